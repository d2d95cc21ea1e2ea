"""The indexer loss entry point that allocates nothing, checked against the workspace one.

Callers that cannot allocate device memory at call time (a runtime that reserved all of HBM
up front, a plugin that only receives its input and output pointers, a thread that must not
risk the synchronisation cudaMalloc/cudaFree can cause) use dsa_indexer_kl_noalloc, whose
per-row scratch is a fixed array inside the library.  Both entry points run the same kernels
and the same fixed-order sum, so the results must be bit-identical.  This file is named so
pytest runs it after every other test: it must pass both on its own in a fresh process and
after them.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import oracle as ref

pytestmark = pytest.mark.gpu


def _case(seed, B, Lq, Lk, k):
    rng = np.random.default_rng(seed)
    scores = (rng.normal(size=(B, Lq, Lk)) * 3).astype(np.float32)
    idx = np.stack([[np.sort(rng.permutation(Lk)[:k]) for _ in range(Lq)] for _ in range(B)])
    idx = idx.astype(np.int32)
    idx[0, 1, k // 2:] = -1
    p = rng.dirichlet(np.ones(k), size=(B, Lq)).astype(np.float32)
    p[0, 1, k // 2:] = 0
    return scores, idx, p


@pytest.fixture(scope="module")
def dsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import sparse_attention_tcgen05_b200 as m
    m.load()
    return m


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def test_noalloc_kl_matches_workspace_entry_point_twice_in_a_row(dsa):
    lib = dsa.load()
    # two calls in a row with different sizes: the second must not see the first's rows
    for seed, (B, Lq, Lk, k) in ((1, (2, 300, 512, 64)), (2, (1, 97, 260, 33))):
        st, it, pt = (torch.from_numpy(a).cuda() for a in _case(seed, B, Lq, Lk, k))
        ref_loss = torch.empty(1, device="cuda")
        ws = torch.empty(dsa.dsa_workspace_bytes(dsa.DSA_OP_INDEXER_KL, B, Lq, Lk, k, 0),
                         dtype=torch.uint8, device="cuda")
        dsa.dsa_indexer_kl(st, it, pt, ref_loss, None, ws)
        loss = torch.full((1,), float("nan"), device="cuda")
        rc = lib.dsa_indexer_kl_noalloc(_ptr(st), _ptr(it), _ptr(pt), B, Lq, Lk, k, _ptr(loss), None,
                                        _stream())
        assert rc == 0, dsa.dsa_status_str(rc)
        assert dsa.dsa_last_device_status() == 0
        assert loss.item() == ref_loss.item()  # bit-identical
    # sizes beyond the fixed array are refused before anything is launched
    big = 1 << 20
    rc = lib.dsa_indexer_kl_noalloc(_ptr(st), _ptr(it), _ptr(pt), 1, big + 1, big + 1, k, _ptr(loss), None,
                                    _stream())
    assert rc == 2  # DSA_ERR_UNSUPPORTED


def test_noalloc_kl_per_row_output_matches_the_oracle(dsa):
    lib = dsa.load()
    B, Lq, Lk, k = 2, 40, 300, 48
    scores, idx, p = _case(5, B, Lq, Lk, k)
    st, it, pt = (torch.from_numpy(a).cuda() for a in (scores, idx, p))
    per = torch.full((B, Lq), float("nan"), device="cuda")
    loss = torch.empty(1, device="cuda")
    rc = lib.dsa_indexer_kl_noalloc(_ptr(st), _ptr(it), _ptr(pt), B, Lq, Lk, k, _ptr(loss), _ptr(per),
                                    _stream())
    assert rc == 0 and dsa.dsa_last_device_status() == 0
    per_ws = torch.empty(B, Lq, device="cuda")
    loss_ws = torch.empty(1, device="cuda")
    dsa.dsa_indexer_kl(st, it, pt, loss_ws, per_ws)
    assert torch.equal(per, per_ws) and loss.item() == loss_ws.item()
    got = per.cpu().numpy()
    for b in range(B):
        for i in range(Lq):
            e = ref.kl_row(scores[b, i].astype(np.float64), idx[b, i], p[b, i].astype(np.float64))
            assert abs(got[b, i] - e) <= 1e-4 * abs(e) + 1e-5, (b, i, got[b, i], e)


def test_noalloc_kl_takes_no_device_memory(dsa):
    lib = dsa.load()
    B, Lq, Lk, k = 1, 500, 700, 64
    st, it, pt = (torch.from_numpy(a).cuda() for a in _case(9, B, Lq, Lk, k))
    loss = torch.empty(1, device="cuda")
    args = (_ptr(st), _ptr(it), _ptr(pt), B, Lq, Lk, k, _ptr(loss), None, _stream())
    assert lib.dsa_indexer_kl_noalloc(*args) == 0  # first call: the array's address is looked up
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    reserved0 = torch.cuda.memory_reserved()
    assert lib.dsa_indexer_kl_noalloc(*args) == 0
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0 and torch.cuda.memory_reserved() == reserved0
    assert dsa.dsa_last_device_status() == 0
