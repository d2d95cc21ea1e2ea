"""The indexer loss entry point that allocates nothing, checked against the workspace one.

Callers that cannot allocate device memory at call time (a runtime that reserved all of HBM
up front, a plugin that only receives its input and output pointers, a thread that must not
risk the synchronisation cudaMalloc/cudaFree can cause) use dsa_indexer_kl_noalloc, whose
per-row scratch is a fixed array inside the library.  This file is named so pytest runs it
after every other test: it must pass both on its own in a fresh process and after them.
"""
import ctypes

import numpy as np
import pytest
import torch

from tests import parity

pytestmark = pytest.mark.gpu


def _case(seed, B, Lq, Lk, k):
    rng = np.random.default_rng(seed)
    scores = (rng.normal(size=(B, Lq, Lk)) * 3).astype(np.float32)
    idx = np.stack([[np.sort(rng.permutation(Lk)[:k]) for _ in range(Lq)] for _ in range(B)])
    idx = idx.astype(np.int32)
    idx[0, 1, k // 2:] = -1
    p = rng.dirichlet(np.ones(k), size=(B, Lq)).astype(np.float32)
    p[0, 1, k // 2:] = 0
    return (torch.from_numpy(a).cuda() for a in (scores, idx, p))


def test_noalloc_kl_matches_workspace_entry_point_twice_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import sparse_attention_tcgen05_b200 as dsa

    lib = dsa.load()
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # two calls in a row with different sizes: the second must not see the first's rows
    for seed, (B, Lq, Lk, k) in ((1, (2, 300, 512, 64)), (2, (1, 97, 260, 33))):
        scores, idx, p = _case(seed, B, Lq, Lk, k)
        ref_loss = torch.empty(1, device="cuda")
        ws = torch.empty(dsa.dsa_workspace_bytes(dsa.DSA_OP_INDEXER_KL, B, Lq, Lk, k, 0),
                         dtype=torch.uint8, device="cuda")
        dsa.dsa_indexer_kl(scores, idx, p, ref_loss, None, ws)
        loss = torch.full((1,), float("nan"), device="cuda")
        rc = lib.dsa_indexer_kl_noalloc(P(scores), P(idx), P(p), B, Lq, Lk, k, P(loss), None, stream)
        assert rc == 0, dsa.dsa_status_str(rc)
        assert dsa.dsa_last_device_status() == 0
        a, b = loss.item(), ref_loss.item()
        assert abs(a - b) <= parity.KL_RTOL * abs(b), (a, b)
    # sizes beyond the fixed array are refused before anything is launched
    big = 1 << 20
    rc = lib.dsa_indexer_kl_noalloc(P(scores), P(idx), P(p), 1, big + 1, big + 1, k, P(loss), None,
                                    stream)
    assert rc == 2  # DSA_ERR_UNSUPPORTED
