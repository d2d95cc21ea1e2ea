"""GPU parity of the paged decode entry points ("DeepSeek-V3.2" analysis page, sec. 5.1: cache pages
and per-row seq_lens) against the fp64 oracle on each sequence's contiguous cache: shuffled page
tables, context lengths that end inside a page and inside a 128-key tile, one shorter than k, and
pages shared by no one; plus equality with the contiguous entry points when every row is full."""
import math

import numpy as np
import pytest
import torch

import dsa_inputs
from oracle import oracle as ref
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import sparse_attention_tcgen05_b200 as m
    m.load()
    return m


def _paged(rng, B, max_len, P, extra_pages=3):
    """A random page table over a shuffled pool: sequence b's logical page j -> physical page."""
    max_pages = -(-max_len // P)
    num_pages = B * max_pages + extra_pages
    perm = rng.permutation(num_pages)[: B * max_pages].reshape(B, max_pages).astype(np.int32)
    return perm, num_pages


def _scatter(cache, table, P, num_pages):
    """[B, max_len, D] contiguous caches -> a [num_pages, P, D] pool laid out by the table."""
    B, L, D = cache.shape
    pool = np.zeros((num_pages, P, D), dtype=cache.dtype)
    for b in range(B):
        for s0 in range(0, L, P):
            n = min(P, L - s0)
            pool[table[b, s0 // P], :n] = cache[b, s0: s0 + n]
    return pool


@pytest.mark.parametrize("B,max_len,P,k", [(6, 5000, 64, 2048), (5, 3000, 256, 512), (4, 20000, 64, 2048)])
def test_paged_decode_matches_the_oracle(dsa, B, max_len, P, k):
    rng = np.random.default_rng(max_len + P)
    wl = dsa_inputs.custom(f"paged_{max_len}_{P}", 4242 + max_len, B, 1, max_len, 64, 128, 16, k, 128, 576, 512,
                           1 / math.sqrt(192.0))
    lens = rng.integers(max_len // 3, max_len + 1, size=B).astype(np.int32)
    lens[0] = max_len            # a full row
    lens[1] = k - 7              # shorter than k: every position selected
    lens[2] = 129 * 3 + P // 2   # ends inside a page and inside a key tile
    table, num_pages = _paged(rng, B, max_len, P)
    kI = dsa_inputs.k_index(wl)        # [B, max_len, 128] e4m3 bytes (only s < len matters)
    kv = dsa_inputs.kv_latent(wl)      # [B, max_len, 576] bf16 bits
    qI = dsa_inputs.q_index(wl)
    w = dsa_inputs.w_index(wl)
    q = dsa_inputs.q_attn(wl)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    kI_pages = dev(_scatter(kI, table, P, num_pages)).view(torch.float8_e4m3fn)
    kv_pages = dev(_scatter(kv.view(np.int16), table, P, num_pages)).view(torch.bfloat16)
    qI_t = dev(qI).view(torch.float8_e4m3fn).reshape(B, 1, 64, 128)
    w_t = dev(w).reshape(B, 1, 64)
    q_t = dev(q.view(np.int16)).view(torch.bfloat16).reshape(B, 1, 128, 576)
    tbl, sl = dev(table), dev(lens)
    scores = torch.full((B, 1, max_len), float("nan"), device="cuda")
    idx = torch.full((B, 1, k), -7, dtype=torch.int32, device="cuda")
    ws_ix = torch.zeros(dsa.dsa_workspace_bytes(dsa.DSA_OP_INDEXER_TOPK, B, 1, max_len, k, 0), dtype=torch.uint8,
                        device="cuda")
    ws = torch.empty(max(16, dsa.dsa_workspace_bytes(dsa.DSA_OP_SPARSE_MLA_FWD, B, 1, max_len, k, 128)),
                     dtype=torch.uint8, device="cuda")
    dsa.dsa_indexer_topk_paged(qI_t, kI_pages, w_t, tbl, sl, scores, idx, ws_ix)
    out = torch.empty(B, 1, 128, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, 1, 128, device="cuda")
    dsa.dsa_sparse_mla_fwd_paged(q_t, kv_pages, idx, tbl, sl, max_len, wl.scale, out, lse, ws)
    assert dsa.dsa_last_device_status() == 0
    g_sc, g_ix = scores.cpu().numpy(), idx.cpu().numpy()
    g_out, g_lse = out.float().cpu().numpy(), lse.cpu().numpy()
    for b in range(B):
        n = int(lens[b])
        t = n - 1
        e_sc = ref.indexer_row(qI[b], kI[b, :n], w[b], t)
        np.testing.assert_array_equal(g_sc[b, 0, :n], e_sc.astype(np.float32), err_msg=f"scores row {b}")
        assert np.all(np.isneginf(g_sc[b, 0, n:])), f"scores past the row, row {b}"
        e_ix, _ = ref.topk_row(e_sc, t, k)
        np.testing.assert_array_equal(g_ix[b, 0], e_ix, err_msg=f"idx row {b}")
        e_out, e_lse, _ = ref.sparse_mla_row(q[b], kv[b, :n], e_ix, 512, wl.scale)
        parity.check_attention_row(g_out[b, 0], e_out, f"out row {b}")
        assert np.abs(g_lse[b, 0] - e_lse).max() <= parity.LSE_ATOL, f"lse row {b}"


def test_paged_full_rows_equal_the_contiguous_path(dsa):
    # every row full and the identity page table: bit-identical to the contiguous entry points
    B, L, P, k = 32, 8192, 128, 2048
    wl = dsa_inputs.custom("paged_identity", 777, B, 1, L, 64, 128, 16, k, 128, 576, 512, 1 / math.sqrt(192.0))
    dw = parity.DeviceWorkload(wl)
    table = torch.arange(B * (L // P), dtype=torch.int32, device="cuda").reshape(B, L // P)
    lens = torch.full((B,), L, dtype=torch.int32, device="cuda")
    s1, s2 = (torch.empty(B, 1, L, device="cuda") for _ in range(2))
    i1, i2 = (torch.empty(B, 1, k, dtype=torch.int32, device="cuda") for _ in range(2))
    ws_ix = torch.zeros(dsa.dsa_workspace_bytes(dsa.DSA_OP_INDEXER_TOPK, B, 1, L, k, 0), dtype=torch.uint8,
                        device="cuda")
    ws = torch.empty(max(16, dsa.dsa_workspace_bytes(dsa.DSA_OP_SPARSE_MLA_FWD, B, 1, L, k, 128)),
                     dtype=torch.uint8, device="cuda")
    dsa.dsa_indexer_topk_paged(dw.qI, dw.kI.reshape(B * L // P, P, 128), dw.w, table, lens, s1, i1, ws_ix)
    dsa.dsa_indexer_topk(dw.qI, dw.kI, dw.w, s2, i2, ws_ix)
    o1, o2 = (torch.empty(B, 1, 128, 512, dtype=torch.bfloat16, device="cuda") for _ in range(2))
    dsa.dsa_sparse_mla_fwd_paged(dw.q, dw.kv.reshape(B * L // P, P, 576), i1, table, lens, L, wl.scale, o1, None, ws)
    dsa.dsa_sparse_mla_fwd(dw.q, dw.kv, i2, wl.scale, o2, None, None, ws)
    assert dsa.dsa_last_device_status() == 0
    assert torch.equal(s1, s2) and torch.equal(i1, i2) and torch.equal(o1, o2)
