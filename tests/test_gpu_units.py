"""GPU parity of each entry point against the fp64 oracle on small inputs that still span
several tiles and a ragged tail, plus edge cases (ties, -inf, empty slots, split rows)."""
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


# ----------------------------------------------------------------------------------- indexer
@pytest.mark.parametrize("H_I,d_I,B,Lq,Lk", [
    (4, 32, 1, 256, 256),      # tiny prefill dims
    (4, 32, 2, 77, 333),       # ragged: Lq < Lk, neither a multiple of 128
    (8, 64, 2, 200, 300),
    (16, 128, 1, 130, 257),
    (32, 128, 3, 1, 1000),     # decode kernel variant
    (32, 128, 2, 40, 700),
    (64, 128, 2, 9, 520),      # prefill variant, few queries
    (64, 128, 5, 1, 3000),     # decode variant
])
def test_indexer_bit_exact(dsa, H_I, d_I, B, Lq, Lk):
    wl = dsa_inputs.custom(f"ix_{H_I}_{d_I}", 1234 + H_I + Lk, B, Lq, Lk, H_I, d_I, 16, 8, 1, 16, 16)
    dw = parity.DeviceWorkload(wl, with_attention=False)
    scores = torch.full((B, Lq, Lk), float("nan"), dtype=torch.float32, device="cuda")
    dsa.dsa_indexer(dw.qI, dw.kI, dw.w, scores)
    got = scores.cpu().numpy()
    assert dsa.dsa_last_device_status() == 0
    qI = dw.qI_np.reshape(B * Lq, H_I, d_I)
    w = dw.w_np.reshape(B * Lq, H_I)
    for r in range(B * Lq):
        b, i = divmod(r, Lq)
        exp = ref.indexer_row(qI[r], dw.kI_np[b], w[r], wl.t_of(i)).astype(np.float32)
        np.testing.assert_array_equal(got[b, i], exp, err_msg=f"row {r}")


def test_indexer_large_batch_decode_walks_whole_rows(dsa):
    # with at least two rows per SM a work item is a whole sequence (33 key tiles here), so the
    # producer refills its 16-tile window of box rows mid-item; contiguous rows against the oracle
    # (sampled), and a shuffled paged copy of the same cache against the contiguous call
    B, Lk, H_I, d_I, k, P = 300, 4224, 64, 128, 256, 64
    wl = dsa_inputs.custom("ix_wide_batch", 4242, B, 1, Lk, H_I, d_I, 16, k, 1, 16, 16)
    dw = parity.DeviceWorkload(wl, with_attention=False)
    scores = torch.full((B, 1, Lk), float("nan"), dtype=torch.float32, device="cuda")
    dsa.dsa_indexer(dw.qI, dw.kI, dw.w, scores)
    got = scores.cpu().numpy()
    assert dsa.dsa_last_device_status() == 0
    qI = dw.qI_np.reshape(B, H_I, d_I)
    w = dw.w_np.reshape(B, H_I)
    for b in (0, 1, 77, 148, 149, 150, 222, 296, 297, 299):
        exp = ref.indexer_row(qI[b], dw.kI_np[b], w[b], Lk - 1).astype(np.float32)
        np.testing.assert_array_equal(got[b, 0], exp, err_msg=f"row {b}")
    # the same cache as pages of 64 keys in a shuffled pool, every row full
    pages = Lk // P
    g = torch.Generator().manual_seed(99)
    table = torch.randperm(B * pages, generator=g).to(torch.int32).reshape(B, pages).cuda()
    pool = torch.empty(B * pages, P, d_I, dtype=dw.kI.dtype, device="cuda")
    pool.view(torch.uint8)[table.flatten().long()] = dw.kI.reshape(B * pages, P, d_I).view(torch.uint8)
    lens = torch.full((B,), Lk, dtype=torch.int32, device="cuda")
    s1, s2 = (torch.empty(B, 1, Lk, device="cuda") for _ in range(2))
    i1, i2 = (torch.empty(B, 1, k, dtype=torch.int32, device="cuda") for _ in range(2))
    ws_ix = torch.zeros(dsa.dsa_workspace_bytes(dsa.DSA_OP_INDEXER_TOPK, B, 1, Lk, k, 0), dtype=torch.uint8,
                        device="cuda")
    dsa.dsa_indexer_topk_paged(dw.qI, pool, dw.w, table, lens, s1, i1, ws_ix)
    dsa.dsa_indexer_topk(dw.qI, dw.kI, dw.w, s2, i2, ws_ix)
    assert dsa.dsa_last_device_status() == 0
    assert torch.equal(s1, scores) and torch.equal(s2, scores) and torch.equal(i1, i2)


def test_indexer_rejects_bad_arguments(dsa):
    q = torch.zeros(1, 4, 64, 128, dtype=torch.float8_e4m3fn, device="cuda")
    k = torch.zeros(1, 8, 128, dtype=torch.float8_e4m3fn, device="cuda")
    w = torch.zeros(1, 4, 64, device="cuda")
    s = torch.zeros(1, 4, 8, device="cuda")
    lib = dsa.load()
    import ctypes
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    assert lib.dsa_indexer(None, P(k), P(w), P(s), 1, 4, 8, 64, 128, None, 0, None) == 1
    assert lib.dsa_indexer(P(q), P(k), P(w), P(s), 1, 9, 8, 64, 128, None, 0, None) == 1  # Lq > Lk
    assert lib.dsa_indexer(P(q), P(k), P(w), P(s), 1, 4, 8, 48, 128, None, 0, None) == 2  # H_I
    assert lib.dsa_indexer(P(q), P(k), P(w), ctypes.c_void_p(s.data_ptr() + 4), 1, 4, 8, 64, 128,
                           None, 0, None) == 1  # misaligned
    assert dsa.dsa_last_device_status() == 0


# ----------------------------------------------------------------------------------- top-k
def _topk_case(dsa, scores_np, Lq, k):
    B, _, Lk = scores_np.shape
    s = torch.from_numpy(scores_np).cuda()
    idx = torch.full((B, Lq, k), -7, dtype=torch.int32, device="cuda")
    dsa.dsa_topk(s, idx)
    got = idx.cpu().numpy()
    assert dsa.dsa_last_device_status() == 0
    for b in range(B):
        for i in range(Lq):
            t = i + Lk - Lq
            exp, n = ref.topk_row(scores_np[b, i].astype(np.float64), t, k)
            np.testing.assert_array_equal(got[b, i], exp, err_msg=f"row ({b},{i})")


@pytest.mark.parametrize("B,Lq,Lk,k,levels", [
    (1, 300, 300, 32, 5),        # many ties, short rows (n <= k fast path included)
    (2, 64, 5000, 100, 3),       # extreme ties
    (100, 1, 16384, 2048, 50),   # few rows: 2-CTA clusters
    (64, 1, 16384, 2048, 7),     # 4-CTA clusters
    (8, 1, 40000, 1000, 1000),   # 8-CTA clusters, slice > one block of threads
    (1, 4, 70000, 4096, 9),      # longest k, 4-CTA by length
    (3, 2, 9999, 512, 20),       # rows not 16-byte aligned: scalar copy into the load stage
])
def test_topk_exact_with_ties(dsa, B, Lq, Lk, k, levels):
    rng = np.random.default_rng(B * 7 + Lk)
    sc = (rng.integers(0, levels, size=(B, Lq, Lk)) / 16.0).astype(np.float32)
    sc[..., ::97] = -sc[..., ::97]
    for i in range(Lq):  # invisible positions hold -inf, as the indexer writes them
        sc[:, i, i + Lk - Lq + 1:] = -np.inf
    _topk_case(dsa, sc, Lq, k)


def test_topk_all_equal_and_signed_zero(dsa):
    sc = np.zeros((2, 1, 5000), np.float32)
    sc[1, 0, ::3] = -0.0
    _topk_case(dsa, sc, 1, 777)


def test_topk_distinct_normal_scores(dsa):
    rng = np.random.default_rng(3)
    sc = rng.normal(size=(3, 1, 131072)).astype(np.float32)
    _topk_case(dsa, sc, 1, 2048)


# ----------------------------------------------------------------------------------- sparse MLA
def _mla_case(dsa, wl, idx_np, emit_p=False, check_p=False):
    dw = parity.DeviceWorkload(wl)
    B, Lq, H = wl.B, wl.Lq, wl.H
    idx = torch.from_numpy(idx_np).cuda()
    out = torch.empty(B, Lq, H, wl.d_v, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, Lq, H, dtype=torch.float32, device="cuda")
    p_sel = torch.full((B, Lq, wl.k), -1.0, dtype=torch.float32, device="cuda") if emit_p else None
    nws = dsa.dsa_workspace_bytes(dsa.DSA_OP_SPARSE_MLA_FWD, B, Lq, wl.Lk, wl.k, H)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device="cuda")
    dsa.dsa_sparse_mla_fwd(dw.q, dw.kv, idx, wl.scale, out, lse, p_sel, ws)
    o = out.float().cpu().numpy()
    l = lse.cpu().numpy()
    ps = p_sel.cpu().numpy() if emit_p else None
    assert dsa.dsa_last_device_status() == 0
    kv = dw.kv_np()
    for r in range(B * Lq):
        b, i = divmod(r, Lq)
        q_row = dsa_inputs.q_attn(wl, r, 1)[0]
        eo, el, P = ref.sparse_mla_row(q_row, kv[b], idx_np[b, i], wl.d_v, wl.scale, want_P=emit_p)
        parity.check_attention_row(o[b, i], eo, f"row {r}")
        # an empty set has lse = -inf on both sides
        fin = ~np.isneginf(el)
        d = np.zeros_like(el)
        d[fin] = np.abs(l[b, i][fin] - el[fin])
        d[~fin & ~np.isneginf(l[b, i])] = np.inf
        assert d.max() <= parity.LSE_ATOL, f"lse row {r}"
        if emit_p:
            parity.check_p_row(ps[b, i], ref.p_sel_row(P, idx_np[b, i]), f"p row {r}")


def test_mla_tiny_dims_random_sets_with_holes(dsa):
    wl = dsa_inputs.custom("mla_tiny", 77, 2, 5, 300, 4, 32, 8, 100, 8, 80, 64)
    rng = np.random.default_rng(5)
    idx = np.stack([np.stack([rng.permutation(300)[:100] for _ in range(5)]) for _ in range(2)])
    idx = idx.astype(np.int32)
    idx[0, 1, 10:30] = -1      # a hole inside the row
    idx[1, 2, 37:] = -1        # padded tail
    idx[1, 3, :99] = -1        # a single valid slot (the last one)
    _mla_case(dsa, wl, idx, emit_p=True)


def test_mla_full_dims_decode_split_and_p(dsa):
    wl = dsa_inputs.custom("mla_full", 91, 3, 1, 5000, 64, 128, 16, 2048, 128, 576, 512,
                           1 / math.sqrt(192))
    rng = np.random.default_rng(9)
    idx = np.stack([rng.permutation(5000)[:2048] for _ in range(3)]).astype(np.int32).reshape(3, 1, 2048)
    idx[2, 0, 1500:] = -1
    _mla_case(dsa, wl, idx)                 # split over several CTAs per row, then combined
    _mla_case(dsa, wl, idx, emit_p=True)    # p emission keeps one CTA per value half


def test_mla_decode_two_splits_combined_in_kernel(dsa):
    # 32 decode rows -> two KV splits per row whose partial results are combined inside the
    # attention kernel (the two pairs of a row form one cluster).  H = 100 leaves the last
    # warp of heads partly empty; some rows have an empty first or second split.
    wl = dsa_inputs.custom("mla_fuse2", 17, 32, 1, 3000, 64, 128, 16, 2048, 100, 576, 512,
                           1 / math.sqrt(192))
    rng = np.random.default_rng(21)
    idx = np.stack([rng.permutation(3000)[:2048] for _ in range(32)]).astype(np.int32)
    idx = idx.reshape(32, 1, 2048)
    idx[0, 0, 600:] = -1        # second split empty
    idx[1, 0, :1500] = -1       # first split empty
    idx[2, 0, 1024:] = -1       # exactly the first split
    idx[3, 0, 40:2000] = -1     # a few entries at both ends
    idx[4, 0, :2047] = -1       # a single valid slot, in the second split
    _mla_case(dsa, wl, idx)


def test_mla_staged_epilogue_fewer_heads(dsa):
    # enough rows for one CTA pair per row (no KV split) and no p emission: the output rows go
    # through the shared-memory tile and are written by whole rows; H = 40 leaves most of the
    # tile's rows unused, and some rows have an empty or a one-entry set
    wl = dsa_inputs.custom("mla_staged_h40", 29, 2, 40, 600, 64, 128, 16, 256, 40, 576, 512,
                           1 / math.sqrt(192))
    rng = np.random.default_rng(31)
    idx = np.stack([np.stack([rng.permutation(600)[:256] for _ in range(40)]) for _ in range(2)])
    idx = idx.astype(np.int32)
    idx[0, 5, :] = -1          # no valid entry
    idx[1, 7, 1:] = -1         # a single entry
    idx[1, 9, 100:] = -1       # a ragged tail
    _mla_case(dsa, wl, idx)


def test_mla_fewer_heads_and_short_sets(dsa):
    wl = dsa_inputs.custom("mla_h20", 13, 1, 6, 700, 64, 128, 16, 40, 20, 576, 512, 0.05)
    rng = np.random.default_rng(2)
    idx = np.full((1, 6, 40), -1, np.int32)
    for i in range(6):
        n = [1, 2, 31, 32, 33, 40][i]
        idx[0, i, :n] = np.sort(rng.permutation(700)[:n])
    _mla_case(dsa, wl, idx, emit_p=True)


# ----------------------------------------------------------------------------------- KL
def test_kl_matches_oracle_rows_and_sum(dsa):
    rng = np.random.default_rng(8)
    B, Lq, Lk, k = 2, 50, 400, 64
    scores = (rng.normal(size=(B, Lq, Lk)) * 3).astype(np.float32)
    idx = np.stack([[np.sort(rng.permutation(Lk)[:k]) for _ in range(Lq)] for _ in range(B)]).astype(np.int32)
    idx[0, 3, 50:] = -1
    p = rng.dirichlet(np.ones(k), size=(B, Lq)).astype(np.float32)
    p[0, 3, 50:] = 0
    p[1, 7, 5] = 0.0
    st, it, pt = (torch.from_numpy(a).cuda() for a in (scores, idx, p))
    loss = torch.empty(1, device="cuda")
    per = torch.empty(B, Lq, device="cuda")
    dsa.dsa_indexer_kl(st, it, pt, loss, per)
    # the workspace path (no per-row output) gives the same loss
    loss2 = torch.empty(1, device="cuda")
    ws = torch.empty(dsa.dsa_workspace_bytes(dsa.DSA_OP_INDEXER_KL, B, Lq, Lk, k, 0), dtype=torch.uint8,
                     device="cuda")
    dsa.dsa_indexer_kl(st, it, pt, loss2, None, ws)
    assert dsa.dsa_last_device_status() == 0
    per = per.cpu().numpy()
    total = 0.0
    for b in range(B):
        for i in range(Lq):
            e = ref.kl_row(scores[b, i].astype(np.float64), idx[b, i], p[b, i].astype(np.float64))
            assert abs(per[b, i] - e) <= 1e-4 * abs(e) + 1e-5, (b, i)
            total += e
    assert abs(loss.item() - total) <= parity.KL_RTOL * abs(total)
    assert loss.item() == loss2.item()


# ----------------------------------------------------------------------------------- fused indexer -> top-k
@pytest.mark.parametrize("H_I,B,Lk,k,w_den", [
    (64, 5, 3000, 512, 16),      # 1-CTA rows, ragged tail tile
    (64, 40, 20000, 2048, 16),   # 2-CTA clusters
    (32, 7, 70000, 2048, 1),     # w in {-1, 0, 1}: heavy ties, 4-CTA clusters
    (64, 3, 131072, 4096, 2),    # the longest rows and the largest k
])
def test_fused_indexer_topk_matches_the_two_calls_and_the_oracle(dsa, H_I, B, Lk, k, w_den):
    wl = dsa_inputs.custom(f"fused_{H_I}_{Lk}", 2468 + Lk, B, 1, Lk, H_I, 128, w_den, k, 1, 16, 16)
    dw = parity.DeviceWorkload(wl, with_attention=False)
    s1 = torch.full((B, 1, Lk), float("nan"), device="cuda")
    s2 = torch.full((B, 1, Lk), float("nan"), device="cuda")
    i1 = torch.full((B, 1, k), -7, dtype=torch.int32, device="cuda")
    i2 = torch.full((B, 1, k), -7, dtype=torch.int32, device="cuda")
    ws = torch.zeros(dsa.dsa_workspace_bytes(dsa.DSA_OP_INDEXER_TOPK, B, 1, Lk, k, 0), dtype=torch.uint8,
                     device="cuda")  # zero-filled once
    for _ in range(3):  # the call leaves the histograms cleared for the next one
        dsa.dsa_indexer_topk(dw.qI, dw.kI, dw.w, s1, i1, ws)
    torch.cuda.synchronize()
    assert int(ws.count_nonzero()) == 0
    dsa.dsa_indexer(dw.qI, dw.kI, dw.w, s2)
    dsa.dsa_topk(s2, i2)
    assert dsa.dsa_last_device_status() == 0
    assert torch.equal(s1, s2) and torch.equal(i1, i2)
    got = i1.cpu().numpy()
    sc = s1.cpu().numpy()
    for b in range(B):
        exp, n = ref.topk_row(sc[b, 0].astype(np.float64), Lk - 1, k)
        np.testing.assert_array_equal(got[b, 0], exp, err_msg=f"row {b}")
    # the scores themselves are checked bit for bit on two rows
    qI = dw.qI_np.reshape(B, H_I, 128)
    w = dw.w_np.reshape(B, H_I)
    for b in (0, B - 1):
        exp = ref.indexer_row(qI[b], dw.kI_np[b], w[b], Lk - 1).astype(np.float32)
        np.testing.assert_array_equal(sc[b, 0], exp)
