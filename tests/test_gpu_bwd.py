"""GPU parity of the indexer-loss gradient (dsa_indexer_bwd) against the fp64 oracle's gradient
(pinned by finite differences and autograd on the CPU), on small ragged shapes with holes, the
dense warm-up form, and decode rows; and, at the sparse-stage workload's full size, sampled rows
of dq and dw plus an identity that holds at any size.

Tolerance: max|err| <= 1e-3 * max|ref| + 1e-5 per row (dq, dw) and over the whole tensor (dk).
The kernel's softmax and sums run in fp32 (about 1e-6 relative per term, sums of up to a few
thousand terms) and G is carried in two fp16 parts (2^-22 relative), so 1e-3 leaves a wide margin
while any wrong index, sign or missing factor fails it by orders of magnitude."""
import numpy as np
import pytest
import torch

import dsa_inputs
from oracle import oracle as ref
from tests import parity

pytestmark = pytest.mark.gpu
RTOL, ATOL = 1e-3, 1e-5


@pytest.fixture(scope="module")
def dsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import sparse_attention_tcgen05_b200 as m
    m.load()
    return m


def _e4m3_f64(b):
    return torch.from_numpy(np.ascontiguousarray(b)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _close(got, exp, what):
    err = np.abs(got.astype(np.float64) - exp).max()
    bound = RTOL * np.abs(exp).max() + ATOL
    assert err <= bound, f"{what}: max|err| {err:.3e} > {bound:.3e}"


def _run(dsa, wl, dw_, idx_np, p_np):
    B, Lq, Lk = wl.B, wl.Lq, wl.Lk
    scores = torch.empty(B, Lq, Lk, device="cuda")
    dsa.dsa_indexer(dw_.qI, dw_.kI, dw_.w, scores)
    idx = None if idx_np is None else torch.from_numpy(idx_np).cuda()
    p = torch.from_numpy(p_np.astype(np.float32)).cuda()
    dq = torch.full((B, Lq, 64, 128), float("nan"), device="cuda")
    dwt = torch.full((B, Lq, 64), float("nan"), device="cuda")
    dk = torch.full((B, Lk, 128), float("nan"), device="cuda")
    dsa.dsa_indexer_bwd(dw_.qI, dw_.kI, dw_.w, scores, idx, p, dq, dwt, dk)
    assert dsa.dsa_last_device_status() == 0
    return scores, dq.cpu().numpy(), dwt.cpu().numpy(), dk.cpu().numpy()


def _oracle(wl, dw_, idx_np, p_np, rows=None):
    B, Lq, Lk = wl.B, wl.Lq, wl.Lk
    q = _e4m3_f64(dw_.qI_np).reshape(B * Lq, 64, 128)
    kk = _e4m3_f64(dw_.kI_np).reshape(B, Lk, 128)
    w = dw_.w_np.reshape(B * Lq, 64).astype(np.float64)
    dk = np.zeros((B, Lk, 128))
    dq, dw = {}, {}
    for r in (range(B * Lq) if rows is None else rows):
        b, i = divmod(r, Lq)
        t = wl.t_of(i)
        if idx_np is None:  # dense: every s <= t
            ix = np.arange(t + 1, dtype=np.int32)
            pr = p_np[b, i, : t + 1].astype(np.float64)
        else:
            ix = idx_np[b, i]
            pr = p_np[b, i].astype(np.float64)
        dq[r], dw[r], _, _ = ref.indexer_grad_row(q[r], kk[b], w[r], ix, pr, dk=dk[b])
    return dq, dw, dk


def _case_sparse(seed, B, Lq, Lk, k, holes=True):
    rng = np.random.default_rng(seed)
    idx = np.full((B, Lq, k), -1, np.int32)
    p = np.zeros((B, Lq, k))
    for b in range(B):
        for i in range(Lq):
            t = i + Lk - Lq
            n = min(k, t + 1)
            idx[b, i, :n] = np.sort(rng.permutation(t + 1)[:n])
            if holes and n > 4 and (b + i) % 3 == 0:
                idx[b, i, n // 2: n // 2 + 2] = -1  # empty slots inside the row
            valid = idx[b, i] >= 0
            pp = rng.dirichlet(np.ones(valid.sum()))
            pp[pp < 0.2 / valid.sum()] = 0.0  # some zero targets
            p[b, i, valid] = pp / pp.sum()
    return idx, p


@pytest.mark.parametrize("B,Lq,Lk,k", [
    (2, 40, 700, 256),    # prefill rows with ragged tiles, holes and zero targets
    (3, 1, 3000, 2048),   # decode rows: 16 tiles each
    (1, 200, 200, 64),    # short causal rows (t + 1 < k for the first ones)
])
def test_sparse_gradient_matches_the_oracle(dsa, B, Lq, Lk, k):
    wl = dsa_inputs.custom(f"bwd_{B}_{Lq}_{Lk}", 1357 + Lk, B, Lq, Lk, 64, 128, 16, k, 1, 16, 16)
    dw_ = parity.DeviceWorkload(wl, with_attention=False)
    idx, p = _case_sparse(Lk + k, B, Lq, Lk, k)
    _, dq, dw, dk = _run(dsa, wl, dw_, idx, p)
    e_dq, e_dw, e_dk = _oracle(wl, dw_, idx, p)
    for r in range(B * Lq):
        b, i = divmod(r, Lq)
        _close(dq[b, i], e_dq[r], f"dq row {r}")
        _close(dw[b, i], e_dw[r], f"dw row {r}")
    _close(dk, e_dk, "dk")


def test_dense_gradient_matches_the_oracle(dsa):
    B, Lq, Lk = 2, 30, 400
    wl = dsa_inputs.custom("bwd_dense", 97531, B, Lq, Lk, 64, 128, 16, Lk, 1, 16, 16)
    dw_ = parity.DeviceWorkload(wl, with_attention=False)
    rng = np.random.default_rng(4)
    p = np.zeros((B, Lq, Lk))
    for b in range(B):
        for i in range(Lq):
            t = i + Lk - Lq
            p[b, i, : t + 1] = rng.dirichlet(np.ones(t + 1))
    _, dq, dw, dk = _run(dsa, wl, dw_, None, p)
    e_dq, e_dw, e_dk = _oracle(wl, dw_, None, p)
    for r in range(B * Lq):
        b, i = divmod(r, Lq)
        _close(dq[b, i], e_dq[r], f"dq row {r}")
        _close(dw[b, i], e_dw[r], f"dw row {r}")
    _close(dk, e_dk, "dk")


def test_sparse_stage_16k_gradient_sampled_rows_and_identity(dsa):
    # the sparse-stage workload at full size: the forward path's own idx and p
    wl = dsa_inputs.WORKLOADS["indexer_kl_16k"]
    dw_ = parity.DeviceWorkload(wl)
    res = parity.run_path(dw_)
    B, Lq, Lk = wl.B, wl.Lq, wl.Lk
    dq = torch.empty(B, Lq, 64, 128, device="cuda")
    dwt = torch.empty(B, Lq, 64, device="cuda")
    dk = torch.empty(B, Lk, 128, device="cuda")
    dsa.dsa_indexer_bwd(dw_.qI, dw_.kI, dw_.w, res["scores"], res["idx"], res["p_sel"], dq, dwt, dk)
    assert dsa.dsa_last_device_status() == 0
    # identity (the indexer score is positively homogeneous of degree 1 in q, in w and in k):
    # sum dq.q = sum dw.w = sum dk.k = sum_t sum_i g_ti I_ti
    qf = dw_.qI.to(torch.float64)
    kf = dw_.kI.to(torch.float64)
    s_q = (dq.double() * qf).sum().item()
    s_w = (dwt.double() * dw_.w.double()).sum().item()
    s_k = (dk.double() * kf).sum().item()
    idx = res["idx"].long()
    valid = idx >= 0
    I = torch.gather(res["scores"], 2, idx.clamp(min=0)).double()
    I = torch.where(valid, I, torch.full_like(I, float("-inf")))
    q_sm = torch.softmax(I, dim=-1)
    pt = res["p_sel"].double()
    g = torch.where(valid, q_sm * pt.sum(-1, keepdim=True) - pt, torch.zeros_like(pt))
    s_g = (g * torch.where(valid, I, torch.zeros_like(I))).sum().item()
    scale = (g.abs() * torch.where(valid, I.abs(), torch.zeros_like(I))).sum().item()
    for name, v in (("dq.q", s_q), ("dw.w", s_w), ("dk.k", s_k)):
        assert abs(v - s_g) <= 1e-4 * scale, (name, v, s_g, scale)
    # sampled rows of dq and dw against the oracle (its inputs drawn afresh)
    rows = dsa_inputs.sample_rows(wl, 24)
    idx_np = res["idx"].cpu().numpy()
    p_np = res["p_sel"].cpu().numpy()
    e_dq, e_dw, _ = _oracle(wl, dw_, idx_np, p_np, rows=rows)
    g_dq = dq.cpu().numpy()
    g_dw = dwt.cpu().numpy()
    for r in rows:
        _close(g_dq[0, r], e_dq[r], f"dq row {r}")
        _close(g_dw[0, r], e_dw[r], f"dw row {r}")
