"""GPU parity of the dense warm-up entry points ("DSA Continued Pre-Training" page, Stage 1;
analysis page eq. (3)) against the fp64 oracle: dense causal attention with its head-summed target
p over every s <= t, and the eq. (3) loss, on small ragged shapes (80/64 and 576/512 latents,
prefill rows and split decode rows) and on sampled rows of the 16K-token warm-up step."""
import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import dsa_inputs
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import sparse_attention_tcgen05_b200 as m
    m.load()
    return m


def _check_rows(wl, dw, res, rows):
    kv = dw.kv_np()
    sc = res["scores"].reshape(wl.rows, wl.Lk)
    out = res["out"].reshape(wl.rows, wl.H, wl.d_v)
    lse = res["lse"].reshape(wl.rows, wl.H)
    pf = res["p_full"].reshape(wl.rows, wl.Lk)
    per = res["loss_rows"].reshape(wl.rows)
    rows_t = torch.tensor(rows, device=sc.device)
    g_sc, g_out, g_lse = sc[rows_t].cpu().numpy(), out[rows_t].float().cpu().numpy(), lse[rows_t].cpu().numpy()
    g_p, g_kl = pf[rows_t].cpu().numpy(), per[rows_t].cpu().numpy()
    # the oracle's rows in parallel (its C calls run without the GIL)
    with ThreadPoolExecutor(max_workers=os.cpu_count() or 1) as ex:
        refs = list(ex.map(lambda r: parity.oracle_dense_row(dw, r, kv), rows))
    for j, r in enumerate(rows):
        e = refs[j]
        t = e["t"]
        np.testing.assert_array_equal(g_sc[j], e["scores"].astype(np.float32), err_msg=f"scores row {r}")
        parity.check_attention_row(g_out[j], e["out"], f"dense out row {r}")
        assert np.abs(g_lse[j] - e["lse"]).max() <= parity.LSE_ATOL, f"lse row {r}"
        parity.check_p_row(g_p[j, : t + 1], e["p"], f"dense p row {r}")
        assert np.all(g_p[j, t + 1:] == 0.0), f"p beyond t, row {r}"
        assert abs(g_kl[j] - e["kl"]) <= parity.KL_RTOL * abs(e["kl"]) + 1e-6, f"KL row {r}: {g_kl[j]} vs {e['kl']}"
    total = res["loss_rows"].double().sum().item()
    assert abs(res["loss"].item() - total) <= 1e-6 * abs(total)


@pytest.mark.parametrize("B,Lq,Lk,H,d_qk,d_v", [
    (2, 150, 150, 8, 80, 64),      # tiny latent, causal prefill, ragged tail
    (1, 40, 700, 128, 576, 512),   # full latent, the last 40 positions of a 700-token context
    (3, 1, 3000, 128, 576, 512),   # full latent, decode rows split over several CTA pairs
    (2, 2, 1500, 100, 576, 512),   # fewer heads
])
def test_dense_warmup_step_matches_the_oracle(dsa, B, Lq, Lk, H, d_qk, d_v):
    H_I, d_I = (4, 32) if d_qk == 80 else (64, 128)
    wl = dsa_inputs.custom(f"dense_{B}_{Lq}_{Lk}", 0xD5A0 + 31 + Lk, B, Lq, Lk, H_I, d_I, 16, Lk, H, d_qk, d_v,
                           1 / math.sqrt(192.0) if d_qk == 576 else None, dense=True)
    dw = parity.DeviceWorkload(wl)
    res = parity.run_path(dw)
    torch.cuda.synchronize()
    _check_rows(wl, dw, res, list(range(wl.rows)))


def test_dense_attention_equals_sparse_attention_over_the_whole_prefix(dsa):
    # the selection kernel given every s <= t must give the dense kernel's results
    wl = dsa_inputs.custom("dense_vs_sparse", 0xD5A0 + 33, 1, 64, 500, 64, 128, 16, 500, 128, 576, 512,
                           1 / math.sqrt(192.0))
    dw = parity.DeviceWorkload(wl)
    idx = torch.full((1, 64, 500), -1, dtype=torch.int32)
    for i in range(64):
        t = wl.t_of(i)
        idx[0, i, : t + 1] = torch.arange(t + 1, dtype=torch.int32)
    idx = idx.cuda()
    o_s = torch.empty(1, 64, 128, 512, dtype=torch.bfloat16, device="cuda")
    o_d = torch.empty_like(o_s)
    p_s = torch.empty(1, 64, 500, device="cuda")
    p_d = torch.empty_like(p_s)
    lse_s = torch.empty(1, 64, 128, device="cuda")
    lse_d = torch.empty_like(lse_s)
    ws = torch.empty(max(16, dsa.dsa_workspace_bytes(dsa.DSA_OP_DENSE_MLA_FWD, 1, 64, 500, 0, 128)),
                     dtype=torch.uint8, device="cuda")
    dsa.dsa_sparse_mla_fwd(dw.q, dw.kv, idx, wl.scale, o_s, lse_s, p_s, ws)
    dsa.dsa_dense_mla_fwd(dw.q, dw.kv, wl.scale, o_d, lse_d, p_d, ws)
    assert dsa.dsa_last_device_status() == 0
    # same kernel, same entries in the same order: identical results
    assert torch.equal(o_s, o_d) and torch.equal(lse_s, lse_d) and torch.equal(p_s, p_d)


def test_dense_warmup_16k_sampled_rows(dsa):
    wl = dsa_inputs.WORKLOADS["dense_warmup_16k"]
    dw = parity.DeviceWorkload(wl)
    res = parity.run_path(dw)
    torch.cuda.synchronize()
    rows = sorted(set([0, 1, 2047, 2048, wl.Lq - 1] + [int(x) for x in dsa_inputs.uniform_int(wl.seed, 99, 27, 0, wl.rows - 1)]))
    _check_rows(wl, dw, res, rows)
