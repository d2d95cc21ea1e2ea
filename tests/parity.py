"""Shared helpers of the parity tests: device upload of seeded workloads, running the
GPU path through the C ABI, and the comparison rules.

Comparison rules (oracle = fp64 CPU code under oracle/):
  indexer scores   bit-exact (integer-valued FP8 inputs make every partial sum exact in fp32)
  top-k sets       exact, as ascending positions padded with -1 (the tie rule makes S_t unique)
  attention out    max|err| <= 1e-2 * max|ref| + 1e-3 per query row (bf16 inputs, fp32 accumulation)
  lse              |err| <= 2e-3 absolute (fp32 logits of bf16 products, natural log)
  p_sel            |err| <= 1e-3 * max p + 1e-6 per row
  KL loss          relative error <= 1e-3
"""
from __future__ import annotations

import numpy as np
import torch

import dsa_inputs

ATT_RTOL, ATT_ATOL = 1e-2, 1e-3
LSE_ATOL = 2e-3
P_RTOL, P_ATOL = 1e-3, 1e-6
KL_RTOL = 1e-3


def bf16_bits_to_torch(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def e4m3_to_torch(b: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(b)).view(torch.float8_e4m3fn)


class DeviceWorkload:
    """All inputs of a workload drawn from the seeded streams and copied to cuda:0."""

    def __init__(self, wl: dsa_inputs.Workload, device: str = "cuda", with_attention: bool = True):
        self.wl = wl
        B, Lq, Lk = wl.B, wl.Lq, wl.Lk
        self.qI_np = dsa_inputs.q_index(wl)
        self.kI_np = dsa_inputs.k_index(wl)
        self.w_np = dsa_inputs.w_index(wl)
        self.qI = e4m3_to_torch(self.qI_np).reshape(B, Lq, wl.H_I, wl.d_I).to(device)
        self.kI = e4m3_to_torch(self.kI_np).reshape(B, Lk, wl.d_I).to(device)
        self.w = torch.from_numpy(self.w_np).reshape(B, Lq, wl.H_I).to(device)
        self.q = self.kv = None
        if with_attention:
            self.q = bf16_bits_to_torch(dsa_inputs.q_attn(wl)).reshape(B, Lq, wl.H, wl.d_qk).to(device)
            self.kv = bf16_bits_to_torch(dsa_inputs.kv_latent(wl)).reshape(B, Lk, wl.d_qk).to(device)

    def q_rows_np(self, rows) -> np.ndarray:
        return np.stack([dsa_inputs.q_attn(self.wl, r, 1)[0] for r in rows])

    def kv_np(self) -> np.ndarray:
        return self.kv.view(torch.int16).cpu().numpy().view(np.uint16)


def run_dense_path(dw: DeviceWorkload):
    """The dense warm-up step through the C ABI: indexer -> dense attention with the target
    p over every s <= t -> eq. (3) loss; returns device tensors."""
    import sparse_attention_tcgen05_b200 as dsa

    wl = dw.wl
    dev = dw.qI.device
    scores = torch.empty(wl.B, wl.Lq, wl.Lk, dtype=torch.float32, device=dev)
    out = torch.empty(wl.B, wl.Lq, wl.H, wl.d_v, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(wl.B, wl.Lq, wl.H, dtype=torch.float32, device=dev)
    p_full = torch.empty(wl.B, wl.Lq, wl.Lk, dtype=torch.float32, device=dev)
    ws_bytes = dsa.dsa_workspace_bytes(dsa.DSA_OP_DENSE_MLA_FWD, wl.B, wl.Lq, wl.Lk, 0, wl.H)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    per = torch.empty(wl.B, wl.Lq, dtype=torch.float32, device=dev)
    dsa.dsa_indexer(dw.qI, dw.kI, dw.w, scores)
    dsa.dsa_dense_mla_fwd(dw.q, dw.kv, wl.scale, out, lse, p_full, ws)
    dsa.dsa_indexer_kl_dense(scores, p_full, loss, per)
    assert dsa.dsa_last_device_status() == 0
    return {"scores": scores, "out": out, "lse": lse, "p_full": p_full, "loss": loss, "loss_rows": per}


def oracle_dense_row(dw: DeviceWorkload, r: int, kv_np=None):
    """The oracle's dense warm-up results for flat row r: scores, out, lse, p[0..t], KL."""
    from oracle import oracle as ref

    wl = dw.wl
    b, i = divmod(r, wl.Lq)
    t = wl.t_of(i)
    kv = dsa_inputs.kv_latent(wl, b) if kv_np is None else kv_np[b]
    q = dsa_inputs.q_attn(wl, r, 1)[0]
    sc = ref.indexer_row(dw.qI_np.reshape(wl.rows, wl.H_I, wl.d_I)[r], dw.kI_np[b],
                         dw.w_np.reshape(wl.rows, wl.H_I)[r], t)
    out, lse, _ = ref.dense_mla_row(q, kv, t, wl.d_v, wl.scale)
    p = ref.dense_p_row(q, kv, t, wl.scale)
    return {"scores": sc, "out": out, "lse": lse, "p": p, "kl": ref.dense_kl_row(sc, t, p), "t": t}


def run_path(dw: DeviceWorkload, emit_p: bool | None = None):
    """indexer -> top-k -> sparse MLA [-> KL] through the C ABI; returns device tensors."""
    import sparse_attention_tcgen05_b200 as dsa

    wl = dw.wl
    if wl.dense:
        return run_dense_path(dw)
    emit_p = wl.emit_p if emit_p is None else emit_p
    dev = dw.qI.device
    scores = torch.empty(wl.B, wl.Lq, wl.Lk, dtype=torch.float32, device=dev)
    idx = torch.empty(wl.B, wl.Lq, wl.k, dtype=torch.int32, device=dev)
    out = torch.empty(wl.B, wl.Lq, wl.H, wl.d_v, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(wl.B, wl.Lq, wl.H, dtype=torch.float32, device=dev)
    p_sel = torch.empty(wl.B, wl.Lq, wl.k, dtype=torch.float32, device=dev) if emit_p else None
    ws_bytes = dsa.dsa_workspace_bytes(dsa.DSA_OP_SPARSE_MLA_FWD, wl.B, wl.Lq, wl.Lk, wl.k, wl.H)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    if wl.Lq == 1:  # decode: the fused indexer -> top-k entry point, as the bench runs it
        ws_ix = torch.zeros(max(16, dsa.dsa_workspace_bytes(dsa.DSA_OP_INDEXER_TOPK, wl.B, 1, wl.Lk, wl.k, 0)),
                            dtype=torch.uint8, device=dev)  # zero-filled once
        dsa.dsa_indexer_topk(dw.qI, dw.kI, dw.w, scores, idx, ws_ix)
    else:
        dsa.dsa_indexer(dw.qI, dw.kI, dw.w, scores)
        dsa.dsa_topk(scores, idx)
    dsa.dsa_sparse_mla_fwd(dw.q, dw.kv, idx, wl.scale, out, lse, p_sel, ws)
    res = {"scores": scores, "idx": idx, "out": out, "lse": lse, "p_sel": p_sel}
    if emit_p:
        loss = torch.empty(1, dtype=torch.float32, device=dev)
        per = torch.empty(wl.B, wl.Lq, dtype=torch.float32, device=dev)
        dsa.dsa_indexer_kl(scores, idx, p_sel, loss, per)
        res["loss"], res["loss_rows"] = loss, per
    assert dsa.dsa_last_device_status() == 0
    return res


def oracle_rows(dw: DeviceWorkload, rows, nthreads: int | None = None, want_scores: bool = True):
    """The oracle's whole-path results for the listed flat rows (inputs drawn afresh)."""
    import os

    from oracle import oracle as ref

    wl = dw.wl
    rows = list(rows)
    qI = dw.qI_np.reshape(wl.rows, wl.H_I, wl.d_I)[rows]
    w = dw.w_np.reshape(wl.rows, wl.H_I)[rows]
    q = np.stack([dsa_inputs.q_attn(wl, r, 1)[0] for r in rows])
    kv = dsa_inputs.kv_latent(wl)
    nthreads = nthreads or max(1, os.cpu_count() or 1)
    return ref.path_rows(wl, rows, qI, dw.kI_np, w, q, kv, rows_packed=True, nthreads=nthreads,
                         want_scores=want_scores)


def check_attention_row(out_gpu: np.ndarray, out_ref: np.ndarray, what: str = "") -> float:
    err = np.abs(out_gpu.astype(np.float64) - out_ref).max()
    bound = ATT_RTOL * np.abs(out_ref).max() + ATT_ATOL
    assert err <= bound, f"{what}: attention max|err| {err:.3e} > {bound:.3e}"
    return err


def check_p_row(p_gpu: np.ndarray, p_ref: np.ndarray, what: str = "") -> None:
    err = np.abs(p_gpu.astype(np.float64) - p_ref).max()
    bound = P_RTOL * np.abs(p_ref).max() + P_ATOL
    assert err <= bound, f"{what}: p max|err| {err:.3e} > {bound:.3e}"
