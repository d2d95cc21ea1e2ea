"""ctypes wrapper around the fp64 CPU oracle (dsa_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by the tests, by the smoke check and by the
bench's CPU-baseline leg.  The GPU product package never imports this module.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libdsa_oracle.so")


def build(force: bool = False) -> str:
    """Compile the oracle with plain IEEE fp64 semantics (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
                               "-pthread", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        vp, i32, i64, f64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.ref_e4m3_to_double.argtypes = [ctypes.c_uint8]
        lib.ref_e4m3_to_double.restype = f64
        lib.ref_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.ref_bf16_to_double.restype = f64
        lib.ref_indexer_row.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp]
        lib.ref_topk_row.argtypes = [vp, i32, i32, vp]
        lib.ref_topk_row.restype = i32
        lib.ref_sparse_mla_row.argtypes = [vp, vp, vp, i32, i32, i32, i32, f64, vp, vp, vp]
        lib.ref_p_sel_row.argtypes = [vp, vp, i32, i32, vp]
        lib.ref_kl_row.argtypes = [vp, vp, vp, i32]
        lib.ref_kl_row.restype = f64
        lib.ref_dense_mla_row.argtypes = [vp, vp, i32, i32, i32, i32, f64, vp, vp, vp]
        lib.ref_dense_p_row.argtypes = [vp, vp, i32, i32, i32, f64, vp]
        lib.ref_dense_kl_row.argtypes = [vp, i32, vp]
        lib.ref_dense_kl_row.restype = f64
        lib.ref_masked_mha_row.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, f64, vp, vp]
        lib.ref_block_mean.argtypes = [vp, i32, i32, i32, vp]
        lib.ref_block_score.argtypes = [vp, vp, vp, i32, i32]
        lib.ref_block_score.restype = f64
        lib.ref_hisa_row.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, vp, vp]
        lib.ref_hisa_row.restype = i32
        lib.ref_indexer_loss_row_f64.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32]
        lib.ref_indexer_loss_row_f64.restype = f64
        lib.ref_indexer_grad_row.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, vp, vp, vp, vp]
        lib.ref_path_rows.argtypes = [vp, vp, vp, vp, vp, i32, vp, i64, i32, i32, i32, i32, i32, i32,
                                      i32, i32, i32, f64, i32, vp, vp, vp, vp, vp, vp, i32]
        _lib = lib
    return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data


def e4m3_to_double(b: int) -> float:
    return _load().ref_e4m3_to_double(int(b))


def bf16_to_double(h: int) -> float:
    return _load().ref_bf16_to_double(int(h))


def indexer_row(q_row, k_seq, w_row, t: int) -> np.ndarray:
    """Scores I[t, 0:Lk] of one query (eq. (1)); q_row [H_I, d_I] e4m3 bytes,
    k_seq [Lk, d_I] e4m3 bytes, w_row [H_I] fp32."""
    q_row, qp = _c(q_row, np.uint8)
    k_seq, kp = _c(k_seq, np.uint8)
    w_row, wp = _c(w_row, np.float32)
    H_I, d_I = q_row.shape
    Lk = k_seq.shape[0]
    out = np.empty(Lk, dtype=np.float64)
    _load().ref_indexer_row(qp, kp, wp, Lk, t, H_I, d_I, out.ctypes.data)
    return out


def topk_row(scores, t: int, k: int) -> tuple[np.ndarray, int]:
    """S_t as ascending positions padded with -1, and its size min(k, t+1)."""
    scores, sp = _c(scores, np.float64)
    idx = np.empty(k, dtype=np.int32)
    n = _load().ref_topk_row(sp, t, k, idx.ctypes.data)
    return idx, n


def sparse_mla_row(q_row, kv_seq, idx, d_v: int, scale: float, want_P: bool = False):
    """(out [H, d_v], lse [H], P [H, k] or None) of one query over the selected latents."""
    q_row, qp = _c(q_row, np.uint16)
    kv_seq, kp = _c(kv_seq, np.uint16)
    idx, ip = _c(idx, np.int32)
    H, d_qk = q_row.shape
    k = idx.shape[0]
    out = np.empty((H, d_v), dtype=np.float64)
    lse = np.empty(H, dtype=np.float64)
    P = np.empty((H, k), dtype=np.float64) if want_P else None
    _load().ref_sparse_mla_row(qp, kp, ip, k, H, d_qk, d_v, float(scale), out.ctypes.data,
                               lse.ctypes.data, P.ctypes.data if want_P else None)
    return out, lse, P


def p_sel_row(P, idx) -> np.ndarray:
    P, pp = _c(P, np.float64)
    idx, ip = _c(idx, np.int32)
    H, k = P.shape
    p = np.empty(k, dtype=np.float64)
    _load().ref_p_sel_row(pp, ip, k, H, p.ctypes.data)
    return p


def kl_row(scores_row, idx, p) -> float:
    scores_row, sp = _c(scores_row, np.float64)
    idx, ip = _c(idx, np.int32)
    p, pp = _c(p, np.float64)
    return _load().ref_kl_row(sp, ip, pp, idx.shape[0])


def dense_mla_row(q_row, kv_seq, t: int, d_v: int, scale: float, want_A: bool = False):
    q_row, qp = _c(q_row, np.uint16)
    kv_seq, kp = _c(kv_seq, np.uint16)
    H, d_qk = q_row.shape
    out = np.empty((H, d_v), dtype=np.float64)
    lse = np.empty(H, dtype=np.float64)
    A = np.empty((H, t + 1), dtype=np.float64) if want_A else None
    _load().ref_dense_mla_row(qp, kp, t, H, d_qk, d_v, float(scale), out.ctypes.data, lse.ctypes.data,
                              A.ctypes.data if want_A else None)
    return out, lse, A


def dense_p_row(q_row, kv_seq, t: int, scale: float) -> np.ndarray:
    """Dense warm-up target p[t, 0..t]: dense MQA attention over every s <= t, summed over
    heads, L1-normalised (Stage 1 of "DSA Continued Pre-Training")."""
    q_row, qp = _c(q_row, np.uint16)
    kv_seq, kp = _c(kv_seq, np.uint16)
    H, d_qk = q_row.shape
    p = np.empty(t + 1, dtype=np.float64)
    _load().ref_dense_p_row(qp, kp, t, H, d_qk, float(scale), p.ctypes.data)
    return p


def dense_kl_row(scores_row, t: int, p) -> float:
    """One row of eq. (3): KL(p[t,:] || Softmax(I[t, 0..t]))."""
    scores_row, sp = _c(scores_row, np.float64)
    p, pp = _c(p, np.float64)
    return _load().ref_dense_kl_row(sp, t, pp)


def masked_mha_row(q_row, k_seq, v_seq, idx, scale: float):
    """MHA-mode attention of one query restricted to the positions of idx: q_row [H, dqk],
    k_seq [L, H, dqk], v_seq [L, H, dv] (real values); returns (out [H, dv], lse [H])."""
    q_row, qp = _c(q_row, np.float64)
    k_seq, kp = _c(k_seq, np.float64)
    v_seq, vp_ = _c(v_seq, np.float64)
    idx, ip = _c(idx, np.int32)
    H, dqk = q_row.shape
    dv = v_seq.shape[2]
    out = np.empty((H, dv))
    lse = np.empty(H)
    _load().ref_masked_mha_row(qp, kp, vp_, ip, idx.shape[0], H, dqk, dv, float(scale), out.ctypes.data,
                               lse.ctypes.data)
    return out, lse


def block_mean(k_seq, s0: int, n: int) -> np.ndarray:
    """Mean of the e4m3 keys [s0, s0+n) of k_seq [Lk, d_I]."""
    k_seq, kp = _c(k_seq, np.uint8)
    out = np.empty(k_seq.shape[1])
    _load().ref_block_mean(kp, s0, n, k_seq.shape[1], out.ctypes.data)
    return out


def block_score(q_row, mean, w_row) -> float:
    """sum_j w_j ReLU(q_j . mean) for e4m3 q_row [H_I, d_I] and a real mean key."""
    q_row, qp = _c(q_row, np.uint8)
    mean, mp = _c(mean, np.float64)
    w_row, wp = _c(w_row, np.float32)
    H_I, d_I = q_row.shape
    return _load().ref_block_score(qp, mp, wp, H_I, d_I)


def hisa_row(q_row, k_seq, w_row, t: int, bsize: int, r: int, k: int):
    """HISA's selection for query t: (idx [k] ascending, -1 padded; kept blocks [r]; |S|)."""
    q_row, qp = _c(q_row, np.uint8)
    k_seq, kp = _c(k_seq, np.uint8)
    w_row, wp = _c(w_row, np.float32)
    H_I, d_I = q_row.shape
    idx = np.empty(k, dtype=np.int32)
    blocks = np.empty(r, dtype=np.int32)
    n = _load().ref_hisa_row(qp, kp, wp, k_seq.shape[0], t, H_I, d_I, bsize, r, k, idx.ctypes.data,
                             blocks.ctypes.data)
    return idx, blocks, n


def indexer_loss_row_f64(q_row, k_seq, w_row, idx, p) -> float:
    """One row's indexer loss from real-valued (fp64) indexer inputs, the selection `idx` fixed."""
    q_row, qp = _c(q_row, np.float64)
    k_seq, kp = _c(k_seq, np.float64)
    w_row, wp = _c(w_row, np.float64)
    idx, ip = _c(idx, np.int32)
    p, pp = _c(p, np.float64)
    H_I, d_I = q_row.shape
    return _load().ref_indexer_loss_row_f64(qp, kp, wp, ip, pp, idx.shape[0], H_I, d_I)


def indexer_grad_row(q_row, k_seq, w_row, idx, p, dk=None):
    """(dq [H_I, d_I], dw [H_I], dk [Lk, d_I], g [k]) of one row's indexer loss; dk accumulates
    into the array passed (zeros if None)."""
    q_row, qp = _c(q_row, np.float64)
    k_seq, kp = _c(k_seq, np.float64)
    w_row, wp = _c(w_row, np.float64)
    idx, ip = _c(idx, np.int32)
    p, pp = _c(p, np.float64)
    H_I, d_I = q_row.shape
    dq = np.empty((H_I, d_I))
    dw = np.empty(H_I)
    if dk is None:
        dk = np.zeros_like(k_seq)
    assert dk.dtype == np.float64 and dk.flags.c_contiguous and dk.shape == k_seq.shape
    g = np.empty(idx.shape[0])
    _load().ref_indexer_grad_row(qp, kp, wp, ip, pp, idx.shape[0], H_I, d_I, dq.ctypes.data, dw.ctypes.data,
                                 dk.ctypes.data, g.ctypes.data)
    return dq, dw, dk, g


def path_rows(wl, rows, qI, kI, w, q, kv, rows_packed: bool, nthreads: int = 1,
              want_scores: bool = True):
    """Whole path (indexer -> top-k -> sparse MLA [-> p -> KL]) for the listed flat rows.

    qI/w/q hold either every row (rows_packed=False) or only the listed rows in order
    (rows_packed=True); kI/kv hold every sequence.  Returns a dict of fp64 results."""
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    n = rows.shape[0]
    qI, qIp = _c(qI, np.uint8)
    kI, kIp = _c(kI, np.uint8)
    w, wp = _c(w, np.float32)
    q, qp = _c(q, np.uint16)
    kv, kvp = _c(kv, np.uint16)
    res = {
        "scores": np.empty((n, wl.Lk), dtype=np.float64) if want_scores else None,
        "idx": np.empty((n, wl.k), dtype=np.int32),
        "out": np.empty((n, wl.H, wl.d_v), dtype=np.float64),
        "lse": np.empty((n, wl.H), dtype=np.float64),
        "p": np.empty((n, wl.k), dtype=np.float64) if wl.emit_p else None,
        "kl": np.empty(n, dtype=np.float64),
    }
    ptr = lambda a: None if a is None else a.ctypes.data
    _load().ref_path_rows(qIp, kIp, wp, qp, kvp, int(rows_packed), rows.ctypes.data, n, wl.B, wl.Lq,
                          wl.Lk, wl.H_I, wl.d_I, wl.k, wl.H, wl.d_qk, wl.d_v, float(wl.scale),
                          int(wl.emit_p), ptr(res["scores"]), ptr(res["idx"]), ptr(res["out"]),
                          ptr(res["lse"]), ptr(res["p"]), ptr(res["kl"]), int(nthreads))
    return res
