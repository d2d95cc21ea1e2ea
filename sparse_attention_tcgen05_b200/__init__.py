"""Python binding of libdsa.so, the DSA hot path on B200 (sm_100a).

Argument marshalling only: every function checks the torch tensors it is given
(device, dtype, shape, contiguity), passes their device pointers and the current
CUDA stream to the C entry point of the same name, and raises DsaError on a
non-zero status.  All arithmetic runs in the library's CUDA kernels; there is no
CPU path.  Layouts and semantics are those of include/dsa.h.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

__all__ = [
    "DsaError", "load", "dsa_status_str", "dsa_version", "dsa_workspace_bytes", "dsa_indexer",
    "dsa_topk", "dsa_sparse_mla_fwd", "dsa_indexer_kl", "dsa_indexer_kl_noalloc",
    "dsa_last_device_status", "dsa_set_wait_limit_ns", "dsa_selftest_wait", "dsa_dense_mla_fwd",
    "dsa_indexer_kl_dense", "dsa_indexer_topk", "dsa_indexer_bwd", "dsa_indexer_topk_paged",
    "dsa_sparse_mla_fwd_paged", "dsa_hisa_workspace_bytes", "dsa_hisa_block_sums", "dsa_hisa_topk",
    "dsa_masked_mha_fwd",
    "DSA_OP_INDEXER", "DSA_OP_TOPK", "DSA_OP_SPARSE_MLA_FWD", "DSA_OP_INDEXER_KL",
    "DSA_OP_DENSE_MLA_FWD", "DSA_OP_INDEXER_KL_DENSE", "DSA_OP_INDEXER_TOPK", "DSA_OP_MASKED_MHA", "EXPORTED",
]

DSA_OP_INDEXER, DSA_OP_TOPK, DSA_OP_SPARSE_MLA_FWD, DSA_OP_INDEXER_KL = 0, 1, 2, 3
DSA_OP_DENSE_MLA_FWD, DSA_OP_INDEXER_KL_DENSE, DSA_OP_INDEXER_TOPK, DSA_OP_MASKED_MHA = 4, 5, 6, 7
EXPORTED = ("dsa_status_str", "dsa_version", "dsa_workspace_bytes", "dsa_indexer", "dsa_topk",
            "dsa_sparse_mla_fwd", "dsa_indexer_kl", "dsa_indexer_kl_noalloc",
            "dsa_last_device_status", "dsa_set_wait_limit_ns", "dsa_selftest_wait",
            "dsa_dense_mla_fwd", "dsa_indexer_kl_dense", "dsa_indexer_topk", "dsa_indexer_bwd",
            "dsa_indexer_topk_paged", "dsa_sparse_mla_fwd_paged", "dsa_hisa_workspace_bytes",
            "dsa_hisa_block_sums", "dsa_hisa_topk", "dsa_masked_mha_fwd")


class DsaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {dsa_status_str(code)} ({code})")
        self.code = code


_lib = None


def load(rebuild: bool = False) -> ctypes.CDLL:
    """Load (building first if missing or stale) the in-tree libdsa.so."""
    global _lib
    if _lib is None or rebuild:
        path = _build.LIB
        if rebuild or _build.stale():
            path = _build.build()
        lib = ctypes.CDLL(path)
        vp, i32, sz, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
        lib.dsa_status_str.argtypes = [i32]
        lib.dsa_status_str.restype = ctypes.c_char_p
        lib.dsa_version.restype = i32
        lib.dsa_workspace_bytes.argtypes = [i32, i32, i32, i32, i32, i32]
        lib.dsa_workspace_bytes.restype = sz
        lib.dsa_indexer.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, vp, sz, vp]
        lib.dsa_topk.argtypes = [vp, vp, i32, i32, i32, i32, vp, sz, vp]
        lib.dsa_sparse_mla_fwd.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, f32, vp,
                                           vp, vp, vp, sz, vp]
        lib.dsa_indexer_kl.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, vp, vp, sz, vp]
        lib.dsa_indexer_kl_noalloc.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, vp, vp]
        lib.dsa_last_device_status.argtypes = [vp]
        lib.dsa_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        lib.dsa_selftest_wait.argtypes = [vp]
        lib.dsa_dense_mla_fwd.argtypes = [vp, vp, i32, i32, i32, i32, i32, i32, f32, vp, vp, vp, vp, sz, vp]
        lib.dsa_indexer_kl_dense.argtypes = [vp, vp, i32, i32, i32, vp, vp, vp, sz, vp]
        lib.dsa_indexer_topk.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, sz, vp]
        lib.dsa_indexer_bwd.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, vp, vp, vp]
        lib.dsa_indexer_topk_paged.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, vp,
                                               sz, vp]
        lib.dsa_sparse_mla_fwd_paged.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, f32,
                                                 vp, vp, vp, sz, vp]
        lib.dsa_hisa_workspace_bytes.argtypes = [i32, i32, i32, i32, i32]
        lib.dsa_hisa_workspace_bytes.restype = sz
        lib.dsa_hisa_block_sums.argtypes = [vp, i32, i32, i32, i32, vp, vp]
        lib.dsa_hisa_topk.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, vp, vp, vp, sz, vp]
        lib.dsa_masked_mha_fwd.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, vp, vp, vp, sz, vp]
        for name in ("dsa_indexer", "dsa_topk", "dsa_sparse_mla_fwd", "dsa_indexer_kl",
                     "dsa_indexer_kl_noalloc", "dsa_last_device_status", "dsa_set_wait_limit_ns",
                     "dsa_selftest_wait", "dsa_dense_mla_fwd", "dsa_indexer_kl_dense", "dsa_indexer_topk",
                     "dsa_indexer_bwd", "dsa_indexer_topk_paged", "dsa_sparse_mla_fwd_paged",
                     "dsa_hisa_block_sums", "dsa_hisa_topk", "dsa_masked_mha_fwd"):
            getattr(lib, name).restype = i32
        _lib = lib
    return _lib


def dsa_status_str(code: int) -> str:
    return load().dsa_status_str(int(code)).decode()


def dsa_version() -> int:
    return load().dsa_version()


def dsa_workspace_bytes(op: int, B: int, Lq: int, Lk: int, k: int, H: int) -> int:
    return int(load().dsa_workspace_bytes(op, B, Lq, Lk, k, H))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(t: torch.Tensor, name: str, dtype, shape) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _raise(fn: str, code: int) -> None:
    if code != 0:
        raise DsaError(fn, code)


def _ws(ws):
    if ws is None:
        return None, 0
    if ws.device.type != "cuda" or not ws.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    return ctypes.c_void_p(ws.data_ptr()), ws.numel() * ws.element_size()


def dsa_indexer(q_fp8: torch.Tensor, k_fp8: torch.Tensor, w: torch.Tensor, scores: torch.Tensor,
                stream=None) -> None:
    """scores[B,Lq,Lk] = lightning-indexer scores (eq. (1)) of q_I [B,Lq,H_I,d_I] e4m3,
    k_I [B,Lk,d_I] e4m3 and w [B,Lq,H_I] fp32; -inf above the causal diagonal."""
    B, Lq, H_I, d_I = q_fp8.shape
    Lk = k_fp8.shape[1]
    _check(q_fp8, "q_fp8", torch.float8_e4m3fn, (B, Lq, H_I, d_I))
    _check(k_fp8, "k_fp8", torch.float8_e4m3fn, (B, Lk, d_I))
    _check(w, "w", torch.float32, (B, Lq, H_I))
    _check(scores, "scores", torch.float32, (B, Lq, Lk))
    _raise("dsa_indexer", load().dsa_indexer(_ptr(q_fp8), _ptr(k_fp8), _ptr(w), _ptr(scores), B, Lq,
                                             Lk, H_I, d_I, None, 0, _stream(stream)))


def dsa_topk(scores: torch.Tensor, idx: torch.Tensor, stream=None) -> None:
    """idx[B,Lq,k] = ascending positions of the top-k scores of each row (s <= t), ties to the
    smaller position, -1 padded."""
    B, Lq, Lk = scores.shape
    k = idx.shape[2]
    _check(scores, "scores", torch.float32, (B, Lq, Lk))
    _check(idx, "idx", torch.int32, (B, Lq, k))
    _raise("dsa_topk", load().dsa_topk(_ptr(scores), _ptr(idx), B, Lq, Lk, k, None, 0,
                                       _stream(stream)))


def dsa_indexer_topk(q_fp8: torch.Tensor, k_fp8: torch.Tensor, w: torch.Tensor, scores: torch.Tensor,
                     idx: torch.Tensor, ws: torch.Tensor | None = None, stream=None) -> None:
    """dsa_indexer then dsa_topk in one call (fused for decode: the indexer counts the top-k's
    first radix digit); ws: dsa_workspace_bytes(DSA_OP_INDEXER_TOPK, ...) bytes."""
    B, Lq, H_I, d_I = q_fp8.shape
    Lk = k_fp8.shape[1]
    k = idx.shape[2]
    _check(q_fp8, "q_fp8", torch.float8_e4m3fn, (B, Lq, H_I, d_I))
    _check(k_fp8, "k_fp8", torch.float8_e4m3fn, (B, Lk, d_I))
    _check(w, "w", torch.float32, (B, Lq, H_I))
    _check(scores, "scores", torch.float32, (B, Lq, Lk))
    _check(idx, "idx", torch.int32, (B, Lq, k))
    wsp, wsb = _ws(ws)
    _raise("dsa_indexer_topk",
           load().dsa_indexer_topk(_ptr(q_fp8), _ptr(k_fp8), _ptr(w), _ptr(scores), _ptr(idx), B, Lq, Lk, H_I,
                                   d_I, k, wsp, wsb, _stream(stream)))


def dsa_sparse_mla_fwd(q: torch.Tensor, kv: torch.Tensor, idx: torch.Tensor, scale: float,
                       out: torch.Tensor, lse: torch.Tensor | None = None,
                       p_sel: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                       stream=None) -> None:
    """MQA-mode attention of q [B,Lq,H,d_qk] over the selected latents kv[b, idx] (bf16);
    out [B,Lq,H,d_v] bf16, optional lse [B,Lq,H] and head-summed p_sel [B,Lq,k] (fp32)."""
    B, Lq, H, d_qk = q.shape
    Lk = kv.shape[1]
    k = idx.shape[2]
    d_v = out.shape[3]
    _check(q, "q", torch.bfloat16, (B, Lq, H, d_qk))
    _check(kv, "kv", torch.bfloat16, (B, Lk, d_qk))
    _check(idx, "idx", torch.int32, (B, Lq, k))
    _check(out, "out", torch.bfloat16, (B, Lq, H, d_v))
    if lse is not None:
        _check(lse, "lse", torch.float32, (B, Lq, H))
    if p_sel is not None:
        _check(p_sel, "p_sel", torch.float32, (B, Lq, k))
    wsp, wsb = _ws(ws)
    _raise("dsa_sparse_mla_fwd",
           load().dsa_sparse_mla_fwd(_ptr(q), _ptr(kv), _ptr(idx), B, Lq, Lk, H, d_qk, d_v, k,
                                     float(scale), _ptr(out), _ptr(lse), _ptr(p_sel), wsp, wsb,
                                     _stream(stream)))


def dsa_indexer_kl(scores: torch.Tensor, idx: torch.Tensor, p_sel: torch.Tensor, loss: torch.Tensor,
                   loss_per_query: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                   stream=None) -> None:
    """loss[0] = sum over rows of KL(p_sel || Softmax(scores[idx])) (eq. (4))."""
    B, Lq, Lk = scores.shape
    k = idx.shape[2]
    _check(scores, "scores", torch.float32, (B, Lq, Lk))
    _check(idx, "idx", torch.int32, (B, Lq, k))
    _check(p_sel, "p_sel", torch.float32, (B, Lq, k))
    _check(loss, "loss", torch.float32, (1,))
    if loss_per_query is not None:
        _check(loss_per_query, "loss_per_query", torch.float32, (B, Lq))
    wsp, wsb = _ws(ws)
    _raise("dsa_indexer_kl",
           load().dsa_indexer_kl(_ptr(scores), _ptr(idx), _ptr(p_sel), B, Lq, Lk, k, _ptr(loss),
                                 _ptr(loss_per_query), wsp, wsb, _stream(stream)))


def dsa_dense_mla_fwd(q: torch.Tensor, kv: torch.Tensor, scale: float, out: torch.Tensor,
                      lse: torch.Tensor | None = None, p_full: torch.Tensor | None = None,
                      ws: torch.Tensor | None = None, stream=None) -> None:
    """Dense causal MQA of q [B,Lq,H,d_qk] over every kv[b, s<=t] (the dense warm-up's main
    attention); out [B,Lq,H,d_v] bf16, optional lse [B,Lq,H] and the head-summed target
    p_full [B,Lq,Lk] (fp32, 0 for s > t)."""
    B, Lq, H, d_qk = q.shape
    Lk = kv.shape[1]
    d_v = out.shape[3]
    _check(q, "q", torch.bfloat16, (B, Lq, H, d_qk))
    _check(kv, "kv", torch.bfloat16, (B, Lk, d_qk))
    _check(out, "out", torch.bfloat16, (B, Lq, H, d_v))
    if lse is not None:
        _check(lse, "lse", torch.float32, (B, Lq, H))
    if p_full is not None:
        _check(p_full, "p_full", torch.float32, (B, Lq, Lk))
    wsp, wsb = _ws(ws)
    _raise("dsa_dense_mla_fwd",
           load().dsa_dense_mla_fwd(_ptr(q), _ptr(kv), B, Lq, Lk, H, d_qk, d_v, float(scale), _ptr(out),
                                    _ptr(lse), _ptr(p_full), wsp, wsb, _stream(stream)))


def dsa_indexer_kl_dense(scores: torch.Tensor, p_full: torch.Tensor, loss: torch.Tensor,
                         loss_per_query: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                         stream=None) -> None:
    """loss[0] = sum over rows of KL(p_full[t, 0..t] || Softmax(scores[t, 0..t])) (eq. (3))."""
    B, Lq, Lk = scores.shape
    _check(scores, "scores", torch.float32, (B, Lq, Lk))
    _check(p_full, "p_full", torch.float32, (B, Lq, Lk))
    _check(loss, "loss", torch.float32, (1,))
    if loss_per_query is not None:
        _check(loss_per_query, "loss_per_query", torch.float32, (B, Lq))
    wsp, wsb = _ws(ws)
    _raise("dsa_indexer_kl_dense",
           load().dsa_indexer_kl_dense(_ptr(scores), _ptr(p_full), B, Lq, Lk, _ptr(loss),
                                       _ptr(loss_per_query), wsp, wsb, _stream(stream)))


def dsa_indexer_bwd(q_fp8: torch.Tensor, k_fp8: torch.Tensor, w: torch.Tensor, scores: torch.Tensor,
                    idx: torch.Tensor | None, p_sel: torch.Tensor, dq: torch.Tensor, dw: torch.Tensor,
                    dk: torch.Tensor, stream=None) -> None:
    """Gradients (dq, dw, dk) of the indexer loss with respect to q_I, w and k_I, the selection
    idx held fixed (idx None: the dense warm-up loss over every s <= t, p_sel [B,Lq,Lk])."""
    B, Lq, H_I, d_I = q_fp8.shape
    Lk = k_fp8.shape[1]
    k = Lk if idx is None else idx.shape[2]
    _check(q_fp8, "q_fp8", torch.float8_e4m3fn, (B, Lq, H_I, d_I))
    _check(k_fp8, "k_fp8", torch.float8_e4m3fn, (B, Lk, d_I))
    _check(w, "w", torch.float32, (B, Lq, H_I))
    _check(scores, "scores", torch.float32, (B, Lq, Lk))
    if idx is not None:
        _check(idx, "idx", torch.int32, (B, Lq, k))
    _check(p_sel, "p_sel", torch.float32, (B, Lq, k))
    _check(dq, "dq", torch.float32, (B, Lq, H_I, d_I))
    _check(dw, "dw", torch.float32, (B, Lq, H_I))
    _check(dk, "dk", torch.float32, (B, Lk, d_I))
    _raise("dsa_indexer_bwd",
           load().dsa_indexer_bwd(_ptr(q_fp8), _ptr(k_fp8), _ptr(w), _ptr(scores), _ptr(idx), _ptr(p_sel), B, Lq,
                                  Lk, H_I, d_I, k, _ptr(dq), _ptr(dw), _ptr(dk), _stream(stream)))


def dsa_indexer_topk_paged(q_fp8: torch.Tensor, k_pages: torch.Tensor, w: torch.Tensor,
                           block_table: torch.Tensor, seq_lens: torch.Tensor, scores: torch.Tensor,
                           idx: torch.Tensor, ws: torch.Tensor | None = None, stream=None) -> None:
    """Decode indexer + top-k over a paged k_I cache: k_pages [num_pages, page_size, d_I] e4m3,
    block_table [B, max_pages] int32, seq_lens [B] int32; scores [B,1,max_len], idx [B,1,k]."""
    B, Lq, H_I, d_I = q_fp8.shape
    num_pages, page_size = k_pages.shape[0], k_pages.shape[1]
    max_len = scores.shape[2]
    k = idx.shape[2]
    _check(q_fp8, "q_fp8", torch.float8_e4m3fn, (B, 1, H_I, d_I))
    _check(k_pages, "k_pages", torch.float8_e4m3fn, (num_pages, page_size, d_I))
    _check(w, "w", torch.float32, (B, 1, H_I))
    _check(block_table, "block_table", torch.int32, (B, -(-max_len // page_size)))
    _check(seq_lens, "seq_lens", torch.int32, (B,))
    _check(scores, "scores", torch.float32, (B, 1, max_len))
    _check(idx, "idx", torch.int32, (B, 1, k))
    wsp, wsb = _ws(ws)
    _raise("dsa_indexer_topk_paged",
           load().dsa_indexer_topk_paged(_ptr(q_fp8), _ptr(k_pages), _ptr(w), _ptr(block_table), _ptr(seq_lens),
                                         _ptr(scores), _ptr(idx), B, max_len, num_pages, page_size, H_I, d_I, k,
                                         wsp, wsb, _stream(stream)))


def dsa_sparse_mla_fwd_paged(q: torch.Tensor, kv_pages: torch.Tensor, idx: torch.Tensor,
                             block_table: torch.Tensor, seq_lens: torch.Tensor, max_len: int, scale: float,
                             out: torch.Tensor, lse: torch.Tensor | None = None,
                             ws: torch.Tensor | None = None, stream=None) -> None:
    """Decode sparse MLA over a paged latent cache kv_pages [num_pages, page_size, 576] bf16."""
    B, Lq, H, d_qk = q.shape
    num_pages, page_size = kv_pages.shape[0], kv_pages.shape[1]
    k = idx.shape[2]
    d_v = out.shape[3]
    _check(q, "q", torch.bfloat16, (B, 1, H, d_qk))
    _check(kv_pages, "kv_pages", torch.bfloat16, (num_pages, page_size, d_qk))
    _check(idx, "idx", torch.int32, (B, 1, k))
    _check(block_table, "block_table", torch.int32, (B, -(-max_len // page_size)))
    _check(seq_lens, "seq_lens", torch.int32, (B,))
    _check(out, "out", torch.bfloat16, (B, 1, H, d_v))
    if lse is not None:
        _check(lse, "lse", torch.float32, (B, 1, H))
    wsp, wsb = _ws(ws)
    _raise("dsa_sparse_mla_fwd_paged",
           load().dsa_sparse_mla_fwd_paged(_ptr(q), _ptr(kv_pages), _ptr(idx), _ptr(block_table), _ptr(seq_lens), B,
                                           max_len, num_pages, page_size, H, d_qk, d_v, k, float(scale), _ptr(out),
                                           _ptr(lse), wsp, wsb, _stream(stream)))


def dsa_hisa_workspace_bytes(B: int, Lk: int, block: int, r: int, k: int) -> int:
    return int(load().dsa_hisa_workspace_bytes(B, Lk, block, r, k))


def dsa_hisa_block_sums(k_fp8: torch.Tensor, block: int, sums: torch.Tensor, stream=None) -> None:
    """Per-block key sums of a k_I cache [B, Lk, d_I] e4m3 -> sums [B, ceil(Lk/block), d_I] fp32."""
    B, Lk, d_I = k_fp8.shape
    _check(k_fp8, "k_fp8", torch.float8_e4m3fn, (B, Lk, d_I))
    _check(sums, "sums", torch.float32, (B, -(-Lk // block), d_I))
    _raise("dsa_hisa_block_sums",
           load().dsa_hisa_block_sums(_ptr(k_fp8), B, Lk, d_I, block, _ptr(sums), _stream(stream)))


def dsa_hisa_topk(q_fp8: torch.Tensor, k_fp8: torch.Tensor, w: torch.Tensor, sums: torch.Tensor, block: int,
                  r: int, idx: torch.Tensor, blocks: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                  stream=None) -> None:
    """HISA decode selection: the r best blocks by their mean key, then the exact top-k inside."""
    B, Lq, H_I, d_I = q_fp8.shape
    Lk = k_fp8.shape[1]
    k = idx.shape[2]
    _check(q_fp8, "q_fp8", torch.float8_e4m3fn, (B, 1, H_I, d_I))
    _check(k_fp8, "k_fp8", torch.float8_e4m3fn, (B, Lk, d_I))
    _check(w, "w", torch.float32, (B, 1, H_I))
    _check(sums, "sums", torch.float32, (B, -(-Lk // block), d_I))
    _check(idx, "idx", torch.int32, (B, 1, k))
    if blocks is not None:
        _check(blocks, "blocks", torch.int32, (B, 1, r))
    wsp, wsb = _ws(ws)
    _raise("dsa_hisa_topk",
           load().dsa_hisa_topk(_ptr(q_fp8), _ptr(k_fp8), _ptr(w), _ptr(sums), B, Lk, H_I, d_I, block, r, k,
                                _ptr(idx), _ptr(blocks), wsp, wsb, _stream(stream)))


def dsa_masked_mha_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, idx: torch.Tensor, scale: float,
                       out: torch.Tensor, lse: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                       stream=None) -> None:
    """MHA-mode causal prefill attention of q/k [B,L,H,192], v [B,L,H,128] (bf16) restricted to each
    query's top-k set idx [B,L,k]; out [B,L,H,128] bf16, optional lse [B,L,H]."""
    B, L, H, d_qk = q.shape
    kk = idx.shape[2]
    d_v = v.shape[3]
    _check(q, "q", torch.bfloat16, (B, L, H, d_qk))
    _check(k, "k", torch.bfloat16, (B, L, H, d_qk))
    _check(v, "v", torch.bfloat16, (B, L, H, d_v))
    _check(idx, "idx", torch.int32, (B, L, kk))
    _check(out, "out", torch.bfloat16, (B, L, H, d_v))
    if lse is not None:
        _check(lse, "lse", torch.float32, (B, L, H))
    wsp, wsb = _ws(ws)
    _raise("dsa_masked_mha_fwd",
           load().dsa_masked_mha_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(idx), B, L, H, d_qk, d_v, kk, float(scale),
                                     _ptr(out), _ptr(lse), wsp, wsb, _stream(stream)))


def dsa_indexer_kl_noalloc(scores: torch.Tensor, idx: torch.Tensor, p_sel: torch.Tensor,
                           loss: torch.Tensor, loss_per_query: torch.Tensor | None = None,
                           stream=None) -> None:
    """dsa_indexer_kl for callers that cannot provide scratch memory: the per-row terms use a
    fixed array inside the library (at most 1048576 rows; calls that overlap on the GPU race
    on it)."""
    B, Lq, Lk = scores.shape
    k = idx.shape[2]
    _check(scores, "scores", torch.float32, (B, Lq, Lk))
    _check(idx, "idx", torch.int32, (B, Lq, k))
    _check(p_sel, "p_sel", torch.float32, (B, Lq, k))
    _check(loss, "loss", torch.float32, (1,))
    if loss_per_query is not None:
        _check(loss_per_query, "loss_per_query", torch.float32, (B, Lq))
    _raise("dsa_indexer_kl_noalloc",
           load().dsa_indexer_kl_noalloc(_ptr(scores), _ptr(idx), _ptr(p_sel), B, Lq, Lk, k,
                                         _ptr(loss), _ptr(loss_per_query), _stream(stream)))


def dsa_set_wait_limit_ns(ns: int) -> None:
    """Bound (ns) of every in-kernel wait for kernels launched afterwards on the current device;
    0 restores the default of 2 s."""
    _raise("dsa_set_wait_limit_ns", load().dsa_set_wait_limit_ns(int(ns)))


def dsa_selftest_wait(stream=None) -> None:
    """Launch one warp that waits on an mbarrier nothing arrives on (it gives up after the wait
    limit and records DSA_ERR_TIMEOUT)."""
    _raise("dsa_selftest_wait", load().dsa_selftest_wait(_stream(stream)))


def dsa_last_device_status(stream=None) -> int:
    """Synchronise `stream` and return (and clear) the kernels' device status code."""
    return int(load().dsa_last_device_status(_stream(stream)))
