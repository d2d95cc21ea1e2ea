"""Seeded synthetic inputs for the DSA hot path.

This module only draws random numbers and packs them into the storage types the
path consumes (FP8 e4m3 bytes, fp32, bf16 bits).  It holds no step of the
method's arithmetic; the CPU oracle's tests and the GPU path's tests and bench
both take their inputs from here, so neither side ever produces the other's
inputs.

Workloads (DeepSeek-V3.2 DSA shapes; "Lightning indexer" and "MLA MQA mode"
sections of the V3.2 analysis page):
  tiny_prefill      B=1, L=256 causal, H_I=4, d_I=32, w in {-8..8}/8, k=32,
                    H=8, d_qk=80, d_v=64, scale 1/sqrt(80)
  decode_32k        B=32 queries, each with its own context of 32768,
                    H_I=64, d_I=128, w in {-16..16}/16, k=2048, H=128,
                    d_qk=576, d_v=512, scale 1/sqrt(192)
  decode_128k       decode_32k at a 131072-token context
  prefill_2x8k      B=2, L=8192 causal, dims of decode_32k
  long_prefill_32k  B=1, L=32768 causal, dims of decode_32k
  indexer_kl_16k    B=1, L=16384 causal, dims of decode_32k, plus p and L^I
  dense_warmup_16k  B=1, L=16384 causal, dims of decode_32k: the dense warm-up step
                    (indexer, dense attention with its target p over every s <= t, eq. (3))
q_I and k_I are integers uniform in [-3, 3] stored as e4m3; q and kv are
N(0,1) rounded to bf16.  The stream recipe is in gen.c.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gen.c")
_LIB_PATH = os.path.join(_HERE, "libdsa_inputs.so")

TENSOR_Q_I, TENSOR_K_I, TENSOR_W, TENSOR_Q, TENSOR_KV = 1, 2, 3, 4, 5

# e4m3fn encodings of the integers -3..3 (OCP FP8 E4M3: bias 7, 3 mantissa bits).
_E4M3_OF_INT = {-3: 0xC4, -2: 0xC0, -1: 0xB8, 0: 0x00, 1: 0x38, 2: 0x40, 3: 0x44}
_E4M3_TABLE = np.array([_E4M3_OF_INT[v] for v in range(-3, 4)], dtype=np.uint8)


def build(force: bool = False) -> str:
    """Compile gen.c into libdsa_inputs.so beside it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        u64, i64, i32, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p
        lib.dsa_gen_words.argtypes = [u64, u64, i64, i64, vp]
        lib.dsa_gen_uniform_int.argtypes = [u64, u64, i64, i64, i32, i32, vp]
        lib.dsa_gen_normal_f64.argtypes = [u64, u64, i64, i64, vp]
        lib.dsa_gen_normal_bf16.argtypes = [u64, u64, i64, i64, vp]
        lib.dsa_gen_e4m3_small_int.argtypes = [u64, u64, i64, i64, vp]
        _lib = lib
    return _lib


def words(seed: int, tensor_id: int, n: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    _load().dsa_gen_words(seed, tensor_id, offset, n, out.ctypes.data)
    return out


def uniform_int(seed: int, tensor_id: int, n: int, lo: int, hi: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    _load().dsa_gen_uniform_int(seed, tensor_id, offset, n, lo, hi, out.ctypes.data)
    return out


def normal_f64(seed: int, tensor_id: int, n: int, offset: int = 0) -> np.ndarray:
    assert offset % 2 == 0
    out = np.empty(n, dtype=np.float64)
    _load().dsa_gen_normal_f64(seed, tensor_id, offset, n, out.ctypes.data)
    return out


def normal_bf16_bits(seed: int, tensor_id: int, n: int, offset: int = 0) -> np.ndarray:
    """N(0,1) values rounded fp64 -> fp32 (RNE) -> bf16 (RNE), as uint16 bit patterns."""
    assert offset % 2 == 0
    out = np.empty(n, dtype=np.uint16)
    _load().dsa_gen_normal_bf16(seed, tensor_id, offset, n, out.ctypes.data)
    return out


def e4m3_small_int(seed: int, tensor_id: int, n: int, offset: int = 0) -> np.ndarray:
    """The [-3, 3] integer stream (same draws as uniform_int(..., -3, 3)) as e4m3 bytes."""
    out = np.empty(n, dtype=np.uint8)
    _load().dsa_gen_e4m3_small_int(seed, tensor_id, offset, n, out.ctypes.data)
    return out


def int_to_e4m3(v: np.ndarray) -> np.ndarray:
    """Encode integers in [-3, 3] as e4m3fn bytes (exact)."""
    v = np.asarray(v)
    if v.size and (v.min() < -3 or v.max() > 3):
        raise ValueError("only integers in [-3, 3] are encoded here")
    return _E4M3_TABLE[(v + 3).astype(np.int64)]


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    B: int
    Lq: int
    Lk: int
    H_I: int
    d_I: int
    w_den: int  # w = integer in [-w_den, w_den] / w_den
    k: int
    H: int
    d_qk: int
    d_v: int
    scale: float
    emit_p: bool = False
    dense: bool = False  # the dense warm-up step: no top-k, attention and KL over every s <= t
    notes: str = field(default="", compare=False)

    @property
    def rows(self) -> int:
        return self.B * self.Lq

    def t_of(self, i: int) -> int:
        """Absolute position of query i: it sees keys s <= t."""
        return i + self.Lk - self.Lq


WORKLOADS = {
    "tiny_prefill": Workload("tiny_prefill", 0xD5A0 + 1, 1, 256, 256, 4, 32, 8, 32, 8, 80, 64,
                             1.0 / math.sqrt(80.0)),
    "decode_32k": Workload("decode_32k", 0xD5A0 + 2, 32, 1, 32768, 64, 128, 16, 2048, 128, 576, 512,
                           1.0 / math.sqrt(192.0)),
    "prefill_2x8k": Workload("prefill_2x8k", 0xD5A0 + 3, 2, 8192, 8192, 64, 128, 16, 2048, 128, 576,
                             512, 1.0 / math.sqrt(192.0)),
    "long_prefill_32k": Workload("long_prefill_32k", 0xD5A0 + 4, 1, 32768, 32768, 64, 128, 16, 2048,
                                 128, 576, 512, 1.0 / math.sqrt(192.0)),
    "indexer_kl_16k": Workload("indexer_kl_16k", 0xD5A0 + 5, 1, 16384, 16384, 64, 128, 16, 2048, 128,
                               576, 512, 1.0 / math.sqrt(192.0), emit_p=True),
    "decode_128k": Workload("decode_128k", 0xD5A0 + 6, 32, 1, 131072, 64, 128, 16, 2048, 128, 576, 512,
                            1.0 / math.sqrt(192.0)),
    "dense_warmup_16k": Workload("dense_warmup_16k", 0xD5A0 + 9, 1, 16384, 16384, 64, 128, 16, 16384, 128,
                                 576, 512, 1.0 / math.sqrt(192.0), emit_p=True, dense=True),
    # a 4K-token prefill with the full dims: small enough for counter captures (about 1 GB on
    # the device) while its inputs still exceed the 126 MB L2
    "prefill_1x4k": Workload("prefill_1x4k", 0xD5A0 + 8, 1, 4096, 4096, 64, 128, 16, 2048, 128, 576,
                             512, 1.0 / math.sqrt(192.0)),
}


def custom(name: str, seed: int, B: int, Lq: int, Lk: int, H_I: int, d_I: int, w_den: int, k: int,
           H: int, d_qk: int, d_v: int, scale: float | None = None, emit_p: bool = False,
           dense: bool = False) -> Workload:
    if scale is None:
        scale = 1.0 / math.sqrt(d_qk)
    return Workload(name, seed, B, Lq, Lk, H_I, d_I, w_den, Lk if dense else k, H, d_qk, d_v, scale,
                    emit_p or dense, dense)


# ---- per-tensor draws ------------------------------------------------------------------------
# Each tensor is a flat stream in the row-major layout of the C ABI, so any row range can be
# drawn on its own (used to feed the oracle only the rows it checks).

def q_index(wl: Workload, row0: int = 0, nrows: int | None = None) -> np.ndarray:
    """q_I rows [row0, row0+nrows) of [B*Lq, H_I, d_I], e4m3 bytes."""
    nrows = wl.rows - row0 if nrows is None else nrows
    per = wl.H_I * wl.d_I
    return e4m3_small_int(wl.seed, TENSOR_Q_I, nrows * per, offset=row0 * per).reshape(
        nrows, wl.H_I, wl.d_I)


def k_index(wl: Workload, b: int | None = None) -> np.ndarray:
    """k_I of sequence b ([Lk, d_I]) or of all sequences ([B, Lk, d_I]), e4m3 bytes."""
    per = wl.Lk * wl.d_I
    if b is None:
        return e4m3_small_int(wl.seed, TENSOR_K_I, wl.B * per).reshape(wl.B, wl.Lk, wl.d_I)
    return e4m3_small_int(wl.seed, TENSOR_K_I, per, offset=b * per).reshape(wl.Lk, wl.d_I)


def w_index(wl: Workload, row0: int = 0, nrows: int | None = None) -> np.ndarray:
    """w rows of [B*Lq, H_I] as fp32 multiples of 1/w_den in [-1, 1]."""
    nrows = wl.rows - row0 if nrows is None else nrows
    v = uniform_int(wl.seed, TENSOR_W, nrows * wl.H_I, -wl.w_den, wl.w_den, offset=row0 * wl.H_I)
    return (v.astype(np.float32) / np.float32(wl.w_den)).reshape(nrows, wl.H_I)


def q_attn(wl: Workload, row0: int = 0, nrows: int | None = None) -> np.ndarray:
    """q rows of [B*Lq, H, d_qk] as bf16 bit patterns (uint16)."""
    nrows = wl.rows - row0 if nrows is None else nrows
    per = wl.H * wl.d_qk
    return normal_bf16_bits(wl.seed, TENSOR_Q, nrows * per, offset=row0 * per).reshape(
        nrows, wl.H, wl.d_qk)


def kv_latent(wl: Workload, b: int | None = None) -> np.ndarray:
    """Latent cache c of sequence b ([Lk, d_qk]) or all ([B, Lk, d_qk]) as bf16 bits."""
    per = wl.Lk * wl.d_qk
    if b is None:
        return normal_bf16_bits(wl.seed, TENSOR_KV, wl.B * per).reshape(wl.B, wl.Lk, wl.d_qk)
    return normal_bf16_bits(wl.seed, TENSOR_KV, per, offset=b * per).reshape(wl.Lk, wl.d_qk)


def sample_rows(wl: Workload, n_random: int = 512) -> list[int]:
    """Query rows (flat b*Lq+i) checked at full size: the edges of the selection regime
    (t in {0, 1, k-2, k-1, k, L-1} for every sequence) plus seeded uniform rows."""
    rows = set()
    for b in range(wl.B):
        for t in (0, 1, wl.k - 2, wl.k - 1, wl.k, wl.Lk - 1):
            i = t - (wl.Lk - wl.Lq)
            if 0 <= i < wl.Lq:
                rows.add(b * wl.Lq + i)
    if n_random > 0:
        r = uniform_int(wl.seed, 99, n_random, 0, wl.rows - 1)
        rows.update(int(x) for x in r)
    return sorted(rows)
