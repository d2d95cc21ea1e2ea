// Masked MHA for short prefill ("DeepSeek-V3.2-Exp" page, sec. 3, inference costs: short
// prefills run MLA's MHA mode with a mask that keeps each query's top-k set, which simulates DSA;
// the analysis page's MHA/MQA-mode paragraph and Fig. 7).  In MHA mode every head has its own
// decompressed keys (d_qk = 192: 128 + 64 rope dims) and values (d_v = 128); query t of head h
// attends to the positions s <= t that its top-k set S_t holds.
//
// One CTA per (sequence, head, tile of 128 queries); key tiles of 128 from 0 to the diagonal:
//   TMA warp     the query tile once, then key and value tiles (two stages); q, k, v are read as
//                2-D maps [B * L rows, H * d cols] whose boxes are one head's 64-dim slices
//   MMA thread   S = Q K^T (M = 128 queries, N = 128 keys, K = 192) into one of two TMEM
//                buffers; O += P V (K = 128 keys, N = 128 value dims, P from TMEM)
//   softmax      thread = query row: mask (s <= t and s in S_t, from a selection bitmap),
//                online softmax with lazy rescaling (the reference max moves only when a
//                tile exceeds it by 2^8), P -> bf16 -> TMEM; at the end O / l -> bf16 and lse
// TMEM: S 2 x 128 [0, 256), O 128 [256, 384), P 2 x 64 [384, 512).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace dsa {
namespace mmha {

constexpr int kBM = 128, kBN = 128;
constexpr int kDQK = 192, kDV = 128;
constexpr int kThreads = 256;  // warps 0-3 softmax, 4 TMA, 5 MMA + TMEM
constexpr int kBox = kBM * 128;                 // 128 rows x 64 bf16 (128 B, SW128)
constexpr int kQBytes = 3 * kBox;               // 48 KB
constexpr int kKBytes = 3 * kBox;               // 48 KB
constexpr int kVBytes = 2 * kBox;               // 32 KB
constexpr int kStage = kKBytes + kVBytes;
constexpr int kOffQ = 0;
constexpr int kOffKV = kOffQ + kQBytes;         // [2] key tile + value tile
constexpr int kOffBar = kOffKV + 2 * kStage;
constexpr int kOffMisc = kOffBar + 16 * 8;
constexpr int kSmemBytes = kOffMisc + 32 + 1024;
constexpr uint32_t kTmemS = 0, kTmemO = 256, kTmemP = 384;
constexpr uint32_t kIdescS = make_idesc(1, 1, false, false, kBM, kBN);
constexpr uint32_t kIdescO = make_idesc(1, 1, false, true, kBM, kDV);
constexpr float kRescaleLog2 = 8.0f;
static_assert(kSmemBytes <= 232448, "shared memory");

__device__ __forceinline__ uint32_t pack_bf16_pair(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

struct Params {
  const uint32_t* sel;  // [B * L][words] selection bitmap: bit s of row t is set iff s is in S_t
                        // (words: a multiple of 4, so that a key tile's 128 bits load as one uint4)
  __nv_bfloat16* out;   // [B, L, H, 128]
  float* lse;           // [B, L, H] (nullable)
  int B, L, H, words;
  float scale_log2;
};

// Selection bitmap of one row per CTA: bit s of word s / 32 is set iff idx holds s (valid slots).
__global__ void __launch_bounds__(256) build_selection_kernel(const int32_t* __restrict__ idx, int L, int k,
                                                              int words, uint32_t* __restrict__ sel) {
  extern __shared__ uint32_t bits[];
  pdl_launch_dependents();
  for (int x = threadIdx.x; x < words; x += blockDim.x) bits[x] = 0u;
  __syncthreads();
  pdl_wait();
  const size_t row = blockIdx.x;
  for (int j = threadIdx.x; j < k; j += blockDim.x) {
    const int s = __ldg(idx + row * k + j);
    if (static_cast<unsigned>(s) < static_cast<unsigned>(L)) atomicOr(&bits[s >> 5], 1u << (s & 31));
    else if (s >= L) record_bad_index();
  }
  __syncthreads();
  for (int x = threadIdx.x; x < words; x += blockDim.x) sel[row * words + x] = bits[x];
}

__global__ void __launch_bounds__(kThreads, 1)
    masked_mha_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + kOffQ;
  uint8_t* sKV = smem + kOffKV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;   // [2]
  uint64_t* kv_empty = bars + 3;  // [2]
  uint64_t* s_full = bars + 5;    // [2]
  uint64_t* s_empty = bars + 7;   // [2] 128 softmax arrivals
  uint64_t* p_full = bars + 9;    // [2] 128 softmax arrivals
  uint64_t* o_done = bars + 11;   // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // CTA -> (sequence, head, query tile); the last query tiles (the most key tiles) first
  const int n_qt = (p.L + kBM - 1) / kBM;
  const int qt = n_qt - 1 - static_cast<int>(blockIdx.x % n_qt);
  const int h = static_cast<int>((blockIdx.x / n_qt) % p.H);
  const int b = static_cast<int>(blockIdx.x / (static_cast<unsigned>(n_qt) * p.H));
  const int n_kt = qt + 1;  // key tiles up to the diagonal
  const int row0 = b * p.L;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 128);
      mbar_init(&p_full[i], 128);
      mbar_init(&o_done[i], 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  pdl_launch_dependents();
  if (warp == 5) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();

  if (warp == 4) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(q_full, kQBytes);
#pragma unroll
      for (int i = 0; i < 3; ++i) tma_load_2d(sQ + i * kBox, &tm_q, q_full, h * kDQK + 64 * i, row0 + qt * kBM);
      for (int j = 0; j < n_kt; ++j) {
        const int st = j & 1;
        if (!mbar_wait(&kv_empty[st], ((j >> 1) & 1) ^ 1, abort_flag, 110)) break;
        uint8_t* dst = sKV + st * kStage;
        mbar_arrive_expect_tx(&kv_full[st], kStage);
#pragma unroll
        for (int i = 0; i < 3; ++i) tma_load_2d(dst + i * kBox, &tm_k, &kv_full[st], h * kDQK + 64 * i, row0 + j * kBN);
#pragma unroll
        for (int i = 0; i < 2; ++i)
          tma_load_2d(dst + kKBytes + i * kBox, &tm_v, &kv_full[st], h * kDV + 64 * i, row0 + j * kBN);
      }
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      bool ok = mbar_wait(q_full, 0, abort_flag, 111);
      tc_fence_after();
      const uint32_t q_addr = smem_u32(sQ);
      auto issue_s = [&](int j) {
        const int st = j & 1;
        const uint32_t k_addr = smem_u32(sKV + st * kStage);
#pragma unroll
        for (int kk = 0; kk < kDQK / 16; ++kk) {
          const int bx = kk >> 2, kin = kk & 3;
          mma_f16_ss(tmem + kTmemS + st * kBN, make_smem_desc(q_addr + bx * kBox + kin * 32, 16, 1024, kSw128),
                     make_smem_desc(k_addr + bx * kBox + kin * 32, 16, 1024, kSw128), kIdescS, kk > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[st]);
      };
      auto issue_pv = [&](int j) {
        const int st = j & 1;
        const uint32_t v_addr = smem_u32(sKV + st * kStage + kKBytes);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          mma_f16_ts(tmem + kTmemO, tmem + kTmemP + st * (kBN / 2) + 8 * kk,
                     make_smem_desc(v_addr + kk * 16 * 128, kBox, 1024, kSw128), kIdescO, (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&o_done[st]);
        mma_commit(&kv_empty[st]);
      };
      for (int j = 0; ok && j < n_kt; ++j) {
        const int st = j & 1;
        ok = mbar_wait(&kv_full[st], (j >> 1) & 1, abort_flag, 112) &&
             mbar_wait(&s_empty[st], ((j >> 1) & 1) ^ 1, abort_flag, 113);
        if (!ok) break;
        tc_fence_after();
        issue_s(j);
        if (j > 0) {
          ok = mbar_wait(&p_full[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag, 114);
          if (!ok) break;
          tc_fence_after();
          issue_pv(j - 1);
        }
      }
      if (ok && mbar_wait(&p_full[(n_kt - 1) & 1], ((n_kt - 1) >> 1) & 1, abort_flag, 115)) {
        tc_fence_after();
        issue_pv(n_kt - 1);
      }
    }
  } else if (warp < 4) {
    // ---------------------------------------------------------------- softmax / epilogue
    const int r = threadIdx.x;  // query row of the tile = TMEM lane
    const int t = qt * kBM + r;
    const bool row_ok = t < p.L;
    const uint32_t tl = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const uint32_t* sel_row = p.sel + static_cast<size_t>(row0 + min(t, p.L - 1)) * p.words;
    const float sc = p.scale_log2;
    float ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kt; ++j) {
      const int st = j & 1;
      if (ok && !mbar_wait(&s_full[st], (j >> 1) & 1, abort_flag, 116)) ok = false;
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) break;
      tc_fence_after();
      // this row's 128 scores of key tile j, masked: s <= t and s in S_t
      const uint4 m4 = row_ok ? *reinterpret_cast<const uint4*>(sel_row + j * 4) : make_uint4(0u, 0u, 0u, 0u);
      const uint32_t mw[4] = {m4.x, m4.y, m4.z, m4.w};
      float z[kBN];
#pragma unroll
      for (int c0 = 0; c0 < kBN; c0 += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tl + kTmemS + st * kBN + c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int s = j * kBN + c0 + c;
          const bool keep = ((mw[c0 >> 5] >> c) & 1u) && s <= t;
          z[c0 + c] = keep ? __uint_as_float(v[c]) * sc : -INFINITY;
        }
      }
      tc_fence_before();
      mbar_arrive(&s_empty[st]);
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < kBN; ++c) mx = fmaxf(mx, z[c]);
      const float rq = (ref == -INFINITY) ? mx : ((mx > ref + kRescaleLog2) ? mx : ref);
      const bool moved = ref != -INFINITY && rq != ref;
      // O may change only between PV(j - 1) and PV(j); P buffer st was last read by PV(j - 2)
      if (j >= 1 && __any_sync(0xFFFFFFFFu, moved)) {
        const bool got = mbar_wait(&o_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag, 117);
        ok = __all_sync(0xFFFFFFFFu, got);
        if (!ok) break;
        tc_fence_after();
        const float f = moved ? ex2_approx(ref - rq) : 1.f;
#pragma unroll 1
        for (int c0 = 0; c0 < kDV; c0 += 16) {
          uint32_t o[16];
          tmem_ld_32x32b_x16(tl + kTmemO + c0, o);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 16; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * f);
          tmem_st_32x32b_x16(tl + kTmemO + c0, o);
        }
        tmem_st_wait();
      } else if (j >= 2) {
        const bool got = mbar_wait(&o_done[st], ((j - 2) >> 1) & 1, abort_flag, 118);
        ok = __all_sync(0xFFFFFFFFu, got);
        if (!ok) break;
      }
      if (moved) l *= ex2_approx(ref - rq);
      ref = rq;
      const bool live = rq != -INFINITY;
#pragma unroll
      for (int c0 = 0; c0 < kBN; c0 += 32) {
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float p0 = live ? ex2_approx(z[c0 + c] - rq) : 0.f;
          const float p1 = live ? ex2_approx(z[c0 + c + 1] - rq) : 0.f;
          l += p0 + p1;
          pk[c >> 1] = pack_bf16_pair(p0, p1);
        }
        tmem_st_32x32b_x16(tl + kTmemP + st * (kBN / 2) + (c0 >> 1), pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[st]);
    }
    // epilogue: O / l -> bf16, lse
    if (ok) {
      const int jl = n_kt - 1;
      const bool got = mbar_wait(&o_done[jl & 1], (jl >> 1) & 1, abort_flag, 119);
      ok = __all_sync(0xFFFFFFFFu, got);
    }
    if (ok) {
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* orow = p.out + ((static_cast<size_t>(row0) + t) * p.H + h) * kDV;
#pragma unroll 1
      for (int c0 = 0; c0 < kDV; c0 += 16) {
        uint32_t o[16];
        tmem_ld_32x32b_x16(tl + kTmemO + c0, o);
        tmem_ld_wait();
        if (row_ok) {
          uint32_t w[8];
#pragma unroll
          for (int c = 0; c < 16; c += 2)
            w[c >> 1] = pack_bf16_pair(__uint_as_float(o[c]) * inv_l, __uint_as_float(o[c + 1]) * inv_l);
          *reinterpret_cast<uint4*>(orow + c0) = make_uint4(w[0], w[1], w[2], w[3]);
          *reinterpret_cast<uint4*>(orow + c0 + 8) = make_uint4(w[4], w[5], w[6], w[7]);
        }
      }
      if (row_ok && p.lse)
        p.lse[(static_cast<size_t>(row0) + t) * p.H + h] = l > 0.f ? (ref + log2f(l)) * 0.6931471805599453f : -INFINITY;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace mmha
}  // namespace dsa
