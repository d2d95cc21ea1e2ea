// Gradient of the indexer loss with respect to the indexer's inputs.  The indexer is trained from
// L^I alone, on a detached input ("DSA Continued Pre-Training" page, Stage 2; "DeepSeek-V3.2"
// analysis page, eq. (4) and the detached-input paragraph; eq. (3) for the dense warm-up), and
// top-k selection is piecewise constant, so the selected set is held fixed:
//   g_i       = dL/dI[t, s_i] = Softmax_i(I[t, S_t]) * sum_i p_i - p_i        (s_i = idx_i)
//   dw[t,j]   = sum_i g_i ReLU(a_ji),                a_ji = q_I[t,j] . k_I[s_i]
//   dq[t,j,:] = sum_i g_i w[t,j] [a_ji > 0] k_I[s_i]
//   dk[s,:]  += sum_{t, i : s_i = s} g_i sum_j w[t,j] [a_ji > 0] q_I[t,j]
// with ReLU'(0) = 0.
//
// One CTA of 128 threads per query row (two CTAs per SM), tiles of 128 selected slots; thread i
// owns slot i of a tile, which is TMEM lane i:
//   1. the tile's k_I rows are gathered (cp.async, 128B-swizzled) and also widened to fp16 (every
//      e4m3 value is exact in fp16) in the MN-major layout of the dq product;
//   2. a = K q^T on the tensor cores (kind::f8f6f4, M = 128 slots, N = 64 heads, K = 128);
//   3. each thread forms its slot's row G_j = g w_j [a_j > 0], split into fp16 hi + lo parts
//      (G = hi + lo to about 2^-22), and adds g ReLU(a_j) to its dw partials;
//   4. dq^T += K^T G (M = 128 dims, N = 64 heads, K = 128 slots) accumulates in TMEM over the
//      row's tiles, and the tile's dk rows G q (M = 128 slots, N = 128 dims, K = 64 heads) are
//      computed into TMEM (kind::f16, hi and lo parts);
//   5. each thread adds its slot's dk row to global memory (vector reductions, fp32).
// At the row's end dq^T is read from TMEM (lane = dim) and dw is reduced over the threads.
// Dense mode (eq. (3)'s gradient): no idx, slot j is position j for j <= t, p has Lk columns.
#pragma once

#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace dsa {
namespace bwd {

constexpr int kThreads = 128;
constexpr int kTile = 128;  // selected slots per tile
constexpr int kHI = 64;     // indexer heads
constexpr int kDI = 128;    // indexer dim

struct Params {
  const uint8_t* q;     // q_I [rows][64][128] e4m3
  const uint8_t* kI;    // k_I [B * Lk][128] e4m3
  const float* w;       // [rows][64]
  const float* scores;  // [rows][Lk], the forward indexer's output
  const int32_t* idx;   // [rows][k]; NULL: dense (slot j is position j, k == Lk)
  const float* p;       // [rows][k] target over the slots
  float* dq;            // [rows][64][128]
  float* dw;            // [rows][64]
  float* dk;            // [B * Lk][128], accumulated (cleared by the host first)
  int B, Lq, Lk, k;
};

// shared memory (offsets from a 1024-aligned base); every operand tile is 128B-swizzled
constexpr int kOffQ8 = 0;                      // q_I row, e4m3 K-major: [64 heads][128 B]
constexpr int kOffQ16 = kOffQ8 + 8192;         // q_I row, fp16 MN-major: 2 atoms (dims 0-63, 64-127) x [64 heads][128 B]
constexpr int kOffK8 = kOffQ16 + 16384;        // gathered k_I rows, e4m3 K-major: [128 slots][128 B]
constexpr int kOffK16 = kOffK8 + 16384;        // the same in fp16, MN-major: 2 atoms x [128 slots][128 B]
constexpr int kOffGhi = kOffK16 + 32768;       // G hi parts, fp16: [128 slots][64 heads]
constexpr int kOffGlo = kOffGhi + 16384;       // G lo parts
constexpr int kOffW = kOffGlo + 16384;         // [64] w of the row
constexpr int kOffRed = kOffW + kHI * 4;       // [4 warps][64] dw partials; [4 warps][4] block reductions
constexpr int kOffBar = kOffRed + 4 * kHI * 4 + 64;
constexpr int kOffMisc = kOffBar + 16;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;
constexpr uint32_t kTmemCols = 256;            // D1 a [0, 64), D2 dq^T [64, 128), D3 dk tile [128, 256)
constexpr uint32_t kColA = 0, kColDq = 64, kColDk = 128;
constexpr uint32_t kIdescA = make_idesc(0, 0, false, false, 128, kHI);    // e4m3 x e4m3
constexpr uint32_t kIdescDq = make_idesc(0, 0, true, true, 128, kHI);     // f16: A, B MN-major
constexpr uint32_t kIdescDk = make_idesc(0, 0, false, true, 128, kDI);    // f16: B MN-major
static_assert(2 * kSmemBytes <= 232448, "two CTAs per SM");

// Byte offset of element `e` (0-63, fp16) of row `r` in a 128-byte-row, 128B-swizzled tile.
__device__ __forceinline__ uint32_t sw16(uint32_t r, uint32_t e) {
  return r * 128u + ((((e >> 3) ^ (r & 7u)) & 7u) << 4) + (e & 7u) * 2u;
}

// 16 e4m3 values (one 16-byte chunk) widened to fp16, as two 16-byte chunks.
__device__ __forceinline__ void e4m3x16_to_f16(const uint4 v, uint4& lo, uint4& hi) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2_raw a = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w[i] & 0xFFFFu), __NV_E4M3);
    const __half2_raw b = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w[i] >> 16), __NV_E4M3);
    o[2 * i] = static_cast<uint32_t>(a.x) | (static_cast<uint32_t>(a.y) << 16);
    o[2 * i + 1] = static_cast<uint32_t>(b.x) | (static_cast<uint32_t>(b.y) << 16);
  }
  lo = make_uint4(o[0], o[1], o[2], o[3]);
  hi = make_uint4(o[4], o[5], o[6], o[7]);
}

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

// Sum of v over the CTA's 128 threads (red: 4 + 4 words), returned to every thread.
__device__ __forceinline__ float cta_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  const float r = red[0] + red[1] + red[2] + red[3];
  __syncthreads();
  return r;
}
__device__ __forceinline__ float cta_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  const float r = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kThreads, 2) indexer_bwd_kernel(const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ8 = smem + kOffQ8;
  uint8_t* sQ16 = smem + kOffQ16;
  uint8_t* sK8 = smem + kOffK8;
  uint8_t* sK16 = smem + kOffK16;
  uint8_t* sGhi = smem + kOffGhi;
  uint8_t* sGlo = smem + kOffGlo;
  float* sW = reinterpret_cast<float*>(smem + kOffW);
  float* sRed = reinterpret_cast<float*>(smem + kOffRed);
  float* sRed2 = sRed + 4 * kHI;
  uint64_t* bar_mma = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    mbar_init(bar_mma, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  pdl_launch_dependents();
  if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tl = tmem + (static_cast<uint32_t>(warp * 32) << 16);  // this warp's TMEM lanes
  pdl_wait();

  const bool dense = p.idx == nullptr;
  const int rows = p.B * p.Lq;
  uint32_t mph = 0;  // phase of bar_mma
  bool ok = true;
  // Every thread waits for the MMAs just committed; the CTA then agrees on the outcome (so that
  // every thread leaves the loops together and no barrier is left waiting).
  auto mma_done = [&]() {
    const bool got = !ok || mbar_wait(bar_mma, mph, abort_flag, 100);
    mph ^= 1;
    ok = __syncthreads_and(ok && got) != 0;
    tc_fence_after();
  };

  for (int r = blockIdx.x; r < rows && ok; r += gridDim.x) {
    const int row = dense ? rows - 1 - r : r;  // dense rows: the longest first
    const int b = row / p.Lq;
    const int t = row % p.Lq + p.Lk - p.Lq;
    const int n_slots = dense ? min(p.k, t + 1) : p.k;
    const int32_t* idx_row = dense ? nullptr : p.idx + static_cast<size_t>(row) * p.k;
    const float* p_row = p.p + static_cast<size_t>(row) * p.k;
    const float* s_row = p.scores + static_cast<size_t>(row) * p.Lk;
    auto pos = [&](int slot) {  // latent position of a slot, -1 if empty
      if (slot >= n_slots) return -1;
      const int s = dense ? slot : __ldg(idx_row + slot);
      if (s >= p.Lk) record_bad_index();
      return (static_cast<unsigned>(s) < static_cast<unsigned>(p.Lk)) ? s : -1;
    };

    // ---- the row's q_I (e4m3 and fp16) and w; the softmax normaliser of its selected scores
    {
      const uint8_t* qg = p.q + static_cast<size_t>(row) * kHI * kDI;
      for (int c = tid; c < kHI * 8; c += kThreads) {  // 64 heads x 8 chunks of 16 bytes
        const int j = c >> 3, ch = c & 7;
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(qg + j * kDI + ch * 16));
        *reinterpret_cast<uint4*>(sQ8 + swizzled_offset(j, ch, 128)) = v;
        uint4 lo, hi;
        e4m3x16_to_f16(v, lo, hi);  // dims 16ch .. 16ch+15 of head j
        const int d0 = ch * 16;
        uint8_t* atom = sQ16 + (d0 >> 6) * 8192;
        *reinterpret_cast<uint4*>(atom + sw16(j, d0 & 63)) = lo;
        *reinterpret_cast<uint4*>(atom + sw16(j, (d0 & 63) + 8)) = hi;
      }
      if (tid < kHI) sW[tid] = __ldg(p.w + static_cast<size_t>(row) * kHI + tid);
    }
    float m = -INFINITY, ptot = 0.f;
    for (int slot = tid; slot < n_slots; slot += kThreads) {
      const int s = pos(slot);
      if (s >= 0) {
        m = fmaxf(m, __ldg(s_row + s));
        ptot += __ldg(p_row + slot);
      }
    }
    m = cta_max(m, sRed2);
    ptot = cta_sum(ptot, sRed2);
    float z = 0.f;
    for (int slot = tid; slot < n_slots; slot += kThreads) {
      const int s = pos(slot);
      if (s >= 0) z += expf(__ldg(s_row + s) - m);
    }
    z = cta_sum(z, sRed2);
    const float lse = m + logf(z);  // only used when the row has a valid slot
    fence_proxy_async_smem();

    float dwacc[kHI];
#pragma unroll
    for (int j = 0; j < kHI; ++j) dwacc[j] = 0.f;
    const int n_tiles = (n_slots + kTile - 1) / kTile;
    for (int n = 0; n < n_tiles && ok; ++n) {
      // ---- 1. gather this thread's slot (one k_I row of 128 bytes) and widen it to fp16
      const int slot = n * kTile + tid;
      const int s = pos(slot);
      const float g = s >= 0 ? expf(__ldg(s_row + s) - lse) * ptot - __ldg(p_row + slot) : 0.f;
      const uint8_t* src = p.kI + (static_cast<size_t>(b) * p.Lk + (s >= 0 ? s : 0)) * kDI;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) cp_async_16(smem_u32(sK8 + swizzled_offset(tid, ch, 128)), src + ch * 16, s >= 0);
      cp_async_commit();
      cp_async_wait_group<0>();
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        const uint4 v = *reinterpret_cast<const uint4*>(sK8 + swizzled_offset(tid, ch, 128));
        uint4 lo, hi;
        e4m3x16_to_f16(v, lo, hi);
        const int d0 = ch * 16;
        uint8_t* atom = sK16 + (d0 >> 6) * 16384;
        *reinterpret_cast<uint4*>(atom + sw16(tid, d0 & 63)) = lo;
        *reinterpret_cast<uint4*>(atom + sw16(tid, (d0 & 63) + 8)) = hi;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      // ---- 2. a = K q^T
      if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kDI / 32; ++kk)
          mma_f8f6f4_ss(tmem + kColA, make_smem_desc(smem_u32(sK8) + kk * 32, 16, 1024, kSw128),
                        make_smem_desc(smem_u32(sQ8) + kk * 32, 16, 1024, kSw128), kIdescA, kk > 0 ? 1u : 0u);
        mma_commit(bar_mma);
      }
      mma_done();
      if (!ok) break;
      // ---- 3. this slot's G row (hi, lo) and dw partials
      {
        uint32_t a[kHI];
        tmem_ld_32x32b_x32(tl + kColA, *reinterpret_cast<uint32_t(*)[32]>(&a[0]));
        tmem_ld_32x32b_x32(tl + kColA + 32, *reinterpret_cast<uint32_t(*)[32]>(&a[32]));
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < kHI / 8; ++c) {
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            float gh[2], gl[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int j = c * 8 + e + u;
              const float x = __uint_as_float(a[j]);
              dwacc[j] = fmaf(g, fmaxf(x, 0.f), dwacc[j]);
              const float G = x > 0.f ? g * sW[j] : 0.f;
              const __half h = __float2half_rn(G);
              gh[u] = __half2float(h);
              gl[u] = G - gh[u];
            }
            const __half2 h2 = __floats2half2_rn(gh[0], gh[1]);
            const __half2 l2 = __floats2half2_rn(gl[0], gl[1]);
            hw[e / 2] = *reinterpret_cast<const uint32_t*>(&h2);
            lw[e / 2] = *reinterpret_cast<const uint32_t*>(&l2);
          }
          *reinterpret_cast<uint4*>(sGhi + sw16(tid, c * 8)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4*>(sGlo + sw16(tid, c * 8)) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      // ---- 4. dq^T += K^T G;  dk tile = G q
      if (tid == 0) {
        tc_fence_after();
        const uint32_t k16 = smem_u32(sK16), q16 = smem_u32(sQ16);
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const uint32_t gb = smem_u32(part == 0 ? sGhi : sGlo);
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            mma_f16_ss(tmem + kColDq, make_smem_desc(k16 + kk * 2048, 16384, 1024, kSw128),
                       make_smem_desc(gb + kk * 2048, 16384, 1024, kSw128), kIdescDq,
                       (n > 0 || part > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < kHI / 16; ++kk)
            mma_f16_ss(tmem + kColDk, make_smem_desc(gb + kk * 32, 16, 1024, kSw128),
                       make_smem_desc(q16 + kk * 2048, 8192, 1024, kSw128), kIdescDk,
                       (part > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar_mma);
      }
      mma_done();
      if (!ok) break;
      // ---- 5. this slot's dk row into global memory
#pragma unroll 1
      for (int c0 = 0; c0 < kDI; c0 += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tl + kColDk + c0, v);
        tmem_ld_wait();
        if (s >= 0) {
          float* dst = p.dk + (static_cast<size_t>(b) * p.Lk + s) * kDI + c0;
#pragma unroll
          for (int c = 0; c < 32; c += 4)
            red_add_v4(dst + c, __uint_as_float(v[c]), __uint_as_float(v[c + 1]), __uint_as_float(v[c + 2]),
                       __uint_as_float(v[c + 3]));
        }
      }
      tc_fence_before();
      __syncthreads();  // the next tile rewrites the operand tiles and D1/D3
    }
    if (!ok) break;

    // ---- row end: dq (lane = dim, column = head) and dw
    {
      float* dq_row = p.dq + static_cast<size_t>(row) * kHI * kDI;
#pragma unroll 1
      for (int c0 = 0; c0 < kHI; c0 += 32) {
        uint32_t v[32];
        if (n_tiles > 0) {
          tmem_ld_32x32b_x32(tl + kColDq + c0, v);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) v[c] = 0u;
        }
#pragma unroll
        for (int c = 0; c < 32; ++c) dq_row[(c0 + c) * kDI + tid] = __uint_as_float(v[c]);
      }
      // dw: butterfly reduce-scatter over the warp (lane L keeps heads L and 32 + L), then
      // the four warps' partials through shared memory
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float* v = dwacc + half * 32;
#pragma unroll
        for (int off2 = 16; off2 >= 1; off2 >>= 1) {
          const bool upper = (lane & off2) != 0;
#pragma unroll
          for (int i = 0; i < off2; ++i) {
            const float send = upper ? v[i] : v[i + off2];
            const float keep = upper ? v[i + off2] : v[i];
            v[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, off2);
          }
        }
        sRed[warp * kHI + half * 32 + lane] = v[0];
      }
      __syncthreads();
      if (tid < kHI)
        p.dw[static_cast<size_t>(row) * kHI + tid] =
            sRed[tid] + sRed[kHI + tid] + sRed[2 * kHI + tid] + sRed[3 * kHI + tid];
      tc_fence_before();
      __syncthreads();  // sRed, the q tiles and D2 are reused by the next row
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace bwd
}  // namespace dsa
