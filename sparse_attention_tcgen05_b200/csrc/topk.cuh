// Top-k selection S_t ("DeepSeek-V3.2" analysis page, sec. 1.1, eq. (2) and the S_t of eq. (4)):
// the min(k, t+1) positions s <= t with the largest scores, ties to the smaller position.
//
// One row per cluster of C CTAs; each CTA takes a contiguous slice of the row and each of its
// 1024 threads a contiguous run of KPT keys, held in registers as order-preserving 32-bit keys
// (read from HBM once).  Radix select in three digit passes (11, 11, 10 bits): shared-memory
// histograms (summed over the cluster through distributed shared memory when C > 1) give the
// digit holding the k-th largest key; later passes only count keys that still match the
// chosen prefix.  The threshold key T and the number r of T-ties to keep fix the set exactly.
// Because every thread owns a contiguous run, one exclusive scan of the per-thread counts of
// (key > T, key == T) gives every selected position's place in ascending order.
#pragma once

#include <cuda_runtime.h>

#include "ptx.cuh"

namespace dsa {
namespace topk {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxKpt = 32;
constexpr int kMaxSlice = kThreads * kMaxKpt;  // keys per CTA

// Every finite or infinite score maps to a key >= 0x007FFFFF; 0 marks an empty register slot
// and can never be selected (at least k real keys exist whenever a row is selected).
__device__ __forceinline__ uint32_t ordered_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;  // -0 ties with +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint32_t ld_peer_u32(const uint32_t* local, uint32_t rank) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(map_to_rank(smem_u32(local), rank))
               : "memory");
  return v;
}

// Digit (of `nbins`) holding the k_rem-th largest counted key, and k_rem within that digit.
// hist: this CTA's counts; with C > 1 the cluster's counts are summed through DSMEM.
template <int C>
__device__ __forceinline__ void select_digit(const uint32_t* hist, int nbins, uint32_t k_rem,
                                             uint32_t* scan, uint32_t* result, uint32_t& digit,
                                             uint32_t& k_out) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = nbins / kThreads;  // bins per thread (1 or 2), taken in descending order
  uint32_t cnt[2] = {0, 0};
  uint32_t mine = 0;
  for (int i = 0; i < per; ++i) {
    const int d = nbins - 1 - (tid * per + i);
    uint32_t c = 0;
    if (C > 1) {
      for (int r = 0; r < C; ++r) c += ld_peer_u32(&hist[d], r);
    } else {
      c = hist[d];
    }
    cnt[i] = c;
    mine += c;
  }
  // exclusive scan of `mine` over threads (descending digits)
  uint32_t inc = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t nb = __shfl_up_sync(0xFFFFFFFFu, inc, o);
    if (lane >= o) inc += nb;
  }
  if (lane == 31) scan[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const uint32_t v = scan[lane];
    uint32_t wi = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t nb = __shfl_up_sync(0xFFFFFFFFu, wi, o);
      if (lane >= o) wi += nb;
    }
    scan[32 + lane] = wi - v;
  }
  __syncthreads();
  uint32_t above = scan[32 + warp] + inc - mine;  // keys in digits larger than this thread's
  for (int i = 0; i < per; ++i) {
    if (above < k_rem && k_rem <= above + cnt[i]) {
      result[0] = nbins - 1 - (tid * per + i);
      result[1] = k_rem - above;
    }
    above += cnt[i];
  }
  __syncthreads();
  digit = result[0];
  k_out = result[1];
}

template <int C, int KPT>
__global__ void __launch_bounds__(kThreads, 1)
    topk_kernel(const float* __restrict__ scores, int32_t* __restrict__ idx, int B, int Lq, int Lk,
                int k) {
  __shared__ uint32_t hist[2][2048];
  __shared__ uint32_t scan[72];
  __shared__ uint32_t result[2];
  __shared__ uint32_t totals[2];  // this CTA's (count > T, count == T), read by later ranks

  pdl_launch_dependents();
  pdl_wait();
  const int row = blockIdx.x / C;
  const uint32_t rank = (C > 1) ? cluster_ctarank() : 0u;
  const int i = row % Lq;
  const int t = i + Lk - Lq;
  const int n = t + 1;  // candidates s in [0, n)
  int32_t* out = idx + static_cast<size_t>(row) * k;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  if (n <= k) {  // every visible position is selected
    for (int x = rank * kThreads + tid; x < k; x += C * kThreads) out[x] = x < n ? x : -1;
    return;
  }

  // ---- this thread's keys: positions [p0, p0 + KPT) of the row, clipped to the slice
  const int slice = (((n + C - 1) / C) + 3) & ~3;  // multiple of 4: aligned vector loads
  const int lo = min(n, static_cast<int>(rank) * slice);
  const int hi = min(n, lo + slice);
  const int p0 = lo + tid * KPT;
  const float* src = scores + static_cast<size_t>(row) * Lk;
  uint32_t key[KPT];
  const bool vec = ((reinterpret_cast<uintptr_t>(src + p0) & 15u) == 0) && (p0 + KPT <= hi);
  if (vec) {
#pragma unroll
    for (int j = 0; j < KPT; j += 4) {
      const float4 f = __ldg(reinterpret_cast<const float4*>(src + p0 + j));
      key[j] = ordered_key(f.x);
      key[j + 1] = ordered_key(f.y);
      key[j + 2] = ordered_key(f.z);
      key[j + 3] = ordered_key(f.w);
    }
  } else {
#pragma unroll
    for (int j = 0; j < KPT; ++j) key[j] = (p0 + j < hi) ? ordered_key(__ldg(src + p0 + j)) : 0u;
  }

  // ---- pass 1: top 11 bits
  for (int x = tid; x < 2048; x += kThreads) {
    hist[0][x] = 0u;
    hist[1][x] = 0u;
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < KPT; ++j)
    if (key[j]) atomicAdd(&hist[0][key[j] >> 21], 1u);
  __syncthreads();
  if (C > 1) cluster_barrier();
  uint32_t d1, k1;
  select_digit<C>(hist[0], 2048, static_cast<uint32_t>(k), scan, result, d1, k1);

  // ---- pass 2: bits 10..20 of keys whose top 11 bits are d1
#pragma unroll
  for (int j = 0; j < KPT; ++j)
    if (key[j] && (key[j] >> 21) == d1) atomicAdd(&hist[1][(key[j] >> 10) & 2047u], 1u);
  __syncthreads();
  if (C > 1) cluster_barrier();  // also: every CTA has finished reading the others' pass-1 counts
  uint32_t d2, k2;
  select_digit<C>(hist[1], 2048, k1, scan, result, d2, k2);
  const uint32_t pre2 = (d1 << 11) | d2;

  // ---- pass 3: bits 0..9 of keys whose top 22 bits are pre2 (hist[0] is free again)
  for (int x = tid; x < 1024; x += kThreads) hist[0][x] = 0u;
  __syncthreads();
#pragma unroll
  for (int j = 0; j < KPT; ++j)
    if (key[j] && (key[j] >> 10) == pre2) atomicAdd(&hist[0][key[j] & 1023u], 1u);
  __syncthreads();
  if (C > 1) cluster_barrier();
  uint32_t d3, r_ties;
  select_digit<C>(hist[0], 1024, k2, scan, result, d3, r_ties);
  const uint32_t T = (pre2 << 10) | d3;  // the threshold key; r_ties keys equal to it are kept

  // ---- output: one exclusive scan of (count > T, count == T) in position order
  uint32_t gt = 0, eq = 0;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    gt += key[j] > T;
    eq += key[j] == T;
  }
  uint32_t igt = gt, ieq = eq;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t a = __shfl_up_sync(0xFFFFFFFFu, igt, o);
    const uint32_t b2 = __shfl_up_sync(0xFFFFFFFFu, ieq, o);
    if (lane >= o) {
      igt += a;
      ieq += b2;
    }
  }
  if (lane == 31) {
    scan[warp] = igt;
    scan[32 + warp] = ieq;
  }
  __syncthreads();
  if (warp == 0) {
    const uint32_t vg = scan[lane], ve = scan[32 + lane];
    uint32_t wsum_g = vg, wsum_e = ve;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t a = __shfl_up_sync(0xFFFFFFFFu, wsum_g, o);
      const uint32_t b2 = __shfl_up_sync(0xFFFFFFFFu, wsum_e, o);
      if (lane >= o) {
        wsum_g += a;
        wsum_e += b2;
      }
    }
    __syncwarp();
    scan[lane] = wsum_g - vg;  // exclusive offsets of each warp
    scan[32 + lane] = wsum_e - ve;
    if (lane == 31) {
      totals[0] = wsum_g;
      totals[1] = wsum_e;
    }
  }
  __syncthreads();
  uint32_t gt_before = scan[warp] + igt - gt;
  uint32_t eq_before = scan[32 + warp] + ieq - eq;
  if (C > 1) {
    cluster_barrier();  // every CTA's totals are written
    for (uint32_t r = 0; r < rank; ++r) {
      gt_before += ld_peer_u32(&totals[0], r);
      eq_before += ld_peer_u32(&totals[1], r);
    }
    cluster_barrier();  // no CTA leaves while a peer may still read its shared memory
  }
  uint32_t pos = gt_before + min(eq_before, r_ties);
  uint32_t eq_rank = eq_before;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    bool sel = key[j] > T;
    if (key[j] == T) {
      sel = eq_rank < r_ties;
      ++eq_rank;
    }
    if (sel && pos < static_cast<uint32_t>(k)) out[pos++] = p0 + j;
  }
}

}  // namespace topk
}  // namespace dsa
