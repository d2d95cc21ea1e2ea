// Top-k selection S_t ("DeepSeek-V3.2" analysis page, sec. 1.1, eq. (2) and the S_t of eq. (4)):
// the min(k, t+1) positions s <= t with the largest scores, ties to the smaller position.
//
// Radix select over order-preserving 32-bit keys, one row per cluster of C CTAs.  Each CTA
// stages its slice of the row in shared memory once (the only HBM read), then four 8-bit
// digit passes build warp-aggregated shared histograms; with C > 1 the C histograms are
// summed through distributed shared memory.  The threshold key T and the number r of
// threshold ties to keep fix the set exactly; a final ordered pass (ballot + popc prefix
// sums) writes the selected positions in ascending order.
#pragma once

#include <cuda_runtime.h>

#include "ptx.cuh"

namespace dsa {
namespace topk {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxSlice = 32768;  // keys per CTA held in shared memory (128 KiB)

__device__ __forceinline__ uint32_t ordered_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;  // -0 ties with +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

__device__ __forceinline__ uint32_t ld_peer_u32(const uint32_t* local, uint32_t rank) {
  uint32_t remote, v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(remote) : "memory");
  return v;
}

// Warp-aggregated histogram increment (all 32 lanes must call; `valid` selects contributors).
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool valid) {
  const uint32_t key = valid ? bin : 0xFFFFFFFFu;
  const uint32_t peers = __match_any_sync(0xFFFFFFFFu, key);
  const int leader = __ffs(peers) - 1;
  if (valid && static_cast<int>(threadIdx.x & 31) == leader) atomicAdd(&hist[bin], __popc(peers));
}

// Block-wide exclusive scan of one value per warp (result for the calling warp) + total.
__device__ __forceinline__ uint32_t warp_offsets(uint32_t warp_total, uint32_t* scratch,
                                                 uint32_t& block_total) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) scratch[warp] = warp_total;
  __syncthreads();
  if (warp == 0) {
    uint32_t v = scratch[lane];
    uint32_t inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t n = __shfl_up_sync(0xFFFFFFFFu, inc, o);
      if (lane >= o) inc += n;
    }
    scratch[32 + lane] = inc - v;
    if (lane == 31) scratch[64] = inc;
  }
  __syncthreads();
  const uint32_t off = scratch[32 + warp];
  block_total = scratch[64];
  __syncthreads();
  return off;
}

template <int C>
__global__ void __launch_bounds__(kThreads, 1)
    topk_kernel(const float* __restrict__ scores, int32_t* __restrict__ idx, int B, int Lq, int Lk,
                int k) {
  extern __shared__ uint32_t keys[];  // [slice]
  __shared__ uint32_t hist[2][256];
  __shared__ uint32_t scan[72];
  __shared__ uint32_t sel_state[4];  // [0] digit, [1] k_remaining, [2] count_gt, [3] count_eq
  __shared__ uint32_t counts[2];     // this CTA's (count_gt, count_eq) for the output pass

  const int row = blockIdx.x / C;
  const uint32_t rank = (C > 1) ? cluster_rank() : 0u;
  const int i = row % Lq;
  const int t = i + Lk - Lq;
  const int n = t + 1;  // candidates s in [0, n)
  int32_t* out = idx + static_cast<size_t>(row) * k;
  const int tid = threadIdx.x, lane = tid & 31;

  if (n <= k) {  // every visible position is selected
    for (int x = rank * kThreads + tid; x < k; x += C * kThreads) out[x] = x < n ? x : -1;
    return;
  }

  const int slice = (n + C - 1) / C;
  const int lo = min(n, static_cast<int>(rank) * slice);
  const int hi = min(n, lo + slice);
  const int len = hi - lo;
  const float* src = scores + static_cast<size_t>(row) * Lk + lo;

  // ---- stage the slice as ordered keys; histogram of the top digit on the way
  for (int x = tid; x < 256; x += kThreads) hist[0][x] = 0u;
  __syncthreads();
  const int len_r = (len + kThreads - 1) / kThreads * kThreads;
  for (int x = tid; x < len_r; x += kThreads) {
    uint32_t key = 0;
    const bool v = x < len;
    if (v) {
      key = ordered_key(__ldg(src + x));
      keys[x] = key;
    }
    hist_add(hist[0], key >> 24, v);
  }

  uint32_t prefix = 0, mask = 0;
  uint32_t k_rem = static_cast<uint32_t>(k);
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    uint32_t* h = hist[pass & 1];
    if (pass > 0) {
      for (int x = tid; x < 256; x += kThreads) h[x] = 0u;
      __syncthreads();
      for (int x = tid; x < len_r; x += kThreads) {
        const bool v = x < len && ((keys[x] & mask) == prefix);
        const uint32_t key = x < len ? keys[x] : 0u;
        hist_add(h, (key >> shift) & 0xFFu, v);
      }
    }
    __syncthreads();
    if (C > 1) cluster_sync();
    // Digit holding the k_rem-th largest key among those matching the prefix.  Thread
    // tid < 256 handles digit d = 255 - tid, so an inclusive scan over tid counts the keys
    // whose digit is >= d.  Counts are summed over the cluster through DSMEM.
    uint32_t cd = 0, inc = 0;
    if (tid < 256) {
      const uint32_t d = 255u - tid;
      if (C > 1) {
        for (int r = 0; r < C; ++r) cd += ld_peer_u32(&h[d], r);
      } else {
        cd = h[d];
      }
      inc = cd;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t nb = __shfl_up_sync(0xFFFFFFFFu, inc, o);
        if (lane >= o) inc += nb;
      }
      if (lane == 31) scan[tid >> 5] = inc;
    }
    __syncthreads();
    if (tid < 256) {
      for (int x = 0; x < (tid >> 5); ++x) inc += scan[x];
      const uint32_t above = inc - cd;  // keys with a larger digit
      if (above < k_rem && k_rem <= inc) {
        sel_state[0] = 255u - tid;
        sel_state[1] = k_rem - above;
      }
    }
    __syncthreads();
    const uint32_t d = sel_state[0];
    k_rem = sel_state[1];
    prefix |= d << shift;
    mask |= 0xFFu << shift;
  }
  const uint32_t T = prefix;      // the threshold key
  const uint32_t r_ties = k_rem;  // keys equal to T that are kept (>= 1)

  // ---- counts of keys > T and == T in this slice, shared over the cluster
  uint32_t my_gt = 0, my_eq = 0;
  for (int x = tid; x < len; x += kThreads) {
    const uint32_t key = keys[x];
    my_gt += key > T;
    my_eq += key == T;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    my_gt += __shfl_xor_sync(0xFFFFFFFFu, my_gt, o);
    my_eq += __shfl_xor_sync(0xFFFFFFFFu, my_eq, o);
  }
  if (tid == 0) {
    counts[0] = 0;
    counts[1] = 0;
  }
  __syncthreads();
  if (lane == 0) {
    atomicAdd(&counts[0], my_gt);
    atomicAdd(&counts[1], my_eq);
  }
  __syncthreads();
  uint32_t gt_before = 0, eq_before = 0;
  if (C > 1) {
    cluster_sync();
    for (uint32_t r = 0; r < rank; ++r) {
      gt_before += ld_peer_u32(&counts[0], r);
      eq_before += ld_peer_u32(&counts[1], r);
    }
    cluster_sync();  // no CTA leaves while a peer may still read its counters
  }
  const uint32_t sel_before = gt_before + min(eq_before, r_ties);

  // ---- ordered output pass
  uint32_t run_eq = 0, run_sel = 0;
  for (int base = 0; base < len; base += kThreads) {
    const int x = base + tid;
    const uint32_t key = x < len ? keys[x] : 0u;
    const bool is_gt = x < len && key > T;
    const bool is_eq = x < len && key == T;
    const uint32_t lt = (1u << lane) - 1u;
    const uint32_t b_eq = __ballot_sync(0xFFFFFFFFu, is_eq);
    uint32_t eq_total;
    const uint32_t eq_off = warp_offsets(__popc(b_eq), scan, eq_total);
    const uint32_t eq_rank = eq_before + run_eq + eq_off + __popc(b_eq & lt);
    const bool sel = is_gt || (is_eq && eq_rank < r_ties);
    const uint32_t b_sel = __ballot_sync(0xFFFFFFFFu, sel);
    uint32_t sel_total;
    const uint32_t sel_off = warp_offsets(__popc(b_sel), scan, sel_total);
    const uint32_t pos = sel_before + run_sel + sel_off + __popc(b_sel & lt);
    if (sel && pos < static_cast<uint32_t>(k)) out[pos] = lo + x;
    run_eq += eq_total;
    run_sel += sel_total;
  }
}

}  // namespace topk
}  // namespace dsa
