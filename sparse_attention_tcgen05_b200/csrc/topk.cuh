// Top-k selection S_t ("DeepSeek-V3.2" analysis page, sec. 1.1, eq. (2) and the S_t of eq. (4)):
// the min(k, t+1) positions s <= t with the largest scores, ties to the smaller position.
//
// One row per cluster of C CTAs; each CTA takes a contiguous slice of the row (up to 1024 * KPT
// keys), brought into shared memory by bulk copies and turned in place into order-preserving
// 32-bit keys (read from HBM once).  The k-th largest key T is found by radix select on digits
// of 11, 11 and 10 bits:
//   1. every CTA counts its keys by the top digit; the cluster's counts (summed through
//      distributed shared memory, two bins per request) give the digit d1 that holds T.  When
//      the indexer already counted the row's top digits (the fused decode path, `ghist`), that
//      histogram gives d1 directly and this pass and its cluster round are skipped; the row's
//      histogram is cleared again once every CTA of the row has read it, so the buffer is all
//      zeros between calls;
//   2. the candidates - keys whose top digit is d1, usually a few thousand per row - are pushed
//      with their positions into every CTA of the cluster, together with each CTA's count of
//      keys above d1; after one cluster barrier every CTA settles the two lower digits on the
//      candidates alone, with no further cluster traffic;
//   3. if the candidates overflow the buffer (heavy ties), or the row has a single CTA, the two
//      lower digits are settled over the whole slices instead, one cluster round per digit.
// T and the number r of T-ties to keep fix the set exactly.  The selected positions are marked
// in bitmaps; exclusive scans of the per-word counts of (key > T, key == T) give every selected
// position its place in ascending order.
#pragma once

#include <cuda_runtime.h>

#include "ptx.cuh"

namespace dsa {
namespace topk {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxKpt = 32;
constexpr int kMaxSlice = kThreads * kMaxKpt;  // keys per CTA
constexpr int kMaxCluster = 8;
constexpr int kCandBytes = 48 * 1024;  // candidate buffer: 6144 (key, position) pairs
constexpr uint32_t kBulkPiece = 32768;   // bytes per bulk copy of the slice
// Dynamic shared memory: the slice's keys, then the candidate buffer.
template <int KPT>
__host__ __device__ constexpr int stage_bytes() { return kThreads * KPT * 4; }
template <int KPT>
__host__ __device__ constexpr int dyn_smem_bytes() { return stage_bytes<KPT>() + kCandBytes; }

__device__ __forceinline__ uint32_t ld_peer_u32(const uint32_t* local, uint32_t rank) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(map_to_rank(smem_u32(local), rank))
               : "memory");
  return v;
}

__device__ __forceinline__ uint2 ld_peer_v2(const uint32_t* local, uint32_t rank) {
  uint2 v;
  asm volatile("ld.shared::cluster.v2.u32 {%0, %1}, [%2];"
               : "=r"(v.x), "=r"(v.y)
               : "r"(map_to_rank(smem_u32(local), rank))
               : "memory");
  return v;
}

// Add v to a counter in the shared memory of CTA `rank` of the cluster (this CTA included);
// returns the old value.
__device__ __forceinline__ uint32_t atom_add_peer(uint32_t* local, uint32_t rank, uint32_t v) {
  uint32_t old;
  asm volatile("atom.shared::cluster.add.u32 %0, [%1], %2;"
               : "=r"(old)
               : "r"(map_to_rank(smem_u32(local), rank)), "r"(v)
               : "memory");
  return old;
}

__device__ __forceinline__ void st_peer_u32(uint32_t* local, uint32_t rank, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(map_to_rank(smem_u32(local), rank)), "r"(v) : "memory");
}

__device__ __forceinline__ void st_peer_v2(void* local, uint32_t rank, uint32_t a, uint32_t b) {
  asm volatile("st.shared::cluster.v2.u32 [%0], {%1, %2};" ::"r"(map_to_rank(smem_u32(local), rank)), "r"(a),
               "r"(b)
               : "memory");
}

// Digit (of `nbins`, 1024 or 2048) holding the k_rem-th largest counted key, and k_rem within
// that digit.  hist: this CTA's counts; with C > 1 the cluster's counts are summed through
// DSMEM.  Thread t < nbins / 2 owns bins [2t, 2t + 2) (one 8-byte load per CTA); the keys in
// higher bins are a suffix sum over those threads.
template <int C>
__device__ __forceinline__ void select_digit(const uint32_t* hist, int nbins, uint32_t k_rem,
                                             uint32_t* scan, uint32_t* result, uint32_t& digit,
                                             uint32_t& k_out) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nt = nbins / 2;
  uint2 cnt = make_uint2(0u, 0u);
  if (tid < nt) {
#pragma unroll
    for (int r = 0; r < C; ++r) {
      const uint2 w = (C > 1) ? ld_peer_v2(&hist[2 * tid], r) : *reinterpret_cast<const uint2*>(&hist[2 * tid]);
      cnt.x += w.x;
      cnt.y += w.y;
    }
  }
  const uint32_t mine = cnt.x + cnt.y;
  // inclusive suffix sum over the lanes of the warp (lane .. 31)
  uint32_t inc = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t nb = __shfl_down_sync(0xFFFFFFFFu, inc, o);
    if (lane + o < 32) inc += nb;
  }
  if (lane == 0 && warp < nt / 32) scan[warp] = inc;  // the warp's total
  __syncthreads();
  if (warp == 0) {  // keys in the warps above each warp
    const uint32_t v = lane < nt / 32 ? scan[lane] : 0u;
    uint32_t sfx = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t nb = __shfl_down_sync(0xFFFFFFFFu, sfx, o);
      if (lane + o < 32) sfx += nb;
    }
    scan[32 + lane] = sfx - v;
  }
  __syncthreads();
  if (tid < nt) {
    uint32_t above = inc - mine + scan[32 + warp];  // keys in higher warps and higher lanes
    if (above < k_rem && k_rem <= above + cnt.y) {
      result[0] = static_cast<uint32_t>(2 * tid + 1);
      result[1] = k_rem - above;
    }
    above += cnt.y;
    if (above < k_rem && k_rem <= above + cnt.x) {
      result[0] = static_cast<uint32_t>(2 * tid);
      result[1] = k_rem - above;
    }
  }
  __syncthreads();
  digit = result[0];
  k_out = result[1];
}

// Sums of (a, b) over the CTA, returned to every thread; red: 64 words of scratch.
__device__ __forceinline__ uint2 block_sum2(uint32_t a, uint32_t b, uint32_t* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xFFFFFFFFu, a, o);
    b += __shfl_xor_sync(0xFFFFFFFFu, b, o);
  }
  if (lane == 0) {
    red[warp] = a;
    red[32 + warp] = b;
  }
  __syncthreads();
  uint32_t sa = red[lane], sb = red[32 + lane];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sa += __shfl_xor_sync(0xFFFFFFFFu, sa, o);
    sb += __shfl_xor_sync(0xFFFFFFFFu, sb, o);
  }
  __syncthreads();  // red may be reused
  return make_uint2(sa, sb);
}

// Exclusive prefix of (a, b) over the threads of the CTA in thread order; red: 64 words.
__device__ __forceinline__ uint2 block_exclusive2(uint32_t a, uint32_t b, uint32_t* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t ia = a, ib = b;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t na = __shfl_up_sync(0xFFFFFFFFu, ia, o);
    const uint32_t nb = __shfl_up_sync(0xFFFFFFFFu, ib, o);
    if (lane >= o) {
      ia += na;
      ib += nb;
    }
  }
  if (lane == 31) {
    red[warp] = ia;
    red[32 + warp] = ib;
  }
  __syncthreads();
  if (warp == 0) {
    const uint32_t va = red[lane], vb = red[32 + lane];
    uint32_t sa = va, sb = vb;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t na = __shfl_up_sync(0xFFFFFFFFu, sa, o);
      const uint32_t nb = __shfl_up_sync(0xFFFFFFFFu, sb, o);
      if (lane >= o) {
        sa += na;
        sb += nb;
      }
    }
    __syncwarp();
    red[lane] = sa - va;  // exclusive offsets of each warp
    red[32 + lane] = sb - vb;
  }
  __syncthreads();
  const uint2 r = make_uint2(red[warp] + ia - a, red[32 + warp] + ib - b);
  __syncthreads();  // red may be reused
  return r;
}

// The slice's keys live in shared memory in position order, converted in place from the scores.
// Thread t owns the 16-byte chunks g = t + 1024 c (c < KPT / 4): a warp touching one chunk per
// thread reads 512 consecutive bytes.  Selected positions are collected in two bitmaps (key > T,
// key == T) whose word w covers slice positions [32 w, 32 w + 32); chunk g is nibble g % 8 of
// word g / 8.
template <int C, int KPT>
__global__ void __launch_bounds__(kThreads, 1)
    topk_kernel(const float* __restrict__ scores, int32_t* __restrict__ idx, int B, int Lq, int Lk,
                int k, uint32_t* __restrict__ ghist, const int32_t* __restrict__ seq_lens) {
  static_assert(KPT == 4 || KPT == 8 || KPT == 16 || KPT == 32, "keys per thread");
  static_assert(C == 1 || C == 2 || C == 4 || C == kMaxCluster, "cluster size");
  constexpr int kCpr = KPT / 4;  // chunks per thread
  __shared__ __align__(16) uint32_t hist[2][2048];
  __shared__ __align__(16) uint32_t bm[2][kThreads * KPT / 32];
  __shared__ uint32_t scan[72];
  __shared__ uint32_t result[2];
  __shared__ uint32_t red[64];
  __shared__ uint32_t n_cand;                 // candidates pushed into this CTA's buffer
  __shared__ uint32_t above_of[kMaxCluster];  // per CTA of the cluster: its keys above digit d1
  __shared__ uint32_t totals[2];              // (count > T, count == T) of this CTA (fallback)
  __shared__ uint32_t offs[kMaxCluster + 1];  // this CTA's list in each CTA's buffer; its length
  __shared__ __align__(8) uint64_t load_bar;
  __shared__ int abort_flag;
  extern __shared__ __align__(16) uint8_t dyn[];

  pdl_launch_dependents();
  const int row = blockIdx.x / C;
  const uint32_t rank = (C > 1) ? cluster_ctarank() : 0u;
  const int i = row % Lq;
  // decode rows of a paged cache (Lq == 1) see their own context length, clamped to [0, Lk]; the
  // lengths may come from an earlier kernel of the stream, so wait for it first
  if (seq_lens) pdl_wait();
  const int t = seq_lens ? min(max(__ldg(seq_lens + row / Lq), 0), Lk) - 1 : i + Lk - Lq;
  const int n = t + 1;  // candidates s in [0, n)
  int32_t* out = idx + static_cast<size_t>(row) * k;
  const int tid = threadIdx.x;

  if (n <= k) {  // every visible position is selected
    pdl_wait();
    for (int x = rank * kThreads + tid; x < k; x += C * kThreads) out[x] = x < n ? x : -1;
    if (ghist != nullptr && rank == 0)  // leave the row's histogram cleared
      for (int x = tid; x < 2048; x += kThreads) ghist[static_cast<size_t>(row) * 2048 + x] = 0u;
    return;
  }

  // ---- the slice [lo, hi) of the row into shared memory: bulk copies of its 16-byte-aligned
  // part, plain loads for the rest (all of it when the row is not 16-byte aligned)
  const int slice = (((n + C - 1) / C) + 3) & ~3;  // multiple of 4
  const int lo = min(n, static_cast<int>(rank) * slice);
  const int hi = min(n, lo + slice);
  const int cnt = hi - lo;
  const float* base = scores + static_cast<size_t>(row) * Lk + lo;
  uint4* stk = reinterpret_cast<uint4*>(dyn);
  const uint32_t nbulk = ((reinterpret_cast<uintptr_t>(base) & 15u) == 0) ? (static_cast<uint32_t>(cnt) * 4u) & ~15u : 0u;
  if (tid == 0) {
    mbar_init(&load_bar, 1);
    abort_flag = 0;
    n_cand = 0u;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  for (int x = tid; x < 2048; x += kThreads) {
    hist[0][x] = 0u;
    hist[1][x] = 0u;
  }
  __syncthreads();
  // With the indexer's histogram no cluster round precedes the candidate push, so every CTA's
  // n_cand must be zero before any peer reserves room in it: one cluster barrier here, which
  // overlaps the previous kernel's tail.
  const bool pre = ghist != nullptr;
  if (C > 1 && pre) cluster_barrier();
  pdl_wait();  // the scores are written by the previous kernel
  if (tid == 0 && nbulk > 0u) {
    mbar_arrive_expect_tx(&load_bar, nbulk);
    for (uint32_t off = 0; off < nbulk; off += kBulkPiece)
      bulk_load(dyn + off, reinterpret_cast<const uint8_t*>(base) + off, min(kBulkPiece, nbulk - off), &load_bar);
  }
  {
    float* stf = reinterpret_cast<float*>(dyn);
    const int first = static_cast<int>(nbulk / 4u);
    float v[KPT];
#pragma unroll
    for (int it = 0; it < KPT; ++it) {  // every load in flight before the first store
      const int x = first + tid + kThreads * it;
      v[it] = 0.f;
      if (x < cnt) v[it] = __ldg(base + x);
    }
#pragma unroll
    for (int it = 0; it < KPT; ++it) {
      const int x = first + tid + kThreads * it;
      if (x < cnt) stf[x] = v[it];
    }
  }
  if (nbulk > 0u) mbar_wait(&load_bar, 0, &abort_flag, 80);
  __syncthreads();

  // ---- keys in place, and digit 1 (top 11 bits) counted over the cluster
#pragma unroll
  for (int c = 0; c < kCpr; ++c) {
    const int g = tid + kThreads * c;
    const int x = 4 * g;
    const float4 f = reinterpret_cast<const float4*>(dyn)[g];
    const uint4 q = make_uint4(x < cnt ? ordered_key(f.x) : 0u, x + 1 < cnt ? ordered_key(f.y) : 0u,
                               x + 2 < cnt ? ordered_key(f.z) : 0u, x + 3 < cnt ? ordered_key(f.w) : 0u);
    stk[g] = q;
    if (!pre) {
      if (q.x) atomicAdd(&hist[0][q.x >> 21], 1u);
      if (q.y) atomicAdd(&hist[0][q.y >> 21], 1u);
      if (q.z) atomicAdd(&hist[0][q.z >> 21], 1u);
      if (q.w) atomicAdd(&hist[0][q.w >> 21], 1u);
    }
  }
  __syncthreads();
  uint32_t d1, k1;
  if (pre) {  // the whole row's top-digit counts, from the indexer
    select_digit<1>(ghist + static_cast<size_t>(row) * 2048, 2048, static_cast<uint32_t>(k), scan, result, d1, k1);
  } else {
    if (C > 1) cluster_barrier();  // every CTA's counts are complete and its n_cand is zero
    select_digit<C>(hist[0], 2048, static_cast<uint32_t>(k), scan, result, d1, k1);
  }

  // ---- the candidates (keys in digit d1) with their positions, into every CTA's buffer
  uint2* cand = reinterpret_cast<uint2*>(dyn + stage_bytes<KPT>());
  constexpr uint32_t kCap = kCandBytes / sizeof(uint2);
  const uint32_t lo1 = d1 << 21, hi1 = lo1 | 0x1FFFFFu;  // the keys of digit d1 (real keys: d1 >= 3)
  uint32_t mabove = 0u, mcand = 0u;                      // bit 4c + e: key e of chunk c
  uint32_t nc = 0u;     // this thread's candidates
  uint32_t cbase = 0u;  // slot of this thread's first candidate in the own buffer
  if constexpr (C > 1) {  // a single CTA settles digits 2 and 3 over its slice (no cluster round to save)
#pragma unroll
    for (int c = 0; c < kCpr; ++c) {
      const uint4 q = stk[tid + kThreads * c];
      const uint32_t kq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        mabove |= (kq[e] > hi1 ? 1u : 0u) << (4 * c + e);
        mcand |= (kq[e] >= lo1 && kq[e] <= hi1 ? 1u : 0u) << (4 * c + e);
      }
    }
    const uint32_t above = __popc(mabove);
    nc = __popc(mcand);
    {
      // This CTA's list: reserve room in every CTA's buffer, write it into the own buffer, then
      // copy it to the peers.
      const uint2 ex = block_exclusive2(nc, above, red);
      if (tid == kThreads - 1) {
        const uint32_t tot_c = ex.x + nc, tot_a = ex.y + above;
        uint32_t o[C];  // every reservation in flight before the first result is used
#pragma unroll
        for (int r = 0; r < C; ++r) o[r] = (C > 1) ? atom_add_peer(&n_cand, r, tot_c) : atomicAdd(&n_cand, tot_c);
#pragma unroll
        for (int r = 0; r < C; ++r) {
          if (C > 1)
            st_peer_u32(&above_of[rank], r, tot_a);
          else
            above_of[0] = tot_a;
        }
#pragma unroll
        for (int r = 0; r < C; ++r) offs[r] = o[r];
        offs[kMaxCluster] = tot_c;
      }
      __syncthreads();
      cbase = offs[rank] + ex.x;
      uint32_t s = cbase;
      for (uint32_t cm = mcand; cm != 0u;) {  // only the chunks holding candidates
        const int c = (__ffs(cm) - 1) >> 2;
        const uint32_t nib = (cm >> (4 * c)) & 0xFu;
        cm &= ~(0xFu << (4 * c));
        const int g = tid + kThreads * c;
        const uint4 q = stk[g];
        const uint32_t kq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if ((nib >> e) & 1u) {
            if (s < kCap) cand[s] = make_uint2(kq[e], static_cast<uint32_t>(lo + 4 * g + e));
            ++s;
          }
        }
      }
      if (C > 1) {
        __syncthreads();
        const uint32_t tot_c = offs[kMaxCluster], own = offs[rank];
        for (uint32_t x = tid; x < tot_c && own + x < kCap; x += kThreads) {
          const uint2 v = cand[own + x];
#pragma unroll
          for (int r = 0; r < C; ++r)
            if (static_cast<uint32_t>(r) != rank && offs[r] + x < kCap) st_peer_v2(&cand[offs[r] + x], r, v.x, v.y);
        }
      }
    }
  }
  for (int x = tid; x < kThreads * KPT / 32; x += kThreads) {
    bm[0][x] = 0u;
    bm[1][x] = 0u;
  }
  if (C > 1)
    cluster_barrier();  // every candidate and count has landed; nothing remote follows on the fast path
  else
    __syncthreads();
  if (pre && rank == 0)  // every CTA of the row has read the row's histogram: clear it for the next call
    for (int x = tid; x < 2048; x += kThreads) ghist[static_cast<size_t>(row) * 2048 + x] = 0u;

  uint32_t T, r_ties, gt_before, eq_before;
  const uint32_t n_c = n_cand;
  if (C > 1 && n_c <= kCap) {
    // ---- digits 2 and 3 on the candidates, which every CTA holds in full
    for (uint32_t c = tid; c < n_c; c += kThreads) atomicAdd(&hist[1][(cand[c].x >> 10) & 2047u], 1u);
    hist[0][tid] = 0u;  // the peers finished reading it before the barrier above
    for (uint32_t cm = mabove; cm != 0u;) {  // keys above d1 are selected
      const int c = (__ffs(cm) - 1) >> 2;
      const uint32_t nib = (cm >> (4 * c)) & 0xFu;
      cm &= ~(0xFu << (4 * c));
      const int g = tid + kThreads * c;
      atomicOr(&bm[0][g >> 3], nib << (4 * (g & 7)));
    }
    __syncthreads();
    uint32_t d2, k2;
    select_digit<1>(hist[1], 2048, k1, scan, result, d2, k2);
    const uint32_t pre2 = (d1 << 11) | d2;
    for (uint32_t c = tid; c < n_c; c += kThreads)
      if ((cand[c].x >> 10) == pre2) atomicAdd(&hist[0][cand[c].x & 1023u], 1u);
    __syncthreads();
    uint32_t d3;
    select_digit<1>(hist[0], 1024, k2, scan, result, d3, r_ties);
    T = (pre2 << 10) | d3;
    // selected keys of lower-ranked CTAs: all their keys above d1 and their candidates > T;
    // and their T-ties
    uint32_t g = 0, e = 0;
    for (uint32_t c = tid; c < n_c; c += kThreads) {
      const uint2 v = cand[c];
      if (static_cast<int>(v.y) < lo) {
        g += v.x > T ? 1u : 0u;
        e += v.x == T ? 1u : 0u;
      }
    }
    for (uint32_t c = 0; c < nc; ++c) {  // this thread's own candidates
      const uint2 v = cand[cbase + c];
      const uint32_t off = v.y - static_cast<uint32_t>(lo);
      if (v.x > T) atomicOr(&bm[0][off >> 5], 1u << (off & 31u));
      if (v.x == T) atomicOr(&bm[1][off >> 5], 1u << (off & 31u));
    }
    const uint2 be = block_sum2(g, e, red);
    gt_before = be.x;
    eq_before = be.y;
    for (uint32_t r = 0; r < rank; ++r) gt_before += above_of[r];
  } else {
    // ---- too many candidates: digits 2 and 3 over the whole slices, one cluster round each
#pragma unroll
    for (int c = 0; c < kCpr; ++c) {
      const uint4 q = stk[tid + kThreads * c];
      const uint32_t kq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (kq[e] >= lo1 && kq[e] <= hi1) atomicAdd(&hist[1][(kq[e] >> 10) & 2047u], 1u);
    }
    __syncthreads();
    if (C > 1) cluster_barrier();
    uint32_t d2, k2;
    select_digit<C>(hist[1], 2048, k1, scan, result, d2, k2);
    const uint32_t pre2 = (d1 << 11) | d2;
    hist[0][tid] = 0u;  // the peers finished reading it before the candidate barrier
    __syncthreads();
#pragma unroll
    for (int c = 0; c < kCpr; ++c) {
      const uint4 q = stk[tid + kThreads * c];
      const uint32_t kq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (kq[e] && (kq[e] >> 10) == pre2) atomicAdd(&hist[0][kq[e] & 1023u], 1u);
    }
    __syncthreads();
    if (C > 1) cluster_barrier();
    uint32_t d3;
    select_digit<C>(hist[0], 1024, k2, scan, result, d3, r_ties);
    T = (pre2 << 10) | d3;
    uint32_t g = 0, e = 0;
#pragma unroll
    for (int c = 0; c < kCpr; ++c) {
      const int gi = tid + kThreads * c;
      const uint4 q = stk[gi];
      const uint32_t kq[4] = {q.x, q.y, q.z, q.w};
      uint32_t ngt = 0u, neq = 0u;
#pragma unroll
      for (int e2 = 0; e2 < 4; ++e2) {
        ngt |= (kq[e2] > T ? 1u : 0u) << e2;
        neq |= (kq[e2] == T ? 1u : 0u) << e2;
      }
      if (ngt) atomicOr(&bm[0][gi >> 3], ngt << (4 * (gi & 7)));
      if (neq) atomicOr(&bm[1][gi >> 3], neq << (4 * (gi & 7)));
      g += __popc(ngt);
      e += __popc(neq);
    }
    // this CTA's counts, then those of the lower-ranked CTAs through DSMEM
    const uint2 s = block_sum2(g, e, red);
    gt_before = 0u;
    eq_before = 0u;
    if (C > 1) {
      if (tid == 0) {
        totals[0] = s.x;
        totals[1] = s.y;
      }
      cluster_barrier();  // every CTA's totals are written
      for (uint32_t r = 0; r < rank; ++r) {
        gt_before += ld_peer_u32(&totals[0], r);
        eq_before += ld_peer_u32(&totals[1], r);
      }
      cluster_barrier();  // no CTA leaves while a peer may still read its shared memory
    }
  }
  __syncthreads();  // the bitmaps are complete

  // ---- output: thread w writes the selected positions of bitmap word w, in ascending order
  const int nwords = (cnt + 31) / 32;
  const uint32_t wgt = tid < nwords ? bm[0][tid] : 0u, weq = tid < nwords ? bm[1][tid] : 0u;
  const uint32_t g = __popc(wgt), e = __popc(weq);
  const uint2 ex = block_exclusive2(g, e, red);
  const uint32_t eqb = eq_before + ex.y;  // T-ties at smaller positions in the row
  uint32_t pos = gt_before + ex.x + min(eqb, r_ties);
  const uint32_t keep = eqb >= r_ties ? 0u : min(e, r_ties - eqb);
  uint32_t m = wgt, mm = weq;
  for (uint32_t a = 0; a < keep; ++a) {  // the first `keep` ties of this word
    const uint32_t low = mm & (~mm + 1u);
    m |= low;
    mm ^= low;
  }
  const int p0 = lo + 32 * tid;
  while (m != 0u) {
    const int j = __ffs(m) - 1;
    m &= m - 1u;
    if (pos < static_cast<uint32_t>(k)) out[pos++] = p0 + j;
  }
}

}  // namespace topk
}  // namespace dsa
