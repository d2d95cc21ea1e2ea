// Lightning indexer ("DeepSeek-V3.2" analysis page, sec. 1.1, eq. (1)) on sm_100a:
//   I[t,s] = sum_j w[t,j] * ReLU(q_I[t,j] . k_I[s])   (s <= t),   -inf for s > t.
//
// One FP8 tcgen05 GEMM per tile: keys along M (128 TMEM lanes), (query, head) pairs along N
// (G queries x H_I heads), K = d_I.  A thread of the epilogue owns one key row of the fp32
// accumulator, so the ReLU, the w-weighted head sum and the causal mask are applied in
// registers without any cross-lane reduction; only the [Lq, Lk] scores reach HBM.
//
// Persistent, warp-specialised CTA (one per SM):
//   warp 0        TMA producer: the q_I group once per work item, then k_I tiles (12 stages
//                 for decode, 6 otherwise).  Decode loads each 128-key tile as two boxes of 64
//                 keys (so that a paged cache can place them in different pages) and marks k_I
//                 evict-first in L2: it is read once, and the scores written meanwhile should stay
//                 there for the top-k.
//   warp 1        MMA issuer (one thread): d_I/32 MMAs of 128 x N x 32 per tile
//   warp 2        TMEM allocator (2 accumulators of N columns, double-buffered)
//   warps 4..     epilogue, 2 or 4 warpgroups: tcgen05.ld -> ReLU * w -> head sum -> mask ->
//                 store; for decode
//                 with a `hist` buffer (the fused indexer -> top-k path) it also counts every
//                 visible score of the row by the top 11 bits of its order-preserving key, the
//                 top-k's first radix digit (shared-memory counts per work item, added to the
//                 row's global histogram at the item's end).
// Work item = (sequence, group of G queries, chunk of key tiles); key tiles beyond the
// group's last visible position skip the MMA and are written as -inf directly.
#pragma once

#include <cuda_runtime.h>

#include "ptx.cuh"

namespace dsa {
namespace indexer {

constexpr int kTileKeys = 128;

struct Params {
  const float* w;
  float* scores;
  uint32_t* hist;    // nullable, decode only: [B * Lq][2048] counts of the scores' top digit
  // Paged decode cache (nullable block_table): key s of sequence b is row
  // block_table[b * max_pages + s / page_size] * page_size + s % page_size of k, and the query
  // sits at t = seq_lens[b] - 1 (clamped to [-1, Lk - 1]; Lk is then the longest context).
  const int32_t* block_table;
  const int32_t* seq_lens;
  int page_size, max_pages, num_pages;  // page_size: a multiple of 64
  int k_rows;                           // rows of the k tensor (one past it reads as zeros)
  int B, Lq, Lk;
  int n_qg;   // query groups per sequence
  int n_kt;   // key tiles per sequence
  int kc;     // key tiles per work chunk
  int n_kc;   // chunks per query group
  int n_items;
};

template <int H_I, int D_I, int G>
struct Cfg {
  // k_I ring depth: decode streams k_I from HBM with little else per tile, so it keeps twice
  // as many tiles in flight
  static constexpr int kStages = (G == 1) ? 12 : 6;
  static constexpr int kKBox = (G == 1) ? 64 : kTileKeys;  // keys per k_I TMA box
  static constexpr int N = G * H_I;                      // MMA N (columns per accumulator)
  static constexpr int kQBytes = N * D_I;                // q_I group tile
  static constexpr int kKBytes = kTileKeys * D_I;        // k_I tile
  static constexpr int kTmemCols = (2 * N <= 32) ? 32 : (2 * N <= 64) ? 64 : (2 * N <= 128) ? 128
                                   : (2 * N <= 256) ? 256 : 512;
  // Epilogue warpgroups: four for prefill with at least 32 heads (the ReLU-weighted head sum is
  // the kernel's ALU load, spread over 16 warps), two otherwise.
  static constexpr int kEpiGroups = (G >= 4 && H_I >= 32) ? 4 : 2;
  static constexpr int kEpiThreads = kEpiGroups * 128;
  static constexpr int kThreads = 128 + kEpiThreads;
  static constexpr bool kSplitWG = (G >= 2);             // the epilogue warpgroups split queries
  static constexpr int kColsPerWG = kSplitWG ? N / kEpiGroups : N;
  static constexpr int kQPerWG = kSplitWG ? G / kEpiGroups : 1;
  static constexpr int kEpiWorkers = kSplitWG ? kEpiThreads : 128;
  static constexpr uint32_t kSwizzle = D_I == 128 ? kSw128 : D_I == 64 ? kSw64 : kSw32;
  static constexpr uint32_t kIdesc = make_idesc(0, 0, false, false, 128, N);
  // shared memory layout (offsets from a 1024-aligned base)
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + 2 * ((kQBytes + 1023) / 1024) * 1024;
  static constexpr int kOffW = kOffK + kStages * kKBytes;
  static constexpr int kOffHist = kOffW + 2 * N * 4;                 // decode: [2 groups][2048] digit counts
  static constexpr int kOffBar = kOffHist + (G == 1 ? 2 * 2048 * 4 : 0);
  static constexpr int kNumBars = 2 * kStages + 8;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack
  static_assert(N % 16 == 0 && N >= 16 && N <= 256, "MMA N");
  static_assert(kColsPerWG % 32 == 0, "epilogue column split");
  static_assert(D_I % 32 == 0 && D_I <= 128, "d_I");
};

__device__ __forceinline__ void decode_item(const Params& p, int u, int& b, int& qg, int& kc) {
  const int per = p.B * p.n_kc;
  const int qg_rev = u / per;  // later (longer) query groups first
  const int rem = u - qg_rev * per;
  b = rem / p.n_kc;
  kc = rem - b * p.n_kc;
  qg = p.n_qg - 1 - qg_rev;
}

// Position of query i of sequence b: i + Lk - Lq, or seq_lens[b] - 1 for a paged decode cache.
__device__ __forceinline__ int query_pos(const Params& p, int b, int i) {
  if (p.seq_lens == nullptr) return i + p.Lk - p.Lq;
  const int n = __ldg(p.seq_lens + b);
  if (n > p.Lk) record_bad_index();
  return min(max(n, 0), p.Lk) - 1;
}

// Tiles [kt0, kt1) of the item; the first n_comp of them hold visible keys and need the MMA.
template <int G>
__device__ __forceinline__ void item_tiles(const Params& p, int b, int qg, int kc, int& kt0, int& kt1,
                                           int& n_comp) {
  kt0 = kc * p.kc;
  kt1 = min(kt0 + p.kc, p.n_kt);
  const int i_last = min(qg * G + G, p.Lq) - 1;
  const int t_max = query_pos(p, b, i_last);
  const int last_visible_tile = t_max < 0 ? -1 : t_max / kTileKeys;
  n_comp = max(0, min(kt1, last_visible_tile + 1) - kt0);
}

// Row of k holding key s of sequence b (-1: a bad page index, recorded).  In a paged cache the 64
// keys from a multiple of 64 lie in one page.
__device__ __forceinline__ long key_row(const Params& p, int b, int s) {
  if (p.block_table == nullptr) return static_cast<long>(b) * p.Lk + s;
  const int page = __ldg(p.block_table + static_cast<size_t>(b) * p.max_pages + s / p.page_size);
  if (static_cast<unsigned>(page) >= static_cast<unsigned>(p.num_pages)) {
    record_bad_index();
    return -1;
  }
  return static_cast<long>(page) * p.page_size + s % p.page_size;
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

template <int H_I, int D_I, int G>
__global__ void __launch_bounds__(Cfg<H_I, D_I, G>::kThreads, 1)
    indexer_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const Params p) {
  using C = Cfg<H_I, D_I, G>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sK = smem + C::kOffK;
  float* sW = reinterpret_cast<float*>(smem + C::kOffW);
  uint32_t* sHist = reinterpret_cast<uint32_t*>(smem + C::kOffHist);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* k_full = bars;
  uint64_t* k_empty = bars + C::kStages;
  uint64_t* q_full = bars + 2 * C::kStages;
  uint64_t* q_empty = q_full + 2;
  uint64_t* acc_full = q_full + 4;
  uint64_t* acc_empty = q_full + 6;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], C::kEpiWorkers);
    }
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  pdl_launch_dependents();
  if (warp == 2) tmem_alloc(tmem_slot, C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // first global access below

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    // The whole warp walks the items; lane 0 waits and issues the copies.  Decode: the rows of
    // the next 16 tiles' 64-key boxes are looked up together, one per lane (a paged cache reads
    // its block table: 32 loads in flight instead of one at a time in the issuing thread).
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
    }
    const uint64_t evict_first = l2_evict_first_policy();
    int ks = 0;
    uint32_t kph = 0;
    int qi = 0;
    for (int u = blockIdx.x; u < p.n_items; u += gridDim.x) {
      int b, qg, kc, kt0, kt1, n_comp;
      decode_item(p, u, b, qg, kc);
      item_tiles<G>(p, b, qg, kc, kt0, kt1, n_comp);
      if (n_comp == 0) continue;
      const int qb = qi & 1;
      const uint32_t qph = (qi >> 1) & 1;
      bool got = true;
      if (lane == 0) {
        got = mbar_wait(&q_empty[qb], qph ^ 1, abort_flag, 1);
        if (got) {
          mbar_arrive_expect_tx(&q_full[qb], C::kQBytes);
          tma_load_2d(sQ + qb * ((C::kQBytes + 1023) / 1024) * 1024, &tm_q, &q_full[qb], 0,
                      (b * p.Lq + qg * G) * H_I);
        }
      }
      if (!__all_sync(0xFFFFFFFFu, got)) goto done;
      const int t_row = (G == 1) ? query_pos(p, b, qg) : 0;  // decode: the query's position
      long my_row = -1;                                      // decode: box `lane` of the window
      for (int tt = 0; tt < n_comp; ++tt) {
        if constexpr (G == 1) {
          if ((tt & 15) == 0) {
            // a box past the query (or the sequence) is read as zeros from one row past the
            // tensor, never through the page table
            const int s0 = (kt0 + tt + (lane >> 1)) * kTileKeys + (lane & 1) * C::kKBox;
            my_row = (tt + (lane >> 1) < n_comp && s0 <= t_row) ? key_row(p, b, s0) : -1;
          }
        }
        const long y0 = __shfl_sync(0xFFFFFFFFu, my_row, 2 * (tt & 15));
        const long y1 = __shfl_sync(0xFFFFFFFFu, my_row, 2 * (tt & 15) + 1);
        if (lane == 0) {
          got = mbar_wait(&k_empty[ks], kph ^ 1, abort_flag, 2);
          if (got) {
            mbar_arrive_expect_tx(&k_full[ks], C::kKBytes);
            if constexpr (G == 1) {
              tma_load_2d_hint(sK + ks * C::kKBytes, &tm_k, &k_full[ks], 0,
                               y0 >= 0 ? static_cast<int32_t>(y0) : p.k_rows, evict_first);
              tma_load_2d_hint(sK + ks * C::kKBytes + C::kKBox * D_I, &tm_k, &k_full[ks], 0,
                               y1 >= 0 ? static_cast<int32_t>(y1) : p.k_rows, evict_first);
            } else {
              tma_load_2d(sK + ks * C::kKBytes, &tm_k, &k_full[ks], 0, b * p.Lk + (kt0 + tt) * kTileKeys);
            }
          }
        }
        if (!__all_sync(0xFFFFFFFFu, got)) goto done;
        if (++ks == C::kStages) {
          ks = 0;
          kph ^= 1;
        }
      }
      ++qi;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int ks = 0;
      uint32_t kph = 0;
      int ab = 0;
      uint32_t aph = 0;
      int qi = 0;
      for (int u = blockIdx.x; u < p.n_items; u += gridDim.x) {
        int b, qg, kc, kt0, kt1, n_comp;
        decode_item(p, u, b, qg, kc);
        item_tiles<G>(p, b, qg, kc, kt0, kt1, n_comp);
        if (n_comp == 0) continue;
        const int qb = qi & 1;
        const uint32_t qph = (qi >> 1) & 1;
        if (!mbar_wait(&q_full[qb], qph, abort_flag, 3)) goto done;
        const uint32_t q_addr = smem_u32(sQ + qb * ((C::kQBytes + 1023) / 1024) * 1024);
        for (int tt = 0; tt < n_comp; ++tt) {
          if (!mbar_wait(&acc_empty[ab], aph ^ 1, abort_flag, 4)) goto done;
          if (!mbar_wait(&k_full[ks], kph, abort_flag, 5)) goto done;
          tc_fence_after();
          const uint32_t k_addr = smem_u32(sK + ks * C::kKBytes);
          const uint32_t d_tmem = tmem_base + ab * C::N;
#pragma unroll
          for (int kk = 0; kk < D_I / 32; ++kk) {
            const uint64_t adesc = make_smem_desc(k_addr + kk * 32, 16, 8 * D_I, C::kSwizzle);
            const uint64_t bdesc = make_smem_desc(q_addr + kk * 32, 16, 8 * D_I, C::kSwizzle);
            mma_f8f6f4_ss(d_tmem, adesc, bdesc, C::kIdesc, kk > 0 ? 1u : 0u);
          }
          mma_commit(&k_empty[ks]);
          mma_commit(&acc_full[ab]);
          if (++ks == C::kStages) {
            ks = 0;
            kph ^= 1;
          }
          ab ^= 1;
          if (ab == 0) aph ^= 1;
        }
        mma_commit(&q_empty[qb]);
        ++qi;
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ epilogue
    const int e = threadIdx.x - 128;  // 0 .. kEpiThreads - 1
    const int wg = e >> 7;            // epilogue warpgroup
    const int sp = warp & 3;          // TMEM sub-partition this warp may access
    const int row = sp * 32 + lane;   // accumulator row = key within the tile
    // G >= 2: both groups take every tile (half of the queries each).  G == 1: the groups take
    // turns by tile, each owning one of the two accumulator buffers.
    bool ok = true;
    int gt = 0;  // tiles with an MMA seen so far, over all items (both groups count every one)
    int it = 0;
    const bool count = (G == 1) && p.hist != nullptr;
    uint32_t* gHist = sHist + wg * 2048;  // this warpgroup's counts (decode: the groups take turns by tile)
    if (count)
      for (int x = e & 127; x < 2048; x += 128) gHist[x] = 0u;  // ordered by the item's first barrier
    for (int u = blockIdx.x; u < p.n_items; u += gridDim.x, ++it) {
      int b, qg, kc, kt0, kt1, n_comp;
      decode_item(p, u, b, qg, kc);
      item_tiles<G>(p, b, qg, kc, kt0, kt1, n_comp);
      const int i0 = qg * G;
      int t_item = 0;  // decode: the query's position, read once per item
      if constexpr (G == 1) t_item = query_pos(p, b, i0);
      float* wbuf = sW + (it & 1) * C::N;
      for (int x = e; x < C::N; x += C::kEpiThreads) {
        const int i = i0 + x / H_I;
        wbuf[x] = (i < p.Lq) ? p.w[(static_cast<size_t>(b) * p.Lq + i) * H_I + (x % H_I)] : 0.f;
      }
      named_bar_sync(1, C::kEpiThreads);
      const size_t row_base = static_cast<size_t>(b) * p.Lq;
      for (int tt = 0; tt < n_comp; ++tt, ++gt) {
        const int ab = gt & 1;
        const uint32_t aph = (gt >> 1) & 1;
        if (!(C::kSplitWG || ab == wg) || !ok) continue;
        const bool got = mbar_wait(&acc_full[ab], aph, abort_flag, 6);
        if (!__all_sync(0xFFFFFFFFu, got)) {  // tcgen05.ld below is warp-collective
          ok = false;  // keep reaching the named barriers; skip the remaining work
          continue;
        }
        tc_fence_after();
        float acc[C::kQPerWG];
#pragma unroll
        for (int g = 0; g < C::kQPerWG; ++g) acc[g] = 0.f;
        const int col0 = C::kSplitWG ? wg * C::kColsPerWG : 0;
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(sp * 32) << 16) + ab * C::N + col0;
#pragma unroll
        for (int ch = 0; ch < C::kColsPerWG / 32; ++ch) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(taddr + ch * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int col = ch * 32 + c;
            acc[col / H_I] = fmaf(wbuf[col0 + col], fmaxf(__uint_as_float(v[c]), 0.f), acc[col / H_I]);
          }
        }
        tc_fence_before();
        mbar_arrive(&acc_empty[ab]);
        const int s = (kt0 + tt) * kTileKeys + row;
        if (s < p.Lk) {
#pragma unroll
          for (int g = 0; g < C::kQPerWG; ++g) {
            const int i = i0 + wg * C::kQPerWG * (C::kSplitWG ? 1 : 0) + g;
            if (i < p.Lq) {
              const int t = (G == 1) ? t_item : query_pos(p, b, i);
              p.scores[(row_base + i) * p.Lk + s] = (s <= t) ? acc[g] : -INFINITY;
            }
          }
        }
        if constexpr (G == 1) {
          if (count) {
            // the tile's visible scores by top digit (plain shared atomics: aggregating equal
            // digits over the warp first measured slower)
            if (s < p.Lk && s <= t_item) atomicAdd(&gHist[ordered_key(acc[0]) >> 21], 1u);
          }
        }
      }
      if (count) {  // this group's counts of the item into the row's histogram; the next item starts
                    // from zero (the groups flush independently, each behind its own barrier)
        named_bar_sync(2 + wg, 128);
        uint32_t* gh = p.hist + (row_base + i0) * 2048;
        for (int x = e & 127; x < 2048; x += 128) {
          const uint32_t v = gHist[x];
          if (v) {
            atomicAdd(gh + x, v);
            gHist[x] = 0u;
          }
        }
      }
      // fully masked tiles: no MMA, just -inf
      for (int kt = kt0 + n_comp; ok && kt < kt1; ++kt) {
        for (int x = e; x < G * kTileKeys; x += C::kEpiThreads) {
          const int i = i0 + x / kTileKeys;
          const int s = kt * kTileKeys + (x % kTileKeys);
          if (i < p.Lq && s < p.Lk) p.scores[(row_base + i) * p.Lk + s] = -INFINITY;
        }
      }
    }
  }
done:
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

}  // namespace indexer
}  // namespace dsa
