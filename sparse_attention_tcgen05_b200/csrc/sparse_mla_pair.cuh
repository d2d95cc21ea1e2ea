// Sparse attention in MLA's MQA mode over the top-k selected latents ("DeepSeek-V3.2" analysis
// page, sec. 1.1, eq. (2) and the MQA-mode paragraph; renormalised form eq. (19)), with the
// optional head-summed target p ("DSA Continued Pre-Training", Stage 1/2), for the 576-d
// latent (512 value + 64 rope dims) shared by up to 128 query heads.
//
// A cluster of two CTAs serves one (query row, KV split).  The fp32 accumulator of all 512
// value dims would fill the whole tensor memory, so each CTA owns half of them, and the 576
// key dims are split evenly so that each CTA gathers only its 288 dims of every entry:
//   rank 0: value dims [0, 256)   + rope dims [512, 544)
//   rank 1: value dims [256, 512) + rope dims [544, 576)
// Each CTA computes a partial S over its dims on the tensor cores, stages the 128 x 32 fp32
// partial in shared memory and ships it to its peer with one bulk copy (counted on the peer's
// mbarrier); both then hold the same full S (fp32 addition commutes), take the same softmax
// decisions and accumulate O for their own 256 value dims.
//
// Tensor memory (512 columns): O [0, 256) fp32, S 2 x 32 fp32 [256, 320), and this CTA's
// slice of Q, 128 heads x 288 bf16, as the A operand of S = Q K^T [320, 464).  Keeping Q in
// tensor memory means a 32-wide S block only streams its 18 KB gathered tile from shared
// memory, and frees shared memory for an 8-deep gather ring.
//
// Pipeline (per CTA, blocks of 32 selected entries; a p sweep revisits every block):
//   gather warps   TMA tile::gather4: 4 selected rows per instruction, landing in the
//                  swizzled K-major tiles the MMA reads (6 stages, 40 instructions a block).
//                  A single issuing warp caps the gather near 9 GB/s per SM, so six warps
//                  take turns by block (warp w always refills stage w).
//   MMA thread     polls: S(j) = Q K_j^T as soon as block j and an S buffer are free;
//                  O += P(i) V_i as soon as P(i) is written (never waits behind a late gather)
//   softmax        two warpgroups on the same 128 TMEM lanes (thread = head row), each owning
//                  16 of the block's 32 columns.  Iteration q loads S(q+1) and ships it to the
//                  peer one block ahead, then adds the peer's part of S(q), combines the two
//                  half-row maxima, runs the online softmax with lazy rescaling and writes P(q).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"
#include "sparse_mla.cuh"

namespace dsa {
namespace mla_pair {

using mla::Params;
using mla::pack_bf16x2;
using mla::named_bar_sync;

constexpr int kBN = 32;             // selected entries per block
constexpr int kStages = 6;          // gather ring depth (a multiple of kGatherWarps)
constexpr int kRecvSlots = 4;       // partial-S receive slots (see the exchange argument below)
constexpr int kThreads = 480;       // warps 0-7 softmax, 8 MMA, 9-14 gather
constexpr int kSoftmaxThreads = 256;
constexpr int kHalf = 16;           // S columns per softmax warpgroup
constexpr int kMmaWarp = 8;
constexpr int kGatherWarp0 = 9;
constexpr int kGatherWarps = 6;
constexpr int kDQK = 576, kDV = 512, kDvCta = 256, kRopeCta = 32;
constexpr int kDimsCta = kDvCta + kRopeCta;         // 288 key dims per CTA
constexpr int kMainBox = kBN * 128;                 // 32 entries x 64 dims (SW128)
constexpr int kRopeTile = kBN * 64;                 // 32 entries x 32 dims (SW64)
constexpr int kKvStage = 4 * kMainBox + kRopeTile;  // 18 KB
constexpr int kPBytes = 128 * kBN * 2;
constexpr int kXSlot = 128 * kBN * 4;               // one partial S (fp32, 16 KB)
constexpr int kOffKV = 0;
constexpr int kOffX = kOffKV + kStages * kKvStage;  // [kRecvSlots] the peer's partials
constexpr int kOffXs = kOffX + kRecvSlots * kXSlot; // [2] own partials staged for the bulk copy
constexpr int kOffP = kOffXs + 2 * kXSlot;
constexpr int kOffRed = kOffP + 2 * kPBytes;   // [2][8 warps][16] p partial sums
constexpr int kOffMax = kOffRed + 2 * 8 * 16 * 4;  // [2][2][128] half-row maxima
constexpr int kOffL = kOffMax + 2 * 2 * 128 * 4;   // [2][128] half-row normalisers
constexpr int kOffBar = kOffL + 2 * 128 * 4;
constexpr int kNumBars = 2 * kStages + 8 + kRecvSlots + 1;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 64 + 1024;
constexpr int kTmemCols = 512;
constexpr uint32_t kTmemO = 0, kTmemS = 256, kTmemQ = 320;
constexpr uint32_t kIdescQK = make_idesc(1, 1, false, false, 128, kBN);
constexpr uint32_t kIdescPV = make_idesc(1, 1, false, true, 128, kDvCta);
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleLog2 = 8.0f;
// named barriers of the 256 softmax threads
constexpr int kBarRed = 1;  // p sweep partial sums
constexpr int kBarXs = 2;   // outgoing partial S staged
constexpr int kBarMax = 3;  // half-row maxima
constexpr int kBarL = 4;    // half-row normalisers
static_assert(kSmemBytes <= 232448, "shared memory");
static_assert(kKvStage % 1024 == 0, "stage alignment (128B-swizzle atoms)");
// A gather warp waits on a stage's barrier for the phase of its own previous block there; if
// the stage also served another warp's blocks, that warp could see the phase two steps ahead.
static_assert(kStages % kGatherWarps == 0, "a stage must always cycle through the same gather warp");
static_assert(kTmemQ + kDimsCta / 2 <= kTmemCols, "tensor memory");

// S = Q K^T over this CTA's 288 key dims: 16 K-steps over the four 64-dim boxes (SW128) and 2
// over the 32 rope dims (SW64).  A (Q) comes from tensor memory, 8 columns per K-step.
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_tmem, uint32_t kv_addr) {
  const uint64_t kb = make_smem_desc(kv_addr, 16, 1024, kSw128);
  const uint64_t rb = make_smem_desc(kv_addr + 4 * kMainBox, 16, 512, kSw64);
#pragma unroll
  for (int kk = 0; kk < 16; ++kk) {
    const int bx = kk >> 2, kin = kk & 3;
    mma_f16_ts(d_tmem, q_tmem + 8 * kk, kb + static_cast<uint64_t>((bx * kMainBox + kin * 32) >> 4),
               kIdescQK, kk > 0 ? 1u : 0u);
  }
#pragma unroll
  for (int kk = 0; kk < 2; ++kk)
    mma_f16_ts(d_tmem, q_tmem + 8 * (16 + kk), rb + static_cast<uint64_t>((kk * 32) >> 4), kIdescQK, 1u);
}

// O (+)= P V: A = P (128 x 32 bf16, SW64 K-major), B = the gathered value dims read MN-major
// (4 boxes of 64 dims at LBO = one box), 2 K-steps of 16 entries.
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_addr, uint32_t kv_addr,
                                         bool first) {
  const uint64_t pd = make_smem_desc(p_addr, 16, 512, kSw64);
  const uint64_t vd = make_smem_desc(kv_addr, kMainBox, 1024, kSw128);
#pragma unroll
  for (int kk = 0; kk < kBN / 16; ++kk)
    mma_f16_ss(o_tmem, pd + static_cast<uint64_t>((kk * 32) >> 4),
               vd + static_cast<uint64_t>((kk * 16 * 128) >> 4), kIdescPV, (!first || kk > 0) ? 1u : 0u);
}

// The 32 idx slots of block `blk` as seen by lane `lane` (-1 past the effective length).
__device__ __forceinline__ int block_slot(const int32_t* idx_row, int e0, int len, int blk, int lane) {
  const int slot = e0 + blk * kBN + lane;
  return (slot < e0 + len) ? __ldg(idx_row + slot) : -1;
}

__global__ void __launch_bounds__(kThreads, 1)
    sparse_mla_pair_kernel(const __grid_constant__ CUtensorMap tm_main,
                           const __grid_constant__ CUtensorMap tm_rope, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sKV = smem + kOffKV;
  uint8_t* sP = smem + kOffP;
  float* sX = reinterpret_cast<float*>(smem + kOffX);
  uint8_t* sXs = smem + kOffXs;
  float* sRed = reinterpret_cast<float*>(smem + kOffRed);
  float* sMax = reinterpret_cast<float*>(smem + kOffMax);
  float* sL = reinterpret_cast<float*>(smem + kOffL);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* kv_full = bars;                 // [kStages] expect_tx + the gathered bytes
  uint64_t* kv_empty = bars + kStages;      // [kStages] MMA commit
  uint64_t* s_full = bars + 2 * kStages;    // [2] MMA commit
  uint64_t* s_empty = s_full + 2;           // [2] 256 softmax arrivals
  uint64_t* p_full = s_full + 4;            // [2] 256 softmax arrivals
  uint64_t* o_done = s_full + 6;            // [2] MMA commit (PV of blocks i, i % 2)
  uint64_t* x_full = s_full + 8;            // [kRecvSlots] own expect_tx + the peer's bytes
  uint64_t* q_ready = x_full + kRecvSlots;  // 256 softmax arrivals: Q is in tensor memory
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  int* s_len = reinterpret_cast<int*>(smem + kOffMisc + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;

  const int pair = blockIdx.x >> 1;
  const int split = pair % p.n_split;
  const int row = pair / p.n_split;
  const int b = row / p.Lq;
  const int32_t* idx_row = p.idx + static_cast<size_t>(row) * p.k;
  const int e0 = split * p.per_split;
  const int e1 = min(p.k, e0 + p.per_split);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], kSoftmaxThreads);
      mbar_init(&p_full[i], kSoftmaxThreads);
      mbar_init(&o_done[i], 1);
    }
    for (int i = 0; i < kRecvSlots; ++i) mbar_init(&x_full[i], 1);
    mbar_init(q_ready, kSoftmaxThreads);
    *abort_flag = 0;
    *s_len = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == kMmaWarp) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  // the peer's barriers must be initialised before any remote store completes on them
  cluster_barrier();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // Effective length: slots after the last valid one in [e0, e1) need no work (same on both).
  {
    int last = -1;
    for (int x = e0 + static_cast<int>(threadIdx.x); x < e1; x += kThreads)
      if (__ldg(idx_row + x) >= 0) last = x;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) last = max(last, __shfl_xor_sync(0xFFFFFFFFu, last, o));
    if (lane == 0 && last >= 0) atomicMax(s_len, last - e0 + 1);
    __syncthreads();
  }
  const int len = *s_len;
  const int nblk = (len + kBN - 1) / kBN;
  const int total = nblk + ((p.p_sel != nullptr) ? nblk : 0);  // the p sweep revisits every block

  if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer (polling)
    if (lane == 0 && total > 0) {
      if (!mbar_wait(q_ready, 0, abort_flag, 60)) goto done;
      tc_fence_after();
      const uint32_t q_tmem = tmem_base + kTmemQ;
      int nq = 0, np = 0;  // next S block to compute, next PV block
      uint64_t t_idle = 0;
      while (nq < total || np < nblk) {
        bool progress = false;
        if (nq < total && mbar_test_wait(&kv_full[nq % kStages], (nq / kStages) & 1) &&
            mbar_test_wait(&s_empty[nq & 1], ((nq >> 1) & 1) ^ 1)) {
          tc_fence_after();
          const int st = nq % kStages;
          issue_qk(tmem_base + kTmemS + (nq & 1) * kBN, q_tmem, smem_u32(sKV + st * kKvStage));
          mma_commit(&s_full[nq & 1]);
          if (nq >= nblk) mma_commit(&kv_empty[st]);  // p sweep: no PV reads this block
          ++nq;
          progress = true;
        }
        if (np < nblk && np < nq && mbar_test_wait(&p_full[np & 1], (np >> 1) & 1)) {
          tc_fence_after();
          const int st = np % kStages;
          issue_pv(tmem_base + kTmemO, smem_u32(sP + (np & 1) * kPBytes), smem_u32(sKV + st * kKvStage),
                   np == 0);
          mma_commit(&kv_empty[st]);
          mma_commit(&o_done[np & 1]);
          ++np;
          progress = true;
        }
        if (progress) {
          t_idle = 0;
        } else {
          __nanosleep(32);  // back off: the warps sharing this SMSP do the softmax
          if (*abort_flag) goto done;
          const uint64_t now = global_timer_ns();
          if (t_idle == 0) {
            t_idle = now;
          } else if (now - t_idle > kWaitLimitNs) {
            record_timeout(61);
            *abort_flag = 1;
            goto done;
          }
        }
      }
    }
  } else if (warp >= kGatherWarp0) {
    // ------------------------------------------------------------------ gather (TMA)
    // Gather warp w takes blocks j = w, w + 6, ... (all of them in stage w)  Lane r holds the block's r-th index; lane
    // g < 8 gathers entries 4g..4g+3: the four 64-dim boxes of this CTA's value dims and its
    // 32 rope dims.  Invalid slots point one row past
    // the tensor, which the TMA fills with zeros.
    const int row0 = b * p.Lk;
    const int oob = p.B * p.Lk;
    const int g = lane & 7;
    const int main0 = static_cast<int>(rank) * kDvCta;         // first value dim of this CTA
    const int rope0 = kDV + static_cast<int>(rank) * kRopeCta;  // first rope dim of this CTA
    const int w = warp - kGatherWarp0;
    int next_s = (w < total) ? block_slot(idx_row, e0, len, w < nblk ? w : w - nblk, lane) : -1;
    int issued = w;  // one past the last block this warp issued
    if (lane == 0) {
      tma_prefetch_desc(&tm_main);
      tma_prefetch_desc(&tm_rope);
    }
    for (int j = w; j < total; j += kGatherWarps) {
      const int st = j % kStages;
      const bool got = mbar_wait(&kv_empty[st], ((j / kStages) & 1) ^ 1, abort_flag, 62);
      if (!__all_sync(0xFFFFFFFFu, got)) break;  // the shuffles below need the whole warp
      const int my_s = next_s;
      const int jn = j + kGatherWarps;
      if (jn < total) next_s = block_slot(idx_row, e0, len, jn < nblk ? jn : jn - nblk, lane);
      if (my_s >= p.Lk) record_bad_index();
      const int y = (static_cast<unsigned>(my_s) < static_cast<unsigned>(p.Lk)) ? row0 + my_s : oob;
      const int y0 = __shfl_sync(0xFFFFFFFFu, y, 4 * g);
      const int y1 = __shfl_sync(0xFFFFFFFFu, y, 4 * g + 1);
      const int y2 = __shfl_sync(0xFFFFFFFFu, y, 4 * g + 2);
      const int y3 = __shfl_sync(0xFFFFFFFFu, y, 4 * g + 3);
      if (lane == 0) mbar_arrive_expect_tx(&kv_full[st], kKvStage);
      __syncwarp();
      if (lane < 8) {
        uint8_t* dst = sKV + st * kKvStage;
#pragma unroll
        for (int bx = 0; bx < 4; ++bx)
          tma_gather4(dst + bx * kMainBox + g * 512, &tm_main, &kv_full[st], main0 + bx * 64, y0, y1, y2, y3);
        tma_gather4(dst + 4 * kMainBox + g * 256, &tm_rope, &kv_full[st], rope0, y0, y1, y2, y3);
      }
      issued = j + 1;
    }
    // Nothing of ours may still be landing when the CTA exits.  On the normal path the MMA
    // consumed every block; after an abort, wait (bounded) for this warp's last blocks.
    if (lane == 0 && *abort_flag) {
      const int lo = max(w, issued - kStages);
      for (int j = lo + (w - lo % kGatherWarps + kGatherWarps) % kGatherWarps; j < issued; j += kGatherWarps)
        mbar_drain(&kv_full[j % kStages], (j / kStages) & 1);
    }
  } else {
    // ------------------------------------------------------------------ softmax / epilogue
    // Warpgroup wg owns S columns [16 wg, 16 wg + 16) of every block and O columns
    // [128 wg, 128 wg + 128) of this CTA's value half; both hold the same per-row state.
    const int wg = warp >> 2;
    const int wq = warp & 3;
    const int h = (wq << 5) + lane;  // head row = TMEM lane (warp w owns lanes 32(w%4)..)
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tm = tmem_base + lane_off;
    const int col0 = wg * kHalf;
    const uint32_t o_cols = static_cast<uint32_t>(wg * (kDvCta / 2));
    const uint32_t peer_recv = map_to_rank(smem_u32(sX), peer);
    const uint32_t peer_x_full = map_to_rank(smem_u32(x_full), peer);
    const uint32_t hsw = static_cast<uint32_t>(h & 7);
    const size_t orow = static_cast<size_t>(row) * p.H + h;
    const bool head_ok = h < p.H;
    bool ok = true;

    if (total > 0) {
      // This CTA's 288 dims of Q into tensor memory: dims [8j, 8j+8) of the slice -> columns
      // [4j, 4j+4), in 9 groups of 16 columns (warpgroup 0 takes groups 0-4, 1 takes 5-8).
      // Heads >= H get zeros.
      const __nv_bfloat16* qrow = p.q + orow * kDQK;
#pragma unroll 1
      for (int grp = wg * 5; grp < (wg == 0 ? 5 : 9); ++grp) {
        uint4 v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int j = grp * 4 + i;
          const int d = j < 32 ? static_cast<int>(rank) * kDvCta + j * 8
                               : kDV + static_cast<int>(rank) * kRopeCta + (j - 32) * 8;
          v[i] = head_ok ? __ldg(reinterpret_cast<const uint4*>(qrow + d)) : make_uint4(0u, 0u, 0u, 0u);
        }
        const uint32_t r[16] = {v[0].x, v[0].y, v[0].z, v[0].w, v[1].x, v[1].y, v[1].z, v[1].w,
                                v[2].x, v[2].y, v[2].z, v[2].w, v[3].x, v[3].y, v[3].z, v[3].w};
        tmem_st_32x32b_x16(tm + kTmemQ + grp * 16, r);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(q_ready);
    }

    auto blk_of = [&](int q) { return q < nblk ? q : q - nblk; };
    auto mask_of = [&](int s) {
      return __ballot_sync(0xFFFFFFFFu, static_cast<unsigned>(s) < static_cast<unsigned>(p.Lk));
    };
    // validity masks of blocks q and q+1, and the pending slot load of block q+2
    uint32_t m_cur = 0, m_nxt = 0;
    int s_pf = -1;
    if (total > 0) m_cur = mask_of(block_slot(idx_row, e0, len, 0, lane));
    if (total > 1) m_nxt = mask_of(block_slot(idx_row, e0, len, blk_of(1), lane));
    if (total > 2) s_pf = block_slot(idx_row, e0, len, blk_of(2), lane);

    // Load this CTA's partial S(j) (this warpgroup's 16 columns) from tensor memory, stage it in
    // shared memory and ship the whole 128 x 32 partial to the peer's receive slot
    // j % kRecvSlots with one bulk copy.  Remote stores from the threads were measured slower:
    // 16 KB of 16-byte st.async per block takes about 1000 cycles to issue.  Row h takes 128 B,
    // 16-byte chunk c kept at chunk c ^ (h % 8) so that a warp's accesses spread over all banks.
    //   Receive slots: four make reuse safe without a back-signal.  This CTA sends block j+1 only
    //   after it received the peer's block j-1, which the peer sends only after it finished
    //   reading the slot of block j-3 = (j+1) - 4.
    //   Staging slots: j % 2.  Before the barrier of block j, thread 0 waits until its copies of
    //   blocks <= j-1 have read their source, so slot (j+1) % 2 is free once all have passed it.
    auto load_and_send = [&](int j, uint32_t (&dst)[kHalf]) {
      if (ok && !mbar_wait(&s_full[j & 1], (j >> 1) & 1, abort_flag, 63)) ok = false;
      ok = __all_sync(0xFFFFFFFFu, ok);  // tcgen05.ld is warp-collective
      if (ok) {
        tc_fence_after();
        tmem_ld_32x32b_x16(tm + kTmemS + (j & 1) * kBN + col0, dst);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&s_empty[j & 1]);
        uint8_t* stg = sXs + (j & 1) * kXSlot + h * (kBN * 4);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t c = static_cast<uint32_t>(4 * wg + i);
          *reinterpret_cast<uint4*>(stg + ((c ^ hsw) << 4)) =
              make_uint4(dst[4 * i], dst[4 * i + 1], dst[4 * i + 2], dst[4 * i + 3]);
        }
        fence_proxy_async_smem();  // the bulk copy reads through the async proxy
      } else {
#pragma unroll
        for (int c = 0; c < kHalf; ++c) dst[c] = 0u;
      }
      if (threadIdx.x == 0) bulk_wait_read_all();
      named_bar_sync(kBarXs, kSoftmaxThreads);
      if (threadIdx.x == 0 && ok) {
        const int sl = j % kRecvSlots;
        bulk_copy_to_peer(peer_recv + static_cast<uint32_t>(sl * kXSlot), smem_u32(sXs + (j & 1) * kXSlot),
                          kXSlot, peer_x_full + sl * 8);
        bulk_commit_group();
      }
    };

    float m_ref = -INFINITY;  // running reference max (log2 domain), identical in all copies
    float l = 0.f;            // this warpgroup's part of the normaliser, relative to m_ref
    float lse2 = -INFINITY;
    const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
    uint32_t cur[kHalf], nxt[kHalf];
    if (total > 0) load_and_send(0, cur);
    for (int q = 0; q < total; ++q) {
      if (q + 1 < total) load_and_send(q + 1, nxt);

      // ---- y = (own part + the peer's part of S(q)) * scale * log2(e) - off, where off is the
      // reference the block is measured against: the running max (main blocks; 0 before the
      // first valid entry) or the final lse (p sweep).  Invalid slots get -inf.
      const int sl = q % kRecvSlots;
      if (threadIdx.x == 0) mbar_arrive_expect_tx(&x_full[sl], kXSlot);
      if (ok && !mbar_wait_cluster(&x_full[sl], (q / kRecvSlots) & 1, abort_flag, 64)) ok = false;
      ok = __all_sync(0xFFFFFFFFu, ok);
      const uint32_t vm = (m_cur >> col0) & 0xFFFFu;  // the same in every warp of the group
      const bool main_blk = q < nblk;
      const float off = main_blk ? (m_ref == -INFINITY ? 0.f : m_ref) : lse2;
      float y[kHalf];
      {
        const uint8_t* mine = reinterpret_cast<const uint8_t*>(sX) + sl * kXSlot + h * (kBN * 4);
        const float2 o2 = make_float2(-off, -off);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t c = static_cast<uint32_t>(4 * wg + i);
          const float4 u = ok ? *reinterpret_cast<const float4*>(mine + ((c ^ hsw) << 4))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
          float2 a0 = add2(make_float2(__uint_as_float(cur[4 * i]), __uint_as_float(cur[4 * i + 1])),
                           make_float2(u.x, u.y));
          float2 a1 = add2(make_float2(__uint_as_float(cur[4 * i + 2]), __uint_as_float(cur[4 * i + 3])),
                           make_float2(u.z, u.w));
          a0 = fma2(a0, sc2, o2);
          a1 = fma2(a1, sc2, o2);
          y[4 * i] = a0.x;
          y[4 * i + 1] = a0.y;
          y[4 * i + 2] = a1.x;
          y[4 * i + 3] = a1.y;
        }
        if (vm != 0xFFFFu) {
#pragma unroll
          for (int c = 0; c < kHalf; ++c)
            if (!((vm >> c) & 1u)) y[c] = -INFINITY;
        }
      }
      // advance the mask pipeline (the load of block q+2 was issued one iteration ago)
      m_cur = m_nxt;
      m_nxt = mask_of(s_pf);
      s_pf = (q + 3 < total) ? block_slot(idx_row, e0, len, blk_of(q + 3), lane) : -1;

      if (main_blk) {
        // ---- online softmax of block q; y is measured against m_ref
        float t8[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) t8[c] = fmaxf(y[c], y[c + 8]);
#pragma unroll
        for (int c = 0; c < 4; ++c) t8[c] = fmaxf(t8[c], t8[c + 4]);
        float by = fmaxf(fmaxf(t8[0], t8[2]), fmaxf(t8[1], t8[3]));
        float* mx = sMax + (q & 1) * 256;  // double-buffered by block parity
        mx[wg * 128 + h] = by;
        named_bar_sync(kBarMax, kSoftmaxThreads);
        by = fmaxf(by, mx[(wg ^ 1) * 128 + h]);
        const int pb = q & 1;
        if (ok && q >= 2) {  // P buffer pb was last read by PV(q-2)
          const bool got = mbar_wait(&o_done[pb], ((q - 2) >> 1) & 1, abort_flag, 65);
          ok = __all_sync(0xFFFFFFFFu, got);
        }
        // Lazy rescale: the reference only moves (by the block's excess d) on the first valid
        // entry or when a block exceeds it by more than 2^8, so P <= 256 stays well inside bf16
        // range.  O is rescaled in tensor memory once PV(q-1) has landed (tcgen05.ld/st are
        // warp-collective, so the whole warp walks its rows); each warpgroup its 128 columns.
        const bool first = (m_ref == -INFINITY);
        const bool move = first ? (by > -INFINITY) : (by > kRescaleLog2);
        const float d = move ? by : 0.f;
        if (ok) {
          const bool scale_o = move && !first;
          const float f = scale_o ? ex2_approx(-by) : 1.f;
          if (__any_sync(0xFFFFFFFFu, scale_o)) {
            const bool got = mbar_wait(&o_done[(q - 1) & 1], ((q - 1) >> 1) & 1, abort_flag, 66);
            ok = __all_sync(0xFFFFFFFFu, got);
            if (ok) {
              tc_fence_after();
#pragma unroll 1
              for (int c0 = 0; c0 < kDvCta / 2; c0 += 16) {
                uint32_t o[16];
                tmem_ld_32x32b_x16(tm + kTmemO + o_cols + c0, o);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < 16; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * f);
                tmem_st_32x32b_x16(tm + kTmemO + o_cols + c0, o);
              }
              tmem_st_wait();
            }
          }
          l *= f;
          if (move) m_ref = first ? by : m_ref + by;
        }
        if (ok) {
          if (__any_sync(0xFFFFFFFFu, move)) {
#pragma unroll
            for (int c = 0; c < kHalf; ++c) y[c] -= d;
          }
          uint32_t pk[kHalf / 2];
          float2 rs[4];
#pragma unroll
          for (int c = 0; c < kHalf; c += 2) {
            const float2 pp = make_float2(ex2_approx(y[c]), ex2_approx(y[c + 1]));
            rs[(c >> 1) & 3] = (c < 8) ? pp : add2(rs[(c >> 1) & 3], pp);
            pk[c >> 1] = pack_bf16x2(pp.x, pp.y);
          }
          const float2 r2 = add2(add2(rs[0], rs[1]), add2(rs[2], rs[3]));
          l += r2.x + r2.y;
          uint8_t* pbuf = sP + pb * kPBytes;  // row h: 64 B, 64B-swizzled; this half = chunks 2wg, 2wg+1
          *reinterpret_cast<uint4*>(pbuf + swizzled_offset(h, 2 * wg, 64)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          *reinterpret_cast<uint4*>(pbuf + swizzled_offset(h, 2 * wg + 1, 64)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          fence_proxy_async_smem();
          tc_fence_before();
          mbar_arrive(&p_full[pb]);
        }
        if (q == nblk - 1) {
          // ---- final O: total normaliser from both halves, wait for the last PV, store this
          // warpgroup's 128 value columns
          sL[wg * 128 + h] = l;
          named_bar_sync(kBarL, kSoftmaxThreads);
          const float l_tot = sL[h] + sL[128 + h];
          if (ok) {
            const bool got = mbar_wait(&o_done[pb], (q >> 1) & 1, abort_flag, 67);
            ok = __all_sync(0xFFFFFFFFu, got);
          }
          if (ok) {
            tc_fence_after();
            const float inv_l = l_tot > 0.f ? 1.f / l_tot : 0.f;
            lse2 = l_tot > 0.f ? m_ref + log2f(l_tot) : -INFINITY;
#pragma unroll 1
            for (int c0 = 0; c0 < kDvCta / 2; c0 += 16) {
              uint32_t o[16];
              tmem_ld_32x32b_x16(tm + kTmemO + o_cols + c0, o);
              tmem_ld_wait();
              if (!head_ok) continue;
              const int col = static_cast<int>(rank) * kDvCta + static_cast<int>(o_cols) + c0;
              if (p.n_split == 1) {
                uint4 w0, w1;
                w0.x = pack_bf16x2(__uint_as_float(o[0]) * inv_l, __uint_as_float(o[1]) * inv_l);
                w0.y = pack_bf16x2(__uint_as_float(o[2]) * inv_l, __uint_as_float(o[3]) * inv_l);
                w0.z = pack_bf16x2(__uint_as_float(o[4]) * inv_l, __uint_as_float(o[5]) * inv_l);
                w0.w = pack_bf16x2(__uint_as_float(o[6]) * inv_l, __uint_as_float(o[7]) * inv_l);
                w1.x = pack_bf16x2(__uint_as_float(o[8]) * inv_l, __uint_as_float(o[9]) * inv_l);
                w1.y = pack_bf16x2(__uint_as_float(o[10]) * inv_l, __uint_as_float(o[11]) * inv_l);
                w1.z = pack_bf16x2(__uint_as_float(o[12]) * inv_l, __uint_as_float(o[13]) * inv_l);
                w1.w = pack_bf16x2(__uint_as_float(o[14]) * inv_l, __uint_as_float(o[15]) * inv_l);
                uint4* dst = reinterpret_cast<uint4*>(p.out + orow * kDV + col);
                dst[0] = w0;
                dst[1] = w1;
              } else {
                float4* dst = reinterpret_cast<float4*>(
                    p.part_o + (static_cast<size_t>(split) * p.B * p.Lq * p.H + orow) * kDV + col);
#pragma unroll
                for (int c = 0; c < 16; c += 4)
                  dst[c / 4] = make_float4(__uint_as_float(o[c]) * inv_l, __uint_as_float(o[c + 1]) * inv_l,
                                           __uint_as_float(o[c + 2]) * inv_l, __uint_as_float(o[c + 3]) * inv_l);
              }
            }
            if (head_ok && rank == 0 && wg == 0) {
              const float lse_nat = lse2 * kLn2;
              if (p.n_split == 1) {
                if (p.lse) p.lse[orow] = lse_nat;
              } else {
                p.part_lse[static_cast<size_t>(split) * p.B * p.Lq * p.H + orow] = lse_nat;
              }
            }
          }
        }
      } else {
        // ---- p sweep: P = exp2(y) (y measured against lse) summed over heads h < H, / H.  Blocks
        // alternate between the two CTAs (both computed the same S); each warpgroup sums its 16
        // columns.
        const int blk = blk_of(q);
        if ((blk & 1) == static_cast<int>(rank)) {
          const bool live = ok && head_ok && lse2 != -INFINITY;
          float v[kHalf];
#pragma unroll
          for (int c = 0; c < kHalf; ++c) v[c] = live ? ex2_approx(y[c]) : 0.f;
          // butterfly reduce-scatter: lane L ends with column L % 16 summed over its 16-lane
          // half, then over the whole warp
#pragma unroll
          for (int off2 = 8; off2 >= 1; off2 >>= 1) {
            const bool upper = (lane & off2) != 0;
#pragma unroll
            for (int i = 0; i < off2; ++i) {
              const float send = upper ? v[i] : v[i + off2];
              const float keep = upper ? v[i + off2] : v[i];
              v[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, off2);
            }
          }
          v[0] += __shfl_xor_sync(0xFFFFFFFFu, v[0], 16);
          float* red = sRed + ((blk >> 1) & 1) * 128;  // double-buffered by own-block parity
          if (lane < 16) red[warp * 16 + lane] = v[0];
          named_bar_sync(kBarRed, kSoftmaxThreads);
          if (wq == 0 && lane < 16 && ok) {
            const float* r4 = red + wg * 64;  // warps 4wg .. 4wg+3
            const float tot = r4[lane] + r4[16 + lane] + r4[32 + lane] + r4[48 + lane];
            const int slot2 = e0 + blk * kBN + col0 + lane;
            if (slot2 < e1)
              p.p_sel[static_cast<size_t>(row) * p.k + slot2] = ((vm >> lane) & 1u) ? tot / p.H : 0.f;
          }
        }
      }
#pragma unroll
      for (int c = 0; c < kHalf; ++c) cur[c] = nxt[c];
    }

    // p emission: slots past the effective length are empty (p = 0)
    if (p.p_sel != nullptr && rank == 0) {
      for (int x2 = e0 + nblk * kBN + static_cast<int>(threadIdx.x); x2 < e1; x2 += kSoftmaxThreads)
        p.p_sel[static_cast<size_t>(row) * p.k + x2] = 0.f;
    }
    if (nblk == 0 && head_ok) {  // no valid entry in this split
      for (int c = 0; c < kDvCta / 2; ++c) {
        const int col = static_cast<int>(rank) * kDvCta + static_cast<int>(o_cols) + c;
        if (p.n_split == 1)
          p.out[orow * kDV + col] = __float2bfloat16_rn(0.f);
        else
          p.part_o[(static_cast<size_t>(split) * p.B * p.Lq * p.H + orow) * kDV + col] = 0.f;
      }
      if (rank == 0 && wg == 0) {
        if (p.n_split == 1) {
          if (p.lse) p.lse[orow] = -INFINITY;
        } else {
          p.part_lse[static_cast<size_t>(split) * p.B * p.Lq * p.H + orow] = -INFINITY;
        }
      }
    }
  }
done:
  tc_fence_before();
  __syncthreads();
  // neither CTA may leave while its peer can still store into its shared memory
  cluster_barrier();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace mla_pair
}  // namespace dsa
