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
// Tensor memory (512 columns): O [0, 256) fp32, S 2 x 32 fp32 [256, 320), this CTA's slice of
// Q, 128 heads x 288 bf16, as the A operand of S = Q K^T [320, 464), and P 2 x 16 [464, 496)
// (bf16, the A operand of O += P V).  Keeping Q in tensor memory means S only streams the
// gathered tile (36 KB per pair of blocks) from shared memory, and leaves shared memory to
// the 4-stage gather ring and the partial-S receive slots (which also stage the outgoing
// partials, see the exchange argument in the softmax role).
//
// Pipeline (per CTA, blocks of 32 selected entries; a p sweep revisits every block):
//   gather warps   TMA tile::gather4: 4 selected rows per instruction, landing in the
//                  swizzled K-major tiles the MMA reads (4 stages of a pair of blocks, 80
//                  instructions each); all seven warps share every stage.
//   MMA thread     polls: S = Q K^T of a pair of blocks (N = 64) as soon as its stage landed
//                  and the previous pair's S was read;
//                  O += P(i) V_i as soon as P(i) is written (never waits behind a late gather)
//   softmax        two warpgroups on the same 128 TMEM lanes (thread = head row) take turns by
//                  block, so two blocks are in flight: each loads its partial S, ships it to the
//                  peer, adds the peer's part, settles the block's per-row reference max with
//                  the other group (the only serial link), and writes P.  See the softmax role.
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

constexpr int kBN = 32;             // selected entries per softmax block
constexpr int kPairN = 2 * kBN;     // entries per gathered stage and per S = Q K^T (MMA N = 64)
constexpr int kStages = 4;          // gather ring depth (pairs of blocks)
constexpr int kRecvSlots = 4;       // partial-S receive slots (see the exchange argument below)
constexpr int kThreads = 512;       // warps 0-7 softmax, 8 MMA, 9-15 gather
constexpr int kSoftmaxThreads = 256;  // two warpgroups taking turns by block
constexpr int kMmaWarp = 8;
constexpr int kGatherWarp0 = 9;
constexpr int kGatherWarps = 7;
constexpr int kDQK = 576, kDV = 512, kDvCta = 256, kRopeCta = 32;
constexpr int kDimsCta = kDvCta + kRopeCta;         // 288 key dims per CTA
constexpr int kMainBox = kPairN * 128;              // 64 entries x 64 dims (SW128)
constexpr int kRopeTile = kPairN * 64;              // 64 entries x 32 dims (SW64)
constexpr int kKvStage = 4 * kMainBox + kRopeTile;  // 36 KB
constexpr int kXSlot = 128 * kBN * 4;               // one partial S (fp32, 16 KB)
constexpr int kOffKV = 0;
constexpr int kOffX = kOffKV + kStages * kKvStage;  // [kRecvSlots] the peer's partials; slot
                                                    // (q + 2) % 4 also stages block q's own
constexpr int kOffRef = kOffX + kRecvSlots * kXSlot;  // [2][128] per-row reference of a block
constexpr int kOffRed = kOffRef;                   // [2 groups][4 warps][32] p partial sums: the p
                                                   // sweep starts after every reference was read
constexpr int kOffFin = kOffRef + 2 * 128 * 4;     // [2 groups][2][128] final (l, reference)
constexpr int kOffBar = kOffFin + 2 * 2 * 128 * 4;
constexpr int kNumBars = 2 * kStages + 8 + kRecvSlots + 4;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 64 + 1024;
constexpr int kTmemCols = 512;
constexpr uint32_t kTmemO = 0, kTmemS = 256, kTmemQ = 320, kTmemP = 464;
constexpr uint32_t kIdescQK = make_idesc(1, 1, false, false, 128, kPairN);
constexpr uint32_t kIdescPV = make_idesc(1, 1, false, true, 128, kDvCta);
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleLog2 = 8.0f;
// named barriers: per softmax warpgroup (128 threads) + g, and one of all 256
constexpr int kBarXs0 = 1;   // outgoing partial S staged
constexpr int kBarRed0 = 3;  // p sweep partial sums
constexpr int kBarFin = 5;   // final normaliser of both groups
static_assert(kSmemBytes <= 232448, "shared memory");
static_assert(kKvStage % 1024 == 0, "stage alignment (128B-swizzle atoms)");
// Epilogue tiles in the gather ring (idle once the last PV is done, without a p sweep): rows of
// one head, padded by 16 bytes so that a warp writing one chunk of each of 32 rows is free of
// bank conflicts, then copied to HBM by whole rows (coalesced).
constexpr int kPitchF = kDvCta * 4 + 16;   // fp32 row (a partial O exported between splits)
constexpr int kPitchB = kDvCta * 2 + 16;   // bf16 row (the output)
constexpr int kOffOutTile = 64 * kPitchF;  // the combined output tile, after the import tile
static_assert(128 * kPitchB <= kStages * kKvStage && kOffOutTile + 64 * kPitchB <= kStages * kKvStage,
              "epilogue tiles fit in the gather ring");
// This CTA's Q slice (128 head rows x 288 dims) is staged by TMA in gather stages 1.. before the
// first gathers need them: four 64-dim boxes (SW128) and the 32 rope dims (SW64).
constexpr int kQBox = 128 * 128;
constexpr int kQBytes = 4 * kQBox + 128 * 64;
static_assert(kQBytes <= (kStages - 1) * kKvStage, "Q staging fits in stages 1..");
static_assert(kGatherWarps * 12 >= 80, "every gather operation of a stage has a lane");
static_assert(kTmemQ + kDimsCta / 2 <= kTmemP && kTmemP + 2 * kBN / 2 <= kTmemCols, "tensor memory");

// S = Q K^T of a pair of blocks (64 entries, N = 64: an M = 128, K = 16 MMA costs the same ~51
// cycles at N = 32 and N = 64, and reaches full rate only from N = 128) over this CTA's 288 key
// dims: 16 K-steps over the four 64-dim boxes (SW128) and 2 over the 32 rope dims (SW64).  A (Q)
// comes from tensor memory, 8 columns per K-step; D is the pair's 64 S columns.
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

// O (+)= P V of one block: A = P (128 x 32 bf16 in tensor memory, 16 columns, written by the
// softmax threads), B = the block's half (rows 32 half.. of each box) of the gathered value dims
// read MN-major (4 boxes of 64 dims at LBO = one box), 2 K-steps of 16 entries.
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint32_t kv_addr, int half, bool first) {
  const uint64_t vd = make_smem_desc(kv_addr + half * (kBN * 128), kMainBox, 1024, kSw128);
#pragma unroll
  for (int kk = 0; kk < kBN / 16; ++kk)
    mma_f16_ts(o_tmem, p_tmem + 8 * kk, vd + static_cast<uint64_t>((kk * 16 * 128) >> 4), kIdescPV,
               (!first || kk > 0) ? 1u : 0u);
}

// The 32 idx slots of block `blk` as seen by lane `lane` (-1 past the effective length).
__device__ __forceinline__ int block_slot(const Params& p, const int32_t* idx_row, int e0, int len, int blk,
                                          int lane) {
  const int slot = e0 + blk * kBN + lane;
  return (slot < e0 + len) ? mla::slot_position(p, idx_row, slot) : -1;
}

__global__ void __launch_bounds__(kThreads, 1)
    sparse_mla_pair_kernel(const __grid_constant__ CUtensorMap tm_main,
                           const __grid_constant__ CUtensorMap tm_rope,
                           const __grid_constant__ CUtensorMap tm_q_main,
                           const __grid_constant__ CUtensorMap tm_q_rope, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sKV = smem + kOffKV;
  float* sX = reinterpret_cast<float*>(smem + kOffX);
  float* sRed = reinterpret_cast<float*>(smem + kOffRed);
  float* sRef = reinterpret_cast<float*>(smem + kOffRef);
  float* sFin = reinterpret_cast<float*>(smem + kOffFin);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* kv_full = bars;                 // [kStages] expect_tx + the gathered bytes
  uint64_t* kv_empty = bars + kStages;      // [kStages] MMA commit
  uint64_t* s_full = bars + 2 * kStages;    // [1 used] MMA commit of a pair's S
  uint64_t* s_empty = s_full + 2;           // [2] per half of a pair: 128 arrivals of its warpgroup
  uint64_t* p_full = s_full + 4;            // [2] 128 arrivals of the block's warpgroup
  uint64_t* o_done = s_full + 6;            // [2] MMA commit (PV of blocks i, i % 2)
  uint64_t* x_full = s_full + 8;            // [kRecvSlots] own expect_tx + the peer's bytes
  uint64_t* q_ready = x_full + kRecvSlots;  // 256 softmax arrivals: Q is in tensor memory
  uint64_t* ref_full = q_ready + 1;         // [2] 128 arrivals: a block's reference is published
  uint64_t* q_full = ref_full + 2;          // expect_tx + the staged Q slice
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  int* s_len = reinterpret_cast<int*>(smem + kOffMisc + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t crank = cluster_ctarank();
  const uint32_t rank = crank & 1u;  // which half of the dims (within the pair)
  const uint32_t peer = crank ^ 1u;  // cluster rank of the pair's other CTA

  const int pair = blockIdx.x >> 1;
  const int split = pair % p.n_split;
  const int row = mla::work_row(p, pair / p.n_split);
  const int b = row / p.Lq;
  const int32_t* idx_row = p.dense ? nullptr : p.idx + static_cast<size_t>(row) * p.k;
  const int e0 = split * p.per_split;
  const int e1 = min(p.k, e0 + p.per_split);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 128);
      mbar_init(&p_full[i], 128);
      mbar_init(&ref_full[i], 128);
      mbar_init(&o_done[i], 1);
    }
    for (int i = 0; i < kRecvSlots; ++i) mbar_init(&x_full[i], 1);
    mbar_init(q_ready, kSoftmaxThreads);
    mbar_init(q_full, 1);
    *abort_flag = 0;
    *s_len = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  pdl_launch_dependents();
  if (threadIdx.x == kMmaWarp * 32) {
    // this CTA's Q slice into L2 while the previous kernel of the stream finishes (a prefetch
    // only warms the cache; the loads below come after the dependency wait)
#pragma unroll
    for (int i = 0; i < 4; ++i) tma_prefetch_2d(&tm_q_main, static_cast<int>(rank) * kDvCta + i * 64, row * p.H);
    tma_prefetch_2d(&tm_q_rope, kDV + static_cast<int>(rank) * kRopeCta, row * p.H);
  }
  if (warp == kMmaWarp) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  // the peer's barriers must be initialised before any remote store completes on them
  cluster_barrier();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // first global access below
  if (threadIdx.x == kMmaWarp * 32) {
    // Q rows row*H .. row*H+127 (rows past H belong to other queries or lie outside the tensor
    // and are zeroed by the readers), this CTA's dims
    uint8_t* qs = sKV + kKvStage;
    const int y = row * p.H;
    mbar_arrive_expect_tx(q_full, kQBytes);
#pragma unroll
    for (int i = 0; i < 4; ++i) tma_load_2d(qs + i * kQBox, &tm_q_main, q_full, static_cast<int>(rank) * kDvCta + i * 64, y);
    tma_load_2d(qs + 4 * kQBox, &tm_q_rope, q_full, kDV + static_cast<int>(rank) * kRopeCta, y);
  }

  // Effective length: slots after the last valid one in [e0, e1) need no work (same on both).
  if (!p.dense) {
    int last = -1;
    for (int x = e0 + static_cast<int>(threadIdx.x); x < e1; x += kThreads)
      if (__ldg(idx_row + x) >= 0) last = x;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) last = max(last, __shfl_xor_sync(0xFFFFFFFFu, last, o));
    if (lane == 0 && last >= 0) atomicMax(s_len, last - e0 + 1);
    __syncthreads();
  }
  const int len = p.dense ? mla::dense_len(p, row, e0, e1) : *s_len;
  const int nblk = (len + kBN - 1) / kBN;
  const int total = nblk + ((p.p_sel != nullptr) ? nblk : 0);  // the p sweep revisits every block

  if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer (polling)
    if (lane == 0 && total > 0) {
      if (!mbar_wait_spin(q_ready, 0, abort_flag, 60)) goto done;
      tc_fence_after();
      const uint32_t q_tmem = tmem_base + kTmemQ;
      const int npairs = (total + 1) / 2;
      int nq = 0, np = 0;  // next pair to compute S for, next block to run PV for
      uint64_t t_idle = 0;
      while (nq < npairs || np < nblk) {
        bool progress = false;
        // S of pair nq once its stage has landed and both halves of pair nq-1 were read
        if (nq < npairs && mbar_test_wait(&kv_full[nq % kStages], (nq / kStages) & 1) &&
            mbar_test_wait(&s_empty[0], (nq & 1) ^ 1) && mbar_test_wait(&s_empty[1], (nq & 1) ^ 1)) {
          tc_fence_after();
          const int st = nq % kStages;
          issue_qk(tmem_base + kTmemS, q_tmem, smem_u32(sKV + st * kKvStage));
          mma_commit(&s_full[0]);
          if (2 * nq >= nblk) mma_commit(&kv_empty[st]);  // no PV reads this stage (p sweep)
          ++nq;
          progress = true;
        }
        // PV of block np; the stage is released after the last MMA that reads it
        if (np < nblk && (np >> 1) < nq && mbar_test_wait(&p_full[np & 1], (np >> 1) & 1)) {
          tc_fence_after();
          const int st = (np >> 1) % kStages;
          issue_pv(tmem_base + kTmemO, tmem_base + kTmemP + (np & 1) * (kBN / 2), smem_u32(sKV + st * kKvStage),
                   np & 1, np == 0);
          if ((np & 1) || np + 1 >= nblk) mma_commit(&kv_empty[st]);
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
          } else if (now - t_idle > wait_limit_ns()) {
            record_timeout(61);
            *abort_flag = 1;
            goto done;
          }
        }
      }
    }
  } else if (warp >= kGatherWarp0) {
    // ------------------------------------------------------------------ gather (TMA)
    // A stage holds a pair of blocks (64 entries): 80 gather4 operations (16 groups of four
    // entries x the four 64-dim boxes of this CTA's value dims and its 32 rope dims).  All gather
    // warps share every stage - warp w issues operations w, w + 7, ... (lanes 0-11) - since one
    // warp issues them about 80 cycles apart.  Every warp waits on the same stage barrier for
    // every pair; none can run two phases ahead, since pair jp + kStages needs pair jp consumed,
    // which needs pair jp landed.  Lane r holds the r-th index of each block of the pair;
    // invalid slots (and the missing half of an odd last pair) point one row past the tensor,
    // which the TMA fills with zeros.
    const int len_b = mla::row_len(p, b);
    const int w = warp - kGatherWarp0;
    const int op = w + kGatherWarps * lane;  // this lane's operation of each stage
    const bool has_op = lane < 12 && op < 80;
    const int g = has_op ? op / 5 : 0;       // entry group: entries 4g..4g+3 of the pair
    const int bx = has_op ? op % 5 : 0;      // 0-3: value box, 4: rope dims
    const int x0 = bx < 4 ? static_cast<int>(rank) * kDvCta + bx * 64 : kDV + static_cast<int>(rank) * kRopeCta;
    const CUtensorMap* tmap = bx < 4 ? &tm_main : &tm_rope;
    const uint32_t dst_off = bx < 4 ? static_cast<uint32_t>(bx * kMainBox + g * 512) : static_cast<uint32_t>(4 * kMainBox + g * 256);
    const int npairs = (total + 1) / 2;
    auto slot_of = [&](int j) { return j < total ? block_slot(p, idx_row, e0, len, j < nblk ? j : j - nblk, lane) : -1; };
    // two-deep pipeline of the lookups: the slots (idx loads) two pairs ahead, the rows (a block
    // table load for a paged cache) one pair ahead
    auto row_of = [&](int sv) {
      if (sv >= len_b) record_bad_index();
      return mla::kv_row(p, b, len_b, sv);
    };
    int y_nlo = row_of((total > 0) ? slot_of(0) : -1), y_nhi = row_of((total > 1) ? slot_of(1) : -1);
    int s_nlo = slot_of(2), s_nhi = slot_of(3);
    int issued = 0;
    if (lane == 0) {
      tma_prefetch_desc(&tm_main);
      tma_prefetch_desc(&tm_rope);
    }
    for (int jp = 0; jp < npairs; ++jp) {
      const int st = jp % kStages;
      // stages 1.. hold the staged Q until it is in tensor memory
      bool got = jp != 1 || mbar_wait_spin(q_ready, 0, abort_flag, 66);
      got = got && mbar_wait_spin(&kv_empty[st], ((jp / kStages) & 1) ^ 1, abort_flag, 62);
      if (!__all_sync(0xFFFFFFFFu, got)) break;  // the shuffles below need the whole warp
      const int y_lo = y_nlo, y_hi = y_nhi;
      if (jp + 1 < npairs) {
        y_nlo = row_of(s_nlo);
        y_nhi = row_of(s_nhi);
        s_nlo = slot_of(2 * jp + 4);
        s_nhi = slot_of(2 * jp + 5);
      }
      const int src = 4 * (g & 7);
      int yv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int a = __shfl_sync(0xFFFFFFFFu, y_lo, src + i);
        const int c = __shfl_sync(0xFFFFFFFFu, y_hi, src + i);
        yv[i] = g < 8 ? a : c;
      }
      if (w == 0 && lane == 0) mbar_arrive_expect_tx(&kv_full[st], kKvStage);
      if (has_op) tma_gather4(sKV + st * kKvStage + dst_off, tmap, &kv_full[st], x0, yv[0], yv[1], yv[2], yv[3]);
      issued = jp + 1;
    }
    // Nothing of ours may still be landing when the CTA exits.  On the normal path the MMA
    // consumed every stage; after an abort, wait (bounded) for the last stages.
    if (w == 0 && lane == 0 && *abort_flag)
      for (int j = max(0, issued - kStages); j < issued; ++j) mbar_drain(&kv_full[j % kStages], (j / kStages) & 1);
  } else {
    // ------------------------------------------------------------------ softmax / epilogue
    // Warpgroup wg handles blocks q = wg, wg + 2, ... (thread = head row over all 32 columns),
    // so two blocks are in flight.  Per block:
    //   1. load the own partial S(q), stage it and bulk-copy it to the peer's receive slot;
    //   2. add the peer's part: z = S * scale * log2(e), invalid slots -inf; row max bz;
    //   3. the block's per-row reference r_q: take r_{q-1} from the other group (published in
    //      shared memory with an mbarrier), keep it unless bz exceeds it by more than 2^8 (lazy
    //      rescaling, so P <= 256), publish r_q - the only serial link between the groups;
    //   4. if the reference moved, rescale O in tensor memory between PV(q-1) and PV(q);
    //      P = 2^(z - r_q) -> bf16 -> the group's P buffer; l accumulates relative to r_q.
    // Both CTAs of the pair see identical S and take identical decisions.
    const int wg = warp >> 2;
    const int wq = warp & 3;
    const int h = (wq << 5) + lane;  // head row = TMEM lane (warp w owns lanes 32(w%4)..)
    const int wtid = threadIdx.x & 127;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tm = tmem_base + lane_off;
    const uint32_t peer_recv = map_to_rank(smem_u32(sX), peer);
    const uint32_t peer_x_full = map_to_rank(smem_u32(x_full), peer);
    const uint32_t hsw = static_cast<uint32_t>(h & 7);
    const size_t orow = static_cast<size_t>(row) * p.H + h;
    const bool head_ok = h < p.H;
    const int bar_xs = kBarXs0 + wg, bar_red = kBarRed0 + wg;
    bool ok = true;

    // This CTA's 288 dims of Q into tensor memory: dims [8j, 8j+8) of the slice -> columns
    // [4j, 4j+4), in 9 groups of 16 columns (warpgroup 0 takes groups 0-4, 1 takes 5-8), read
    // from the TMA-staged slice (row h of a box; 16-byte chunk c sits at c ^ (h & 7) in a
    // 128-byte row, at c ^ ((h >> 1) & 3) in a 64-byte rope row).  Heads >= H get zeros.  The
    // staged slice is waited for even with no work, so no copy is in flight at exit.
    if (!mbar_wait_spin(q_full, 0, abort_flag, 65)) {
      ok = false;
      if (threadIdx.x == 0) mbar_drain(q_full, 0);  // let the staged copy land before exit
    }
    if (ok && total > 0) {
      const uint8_t* qs = sKV + kKvStage;
      const int g0 = wg * 5, ng = wg == 0 ? 5 : 4;
#pragma unroll
      for (int gi = 0; gi < 5; ++gi) {
        if (gi < ng) {
          const int gg = g0 + gi;
          uint4 v[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint8_t* src = gg < 8 ? qs + (gg >> 1) * kQBox + h * 128 + ((((gg & 1) * 4 + c) ^ (h & 7)) << 4)
                                        : qs + 4 * kQBox + h * 64 + ((c ^ ((h >> 1) & 3)) << 4);
            v[c] = head_ok ? *reinterpret_cast<const uint4*>(src) : make_uint4(0u, 0u, 0u, 0u);
          }
          const uint32_t r[16] = {v[0].x, v[0].y, v[0].z, v[0].w, v[1].x, v[1].y, v[1].z, v[1].w,
                                  v[2].x, v[2].y, v[2].z, v[2].w, v[3].x, v[3].y, v[3].z, v[3].w};
          tmem_st_32x32b_x16(tm + kTmemQ + gg * 16, r);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(q_ready);
    }

    auto blk_of = [&](int q) { return q < nblk ? q : q - nblk; };
    const int len_s = mla::row_len(p, b);
    auto mask_of = [&](int s) {
      return __ballot_sync(0xFFFFFFFFu, static_cast<unsigned>(s) < static_cast<unsigned>(len_s));
    };

    // Steps 1-2 for block q: z[] = the full S(q) (unscaled), -inf at invalid slots.
    // Receive slots q % 4: four make reuse safe without a back-signal.  This group sends block
    // q+4 only after it received the peer group's block q+2, which that group sends only after
    // it finished reading the slot of block q.
    // Staging: the own partial of block q goes out from this CTA's receive slot (q + 2) % 4.  This
    // group finished reading it (the peer's block q-2) before starting block q, and the peer
    // writes it next with its block q+2, which it sends only after it received this group's
    // block q - that is, after the bulk copy read the staged rows.  The group's leader also waits
    // until its previous copy has read its source before the slot is rewritten.
    auto full_s = [&](int q, uint32_t vm, float (&z)[32]) {
      uint8_t* stg = reinterpret_cast<uint8_t*>(sX) + ((q + 2) % kRecvSlots) * kXSlot;
      uint8_t* stg_row = stg + h * (kBN * 4);
      if (wtid == 0) bulk_wait_read_all();
      named_bar_sync(bar_xs, 128);
      uint32_t v[32];
      if (ok && !mbar_wait_spin(&s_full[0], (q >> 1) & 1, abort_flag, 63)) ok = false;
      ok = __all_sync(0xFFFFFFFFu, ok);  // tcgen05.ld is warp-collective
      if (ok) {
        tc_fence_after();
        tmem_ld_32x32b_x32(tm + kTmemS + (q & 1) * kBN, v);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&s_empty[q & 1]);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          *reinterpret_cast<uint4*>(stg_row + ((static_cast<uint32_t>(i) ^ hsw) << 4)) =
              make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        fence_proxy_async_smem();  // the bulk copy reads through the async proxy
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) v[c] = 0u;
      }
      named_bar_sync(bar_xs, 128);
      const int sl = q % kRecvSlots;
      if (wtid == 0) {
        if (ok)
          bulk_copy_to_peer(peer_recv + static_cast<uint32_t>(sl * kXSlot), smem_u32(stg), kXSlot,
                            peer_x_full + sl * 8);
        bulk_commit_group();
        mbar_arrive_expect_tx(&x_full[sl], kXSlot);
      }
      if (ok && !mbar_wait_cluster(&x_full[sl], (q / kRecvSlots) & 1, abort_flag, 64)) ok = false;
      ok = __all_sync(0xFFFFFFFFu, ok);
      const uint8_t* mine = reinterpret_cast<const uint8_t*>(sX) + sl * kXSlot + h * (kBN * 4);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 u = ok ? *reinterpret_cast<const float4*>(mine + ((static_cast<uint32_t>(i) ^ hsw) << 4))
                            : make_float4(0.f, 0.f, 0.f, 0.f);
        const float2 a0 = add2(make_float2(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1])), make_float2(u.x, u.y));
        const float2 a1 = add2(make_float2(__uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3])), make_float2(u.z, u.w));
        z[4 * i] = a0.x;
        z[4 * i + 1] = a0.y;
        z[4 * i + 2] = a1.x;
        z[4 * i + 3] = a1.y;
      }
      if (vm != 0xFFFFFFFFu) {
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if (!((vm >> c) & 1u)) z[c] = -INFINITY;
      }
    };

    const float sc = p.scale_log2;  // > 0, so max(t) * sc = max(t * sc)
    // Fused combine of two splits: this CTA finalises heads [64 split, 64 split + 64) and
    // exports the other heads' normalised partial O and lse for the other split's CTA.
    const bool own_head = (h >> 6) == split;
    float own_inv_l = 0.f;
    // the epilogue goes through shared-memory tiles when the gather ring is idle by then
    const bool staged = p.fuse2 || (p.n_split == 1 && p.p_sel == nullptr);
    const size_t rows_h = static_cast<size_t>(p.B) * p.Lq * p.H;
    float r = -INFINITY;  // reference of this group's previous block; l is relative to it
    float l = 0.f;
    float lse2 = -INFINITY;
    bool fin = false;
    // Final normaliser and O: both groups' l brought to the last block's reference, which is
    // the largest (references never decrease); each group stores its 128 value columns.
    auto finish = [&]() {
      sFin[(wg * 2) * 128 + h] = l;
      sFin[(wg * 2 + 1) * 128 + h] = r;
      named_bar_sync(kBarFin, kSoftmaxThreads);
      const float l0 = sFin[h], r0 = sFin[128 + h], l1 = sFin[256 + h], r1 = sFin[384 + h];
      const float rf = fmaxf(r0, r1);
      const float l_tot = (r0 == -INFINITY ? 0.f : l0 * ex2_approx(r0 - rf)) +
                          (r1 == -INFINITY ? 0.f : l1 * ex2_approx(r1 - rf));
      lse2 = l_tot > 0.f ? rf + log2f(l_tot) : -INFINITY;
      if (nblk == 0) return;
      const int ql = nblk - 1;
      if (ok) {
        const bool got = mbar_wait_spin(&o_done[ql & 1], (ql >> 1) & 1, abort_flag, 67);
        ok = __all_sync(0xFFFFFFFFu, got);
      }
      if (!ok) return;
      tc_fence_after();
      const float inv_l = l_tot > 0.f ? 1.f / l_tot : 0.f;
      own_inv_l = inv_l;
      const uint32_t o_cols = static_cast<uint32_t>(wg * (kDvCta / 2));
      if (p.fuse2 && own_head) return;  // finalised after the cluster barrier, from tensor memory
      // staged: this thread's row goes to an epilogue tile (copied out by whole rows below)
      uint8_t* trow = p.fuse2 ? sKV + (h & 63) * kPitchF + wg * (kDvCta / 2) * 4
                              : sKV + h * kPitchB + wg * (kDvCta / 2) * 2;
#pragma unroll 1
      for (int c0 = 0; c0 < kDvCta / 2; c0 += 16) {
        uint32_t o[16];
        tmem_ld_32x32b_x16(tm + kTmemO + o_cols + c0, o);
        tmem_ld_wait();
        if (!head_ok) continue;
        const int col = static_cast<int>(rank) * kDvCta + static_cast<int>(o_cols) + c0;
        if (staged && !p.fuse2) {
          uint4* dst = reinterpret_cast<uint4*>(trow + c0 * 2);
          dst[0] = make_uint4(pack_bf16x2(__uint_as_float(o[0]) * inv_l, __uint_as_float(o[1]) * inv_l),
                              pack_bf16x2(__uint_as_float(o[2]) * inv_l, __uint_as_float(o[3]) * inv_l),
                              pack_bf16x2(__uint_as_float(o[4]) * inv_l, __uint_as_float(o[5]) * inv_l),
                              pack_bf16x2(__uint_as_float(o[6]) * inv_l, __uint_as_float(o[7]) * inv_l));
          dst[1] = make_uint4(pack_bf16x2(__uint_as_float(o[8]) * inv_l, __uint_as_float(o[9]) * inv_l),
                              pack_bf16x2(__uint_as_float(o[10]) * inv_l, __uint_as_float(o[11]) * inv_l),
                              pack_bf16x2(__uint_as_float(o[12]) * inv_l, __uint_as_float(o[13]) * inv_l),
                              pack_bf16x2(__uint_as_float(o[14]) * inv_l, __uint_as_float(o[15]) * inv_l));
        } else if (p.fuse2) {
          float4* dst = reinterpret_cast<float4*>(trow + c0 * 4);
#pragma unroll
          for (int c = 0; c < 16; c += 4)
            dst[c / 4] = make_float4(__uint_as_float(o[c]) * inv_l, __uint_as_float(o[c + 1]) * inv_l,
                                     __uint_as_float(o[c + 2]) * inv_l, __uint_as_float(o[c + 3]) * inv_l);
        } else if (p.n_split == 1) {
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
          float4* dst = reinterpret_cast<float4*>(p.part_o + (static_cast<size_t>(split) * p.B * p.Lq * p.H + orow) * kDV + col);
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
    };

    // mask of this group's next block and the pending slot load of the one after
    uint32_t m_cur = mask_of((wg < total) ? block_slot(p, idx_row, e0, len, blk_of(wg), lane) : -1);
    int s_pf = (wg + 2 < total) ? block_slot(p, idx_row, e0, len, blk_of(wg + 2), lane) : -1;
    for (int q = wg; q < total; q += 2) {
      const uint32_t vm = m_cur;
      m_cur = mask_of(s_pf);
      s_pf = (q + 4 < total) ? block_slot(p, idx_row, e0, len, blk_of(q + 4), lane) : -1;
      if (q >= nblk && !fin) {
        finish();
        fin = true;
      }
      float t[32];
      full_s(q, vm, t);
      if (q < nblk) {
        // ---- step 3: the block's reference
        float m8[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) m8[c] = fmaxf(fmaxf(t[c], t[c + 8]), fmaxf(t[c + 16], t[c + 24]));
        const float bz = fmaxf(fmaxf(fmaxf(m8[0], m8[4]), fmaxf(m8[1], m8[5])),
                               fmaxf(fmaxf(m8[2], m8[6]), fmaxf(m8[3], m8[7]))) * sc;
        float rp = -INFINITY;
        if (q > 0) {
          if (ok && !mbar_wait_spin(&ref_full[(q - 1) & 1], ((q - 1) >> 1) & 1, abort_flag, 68)) ok = false;
          ok = __all_sync(0xFFFFFFFFu, ok);
          rp = sRef[((q - 1) & 1) * 128 + h];
        }
        const float rq = (rp == -INFINITY) ? bz : ((bz > rp + kRescaleLog2) ? bz : rp);
        sRef[(q & 1) * 128 + h] = rq;
        mbar_arrive(&ref_full[q & 1]);
        // ---- step 4: rescale O if the reference moved, then P
        const int pb = q & 1;
        if (ok && q >= 2) {  // P buffer pb was last read by PV(q-2)
          const bool got = mbar_wait_spin(&o_done[pb], ((q - 2) >> 1) & 1, abort_flag, 65);
          ok = __all_sync(0xFFFFFFFFu, got);
        }
        const bool moved = (rp != -INFINITY) && (rq != rp);
        if (ok && __any_sync(0xFFFFFFFFu, moved)) {
          const bool got = mbar_wait_spin(&o_done[(q - 1) & 1], ((q - 1) >> 1) & 1, abort_flag, 66);
          ok = __all_sync(0xFFFFFFFFu, got);
          if (ok) {
            const float f = moved ? ex2_approx(rp - rq) : 1.f;
            tc_fence_after();
#pragma unroll 1
            for (int c0 = 0; c0 < kDvCta; c0 += 16) {
              uint32_t o[16];
              tmem_ld_32x32b_x16(tm + kTmemO + c0, o);
              tmem_ld_wait();
#pragma unroll
              for (int c = 0; c < 16; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * f);
              tmem_st_32x32b_x16(tm + kTmemO + c0, o);
            }
            tmem_st_wait();
          }
        }
        if (r != -INFINITY && r != rq) l *= ex2_approx(r - rq);
        r = rq;
        if (ok) {
          const bool live = rq != -INFINITY;
          const float2 nr2 = make_float2(-rq, -rq), sc2 = make_float2(sc, sc);
          uint32_t pk[16];
          float2 rs[4];
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const float2 y2 = fma2(make_float2(t[c], t[c + 1]), sc2, nr2);
            const float2 pp = live ? make_float2(ex2_approx(y2.x), ex2_approx(y2.y)) : make_float2(0.f, 0.f);
            rs[(c >> 1) & 3] = (c < 8) ? pp : add2(rs[(c >> 1) & 3], pp);
            pk[c >> 1] = pack_bf16x2(pp.x, pp.y);
          }
          const float2 r2 = add2(add2(rs[0], rs[1]), add2(rs[2], rs[3]));
          l += r2.x + r2.y;
          tmem_st_32x32b_x16(tm + kTmemP + pb * (kBN / 2), pk);  // row h, 32 bf16 = 16 columns
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&p_full[pb]);
        }
      } else {
        // ---- p sweep: P = 2^(t * sc - lse2) summed over heads h < H, divided by H.  Blocks
        // alternate between the two CTAs (both computed the same S).
        const int blk = blk_of(q);
        if ((blk & 1) == static_cast<int>(rank)) {
          const bool live = ok && head_ok && lse2 != -INFINITY;
          float v[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) v[c] = live ? ex2_approx(fmaf(t[c], sc, -lse2)) : 0.f;
          // butterfly reduce-scatter over the warp: lane L ends with column L summed over the
          // warp's 32 heads
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
          float* red = sRed + wg * 128;
          red[wq * 32 + lane] = v[0];
          named_bar_sync(bar_red, 128);
          if (wq == 0 && ok) {
            const float tot = red[lane] + red[32 + lane] + red[64 + lane] + red[96 + lane];
            const int slot2 = e0 + blk * kBN + lane;
            if (slot2 < e1) p.p_sel[static_cast<size_t>(row) * p.k + slot2] = ((vm >> lane) & 1u) ? tot / p.H : 0.f;
          }
        }
      }
    }
    if (!fin) finish();
    if (staged) {  // the staged rows to HBM, whole rows per warp
      named_bar_sync(kBarFin, kSoftmaxThreads);
      if (nblk > 0) {
        if (p.fuse2) {
          const int hb = 64 * (split ^ 1);  // the heads this CTA exports
          const int nrows = max(0, min(64, p.H - hb));
          float* dst0 = p.part_o + (static_cast<size_t>(split) * rows_h + static_cast<size_t>(row) * p.H + hb) * kDV +
                        static_cast<int>(rank) * kDvCta;
          for (int f = threadIdx.x; f < nrows * (kDvCta / 4); f += kSoftmaxThreads) {
            const int r2 = f / (kDvCta / 4), c = f % (kDvCta / 4);
            *reinterpret_cast<float4*>(dst0 + static_cast<size_t>(r2) * kDV + 4 * c) =
                *reinterpret_cast<const float4*>(sKV + r2 * kPitchF + 16 * c);
          }
        } else {
          __nv_bfloat16* dst0 = p.out + static_cast<size_t>(row) * p.H * kDV + static_cast<int>(rank) * kDvCta;
          for (int f = threadIdx.x; f < p.H * (kDvCta / 8); f += kSoftmaxThreads) {
            const int r2 = f / (kDvCta / 8), c = f % (kDvCta / 8);
            *reinterpret_cast<uint4*>(dst0 + static_cast<size_t>(r2) * kDV + 8 * c) =
                *reinterpret_cast<const uint4*>(sKV + r2 * kPitchB + 16 * c);
          }
        }
      }
    }

    // p emission: slots past the effective length are empty (p = 0)
    if (p.p_sel != nullptr && rank == 0) {
      for (int x2 = e0 + nblk * kBN + static_cast<int>(threadIdx.x); x2 < e1; x2 += kSoftmaxThreads)
        p.p_sel[static_cast<size_t>(row) * p.k + x2] = 0.f;
    }
    if (nblk == 0 && head_ok && !(p.fuse2 && own_head)) {  // no valid entry in this split
      const uint32_t o_cols = static_cast<uint32_t>(wg * (kDvCta / 2));
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
    if (p.fuse2) {
      // ---- combine with the other split: its exports are visible after the cluster barrier
      // (release/acquire at cluster scope); every thread of all four CTAs takes it once here
      // (the other roles at the end).  out = w_own * O_own + w_other * O_other, w = e^(lse - lse_all).
      tc_fence_before();
      __syncwarp();
      cluster_barrier();
      // the other split's export of this CTA's heads into the import tile, whole rows per warp
      const int hb = 64 * split;
      const int nrows = max(0, min(64, p.H - hb));
      {
        const float* src0 = p.part_o + (static_cast<size_t>(split ^ 1) * rows_h + static_cast<size_t>(row) * p.H + hb) * kDV +
                            static_cast<int>(rank) * kDvCta;
        for (int f = threadIdx.x; f < nrows * (kDvCta / 4); f += kSoftmaxThreads) {
          const int r2 = f / (kDvCta / 4), c = f % (kDvCta / 4);
          *reinterpret_cast<float4*>(sKV + r2 * kPitchF + 16 * c) =
              *reinterpret_cast<const float4*>(src0 + static_cast<size_t>(r2) * kDV + 4 * c);
        }
      }
      named_bar_sync(kBarFin, kSoftmaxThreads);
      if (own_head) {  // warp-uniform (a warp covers 32 heads of one 64-head half)
        const float lse_o = head_ok ? p.part_lse[static_cast<size_t>(split ^ 1) * rows_h + orow] : -INFINITY;
        const float lse_m = (ok && nblk > 0 && head_ok) ? lse2 * kLn2 : -INFINITY;  // natural log
        const float mx = fmaxf(lse_m, lse_o);
        const float em = lse_m == -INFINITY ? 0.f : expf(lse_m - mx);
        const float eo = lse_o == -INFINITY ? 0.f : expf(lse_o - mx);
        const float den = em + eo;
        const float wm = den > 0.f ? em / den * own_inv_l : 0.f;  // own O is not yet normalised
        const float wo = den > 0.f ? eo / den : 0.f;
        const uint32_t o_cols = static_cast<uint32_t>(wg * (kDvCta / 2));
        const uint8_t* other = sKV + (h & 63) * kPitchF;                              // import tile row
        uint8_t* orow_t = sKV + kOffOutTile + (h & 63) * kPitchB + o_cols * 2;  // output tile row
        const bool need_tm = __any_sync(0xFFFFFFFFu, em > 0.f);  // tcgen05.ld is warp-collective
        if (need_tm) tc_fence_after();
#pragma unroll 1
        for (int c0 = 0; c0 < kDvCta / 2; c0 += 16) {
          uint32_t o[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) o[c] = 0u;
          if (need_tm) {
            tmem_ld_32x32b_x16(tm + kTmemO + o_cols + c0, o);
            tmem_ld_wait();
          }
          if (!head_ok) continue;
          float r[16];
#pragma unroll
          for (int c = 0; c < 16; c += 4) {
            const float4 u = wo > 0.f ? *reinterpret_cast<const float4*>(other + (o_cols + c0 + c) * 4)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
            r[c] = fmaf(wo, u.x, em > 0.f ? wm * __uint_as_float(o[c]) : 0.f);
            r[c + 1] = fmaf(wo, u.y, em > 0.f ? wm * __uint_as_float(o[c + 1]) : 0.f);
            r[c + 2] = fmaf(wo, u.z, em > 0.f ? wm * __uint_as_float(o[c + 2]) : 0.f);
            r[c + 3] = fmaf(wo, u.w, em > 0.f ? wm * __uint_as_float(o[c + 3]) : 0.f);
          }
          uint4 w0, w1;
          w0.x = pack_bf16x2(r[0], r[1]);
          w0.y = pack_bf16x2(r[2], r[3]);
          w0.z = pack_bf16x2(r[4], r[5]);
          w0.w = pack_bf16x2(r[6], r[7]);
          w1.x = pack_bf16x2(r[8], r[9]);
          w1.y = pack_bf16x2(r[10], r[11]);
          w1.z = pack_bf16x2(r[12], r[13]);
          w1.w = pack_bf16x2(r[14], r[15]);
          uint4* dst = reinterpret_cast<uint4*>(orow_t + c0 * 2);
          dst[0] = w0;
          dst[1] = w1;
        }
        if (head_ok && rank == 0 && wg == 0 && p.lse) p.lse[orow] = den > 0.f ? mx + logf(den) : -INFINITY;
      }
      named_bar_sync(kBarFin, kSoftmaxThreads);
      __nv_bfloat16* dst0 = p.out + (static_cast<size_t>(row) * p.H + hb) * kDV + static_cast<int>(rank) * kDvCta;
      for (int f = threadIdx.x; f < nrows * (kDvCta / 8); f += kSoftmaxThreads) {
        const int r2 = f / (kDvCta / 8), c = f % (kDvCta / 8);
        *reinterpret_cast<uint4*>(dst0 + static_cast<size_t>(r2) * kDV + 8 * c) =
            *reinterpret_cast<const uint4*>(sKV + kOffOutTile + r2 * kPitchB + 16 * c);
      }
    }
  }
done:
  if (p.fuse2 && warp >= kMmaWarp) {  // the softmax roles took this one above
    __syncwarp();
    cluster_barrier();
  }
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
