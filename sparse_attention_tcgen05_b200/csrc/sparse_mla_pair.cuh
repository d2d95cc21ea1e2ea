// Sparse attention in MLA's MQA mode over the top-k selected latents ("DeepSeek-V3.2" analysis
// page, sec. 1.1, eq. (2) and the MQA-mode paragraph; renormalised form eq. (19)), with the
// optional head-summed target p ("DSA Continued Pre-Training", Stage 1/2), for the 576-d
// latent (512 value + 64 rope dims) shared by up to 128 query heads.
//
// A cluster of two CTAs serves one (query row, KV split).  The 576 latent dims are split:
//   rank 0: QK dims [0, 256)   (Q boxes 0-3),  value dims [0, 256)
//   rank 1: QK dims [256, 576) (Q boxes 4-8),  value dims [256, 512)
// so each CTA gathers only its own dims of every selected entry (each latent byte is read
// once per pair) and holds only its slice of Q.  Each CTA computes a partial S over its dims
// on the tensor cores (tcgen05 kind::f16, heads on the 128 TMEM lanes), ships the 128 x 32
// fp32 partial to its peer with asynchronous remote stores (st.async, counted on the peer's
// mbarrier), and adds the peer's partial: both CTAs then hold the
// same full S (fp32 addition commutes), run the same online softmax and accumulate O for
// their own 256 value dims in TMEM.
//
// Roles per CTA (13 warps):
//   warps 0-7   softmax/epilogue: two warpgroups on the same 128 TMEM lanes (thread = head
//               row); warpgroup g owns columns [16g, 16g+16) of every 32-entry block and
//               value columns [128g, 128g+128) of this CTA's half
//   warp 8      TMA (Q) + MMA issue (one thread) + TMEM allocation
//   warps 9-12  gather: 16-byte cp.async straight into the 128B-swizzled K-major tiles,
//               completion tracked by the hardware (cp.async.mbarrier.arrive.noinc)
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

constexpr int kBN = 32;          // selected entries per block
constexpr int kHalf = kBN / 2;   // columns per softmax warpgroup
constexpr int kStages = 4;       // gather ring
constexpr int kThreads = 416;
constexpr int kSoftmaxThreads = 256;
constexpr int kMmaWarp = 8;
constexpr int kProducerThread0 = 288;
constexpr int kDQK = 576, kDV = 512, kDvCta = 256;
constexpr int kQBox = 128 * 128;       // 128 rows x 128 B
constexpr int kKvBox = kBN * 128;      // 32 entries x 128 B
constexpr int kMaxBoxes = 5;
constexpr int kKvStage = kMaxBoxes * kKvBox;
constexpr int kPBytes = 128 * kBN * 2;
constexpr int kXSlot = 128 * kBN * 4;  // one partial S (fp32)
constexpr int kOffQ = 0;
constexpr int kOffKV = kOffQ + kMaxBoxes * kQBox;
constexpr int kOffP = kOffKV + kStages * kKvStage;
constexpr int kOffX = kOffP + 2 * kPBytes;     // 2 slots received from the peer
constexpr int kOffRed = kOffX + 2 * kXSlot;    // [8 warps][16] p partial sums
constexpr int kOffMax = kOffRed + 8 * 16 * 4;  // [2][128] row-max exchange
constexpr int kOffL = kOffMax + 2 * 128 * 4;   // [2][128] normaliser exchange
constexpr int kOffBar = kOffL + 2 * 128 * 4;
constexpr int kNumBars = 2 * kStages + 11;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 64 + 1024;
constexpr int kTmemCols = 512;  // O (256) + 2 x S (32)
constexpr uint32_t kIdescQK = make_idesc(1, 1, false, false, 128, kBN);
constexpr uint32_t kIdescPV = make_idesc(1, 1, false, true, 128, kDvCta);
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleLog2 = 8.0f;
constexpr int kBarSoftmax = 1;  // named barriers of the 256 softmax threads: 1 (per block), 2
static_assert(kSmemBytes <= 232448, "shared memory");

// S = Q K^T over this CTA's NBOX 64-dim boxes: 4 K-steps of 16 per box.  Descriptors are built
// once and advanced through their start-address field.
template <int NBOX>
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_addr, uint32_t kv_addr) {
  const uint64_t qa = make_smem_desc(q_addr, 16, 1024, kSw128);
  const uint64_t kb = make_smem_desc(kv_addr, 16, 1024, kSw128);
#pragma unroll
  for (int kk = 0; kk < NBOX * 4; ++kk) {
    const int bx = kk >> 2, kin = kk & 3;
    mma_f16_ss(d_tmem, qa + static_cast<uint64_t>((bx * kQBox + kin * 32) >> 4),
               kb + static_cast<uint64_t>((bx * kKvBox + kin * 32) >> 4), kIdescQK, kk > 0 ? 1u : 0u);
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    sparse_mla_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + kOffQ;
  uint8_t* sKV = smem + kOffKV;
  uint8_t* sP = smem + kOffP;
  float* sX = reinterpret_cast<float*>(smem + kOffX);
  float* sRed = reinterpret_cast<float*>(smem + kOffRed);
  float* sMax = reinterpret_cast<float*>(smem + kOffMax);
  float* sL = reinterpret_cast<float*>(smem + kOffL);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* kv_full = bars;                 // [kStages] 128 producer arrivals (async)
  uint64_t* kv_empty = bars + kStages;      // [kStages] MMA commit
  uint64_t* s_full = bars + 2 * kStages;    // [2] MMA commit
  uint64_t* s_empty = s_full + 2;           // [2] 256 softmax arrivals
  uint64_t* p_full = s_full + 4;            // [2] 256 softmax arrivals
  uint64_t* o_done = s_full + 6;            // [2] MMA commit (PV of blocks q, q % 2)
  uint64_t* x_full = s_full + 8;            // [2] own expect_tx + the peer's stored bytes
  uint64_t* q_full = s_full + 10;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  int* s_len = reinterpret_cast<int*>(smem + kOffMisc + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int nbox = 4 + static_cast<int>(rank);  // Q/KV boxes this CTA holds
  const int box0 = 4 * static_cast<int>(rank);  // first global 64-dim box

  const int pair = blockIdx.x >> 1;
  const int split = pair % p.n_split;
  const int row = pair / p.n_split;
  const int b = row / p.Lq;
  const int32_t* idx_row = p.idx + static_cast<size_t>(row) * p.k;
  const int e0 = split * p.per_split;
  const int e1 = min(p.k, e0 + p.per_split);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&kv_full[i], 128);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], kSoftmaxThreads);
      mbar_init(&p_full[i], kSoftmaxThreads);
      mbar_init(&o_done[i], 1);
      mbar_init(&x_full[i], 1);
    }
    mbar_init(q_full, 1);
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
  const uint32_t tmem_o = tmem_base;
  const uint32_t tmem_s = tmem_base + kDvCta;

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
  const int n_main = nblk;
  const int total = nblk + ((p.p_sel != nullptr) ? nblk : 0);  // p sweep revisits every block
  auto block_of = [&](int q) { return q < n_main ? q : q - n_main; };

  if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ TMA + MMA issuer
    if (lane == 0 && nblk > 0) {
      tma_prefetch_desc(&tm_q);
      mbar_arrive_expect_tx(q_full, nbox * kQBox);
      for (int bx = 0; bx < nbox; ++bx)
        tma_load_2d(sQ + bx * kQBox, &tm_q, q_full, (box0 + bx) * 64, row * p.H);
      if (!mbar_wait(q_full, 0, abort_flag, 40)) goto done;
      const uint32_t q_addr = smem_u32(sQ);
      const uint64_t p_desc = make_smem_desc(smem_u32(sP), 16, 512, kSw64);
      auto issue_s = [&](int q) -> bool {
        const int st = q % kStages, sb = q & 1;
        if (!mbar_wait(&kv_full[st], (q / kStages) & 1, abort_flag, 41)) return false;
        fence_proxy_async_smem();  // the gathered block was written by cp.async
        if (!mbar_wait(&s_empty[sb], ((q >> 1) & 1) ^ 1, abort_flag, 42)) return false;
        tc_fence_after();
        const uint32_t kv_addr = smem_u32(sKV + st * kKvStage);
        if (rank == 0)
          issue_qk<4>(tmem_s + sb * kBN, q_addr, kv_addr);
        else
          issue_qk<5>(tmem_s + sb * kBN, q_addr, kv_addr);
        mma_commit(&s_full[sb]);
        if (q >= n_main) mma_commit(&kv_empty[st]);  // p sweep: no PV reads this block
        return true;
      };
      if (!issue_s(0)) goto done;
      for (int q = 0; q < total; ++q) {
        if (q + 1 < total && !issue_s(q + 1)) goto done;
        if (q >= n_main) continue;
        const int pb = q & 1;
        if (!mbar_wait(&p_full[pb], (q >> 1) & 1, abort_flag, 43)) goto done;
        tc_fence_after();
        const int st = q % kStages;
        // value dims = local boxes 0-3, read MN-major: 4 chunks of 64 dims at LBO = one box
        const uint64_t v_desc = make_smem_desc(smem_u32(sKV + st * kKvStage), kKvBox, 1024, kSw128);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          mma_f16_ss(tmem_o, p_desc + static_cast<uint64_t>((pb * kPBytes + kk * 32) >> 4),
                     v_desc + static_cast<uint64_t>((kk * 16 * 128) >> 4), kIdescPV,
                     (q > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&kv_empty[st]);
        mma_commit(&o_done[pb]);
      }
    }
  } else if (warp > kMmaWarp) {
    // ------------------------------------------------------------------ gather producers
    // Each block's completion is tracked by the hardware, so the producers run up to kStages
    // blocks ahead without waiting for their own copies.
    const int pt = threadIdx.x - kProducerThread0;  // 0..127
    const __nv_bfloat16* kv_seq = p.kv + static_cast<size_t>(b) * p.Lk * kDQK;
    const int chunks = nbox * 8;  // 16-byte chunks of this CTA's dims per entry
    for (int q = 0; q < total; ++q) {
      const int st = q % kStages;
      const bool got = mbar_wait(&kv_empty[st], ((q / kStages) & 1) ^ 1, abort_flag, 44);
      if (!__all_sync(0xFFFFFFFFu, got)) break;  // the shuffles below need the whole warp
      const int blk = block_of(q);
      const int myslot = e0 + blk * kBN + lane;  // lane r holds the block's r-th index
      const int my_s = (myslot < e0 + len) ? __ldg(idx_row + myslot) : -1;
      const uint32_t dst = smem_u32(sKV + st * kKvStage);
      for (int c = pt; c < kBN * chunks; c += 128) {  // same trip count in every lane
        const int r = c / chunks;
        const int cl = c - r * chunks;
        const int s = __shfl_sync(0xFFFFFFFFu, my_s, r);
        const bool valid = static_cast<unsigned>(s) < static_cast<unsigned>(p.Lk);
        if (s >= p.Lk) record_bad_index();
        const __nv_bfloat16* srcp = kv_seq + static_cast<size_t>(valid ? s : 0) * kDQK + (box0 * 8 + cl) * 8;
        cp_async_16(dst + (cl >> 3) * kKvBox + swizzled_offset(r, cl & 7, 128), srcp, valid);
      }
      cp_async_arrive_noinc(&kv_full[st]);
    }
    cp_async_wait_group<0>();  // nothing of ours may still be landing when the CTA exits
  } else {
    // ------------------------------------------------------------------ softmax / epilogue
    const int wg = warp >> 2;                // column half of each block
    const int h = ((warp & 3) << 5) + lane;  // head row; warp w owns TMEM lanes 32(w%4)..
    const int col0 = wg * kHalf;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t o_cols = static_cast<uint32_t>(wg * (kDvCta / 2));
    // Exchange of partial S: at step q every thread stores its 16 values into slot q % 2 of the
    // peer's receive buffer (row h = 128 B, 16-byte chunk j kept at chunk j ^ (h % 8) so that a
    // warp's accesses spread over all banks).  Two slots suffice without a back-signal: before
    // this CTA reuses a slot (step q + 2) it has received all of the peer's step q + 1 stores,
    // which the peer issues only after it consumed step q.
    const uint32_t peer_recv = map_to_rank(smem_u32(sX), peer);
    const uint32_t peer_x_full = map_to_rank(smem_u32(x_full), peer);
    float m_ref = -INFINITY;  // running reference max (log2 domain), identical in both halves
    float l = 0.f;            // this half's share of the normaliser
    float lse2 = -INFINITY;
    bool ok = true;
    // Every named barrier below is reached by all 256 threads on every step, whatever `ok`
    // says; an expired wait only makes the thread skip TMEM, the peer and the outputs.
    for (int q = 0; q < total; ++q) {
      const int sb = q & 1;
      const uint32_t ph = (q >> 1) & 1;
      const int blk = block_of(q);
      const int slot = e0 + blk * kBN + lane;
      const int sidx = (slot < e0 + len) ? __ldg(idx_row + slot) : -1;
      const bool svalid = static_cast<unsigned>(sidx) < static_cast<unsigned>(p.Lk);
      const uint32_t vmask = __ballot_sync(0xFFFFFFFFu, svalid) >> col0;  // this half's columns
      if (ok && !mbar_wait(&s_full[sb], ph, abort_flag, 45)) ok = false;
      ok = __all_sync(0xFFFFFFFFu, ok);  // TMEM accesses below are warp-collective
      uint32_t v[kHalf];
      float x[kHalf];
      const uint32_t xrow = static_cast<uint32_t>(sb * kXSlot + h * (kBN * 4));
      const uint32_t hsw = static_cast<uint32_t>(h & 7);
      if (ok) {
        tc_fence_after();
        tmem_ld_32x32b_x16(tmem_s + sb * kBN + col0 + lane_off, v);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&s_empty[sb]);
        if (threadIdx.x == 0) mbar_arrive_expect_tx(&x_full[sb], kXSlot);
#pragma unroll
        for (int i = 0; i < kHalf / 4; ++i) {
          const uint32_t j = static_cast<uint32_t>(wg * 4 + i);
          st_async_v4(peer_recv + xrow + ((j ^ hsw) << 4), __uint_as_float(v[4 * i]),
                      __uint_as_float(v[4 * i + 1]), __uint_as_float(v[4 * i + 2]),
                      __uint_as_float(v[4 * i + 3]), peer_x_full + sb * 8);
        }
      } else {
#pragma unroll
        for (int c = 0; c < kHalf; ++c) v[c] = 0u;
      }
      if (ok && !mbar_wait_cluster(&x_full[sb], ph, abort_flag, 47)) ok = false;
      ok = __all_sync(0xFFFFFFFFu, ok);
      float bm = -INFINITY;
      {
        const uint8_t* mine = reinterpret_cast<const uint8_t*>(sX) + xrow;
#pragma unroll
        for (int i = 0; i < kHalf / 4; ++i) {
          const uint32_t j = static_cast<uint32_t>(wg * 4 + i);
          const float4 u = ok ? *reinterpret_cast<const float4*>(mine + ((j ^ hsw) << 4))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
          x[4 * i] = __uint_as_float(v[4 * i]) + u.x;
          x[4 * i + 1] = __uint_as_float(v[4 * i + 1]) + u.y;
          x[4 * i + 2] = __uint_as_float(v[4 * i + 2]) + u.z;
          x[4 * i + 3] = __uint_as_float(v[4 * i + 3]) + u.w;
        }
#pragma unroll
        for (int c = 0; c < kHalf; ++c) {
          x[c] = ((vmask >> c) & 1u) ? x[c] * p.scale_log2 : -INFINITY;
          bm = fmaxf(bm, x[c]);
        }
      }

      if (q < n_main) {
        // row max over the whole block: combine the two halves
        sMax[wg * 128 + h] = bm;
        named_bar_sync(kBarSoftmax, kSoftmaxThreads);
        bm = fmaxf(bm, sMax[(wg ^ 1) * 128 + h]);
        const int pb = q & 1;
        if (ok && q >= 2) {  // P buffer pb was last read by PV(q-2)
          const bool got = mbar_wait(&o_done[pb], ((q - 2) >> 1) & 1, abort_flag, 48);
          ok = __all_sync(0xFFFFFFFFu, got);
        }
        if (ok) {
          // Lazy rescale: the reference max moves only when a block max exceeds it by 2^8.
          // Both halves take the same decision; each walks its 128 value columns of O
          // (tcgen05.ld/st are warp-collective) once PV(q-1) has landed.
          const bool move = bm > m_ref + kRescaleLog2;
          const bool scale_o = move && q > 0 && m_ref != -INFINITY;
          const float f = scale_o ? ex2_approx(m_ref - bm) : 1.f;
          if (__any_sync(0xFFFFFFFFu, scale_o)) {
            const bool got = mbar_wait(&o_done[(q - 1) & 1], ((q - 1) >> 1) & 1, abort_flag, 49);
            ok = __all_sync(0xFFFFFFFFu, got);
            if (ok) {
              tc_fence_after();
#pragma unroll 1
              for (int c0 = 0; c0 < kDvCta / 2; c0 += 16) {
                uint32_t o[16];
                tmem_ld_32x32b_x16(tmem_o + o_cols + lane_off + c0, o);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < 16; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * f);
                tmem_st_32x32b_x16(tmem_o + o_cols + lane_off + c0, o);
              }
              tmem_st_wait();
            }
          }
          l *= f;
          if (move) m_ref = bm;
        }
        if (ok) {
          uint32_t pk[kHalf / 2];
          float rs = 0.f;
#pragma unroll
          for (int c = 0; c < kHalf; c += 2) {
            const float p0 = ((vmask >> c) & 1u) ? ex2_approx(x[c] - m_ref) : 0.f;
            const float p1 = ((vmask >> (c + 1)) & 1u) ? ex2_approx(x[c + 1] - m_ref) : 0.f;
            rs += p0 + p1;
            pk[c >> 1] = pack_bf16x2(p0, p1);
          }
          l += rs;
          uint8_t* pbuf = sP + pb * kPBytes;  // row h: 64 B, 64B-swizzled; this half = chunks 2wg, 2wg+1
          *reinterpret_cast<uint4*>(pbuf + swizzled_offset(h, 2 * wg, 64)) =
              make_uint4(pk[0], pk[1], pk[2], pk[3]);
          *reinterpret_cast<uint4*>(pbuf + swizzled_offset(h, 2 * wg + 1, 64)) =
              make_uint4(pk[4], pk[5], pk[6], pk[7]);
          fence_proxy_async_smem();
          tc_fence_before();
          mbar_arrive(&p_full[pb]);
        }
        if (q == n_main - 1) {
          // ---- final O: total normaliser from both halves, wait for the last PV, store
          sL[wg * 128 + h] = l;
          named_bar_sync(kBarSoftmax + 1, kSoftmaxThreads);
          const float l_tot = (wg == 0) ? l + sL[128 + h] : sL[h] + l;  // same order in both
          if (ok) {
            const bool got = mbar_wait(&o_done[pb], (q >> 1) & 1, abort_flag, 50);
            ok = __all_sync(0xFFFFFFFFu, got);
          }
          if (ok) {
            tc_fence_after();
            const float inv_l = l_tot > 0.f ? 1.f / l_tot : 0.f;
            lse2 = l_tot > 0.f ? m_ref + log2f(l_tot) : -INFINITY;
            const bool head_ok = h < p.H;
            const size_t orow = static_cast<size_t>(row) * p.H + h;
#pragma unroll 1
            for (int c0 = 0; c0 < kDvCta / 2; c0 += 16) {
              uint32_t o[16];
              tmem_ld_32x32b_x16(tmem_o + o_cols + lane_off + c0, o);
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
      } else if ((blk & 1) == static_cast<int>(rank)) {
        // ---- p sweep, blocks alternate between the two CTAs: P = exp2(x - lse2) summed over
        // heads h < H, divided by H; each warpgroup handles its 16 columns
        float pv[kHalf];
#pragma unroll
        for (int c = 0; c < kHalf; ++c)
          pv[c] = (ok && h < p.H && ((vmask >> c) & 1u)) ? ex2_approx(x[c] - lse2) : 0.f;
#pragma unroll
        for (int off = 8; off >= 1; off >>= 1) {  // lane ends with column (lane & 15) summed over
          const bool upper = (lane & off) != 0;   // its 16-lane half, then over the whole warp
#pragma unroll
          for (int i2 = 0; i2 < off; ++i2) {
            const float send = upper ? pv[i2] : pv[i2 + off];
            const float keep = upper ? pv[i2 + off] : pv[i2];
            pv[i2] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, off);
          }
        }
        pv[0] += __shfl_xor_sync(0xFFFFFFFFu, pv[0], 16);
        if (lane < 16) sRed[warp * 16 + lane] = pv[0];
        named_bar_sync(kBarSoftmax, kSoftmaxThreads);
        if ((warp & 3) == 0 && lane < 16 && ok) {
          const int w0 = warp;  // warps w0..w0+3 hold this half's partial sums
          const float tot = sRed[w0 * 16 + lane] + sRed[(w0 + 1) * 16 + lane] + sRed[(w0 + 2) * 16 + lane] +
                            sRed[(w0 + 3) * 16 + lane];
          const int slot2 = e0 + blk * kBN + col0 + lane;
          const bool v2 = (vmask >> lane) & 1u;
          if (slot2 < e1) p.p_sel[static_cast<size_t>(row) * p.k + slot2] = v2 ? tot / p.H : 0.f;
        }
      }
    }
    // p emission: slots past the effective length are empty (p = 0)
    const int st_id = static_cast<int>(threadIdx.x);  // 0..255
    if (p.p_sel != nullptr && rank == 0) {
      for (int x2 = e0 + nblk * kBN + st_id; x2 < e1; x2 += kSoftmaxThreads)
        p.p_sel[static_cast<size_t>(row) * p.k + x2] = 0.f;
    }
    if (nblk == 0 && h < p.H) {  // no valid entry in this split
      const size_t orow = static_cast<size_t>(row) * p.H + h;
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
  // neither CTA may leave while its peer can still copy into its shared memory
  cluster_barrier();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace mla_pair
}  // namespace dsa
