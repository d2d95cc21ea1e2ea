// Sparse attention in MLA's MQA mode over the top-k selected latents ("DeepSeek-V3.2"
// analysis page, sec. 1.1, eq. (2) and the MQA-mode paragraph; renormalised form eq. (19)),
// with the optional head-summed target p ("DSA Continued Pre-Training", Stage 1/2).
//
// One CTA per (query row, half of the value dims, KV split).  Every gathered latent entry
// (d_qk bf16) is shared by all query heads: heads run along M = 128 TMEM lanes, so one
// thread of the softmax warpgroup owns one head's row of S and its softmax state.
//   S = Q K^T   : tcgen05 kind::f16, A = Q (128 x d_qk, K-major, SW128, resident in smem),
//                 B = gathered block (32 entries x d_qk, K-major, SW128), N = 32
//   O += P V    : A = P (128 x 32 bf16, K-major, SW64, written by the softmax threads),
//                 B = the same gathered block read MN-major (value dims contiguous), N = 256
// O (fp32, 256 columns) and a double-buffered S (2 x 32 columns) live in TMEM.  The fp32
// accumulator of all 512 value dims would fill the whole TMEM, so the value dims are split
// over two CTAs that both compute S.
//
// Softmax is online with lazy rescaling: the running reference max m only moves (and O is
// rescaled in TMEM) when a block's max exceeds it by more than 2^8, so P <= 256 stays exact
// in bf16 range; the final 1/l and lse use the same reference.
// Roles: warps 0-3 softmax/epilogue, warp 4 TMA(Q) + MMA issue + TMEM alloc, warps 5-8
// gather producers (cp.async 16 B, written in the swizzled layout).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace dsa {
namespace mla {

constexpr int kBN = 32;       // selected entries per block
constexpr int kStages = 2;    // gathered blocks in flight
constexpr int kThreads = 288; // 9 warps
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleLog2 = 8.0f;

struct Params {
  const __nv_bfloat16* q;  // [rows][H][d_qk] (read directly by the 576-d pair kernel)
  const __nv_bfloat16* kv;
  const int32_t* idx;
  __nv_bfloat16* out;   // final output (n_split == 1, or fuse2)
  float* lse;           // nullable (n_split == 1, or fuse2)
  float* p_sel;         // nullable
  float* part_o;        // [n_split][rows][H][d_v] fp32 (n_split > 1)
  float* part_lse;      // [n_split][rows][H]       fp32 (n_split > 1)
  int B, Lq, Lk, H, k;
  int n_split, per_split;  // entries of the idx row per split (multiple of kBN)
  float scale_log2;        // softmax scale * log2(e)
  int fuse2;               // 576-d pair kernel, n_split == 2: both splits of a row form one
                           // cluster of four and combine in the kernel (no combine launch)
  int dense;               // dense causal attention: no idx, slot j is position j for j <= t,
                           // k == Lk (the dense warm-up's main attention and its target p)
  // Paged decode cache (576-d kernel; nullable block_table): latent s of sequence b is row
  // block_table[b * max_pages + s / page_size] * page_size + s % page_size of kv, and only
  // s < seq_lens[b] are valid.  kv_rows: rows of the kv tensor (one past is the zero-fill row).
  const int32_t* block_table;
  const int32_t* seq_lens;
  int page_size, max_pages, num_pages;
  int kv_rows;
};

// Valid latent positions of sequence b: [0, Lk), or [0, seq_lens[b]) for a paged cache.
__device__ __forceinline__ int row_len(const Params& p, int b) {
  return p.seq_lens ? min(max(__ldg(p.seq_lens + b), 0), p.Lk) : p.Lk;
}

// Row of kv holding latent s of sequence b; kv_rows (one past the tensor, zero-filled by the
// TMA) for an empty slot.
__device__ __forceinline__ int kv_row(const Params& p, int b, int len_b, int s) {
  if (static_cast<unsigned>(s) >= static_cast<unsigned>(len_b)) return p.kv_rows;
  if (p.block_table == nullptr) return b * p.Lk + s;
  const int page = __ldg(p.block_table + static_cast<size_t>(b) * p.max_pages + s / p.page_size);
  if (static_cast<unsigned>(page) >= static_cast<unsigned>(p.num_pages)) {
    record_bad_index();
    return p.kv_rows;
  }
  return page * p.page_size + s % p.page_size;
}

// Query row served by the r-th row of the grid: in dense mode the latest (longest) rows go
// first, so that the shortest ones fill the tail.
__device__ __forceinline__ int work_row(const Params& p, int r) { return p.dense ? p.B * p.Lq - 1 - r : r; }

// Latent position of selection slot `slot` of a row: the caller's index, or the slot itself in
// dense mode.
__device__ __forceinline__ int slot_position(const Params& p, const int32_t* idx_row, int slot) {
  return p.dense ? slot : __ldg(idx_row + slot);
}

// Dense mode: slots [e0, e1) of row `row` that hold visible positions (s <= t).
__device__ __forceinline__ int dense_len(const Params& p, int row, int e0, int e1) {
  const int t = (row % p.Lq) + p.Lk - p.Lq;
  return max(0, min(e1, t + 1) - e0);
}

template <int D_QK, int D_V>
struct Cfg {
  static constexpr int kBoxes = (D_QK + 63) / 64;        // 64-dim (128 B) column boxes
  static constexpr int kDvCta = D_V > 256 ? 256 : D_V;   // value dims per CTA
  static constexpr int kNdv = D_V / kDvCta;              // CTAs across the value dims
  static constexpr int kQBox = 128 * 128;                // 128 heads x 128 B
  static constexpr int kKvBox = kBN * 128;               // 32 entries x 128 B
  static constexpr int kKvStage = kBoxes * kKvBox;
  static constexpr int kChunksPerRow = D_QK * 2 / 16;    // 16-byte chunks of one latent
  static constexpr int kKSteps = D_QK / 16;
  static constexpr int kTmemCols = (kDvCta + 2 * kBN) <= 128 ? 128 : (kDvCta + 2 * kBN) <= 256 ? 256 : 512;
  static constexpr uint32_t kIdescQK = make_idesc(1, 1, false, false, 128, kBN);
  static constexpr uint32_t kIdescPV = make_idesc(1, 1, false, true, 128, kDvCta);
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = kOffQ + kBoxes * kQBox;
  static constexpr int kOffP = kOffKV + kStages * kKvStage;
  static constexpr int kOffRed = kOffP + 128 * kBN * 2;
  static constexpr int kOffBar = kOffRed + 4 * 32 * 4;
  static constexpr int kOffMisc = kOffBar + 16 * 8;
  static constexpr int kSmemBytes = kOffMisc + 64 + 1024;
  static_assert(D_QK % 16 == 0 && D_V % 64 == 0, "dims");
  static_assert(kDvCta % 64 == 0 && kDvCta <= 256, "PV N");
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Steps of a CTA: n_main attention blocks, then (p emission) the blocks this CTA sweeps again.
struct Steps {
  int n_main, n_p, nd, hv;
  __device__ __forceinline__ int total() const { return n_main + n_p; }
  __device__ __forceinline__ bool is_p(int q) const { return q >= n_main; }
  __device__ __forceinline__ int block(int q) const { return q < n_main ? q : hv + nd * (q - n_main); }
};

template <int D_QK, int D_V>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_mla_kernel(const __grid_constant__ CUtensorMap tm_q, const Params p) {
  using C = Cfg<D_QK, D_V>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sKV = smem + C::kOffKV;
  uint8_t* sP = smem + C::kOffP;
  float* sRed = reinterpret_cast<float*>(smem + C::kOffRed);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* kv_full = bars;       // [2]
  uint64_t* kv_empty = bars + 2;  // [2]
  uint64_t* s_full = bars + 4;    // [2]
  uint64_t* s_empty = bars + 6;   // [2]
  uint64_t* q_full = bars + 8;
  uint64_t* p_full = bars + 9;
  uint64_t* o_done = bars + 10;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  int* s_len = reinterpret_cast<int*>(smem + C::kOffMisc + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // CTA -> (query row, value-dim half, split)
  const int hv = blockIdx.x % C::kNdv;
  const int split = (blockIdx.x / C::kNdv) % p.n_split;
  const int row = work_row(p, blockIdx.x / (C::kNdv * p.n_split));
  const int b = row / p.Lq;
  const int32_t* idx_row = p.dense ? nullptr : p.idx + static_cast<size_t>(row) * p.k;
  const int e0 = split * p.per_split;
  const int e1 = min(p.k, e0 + p.per_split);

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kv_full[i], 128);
      mbar_init(&kv_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 128);
    }
    mbar_init(q_full, 1);
    mbar_init(p_full, 128);
    mbar_init(o_done, 1);
    *abort_flag = 0;
    *s_len = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  pdl_launch_dependents();
  if (warp == 4) tmem_alloc(tmem_slot, C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // first global access below
  const uint32_t tmem_o = tmem_base;
  const uint32_t tmem_s = tmem_base + C::kDvCta;

  // Effective length: slots after the last valid one in [e0, e1) need no work.
  if (!p.dense) {
    int last = -1;
    for (int x = e0 + static_cast<int>(threadIdx.x); x < e1; x += kThreads)
      if (__ldg(idx_row + x) >= 0) last = x;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) last = max(last, __shfl_xor_sync(0xFFFFFFFFu, last, o));
    if (lane == 0 && last >= 0) atomicMax(s_len, last - e0 + 1);
    __syncthreads();
  }
  const int len = p.dense ? dense_len(p, row, e0, e1) : *s_len;
  const int nblk = (len + kBN - 1) / kBN;
  Steps st;
  st.n_main = nblk;
  st.nd = C::kNdv;
  st.hv = hv;
  st.n_p = (p.p_sel != nullptr && nblk > hv) ? (nblk - hv + C::kNdv - 1) / C::kNdv : 0;

  if (warp == 4) {
    // ------------------------------------------------------------------ TMA + MMA issuer
    if (lane == 0 && nblk > 0) {
      tma_prefetch_desc(&tm_q);
      mbar_arrive_expect_tx(q_full, C::kBoxes * C::kQBox);
      for (int bx = 0; bx < C::kBoxes; ++bx)
        tma_load_2d(sQ + bx * C::kQBox, &tm_q, q_full, bx * 64, row * p.H);
      if (!mbar_wait(q_full, 0, abort_flag, 20)) goto done;
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t p_addr = smem_u32(sP);
      auto issue_s = [&](int q) -> bool {
        const int sb = q & 1;
        const uint32_t ph = (q >> 1) & 1;
        if (!mbar_wait(&kv_full[sb], ph, abort_flag, 21)) return false;
        if (!mbar_wait(&s_empty[sb], ph ^ 1, abort_flag, 22)) return false;
        tc_fence_after();
        const uint32_t kv_addr = smem_u32(sKV + sb * C::kKvStage);
#pragma unroll
        for (int kk = 0; kk < C::kKSteps; ++kk) {
          const int bx = kk >> 2, kin = kk & 3;
          const uint64_t a = make_smem_desc(q_addr + bx * C::kQBox + kin * 32, 16, 1024, kSw128);
          const uint64_t bd = make_smem_desc(kv_addr + bx * C::kKvBox + kin * 32, 16, 1024, kSw128);
          mma_f16_ss(tmem_s + sb * kBN, a, bd, C::kIdescQK, kk > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[sb]);
        if (st.is_p(q)) mma_commit(&kv_empty[sb]);  // no PV reads this block
        return true;
      };
      const int total = st.total();
      if (!issue_s(0)) goto done;
      for (int q = 0; q < total; ++q) {
        if (q + 1 < total && !issue_s(q + 1)) goto done;
        if (st.is_p(q)) continue;
        // O += P V for main block q
        if (!mbar_wait(p_full, q & 1, abort_flag, 23)) goto done;
        tc_fence_after();
        const int sb = q & 1;
        const uint32_t v_addr = smem_u32(sKV + sb * C::kKvStage) + (hv * C::kDvCta / 64) * C::kKvBox;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint64_t a = make_smem_desc(p_addr + kk * 32, 16, 512, kSw64);
          const uint64_t bd = make_smem_desc(v_addr + kk * 16 * 128, C::kKvBox, 1024, kSw128);
          mma_f16_ss(tmem_o, a, bd, C::kIdescPV, (q > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&kv_empty[sb]);
        mma_commit(o_done);
      }
    }
  } else if (warp >= 5) {
    // ------------------------------------------------------------------ gather producers
    const int pt = threadIdx.x - 160;  // 0..127
    const __nv_bfloat16* kv_seq = p.kv + static_cast<size_t>(b) * p.Lk * D_QK;
    const int total = st.total();
    for (int q = 0; q < total; ++q) {
      const int sb = q & 1;
      const uint32_t ph = (q >> 1) & 1;
      if (!mbar_wait(&kv_empty[sb], ph ^ 1, abort_flag, 24)) break;
      const int blk = st.block(q);
      const uint32_t dst = smem_u32(sKV + sb * C::kKvStage);
      for (int c = pt; c < kBN * C::kChunksPerRow; c += 128) {
        const int r = c / C::kChunksPerRow;
        const int ch = c - r * C::kChunksPerRow;
        const int slot = e0 + blk * kBN + r;
        const int s = (slot < e0 + len) ? slot_position(p, idx_row, slot) : -1;
        const bool valid = static_cast<unsigned>(s) < static_cast<unsigned>(p.Lk);
        if (s >= p.Lk) record_bad_index();
        const __nv_bfloat16* srcp = kv_seq + static_cast<size_t>(valid ? s : 0) * D_QK + ch * 8;
        const uint32_t off = (ch >> 3) * C::kKvBox + swizzled_offset(r, ch & 7, 128);
        cp_async_16(dst + off, srcp, valid);
      }
      cp_async_commit();
      cp_async_wait_group<0>();
      fence_proxy_async_smem();
      mbar_arrive(&kv_full[sb]);
    }
  } else {
    // ------------------------------------------------------------------ softmax / epilogue
    const int h = threadIdx.x;  // head row 0..127 (warp w owns TMEM lanes 32w..32w+31)
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    float m_ref = -INFINITY;  // running reference max (log2 domain)
    float l = 0.f;
    bool ok = true;
    const int total = st.total();
    float lse2 = -INFINITY;
    for (int q = 0; q < total; ++q) {
      // On an expired wait (ok == false) the loop keeps running without touching TMEM, so
      // every thread still reaches the p-emission named barriers.
      const int sb = q & 1;
      const uint32_t ph = (q >> 1) & 1;
      const int blk = st.block(q);
      const int slot = e0 + blk * kBN + lane;
      const int sidx = (slot < e0 + len) ? slot_position(p, idx_row, slot) : -1;
      const bool svalid = static_cast<unsigned>(sidx) < static_cast<unsigned>(p.Lk);
      const uint32_t vmask = __ballot_sync(0xFFFFFFFFu, svalid);
      if (ok && !mbar_wait(&s_full[sb], ph, abort_flag, 25)) ok = false;
      ok = __all_sync(0xFFFFFFFFu, ok);  // TMEM accesses below are warp-collective
      uint32_t v[32];
      if (ok) {
        tc_fence_after();
        tmem_ld_32x32b_x32(tmem_s + sb * kBN + lane_off, v);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&s_empty[sb]);
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) v[c] = 0u;
      }
      float x[32];
#pragma unroll
      for (int c = 0; c < 32; ++c)
        x[c] = ((vmask >> c) & 1u) ? __uint_as_float(v[c]) * p.scale_log2 : -INFINITY;

      if (!st.is_p(q)) {
        if (!ok) continue;
        float bm = -INFINITY;
#pragma unroll
        for (int c = 0; c < 32; ++c) bm = fmaxf(bm, x[c]);
        // P and O of block q-1 must be consumed before P is rewritten or O rescaled
        if (q > 0) {
          const bool got = mbar_wait(o_done, (q - 1) & 1, abort_flag, 26);
          ok = __all_sync(0xFFFFFFFFu, got);
          if (!ok) continue;
        }
        tc_fence_after();
        // The reference max moves per head row, but tcgen05.ld/st are warp-collective
        // (.sync.aligned): when any row of the warp rescales, the whole warp walks O and
        // rows that keep their reference multiply by 1.
        const bool move = bm > m_ref + kRescaleLog2;
        const bool scale_o = move && q > 0 && m_ref != -INFINITY;
        const float f = scale_o ? exp2f(m_ref - bm) : 1.f;
        if (__any_sync(0xFFFFFFFFu, scale_o)) {
#pragma unroll 1
          for (int c0 = 0; c0 < C::kDvCta; c0 += 16) {
            uint32_t o[16];
            tmem_ld_32x32b_x16(tmem_o + lane_off + c0, o);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 16; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * f);
            tmem_st_32x32b_x16(tmem_o + lane_off + c0, o);
          }
          tmem_st_wait();
        }
        l *= f;
        if (move) m_ref = bm;
        uint32_t pk[16];
        float rs = 0.f;
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float p0 = ((vmask >> c) & 1u) ? exp2f(x[c] - m_ref) : 0.f;
          const float p1 = ((vmask >> (c + 1)) & 1u) ? exp2f(x[c + 1] - m_ref) : 0.f;
          rs += p0 + p1;  // fp32 probabilities: the normaliser and lse keep fp32 accuracy
          pk[c >> 1] = pack_bf16x2(p0, p1);
        }
        l += rs;
        // P row h: 64 bytes = four 16-byte chunks, 64B-swizzled K-major layout
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const uint32_t off = swizzled_offset(h, ch, 64);
          uint4 val = make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
          *reinterpret_cast<uint4*>(sP + off) = val;
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(p_full);
        if (q == st.n_main - 1) {
          // ---- final O: wait for the last PV, normalise, store
          const bool got = mbar_wait(o_done, q & 1, abort_flag, 27);
          ok = __all_sync(0xFFFFFFFFu, got);
          if (!ok) continue;
          tc_fence_after();
          const float inv_l = l > 0.f ? 1.f / l : 0.f;
          lse2 = l > 0.f ? m_ref + log2f(l) : -INFINITY;
          const bool head_ok = h < p.H;
          const size_t orow = static_cast<size_t>(row) * p.H + h;
#pragma unroll 1
          for (int c0 = 0; c0 < C::kDvCta; c0 += 16) {
            uint32_t o[16];
            tmem_ld_32x32b_x16(tmem_o + lane_off + c0, o);
            tmem_ld_wait();
            if (!head_ok) continue;
            const int col = hv * C::kDvCta + c0;
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
              uint4* dst = reinterpret_cast<uint4*>(p.out + orow * D_V + col);
              dst[0] = w0;
              dst[1] = w1;
            } else {
              float4* dst = reinterpret_cast<float4*>(
                  p.part_o + (static_cast<size_t>(split) * p.B * p.Lq * p.H + orow) * D_V + col);
#pragma unroll
              for (int c = 0; c < 16; c += 4)
                dst[c / 4] = make_float4(__uint_as_float(o[c]) * inv_l, __uint_as_float(o[c + 1]) * inv_l,
                                         __uint_as_float(o[c + 2]) * inv_l, __uint_as_float(o[c + 3]) * inv_l);
            }
          }
          if (head_ok && hv == 0) {
            const float lse_nat = lse2 * kLn2;
            if (p.n_split == 1) {
              if (p.lse) p.lse[orow] = lse_nat;
            } else {
              p.part_lse[static_cast<size_t>(split) * p.B * p.Lq * p.H + orow] = lse_nat;
            }
          }
        }
      } else {
        // ---- p emission: P = exp2(x - lse2) summed over heads h < H, divided by H
        float pv[32];
#pragma unroll
        for (int c = 0; c < 32; ++c)
          pv[c] = (ok && h < p.H && ((vmask >> c) & 1u)) ? exp2f(x[c] - lse2) : 0.f;
        // reduce-scatter across the warp: lane c ends with the warp's sum for column c
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
          const bool upper = (lane & off) != 0;
#pragma unroll
          for (int i2 = 0; i2 < off; ++i2) {
            const float send = upper ? pv[i2] : pv[i2 + off];
            const float keep = upper ? pv[i2 + off] : pv[i2];
            pv[i2] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, off);
          }
        }
        named_bar_sync(2, 128);  // previous block's partials have been consumed
        sRed[warp * 32 + lane] = pv[0];
        named_bar_sync(2, 128);
        if (warp == 0) {
          const float tot = sRed[lane] + sRed[32 + lane] + sRed[64 + lane] + sRed[96 + lane];
          const int slot2 = e0 + blk * kBN + lane;
          if (slot2 < e1) p.p_sel[static_cast<size_t>(row) * p.k + slot2] = svalid ? tot / p.H : 0.f;
        }
      }
    }
    // p emission: slots past the effective length are empty (p = 0)
    if (p.p_sel != nullptr && hv == 0) {
      for (int x2 = e0 + nblk * kBN + h; x2 < e1; x2 += 128) p.p_sel[static_cast<size_t>(row) * p.k + x2] = 0.f;
    }
    if (nblk == 0 && h < p.H) {  // no valid entry in this split
      const size_t orow = static_cast<size_t>(row) * p.H + h;
      for (int c = 0; c < C::kDvCta; ++c) {
        const int col = hv * C::kDvCta + c;
        if (p.n_split == 1)
          p.out[orow * D_V + col] = __float2bfloat16_rn(0.f);
        else
          p.part_o[(static_cast<size_t>(split) * p.B * p.Lq * p.H + orow) * D_V + col] = 0.f;
      }
      if (hv == 0) {
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
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// Split-KV combine: out = sum_s exp(lse_s - lse) * O_s,  lse = ln sum_s exp(lse_s).
// Split-KV combine: out[rh, :] = sum_s w_s * part_o[s, rh, :] with w_s = exp(lse_s - lse_all),
// lse_all = log sum_s exp(lse_s).  One warp per (row, head): the splits' lse values are
// reduced with shuffles and every lane streams D_V / 32 contiguous columns of each split, so a
// warp issues all of its loads at once.
constexpr int kCombineWarps = 8;

template <int D_V>
__global__ void __launch_bounds__(kCombineWarps * 32)
    combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse, int n_split,
                   int rows_h, __nv_bfloat16* __restrict__ out, float* lse) {
  constexpr int kPer = D_V / 32;  // columns per lane
  static_assert(kPer % 2 == 0, "D_V");
  pdl_launch_dependents();
  pdl_wait();
  const int rh = blockIdx.x * kCombineWarps + static_cast<int>(threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (rh >= rows_h) return;  // warp-uniform
  float m = -INFINITY;
  for (int s = lane; s < n_split; s += 32) m = fmaxf(m, part_lse[static_cast<size_t>(s) * rows_h + rh]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  float denom = 0.f;
  for (int s = lane; s < n_split; s += 32) {
    const float ls = part_lse[static_cast<size_t>(s) * rows_h + rh];
    denom += (ls == -INFINITY) ? 0.f : expf(ls - m);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) denom += __shfl_xor_sync(0xFFFFFFFFu, denom, o);
  const float lse_all = (denom > 0.f) ? m + logf(denom) : -INFINITY;
  float acc[kPer];
#pragma unroll
  for (int c = 0; c < kPer; ++c) acc[c] = 0.f;
#pragma unroll 2
  for (int s = 0; s < n_split; ++s) {
    const float ls = part_lse[static_cast<size_t>(s) * rows_h + rh];
    if (ls == -INFINITY) continue;  // warp-uniform
    const float w = expf(ls - lse_all);
    const float* src = part_o + (static_cast<size_t>(s) * rows_h + rh) * D_V + lane * kPer;
#pragma unroll
    for (int c = 0; c < kPer; c += 2) {
      const float2 v = *reinterpret_cast<const float2*>(src + c);
      acc[c] = fmaf(w, v.x, acc[c]);
      acc[c + 1] = fmaf(w, v.y, acc[c + 1]);
    }
  }
  __nv_bfloat16* dst = out + static_cast<size_t>(rh) * D_V + lane * kPer;
#pragma unroll
  for (int c = 0; c < kPer; c += 2) {
    const __nv_bfloat162 pr = __floats2bfloat162_rn(acc[c], acc[c + 1]);
    *reinterpret_cast<__nv_bfloat162*>(dst + c) = pr;
  }
  if (lane == 0 && lse != nullptr) lse[rh] = lse_all;
}

}  // namespace mla
}  // namespace dsa
