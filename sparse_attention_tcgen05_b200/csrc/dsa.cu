// Host side of the C ABI declared in include/dsa.h: argument validation, launch-shape
// selection, TMA descriptor encoding and kernel launches.  All kernels of the library are
// compiled in this one translation unit so they share the device status word.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>
#include <utility>

#include "../../include/dsa.h"
#include "hisa.cuh"
#include "indexer.cuh"
#include "indexer_bwd.cuh"
#include "indexer_kl.cuh"
#include "masked_mha.cuh"
#include "ptx.cuh"
#include "sparse_mla.cuh"
#include "sparse_mla_pair.cuh"
#include "status.cuh"
#include "topk.cuh"

namespace {

using dsa::g_device_status;

// ------------------------------------------------------------------------------ device info
struct DeviceInfo {
  bool ok = false;
  bool sm100 = false;
  int sms = 0;
};

constexpr int kMaxDevices = 64;
// Per-device facts, looked up once and cached only when the lookup succeeded (a failed lookup,
// e.g. before the context is ready, is retried on the next call).
DeviceInfo g_dev[kMaxDevices];
std::atomic<bool> g_dev_ok[kMaxDevices];
std::mutex g_mu;

dsa_status current_device(DeviceInfo& out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DSA_ERR_CUDA;
  if (!g_dev_ok[dev].load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_dev_ok[dev].load(std::memory_order_relaxed)) {
      int major = 0, minor = 0, sms = 0;
      if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return DSA_ERR_CUDA;
      g_dev[dev].sm100 = (major == 10 && minor == 0);
      g_dev[dev].sms = sms;
      g_dev[dev].ok = true;
      g_dev_ok[dev].store(true, std::memory_order_release);
    }
  }
  if (!g_dev[dev].sm100) return DSA_ERR_NO_SM100;
  out = g_dev[dev];
  return DSA_OK;
}

int sm_count_or_default() {
  DeviceInfo d;
  if (current_device(d) == DSA_OK) return d.sms;
  return 148;
}

// ------------------------------------------------------------------------------ TMA encode
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static std::atomic<EncodeTiledFn> cached{nullptr};
  EncodeTiledFn fn = cached.load(std::memory_order_acquire);
  if (fn) return fn;
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess) {
    fn = reinterpret_cast<EncodeTiledFn>(p);
    cached.store(fn, std::memory_order_release);
  }
  return fn;  // nullptr: looked up again on the next call
}

// 2-D row-major tensor [outer, inner] with `row_bytes` between rows; box [box_outer, box_inner].
bool encode_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner,
               uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
               CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A paged decode cache: key/latent s of sequence b lives in row
// block_table[b * max_pages + s / page_size] * page_size + s % page_size of the page pool, and
// sequence b's context is seq_lens[b] long.
struct Paging {
  const int32_t* block_table;
  const int32_t* seq_lens;
  int page_size, max_pages, num_pages;
};

inline dsa_status launch_result() {
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// Every kernel of the library is launched as a programmatic dependent of the previous launch in
// the stream (see pdl_wait in ptx.cuh), optionally as clusters of `cluster` CTAs.
template <typename... KArgs, typename... Args>
dsa_status launch(void (*kern)(KArgs...), unsigned grid, unsigned block, size_t smem, cudaStream_t stream,
                  unsigned cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  if (cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...) != cudaSuccess) return DSA_ERR_CUDA;
  return launch_result();
}

// ------------------------------------------------------------------------------ indexer
template <int H_I, int D_I, int G>
dsa_status launch_indexer(const void* q, const void* kk, const float* w, float* scores, int B,
                          int Lq, int Lk, int sms, cudaStream_t stream, uint32_t* hist = nullptr,
                          const Paging* pg = nullptr) {
  using Cfg = dsa::indexer::Cfg<H_I, D_I, G>;
  const CUtensorMapSwizzle swz = D_I == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                 : D_I == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                             : CU_TENSOR_MAP_SWIZZLE_32B;
  CUtensorMap tm_q, tm_k;
  if (!encode_2d(&tm_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, D_I, static_cast<uint64_t>(B) * Lq * H_I,
                 D_I, D_I, Cfg::N, swz))
    return DSA_ERR_CUDA;
  const uint64_t k_rows = pg ? static_cast<uint64_t>(pg->num_pages) * pg->page_size : static_cast<uint64_t>(B) * Lk;
  if (k_rows >= INT32_MAX) return DSA_ERR_UNSUPPORTED;
  if (!encode_2d(&tm_k, CU_TENSOR_MAP_DATA_TYPE_UINT8, kk, D_I, k_rows, D_I, D_I, Cfg::kKBox, swz))
    return DSA_ERR_CUDA;
  dsa::indexer::Params p{};
  p.k_rows = static_cast<int>(k_rows);
  if (pg) {
    p.block_table = pg->block_table;
    p.seq_lens = pg->seq_lens;
    p.page_size = pg->page_size;
    p.max_pages = pg->max_pages;
    p.num_pages = pg->num_pages;
  }
  p.w = w;
  p.scores = scores;
  p.hist = hist;
  p.B = B;
  p.Lq = Lq;
  p.Lk = Lk;
  p.n_qg = (Lq + G - 1) / G;
  p.n_kt = (Lk + dsa::indexer::kTileKeys - 1) / dsa::indexer::kTileKeys;
  const long base = static_cast<long>(B) * p.n_qg;
  if (base >= 2L * sms) {
    p.kc = p.n_kt;
  } else {
    // about 16 items per CTA, so that whole items left over at the end cost little
    const long splits = (16L * sms + base - 1) / base;
    p.kc = static_cast<int>(std::max<long>(4, (p.n_kt + splits - 1) / splits));
  }
  p.kc = std::min(p.kc, p.n_kt);
  p.n_kc = (p.n_kt + p.kc - 1) / p.kc;
  const long items = base * p.n_kc;
  if (items > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  p.n_items = static_cast<int>(items);
  auto kern = dsa::indexer::indexer_kernel<H_I, D_I, G>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes) !=
      cudaSuccess)
    return DSA_ERR_CUDA;
  const int grid = static_cast<int>(std::min<long>(items, sms));
  return launch(kern, static_cast<unsigned>(grid), Cfg::kThreads, Cfg::kSmemBytes, stream, 1, tm_q, tm_k, p);
}

// ------------------------------------------------------------------------------ top-k
template <int C, int KPT>
dsa_status launch_topk(const float* scores, int32_t* idx, int B, int Lq, int Lk, int k,
                       cudaStream_t stream, uint32_t* ghist, const int32_t* seq_lens) {
  auto kern = dsa::topk::topk_kernel<C, KPT>;
  constexpr int smem = dsa::topk::dyn_smem_bytes<KPT>();
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return DSA_ERR_CUDA;
  return launch(kern, static_cast<unsigned>(B) * Lq * C, dsa::topk::kThreads, smem, stream, C, scores, idx, B, Lq,
                Lk, k, ghist, seq_lens);
}

// Keys per CTA for a row split over c CTAs (a multiple of 4, as the kernel computes it).
inline int topk_slice(int Lk, int c) { return (((Lk + c - 1) / c) + 3) & ~3; }

int topk_cluster_size(int rows, int Lk, int sms) {
  int c = 1;
  while (c < 8 && topk_slice(Lk, c) > dsa::topk::kMaxSlice) c *= 2;
  // more CTAs per row only while the doubled grid still runs in one wave
  while (c < 8 && static_cast<long>(rows) * 2 * c <= sms && topk_slice(Lk, 2 * c) >= 4096) c *= 2;
  return c;
}

template <int C>
dsa_status launch_topk_c(const float* scores, int32_t* idx, int B, int Lq, int Lk, int k,
                         cudaStream_t st, uint32_t* ghist, const int32_t* sl) {
  const int slice = topk_slice(Lk, C);
  if (slice <= 4 * dsa::topk::kThreads) return launch_topk<C, 4>(scores, idx, B, Lq, Lk, k, st, ghist, sl);
  if (slice <= 8 * dsa::topk::kThreads) return launch_topk<C, 8>(scores, idx, B, Lq, Lk, k, st, ghist, sl);
  if (slice <= 16 * dsa::topk::kThreads) return launch_topk<C, 16>(scores, idx, B, Lq, Lk, k, st, ghist, sl);
  return launch_topk<C, 32>(scores, idx, B, Lq, Lk, k, st, ghist, sl);
}

// Top-k with the validated sizes; ghist (nullable) holds each row's top-digit counts, seq_lens
// (nullable, Lq == 1) each row's context length.
dsa_status run_topk(const float* scores, int32_t* idx, int B, int Lq, int Lk, int k, int sms, cudaStream_t st,
                    uint32_t* ghist, const int32_t* seq_lens = nullptr) {
  switch (topk_cluster_size(B * Lq, Lk, sms)) {
    case 1: return launch_topk_c<1>(scores, idx, B, Lq, Lk, k, st, ghist, seq_lens);
    case 2: return launch_topk_c<2>(scores, idx, B, Lq, Lk, k, st, ghist, seq_lens);
    case 4: return launch_topk_c<4>(scores, idx, B, Lq, Lk, k, st, ghist, seq_lens);
    default: return launch_topk_c<8>(scores, idx, B, Lq, Lk, k, st, ghist, seq_lens);
  }
}

// Indexer with the validated sizes.  hist (nullable, decode kernels only) receives each row's
// top-digit counts; returns DSA_ERR_UNSUPPORTED for shapes outside the compiled kernels.
dsa_status run_indexer(const void* q_fp8, const void* k_fp8, const float* w, float* scores, int B, int Lq, int Lk,
                       int H_I, int d_I, int sms, cudaStream_t st, uint32_t* hist, const Paging* pg = nullptr) {
  const bool decode = (Lq == 1);
  if (pg && !(decode && d_I == 128 && (H_I == 64 || H_I == 32))) return DSA_ERR_UNSUPPORTED;
  if (H_I == 64 && d_I == 128)
    return decode ? launch_indexer<64, 128, 1>(q_fp8, k_fp8, w, scores, B, Lq, Lk, sms, st, hist, pg)
                  : launch_indexer<64, 128, 4>(q_fp8, k_fp8, w, scores, B, Lq, Lk, sms, st);
  if (H_I == 32 && d_I == 128)
    return decode ? launch_indexer<32, 128, 1>(q_fp8, k_fp8, w, scores, B, Lq, Lk, sms, st, hist, pg)
                  : launch_indexer<32, 128, 8>(q_fp8, k_fp8, w, scores, B, Lq, Lk, sms, st);
  if (H_I == 16 && d_I == 128) return launch_indexer<16, 128, 16>(q_fp8, k_fp8, w, scores, B, Lq, Lk, sms, st);
  if (H_I == 8 && d_I == 64) return launch_indexer<8, 64, 32>(q_fp8, k_fp8, w, scores, B, Lq, Lk, sms, st);
  if (H_I == 4 && d_I == 32) return launch_indexer<4, 32, 64>(q_fp8, k_fp8, w, scores, B, Lq, Lk, sms, st);
  return DSA_ERR_UNSUPPORTED;
}

// Whether the indexer of this shape has the decode kernel that counts top digits.
inline bool fused_topk_shape(int Lq, int H_I, int d_I) {
  return Lq == 1 && d_I == 128 && (H_I == 64 || H_I == 32);
}

// ------------------------------------------------------------------------------ sparse MLA
struct MlaSplit {
  int n_split;
  int per_split;
};

MlaSplit mla_split(int rows, int k, int n_dv, int sms, bool want_p) {
  MlaSplit s{1, ((k + dsa::mla::kBN - 1) / dsa::mla::kBN) * dsa::mla::kBN};
  const long ctas = static_cast<long>(rows) * n_dv;
  if (want_p || ctas >= sms) return s;
  int n = static_cast<int>(sms / ctas);
  const int max_by_len = std::max(1, (k + 4 * dsa::mla::kBN - 1) / (4 * dsa::mla::kBN));
  n = std::max(1, std::min(n, max_by_len));
  const int blocks = (k + dsa::mla::kBN - 1) / dsa::mla::kBN;
  s.per_split = ((blocks + n - 1) / n) * dsa::mla::kBN;
  s.n_split = (k + s.per_split - 1) / s.per_split;
  return s;
}

size_t mla_ws_bytes(int rows, int k, int H, int d_v, int sms) {
  const int n_dv = d_v > 256 ? d_v / 256 : 1;
  const MlaSplit s = mla_split(rows, k, n_dv, sms, false);
  if (s.n_split <= 1) return 0;
  return static_cast<size_t>(s.n_split) * rows * H * (static_cast<size_t>(d_v) + 1) * sizeof(float);
}

template <int D_QK, int D_V>
dsa_status launch_mla(const void* q, const void* kv, const int32_t* idx, int B, int Lq, int Lk,
                      int H, int k, float scale, void* out, float* lse, float* p_sel, void* ws,
                      size_t ws_bytes, int sms, cudaStream_t stream, int dense = 0,
                      const Paging* pg = nullptr) {
  using Cfg = dsa::mla::Cfg<D_QK, D_V>;
  const int rows = B * Lq;
  const MlaSplit sp = mla_split(rows, k, Cfg::kNdv, sms, p_sel != nullptr);
  dsa::mla::Params p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.kv = static_cast<const __nv_bfloat16*>(kv);
  p.idx = idx;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.p_sel = p_sel;
  p.B = B;
  p.Lq = Lq;
  p.Lk = Lk;
  p.H = H;
  p.k = k;
  p.n_split = sp.n_split;
  p.per_split = sp.per_split;
  p.scale_log2 = scale * dsa::mla::kLog2e;
  p.dense = dense;
  const long kv_rows = pg ? static_cast<long>(pg->num_pages) * pg->page_size : static_cast<long>(B) * Lk;
  if (kv_rows >= INT32_MAX) return DSA_ERR_UNSUPPORTED;
  p.kv_rows = static_cast<int>(kv_rows);
  if (pg) {
    p.block_table = pg->block_table;
    p.seq_lens = pg->seq_lens;
    p.page_size = pg->page_size;
    p.max_pages = pg->max_pages;
    p.num_pages = pg->num_pages;
  }
  if (sp.n_split > 1) {
    const size_t need = static_cast<size_t>(sp.n_split) * rows * H * (static_cast<size_t>(D_V) + 1) * sizeof(float);
    if (ws == nullptr || ws_bytes < need || !aligned16(ws)) return DSA_ERR_INVALID_ARG;
    p.part_o = static_cast<float*>(ws);
    p.part_lse = p.part_o + static_cast<size_t>(sp.n_split) * rows * H * D_V;
  }
  const long grid = static_cast<long>(rows) * Cfg::kNdv * sp.n_split;
  if (grid > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  if constexpr (D_QK == dsa::mla_pair::kDQK && D_V == dsa::mla_pair::kDV) {
    // cluster of two CTAs per (row, split): QK dims and value dims split between them; with two
    // splits, both pairs of a row form one cluster of four that combines in the kernel
    p.fuse2 = (sp.n_split == 2) ? 1 : 0;
    // kv as [B * Lk rows, 576 dims]: one-row boxes of 64 dims (SW128) and of the 32 rope dims
    // (SW64) for the row gathers
    CUtensorMap tm_main, tm_rope;
    if (!encode_2d(&tm_main, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kv, D_QK, static_cast<uint64_t>(kv_rows),
                   static_cast<uint64_t>(D_QK) * 2, 64, 1, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_2d(&tm_rope, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kv, D_QK, static_cast<uint64_t>(kv_rows),
                   static_cast<uint64_t>(D_QK) * 2, 32, 1, CU_TENSOR_MAP_SWIZZLE_64B))
      return DSA_ERR_CUDA;
    // q as [rows * H, 576]: 128 head rows x 64 dims (SW128) and x the 32 rope dims (SW64)
    CUtensorMap tm_q_main, tm_q_rope;
    if (!encode_2d(&tm_q_main, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q, D_QK, static_cast<uint64_t>(rows) * H,
                   static_cast<uint64_t>(D_QK) * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_2d(&tm_q_rope, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q, D_QK, static_cast<uint64_t>(rows) * H,
                   static_cast<uint64_t>(D_QK) * 2, 32, 128, CU_TENSOR_MAP_SWIZZLE_64B))
      return DSA_ERR_CUDA;
    auto kern = dsa::mla_pair::sparse_mla_pair_kernel;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             dsa::mla_pair::kSmemBytes) != cudaSuccess)
      return DSA_ERR_CUDA;
    const dsa_status st = launch(kern, static_cast<unsigned>(grid), dsa::mla_pair::kThreads, dsa::mla_pair::kSmemBytes,
                                 stream, p.fuse2 ? 4u : 2u, tm_main, tm_rope, tm_q_main, tm_q_rope, p);
    if (st != DSA_OK || p.fuse2) return st;
  } else {
    CUtensorMap tm_q;
    if (!encode_2d(&tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q, D_QK, static_cast<uint64_t>(rows) * H,
                   static_cast<uint64_t>(D_QK) * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
      return DSA_ERR_CUDA;
    auto kern = dsa::mla::sparse_mla_kernel<D_QK, D_V>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes) !=
        cudaSuccess)
      return DSA_ERR_CUDA;
    const dsa_status st = launch(kern, static_cast<unsigned>(grid), dsa::mla::kThreads, Cfg::kSmemBytes, stream, 1,
                                 tm_q, p);
    if (st != DSA_OK) return st;
  }
  if (sp.n_split > 1) {
    const int cgrid = (rows * H + dsa::mla::kCombineWarps - 1) / dsa::mla::kCombineWarps;
    return launch(dsa::mla::combine_kernel<D_V>, static_cast<unsigned>(cgrid), dsa::mla::kCombineWarps * 32, 0, stream,
                  1, static_cast<const float*>(p.part_o), static_cast<const float*>(p.part_lse), sp.n_split, rows * H,
                  static_cast<__nv_bfloat16*>(out), lse);
  }
  return DSA_OK;
}

// ------------------------------------------------------------------------------ indexer KL without
// caller scratch.  The per-row KL terms go to a fixed device array that every GPU loading the
// library holds until the process exits; its address is looked up once per device.
constexpr int kKlNoAllocMaxRows = 1 << 20;  // 4 MiB of fp32 per device
static __device__ __align__(256) float g_kl_rows_scratch[kKlNoAllocMaxRows];

float* g_kl_scratch_ptr[kMaxDevices];
std::atomic<bool> g_kl_scratch_ok[kMaxDevices];

// Device address of g_kl_rows_scratch on the current device.  The name itself is only a host
// stand-in, so the address must come from cudaGetSymbolAddress with that device current.  Only a
// successful lookup is cached; a failed one is retried on the next call.
dsa_status kl_scratch_for_current_device(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DSA_ERR_CUDA;
  if (!g_kl_scratch_ok[dev].load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_kl_scratch_ok[dev].load(std::memory_order_relaxed)) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_kl_rows_scratch) != cudaSuccess || p == nullptr) {
        cudaGetLastError();  // clear the (non-sticky) error so that the next call starts clean
        return DSA_ERR_CUDA;
      }
      g_kl_scratch_ptr[dev] = static_cast<float*>(p);
      g_kl_scratch_ok[dev].store(true, std::memory_order_release);
    }
  }
  *out = g_kl_scratch_ptr[dev];
  return DSA_OK;
}

// ------------------------------------------------------------------------------ wait self-test
// One warp waits on an mbarrier that nothing arrives on: the bounded wait gives up after the
// limit in force and records DSA_ERR_TIMEOUT (site 90), and the kernel returns.
__global__ void wait_selftest_kernel() {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    dsa::mbar_init(&bar, 1);
    abort_flag = 0;
    dsa::fence_barrier_init();
  }
  __syncwarp();
  dsa::mbar_wait(&bar, 0, &abort_flag, 90);
}

// ------------------------------------------------------------------------------ HISA workspace
struct HisaWs {  // workspace regions of dsa_hisa_topk (each 256-byte aligned)
  size_t bscores, bidx, pages, seq, cscores, cidx, hist, total;
};
inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
HisaWs hisa_ws(int B, int Lk, int block, int r, int k) {
  HisaWs w{};
  const size_t nb = static_cast<size_t>((Lk + block - 1) / block);
  size_t o = 0;
  w.bscores = o; o = align256(o + static_cast<size_t>(B) * nb * 4);
  w.bidx = o;    o = align256(o + static_cast<size_t>(B) * r * 4);
  w.pages = o;   o = align256(o + static_cast<size_t>(B) * r * 4);
  w.seq = o;     o = align256(o + static_cast<size_t>(B) * 4);
  w.cscores = o; o = align256(o + static_cast<size_t>(B) * r * block * 4);
  w.cidx = o;    o = align256(o + static_cast<size_t>(B) * k * 4);
  w.hist = o;    o = align256(o + static_cast<size_t>(B) * 2048 * 4);
  w.total = o;
  return w;
}

__global__ void hisa_seq_lens_kernel(int32_t* seq, int B, int n) {
  dsa::pdl_launch_dependents();
  dsa::pdl_wait();
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < B; b += gridDim.x * blockDim.x) seq[b] = n;
}

}  // namespace

// ================================================================================ C ABI
extern "C" {

const char* dsa_status_str(dsa_status s) {
  switch (s) {
    case DSA_OK: return "DSA_OK";
    case DSA_ERR_INVALID_ARG: return "DSA_ERR_INVALID_ARG";
    case DSA_ERR_UNSUPPORTED: return "DSA_ERR_UNSUPPORTED";
    case DSA_ERR_CUDA: return "DSA_ERR_CUDA";
    case DSA_ERR_NO_SM100: return "DSA_ERR_NO_SM100";
    case DSA_ERR_TIMEOUT: return "DSA_ERR_TIMEOUT";
  }
  return "DSA_ERR_UNKNOWN";
}

int dsa_version(void) { return 101; }

size_t dsa_workspace_bytes(int op, int B, int Lq, int Lk, int k, int H) {
  if (B <= 0 || Lq <= 0) return 0;
  const long rows = static_cast<long>(B) * Lq;
  switch (op) {
    case DSA_OP_SPARSE_MLA_FWD: {
      if (k <= 0 || H <= 0) return 0;
      const int sms = sm_count_or_default();
      // an upper bound over every supported value width
      return std::max(mla_ws_bytes(static_cast<int>(rows), k, H, 512, sms),
                      mla_ws_bytes(static_cast<int>(rows), k, H, 64, sms));
    }
    case DSA_OP_DENSE_MLA_FWD: {
      if (Lk <= 0 || H <= 0) return 0;
      const int sms = sm_count_or_default();
      return std::max(mla_ws_bytes(static_cast<int>(rows), Lk, H, 512, sms),
                      mla_ws_bytes(static_cast<int>(rows), Lk, H, 64, sms));
    }
    case DSA_OP_MASKED_MHA:  // the selection bitmap, rows of a multiple of 4 words
      return static_cast<size_t>(rows) * (((Lk + 127) / 128) * 4) * sizeof(uint32_t);
    case DSA_OP_INDEXER_TOPK:
      // the decode kernels' top-digit histograms (no workspace for other shapes)
      return Lq == 1 ? static_cast<size_t>(rows) * 2048 * sizeof(uint32_t) : 0;
    case DSA_OP_INDEXER_KL:
    case DSA_OP_INDEXER_KL_DENSE:
      return static_cast<size_t>(rows) * sizeof(float);
    default:
      return 0;
  }
}

dsa_status dsa_indexer(const void* q_fp8, const void* k_fp8, const float* w, float* scores, int B,
                       int Lq, int Lk, int H_I, int d_I, void* ws, size_t ws_bytes,
                       dsa_stream_t stream) {
  (void)ws;
  (void)ws_bytes;
  if (!q_fp8 || !k_fp8 || !w || !scores) return DSA_ERR_INVALID_ARG;
  if (B <= 0 || Lq <= 0 || Lk <= 0 || Lq > Lk || H_I <= 0 || d_I <= 0) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_fp8) || !aligned16(k_fp8) || !aligned16(w) || !aligned16(scores))
    return DSA_ERR_INVALID_ARG;
  if (static_cast<long>(B) * Lk > INT32_MAX || static_cast<long>(B) * Lq * H_I > INT32_MAX)
    return DSA_ERR_UNSUPPORTED;
  DeviceInfo dev;
  const dsa_status ds = current_device(dev);
  if (ds != DSA_OK) return ds;
  return run_indexer(q_fp8, k_fp8, w, scores, B, Lq, Lk, H_I, d_I, dev.sms, static_cast<cudaStream_t>(stream),
                     nullptr);
}

dsa_status dsa_topk(const float* scores, int32_t* idx, int B, int Lq, int Lk, int k, void* ws,
                    size_t ws_bytes, dsa_stream_t stream) {
  (void)ws;
  (void)ws_bytes;
  if (!scores || !idx) return DSA_ERR_INVALID_ARG;
  if (B <= 0 || Lq <= 0 || Lk <= 0 || Lq > Lk || k <= 0) return DSA_ERR_INVALID_ARG;
  if (!aligned16(scores) || !aligned16(idx)) return DSA_ERR_INVALID_ARG;
  if (k > 4096 || topk_slice(Lk, 8) > dsa::topk::kMaxSlice) return DSA_ERR_UNSUPPORTED;
  if (static_cast<long>(B) * Lq * 8 > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  DeviceInfo dev;
  const dsa_status ds = current_device(dev);
  if (ds != DSA_OK) return ds;
  return run_topk(scores, idx, B, Lq, Lk, k, dev.sms, static_cast<cudaStream_t>(stream), nullptr);
}

dsa_status dsa_indexer_topk(const void* q_fp8, const void* k_fp8, const float* w, float* scores, int32_t* idx,
                            int B, int Lq, int Lk, int H_I, int d_I, int k, void* ws, size_t ws_bytes,
                            dsa_stream_t stream) {
  if (!q_fp8 || !k_fp8 || !w || !scores || !idx) return DSA_ERR_INVALID_ARG;
  if (B <= 0 || Lq <= 0 || Lk <= 0 || Lq > Lk || H_I <= 0 || d_I <= 0 || k <= 0) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_fp8) || !aligned16(k_fp8) || !aligned16(w) || !aligned16(scores) || !aligned16(idx))
    return DSA_ERR_INVALID_ARG;
  if (static_cast<long>(B) * Lk > INT32_MAX || static_cast<long>(B) * Lq * H_I > INT32_MAX)
    return DSA_ERR_UNSUPPORTED;
  if (k > 4096 || topk_slice(Lk, 8) > dsa::topk::kMaxSlice) return DSA_ERR_UNSUPPORTED;
  if (static_cast<long>(B) * Lq * 8 > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  const bool fused = fused_topk_shape(Lq, H_I, d_I);
  const size_t need = fused ? static_cast<size_t>(B) * Lq * 2048 * sizeof(uint32_t) : 0;
  if (fused && (ws == nullptr || ws_bytes < need || !aligned16(ws))) return DSA_ERR_INVALID_ARG;
  DeviceInfo dev;
  const dsa_status ds = current_device(dev);
  if (ds != DSA_OK) return ds;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t* hist = fused ? static_cast<uint32_t*>(ws) : nullptr;  // zero-filled between calls
  const dsa_status si = run_indexer(q_fp8, k_fp8, w, scores, B, Lq, Lk, H_I, d_I, dev.sms, st, hist);
  if (si != DSA_OK) return si;
  return run_topk(scores, idx, B, Lq, Lk, k, dev.sms, st, hist);
}

dsa_status dsa_sparse_mla_fwd(const void* q_bf16, const void* kv_bf16, const int32_t* idx, int B,
                              int Lq, int Lk, int H, int d_qk, int d_v, int k, float scale,
                              void* out_bf16, float* lse, float* p_sel, void* ws, size_t ws_bytes,
                              dsa_stream_t stream) {
  if (!q_bf16 || !kv_bf16 || !idx || !out_bf16) return DSA_ERR_INVALID_ARG;
  if (B <= 0 || Lq <= 0 || Lk <= 0 || Lq > Lk || H <= 0 || k <= 0) return DSA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_bf16) || !aligned16(kv_bf16) || !aligned16(idx) || !aligned16(out_bf16) ||
      (lse && !aligned16(lse)) || (p_sel && !aligned16(p_sel)))
    return DSA_ERR_INVALID_ARG;
  if (H > 128 || k > 65536 || static_cast<long>(B) * Lk >= INT32_MAX) return DSA_ERR_UNSUPPORTED;
  if (static_cast<long>(B) * Lq * H * 2 * 8 > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  DeviceInfo dev;
  const dsa_status ds = current_device(dev);
  if (ds != DSA_OK) return ds;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d_qk == 576 && d_v == 512)
    return launch_mla<576, 512>(q_bf16, kv_bf16, idx, B, Lq, Lk, H, k, scale, out_bf16, lse, p_sel,
                                ws, ws_bytes, dev.sms, st);
  if (d_qk == 80 && d_v == 64)
    return launch_mla<80, 64>(q_bf16, kv_bf16, idx, B, Lq, Lk, H, k, scale, out_bf16, lse, p_sel,
                              ws, ws_bytes, dev.sms, st);
  return DSA_ERR_UNSUPPORTED;
}

dsa_status dsa_indexer_kl(const float* scores, const int32_t* idx, const float* p_sel, int B,
                          int Lq, int Lk, int k, float* loss, float* loss_per_query, void* ws,
                          size_t ws_bytes, dsa_stream_t stream) {
  if (!scores || !idx || !p_sel || !loss) return DSA_ERR_INVALID_ARG;
  if (B <= 0 || Lq <= 0 || Lk <= 0 || Lq > Lk || k <= 0) return DSA_ERR_INVALID_ARG;
  if (!aligned16(scores) || !aligned16(idx) || !aligned16(p_sel) || (reinterpret_cast<uintptr_t>(loss) & 3u) ||
      (loss_per_query && !aligned16(loss_per_query)))
    return DSA_ERR_INVALID_ARG;
  const long rows = static_cast<long>(B) * Lq;
  if (rows > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  float* per_row = loss_per_query;
  if (per_row == nullptr) {
    if (ws == nullptr || ws_bytes < static_cast<size_t>(rows) * sizeof(float) || !aligned16(ws))
      return DSA_ERR_INVALID_ARG;
    per_row = static_cast<float*>(ws);
  }
  DeviceInfo dev;
  const dsa_status ds = current_device(dev);
  if (ds != DSA_OK) return ds;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const dsa_status sr = launch(dsa::kl::kl_rows_kernel, static_cast<unsigned>(rows), dsa::kl::kRowThreads, 0, st, 1,
                               scores, idx, p_sel, Lq, Lk, k, per_row);
  if (sr != DSA_OK) return sr;
  return launch(dsa::kl::kl_sum_kernel, 1u, dsa::kl::kSumThreads, 0, st, 1, static_cast<const float*>(per_row),
                static_cast<int>(rows), loss);
}

dsa_status dsa_indexer_kl_noalloc(const float* scores, const int32_t* idx, const float* p_sel,
                                  int B, int Lq, int Lk, int k, float* loss,
                                  float* loss_per_query, dsa_stream_t stream) {
  if (!scores || !idx || !p_sel || !loss) return DSA_ERR_INVALID_ARG;
  if (B <= 0 || Lq <= 0 || Lk <= 0 || Lq > Lk || k <= 0) return DSA_ERR_INVALID_ARG;
  if (!aligned16(scores) || !aligned16(idx) || !aligned16(p_sel) || (reinterpret_cast<uintptr_t>(loss) & 3u) ||
      (loss_per_query && !aligned16(loss_per_query)))
    return DSA_ERR_INVALID_ARG;
  const long rows = static_cast<long>(B) * Lq;
  if (rows > kKlNoAllocMaxRows) return DSA_ERR_UNSUPPORTED;
  DeviceInfo dev;
  const dsa_status ds = current_device(dev);
  if (ds != DSA_OK) return ds;
  float* per_row = loss_per_query;
  if (per_row == nullptr) {
    const dsa_status ss = kl_scratch_for_current_device(&per_row);
    if (ss != DSA_OK) return ss;
  }
  // Every row's term is written before the sum reads it, so the shared array needs no clearing.
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const dsa_status sr = launch(dsa::kl::kl_rows_kernel, static_cast<unsigned>(rows), dsa::kl::kRowThreads, 0, st, 1,
                               scores, idx, p_sel, Lq, Lk, k, per_row);
  if (sr != DSA_OK) return sr;
  return launch(dsa::kl::kl_sum_kernel, 1u, dsa::kl::kSumThreads, 0, st, 1, static_cast<const float*>(per_row),
                static_cast<int>(rows), loss);
}

dsa_status dsa_dense_mla_fwd(const void* q_bf16, const void* kv_bf16, int B, int Lq, int Lk, int H,
                             int d_qk, int d_v, float scale, void* out_bf16, float* lse, float* p_full,
                             void* ws, size_t ws_bytes, dsa_stream_t stream) {
  if (!q_bf16 || !kv_bf16 || !out_bf16) return DSA_ERR_INVALID_ARG;
  if (B <= 0 || Lq <= 0 || Lk <= 0 || Lq > Lk || H <= 0) return DSA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_bf16) || !aligned16(kv_bf16) || !aligned16(out_bf16) || (lse && !aligned16(lse)) ||
      (p_full && !aligned16(p_full)))
    return DSA_ERR_INVALID_ARG;
  if (H > 128 || Lk > 65536 || static_cast<long>(B) * Lk >= INT32_MAX) return DSA_ERR_UNSUPPORTED;
  if (static_cast<long>(B) * Lq * H * 2 * 8 > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  DeviceInfo dev;
  const dsa_status ds = current_device(dev);
  if (ds != DSA_OK) return ds;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // dense causal attention = the selection kernel with slot j read as position j (k = Lk)
  if (d_qk == 576 && d_v == 512)
    return launch_mla<576, 512>(q_bf16, kv_bf16, nullptr, B, Lq, Lk, H, Lk, scale, out_bf16, lse, p_full, ws,
                                ws_bytes, dev.sms, st, 1);
  if (d_qk == 80 && d_v == 64)
    return launch_mla<80, 64>(q_bf16, kv_bf16, nullptr, B, Lq, Lk, H, Lk, scale, out_bf16, lse, p_full, ws,
                              ws_bytes, dev.sms, st, 1);
  return DSA_ERR_UNSUPPORTED;
}

dsa_status dsa_indexer_kl_dense(const float* scores, const float* p_full, int B, int Lq, int Lk, float* loss,
                                float* loss_per_query, void* ws, size_t ws_bytes, dsa_stream_t stream) {
  if (!scores || !p_full || !loss) return DSA_ERR_INVALID_ARG;
  if (B <= 0 || Lq <= 0 || Lk <= 0 || Lq > Lk) return DSA_ERR_INVALID_ARG;
  if (!aligned16(scores) || !aligned16(p_full) || (reinterpret_cast<uintptr_t>(loss) & 3u) ||
      (loss_per_query && !aligned16(loss_per_query)))
    return DSA_ERR_INVALID_ARG;
  const long rows = static_cast<long>(B) * Lq;
  if (rows > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  float* per_row = loss_per_query;
  if (per_row == nullptr) {
    if (ws == nullptr || ws_bytes < static_cast<size_t>(rows) * sizeof(float) || !aligned16(ws))
      return DSA_ERR_INVALID_ARG;
    per_row = static_cast<float*>(ws);
  }
  DeviceInfo dev;
  const dsa_status ds = current_device(dev);
  if (ds != DSA_OK) return ds;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const dsa_status sr = launch(dsa::kl::kl_rows_kernel, static_cast<unsigned>(rows), dsa::kl::kRowThreads, 0, st, 1,
                               scores, static_cast<const int32_t*>(nullptr), p_full, Lq, Lk, Lk, per_row);
  if (sr != DSA_OK) return sr;
  return launch(dsa::kl::kl_sum_kernel, 1u, dsa::kl::kSumThreads, 0, st, 1, static_cast<const float*>(per_row),
                static_cast<int>(rows), loss);
}

dsa_status dsa_indexer_bwd(const void* q_fp8, const void* k_fp8, const float* w, const float* scores,
                           const int32_t* idx, const float* p_sel, int B, int Lq, int Lk, int H_I, int d_I, int k,
                           float* dq, float* dw, float* dk, dsa_stream_t stream) {
  if (!q_fp8 || !k_fp8 || !w || !scores || !p_sel || !dq || !dw || !dk) return DSA_ERR_INVALID_ARG;
  if (B <= 0 || Lq <= 0 || Lk <= 0 || Lq > Lk || H_I <= 0 || d_I <= 0 || k <= 0) return DSA_ERR_INVALID_ARG;
  if (idx == nullptr && k != Lk) return DSA_ERR_INVALID_ARG;  // dense: every position is a slot
  if (!aligned16(q_fp8) || !aligned16(k_fp8) || !aligned16(w) || !aligned16(scores) || (idx && !aligned16(idx)) ||
      !aligned16(p_sel) || !aligned16(dq) || !aligned16(dw) || !aligned16(dk))
    return DSA_ERR_INVALID_ARG;
  if (H_I != dsa::bwd::kHI || d_I != dsa::bwd::kDI) return DSA_ERR_UNSUPPORTED;
  if (static_cast<long>(B) * Lk >= INT32_MAX || static_cast<long>(B) * Lq >= INT32_MAX) return DSA_ERR_UNSUPPORTED;
  DeviceInfo dev;
  const dsa_status ds = current_device(dev);
  if (ds != DSA_OK) return ds;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // dk accumulates over every query that selected a key
  if (cudaMemsetAsync(dk, 0, static_cast<size_t>(B) * Lk * d_I * sizeof(float), st) != cudaSuccess)
    return DSA_ERR_CUDA;
  dsa::bwd::Params p{};
  p.q = static_cast<const uint8_t*>(q_fp8);
  p.kI = static_cast<const uint8_t*>(k_fp8);
  p.w = w;
  p.scores = scores;
  p.idx = idx;
  p.p = p_sel;
  p.dq = dq;
  p.dw = dw;
  p.dk = dk;
  p.B = B;
  p.Lq = Lq;
  p.Lk = Lk;
  p.k = k;
  auto kern = dsa::bwd::indexer_bwd_kernel;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, dsa::bwd::kSmemBytes) != cudaSuccess)
    return DSA_ERR_CUDA;
  const long rows = static_cast<long>(B) * Lq;
  const unsigned grid = static_cast<unsigned>(std::min<long>(rows, 2L * dev.sms));
  return launch(kern, grid, dsa::bwd::kThreads, dsa::bwd::kSmemBytes, st, 1, p);
}

// Shared checks of the paged decode entry points; fills *pg.
dsa_status check_paging(const int32_t* block_table, const int32_t* seq_lens, int B, int max_len, int num_pages,
                        int page_size, Paging* pg) {
  if (!block_table || !seq_lens) return DSA_ERR_INVALID_ARG;
  if (B <= 0 || max_len <= 0 || num_pages <= 0 || page_size <= 0) return DSA_ERR_INVALID_ARG;
  if (!aligned16(block_table) || !aligned16(seq_lens)) return DSA_ERR_INVALID_ARG;
  if (page_size % 64 != 0) return DSA_ERR_UNSUPPORTED;  // the indexer loads pages in boxes of 64 keys
  if (static_cast<long>(num_pages) * page_size >= INT32_MAX || static_cast<long>(B) * max_len >= INT32_MAX)
    return DSA_ERR_UNSUPPORTED;
  pg->block_table = block_table;
  pg->seq_lens = seq_lens;
  pg->page_size = page_size;
  pg->max_pages = (max_len + page_size - 1) / page_size;
  pg->num_pages = num_pages;
  return DSA_OK;
}

dsa_status dsa_indexer_topk_paged(const void* q_fp8, const void* k_pages, const float* w, const int32_t* block_table,
                                  const int32_t* seq_lens, float* scores, int32_t* idx, int B, int max_len,
                                  int num_pages, int page_size, int H_I, int d_I, int k, void* ws, size_t ws_bytes,
                                  dsa_stream_t stream) {
  if (!q_fp8 || !k_pages || !w || !scores || !idx || H_I <= 0 || d_I <= 0 || k <= 0) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_fp8) || !aligned16(k_pages) || !aligned16(w) || !aligned16(scores) || !aligned16(idx))
    return DSA_ERR_INVALID_ARG;
  Paging pg;
  const dsa_status sp = check_paging(block_table, seq_lens, B, max_len, num_pages, page_size, &pg);
  if (sp != DSA_OK) return sp;
  if (!fused_topk_shape(1, H_I, d_I)) return DSA_ERR_UNSUPPORTED;
  if (k > 4096 || topk_slice(max_len, 8) > dsa::topk::kMaxSlice) return DSA_ERR_UNSUPPORTED;
  const size_t need = static_cast<size_t>(B) * 2048 * sizeof(uint32_t);
  if (ws == nullptr || ws_bytes < need || !aligned16(ws)) return DSA_ERR_INVALID_ARG;
  DeviceInfo dev;
  const dsa_status ds = current_device(dev);
  if (ds != DSA_OK) return ds;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t* hist = static_cast<uint32_t*>(ws);  // zero-filled between calls
  const dsa_status si = run_indexer(q_fp8, k_pages, w, scores, B, 1, max_len, H_I, d_I, dev.sms, st, hist, &pg);
  if (si != DSA_OK) return si;
  return run_topk(scores, idx, B, 1, max_len, k, dev.sms, st, hist, seq_lens);
}

dsa_status dsa_sparse_mla_fwd_paged(const void* q_bf16, const void* kv_pages, const int32_t* idx,
                                    const int32_t* block_table, const int32_t* seq_lens, int B, int max_len,
                                    int num_pages, int page_size, int H, int d_qk, int d_v, int k, float scale,
                                    void* out_bf16, float* lse, void* ws, size_t ws_bytes, dsa_stream_t stream) {
  if (!q_bf16 || !kv_pages || !idx || !out_bf16 || H <= 0 || k <= 0) return DSA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_bf16) || !aligned16(kv_pages) || !aligned16(idx) || !aligned16(out_bf16) || (lse && !aligned16(lse)))
    return DSA_ERR_INVALID_ARG;
  Paging pg;
  const dsa_status sp = check_paging(block_table, seq_lens, B, max_len, num_pages, page_size, &pg);
  if (sp != DSA_OK) return sp;
  if (d_qk != 576 || d_v != 512 || H > 128 || k > 65536) return DSA_ERR_UNSUPPORTED;
  DeviceInfo dev;
  const dsa_status ds = current_device(dev);
  if (ds != DSA_OK) return ds;
  return launch_mla<576, 512>(q_bf16, kv_pages, idx, B, 1, max_len, H, k, scale, out_bf16, lse, nullptr, ws, ws_bytes,
                              dev.sms, static_cast<cudaStream_t>(stream), 0, &pg);
}


size_t dsa_hisa_workspace_bytes(int B, int Lk, int block, int r, int k) {
  if (B <= 0 || Lk <= 0 || block <= 0 || r <= 0 || k <= 0) return 0;
  return hisa_ws(B, Lk, block, r, k).total;
}

dsa_status dsa_hisa_block_sums(const void* k_fp8, int B, int Lk, int d_I, int block, float* sums,
                                          dsa_stream_t stream) {
  if (!k_fp8 || !sums || B <= 0 || Lk <= 0 || block <= 0 || d_I <= 0) return DSA_ERR_INVALID_ARG;
  if (!aligned16(k_fp8) || !aligned16(sums)) return DSA_ERR_INVALID_ARG;
  if (d_I != dsa::hisa::kDI) return DSA_ERR_UNSUPPORTED;
  const long n_blocks = (Lk + block - 1) / block;
  if (static_cast<long>(B) * n_blocks > INT32_MAX || static_cast<long>(B) * Lk >= INT32_MAX) return DSA_ERR_UNSUPPORTED;
  DeviceInfo dev;
  const dsa_status ds = current_device(dev);
  if (ds != DSA_OK) return ds;
  return launch(dsa::hisa::block_sums_kernel, static_cast<unsigned>(B * n_blocks), dsa::hisa::kSumThreads, 0,
                static_cast<cudaStream_t>(stream), 1, static_cast<const uint8_t*>(k_fp8), Lk, block,
                static_cast<int>(n_blocks), sums);
}

dsa_status dsa_hisa_topk(const void* q_fp8, const void* k_fp8, const float* w, const float* block_sums,
                                    int B, int Lk, int H_I, int d_I, int block, int r, int k, int32_t* idx,
                                    int32_t* blocks, void* ws, size_t ws_bytes, dsa_stream_t stream) {
  if (!q_fp8 || !k_fp8 || !w || !block_sums || !idx || !ws) return DSA_ERR_INVALID_ARG;
  if (B <= 0 || Lk <= 0 || block <= 0 || r <= 0 || k <= 0) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_fp8) || !aligned16(k_fp8) || !aligned16(w) || !aligned16(block_sums) || !aligned16(idx) ||
      (blocks && !aligned16(blocks)) || !aligned16(ws))
    return DSA_ERR_INVALID_ARG;
  if (Lk % block != 0 || block % 64 != 0) return DSA_ERR_UNSUPPORTED;  // whole blocks, loaded 64 keys at a time
  if (!fused_topk_shape(1, H_I, d_I)) return DSA_ERR_UNSUPPORTED;
  const int n_blocks = Lk / block;
  const int r_eff = std::min(r, n_blocks);
  if (k > 4096 || r > 4096 || static_cast<long>(r) * block > 262144 || n_blocks > 262144) return DSA_ERR_UNSUPPORTED;
  if (static_cast<long>(B) * Lk >= INT32_MAX) return DSA_ERR_UNSUPPORTED;
  const HisaWs L = hisa_ws(B, Lk, block, r, k);
  if (ws_bytes < L.total) return DSA_ERR_INVALID_ARG;
  DeviceInfo dev;
  const dsa_status ds = current_device(dev);
  if (ds != DSA_OK) return ds;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  float* bscores = reinterpret_cast<float*>(base + L.bscores);
  int32_t* bidx = blocks ? blocks : reinterpret_cast<int32_t*>(base + L.bidx);
  int32_t* pages = reinterpret_cast<int32_t*>(base + L.pages);
  int32_t* seq = reinterpret_cast<int32_t*>(base + L.seq);
  float* cscores = reinterpret_cast<float*>(base + L.cscores);
  int32_t* cidx = reinterpret_cast<int32_t*>(base + L.cidx);
  uint32_t* hist = reinterpret_cast<uint32_t*>(base + L.hist);
  // 1. coarse scores of every block; 2. the r best blocks (ascending)
  const dim3 sgrid(static_cast<unsigned>(B), static_cast<unsigned>((n_blocks + dsa::hisa::kScoreThreads - 1) /
                                                                    dsa::hisa::kScoreThreads));
  if (H_I == 64)
    dsa::hisa::block_scores_kernel<64><<<sgrid, dsa::hisa::kScoreThreads, 0, st>>>(
        static_cast<const uint8_t*>(q_fp8), w, block_sums, Lk, block, n_blocks, bscores);
  else
    dsa::hisa::block_scores_kernel<32><<<sgrid, dsa::hisa::kScoreThreads, 0, st>>>(
        static_cast<const uint8_t*>(q_fp8), w, block_sums, Lk, block, n_blocks, bscores);
  if (launch_result() != DSA_OK) return DSA_ERR_CUDA;
  dsa_status s = run_topk(bscores, bidx, B, 1, n_blocks, r, dev.sms, st, nullptr);
  if (s != DSA_OK) return s;
  // 3. the kept blocks as the pages of the exact stage, every candidate slot valid
  s = launch(dsa::hisa::block_pages_kernel, static_cast<unsigned>(B), 128u, 0, st, 1,
             static_cast<const int32_t*>(bidx), r, n_blocks, pages);
  if (s != DSA_OK) return s;
  s = launch(hisa_seq_lens_kernel, static_cast<unsigned>((B + 255) / 256), 256u, 0, st, 1, seq, B, r_eff * block);
  if (s != DSA_OK) return s;
  // 4. exact indexer scores on the candidates and their top-k (the paged decode path)
  Paging pg{pages, seq, block, r, B * n_blocks};  // hist: zero-filled between calls
  s = run_indexer(q_fp8, k_fp8, w, cscores, B, 1, r * block, H_I, d_I, dev.sms, st, hist, &pg);
  if (s != DSA_OK) return s;
  s = run_topk(cscores, cidx, B, 1, r * block, k, dev.sms, st, hist, seq);
  if (s != DSA_OK) return s;
  // 5. candidate slots -> positions
  return launch(dsa::hisa::slots_to_positions_kernel, static_cast<unsigned>(B), 256u, 0, st, 1,
                static_cast<const int32_t*>(cidx), static_cast<const int32_t*>(bidx), r, block, k, idx);
}

dsa_status dsa_masked_mha_fwd(const void* q_bf16, const void* k_bf16, const void* v_bf16, const int32_t* idx, int B,
                              int L, int H, int d_qk, int d_v, int k, float scale, void* out_bf16, float* lse,
                              void* ws, size_t ws_bytes, dsa_stream_t stream) {
  if (!q_bf16 || !k_bf16 || !v_bf16 || !idx || !out_bf16 || !ws) return DSA_ERR_INVALID_ARG;
  if (B <= 0 || L <= 0 || H <= 0 || k <= 0) return DSA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_bf16) || !aligned16(k_bf16) || !aligned16(v_bf16) || !aligned16(idx) || !aligned16(out_bf16) ||
      (lse && !aligned16(lse)) || !aligned16(ws))
    return DSA_ERR_INVALID_ARG;
  if (d_qk != dsa::mmha::kDQK || d_v != dsa::mmha::kDV || L > 65536) return DSA_ERR_UNSUPPORTED;
  const int words = ((L + 127) / 128) * 4;
  const size_t need = static_cast<size_t>(B) * L * words * sizeof(uint32_t);
  if (ws_bytes < need) return DSA_ERR_INVALID_ARG;
  const long n_qt = (L + dsa::mmha::kBM - 1) / dsa::mmha::kBM;
  if (static_cast<long>(B) * L * H >= INT32_MAX || static_cast<long>(B) * H * n_qt >= INT32_MAX ||
      static_cast<long>(B) * L >= INT32_MAX)
    return DSA_ERR_UNSUPPORTED;
  DeviceInfo dev;
  const dsa_status ds = current_device(dev);
  if (ds != DSA_OK) return ds;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t* sel = static_cast<uint32_t*>(ws);
  if (cudaFuncSetAttribute(dsa::mmha::build_selection_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           words * 4) != cudaSuccess)
    return DSA_ERR_CUDA;
  dsa_status s = launch(dsa::mmha::build_selection_kernel, static_cast<unsigned>(B * L), 256u,
                        static_cast<size_t>(words) * 4, st, 1, idx, L, k, words, sel);
  if (s != DSA_OK) return s;
  // q, k: [B * L rows, H * 192 cols]; v: [B * L rows, H * 128 cols]; boxes of 64 cols x 128 rows
  CUtensorMap tm_q, tm_k, tm_v;
  const uint64_t rows = static_cast<uint64_t>(B) * L;
  if (!encode_2d(&tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q_bf16, static_cast<uint64_t>(H) * d_qk, rows,
                 static_cast<uint64_t>(H) * d_qk * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&tm_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, k_bf16, static_cast<uint64_t>(H) * d_qk, rows,
                 static_cast<uint64_t>(H) * d_qk * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&tm_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, v_bf16, static_cast<uint64_t>(H) * d_v, rows,
                 static_cast<uint64_t>(H) * d_v * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
    return DSA_ERR_CUDA;
  dsa::mmha::Params p{};
  p.sel = sel;
  p.out = static_cast<__nv_bfloat16*>(out_bf16);
  p.lse = lse;
  p.B = B;
  p.L = L;
  p.H = H;
  p.words = words;
  p.scale_log2 = scale * dsa::mla::kLog2e;
  auto kern = dsa::mmha::masked_mha_kernel;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, dsa::mmha::kSmemBytes) != cudaSuccess)
    return DSA_ERR_CUDA;
  return launch(kern, static_cast<unsigned>(B * H * n_qt), dsa::mmha::kThreads, dsa::mmha::kSmemBytes, st, 1, tm_q,
                tm_k, tm_v, p);
}

dsa_status dsa_set_wait_limit_ns(uint64_t ns) {
  const unsigned long long v = ns == 0 ? dsa::kWaitLimitNs : static_cast<unsigned long long>(ns);
  if (cudaMemcpyToSymbol(dsa::g_wait_limit_ns, &v, sizeof(v)) != cudaSuccess) return DSA_ERR_CUDA;
  return DSA_OK;
}

dsa_status dsa_selftest_wait(dsa_stream_t stream) {
  DeviceInfo dev;
  const dsa_status ds = current_device(dev);
  if (ds != DSA_OK) return ds;
  wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
  return launch_result();
}

dsa_status dsa_last_device_status(dsa_stream_t stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return DSA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return DSA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return DSA_ERR_CUDA;
  return static_cast<dsa_status>(v & 0xFF);
}

}  // extern "C"
