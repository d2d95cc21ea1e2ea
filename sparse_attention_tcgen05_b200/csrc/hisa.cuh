// HISA, block -> token retrieval for decode ("DeepSeek-V3.2" analysis page, sec. 5.3: a coarse
// stage over block representatives, then exact indexer scores inside the kept blocks; cost
// model eq. (25), recall decomposition eq. (24)).
//
// The cache is cut into blocks of `block` keys.  A block is represented by the mean of its keys;
// its coarse score for a query is the indexer's formula applied to that mean key,
//   score_B = sum_j w_j ReLU(q_j . mean_B) = (1 / n_B) sum_j w_j ReLU(q_j . sum_B),
// (n_B > 0 keys in the block).  The block sums are a cache summary, computed once when the
// cache is written (block_sums_kernel); the per-step coarse stage reads 1/block of the bytes
// the full indexer reads.  The kept blocks then act as the pages of a paged cache for the
// exact stage (the paged decode indexer and its fused top-k), and the selected candidate slots
// map back to positions (both orders are monotone, so ascending slots give ascending positions).
#pragma once

#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace dsa {
namespace hisa {

constexpr int kDI = 128;
constexpr int kSumThreads = 128;  // one dim per thread
constexpr int kScoreThreads = 128;  // one block per thread

__device__ __forceinline__ float e4m3_to_float(uint8_t b) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(b), __NV_E4M3);
  return __half2float(__half(h));
}

// sums[b, B, :] = sum of the keys of block B of sequence b (fp32; exact for integer-valued keys).
// Grid: B * n_blocks CTAs of 128 threads (thread = dim).
__global__ void __launch_bounds__(kSumThreads) block_sums_kernel(const uint8_t* __restrict__ k, int Lk, int block,
                                                                int n_blocks, float* __restrict__ sums) {
  pdl_launch_dependents();
  pdl_wait();
  const int bb = blockIdx.x;  // b * n_blocks + block index
  const int b = bb / n_blocks, blk = bb - b * n_blocks;
  const int s0 = blk * block, s1 = min(Lk, s0 + block);
  const uint8_t* base = k + static_cast<size_t>(b) * Lk * kDI + threadIdx.x;
  float acc = 0.f;
  for (int s = s0; s < s1; ++s) acc += e4m3_to_float(__ldg(base + static_cast<size_t>(s) * kDI));
  sums[static_cast<size_t>(bb) * kDI + threadIdx.x] = acc;
}

// Coarse scores of every block for the decode query of each sequence (t = Lk - 1: every block is
// visible, the last one may be short).  Grid: (B, ceil(n_blocks / 128)), 128 threads.
template <int H_I>
__global__ void __launch_bounds__(kScoreThreads) block_scores_kernel(const uint8_t* __restrict__ q,
                                                                    const float* __restrict__ w,
                                                                    const float* __restrict__ sums, int Lk,
                                                                    int block, int n_blocks,
                                                                    float* __restrict__ scores) {
  __shared__ float sq[H_I][kDI];
  __shared__ float sw[H_I];
  pdl_launch_dependents();
  pdl_wait();
  const int b = blockIdx.x;
  for (int x = threadIdx.x; x < H_I * kDI; x += kScoreThreads)
    sq[x / kDI][x % kDI] = e4m3_to_float(__ldg(q + static_cast<size_t>(b) * H_I * kDI + x));
  if (threadIdx.x < H_I) sw[threadIdx.x] = __ldg(w + static_cast<size_t>(b) * H_I + threadIdx.x);
  __syncthreads();
  const int blk = blockIdx.y * kScoreThreads + threadIdx.x;
  if (blk >= n_blocks) return;
  const float* sum = sums + (static_cast<size_t>(b) * n_blocks + blk) * kDI;
  float acc[H_I];
#pragma unroll
  for (int j = 0; j < H_I; ++j) acc[j] = 0.f;
#pragma unroll 1
  for (int d0 = 0; d0 < kDI; d0 += 16) {
    float v[16];
#pragma unroll
    for (int c = 0; c < 16; c += 4) {
      const float4 f = __ldg(reinterpret_cast<const float4*>(sum + d0 + c));
      v[c] = f.x;
      v[c + 1] = f.y;
      v[c + 2] = f.z;
      v[c + 3] = f.w;
    }
#pragma unroll
    for (int j = 0; j < H_I; ++j)
#pragma unroll
      for (int c = 0; c < 16; ++c) acc[j] = fmaf(sq[j][d0 + c], v[c], acc[j]);
  }
  float num = 0.f;
#pragma unroll
  for (int j = 0; j < H_I; ++j) num = fmaf(sw[j], fmaxf(acc[j], 0.f), num);
  const int n = min(block, Lk - blk * block);  // keys in the block (> 0)
  scores[static_cast<size_t>(b) * n_blocks + blk] = num / static_cast<float>(n);
}

// The kept blocks (ascending, per sequence) as page indices of the whole cache viewed as pages of
// `block` keys: page = b * n_blocks + block index.  Grid: B, threads: up to r (strided).
__global__ void block_pages_kernel(const int32_t* __restrict__ blocks, int r, int n_blocks,
                                   int32_t* __restrict__ pages) {
  pdl_launch_dependents();
  pdl_wait();
  const int b = blockIdx.x;
  for (int j = threadIdx.x; j < r; j += blockDim.x) {
    const int blk = __ldg(blocks + static_cast<size_t>(b) * r + j);
    pages[static_cast<size_t>(b) * r + j] = blk >= 0 ? b * n_blocks + blk : -1;
  }
}

// Selected candidate slots -> positions: slot c of sequence b is key
// blocks[b, c / block] * block + c % block.  Grid: B, threads strided over k.
__global__ void slots_to_positions_kernel(const int32_t* __restrict__ cand, const int32_t* __restrict__ blocks,
                                          int r, int block, int k, int32_t* __restrict__ idx) {
  pdl_launch_dependents();
  pdl_wait();
  const int b = blockIdx.x;
  for (int j = threadIdx.x; j < k; j += blockDim.x) {
    const int c = __ldg(cand + static_cast<size_t>(b) * k + j);
    int s = -1;
    if (c >= 0) {
      const int blk = __ldg(blocks + static_cast<size_t>(b) * r + c / block);
      s = blk >= 0 ? blk * block + c % block : -1;
    }
    idx[static_cast<size_t>(b) * k + j] = s;
  }
}

}  // namespace hisa
}  // namespace dsa
