// Sparse-stage indexer loss ("DSA Continued Pre-Training" page, Stage 2; "DeepSeek-V3.2"
// analysis page, eq. (4)):  L^I = sum_t KL(p[t,S_t] || Softmax(I[t,S_t])), and in dense mode the
// warm-up loss of eq. (3) (Stage 1), the same sum over every s <= t (idx = NULL, k = Lk, slot j is
// position j).
// Per row (one CTA): gather I[t, idx], log-sum-exp over the valid slots, then
// sum_j p_j (ln p_j - (I_j - lse)) with 0 ln 0 = 0, all in fp32.  The sum over rows runs
// in a second single-CTA kernel in a fixed order (fp64 accumulation), so the loss is
// deterministic.
#pragma once

#include <cuda_runtime.h>

#include "ptx.cuh"

namespace dsa {
namespace kl {

constexpr int kRowThreads = 256;
constexpr int kSumThreads = 1024;

__device__ __forceinline__ float block_reduce_max(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = -INFINITY;
  for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) r = fmaxf(r, red[w]);
  __syncthreads();
  return r;
}

__device__ __forceinline__ float block_reduce_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = 0.f;
  for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) r += red[w];
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kRowThreads)
    kl_rows_kernel(const float* __restrict__ scores, const int32_t* __restrict__ idx,
                   const float* __restrict__ p_sel, int Lq, int Lk, int k, float* __restrict__ kl_rows) {
  __shared__ float red[32];
  pdl_launch_dependents();
  pdl_wait();
  const size_t row = blockIdx.x;
  const float* srow = scores + row * Lk;
  const bool dense = idx == nullptr;
  const int32_t* irow = dense ? nullptr : idx + row * k;
  const float* prow = p_sel + row * k;
  // slots of this row: the k selected ones, or every visible position s <= t in dense mode
  const int n = dense ? min(k, static_cast<int>(row % Lq) + Lk - Lq + 1) : k;
  auto pos = [&](int j) { return dense ? j : __ldg(irow + j); };
  float m = -INFINITY;
  for (int j = threadIdx.x; j < n; j += kRowThreads) {
    const int s = pos(j);
    if (static_cast<unsigned>(s) < static_cast<unsigned>(Lk)) m = fmaxf(m, __ldg(srow + s));
  }
  m = block_reduce_max(m, red);
  float z = 0.f;
  for (int j = threadIdx.x; j < n; j += kRowThreads) {
    const int s = pos(j);
    if (static_cast<unsigned>(s) < static_cast<unsigned>(Lk)) z += expf(__ldg(srow + s) - m);
  }
  z = block_reduce_sum(z, red);
  const float lse = m + logf(z);
  float acc = 0.f;
  for (int j = threadIdx.x; j < n; j += kRowThreads) {
    const int s = pos(j);
    const float pj = __ldg(prow + j);
    if (static_cast<unsigned>(s) < static_cast<unsigned>(Lk) && pj > 0.f)
      acc += pj * (logf(pj) - (__ldg(srow + s) - lse));
  }
  acc = block_reduce_sum(acc, red);
  if (threadIdx.x == 0) kl_rows[row] = acc;
}

__global__ void __launch_bounds__(kSumThreads)
    kl_sum_kernel(const float* __restrict__ kl_rows, int rows, float* __restrict__ loss) {
  __shared__ double red[kSumThreads];
  pdl_launch_dependents();
  pdl_wait();
  double acc = 0.0;
  for (int r = threadIdx.x; r < rows; r += kSumThreads) acc += static_cast<double>(kl_rows[r]);
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int w = kSumThreads / 2; w > 0; w >>= 1) {
    if (static_cast<int>(threadIdx.x) < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) *loss = static_cast<float>(red[0]);
}

}  // namespace kl
}  // namespace dsa
