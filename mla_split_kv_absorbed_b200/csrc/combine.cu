// Step A9, the second kernel: log-sum-exp merge of the split partials.
//
// "SGLang & Miles ... Vera Rubin" article, section "Kimi K3 的 MLA", bullet
// "更快的 split-KV 归约": the merge used to load one partial, wait, then load
// the next, paying one L2 latency per partial; issuing every load first and
// then accumulating from registers made batch-1 / 128K FP8 MLA up to ~20%
// faster.  This kernel does exactly that: each thread owns one latent column
// of one row and issues the loads of all of its row's partials (in groups of
// up to 64 registers) before the first multiply-add.
//
// Per row: M = max_s LSE_s, w_s = e^{LSE_s - M}, O = sum w_s O_s / sum w_s,
// LSE = M + ln sum w_s.  Grid: (rows, 512 / 128), 128 threads; the split
// weights of the row are computed once per block into shared memory while the
// partial loads are in flight.
#include <cstdint>
#include <cuda_bf16.h>

#include "kernels.cuh"

namespace mla {

constexpr int kCombineThreads = 128;
constexpr int kCombineGroup = 64;  // partial loads in flight per thread

__global__ void __launch_bounds__(kCombineThreads) combine_kernel(
    const float* __restrict__ part_o, const float* __restrict__ part_lse,
    const int32_t* __restrict__ num_splits, int max_splits, int rows_per_batch,
    uint16_t* __restrict__ out, float* __restrict__ out_lse) {
  extern __shared__ float w_smem[];  // [max_splits] weights, then [1] inverse sum
  const int row = blockIdx.x;
  const int d = blockIdx.y * kCombineThreads + threadIdx.x;
  const int b = row / rows_per_batch;
  int S = num_splits[b];
  S = S < 0 ? 0 : (S > max_splits ? max_splits : S);
  const float* po = part_o + (size_t)row * max_splits * 512 + d;

  // issue the first group of partial loads before anything else
  float v[kCombineGroup];
#pragma unroll
  for (int j = 0; j < kCombineGroup; ++j) v[j] = (j < S) ? __ldg(po + (size_t)j * 512) : 0.0f;

  // split weights (overlaps the loads above)
  const float* pl = part_lse + (size_t)row * max_splits;
  __shared__ float red[kCombineThreads / 32];
  float m = -INFINITY;
  for (int s = threadIdx.x; s < S; s += kCombineThreads) m = fmaxf(m, pl[s]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  m = red[0];
#pragma unroll
  for (int i = 1; i < kCombineThreads / 32; ++i) m = fmaxf(m, red[i]);
  __syncthreads();
  float wsum_part = 0.0f;
  for (int s = threadIdx.x; s < S; s += kCombineThreads) {
    const float l = pl[s];
    const float w = (l == -INFINITY) ? 0.0f : expf(l - m);
    w_smem[s] = w;
  }
  __syncthreads();
  // every thread sums the weights in the same order (deterministic)
  for (int s = 0; s < S; ++s) wsum_part += w_smem[s];

  float acc = 0.0f;
  for (int g0 = 0; g0 < S; g0 += kCombineGroup) {
    if (g0 > 0) {
#pragma unroll
      for (int j = 0; j < kCombineGroup; ++j)
        v[j] = (g0 + j < S) ? __ldg(po + (size_t)(g0 + j) * 512) : 0.0f;
    }
#pragma unroll
    for (int j = 0; j < kCombineGroup; ++j)
      if (g0 + j < S) acc = fmaf(w_smem[g0 + j], v[j], acc);
  }

  const bool empty = (m == -INFINITY) || !(wsum_part > 0.0f);
  const float o = empty ? 0.0f : acc / wsum_part;
  out[(size_t)row * 512 + d] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
  if (out_lse != nullptr && blockIdx.y == 0 && threadIdx.x == 0)
    out_lse[row] = empty ? -INFINITY : m + logf(wsum_part);
}

cudaError_t launch_combine(const float* part_o, const float* part_lse, const int32_t* num_splits,
                           int max_splits, int B, int q_len, int H, uint16_t* out, float* out_lse,
                           cudaStream_t stream) {
  const int rows = B * q_len * H;
  if (rows == 0) return cudaSuccess;
  dim3 grid(rows, 512 / kCombineThreads);
  const size_t smem = sizeof(float) * (size_t)max_splits;
  combine_kernel<<<grid, kCombineThreads, smem, stream>>>(part_o, part_lse, num_splits, max_splits,
                                                          q_len * H, out, out_lse);
  return cudaGetLastError();
}

}  // namespace mla
