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
// partial loads are in flight.  Up to 256 splits (two per thread for the
// weights).  The same kernel, with an fp32 output, merges one rank's splits
// into a single partial per row, and, with the partials laid out one per rank,
// merges the ranks' partials of a sequence-sharded decode (the same merge one
// level up).
#include <cstdint>
#include <cuda_bf16.h>

#include "kernels.cuh"

namespace mla {

constexpr int kCombineThreads = 128;
constexpr int kCombineGroup = 64;  // partial loads in flight per thread

// Where the partials of a row live: partial s of row r starts at
// part_o + r * o_row + s * o_split (512 fp32) with its LSE at
// part_lse[r * l_row + s * l_split].  The split-KV workspace has o_split = 512,
// o_row = max_splits * 512; partials gathered from several ranks, one per
// rank, have o_split = rows * 512, o_row = 512.
struct PartialLayout {
  int64_t o_row, o_split, l_row, l_split;
};

template <bool kOutF32>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(
    const float* __restrict__ part_o, const float* __restrict__ part_lse,
    const int32_t* __restrict__ num_splits, int splits_const, int max_splits, int rows_per_batch,
    PartialLayout lay, void* __restrict__ out, float* __restrict__ out_lse) {
  extern __shared__ float w_smem[];  // [max_splits] split weights
  __shared__ float red[2][kCombineThreads / 32];
  const int row = blockIdx.x;
  const int d = blockIdx.y * kCombineThreads + threadIdx.x;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int b = row / rows_per_batch;
  const float* po = part_o + (int64_t)row * lay.o_row + d;
  const float* pl = part_lse + (int64_t)row * lay.l_row;

  // launched as a programmatic dependent of the kernel before it on the
  // stream: everything above overlapped that kernel's tail; memory it may have
  // written (the partials, and num_splits too) is read only after it completes
  asm volatile("griddepcontrol.wait;" ::: "memory");
  int S = num_splits != nullptr ? num_splits[b] : splits_const;
  S = S < 0 ? 0 : (S > max_splits ? max_splits : S);

  // issue the first group of partial loads before anything else
  float v[kCombineGroup];
#pragma unroll
  for (int j = 0; j < kCombineGroup; ++j) v[j] = (j < S) ? __ldg(po + (int64_t)j * lay.o_split) : 0.0f;

  // split weights while those loads are in flight: M = max LSE, w_s = e^(LSE_s - M)
  float lse[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int sidx = threadIdx.x + k * kCombineThreads;
    lse[k] = sidx < S ? pl[(int64_t)sidx * lay.l_split] : -INFINITY;
  }
  float m = fmaxf(lse[0], lse[1]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[0][wid] = m;
  __syncthreads();
  m = fmaxf(fmaxf(red[0][0], red[0][1]), fmaxf(red[0][2], red[0][3]));
  float wpart = 0.0f;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int sidx = threadIdx.x + k * kCombineThreads;
    const float w = (lse[k] == -INFINITY) ? 0.0f : expf(lse[k] - m);
    if (sidx < S) w_smem[sidx] = w;
    wpart += w;
  }
  // fixed-shape tree sum of the weights (deterministic)
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) wpart += __shfl_xor_sync(0xffffffffu, wpart, o);
  if (lane == 0) red[1][wid] = wpart;
  __syncthreads();
  const float wsum = (red[1][0] + red[1][1]) + (red[1][2] + red[1][3]);

  // accumulate in four independent chains, summed in a fixed order
  float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  for (int g0 = 0; g0 < S; g0 += kCombineGroup) {
    if (g0 > 0) {
#pragma unroll
      for (int j = 0; j < kCombineGroup; ++j)
        v[j] = (g0 + j < S) ? __ldg(po + (int64_t)(g0 + j) * lay.o_split) : 0.0f;
    }
#pragma unroll
    for (int j = 0; j < kCombineGroup; ++j)
      if (g0 + j < S) acc[j & 3] = fmaf(w_smem[g0 + j], v[j], acc[j & 3]);
  }
  const float a = (acc[0] + acc[1]) + (acc[2] + acc[3]);

  const bool empty = (m == -INFINITY) || !(wsum > 0.0f);
  const float o = empty ? 0.0f : a / wsum;
  if (kOutF32)
    static_cast<float*>(out)[(int64_t)row * 512 + d] = o;
  else
    static_cast<uint16_t*>(out)[(int64_t)row * 512 + d] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
  if (out_lse != nullptr && blockIdx.y == 0 && threadIdx.x == 0)
    out_lse[row] = empty ? -INFINITY : m + logf(wsum);
}

template <bool kOutF32>
static cudaError_t launch_combine_any(const float* part_o, const float* part_lse,
                                      const int32_t* num_splits, int splits_const, int max_splits,
                                      int rows, int rows_per_batch, const PartialLayout& lay,
                                      void* out, float* out_lse, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(rows, 512 / kCombineThreads);
  cfg.blockDim = dim3(kCombineThreads);
  cfg.dynamicSmemBytes = sizeof(float) * (size_t)max_splits;
  cfg.stream = stream;
  // programmatic dependent launch: the grid may be scheduled while the
  // kernel before it on the stream is still running
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, combine_kernel<kOutF32>, part_o, part_lse, num_splits,
                            splits_const, max_splits, rows_per_batch, lay, out, out_lse);
}

cudaError_t launch_combine(const float* part_o, const float* part_lse, const int32_t* num_splits,
                           int max_splits, int B, int q_len, int H, uint16_t* out, float* out_lse,
                           cudaStream_t stream) {
  const PartialLayout lay = {(int64_t)max_splits * 512, 512, max_splits, 1};
  return launch_combine_any<false>(part_o, part_lse, num_splits, 0, max_splits, B * q_len * H,
                                   q_len * H, lay, out, out_lse, stream);
}

cudaError_t launch_combine_f32(const float* part_o, const float* part_lse,
                               const int32_t* num_splits, int max_splits, int B, int q_len, int H,
                               float* out, float* out_lse, cudaStream_t stream) {
  const PartialLayout lay = {(int64_t)max_splits * 512, 512, max_splits, 1};
  return launch_combine_any<true>(part_o, part_lse, num_splits, 0, max_splits, B * q_len * H,
                                  q_len * H, lay, out, out_lse, stream);
}

cudaError_t launch_merge_ranks(const float* rank_o, const float* rank_lse, int n_ranks, int rows,
                               uint16_t* out, float* out_lse, cudaStream_t stream) {
  const PartialLayout lay = {512, (int64_t)rows * 512, 1, rows};
  return launch_combine_any<false>(rank_o, rank_lse, nullptr, n_ranks, n_ranks, rows, rows, lay,
                                   out, out_lse, stream);
}

}  // namespace mla
