// KV append, the step before the decode path: each new token's latent (512)
// and RoPE key (64) go into the paged FP8 cache in one kernel.
//
// "Muse Spark Open" article (theainews.cc), section "内核优化：解码吞吐 3 倍",
// bullet "RoPE 与 KV 缓存写入融合": the rotary embedding is applied by the same
// kernel that writes the decode KV cache, so no separate kernel runs for it.
// "SGLang & Miles ... Vera Rubin" article, bullet "原生 FP8 转换": the cache
// holds saturating E4M3 codes (overflow clamps to +-448, never NaN), produced
// by the packed hardware conversion.
//
// Token j of request b has position pos = seq_lens[b] - n_new + j and goes to
// row pos % 64 of page block_table[b][pos / 64]:
//   latent dim d:  code = E4M3_satfinite(fl32(x_d * inv_scale))
//   RoPE pair i:   (c, s) = cos_sin[pos][i]; in fp32 with every operation
//                  rounded (no fused multiply-add) y0 = x0 c - x1 s,
//                  y1 = x0 s + x1 c; codes E4M3_satfinite(fl32(y * inv_scale))
// (pairs are consecutive dims 2i, 2i+1: the original rotary embedding).
//
// One warp per token, grid-stride over the tokens: lane l converts latent
// dims 16l .. 16l+15 (two 16-byte loads, one 16-byte store) and RoPE pair l.
// A short decode append is launch-latency bound; a long one (a prompt) is an
// HBM stream of 1152 bytes in and 576 out per token.
#include <cstdint>

#include "kernels.cuh"
#include "mla.h"
#include "ptx.cuh"

namespace mla {

constexpr int kAppendThreads = 256;

__global__ void __launch_bounds__(kAppendThreads) append_kv_fp8_kernel(AppendArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (kAppendThreads / 32);
  const int64_t tokens = (int64_t)a.B * a.n_new;
  for (int64_t tk = (int64_t)blockIdx.x * (kAppendThreads / 32) + (threadIdx.x >> 5); tk < tokens;
       tk += warps) {
    const int b = (int)(tk / a.n_new);
    const int j = (int)(tk % a.n_new);
    const int64_t pos = (int64_t)a.seq_lens[b] - a.n_new + j;
    if (pos < 0 || pos >= a.max_pos || pos / 64 >= a.max_pages) {
      if (lane == 0 && a.dev_error != nullptr) atomicOr(a.dev_error, MLA_DEVERR_BAD_SEQLEN);
      continue;
    }
    const int64_t page = a.block_table[(int64_t)b * a.max_pages + pos / 64];
    if (page < 0 || page >= a.num_pages) {
      if (lane == 0 && a.dev_error != nullptr) atomicOr(a.dev_error, MLA_DEVERR_BAD_PAGE);
      continue;
    }
    uint8_t* row = a.kv_pages + (page * 64 + pos % 64) * 576;
    // latent: 16 dims per lane
    const uint4* src = reinterpret_cast<const uint4*>(a.c_kv + tk * 512 + 16 * lane);
    const uint4 v0 = src[0], v1 = src[1];
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    uint32_t codes[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t lo = cvt_e4m3x2(__fmul_rn(__uint_as_float(w[2 * k] << 16), a.inv_scale),
                                     __fmul_rn(__uint_as_float(w[2 * k] & 0xFFFF0000u), a.inv_scale));
      const uint32_t hi =
          cvt_e4m3x2(__fmul_rn(__uint_as_float(w[2 * k + 1] << 16), a.inv_scale),
                     __fmul_rn(__uint_as_float(w[2 * k + 1] & 0xFFFF0000u), a.inv_scale));
      codes[k] = lo | (hi << 16);
    }
    *reinterpret_cast<uint4*>(row + 16 * lane) = make_uint4(codes[0], codes[1], codes[2], codes[3]);
    // RoPE pair `lane`
    const uint32_t xr = *reinterpret_cast<const uint32_t*>(a.k_rope + tk * 64 + 2 * lane);
    const float x0 = __uint_as_float(xr << 16), x1 = __uint_as_float(xr & 0xFFFF0000u);
    const float2 cs = *reinterpret_cast<const float2*>(a.cos_sin + (pos * 32 + lane) * 2);
    const float y0 = __fsub_rn(__fmul_rn(x0, cs.x), __fmul_rn(x1, cs.y));
    const float y1 = __fadd_rn(__fmul_rn(x0, cs.y), __fmul_rn(x1, cs.x));
    const uint32_t rc = cvt_e4m3x2(__fmul_rn(y0, a.inv_scale), __fmul_rn(y1, a.inv_scale));
    *reinterpret_cast<uint16_t*>(row + 512 + 2 * lane) = (uint16_t)rc;
  }
}

cudaError_t launch_append_kv_fp8(const AppendArgs& a, int num_sms, cudaStream_t stream) {
  const int64_t tokens = (int64_t)a.B * a.n_new;
  if (tokens == 0) return cudaSuccess;
  const int64_t per_block = kAppendThreads / 32;
  int64_t blocks = (tokens + per_block - 1) / per_block;
  const int64_t cap = (int64_t)num_sms * 8;  // 64 warps per SM: enough loads in flight for a stream
  if (blocks > cap) blocks = cap;
  append_kv_fp8_kernel<<<(unsigned)blocks, kAppendThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace mla
