// Step A1, the prep kernel: saturating bf16 -> FP8 E4M3 conversion.
//
// "SGLang & Miles ... Vera Rubin" article, section "Kimi K3 的 MLA", bullet
// "原生 FP8 转换": converting KV/Q to FP8 without saturation keeps the compiler
// off the packed hardware conversion; with a saturating conversion (overflow
// clamps to +-448 instead of NaN) the prep kernel was 2.5x faster.  Here every
// pair of values goes through one packed cvt.rn.satfinite.e4m3x2.f32.
//
// y[i] = E4M3_RN_satfinite(fl32(float(x[i]) * inv_scale)).  The kernel is a
// pure HBM stream (2 bytes in, 1 byte out per element): each thread issues
// eight 16-byte non-allocating loads (two 32-element groups, 128 bytes of
// bf16) before converting, and writes 64 bytes of codes, grid-stride over a
// grid of four 256-thread blocks per SM (128 KiB of loads in flight per SM).
#include <cstdint>

#include "kernels.cuh"
#include "ptx.cuh"

namespace mla {

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ void st_stream_v4(void* p, uint4 v) {
  asm volatile("st.global.L1::no_allocate.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x),
               "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// Two bf16 (one 32-bit word, element 0 in the low half) -> two codes.
__device__ __forceinline__ uint32_t quant_pair(uint32_t w, float inv_scale) {
  const float a = __fmul_rn(__uint_as_float(w << 16), inv_scale);
  const float b = __fmul_rn(__uint_as_float(w & 0xFFFF0000u), inv_scale);
  return cvt_e4m3x2(a, b);
}
// Four bf16 (two words) -> four codes packed little-endian in one word.
__device__ __forceinline__ uint32_t quant_quad(uint32_t w0, uint32_t w1, float inv_scale) {
  return quant_pair(w0, inv_scale) | (quant_pair(w1, inv_scale) << 16);
}

__global__ void __launch_bounds__(256) quantize_fp8_vec_kernel(const uint16_t* __restrict__ x,
                                                               uint8_t* __restrict__ y,
                                                               int64_t n32, float inv_scale) {
  // n32 = number of 32-element groups; x and y are 16-byte aligned.  Each
  // thread handles two groups per iteration, all eight loads issued first.
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (; g + stride < n32; g += 2 * stride) {
    const uint16_t* s0 = x + g * 32;
    const uint16_t* s1 = x + (g + stride) * 32;
    uint4 v[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) v[k] = ld_stream_v4(s0 + 8 * k);
#pragma unroll
    for (int k = 0; k < 4; ++k) v[4 + k] = ld_stream_v4(s1 + 8 * k);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint4 o0, o1;
      o0.x = quant_quad(v[4 * h + 0].x, v[4 * h + 0].y, inv_scale);
      o0.y = quant_quad(v[4 * h + 0].z, v[4 * h + 0].w, inv_scale);
      o0.z = quant_quad(v[4 * h + 1].x, v[4 * h + 1].y, inv_scale);
      o0.w = quant_quad(v[4 * h + 1].z, v[4 * h + 1].w, inv_scale);
      o1.x = quant_quad(v[4 * h + 2].x, v[4 * h + 2].y, inv_scale);
      o1.y = quant_quad(v[4 * h + 2].z, v[4 * h + 2].w, inv_scale);
      o1.z = quant_quad(v[4 * h + 3].x, v[4 * h + 3].y, inv_scale);
      o1.w = quant_quad(v[4 * h + 3].z, v[4 * h + 3].w, inv_scale);
      uint8_t* dst = y + (g + h * stride) * 32;
      st_stream_v4(dst, o0);
      st_stream_v4(dst + 16, o1);
    }
  }
  if (g < n32) {
    const uint16_t* src = x + g * 32;
    const uint4 a = ld_stream_v4(src);
    const uint4 b = ld_stream_v4(src + 8);
    const uint4 c = ld_stream_v4(src + 16);
    const uint4 d = ld_stream_v4(src + 24);
    uint4 o0, o1;
    o0.x = quant_quad(a.x, a.y, inv_scale);
    o0.y = quant_quad(a.z, a.w, inv_scale);
    o0.z = quant_quad(b.x, b.y, inv_scale);
    o0.w = quant_quad(b.z, b.w, inv_scale);
    o1.x = quant_quad(c.x, c.y, inv_scale);
    o1.y = quant_quad(c.z, c.w, inv_scale);
    o1.z = quant_quad(d.x, d.y, inv_scale);
    o1.w = quant_quad(d.z, d.w, inv_scale);
    st_stream_v4(y + g * 32, o0);
    st_stream_v4(y + g * 32 + 16, o1);
  }
}

// Element-wise path for unaligned pointers and for the tail.
__global__ void __launch_bounds__(256) quantize_fp8_scalar_kernel(const uint16_t* __restrict__ x,
                                                                  uint8_t* __restrict__ y,
                                                                  int64_t n, float inv_scale) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    const float v = __fmul_rn(__uint_as_float((uint32_t)x[i] << 16), inv_scale);
    y[i] = (uint8_t)(cvt_e4m3x2(v, 0.0f) & 0xFFu);
  }
}

cudaError_t launch_quantize_fp8(const uint16_t* x, uint8_t* y, int64_t n, float inv_scale,
                                int num_sms, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const bool aligned = ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(y)) & 15) == 0;
  int64_t done = 0;
  if (aligned) {
    const int64_t n32 = n / 32;
    if (n32 > 0) {
      int64_t blocks = (n32 + 255) / 256;
      const int64_t cap = (int64_t)num_sms * 4;
      if (blocks > cap) blocks = cap;
      quantize_fp8_vec_kernel<<<(unsigned)blocks, 256, 0, stream>>>(x, y, n32, inv_scale);
      done = n32 * 32;
    }
  }
  if (done < n) {
    const int64_t rem = n - done;
    int64_t blocks = (rem + 255) / 256;
    const int64_t cap = (int64_t)num_sms * 8;
    if (blocks > cap) blocks = cap;
    quantize_fp8_scalar_kernel<<<(unsigned)blocks, 256, 0, stream>>>(x + done, y + done, rem,
                                                                      inv_scale);
  }
  return cudaGetLastError();
}

}  // namespace mla
