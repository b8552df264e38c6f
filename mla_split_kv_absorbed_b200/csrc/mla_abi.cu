// C ABI of the library (declarations and contracts in include/mla.h):
// argument validation, TMA descriptor encoding and kernel launches.  Nothing
// here allocates, frees or synchronises; every launch goes to the caller's
// stream.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cmath>
#include <cstring>

#include "kernels.cuh"
#include "mla.h"

namespace {

std::atomic<int> g_inject_stall{0};  // mla_debug_inject_stall
std::atomic<int> g_merge_plan{0};    // mla_debug_merge_plan: 16 * V + gpi, 0 = automatic

constexpr int kPage = 64;
constexpr int kRow = 576;
constexpr int kSplitTokens = 2048;  // mla_choose_splits: the fewest tokens per split

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// SM count of the current device, looked up once per device (the partial
// kernel's grid plan depends on it; a process may drive several devices).
constexpr int kMaxDevices = 64;
std::atomic<int> g_num_sms[kMaxDevices] = {};

int num_sms_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
  if (dev < kMaxDevices) {
    const int cached = g_num_sms[dev].load(std::memory_order_relaxed);
    if (cached > 0) return cached;
  }
  int v = 0;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
    return 148;
  if (dev < kMaxDevices) g_num_sms[dev].store(v, std::memory_order_relaxed);
  return v;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// TMA map over kv_pages viewed as [num_pages][64][576] elements with a box of
// {box_x elements, 64 rows, 1 page} and the given swizzle.
int make_kv_map(CUtensorMap* map, const void* kv_pages, int kv_dtype, int64_t num_pages,
                cuuint32_t box_x, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return MLA_ERR_CUDA;
  const cuuint64_t esz = kv_dtype == MLA_KV_FP8_E4M3 ? 1 : 2;
  const cuuint64_t dims[3] = {(cuuint64_t)kRow, (cuuint64_t)kPage, (cuuint64_t)num_pages};
  const cuuint64_t strides[2] = {kRow * esz, (cuuint64_t)kPage * kRow * esz};
  const cuuint32_t box[3] = {box_x, 64, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map,
                        kv_dtype == MLA_KV_FP8_E4M3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                                    : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                        3, const_cast<void*>(kv_pages), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_INVALID_ARG;
}

int status_of(cudaError_t e) { return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA; }

// FP8 partial-kernel grid over units (64-row query group, split, request).
// When the units fill at most half of the SMs, every split is cut into 2 or 4
// runs of tiles, one CTA each, merged on chip by its cluster; when they fill
// several waves and the last wave is at most half full, only the units of that
// last wave are cut in two.  The partial per split is the same either way.
// out = {CTAs, pieces, first cut unit, idle CTAs before the cut units}.
void plan_grid(int B, int q_len, int H, int max_splits, int kv_dtype, int sms, int32_t* out) {
  const long long groups = (q_len * H + 63) / 64;
  const long long units = groups * max_splits * B;
  int pieces = 1;
  long long split_from = units;
  if (kv_dtype == MLA_KV_FP8_E4M3 && sms > 0) {
    if (units * 2 <= sms) {
      while (pieces < 4 && units * pieces * 2 <= sms) pieces *= 2;
      split_from = 0;
    } else if (units > sms) {
      const long long tail = units % sms;
      if (tail > 0 && tail * 2 <= sms) {
        pieces = 2;
        split_from = units - tail;
      }
    }
  }
  const long long pad = pieces > 1 ? (pieces - split_from % pieces) % pieces : 0;
  out[0] = (int32_t)(split_from + pad + (units - split_from) * pieces);
  out[1] = pieces;
  out[2] = (int32_t)split_from;
  out[3] = (int32_t)pad;
}

}  // namespace

extern "C" {

int mla_quantize_fp8(const uint16_t* x_bf16, uint8_t* y_e4m3, int64_t n, float inv_scale,
                     void* stream) {
  if (n < 0) return MLA_ERR_INVALID_ARG;
  if (n == 0) return MLA_OK;
  if (x_bf16 == nullptr || y_e4m3 == nullptr) return MLA_ERR_INVALID_ARG;
  return status_of(mla::launch_quantize_fp8(x_bf16, y_e4m3, n, inv_scale, num_sms_current_device(),
                                            static_cast<cudaStream_t>(stream)));
}

size_t mla_partial_workspace_bytes(int B, int q_len, int H, int max_splits) {
  if (B <= 0 || q_len <= 0 || H <= 0 || max_splits <= 0) return 0;
  const size_t rows = (size_t)B * q_len * H * max_splits;
  return rows * 512 * sizeof(float) + rows * sizeof(float);
}

}  // extern "C"

namespace {

// Checks shared by the partial and the single-launch entry points; fills the
// kernel arguments (all but the output pointers) and the tensor maps.
int setup_decode(const uint16_t* q_nope, const uint16_t* q_rope, const void* kv_pages, int kv_dtype,
                 float kv_scale, int64_t num_pages, const int32_t* block_table,
                 int max_pages_per_req, const int32_t* seq_lens, const int32_t* num_splits,
                 int max_splits, int B, int q_len, int H, float softmax_scale,
                 int32_t* dev_error, mla::DecodeArgs* a, CUtensorMap* map, CUtensorMap* rope_map,
                 int splits_const = 0) {
  // splits_const > 0: every request has max_splits splits and num_splits is unused
  if (q_nope == nullptr || q_rope == nullptr || kv_pages == nullptr || block_table == nullptr ||
      seq_lens == nullptr || (num_splits == nullptr && splits_const == 0))
    return MLA_ERR_INVALID_ARG;
  if (!aligned16(q_nope) || !aligned16(q_rope) || !aligned16(kv_pages)) return MLA_ERR_INVALID_ARG;
  if (B <= 0 || q_len <= 0 || H <= 0 || num_pages <= 0 || max_pages_per_req <= 0 ||
      max_splits <= 0)
    return MLA_ERR_INVALID_ARG;
  if (num_pages > 0x7FFFFFFFll || (int64_t)max_pages_per_req * kPage > 0x7FFFFFFFll)
    return MLA_ERR_INVALID_ARG;
  if (kv_dtype != MLA_KV_FP8_E4M3 && kv_dtype != MLA_KV_BF16) return MLA_ERR_INVALID_ARG;
  if (!(softmax_scale == softmax_scale) || !(kv_scale == kv_scale) || kv_scale <= 0.0f)
    return MLA_ERR_INVALID_ARG;
  if (kv_dtype == MLA_KV_BF16 && kv_scale != 1.0f) return MLA_ERR_INVALID_ARG;
  if (q_len > 4 || q_len * H > 512 || max_splits > 256 || B > 65535 || (q_len * H) % 16 != 0)
    return MLA_ERR_UNSUPPORTED;

  // FP8: the latent dims as 128-byte rows (128-byte swizzle) and the RoPE dims
  // as 64-byte rows (64-byte swizzle); bf16: 64-element (128-byte) rows
  std::memset(map, 0, sizeof(*map));
  std::memset(rope_map, 0, sizeof(*rope_map));
  int st = kv_dtype == MLA_KV_FP8_E4M3
               ? make_kv_map(map, kv_pages, kv_dtype, num_pages, 128, CU_TENSOR_MAP_SWIZZLE_128B)
               : make_kv_map(map, kv_pages, kv_dtype, num_pages, 64, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != MLA_OK) return st;
  if (kv_dtype == MLA_KV_FP8_E4M3) {
    st = make_kv_map(rope_map, kv_pages, kv_dtype, num_pages, 64, CU_TENSOR_MAP_SWIZZLE_64B);
    if (st != MLA_OK) return st;
  }

  *a = mla::DecodeArgs{};
  a->q_nope = q_nope;
  a->q_rope = q_rope;
  a->kv_pages = static_cast<const uint8_t*>(kv_pages);
  a->block_table = block_table;
  a->seq_lens = seq_lens;
  a->num_splits = num_splits;
  a->splits_const = splits_const > 0 ? max_splits : 0;
  a->dev_error = dev_error;
  a->num_pages = num_pages;
  a->max_pages = max_pages_per_req;
  a->max_splits = max_splits;
  a->B = B;
  a->q_len = q_len;
  a->H = H;
  a->qk_scale_log2 = softmax_scale * kv_scale * 1.4426950408889634f;
  a->kv_scale = kv_scale;
  a->inject_stall = g_inject_stall.load(std::memory_order_relaxed);
  const int plan_mv = g_merge_plan.load(std::memory_order_relaxed);
  a->merge_v = plan_mv >> 4;  // 0: the launcher chooses
  a->merge_gpi = plan_mv & 15;
  int32_t plan[4];
  plan_grid(B, q_len, H, max_splits, kv_dtype, num_sms_current_device(), plan);
  a->groups = (q_len * H + 63) / 64;
  a->pieces = plan[1];
  a->split_from = plan[2];
  a->pad = plan[3];
  return MLA_OK;
}

constexpr size_t kFusedCounterBytes = 256;  // two int32 counters, padded
constexpr int kFusedMaxEntries = 256;       // splits per row the single launch's merge takes

}  // namespace

extern "C" {

int mla_decode_partial(const uint16_t* q_nope, const uint16_t* q_rope, const void* kv_pages,
                       int kv_dtype, float kv_scale, int64_t num_pages,
                       const int32_t* block_table, int max_pages_per_req,
                       const int32_t* seq_lens, const int32_t* num_splits, int max_splits, int B,
                       int q_len, int H, float softmax_scale, float* part_o, float* part_lse,
                       int32_t* dev_error, void* stream) {
  if (part_o == nullptr || part_lse == nullptr || !aligned16(part_o)) return MLA_ERR_INVALID_ARG;
  mla::DecodeArgs a;
  CUtensorMap map, rope_map;
  const int st = setup_decode(q_nope, q_rope, kv_pages, kv_dtype, kv_scale, num_pages, block_table,
                              max_pages_per_req, seq_lens, num_splits, max_splits, B, q_len, H,
                              softmax_scale, dev_error, &a, &map, &rope_map);
  if (st != MLA_OK) return st;
  a.part_o = part_o;
  a.part_lse = part_lse;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return status_of(kv_dtype == MLA_KV_FP8_E4M3 ? mla::launch_decode_fp8(a, map, rope_map, s)
                                               : mla::launch_decode_bf16(a, map, s));
}

int mla_decode_partial_q8(const uint8_t* q8, float q_scale, const void* kv_pages, float kv_scale,
                          int64_t num_pages, const int32_t* block_table, int max_pages_per_req,
                          const int32_t* seq_lens, const int32_t* num_splits, int max_splits,
                          int B, int q_len, int H, float softmax_scale, float* part_o,
                          float* part_lse, int32_t* dev_error, void* stream) {
  if (q8 == nullptr || !aligned16(q8) || part_o == nullptr || part_lse == nullptr ||
      !aligned16(part_o))
    return MLA_ERR_INVALID_ARG;
  if (!(q_scale > 0.0f) || !(q_scale < INFINITY)) return MLA_ERR_INVALID_ARG;
  mla::DecodeArgs a;
  CUtensorMap map, rope_map;
  // the query pointers of the bf16 form are not read in this mode: q8 stands in
  const uint16_t* qq = reinterpret_cast<const uint16_t*>(q8);
  const int st = setup_decode(qq, qq, kv_pages, MLA_KV_FP8_E4M3, kv_scale, num_pages, block_table,
                              max_pages_per_req, seq_lens, num_splits, max_splits, B, q_len, H,
                              softmax_scale, dev_error, &a, &map, &rope_map);
  if (st != MLA_OK) return st;
  a.part_o = part_o;
  a.part_lse = part_lse;
  a.q8 = q8;
  a.q_scale = q_scale;
  return status_of(mla::launch_decode_fp8(a, map, rope_map, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {

// Split count of the single launch: every request cut into as many splits as
// one wave of CTAs allows, one CTA per (row group, split, request).
int fused_splits(int B, int q_len, int H, int num_sms) {
  const long long units_per_split = (long long)((q_len * H + 63) / 64) * B;
  if (units_per_split <= 0 || num_sms <= 0) return 0;
  long long S = num_sms / units_per_split;
  return (int)(S > kFusedMaxEntries ? kFusedMaxEntries : S);
}

// counters, then the entries' O (fp16), then their LSE (fp32)
size_t fused_bytes(int B, int q_len, int H, int S) {
  const size_t entries = (size_t)B * q_len * H * S;
  return kFusedCounterBytes + entries * 512 * sizeof(uint16_t) + entries * sizeof(float);
}

}  // namespace

extern "C" {

int mla_fused_splits(int B, int q_len, int H, int num_sms) {
  if (B <= 0 || q_len <= 0 || H <= 0 || num_sms <= 0) return 0;
  return fused_splits(B, q_len, H, num_sms);
}

size_t mla_fused_workspace_bytes(int B, int q_len, int H, int num_sms) {
  if (B <= 0 || q_len <= 0 || H <= 0 || num_sms <= 0) return 0;
  const int S = fused_splits(B, q_len, H, num_sms);
  return S < 1 ? 0 : fused_bytes(B, q_len, H, S);
}

int mla_decode_fused(const uint16_t* q_nope, const uint16_t* q_rope, const void* kv_pages,
                     int kv_dtype, float kv_scale, int64_t num_pages, const int32_t* block_table,
                     int max_pages_per_req, const int32_t* seq_lens, int B, int q_len, int H,
                     float softmax_scale, void* workspace, size_t workspace_bytes,
                     uint16_t* out_bf16, float* out_lse, int32_t* dev_error, void* stream) {
  if (workspace == nullptr || out_bf16 == nullptr || !aligned16(workspace))
    return MLA_ERR_INVALID_ARG;
  if (B <= 0 || q_len <= 0 || H <= 0) return MLA_ERR_INVALID_ARG;
  // one launch only when every CTA of the grid is resident at once: an FP8
  // cache and at least one split per (row group, request) in one wave
  const int S = fused_splits(B, q_len, H, num_sms_current_device());
  if (kv_dtype != MLA_KV_FP8_E4M3 || S < 1) return MLA_ERR_UNSUPPORTED;
  if (workspace_bytes < fused_bytes(B, q_len, H, S)) return MLA_ERR_INVALID_ARG;
  mla::DecodeArgs a;
  CUtensorMap map, rope_map;
  const int st = setup_decode(q_nope, q_rope, kv_pages, kv_dtype, kv_scale, num_pages, block_table,
                              max_pages_per_req, seq_lens, nullptr, S, B, q_len, H,
                              softmax_scale, dev_error, &a, &map, &rope_map, /*splits_const=*/1);
  if (st != MLA_OK) return st;
  const int units = a.groups * S * B;
  a.pieces = 1;  // one CTA per unit, no cluster: the grid is exactly one wave
  a.split_from = units;
  a.pad = 0;
  const size_t entries = (size_t)B * q_len * H * S;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.fused = 1;
  a.sync = reinterpret_cast<int32_t*>(ws);
  a.part_o = nullptr;
  a.part_o16 = reinterpret_cast<uint16_t*>(ws + kFusedCounterBytes);
  a.part_lse = reinterpret_cast<float*>(a.part_o16 + entries * 512);
  a.out = out_bf16;
  a.out_lse = out_lse;
  return status_of(mla::launch_decode_fp8(a, map, rope_map, static_cast<cudaStream_t>(stream)));
}

int mla_combine(const float* part_o, const float* part_lse, const int32_t* num_splits,
                int max_splits, int B, int q_len, int H, uint16_t* out_bf16, float* out_lse,
                void* stream) {
  if (part_o == nullptr || part_lse == nullptr || num_splits == nullptr || out_bf16 == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (B <= 0 || q_len <= 0 || H <= 0 || max_splits <= 0) return MLA_ERR_INVALID_ARG;
  if (max_splits > 256 || q_len > 4 || q_len * H > 512) return MLA_ERR_UNSUPPORTED;
  return status_of(mla::launch_combine(part_o, part_lse, num_splits, max_splits, B, q_len, H,
                                       out_bf16, out_lse, static_cast<cudaStream_t>(stream)));
}

int mla_combine_f32(const float* part_o, const float* part_lse, const int32_t* num_splits,
                    int max_splits, int B, int q_len, int H, float* out_o, float* out_lse,
                    void* stream) {
  if (part_o == nullptr || part_lse == nullptr || num_splits == nullptr || out_o == nullptr ||
      out_lse == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (B <= 0 || q_len <= 0 || H <= 0 || max_splits <= 0) return MLA_ERR_INVALID_ARG;
  if (max_splits > 256 || q_len > 4 || q_len * H > 512) return MLA_ERR_UNSUPPORTED;
  return status_of(mla::launch_combine_f32(part_o, part_lse, num_splits, max_splits, B, q_len, H,
                                           out_o, out_lse, static_cast<cudaStream_t>(stream)));
}

int mla_merge_rank_partials(const float* rank_o, const float* rank_lse, int n_ranks, int B,
                            int q_len, int H, uint16_t* out_bf16, float* out_lse, void* stream) {
  if (rank_o == nullptr || rank_lse == nullptr || out_bf16 == nullptr) return MLA_ERR_INVALID_ARG;
  if (n_ranks <= 0 || B <= 0 || q_len <= 0 || H <= 0) return MLA_ERR_INVALID_ARG;
  if (n_ranks > 256 || q_len > 4 || q_len * H > 512) return MLA_ERR_UNSUPPORTED;
  const int64_t rows = (int64_t)B * q_len * H;
  if (rows > 0x7FFFFFFF) return MLA_ERR_UNSUPPORTED;
  return status_of(mla::launch_merge_ranks(rank_o, rank_lse, n_ranks, (int)rows, out_bf16, out_lse,
                                           static_cast<cudaStream_t>(stream)));
}

int mla_choose_splits(const int32_t* seq_lens_host, int B, int num_sms, int max_splits,
                      int32_t* out_host) {
  if (seq_lens_host == nullptr || out_host == nullptr || B <= 0 || num_sms <= 0 || max_splits <= 0)
    return MLA_ERR_INVALID_ARG;
  for (int b = 0; b < B; ++b)
    if (seq_lens_host[b] < 1) return MLA_ERR_INVALID_ARG;
  // T = max(2048, ceil(sum_b L_b / max(1, num_sms - B))) tokens per split,
  // and every request gets ceil(L_b / T) splits, at least one, at most
  // max_splits: sum_b ceil(L_b / T) <= sum_b L_b / T + B <= num_sms
  int64_t total = 0;
  for (int b = 0; b < B; ++b) total += seq_lens_host[b];
  const int64_t slots = num_sms - B > 1 ? num_sms - B : 1;
  int64_t T = (total + slots - 1) / slots;
  if (T < kSplitTokens) T = kSplitTokens;
  for (int b = 0; b < B; ++b) {
    int64_t sp = ((int64_t)seq_lens_host[b] + T - 1) / T;
    if (sp < 1) sp = 1;
    if (sp > max_splits) sp = max_splits;
    out_host[b] = (int32_t)sp;
  }
  return MLA_OK;
}

int mla_device_error_status(int32_t dev_error_word) {
  return dev_error_word == 0 ? MLA_OK : MLA_ERR_DEVICE;
}

int mla_append_kv_fp8(const uint16_t* c_kv, const uint16_t* k_rope, const float* cos_sin,
                      int64_t max_pos, const int32_t* block_table, int max_pages_per_req,
                      const int32_t* seq_lens, int B, int n_new, float inv_scale, uint8_t* kv_pages,
                      int64_t num_pages, int32_t* dev_error, void* stream) {
  if (B <= 0 || n_new < 0 || max_pos <= 0 || max_pages_per_req <= 0 || num_pages <= 0)
    return MLA_ERR_INVALID_ARG;
  if (n_new == 0) return MLA_OK;
  if (c_kv == nullptr || k_rope == nullptr || cos_sin == nullptr || block_table == nullptr ||
      seq_lens == nullptr || kv_pages == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (!aligned16(c_kv) || !aligned16(kv_pages) || (reinterpret_cast<uintptr_t>(k_rope) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(cos_sin) & 7u) != 0)
    return MLA_ERR_INVALID_ARG;
  if (!(inv_scale == inv_scale) || !(inv_scale > 0.0f)) return MLA_ERR_INVALID_ARG;
  mla::AppendArgs a = {};
  a.c_kv = c_kv;
  a.k_rope = k_rope;
  a.cos_sin = cos_sin;
  a.block_table = block_table;
  a.seq_lens = seq_lens;
  a.kv_pages = kv_pages;
  a.dev_error = dev_error;
  a.max_pos = max_pos;
  a.num_pages = num_pages;
  a.max_pages = max_pages_per_req;
  a.B = B;
  a.n_new = n_new;
  a.inv_scale = inv_scale;
  return status_of(mla::launch_append_kv_fp8(a, num_sms_current_device(),
                                             static_cast<cudaStream_t>(stream)));
}

int mla_rope_cos_sin_table(float* cos_sin_host, int64_t max_pos, double base) {
  if (cos_sin_host == nullptr || max_pos <= 0 || !(base > 1.0)) return MLA_ERR_INVALID_ARG;
  for (int64_t pos = 0; pos < max_pos; ++pos) {
    for (int i = 0; i < 32; ++i) {
      // theta_i = base^(-2i/64); angle, cosine and sine in double, rounded once
      const double angle = (double)pos * std::pow(base, -(double)(2 * i) / 64.0);
      cos_sin_host[(pos * 32 + i) * 2] = (float)std::cos(angle);
      cos_sin_host[(pos * 32 + i) * 2 + 1] = (float)std::sin(angle);
    }
  }
  return MLA_OK;
}

const char* mla_status_string(int status) {
  switch (status) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
    case MLA_ERR_DEVICE: return "MLA_ERR_DEVICE";
    case MLA_ERR_SCRATCH_LIMIT: return "MLA_ERR_SCRATCH_LIMIT";
    default: return "MLA_ERR_UNKNOWN";
  }
}

int mla_partial_grid(int B, int q_len, int H, int max_splits, int kv_dtype, int num_sms,
                     int32_t* out4) {
  if (out4 == nullptr || B < 1 || q_len < 1 || H < 1 || max_splits < 1 || num_sms < 1)
    return MLA_ERR_INVALID_ARG;
  if (kv_dtype != MLA_KV_FP8_E4M3 && kv_dtype != MLA_KV_BF16) return MLA_ERR_INVALID_ARG;
  plan_grid(B, q_len, H, max_splits, kv_dtype, num_sms, out4);
  if (kv_dtype == MLA_KV_BF16) out4[0] = ((q_len * H + 63) / 64) * max_splits * B;
  return MLA_OK;
}

int mla_debug_inject_stall(int enable) {
  return g_inject_stall.exchange(enable != 0 ? 1 : 0, std::memory_order_relaxed);
}

int mla_debug_merge_plan(int v, int gpi) {
  if (v == 0 && gpi == 0) {
    g_merge_plan.store(0, std::memory_order_relaxed);
    return MLA_OK;
  }
  if ((v != 1 && v != 2 && v != 4) || (gpi != 1 && gpi != 2 && gpi != 3 && gpi != 6))
    return MLA_ERR_INVALID_ARG;
  g_merge_plan.store(16 * v + gpi, std::memory_order_relaxed);
  return MLA_OK;
}

}  // extern "C"
