// Allocation-free decode: partial attention + merge with the split workspace
// held in a fixed, file-scope device array instead of caller memory.
//
// Who needs this: callers that cannot allocate device memory themselves —
// for example a plugin whose host application owns the whole device memory
// pool and gives plugins no allocator, or a latency-critical loop that must
// not call cudaMalloc because cudaMalloc may synchronise the device.  Such a
// caller passes only the inputs and the outputs; the library allocates
// nothing either (no cudaMalloc, no cudaFree, no allocating library call).
//
// The cost: every process that loads the library holds kScratchRowSplits *
// 513 * 4 bytes (about 16 MiB) of device memory on each GPU it uses, until
// the process exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "mla.h"

namespace {

// Capacity in (query row, split) pairs: B * q_len * H * max_splits <= 8192,
// e.g. batch 1 x 64 heads x 128 splits, or batch 2 x 64 heads x 64 splits.
constexpr int64_t kScratchRowSplits = 8192;

// Partial outputs of every call: part_o (512 fp32 per row-split) followed by
// part_lse (1 fp32 per row-split).  Shared by all calls on a device.
static __device__ __align__(256) float g_partials_scratch[kScratchRowSplits * 513];

constexpr int kMaxDevices = 64;

// The cached address is tagged with the CUDA context it was looked up in: a
// context that is destroyed and created again (cudaDeviceReset, a primary
// context released and retained again) reloads the module, and the array may
// then live elsewhere, so a changed context id triggers a new look-up.
struct ScratchEntry {
  float* ptr = nullptr;
  unsigned long long ctx_id = 0;
};
ScratchEntry g_scratch[kMaxDevices];
std::mutex g_scratch_mutex;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique id of the current context (0 if it cannot be had).
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static bool looked_up = false;
  if (!looked_up) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
    looked_up = true;
  }
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS ||
      ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of g_partials_scratch on the current device.  In host code
// the symbol's name is only a host-side stand-in; the address the kernels
// may use is the one cudaGetSymbolAddress returns with the device current.
int scratch_for_current_device(float** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return MLA_ERR_CUDA;
  if (dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  // (before the device's first runtime call there is no current context and
  // the id is 0: the look-up below creates the context and is repeated once
  // on the next call, which then finds the context's id)
  const unsigned long long ctx = current_context_id();
  ScratchEntry& e = g_scratch[dev];
  if (e.ptr == nullptr || ctx == 0 || e.ctx_id != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_partials_scratch) != cudaSuccess || p == nullptr)
      return MLA_ERR_CUDA;
    e.ptr = static_cast<float*>(p);
    e.ctx_id = ctx;
  }
  *out = e.ptr;
  return MLA_OK;
}

}  // namespace

extern "C" {

int mla_decode_noalloc(const uint16_t* q_nope, const uint16_t* q_rope, const void* kv_pages,
                       int kv_dtype, float kv_scale, int64_t num_pages,
                       const int32_t* block_table, int max_pages_per_req,
                       const int32_t* seq_lens, const int32_t* num_splits, int max_splits, int B,
                       int q_len, int H, float softmax_scale, uint16_t* out_bf16, float* out_lse,
                       int32_t* dev_error, void* stream) {
  if (B <= 0 || q_len <= 0 || H <= 0 || max_splits <= 0) return MLA_ERR_INVALID_ARG;
  const int64_t row_splits = (int64_t)B * q_len * H * max_splits;
  if (row_splits > kScratchRowSplits) return MLA_ERR_SCRATCH_LIMIT;
  if (out_bf16 == nullptr) return MLA_ERR_INVALID_ARG;
  float* scratch = nullptr;
  int st = scratch_for_current_device(&scratch);
  if (st != MLA_OK) return st;
  // Every (row, split) entry the merge reads is written by the partial kernel
  // of the same call (empty splits included), so nothing needs clearing
  // between calls.
  float* part_o = scratch;
  float* part_lse = scratch + row_splits * 512;
  st = mla_decode_partial(q_nope, q_rope, kv_pages, kv_dtype, kv_scale, num_pages, block_table,
                          max_pages_per_req, seq_lens, num_splits, max_splits, B, q_len, H,
                          softmax_scale, part_o, part_lse, dev_error, stream);
  if (st != MLA_OK) return st;
  return mla_combine(part_o, part_lse, num_splits, max_splits, B, q_len, H, out_bf16, out_lse,
                     stream);
}

}  // extern "C"
