// Internal launcher declarations shared by the kernel files and the C ABI.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace mla {

cudaError_t launch_quantize_fp8(const uint16_t* x, uint8_t* y, int64_t n, float inv_scale,
                                int num_sms, cudaStream_t stream);

cudaError_t launch_combine(const float* part_o, const float* part_lse, const int32_t* num_splits,
                           int max_splits, int B, int q_len, int H, uint16_t* out, float* out_lse,
                           cudaStream_t stream);
// The same merge with an fp32 output: one partial per row (O [rows][512], LSE).
cudaError_t launch_combine_f32(const float* part_o, const float* part_lse,
                               const int32_t* num_splits, int max_splits, int B, int q_len, int H,
                               float* out, float* out_lse, cudaStream_t stream);
// Merge of per-rank partials laid out [n_ranks][rows][512] and [n_ranks][rows].
cudaError_t launch_merge_ranks(const float* rank_o, const float* rank_lse, int n_ranks, int rows,
                               uint16_t* out, float* out_lse, cudaStream_t stream);

// Arguments of the split-KV partial kernels (device pointers; see mla.h).
struct DecodeArgs {
  const uint16_t* q_nope;
  const uint16_t* q_rope;
  const uint8_t* kv_pages;   // the page pool, [num_pages][64][576] elements
  const int32_t* block_table;
  const int32_t* seq_lens;
  const int32_t* num_splits;
  float* part_o;
  float* part_lse;
  int32_t* dev_error;
  int64_t num_pages;
  int max_pages;
  int max_splits;
  int B;
  int q_len;
  int H;
  float qk_scale_log2;  // softmax_scale * kv_scale * log2(e)
  float kv_scale;
  // FP8 grid, one dimension: units are (query-row group, split, request)
  // triples, unit = g + groups * (s + max_splits * b).  Units below split_from
  // run one CTA each; then come `pad` idle CTAs (cluster alignment); every
  // later unit runs `pieces` CTAs, one cluster, each over a contiguous run of
  // the split's tiles, merged on chip.
  int groups;
  int split_from;
  int pad;
  int pieces;
  int inject_stall;     // test hook: leave the first load of CTA (0, 0, 0) unissued
  // FP8 query (FP8 kernel only): when q8 is set, query row r is the 576 E4M3
  // codes q8[576 r ..] (latent then RoPE dims) of value code * q_scale, and
  // q_nope / q_rope are not read.
  const uint8_t* q8;
  float q_scale;
  // Single-launch mode (FP8, every CTA resident, cooperative launch without
  // clusters): each piece writes its own normalised partial to entry
  // s * pieces + piece of its rows (part_o16 / part_lse then hold
  // max_splits * pieces entries per row; O as fp16 in units of kv_scale,
  // part_o is not used), and after a grid barrier on sync[0] the grid merges
  // them into out / out_lse; sync[1] counts the CTAs that have finished, and
  // the last one resets both to zero.
  int fused;
  uint16_t* part_o16;   // [rows][entries][512] fp16, O / (l kv_scale)
  int splits_const;     // > 0: every request has this many splits (num_splits is not read)
  int merge_v;          // single launch: dims per thread in the merge (1, 2 or 4)
  int merge_gpi;        // single launch: 128-thread groups per merge item (1, 2, 3 or 6)
  uint16_t* out;        // [rows][512] bf16
  float* out_lse;       // [rows], may be null
  int32_t* sync;        // two counters, zero before the launch
};

// FP8 E4M3 cache: kv_map and rope_map are 3-D tiled TMA maps over kv_pages
// viewed as [num_pages][64][576] bytes: kv_map with box {128 B, 64 rows,
// 1 page} and the 128-byte swizzle (the latent dims), rope_map with box
// {64 B, 64 rows, 1 page} and the 64-byte swizzle (the RoPE dims).
cudaError_t launch_decode_fp8(const DecodeArgs& a, const CUtensorMap& kv_map,
                              const CUtensorMap& rope_map, cudaStream_t stream);

// bf16 cache: kv_map over [num_pages][64][576] bf16, box {64 elems, 64 rows,
// 1 page}, 128-byte swizzle.
cudaError_t launch_decode_bf16(const DecodeArgs& a, const CUtensorMap& kv_map,
                               cudaStream_t stream);

// Arguments of the KV-append kernel (device pointers; see mla.h).
struct AppendArgs {
  const uint16_t* c_kv;        // [B][n_new][512] bf16
  const uint16_t* k_rope;      // [B][n_new][64] bf16, before rotation
  const float* cos_sin;        // [max_pos][32][2] fp32
  const int32_t* block_table;  // [B][max_pages]
  const int32_t* seq_lens;     // [B], including the n_new tokens
  uint8_t* kv_pages;           // [num_pages][64][576] E4M3
  int32_t* dev_error;
  int64_t max_pos;
  int64_t num_pages;
  int max_pages;
  int B;
  int n_new;
  float inv_scale;
};

cudaError_t launch_append_kv_fp8(const AppendArgs& a, int num_sms, cudaStream_t stream);

}  // namespace mla
