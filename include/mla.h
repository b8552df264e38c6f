/*
 * mla.h — C ABI of the B200 (sm_100a) absorbed-MLA split-KV decode library.
 *
 * What the library computes (decode over a paged latent KV cache):
 *   One KV row per token: 576 values = a 512-wide compressed latent (which is
 *   also V) followed by a 64-wide decoupled RoPE key, stored as FP8 E4M3 codes
 *   with one per-tensor scale, or as bf16.  For each query row (b, q, h):
 *     s_t = softmax_scale * (q_nope . c_t[0:512] + q_rope . c_t[512:576])
 *     O   = sum_t e^{s_t} c_t[0:512] / sum_t e^{s_t},  LSE = ln sum_t e^{s_t}
 *   over the tokens the row sees.  q_nope is the already-absorbed 512-wide
 *   query; absorption and the output up-projection belong to the caller.
 *
 * Sources: "SGLang & Miles ... Vera Rubin" article (arex-research.com),
 * section "Kimi K3 的 MLA：更深的流水线、更快的 split-KV 归约":
 *   - bullet "更快的 split-KV 归约": at low concurrency one request's KV is cut
 *     across many CTAs, each producing a partial result, and a second kernel
 *     merges the partials; the merge issues all partial loads first and then
 *     accumulates from registers  -> mla_decode_partial + mla_combine;
 *   - bullet "64 路 split-KV": batch-1 decode needs enough splits to occupy the
 *     SMs  -> per-request num_splits, mla_choose_splits;
 *   - bullet "原生 FP8 转换": KV/Q converted to FP8 with a saturating
 *     conversion, overflow clamped to +-448 instead of NaN  -> mla_quantize_fp8.
 *
 * Conventions for every entry point:
 *   - Pointers are DEVICE pointers unless a name ends in _host.  The caller
 *     owns all memory; the library allocates, frees and synchronises nothing.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and is stream-ordered; the return value reports argument and
 *     launch errors only.  Errors found by the GPU (bad page id, a wait that
 *     timed out) are recorded in the caller's dev_error word, read after a
 *     stream synchronisation.
 *   - Arrays are dense, C order, as laid out below.  Device pointers must be
 *     16-byte aligned (mla_quantize_fp8 also accepts unaligned pointers).
 *   - Return 0 (MLA_OK) or one of the MLA_ERR_* codes; nothing is launched when
 *     an argument is rejected.  No exceptions, no logging.  The only global
 *     state is per device and thread-safe: each device's SM count, looked up
 *     on first use, and the kernels' shared-memory opt-in, set on every launch.
 *     Calls may target any device the caller makes current.
 */
#ifndef MLA_B200_H
#define MLA_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MLA_API __attribute__((visibility("default")))
#else
#define MLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misalignment, out of range */
  MLA_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. H*q_len not a multiple of 16) */
  MLA_ERR_CUDA = 3,         /* a CUDA runtime/driver call or launch failed */
  MLA_ERR_DEVICE = 4,       /* the GPU set dev_error (mla_device_error_status) */
  MLA_ERR_SCRATCH_LIMIT = 5 /* mla_decode_noalloc: problem larger than its fixed scratch */
};

enum {
  MLA_KV_FP8_E4M3 = 0,      /* kv_pages holds E4M3 codes, value = code * kv_scale */
  MLA_KV_BF16 = 1           /* kv_pages holds bf16 values, kv_scale must be 1 */
};

/* Bits the GPU ORs into *dev_error (zero it before the launch). */
enum {
  MLA_DEVERR_BAD_PAGE = 1,      /* block_table entry outside [0, num_pages); tile skipped */
  MLA_DEVERR_BAD_SEQLEN = 2,    /* seq_len < q_len or above max_pages*64; request skipped */
  MLA_DEVERR_TIMEOUT = 4,       /* a pipeline wait exceeded its time limit; CTA aborted */
  MLA_DEVERR_BAD_SPLITS = 8,    /* num_splits[b] outside [1, max_splits]; request skipped */
  MLA_DEVERR_SMEM_ALIGN = 16    /* dynamic shared memory base not 1 KiB aligned */
};

/* ---------------------------------------------------------------------------
 * Step A1, prep: saturating FP8 conversion (article bullet "原生 FP8 转换").
 *   y[i] = E4M3_RN_satfinite( fl32( float(x[i]) * inv_scale ) )
 * x: n bf16 values (bit patterns), y: n E4M3 codes.  Exactly one fp32 multiply
 * (round to nearest) then one E4M3 rounding, ties to even; |v| >= 448 and
 * +-inf give +-448 (0x7E/0xFE), never NaN; NaN input gives an E4M3 NaN code.
 * inv_scale is the caller's fp32 reciprocal of the dequantisation scale.
 * n may be 0.  x and y may have any alignment (16-byte aligned is fastest).
 * ------------------------------------------------------------------------- */
MLA_API int mla_quantize_fp8(const uint16_t* x_bf16, uint8_t* y_e4m3, int64_t n,
                     float inv_scale, void* stream);

/* Bytes of the split workspace that holds the per-split partial results
 * (article bullet "更快的 split-KV 归约": each CTA's partial result, merged
 * by the second kernel): part_o (B*q_len*H*max_splits*512 fp32) followed by
 * part_lse (B*q_len*H*max_splits fp32).  Returns 0 for invalid
 * sizes.  A caller may carve both arrays from one allocation of this size
 * (part_lse = part_o + B*q_len*H*max_splits*512). */
MLA_API size_t mla_partial_workspace_bytes(int B, int q_len, int H, int max_splits);

/* ---------------------------------------------------------------------------
 * Steps A2-A8: split-KV partial attention (article bullet "更快的 split-KV 归约").
 *
 * q_nope     [B][q_len][H][512] bf16   absorbed query (latent part)
 * q_rope     [B][q_len][H][64]  bf16   RoPE part of the query
 * kv_pages   [num_pages][64][576]      E4M3 codes (kv_dtype 0) or bf16 (1)
 * block_table[B][max_pages_per_req] int32: token t of request b is row t%64
 *            of page block_table[b][t/64]
 * seq_lens   [B] int32, tokens in the cache including the q_len new ones
 *            (q_len <= seq_len <= max_pages_per_req*64)
 * num_splits [B] int32 in [1, max_splits]
 * Causality: query position q of request b sees tokens 0 .. seq_len-q_len+q.
 * Split s of request b covers pages [s*c, min((s+1)*c, n)) with
 * n = ceil(seq_len/64) and c = ceil(n/num_splits[b]).
 * Outputs, for s < num_splits[b] (entries s >= num_splits[b] are not written):
 *   part_o  [B][q_len][H][max_splits][512] fp32  O_s = sum_t w_t v_t / sum_t w_t
 *   part_lse[B][q_len][H][max_splits]      fp32  LSE_s (natural log of the
 *           scaled-score sum); an empty split gives O_s = 0, LSE_s = -inf.
 * softmax_scale multiplies q.k; kv_scale (FP8 only) multiplies every code.
 * Supported: H*q_len a multiple of 16 and at most 512, q_len in 1..4,
 * max_splits in 1..256.  dev_error may be NULL.
 * ------------------------------------------------------------------------- */
MLA_API int mla_decode_partial(const uint16_t* q_nope, const uint16_t* q_rope,
                       const void* kv_pages, int kv_dtype, float kv_scale,
                       int64_t num_pages, const int32_t* block_table,
                       int max_pages_per_req, const int32_t* seq_lens,
                       const int32_t* num_splits, int max_splits, int B, int q_len,
                       int H, float softmax_scale, float* part_o, float* part_lse,
                       int32_t* dev_error, void* stream);

/* ---------------------------------------------------------------------------
 * Steps A2-A8 with an FP8 query (article bullet "原生 FP8 转换": the prep
 * converts Q to FP8 as well as KV).  An option beside mla_decode_partial, not
 * its replacement: the query itself is then quantised, which the bf16-query
 * entry point avoids (it splits Q into two exact FP8 terms), so results
 * differ from it by the query's rounding.  The MMAs take the same time.
 * q8 [B][q_len][H][576] E4M3 codes (the 512 latent dims, then the 64 RoPE
 * dims; e.g. from mla_quantize_fp8 of the concatenated bf16 query), 16-byte
 * aligned; the value of a code is e4m3(code) * q_scale (q_scale > 0, finite).
 * kv_pages must be FP8 E4M3.  Every other argument, the outputs and the
 * error behaviour are those of mla_decode_partial; merge with mla_combine.
 * ------------------------------------------------------------------------- */
MLA_API int mla_decode_partial_q8(const uint8_t* q8, float q_scale, const void* kv_pages,
                                  float kv_scale, int64_t num_pages,
                                  const int32_t* block_table, int max_pages_per_req,
                                  const int32_t* seq_lens, const int32_t* num_splits,
                                  int max_splits, int B, int q_len, int H, float softmax_scale,
                                  float* part_o, float* part_lse, int32_t* dev_error,
                                  void* stream);

/* ---------------------------------------------------------------------------
 * Step A9: the second kernel, LSE merge of the partials (same bullet): per row
 *   M = max_s LSE_s, w_s = e^{LSE_s - M},
 *   O = sum_s w_s O_s / sum_s w_s (rounded to bf16, nearest-even),
 *   LSE = M + ln sum_s w_s   (fp32),
 * over s < num_splits[b]; all splits empty gives O = 0, LSE = -inf.  Every
 * partial load of a row is issued before the accumulation starts.
 * out_bf16 [B][q_len][H][512], out_lse [B][q_len][H] (out_lse may be NULL).
 * ------------------------------------------------------------------------- */
MLA_API int mla_combine(const float* part_o, const float* part_lse, const int32_t* num_splits,
                int max_splits, int B, int q_len, int H, uint16_t* out_bf16,
                float* out_lse, void* stream);

/* ---------------------------------------------------------------------------
 * Single-launch decode, steps A2-A9 in one kernel ("SGLang & Miles ... Vera
 * Rubin" article, section "Vera Rubin 的三处硬件变化": kernel launches are
 * among the overheads the team removed).  The call picks its own partition:
 * every request is cut into S equal page ranges (step A2 with the same S for
 * all requests), S = min(256, floor(SMs / (G * B))), G = ceil(q_len*H / 64)
 * query-row groups, SMs those of the current device, so that the grid holds
 * one CTA per (row group, split, request) and is a single wave: every CTA is
 * resident at once and none waits for a free SM.  Requires an FP8 cache
 * (kv_dtype 0) and S >= 1 (G * B <= SMs, e.g. batch 16 with 64 heads and
 * one query token per request on 148 SMs gives S = 9); otherwise it returns
 * MLA_ERR_UNSUPPORTED and launches nothing: use mla_decode_partial +
 * mla_combine.  Other arguments and the outputs are those of
 * mla_decode_partial followed by mla_combine.
 * The kernel is a cooperative launch.  Every CTA writes the partial of its
 * split (O/l, as fp16 in units of kv_scale, and the fp32 LSE) to the workspace, the CTAs meet at a grid barrier (a
 * counter in the workspace, bounded wait), and the grid then merges each
 * row's S partials as mla_combine does, in a fixed order (deterministic); the
 * result equals partial + combine with S splits up to rounding.
 *   mla_fused_splits: the S that a call with these sizes uses on a GPU with
 *     num_sms SMs (0: no single launch for these sizes).
 *   workspace: mla_fused_workspace_bytes(B, q_len, H, num_sms) bytes with the
 *     current device's SM count (256 + B*q_len*H*S*(512*2 + 4): per (row,
 *     split) the partial O as fp16 in units of kv_scale and its fp32 LSE; 0
 *     when S = 0),
 *     passed with its size; 16-byte aligned; its first 8 bytes (two int32
 *     counters) must be zero before the first call; every call that
 *     completes leaves them zero.  After MLA_DEVERR_TIMEOUT, zero them again
 *     before the next call.  Calls that share a workspace must not overlap on
 *     the GPU.  A workspace smaller than the call needs: MLA_ERR_INVALID_ARG.
 *   out_bf16 [B][q_len][H][512], out_lse [B][q_len][H] (nullable).
 * ------------------------------------------------------------------------- */
MLA_API int mla_fused_splits(int B, int q_len, int H, int num_sms);
MLA_API size_t mla_fused_workspace_bytes(int B, int q_len, int H, int num_sms);
MLA_API int mla_decode_fused(const uint16_t* q_nope, const uint16_t* q_rope,
                             const void* kv_pages, int kv_dtype, float kv_scale,
                             int64_t num_pages, const int32_t* block_table,
                             int max_pages_per_req, const int32_t* seq_lens, int B, int q_len,
                             int H, float softmax_scale, void* workspace, size_t workspace_bytes,
                             uint16_t* out_bf16, float* out_lse, int32_t* dev_error,
                             void* stream);

/* ---------------------------------------------------------------------------
 * Sequence-sharded decode over several GPUs (the merge of "更快的 split-KV 归约"
 * one level up): each rank holds a disjoint page range of every request, runs
 * mla_decode_partial over it, folds its own splits into one partial per row
 * with mla_combine_f32, the ranks exchange those (an all-gather of
 * rows*513 fp32 per rank), and mla_merge_rank_partials merges them.
 *
 * mla_combine_f32: the merge of mla_combine with an fp32 output and the
 * merged LSE: out_o [B][q_len][H][512] fp32, out_lse [B][q_len][H] fp32 (both
 * required).  A row whose splits are all empty gives O = 0, LSE = -inf.
 * ------------------------------------------------------------------------- */
MLA_API int mla_combine_f32(const float* part_o, const float* part_lse,
                            const int32_t* num_splits, int max_splits, int B, int q_len, int H,
                            float* out_o, float* out_lse, void* stream);

/* mla_merge_rank_partials: rank_o [n_ranks][B][q_len][H][512] fp32 and
 * rank_lse [n_ranks][B][q_len][H] fp32 (each rank's mla_combine_f32 output,
 * stacked in rank order, as an all-gather lays them out) -> out_bf16
 * [B][q_len][H][512] (nearest-even) and out_lse (nullable), by the same LSE
 * merge over the ranks.  n_ranks in 1..256. */
MLA_API int mla_merge_rank_partials(const float* rank_o, const float* rank_lse, int n_ranks,
                                    int B, int q_len, int H, uint16_t* out_bf16, float* out_lse,
                                    void* stream);

/* ---------------------------------------------------------------------------
 * Allocation-free decode (steps A2-A9 in one call).  The pages have no
 * counterpart to this entry point; it exists for callers that cannot allocate
 * device memory (a plugin whose host owns the whole device memory pool and
 * offers no allocator, a latency-critical loop that must not call cudaMalloc
 * because it may synchronise the device).  Arguments and outputs are those of
 * mla_decode_partial followed by mla_combine, minus the workspace: the split
 * partials live in a file-scope device array inside the library, and the
 * library allocates nothing (no cudaMalloc, no cudaFree).
 *   - Limit: B*q_len*H*max_splits <= 8192 (row, split) pairs, e.g. batch 1 x
 *     64 heads x 128 splits; larger problems return MLA_ERR_SCRATCH_LIMIT and
 *     launch nothing.  Every GPU on which the library is loaded holds that
 *     array (8192*513 fp32, about 16 MiB) until the process exits.
 *   - The first call on each device looks up the array's device address with
 *     that device current (cudaGetSymbolAddress); make that first call before
 *     any stream capture.  Later calls reuse the address while the device's
 *     CUDA context stays the same; after cudaDeviceReset (a new context) the
 *     next call looks it up again, so make that call outside a capture too.
 *   - All calls on a device share the array and it keeps the last call's
 *     contents.  Each call writes every entry it reads, so nothing needs to
 *     start at zero, but calls that overlap on the GPU (different streams,
 *     host threads) race on it: order them on one stream.
 *   - If dev_error reports an error the outputs are undefined.
 * ------------------------------------------------------------------------- */
MLA_API int mla_decode_noalloc(const uint16_t* q_nope, const uint16_t* q_rope,
                               const void* kv_pages, int kv_dtype, float kv_scale,
                               int64_t num_pages, const int32_t* block_table,
                               int max_pages_per_req, const int32_t* seq_lens,
                               const int32_t* num_splits, int max_splits, int B, int q_len,
                               int H, float softmax_scale, uint16_t* out_bf16, float* out_lse,
                               int32_t* dev_error, void* stream);

/* ---------------------------------------------------------------------------
 * KV append, the step before the decode path ("Muse Spark Open" article,
 * section "内核优化：解码吞吐 3 倍", bullet "RoPE 与 KV 缓存写入融合": RoPE is
 * applied in the kernel that writes the decode KV cache; "SGLang & Miles ...
 * Vera Rubin" article, bullet "原生 FP8 转换": saturating E4M3 storage).
 *
 * c_kv       [B][n_new][512] bf16   new tokens' compressed latent
 * k_rope     [B][n_new][64]  bf16   new tokens' RoPE key, before rotation
 * cos_sin    [max_pos][32][2] fp32  (cos, sin) of pos * theta_i, theta_i =
 *            base^(-2i/64) (see mla_rope_cos_sin_table)
 * block_table[B][max_pages_per_req], seq_lens [B] (lengths including the
 *            n_new tokens, as for mla_decode_partial)
 * kv_pages   [num_pages][64][576] E4M3 codes, written in place
 * Token j of request b has position pos = seq_lens[b] - n_new + j and is
 * written to row pos % 64 of page block_table[b][pos / 64]:
 *   latent d:   E4M3_satfinite(fl32(x_d * inv_scale))
 *   RoPE pair i (dims 2i, 2i+1), (c, s) = cos_sin[pos][i], fp32 with every
 *   operation rounded to nearest and no fused multiply-add:
 *     y0 = x0*c - x1*s,  y1 = x0*s + x1*c;  codes E4M3_satfinite(fl32(y*inv_scale)).
 * A token whose position is outside [0, max_pos) or beyond the block table
 * sets MLA_DEVERR_BAD_SEQLEN, one whose page id is outside [0, num_pages) sets
 * MLA_DEVERR_BAD_PAGE; such tokens are not written, the others are.
 * c_kv and kv_pages must be 16-byte aligned, k_rope 4-byte, cos_sin 8-byte.
 * n_new may be 0.  dev_error may be NULL.
 * ------------------------------------------------------------------------- */
MLA_API int mla_append_kv_fp8(const uint16_t* c_kv, const uint16_t* k_rope, const float* cos_sin,
                              int64_t max_pos, const int32_t* block_table,
                              int max_pages_per_req, const int32_t* seq_lens, int B, int n_new,
                              float inv_scale, uint8_t* kv_pages, int64_t num_pages,
                              int32_t* dev_error, void* stream);

/* Host helper for mla_append_kv_fp8: fills the HOST array cos_sin_host
 * [max_pos][32][2] with (cos, sin) of pos * base^(-2i/64), each computed in
 * double and rounded once to fp32 (the original rotary embedding; base is
 * 10000 in the paper that introduced it).  base must be > 1. */
MLA_API int mla_rope_cos_sin_table(float* cos_sin_host, int64_t max_pos, double base);

/* Host helper (article bullet "64 路 split-KV": batch-1 decode needs enough
 * splits to occupy the SMs; the pages fix no rule, so this is a reading):
 * a batch's tokens are cut into at most about num_sms splits of equal length,
 *   T = max(2048, ceil(sum_b seq_lens_host[b] / max(1, num_sms - B))) tokens,
 *   out_host[b] = min(max_splits, max(1, ceil(seq_lens_host[b] / T))),
 * so that no split is longer than T and, for B < num_sms, the batch has at
 * most num_sms splits.  A single 128K-token request gets 64 splits (T =
 * 2048); 16 such requests on 148 SMs get 9 each (one wave).  When the grid
 * still underfills the GPU, mla_decode_partial cuts each split across a CTA
 * cluster on its own (see mla_partial_grid).  seq_lens_host and out_host are
 * HOST arrays of B int32; every seq_len must be >= 1.  Returns
 * MLA_ERR_INVALID_ARG for null pointers, sizes <= 0 or num_sms <= 0. */
MLA_API int mla_choose_splits(const int32_t* seq_lens_host, int B, int num_sms, int max_splits,
                              int32_t* out_host);

/* Fold a device error word (read back from dev_error after the stream has
 * synchronised) into a status: MLA_OK for 0, MLA_ERR_DEVICE otherwise (the
 * MLA_DEVERR_* bits say what the GPU found). */
MLA_API int mla_device_error_status(int32_t dev_error_word);

/* Host helper, no GPU needed: how mla_decode_partial lays out its CTAs for
 * a problem shape on num_sms SMs.  Units are (64-row query group, split,
 * request) triples.  FP8: when the units fill at most half of the SMs, every
 * split is cut into 2 or 4 contiguous runs of tiles, one CTA each, launched as
 * a cluster that merges on chip; when they fill several waves and the last
 * wave is at most half full, only that wave's units are cut in two.  bf16: one
 * CTA per unit.  The partials are the same either way (rounding aside).
 * out4 (HOST, 4 int32) = {CTAs launched, pieces per cut unit, index of the
 * first cut unit, idle CTAs placed before the cut units so that clusters
 * align}.  Returns MLA_ERR_INVALID_ARG for non-positive sizes or an unknown
 * kv_dtype. */
MLA_API int mla_partial_grid(int B, int q_len, int H, int max_splits, int kv_dtype, int num_sms,
                             int32_t* out4);

/* ---------------------------------------------------------------------------
 * mla_debug_inject_stall: a test hook for the failure path; the pages have no
 * counterpart.  While enabled (enable != 0), every FP8 mla_decode_partial
 * launch leaves the first KV load of its first CTA (first tile, first latent
 * pair) unissued, so the waits on that load run out: after the 2 s bound the
 * kernel sets MLA_DEVERR_TIMEOUT in dev_error, all of its warps leave their
 * loops, it frees its tensor memory and returns.  Nothing traps or faults and
 * the CUDA context stays usable; the outputs of such a launch are undefined.
 * Returns the previous setting.  Process-wide; not for production use.
 * ------------------------------------------------------------------------- */
MLA_API int mla_debug_inject_stall(int enable);

/* mla_debug_merge_plan: a test hook with no counterpart on the pages.  The
 * merge inside mla_decode_fused runs each row's entries as items of 128*v
 * dims (v = 1, 2 or 4 dims per thread), gpi = 1, 2, 3 or 6 128-thread groups
 * per item, and picks (v, gpi) per launch from the shape.  While set, every
 * later mla_decode_fused call uses the given plan instead, so that tests can
 * run each one; (0, 0) restores the automatic choice.  Every plan gives the
 * same result up to the order of the sums.  Returns MLA_ERR_INVALID_ARG for
 * other values.  Process-wide; not for production use. */
MLA_API int mla_debug_merge_plan(int v, int gpi);

/* Static, human-readable name of a status code. */
MLA_API const char* mla_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* MLA_B200_H */
