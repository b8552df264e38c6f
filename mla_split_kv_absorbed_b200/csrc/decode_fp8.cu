// Steps A2-A8 for an FP8 E4M3 latent cache: split-KV partial attention on
// sm_100a tensor cores (tcgen05), fed by TMA.
//
// "SGLang & Miles ... Vera Rubin" article, section "Kimi K3 的 MLA":
//  - bullet "更深的 MLA 流水线": long-context MLA decode waits on HBM KV
//    reads; the fix is more reads in flight, i.e. a deep K/V shared-memory
//    stage ring, with output bit-identical across pipeline depths;
//  - bullet "更快的 split-KV 归约": one request's KV is cut across many CTAs,
//    each writing a partial result (normalised O and its log-sum-exp) that a
//    second kernel merges.
//
// Work unit = (query-row group g of up to 64 rows, split s, request b); the
// rows of a group are (q, h) pairs in [q_len][H] order.  The grid is one-
// dimensional: one CTA per unit, except that units can be cut into 2 or 4
// contiguous runs of the split's tiles, one CTA each, launched as a cluster
// that merges its results on chip (merge_pieces) - all units when they fill at
// most half of the GPU, or only those of a partly filled last wave.
//
// Exact two-term FP8 operands: the cache is E4M3, and kind::f8f6f4 needs both
// operands E4M3.  Q (bf16, 8 significant bits) is scaled per row by a power
// of two and split as Q = Q_hi + Q_lo with Q_hi = Q rounded to 4 significant
// bits and Q_lo = E4M3(Q - Q_hi); this is exact for every element within a
// factor 2^-9 of the row maximum.  The softmax weights are scaled by 2^3.5,
// p' = 2^(s - m + 3.5), and split the same way, P = P_hi + P_lo: about 8
// significant bits (like bf16) for every p' >= 2^-1 and an absolute error of
// at most 2^-10 for smaller weights, while the largest weight of a row is at
// least 2^3.5.  The scale cancels in O / l and is removed from the LSE.
//
// Tensor-core mapping.  QK^T takes the 128 two-term query rows as M and the
// 128 tokens of a tile as N:
//   S'[m][t] = Q'[m][:] . K[t][:]      A = Q' (tensor memory for the 512
//                                      latent dims, shared memory for the 64
//                                      RoPE dims), B = K tile (K-major)
// Row m = 32 qd + l of Q' (qd = TMEM lane quadrant, l = lane) is query row
// n = 16 qd + (l & 15), term hi for l < 16 and lo for l >= 16, so the two
// terms of a score sit in lanes l and l ^ 16 of one warp and are added with
// one shuffle.  Keeping the 512 latent dims of Q' in tensor memory frees 64
// KiB of shared memory for the KV ring.  PV keeps the tokens as K and the
// latent dims as M (a 64 x 512 fp32 O with rows as M would not fit in tensor
// memory beside S'):
//   O^T[d][n] += V^T[d][t] . P[t][n]   A = V tile (MN-major), B = P (K-major)
// for d in four 128-wide blocks; the hi and lo MMAs of one block and K step
// share A through the MMA's A-operand collector, so V is read from shared
// memory once.  V is the first 512 columns of the same resident tile that fed
// K, so every KV byte crosses HBM once.
//
// Online softmax (log2 domain, scores pre-multiplied by log2 e), with a lazy
// running max: the max m used for a row only moves when a tile's max exceeds
// it by more than 5.25 (log2 units), so p' stays <= 2^8.75 < 448, the E4M3
// maximum.  A tile in which no score of a quadrant's rows exceeds its max by
// that much (the common case once the max has settled) skips the max
// reduction altogether: one barrier vote decides it.  O^T columns and row
// sums are rescaled (by 2^(m_old - m_new)) only for rows whose max moved.
//
// Warp roles (768 threads):
//   warp 0        TMA producer: pages -> 128-byte-swizzled 128-dim pairs
//                 (one 8 KiB box per page and pair) in an 11-slot ring (2.75
//                 tiles) plus one RoPE slot (64-byte swizzle), each tile's
//                 pages bulk-prefetched into L2 just before its loads, its
//                 RoPE chunk loaded before its latent pairs
//   warp 1        UMMA issuer (warp-uniform polling of readiness; the QK
//                 MMAs whose operands have landed go before a ready PV, which
//                 measured faster than the reverse; one elected lane issues)
//                 and TMEM owner
//   warps 4-19    softmax: warp w works on TMEM lane quadrant w % 4 (16 query
//                 rows) and token slice (w - 4) / 4 (32 tokens of the tile)
//   warps 20-23   O^T rescaling between tiles (thread = latent dim)
//   warps 4-23    epilogue: O^T / l from TMEM to the partial output
//   warps 4-19    also convert Q to the split FP8 operand at the start
// TMEM (512 columns): O^T blocks at 64 j (0-255), Q' latent at 256-383, S' at
// 384-511.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kernels.cuh"
#include "mla.h"
#include "ptx.cuh"

namespace mla {
namespace fp8k {

constexpr int kThreads = 768;
constexpr int kSoftWarps = 16;
constexpr int kSoftThreads = 32 * kSoftWarps;
constexpr int kRows = 64;           // query rows per CTA (UMMA N for PV)
constexpr int kTile = 128;          // tokens per tile (UMMA N for QK, K for PV)
constexpr int kChunk = 128 * 64;    // 128 tokens x 64 dims of E4M3 = 8 KiB
constexpr int kPair = 2 * kChunk;   // 128 latent dims of a tile
constexpr int kRingPairs = 11;      // latent pair slots: 2.75 tiles in flight
constexpr int kRopeSlots = 1;      // freed by its tile's QK, refilled first for the next tile
constexpr int kPBufs = 2;          // P buffers (1 or 2): with 2 the softmax of tile i+1 need not wait for PV(i)
static_assert(kPBufs == 1 || kPBufs == 2, "the alpha and PV-done handshakes assume at most 2");
constexpr float kPShift = 3.5f;     // log2 of the factor carried by the softmax weights
constexpr float kLazy = 5.25f;      // the used max moves only when exceeded by more than this
static_assert(kLazy + kPShift <= 8.8f, "p' must stay below 448, the E4M3 maximum");

constexpr int kOffRing = 0;                                  // 11 pairs
constexpr int kOffRope = kOffRing + kRingPairs * kPair;      // 180224: 2 RoPE chunks
constexpr int kOffQr = kOffRope + kRopeSlots * kChunk;       // 196608: Q' RoPE dims [128][64 B]
constexpr int kOffP = kOffQr + kChunk;                       // buffer b: P_hi [64 rows][128 B] at
                                                             // kOffP + 16 KiB b, P_lo 8 KiB after it
constexpr int kOffScratch = kOffP + kPBufs * 2 * kChunk;
constexpr int kSmemBytes = 232448;                           // 227 KiB

constexpr uint32_t kTmemO = 0;      // O^T block j at 64 j
constexpr uint32_t kTmemQ = 256;    // Q' latent dims: K step k at 256 + 8 k
constexpr uint32_t kTmemS = 384;    // S' [128 rows][128 tokens]

// barrier indices
constexpr int kBarFull = 0;                           // kRingPairs
constexpr int kBarEmpty = kBarFull + kRingPairs;      // kRingPairs
constexpr int kBarRopeFull = kBarEmpty + kRingPairs;  // kRopeSlots
constexpr int kBarRopeEmpty = kBarRopeFull + kRopeSlots;
constexpr int kBarSFull = kBarRopeEmpty + kRopeSlots;
constexpr int kBarSEmpty = kBarSFull + 1;      // one arrival per softmax warp
constexpr int kBarPFull = kBarSEmpty + 1;      // kPBufs, one arrival per softmax warp
constexpr int kBarPEmpty = kBarPFull + kPBufs;  // kPBufs
constexpr int kBarOReady = kBarPEmpty + kPBufs;  // 2: per tile parity
constexpr int kBarPvDone = kBarOReady + 2;
constexpr int kBarQReady = kBarPvDone + 1;
constexpr int kBarAlphaFull = kBarQReady + 1;  // 2: per tile parity, one arrival per lane quadrant
constexpr int kBarDrain = kBarAlphaFull + 2;
constexpr int kBarPvAll = kBarDrain + 1;
constexpr int kNumBars = kBarPvAll + 1;

struct Scratch {
  uint64_t bars[40];
  uint32_t tmem_base;
  int abort;
  int merge_fail;            // single-launch mode: the grid barrier timed out
  int pad;
  float red[4][64];          // per token slice, per query row: amax, tile max, row sums
  float m_run[64];           // max used per query row (log2 units), for the epilogue/merge
  float inv_l[64];           // per query row: kv_scale / l (0 when l == 0), or raw l when cut
  float alpha[2][64];        // per tile parity: rescale factor per query row
  uint32_t changed[2][4];    // per tile parity, per lane quadrant: rows whose max moved
};
static_assert(kOffScratch + sizeof(Scratch) <= kSmemBytes, "shared memory overflow");
static_assert(kNumBars <= 40, "barrier array");

// 64-byte swizzle of a 64-byte-row layout: 16-byte unit u of row r lives at
// unit u ^ ((r >> 1) & 3).  Matches the TMA 64B swizzle and the UMMA SW64
// canonical layout when the atom base is 512-byte aligned.
__device__ __forceinline__ uint32_t sw64(uint32_t row, uint32_t byte_in_row) {
  return row * 64u + ((((byte_in_row >> 4) ^ ((row >> 1) & 3u)) << 4) | (byte_in_row & 15u));
}
// 128-byte swizzle of a 128-byte-row layout: unit u of row r at u ^ (r & 7)
// (UMMA SW128 canonical layout for a 1024-byte-aligned atom base).
__device__ __forceinline__ uint32_t sw128(uint32_t row, uint32_t byte_in_row) {
  return row * 128u + ((((byte_in_row >> 4) ^ (row & 7u)) << 4) | (byte_in_row & 15u));
}

__device__ __forceinline__ void set_error(int32_t* err, int bit) {
  if (err != nullptr) atomicOr(err, bit);
}

// Descriptor for a start address `bytes` past the one `base` encodes (the
// start field holds address >> 4 in its low 14 bits; addresses stay below
// 256 KiB, so the add never carries out of the field).
__device__ __forceinline__ uint64_t desc_at(uint64_t base, uint32_t bytes) {
  return base + (uint64_t)(bytes >> 4);
}

// x rounded to 4 significant bits (round half away from zero on the bit
// pattern): an exact E4M3 value for |x| in the normal range.
__device__ __forceinline__ float hi4(float x) {
  return __uint_as_float((__float_as_uint(x) + 0x80000u) & 0xFFF00000u);
}

// Split 16 fp32 values into two E4M3 terms each: hi = hi4(x), lo = E4M3(x -
// hi).  Result bytes are in element order (16 bytes per term).
__device__ __forceinline__ void split16(const float* x, uint4& hi, uint4& lo) {
  uint32_t h[8], l[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float a = x[2 * k], b = x[2 * k + 1];
    const float ha = hi4(a), hb = hi4(b);
    h[k] = cvt_e4m3x2(ha, hb);
    l[k] = cvt_e4m3x2(a - ha, b - hb);
  }
  hi = make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16), h[6] | (h[7] << 16));
  lo = make_uint4(l[0] | (l[1] << 16), l[2] | (l[3] << 16), l[4] | (l[5] << 16), l[6] | (l[7] << 16));
}

// One term (hi or lo) of 8 fp32 values as E4M3 codes, element order.
__device__ __forceinline__ uint2 term8(const float* x, bool lo) {
  uint32_t c[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float a = x[2 * k], b = x[2 * k + 1];
    const float ha = hi4(a), hb = hi4(b);
    c[k] = lo ? cvt_e4m3x2(a - ha, b - hb) : cvt_e4m3x2(ha, hb);
  }
  return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

// Merge of the P CTAs (one cluster) that share a split, each having staged
// its unnormalised O ([64][512] fp32 at kOffRing), its used max m (sc.m_run)
// and row sum l (sc.inv_l) in its own shared memory.  With M = max m_k over
// the pieces that saw a token and l = sum_k l_k 2^(m_k - M), the split's
// partial is O = sum_k O_k 2^(m_k - M) kv_scale / l and
// LSE = (M - 7 + log2 l) ln 2, the values one CTA over the whole split
// produces.  Rank r of the cluster writes rows [r 64/P, (r+1) 64/P).  Every
// thread of every CTA of the cluster calls this; all distributed shared
// memory loads of a thread are issued before the first is used.
template <int P>
__device__ __forceinline__ void merge_pieces(const DecodeArgs& args, uint8_t* smem, Scratch& sc,
                                             int64_t row_base, int rows_valid, int s) {
  constexpr int kRowsPer = kRows / P;
  constexpr int kIters = (kRowsPer * 128 + kThreads - 1) / kThreads;  // float4 per thread
  const int tid = threadIdx.x;
  const uint32_t rank = cluster_ctarank();
  cluster_sync_all();  // every piece's O, m and l are staged
  const int n0 = (int)rank * kRowsPer;
  float* wgt = reinterpret_cast<float*>(smem + kOffP);  // [P][64] piece weights (P buffers are free)
  if (tid < kRowsPer) {
    const int n = n0 + tid;
    float mk[P], lk[P];
#pragma unroll
    for (int k = 0; k < P; ++k) {
      mk[k] = ld_cluster_f32(mapa_shared(smem_u32(&sc.m_run[n]), k));
      lk[k] = ld_cluster_f32(mapa_shared(smem_u32(&sc.inv_l[n]), k));
    }
    float M = -INFINITY;
#pragma unroll
    for (int k = 0; k < P; ++k)
      if (lk[k] > 0.0f) M = fmaxf(M, mk[k]);
    float l = 0.0f;
#pragma unroll
    for (int k = 0; k < P; ++k)
      if (lk[k] > 0.0f) l += lk[k] * exp2f(mk[k] - M);
#pragma unroll
    for (int k = 0; k < P; ++k)
      wgt[k * kRows + n] = (lk[k] > 0.0f && l > 0.0f) ? exp2f(mk[k] - M) * args.kv_scale / l : 0.0f;
    if (n < rows_valid)
      args.part_lse[(row_base + n) * args.max_splits + s] =
          l > 0.0f ? (M - kPShift + log2f(l)) * 0.69314718055994530942f : -INFINITY;
  }
  __syncthreads();
  const uint32_t staged = smem_u32(smem + kOffRing);
  float4 o[kIters][P];
  float w[kIters][P];
#pragma unroll
  for (int it = 0; it < kIters; ++it) {
    const int idx = tid + it * kThreads;
    const int n = n0 + (idx >> 7);
    const int q4 = idx & 127;  // dims 4*q4 .. 4*q4+3
    const bool live = idx < kRowsPer * 128 && n < rows_valid;
#pragma unroll
    for (int k = 0; k < P; ++k) {
      w[it][k] = live ? wgt[k * kRows + n] : 0.0f;
      // an empty piece (weight 0) staged nothing: skip its load
      o[it][k] = w[it][k] != 0.0f
                     ? ld_cluster_f32x4(mapa_shared(staged + (uint32_t)(n * 512 + 4 * q4) * 4u, k))
                     : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    }
  }
#pragma unroll
  for (int it = 0; it < kIters; ++it) {
    const int idx = tid + it * kThreads;
    const int n = n0 + (idx >> 7);
    const int q4 = idx & 127;
    if (idx < kRowsPer * 128 && n < rows_valid) {
      float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
      for (int k = 0; k < P; ++k) {
        acc.x = fmaf(w[it][k], o[it][k].x, acc.x);
        acc.y = fmaf(w[it][k], o[it][k].y, acc.y);
        acc.z = fmaf(w[it][k], o[it][k].z, acc.z);
        acc.w = fmaf(w[it][k], o[it][k].w, acc.w);
      }
      *reinterpret_cast<float4*>(args.part_o + ((row_base + n) * args.max_splits + s) * 512 +
                                 4 * q4) = acc;
    }
  }
  cluster_sync_all();  // no CTA leaves while a peer still reads its shared memory
}

__device__ __forceinline__ void merge_pieces(int npieces, const DecodeArgs& args, uint8_t* smem,
                                             Scratch& sc, int64_t row_base, int rows_valid, int s) {
  if (npieces == 2)
    merge_pieces<2>(args, smem, sc, row_base, rows_valid, s);
  else
    merge_pieces<4>(args, smem, sc, row_base, rows_valid, s);
}

// Steps A2-A8 for one CTA: its piece of one unit.  Every early return is
// uniform across the CTA.
template <bool kBlock0First>
__device__ __forceinline__ void partial_body(const DecodeArgs& args, const CUtensorMap* kv_map,
                                             const CUtensorMap* rope_map, uint8_t* smem) {
  Scratch& sc = *reinterpret_cast<Scratch*>(smem + kOffScratch);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  const int QH = args.q_len * args.H;
  // the merge kernel that follows may be scheduled now; it waits for this
  // grid's completion before it reads any partial
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // unit (query-row group g, split s, request b) and this CTA's piece of it
  int unit, piece = 0, npieces = 1;
  if ((int)blockIdx.x < args.split_from) {
    unit = blockIdx.x;
  } else if ((int)blockIdx.x < args.split_from + args.pad) {
    return;  // idle: only aligns the clusters of the split units
  } else {
    const int j = (int)blockIdx.x - args.split_from - args.pad;
    unit = args.split_from + j / args.pieces;
    piece = j % args.pieces;  // this CTA's run of the split's tiles
    npieces = args.pieces;
  }
  // Where this CTA's partial goes: split s of its rows, or, in the
  // single-launch mode, entry s * pieces + piece of its rows (every piece
  // writes its own normalised partial, merged with the rest after the grid
  // barrier; no cluster merge).
  const bool own = npieces == 1 || args.fused;
  const int g = unit % args.groups;
  const int s = (unit / args.groups) % args.max_splits;
  const int b = unit / (args.groups * args.max_splits);
  // ---------------------------------------------------------------- split range (step A2)
  const int L = args.seq_lens[b];
  const int S_b = args.splits_const > 0 ? args.splits_const : args.num_splits[b];
  if (S_b < 1 || S_b > args.max_splits) {
    if (tid == 0 && s == 0 && g == 0 && piece == 0) set_error(args.dev_error, MLA_DEVERR_BAD_SPLITS);
    return;
  }
  if (s >= S_b) return;
  if (L < args.q_len || (int64_t)L > (int64_t)args.max_pages * 64) {
    if (tid == 0 && s == 0 && g == 0 && piece == 0) set_error(args.dev_error, MLA_DEVERR_BAD_SEQLEN);
    return;
  }
  const int n_pages = (L + 63) / 64;
  const int cpages = (n_pages + S_b - 1) / S_b;
  const int p0 = min(s * cpages, n_pages);
  const int p1 = min(p0 + cpages, n_pages);
  const int r0 = g * kRows;
  const int rows_valid = min(kRows, QH - r0);
  const int q_max = (r0 + rows_valid - 1) / args.H;
  const int vis_base = L - args.q_len + 1;  // visible length of q = 0
  const int t0s = p0 * 64;                         // the split's tokens [t0s, t1s)
  const int t1s = min(p1 * 64, vis_base + q_max);
  const int64_t row_base = (int64_t)b * QH + r0;
  const int slots = args.fused ? args.max_splits * args.pieces : args.max_splits;  // per row
  const int slot = args.fused ? s * npieces + piece : s;
  // an empty partial: O = 0, LSE = -inf
  auto write_empty = [&]() {
    for (int i = tid; i < rows_valid * 512; i += kThreads) {
      const int n = i >> 9;
      const int64_t at = ((row_base + n) * slots + slot) * 512 + (i & 511);
      if (args.fused)
        args.part_o16[at] = 0;
      else
        args.part_o[at] = 0.0f;
    }
    if (tid < rows_valid) args.part_lse[(row_base + tid) * slots + slot] = -INFINITY;
  };

  if (t1s <= t0s) {  // empty split for every row of the group
    if (piece == 0 || args.fused) write_empty();
    return;
  }
  // this CTA's run: tiles [tile0, tile0 + T) of the split's Ts tiles
  const int Ts = (t1s - t0s + kTile - 1) / kTile;
  const int per = (Ts + npieces - 1) / npieces;
  const int tile0 = min(piece * per, Ts);
  const int T = min(per, Ts - tile0);  // 0 only for a trailing piece of a short split
  const int pg0 = p0 + 2 * tile0;      // block-table index of the run's first page
  const int t0 = t0s + tile0 * kTile;
  const int t1 = min(t1s, t0 + T * kTile);

  // ---------------------------------------------------------------- setup
  if ((smem_u32(smem) & 1023u) != 0) {  // same for every CTA of the grid
    if (tid == 0) set_error(args.dev_error, MLA_DEVERR_SMEM_ALIGN);
    return;
  }
  if (T == 0 && args.fused) {  // no tiles in this piece: an empty entry
    write_empty();
    return;
  }
  if (T == 0) {
    // no tiles in this piece: it joins the cluster merge with an empty result
    if (tid < 64) {
      sc.m_run[tid] = -INFINITY;
      sc.inv_l[tid] = 0.0f;
    }
    __syncthreads();
    merge_pieces(npieces, args, smem, sc, row_base, rows_valid, s);
    return;
  }
  if (tid == 0) {
    for (int i = 0; i < kRingPairs; ++i) {
      mbar_init(&sc.bars[kBarFull + i], 1);
      mbar_init(&sc.bars[kBarEmpty + i], 1);
    }
    for (int i = 0; i < kRopeSlots; ++i) {
      mbar_init(&sc.bars[kBarRopeFull + i], 1);
      mbar_init(&sc.bars[kBarRopeEmpty + i], 1);
    }
    mbar_init(&sc.bars[kBarSFull], 1);
    mbar_init(&sc.bars[kBarSEmpty], kSoftWarps);
    for (int i = 0; i < kPBufs; ++i) {
      mbar_init(&sc.bars[kBarPFull + i], kSoftWarps);
      mbar_init(&sc.bars[kBarPEmpty + i], 1);
    }
    mbar_init(&sc.bars[kBarPvAll], 1);
    for (int i = 0; i < 2; ++i) mbar_init(&sc.bars[kBarOReady + i], 4);
    mbar_init(&sc.bars[kBarPvDone], 1);
    mbar_init(&sc.bars[kBarQReady], kSoftWarps);
    for (int i = 0; i < 2; ++i) mbar_init(&sc.bars[kBarAlphaFull + i], 4);
    mbar_init(&sc.bars[kBarDrain], 1);
    sc.abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sc.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sc.tmem_base;
  volatile int* abort_flag = &sc.abort;
  uint64_t* bars = sc.bars;

  if (warp == 0) {
    // ============================================================ TMA producer
    // The whole warp runs this loop with warp-uniform values; one elected
    // lane issues each TMA instruction and barrier arrival.  Latent pair j of
    // tile i is load number u = 4 i + j and goes to ring slot u % 11; the
    // RoPE chunk of tile i goes to slot i % 2 of its own ring.
    if (lane == 0) {
      prefetch_tensormap(kv_map);
      prefetch_tensormap(rope_map);
    }
    __syncwarp();
    const int32_t* bt = args.block_table + (int64_t)b * args.max_pages;
    // Page ids of this run, 32 at a time (one load per lane instead of a
    // dependent load per tile): lane l of window w holds block-table entry
    // pg0 + 32 w + l (-1 past the row); the next window is loaded ahead.
    auto load_window = [&](int w) -> int {
      const int k = pg0 + 32 * w + lane;
      return k < args.max_pages ? bt[k] : -1;
    };
    int win = 0;
    int win_lo = load_window(0), win_hi = load_window(1);
    auto page_at = [&](int k) -> int {  // run page index k, warp-uniform
      return __shfl_sync(0xffffffffu, (k >> 5) == win ? win_lo : win_hi, k & 31);
    };
    // An untiled bulk L2 prefetch of each of the tile's two pages (36 KiB
    // contiguous each) right before the tile's TMA loads: measured a little
    // faster than the TMA loads alone, and faster than prefetching further
    // ahead (which only adds to the queues in front of the loads).
    constexpr uint32_t kPageBytes = 64 * 576;
    auto prefetch_tile = [&](int i) {
      const int tok0 = t0 + i * kTile;
      const int pa = page_at(2 * i);
      const bool want_b = tok0 + 64 < t1;
      const int pb = page_at(2 * i + 1);
      if (pa >= 0 && (int64_t)pa < args.num_pages)
        bulk_prefetch_l2_elect(args.kv_pages + (int64_t)pa * kPageBytes, kPageBytes);
      if (want_b && pb >= 0 && (int64_t)pb < args.num_pages)
        bulk_prefetch_l2_elect(args.kv_pages + (int64_t)pb * kPageBytes, kPageBytes);
    };
    int last_parity[kRingPairs];
    bool armed[kRingPairs];
    for (int i = 0; i < kRingPairs; ++i) armed[i] = false;
    int rope_last[kRopeSlots];
    for (int q = 0; q < kRopeSlots; ++q) rope_last[q] = -1;
    bool ok = true;
    int u = 0;  // load number of the next latent pair
    for (int i = 0; i < T && ok; ++i) {
      if ((2 * i) >> 5 > win) {  // the loads moved into the next window
        win_lo = win_hi;
        ++win;
        win_hi = load_window(win + 1);
      }
      // with several query-row groups the split's CTAs read the same pages
      // (the first reader brings them into L2) and the prefetches only add
      // to the queues: measured 2.4% faster at q_len 4 without them
      if (args.groups == 1) prefetch_tile(i);
      const int tok0 = t0 + i * kTile;
      const int pa = page_at(2 * i);
      const bool want_b = tok0 + 64 < t1;
      const int pb = want_b ? page_at(2 * i + 1) : 0;
      const bool la = pa >= 0 && (int64_t)pa < args.num_pages;
      const bool lb = want_b && pb >= 0 && (int64_t)pb < args.num_pages;
      if (lane == 0 && (!la || (want_b && !lb))) set_error(args.dev_error, MLA_DEVERR_BAD_PAGE);
      const uint32_t bytes_pair = (la ? 8192u : 0u) + (lb ? 8192u : 0u);  // 128 dims of both pages
      const uint32_t bytes_rope = (la ? 4096u : 0u) + (lb ? 4096u : 0u);
      const int rs = i % kRopeSlots;
      if (i >= kRopeSlots) {
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&bars[kBarRopeEmpty + rs], ((i / kRopeSlots) - 1) & 1, abort_flag));
        if (!ok) break;
      }
      uint64_t* rfull = &bars[kBarRopeFull + rs];
      mbar_arrive_expect_tx_elect(rfull, bytes_rope);
      rope_last[rs] = i;
      uint8_t* rdst = smem + kOffRope + rs * kChunk;
      if (la) tma_load_3d_elect(rdst, rope_map, rfull, 512, 0, pa);
      if (lb) tma_load_3d_elect(rdst + 4096, rope_map, rfull, 512, 0, pb);
      for (int j = 0; j < 4; ++j, ++u) {
        const int slot = u % kRingPairs;
        const int use = u / kRingPairs;  // how many times the slot was filled before
        if (use >= 1) {
          ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarEmpty + slot], (use - 1) & 1, abort_flag));
          if (!ok) break;
        }
        uint64_t* full = &bars[kBarFull + slot];
        if (args.inject_stall && i == 0 && j == 0 && blockIdx.x == 0)
          continue;  // test hook: this slot is never armed, so its waits run out
        mbar_arrive_expect_tx_elect(full, bytes_pair);
        armed[slot] = true;
        last_parity[slot] = use & 1;
        // latent dims [128 j, 128 j + 128) of the tile: [128 tokens][128 B],
        // 128-byte swizzle, the second page's 64 tokens 8 KiB in
        uint8_t* dst = smem + kOffRing + slot * kPair;
        if (la) tma_load_3d_elect(dst, kv_map, full, 128 * j, 0, pa);
        if (lb) tma_load_3d_elect(dst + 8192, kv_map, full, 128 * j, 0, pb);
      }
      if (!ok) break;
    }
    // drain: every armed transaction has landed before the CTA may exit
    const uint64_t t_start = globaltimer_ns();
    for (int i = 0; i < kRingPairs; ++i)
      if (armed[i])
        while (!mbar_try_wait(&bars[kBarFull + i], last_parity[i]) &&
               globaltimer_ns() - t_start < kWaitLimitNs) {
        }
    for (int rs = 0; rs < kRopeSlots; ++rs)
      if (rope_last[rs] >= 0)
        while (!mbar_try_wait(&bars[kBarRopeFull + rs], (rope_last[rs] / kRopeSlots) & 1) &&
               globaltimer_ns() - t_start < kWaitLimitNs) {
        }
  } else if (warp == 1) {
    // ============================================================ UMMA issuer
    // Warp-uniform scheduler; one elected lane issues each MMA and commit.
    const uint32_t idesc_qk = instr_desc(0, 0, 0, 0, 128, 128);  // E4M3, A K-major (TMEM or smem), B K-major, N=128
    const uint32_t idesc_pv = instr_desc(0, 0, 1, 0, 128, 64);   // A MN-major, B K-major, N=64
    // Latent pairs are [128 tokens][128 B] with the 128-byte swizzle: K-major
    // for QK (8-row groups 1 KiB apart) and MN-major for PV (one 128-dim atom
    // across M, 8-token groups 1 KiB apart).  The RoPE chunks and the Q' RoPE
    // operand are K-major with the 64-byte swizzle (8-row groups 512 B apart);
    // P is K-major with the 128-byte swizzle.
    const uint64_t dRingK = smem_desc(smem_u32(smem + kOffRing), 16, 1024, 2);
    const uint64_t dRope = smem_desc(smem_u32(smem + kOffRope), 16, 512, 4);
    const uint64_t dQr = smem_desc(smem_u32(smem + kOffQr), 16, 512, 4);
    const uint64_t dRingMN = smem_desc(smem_u32(smem + kOffRing), kPair, 1024, 2);
    const uint64_t dP = smem_desc(smem_u32(smem + kOffP), 16, 1024, 2);  // buffer 0, P_hi
    const uint32_t d_s = tmem + kTmemS;
    auto ready = [&](int bar, int parity) {
      return __any_sync(0xffffffffu, mbar_test_wait(&bars[bar], parity));
    };
    bool ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarQReady], 0, abort_flag));
    tc_fence_after();
    int nq = 0, qpair = 0, np = 0;
    bool s_free = false, rope_done = false;
    uint64_t idle_since = 0;
    uint32_t idle_spins = 0;
    // kBlock0First (the instance launched when a split has several query-row
    // groups, q_len > 1): block 0 of PV(np) goes ahead of a ready QK, since its
    // ring slot takes the last latent pair of tile np + 2, whose load is on
    // the critical loop (measured 3% faster at q_len 4; 2-3% slower at batch
    // 1, where the order stays QK first).
    constexpr bool pv_block0_first = kBlock0First;
    bool pv0 = false;  // block 0 of PV(np) issued
    while (ok && np < T) {
      bool progress = false;
      if (pv_block0_first && !pv0 && np < nq && ready(kBarPFull + np % kPBufs, (np / kPBufs) & 1) &&
          ready(kBarOReady + (np & 1), (np >> 1) & 1)) {
        tc_fence_after();
        const uint64_t dPhi = desc_at(dP, (np % kPBufs) * 2 * kChunk), dPlo = desc_at(dPhi, kChunk);
        const int slot = (4 * np) % kRingPairs;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t a = desc_at(dRingMN, slot * kPair + kk * 4096);
          umma_f8_fill_elect(tmem + kTmemO, a, desc_at(dPhi, kk * 32), idesc_pv,
                             (np > 0 || kk > 0) ? 1u : 0u);
          umma_f8_lastuse_elect(tmem + kTmemO, a, desc_at(dPlo, kk * 32), idesc_pv, 1u);
        }
        umma_commit_elect(&bars[kBarEmpty + slot]);
        pv0 = true;
        progress = true;
      }
      // ---------------- S'(nq) = Q' . K(nq)^T, one 128-dim pair at a time
      if (nq < T) {
        if (!s_free) {
          s_free = nq < 1 || ready(kBarSEmpty, (nq - 1) & 1);
          if (s_free) tc_fence_after();
        }
        // the RoPE chunk (loaded first) goes first when it has landed; the
        // first MMA of a tile starts S' afresh
        if (s_free && !rope_done && ready(kBarRopeFull + nq % kRopeSlots, (nq / kRopeSlots) & 1)) {
          tc_fence_after();
          const uint32_t r_off = (nq % kRopeSlots) * kChunk;
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            umma_f8_elect(d_s, desc_at(dQr, kk * 32), desc_at(dRope, r_off + kk * 32), idesc_qk,
                          (qpair > 0 || kk > 0) ? 1u : 0u);
          umma_commit_elect(&bars[kBarRopeEmpty + nq % kRopeSlots]);
          rope_done = true;
          progress = true;
        }
        while (s_free && qpair < 4 &&
               ready(kBarFull + (4 * nq + qpair) % kRingPairs, ((4 * nq + qpair) / kRingPairs) & 1)) {
          tc_fence_after();
          const uint32_t b_off = ((4 * nq + qpair) % kRingPairs) * kPair;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const int ks = 4 * qpair + kk;  // K step of 32 latent dims
            umma_f8_ts_elect(d_s, tmem + kTmemQ + 8 * ks, desc_at(dRingK, b_off + kk * 32), idesc_qk,
                             (rope_done || ks != 0) ? 1u : 0u);
          }
          ++qpair;
          progress = true;
        }
        if (s_free && qpair == 4 && rope_done) {
          umma_commit_elect(&bars[kBarSFull]);
          ++nq;
          qpair = 0;
          rope_done = false;
          s_free = false;
          progress = true;
        }
      }
      // ---------------- O^T += V(np)^T . (P_hi + P_lo), after any QK that was ready
      // (with block 0 first, the rest follows only in a pass that issued it
      // at the top, after any QK that was ready)
      if (pv0 || (!pv_block0_first && np < nq && ready(kBarPFull + np % kPBufs, (np / kPBufs) & 1) &&
                  ready(kBarOReady + (np & 1), (np >> 1) & 1))) {
        tc_fence_after();
        const uint64_t dPhi = desc_at(dP, (np % kPBufs) * 2 * kChunk), dPlo = desc_at(dPhi, kChunk);
        // block by block, so each latent pair can be refilled as soon as its
        // block is done (block 0 may have gone already)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (j == 0 && pv0) continue;
          const int slot = (4 * np + j) % kRingPairs;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t a = desc_at(dRingMN, slot * kPair + kk * 4096);  // tokens 32 kk ..
            umma_f8_fill_elect(tmem + kTmemO + 64 * j, a, desc_at(dPhi, kk * 32), idesc_pv,
                               (np > 0 || kk > 0) ? 1u : 0u);
            umma_f8_lastuse_elect(tmem + kTmemO + 64 * j, a, desc_at(dPlo, kk * 32), idesc_pv, 1u);
          }
          // latent pair j of this tile is free once its block's MMAs complete
          umma_commit_elect(&bars[kBarEmpty + slot]);
        }
        umma_commit_elect(&bars[kBarPEmpty + np % kPBufs]);
        umma_commit_elect(&bars[kBarPvDone]);
        if (np == T - 1) umma_commit_elect(&bars[kBarPvAll]);
        ++np;
        pv0 = false;
        progress = true;
      }
      if (progress) {
        idle_spins = 0;
      } else if ((++idle_spins & 63) == 0) {
        const uint64_t now = __shfl_sync(0xffffffffu, globaltimer_ns(), 0);
        if (idle_spins == 64) idle_since = now;
        if (__any_sync(0xffffffffu, *abort_flag != 0)) {
          ok = false;
        } else if (now - idle_since > kWaitLimitNs) {
          if (lane == 0) *abort_flag = 1;
          ok = false;
        }
      }
    }
    // drain: all issued MMAs complete before TMEM is released
    umma_commit_elect(&bars[kBarDrain]);
    const uint64_t t_start = globaltimer_ns();
    while (!mbar_try_wait(&bars[kBarDrain], 0) && globaltimer_ns() - t_start < kWaitLimitNs) {
    }
  } else if (warp >= 4 && warp < 4 + kSoftWarps) {
    // ============================================================ Q split + softmax
    const int qd = warp & 3;           // TMEM lane quadrant
    const int c = (warp - 4) >> 2;     // token slice: tokens 32c .. 32c+31 of a tile
    const int part = lane >> 4;        // 0: hi term, 1: lo term
    const int n = 16 * qd + (lane & 15);  // query row of this thread
    const bool valid = n < rows_valid;
    const int bar_id = 1 + qd;         // the four warps of this quadrant
    float c_head;                      // softmax_scale * kv_scale * log2(e) * 2^-e
    if (args.q8 != nullptr) {
      // ---- FP8 query: row n's slice c is its own E4M3 codes, used as they
      // are (a single term: the hi lanes hold the codes, the lo lanes zeros),
      // with the per-tensor scale folded into the score factor.
      const uint8_t* qrow = args.q8 + (row_base + n) * 576;
      const bool mine = valid && part == 0;
      uint32_t w[32];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint4 x = mine ? *reinterpret_cast<const uint4*>(qrow + 128 * c + 16 * k)
                             : make_uint4(0, 0, 0, 0);
        w[4 * k] = x.x;
        w[4 * k + 1] = x.y;
        w[4 * k + 2] = x.z;
        w[4 * k + 3] = x.w;
      }
      const uint4 r8 = mine ? *reinterpret_cast<const uint4*>(qrow + 512 + 16 * c)
                            : make_uint4(0, 0, 0, 0);
      c_head = valid ? args.qk_scale_log2 * args.q_scale : 0.0f;
      const uint32_t t_q = tmem + ((uint32_t)(32 * qd) << 16) + kTmemQ + 32 * c;
      float first[16], second[16];  // slice dims [0, 64) and [64, 128)
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        first[k] = __uint_as_float(w[k]);
        second[k] = __uint_as_float(w[16 + k]);
      }
      tmem_st16(t_q, first);
      tmem_st16(t_q + 16, second);
      *reinterpret_cast<uint4*>(smem + kOffQr + sw64(32 * qd + lane, 16 * c)) = r8;
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kBarQReady]);
    } else {
      // ---- Q -> Q' = [Q_hi ; Q_lo] with a power-of-two scale per query row.
      // Row n's slice c is latent dims [128c, 128c+128) and RoPE dims
      // [16c, 16c+16); the two lanes of the row (l and l ^ 16) each load one
      // half of it in a single round of loads, compute both terms of their
      // half, and swap the term the other lane needs.  The latent bytes go to
      // TMEM lane 32 qd + lane, the RoPE bytes to shared memory row 32 qd +
      // lane.  The row's amax is taken over all 576 dims (both halves of the
      // four slices).
      const uint16_t* qn = args.q_nope + (row_base + n) * 512 + 128 * c + 64 * part;
      const uint16_t* qr = args.q_rope + (row_base + n) * 64 + 16 * c + 8 * part;
      uint4 v[9];
#pragma unroll
      for (int k = 0; k < 8; ++k)
        v[k] = valid ? *reinterpret_cast<const uint4*>(qn + 8 * k) : make_uint4(0, 0, 0, 0);
      v[8] = valid ? *reinterpret_cast<const uint4*>(qr) : make_uint4(0, 0, 0, 0);
      uint32_t amax_bits = 0;
#pragma unroll
      for (int k = 0; k < 9; ++k) {
        const uint32_t w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          amax_bits = max(amax_bits, (w[e] << 16) & 0x7FFFFFFFu);
          amax_bits = max(amax_bits, w[e] & 0x7FFF0000u);
        }
      }
      amax_bits = max(amax_bits, __shfl_xor_sync(0xffffffffu, amax_bits, 16));
      if (part == 0) sc.red[c][n] = __uint_as_float(amax_bits);
      named_bar_sync(bar_id, 128);
      const float amax = fmaxf(fmaxf(sc.red[0][n], sc.red[1][n]), fmaxf(sc.red[2][n], sc.red[3][n]));
      int e = 0;
      if (amax > 0.0f && __float_as_uint(amax) < 0x7F800000u) {
        int E;
        frexpf(amax, &E);    // amax in [2^(E-1), 2^E)
        e = min(max(8 - E, -126), 126);  // amax * 2^e in [128, 256)
      }
      c_head = valid ? args.qk_scale_log2 * __uint_as_float((uint32_t)(127 - e) << 23) : 0.0f;
      const float sc_up = __uint_as_float((uint32_t)(127 + e) << 23);
      // this lane's term of its own 8 dims (mine) and of the partner's 8 dims
      // of the same position (got), for load k
      auto terms = [&](int k, uint2& mine, uint2& got) {
        const uint32_t w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
        float x[8];
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) {
          x[2 * e2] = __uint_as_float(w[e2] << 16) * sc_up;
          x[2 * e2 + 1] = __uint_as_float(w[e2] & 0xFFFF0000u) * sc_up;
        }
        const uint2 hi = term8(x, false), lo = term8(x, true);
        mine = part ? lo : hi;
        const uint2 give = part ? hi : lo;  // the partner's term of my dims
        got.x = __shfl_xor_sync(0xffffffffu, give.x, 16);
        got.y = __shfl_xor_sync(0xffffffffu, give.y, 16);
      };
      const uint32_t t_q = tmem + ((uint32_t)(32 * qd) << 16) + kTmemQ + 32 * c;
      {
        float first[16], second[16];  // slice dims [0, 64) and [64, 128) of this lane's term
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          uint2 mine, got;
          terms(k, mine, got);
          first[2 * k] = __uint_as_float(part ? got.x : mine.x);
          first[2 * k + 1] = __uint_as_float(part ? got.y : mine.y);
          second[2 * k] = __uint_as_float(part ? mine.x : got.x);
          second[2 * k + 1] = __uint_as_float(part ? mine.y : got.y);
        }
        tmem_st16(t_q, first);
        tmem_st16(t_q + 16, second);
      }
      {
        uint2 mine, got;
        terms(8, mine, got);
        const uint2 lo8 = part ? got : mine, hi8 = part ? mine : got;  // RoPE dims 0-7, 8-15 of the slice
        *reinterpret_cast<uint4*>(smem + kOffQr + sw64(32 * qd + lane, 16 * c)) =
            make_uint4(lo8.x, lo8.y, hi8.x, hi8.y);
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kBarQReady]);
    }

    // ---- softmax over S': this thread ends up with the scores of row n for
    // the 16 tokens 32c + 16 part .. +15 of each tile
    const int q_of_row = (r0 + n) / args.H;
    const int lim = valid ? min(t1, vis_base + q_of_row) : t0;  // tokens >= lim are invisible
    const uint32_t t_s = tmem + ((uint32_t)(32 * qd) << 16) + kTmemS + 32 * c;
    const int tid_s = tid - 128;       // 0..511
    float m_run = -INFINITY;           // max used for row n (log2 units)
    float l_run = 0.0f;                // this thread's share of row n's sum
    bool bad = false;
    for (int i = 0; i < T; ++i) {
      const int tok_base = t0 + i * kTile + 32 * c + 16 * part;
      bad |= !mbar_wait(&bars[kBarSFull], i & 1, abort_flag);
      tc_fence_after();
      float sv[16];
      {
        uint32_t r[32];
        tmem_ld32_nowait(t_s, r);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[kBarSEmpty]);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float keep = __uint_as_float(part ? r[16 + j] : r[j]);
          const float give = __uint_as_float(part ? r[j] : r[16 + j]);
          sv[j] = (keep + __shfl_xor_sync(0xffffffffu, give, 16)) * c_head;
        }
      }
      // visibility mask (split end, causal limit of the row, sequence end)
      if (tok_base + 16 > lim) {
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (tok_base + j >= lim) sv[j] = -INFINITY;
      }
      // does any score exceed the used max by more than the lazy threshold?
      bool exceed = false;
      const float thr = m_run + kLazy;
#pragma unroll
      for (int j = 0; j < 16; ++j) exceed |= sv[j] > thr;
      float alpha = 1.0f;
      bool moved = false;
      // One vote per quadrant and tile; its result is the same for all 128
      // threads, so they take the same barriers.  After a failed wait (bad)
      // a thread keeps looping: its waits return at once, the results are
      // discarded, and no thread is left at a named barrier.
      if (named_bar_or(bar_id, 128, exceed || bad)) {
        // some row of this quadrant may move: tile max per row over the 128 tokens
        float tm = sv[0];
#pragma unroll
        for (int j = 1; j < 16; ++j) tm = fmaxf(tm, sv[j]);
        tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 16));
        if (part == 0) sc.red[c][n] = tm;
        named_bar_sync(bar_id, 128);
        tm = fmaxf(fmaxf(sc.red[0][n], sc.red[1][n]), fmaxf(sc.red[2][n], sc.red[3][n]));
        moved = tm > thr;
        if (moved) {
          alpha = m_run == -INFINITY ? 0.0f : ex2_approx(m_run - tm);
          m_run = tm;
        }
      }
      // P buffer i % kPBufs free: PV of tile i - kPBufs done.  Waited for
      // before this tile's alpha goes out: PV(i - kPBufs) waited for the
      // rescale of that tile, so the alpha slot i % 2 has been read, and the
      // PV-done count the rescale warps test is at least i - 1.
      if (i >= kPBufs)
        bad |= !mbar_wait(&bars[kBarPEmpty + i % kPBufs], ((i / kPBufs) - 1) & 1, abort_flag);
      // the rescale warps learn, per tile, which rows moved and by how much
      if (c == 0) {
        const uint32_t mask = __ballot_sync(0xffffffffu, moved && part == 0);
        if (part == 0) sc.alpha[i & 1][n] = alpha;
        if (lane == 0) sc.changed[i & 1][qd] = mask & 0xFFFFu;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[kBarAlphaFull + (i & 1)]);
      }
      // weights carry a 2^3.5 factor: p' = 2^(s - m + 3.5) <= 2^8.75
      float pv[16];
      float psum = 0.0f;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        pv[j] = (sv[j] == -INFINITY) ? 0.0f : ex2_approx(sv[j] - m_run + kPShift);
        psum += pv[j];
      }
      l_run = fmaf(l_run, alpha, psum);
      uint4 phi, plo;
      split16(pv, phi, plo);
      const uint32_t p_off = kOffP + (i % kPBufs) * 2 * kChunk + sw128(n, 32 * c + 16 * part);
      *reinterpret_cast<uint4*>(smem + p_off) = phi;
      *reinterpret_cast<uint4*>(smem + p_off + kChunk) = plo;
      if (t0 + i * kTile + kTile > t1) {
        // token rows past the visible range: clear their V bytes so that
        // 0 * garbage cannot be NaN (thread: token row tid_s & 127, pair tid_s >> 7)
        const int r = tid_s & 127;
        if (t0 + i * kTile + r >= t1) {
          const int slot = (4 * i + (tid_s >> 7)) % kRingPairs;
          uint4* row = reinterpret_cast<uint4*>(smem + kOffRing + slot * kPair + r * 128);
#pragma unroll
          for (int k = 0; k < 8; ++k) row[k] = make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kBarPFull + i % kPBufs]);
    }
    // ---- row sums: reduce l over the 8 threads of row n, in a fixed order
    {
      const float l2 = l_run + __shfl_xor_sync(0xffffffffu, l_run, 16);
      named_bar_sync(bar_id, 128);  // red no longer read
      if (part == 0) sc.red[c][n] = l2;
      named_bar_sync(bar_id, 128);
      if (c == 0 && part == 0) {
        const float l = (sc.red[0][n] + sc.red[1][n]) + (sc.red[2][n] + sc.red[3][n]);
        const bool nonempty = !bad && l > 0.0f;
        sc.m_run[n] = m_run;
        if (own) {
          // the single launch keeps O in units of kv_scale (|O| <= 448 fits fp16)
          sc.inv_l[n] = nonempty ? (args.fused ? 1.0f : args.kv_scale) / l : 0.0f;
          if (valid)
            args.part_lse[(row_base + n) * slots + slot] =
                nonempty ? (m_run - kPShift + log2f(l)) * 0.69314718055994530942f : -INFINITY;
        } else {
          sc.inv_l[n] = nonempty ? l : 0.0f;  // raw row sum, merged across the cluster
        }
      }
    }
    named_bar_sync(6, kSoftThreads + 128);  // inv_l ready, every PV complete
  } else if (warp >= 4 + kSoftWarps) {
    // ============================================================ O^T rescale between tiles
    // The O-ready barriers are per tile parity because this loop may run one
    // tile ahead of the PV issue, but never two: the softmax of tile i + 2
    // sends its alpha only after PV(i), which waited for this loop's tile i.
    const int wq = warp & 3;            // thread = latent dim wq * 32 + lane of a block
    const uint32_t t_lane = tmem + ((uint32_t)(wq * 32) << 16);
    bool ok = true;
    for (int i = 0; i < T; ++i) {
      if (wq == 0 && lane == 0) mbar_wait(&bars[kBarAlphaFull + (i & 1)], (i >> 1) & 1, abort_flag);
      if (named_bar_or(5, 128, *abort_flag != 0)) {
        ok = false;
        break;
      }
      const uint32_t ch0 = i >= 1 ? sc.changed[i & 1][0] : 0u, ch1 = i >= 1 ? sc.changed[i & 1][1] : 0u;
      const uint32_t ch2 = i >= 1 ? sc.changed[i & 1][2] : 0u, ch3 = i >= 1 ? sc.changed[i & 1][3] : 0u;
      if ((ch0 | ch1 | ch2 | ch3) != 0) {
        // some row's max moved: O^T is rescaled once PV of the previous tile is done
        if (wq == 0 && lane == 0) mbar_wait(&bars[kBarPvDone], (i - 1) & 1, abort_flag);
        named_bar_sync(5, 128);
        tc_fence_after();
#pragma unroll 1
        for (int grp = 0; grp < 4; ++grp) {  // grp = lane quadrant = 16 query rows
          const uint32_t bits = grp == 0 ? ch0 : grp == 1 ? ch1 : grp == 2 ? ch2 : ch3;
          if (bits == 0) continue;
          float a[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) a[k] = sc.alpha[i & 1][grp * 16 + k];
#pragma unroll 1
          for (int j = 0; j < 4; ++j) {
            const uint32_t ta = t_lane + kTmemO + 64 * j + 16 * grp;
            float v[16];
            tmem_ld16(ta, v);
#pragma unroll
            for (int k = 0; k < 16; ++k) v[k] *= a[k];
            tmem_st16(ta, v);
          }
        }
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kBarOReady + (i & 1)]);
    }
    // every PV complete (a barrier of its own: the PV-done count may be one
    // or two tiles behind here, which one parity test cannot tell apart)
    if (ok && wq == 0 && lane == 0) mbar_wait(&bars[kBarPvAll], 0, abort_flag);
    named_bar_sync(5, 128);
    tc_fence_before();
    named_bar_sync(6, kSoftThreads + 128);  // inv_l ready, every PV complete
  }
  if (warp >= 4) {
    // ============================================================ epilogue (warps 4-23)
    // O^T -> shared memory, the sixteen [128 dims x 16 rows] TMEM chunks
    // spread over the five warpgroups (thread = latent dim of a block), as
    // row-major [64 rows][512 dims] in the free ring: O/l (fp32, or fp16 in
    // units of kv_scale in the single launch) when this CTA writes its own
    // partial, which then leaves row by row in 16-byte stores; unnormalised
    // fp32 O when the cut unit's pieces merge it across the cluster.
    tc_fence_after();
    const int ewg = (warp - 4) >> 2;  // 0..4
    const int wq = warp & 3;
    const int d_lane = wq * 32 + lane;
    const uint32_t t_lane = tmem + ((uint32_t)(wq * 32) << 16);
    float* staged = reinterpret_cast<float*>(smem + kOffRing);           // [64][512] fp32
    uint16_t* staged_h = reinterpret_cast<uint16_t*>(smem + kOffRing);   // [64][512] fp16
    if (*abort_flag == 0) {
#pragma unroll 1
      for (int ch = ewg; ch < 16; ch += 5) {
        const int j = ch >> 2, grp = ch & 3;
        float v[16];
        tmem_ld16(t_lane + kTmemO + 64 * j + 16 * grp, v);
        if (own && args.fused) {
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const int nn = grp * 16 + k;
            staged_h[nn * 512 + 128 * j + d_lane] = __half_as_ushort(__float2half_rn(v[k] * sc.inv_l[nn]));
          }
        } else if (own) {
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const int nn = grp * 16 + k;
            staged[nn * 512 + 128 * j + d_lane] = v[k] * sc.inv_l[nn];
          }
        } else {
#pragma unroll
          for (int k = 0; k < 16; ++k) staged[(grp * 16 + k) * 512 + 128 * j + d_lane] = v[k];
        }
      }
    }
    if (own) {
      named_bar_sync(6, kSoftThreads + 128);  // the staged rows are complete
      if (*abort_flag == 0) {
        const int vpr = args.fused ? 64 : 128;  // 16-byte vectors per row
        const uint4* src = reinterpret_cast<const uint4*>(smem + kOffRing);
        for (int i = tid - 128; i < rows_valid * vpr; i += kSoftThreads + 128) {
          const int n = i / vpr, c = i - n * vpr;
          const int64_t at = ((row_base + n) * slots + slot) * 512;
          uint4* dst = args.fused ? reinterpret_cast<uint4*>(args.part_o16 + at)
                                  : reinterpret_cast<uint4*>(args.part_o + at);
          dst[c] = src[i];
        }
      }
    }
  }
  // warps 2-3 and idle lanes fall through
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && tid == 0) set_error(args.dev_error, MLA_DEVERR_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (!own) merge_pieces(npieces, args, smem, sc, row_base, rows_valid, s);
}

// Single-launch mode, after every CTA's partial body: a grid barrier (the
// launch is cooperative, so every CTA is resident), then the log-sum-exp
// merge of each row's entries, spread over the grid.  An item is a run of
// 128 V dims of one row (thread t: dims t V .. t V + V - 1); gpi 128-thread
// groups of one CTA share an item, group j taking entries j, j + gpi, ...;
// a CTA works on 6 / gpi items at a time.  Each group merges its entries
// against its own maximum LSE (every entry load of a batch issued before the
// weights are applied), and the groups' results are combined through shared
// memory, so every sum has a fixed order (deterministic).  Each batch's LSEs
// are loaded with its values and folded into a running maximum, so a batch
// costs one round trip to L2.  V and gpi are
// chosen per launch by the launcher (merge_v, merge_gpi).  The last CTA to
// leave resets the two counters for the next launch.
constexpr int kMergeGroups = kThreads / 128;

// The raw words of V consecutive fp16 entries, loaded as they are (one
// register per entry for V <= 2, two for V = 4) and converted when used.
template <int V>
struct MergeRaw;
template <>
struct MergeRaw<1> {
  using T = unsigned short;
  __device__ static T load(const uint16_t* p) { return __ldcg(reinterpret_cast<const unsigned short*>(p)); }
  __device__ static T zero() { return 0; }
  __device__ static float at(T r, int) { return __half2float(__ushort_as_half(r)); }
};
template <>
struct MergeRaw<2> {
  using T = unsigned int;
  __device__ static T load(const uint16_t* p) { return __ldcg(reinterpret_cast<const unsigned int*>(p)); }
  __device__ static T zero() { return 0u; }
  __device__ static float at(T r, int v) {
    return __half2float(__ushort_as_half((unsigned short)(v ? r >> 16 : r & 0xFFFFu)));
  }
};
template <>
struct MergeRaw<4> {
  using T = uint2;
  __device__ static T load(const uint16_t* p) { return __ldcg(reinterpret_cast<const uint2*>(p)); }
  __device__ static T zero() { return make_uint2(0u, 0u); }
  __device__ static float at(T r, int v) {
    const uint32_t w = v < 2 ? r.x : r.y;
    return __half2float(__ushort_as_half((unsigned short)((v & 1) ? w >> 16 : w & 0xFFFFu)));
  }
};

template <int V>
__device__ __forceinline__ void merge_items(const DecodeArgs& a, uint8_t* smem) {
  constexpr int kB = V == 4 ? 12 : 32;  // entries per batch: 24-32 registers of loads in flight
  const int tid = threadIdx.x, grp = tid >> 7, t = tid & 127, lane = tid & 31;
  const int gpi = a.merge_gpi, ipc = kMergeGroups / gpi;
  const int sub = grp / gpi, j = grp % gpi;
  const int chunks = 4 / V;
  const int QH = a.q_len * a.H;
  const int items = a.B * QH * chunks;
  const int slots = a.max_splits * a.pieces;
  // exchange: [sub][buffer][group][128 V acc | m | w], the ring is free
  const int xstride = 128 * V + 2;
  float* xbase = reinterpret_cast<float*>(smem + kOffRing) + sub * 2 * gpi * xstride;
  int it = 0;
  for (int item = (int)blockIdx.x + sub * (int)gridDim.x; item < items;
       item += ipc * (int)gridDim.x, ++it) {
    const int row = item / chunks, d = (item % chunks) * 128 * V + t * V;
    const int bq = row / QH;
    int S = a.splits_const > 0 ? a.splits_const : a.num_splits[bq];
    S = S < 1 ? 0 : (S > a.max_splits ? a.max_splits : S);
    const int E = S * a.pieces;
    const int nj = E > j ? (E - j + gpi - 1) / gpi : 0;  // this group's entries
    const uint16_t* po = a.part_o16 + (int64_t)row * slots * 512 + d;
    const float* pl = a.part_lse + (int64_t)row * slots;
    // the group's entries in batches of kB, each batch's LSEs loaded with its
    // values (lane q: entry k0 + q), against a running maximum mj
    float mj = -INFINITY, acc[V], wsum = 0.0f;
#pragma unroll
    for (int v = 0; v < V; ++v) acc[v] = 0.0f;
    for (int k0 = 0; k0 < nj; k0 += kB) {
      typename MergeRaw<V>::T x[kB];
#pragma unroll
      for (int q = 0; q < kB; ++q)
        x[q] = k0 + q < nj ? MergeRaw<V>::load(po + (int64_t)(j + gpi * (k0 + q)) * 512)
                           : MergeRaw<V>::zero();
      const float lq = (lane < kB && k0 + lane < nj) ? __ldcg(pl + j + gpi * (k0 + lane)) : -INFINITY;
      float mb = lq;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, o));
      if (mb > mj) {  // warp-uniform; the sums so far are rescaled to the new maximum
        const float r = mj == -INFINITY ? 0.0f : expf(mj - mb);
        wsum *= r;
#pragma unroll
        for (int v = 0; v < V; ++v) acc[v] *= r;
        mj = mb;
      }
      const float wl = lq == -INFINITY ? 0.0f : expf(lq - mj);
#pragma unroll
      for (int q = 0; q < kB; ++q) {
        const float w = __shfl_sync(0xffffffffu, wl, q);
        wsum += w;
#pragma unroll
        for (int v = 0; v < V; ++v) acc[v] = fmaf(w, MergeRaw<V>::at(x[q], v), acc[v]);
      }
    }
    float M = mj, W = wsum;
    if (gpi > 1) {
      float* xb = xbase + (it & 1) * gpi * xstride;
      float* mine = xb + j * xstride;
#pragma unroll
      for (int v = 0; v < V; ++v) mine[t * V + v] = acc[v];
      if (t == 0) {
        mine[128 * V] = mj;
        mine[128 * V + 1] = wsum;
      }
      named_bar_sync(7 + sub, 128 * gpi);
      if (j == 0) {
        M = -INFINITY;
        for (int g = 0; g < gpi; ++g) M = fmaxf(M, xb[g * xstride + 128 * V]);
        W = 0.0f;
#pragma unroll
        for (int v = 0; v < V; ++v) acc[v] = 0.0f;
        for (int g = 0; g < gpi; ++g) {
          const float mg = xb[g * xstride + 128 * V];
          const float f = mg == -INFINITY ? 0.0f : expf(mg - M);
          W = fmaf(f, xb[g * xstride + 128 * V + 1], W);
#pragma unroll
          for (int v = 0; v < V; ++v) acc[v] = fmaf(f, xb[g * xstride + t * V + v], acc[v]);
        }
      }
    }
    if (j == 0) {
      const bool empty = M == -INFINITY || !(W > 0.0f);
      const float f = empty ? 0.0f : a.kv_scale / W;  // the entries are in units of kv_scale
      uint16_t h[V];
#pragma unroll
      for (int v = 0; v < V; ++v) h[v] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[v] * f));
      uint16_t* dst = a.out + (int64_t)row * 512 + d;
      if constexpr (V == 4) {
        *reinterpret_cast<uint2*>(dst) =
            make_uint2(h[0] | ((uint32_t)h[1] << 16), h[2] | ((uint32_t)h[3] << 16));
      } else if constexpr (V == 2) {
        *reinterpret_cast<uint32_t*>(dst) = h[0] | ((uint32_t)h[1] << 16);
      } else {
        dst[0] = h[0];
      }
      if (a.out_lse != nullptr && d == 0) a.out_lse[row] = empty ? -INFINITY : M + logf(W);
    }
  }
}

__device__ __forceinline__ void fused_merge(const DecodeArgs& a, uint8_t* smem) {
  Scratch& sc = *reinterpret_cast<Scratch*>(smem + kOffScratch);
  const int tid = threadIdx.x;
  __syncthreads();
  if (tid == 0) {
    __threadfence();  // this CTA's partial stores, ordered by the barrier above
    atomicAdd(a.sync, 1);
    const uint64_t t0 = globaltimer_ns();
    bool ok = true;
    while (*reinterpret_cast<volatile int32_t*>(a.sync) < (int)gridDim.x) {
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        ok = false;
        break;
      }
    }
    __threadfence();
    sc.merge_fail = ok ? 0 : 1;
    if (!ok) set_error(a.dev_error, MLA_DEVERR_TIMEOUT);
  }
  __syncthreads();
  if (sc.merge_fail == 0) {
    if (a.merge_v == 4)
      merge_items<4>(a, smem);
    else if (a.merge_v == 2)
      merge_items<2>(a, smem);
    else
      merge_items<1>(a, smem);
  }
  __syncthreads();
  if (tid == 0 && atomicAdd(a.sync + 1, 1) == (int)gridDim.x - 1) {
    // every CTA has passed the barrier: leave both counters at zero
    atomicExch(a.sync, 0);
    atomicExch(a.sync + 1, 0);
  }
}

template <bool kBlock0First>
__global__ void __launch_bounds__(kThreads, 1)
    decode_fp8_kernel(const DecodeArgs args, const __grid_constant__ CUtensorMap kv_map,
                      const __grid_constant__ CUtensorMap rope_map) {
  extern __shared__ __align__(1024) uint8_t smem[];
  partial_body<kBlock0First>(args, &kv_map, &rope_map, smem);
  if (args.fused) fused_merge(args, smem);
}

}  // namespace fp8k

cudaError_t launch_decode_fp8(const DecodeArgs& a, const CUtensorMap& kv_map,
                              const CUtensorMap& rope_map, cudaStream_t stream) {
  // the PV-order instance: block 0 first when a split has several row groups
  auto* kernel = a.groups > 1 ? fp8k::decode_fp8_kernel<true> : fp8k::decode_fp8_kernel<false>;
  // the shared-memory opt-in is a per-device attribute of the kernel: set it
  // on every launch (a cheap host call) so that any device the caller makes
  // current is configured
  cudaError_t e = cudaFuncSetAttribute(kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       fp8k::kSmemBytes);
  if (e != cudaSuccess) return e;
  const long long units = (long long)a.groups * a.max_splits * a.B;
  const long long ctas = a.split_from + a.pad + (units - a.split_from) * a.pieces;
  if (a.fused) {
    // the merge plan: vector width V and groups per item with the fewest
    // rounds of entry loads per CTA, (items per CTA slot) x (batches + 1)
    DecodeArgs f = a;
    const long long rows = (long long)a.B * a.q_len * a.H;
    const int E = a.max_splits * a.pieces;
    long long best = a.merge_v > 0 ? 0 : -1;  // a plan set by the test hook stands
    for (int V : {4, 2, 1}) {
      for (int gpi : {1, 2, 3, 6}) {
        const long long items = rows * (4 / V);
        const long long slots_per_round = ctas * (fp8k::kMergeGroups / gpi);
        const long long per = (E + gpi - 1) / gpi;
        const long long kb = V == 4 ? 12 : 32;  // entries per load batch
        const long long cost =
            ((items + slots_per_round - 1) / slots_per_round) * ((per + kb - 1) / kb + 1);
        if (best < 0 || (a.merge_v == 0 && cost < best)) {
          best = cost;
          f.merge_v = V;
          f.merge_gpi = gpi;
        }
      }
    }
    // every CTA must be resident for the grid barrier: a cooperative launch
    // guarantees it (or fails), and the pieces need no cluster here
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)ctas);
    cfg.blockDim = dim3(fp8k::kThreads);
    cfg.dynamicSmemBytes = fp8k::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, f, kv_map, rope_map);
  }
  if (a.pieces == 1) {
    kernel<<<(unsigned)ctas, fp8k::kThreads, fp8k::kSmemBytes, stream>>>(a, kv_map,
                                                                                         rope_map);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)ctas);
  cfg.blockDim = dim3(fp8k::kThreads);
  cfg.dynamicSmemBytes = fp8k::kSmemBytes;
  cfg.stream = stream;
  // the pieces of one split form a cluster (they merge through distributed
  // shared memory); the one-CTA units are paired into clusters that do not
  // interact
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)a.pieces;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, a, kv_map, rope_map);
}

}  // namespace mla
