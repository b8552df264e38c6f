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
// Tensor-core mapping (tokens as M): with at most 64 query rows per CTA,
// using the rows as M would run the half-width M=64 UMMA shape and would need
// a 64x512 fp32 O accumulator beside S, which does not fit TMEM.  Instead the
// 128 tokens of a tile are M=128:
//   S^T[t][n] = K[t][:] . Q[n][:]        A = K tile (K-major), B = Q (K-major)
//   O^T[d][n] += V^T[d][t] . P[t][n]     A = V tile (MN-major), B = P (MN-major)
// for d in four 128-wide blocks of the 512 latent dims.  V is the first 512
// columns of the same resident tile that fed K, so every KV byte crosses HBM
// once and shared memory once.
//
// Exact two-term FP8 operands: the cache is E4M3, and kind::f8f6f4 needs both
// operands E4M3.  Q (bf16, 8 significant bits) is scaled per row by a power
// of two and split as Q = Q_hi + Q_lo with Q_hi = Q rounded to 4 significant
// bits and Q_lo = E4M3(Q - Q_hi); this is exact for every element within a
// factor 2^-9 of the row maximum (smaller ones carry an absolute error of at
// most 2^-16 of the maximum).  B = [Q_hi ; Q_lo] is one N=128 operand, so S_hi and S_lo
// come out of one MMA and the softmax adds them.  The softmax weights are
// scaled by 2^7, p' = 2^(s - m + 7), and split the same way, P = P_hi + P_lo:
// about 8 significant bits (like bf16) for every p' >= 2^-2 and an absolute
// error of at most 2^-9 for smaller weights.  PV accumulates both terms; the scale
// cancels in O / l and is removed from the LSE.
//
// Online softmax (log2 domain, scores pre-multiplied by log2 e), with a lazy
// running max: the max m used for a row only moves when a tile's max exceeds
// it by more than 1.75 (log2 units), so p' stays <= 2^8.75 < 448, the E4M3
// maximum, and rescaling of the O^T columns and row sums (by
// 2^(m_old - m_new)) is rare.  A tile whose max moved nowhere does not wait
// for the previous tile's PV before its own PV is released.
//
// Warp roles (768 threads):
//   warp 0        TMA producer: pages -> 64-byte-swizzled chunks, plus L2
//                 prefetch of tiles up to three ahead
//   warp 1        UMMA issuer (warp-uniform polling of readiness, so a ready
//                 PV is never held behind QK data still in flight; one
//                 elected lane issues) and TMEM owner
//   warps 4-19    softmax in four warpgroups of 16 query columns each
//                 (thread = token row of S^T); the softmax of a tile is on
//                 the critical path of the two-tile ring, so it gets the
//                 most warps that the register file allows
//   warps 20-23   O^T rescaling between tiles (thread = latent dim)
//   warps 4-23    epilogue: O^T / l from TMEM to the partial output
//   warps 4-19    also convert Q to the split FP8 operand at the start
// TMEM (512 columns): S^T buffers at 0 and 128 (S_hi 0-63 | S_lo 64-127),
// O^T blocks at 256 + 64*j.
#include <cstdint>
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "mla.h"
#include "ptx.cuh"

namespace mla {
namespace fp8k {

constexpr int kThreads = 768;
constexpr int kSoftGroups = 4;      // softmax warpgroups
constexpr int kCols = 16;           // query columns per softmax warpgroup
constexpr int kSoftThreads = 128 * kSoftGroups;
constexpr int kRows = 64;           // query rows per CTA (UMMA N for PV)
constexpr int kTile = 128;          // tokens per tile (UMMA M)
constexpr int kChunk = 128 * 64;    // 128 tokens x 64 dims of E4M3 = 8 KiB
constexpr int kPair = 2 * kChunk;   // 128 latent dims of a tile
constexpr uint32_t kPageBytes = 64 * 576;  // one page of the pool
constexpr int kRingPairs = 8;       // two tiles of latent dims in flight
constexpr float kPShift = 7.0f;     // log2 of the factor carried by the softmax weights
constexpr float kLazy = 1.75f;       // the used max moves only when exceeded by more than this

constexpr int kOffQ = 0;                                 // 9 chunks, rows hi 0-63 | lo 64-127
constexpr int kOffRing = kOffQ + 9 * kChunk;             // 73728
constexpr int kOffRope = kOffRing + kRingPairs * kPair;  // 204800
constexpr int kOffPhi = kOffRope + kChunk;               // 212992
constexpr int kOffPlo = kOffPhi + kChunk;                // 221184
constexpr int kOffScratch = kOffPlo + kChunk;            // 229376
constexpr int kSmemBytes = 232448;                       // 227 KiB

// barrier indices
constexpr int kBarNopeFull = 0;    // 8
constexpr int kBarNopeEmpty = 8;   // 8
constexpr int kBarRopeFull = 16;
constexpr int kBarRopeEmpty = 17;
constexpr int kBarSFull = 18;      // 2
constexpr int kBarSEmpty = 20;     // 2
constexpr int kBarPFull = 22;
constexpr int kBarPEmpty = 23;
constexpr int kBarOReady = 24;     // 2: per tile parity (the rescale loop may run a tile ahead)
constexpr int kBarPvDone = 26;
constexpr int kBarQReady = 27;
constexpr int kBarAlphaFull = 28;  // 2: per tile parity (the softmax groups may be a tile apart)
constexpr int kBarDrain = 30;

struct Scratch {
  uint64_t bars[32];
  uint32_t tmem_base;
  int abort;
  int pad[2];
  float warp_max[4][4][16];  // per softmax group, per warp, per column; reused for row sums
  float m_run[64];           // max used per column (log2 units)
  float alpha[2][64];        // per tile parity: rescale factor per column
  uint32_t changed[2][4];    // per tile parity, per softmax group: columns whose max moved
  float c_head[64];          // per column: softmax_scale * kv_scale * log2(e) * 2^-e
  float inv_l[64];           // per column: kv_scale / l  (0 when l == 0)
  uint8_t qcol[64];          // per column: its query position q
};
static_assert(kOffScratch + sizeof(Scratch) <= kSmemBytes, "shared memory overflow");

// 64-byte swizzle of a 64-byte-row layout: 16-byte unit u of row r lives at
// unit u ^ ((r >> 1) & 3).  Matches the TMA 64B swizzle and the UMMA SW64
// canonical layout when the atom base is 512-byte aligned.
__device__ __forceinline__ uint32_t sw64(uint32_t row, uint32_t byte_in_row) {
  return row * 64u + ((((byte_in_row >> 4) ^ ((row >> 1) & 3u)) << 4) | (byte_in_row & 15u));
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

// Split 8 fp32 values into two E4M3 terms each: hi = x rounded to 4
// significant bits (round half away from zero on the bit pattern; an exact
// E4M3 value for |x| in the normal range), lo = E4M3(x - hi).  Result bytes
// are in element order.
__device__ __forceinline__ void split8(const float* x, uint2& hi, uint2& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float a = x[2 * k], b = x[2 * k + 1];
    const float ha = __uint_as_float((__float_as_uint(a) + 0x80000u) & 0xFFF00000u);
    const float hb = __uint_as_float((__float_as_uint(b) + 0x80000u) & 0xFFF00000u);
    h[k] = cvt_e4m3x2(ha, hb);
    l[k] = cvt_e4m3x2(a - ha, b - hb);
  }
  hi.x = h[0] | (h[1] << 16);
  hi.y = h[2] | (h[3] << 16);
  lo.x = l[0] | (l[1] << 16);
  lo.y = l[2] | (l[3] << 16);
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
  float* wgt = reinterpret_cast<float*>(smem + kOffPhi);  // [P][64] piece weights (P buffers are free)
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

__global__ void __launch_bounds__(kThreads, 1)
    decode_fp8_kernel(const DecodeArgs args, const __grid_constant__ CUtensorMap kv_map) {
  extern __shared__ __align__(1024) uint8_t smem[];
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
  const int g = unit % args.groups;
  const int s = (unit / args.groups) % args.max_splits;
  const int b = unit / (args.groups * args.max_splits);

  // ---------------------------------------------------------------- split range (step A2)
  const int L = args.seq_lens[b];
  const int S_b = args.num_splits[b];
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
  const int q_min = r0 / args.H;
  const int q_max = (r0 + rows_valid - 1) / args.H;
  const int vis_base = L - args.q_len + 1;  // visible length of q = 0
  const int t0s = p0 * 64;                         // the split's tokens [t0s, t1s)
  const int t1s = min(p1 * 64, vis_base + q_max);
  const int64_t row_base = (int64_t)b * QH + r0;

  if (t1s <= t0s) {  // empty split for every row of the group
    if (piece == 0) {
      for (int i = tid; i < rows_valid * 512; i += kThreads) {
        const int n = i >> 9;
        args.part_o[((row_base + n) * args.max_splits + s) * 512 + (i & 511)] = 0.0f;
      }
      if (tid < rows_valid) args.part_lse[(row_base + tid) * args.max_splits + s] = -INFINITY;
    }
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
  const int t_all = min(t1, vis_base + q_min);  // every column sees every token < t_all

  // ---------------------------------------------------------------- setup
  if ((smem_u32(smem) & 1023u) != 0) {  // same for every CTA of the grid
    if (tid == 0) set_error(args.dev_error, MLA_DEVERR_SMEM_ALIGN);
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
      mbar_init(&sc.bars[kBarNopeFull + i], 1);
      mbar_init(&sc.bars[kBarNopeEmpty + i], 1);
    }
    mbar_init(&sc.bars[kBarRopeFull], 1);
    mbar_init(&sc.bars[kBarRopeEmpty], 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sc.bars[kBarSFull + i], 1);
      mbar_init(&sc.bars[kBarSEmpty + i], kSoftThreads);
    }
    mbar_init(&sc.bars[kBarPFull], kSoftThreads);
    mbar_init(&sc.bars[kBarPEmpty], 1);
    for (int i = 0; i < 2; ++i) mbar_init(&sc.bars[kBarOReady + i], 128);
    mbar_init(&sc.bars[kBarPvDone], 1);
    mbar_init(&sc.bars[kBarQReady], 4 * kSoftGroups);
    for (int i = 0; i < 2; ++i) mbar_init(&sc.bars[kBarAlphaFull + i], kSoftGroups);
    mbar_init(&sc.bars[kBarDrain], 1);
    sc.abort = 0;
    fence_barrier_init();
  }
  if (tid < 64) {
    sc.m_run[tid] = -INFINITY;
    sc.qcol[tid] = (uint8_t)min((r0 + tid) / args.H, 255);
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
    // lane issues each TMA instruction and barrier arrival.
    if (lane == 0) prefetch_tensormap(&kv_map);
    __syncwarp();
    const int32_t* bt = args.block_table + (int64_t)b * args.max_pages;
    // L2 prefetch of a whole tile: each page is one contiguous 36 KiB block,
    // so one untiled bulk prefetch per page; page ids out of range are
    // skipped here and reported by the load path
    auto prefetch_tile = [&](int i) {
      const int tok0 = t0 + i * kTile;
      const int pa = bt[pg0 + 2 * i];
      const bool want_b = tok0 + 64 < t1;
      const int pb = want_b ? bt[pg0 + 2 * i + 1] : -1;
      if (pa >= 0 && (int64_t)pa < args.num_pages)
        bulk_prefetch_l2_elect(args.kv_pages + (int64_t)pa * kPageBytes, kPageBytes);
      if (want_b && pb >= 0 && (int64_t)pb < args.num_pages)
        bulk_prefetch_l2_elect(args.kv_pages + (int64_t)pb * kPageBytes, kPageBytes);
    };
    if (T > 2) prefetch_tile(2);
    int last_nope_parity[kRingPairs];
    bool armed[kRingPairs];
    for (int i = 0; i < kRingPairs; ++i) armed[i] = false;
    int rope_armed_tiles = 0;
    bool ok = true;
    for (int i = 0; i < T && ok; ++i) {
      if (i + 3 < T) prefetch_tile(i + 3);
      const int tok0 = t0 + i * kTile;
      const int pa = bt[pg0 + 2 * i];
      const bool want_b = tok0 + 64 < t1;
      const int pb = want_b ? bt[pg0 + 2 * i + 1] : 0;
      const bool la = pa >= 0 && (int64_t)pa < args.num_pages;
      const bool lb = want_b && pb >= 0 && (int64_t)pb < args.num_pages;
      if (lane == 0 && (!la || (want_b && !lb))) set_error(args.dev_error, MLA_DEVERR_BAD_PAGE);
      const uint32_t bytes_chunk = (la ? 4096u : 0u) + (lb ? 4096u : 0u);
      for (int j = 0; j < 4; ++j) {
        const int slot = (i & 1) * 4 + j;
        if (i >= 2) {
          ok = __all_sync(0xffffffffu,
                          mbar_wait(&bars[kBarNopeEmpty + slot], ((i - 2) >> 1) & 1, abort_flag));
          if (!ok) break;
        }
        uint64_t* full = &bars[kBarNopeFull + slot];
        if (args.inject_stall && i == 0 && j == 0 && blockIdx.x == 0)
          continue;  // test hook: this slot is never armed, so its waits run out
        mbar_arrive_expect_tx_elect(full, 2 * bytes_chunk);
        armed[slot] = true;
        last_nope_parity[slot] = (i >> 1) & 1;
        uint8_t* dst = smem + kOffRing + slot * kPair;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int chunk = 2 * j + cc;
          if (la) tma_load_3d_elect(dst + cc * kChunk, &kv_map, full, chunk * 64, 0, pa);
          if (lb) tma_load_3d_elect(dst + cc * kChunk + 4096, &kv_map, full, chunk * 64, 0, pb);
        }
      }
      if (!ok) break;
      if (i >= 1) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarRopeEmpty], (i - 1) & 1, abort_flag));
        if (!ok) break;
      }
      uint64_t* rfull = &bars[kBarRopeFull];
      mbar_arrive_expect_tx_elect(rfull, bytes_chunk);
      rope_armed_tiles = i + 1;
      if (la) tma_load_3d_elect(smem + kOffRope, &kv_map, rfull, 512, 0, pa);
      if (lb) tma_load_3d_elect(smem + kOffRope + 4096, &kv_map, rfull, 512, 0, pb);
    }
    // drain: every armed transaction has landed before the CTA may exit
    const uint64_t t_start = globaltimer_ns();
    for (int i = 0; i < kRingPairs; ++i)
      if (armed[i])
        while (!mbar_try_wait(&bars[kBarNopeFull + i], last_nope_parity[i]) &&
               globaltimer_ns() - t_start < kWaitLimitNs) {
        }
    if (rope_armed_tiles > 0)
      while (!mbar_try_wait(&bars[kBarRopeFull], (rope_armed_tiles - 1) & 1) &&
             globaltimer_ns() - t_start < kWaitLimitNs) {
      }
  } else if (warp == 1) {
    // ============================================================ UMMA issuer
    // Warp-uniform scheduler; one elected lane issues each MMA and commit.
    const uint32_t idesc_qk = instr_desc(0, 0, 0, 0, 128, 128);  // E4M3 K-major x K-major, N=128
    const uint32_t idesc_pv = instr_desc(0, 0, 1, 1, 128, 64);   // MN-major x MN-major, N=64
    // K-major SW64 (8-row groups 512 B apart) and MN-major SW64 (64-element
    // atoms 8 KiB apart, 8-row groups 512 B apart) descriptor bases
    const uint64_t dRingK = smem_desc(smem_u32(smem + kOffRing), 16, 512, 4);
    const uint64_t dRope = smem_desc(smem_u32(smem + kOffRope), 16, 512, 4);
    const uint64_t dQ = smem_desc(smem_u32(smem + kOffQ), 16, 512, 4);
    const uint64_t dRingMN = smem_desc(smem_u32(smem + kOffRing), kChunk, 512, 4);
    const uint64_t dPhi = smem_desc(smem_u32(smem + kOffPhi), kChunk, 512, 4);
    const uint64_t dPlo = smem_desc(smem_u32(smem + kOffPlo), kChunk, 512, 4);
    auto ready = [&](int bar, int parity) {
      return __any_sync(0xffffffffu, mbar_test_wait(&bars[bar], parity));
    };
    bool ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarQReady], 0, abort_flag));
    tc_fence_after();
    int nq = 0, qpair = 0, np = 0;
    bool s_free = false;
    uint64_t idle_since = 0;
    uint32_t idle_spins = 0;
    while (ok && np < T) {
      bool progress = false;
      // ---------------- S^T(nq) = K(nq) . [Q_hi ; Q_lo]^T, one 128-dim pair at a time
      if (nq < T) {
        const int sb = nq & 1;
        const uint32_t d_s = tmem + sb * 128;
        if (!s_free) {
          s_free = nq < 2 || ready(kBarSEmpty + sb, ((nq - 2) >> 1) & 1);
          if (s_free) tc_fence_after();
        }
        while (s_free && qpair < 4 && ready(kBarNopeFull + (nq & 1) * 4 + qpair, (nq >> 1) & 1)) {
          tc_fence_after();
          const uint32_t a_off = ((nq & 1) * 4 + qpair) * kPair;
          const uint32_t b_off = 2 * qpair * kChunk;
#pragma unroll
          for (int cc = 0; cc < 2; ++cc)
#pragma unroll
            for (int kk = 0; kk < 2; ++kk)
              umma_f8_elect(d_s, desc_at(dRingK, a_off + cc * kChunk + kk * 32),
                            desc_at(dQ, b_off + cc * kChunk + kk * 32), idesc_qk,
                            (qpair | cc | kk) != 0 ? 1u : 0u);
          ++qpair;
          progress = true;
        }
        if (s_free && qpair == 4 && ready(kBarRopeFull, nq & 1)) {
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            umma_f8_elect(d_s, desc_at(dRope, kk * 32), desc_at(dQ, 8 * kChunk + kk * 32),
                          idesc_qk, 1u);
          umma_commit_elect(&bars[kBarSFull + sb]);
          umma_commit_elect(&bars[kBarRopeEmpty]);
          ++nq;
          qpair = 0;
          s_free = false;
          progress = true;
        }
      }
      // ---------------- O^T += V(np)^T . (P_hi + P_lo)
      if (np < nq && ready(kBarPFull, np & 1) && ready(kBarOReady + (np & 1), (np >> 1) & 1)) {
        tc_fence_after();
        const uint32_t slot0 = (np & 1) * 4 * kPair;
        // block by block, so each latent pair can be refilled as soon as its
        // block is done
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
#pragma unroll
            for (int hl = 0; hl < 2; ++hl)
              umma_f8_elect(tmem + 256 + 64 * j, desc_at(dRingMN, slot0 + j * kPair + kk * 2048),
                            desc_at(hl ? dPlo : dPhi, kk * 2048), idesc_pv,
                            (np > 0 || kk > 0 || hl > 0) ? 1u : 0u);
          // latent pair j of this tile is free once its block's MMAs complete
          umma_commit_elect(&bars[kBarNopeEmpty + (np & 1) * 4 + j]);
        }
        umma_commit_elect(&bars[kBarPEmpty]);
        umma_commit_elect(&bars[kBarPvDone]);
        ++np;
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
  } else if (warp >= 4 && warp < 4 + 4 * kSoftGroups) {
    // ============================================================ Q split + softmax
    const int wg = (warp - 4) >> 2;  // softmax group: query columns 16*wg .. 16*wg+15
    const int wq = warp & 3;         // TMEM lane quadrant
    {
      // ---- Q -> [Q_hi ; Q_lo] in K-major SW64 chunks, per-row power-of-two scale
      const int pw = warp - 4;  // rows pw, pw + 16, ...
      for (int n = pw; n < kRows; n += 4 * kSoftGroups) {
        const bool valid = n < rows_valid;
        const uint16_t* qn = args.q_nope + (row_base + n) * 512;
        const uint16_t* qr = args.q_rope + (row_base + n) * 64;
        uint4 v[3];
        const int nch = lane < 8 ? 3 : 2;
        const int dim0[3] = {lane * 8, 256 + lane * 8, 512 + lane * 8};
        v[0] = valid ? *reinterpret_cast<const uint4*>(qn + lane * 8) : make_uint4(0, 0, 0, 0);
        v[1] = valid ? *reinterpret_cast<const uint4*>(qn + 256 + lane * 8) : make_uint4(0, 0, 0, 0);
        v[2] = (valid && lane < 8) ? *reinterpret_cast<const uint4*>(qr + lane * 8)
                                   : make_uint4(0, 0, 0, 0);
        uint32_t amax_bits = 0;
        for (int c = 0; c < nch; ++c) {
          const uint32_t w[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            amax_bits = max(amax_bits, (w[k] << 16) & 0x7FFFFFFFu);
            amax_bits = max(amax_bits, w[k] & 0x7FFF0000u);
          }
        }
        amax_bits = __reduce_max_sync(0xffffffffu, amax_bits);
        const float amax = __uint_as_float(amax_bits);
        int e = 0;
        if (amax > 0.0f && amax_bits < 0x7F800000u) {
          int E;
          frexpf(amax, &E);    // amax in [2^(E-1), 2^E)
          e = min(max(8 - E, -126), 126);  // amax * 2^e in [128, 256)
        }
        const float sc_up = __uint_as_float((uint32_t)(127 + e) << 23);
        for (int c = 0; c < nch; ++c) {
          const uint32_t w[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
          float x[8];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            x[2 * k] = __uint_as_float(w[k] << 16) * sc_up;
            x[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u) * sc_up;
          }
          uint2 hi, lo;
          split8(x, hi, lo);
          const int chunk = dim0[c] >> 6;
          const uint32_t bo = dim0[c] & 63;
          uint8_t* base = smem + kOffQ + chunk * kChunk;
          *reinterpret_cast<uint2*>(base + sw64(n, bo)) = hi;
          *reinterpret_cast<uint2*>(base + sw64(64 + n, bo)) = lo;
        }
        if (lane == 0)
          sc.c_head[n] = valid ? args.qk_scale_log2 * __uint_as_float((uint32_t)(127 - e) << 23)
                               : 0.0f;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kBarQReady]);
      named_bar_sync(7, kSoftThreads);  // c_head visible to every softmax group
    }

    // ---- softmax over S^T: thread = token row r of the tile, 16 query columns
    const int r = wq * 32 + lane;
    const int col0 = wg * kCols;
    const uint32_t t_lane = tmem + ((uint32_t)(wq * 32) << 16);
    const float4* c4 = reinterpret_cast<const float4*>(sc.c_head + col0);
    float l_part[kCols];
#pragma unroll
    for (int j = 0; j < kCols; ++j) l_part[j] = 0.0f;
    const int bar_id = 1 + wg;
    bool ok = true;
    bool bad = false;
    for (int i = 0; i < T; ++i) {
      const int sb = i & 1;
      const int tok = t0 + i * kTile + r;
      bad |= !mbar_wait(&bars[kBarSFull + sb], (i >> 1) & 1, abort_flag);
      tc_fence_after();
      float sv[kCols];
      {
        float hi[kCols], lo[kCols];
        const uint32_t ts = t_lane + sb * 128 + col0;
        tmem_ld16x2(ts, ts + 64, hi, lo);
#pragma unroll
        for (int j4 = 0; j4 < kCols / 4; ++j4) {
          const float4 c = c4[j4];
          sv[4 * j4 + 0] = (hi[4 * j4 + 0] + lo[4 * j4 + 0]) * c.x;
          sv[4 * j4 + 1] = (hi[4 * j4 + 1] + lo[4 * j4 + 1]) * c.y;
          sv[4 * j4 + 2] = (hi[4 * j4 + 2] + lo[4 * j4 + 2]) * c.z;
          sv[4 * j4 + 3] = (hi[4 * j4 + 3] + lo[4 * j4 + 3]) * c.w;
        }
      }
      tc_fence_before();
      mbar_arrive(&bars[kBarSEmpty + sb]);
      // visibility mask (split end, causal limit per column, sequence end)
      if (t0 + i * kTile + kTile > t_all) {
        const int qq = tok - vis_base;  // token invisible to columns whose q <= qq
#pragma unroll
        for (int j = 0; j < kCols; ++j)
          if (tok >= t1 || (qq >= 0 && (int)sc.qcol[col0 + j] <= qq)) sv[j] = -INFINITY;
      }
      // per-column tile max: warp redux, then across the 4 warps
      float mine = -INFINITY;
#pragma unroll
      for (int j = 0; j < kCols; ++j) {
        const float wm = warp_max_f32(sv[j]);
        mine = (lane == j) ? wm : mine;
      }
      if (lane < kCols) sc.warp_max[wg][wq][lane] = mine;
      if (named_bar_or(bar_id, 128, bad || *abort_flag != 0)) {
        ok = false;
        break;
      }
      if (wq == 0) {
        const int n = col0 + lane;
        bool moved = false;
        if (lane < kCols) {
          const float tm = fmaxf(fmaxf(sc.warp_max[wg][0][lane], sc.warp_max[wg][1][lane]),
                                 fmaxf(sc.warp_max[wg][2][lane], sc.warp_max[wg][3][lane]));
          const float m_old = sc.m_run[n];
          moved = tm > m_old + kLazy;
          const float m_new = moved ? tm : m_old;
          const float a = moved ? (m_old == -INFINITY ? 0.0f : ex2_approx(m_old - m_new)) : 1.0f;
          sc.m_run[n] = m_new;
          sc.alpha[i & 1][n] = a;
        }
        const uint32_t mask = __ballot_sync(0xffffffffu, moved);
        if (lane == 0) sc.changed[i & 1][wg] = mask;
      }
      named_bar_sync(bar_id, 128);
      if (wq == 0 && lane == 0) mbar_arrive(&bars[kBarAlphaFull + (i & 1)]);
      const float4* m4 = reinterpret_cast<const float4*>(sc.m_run + col0);
      const float4* a4 = reinterpret_cast<const float4*>(sc.alpha[i & 1] + col0);
      uint2 phi[kCols / 8], plo[kCols / 8];
#pragma unroll
      for (int q8 = 0; q8 < kCols / 8; ++q8) {
        const float4 ma = m4[2 * q8], mb = m4[2 * q8 + 1];
        const float4 aa = a4[2 * q8], ab = a4[2 * q8 + 1];
        const float mm[8] = {ma.x, ma.y, ma.z, ma.w, mb.x, mb.y, mb.z, mb.w};
        const float al[8] = {aa.x, aa.y, aa.z, aa.w, ab.x, ab.y, ab.z, ab.w};
        float pv[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int j = 8 * q8 + k;
          // weights carry a 2^7 factor: p' = 2^(s - m + 7) <= 2^8.75
          pv[k] = (sv[j] == -INFINITY) ? 0.0f : ex2_approx(sv[j] - mm[k] + kPShift);
          l_part[j] = fmaf(l_part[j], al[k], pv[k]);
        }
        split8(pv, phi[q8], plo[q8]);
      }
      // P buffer (and the V rows cleared below) free: PV of the previous tile done
      if (i >= 1) bad |= !mbar_wait(&bars[kBarPEmpty], (i - 1) & 1, abort_flag);
      *reinterpret_cast<uint4*>(smem + kOffPhi + sw64(r, col0)) =
          make_uint4(phi[0].x, phi[0].y, phi[1].x, phi[1].y);
      *reinterpret_cast<uint4*>(smem + kOffPlo + sw64(r, col0)) =
          make_uint4(plo[0].x, plo[0].y, plo[1].x, plo[1].y);
      if (tok >= t1) {
        // rows past the visible range: clear their V bytes so 0 * garbage cannot be NaN
        // (softmax group g clears latent pair g)
        const int pair = (i & 1) * 4 + wg;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          uint4* row = reinterpret_cast<uint4*>(smem + kOffRing + pair * kPair + cc * kChunk + r * 64);
#pragma unroll
          for (int u = 0; u < 4; ++u) row[u] = make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&bars[kBarPFull]);
    }
    // ---- row sums: reduce l_part over the 128 token rows of this group
    {
      float mine = 0.0f;
#pragma unroll
      for (int j = 0; j < kCols; ++j) {
        float v = l_part[j];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        mine = (lane == j) ? v : mine;
      }
      named_bar_sync(bar_id, 128);  // warp_max no longer read
      if (lane < kCols) sc.warp_max[wg][wq][lane] = mine;
      named_bar_sync(bar_id, 128);
      if (wq == 0 && lane < kCols) {
        const int n = col0 + lane;
        const float l = (sc.warp_max[wg][0][lane] + sc.warp_max[wg][1][lane]) +
                        (sc.warp_max[wg][2][lane] + sc.warp_max[wg][3][lane]);
        const bool nonempty = ok && l > 0.0f;
        if (npieces == 1) {
          sc.inv_l[n] = nonempty ? args.kv_scale / l : 0.0f;
          if (n < rows_valid)
            args.part_lse[(row_base + n) * args.max_splits + s] =
                nonempty ? (sc.m_run[n] - kPShift + log2f(l)) * 0.69314718055994530942f
                         : -INFINITY;
        } else {
          sc.inv_l[n] = nonempty ? l : 0.0f;  // raw row sum, merged across the cluster
        }
      }
    }
    named_bar_sync(6, kSoftThreads + 128);  // inv_l ready, every PV complete
  } else if (warp >= 4 + 4 * kSoftGroups) {
    // ============================================================ O^T rescale between tiles
    // The O-ready barriers are per tile parity because this loop may run one
    // tile ahead of the PV issue, but never two: tile i + 2 needs the ring
    // slots that PV(i) frees, and so its max and alpha.
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
        // some column's max moved: O^T is rescaled once PV of the previous tile is done
        if (wq == 0 && lane == 0) mbar_wait(&bars[kBarPvDone], (i - 1) & 1, abort_flag);
        named_bar_sync(5, 128);
        tc_fence_after();
#pragma unroll 1
        for (int grp = 0; grp < 4; ++grp) {  // grp = softmax group = 16 columns
          const uint32_t bits = grp == 0 ? ch0 : grp == 1 ? ch1 : grp == 2 ? ch2 : ch3;
          if (bits == 0) continue;
          float a[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) a[c] = sc.alpha[i & 1][grp * 16 + c];
#pragma unroll 1
          for (int j = 0; j < 4; ++j) {
            const uint32_t ta = t_lane + 256 + 64 * j + 16 * grp;
            float v[16];
            tmem_ld16(ta, v);
#pragma unroll
            for (int c = 0; c < 16; ++c) v[c] *= a[c];
            tmem_st16(ta, v);
          }
        }
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(&bars[kBarOReady + (i & 1)]);
    }
    // This loop may have run a tile ahead of PV, so the barrier can still be
    // one phase short of tile T-2: wait for that phase first, or the parity
    // test for T-1 would match the older phase T-3.
    if (ok && wq == 0 && lane == 0) {
      if (T >= 2) mbar_wait(&bars[kBarPvDone], (T - 2) & 1, abort_flag);
      mbar_wait(&bars[kBarPvDone], (T - 1) & 1, abort_flag);
    }
    named_bar_sync(5, 128);
    tc_fence_before();
    named_bar_sync(6, kSoftThreads + 128);  // inv_l ready, every PV complete
  }
  if (warp >= 4) {
    // ============================================================ epilogue (warps 4-23)
    // O^T / l -> part_o, the sixteen [128 dims x 16 columns] TMEM chunks
    // spread over the five warpgroups (thread = latent dim of a block)
    tc_fence_after();
    if (*abort_flag == 0) {
      const int ewg = (warp - 4) >> 2;  // 0..4
      const int wq = warp & 3;
      const int d_lane = wq * 32 + lane;
      const uint32_t t_lane = tmem + ((uint32_t)(wq * 32) << 16);
      float* po = args.part_o + (row_base * args.max_splits + s) * 512;
      const int64_t row_stride = (int64_t)args.max_splits * 512;
      float* staged = reinterpret_cast<float*>(smem + kOffRing);  // [64][512], ring is free
#pragma unroll 1
      for (int c = ewg; c < 16; c += 5) {
        const int j = c >> 2, grp = c & 3;
        float v[16];
        tmem_ld16(t_lane + 256 + 64 * j + 16 * grp, v);
        if (npieces == 1) {
#pragma unroll
          for (int cc = 0; cc < 16; ++cc) {
            const int n = grp * 16 + cc;
            if (n < rows_valid) po[n * row_stride + 128 * j + d_lane] = v[cc] * sc.inv_l[n];
          }
        } else {
          // unnormalised O, merged across the cluster below
#pragma unroll
          for (int cc = 0; cc < 16; ++cc) staged[(grp * 16 + cc) * 512 + 128 * j + d_lane] = v[cc];
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
  if (npieces > 1) merge_pieces(npieces, args, smem, sc, row_base, rows_valid, s);
}

}  // namespace fp8k

cudaError_t launch_decode_fp8(const DecodeArgs& a, const CUtensorMap& kv_map, cudaStream_t stream) {
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(fp8k::decode_fp8_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         fp8k::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const long long units = (long long)a.groups * a.max_splits * a.B;
  const long long ctas = a.split_from + a.pad + (units - a.split_from) * a.pieces;
  if (a.pieces == 1) {
    fp8k::decode_fp8_kernel<<<(unsigned)ctas, fp8k::kThreads, fp8k::kSmemBytes, stream>>>(a, kv_map);
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
  return cudaLaunchKernelEx(&cfg, fp8k::decode_fp8_kernel, a, kv_map);
}

}  // namespace mla
