// Steps A2-A8 for a bf16 latent cache: split-KV partial attention on sm_100a
// tensor cores (tcgen05 kind::f16), fed by TMA.
//
// "SGLang & Miles ... Vera Rubin" article, section "Kimi K3 的 MLA", bullets
// "更深的 MLA 流水线" (keep more KV reads in flight) and "更快的 split-KV 归约"
// (per-CTA partial results merged by a second kernel).
//
// Tensor-core mapping as in the FP8 kernel (tokens as UMMA M = 128, up to 64
// query rows as N, O^T accumulated in TMEM in four 128-dim blocks), with bf16
// operands.  One CTA per (64-row query group, split, request), a 3-D grid:
//   S^T[t][n] = K[t][:] . Q[n][:]        A = K chunk (K-major SW128), B = Q
//   O^T[d][n] += V^T[d][t] . P[t][n]     A = V pair (MN-major SW128), B = P (bf16)
// The query is exact in bf16, so no operand split is needed.
//
// A resident bf16 tile (144 KiB) does not fit beside the 72 KiB query, so the
// KV is streamed through a ring of four 32 KiB slots, each holding a 128-dim
// pair of chunks (or the 64-dim RoPE chunk) of one 128-token tile.  Loads and
// MMAs walk the same fixed order:
//   K(0) K(1) V(0) K(2) V(1) ... K(T-1) V(T-2) V(T-1)
// where K(i) is the five slots QK of tile i reads (four latent pairs and the
// RoPE chunk) and V(i) the four latent pairs PV of tile i reads.  V is loaded a
// second time, shortly after K, so that second read is served by L2; HBM sees
// every KV byte once, and each slot is held only from its load until its
// MMAs complete, which keeps up to 128 KiB of loads in flight.
//
// Warp roles (512 threads): producer (warp 0), warp-uniform MMA issuer
// (warp 1), two softmax warpgroups (warps 4-11, 32 query columns each, thread
// = token row), O^T rescale between tiles and epilogue (warps 12-15, thread =
// latent dim).  The online softmax (log2 domain, lazy running max moving only
// when exceeded by more than 8: bf16 weights up to 2^8 keep their 8
// significant bits, and the O^T rescale is rarely needed; 0.4-0.8% faster
// than a threshold of 1) and the bounded waits follow the FP8 kernel.
#include <cstdint>
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "mla.h"
#include "ptx.cuh"

namespace mla {
namespace bf16k {

constexpr int kThreads = 512;
constexpr int kRows = 64;            // query rows per CTA (UMMA N)
constexpr int kTile = 128;           // tokens per tile (UMMA M)
constexpr int kChunk = 128 * 128;    // 128 tokens x 64 dims bf16 = 16 KiB (rows of 128 B)
constexpr int kSlot = 2 * kChunk;    // a pair of chunks
constexpr int kSlots = 4;
constexpr int kQChunk = 64 * 128;    // 64 query rows x 64 dims bf16 = 8 KiB

constexpr int kOffQ = 0;                              // 9 chunks of [64 rows][128 B]
constexpr int kOffRing = kOffQ + 9 * kQChunk;         // 73728
constexpr int kOffP = kOffRing + kSlots * kSlot;      // 204800: [128 tokens][128 B]
constexpr int kOffScratch = kOffP + kTile * 128;      // 221184
constexpr int kSmemBytes = kOffScratch + 4096;        // 225280

constexpr int kBarFull = 0;       // 4
constexpr int kBarEmpty = 4;      // 4
constexpr int kBarSFull = 8;      // 2
constexpr int kBarSEmpty = 10;    // 2
constexpr int kBarPFull = 12;
constexpr int kBarPEmpty = 13;
constexpr int kBarOReady = 14;
constexpr int kBarPvDone = 15;
constexpr int kBarQReady = 16;
constexpr int kBarAlphaFull = 17;  // 2: per tile parity (the softmax groups may be a tile apart)
constexpr int kBarDrain = 19;

struct Scratch {
  uint64_t bars[24];
  uint32_t tmem_base;
  int abort;
  int pad[2];
  float warp_max[2][4][32];
  float m_run[64];
  float alpha[2][64];
  uint32_t changed[2][2];
  float c_head[64];
  float inv_l[64];
  uint8_t qcol[64];
};
static_assert(sizeof(Scratch) <= 4096, "scratch overflow");
static_assert(kSmemBytes <= 232448, "shared memory overflow");

// 128-byte swizzle of a 128-byte-row layout: 16-byte unit u of row r lives at
// unit u ^ (r & 7) (matches TMA SWIZZLE_128B and the UMMA SW128 layouts for a
// 1024-byte-aligned atom base).
__device__ __forceinline__ uint32_t sw128(uint32_t row, uint32_t byte_in_row) {
  return row * 128u + ((((byte_in_row >> 4) ^ (row & 7u)) << 4) | (byte_in_row & 15u));
}
__device__ __forceinline__ void set_error(int32_t* err, int bit) {
  if (err != nullptr) atomicOr(err, bit);
}
__device__ __forceinline__ uint64_t desc_at(uint64_t base, uint32_t bytes) {
  return base + (uint64_t)(bytes >> 4);
}

// Position of load number `u` in the fixed order K(0) K(1) V(0) K(2) V(1) ...:
// returns the tile and whether it is a V pair (else a K slot), and the index
// within that group (0-4 for K, 0-3 for V).  K(i) has 5 loads, V(i) 4.
__device__ __forceinline__ void load_at(int u, int T, int& tile, bool& is_v, int& idx) {
  // groups: K0 (5), then for i = 1..T-1: K(i) (5), V(i-1) (4); then V(T-1) (4)
  if (u < 5) {
    tile = 0;
    is_v = false;
    idx = u;
    return;
  }
  const int v = u - 5;
  const int grp = v / 9;  // pairs (K(grp+1), V(grp))
  const int in = v % 9;
  if (grp < T - 1) {
    if (in < 5) {
      tile = grp + 1;
      is_v = false;
      idx = in;
    } else {
      tile = grp;
      is_v = true;
      idx = in - 5;
    }
  } else {
    tile = T - 1;
    is_v = true;
    idx = v - 9 * (T - 1);
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    decode_bf16_kernel(const DecodeArgs args, const __grid_constant__ CUtensorMap kv_map) {
  extern __shared__ __align__(1024) uint8_t smem[];
  Scratch& sc = *reinterpret_cast<Scratch*>(smem + kOffScratch);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int g = blockIdx.x;
  const int s = blockIdx.y;
  const int b = blockIdx.z;
  const int QH = args.q_len * args.H;
  // the merge kernel that follows may be scheduled now; it waits for this
  // grid's completion before it reads any partial
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // ---------------------------------------------------------------- split range (step A2)
  const int L = args.seq_lens[b];
  const int S_b = args.num_splits[b];
  if (S_b < 1 || S_b > args.max_splits) {
    if (tid == 0 && s == 0 && g == 0) set_error(args.dev_error, MLA_DEVERR_BAD_SPLITS);
    return;
  }
  if (s >= S_b) return;
  if (L < args.q_len || (int64_t)L > (int64_t)args.max_pages * 64) {
    if (tid == 0 && s == 0 && g == 0) set_error(args.dev_error, MLA_DEVERR_BAD_SEQLEN);
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
  const int vis_base = L - args.q_len + 1;
  const int t0 = p0 * 64;
  const int t1 = min(p1 * 64, vis_base + q_max);
  const int t_all = min(t1, vis_base + q_min);
  const int64_t row_base = (int64_t)b * QH + r0;
  if (t1 <= t0) {
    for (int i = tid; i < rows_valid * 512; i += kThreads) {
      const int n = i >> 9;
      args.part_o[((row_base + n) * args.max_splits + s) * 512 + (i & 511)] = 0.0f;
    }
    if (tid < rows_valid) args.part_lse[(row_base + tid) * args.max_splits + s] = -INFINITY;
    return;
  }
  const int T = (t1 - t0 + kTile - 1) / kTile;
  const int n_loads = 9 * T;

  if ((smem_u32(smem) & 1023u) != 0) {
    if (tid == 0) set_error(args.dev_error, MLA_DEVERR_SMEM_ALIGN);
    return;
  }
  if (tid == 0) {
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(&sc.bars[kBarFull + i], 1);
      mbar_init(&sc.bars[kBarEmpty + i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sc.bars[kBarSFull + i], 1);
      mbar_init(&sc.bars[kBarSEmpty + i], 256);
    }
    mbar_init(&sc.bars[kBarPFull], 256);
    mbar_init(&sc.bars[kBarPEmpty], 1);
    mbar_init(&sc.bars[kBarOReady], 128);
    mbar_init(&sc.bars[kBarPvDone], 1);
    mbar_init(&sc.bars[kBarQReady], 8);
    for (int i = 0; i < 2; ++i) mbar_init(&sc.bars[kBarAlphaFull + i], 2);
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
    if (lane == 0) prefetch_tensormap(&kv_map);
    __syncwarp();
    const int32_t* bt = args.block_table + (int64_t)b * args.max_pages;
    bool ok = true;
    int last_parity[kSlots] = {0, 0, 0, 0};
    bool armed[kSlots] = {false, false, false, false};
    for (int u = 0; u < n_loads && ok; ++u) {
      int tile, idx;
      bool is_v;
      load_at(u, T, tile, is_v, idx);
      const int slot = u % kSlots;
      const int use = u / kSlots;
      if (use >= 1) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarEmpty + slot], (use - 1) & 1, abort_flag));
        if (!ok) break;
      }
      const int tok0 = t0 + tile * kTile;
      const int pa = bt[p0 + 2 * tile];
      const bool want_b = tok0 + 64 < t1;
      const int pb = want_b ? bt[p0 + 2 * tile + 1] : 0;
      const bool la = pa >= 0 && (int64_t)pa < args.num_pages;
      const bool lb = want_b && pb >= 0 && (int64_t)pb < args.num_pages;
      if (lane == 0 && (!la || (want_b && !lb))) set_error(args.dev_error, MLA_DEVERR_BAD_PAGE);
      const int nch = (!is_v && idx == 4) ? 1 : 2;  // the RoPE load is one chunk
      const uint32_t bytes = (uint32_t)nch * ((la ? 8192u : 0u) + (lb ? 8192u : 0u));
      uint64_t* full = &bars[kBarFull + slot];
      mbar_arrive_expect_tx_elect(full, bytes);
      armed[slot] = true;
      last_parity[slot] = use & 1;
      uint8_t* dst = smem + kOffRing + slot * kSlot;
      for (int c = 0; c < nch; ++c) {
        const int dim0 = (!is_v && idx == 4) ? 512 : 128 * idx + 64 * c;
        if (la) tma_load_3d_elect(dst + c * kChunk, &kv_map, full, dim0, 0, pa);
        if (lb) tma_load_3d_elect(dst + c * kChunk + 8192, &kv_map, full, dim0, 0, pb);
      }
    }
    const uint64_t t_start = globaltimer_ns();
    for (int i = 0; i < kSlots; ++i)
      if (armed[i])
        while (!mbar_try_wait(&bars[kBarFull + i], last_parity[i]) &&
               globaltimer_ns() - t_start < kWaitLimitNs) {
        }
  } else if (warp == 1) {
    // ============================================================ UMMA issuer
    const uint32_t idesc_qk = instr_desc(1, 1, 0, 0, 128, 64);  // bf16 K-major x K-major, N=64
    const uint32_t idesc_pv = instr_desc(1, 1, 1, 1, 128, 64);  // bf16 MN-major x MN-major
    const uint64_t dRingK = smem_desc(smem_u32(smem + kOffRing), 16, 1024, 2);
    const uint64_t dQ = smem_desc(smem_u32(smem + kOffQ), 16, 1024, 2);
    const uint64_t dRingMN = smem_desc(smem_u32(smem + kOffRing), kChunk, 1024, 2);
    const uint64_t dP = smem_desc(smem_u32(smem + kOffP), kChunk, 1024, 2);
    bool ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarQReady], 0, abort_flag));
    tc_fence_after();
    auto wait_slot = [&](int u) {
      return __all_sync(0xffffffffu,
                        mbar_wait(&bars[kBarFull + (u % kSlots)], (u / kSlots) & 1, abort_flag));
    };
    for (int u = 0; u < n_loads && ok;) {
      int tile, idx;
      bool is_v;
      load_at(u, T, tile, is_v, idx);
      if (!is_v) {
        // ---------------- S^T(tile) = K(tile) . Q^T over five slots
        const int sb = tile & 1;
        const uint32_t d_s = tmem + sb * 64;
        if (tile >= 2) {
          ok = __all_sync(0xffffffffu,
                          mbar_wait(&bars[kBarSEmpty + sb], ((tile - 2) >> 1) & 1, abort_flag));
          if (!ok) break;
        }
        tc_fence_after();
        for (int k5 = 0; k5 < 5 && ok; ++k5, ++u) {
          if (!(ok = wait_slot(u))) break;
          tc_fence_after();
          const uint32_t a_off = (u % kSlots) * kSlot;
          const int nch = k5 == 4 ? 1 : 2;
          for (int c = 0; c < nch; ++c) {
            const int qchunk = k5 == 4 ? 8 : 2 * k5 + c;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_f16_elect(d_s, desc_at(dRingK, a_off + c * kChunk + kk * 32),
                             desc_at(dQ, qchunk * kQChunk + kk * 32), idesc_qk,
                             (k5 | c | kk) != 0 ? 1u : 0u);
          }
          umma_commit_elect(&bars[kBarEmpty + (u % kSlots)]);
        }
        if (!ok) break;
        umma_commit_elect(&bars[kBarSFull + sb]);
      } else {
        // ---------------- O^T += V(tile)^T . P(tile) over four slots
        ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarPFull], tile & 1, abort_flag)) &&
             __all_sync(0xffffffffu, mbar_wait(&bars[kBarOReady], tile & 1, abort_flag));
        if (!ok) break;
        tc_fence_after();
        const bool tail = t0 + tile * kTile + kTile > t1;
        for (int j = 0; j < 4 && ok; ++j, ++u) {
          if (!(ok = wait_slot(u))) break;
          uint8_t* slot = smem + kOffRing + (u % kSlots) * kSlot;
          if (tail) {
            // rows past the visible range may hold anything (NaN included):
            // clear them so that 0 * garbage cannot reach O
            const int valid = t1 - (t0 + tile * kTile);
            for (int row = valid + lane; row < kTile; row += 32) {
              uint4* r0p = reinterpret_cast<uint4*>(slot + row * 128);
              uint4* r1p = reinterpret_cast<uint4*>(slot + kChunk + row * 128);
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                r0p[q] = make_uint4(0, 0, 0, 0);
                r1p[q] = make_uint4(0, 0, 0, 0);
              }
            }
            fence_proxy_async_smem();
            __syncwarp();
          }
          tc_fence_after();
          const uint32_t a_off = (u % kSlots) * kSlot;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_f16_elect(tmem + 128 + 64 * j, desc_at(dRingMN, a_off + kk * 2048),
                           desc_at(dP, kk * 2048), idesc_pv, (tile > 0 || kk > 0) ? 1u : 0u);
          umma_commit_elect(&bars[kBarEmpty + (u % kSlots)]);
        }
        if (!ok) break;
        umma_commit_elect(&bars[kBarPEmpty]);
        umma_commit_elect(&bars[kBarPvDone]);
      }
    }
    umma_commit_elect(&bars[kBarDrain]);
    const uint64_t t_start = globaltimer_ns();
    while (!mbar_try_wait(&bars[kBarDrain], 0) && globaltimer_ns() - t_start < kWaitLimitNs) {
    }
  } else if (warp >= 4 && warp < 12) {
    // ============================================================ Q copy + softmax
    const int wg = (warp - 4) >> 2;
    const int wq = warp & 3;
    {
      // ---- Q (bf16) -> K-major SW128 chunks of [64 rows][64 dims]
      const int pw = warp - 4;
      for (int n = pw; n < kRows; n += 8) {
        const bool valid = n < rows_valid;
        const uint16_t* qn = args.q_nope + (row_base + n) * 512;
        const uint16_t* qr = args.q_rope + (row_base + n) * 64;
        // 72 16-byte pieces per row: lanes take pieces lane, lane+32, lane+64
        for (int pc = lane; pc < 72; pc += 32) {
          uint4 v = make_uint4(0, 0, 0, 0);
          if (valid) v = pc < 64 ? *reinterpret_cast<const uint4*>(qn + pc * 8)
                                 : *reinterpret_cast<const uint4*>(qr + (pc - 64) * 8);
          const int dim0 = pc * 8;
          *reinterpret_cast<uint4*>(smem + kOffQ + (dim0 >> 6) * kQChunk + sw128(n, (dim0 & 63) * 2)) = v;
        }
        if (lane == 0) sc.c_head[n] = valid ? args.qk_scale_log2 : 0.0f;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kBarQReady]);
      named_bar_sync(5, 256);
    }
    const int r = wq * 32 + lane;
    const int col0 = wg * 32;
    const uint32_t t_lane = tmem + ((uint32_t)(wq * 32) << 16);
    const float4* c4 = reinterpret_cast<const float4*>(sc.c_head + col0);
    float l_part[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) l_part[j] = 0.0f;
    const int bar_id = 1 + wg;
    bool ok = true;
    bool bad = false;
    for (int i = 0; i < T; ++i) {
      const int sb = i & 1;
      const int tok = t0 + i * kTile + r;
      bad |= !mbar_wait(&bars[kBarSFull + sb], (i >> 1) & 1, abort_flag);
      tc_fence_after();
      float sv[32];
      {
        const uint32_t ts = t_lane + sb * 64 + col0;
        tmem_ld16x2(ts, ts + 16, sv, sv + 16);
#pragma unroll
        for (int j4 = 0; j4 < 8; ++j4) {
          const float4 c = c4[j4];
          sv[4 * j4 + 0] *= c.x;
          sv[4 * j4 + 1] *= c.y;
          sv[4 * j4 + 2] *= c.z;
          sv[4 * j4 + 3] *= c.w;
        }
      }
      tc_fence_before();
      mbar_arrive(&bars[kBarSEmpty + sb]);
      if (t0 + i * kTile + kTile > t_all) {
        const int qq = tok - vis_base;
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (tok >= t1 || (qq >= 0 && (int)sc.qcol[col0 + j] <= qq)) sv[j] = -INFINITY;
      }
      // does any score of this group's columns exceed its used max by more
      // than the lazy threshold?  If none does (the common case once the max
      // has settled), the column maxima are not reduced at all.
      bool exceed = false;
      {
        const float4* mo4 = reinterpret_cast<const float4*>(sc.m_run + col0);
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) {
          const float4 mo = mo4[q4];
          exceed |= sv[4 * q4] > mo.x + 8.0f;
          exceed |= sv[4 * q4 + 1] > mo.y + 8.0f;
          exceed |= sv[4 * q4 + 2] > mo.z + 8.0f;
          exceed |= sv[4 * q4 + 3] > mo.w + 8.0f;
        }
      }
      if (named_bar_or(bar_id, 128, bad || *abort_flag != 0)) {
        ok = false;
        break;
      }
      if (named_bar_or(bar_id, 128, exceed)) {
        float mine = -INFINITY;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float wm = warp_max_f32(sv[j]);
          mine = (lane == j) ? wm : mine;
        }
        sc.warp_max[wg][wq][lane] = mine;
        named_bar_sync(bar_id, 128);
        if (wq == 0) {
          const int n = col0 + lane;
          const float tm = fmaxf(fmaxf(sc.warp_max[wg][0][lane], sc.warp_max[wg][1][lane]),
                                 fmaxf(sc.warp_max[wg][2][lane], sc.warp_max[wg][3][lane]));
          const float m_old = sc.m_run[n];
          const bool moved = tm > m_old + 8.0f;
          const float m_new = moved ? tm : m_old;
          const float a = moved ? (m_old == -INFINITY ? 0.0f : ex2_approx(m_old - m_new)) : 1.0f;
          sc.m_run[n] = m_new;
          sc.alpha[i & 1][n] = a;
          const uint32_t mask = __ballot_sync(0xffffffffu, moved);
          if (lane == 0) sc.changed[i & 1][wg] = mask;
        }
      } else if (wq == 0) {
        sc.alpha[i & 1][col0 + lane] = 1.0f;
        if (lane == 0) sc.changed[i & 1][wg] = 0u;
      }
      named_bar_sync(bar_id, 128);
      if (wq == 0 && lane == 0) mbar_arrive(&bars[kBarAlphaFull + (i & 1)]);
      const float4* m4 = reinterpret_cast<const float4*>(sc.m_run + col0);
      const float4* a4 = reinterpret_cast<const float4*>(sc.alpha[i & 1] + col0);
      uint32_t pk[16];
#pragma unroll
      for (int q8 = 0; q8 < 4; ++q8) {
        const float4 ma = m4[2 * q8], mb = m4[2 * q8 + 1];
        const float4 aa = a4[2 * q8], ab = a4[2 * q8 + 1];
        const float mm[8] = {ma.x, ma.y, ma.z, ma.w, mb.x, mb.y, mb.z, mb.w};
        const float al[8] = {aa.x, aa.y, aa.z, aa.w, ab.x, ab.y, ab.z, ab.w};
#pragma unroll
        for (int k = 0; k < 8; k += 2) {
          const int j = 8 * q8 + k;
          // p = 2^(s - m) <= 2^8 with the lazy max; rounded to bf16 for the MMA,
          // and the row sum accumulates the rounded values
          const float p0 = (sv[j] == -INFINITY) ? 0.0f : ex2_approx(sv[j] - mm[k]);
          const float p1 = (sv[j + 1] == -INFINITY) ? 0.0f : ex2_approx(sv[j + 1] - mm[k + 1]);
          const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
          const float2 pr = __bfloat1622float2(pb);
          l_part[j] = fmaf(l_part[j], al[k], pr.x);
          l_part[j + 1] = fmaf(l_part[j + 1], al[k + 1], pr.y);
          pk[j >> 1] = *reinterpret_cast<const uint32_t*>(&pb);
        }
      }
      if (i >= 1) bad |= !mbar_wait(&bars[kBarPEmpty], (i - 1) & 1, abort_flag);
      {
        uint8_t* pp = smem + kOffP;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<uint4*>(pp + sw128(r, col0 * 2 + 16 * q)) =
              make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
      }
      fence_proxy_async_smem();
      mbar_arrive(&bars[kBarPFull]);
    }
    {
      float mine = 0.0f;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        float v = l_part[j];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        mine = (lane == j) ? v : mine;
      }
      named_bar_sync(bar_id, 128);
      sc.warp_max[wg][wq][lane] = mine;
      named_bar_sync(bar_id, 128);
      if (wq == 0) {
        const int n = col0 + lane;
        const float l = (sc.warp_max[wg][0][lane] + sc.warp_max[wg][1][lane]) +
                        (sc.warp_max[wg][2][lane] + sc.warp_max[wg][3][lane]);
        const bool nonempty = ok && l > 0.0f;
        sc.inv_l[n] = nonempty ? 1.0f / l : 0.0f;
        if (n < rows_valid)
          args.part_lse[(row_base + n) * args.max_splits + s] =
              nonempty ? (sc.m_run[n] + log2f(l)) * 0.69314718055994530942f : -INFINITY;
      }
    }
    named_bar_sync(4, 384);
  } else if (warp >= 12) {
    // ============================================================ O^T rescale + epilogue
    const int wq = warp & 3;
    const int d_lane = wq * 32 + lane;
    const uint32_t t_lane = tmem + ((uint32_t)(wq * 32) << 16);
    bool ok = true;
    for (int i = 0; i < T; ++i) {
      if (warp == 12 && lane == 0) {
        mbar_wait(&bars[kBarAlphaFull + (i & 1)], (i >> 1) & 1, abort_flag);
        if (i >= 1) mbar_wait(&bars[kBarPvDone], (i - 1) & 1, abort_flag);
      }
      if (named_bar_or(3, 128, *abort_flag != 0)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (i >= 1) {
        const uint32_t ch0 = sc.changed[i & 1][0], ch1 = sc.changed[i & 1][1];
        if ((ch0 | ch1) != 0) {
#pragma unroll 1
          for (int grp = 0; grp < 4; ++grp) {
            const uint32_t bits = ((grp < 2 ? ch0 : ch1) >> ((grp & 1) * 16)) & 0xFFFFu;
            if (bits == 0) continue;
            float a[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) a[c] = sc.alpha[i & 1][grp * 16 + c];
#pragma unroll 1
            for (int j = 0; j < 4; ++j) {
              const uint32_t ta = t_lane + 128 + 64 * j + 16 * grp;
              float v[16];
              tmem_ld16(ta, v);
#pragma unroll
              for (int c = 0; c < 16; ++c) v[c] *= a[c];
              tmem_st16(ta, v);
            }
          }
          tmem_wait_st();
        }
      }
      tc_fence_before();
      mbar_arrive(&bars[kBarOReady]);
    }
    if (ok && warp == 12 && lane == 0) mbar_wait(&bars[kBarPvDone], (T - 1) & 1, abort_flag);
    const bool bad = named_bar_or(3, 128, !ok || *abort_flag != 0);
    named_bar_sync(4, 384);
    if (!bad) {
      tc_fence_after();
      float* po = args.part_o + (row_base * args.max_splits + s) * 512;
      const int64_t row_stride = (int64_t)args.max_splits * 512;
#pragma unroll 1
      for (int j = 0; j < 4; ++j) {
#pragma unroll 1
        for (int grp = 0; grp < 4; ++grp) {
          float v[16];
          tmem_ld16(t_lane + 128 + 64 * j + 16 * grp, v);
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int n = grp * 16 + c;
            if (n < rows_valid) po[n * row_stride + 128 * j + d_lane] = v[c] * sc.inv_l[n];
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && tid == 0) set_error(args.dev_error, MLA_DEVERR_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace bf16k

cudaError_t launch_decode_bf16(const DecodeArgs& a, const CUtensorMap& kv_map,
                               cudaStream_t stream) {
  // the shared-memory opt-in is a per-device attribute of the kernel: set it
  // on every launch (a cheap host call) so that any device the caller makes
  // current is configured
  cudaError_t e = cudaFuncSetAttribute(bf16k::decode_bf16_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       bf16k::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int groups = (a.q_len * a.H + bf16k::kRows - 1) / bf16k::kRows;
  dim3 grid(groups, a.max_splits, a.B);
  bf16k::decode_bf16_kernel<<<grid, bf16k::kThreads, bf16k::kSmemBytes, stream>>>(a, kv_map);
  return cudaGetLastError();
}

}  // namespace mla
