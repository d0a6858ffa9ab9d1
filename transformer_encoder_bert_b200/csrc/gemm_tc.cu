// FP16 x FP16 -> FP32 tensor-core GEMM for sm_100a (tcgen05 + TMEM + TMA).
//
// The four matrix multiplies of an encoder layer (QKV, attention output,
// FFN1, FFN2) run here.  The source page ("Faster Transformer 优化原理")
// computes them with cuBLAS on Volta/Turing tensor cores and fuses the
// element-wise work around them into separate kernels; on B200 the
// element-wise work that follows a GEMM (add-bias + GELU, add-bias + Q/K/V
// head split) runs in this kernel's epilogue instead.
//
// C[M,N] = A[M,K] * B[N,K]^T, A and B K-major in global memory.
// Persistent kernel, one CTA per SM, warp roles:
//   warp 0      TMA producer: 128x64 A tile and BNx64 B tile per stage
//               (128-byte swizzle) into a STAGES-deep shared-memory ring.
//   warp 1      TMEM owner; one thread issues tcgen05.mma (M=128, N=BN, K=16,
//               four per 64-wide k-block) into one of two TMEM accumulators.
//   warps 2..9  epilogue: two warps per TMEM lane quadrant (32 rows), each
//               taking half of the tile's columns: tcgen05.ld, bias / GELU /
//               head split, TMA stores from a shared staging buffer.
// The two accumulators let the epilogue of tile i overlap the MMAs of tile
// i+1.  Every mbarrier wait is bounded (kWaitLimitNs); a wait that gives up
// records kStatusWaitTimeout in the status word and the CTA drains its copies
// and MMAs, frees TMEM and exits.
#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <mutex>

#include <cudaTypedefs.h>

#include "gelu.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace enc {
namespace {

using namespace sm100;

constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s
// Every wait in these kernels sleeps until its phase completes (suspend-time
// hint 100 us) rather than polling: the polling warps (epilogue warps waiting
// out a whole main loop, producer and MMA threads) otherwise take issue slots
// from the warps doing work.  Measured 8-10 % faster GEMMs.
constexpr uint32_t kSleepNs = 100000;
constexpr int kBM = 128;
constexpr int kBK = 64;
// Epilogue warps: 8 (two per TMEM lane quadrant) measured faster than 16 on
// every GEMM of the encoder (16 warps cap the registers at 96 per thread).
#ifndef ENC_EPI_WARPS
#define ENC_EPI_WARPS 8
#endif
constexpr int kEpiWarps = ENC_EPI_WARPS;     // 8 or 16: 2 or 4 warps per TMEM lane quadrant
constexpr int kEpiSlices = kEpiWarps / 4;    // column slices of a tile
constexpr int kThreads = 64 + 32 * kEpiWarps;

template <int BN>
struct Cfg {
  static constexpr int kStages = BN == 256 ? 3 : 5;
  static constexpr int kABytes = kBM * kBK * 2;
  static constexpr int kBBytes = BN * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = 2 * BN;
  // full[kStages], empty[kStages], tfull[2], tempty[2], drain, then two residual barriers per epilogue warp
  static constexpr int kResBar0 = 2 * kStages + 5;
  static constexpr int kNumBars = kResBar0 + 2 * kEpiWarps;
  static constexpr int kBiasOffset = (kStages * kStageBytes + kNumBars * 8 + 16 + 15) / 16 * 16;
  static constexpr int kStoreOffset = (kBiasOffset + kEpiWarps * (BN / kEpiSlices) * 4 + 1023) / 1024 * 1024;
  static constexpr int kSmem = 1024 + kStoreOffset + kEpiWarps * 2 * (32 * 32 * 2);   // two staging buffers per warp
};

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Per-thread destination of one output row: for the head split, the part of
// the address that depends on the token only (b, s); otherwise row * N.
template <Epi EPI>
__device__ __forceinline__ size_t row_offset(int row, int N, const SplitShape& sp) {
  if constexpr (EPI == Epi::kBiasQkvSplit) {
    const int b = row / sp.seq;
    const int s = row - b * sp.seq;
    return ((size_t)b * sp.head_num * sp.seq + s) * sp.size_per_head;
  } else {
    return (size_t)row * N;
  }
}

// The part that depends on the column (uniform across the warp): for the head
// split, column n = t*H + h*d + c goes to block t, head h, offset c.
template <Epi EPI>
__device__ __forceinline__ size_t col_offset(int col0, const SplitShape& sp) {
  if constexpr (EPI == Epi::kBiasQkvSplit) {
    const int H = sp.head_num * sp.size_per_head;
    const int t = col0 / H;
    const int rem = col0 - t * H;
    const int h = rem / sp.size_per_head;
    const int c = rem - h * sp.size_per_head;
    return ((size_t)t * sp.batch * sp.head_num + h) * sp.seq * sp.size_per_head + c;
  } else {
    return (size_t)col0;
  }
}

// Epilogue math for one thread: 32 accumulator columns of one row, plus bias
// and the element-wise function.  `bias_s` holds the bias of these 32 columns
// (shared memory, read as a broadcast).
template <Epi EPI>
__device__ __forceinline__ void epilogue_values(const uint32_t (&r)[32], const float* bias_s, float (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
  if constexpr (EPI != Epi::kStore) {
#pragma unroll
    for (int i = 0; i < 32; i += 4) {
      const float4 b = *reinterpret_cast<const float4*>(bias_s + i);
      v[i] += b.x; v[i + 1] += b.y; v[i + 2] += b.z; v[i + 3] += b.w;
    }
  }
  if constexpr (EPI == Epi::kBiasGelu) {
#pragma unroll
    for (int i = 0; i < 32; i += 2) act::gelu_erf_pair(v[i], v[i + 1]);
  }
  if constexpr (EPI == Epi::kBiasGeluTanh) {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = act::gelu_tanh(v[i]);
  }
}

// v += 8 halves (one 16-byte unit) of the residual, columns 8u .. 8u+7.
__device__ __forceinline__ void add_residual_unit(float (&v)[32], int u, const uint4& res) {
  const __half2* h = reinterpret_cast<const __half2*>(&res);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 f = __half22float2(h[j]);
    v[8 * u + 2 * j] += f.x;
    v[8 * u + 2 * j + 1] += f.y;
  }
}

// Bytes of one warp's staging buffer: a 32x32 FP16 chunk.
constexpr int kStageChunkBytes = 32 * 32 * 2;

// Byte offset of 16-byte unit u (0..3) of row r in a staging buffer with the
// output map's 64-byte swizzle: unit u of row r sits at unit u ^ ((r >> 1) & 3).
__device__ __forceinline__ int stage_unit(int r, int u) { return r * 64 + 16 * (u ^ ((r >> 1) & 3)); }

// An epilogue warp's state across tiles: two staging buffers used in turn
// (chunk i in buffer i & 1), and for kBiasResidStore through TMA the two
// mbarriers on which the residual chunk loaded into each buffer completes.
struct EpiWarpState {
  uint8_t* stage;             // 2 x kStageChunkBytes
  uint32_t seq = 0;           // chunks written so far
  const CUtensorMap* tm_r = nullptr;
  uint32_t res_bar = 0;       // buffer k's barrier at res_bar + 8k
  uint32_t res_phase = 0;     // bit k: parity of buffer k's next completion
};

// One epilogue warp's share of a tile: rows [32*quad, 32*quad+32) of the
// accumulator (one row per lane), global columns [col_begin, col_begin +
// 32*CHUNKS), whose first column sits at TMEM address t_cols (lane field
// included); `row0` is the global row of lane 0.
// The bias of those columns is staged in the warp's shared-memory slot before
// the accumulator is awaited; the TMEM load of chunk j+1 is in flight while
// chunk j is converted and stored.  `release` runs once the last TMEM load of
// the tile has completed (it frees the accumulator for the next tile).
// Stores: with an output map (tm_c != nullptr) each 32x32 chunk is written to
// a staging buffer in the map's 64-byte swizzle and stored by a TMA bulk copy
// (full lines, no per-lane stores).  Otherwise each lane stores its row with
// 16-byte stores.
// Residual (kBiasResidStore): with an output map, the residual chunk is
// brought into the chunk's staging buffer by a TMA load (the next chunk's
// while this one is processed) and added in place; otherwise each lane loads
// its row's halves.
template <Epi EPI, int CHUNKS, int NBUF = 2, typename WaitFull, typename Release>
__device__ __forceinline__ bool epilogue_warp_tile(uint32_t t_cols, int row0, int col_begin, int M, int N,
                                                   const float* __restrict__ bias, float* bias_s,
                                                   __half* __restrict__ C, const SplitShape& sp,
                                                   const CUtensorMap* tm_c, EpiWarpState& ws,
                                                   const __half* __restrict__ resid, WaitFull wait_full,
                                                   Release release) {
  const int lane = threadIdx.x & 31;
  if constexpr (EPI != Epi::kStore) {
    for (int i = lane * 4; i < 32 * CHUNKS; i += 128) {   // CHUNKS <= 4
      float4 b = make_float4(0.f, 0.f, 0.f, 0.f);
      if (col_begin + i < N) b = *reinterpret_cast<const float4*>(bias + col_begin + i);
      *reinterpret_cast<float4*>(bias_s + i) = b;
    }
  }
  const int row = row0 + lane;
  const bool row_ok = row < M;
  const size_t roff = row_ok ? row_offset<EPI>(row, N, sp) : 0;
  // Token coordinates of the chunk's first row for the head-split store map.
  const int b0 = EPI == Epi::kBiasQkvSplit ? row0 / sp.seq : 0;
  const int s0 = EPI == Epi::kBiasQkvSplit ? row0 - b0 * sp.seq : 0;
  constexpr bool kResid = EPI == Epi::kBiasResidStore;
  const bool tma_resid = kResid && tm_c != nullptr && ws.tm_r != nullptr;
  // With a buffer per chunk (NBUF >= CHUNKS) every residual chunk of the tile
  // is requested before the accumulator is awaited, chunk j into buffer j;
  // otherwise two buffers alternate and the residual runs one chunk ahead.
  constexpr bool kAllAhead = NBUF >= CHUNKS;
  auto buf_of = [&](uint32_t seq) {
    return ws.stage + (kAllAhead ? (seq % (uint32_t)NBUF) : (seq & 1u)) * kStageChunkBytes;
  };
  // Lane 0: residual chunk j into the buffer of chunk number `seq`, once every
  // store this thread issued has read its buffer.
  auto issue_res = [&](uint32_t seq, int j) {
    if (!kAllAhead) sm100::bulk_wait_group_read<0>();
    const uint32_t bar = ws.res_bar + 8u * (kAllAhead ? (seq % (uint32_t)NBUF) : (seq & 1u));
    sm100::mbar_arrive_expect_tx(bar, kStageChunkBytes);
    sm100::tma_load_2d(ws.tm_r, sm100::smem_u32(buf_of(seq)), bar, col_begin + 32 * j, row0);
  };
  if (tma_resid && lane == 0) {
    if constexpr (kAllAhead) {
      sm100::bulk_wait_group_read<0>();        // the previous tile's stores have read every buffer
      for (int j = 0; j < CHUNKS; ++j)
        if (col_begin + 32 * j < N) issue_res(ws.seq + j, j);
    } else if (col_begin < N) {
      issue_res(ws.seq, 0);
    }
  }
  // Per-lane residual path: chunk 0 before the accumulator is awaited, chunk
  // j+1 while chunk j is processed.
  uint4 res_a[4] = {}, res_b[kResid ? 4 : 1] = {};
  auto load_res = [&](int j, uint4* dst) {
    const int c0 = col_begin + 32 * j;
    if (!row_ok || c0 >= N) return;
    const uint4* rp = reinterpret_cast<const uint4*>(resid + (size_t)row * N + c0);
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (c0 + 8 * u < N) dst[u] = rp[u];
  };
  if (kResid && !tma_resid) load_res(0, res_a);
  int got = 0;
  if (lane == 0) got = wait_full() ? 1 : 0;
  got = __shfl_sync(0xffffffffu, got, 0);     // also orders the bias staging before its use
  if (!got) return false;
  sm100::tc_fence_after();
  // With more than two chunks per warp the next chunk's TMEM load is issued
  // before the current one is processed; with one or two, other warps hide it.
  constexpr bool kPrefetch = CHUNKS > 2;
  uint32_t ra[32], rb[kPrefetch ? 32 : 1];
  if constexpr (kPrefetch) sm100::tmem_ld_32x32b_x32_async(t_cols, ra);
#pragma unroll
  for (int j = 0; j < CHUNKS; ++j) {
    uint32_t* cur_p;
    if constexpr (kPrefetch) {
      uint32_t(&cur)[32] = (j & 1) ? *reinterpret_cast<uint32_t(*)[32]>(rb) : ra;
      uint32_t(&nxt)[32] = (j & 1) ? ra : *reinterpret_cast<uint32_t(*)[32]>(rb);
      sm100::tmem_wait_ld(cur);
      if (j + 1 < CHUNKS) sm100::tmem_ld_32x32b_x32_async(t_cols + 32 * (j + 1), nxt);
      cur_p = cur;
    } else {
      sm100::tmem_ld_32x32b_x32(t_cols + 32 * j, ra);
      cur_p = ra;
    }
    if (j + 1 == CHUNKS) {
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) release();
    }
    uint32_t(&cur)[32] = *reinterpret_cast<uint32_t(*)[32]>(cur_p);
    const int col0 = col_begin + 32 * j;
    if (col0 >= N) continue;
    if (kResid && !tma_resid && j + 1 < CHUNKS) load_res(j + 1, (j & 1) ? res_a : res_b);
    if (!kAllAhead && tma_resid && lane == 0 && j + 1 < CHUNKS && col0 + 32 < N) issue_res(ws.seq + 1, j + 1);
    float v[32];
    epilogue_values<EPI>(cur, bias_s + 32 * j, v);
    uint8_t* buf = buf_of(ws.seq);
    if (tma_resid) {
      const uint32_t k = kAllAhead ? (ws.seq % (uint32_t)NBUF) : (ws.seq & 1u);
      int ok = 0;
      if (lane == 0) ok = mbar_wait<kSleepNs>(ws.res_bar + 8u * k, (ws.res_phase >> k) & 1u, kWaitLimitNs) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) return false;
      ws.res_phase ^= 1u << k;
#pragma unroll
      for (int u = 0; u < 4; ++u) add_residual_unit(v, u, *reinterpret_cast<const uint4*>(buf + stage_unit(lane, u)));
    } else if constexpr (kResid) {
      const uint4* res = (j & 1) ? res_b : res_a;
#pragma unroll
      for (int u = 0; u < 4; ++u) add_residual_unit(v, u, res[u]);
    }
    uint32_t p[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) p[i] = pack_half2(v[2 * i], v[2 * i + 1]);
    if (tm_c != nullptr) {
      // The buffer was last read by the store two chunks back (with a TMA
      // residual load, that wait came before the load was issued).
      if (!tma_resid && lane == 0) sm100::bulk_wait_group_read<1>();
      __syncwarp();
#pragma unroll
      for (int u = 0; u < 4; ++u)
        *reinterpret_cast<uint4*>(buf + stage_unit(lane, u)) =
            make_uint4(p[4 * u], p[4 * u + 1], p[4 * u + 2], p[4 * u + 3]);
      sm100::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        if constexpr (EPI == Epi::kBiasQkvSplit) {
          const int H = sp.head_num * sp.size_per_head;
          const int t = col0 / H;
          const int rem = col0 - t * H;
          const int h = rem / sp.size_per_head;
          const int c = rem - h * sp.size_per_head;
          if (b0 < sp.batch) sm100::tma_store_5d(tm_c, sm100::smem_u32(buf), c, s0, h, b0, t);
        } else {
          sm100::tma_store_2d(tm_c, sm100::smem_u32(buf), col0, row0);
        }
        sm100::bulk_commit_group();
      }
      ++ws.seq;
    } else if (row_ok) {
      __half* dst = C + roff + col_offset<EPI>(col0, sp);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (col0 + 8 * u < N)
          *reinterpret_cast<uint4*>(dst + 8 * u) = make_uint4(p[4 * u], p[4 * u + 1], p[4 * u + 2], p[4 * u + 3]);
      }
    }
  }
  return true;
}

// ---------------------------------------------------------------------------
// Fused LayerNorm epilogue (kBiasResidLN) for the 2-CTA kernel run in clusters
// of P pairs that cover a whole row of N = 256 P columns.  The source page
// ("Faster Transformer 优化原理") runs add-bias + residual + LayerNorm as a
// separate kernel after the GEMM; here the GEMM writes the normalised row.
//   Pass 1: each epilogue warp forms z = acc + bias + residual for its 32 rows
//     x 128 columns (residual by TMA, two chunks ahead), writes z back
//     into the accumulator's TMEM columns and keeps per-row (mean, M2) of its
//     128 values, merged chunk by chunk with the pairwise update of Chan,
//     Golub and LeVeque (1979), which has no E[z^2] - E[z]^2 cancellation.
//   Exchange: the (mean, M2) halves go to shared memory; once the CTA's 8 warps
//     have written theirs, one thread arrives (release, cluster scope) on the
//     matching barrier of the CTA with the same rows in each other pair; each
//     CTA then reads the other pairs' halves through distributed shared
//     memory and merges all 2P of them in a fixed order.
//   Pass 2: out = (z - mean) * rsqrt(M2 / N + eps) * gamma + beta, from TMEM,
//     stored as FP16 through the staging buffers and TMA stores.
// The accumulator is released only after pass 2.  Releasing it after pass 1
// (z kept as FP16 in registers) was measured slower: the next tile's MMAs
// then run under the whole epilogue, and their operand traffic through
// shared memory slows every epilogue phase more than the overlap gains.
// The statistics are double-buffered by tile parity: a pair writes buffer b
// again only two tiles later, after every other pair has signalled the tile in
// between, i.e. after they have read buffer b.
// ---------------------------------------------------------------------------
struct LnCtx {
  float2* stats;          // [2 buffers][column slices][128 rows] (mean, M2)
  uint32_t local_bar;     // 8 epilogue warps of this CTA, one phase per tile
  uint32_t ready_bar0;    // + 8 * buffer: one arrival from each other pair
  int pairs;              // P
  int pair;               // this CTA's pair in the cluster
  int rir;                // this CTA's index in its pair (its 128 rows)
};

// Pairwise update (Chan, Golub and LeVeque 1979) of (count, mean, M2) with a
// group of nb values whose mean is mb and sum of squared deviations qb.
__device__ __forceinline__ void chan_merge(float& n, float& mean, float& m2, float nb, float mb, float qb) {
  const float nn = n + nb;
  const float d = mb - mean;
  mean = fmaf(d, nb / nn, mean);
  m2 = m2 + qb + d * d * (n * nb / nn);
  n = nn;
}

constexpr int kMaxLnPairs = 4;                 // clusters of up to 8 CTAs (N <= 1024)

template <typename WaitFull, typename Release>
__device__ __forceinline__ bool epilogue_ln_tile(uint32_t t_cols, int row0, int col_begin, int N,
                                                 const float* __restrict__ bias, const float* __restrict__ gamma,
                                                 const float* __restrict__ beta, float* par_s, const CUtensorMap* tm_c,
                                                 EpiWarpState& ws, const LnCtx& ln, int slice, int rloc,
                                                 bool signaller, uint32_t local, bool prefetch, int next_row0,
                                                 WaitFull wait_full, Release release) {
  constexpr int kCols = 256 / kEpiSlices;      // columns per warp (128 with 8 epilogue warps)
  constexpr int CHUNKS = kCols / 32;
  const int lane = threadIdx.x & 31;
  {
    const int i = lane * 4;                    // bias, gamma, beta of the warp's columns
    float4 b = make_float4(0.f, 0.f, 0.f, 0.f), g = b, t = b;
    if (i < kCols && col_begin + i < N) {
      b = __ldg(reinterpret_cast<const float4*>(bias + col_begin + i));
      g = __ldg(reinterpret_cast<const float4*>(gamma + col_begin + i));
      t = __ldg(reinterpret_cast<const float4*>(beta + col_begin + i));
    }
    if (i < kCols) {
      *reinterpret_cast<float4*>(par_s + i) = b;
      *reinterpret_cast<float4*>(par_s + kCols + i) = g;
      *reinterpret_cast<float4*>(par_s + 2 * kCols + i) = t;
    }
  }
  auto buf_of = [&](int j) { return ws.stage + ((ws.seq + j) & 1u) * kStageChunkBytes; };
  auto issue_res = [&](int j) {                // lane 0: residual chunk j into buffer (seq + j) & 1
    const uint32_t bar = ws.res_bar + 8u * ((ws.seq + j) & 1u);
    sm100::mbar_arrive_expect_tx(bar, kStageChunkBytes);
    sm100::tma_load_2d(ws.tm_r, sm100::smem_u32(buf_of(j)), bar, col_begin + 32 * j, row0);
  };
  // Residual chunks 0 and 1 before the accumulator is awaited (once the
  // previous tile's stores have read both buffers); chunk j + 2 once chunk j's
  // residual has been read out of its buffer.
  // With `prefetch`, the rest of this tile's residual (first tile) and the next
  // tile's (at row next_row0, if any) are requested into L2 now, so that the
  // loads of pass 1 find them there.
  if (lane == 0) {
    sm100::bulk_wait_group_read<0>();
    issue_res(0);
    issue_res(1);
    if (prefetch && local == 0)
      for (int j = 2; j < CHUNKS; ++j) sm100::tma_prefetch_2d_l2(ws.tm_r, col_begin + 32 * j, row0);
    if (prefetch && next_row0 >= 0)
      for (int j = 0; j < CHUNKS; ++j) sm100::tma_prefetch_2d_l2(ws.tm_r, col_begin + 32 * j, next_row0);
  }
  int got = 0;
  if (lane == 0) got = wait_full() ? 1 : 0;
  got = __shfl_sync(0xffffffffu, got, 0);      // also orders the parameter staging before its use
  if (!got) return false;
  sm100::tc_fence_after();

  // Pass 1.
  float n = 0.f, mean = 0.f, m2 = 0.f;
  uint32_t ra[32], rb[32];
  sm100::tmem_ld_32x32b_x32_async(t_cols, ra);
#pragma unroll
  for (int j = 0; j < CHUNKS; ++j) {
    uint32_t(&cur)[32] = (j & 1) ? rb : ra;
    uint32_t(&nxt)[32] = (j & 1) ? ra : rb;
    sm100::tmem_wait_ld(cur);
    if (j + 1 < CHUNKS) sm100::tmem_ld_32x32b_x32_async(t_cols + 32 * (j + 1), nxt);
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; i += 4) {          // bias: one 16-byte broadcast read per 4 columns
      const float4 b4 = *reinterpret_cast<const float4*>(par_s + 32 * j + i);
      v[i] = __uint_as_float(cur[i]) + b4.x;
      v[i + 1] = __uint_as_float(cur[i + 1]) + b4.y;
      v[i + 2] = __uint_as_float(cur[i + 2]) + b4.z;
      v[i + 3] = __uint_as_float(cur[i + 3]) + b4.w;
    }
    const uint32_t k = (ws.seq + j) & 1u;
    int ok = 0;
    if (lane == 0) ok = mbar_wait<kSleepNs>(ws.res_bar + 8u * k, (ws.res_phase >> k) & 1u, kWaitLimitNs) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok) return false;
    ws.res_phase ^= 1u << k;
    const uint8_t* buf = buf_of(j);
#pragma unroll
    for (int u = 0; u < 4; ++u) add_residual_unit(v, u, *reinterpret_cast<const uint4*>(buf + stage_unit(lane, u)));
    float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < 32; ++i) s4[i & 3] += v[i];
    const float mc = ((s4[0] + s4[1]) + (s4[2] + s4[3])) * (1.0f / 32.0f);
    float q4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float d = v[i] - mc;
      q4[i & 3] = fmaf(d, d, q4[i & 3]);
    }
    chan_merge(n, mean, m2, 32.0f, mc, (q4[0] + q4[1]) + (q4[2] + q4[3]));
    if (j + 2 < CHUNKS) {
      __syncwarp();                            // every lane has used the residual it read from the buffer
      if (lane == 0) issue_res(j + 2);
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) cur[i] = __float_as_uint(v[i]);
    sm100::tmem_st_32x32b_x32(t_cols + 32 * j, cur);     // z replaces the accumulator
  }

  // Exchange.
  const uint32_t b = local & 1u;
  ln.stats[(b * kEpiSlices + slice) * 128 + rloc] = make_float2(mean, m2);
  __syncwarp();
  int ok = 1;
  if (lane == 0) {
    mbar_arrive(ln.local_bar);
    ok = mbar_wait<kSleepNs>(ln.local_bar, local & 1u, kWaitLimitNs) ? 1 : 0;
    if (ok && signaller) {
      for (int p = 0; p < ln.pairs; ++p)
        if (p != ln.pair) mbar_arrive_remote_release(mapa_shared(ln.ready_bar0 + 8u * b, 2 * p + ln.rir));
    }
    if (ok && ln.pairs > 1)
      ok = mbar_wait_acquire_cluster<kSleepNs>(ln.ready_bar0 + 8u * b, (local >> 1) & 1u, kWaitLimitNs) ? 1 : 0;
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (!ok) return false;
  // Every pair's statistics of the row are requested before the first merge
  // (one remote-load latency); merged in pair order.
  float tn = 0.f, tmean = 0.f, tm2 = 0.f;
  const uint32_t st0 = sm100::smem_u32(ln.stats + (b * kEpiSlices) * 128 + rloc);
  float2 hs[kMaxLnPairs][kEpiSlices];
#pragma unroll
  for (int p = 0; p < kMaxLnPairs; ++p) {
    if (p < ln.pairs) {
#pragma unroll
      for (int hf = 0; hf < kEpiSlices; ++hf)
        hs[p][hf] = p == ln.pair ? ln.stats[(b * kEpiSlices + hf) * 128 + rloc]
                                 : ld_cluster_f2(mapa_shared(st0 + hf * 128 * 8, 2 * p + ln.rir));
    }
  }
#pragma unroll
  for (int p = 0; p < kMaxLnPairs; ++p) {
    if (p < ln.pairs) {
#pragma unroll
      for (int hf = 0; hf < kEpiSlices; ++hf) chan_merge(tn, tmean, tm2, (float)kCols, hs[p][hf].x, hs[p][hf].y);
    }
  }
  const float rstd = rsqrtf(tm2 / (float)N + kLnEps);

  // Pass 2.
  sm100::tmem_ld_32x32b_x32_async(t_cols, ra);
#pragma unroll
  for (int j = 0; j < CHUNKS; ++j) {
    uint32_t(&cur)[32] = (j & 1) ? rb : ra;
    uint32_t(&nxt)[32] = (j & 1) ? ra : rb;
    sm100::tmem_wait_ld(cur);
    if (j + 1 < CHUNKS) sm100::tmem_ld_32x32b_x32_async(t_cols + 32 * (j + 1), nxt);
    if (j + 1 == CHUNKS) {
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) release();
    }
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 32; i += 4) {          // gamma, beta: 16-byte broadcast reads
      const float4 g4 = *reinterpret_cast<const float4*>(par_s + kCols + 32 * j + i);
      const float4 t4 = *reinterpret_cast<const float4*>(par_s + 2 * kCols + 32 * j + i);
      const float o0 = fmaf((__uint_as_float(cur[i]) - tmean) * rstd, g4.x, t4.x);
      const float o1 = fmaf((__uint_as_float(cur[i + 1]) - tmean) * rstd, g4.y, t4.y);
      const float o2 = fmaf((__uint_as_float(cur[i + 2]) - tmean) * rstd, g4.z, t4.z);
      const float o3 = fmaf((__uint_as_float(cur[i + 3]) - tmean) * rstd, g4.w, t4.w);
      pk[i >> 1] = pack_half2(o0, o1);
      pk[(i >> 1) + 1] = pack_half2(o2, o3);
    }
    uint8_t* buf = buf_of(j);
    if (lane == 0) sm100::bulk_wait_group_read<1>();   // the store two chunks back has read buf
    __syncwarp();
#pragma unroll
    for (int u = 0; u < 4; ++u)
      *reinterpret_cast<uint4*>(buf + stage_unit(lane, u)) =
          make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
    sm100::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      sm100::tma_store_2d(tm_c, sm100::smem_u32(buf), col_begin + 32 * j, row0);
      sm100::bulk_commit_group();
    }
  }
  ws.seq += CHUNKS;
  return true;
}

template <int BN, Epi EPI>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                   const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_r,
                   int use_tma_store, int M_max, int N, int K,
                   const float* __restrict__ bias, __half* __restrict__ C, SplitShape sp, int* __restrict__ status,
                   const int* __restrict__ m_dev, const __half* __restrict__ resid) {
  using G = Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + G::kStages * G::kABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + G::kStages * G::kBBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + G::kNumBars);
  float* bias_smem = reinterpret_cast<float*>(smem + G::kBiasOffset);
  uint8_t* store_smem = smem + G::kStoreOffset;

  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (G::kStages + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * G::kStages + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * G::kStages + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * G::kStages + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < G::kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), kEpiWarps);
    }
    mbar_init(drain_bar, 1);
    for (int i = 0; i < 2 * kEpiWarps; ++i) mbar_init(bar0 + 8u * (G::kResBar0 + i), 1);
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), G::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int num_n = (N + BN - 1) / BN;
  const int num_kb = (K + kBK - 1) / kBK;
  // The weights do not depend on the previous kernel: with a fixed row count
  // (the grid's first tiles all exist) the producer requests the first stages'
  // weight tiles of its first tile before waiting for it.
  int pre = 0;
  if (!m_dev && warp == 0 && lane == 0) {
    pre = min(G::kStages, num_kb);
    const int n_blk = (int)blockIdx.x % num_n;
    for (int i = 0; i < pre; ++i) {
      mbar_arrive_expect_tx(full_bar(i), G::kStageBytes);
      tma_load_2d(&tm_b, smem_u32(sB + i * G::kBBytes), full_bar(i), i * kBK, n_blk * BN);
    }
  }
  pdl_wait();                                  // the previous kernel's writes (A, m_dev) are visible
  pdl_trigger();
  const int M = m_dev ? min(*m_dev, M_max) : M_max;
  const int num_m = (M + kBM - 1) / kBM;
  const int num_tiles = num_m * num_n;

  bool ok = true;
  if (warp == 0) {
    if (lane == 0) {
      uint32_t it = 0;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int m_blk = tile / num_n;
        const int n_blk = tile - m_blk * num_n;
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const int s = it % G::kStages;
          const uint32_t ph = (it / G::kStages) & 1u;
          if ((int)it < pre) {                   // the weight tile is already on its way
            tma_load_2d(&tm_a, smem_u32(sA + s * G::kABytes), full_bar(s), kb * kBK, m_blk * kBM);
            continue;
          }
          if (!mbar_wait<kSleepNs>(empty_bar(s), ph ^ 1u, kWaitLimitNs)) { ok = false; break; }
          mbar_arrive_expect_tx(full_bar(s), G::kStageBytes);
          tma_load_2d(&tm_a, smem_u32(sA + s * G::kABytes), full_bar(s), kb * kBK, m_blk * kBM);
          tma_load_2d(&tm_b, smem_u32(sB + s * G::kBBytes), full_bar(s), kb * kBK, n_blk * BN);
        }
      }
      // Let every copy this thread issued land before the CTA can exit.
      const uint32_t first = it > (uint32_t)G::kStages ? it - G::kStages : 0u;
      for (uint32_t j = first; j < it; ++j)
        mbar_wait<kSleepNs>(full_bar(j % G::kStages), (j / G::kStages) & 1u, kWaitLimitNs);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(kBM, BN);
      uint32_t it = 0, local = 0;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++local) {
        const uint32_t acc = local & 1u;
        const uint32_t aph = (local >> 1) & 1u;
        if (!mbar_wait<kSleepNs>(tempty_bar(acc), aph ^ 1u, kWaitLimitNs)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const int s = it % G::kStages;
          const uint32_t ph = (it / G::kStages) & 1u;
          if (!mbar_wait<kSleepNs>(full_bar(s), ph, kWaitLimitNs)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + s * G::kABytes);
          const uint32_t b_addr = smem_u32(sB + s * G::kBBytes);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            mma_f16_ss(d_tmem, smem_desc_sw128(a_addr + kk * 32), smem_desc_sw128(b_addr + kk * 32),
                       idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(empty_bar(s));
        }
        if (!ok) break;
        mma_commit(tfull_bar(acc));
      }
      // Every MMA this thread issued has completed once drain_bar flips.
      mma_commit(drain_bar);
      mbar_wait<kSleepNs>(drain_bar, 0, kWaitLimitNs);
    }
  } else {
    const int quad = warp & 3;                 // TMEM lanes 32*quad .. 32*quad+31
    const int slice = (warp - 2) >> 2;         // which column slice of the tile
    constexpr int kCols = BN / kEpiSlices;
    constexpr int kChunks = kCols / 32;        // 32-column chunks per warp
    float* bias_s = bias_smem + (warp - 2) * kCols;
    const CUtensorMap* tmc = (use_tma_store & 1) ? &tm_c : nullptr;
    EpiWarpState ws;
    ws.stage = store_smem + (warp - 2) * 2 * kStageChunkBytes;
    ws.tm_r = (use_tma_store & 2) ? &tm_r : nullptr;     // residual through TMA (kBiasResidStore)
    ws.res_bar = bar0 + 8u * (G::kResBar0 + 2 * (warp - 2));
    uint32_t local = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
      const int m_blk = tile / num_n;
      const int n_blk = tile - m_blk * num_n;
      const uint32_t acc = local & 1u;
      const uint32_t aph = (local >> 1) & 1u;
      const uint32_t t_cols = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * BN + slice * kCols;
      const int row0 = m_blk * kBM + quad * 32;
      const bool got = epilogue_warp_tile<EPI, kChunks>(
          t_cols, row0, n_blk * BN + slice * kCols, M, N, bias, bias_s, C, sp, tmc, ws, resid,
          [&] { return mbar_wait<kSleepNs>(tfull_bar(acc), aph, kWaitLimitNs); },
          [&] { mbar_arrive(tempty_bar(acc)); });
      if (!got) { ok = false; break; }
    }
    if (lane == 0) bulk_wait_group_all();      // every TMA store of this warp has completed
    __syncwarp();
  }

  if (!ok) atomicCAS(status, 0, kStatusWaitTimeout);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, G::kTmemCols);
  }
}


// ---------------------------------------------------------------------------
// 2-CTA variant: a cluster of two CTAs computes a 256x256 tile with
// tcgen05.mma.cta_group::2 (M = 256, N = 256).  CTA r holds rows
// [128r, 128r+128) of the A tile and rows [128r, 128r+128) of the B tile
// in its own shared memory, at the same offsets in both CTAs, and receives
// rows [128r, 128r+128) of the accumulator in its TMEM.  Per SM and k-block
// that is 32 KB of operands for 4.2 MFLOP (128 flop/byte) instead of 48 KB for
// the same work with a 128x256 one-CTA tile, which is what keeps the L2->SM
// traffic below what the tensor cores consume.
//   - Both CTAs' producers load their halves; the transaction bytes of both
//     complete on the leader CTA's full barrier (count 2).
//   - The leader's single MMA thread issues the MMAs and commits to the
//     empty / accumulator-full barriers of both CTAs at once.
//   - Both CTAs' epilogue warps release an accumulator on the leader's
//     accumulator-empty barrier (count 2 x kEpiWarps).
// ---------------------------------------------------------------------------
// The bias + residual epilogue (output projection, FFN2 without the fused
// LayerNorm) keeps four staging buffers per warp instead of two, so that the
// residual of all four of a warp's 32-column chunks is fetched while the
// tile's MMAs run; one operand stage fewer pays for them.
template <Epi EPI>
struct PairCfgT {
  static constexpr bool kResAll = EPI == Epi::kBiasResidStore;
  static constexpr int kStoreBufs = kResAll ? 4 : 2;          // staging buffers per epilogue warp
  static constexpr int kStages = kResAll ? 4 : 5;
  static constexpr int kABytes = 128 * kBK * 2;
  static constexpr int kBBytes = 128 * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = 512;             // two 256-column accumulators
  static constexpr int kResBar0 = 2 * kStages + 5;
  static constexpr int kLnBar0 = kResBar0 + kStoreBufs * kEpiWarps;   // LayerNorm: local, ready[2]
  static constexpr int kNumBars = kLnBar0 + 3;
  static constexpr int kBiasOffset = (kStages * kStageBytes + kNumBars * 8 + 16 + 15) / 16 * 16;
  // Per epilogue warp: bias (and, for the fused LayerNorm, gamma and beta) of its columns.
  static constexpr int kParamFloats = 3 * (256 / kEpiSlices);
  static constexpr int kStatsOffset = (kBiasOffset + kEpiWarps * kParamFloats * 4 + 15) / 16 * 16;
  static constexpr int kStatsBytes = 2 * kEpiSlices * 128 * 8;   // LayerNorm statistics, [2][slices][128] float2
  static constexpr int kStoreOffset = (kStatsOffset + kStatsBytes + 1023) / 1024 * 1024;
  static constexpr int kSmem = 1024 + kStoreOffset + kEpiWarps * kStoreBufs * (32 * 32 * 2);
  static_assert(kSmem <= 227 * 1024, "dynamic shared memory of one CTA");
};

// CL = CTAs per cluster: 2 (one pair) for every epilogue but the fused
// LayerNorm, which runs N / 128 CTAs (N / 256 pairs) per cluster, one pair
// per 256-column block of the same 256 rows.  The pair of CTA rank r is
// {r & ~1, r | 1}; its leader is r & ~1.
template <Epi EPI, int CL>
__global__ void __cluster_dims__(CL, 1, 1) __launch_bounds__(kThreads, 1)
    gemm_tc_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                        const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_r,
                        int use_tma_store, int M_max, int N, int K,
                        const float* __restrict__ bias, __half* __restrict__ C, SplitShape sp,
                        int* __restrict__ status, const int* __restrict__ m_dev, const __half* __restrict__ resid,
                        const float* __restrict__ ln_gamma, const float* __restrict__ ln_beta) {
  constexpr bool kLn = EPI == Epi::kBiasResidLN;
  using G = PairCfgT<EPI>;
  constexpr int BN = 256;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + G::kStages * G::kABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + G::kStages * G::kBBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + G::kNumBars);
  float* bias_smem = reinterpret_cast<float*>(smem + G::kBiasOffset);
  uint8_t* store_smem = smem + G::kStoreOffset;

  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (G::kStages + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * G::kStages + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * G::kStages + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * G::kStages + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t rir = rank & 1u;                 // CTA within its pair: rows [128 rir, 128 rir + 128)
  const uint32_t lead = rank & ~1u;               // the pair's leader (issues the MMAs)
  const uint16_t pair_mask = static_cast<uint16_t>(3u << lead);
  const int pic = static_cast<int>(rank >> 1);    // pair within the cluster (column block, fused LayerNorm)
  const int cluster = blockIdx.x / CL;
  const int num_clusters = gridDim.x / CL;

  if (threadIdx.x == 0) {
    for (int s = 0; s < G::kStages; ++s) {
      mbar_init(full_bar(s), 2);              // both CTAs' producers arrive (leader's copy is used)
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 2 * kEpiWarps);
    }
    mbar_init(drain_bar, 1);
    for (int i = 0; i < G::kStoreBufs * kEpiWarps; ++i) mbar_init(bar0 + 8u * (G::kResBar0 + i), 1);
    mbar_init(bar0 + 8u * G::kLnBar0, kEpiWarps);
    for (int i = 1; i <= 2; ++i) mbar_init(bar0 + 8u * (G::kLnBar0 + i), CL > 2 ? CL / 2 - 1 : 1);
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), G::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync();                               // barriers of both CTAs are initialised
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int num_n = (N + BN - 1) / BN;
  const int num_kb = (K + kBK - 1) / kBK;
  // The weights do not depend on the previous kernel: with a fixed row count
  // (the grid's first work items all exist) each CTA's producer requests the
  // first stages' weight halves of its first work item before waiting for it.
  int pre = 0;
  if (!m_dev && warp == 0 && lane == 0) {
    pre = min(G::kStages, num_kb);
    const int n_blk = kLn ? pic : cluster % num_n;
    for (int i = 0; i < pre; ++i) {
      const uint32_t leader_full = mapa_shared(full_bar(i), lead);
      mbar_arrive_expect_tx_cluster(leader_full, G::kStageBytes);
      tma_load_2d_pair(&tm_b, smem_u32(sB + i * G::kBBytes), leader_full, i * kBK, n_blk * BN + (int)rir * 128);
    }
  }
  pdl_wait();                                   // the previous kernel's writes (A, m_dev) are visible
  pdl_trigger();
  const int M = m_dev ? min(*m_dev, M_max) : M_max;
  const int num_m = (M + 255) / 256;
  // Work items walked by each cluster: 256x256 tiles, or (fused LayerNorm)
  // 256-row blocks whose column block is the pair's index in the cluster.
  const int num_work = kLn ? num_m : num_m * num_n;
  auto work_tile = [&](int w, int& m_blk, int& n_blk) {
    if (kLn) {
      m_blk = w;
      n_blk = pic;
    } else {
      m_blk = w / num_n;
      n_blk = w - m_blk * num_n;
    }
  };

  bool ok = true;
  uint32_t issued = 0;
  if (warp == 0) {
    if (lane == 0) {
      for (int w = cluster; w < num_work && ok; w += num_clusters) {
        int m_blk, n_blk;
        work_tile(w, m_blk, n_blk);
        const int a_row = m_blk * 256 + (int)rir * 128;
        const int b_row = n_blk * BN + (int)rir * 128;
        for (int kb = 0; kb < num_kb; ++kb, ++issued) {
          const int s = issued % G::kStages;
          const uint32_t ph = (issued / G::kStages) & 1u;
          if ((int)issued < pre) {               // the weight half is already on its way
            tma_load_2d_pair(&tm_a, smem_u32(sA + s * G::kABytes), mapa_shared(full_bar(s), lead), kb * kBK, a_row);
            continue;
          }
          if (!mbar_wait<kSleepNs>(empty_bar(s), ph ^ 1u, kWaitLimitNs)) { ok = false; break; }
          const uint32_t leader_full = mapa_shared(full_bar(s), lead);
          mbar_arrive_expect_tx_cluster(leader_full, G::kStageBytes);
          tma_load_2d_pair(&tm_a, smem_u32(sA + s * G::kABytes), leader_full, kb * kBK, a_row);
          tma_load_2d_pair(&tm_b, smem_u32(sB + s * G::kBBytes), leader_full, kb * kBK, b_row);
        }
      }
      if (rir == 0) {
        // Every copy of both CTAs counted on the leader's full barriers has landed.
        const uint32_t first = issued > (uint32_t)G::kStages ? issued - G::kStages : 0u;
        for (uint32_t j = first; j < issued; ++j)
          mbar_wait<kSleepNs>(full_bar(j % G::kStages), (j / G::kStages) & 1u, kWaitLimitNs);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rir == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(256, BN);
      uint32_t it = 0, local = 0;
      for (int w = cluster; w < num_work && ok; w += num_clusters, ++local) {
        const uint32_t acc = local & 1u;
        const uint32_t aph = (local >> 1) & 1u;
        if (!mbar_wait<kSleepNs>(tempty_bar(acc), aph ^ 1u, kWaitLimitNs)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const int s = it % G::kStages;
          const uint32_t ph = (it / G::kStages) & 1u;
          if (!mbar_wait<kSleepNs>(full_bar(s), ph, kWaitLimitNs)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + s * G::kABytes);
          const uint32_t b_addr = smem_u32(sB + s * G::kBBytes);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            mma_f16_ss_pair(d_tmem, smem_desc_sw128(a_addr + kk * 32), smem_desc_sw128(b_addr + kk * 32), idesc,
                            (kb > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit_pair(empty_bar(s), pair_mask);
        }
        if (!ok) break;
        mma_commit_pair(tfull_bar(acc), pair_mask);
      }
      mma_commit_pair(drain_bar, pair_mask);
    }
    if (lane == 0) mbar_wait<kSleepNs>(drain_bar, 0, kWaitLimitNs);   // the leader's MMAs are done
    __syncwarp();
  } else {
    const int quad = warp & 3;
    const int slice = (warp - 2) >> 2;
    constexpr int kCols = BN / kEpiSlices;
    constexpr int kChunks = kCols / 32;
    float* bias_s = bias_smem + (warp - 2) * kCols;
    const CUtensorMap* tmc = (use_tma_store & 1) ? &tm_c : nullptr;
    EpiWarpState ws;
    ws.stage = store_smem + (warp - 2) * G::kStoreBufs * kStageChunkBytes;
    ws.tm_r = (use_tma_store & 2) ? &tm_r : nullptr;     // residual through TMA (kBiasResidStore)
    ws.res_bar = bar0 + 8u * (G::kResBar0 + G::kStoreBufs * (warp - 2));
    const uint32_t leader_tempty0 = mapa_shared(tempty_bar(0), lead);
    const uint32_t leader_tempty1 = mapa_shared(tempty_bar(1), lead);
    LnCtx ln;
    ln.stats = reinterpret_cast<float2*>(smem + G::kStatsOffset);
    ln.local_bar = bar0 + 8u * G::kLnBar0;
    ln.ready_bar0 = bar0 + 8u * (G::kLnBar0 + 1);
    ln.pairs = CL / 2;
    ln.pair = pic;
    ln.rir = static_cast<int>(rir);
    float* par_s = reinterpret_cast<float*>(smem + G::kBiasOffset) + (warp - 2) * G::kParamFloats;
    uint32_t local = 0;
    for (int w = cluster; w < num_work; w += num_clusters, ++local) {
      int m_blk, n_blk;
      work_tile(w, m_blk, n_blk);
      const uint32_t acc = local & 1u;
      const uint32_t aph = (local >> 1) & 1u;
      const uint32_t t_cols = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * BN + slice * kCols;
      const int row0 = m_blk * 256 + (int)rir * 128 + quad * 32;
      auto wait_full = [&] { return mbar_wait<kSleepNs>(tfull_bar(acc), aph, kWaitLimitNs); };
      auto release = [&] { mbar_arrive_cluster(acc ? leader_tempty1 : leader_tempty0); };
      bool got;
      if constexpr (kLn) {
        // Residual prefetch into L2 where the epilogue outlasts the main loop
        // (K <= 1024, the output projection); with FFN2's K = F it measured slower.
        const bool prefetch = K <= 1024;
        const int next_row0 = w + num_clusters < num_work ? row0 + num_clusters * 256 : -1;
        got = epilogue_ln_tile(t_cols, row0, n_blk * BN + slice * kCols, N, bias, ln_gamma, ln_beta, par_s, tmc,
                               ws, ln, slice, quad * 32 + lane, warp == 2, local, prefetch, next_row0, wait_full,
                               release);
      } else {
        got = epilogue_warp_tile<EPI, kChunks, G::kStoreBufs>(t_cols, row0, n_blk * BN + slice * kCols, M, N, bias,
                                                              bias_s, C, sp, tmc, ws, resid, wait_full, release);
      }
      if (!got) { ok = false; break; }
    }
    if (lane == 0) bulk_wait_group_all();      // every TMA store of this warp has completed
    __syncwarp();
  }

  if (!ok) atomicCAS(status, 0, kStatusWaitTimeout);
  tc_fence_before();
  __syncwarp();
  cluster_sync();                               // no CTA leaves while its peer may still signal it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, G::kTmemCols);
  }
}

// Epilogue store flags: bit 0 = TMA stores through tmap_c, bit 1 = residual
// tiles through tmap_r (only with TMA stores).
int store_flags(const TcGemmArgs& a) { return (a.tmap_c ? 1 : 0) | (a.tmap_c && a.tmap_r ? 2 : 0); }

// Clusters of CL CTAs of this kernel that fit on the GPU at once (a persistent
// grid larger than that would run its last clusters as a second wave).
template <Epi EPI, int CL>
int pair_max_clusters(cudaError_t& err) {
  using G = PairCfgT<EPI>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  static int max_clusters = 0;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(gemm_tc_pair_kernel<EPI, CL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    G::kSmem);
    if (attr_err != cudaSuccess) return;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(CL * 256, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = G::kSmem;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = CL;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    attr_err = cudaOccupancyMaxActiveClusters(&max_clusters, gemm_tc_pair_kernel<EPI, CL>, &cfg);
  });
  err = attr_err;
  return max_clusters;
}

template <Epi EPI, int CL>
cudaError_t launch_pair(const TcGemmArgs& a, cudaStream_t stream) {
  using G = PairCfgT<EPI>;
  cudaError_t err;
  const int max_clusters = pair_max_clusters<EPI, CL>(err);
  if (err != cudaSuccess) return err;
  if (max_clusters <= 0) return cudaErrorInvalidConfiguration;
  const int num_m = (a.M + 255) / 256;
  const int work = EPI == Epi::kBiasResidLN ? num_m : num_m * ((a.N + 255) / 256);
  const int clusters = work < max_clusters ? work : max_clusters;
  return launch_kernel(gemm_tc_pair_kernel<EPI, CL>, dim3(CL * clusters), dim3(kThreads), G::kSmem, stream, nullptr,
                       0, *a.tmap_a, *a.tmap_b, a.tmap_c ? *a.tmap_c : *a.tmap_a, a.tmap_r ? *a.tmap_r : *a.tmap_a,
                       store_flags(a), a.M, a.N, a.K, a.bias, a.c, a.split, a.status, a.m_dev, a.resid, a.ln_gamma,
                       a.ln_beta);
}

// ---------------------------------------------------------------------------
// Split-K variant for small M, where 128x128 tiles alone would leave most SMs
// idle while a few stream all of the weights.  A cluster of `splits` CTAs
// (one per SM) shares each tile; CTA r (its rank in the cluster) accumulates
// the r-th balanced range of the k-blocks in TMEM:
//   warp 0      TMA producer (4-stage ring of 128x64 A and B tiles)
//   warp 1      TMEM owner and MMA issuer (M=128, N=128, K=16)
//   warps 2..9  copy the FP32 partial tile from TMEM to this CTA's shared
//               memory; after a cluster barrier each CTA reduces its band of
//               128/splits rows over all CTAs' partials through distributed
//               shared memory, in rank order (so the sum does not depend on
//               timing), applies the epilogue and stores FP16.
// Nothing goes through global memory but the operands and the result.
// ---------------------------------------------------------------------------
struct SplitCfg {
  static constexpr int kBN = 128;
  static constexpr int kStages = 4;
  static constexpr int kABytes = kBM * kBK * 2;
  static constexpr int kBBytes = kBN * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kPartOffset = kStages * kStageBytes;      // FP32 partial, 128 rows x 512 bytes
  static constexpr int kPartBytes = kBM * kBN * 4;
  static constexpr int kBarOffset = kPartOffset + kPartBytes;
  static constexpr int kNumBars = 2 * kStages + 2;                // full, empty, tfull, drain
  static constexpr int kSmem = 1024 + kBarOffset + kNumBars * 8 + 16;
  static constexpr int kTmemCols = 128;
  static constexpr int kMaxSplits = 16;
};

// Byte offset of float4 unit u (0..31) of partial row r: units swizzled by r
// so that a warp writing 32 rows (one unit each) and a warp reading one row
// (all 32 units) both spread over the banks.
__device__ __forceinline__ uint32_t part_offset(int r, int u) {
  return SplitCfg::kPartOffset + r * 512 + 16 * (u ^ (r & 31));
}

// Bias `b`, residual `u` (4 halves) and the epilogue's element-wise function
// on 4 consecutive columns of a row; both operands were loaded by the caller
// ahead of the partial sums they are added to.
template <Epi EPI>
__device__ __forceinline__ void epilogue4(float (&v)[4], const float4& b, const uint2& u) {
  if constexpr (EPI != Epi::kStore) {
    v[0] += b.x; v[1] += b.y; v[2] += b.z; v[3] += b.w;
  }
  if constexpr (EPI == Epi::kBiasResidStore) {
    const float2 lo = __half22float2(*reinterpret_cast<const __half2*>(&u.x));
    const float2 hi = __half22float2(*reinterpret_cast<const __half2*>(&u.y));
    v[0] += lo.x; v[1] += lo.y; v[2] += hi.x; v[3] += hi.y;
  }
  if constexpr (EPI == Epi::kBiasGelu) {
    act::gelu_erf_pair(v[0], v[1]);
    act::gelu_erf_pair(v[2], v[3]);
  }
  if constexpr (EPI == Epi::kBiasGeluTanh) {
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = act::gelu_tanh(v[i]);
  }
}

template <Epi EPI>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_splitk_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                          int M_max, int N, int K, const float* __restrict__ bias, __half* __restrict__ C,
                          SplitShape sp, int* __restrict__ status, const int* __restrict__ m_dev, int splits,
                          const __half* __restrict__ resid) {
  using G = SplitCfg;
  const int num_n = (N + G::kBN - 1) / G::kBN;
  const int tile = blockIdx.x / splits;
  const int ks = static_cast<int>(cluster_ctarank());
  const int m_blk = tile / num_n;
  const int n_blk = tile - m_blk * num_n;
  const int num_kb = (K + kBK - 1) / kBK;
  const int kb0 = ks * num_kb / splits;
  const int kb1 = (ks + 1) * num_kb / splits;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + G::kBarOffset);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + G::kNumBars);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (G::kStages + s); };
  const uint32_t tfull_bar = bar0 + 8u * (2 * G::kStages);
  const uint32_t drain_bar = bar0 + 8u * (2 * G::kStages + 1);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < G::kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(tfull_bar, 1);
    mbar_init(drain_bar, 1);
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), G::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The weights do not depend on the previous kernel: with a fixed row count
  // (no device count, so no tile of this grid can turn out empty) the producer
  // requests the first stages' weight tiles before waiting for it, so that
  // their latency overlaps its tail.
  int pre = 0;
  if (!m_dev && warp == 0 && lane == 0) {
    pre = min(G::kStages, kb1 - kb0);
    for (int i = 0; i < pre; ++i) {
      mbar_arrive_expect_tx(full_bar(i), G::kStageBytes);
      tma_load_2d(&tm_b, sbase + i * G::kStageBytes + G::kABytes, full_bar(i), (kb0 + i) * kBK, n_blk * G::kBN);
    }
  }
  pdl_wait();                                 // the previous kernel's writes (A, m_dev) are visible
  pdl_trigger();
  const int M = m_dev ? min(*m_dev, M_max) : M_max;
  if (m_blk * kBM >= M) {                     // a tile past the device row count: the whole cluster leaves
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc(tmem, G::kTmemCols);
    }
    return;
  }

  bool ok = true;
  float4 b4 = make_float4(0.f, 0.f, 0.f, 0.f);
  if (warp == 0) {
    if (lane == 0) {
      uint32_t it = 0;
      for (int kb = kb0; kb < kb1; ++kb, ++it) {
        const int s = it % G::kStages;
        const uint32_t ph = (it / G::kStages) & 1u;
        if ((int)it < pre) {                  // the weight tile is already on its way
          tma_load_2d(&tm_a, sbase + s * G::kStageBytes, full_bar(s), kb * kBK, m_blk * kBM);
          continue;
        }
        if (!mbar_wait<kSleepNs>(empty_bar(s), ph ^ 1u, kWaitLimitNs)) { ok = false; break; }
        mbar_arrive_expect_tx(full_bar(s), G::kStageBytes);
        tma_load_2d(&tm_a, sbase + s * G::kStageBytes, full_bar(s), kb * kBK, m_blk * kBM);
        tma_load_2d(&tm_b, sbase + s * G::kStageBytes + G::kABytes, full_bar(s), kb * kBK, n_blk * G::kBN);
      }
      const uint32_t first = it > (uint32_t)G::kStages ? it - G::kStages : 0u;
      for (uint32_t j = first; j < it; ++j)
        mbar_wait<kSleepNs>(full_bar(j % G::kStages), (j / G::kStages) & 1u, kWaitLimitNs);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(kBM, G::kBN);
      uint32_t it = 0;
      for (int kb = kb0; kb < kb1; ++kb, ++it) {
        const int s = it % G::kStages;
        const uint32_t ph = (it / G::kStages) & 1u;
        if (!mbar_wait<kSleepNs>(full_bar(s), ph, kWaitLimitNs)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_addr = sbase + s * G::kStageBytes;
        const uint32_t b_addr = a_addr + G::kABytes;
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk)
          mma_f16_ss(tmem, smem_desc_sw128(a_addr + kk * 32), smem_desc_sw128(b_addr + kk * 32), idesc,
                     (kb > kb0 || kk > 0) ? 1u : 0u);
        mma_commit(empty_bar(s));
      }
      if (ok) mma_commit(tfull_bar);
      mma_commit(drain_bar);
      mbar_wait<kSleepNs>(drain_bar, 0, kWaitLimitNs);
    }
  } else {
    // The bias of this thread's reduction columns, before the accumulator is awaited.
    const int col = n_blk * G::kBN + 4 * lane;
    if constexpr (EPI != Epi::kStore)
      if (col < N) b4 = __ldg(reinterpret_cast<const float4*>(bias + col));
    // TMEM lanes of quadrant warp % 4; columns [64 * slice, 64 * slice + 64).
    const int quad = warp & 3;
    const int slice = (warp - 2) >> 2;
    const int r = quad * 32 + lane;
    int got = 0;
    if (lane == 0) got = mbar_wait<kSleepNs>(tfull_bar, 0, kWaitLimitNs) ? 1 : 0;
    got = __shfl_sync(0xffffffffu, got, 0);
    // Only rows that exist are reduced: a quadrant past them copies nothing.
    if (got && quad * 32 < M - m_blk * kBM) {
      tc_fence_after();
      uint32_t v[32];
#pragma unroll 1
      for (int j = 0; j < 2; ++j) {
        tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + slice * 64 + 32 * j, v);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          *reinterpret_cast<uint4*>(smem + part_offset(r, slice * 16 + 8 * j + q)) =
              make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
      }
    } else if (!got) {
      ok = false;
    }
  }
  __syncwarp();
  cluster_sync();                             // every CTA's partial is in its shared memory

  if (warp >= 2) {
    // Rows [row0, row1) of the tile, 8 rows per pass, one float4 column unit per
    // lane.  The tile's rows that exist (fewer than 128 in the last row block,
    // e.g. 32 at batch 1) are shared evenly by the cluster's CTAs: the cluster
    // waits for its slowest reducer at the barrier below.
    const int t = threadIdx.x - 64;
    const int u = t & 31;
    const int valid = min(M - m_blk * kBM, kBM);
    const int row0 = ks * valid / splits;
    const int row1 = (ks + 1) * valid / splits;
    const int col = n_blk * G::kBN + 4 * u;
    if (col < N) {
      for (int r = row0 + (t >> 5); r < row1; r += 8) {
        const int grow = m_blk * kBM + r;
        if (grow >= M) break;
        // The residual and every CTA's partial are requested before any is
        // used, so the row costs one remote-load latency, not one per split.
        uint2 ru = make_uint2(0u, 0u);
        if constexpr (EPI == Epi::kBiasResidStore) ru = *reinterpret_cast<const uint2*>(resid + (size_t)grow * N + col);
        const uint32_t off = sbase + part_offset(r, u);
        float4 p[G::kMaxSplits];
#pragma unroll
        for (int s = 0; s < G::kMaxSplits; ++s)
          if (s < splits) p[s] = ld_cluster_f4(mapa_shared(off, (uint32_t)s));
        float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int s = 0; s < G::kMaxSplits; ++s) {   // rank order: the same sum on every run
          if (s < splits) {
            a[0] += p[s].x; a[1] += p[s].y; a[2] += p[s].z; a[3] += p[s].w;
          }
        }
        epilogue4<EPI>(a, b4, ru);
        __half* dst = C + row_offset<EPI>(grow, N, sp) + col_offset<EPI>(col, sp);
        *reinterpret_cast<uint2*>(dst) = make_uint2(pack_half2(a[0], a[1]), pack_half2(a[2], a[3]));
      }
    }
  }
  __syncwarp();
  cluster_sync();                             // no CTA leaves while a peer may still read its partial

  if (!ok) atomicCAS(status, 0, kStatusWaitTimeout);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, G::kTmemCols);
  }
}

// Most clusters of `size` split-K CTAs resident at once (0 when none fit).
int splitk_max_clusters(int size) {
  static std::mutex mu;
  static int cache[16][SplitCfg::kMaxSplits + 1] = {};
  static bool done[16][SplitCfg::kMaxSplits + 1] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 16 || size < 1 || size > SplitCfg::kMaxSplits) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (!done[dev][size]) {
    auto kern = gemm_tc_splitk_kernel<Epi::kStore>;    // every epilogue has the same resources
    int n = 0;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SplitCfg::kSmem) == cudaSuccess &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(size * 64, 1, 1);
      cfg.blockDim = dim3(kThreads, 1, 1);
      cfg.dynamicSmemBytes = SplitCfg::kSmem;
      cudaLaunchAttribute attr;
      attr.id = cudaLaunchAttributeClusterDimension;
      attr.val.clusterDim.x = size;
      attr.val.clusterDim.y = 1;
      attr.val.clusterDim.z = 1;
      cfg.attrs = &attr;
      cfg.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) n = 0;
    }
    cudaGetLastError();
    cache[dev][size] = n;
    done[dev][size] = true;
  }
  return cache[dev][size];
}

template <Epi EPI>
cudaError_t launch_splitk(const TcGemmArgs& a, cudaStream_t stream) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(gemm_tc_splitk_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    SplitCfg::kSmem);
    if (attr_err == cudaSuccess)
      attr_err = cudaFuncSetAttribute(gemm_tc_splitk_kernel<EPI>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const int tiles = ((a.M + kBM - 1) / kBM) * ((a.N + SplitCfg::kBN - 1) / SplitCfg::kBN);
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = a.splits;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  return launch_kernel(gemm_tc_splitk_kernel<EPI>, dim3(tiles * a.splits), dim3(kThreads), SplitCfg::kSmem, stream,
                       &attr, 1, *a.tmap_a, *a.tmap_b, a.M, a.N, a.K, a.bias, a.c, a.split, a.status, a.m_dev,
                       a.splits, a.resid);
}

template <int BN, Epi EPI>
cudaError_t launch_impl(const TcGemmArgs& a, cudaStream_t stream) {
  using G = Cfg<BN>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(gemm_tc_kernel<BN, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    G::kSmem);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const int tiles = ((a.M + kBM - 1) / kBM) * ((a.N + BN - 1) / BN);
  const int grid = tiles < a.num_sms ? tiles : a.num_sms;
  return launch_kernel(gemm_tc_kernel<BN, EPI>, dim3(grid), dim3(kThreads), G::kSmem, stream, nullptr, 0, *a.tmap_a,
                       *a.tmap_b, a.tmap_c ? *a.tmap_c : *a.tmap_a, a.tmap_r ? *a.tmap_r : *a.tmap_a, store_flags(a),
                       a.M, a.N, a.K, a.bias, a.c, a.split, a.status, a.m_dev, a.resid);
}

template <int BN>
cudaError_t launch_bn(const TcGemmArgs& a, cudaStream_t stream) {
  switch (a.epi) {
    case Epi::kStore: return launch_impl<BN, Epi::kStore>(a, stream);
    case Epi::kBiasGelu: return launch_impl<BN, Epi::kBiasGelu>(a, stream);
    case Epi::kBiasQkvSplit: return launch_impl<BN, Epi::kBiasQkvSplit>(a, stream);
    case Epi::kBiasGeluTanh: return launch_impl<BN, Epi::kBiasGeluTanh>(a, stream);
    case Epi::kBiasStore: return launch_impl<BN, Epi::kBiasStore>(a, stream);
    case Epi::kBiasResidStore: return launch_impl<BN, Epi::kBiasResidStore>(a, stream);
  }
  return cudaErrorInvalidValue;
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

}  // namespace

bool encode_kmajor_fp16_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                            uint32_t box_rows) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_output_map_2d(CUtensorMap* map, void* base, uint64_t rows, uint64_t cols) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {32, 32};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

bool encode_output_map_split(CUtensorMap* map, void* base, const SplitShape& sp) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  const uint64_t d = sp.size_per_head, S = sp.seq, nh = sp.head_num, B = sp.batch;
  const cuuint64_t dims[5] = {d, S, nh, B, 3};
  const cuuint64_t strides[4] = {d * 2, S * d * 2, nh * S * d * 2, B * nh * S * d * 2};
  const cuuint32_t box[5] = {32, 32, 1, 1, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 5, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

bool gemm_ln_supported(int M, int N) { return M >= 256 && N % 256 == 0 && N <= 1024; }

bool gemm_ln_wave_efficiency(int M, int N, float& fused, float& unfused) {
  cudaError_t e_ln = cudaSuccess, e_pair = cudaSuccess;
  int ln_slots = 0;
  switch (N) {
    case 256: ln_slots = pair_max_clusters<Epi::kBiasResidLN, 2>(e_ln); break;
    case 512: ln_slots = pair_max_clusters<Epi::kBiasResidLN, 4>(e_ln); break;
    case 768: ln_slots = pair_max_clusters<Epi::kBiasResidLN, 6>(e_ln); break;
    case 1024: ln_slots = pair_max_clusters<Epi::kBiasResidLN, 8>(e_ln); break;
    default: return false;
  }
  const int pair_slots = pair_max_clusters<Epi::kBiasResidStore, 2>(e_pair);
  if (e_ln != cudaSuccess || e_pair != cudaSuccess || ln_slots <= 0 || pair_slots <= 0 || M <= 0) return false;
  auto eff = [](int work, int slots) {
    const int waves = (work + slots - 1) / slots;
    return static_cast<float>(work) / static_cast<float>(waves * slots);
  };
  const int num_m = (M + 255) / 256;
  fused = eff(num_m, ln_slots);
  unfused = eff(num_m * (N / 256), pair_slots);
  return true;
}

int choose_gemm_splits(int tiles, int num_kb, int num_sms) {
  if (tiles <= 0) return 1;
  for (int s = std::min(SplitCfg::kMaxSplits, num_kb); s >= 2; --s)
    if ((long)tiles * s <= num_sms && tiles <= splitk_max_clusters(s)) return s;
  return 1;
}

cudaError_t launch_gemm_tc(const TcGemmArgs& a, cudaStream_t stream) {
  if (a.M <= 0 || a.N <= 0 || a.K <= 0 || (a.N % 8) != 0 || (a.K % 8) != 0) return cudaErrorInvalidValue;
  if (a.epi == Epi::kBiasQkvSplit && (a.split.size_per_head % 32) != 0) return cudaErrorInvalidValue;
  if (a.epi == Epi::kBiasResidStore && !a.resid) return cudaErrorInvalidValue;
  // The head-split store map needs every 32-row chunk inside one sequence.
  if (a.epi == Epi::kBiasQkvSplit && a.tmap_c && (a.split.seq % 32) != 0) return cudaErrorInvalidValue;
  if (a.splits > 1) {
    // every CTA of a cluster needs at least one k-block
    if (a.bn != 128 || a.splits > SplitCfg::kMaxSplits || a.splits > (a.K + kBK - 1) / kBK)
      return cudaErrorInvalidValue;
    switch (a.epi) {
      case Epi::kStore: return launch_splitk<Epi::kStore>(a, stream);
      case Epi::kBiasGelu: return launch_splitk<Epi::kBiasGelu>(a, stream);
      case Epi::kBiasQkvSplit: return launch_splitk<Epi::kBiasQkvSplit>(a, stream);
      case Epi::kBiasGeluTanh: return launch_splitk<Epi::kBiasGeluTanh>(a, stream);
      case Epi::kBiasStore: return launch_splitk<Epi::kBiasStore>(a, stream);
      case Epi::kBiasResidStore: return launch_splitk<Epi::kBiasResidStore>(a, stream);
    }
    return cudaErrorInvalidValue;
  }
  if (a.bn == kPairTile) {
    if ((a.N % 256) != 0) return cudaErrorInvalidValue;
    switch (a.epi) {
      case Epi::kStore: return launch_pair<Epi::kStore, 2>(a, stream);
      case Epi::kBiasGelu: return launch_pair<Epi::kBiasGelu, 2>(a, stream);
      case Epi::kBiasQkvSplit: return launch_pair<Epi::kBiasQkvSplit, 2>(a, stream);
      case Epi::kBiasGeluTanh: return launch_pair<Epi::kBiasGeluTanh, 2>(a, stream);
      case Epi::kBiasStore: return launch_pair<Epi::kBiasStore, 2>(a, stream);
      case Epi::kBiasResidStore: return launch_pair<Epi::kBiasResidStore, 2>(a, stream);
      case Epi::kBiasResidLN:
        // one cluster of N/128 CTAs per 256-row block; residual and output through TMA
        if (!a.tmap_c || !a.tmap_r || !a.ln_gamma || !a.ln_beta) return cudaErrorInvalidValue;
        switch (a.N) {
          case 256: return launch_pair<Epi::kBiasResidLN, 2>(a, stream);
          case 512: return launch_pair<Epi::kBiasResidLN, 4>(a, stream);
          case 768: return launch_pair<Epi::kBiasResidLN, 6>(a, stream);
          case 1024: return launch_pair<Epi::kBiasResidLN, 8>(a, stream);
        }
        return cudaErrorInvalidValue;
    }
    return cudaErrorInvalidValue;
  }
  if (a.bn == 256) return launch_bn<256>(a, stream);
  if (a.bn == 128) return launch_bn<128>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace enc
