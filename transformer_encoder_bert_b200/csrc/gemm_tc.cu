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
//               head split, 16-byte stores to global memory.
// The two accumulators let the epilogue of tile i overlap the MMAs of tile
// i+1.  Every mbarrier wait is bounded (kWaitLimitNs); a wait that gives up
// records kStatusWaitTimeout in the status word and the CTA drains its copies
// and MMAs, frees TMEM and exits.
#include <cstdio>
#include <cstdlib>
#include <mutex>

#include <cudaTypedefs.h>

#include "internal.h"
#include "sm100.cuh"

namespace enc {
namespace {

using namespace sm100;

constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s
constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;

template <int BN>
struct Cfg {
  static constexpr int kStages = BN == 256 ? 4 : 6;
  static constexpr int kABytes = kBM * kBK * 2;
  static constexpr int kBBytes = BN * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = 2 * BN;
  static constexpr int kNumBars = 2 * kStages + 5;
  static constexpr int kBiasOffset = (kStages * kStageBytes + kNumBars * 8 + 16 + 15) / 16 * 16;
  static constexpr int kSmem = 1024 + kBiasOffset + kEpiWarps * (BN / 2) * 4;
};

// GELU(v) = v * Phi(v) = 0.5 v (1 + erf(v / sqrt 2)), with erf from the rational
// approximation of Hastings (Abramowitz & Stegun, Handbook of Mathematical
// Functions, formula 7.1.26): for z >= 0,
//   erf(z) = 1 - (a1 t + a2 t^2 + a3 t^3 + a4 t^4 + a5 t^5) exp(-z^2),  t = 1/(1 + p z),
// |error| <= 1.5e-7, and erf(-z) = -erf(z).  One reciprocal and one exponential
// per element keep the epilogue of the FFN1 GEMM off the critical path; the
// error is far below the FP16 rounding of the stored result.
__device__ __forceinline__ float gelu_erf(float v) {
  const float z = fabsf(v) * 0.70710678118654752f;
  const float t = __fdividef(1.0f, fmaf(0.3275911f, z, 1.0f));
  float poly = fmaf(t, 1.061405429f, -1.453152027f);
  poly = fmaf(t, poly, 1.421413741f);
  poly = fmaf(t, poly, -0.284496736f);
  poly = fmaf(t, poly, 0.254829592f);
  poly *= t;
  const float erf_abs = fmaf(-poly, __expf(-z * z), 1.0f);
  return 0.5f * v * (1.0f + copysignf(erf_abs, v));
}

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

// Epilogue for one thread: 32 accumulator columns of one row.  `bias_s` holds
// the bias of these 32 columns (shared memory, read as a broadcast).
template <Epi EPI>
__device__ __forceinline__ void store_chunk(const uint32_t (&r)[32], bool row_ok, int col0, int N,
                                            const float* bias_s, __half* __restrict__ dst) {
  if (!row_ok) return;
  float v[32];
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
    for (int i = 0; i < 32; ++i) v[i] = gelu_erf(v[i]);
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    if (col0 + 8 * j < N) {
      uint4 w;
      w.x = pack_half2(v[8 * j + 0], v[8 * j + 1]);
      w.y = pack_half2(v[8 * j + 2], v[8 * j + 3]);
      w.z = pack_half2(v[8 * j + 4], v[8 * j + 5]);
      w.w = pack_half2(v[8 * j + 6], v[8 * j + 7]);
      *reinterpret_cast<uint4*>(dst + 8 * j) = w;
    }
  }
}

// One epilogue warp's share of a tile: rows [32*quad, 32*quad+32) of the
// accumulator (one row per lane), global columns [col_begin, col_begin +
// 32*CHUNKS), whose first column sits at TMEM address t_cols (lane field
// included).
// The bias of those columns is staged in the warp's shared-memory slot before
// the accumulator is awaited; the TMEM load of chunk j+1 is in flight while
// chunk j is converted and stored.  `release` runs once the last TMEM load of
// the tile has completed (it frees the accumulator for the next tile).
template <Epi EPI, int CHUNKS, typename WaitFull, typename Release>
__device__ __forceinline__ bool epilogue_warp_tile(uint32_t t_cols, int row, int col_begin, int M, int N,
                                                   const float* __restrict__ bias, float* bias_s,
                                                   __half* __restrict__ C, const SplitShape& sp,
                                                   WaitFull wait_full, Release release) {
  const int lane = threadIdx.x & 31;
  if constexpr (EPI != Epi::kStore) {
    for (int i = lane * 4; i < 32 * CHUNKS; i += 128) {
      float4 b = make_float4(0.f, 0.f, 0.f, 0.f);
      if (col_begin + i < N) b = *reinterpret_cast<const float4*>(bias + col_begin + i);
      *reinterpret_cast<float4*>(bias_s + i) = b;
    }
  }
  const bool row_ok = row < M;
  const size_t roff = row_ok ? row_offset<EPI>(row, N, sp) : 0;
  int got = 0;
  if (lane == 0) got = wait_full() ? 1 : 0;
  got = __shfl_sync(0xffffffffu, got, 0);     // also orders the bias staging before its use
  if (!got) return false;
  sm100::tc_fence_after();
  uint32_t ra[32], rb[32];
  sm100::tmem_ld_32x32b_x32_async(t_cols, ra);
#pragma unroll
  for (int j = 0; j < CHUNKS; ++j) {
    uint32_t(&cur)[32] = (j & 1) ? rb : ra;
    uint32_t(&nxt)[32] = (j & 1) ? ra : rb;
    sm100::tmem_wait_ld(cur);
    if (j + 1 < CHUNKS) {
      sm100::tmem_ld_32x32b_x32_async(t_cols + 32 * (j + 1), nxt);
    } else {
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) release();
    }
    const int col0 = col_begin + 32 * j;
    if (col0 < N) store_chunk<EPI>(cur, row_ok, col0, N, bias_s + 32 * j, C + roff + col_offset<EPI>(col0, sp));
  }
  return true;
}

template <int BN, Epi EPI>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                   int M, int N, int K, const float* __restrict__ bias, __half* __restrict__ C,
                   SplitShape sp, int* __restrict__ status) {
  using G = Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + G::kStages * G::kABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + G::kStages * G::kBBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + G::kNumBars);
  float* bias_smem = reinterpret_cast<float*>(smem + G::kBiasOffset);

  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (G::kStages + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * G::kStages + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * G::kStages + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * G::kStages + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_m = (M + kBM - 1) / kBM;
  const int num_n = (N + BN - 1) / BN;
  const int num_tiles = num_m * num_n;
  const int num_kb = (K + kBK - 1) / kBK;

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
          if (!mbar_wait(empty_bar(s), ph ^ 1u, kWaitLimitNs)) { ok = false; break; }
          mbar_arrive_expect_tx(full_bar(s), G::kStageBytes);
          tma_load_2d(&tm_a, smem_u32(sA + s * G::kABytes), full_bar(s), kb * kBK, m_blk * kBM);
          tma_load_2d(&tm_b, smem_u32(sB + s * G::kBBytes), full_bar(s), kb * kBK, n_blk * BN);
        }
      }
      // Let every copy this thread issued land before the CTA can exit.
      const uint32_t first = it > (uint32_t)G::kStages ? it - G::kStages : 0u;
      for (uint32_t j = first; j < it; ++j)
        mbar_wait(full_bar(j % G::kStages), (j / G::kStages) & 1u, kWaitLimitNs);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(kBM, BN);
      uint32_t it = 0, local = 0;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++local) {
        const uint32_t acc = local & 1u;
        const uint32_t aph = (local >> 1) & 1u;
        if (!mbar_wait(tempty_bar(acc), aph ^ 1u, kWaitLimitNs)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const int s = it % G::kStages;
          const uint32_t ph = (it / G::kStages) & 1u;
          if (!mbar_wait(full_bar(s), ph, kWaitLimitNs)) { ok = false; break; }
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
      mbar_wait(drain_bar, 0, kWaitLimitNs);
    }
  } else {
    const int quad = warp & 3;                 // TMEM lanes 32*quad .. 32*quad+31
    const int half = (warp - 2) >> 2;          // which half of the tile's columns
    constexpr int kChunks = BN / 64;           // 32-column chunks per warp
    float* bias_s = bias_smem + (warp - 2) * (BN / 2);
    uint32_t local = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
      const int m_blk = tile / num_n;
      const int n_blk = tile - m_blk * num_n;
      const uint32_t acc = local & 1u;
      const uint32_t aph = (local >> 1) & 1u;
      const uint32_t t_cols = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * BN + half * (BN / 2);
      const int row = m_blk * kBM + quad * 32 + lane;
      const bool got = epilogue_warp_tile<EPI, kChunks>(
          t_cols, row, n_blk * BN + half * (BN / 2), M, N, bias, bias_s, C, sp,
          [&] { return mbar_wait(tfull_bar(acc), aph, kWaitLimitNs); },
          [&] { mbar_arrive(tempty_bar(acc)); });
      if (!got) { ok = false; break; }
    }
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
struct PairCfg {
  static constexpr int kStages = 6;
  static constexpr int kABytes = 128 * kBK * 2;
  static constexpr int kBBytes = 128 * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = 512;             // two 256-column accumulators
  static constexpr int kNumBars = 2 * kStages + 5;
  static constexpr int kBiasOffset = (kStages * kStageBytes + kNumBars * 8 + 16 + 15) / 16 * 16;
  static constexpr int kSmem = 1024 + kBiasOffset + kEpiWarps * 128 * 4;
};

template <Epi EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gemm_tc_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                        int M, int N, int K, const float* __restrict__ bias, __half* __restrict__ C,
                        SplitShape sp, int* __restrict__ status) {
  using G = PairCfg;
  constexpr int BN = 256;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + G::kStages * G::kABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + G::kStages * G::kBBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + G::kNumBars);
  float* bias_smem = reinterpret_cast<float*>(smem + G::kBiasOffset);

  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (G::kStages + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * G::kStages + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * G::kStages + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * G::kStages + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int num_pairs = gridDim.x >> 1;
  const int num_m = (M + 255) / 256;
  const int num_n = (N + BN - 1) / BN;
  const int num_tiles = num_m * num_n;
  const int num_kb = (K + kBK - 1) / kBK;

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

  bool ok = true;
  uint32_t issued = 0;
  if (warp == 0) {
    if (lane == 0) {
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
        const int m_blk = tile / num_n;
        const int n_blk = tile - m_blk * num_n;
        const int a_row = m_blk * 256 + (int)rank * 128;
        const int b_row = n_blk * BN + (int)rank * 128;
        for (int kb = 0; kb < num_kb; ++kb, ++issued) {
          const int s = issued % G::kStages;
          const uint32_t ph = (issued / G::kStages) & 1u;
          if (!mbar_wait(empty_bar(s), ph ^ 1u, kWaitLimitNs)) { ok = false; break; }
          const uint32_t leader_full = mapa_shared(full_bar(s), 0);
          mbar_arrive_expect_tx_cluster(leader_full, G::kStageBytes);
          tma_load_2d_pair(&tm_a, smem_u32(sA + s * G::kABytes), leader_full, kb * kBK, a_row);
          tma_load_2d_pair(&tm_b, smem_u32(sB + s * G::kBBytes), leader_full, kb * kBK, b_row);
        }
      }
      if (rank == 0) {
        // Every copy of both CTAs counted on the leader's full barriers has landed.
        const uint32_t first = issued > (uint32_t)G::kStages ? issued - G::kStages : 0u;
        for (uint32_t j = first; j < issued; ++j)
          mbar_wait(full_bar(j % G::kStages), (j / G::kStages) & 1u, kWaitLimitNs);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(256, BN);
      uint32_t it = 0, local = 0;
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs, ++local) {
        const uint32_t acc = local & 1u;
        const uint32_t aph = (local >> 1) & 1u;
        if (!mbar_wait(tempty_bar(acc), aph ^ 1u, kWaitLimitNs)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const int s = it % G::kStages;
          const uint32_t ph = (it / G::kStages) & 1u;
          if (!mbar_wait(full_bar(s), ph, kWaitLimitNs)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + s * G::kABytes);
          const uint32_t b_addr = smem_u32(sB + s * G::kBBytes);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            mma_f16_ss_pair(d_tmem, smem_desc_sw128(a_addr + kk * 32), smem_desc_sw128(b_addr + kk * 32), idesc,
                            (kb > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit_pair(empty_bar(s), 0x3);
        }
        if (!ok) break;
        mma_commit_pair(tfull_bar(acc), 0x3);
      }
      mma_commit_pair(drain_bar, 0x3);
    }
    if (lane == 0) mbar_wait(drain_bar, 0, kWaitLimitNs);   // the leader's MMAs are done
    __syncwarp();
  } else {
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    constexpr int kChunks = BN / 64;
    float* bias_s = bias_smem + (warp - 2) * (BN / 2);
    const uint32_t leader_tempty0 = mapa_shared(tempty_bar(0), 0);
    const uint32_t leader_tempty1 = mapa_shared(tempty_bar(1), 0);
    uint32_t local = 0;
    for (int tile = pair; tile < num_tiles; tile += num_pairs, ++local) {
      const int m_blk = tile / num_n;
      const int n_blk = tile - m_blk * num_n;
      const uint32_t acc = local & 1u;
      const uint32_t aph = (local >> 1) & 1u;
      const uint32_t t_cols = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * BN + half * (BN / 2);
      const int row = m_blk * 256 + (int)rank * 128 + quad * 32 + lane;
      const bool got = epilogue_warp_tile<EPI, kChunks>(
          t_cols, row, n_blk * BN + half * (BN / 2), M, N, bias, bias_s, C, sp,
          [&] { return mbar_wait(tfull_bar(acc), aph, kWaitLimitNs); },
          [&] { mbar_arrive_cluster(acc ? leader_tempty1 : leader_tempty0); });
      if (!got) { ok = false; break; }
    }
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

template <Epi EPI>
cudaError_t launch_pair(const TcGemmArgs& a, cudaStream_t stream) {
  using G = PairCfg;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  static int max_clusters = 0;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(gemm_tc_pair_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    G::kSmem);
    if (attr_err != cudaSuccess) return;
    // How many 2-CTA clusters of this kernel fit on the GPU at once: a persistent
    // grid larger than that would run its last clusters as a second wave.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * 512, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = G::kSmem;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    attr_err = cudaOccupancyMaxActiveClusters(&max_clusters, gemm_tc_pair_kernel<EPI>, &cfg);
    if (getenv("ENC_DEBUG")) fprintf(stderr, "[enc] pair GEMM: %d co-resident clusters\n", max_clusters);
  });
  if (attr_err != cudaSuccess) return attr_err;
  if (max_clusters <= 0) return cudaErrorInvalidConfiguration;
  const int tiles = ((a.M + 255) / 256) * ((a.N + 255) / 256);
  const int pairs = tiles < max_clusters ? tiles : max_clusters;
  gemm_tc_pair_kernel<EPI><<<2 * pairs, kThreads, G::kSmem, stream>>>(*a.tmap_a, *a.tmap_b, a.M, a.N, a.K,
                                                                      a.bias, a.c, a.split, a.status);
  return cudaGetLastError();
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
  gemm_tc_kernel<BN, EPI><<<grid, kThreads, G::kSmem, stream>>>(*a.tmap_a, *a.tmap_b, a.M, a.N, a.K,
                                                               a.bias, a.c, a.split, a.status);
  return cudaGetLastError();
}

template <int BN>
cudaError_t launch_bn(const TcGemmArgs& a, cudaStream_t stream) {
  switch (a.epi) {
    case Epi::kStore: return launch_impl<BN, Epi::kStore>(a, stream);
    case Epi::kBiasGelu: return launch_impl<BN, Epi::kBiasGelu>(a, stream);
    case Epi::kBiasQkvSplit: return launch_impl<BN, Epi::kBiasQkvSplit>(a, stream);
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

cudaError_t launch_gemm_tc(const TcGemmArgs& a, cudaStream_t stream) {
  if (a.M <= 0 || a.N <= 0 || a.K <= 0 || (a.N % 8) != 0 || (a.K % 8) != 0) return cudaErrorInvalidValue;
  if (a.epi == Epi::kBiasQkvSplit && (a.split.size_per_head % 32) != 0) return cudaErrorInvalidValue;
  if (a.bn == kPairTile) {
    if ((a.N % 256) != 0) return cudaErrorInvalidValue;
    switch (a.epi) {
      case Epi::kStore: return launch_pair<Epi::kStore>(a, stream);
      case Epi::kBiasGelu: return launch_pair<Epi::kBiasGelu>(a, stream);
      case Epi::kBiasQkvSplit: return launch_pair<Epi::kBiasQkvSplit>(a, stream);
    }
    return cudaErrorInvalidValue;
  }
  if (a.bn == 256) return launch_bn<256>(a, stream);
  if (a.bn == 128) return launch_bn<128>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace enc
