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
//   warps 2..5  epilogue: tcgen05.ld of their 32 TMEM lanes (32 rows),
//               bias / GELU / head split, 16-byte stores to global memory.
// The two accumulators let the epilogue of tile i overlap the MMAs of tile
// i+1.  Every mbarrier wait is bounded (kWaitLimitNs); a wait that gives up
// records kStatusWaitTimeout in the status word and the CTA drains its copies
// and MMAs, frees TMEM and exits.
#include <cstdio>
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
constexpr int kEpiWarps = 4;
constexpr int kThreads = 64 + 32 * kEpiWarps;

template <int BN>
struct Cfg {
  static constexpr int kStages = BN == 256 ? 4 : 6;
  static constexpr int kABytes = kBM * kBK * 2;
  static constexpr int kBBytes = BN * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = 2 * BN;
  static constexpr int kNumBars = 2 * kStages + 5;
  static constexpr int kSmem = 1024 + kStages * kStageBytes + kNumBars * 8 + 16;
};

__device__ __forceinline__ float gelu_erf(float v) {
  return 0.5f * v * (1.0f + erff(v * 0.70710678118654752f));
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Epilogue for one thread: 32 accumulator columns of one row.
template <Epi EPI>
__device__ __forceinline__ void store_chunk(const uint32_t (&r)[32], int row, int col0, int M,
                                            int N, const float* __restrict__ bias,
                                            __half* __restrict__ C, const SplitShape& sp) {
  if (row >= M) return;
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
  if constexpr (EPI != Epi::kStore) {
#pragma unroll
    for (int i = 0; i < 32; i += 4) {
      if (col0 + i < N) {
        const float4 b = *reinterpret_cast<const float4*>(bias + col0 + i);
        v[i] += b.x; v[i + 1] += b.y; v[i + 2] += b.z; v[i + 3] += b.w;
      }
    }
  }
  if constexpr (EPI == Epi::kBiasGelu) {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = gelu_erf(v[i]);
  }
  __half* dst;
  if constexpr (EPI == Epi::kBiasQkvSplit) {
    const int H = sp.head_num * sp.size_per_head;
    const int t = col0 / H;
    const int rem = col0 - t * H;
    const int h = rem / sp.size_per_head;
    const int c = rem - h * sp.size_per_head;
    const int b = row / sp.seq;
    const int s = row - b * sp.seq;
    dst = C + ((((size_t)t * sp.batch + b) * sp.head_num + h) * sp.seq + s) * sp.size_per_head + c;
  } else {
    dst = C + (size_t)row * N + col0;
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
    uint32_t local = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
      const int m_blk = tile / num_n;
      const int n_blk = tile - m_blk * num_n;
      const uint32_t acc = local & 1u;
      const uint32_t aph = (local >> 1) & 1u;
      int got = 0;
      if (lane == 0) got = mbar_wait(tfull_bar(acc), aph, kWaitLimitNs) ? 1 : 0;
      got = __shfl_sync(0xffffffffu, got, 0);
      if (!got) { ok = false; break; }
      tc_fence_after();
      const int row = m_blk * kBM + quad * 32 + lane;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * BN;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(t_row + c * 32, r);
        if (c == BN / 32 - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(tempty_bar(acc));
        }
        const int col0 = n_blk * BN + c * 32;
        if (col0 < N) store_chunk<EPI>(r, row, col0, M, N, bias, C, sp);
      }
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
  if (a.bn == 256) return launch_bn<256>(a, stream);
  if (a.bn == 128) return launch_bn<128>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace enc
