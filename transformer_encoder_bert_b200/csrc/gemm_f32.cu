// FP32 GEMM on CUDA cores (FFMA, no TF32) for the FP32 computation mode.
//
// The source page ("什么是 Faster Transformer") offers an FP32 mode beside
// FP16; tcgen05 has no exact-FP32 kind, so FP32 mode runs its matrix
// multiplies here.  C = A[M,K] * W[K,N] with the same epilogues as the
// tensor-core GEMM (plain, add-bias + GELU, add-bias + Q/K/V head split).
// 64x64 output tile per 256-thread block, 4x4 outputs per thread, K in
// steps of 16 staged through shared memory.
#include "internal.h"

namespace enc {
namespace {

constexpr int TM = 64, TN = 64, TK = 16;

template <Epi EPI>
__global__ void __launch_bounds__(256) gemm_f32_kernel(const float* __restrict__ A,
                                                       const float* __restrict__ W, int M, int N,
                                                       int K, const float* __restrict__ bias,
                                                       float* __restrict__ C, SplitShape sp,
                                                       const float* __restrict__ resid) {
  __shared__ float As[TK][TM + 4];
  __shared__ float Ws[TK][TN + 4];
  pdl_wait();
  pdl_trigger();
  const int tx = threadIdx.x & 15;   // column group
  const int ty = threadIdx.x >> 4;   // row group
  const int m0 = blockIdx.y * TM;
  const int n0 = blockIdx.x * TN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += TK) {
    // A tile: 64 rows x 16 k, stored k-major in shared memory.
    for (int i = threadIdx.x; i < TM * TK; i += 256) {
      const int r = i / TK, k = i % TK;
      const int gm = m0 + r, gk = k0 + k;
      As[k][r] = (gm < M && gk < K) ? A[(size_t)gm * K + gk] : 0.0f;
    }
    for (int i = threadIdx.x; i < TK * TN; i += 256) {
      const int k = i / TN, c = i % TN;
      const int gk = k0 + k, gn = n0 + c;
      Ws[k][c] = (gk < K && gn < N) ? W[(size_t)gk * N + gn] : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < TK; ++k) {
      float a[4], w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[k][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) w[j] = Ws[k][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= N) continue;
      float v = acc[i][j];
      if constexpr (EPI != Epi::kStore) v += bias[n];
      if constexpr (EPI == Epi::kBiasResidStore) v += resid[(size_t)m * N + n];
      if constexpr (EPI == Epi::kBiasGelu) v = 0.5f * v * (1.0f + erff(v * 0.70710678118654752f));
      if constexpr (EPI == Epi::kBiasGeluTanh)
        v = 0.5f * v * (1.0f + tanhf(0.7978845608028654f * (v + 0.044715f * v * v * v)));
      if constexpr (EPI == Epi::kBiasQkvSplit) {
        const int H = sp.head_num * sp.size_per_head;
        const int t = n / H, rem = n - t * H;
        const int h = rem / sp.size_per_head, c = rem - h * sp.size_per_head;
        const int b = m / sp.seq, s = m - b * sp.seq;
        C[((((size_t)t * sp.batch + b) * sp.head_num + h) * sp.seq + s) * sp.size_per_head + c] = v;
      } else {
        C[(size_t)m * N + n] = v;
      }
    }
  }
}

}  // namespace

cudaError_t launch_gemm_f32(const float* A, const float* W, int M, int N, int K, Epi epi,
                            const float* bias, float* C, SplitShape split, cudaStream_t stream,
                            const float* resid) {
  if (M <= 0 || N <= 0 || K <= 0) return cudaErrorInvalidValue;
  const dim3 grid((N + TN - 1) / TN, (M + TM - 1) / TM);
  switch (epi) {
    case Epi::kStore:
      return launch_kernel(gemm_f32_kernel<Epi::kStore>, grid, dim3(256), 0, stream, nullptr, 0, A, W, M, N, K, bias,
                           C, split, resid);
    case Epi::kBiasGelu:
      return launch_kernel(gemm_f32_kernel<Epi::kBiasGelu>, grid, dim3(256), 0, stream, nullptr, 0, A, W, M, N, K, bias,
                           C, split, resid);
    case Epi::kBiasQkvSplit:
      return launch_kernel(gemm_f32_kernel<Epi::kBiasQkvSplit>, grid, dim3(256), 0, stream, nullptr, 0, A, W, M, N, K, bias,
                           C, split, resid);
    case Epi::kBiasGeluTanh:
      return launch_kernel(gemm_f32_kernel<Epi::kBiasGeluTanh>, grid, dim3(256), 0, stream, nullptr, 0, A, W, M, N, K, bias,
                           C, split, resid);
    case Epi::kBiasStore:
      return launch_kernel(gemm_f32_kernel<Epi::kBiasStore>, grid, dim3(256), 0, stream, nullptr, 0, A, W, M, N, K, bias,
                           C, split, resid);
    case Epi::kBiasResidStore:
      if (!resid) return cudaErrorInvalidValue;
      return launch_kernel(gemm_f32_kernel<Epi::kBiasResidStore>, grid, dim3(256), 0, stream, nullptr, 0, A, W, M, N,
                           K, bias, C, split, resid);
  }
  return cudaErrorInvalidValue;
}

}  // namespace enc
