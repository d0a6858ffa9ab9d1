// LayerNorm of rows that already hold z = a + bias + residual.
//
// The source page ("Faster Transformer 优化原理") fuses add-bias, residual
// and Layer Normalization into one custom kernel (run twice per layer), reads
// FP16 data as half2 but sums in float, reduces rows with warp shuffles and
// uses rsqrtf for 1/sqrt.  Here the add-bias and residual move one step
// earlier, into the epilogue of the GEMM that produces `a` (which reads the
// residual tile while its tensor cores run), so this kernel reads one input
// row instead of two: 4 bytes per element of HBM traffic instead of 6.
// Each lane moves 16-byte vectors (8 halves or 4 floats) and keeps its share
// of the row in registers, so the row is read once; mean and variance are two
// in-register passes (variance of deviations, no E[x^2] - E[x]^2
// cancellation), all in FP32.
//   out = gamma * (z - mean) * rsqrt(var + eps) + beta.
#include "internal.h"

namespace enc {
namespace {

template <typename T>
struct Vec;
template <>
struct Vec<__half> {
  static constexpr int kN = 8;
  using Raw = uint4;
  __device__ static void unpack(const uint4& u, float (&v)[8]) {
    const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __half22float2(h[i]);
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  }
  __device__ static void store(__half* p, const float (&v)[8]) {
    uint4 u;
    __half2* h = reinterpret_cast<__half2*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(v[2 * i], v[2 * i + 1]);
    *reinterpret_cast<uint4*>(p) = u;
  }
};
template <>
struct Vec<float> {
  static constexpr int kN = 4;
  using Raw = float4;
  __device__ static void unpack(const float4& f, float (&v)[4]) {
    v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
  }
  __device__ static void store(float* p, const float (&v)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// Shared-memory copy of gamma and beta in the row's own element type: for
// FP16 rows the parameters came from the caller as halves (the handle widened
// them to FP32), so narrowing them back is exact, and a lane then reads each
// parameter's 8 elements as one conflict-free 16-byte load.
template <typename T>
__device__ __forceinline__ void store_param4(T* dst, float4 v);
template <>
__device__ __forceinline__ void store_param4<float>(float* dst, float4 v) {
  *reinterpret_cast<float4*>(dst) = v;
}
template <>
__device__ __forceinline__ void store_param4<__half>(__half* dst, float4 v) {
  __half2 lo = __floats2half2_rn(v.x, v.y), hi = __floats2half2_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&lo);
  u.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(dst) = u;
}

// Normalises one row held as VPT 16-byte vectors per lane (lane l owns vectors
// l, l + 32, ...) and stores it; gamma/beta vectors come from `param(c)`.
template <typename T, int VPT, typename Params>
__device__ __forceinline__ void normalise_row(const typename Vec<T>::Raw (&zr)[VPT], int lane, int nvec, int H,
                                              T* orow, Params param) {
  constexpr int E = Vec<T>::kN;
  float z[VPT][E];
  float sum = 0.f;
#pragma unroll
  for (int v = 0; v < VPT; ++v) {
    if (lane + 32 * v < nvec) {
      Vec<T>::unpack(zr[v], z[v]);
#pragma unroll
      for (int e = 0; e < E; ++e) sum += z[v][e];
    }
  }
  const float mean = warp_sum(sum) / (float)H;
  float sq = 0.f;
#pragma unroll
  for (int v = 0; v < VPT; ++v) {
    if (lane + 32 * v < nvec) {
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const float d = z[v][e] - mean;
        sq = fmaf(d, d, sq);
      }
    }
  }
  const float rstd = rsqrtf(warp_sum(sq) / (float)H + kLnEps);
#pragma unroll
  for (int v = 0; v < VPT; ++v) {
    const int c = lane + 32 * v;
    if (c < nvec) {
      float o[E], gg[E], tt[E];
      param(v, c, gg, tt);
#pragma unroll
      for (int e = 0; e < E; ++e) o[e] = fmaf((z[v][e] - mean) * rstd, gg[e], tt[e]);
      Vec<T>::store(orow + c * E, o);
    }
  }
}

// VPT = 16-byte vectors per lane (the row holds at most 32*VPT vectors).
// A block of 8 warps stages gamma and beta in shared memory once; each warp
// then walks rows warp_id, warp_id + num_warps, ..., loading the next row
// while it normalises the current one.  Used for FP32 rows and H > 1024.
constexpr int kLnWarps = 8;

template <typename T, int VPT>
__global__ void __launch_bounds__(kLnWarps * 32)
    layernorm_kernel(const T* __restrict__ zin, const float* __restrict__ gamma, const float* __restrict__ beta,
                     T* __restrict__ out, int rows, int H) {
  constexpr int E = Vec<T>::kN;
  using Raw = typename Vec<T>::Raw;
  extern __shared__ __align__(16) uint8_t params_raw[];   // [2][H] of T: gamma, beta
  T* params = reinterpret_cast<T*>(params_raw);
  for (int i = threadIdx.x * 4; i < H; i += blockDim.x * 4) {   // parameters: written by no kernel
    store_param4<T>(params + i, *reinterpret_cast<const float4*>(gamma + i));
    store_param4<T>(params + H + i, *reinterpret_cast<const float4*>(beta + i));
  }
  pdl_wait();                                   // the rows of the previous kernels are visible
  pdl_trigger();
  __syncthreads();
  const T* sg = params;
  const T* st = params + H;
  const int lane = threadIdx.x & 31;
  const int nvec = H / E;
  const int warps = gridDim.x * kLnWarps;
  auto load_row = [&](int r, Raw (&x)[VPT]) {
#pragma unroll
    for (int v = 0; v < VPT; ++v) {
      const int c = lane + 32 * v;
      if (c < nvec) x[v] = *reinterpret_cast<const Raw*>(zin + (size_t)r * H + c * E);
    }
  };
  auto param = [&](int, int c, float (&gg)[E], float (&tt)[E]) {
    Vec<T>::unpack(*reinterpret_cast<const Raw*>(sg + c * E), gg);
    Vec<T>::unpack(*reinterpret_cast<const Raw*>(st + c * E), tt);
  };
  Raw za[VPT];
  int row = blockIdx.x * kLnWarps + (threadIdx.x >> 5);
  if (row < rows) load_row(row, za);
  for (; row < rows; row += warps) {
    Raw zn[VPT];
    const int next = row + warps;
    if (next < rows) load_row(next, zn);
    normalise_row<T, VPT>(za, lane, nvec, H, out + (size_t)row * H, param);
#pragma unroll
    for (int v = 0; v < VPT; ++v) za[v] = zn[v];
  }
}

int blocks_per_sm(const void* fn, size_t dyn_smem) {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, kLnWarps * 32, dyn_smem) != cudaSuccess || n < 1) n = 1;
  return n;
}

// FP16 rows, one row per warp and no row loop: many small blocks keep many
// rows in flight; gamma and beta are read as halves (the handle keeps FP16
// copies, exact in FP16 mode) through L1, 16 bytes per 8 elements.
template <int VPT>
__global__ void __launch_bounds__(128)
    layernorm_rowwarp_kernel(const __half* __restrict__ zin, const __half* __restrict__ gamma,
                             const __half* __restrict__ beta, __half* __restrict__ out, int rows, int H,
                             const int* __restrict__ rows_dev) {
  constexpr int E = 8;
  const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int nvec = H / E;
  // gamma and beta do not depend on the previous kernel: requested before
  // waiting for it.
  uint4 gv[VPT], bv[VPT];
#pragma unroll
  for (int v = 0; v < VPT; ++v) {
    const int c = lane + 32 * v;
    if (c < nvec) {
      gv[v] = __ldg(reinterpret_cast<const uint4*>(gamma + c * E));
      bv[v] = __ldg(reinterpret_cast<const uint4*>(beta + c * E));
    }
  }
  pdl_wait();                                   // the rows of the previous kernels are visible
  pdl_trigger();
  if (rows_dev) rows = min(rows, *rows_dev);   // packed tokens: the row count lives on the device
  if (row >= rows) return;
  uint4 za[VPT];
#pragma unroll
  for (int v = 0; v < VPT; ++v) {
    const int c = lane + 32 * v;
    if (c < nvec) za[v] = __ldg(reinterpret_cast<const uint4*>(zin + (size_t)row * H + c * E));
  }
  normalise_row<__half, VPT>(za, lane, nvec, H, out + (size_t)row * H, [&](int v, int, float (&gg)[E], float (&tt)[E]) {
    Vec<__half>::unpack(gv[v], gg);
    Vec<__half>::unpack(bv[v], tt);
  });
}

template <typename T>
cudaError_t launch_ln(const T* z, const float* gamma, const float* beta, T* out, int rows, int H,
                      cudaStream_t stream) {
  constexpr int E = Vec<T>::kN;
  if (rows <= 0 || H <= 0 || H % E != 0 || H % 4 != 0) return cudaErrorInvalidValue;
  const int vpt = (H / E + 31) / 32;
  const int want = (rows + kLnWarps - 1) / kLnWarps;
  const size_t smem = (size_t)2 * H * sizeof(T);
  // Persistent grid: exactly the blocks that are resident at once (a larger
  // grid would run its row loops in waves), each warp walking several rows.
#define ENC_LN_CASE(V)                                                                                 \
  if (vpt <= V) {                                                                                      \
    const int cap = blocks_per_sm((const void*)layernorm_kernel<T, V>, smem) * device_sm_count();      \
    const dim3 grid(want < cap ? want : cap);                                                          \
    return launch_kernel(layernorm_kernel<T, V>, grid, dim3(kLnWarps * 32), smem, stream, nullptr, 0, z, \
                         gamma, beta, out, rows, H);                                                   \
  }
  ENC_LN_CASE(1)
  ENC_LN_CASE(2)
  ENC_LN_CASE(3)
  ENC_LN_CASE(4)
  ENC_LN_CASE(6)
  ENC_LN_CASE(8)
#undef ENC_LN_CASE
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_layernorm_f16h(const __half* z, const __half* gamma, const __half* beta, __half* out, int rows,
                                  int hidden, cudaStream_t stream, const int* rows_dev) {
  if (rows <= 0 || hidden <= 0 || hidden % 8 != 0) return cudaErrorInvalidValue;
  const int vpt = (hidden / 8 + 31) / 32;
  const dim3 grid((rows + 3) / 4);
#define ENC_LN_ROW_CASE(V)                                                                                 \
  if (vpt <= V) {                                                                                          \
    return launch_kernel(layernorm_rowwarp_kernel<V>, grid, dim3(128), 0, stream, nullptr, 0, z, gamma, beta, \
                         out, rows, hidden, rows_dev);                                                     \
  }
  ENC_LN_ROW_CASE(1)
  ENC_LN_ROW_CASE(2)
  ENC_LN_ROW_CASE(3)
  ENC_LN_ROW_CASE(4)
#undef ENC_LN_ROW_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_layernorm_f16(const __half* z, const float* gamma, const float* beta, __half* out, int rows,
                                 int hidden, cudaStream_t stream) {
  return launch_ln<__half>(z, gamma, beta, out, rows, hidden, stream);
}

cudaError_t launch_layernorm_f32(const float* z, const float* gamma, const float* beta, float* out, int rows,
                                 int hidden, cudaStream_t stream) {
  return launch_ln<float>(z, gamma, beta, out, rows, hidden, stream);
}

}  // namespace enc
