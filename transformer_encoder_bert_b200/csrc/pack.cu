// Padding removal: pack the valid tokens of a [batch, seq, H] batch into
// [T, H] (T = total valid tokens) and scatter results back.
//
// The source page fixes the sequence length "for performance" and plans
// arbitrary lengths ("什么是 Faster Transformer"); with the valid lengths of a
// batch known on the device, the projections, FFN and LayerNorms can run on
// the T valid rows only, and attention reads each sequence's rows through
// per-sequence offsets.  Everything stays on the device: the row count T is
// written to offsets[batch] and read there by the kernels that follow, so a
// packed forward needs no host synchronisation and can be recorded in a graph.
#include "internal.h"

namespace enc {
namespace {

constexpr int kScanThreads = 1024;

// offsets[b] = sum of clamp(valid_len[b'], 0, seq) over b' < b; offsets[batch] = T.
// One block: each thread sums a contiguous slice of sequences, the block scans
// the slice totals with warp shuffles, then each thread writes its slice.
__global__ void __launch_bounds__(kScanThreads)
    valid_offsets_kernel(const int32_t* __restrict__ valid_len, int batch, int seq, int32_t* __restrict__ offsets) {
  __shared__ int warp_tot[kScanThreads / 32];
  pdl_wait();
  pdl_trigger();
  const int per = (batch + kScanThreads - 1) / kScanThreads;
  const int b0 = threadIdx.x * per;
  const int b1 = min(b0 + per, batch);
  int local = 0;
  for (int b = b0; b < b1; ++b) local += min(max(valid_len[b], 0), seq);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kScanThreads / 32 ? warp_tot[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, w, off);
      if (lane >= off) w += v;
    }
    if (lane < kScanThreads / 32) warp_tot[lane] = w;   // inclusive totals of warps
  }
  __syncthreads();
  int run = (warp > 0 ? warp_tot[warp - 1] : 0) + incl - local;   // exclusive prefix of this slice
  for (int b = b0; b < b1; ++b) {
    offsets[b] = run;
    run += min(max(valid_len[b], 0), seq);
  }
  if (threadIdx.x == kScanThreads - 1) offsets[batch] = warp_tot[kScanThreads / 32 - 1];
}

// One warp per (sequence, position): 16-byte moves of a row of `hidden` halves.
template <bool PACK>
__global__ void __launch_bounds__(128)
    move_rows_kernel(const __half* __restrict__ src, const int32_t* __restrict__ valid_len,
                     const int32_t* __restrict__ offsets, __half* __restrict__ dst, int batch, int seq, int hidden) {
  pdl_wait();
  pdl_trigger();
  const long tok = (long)blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (tok >= (long)batch * seq) return;
  const int b = (int)(tok / seq), s = (int)(tok - (long)b * seq);
  const int n = min(max(valid_len[b], 0), seq);
  const int nvec = hidden / 8;
  if (PACK) {
    if (s >= n) return;
    const uint4* in = reinterpret_cast<const uint4*>(src + tok * hidden);
    uint4* out = reinterpret_cast<uint4*>(dst + ((long)offsets[b] + s) * hidden);
    for (int c = lane; c < nvec; c += 32) out[c] = in[c];
  } else {
    uint4* out = reinterpret_cast<uint4*>(dst + tok * hidden);
    if (s < n) {
      const uint4* in = reinterpret_cast<const uint4*>(src + ((long)offsets[b] + s) * hidden);
      for (int c = lane; c < nvec; c += 32) out[c] = in[c];
    } else {
      for (int c = lane; c < nvec; c += 32) out[c] = make_uint4(0, 0, 0, 0);
    }
  }
}

}  // namespace

cudaError_t launch_valid_offsets(const int32_t* valid_len, int batch, int seq, int32_t* offsets,
                                 cudaStream_t stream) {
  if (batch <= 0 || seq <= 0) return cudaErrorInvalidValue;
  return launch_kernel(valid_offsets_kernel, dim3(1), dim3(kScanThreads), 0, stream, nullptr, 0, valid_len, batch, seq,
                       offsets);
}

cudaError_t launch_pack_rows(const __half* x, const int32_t* valid_len, const int32_t* offsets, __half* xp,
                             int batch, int seq, int hidden, cudaStream_t stream) {
  if (batch <= 0 || seq <= 0 || hidden % 8 != 0) return cudaErrorInvalidValue;
  const long tokens = (long)batch * seq;
  return launch_kernel(move_rows_kernel<true>, dim3((unsigned)((tokens + 3) / 4)), dim3(128), 0, stream, nullptr, 0, x,
                       valid_len, offsets, xp, batch, seq, hidden);
}

cudaError_t launch_unpack_rows(const __half* yp, const int32_t* valid_len, const int32_t* offsets, __half* out,
                               int batch, int seq, int hidden, cudaStream_t stream) {
  if (batch <= 0 || seq <= 0 || hidden % 8 != 0) return cudaErrorInvalidValue;
  const long tokens = (long)batch * seq;
  return launch_kernel(move_rows_kernel<false>, dim3((unsigned)((tokens + 3) / 4)), dim3(128), 0, stream, nullptr, 0,
                       yp, valid_len, offsets, out, batch, seq, hidden);
}

}  // namespace enc
