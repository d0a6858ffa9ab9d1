// Masked scaled-dot-product attention on the 5th-generation tensor cores
// (tcgen05 + TMEM + TMA) for size_per_head 64 and 64 < seq <= 128, where one
// block of 128 keys covers every key of a sequence.
//
// The source page ("Faster Transformer 优化原理") runs attention as two batched
// GEMMs around a SoftMax kernel.  Here both products run on tcgen05 and the
// score tile never leaves the SM: one CTA per (sequence, head), 160 threads:
//   warps 0..3  softmax: thread r owns query row r = TMEM lane r.  It reads its
//               row of S from TMEM, takes the row max over the valid keys (the
//               row is in one thread: no shuffles), forms
//               P = exp(S/sqrt(d) - max) in FP32, sums it, and writes P as FP16
//               in the 128-byte-swizzled K-major layout the next MMA reads.
//               After P V it scales its row of O by 1/sum and stores it.
//   warp 4      one thread issues the TMA loads of Q, K and V and the MMAs
//                 S = Q K^T   M=128, N=128, K=64  (A, B K-major)
//                 O = P V     M=128, N=64,  K=128 (A K-major; B = V read
//                             MN-major straight from its token-major tile)
// The valid length n is the same for every row of the CTA, so every masking
// decision is a warp-uniform branch: 32-key chunks wholly past n are skipped,
// chunks wholly inside n run unmasked, and at most one chunk is masked per
// element.  Keys j >= n get weight exactly 0.
//
// Footprint, so that four CTAs share an SM (their loads, MMAs and softmax
// overlap one another): P (32 KB) overwrites the Q and K tiles once S = Q K^T
// has completed, the output rows are staged in the V tile once O = P V has
// completed, and O takes S's TMEM columns [0, 64) (128 columns per CTA).
// Every mbarrier wait is bounded in time.
//
// Q, K and V are read through one 2-D tensor map with rows of 64 halves:
// the split layout [3, B, nh, S, 64] (rows = ((t*B + b)*nh + h)*S + s) or the
// packed [T, 3H] layout (column offset t*H + h*64, rows = offsets[b] + s).
#include <mutex>

#include <cudaTypedefs.h>

#include "internal.h"
#include "sm100.cuh"

namespace enc {
namespace {

using namespace sm100;

constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr int kD = 64;
constexpr int kRows = 128;                        // query rows = keys per CTA
constexpr int kSoftmaxWarps = 4;
constexpr int kThreads = 32 * (kSoftmaxWarps + 1);
constexpr int kTileBytes = kRows * kD * 2;        // 16 KB: 128 rows x 64 halves
constexpr int kTmemCols = 128;
constexpr float kLog2e = 1.4426950408889634f;

// Shared memory (offsets from a 1024-byte-aligned base).
constexpr int kQ = 0;                             // Q tile, then P keys 0..63
constexpr int kK = kTileBytes;                    // K tile, then P keys 64..127
constexpr int kP = 0;                             // P: two 64-key K-major atoms
constexpr int kV = 2 * kTileBytes;                // V tile, then the output rows
constexpr int kBars = 3 * kTileBytes;
// qk_full, v_full, s_full, p_full, o_full, drain
constexpr int kNumBars = 6;
constexpr int kSlot = kBars + kNumBars * 8;
constexpr int kSmemTotal = 1024 + kSlot + 16;

// MN-major operand, 128-byte swizzle: 64 contiguous MN elements (128 bytes) per
// row, K rows 128 bytes apart in groups of 8 that are 1 KB apart (stride byte
// offset); one 64-element MN atom, so the leading byte offset is not used.
__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(1u) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// kind::f16 instruction descriptor with B MN-major (bit 16).
__host__ __device__ constexpr uint32_t idesc_f16_f32_bmn(int m, int n) { return idesc_f16_f32(m, n) | (1u << 16); }

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t cvt_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Waits on one lane, result broadcast to the warp.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity) {
  int got = 0;
  if ((threadIdx.x & 31) == 0) got = mbar_wait(bar, parity, kWaitLimitNs) ? 1 : 0;
  return __shfl_sync(0xffffffffu, got, 0) != 0;
}

// Stores 16-byte unit `unit` (0..15) of a 128-key FP16 row r of P: keys
// 64a .. 64a+63 form atom a (rows of 128 bytes), units swizzled by r & 7.
__device__ __forceinline__ void store_p_unit(uint8_t* prow, int unit, int r, uint4 v) {
  *reinterpret_cast<uint4*>(prow + (unit >> 3) * kTileBytes + 16 * ((unit & 7) ^ (r & 7))) = v;
}

// P of 32 keys (chunk c of the row) from 32 raw scores: p = 2^(s*c2 - m*c2)
// for the first `lim` keys, 0 for the rest; adds to the pair sum and writes
// the FP16 values as four 16-byte units of the row.
template <bool MASKED>
__device__ __forceinline__ void p_chunk(const uint32_t (&sv)[32], int lim, uint64_t scale2, uint64_t neg_m2,
                                        uint64_t& sum2, uint8_t* prow, int c, int r) {
  uint32_t pk[16];
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    const uint64_t t = f2_fma(f2_pack(__uint_as_float(sv[i]), __uint_as_float(sv[i + 1])), scale2, neg_m2);
    float t0, t1;
    f2_unpack(t, t0, t1);
    float p0 = ex2(t0), p1 = ex2(t1);
    if (MASKED) {
      p0 = i < lim ? p0 : 0.f;
      p1 = i + 1 < lim ? p1 : 0.f;
    }
    sum2 = f2_add(sum2, f2_pack(p0, p1));
    pk[i >> 1] = cvt_half2(p0, p1);
  }
#pragma unroll
  for (int u = 0; u < 4; ++u)
    store_p_unit(prow, 4 * c + u, r, make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]));
}

template <bool PACKED>
__global__ void __launch_bounds__(kThreads, 4)   // four CTAs per SM (TMEM 4 x 128 columns)
    attention_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv, const int32_t* __restrict__ valid_len,
                        const int32_t* __restrict__ offsets, __half* __restrict__ ctx, int B, int S, int NH,
                        float score_scale_log2, int* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + kBars;
  const uint32_t qk_full = bar0, v_full = bar0 + 8, s_full = bar0 + 16, p_full = bar0 + 24, o_full = bar0 + 32,
                 drain = bar0 + 40;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kSlot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x, b = blockIdx.y;
  pdl_wait();                                          // Q/K/V (and offsets) of the previous kernels are visible
  int n = valid_len[b];
  n = n < 0 ? 0 : (n > S ? S : n);
  if (PACKED && n == 0) return;                        // the sequence has no rows (uniform per CTA)
  const int rows_exist = PACKED ? n : S;
  const int H = NH * kD;

  // Tensor-map coordinates of row s of block t (0 = Q, 1 = K, 2 = V).
  auto coord_x = [&](int t) { return PACKED ? t * H + h * kD : 0; };
  auto coord_y = [&](int t, int s) { return PACKED ? offsets[b] + s : ((t * B + b) * NH + h) * S + s; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) mbar_init(bar0 + 8 * i, bar0 + 8 * i == p_full ? kSoftmaxWarps : 1);
    fence_barrier_init();
  }
  if (warp == kSoftmaxWarps) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;                    // S in columns [0, 128); O in [0, 64) after softmax
  pdl_trigger();                                       // after taking TMEM

  bool ok = true;
  if (warp == kSoftmaxWarps) {
    if (lane == 0 && n > 0) {
      prefetch_tmap(&tm_qkv);
      mbar_arrive_expect_tx(qk_full, 2 * kTileBytes);
      tma_load_2d(&tm_qkv, sbase + kQ, qk_full, coord_x(0), coord_y(0, 0));
      tma_load_2d(&tm_qkv, sbase + kK, qk_full, coord_x(1), coord_y(1, 0));
      mbar_arrive_expect_tx(v_full, kTileBytes);
      tma_load_2d(&tm_qkv, sbase + kV, v_full, coord_x(2), coord_y(2, 0));
      constexpr uint32_t idesc_s = idesc_f16_f32(kRows, kRows);
      constexpr uint32_t idesc_o = idesc_f16_f32_bmn(kRows, kD);
      if (mbar_wait(qk_full, 0, kWaitLimitNs)) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk)
          mma_f16_ss(tmem, smem_desc_sw128(sbase + kQ + kk * 32), smem_desc_sw128(sbase + kK + kk * 32), idesc_s,
                     kk > 0 ? 1u : 0u);
        mma_commit(s_full);
        // P written by the softmax warps (which have read all of S and zeroed
        // the V rows of keys >= n).
        if (mbar_wait(p_full, 0, kWaitLimitNs) && mbar_wait(v_full, 0, kWaitLimitNs)) {
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kRows / 16; ++kk)
            mma_f16_ss(tmem, smem_desc_sw128(sbase + kP + (kk >> 2) * kTileBytes + (kk & 3) * 32),
                       desc_mn_sw128(sbase + kV + kk * 16 * 128), idesc_o, kk > 0 ? 1u : 0u);
          mma_commit(o_full);
        } else {
          ok = false;
        }
      } else {
        ok = false;
      }
      mma_commit(drain);                               // every MMA issued here has completed
      mbar_wait(drain, 0, kWaitLimitNs);
      if (!ok) {                                       // let the copies land before the CTA exits
        mbar_wait(qk_full, 0, kWaitLimitNs);
        mbar_wait(v_full, 0, kWaitLimitNs);
      }
    }
  } else {
    const int r = warp * 32 + lane;                    // query row = TMEM lane
    const uint32_t t_row = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const int nchunks = (n + 31) >> 5;                 // 32-key chunks holding valid keys
    uint8_t* prow = smem + kP + r * 128;
    uint32_t sa[32], sb[32];                           // two chunks: one in use, one loading
    uint64_t sum2 = 0;                                 // two partial row sums (0.0f, 0.0f)
    if (n > 0) {
      ok = warp_wait(s_full, 0);
      if (ok) {
        tc_fence_after();
        // Pass 1: row max over the valid keys.  The next chunk's TMEM load is
        // in flight while the current one is scanned.
        float mx = -INFINITY;
        tmem_ld_32x32b_x32_async(t_row, sa);
#pragma unroll
        for (int c = 0; c < kRows / 32; ++c) {
          if (c < nchunks) {
            uint32_t(&cur)[32] = (c & 1) ? sb : sa;
            uint32_t(&nxt)[32] = (c & 1) ? sa : sb;
            tmem_wait_ld(cur);
            if (c + 1 < nchunks) tmem_ld_32x32b_x32_async(t_row + 32 * (c + 1), nxt);
            const int lim = n - 32 * c;
            if (lim >= 32) {
#pragma unroll
              for (int i = 0; i < 32; ++i) mx = fmaxf(mx, __uint_as_float(cur[i]));
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (i < lim) mx = fmaxf(mx, __uint_as_float(cur[i]));
            }
          }
        }
        const uint64_t scale2 = f2_pack(score_scale_log2, score_scale_log2);
        const uint64_t neg_m2 = f2_pack(-mx * score_scale_log2, -mx * score_scale_log2);
        // Pass 2: P, its row sum, FP16 P into the swizzled tile (over Q and K);
        // chunks past n get P = 0.
        tmem_ld_32x32b_x32_async(t_row, sa);
#pragma unroll
        for (int c = 0; c < kRows / 32; ++c) {
          if (c < nchunks) {
            uint32_t(&cur)[32] = (c & 1) ? sb : sa;
            uint32_t(&nxt)[32] = (c & 1) ? sa : sb;
            tmem_wait_ld(cur);
            if (c + 1 < nchunks) tmem_ld_32x32b_x32_async(t_row + 32 * (c + 1), nxt);
            const int lim = n - 32 * c;
            if (lim >= 32)
              p_chunk<false>(cur, 32, scale2, neg_m2, sum2, prow, c, r);
            else
              p_chunk<true>(cur, lim, scale2, neg_m2, sum2, prow, c, r);
          } else {
#pragma unroll
            for (int u = 0; u < 4; ++u) store_p_unit(prow, 4 * c + u, r, make_uint4(0, 0, 0, 0));
          }
        }
        // V rows of keys >= n: their P is 0, but a row the TMA box brought in
        // from outside the sequence may hold non-finite data (0 * NaN = NaN in
        // the MMA), so zero them.  Row r of the tile is key r.
        if (n < kRows) {
          ok = warp_wait(v_full, 0);
          if (ok && r >= n) {
            uint4* vrow = reinterpret_cast<uint4*>(smem + kV + r * 128);
#pragma unroll
            for (int u = 0; u < 8; ++u) vrow[u] = make_uint4(0, 0, 0, 0);
          }
        }
        fence_proxy_async_smem();                      // P (and zeroed V rows) visible to the tensor core
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
        if (ok) ok = warp_wait(o_full, 0);
      }
    }
    if (ok) {
      // Row r of O, scaled by 1/sum, as FP16 into the V tile (free once P V has
      // completed): 128 bytes per row, 16-byte units swizzled by r & 7.
      tc_fence_after();
      float s0, s1;
      f2_unpack(sum2, s0, s1);
      const float l = s0 + s1;
      const float inv = l > 0.f ? 1.f / l : 0.f;       // n == 0: ctx = 0
      const uint64_t inv2 = f2_pack(inv, inv);
      uint8_t* orow = smem + kV + r * 128;
      if (n > 0) {
        tmem_ld_32x32b_x32_async(t_row, sa);
        tmem_ld_32x32b_x32_async(t_row + 32, sb);
        tmem_wait_ld(sa);
        tmem_wait_ld(sb);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) sa[i] = sb[i] = 0u;
      }
#pragma unroll
      for (int c = 0; c < kD / 32; ++c) {
        const uint32_t(&sv)[32] = c ? sb : sa;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint32_t w[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            float o0, o1;
            f2_unpack(f2_mul(f2_pack(__uint_as_float(sv[8 * u + 2 * j]), __uint_as_float(sv[8 * u + 2 * j + 1])),
                             inv2),
                      o0, o1);
            w[j] = cvt_half2(o0, o1);
          }
          const int unit = 4 * c + u;
          *reinterpret_cast<uint4*>(orow + 16 * (unit ^ (r & 7))) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      __syncwarp();
      // The warp's 32 rows, stored coalesced: 8 lanes per 128-byte row, 4 rows
      // per instruction.
      const int unit = lane & 7;
#pragma unroll 1
      for (int it = 0; it < 8; ++it) {
        const int rr = warp * 32 + it * 4 + (lane >> 3);
        if (rr < rows_exist) {
          const uint4 v = *reinterpret_cast<const uint4*>(smem + kV + rr * 128 + 16 * (unit ^ (rr & 7)));
          const size_t out_row = PACKED ? (size_t)offsets[b] + rr : (size_t)b * S + rr;
          *reinterpret_cast<uint4*>(ctx + out_row * H + h * kD + unit * 8) = v;
        }
      }
    }
  }

  if (!ok) atomicCAS(status, 0, kStatusWaitTimeout);
  tc_fence_before();
  __syncthreads();
  if (warp == kSoftmaxWarps) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

template <bool PACKED>
cudaError_t launch_tc(const __half* qkv, const int32_t* vl, const int32_t* offsets, __half* ctx, int B, int S,
                      int NH, int* status, cudaStream_t stream) {
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  std::call_once(once, [] {
    attr = cudaFuncSetAttribute(attention_tc_kernel<PACKED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kSmemTotal);
  });
  if (attr != cudaSuccess) return attr;
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  // Rows of 64 halves: the split layout has 3*B*nh*S of them; the packed
  // layout is [B*S (most tokens), 3H].
  const uint64_t H = (uint64_t)NH * kD;
  cuuint64_t dims[2], strides[1];
  if (PACKED) {
    dims[0] = 3 * H; dims[1] = (uint64_t)B * S; strides[0] = 3 * H * 2;
  } else {
    dims[0] = kD; dims[1] = 3ull * B * NH * S; strides[0] = kD * 2;
  }
  const cuuint32_t box[2] = {kD, kRows};
  const cuuint32_t estr[2] = {1, 1};
  CUtensorMap map;
  if (fn(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<__half*>(qkv), dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const dim3 grid(NH, B);
  const float scale_log2 = kLog2e / sqrtf((float)kD);
  return launch_kernel(attention_tc_kernel<PACKED>, grid, dim3(kThreads), kSmemTotal, stream, nullptr, 0, map, vl,
                       offsets, ctx, B, S, NH, scale_log2, status);
}

}  // namespace

bool attention_tc_supported(int size_per_head, int seq) { return size_per_head == kD && seq > 64 && seq <= kRows; }

cudaError_t launch_attention_tc(const __half* qkv, const int32_t* valid_len, const int32_t* offsets, __half* ctx,
                                int batch, int seq, int head_num, int* status, cudaStream_t stream) {
  if (batch <= 0 || batch > 65535 || head_num <= 0 || head_num > 65535 || !attention_tc_supported(kD, seq))
    return cudaErrorInvalidValue;
  if (offsets) return launch_tc<true>(qkv, valid_len, offsets, ctx, batch, seq, head_num, status, stream);
  return launch_tc<false>(qkv, valid_len, nullptr, ctx, batch, seq, head_num, status, stream);
}

}  // namespace enc
