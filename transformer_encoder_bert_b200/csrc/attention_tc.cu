// Masked scaled-dot-product attention on the 5th-generation tensor cores
// (tcgen05 + TMEM + TMA) for size_per_head 64 and seq > 64.  Two kernels:
// attention_tc_kernel for seq <= 128, where one block of 128 keys covers every
// key of a sequence (described here), and attention_tc_long_kernel for longer
// sequences (described where it is defined).
//
// The source page ("Faster Transformer 优化原理") runs attention as two batched
// GEMMs around a SoftMax kernel.  Here both products run on tcgen05 and the
// score tile never leaves the SM.  The one-block kernel is persistent: about
// four CTAs per SM, each taking (sequence, head) items in turn, 160 threads:
//   warps 0..3  softmax: thread r owns query row r = TMEM lane r.  It reads its
//               row of S from TMEM, takes the row max over the valid keys (the
//               row is in one thread: no shuffles), forms
//               P = exp(S/sqrt(d) - max) in FP32, sums it, and writes P as FP16
//               back into TMEM over the scores it has read.  After P V it
//               scales its row of O by 1/sum and stores it.
//   warp 4      one thread issues the TMA loads of Q, K and V and the MMAs
//                 S = Q K^T   M=128, N=128, K=64  (A, B K-major, both in smem)
//                 O = P V     M=128, N=64,  K=16 per valid 16-key group (A = P
//                             read from TMEM; B = V read MN-major straight from
//                             its token-major tile)
// The valid length n is the same for every row of an item, so every masking
// decision is a warp-uniform branch: 32-key chunks wholly past n are skipped,
// chunks wholly inside n run unmasked, and at most one chunk is masked per
// element.  Keys j >= n get weight exactly 0.
//
// P in TMEM frees the Q and K tiles as soon as S = Q K^T has completed, so the
// next item's Q and K load while this item's softmax, P V and output run; its
// V loads once the output rows staged in the V tile have been read by their
// TMA stores.  TMEM: S in columns [0, 128), P (two halves per column) over
// [0, 64), O in [64, 128); the next S waits until O has been read.  Footprint
// per CTA: 48 KB of tiles and 128 TMEM columns.  Every mbarrier wait is
// bounded in time.
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

// Shared memory of the one-block kernel (offsets from a 1024-byte-aligned base).
constexpr int kQ = 0;                             // Q tile
constexpr int kK = kTileBytes;                    // K tile
constexpr int kV = 2 * kTileBytes;                // V tile, then the output rows
constexpr int kBars = 3 * kTileBytes;
// qk_full, v_full, s_full, p_full, o_full, o_free, v_free, drain
constexpr int kNumBars = 8;
constexpr int kSlot = kBars + kNumBars * 8;
constexpr int kSmemTotal = 1024 + kSlot + 16;
constexpr int kOCol = 64;                         // O's TMEM columns [64, 128)
constexpr int kCtasPerSm = 4;                     // TMEM 4 x 128 columns, shared memory 4 x 50 KB
static_assert(kCtasPerSm * (kSmemTotal + 1024) <= 228 * 1024, "four CTAs per SM");

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

// P of 32 keys (chunk c of the row) from 32 raw scores: p = 2^(s*c2 - m*c2)
// for the first `lim` keys, 0 for the rest; adds to the pair sum and writes
// the FP16 values into TMEM as 16 columns (two keys per column) of this lane.
template <bool MASKED>
__device__ __forceinline__ void p_chunk_tmem(const uint32_t (&sv)[32], int lim, uint64_t scale2, uint64_t neg_m2,
                                             uint64_t& sum2, uint32_t t_p) {
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
  tmem_st_32x32b_x16_async(t_p, pk);
}

template <bool PACKED>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    attention_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv, const int32_t* __restrict__ valid_len,
                        const int32_t* __restrict__ offsets, __half* __restrict__ ctx, int B, int S, int NH,
                        float score_scale_log2, const __grid_constant__ CUtensorMap tm_ctx,
                        int* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + kBars;
  const uint32_t qk_full = bar0, v_full = bar0 + 8, s_full = bar0 + 16, p_full = bar0 + 24, o_full = bar0 + 32,
                 o_free = bar0 + 40, v_free = bar0 + 48, drain = bar0 + 56;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kSlot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = NH * kD;
  const int items = B * NH;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) {
      const uint32_t bar = bar0 + 8 * i;
      mbar_init(bar, (bar == p_full || bar == o_free || bar == v_free) ? kSoftmaxWarps : 1);
    }
    fence_barrier_init();
  }
  if (warp == kSoftmaxWarps) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;                    // S [0, 128); P over [0, 64); O [64, 128)
  pdl_wait();                                          // Q/K/V (and offsets) of the previous kernels are visible
  pdl_trigger();                                       // after taking TMEM

  // Item i is (sequence B-1-i/nh, head i%nh): the sequences are taken last to
  // first, since the QKV GEMM before this kernel writes the rows of the last
  // sequences last, so those are the ones still in L2.
  auto seq_of = [&](int item) { return B - 1 - item / NH; };
  auto seq_len = [&](int item) {
    const int n = valid_len[seq_of(item)];
    return n < 0 ? 0 : (n > S ? S : n);
  };
  // Tensor-map coordinates of row 0 of block t (0 = Q, 1 = K, 2 = V).
  auto coord_x = [&](int t, int h) { return PACKED ? t * H + h * kD : 0; };
  auto coord_y = [&](int t, int b, int h) { return PACKED ? offsets[b] : ((t * B + b) * NH + h) * S; };

  bool ok = true;
  if (warp == kSoftmaxWarps) {
    if (lane == 0) {
      prefetch_tmap(&tm_qkv);
      prefetch_tmap(&tm_ctx);
      constexpr uint32_t idesc_s = idesc_f16_f32(kRows, kRows);
      constexpr uint32_t idesc_o = idesc_f16_f32_bmn(kRows, kD);
      const int G = static_cast<int>(gridDim.x);
      auto next_loaded = [&](int item) {                // items with no valid key load nothing
        while (item < items && seq_len(item) == 0) item += G;
        return item;
      };
      auto load_qk = [&](int item) {
        const int b = seq_of(item), h = item % NH;
        mbar_arrive_expect_tx(qk_full, 2 * kTileBytes);
        tma_load_2d(&tm_qkv, sbase + kQ, qk_full, coord_x(0, h), coord_y(0, b, h));
        tma_load_2d(&tm_qkv, sbase + kK, qk_full, coord_x(1, h), coord_y(1, b, h));
      };
      auto load_v = [&](int item) {
        const int b = seq_of(item), h = item % NH;
        mbar_arrive_expect_tx(v_full, kTileBytes);
        tma_load_2d(&tm_qkv, sbase + kV, v_full, coord_x(2, h), coord_y(2, b, h));
      };
      // Copies issued and not yet waited for, with the parity they complete.
      int qk_pending = -1, v_pending = -1;
      int cur = next_loaded(blockIdx.x);
      if (cur < items) {
        load_qk(cur);
        load_v(cur);
        qk_pending = v_pending = 0;
      }
      for (int it = 0; cur < items; ++it) {
        const uint32_t ph = it & 1;
        const int n = seq_len(cur);
        const int nxt = next_loaded(cur + G);
        if (!(ok = mbar_wait(qk_full, ph, kWaitLimitNs))) break;
        qk_pending = -1;
        // S goes into the columns that held the previous item's O.
        if (it > 0 && !(ok = mbar_wait(o_free, ph ^ 1, kWaitLimitNs))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk)
          mma_f16_ss(tmem, smem_desc_sw128(sbase + kQ + kk * 32), smem_desc_sw128(sbase + kK + kk * 32), idesc_s,
                     kk > 0 ? 1u : 0u);
        mma_commit(s_full);
        if (it > 0) {                                    // the V tile held the previous item's output rows
          if (!(ok = mbar_wait(v_free, ph ^ 1, kWaitLimitNs))) break;
          load_v(cur);
          v_pending = ph;
        }
        if (nxt < items) {                               // the next Q and K, once S = Q K^T has read these
          if (!(ok = mbar_wait(s_full, ph, kWaitLimitNs))) break;
          load_qk(nxt);
          qk_pending = ph ^ 1;
        }
        // P written to TMEM by the softmax warps (which have read all of S and
        // zeroed the V rows of keys in [n, n rounded up to 16)).
        if (!(ok = mbar_wait(p_full, ph, kWaitLimitNs))) break;
        if (!(ok = mbar_wait(v_full, ph, kWaitLimitNs))) break;
        v_pending = -1;
        tc_fence_after();
        const int ksteps = (n + 15) >> 4;                // key groups of 16 holding valid keys
        for (int kk = 0; kk < ksteps; ++kk)
          mma_f16_ts(tmem + kOCol, tmem + 8 * kk, desc_mn_sw128(sbase + kV + kk * 16 * 128), idesc_o,
                     kk > 0 ? 1u : 0u);
        mma_commit(o_full);
        cur = nxt;
      }
      mma_commit(drain);                                 // every MMA issued here has completed
      mbar_wait(drain, 0, kWaitLimitNs);
      // After a failed wait, let the copies in flight land before the CTA exits.
      if (qk_pending >= 0) mbar_wait(qk_full, qk_pending, kWaitLimitNs);
      if (v_pending >= 0) mbar_wait(v_full, v_pending, kWaitLimitNs);
    }
  } else {
    const int r = warp * 32 + lane;                      // query row = TMEM lane
    const uint32_t t_row = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const int unit = lane & 7;                           // plain stores: 8 lanes per 128-byte row
    uint32_t sa[32], sb[32];                             // two chunks: one in use, one loading
    int it = 0;
    for (int item = blockIdx.x; item < items; item += gridDim.x) {
      const int b = seq_of(item), h = item % NH;
      const int n = seq_len(item);
      if (n == 0) {                                      // no valid key: ctx = 0 (packed: no rows)
        if (!PACKED) {
          __half* out = ctx + (size_t)b * S * H + h * kD;
#pragma unroll 1
          for (int k = 0; k < 8; ++k) {
            const int rr = warp * 32 + k * 4 + (lane >> 3);
            if (rr < S) *reinterpret_cast<uint4*>(out + (size_t)rr * H + unit * 8) = make_uint4(0, 0, 0, 0);
          }
        }
        continue;
      }
      const uint32_t ph = it & 1;
      ++it;
      const int nchunks = (n + 31) >> 5;                 // 32-key chunks holding valid keys
      uint64_t sum2 = 0;                                 // two partial row sums (0.0f, 0.0f)
      if (!(ok = warp_wait(s_full, ph))) break;
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
      // Pass 2: P and its row sum; FP16 P of chunk c goes to columns
      // [16c, 16c + 16), which hold scores this thread has already read.
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
            p_chunk_tmem<false>(cur, 32, scale2, neg_m2, sum2, t_row + 16 * c);
          else
            p_chunk_tmem<true>(cur, lim, scale2, neg_m2, sum2, t_row + 16 * c);
        }
      }
      // P V reads the keys of the 16-key groups holding valid keys.  Keys in
      // [n, n16) have P = 0, but a V row the TMA box brought in from outside the
      // sequence may hold non-finite data (0 * NaN = NaN in the MMA), so they
      // are zeroed; those rows all lie in warp n / 32.  Row r of the tile is key r.
      const int n16 = (n + 15) & ~15;
      if (n < n16 && warp == (n >> 5)) {
        if (!(ok = warp_wait(v_full, ph))) break;
        if (r >= n && r < n16) {
          uint4* vrow = reinterpret_cast<uint4*>(smem + kV + r * 128);
#pragma unroll
          for (int u = 0; u < 8; ++u) vrow[u] = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();                        // zeroed V rows visible to the tensor core
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
      if (!(ok = warp_wait(o_full, ph))) break;
      tc_fence_after();
      tmem_ld_32x32b_x32_async(t_row + kOCol, sa);
      tmem_ld_32x32b_x32_async(t_row + kOCol + 32, sb);
      tmem_wait_ld(sa);
      tmem_wait_ld(sb);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_free);                // the next S may overwrite O
      // Row r of O, scaled by 1/sum, as FP16 into the V tile (free once P V has
      // completed): 128 bytes per row, 16-byte units swizzled by r & 7, the
      // layout of a 128-byte-swizzled TMA box.
      float s0, s1;
      f2_unpack(sum2, s0, s1);
      const float inv = 1.f / (s0 + s1);                 // n > 0: the sum holds P = 1 at the row max
      const uint64_t inv2 = f2_pack(inv, inv);
      uint8_t* orow = smem + kV + r * 128;
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
          const int un = 4 * c + u;
          *reinterpret_cast<uint4*>(orow + 16 * (un ^ (r & 7))) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      fence_proxy_async_smem();                          // the rows visible to the TMA store
      __syncwarp();
      // The warp's 32 rows: one TMA store when all of them exist; else the rows
      // that do, stored coalesced (8 lanes per 128-byte row, 4 rows per
      // instruction).  The V tile is released once the rows have been read.
      const int rows_exist = PACKED ? n : S;
      const int row0 = PACKED ? offsets[b] : b * S;
      if (warp * 32 + 32 <= rows_exist) {
        if (lane == 0) {
          tma_store_2d(&tm_ctx, sbase + kV + warp * 32 * 128, h * kD, row0 + warp * 32);
          bulk_commit_group();
          bulk_wait_group_read<0>();
        }
      } else {
        __half* out = ctx + (size_t)row0 * H + h * kD;
#pragma unroll 1
        for (int k = 0; k < 8; ++k) {
          const int rr = warp * 32 + k * 4 + (lane >> 3);
          if (rr < rows_exist) {
            const uint4 v = *reinterpret_cast<const uint4*>(smem + kV + rr * 128 + 16 * (unit ^ (rr & 7)));
            *reinterpret_cast<uint4*>(out + (size_t)rr * H + unit * 8) = v;
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(v_free);
    }
    if (lane == 0) bulk_wait_group_all();                // this warp's TMA stores have completed
  }

  if (!ok) atomicCAS(status, 0, kStatusWaitTimeout);
  tc_fence_before();
  __syncthreads();
  if (warp == kSoftmaxWarps) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Sequences longer than one key block (seq > 128): the same per-row softmax
// over key blocks of 32 with a reference maximum (online softmax).  One CTA per
// (sequence, head, 128 query rows), 160 threads, four CTAs per SM:
//   warps 0..3  softmax: thread r owns query row r = TMEM lane r.  For key
//               block j it reads its row of S_j = Q K_j^T from TMEM, writes
//               P_j = exp(S_j/sqrt(d) - m) as FP16 back into S_j's columns and
//               adds its row sum to l.  m is a reference maximum: it moves only
//               when a block's maximum exceeds it by more than 2^8 in the
//               exponent, and then O (in TMEM) and l are scaled by
//               exp(m_old - m_new) before the next P V accumulates.  At the end
//               it stores O / l.
//   warp 4      one thread issues every TMA load (Q once; K and V blocks
//               through four-stage rings) and every MMA:
//                 S_j = Q K_j^T   M=128, N=32, K=64 into S buffer j % 2
//                 O += P_j V_j    M=128, N=64, K=16 per 16-key group (A = P_j
//                                 read from TMEM; B = V_j MN-major from smem)
// The two S buffers let S_{j+1} be computed while the softmax warps work on
// S_j, and S_{j+2} goes into S_j's buffer as soon as P_j V_j has read P_j.
// TMEM (128 columns): S buffers at [0, 32) and [32, 64), P_j (two halves per
// column) over the first 16 columns of its buffer, O at [64, 128).  Key blocks
// past n are never loaded; in the last block, keys >= n get weight 0 and the
// V rows of keys in [n, n rounded up to 16) are zeroed.
namespace lng {
constexpr int kThreads = 32 * (kSoftmaxWarps + 1);
constexpr int kBK = 32;                                     // keys per block
constexpr int kStages = 4;                                  // K and V ring depth
constexpr int kKVBytes = kBK * kD * 2;                      // 4 KB: 32 keys x 64 halves
constexpr int kQ = 0;                                       // Q tile, later the output rows
constexpr int kK = kTileBytes;                              // K stages
constexpr int kV = kK + kStages * kKVBytes;                 // V stages
constexpr int kBars = kV + kStages * kKVBytes;
// q_full, k_full[4], v_full[4], s_full[2], p_full[2], o_done, drain
constexpr int kNumBars = 15;
constexpr int kSlot = kBars + kNumBars * 8;
constexpr int kSmemTotal = 1024 + kSlot + 16;
constexpr int kTmemCols = 128;
constexpr int kOCol = 2 * kBK;
constexpr int kCtasPerSm = 4;                               // TMEM 4 x 128 columns
constexpr float kRescaleLog2 = 8.f;                         // P < 2^8 between rescales
static_assert(kCtasPerSm * (kSmemTotal + 1024) <= 228 * 1024, "four CTAs per SM");
}  // namespace lng

template <bool PACKED>
__global__ void __launch_bounds__(lng::kThreads, lng::kCtasPerSm)
    attention_tc_long_kernel(const __grid_constant__ CUtensorMap tm_qkv, const __grid_constant__ CUtensorMap tm_kv,
                             const int32_t* __restrict__ valid_len, const int32_t* __restrict__ offsets,
                             __half* __restrict__ ctx, int B, int S, int NH, float score_scale_log2,
                             int* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + lng::kBars;
  const uint32_t q_full = bar0, o_done = bar0 + 104, drain = bar0 + 112;
  auto k_full = [&](int st) { return bar0 + 8 + 8 * st; };
  auto v_full = [&](int st) { return bar0 + 40 + 8 * st; };
  auto s_full = [&](int bf) { return bar0 + 72 + 8 * bf; };
  auto p_full = [&](int bf) { return bar0 + 88 + 8 * bf; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + lng::kSlot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, b = B - 1 - (int)blockIdx.z;   // last sequences first, as above
  const int q0 = blockIdx.x * kRows;
  pdl_wait();
  int n = valid_len[b];
  n = n < 0 ? 0 : (n > S ? S : n);
  const int rows_exist = PACKED ? n : S;
  if (q0 >= rows_exist) return;                        // no query rows here (uniform per CTA)
  const int H = NH * kD;
  const size_t row0 = PACKED ? (size_t)offsets[b] : (size_t)b * S;
  if (n == 0) {                                        // fixed-length layout, empty sequence: ctx = 0
    const int rows = min(kRows, S - q0);
    for (int i = threadIdx.x; i < rows * 8; i += lng::kThreads)
      *reinterpret_cast<uint4*>(ctx + (row0 + q0 + (i >> 3)) * H + h * kD + (i & 7) * 8) = make_uint4(0, 0, 0, 0);
    return;
  }
  const int nb = (n + lng::kBK - 1) / lng::kBK;        // key blocks holding valid keys

  auto coord_x = [&](int t) { return PACKED ? t * H + h * kD : 0; };
  auto coord_y = [&](int t, int s) { return PACKED ? offsets[b] + s : ((t * B + b) * NH + h) * S + s; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < lng::kNumBars; ++i) {
      const uint32_t bar = bar0 + 8 * i;
      mbar_init(bar, (bar == p_full(0) || bar == p_full(1)) ? kSoftmaxWarps : 1);
    }
    fence_barrier_init();
  }
  if (warp == kSoftmaxWarps) {
    tmem_alloc(smem_u32(tmem_slot), lng::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_trigger();                                       // after taking TMEM

  bool ok = true;
  if (warp == kSoftmaxWarps) {
    if (lane == 0) {
      prefetch_tmap(&tm_qkv);
      prefetch_tmap(&tm_kv);
      // K_j and V_j go to stage j % kStages (one key block per box, same rows as the Q map).
      auto load_k = [&](int j) {
        const int st = j % lng::kStages;
        mbar_arrive_expect_tx(k_full(st), lng::kKVBytes);
        tma_load_2d(&tm_kv, sbase + lng::kK + st * lng::kKVBytes, k_full(st), coord_x(1), coord_y(1, j * lng::kBK));
      };
      auto load_v = [&](int j) {
        const int st = j % lng::kStages;
        mbar_arrive_expect_tx(v_full(st), lng::kKVBytes);
        tma_load_2d(&tm_kv, sbase + lng::kV + st * lng::kKVBytes, v_full(st), coord_x(2), coord_y(2, j * lng::kBK));
      };
      mbar_arrive_expect_tx(q_full, kTileBytes);
      tma_load_2d(&tm_qkv, sbase + lng::kQ, q_full, coord_x(0), coord_y(0, q0));
      for (int j = 0; j < nb && j < lng::kStages; ++j) {
        load_k(j);
        load_v(j);
      }
      int loaded = nb < lng::kStages ? nb : lng::kStages;   // K and V blocks requested
      constexpr uint32_t idesc_s = idesc_f16_f32(kRows, lng::kBK);
      constexpr uint32_t idesc_o = idesc_f16_f32_bmn(kRows, kD);
      auto issue_s = [&](int j) {                      // S_j into buffer j % 2
        const int st = j % lng::kStages;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk)
          mma_f16_ss(tmem + (j & 1) * lng::kBK, smem_desc_sw128(sbase + lng::kQ + kk * 32),
                     smem_desc_sw128(sbase + lng::kK + st * lng::kKVBytes + kk * 32), idesc_s, kk > 0 ? 1u : 0u);
        mma_commit(s_full(j & 1));
      };
      ok = mbar_wait(q_full, 0, kWaitLimitNs);
      for (int j = 0; j < 2 && j < nb && ok; ++j) {
        if (!(ok = mbar_wait(k_full(j), 0, kWaitLimitNs))) break;
        tc_fence_after();
        issue_s(j);
      }
      for (int j = 0; j < nb && ok; ++j) {
        const int st = j % lng::kStages;
        const uint32_t rph = (j / lng::kStages) & 1;
        // P_j is written (so S_j has been read and O rescaled) and V_j has landed.
        if (!(ok = mbar_wait(p_full(j & 1), (j >> 1) & 1, kWaitLimitNs))) break;
        if (!(ok = mbar_wait(v_full(st), rph, kWaitLimitNs))) break;
        tc_fence_after();
        const int lim_blk = min(n - j * lng::kBK, lng::kBK);
        const int ksteps = (lim_blk + 15) >> 4;
        for (int kk = 0; kk < ksteps; ++kk)            // O += P_j V_j
          mma_f16_ts(tmem + lng::kOCol, tmem + (j & 1) * lng::kBK + 8 * kk,
                     desc_mn_sw128(sbase + lng::kV + st * lng::kKVBytes + kk * 16 * 128), idesc_o,
                     (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(o_done);
        if (j + 2 < nb) {
          // P_j V_j has read P_j (S_j's buffer is free) and V_j (its stage is free);
          // S_j, long complete, has read K_j.
          if (!(ok = mbar_wait(o_done, j & 1, kWaitLimitNs))) break;
          if (j + lng::kStages < nb) {
            load_k(j + lng::kStages);
            load_v(j + lng::kStages);
            loaded = j + lng::kStages + 1;
          }
          if (j + 2 < nb) {
            const int st2 = (j + 2) % lng::kStages;
            if (!(ok = mbar_wait(k_full(st2), ((j + 2) / lng::kStages) & 1, kWaitLimitNs))) break;
            tc_fence_after();
            issue_s(j + 2);
          }
        }
      }
      mma_commit(drain);                               // every MMA issued here has completed
      mbar_wait(drain, 0, kWaitLimitNs);
      if (!ok) {                                       // let the copies land before the CTA exits
        mbar_wait(q_full, 0, kWaitLimitNs);
        for (int j = loaded > lng::kStages ? loaded - lng::kStages : 0; j < loaded; ++j) {
          mbar_wait(k_full(j % lng::kStages), (j / lng::kStages) & 1, kWaitLimitNs);
          mbar_wait(v_full(j % lng::kStages), (j / lng::kStages) & 1, kWaitLimitNs);
        }
      }
    }
  } else {
    const int r = warp * 32 + lane;                    // query row = TMEM lane
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const uint32_t t_o = t_lane + lng::kOCol;
    const uint64_t scale2 = f2_pack(score_scale_log2, score_scale_log2);
    uint32_t sa[32], sb[32];
    uint64_t sum2 = 0;                                 // two partial row sums (0.0f, 0.0f)
    float m_ref = 0.f;                                 // the max that P, O and l are taken against
    for (int j = 0; j < nb && ok; ++j) {
      const uint32_t t_s = t_lane + (j & 1) * lng::kBK;
      if (!(ok = warp_wait(s_full(j & 1), (j >> 1) & 1))) break;
      tc_fence_after();
      const int lim_blk = min(n - j * lng::kBK, lng::kBK);   // valid keys in this block (>= 1)
      // The block's 32 scores of this row in registers.
      tmem_ld_32x32b_x32(t_s, sa);
      float bmax = -INFINITY;
      if (lim_blk >= lng::kBK) {
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int i = 0; i < 32; ++i) m4[i & 3] = fmaxf(m4[i & 3], __uint_as_float(sa[i]));
        bmax = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (i < lim_blk) bmax = fmaxf(bmax, __uint_as_float(sa[i]));
      }
      // Every P, and every term of O and l, is taken against the same reference
      // m, so O / l is the softmax-weighted sum whatever m is; m moves (and O and
      // l are rescaled by alpha = exp(m_old - m_new)) only to keep P below 2^8.
      float alpha = 1.f;
      bool moved = false;
      if (j == 0) {
        m_ref = bmax;
      } else if ((bmax - m_ref) * score_scale_log2 > lng::kRescaleLog2) {
        alpha = ex2((m_ref - bmax) * score_scale_log2);
        m_ref = bmax;
        moved = true;
      }
      if (__any_sync(0xffffffffu, moved)) {            // O *= alpha (alpha = 1 on rows that keep theirs)
        if (!(ok = warp_wait(o_done, (j - 1) & 1))) break;   // P_{j-1} V_{j-1} has completed
        tc_fence_after();
        uint32_t oa[32];
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          tmem_ld_32x32b_x32(t_o + 32 * half, oa);
#pragma unroll
          for (int i = 0; i < 32; ++i) oa[i] = __float_as_uint(__uint_as_float(oa[i]) * alpha);
          tmem_st_32x32b_x32(t_o + 32 * half, oa);
        }
      }
      sum2 = f2_mul(sum2, f2_pack(alpha, alpha));
      const uint64_t neg_m2 = f2_pack(-m_ref * score_scale_log2, -m_ref * score_scale_log2);
      // P_j and its row sum; FP16 P goes to the first 16 columns of S_j's
      // buffer, which hold scores this thread has already read.
      if (lim_blk >= lng::kBK) {
        p_chunk_tmem<false>(sa, 32, scale2, neg_m2, sum2, t_s);
      } else {
        p_chunk_tmem<true>(sa, lim_blk, scale2, neg_m2, sum2, t_s);
        // V rows of keys in [lim_blk, lim_blk rounded up to 16) are read by
        // P V; a row the TMA box brought in from outside the sequence may hold
        // non-finite data (0 * NaN = NaN in the MMA), so zero them.  Those rows
        // of the 32-row V tile are rows of warp 0.
        const int n16 = (lim_blk + 15) & ~15;
        if (lim_blk < n16 && warp == 0) {
          if (!(ok = warp_wait(v_full(j % lng::kStages), (j / lng::kStages) & 1))) break;
          if (r >= lim_blk && r < n16) {
            uint4* vrow = reinterpret_cast<uint4*>(smem + lng::kV + (j % lng::kStages) * lng::kKVBytes + r * 128);
#pragma unroll
            for (int u = 0; u < 8; ++u) vrow[u] = make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();                    // zeroed V rows visible to the tensor core
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full(j & 1));
    }
    if (ok) {
      ok = warp_wait(o_done, (nb - 1) & 1);
      if (ok) {
        tc_fence_after();
        tmem_ld_32x32b_x32_async(t_o, sa);
        tmem_ld_32x32b_x32_async(t_o + 32, sb);
        tmem_wait_ld(sa);
        tmem_wait_ld(sb);
      }
    }
    if (ok) {
      // Row r of O / l as FP16 into the Q tile (its last reader, the MMA of
      // the last S, has completed), then coalesced stores.
      float s0, s1;
      f2_unpack(sum2, s0, s1);
      const float inv = 1.f / (s0 + s1);               // n >= 1: the sum holds P = 1 at the first block's max
      uint8_t* orow = smem + lng::kQ + r * 128;
#pragma unroll
      for (int unit = 0; unit < 8; ++unit) {
        const uint32_t(&sv)[32] = unit < 4 ? sa : sb;
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int i = 8 * (unit & 3) + 2 * k;
          w[k] = cvt_half2(__uint_as_float(sv[i]) * inv, __uint_as_float(sv[i + 1]) * inv);
        }
        *reinterpret_cast<uint4*>(orow + 16 * (unit ^ (r & 7))) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      __syncwarp();
      const int unit = lane & 7;
#pragma unroll 1
      for (int it = 0; it < 8; ++it) {
        const int rr = warp * 32 + it * 4 + (lane >> 3);
        if (q0 + rr < rows_exist) {
          const uint4 v = *reinterpret_cast<const uint4*>(smem + lng::kQ + rr * 128 + 16 * (unit ^ (rr & 7)));
          *reinterpret_cast<uint4*>(ctx + (row0 + q0 + rr) * H + h * kD + unit * 8) = v;
        }
      }
    }
  }

  if (!ok) atomicCAS(status, 0, kStatusWaitTimeout);
  tc_fence_before();
  __syncthreads();
  if (warp == kSoftmaxWarps) {
    tc_fence_after();
    tmem_dealloc(tmem, lng::kTmemCols);
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
    if (attr == cudaSuccess)
      attr = cudaFuncSetAttribute(attention_tc_long_kernel<PACKED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  lng::kSmemTotal);
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
  const float scale_log2 = kLog2e / sqrtf((float)kD);
  if (S > kRows) {
    // K and V blocks through a second map over the same rows, with boxes of
    // one key block.
    const cuuint32_t kvbox[2] = {kD, lng::kBK};
    CUtensorMap kvmap;
    if (fn(&kvmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<__half*>(qkv), dims, strides, kvbox, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    const dim3 grid((unsigned)((S + kRows - 1) / kRows), NH, B);
    return launch_kernel(attention_tc_long_kernel<PACKED>, grid, dim3(lng::kThreads), lng::kSmemTotal, stream,
                         nullptr, 0, map, kvmap, vl, offsets, ctx, B, S, NH, scale_log2, status);
  }
  // Persistent: four CTAs per SM, the footprint the kernel is built for
  // (launch bounds, shared memory and TMEM above).  The occupancy calculator
  // reports one CTA per SM for this kernel, so it is not asked.
  static const int resident = kCtasPerSm * device_sm_count();
  const long long items = (long long)B * NH;
  const dim3 grid((unsigned)(items < resident ? items : resident));
  // ctx [B*S, H] (the packed layout uses its first T rows), stored in boxes
  // of 32 rows x 64 halves with the 128-byte swizzle of the staged rows.
  const cuuint64_t cdims[2] = {H, (cuuint64_t)B * S};
  const cuuint64_t cstrides[1] = {H * 2};
  const cuuint32_t cbox[2] = {kD, 32};
  CUtensorMap cmap;
  if (fn(&cmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, ctx, cdims, cstrides, cbox, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  return launch_kernel(attention_tc_kernel<PACKED>, grid, dim3(kThreads), kSmemTotal, stream, nullptr, 0, map, vl,
                       offsets, ctx, B, S, NH, scale_log2, cmap, status);
}

}  // namespace

bool attention_tc_supported(int size_per_head, int seq) { return size_per_head == kD && seq > 64; }

cudaError_t launch_attention_tc(const __half* qkv, const int32_t* valid_len, const int32_t* offsets, __half* ctx,
                                int batch, int seq, int head_num, int* status, cudaStream_t stream) {
  if (batch <= 0 || batch > 65535 || head_num <= 0 || head_num > 65535 || !attention_tc_supported(kD, seq))
    return cudaErrorInvalidValue;
  if (3ll * batch * head_num * seq > 0x7fffffffll) return cudaErrorInvalidValue;   // int32 tensor-map rows
  if (offsets) return launch_tc<true>(qkv, valid_len, offsets, ctx, batch, seq, head_num, status, stream);
  return launch_tc<false>(qkv, valid_len, nullptr, ctx, batch, seq, head_num, status, stream);
}

}  // namespace enc
