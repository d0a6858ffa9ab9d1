// Fused masked scaled-dot-product attention: scaled QK^T + padding mask,
// softmax, PV and the merge of heads back to [tokens, hidden], one kernel.
//
// The source page ("Faster Transformer 优化原理") runs this as two batched
// cuBLAS GEMMs around a SoftMax kernel (two SoftMax versions for different
// shapes), with row sums by warp shuffle and FP32 sums for FP16 data, plus a
// transpose kernel.  Here the score tile never leaves the chip: each warp
// keeps 16 query rows' scores in registers, takes the row max and row sum
// with quad shuffles in FP32, and streams keys in blocks of 32 or 64 with an online
// softmax, so short (one key block) and long sequences share one kernel.
// Only key blocks that hold valid keys (j < n) are visited.
//
// FP16 path: mma.sync m16n8k16 (FP16 in, FP32 accumulate).  FP32 path: a
// plain CUDA-core kernel (no TF32) for the FP32 mode.
#include <mutex>

#include "internal.h"

namespace enc {
namespace {

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;   // 0 source bytes: the 16 destination bytes are zero-filled
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// One CTA = NW warps = 16*NW query rows of one (sequence, head); keys are
// streamed in blocks of BKV (32 for sequences of at most 32 tokens, so that no
// score MMA is spent on padding, else 64).
// Where one (sequence, head) lives.  Split layout: Q, K, V are [3, B, nh, S, d]
// (row stride d, S rows).  Packed layout (padding removed): the [T, 3H] output
// of the QKV projection, sequence b at rows offsets[b] .. offsets[b] + n - 1
// (row stride 3H, n rows); ctx is [T, H].
struct HeadView {
  const __half* q;
  const __half* k;
  const __half* v;
  size_t ld;        // row stride of Q/K/V (elements)
  size_t out_row0;  // ctx row of the sequence's first token
  int rows;         // rows that exist
};

template <bool PACKED>
__device__ __forceinline__ HeadView head_view(const __half* qkv, const int32_t* offsets, int b, int h, int B,
                                              int S, int NH, int D, int n) {
  HeadView hv;
  if constexpr (PACKED) {
    const size_t H = (size_t)NH * D;
    const size_t o = (size_t)offsets[b];
    hv.ld = 3 * H;
    hv.q = qkv + o * hv.ld + (size_t)h * D;
    hv.k = hv.q + H;
    hv.v = hv.q + 2 * H;
    hv.out_row0 = o;
    hv.rows = n;
  } else {
    const size_t he = (size_t)S * D;
    hv.q = qkv + (((size_t)0 * B + b) * NH + h) * he;
    hv.k = qkv + (((size_t)1 * B + b) * NH + h) * he;
    hv.v = qkv + (((size_t)2 * B + b) * NH + h) * he;
    hv.ld = D;
    hv.out_row0 = (size_t)b * S;
    hv.rows = S;
  }
  return hv;
}

__device__ __forceinline__ int clamp_len(const int32_t* valid_len, int b, int S) {
  const int n = valid_len[b];
  return n < 0 ? 0 : (n > S ? S : n);
}

// STAGES = 2 double-buffers the K/V blocks; STAGES = 1 when one block covers
// every key (S <= BKV).  MT = 16-row tiles per warp: with MT = 2 every K/V
// fragment read from shared memory feeds two MMAs, which halves the
// shared-memory traffic per MMA (the limiter once the scores stay on chip).
template <int D, int NW, int BKV, int STAGES, int MT>
struct AttnCfg {
  static constexpr int kBQ = 16 * MT * NW;
  static constexpr int kLd = D + 8;                         // padded row (halves): conflict-free ldmatrix
  static constexpr int kQElems = kBQ * kLd;
  static constexpr int kKVElems = BKV * kLd;
  static constexpr int kSmem = (kQElems + 2 * STAGES * kKVElems) * 2;  // Q + STAGES x (K, V)
};

template <int D, int NW, int BKV, int STAGES, int MT, bool PACKED>
__global__ void __launch_bounds__(NW * 32)
    attention_f16_kernel(const __half* __restrict__ qkv, const int32_t* __restrict__ valid_len,
                         const int32_t* __restrict__ offsets, __half* __restrict__ ctx, int B, int S, int NH,
                         float score_scale_log2) {
  using C = AttnCfg<D, NW, BKV, STAGES, MT>;
  constexpr int kBKV = BKV;
  extern __shared__ __align__(16) __half sm[];
  pdl_wait();                                   // Q/K/V (and offsets) of the previous kernels are visible
  pdl_trigger();
  __half* Qs = sm;
  __half* Ks = sm + C::kQElems;                 // [STAGES][kBKV][kLd]
  __half* Vs = Ks + STAGES * C::kKVElems;       // [STAGES][kBKV][kLd]

  const int b = blockIdx.z, h = blockIdx.y, q0 = blockIdx.x * C::kBQ;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int n = clamp_len(valid_len, b, S);
  if (PACKED && q0 >= n) return;               // packed: no rows of this sequence in this block
  const HeadView hv = head_view<PACKED>(qkv, offsets, b, h, B, S, NH, D, n);
  constexpr int kChunks = D / 8;                // 16-byte chunks per row

  // Q block (rows that do not exist are zero-filled).
  for (int i = threadIdx.x; i < C::kBQ * kChunks; i += NW * 32) {
    const int r = i / kChunks, c = i % kChunks;
    const int row = q0 + r;
    const bool v = row < hv.rows;
    cp_async16(smem_addr(Qs + r * C::kLd + c * 8), hv.q + (size_t)(v ? row : 0) * hv.ld + c * 8, v);
  }
  auto load_kv = [&](int kb, int stage) {
    __half* kd = Ks + stage * C::kKVElems;
    __half* vd = Vs + stage * C::kKVElems;
    for (int i = threadIdx.x; i < kBKV * kChunks; i += NW * 32) {
      const int r = i / kChunks, c = i % kChunks;
      const int key = kb * kBKV + r;
      const bool v = key < hv.rows;
      const size_t off = (size_t)(v ? key : 0) * hv.ld + c * 8;
      cp_async16(smem_addr(kd + r * C::kLd + c * 8), hv.k + off, v);
      cp_async16(smem_addr(vd + r * C::kLd + c * 8), hv.v + off, v);
    }
  };
  const int num_kb = (n + kBKV - 1) / kBKV;
  if (num_kb > 0) load_kv(0, 0);
  cp_async_commit();

  float o[MT][D / 8][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int i = 0; i < D / 8; ++i) o[mt][i][0] = o[mt][i][1] = o[mt][i][2] = o[mt][i][3] = 0.f;
  float m_run[MT][2], l_run[MT][2];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    m_run[mt][0] = m_run[mt][1] = -INFINITY;
    l_run[mt][0] = l_run[mt][1] = 0.f;
  }
  uint32_t qf[MT][D / 16][4];

  for (int kb = 0; kb < num_kb; ++kb) {
    if (STAGES > 1 && kb + 1 < num_kb) load_kv(kb + 1, (kb + 1) % STAGES);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (kb == 0) {
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int r = (warp * MT + mt) * 16 + (lane & 15);
          const int c = kk * 16 + (lane >> 4) * 8;
          ldsm_x4(smem_addr(Qs + r * C::kLd + c), qf[mt][kk][0], qf[mt][kk][1], qf[mt][kk][2], qf[mt][kk][3]);
        }
    }
    const __half* kbuf = Ks + (kb % STAGES) * C::kKVElems;
    const __half* vbuf = Vs + (kb % STAGES) * C::kKVElems;

    // Scores for this warp's 16*MT rows x kBKV keys.  Groups of 16 keys that lie
    // wholly at or past n are masked: their scores are never formed and their
    // PV terms are skipped (their weight is exactly 0).
    const int key_base = kb * kBKV;
    float s[MT][kBKV / 8][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int i = 0; i < kBKV / 8; ++i) s[mt][i][0] = s[mt][i][1] = s[mt][i][2] = s[mt][i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int np = 0; np < kBKV / 16; ++np) {
        if (key_base + np * 16 >= n) continue;
        const int key = np * 16 + (lane >> 4) * 8 + (lane & 7);
        const int dim = kk * 16 + ((lane >> 3) & 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(smem_addr(kbuf + key * C::kLd + dim), b0, b1, b2, b3);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          mma16816(s[mt][2 * np], qf[mt][kk][0], qf[mt][kk][1], qf[mt][kk][2], qf[mt][kk][3], b0, b1);
          mma16816(s[mt][2 * np + 1], qf[mt][kk][0], qf[mt][kk][1], qf[mt][kk][2], qf[mt][kk][3], b2, b3);
        }
      }
    }
    // Mask keys j >= n, then the online-softmax update (FP32).
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      float mx[2] = {m_run[mt][0], m_run[mt][1]};
#pragma unroll
      for (int nt = 0; nt < kBKV / 8; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = key_base + nt * 8 + 2 * t + (e & 1);
          if (j >= n) s[mt][nt][e] = -INFINITY;
          mx[e >> 1] = fmaxf(mx[e >> 1], s[mt][nt][e]);
        }
      }
      float alpha[2], mscaled[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
        mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
        alpha[r] = exp2f((m_run[mt][r] - mx[r]) * score_scale_log2);   // first block: exp2(-inf) = 0
        m_run[mt][r] = mx[r];
        mscaled[r] = mx[r] * score_scale_log2;
        l_run[mt][r] *= alpha[r];
      }
#pragma unroll
      for (int nt = 0; nt < kBKV / 8; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float p = exp2f(fmaf(s[mt][nt][e], score_scale_log2, -mscaled[e >> 1]));
          s[mt][nt][e] = p;
          l_run[mt][e >> 1] += p;
        }
      }
#pragma unroll
      for (int i = 0; i < D / 8; ++i) {
        o[mt][i][0] *= alpha[0]; o[mt][i][1] *= alpha[0];
        o[mt][i][2] *= alpha[1]; o[mt][i][3] *= alpha[1];
      }
    }
    // O += P V: P (16*MT x kBKV keys) from registers as FP16 A fragments.
#pragma unroll
    for (int kc = 0; kc < kBKV / 16; ++kc) {
      if (key_base + kc * 16 >= n) continue;
      uint32_t pa[MT][4];
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        pa[mt][0] = pack_h2(s[mt][2 * kc][0], s[mt][2 * kc][1]);
        pa[mt][1] = pack_h2(s[mt][2 * kc][2], s[mt][2 * kc][3]);
        pa[mt][2] = pack_h2(s[mt][2 * kc + 1][0], s[mt][2 * kc + 1][1]);
        pa[mt][3] = pack_h2(s[mt][2 * kc + 1][2], s[mt][2 * kc + 1][3]);
      }
#pragma unroll
      for (int dp = 0; dp < D / 16; ++dp) {
        const int key = kc * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
        const int dim = dp * 16 + (lane >> 4) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(smem_addr(vbuf + key * C::kLd + dim), b0, b1, b2, b3);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          mma16816(o[mt][2 * dp], pa[mt][0], pa[mt][1], pa[mt][2], pa[mt][3], b0, b1);
          mma16816(o[mt][2 * dp + 1], pa[mt][0], pa[mt][1], pa[mt][2], pa[mt][3], b2, b3);
        }
      }
    }
    __syncthreads();   // this stage is refilled by the next iteration's prefetch
  }
  cp_async_wait<0>();
  __syncthreads();   // with n == 0 the Q copies of other threads may still be landing

  // Normalise and stage this warp's rows in shared memory (its own Q rows).
  const int H = NH * D;
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      l_run[mt][r] += __shfl_xor_sync(0xffffffffu, l_run[mt][r], 1);
      l_run[mt][r] += __shfl_xor_sync(0xffffffffu, l_run[mt][r], 2);
    }
    const float inv0 = l_run[mt][0] > 0.f ? 1.f / l_run[mt][0] : 0.f;   // n == 0: ctx = 0
    const float inv1 = l_run[mt][1] > 0.f ? 1.f / l_run[mt][1] : 0.f;
    __syncwarp();
    __half* orow = Qs + (warp * MT + mt) * 16 * C::kLd;
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      *reinterpret_cast<uint32_t*>(orow + g * C::kLd + i * 8 + 2 * t) =
          pack_h2(o[mt][i][0] * inv0, o[mt][i][1] * inv0);
      *reinterpret_cast<uint32_t*>(orow + (g + 8) * C::kLd + i * 8 + 2 * t) =
          pack_h2(o[mt][i][2] * inv1, o[mt][i][3] * inv1);
    }
    __syncwarp();
    for (int i = lane; i < 16 * kChunks; i += 32) {
      const int r = i / kChunks, c = i % kChunks;
      const int row = q0 + (warp * MT + mt) * 16 + r;
      if (row < hv.rows) {
        *reinterpret_cast<uint4*>(ctx + (hv.out_row0 + row) * H + h * D + c * 8) =
            *reinterpret_cast<const uint4*>(orow + r * C::kLd + c * 8);
      }
    }
  }
}

template <int D, int NW, int BKV, int STAGES, int MT, bool PACKED>
cudaError_t launch_f16(const __half* qkv, const int32_t* vl, const int32_t* offsets, __half* ctx, int B, int S,
                       int NH, cudaStream_t stream) {
  using C = AttnCfg<D, NW, BKV, STAGES, MT>;
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  std::call_once(once, [] {
    attr = cudaFuncSetAttribute(attention_f16_kernel<D, NW, BKV, STAGES, MT, PACKED>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  });
  if (attr != cudaSuccess) return attr;
  const dim3 grid((S + C::kBQ - 1) / C::kBQ, NH, B);
  const float scale_log2 = kLog2e / sqrtf((float)D);
  return launch_kernel(attention_f16_kernel<D, NW, BKV, STAGES, MT, PACKED>, grid, dim3(NW * 32), C::kSmem, stream,
                       nullptr, 0, qkv, vl, offsets, ctx, B, S, NH, scale_log2);
}


// ---------------------------------------------------------------------------
// Short sequences (S <= BKV, so one query block of 16*NW rows and one key
// block cover a whole (sequence, head)): a persistent CTA walks (sequence,
// head) items with two shared-memory buffers, so the next item's Q/K/V copies
// are in flight while the current item is computed.  The single key block
// needs no online rescaling: row max, exponentials, row sum, PV.
// ---------------------------------------------------------------------------
template <int D, int NW, int BKV>
struct ShortCfg {
  static constexpr int kBQ = 16 * NW;
  static constexpr int kLd = D + 8;
  static constexpr int kBufElems = (kBQ + 2 * BKV) * kLd;   // Q, K, V of one item
  static constexpr int kSmem = 2 * kBufElems * 2;
};

template <int D, int NW, int BKV, bool PACKED>
__global__ void __launch_bounds__(NW * 32)
    attention_f16_short_kernel(const __half* __restrict__ qkv, const int32_t* __restrict__ valid_len,
                               const int32_t* __restrict__ offsets, __half* __restrict__ ctx, int B, int S,
                               int NH, float score_scale_log2) {
  using C = ShortCfg<D, NW, BKV>;
  static_assert(C::kBQ <= BKV || C::kBQ == 16 * NW, "one query block");
  extern __shared__ __align__(16) __half sm[];
  pdl_wait();                                   // Q/K/V (and offsets) of the previous kernels are visible
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  constexpr int kChunks = D / 8;
  const int items = B * NH;
  const int H = NH * D;

  auto issue_loads = [&](int item, int buf) {
    const int b = item / NH, h = item - b * NH;
    const HeadView hv = head_view<PACKED>(qkv, offsets, b, h, B, S, NH, D, clamp_len(valid_len, b, S));
    __half* qs = sm + buf * C::kBufElems;
    __half* ks = qs + C::kBQ * C::kLd;
    __half* vs = ks + BKV * C::kLd;
    for (int i = threadIdx.x; i < BKV * kChunks; i += NW * 32) {
      const int r = i / kChunks, c = i % kChunks;
      const bool v = r < hv.rows;
      const size_t off = (size_t)(v ? r : 0) * hv.ld + c * 8;
      if (r < C::kBQ) cp_async16(smem_addr(qs + r * C::kLd + c * 8), hv.q + off, v);
      cp_async16(smem_addr(ks + r * C::kLd + c * 8), hv.k + off, v);
      cp_async16(smem_addr(vs + r * C::kLd + c * 8), hv.v + off, v);
    }
  };

  int item = blockIdx.x;
  if (item < items) issue_loads(item, 0);
  cp_async_commit();
  for (int it = 0; item < items; ++it, item += gridDim.x) {
    const int buf = it & 1;
    const int next = item + gridDim.x;
    if (next < items) issue_loads(next, buf ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();

    const int b = item / NH, h = item - b * NH;
    const int n = clamp_len(valid_len, b, S);
    const HeadView hv = head_view<PACKED>(qkv, offsets, b, h, B, S, NH, D, n);
    __half* qs = sm + buf * C::kBufElems;
    const __half* ks = qs + C::kBQ * C::kLd;
    const __half* vs = ks + BKV * C::kLd;

    uint32_t qf[D / 16][4];
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int r = warp * 16 + (lane & 15);
      const int c = kk * 16 + (lane >> 4) * 8;
      ldsm_x4(smem_addr(qs + r * C::kLd + c), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
    }
    float o[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float l_run[2] = {0.f, 0.f};
    if (n > 0) {
      float s[BKV / 8][4];
#pragma unroll
      for (int i = 0; i < BKV / 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
        for (int np = 0; np < BKV / 16; ++np) {
          if (np * 16 >= n) continue;   // wholly masked group of 16 keys
          const int key = np * 16 + (lane >> 4) * 8 + (lane & 7);
          const int dim = kk * 16 + ((lane >> 3) & 1) * 8;
          uint32_t b0, b1, b2, b3;
          ldsm_x4(smem_addr(ks + key * C::kLd + dim), b0, b1, b2, b3);
          mma16816(s[2 * np], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b0, b1);
          mma16816(s[2 * np + 1], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b2, b3);
        }
      }
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int nt = 0; nt < BKV / 8; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = nt * 8 + 2 * t + (e & 1);
          if (j >= n) s[nt][e] = -INFINITY;
          mx[e >> 1] = fmaxf(mx[e >> 1], s[nt][e]);
        }
      }
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
        mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
        mx[r] *= score_scale_log2;
      }
#pragma unroll
      for (int nt = 0; nt < BKV / 8; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float p = exp2f(fmaf(s[nt][e], score_scale_log2, -mx[e >> 1]));
          s[nt][e] = p;
          l_run[e >> 1] += p;
        }
      }
#pragma unroll
      for (int kc = 0; kc < BKV / 16; ++kc) {
        if (kc * 16 >= n) continue;
        const uint32_t a0 = pack_h2(s[2 * kc][0], s[2 * kc][1]);
        const uint32_t a1 = pack_h2(s[2 * kc][2], s[2 * kc][3]);
        const uint32_t a2 = pack_h2(s[2 * kc + 1][0], s[2 * kc + 1][1]);
        const uint32_t a3 = pack_h2(s[2 * kc + 1][2], s[2 * kc + 1][3]);
#pragma unroll
        for (int dp = 0; dp < D / 16; ++dp) {
          const int key = kc * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
          const int dim = dp * 16 + (lane >> 4) * 8;
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(smem_addr(vs + key * C::kLd + dim), b0, b1, b2, b3);
          mma16816(o[2 * dp], a0, a1, a2, a3, b0, b1);
          mma16816(o[2 * dp + 1], a0, a1, a2, a3, b2, b3);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 1);
      l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 2);
    }
    const float inv0 = l_run[0] > 0.f ? 1.f / l_run[0] : 0.f;   // n == 0: ctx = 0
    const float inv1 = l_run[1] > 0.f ? 1.f / l_run[1] : 0.f;
    // Stage this warp's 16 output rows over its own Q rows (already in registers).
    __syncwarp();
    __half* orow = qs + warp * 16 * C::kLd;
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      *reinterpret_cast<uint32_t*>(orow + g * C::kLd + i * 8 + 2 * t) = pack_h2(o[i][0] * inv0, o[i][1] * inv0);
      *reinterpret_cast<uint32_t*>(orow + (g + 8) * C::kLd + i * 8 + 2 * t) = pack_h2(o[i][2] * inv1, o[i][3] * inv1);
    }
    __syncwarp();
    for (int i = lane; i < 16 * kChunks; i += 32) {
      const int r = i / kChunks, c = i % kChunks;
      const int row = warp * 16 + r;
      if (row < hv.rows) {
        *reinterpret_cast<uint4*>(ctx + (hv.out_row0 + row) * H + h * D + c * 8) =
            *reinterpret_cast<const uint4*>(orow + r * C::kLd + c * 8);
      }
    }
    __syncthreads();   // buffer `buf` is refilled by the prefetch two items ahead
  }
  cp_async_wait<0>();
}

template <int D, int NW, int BKV, bool PACKED>
cudaError_t launch_short(const __half* qkv, const int32_t* vl, const int32_t* offsets, __half* ctx, int B, int S,
                         int NH, cudaStream_t stream) {
  using C = ShortCfg<D, NW, BKV>;
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  static int per_sm = 1;
  std::call_once(once, [] {
    attr = cudaFuncSetAttribute(attention_f16_short_kernel<D, NW, BKV, PACKED>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (attr == cudaSuccess)
      attr = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, attention_f16_short_kernel<D, NW, BKV, PACKED>, NW * 32,
                                                           C::kSmem);
    if (per_sm < 1) per_sm = 1;
  });
  if (attr != cudaSuccess) return attr;
  const int items = B * NH;
  const int cap = per_sm * device_sm_count();
  const float scale_log2 = kLog2e / sqrtf((float)D);
  return launch_kernel(attention_f16_short_kernel<D, NW, BKV, PACKED>, dim3(items < cap ? items : cap), dim3(NW * 32),
                       C::kSmem, stream, nullptr, 0, qkv, vl, offsets, ctx, B, S, NH, scale_log2);
}


// Launch shape by sequence length ([FT] "Faster Transformer 优化原理" keeps
// several SoftMax versions and picks grid/block sizes from the shape).
template <int D, bool PACKED>
cudaError_t launch_f16_d(const __half* qkv, const int32_t* vl, const int32_t* offsets, __half* ctx, int B, int S,
                         int NH, cudaStream_t stream) {
  if (S <= 16) return launch_short<D, 1, 32, PACKED>(qkv, vl, offsets, ctx, B, S, NH, stream);
  if (S <= 32) return launch_short<D, 2, 32, PACKED>(qkv, vl, offsets, ctx, B, S, NH, stream);
  if (S <= 64) return launch_short<D, 4, 64, PACKED>(qkv, vl, offsets, ctx, B, S, NH, stream);
#ifndef ENC_ATTN_MT
#define ENC_ATTN_MT 2
#endif
  if constexpr (D <= 64 && ENC_ATTN_MT == 2)
    return launch_f16<D, 4, 32, 2, 2, PACKED>(qkv, vl, offsets, ctx, B, S, NH, stream);
  return launch_f16<D, 8, 64, 2, 1, PACKED>(qkv, vl, offsets, ctx, B, S, NH, stream);
}

// ---------------------------------------------------------------- FP32 (CUDA cores)
// One warp per query row; lanes own head dimensions c = lane, lane+32, ...; keys
// are visited in order with an online softmax (running max and sum, FP32).
template <int D>
__global__ void __launch_bounds__(128)
    attention_f32_kernel(const float* __restrict__ qkv, const int32_t* __restrict__ valid_len,
                         float* __restrict__ ctx, int B, int S, int NH) {
  constexpr int kPer = D / 32;
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.z, h = blockIdx.y;
  const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= S) return;
  int n = valid_len[b];
  n = n < 0 ? 0 : (n > S ? S : n);
  const size_t head_elems = (size_t)S * D;
  const float* Qg = qkv + (((size_t)0 * B + b) * NH + h) * head_elems;
  const float* Kg = qkv + (((size_t)1 * B + b) * NH + h) * head_elems;
  const float* Vg = qkv + (((size_t)2 * B + b) * NH + h) * head_elems;
  const float scale = 1.0f / sqrtf((float)D);
  float q[kPer], acc[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    q[i] = Qg[(size_t)row * D + lane + 32 * i];
    acc[i] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int j = 0; j < n; ++j) {
    float part = 0.f;
#pragma unroll
    for (int i = 0; i < kPer; ++i) part = fmaf(q[i], Kg[(size_t)j * D + lane + 32 * i], part);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    const float sc = part * scale;
    const float m_new = fmaxf(m, sc);
    const float alpha = expf(m - m_new);
    const float p = expf(sc - m_new);
    l = l * alpha + p;
#pragma unroll
    for (int i = 0; i < kPer; ++i) acc[i] = fmaf(p, Vg[(size_t)j * D + lane + 32 * i], acc[i] * alpha);
    m = m_new;
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  const int H = NH * D;
#pragma unroll
  for (int i = 0; i < kPer; ++i) ctx[((size_t)b * S + row) * H + h * D + lane + 32 * i] = acc[i] * inv;
}

}  // namespace

cudaError_t launch_attention_f16(const __half* qkv, const int32_t* valid_len, __half* ctx, int batch,
                                 int seq, int head_num, int size_per_head, cudaStream_t stream) {
  if (batch <= 0 || seq <= 0 || head_num <= 0 || head_num > 65535 || batch > 65535) return cudaErrorInvalidValue;
  switch (size_per_head) {
    case 32: return launch_f16_d<32, false>(qkv, valid_len, nullptr, ctx, batch, seq, head_num, stream);
    case 64: return launch_f16_d<64, false>(qkv, valid_len, nullptr, ctx, batch, seq, head_num, stream);
    case 128: return launch_f16_d<128, false>(qkv, valid_len, nullptr, ctx, batch, seq, head_num, stream);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_attention_f16_packed(const __half* qkv, const int32_t* valid_len, const int32_t* offsets,
                                        __half* ctx, int batch, int seq, int head_num, int size_per_head,
                                        cudaStream_t stream) {
  if (batch <= 0 || seq <= 0 || head_num <= 0 || head_num > 65535 || batch > 65535) return cudaErrorInvalidValue;
  switch (size_per_head) {
    case 32: return launch_f16_d<32, true>(qkv, valid_len, offsets, ctx, batch, seq, head_num, stream);
    case 64: return launch_f16_d<64, true>(qkv, valid_len, offsets, ctx, batch, seq, head_num, stream);
    case 128: return launch_f16_d<128, true>(qkv, valid_len, offsets, ctx, batch, seq, head_num, stream);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_attention_f32(const float* qkv, const int32_t* valid_len, float* ctx, int batch,
                                 int seq, int head_num, int size_per_head, cudaStream_t stream) {
  if (batch <= 0 || seq <= 0 || head_num <= 0 || head_num > 65535 || batch > 65535) return cudaErrorInvalidValue;
  const dim3 grid((seq + 3) / 4, head_num, batch);
  switch (size_per_head) {
    case 32:
      return launch_kernel(attention_f32_kernel<32>, grid, dim3(128), 0, stream, nullptr, 0, qkv, valid_len, ctx,
                           batch, seq, head_num);
    case 64:
      return launch_kernel(attention_f32_kernel<64>, grid, dim3(128), 0, stream, nullptr, 0, qkv, valid_len, ctx,
                           batch, seq, head_num);
    case 128:
      return launch_kernel(attention_f32_kernel<128>, grid, dim3(128), 0, stream, nullptr, 0, qkv, valid_len, ctx,
                           batch, seq, head_num);
  }
  return cudaErrorInvalidValue;
}

}  // namespace enc
