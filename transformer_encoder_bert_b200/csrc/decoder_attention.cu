// Attention of the decoder forward: causal self-attention over the target
// tokens and cross-attention from the target to the memory (an encoder
// output), one kernel for both.
//
// The source page ([FT] "什么是 Faster Transformer") plans a decoder without
// describing it; the layer read here is the post-LN Transformer decoder layer
// over a whole target sequence.  Its attention differs from the encoder's in
// two ways: the queries and the keys come from different tensors of different
// lengths (T target tokens, S memory tokens for cross-attention), and
// self-attention is causal (query i sees keys j <= i).
//
//   q:  [B, nh, T, d]  (head-split, as the Q-projection GEMM epilogue writes it)
//   k, v: [B, nh, Skv, d]
//   kv_len[b]: keys j < n = clamp(kv_len[b], 0, Skv) are valid; with `causal`
//   query i also needs j <= i.  ctx [B*T, nh*d]: row b*T + i, head h at
//   columns h*d .. h*d+d-1.  A row without a valid key (n == 0) gets ctx = 0.
//
// One CTA per (block of 64 query rows, head, sequence), 4 warps of 16 rows.
// Keys stream in blocks of 64 through a two-stage cp.async ring; scores stay in
// registers (mma.sync m16n8k16, FP16 in, FP32 accumulate); online softmax in
// FP32 with quad-shuffle row max and sum; P rounded to FP16 for P V.  With the
// causal mask a query block never loads the key blocks past its last row.
// Every row has a valid key in the first key block (key 0) whenever n >= 1,
// so the running maximum is finite from the first block on.
#include <mutex>

#include "internal.h"

namespace enc {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kNW = 4;             // warps per CTA
constexpr int kBQ = 16 * kNW;      // query rows per CTA
constexpr int kBKV = 64;           // keys per block

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;    // 0 source bytes: the 16 destination bytes are zero-filled
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

template <int D>
struct DecAttnCfg {
  static constexpr int kLd = D + 8;                          // padded row (halves): conflict-free ldmatrix
  static constexpr int kQElems = kBQ * kLd;
  static constexpr int kKVElems = kBKV * kLd;
  static constexpr int kSmem = (kQElems + 4 * kKVElems) * 2;  // Q, two stages of (K, V)
};

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kNW * 32)
    decoder_attention_kernel(const __half* __restrict__ q, const __half* __restrict__ k, const __half* __restrict__ v,
                             const int32_t* __restrict__ kv_len, __half* __restrict__ ctx, int B, int NH, int T,
                             int Skv, float score_scale_log2) {
  using C = DecAttnCfg<D>;
  extern __shared__ __align__(16) __half sm[];
  pdl_wait();                                   // Q/K/V of the previous kernels are visible
  pdl_trigger();
  __half* Qs = sm;
  __half* Ks = sm + C::kQElems;                 // [2][kBKV][kLd]
  __half* Vs = Ks + 2 * C::kKVElems;            // [2][kBKV][kLd]
  const int b = blockIdx.z, h = blockIdx.y, q0 = blockIdx.x * kBQ;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  int n = kv_len[b];
  n = n < 0 ? 0 : (n > Skv ? Skv : n);
  constexpr int kChunks = D / 8;
  const __half* qh = q + ((size_t)b * NH + h) * T * D;
  const __half* kh = k + ((size_t)b * NH + h) * Skv * D;
  const __half* vh = v + ((size_t)b * NH + h) * Skv * D;

  for (int i = threadIdx.x; i < kBQ * kChunks; i += kNW * 32) {
    const int r = i / kChunks, c = i % kChunks;
    const int row = q0 + r;
    const bool ok = row < T;
    cp_async16(smem_addr(Qs + r * C::kLd + c * 8), qh + (size_t)(ok ? row : 0) * D + c * 8, ok);
  }
  auto load_kv = [&](int kb, int stage) {
    __half* kd = Ks + stage * C::kKVElems;
    __half* vd = Vs + stage * C::kKVElems;
    for (int i = threadIdx.x; i < kBKV * kChunks; i += kNW * 32) {
      const int r = i / kChunks, c = i % kChunks;
      const int key = kb * kBKV + r;
      const bool ok = key < n;
      const size_t off = (size_t)(ok ? key : 0) * D + c * 8;
      cp_async16(smem_addr(kd + r * C::kLd + c * 8), kh + off, ok);
      cp_async16(smem_addr(vd + r * C::kLd + c * 8), vh + off, ok);
    }
  };
  // Keys this query block can see: j < n, and with the causal mask j <= q0 + kBQ - 1.
  const int kmax = CAUSAL ? min(n, q0 + kBQ) : n;
  const int num_kb = (kmax + kBKV - 1) / kBKV;
  if (num_kb > 0) load_kv(0, 0);
  cp_async_commit();

  float o[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  uint32_t qf[D / 16][4];
  const int row_lo = q0 + warp * 16 + g;        // this thread's two query rows: row_lo, row_lo + 8

  for (int kb = 0; kb < num_kb; ++kb) {
    if (kb + 1 < num_kb) load_kv(kb + 1, (kb + 1) & 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (kb == 0) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int r = warp * 16 + (lane & 15);
        const int c = kk * 16 + (lane >> 4) * 8;
        ldsm_x4(smem_addr(Qs + r * C::kLd + c), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
      }
    }
    const __half* kbuf = Ks + (kb & 1) * C::kKVElems;
    const __half* vbuf = Vs + (kb & 1) * C::kKVElems;
    const int key_base = kb * kBKV;
    float s[kBKV / 8][4];
#pragma unroll
    for (int i = 0; i < kBKV / 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int np = 0; np < kBKV / 16; ++np) {
        if (key_base + np * 16 >= kmax) continue;
        const int key = np * 16 + (lane >> 4) * 8 + (lane & 7);
        const int dim = kk * 16 + ((lane >> 3) & 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(smem_addr(kbuf + key * C::kLd + dim), b0, b1, b2, b3);
        mma16816(s[2 * np], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b0, b1);
        mma16816(s[2 * np + 1], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b2, b3);
      }
    }
    // Mask (j >= n, and j > i with the causal mask), then the online softmax.
    float mx[2] = {m_run[0], m_run[1]};
#pragma unroll
    for (int nt = 0; nt < kBKV / 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = key_base + nt * 8 + 2 * t + (e & 1);
        const int i = row_lo + 8 * (e >> 1);
        if (j >= n || (CAUSAL && j > i)) s[nt][e] = -INFINITY;
        mx[e >> 1] = fmaxf(mx[e >> 1], s[nt][e]);
      }
    }
    float alpha[2], mscaled[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
      alpha[r] = exp2f((m_run[r] - mx[r]) * score_scale_log2);   // first block: exp2(-inf) = 0
      m_run[r] = mx[r];
      mscaled[r] = mx[r] * score_scale_log2;
      l_run[r] *= alpha[r];
    }
#pragma unroll
    for (int nt = 0; nt < kBKV / 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float p = exp2f(fmaf(s[nt][e], score_scale_log2, -mscaled[e >> 1]));   // masked: exp2(-inf) = 0
        s[nt][e] = p;
        l_run[e >> 1] += p;
      }
    }
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      o[i][0] *= alpha[0]; o[i][1] *= alpha[0];
      o[i][2] *= alpha[1]; o[i][3] *= alpha[1];
    }
#pragma unroll
    for (int kc = 0; kc < kBKV / 16; ++kc) {
      if (key_base + kc * 16 >= kmax) continue;
      const uint32_t pa0 = pack_h2(s[2 * kc][0], s[2 * kc][1]);
      const uint32_t pa1 = pack_h2(s[2 * kc][2], s[2 * kc][3]);
      const uint32_t pa2 = pack_h2(s[2 * kc + 1][0], s[2 * kc + 1][1]);
      const uint32_t pa3 = pack_h2(s[2 * kc + 1][2], s[2 * kc + 1][3]);
#pragma unroll
      for (int dp = 0; dp < D / 16; ++dp) {
        const int key = kc * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
        const int dim = dp * 16 + (lane >> 4) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(smem_addr(vbuf + key * C::kLd + dim), b0, b1, b2, b3);
        mma16816(o[2 * dp], pa0, pa1, pa2, pa3, b0, b1);
        mma16816(o[2 * dp + 1], pa0, pa1, pa2, pa3, b2, b3);
      }
    }
    __syncthreads();   // this stage is refilled by the next iteration's prefetch
  }
  cp_async_wait<0>();
  __syncthreads();     // with no key block the Q copies of other threads may still be landing

  const int H = NH * D;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 1);
    l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 2);
  }
  const float inv0 = l_run[0] > 0.f ? 1.f / l_run[0] : 0.f;    // n == 0: ctx = 0
  const float inv1 = l_run[1] > 0.f ? 1.f / l_run[1] : 0.f;
  __half* orow = Qs + warp * 16 * C::kLd;       // this warp's own Q rows, reused for staging
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
    *reinterpret_cast<uint32_t*>(orow + g * C::kLd + i * 8 + 2 * t) = pack_h2(o[i][0] * inv0, o[i][1] * inv0);
    *reinterpret_cast<uint32_t*>(orow + (g + 8) * C::kLd + i * 8 + 2 * t) = pack_h2(o[i][2] * inv1, o[i][3] * inv1);
  }
  __syncwarp();
  for (int i = lane; i < 16 * kChunks; i += 32) {
    const int r = i / kChunks, c = i % kChunks;
    const int row = q0 + warp * 16 + r;
    if (row < T)
      *reinterpret_cast<uint4*>(ctx + ((size_t)b * T + row) * H + h * D + c * 8) =
          *reinterpret_cast<const uint4*>(orow + r * C::kLd + c * 8);
  }
}

template <int D, bool CAUSAL>
cudaError_t launch_dec(const __half* q, const __half* k, const __half* v, const int32_t* kv_len, __half* ctx, int B,
                       int NH, int T, int Skv, cudaStream_t stream) {
  using C = DecAttnCfg<D>;
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  std::call_once(once, [] {
    attr = cudaFuncSetAttribute(decoder_attention_kernel<D, CAUSAL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                C::kSmem);
  });
  if (attr != cudaSuccess) return attr;
  const dim3 grid((T + kBQ - 1) / kBQ, NH, B);
  const float scale_log2 = kLog2e / sqrtf((float)D);
  return launch_kernel(decoder_attention_kernel<D, CAUSAL>, grid, dim3(kNW * 32), C::kSmem, stream, nullptr, 0, q, k,
                       v, kv_len, ctx, B, NH, T, Skv, scale_log2);
}

}  // namespace

cudaError_t launch_decoder_attention(const __half* q, const __half* k, const __half* v, const int32_t* kv_len,
                                     __half* ctx, int batch, int head_num, int size_per_head, int tgt_seq, int kv_seq,
                                     bool causal, cudaStream_t stream) {
  if (batch <= 0 || batch > 65535 || head_num <= 0 || head_num > 65535 || tgt_seq <= 0 || kv_seq <= 0)
    return cudaErrorInvalidValue;
#define ENC_DEC_CASE(DD)                                                                                   \
  if (size_per_head == DD)                                                                                 \
    return causal ? launch_dec<DD, true>(q, k, v, kv_len, ctx, batch, head_num, tgt_seq, kv_seq, stream)   \
                  : launch_dec<DD, false>(q, k, v, kv_len, ctx, batch, head_num, tgt_seq, kv_seq, stream);
  ENC_DEC_CASE(32)
  ENC_DEC_CASE(64)
  ENC_DEC_CASE(128)
#undef ENC_DEC_CASE
  return cudaErrorInvalidValue;
}

}  // namespace enc
