// Internal declarations shared by the kernels and the C-ABI layer.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "enc.h"

namespace enc {

constexpr float kLnEps = 1e-12f;   // LayerNorm epsilon (the original BERT value; the source page gives none)

// What a GEMM does with its FP32 accumulator tile before storing it.
enum class Epi : int {
  kStore = 0,        // C[m][n] = acc
  kBiasGelu = 1,     // C[m][n] = GELU(acc + bias[n]), erf form
  kBiasQkvSplit = 2, // Q/K/V head split: dst[t][b][h][s][c] = acc + bias[n]
  kBiasGeluTanh = 3, // C[m][n] = GELU_tanh(acc + bias[n])
  kBiasStore = 4,    // C[m][n] = acc + bias[n]
  kBiasResidStore = 5,  // C[m][n] = acc + bias[n] + R[m][n]  (R: the residual, [M, N] like C)
  kBiasResidLN = 6      // C[m][:] = LayerNorm(acc + bias + R)[m][:] over the row (gamma, beta)
};

// Addressing for the head-split epilogue (n = t*H + h*d + c, m = b*seq + s).
struct SplitShape {
  int batch, seq, head_num, size_per_head;
};

// Device status codes written by kernels (first failure wins).
constexpr int kStatusWaitTimeout = 1;

// ---- programmatic dependent launch ----
// The kernels of a forward are launched with programmatic stream
// serialization: a kernel may start while the previous kernel on the stream is
// still running.  It sets up what needs no memory the predecessor may touch
// (barriers, TMEM, tensor-map prefetch), then pdl_wait() returns once the
// predecessor has completed and its writes are visible; pdl_trigger() lets the
// successor begin launching (every kernel calls it only after taking its TMEM,
// so that a successor cannot hold TMEM a running kernel still has to allocate).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// The handle's ENC_OPT_PDL for the entry point running on this thread (plain
// stream order when off, for comparison runs).
bool pdl_enabled();

// <<<grid, block, smem, stream>>> with programmatic stream serialization
// (unless disabled); extra launch attributes (e.g. a cluster shape) may be
// passed in `extra`.
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                          const cudaLaunchAttribute* extra, int num_extra, Args... args) {
  cudaLaunchAttribute attrs[4];
  int n = 0;
  for (int i = 0; i < num_extra && n < 3; ++i) attrs[n++] = extra[i];
  if (pdl_enabled()) {
    attrs[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attrs;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// ---- FP16 tensor-core GEMM (tcgen05 + TMEM + TMA), gemm_tc.cu ----
// TcGemmArgs::bn selects the tile: 128 or 256 (one CTA, 128 x bn), or kPairTile
// (a 2-CTA cluster per 256 x 256 tile; B map box of 128 rows; N % 256 == 0).
constexpr int kPairTile = 2;
// C = A[M,K] * B[N,K]^T; A and B are K-major FP16 in global memory.
struct TcGemmArgs {
  const CUtensorMap* tmap_a;   // dims {K, M}, box {64, 128}, 128B swizzle
  const CUtensorMap* tmap_b;   // dims {K, N}, box {64, bn} (128 rows for kPairTile), 128B swizzle
  const CUtensorMap* tmap_c;   // output map with a 32x32 box, 64B swizzle, or nullptr (direct stores):
                               // C [M, N] as dims {N, M}; the head split as dims {d, seq, heads, batch, 3}
  int M, N, K;
  int bn;                      // 128, 256 or kPairTile
  Epi epi;
  const float* bias;           // [N] (kBiasGelu, kBiasQkvSplit)
  __half* c;                   // [M, N] or the split destination
  SplitShape split;
  int* status;                 // device status word
  int num_sms;
  const int* m_dev = nullptr;  // optional device row count (<= M): rows past it are neither computed nor stored
  // Split-K (bn == 128 only): a cluster of `splits` CTAs shares each 128 x 128
  // tile, CTA r taking the r-th of `splits` balanced ranges of the k-blocks;
  // the partial sums meet in the cluster's shared memory (no global scratch).
  int splits = 1;
  const __half* resid = nullptr;  // [M, N] (kBiasResidStore)
  const CUtensorMap* tmap_r = nullptr;  // the residual as an output-style map (32x32 box), or nullptr
  const float* ln_gamma = nullptr;      // [N] (kBiasResidLN)
  const float* ln_beta = nullptr;       // [N] (kBiasResidLN)
};
// The split count for a GEMM of `tiles` 128 x 128 tiles and `num_kb` 64-wide
// k-blocks: the largest s <= min(16, num_kb) whose clusters of s CTAs all fit
// on the GPU at once with tiles * s <= num_sms; 1 when no s >= 2 does.
int choose_gemm_splits(int tiles, int num_kb, int num_sms);
// Whether kBiasResidLN can run for an [M, N] GEMM: the row of N columns is
// covered by one cluster of N/128 CTAs (N a multiple of 256, N <= 1024), M >= 256.
bool gemm_ln_supported(int M, int N);
// Wave efficiency (work items / (waves x resident slots)) of an [M, N] GEMM with
// 2-CTA tiles: `fused` for the LayerNorm-fused kernel (one cluster of N/128 CTAs
// per 256 rows), `unfused` for the plain bias + residual kernel (one CTA pair
// per 256x256 tile).  False when N is not a LayerNorm width or the occupancy
// query fails.
bool gemm_ln_wave_efficiency(int M, int N, float& fused, float& unfused);
cudaError_t launch_gemm_tc(const TcGemmArgs& a, cudaStream_t stream);

// Encode a 2-D K-major FP16 tensor map over [rows, cols=K] with a {64, box_rows} box.
bool encode_kmajor_fp16_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                            uint32_t box_rows);
// Output maps for the GEMM epilogue's TMA stores (32x32 boxes, 64-byte swizzle).
bool encode_output_map_2d(CUtensorMap* map, void* base, uint64_t rows, uint64_t cols);
bool encode_output_map_split(CUtensorMap* map, void* base, const SplitShape& sp);

// ---- padding removal, pack.cu ----
// offsets[b] = sum_{b' < b} clamp(valid_len[b'], 0, seq); offsets[batch] = total valid tokens.
cudaError_t launch_valid_offsets(const int32_t* valid_len, int batch, int seq, int32_t* offsets,
                                 cudaStream_t stream);
// xp[offsets[b] + s] = x[b][s] for s < n_b (rows of `hidden` halves).
cudaError_t launch_pack_rows(const __half* x, const int32_t* valid_len, const int32_t* offsets, __half* xp,
                             int batch, int seq, int hidden, cudaStream_t stream);
// out[b][s] = yp[offsets[b] + s] for s < n_b, 0 otherwise.
cudaError_t launch_unpack_rows(const __half* yp, const int32_t* valid_len, const int32_t* offsets, __half* out,
                               int batch, int seq, int hidden, cudaStream_t stream);

// ---- FP32 SIMT GEMM (FP32 mode, no TF32), gemm_f32.cu ----
// C = A[M,K] * W[K,N] (W row-major [K,N]).
cudaError_t launch_gemm_f32(const float* A, const float* W, int M, int N, int K, Epi epi,
                            const float* bias, float* C, SplitShape split, cudaStream_t stream,
                            const float* resid = nullptr);

// ---- attention, attention.cu ----
cudaError_t launch_attention_f16(const __half* qkv, const int32_t* valid_len, __half* ctx,
                                 int batch, int seq, int head_num, int size_per_head,
                                 cudaStream_t stream);
// Packed tokens: qkv is [T, 3H] (Q | K | V per token), sequence b occupies rows
// offsets[b] .. offsets[b] + n_b - 1; ctx is [T, H].
cudaError_t launch_attention_f16_packed(const __half* qkv, const int32_t* valid_len, const int32_t* offsets,
                                        __half* ctx, int batch, int seq, int head_num, int size_per_head,
                                        cudaStream_t stream);
cudaError_t launch_attention_f32(const float* qkv, const int32_t* valid_len, float* ctx,
                                 int batch, int seq, int head_num, int size_per_head,
                                 cudaStream_t stream);

// Tensor-core attention (attention_tc.cu): size_per_head 64 and seq > 64
// (attention_tc_supported); offsets == nullptr reads the split layout
// [3, B, nh, S, 64], else the packed [T, 3H] layout.
bool attention_tc_supported(int size_per_head, int seq);
cudaError_t launch_attention_tc(const __half* qkv, const int32_t* valid_len, const int32_t* offsets, __half* ctx,
                                int batch, int seq, int head_num, int* status, cudaStream_t stream);

// ---- LayerNorm of z = a + bias + residual (added by the GEMM epilogue), layernorm.cu ----
cudaError_t launch_layernorm_f16(const __half* z, const float* gamma, const float* beta, __half* out, int rows,
                                 int hidden, cudaStream_t stream);
// FP16 rows with FP16 parameters (hidden <= 1024): one row per warp.
cudaError_t launch_layernorm_f16h(const __half* z, const __half* gamma, const __half* beta, __half* out, int rows,
                                  int hidden, cudaStream_t stream, const int* rows_dev = nullptr);
cudaError_t launch_layernorm_f32(const float* z, const float* gamma, const float* beta, float* out, int rows,
                                 int hidden, cudaStream_t stream);

// ---- decoder attention, decoder_attention.cu ----
// q [B, nh, T, d], k and v [B, nh, Skv, d] (head-split); keys j < clamp(kv_len[b],
// 0, Skv), and with `causal` j <= i for query i; ctx [B*T, nh*d].
cudaError_t launch_decoder_attention(const __half* q, const __half* k, const __half* v, const int32_t* kv_len,
                                     __half* ctx, int batch, int head_num, int size_per_head, int tgt_seq, int kv_seq,
                                     bool causal, cudaStream_t stream);

// ---- single-launch forward for small batches, persistent.cu ----
constexpr int kPersistMaxTokens = 256;   // batch * seq
constexpr int kPersistMaxSplits = 4;     // K splits of FFN2
// One layer's parameters as the handle stores them: FP16 weights transposed to
// [out, in] (K-major), FP32 biases and LayerNorm parameters.
struct PersistLayer {
  const __half *w_qkv, *w_o, *w_ff1, *w_ff2;
  const float *b_qkv, *b_o, *b_ff1, *b_ff2, *ln1_g, *ln1_b, *ln2_g, *ln2_b;
};
struct PersistArgs {
  // A operands, FP16 [M, K] with a box of 64 columns x 16 ceil(M / 16) rows and
  // 128-byte swizzle: x, z2, ctx, z1 ([M, H]) and u ([M, F]).
  alignas(64) CUtensorMap amap[5];
  const CUtensorMap* wmaps;     // device [L][4]: Wqkv^T, Wo^T, W1^T, W2^T ([N, K], box 64 x 32, 128-byte swizzle)
  const PersistLayer* layers;   // device array [L]
  int L;
  const __half* x;              // [B*S, H]
  const int32_t* valid_len;     // [B]
  __half* out;                  // [B*S, H]
  int B, S, NH, D, F;
  // Workspace [B*S, ...]: qkv [M, 3H] (Q | K | V per token), ctx, z1, h1 [M, H],
  // u [M, F], z2 [M, H], xl [M, H] (the LayerNorm-2 output of the previous layer).
  __half *qkv, *ctx, *z1, *h1, *u, *z2, *xl;
  float* partial;               // FFN2 split-K partial tiles, FP32 [splits][M][H]
  unsigned* tile_cnt;           // FFN2 per-tile counters [H / 32]
  int gelu_tanh;
  unsigned* bar;                // 4 words, zero between launches: arrivals, epoch, exits, a flag never set
  int* status;
  unsigned long long wait_ns;   // limit of every wait
  int stall_test;               // failure-detection test: CTA 0 never joins the first barrier
};
bool persistent_supported(int B, int S, int NH, int D, int F, int num_sms);
// Device bytes of the FFN2 partial tiles and tile counters for hidden size H.
size_t persistent_partial_bytes(int H, int F);
cudaError_t launch_persistent(const PersistArgs& args, cudaStream_t stream);

// ---- weight repack, encoder.cu ----
int device_sm_count();

}  // namespace enc
