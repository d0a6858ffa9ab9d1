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
  kBiasStore = 4     // C[m][n] = acc + bias[n]
};

// Addressing for the head-split epilogue (n = t*H + h*d + c, m = b*seq + s).
struct SplitShape {
  int batch, seq, head_num, size_per_head;
};

// Device status codes written by kernels (first failure wins).
constexpr int kStatusWaitTimeout = 1;

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
};
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
                            const float* bias, float* C, SplitShape split, cudaStream_t stream);

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

// Tensor-core attention (attention_tc.cu): size_per_head 64 and 64 < seq <= 128
// (attention_tc_supported); offsets == nullptr reads the split layout
// [3, B, nh, S, 64], else the packed [T, 3H] layout.
bool attention_tc_supported(int size_per_head, int seq);
cudaError_t launch_attention_tc(const __half* qkv, const int32_t* valid_len, const int32_t* offsets, __half* ctx,
                                int batch, int seq, int head_num, int* status, cudaStream_t stream);

// ---- add-bias + residual + LayerNorm, layernorm.cu ----
cudaError_t launch_bias_residual_ln_f16(const __half* a, const float* bias, const __half* resid,
                                        const float* gamma, const float* beta, __half* out,
                                        int rows, int hidden, cudaStream_t stream);
// FP16 rows with FP16 parameters (hidden <= 1024): one row per warp.
cudaError_t launch_bias_residual_ln_f16h(const __half* a, const __half* bias, const __half* resid,
                                         const __half* gamma, const __half* beta, __half* out,
                                         int rows, int hidden, cudaStream_t stream,
                                         const int* rows_dev = nullptr);
cudaError_t launch_bias_residual_ln_f32(const float* a, const float* bias, const float* resid,
                                        const float* gamma, const float* beta, float* out,
                                        int rows, int hidden, cudaStream_t stream);

// ---- weight repack, encoder.cu ----
int device_sm_count();

}  // namespace enc
