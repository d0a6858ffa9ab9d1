// C-ABI layer: handle, weight repacking, workspace, the per-layer step
// sequence and the entry points declared in enc.h.
//
// Per layer, enc_forward launches (FP16 mode):
//   1 tcgen05 GEMM  x Wqkv, epilogue + bqkv and Q/K/V head split
//   2 attention     masked scaled softmax(QK^T) V, heads merged to [M, H]
//   3 tcgen05 GEMM  ctx Wo
//   4 LayerNorm     LN(x + a + bo)
//   5 tcgen05 GEMM  h1 W1, epilogue + b1 and GELU
//   6 tcgen05 GEMM  u W2
//   7 LayerNorm     LN(h1 + y + b2)
// i.e. 7 launches for the page's 14 ("Faster Transformer 优化原理": 8 cuBLAS
// GEMMs + 6 custom kernels).  FP32 mode runs the same sequence with the
// CUDA-core GEMM and attention kernels.
#include <cstdarg>
#include <cstdio>
#include <algorithm>
#include <atomic>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "internal.h"

namespace {

thread_local std::string g_last_error;
// The device of the first handle: kernel launch attributes (dynamic shared
// memory sizes, cluster occupancy) are set once per process, for that device.
std::atomic<int> g_process_device{-1};

enc_status fail(enc_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

enc_status ok() {
  g_last_error.clear();
  return ENC_OK;
}

enc_status cuda_fail(cudaError_t e, const char* what) {
  return fail(ENC_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// [rows, cols] -> [cols, rows] for FP16 weights (tensor-core B operands are K-major).
__global__ void transpose_f16_kernel(const __half* __restrict__ in, __half* __restrict__ out, int rows,
                                     int cols) {
  __shared__ __half tile[32][33];
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int r = r0 + i, c = c0 + threadIdx.x;
    if (r < rows && c < cols) tile[i][threadIdx.x] = in[(size_t)r * cols + c];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int c = c0 + i, r = r0 + threadIdx.x;
    if (c < cols && r < rows) out[(size_t)c * rows + r] = tile[threadIdx.x][i];
  }
}

template <typename T>
__global__ void widen_to_f32_kernel(const T* __restrict__ in, float* __restrict__ out, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = static_cast<float>(in[i]);
}

struct LayerDev {
  void* w_qkv = nullptr;   // FP16: [3H, H]; FP32: [H, 3H]
  void* w_o = nullptr;     // FP16: [H, H] transposed; FP32: [H, H]
  void* w_ff1 = nullptr;   // FP16: [F, H]; FP32: [H, F]
  void* w_ff2 = nullptr;   // FP16: [H, F]; FP32: [F, H]
  float *b_qkv = nullptr, *b_o = nullptr, *b_ff1 = nullptr, *b_ff2 = nullptr;
  float *ln1_g = nullptr, *ln1_b = nullptr, *ln2_g = nullptr, *ln2_b = nullptr;
  // FP16 copies (FP16 mode only; exact, the caller supplied halves) for the LayerNorm kernel:
  // b_o, ln1_g, ln1_b, b_ff2, ln2_g, ln2_b.
  __half *h_ln1_g = nullptr, *h_ln1_b = nullptr, *h_ln2_g = nullptr, *h_ln2_b = nullptr;
  CUtensorMap tm_qkv[2], tm_o[2], tm_ff1[2], tm_ff2[2];   // [0]: 128-row box, [1]: 256-row box
};

// One decoder layer on the device: FP16 weights transposed to [out, in] with
// their tensor maps (128- and 256-row boxes), FP32 biases and LayerNorm
// parameters, FP16 copies of the LayerNorm parameters for the LayerNorm kernel.
struct DecLayerDev {
  void *w_qkv, *w_o, *w_q2, *w_kv2, *w_o2, *w_ff1, *w_ff2;
  float *b_qkv, *b_o, *b_q2, *b_kv2, *b_o2, *b_ff1, *b_ff2;
  __half *ln_g[3], *ln_b[3];                 // FP16 (LayerNorm kernel)
  float *ln_gf[3], *ln_bf[3];                // FP32 (LayerNorm fused into a GEMM epilogue)
  CUtensorMap tm_qkv[2], tm_o[2], tm_q2[2], tm_kv2[2], tm_o2[2], tm_ff1[2], tm_ff2[2];
};

}  // namespace

struct enc_handle {
  int nh = 0, d = 0, H = 0, F = 0, L = 0;
  enc_dtype dtype = ENC_FP16;
  int device = 0;
  int num_sms = 0;
  size_t esize = 2;
  std::vector<LayerDev> layers;
  void* param_block = nullptr;
  void* ws = nullptr;
  size_t ws_bytes = 0;
  void* stage = nullptr;            // enc_forward_host device staging
  size_t stage_bytes = 0;
  cudaStream_t copy_in = nullptr;   // enc_forward_host: host-to-device copies
  cudaStream_t copy_out = nullptr;  // enc_forward_host: device-to-host copies
  static constexpr int kMaxChunks = 4;
  cudaEvent_t ev_in[kMaxChunks] = {}, ev_done[kMaxChunks] = {}, ev_out = nullptr, ev_start = nullptr;
  // enc_forward_host_async: two staging slots used in turn; per slot, its input
  // copy landed, its encoder run done, its output copy done (slot free again).
  int host_slot = 0;
  cudaEvent_t ev_slot_in[2] = {}, ev_slot_done[2] = {}, ev_slot_free[2] = {};
  int* status = nullptr;
  uint64_t launches = 0;            // kernels launched through this handle
  int graphs_alive = 0;             // recorded forwards that reference the workspace
  enc_gelu gelu = ENC_GELU_ERF;
  bool packed = false;              // padding removal (enc_set_packing)
  int host_chunks = 1;              // enc_forward_host: most chunks the batch is cut into (see enc.h)
  // Kernel-path switches (enc_set_option); the defaults are the fastest measured paths.
  bool pair_tiles = true;           // ENC_OPT_PAIR_TILES: 2-CTA 256x256 GEMM tiles where they fill the GPU
  bool tma_store = true;            // ENC_OPT_TMA_STORE: GEMM epilogues store (and read the residual) by TMA
  bool tc_attn = true;              // ENC_OPT_TC_ATTENTION: tcgen05 attention for d = 64, seq > 64
  bool splitk = true;               // ENC_OPT_SPLIT_K: split-K clusters for GEMMs that would idle most SMs
  // ENC_OPT_LN_FUSE_FFN2 / _OUT_PROJ: the GEMM writes the LayerNorm of its rows
  // (0 never, 1 where measured faster: hidden size <= 768, 2 wherever supported)
  int ln_fuse_ffn2 = 1;
  int ln_fuse_oproj = 1;
  bool pdl = true;                  // ENC_OPT_PDL: programmatic dependent launch between kernels
  bool persistent = false;          // ENC_OPT_PERSISTENT: single-launch forward for small batches
  bool stall_test = false;          // ENC_OPT_TEST_STALL: failure-detection test of that forward
  enc::PersistLayer* d_players = nullptr;   // device copy of every layer's pointers (FP16 mode)
  CUtensorMap* d_wmaps = nullptr;           // device [L][4] weight maps of the single-launch forward
  void* persist_partial = nullptr;          // its FFN2 partial tiles and tile counters
  std::vector<cudaEvent_t> trace;   // optional per-kernel events for enc_forward
  bool decoder = false;             // created by enc_decoder_create (its layers in dlayers)
  std::vector<struct DecLayerDev> dlayers;
};

namespace {

struct Workspace {
  void *qkv, *ctx, *a, *h1, *u, *x0, *x1;
  int32_t* offsets;   // packed mode: [batch + 1] token offsets of the sequences
};

size_t workspace_bytes(const enc_handle* h, size_t tokens) {
  const size_t es = h->esize;
  const size_t mh = align_up(tokens * h->H * es, 256);
  const size_t mf = align_up(tokens * h->F * es, 256);
  return 3 * mh + mh + mh + mh + mf + 2 * mh + align_up((tokens + 1) * 4, 256);
}

Workspace carve(const enc_handle* h, size_t tokens) {
  const size_t es = h->esize;
  const size_t mh = align_up(tokens * h->H * es, 256);
  const size_t mf = align_up(tokens * h->F * es, 256);
  char* p = static_cast<char*>(h->ws);
  Workspace w;
  w.qkv = p; p += 3 * mh;
  w.ctx = p; p += mh;
  w.a = p; p += mh;
  w.h1 = p; p += mh;
  w.u = p; p += mf;
  w.x0 = p; p += mh;
  w.x1 = p; p += mh;
  w.offsets = reinterpret_cast<int32_t*>(p);
  return w;
}

enc_status ensure_workspace(enc_handle* h, size_t tokens) {
  const size_t need = workspace_bytes(h, tokens);
  if (need <= h->ws_bytes) return ENC_OK;
  if (h->graphs_alive > 0)
    return fail(ENC_ERR_INVALID_ARG, "workspace of %zu bytes needed but %d recorded graph(s) pin the current one",
                need, h->graphs_alive);
  if (h->ws) {
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize before workspace growth");
    cudaFree(h->ws);
    h->ws = nullptr;
    h->ws_bytes = 0;
  }
  void* p = nullptr;
  if (cudaMalloc(&p, need) != cudaSuccess) {
    cudaGetLastError();
    return fail(ENC_ERR_OOM, "workspace allocation of %zu bytes failed", need);
  }
  h->ws = p;
  h->ws_bytes = need;
  return ENC_OK;
}

enc_status check_handle(const enc_handle* h) {
  if (!h) return fail(ENC_ERR_INVALID_ARG, "null handle");
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != h->device)
    return fail(ENC_ERR_INVALID_ARG, "current device %d is not the handle's device %d", dev, h->device);
  return ENC_OK;
}

// GEMM tiling.  The 2-CTA 256x256 tile when it still gives at least a quarter
// of the SMs a cluster each; else 128x256 one-CTA tiles when they fill the
// GPU; else 128x128.
int choose_bn(const enc_handle* h, int M, int N) {
  if (N % 256 == 0 && M >= 256 && h->pair_tiles) {
    const long pair_tiles = (long)((M + 255) / 256) * (N / 256);
    if (4 * pair_tiles >= h->num_sms) return enc::kPairTile;
  }
  if (N % 256 != 0) return 128;
  const long tiles256 = (long)((M + 127) / 128) * (N / 256);
  return tiles256 >= h->num_sms ? 256 : 128;
}

// Split-K for GEMMs whose 128x128 tiles would leave more than half the SMs
// idle (small batches): the k-blocks of a tile are shared by a cluster of CTAs,
// so that the weights are streamed by most SMs instead of a few.
int choose_splits(const enc_handle* h, int M, int N, int K, int bn) {
  if (bn != 128 || !h->splitk) return 1;
  const long tiles = (long)((M + 127) / 128) * ((N + 127) / 128);
  if (2 * tiles > h->num_sms) return 1;
  return enc::choose_gemm_splits((int)tiles, (K + 63) / 64, h->num_sms);
}

// One GEMM step: C = A * W (+ epilogue), dispatched on the handle's dtype.
enc_status run_gemm(enc_handle* h, const void* A, int M, int K, void* W, const CUtensorMap* wmaps, int N,
                    enc::Epi epi, const float* bias, void* C, enc::SplitShape sp, cudaStream_t st,
                    const int* m_dev = nullptr, const void* resid = nullptr, const float* ln_g = nullptr,
                    const float* ln_b = nullptr) {
  if (h->dtype == ENC_FP16) {
    const int bn = choose_bn(h, M, N);
    CUtensorMap ta;
    if (!enc::encode_kmajor_fp16_map(&ta, A, (uint64_t)M, (uint64_t)K, 128))
      return fail(ENC_ERR_CUDA, "cuTensorMapEncodeTiled failed for an activation operand [%d, %d]", M, K);
    // Output through TMA stores (32x32 boxes); the head split needs whole
    // 32-token chunks per sequence, otherwise its epilogue stores directly.
    CUtensorMap tc;
    bool use_tc = h->tma_store;
    if (use_tc) {
      if (epi == enc::Epi::kBiasQkvSplit)
        use_tc = (sp.seq % 32 == 0) && enc::encode_output_map_split(&tc, C, sp);
      else
        use_tc = enc::encode_output_map_2d(&tc, C, (uint64_t)M, (uint64_t)N);
    }
    // The residual of kBiasResidStore / kBiasResidLN comes in by TMA in the same 32x32 boxes
    // the output leaves in (only with TMA stores).
    CUtensorMap tr;
    const bool use_tr = use_tc && (epi == enc::Epi::kBiasResidStore || epi == enc::Epi::kBiasResidLN) && resid &&
                        enc::encode_output_map_2d(&tr, const_cast<void*>(resid), (uint64_t)M, (uint64_t)N);
    enc::TcGemmArgs a;
    a.tmap_a = &ta;
    a.tmap_c = use_tc ? &tc : nullptr;
    a.tmap_r = use_tr ? &tr : nullptr;
    a.tmap_b = &wmaps[bn == 256 ? 1 : 0];      // the pair tile loads 128-row halves of B
    a.M = M; a.N = N; a.K = K; a.bn = bn; a.epi = epi; a.bias = bias;
    a.c = static_cast<__half*>(C);
    a.split = sp;
    a.status = h->status;
    a.num_sms = h->num_sms;
    a.m_dev = m_dev;
    a.splits = choose_splits(h, M, N, K, bn);
    a.resid = static_cast<const __half*>(resid);
    a.ln_gamma = ln_g;
    a.ln_beta = ln_b;
    if (epi == enc::Epi::kBiasResidLN && (bn != enc::kPairTile || a.splits != 1 || !use_tr))
      return fail(ENC_ERR_UNSUPPORTED, "fused LayerNorm GEMM needs 2-CTA tiles and TMA residual/output maps");
    cudaError_t e = enc::launch_gemm_tc(a, st);
    if (e != cudaSuccess) return cuda_fail(e, "tensor-core GEMM launch");
    ++h->launches;
  } else {
    cudaError_t e = enc::launch_gemm_f32(static_cast<const float*>(A), static_cast<const float*>(W), M, N, K,
                                         epi, bias, static_cast<float*>(C), sp, st, static_cast<const float*>(resid));
    if (e != cudaSuccess) return cuda_fail(e, "FP32 GEMM launch");
    ++h->launches;
  }
  return ENC_OK;
}

enc_status step_qkv(enc_handle* h, int l, const void* x, void* qkv, int batch, int seq, cudaStream_t st) {
  LayerDev& L = h->layers[l];
  enc::SplitShape sp{batch, seq, h->nh, h->d};
  return run_gemm(h, x, batch * seq, h->H, L.w_qkv, L.tm_qkv, 3 * h->H, enc::Epi::kBiasQkvSplit, L.b_qkv, qkv,
                  sp, st);
}

// Attention kernel choice: the tensor-core kernels for size_per_head 64 and
// sequences longer than the short kernel's 64-row tiles (one 128-key block up to
// 128, key blocks with a running maximum beyond); mma.sync otherwise (and for
// every length with the tc_attention option off).
bool use_tc_attention(const enc_handle* h, int seq) {
  return enc::attention_tc_supported(h->d, seq) && h->tc_attn;
}

enc_status step_attention(enc_handle* h, const void* qkv, const int32_t* vl, void* ctx, int batch, int seq,
                          cudaStream_t st) {
  cudaError_t e;
  if (h->dtype == ENC_FP16 && use_tc_attention(h, seq))
    e = enc::launch_attention_tc(static_cast<const __half*>(qkv), vl, nullptr, static_cast<__half*>(ctx), batch, seq,
                                 h->nh, h->status, st);
  else if (h->dtype == ENC_FP16)
    e = enc::launch_attention_f16(static_cast<const __half*>(qkv), vl, static_cast<__half*>(ctx), batch, seq,
                                  h->nh, h->d, st);
  else
    e = enc::launch_attention_f32(static_cast<const float*>(qkv), vl, static_cast<float*>(ctx), batch, seq,
                                  h->nh, h->d, st);
  if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  ++h->launches;
  return ENC_OK;
}

// Output projection with add-bias and residual in the epilogue:
// z = ctx Wo + bo + resid (resid = the layer input).
enc_status step_out_proj(enc_handle* h, int l, const void* ctx, const void* resid, void* z, int tokens,
                         cudaStream_t st, const int* m_dev = nullptr) {
  LayerDev& L = h->layers[l];
  return run_gemm(h, ctx, tokens, h->H, L.w_o, L.tm_o, h->H, enc::Epi::kBiasResidStore, L.b_o, z, {}, st, m_dev,
                  resid);
}

// Whether GEMM `which` (1: output projection, 2: FFN2) writes the LayerNorm of
// its rows (kBiasResidLN) instead of z = acc + bias + residual for a LayerNorm
// kernel.  Needs the 2-CTA tiles to be the ones chosen for the shape (large M)
// and H a multiple of 256.  The fused kernel runs one cluster of H/128 CTAs per
// 256 rows (22 six-CTA clusters fit at once for H = 768), the unfused one a CTA
// pair per 256x256 tile (74 pairs), so the two fill their last wave
// differently.  Measured on BERT-Base shapes (forwards of 6144 to 32768
// tokens): FFN2's fused epilogue hides behind its long K = F main loop and pays
// off unless its last wave is far emptier than the unfused kernel's (24
// clusters' worth of rows on 22 slots: 13 % slower); the output projection's
// short K = H main loop cannot hide it, and fusing pays off only where the
// fused kernel fills its waves clearly better (64 and 128 row blocks: 1-3 %
// faster; 24, 32, 48 and 96: 0.3-5 % slower).  With 8-CTA clusters (H = 1024)
// fusion measured slower: those shapes keep the separate LayerNorm kernel
// unless the option asks for fusion wherever supported (2).
bool ln_fused(const enc_handle* h, int tokens, int which) {
  if (h->dtype != ENC_FP16 || !h->tma_store || !enc::gemm_ln_supported(tokens, h->H) ||
      choose_bn(h, tokens, h->H) != enc::kPairTile)
    return false;
  const int mode = which == 2 ? h->ln_fuse_ffn2 : h->ln_fuse_oproj;
  if (mode == 2) return true;
  if (mode != 1 || h->H > 768) return false;
  float fused = 0.f, unfused = 0.f;
  if (!enc::gemm_ln_wave_efficiency(tokens, h->H, fused, unfused)) return false;
  return which == 2 ? fused >= unfused - 0.3f : fused >= unfused + 0.1f;
}

// The single-launch forward (persistent.cu): FP16, padding kept, few enough
// tokens that every GEMM is a weight stream.
bool use_persistent(const enc_handle* h, int batch, int seq) {
  return h->dtype == ENC_FP16 && !h->packed && h->persistent && h->persist_partial && h->d_wmaps &&
         enc::persistent_supported(batch, seq, h->nh, h->d, h->F, h->num_sms);
}

enc_status run_persistent(enc_handle* h, const void* x, const int32_t* valid_len, void* out, int batch, int seq,
                          const Workspace& w, cudaStream_t st) {
  enc::PersistArgs a;
  const int M = batch * seq;
  const uint32_t box_rows = (uint32_t)(16 * ((M + 15) / 16));
  const void* abase[5] = {x, w.x0, w.ctx, w.a, w.u};        // x, z2, ctx, z1, u
  for (int i = 0; i < 5; ++i)
    if (!enc::encode_kmajor_fp16_map(&a.amap[i], abase[i], (uint64_t)M, (uint64_t)(i == 4 ? h->F : h->H), box_rows))
      return fail(ENC_ERR_CUDA, "cuTensorMapEncodeTiled failed for an activation operand");
  a.wmaps = h->d_wmaps;
  a.layers = h->d_players;
  a.L = h->L;
  a.x = static_cast<const __half*>(x);
  a.valid_len = valid_len;
  a.out = static_cast<__half*>(out);
  a.B = batch; a.S = seq; a.NH = h->nh; a.D = h->d; a.F = h->F;
  a.qkv = static_cast<__half*>(w.qkv);
  a.ctx = static_cast<__half*>(w.ctx);
  a.z1 = static_cast<__half*>(w.a);
  a.h1 = static_cast<__half*>(w.h1);
  a.u = static_cast<__half*>(w.u);
  a.z2 = static_cast<__half*>(w.x0);
  a.xl = static_cast<__half*>(w.x1);
  a.partial = static_cast<float*>(h->persist_partial);
  a.tile_cnt = reinterpret_cast<unsigned*>(static_cast<char*>(h->persist_partial) +
                                           (size_t)enc::kPersistMaxSplits * enc::kPersistMaxTokens * h->H * 4);
  a.gelu_tanh = h->gelu == ENC_GELU_TANH ? 1 : 0;
  a.bar = reinterpret_cast<unsigned*>(h->status + 4);
  a.status = h->status;
  a.stall_test = h->stall_test ? 1 : 0;
  a.wait_ns = h->stall_test ? 20000000ull : 2000000000ull;   // 20 ms in the failure test, else 2 s
  cudaError_t e = enc::launch_persistent(a, st);
  if (e != cudaSuccess) return cuda_fail(e, "single-launch forward");
  ++h->launches;
  return ENC_OK;
}

int kernels_per_layer(const enc_handle* h, int tokens) {
  return 7 - (ln_fused(h, tokens, 1) ? 1 : 0) - (ln_fused(h, tokens, 2) ? 1 : 0);
}

// LayerNorm `which` (1 or 2) of z (bias and residual already added).
enc_status step_ln(enc_handle* h, int l, int which, const void* z, void* out, int tokens, cudaStream_t st,
                   const int* rows_dev = nullptr) {
  LayerDev& L = h->layers[l];
  cudaError_t e;
  if (h->dtype == ENC_FP16 && h->H <= 1024)
    e = enc::launch_layernorm_f16h(static_cast<const __half*>(z), which == 1 ? L.h_ln1_g : L.h_ln2_g,
                                   which == 1 ? L.h_ln1_b : L.h_ln2_b, static_cast<__half*>(out), tokens, h->H, st,
                                   rows_dev);
  else if (h->dtype == ENC_FP16)
    e = enc::launch_layernorm_f16(static_cast<const __half*>(z), which == 1 ? L.ln1_g : L.ln2_g,
                                  which == 1 ? L.ln1_b : L.ln2_b, static_cast<__half*>(out), tokens, h->H, st);
  else
    e = enc::launch_layernorm_f32(static_cast<const float*>(z), which == 1 ? L.ln1_g : L.ln2_g,
                                  which == 1 ? L.ln1_b : L.ln2_b, static_cast<float*>(out), tokens, h->H, st);
  if (e != cudaSuccess) return cuda_fail(e, "LayerNorm launch");
  ++h->launches;
  return ENC_OK;
}

enc_status step_ffn1(enc_handle* h, int l, const void* h1, void* u, int tokens, cudaStream_t st) {
  LayerDev& L = h->layers[l];
  const enc::Epi epi = h->gelu == ENC_GELU_TANH ? enc::Epi::kBiasGeluTanh : enc::Epi::kBiasGelu;
  return run_gemm(h, h1, tokens, h->H, L.w_ff1, L.tm_ff1, h->F, epi, L.b_ff1, u, {}, st);
}

// Output projection + add-bias + residual + LayerNorm 1 in one GEMM:
// out = LN1(ctx Wo + bo + resid).
enc_status step_out_proj_ln(enc_handle* h, int l, const void* ctx, const void* resid, void* out, int tokens,
                            cudaStream_t st, const int* m_dev = nullptr) {
  LayerDev& L = h->layers[l];
  return run_gemm(h, ctx, tokens, h->H, L.w_o, L.tm_o, h->H, enc::Epi::kBiasResidLN, L.b_o, out, {}, st, m_dev, resid,
                  L.ln1_g, L.ln1_b);
}

// FFN2 with add-bias and residual in the epilogue: z = u W2 + b2 + resid
// (resid = the first LayerNorm's output).
enc_status step_ffn2(enc_handle* h, int l, const void* u, const void* resid, void* z, int tokens, cudaStream_t st,
                     const int* m_dev = nullptr) {
  LayerDev& L = h->layers[l];
  return run_gemm(h, u, tokens, h->F, L.w_ff2, L.tm_ff2, h->H, enc::Epi::kBiasResidStore, L.b_ff2, z, {}, st, m_dev,
                  resid);
}

// FFN2 + add-bias + residual + LayerNorm 2 in one GEMM: out = LN2(u W2 + b2 + resid).
enc_status step_ffn2_ln(enc_handle* h, int l, const void* u, const void* resid, void* out, int tokens,
                        cudaStream_t st, const int* m_dev = nullptr) {
  LayerDev& L = h->layers[l];
  return run_gemm(h, u, tokens, h->F, L.w_ff2, L.tm_ff2, h->H, enc::Epi::kBiasResidLN, L.b_ff2, out, {}, st, m_dev,
                  resid, L.ln2_g, L.ln2_b);
}

enc_status check_tokens(int batch, int seq) {
  if (batch <= 0 || seq <= 0) return fail(ENC_ERR_INVALID_ARG, "batch (%d) and seq (%d) must be >= 1", batch, seq);
  if (batch > 65535) return fail(ENC_ERR_UNSUPPORTED, "batch %d exceeds 65535", batch);
  if ((long long)batch * seq > (1LL << 30)) return fail(ENC_ERR_UNSUPPORTED, "batch*seq too large");
  return ENC_OK;
}

enc_status check_ptrs(std::initializer_list<const void*> ps) {
  for (const void* p : ps) {
    if (!p) return fail(ENC_ERR_INVALID_ARG, "null buffer pointer");
    if (!aligned16(p)) return fail(ENC_ERR_INVALID_ARG, "buffer %p is not 16-byte aligned", p);
  }
  return ENC_OK;
}

void free_handle(enc_handle* h) {
  if (!h) return;
  for (int i = 0; i < enc_handle::kMaxChunks; ++i) {
    if (h->ev_in[i]) cudaEventDestroy(h->ev_in[i]);
    if (h->ev_done[i]) cudaEventDestroy(h->ev_done[i]);
  }
  if (h->ev_out) cudaEventDestroy(h->ev_out);
  if (h->ev_start) cudaEventDestroy(h->ev_start);
  for (int i = 0; i < 2; ++i) {
    if (h->ev_slot_in[i]) cudaEventDestroy(h->ev_slot_in[i]);
    if (h->ev_slot_done[i]) cudaEventDestroy(h->ev_slot_done[i]);
    if (h->ev_slot_free[i]) cudaEventDestroy(h->ev_slot_free[i]);
  }
  if (h->copy_in) cudaStreamDestroy(h->copy_in);
  if (h->copy_out) cudaStreamDestroy(h->copy_out);
  if (h->param_block) cudaFree(h->param_block);
  if (h->ws) cudaFree(h->ws);
  if (h->stage) cudaFree(h->stage);
  if (h->status) cudaFree(h->status);
  if (h->d_players) cudaFree(h->d_players);
  if (h->d_wmaps) cudaFree(h->d_wmaps);
  if (h->persist_partial) cudaFree(h->persist_partial);
  delete h;
}

// Device staging for the host entry points: two slots of {x, out, valid_len}
// for a batch*seq-token run (slot 0 serves enc_forward_host), plus the copy
// streams and events.  Growing the staging synchronises the device.
size_t host_slot_bytes(const enc_handle* h, int batch, int seq) {
  const size_t act_al = align_up((size_t)batch * seq * h->H * h->esize, 256);
  return 2 * act_al + align_up((size_t)batch * 4, 256);
}

enc_status host_setup(enc_handle* h, int batch, int seq) {
  const size_t need = 2 * host_slot_bytes(h, batch, seq);
  if (need > h->stage_bytes) {
    if (h->stage) {
      cudaDeviceSynchronize();
      cudaFree(h->stage);
      h->stage = nullptr;
      h->stage_bytes = 0;
    }
    if (cudaMalloc(&h->stage, need) != cudaSuccess) {
      cudaGetLastError();
      return fail(ENC_ERR_OOM, "staging allocation of %zu bytes failed", need);
    }
    h->stage_bytes = need;
  }
  if (!h->copy_in) {
    cudaError_t e = cudaStreamCreateWithFlags(&h->copy_in, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&h->copy_out, cudaStreamNonBlocking);
    for (int i = 0; i < enc_handle::kMaxChunks && e == cudaSuccess; ++i) {
      e = cudaEventCreateWithFlags(&h->ev_in[i], cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev_done[i], cudaEventDisableTiming);
    }
    for (int i = 0; i < 2 && e == cudaSuccess; ++i) {
      e = cudaEventCreateWithFlags(&h->ev_slot_in[i], cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev_slot_done[i], cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev_slot_free[i], cudaEventDisableTiming);
    }
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev_out, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev_start, cudaEventDisableTiming);
    if (e != cudaSuccess) return cuda_fail(e, "copy stream setup");
  }
  return ENC_OK;
}

}  // namespace

namespace {
// Whether the launches of the entry point running on this thread use
// programmatic dependent launch: the handle's ENC_OPT_PDL, set for the
// duration of each entry point by a PdlScope.
thread_local bool t_pdl = true;

struct PdlScope {
  bool prev;
  explicit PdlScope(const enc_handle* h) : prev(t_pdl) { t_pdl = h ? h->pdl : true; }
  ~PdlScope() { t_pdl = prev; }
};
}  // namespace

bool enc::pdl_enabled() { return t_pdl; }

int enc::device_sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

extern "C" {

const char* enc_last_error(void) { return g_last_error.c_str(); }

enc_status enc_create(int head_num, int size_per_head, int ffn_dim, int num_layers, enc_dtype dtype,
                      const enc_layer_weights* weights, enc_t* out) {
  if (!out) return fail(ENC_ERR_INVALID_ARG, "out is null");
  *out = nullptr;
  if (head_num <= 0 || size_per_head <= 0 || ffn_dim <= 0 || num_layers <= 0)
    return fail(ENC_ERR_INVALID_ARG, "head_num, size_per_head, ffn_dim and num_layers must be > 0");
  if (size_per_head != 32 && size_per_head != 64 && size_per_head != 128)
    return fail(ENC_ERR_UNSUPPORTED, "size_per_head %d not in {32, 64, 128}", size_per_head);
  if (dtype != ENC_FP16 && dtype != ENC_FP32) return fail(ENC_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
  if (ffn_dim % 8 != 0) return fail(ENC_ERR_INVALID_ARG, "ffn_dim %d is not a multiple of 8", ffn_dim);
  const int H = head_num * size_per_head;
  const int max_h = dtype == ENC_FP16 ? 2048 : 1024;
  if (H > max_h) return fail(ENC_ERR_UNSUPPORTED, "hidden size %d exceeds %d", H, max_h);
  if (!weights) return fail(ENC_ERR_INVALID_ARG, "weights is null");
  for (int l = 0; l < num_layers; ++l) {
    const enc_layer_weights& w = weights[l];
    const void* ps[] = {w.w_qkv, w.b_qkv, w.w_o, w.b_o, w.ln1_g, w.ln1_b,
                        w.w_ff1, w.b_ff1, w.w_ff2, w.b_ff2, w.ln2_g, w.ln2_b};
    for (const void* p : ps)
      if (!p) return fail(ENC_ERR_INVALID_ARG, "layer %d has a null parameter pointer", l);
  }

  int cur_dev = -1;
  if (cudaGetDevice(&cur_dev) != cudaSuccess) return fail(ENC_ERR_CUDA, "no CUDA device");
  int first = -1;
  if (!g_process_device.compare_exchange_strong(first, cur_dev) && first != cur_dev)
    return fail(ENC_ERR_UNSUPPORTED, "handles of one process share one CUDA device (%d); the current device is %d",
                first, cur_dev);

  enc_handle* h = new enc_handle();
  h->nh = head_num; h->d = size_per_head; h->H = H; h->F = ffn_dim; h->L = num_layers;
  h->dtype = dtype;
  h->esize = dtype == ENC_FP16 ? 2 : 4;
  cudaGetDevice(&h->device);
  h->num_sms = enc::device_sm_count();
  if (h->num_sms <= 0) { free_handle(h); return fail(ENC_ERR_CUDA, "no CUDA device"); }
  if (dtype == ENC_FP16) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, h->device) != cudaSuccess || prop.major != 10) {
      free_handle(h);
      return fail(ENC_ERR_UNSUPPORTED, "FP16 mode needs an sm_100 (B200-class) device");
    }
  }
  // The status word, then (16 bytes on) the four barrier words of the single-launch forward.
  if (cudaMalloc(&h->status, 8 * sizeof(int)) != cudaSuccess ||
      cudaMemset(h->status, 0, 8 * sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    free_handle(h);
    return fail(ENC_ERR_OOM, "status word allocation failed");
  }

  const size_t es = h->esize;
  const size_t F = ffn_dim;
  const size_t wsz[4] = {(size_t)H * 3 * H, (size_t)H * H, (size_t)H * F, F * H};
  const size_t vsz[8] = {3 * (size_t)H, (size_t)H, F, (size_t)H, (size_t)H, (size_t)H, (size_t)H, (size_t)H};
  size_t per_layer = 0;
  for (size_t s : wsz) per_layer += align_up(s * es, 256);
  for (size_t s : vsz) per_layer += align_up(s * 4, 256);
  if (dtype == ENC_FP16) per_layer += 4 * align_up((size_t)H * 2, 256);
  size_t staging = 0;
  for (size_t s : wsz) staging = std::max(staging, align_up(s * es, 256));
  if (cudaMalloc(&h->param_block, per_layer * num_layers + staging) != cudaSuccess) {
    cudaGetLastError();
    free_handle(h);
    return fail(ENC_ERR_OOM, "parameter allocation of %zu bytes failed", per_layer * num_layers + staging);
  }
  char* p = static_cast<char*>(h->param_block);
  char* stage = p + per_layer * num_layers;
  h->layers.resize(num_layers);
  cudaStream_t st = nullptr;
  for (int l = 0; l < num_layers; ++l) {
    const enc_layer_weights& w = weights[l];
    LayerDev& L = h->layers[l];
    const void* wsrc[4] = {w.w_qkv, w.w_o, w.w_ff1, w.w_ff2};
    void** wdst[4] = {&L.w_qkv, &L.w_o, &L.w_ff1, &L.w_ff2};
    const int rows[4] = {H, H, H, ffn_dim};           // "in" dimension of each [in, out] matrix
    const int cols[4] = {3 * H, H, ffn_dim, H};
    for (int i = 0; i < 4; ++i) {
      *wdst[i] = p;
      const size_t bytes = wsz[i] * es;
      if (dtype == ENC_FP16) {
        cudaError_t e = cudaMemcpy(stage, wsrc[i], bytes, cudaMemcpyDefault);
        if (e != cudaSuccess) { free_handle(h); return cuda_fail(e, "weight upload"); }
        const dim3 grid((cols[i] + 31) / 32, (rows[i] + 31) / 32);
        transpose_f16_kernel<<<grid, dim3(32, 8), 0, st>>>(reinterpret_cast<const __half*>(stage),
                                                          reinterpret_cast<__half*>(p), rows[i], cols[i]);
        e = cudaDeviceSynchronize();
        if (e == cudaSuccess) e = cudaGetLastError();
        if (e != cudaSuccess) { free_handle(h); return cuda_fail(e, "weight repack"); }
      } else {
        cudaError_t e = cudaMemcpy(p, wsrc[i], bytes, cudaMemcpyDefault);
        if (e != cudaSuccess) { free_handle(h); return cuda_fail(e, "weight upload"); }
      }
      p += align_up(bytes, 256);
    }
    const void* vsrc[8] = {w.b_qkv, w.b_o, w.b_ff1, w.b_ff2, w.ln1_g, w.ln1_b, w.ln2_g, w.ln2_b};
    float** vdst[8] = {&L.b_qkv, &L.b_o, &L.b_ff1, &L.b_ff2, &L.ln1_g, &L.ln1_b, &L.ln2_g, &L.ln2_b};
    for (int i = 0; i < 8; ++i) {
      *vdst[i] = reinterpret_cast<float*>(p);
      const size_t n = vsz[i];
      cudaError_t e = cudaMemcpy(stage, vsrc[i], n * es, cudaMemcpyDefault);
      if (e != cudaSuccess) { free_handle(h); return cuda_fail(e, "parameter upload"); }
      if (dtype == ENC_FP16)
        widen_to_f32_kernel<__half><<<(unsigned)((n + 255) / 256), 256, 0, st>>>(
            reinterpret_cast<const __half*>(stage), *vdst[i], (int)n);
      else
        widen_to_f32_kernel<float><<<(unsigned)((n + 255) / 256), 256, 0, st>>>(
            reinterpret_cast<const float*>(stage), *vdst[i], (int)n);
      e = cudaDeviceSynchronize();
      if (e == cudaSuccess) e = cudaGetLastError();
      if (e != cudaSuccess) { free_handle(h); return cuda_fail(e, "parameter widen"); }
      p += align_up(n * 4, 256);
    }
    if (dtype == ENC_FP16) {
      const void* hsrc[4] = {w.ln1_g, w.ln1_b, w.ln2_g, w.ln2_b};
      __half** hdst[4] = {&L.h_ln1_g, &L.h_ln1_b, &L.h_ln2_g, &L.h_ln2_b};
      for (int i = 0; i < 4; ++i) {
        *hdst[i] = reinterpret_cast<__half*>(p);
        cudaError_t e = cudaMemcpy(p, hsrc[i], (size_t)H * 2, cudaMemcpyDefault);
        if (e != cudaSuccess) { free_handle(h); return cuda_fail(e, "parameter upload"); }
        p += align_up((size_t)H * 2, 256);
      }
    }
    if (dtype == ENC_FP16) {
      // B operands [N, K]: Wqkv^T [3H, H], Wo^T [H, H], W1^T [F, H], W2^T [H, F].
      struct { CUtensorMap* m; void* w; int n, k; } maps[4] = {
          {L.tm_qkv, L.w_qkv, 3 * H, H}, {L.tm_o, L.w_o, H, H}, {L.tm_ff1, L.w_ff1, ffn_dim, H},
          {L.tm_ff2, L.w_ff2, H, ffn_dim}};
      for (auto& m : maps) {
        if (!enc::encode_kmajor_fp16_map(&m.m[0], m.w, m.n, m.k, 128) ||
            !enc::encode_kmajor_fp16_map(&m.m[1], m.w, m.n, m.k, 256)) {
          free_handle(h);
          return fail(ENC_ERR_CUDA, "cuTensorMapEncodeTiled failed for a weight operand");
        }
      }
    }
  }
  if (dtype == ENC_FP16) {
    std::vector<enc::PersistLayer> pl(num_layers);
    for (int l = 0; l < num_layers; ++l) {
      const LayerDev& L = h->layers[l];
      pl[l] = {static_cast<const __half*>(L.w_qkv), static_cast<const __half*>(L.w_o),
               static_cast<const __half*>(L.w_ff1), static_cast<const __half*>(L.w_ff2),
               L.b_qkv, L.b_o, L.b_ff1, L.b_ff2, L.ln1_g, L.ln1_b, L.ln2_g, L.ln2_b};
    }
    const size_t bytes = sizeof(enc::PersistLayer) * num_layers;
    if (cudaMalloc(&h->d_players, bytes) != cudaSuccess) {
      cudaGetLastError();
      free_handle(h);
      return fail(ENC_ERR_OOM, "layer table allocation failed");
    }
    cudaError_t e = cudaMemcpy(h->d_players, pl.data(), bytes, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) { free_handle(h); return cuda_fail(e, "layer table upload"); }
    // Weight maps of the single-launch forward: box of 64 columns x 32 rows.
    std::vector<CUtensorMap> wm((size_t)num_layers * 4);
    for (int l = 0; l < num_layers; ++l) {
      const LayerDev& L = h->layers[l];
      const struct { void* w; int n, k; } ws[4] = {
          {L.w_qkv, 3 * H, H}, {L.w_o, H, H}, {L.w_ff1, ffn_dim, H}, {L.w_ff2, H, ffn_dim}};
      for (int i = 0; i < 4; ++i)
        if (!enc::encode_kmajor_fp16_map(&wm[(size_t)l * 4 + i], ws[i].w, ws[i].n, ws[i].k, 32)) {
          free_handle(h);
          return fail(ENC_ERR_CUDA, "cuTensorMapEncodeTiled failed for a weight operand");
        }
    }
    if (cudaMalloc(&h->d_wmaps, wm.size() * sizeof(CUtensorMap)) != cudaSuccess) {
      cudaGetLastError();
      free_handle(h);
      return fail(ENC_ERR_OOM, "weight map allocation failed");
    }
    e = cudaMemcpy(h->d_wmaps, wm.data(), wm.size() * sizeof(CUtensorMap), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) { free_handle(h); return cuda_fail(e, "weight map upload"); }
    if (H % 32 == 0) {
      const size_t pb = enc::persistent_partial_bytes(H, ffn_dim);
      if (cudaMalloc(&h->persist_partial, pb) != cudaSuccess || cudaMemset(h->persist_partial, 0, pb) != cudaSuccess) {
        cudaGetLastError();
        free_handle(h);
        return fail(ENC_ERR_OOM, "partial-tile allocation of %zu bytes failed", pb);
      }
    }
  }
  *out = h;
  return ok();
}

size_t enc_workspace_bytes(enc_t h, int batch, int seq) {
  if (!h || batch <= 0 || seq <= 0) return 0;
  return workspace_bytes(h, (size_t)batch * seq);
}

enc_status enc_reserve(enc_t h, int batch, int seq) {
  enc_status s = check_handle(h);
  if (s != ENC_OK) return s;
  if ((s = check_tokens(batch, seq)) != ENC_OK) return s;
  if ((s = ensure_workspace(h, (size_t)batch * seq)) != ENC_OK) return s;
  return ok();
}

}  // extern "C"

namespace {

// Padding removal: offsets <- prefix sum of the valid lengths (T = offsets[batch]
// on the device); the valid tokens are packed into [T, H]; every layer runs on
// T rows (GEMMs and LayerNorms read T from the device, attention walks each
// sequence through its offset); the last layer's rows are scattered back into
// out, with zeros in the padded positions.  Kernels: 2 + 7 per layer + 1.
template <typename Mark>
enc_status forward_packed(enc_handle* h, const void* x, const int32_t* valid_len, void* out, int batch, int seq,
                          cudaStream_t st, const Workspace& w, Mark& mark) {
  const int M = batch * seq;                 // most rows any step can hold
  const int H = h->H;
  const int* T = w.offsets + batch;
  cudaError_t e;
  mark();
  e = enc::launch_valid_offsets(valid_len, batch, seq, w.offsets, st);
  if (e != cudaSuccess) return cuda_fail(e, "offsets launch");
  ++h->launches;
  mark();
  e = enc::launch_pack_rows(static_cast<const __half*>(x), valid_len, w.offsets, static_cast<__half*>(w.x1), batch,
                            seq, H, st);
  if (e != cudaSuccess) return cuda_fail(e, "pack launch");
  ++h->launches;
  enc_status s;
  void* last = nullptr;
  for (int l = 0; l < h->L; ++l) {
    LayerDev& L = h->layers[l];
    void* xin = l == 0 ? w.x1 : (((l - 1) & 1) ? w.x1 : w.x0);
    void* xout = (l & 1) ? w.x1 : w.x0;
    mark();
    if ((s = run_gemm(h, xin, M, H, L.w_qkv, L.tm_qkv, 3 * H, enc::Epi::kBiasStore, L.b_qkv, w.qkv, {}, st, T)) !=
        ENC_OK)
      return s;
    mark();
    if (use_tc_attention(h, seq))
      e = enc::launch_attention_tc(static_cast<const __half*>(w.qkv), valid_len, w.offsets,
                                   static_cast<__half*>(w.ctx), batch, seq, h->nh, h->status, st);
    else
      e = enc::launch_attention_f16_packed(static_cast<const __half*>(w.qkv), valid_len, w.offsets,
                                           static_cast<__half*>(w.ctx), batch, seq, h->nh, h->d, st);
    if (e != cudaSuccess) return cuda_fail(e, "attention launch");
    ++h->launches;
    mark();
    if (ln_fused(h, M, 1)) {
      if ((s = step_out_proj_ln(h, l, w.ctx, xin, w.h1, M, st, T)) != ENC_OK) return s;
    } else {
      if ((s = step_out_proj(h, l, w.ctx, xin, w.a, M, st, T)) != ENC_OK) return s;
      mark();
      if ((s = step_ln(h, l, 1, w.a, w.h1, M, st, T)) != ENC_OK) return s;
    }
    mark();
    const enc::Epi gelu = h->gelu == ENC_GELU_TANH ? enc::Epi::kBiasGeluTanh : enc::Epi::kBiasGelu;
    if ((s = run_gemm(h, w.h1, M, H, L.w_ff1, L.tm_ff1, h->F, gelu, L.b_ff1, w.u, {}, st, T)) != ENC_OK) return s;
    mark();
    if (ln_fused(h, M, 2)) {
      if ((s = step_ffn2_ln(h, l, w.u, w.h1, xout, M, st, T)) != ENC_OK) return s;
    } else {
      if ((s = step_ffn2(h, l, w.u, w.h1, w.a, M, st, T)) != ENC_OK) return s;
      mark();
      if ((s = step_ln(h, l, 2, w.a, xout, M, st, T)) != ENC_OK) return s;
    }
    last = xout;
  }
  mark();
  e = enc::launch_unpack_rows(static_cast<const __half*>(last), valid_len, w.offsets, static_cast<__half*>(out), batch,
                              seq, H, st);
  if (e != cudaSuccess) return cuda_fail(e, "unpack launch");
  ++h->launches;
  mark();
  return ENC_OK;
}

// The 7 launches of one dense layer: xin [batch*seq, H] -> xout, with the
// intermediate buffers of `w` (carved for at least batch*seq tokens).
template <typename Mark>
enc_status run_layer(enc_handle* h, int l, const void* xin, void* xout, const int32_t* valid_len, int batch, int seq,
                     const Workspace& w, cudaStream_t st, Mark& mark) {
  const int tokens = batch * seq;
  enc_status s;
  mark();
  if ((s = step_qkv(h, l, xin, w.qkv, batch, seq, st)) != ENC_OK) return s;
  mark();
  if ((s = step_attention(h, w.qkv, valid_len, w.ctx, batch, seq, st)) != ENC_OK) return s;
  mark();
  if (ln_fused(h, tokens, 1)) {
    if ((s = step_out_proj_ln(h, l, w.ctx, xin, w.h1, tokens, st)) != ENC_OK) return s;
  } else {
    if ((s = step_out_proj(h, l, w.ctx, xin, w.a, tokens, st)) != ENC_OK) return s;
    mark();
    if ((s = step_ln(h, l, 1, w.a, w.h1, tokens, st)) != ENC_OK) return s;
  }
  mark();
  if ((s = step_ffn1(h, l, w.h1, w.u, tokens, st)) != ENC_OK) return s;
  mark();
  if (ln_fused(h, tokens, 2)) return step_ffn2_ln(h, l, w.u, w.h1, xout, tokens, st);
  if ((s = step_ffn2(h, l, w.u, w.h1, w.a, tokens, st)) != ENC_OK) return s;
  mark();
  return step_ln(h, l, 2, w.a, xout, tokens, st);
}

// Checks, workspace, and the per-layer launches of one forward on `st`.
enc_status forward_impl(enc_handle* h, const void* x, const int32_t* valid_len, void* out, int batch, int seq,
                        cudaStream_t st, bool tracing) {
  enc_status s = check_handle(h);
  if (s != ENC_OK) return s;
  if (h->decoder) return fail(ENC_ERR_INVALID_ARG, "a decoder handle runs enc_decoder_forward");
  if ((s = check_tokens(batch, seq)) != ENC_OK) return s;
  if ((s = check_ptrs({x, out})) != ENC_OK) return s;
  if (!valid_len) return fail(ENC_ERR_INVALID_ARG, "valid_len is null");
  const size_t M = (size_t)batch * seq;
  const size_t bytes = M * h->H * h->esize;
  const char* xb = static_cast<const char*>(x);
  const char* ob = static_cast<const char*>(out);
  if (xb < ob + bytes && ob < xb + bytes) return fail(ENC_ERR_INVALID_ARG, "out overlaps x");
  if ((s = ensure_workspace(h, M)) != ENC_OK) return s;
  Workspace w = carve(h, M);
  const int tokens = (int)M;
  tracing = tracing && !h->trace.empty();
  if (tracing && (int)h->trace.size() < enc_kernels_per_forward(h, batch, seq) + 1)
    return fail(ENC_ERR_INVALID_ARG, "need %d trace events for this forward, got %d",
                enc_kernels_per_forward(h, batch, seq) + 1, (int)h->trace.size());
  int k = 0;
  auto mark = [&]() {
    if (tracing) cudaEventRecord(h->trace[k++], st);
  };
  if (h->packed) return forward_packed(h, x, valid_len, out, batch, seq, st, w, mark);
  if (use_persistent(h, batch, seq)) {
    mark();
    if ((s = run_persistent(h, x, valid_len, out, batch, seq, w, st)) != ENC_OK) return s;
    mark();
    return ENC_OK;
  }
  (void)tokens;
  for (int l = 0; l < h->L; ++l) {
    const void* xin = l == 0 ? x : (((l - 1) & 1) ? w.x1 : w.x0);
    void* xout = l == h->L - 1 ? out : ((l & 1) ? w.x1 : w.x0);
    if ((s = run_layer(h, l, xin, xout, valid_len, batch, seq, w, st, mark)) != ENC_OK) return s;
  }
  mark();
  return ENC_OK;
}

}  // namespace

struct enc_graph_s {
  enc_handle* h = nullptr;
  int kernels = 0;          // launches one replay issues
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
};

extern "C" {

enc_status enc_forward(enc_t h, const void* x, const int32_t* valid_len, void* out, int batch, int seq,
                       enc_stream_t stream) {
  PdlScope pdl(h);
  enc_status s = forward_impl(h, x, valid_len, out, batch, seq, reinterpret_cast<cudaStream_t>(stream), true);
  return s == ENC_OK ? ok() : s;
}

enc_status enc_graph_create(enc_t h, const void* x, const int32_t* valid_len, void* out, int batch, int seq,
                            enc_graph_t* graph) {
  if (!graph) return fail(ENC_ERR_INVALID_ARG, "graph is null");
  *graph = nullptr;
  enc_status s = check_handle(h);
  if (s != ENC_OK) return s;
  if ((s = check_tokens(batch, seq)) != ENC_OK) return s;
  if ((s = ensure_workspace(h, (size_t)batch * seq)) != ENC_OK) return s;   // no allocation while recording
  PdlScope pdl(h);
  cudaStream_t st = nullptr;
  cudaError_t e = cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamCreate");
  const uint64_t launches_before = h->launches;
  e = cudaStreamBeginCapture(st, cudaStreamCaptureModeThreadLocal);
  if (e != cudaSuccess) {
    cudaStreamDestroy(st);
    return cuda_fail(e, "cudaStreamBeginCapture");
  }
  s = forward_impl(h, x, valid_len, out, batch, seq, st, false);
  cudaGraph_t g = nullptr;
  e = cudaStreamEndCapture(st, &g);
  cudaStreamDestroy(st);
  const int recorded = static_cast<int>(h->launches - launches_before);
  h->launches = launches_before;            // recording launches nothing
  if (s != ENC_OK) {
    if (g) cudaGraphDestroy(g);
    return s;
  }
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamEndCapture");
  cudaGraphExec_t exec = nullptr;
  e = cudaGraphInstantiate(&exec, g, 0);
  if (e != cudaSuccess) {
    cudaGraphDestroy(g);
    return cuda_fail(e, "cudaGraphInstantiate");
  }
  enc_graph_s* out_g = new enc_graph_s();
  out_g->h = h;
  out_g->kernels = recorded;
  out_g->graph = g;
  out_g->exec = exec;
  ++h->graphs_alive;
  *graph = out_g;
  return ok();
}

enc_status enc_graph_launch(enc_graph_t graph, enc_stream_t stream) {
  if (!graph) return fail(ENC_ERR_INVALID_ARG, "null graph");
  cudaError_t e = cudaGraphLaunch(graph->exec, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaGraphLaunch");
  graph->h->launches += graph->kernels;
  return ok();
}

enc_status enc_graph_destroy(enc_graph_t graph) {
  if (!graph) return ok();
  cudaDeviceSynchronize();
  if (graph->exec) cudaGraphExecDestroy(graph->exec);
  if (graph->graph) cudaGraphDestroy(graph->graph);
  if (graph->h) --graph->h->graphs_alive;
  delete graph;
  return ok();
}

}  // extern "C"

// ------------------------------------------------- forward without allocation

// Scratch of enc_forward_noalloc: a fixed array in the library's own device
// image, so that the entry point needs no cudaMalloc.  Every GPU that loads the
// library holds it until the process exits.
static __device__ __align__(256) unsigned char g_static_workspace[ENC_STATIC_WORKSPACE_BYTES];

namespace {

// In host code g_static_workspace names a host-side stand-in, not device
// memory; its device address is looked up once per device, with that device
// current, and kept here.
constexpr int kMaxStaticDevices = 64;
std::mutex g_static_ws_mutex;
void* g_static_ws_addr[kMaxStaticDevices] = {};

enc_status static_workspace_address(int device, void** ptr) {
  if (device < 0 || device >= kMaxStaticDevices)
    return fail(ENC_ERR_UNSUPPORTED, "device %d is beyond the %d the static workspace table holds", device,
                kMaxStaticDevices);
  std::lock_guard<std::mutex> lock(g_static_ws_mutex);
  if (!g_static_ws_addr[device]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_static_workspace);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the static workspace");
    g_static_ws_addr[device] = p;
  }
  *ptr = g_static_ws_addr[device];
  return ENC_OK;
}

// The workspace layout of carve(), laid out from `base` instead of the
// handle's own allocation.
Workspace carve_at(const enc_handle* h, void* base, size_t tokens) {
  const size_t es = h->esize;
  const size_t mh = align_up(tokens * h->H * es, 256);
  const size_t mf = align_up(tokens * h->F * es, 256);
  char* p = static_cast<char*>(base);
  Workspace w;
  w.qkv = p; p += 3 * mh;
  w.ctx = p; p += mh;
  w.a = p; p += mh;
  w.h1 = p; p += mh;
  w.u = p; p += mf;
  w.x0 = p; p += mh;
  w.x1 = p; p += mh;
  w.offsets = reinterpret_cast<int32_t*>(p);
  return w;
}

}  // namespace

extern "C" {

enc_status enc_forward_noalloc(enc_t h, const void* x, const int32_t* valid_len, void* out, int batch, int seq,
                               enc_stream_t stream) {
  enc_status s = check_handle(h);
  if (s != ENC_OK) return s;
  if ((s = check_tokens(batch, seq)) != ENC_OK) return s;
  if ((s = check_ptrs({x, out})) != ENC_OK) return s;
  if (!valid_len) return fail(ENC_ERR_INVALID_ARG, "valid_len is null");
  const size_t M = (size_t)batch * seq;
  const size_t bytes = M * h->H * h->esize;
  const char* xb = static_cast<const char*>(x);
  const char* ob = static_cast<const char*>(out);
  if (xb < ob + bytes && ob < xb + bytes) return fail(ENC_ERR_INVALID_ARG, "out overlaps x");
  const size_t need = workspace_bytes(h, M);
  if (need > ENC_STATIC_WORKSPACE_BYTES)
    return fail(ENC_ERR_UNSUPPORTED,
                "batch %d x seq %d needs %zu bytes of scratch; the static workspace of enc_forward_noalloc holds %zu",
                batch, seq, need, (size_t)ENC_STATIC_WORKSPACE_BYTES);
  void* base = nullptr;
  if ((s = static_workspace_address(h->device, &base)) != ENC_OK) return s;
  PdlScope pdl(h);
  const Workspace w = carve_at(h, base, M);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  auto no_mark = [] {};
  if (h->packed) {
    s = forward_packed(h, x, valid_len, out, batch, seq, st, w, no_mark);
    return s == ENC_OK ? ok() : s;
  }
  for (int l = 0; l < h->L; ++l) {
    const void* xin = l == 0 ? x : (((l - 1) & 1) ? w.x1 : w.x0);
    void* xout = l == h->L - 1 ? out : ((l & 1) ? w.x1 : w.x0);
    if ((s = run_layer(h, l, xin, xout, valid_len, batch, seq, w, st, no_mark)) != ENC_OK) return s;
  }
  return ok();
}

enc_status enc_forward_host(enc_t h, const void* x, const int32_t* valid_len, void* out, int batch, int seq,
                            enc_stream_t stream) {
  enc_status s = check_handle(h);
  if (s != ENC_OK) return s;
  PdlScope pdl(h);
  if ((s = check_tokens(batch, seq)) != ENC_OK) return s;
  if (!x || !valid_len || !out) return fail(ENC_ERR_INVALID_ARG, "null host buffer");
  const size_t seq_bytes = (size_t)seq * h->H * h->esize;
  const size_t act_al = align_up((size_t)batch * seq_bytes, 256);
  if ((s = host_setup(h, batch, seq)) != ENC_OK) return s;
  // Sequences are independent, so the batch can be cut into chunks: the first
  // layer runs chunk by chunk as each chunk's input lands, the middle layers
  // run on the whole batch, and the last layer runs chunk by chunk so that each
  // chunk's output is copied out while the next one is computed.  Only the
  // first and last layers pay the smaller GEMMs.  One chunk, a packed forward,
  // or fewer than 2 layers: copy in, run, copy out.
  const long tokens = (long)batch * seq;
  int chunks = (int)std::min<long>(h->host_chunks, std::max<long>(1, tokens / 2048));
  chunks = std::min(chunks, batch);
  if (h->packed || h->L < 2) chunks = 1;
  char* base = static_cast<char*>(h->stage);
  char* dx = base;
  char* dout = base + act_al;
  int32_t* dvl = reinterpret_cast<int32_t*>(base + 2 * act_al);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const char* hx = static_cast<const char*>(x);
  char* hout = static_cast<char*>(out);
  // Copies start after the caller's earlier work on `st` and after any output
  // copy of enc_forward_host_async still reading the staging.
  cudaError_t e = cudaEventRecord(h->ev_start, st);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(h->copy_in, h->ev_start, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(h->copy_out, h->ev_start, 0);
  for (int k = 0; k < 2 && e == cudaSuccess; ++k) e = cudaStreamWaitEvent(h->copy_in, h->ev_slot_free[k], 0);
  if (e == cudaSuccess) e = cudaMemcpyAsync(dvl, valid_len, (size_t)batch * 4, cudaMemcpyHostToDevice, h->copy_in);
  if (e != cudaSuccess) return cuda_fail(e, "host-to-device copy");
  int cb[enc_handle::kMaxChunks + 1];
  cb[0] = 0;
  for (int c = 0; c < chunks; ++c) cb[c + 1] = cb[c] + batch / chunks + (c < batch % chunks ? 1 : 0);
  for (int c = 0; c < chunks; ++c) {
    const size_t off = (size_t)cb[c] * seq_bytes, bytes = (size_t)(cb[c + 1] - cb[c]) * seq_bytes;
    e = cudaMemcpyAsync(dx + off, hx + off, bytes, cudaMemcpyHostToDevice, h->copy_in);
    if (e == cudaSuccess) e = cudaEventRecord(h->ev_in[c], h->copy_in);
    if (e != cudaSuccess) return cuda_fail(e, "host-to-device copy");
  }
  auto copy_out_chunk = [&](int c) -> enc_status {
    const size_t off = (size_t)cb[c] * seq_bytes, bytes = (size_t)(cb[c + 1] - cb[c]) * seq_bytes;
    cudaError_t ce = cudaEventRecord(h->ev_done[c], st);
    if (ce == cudaSuccess) ce = cudaStreamWaitEvent(h->copy_out, h->ev_done[c], 0);
    if (ce == cudaSuccess) ce = cudaMemcpyAsync(hout + off, dout + off, bytes, cudaMemcpyDeviceToHost, h->copy_out);
    return ce == cudaSuccess ? ENC_OK : cuda_fail(ce, "device-to-host copy");
  };
  if (chunks == 1) {
    e = cudaStreamWaitEvent(st, h->ev_in[0], 0);
    if (e != cudaSuccess) return cuda_fail(e, "stream wait");
    if ((s = forward_impl(h, dx, dvl, dout, batch, seq, st, false)) != ENC_OK) return s;
    if ((s = copy_out_chunk(0)) != ENC_OK) return s;
  } else {
    if ((s = check_handle(h)) != ENC_OK) return s;
    if ((s = ensure_workspace(h, (size_t)tokens)) != ENC_OK) return s;
    const Workspace w = carve(h, (size_t)tokens);
    auto no_mark = [] {};
    const int L = h->L;
    for (int c = 0; c < chunks; ++c) {          // layer 0, chunk by chunk
      const size_t off = (size_t)cb[c] * seq_bytes;
      e = cudaStreamWaitEvent(st, h->ev_in[c], 0);
      if (e != cudaSuccess) return cuda_fail(e, "stream wait");
      if ((s = run_layer(h, 0, dx + off, static_cast<char*>(w.x0) + off, dvl + cb[c], cb[c + 1] - cb[c], seq, w, st,
                         no_mark)) != ENC_OK)
        return s;
    }
    for (int l = 1; l < L - 1; ++l) {            // middle layers, whole batch
      const void* xin = ((l - 1) & 1) ? w.x1 : w.x0;
      void* xo = (l & 1) ? w.x1 : w.x0;
      if ((s = run_layer(h, l, xin, xo, dvl, batch, seq, w, st, no_mark)) != ENC_OK) return s;
    }
    const char* xlast = static_cast<const char*>(((L - 2) & 1) ? w.x1 : w.x0);
    for (int c = 0; c < chunks; ++c) {          // last layer, chunk by chunk, each copied out at once
      const size_t off = (size_t)cb[c] * seq_bytes;
      if ((s = run_layer(h, L - 1, xlast + off, dout + off, dvl + cb[c], cb[c + 1] - cb[c], seq, w, st, no_mark)) !=
          ENC_OK)
        return s;
      if ((s = copy_out_chunk(c)) != ENC_OK) return s;
    }
  }
  e = cudaEventRecord(h->ev_out, h->copy_out);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st, h->ev_out, 0);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "device-to-host copy");
  return ok();
}

enc_status enc_forward_host_async(enc_t h, const void* x, const int32_t* valid_len, void* out, int batch, int seq,
                                  enc_stream_t stream) {
  enc_status s = check_handle(h);
  if (s != ENC_OK) return s;
  PdlScope pdl(h);
  if ((s = check_tokens(batch, seq)) != ENC_OK) return s;
  if (!x || !valid_len || !out) return fail(ENC_ERR_INVALID_ARG, "null host buffer");
  if ((s = host_setup(h, batch, seq)) != ENC_OK) return s;
  const int k = h->host_slot;
  const size_t act = (size_t)batch * seq * h->H * h->esize;
  const size_t act_al = align_up(act, 256);
  // The two slots split the staging allocation in halves, whatever the shape of
  // the call that allocated it: a call smaller than the previous one must not
  // place its slot inside the other slot, whose run may still be in flight.
  const size_t slot_stride = h->stage_bytes / 2;
  if (host_slot_bytes(h, batch, seq) > slot_stride)
    return fail(ENC_ERR_CUDA, "staging slot of %zu bytes is smaller than the %zu this call needs", slot_stride,
                host_slot_bytes(h, batch, seq));
  char* base = static_cast<char*>(h->stage) + (size_t)k * slot_stride;
  char* dx = base;
  char* dout = base + act_al;
  int32_t* dvl = reinterpret_cast<int32_t*>(base + 2 * act_al);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // The slot's previous run (two calls ago) has copied its output out.
  cudaError_t e = cudaStreamWaitEvent(h->copy_in, h->ev_slot_free[k], 0);
  if (e == cudaSuccess) e = cudaMemcpyAsync(dvl, valid_len, (size_t)batch * 4, cudaMemcpyHostToDevice, h->copy_in);
  if (e == cudaSuccess) e = cudaMemcpyAsync(dx, x, act, cudaMemcpyHostToDevice, h->copy_in);
  if (e == cudaSuccess) e = cudaEventRecord(h->ev_slot_in[k], h->copy_in);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st, h->ev_slot_in[k], 0);
  if (e != cudaSuccess) return cuda_fail(e, "host-to-device copy");
  if ((s = forward_impl(h, dx, dvl, dout, batch, seq, st, false)) != ENC_OK) return s;
  e = cudaEventRecord(h->ev_slot_done[k], st);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(h->copy_out, h->ev_slot_done[k], 0);
  if (e == cudaSuccess) e = cudaMemcpyAsync(out, dout, act, cudaMemcpyDeviceToHost, h->copy_out);
  if (e == cudaSuccess) e = cudaEventRecord(h->ev_slot_free[k], h->copy_out);
  if (e != cudaSuccess) return cuda_fail(e, "device-to-host copy");
  h->host_slot = k ^ 1;
  return ok();
}

enc_status enc_host_join(enc_t h, enc_stream_t stream) {
  enc_status s = check_handle(h);
  if (s != ENC_OK) return s;
  if (!h->copy_out) return ok();                       // no host call yet
  cudaError_t e = cudaEventRecord(h->ev_out, h->copy_out);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(reinterpret_cast<cudaStream_t>(stream), h->ev_out, 0);
  if (e != cudaSuccess) return cuda_fail(e, "join");
  return ok();
}

enc_status enc_destroy(enc_t h) {
  if (!h) return ok();
  cudaDeviceSynchronize();
  free_handle(h);
  return ok();
}

enc_status enc_device_status(enc_t h, int32_t* code) {
  enc_status s = check_handle(h);
  if (s != ENC_OK) return s;
  if (!code) return fail(ENC_ERR_INVALID_ARG, "code is null");
  int v = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(&v, h->status, sizeof(int), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(h->status, 0, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  *code = v;
  if (v != 0) return fail(ENC_ERR_DEVICE, "a kernel reported device status %d", v);
  return ok();
}

int enc_kernels_per_forward(enc_t h, int batch, int seq) {
  if (!h || batch <= 0 || seq <= 0) return 0;
  if (use_persistent(h, batch, seq)) return 1;
  return kernels_per_layer(h, batch * seq) * h->L + (h->packed ? 3 : 0);
}

enc_status enc_set_packing(enc_t h, int enable) {
  if (!h) return fail(ENC_ERR_INVALID_ARG, "null handle");
  if (enable && (h->dtype != ENC_FP16 || h->H > 1024))
    return fail(ENC_ERR_UNSUPPORTED, "padding removal needs FP16 mode and hidden size <= 1024");
  h->packed = enable != 0;
  return ok();
}

enc_status enc_set_option(enc_t h, enc_option option, int value) {
  if (!h) return fail(ENC_ERR_INVALID_ARG, "null handle");
  const bool three = option == ENC_OPT_LN_FUSE_FFN2 || option == ENC_OPT_LN_FUSE_OUT_PROJ;
  if (value < 0 || value > (three ? 2 : 1))
    return fail(ENC_ERR_INVALID_ARG, "option %d takes 0..%d, not %d", (int)option, three ? 2 : 1, value);
  const bool v = value != 0;
  switch (option) {
    case ENC_OPT_PAIR_TILES: h->pair_tiles = v; break;
    case ENC_OPT_TMA_STORE: h->tma_store = v; break;
    case ENC_OPT_TC_ATTENTION: h->tc_attn = v; break;
    case ENC_OPT_SPLIT_K: h->splitk = v; break;
    case ENC_OPT_LN_FUSE_FFN2: h->ln_fuse_ffn2 = value; break;
    case ENC_OPT_LN_FUSE_OUT_PROJ: h->ln_fuse_oproj = value; break;
    case ENC_OPT_PDL: h->pdl = v; break;
    case ENC_OPT_PERSISTENT: h->persistent = v; break;
    case ENC_OPT_TEST_STALL: h->stall_test = v; break;
    default: return fail(ENC_ERR_INVALID_ARG, "unknown option %d", (int)option);
  }
  return ok();
}

enc_status enc_get_option(enc_t h, enc_option option, int* value) {
  if (!h) return fail(ENC_ERR_INVALID_ARG, "null handle");
  if (!value) return fail(ENC_ERR_INVALID_ARG, "value is null");
  int v;
  switch (option) {
    case ENC_OPT_PAIR_TILES: v = h->pair_tiles; break;
    case ENC_OPT_TMA_STORE: v = h->tma_store; break;
    case ENC_OPT_TC_ATTENTION: v = h->tc_attn; break;
    case ENC_OPT_SPLIT_K: v = h->splitk; break;
    case ENC_OPT_LN_FUSE_FFN2: v = h->ln_fuse_ffn2; break;
    case ENC_OPT_LN_FUSE_OUT_PROJ: v = h->ln_fuse_oproj; break;
    case ENC_OPT_PDL: v = h->pdl; break;
    case ENC_OPT_PERSISTENT: v = h->persistent; break;
    case ENC_OPT_TEST_STALL: v = h->stall_test; break;
    default: return fail(ENC_ERR_INVALID_ARG, "unknown option %d", (int)option);
  }
  *value = v;
  return ok();
}

enc_status enc_set_host_chunks(enc_t h, int chunks) {
  if (!h) return fail(ENC_ERR_INVALID_ARG, "null handle");
  if (chunks < 1 || chunks > enc_handle::kMaxChunks)
    return fail(ENC_ERR_INVALID_ARG, "chunks must be in [1, %d]", enc_handle::kMaxChunks);
  h->host_chunks = chunks;
  return ok();
}

enc_status enc_set_gelu(enc_t h, enc_gelu form) {
  if (!h) return fail(ENC_ERR_INVALID_ARG, "null handle");
  if (form != ENC_GELU_ERF && form != ENC_GELU_TANH) return fail(ENC_ERR_INVALID_ARG, "unknown GELU form %d", (int)form);
  h->gelu = form;
  return ok();
}

uint64_t enc_launch_count(enc_t h) { return h ? h->launches : 0; }

enc_status enc_set_trace_events(enc_t h, void* const* events, int count) {
  if (!h) return fail(ENC_ERR_INVALID_ARG, "null handle");
  if (!events || count == 0) {
    h->trace.clear();
    return ok();
  }
  if (count < 2) return fail(ENC_ERR_INVALID_ARG, "need at least 2 trace events, got %d", count);
  h->trace.assign(reinterpret_cast<cudaEvent_t const*>(events), reinterpret_cast<cudaEvent_t const*>(events) + count);
  return ok();
}

// ---------------------------------------------------------------- single steps

static enc_status op_prologue(enc_t h, int layer, bool needs_layer, int tokens) {
  enc_status s = check_handle(h);
  if (s != ENC_OK) return s;
  if (h->decoder) return fail(ENC_ERR_INVALID_ARG, "single encoder steps need an encoder handle");
  if (needs_layer && (layer < 0 || layer >= h->L)) return fail(ENC_ERR_INVALID_ARG, "layer %d out of range", layer);
  if (tokens <= 0) return fail(ENC_ERR_INVALID_ARG, "token count must be >= 1");
  return ENC_OK;
}

enc_status enc_op_qkv(enc_t h, int layer, const void* x, void* qkv, int batch, int seq, enc_stream_t stream) {
  enc_status s = op_prologue(h, layer, true, batch > 0 && seq > 0 ? batch * seq : 0);
  if (s != ENC_OK) return s;
  PdlScope pdl(h);
  if ((s = check_tokens(batch, seq)) != ENC_OK) return s;
  if ((s = check_ptrs({x, qkv})) != ENC_OK) return s;
  if ((s = step_qkv(h, layer, x, qkv, batch, seq, reinterpret_cast<cudaStream_t>(stream))) != ENC_OK) return s;
  return ok();
}

enc_status enc_op_attention(enc_t h, const void* qkv, const int32_t* valid_len, void* ctx, int batch, int seq,
                            enc_stream_t stream) {
  enc_status s = op_prologue(h, 0, false, batch > 0 && seq > 0 ? batch * seq : 0);
  if (s != ENC_OK) return s;
  PdlScope pdl(h);
  if ((s = check_tokens(batch, seq)) != ENC_OK) return s;
  if ((s = check_ptrs({qkv, ctx})) != ENC_OK) return s;
  if (!valid_len) return fail(ENC_ERR_INVALID_ARG, "valid_len is null");
  if ((s = step_attention(h, qkv, valid_len, ctx, batch, seq, reinterpret_cast<cudaStream_t>(stream))) != ENC_OK)
    return s;
  return ok();
}

enc_status enc_op_out_proj_ln(enc_t h, int layer, const void* ctx, const void* resid, void* out, int tokens,
                              enc_stream_t stream) {
  enc_status s = op_prologue(h, layer, true, tokens);
  if (s != ENC_OK) return s;
  PdlScope pdl(h);
  if ((s = check_ptrs({ctx, resid, out})) != ENC_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (ln_fused(h, tokens, 1)) {
    if ((s = step_out_proj_ln(h, layer, ctx, resid, out, tokens, st)) != ENC_OK) return s;
    return ok();
  }
  if ((s = ensure_workspace(h, (size_t)tokens)) != ENC_OK) return s;   // z in the workspace
  const Workspace w = carve(h, (size_t)tokens);
  if ((s = step_out_proj(h, layer, ctx, resid, w.a, tokens, st)) != ENC_OK) return s;
  if ((s = step_ln(h, layer, 1, w.a, out, tokens, st)) != ENC_OK) return s;
  return ok();
}

enc_status enc_op_ffn1(enc_t h, int layer, const void* h1, void* u, int tokens, enc_stream_t stream) {
  enc_status s = op_prologue(h, layer, true, tokens);
  if (s != ENC_OK) return s;
  PdlScope pdl(h);
  if ((s = check_ptrs({h1, u})) != ENC_OK) return s;
  if ((s = step_ffn1(h, layer, h1, u, tokens, reinterpret_cast<cudaStream_t>(stream))) != ENC_OK) return s;
  return ok();
}

enc_status enc_op_ffn2_ln(enc_t h, int layer, const void* u, const void* resid, void* out, int tokens,
                          enc_stream_t stream) {
  enc_status s = op_prologue(h, layer, true, tokens);
  if (s != ENC_OK) return s;
  PdlScope pdl(h);
  if ((s = check_ptrs({u, resid, out})) != ENC_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (ln_fused(h, tokens, 2)) {
    if ((s = step_ffn2_ln(h, layer, u, resid, out, tokens, st)) != ENC_OK) return s;
    return ok();
  }
  if ((s = ensure_workspace(h, (size_t)tokens)) != ENC_OK) return s;   // z in the workspace
  const Workspace w = carve(h, (size_t)tokens);
  if ((s = step_ffn2(h, layer, u, resid, w.a, tokens, st)) != ENC_OK) return s;
  if ((s = step_ln(h, layer, 2, w.a, out, tokens, st)) != ENC_OK) return s;
  return ok();
}

}  // extern "C"

// ------------------------------------------------------------------ decoder forward
//
// [FT] "什么是 Faster Transformer" plans a decoder without describing it.  The
// layer here is the post-LN Transformer decoder layer over a whole target
// sequence, with the encoder's conventions (see enc.h), run as 12 launches:
//   1 GEMM   y Wqkv + bqkv, head split [3, B, nh, T, d]
//   2 attention (causal, keys j < tgt_len)
//   3 GEMM   ctx Wo + bo + y           4 LayerNorm 1 -> h1
//   5 GEMM   h1 Wq2 + bq2, head split [1, B, nh, T, d]
//   6 GEMM   mem Wkv2 + bkv2, head split [2, B, nh, S, d]
//   7 attention (cross, keys j < mem_len)
//   8 GEMM   ctx2 Wo2 + bo2 + h1       9 LayerNorm 2 -> h2
//  10 GEMM   GELU(h2 W1 + b1)         11 GEMM u W2 + b2 + h2     12 LayerNorm 3

namespace {

// Workspace of a decoder forward: qkv 3Mt H, ctx, z, h1, h2, q2 (Mt H each),
// kv2 2 Ms H, u Mt F, two ping-pong layer outputs (Mt H each).
struct DecWorkspace {
  void *qkv, *ctx, *z, *h1, *h2, *q2, *kv2, *u, *x0, *x1;
};

size_t dec_workspace_bytes(const enc_handle* h, size_t mt, size_t ms) {
  const size_t mh = align_up(mt * h->H * 2, 256), sh = align_up(ms * h->H * 2, 256);
  const size_t mf = align_up(mt * h->F * 2, 256);
  return 3 * mh + 5 * mh + 2 * sh + mf + 2 * mh;
}

DecWorkspace dec_carve(const enc_handle* h, size_t mt, size_t ms) {
  const size_t mh = align_up(mt * h->H * 2, 256), sh = align_up(ms * h->H * 2, 256);
  const size_t mf = align_up(mt * h->F * 2, 256);
  char* p = static_cast<char*>(h->ws);
  DecWorkspace w;
  w.qkv = p; p += 3 * mh;
  w.ctx = p; p += mh;
  w.z = p; p += mh;
  w.h1 = p; p += mh;
  w.h2 = p; p += mh;
  w.q2 = p; p += mh;
  w.kv2 = p; p += 2 * sh;
  w.u = p; p += mf;
  w.x0 = p; p += mh;
  w.x1 = p;
  return w;
}

enc_status ensure_bytes(enc_handle* h, size_t need) {
  if (need <= h->ws_bytes) return ENC_OK;
  if (h->graphs_alive > 0)
    return fail(ENC_ERR_INVALID_ARG, "workspace of %zu bytes needed but %d recorded graph(s) pin the current one",
                need, h->graphs_alive);
  if (h->ws) {
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize before workspace growth");
    cudaFree(h->ws);
    h->ws = nullptr;
    h->ws_bytes = 0;
  }
  void* p = nullptr;
  if (cudaMalloc(&p, need) != cudaSuccess) {
    cudaGetLastError();
    return fail(ENC_ERR_OOM, "workspace allocation of %zu bytes failed", need);
  }
  h->ws = p;
  h->ws_bytes = need;
  return ENC_OK;
}

enc_status dec_ln(enc_handle* h, const void* z, const __half* g, const __half* b, void* out, int rows,
                  cudaStream_t st) {
  cudaError_t e = enc::launch_layernorm_f16h(static_cast<const __half*>(z), g, b, static_cast<__half*>(out), rows,
                                             h->H, st);
  if (e != cudaSuccess) return cuda_fail(e, "LayerNorm launch");
  ++h->launches;
  return ENC_OK;
}

enc_status dec_attention(enc_handle* h, const void* q, const void* k, const void* v, const int32_t* kv_len, void* ctx,
                         int batch, int tgt_seq, int kv_seq, bool causal, cudaStream_t st) {
  cudaError_t e = enc::launch_decoder_attention(static_cast<const __half*>(q), static_cast<const __half*>(k),
                                                static_cast<const __half*>(v), kv_len, static_cast<__half*>(ctx),
                                                batch, h->nh, h->d, tgt_seq, kv_seq, causal, st);
  if (e != cudaSuccess) return cuda_fail(e, "decoder attention launch");
  ++h->launches;
  return ENC_OK;
}

enc_status dec_layer(enc_handle* h, int l, const void* yin, void* yout, const int32_t* tgt_len, const void* mem,
                     const int32_t* mem_len, int B, int T, int S, const DecWorkspace& w, cudaStream_t st) {
  DecLayerDev& L = h->dlayers[l];
  const int H = h->H, Mt = B * T, Ms = B * S;
  const size_t hd = (size_t)B * h->nh * h->d;   // elements of one [B, nh, ., d] block per token
  enc_status s;
  const enc::SplitShape spt{B, T, h->nh, h->d}, sps{B, S, h->nh, h->d};
  if ((s = run_gemm(h, yin, Mt, H, L.w_qkv, L.tm_qkv, 3 * H, enc::Epi::kBiasQkvSplit, L.b_qkv, w.qkv, spt, st)) !=
      ENC_OK)
    return s;
  const __half* qkv = static_cast<const __half*>(w.qkv);
  if ((s = dec_attention(h, qkv, qkv + hd * T, qkv + 2 * hd * T, tgt_len, w.ctx, B, T, T, true, st)) != ENC_OK)
    return s;
  // GEMM + bias + residual + LayerNorm i: in the GEMM epilogue where the
  // encoder fuses it (2-CTA tiles, the same options), else through z and the
  // LayerNorm kernel.
  auto resid_ln = [&](const void* A, int K, void* W, const CUtensorMap* tm, const float* b, const void* resid, int i,
                      int which, void* out) -> enc_status {
    if (ln_fused(h, Mt, which))
      return run_gemm(h, A, Mt, K, W, tm, H, enc::Epi::kBiasResidLN, b, out, {}, st, nullptr, resid, L.ln_gf[i],
                      L.ln_bf[i]);
    enc_status r = run_gemm(h, A, Mt, K, W, tm, H, enc::Epi::kBiasResidStore, b, w.z, {}, st, nullptr, resid);
    return r != ENC_OK ? r : dec_ln(h, w.z, L.ln_g[i], L.ln_b[i], out, Mt, st);
  };
  if ((s = resid_ln(w.ctx, H, L.w_o, L.tm_o, L.b_o, yin, 0, 1, w.h1)) != ENC_OK) return s;
  if ((s = run_gemm(h, w.h1, Mt, H, L.w_q2, L.tm_q2, H, enc::Epi::kBiasQkvSplit, L.b_q2, w.q2, spt, st)) != ENC_OK)
    return s;
  if ((s = run_gemm(h, mem, Ms, H, L.w_kv2, L.tm_kv2, 2 * H, enc::Epi::kBiasQkvSplit, L.b_kv2, w.kv2, sps, st)) !=
      ENC_OK)
    return s;
  const __half* kv2 = static_cast<const __half*>(w.kv2);
  if ((s = dec_attention(h, w.q2, kv2, kv2 + hd * S, mem_len, w.ctx, B, T, S, false, st)) != ENC_OK) return s;
  if ((s = resid_ln(w.ctx, H, L.w_o2, L.tm_o2, L.b_o2, w.h1, 1, 1, w.h2)) != ENC_OK) return s;
  const enc::Epi gelu = h->gelu == ENC_GELU_TANH ? enc::Epi::kBiasGeluTanh : enc::Epi::kBiasGelu;
  if ((s = run_gemm(h, w.h2, Mt, H, L.w_ff1, L.tm_ff1, h->F, gelu, L.b_ff1, w.u, {}, st)) != ENC_OK) return s;
  return resid_ln(w.u, h->F, L.w_ff2, L.tm_ff2, L.b_ff2, w.h2, 2, 2, yout);
}

}  // namespace

extern "C" {

enc_status enc_decoder_create(int head_num, int size_per_head, int ffn_dim, int num_layers, enc_dtype dtype,
                              const enc_decoder_layer_weights* weights, enc_t* out) {
  if (!out) return fail(ENC_ERR_INVALID_ARG, "out is null");
  *out = nullptr;
  if (head_num <= 0 || size_per_head <= 0 || ffn_dim <= 0 || num_layers <= 0)
    return fail(ENC_ERR_INVALID_ARG, "head_num, size_per_head, ffn_dim and num_layers must be > 0");
  if (size_per_head != 32 && size_per_head != 64 && size_per_head != 128)
    return fail(ENC_ERR_UNSUPPORTED, "size_per_head %d not in {32, 64, 128}", size_per_head);
  if (dtype != ENC_FP16) return fail(ENC_ERR_UNSUPPORTED, "the decoder runs in FP16 mode only");
  if (ffn_dim % 8 != 0) return fail(ENC_ERR_INVALID_ARG, "ffn_dim %d is not a multiple of 8", ffn_dim);
  const int H = head_num * size_per_head;
  if (H > 1024) return fail(ENC_ERR_UNSUPPORTED, "hidden size %d exceeds 1024", H);
  if (!weights) return fail(ENC_ERR_INVALID_ARG, "weights is null");
  for (int l = 0; l < num_layers; ++l) {
    const void* const* ps = reinterpret_cast<const void* const*>(&weights[l]);
    for (size_t i = 0; i < sizeof(enc_decoder_layer_weights) / sizeof(void*); ++i)
      if (!ps[i]) return fail(ENC_ERR_INVALID_ARG, "decoder layer %d has a null parameter pointer", l);
  }
  int cur_dev = -1;
  if (cudaGetDevice(&cur_dev) != cudaSuccess) return fail(ENC_ERR_CUDA, "no CUDA device");
  int first = -1;
  if (!g_process_device.compare_exchange_strong(first, cur_dev) && first != cur_dev)
    return fail(ENC_ERR_UNSUPPORTED, "handles of one process share one CUDA device (%d); the current device is %d",
                first, cur_dev);
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, cur_dev) != cudaSuccess || prop.major != 10)
    return fail(ENC_ERR_UNSUPPORTED, "FP16 mode needs an sm_100 (B200-class) device");

  enc_handle* h = new enc_handle();
  h->decoder = true;
  h->nh = head_num; h->d = size_per_head; h->H = H; h->F = ffn_dim; h->L = num_layers;
  h->dtype = ENC_FP16;
  h->esize = 2;
  h->device = cur_dev;
  h->num_sms = enc::device_sm_count();
  if (cudaMalloc(&h->status, 8 * sizeof(int)) != cudaSuccess ||
      cudaMemset(h->status, 0, 8 * sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    free_handle(h);
    return fail(ENC_ERR_OOM, "status word allocation failed");
  }
  const size_t F = ffn_dim;
  // Matrices [in, out]: Wqkv [H,3H], Wo [H,H], Wq2 [H,H], Wkv2 [H,2H], Wo2 [H,H], W1 [H,F], W2 [F,H].
  const size_t mrows[7] = {(size_t)H, (size_t)H, (size_t)H, (size_t)H, (size_t)H, (size_t)H, F};
  const size_t mcols[7] = {3 * (size_t)H, (size_t)H, (size_t)H, 2 * (size_t)H, (size_t)H, F, (size_t)H};
  const size_t vlen[7] = {3 * (size_t)H, (size_t)H, (size_t)H, 2 * (size_t)H, (size_t)H, F, (size_t)H};
  size_t per_layer = 6 * (align_up((size_t)H * 2, 256) + align_up((size_t)H * 4, 256)), staging = 0;
  for (int i = 0; i < 7; ++i) {
    per_layer += align_up(mrows[i] * mcols[i] * 2, 256) + align_up(vlen[i] * 4, 256);
    staging = std::max(staging, align_up(mrows[i] * mcols[i] * 2, 256));
  }
  if (cudaMalloc(&h->param_block, per_layer * num_layers + staging) != cudaSuccess) {
    cudaGetLastError();
    free_handle(h);
    return fail(ENC_ERR_OOM, "parameter allocation failed");
  }
  char* p = static_cast<char*>(h->param_block);
  char* stage = p + per_layer * num_layers;
  h->dlayers.resize(num_layers);
  for (int l = 0; l < num_layers; ++l) {
    const enc_decoder_layer_weights& wsrc = weights[l];
    DecLayerDev& L = h->dlayers[l];
    const void* msrc[7] = {wsrc.w_qkv, wsrc.w_o, wsrc.w_q2, wsrc.w_kv2, wsrc.w_o2, wsrc.w_ff1, wsrc.w_ff2};
    void** mdst[7] = {&L.w_qkv, &L.w_o, &L.w_q2, &L.w_kv2, &L.w_o2, &L.w_ff1, &L.w_ff2};
    CUtensorMap* maps[7] = {L.tm_qkv, L.tm_o, L.tm_q2, L.tm_kv2, L.tm_o2, L.tm_ff1, L.tm_ff2};
    const void* vsrc[7] = {wsrc.b_qkv, wsrc.b_o, wsrc.b_q2, wsrc.b_kv2, wsrc.b_o2, wsrc.b_ff1, wsrc.b_ff2};
    float** vdst[7] = {&L.b_qkv, &L.b_o, &L.b_q2, &L.b_kv2, &L.b_o2, &L.b_ff1, &L.b_ff2};
    for (int i = 0; i < 7; ++i) {
      *mdst[i] = p;
      const size_t bytes = mrows[i] * mcols[i] * 2;
      cudaError_t e = cudaMemcpy(stage, msrc[i], bytes, cudaMemcpyDefault);
      if (e != cudaSuccess) { free_handle(h); return cuda_fail(e, "decoder weight upload"); }
      const dim3 grid((unsigned)((mcols[i] + 31) / 32), (unsigned)((mrows[i] + 31) / 32));
      transpose_f16_kernel<<<grid, dim3(32, 8)>>>(reinterpret_cast<const __half*>(stage), reinterpret_cast<__half*>(p),
                                                  (int)mrows[i], (int)mcols[i]);
      e = cudaDeviceSynchronize();
      if (e == cudaSuccess) e = cudaGetLastError();
      if (e != cudaSuccess) { free_handle(h); return cuda_fail(e, "decoder weight repack"); }
      // B operand [N = out, K = in]
      if (!enc::encode_kmajor_fp16_map(&maps[i][0], p, mcols[i], mrows[i], 128) ||
          !enc::encode_kmajor_fp16_map(&maps[i][1], p, mcols[i], mrows[i], 256)) {
        free_handle(h);
        return fail(ENC_ERR_CUDA, "cuTensorMapEncodeTiled failed for a decoder weight");
      }
      p += align_up(bytes, 256);
      *vdst[i] = reinterpret_cast<float*>(p);
      e = cudaMemcpy(stage, vsrc[i], vlen[i] * 2, cudaMemcpyDefault);
      if (e != cudaSuccess) { free_handle(h); return cuda_fail(e, "decoder bias upload"); }
      widen_to_f32_kernel<__half><<<(unsigned)((vlen[i] + 255) / 256), 256>>>(reinterpret_cast<const __half*>(stage),
                                                                              *vdst[i], (int)vlen[i]);
      e = cudaDeviceSynchronize();
      if (e == cudaSuccess) e = cudaGetLastError();
      if (e != cudaSuccess) { free_handle(h); return cuda_fail(e, "decoder bias widen"); }
      p += align_up(vlen[i] * 4, 256);
    }
    const void* lsrc[6] = {wsrc.ln1_g, wsrc.ln1_b, wsrc.ln2_g, wsrc.ln2_b, wsrc.ln3_g, wsrc.ln3_b};
    for (int i = 0; i < 6; ++i) {
      __half* dst = reinterpret_cast<__half*>(p);
      cudaError_t e = cudaMemcpy(dst, lsrc[i], (size_t)H * 2, cudaMemcpyDefault);
      if (e != cudaSuccess) { free_handle(h); return cuda_fail(e, "decoder LayerNorm upload"); }
      if (i % 2 == 0) L.ln_g[i / 2] = dst; else L.ln_b[i / 2] = dst;
      p += align_up((size_t)H * 2, 256);
      float* dstf = reinterpret_cast<float*>(p);
      widen_to_f32_kernel<__half><<<(unsigned)((H + 255) / 256), 256>>>(dst, dstf, H);
      e = cudaDeviceSynchronize();
      if (e == cudaSuccess) e = cudaGetLastError();
      if (e != cudaSuccess) { free_handle(h); return cuda_fail(e, "decoder LayerNorm widen"); }
      if (i % 2 == 0) L.ln_gf[i / 2] = dstf; else L.ln_bf[i / 2] = dstf;
      p += align_up((size_t)H * 4, 256);
    }
  }
  *out = h;
  return ok();
}

enc_status enc_decoder_forward(enc_t h, const void* y, const int32_t* tgt_len, const void* mem,
                               const int32_t* mem_len, void* out, int batch, int tgt_seq, int mem_seq,
                               enc_stream_t stream) {
  enc_status s = check_handle(h);
  if (s != ENC_OK) return s;
  if (!h->decoder) return fail(ENC_ERR_INVALID_ARG, "an encoder handle runs enc_forward");
  if ((s = check_tokens(batch, tgt_seq)) != ENC_OK) return s;
  if ((s = check_tokens(batch, mem_seq)) != ENC_OK) return s;
  if ((s = check_ptrs({y, mem, out})) != ENC_OK) return s;
  if (!tgt_len || !mem_len) return fail(ENC_ERR_INVALID_ARG, "tgt_len and mem_len must not be null");
  const size_t mt = (size_t)batch * tgt_seq, ms = (size_t)batch * mem_seq;
  const size_t bytes = mt * h->H * 2;
  const char* yb = static_cast<const char*>(y);
  const char* ob = static_cast<const char*>(out);
  if (yb < ob + bytes && ob < yb + bytes) return fail(ENC_ERR_INVALID_ARG, "out overlaps y");
  if ((s = ensure_bytes(h, dec_workspace_bytes(h, mt, ms))) != ENC_OK) return s;
  const DecWorkspace w = dec_carve(h, mt, ms);
  PdlScope pdl(h);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  for (int l = 0; l < h->L; ++l) {
    const void* yin = l == 0 ? y : ((l - 1) & 1 ? w.x1 : w.x0);
    void* yout = l == h->L - 1 ? out : (l & 1 ? w.x1 : w.x0);
    if ((s = dec_layer(h, l, yin, yout, tgt_len, mem, mem_len, batch, tgt_seq, mem_seq, w, st)) != ENC_OK) return s;
  }
  return ok();
}

}  // extern "C"
