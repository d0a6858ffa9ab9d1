/*
 * enc.h - C ABI of a B200 (sm_100a) library for the forward pass of a
 * BERT-style post-LayerNorm Transformer encoder stack.
 *
 * Source page: "有钱任性：英伟达训练80亿参数量GPT-2，1475块V100 53分钟训练BERT"
 * (机器之心; the Faster Transformer write-up), cited as [FT] with a section.
 *
 *  - [FT] "什么是 Faster Transformer": the encoder forward is the whole
 *    product; the network structure is fixed by head_num and size_per_head,
 *    and batch size and maximum sequence length are given per run; the
 *    computation runs in FP32 or in FP16 (FP16 on tensor cores); the library
 *    offers a C++ API.  Unlike the page's fixed lengths (32/64/128), any
 *    sequence length >= 1 is accepted here.
 *  - [FT] "Faster Transformer 优化原理": per layer, the matrix multiplies run
 *    on tensor cores and every other operation is fused into as few kernels
 *    as possible (add-bias/transposes, SoftMax, add-bias + residual +
 *    LayerNorm, add-bias + GELU).
 *
 * Per layer (x: [batch, seq, H], H = head_num * size_per_head, F = ffn_dim):
 *   QKV = x Wqkv + bqkv;  per head: ctx = softmax(Q K^T / sqrt(d), keys j < n) V
 *   H1  = LN(x + ctx Wo + bo; ln1);   U = GELU(H1 W1 + b1)  (erf form)
 *   out = LN(H1 + U W2 + b2; ln2)
 * with n = clamp(valid_len[b], 0, seq); LN eps = 1e-12, biased variance.
 * Query rows i >= n are computed (attending to the n valid keys) but are not
 * meaningful to callers; n == 0 gives ctx = 0 for that sequence.
 *
 * Numerics: FP16 mode stores every tensor in IEEE half and accumulates every
 * matmul, softmax and LayerNorm in FP32 (no half accumulation).  FP32 mode
 * stores and computes in FP32 on CUDA cores (no TF32).
 *
 * Threading and streams: every call is asynchronous on the given stream
 * unless stated.  A handle owns one workspace, so it must not be used by two
 * streams at once.  Device-side faults surface at the caller's next
 * synchronisation, as with any CUDA launch.
 */
#ifndef BERT_ENCODER_B200_ENC_H
#define BERT_ENCODER_B200_ENC_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ENC_API __attribute__((visibility("default")))
#else
#define ENC_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream (a pointer to the driver's stream object); NULL = legacy default stream. */
typedef struct CUstream_st* enc_stream_t;

typedef struct enc_handle* enc_t;
typedef struct enc_graph_s* enc_graph_t;

typedef enum {
  ENC_OK = 0,
  ENC_ERR_INVALID_ARG = 1,   /* a host-side argument check failed; nothing was enqueued */
  ENC_ERR_UNSUPPORTED = 2,   /* valid but not supported (e.g. size_per_head not in {32,64,128}) */
  ENC_ERR_OOM = 3,           /* a device allocation failed; the handle stays usable */
  ENC_ERR_CUDA = 4,          /* a CUDA runtime/driver call or launch failed; see enc_last_error() */
  ENC_ERR_DEVICE = 5         /* a kernel reported a failure through the handle's device status word */
} enc_status;

typedef enum { ENC_FP32 = 0, ENC_FP16 = 1 } enc_dtype;

/* FFN activation.  ENC_GELU_ERF: 0.5 t (1 + erf(t / sqrt 2)) (default).
 * ENC_GELU_TANH: 0.5 t (1 + tanh(sqrt(2/pi) (t + 0.044715 t^3))), the form the
 * source page implies when it replaces pow(x, 3) by x*x*x ([FT] "Faster
 * Transformer 优化原理"). */
typedef enum { ENC_GELU_ERF = 0, ENC_GELU_TANH = 1 } enc_gelu;

/* One layer's parameters.  Element type = the handle's dtype (float or IEEE half).
 * Matrices are [in, out] row-major (y = x W + b).  Wqkv's columns are Q | K | V,
 * and inside each block head h owns columns h*d .. h*d+d-1.  The pointers may be
 * host or device memory (detected per pointer); they are only read during
 * enc_create. */
typedef struct {
  const void* w_qkv; const void* b_qkv;   /* [H, 3H], [3H] */
  const void* w_o;   const void* b_o;     /* [H, H],  [H]  */
  const void* ln1_g; const void* ln1_b;   /* [H], [H] */
  const void* w_ff1; const void* b_ff1;   /* [H, F],  [F]  */
  const void* w_ff2; const void* b_ff2;   /* [F, H],  [H]  */
  const void* ln2_g; const void* ln2_b;   /* [H], [H] */
} enc_layer_weights;

/* enc_create - build a handle on the current CUDA device.  Every handle of a
 * process lives on the device of the first one (kernel launch attributes are
 * set once per process); on another device enc_create returns
 * ENC_ERR_UNSUPPORTED.  Use one process per GPU.
 * [FT] "什么是 Faster Transformer": head_num and size_per_head are the two
 * structural parameters; ffn_dim and num_layers complete the stack.
 *   head_num, ffn_dim, num_layers > 0; size_per_head in {32, 64, 128}
 *   (else ENC_ERR_UNSUPPORTED); ffn_dim a multiple of 8; hidden size
 *   H = head_num * size_per_head at most 2048 in FP16 mode and 1024 in FP32
 *   mode (else ENC_ERR_UNSUPPORTED: a LayerNorm row lives in one warp's
 *   registers).
 *   weights: array of num_layers structs (see enc_layer_weights).
 * The handle copies and repacks every parameter into its own device memory
 * (FP16 weights are stored transposed, [out, in], for the tensor-core GEMMs;
 * biases and LayerNorm parameters are widened to FP32), so the caller may free
 * its buffers on return.  Synchronous.  On error *out is set to NULL. */
ENC_API enc_status enc_create(int head_num, int size_per_head, int ffn_dim, int num_layers,
                      enc_dtype dtype, const enc_layer_weights* weights, enc_t* out);

/* enc_set_gelu - choose the FFN activation of every later call on this handle
 * (host-side setting; takes effect at the next launch). */
ENC_API enc_status enc_set_gelu(enc_t h, enc_gelu form);

/* Kernel-path switches.  Every choice computes the same result to rounding;
 * the defaults are the measured-fastest paths, and the others exist so that
 * each alternative kernel can be compared and checked on any shape. */
typedef enum {
  /* 1 (default): 2-CTA 256x256 GEMM tiles where they still give a quarter of
   * the SMs a tile; 0: one-CTA 128-row tiles only. */
  ENC_OPT_PAIR_TILES = 0,
  /* 1 (default): GEMM epilogues store their output, and read the residual,
   * through TMA; 0: plain 16-byte stores and loads (also turns off both
   * LayerNorm fusions, which need TMA). */
  ENC_OPT_TMA_STORE = 1,
  /* 1 (default): tcgen05 attention for size-64 heads on sequences longer than
   * 64; 0: the mma.sync attention kernels for every length. */
  ENC_OPT_TC_ATTENTION = 2,
  /* 1 (default): split-K thread-block clusters for GEMMs whose tiles would
   * leave more than half the SMs idle; 0: never split K. */
  ENC_OPT_SPLIT_K = 3,
  /* Whether the FFN2 GEMM writes LayerNorm 2 of its rows itself (row
   * statistics exchanged across the thread-block cluster that covers a row;
   * needs the 2-CTA tiles and a hidden size that is a multiple of 256, at most
   * 1024): 0 never (a separate LayerNorm kernel), 1 (default) where it measured
   * faster (hidden size <= 768, clusters of at most 6 CTAs, and a token count
   * whose row blocks fill the clusters' waves about as well as the unfused
   * GEMM's tiles fill its waves), 2 wherever supported. */
  ENC_OPT_LN_FUSE_FFN2 = 4,
  /* The same for the output-projection GEMM and LayerNorm 1 (0, 1 = default, 2);
   * its default asks for clearly better-filled waves than FFN2's, since its
   * short K = hidden main loop does not hide the fused epilogue. */
  ENC_OPT_LN_FUSE_OUT_PROJ = 5,
  /* 1 (default): kernels are launched with programmatic dependent launch, so
   * each one's set-up overlaps its predecessor's tail; 0: plain stream order. */
  ENC_OPT_PDL = 6,
  /* 0 (default): the per-step kernels; 1: FP16 forwards of at most 256 tokens
   * (batch * seq) without padding removal run as ONE persistent kernel for the
   * whole stack, with grid-wide barriers between the steps ([FT] "Faster
   * Transformer 优化原理": at small batch the launches, not the arithmetic, set
   * the time).  Needs hidden and ffn sizes that are multiples of 64, hidden <=
   * 1024; other shapes keep the per-step kernels.  Off by default because the
   * per-step kernels, replayed as a CUDA graph with programmatic dependent
   * launch, measured faster at every batch size. */
  ENC_OPT_PERSISTENT = 7,
  /* Failure-detection test of that single-launch forward, 0 by default: with
   * 1, one CTA waits on a flag that nothing sets instead of joining the first
   * grid-wide barrier, every wait of the launch gives up after 20 ms, and the
   * launch reports status 1 through enc_device_status; the outputs of that
   * forward are undefined and the context stays usable. */
  ENC_OPT_TEST_STALL = 8
} enc_option;

/* enc_set_option - set one kernel-path switch of this handle (0 or 1; 0, 1 or 2
 * for the two LayerNorm fusions; else ENC_ERR_INVALID_ARG).  Host-side; takes effect at the next launch.  A
 * recorded forward (enc_graph_create) keeps the kernels it recorded.  Not part
 * of the source pages' design: it exposes this library's own alternatives. */
ENC_API enc_status enc_set_option(enc_t h, enc_option option, int value);

/* enc_get_option - read one switch into *value. */
ENC_API enc_status enc_get_option(enc_t h, enc_option option, int* value);

/* enc_set_packing - padding removal for every later forward (FP16 mode, H <=
 * 1024; else ENC_ERR_UNSUPPORTED).  With it on, the valid tokens of the batch
 * are packed on the device into [T, H] (T = sum of the clamped valid lengths),
 * every GEMM, LayerNorm and attention step runs on those T rows only, and out
 * receives the valid rows with ZEROS in the padded positions i >= n (the
 * default mode computes those rows; their values are not meaningful in either
 * mode).  Valid outputs agree with the default mode to rounding.  The page
 * fixes the sequence length for performance and plans arbitrary lengths
 * ([FT] "什么是 Faster Transformer"); this removes the padding's cost instead.
 * A forward then launches 3 kernels more (offsets, pack, unpack);
 * enc_kernels_per_forward gives the total. */
ENC_API enc_status enc_set_packing(enc_t h, int enable);

/* enc_set_host_chunks - most chunks enc_forward_host cuts a batch into (1..4,
 * default 1 = no overlap of copies with the encoder). */
ENC_API enc_status enc_set_host_chunks(enc_t h, int chunks);

/* enc_forward - run the whole encoder stack on `stream`.
 * [FT] "什么是 Faster Transformer" (batch size and sequence length per run)
 * and "Faster Transformer 优化原理" (the fused per-layer kernels).
 *   x:         device [batch, seq, H] in the handle's dtype, row-major.
 *   valid_len: device int32 [batch]; values are clamped to [0, seq] on device.
 *   out:       device [batch, seq, H]; must not overlap x.
 *   1 <= batch <= 65535, seq >= 1.  x and out must be 16-byte aligned.
 * The handle's workspace grows (cudaMalloc) when batch*seq exceeds what it
 * holds; call enc_reserve first to keep allocation out of a timed or captured
 * region.  No host synchronisation inside; errors in host checks are returned
 * before anything is enqueued. */
ENC_API enc_status enc_forward(enc_t h, const void* x, const int32_t* valid_len, void* out,
                       int batch, int seq, enc_stream_t stream);

/* Size of the fixed device array that enc_forward_noalloc uses as its scratch:
 * 32 MiB.  Every GPU that loads this library holds it until the process exits. */
#define ENC_STATIC_WORKSPACE_BYTES ((size_t)32 << 20)

/* enc_forward_noalloc - enc_forward without any device allocation.  The source
 * pages have no counterpart: this serves callers that cannot call cudaMalloc
 * when they run the encoder, such as a server whose device memory is all handed
 * out by its own pool allocator (so a library allocation fails or takes memory
 * the pool counts on), or a latency-bound loop that cannot afford cudaMalloc /
 * cudaFree, which may synchronise the whole device.  The handle still comes
 * from enc_create, which does allocate, at set-up time.
 *   Same arguments, layout, results and kernels as enc_forward.  The
 *   intermediates live in one fixed device array of ENC_STATIC_WORKSPACE_BYTES
 *   compiled into the library instead of the handle's workspace, so the call
 *   accepts a batch only when enc_workspace_bytes(h, batch, seq) <=
 *   ENC_STATIC_WORKSPACE_BYTES (BERT-Base needs 18,432 bytes per token, so at
 *   most 1,820 tokens, e.g. batch 14 at seq 128); larger ones return
 *   ENC_ERR_UNSUPPORTED before anything is enqueued.
 *   The first call on a device looks up the array's device address there
 *   (cudaGetSymbolAddress, with that device current); make that first call
 *   before any stream capture.  Later calls only launch kernels.
 *   The array is shared by every call on the device, from every handle and
 *   stream, and keeps the last call's contents.  Nothing in it needs to start
 *   at zero: each forward writes every intermediate before reading it.  Calls
 *   that overlap on the GPU race on the array and corrupt each other's
 *   results: order them, e.g. on one stream. */
ENC_API enc_status enc_forward_noalloc(enc_t h, const void* x, const int32_t* valid_len, void* out,
                                       int batch, int seq, enc_stream_t stream);

/* enc_forward_host - enc_forward on HOST buffers: copies x and valid_len to
 * handle-owned device staging buffers, runs the stack and copies the result
 * back into out, then synchronises `stream`.  The copies run on two
 * handle-owned streams, ordered after the caller's earlier work on `stream`.
 * With enc_set_host_chunks(h, c > 1) the batch is cut into up to c chunks of
 * sequences (at least 2048 tokens each), so that copying chunk i+1 in and
 * chunk i-1 out overlaps the encoder on chunk i; the default is one chunk,
 * which measured fastest for BERT-Base at 16384 tokens (smaller chunks cost
 * the GEMMs more than the overlap saves).  Host buffers may be pageable or
 * pinned (pinned gives asynchronous DMA).
 *   x: host [batch, seq, H]; valid_len: host int32 [batch]; out: host [batch, seq, H]. */
ENC_API enc_status enc_forward_host(enc_t h, const void* x, const int32_t* valid_len, void* out,
                            int batch, int seq, enc_stream_t stream);

/* enc_forward_host_async - enc_forward_host for a stream of batches: returns
 * once the work is enqueued, without synchronising.  Consecutive calls use two
 * handle-owned device staging slots in turn, so that the input copy of call
 * i+1 and the output copy of call i overlap the encoder runs (copies on two
 * handle-owned streams, the encoder on `stream`).  Host buffers should be
 * pinned; the caller keeps x and valid_len unchanged and out untouched until
 * the call's copies are done, which enc_host_join makes `stream` wait for.
 * Calls of one handle must use one `stream`.  Same arguments and errors as
 * enc_forward_host.  Not part of the source pages' design (they describe the
 * device computation only): it serves throughput from host memory. */
ENC_API enc_status enc_forward_host_async(enc_t h, const void* x, const int32_t* valid_len, void* out,
                                          int batch, int seq, enc_stream_t stream);

/* enc_host_join - make `stream` wait until every copy enqueued by earlier
 * enc_forward_host_async calls has completed (no host synchronisation).  After
 * `stream` reaches that point the outputs are in host memory. */
ENC_API enc_status enc_host_join(enc_t h, enc_stream_t stream);

/* enc_reserve - grow the workspace to hold batch*seq tokens now (synchronous). */
ENC_API enc_status enc_reserve(enc_t h, int batch, int seq);

/* enc_workspace_bytes - device bytes enc_forward needs for a batch*seq-token run. */
ENC_API size_t enc_workspace_bytes(enc_t h, int batch, int seq);

/* enc_destroy - free every device buffer the handle owns (synchronises the device). NULL is a no-op. */
ENC_API enc_status enc_destroy(enc_t h);

/* enc_last_error - message for the last non-OK status on the calling thread ("" if none).
 * The string is thread-local and valid until the next library call on this thread. */
ENC_API const char* enc_last_error(void);

/* enc_device_status - read and clear the handle's device status word (synchronises
 * the device).  *code is 0 when no kernel has reported a failure since the last
 * read; otherwise the code of the first failure (1 = a bounded wait inside a
 * tensor-core GEMM or attention kernel gave up).  Returns ENC_ERR_DEVICE when
 * *code != 0. */
ENC_API enc_status enc_device_status(enc_t h, int32_t* code);

/* enc_graph_create - record one enc_forward (these exact buffers, batch and seq)
 * as an instantiated CUDA graph, so that it replays with a single launch.
 * [FT] "Faster Transformer 优化原理": at small batch the cost is kernel
 * launches, not arithmetic.  The workspace is reserved first; while any graph
 * of the handle exists the workspace is pinned, and an enc_forward that would
 * need a larger one returns ENC_ERR_INVALID_ARG.  Synchronous.  The graph
 * reads x and valid_len and writes out at replay time; the caller keeps those
 * buffers alive until enc_graph_destroy. */
ENC_API enc_status enc_graph_create(enc_t h, const void* x, const int32_t* valid_len, void* out,
                                    int batch, int seq, enc_graph_t* graph);

/* enc_graph_launch - replay a recorded forward on `stream` (asynchronous). */
ENC_API enc_status enc_graph_launch(enc_graph_t graph, enc_stream_t stream);

/* enc_graph_destroy - release a recorded forward (synchronises the device). NULL is a no-op. */
ENC_API enc_status enc_graph_destroy(enc_graph_t graph);

/* enc_kernels_per_forward - kernel launches one enc_forward of batch x seq
 * issues: 1 when the single-launch forward runs (ENC_OPT_PERSISTENT);
 * otherwise per layer 7, less one for each of the output-projection and FFN2
 * GEMMs that writes the LayerNorm of its rows itself (FP16, enough tokens for
 * the 2-CTA tiles, hidden size 256, 512 or 768 by default; which of the two
 * follows ENC_OPT_LN_FUSE_FFN2 and ENC_OPT_LN_FUSE_OUT_PROJ); plus 3 with
 * padding removal.  0 for invalid arguments. */
ENC_API int enc_kernels_per_forward(enc_t h, int batch, int seq);

/* enc_launch_count - kernel launches this handle has issued since enc_create
 * (forward passes and single steps), for checking what ran. */
ENC_API uint64_t enc_launch_count(enc_t h);

/* enc_set_trace_events - optional per-kernel timing of enc_forward.  events
 * holds count CUDA events (cudaEvent_t, created by the caller; at least 2, and
 * a forward needing more than count fails with ENC_ERR_INVALID_ARG);
 * with count >= enc_kernels_per_forward(h, batch, seq) + 1, each enc_forward records events[k] on its
 * stream just before its k-th kernel and events[kernels] after the last, so
 * cudaEventElapsedTime(events[k], events[k+1]) is kernel k's duration.
 * Kernel order per layer: QKV GEMM, attention, output GEMM, LayerNorm 1,
 * FFN1 GEMM, FFN2 GEMM, LayerNorm 2 (without the two LayerNorm kernels when
 * the GEMMs write the normalised rows); with padding removal the offsets and
 * pack kernels come first and the unpack kernel last.  events = NULL or count = 0 switches
 * tracing off.  The handle keeps the pointers; the caller keeps the events
 * alive while tracing is on. */
ENC_API enc_status enc_set_trace_events(enc_t h, void* const* events, int count);

/* ------------------------------------------------------------------------------
 * Decoder forward.  [FT] "什么是 Faster Transformer" says a decoder follows the
 * encoder in a later release and gives no design.  The layer here is the
 * post-LN Transformer decoder layer run over a whole target sequence (every
 * target token at once), with the encoder's conventions (LN eps 1e-12,
 * biased variance, scale 1/sqrt(d), masked keys weigh exactly 0, erf GELU
 * unless enc_set_gelu chooses tanh):
 *   QKV = y Wqkv + bqkv;  per head: A1 = softmax(Q K^T / sqrt(d)) V over keys
 *     j <= i and j < nt = clamp(tgt_len[b], 0, T)  (causal self-attention);
 *   H1 = LN1(y + A1 Wo + bo);
 *   Q2 = H1 Wq2 + bq2,  [K2 | V2] = mem Wkv2 + bkv2;  A2 = softmax(Q2 K2^T /
 *     sqrt(d)) V2 over memory keys j < nm = clamp(mem_len[b], 0, S);
 *   H2 = LN2(H1 + A2 Wo2 + bo2);
 *   out = LN3(H2 + GELU(H2 W1 + b1) W2 + b2).
 * Every layer attends to the same memory (e.g. the encoder output).  A query
 * row with no valid key gets a zero attention context.
 * ---------------------------------------------------------------------------- */

/* One decoder layer's parameters, IEEE half, matrices [in, out] row-major.
 * Wqkv's columns are Q | K | V and Wkv2's are K | V, head h at columns
 * h*d .. h*d+d-1 inside each block.  Host or device pointers, read only
 * during enc_decoder_create. */
typedef struct {
  const void* w_qkv; const void* b_qkv;   /* [H, 3H], [3H]  self-attention */
  const void* w_o;   const void* b_o;     /* [H, H],  [H]   */
  const void* ln1_g; const void* ln1_b;   /* [H], [H] */
  const void* w_q2;  const void* b_q2;    /* [H, H],  [H]   cross-attention query */
  const void* w_kv2; const void* b_kv2;   /* [H, 2H], [2H]  cross-attention keys | values, from the memory */
  const void* w_o2;  const void* b_o2;    /* [H, H],  [H]   */
  const void* ln2_g; const void* ln2_b;   /* [H], [H] */
  const void* w_ff1; const void* b_ff1;   /* [H, F],  [F]   */
  const void* w_ff2; const void* b_ff2;   /* [F, H],  [H]   */
  const void* ln3_g; const void* ln3_b;   /* [H], [H] */
} enc_decoder_layer_weights;

/* enc_decoder_create - a decoder handle (FP16 only: ENC_FP32 gives
 * ENC_ERR_UNSUPPORTED; size_per_head in {32, 64, 128}, hidden size <= 1024,
 * ffn_dim a multiple of 8).  Copies and repacks every parameter like
 * enc_create; release it with enc_destroy.  Synchronous.  enc_set_gelu and
 * enc_set_option apply to it; the encoder-only calls (enc_forward and the
 * enc_op_* steps) return ENC_ERR_INVALID_ARG on it. */
ENC_API enc_status enc_decoder_create(int head_num, int size_per_head, int ffn_dim, int num_layers,
                                      enc_dtype dtype, const enc_decoder_layer_weights* weights, enc_t* out);

/* enc_decoder_forward - the decoder stack on `stream`.
 *   y:        device [batch, tgt_seq, H] target hidden states;
 *   tgt_len:  device int32 [batch], clamped to [0, tgt_seq] on device;
 *   mem:      device [batch, mem_seq, H] memory (e.g. the encoder output);
 *   mem_len:  device int32 [batch], clamped to [0, mem_seq] on device;
 *   out:      device [batch, tgt_seq, H]; must not overlap y.
 * 16-byte-aligned buffers; the workspace grows like enc_forward's.  12 kernel
 * launches per layer, 9 where the three bias + residual + LayerNorm steps run
 * in their GEMMs' epilogues (the encoder's rule and options: 2-CTA tiles,
 * hidden size <= 768 by default).  Asynchronous; host checks fail before
 * anything is enqueued. */
ENC_API enc_status enc_decoder_forward(enc_t h, const void* y, const int32_t* tgt_len, const void* mem,
                                       const int32_t* mem_len, void* out, int batch, int tgt_seq, int mem_seq,
                                       enc_stream_t stream);

/* ------------------------------------------------------------------------------
 * Single steps of one layer, for checking each kernel alone.  Each runs exactly
 * the kernel enc_forward runs for that step, with layer `layer`'s parameters,
 * on caller-owned device buffers (same dtype as the handle, 16-byte aligned,
 * non-overlapping).  M = batch * seq tokens.  Asynchronous on `stream`.
 * ---------------------------------------------------------------------------- */

/* Steps QKV projection + add-bias + head split ([FT] "Faster Transformer 优化原理":
 * the Q/K/V matrix multiplies and the add-bias/transpose custom kernel, fused here
 * into one GEMM epilogue):
 *   qkv[t][b][h][s][c] = (x Wqkv + bqkv)[b*seq+s][t*H + h*d + c],
 *   x: [M, H];  qkv: [3, batch, head_num, seq, d]. */
ENC_API enc_status enc_op_qkv(enc_t h, int layer, const void* x, void* qkv, int batch, int seq,
                      enc_stream_t stream);

/* Steps scaled QK^T + padding mask, softmax, PV and head merge ([FT] "Faster
 * Transformer 优化原理": the batched matrix multiplies around the SoftMax kernel
 * and the transpose back to [tokens, hidden]), one fused kernel:
 *   qkv: [3, batch, head_num, seq, d];  valid_len: device int32 [batch];
 *   ctx: [M, H], ctx[b*seq+i][h*d + c]. */
ENC_API enc_status enc_op_attention(enc_t h, const void* qkv, const int32_t* valid_len, void* ctx,
                            int batch, int seq, enc_stream_t stream);

/* Steps output projection + add-bias + residual + LayerNorm 1 ([FT] "Faster
 * Transformer 优化原理": the output GEMM and the add-bias + residual + Layer
 * Normalization kernel):
 *   out = LN1(ctx Wo + bo + resid),  ctx, resid, out: [tokens, H]  (resid = the
 *   layer input); LN over H, biased variance, eps 1e-12.
 * One kernel when the GEMM writes the normalised rows itself (see
 * enc_kernels_per_forward); otherwise the GEMM writes ctx Wo + bo + resid into
 * the handle's workspace (which grows as enc_forward's does) and a LayerNorm
 * kernel follows. */
ENC_API enc_status enc_op_out_proj_ln(enc_t h, int layer, const void* ctx, const void* resid, void* out,
                                      int tokens, enc_stream_t stream);

/* Step FFN1 + add-bias + GELU (erf form) fused in the GEMM epilogue:
 *   u = GELU(h1 W1 + b1),  h1: [tokens, H], u: [tokens, F]. */
ENC_API enc_status enc_op_ffn1(enc_t h, int layer, const void* h1, void* u, int tokens,
                       enc_stream_t stream);

/* Steps FFN2 + add-bias + residual + LayerNorm 2, like enc_op_out_proj_ln:
 *   out = LN2(u W2 + b2 + resid),  u: [tokens, F], resid, out: [tokens, H]
 *   (resid = h1, the first LayerNorm's output). */
ENC_API enc_status enc_op_ffn2_ln(enc_t h, int layer, const void* u, const void* resid, void* out, int tokens,
                                  enc_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* BERT_ENCODER_B200_ENC_H */
