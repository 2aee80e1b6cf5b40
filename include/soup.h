/*
 * soup.h - C ABI of the B200 (sm_100a) layer-streamed LoRA training library.
 *
 * What the library computes (the method of the Soup "layer streaming" pages):
 * LoRA fine-tuning over a frozen base model whose weights live in pinned host
 * RAM as per-layer NF4 (or bf16) shards and are fed one decoder layer at a
 * time into a small ring of preallocated device slots by a separate copy
 * stream.  Each adapted projection computes  y = W x + (alpha/r) B A x;  the
 * backward pass re-reads and recomputes the layer and produces
 * dL/dx = W^T dL/dy plus the adapter terms, and dA, dB, while W stays frozen.
 *
 * Sections below: status and profiling; NF4 quantisation; the LoRA linear
 * layer; the decoder layer (forward, recompute backward, kept q|k|v); the
 * stream plan (slot ring, copies, waits); the disk tier (shard files read
 * ahead into staging buffers); layer blob layout; embedding, output head,
 * cross-entropy and DPO; SimPO and ORPO; the AdamW step on the adapters.
 *
 * Conventions for every entry point
 *  - Every function returns a soup_status; SOUP_OK (0) on success.  On failure
 *    soup_last_error() returns a message for the calling thread.  Nothing
 *    aborts the process and no argument is silently clamped: an argument that
 *    is out of range is refused.
 *  - Pointers named *_dev, and all tensor pointers unless stated otherwise,
 *    are CUDA device pointers owned by the caller.  The library allocates no
 *    device memory except the slot arena of soup_stream_plan (and the
 *    disk tier's page-locked host staging buffers, in soup_disk_open).
 *  - "bf16" tensors are passed as uint16_t bit patterns (IEEE bfloat16).
 *  - Matrices are row-major.  [R, C] means R rows of C contiguous elements.
 *  - `stream` is a cudaStream_t passed as void*; work is enqueued on it and
 *    the call returns without waiting, except where a function says it
 *    synchronises.
 *  - A kernel whose internal wait exceeds its time limit records a code in a
 *    device error word instead of hanging; soup_device_error() reads it.
 */
#ifndef SOUP_H_
#define SOUP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t soup_status;
#define SOUP_OK 0
#define SOUP_ERR_INVALID_ARG 1 /* null pointer, value out of range */
#define SOUP_ERR_SHAPE 2       /* dimensions the kernels do not support */
#define SOUP_ERR_ALIGN 3       /* pointer or stride misaligned */
#define SOUP_ERR_NONFINITE 4   /* NaN or Inf in an input that must be finite */
#define SOUP_ERR_OOM_PLAN 5    /* a stream plan does not fit the device cap */
#define SOUP_ERR_TIMEOUT 6     /* a host wait or a kernel's bounded wait expired */
#define SOUP_ERR_CUDA 7        /* a CUDA runtime call failed */
#define SOUP_ERR_IO 8          /* a shard file could not be opened or read */

/* Message describing the last failure on the calling thread ("" if none). */
const char* soup_last_error(void);

/* Reads and clears the device error word of the current device (synchronises
 * the device).  *code_out = 0 when no kernel reported a problem; otherwise
 * the OR of the codes the kernels recorded: 1 = a bounded wait on an mbarrier
 * expired in a GEMM, 2 = a token id outside the vocabulary in soup_embed (its
 * row is written as zeros), 4 = a bounded wait expired in an attention kernel.
 * Returns SOUP_OK, or SOUP_ERR_CUDA if the read itself failed. */
soup_status soup_device_error(int32_t* code_out);

/* Test of the kernels' bounded waits, with no fault and no hang: computes
 * C[M, N] (fp32, row-major) = A[M, K] B[N, K]^T (bf16, row-major, device
 * pointers) with the one-CTA tcgen05 GEMM engine, whose mbarrier waits give
 * up after wait_limit_cycles SM clock cycles (0 = the default, ~2 s).  With
 * skip_producer_arrivals != 0 the engine's TMA producer issues nothing and
 * never arrives, so the MMA warp's wait runs out: the CTA records code 1 in
 * the device error word (soup_device_error), issues no tensor-core work,
 * frees its tensor memory and returns; C is left unwritten and the context
 * stays usable.  Sizes in (0, 4096], K % 8 == 0, N % 4 == 0.  Async on
 * `stream`. */
soup_status soup_debug_gemm_bounded_wait(const uint16_t* A, const uint16_t* B, int64_t M, int64_t N, int64_t K,
                                         float* C, int64_t wait_limit_cycles, int32_t skip_producer_arrivals,
                                         void* stream);

/* Number of kernels this library has launched in this process. */
int64_t soup_launch_count(void);

/* Optional timing of kernel launches: while enabled, every launch of a class
 * in class_mask (bit c = class c) is bracketed by CUDA events recorded on its
 * own stream and tagged with its algorithmic work.  soup_profile_read
 * synchronises those events and sums them per class:
 * 0 = fused NF4-decode GEMM (forward, W), 1 = fused NF4-decode GEMM
 * (backward, W^T), 2 = other GEMMs with N > 64, 3 = skinny LoRA GEMMs
 * (N <= 64), 4 = fused NF4-decode GEMMs with a hi + lo A pair (either
 * direction), 5 = attention (forward and backward kernels; flops 4 B Hq d
 * S(S+1)/2 forward, 2.5x that backward), 6 = RMSNorm forward / backward,
 * 7 = split-K reductions, 8 = other elementwise kernels (RoPE tables, LoRA
 * operand preparation, conversions, attention row dots, embedding gather),
 * 9 = cross-entropy rows of the output head, 10 = AdamW.  Classes 6..10
 * carry algorithmic bytes (each operand read once, each output written
 * once) and no flops.  Enabling resets the records; class_mask 0 disables. */
typedef struct soup_gemm_profile {
  int64_t launches;
  double total_ms;
  double flops;  /* GEMMs: 2 M N (K + r_tail) summed over launches; attention as above */
  double bytes;  /* operands read once + outputs written once */
} soup_gemm_profile;
soup_status soup_profile_enable(int32_t class_mask);
soup_status soup_profile_read(soup_gemm_profile* out, int32_t n_classes);

/* ------------------------------------------------------------------ NF4 ---
 * NF4 block quantisation of the frozen base (the pages' `quantization: 4bit`
 * storage of the streamed base; Soup pages, "configuration and training" and
 * the published-numbers table).  Data type: QLoRA's 16-level NormalFloat
 * codebook.  Blocks of 64 consecutive elements along the input dimension of a
 * row share one fp32 absmax (no double quantisation).  A weight w in a block
 * with absmax a gets the code of the codebook value nearest to fl32(w / a)
 * (ties to the lower code); an all-zero block gets code 7 (exact zero).
 * Packing: byte j of a row holds element 2j in bits 7..4 and 2j+1 in bits 3..0.
 */

/* W [out, in] fp32 -> codes [out, in/2] u8, absmax [out, in/64] fp32.
 * in must be a positive multiple of 64.  flag_dev: caller-owned device int32
 * used as scratch (the call zeroes it, the kernel sets it when it meets a
 * non-finite weight).  This call SYNCHRONISES `stream` and returns
 * SOUP_ERR_NONFINITE if any weight was NaN/Inf (codes/absmax are then
 * unspecified). */
soup_status soup_nf4_quantize(const float* W, int64_t out, int64_t in, uint8_t* codes,
                              float* absmax, int32_t* flag_dev, void* stream);

/* codes [out, in/2], absmax [out, in/64] -> W [out, in] bf16 where each value
 * is round-to-nearest-even-to-bf16 of the fp32 product codebook[code]*absmax. */
soup_status soup_nf4_dequant(const uint8_t* codes, const float* absmax, int64_t out,
                             int64_t in, uint16_t* W_bf16, void* stream);

/* ----------------------------------------------------------- LoRA linear ---
 * One adapted projection, y = x W^T + s (x A^T) B^T with s = alpha/r
 * (row-vector form of y = W x + (alpha/r) B A x), W frozen.
 *
 * Precision contract: bf16 operands, fp32 accumulation on tensor cores.  The
 * down-projection result is stored as u_save = bf16(s * A x), transposed
 * [r, ldT] with ldT = round_up(T, 8); the up-projection consumes that bf16
 * value.  y is rounded once to bf16 from the fp32 sum.
 */
#define SOUP_WEIGHT_NF4 0
#define SOUP_WEIGHT_BF16 1

typedef struct soup_weight {
  int32_t kind;          /* SOUP_WEIGHT_NF4 or SOUP_WEIGHT_BF16 */
  int64_t out_features;  /* rows of W (N) */
  int64_t in_features;   /* columns of W (K); a multiple of 64 */
  const uint8_t* codes;  /* NF4: [out, in/2] */
  const float* absmax;   /* NF4: [out, in/64] */
  const uint16_t* w;     /* BF16: [out, in] */
} soup_weight;

/* Forward.  A [r, in] bf16, B [out, r] bf16 (r a multiple of 8, 8 <= r <= 64),
 * x [T, in] bf16, y [T, out] bf16, u_save [r, round_up(T, 8)] bf16.
 * T >= 1; out a multiple of 16; in a multiple of 64; all pointers 16-byte
 * aligned. */
soup_status soup_lora_linear_fwd(const soup_weight* W, const uint16_t* A, const uint16_t* B,
                                 int32_t r, float scale, const uint16_t* x, int64_t T,
                                 uint16_t* y, uint16_t* u_save, void* stream);

/* Workspace bytes soup_lora_linear_bwd needs for (T, r, out). */
size_t soup_lora_linear_bwd_workspace(int64_t T, int32_t r, int64_t out_features);

/* Backward.  dy [T, out] bf16 -> dx [T, in] bf16, dA [r, in] fp32 and
 * dB [out, r] fp32 (overwritten, not accumulated):
 *   g' = bf16(s * dy B)        (stored transposed in the workspace)
 *   dx = dy W + g' A,   dA = g'^T x,   dB = dy^T u_save^T
 * u_save is the tensor soup_lora_linear_fwd wrote for the same x.
 * workspace: device memory of at least soup_lora_linear_bwd_workspace() bytes,
 * 256-byte aligned. */
soup_status soup_lora_linear_bwd(const soup_weight* W, const uint16_t* A, const uint16_t* B,
                                 int32_t r, float scale, const uint16_t* x,
                                 const uint16_t* u_save, const uint16_t* dy, int64_t T,
                                 uint16_t* dx, float* dA, float* dB, void* workspace,
                                 size_t workspace_bytes, void* stream);

/* Allocation-free variant of soup_lora_linear_bwd (the pages have no
 * counterpart: this is an integration convenience).  For callers that cannot
 * allocate device memory when they run the backward, e.g. an integration
 * whose device memory is entirely owned by another allocator's pool, or a
 * latency-critical path where cudaMalloc (which may synchronise the device)
 * is not allowed.  Same arguments and results as soup_lora_linear_bwd minus
 * the workspace: the scratch lives in a static device array of
 * soup_lora_linear_bwd_noalloc_max_scratch() bytes (8 MiB) that every GPU
 * loading the library holds until the process exits.
 *  - Sizes whose scratch, soup_lora_linear_bwd_workspace(T, r, out), exceeds
 *    that maximum are refused with SOUP_ERR_SHAPE and a message (nothing runs).
 *  - The first call on each device does a one-time set-up (it looks up the
 *    array's device address with that device current and caches it with the
 *    device's context; a call in a new context, e.g. after cudaDeviceReset,
 *    looks it up again); make that first call before any stream capture.
 *  - Every call shares the one array and it keeps the last call's contents:
 *    calls that overlap on the GPU (different streams, or different host
 *    threads on one device) race and corrupt each other's results; serialise
 *    them.  No part of the scratch has to start at zero.
 *  - Never calls cudaMalloc, cudaFree or any allocating routine. */
size_t soup_lora_linear_bwd_noalloc_max_scratch(void);
/* Device bytes the library holds in module-static arrays (the scratch above)
 * on every device that loads it: memory outside any allocator, to be counted
 * against a device budget. */
size_t soup_static_device_bytes(void);
soup_status soup_lora_linear_bwd_noalloc(const soup_weight* W, const uint16_t* A, const uint16_t* B,
                                         int32_t r, float scale, const uint16_t* x,
                                         const uint16_t* u_save, const uint16_t* dy, int64_t T,
                                         uint16_t* dx, float* dA, float* dB, void* stream);

/* ------------------------------------------------------------- attention ---
 * The decoder layer's causal GQA attention on its own (Soup pages, "how layer
 * streaming works": the layer the stream feeds; the attention itself is the
 * Llama-3.1-8B layer's: causal within each sequence, kv head = q head /
 * (n_q_heads / n_kv_heads), scale 1/sqrt(128)).  head_dim is 128.
 * Token layout: `batch` sequences of `seq` tokens.  prefix_share <= 1: each
 * sequence is its own `seq` rows (sequence b = rows [b*seq, (b+1)*seq)).
 * prefix_share = G > 1: consecutive groups of G sequences share their first
 * prefix_len tokens (a positive multiple of 128, < seq), stored once: a
 * group's rows are [prefix | continuation of its sequence 0 | ... | of its
 * sequence G-1], G * (seq - prefix_len) + prefix_len rows per group (the
 * preference pairs of a DPO step with one prompt); the prefix's own queries
 * belong to sequence 0 of the group; dk, dv of a prefix row sum the
 * contributions of every sequence of the group.  T = number of rows.
 * qkv: [T, ld] fp16 (ld >= (n_q + 2 n_kv) * 128, ld % 8 == 0, base 16-byte
 * aligned): q heads at columns [0, 128 n_q), k heads after them, then v heads;
 * q and k as they enter the dot products (after RoPE).
 * soup_attention_fwd: out [T, 128 n_q] bf16, out16 (may be NULL) the same
 * values in fp16, lse [n_q, T] fp32 = log2 of each row's softmax denominator
 * including the row maximum (log2 units).
 * soup_attention_bwd: from the forward's out16 and lse and dout [T, 128 n_q]
 * fp16, writes D [n_q, T] (rowsum(dout * out), a buffer the caller provides)
 * and dq, dk, dv (bf16) into dqkv at qkv's layout (dq includes the
 * 1/sqrt(128) scale; row stride ld), and the same values in fp32 into dqkv32
 * when it is not NULL.  Both run on the tensor cores (tcgen05, accumulators
 * in tensor memory), are deterministic, and are async on `stream`.
 * Refusals: SOUP_ERR_SHAPE (bad sizes, n_q % n_kv != 0, a prefix layout that
 * does not fit), SOUP_ERR_ALIGN. */
soup_status soup_attention_fwd(const uint16_t* qkv, int64_t ld, int64_t batch, int64_t seq, int32_t n_q_heads,
                               int32_t n_kv_heads, int32_t prefix_share, int64_t prefix_len, uint16_t* out,
                               uint16_t* out16, float* lse, void* stream);
soup_status soup_attention_bwd(const uint16_t* qkv, int64_t ld, int64_t batch, int64_t seq, int32_t n_q_heads,
                               int32_t n_kv_heads, int32_t prefix_share, int64_t prefix_len, const uint16_t* out16,
                               const uint16_t* dout, const float* lse, float* D, uint16_t* dqkv, float* dqkv32,
                               void* stream);

/* --------------------------------------------------------- decoder layer ---
 * One Llama-style decoder layer with LoRA on all seven projections (the unit
 * the pages stream "one decoder layer at a time"; Soup pages, "layer
 * streaming" and "how layer streaming works"):
 *   x1 = RMSNorm(h; norm1); q,k,v = LoRA projections of x1; RoPE(q, k);
 *   h2 = h + LoRA_o(causal GQA attention(q, k, v));
 *   x2 = RMSNorm(h2; norm2); h_out = h2 + LoRA_down(silu(LoRA_gate(x2)) * LoRA_up(x2)).
 * RMSNorm y = x / sqrt(mean(x^2) + eps) * w (w frozen); RoPE rotates pairs
 * (i, i + d/2) by pos * theta^(-2i/d), positions restarting in every sequence;
 * attention scale 1/sqrt(d), kv head = q_head / (Hq / Hkv); no biases.
 * Activations are [T, features] bf16 with T = batch * seq (batch-major).
 */
typedef struct soup_layer_cfg {
  int32_t hidden;        /* H: a multiple of 256 */
  int32_t n_q_heads;     /* Hq */
  int32_t n_kv_heads;    /* Hkv: divides Hq */
  int32_t head_dim;      /* d: must be 128 */
  int32_t intermediate;  /* I: a multiple of 128 */
  int32_t rank;          /* r: must be 16 */
  float alpha;           /* LoRA scale s = alpha / r */
  float eps;             /* RMSNorm epsilon */
  float theta;           /* RoPE base */
  /* Token layout of the layer calls' `batch` sequences of `seq` tokens.
   * prefix_share <= 1: sequence b is token rows [b*seq, (b+1)*seq).
   * prefix_share = G > 1: consecutive groups of G sequences share their
   * first prefix_len tokens (a positive multiple of 128, < seq), stored once
   * per group as [prefix | continuation of sequence 0 | ... | of sequence
   * G-1]: a preference pair's prompt is computed once (G = 2).  Every
   * activation buffer of the layer calls then holds
   * batch / G * (prefix_len + G * (seq - prefix_len)) rows. */
  int32_t prefix_share;
  int32_t prefix_len;
} soup_layer_cfg;

/* The frozen base of one layer (all NF4 or all bf16), as it sits in a device
 * slot.  Fused row layouts: qkv = [q; k; v] rows ([(Hq + 2 Hkv) d, H]),
 * gate_up = [gate; up] rows ([2 I, H]); o [H, Hq d]; down [H, I]. */
typedef struct soup_layer_weights {
  soup_weight qkv, o, gate_up, down;
  const uint16_t* norm1; /* [H] bf16 */
  const uint16_t* norm2; /* [H] bf16 */
} soup_layer_weights;

/* LoRA factors (bf16), concatenated in the same row order as the base:
 * A_qkv [3r, H] = [A_q; A_k; A_v], B_qkv [(Hq + 2 Hkv) d, r] = [B_q; B_k; B_v],
 * A_o [r, Hq d], B_o [H, r], A_gu [2r, H] = [A_gate; A_up],
 * B_gu [2I, r] = [B_gate; B_up], A_down [r, I], B_down [H, r]. */
typedef struct soup_layer_lora {
  const uint16_t *A_qkv, *B_qkv, *A_o, *B_o, *A_gu, *B_gu, *A_down, *B_down;
} soup_layer_lora;

/* fp32 gradients of the LoRA factors, same shapes as soup_layer_lora
 * (overwritten by soup_decoder_layer_bwd). */
typedef struct soup_layer_grads {
  float *dA_qkv, *dB_qkv, *dA_o, *dB_o, *dA_gu, *dB_gu, *dA_down, *dB_down;
} soup_layer_grads;

/* Workspace bytes the layer calls need for (batch, seq). */
size_t soup_decoder_layer_workspace(const soup_layer_cfg* cfg, int64_t batch, int64_t seq);

/* Forward: h_in [T, H] bf16 -> h_out [T, H] bf16.  adapters_on = 0 drops
 * every LoRA term (the adapters-off reference model used for DPO).
 * workspace: >= soup_decoder_layer_workspace bytes, 256-byte aligned. */
soup_status soup_decoder_layer_fwd(const soup_layer_weights* W, const soup_layer_lora* lora,
                                   const soup_layer_cfg* cfg, const uint16_t* h_in, int64_t batch,
                                   int64_t seq, uint16_t* h_out, int32_t adapters_on, void* workspace,
                                   size_t workspace_bytes, void* stream);

/* Recompute-backward: re-runs the forward from h_in (keeping intermediates),
 * then back-propagates dh_out [T, H] fp32 (gradient w.r.t. h_out) to
 * dh_in [T, H] fp32 and fills the LoRA gradients.  W gets no gradient.
 * dh_in may alias dh_out.  With adapters_on = 0 the grads are not written.
 * The LoRA-factor gradients (dA, dB) run on a library-internal stream of the
 * device, forked from `stream` by events and joined back into it before the
 * call returns: to the caller all of the layer's work is ordered on
 * `stream` as usual (the dA / dB GEMMs overlap the dx chain on the GPU). */
soup_status soup_decoder_layer_bwd(const soup_layer_weights* W, const soup_layer_lora* lora,
                                   const soup_layer_cfg* cfg, const uint16_t* h_in,
                                   const float* dh_out, int64_t batch, int64_t seq, float* dh_in,
                                   const soup_layer_grads* grads, int32_t adapters_on,
                                   void* workspace, size_t workspace_bytes, void* stream);

/* Selective keep of the layer's q|k|v between its two reads (the pages'
 * forward read and recompute read of every layer; deep dive, section "How
 * layer streaming works"): the forward pass, which waits on its copy stream
 * anyway, computes q|k|v from the fp32-accurate normalised input (the same
 * values the recompute would produce) and leaves them in qkv_keep; the
 * backward then skips its q|k|v GEMM.  Results are bit-identical to the
 * fwd + recompute pair above.  qkv_keep: fp16 [T, (Hq + 2 Hkv) * head_dim],
 * soup_decoder_layer_keep_bytes bytes, 16-byte aligned, owned by the caller
 * and kept untouched between the two calls of the same layer. */
size_t soup_decoder_layer_keep_bytes(const soup_layer_cfg* cfg, int64_t batch, int64_t seq);
soup_status soup_decoder_layer_fwd_keep(const soup_layer_weights* W, const soup_layer_lora* lora,
                                        const soup_layer_cfg* cfg, const uint16_t* h_in, int64_t batch,
                                        int64_t seq, uint16_t* h_out, int32_t adapters_on, uint16_t* qkv_keep,
                                        void* workspace, size_t workspace_bytes, void* stream);
soup_status soup_decoder_layer_bwd_kept(const soup_layer_weights* W, const soup_layer_lora* lora,
                                        const soup_layer_cfg* cfg, const uint16_t* h_in,
                                        const float* dh_out, int64_t batch, int64_t seq, float* dh_in,
                                        const soup_layer_grads* grads, int32_t adapters_on,
                                        const uint16_t* qkv_kept, void* workspace, size_t workspace_bytes,
                                        void* stream);

/* Keep-activations form (the pages' `stream_recompute` key: keep the
 * layer's activations instead of recomputing them; Soup pages, the streaming
 * configuration keys).  soup_decoder_layer_fwd_save runs the forward pass and
 * leaves every intermediate the backward reads (the normalised inputs, q|k|v
 * from the hi + lo input, the attention output and log-sum-exp, the mid
 * residual, the SwiGLU inputs and output, the LoRA down-projections, ...) in
 * `saved`, soup_decoder_layer_saved_bytes bytes, 256-byte aligned, owned by
 * the caller and left untouched until soup_decoder_layer_bwd_saved of the
 * same layer, which then runs no forward recompute at all (the layer is still
 * read a second time: the backward needs W^T).  Results are bit-identical to
 * the soup_decoder_layer_fwd_keep / soup_decoder_layer_bwd_kept pair (same
 * kernels on the same values).  The workspace is the same as for the other
 * forms. */
size_t soup_decoder_layer_saved_bytes(const soup_layer_cfg* cfg, int64_t batch, int64_t seq);
soup_status soup_decoder_layer_fwd_save(const soup_layer_weights* W, const soup_layer_lora* lora,
                                        const soup_layer_cfg* cfg, const uint16_t* h_in, int64_t batch,
                                        int64_t seq, uint16_t* h_out, int32_t adapters_on, void* saved,
                                        void* workspace, size_t workspace_bytes, void* stream);
soup_status soup_decoder_layer_bwd_saved(const soup_layer_weights* W, const soup_layer_lora* lora,
                                         const soup_layer_cfg* cfg, const uint16_t* h_in,
                                         const float* dh_out, int64_t batch, int64_t seq, float* dh_in,
                                         const soup_layer_grads* grads, int32_t adapters_on, const void* saved,
                                         void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------- layer streaming ---
 * The frozen base lives in pinned host RAM as one blob per decoder layer
 * (Soup pages, "how layer streaming works": per-layer shards in page-locked
 * host memory; `stream_buffers` preallocated device buffers, 2..8, default 2;
 * a dedicated CUDA stream copies the next layer while the current one
 * computes; the vocab-sized embed_tokens and an untied lm_head share one
 * slot).  A plan owns the only device memory this library allocates: an
 * arena of n_buffers layer slots plus one vocab slot, a copy stream and
 * events.  Slots are reused least-recently-released first; prefetching an
 * item that is still resident in a released slot makes no copy.
 */
#define SOUP_ITEM_NONE (-100)
#define SOUP_ITEM_EMBED (-1) /* the embed_tokens matrix, into the vocab slot */
#define SOUP_ITEM_HEAD (-2)  /* the lm_head matrix, into the vocab slot */

typedef struct soup_plan soup_plan; /* opaque */

typedef struct soup_stream_desc {
  int32_t n_layers;
  size_t layer_bytes;              /* bytes of one layer blob (multiple of 256) */
  const void* const* host_layers;  /* n_layers pinned host blobs, or NULL when every layer copy
                                      comes from soup_stream_prefetch_from (disk tier) */
  size_t vocab_bytes;              /* bytes of the vocab slot (0: none; multiple of 256) */
  const void* host_embed;          /* pinned host embed_tokens blob (vocab_bytes) or NULL */
  const void* host_head;           /* pinned host lm_head blob or NULL (tied: same as embed) */
  int32_t n_buffers;               /* stream_buffers: 2..8 */
  size_t device_cap_bytes;         /* 0: no cap; else refuse plans that exceed it */
  size_t reserve_bytes;            /* device bytes the caller holds besides the plan */
} soup_stream_desc;

typedef struct soup_stream_stats_t {
  int64_t copies;      /* H2D copies issued */
  int64_t reuses;      /* prefetches served by a still-resident slot */
  size_t bytes_copied;
  size_t arena_bytes;
  int64_t waits;       /* soup_stream_wait calls */
  double stall_ms;     /* total time the compute stream spent inside those waits */
  double copy_ms;      /* total duration of the copies on the copy stream */
} soup_stream_stats_t;

/* Allocates the slot arena and the copy stream.  Refuses (no allocation)
 * with SOUP_ERR_INVALID_ARG when n_buffers is outside [2, 8], and with
 * SOUP_ERR_OOM_PLAN when n_buffers * layer_bytes + vocab_bytes +
 * reserve_bytes exceeds a nonzero device_cap_bytes. */
soup_status soup_stream_plan(const soup_stream_desc* desc, soup_plan** plan_out);
soup_status soup_stream_plan_free(soup_plan* plan);

/* Enqueues the copy of `item` (a layer index, SOUP_ITEM_EMBED or
 * SOUP_ITEM_HEAD) into a free slot on the plan's copy stream; the copy first
 * waits (on the device) until the compute stream released the slot's
 * previous item.  Copies of 8 MiB or more are split in two halves, the
 * second on a second copy stream (a second DMA engine), joined back before
 * the item is marked ready.  Refuses when every slot of the kind holds an
 * unreleased item or the item is already held. */
soup_status soup_stream_prefetch(soup_plan* plan, int32_t item);

/* As soup_stream_prefetch for a layer, but the copy reads `host_src` (a
 * page-locked buffer of layer_bytes, e.g. a disk-tier staging buffer) and,
 * when copy_done_event (a cudaEvent_t) is not NULL, records it on the copy
 * stream once the copy has finished reading host_src.  A layer still
 * resident in a released slot is reused as by soup_stream_prefetch (no copy,
 * the event is not recorded).  Layers of a plan made without host_layers
 * can only be brought in this way. */
soup_status soup_stream_prefetch_from(soup_plan* plan, int32_t layer, const void* host_src,
                                      void* copy_done_event);

/* *resident <- 1 if a slot holds `item` (a prefetch of it makes no copy;
 * while it is still held, a prefetch refuses), else 0.  Host only. */
soup_status soup_stream_resident(soup_plan* plan, int32_t item, int32_t* resident);

/* Makes `compute_stream` wait (on the device) until the item's copy is done
 * and returns the slot's device address in *slot_dev. */
soup_status soup_stream_wait(soup_plan* plan, int32_t item, void* compute_stream, void** slot_dev);

/* Host-side wait for the item's copy, at most timeout_ms; SOUP_ERR_TIMEOUT
 * when it does not finish in time (the copy is left in flight). */
soup_status soup_stream_wait_host(soup_plan* plan, int32_t item, int32_t timeout_ms);

/* Marks the item's slot reusable once `compute_stream` reaches this point. */
soup_status soup_stream_release(soup_plan* plan, int32_t item, void* compute_stream);

/* Copy/stall statistics since the plan was made or last reset (synchronises
 * the copy stream and the recorded events).  The timing events form two
 * fixed rings of 256 (start, end) pairs (one for copies, one for waits):
 * an entry's elapsed time is folded into a running total before the entry
 * is reused, so a run of any length holds a bounded number of events. */
soup_status soup_stream_stats(soup_plan* plan, soup_stream_stats_t* out);
soup_status soup_stream_stats_reset(soup_plan* plan);

/* The plan's copy stream (cudaStream_t as void*). */
void* soup_stream_copy_stream(soup_plan* plan);

/* Number of CUDA events the plan holds for its statistics (at most 1024;
 * -1 for a NULL plan).  Host only. */
int64_t soup_stream_debug_timing_events(soup_plan* plan);

/* Fault-injection hooks for tests (host side only): the next prefetch fails
 * with SOUP_ERR_CUDA without copying; or the next copy first waits on
 * `event` (a cudaEvent_t). */
soup_status soup_stream_debug_fail_next_copy(soup_plan* plan);
soup_status soup_stream_debug_gate_next_copy(soup_plan* plan, void* event);

/* ------------------------------------------------------------ disk tier ---
 * The pages' `stream_source: disk` with `stream_read_ahead` (1..8): the
 * frozen base's per-layer shards are files (one per layer, layer_bytes each,
 * the blob layout below), read ahead into `read_ahead` host staging buffers
 * by `io_threads` threads, each read cut into 8 MiB requests (Soup pages,
 * "how layer streaming works" and the streaming configuration keys).
 * The reader follows a cyclic layer visit order (soup_disk_schedule: one
 * training step's visits, e.g. 0..L-1 then L-1..0) and replays the plan's
 * slot ring (n_slots = stream_buffers, least recently used first) over it, so
 * it reads only the visits that need a copy.  A consumer that visits layers
 * in that order calls, for a layer that soup_stream_resident reports absent:
 * soup_disk_acquire -> soup_stream_prefetch_from(host, event) ->
 * soup_disk_release.  A staging buffer is refilled only after its
 * copy-done event has completed.  Visits the consumer passes over are
 * dropped (stats.skipped); a layer acquired out of order resynchronises the
 * reader on its next visit: results never depend on the schedule.
 * flags: SOUP_DISK_PINNED: page-locked staging buffers (cudaHostAlloc) and
 * one CUDA event per buffer for the copy hand-off (needs a device); without
 * it, plain page-aligned host memory and no CUDA call at all (host-side use
 * and tests).  SOUP_DISK_DIRECT: O_DIRECT reads (no page-cache copy), per
 * file, where the file system accepts them (else buffered reads).
 * Errors: SOUP_ERR_IO (a file cannot be opened or read; a read error is
 * reported by the acquire of that visit), SOUP_ERR_SHAPE (a file's size is
 * not layer_bytes), SOUP_ERR_TIMEOUT (acquire waited timeout_ms), and
 * SOUP_ERR_INVALID_ARG (out-of-range arguments, a layer not in the
 * schedule, a layer acquired twice or released without being held). */
#define SOUP_DISK_PINNED 1
#define SOUP_DISK_DIRECT 2

typedef struct soup_disk soup_disk; /* opaque */

typedef struct soup_disk_stats_t {
  int64_t reads;       /* staging buffers filled with a visit that was then acquired or is waiting */
  int64_t skipped;     /* visits read (or being read) and then passed over */
  int64_t acquires;
  uint64_t bytes_read;
  double read_ms;      /* sum over reads of the time from start to last byte (reads overlap) */
  double wait_ms;      /* total time acquire calls waited */
  int32_t direct_files;/* shards read with O_DIRECT */
} soup_disk_stats_t;

soup_status soup_disk_open(const char* const* paths, int32_t n_layers, size_t layer_bytes, int32_t read_ahead,
                           int32_t n_slots, int32_t io_threads, int32_t flags, soup_disk** out);
soup_status soup_disk_close(soup_disk* disk);
/* Sets the cyclic visit order (layer indices, each < n_layers) and restarts
 * the reader on it; refused while a staging buffer is held. */
soup_status soup_disk_schedule(soup_disk* disk, const int32_t* order, int32_t n);
/* Waits (at most timeout_ms) for the staging buffer of `layer`'s next copied
 * visit; *host <- its address (layer_bytes valid), *copy_done_event <- the
 * buffer's cudaEvent_t (NULL without SOUP_DISK_PINNED).  The buffer is held
 * until soup_disk_release. */
soup_status soup_disk_acquire(soup_disk* disk, int32_t layer, int32_t timeout_ms, const void** host,
                              void** copy_done_event);
soup_status soup_disk_release(soup_disk* disk, int32_t layer);
soup_status soup_disk_stats(soup_disk* disk, soup_disk_stats_t* out);

/* Layer blob layout (host arithmetic, no device access).  NF4 blob: qkv
 * codes | qkv absmax | o codes | o absmax | gate_up codes | gate_up absmax |
 * down codes | down absmax | norm1 | norm2; bf16 blob: qkv | o | gate_up |
 * down | norm1 | norm2; every part 256-byte aligned.  soup_layer_blob_views
 * fills *out with pointers into a blob at `base`. */
size_t soup_layer_blob_bytes(const soup_layer_cfg* cfg, int32_t kind);
soup_status soup_layer_blob_views(const soup_layer_cfg* cfg, int32_t kind, const void* base,
                                  soup_layer_weights* out);

/* ------------------------------------------------------- embedding, head ---
 * Token embedding gather: h[t] = E[ids[t]] (E [V, H] bf16 in the vocab slot,
 * ids [T] int32).  An id outside [0, V) writes a zero row and sets code 2 in
 * the device error word. */
soup_status soup_embed(const uint16_t* E, int64_t V, int64_t H, const int32_t* ids, int64_t T,
                       uint16_t* h, void* stream);

/* Final RMSNorm + lm_head + next-token log-probabilities, `chunk` tokens at a
 * time (the pages' stream_loss_chunk):  x = RMSNorm(h; w_final),
 * logp[b, s] = log softmax(x_t E^T)[ids[b, s+1]] for t = b*seq + s, s < seq-1.
 * h [batch*seq, H] bf16, E [V, H] bf16 (lm_head), ids [batch, seq] int32,
 * logp [batch, seq-1] fp32.  When coef [batch, seq-1] (= dL/dlogp) is given,
 * also dh [batch*seq, H] fp32 = dL/dh.  Logits are fp32; dL/dlogits enter the
 * backward GEMM in bf16. */
size_t soup_head_workspace(int64_t V, int64_t H, int64_t batch, int64_t seq, int32_t chunk);
soup_status soup_head_fwd_bwd(const uint16_t* h, const uint16_t* w_final, const uint16_t* E, int64_t V,
                              int64_t H, const int32_t* ids, int64_t batch, int64_t seq, float eps,
                              int32_t chunk, const float* coef, float* logp, float* dh, void* workspace,
                              size_t workspace_bytes, void* stream);

/* Row gather: dst[i] = src[idx[i]] for i < n, rows of row_bytes bytes (a
 * multiple of 4; device pointers).  Used to lay out a preference batch's
 * tokens with the shared prompt stored once and to collect the rows the
 * output head reads.  Async on `stream`. */
soup_status soup_gather_rows(const void* src, int64_t row_bytes, const int32_t* idx, int64_t n, void* dst,
                             void* stream);
/* Row sums in a fixed order: dst[d] = sum over k in [start[d], start[d+1]) of
 * src[src_idx[k]] (fp32 rows of H values; an empty range gives zeros), for
 * d < n_dst.  Scatters the head's dL/dh back to the token rows, adding the
 * contributions of both sequences of a pair at their shared prompt row
 * (deterministic).  Async on `stream`. */
soup_status soup_sum_rows_f32(const float* src, int64_t H, const int32_t* src_idx, const int32_t* start,
                              int64_t n_dst, float* dst, void* stream);

/* Mean next-token cross-entropy over batch*(seq-1) targets into *loss (a
 * device float; optional, then logp may be NULL); coef (optional) <-
 * dL/dlogp = -1/(batch*(seq-1)), which does not depend on logp and so can be
 * produced before the head runs. */
soup_status soup_ce_loss(const float* logp, int64_t batch, int64_t seq, float* loss, float* coef,
                         void* stream);

/* DPO loss (Rafailov et al. 2023) over `pairs` preference pairs; rows 2p /
 * 2p+1 of the [2*pairs, seq-1] log-prob arrays are the chosen / rejected
 * sequence of pair p, sharing a prompt of prompt_len tokens.  Sequence
 * log-probs sum the targets at positions >= prompt_len (continuation tokens).
 *   L = -(1/P) sum_p log sigmoid(beta [(pi_c - ref_c) - (pi_r - ref_r)])
 * logp_policy: adapters on; logp_ref: the same streamed base with adapters
 * off (the pages' memory-free reference model).  *loss (device) <- L;
 * seq_sums (optional, [4*pairs]) <- policy sums then reference sums;
 * coef [2*pairs, seq-1] <- dL/dlogp_policy (zero on prompt positions). */
soup_status soup_dpo_loss(const float* logp_policy, const float* logp_ref, int64_t pairs, int64_t seq,
                          int64_t prompt_len, float beta, float* loss, float* seq_sums, float* coef,
                          void* stream);

/* Reference-free preference losses (the pages name ORPO and SimPO as the
 * methods without DPO's reference reads: "memory-free reference model").
 * logp [2*pairs, seq-1] holds the policy's next-token log-probs; rows 2p /
 * 2p+1 are the chosen / rejected sequence of pair p, sharing a prompt of
 * prompt_len tokens, so each row has n = seq - max(prompt_len, 1)
 * continuation targets (positions j with j + 1 >= prompt_len).  With s a
 * row's summed continuation log-probs and m = s / n:
 *   SimPO (Meng, Xia & Chen 2024):
 *     L = -(1/P) sum_p log sigmoid(beta (m_c - m_r) - gamma)
 *   ORPO (Hong, Lee & Thorne 2024), lo = m - log(1 - exp(m)) the log odds:
 *     L = (1/P) sum_p [ -m_c - lam log sigmoid(lo_c - lo_r) ]
 * *loss (device float) <- L; seq_sums (optional, [2*pairs]) <- s per row;
 * coef [2*pairs, seq-1] <- dL/dlogp (0 on prompt positions).  One kernel
 * launch; SOUP_ERR_SHAPE unless 1 <= pairs <= 2048, seq >= 2 and
 * 0 <= prompt_len < seq.  A row whose mean log-likelihood is 0 (probability
 * 1) has infinite log odds: ORPO is then not finite. */
soup_status soup_simpo_loss(const float* logp, int64_t pairs, int64_t seq, int64_t prompt_len, float beta,
                            float gamma, float* loss, float* seq_sums, float* coef, void* stream);
soup_status soup_orpo_loss(const float* logp, int64_t pairs, int64_t seq, int64_t prompt_len, float lam,
                           float* loss, float* seq_sums, float* coef, void* stream);

/* ---------------------------------------------------------------- AdamW ---
 * One AdamW step over the LoRA adapters, which stay resident in device memory
 * with their gradients and optimiser state while the base streams (Soup
 * pages, "how layer streaming works").  AdamW is Adam with decoupled weight
 * decay (Loshchilov & Hutter, "Decoupled Weight Decay Regularization", ICLR
 * 2019), the decay folded into the learning rate.  For i < n, with
 * g = grad_scale * grad[i]:
 *   theta <- theta * (1 - lr * weight_decay)
 *   m     <- beta1 * m + (1 - beta1) * g
 *   v     <- beta2 * v + (1 - beta2) * g^2
 *   theta <- theta - (lr / (1 - beta1^t)) * m / (sqrt(v) / sqrt(1 - beta2^t) + eps)
 * theta (the fp32 master copy), m, v: fp32 [n], updated in place.  grad:
 * fp32 [n], read, then set to zero when zero_grad != 0 (a backward pass that
 * accumulates can then run straight into it).  theta_bf16 (optional, NULL to
 * skip): bf16 [n] <- round-to-nearest-even of the new theta, the working copy
 * the GEMMs read.  t >= 1 is this step's index; the bias corrections are
 * formed on the host in double.  grad_scale multiplies the incoming gradient
 * (1/world when it arrives as a data-parallel sum).  nonfinite_dev (optional):
 * a device int32 set to 1 when a gradient element is NaN or Inf (the update
 * is still applied; the call never clears it).
 * Errors: SOUP_ERR_ALIGN unless theta, grad, m, v are 16-byte and theta_bf16
 * 8-byte aligned; SOUP_ERR_INVALID_ARG for t < 1, a beta outside [0, 1),
 * eps <= 0, or a negative lr / weight_decay.  n = 0 is a no-op.  One kernel
 * launch, asynchronous on `stream`; the caller owns every buffer. */
soup_status soup_adamw_step(float* theta, uint16_t* theta_bf16, float* grad, float* m, float* v, int64_t n,
                            float lr, float beta1, float beta2, float eps, float weight_decay,
                            float grad_scale, int64_t t, int32_t zero_grad, int32_t* nonfinite_dev,
                            void* stream);

#ifdef __cplusplus
}
#endif
#endif /* SOUP_H_ */
