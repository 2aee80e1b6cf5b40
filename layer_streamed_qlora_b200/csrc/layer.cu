// One decoder layer, forward and recompute-backward, as a sequence of the
// library's kernels on one stream:
//
// forward:  RMSNorm -> [u_qkv] -> QKV GEMM (NF4 decode + 3-segment LoRA tail,
//           RoPE on q/k in the epilogue, fp16 out) -> attention -> [u_o]
//           -> O GEMM (+ residual, fp32 out) -> RMSNorm -> [u_gu]
//           -> gate|up GEMM on paired tiles with SwiGLU in the epilogue
//           -> [u_d] -> down GEMM (+ fp32 residual, bf16 out)
// backward: the forward again from the saved layer input (the layer was read
//           a second time for this; the down GEMM's output is not needed and
//           is skipped), then in reverse: g = dy B (per adapter), dx = dy W +
//           g' A (NF4 decode of W^T + tail; the down projection's epilogue
//           applies the SwiGLU backward), dB = dy^T u, dA = g'^T x for each
//           projection group, with RMSNorm / attention backward in between
//           (inverse RoPE in the attention-backward epilogues).  The
//           residual-stream gradient and the mid-layer residual h2 stay fp32.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "elementwise.h"
#include "lora_internal.h"

namespace soup {
namespace {

struct Dims {
  int T, S, B, H, Hq, Hkv, d, I, r, qkv_w, o_in;
  int G, Lp;  // groups of G sequences sharing Lp prefix tokens (G = 1: none); T = token rows
  int64_t ldT;
  float s;
};

// Workspace layout (byte offsets, each 256-aligned).
struct WS {
  size_t x1, rinv1, qkv, attn, lse, h2, x2, rinv2, gu16, act, u_qkv, u_o, u_gu, u_d, cosb, sinb;
  size_t dh_b, g_d, g_gu, g_o, g_qkv, d_gu, dx2, dh2, dh2_b, d_attn, D, d_qkv, dx1, attn16, gamax;
  size_t x1_32, dqkv32, u32, g32, A32;  // fp32 operands of the q/k/v LoRA-gradient GEMMs (tf32)
  size_t x1_lo, dh2_lo;                       // bf16 rounding residuals (dual-A GEMM inputs)
  size_t attn32, uo32, go32, Ao32;            // fp32 operands of the o LoRA-gradient GEMMs (tf32)
  size_t splitk, splitk_bytes;                // fp32 partial products of split-K LoRA GEMMs
  size_t splitk2;                             // the same for the GEMMs of the side stream (backward)
  size_t u_gu_lo, g_d_lo, u_d32;     // MLP LoRA-gradient operands beyond bf16 (residuals, fp32)
  size_t x2_32, Agu32, g_gu32, d_gu_lo;
  size_t Bt_down32, Bt_o32, Bbd_qkv32, Bbd_gu;  // B factors prepared for the g GEMMs (transposed, block-diagonal)
  size_t fwd_bytes;  // [0, fwd_bytes): the fields the forward pass leaves for the backward
  size_t total;
};

WS layout(const Dims& m) {
  WS w;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    size_t at = o;
    o += align256(bytes);
    return at;
  };
  const size_t T = m.T, H = m.H, I = m.I, r = m.r, ldT = m.ldT;
  // ---- fields the forward pass computes and the backward reads (the part a
  // saved layer keeps): offsets [0, fwd_bytes)
  w.x1 = take(T * H * 2);
  w.rinv1 = take(T * 4);
  w.qkv = take(T * m.qkv_w * 2);  // fp16
  w.attn = take(T * m.o_in * 2);
  w.lse = take((size_t)m.Hq * T * 4);
  w.h2 = take(T * H * 4);  // fp32
  w.x2 = take(T * H * 2);
  w.rinv2 = take(T * 4);
  w.gu16 = take(T * 2 * I * 2);  // fp16 g | u saved for the SwiGLU backward
  w.act = take(T * I * 2);
  w.u_qkv = take(3 * r * ldT * 2);
  w.u_o = take(r * ldT * 2);
  w.u_gu = take(2 * r * ldT * 2);
  w.u_d = take(r * ldT * 2);
  w.cosb = take((size_t)m.S * (m.d / 2) * 4);
  w.sinb = take((size_t)m.S * (m.d / 2) * 4);
  w.attn16 = take(T * m.o_in * 2);  // fp16 copy of the attention output (for D = rowsum(dO * O))
  w.x1_32 = take(T * H * 4);
  w.u32 = take(3 * r * ldT * 4);
  w.A32 = take(3 * r * H * 4);
  w.x1_lo = take(T * H * 2);
  w.attn32 = take(T * m.o_in * 4);
  w.uo32 = take(r * ldT * 4);
  w.Ao32 = take(r * (size_t)m.o_in * 4);
  w.u_gu_lo = take(2 * r * ldT * 2);
  w.u_d32 = take(r * ldT * 4);
  w.x2_32 = take(T * H * 4);
  w.Agu32 = take(2 * r * H * 4);
  w.fwd_bytes = o;
  // ---- backward-only fields and scratch
  w.dh_b = take(T * H * 2);
  w.g_d = take(r * ldT * 2);
  w.g_gu = take(2 * r * ldT * 2);
  w.g_o = take(r * ldT * 2);
  w.g_qkv = take(3 * r * ldT * 2);
  w.d_gu = take(T * 2 * I * 2);
  w.dx2 = take(T * H * 2);
  w.dh2 = take(T * H * 4);
  w.dh2_b = take(T * H * 2);
  w.d_attn = take(T * m.o_in * 2);  // fp16
  w.D = take((size_t)m.Hq * T * 4);
  w.d_qkv = take(T * m.qkv_w * 2);
  w.dx1 = take(T * H * 2);
  w.gamax = take(4);                // max |dh2| bit pattern (gradient scale of dO)
  w.dqkv32 = take(T * m.qkv_w * 4);
  w.g32 = take(3 * r * ldT * 4);
  w.dh2_lo = take(T * H * 2);
  w.go32 = take(r * ldT * 4);
  w.splitk_bytes = 8 * T * 64 * 4;
  w.splitk = take(w.splitk_bytes);
  w.splitk2 = take(w.splitk_bytes);
  w.g_d_lo = take(r * ldT * 2);
  w.g_gu32 = take(2 * r * ldT * 4);
  w.d_gu_lo = take(T * 2 * I * 2);
  w.Bt_down32 = take(r * H * 4);
  w.Bt_o32 = take(r * H * 4);
  w.Bbd_qkv32 = take(3 * r * (size_t)m.qkv_w * 4);
  w.Bbd_gu = take(2 * r * 2 * I * 2);
  w.total = o;
  return w;
}

soup_status make_dims(const soup_layer_cfg* c, int64_t batch, int64_t seq, Dims* m) {
  SOUP_CHECK(c, SOUP_ERR_INVALID_ARG, "decoder layer: null cfg");
  SOUP_CHECK(c->head_dim == 128, SOUP_ERR_SHAPE, "decoder layer: head_dim must be 128 (got %d)", c->head_dim);
  SOUP_CHECK(c->rank == 16, SOUP_ERR_SHAPE, "decoder layer: rank must be 16 (got %d)", c->rank);
  SOUP_CHECK(c->hidden > 0 && c->hidden % 256 == 0, SOUP_ERR_SHAPE, "decoder layer: hidden %% 256");
  SOUP_CHECK(c->n_q_heads > 0 && c->n_kv_heads > 0 && c->n_q_heads % c->n_kv_heads == 0, SOUP_ERR_SHAPE,
             "decoder layer: heads %d/%d", c->n_q_heads, c->n_kv_heads);
  SOUP_CHECK(c->intermediate > 0 && c->intermediate % 128 == 0, SOUP_ERR_SHAPE,
             "decoder layer: intermediate must be a multiple of 128");
  SOUP_CHECK(batch >= 1 && seq >= 1 && batch * seq < (1 << 24), SOUP_ERR_SHAPE, "decoder layer: batch/seq");
  SOUP_CHECK(c->eps >= 0.f && c->theta > 0.f, SOUP_ERR_INVALID_ARG, "decoder layer: eps/theta");
  const int G = c->prefix_share > 1 ? c->prefix_share : 1;
  const int Lp = G > 1 ? c->prefix_len : 0;
  SOUP_CHECK(G == 1 || (batch % G == 0 && Lp > 0 && Lp < seq && Lp % 128 == 0), SOUP_ERR_SHAPE,
             "decoder layer: prefix sharing needs groups of %d sequences dividing the batch (%lld) and a shared "
             "prefix that is a positive multiple of 128 shorter than the sequence (%d of %lld)", G, (long long)batch,
             Lp, (long long)seq);
  m->G = G; m->Lp = Lp;
  m->B = (int)batch; m->S = (int)seq;
  m->T = (int)((batch / G) * (Lp + G * (seq - Lp)));
  m->H = c->hidden; m->Hq = c->n_q_heads; m->Hkv = c->n_kv_heads; m->d = c->head_dim;
  m->I = c->intermediate; m->r = c->rank;
  m->qkv_w = (m->Hq + 2 * m->Hkv) * m->d;
  m->o_in = m->Hq * m->d;
  m->ldT = round_up8(m->T);
  m->s = c->alpha / (float)c->rank;
  return SOUP_OK;
}

soup_status check_weights(const soup_layer_weights* W, const Dims& m) {
  SOUP_CHECK(W && W->norm1 && W->norm2, SOUP_ERR_INVALID_ARG, "decoder layer: null weights");
  SOUP_TRY(check_weight(&W->qkv, "decoder layer qkv"));
  SOUP_TRY(check_weight(&W->o, "decoder layer o"));
  SOUP_TRY(check_weight(&W->gate_up, "decoder layer gate_up"));
  SOUP_TRY(check_weight(&W->down, "decoder layer down"));
  SOUP_CHECK(W->qkv.out_features == m.qkv_w && W->qkv.in_features == m.H, SOUP_ERR_SHAPE, "qkv shape");
  SOUP_CHECK(W->o.out_features == m.H && W->o.in_features == m.o_in, SOUP_ERR_SHAPE, "o shape");
  SOUP_CHECK(W->gate_up.out_features == 2 * m.I && W->gate_up.in_features == m.H, SOUP_ERR_SHAPE, "gate_up shape");
  SOUP_CHECK(W->down.out_features == m.H && W->down.in_features == m.I, SOUP_ERR_SHAPE, "down shape");
  return SOUP_OK;
}

// Field addresses: the forward pass's fields [0, fwd_bytes) live at `fb` (the
// layer workspace itself, or a saved layer's own region), the backward-only
// fields and scratch at `base` (the layer workspace).
#define FIELD(off) ((ws.off) < ws.fwd_bytes ? fb + (ws.off) : base + (ws.off))
#define P(off) (reinterpret_cast<uint16_t*>(FIELD(off)))
#define PF(off) (reinterpret_cast<float*>(FIELD(off)))

// Device memory a big GEMM may use for the partials of its split last
// round of tiles (nothing else reads or writes it during the call).
struct Scratch {
  void* p = nullptr;
  size_t bytes = 0;
};

// y = x W^T (+ tail u B^T) (+ resid) into out [T, N]
struct ProjOpts {
  int out_kind = OUT_BF16;
  const uint16_t* resid = nullptr;
  const float* resid_f32 = nullptr;
  int rope_cols = 0, rope_S = 0;
  const float* rope_cos = nullptr;
  const float* rope_sin = nullptr;
  int rope_prefix = 0, rope_group = 1;
  int swiglu_I = 0;          // > 0: paired gate|up tiles with the SwiGLU epilogue
  uint16_t* aux16 = nullptr; // SwiGLU: fp16 g | u output (may be null)
  const uint16_t* x_lo = nullptr;  // dual-A: bf16 rounding residual of x
  Scratch sk;
};

soup_status proj_fwd(const soup_weight* W, const uint16_t* x, int T, const uint16_t* u, int64_t ldT, int u_rows,
                     const uint16_t* Bl, int r, int nseg, const int* seg_end, const int* seg_row, bool on,
                     uint16_t* out, cudaStream_t st, const ProjOpts& o = ProjOpts()) {
  GemmDesc g;
  g.M = T; g.N = (int)W->out_features; g.K = (int)W->in_features;
  g.A = Mat{x, T, W->in_features, W->in_features};
  if (o.x_lo) g.A_lo = Mat{o.x_lo, T, W->in_features, W->in_features};
  set_weight_fwd(g, W);
  if (on) {
    g.tail_ksteps = r / 16;
    g.tailA = Mat{u, u_rows, T, ldT};
    g.tailB = Mat{Bl, W->out_features, r, r};
    g.nseg = nseg;
    for (int i = 0; i < nseg; ++i) { g.seg_end[i] = seg_end[i]; g.seg_row[i] = seg_row[i]; }
  }
  g.out_kind = o.out_kind; g.out = out; g.ldo = W->out_features;
  g.resid = o.resid; g.resid_f32 = o.resid_f32; g.ldr = W->out_features;
  g.rope_cols = o.rope_cols; g.rope_S = o.rope_S; g.rope_cos = o.rope_cos; g.rope_sin = o.rope_sin;
  g.rope_prefix = o.rope_prefix; g.rope_group = o.rope_group;
  g.sk_scratch = o.sk.p; g.sk_scratch_bytes = o.sk.bytes;
  if (o.swiglu_I > 0) {
    g.pair_off = o.swiglu_I;
    g.nseg = 1;
    g.epi = EPI_SWIGLU;
    g.swiglu_I = o.swiglu_I;
    g.ldo = o.swiglu_I;
    g.aux16 = o.aux16;
    g.ld_aux = 2 * (int64_t)o.swiglu_I;
  }
  return gemm(g, st);
}

// Split-K workspace handed to the skinny LoRA GEMMs.
struct SplitWS {
  float* p = nullptr;
  size_t bytes = 0;
};
void use_split(GemmDesc& g, const SplitWS& sw) {
  g.split_ws = sw.p;
  g.split_ws_bytes = sw.bytes;
}

// u' = bf16(s * x A^T), transposed [rows, ldT]
// (optionally also the fp32 values u32 and the rounding residual ulo)
soup_status lora_down(const uint16_t* x, int T, int K, const uint16_t* A, int rows, float s, uint16_t* u,
                      int64_t ldT, cudaStream_t st, const SplitWS& sw, float* u32 = nullptr,
                      uint16_t* ulo = nullptr) {
  GemmDesc g;
  g.M = T; g.N = rows; g.K = K;
  g.A = Mat{x, T, K, K};
  g.b_mode = B_TMA_K;
  g.B = Mat{A, rows, K, K};
  g.out_kind = OUT_BF16_T; g.out = u; g.ldo = ldT; g.alpha = s;
  g.out2 = u32; g.out_lo = ulo;
  use_split(g, sw);
  return gemm(g, st);
}


// g' = bf16(s * dy Bt^T) with a prepared Bt [rows, n] (transposed, possibly
// block-diagonal over segments of dy's columns): one GEMM for all segments;
// optionally dy's residual dy_lo (a second A), and the fp32 values g32 and
// residual glo as extra outputs.  tf32: dy, Bt fp32.
soup_status lora_g_prepared(const void* dy, const void* dy_lo, int64_t ld, int T, int n, const void* Bt, int rows,
                            float s, bool tf32, uint16_t* gout, float* g32, uint16_t* glo, int64_t ldT,
                            cudaStream_t st, const SplitWS& sw) {
  GemmDesc g;
  g.tf32 = tf32;
  g.M = T; g.N = rows; g.K = n;
  g.A = Mat{dy, T, n, ld};
  if (dy_lo) g.A_lo = Mat{dy_lo, T, n, ld};
  g.b_mode = B_TMA_K;
  g.B = Mat{Bt, rows, n, n};
  g.out_kind = OUT_BF16_T; g.out = gout; g.out2 = g32; g.out_lo = glo; g.ldo = ldT; g.alpha = s;
  use_split(g, sw);
  return gemm(g, st);
}

// dA [rows, K] = (g' + g_lo)^T x, with g' and its rounding residual g_lo
// stored transposed [rows, ldT] (a K-major A of M = rows) and x [T, K] the
// MN-major B: two bf16 MMAs per k-step give an fp32-accurate g.
soup_status lora_dA_dual(const uint16_t* gt, const uint16_t* gt_lo, int rows, int64_t ldT, const uint16_t* x, int T,
                         int K, float* dA, cudaStream_t st, const SplitWS& sw) {
  GemmDesc g;
  g.M = rows; g.N = K; g.K = T;
  g.A = Mat{gt, rows, T, ldT};
  g.A_lo = Mat{gt_lo, rows, T, ldT};
  g.b_mode = B_TMA_MN;
  g.B = Mat{x, T, K, K};
  g.out_kind = OUT_F32; g.out = dA; g.ldo = K;
  use_split(g, sw);
  return gemm(g, st);
}

// dB [n, r] = dy_seg^T (u' + u_lo)^T, computed as (u' + u_lo) dy_seg = dB^T
// (M = r) and stored transposed; dy = columns [c0, c0+n) of a [T, ld] buffer.
soup_status lora_dB_dual(const uint16_t* dy, int64_t ld, int T, int n, const uint16_t* ut, const uint16_t* ut_lo,
                         int r, int64_t ldT, float* dB, cudaStream_t st, const SplitWS& sw) {
  GemmDesc g;
  g.M = r; g.N = n; g.K = T;
  g.A = Mat{ut, r, T, ldT};
  g.A_lo = Mat{ut_lo, r, T, ldT};
  g.b_mode = B_TMA_MN;
  g.B = Mat{dy, T, n, ld};
  g.out_kind = OUT_F32_T; g.out = dB; g.ldo = r;
  use_split(g, sw);
  return gemm(g, st);
}

// tf32 variants of the LoRA GEMMs on fp32 operands: u = s x A^T (bf16 copy
// u' for the tail, fp32 copy for dB), dA = g^T x, dB = dy^T u.
soup_status lora_down_tf32(const float* x, int T, int K, const float* A32, int rows, float s, uint16_t* u,
                           float* u32, int64_t ldT, cudaStream_t st, const SplitWS& sw, uint16_t* ulo = nullptr) {
  GemmDesc g;
  g.tf32 = true;
  g.M = T; g.N = rows; g.K = K;
  g.A = Mat{x, T, K, K};
  g.b_mode = B_TMA_K;
  g.B = Mat{A32, rows, K, K};
  g.out_kind = OUT_BF16_T; g.out = u; g.out2 = u32; g.ldo = ldT; g.alpha = s;
  g.out_lo = ulo;
  use_split(g, sw);
  return gemm(g, st);
}


soup_status lora_dB_tf32(const float* dy, int64_t ld, int T, int n, const float* u32, int r, int64_t ldT, float* dB,
                         cudaStream_t st, const SplitWS& sw) {
  GemmDesc g;
  g.tf32 = true;
  g.M = n; g.N = r; g.K = T;
  g.a_major = A_MN;
  g.A = Mat{dy, T, n, ld};
  g.b_mode = B_TMA_K;
  g.B = Mat{u32, r, T, ldT};
  g.out_kind = OUT_F32; g.out = dB; g.ldo = r;
  use_split(g, sw);
  return gemm(g, st);
}

soup_status lora_dA_tf32(const float* x, int T, int K, const float* g32, int rows, int64_t ldT, float* dA,
                         cudaStream_t st, const SplitWS& sw) {
  GemmDesc g;
  g.tf32 = true;
  g.M = K; g.N = rows; g.K = T;
  g.a_major = A_MN;
  g.A = Mat{x, T, K, K};
  g.b_mode = B_TMA_K;
  g.B = Mat{g32, rows, T, ldT};
  g.out_kind = OUT_F32_T; g.out = dA; g.ldo = K;
  use_split(g, sw);
  return gemm(g, st);
}

// dx = dy W (+ g' A); with swiglu_I > 0 the epilogue turns dL/d(act) into
// [dL/dg | dL/du] (bf16, [T, 2I]) using the fp16 g | u saved by the forward.
soup_status proj_bwd(const soup_weight* W, const uint16_t* dy, int T, const uint16_t* gt, int64_t ldT, int g_rows,
                     const uint16_t* Al, bool on, uint16_t* dx, cudaStream_t st, int out_kind = OUT_BF16,
                     int swiglu_I = 0, uint16_t* aux16 = nullptr, const unsigned int* scale_amax = nullptr,
                     const uint16_t* dy_lo = nullptr, uint16_t* out_lo = nullptr, Scratch sk = Scratch()) {
  GemmDesc g;
  g.sk_scratch = sk.p; g.sk_scratch_bytes = sk.bytes;
  g.scale_amax = scale_amax;
  g.out_lo = out_lo;
  if (dy_lo) g.A_lo = Mat{dy_lo, T, W->out_features, W->out_features};
  g.M = T; g.N = (int)W->in_features; g.K = (int)W->out_features;
  g.A = Mat{dy, T, W->out_features, W->out_features};
  set_weight_bwd(g, W);
  if (on) {
    g.tail_ksteps = g_rows / 16;
    g.tailA = Mat{gt, g_rows, T, ldT};
    g.tailB = Mat{Al, g_rows, W->in_features, W->in_features};
  }
  g.out_kind = out_kind; g.out = dx; g.ldo = W->in_features;
  if (swiglu_I > 0) {
    g.epi = EPI_SWIGLU_BWD;
    g.swiglu_I = swiglu_I;
    g.aux16 = aux16;
    g.ld_aux = 2 * (int64_t)swiglu_I;
    g.ldo = 2 * (int64_t)swiglu_I;
  }
  return gemm(g, st);
}

// Forward through the layer.  save: also produce what only the backward
// reads (fp16 g | u for the SwiGLU backward, the fp16 attention output for
// D, q|k|v from the hi + lo x1 pair); want_out: run the final down GEMM
// (the recompute inside the backward does not need its output).  The
// forward fields go to `fb` (FIELD), scratch to `base`.
// keep (forward pass only): also compute q|k|v with the hi + lo A pair and
// leave them (fp16, [T, qkv_w]) in `keep` for the backward; kept (recompute
// only): q|k|v of this layer kept by the forward pass, whose GEMM is skipped.
// The backward's side stream: the LoRA-factor gradients (dA, dB) feed only
// the optimiser, so they run on a second stream of the device beside the
// dx chain (on CTAs the big GEMMs' last rounds leave free), joined at the end
// of the layer.  One stream and six fork / join events per device, created
// once, again for a new CUDA context.
struct SideStream {
  void* ctx = nullptr;
  cudaStream_t st = nullptr;
  cudaEvent_t ev[11] = {};  // 0-4, 7-10: chain steps the side stream waits for; 5, 6: side-stream milestones
  std::mutex issue;  // held while one layer call issues its work: calls from
                     // several threads then share the side stream in turn
};
SideStream g_side[64];
std::mutex g_side_mu;

soup_status side_stream(SideStream** out) {
  int dev = 0;
  SOUP_CUDA_TRY(cudaGetDevice(&dev));
  SOUP_CHECK(dev >= 0 && dev < 64, SOUP_ERR_INVALID_ARG, "device %d out of range", dev);
  void* ctx = current_context();
  std::lock_guard<std::mutex> lk(g_side_mu);
  SideStream& s = g_side[dev];
  if (s.st == nullptr || ctx == nullptr || s.ctx != ctx) {
    SOUP_CUDA_TRY(cudaStreamCreateWithFlags(&s.st, cudaStreamNonBlocking));
    for (auto& e : s.ev) SOUP_CUDA_TRY(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
    s.ctx = ctx;
  }
  *out = &s;
  return SOUP_OK;
}

// The backward's recompute may hand LoRA down-projections that only the
// LoRA-factor gradients read (u_qkv of a layer whose q|k|v were kept: no
// q|k|v GEMM consumes it; u_down: the down product is not recomputed) to the
// side stream, after an event on the chain marks their input ready.
struct RecomputeSide {
  SideStream* side = nullptr;
  SplitWS sw{nullptr, 0};
};

soup_status forward(const soup_layer_weights* W, const soup_layer_lora* L, const soup_layer_cfg* c, const Dims& m,
                    const WS& ws, char* base, char* fb, const uint16_t* h_in, uint16_t* h_out, bool on, bool save,
                    bool want_out, cudaStream_t st, uint16_t* keep = nullptr, const uint16_t* kept = nullptr,
                    const RecomputeSide& rs = RecomputeSide()) {
  const int T = m.T, r = m.r;
  const SplitWS SW{PF(splitk), ws.splitk_bytes};
  // the backward's d_gu residual field is unused during a forward pass or
  // recompute: the big GEMMs' split last round keeps its partials there
  const Scratch SK{base + ws.d_gu_lo, (size_t)T * 2 * m.I * 2};
  // the RoPE table, with adapters on in the same launch as the fp32 copies of
  // the three A factors (tf32 operands)
  if (on) {
    PrepJobs pj;
    pj.njobs = 4;
    pj.job[0].in = L->A_qkv; pj.job[0].out = PF(A32); pj.job[0].rows = 3 * r; pj.job[0].cols = m.H;
    pj.job[1].in = L->A_o; pj.job[1].out = PF(Ao32); pj.job[1].rows = r; pj.job[1].cols = m.o_in;
    pj.job[2].in = L->A_gu; pj.job[2].out = PF(Agu32); pj.job[2].rows = 2 * r; pj.job[2].cols = m.H;
    PrepJob& rp = pj.job[3];
    rp.kind = PREP_ROPE; rp.out = PF(cosb); rp.out2 = PF(sinb); rp.N = m.S; rp.r = m.d / 2;
    rp.theta = (double)c->theta;
    SOUP_TRY(lora_prep(pj, st));
  } else {
    SOUP_TRY(rope_table(m.S, m.d, (double)c->theta, PF(cosb), PF(sinb), st));
  }
  const bool precise_qkv = (save && !kept) || keep;  // q|k|v from the hi + lo x1 pair
  SOUP_TRY(rmsnorm_fwd(h_in, nullptr, W->norm1, T, m.H, c->eps, P(x1), PF(rinv1), st, on ? PF(x1_32) : nullptr,
                       precise_qkv ? P(x1_lo) : nullptr));
  if (on) {
    // q/k/v adapters: u from the fp32 normalised input (tf32 tensor cores); the
    // tail consumes its bf16 copy, the dB GEMM its fp32 copy
    if (kept && rs.side) {
      SOUP_CUDA_TRY(cudaEventRecord(rs.side->ev[9], st));
      SOUP_CUDA_TRY(cudaStreamWaitEvent(rs.side->st, rs.side->ev[9], 0));
      SOUP_TRY(lora_down_tf32(PF(x1_32), T, m.H, PF(A32), 3 * r, m.s, P(u_qkv), PF(u32), m.ldT, rs.side->st, rs.sw));
    } else {
      SOUP_TRY(lora_down_tf32(PF(x1_32), T, m.H, PF(A32), 3 * r, m.s, P(u_qkv), PF(u32), m.ldT, st, SW));
    }
  }
  {
    const int se[3] = {m.Hq * m.d, (m.Hq + m.Hkv) * m.d, m.qkv_w};
    const int sr[3] = {0, r, 2 * r};
    ProjOpts o;
    o.out_kind = OUT_F16;  // q, k, v feed only the attention kernels
    o.rope_cols = (m.Hq + m.Hkv) * m.d;
    o.rope_S = m.S; o.rope_cos = PF(cosb); o.rope_sin = PF(sinb);
    o.rope_prefix = m.Lp; o.rope_group = m.G;
    // for the backward, q/k/v from an fp32-accurate x1 (hi + lo parts): the
    // attention backward amplifies the bf16 rounding of x1 into the q/k/v
    // adapter gradients
    if (precise_qkv) o.x_lo = P(x1_lo);
    o.sk = SK;
    if (!kept)
      SOUP_TRY(proj_fwd(&W->qkv, P(x1), T, P(u_qkv), m.ldT, 3 * r, L ? L->B_qkv : nullptr, r, 3, se, sr, on,
                        keep ? keep : P(qkv), st, o));
  }
  const uint16_t* qkvp = kept ? kept : (keep ? keep : P(qkv));
  SOUP_TRY(attention_fwd(qkvp, m.qkv_w, m.B, m.S, m.Hq, m.Hkv, P(attn), PF(lse), st,
                         save ? P(attn16) : nullptr, on ? PF(attn32) : nullptr, m.G, m.Lp));
  if (on) {
    SOUP_TRY(lora_down_tf32(PF(attn32), T, m.o_in, PF(Ao32), r, m.s, P(u_o), PF(uo32), m.ldT, st, SW));
  }
  {
    const int se[1] = {m.H};
    const int sr[1] = {0};
    ProjOpts o;
    o.out_kind = OUT_F32;  // h2 = h + o kept in fp32
    o.resid = h_in;
    o.sk = SK;
    SOUP_TRY(proj_fwd(&W->o, P(attn), T, P(u_o), m.ldT, r, L ? L->B_o : nullptr, r, 1, se, sr, on,
                      reinterpret_cast<uint16_t*>(PF(h2)), st, o));
  }
  SOUP_TRY(rmsnorm_fwd(nullptr, PF(h2), W->norm2, T, m.H, c->eps, P(x2), PF(rinv2), st, on ? PF(x2_32) : nullptr));
  if (on) {
    // u_gu from the unrounded x2 (tf32), with its rounding residual for dB
    SOUP_TRY(lora_down_tf32(PF(x2_32), T, m.H, PF(Agu32), 2 * r, m.s, P(u_gu), nullptr, m.ldT, st, SW, P(u_gu_lo)));
  }
  {
    const int se[1] = {2 * m.I};
    const int sr[1] = {0};
    ProjOpts o;
    o.swiglu_I = m.I;
    o.aux16 = save ? P(gu16) : nullptr;  // g | u are needed only by the backward
    o.sk = SK;
    SOUP_TRY(proj_fwd(&W->gate_up, P(x2), T, P(u_gu), m.ldT, 2 * r, L ? L->B_gu : nullptr, r, 1, se, sr, on,
                      P(act), st, o));
  }
  if (on) {
    if (!want_out && rs.side) {
      SOUP_CUDA_TRY(cudaEventRecord(rs.side->ev[10], st));
      SOUP_CUDA_TRY(cudaStreamWaitEvent(rs.side->st, rs.side->ev[10], 0));
      SOUP_TRY(lora_down(P(act), T, m.I, L->A_down, r, m.s, P(u_d), m.ldT, rs.side->st, rs.sw, PF(u_d32)));
    } else {
      SOUP_TRY(lora_down(P(act), T, m.I, L->A_down, r, m.s, P(u_d), m.ldT, st, SW, PF(u_d32)));
    }
  }
  if (want_out) {
    const int se[1] = {m.H};
    const int sr[1] = {0};
    ProjOpts o;
    o.resid_f32 = PF(h2);
    o.sk = SK;
    SOUP_TRY(proj_fwd(&W->down, P(act), T, P(u_d), m.ldT, r, L ? L->B_down : nullptr, r, 1, se, sr, on, h_out, st,
                      o));
  }
  return SOUP_OK;
}

}  // namespace
}  // namespace soup

using namespace soup;

extern "C" size_t soup_decoder_layer_workspace(const soup_layer_cfg* cfg, int64_t batch, int64_t seq) {
  Dims m;
  if (make_dims(cfg, batch, seq, &m) != SOUP_OK) return 0;
  return layout(m).total;
}

extern "C" size_t soup_decoder_layer_saved_bytes(const soup_layer_cfg* cfg, int64_t batch, int64_t seq) {
  Dims m;
  if (make_dims(cfg, batch, seq, &m) != SOUP_OK) return 0;
  return layout(m).fwd_bytes;
}

extern "C" size_t soup_decoder_layer_keep_bytes(const soup_layer_cfg* cfg, int64_t batch, int64_t seq) {
  Dims m;
  if (make_dims(cfg, batch, seq, &m) != SOUP_OK) return 0;
  return (size_t)m.T * m.qkv_w * 2;
}

static soup_status layer_fwd_impl(const soup_layer_weights* W, const soup_layer_lora* lora, const soup_layer_cfg* cfg,
                                  const uint16_t* h_in, int64_t batch, int64_t seq, uint16_t* h_out,
                                  int32_t adapters_on, void* workspace, size_t workspace_bytes, void* stream,
                                  uint16_t* keep, void* saved = nullptr) {
  Dims m;
  SOUP_TRY(make_dims(cfg, batch, seq, &m));
  SOUP_TRY(check_weights(W, m));
  SOUP_CHECK(h_in && h_out && workspace, SOUP_ERR_INVALID_ARG, "soup_decoder_layer_fwd: null pointer");
  SOUP_CHECK(!adapters_on || (lora && lora->A_qkv && lora->B_qkv && lora->A_o && lora->B_o && lora->A_gu &&
                              lora->B_gu && lora->A_down && lora->B_down),
             SOUP_ERR_INVALID_ARG, "soup_decoder_layer_fwd: adapters on but LoRA factors missing");
  const WS ws = layout(m);
  SOUP_CHECK(workspace_bytes >= ws.total && soup_aligned(workspace, 256), SOUP_ERR_INVALID_ARG,
             "soup_decoder_layer_fwd: workspace %zu < %zu bytes or misaligned", workspace_bytes, ws.total);
  char* base = static_cast<char*>(workspace);
  if (saved) {  // everything the backward reads stays in the layer's saved region
    SOUP_CHECK(soup_aligned(saved, 256), SOUP_ERR_ALIGN, "soup_decoder_layer_fwd_save: saved region not 256-byte aligned");
    return forward(W, lora, cfg, m, ws, base, static_cast<char*>(saved), h_in, h_out, adapters_on != 0, true, true,
                   static_cast<cudaStream_t>(stream));
  }
  return forward(W, lora, cfg, m, ws, base, base, h_in, h_out, adapters_on != 0, false, true,
                 static_cast<cudaStream_t>(stream), keep);
}

extern "C" soup_status soup_decoder_layer_fwd(const soup_layer_weights* W, const soup_layer_lora* lora,
                                              const soup_layer_cfg* cfg, const uint16_t* h_in, int64_t batch,
                                              int64_t seq, uint16_t* h_out, int32_t adapters_on, void* workspace,
                                              size_t workspace_bytes, void* stream) {
  return layer_fwd_impl(W, lora, cfg, h_in, batch, seq, h_out, adapters_on, workspace, workspace_bytes, stream,
                        nullptr);
}

extern "C" soup_status soup_decoder_layer_fwd_keep(const soup_layer_weights* W, const soup_layer_lora* lora,
                                                   const soup_layer_cfg* cfg, const uint16_t* h_in, int64_t batch,
                                                   int64_t seq, uint16_t* h_out, int32_t adapters_on,
                                                   uint16_t* qkv_keep, void* workspace, size_t workspace_bytes,
                                                   void* stream) {
  SOUP_CHECK(qkv_keep && soup_aligned(qkv_keep, 16), SOUP_ERR_INVALID_ARG,
             "soup_decoder_layer_fwd_keep: null or misaligned keep buffer");
  return layer_fwd_impl(W, lora, cfg, h_in, batch, seq, h_out, adapters_on, workspace, workspace_bytes, stream,
                        qkv_keep);
}

extern "C" soup_status soup_decoder_layer_fwd_save(const soup_layer_weights* W, const soup_layer_lora* lora,
                                                   const soup_layer_cfg* cfg, const uint16_t* h_in, int64_t batch,
                                                   int64_t seq, uint16_t* h_out, int32_t adapters_on, void* saved,
                                                   void* workspace, size_t workspace_bytes, void* stream) {
  SOUP_CHECK(saved, SOUP_ERR_INVALID_ARG, "soup_decoder_layer_fwd_save: null saved region");
  return layer_fwd_impl(W, lora, cfg, h_in, batch, seq, h_out, adapters_on, workspace, workspace_bytes, stream,
                        nullptr, saved);
}

static soup_status layer_bwd_impl(const soup_layer_weights* W, const soup_layer_lora* L, const soup_layer_cfg* cfg,
                                  const uint16_t* h_in, const float* dh_out, int64_t batch, int64_t seq, float* dh_in,
                                  const soup_layer_grads* G, int32_t adapters_on, void* workspace,
                                  size_t workspace_bytes, void* stream, const uint16_t* kept,
                                  const void* saved = nullptr) {
  Dims m;
  SOUP_TRY(make_dims(cfg, batch, seq, &m));
  SOUP_TRY(check_weights(W, m));
  SOUP_CHECK(h_in && dh_out && dh_in && workspace, SOUP_ERR_INVALID_ARG, "soup_decoder_layer_bwd: null pointer");
  const bool on = adapters_on != 0;
  SOUP_CHECK(!on || (L && G && G->dA_qkv && G->dB_qkv && G->dA_o && G->dB_o && G->dA_gu && G->dB_gu && G->dA_down &&
                     G->dB_down),
             SOUP_ERR_INVALID_ARG, "soup_decoder_layer_bwd: adapters on but LoRA factors/grads missing");
  const WS ws = layout(m);
  SOUP_CHECK(workspace_bytes >= ws.total && soup_aligned(workspace, 256), SOUP_ERR_INVALID_ARG,
             "soup_decoder_layer_bwd: workspace %zu < %zu bytes or misaligned", workspace_bytes, ws.total);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* base = static_cast<char*>(workspace);
  char* fb = base;  // forward fields (below: or the saved region)
  const SplitWS SW{PF(splitk), ws.splitk_bytes};
  const int T = m.T, r = m.r, H = m.H, I = m.I;
  const int64_t ldT = m.ldT;

  // LoRA-factor gradients go to the side stream: each group waits (event)
  // for the main-stream step that produced its inputs.  The MLP groups are
  // issued after the next big GEMM; dB_o and dB_qkv, which need only dy and
  // the forward's u, start beside the skinny g GEMM before the o / q|k|v
  // dx product (measured: 2 ms less per 32-layer backward than issuing them
  // after it), so less of the side stream is left when the layer joins it.
  // The recompute hands it the down-projections only they read.
  SideStream* side = nullptr;
  if (on) SOUP_TRY(side_stream(&side));
  std::unique_lock<std::mutex> issue_lock;
  if (side) issue_lock = std::unique_lock<std::mutex>(side->issue);

  // forward fields: recomputed into the workspace (the layer was read again
  // for this), or what a saved forward pass left in the layer's own region
  if (saved) {
    SOUP_CHECK(soup_aligned(saved, 256), SOUP_ERR_ALIGN, "soup_decoder_layer_bwd_saved: saved region not 256-byte aligned");
    fb = static_cast<char*>(const_cast<void*>(saved));
  } else {
    RecomputeSide rs;
    rs.side = side;
    rs.sw = SplitWS{PF(splitk2), ws.splitk_bytes};
    SOUP_TRY(forward(W, L, cfg, m, ws, base, fb, h_in, nullptr, on, true, false, st, nullptr, kept, rs));
  }
  const uint16_t* qkvp = kept ? kept : P(qkv);

  // ---- B factors for the g GEMMs, one launch: B_down^T and B_o^T (fp32),
  // block-diagonal transposes of B_qkv (fp32, 3 segments) and B_gu (bf16,
  // 2 segments), so each g = s dy B is one GEMM over all its segments; the
  // same launch converts dh_out to bf16 (the down product's A operand) and
  // zeroes gamax (max |dh2| of the norm2 backward accumulates into it)
  unsigned int* gamax = reinterpret_cast<unsigned int*>(base + ws.gamax);
  if (on) {
    PrepJobs pj;
    pj.njobs = 5;
    pj.zero_word = gamax;
    PrepJob& cv = pj.job[4];
    cv.kind = PREP_F32_TO_BF16; cv.in32 = dh_out; cv.out = P(dh_b); cv.n = (long long)T * H;
    PrepJob& a = pj.job[0];
    a.kind = PREP_BLOCKDIAG_T; a.in = L->B_down; a.out = PF(Bt_down32); a.N = H; a.r = r;
    PrepJob& b = pj.job[1];
    b.kind = PREP_BLOCKDIAG_T; b.in = L->B_o; b.out = PF(Bt_o32); b.N = H; b.r = r;
    PrepJob& c = pj.job[2];
    c.kind = PREP_BLOCKDIAG_T; c.in = L->B_qkv; c.out = PF(Bbd_qkv32); c.N = m.qkv_w; c.r = r; c.nseg = 3;
    c.seg_end[0] = m.Hq * m.d; c.seg_end[1] = (m.Hq + m.Hkv) * m.d; c.seg_end[2] = m.qkv_w;
    PrepJob& d = pj.job[3];
    d.kind = PREP_BLOCKDIAG_T; d.out_bf16 = 1; d.in = L->B_gu; d.out = P(Bbd_gu); d.N = 2 * I; d.r = r; d.nseg = 2;
    d.seg_end[0] = I; d.seg_end[1] = 2 * I;
    SOUP_TRY(lora_prep(pj, st));
  }

  const SplitWS SW2{PF(splitk2), ws.splitk_bytes};
  cudaStream_t s2 = side ? side->st : st;
  auto mark = [&](int e) -> soup_status {  // the side stream may consume what st has produced so far
    SOUP_CUDA_TRY(cudaEventRecord(side->ev[e], st));
    return SOUP_OK;
  };
  auto after = [&](int e) -> soup_status {
    SOUP_CUDA_TRY(cudaStreamWaitEvent(s2, side->ev[e], 0));
    return SOUP_OK;
  };

  // ---- MLP block
  if (!on) SOUP_TRY(f32_to_bf16(dh_out, (size_t)T * H, P(dh_b), st, gamax));
  // LoRA gradients of the MLP: g_down from the fp32 dh (tf32), the others
  // from hi + lo (rounding residual) operand pairs, so no operand of a
  // LoRA-gradient GEMM carries more than the bf16 rounding of d_gu
  if (on) {
    SOUP_TRY(lora_g_prepared(dh_out, nullptr, H, T, H, PF(Bt_down32), r, m.s, true, P(g_d), nullptr, P(g_d_lo), ldT,
                             st, SW));
    SOUP_TRY(mark(0));
  }
  // d_gu = SwiGLU backward of (dh W_down + g' A_down), fused in the epilogue
  // split-round partials: in dx2 for the down product (it writes d_gu's
  // residual), then in that residual, which nothing reads after g_gu
  const Scratch SK_dx2{P(dx2), (size_t)T * H * 2}, SK_lo{P(d_gu_lo), (size_t)T * 2 * I * 2};
  SOUP_TRY(proj_bwd(&W->down, P(dh_b), T, P(g_d), ldT, r, on ? L->A_down : nullptr, on, P(d_gu), st, OUT_BF16, I,
                    P(gu16), nullptr, nullptr, on ? P(d_gu_lo) : nullptr, SK_dx2));
  if (on) {
    SOUP_TRY(mark(1));
    SOUP_TRY(after(0));
    SOUP_TRY(lora_dB_tf32(dh_out, H, T, H, PF(u_d32), r, ldT, G->dB_down, s2, SW2));
    // dh_in may alias dh_out: its writer (the norm1 backward) waits for this read
    SOUP_CUDA_TRY(cudaEventRecord(side->ev[6], s2));
    SOUP_TRY(lora_dA_dual(P(g_d), P(g_d_lo), r, ldT, P(act), T, I, G->dA_down, s2, SW2));
  }
  uint16_t* d_gu = P(d_gu);
  if (on) {  // g_gate | g_up in one GEMM (block-diagonal B_gu^T), d_gu hi + lo
    SOUP_TRY(lora_g_prepared(d_gu, P(d_gu_lo), 2 * I, T, 2 * I, P(Bbd_gu), 2 * r, m.s, false, P(g_gu), PF(g_gu32),
                             nullptr, ldT, st, SW));
    SOUP_TRY(mark(2));
  }
  SOUP_TRY(proj_bwd(&W->gate_up, d_gu, T, P(g_gu), ldT, 2 * r, on ? L->A_gu : nullptr, on, P(dx2), st, OUT_BF16, 0,
                    nullptr, nullptr, nullptr, nullptr, SK_lo));
  if (on) {
    SOUP_TRY(after(1));
    for (int sg = 0; sg < 2; ++sg)
      SOUP_TRY(lora_dB_dual(d_gu + (size_t)sg * I, 2 * I, T, I, P(u_gu) + (size_t)sg * r * ldT,
                            P(u_gu_lo) + (size_t)sg * r * ldT, r, ldT, G->dB_gu + (size_t)sg * I * r, s2, SW2));
    SOUP_TRY(after(2));
    SOUP_TRY(lora_dA_tf32(PF(x2_32), T, H, PF(g_gu32), 2 * r, ldT, G->dA_gu, s2, SW2));
  }
  SOUP_TRY(rmsnorm_bwd(nullptr, PF(h2), W->norm2, PF(rinv2), P(dx2), dh_out, T, H, PF(dh2), P(dh2_b), st, gamax,
                       P(dh2_lo)));

  // ---- attention block
  if (on) {
    SOUP_TRY(mark(8));
    SOUP_TRY(after(8));
    SOUP_TRY(lora_dB_tf32(PF(dh2), H, T, H, PF(uo32), r, ldT, G->dB_o, s2, SW2));
    SOUP_TRY(lora_g_prepared(PF(dh2), nullptr, H, T, H, PF(Bt_o32), r, m.s, true, P(g_o), PF(go32), nullptr, ldT, st,
                             SW));
    SOUP_TRY(mark(3));
  }
  // dO for the attention backward: from the fp32-accurate dh2 (hi + lo parts),
  // stored fp16 scaled by a power of two derived from max |dh2|
  SOUP_TRY(proj_bwd(&W->o, P(dh2_b), T, P(g_o), ldT, r, on ? L->A_o : nullptr, on, P(d_attn), st, OUT_F16, 0,
                    nullptr, gamax, P(dh2_lo), nullptr, SK_lo));
  if (on) {
    SOUP_TRY(after(3));
    SOUP_TRY(lora_dA_tf32(PF(attn32), T, m.o_in, PF(go32), r, ldT, G->dA_o, s2, SW2));
  }
  SOUP_TRY(attn_rowdot(P(d_attn), P(attn16), T, m.Hq, PF(D), st));
  // dq and dk leave the attention backward already rotated back (inverse RoPE in its epilogues)
  SOUP_TRY(attention_bwd(qkvp, m.qkv_w, m.B, m.S, m.Hq, m.Hkv, P(d_attn), PF(lse), PF(D), P(d_qkv), PF(cosb),
                         PF(sinb), gamax, st, on ? PF(dqkv32) : nullptr, m.G, m.Lp));
  const int seg_n[3] = {m.Hq * m.d, m.Hkv * m.d, m.Hkv * m.d};
  const int seg_c[3] = {0, m.Hq * m.d, (m.Hq + m.Hkv) * m.d};
  if (on) {
    SOUP_TRY(mark(7));
    SOUP_TRY(after(7));
    for (int sg = 0; sg < 3; ++sg)
      SOUP_TRY(lora_dB_tf32(PF(dqkv32) + seg_c[sg], m.qkv_w, T, seg_n[sg], PF(u32) + (size_t)sg * r * ldT, r, ldT,
                            G->dB_qkv + (size_t)seg_c[sg] * r, s2, SW2));
    // g_q | g_k | g_v in one GEMM (block-diagonal B_qkv^T)
    SOUP_TRY(lora_g_prepared(PF(dqkv32), nullptr, m.qkv_w, T, m.qkv_w, PF(Bbd_qkv32), 3 * r, m.s, true, P(g_qkv),
                             PF(g32), nullptr, ldT, st, SW));
    SOUP_TRY(mark(4));
  }
  SOUP_TRY(proj_bwd(&W->qkv, P(d_qkv), T, P(g_qkv), ldT, 3 * r, on ? L->A_qkv : nullptr, on, P(dx1), st, OUT_BF16, 0,
                    nullptr, nullptr, nullptr, nullptr, SK_lo));
  if (on) {
    SOUP_TRY(after(4));
    SOUP_TRY(lora_dA_tf32(PF(x1_32), T, H, PF(g32), 3 * r, ldT, G->dA_qkv, s2, SW2));
    // join: the layer's work is done on st only when the side stream's is
    SOUP_CUDA_TRY(cudaEventRecord(side->ev[5], s2));
  }
  if (on) SOUP_CUDA_TRY(cudaStreamWaitEvent(st, side->ev[6], 0));
  SOUP_TRY(rmsnorm_bwd(h_in, nullptr, W->norm1, PF(rinv1), P(dx1), PF(dh2), T, H, dh_in, nullptr, st));
  if (on) SOUP_CUDA_TRY(cudaStreamWaitEvent(st, side->ev[5], 0));
  return SOUP_OK;
}

namespace {
struct BlobPart {
  int64_t out, in;
};
}  // namespace

extern "C" size_t soup_layer_blob_bytes(const soup_layer_cfg* cfg, int32_t kind) {
  soup_layer_weights w;
  if (soup_layer_blob_views(cfg, kind, nullptr, &w) != SOUP_OK) return 0;
  // the last part is norm2 of `hidden` bf16 values
  return reinterpret_cast<size_t>(w.norm2) + align256((size_t)cfg->hidden * 2);
}

extern "C" soup_status soup_layer_blob_views(const soup_layer_cfg* cfg, int32_t kind, const void* base,
                                             soup_layer_weights* out) {
  SOUP_CHECK(cfg, SOUP_ERR_INVALID_ARG, "soup_layer_blob_views: null cfg");
  soup_layer_cfg one = *cfg;  // the blob does not depend on the token layout
  one.prefix_share = 0;
  one.prefix_len = 0;
  Dims m;
  SOUP_TRY(make_dims(&one, 1, 1, &m));
  SOUP_CHECK(out, SOUP_ERR_INVALID_ARG, "soup_layer_blob_views: null out");
  SOUP_CHECK(kind == SOUP_WEIGHT_NF4 || kind == SOUP_WEIGHT_BF16, SOUP_ERR_INVALID_ARG, "bad weight kind %d", kind);
  SOUP_CHECK(soup_aligned(base, 256), SOUP_ERR_ALIGN, "soup_layer_blob_views: base not 256-byte aligned");
  const char* b = static_cast<const char*>(base);
  size_t o = 0;
  const BlobPart parts[4] = {{m.qkv_w, m.H}, {m.H, m.o_in}, {2 * (int64_t)m.I, m.H}, {m.H, m.I}};
  soup_weight* dst[4] = {&out->qkv, &out->o, &out->gate_up, &out->down};
  for (int i = 0; i < 4; ++i) {
    soup_weight& w = *dst[i];
    memset(&w, 0, sizeof(w));
    w.kind = kind;
    w.out_features = parts[i].out;
    w.in_features = parts[i].in;
    const size_t n = (size_t)parts[i].out * parts[i].in;
    if (kind == SOUP_WEIGHT_NF4) {
      w.codes = reinterpret_cast<const uint8_t*>(b + o);
      o += align256(n / 2);
      w.absmax = reinterpret_cast<const float*>(b + o);
      o += align256(n / 64 * 4);
    } else {
      w.w = reinterpret_cast<const uint16_t*>(b + o);
      o += align256(n * 2);
    }
  }
  out->norm1 = reinterpret_cast<const uint16_t*>(b + o);
  o += align256((size_t)m.H * 2);
  out->norm2 = reinterpret_cast<const uint16_t*>(b + o);
  return SOUP_OK;
}

extern "C" soup_status soup_decoder_layer_bwd(const soup_layer_weights* W, const soup_layer_lora* L,
                                              const soup_layer_cfg* cfg, const uint16_t* h_in, const float* dh_out,
                                              int64_t batch, int64_t seq, float* dh_in,
                                              const soup_layer_grads* G, int32_t adapters_on, void* workspace,
                                              size_t workspace_bytes, void* stream) {
  return layer_bwd_impl(W, L, cfg, h_in, dh_out, batch, seq, dh_in, G, adapters_on, workspace, workspace_bytes,
                        stream, nullptr);
}

extern "C" soup_status soup_decoder_layer_bwd_kept(const soup_layer_weights* W, const soup_layer_lora* L,
                                                   const soup_layer_cfg* cfg, const uint16_t* h_in,
                                                   const float* dh_out, int64_t batch, int64_t seq, float* dh_in,
                                                   const soup_layer_grads* G, int32_t adapters_on,
                                                   const uint16_t* qkv_kept, void* workspace,
                                                   size_t workspace_bytes, void* stream) {
  SOUP_CHECK(qkv_kept && soup_aligned(qkv_kept, 16), SOUP_ERR_INVALID_ARG,
             "soup_decoder_layer_bwd_kept: null or misaligned kept buffer");
  return layer_bwd_impl(W, L, cfg, h_in, dh_out, batch, seq, dh_in, G, adapters_on, workspace, workspace_bytes,
                        stream, qkv_kept);
}

extern "C" soup_status soup_decoder_layer_bwd_saved(const soup_layer_weights* W, const soup_layer_lora* L,
                                                    const soup_layer_cfg* cfg, const uint16_t* h_in,
                                                    const float* dh_out, int64_t batch, int64_t seq, float* dh_in,
                                                    const soup_layer_grads* G, int32_t adapters_on, const void* saved,
                                                    void* workspace, size_t workspace_bytes, void* stream) {
  SOUP_CHECK(saved, SOUP_ERR_INVALID_ARG, "soup_decoder_layer_bwd_saved: null saved region");
  return layer_bwd_impl(W, L, cfg, h_in, dh_out, batch, seq, dh_in, G, adapters_on, workspace, workspace_bytes,
                        stream, nullptr, saved);
}
