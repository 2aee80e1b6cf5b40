// One LoRA-adapted projection over a frozen base (NF4 or bf16), forward and
// backward, built from the tcgen05 GEMM engine:
//
//   forward   u'  = bf16(s * x A^T)         -> u_save [r, ldT] (transposed)
//             y   = x W^T + u' B^T           (NF4 decode + LoRA tail fused)
//   backward  g'  = bf16(s * dy B)           -> workspace [r, ldT] (transposed)
//             dx  = dy W + g' A              (NF4 decode of W^T + LoRA tail fused)
//             dB  = dy^T u'^T ,  dA = g'^T x (fp32, one CTA per output tile,
//                                             fixed-order reduction over T)
// W gets no gradient: the pages' backward through a frozen layer needs only
// dL/dx = W^T dL/dy plus the adapter terms (Soup pages, "how layer streaming
// works").
#include <cuda_bf16.h>

#include <mutex>

#include "gemm.h"
#include "lora_internal.h"

namespace soup {
namespace {

__global__ void transpose_bf16_kernel(const uint16_t* __restrict__ in, int rows, int cols,
                                      uint16_t* __restrict__ out) {
  // in [rows, cols] -> out [cols, rows]
  __shared__ uint16_t tile[32][33];
  const int bx = blockIdx.x * 32, by = blockIdx.y * 32;
  for (int j = threadIdx.y; j < 32; j += blockDim.y) {
    const int r = by + j, c = bx + threadIdx.x;
    if (r < rows && c < cols) tile[j][threadIdx.x] = in[(size_t)r * cols + c];
  }
  __syncthreads();
  for (int j = threadIdx.y; j < 32; j += blockDim.y) {
    const int c = bx + j, r = by + threadIdx.x;
    if (r < rows && c < cols) out[(size_t)c * rows + r] = tile[threadIdx.x][j];
  }
}

}  // namespace

soup_status transpose_bf16(const uint16_t* in, int rows, int cols, uint16_t* out, cudaStream_t st) {
  dim3 grid((cols + 31) / 32, (rows + 31) / 32);
  transpose_bf16_kernel<<<grid, dim3(32, 8), 0, st>>>(in, rows, cols, out);
  SOUP_LAUNCH_CHECK();
  return SOUP_OK;
}

soup_status check_weight(const soup_weight* W, const char* fn) {
  SOUP_CHECK(W, SOUP_ERR_INVALID_ARG, "%s: null weight", fn);
  SOUP_CHECK(W->kind == SOUP_WEIGHT_NF4 || W->kind == SOUP_WEIGHT_BF16, SOUP_ERR_INVALID_ARG,
             "%s: unknown weight kind %d", fn, W->kind);
  SOUP_CHECK(W->out_features > 0 && W->in_features > 0 && W->in_features % 64 == 0 &&
                 W->out_features % 16 == 0 && W->out_features < (1 << 30) && W->in_features < (1 << 30),
             SOUP_ERR_SHAPE, "%s: W must be [out, in] with out %% 16 == 0 and in %% 64 == 0 (got %lld x %lld)",
             fn, (long long)W->out_features, (long long)W->in_features);
  if (W->kind == SOUP_WEIGHT_NF4) {
    SOUP_CHECK(W->codes && W->absmax, SOUP_ERR_INVALID_ARG, "%s: NF4 weight without codes/absmax", fn);
    SOUP_CHECK(soup_aligned(W->codes, 16) && soup_aligned(W->absmax, 4), SOUP_ERR_ALIGN,
               "%s: NF4 codes must be 16-byte aligned", fn);
  } else {
    SOUP_CHECK(W->w && soup_aligned(W->w, 16), SOUP_ERR_ALIGN, "%s: bf16 weight null or misaligned", fn);
  }
  return SOUP_OK;
}

// Shared by the layer: a projection's forward GEMM (x W^T + tail), with the
// tail description supplied by the caller.
void set_weight_fwd(GemmDesc& g, const soup_weight* W) {
  if (W->kind == SOUP_WEIGHT_NF4) {
    g.b_mode = B_NF4_K;
    g.codes = W->codes;
    g.absmax = W->absmax;
  } else {
    g.b_mode = B_TMA_K;
    g.B = Mat{W->w, W->out_features, W->in_features, W->in_features};
  }
}

void set_weight_bwd(GemmDesc& g, const soup_weight* W) {
  if (W->kind == SOUP_WEIGHT_NF4) {
    g.b_mode = B_NF4_MN;
    g.codes = W->codes;
    g.absmax = W->absmax;
  } else {
    g.b_mode = B_TMA_MN;
    g.B = Mat{W->w, W->out_features, W->in_features, W->in_features};
  }
}

}  // namespace soup

using namespace soup;

extern "C" soup_status soup_lora_linear_fwd(const soup_weight* W, const uint16_t* A, const uint16_t* B,
                                            int32_t r, float scale, const uint16_t* x, int64_t T,
                                            uint16_t* y, uint16_t* u_save, void* stream) {
  SOUP_TRY(check_weight(W, "soup_lora_linear_fwd"));
  SOUP_CHECK(A && B && x && y && u_save, SOUP_ERR_INVALID_ARG, "soup_lora_linear_fwd: null pointer");
  SOUP_CHECK(r >= 8 && r <= 64 && r % 8 == 0, SOUP_ERR_SHAPE, "soup_lora_linear_fwd: r=%d (need 8..64, %%8)", r);
  SOUP_CHECK(T >= 1 && T < (1 << 30), SOUP_ERR_SHAPE, "soup_lora_linear_fwd: T=%lld", (long long)T);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t in = W->in_features, out = W->out_features, ldT = round_up8(T);
  // u' = bf16(s * x A^T), stored transposed
  GemmDesc g1;
  g1.M = (int)T; g1.N = r; g1.K = (int)in;
  g1.A = Mat{x, T, in, in};
  g1.b_mode = B_TMA_K;
  g1.B = Mat{A, r, in, in};
  g1.out_kind = OUT_BF16_T; g1.out = u_save; g1.ldo = ldT; g1.alpha = scale;
  SOUP_TRY(gemm(g1, st));
  // y = x W^T + u' B^T
  GemmDesc g2;
  g2.M = (int)T; g2.N = (int)out; g2.K = (int)in;
  g2.A = Mat{x, T, in, in};
  set_weight_fwd(g2, W);
  g2.tail_ksteps = (r + 15) / 16;
  g2.tailA = Mat{u_save, r, T, ldT};
  g2.tailB = Mat{B, out, r, r};
  g2.out_kind = OUT_BF16; g2.out = y; g2.ldo = out;
  return gemm(g2, st);
}

extern "C" size_t soup_lora_linear_bwd_workspace(int64_t T, int32_t r, int64_t out_features) {
  if (T <= 0 || r <= 0 || out_features <= 0) return 0;
  return align256((size_t)r * out_features * 2) + align256((size_t)r * round_up8(T) * 2);
}

extern "C" soup_status soup_lora_linear_bwd(const soup_weight* W, const uint16_t* A, const uint16_t* B,
                                            int32_t r, float scale, const uint16_t* x,
                                            const uint16_t* u_save, const uint16_t* dy, int64_t T,
                                            uint16_t* dx, float* dA, float* dB, void* workspace,
                                            size_t workspace_bytes, void* stream) {
  SOUP_TRY(check_weight(W, "soup_lora_linear_bwd"));
  SOUP_CHECK(A && B && x && u_save && dy && dx && dA && dB && workspace, SOUP_ERR_INVALID_ARG,
             "soup_lora_linear_bwd: null pointer");
  SOUP_CHECK(r >= 8 && r <= 64 && r % 8 == 0, SOUP_ERR_SHAPE, "soup_lora_linear_bwd: r=%d", r);
  SOUP_CHECK(T >= 1 && T < (1 << 30), SOUP_ERR_SHAPE, "soup_lora_linear_bwd: T=%lld", (long long)T);
  const int64_t in = W->in_features, out = W->out_features, ldT = round_up8(T);
  SOUP_CHECK(workspace_bytes >= soup_lora_linear_bwd_workspace(T, r, out) && soup_aligned(workspace, 256),
             SOUP_ERR_INVALID_ARG, "soup_lora_linear_bwd: workspace too small or not 256-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint16_t* Bt = static_cast<uint16_t*>(workspace);
  uint16_t* gt = reinterpret_cast<uint16_t*>(static_cast<char*>(workspace) + align256((size_t)r * out * 2));
  SOUP_TRY(transpose_bf16(B, (int)out, r, Bt, st));
  // g' = bf16(s * dy B), transposed [r, ldT]
  GemmDesc g1;
  g1.M = (int)T; g1.N = r; g1.K = (int)out;
  g1.A = Mat{dy, T, out, out};
  g1.b_mode = B_TMA_K;
  g1.B = Mat{Bt, r, out, out};
  g1.out_kind = OUT_BF16_T; g1.out = gt; g1.ldo = ldT; g1.alpha = scale;
  SOUP_TRY(gemm(g1, st));
  // dx = dy W + g' A
  GemmDesc g2;
  g2.M = (int)T; g2.N = (int)in; g2.K = (int)out;
  g2.A = Mat{dy, T, out, out};
  set_weight_bwd(g2, W);
  g2.tail_ksteps = (r + 15) / 16;
  g2.tailA = Mat{gt, r, T, ldT};
  g2.tailB = Mat{A, r, in, in};
  g2.out_kind = OUT_BF16; g2.out = dx; g2.ldo = in;
  SOUP_TRY(gemm(g2, st));
  // dB = dy^T u'^T   [out, r]
  GemmDesc g3;
  g3.M = (int)out; g3.N = r; g3.K = (int)T;
  g3.a_major = A_MN;
  g3.A = Mat{dy, T, out, out};
  g3.b_mode = B_TMA_K;
  g3.B = Mat{u_save, r, T, ldT};
  g3.out_kind = OUT_F32; g3.out = dB; g3.ldo = r;
  SOUP_TRY(gemm(g3, st));
  // dA = g'^T x  computed as dA^T = x^T g' and stored transposed into [r, in]
  GemmDesc g4;
  g4.M = (int)in; g4.N = r; g4.K = (int)T;
  g4.a_major = A_MN;
  g4.A = Mat{x, T, in, in};
  g4.b_mode = B_TMA_K;
  g4.B = Mat{gt, r, T, ldT};
  g4.out_kind = OUT_F32_T; g4.out = dA; g4.ldo = in;
  return gemm(g4, st);
}

// ---------------------------------------------------------------------------
// Allocation-free variant of the LoRA linear backward.
//
// For callers that cannot allocate device memory when they run the backward
// (for example an integration whose device memory is entirely owned by
// another allocator's pool, or a latency-critical path where cudaMalloc,
// which may synchronise the device, is not allowed).  Its scratch (the
// transposed B and the g' = bf16(s dy B) buffer) lives in this file-scope
// array instead of a caller-provided workspace.  Every GPU that loads the
// library holds the array until the process exits.
#define SOUP_NOALLOC_SCRATCH_BYTES (8u << 20)
static __device__ __align__(256) uint8_t g_lora_noalloc_scratch[SOUP_NOALLOC_SCRATCH_BYTES];


extern "C" size_t soup_lora_linear_bwd_noalloc_max_scratch(void) { return SOUP_NOALLOC_SCRATCH_BYTES; }

extern "C" size_t soup_static_device_bytes(void) { return SOUP_NOALLOC_SCRATCH_BYTES + gemm_static_device_bytes(); }

extern "C" soup_status soup_lora_linear_bwd_noalloc(const soup_weight* W, const uint16_t* A, const uint16_t* B,
                                                    int32_t r, float scale, const uint16_t* x,
                                                    const uint16_t* u_save, const uint16_t* dy, int64_t T,
                                                    uint16_t* dx, float* dA, float* dB, void* stream) {
  SOUP_CHECK(W, SOUP_ERR_INVALID_ARG, "soup_lora_linear_bwd_noalloc: null weight");
  const size_t need = soup_lora_linear_bwd_workspace(T, r, W->out_features);
  SOUP_CHECK(need > 0, SOUP_ERR_SHAPE, "soup_lora_linear_bwd_noalloc: bad sizes (T=%lld r=%d out=%lld)",
             (long long)T, r, (long long)W->out_features);
  SOUP_CHECK(need <= SOUP_NOALLOC_SCRATCH_BYTES, SOUP_ERR_SHAPE,
             "soup_lora_linear_bwd_noalloc: T=%lld, r=%d, out=%lld need %zu bytes of scratch, more than the "
             "static maximum of %u bytes; use soup_lora_linear_bwd with a workspace",
             (long long)T, r, (long long)W->out_features, need, SOUP_NOALLOC_SCRATCH_BYTES);
  void* ws = nullptr;
  SOUP_TRY(static_symbol_address(SYM_NOALLOC_SCRATCH, reinterpret_cast<const void*>(g_lora_noalloc_scratch), &ws));
  // Every byte of the scratch that this call reads it first writes (the
  // transpose fills B^T, the GEMM fills g' for columns [0, T), the only ones
  // read), so nothing left by an earlier call needs clearing.
  return soup_lora_linear_bwd(W, A, B, r, scale, x, u_save, dy, T, dx, dA, dB, ws, SOUP_NOALLOC_SCRATCH_BYTES,
                              stream);
}
