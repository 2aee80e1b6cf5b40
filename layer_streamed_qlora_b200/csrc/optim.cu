// AdamW step over the resident LoRA adapters.
//
// The Soup pages ("how layer streaming works") keep the adapters, their
// gradients and the optimiser state in device memory for the whole run; only
// the frozen base streams.  The update is AdamW: Adam with decoupled weight
// decay (Loshchilov & Hutter, "Decoupled Weight Decay Regularization", ICLR
// 2019), with the decay folded into the learning rate as PyTorch does:
//
//   g     = grad_scale * grad
//   theta = theta * (1 - lr * weight_decay)
//   m     = beta1 * m + (1 - beta1) * g
//   v     = beta2 * v + (1 - beta2) * g^2
//   theta = theta - (lr / (1 - beta1^t)) * m / (sqrt(v) / sqrt(1 - beta2^t) + eps)
//
// One fp32 master copy of every adapter parameter is updated; its
// round-to-nearest-even bf16 copy (what the GEMMs read) is rewritten in the
// same pass, and the gradient is cleared for the next step's backward, which
// accumulates.  The pass is bound by HBM: per parameter it reads theta, grad,
// m and v (16 bytes) and writes theta, m, v, grad (16 bytes) and the bf16
// copy (2 bytes).  Each thread moves four parameters per iteration with
// 16-byte accesses; the grid is a multiple of the SM count.
#include <cmath>

#include <cuda_bf16.h>

#include "soup_internal.h"

namespace soup {
namespace {

struct AdamWArgs {
  float decay;         // 1 - lr * weight_decay
  float beta1, one_minus_beta1;
  float beta2, one_minus_beta2;
  float step_size;     // lr / (1 - beta1^t)
  float inv_sqrt_bc2;  // 1 / sqrt(1 - beta2^t)
  float eps;
  float grad_scale;
  int zero_grad;
};

__device__ __forceinline__ bool nonfinite(float x) {
  return (__float_as_uint(x) & 0x7f800000u) == 0x7f800000u;
}

__device__ __forceinline__ float adamw_one(const AdamWArgs& a, float p, float g_raw, float& m, float& v,
                                           bool& bad) {
  bad |= nonfinite(g_raw);
  const float g = g_raw * a.grad_scale;
  p = p * a.decay;
  m = a.beta1 * m + a.one_minus_beta1 * g;
  v = a.beta2 * v + a.one_minus_beta2 * (g * g);
  const float denom = sqrtf(v) * a.inv_sqrt_bc2 + a.eps;
  return p - a.step_size * (m / denom);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&b);
}

// n4 = n / 4 vector groups; the last n % 4 parameters are handled by the
// first threads of block 0.
__global__ void __launch_bounds__(256) adamw_kernel(float4* __restrict__ theta, uint2* __restrict__ theta_bf16,
                                                    float4* __restrict__ grad, float4* __restrict__ m,
                                                    float4* __restrict__ v, int64_t n4, int64_t n, AdamWArgs a,
                                                    int32_t* __restrict__ nonfinite_flag) {
  bool bad = false;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 p = theta[i], g = grad[i], mm = m[i], vv = v[i];
    p.x = adamw_one(a, p.x, g.x, mm.x, vv.x, bad);
    p.y = adamw_one(a, p.y, g.y, mm.y, vv.y, bad);
    p.z = adamw_one(a, p.z, g.z, mm.z, vv.z, bad);
    p.w = adamw_one(a, p.w, g.w, mm.w, vv.w, bad);
    theta[i] = p;
    m[i] = mm;
    v[i] = vv;
    if (a.zero_grad) grad[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (theta_bf16) theta_bf16[i] = make_uint2(pack_bf16x2(p.x, p.y), pack_bf16x2(p.z, p.w));
  }
  if (blockIdx.x == 0) {
    const int64_t j = n4 * 4 + threadIdx.x;
    if (j < n) {
      float* th = reinterpret_cast<float*>(theta);
      float* gr = reinterpret_cast<float*>(grad);
      float* ms = reinterpret_cast<float*>(m);
      float* vs = reinterpret_cast<float*>(v);
      float mj = ms[j], vj = vs[j];
      const float p = adamw_one(a, th[j], gr[j], mj, vj, bad);
      th[j] = p;
      ms[j] = mj;
      vs[j] = vj;
      if (a.zero_grad) gr[j] = 0.f;
      if (theta_bf16) reinterpret_cast<__nv_bfloat16*>(theta_bf16)[j] = __float2bfloat16_rn(p);
    }
  }
  if (bad && nonfinite_flag) *nonfinite_flag = 1;
}

}  // namespace
}  // namespace soup

extern "C" soup_status soup_adamw_step(float* theta, uint16_t* theta_bf16, float* grad, float* m, float* v,
                                       int64_t n, float lr, float beta1, float beta2, float eps,
                                       float weight_decay, float grad_scale, int64_t t, int32_t zero_grad,
                                       int32_t* nonfinite_dev, void* stream) {
  using namespace soup;
  SOUP_CHECK(n >= 0, SOUP_ERR_SHAPE, "soup_adamw_step: n must be >= 0");
  SOUP_CHECK(t >= 1, SOUP_ERR_INVALID_ARG, "soup_adamw_step: the step index t starts at 1");
  SOUP_CHECK(beta1 >= 0.f && beta1 < 1.f && beta2 >= 0.f && beta2 < 1.f && eps > 0.f && lr >= 0.f &&
                 weight_decay >= 0.f,
             SOUP_ERR_INVALID_ARG, "soup_adamw_step: need 0 <= beta < 1, eps > 0, lr >= 0, weight_decay >= 0");
  if (n == 0) return SOUP_OK;
  SOUP_CHECK(theta && grad && m && v, SOUP_ERR_INVALID_ARG, "soup_adamw_step: null pointer");
  SOUP_CHECK(soup_aligned(theta, 16) && soup_aligned(grad, 16) && soup_aligned(m, 16) && soup_aligned(v, 16) &&
                 (!theta_bf16 || soup_aligned(theta_bf16, 8)),
             SOUP_ERR_ALIGN, "soup_adamw_step: theta, grad, m, v must be 16-byte and theta_bf16 8-byte aligned");
  // bias corrections in double on the host
  const double bc1 = 1.0 - std::pow((double)beta1, (double)t);
  const double bc2 = 1.0 - std::pow((double)beta2, (double)t);
  AdamWArgs a;
  a.decay = (float)(1.0 - (double)lr * (double)weight_decay);
  a.beta1 = beta1;
  a.one_minus_beta1 = (float)(1.0 - (double)beta1);
  a.beta2 = beta2;
  a.one_minus_beta2 = (float)(1.0 - (double)beta2);
  a.step_size = (float)((double)lr / bc1);
  a.inv_sqrt_bc2 = (float)(1.0 / std::sqrt(bc2));
  a.eps = eps;
  a.grad_scale = grad_scale;
  a.zero_grad = zero_grad ? 1 : 0;
  const int64_t n4 = n / 4;
  int64_t blocks = (n4 + 255) / 256;
  const int64_t cap = (int64_t)sm_count() * 8;  // 8 resident 256-thread blocks per SM
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;  // the scalar tail runs in block 0
  // algorithmic bytes: theta, g, m, v read (16 B); theta, m, v written (12 B),
  // g cleared (4 B) and the bf16 copy (2 B) when asked
  profile_begin(static_cast<cudaStream_t>(stream), GC_ADAMW, 0.0,
                (double)n * (28.0 + (zero_grad ? 4.0 : 0.0) + (theta_bf16 ? 2.0 : 0.0)));
  adamw_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<float4*>(theta), reinterpret_cast<uint2*>(theta_bf16), reinterpret_cast<float4*>(grad),
      reinterpret_cast<float4*>(m), reinterpret_cast<float4*>(v), n4, n, a, nonfinite_dev);
  SOUP_LAUNCH_CHECK();
  profile_end(static_cast<cudaStream_t>(stream));
  return SOUP_OK;
}
