#include <algorithm>
// Memory-bound kernels of the decoder layer: RMSNorm forward/backward, the
// RoPE angle table, the attention-backward row dot D = rowsum(dO * O), and
// dtype conversions.  (RoPE itself is applied in the QKV GEMM epilogue and in
// the attention-backward epilogues; SwiGLU in the gate|up and down GEMM
// epilogues.)  All accesses are 16-byte
// vectorised and coalesced; row reductions use warp shuffles.  Layouts are
// token-major: [T, features] with T = batch * seq.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "elementwise.h"

namespace soup {
namespace {

__device__ __forceinline__ float b2f(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }
__device__ __forceinline__ void unpack8(const uint4 v, float* f) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ uint4 pack8(const float* f) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    w[i] = *reinterpret_cast<uint32_t*>(&h);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Loads 8 consecutive elements of row `row` (chunk c8) from bf16 or fp32 storage.
__device__ __forceinline__ void load8(const uint16_t* xb, const float* xf, size_t off, float* f) {
  if (xf) {
    const float4 a = reinterpret_cast<const float4*>(xf + off)[0];
    const float4 b = reinterpret_cast<const float4*>(xf + off)[1];
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  } else {
    unpack8(*reinterpret_cast<const uint4*>(xb + off), f);
  }
}

// One warp per row; H % 256 == 0 so every lane owns H/256 chunks of 8.
__global__ void rmsnorm_fwd_kernel(const uint16_t* __restrict__ x, const float* __restrict__ xf,
                                   const uint16_t* __restrict__ w, int T, int H, float eps, uint16_t* __restrict__ y,
                                   float* __restrict__ rinv, float* __restrict__ y32, uint16_t* __restrict__ ylo) {
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= T) return;
  const size_t rb = (size_t)row * H;
  float ss = 0.f;
  const int nch = H / 256;
  for (int c = 0; c < nch; ++c) {
    float f[8];
    load8(x, xf, rb + (size_t)(c * 32 + lane) * 8, f);
#pragma unroll
    for (int i = 0; i < 8; ++i) ss += f[i] * f[i];
  }
  ss = warp_sum(ss);
  const float r = 1.0f / sqrtf(ss / (float)H + eps);
  if (lane == 0 && rinv) rinv[row] = r;
  const uint4* wr = reinterpret_cast<const uint4*>(w);
  uint4* yr = reinterpret_cast<uint4*>(y + rb);
  for (int c = 0; c < nch; ++c) {
    float f[8], g[8];
    load8(x, xf, rb + (size_t)(c * 32 + lane) * 8, f);
    unpack8(wr[c * 32 + lane], g);
#pragma unroll
    for (int i = 0; i < 8; ++i) f[i] = (f[i] * r) * g[i];
    const uint4 hi = pack8(f);
    yr[c * 32 + lane] = hi;
    if (ylo) {  // rounding residual: y = hi + lo to ~16 significant bits
      float fh[8], fl[8];
      unpack8(hi, fh);
#pragma unroll
      for (int i = 0; i < 8; ++i) fl[i] = f[i] - fh[i];
      reinterpret_cast<uint4*>(ylo + rb)[c * 32 + lane] = pack8(fl);
    }
    if (y32) {
      float4* o = reinterpret_cast<float4*>(y32 + rb + (size_t)(c * 32 + lane) * 8);
      o[0] = make_float4(f[0], f[1], f[2], f[3]);
      o[1] = make_float4(f[4], f[5], f[6], f[7]);
    }
  }
}

// dh = dres + rinv * (dy*w - xh * mean(dy*w*xh)),  xh = x * rinv
__global__ void rmsnorm_bwd_kernel(const uint16_t* __restrict__ x, const float* __restrict__ xf,
                                   const uint16_t* __restrict__ w, const float* __restrict__ rinv,
                                   const uint16_t* __restrict__ dy, const float* __restrict__ dyf,
                                   const float* __restrict__ dres, int T, int H, float* __restrict__ dh,
                                   uint16_t* __restrict__ dh_bf16, unsigned int* __restrict__ amax,
                                   uint16_t* __restrict__ dh_lo) {
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= T) return;
  const float r = rinv[row];
  const size_t rb = (size_t)row * H;
  const uint4* wr = reinterpret_cast<const uint4*>(w);
  const int nch = H / 256;
  float dot = 0.f;
  for (int c = 0; c < nch; ++c) {
    float a[8], b[8], g[8];
    load8(x, xf, rb + (size_t)(c * 32 + lane) * 8, a);
    load8(dy, dyf, rb + (size_t)(c * 32 + lane) * 8, b);
    unpack8(wr[c * 32 + lane], g);
#pragma unroll
    for (int i = 0; i < 8; ++i) dot += (b[i] * g[i]) * (a[i] * r);
  }
  dot = warp_sum(dot) / (float)H;
  float mx = 0.f;
  for (int c = 0; c < nch; ++c) {
    float a[8], b[8], g[8], o[8];
    load8(x, xf, rb + (size_t)(c * 32 + lane) * 8, a);
    load8(dy, dyf, rb + (size_t)(c * 32 + lane) * 8, b);
    unpack8(wr[c * 32 + lane], g);
    const size_t base = rb + (size_t)(c * 32 + lane) * 8;
    const float4 d0 = dres ? reinterpret_cast<const float4*>(dres + base)[0] : make_float4(0, 0, 0, 0);
    const float4 d1 = dres ? reinterpret_cast<const float4*>(dres + base)[1] : make_float4(0, 0, 0, 0);
    const float dr[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = dr[i] + r * (b[i] * g[i] - (a[i] * r) * dot);
    reinterpret_cast<float4*>(dh + base)[0] = make_float4(o[0], o[1], o[2], o[3]);
    reinterpret_cast<float4*>(dh + base)[1] = make_float4(o[4], o[5], o[6], o[7]);
    if (dh_bf16) {
      const uint4 hi = pack8(o);
      reinterpret_cast<uint4*>(dh_bf16 + base)[0] = hi;
      if (dh_lo) {
        float oh[8], ol[8];
        unpack8(hi, oh);
#pragma unroll
        for (int i = 0; i < 8; ++i) ol[i] = o[i] - oh[i];
        reinterpret_cast<uint4*>(dh_lo + base)[0] = pack8(ol);
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) mx = fmaxf(mx, fabsf(o[i]));
  }
  if (amax) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    // non-negative floats order like their bit patterns: an integer max is exact and order-independent
    if (lane == 0) atomicMax(amax, __float_as_uint(mx));
  }
}

// The same backward with one 128-thread CTA per row: every thread loads its
// (at most CPT) 8-element chunks of x, dy and dres once, up front, and keeps
// them in registers across the row reduction, so the row streams through
// memory once with all its loads in flight together.  H / 8 <= 128 * CPT.
template <int CPT>
__global__ void __launch_bounds__(128) rmsnorm_bwd_row_kernel(
    const uint16_t* __restrict__ x, const float* __restrict__ xf, const uint16_t* __restrict__ w,
    const float* __restrict__ rinv, const uint16_t* __restrict__ dy, const float* __restrict__ dyf,
    const float* __restrict__ dres, int T, int H, float* __restrict__ dh, uint16_t* __restrict__ dh_bf16,
    unsigned int* __restrict__ amax, uint16_t* __restrict__ dh_lo) {
  __shared__ float red_dot[4], red_max[4];
  const int row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int nc = H / 8;
  const size_t rb = (size_t)row * H;
  const float r = rinv[row];
  float a[CPT][8], b[CPT][8], d[CPT][8];
#pragma unroll
  for (int k = 0; k < CPT; ++k) {
    const int c = tid + k * 128;
    if (c < nc) {
      const size_t off = rb + (size_t)c * 8;
      load8(x, xf, off, a[k]);
      load8(dy, dyf, off, b[k]);
      if (dres) {
        const float4 d0 = reinterpret_cast<const float4*>(dres + off)[0];
        const float4 d1 = reinterpret_cast<const float4*>(dres + off)[1];
        d[k][0] = d0.x; d[k][1] = d0.y; d[k][2] = d0.z; d[k][3] = d0.w;
        d[k][4] = d1.x; d[k][5] = d1.y; d[k][6] = d1.z; d[k][7] = d1.w;
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) d[k][i] = 0.f;
      }
    }
  }
  const uint4* wr = reinterpret_cast<const uint4*>(w);
  float dot = 0.f;
#pragma unroll
  for (int k = 0; k < CPT; ++k) {
    const int c = tid + k * 128;
    if (c < nc) {
      float g[8];
      unpack8(wr[c], g);
#pragma unroll
      for (int i = 0; i < 8; ++i) dot += (b[k][i] * g[i]) * (a[k][i] * r);
    }
  }
  dot = warp_sum(dot);
  if (lane == 0) red_dot[wid] = dot;
  __syncthreads();
  dot = ((red_dot[0] + red_dot[1]) + (red_dot[2] + red_dot[3])) / (float)H;
  float mx = 0.f;
#pragma unroll
  for (int k = 0; k < CPT; ++k) {
    const int c = tid + k * 128;
    if (c < nc) {
      float g[8], o[8];
      unpack8(wr[c], g);
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = d[k][i] + r * (b[k][i] * g[i] - (a[k][i] * r) * dot);
      const size_t base = rb + (size_t)c * 8;
      reinterpret_cast<float4*>(dh + base)[0] = make_float4(o[0], o[1], o[2], o[3]);
      reinterpret_cast<float4*>(dh + base)[1] = make_float4(o[4], o[5], o[6], o[7]);
      if (dh_bf16) {
        const uint4 hi = pack8(o);
        reinterpret_cast<uint4*>(dh_bf16 + base)[0] = hi;
        if (dh_lo) {
          float oh[8], ol[8];
          unpack8(hi, oh);
#pragma unroll
          for (int i = 0; i < 8; ++i) ol[i] = o[i] - oh[i];
          reinterpret_cast<uint4*>(dh_lo + base)[0] = pack8(ol);
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) mx = fmaxf(mx, fabsf(o[i]));
    }
  }
  if (amax) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    if (lane == 0) red_max[wid] = mx;
    __syncthreads();
    // non-negative floats order like their bit patterns: an integer max is exact and order-independent
    if (tid == 0)
      atomicMax(amax, __float_as_uint(fmaxf(fmaxf(red_max[0], red_max[1]), fmaxf(red_max[2], red_max[3]))));
  }
}

// cos/sin of pos * theta^(-2i/d), computed in fp64 and rounded to fp32.
__global__ void rope_table_kernel(int S, int half, double theta, float* __restrict__ cosb, float* __restrict__ sinb) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= S * half) return;
  const int pos = i / half, j = i % half;
  const double inv = pow(theta, -(2.0 * j) / (2.0 * half));
  const double a = (double)pos * inv;
  cosb[i] = (float)cos(a);
  sinb[i] = (float)sin(a);
}

// D[h, t] = sum_d dO[t, h*128 + d] * O[t, h*128 + d]; one warp per (t, h).
__global__ void attn_rowdot_kernel(const uint16_t* __restrict__ dO, const uint16_t* __restrict__ O, int T, int Hq,
                                   float* __restrict__ D) {
  const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= T * Hq) return;
  const int t = gw / Hq, h = gw % Hq;
  const size_t off = (size_t)t * Hq * 128 + h * 128 + lane * 4;
  const uint2 a = *reinterpret_cast<const uint2*>(dO + off);
  const uint2 b = *reinterpret_cast<const uint2*>(O + off);
  // dO and O are both fp16 here (O: the attention forward's fp16 copy)
  const float2 d01 = __half22float2(*reinterpret_cast<const __half2*>(&a.x));
  const float2 d23 = __half22float2(*reinterpret_cast<const __half2*>(&a.y));
  const float2 o01 = __half22float2(*reinterpret_cast<const __half2*>(&b.x));
  const float2 o23 = __half22float2(*reinterpret_cast<const __half2*>(&b.y));
  float s = d01.x * o01.x + d01.y * o01.y + d23.x * o23.x + d23.y * o23.y;
  s = warp_sum(s);
  if (lane == 0) D[(size_t)h * T + t] = s;
}

__global__ void f32_to_bf16_kernel(const float* __restrict__ in, size_t n, uint16_t* __restrict__ out,
                                   unsigned int* __restrict__ zero_word) {
  if (zero_word && blockIdx.x == 0 && threadIdx.x == 0) *zero_word = 0u;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n / 8; i += (size_t)gridDim.x * blockDim.x) {
    const float4 a = reinterpret_cast<const float4*>(in)[2 * i];
    const float4 b = reinterpret_cast<const float4*>(in)[2 * i + 1];
    const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    reinterpret_cast<uint4*>(out)[i] = pack8(f);
  }
}

__global__ void bf16_to_f32_kernel(const uint16_t* __restrict__ in, size_t n, float* __restrict__ out) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n / 8; i += (size_t)gridDim.x * blockDim.x) {
    float f[8];
    unpack8(reinterpret_cast<const uint4*>(in)[i], f);
    reinterpret_cast<float4*>(out)[2 * i] = make_float4(f[0], f[1], f[2], f[3]);
    reinterpret_cast<float4*>(out)[2 * i + 1] = make_float4(f[4], f[5], f[6], f[7]);
  }
}

// in [rows, cols] bf16 -> out [cols, rows] fp32 (exact)
__global__ void transpose_bf16_f32_kernel(const uint16_t* __restrict__ in, int rows, int cols,
                                          float* __restrict__ out) {
  __shared__ float tile[32][33];
  const int bx = blockIdx.x * 32, by = blockIdx.y * 32;
  for (int j = threadIdx.y; j < 32; j += blockDim.y) {
    const int r = by + j, c = bx + threadIdx.x;
    if (r < rows && c < cols) tile[j][threadIdx.x] = b2f(in[(size_t)r * cols + c]);
  }
  __syncthreads();
  for (int j = threadIdx.y; j < 32; j += blockDim.y) {
    const int c = bx + j, r = by + threadIdx.x;
    if (r < rows && c < cols) out[(size_t)c * rows + r] = tile[threadIdx.x][j];
  }
}

unsigned grid_for(size_t work, int threads) {
  size_t g = (work + threads - 1) / threads;
  const size_t cap = (size_t)sm_count() * 16;
  return (unsigned)(g < 1 ? 1 : (g > cap ? cap : g));
}

}  // namespace

soup_status rmsnorm_fwd(const uint16_t* x, const float* x_f32, const uint16_t* w, int T, int H, float eps,
                        uint16_t* y, float* rinv, cudaStream_t st, float* y32, uint16_t* ylo) {
  SOUP_CHECK(H % 256 == 0, SOUP_ERR_SHAPE, "rmsnorm: hidden %d not a multiple of 256", H);
  const double n = (double)T * H;
  profile_begin(st, GC_RMSNORM, 0.0,
                n * (x_f32 ? 4 : 2) + H * 2.0 + n * 2 + T * 4.0 + (y32 ? n * 4 : 0.0) + (ylo ? n * 2 : 0.0));
  rmsnorm_fwd_kernel<<<(T + 7) / 8, 256, 0, st>>>(x, x_f32, w, T, H, eps, y, rinv, y32, ylo);
  SOUP_LAUNCH_CHECK();
  profile_end(st);
  return SOUP_OK;
}

soup_status rmsnorm_bwd(const uint16_t* x, const float* x_f32, const uint16_t* w, const float* rinv,
                        const uint16_t* dy, const float* dres, int T, int H, float* dh, uint16_t* dh_bf16,
                        cudaStream_t st, unsigned int* amax, uint16_t* dh_lo) {
  SOUP_CHECK(H % 256 == 0, SOUP_ERR_SHAPE, "rmsnorm: hidden %d not a multiple of 256", H);
  const double n = (double)T * H;
  profile_begin(st, GC_RMSNORM, 0.0,
                n * (x_f32 ? 4 : 2) + H * 2.0 + T * 4.0 + n * 2 + (dres ? n * 4 : 0.0) + n * 4 +
                    (dh_bf16 ? n * 2 : 0.0) + (dh_lo ? n * 2 : 0.0));
  if (H <= 128 * 8 * 4)
    rmsnorm_bwd_row_kernel<4><<<T, 128, 0, st>>>(x, x_f32, w, rinv, dy, nullptr, dres, T, H, dh, dh_bf16, amax, dh_lo);
  else
    rmsnorm_bwd_kernel<<<(T + 7) / 8, 256, 0, st>>>(x, x_f32, w, rinv, dy, nullptr, dres, T, H, dh, dh_bf16, amax,
                                                    dh_lo);
  SOUP_LAUNCH_CHECK();
  profile_end(st);
  return SOUP_OK;
}

soup_status rmsnorm_bwd_f32dy(const uint16_t* x, const uint16_t* w, const float* rinv, const float* dy, int T, int H,
                              float* dh, cudaStream_t st) {
  SOUP_CHECK(H % 256 == 0, SOUP_ERR_SHAPE, "rmsnorm: hidden %d not a multiple of 256", H);
  if (H <= 128 * 8 * 4)
    rmsnorm_bwd_row_kernel<4><<<T, 128, 0, st>>>(x, nullptr, w, rinv, nullptr, dy, nullptr, T, H, dh, nullptr, nullptr,
                                                 nullptr);
  else
    rmsnorm_bwd_kernel<<<(T + 7) / 8, 256, 0, st>>>(x, nullptr, w, rinv, nullptr, dy, nullptr, T, H, dh, nullptr,
                                                    nullptr, nullptr);
  SOUP_LAUNCH_CHECK();
  return SOUP_OK;
}

soup_status transpose_bf16_f32(const uint16_t* in, int rows, int cols, float* out, cudaStream_t st) {
  dim3 grid((cols + 31) / 32, (rows + 31) / 32);
  transpose_bf16_f32_kernel<<<grid, dim3(32, 8), 0, st>>>(in, rows, cols, out);
  SOUP_LAUNCH_CHECK();
  return SOUP_OK;
}

soup_status rope_table(int S, int head_dim, double theta, float* cosb, float* sinb, cudaStream_t st) {
  const int n = S * head_dim / 2;
  profile_begin(st, GC_ELEM, 0.0, n * 8.0);
  rope_table_kernel<<<(n + 255) / 256, 256, 0, st>>>(S, head_dim / 2, theta, cosb, sinb);
  SOUP_LAUNCH_CHECK();
  profile_end(st);
  return SOUP_OK;
}

soup_status attn_rowdot(const uint16_t* dO, const uint16_t* O, int T, int Hq, float* D, cudaStream_t st) {
  profile_begin(st, GC_ELEM, 0.0, (double)T * Hq * (128 * 2 * 2 + 4));
  attn_rowdot_kernel<<<(T * Hq + 7) / 8, 256, 0, st>>>(dO, O, T, Hq, D);
  SOUP_LAUNCH_CHECK();
  profile_end(st);
  return SOUP_OK;
}

soup_status f32_to_bf16(const float* in, size_t n, uint16_t* out, cudaStream_t st, unsigned int* zero_word) {
  SOUP_CHECK(n % 8 == 0, SOUP_ERR_SHAPE, "f32_to_bf16: n %% 8");
  profile_begin(st, GC_ELEM, 0.0, n * 6.0);
  f32_to_bf16_kernel<<<grid_for(n / 8, 256), 256, 0, st>>>(in, n, out, zero_word);
  SOUP_LAUNCH_CHECK();
  profile_end(st);
  return SOUP_OK;
}

soup_status bf16_to_f32(const uint16_t* in, size_t n, float* out, cudaStream_t st) {
  SOUP_CHECK(n % 8 == 0, SOUP_ERR_SHAPE, "bf16_to_f32: n %% 8");
  bf16_to_f32_kernel<<<grid_for(n / 8, 256), 256, 0, st>>>(in, n, out);
  SOUP_LAUNCH_CHECK();
  return SOUP_OK;
}


namespace {
struct PrepArgs {
  PrepJobs jobs;
  long long start[6];  // prefix sums of the jobs' unit counts
};

__global__ void lora_prep_kernel(const PrepArgs a) {
  if (a.jobs.zero_word && blockIdx.x == 0 && threadIdx.x == 0) *a.jobs.zero_word = 0u;
  const long long total = a.start[a.jobs.njobs];
  for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    int k = 0;
    while (k + 1 < a.jobs.njobs && idx >= a.start[k + 1]) ++k;
    const PrepJob& J = a.jobs.job[k];
    const long long i = idx - a.start[k];
    if (J.kind == PREP_COPY_F32) {
      static_cast<float*>(J.out)[i] = b2f(J.in[i]);
    } else if (J.kind == PREP_F32_TO_BF16) {  // unit i: elements 8i .. 8i+7
      const float4 x0 = reinterpret_cast<const float4*>(J.in32)[2 * i];
      const float4 x1 = reinterpret_cast<const float4*>(J.in32)[2 * i + 1];
      const float f[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
      reinterpret_cast<uint4*>(J.out)[i] = pack8(f);
    } else if (J.kind == PREP_ROPE) {
      const int pos = (int)(i / J.r), j = (int)(i % J.r);
      const double inv = pow(J.theta, -(2.0 * j) / (2.0 * J.r));
      const double ang = (double)pos * inv;
      static_cast<float*>(J.out)[i] = (float)cos(ang);
      static_cast<float*>(J.out2)[i] = (float)sin(ang);
    } else {
      // 32-bit division: a job has fewer than 2^31 elements (checked on the host)
      const unsigned R = (unsigned)i / (unsigned)J.N, n = (unsigned)i - R * (unsigned)J.N;
      const int s = (int)R / J.r, j = (int)R % J.r;
      int seg = 0;
      while (seg + 1 < J.nseg && (int)n >= J.seg_end[seg]) ++seg;
      const uint16_t v = seg == s ? J.in[(size_t)n * J.r + j] : static_cast<uint16_t>(0);
      if (J.out_bf16) static_cast<uint16_t*>(J.out)[i] = v;
      else static_cast<float*>(J.out)[i] = b2f(v);
    }
  }
}
}  // namespace

soup_status lora_prep(const PrepJobs& jobs, cudaStream_t st) {
  SOUP_CHECK(jobs.njobs >= 1 && jobs.njobs <= 5, SOUP_ERR_INVALID_ARG, "lora_prep: %d jobs", jobs.njobs);
  PrepArgs a;
  a.jobs = jobs;
  a.start[0] = 0;
  for (int k = 0; k < jobs.njobs; ++k) {
    const PrepJob& J = jobs.job[k];
    long long n = 0;
    bool ok = false;
    switch (J.kind) {
      case PREP_COPY_F32:
        n = (long long)J.rows * J.cols;
        ok = J.in && J.out;
        break;
      case PREP_BLOCKDIAG_T:
        n = (long long)J.nseg * J.r * J.N;
        ok = J.in && J.out && J.r > 0 && J.nseg >= 1 && J.nseg <= 3;
        break;
      case PREP_F32_TO_BF16:
        n = J.n / 8;
        ok = J.in32 && J.out && J.n % 8 == 0 && soup_aligned(J.in32, 16) && soup_aligned(J.out, 16);
        break;
      case PREP_ROPE:
        n = (long long)J.N * J.r;
        ok = J.out && J.out2 && J.r > 0 && J.theta > 0.0;
        break;
    }
    SOUP_CHECK(ok && n > 0 && n < (1LL << 31), SOUP_ERR_SHAPE, "lora_prep: bad job %d", k);
    a.start[k + 1] = a.start[k] + n;
  }
  const long long total = a.start[jobs.njobs];
  const int blocks = (int)std::min<long long>((total + 255) / 256, (long long)sm_count() * 8);
  double bytes = 0;  // each output element written once, each input element read once
  for (int k = 0; k < jobs.njobs; ++k) {
    const PrepJob& J = jobs.job[k];
    const double outs = (double)(a.start[k + 1] - a.start[k]);
    if (J.kind == PREP_COPY_F32) bytes += outs * 6.0;
    else if (J.kind == PREP_F32_TO_BF16) bytes += outs * 48.0;  // 8 x (4 in + 2 out)
    else if (J.kind == PREP_ROPE) bytes += outs * 8.0;
    else bytes += outs * (J.out_bf16 ? 2 : 4) + (double)J.N * J.r * 2;
  }
  profile_begin(st, GC_ELEM, 0.0, bytes);
  lora_prep_kernel<<<blocks, 256, 0, st>>>(a);
  SOUP_LAUNCH_CHECK();
  profile_end(st);
  return SOUP_OK;
}

}  // namespace soup
