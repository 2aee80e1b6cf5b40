// NF4 block quantisation (shard building) and standalone dequantisation.
//
// Quantise: one warp per 64-element block, two elements per lane.  absmax is
// a warp max-reduction of |w| (exact); n = w / absmax is an IEEE
// correctly-rounded fp32 division; the code is the number of codebook
// midpoints strictly below n.  Midpoints (c_i + c_{i+1}) / 2 are exact in
// fp64; comparing the fp32 n against each midpoint rounded toward -inf to
// fp32 gives the same answer as comparing against the exact midpoint, so a
// value exactly on a midpoint goes to the lower code (nearest code, ties to
// the lower index).
//
// Dequantise: value = RNE_bf16(fp32(c_code * absmax)); one thread per 8
// codes, 16-byte stores.  The fused GEMM decodes with the same arithmetic, so
// its B operand is bit-identical to this kernel's output.
#include <cuda_bf16.h>

#include "nf4_codebook.cuh"
#include "soup_internal.h"

namespace soup {
namespace {

__global__ void nf4_quantize_kernel(const float* __restrict__ W, int64_t n_blocks, int64_t blocks_per_row,
                                    int64_t in, uint8_t* __restrict__ codes, float* __restrict__ absmax,
                                    int32_t* flag) {
  __shared__ float thr[15];
  if (threadIdx.x < 15) {
    const double lo = (double)__uint_as_float(nf4_code_bits(threadIdx.x));
    const double hi = (double)__uint_as_float(nf4_code_bits(threadIdx.x + 1));
    thr[threadIdx.x] = __double2float_rd(0.5 * (lo + hi));
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t warps_total = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t b = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); b < n_blocks; b += warps_total) {
    const int64_t row = b / blocks_per_row, col_blk = b % blocks_per_row;
    const float* src = W + row * in + col_blk * 64;
    const float2 w = reinterpret_cast<const float2*>(src)[lane];
    const bool finite = isfinite(w.x) && isfinite(w.y);
    if (!finite) atomicOr(flag, 1);
    float m = fmaxf(fabsf(w.x), fabsf(w.y));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    uint32_t c0 = 7, c1 = 7;
    if (m > 0.f) {
      const float n0 = __fdiv_rn(w.x, m), n1 = __fdiv_rn(w.y, m);
      c0 = 0; c1 = 0;
#pragma unroll
      for (int j = 0; j < 15; ++j) {
        c0 += (n0 > thr[j]) ? 1u : 0u;
        c1 += (n1 > thr[j]) ? 1u : 0u;
      }
    }
    codes[row * (in / 2) + col_blk * 32 + lane] = static_cast<uint8_t>((c0 << 4) | c1);
    if (lane == 0) absmax[b] = m;
  }
}

__global__ void nf4_dequant_kernel(const uint32_t* __restrict__ codes, const float* __restrict__ absmax,
                                   int64_t n_words, uint4* __restrict__ out) {
  __shared__ float cb[16];
  if (threadIdx.x < 16) cb[threadIdx.x] = __uint_as_float(nf4_code_bits(threadIdx.x));
  __syncthreads();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_words; i += (int64_t)gridDim.x * blockDim.x) {
    const uint32_t w = codes[i];
    const float am = absmax[i >> 3];  // 8 words (64 elements) per block
    uint32_t o[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const float f0 = cb[(w >> (8 * p + 4)) & 15u] * am;
      const float f1 = cb[(w >> (8 * p)) & 15u] * am;
      __nv_bfloat162 v = __floats2bfloat162_rn(f0, f1);
      o[p] = *reinterpret_cast<uint32_t*>(&v);
    }
    out[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace
}  // namespace soup

extern "C" soup_status soup_nf4_quantize(const float* W, int64_t out, int64_t in, uint8_t* codes,
                                         float* absmax, int32_t* flag_dev, void* stream) {
  using namespace soup;
  SOUP_CHECK(W && codes && absmax && flag_dev, SOUP_ERR_INVALID_ARG, "soup_nf4_quantize: null pointer");
  SOUP_CHECK(out > 0 && in > 0 && in % 64 == 0, SOUP_ERR_SHAPE,
             "soup_nf4_quantize: need out > 0 and in a positive multiple of 64 (out=%lld in=%lld)",
             (long long)out, (long long)in);
  SOUP_CHECK(soup_aligned(W, 8) && soup_aligned(absmax, 4) && soup_aligned(flag_dev, 4), SOUP_ERR_ALIGN,
             "soup_nf4_quantize: misaligned pointer");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SOUP_CUDA_TRY(cudaMemsetAsync(flag_dev, 0, sizeof(int32_t), st));
  const int64_t n_blocks = out * (in / 64);
  const int threads = 256;
  int64_t grid = (n_blocks + 7) / 8;
  const int64_t cap = (int64_t)sm_count() * 16;
  if (grid > cap) grid = cap;
  nf4_quantize_kernel<<<(unsigned)grid, threads, 0, st>>>(W, n_blocks, in / 64, in, codes, absmax, flag_dev);
  SOUP_LAUNCH_CHECK();
  int32_t flag = 0;
  SOUP_CUDA_TRY(cudaMemcpyAsync(&flag, flag_dev, sizeof(int32_t), cudaMemcpyDeviceToHost, st));
  SOUP_CUDA_TRY(cudaStreamSynchronize(st));
  if (flag) return fail(SOUP_ERR_NONFINITE, "soup_nf4_quantize: non-finite weight");
  return SOUP_OK;
}

extern "C" soup_status soup_nf4_dequant(const uint8_t* codes, const float* absmax, int64_t out, int64_t in,
                                        uint16_t* W_bf16, void* stream) {
  using namespace soup;
  SOUP_CHECK(codes && absmax && W_bf16, SOUP_ERR_INVALID_ARG, "soup_nf4_dequant: null pointer");
  SOUP_CHECK(out > 0 && in > 0 && in % 64 == 0, SOUP_ERR_SHAPE,
             "soup_nf4_dequant: need in a positive multiple of 64");
  SOUP_CHECK(soup_aligned(codes, 4) && soup_aligned(W_bf16, 16) && soup_aligned(absmax, 4), SOUP_ERR_ALIGN,
             "soup_nf4_dequant: codes must be 4-byte and W 16-byte aligned");
  const int64_t n_words = out * in / 8;
  int64_t grid = (n_words + 255) / 256;
  const int64_t cap = (int64_t)sm_count() * 32;
  if (grid > cap) grid = cap;
  nf4_dequant_kernel<<<(unsigned)grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const uint32_t*>(codes), absmax, n_words, reinterpret_cast<uint4*>(W_bf16));
  SOUP_LAUNCH_CHECK();
  return SOUP_OK;
}
