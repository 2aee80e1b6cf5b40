// Vocab-side kernels of the streamed step: token-embedding gather from the
// vocab slot, final RMSNorm + lm_head + next-token log-probabilities computed
// `chunk` tokens at a time (the pages' `stream_loss_chunk`: the output head
// and the loss are evaluated N tokens at a time so the [tokens, vocab] logits
// never exist in full), the gradient back to the last hidden state, the
// cross-entropy reduction and the DPO loss with its per-token coefficients.
#include <cuda_bf16.h>

#include "elementwise.h"
#include "gemm.h"
#include "lora_internal.h"

namespace soup {
namespace {

// one warp per token: h[t] = E[ids[t]]
__global__ void embed_kernel(const uint16_t* __restrict__ E, int64_t V, int H, const int32_t* __restrict__ ids,
                             int T, uint16_t* __restrict__ h, int* err) {
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  const int id = ids[t];
  uint4* dst = reinterpret_cast<uint4*>(h + (size_t)t * H);
  if (id < 0 || id >= V) {
    if (lane == 0) atomicOr(err, 2);
    for (int c = lane; c < H / 8; c += 32) dst[c] = make_uint4(0, 0, 0, 0);
    return;
  }
  const uint4* src = reinterpret_cast<const uint4*>(E + (size_t)id * H);
  for (int c = lane; c < H / 8; c += 32) dst[c] = src[c];
}

__device__ __forceinline__ float block_reduce(float v, bool is_max, float* sh) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float w = __shfl_xor_sync(0xffffffffu, v, o);
    v = is_max ? fmaxf(v, w) : v + w;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  __syncthreads();
  if (lane == 0) sh[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = lane < nw ? sh[lane] : (is_max ? -INFINITY : 0.f);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float w = __shfl_xor_sync(0xffffffffu, v, o);
      v = is_max ? fmaxf(v, w) : v + w;
    }
    if (lane == 0) sh[0] = v;
  }
  __syncthreads();
  return sh[0];
}

// One CTA per token row of the chunk: log-softmax at the label, and (when
// coef is given) dlogits = coef * (onehot(label) - softmax) in bf16.
__global__ void __launch_bounds__(1024) ce_rows_kernel(const float* __restrict__ logits, int64_t V,
                                                       const int32_t* __restrict__ ids, int t0, int S,
                                                       const float* __restrict__ coef, float* __restrict__ logp,
                                                       uint16_t* __restrict__ dlogits) {
  __shared__ float sh[32];
  const int i = blockIdx.x;
  const int t = t0 + i;
  const int b = t / S, s = t % S;
  const bool has_label = s < S - 1;
  const int label = has_label ? ids[t + 1] : -1;
  const float* row = logits + (size_t)i * V;
  // one pass for the row's maximum and its sum of exponentials: each thread
  // keeps a running maximum and rescales its partial sum when it grows, then
  // the block combines the (maximum, sum) pairs (V % 8 == 0: float4 loads)
  float tm = -INFINITY, ts = 0.f;
  const float4* row4 = reinterpret_cast<const float4*>(row);
  for (int64_t j = threadIdx.x; j < V / 4; j += blockDim.x) {
    const float4 x = row4[j];
    const float mx = fmaxf(fmaxf(x.x, x.y), fmaxf(x.z, x.w));
    const float mn = fmaxf(tm, mx);
    ts = ts * expf(tm - mn) + (expf(x.x - mn) + expf(x.y - mn)) + (expf(x.z - mn) + expf(x.w - mn));
    tm = mn;
  }
  const float m = block_reduce(tm, true, sh);
  float sum = block_reduce(tm == -INFINITY ? 0.f : ts * expf(tm - m), false, sh);
  const float lse = m + logf(sum);
  const bool label_ok = has_label && label >= 0 && label < V;
  if (threadIdx.x == 0 && has_label) logp[(size_t)b * (S - 1) + s] = label_ok ? row[label] - lse : 0.f;
  if (dlogits) {
    const float c = (coef && label_ok) ? coef[(size_t)b * (S - 1) + s] : 0.f;
    uint16_t* drow = dlogits + (size_t)i * V;
    const float inv = 1.0f / sum;
    for (int64_t j = threadIdx.x; j < V / 4; j += blockDim.x) {
      const float4 x = row4[j];
      const float xs[4] = {x.x, x.y, x.z, x.w};
      uint32_t w[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int64_t j0 = 4 * j + 2 * e;
        const float g0 = c * ((j0 == label ? 1.f : 0.f) - expf(xs[2 * e] - m) * inv);
        const float g1 = c * ((j0 + 1 == label ? 1.f : 0.f) - expf(xs[2 * e + 1] - m) * inv);
        __nv_bfloat162 hv = __floats2bfloat162_rn(g0, g1);
        w[e] = *reinterpret_cast<uint32_t*>(&hv);
      }
      reinterpret_cast<uint2*>(drow)[j] = make_uint2(w[0], w[1]);
    }
  }
}

// Mean next-token cross-entropy: loss = -sum(logp) / count (one CTA).
__global__ void ce_mean_kernel(const float* __restrict__ logp, int64_t n, float* __restrict__ loss) {
  __shared__ float sh[32];
  float s = 0.f;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) s += logp[i];
  s = block_reduce(s, false, sh);
  if (threadIdx.x == 0) *loss = -s / (float)n;
}

__global__ void fill_kernel(float* __restrict__ p, int64_t n, float v) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    p[i] = v;
}

// DPO: rows 2p (chosen) / 2p+1 (rejected).  seq[r] = sum of logp over the
// continuation positions (target index s+1 >= prompt_len).
//   z_p = beta * ((pi_c - ref_c) - (pi_r - ref_r)),  L = mean_p softplus(-z_p)
//   dL/dpi_c = -beta * sigmoid(-z_p) / P,  dL/dpi_r = +beta * sigmoid(-z_p) / P
// coef[r, s] = dL/dpi_row(r) on continuation positions, 0 on prompt positions.
__global__ void dpo_kernel(const float* __restrict__ lp_pol, const float* __restrict__ lp_ref, int pairs, int S,
                           int prompt_len, float beta, float* __restrict__ loss, float* __restrict__ seq_out,
                           float* __restrict__ coef) {
  extern __shared__ float sh[];  // [2*pairs] policy sums, [2*pairs] reference sums
  const int rows = 2 * pairs;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  for (int r = warp; r < 2 * rows; r += nw) {
    const float* lp = (r < rows) ? lp_pol + (size_t)r * (S - 1) : lp_ref + (size_t)(r - rows) * (S - 1);
    float s = 0.f;
    for (int j = lane; j < S - 1; j += 32)
      if (j + 1 >= prompt_len) s += lp[j];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) sh[r] = s;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float L = 0.f;
    for (int p = 0; p < pairs; ++p) {
      const float z = beta * ((sh[2 * p] - sh[rows + 2 * p]) - (sh[2 * p + 1] - sh[rows + 2 * p + 1]));
      L += (z > 0.f) ? log1pf(expf(-z)) : (-z + log1pf(expf(z)));
    }
    *loss = L / (float)pairs;
  }
  if (seq_out)
    for (int r = threadIdx.x; r < 2 * rows; r += blockDim.x) seq_out[r] = sh[r];
  for (int64_t i = threadIdx.x; i < (int64_t)rows * (S - 1); i += blockDim.x) {
    const int r = (int)(i / (S - 1)), j = (int)(i % (S - 1));
    const int p = r >> 1;
    const float z = beta * ((sh[2 * p] - sh[rows + 2 * p]) - (sh[2 * p + 1] - sh[rows + 2 * p + 1]));
    const float sig = 1.0f / (1.0f + expf(z));  // sigmoid(-z)
    const float d = beta * sig / (float)pairs;
    coef[i] = (j + 1 >= prompt_len) ? ((r & 1) ? d : -d) : 0.f;
  }
}

struct HeadWS {
  size_t xn, rinv, logits, dlogits, dxn, splitk, splitk_bytes, total;
};

HeadWS head_layout(int64_t V, int64_t H, int64_t T, int chunk) {
  HeadWS w;
  size_t o = 0;
  auto take = [&](size_t b) {
    size_t at = o;
    o += align256(b);
    return at;
  };
  w.xn = take((size_t)T * H * 2);
  w.rinv = take((size_t)T * 4);
  w.logits = take((size_t)chunk * V * 4);
  w.dlogits = take((size_t)chunk * V * 2);
  w.dxn = take((size_t)T * H * 4);
  // dxn = dlogits E has K = V but only (chunk/256)·(H/256) output tiles of
  // the CTA-pair engine: scratch for the fp32 partials of its K slices
  w.splitk_bytes = (size_t)6 * chunk * H * 4;
  w.splitk = take(w.splitk_bytes);
  w.total = o;
  return w;
}

}  // namespace
}  // namespace soup

using namespace soup;

extern "C" soup_status soup_embed(const uint16_t* E, int64_t V, int64_t H, const int32_t* ids, int64_t T, uint16_t* h,
                                  void* stream) {
  SOUP_CHECK(E && ids && h, SOUP_ERR_INVALID_ARG, "soup_embed: null pointer");
  SOUP_CHECK(V > 0 && H > 0 && H % 8 == 0 && T > 0, SOUP_ERR_SHAPE, "soup_embed: bad shape");
  SOUP_CHECK(soup_aligned(E, 16) && soup_aligned(h, 16), SOUP_ERR_ALIGN, "soup_embed: alignment");
  int* err = device_error_word();
  SOUP_CHECK(err, SOUP_ERR_CUDA, "device error word unavailable");
  profile_begin(static_cast<cudaStream_t>(stream), GC_ELEM, 0.0, (double)T * (H * 4.0 + 4.0));
  embed_kernel<<<(unsigned)((T + 7) / 8), 256, 0, static_cast<cudaStream_t>(stream)>>>(E, V, (int)H, ids, (int)T, h,
                                                                                        err);
  SOUP_LAUNCH_CHECK();
  profile_end(static_cast<cudaStream_t>(stream));
  return SOUP_OK;
}

extern "C" size_t soup_head_workspace(int64_t V, int64_t H, int64_t batch, int64_t seq, int32_t chunk) {
  if (V <= 0 || H <= 0 || batch <= 0 || seq <= 0 || chunk <= 0) return 0;
  return head_layout(V, H, batch * seq, chunk).total;
}

extern "C" soup_status soup_head_fwd_bwd(const uint16_t* h, const uint16_t* w_final, const uint16_t* E, int64_t V,
                                         int64_t H, const int32_t* ids, int64_t batch, int64_t seq, float eps,
                                         int32_t chunk, const float* coef, float* logp, float* dh, void* workspace,
                                         size_t workspace_bytes, void* stream) {
  SOUP_CHECK(h && w_final && E && ids && logp && workspace, SOUP_ERR_INVALID_ARG, "soup_head_fwd_bwd: null pointer");
  SOUP_CHECK(!coef == !dh, SOUP_ERR_INVALID_ARG, "soup_head_fwd_bwd: coef and dh go together");
  SOUP_CHECK(V > 0 && V < (1LL << 31) && H % 256 == 0 && batch >= 1 && seq >= 2, SOUP_ERR_SHAPE,
             "soup_head_fwd_bwd: bad shape");
  SOUP_CHECK(chunk >= 1 && chunk <= 4096 && V % 8 == 0, SOUP_ERR_SHAPE, "soup_head_fwd_bwd: chunk/vocab");
  const int64_t T = batch * seq;
  const HeadWS ws = head_layout(V, H, T, chunk);
  SOUP_CHECK(workspace_bytes >= ws.total && soup_aligned(workspace, 256), SOUP_ERR_INVALID_ARG,
             "soup_head_fwd_bwd: workspace %zu < %zu or misaligned", workspace_bytes, ws.total);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* base = static_cast<char*>(workspace);
  uint16_t* xn = reinterpret_cast<uint16_t*>(base + ws.xn);
  float* rinv = reinterpret_cast<float*>(base + ws.rinv);
  float* logits = reinterpret_cast<float*>(base + ws.logits);
  uint16_t* dlog = reinterpret_cast<uint16_t*>(base + ws.dlogits);
  float* dxn = reinterpret_cast<float*>(base + ws.dxn);
  SOUP_TRY(rmsnorm_fwd(h, nullptr, w_final, (int)T, (int)H, eps, xn, rinv, st));
  for (int64_t t0 = 0; t0 < T; t0 += chunk) {
    const int c = (int)std::min<int64_t>(chunk, T - t0);
    GemmDesc g;  // logits[c, V] = xn[t0:t0+c] E^T
    g.M = c; g.N = (int)V; g.K = (int)H;
    g.A = Mat{xn + (size_t)t0 * H, c, H, H};
    g.b_mode = B_TMA_K;
    g.B = Mat{E, V, H, H};
    g.out_kind = OUT_F32; g.out = logits; g.ldo = V;
    SOUP_TRY(gemm(g, st));
    profile_begin(st, GC_CE, 0.0, (double)c * V * (4.0 + (coef ? 2.0 : 0.0)) + c * 12.0);
    ce_rows_kernel<<<c, 1024, 0, st>>>(logits, V, ids, (int)t0, (int)seq, coef, logp, coef ? dlog : nullptr);
    SOUP_LAUNCH_CHECK();
    profile_end(st);
    if (coef) {
      GemmDesc g2;  // dxn[t0:t0+c] = dlogits E
      g2.M = c; g2.N = (int)H; g2.K = (int)V;
      g2.A = Mat{dlog, c, V, V};
      g2.b_mode = B_TMA_MN;
      g2.B = Mat{E, V, H, H};
      g2.out_kind = OUT_F32; g2.out = dxn + (size_t)t0 * H; g2.ldo = H;
      // few output tiles, long K: the persistent CTA-pair engine cuts the
      // tiles into K slices (fp32 partials in this scratch, summed in slice
      // order by the last slice of each tile)
      g2.sk_scratch = base + ws.splitk;
      g2.sk_scratch_bytes = ws.splitk_bytes;
      SOUP_TRY(gemm(g2, st));
    }
  }
  if (coef) SOUP_TRY(rmsnorm_bwd_f32dy(h, w_final, rinv, dxn, (int)T, (int)H, dh, st));
  return SOUP_OK;
}

extern "C" soup_status soup_ce_loss(const float* logp, int64_t batch, int64_t seq, float* loss, float* coef,
                                    void* stream) {
  SOUP_CHECK((loss || coef) && batch >= 1 && seq >= 2, SOUP_ERR_INVALID_ARG, "soup_ce_loss: bad argument");
  SOUP_CHECK(!loss || logp, SOUP_ERR_INVALID_ARG, "soup_ce_loss: loss needs logp");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t n = batch * (seq - 1);
  if (loss) {
    ce_mean_kernel<<<1, 1024, 0, st>>>(logp, n, loss);
    SOUP_LAUNCH_CHECK();
  }
  if (coef) {
    fill_kernel<<<(unsigned)std::min<int64_t>((n + 255) / 256, 1024), 256, 0, st>>>(coef, n, -1.0f / (float)n);
    SOUP_LAUNCH_CHECK();
  }
  return SOUP_OK;
}

extern "C" soup_status soup_dpo_loss(const float* logp_policy, const float* logp_ref, int64_t pairs, int64_t seq,
                                     int64_t prompt_len, float beta, float* loss, float* seq_sums, float* coef,
                                     void* stream) {
  SOUP_CHECK(logp_policy && logp_ref && loss && coef, SOUP_ERR_INVALID_ARG, "soup_dpo_loss: null pointer");
  SOUP_CHECK(pairs >= 1 && pairs <= 2048 && seq >= 2 && prompt_len >= 1 && prompt_len < seq, SOUP_ERR_SHAPE,
             "soup_dpo_loss: bad shape");
  dpo_kernel<<<1, 1024, (size_t)4 * pairs * sizeof(float), static_cast<cudaStream_t>(stream)>>>(
      logp_policy, logp_ref, (int)pairs, (int)seq, (int)prompt_len, beta, loss, seq_sums, coef);
  SOUP_LAUNCH_CHECK();
  return SOUP_OK;
}

namespace soup {
namespace {

// One warp per output row: 16-byte words when the row and both bases allow,
// else 4-byte words.
__global__ void gather_rows_kernel(const uint8_t* __restrict__ src, int64_t row_bytes, const int32_t* __restrict__ idx,
                                   int64_t n, uint8_t* __restrict__ dst, int vec16) {
  const int lane = threadIdx.x & 31;
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < n;
       r += (int64_t)gridDim.x * (blockDim.x >> 5)) {
    const uint8_t* s = src + (int64_t)idx[r] * row_bytes;
    uint8_t* d = dst + r * row_bytes;
    if (vec16) {
      for (int64_t w = lane; w < row_bytes / 16; w += 32)
        reinterpret_cast<uint4*>(d)[w] = reinterpret_cast<const uint4*>(s)[w];
    } else {
      for (int64_t w = lane; w < row_bytes / 4; w += 32)
        reinterpret_cast<uint32_t*>(d)[w] = reinterpret_cast<const uint32_t*>(s)[w];
    }
  }
}

// dst[d] = sum over k in [start[d], start[d+1]) of src[src_idx[k]], in k order.
__global__ void sum_rows_kernel(const float* __restrict__ src, int64_t H, const int32_t* __restrict__ src_idx,
                                const int32_t* __restrict__ start, int64_t n_dst, float* __restrict__ dst) {
  for (int64_t d = blockIdx.x; d < n_dst; d += gridDim.x) {
    const int k0 = start[d], k1 = start[d + 1];
    for (int64_t c = threadIdx.x; c < H; c += blockDim.x) {
      float acc = 0.f;
      for (int k = k0; k < k1; ++k) acc += src[(int64_t)src_idx[k] * H + c];
      dst[d * H + c] = acc;
    }
  }
}

}  // namespace
}  // namespace soup

extern "C" soup_status soup_gather_rows(const void* src, int64_t row_bytes, const int32_t* idx, int64_t n, void* dst,
                                        void* stream) {
  SOUP_CHECK(src && idx && dst, SOUP_ERR_INVALID_ARG, "soup_gather_rows: null pointer");
  SOUP_CHECK(row_bytes > 0 && row_bytes % 4 == 0 && n >= 0, SOUP_ERR_SHAPE, "soup_gather_rows: rows of %lld bytes",
             (long long)row_bytes);
  SOUP_CHECK(soup_aligned(src, 4) && soup_aligned(dst, 4), SOUP_ERR_ALIGN, "soup_gather_rows: alignment");
  if (n == 0) return SOUP_OK;
  const int vec16 = row_bytes % 16 == 0 && soup_aligned(src, 16) && soup_aligned(dst, 16);
  const unsigned blocks = (unsigned)std::min<int64_t>((n + 7) / 8, (int64_t)sm_count() * 8);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  profile_begin(st, GC_ELEM, 0.0, 2.0 * n * row_bytes + 4.0 * n);
  gather_rows_kernel<<<blocks, 256, 0, st>>>(static_cast<const uint8_t*>(src), row_bytes, idx, n,
                                             static_cast<uint8_t*>(dst), vec16);
  SOUP_LAUNCH_CHECK();
  profile_end(st);
  return SOUP_OK;
}

extern "C" soup_status soup_sum_rows_f32(const float* src, int64_t H, const int32_t* src_idx, const int32_t* start,
                                         int64_t n_dst, float* dst, void* stream) {
  SOUP_CHECK(src && src_idx && start && dst, SOUP_ERR_INVALID_ARG, "soup_sum_rows_f32: null pointer");
  SOUP_CHECK(H > 0 && n_dst >= 0, SOUP_ERR_SHAPE, "soup_sum_rows_f32: bad shape");
  if (n_dst == 0) return SOUP_OK;
  const unsigned blocks = (unsigned)std::min<int64_t>(n_dst, (int64_t)sm_count() * 16);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  profile_begin(st, GC_ELEM, 0.0, 8.0 * n_dst * H);
  sum_rows_kernel<<<blocks, 256, 0, st>>>(src, H, src_idx, start, n_dst, dst);
  SOUP_LAUNCH_CHECK();
  profile_end(st);
  return SOUP_OK;
}
