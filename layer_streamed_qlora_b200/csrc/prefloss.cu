// Reference-free preference losses over the policy's next-token log-probs:
// SimPO (Meng, Xia & Chen 2024) and ORPO (Hong, Lee & Thorne 2024), the two
// methods the Soup pages name as needing no reference model, so a step reads
// every layer twice like SFT ("memory-free reference model").
//
// Rows 2p / 2p+1 of logp [2P, S-1] are the chosen / rejected sequence of pair
// p; both share a prompt of prompt_len tokens, so every row has
// n = S - max(prompt_len, 1) continuation targets (positions j with
// j + 1 >= prompt_len).  With s the summed continuation log-probs of a row
// and m = s / n its length-normalised log-likelihood:
//   SimPO: L = -(1/P) sum_p log sigmoid(beta (m_c - m_r) - gamma)
//   ORPO:  L =  (1/P) sum_p [ -m_c - lam log sigmoid(lo_c - lo_r) ],
//          lo = m - log(1 - exp(m)) (log odds of the mean likelihood)
// The kernel also writes coef = dL/dlogp (dL/ds / n on continuation
// positions, 0 on the prompt) for the head's backward pass.  One block: the
// work is a few thousand log-probs.
#include "soup_internal.h"

namespace soup {
namespace {

enum PrefKind { PREF_SIMPO = 0, PREF_ORPO = 1 };

__device__ __forceinline__ float softplus_neg(float z) {  // log(1 + exp(-z)) = -log sigmoid(z)
  return (z > 0.f) ? log1pf(expf(-z)) : (-z + log1pf(expf(z)));
}

__device__ __forceinline__ float log1mexp(float m) {  // log(1 - exp(m)), m < 0
  return (m > -0.69314718f) ? logf(-expm1f(m)) : log1pf(-expf(m));
}

template <int KIND>
__global__ void __launch_bounds__(1024) pref_kernel(const float* __restrict__ lp, int pairs, int S, int prompt_len,
                                                    float p1, float p2, float* __restrict__ loss,
                                                    float* __restrict__ seq_out, float* __restrict__ coef) {
  extern __shared__ float sh[];  // [2P] sums | [2P] dL/dsum | [P] per-pair loss
  const int rows = 2 * pairs;
  float* dsum = sh + rows;
  float* lpair = sh + 2 * rows;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  for (int r = warp; r < rows; r += nw) {
    const float* row = lp + (size_t)r * (S - 1);
    float s = 0.f;
    for (int j = lane; j < S - 1; j += 32)
      if (j + 1 >= prompt_len) s += row[j];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) sh[r] = s;
  }
  __syncthreads();
  const float n = (float)(S - (prompt_len > 1 ? prompt_len : 1));
  const float inv_pn = 1.0f / ((float)pairs * n);
  for (int p = threadIdx.x; p < pairs; p += blockDim.x) {
    const float m_c = sh[2 * p] / n, m_r = sh[2 * p + 1] / n;
    float Lp, dc, dr;
    if (KIND == PREF_SIMPO) {  // p1 = beta, p2 = gamma
      const float z = p1 * (m_c - m_r) - p2;
      const float sg = 1.0f / (1.0f + expf(z));  // sigmoid(-z)
      Lp = softplus_neg(z);
      dc = -p1 * sg * inv_pn;
      dr = p1 * sg * inv_pn;
    } else {  // p1 = lam
      const float z = (m_c - log1mexp(m_c)) - (m_r - log1mexp(m_r));
      const float sg = 1.0f / (1.0f + expf(z));
      Lp = -m_c + p1 * softplus_neg(z);
      dc = (-1.0f - p1 * sg / -expm1f(m_c)) * inv_pn;
      dr = (p1 * sg / -expm1f(m_r)) * inv_pn;
    }
    lpair[p] = Lp;
    dsum[2 * p] = dc;
    dsum[2 * p + 1] = dr;
  }
  __syncthreads();
  if (threadIdx.x == 0) {  // fixed order: the same bits every run
    float L = 0.f;
    for (int p = 0; p < pairs; ++p) L += lpair[p];
    *loss = L / (float)pairs;
  }
  if (seq_out)
    for (int r = threadIdx.x; r < rows; r += blockDim.x) seq_out[r] = sh[r];
  for (int64_t i = threadIdx.x; i < (int64_t)rows * (S - 1); i += blockDim.x) {
    const int r = (int)(i / (S - 1)), j = (int)(i % (S - 1));
    coef[i] = (j + 1 >= prompt_len) ? dsum[r] : 0.f;
  }
}

template <int KIND>
soup_status pref_launch(const char* fn, const float* logp, int64_t pairs, int64_t seq, int64_t prompt_len, float p1,
                        float p2, float* loss, float* seq_sums, float* coef, void* stream) {
  SOUP_CHECK(logp && loss && coef, SOUP_ERR_INVALID_ARG, "%s: null pointer", fn);
  SOUP_CHECK(pairs >= 1 && pairs <= 2048 && seq >= 2 && prompt_len >= 0 && prompt_len < seq, SOUP_ERR_SHAPE,
             "%s: need 1 <= pairs <= 2048, seq >= 2 and 0 <= prompt_len < seq", fn);
  pref_kernel<KIND><<<1, 1024, (size_t)5 * pairs * sizeof(float), static_cast<cudaStream_t>(stream)>>>(
      logp, (int)pairs, (int)seq, (int)prompt_len, p1, p2, loss, seq_sums, coef);
  SOUP_LAUNCH_CHECK();
  return SOUP_OK;
}

}  // namespace
}  // namespace soup

extern "C" soup_status soup_simpo_loss(const float* logp, int64_t pairs, int64_t seq, int64_t prompt_len, float beta,
                                       float gamma, float* loss, float* seq_sums, float* coef, void* stream) {
  return soup::pref_launch<soup::PREF_SIMPO>("soup_simpo_loss", logp, pairs, seq, prompt_len, beta, gamma, loss,
                                             seq_sums, coef, stream);
}

extern "C" soup_status soup_orpo_loss(const float* logp, int64_t pairs, int64_t seq, int64_t prompt_len, float lam,
                                      float* loss, float* seq_sums, float* coef, void* stream) {
  return soup::pref_launch<soup::PREF_ORPO>("soup_orpo_loss", logp, pairs, seq, prompt_len, lam, 0.f, loss,
                                            seq_sums, coef, stream);
}
