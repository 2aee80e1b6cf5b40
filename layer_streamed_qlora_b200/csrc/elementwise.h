// Internal launchers of the memory-bound decoder-layer kernels.
#pragma once

#include "soup_internal.h"

namespace soup {

// RMSNorm over rows of x (bf16 when x_f32 is null, else fp32 x_f32); y32
// (optional) receives the fp32 values before their bf16 rounding, ylo
// (optional) the bf16 rounding residual (y ~= y_bf16 + ylo).
soup_status rmsnorm_fwd(const uint16_t* x, const float* x_f32, const uint16_t* w, int T, int H, float eps,
                        uint16_t* y, float* rinv, cudaStream_t st, float* y32 = nullptr, uint16_t* ylo = nullptr);
// in [rows, cols] bf16 -> out [cols, rows] fp32
soup_status transpose_bf16_f32(const uint16_t* in, int rows, int cols, float* out, cudaStream_t st);
// amax (optional): atomically maxed with the bit pattern of max |dh| (the
// caller zeroes it first); dh_lo (optional, with dh_bf16): the bf16 rounding
// residual of dh.
soup_status rmsnorm_bwd(const uint16_t* x, const float* x_f32, const uint16_t* w, const float* rinv,
                        const uint16_t* dy, const float* dres, int T, int H, float* dh, uint16_t* dh_bf16,
                        cudaStream_t st, unsigned int* amax = nullptr, uint16_t* dh_lo = nullptr);
// Same with an fp32 upstream gradient and no residual (the final norm).
soup_status rmsnorm_bwd_f32dy(const uint16_t* x, const uint16_t* w, const float* rinv, const float* dy, int T, int H,
                              float* dh, cudaStream_t st);
soup_status rope_table(int S, int head_dim, double theta, float* cosb, float* sinb, cudaStream_t st);
soup_status rope_apply(uint16_t* buf, int T, int S, int ld, int col0, int nh, const float* cosb, const float* sinb,
                       bool inverse, cudaStream_t st);
// D[h, t] = sum_d dO (fp16) * O (fp16)
soup_status attn_rowdot(const uint16_t* dO, const uint16_t* O, int T, int Hq, float* D, cudaStream_t st);
// out = bf16(in) (RNE), n % 8 == 0; zero_word (optional) is set to 0 by the
// same launch (a counter the next kernels accumulate into).
soup_status f32_to_bf16(const float* in, size_t n, uint16_t* out, cudaStream_t st, unsigned int* zero_word = nullptr);
soup_status bf16_to_f32(const uint16_t* in, size_t n, float* out, cudaStream_t st);

// LoRA operand preparation in one launch (up to 5 jobs):
//   PREP_COPY_F32:   out[i] = fp32(in[i]), i < rows * cols (in and out [rows, cols])
//   PREP_BLOCKDIAG_T: in = B [N, r] (rows grouped in nseg segments ending at
//     seg_end[]), out [nseg * r, N] = the block-diagonal transpose: row
//     s*r + j, column n holds B[n, j] when n lies in segment s, else 0
//     (fp32, or bf16 with out_bf16)
//   PREP_F32_TO_BF16: out [n] bf16 = RNE(in32 [n] fp32), n % 8 == 0 (the
//     activation conversion that shares the launch with the factor prep)
//   PREP_ROPE: out / out2 [N positions, r] fp32 = cos / sin of
//     pos * theta^(-2j / 2r), computed in fp64 (the same values as rope_table)
enum PrepKind : int { PREP_COPY_F32 = 0, PREP_BLOCKDIAG_T = 1, PREP_F32_TO_BF16 = 2, PREP_ROPE = 3 };
struct PrepJob {
  int kind = PREP_COPY_F32;
  int out_bf16 = 0;
  const uint16_t* in = nullptr;
  void* out = nullptr;
  int rows = 0, cols = 0;  // PREP_COPY_F32
  int N = 0, r = 0, nseg = 1;
  int seg_end[3] = {0, 0, 0};
  const float* in32 = nullptr;  // PREP_F32_TO_BF16
  long long n = 0;              // PREP_F32_TO_BF16
  void* out2 = nullptr;         // PREP_ROPE: the sin table
  double theta = 0.0;           // PREP_ROPE
};
struct PrepJobs {
  int njobs = 0;
  PrepJob job[5];
  unsigned int* zero_word = nullptr;  // optional: set to 0 by the same launch
};
soup_status lora_prep(const PrepJobs& jobs, cudaStream_t st);

// Causal GQA flash attention, head_dim 128.  qkv [T, ld] (fp16) holds q heads
// at columns [0, Hq*128), k heads at [Hq*128, (Hq+Hkv)*128), v after them;
// T = Bsz * S tokens, batch-major.  out [T, Hq*128] bf16; lse [Hq, T] (log2
// units); out16 (optional) [T, Hq*128] fp16 copy of the output, out32
// (optional) an fp32 copy.
// Sequences may come in groups of G sharing their first Lp tokens (Lp a
// multiple of 128), stored once per group as [prefix | continuation of each
// sequence]; T = Bsz / G * (Lp + G * (S - Lp)) token rows.
soup_status attention_fwd(const uint16_t* qkv, int ld, int Bsz, int S, int Hq, int Hkv, uint16_t* out,
                          float* lse, cudaStream_t st, uint16_t* out16 = nullptr, float* out32 = nullptr, int G = 1,
                          int Lp = 0);
// Backward: dout [T, Hq*128] fp16; D [Hq, T] = rowsum(dout * out); dqkv bf16; writes dq, dk,
// dv into dqkv [T, ld] at the same column layout as qkv.  q and k in qkv are
// post-RoPE; when rope_cos/rope_sin ([S, 64]) are given, dq and dk are
// rotated back (gradient w.r.t. the pre-RoPE q, k) before they are stored.
// dout carries the power-of-two gradient scale derived from *amax (gscale.cuh);
// dq, dk, dv are unscaled exactly before they are stored; dqkv32 (optional)
// receives them unrounded in fp32, same layout.
soup_status attention_bwd(const uint16_t* qkv, int ld, int Bsz, int S, int Hq, int Hkv, const uint16_t* dout,
                          const float* lse, const float* D, uint16_t* dqkv, const float* rope_cos,
                          const float* rope_sin, const unsigned int* amax, cudaStream_t st,
                          float* dqkv32 = nullptr, int G = 1, int Lp = 0);

}  // namespace soup
