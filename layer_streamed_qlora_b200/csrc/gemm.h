// Internal interface of the tcgen05 GEMM engine used by every contraction of
// the training step: D[M, N] = A[M, K] * B[N, K]^T (+ tail) with bf16
// operands and fp32 accumulation in tensor memory.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "soup_internal.h"

namespace soup {

// A bf16 matrix in device memory, row-major [rows, cols], row stride `ld`
// elements (ld*2 must be a multiple of 16 bytes for TMA).
struct Mat {
  const void* ptr = nullptr;
  int64_t rows = 0, cols = 0, ld = 0;
};

enum AMajor : int { A_K = 0, A_MN = 1 };           // A stored [M, K] or [K, M]
enum BMode : int {
  B_TMA_K = 0,   // B stored [N, K] bf16
  B_TMA_MN = 1,  // B stored [K, N] bf16
  B_NF4_K = 2,   // B = dequant(codes [N, K/2], absmax [N, K/64])      (forward W)
  B_NF4_MN = 3,  // B = dequant(codes [K, N/2], absmax [K, N/64])^T    (backward W^T)
};
enum OutKind : int { OUT_BF16 = 0, OUT_BF16_T = 1, OUT_F32 = 2, OUT_F32_T = 3 };

struct GemmDesc {
  int M = 0, N = 0, K = 0;
  int a_major = A_K;
  Mat A;                    // [M, K] (A_K) or [K, M] (A_MN)
  int b_mode = B_TMA_K;
  Mat B;                    // bf16 B for TMA modes
  const uint8_t* codes = nullptr;
  const float* absmax = nullptr;
  // Optional extra K-block appended after the main loop ("tail"): a LoRA
  // up-projection folded into the same accumulator.  tailA is stored
  // transposed, [rows, M] (row offset chosen per N segment), tailB has the
  // same major-ness as B: [N, r] for K-major modes, [r, N] for MN-major ones.
  int tail_ksteps = 0;      // 16-wide k-steps of the tail (0 = none, max 4)
  Mat tailA, tailB;
  int nseg = 1;             // N segments (tiles never straddle a segment end)
  int seg_end[4] = {0, 0, 0, 0};
  int seg_row[4] = {0, 0, 0, 0};
  // Epilogue: out = alpha * acc (+ resid), rounded once.
  int out_kind = OUT_BF16;
  void* out = nullptr;
  int64_t ldo = 0;
  const uint16_t* resid = nullptr;  // bf16 [M, N] row stride ldr (OUT_BF16 only)
  int64_t ldr = 0;
  float alpha = 1.f;
  int bn = 0;               // N tile (0 = pick)
};

soup_status gemm(const GemmDesc& d, cudaStream_t stream);

}  // namespace soup
