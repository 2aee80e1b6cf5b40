// Internal interface of the tcgen05 GEMM engine used by every contraction of
// the training step: D[M, N] = A[M, K] * B[N, K]^T (+ tail) with bf16
// operands and fp32 accumulation in tensor memory, followed by a fused
// epilogue.
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
// Output element type and layout: row-major [M, N] or transposed [N, M].
enum OutKind : int { OUT_BF16 = 0, OUT_BF16_T = 1, OUT_F32 = 2, OUT_F32_T = 3, OUT_F16 = 4 };
enum Epi : int {
  EPI_STORE = 0,       // out = alpha * acc (+ resid), one rounding
  EPI_SWIGLU = 1,      // paired gate|up tile: out = bf16(silu(g) * u), aux16 <- fp16 g | u
  EPI_SWIGLU_BWD = 2,  // acc = dL/d(act): reads fp16 g | u from aux16, out <- bf16 dL/dg | dL/du
};

struct GemmDesc {
  int M = 0, N = 0, K = 0;
  // tf32 mode: every TMA operand is fp32 (Mat sizes in fp32 elements) and the
  // MMA is kind::tf32 (skinny K-major-B GEMMs only, no tail).
  bool tf32 = false;
  int a_major = A_K;
  Mat A;                    // [M, K] (A_K) or [K, M] (A_MN)
  // Dual-A (when A_lo.ptr is set): A is the sum of two bf16 tensors, the
  // rounded value (A) and its rounding residual (A_lo); each k-step issues
  // both MMAs against the same B tile, so an fp32-accurate A costs no extra
  // B traffic or NF4 decoding.
  Mat A_lo;
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
  // Paired tiles (gate|up): when pair_off > 0, B has 2*pair_off rows and the
  // CTA of N-tile j computes columns [j*BN/2, (j+1)*BN/2) of both halves
  // (rows of B at j*BN/2 and pair_off + j*BN/2) into one BN-wide
  // accumulator; the tail then uses tailA rows [0, 16) for the first half and
  // [16, 32) for the second.  N must equal 2*pair_off.
  int pair_off = 0;
  // Epilogue.
  int epi = EPI_STORE;
  int out_kind = OUT_BF16;
  void* out = nullptr;
  float* out2 = nullptr;            // OUT_BF16_T only: also the unrounded fp32 values, same layout
  uint16_t* out_lo = nullptr;       // OUT_BF16_T and EPI_SWIGLU_BWD: also the rounding residual
                                    // bf16(v - bf16(v)), same layout
  int64_t ldo = 0;
  const uint16_t* resid = nullptr;  // bf16 [M, N] row stride ldr (row-major outputs)
  const float* resid_f32 = nullptr; // fp32 [M, N] row stride ldr (row-major outputs)
  int64_t ldr = 0;
  float alpha = 1.f;
  // Optional power-of-two gradient scale (gscale.cuh) multiplied into alpha,
  // derived on the device from the bit pattern of an amax value.
  const unsigned int* scale_amax = nullptr;
  uint16_t* aux16 = nullptr;        // fp16 [M, 2*I] g | u (SwiGLU modes), row stride ld_aux
  int64_t ld_aux = 0;
  int swiglu_I = 0;                 // I: offset of u within aux16 / of dL/du within out
  // Optional RoPE on output columns [0, rope_cols) (128-wide heads): pairs
  // (i, i+64) of each head rotated by the angle of position row % rope_S,
  // cos/sin tables [rope_S, 64] fp32, applied to the fp32 accumulator.
  int rope_cols = 0, rope_S = 0;
  const float* rope_cos = nullptr;
  const float* rope_sin = nullptr;
  // Rows in groups of rope_group sequences sharing their first rope_prefix
  // positions (stored once: [prefix | continuation of each sequence]): the
  // position of a row is then its position within its sequence (rope_S =
  // the sequence length).  rope_group <= 1: position = row % rope_S.
  int rope_prefix = 0, rope_group = 1;
  int bn = 0;               // N tile (0 = pick)
  // NF4 GEMMs on CTA pairs: persistent tile loop with two accumulators (the
  // epilogue of one tile overlaps the next tile's main loop) or one tile
  // per pair
  bool persistent = true;
  // Persistent kernel: scratch for the fp32 partials of a split last round
  // of tiles (256 KB per slice; null: whole tiles only).  Device memory
  // that nothing else uses during the call.
  void* sk_scratch = nullptr;
  size_t sk_scratch_bytes = 0;
  // Optional split-K for skinny GEMMs (N <= 64, TMA operands, plain store
  // epilogue): when a workspace is given and the M x N tiles alone cannot
  // fill the GPU, the K range is cut into up to 8 slices whose fp32 partial
  // products land in split_ws ([slices, M, N]); a second kernel sums them
  // in slice order (deterministic) and applies the epilogue.
  float* split_ws = nullptr;
  size_t split_ws_bytes = 0;
  // Clock cycles a bounded mbarrier wait in the kernel may take before the
  // CTA records an error and winds down (0 = the default, ~2 s).
  long long wait_limit = 0;
  // Test hook, honoured by the one-CTA engine only: the TMA producer issues
  // no loads and never arrives, so the MMA warp's bounded wait runs out.
  int debug_skip_producer = 0;
};

soup_status gemm(const GemmDesc& d, cudaStream_t stream);

}  // namespace soup
