// tcgen05 GEMM engine for sm_100a.
//
// D[M, N] (fp32, tensor memory) = A[M, K] * B[N, K]^T  (+ tailA * tailB^T)
//
// * 128 x BN x 64 CTA tiles, one CTA per SM (shared memory ~196 KB), a ring of
//   STAGES shared-memory stages, warp-specialised:
//     warp 0      one elected thread issues TMA loads (A, bf16 B, tail tiles)
//     warp 1      allocates tensor memory; one elected thread issues
//                 tcgen05.mma (M=128, N=BN, K=16) and tcgen05.commit
//     warps 2..   NF4 modes: 8 warps decode the packed 4-bit weights straight
//                 into the 128-byte-swizzled B stage (the "NF4 dequant
//                 prologue"), then all of them run the epilogue;
//                 bf16 modes: 4 epilogue warps.
// * The LoRA up-projection is folded in as one extra K-block ("tail"): after
//   the main loop the same accumulator receives u[M, r] * B_lora[N, r]^T
//   (forward) or g'[M, r] * A_lora[r, N] (backward), so the adapter term costs
//   at most one more 64-wide k-stage and no extra pass over y.
// * Every mbarrier wait is bounded in time; on expiry the CTA records an error
//   in the device error word and winds down (no hang).
//
// Operand layouts in shared memory (128-byte swizzle, 1024-byte atoms):
//   K-major tile [rows, 64]: row i at i*128 bytes, 16-byte unit u stored at
//     unit position u ^ (i % 8); descriptor SBO = 1024, k-step advance 32 B.
//   MN-major tile [64 k-rows, 64*c MN]: chunk c (64 MN elements) at c*8192,
//     k-row j at j*128, unit u at u ^ (j % 8); descriptor LBO = 8192 (chunk
//     stride), SBO = 1024, k-step advance 2048 B.
#include <cuda.h>

#include <algorithm>
#include <atomic>

#include "gemm.h"
#include "nf4_codebook.cuh"
#include "ptx.cuh"
#include "gscale.cuh"
#include <cuda_fp16.h>

namespace soup {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int A_STAGE_BYTES = BM * BK * 2;  // 16 KB

template <int BN, bool DUAL = false, int CG = 1, bool NF4B = true>
struct Cfg {
  // DUAL: each stage holds two A tiles (the hi and lo bf16 parts of a more
  // precise A), multiplied against the same B tile.  CG = 2: the tile is
  // shared by a CTA pair (M = 256 over the pair, each CTA holds half of B).
  // NF4B (CTA pairs): B is decoded from NF4 codes; otherwise bf16 B tiles
  // come straight from TMA and there is no decode table.
  static constexpr int A_STAGE = A_STAGE_BYTES * (DUAL ? 2 : 1);
  static constexpr int B_STAGE = (BN / CG) * BK * 2;
  // NF4 CTA pairs also stage the packed codes (128 rows x 32 bytes, or 64
  // k-rows x 64 bytes) and a 4-block-wide absmax box per stage through TMA
  static constexpr int C_STAGE = (CG == 2 && NF4B) ? 4096 : 0;
  static constexpr int S_STAGE = (CG == 2 && NF4B) ? 2048 : 0;
  static constexpr int TMEM_COLS = BN <= 32 ? 32 : (BN <= 64 ? 64 : (BN <= 128 ? 128 : 256));
  static constexpr int BAR_BYTES = 256;
  // CTA pairs: byte-indexed NF4 table (256 code pairs x 32 lanes x float2;
  // x 16 half-warp lanes when two A tiles per stage leave no room) at the
  // start of shared memory; single CTAs: nibble table after the barriers
  static constexpr int LUT_LANES = DUAL ? 16 : 32;
  static constexpr int LUT_BYTES = CG == 2 ? (NF4B ? 256 * LUT_LANES * 8 : 0) : 16 * 32 * 4;
  static constexpr int STAGE_BYTES = A_STAGE + B_STAGE + C_STAGE + S_STAGE;
  static constexpr int STAGE_BUDGET = CG == 2 ? (232448 - 1024 - BAR_BYTES - LUT_BYTES) : 196608;
  static constexpr int STAGES = (STAGE_BUDGET / STAGE_BYTES) > 8 ? 8 : (STAGE_BUDGET / STAGE_BYTES);
  static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + BAR_BYTES + LUT_BYTES;
};

struct KArgs {
  int M, N, K, num_kb;
  int kb_split;  // split-K: k-blocks per slice (blockIdx.z = slice), 0 = no split
  const uint8_t* codes;
  const float* absmax;
  int tail_ksteps, nseg;
  int seg_end[4], seg_row[4];
  int pair_off;
  int epi, out_kind;
  void* out;
  float* out2;
  uint16_t* out_lo;
  long long ldo;
  const uint16_t* resid;
  const float* resid_f32;
  long long ldr;
  float alpha;
  const unsigned int* scale_amax;
  uint16_t* aux16;
  long long ld_aux;
  int swiglu_I;
  int vec_ok;
  int rope_cols, rope_S, rope_Lp, rope_G;
  const float* rope_cos;
  const float* rope_sin;
  int* err;
  long long wait_limit;  // clock cycles a bounded mbarrier wait may take before it gives up
  int skip_producer;     // test hook (one-CTA kernel): the TMA producer issues nothing and never arrives
  // Persistent kernel, last partial round split along K: every pair first
  // takes sk_full whole tiles (t = pair + j * pairs), then the slice units
  // u = pair, pair + pairs, ... < sk_units, unit u being k-slice u % sk_k of
  // leftover tile sk_full * pairs + u / sk_k.  A slice stores its fp32
  // partial ([256 columns][128 rows] per CTA) in sk_ws; the last slice of a
  // tile to finish (counted in sk_cnt, tagged with sk_epoch) sums the
  // tile's partials in slice order and runs the epilogue.  sk_k < 2: whole
  // tiles only.
  int sk_full, sk_units, sk_k;
  float* sk_ws;
  unsigned long long* sk_cnt;
  unsigned int sk_epoch;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}
__device__ __forceinline__ float f16_to_f32(uint16_t b) {
  return __half2float(__ushort_as_half(b));
}

// Stores 16 consecutive values of one row (row-major 16-bit or fp32 output),
// vectorised when the whole chunk is in range and aligned (vec: 0 scalar,
// 1 16-byte, 2 32-byte accesses).
__device__ __forceinline__ void store_row16(void* out, int out_kind, long long ldo, int row, int n, int N,
                                            const float (&f)[16], int vec) {
  const bool full = vec && (n + 16 <= N);
  if (out_kind == OUT_F32) {
    float* o = static_cast<float*>(out) + (size_t)row * ldo + n;
    if (full && vec == 2) {
      uint32_t w[8];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = __float_as_uint(f[8 * h + i]);
        ptx::st_global_32B(o + 8 * h, w);
      }
    } else if (full) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        reinterpret_cast<float4*>(o)[i] = make_float4(f[4 * i], f[4 * i + 1], f[4 * i + 2], f[4 * i + 3]);
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (n + i < N) o[i] = f[i];
    }
    return;
  }
  uint16_t* o = static_cast<uint16_t*>(out) + (size_t)row * ldo + n;
  const bool h = out_kind == OUT_F16;
  if (full) {
    uint32_t p[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) p[i] = h ? pack_f16x2(f[2 * i], f[2 * i + 1]) : pack_bf16x2(f[2 * i], f[2 * i + 1]);
    if (vec == 2) {
      ptx::st_global_32B(o, p);
    } else {
      reinterpret_cast<uint4*>(o)[0] = make_uint4(p[0], p[1], p[2], p[3]);
      reinterpret_cast<uint4*>(o)[1] = make_uint4(p[4], p[5], p[6], p[7]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (n + i < N) {
        const uint32_t w = h ? pack_f16x2(f[i], 0.f) : pack_bf16x2(f[i], 0.f);
        o[i] = static_cast<uint16_t>(w & 0xFFFF);
      }
  }
}

// 16 consecutive 16-bit values as 8 packed words (element 2i in the low half)
__device__ __forceinline__ void load8_u32(const uint16_t* p, uint32_t (&w)[8], int vec) {
  if (vec == 2) {
    ptx::ld_global_32B(p, w);
  } else {
    const uint4 a = *reinterpret_cast<const uint4*>(p);
    const uint4 b = *reinterpret_cast<const uint4*>(p + 8);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  }
}

__device__ __forceinline__ void load16_u16(const uint16_t* p, uint16_t (&v)[16], int vec) {
  uint32_t w[8];
  if (vec == 2) {
    ptx::ld_global_32B(p, w);
  } else {
    const uint4 a = *reinterpret_cast<const uint4*>(p);
    const uint4 b = *reinterpret_cast<const uint4*>(p + 8);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[2 * i] = static_cast<uint16_t>(w[i] & 0xFFFF);
    v[2 * i + 1] = static_cast<uint16_t>(w[i] >> 16);
  }
}

__device__ __forceinline__ float sigmoid_f(float g) { return 1.0f / (1.0f + expf(-g)); }

// 8 NF4 codes (one 32-bit word: byte p holds element 2p high, 2p+1 low) ->
// 8 bf16 values RNE(fp32(c * absmax)) packed in a uint4.
__device__ __forceinline__ uint4 decode8(uint32_t w, const float* lut_lane, float am) {
  uint32_t o[4];
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const uint32_t c0 = (w >> (8 * p + 4)) & 15u;
    const uint32_t c1 = (w >> (8 * p)) & 15u;
    const float f0 = lut_lane[c0 * 32] * am;
    const float f1 = lut_lane[c1 * 32] * am;
    o[p] = pack_bf16x2(f0, f1);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Same result from the byte-indexed table of the pair kernels: entry b of
// lane l holds the codebook values of the two codes packed in byte b (high
// nibble first), at byte offset b*256 + l*8 (LANES = 32; lane_b = l*8) or, in
// the half-size table, b*128 + (l % 16)*8 (LANES = 16; lane_b = (l % 16)*16,
// the offset halved after the permute), so that the lanes reading one 8-byte
// wavefront hit distinct banks.  One byte permute forms the offset, one
// 8-byte shared load fetches both values, one packed multiply scales them,
// and the products are rounded exactly as above.
template <int LANES>
__device__ __forceinline__ uint4 decode8_pairs(uint32_t w, const uint8_t* lut_bytes, uint32_t lane_b, float am) {
  uint32_t o[4];
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    uint32_t off = __byte_perm(w, lane_b, 0x5504u | ((uint32_t)p << 4));
    if (LANES == 16) off >>= 1;
    const float2 c = *reinterpret_cast<const float2*>(lut_bytes + off);
    const float2 f = ptx::mul_f32x2(c, am);
    o[p] = pack_bf16x2(f.x, f.y);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ void st_shared_v4(void* p, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(ptx::smem_u32(p)), "r"(v.x),
               "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

template <int NWORDS>
__device__ __forceinline__ void load_codes(const uint8_t* src, uint32_t (&w)[NWORDS]) {
  if constexpr (NWORDS == 8) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(src));
    const uint4 b = __ldg(reinterpret_cast<const uint4*>(src) + 1);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  } else if constexpr (NWORDS == 4) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(src));
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
  } else {
    const uint2 a = __ldg(reinterpret_cast<const uint2*>(src));
    w[0] = a.x; w[1] = a.y;
  }
}

// Epilogue of one accumulator tile: the warp owns TMEM lanes 32q..32q+31
// (output rows m0 + 32q + lane) of the accumulator at column `tacc`, and its
// 16-column chunks ch0, ch0 + chs, ...
//
// The accumulator comes from tensor memory, or (split tile: parts != null)
// is the sum, in slice order, of nparts fp32 partials stored column-major
// ([256 columns][128 rows] per CTA, slices 2 * 32768 floats apart).
constexpr int SK_HALF = 256 * 128;  // floats of one CTA's partial
__device__ __forceinline__ void acc_ld16(uint32_t taddr, int c, uint32_t (&v)[16], const float* parts, int nparts,
                                         int prow) {
  if (!parts) {
    ptx::tmem_ld16(taddr + c, v);
    ptx::tmem_ld_wait();
    return;
  }
  float a[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) a[i] = 0.f;
  for (int z = 0; z < nparts; ++z) {
    const float* pz = parts + (size_t)z * 2 * SK_HALF + (size_t)c * 128 + prow;
#pragma unroll
    for (int i = 0; i < 16; ++i) a[i] += __ldcg(pz + i * 128);
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __float_as_uint(a[i]);
}

template <int BN>
__device__ __forceinline__ void epilogue_tile(const KArgs& args, void* outp, uint32_t tacc, int m0, int n0, int nb,
                                              int q, int lane, int ch0, int chs, const float* parts = nullptr,
                                              int nparts = 0) {
  const uint32_t trow = tacc + ((uint32_t)(q * 32) << 16);
  const int prow = q * 32 + lane;
  const int row = m0 + q * 32 + lane;
  const bool row_ok = row < args.M;
  constexpr int NCH = BN / 16;
  const float alpha =
      args.scale_amax ? args.alpha * grad_scale_from_amax(__uint_as_float(*args.scale_amax)) : args.alpha;
  const int vec = args.vec_ok;
  if (args.epi == EPI_SWIGLU) {
    // paired gate|up tile: chunk c (gate) pairs with c + NCH/2 (up); both
    // owned by this warp (NCH/2 is even)
    const int I = args.swiglu_I;
    for (int ch = ch0; ch < NCH / 2; ch += chs) {
      uint32_t vg[16], vu[16];
      acc_ld16(trow, ch * 16, vg, parts, nparts, prow);
      acc_ld16(trow, (ch + NCH / 2) * 16, vu, parts, nparts, prow);
      const int n = nb + ch * 16;
      if (!row_ok || n >= I) continue;
      float a[16], gg[16], uu[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        gg[i] = __uint_as_float(vg[i]) * alpha;
        uu[i] = __uint_as_float(vu[i]) * alpha;
        a[i] = gg[i] * sigmoid_f(gg[i]) * uu[i];
      }
      store_row16(outp, OUT_BF16, args.ldo, row, n, I, a, vec);
      if (args.aux16) {
        store_row16(args.aux16, OUT_F16, args.ld_aux, row, n, I, gg, vec);
        store_row16(args.aux16 + I, OUT_F16, args.ld_aux, row, n, I, uu, vec);
      }
    }
  } else if ((BN >= 128) && args.rope_cols > 0 && n0 < args.rope_cols) {
    // RoPE (q/k heads of the fused QKV projection): the pair (i, i + 64)
    // of a 128-wide head lives in chunks c and c + 4 of the head, which
    // the same warp owns; rotate the fp32 accumulators, then round once.
    for (int ch = ch0; ch < NCH; ch += chs) {
      if ((ch & 7) >= 4) continue;
      uint32_t v0[16], v1[16];
      acc_ld16(trow, ch * 16, v0, parts, nparts, prow);
      acc_ld16(trow, (ch + 4) * 16, v1, parts, nparts, prow);
      const int n = n0 + ch * 16;
      if (!row_ok || n >= args.N) continue;
      int pos = row % args.rope_S;
      if (args.rope_G > 1) {  // shared-prefix layout: position within the row's sequence
        const int lc = args.rope_S - args.rope_Lp;
        const int r = row % (args.rope_Lp + args.rope_G * lc);
        pos = r < args.rope_Lp ? r : args.rope_Lp + (r - args.rope_Lp) % lc;
      }
      const float* cs = args.rope_cos + (size_t)pos * 64 + (ch & 7) * 16;
      const float* sn = args.rope_sin + (size_t)pos * 64 + (ch & 7) * 16;
      // the position's 16 angles of the chunk, 8 at a time: 32-byte loads
      // where aligned (each thread owns a row, so scalar loads would touch
      // 32 rows apiece)
      float a[16], b[16];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t cw[8], sw[8];
        if (vec == 2) {
          ptx::ld_global_32B(cs + 8 * hh, cw);
          ptx::ld_global_32B(sn + 8 * hh, sw);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            cw[i] = __float_as_uint(__ldg(cs + 8 * hh + i));
            sw[i] = __float_as_uint(__ldg(sn + 8 * hh + i));
          }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int e = 8 * hh + i;
          const float x0 = __uint_as_float(v0[e]) * alpha, x1 = __uint_as_float(v1[e]) * alpha;
          const float c = __uint_as_float(cw[i]), sv = __uint_as_float(sw[i]);
          a[e] = x0 * c - x1 * sv;
          b[e] = x1 * c + x0 * sv;
        }
      }
      store_row16(outp, args.out_kind, args.ldo, row, n, args.N, a, vec);
      store_row16(outp, args.out_kind, args.ldo, row, n + 64, args.N, b, vec);
    }
  } else if (args.epi == EPI_SWIGLU_BWD) {
    // acc = dL/d(act); g, u from the forward (fp16); out = [dL/dg | dL/du]
    // bf16 (+ rounding residuals)
    const int I = args.swiglu_I;
    for (int ch = ch0; ch < NCH; ch += chs) {
      const int n = n0 + ch * 16;
      uint32_t v[16];
      acc_ld16(trow, ch * 16, v, parts, nparts, prow);
      if (!row_ok || n >= args.N) continue;
      const bool full16 = vec && (n + 16 <= args.N);
      uint32_t gw[8], uw[8];  // fp16 pairs (element 2i low)
      const uint16_t* gp = args.aux16 + (size_t)row * args.ld_aux + n;
      if (full16) {
        load8_u32(gp, gw, vec);
        load8_u32(gp + I, uw, vec);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t g0 = (n + 2 * i < args.N) ? gp[2 * i] : 0, g1 = (n + 2 * i + 1 < args.N) ? gp[2 * i + 1] : 0;
          const uint32_t u0 = (n + 2 * i < args.N) ? gp[I + 2 * i] : 0,
                         u1 = (n + 2 * i + 1 < args.N) ? gp[I + 2 * i + 1] : 0;
          gw[i] = g0 | (g1 << 16);
          uw[i] = u0 | (u1 << 16);
        }
      }
      float dg[16], du[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float f = __uint_as_float(v[i]) * alpha;
        const float g = f16_to_f32(static_cast<uint16_t>(gw[i >> 1] >> (16 * (i & 1)))),
                    u = f16_to_f32(static_cast<uint16_t>(uw[i >> 1] >> (16 * (i & 1))));
        const float sg = sigmoid_f(g);
        dg[i] = f * u * sg * (1.0f + g * (1.0f - sg));
        du[i] = f * g * sg;
      }
      store_row16(outp, OUT_BF16, args.ldo, row, n, args.N, dg, vec);
      store_row16(static_cast<uint16_t*>(outp) + I, OUT_BF16, args.ldo, row, n, args.N, du, vec);
      if (args.out_lo) {  // rounding residuals of both halves, same layout
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          dg[i] -= bf16_to_f32(static_cast<uint16_t>(pack_bf16x2(dg[i], 0.f) & 0xFFFF));
          du[i] -= bf16_to_f32(static_cast<uint16_t>(pack_bf16x2(du[i], 0.f) & 0xFFFF));
        }
        store_row16(args.out_lo, OUT_BF16, args.ldo, row, n, args.N, dg, vec);
        store_row16(args.out_lo + I, OUT_BF16, args.ldo, row, n, args.N, du, vec);
      }
    }
  } else {
    for (int ch = ch0; ch < NCH; ch += chs) {
      uint32_t v[16];
      acc_ld16(trow, ch * 16, v, parts, nparts, prow);
      const int n = n0 + ch * 16;
      if (!row_ok || n >= args.N) continue;
      float f[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) f[i] = __uint_as_float(v[i]) * alpha;
      const bool full16 = vec && (n + 16 <= args.N);
      if (args.out_kind == OUT_BF16_T || args.out_kind == OUT_F32_T) {
        if (args.out_kind == OUT_BF16_T) {
          uint16_t* o = static_cast<uint16_t*>(outp);
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (n + i < args.N)
              o[(size_t)(n + i) * args.ldo + row] = static_cast<uint16_t>(pack_bf16x2(f[i], 0.f) & 0xFFFF);
          if (args.out2) {  // the same values unrounded, fp32, same layout
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (n + i < args.N) args.out2[(size_t)(n + i) * args.ldo + row] = f[i];
          }
          if (args.out_lo) {  // rounding residual: hi + lo carries ~16 significant bits
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (n + i < args.N) {
                const uint16_t hb = static_cast<uint16_t>(pack_bf16x2(f[i], 0.f) & 0xFFFF);
                args.out_lo[(size_t)(n + i) * args.ldo + row] =
                    static_cast<uint16_t>(pack_bf16x2(f[i] - bf16_to_f32(hb), 0.f) & 0xFFFF);
              }
          }
        } else {
          float* o = static_cast<float*>(outp);
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (n + i < args.N) o[(size_t)(n + i) * args.ldo + row] = f[i];
        }
        continue;
      }
      if (args.resid) {
        const uint16_t* r = args.resid + (size_t)row * args.ldr + n;
        if (full16) {
          uint16_t rb[16];
          load16_u16(r, rb, vec);
#pragma unroll
          for (int i = 0; i < 16; ++i) f[i] += bf16_to_f32(rb[i]);
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (n + i < args.N) f[i] += bf16_to_f32(r[i]);
        }
      } else if (args.resid_f32) {
        const float* r = args.resid_f32 + (size_t)row * args.ldr + n;
        if (full16 && vec == 2) {
          uint32_t w[8];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            ptx::ld_global_32B(r + 8 * h, w);
#pragma unroll
            for (int i = 0; i < 8; ++i) f[8 * h + i] += __uint_as_float(w[i]);
          }
        } else if (full16) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float4 x = reinterpret_cast<const float4*>(r)[i];
            f[4 * i] += x.x; f[4 * i + 1] += x.y; f[4 * i + 2] += x.z; f[4 * i + 3] += x.w;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (n + i < args.N) f[i] += r[i];
        }
      }
      store_row16(outp, args.out_kind, args.ldo, row, n, args.N, f, vec);
    }
  }
}

template <int BN, int AMJ, int BMD, bool TF, bool DUAL, int CG>
__global__ void __launch_bounds__(32 * (2 + (BMD >= B_NF4_K ? 8 : 4)), 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmTA,
                const __grid_constant__ CUtensorMap tmTB, const __grid_constant__ CUtensorMap tmA2,
                const __grid_constant__ CUtensorMap tmA3,
                const KArgs args) {
  using C = Cfg<BN, DUAL, CG>;
  static_assert(!DUAL || (AMJ == A_K && !TF), "dual-A: K-major bf16 A only");
  static_assert(CG == 1 || (BN == 256 && AMJ == A_K && BMD >= B_NF4_K && !TF),
                "CTA pairs: NF4 B, K-major bf16 A, 256-wide tiles");
  constexpr bool NF4 = BMD >= B_NF4_K;
  constexpr bool B_MN = (BMD == B_TMA_MN || BMD == B_NF4_MN);
  constexpr int STAGES = C::STAGES;
  constexpr int NEPI = NF4 ? 8 : 4;
  // Element geometry: every stage row is one 128-byte swizzle row.  bf16:
  // 64 K-elements per stage, K = 16 per MMA, 64-wide MN-major chunks; tf32
  // (fp32 operands): 32 K-elements per stage, K = 8 per MMA, 32-wide chunks.
  constexpr int BKE = TF ? 32 : 64;          // K elements per stage
  constexpr int KI = TF ? 8 : 16;            // K per MMA instruction
  constexpr int CW = TF ? 32 : 64;           // MN-major chunk width (elements)
  constexpr int CHUNK_BYTES = BKE * 128;     // one MN-major chunk of a stage
  constexpr int KSTEP_MN = KI * 128;         // MN-major descriptor advance per MMA
  static_assert(!TF || (BMD == B_TMA_K), "tf32 mode: TMA-fed K-major B only");

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  constexpr int LUT_FRONT = CG == 2 ? C::LUT_BYTES : 0;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw + LUT_FRONT) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * C::A_STAGE;
  uint8_t* sC = sB + STAGES * C::B_STAGE;     // CTA pairs: packed codes per stage
  uint8_t* sS = sC + STAGES * C::C_STAGE;     // CTA pairs: absmax box per stage
  uint64_t* full = reinterpret_cast<uint64_t*>(sS + STAGES * C::S_STAGE);
  uint64_t* empty = full + STAGES;
  uint64_t* cfull = empty + STAGES;           // CTA pairs: codes + absmax of the stage landed
  uint64_t* accf = cfull + (CG == 2 ? STAGES : 0);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* lut = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(full) + C::BAR_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // CTA pairs: blockIdx.x = 2 * (pair M tile) + rank; this CTA owns rows
  // [m0, m0 + 128) of A and of the accumulator either way
  const uint32_t rank = CG == 2 ? ptx::cluster_ctarank() : 0u;
  const int m0 = blockIdx.x * BM;
  const bool paired = args.pair_off > 0;
  // paired: the tile covers columns [nb, nb + BN/2) of both halves
  const int nb = paired ? blockIdx.y * (BN / 2) : blockIdx.y * BN;
  const int n0 = nb;  // first B row / output column of the tile (first half when paired)
  // split-K: this CTA's slice of k-blocks and its fp32 partial-product plane
  const int kz = args.kb_split > 0 ? (int)blockIdx.z * args.kb_split : 0;
  const int num_kb = args.kb_split > 0 ? min(args.kb_split, args.num_kb - kz) : args.num_kb;
  const int n_iters = num_kb + (args.tail_ksteps > 0 ? 1 : 0);
  void* const outp = args.kb_split > 0 ? static_cast<void*>(static_cast<float*>(args.out) +
                                                           (size_t)blockIdx.z * args.M * args.N)
                                       : args.out;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(&full[s], CG == 2 ? 1 + 16 : 1 + (NF4 ? 8 : 0));
      ptx::mbar_init(&empty[s], 1);
      if (CG == 2) ptx::mbar_init(&cfull[s], 1);
    }
    ptx::mbar_init(accf, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tmA);
    if (DUAL || CG == 2) ptx::prefetch_tmap(&tmA2);
    if (DUAL && CG == 2) ptx::prefetch_tmap(&tmA3);
    if (!NF4 || CG == 2) ptx::prefetch_tmap(&tmB);
    if (args.tail_ksteps > 0) {
      ptx::prefetch_tmap(&tmTA);
      ptx::prefetch_tmap(&tmTB);
    }
  }
  if (NF4 && threadIdx.x >= 64) {
    if constexpr (CG == 2) {
      // entry b of every lane: (c[b >> 4], c[b & 15])
      float2* lut2 = reinterpret_cast<float2*>(smem_raw);
      for (int i = threadIdx.x - 64; i < 256 * C::LUT_LANES; i += 256) {
        const int b = i / C::LUT_LANES;
        lut2[i] = make_float2(__uint_as_float(c_nf4_bits[b >> 4]), __uint_as_float(c_nf4_bits[b & 15]));
      }
    } else {
      for (int i = threadIdx.x - 64; i < 16 * 32; i += 256) lut[i] = __uint_as_float(c_nf4_bits[i >> 5]);
    }
  }
  if (warp == 1) {
    if constexpr (CG == 2) {
      ptx::tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
      ptx::tmem_relinquish_pair();
    } else {
      ptx::tmem_alloc(tmem_slot, C::TMEM_COLS);
      ptx::tmem_relinquish();
    }
  }
  ptx::tc_fence_before();
  if constexpr (CG == 2) ptx::cluster_sync();  // both CTAs' barriers exist before any cross-CTA signal
  else __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // tail row offset of this tile's N segment (no dynamic indexing of the
  // parameter arrays, which would spill them to local memory)
  int tail_row = args.seg_row[0];
  if (args.nseg > 1 && n0 >= args.seg_end[0]) tail_row = args.seg_row[1];
  if (args.nseg > 2 && n0 >= args.seg_end[1]) tail_row = args.seg_row[2];
  if (args.nseg > 3 && n0 >= args.seg_end[2]) tail_row = args.seg_row[3];
  if (paired) tail_row = 0;

  if (CG == 2 && warp == 0) {
    // ------------------------------------------- TMA producer (CTA pair)
    // Each CTA loads its own A rows (and its half of the tail B); the
    // transaction bytes of both land on the even CTA's full barrier.
    if (lane == 0) {
      const uint32_t full0 = ptx::mapa_shared(ptx::smem_u32(full), 0);
      for (int ip = 0; ip < 12 && ip < num_kb; ++ip) {  // warm L2 with the first stages' codes
        if (!B_MN) {
          const int r0 = paired ? (rank == 0 ? nb : args.pair_off + nb) : n0 + (int)rank * 128;
          ptx::tma_prefetch_l2_2d(&tmB, ip * 32, r0);
          if ((ip & 3) == 0) ptx::tma_prefetch_l2_2d(&tmA2, ip, r0);
        } else {
          const int c0 = n0 + (int)rank * 128;
          ptx::tma_prefetch_l2_2d(&tmB, c0 / 2, ip * BK);
          ptx::tma_prefetch_l2_2d(&tmA2, (c0 / 64) & ~3, ip * BK);
        }
      }
      for (int it = 0; it < n_iters; ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (!ptx::mbar_wait_bounded(&empty[s], ph ^ 1, abort_flag, args.wait_limit)) {
          atomicOr(args.err, 1);
          *abort_flag = 1;
          break;
        }
        uint8_t* a = sA + s * C::A_STAGE;
        uint8_t* b = sB + s * C::B_STAGE;
        const bool tail = it >= num_kb;
        const uint32_t bytes = tail ? (uint32_t)(A_STAGE_BYTES + C::B_STAGE) : (uint32_t)C::A_STAGE;
        if (rank == 0) ptx::mbar_arrive_expect_tx(&full[s], 2 * bytes);
        const uint32_t bar = full0 + s * 8;
        if (!tail) {
          ptx::tma_load_2d_pair(a, &tmA, bar, it * BKE, m0);
          // hi + lo A pair: the rounding residual tile (tmA3) beside it
          if (DUAL) ptx::tma_load_2d_pair(a + A_STAGE_BYTES, &tmA3, bar, it * BKE, m0);
          // this CTA's codes and absmax for the stage (tmB: codes bytes,
          // tmA2: absmax fp32; boxes out of range read as zeros), and an L2
          // prefetch of those of stage it + PF, so that a slot refill, issued
          // only when the slot frees, waits for L2 rather than DRAM
          uint8_t* c = sC + s * C::C_STAGE;
          uint8_t* sc = sS + s * C::S_STAGE;
          constexpr int PF = 12;
          const int ip = it + PF;
          ptx::mbar_arrive_expect_tx(&cfull[s], (uint32_t)(C::C_STAGE + (B_MN ? 1024 : 2048)));
          if (!B_MN) {
            const int r0 = paired ? (rank == 0 ? nb : args.pair_off + nb) : n0 + (int)rank * 128;
            ptx::tma_load_2d(c, &tmB, &cfull[s], it * 32, r0);
            ptx::tma_load_2d(sc, &tmA2, &cfull[s], it & ~3, r0);
            if (ip < num_kb) {
              ptx::tma_prefetch_l2_2d(&tmB, ip * 32, r0);
              if ((ip & 3) == 0) ptx::tma_prefetch_l2_2d(&tmA2, ip, r0);
            }
          } else {
            const int c0 = n0 + (int)rank * 128;
            ptx::tma_load_2d(c, &tmB, &cfull[s], c0 / 2, it * BK);
            ptx::tma_load_2d(sc, &tmA2, &cfull[s], (c0 / 64) & ~3, it * BK);
            if (ip < num_kb) {
              ptx::tma_prefetch_l2_2d(&tmB, c0 / 2, ip * BK);
              ptx::tma_prefetch_l2_2d(&tmA2, (c0 / 64) & ~3, ip * BK);
            }
          }
        } else {
          ptx::tma_load_2d_pair(a, &tmTA, bar, m0, tail_row);
          ptx::tma_load_2d_pair(a + 8192, &tmTA, bar, m0 + 64, tail_row);
          if (!B_MN) {
            if (paired) {  // 64 rows of each half per CTA
              ptx::tma_load_2d_pair(b, &tmTB, bar, 0, nb + (int)rank * 64);
              ptx::tma_load_2d_pair(b + 8192, &tmTB, bar, 0, args.pair_off + nb + (int)rank * 64);
            } else {
              ptx::tma_load_2d_pair(b, &tmTB, bar, 0, n0 + (int)rank * 128);
            }
          } else {
            ptx::tma_load_2d_pair(b, &tmTB, bar, n0 + (int)rank * 128, 0);
            ptx::tma_load_2d_pair(b + 8192, &tmTB, bar, n0 + (int)rank * 128 + 64, 0);
          }
        }
      }
    }
  } else if (CG == 2 && warp == 1) {
    // ------------------------------------- MMA issuer (even CTA of the pair)
    if (rank == 0 && lane == 0) {
      constexpr uint32_t idesc_main = ptx::idesc_bf16(2 * BM, BN, 0, B_MN ? 1 : 0);
      constexpr uint32_t idesc_tail = ptx::idesc_bf16(2 * BM, BN, 1, B_MN ? 1 : 0);
      constexpr uint32_t idesc_half = ptx::idesc_bf16(2 * BM, BN / 2, 1, B_MN ? 1 : 0);
      bool ok = true;
      for (int it = 0; it < n_iters; ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (!ptx::mbar_wait_bounded(&full[s], ph, abort_flag, args.wait_limit)) {
          atomicOr(args.err, 1);
          *abort_flag = 1;
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t a_base = ptx::smem_u32(sA + s * C::A_STAGE);
        const uint32_t b_base = ptx::smem_u32(sB + s * C::B_STAGE);
        const bool tail = it >= num_kb;
        if (tail && paired) {
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const uint64_t ad = ptx::smem_desc_sw128(a_base + hf * 2048, 8192, 1024);
            const uint64_t bd = ptx::smem_desc_sw128(b_base + hf * 8192, 16, 1024);
            ptx::mma_bf16_pair(tmem + hf * (BN / 2), ad, bd, idesc_half, 1u);
          }
        } else {
          const int nk = tail ? args.tail_ksteps : BKE / KI;
          for (int k = 0; k < nk; ++k) {
            const uint64_t ad = tail ? ptx::smem_desc_sw128(a_base + k * KSTEP_MN, CHUNK_BYTES, 1024)
                                     : ptx::smem_desc_sw128(a_base + k * 32, 16, 1024);
            const uint64_t bd = B_MN ? ptx::smem_desc_sw128(b_base + k * KSTEP_MN, CHUNK_BYTES, 1024)
                                     : ptx::smem_desc_sw128(b_base + k * 32, 16, 1024);
            ptx::mma_bf16_pair(tmem, ad, bd, tail ? idesc_tail : idesc_main, (it > 0 || k > 0) ? 1u : 0u);
            if (DUAL && !tail)  // lo part of A against the same B tile
              ptx::mma_bf16_pair(tmem, ptx::smem_desc_sw128(a_base + A_STAGE_BYTES + k * 32, 16, 1024), bd, idesc_main,
                                 1u);
          }
        }
        ptx::mma_commit_pair(&empty[s], 3);
      }
      if (ok) ptx::mma_commit_pair(accf, 3);
    }
  } else if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && !args.skip_producer) {
      for (int it = 0; it < n_iters; ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (!ptx::mbar_wait_bounded(&empty[s], ph ^ 1, abort_flag, args.wait_limit)) {
          atomicOr(args.err, 1);
          *abort_flag = 1;
          break;
        }
        uint8_t* a = sA + s * C::A_STAGE;
        uint8_t* b = sB + s * C::B_STAGE;
        const bool tail = it >= num_kb;
        const uint32_t bytes = ((DUAL && !tail) ? C::A_STAGE : A_STAGE_BYTES) + ((!NF4 || tail) ? C::B_STAGE : 0);
        ptx::mbar_arrive_expect_tx(&full[s], bytes);
        if (!tail) {
          const int k0 = (kz + it) * BKE;
          if (AMJ == A_K) {
            ptx::tma_load_2d(a, &tmA, &full[s], k0, m0);
            if (DUAL) ptx::tma_load_2d(a + A_STAGE_BYTES, &tmA2, &full[s], k0, m0);
          } else {
#pragma unroll
            for (int c = 0; c < BM / CW; ++c) ptx::tma_load_2d(a + c * CHUNK_BYTES, &tmA, &full[s], m0 + c * CW, k0);
          }
          if (!NF4) {
            if (!B_MN) {
              if (paired) {
                ptx::tma_load_2d(b, &tmB, &full[s], k0, nb);
                ptx::tma_load_2d(b + (BN / 2) * 128, &tmB, &full[s], k0, args.pair_off + nb);
              } else {
                ptx::tma_load_2d(b, &tmB, &full[s], k0, n0);
              }
            } else {
#pragma unroll
              for (int c = 0; c < BN / 64; ++c) ptx::tma_load_2d(b + c * 8192, &tmB, &full[s], n0 + 64 * c, k0);
            }
          }
        } else {
          ptx::tma_load_2d(a, &tmTA, &full[s], m0, tail_row);
          ptx::tma_load_2d(a + 8192, &tmTA, &full[s], m0 + 64, tail_row);
          if (!B_MN) {
            if (paired) {
              ptx::tma_load_2d(b, &tmTB, &full[s], 0, nb);
              ptx::tma_load_2d(b + (BN / 2) * 128, &tmTB, &full[s], 0, args.pair_off + nb);
            } else {
              ptx::tma_load_2d(b, &tmTB, &full[s], 0, n0);
            }
          } else {
#pragma unroll
            for (int c = 0; c < (BN >= 64 ? BN / 64 : 1); ++c)
              ptx::tma_load_2d(b + c * 8192, &tmTB, &full[s], n0 + 64 * c, 0);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_main = ptx::idesc_fmt(BM, BN, AMJ, B_MN ? 1 : 0, TF ? 2u : 1u);
      constexpr uint32_t idesc_tail = ptx::idesc_bf16(BM, BN, 1, B_MN ? 1 : 0);
      constexpr uint32_t idesc_half = ptx::idesc_bf16(BM, BN >= 32 ? BN / 2 : BN, 1, B_MN ? 1 : 0);
      bool ok = true;
      for (int it = 0; it < n_iters; ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (!ptx::mbar_wait_bounded(&full[s], ph, abort_flag, args.wait_limit)) {
          atomicOr(args.err, 1);
          *abort_flag = 1;
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t a_base = ptx::smem_u32(sA + s * C::A_STAGE);
        const uint32_t b_base = ptx::smem_u32(sB + s * C::B_STAGE);
        const bool tail = it >= num_kb;
        if (tail && paired) {
          // two half-width MMAs: adapter rows [0,16) for the first half of
          // the tile, [16,32) for the second
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const uint64_t ad = ptx::smem_desc_sw128(a_base + hf * 2048, 8192, 1024);
            const uint64_t bd = ptx::smem_desc_sw128(b_base + hf * (BN / 2) * 128, 16, 1024);
            ptx::mma_bf16(tmem + hf * (BN / 2), ad, bd, idesc_half, 1u);
          }
        } else {
          const int nk = tail ? args.tail_ksteps : BKE / KI;
          const bool a_mn = tail || AMJ == A_MN;
          for (int k = 0; k < nk; ++k) {
            uint64_t ad;
            if constexpr (TF)  // MN-major tf32: 32-byte-atom swizzle, 4-row period (SBO 512 B)
              ad = a_mn ? ptx::smem_desc_sw128_32b(a_base + k * KSTEP_MN, CHUNK_BYTES, 512)
                        : ptx::smem_desc_sw128(a_base + k * 32, 16, 1024);
            else
              ad = a_mn ? ptx::smem_desc_sw128(a_base + k * KSTEP_MN, CHUNK_BYTES, 1024)
                        : ptx::smem_desc_sw128(a_base + k * 32, 16, 1024);
            const uint64_t bd = B_MN ? ptx::smem_desc_sw128(b_base + k * KSTEP_MN, CHUNK_BYTES, 1024)
                                     : ptx::smem_desc_sw128(b_base + k * 32, 16, 1024);
            if constexpr (TF)
              ptx::mma_tf32(tmem, ad, bd, idesc_main, (it > 0 || k > 0) ? 1u : 0u);
            else
              ptx::mma_bf16(tmem, ad, bd, tail ? idesc_tail : idesc_main, (it > 0 || k > 0) ? 1u : 0u);
            if constexpr (DUAL) {
              if (!tail) {  // lo part of A against the same B tile
                const uint64_t ad2 = ptx::smem_desc_sw128(a_base + A_STAGE_BYTES + k * 32, 16, 1024);
                ptx::mma_bf16(tmem, ad2, bd, idesc_main, 1u);
              }
            }
          }
        }
        ptx::mma_commit(&empty[s]);
      }
      if (ok) ptx::mma_commit(accf);
    }
  } else {
    const int t = threadIdx.x - 64;  // 0 .. (NF4 ? 255 : 127)
    if constexpr (NF4 && CG == 2) {
      // ------------------------------------------ NF4 decode warps (CTA pair)
      // This CTA decodes its 128 of the tile's 256 B rows (K-major: weight
      // rows; transposed: weight columns); each thread one 32-element run
      // per stage (one absmax), codes of stage it+1 prefetched in registers.
      // Arrivals go to the even CTA's full barrier.
      const uint32_t full0 = ptx::mapa_shared(ptx::smem_u32(full), 0);
      const uint32_t lane_b = C::LUT_LANES == 32 ? (uint32_t)lane * 8u : (uint32_t)(lane & 15) * 16u;
      const uint8_t* lutb = smem_raw;
      // thread -> (shared row of the B stage, first 16-byte unit, chunk),
      // its 16 code bytes within the staged codes tile, and its absmax
      // within the staged absmax box (fp32 index)
      int srow, unit0, chunk, coff, soff;
      bool valid;
      if constexpr (BMD == B_NF4_K) {
        const int row = t >> 1, h = t & 1;
        const int n = paired ? (rank == 0 ? nb + row : args.pair_off + nb + row) : n0 + (int)rank * 128 + row;
        valid = n < args.N;
        srow = row;
        unit0 = h * 4;
        chunk = 0;
        coff = row * 32 + h * 16;
        soff = row * 4;  // + (it & 3)
      } else {
        const int q = t & 3, kr = t >> 2;
        const int col = n0 + (int)rank * 128 + q * 32;
        valid = col < args.N;
        srow = kr;
        unit0 = (q & 1) * 4;
        chunk = q >> 1;
        coff = kr * 64 + q * 16;
        soff = kr * 4 + ((n0 + (int)rank * 128) / 64 & 3) + (q >> 1);
      }
      uint8_t* const drow = sB + chunk * 8192 + srow * 128;
      for (int it = 0; it < n_iters; ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (!ptx::mbar_wait_bounded(&empty[s], ph ^ 1, abort_flag, args.wait_limit)) {
          atomicOr(args.err, 1);
          *abort_flag = 1;
          break;
        }
        if (it < num_kb) {
          if (!ptx::mbar_wait_bounded(&cfull[s], ph, abort_flag, args.wait_limit)) {
            atomicOr(args.err, 1);
            *abort_flag = 1;
            break;
          }
          const uint4 w = *reinterpret_cast<const uint4*>(sC + s * C::C_STAGE + coff);
          const float am =
              reinterpret_cast<const float*>(sS + s * C::S_STAGE)[soff + (BMD == B_NF4_K ? (it & 3) : 0)];
          uint8_t* b = drow + s * C::B_STAGE;
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const uint4 v = valid ? decode8_pairs<C::LUT_LANES>(ws[u], lutb, lane_b, am) : make_uint4(0, 0, 0, 0);
            st_shared_v4(b + (((unit0 + u) ^ (srow & 7)) << 4), v);
          }
          ptx::fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_cluster(full0 + s * 8);
      }
    } else if constexpr (NF4) {
      // ----------------------------------------------------- NF4 decode warps
      // Each thread decodes one row-segment of the B tile per stage; the
      // codes of stage it+1 are loaded into registers while stage it is
      // decoded, so the global-load latency overlaps the decode.
      const float* lut_lane = lut + lane;
      if constexpr (BMD == B_NF4_K) {
        constexpr int TPR = 256 / BN;      // threads per row
        constexpr int EPT = 64 / TPR;      // elements per thread
        constexpr int NW = EPT / 8;        // 32-bit code words per thread
        const int row = t / TPR, h = t % TPR;
        const int n = paired ? (row < BN / 2 ? nb + row : args.pair_off + nb + row - BN / 2) : n0 + row;
        const bool nvalid = n < args.N;
        const uint8_t* src = args.codes + (size_t)(nvalid ? n : 0) * (args.K / 2) + h * (EPT / 2);
        const float* amp = args.absmax + (size_t)(nvalid ? n : 0) * (args.K / 64);
        uint32_t wn[NW];
        float amn = 0.f;
        if (nvalid && num_kb > 0) {
          load_codes(src, wn);
          amn = __ldg(amp);
        }
        for (int it = 0; it < n_iters; ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          uint32_t w[NW];
#pragma unroll
          for (int u = 0; u < NW; ++u) w[u] = wn[u];
          const float am = amn;
          if (nvalid && it + 1 < num_kb) {
            load_codes(src + (size_t)(it + 1) * 32, wn);
            amn = __ldg(amp + it + 1);
          }
          if (!ptx::mbar_wait_bounded(&empty[s], ph ^ 1, abort_flag, args.wait_limit)) {
            atomicOr(args.err, 1);
            *abort_flag = 1;
            break;
          }
          if (it < num_kb) {
            uint8_t* b = sB + s * C::B_STAGE;
#pragma unroll
            for (int u = 0; u < NW; ++u) {
              const int unit = h * NW + u;
              const uint4 v = nvalid ? decode8(w[u], lut_lane, am) : make_uint4(0, 0, 0, 0);
              st_shared_v4(b + row * 128 + ((unit ^ (row & 7)) << 4), v);
            }
            ptx::fence_proxy_async_smem();
          }
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&full[s]);
        }
      } else {
        // B tile [64 k-rows, BN cols]: codes [K, N/2], absmax [K, N/64]
        constexpr int CPT = BN / 4;        // columns per thread
        constexpr int NW = CPT / 8;
        const int kr = t & 63, q = t >> 6;
        const int c0 = q * CPT;
        const uint8_t* src = args.codes + (size_t)kr * (args.N / 2) + (n0 + c0) / 2;
        const float* amp = args.absmax + (size_t)kr * (args.N / 64) + (n0 + c0) / 64;
        const size_t cstep = (size_t)BK * (args.N / 2), astep = (size_t)BK * (args.N / 64);
        uint32_t wn[NW];
        float amn = 0.f;
        if (kr < args.K && num_kb > 0) {
          load_codes(src, wn);
          amn = __ldg(amp);
        }
        for (int it = 0; it < n_iters; ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          uint32_t w[NW];
#pragma unroll
          for (int u = 0; u < NW; ++u) w[u] = wn[u];
          const float am = amn;
          const bool kvalid = it * BK + kr < args.K;
          if (it + 1 < num_kb && (it + 1) * BK + kr < args.K) {
            load_codes(src + (size_t)(it + 1) * cstep, wn);
            amn = __ldg(amp + (size_t)(it + 1) * astep);
          }
          if (!ptx::mbar_wait_bounded(&empty[s], ph ^ 1, abort_flag, args.wait_limit)) {
            atomicOr(args.err, 1);
            *abort_flag = 1;
            break;
          }
          if (it < num_kb) {
            uint8_t* b = sB + s * C::B_STAGE;
#pragma unroll
            for (int u = 0; u < NW; ++u) {
              const int col = c0 + 8 * u;
              const int chunk = col >> 6, unit = (col >> 3) & 7;
              const uint4 v = kvalid ? decode8(w[u], lut_lane, am) : make_uint4(0, 0, 0, 0);
              st_shared_v4(b + chunk * 8192 + kr * 128 + ((unit ^ (kr & 7)) << 4), v);
            }
            ptx::fence_proxy_async_smem();
          }
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&full[s]);
        }
      }
    }
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;
    const int q = warp & 3;
    const bool got = ptx::mbar_wait_bounded(accf, 0, abort_flag);
    if (!got) {
      atomicOr(args.err, 1);
      *abort_flag = 1;
    } else {
      ptx::tc_fence_after();
      epilogue_tile<BN>(args, outp, tmem, m0, n0, nb, q, lane, NEPI == 8 ? ew / 4 : 0, NEPI == 8 ? 2 : 1);
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // let copies and MMAs already in flight land before the CTA releases its
    // shared and tensor memory (bounded: ~1 ms)
    const long long t0 = clock64();
    while (clock64() - t0 < 2000000LL) {
    }
    __syncthreads();
  }
  if constexpr (CG == 2) ptx::cluster_sync();  // no CTA leaves while its pair may still signal it
  if (warp == 1) {
    ptx::tc_fence_after();
    if constexpr (CG == 2) ptx::tmem_dealloc_pair(tmem, C::TMEM_COLS);
    else ptx::tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Persistent form of the CTA-pair NF4 GEMM: each pair loops over 256x256
// output tiles (t = pair, pair + pairs, ...; M tiles fastest) with two
// accumulators in tensor memory (2 x 256 columns), so that 8 epilogue warps
// drain tile i while the MMA warp already accumulates tile i + 1.  Roles:
// warp 0 TMA producer, warp 1 TMEM owner + MMA issuer (even CTA), warps 2..9
// NF4 decode, warps 10..17 epilogue (two per TMEM lane quadrant).  The shared-memory ring, decode, tail
// K-block and epilogues are those of gemm_kernel with CTA pairs; the stage
// counter runs on across tiles and the decode table is built once.
constexpr int PERSIST_THREADS = 32 * 18;

struct PairTile {
  int m0, n0, nb, tail_row;
};

// A pair's j-th work item: a whole tile, or (last partial round split along
// K) k-blocks [kb0, kb1) of a leftover tile; unit >= 0 for a slice.
struct PairItem {
  int t, kb0, kb1, unit;
};
__device__ __forceinline__ int pair_items(const KArgs& a, int pair, int npairs, int ntiles_total) {
  if (a.sk_k > 1) return a.sk_full + (pair < a.sk_units ? (a.sk_units - pair + npairs - 1) / npairs : 0);
  return pair < ntiles_total ? (ntiles_total - pair + npairs - 1) / npairs : 0;
}
__device__ __forceinline__ PairItem pair_item(const KArgs& a, int j, int pair, int npairs) {
  PairItem w;
  if (a.sk_k > 1 && j >= a.sk_full) {
    const int u = pair + (j - a.sk_full) * npairs;
    const int z = u % a.sk_k;
    w.t = a.sk_full * npairs + u / a.sk_k;
    w.kb0 = (int)((long long)z * a.num_kb / a.sk_k);
    w.kb1 = (int)((long long)(z + 1) * a.num_kb / a.sk_k);
    w.unit = u;
  } else {
    w.t = pair + j * npairs;
    w.kb0 = 0;
    w.kb1 = a.num_kb;
    w.unit = -1;
  }
  return w;
}

__device__ __forceinline__ PairTile pair_tile(const KArgs& args, int t, int mtiles, uint32_t rank) {
  constexpr int BN = 256;
  PairTile p;
  const int mt = t % mtiles, nt = t / mtiles;
  p.m0 = mt * 256 + (int)rank * 128;
  const bool paired = args.pair_off > 0;
  p.nb = paired ? nt * (BN / 2) : nt * BN;
  p.n0 = p.nb;
  int tr = args.seg_row[0];
  if (args.nseg > 1 && p.n0 >= args.seg_end[0]) tr = args.seg_row[1];
  if (args.nseg > 2 && p.n0 >= args.seg_end[1]) tr = args.seg_row[2];
  if (args.nseg > 3 && p.n0 >= args.seg_end[2]) tr = args.seg_row[3];
  p.tail_row = paired ? 0 : tr;
  return p;
}

template <int BMD, bool DUAL>
__global__ void __launch_bounds__(PERSIST_THREADS, 1)
    gemm_pair_persistent(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                         const __grid_constant__ CUtensorMap tmTA, const __grid_constant__ CUtensorMap tmTB,
                         const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmA3,
                         const KArgs args, int mtiles, int ntiles_total) {
  constexpr int BN = 256;
  constexpr bool NF4 = BMD >= B_NF4_K;  // else bf16 B tiles by TMA, no decode
  using C = Cfg<BN, DUAL, 2, NF4>;
  constexpr bool B_MN = BMD == B_NF4_MN || BMD == B_TMA_MN;
  constexpr int STAGES = C::STAGES;
  constexpr int KSTEP_MN = 16 * 128;
  constexpr int CHUNK_BYTES = 64 * 128;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw + C::LUT_BYTES) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * C::A_STAGE;
  uint8_t* sC = sB + STAGES * C::B_STAGE;
  uint8_t* sS = sC + STAGES * C::C_STAGE;
  uint64_t* full = reinterpret_cast<uint64_t*>(sS + STAGES * C::S_STAGE);
  uint64_t* empty = full + STAGES;
  uint64_t* cfull = empty + STAGES;
  uint64_t* acc_full = cfull + STAGES;   // [2] MMA of a tile done (both CTAs, multicast commit)
  uint64_t* acc_empty = acc_full + 2;    // [2] even CTA: both CTAs' epilogues drained the buffer
  uint64_t* sk_done = acc_empty + 2;     // split slice: the 8 epilogue warps stored their partial
  uint64_t* sk_go = sk_done + 1;         // split slice: whether this CTA sums the tile was decided
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sk_go + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* sk_last = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int num_kb = args.num_kb;
  const bool paired = args.pair_off > 0;
  const int nitems = pair_items(args, pair, npairs, ntiles_total);
  // iterations of an item: its k-blocks, plus the LoRA tail step for the
  // item that ends the tile's K range
  auto item_end = [&](const PairItem& w) { return w.kb1 + ((args.tail_ksteps > 0 && w.kb1 == num_kb) ? 1 : 0); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(&full[s], NF4 ? 1 + 16 : 1);
      ptx::mbar_init(&empty[s], 1);
      ptx::mbar_init(&cfull[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&acc_full[b], 1);
      ptx::mbar_init(&acc_empty[b], 16);
    }
    ptx::mbar_init(sk_done, 8);
    ptx::mbar_init(sk_go, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tmA);
    ptx::prefetch_tmap(&tmB);
    if (NF4) ptx::prefetch_tmap(&tmA2);
    if (DUAL) ptx::prefetch_tmap(&tmA3);
    if (args.tail_ksteps > 0) {
      ptx::prefetch_tmap(&tmTA);
      ptx::prefetch_tmap(&tmTB);
    }
  }
  if (NF4 && warp >= 2 && warp < 10) {
    float2* lut2 = reinterpret_cast<float2*>(smem_raw);
    for (int i = threadIdx.x - 64; i < 256 * C::LUT_LANES; i += 256) {
      const int b = i / C::LUT_LANES;
      lut2[i] = make_float2(__uint_as_float(c_nf4_bits[b >> 4]), __uint_as_float(c_nf4_bits[b & 15]));
    }
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(tmem_slot, 512);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  ptx::cluster_sync();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint32_t full0 = ptx::mapa_shared(ptx::smem_u32(full), 0);
      int gi = 0;
      bool ok = true;
      for (int j = 0; j < nitems && ok; ++j) {
        const PairItem wi = pair_item(args, j, pair, npairs);
        const PairTile tl = pair_tile(args, wi.t, mtiles, rank);
        const int r0 = paired ? (rank == 0 ? tl.nb : args.pair_off + tl.nb) : tl.n0 + (int)rank * 128;
        const int c0 = tl.n0 + (int)rank * 128;
        const int it_end = item_end(wi);
        for (int it = wi.kb0; it < it_end; ++it, ++gi) {
          const int s = gi % STAGES;
          const uint32_t ph = (gi / STAGES) & 1;
          if (!ptx::mbar_wait_bounded(&empty[s], ph ^ 1, abort_flag)) {
            atomicOr(args.err, 1);
            *abort_flag = 1;
            ok = false;
            break;
          }
          uint8_t* a = sA + s * C::A_STAGE;
          uint8_t* b = sB + s * C::B_STAGE;
          const bool tail = it >= num_kb;
          const uint32_t bytes = tail ? (uint32_t)(A_STAGE_BYTES + C::B_STAGE)
                                      : (uint32_t)(C::A_STAGE + (NF4 ? 0 : C::B_STAGE));
          if (rank == 0) ptx::mbar_arrive_expect_tx(&full[s], 2 * bytes);
          const uint32_t bar = full0 + s * 8;
          if (!tail) {
            ptx::tma_load_2d_pair(a, &tmA, bar, it * BK, tl.m0);
            if (DUAL) ptx::tma_load_2d_pair(a + A_STAGE_BYTES, &tmA3, bar, it * BK, tl.m0);
            if constexpr (!NF4) {
              // bf16 B: this CTA's 128 rows (K-major; paired tiles: its half
              // of the pair) or 128 columns as two 64-wide chunks (MN-major)
              if constexpr (!B_MN) {
                ptx::tma_load_2d_pair(b, &tmB, bar, it * BK, r0);
              } else {
                ptx::tma_load_2d_pair(b, &tmB, bar, c0, it * BK);
                ptx::tma_load_2d_pair(b + 8192, &tmB, bar, c0 + 64, it * BK);
              }
              continue;
            }
            uint8_t* c = sC + s * C::C_STAGE;
            uint8_t* sc = sS + s * C::S_STAGE;
            const int ip = it + 12;
            ptx::mbar_arrive_expect_tx(&cfull[s], (uint32_t)(C::C_STAGE + (B_MN ? 1024 : 2048)));
            if (!B_MN) {
              ptx::tma_load_2d(c, &tmB, &cfull[s], it * 32, r0);
              ptx::tma_load_2d(sc, &tmA2, &cfull[s], it & ~3, r0);
              if (ip < num_kb) {
                ptx::tma_prefetch_l2_2d(&tmB, ip * 32, r0);
                if ((ip & 3) == 0) ptx::tma_prefetch_l2_2d(&tmA2, ip, r0);
              }
            } else {
              ptx::tma_load_2d(c, &tmB, &cfull[s], c0 / 2, it * BK);
              ptx::tma_load_2d(sc, &tmA2, &cfull[s], (c0 / 64) & ~3, it * BK);
              if (ip < num_kb) {
                ptx::tma_prefetch_l2_2d(&tmB, c0 / 2, ip * BK);
                ptx::tma_prefetch_l2_2d(&tmA2, (c0 / 64) & ~3, ip * BK);
              }
            }
          } else {
            if (NF4) ptx::mbar_arrive(&cfull[s]);  // keeps cfull's phase in step with the slot's uses
            ptx::tma_load_2d_pair(a, &tmTA, bar, tl.m0, tl.tail_row);
            ptx::tma_load_2d_pair(a + 8192, &tmTA, bar, tl.m0 + 64, tl.tail_row);
            if (!B_MN) {
              if (paired) {
                ptx::tma_load_2d_pair(b, &tmTB, bar, 0, tl.nb + (int)rank * 64);
                ptx::tma_load_2d_pair(b + 8192, &tmTB, bar, 0, args.pair_off + tl.nb + (int)rank * 64);
              } else {
                ptx::tma_load_2d_pair(b, &tmTB, bar, 0, tl.n0 + (int)rank * 128);
              }
            } else {
              ptx::tma_load_2d_pair(b, &tmTB, bar, c0, 0);
              ptx::tma_load_2d_pair(b + 8192, &tmTB, bar, c0 + 64, 0);
            }
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------- MMA issuer (even CTA of the pair)
    if (rank == 0 && lane == 0) {
      constexpr uint32_t idesc_main = ptx::idesc_bf16(2 * BM, BN, 0, B_MN ? 1 : 0);
      constexpr uint32_t idesc_tail = ptx::idesc_bf16(2 * BM, BN, 1, B_MN ? 1 : 0);
      constexpr uint32_t idesc_half = ptx::idesc_bf16(2 * BM, BN / 2, 1, B_MN ? 1 : 0);
      int gi = 0, lt = 0;
      bool ok = true;
      for (int j = 0; j < nitems && ok; ++j, ++lt) {
        const PairItem wi = pair_item(args, j, pair, npairs);
        const int it_end = item_end(wi);
        const int ab = lt & 1;
        if (!ptx::mbar_wait_bounded(&acc_empty[ab], ((lt >> 1) & 1) ^ 1, abort_flag)) {
          atomicOr(args.err, 1);
          *abort_flag = 1;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t tacc = tmem + (uint32_t)(ab * BN);
        for (int it = wi.kb0; it < it_end; ++it, ++gi) {
          const int s = gi % STAGES;
          const uint32_t ph = (gi / STAGES) & 1;
          if (!ptx::mbar_wait_bounded(&full[s], ph, abort_flag)) {
            atomicOr(args.err, 1);
            *abort_flag = 1;
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t a_base = ptx::smem_u32(sA + s * C::A_STAGE);
          const uint32_t b_base = ptx::smem_u32(sB + s * C::B_STAGE);
          const bool tail = it >= num_kb;
          if (tail && paired) {
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              const uint64_t ad = ptx::smem_desc_sw128(a_base + hf * 2048, 8192, 1024);
              const uint64_t bd = ptx::smem_desc_sw128(b_base + hf * 8192, 16, 1024);
              ptx::mma_bf16_pair(tacc + hf * (BN / 2), ad, bd, idesc_half, 1u);
            }
          } else {
            const int nk = tail ? args.tail_ksteps : 4;
            for (int k = 0; k < nk; ++k) {
              const uint64_t ad = tail ? ptx::smem_desc_sw128(a_base + k * KSTEP_MN, CHUNK_BYTES, 1024)
                                       : ptx::smem_desc_sw128(a_base + k * 32, 16, 1024);
              const uint64_t bd = B_MN ? ptx::smem_desc_sw128(b_base + k * KSTEP_MN, CHUNK_BYTES, 1024)
                                       : ptx::smem_desc_sw128(b_base + k * 32, 16, 1024);
              ptx::mma_bf16_pair(tacc, ad, bd, tail ? idesc_tail : idesc_main, (it > wi.kb0 || k > 0) ? 1u : 0u);
              if (DUAL && !tail)
                ptx::mma_bf16_pair(tacc, ptx::smem_desc_sw128(a_base + A_STAGE_BYTES + k * 32, 16, 1024), bd,
                                   idesc_main, 1u);
            }
          }
          ptx::mma_commit_pair(&empty[s], 3);
        }
        if (ok) ptx::mma_commit_pair(&acc_full[ab], 3);
      }
    }
  } else if (warp < 10) {
    // ----------------------------------------------------- NF4 decode warps
    // (bf16 B: the TMA brings the B tiles, these warps have nothing to do)
    if constexpr (NF4) {
    const int td = threadIdx.x - 64;
    const uint32_t full0 = ptx::mapa_shared(ptx::smem_u32(full), 0);
    const uint32_t lane_b = C::LUT_LANES == 32 ? (uint32_t)lane * 8u : (uint32_t)(lane & 15) * 16u;
    const uint8_t* lutb = smem_raw;
    int gi = 0;
    bool ok = true;
    for (int j = 0; j < nitems && ok; ++j) {
      const PairItem wi = pair_item(args, j, pair, npairs);
      const PairTile tl = pair_tile(args, wi.t, mtiles, rank);
      const int it_end = item_end(wi);
      int srow, unit0, chunk, coff, soff;
      bool valid;
      if constexpr (BMD == B_NF4_K) {
        const int row = td >> 1, h = td & 1;
        const int n = paired ? (rank == 0 ? tl.nb + row : args.pair_off + tl.nb + row) : tl.n0 + (int)rank * 128 + row;
        valid = n < args.N;
        srow = row;
        unit0 = h * 4;
        chunk = 0;
        coff = row * 32 + h * 16;
        soff = row * 4;
      } else {
        const int q = td & 3, kr = td >> 2;
        const int col = tl.n0 + (int)rank * 128 + q * 32;
        valid = col < args.N;
        srow = kr;
        unit0 = (q & 1) * 4;
        chunk = q >> 1;
        coff = kr * 64 + q * 16;
        soff = kr * 4 + ((tl.n0 + (int)rank * 128) / 64 & 3) + (q >> 1);
      }
      uint8_t* const drow = sB + chunk * 8192 + srow * 128;
      for (int it = wi.kb0; it < it_end; ++it, ++gi) {
        const int s = gi % STAGES;
        const uint32_t ph = (gi / STAGES) & 1;
        // cfull completes once per use of the slot (the tail stage arrives without bytes)
        if (!ptx::mbar_wait_bounded(&empty[s], ph ^ 1, abort_flag) ||
            !ptx::mbar_wait_bounded(&cfull[s], ph, abort_flag)) {
          atomicOr(args.err, 1);
          *abort_flag = 1;
          ok = false;
          break;
        }
        if (it < num_kb) {
          const uint4 w = *reinterpret_cast<const uint4*>(sC + s * C::C_STAGE + coff);
          const float am =
              reinterpret_cast<const float*>(sS + s * C::S_STAGE)[soff + (BMD == B_NF4_K ? (it & 3) : 0)];
          uint8_t* b = drow + s * C::B_STAGE;
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const uint4 v = valid ? decode8_pairs<C::LUT_LANES>(ws[u], lutb, lane_b, am) : make_uint4(0, 0, 0, 0);
            st_shared_v4(b + (((unit0 + u) ^ (srow & 7)) << 4), v);
          }
          ptx::fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_cluster(full0 + s * 8);
      }
    }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // warps 10..17 own TMEM lane quadrants 2, 3, 0, 1 (twice); each drains
    // every other 16-column chunk of its 32 rows, then frees the buffer on
    // the even CTA
    const int q = warp & 3, ew = warp - 10;
    const uint32_t acc_empty0 = ptx::mapa_shared(ptx::smem_u32(acc_empty), 0);
    int lt = 0, ns = 0;  // ns: slices handled (phase of sk_done / sk_go)
    for (int j = 0; j < nitems; ++j, ++lt) {
      const PairItem wi = pair_item(args, j, pair, npairs);
      const PairTile tl = pair_tile(args, wi.t, mtiles, rank);
      const int ab = lt & 1;
      if (!ptx::mbar_wait_bounded(&acc_full[ab], (lt >> 1) & 1, abort_flag)) {
        atomicOr(args.err, 1);
        *abort_flag = 1;
        break;
      }
      ptx::tc_fence_after();
      const uint32_t tacc = tmem + (uint32_t)(ab * BN);
      if (wi.unit < 0) {
        epilogue_tile<BN>(args, args.out, tacc, tl.m0, tl.n0, tl.nb, q, lane, ew / 4, 2);
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_cluster(acc_empty0 + ab * 8);
        continue;
      }
      // ---- k-slice of a split tile: store this CTA's partial (column-major),
      // free the accumulator, count the slice; the last of the tile's slices
      // to finish sums all of them (slice order) and runs the epilogue
      const int u0 = wi.unit - wi.unit % args.sk_k;  // the tile's first slice
      {
        float* part = args.sk_ws + ((size_t)wi.unit * 2 + rank) * SK_HALF + q * 32 + lane;
        const uint32_t trow = tacc + ((uint32_t)(q * 32) << 16);
        for (int ch = ew / 4; ch < BN / 16; ch += 2) {
          uint32_t v[16];
          ptx::tmem_ld16(trow + ch * 16, v);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) __stcg(part + (size_t)(ch * 16 + i) * 128, __uint_as_float(v[i]));
        }
      }
      __threadfence();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        ptx::mbar_arrive_cluster(acc_empty0 + ab * 8);
        ptx::mbar_arrive(sk_done);
      }
      if (ew == 0 && lane == 0) {
        int last = 0;
        if (ptx::mbar_wait_bounded(sk_done, (uint32_t)(ns & 1), abort_flag, args.wait_limit)) {
          // count this CTA's slice on the tile's (epoch-tagged) counter
          unsigned long long* cnt = args.sk_cnt + (size_t)(wi.unit / args.sk_k) * 2 + rank;
          unsigned long long old = *reinterpret_cast<volatile unsigned long long*>(cnt), nw;
          while (true) {
            nw = (unsigned int)(old >> 32) == args.sk_epoch ? old + 1
                                                             : (((unsigned long long)args.sk_epoch << 32) | 1ull);
            const unsigned long long prev = atomicCAS(cnt, old, nw);
            if (prev == old) break;
            old = prev;
          }
          last = (int)(nw & 0xFFFFFFFFull) == args.sk_k ? 1 : 0;
          __threadfence();
        } else {
          atomicOr(args.err, 1);
          *abort_flag = 1;
          last = -1;
        }
        *sk_last = last;
        ptx::mbar_arrive(sk_go);
      }
      if (!ptx::mbar_wait_bounded(sk_go, (uint32_t)(ns & 1), abort_flag, args.wait_limit)) {
        atomicOr(args.err, 1);
        *abort_flag = 1;
        break;
      }
      ++ns;
      if (*sk_last == 1) {
        __threadfence();
        epilogue_tile<BN>(args, args.out, tacc, tl.m0, tl.n0, tl.nb, q, lane, ew / 4, 2,
                          args.sk_ws + ((size_t)u0 * 2 + rank) * SK_HALF, args.sk_k);
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    const long long t0 = clock64();
    while (clock64() - t0 < 2000000LL) {
    }
    __syncthreads();
  }
  ptx::cluster_sync();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem, 512);
  }
}

// Split-K epilogue: out = alpha * sum over slices (in slice order) of the
// fp32 partial products ws[z] ([M, N], or [N, M] for a transposed output),
// stored as the GEMM's own epilogue would.
__global__ void splitk_reduce_kernel(const float* __restrict__ ws, int splits, int M, int N, int out_kind,
                                     void* out, float* out2, uint16_t* out_lo, long long ldo, float alpha,
                                     const unsigned int* scale_amax) {
  const float a = scale_amax ? alpha * grad_scale_from_amax(__uint_as_float(*scale_amax)) : alpha;
  const bool tr = out_kind == OUT_BF16_T || out_kind == OUT_F32_T;
  const size_t total = (size_t)M * N, plane = (size_t)M * N;
  for (size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total; idx += (size_t)gridDim.x * blockDim.x) {
    // transposed outputs: consecutive threads take consecutive rows m
    const int m = tr ? (int)(idx % M) : (int)(idx / N);
    const int n = tr ? (int)(idx / M) : (int)(idx % N);
    float acc = 0.f;
    const size_t pi = tr ? (size_t)n * M + m : (size_t)m * N + n;  // planes are [N, M] for transposed outputs
    for (int z = 0; z < splits; ++z) acc += ws[z * plane + pi];
    const float v = acc * a;
    const size_t o = tr ? (size_t)n * ldo + m : (size_t)m * ldo + n;
    if (out_kind == OUT_F32 || out_kind == OUT_F32_T) {
      static_cast<float*>(out)[o] = v;
    } else {
      const uint32_t w = out_kind == OUT_F16 ? pack_f16x2(v, 0.f) : pack_bf16x2(v, 0.f);
      static_cast<uint16_t*>(out)[o] = static_cast<uint16_t>(w & 0xFFFF);
      if (out2 && out_kind == OUT_BF16_T) out2[o] = v;
      if (out_lo && out_kind == OUT_BF16_T)
        out_lo[o] = static_cast<uint16_t>(pack_bf16x2(v - bf16_to_f32(static_cast<uint16_t>(w & 0xFFFF)), 0.f) & 0xFFFF);
    }
  }
}

// ----------------------------------------------------------------- host side
constexpr int CU_DT_BF16 = 9;       // CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
constexpr int CU_SWIZZLE_128B = 3;  // CU_TENSOR_MAP_SWIZZLE_128B
constexpr int CU_L2_256B = 3;       // CU_TENSOR_MAP_L2_PROMOTION_L2_256B

constexpr int CU_DT_F32 = 7;        // CU_TENSOR_MAP_DATA_TYPE_FLOAT32
constexpr int CU_SWIZZLE_128B_ATOM_32B = 4;  // 32-byte chunks within a 128-byte span

soup_status make_map(CUtensorMap* m, const Mat& mat, uint32_t box0, uint32_t box1, const char* what,
                     bool f32 = false, int swizzle = CU_SWIZZLE_128B) {
  const int es = f32 ? 4 : 2;
  SOUP_CHECK(mat.ptr && mat.rows > 0 && mat.cols > 0, SOUP_ERR_INVALID_ARG, "gemm: %s is empty", what);
  SOUP_CHECK(soup_aligned(mat.ptr, 16), SOUP_ERR_ALIGN, "gemm: %s base not 16-byte aligned", what);
  SOUP_CHECK((mat.ld * es) % 16 == 0 && mat.ld >= mat.cols, SOUP_ERR_ALIGN,
             "gemm: %s row stride %lld elements is not a multiple of 16 bytes (or < cols)", what,
             (long long)mat.ld);
  EncodeTiledFn enc = encode_tiled();
  SOUP_CHECK(enc != nullptr, SOUP_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const uint64_t gdim[2] = {(uint64_t)mat.cols, (uint64_t)mat.rows};
  const uint64_t gstride[1] = {(uint64_t)mat.ld * es};
  const uint32_t box[2] = {box0, box1};
  const uint32_t estr[2] = {1, 1};
  int r = enc(m, f32 ? CU_DT_F32 : CU_DT_BF16, 2, const_cast<void*>(mat.ptr), gdim, gstride, box, estr, 0,
              swizzle, CU_L2_256B, 0);
  SOUP_CHECK(r == 0, SOUP_ERR_CUDA, "cuTensorMapEncodeTiled(%s) failed with %d", what, r);
  return SOUP_OK;
}

// Un-swizzled tensor map over a row-major [rows, cols] array of 1- or 4-byte
// elements (the NF4 codes / absmax staging of the pair kernels).
soup_status make_plain_map(CUtensorMap* m, const void* ptr, int64_t rows, int64_t cols, int es, int dtype,
                           uint32_t box0, uint32_t box1, const char* what) {
  SOUP_CHECK(ptr && rows > 0 && cols > 0, SOUP_ERR_INVALID_ARG, "gemm: %s is empty", what);
  SOUP_CHECK(soup_aligned(ptr, 16), SOUP_ERR_ALIGN, "gemm: %s base not 16-byte aligned", what);
  SOUP_CHECK((cols * es) % 16 == 0, SOUP_ERR_ALIGN, "gemm: %s row of %lld bytes is not a multiple of 16", what,
             (long long)(cols * es));
  EncodeTiledFn enc = encode_tiled();
  SOUP_CHECK(enc != nullptr, SOUP_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const uint64_t gdim[2] = {(uint64_t)cols, (uint64_t)rows};
  const uint64_t gstride[1] = {(uint64_t)(cols * es)};
  const uint32_t box[2] = {box0, box1};
  const uint32_t estr[2] = {1, 1};
  int r = enc(m, dtype, 2, const_cast<void*>(ptr), gdim, gstride, box, estr, 0, 0 /* no swizzle */, CU_L2_256B, 0);
  SOUP_CHECK(r == 0, SOUP_ERR_CUDA, "cuTensorMapEncodeTiled(%s) failed with %d", what, r);
  return SOUP_OK;
}
constexpr int CU_DT_U8 = 0;  // CU_TENSOR_MAP_DATA_TYPE_UINT8

// Per-device slice counters of the persistent kernel's split last round
// (one per leftover tile and CTA of the pair, tagged with a launch-unique
// epoch, so none ever needs clearing).
constexpr int SK_MAX_TILES = 128;
__device__ __align__(256) unsigned long long g_sk_cnt[2 * SK_MAX_TILES];
std::atomic<unsigned int> g_sk_epoch{0};

// The split of the last partial round: leftover tiles L after the full
// rounds on P pairs are cut into k slices (2 <= k <= 8, >= 64 k-blocks
// each: a slice pays a pipeline fill, a 128 KB partial store per CTA and
// its share of the sums) handed round-robin to the pairs; picked to
// minimise the rounds the leftover then takes, ceil(L k / P) / k of a tile,
// if that saves at least a tenth of a tile and the partials (L k x 256 KB)
// fit the scratch.
int pick_split(int total, int P, int num_kb, size_t scratch_bytes) {
  const int F = total / P, L = total - F * P;
  if (L == 0 || L > SK_MAX_TILES) return 0;
  int best = 0;
  double best_cost = 0.9;
  for (int k = 2; k <= 8; ++k) {
    if (num_kb / k < 64) break;
    if ((size_t)L * k * 2 * 256 * 128 * sizeof(float) > scratch_bytes) break;
    const double cost = (double)((L * k + P - 1) / P) / k + 0.01 * k;  // + a little per slice for the sums
    if (cost < best_cost) {
      best_cost = cost;
      best = k;
    }
  }
  return best;
}

template <int BN, int AMJ, int BMD, bool TF = false, bool DUAL = false, int CG = 1, bool PERSIST = false>
soup_status launch(const GemmDesc& d, const KArgs& ka, cudaStream_t st) {
  static_assert(!PERSIST || (CG == 2 && BN == 256 && AMJ == A_K && !TF), "persistent: CTA pairs, K-major A");
  using C = Cfg<BN, DUAL, CG, (CG == 1 || BMD >= B_NF4_K)>;
  CUtensorMap mA, mB, mTA, mTB, mA2, mA3;
  memset(&mA2, 0, sizeof(mA2));
  memset(&mA3, 0, sizeof(mA3));
  if (DUAL) SOUP_TRY(make_map(CG == 2 ? &mA3 : &mA2, d.A_lo, 64, 128, "A (lo part)"));
  memset(&mA, 0, sizeof(mA));
  memset(&mB, 0, sizeof(mB));
  memset(&mTA, 0, sizeof(mTA));
  memset(&mTB, 0, sizeof(mTB));
  const bool paired = d.pair_off > 0;
  constexpr uint32_t EW = TF ? 32 : 64;  // elements per 128-byte row
  if (AMJ == A_K) SOUP_TRY(make_map(&mA, d.A, EW, 128, "A", TF));
  else SOUP_TRY(make_map(&mA, d.A, EW, EW, "A (MN-major)", TF, TF ? CU_SWIZZLE_128B_ATOM_32B : CU_SWIZZLE_128B));
  constexpr bool B_MN = (BMD == B_TMA_MN || BMD == B_NF4_MN);
  // K-major B boxes: the tile's rows (CTA pairs: this CTA's 128 of them;
  // paired gate|up tiles: one half of the pair's rows)
  if (BMD == B_TMA_K) SOUP_TRY(make_map(&mB, d.B, EW, CG == 2 ? 128 : (paired ? BN / 2 : BN), "B", TF));
  if (BMD == B_TMA_MN) SOUP_TRY(make_map(&mB, d.B, 64, 64, "B (MN-major)"));
  if (CG == 2 && BMD >= B_NF4_K) {
    // codes and absmax staged per stage: K-major 128 rows x 32 bytes and a
    // 128 x 4 absmax box; transposed 64 k-rows x 64 bytes and a 64 x 4 box
    if (BMD == B_NF4_K) {
      SOUP_TRY(make_plain_map(&mB, d.codes, d.N, d.K / 2, 1, CU_DT_U8, 32, 128, "NF4 codes"));
      SOUP_TRY(make_plain_map(&mA2, d.absmax, d.N, d.K / 64, 4, CU_DT_F32, 4, 128, "NF4 absmax"));
    } else {
      SOUP_TRY(make_plain_map(&mB, d.codes, d.K, d.N / 2, 1, CU_DT_U8, 64, 64, "NF4 codes (transposed)"));
      SOUP_TRY(make_plain_map(&mA2, d.absmax, d.K, d.N / 64, 4, CU_DT_F32, 4, 64, "NF4 absmax (transposed)"));
    }
  }
  if (d.tail_ksteps > 0) {
    SOUP_TRY(make_map(&mTA, d.tailA, 64, 64, "tail A"));
    // K-major tail B rows per box: the tile's (CTA pairs: this CTA's half of
    // it; paired gate|up tiles: one half of the pair's half)
    if (!B_MN) SOUP_TRY(make_map(&mTB, d.tailB, 64, (paired ? BN / 2 : BN) / CG, "tail B"));
    else SOUP_TRY(make_map(&mTB, d.tailB, 64, 64, "tail B (MN-major)"));
  }
  if constexpr (PERSIST) {
    auto kp = gemm_pair_persistent<BMD, DUAL>;
    static int max_pairs = 0;  // per instantiation: co-resident CTA pairs
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.blockDim = dim3(PERSIST_THREADS);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    if (max_pairs == 0) {
      SOUP_CUDA_TRY(cudaFuncSetAttribute(kp, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM));
      cfg.gridDim = dim3(2 * (sm_count() / 2));
      int nc = 0;
      if (cudaOccupancyMaxActiveClusters(&nc, kp, &cfg) != cudaSuccess || nc <= 0) {
        cudaGetLastError();
        nc = sm_count() / 2;
      }
      max_pairs = nc;
    }
    const int mtiles = (d.M + 2 * BM - 1) / (2 * BM);
    const int ntiles = paired ? d.pair_off / (BN / 2) : (d.N + BN - 1) / BN;
    const int total = mtiles * ntiles;
    int npairs = std::min(total, max_pairs);
    KArgs kx = ka;
    kx.sk_k = 0;
    if (d.sk_scratch && d.sk_scratch_bytes > 0 && soup_aligned(d.sk_scratch, 16)) {
      const int k = pick_split(total, max_pairs, ka.num_kb, d.sk_scratch_bytes);
      if (k >= 2) {
        void* cnt = nullptr;
        SOUP_TRY(static_symbol_address(SYM_SPLIT_COUNTERS, reinterpret_cast<const void*>(g_sk_cnt), &cnt));
        const int F = total / max_pairs;
        kx.sk_full = F;
        kx.sk_units = (total - F * max_pairs) * k;
        kx.sk_k = k;
        kx.sk_ws = static_cast<float*>(d.sk_scratch);
        kx.sk_cnt = static_cast<unsigned long long*>(cnt);
        kx.sk_epoch = g_sk_epoch.fetch_add(1) + 1;
        npairs = F > 0 ? max_pairs : std::min(kx.sk_units, max_pairs);
      }
    }
    cfg.gridDim = dim3(2 * npairs);
    if (profiling()) {
      const int cls = BMD < B_NF4_K ? GC_BF16
                                    : (DUAL ? GC_NF4_DUAL : (BMD == B_NF4_K ? GC_NF4_FWD : GC_NF4_BWD));
      const double tail_k = d.tail_ksteps > 0 ? (double)d.tailA.rows : 0.0;
      const double flops = 2.0 * d.M * d.N * ((double)d.K * (DUAL ? 2 : 1) + (paired ? 16.0 : tail_k));
      const double wbytes = BMD >= B_NF4_K ? (double)d.N * d.K * (0.5 + 4.0 / 64) : (double)d.N * d.K * 2;
      const double bytes = (double)d.M * d.K * 2 + wbytes +
                           (double)d.M * d.N * ((d.out_kind == OUT_F32 || d.out_kind == OUT_F32_T) ? 4 : 2);
      profile_begin(st, cls, flops, bytes);
    }
    SOUP_CUDA_TRY(cudaLaunchKernelEx(&cfg, kp, mA, mB, mTA, mTB, mA2, mA3, kx, mtiles, total));
    SOUP_LAUNCH_CHECK();
    profile_end(st);
    return SOUP_OK;
  } else {
  auto kern = gemm_kernel<BN, AMJ, BMD, TF, DUAL, CG>;
  static bool attr_set = false;  // per instantiation
  if (!attr_set) {
    SOUP_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM));
    attr_set = true;
  }
  constexpr int NT = 32 * (2 + (BMD >= B_NF4_K ? 8 : 4));
  const int ntiles = paired ? (d.pair_off + BN / 2 - 1) / (BN / 2) : (d.N + BN - 1) / BN;
  const int nz = ka.kb_split > 0 ? (ka.num_kb + ka.kb_split - 1) / ka.kb_split : 1;
  dim3 grid(CG == 2 ? 2 * ((d.M + 2 * BM - 1) / (2 * BM)) : (d.M + BM - 1) / BM, ntiles, nz);
  if (profiling()) {
    // algorithmic work: 2 M N K (+ 2 M N r for the LoRA tail); bytes: the
    // operands read once and the output written once
    const int cls = (DUAL && BMD >= B_NF4_K) ? GC_NF4_DUAL
                    : BMD == B_NF4_K ? GC_NF4_FWD : (BMD == B_NF4_MN ? GC_NF4_BWD : (d.N <= 64 ? GC_SKINNY : GC_BF16));
    const double tail_k = d.tail_ksteps > 0 ? (double)d.tailA.rows : 0.0;
    const double flops = 2.0 * d.M * d.N * ((double)d.K * (DUAL ? 2 : 1) + (paired ? 16.0 : tail_k));
    const double wbytes = (BMD >= B_NF4_K) ? (double)d.N * d.K * (0.5 + 4.0 / 64) : (double)d.N * d.K * 2;
    const int oes = (d.out_kind == OUT_F32 || d.out_kind == OUT_F32_T) ? 4 : 2;
    const double bytes = (double)d.M * d.K * 2 + wbytes + (double)d.M * d.N * oes;
    profile_begin(st, cls, flops, bytes);
  }
  if constexpr (CG == 2) {
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = grid;
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    SOUP_CUDA_TRY(cudaLaunchKernelEx(&cfg, kern, mA, mB, mTA, mTB, mA2, mA3, ka));
  } else {
    kern<<<grid, NT, C::SMEM, st>>>(mA, mB, mTA, mTB, mA2, mA3, ka);
  }
  SOUP_LAUNCH_CHECK();
  profile_end(st);
  return SOUP_OK;
  }
}

int pick_bn(const GemmDesc& d) {
  if (d.bn) return d.bn;
  const bool nf4 = d.b_mode >= B_NF4_K;
  const bool mn = d.b_mode == B_TMA_MN || d.b_mode == B_NF4_MN;
  auto fits = [&](int bn) {
    for (int i = 0; i < d.nseg - 1; ++i)
      if (d.seg_end[i] % bn) return false;
    return true;
  };
  if (d.pair_off > 0) return 256;
  if (!nf4 && !mn && d.N <= 64) return ((d.N + 15) / 16) * 16;
  if (d.N >= 256 && (d.N % 256 == 0 || d.N >= 1024) && fits(256)) return 256;
  if (d.N >= 128 && fits(128)) return 128;
  return 64;
}

// Kernel selection for one launch (after the descriptor checks).
soup_status dispatch(const GemmDesc& d, const KArgs& ka, int bn, cudaStream_t st) {
  const bool nf4 = d.b_mode >= B_NF4_K;
  if (d.tf32) {
    SOUP_CHECK(d.b_mode == B_TMA_K && d.tail_ksteps == 0 && d.pair_off == 0 && d.epi == EPI_STORE && bn <= 64,
               SOUP_ERR_SHAPE, "gemm: tf32 mode supports skinny (N <= 64) K-major-B GEMMs without tail");
#define SOUP_GEMM_TF(BN_, AM_) \
  if (bn == BN_ && d.a_major == AM_) return launch<BN_, AM_, B_TMA_K, true>(d, ka, st);
    SOUP_GEMM_TF(64, A_K) SOUP_GEMM_TF(48, A_K) SOUP_GEMM_TF(32, A_K) SOUP_GEMM_TF(16, A_K)
    SOUP_GEMM_TF(64, A_MN) SOUP_GEMM_TF(48, A_MN) SOUP_GEMM_TF(32, A_MN) SOUP_GEMM_TF(16, A_MN)
#undef SOUP_GEMM_TF
    return fail(SOUP_ERR_SHAPE, "gemm: no tf32 kernel for BN=%d", bn);
  }
  // bf16 B with 256-wide tiles and at least one 256-row M tile: the
  // persistent CTA-pair engine with TMA-fed B (no split-K, single A)
  if (!nf4 && !d.A_lo.ptr && bn == 256 && d.a_major == A_K && d.M >= 256 && ka.kb_split == 0 && d.persistent &&
      (d.b_mode == B_TMA_K || (d.b_mode == B_TMA_MN && d.N % 256 == 0))) {
    if (d.b_mode == B_TMA_K) return launch<256, A_K, B_TMA_K, false, false, 2, true>(d, ka, st);
    return launch<256, A_K, B_TMA_MN, false, false, 2, true>(d, ka, st);
  }
  // NF4 B with 256-wide tiles: CTA pairs (half the decode per CTA)
  const bool pair_ok = nf4 && bn == 256 && d.a_major == A_K && soup_aligned(d.absmax, 16) &&
                       (d.b_mode == B_NF4_K ? d.K % 256 == 0 : d.N % 256 == 0);
  if (d.A_lo.ptr) {
    if (pair_ok && d.A_lo.rows == d.A.rows && d.A_lo.cols == d.A.cols) {
      if (d.persistent) {
        if (d.b_mode == B_NF4_K) return launch<256, A_K, B_NF4_K, false, true, 2, true>(d, ka, st);
        return launch<256, A_K, B_NF4_MN, false, true, 2, true>(d, ka, st);
      }
      if (d.b_mode == B_NF4_K) return launch<256, A_K, B_NF4_K, false, true, 2>(d, ka, st);
      return launch<256, A_K, B_NF4_MN, false, true, 2>(d, ka, st);
    }
    SOUP_CHECK(d.a_major == A_K && !d.tf32 && (bn == 256 || bn == 128 || (bn <= 32 && d.b_mode == B_TMA_K)) &&
                   d.A_lo.rows == d.A.rows &&
                   d.A_lo.cols == d.A.cols,
               SOUP_ERR_SHAPE, "gemm: dual-A needs a K-major bf16 A, N tile 128/256 (16/32 for skinny K-major B) "
               "and matching hi/lo shapes");
#define SOUP_GEMM_DUAL(BN_, BMD_) \
  if (bn == BN_ && d.b_mode == BMD_) return launch<BN_, A_K, BMD_, false, true>(d, ka, st);
    SOUP_GEMM_DUAL(256, B_NF4_K) SOUP_GEMM_DUAL(128, B_NF4_K) SOUP_GEMM_DUAL(256, B_NF4_MN)
    SOUP_GEMM_DUAL(128, B_NF4_MN) SOUP_GEMM_DUAL(256, B_TMA_K) SOUP_GEMM_DUAL(128, B_TMA_K)
    SOUP_GEMM_DUAL(256, B_TMA_MN) SOUP_GEMM_DUAL(128, B_TMA_MN)
    SOUP_GEMM_DUAL(32, B_TMA_K) SOUP_GEMM_DUAL(16, B_TMA_K)
#undef SOUP_GEMM_DUAL
    return fail(SOUP_ERR_SHAPE, "gemm: no dual-A kernel for BN=%d b_mode=%d", bn, d.b_mode);
  }
  if (pair_ok) {
    if (d.persistent) {
      if (d.b_mode == B_NF4_K) return launch<256, A_K, B_NF4_K, false, false, 2, true>(d, ka, st);
      return launch<256, A_K, B_NF4_MN, false, false, 2, true>(d, ka, st);
    }
    if (d.b_mode == B_NF4_K) return launch<256, A_K, B_NF4_K, false, false, 2>(d, ka, st);
    return launch<256, A_K, B_NF4_MN, false, false, 2>(d, ka, st);
  }
#define SOUP_GEMM_CASE(BN_, AM_, BMD_) \
  if (bn == BN_ && d.a_major == AM_ && d.b_mode == BMD_) return launch<BN_, AM_, BMD_>(d, ka, st);
  SOUP_GEMM_CASE(256, A_K, B_NF4_K)
  SOUP_GEMM_CASE(128, A_K, B_NF4_K)
  SOUP_GEMM_CASE(64, A_K, B_NF4_K)
  SOUP_GEMM_CASE(256, A_K, B_NF4_MN)
  SOUP_GEMM_CASE(128, A_K, B_NF4_MN)
  SOUP_GEMM_CASE(64, A_K, B_NF4_MN)
  SOUP_GEMM_CASE(256, A_K, B_TMA_K)
  SOUP_GEMM_CASE(128, A_K, B_TMA_K)
  SOUP_GEMM_CASE(64, A_K, B_TMA_K)
  SOUP_GEMM_CASE(48, A_K, B_TMA_K)
  SOUP_GEMM_CASE(32, A_K, B_TMA_K)
  SOUP_GEMM_CASE(16, A_K, B_TMA_K)
  SOUP_GEMM_CASE(256, A_K, B_TMA_MN)
  SOUP_GEMM_CASE(128, A_K, B_TMA_MN)
  SOUP_GEMM_CASE(64, A_K, B_TMA_MN)
  SOUP_GEMM_CASE(64, A_MN, B_TMA_K)
  SOUP_GEMM_CASE(48, A_MN, B_TMA_K)
  SOUP_GEMM_CASE(32, A_MN, B_TMA_K)
  SOUP_GEMM_CASE(16, A_MN, B_TMA_K)
#undef SOUP_GEMM_CASE
  return fail(SOUP_ERR_SHAPE, "gemm: no kernel for BN=%d a_major=%d b_mode=%d (M=%d N=%d K=%d)", bn,
              d.a_major, d.b_mode, d.M, d.N, d.K);
}

}  // namespace

size_t gemm_static_device_bytes() { return sizeof(g_sk_cnt); }

soup_status gemm(const GemmDesc& d, cudaStream_t st) {
  SOUP_CHECK(d.M > 0 && d.N > 0 && d.K > 0, SOUP_ERR_SHAPE, "gemm: empty problem %dx%dx%d", d.M, d.N, d.K);
  SOUP_CHECK(d.out != nullptr, SOUP_ERR_INVALID_ARG, "gemm: null output");
  SOUP_CHECK(d.tail_ksteps >= 0 && d.tail_ksteps <= 4, SOUP_ERR_SHAPE, "gemm: tail_ksteps %d", d.tail_ksteps);
  SOUP_CHECK(d.nseg >= 1 && d.nseg <= 4, SOUP_ERR_SHAPE, "gemm: nseg %d", d.nseg);
  const bool nf4 = d.b_mode >= B_NF4_K;
  if (nf4) {
    SOUP_CHECK(d.codes && d.absmax, SOUP_ERR_INVALID_ARG, "gemm: NF4 operand missing");
    SOUP_CHECK(d.a_major == A_K, SOUP_ERR_SHAPE, "gemm: NF4 B needs a K-major A");
    SOUP_CHECK(d.K % 64 == 0, SOUP_ERR_SHAPE, "gemm: NF4 needs K %% 64 == 0 (K=%d)", d.K);
    if (d.b_mode == B_NF4_MN)
      SOUP_CHECK(d.N % 64 == 0, SOUP_ERR_SHAPE, "gemm: NF4 (transposed) needs N %% 64 == 0");
    SOUP_CHECK(soup_aligned(d.codes, 16), SOUP_ERR_ALIGN, "gemm: NF4 codes misaligned");
  }
  const int bn = pick_bn(d);
  for (int i = 0; i < d.nseg - 1; ++i)
    SOUP_CHECK(d.seg_end[i] % bn == 0, SOUP_ERR_SHAPE, "gemm: segment end %d not a multiple of the tile %d",
               d.seg_end[i], bn);
  if (d.pair_off > 0) {
    SOUP_CHECK(d.N == 2 * d.pair_off && d.pair_off % 128 == 0 && bn == 256 &&
                   (d.b_mode == B_NF4_K || d.b_mode == B_TMA_K) && d.a_major == A_K,
               SOUP_ERR_SHAPE, "gemm: paired tiles need N = 2*pair_off, pair_off %% 128 == 0, K-major B");
    SOUP_CHECK(d.tail_ksteps == 0 || d.tail_ksteps == 1, SOUP_ERR_SHAPE, "gemm: paired tiles take one tail step per half");
  }
  if (d.epi == EPI_SWIGLU) {
    SOUP_CHECK(d.pair_off > 0 && d.swiglu_I == d.pair_off, SOUP_ERR_SHAPE, "gemm: SwiGLU epilogue needs paired tiles");
  }
  if (d.epi == EPI_SWIGLU_BWD) {
    SOUP_CHECK(d.aux16 && d.swiglu_I == d.N && d.out_kind == OUT_BF16, SOUP_ERR_INVALID_ARG,
               "gemm: SwiGLU backward epilogue needs g|u and a bf16 [M, 2N] output");
  }
  KArgs ka;
  memset(&ka, 0, sizeof(ka));
  ka.M = d.M; ka.N = d.N; ka.K = d.K;
  ka.num_kb = d.tf32 ? (d.K + 31) / 32 : (d.K + BK - 1) / BK;
  ka.codes = d.codes; ka.absmax = d.absmax;
  ka.tail_ksteps = d.tail_ksteps; ka.nseg = d.nseg;
  for (int i = 0; i < 4; ++i) { ka.seg_end[i] = d.seg_end[i]; ka.seg_row[i] = d.seg_row[i]; }
  ka.pair_off = d.pair_off;
  ka.epi = d.epi;
  ka.out_kind = d.out_kind; ka.out = d.out; ka.ldo = d.ldo; ka.out2 = d.out2; ka.out_lo = d.out_lo;
  ka.resid = d.resid; ka.resid_f32 = d.resid_f32; ka.ldr = d.ldr; ka.alpha = d.alpha;
  ka.scale_amax = d.scale_amax;
  ka.aux16 = d.aux16; ka.ld_aux = d.ld_aux; ka.swiglu_I = d.swiglu_I;
  const int esz = (d.out_kind == OUT_F32 || d.out_kind == OUT_F32_T) ? 4 : 2;
  // row-chunk accesses of the epilogue: 32 bytes per instruction where every
  // row pointer it forms is 32-byte aligned, else 16 bytes, else scalar
  auto rows_aligned = [&](size_t a) {
    return soup_aligned(d.out, a) && ((d.ldo * esz) % a == 0) && (!d.out_lo || soup_aligned(d.out_lo, a)) &&
           (!d.resid || (soup_aligned(d.resid, a) && (d.ldr * 2) % a == 0)) &&
           (!d.resid_f32 || (soup_aligned(d.resid_f32, a) && (d.ldr * 4) % a == 0)) &&
           (!d.aux16 || (soup_aligned(d.aux16, a) && (d.ld_aux * 2) % a == 0 && (d.swiglu_I * 2) % a == 0)) &&
           (!d.rope_cols || (soup_aligned(d.rope_cos, a) && soup_aligned(d.rope_sin, a)));
  };
  ka.vec_ok = rows_aligned(32) ? 2 : (rows_aligned(16) ? 1 : 0);
  ka.wait_limit = d.wait_limit > 0 ? d.wait_limit : 4000000000LL;
  ka.skip_producer = d.debug_skip_producer;
  ka.rope_cols = d.rope_cols; ka.rope_S = d.rope_S;
  ka.rope_Lp = d.rope_group > 1 ? d.rope_prefix : 0;
  ka.rope_G = d.rope_group > 1 ? d.rope_group : 1;
  ka.rope_cos = d.rope_cos; ka.rope_sin = d.rope_sin;
  if (d.rope_cols > 0) {
    SOUP_CHECK((d.out_kind == OUT_BF16 || d.out_kind == OUT_F16) && !d.resid && !d.resid_f32 && d.rope_cos &&
                   d.rope_sin && d.rope_S > 0 && d.rope_cols % 128 == 0 && bn >= 128,
               SOUP_ERR_SHAPE, "gemm: RoPE epilogue needs a plain 16-bit output, 128-aligned heads and BN >= 128");
  }
  ka.err = device_error_word();
  SOUP_CHECK(ka.err != nullptr, SOUP_ERR_CUDA, "device error word unavailable");

  if (d.split_ws && d.split_ws_bytes > 0 && !nf4 && d.epi == EPI_STORE && d.tail_ksteps == 0 &&
      !d.resid && !d.resid_f32 && d.pair_off == 0 && d.rope_cols == 0 &&
      (d.out_kind == OUT_BF16_T || d.out_kind == OUT_F32 || d.out_kind == OUT_F32_T || d.out_kind == OUT_BF16) &&
      d.N % 4 == 0 && soup_aligned(d.split_ws, 16)) {
    const int sms = sm_count();
    const int tiles = ((d.M + BM - 1) / BM) * ((d.N + bn - 1) / bn);
    int splits = std::min(8, std::min(ka.num_kb / 2, (sms + tiles - 1) / tiles));
    while (splits > 1 && (size_t)splits * d.M * d.N * 4 > d.split_ws_bytes) --splits;
    if (splits > 1) {
      KArgs kz = ka;
      kz.kb_split = (ka.num_kb + splits - 1) / splits;
      splits = (ka.num_kb + kz.kb_split - 1) / kz.kb_split;
      // partial planes in the output's own orientation ([M, N], or [N, M]
      // for transposed outputs), so that the reduction reads and writes
      // consecutive addresses with consecutive threads
      const bool tr = d.out_kind == OUT_BF16_T || d.out_kind == OUT_F32_T;
      kz.out = d.split_ws;
      kz.out_kind = tr ? OUT_F32_T : OUT_F32;
      kz.ldo = tr ? d.M : d.N;
      kz.out2 = nullptr;
      kz.out_lo = nullptr;
      kz.alpha = 1.f;
      kz.scale_amax = nullptr;
      kz.vec_ok = (soup_aligned(d.split_ws, 32) && (kz.ldo * 4) % 32 == 0) ? 2 : 1;
      SOUP_TRY(dispatch(d, kz, bn, st));
      const size_t total = (size_t)d.M * d.N;
      const int blocks = (int)std::min<size_t>((total + 255) / 256, (size_t)sms * 8);
      const int oes = (d.out_kind == OUT_F32 || d.out_kind == OUT_F32_T) ? 4 : 2;
      profile_begin(st, GC_SPLITK, 0.0,
                    (double)total * (4.0 * splits + oes + (d.out2 ? 4 : 0) + (d.out_lo ? 2 : 0)));
      splitk_reduce_kernel<<<blocks, 256, 0, st>>>(d.split_ws, splits, d.M, d.N, d.out_kind, d.out, d.out2,
                                                   d.out_lo, d.ldo, d.alpha, d.scale_amax);
      SOUP_LAUNCH_CHECK();
      profile_end(st);
      return SOUP_OK;
    }
  }
  return dispatch(d, ka, bn, st);
}

}  // namespace soup

using namespace soup;

extern "C" soup_status soup_debug_gemm_bounded_wait(const uint16_t* A, const uint16_t* B, int64_t M, int64_t N,
                                                    int64_t K, float* C, int64_t wait_limit_cycles,
                                                    int32_t skip_producer_arrivals, void* stream) {
  SOUP_CHECK(A && B && C, SOUP_ERR_INVALID_ARG, "soup_debug_gemm_bounded_wait: null pointer");
  SOUP_CHECK(M > 0 && N > 0 && K > 0 && M <= 4096 && N <= 4096 && K <= 4096 && K % 8 == 0 && N % 4 == 0,
             SOUP_ERR_SHAPE, "soup_debug_gemm_bounded_wait: sizes must be in (0, 4096], K %% 8 == 0, N %% 4 == 0");
  SOUP_CHECK(wait_limit_cycles >= 0, SOUP_ERR_INVALID_ARG, "soup_debug_gemm_bounded_wait: negative wait limit");
  GemmDesc g;  // bf16 K-major operands: the one-CTA engine, no split-K
  g.M = (int)M; g.N = (int)N; g.K = (int)K;
  g.A = Mat{A, M, K, K};
  g.b_mode = B_TMA_K;
  g.B = Mat{B, N, K, K};
  g.out_kind = OUT_F32; g.out = C; g.ldo = N;
  g.wait_limit = wait_limit_cycles;
  g.debug_skip_producer = skip_producer_arrivals ? 1 : 0;
  return gemm(g, static_cast<cudaStream_t>(stream));
}
