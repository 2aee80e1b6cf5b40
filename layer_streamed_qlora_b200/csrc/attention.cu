// Causal GQA attention (head_dim 128) of the decoder layer on the fifth-
// generation tensor cores: tcgen05.mma with the accumulators in tensor memory,
// operand tiles brought into 128-byte-swizzled shared memory by TMA (no
// cluster multicast), warp-specialised CTAs (one TMA thread, one MMA thread,
// eight softmax / elementwise warps: two per query or key row, each taking
// half of the row's columns).
//
//   forward   per (128-query tile, q head): S_j = Q K_j^T into tensor memory,
//             online softmax in fp32 (log2 domain) from a two-pass read of the
//             row (max, then 2^(s - m) and the row sum), P_j in fp16 into
//             shared memory, O_j = P_j V_j into a fresh tensor-memory
//             accumulator, folded into the row's fp32 running output in
//             registers with the online-softmax correction.  S and O are
//             double-buffered in tensor memory (4 x 128 columns), so the
//             tensor cores compute S_{j+1} and O_j while the softmax warps
//             work on block j.
//   backward  two passes in one launch, no atomics (every run gives the same
//             bits):
//             pass 1 per (128-key block, kv head): for each q head of the group
//             and each 64-query tile at or after the block, S^T = K Q^T and
//             dP^T = V dO^T (tensor memory), P^T = 2^(S^T scale - L) and
//             dS^T = P^T (dP^T - D) in fp16 into shared memory, then
//             dV += P^T dO and dK += dS^T Q accumulated in tensor memory;
//             pass 2 per (128-query tile, q head): S = Q K^T, dP = dO V^T per
//             64-key block, dS into shared memory, dQ += dS K in tensor memory.
//             The passes write disjoint outputs, so their CTAs share the grid
//             (heaviest pass-1 key blocks first, then pass-2 query tiles).
//             Q, dO (pass 1) and K (pass 2) tiles serve both as K-major and as
//             MN-major operands of the same shared-memory bytes.
//
// Inputs q, k, v and dO are fp16 (the projections write them in fp16: same
// 16-bit traffic as bf16 with 8x finer rounding for these O(1) values), P and
// dS enter the MMAs as fp16, accumulation is fp32; the saved log-sum-exp is
// in log2 units.  Outputs (attention output, dq, dk, dv) are bf16, with
// optional fp16 / fp32 copies.  Every mbarrier wait is bounded: on expiry the
// CTA records code 4 in the device error word, stops issuing work, lets copies
// and MMAs in flight land, frees its tensor memory and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "elementwise.h"
#include "gscale.cuh"
#include "ptx.cuh"

namespace soup {
namespace {

constexpr int HD = 128;          // head dim
constexpr int ERR_ATTN_WAIT = 4;  // device error code: a bounded wait of an attention kernel expired

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ uint32_t pack_b2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
// One 16-byte unit (8 16-bit values) of row r of a K-major 128-byte-swizzled
// tile (rows of 128 bytes; unit u of row r stored at unit u ^ (r % 8)).
__device__ __forceinline__ void st_unit(uint8_t* tile, int r, int u, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  *reinterpret_cast<uint4*>(tile + r * 128 + ((u ^ (r & 7)) << 4)) = make_uint4(a, b, c, d);
}
// 2^x on the special-function unit (PTX ex2.approx.ftz.f32: relative error
// about 2^-22, results below 2^-126 flushed to zero).  Every argument here is
// a scaled score minus a running maximum or log-sum-exp (<= 0 up to
// rounding), or -inf for a masked key, whose power is 0.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~static_cast<uintptr_t>(1023));
}
// K-major operand descriptor: 128-byte rows, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t kdesc(uint32_t saddr) { return ptx::smem_desc_sw128(saddr, 16, 1024); }
// MN-major operand descriptor: 64-element MN chunks `chunk` bytes apart.
__device__ __forceinline__ uint64_t mndesc(uint32_t saddr, uint32_t chunk) {
  return ptx::smem_desc_sw128(saddr, chunk, 1024);
}

struct AttnArgs {
  int S, Hq, Hkv, T;  // S: tokens per sequence; T: token rows in memory
  int nseq;           // sequences (forward grid)
  // Sequences come in groups of G that share their first Lp positions,
  // stored once: a group's rows are [prefix | continuation of sequence 0 |
  // ... | continuation of sequence G-1] (G = 1, Lp = 0: sequence v is rows
  // [v S, (v + 1) S)).  Queries of the shared prefix belong to sequence 0.
  int G, Lp;
  float scale_log2;  // log2(e) / sqrt(head_dim)
  float scale;       // 1 / sqrt(head_dim)
  // forward
  uint16_t* out;
  float* lse;
  uint16_t* out16;
  float* out32;
  // backward
  const float* L;  // [Hq, T] log2-domain log-sum-exp of the forward pass
  const float* D;  // [Hq, T] rowsum(dO * O)
  uint16_t* dqkv;  // [T, ld] bf16
  float* dqkv32;   // [T, ld] fp32 or null
  int ld;
  const float* rcos;  // [S, 64] or null: rotate dq / dk back
  const float* rsin;
  const unsigned int* amax;  // dO's power-of-two gradient scale, or null
  // 1: every output pointer (and RoPE table) the epilogues form is 32-byte
  // aligned, so they move a row's values with 32-byte accesses
  int v32;
  int* err;
  long long wait_limit;
};

// Physical token row of position t of sequence v.
__device__ __forceinline__ int vrow(const AttnArgs& a, int v, int t) {
  const int Lc = a.S - a.Lp;
  const int g = v / a.G, i = v - g * a.G;
  return g * (a.Lp + a.G * Lc) + (t < a.Lp ? t : a.Lp + i * Lc + (t - a.Lp));
}

#define ATTN_WAIT(bar, parity)                                                   \
  (ptx::mbar_wait_bounded((bar), (parity), abort_flag, a.wait_limit) ||          \
   (atomicOr(a.err, ERR_ATTN_WAIT), *abort_flag = 1, false))

// Tail of every attention kernel: all threads meet, a CTA that gave up lets
// copies and MMAs in flight land (~1 ms, bounded), then warp 1 frees the
// tensor memory.
__device__ __forceinline__ void attn_teardown(volatile int* abort_flag, int warp, uint32_t tmem) {
  ptx::tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    const long long t0 = clock64();
    while (clock64() - t0 < 2000000LL) {
    }
    __syncthreads();
  }
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

// 32 fp32 values -> 32 bf16 (or fp16) at o: 16-byte stores, or 32-byte ones
// when v32 (o 32-byte aligned).
template <bool HALF>
__device__ __forceinline__ void store32_16bit(uint16_t* o, const float (&f)[32], bool v32) {
  if (v32) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      uint32_t w[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        w[i] = HALF ? pack_h2(f[16 * u + 2 * i], f[16 * u + 2 * i + 1]) : pack_b2(f[16 * u + 2 * i], f[16 * u + 2 * i + 1]);
      ptx::st_global_32B(o + 16 * u, w);
    }
  } else {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        w[i] = HALF ? pack_h2(f[8 * u + 2 * i], f[8 * u + 2 * i + 1]) : pack_b2(f[8 * u + 2 * i], f[8 * u + 2 * i + 1]);
      reinterpret_cast<uint4*>(o)[u] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}
// 32 fp32 values at p: 16-byte stores, or 32-byte ones when v32.
__device__ __forceinline__ void store32_f32(float* p, const float (&f)[32], bool v32) {
  if (v32) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      uint32_t w[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) w[i] = __float_as_uint(f[8 * u + i]);
      ptx::st_global_32B(p + 8 * u, w);
    }
  } else {
#pragma unroll
    for (int u = 0; u < 8; ++u)
      reinterpret_cast<float4*>(p)[u] = make_float4(f[4 * u], f[4 * u + 1], f[4 * u + 2], f[4 * u + 3]);
  }
}
// 32 consecutive fp32 table values at t (128-byte aligned when v32).
__device__ __forceinline__ void load32_f32(const float* t, float (&f)[32], bool v32) {
  if (v32) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      uint32_t w[8];
      ptx::ld_global_32B(t + 8 * u, w);
#pragma unroll
      for (int i = 0; i < 8; ++i) f[8 * u + i] = __uint_as_float(w[i]);
    }
  } else {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float4 x = __ldg(reinterpret_cast<const float4*>(t) + u);
      f[4 * u] = x.x; f[4 * u + 1] = x.y; f[4 * u + 2] = x.z; f[4 * u + 3] = x.w;
    }
  }
}

// Rotates the pair (i, i + 64) of a 128-wide head back by the position's
// angle: (a, b) -> (a c + b s, b c - a s).
__device__ __forceinline__ void rope_back(float& x0, float& x1, float c, float s) {
  const float a = x0 * c + x1 * s, b = x1 * c - x0 * s;
  x0 = a;
  x1 = b;
}

// ====================================================================== forward
// Shared memory: Q tile (2 chunks x 16 KB), 2 K|V stages (64 KB each), 2 P
// buffers (32 KB each), barriers, the partial row sums.  Warps: 0 TMA, 1 MMA,
// 2..9 softmax (two per row).
constexpr int F_Q = 0, F_KV = 32768, F_P = F_KV + 2 * 65536, F_BAR = F_P + 2 * 32768;
constexpr int F_SMEM = F_BAR + 256 + 1024 + 1024;

__global__ void __launch_bounds__(320, 1) attn_fwd_tc(const __grid_constant__ CUtensorMap tm, const AttnArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + F_BAR);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = bars + 3;
  uint64_t* s_full = bars + 5;
  uint64_t* s_free = bars + 7;
  uint64_t* p_full = bars + 9;
  uint64_t* p_empty = bars + 11;
  uint64_t* o_full = bars + 13;
  uint64_t* o_free = bars + 15;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 17);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* lsum = reinterpret_cast<float*>(sm + F_BAR + 256);  // [2][128] partial row sums

  const int S = a.S;
  const int nqt = (S + 127) / 128;
  // one-dimensional grid, query tile outermost: the tiles with the most key
  // blocks (the last ones) of every head and sequence start first
  const int hv = (int)blockIdx.x % (a.Hq * a.nseq), qb = nqt - 1 - (int)blockIdx.x / (a.Hq * a.nseq);
  const int h = hv % a.Hq, v = hv / a.Hq;  // q head, sequence
  if (v % a.G != 0 && qb * 128 < a.Lp) return;  // shared-prefix queries: sequence 0 of the group computes them
  const int g = h / (a.Hq / a.Hkv);
  const int nkb = qb + 1;
  const int qcol = h * HD, kcol = (a.Hq + g) * HD, vcol = (a.Hq + a.Hkv + g) * HD;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    ptx::mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&kv_full[i], 1);
      ptx::mbar_init(&kv_empty[i], 1);
      ptx::mbar_init(&s_full[i], 1);
      ptx::mbar_init(&s_free[i], 8);
      ptx::mbar_init(&p_full[i], 8);
      ptx::mbar_init(&p_empty[i], 1);
      ptx::mbar_init(&o_full[i], 1);
      ptx::mbar_init(&o_free[i], 8);
    }
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tm);
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;  // columns: S[0] 0, S[1] 128, O[0] 256, O[1] 384
  bool ok = true;
  float o[64];  // softmax warps: this thread's 64 output columns, unnormalised
  float m = -INFINITY;

  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      const int qrow = vrow(a, v, qb * 128);
      ptx::mbar_arrive_expect_tx(q_full, 32768);
      ptx::tma_load_2d(sm + F_Q, &tm, q_full, qcol, qrow);
      ptx::tma_load_2d(sm + F_Q + 16384, &tm, q_full, qcol + 64, qrow);
      for (int j = 0; j < nkb; ++j) {
        const int s = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!ATTN_WAIT(&kv_empty[s], ph ^ 1)) break;
        uint8_t* kv = sm + F_KV + s * 65536;
        const int r = vrow(a, v, j * 128);
        ptx::mbar_arrive_expect_tx(&kv_full[s], 65536);
        ptx::tma_load_2d(kv, &tm, &kv_full[s], kcol, r);
        ptx::tma_load_2d(kv + 16384, &tm, &kv_full[s], kcol + 64, r);
        ptx::tma_load_2d(kv + 32768, &tm, &kv_full[s], vcol, r);
        ptx::tma_load_2d(kv + 49152, &tm, &kv_full[s], vcol + 64, r);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_s = ptx::idesc_fmt(128, 128, 0, 0, 0u);  // fp16 A, B; fp32 D
      constexpr uint32_t id_o = ptx::idesc_fmt(128, 128, 0, 1, 0u);  // V: MN-major B
      const uint32_t qa = ptx::smem_u32(sm + F_Q);
      const bool go = ATTN_WAIT(q_full, 0);
      for (int jj = 0; go && jj <= nkb; ++jj) {
        if (jj < nkb) {  // S_jj = Q K_jj^T
          const int s = jj & 1;
          const uint32_t ph = (jj >> 1) & 1;
          if (!ATTN_WAIT(&kv_full[s], ph) || !ATTN_WAIT(&s_free[s], ph ^ 1)) break;
          ptx::tc_fence_after();
          const uint32_t ka = ptx::smem_u32(sm + F_KV + s * 65536);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            ptx::mma_bf16(tmem + s * 128, kdesc(qa + (k >> 2) * 16384 + (k & 3) * 32),
                          kdesc(ka + (k >> 2) * 16384 + (k & 3) * 32), id_s, k > 0 ? 1u : 0u);
          ptx::mma_commit(&s_full[s]);
        }
        if (jj >= 1) {  // O_j = P_j V_j, j = jj - 1
          const int j = jj - 1, s = j & 1;
          const uint32_t ph = (j >> 1) & 1;
          if (!ATTN_WAIT(&p_full[s], ph) || !ATTN_WAIT(&o_free[s], ph ^ 1)) break;
          ptx::tc_fence_after();
          const uint32_t pa = ptx::smem_u32(sm + F_P + s * 32768);
          const uint32_t va = ptx::smem_u32(sm + F_KV + s * 65536 + 32768);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            ptx::mma_bf16(tmem + 256 + s * 128, kdesc(pa + (k >> 2) * 16384 + (k & 3) * 32), mndesc(va + k * 2048, 16384),
                          id_o, k > 0 ? 1u : 0u);
          ptx::mma_commit(&o_full[s]);
          ptx::mma_commit(&kv_empty[s]);
          ptx::mma_commit(&p_empty[s]);
        }
      }
    }
  } else {
    // ------------------------------- softmax warps: two per row (64 columns each)
    // Both warps of a pair read the whole row of S for its maximum (the same
    // values in the same order, so the same maximum), then each computes P
    // and folds O for its half of the columns, with a partial row sum.
    const int quad = warp & 3, half = (warp - 2) >> 2;
    const int row = quad * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
    const int qi = qb * 128 + row;  // query position in the sequence
    const float sl2 = a.scale_log2;
#pragma unroll
    for (int i = 0; i < 64; ++i) o[i] = 0.f;
    float l = 0.f, m_o = -INFINITY, m_pend = -INFINITY;
    auto fold_o = [&](int jo, float mj) -> bool {
      const int s = jo & 1;
      const uint32_t ph = (jo >> 1) & 1;
      if (!ATTN_WAIT(&o_full[s], ph)) return false;
      ptx::tc_fence_after();
      const float alpha = ex2(m_o - mj);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t v[32];
        ptx::tmem_ld32(tl + 256 + s * 128 + half * 64 + c * 32, v);
        ptx::tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) o[c * 32 + i] = fmaf(o[c * 32 + i], alpha, __uint_as_float(v[i]));
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&o_free[s]);
      m_o = mj;
      return true;
    };
    for (int j = 0; j < nkb; ++j) {
      const int s = j & 1;
      const uint32_t ph = (j >> 1) & 1;
      if (!ATTN_WAIT(&s_full[s], ph)) { ok = false; break; }
      ptx::tc_fence_after();
      const int key0 = j * 128;
      const bool edge = key0 + 127 > qi || key0 + 128 > S;  // some key of the block is masked for this row
      // pass 1: the row's maximum over the block, of the raw scores (the
      // scale is positive: it multiplies the maximum once)
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t v[32];
        ptx::tmem_ld32(tl + s * 128 + c * 32, v);
        ptx::tmem_ld_wait();
        if (edge) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int key = key0 + c * 32 + i;
            if (key <= qi && key < S) mx = fmaxf(mx, __uint_as_float(v[i]));
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) mx = fmaxf(mx, __uint_as_float(v[i]));
        }
      }
      const float m_new = fmaxf(m, mx * sl2);
      // pass 2 (this warp's 64 keys): p = 2^(x - m_new) (0 where masked),
      // partial row sum, P in fp16
      if (!ATTN_WAIT(&p_empty[s], ph ^ 1)) { ok = false; break; }
      uint8_t* P = sm + F_P + s * 32768 + half * 16384;  // keys 0..63 | 64..127
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t v[32];
        ptx::tmem_ld32(tl + s * 128 + half * 64 + c * 32, v);
        ptx::tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const int key = key0 + half * 64 + c * 32 + i;
          // one FMA per exponent argument: x * scale - m
          float x0 = fmaf(__uint_as_float(v[i]), sl2, -m_new), x1 = fmaf(__uint_as_float(v[i + 1]), sl2, -m_new);
          if (edge) {
            if (key > qi || key >= S) x0 = -INFINITY;
            if (key + 1 > qi || key + 1 >= S) x1 = -INFINITY;
          }
          const float p0 = ex2(x0), p1 = ex2(x1);
          sum += p0 + p1;
          pk[i >> 1] = pack_h2(p0, p1);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
          st_unit(P, row, c * 4 + u, pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
      }
      ptx::tc_fence_before();
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        ptx::mbar_arrive(&s_free[s]);
        ptx::mbar_arrive(&p_full[s]);
      }
      l = l * ex2(m - m_new) + sum;
      m = m_new;
      if (j >= 1 && !fold_o(j - 1, m_pend)) { ok = false; break; }
      m_pend = m_new;
    }
    if (ok) ok = fold_o(nkb - 1, m_pend);
    lsum[half * 128 + row] = l;
  }
  // the two partial row sums meet here; then each softmax thread stores its
  // 64 output columns (and half 0 the log-sum-exp)
  __syncthreads();
  if (warp >= 2 && ok) {
    const int quad = warp & 3, half = (warp - 2) >> 2;
    const int row = quad * 32 + lane;
    const int qi = qb * 128 + row;
    if (qi < S) {
      const float l = lsum[row] + lsum[128 + row];
      const float inv = 1.f / l;
      const int prow = vrow(a, v, qi);
      const size_t off = (size_t)prow * (a.Hq * HD) + h * HD + half * 64;
      const bool v32 = a.v32 != 0;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        float f[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) f[i] = o[u * 32 + i] * inv;
        store32_16bit<false>(a.out + off + 32 * u, f, v32);
        if (a.out16) store32_16bit<true>(a.out16 + off + 32 * u, f, v32);
        if (a.out32) store32_f32(a.out32 + off + 32 * u, f, v32);
      }
      if (half == 0) a.lse[(size_t)h * a.T + prow] = m + log2f(l);
    }
  }
  attn_teardown(abort_flag, warp, tmem);
}

// ================================================ backward pass 1: dK and dV
// Shared memory: K and V of the block (32 KB each, K-major, 128 rows), NS
// stages of (Q tile | dO tile) (64 rows: 16 KB each) with their L and D
// values, 2 P^T and 2 dS^T buffers ([128 keys, 64 queries] fp16, 16 KB each).
constexpr int B1_NS = 3;
constexpr int B1_K = 0, B1_V = 32768, B1_ST = 65536;
constexpr int B1_STAGE = 32768;
constexpr int B1_P = B1_ST + B1_NS * B1_STAGE;  // 2 x 16 KB
constexpr int B1_DS = B1_P + 2 * 16384;         // 2 x 16 KB
constexpr int B1_LD = B1_DS + 2 * 16384;        // NS x (64 L + 64 D) floats
constexpr int B1_BAR = B1_LD + B1_NS * 512;
constexpr int B1_SMEM = B1_BAR + 256 + 1024;

// One CTA of pass 1 (key block bx of sequence group bz, kv head by).
__device__ __forceinline__ void attn_bwd_dkdv_cta(const CUtensorMap& tm128, const CUtensorMap& tm64,
                                                  const CUtensorMap& tmdo64, const AttnArgs& a, int bx, int by,
                                                  int bz) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + B1_BAR);
  uint64_t* kv_full = bars;               // 1
  uint64_t* full = bars + 1;              // [NS]
  uint64_t* empty = full + B1_NS;         // [NS]
  uint64_t* st_full = empty + B1_NS;      // [2]
  uint64_t* st_free = st_full + 2;        // [2]
  uint64_t* p_full = st_free + 2;         // [2]
  uint64_t* p_empty = p_full + 2;         // [2]
  uint64_t* acc_full = p_empty + 2;       // 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int S = a.S;
  // physical key block pb of sequence group gq: a block of the shared prefix
  // (every sequence of the group attends to it) or a continuation block of
  // one sequence; the first blocks have the most query tiles
  const int g = by, gq = bz;
  const int nb_pre = a.Lp / 128, nbc = (S - a.Lp + 127) / 128;
  const int pb = bx;
  const bool prefix = pb < nb_pre;
  const int own = prefix ? 0 : (pb - nb_pre) / nbc;            // sequence of the group owning the block
  const int kb = prefix ? pb : nb_pre + (pb - nb_pre) % nbc;    // block index within the sequence
  const int v0 = gq * a.G + own;
  const int grp = a.Hq / a.Hkv;
  const int kcol = (a.Hq + g) * HD, vcol = (a.Hq + a.Hkv + g) * HD;
  const int nqt = (S + 63) / 64;
  // work items (sequence of the group, q head of the kv group, 64-query
  // tile): the owner's tiles from the block on; for a prefix block also the
  // other sequences' continuation tiles
  const int per0 = nqt - 2 * kb, perR = nqt - a.Lp / 64;
  const int seg0 = grp * per0;
  const int n_it = seg0 + (prefix ? (a.G - 1) * grp * perR : 0);
  auto item = [&](int it, int& vseq, int& hh, int& qt) {
    if (it < seg0) {
      vseq = v0;
      hh = it / per0;
      qt = 2 * kb + it % per0;
    } else {
      const int r = it - seg0, segR = grp * perR;
      vseq = gq * a.G + 1 + r / segR;
      hh = (r % segR) / perR;
      qt = a.Lp / 64 + (r % segR) % perR;
    }
  };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    ptx::mbar_init(kv_full, 1);
    for (int i = 0; i < B1_NS; ++i) {
      ptx::mbar_init(&full[i], 1);
      ptx::mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&st_full[i], 1);
      ptx::mbar_init(&st_free[i], 8);
      ptx::mbar_init(&p_full[i], 8);
      ptx::mbar_init(&p_empty[i], 1);
    }
    ptx::mbar_init(acc_full, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tm128);
    ptx::prefetch_tmap(&tm64);
    ptx::prefetch_tmap(&tmdo64);
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  // columns: S^T[0] 0, S^T[1] 64, dP^T[0] 128, dP^T[1] 192, dV 256, dK 384
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------- TMA producer (whole warp)
    if (lane == 0) {
      ptx::mbar_arrive_expect_tx(kv_full, 65536);
      const int r = vrow(a, v0, kb * 128);
      ptx::tma_load_2d(sm + B1_K, &tm128, kv_full, kcol, r);
      ptx::tma_load_2d(sm + B1_K + 16384, &tm128, kv_full, kcol + 64, r);
      ptx::tma_load_2d(sm + B1_V, &tm128, kv_full, vcol, r);
      ptx::tma_load_2d(sm + B1_V + 16384, &tm128, kv_full, vcol + 64, r);
    }
    for (int it = 0; it < n_it; ++it) {
      const int s = it % B1_NS;
      const uint32_t ph = (it / B1_NS) & 1;
      int okw = 1;
      if (lane == 0) okw = ATTN_WAIT(&empty[s], ph ^ 1) ? 1 : 0;
      okw = __shfl_sync(0xffffffffu, okw, 0);
      if (!okw) break;
      int vs, hh, qt;
      item(it, vs, hh, qt);
      const int h = g * grp + hh;
      const int q0 = qt * 64;
      const int qrow0 = vrow(a, vs, q0);
      // this tile's L and D (the softmax warps read them after the stage's full barrier)
      float* LD = reinterpret_cast<float*>(sm + B1_LD + s * 512);
#pragma unroll
      for (int i = lane; i < 64; i += 32) {
        const bool in = q0 + i < S;
        LD[i] = in ? a.L[(size_t)h * a.T + qrow0 + i] : 0.f;
        LD[64 + i] = in ? a.D[(size_t)h * a.T + qrow0 + i] : 0.f;
      }
      __syncwarp();
      if (lane == 0) {
        uint8_t* st = sm + B1_ST + s * B1_STAGE;
        ptx::mbar_arrive_expect_tx(&full[s], 32768);
        ptx::tma_load_2d(st, &tm64, &full[s], h * HD, qrow0);            // Q
        ptx::tma_load_2d(st + 8192, &tm64, &full[s], h * HD + 64, qrow0);
        ptx::tma_load_2d(st + 16384, &tmdo64, &full[s], h * HD, qrow0);  // dO
        ptx::tma_load_2d(st + 24576, &tmdo64, &full[s], h * HD + 64, qrow0);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_st = ptx::idesc_fmt(128, 64, 0, 0, 0u);    // S^T, dP^T: [128 keys, 64 queries]
      constexpr uint32_t id_acc = ptx::idesc_fmt(128, 128, 0, 1, 0u);  // dV, dK: B (dO, Q) MN-major
      const uint32_t ka = ptx::smem_u32(sm + B1_K), va = ptx::smem_u32(sm + B1_V);
      bool ok = ATTN_WAIT(kv_full, 0);
      for (int jj = 0; ok && jj <= n_it; ++jj) {
        if (jj < n_it) {
          const int s = jj % B1_NS, bb = jj & 1;
          const uint32_t ph = (jj / B1_NS) & 1, pb = (jj >> 1) & 1;
          if (!ATTN_WAIT(&full[s], ph) || !ATTN_WAIT(&st_free[bb], pb ^ 1)) break;
          ptx::tc_fence_after();
          const uint32_t qa = ptx::smem_u32(sm + B1_ST + s * B1_STAGE), oa = qa + 16384;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t off = (k >> 2) * 8192 + (k & 3) * 32;
            ptx::mma_bf16(tmem + bb * 64, kdesc(ka + (k >> 2) * 16384 + (k & 3) * 32), kdesc(qa + off), id_st,
                          k > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t off = (k >> 2) * 8192 + (k & 3) * 32;
            ptx::mma_bf16(tmem + 128 + bb * 64, kdesc(va + (k >> 2) * 16384 + (k & 3) * 32), kdesc(oa + off), id_st,
                          k > 0 ? 1u : 0u);
          }
          ptx::mma_commit(&st_full[bb]);
        }
        if (jj >= 1) {  // dV += P^T dO, dK += dS^T Q for iteration it = jj - 1
          const int it = jj - 1, s = it % B1_NS, bb = it & 1;
          const uint32_t pb = (it >> 1) & 1;
          if (!ATTN_WAIT(&p_full[bb], pb)) break;
          ptx::tc_fence_after();
          const uint32_t qa = ptx::smem_u32(sm + B1_ST + s * B1_STAGE), oa = qa + 16384;
          const uint32_t pa = ptx::smem_u32(sm + B1_P + bb * 16384), da = ptx::smem_u32(sm + B1_DS + bb * 16384);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            ptx::mma_bf16(tmem + 256, kdesc(pa + k * 32), mndesc(oa + k * 2048, 8192), id_acc,
                          (it > 0 || k > 0) ? 1u : 0u);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            ptx::mma_bf16(tmem + 384, kdesc(da + k * 32), mndesc(qa + k * 2048, 8192), id_acc,
                          (it > 0 || k > 0) ? 1u : 0u);
          ptx::mma_commit(&p_empty[bb]);
          ptx::mma_commit(&empty[s]);
        }
      }
      if (ok && n_it > 0) ptx::mma_commit(acc_full);
    }
  } else {
    // ---------------- elementwise warps: two per key row, 32 queries each
    const int quad = warp & 3, half = (warp - 2) >> 2;
    const int row = quad * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
    const int key = kb * 128 + row;
    const float sl2 = a.scale_log2;
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int s = it % B1_NS, bb = it & 1;
      const uint32_t pb = (it >> 1) & 1;
      int vs, hh, qt;
      item(it, vs, hh, qt);
      const int q0 = qt * 64;
      // the stage's full barrier also publishes the L and D values the
      // producer warp stored next to the tiles (it cannot move on to the
      // stage's next use before these warps release this iteration)
      if (!ATTN_WAIT(&full[s], (it / B1_NS) & 1) || !ATTN_WAIT(&st_full[bb], pb)) { ok = false; break; }
      ptx::tc_fence_after();
      const float* LD = reinterpret_cast<const float*>(sm + B1_LD + s * 512);
      if (!ATTN_WAIT(&p_empty[bb], pb ^ 1)) { ok = false; break; }
      uint8_t* P = sm + B1_P + bb * 16384;
      uint8_t* DS = sm + B1_DS + bb * 16384;
      const bool edge = q0 < key || q0 + 64 > S || key >= S;  // some query of the tile is masked for this key
      {
        const int c = half;  // this warp's 32 queries of the tile
        uint32_t sv[32], dv[32];
        ptx::tmem_ld32(tl + bb * 64 + c * 32, sv);
        ptx::tmem_ld32(tl + 128 + bb * 64 + c * 32, dv);
        ptx::tmem_ld_wait();
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float p[2], d[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int qi = c * 32 + i + e;
            const int q = q0 + qi;
            float x = fmaf(__uint_as_float(sv[i + e]), sl2, -LD[qi]);
            if (edge && (q < key || q >= S || key >= S)) x = -INFINITY;
            p[e] = ex2(x);
            d[e] = p[e] * (__uint_as_float(dv[i + e]) - LD[64 + qi]);
          }
          pk[i >> 1] = pack_h2(p[0], p[1]);
          dk[i >> 1] = pack_h2(d[0], d[1]);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          st_unit(P, row, c * 4 + u, pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
          st_unit(DS, row, c * 4 + u, dk[4 * u], dk[4 * u + 1], dk[4 * u + 2], dk[4 * u + 3]);
        }
      }
      ptx::tc_fence_before();
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        ptx::mbar_arrive(&st_free[bb]);
        ptx::mbar_arrive(&p_full[bb]);
      }
    }
    // epilogue: dK (x scale, RoPE back) from the second warp of a row, dV
    // (unscaled) from the first, out of tensor memory
    if (ok && n_it > 0 && ATTN_WAIT(acc_full, 0)) {
      ptx::tc_fence_after();
      const float unscale = a.amax ? 1.f / grad_scale_from_amax(__uint_as_float(*a.amax)) : 1.f;
      const bool in = key < S;
      const size_t r = (size_t)(in ? vrow(a, v0, key) : 0) * a.ld;
      {
        const int which = half;  // 0: dV, 1: dK
        const uint32_t col0 = which ? 384 : 256;
        const float mul = which ? a.scale * unscale : unscale;
        const int dcol = which ? kcol : vcol;
#pragma unroll
        for (int c = 0; c < 2; ++c) {  // pairs (c*32 + i, c*32 + i + 64)
          uint32_t v0[32], v1[32];
          ptx::tmem_ld32(tl + col0 + c * 32, v0);
          ptx::tmem_ld32(tl + col0 + 64 + c * 32, v1);
          ptx::tmem_ld_wait();
          float f0[32], f1[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            f0[i] = __uint_as_float(v0[i]) * mul;
            f1[i] = __uint_as_float(v1[i]) * mul;
          }
          const bool v32 = a.v32 != 0;
          if (which && a.rcos && in) {
            float cs[32], sn[32];
            load32_f32(a.rcos + (size_t)key * 64 + c * 32, cs, v32);
            load32_f32(a.rsin + (size_t)key * 64 + c * 32, sn, v32);
#pragma unroll
            for (int i = 0; i < 32; ++i) rope_back(f0[i], f1[i], cs[i], sn[i]);
          }
          if (in) {
            uint16_t* o0 = a.dqkv + r + dcol + c * 32;
            store32_16bit<false>(o0, f0, v32);
            store32_16bit<false>(o0 + 64, f1, v32);
            if (a.dqkv32) {
              float* p0 = a.dqkv32 + r + dcol + c * 32;
              store32_f32(p0, f0, v32);
              store32_f32(p0 + 64, f1, v32);
            }
          }
        }
      }
    }
  }
  attn_teardown(abort_flag, warp, tmem);
}

// ======================================================= backward pass 2: dQ
// Shared memory: Q and dO of the tile (32 KB each, 128 rows), NS stages of
// (K block | V block) (64 rows: 16 KB each), 2 dS buffers ([128 queries, 64
// keys] fp16, 16 KB each).
constexpr int B2_NS = 3;
constexpr int B2_Q = 0, B2_O = 32768, B2_ST = 65536;
constexpr int B2_STAGE = 32768;
constexpr int B2_DS = B2_ST + B2_NS * B2_STAGE;
constexpr int B2_BAR = B2_DS + 2 * 16384;
constexpr int B2_SMEM = B2_BAR + 256 + 1024;

// One CTA of pass 2 (query tile nqt - 1 - bx of sequence bz, q head by).
__device__ __forceinline__ void attn_bwd_dq_cta(const CUtensorMap& tm128, const CUtensorMap& tm64,
                                                const CUtensorMap& tmdo128, const AttnArgs& a, int bx, int by,
                                                int bz) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + B2_BAR);
  uint64_t* qo_full = bars;               // 1
  uint64_t* full = bars + 1;              // [NS]
  uint64_t* empty = full + B2_NS;         // [NS]
  uint64_t* st_full = empty + B2_NS;      // [2]
  uint64_t* st_free = st_full + 2;        // [2]
  uint64_t* ds_full = st_free + 2;        // [2]
  uint64_t* ds_empty = ds_full + 2;       // [2]
  uint64_t* acc_full = ds_empty + 2;      // 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int S = a.S;
  const int nqt = (S + 127) / 128;
  const int qb = nqt - 1 - bx;  // the longest rows first
  const int h = by, v = bz;     // q head, sequence
  if (v % a.G != 0 && qb * 128 < a.Lp) return;  // shared-prefix queries: sequence 0 of the group
  const int g = h / (a.Hq / a.Hkv);
  const int kcol = (a.Hq + g) * HD, vcol = (a.Hq + a.Hkv + g) * HD;
  const int n_it = min(2 * qb + 2, (S + 63) / 64);  // 64-key blocks up to the diagonal and the sequence end
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    ptx::mbar_init(qo_full, 1);
    for (int i = 0; i < B2_NS; ++i) {
      ptx::mbar_init(&full[i], 1);
      ptx::mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&st_full[i], 1);
      ptx::mbar_init(&st_free[i], 8);
      ptx::mbar_init(&ds_full[i], 8);
      ptx::mbar_init(&ds_empty[i], 1);
    }
    ptx::mbar_init(acc_full, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tm128);
    ptx::prefetch_tmap(&tm64);
    ptx::prefetch_tmap(&tmdo128);
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  // columns: S[0] 0, S[1] 64, dP[0] 128, dP[1] 192, dQ 256
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      const int qrow = vrow(a, v, qb * 128);
      ptx::mbar_arrive_expect_tx(qo_full, 65536);
      ptx::tma_load_2d(sm + B2_Q, &tm128, qo_full, h * HD, qrow);
      ptx::tma_load_2d(sm + B2_Q + 16384, &tm128, qo_full, h * HD + 64, qrow);
      ptx::tma_load_2d(sm + B2_O, &tmdo128, qo_full, h * HD, qrow);
      ptx::tma_load_2d(sm + B2_O + 16384, &tmdo128, qo_full, h * HD + 64, qrow);
      for (int j = 0; j < n_it; ++j) {
        const int s = j % B2_NS;
        const uint32_t ph = (j / B2_NS) & 1;
        if (!ATTN_WAIT(&empty[s], ph ^ 1)) break;
        uint8_t* st = sm + B2_ST + s * B2_STAGE;
        const int r = vrow(a, v, j * 64);
        ptx::mbar_arrive_expect_tx(&full[s], 32768);
        ptx::tma_load_2d(st, &tm64, &full[s], kcol, r);
        ptx::tma_load_2d(st + 8192, &tm64, &full[s], kcol + 64, r);
        ptx::tma_load_2d(st + 16384, &tm64, &full[s], vcol, r);
        ptx::tma_load_2d(st + 24576, &tm64, &full[s], vcol + 64, r);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t id_s = ptx::idesc_fmt(128, 64, 0, 0, 0u);    // S, dP: [128 queries, 64 keys]
      constexpr uint32_t id_q = ptx::idesc_fmt(128, 128, 0, 1, 0u);   // dQ: B (K) MN-major
      const uint32_t qa = ptx::smem_u32(sm + B2_Q), oa = ptx::smem_u32(sm + B2_O);
      bool ok = ATTN_WAIT(qo_full, 0);
      for (int jj = 0; ok && jj <= n_it; ++jj) {
        if (jj < n_it) {
          const int s = jj % B2_NS, bb = jj & 1;
          const uint32_t ph = (jj / B2_NS) & 1, pb = (jj >> 1) & 1;
          if (!ATTN_WAIT(&full[s], ph) || !ATTN_WAIT(&st_free[bb], pb ^ 1)) break;
          ptx::tc_fence_after();
          const uint32_t ka = ptx::smem_u32(sm + B2_ST + s * B2_STAGE), va = ka + 16384;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t off = (k >> 2) * 8192 + (k & 3) * 32;
            ptx::mma_bf16(tmem + bb * 64, kdesc(qa + (k >> 2) * 16384 + (k & 3) * 32), kdesc(ka + off), id_s,
                          k > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t off = (k >> 2) * 8192 + (k & 3) * 32;
            ptx::mma_bf16(tmem + 128 + bb * 64, kdesc(oa + (k >> 2) * 16384 + (k & 3) * 32), kdesc(va + off), id_s,
                          k > 0 ? 1u : 0u);
          }
          ptx::mma_commit(&st_full[bb]);
        }
        if (jj >= 1) {  // dQ += dS_j K_j, j = jj - 1
          const int j = jj - 1, s = j % B2_NS, bb = j & 1;
          const uint32_t pb = (j >> 1) & 1;
          if (!ATTN_WAIT(&ds_full[bb], pb)) break;
          ptx::tc_fence_after();
          const uint32_t ka = ptx::smem_u32(sm + B2_ST + s * B2_STAGE);
          const uint32_t da = ptx::smem_u32(sm + B2_DS + bb * 16384);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            ptx::mma_bf16(tmem + 256, kdesc(da + k * 32), mndesc(ka + k * 2048, 8192), id_q,
                          (j > 0 || k > 0) ? 1u : 0u);
          ptx::mma_commit(&ds_empty[bb]);
          ptx::mma_commit(&empty[s]);
        }
      }
      if (ok) ptx::mma_commit(acc_full);
    }
  } else {
    // ---------------- elementwise warps: two per query row, 32 keys each
    const int quad = warp & 3, half = (warp - 2) >> 2;
    const int row = quad * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
    const int qi = qb * 128 + row;
    const bool qin = qi < S;
    const int prow = qin ? vrow(a, v, qi) : 0;
    const float Lr = qin ? a.L[(size_t)h * a.T + prow] : 0.f;
    const float Dr = qin ? a.D[(size_t)h * a.T + prow] : 0.f;
    const float sl2 = a.scale_log2;
    bool ok = true;
    for (int j = 0; j < n_it; ++j) {
      const int bb = j & 1;
      const uint32_t pb = (j >> 1) & 1;
      const int key0 = j * 64;
      if (!ATTN_WAIT(&st_full[bb], pb)) { ok = false; break; }
      ptx::tc_fence_after();
      if (!ATTN_WAIT(&ds_empty[bb], pb ^ 1)) { ok = false; break; }
      uint8_t* DS = sm + B2_DS + bb * 16384;
      const bool edge = key0 + 63 > qi || key0 + 64 > S || !qin;
      {
        const int c = half;  // this warp's 32 keys of the block
        uint32_t sv[32], dv[32];
        ptx::tmem_ld32(tl + bb * 64 + c * 32, sv);
        ptx::tmem_ld32(tl + 128 + bb * 64 + c * 32, dv);
        ptx::tmem_ld_wait();
        uint32_t dk[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float d[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int key = key0 + c * 32 + i + e;
            float x = fmaf(__uint_as_float(sv[i + e]), sl2, -Lr);
            if (edge && (key > qi || key >= S || !qin)) x = -INFINITY;
            const float p = ex2(x);
            d[e] = p * (__uint_as_float(dv[i + e]) - Dr);
          }
          dk[i >> 1] = pack_h2(d[0], d[1]);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) st_unit(DS, row, c * 4 + u, dk[4 * u], dk[4 * u + 1], dk[4 * u + 2], dk[4 * u + 3]);
      }
      ptx::tc_fence_before();
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        ptx::mbar_arrive(&st_free[bb]);
        ptx::mbar_arrive(&ds_full[bb]);
      }
    }
    if (ok && ATTN_WAIT(acc_full, 0)) {
      ptx::tc_fence_after();
      const float unscale = a.amax ? 1.f / grad_scale_from_amax(__uint_as_float(*a.amax)) : 1.f;
      const float mul = a.scale * unscale;
      const size_t r = (size_t)prow * a.ld + h * HD;
      {
        const int c = half;  // pairs (c*32 + i, c*32 + i + 64)
        uint32_t v0[32], v1[32];
        ptx::tmem_ld32(tl + 256 + c * 32, v0);
        ptx::tmem_ld32(tl + 256 + 64 + c * 32, v1);
        ptx::tmem_ld_wait();
        float f0[32], f1[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          f0[i] = __uint_as_float(v0[i]) * mul;
          f1[i] = __uint_as_float(v1[i]) * mul;
        }
        if (qin) {
          const bool v32 = a.v32 != 0;
          if (a.rcos) {
            float cs[32], sn[32];
            load32_f32(a.rcos + (size_t)qi * 64 + c * 32, cs, v32);
            load32_f32(a.rsin + (size_t)qi * 64 + c * 32, sn, v32);
#pragma unroll
            for (int i = 0; i < 32; ++i) rope_back(f0[i], f1[i], cs[i], sn[i]);
          }
          uint16_t* o0 = a.dqkv + r + c * 32;
          store32_16bit<false>(o0, f0, v32);
          store32_16bit<false>(o0 + 64, f1, v32);
          if (a.dqkv32) {
            float* p0 = a.dqkv32 + r + c * 32;
            store32_f32(p0, f0, v32);
            store32_f32(p0 + 64, f1, v32);
          }
        }
      }
    }
  }
  attn_teardown(abort_flag, warp, tmem);
}

// Both backward passes in one launch (they write disjoint columns of dq|dk|dv
// and only read the forward's outputs): CTAs [0, n1) are pass-1 key blocks,
// heaviest (most query tiles) first, the rest pass-2 query tiles, longest
// first, so the scheduler fills the SMs the uneven causal pass 1 leaves.
constexpr int B_SMEM = B1_SMEM > B2_SMEM ? B1_SMEM : B2_SMEM;
__global__ void __launch_bounds__(320, 1) attn_bwd_tc(const __grid_constant__ CUtensorMap tm128,
                                                      const __grid_constant__ CUtensorMap tm64,
                                                      const __grid_constant__ CUtensorMap tmdo64,
                                                      const __grid_constant__ CUtensorMap tmdo128, const AttnArgs a,
                                                      int x1, int y1, int z1, int y2, int z2) {
  int i = (int)blockIdx.x;
  const int n1 = x1 * y1 * z1;
  if (i < n1) {
    const int yz = y1 * z1;
    attn_bwd_dkdv_cta(tm128, tm64, tmdo64, a, i / yz, (i % yz) % y1, (i % yz) / y1);
  } else {
    i -= n1;
    const int yz = y2 * z2;
    attn_bwd_dq_cta(tm128, tm64, tmdo128, a, i / yz, (i % yz) % y2, (i % yz) / y2);
  }
}

#undef ATTN_WAIT

// 2-D fp16 tensor map over [rows, cols] (row stride ld elements), box of
// 64 columns (128 bytes) x box_rows rows, 128-byte swizzle.
soup_status fp16_map(CUtensorMap* m, const uint16_t* p, int64_t rows, int64_t cols, int64_t ld, uint32_t box_rows,
                     const char* what) {
  SOUP_CHECK(p && rows > 0 && cols > 0, SOUP_ERR_INVALID_ARG, "attention: %s is empty", what);
  SOUP_CHECK(soup_aligned(p, 16) && (ld * 2) % 16 == 0, SOUP_ERR_ALIGN, "attention: %s base / row stride alignment",
             what);
  EncodeTiledFn enc = encode_tiled();
  SOUP_CHECK(enc != nullptr, SOUP_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const uint64_t gdim[2] = {(uint64_t)cols, (uint64_t)rows};
  const uint64_t gstride[1] = {(uint64_t)(ld * 2)};
  const uint32_t box[2] = {64, box_rows};
  const uint32_t estr[2] = {1, 1};
  const int r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<uint16_t*>(p), gdim, gstride, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  SOUP_CHECK(r == 0, SOUP_ERR_CUDA, "cuTensorMapEncodeTiled(%s) failed with %d", what, r);
  return SOUP_OK;
}

soup_status attn_init() {
  static bool init = false;
  if (!init) {
    SOUP_CUDA_TRY(cudaFuncSetAttribute(attn_fwd_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, F_SMEM));
    SOUP_CUDA_TRY(cudaFuncSetAttribute(attn_bwd_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, B_SMEM));
    init = true;
  }
  return SOUP_OK;
}

soup_status attn_check(int ld, int Bsz, int S, int Hq, int Hkv, int G, int Lp) {
  SOUP_CHECK(Hkv > 0 && Hq % Hkv == 0 && S > 0 && Bsz > 0, SOUP_ERR_SHAPE, "attention: bad heads/shape");
  SOUP_CHECK(ld >= (Hq + 2 * Hkv) * HD && ld % 8 == 0, SOUP_ERR_SHAPE, "attention: row stride %d", ld);
  SOUP_CHECK((int64_t)Bsz * S < (1LL << 31), SOUP_ERR_SHAPE, "attention: too many tokens");
  SOUP_CHECK(G >= 1 && Bsz % G == 0 && (G == 1 ? Lp == 0 : (Lp > 0 && Lp < S && Lp % 128 == 0)), SOUP_ERR_SHAPE,
             "attention: prefix sharing needs groups of G sequences dividing the batch and a shared prefix that is "
             "a positive multiple of 128 shorter than the sequence (G=%d, prefix %d, seq %d)", G, Lp, S);
  return SOUP_OK;
}

// Token rows of Bsz sequences of S tokens in groups of G sharing Lp.
int attn_rows(int Bsz, int S, int G, int Lp) { return (Bsz / G) * (Lp + G * (S - Lp)); }

}  // namespace

soup_status attention_fwd(const uint16_t* qkv, int ld, int Bsz, int S, int Hq, int Hkv, uint16_t* out, float* lse,
                          cudaStream_t st, uint16_t* out16, float* out32, int G, int Lp) {
  SOUP_TRY(attn_check(ld, Bsz, S, Hq, Hkv, G, Lp));
  SOUP_CHECK(soup_aligned(qkv, 16) && soup_aligned(out, 16) && (!out16 || soup_aligned(out16, 16)) &&
                 (!out32 || soup_aligned(out32, 16)) && lse,
             SOUP_ERR_ALIGN, "attention: alignment");
  SOUP_TRY(attn_init());
  const int T = attn_rows(Bsz, S, G, Lp);
  CUtensorMap tm;
  SOUP_TRY(fp16_map(&tm, qkv, T, (Hq + 2 * Hkv) * HD, ld, 128, "q|k|v"));
  AttnArgs a;
  memset(&a, 0, sizeof(a));
  a.S = S; a.Hq = Hq; a.Hkv = Hkv; a.T = T; a.G = G; a.Lp = Lp;
  a.scale = 1.0f / sqrtf((float)HD);
  a.scale_log2 = 1.4426950408889634f * a.scale;
  a.out = out; a.lse = lse; a.out16 = out16; a.out32 = out32;
  a.v32 = soup_aligned(out, 32) && (!out16 || soup_aligned(out16, 32)) && (!out32 || soup_aligned(out32, 32));
  a.err = device_error_word();
  SOUP_CHECK(a.err, SOUP_ERR_CUDA, "device error word unavailable");
  a.wait_limit = 4000000000LL;
  const double fl = 4.0 * Bsz * Hq * (double)HD * ((double)S * (S + 1) / 2);
  profile_begin(st, GC_ATTN, fl, 0.0);
  a.nseq = Bsz;
  attn_fwd_tc<<<((S + 127) / 128) * Hq * Bsz, 320, F_SMEM, st>>>(tm, a);
  SOUP_LAUNCH_CHECK();
  profile_end(st);
  return SOUP_OK;
}

soup_status attention_bwd(const uint16_t* qkv, int ld, int Bsz, int S, int Hq, int Hkv, const uint16_t* dout,
                          const float* lse, const float* D, uint16_t* dqkv, const float* rope_cos,
                          const float* rope_sin, const unsigned int* amax, cudaStream_t st, float* dqkv32, int G,
                          int Lp) {
  SOUP_TRY(attn_check(ld, Bsz, S, Hq, Hkv, G, Lp));
  SOUP_CHECK(soup_aligned(qkv, 16) && soup_aligned(dout, 16) && soup_aligned(dqkv, 16) &&
                 (!dqkv32 || soup_aligned(dqkv32, 16)) && lse && D,
             SOUP_ERR_ALIGN, "attention backward: alignment");
  SOUP_CHECK(!rope_cos == !rope_sin, SOUP_ERR_INVALID_ARG, "attention backward: RoPE tables go together");
  SOUP_TRY(attn_init());
  const int T = attn_rows(Bsz, S, G, Lp);
  CUtensorMap tm128, tm64, tmdo64, tmdo128;
  SOUP_TRY(fp16_map(&tm128, qkv, T, (Hq + 2 * Hkv) * HD, ld, 128, "q|k|v"));
  SOUP_TRY(fp16_map(&tm64, qkv, T, (Hq + 2 * Hkv) * HD, ld, 64, "q|k|v"));
  SOUP_TRY(fp16_map(&tmdo64, dout, T, Hq * HD, Hq * HD, 64, "dO"));
  SOUP_TRY(fp16_map(&tmdo128, dout, T, Hq * HD, Hq * HD, 128, "dO"));
  AttnArgs a;
  memset(&a, 0, sizeof(a));
  a.S = S; a.Hq = Hq; a.Hkv = Hkv; a.T = T; a.G = G; a.Lp = Lp;
  a.scale = 1.0f / sqrtf((float)HD);
  a.scale_log2 = 1.4426950408889634f * a.scale;
  a.L = lse; a.D = D; a.dqkv = dqkv; a.dqkv32 = dqkv32; a.ld = ld;
  a.rcos = rope_cos; a.rsin = rope_sin; a.amax = amax;
  a.v32 = soup_aligned(dqkv, 32) && (!dqkv32 || soup_aligned(dqkv32, 32)) && (ld * 2) % 32 == 0 &&
          (!rope_cos || (soup_aligned(rope_cos, 32) && soup_aligned(rope_sin, 32)));
  a.err = device_error_word();
  SOUP_CHECK(a.err, SOUP_ERR_CUDA, "device error word unavailable");
  a.wait_limit = 4000000000LL;
  const double fl = 2.5 * 4.0 * Bsz * Hq * (double)HD * ((double)S * (S + 1) / 2);
  profile_begin(st, GC_ATTN, fl, 0.0);
  const int x1 = Lp / 128 + G * ((S - Lp + 127) / 128), y1 = Hkv, z1 = Bsz / G;  // pass 1
  const int x2 = (S + 127) / 128, y2 = Hq, z2 = Bsz;                              // pass 2
  attn_bwd_tc<<<x1 * y1 * z1 + x2 * y2 * z2, 320, B_SMEM, st>>>(tm128, tm64, tmdo64, tmdo128, a, x1, y1, z1, y2, z2);
  SOUP_LAUNCH_CHECK();
  profile_end(st);
  return SOUP_OK;
}

}  // namespace soup

using namespace soup;

extern "C" soup_status soup_attention_fwd(const uint16_t* qkv, int64_t ld, int64_t batch, int64_t seq, int32_t n_q_heads,
                                          int32_t n_kv_heads, int32_t prefix_share, int64_t prefix_len, uint16_t* out,
                                          uint16_t* out16, float* lse, void* stream) {
  SOUP_CHECK(qkv && out && lse, SOUP_ERR_INVALID_ARG, "soup_attention_fwd: null pointer");
  SOUP_CHECK(batch > 0 && seq > 0 && batch * seq < (1LL << 31) && ld > 0 && ld < (1LL << 31), SOUP_ERR_SHAPE,
             "soup_attention_fwd: bad shape");
  SOUP_CHECK(prefix_len >= 0 && prefix_len < seq, SOUP_ERR_SHAPE, "soup_attention_fwd: prefix length");
  const int G = prefix_share > 1 ? prefix_share : 1;
  return attention_fwd(qkv, (int)ld, (int)batch, (int)seq, n_q_heads, n_kv_heads, out, lse,
                       static_cast<cudaStream_t>(stream), out16, nullptr, G, G > 1 ? (int)prefix_len : 0);
}

extern "C" soup_status soup_attention_bwd(const uint16_t* qkv, int64_t ld, int64_t batch, int64_t seq,
                                          int32_t n_q_heads, int32_t n_kv_heads, int32_t prefix_share,
                                          int64_t prefix_len, const uint16_t* out16,
                                          const uint16_t* dout, const float* lse, float* D, uint16_t* dqkv,
                                          float* dqkv32, void* stream) {
  SOUP_CHECK(qkv && out16 && dout && lse && D && dqkv, SOUP_ERR_INVALID_ARG, "soup_attention_bwd: null pointer");
  SOUP_CHECK(batch > 0 && seq > 0 && batch * seq < (1LL << 31) && ld > 0 && ld < (1LL << 31), SOUP_ERR_SHAPE,
             "soup_attention_bwd: bad shape");
  SOUP_CHECK(prefix_len >= 0 && prefix_len < seq, SOUP_ERR_SHAPE, "soup_attention_bwd: prefix length");
  const int G = prefix_share > 1 ? prefix_share : 1;
  const int Lp = G > 1 ? (int)prefix_len : 0;
  SOUP_TRY(attn_check((int)ld, (int)batch, (int)seq, n_q_heads, n_kv_heads, G, Lp));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SOUP_TRY(attn_rowdot(dout, out16, attn_rows((int)batch, (int)seq, G, Lp), n_q_heads, D, st));
  return attention_bwd(qkv, (int)ld, (int)batch, (int)seq, n_q_heads, n_kv_heads, dout, lse, D, dqkv, nullptr,
                       nullptr, nullptr, st, dqkv32, G, Lp);
}
