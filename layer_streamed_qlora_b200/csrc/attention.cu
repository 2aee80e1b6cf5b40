// Causal GQA attention (head_dim 128) for the decoder layer: flash-style
// forward with online softmax, and a two-pass backward that needs no atomics
// (pass 1: dK, dV per key block, summing the q heads of the group in a fixed
// order; pass 2: dQ per query block), so every run gives the same bits.
//
// Tensor-core path: warp-level mma.sync m16n8k16 with fp16 operands and fp32
// accumulation, ldmatrix operand loads from padded shared-memory tiles;
// softmax in fp32 in the log2 domain; the saved log-sum-exp is in log2 units.
// Inputs q, k, v and dO are fp16 (the projections write them in fp16: same
// 16-bit traffic as bf16 with 8x finer rounding for these O(1) values), the
// probabilities P and dS enter the MMAs as fp16; outputs (attention output,
// dq, dk, dv) are bf16, the operand type of the projection GEMMs.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "elementwise.h"
#include "gscale.cuh"

namespace soup {
namespace {

constexpr int HD = 128;   // head dim
constexpr int LDS = 136;  // padded smem row (elements): conflict-free ldmatrix

__device__ __forceinline__ uint32_t su32(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(su32(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(su32(p)));
}
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t packbf(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ uint32_t packh(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(su32(dst)), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Loads `rows` rows of a head (128 bf16 each) starting at token row `r0` of
// sequence-local index `s0` (rows with s0 + r >= S are zero-filled).
__device__ __forceinline__ void load_tile(uint16_t* dst, const uint16_t* base, int ld, int col, int r0, int s0,
                                          int S, int rows, int tid, int nthr) {
  for (int idx = tid; idx < rows * 16; idx += nthr) {
    const int r = idx >> 4, c = (idx & 15) * 8;
    const bool ok = (s0 + r) < S;
    const uint16_t* src = base + (size_t)(ok ? r0 + r : r0) * ld + col + c;
    cp_async16(dst + r * LDS + c, src, ok);
  }
}

// A fragment (16x16) address for this lane from a row-major tile.
__device__ __forceinline__ const uint16_t* a_addr(const uint16_t* tile, int row0, int col0, int lane) {
  const int mi = lane >> 3, ri = lane & 7;
  return tile + (row0 + (mi & 1) * 8 + ri) * LDS + col0 + (mi >> 1) * 8;
}
// Two B fragments (n-tiles n0, n0+8; k16) from a tile stored [n][k] (non-trans).
__device__ __forceinline__ const uint16_t* bn_addr(const uint16_t* tile, int n0, int k0, int lane) {
  const int mi = lane >> 3, ri = lane & 7;
  return tile + (n0 + (mi >> 1) * 8 + ri) * LDS + k0 + (mi & 1) * 8;
}
// Two B fragments (n-tiles n0, n0+8; k16) from a tile stored [k][n] (trans).
__device__ __forceinline__ const uint16_t* bk_addr(const uint16_t* tile, int k0, int n0, int lane) {
  const int mi = lane >> 3, ri = lane & 7;
  return tile + (k0 + (mi & 1) * 8 + ri) * LDS + n0 + (mi >> 1) * 8;
}


// Stores one row (this lane's 16 x 2 columns of a 128-wide head) scaled by
// `scale`, rotating pairs (i, i+64) back by the position's angle when tables
// are given: (a, b) -> (a c + b s, b c - a s).
__device__ __forceinline__ void store_row_rot(uint16_t* p, const float (&acc)[16][4], int e0, float scale,
                                              const float* cosr, const float* sinr, int t4, float* p32 = nullptr) {
#pragma unroll
  for (int dt = 0; dt < 8; ++dt) {
    float a0 = acc[dt][e0] * scale, a1 = acc[dt][e0 + 1] * scale;
    float b0 = acc[dt + 8][e0] * scale, b1 = acc[dt + 8][e0 + 1] * scale;
    if (cosr) {
      const int c = dt * 8 + 2 * t4;
      const float c0 = cosr[c], c1 = cosr[c + 1], s0 = sinr[c], s1 = sinr[c + 1];
      const float ra0 = a0 * c0 + b0 * s0, rb0 = b0 * c0 - a0 * s0;
      const float ra1 = a1 * c1 + b1 * s1, rb1 = b1 * c1 - a1 * s1;
      a0 = ra0; a1 = ra1; b0 = rb0; b1 = rb1;
    }
    *reinterpret_cast<uint32_t*>(p + dt * 8 + 2 * t4) = packbf(a0, a1);
    *reinterpret_cast<uint32_t*>(p + 64 + dt * 8 + 2 * t4) = packbf(b0, b1);
    if (p32) {
      *reinterpret_cast<float2*>(p32 + dt * 8 + 2 * t4) = make_float2(a0, a1);
      *reinterpret_cast<float2*>(p32 + 64 + dt * 8 + 2 * t4) = make_float2(b0, b1);
    }
  }
}

// ------------------------------------------------------------------ forward
__global__ void __launch_bounds__(128) attn_fwd_kernel(const uint16_t* __restrict__ qkv, int ld, int S, int Hq,
                                                        int Hkv, uint16_t* __restrict__ out,
                                                        float* __restrict__ lse, float scale_log2,
                                                        uint16_t* __restrict__ out16, float* __restrict__ out32) {
  extern __shared__ __align__(16) uint16_t sm[];
  uint16_t* Qs = sm;
  uint16_t* Ks = Qs + 64 * LDS;   // 2 buffers
  uint16_t* Vs = Ks + 2 * 64 * LDS;
  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g4 = lane >> 2, t4 = lane & 3;
  const int T = gridDim.z * S;
  const int grp = Hq / Hkv, kvh = h / grp;
  const int qcol = h * HD, kcol = (Hq + kvh) * HD, vcol = (Hq + Hkv + kvh) * HD;
  const int row0 = b * S;
  load_tile(Qs, qkv, ld, qcol, row0 + qb * 64, qb * 64, S, 64, tid, 128);
  load_tile(Ks, qkv, ld, kcol, row0, 0, S, 64, tid, 128);
  load_tile(Vs, qkv, ld, vcol, row0, 0, S, 64, tid, 128);
  cp_commit();
  cp_wait<0>();
  __syncthreads();
  uint32_t qf[8][4];
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) ldsm_x4(qf[kk], a_addr(Qs, warp * 16, kk * 16, lane));
  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const int qr0 = qb * 64 + warp * 16 + g4, qr1 = qr0 + 8;
  const int nkb = qb + 1;
  for (int j = 0; j < nkb; ++j) {
    if (j + 1 < nkb) {
      load_tile(Ks + ((j + 1) & 1) * 64 * LDS, qkv, ld, kcol, row0 + (j + 1) * 64, (j + 1) * 64, S, 64, tid, 128);
      load_tile(Vs + ((j + 1) & 1) * 64 * LDS, qkv, ld, vcol, row0 + (j + 1) * 64, (j + 1) * 64, S, 64, tid, 128);
      cp_commit();
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
    const uint16_t* Kb = Ks + (j & 1) * 64 * LDS;
    const uint16_t* Vb = Vs + (j & 1) * 64 * LDS;
    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
      for (int nt2 = 0; nt2 < 4; ++nt2) {
        uint32_t bf[4];
        ldsm_x4(bf, bn_addr(Kb, nt2 * 16, kk * 16, lane));
        mma16816(s[2 * nt2], qf[kk], bf[0], bf[1]);
        mma16816(s[2 * nt2 + 1], qf[kk], bf[2], bf[3]);
      }
    }
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = j * 64 + nt * 8 + 2 * t4 + (e & 1);
        const int qr = (e < 2) ? qr0 : qr1;
        float v = s[nt][e] * scale_log2;
        if (key > qr || key >= S) v = -INFINITY;
        s[nt][e] = v;
      }
      mx0 = fmaxf(mx0, fmaxf(s[nt][0], s[nt][1]));
      mx1 = fmaxf(mx1, fmaxf(s[nt][2], s[nt][3]));
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float c0 = (mn0 == -INFINITY) ? 1.f : exp2f(m0 - mn0);
    const float c1 = (mn1 == -INFINITY) ? 1.f : exp2f(m1 - mn1);
    m0 = mn0;
    m1 = mn1;
    float sum0 = 0.f, sum1 = 0.f;
    uint32_t pa[4][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const float p0 = (s[nt][0] == -INFINITY) ? 0.f : exp2f(s[nt][0] - mn0);
      const float p1 = (s[nt][1] == -INFINITY) ? 0.f : exp2f(s[nt][1] - mn0);
      const float p2 = (s[nt][2] == -INFINITY) ? 0.f : exp2f(s[nt][2] - mn1);
      const float p3 = (s[nt][3] == -INFINITY) ? 0.f : exp2f(s[nt][3] - mn1);
      sum0 += p0 + p1;
      sum1 += p2 + p3;
      pa[nt >> 1][(nt & 1) * 2 + 0] = packh(p0, p1);
      pa[nt >> 1][(nt & 1) * 2 + 1] = packh(p2, p3);
    }
    l0 = l0 * c0 + sum0;
    l1 = l1 * c1 + sum1;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      o[i][0] *= c0; o[i][1] *= c0; o[i][2] *= c1; o[i][3] *= c1;
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
      for (int dt2 = 0; dt2 < 8; ++dt2) {
        uint32_t bf[4];
        ldsm_x4_t(bf, bk_addr(Vb, kk * 16, dt2 * 16, lane));
        mma16816(o[2 * dt2], pa[kk], bf[0], bf[1]);
        mma16816(o[2 * dt2 + 1], pa[kk], bf[2], bf[3]);
      }
    }
    __syncthreads();
  }
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float i0 = 1.f / l0, i1 = 1.f / l1;
  const int ldo = Hq * HD;
  if (qr0 < S) {
    const size_t off = (size_t)(row0 + qr0) * ldo + h * HD;
#pragma unroll
    for (int dt = 0; dt < 16; ++dt) {
      *reinterpret_cast<uint32_t*>(out + off + dt * 8 + 2 * t4) = packbf(o[dt][0] * i0, o[dt][1] * i0);
      if (out16) *reinterpret_cast<uint32_t*>(out16 + off + dt * 8 + 2 * t4) = packh(o[dt][0] * i0, o[dt][1] * i0);
      if (out32) *reinterpret_cast<float2*>(out32 + off + dt * 8 + 2 * t4) = make_float2(o[dt][0] * i0, o[dt][1] * i0);
    }
    if (t4 == 0) lse[(size_t)h * T + row0 + qr0] = m0 + log2f(l0);
  }
  if (qr1 < S) {
    const size_t off = (size_t)(row0 + qr1) * ldo + h * HD;
#pragma unroll
    for (int dt = 0; dt < 16; ++dt) {
      *reinterpret_cast<uint32_t*>(out + off + dt * 8 + 2 * t4) = packbf(o[dt][2] * i1, o[dt][3] * i1);
      if (out16) *reinterpret_cast<uint32_t*>(out16 + off + dt * 8 + 2 * t4) = packh(o[dt][2] * i1, o[dt][3] * i1);
      if (out32) *reinterpret_cast<float2*>(out32 + off + dt * 8 + 2 * t4) = make_float2(o[dt][2] * i1, o[dt][3] * i1);
    }
    if (t4 == 0) lse[(size_t)h * T + row0 + qr1] = m1 + log2f(l1);
  }
}

// --------------------------------------------------- backward pass 1: dK, dV
// CTA = 64 keys (4 warps x 16) of one kv head; loops over the group's q heads
// and over query blocks of 32 at or after the key block.
__global__ void __launch_bounds__(128) attn_bwd_dkdv_kernel(const uint16_t* __restrict__ qkv, int ld, int S, int Hq,
                                                             int Hkv, const uint16_t* __restrict__ dout,
                                                             const float* __restrict__ lse,
                                                             const float* __restrict__ Dd,
                                                             uint16_t* __restrict__ dqkv, float scale_log2,
                                                             float scale, const float* __restrict__ rcos,
                                                             const float* __restrict__ rsin,
                                                             const unsigned int* __restrict__ amax,
                                                             float* __restrict__ dqkv32) {
  extern __shared__ __align__(16) uint16_t sm[];
  uint16_t* Ks = sm;
  uint16_t* Vs = Ks + 64 * LDS;
  uint16_t* Qs = Vs + 64 * LDS;        // 2 x 32 rows
  uint16_t* Os = Qs + 2 * 32 * LDS;    // dO, 2 x 32 rows
  float* Ls = reinterpret_cast<float*>(Os + 2 * 32 * LDS);  // 2 x 32
  float* Ds = Ls + 64;                                       // 2 x 32
  const int kb = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g4 = lane >> 2, t4 = lane & 3;
  const int T = gridDim.z * S;
  const int grp = Hq / Hkv;
  const int kcol = (Hq + kvh) * HD, vcol = (Hq + Hkv + kvh) * HD;
  const int row0 = b * S;
  const int ldo = Hq * HD;
  load_tile(Ks, qkv, ld, kcol, row0 + kb * 64, kb * 64, S, 64, tid, 128);
  load_tile(Vs, qkv, ld, vcol, row0 + kb * 64, kb * 64, S, 64, tid, 128);
  cp_commit();
  const int qb_first = (kb * 64) / 32;
  const int nqb = (S + 31) / 32;
  const int per_head = nqb - qb_first;
  const int n_it = per_head * grp;
  auto issue = [&](int it, int buf) {
    const int hh = it / per_head, qb2 = qb_first + it % per_head;
    const int h = kvh * grp + hh;
    load_tile(Qs + buf * 32 * LDS, qkv, ld, h * HD, row0 + qb2 * 32, qb2 * 32, S, 32, tid, 128);
    load_tile(Os + buf * 32 * LDS, dout, ldo, h * HD, row0 + qb2 * 32, qb2 * 32, S, 32, tid, 128);
    if (tid < 32) {
      const int q = qb2 * 32 + tid;
      Ls[buf * 32 + tid] = (q < S) ? lse[(size_t)h * T + row0 + q] : 0.f;
      Ds[buf * 32 + tid] = (q < S) ? Dd[(size_t)h * T + row0 + q] : 0.f;
    }
  };
  float dk[16][4], dv[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    dk[i][0] = dk[i][1] = dk[i][2] = dk[i][3] = 0.f;
    dv[i][0] = dv[i][1] = dv[i][2] = dv[i][3] = 0.f;
  }
  const int key0 = kb * 64 + warp * 16 + g4, key1 = key0 + 8;
  if (n_it > 0) issue(0, 0);
  cp_commit();
  for (int it = 0; it < n_it; ++it) {
    const int buf = it & 1;
    if (it + 1 < n_it) {
      __syncthreads();  // everyone done with buffer buf^1 (iteration it-1)
      issue(it + 1, buf ^ 1);
      cp_commit();
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
    const int qb2 = qb_first + it % per_head;
    const uint16_t* Qb = Qs + buf * 32 * LDS;
    const uint16_t* Ob = Os + buf * 32 * LDS;
    const float* Lb = Ls + buf * 32;
    const float* Db = Ds + buf * 32;
    // S^T = K Q^T and dP^T = V dO^T  (16 keys x 32 queries)
    float st[4][4], dpt[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      st[i][0] = st[i][1] = st[i][2] = st[i][3] = 0.f;
      dpt[i][0] = dpt[i][1] = dpt[i][2] = dpt[i][3] = 0.f;
    }
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      uint32_t ka[4], va[4];
      ldsm_x4(ka, a_addr(Ks, warp * 16, kk * 16, lane));
      ldsm_x4(va, a_addr(Vs, warp * 16, kk * 16, lane));
#pragma unroll
      for (int nt2 = 0; nt2 < 2; ++nt2) {
        uint32_t bq[4], bo[4];
        ldsm_x4(bq, bn_addr(Qb, nt2 * 16, kk * 16, lane));
        ldsm_x4(bo, bn_addr(Ob, nt2 * 16, kk * 16, lane));
        mma16816(st[2 * nt2], ka, bq[0], bq[1]);
        mma16816(st[2 * nt2 + 1], ka, bq[2], bq[3]);
        mma16816(dpt[2 * nt2], va, bo[0], bo[1]);
        mma16816(dpt[2 * nt2 + 1], va, bo[2], bo[3]);
      }
    }
    uint32_t pa[2][4], da[2][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      float p[4], ds[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int ql = nt * 8 + 2 * t4 + (e & 1);
        const int q = qb2 * 32 + ql;
        const int key = (e < 2) ? key0 : key1;
        const bool ok = (q >= key) && (q < S) && (key < S);
        p[e] = ok ? exp2f(st[nt][e] * scale_log2 - Lb[ql]) : 0.f;
        ds[e] = p[e] * (dpt[nt][e] - Db[ql]);
      }
      pa[nt >> 1][(nt & 1) * 2 + 0] = packh(p[0], p[1]);
      pa[nt >> 1][(nt & 1) * 2 + 1] = packh(p[2], p[3]);
      da[nt >> 1][(nt & 1) * 2 + 0] = packh(ds[0], ds[1]);
      da[nt >> 1][(nt & 1) * 2 + 1] = packh(ds[2], ds[3]);
    }
    // dV += P^T dO ; dK += dS^T Q
#pragma unroll
    for (int kq = 0; kq < 2; ++kq) {
#pragma unroll
      for (int dt2 = 0; dt2 < 8; ++dt2) {
        uint32_t bo[4], bq[4];
        ldsm_x4_t(bo, bk_addr(Ob, kq * 16, dt2 * 16, lane));
        ldsm_x4_t(bq, bk_addr(Qb, kq * 16, dt2 * 16, lane));
        mma16816(dv[2 * dt2], pa[kq], bo[0], bo[1]);
        mma16816(dv[2 * dt2 + 1], pa[kq], bo[2], bo[3]);
        mma16816(dk[2 * dt2], da[kq], bq[0], bq[1]);
        mma16816(dk[2 * dt2 + 1], da[kq], bq[2], bq[3]);
      }
    }
  }
  // dO carried the power-of-two gradient scale: undo it (exact)
  const float unscale = amax ? 1.f / grad_scale_from_amax(__uint_as_float(*amax)) : 1.f;
  if (key0 < S) {
    const size_t r = (size_t)(row0 + key0) * ld;
    store_row_rot(dqkv + r + kcol, dk, 0, scale * unscale, rcos ? rcos + (size_t)key0 * 64 : nullptr,
                  rsin ? rsin + (size_t)key0 * 64 : nullptr, t4, dqkv32 ? dqkv32 + r + kcol : nullptr);
    store_row_rot(dqkv + r + vcol, dv, 0, unscale, nullptr, nullptr, t4, dqkv32 ? dqkv32 + r + vcol : nullptr);
  }
  if (key1 < S) {
    const size_t r = (size_t)(row0 + key1) * ld;
    store_row_rot(dqkv + r + kcol, dk, 2, scale * unscale, rcos ? rcos + (size_t)key1 * 64 : nullptr,
                  rsin ? rsin + (size_t)key1 * 64 : nullptr, t4, dqkv32 ? dqkv32 + r + kcol : nullptr);
    store_row_rot(dqkv + r + vcol, dv, 2, unscale, nullptr, nullptr, t4, dqkv32 ? dqkv32 + r + vcol : nullptr);
  }
}

// ------------------------------------------------------- backward pass 2: dQ
__global__ void __launch_bounds__(128) attn_bwd_dq_kernel(const uint16_t* __restrict__ qkv, int ld, int S, int Hq,
                                                           int Hkv, const uint16_t* __restrict__ dout,
                                                           const float* __restrict__ lse,
                                                           const float* __restrict__ Dd,
                                                           uint16_t* __restrict__ dqkv, float scale_log2,
                                                           float scale, const float* __restrict__ rcos,
                                                           const float* __restrict__ rsin,
                                                           const unsigned int* __restrict__ amax,
                                                           float* __restrict__ dqkv32) {
  extern __shared__ __align__(16) uint16_t sm[];
  uint16_t* Qs = sm;
  uint16_t* Os = Qs + 64 * LDS;
  uint16_t* Ks = Os + 64 * LDS;  // 2 buffers
  uint16_t* Vs = Ks + 2 * 64 * LDS;
  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g4 = lane >> 2, t4 = lane & 3;
  const int T = gridDim.z * S;
  const int grp = Hq / Hkv, kvh = h / grp;
  const int kcol = (Hq + kvh) * HD, vcol = (Hq + Hkv + kvh) * HD;
  const int row0 = b * S;
  const int ldo = Hq * HD;
  load_tile(Qs, qkv, ld, h * HD, row0 + qb * 64, qb * 64, S, 64, tid, 128);
  load_tile(Os, dout, ldo, h * HD, row0 + qb * 64, qb * 64, S, 64, tid, 128);
  load_tile(Ks, qkv, ld, kcol, row0, 0, S, 64, tid, 128);
  load_tile(Vs, qkv, ld, vcol, row0, 0, S, 64, tid, 128);
  cp_commit();
  const int qr0 = qb * 64 + warp * 16 + g4, qr1 = qr0 + 8;
  const float L0 = (qr0 < S) ? lse[(size_t)h * T + row0 + qr0] : 0.f;
  const float L1 = (qr1 < S) ? lse[(size_t)h * T + row0 + qr1] : 0.f;
  const float D0 = (qr0 < S) ? Dd[(size_t)h * T + row0 + qr0] : 0.f;
  const float D1 = (qr1 < S) ? Dd[(size_t)h * T + row0 + qr1] : 0.f;
  float dq[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) dq[i][0] = dq[i][1] = dq[i][2] = dq[i][3] = 0.f;
  const int nkb = qb + 1;
  for (int j = 0; j < nkb; ++j) {
    if (j + 1 < nkb) {
      load_tile(Ks + ((j + 1) & 1) * 64 * LDS, qkv, ld, kcol, row0 + (j + 1) * 64, (j + 1) * 64, S, 64, tid, 128);
      load_tile(Vs + ((j + 1) & 1) * 64 * LDS, qkv, ld, vcol, row0 + (j + 1) * 64, (j + 1) * 64, S, 64, tid, 128);
      cp_commit();
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
    const uint16_t* Kb = Ks + (j & 1) * 64 * LDS;
    const uint16_t* Vb = Vs + (j & 1) * 64 * LDS;
    float s[8][4], dp[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
      dp[i][0] = dp[i][1] = dp[i][2] = dp[i][3] = 0.f;
    }
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      uint32_t qa[4], oa[4];
      ldsm_x4(qa, a_addr(Qs, warp * 16, kk * 16, lane));
      ldsm_x4(oa, a_addr(Os, warp * 16, kk * 16, lane));
#pragma unroll
      for (int nt2 = 0; nt2 < 4; ++nt2) {
        uint32_t bk[4], bv[4];
        ldsm_x4(bk, bn_addr(Kb, nt2 * 16, kk * 16, lane));
        ldsm_x4(bv, bn_addr(Vb, nt2 * 16, kk * 16, lane));
        mma16816(s[2 * nt2], qa, bk[0], bk[1]);
        mma16816(s[2 * nt2 + 1], qa, bk[2], bk[3]);
        mma16816(dp[2 * nt2], oa, bv[0], bv[1]);
        mma16816(dp[2 * nt2 + 1], oa, bv[2], bv[3]);
      }
    }
    uint32_t da[4][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      float ds[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = j * 64 + nt * 8 + 2 * t4 + (e & 1);
        const int qr = (e < 2) ? qr0 : qr1;
        const bool ok = (key <= qr) && (key < S) && (qr < S);
        const float p = ok ? exp2f(s[nt][e] * scale_log2 - ((e < 2) ? L0 : L1)) : 0.f;
        ds[e] = p * (dp[nt][e] - ((e < 2) ? D0 : D1));
      }
      da[nt >> 1][(nt & 1) * 2 + 0] = packh(ds[0], ds[1]);
      da[nt >> 1][(nt & 1) * 2 + 1] = packh(ds[2], ds[3]);
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
      for (int dt2 = 0; dt2 < 8; ++dt2) {
        uint32_t bk[4];
        ldsm_x4_t(bk, bk_addr(Kb, kk * 16, dt2 * 16, lane));
        mma16816(dq[2 * dt2], da[kk], bk[0], bk[1]);
        mma16816(dq[2 * dt2 + 1], da[kk], bk[2], bk[3]);
      }
    }
    __syncthreads();
  }
  const float unscale = amax ? 1.f / grad_scale_from_amax(__uint_as_float(*amax)) : 1.f;
  if (qr0 < S) {
    const size_t r = (size_t)(row0 + qr0) * ld + h * HD;
    store_row_rot(dqkv + r, dq, 0, scale * unscale, rcos ? rcos + (size_t)qr0 * 64 : nullptr,
                  rsin ? rsin + (size_t)qr0 * 64 : nullptr, t4, dqkv32 ? dqkv32 + r : nullptr);
  }
  if (qr1 < S) {
    const size_t r = (size_t)(row0 + qr1) * ld + h * HD;
    store_row_rot(dqkv + r, dq, 2, scale * unscale, rcos ? rcos + (size_t)qr1 * 64 : nullptr,
                  rsin ? rsin + (size_t)qr1 * 64 : nullptr, t4, dqkv32 ? dqkv32 + r : nullptr);
  }
}

constexpr int FWD_SMEM = 5 * 64 * LDS * 2;
constexpr int DKDV_SMEM = (2 * 64 + 4 * 32) * LDS * 2 + 4 * 32 * 4;
constexpr int DQ_SMEM = 6 * 64 * LDS * 2;

soup_status attn_init() {
  static bool init = false;
  if (!init) {
    SOUP_CUDA_TRY(cudaFuncSetAttribute(attn_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, FWD_SMEM));
    SOUP_CUDA_TRY(cudaFuncSetAttribute(attn_bwd_dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DKDV_SMEM));
    SOUP_CUDA_TRY(cudaFuncSetAttribute(attn_bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DQ_SMEM));
    init = true;
  }
  return SOUP_OK;
}

}  // namespace

soup_status attention_fwd(const uint16_t* qkv, int ld, int Bsz, int S, int Hq, int Hkv, uint16_t* out, float* lse,
                          cudaStream_t st, uint16_t* out16, float* out32) {
  SOUP_CHECK(Hq % Hkv == 0 && S > 0 && Bsz > 0, SOUP_ERR_SHAPE, "attention: bad heads/shape");
  SOUP_CHECK(ld % 8 == 0 && soup_aligned(qkv, 16) && soup_aligned(out, 16), SOUP_ERR_ALIGN, "attention: alignment");
  SOUP_TRY(attn_init());
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)HD);
  dim3 grid((S + 63) / 64, Hq, Bsz);
  const double fl = 4.0 * Bsz * Hq * (double)HD * ((double)S * (S + 1) / 2);
  profile_begin(st, GC_ATTN, fl, 0.0);
  attn_fwd_kernel<<<grid, 128, FWD_SMEM, st>>>(qkv, ld, S, Hq, Hkv, out, lse, scale_log2, out16, out32);
  SOUP_LAUNCH_CHECK();
  profile_end(st);
  return SOUP_OK;
}

soup_status attention_bwd(const uint16_t* qkv, int ld, int Bsz, int S, int Hq, int Hkv, const uint16_t* dout,
                          const float* lse, const float* D, uint16_t* dqkv, const float* rope_cos,
                          const float* rope_sin, const unsigned int* amax, cudaStream_t st, float* dqkv32) {
  SOUP_CHECK(Hq % Hkv == 0 && S > 0 && Bsz > 0, SOUP_ERR_SHAPE, "attention: bad heads/shape");
  SOUP_TRY(attn_init());
  const float scale = 1.0f / sqrtf((float)HD);
  const float scale_log2 = 1.4426950408889634f * scale;
  const double fl = 2.5 * 4.0 * Bsz * Hq * (double)HD * ((double)S * (S + 1) / 2);
  profile_begin(st, GC_ATTN, fl, 0.0);
  dim3 g1((S + 63) / 64, Hkv, Bsz);
  attn_bwd_dkdv_kernel<<<g1, 128, DKDV_SMEM, st>>>(qkv, ld, S, Hq, Hkv, dout, lse, D, dqkv, scale_log2, scale,
                                                   rope_cos, rope_sin, amax, dqkv32);
  SOUP_LAUNCH_CHECK();
  dim3 g2((S + 63) / 64, Hq, Bsz);
  attn_bwd_dq_kernel<<<g2, 128, DQ_SMEM, st>>>(qkv, ld, S, Hq, Hkv, dout, lse, D, dqkv, scale_log2, scale,
                                               rope_cos, rope_sin, amax, dqkv32);
  SOUP_LAUNCH_CHECK();
  profile_end(st);
  return SOUP_OK;
}

}  // namespace soup
