// Symmetric sweep operator over the lower block-triangle of a D x D matrix,
// held in registers by 64 threads on an 8 x 8 grid.
// Paper: "Video DeltaNet: A Video-Native Hybrid Attention for Livestream
// Video Generation" (summary page), "Core method" (the closed form needs
// (I + A_t)^{-1}) and "Method steps" step (3) (factor I + A_t per frame).
//
// Sweeping pivot k of a symmetric G maps
//   G[k][k] -> -1/G[k][k],   G[i][k] = G[k][i] -> G[i][k]/G[k][k],
//   G[i][j] -> G[i][j] - G[i][k] G[k][j] / G[k][k]       (i, j != k),
// and after every pivot has been swept once G has become -G^{-1}. For a
// symmetric positive definite G every pivot is positive, so no pivoting is
// needed; a non-positive or non-finite pivot is reported to the caller.
//
// Thread (rg, cg) owns the elements (rg + 8a, cg + 8b) with a >= b: pairs of
// block columns (b = 2q, 2q + 1 <= a) as float2 for the packed fp32x2 FMA of
// sm_100, and the diagonal block of even rows (b = a) as a scalar, so
// R (R + 1) / 2 values per thread with no padding (R = D / 8).
#pragma once
#include "common.cuh"

namespace vdn {

// Reciprocal by the hardware approximation (PTX rcp.approx.ftz.f32, about
// one ulp): the pivot reciprocal sits on the sweep's step-to-step critical path.
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

constexpr int kSweepGrid = 8;
constexpr int kSweepThreads = kSweepGrid * kSweepGrid;  // 64

template <int D>
struct Sweep {
  static constexpr int R = D / kSweepGrid;  // blocks per dimension
  static constexpr int P = (R + 1) / 2;
  float2 XP[R][P];
  float XS[P];

  // element (rg + 8a, cg + 8b), a >= b; a and b are compile-time after unrolling
  __device__ __forceinline__ float &at(int a, int b) {
    return ((a & 1) == 0 && b == a) ? XS[a >> 1] : ((b & 1) ? XP[a][b >> 1].y : XP[a][b >> 1].x);
  }

  // Sweep every pivot. `cbuf` is 2 x D floats of shared memory private to the
  // 64 participating threads; `sync` is a barrier over exactly those threads.
  // Returns false if any pivot was non-positive or non-finite.
  template <class Sync>
  __device__ __forceinline__ bool run(float (*cbuf)[D], int rg, int cg, Sync sync) {
    bool bad = false;
    // Pivot block kb is a compile-time constant (outer loop unrolled), so the
    // pivot row/column registers are addressed statically and only the lanes
    // that own them act on them; the 8 pivots of a block run in a plain loop.
    // c[x] lives at slot (x % 8) * R + x / 8: a thread's entries rg + 8a are contiguous.
#pragma unroll
    for (int kb = 0; kb < R; ++kb) {
#pragma unroll 1
      for (int kr = 0; kr < kSweepGrid; ++kr) {
        float *c = cbuf[kr & 1];
        // publish c_x = G[x][k] for all x: column k at and below the diagonal
        // block (lanes with cg == kr), row k to its left (lanes with rg == kr)
        if (cg == kr) {
#pragma unroll
          for (int a = kb; a < R; ++a) c[rg * R + a] = at(a, kb);
        }
        if (rg == kr) {
#pragma unroll
          for (int b = 0; b < kb; ++b) c[cg * R + b] = at(kb, b);
        }
        sync();
        const float piv = c[kr * R + kb];
        bad |= !(piv > 0.f) || !isfinite(piv);
        const float rp = rcp_approx(piv);
        // c_i for this thread's rows is read from shared memory where it is used
        const float *ci = &c[rg * R];
        float2 cj2[P];  // c_j / piv for this thread's columns, as pairs
        if constexpr (R % 4 == 0) {
          const float2 rp2 = make_float2(rp, rp);
#pragma unroll
          for (int a = 0; a < R; a += 4) {
            const float4 w = *reinterpret_cast<const float4 *>(&c[cg * R + a]);
            cj2[a / 2] = __fmul2_rn(make_float2(w.x, w.y), rp2);
            cj2[a / 2 + 1] = __fmul2_rn(make_float2(w.z, w.w), rp2);
          }
        } else {
#pragma unroll
          for (int q = 0; q < P; ++q)
            cj2[q] = make_float2(c[cg * R + 2 * q] * rp, (2 * q + 1 < R) ? c[cg * R + 2 * q + 1] * rp : 0.f);
        }
#define VDN_CJ(b) (((b) & 1) ? cj2[(b) >> 1].y : cj2[(b) >> 1].x)
#pragma unroll
        for (int a = 0; a < R; ++a) {
          const float nc = -ci[a];
          const float2 na = make_float2(nc, nc);
#pragma unroll
          for (int q = 0; q < (a + 1) / 2; ++q) XP[a][q] = __ffma2_rn(na, cj2[q], XP[a][q]);
          if ((a & 1) == 0) XS[a >> 1] = fmaf(nc, VDN_CJ(a), XS[a >> 1]);
        }
        // row/column k: G[x][k] / piv, and the pivot -> -1/piv
        if (cg == kr) {
#pragma unroll
          for (int a = kb; a < R; ++a) at(a, kb) = ci[a] * rp;
        }
        if (rg == kr) {
#pragma unroll
          for (int b = 0; b < kb; ++b) at(kb, b) = VDN_CJ(b);
          at(kb, kb) = (cg == kr) ? -rp : VDN_CJ(kb);
        }
#undef VDN_CJ
      }
    }
    return !bad;
  }

  // The same result two pivots at a time: sweeping the pair K = {k, k + 1}
  // at once maps G_KK -> -G_KK^{-1}, G_iK -> G_iK G_KK^{-1} and
  // G_ij -> G_ij - G_iK G_KK^{-1} G_Kj (sweeps compose, so this equals
  // sweeping k and then k + 1). One barrier and one reciprocal (of the 2 x 2
  // block's determinant) per pair. `cbuf` is 2 x 2 x D floats here.
  template <class Sync>
  __device__ __forceinline__ bool run2(float (*cbuf)[2][D], int rg, int cg, Sync sync) {
    static_assert(kSweepGrid % 2 == 0, "pivot pairs stay inside a block of 8");
    bool bad = false;
#pragma unroll
    for (int kb = 0; kb < R; ++kb) {
#pragma unroll 1
      for (int kr = 0; kr < kSweepGrid; kr += 2) {
        float *c0 = cbuf[(kr >> 1) & 1][0], *c1 = cbuf[(kr >> 1) & 1][1];
        // publish columns k and k + 1 (slot (x % 8) * R + x / 8 as in run)
        if (cg == kr || cg == kr + 1) {
          float *c = cg == kr ? c0 : c1;
#pragma unroll
          for (int a = kb; a < R; ++a) c[rg * R + a] = at(a, kb);
        }
        if (rg == kr || rg == kr + 1) {
          float *c = rg == kr ? c0 : c1;
#pragma unroll
          for (int b = 0; b < kb; ++b) c[cg * R + b] = at(kb, b);
        }
        sync();
        const float p00 = c0[kr * R + kb], p01 = c0[(kr + 1) * R + kb], p11 = c1[(kr + 1) * R + kb];
        const float det = fmaf(p00, p11, -p01 * p01);
        bad |= !(p00 > 0.f) || !(det > 0.f) || !isfinite(p00) || !isfinite(det);
        const float rd = rcp_approx(det);
        const float q00 = p11 * rd, q01 = -p01 * rd, q11 = p00 * rd;  // G_KK^{-1}
        const float *ci0 = &c0[rg * R], *ci1 = &c1[rg * R];
        // e_j = G_KK^{-1} (c0_j, c1_j) for this thread's columns, as pairs
        float2 e0[P], e1[P];
        {
          const float2 Q00 = make_float2(q00, q00), Q01 = make_float2(q01, q01), Q11 = make_float2(q11, q11);
#pragma unroll
          for (int q = 0; q < P; ++q) {
            float2 x0, x1;
            if constexpr (R % 2 == 0) {
              x0 = *reinterpret_cast<const float2 *>(&c0[cg * R + 2 * q]);
              x1 = *reinterpret_cast<const float2 *>(&c1[cg * R + 2 * q]);
            } else {
              x0 = make_float2(c0[cg * R + 2 * q], (2 * q + 1 < R) ? c0[cg * R + 2 * q + 1] : 0.f);
              x1 = make_float2(c1[cg * R + 2 * q], (2 * q + 1 < R) ? c1[cg * R + 2 * q + 1] : 0.f);
            }
            e0[q] = __ffma2_rn(Q01, x1, __fmul2_rn(Q00, x0));
            e1[q] = __ffma2_rn(Q11, x1, __fmul2_rn(Q01, x0));
          }
        }
#define VDN_E(e, b) (((b) & 1) ? e[(b) >> 1].y : e[(b) >> 1].x)
#pragma unroll
        for (int a = 0; a < R; ++a) {
          const float n0 = -ci0[a], n1 = -ci1[a];
          const float2 m0 = make_float2(n0, n0), m1 = make_float2(n1, n1);
#pragma unroll
          for (int q = 0; q < (a + 1) / 2; ++q) XP[a][q] = __ffma2_rn(m1, e1[q], __ffma2_rn(m0, e0[q], XP[a][q]));
          if ((a & 1) == 0) XS[a >> 1] = fmaf(n1, VDN_E(e1, a), fmaf(n0, VDN_E(e0, a), XS[a >> 1]));
        }
        // columns k, k + 1 (rows at and below the diagonal block): c_i^T G_KK^{-1}
        if (cg == kr || cg == kr + 1) {
          const float u0 = cg == kr ? q00 : q01, u1 = cg == kr ? q01 : q11;
#pragma unroll
          for (int a = kb; a < R; ++a) at(a, kb) = fmaf(ci1[a], u1, ci0[a] * u0);
        }
        // rows k, k + 1 (left of and in the diagonal block): G_KK^{-1} c_j, and
        // -G_KK^{-1} on the pair itself
        if (rg == kr || rg == kr + 1) {
          const bool r0 = rg == kr;
#pragma unroll
          for (int b = 0; b < kb; ++b) at(kb, b) = r0 ? VDN_E(e0, b) : VDN_E(e1, b);
          if (cg == kr || cg == kr + 1) {
            const bool c0k = cg == kr;
            at(kb, kb) = r0 ? (c0k ? -q00 : -q01) : (c0k ? -q01 : -q11);
          } else {
            at(kb, kb) = r0 ? VDN_E(e0, kb) : VDN_E(e1, kb);
          }
        }
#undef VDN_E
      }
    }
    return !bad;
  }
};

// -G^{-1} of a 64 x 64 block from the sweep, stored as the bf16 hi/lo tile of
// G^{-1} (both triangles; 64 rows of 128 bytes per part, K-major with the
// 128-byte swizzle, hi part then lo part 8 KB later) that the tensor cores read.
__device__ __forceinline__ void store_swept_tile(Sweep<64> &X, uint8_t *tile, int rg, int cg) {
  constexpr int kPart = 64 * 128;
#pragma unroll
  for (int a = 0; a < Sweep<64>::R; ++a)
#pragma unroll
    for (int b = 0; b <= a; ++b) {
      const int i = rg + kSweepGrid * a, j = cg + kSweepGrid * b;
      __nv_bfloat16 h, l;
      split_bf16(-X.at(a, b), h, l);
      const uint32_t oij = kmajor_sw128_offset(i, j, 64), oji = kmajor_sw128_offset(j, i, 64);
      *reinterpret_cast<__nv_bfloat16 *>(tile + oij) = h;
      *reinterpret_cast<__nv_bfloat16 *>(tile + kPart + oij) = l;
      if (a != b) {
        *reinterpret_cast<__nv_bfloat16 *>(tile + oji) = h;
        *reinterpret_cast<__nv_bfloat16 *>(tile + kPart + oji) = l;
      }
    }
}

}  // namespace vdn
