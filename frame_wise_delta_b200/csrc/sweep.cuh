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
        const float rp = 1.0f / piv;
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
};

}  // namespace vdn
