// The first half of the 2 x 2 block inverse of G = I + A_t (d = 128): P^{-1},
// X^T = Q^T P^{-1} and the Schur complement S = R - Q^T X, on the CUDA cores
// in fp32, by the 64 threads of a sweep grid.
// Paper: "Video DeltaNet: A Video-Native Hybrid Attention for Livestream
// Video Generation" (summary page), "Core method" (the closed form needs
// (I + A_t)^{-1}) and "Method steps" step (3) (factor I + A_t per frame, all
// frames in parallel).
//
// With G = [[P, Q], [Q^T, R]] in 64 x 64 blocks, G^{-1} follows from P^{-1},
// X = P^{-1} Q and S^{-1} (the tensor-core kernel finishes it). S is formed
// here in fp32: when I + A is ill-conditioned S is much smaller than R and
// Q^T X, so this subtraction is where precision matters.
//
// Outputs per frame, all fp32: P^{-1} and X^T as 64 x 64 matrices whose rows
// hold their 16-byte chunks permuted (chunk c of row i at c ^ (i & 15), the
// shared-memory layout that makes this step's reads conflict-free, copied out
// in bulk); S as the 36 values each sweep thread of the next kernel loads
// (value v of thread t at v * 64 + t, so both sides move 32 consecutive floats
// per warp access).
#pragma once
#include "common.cuh"
#include "sweep.cuh"

namespace vdn {

// In the fused frame path the first 64 rows of each frame's A buffer are not
// read once P has been staged: X^T and S are written there (float offsets).
constexpr long long kSchurXT = 0;
constexpr long long kSchurS = 64 * 64;
constexpr int kSchurSPerThread = Sweep<64>::R * (Sweep<64>::R + 1) / 2;  // 36
constexpr int kSchurBytes = 64 * 64 * 4;  // one fp32 64 x 64 block

// element (i, j) of a 64 x 64 fp32 block in the permuted-chunk layout
__device__ __forceinline__ int swz64(int i, int j) { return i * 64 + (((j >> 2) ^ (i & 15)) << 2) + (j & 3); }

// X holds the sweep of P (-P^{-1} on the grid's lower blocks). qs holds Q^T
// (row i = row 64 + i of A, columns 0..63) in shared memory in the
// permuted-chunk layout; R points at element (64, 64) of the frame's A
// (row-major, 128 floats a row), written by this kernel or an earlier one.
// bp is a 16 KB shared-memory buffer (16-byte aligned): it takes P^{-1},
// then X^T. sync is a barrier over exactly the 64 participating threads.
// The bulk copies out of bp have been read when the call returns, and qs and
// bp are free again.
template <class Sync>
__device__ __forceinline__ void schur_prep(Sweep<64> &X, const float *qs, const float *R, float *bp,
                                           float *g_pinv, float *g_xt, float *g_s, int st, Sync sync) {
  const int rg = st / kSweepGrid, cg = st % kSweepGrid;
  // P^{-1}, both triangles (the diagonal blocks are held whole by the grid)
#pragma unroll
  for (int a = 0; a < Sweep<64>::R; ++a)
#pragma unroll
    for (int b = 0; b <= a; ++b) {
      const int i = rg + kSweepGrid * a, j = cg + kSweepGrid * b;
      const float v = -X.at(a, b);
      bp[swz64(i, j)] = v;
      if (a != b) bp[swz64(j, i)] = v;
    }
  fence_proxy_async_smem();
  sync();
  if (st == 0) {
    bulk_store(g_pinv, smem_u32(bp), kSchurBytes);
    bulk_commit();
  }
  // X^T[i][j] = sum_k Q^T[i][k] P^{-1}[k][j] for rows i = rg + 8a and the
  // eight consecutive columns j = 8cg .. 8cg + 7, as pairs of columns for the
  // packed fp32x2 FMA (P^{-1} symmetric: its row k is read)
  float2 acc[8][4];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[a][e] = make_float2(0.f, 0.f);
#pragma unroll 1
  for (int kq = 0; kq < 16; ++kq) {
    float4 qa[8];
#pragma unroll
    for (int a = 0; a < 8; ++a) qa[a] = *reinterpret_cast<const float4 *>(qs + swz64(rg + 8 * a, 4 * kq));
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const int k = 4 * kq + kk;
      const float4 p0 = *reinterpret_cast<const float4 *>(bp + swz64(k, 8 * cg));
      const float4 p1 = *reinterpret_cast<const float4 *>(bp + swz64(k, 8 * cg + 4));
      const float2 pj[4] = {make_float2(p0.x, p0.y), make_float2(p0.z, p0.w), make_float2(p1.x, p1.y),
                            make_float2(p1.z, p1.w)};
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        const float q = kk == 0 ? qa[a].x : kk == 1 ? qa[a].y : kk == 2 ? qa[a].z : qa[a].w;
        const float2 q2 = make_float2(q, q);
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[a][e] = __ffma2_rn(q2, pj[e], acc[a][e]);
      }
    }
  }
  if (st == 0) bulk_wait_read<0>();  // the P^{-1} copy has read bp
  sync();                            // and so has every thread
  // X^T replaces P^{-1}
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const int i = rg + 8 * a;
    *reinterpret_cast<float4 *>(bp + swz64(i, 8 * cg)) = make_float4(acc[a][0].x, acc[a][0].y, acc[a][1].x, acc[a][1].y);
    *reinterpret_cast<float4 *>(bp + swz64(i, 8 * cg + 4)) =
        make_float4(acc[a][2].x, acc[a][2].y, acc[a][3].x, acc[a][3].y);
  }
  fence_proxy_async_smem();
  sync();
  if (st == 0) {
    bulk_store(g_xt, smem_u32(bp), kSchurBytes);
    bulk_commit();
  }
  // S[i][j] = R[i][j] + [i == j] - sum_k X^T[i][k] Q^T[j][k] on the sweep
  // grid's lower blocks (i = rg + 8a, j = cg + 8b, b <= a), each as two
  // partial sums (even and odd k) for the packed FMA; R's values are loaded
  // first, all in flight at once
  float2 t[kSchurSPerThread];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int b = 0; b <= a; ++b) t[a * (a + 1) / 2 + b] = make_float2(R[(rg + 8 * a) * 128 + cg + 8 * b], 0.f);
#pragma unroll 1
  for (int kq = 0; kq < 16; ++kq) {
    float4 xa[8];
#pragma unroll
    for (int a = 0; a < 8; ++a) {
      const float4 x = *reinterpret_cast<const float4 *>(bp + swz64(rg + 8 * a, 4 * kq));
      xa[a] = make_float4(-x.x, -x.y, -x.z, -x.w);
    }
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      const float4 qb = *reinterpret_cast<const float4 *>(qs + swz64(cg + 8 * b, 4 * kq));
#pragma unroll
      for (int a = b; a < 8; ++a) {
        float2 &u = t[a * (a + 1) / 2 + b];
        u = __ffma2_rn(make_float2(xa[a].x, xa[a].y), make_float2(qb.x, qb.y), u);
        u = __ffma2_rn(make_float2(xa[a].z, xa[a].w), make_float2(qb.z, qb.w), u);
      }
    }
  }
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int b = 0; b <= a; ++b) {
      const int v = a * (a + 1) / 2 + b;
      g_s[v * 64 + st] = (t[v].x + t[v].y) + (a == b && rg == cg ? 1.f : 0.f);
    }
  if (st == 0) bulk_wait_read<0>();  // the X^T copy has read bp
  sync();
}

}  // namespace vdn
