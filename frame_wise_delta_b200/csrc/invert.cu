// W_t = (I + A_t)^{-1} for every frame, on the CUDA cores.
// Paper: "Video DeltaNet: A Video-Native Hybrid Attention for Livestream
// Video Generation" (summary page), "Core method" (closed form
// S_t = (Sbar_t + B_t)(I + A_t)^{-1}) and "Method steps" step (3) (factor
// I + A_t in batch, independent of the state, all frames in parallel).
//
// Symmetric sweep operator, one pivot at a time: sweeping pivot k of a
// symmetric G maps
//   G[k][k] -> -1/G[k][k],   G[i][k] = G[k][i] -> G[i][k]/G[k][k],
//   G[i][j] -> G[i][j] - G[i][k] G[k][j] / G[k][k]       (i, j != k),
// and after every pivot has been swept once G has become -G^{-1}. I + A is
// symmetric positive definite with eigenvalues >= 1, so every pivot is
// positive and no pivoting is needed. The matrix stays symmetric, so only
// the lower block-triangle is kept: 64 threads on an 8 x 8 grid own the
// elements (rg + 8a, cg + 8b) with a >= b (136 values each, held as float2
// pairs for the packed fp32x2 FMA of sm_100), which is half the work of a
// full Gauss-Jordan and spreads it evenly. Each step
// publishes pivot row k into a shared vector (stored interleaved so that a
// thread's eight-apart entries are contiguous), applies one rank-1 update to
// every owned element, then rewrites row/column k. A non-positive or
// non-finite pivot is reported in *info.
#include "common.cuh"
#include "internal.h"

namespace vdn {
namespace {

constexpr int kGrid = 8;                 // 8 x 8 threads
constexpr int kThreads = kGrid * kGrid;  // 64

// W (fp32, row-major) and Wimg (the hi/lo MMA image, d = 128 only) are each optional.
template <int D>
__global__ void __launch_bounds__(kThreads) invert_sweep_kernel(const float *__restrict__ A,
                                                                float *__restrict__ W,
                                                                uint8_t *__restrict__ Wimg,
                                                                int32_t *__restrict__ info,
                                                                long long frame_base) {
  constexpr int R = D / kGrid;  // blocks per dimension
  // c[x] lives at slot (x % 8) * R + x / 8: a thread's entries rg + 8a are contiguous
  __shared__ __align__(16) float cbuf[2][D];
  const long long f = blockIdx.x;
  const int rg = threadIdx.x / kGrid, cg = threadIdx.x % kGrid;
  const float *Af = A + f * (long long)D * D;

  // X(a, b) for a >= b: full pairs of block columns (b = 2q, 2q + 1 <= a) as
  // float2, so the rank-1 update runs as packed fp32x2 FMAs, and the
  // diagonal block of even rows (b = a) as a scalar: 136 values, no padding.
  constexpr int P = (R + 1) / 2;
  float2 XP[R][P];
  float XS[P];
#define XE(a, b) ((((a) & 1) == 0 && (b) == (a)) ? XS[(a) >> 1] : (((b) & 1) ? XP[a][(b) >> 1].y : XP[a][(b) >> 1].x))
#pragma unroll
  for (int a = 0; a < R; ++a)
#pragma unroll
    for (int b = 0; b <= a; ++b) {
      const int i = rg + kGrid * a, j = cg + kGrid * b;
      XE(a, b) = Af[i * D + j] + (i == j ? 1.f : 0.f);
    }

  bool bad = false;
  // Pivot block kb is a compile-time constant (outer loop unrolled), so the
  // pivot row/column registers X[.][kb], X[kb][.] are addressed statically and
  // only the lanes that own them act on them; the 8 pivots of a block run in
  // an ordinary loop.
#pragma unroll
  for (int kb = 0; kb < R; ++kb) {
#pragma unroll 1
    for (int kr = 0; kr < kGrid; ++kr) {
      const int k = kb * kGrid + kr;
      float *c = cbuf[k & 1];
      // publish c_x = G[x][k] for all x: column k at and below the diagonal
      // block (lanes with cg == kr), row k to its left (lanes with rg == kr)
      if (cg == kr) {
#pragma unroll
        for (int a = kb; a < R; ++a) c[rg * R + a] = XE(a, kb);
      }
      if (rg == kr) {
#pragma unroll
        for (int b = 0; b < kb; ++b) c[cg * R + b] = XE(kb, b);
      }
      __syncthreads();
      const float piv = c[kr * R + kb];
      bad |= !(piv > 0.f) || !isfinite(piv);
      const float rp = 1.0f / piv;
      // c_i for this thread's rows is read from shared memory where it is
      // used (keeps the 144 matrix values plus cj2 within the register file)
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
#define CJ(b) (((b) & 1) ? cj2[(b) >> 1].y : cj2[(b) >> 1].x)
#pragma unroll
      for (int a = 0; a < R; ++a) {
        const float nc = -ci[a];
        const float2 na = make_float2(nc, nc);
#pragma unroll
        for (int q = 0; q < (a + 1) / 2; ++q) XP[a][q] = __ffma2_rn(na, cj2[q], XP[a][q]);
        if ((a & 1) == 0) XS[a >> 1] = fmaf(nc, CJ(a), XS[a >> 1]);
      }
      // row/column k: G[x][k] / piv, and the pivot -> -1/piv
      if (cg == kr) {
#pragma unroll
        for (int a = kb; a < R; ++a) XE(a, kb) = ci[a] * rp;
      }
      if (rg == kr) {
#pragma unroll
        for (int b = 0; b < kb; ++b) XE(kb, b) = CJ(b);
        XE(kb, kb) = (cg == kr) ? -rp : CJ(kb);
      }
    }
  }
  if (bad && threadIdx.x == 0) report_frame_failure(info, frame_base + f);

  // W = -X; write both triangles
  if (W) {
    float *Wf = W + f * (long long)D * D;
#pragma unroll
    for (int a = 0; a < R; ++a)
#pragma unroll
      for (int b = 0; b <= a; ++b) {
        const int i = rg + kGrid * a, j = cg + kGrid * b;
        Wf[i * D + j] = -XE(a, b);
        if (a != b) Wf[j * D + i] = -XE(a, b);
      }
  }
  if constexpr (D == 128) {
    if (Wimg) {
      uint8_t *img = Wimg + f * (long long)kImgBytes;
#pragma unroll
      for (int a = 0; a < R; ++a)
#pragma unroll
        for (int b = 0; b <= a; ++b) {
          const int i = rg + kGrid * a, j = cg + kGrid * b;
          img_store(img, i, j, -XE(a, b));
          if (a != b) img_store(img, j, i, -XE(a, b));
        }
    }
  }
#undef CJ
#undef XE
}

}  // namespace

cudaError_t launch_invert_simt(const float *A, float *W, uint8_t *Wimg, int32_t *info,
                               long long nframes, int D, cudaStream_t st, long long frame_base) {
  if (nframes <= 0) return cudaSuccess;
  if (Wimg && D != 128) return cudaErrorInvalidValue;
  switch (D) {
    case 16: invert_sweep_kernel<16><<<(unsigned)nframes, kThreads, 0, st>>>(A, W, nullptr, info, frame_base); break;
    case 32: invert_sweep_kernel<32><<<(unsigned)nframes, kThreads, 0, st>>>(A, W, nullptr, info, frame_base); break;
    case 64: invert_sweep_kernel<64><<<(unsigned)nframes, kThreads, 0, st>>>(A, W, nullptr, info, frame_base); break;
    case 128: invert_sweep_kernel<128><<<(unsigned)nframes, kThreads, 0, st>>>(A, W, Wimg, info, frame_base); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace vdn
