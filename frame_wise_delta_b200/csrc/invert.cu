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
// elements (rg + 8a, cg + 8b) with a >= b (136 registers each), which is
// half the work of a full Gauss-Jordan and spreads it evenly. Each step
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
                                                                int32_t *__restrict__ info) {
  constexpr int R = D / kGrid;  // blocks per dimension
  // c[x] lives at slot (x % 8) * R + x / 8: a thread's entries rg + 8a are contiguous
  __shared__ __align__(16) float cbuf[2][D];
  const long long f = blockIdx.x;
  const int rg = threadIdx.x / kGrid, cg = threadIdx.x % kGrid;
  const float *Af = A + f * (long long)D * D;

  float X[R][R];  // only a >= b is used
#pragma unroll
  for (int a = 0; a < R; ++a)
#pragma unroll
    for (int b = 0; b <= a; ++b) {
      const int i = rg + kGrid * a, j = cg + kGrid * b;
      X[a][b] = Af[i * D + j] + (i == j ? 1.f : 0.f);
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
        for (int a = kb; a < R; ++a) c[rg * R + a] = X[a][kb];
      }
      if (rg == kr) {
#pragma unroll
        for (int b = 0; b < kb; ++b) c[cg * R + b] = X[kb][b];
      }
      __syncthreads();
      const float piv = c[kr * R + kb];
      bad |= !(piv > 0.f) || !isfinite(piv);
      const float rp = 1.0f / piv;
      float ci[R], cj[R];
      if constexpr (R % 4 == 0) {
#pragma unroll
        for (int a = 0; a < R; a += 4) {
          const float4 v = *reinterpret_cast<const float4 *>(&c[rg * R + a]);
          ci[a] = v.x; ci[a + 1] = v.y; ci[a + 2] = v.z; ci[a + 3] = v.w;
          const float4 w = *reinterpret_cast<const float4 *>(&c[cg * R + a]);
          cj[a] = w.x * rp; cj[a + 1] = w.y * rp; cj[a + 2] = w.z * rp; cj[a + 3] = w.w * rp;
        }
      } else {
#pragma unroll
        for (int a = 0; a < R; ++a) {
          ci[a] = c[rg * R + a];
          cj[a] = c[cg * R + a] * rp;
        }
      }
#pragma unroll
      for (int a = 0; a < R; ++a)
#pragma unroll
        for (int b = 0; b <= a; ++b) X[a][b] = fmaf(-ci[a], cj[b], X[a][b]);
      // row/column k: G[x][k] / piv, and the pivot -> -1/piv
      if (cg == kr) {
#pragma unroll
        for (int a = kb; a < R; ++a) X[a][kb] = ci[a] * rp;
      }
      if (rg == kr) {
#pragma unroll
        for (int b = 0; b < kb; ++b) X[kb][b] = cj[b];
        X[kb][kb] = (cg == kr) ? -rp : cj[kb];
      }
    }
  }
  if (bad && threadIdx.x == 0) report_frame_failure(info, f);

  // W = -X; write both triangles
  if (W) {
    float *Wf = W + f * (long long)D * D;
#pragma unroll
    for (int a = 0; a < R; ++a)
#pragma unroll
      for (int b = 0; b <= a; ++b) {
        const int i = rg + kGrid * a, j = cg + kGrid * b;
        Wf[i * D + j] = -X[a][b];
        if (a != b) Wf[j * D + i] = -X[a][b];
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
          img_store(img, i, j, -X[a][b]);
          if (a != b) img_store(img, j, i, -X[a][b]);
        }
    }
  }
}

}  // namespace

cudaError_t launch_invert_simt(const float *A, float *W, uint8_t *Wimg, int32_t *info,
                               long long nframes, int D, cudaStream_t st) {
  if (nframes <= 0) return cudaSuccess;
  if (Wimg && D != 128) return cudaErrorInvalidValue;
  switch (D) {
    case 16: invert_sweep_kernel<16><<<(unsigned)nframes, kThreads, 0, st>>>(A, W, nullptr, info); break;
    case 32: invert_sweep_kernel<32><<<(unsigned)nframes, kThreads, 0, st>>>(A, W, nullptr, info); break;
    case 64: invert_sweep_kernel<64><<<(unsigned)nframes, kThreads, 0, st>>>(A, W, nullptr, info); break;
    case 128: invert_sweep_kernel<128><<<(unsigned)nframes, kThreads, 0, st>>>(A, W, Wimg, info); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace vdn
