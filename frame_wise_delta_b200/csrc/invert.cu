// W_t = (I + A_t)^{-1} for every frame, on the CUDA cores.
// Paper: "Video DeltaNet: A Video-Native Hybrid Attention for Livestream
// Video Generation" (summary page), "Core method" (closed form
// S_t = (Sbar_t + B_t)(I + A_t)^{-1}) and "Method steps" step (3) (factor
// I + A_t in batch, independent of the state, all frames in parallel).
//
// The symmetric sweep (sweep.cuh) on the whole matrix, one frame per 64-thread
// block; the result -G^{-1} is negated into W and/or the hi/lo MMA image.
#include "common.cuh"
#include "internal.h"
#include "sweep.cuh"

namespace vdn {
namespace {

// W (fp32, row-major) and Wimg (the hi/lo MMA image, d = 128 only) are each optional.
template <int D>
__global__ void __launch_bounds__(kSweepThreads) invert_sweep_kernel(const float *__restrict__ A,
                                                                     float *__restrict__ W,
                                                                     uint8_t *__restrict__ Wimg,
                                                                     int32_t *__restrict__ info,
                                                                     long long frame_base) {
  using S = Sweep<D>;
  constexpr int R = S::R;
  __shared__ __align__(16) float cbuf[2][2][D];
  const long long f = blockIdx.x;
  const int rg = threadIdx.x / kSweepGrid, cg = threadIdx.x % kSweepGrid;
  const float *Af = A + f * (long long)D * D;

  S X;
#pragma unroll
  for (int a = 0; a < R; ++a)
#pragma unroll
    for (int b = 0; b <= a; ++b) {
      const int i = rg + kSweepGrid * a, j = cg + kSweepGrid * b;
      X.at(a, b) = Af[i * D + j] + (i == j ? 1.f : 0.f);
    }
  const bool ok = X.run2(cbuf, rg, cg, [] { __syncthreads(); });
  if (!ok && threadIdx.x == 0) report_frame_failure(info, frame_base + f);

  // W = -X; write both triangles
  if (W) {
    float *Wf = W + f * (long long)D * D;
#pragma unroll
    for (int a = 0; a < R; ++a)
#pragma unroll
      for (int b = 0; b <= a; ++b) {
        const int i = rg + kSweepGrid * a, j = cg + kSweepGrid * b;
        Wf[i * D + j] = -X.at(a, b);
        if (a != b) Wf[j * D + i] = -X.at(a, b);
      }
  }
  if constexpr (D == 128) {
    if (Wimg) {
      uint8_t *img = Wimg + f * (long long)kImgBytes;
#pragma unroll
      for (int a = 0; a < R; ++a)
#pragma unroll
        for (int b = 0; b <= a; ++b) {
          const int i = rg + kSweepGrid * a, j = cg + kSweepGrid * b;
          img_store(img, i, j, -X.at(a, b));
          if (a != b) img_store(img, j, i, -X.at(a, b));
        }
    }
  }
}

}  // namespace

cudaError_t launch_invert_simt(const float *A, float *W, uint8_t *Wimg, int32_t *info,
                               long long nframes, int D, cudaStream_t st, long long frame_base) {
  if (nframes <= 0) return cudaSuccess;
  if (Wimg && D != 128) return cudaErrorInvalidValue;
  switch (D) {
    case 16: invert_sweep_kernel<16><<<(unsigned)nframes, kSweepThreads, 0, st>>>(A, W, nullptr, info, frame_base); break;
    case 32: invert_sweep_kernel<32><<<(unsigned)nframes, kSweepThreads, 0, st>>>(A, W, nullptr, info, frame_base); break;
    case 64: invert_sweep_kernel<64><<<(unsigned)nframes, kSweepThreads, 0, st>>>(A, W, nullptr, info, frame_base); break;
    case 128: invert_sweep_kernel<128><<<(unsigned)nframes, kSweepThreads, 0, st>>>(A, W, Wimg, info, frame_base); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace vdn
