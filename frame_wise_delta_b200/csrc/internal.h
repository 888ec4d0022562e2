// Kernel launchers shared between the translation units of libvdn.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "vdn.h"

namespace vdn {

// Generic CUDA-core kernels: any d in {16, 32, 64, 128}, float32 or bf16 inputs.
cudaError_t launch_gram_simt(const void *K, const void *V, int in_dtype, const float *beta, float *A,
                             float *Bm, long long nframes, int U, int D, cudaStream_t st);
cudaError_t launch_factor_simt(const float *A, const float *Bm, const float *alpha, float *M,
                               float *J, int32_t *info, long long nframes, int T, int anchors, int D,
                               cudaStream_t st);
cudaError_t launch_compose_simt(const float *M, const float *J, float *Mf, float *Jf, float *Mb,
                                float *Jb, long long BH, int T, int chunk, int D, cudaStream_t st);
// dir_mask: bit 0 forward (writes F), bit 1 backward (writes G).
cudaError_t launch_scan_simt(const float *Mf, const float *Jf, const float *Mb, const float *Jb,
                             const float *S_T, float *F, float *G, long long BH, int C, int D,
                             int dir_mask, cudaStream_t st);
cudaError_t launch_readout_simt(const void *Q, int in_dtype, const float *F, const float *G, void *O,
                                int out_dtype, long long BH, int T, int U, int chunk, int anchors,
                                int D, cudaStream_t st);

// Tensor-core kernels (tcgen05 + TMA), bf16 inputs, d = 128.
bool gram_tc_supported(int in_dtype, int D, int U);
cudaError_t launch_gram_tc(const void *K, const void *V, const float *beta, float *A, float *Bm,
                           long long nframes, int U, int32_t *info, cudaStream_t st);
bool readout_tc_supported(int in_dtype, int out_dtype, int D, int U);
cudaError_t launch_readout_tc(const void *Q, const float *F, const float *G, void *O, long long BH,
                              int T, int U, int chunk, int anchors, int32_t *info, cudaStream_t st);

// Message returned by vdn_last_error() on this thread.
void set_last_error(const char *msg);

// Driver entry point for tensor-map encoding (resolved once, thread-safe).
void *tensor_map_encoder();
int device_sm_count();

}  // namespace vdn
