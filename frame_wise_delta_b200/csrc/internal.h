// Kernel launchers shared between the translation units of libvdn.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "vdn.h"

namespace vdn {

// Generic CUDA-core kernels: any d in {16, 32, 64, 128}, float32 or bf16 inputs.
// `anchors` is a mask throughout: bit 0 makes the first frame of each (b, h)
// an anchor, bit 1 the last one (identity transitions, zero reads).
// beta: one gate per frame ([nframes]) or, with per_token, per token ([nframes, U])
cudaError_t launch_gram_simt(const void *K, const void *V, int in_dtype, const float *beta, bool per_token,
                             float *A, float *Bm, long long nframes, int U, int D, cudaStream_t st);
cudaError_t launch_factor_simt(const float *A, const float *Bm, const float *alpha, float *M,
                               float *J, int32_t *info, long long nframes, int T, int anchors, int D,
                               cudaStream_t st);
cudaError_t launch_compose_simt(const float *M, const float *J, float *Mf, float *Jf, float *Mb,
                                float *Jb, long long BH, int T, int chunk, int D, cudaStream_t st);
// dir_mask: bit 0 forward (writes F), bit 1 backward (writes G).
// Both scans start from init_scale * S_T (1/2: the two scans share the text
// state; 1: a forward-only scan from a carried state).
cudaError_t launch_scan_simt(const float *Mf, const float *Jf, const float *Mb, const float *Jb,
                             const float *S_T, float *F, float *G, long long BH, int C, int D,
                             int dir_mask, cudaStream_t st, float init_scale = 0.5f);
// Readout epilogue of step (5): y = o / sqrt(mean o^2 + eps) * w[h] * sigmoid(gate),
// per token over its d channels; gate == nullptr leaves o as it is.
struct OutGate {
  const void *gate;  // [B,H,T,U,d], the input dtype
  const float *w;    // [H, d]
  float eps;
  int H;
};
// R_c = F[max(c - 1, 0)] + G[min(c + 2, C)]; G may be null (forward reads
// only) and F0 ([BH, d, d], may be null) replaces F[0] for chunk 0.
// bridge_alpha ([BH, T, d], may be null): read through the decay bridge,
// R_t = F[max(c - 1, 0)] Diag(pf_t) + G[min(c + 2, C)] Diag(pb_t).
// bridge_prev ([BH, d], may be null): with F0 and the bridge, chunk 0's
// forward factor also carries this decay product (a stream segment's window
// starting in the previous segment's last chunk).
cudaError_t launch_readout_simt(const void *Q, int in_dtype, const float *F, const float *G, void *O,
                                int out_dtype, long long BH, int T, int U, int chunk, int anchors,
                                int D, cudaStream_t st, const OutGate *og = nullptr,
                                const float *F0 = nullptr, const float *bridge_alpha = nullptr,
                                const float *bridge_prev = nullptr);
// Decay product over the last chunk of each b*h's frames, anchors (mask as
// above) counting as 1: out[bh][k] = prod alpha[bh][r][k], r = chunk (C - 1) .. T - 1.
cudaError_t launch_bridge_tail(const float *alpha, float *out, long long BH, int T, int chunk, int anchors, int D,
                               cudaStream_t st);

// Tensor-core kernels (tcgen05 + TMA), bf16 inputs, d = 128.
bool gram_tc_supported(int in_dtype, int D, int U);
// Pinv: null, or where to write each frame's P^{-1} (the leading 64 x 64
// block of I + A inverted): the sweep pairs then also form X^T and the Schur
// complement S (schur.cuh, as launch_schur_prep does) beside the stream, in
// rows 0..63 of each frame of A.
// spare_sms: SMs the persistent grid leaves free for a concurrent stream.
cudaError_t launch_gram_tc(const void *K, const void *V, const float *beta, bool per_token, float *A,
                           float *Bm, long long nframes, int U, int32_t *info, cudaStream_t st,
                           float *Pinv = nullptr, long long frame_base = 0, int spare_sms = 0);
bool readout_tc_supported(int in_dtype, int out_dtype, int D, int U);
cudaError_t launch_readout_tc(const void *Q, const float *F, const float *G, void *O, long long BH,
                              int T, int U, int chunk, int anchors, int32_t *info, cudaStream_t st,
                              const OutGate *og = nullptr, const float *F0 = nullptr,
                              const float *bridge_alpha = nullptr, const float *bridge_prev = nullptr);

// W = (I + A)^{-1} per frame (CUDA cores); W fp32 and/or Wimg (hi/lo MMA
// images of kImgBytes per frame, d = 128 only), each optional.
// frame_base: index of the first frame, for the failure index in *info.
// (I + A)^{-1} of 128 x 128 frames by the tensor-core block inverse, from the
// P^{-1}, X^T and S that launch_schur_prep (or the Gram kernel's sweep pairs)
// left in Pinv and A, as fp32 row-major W and/or hi/lo MMA images (either
// may be null)
cudaError_t launch_invert_tc(const float *A, const float *Pinv, float *W, uint8_t *Wimg, int32_t *info,
                             long long nframes, cudaStream_t st, long long frame_base = 0);
// (I + A)^{-1} of fp32 128 x 128 frames by the blocked symmetric sweep with
// tensor-core updates, as fp32 row-major W and/or hi/lo MMA images (either
// may be null). A must be symmetric: the kernel reads its columns as rows.
cudaError_t launch_invert_bsweep(const float *A, float *W, uint8_t *Wimg, int32_t *info, long long nframes,
                                 cudaStream_t st, long long frame_base);
// P^{-1} (leading 64 x 64 block of I + A, 16 KB fp32) of every frame into
// Pinv, and X^T = Q^T P^{-1} and the Schur complement S into rows 0..63 of
// each frame of A (schur.cuh), from a full fp32 A
constexpr long long kPinvBytes = 16384;
cudaError_t launch_schur_prep(float *A, float *Pinv, int32_t *info, long long nframes, cudaStream_t st,
                              long long frame_base = 0);
cudaError_t launch_invert_simt(const float *A, float *W, uint8_t *Wimg, int32_t *info,
                               long long nframes, int D, cudaStream_t st, long long frame_base = 0);
// Chunk maps from W images (tensor cores, d = 128): per (direction, b*h,
// chunk) the M-chain (Mf/Mb fp32, and if Mimg its transposed image: the
// K-major A operand of the scan) and the J-chain (Jf/Jb, row-major, or
// transposed with j_transposed, as the scan reads it); any output pointer may
// be NULL. ndirs = 1 runs the forward direction only.
cudaError_t launch_compose_tc(const uint8_t *Wimg, const float *Bm, const float *alpha, float *Mf,
                              float *Jf, float *Mb, float *Jb, uint8_t *Mimg, long long BH, int T,
                              int chunk, int anchors, int ndirs, bool j_transposed, int32_t *info,
                              cudaStream_t st);
// Both scans (dir_mask bit 0 forward, bit 1 backward) from the compose's Mc
// images and transposed fp32 Jc (tensor cores, d = 128), started from
// init_scale * S_T.
cudaError_t launch_scan_tc(const uint8_t *Mimg, const float *Jf, const float *Jb, const float *S_T,
                           float *F, float *G, long long BH, int C, int32_t *info, cudaStream_t st,
                           int dir_mask = 3, float init_scale = 0.5f);

// Message returned by vdn_last_error() on this thread.
void set_last_error(const char *msg);

// The shape checks every entry point applies (sizes, d, chunk, flags,
// dtypes, index ranges); on failure the message is set as by the entry points.
vdn_status validate_shape(const vdn_shape *s);

// Driver entry point for tensor-map encoding (resolved once, thread-safe).
void *tensor_map_encoder();
int device_sm_count();

}  // namespace vdn
