// CUDA-core kernels of the VDA hot path, for any width d in {16, 32, 64, 128}
// and float32 or bf16 inputs. They carry the float32 workloads (which need
// ~1e-4 agreement and are too small for the tensor-core tiles) and every
// step that has no tensor-core kernel yet. Paper: "Video DeltaNet: A
// Video-Native Hybrid Attention for Livestream Video Generation" (summary
// page), "Core method" and "Method steps" (2)-(5).
//
// Thread layout used throughout: 256 threads, rg = tid / 16, cg = tid % 16;
// a thread owns rows rg + 16a and columns cg + 16b of its output tiles, so
// shared-memory reads along a column are broadcasts and reads along a row
// are 16 consecutive words (conflict-free).
#include "common.cuh"
#include "internal.h"

namespace vdn {
namespace {

constexpr int kThreads = 256;

// ----------------------------------------------------------------- Grams
// One block per (frame, which): which = 0 -> A = beta K^T K,
// which = 1 -> Bm = beta V^T K. Token tiles of 32 rows are staged in smem.
template <int D, typename Tin>
__global__ void __launch_bounds__(kThreads) gram_simt_kernel(const Tin *__restrict__ K,
                                                            const Tin *__restrict__ V,
                                                            const float *__restrict__ beta,
                                                            bool per_token,
                                                            float *__restrict__ A,
                                                            float *__restrict__ Bm, int U) {
  constexpr int R = D / 16;
  constexpr int TU = 32;
  __shared__ float Xs[TU][D];
  __shared__ float Ks[TU][D];
  const long long f = blockIdx.x;
  const int which = blockIdx.y;
  const Tin *Kf = K + f * (long long)U * D;
  const Tin *Xf = (which == 0 ? K : V) + f * (long long)U * D;
  const int rg = threadIdx.x / 16, cg = threadIdx.x % 16;
  float acc[R][R];
#pragma unroll
  for (int a = 0; a < R; ++a)
#pragma unroll
    for (int b = 0; b < R; ++b) acc[a][b] = 0.f;

  for (int u0 = 0; u0 < U; u0 += TU) {
    for (int e = threadIdx.x; e < TU * D; e += kThreads) {
      const int uu = e / D, c = e % D, u = u0 + uu;
      float xv = 0.f, kv = 0.f;
      if (u < U) {
        xv = to_f32(Xf[(long long)u * D + c]);
        kv = to_f32(Kf[(long long)u * D + c]);
        if (per_token) kv *= beta[f * U + u];  // K^T Diag(beta) [K | V]
      }
      Xs[uu][c] = xv;
      Ks[uu][c] = kv;
    }
    __syncthreads();
#pragma unroll 4
    for (int uu = 0; uu < TU; ++uu) {
      float xr[R], kr[R];
#pragma unroll
      for (int a = 0; a < R; ++a) xr[a] = Xs[uu][rg + 16 * a];
#pragma unroll
      for (int b = 0; b < R; ++b) kr[b] = Ks[uu][cg + 16 * b];
#pragma unroll
      for (int a = 0; a < R; ++a)
#pragma unroll
        for (int b = 0; b < R; ++b) acc[a][b] = fmaf(xr[a], kr[b], acc[a][b]);
    }
    __syncthreads();
  }
  const float bt = per_token ? 1.f : beta[f];
  float *out = (which == 0 ? A : Bm) + f * (long long)D * D;
#pragma unroll
  for (int a = 0; a < R; ++a)
#pragma unroll
    for (int b = 0; b < R; ++b) out[(rg + 16 * a) * D + cg + 16 * b] = bt * acc[a][b];
}

// ---------------------------------------------------------------- factor
// In-place Gauss-Jordan by columns on the stacked matrix X = [I + A_t ; Bm_t]
// ((2d) x d), held in registers. Column step k scales column k by 1/pivot
// and eliminates row k of the top block from every other column; the top
// block's row k is overwritten with the matching row of the inverse (the
// classic in-place scheme). At the end X = [(I+A)^{-1} ; Bm (I+A)^{-1}], so
// M_t = Diag(alpha_t) * top and J_t = bottom. No pivoting is needed: I + A
// is symmetric positive definite with every pivot >= 1.
template <int D>
__global__ void __launch_bounds__(kThreads, 1) factor_simt_kernel(
    const float *__restrict__ A, const float *__restrict__ Bm, const float *__restrict__ alpha,
    float *__restrict__ M, float *__restrict__ J, int32_t *__restrict__ info, int T, int anchors) {
  constexpr int RA = D / 16;       // top-block rows per thread
  constexpr int RA2 = 2 * D / 16;  // stacked rows per thread
  constexpr int RB = D / 16;       // columns per thread
  __shared__ float rowbuf[2][D];
  __shared__ float colbuf[2][2 * D];
  const long long f = blockIdx.x;
  const int t = (int)(f % T);
  const int rg = threadIdx.x / 16, cg = threadIdx.x % 16;
  const long long base = f * (long long)D * D;

  if (((anchors & 1) && t == 0) || ((anchors & 2) && t == T - 1)) {  // identity transition
#pragma unroll
    for (int a = 0; a < RA; ++a)
#pragma unroll
      for (int b = 0; b < RB; ++b) {
        const int i = rg + 16 * a, j = cg + 16 * b;
        if (M) M[base + i * D + j] = (i == j) ? 1.f : 0.f;
        J[base + i * D + j] = 0.f;
      }
    return;
  }

  float X[RA2][RB];
#pragma unroll
  for (int a = 0; a < RA2; ++a)
#pragma unroll
    for (int b = 0; b < RB; ++b) {
      const int i = rg + 16 * a, j = cg + 16 * b;
      if (a < RA)
        X[a][b] = A[base + i * D + j] + (i == j ? 1.f : 0.f);
      else
        X[a][b] = Bm[base + (i - D) * D + j];
    }

  bool bad = false;
  for (int k = 0; k < D; ++k) {
    const int buf = k & 1;
    const int kb = k >> 4, kr = k & 15;
    if (cg == kr) {
#pragma unroll
      for (int b = 0; b < RB; ++b)
        if (b == kb) {
#pragma unroll
          for (int a = 0; a < RA2; ++a) colbuf[buf][rg + 16 * a] = X[a][b];
        }
    }
    if (rg == kr) {
#pragma unroll
      for (int a = 0; a < RA; ++a)
        if (a == kb) {
#pragma unroll
          for (int b = 0; b < RB; ++b) rowbuf[buf][cg + 16 * b] = X[a][b];
        }
    }
    __syncthreads();
    const float piv = rowbuf[buf][k];
    if (!(piv > 0.f) || !isfinite(piv)) bad = true;
    const float p = 1.0f / piv;
    float fr[RB];
#pragma unroll
    for (int b = 0; b < RB; ++b) fr[b] = rowbuf[buf][cg + 16 * b] * p;
#pragma unroll
    for (int a = 0; a < RA2; ++a) {
      const int i = rg + 16 * a;
      if (a < RA && i == k) {
#pragma unroll
        for (int b = 0; b < RB; ++b) X[a][b] = -fr[b];
      } else {
        const float c = colbuf[buf][i];
#pragma unroll
        for (int b = 0; b < RB; ++b) X[a][b] = fmaf(-c, fr[b], X[a][b]);
      }
    }
    // column k: X[i][k] = X_old[i][k] / piv, and the pivot itself becomes 1/piv
    if (cg == kr) {
#pragma unroll
      for (int b = 0; b < RB; ++b)
        if (b == kb) {
#pragma unroll
          for (int a = 0; a < RA2; ++a) {
            const int i = rg + 16 * a;
            X[a][b] = (a < RA && i == k) ? p : colbuf[buf][i] * p;
          }
        }
    }
  }
  if (bad && threadIdx.x == 0) report_frame_failure(info, f);

#pragma unroll
  for (int a = 0; a < RA2; ++a) {
    const int i = rg + 16 * a;
    if (a < RA) {
      if (M) {
        const float al = alpha ? alpha[f * D + i] : 1.f;
#pragma unroll
        for (int b = 0; b < RB; ++b) M[base + i * D + cg + 16 * b] = al * X[a][b];
      }
    } else {
#pragma unroll
      for (int b = 0; b < RB; ++b) J[base + (i - D) * D + cg + 16 * b] = X[a][b];
    }
  }
}

// --------------------------------------------------------------- compose
// One block per (b*h, chunk, direction). X = [Mc ; Jc] ((2d) x d) lives in
// shared memory; each further frame applies X <- X M_t + [0 ; J_t].
template <int D>
__global__ void __launch_bounds__(kThreads, 1) compose_simt_kernel(
    const float *__restrict__ M, const float *__restrict__ J, float *__restrict__ Mf,
    float *__restrict__ Jf, float *__restrict__ Mb, float *__restrict__ Jb, int T, int chunk,
    int C) {
  constexpr int RA2 = 2 * D / 16;
  constexpr int RB = D / 16;
  extern __shared__ __align__(16) float sm[];
  float *Xs = sm;              // [2D][D]
  float *Ms = sm + 2 * D * D;  // [D][D]
  const long long bh = blockIdx.x;
  const int c = blockIdx.y;
  const int dir = blockIdx.z;
  const int rg = threadIdx.x / 16, cg = threadIdx.x % 16;
  const int t0 = c * chunk;
  const int t1 = min(t0 + chunk, T);
  const int n = t1 - t0;
  const long long DD = (long long)D * D;

  auto frame_at = [&](int s) { return dir == 0 ? t0 + s : t1 - 1 - s; };
  {
    const long long fidx = bh * T + frame_at(0);
    const float4 *m4 = reinterpret_cast<const float4 *>(M + fidx * DD);
    const float4 *j4 = reinterpret_cast<const float4 *>(J + fidx * DD);
    float4 *x4 = reinterpret_cast<float4 *>(Xs);
    for (int e = threadIdx.x; e < D * D / 4; e += kThreads) {
      x4[e] = m4[e];
      x4[D * D / 4 + e] = j4[e];
    }
  }
  for (int s = 1; s < n; ++s) {
    const long long fidx = bh * T + frame_at(s);
    const float4 *m4 = reinterpret_cast<const float4 *>(M + fidx * DD);
    float4 *ms4 = reinterpret_cast<float4 *>(Ms);
    for (int e = threadIdx.x; e < D * D / 4; e += kThreads) ms4[e] = m4[e];
    __syncthreads();
    float acc[RA2][RB];
#pragma unroll
    for (int a = 0; a < RA2; ++a)
#pragma unroll
      for (int b = 0; b < RB; ++b) acc[a][b] = 0.f;
#pragma unroll 2
    for (int k = 0; k < D; ++k) {
      float xr[RA2], mr[RB];
#pragma unroll
      for (int a = 0; a < RA2; ++a) xr[a] = Xs[(rg + 16 * a) * D + k];
#pragma unroll
      for (int b = 0; b < RB; ++b) mr[b] = Ms[k * D + cg + 16 * b];
#pragma unroll
      for (int a = 0; a < RA2; ++a)
#pragma unroll
        for (int b = 0; b < RB; ++b) acc[a][b] = fmaf(xr[a], mr[b], acc[a][b]);
    }
    __syncthreads();
    const float *Jt = J + fidx * DD;
#pragma unroll
    for (int a = 0; a < RA2; ++a) {
      const int i = rg + 16 * a;
#pragma unroll
      for (int b = 0; b < RB; ++b) {
        const int j = cg + 16 * b;
        float v = acc[a][b];
        if (i >= D) v += Jt[(i - D) * D + j];
        Xs[i * D + j] = v;
      }
    }
  }
  __syncthreads();
  float *Mo = (dir == 0 ? Mf : Mb) + (bh * C + c) * DD;
  float *Jo = (dir == 0 ? Jf : Jb) + (bh * C + c) * DD;
  const float4 *x4 = reinterpret_cast<const float4 *>(Xs);
  float4 *mo4 = reinterpret_cast<float4 *>(Mo);
  float4 *jo4 = reinterpret_cast<float4 *>(Jo);
  for (int e = threadIdx.x; e < D * D / 4; e += kThreads) {
    mo4[e] = x4[e];
    jo4[e] = x4[D * D / 4 + e];
  }
}

// ------------------------------------------------------------------ scan
// One block per (b*h, direction, 16-row block of the state). Rows of the
// state evolve independently (S_out = S_in Mc + Jc acts row by row), so the
// d_v rows are split over d_v / 16 blocks that each hold their rows on chip
// for the whole sequence of chunk boundaries.
template <int D>
__global__ void __launch_bounds__(kThreads) scan_simt_kernel(
    const float *__restrict__ Mf, const float *__restrict__ Jf, const float *__restrict__ Mb,
    const float *__restrict__ Jb, const float *__restrict__ S_T, float *__restrict__ F,
    float *__restrict__ G, int C, int dir_mask, float init_scale) {
  constexpr int RB = D / 16;
  constexpr int RR = 16;  // state rows per block
  extern __shared__ __align__(16) float sm[];
  float *Ms = sm;           // [D][D]
  float *Ss = sm + D * D;   // [RR][D]
  const long long bh = blockIdx.x;
  const int dir = blockIdx.y;
  const int r0 = blockIdx.z * RR;
  if (!((dir_mask >> dir) & 1)) return;
  const int r = threadIdx.x / 16, cg = threadIdx.x % 16;
  const long long DD = (long long)D * D;
  const float *Mc = dir == 0 ? Mf : Mb;
  const float *Jc = dir == 0 ? Jf : Jb;
  float *out = dir == 0 ? F : G;

  float s[RB];
#pragma unroll
  for (int b = 0; b < RB; ++b) {
    const int j = cg + 16 * b;
    s[b] = init_scale * S_T[bh * DD + (r0 + r) * D + j];
    Ss[r * D + j] = s[b];
    out[(bh * (C + 1) + (dir == 0 ? 0 : C)) * DD + (r0 + r) * D + j] = s[b];
  }
  for (int step = 0; step < C; ++step) {
    const int c = dir == 0 ? step : C - 1 - step;
    const float4 *m4 = reinterpret_cast<const float4 *>(Mc + (bh * C + c) * DD);
    float4 *ms4 = reinterpret_cast<float4 *>(Ms);
    for (int e = threadIdx.x; e < D * D / 4; e += kThreads) ms4[e] = m4[e];
    __syncthreads();
    float acc[RB];
#pragma unroll
    for (int b = 0; b < RB; ++b) acc[b] = Jc[(bh * C + c) * DD + (r0 + r) * D + cg + 16 * b];
#pragma unroll 4
    for (int k = 0; k < D; ++k) {
      const float sv = Ss[r * D + k];
#pragma unroll
      for (int b = 0; b < RB; ++b) acc[b] = fmaf(sv, Ms[k * D + cg + 16 * b], acc[b]);
    }
    __syncthreads();
    const int oi = dir == 0 ? c + 1 : c;
#pragma unroll
    for (int b = 0; b < RB; ++b) {
      const int j = cg + 16 * b;
      Ss[r * D + j] = acc[b];
      out[(bh * (C + 1) + oi) * DD + (r0 + r) * D + j] = acc[b];
    }
  }
}

// --------------------------------------------------------------- readout
// One block per (frame, 64-token tile). R_c = F[max(c-1,0)] + G[min(c+2,C)]
// is staged transposed (padded) in smem, the query tile as float32. With the
// decay bridge (bal = the decay gates alpha [BH, T, D]) frame t reads
// R_t = F[max(c-1,0)] Diag(pf) + G[min(c+2,C)] Diag(pb), pf and pb the
// products of alpha over the window's frames f0..t and t..f1 (anchor frames
// count as 1), formed per channel in smem first.
template <int D, typename Tin, typename Tout>
__global__ void __launch_bounds__(kThreads) readout_simt_kernel(
    const Tin *__restrict__ Q, const float *__restrict__ F, const float *__restrict__ G,
    Tout *__restrict__ O, int T, int U, int chunk, int anchors, int C, OutGate og,
    const float *__restrict__ F0, const float *__restrict__ bal, const float *__restrict__ bprev) {
  constexpr int TU = 64;
  constexpr int RB = D / 16;
  constexpr int LD = D + 1;
  extern __shared__ __align__(16) float sm[];
  float *Rt = sm;            // [D][LD] : Rt[k][i] = R[i][k]
  float *Qs = sm + D * LD;   // [TU][D]
  float *pfb = Qs + TU * D;  // [2][D] bridge factors pf, pb
  const long long f = blockIdx.x;
  const int u0 = blockIdx.y * TU;
  const long long bh = f / T;
  const int t = (int)(f % T);
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  const long long DD = (long long)D * D;
  Tout *Of = O + f * (long long)U * D;

  if (((anchors & 1) && t == 0) || ((anchors & 2) && t == T - 1)) {
    for (int e = threadIdx.x; e < TU * D; e += kThreads) {
      const int u = u0 + e / D;
      if (u < U) store_val(&Of[(long long)u * D + e % D], 0.f);
    }
    return;
  }
  const int c = t / chunk;
  const float *Fs = (c == 0 && F0) ? F0 + bh * DD : F + (bh * (C + 1) + max(c - 1, 0)) * DD;
  const float *Gs = G ? G + (bh * (C + 1) + min(c + 2, C)) * DD : nullptr;
  if (bal) {
    const int f0 = chunk * max(c - 1, 0), f1 = min(chunk * (c + 2), T) - 1;
    for (int k = threadIdx.x; k < D; k += kThreads) {
      const float *al = bal + bh * (long long)T * D + k;
      float pf = 1.f, pb = 1.f;
      for (int r = f0; r <= t; ++r)
        if (!(((anchors & 1) && r == 0) || ((anchors & 2) && r == T - 1))) pf *= al[(long long)r * D];
      for (int r = t; r <= f1; ++r)
        if (!(((anchors & 1) && r == 0) || ((anchors & 2) && r == T - 1))) pb *= al[(long long)r * D];
      if (c == 0 && F0 && bprev) pf *= bprev[bh * D + k];  // a stream segment's window starts before it
      pfb[k] = pf;
      pfb[D + k] = pb;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < D * D; e += kThreads) {
      const int i = e / D, k = e % D;
      Rt[k * LD + i] = fmaf(Fs[e], pfb[k], Gs ? Gs[e] * pfb[D + k] : 0.f);
    }
  } else {
    for (int e = threadIdx.x; e < D * D; e += kThreads) {
      const int i = e / D, k = e % D;
      Rt[k * LD + i] = Fs[e] + (Gs ? Gs[e] : 0.f);
    }
  }
  const Tin *Qf = Q + f * (long long)U * D;
  for (int e = threadIdx.x; e < TU * D; e += kThreads) {
    const int u = u0 + e / D;
    Qs[e] = (u < U) ? to_f32(Qf[(long long)u * D + e % D]) : 0.f;
  }
  __syncthreads();
  float acc[4][RB];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < RB; ++b) acc[a][b] = 0.f;
#pragma unroll 4
  for (int k = 0; k < D; ++k) {
    float q[4], rr[RB];
#pragma unroll
    for (int a = 0; a < 4; ++a) q[a] = Qs[(ty + 16 * a) * D + k];
#pragma unroll
    for (int b = 0; b < RB; ++b) rr[b] = Rt[k * LD + tx + 16 * b];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < RB; ++b) acc[a][b] = fmaf(q[a], rr[b], acc[a][b]);
  }
  if (og.gate) {
    // RMSNorm over each token's D channels (held by the 16 lanes tx of its
    // half-warp), then the per-channel sigmoid gate
    const Tin *Gf = static_cast<const Tin *>(og.gate) + f * (long long)U * D;
    const float *w = og.w + (bh % og.H) * D;
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int u = u0 + ty + 16 * a;
      float ss = 0.f;
#pragma unroll
      for (int b = 0; b < RB; ++b) ss = fmaf(acc[a][b], acc[a][b], ss);
#pragma unroll
      for (int m = 8; m >= 1; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
      const float rs = 1.0f / sqrtf(ss / D + og.eps);
#pragma unroll
      for (int b = 0; b < RB; ++b) {
        const int ch = tx + 16 * b;
        const float gv = u < U ? to_f32(Gf[(long long)u * D + ch]) : 0.f;
        acc[a][b] *= rs * w[ch] / (1.0f + expf(-gv));
      }
    }
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int u = u0 + ty + 16 * a;
    if (u < U) {
#pragma unroll
      for (int b = 0; b < RB; ++b) store_val(&Of[(long long)u * D + tx + 16 * b], acc[a][b]);
    }
  }
}

template <int D>
cudaError_t gram_d(const void *K, const void *V, int in_dtype, const float *beta, bool per_token, float *A,
                   float *Bm, long long nframes, int U, cudaStream_t st) {
  dim3 grid((unsigned)nframes, 2);
  if (in_dtype == VDN_BF16)
    gram_simt_kernel<D, __nv_bfloat16><<<grid, kThreads, 0, st>>>(
        (const __nv_bfloat16 *)K, (const __nv_bfloat16 *)V, beta, per_token, A, Bm, U);
  else
    gram_simt_kernel<D, float><<<grid, kThreads, 0, st>>>((const float *)K, (const float *)V, beta,
                                                          per_token, A, Bm, U);
  return cudaGetLastError();
}

template <int D>
cudaError_t compose_d(const float *M, const float *J, float *Mf, float *Jf, float *Mb, float *Jb,
                      long long BH, int T, int chunk, cudaStream_t st) {
  const int C = (T + chunk - 1) / chunk;
  const size_t smem = (size_t)3 * D * D * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(compose_simt_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)BH, (unsigned)C, 2);
  compose_simt_kernel<D><<<grid, kThreads, smem, st>>>(M, J, Mf, Jf, Mb, Jb, T, chunk, C);
  return cudaGetLastError();
}

template <int D>
cudaError_t scan_d(const float *Mf, const float *Jf, const float *Mb, const float *Jb,
                   const float *S_T, float *F, float *G, long long BH, int C, int dir_mask,
                   float init_scale, cudaStream_t st) {
  const size_t smem = (size_t)(D * D + 16 * D) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(scan_simt_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)BH, 2, D / 16);
  scan_simt_kernel<D><<<grid, kThreads, smem, st>>>(Mf, Jf, Mb, Jb, S_T, F, G, C, dir_mask, init_scale);
  return cudaGetLastError();
}

// Decay product over the last chunk of each b*h's frames (anchors count as
// 1): what the next stream segment's first chunk finds at the start of its
// window. One thread per (b*h, channel); T = 0 leaves the empty product 1.
__global__ void bridge_tail_kernel(const float *__restrict__ alpha, float *__restrict__ out, long long n, int T,
                                   int chunk, int anchors, int D) {
  const long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (e >= n) return;
  const long long bh = e / D;
  const int k = (int)(e % D);
  const int C = (T + chunk - 1) / chunk;
  float p = 1.f;
  for (int r = C > 0 ? chunk * (C - 1) : 0; r < T; ++r)
    if (!(((anchors & 1) && r == 0) || ((anchors & 2) && r == T - 1))) p *= alpha[(bh * T + r) * D + k];
  out[e] = p;
}

template <int D, typename Tin, typename Tout>
cudaError_t readout_dt(const void *Q, const float *F, const float *G, void *O, long long BH, int T,
                       int U, int chunk, int anchors, cudaStream_t st, const OutGate &og, const float *F0,
                       const float *bal, const float *bprev) {
  const int C = (T + chunk - 1) / chunk;
  const size_t smem = (size_t)(D * (D + 1) + 64 * D + 2 * D) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(readout_simt_kernel<D, Tin, Tout>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)(BH * T), (unsigned)((U + 63) / 64));
  readout_simt_kernel<D, Tin, Tout><<<grid, kThreads, smem, st>>>(
      (const Tin *)Q, F, G, (Tout *)O, T, U, chunk, anchors, C, og, F0, bal, bprev);
  return cudaGetLastError();
}

template <int D>
cudaError_t readout_d(const void *Q, int in_dtype, const float *F, const float *G, void *O,
                      int out_dtype, long long BH, int T, int U, int chunk, int anchors,
                      cudaStream_t st, const OutGate &og, const float *F0, const float *bal,
                      const float *bprev) {
  if (in_dtype == VDN_BF16) {
    if (out_dtype == VDN_BF16)
      return readout_dt<D, __nv_bfloat16, __nv_bfloat16>(Q, F, G, O, BH, T, U, chunk, anchors, st, og, F0, bal, bprev);
    return readout_dt<D, __nv_bfloat16, float>(Q, F, G, O, BH, T, U, chunk, anchors, st, og, F0, bal, bprev);
  }
  if (out_dtype == VDN_BF16)
    return readout_dt<D, float, __nv_bfloat16>(Q, F, G, O, BH, T, U, chunk, anchors, st, og, F0, bal, bprev);
  return readout_dt<D, float, float>(Q, F, G, O, BH, T, U, chunk, anchors, st, og, F0, bal, bprev);
}

}  // namespace

#define VDN_DISPATCH_D(D, CALL)                \
  switch (D) {                                 \
    case 16: { constexpr int DD_ = 16; return CALL; }   \
    case 32: { constexpr int DD_ = 32; return CALL; }   \
    case 64: { constexpr int DD_ = 64; return CALL; }   \
    case 128: { constexpr int DD_ = 128; return CALL; } \
    default: return cudaErrorInvalidValue;     \
  }

cudaError_t launch_gram_simt(const void *K, const void *V, int in_dtype, const float *beta, bool per_token,
                             float *A, float *Bm, long long nframes, int U, int D, cudaStream_t st) {
  if (nframes <= 0) return cudaSuccess;
  VDN_DISPATCH_D(D, gram_d<DD_>(K, V, in_dtype, beta, per_token, A, Bm, nframes, U, st))
}

cudaError_t launch_factor_simt(const float *A, const float *Bm, const float *alpha, float *M,
                               float *J, int32_t *info, long long nframes, int T, int anchors, int D,
                               cudaStream_t st) {
  if (nframes <= 0) return cudaSuccess;
  switch (D) {
    case 16: factor_simt_kernel<16><<<(unsigned)nframes, kThreads, 0, st>>>(A, Bm, alpha, M, J, info, T, anchors); break;
    case 32: factor_simt_kernel<32><<<(unsigned)nframes, kThreads, 0, st>>>(A, Bm, alpha, M, J, info, T, anchors); break;
    case 64: factor_simt_kernel<64><<<(unsigned)nframes, kThreads, 0, st>>>(A, Bm, alpha, M, J, info, T, anchors); break;
    case 128: factor_simt_kernel<128><<<(unsigned)nframes, kThreads, 0, st>>>(A, Bm, alpha, M, J, info, T, anchors); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_compose_simt(const float *M, const float *J, float *Mf, float *Jf, float *Mb,
                                float *Jb, long long BH, int T, int chunk, int D, cudaStream_t st) {
  if (BH <= 0 || T <= 0) return cudaSuccess;
  VDN_DISPATCH_D(D, compose_d<DD_>(M, J, Mf, Jf, Mb, Jb, BH, T, chunk, st))
}

cudaError_t launch_scan_simt(const float *Mf, const float *Jf, const float *Mb, const float *Jb,
                             const float *S_T, float *F, float *G, long long BH, int C, int D,
                             int dir_mask, cudaStream_t st, float init_scale) {
  if (BH <= 0) return cudaSuccess;
  VDN_DISPATCH_D(D, scan_d<DD_>(Mf, Jf, Mb, Jb, S_T, F, G, BH, C, dir_mask, init_scale, st))
}

cudaError_t launch_readout_simt(const void *Q, int in_dtype, const float *F, const float *G, void *O,
                                int out_dtype, long long BH, int T, int U, int chunk, int anchors,
                                int D, cudaStream_t st, const OutGate *og, const float *F0,
                                const float *bridge_alpha, const float *bridge_prev) {
  if (BH <= 0 || T <= 0 || U <= 0) return cudaSuccess;
  const OutGate none{nullptr, nullptr, 0.f, 1};
  const OutGate &g = og ? *og : none;
  VDN_DISPATCH_D(D, readout_d<DD_>(Q, in_dtype, F, G, O, out_dtype, BH, T, U, chunk, anchors, st, g, F0,
                                   bridge_alpha, bridge_prev))
}

cudaError_t launch_bridge_tail(const float *alpha, float *out, long long BH, int T, int chunk, int anchors, int D,
                               cudaStream_t st) {
  if (BH <= 0) return cudaSuccess;
  const long long n = BH * D;
  bridge_tail_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(alpha, out, n, T, chunk, anchors, D);
  return cudaGetLastError();
}

}  // namespace vdn
