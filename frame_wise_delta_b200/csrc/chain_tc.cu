// Chunk composition and the bidirectional scan on the 5th-generation tensor
// cores (tcgen05 + TMEM), d = 128, fp32 state carried as bf16 hi + lo.
// Paper: "Video DeltaNet: A Video-Native Hybrid Attention for Livestream
// Video Generation" (summary page), "Technical novelty" (frame-level affine
// transitions composed into chunk-level ones before the scan) and "Method
// steps" step (4) (S_out = S_in M_chunk + J_chunk, both scans started from
// half of the text state).
//
// Both are chains of 128 x 128 x 128 products with the state kept on chip:
//
//  compose, one CTA per (b*h, chunk, direction, part), with W_t = (I+A_t)^{-1}:
//     X <- (X Diag(alpha_t) + [part J] B_t) W_t
//  over the chunk's non-anchor frames in forward or reverse order, from
//  X = I (part M -> Mc) or X = 0 (part J -> Jc). This equals X M_t + J_t
//  with M_t = Diag(alpha_t) W_t and J_t = B_t W_t, so the per-frame (M_t,
//  J_t) are never materialised.
//
//  scan, one CTA per (b*h, direction): X <- X Mc_c + Jc_c over the chunks,
//  from X = S_T / 2, writing every boundary state.
//
// One product: D[m][n] = sum_k Op[k][m] E[n][k], i.e. D = (E Op)^T in TMEM
// (lane m, column n). Op arrives as a ready-made hi/lo image (W_t from the
// factor kernel, Mc_c from the compose) by one bulk copy into a double
// buffer; E is written straight from the previous D by the thread that owns
// lane m (its column m of X is row m of E's MN-major image). Three MMAs
// accumulate hi*hi + hi*lo + lo*hi, so each product keeps ~2^-17 relative
// accuracy: an fp32 state on bf16 tensor cores.
//
// Roles (160 threads): warps 0..3 drain TMEM and build the next E (their
// global reads for the next step are issued before they wait for the MMAs);
// warp 4 allocates TMEM and one lane issues the bulk copies and the MMAs.
// Every wait is bounded.
#include "common.cuh"
#include "internal.h"

namespace vdn {
namespace {

constexpr int kD = 128;
constexpr int kThreads = 160;
constexpr size_t kSmemBytes = 1024 + 3 * (size_t)kImgBytes + 64;
constexpr uint32_t kTmemCols = 128;

enum Mode { kComposeM = 0, kComposeJ = 1, kScan = 2 };

struct ChainArgs {
  const uint8_t *Wimg;      // compose: [BH*T] images
  const float *Bm;          // compose: [BH, T, d, d]
  const float *alpha;       // compose: [BH, T, d]
  float *Mf, *Jf, *Mb, *Jb; // compose outputs / scan inputs (J) [BH, C, d, d]
  uint8_t *Mimg;            // compose output / scan input: [BH, 2, C] images of Mc
  const float *S_T;         // scan: [BH, d, d]
  float *F, *G;             // scan outputs [BH, C+1, d, d]
  int32_t *info;
  int T, chunk, C, anchors, dir_mask;
};

// Write 32 consecutive values of row m (columns n0 .. n0+31) of an image in smem.
__device__ __forceinline__ void write_e32(uint8_t *E, int m, int n0, const float (&v)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    __nv_bfloat16 h[8], l[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) split_bf16(v[q * 8 + e], h[e], l[e]);
    const uint32_t off = mn_off(m, n0 + q * 8);
    *reinterpret_cast<uint4 *>(E + off) = make_uint4(pack2(h[0], h[1]), pack2(h[2], h[3]),
                                                     pack2(h[4], h[5]), pack2(h[6], h[7]));
    *reinterpret_cast<uint4 *>(E + kImgHalf + off) = make_uint4(pack2(l[0], l[1]), pack2(l[2], l[3]),
                                                                pack2(l[4], l[5]), pack2(l[6], l[7]));
  }
}

__device__ __forceinline__ void fail(volatile int *abort, int32_t *info) {
  *abort = 1;
  if (info) atomicExch(info, VDN_INFO_TIMEOUT);
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1) chain_tc_kernel(ChainArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  uint8_t *opimg[2] = {smem, smem + kImgBytes};
  uint8_t *eimg = smem + 2 * kImgBytes;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + 3 * kImgBytes);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 5);
  volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
  const uint32_t ready = smem_u32(bars), done = ready + 8, drain = ready + 16;
  const uint32_t opfull0 = ready + 24;  // two barriers

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long bh = blockIdx.x;
  const long long DD = (long long)kD * kD;

  // ---- the chain this CTA walks
  int dir, nsteps = 0;
  int frames[16];
  int c_cmp = 0;
  if (MODE == kScan) {
    dir = blockIdx.y;
    nsteps = p.C;
    if (!((p.dir_mask >> dir) & 1)) return;
  } else {
    c_cmp = blockIdx.y;
    dir = blockIdx.z;
    const int t0 = c_cmp * p.chunk, t1 = min(t0 + p.chunk, p.T);
    for (int s = 0; s < t1 - t0; ++s) {
      const int t = dir == 0 ? t0 + s : t1 - 1 - s;
      if (p.anchors && (t == 0 || t == p.T - 1)) continue;
      frames[nsteps++] = t;
    }
  }
  // chunk visited at scan step s
  auto scan_c = [&](int s) { return dir == 0 ? s : p.C - 1 - s; };
  auto op_src = [&](int s) -> const uint8_t * {
    if (MODE == kScan) return p.Mimg + ((bh * 2 + dir) * p.C + scan_c(s)) * (long long)kImgBytes;
    return p.Wimg + (bh * p.T + frames[s]) * (long long)kImgBytes;
  };

  if (threadIdx.x == 0) {
    mbar_init(ready, 128);
    mbar_init(done, 1);
    mbar_init(drain, 1);
    mbar_init(opfull0, 1);
    mbar_init(opfull0 + 8, 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 4) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 4) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128, true, true);
      const uint32_t e_hi = smem_u32(eimg), e_lo = e_hi + kImgHalf;
      auto load_op = [&](int s) {
        const uint32_t bar = opfull0 + 8 * (s & 1);
        mbar_arrive_expect_tx(bar, kImgBytes);
        const uint32_t dst = smem_u32(opimg[s & 1]);
        const uint8_t *src = op_src(s);
#pragma unroll
        for (int q = 0; q < 4; ++q) bulk_load(dst + q * (kImgBytes / 4), src + q * (kImgBytes / 4), kImgBytes / 4, bar);
      };
      int loads = 0;
      for (; loads < 2 && loads < nsteps; ++loads) load_op(loads);
      bool ok = true;
      for (int s = 0; s < nsteps; ++s) {
        if (!mbar_wait(ready, (uint32_t)(s & 1), abort) ||
            !mbar_wait(opfull0 + 8 * (s & 1), (uint32_t)((s >> 1) & 1), abort)) {
          fail(abort, p.info);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t o_hi = smem_u32(opimg[s & 1]), o_lo = o_hi + kImgHalf;
#pragma unroll
        for (int part = 0; part < 3; ++part) {
          const uint32_t a0 = part == 2 ? o_lo : o_hi;
          const uint32_t b0 = part == 1 ? e_lo : e_hi;
#pragma unroll
          for (int ks = 0; ks < kD / 16; ++ks) {
            const uint64_t ad = smem_desc_sw128(a0 + ks * 2048, kImgRegion, 1024);
            const uint64_t bd = smem_desc_sw128(b0 + ks * 2048, kImgRegion, 1024);
            tc_mma_bf16(tmem_base, ad, bd, idesc, (part > 0 || ks > 0) ? 1u : 0u);
          }
        }
        tc_commit(done);
        if (loads < nsteps) {
          // buffer s & 1 is free once these MMAs are done
          if (!mbar_wait(done, (uint32_t)(s & 1), abort)) {
            fail(abort, p.info);
            ok = false;
            break;
          }
          load_op(loads++);
        }
      }
      (void)ok;
      // every issued copy has landed and every MMA is done before leaving
      volatile int never = 0;
      for (int s = (loads > 2 ? loads - 2 : 0); s < loads; ++s)
        mbar_wait(opfull0 + 8 * (s & 1), (uint32_t)((s >> 1) & 1), &never);
      tc_commit(drain);
      mbar_wait(drain, 0, &never);
    }
  } else {
    // ---- workers: thread m owns column m of X (TMEM lane m)
    const int m = threadIdx.x;  // warp w -> TMEM sub-partition w
    float *out_base = nullptr;
    uint8_t *out_img = nullptr;
    if (MODE != kScan) {
      const long long cidx = bh * p.C + c_cmp;
      out_base = (dir == 0 ? (MODE == kComposeM ? p.Mf : p.Jf) : (MODE == kComposeM ? p.Mb : p.Jb)) + cidx * DD;
      if (MODE == kComposeM && p.Mimg) out_img = p.Mimg + ((bh * 2 + dir) * p.C + c_cmp) * (long long)kImgBytes;
    }

    // E_0 (and, for the scan, the first boundary state)
    if (MODE == kScan) {
      const float *st = p.S_T + bh * DD;
      float *o = dir == 0 ? p.F + (bh * (p.C + 1)) * DD : p.G + (bh * (p.C + 1) + p.C) * DD;
      for (int n0 = 0; n0 < kD; n0 += 32) {
        float v[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          v[e] = 0.5f * st[(n0 + e) * kD + m];
          o[(n0 + e) * kD + m] = v[e];
        }
        if (nsteps > 0) write_e32(eimg, m, n0, v);
      }
    } else if (nsteps == 0) {  // every frame of the chunk is an anchor: identity map
      for (int n = 0; n < kD; ++n) {
        const float x0 = (MODE == kComposeM && n == m) ? 1.f : 0.f;
        out_base[n * kD + m] = x0;
        if (out_img) img_store(out_img, n, m, x0);
      }
    } else {
      const float al = p.alpha[(bh * p.T + frames[0]) * kD + m];
      const float *Bt = p.Bm + (bh * p.T + frames[0]) * DD;
      for (int n0 = 0; n0 < kD; n0 += 32) {
        float v[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int n = n0 + e;
          v[e] = (MODE == kComposeM) ? (n == m ? al : 0.f) : Bt[n * kD + m];
        }
        write_e32(eimg, m, n0, v);
      }
    }
    if (nsteps > 0) {
      fence_proxy_async_smem();
      mbar_arrive(ready);
    }

    for (int s = 0; s < nsteps; ++s) {
      const bool last = (s + 1 == nsteps);
      // operands of this step's epilogue, fetched while the MMAs run
      float al = 1.f;
      float addv[kD];
      bool has_add = false;
      if (MODE == kScan) {
        const float *J = (dir == 0 ? p.Jf : p.Jb) + (bh * p.C + scan_c(s)) * DD;
#pragma unroll
        for (int n = 0; n < kD; ++n) addv[n] = J[n * kD + m];
        has_add = true;
      } else if (!last) {
        al = p.alpha[(bh * p.T + frames[s + 1]) * kD + m];
        if (MODE == kComposeJ) {
          const float *Bt = p.Bm + (bh * p.T + frames[s + 1]) * DD;
#pragma unroll
          for (int n = 0; n < kD; ++n) addv[n] = Bt[n * kD + m];
          has_add = true;
        }
      }
      const bool ok = __all_sync(0xffffffffu, mbar_wait(done, (uint32_t)(s & 1), abort));
      if (!ok) {
        fail(abort, p.info);
        break;
      }
      tc_fence_after();
      float *o = nullptr;
      if (MODE == kScan) {
        const int c = scan_c(s);
        o = dir == 0 ? p.F + (bh * (p.C + 1) + c + 1) * DD : p.G + (bh * (p.C + 1) + c) * DD;
      } else if (last) {
        o = out_base;
      }
#pragma unroll
      for (int n0 = 0; n0 < kD; n0 += 32) {
        float v[32];
        tmem_ld32(tmem_base + (uint32_t)n0 + ((uint32_t)(warp * 32) << 16), v);
        if (MODE == kScan) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            v[e] += addv[n0 + e];
            o[(n0 + e) * kD + m] = v[e];
          }
          if (!last) write_e32(eimg, m, n0, v);
        } else if (!last) {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = v[e] * al + (has_add ? addv[n0 + e] : 0.f);
          write_e32(eimg, m, n0, v);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            o[(n0 + e) * kD + m] = v[e];
            if (out_img) img_store(out_img, n0 + e, m, v[e]);
          }
        }
      }
      if (!last) {
        tc_fence_before();
        fence_proxy_async_smem();
        mbar_arrive(ready);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

template <int MODE>
cudaError_t launch_mode(dim3 grid, const ChainArgs &a, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(chain_tc_kernel<MODE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  chain_tc_kernel<MODE><<<grid, kThreads, kSmemBytes, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_compose_tc(const uint8_t *Wimg, const float *Bm, const float *alpha, float *Mf,
                              float *Jf, float *Mb, float *Jb, uint8_t *Mimg, long long BH, int T,
                              int chunk, int anchors, int parts, int ndirs, int32_t *info,
                              cudaStream_t st) {
  if (BH <= 0 || T <= 0) return cudaSuccess;
  ChainArgs a{};
  a.Wimg = Wimg;
  a.Bm = Bm;
  a.alpha = alpha;
  a.Mf = Mf;
  a.Jf = Jf;
  a.Mb = Mb;
  a.Jb = Jb;
  a.Mimg = Mimg;
  a.info = info;
  a.T = T;
  a.chunk = chunk;
  a.C = (T + chunk - 1) / chunk;
  a.anchors = anchors;
  dim3 grid((unsigned)BH, (unsigned)a.C, (unsigned)ndirs);
  if (parts & 1) {
    cudaError_t e = launch_mode<kComposeM>(grid, a, st);
    if (e != cudaSuccess) return e;
  }
  if (parts & 2) return launch_mode<kComposeJ>(grid, a, st);
  return cudaSuccess;
}

cudaError_t launch_scan_tc(const uint8_t *Mimg, const float *Jf, const float *Jb, const float *S_T,
                           float *F, float *G, long long BH, int C, int dir_mask, int32_t *info,
                           cudaStream_t st) {
  if (BH <= 0) return cudaSuccess;
  ChainArgs a{};
  a.Mimg = const_cast<uint8_t *>(Mimg);
  a.Jf = const_cast<float *>(Jf);
  a.Jb = const_cast<float *>(Jb);
  a.S_T = S_T;
  a.F = F;
  a.G = G;
  a.info = info;
  a.C = C;
  a.dir_mask = dir_mask;
  return launch_mode<kScan>(dim3((unsigned)BH, 2, 1), a, st);
}

}  // namespace vdn
