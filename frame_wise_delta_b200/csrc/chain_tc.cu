// Chunk composition and the bidirectional scan on the 5th-generation tensor
// cores (tcgen05 + TMEM), d = 128, fp32 state carried as bf16 hi + lo.
// Paper: "Video DeltaNet: A Video-Native Hybrid Attention for Livestream
// Video Generation" (summary page), "Technical novelty" (frame-level affine
// transitions composed into chunk-level ones before the scan) and "Method
// steps" step (4) (S_out = S_in M_chunk + J_chunk, both scans started from
// half of the text state).
//
// Both are chains of products with the state kept on chip:
//
//  compose, one CTA per (direction, b*h, chunk); over the chunk's non-anchor
//  frames in forward or reverse order, with W_t = (I + A_t)^{-1}, the
//  stacked state X = [X_M ; X_J] (256 x 128) follows
//     X <- (X Diag(alpha_t) + [0 ; B_t]) W_t,    X_0 = [I ; 0]
//  and ends as [Mc ; Jc]. This equals X M_t + [0 ; J_t] with
//  M_t = Diag(alpha_t) W_t and J_t = B_t W_t, so the per-frame (M_t, J_t) are
//  never materialised. The M and J rows are independent groups of N = 128.
//
//  scan, one CTA per (b*h, direction, half of the state rows): X <- X Mc_c +
//  Jc_c over the chunks, from X = S_T / 2, writing every boundary state; the
//  rows of X are independent, so each CTA carries 64 of them (N = 64).
//
// One product: D[m][n] = sum_k Op[k][m] E[n][k], i.e. D = (E Op)^T in TMEM
// (lane m = state column, TMEM column n = state row). Op arrives as a
// ready-made hi/lo image (W_t from the factor kernel, Mc_c from the compose)
// by bulk copy; E is written by the threads that own TMEM lane m (state
// column m is row m of E's MN-major image). Three MMAs accumulate
// hi*hi + hi*lo + lo*hi, so each product keeps ~2^-17 relative accuracy: an
// fp32 state on bf16 tensor cores. Owning a state column per thread keeps
// every global access of the epilogue coalesced (a warp reads or writes 32
// consecutive floats of one state row).
//
// Roles (288 threads): warps 0..7 are the epilogue (warp w drains TMEM lanes
// 32(w%4)..+31 for column half w/4; for the compose, half 0 is the M group and
// half 1 the J group, each with its own TMEM accumulator and barriers, so the
// epilogue of one group overlaps the MMAs of the other); warp 8 allocates TMEM
// and one lane issues the bulk copies and the MMAs. The epilogue's fp32 work
// and bf16 splits use packed fp32x2 / bf16x2 instructions. Every wait is
// bounded.
#include "common.cuh"
#include "internal.h"

namespace vdn {
namespace {

constexpr int kD = 128;
constexpr int kWorkers = 256;
constexpr int kThreads = kWorkers + 32;

enum Mode { kCompose = 0, kScan = 1 };

// compose: E (256 rows, 128 KB) + one Op buffer; scan: E (128 rows) + two Op buffers
constexpr size_t kSmemBytes = 1024 + 3 * (size_t)kImgBytes + 128;

struct ChainArgs {
  const uint8_t *Wimg;      // compose: [BH*T] images
  const float *Bm;          // compose: [BH, T, d, d]
  const float *alpha;       // compose: [BH, T, d]
  float *Mf, *Jf, *Mb, *Jb; // compose outputs / scan inputs (J) [BH, C, d, d]
  uint8_t *Mimg;            // compose output / scan input: [BH, 2, C] images of Mc
  const float *S_T;         // scan: [BH, d, d]
  float *F, *G;             // scan outputs [BH, C+1, d, d]
  int32_t *info;
  int T, chunk, C, anchors;
};

__device__ __forceinline__ void fail(volatile int *abort, int32_t *info) {
  *abort = 1;
  if (info) atomicExch(info, VDN_INFO_TIMEOUT);
}

// bf16 hi/lo split of two values with packed instructions: hi = bf16x2(a, b),
// lo = bf16x2 of the fp32 remainders.
__device__ __forceinline__ void split2(float a, float b, uint32_t &hi, uint32_t &lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  const float2 hf = __bfloat1622float2(h);
  const float2 r = __fadd2_rn(make_float2(a, b), make_float2(-hf.x, -hf.y));
  const __nv_bfloat162 l = __floats2bfloat162_rn(r.x, r.y);
  hi = *reinterpret_cast<const uint32_t *>(&h);
  lo = *reinterpret_cast<const uint32_t *>(&l);
}

// Write 32 consecutive values (columns x0 .. x0+31 of image row rr) of an
// MN-major hi/lo image in shared memory whose 64-column regions are `region`
// bytes apart and whose hi and lo halves are `half` bytes apart.
__device__ __forceinline__ void write_img32(uint8_t *img, int rr, int x0, const float (&v)[32],
                                            uint32_t region, uint32_t half) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) split2(v[q * 8 + 2 * e], v[q * 8 + 2 * e + 1], h[e], l[e]);
    const int x = x0 + q * 8;
    const uint32_t off = (uint32_t)(x >> 6) * region + (uint32_t)rr * 128u +
                         ((((uint32_t)(x & 63) >> 3) ^ (uint32_t)(rr & 7)) << 4);
    *reinterpret_cast<uint4 *>(img + off) = make_uint4(h[0], h[1], h[2], h[3]);
    *reinterpret_cast<uint4 *>(img + half + off) = make_uint4(l[0], l[1], l[2], l[3]);
  }
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1) chain_tc_kernel(ChainArgs p) {
  // N: state rows per product; the E image has N/64 regions of kImgRegion bytes
  constexpr int N = MODE == kCompose ? 256 : 64;
  constexpr uint32_t kEHalf = N * kD * 2;  // bytes of one bf16 part of E
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  uint8_t *eimg = smem;                              // 2 * kEHalf bytes
  uint8_t *opbase = smem + 2 * kEHalf;               // compose: 1 buffer, scan: 2
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + 3 * kImgBytes);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 8);
  volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
  // Independent row groups: compose runs the M rows and the J rows as two
  // groups (each N = 128) so one group's epilogue overlaps the other's MMAs;
  // the scan is one group.
  constexpr int NG = MODE == kCompose ? 2 : 1;
  constexpr int kGroupWorkers = kWorkers / NG;
  const uint32_t ready0 = smem_u32(bars);  // ready[g]
  const uint32_t done0 = ready0 + 16;      // done[g]
  const uint32_t opfull0 = ready0 + 32;    // opfull[b]
  const uint32_t drain = ready0 + 48;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long DD = (long long)kD * kD;

  // ---- the chain this CTA walks
  long long bh;
  int dir, c_cmp = 0, nsteps = 0, hz = 0;
  int frames[16];
  if (MODE == kScan) {
    bh = blockIdx.x;
    dir = blockIdx.y;
    hz = blockIdx.z;  // state rows 64 hz .. 64 hz + 63
    nsteps = p.C;
  } else {
    dir = blockIdx.x;
    bh = blockIdx.y;
    c_cmp = blockIdx.z;
    const int t0 = c_cmp * p.chunk, t1 = min(t0 + p.chunk, p.T);
    for (int s = 0; s < t1 - t0; ++s) {
      const int t = dir == 0 ? t0 + s : t1 - 1 - s;
      if (p.anchors && (t == 0 || t == p.T - 1)) continue;
      frames[nsteps++] = t;
    }
  }
  auto scan_c = [&](int s) { return dir == 0 ? s : p.C - 1 - s; };
  auto op_src = [&](int s) -> const uint8_t * {
    if (MODE == kScan) return p.Mimg + ((bh * 2 + dir) * p.C + scan_c(s)) * (long long)kImgBytes;
    return p.Wimg + (bh * p.T + frames[s]) * (long long)kImgBytes;
  };
  constexpr int kBufs = MODE == kCompose ? 1 : 2;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(ready0 + 8 * i, kGroupWorkers);
      mbar_init(done0 + 8 * i, 1);
      mbar_init(opfull0 + 8 * i, 1);
    }
    mbar_init(drain, 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 8) tmem_alloc(smem_u32(tmem_slot), (uint32_t)N);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 8) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, MODE == kCompose ? 128 : 64, true, true);
      const uint32_t e_hi = smem_u32(eimg), e_lo = e_hi + kEHalf;
      auto load = [&](int s) {
        const int b = s % kBufs;
        const uint32_t bar = opfull0 + 8 * b;
        mbar_arrive_expect_tx(bar, kImgBytes);
        const uint32_t dst = smem_u32(opbase + b * kImgBytes);
        const uint8_t *src = op_src(s);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          bulk_load(dst + q * (kImgBytes / 4), src + q * (kImgBytes / 4), kImgBytes / 4, bar);
      };
      int loads = 0;
      for (; loads < kBufs && loads < nsteps; ++loads) load(loads);
      bool ok = true;
      for (int s = 0; ok && s < nsteps; ++s) {
        const int b = s % kBufs;
        if (!mbar_wait(opfull0 + 8 * b, (uint32_t)((s / kBufs) & 1), abort)) {
          fail(abort, p.info);
          break;
        }
        const uint32_t o_hi = smem_u32(opbase + b * kImgBytes), o_lo = o_hi + kImgHalf;
        for (int g = 0; g < NG; ++g) {
          if (!mbar_wait(ready0 + 8 * g, (uint32_t)(s & 1), abort)) {
            fail(abort, p.info);
            ok = false;
            break;
          }
          tc_fence_after();
          // group g: state rows 128g.. (E image regions 2g, 2g+1), TMEM columns 128g..
          const uint32_t eg_hi = e_hi + (uint32_t)(g * 2 * kImgRegion), eg_lo = e_lo + (uint32_t)(g * 2 * kImgRegion);
#pragma unroll
          for (int part = 0; part < 3; ++part) {
            const uint32_t a0 = part == 2 ? o_lo : o_hi;
            const uint32_t b0 = part == 1 ? eg_lo : eg_hi;
#pragma unroll
            for (int ks = 0; ks < kD / 16; ++ks) {
              const uint64_t ad = smem_desc_sw128(a0 + ks * 2048, kImgRegion, 1024);
              const uint64_t bd = smem_desc_sw128(b0 + ks * 2048, kImgRegion, 1024);
              tc_mma_bf16(tmem_base + (uint32_t)(128 * g), ad, bd, idesc, (part > 0 || ks > 0) ? 1u : 0u);
            }
          }
          tc_commit(done0 + 8 * g);
        }
        if (ok && loads < nsteps) {
          // the next load (step s + kBufs) reuses this step's buffer: wait for
          // the MMAs of the last group (hence of every group) to finish
          if (!mbar_wait(done0 + 8 * (NG - 1), (uint32_t)(s & 1), abort)) {
            fail(abort, p.info);
            break;
          }
          load(loads++);
        }
      }
      // every issued copy has landed and every MMA is done before leaving
      volatile int never = 0;
      for (int s = (loads > kBufs ? loads - kBufs : 0); s < loads; ++s)
        mbar_wait(opfull0 + 8 * (s % kBufs), (uint32_t)((s / kBufs) & 1), &never);
      tc_commit(drain);
      mbar_wait(drain, 0, &never);
    }
  } else {
    // ---- epilogue: thread owns state column m (TMEM lane m) for column half h
    const int m = (warp & 3) * 32 + lane;
    const int h = warp >> 2;                     // scan: rows 64hz+32h..+31; compose: group (0 M, 1 J)
    const int grp = MODE == kCompose ? h : 0;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    constexpr int kRows = MODE == kCompose ? 128 : 32;  // state rows handled per thread
    const int row0 = MODE == kCompose ? 0 : 64 * hz + 32 * h;  // first state row of this thread
    const int tcol0 = MODE == kCompose ? 128 * h : 32 * h;     // first TMEM column / E image column

    // ---- E_0 (and, for the scan, the first boundary state)
    if (MODE == kScan) {
      const float *st = p.S_T + bh * DD + m;
      float *o = (dir == 0 ? p.F + (bh * (p.C + 1)) * DD : p.G + (bh * (p.C + 1) + p.C) * DD) + m;
      float x0[kRows];  // every load first: one memory latency, not one per block
#pragma unroll
      for (int e = 0; e < kRows; ++e) x0[e] = 0.5f * st[(row0 + e) * kD];
#pragma unroll
      for (int j = 0; j < kRows / 32; ++j) {
        float v[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          v[e] = x0[32 * j + e];
          o[(row0 + 32 * j + e) * kD] = v[e];
        }
        if (nsteps > 0) write_img32(eimg, m, tcol0 + 32 * j, v, kImgRegion, kEHalf);
      }
    } else {
      const long long cidx = bh * p.C + c_cmp;
      float *out = h == 0 ? (dir == 0 ? p.Mf : p.Mb) : (dir == 0 ? p.Jf : p.Jb);
      uint8_t *out_img = (h == 0 && p.Mimg) ? p.Mimg + ((bh * 2 + dir) * p.C + c_cmp) * (long long)kImgBytes : nullptr;
      if (nsteps == 0) {  // every frame of the chunk is an anchor: identity map
        for (int n = 0; n < kD; ++n) {
          const float x0 = (h == 0 && n == m) ? 1.f : 0.f;
          if (out) out[cidx * DD + n * kD + m] = x0;
          if (out_img) img_store(out_img, n, m, x0);
        }
      } else {
        const float al = p.alpha[(bh * p.T + frames[0]) * kD + m];
        const float *Bt = p.Bm + (bh * p.T + frames[0]) * DD + m;
        float b0[kD];  // every load first: one memory latency, not one per block
        if (h == 1) {
#pragma unroll
          for (int e = 0; e < kD; ++e) b0[e] = Bt[e * kD];
        }
#pragma unroll
        for (int j = 0; j < kD / 32; ++j) {
          float v[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = h == 0 ? ((32 * j + e == m) ? al : 0.f) : b0[32 * j + e];
          write_img32(eimg, m, tcol0 + 32 * j, v, kImgRegion, kEHalf);
        }
      }
    }
    if (nsteps > 0) {
      fence_proxy_async_smem();
      mbar_arrive(ready0 + 8 * grp);
    }

    for (int s = 0; s < nsteps; ++s) {
      const bool last = (s + 1 == nsteps);
      // operands of this step's epilogue, fetched while the MMAs run
      float al = 1.f;
      const float *add = nullptr;
      float *o = nullptr;
      uint8_t *o_img = nullptr;
      if (MODE == kScan) {
        const int c = scan_c(s);
        add = (dir == 0 ? p.Jf : p.Jb) + (bh * p.C + c) * DD + m;
        o = (dir == 0 ? p.F + (bh * (p.C + 1) + c + 1) * DD : p.G + (bh * (p.C + 1) + c) * DD) + m;
      } else if (!last) {
        al = p.alpha[(bh * p.T + frames[s + 1]) * kD + m];
        if (h == 1) add = p.Bm + (bh * p.T + frames[s + 1]) * DD + m;
      } else {
        const long long cidx = bh * p.C + c_cmp;
        float *oo = h == 0 ? (dir == 0 ? p.Mf : p.Mb) : (dir == 0 ? p.Jf : p.Jb);
        o = oo ? oo + cidx * DD + m : nullptr;
        if (h == 0 && p.Mimg) o_img = p.Mimg + ((bh * 2 + dir) * p.C + c_cmp) * (long long)kImgBytes;
      }
      float addv[kRows];
      if (add) {
#pragma unroll
        for (int e = 0; e < kRows; ++e) addv[e] = add[(row0 + e) * kD];
      }
      if (!__all_sync(0xffffffffu, mbar_wait(done0 + 8 * grp, (uint32_t)(s & 1), abort))) {
        fail(abort, p.info);
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int j = 0; j < kRows / 32; ++j) {
        const int n0 = row0 + 32 * j;  // state rows n0 .. n0+31
        float v[32];
        tmem_ld32(tmem_base + lane_off + (uint32_t)(tcol0 + 32 * j), v);
        if (MODE == kScan) {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] += addv[32 * j + e];
#pragma unroll
          for (int e = 0; e < 32; ++e) o[(n0 + e) * kD] = v[e];
          if (!last) write_img32(eimg, m, tcol0 + 32 * j, v, kImgRegion, kEHalf);
        } else if (!last) {
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float2 r2 = __ffma2_rn(make_float2(v[e], v[e + 1]), make_float2(al, al),
                                         add ? make_float2(addv[32 * j + e], addv[32 * j + e + 1]) : make_float2(0.f, 0.f));
            v[e] = r2.x;
            v[e + 1] = r2.y;
          }
          write_img32(eimg, m, tcol0 + n0, v, kImgRegion, kEHalf);
        } else {
          if (o) {
#pragma unroll
            for (int e = 0; e < 32; ++e) o[(n0 + e) * kD] = v[e];
          }
          if (o_img) {
#pragma unroll
            for (int e = 0; e < 32; ++e) img_store(o_img, n0 + e, m, v[e]);
          }
        }
      }
      if (!last) {
        tc_fence_before();
        fence_proxy_async_smem();
        mbar_arrive(ready0 + 8 * grp);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, (uint32_t)N);
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
                              int chunk, int anchors, int ndirs, int32_t *info, cudaStream_t st) {
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
  // direction fastest, so the two CTAs that read the same W images run together
  return launch_mode<kCompose>(dim3((unsigned)ndirs, (unsigned)BH, (unsigned)a.C), a, st);
}

cudaError_t launch_scan_tc(const uint8_t *Mimg, const float *Jf, const float *Jb, const float *S_T,
                           float *F, float *G, long long BH, int C, int32_t *info, cudaStream_t st) {
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
  return launch_mode<kScan>(dim3((unsigned)BH, 2, 2), a, st);
}

}  // namespace vdn
