// The bidirectional scan over chunks on the 5th-generation tensor cores
// (tcgen05 + TMEM), d = 128, fp32 state carried as bf16 hi + lo.
// Paper: "Video DeltaNet: A Video-Native Hybrid Attention for Livestream
// Video Generation" (summary page), "Core method" (forward and backward
// scans) and "Method steps" step (4) (S_out = S_in M_chunk + J_chunk, both
// scans started from half of the text state).
//
// One CTA per (b*h, direction, half of the state rows): X <- X Mc_c + Jc_c
// over the chunks, from X = S_T / 2, writing every boundary state. The rows
// of X are independent, so each CTA carries 64 of them (N = 64).
//
// One product: D[m][n] = sum_k Mc[k][m] E[n][k], i.e. D = (E Mc)^T in TMEM
// (lane m = state column, TMEM column n = state row). Mc arrives as the
// transposed hi/lo image the composition writes (the K-major A operand) by
// bulk copy, double-buffered; E is written by the threads that own TMEM lane m
// (state column m is row m of E's MN-major image). Three MMAs accumulate
// hi*hi + hi*lo + lo*hi, so each product keeps ~2^-17 relative accuracy: an
// fp32 state on bf16 tensor cores. Owning a state column per thread keeps the
// boundary-state writes coalesced (a warp writes 32 consecutive floats of one
// state row). Jc comes transposed and is brought into shared memory by TMA
// with the 128-byte swizzle, two steps ahead with the Mc image, so each
// thread's 32 added values are one conflict-free 128-byte row.
//
// Roles (288 threads): warps 0..7 are the epilogue (warp w drains TMEM lanes
// 32(w%4)..+31 for state rows 32(w/4)..+31 of the CTA's 64); warp 8
// allocates TMEM and one lane issues the copies and the MMAs. Every wait is
// bounded.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"

namespace vdn {
namespace {

constexpr int kD = 128;
constexpr int kN = 64;                      // state rows per CTA
constexpr int kRows = 32;                   // state rows per epilogue thread
constexpr int kThreads = 8 * 32 + 32;
constexpr uint32_t kEHalf = kN * kD * 2;    // bytes of one bf16 part of E
constexpr int kBufs = 2;                    // Mc image and Jc buffers
constexpr uint32_t kJBox = 128 * 32 * 4;    // TMA box of transposed Jc: 128 columns m x 32 rows n
constexpr uint32_t kJBytes = 2 * kJBox;     // the CTA's 64 rows
// E (2 parts) + Mc images + Jc tiles + barriers
constexpr uint32_t kOffOp = 2 * kEHalf;
constexpr uint32_t kOffJ = kOffOp + kBufs * kImgBytes;
constexpr uint32_t kOffBar = kOffJ + kBufs * kJBytes;
constexpr size_t kSmemBytes = 1024 + kOffBar + 128;

struct ScanArgs {
  const uint8_t *Mimg;       // [BH, 2, C] transposed images of Mc
  const float *S_T;          // [BH, d, d]
  float *F, *G;              // [BH, C+1, d, d]
  int32_t *info;
  int C;
  float init_scale;          // the state starts as init_scale * S_T
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

// Write 32 consecutive values (columns x0 .. x0+31 of image row rr, x0 < 64)
// of an MN-major hi/lo image in shared memory whose hi and lo halves are
// `half` bytes apart.
__device__ __forceinline__ void write_img32(uint8_t *img, int rr, int x0, const float (&v)[32], uint32_t half) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) split2(v[q * 8 + 2 * e], v[q * 8 + 2 * e + 1], h[e], l[e]);
    const int x = x0 + q * 8;
    const uint32_t off = (uint32_t)rr * 128u + ((((uint32_t)x >> 3) ^ (uint32_t)(rr & 7)) << 4);
    *reinterpret_cast<uint4 *>(img + off) = make_uint4(h[0], h[1], h[2], h[3]);
    *reinterpret_cast<uint4 *>(img + half + off) = make_uint4(l[0], l[1], l[2], l[3]);
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    scan_tc_kernel(const __grid_constant__ CUtensorMap tmJf, const __grid_constant__ CUtensorMap tmJb, ScanArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  uint8_t *eimg = smem;                    // 2 * kEHalf bytes
  uint8_t *opbase = smem + kOffOp;         // kBufs Mc images
  const uint8_t *jbase = smem + kOffJ;     // kBufs Jc tiles
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 8);
  volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
  const uint32_t ready = smem_u32(bars), done = ready + 8, drain = ready + 16;
  const uint32_t opfull0 = ready + 24;  // opfull[b]: Mc image and Jc tile of a step
  const uint32_t jfree0 = ready + 40;   // jfree[b]: the epilogue has read the Jc tile
  const CUtensorMap *tmJ = blockIdx.y == 0 ? &tmJf : &tmJb;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr long long DD = (long long)kD * kD;
  const long long bh = blockIdx.x;
  const int dir = blockIdx.y;
  const int hz = blockIdx.z;  // state rows 64 hz .. 64 hz + 63
  const int nsteps = p.C;
  auto scan_c = [&](int s) { return dir == 0 ? s : p.C - 1 - s; };

  if (threadIdx.x == 0) {
    mbar_init(ready, 8 * 32);
    mbar_init(done, 1);
    mbar_init(drain, 1);
    for (int i = 0; i < kBufs; ++i) {
      mbar_init(opfull0 + 8 * i, 1);
      mbar_init(jfree0 + 8 * i, 8 * 32);
    }
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 8) tmem_alloc(smem_u32(tmem_slot), (uint32_t)kN);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 8) {
    if (lane == 0) {
      // A = Mc image K-major, B = E MN-major
      constexpr uint32_t idesc = idesc_bf16_f32(128, kN, false, true);
      const uint32_t e_hi = smem_u32(eimg), e_lo = e_hi + kEHalf;
      tma_prefetch_desc(tmJ);
      auto load = [&](int s) {
        const int b = s % kBufs;
        const uint32_t bar = opfull0 + 8 * b;
        mbar_arrive_expect_tx(bar, kImgBytes + kJBytes);
        const uint32_t dst = smem_u32(opbase + b * kImgBytes);
        const long long cidx = (bh * 2 + dir) * p.C + scan_c(s);
        const uint8_t *src = p.Mimg + cidx * (long long)kImgBytes;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          bulk_load(dst + q * (kImgBytes / 4), src + q * (kImgBytes / 4), kImgBytes / 4, bar);
        // transposed Jc of (b*h, chunk): columns n = 64 hz .. 64 hz + 63 of all 128 rows m
#pragma unroll
        for (int q = 0; q < 2; ++q)
          tma_load_3d(smem_u32(jbase + b * kJBytes + q * kJBox), tmJ, bar, 64 * hz + 32 * q, 0,
                      (int)(bh * p.C + scan_c(s)));
      };
      int loads = 0;
      for (; loads < kBufs && loads < nsteps; ++loads) load(loads);
      for (int s = 0; s < nsteps; ++s) {
        const int b = s % kBufs;
        if (!mbar_wait(opfull0 + 8 * b, (uint32_t)((s / kBufs) & 1), abort) ||
            !mbar_wait(ready, (uint32_t)(s & 1), abort)) {
          fail(abort, p.info);
          break;
        }
        tc_fence_after();
        const uint32_t o_hi = smem_u32(opbase + b * kImgBytes), o_lo = o_hi + kImgHalf;
#pragma unroll
        for (int part = 0; part < 3; ++part) {
          const uint32_t a0 = part == 2 ? o_lo : o_hi;
          const uint32_t b0 = part == 1 ? e_lo : e_hi;
#pragma unroll
          for (int ks = 0; ks < kD / 16; ++ks) {
            const uint64_t ad = smem_desc_sw128(a0 + (ks >> 2) * kImgRegion + (ks & 3) * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(b0 + ks * 2048, kImgRegion, 1024);
            tc_mma_bf16(tmem_base, ad, bd, idesc, (part > 0 || ks > 0) ? 1u : 0u);
          }
        }
        tc_commit(done);
        if (loads < nsteps) {
          // the next load (step s + kBufs) reuses this step's buffers: the MMAs
          // have read the image and the epilogue the Jc tile
          if (!mbar_wait(done, (uint32_t)(s & 1), abort) ||
              !mbar_wait(jfree0 + 8 * b, (uint32_t)((s / kBufs) & 1), abort)) {
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
    // ---- epilogue: thread owns state column m (TMEM lane m)
    const int m = (warp & 3) * 32 + lane;
    const int h = warp >> 2;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const int row0 = 64 * hz + 32 * h;  // first state row of this thread
    const int tcol0 = 32 * h;           // its TMEM column / E image column

    // ---- E_0 and the first boundary state
    {
      const float *st = p.S_T + bh * DD + m;
      float *o = (dir == 0 ? p.F + (bh * (p.C + 1)) * DD : p.G + (bh * (p.C + 1) + p.C) * DD) + m;
      float v[kRows];  // every load first: one memory latency, not one per row
#pragma unroll
      for (int e = 0; e < kRows; ++e) v[e] = p.init_scale * st[(row0 + e) * kD];
#pragma unroll
      for (int e = 0; e < kRows; ++e) o[(row0 + e) * kD] = v[e];
      if (nsteps > 0) {
        write_img32(eimg, m, tcol0, v, kEHalf);
        fence_proxy_async_smem();
        mbar_arrive(ready);
      }
    }

    for (int s = 0; s < nsteps; ++s) {
      const bool last = (s + 1 == nsteps);
      const int c = scan_c(s);
      float *o = (dir == 0 ? p.F + (bh * (p.C + 1) + c + 1) * DD : p.G + (bh * (p.C + 1) + c) * DD) + m;
      const int b = s % kBufs;
      if (!__all_sync(0xffffffffu, mbar_wait(opfull0 + 8 * b, (uint32_t)((s / kBufs) & 1), abort) &&
                                       mbar_wait(done, (uint32_t)(s & 1), abort))) {
        fail(abort, p.info);
        break;
      }
      tc_fence_after();
      float v[32];
      tmem_ld32(tmem_base + lane_off + (uint32_t)tcol0, v);
      // + Jc: row m of this thread's box, 16-byte chunks permuted by (m & 7)
      {
        const uint8_t *jrow = jbase + b * kJBytes + h * kJBox + m * 128;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 a4 = *reinterpret_cast<const float4 *>(jrow + ((q ^ (m & 7)) << 4));
          v[4 * q] += a4.x;
          v[4 * q + 1] += a4.y;
          v[4 * q + 2] += a4.z;
          v[4 * q + 3] += a4.w;
        }
      }
      mbar_arrive(jfree0 + 8 * b);
      // the next operand first (the next product waits for it), then the
      // boundary state, whose stores drain under that product
      if (!last) {
        write_img32(eimg, m, tcol0, v, kEHalf);
        tc_fence_before();
        fence_proxy_async_smem();
        mbar_arrive(ready);
      }
#pragma unroll
      for (int e = 0; e < 32; ++e) o[(row0 + e) * kD] = v[e];
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, (uint32_t)kN);
  }
}

// 3-D tensor map over transposed Jc ([maps][128 rows m][128 columns n] fp32)
// with a (32 columns x 128 rows x 1) box and the 128-byte swizzle.
bool make_jt_map(CUtensorMap *m, const float *J, long long maps) {
  auto enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)kD, (cuuint64_t)maps};
  cuuint64_t strides[2] = {(cuuint64_t)kD * 4, (cuuint64_t)kD * kD * 4};
  cuuint32_t box[3] = {32, (cuuint32_t)kD, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float *>(J), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_scan_tc(const uint8_t *Mimg, const float *Jf, const float *Jb, const float *S_T,
                           float *F, float *G, long long BH, int C, int32_t *info, cudaStream_t st,
                           int dir_mask, float init_scale) {
  if (BH <= 0) return cudaSuccess;
  // with no chunks the maps are never read: describe S_T instead of empty Jc
  CUtensorMap tmJf, tmJb;
  const long long maps = C > 0 ? BH * C : BH;
  if (!make_jt_map(&tmJf, C > 0 ? Jf : S_T, maps) || !make_jt_map(&tmJb, C > 0 ? (Jb ? Jb : Jf) : S_T, maps))
    return cudaErrorInvalidValue;
  ScanArgs a{};
  a.Mimg = Mimg;
  a.S_T = S_T;
  a.F = F;
  a.G = G;
  a.info = info;
  a.C = C;
  a.init_scale = init_scale;
  cudaError_t e = cudaFuncSetAttribute(scan_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  // forward only: grid.y = 1 (direction 0); backward only is not needed
  scan_tc_kernel<<<dim3((unsigned)BH, dir_mask == 1 ? 1 : 2, 2), kThreads, kSmemBytes, st>>>(tmJf, tmJb, a);
  return cudaGetLastError();
}

}  // namespace vdn
