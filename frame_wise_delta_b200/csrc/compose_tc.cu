// Chunk composition on the 5th-generation tensor cores (tcgen05), d = 128,
// with the chain state held in tensor memory.
// Paper: "Video DeltaNet: A Video-Native Hybrid Attention for Livestream
// Video Generation" (summary page), "Technical novelty" (frame-level affine
// transitions composed into chunk-level ones before the scan) and "Method
// steps" step (4).
//
// For one (direction, b*h, chunk), over the chunk's non-anchor frames in
// forward or reverse order and with W_t = (I + A_t)^{-1}, the stacked state
// X = [X_M ; X_J] (256 x 128) follows
//     X <- (X Diag(alpha_t) + [0 ; B_t]) W_t,    X_0 = [I ; 0]
// and ends as [Mc ; Jc]. This equals X M_t + [0 ; J_t] with
// M_t = Diag(alpha_t) W_t and J_t = B_t W_t, so the per-frame M_t, J_t are
// never materialised. The M rows and the J rows are independent groups.
//
// One product per group and frame: D[n][m] = sum_k E[n][k] W[k][m], where the
// operand E = X Diag(alpha_t) (+ B_t) lives in TMEM (state row n on lane n, as
// bf16 hi and lo parts) and W is the hi/lo image the factor kernel writes,
// read from shared memory. Three MMAs accumulate hi*hi + lo*hi + hi*lo, so each
// product keeps ~2^-17 relative accuracy: an fp32 state on bf16 tensor cores.
//
// Persistent CTAs (one per SM) take chains blockIdx.x, + gridDim.x, ...; the
// steps of all of a CTA's chains form one stream, so the loads for the next
// chain overlap the last products of the current one.
//
// Roles (320 threads):
//   warps 0..7  epilogue: warp w owns one state row per thread (TMEM lanes
//               32(w % 4) ..) and the column half w / 4 of both groups; it
//               reads accumulator rows with tcgen05.ld and writes the next
//               operand rows with tcgen05.st. The groups have their own
//               accumulators and barriers, so one group's operand update (on
//               all eight warps) overlaps the other group's MMAs;
//   warp 8      allocates TMEM; one lane issues the MMAs;
//   warp 9      one lane issues the loads: W images into two buffers (bulk
//               copies), B_t by TMA in two column halves with the 128-byte
//               swizzle (each thread then reads its own row without bank
//               conflicts), and alpha_t.
// Every wait is bounded.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"

namespace vdn {
namespace {

constexpr int kD = 128;
constexpr int kThreads = 320;
constexpr uint32_t kBBox = 128 * 32 * 4;         // TMA box of B_t: 128 rows x 32 columns fp32
constexpr uint32_t kBHalf = 2 * kBBox;           // columns 64h .. 64h + 63
constexpr uint32_t kAlphaBytes = kD * 4;
// shared memory, from a 1024-byte aligned base
constexpr uint32_t kOffW = 0;                           // two W images
constexpr uint32_t kOffB = kOffW + 2 * kImgBytes;       // B_t: four boxes
constexpr uint32_t kOffAl = kOffB + 2 * kBHalf;         // alpha_t: two slots
constexpr uint32_t kOffBar = kOffAl + 2 * kAlphaBytes;  // barriers, TMEM address, abort flag
constexpr size_t kSmemBytes = 1024 + kOffBar + 256;
// TMEM columns: accumulator of group g at 128 g; operand of group g at
// 256 + 128 g (hi part, 64 columns of bf16 pairs) and 320 + 128 g (lo part)
constexpr uint32_t kColD = 0, kColE = 256, kTmemCols = 512;

struct ComposeArgs {
  const uint8_t *Wimg;       // [BH*T] images of W_t
  const float *alpha;        // [BH, T, d]
  float *Mf, *Jf, *Mb, *Jb;  // [BH, C, d, d], each optional
  uint8_t *Mimg;             // [BH, 2, C] images of Mc, optional
  int32_t *info;
  long long BH, nchains;
  int T, chunk, C, anchors, ndirs;
  int jt;  // J outputs transposed (Jc[n][m] at m * d + n)
};

// A chain and the frames it takes: anchors only sit at t = 0 (anchors bit 0)
// and t = T - 1 (bit 1), so the non-anchor frames of a chunk are the
// contiguous range [lo, hi].
struct Chain {
  long long bh;
  int dir, c, lo, hi, nsteps;
  __device__ __forceinline__ int frame(int s) const { return dir == 0 ? lo + s : hi - s; }
};

__device__ __forceinline__ Chain decode(const ComposeArgs &p, long long q) {
  Chain ch;
  ch.dir = (int)(q % p.ndirs);
  const long long r = q / p.ndirs;
  ch.bh = r % p.BH;
  ch.c = (int)(r / p.BH);
  const int t0 = ch.c * p.chunk, t1 = min(t0 + p.chunk, p.T);
  ch.lo = ((p.anchors & 1) && t0 == 0) ? 1 : t0;
  ch.hi = ((p.anchors & 2) && t1 == p.T) ? p.T - 2 : t1 - 1;
  ch.nsteps = max(ch.hi - ch.lo + 1, 0);
  return ch;
}

__device__ __forceinline__ void fail(volatile int *abort, int32_t *info) {
  *abort = 1;
  if (info) atomicExch(info, VDN_INFO_TIMEOUT);
}

// Row n of an operand chunk (32 columns) as TMEM words: bf16 pairs of
// columns (2i, 2i + 1), hi parts and lo parts.
__device__ __forceinline__ void pack_row32(const float (&v)[32], uint32_t (&hi)[16], uint32_t (&lo)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) split_bf16x2(v[2 * i], v[2 * i + 1], hi[i], lo[i]);
}

// Columns 32j .. 32j + 31 of row n of B_t from its swizzled boxes.
__device__ __forceinline__ void load_b_row32(const uint8_t *bbuf, int j, int n, float (&b)[32]) {
  const uint8_t *row = bbuf + j * kBBox + n * 128;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const float4 x = *reinterpret_cast<const float4 *>(row + ((c ^ (n & 7)) << 4));
    b[4 * c] = x.x;
    b[4 * c + 1] = x.y;
    b[4 * c + 2] = x.z;
    b[4 * c + 3] = x.w;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    compose_tc_kernel(const __grid_constant__ CUtensorMap tmB, ComposeArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
  const uint32_t bar0 = smem_u32(bars);
  const uint32_t wfull = bar0, wfree = bar0 + 16;  // per W buffer
  const uint32_t bfull = bar0 + 32, bfree = bar0 + 48;  // per B half
  const uint32_t ready = bar0 + 64, done = bar0 + 80;   // per group
  const uint32_t afull = bar0 + 96, afree = bar0 + 112; // per alpha slot
  const uint32_t drain = bar0 + 128;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 17);
  volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr long long DD = (long long)kD * kD;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(wfull + 8 * i, 1);
      mbar_init(wfree + 8 * i, 1);
      mbar_init(bfull + 8 * i, 1);
      mbar_init(bfree + 8 * i, 128);
      mbar_init(ready + 8 * i, 256);
      mbar_init(done + 8 * i, 1);
      mbar_init(afull + 8 * i, 1);
      mbar_init(afree + 8 * i, 256);
    }
    mbar_init(drain, 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 8) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 9) {
    // ---------------------------------------------------------------- loads
    if (lane == 0) {
      tma_prefetch_desc(&tmB);
      // loads issued: W images, alpha rows, B halves (one of each per step)
      long long wl = 0, al = 0, bl[2] = {0, 0};
      bool ok = true;
      for (long long q = blockIdx.x; ok && q < p.nchains; q += gridDim.x) {
        const Chain ch = decode(p, q);
        for (int s = 0; ok && s < ch.nsteps; ++s) {
          const long long f = ch.bh * p.T + ch.frame(s);
          // W_t: buffer wl % 2, free once the MMAs of step wl - 2 are done
          const int wb = (int)(wl & 1);
          if (wl >= 2 && !mbar_wait(wfree + 8 * wb, (uint32_t)(((wl - 2) >> 1) & 1), abort)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(wfull + 8 * wb, kImgBytes);
          const uint32_t wdst = smem_u32(smem + kOffW + wb * kImgBytes);
          const uint8_t *wsrc = p.Wimg + f * kImgBytes;
#pragma unroll
          for (int i = 0; i < 4; ++i)
            bulk_load(wdst + i * (kImgBytes / 4), wsrc + i * (kImgBytes / 4), kImgBytes / 4, wfull + 8 * wb);
          ++wl;
          // alpha_t: slot al % 2, free once both groups have read step al - 2
          const int as = (int)(al & 1);
          if (al >= 2 && !mbar_wait(afree + 8 * as, (uint32_t)(((al - 2) >> 1) & 1), abort)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(afull + 8 * as, kAlphaBytes);
          bulk_load(smem_u32(smem + kOffAl + as * kAlphaBytes), p.alpha + f * kD, kAlphaBytes, afull + 8 * as);
          ++al;
          // B_t by column halves, each free once the J group has read it
          for (int h = 0; h < 2; ++h) {
            if (bl[h] >= 1 && !mbar_wait(bfree + 8 * h, (uint32_t)((bl[h] - 1) & 1), abort)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(bfull + 8 * h, kBHalf);
#pragma unroll
            for (int b = 0; b < 2; ++b)
              tma_load_3d(smem_u32(smem + kOffB + (2 * h + b) * kBBox), &tmB, bfull + 8 * h, 32 * (2 * h + b),
                          0, (int)f);
            ++bl[h];
          }
        }
      }
      if (!ok) fail(abort, p.info);
      // every copy issued lands before the CTA may leave (only the newest
      // load on each barrier can still be in flight)
      volatile int never = 0;
      for (long long i = (wl > 2 ? wl - 2 : 0); i < wl; ++i)
        mbar_wait(wfull + 8 * (i & 1), (uint32_t)((i >> 1) & 1), &never);
      for (long long i = (al > 2 ? al - 2 : 0); i < al; ++i)
        mbar_wait(afull + 8 * (i & 1), (uint32_t)((i >> 1) & 1), &never);
      for (int h = 0; h < 2; ++h)
        if (bl[h] > 0) mbar_wait(bfull + 8 * h, (uint32_t)((bl[h] - 1) & 1), &never);
    }
  } else if (warp == 8) {
    // ----------------------------------------------------------------- MMAs
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false, true);  // A from TMEM, B MN-major
      long long gs = 0;
      bool ok = true;
      for (long long q = blockIdx.x; ok && q < p.nchains; q += gridDim.x) {
        const Chain ch = decode(p, q);
        for (int s = 0; s < ch.nsteps; ++s, ++gs) {
          const int wb = (int)(gs & 1);
          if (!mbar_wait(wfull + 8 * wb, (uint32_t)((gs >> 1) & 1), abort)) {
            ok = false;
            break;
          }
          const uint32_t w_hi = smem_u32(smem + kOffW + wb * kImgBytes), w_lo = w_hi + kImgHalf;
          for (int g = 0; g < 2; ++g) {
            if (!mbar_wait(ready + 8 * g, (uint32_t)(gs & 1), abort)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t d = tmem + kColD + 128 * g, e_hi = tmem + kColE + 128 * g, e_lo = e_hi + 64;
#pragma unroll
            for (int ks = 0; ks < kD / 16; ++ks) {
              const uint64_t bh = smem_desc_sw128(w_hi + ks * 2048, kImgRegion, 1024);
              const uint64_t blo = smem_desc_sw128(w_lo + ks * 2048, kImgRegion, 1024);
              tc_mma_bf16_ts(d, e_hi + 8 * ks, bh, idesc, ks > 0 ? 1u : 0u);
              tc_mma_bf16_ts(d, e_lo + 8 * ks, bh, idesc, 1u);
              tc_mma_bf16_ts(d, e_hi + 8 * ks, blo, idesc, 1u);
            }
            tc_commit(done + 8 * g);
          }
          if (!ok) break;
          tc_commit(wfree + 8 * wb);
        }
      }
      if (!ok) fail(abort, p.info);
      volatile int never = 0;
      tc_commit(drain);
      mbar_wait(drain, 0, &never);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Every epilogue warp serves both groups: warp w owns TMEM lanes
    // 32(w % 4) .. + 31 (state rows n) and the column half ch = w / 4 of each
    // accumulator and operand, so a group's operand update runs on all eight
    // warps while the other group's product runs.
    const int ch = warp >> 2;              // columns 64 ch .. 64 ch + 63
    const int n = (warp & 3) * 32 + lane;  // state row (TMEM lane)
    const uint32_t lanes = (uint32_t)((warp & 3) * 32) << 16;
    const uint8_t *bbuf = smem + kOffB;
    auto tD = [&](int g) { return tmem + lanes + kColD + 128 * g + 64 * ch; };
    auto tEh = [&](int g) { return tmem + lanes + kColE + 128 * g + 32 * ch; };
    auto alpha_slot = [&](long long i) {
      return reinterpret_cast<const float *>(smem + kOffAl + (i & 1) * kAlphaBytes) + 64 * ch;
    };
    auto wait_alpha = [&](long long i) {
      return __all_sync(0xffffffffu, mbar_wait(afull + 8 * (i & 1), (uint32_t)((i >> 1) & 1), abort));
    };
    auto wait_b = [&](long long i) {  // this warp's column half of B_t
      return __all_sync(0xffffffffu, mbar_wait(bfull + 8 * ch, (uint32_t)(i & 1), abort));
    };
    // Operand chunk j (of this half) of group g, row n
    auto put_operand = [&](int g, int j, const float (&v)[32]) {
      uint32_t hi[16], lo[16];
      pack_row32(v, hi, lo);
      tmem_st16(tEh(g) + 16 * j, hi);
      tmem_st16(tEh(g) + 64 + 16 * j, lo);
    };
    auto publish = [&](int g) {
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(ready + 8 * g);
    };
    // Columns 64 ch + 32 j .. + 31 of row n of a chain's result. Transposed
    // outputs (the image of Mc, Jc with jt) put the 32 threads of a warp on
    // consecutive addresses for each column m, so those stores coalesce.
    auto write_out = [&](int g, int j, const float (&v)[32], float *oF, uint8_t *oI) {
      const int m0 = 64 * ch + 32 * j;
      if (oF) {
        if (p.jt && g == 1) {
#pragma unroll
          for (int e = 0; e < 32; ++e) oF[(m0 + e) * kD] = v[e];
        } else {
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<float4 *>(oF + m0 + 4 * c) = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
        }
      }
      if (oI) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          __nv_bfloat16 h, l;
          split_bf16(v[e], h, l);
          const uint32_t off = mn_off(m0 + e, n);  // row m, column n
          *reinterpret_cast<__nv_bfloat16 *>(oI + off) = h;
          *reinterpret_cast<__nv_bfloat16 *>(oI + kImgHalf + off) = l;
        }
      }
    };

    // First-step operands of a chain starting at step i: E_M = Diag(alpha),
    // E_J = B (each published as soon as it is written)
    auto first_m = [&](long long i) {
      if (!wait_alpha(i)) return false;
      const float a_n = reinterpret_cast<const float *>(smem + kOffAl + (i & 1) * kAlphaBytes)[n];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float v[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = (64 * ch + 32 * j + e == n) ? a_n : 0.f;
        put_operand(0, j, v);
      }
      mbar_arrive(afree + 8 * (i & 1));
      publish(0);
      return true;
    };
    auto first_j = [&](long long i) {
      if (!wait_b(i)) return false;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float v[32];
        load_b_row32(bbuf, 2 * ch + j, n, v);
        put_operand(1, j, v);
      }
      mbar_arrive(bfree + 8 * ch);
      publish(1);
      return true;
    };

    long long gs = 0;
    bool ok = true;
    for (long long q = blockIdx.x; ok && q < p.nchains; q += gridDim.x) {
      const Chain ch_ = decode(p, q);
      const long long cidx = ch_.bh * p.C + ch_.c;
      float *outM = ch_.dir == 0 ? p.Mf : p.Mb, *outJ = ch_.dir == 0 ? p.Jf : p.Jb;
      if (outM) outM += cidx * DD + (long long)n * kD;
      if (outJ) outJ += cidx * DD + (p.jt ? (long long)n : (long long)n * kD);
      uint8_t *outI = p.Mimg ? p.Mimg + ((ch_.bh * 2 + ch_.dir) * p.C + ch_.c) * (long long)kImgBytes : nullptr;
      if (ch_.nsteps == 0) {
        // every frame of the chunk is an anchor: the identity map
#pragma unroll 1
        for (int j = 0; j < 2; ++j) {
          float v[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = (64 * ch + 32 * j + e == n) ? 1.f : 0.f;
          write_out(0, j, v, outM, outI);
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = 0.f;
          write_out(1, j, v, outJ, nullptr);
        }
        continue;
      }
      // ---- operands of the chain's first step
      if (!first_m(gs) || !first_j(gs)) {
        ok = false;
        break;
      }
      for (int s = 0; s < ch_.nsteps; ++s, ++gs) {
        const bool last = s + 1 == ch_.nsteps;
        if (!last && !wait_alpha(gs + 1)) {
          ok = false;
          break;
        }
        for (int g = 0; g < 2; ++g) {
          if (g == 1 && !last && !wait_b(gs + 1)) {
            ok = false;
            break;
          }
          if (!__all_sync(0xffffffffu, mbar_wait(done + 8 * g, (uint32_t)(gs & 1), abort))) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (!last) {
            // E = D Diag(alpha) (+ B) for the next step
            const float *al = alpha_slot(gs + 1);
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              float v[32], b[32];
              tmem_ld32(tD(g) + 32 * j, v);
              if (g == 1) load_b_row32(bbuf, 2 * ch + j, n, b);
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                const float4 a4 = *reinterpret_cast<const float4 *>(al + 32 * j + 4 * c);
                const float2 b01 = g == 1 ? make_float2(b[4 * c], b[4 * c + 1]) : make_float2(0.f, 0.f);
                const float2 b23 = g == 1 ? make_float2(b[4 * c + 2], b[4 * c + 3]) : make_float2(0.f, 0.f);
                const float2 r01 = __ffma2_rn(make_float2(v[4 * c], v[4 * c + 1]), make_float2(a4.x, a4.y), b01);
                const float2 r23 =
                    __ffma2_rn(make_float2(v[4 * c + 2], v[4 * c + 3]), make_float2(a4.z, a4.w), b23);
                v[4 * c] = r01.x;
                v[4 * c + 1] = r01.y;
                v[4 * c + 2] = r23.x;
                v[4 * c + 3] = r23.y;
              }
              put_operand(g, j, v);
            }
            if (g == 1) {
              mbar_arrive(bfree + 8 * ch);
              mbar_arrive(afree + 8 * ((gs + 1) & 1));
            }
            publish(g);
          } else {
            // the chain's result: Mc (fp32 rows and/or its image) or Jc
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              float v[32];
              tmem_ld32(tD(g) + 32 * j, v);
              if (g == 0)
                write_out(0, j, v, outM, outI);
              else
                write_out(1, j, v, outJ, nullptr);
            }
            // the accumulator is read; the next chain's first operand follows
            tc_fence_before();
          }
        }
        if (!ok) break;
      }
    }
    if (!ok) fail(abort, p.info);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// 3-D tensor map over B_t ([frames][128 rows][128 columns] fp32) with a
// (32 columns x 128 rows x 1) box and the 128-byte swizzle.
bool make_b_map(CUtensorMap *m, const float *Bm, long long frames) {
  auto enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)kD, (cuuint64_t)frames};
  cuuint64_t strides[2] = {(cuuint64_t)kD * 4, (cuuint64_t)kD * kD * 4};
  cuuint32_t box[3] = {32, (cuuint32_t)kD, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float *>(Bm), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_compose_tc(const uint8_t *Wimg, const float *Bm, const float *alpha, float *Mf,
                              float *Jf, float *Mb, float *Jb, uint8_t *Mimg, long long BH, int T,
                              int chunk, int anchors, int ndirs, bool j_transposed, int32_t *info,
                              cudaStream_t st) {
  if (BH <= 0 || T <= 0) return cudaSuccess;
  CUtensorMap tmB;
  if (!make_b_map(&tmB, Bm, BH * T)) return cudaErrorInvalidValue;
  ComposeArgs a{};
  a.Wimg = Wimg;
  a.alpha = alpha;
  a.Mf = Mf;
  a.Jf = Jf;
  a.Mb = Mb;
  a.Jb = Jb;
  a.Mimg = Mimg;
  a.info = info;
  a.BH = BH;
  a.T = T;
  a.chunk = chunk;
  a.C = (T + chunk - 1) / chunk;
  a.anchors = anchors;
  a.ndirs = ndirs;
  a.jt = j_transposed ? 1 : 0;
  // chain index: direction fastest, then b*h, then chunk, so the two
  // directions of a chunk (which read the same W and B) run side by side
  a.nchains = (long long)ndirs * BH * a.C;
  cudaError_t e =
      cudaFuncSetAttribute(compose_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const long long sms = device_sm_count();
  const long long grid = a.nchains < sms ? a.nchains : sms;
  compose_tc_kernel<<<(unsigned)grid, kThreads, kSmemBytes, st>>>(tmB, a);
  return cudaGetLastError();
}

}  // namespace vdn
