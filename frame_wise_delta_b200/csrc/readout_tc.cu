// Chunk readout on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
// Paper: "Video DeltaNet: A Video-Native Hybrid Attention for Livestream
// Video Generation" (summary page), "Core method" (each query chunk reads the
// forward state before its 15-frame window plus the backward state after it)
// and "Method steps" step (5):
//   R_c = F[max(c-1,0)] + G[min(c+2,C)],   o_{t,u} = R_c q_{t,u}.
//
// D = Q_tile R^T with M = 128 tokens, N = 128 (value channel i), K = 128 key
// channels. The fp32 state R is split into bf16 hi + lo parts (R = hi + lo to
// ~2^-17 relative) and both products accumulate into one fp32 TMEM tile, so
// the readout keeps fp32-state accuracy while Q is read once, as bf16.
// Operands are K-major and 128-byte swizzled: Q tiles come from TMA, R is
// written by the CTA into the same layout.
//
// Optional epilogue ("Method steps" step (5): RMSNorm, then a sigmoid gate):
// y = o / sqrt(mean o^2 + eps) * w[h] * sigmoid(g) per token, in two passes
// over the token's TMEM row (mean square, then scale), with the tile's gate
// logits brought by TMA into the staging tile that then receives y.
//
// Decay bridge (optional, step (5)): frame t reads
//   R_t = F[max(c-1,0)] Diag(pf_t) + G[min(c+2,C)] Diag(pb_t),
// pf_t and pb_t the products of the decay gates over the window's frames
// f0..t and t..f1; R is then rebuilt for every frame. In a stream segment
// (F0 given) chunk 0's window starts in the previous segment's last chunk,
// whose decay product (bprev) joins pf.
//
// Persistent kernel, one CTA per SM, 10 warps; each CTA walks a contiguous
// range of frames so consecutive frames usually share a chunk and R is
// rebuilt only when the chunk changes.
//   warp 0     : TMA producer (two 16 KB loads per 128-token stage)
//   warp 1     : TMEM allocator and single-thread MMA issuer
//   warps 2..9 : R builder and epilogue in two groups of four warps that take
//                alternate tiles (TMEM -> bf16 tile in the group's staging
//                buffer in shared memory -> TMA store); anchor frames
//                are written as zeros without touching the tensor cores)
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"

namespace vdn {
namespace {

constexpr int kD = 128;
constexpr int kNT = 128;                      // tokens per tile (MMA N)
constexpr int kStages = 3;
constexpr int kStageBytes = kNT * 128 * 2;    // two 64-channel regions
constexpr int kRegionQ = kNT * 128;           // 16 KB
constexpr int kRBytes = kD * 128 * 2;         // one bf16 R operand, 2 regions
constexpr int kRegionR = kD * 128;
constexpr int kOBytes = kNT * 128 * 2;        // one bf16 O tile, two 64-channel regions
constexpr int kRegionO = kNT * 128;
constexpr int kAcc = 4;                       // TMEM accumulators (128 columns each)
constexpr int kThreads = 320;
constexpr uint32_t kTmemCols = 512;
constexpr int kBarBytes = 8 * (2 * kStages + 2 * kAcc + 2 + 2);
constexpr size_t kSmemBytes =
    1024 + (size_t)kStages * kStageBytes + 2 * kRBytes + 2 * kOBytes + kBarBytes + 16 + 2 * kD * 4;

struct ReadoutArgs {
  const float *F;
  const float *G;   // optional (forward reads only when null)
  const float *F0;  // optional: per-b*h forward state chunk 0 reads instead of F[0]
  const float *bal; // optional: decay gates alpha [BH, T, 128]: read through the decay bridge
  const float *bprev; // optional [BH, 128]: extra decay of chunk 0's forward factor (with F0)
  __nv_bfloat16 *O;
  int32_t *info;
  long long nframes;
  int T, U, chunk, anchors, C, ntiles;
  // gated RMSNorm epilogue (step (5))
  const float *gw;  // [H, 128] RMSNorm weights, nullptr = no epilogue (gate logits through tmG)
  float eps;
  int H;
};

__device__ __forceinline__ void fail(volatile int *abort, int32_t *info) {
  *abort = 1;
  if (info) atomicExch(info, VDN_INFO_TIMEOUT);
}

__device__ __forceinline__ bool is_anchor(const ReadoutArgs &p, long long f) {
  const int t = (int)(f % p.T);
  return ((p.anchors & 1) && t == 0) || ((p.anchors & 2) && t == p.T - 1);
}

// R changes with the chunk, or with every frame through the decay bridge
__device__ __forceinline__ long long chunk_key(const ReadoutArgs &p, long long f) {
  return p.bal ? f : (f / p.T) * p.C + (f % p.T) / p.chunk;
}

// tanh by the hardware approximation (PTX tanh.approx.f32, ~2^-11 relative)
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);  // a in the low half
  return *reinterpret_cast<const uint32_t *>(&h);
}

__global__ void __launch_bounds__(kThreads, 1)
    readout_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
                      const __grid_constant__ CUtensorMap tmG, ReadoutArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  uint8_t *stages = smem;
  uint8_t *Rhi = smem + kStages * kStageBytes;
  uint8_t *Rlo = Rhi + kRBytes;
  uint8_t *Obuf = Rlo + kRBytes;  // two O staging tiles
  uint64_t *bars = reinterpret_cast<uint64_t *>(Obuf + 2 * kOBytes);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(reinterpret_cast<uint8_t *>(bars) + kBarBytes);
  volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
  float *bridge_fb = reinterpret_cast<float *>(tmem_slot + 4);  // [2][128]: pf, pb of the frame being read

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8 * kStages;
  const uint32_t tfull0 = empty0 + 8 * kStages;
  const uint32_t tempty0 = tfull0 + 8 * kAcc;
  const uint32_t rfull = tempty0 + 8 * kAcc;
  const uint32_t drain = rfull + 8;
  const uint32_t gfull0 = drain + 8;  // a group's gate tile has landed in its staging tile

  // contiguous, balanced frame range of this CTA
  const long long f_begin = p.nframes * blockIdx.x / gridDim.x;
  const long long f_end = p.nframes * (blockIdx.x + 1) / gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < kAcc; ++b) {
      mbar_init(tfull0 + 8 * b, 1);
      mbar_init(tempty0 + 8 * b, 128);
    }
    mbar_init(rfull, 1);
    mbar_init(drain, 1);
    mbar_init(gfull0, 1);
    mbar_init(gfull0 + 8, 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      int stage = 0;
      uint32_t phase = 0;
      int armed_parity[kStages];
      for (int s = 0; s < kStages; ++s) armed_parity[s] = -1;
      bool ok = true;
      for (long long f = f_begin; ok && f < f_end; ++f) {
        if (is_anchor(p, f)) continue;
        for (int j = 0; j < p.ntiles; ++j) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1, abort)) {
            fail(abort, p.info);
            ok = false;
            break;
          }
          const uint32_t dst = smem_u32(stages + stage * kStageBytes);
          const uint32_t fb = full0 + 8 * stage;
          mbar_arrive_expect_tx(fb, kStageBytes);
          armed_parity[stage] = (int)phase;
          tma_load_3d(dst, &tmQ, fb, 0, j * kNT, (int)f);
          tma_load_3d(dst + kRegionQ, &tmQ, fb, 64, j * kNT, (int)f);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      volatile int never = 0;
      for (int s = 0; s < kStages; ++s)
        if (armed_parity[s] >= 0) mbar_wait(full0 + 8 * s, (uint32_t)armed_parity[s], &never);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, kNT, false, false);
      const uint32_t rhi = smem_u32(Rhi), rlo = smem_u32(Rlo);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t tile = 0;
      uint32_t rbuilds = 0;
      long long cur = -1;
      bool ok = true;
      for (long long f = f_begin; ok && f < f_end; ++f) {
        if (is_anchor(p, f)) continue;
        const long long key = chunk_key(p, f);
        if (key != cur) {
          if (!mbar_wait(rfull, rbuilds & 1, abort)) {
            fail(abort, p.info);
            break;
          }
          ++rbuilds;
          cur = key;
          tc_fence_after();
        }
        for (int j = 0; j < p.ntiles; ++j, ++tile) {
          const int buf = (int)(tile % kAcc);
          const uint32_t use = tile / kAcc;
          if (!mbar_wait(tempty0 + 8 * buf, (use & 1) ^ 1, abort) ||
              !mbar_wait(full0 + 8 * stage, phase, abort)) {
            fail(abort, p.info);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t q = smem_u32(stages + stage * kStageBytes);
          const uint32_t dcol = tmem_base + (uint32_t)(buf * kNT);
#pragma unroll
          for (int part = 0; part < 2; ++part) {
            const uint32_t r = part == 0 ? rhi : rlo;
#pragma unroll
            for (int ks = 0; ks < kD / 16; ++ks) {
              const uint32_t koff = (uint32_t)(ks & 3) * 32;  // 16 bf16 = 32 B inside the swizzle atom
              const uint64_t adesc = smem_desc_sw128(q + (ks >> 2) * kRegionQ + koff, 16, 1024);
              const uint64_t bdesc = smem_desc_sw128(r + (ks >> 2) * kRegionR + koff, 16, 1024);
              tc_mma_bf16(dcol, adesc, bdesc, idesc, (part > 0 || ks > 0) ? 1u : 0u);
            }
          }
          tc_commit(empty0 + 8 * stage);
          tc_commit(tfull0 + 8 * buf);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      tc_commit(drain);
      volatile int never = 0;
      mbar_wait(drain, 0, &never);
    }
  } else {
    const int et = threadIdx.x - 64;       // 0..255 over both groups
    const int grp = (warp - 2) >> 2;        // tiles with (tile & 1) == grp
    const int gt = et & 127;                // thread of the group
    const int sub = warp & 3;               // TMEM sub-partition
    const int row = sub * 32 + lane;        // token of the tile held by this thread (TMEM lane)
    const int gbar = 1 + grp;               // the group's named barrier
    uint8_t *ob = Obuf + grp * kOBytes;     // the group's staging tile
    uint32_t tile = 0;
    long long cur = -1;
    bool ok = true;  // after a failed wait: keep every barrier, skip the work
    const bool gated = p.gw != nullptr;
    const uint32_t gfull = gfull0 + 8 * grp;
    uint32_t guse = 0;      // gate tiles this group has loaded
    bool garmed = false;    // a gate load is armed and not yet waited for
    for (long long f = f_begin; f < f_end; ++f) {
      __nv_bfloat16 *Of = p.O + f * (long long)p.U * kD;
      if (is_anchor(p, f)) {
        uint4 z = make_uint4(0, 0, 0, 0);
        uint4 *o4 = reinterpret_cast<uint4 *>(Of);
        const long long n16 = (long long)p.U * kD / 8;
        for (long long e = et; e < n16; e += 256) o4[e] = z;
        continue;
      }
      const long long key = chunk_key(p, f);
      if (key != cur) {
        // Both groups have drained every tile of the previous chunk (their
        // MMAs, which read the previous R, have completed) once they meet here.
        asm volatile("bar.sync 3, 256;" ::: "memory");
        cur = key;
        const long long bh = f / p.T;
        const int c = (int)((f % p.T) / p.chunk);
        const float *Fs = (c == 0 && p.F0) ? p.F0 + bh * (long long)(kD * kD)
                                           : p.F + (bh * (p.C + 1) + max(c - 1, 0)) * (long long)(kD * kD);
        const float *Gs = p.G ? p.G + (bh * (p.C + 1) + min(c + 2, p.C)) * (long long)(kD * kD) : nullptr;
        // decay bridge: thread et forms the factor of key channel et & 127,
        // forward (pf, the window's frames f0..t) or backward (pb, t..f1),
        // anchor frames counting as 1; the products go through shared memory
        if (p.bal) {
          const int t = (int)(f % p.T), k = et & 127, dir = et >> 7;
          const int lo = dir ? t : p.chunk * max(c - 1, 0);
          const int hi = dir ? min(p.chunk * (c + 2), p.T) - 1 : t;
          const float *al = p.bal + bh * (long long)p.T * kD + k;
          float prod = 1.f;
#pragma unroll 8
          for (int r = lo; r <= hi; ++r) {
            const float x = __ldg(al + (long long)r * kD);
            if (!(((p.anchors & 1) && r == 0) || ((p.anchors & 2) && r == p.T - 1))) prod *= x;
          }
          // a stream segment's chunk 0: its window starts in the previous segment
          if (dir == 0 && c == 0 && p.F0 && p.bprev) prod *= __ldg(p.bprev + bh * kD + k);
          bridge_fb[dir * kD + k] = prod;
          asm volatile("bar.sync 3, 256;" ::: "memory");
        }
        // R (or R_t) as hi/lo bf16 operand images; each thread covers 8 key
        // channels k0.. of 8 rows, the loads of four rows in flight at once
        const int k0 = (et & 15) * 8;
        float pf[8], pb[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          pf[q] = p.bal ? bridge_fb[k0 + q] : 1.f;
          pb[q] = p.bal ? bridge_fb[kD + k0 + q] : 1.f;
        }
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          float4 fa[4][2], ga[4][2];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int i = (et + 256 * (4 * half + j)) >> 4;
            const float4 *f4 = reinterpret_cast<const float4 *>(Fs + i * kD + k0);
            fa[j][0] = __ldg(f4);
            fa[j][1] = __ldg(f4 + 1);
            if (Gs) {
              const float4 *g4 = reinterpret_cast<const float4 *>(Gs + i * kD + k0);
              ga[j][0] = __ldg(g4);
              ga[j][1] = __ldg(g4 + 1);
            } else {
              ga[j][0] = ga[j][1] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int i = (et + 256 * (4 * half + j)) >> 4;
            const float x[8] = {fa[j][0].x, fa[j][0].y, fa[j][0].z, fa[j][0].w,
                                fa[j][1].x, fa[j][1].y, fa[j][1].z, fa[j][1].w};
            const float y[8] = {ga[j][0].x, ga[j][0].y, ga[j][0].z, ga[j][0].w,
                                ga[j][1].x, ga[j][1].y, ga[j][1].z, ga[j][1].w};
            float r[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) r[q] = p.bal ? fmaf(x[q], pf[q], y[q] * pb[q]) : x[q] + y[q];
            uint4 h, l;
            split_bf16x2(r[0], r[1], h.x, l.x);
            split_bf16x2(r[2], r[3], h.y, l.y);
            split_bf16x2(r[4], r[5], h.z, l.z);
            split_bf16x2(r[6], r[7], h.w, l.w);
            const uint32_t off = kmajor_sw128_offset(i, k0, kD);
            *reinterpret_cast<uint4 *>(Rhi + off) = h;
            *reinterpret_cast<uint4 *>(Rlo + off) = l;
          }
        }
        fence_proxy_async_smem();
        asm volatile("bar.sync 3, 256;" ::: "memory");
        if (et == 0) mbar_arrive(rfull);
      }
      for (int j = 0; j < p.ntiles; ++j, ++tile) {
        if ((int)(tile & 1) != grp) continue;
        const int buf = (int)(tile % kAcc);
        const uint32_t use = tile / kAcc;
        // the group's previous TMA store has finished reading the staging tile
        if (gt == 0) bulk_wait_read<0>();
        asm volatile("bar.sync %0, 128;" ::"r"(gbar) : "memory");
        // the tile's gate logits into the staging tile (same layout as O),
        // coalesced by TMA while the MMA and pass 1 run
        if (gated && ok && gt == 0) {
          mbar_arrive_expect_tx(gfull, kOBytes);
          tma_load_3d(smem_u32(ob), &tmG, gfull, 0, j * kNT, (int)f);
          tma_load_3d(smem_u32(ob + kRegionO), &tmG, gfull, 64, j * kNT, (int)f);
          garmed = true;
        }
        if (ok && !__all_sync(0xffffffffu, mbar_wait(tfull0 + 8 * buf, use & 1, abort))) {
          fail(abort, p.info);
          ok = false;
        }
        float rs = 0.f;
        if (ok && gated) {
          tc_fence_after();
          // pass 1: this token's mean square over its 128 channels
          float ss[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
          for (int cc = 0; cc < kD / 32; ++cc) {
            float v[32];
            tmem_ld32(tmem_base + (uint32_t)(buf * kNT + cc * 32) + ((uint32_t)(sub * 32) << 16), v);
#pragma unroll
            for (int e = 0; e < 32; ++e) ss[e & 3] = fmaf(v[e], v[e], ss[e & 3]);
          }
          rs = rsqrtf((ss[0] + ss[1] + ss[2] + ss[3]) * (1.0f / kD) + p.eps);
          const bool gok = __all_sync(0xffffffffu, mbar_wait(gfull, guse & 1, abort));
          ++guse;
          if (gt == 0) garmed = false;
          if (!gok) {
            fail(abort, p.info);
            ok = false;
          }
        }
        if (ok && gated) {
          // pass 2: y = o * rs * w * sigmoid(g), sigmoid(g) = (1 + tanh(g / 2)) / 2
          const float *wv = p.gw + ((f / p.T) % p.H) * kD;
#pragma unroll
          for (int cc = 0; cc < kD / 32; ++cc) {
            float v[32];
            tmem_ld32(tmem_base + (uint32_t)(buf * kNT + cc * 32) + ((uint32_t)(sub * 32) << 16), v);
            uint8_t *rb = ob + (cc >> 1) * kRegionO + row * 128;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int ch = (cc & 1) * 4 + q;
              uint4 *slot = reinterpret_cast<uint4 *>(rb + ((ch ^ (row & 7)) << 4));
              const uint4 g8 = *slot;
              const uint32_t gw4[4] = {g8.x, g8.y, g8.z, g8.w};
              const float4 w0 = *reinterpret_cast<const float4 *>(wv + cc * 32 + 8 * q);
              const float4 w1 = *reinterpret_cast<const float4 *>(wv + cc * 32 + 8 * q + 4);
              const float wq[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
              uint32_t y[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float g0 = __uint_as_float(gw4[e] << 16), g1 = __uint_as_float(gw4[e] & 0xFFFF0000u);
                const float y0 = v[8 * q + 2 * e] * rs * wq[2 * e] * fmaf(0.5f, tanh_approx(0.5f * g0), 0.5f);
                const float y1 = v[8 * q + 2 * e + 1] * rs * wq[2 * e + 1] * fmaf(0.5f, tanh_approx(0.5f * g1), 0.5f);
                y[e] = pack_bf16(y0, y1);
              }
              *slot = make_uint4(y[0], y[1], y[2], y[3]);
            }
          }
          tc_fence_before();
          mbar_arrive(tempty0 + 8 * buf);
        } else if (ok) {
          tc_fence_after();
          // row `row` of the tile: 128 channels -> bf16, 16-byte chunks swizzled
          // as the tensor map's 128-byte swizzle expects
#pragma unroll
          for (int cc = 0; cc < kD / 32; ++cc) {
            float v[32];
            tmem_ld32(tmem_base + (uint32_t)(buf * kNT + cc * 32) + ((uint32_t)(sub * 32) << 16), v);
            uint8_t *rb = ob + (cc >> 1) * kRegionO + row * 128;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int ch = (cc & 1) * 4 + q;
              *reinterpret_cast<uint4 *>(rb + ((ch ^ (row & 7)) << 4)) =
                  make_uint4(pack_bf16(v[8 * q], v[8 * q + 1]), pack_bf16(v[8 * q + 2], v[8 * q + 3]),
                             pack_bf16(v[8 * q + 4], v[8 * q + 5]), pack_bf16(v[8 * q + 6], v[8 * q + 7]));
            }
          }
          tc_fence_before();
          mbar_arrive(tempty0 + 8 * buf);
        }
        fence_proxy_async_smem();
        asm volatile("bar.sync %0, 128;" ::"r"(gbar) : "memory");
        if (ok && gt == 0) {
          // rows past U fall outside the tensor and are not written
          tma_store_3d(&tmO, smem_u32(ob), 0, j * kNT, (int)f);
          tma_store_3d(&tmO, smem_u32(ob + kRegionO), 64, j * kNT, (int)f);
          bulk_commit();
        }
      }
    }
    if (gt == 0) {
      bulk_wait_all();
      // never leave with a gate load in flight (only after a failed wait)
      volatile int never = 0;
      if (garmed) mbar_wait(gfull, guse & 1, &never);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

bool make_rows_map(CUtensorMap *m, const void *base, long long frames, int rows, int box_rows);

bool readout_tc_supported(int in_dtype, int out_dtype, int D, int U) {
  return in_dtype == VDN_BF16 && out_dtype == VDN_BF16 && D == 128 && U > 0;
}

cudaError_t launch_readout_tc(const void *Q, const float *F, const float *G, void *O, long long BH,
                              int T, int U, int chunk, int anchors, int32_t *info, cudaStream_t st,
                              const OutGate *og, const float *F0, const float *bridge_alpha,
                              const float *bridge_prev) {
  const long long nframes = BH * T;
  if (nframes <= 0) return cudaSuccess;
  CUtensorMap tmQ, tmO, tmG;
  const bool gated = og && og->gate;
  if (!make_rows_map(&tmQ, Q, nframes, U, kNT) || !make_rows_map(&tmO, O, nframes, U, kNT) ||
      !make_rows_map(&tmG, gated ? og->gate : Q, nframes, U, kNT))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(readout_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const int sms = device_sm_count();
  const long long grid = nframes < sms ? nframes : sms;
  ReadoutArgs a{F, G, F0, bridge_alpha, bridge_prev, (__nv_bfloat16 *)O, info, nframes, T, U, chunk, anchors,
                (T + chunk - 1) / chunk, (U + kNT - 1) / kNT,
                gated ? og->w : nullptr, gated ? og->eps : 0.f, gated ? og->H : 1};
  readout_tc_kernel<<<(unsigned)grid, kThreads, kSmemBytes, st>>>(tmQ, tmO, tmG, a);
  return cudaGetLastError();
}

}  // namespace vdn
