// W_t = (I + A_t)^{-1} for every frame (d = 128), as a 2 x 2 block inverse
// whose last three 64 x 64 x 64 products run on the tensor cores.
// Paper: "Video DeltaNet: A Video-Native Hybrid Attention for Livestream
// Video Generation" (summary page), "Core method" (the closed form
// S_t = (Sbar_t + B_t)(I + A_t)^{-1}) and "Method steps" step (3) (factor
// I + A_t per frame, independent of the state, all frames in parallel).
//
// With G = I + A = [[P, Q], [Q^T, R]] (64 x 64 blocks, G symmetric positive
// definite) the Schur complement S = R - Q^T P^{-1} Q is positive definite too
// and, with X = P^{-1} Q and Y = X S^{-1},
//   G^{-1} = [[P^{-1} + Y X^T, -Y], [-Y^T, S^{-1}]].
// P^{-1}, X^T and S arrive in fp32 from the step in schur.cuh (run beside the
// Gram stream, or by schur_prep_kernel below). This kernel sweeps S on the
// CUDA cores (symmetric sweep) and runs Y = X S^{-1}, Y^T = S^{-1} X^T and
// Y X^T as tcgen05 MMAs (M = 128, N = 64, K = 64) on bf16 hi/lo splits
// (hi*hi + hi*lo + lo*hi, ~2^-17 of each operand: these results are at most 2
// in norm and involve no cancellation), accumulating in TMEM. A pivot of S
// that is not positive (G not positive definite) is reported in *info like
// the sweep does.
//
// One CTA of 128 threads works through frames (persistent), four CTAs per SM:
//   warps 0-1 (sweep): load S, sweep it, write the S^{-1} tile -> (SiReady)
//   warps 2-3 (epilogue, TMEM lanes 64-127; thread 64 issues the MMAs):
//            X^T tile from the fp32 rows -> [SiReady] -> Y, Y^T -> Y X^T ->
//            the image's four blocks -> (SiFree)
// The sweep of frame f + 1 runs while the epilogue finishes frame f; only
// the S^{-1} tile's slot is handed back and forth (named barriers).
// Every product keeps its 64 useful rows in lanes 64-127: the A operand's
// descriptor starts 64 rows (8 KB) before the useful rows, so lanes 0-63
// compute throw-away rows from whatever shared memory lies there.
#include "common.cuh"
#include "internal.h"
#include "schur.cuh"
#include "sweep.cuh"

namespace vdn {
namespace {

constexpr int kThreads = 128;
constexpr int kCtasPerSm = 4;          // x 128 TMEM columns <= 512
constexpr int kHalf = 64 * 128;         // one 64 x 64 bf16 tile, 128-byte rows: 8 KB
constexpr int kTile = 2 * kHalf;        // hi + lo: 16 KB
// shared memory slots (offsets from the 1024-aligned base)
constexpr int kSlotTL = 0;              // top-left block of the image
constexpr int kSlotS0 = kTile;          // S^{-1} tile -> -Y tile
constexpr int kSlotXT = 2 * kTile;      // X^T tile -> bottom-left block of the image
constexpr int kSlotMisc = 3 * kTile;    // sweep exchange buffer, barrier, TMEM address, abort flag
constexpr size_t kSmemBytes = 1024 + kSlotMisc + 2 * 2 * 64 * 4 + 64;
constexpr uint32_t kTmemCols = 128;     // two 64-column accumulators
constexpr uint32_t kIdescAmn = idesc_bf16_f32(128, 64, true, false);  // A MN-major
constexpr uint32_t kIdescBmn = idesc_bf16_f32(128, 64, false, true);  // B MN-major

// physical 16-byte chunk of logical chunk c in row r (both tile and image layouts)
__device__ __forceinline__ uint32_t chunk_pos(int r, int c) { return (uint32_t)((c ^ (r & 7)) << 4); }

// hi and lo 16-byte chunks of 8 values (times sign)
__device__ __forceinline__ void pack8(const float *v, float sign, uint4 &h, uint4 &l) {
  split_bf16x2(sign * v[0], sign * v[1], h.x, l.x);
  split_bf16x2(sign * v[2], sign * v[3], h.y, l.y);
  split_bf16x2(sign * v[4], sign * v[5], h.z, l.z);
  split_bf16x2(sign * v[6], sign * v[7], h.w, l.w);
}

// Row r of a hi/lo tile (64 values) written from one thread.
__device__ __forceinline__ void tile_row_store(uint8_t *tile, int r, const float *v, float sign) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint4 h, l;
    pack8(v + 8 * c, sign, h, l);
    const uint32_t o = (uint32_t)r * 128u + chunk_pos(r, c);
    *reinterpret_cast<uint4 *>(tile + o) = h;
    *reinterpret_cast<uint4 *>(tile + kHalf + o) = l;
  }
}

// the 12 MMAs (3 hi/lo parts x 4 k-steps) of one 64-deep product
__device__ __forceinline__ void mma_hilo(uint32_t d, uint32_t a_hi, uint32_t a_lo, uint32_t b_hi,
                                         uint32_t b_lo, bool a_mn, bool b_mn, uint32_t a_lbo,
                                         uint32_t idesc) {
#pragma unroll
  for (int part = 0; part < 3; ++part) {
    const uint32_t a = part == 2 ? a_lo : a_hi;
    const uint32_t b = part == 1 ? b_lo : b_hi;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      // K-major: 16 bf16 = 32 B inside the swizzle row; MN-major: 16 rows of 128 B
      const uint64_t ad = smem_desc_sw128(a + (a_mn ? ks * 2048 : ks * 32), a_mn ? a_lbo : 16, 1024);
      const uint64_t bd = smem_desc_sw128(b + (b_mn ? ks * 2048 : ks * 32), b_mn ? kTile : 16, 1024);
      tc_mma_bf16(d, ad, bd, idesc, (part > 0 || ks > 0) ? 1u : 0u);
    }
  }
}

__device__ __forceinline__ void bar_named(int id) {
  asm volatile("bar.sync %0, 64;" ::"r"(id) : "memory");
}
// hand-offs between the sweep warps and the epilogue warps (128 threads:
// the producers arrive, the consumers wait)
__device__ __forceinline__ void handoff_arrive(int id) {
  __threadfence_block();
  asm volatile("bar.arrive %0, 128;" ::"r"(id) : "memory");
}
__device__ __forceinline__ void handoff_wait(int id) {
  asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory");
}
constexpr int kBarSweep = 1, kBarEpi = 2;  // within each warp pair
constexpr int kBarSiReady = 3, kBarSiFree = 4;

// v = row r of a bf16 hi/lo tile, decoded to fp32
__device__ __forceinline__ void tile_row_load(const uint8_t *tile, int r, float (&v)[64]) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint32_t o = (uint32_t)r * 128u + chunk_pos(r, c);
    const uint4 h = *reinterpret_cast<const uint4 *>(tile + o);
    const uint4 l = *reinterpret_cast<const uint4 *>(tile + kHalf + o);
    const uint32_t hw[4] = {h.x, h.y, h.z, h.w}, lw[4] = {l.x, l.y, l.z, l.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      v[8 * c + 2 * q] = __uint_as_float(hw[q] << 16) + __uint_as_float(lw[q] << 16);
      v[8 * c + 2 * q + 1] = __uint_as_float(hw[q] & 0xFFFF0000u) + __uint_as_float(lw[q] & 0xFFFF0000u);
    }
  }
}

// v (+)= row r of a 64 x 64 fp32 block in schur.cuh's permuted-chunk layout
__device__ __forceinline__ void block_row_load(const float *blk, int r, float (&v)[64], bool add) {
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const float4 x = __ldg(reinterpret_cast<const float4 *>(blk + r * 64 + ((c ^ (r & 15)) << 2)));
    v[4 * c] = add ? v[4 * c] + x.x : x.x;
    v[4 * c + 1] = add ? v[4 * c + 1] + x.y : x.y;
    v[4 * c + 2] = add ? v[4 * c + 2] + x.z : x.z;
    v[4 * c + 3] = add ? v[4 * c + 3] + x.w : x.w;
  }
}

// Row r, columns 64 * region .. + 63 of a row-major fp32 128 x 128 matrix.
__device__ __forceinline__ void w_row_store(float *W, int region, int r, const float *v, float sign) {
  float *dst = W + r * 128 + region * 64;
#pragma unroll
  for (int c = 0; c < 16; ++c)
    *reinterpret_cast<float4 *>(dst + 4 * c) =
        make_float4(sign * v[4 * c], sign * v[4 * c + 1], sign * v[4 * c + 2], sign * v[4 * c + 3]);
}

// 64 TMEM columns of this thread's lane
__device__ __forceinline__ void tmem_row64(uint32_t taddr, float (&v)[64]) {
  tmem_ld32(taddr, *reinterpret_cast<float(*)[32]>(&v[0]));
  tmem_ld32(taddr + 32, *reinterpret_cast<float(*)[32]>(&v[32]));
}

__device__ __forceinline__ void fail(volatile int *abort, int32_t *info) {
  *abort = 1;
  if (info) atomicExch(info, VDN_INFO_TIMEOUT);
}

// P^{-1}, X^T and S of every frame (schur.cuh) from a full A, one CTA of 64
// threads per frame: for Grams computed without the sweep pairs (per-token
// gates, no tokens, CUDA-core Grams).
__global__ void __launch_bounds__(kSweepThreads) schur_prep_kernel(float *__restrict__ A, float *__restrict__ Pinv,
                                                                   int32_t *__restrict__ info, long long frame_base) {
  __shared__ __align__(16) float bp[64 * 64];
  __shared__ __align__(16) float qs[64 * 64];
  __shared__ __align__(16) float cbuf[2][64];
  const long long f = blockIdx.x;
  const int tid = threadIdx.x, rg = tid / kSweepGrid, cg = tid % kSweepGrid;
  float *Af = A + f * 128LL * 128;
  Sweep<64> X;
  // P = I + A[0..63][0..63]; rows 0..63 of A then receive X^T and S
#pragma unroll
  for (int a = 0; a < Sweep<64>::R; ++a)
#pragma unroll
    for (int b = 0; b <= a; ++b) {
      const int r = rg + kSweepGrid * a, c = cg + kSweepGrid * b;
      X.at(a, b) = Af[r * 128 + c] + (r == c ? 1.f : 0.f);
    }
  // Q^T (rows 64..127, columns 0..63) into shared memory
#pragma unroll
  for (int it = 0; it < 16; ++it) {
    const int r = it * 4 + (tid >> 4), c4 = tid & 15;
    *reinterpret_cast<float4 *>(qs + swz64(r, 4 * c4)) =
        *reinterpret_cast<const float4 *>(Af + (64 + r) * 128 + 4 * c4);
  }
  auto sync = [] { __syncthreads(); };
  const bool ok = X.run(cbuf, rg, cg, sync);  // its barriers also publish qs
  if (!ok && tid == 0) report_frame_failure(info, frame_base + f);
  schur_prep(X, qs, Af + 64 * 128 + 64, bp, Pinv + f * 64LL * 64, Af + kSchurXT, Af + kSchurS, tid, sync);
  if (tid == 0) bulk_wait_all();
}

__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    invert_tc_kernel(const float *__restrict__ A, const float *__restrict__ Pinv, float *__restrict__ W,
                     uint8_t *__restrict__ Wimg, int32_t *__restrict__ info, long long nframes,
                     long long frame_base) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *tl_t = sm + kSlotTL, *s0 = sm + kSlotS0, *xt = sm + kSlotXT;
  float(*cbuf)[64] = reinterpret_cast<float(*)[64]>(sm + kSlotMisc);  // sweep exchange buffer
  uint64_t *bar = reinterpret_cast<uint64_t *>(sm + kSlotMisc + 1024);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kSlotMisc + 1032);
  volatile int *abort = reinterpret_cast<volatile int *>(sm + kSlotMisc + 1036);
  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t mbar = smem_u32(bar);
  if (tid == 0) {
    mbar_init(mbar, 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t acc0 = *tmem_slot, acc1 = acc0 + 64;

  if (tid < 64) {
    const int rg = tid / kSweepGrid, cg = tid % kSweepGrid;
    bool first = true;
    for (long long f = blockIdx.x; f < nframes; f += gridDim.x) {
      const float *Sf = A + f * 128LL * 128 + kSchurS;
      Sweep<64> X;
#pragma unroll
      for (int a = 0; a < Sweep<64>::R; ++a)
#pragma unroll
        for (int b = 0; b <= a; ++b) X.at(a, b) = __ldg(Sf + (a * (a + 1) / 2 + b) * 64 + tid);
      const bool ok = X.run(cbuf, rg, cg, [] { bar_named(kBarSweep); });
      // the epilogue is done with the previous frame's S^{-1} and -Y tiles
      if (!first) handoff_wait(kBarSiFree);
      first = false;
      store_swept_tile(X, s0, rg, cg);
      fence_proxy_async_smem();
      handoff_arrive(kBarSiReady);
      if (!ok && tid == 0) report_frame_failure(info, frame_base + f);
    }
  } else {
    const int i = tid - 64;  // TMEM lane 64 + i, row i of every product
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t a_tl = smem_u32(tl_t), a_s0 = smem_u32(s0), a_xt = smem_u32(xt);
    uint32_t nwait = 0;
    auto wait_mma = [&]() {
      if (!mbar_wait(mbar, nwait & 1, abort)) fail(abort, info);
      ++nwait;
      tc_fence_after();
    };
    auto issue = [&](auto body) {  // thread 64, once the operands are visible to the tensor cores
      if (tid == 64 && !*abort) {
        tc_fence_after();
        body();
        tc_commit(mbar);
      }
    };
    for (long long f = blockIdx.x; f < nframes; f += gridDim.x) {
      const float *Af = A + f * 128LL * 128;
      const float *Pf = Pinv + f * 64LL * 64;
      uint8_t *img = Wimg ? Wimg + f * (long long)kImgBytes : nullptr;
      float *Wf = W ? W + f * 128LL * 128 : nullptr;
      // the X^T tile from its fp32 rows (the previous frame's output copies
      // have read the slot)
      float v[64];
      block_row_load(Af + kSchurXT, i, v, false);
      tile_row_store(xt, i, v, 1.f);
      fence_proxy_async_smem();
      if (i == 0 && f + gridDim.x < nframes) {
        // the next frame's inputs into L2 while this one is finished
        const float *An = Af + gridDim.x * 128LL * 128;
        bulk_prefetch_l2(An + kSchurXT, kSchurBytes);
        bulk_prefetch_l2(An + kSchurS, kSchurSPerThread * 64 * 4);
        bulk_prefetch_l2(Pf + gridDim.x * 64LL * 64, kSchurBytes);
      }
      handoff_wait(kBarSiReady);  // the S^{-1} tile is written; so is every row of X^T
      issue([&] {
        // Y = X S^{-1}: A = X, the X^T tile read MN-major as the second 64-row
        // block (lanes 64-127) of a descriptor that starts one tile earlier
        mma_hilo(acc0, a_xt - kTile, a_xt + kHalf - kTile, a_s0, a_s0 + kHalf, true, false, kTile, kIdescAmn);
        // Y^T = S^{-1} X^T: B = X^T read MN-major
        mma_hilo(acc1, a_s0 - kHalf, a_s0, a_xt, a_xt + kHalf, false, true, 16, kIdescBmn);
      });
      wait_mma();
      tmem_row64(acc0 + lane_off, v);  // row i of Y
      if (Wf) {
        w_row_store(Wf, 1, i, v, -1.f);  // top-right block: -Y
        float u[64];
        tile_row_load(s0, i, u);
        w_row_store(Wf, 1, 64 + i, u, 1.f);  // bottom-right block: S^{-1}
      }
      // The image is written as four 64 x 64 blocks by bulk copies of the
      // tiles (rows 64 + i of an image region have the swizzle of rows i of a
      // tile). Bottom-right: the S^{-1} tile as it stands.
      if (img && i == 0) {
        bulk_store(img + kImgRegion + 64 * 128, a_s0, kHalf);
        bulk_store(img + kImgHalf + kImgRegion + 64 * 128, a_s0 + kHalf, kHalf);
        bulk_commit();
        bulk_wait_read<0>();
      }
      bar_named(kBarEpi);  // the S^{-1} tile has been read; it becomes -Y
      tile_row_store(s0, i, v, -1.f);  // -Y: the top-right block and A of the last product
      fence_proxy_async_smem();
      tc_fence_before();
      bar_named(kBarEpi);
      // (-Y) X^T; the top-right block is copied out alongside
      issue([&] { mma_hilo(acc0, a_s0 - kHalf, a_s0, a_xt, a_xt + kHalf, false, true, 16, kIdescBmn); });
      if (img && i == 0) {
        bulk_store(img + kImgRegion, a_s0, kHalf);
        bulk_store(img + kImgHalf + kImgRegion, a_s0 + kHalf, kHalf);
        bulk_commit();
      }
      wait_mma();
      tmem_row64(acc0 + lane_off, v);
      // top-left block: P^{-1} - (-Y) X^T
#pragma unroll
      for (int e = 0; e < 64; ++e) v[e] = -v[e];
      block_row_load(Pf, i, v, true);
      tile_row_store(tl_t, i, v, 1.f);
      if (Wf) w_row_store(Wf, 0, i, v, 1.f);
      // bottom-left block: -Y^T, into the X^T tile (the last product is done)
      tmem_row64(acc1 + lane_off, v);
      tile_row_store(xt, i, v, -1.f);
      if (Wf) w_row_store(Wf, 0, 64 + i, v, -1.f);
      fence_proxy_async_smem();
      bar_named(kBarEpi);
      if (img && i == 0) {
        bulk_store(img, a_tl, kHalf);
        bulk_store(img + kImgHalf, a_tl + kHalf, kHalf);
        bulk_store(img + 64 * 128, a_xt, kHalf);
        bulk_store(img + kImgHalf + 64 * 128, a_xt + kHalf, kHalf);
        bulk_commit();
        bulk_wait_read<0>();  // the top-left, X^T and -Y tiles may be reused
      }
      bar_named(kBarEpi);
      // the sweep warps may now write the next frame's S^{-1} tile
      if (f + gridDim.x < nframes) handoff_arrive(kBarSiFree);
      tc_fence_before();
    }
  }
  if (tid == 64) bulk_wait_all();  // the image's bulk copies have landed
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(acc0, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_invert_tc(const float *A, const float *Pinv, float *W, uint8_t *Wimg, int32_t *info,
                             long long nframes, cudaStream_t st, long long frame_base) {
  if (nframes <= 0) return cudaSuccess;
  if (!A || !Pinv) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(invert_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const long long cap = (long long)kCtasPerSm * device_sm_count();
  const long long grid = nframes < cap ? nframes : cap;
  invert_tc_kernel<<<(unsigned)grid, kThreads, kSmemBytes, st>>>(A, Pinv, W, Wimg, info, nframes, frame_base);
  return cudaGetLastError();
}

cudaError_t launch_schur_prep(float *A, float *Pinv, int32_t *info, long long nframes, cudaStream_t st,
                              long long frame_base) {
  if (nframes <= 0) return cudaSuccess;
  schur_prep_kernel<<<(unsigned)nframes, kSweepThreads, 0, st>>>(A, Pinv, info, frame_base);
  return cudaGetLastError();
}

}  // namespace vdn
