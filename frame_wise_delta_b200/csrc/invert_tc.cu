// W_t = (I + A_t)^{-1} for every frame (d = 128), as a 2 x 2 block inverse
// whose four 64 x 64 x 64 products run on the tensor cores.
// Paper: "Video DeltaNet: A Video-Native Hybrid Attention for Livestream
// Video Generation" (summary page), "Core method" (the closed form
// S_t = (Sbar_t + B_t)(I + A_t)^{-1}) and "Method steps" step (3) (factor
// I + A_t per frame, independent of the state, all frames in parallel).
//
// With G = I + A = [[P, Q], [Q^T, R]] (64 x 64 blocks, G symmetric positive
// definite) the Schur complement S = R - Q^T P^{-1} Q is positive definite too
// and, with X = P^{-1} Q and Y = X S^{-1},
//   G^{-1} = [[P^{-1} + Y X^T, -Y], [-Y^T, S^{-1}]].
// P^{-1} and S^{-1} come from the symmetric sweep on the CUDA cores (a quarter
// of the full sweep's work); the products X^T = Q^T P^{-1}, Q^T X, Y = X S^{-1},
// Y^T = S^{-1} X^T and Y X^T run as tcgen05 MMAs (M = 128, N = 64, K = 64) on
// hi/lo bf16 splits (hi*hi + hi*lo + lo*hi, ~fp32 accuracy), accumulating in
// TMEM. A pivot of P or S that is not positive (G not positive definite) is
// reported in *info like the sweep does.
//
// One CTA of 128 threads per frame at a time (persistent over frames), four
// CTAs per SM: warps 0-1 run the sweeps, warps 2-3 own TMEM lanes 64-127 and
// do the loads, the epilogues and the output; thread 64 issues the MMAs.
// Every product keeps its 64 useful rows in lanes 64-127: the A operand's
// descriptor starts 64 rows (8 KB) before the useful rows, so lanes 0-63
// compute throw-away rows from whatever shared memory lies there.
#include "common.cuh"
#include "internal.h"
#include "sweep.cuh"

namespace vdn {
namespace {

constexpr int kThreads = 128;
constexpr int kHalf = 64 * 128;         // one 64 x 64 bf16 tile, 128-byte rows: 8 KB
constexpr int kTile = 2 * kHalf;        // hi + lo: 16 KB
// shared memory slots (offsets from the 1024-aligned base)
constexpr int kSlotPi = 0;              // P^{-1} image
constexpr int kSlotS0 = kTile;          // Q^T image -> fp32 Q^T X staging -> S^{-1} image -> Y image
constexpr int kSlotXT = 2 * kTile;      // X^T image
constexpr int kSlotMisc = 3 * kTile;    // sweep exchange buffer, barrier, TMEM address, abort flag
constexpr size_t kSmemBytes = 1024 + kSlotMisc + 2 * 64 * 4 + 64;
constexpr uint32_t kTmemCols = 128;     // two 64-column accumulators
constexpr uint32_t kIdesc = idesc_bf16_f32(128, 64, false, false);    // A, B K-major
constexpr uint32_t kIdescAmn = idesc_bf16_f32(128, 64, true, false);  // A MN-major
constexpr uint32_t kIdescBmn = idesc_bf16_f32(128, 64, false, true);  // B MN-major

// element (row, k) of a 64-row K-major 128-byte-swizzled tile (k < 64)
__device__ __forceinline__ uint32_t tile_off(int row, int k) { return kmajor_sw128_offset(row, k, 64); }

// physical 16-byte chunk of logical chunk c in row r (both tile and image layouts)
__device__ __forceinline__ uint32_t chunk_pos(int r, int c) { return (uint32_t)((c ^ (r & 7)) << 4); }

__device__ __forceinline__ uint4 pack8(const float *v, bool lo) {
  uint32_t w[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    __nv_bfloat16 h0, l0, h1, l1;
    split_bf16(v[2 * q], h0, l0);
    split_bf16(v[2 * q + 1], h1, l1);
    w[q] = lo ? pack2(l0, l1) : pack2(h0, h1);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Row r of a hi/lo tile (64 values) written from one thread.
__device__ __forceinline__ void tile_row_store(uint8_t *tile, int r, const float *v, float sign) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float s[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) s[e] = sign * v[8 * c + e];
    const uint32_t o = (uint32_t)r * 128u + chunk_pos(r, c);
    *reinterpret_cast<uint4 *>(tile + o) = pack8(s, false);
    *reinterpret_cast<uint4 *>(tile + kHalf + o) = pack8(s, true);
  }
}

// Row r, columns 64 * region .. + 63 of a global 128 x 128 hi/lo image.
__device__ __forceinline__ void img_row_store(uint8_t *img, int region, int r, const float *v, float sign) {
  uint8_t *base = img + region * kImgRegion + r * 128;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float s[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) s[e] = sign * v[8 * c + e];
    const uint32_t o = chunk_pos(r, c);
    *reinterpret_cast<uint4 *>(base + o) = pack8(s, false);
    *reinterpret_cast<uint4 *>(base + kImgHalf + o) = pack8(s, true);
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

// v (+)= row r of a hi/lo tile, decoded to fp32
__device__ __forceinline__ void tile_row_add(const uint8_t *tile, int r, float (&v)[64], bool add) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint32_t o = (uint32_t)r * 128u + chunk_pos(r, c);
    const uint4 h = *reinterpret_cast<const uint4 *>(tile + o);
    const uint4 l = *reinterpret_cast<const uint4 *>(tile + kHalf + o);
    const uint32_t hw[4] = {h.x, h.y, h.z, h.w}, lw[4] = {l.x, l.y, l.z, l.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float x0 = __uint_as_float(hw[q] << 16) + __uint_as_float(lw[q] << 16);
      const float x1 = __uint_as_float(hw[q] & 0xFFFF0000u) + __uint_as_float(lw[q] & 0xFFFF0000u);
      v[8 * c + 2 * q] = add ? v[8 * c + 2 * q] + x0 : x0;
      v[8 * c + 2 * q + 1] = add ? v[8 * c + 2 * q + 1] + x1 : x1;
    }
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

// -G^{-1} of a 64 x 64 block from the sweep -> hi/lo tile of G^{-1} (both triangles)
__device__ __forceinline__ void store_swept(Sweep<64> &X, uint8_t *tile, int rg, int cg) {
#pragma unroll
  for (int a = 0; a < Sweep<64>::R; ++a)
#pragma unroll
    for (int b = 0; b <= a; ++b) {
      const int i = rg + kSweepGrid * a, j = cg + kSweepGrid * b;
      __nv_bfloat16 h, l;
      split_bf16(-X.at(a, b), h, l);
      *reinterpret_cast<__nv_bfloat16 *>(tile + tile_off(i, j)) = h;
      *reinterpret_cast<__nv_bfloat16 *>(tile + kHalf + tile_off(i, j)) = l;
      if (a != b) {
        *reinterpret_cast<__nv_bfloat16 *>(tile + tile_off(j, i)) = h;
        *reinterpret_cast<__nv_bfloat16 *>(tile + kHalf + tile_off(j, i)) = l;
      }
    }
}

__global__ void __launch_bounds__(kThreads, 4)
    invert_tc_kernel(const float *__restrict__ A, float *__restrict__ W, uint8_t *__restrict__ Wimg,
                     int32_t *__restrict__ info, long long nframes, long long frame_base) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *pi_t = sm + kSlotPi, *s0 = sm + kSlotS0, *xt = sm + kSlotXT;
  float(*cbuf)[64] = reinterpret_cast<float(*)[64]>(sm + kSlotMisc);
  uint64_t *bar = reinterpret_cast<uint64_t *>(sm + kSlotMisc + 512);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kSlotMisc + 520);
  volatile int *abort = reinterpret_cast<volatile int *>(sm + kSlotMisc + 524);
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
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  const uint32_t a_pi = smem_u32(pi_t), a_s0 = smem_u32(s0), a_xt = smem_u32(xt);
  const int rg = (tid & 63) / kSweepGrid, cg = tid % kSweepGrid;  // sweep grid (warps 0-1)
  const int i = tid - 64;                                         // epilogue row (warps 2-3)
  float *stage = reinterpret_cast<float *>(s0);                   // fp32 Q^T X, swizzled rows
  uint32_t nwait = 0;
  auto wait_mma = [&]() {
    if (!mbar_wait(mbar, nwait & 1, abort)) fail(abort, info);
    ++nwait;
    tc_fence_after();
  };
  auto issue = [&](auto body) {  // thread 64, after the operands are visible to the tensor cores
    if (tid == 64 && !*abort) {
      tc_fence_after();
      body();
      tc_commit(mbar);
    }
  };

  for (long long f = blockIdx.x; f < nframes; f += gridDim.x) {
    const float *Af = A + f * 128LL * 128;
    uint8_t *img = Wimg ? Wimg + f * (long long)kImgBytes : nullptr;
    float *Wf = W ? W + f * 128LL * 128 : nullptr;
    bool ok = true;
    if (tid < 64) {
      // P^{-1} by the sweep
      Sweep<64> X;
#pragma unroll
      for (int a = 0; a < Sweep<64>::R; ++a)
#pragma unroll
        for (int b = 0; b <= a; ++b) {
          const int r = rg + kSweepGrid * a, c = cg + kSweepGrid * b;
          X.at(a, b) = Af[r * 128 + c] + (r == c ? 1.f : 0.f);
        }
      ok = X.run(cbuf, rg, cg, [] { bar_named(1); });
      store_swept(X, pi_t, rg, cg);
    } else {
      // Q^T = G[64 + r][0 .. 63] as a hi/lo tile, read row-contiguously
      const int e = i;
#pragma unroll 4
      for (int it = 0; it < 16; ++it) {
        const int r = it * 4 + (e >> 4), c4 = e & 15;
        const float4 x = __ldg(reinterpret_cast<const float4 *>(Af + (64 + r) * 128 + 4 * c4));
        __nv_bfloat16 h[4], l[4];
        split_bf16(x.x, h[0], l[0]);
        split_bf16(x.y, h[1], l[1]);
        split_bf16(x.z, h[2], l[2]);
        split_bf16(x.w, h[3], l[3]);
        const uint32_t o = tile_off(r, 4 * c4);
        *reinterpret_cast<uint2 *>(s0 + o) = make_uint2(pack2(h[0], h[1]), pack2(h[2], h[3]));
        *reinterpret_cast<uint2 *>(s0 + kHalf + o) = make_uint2(pack2(l[0], l[1]), pack2(l[2], l[3]));
      }
    }
    fence_proxy_async_smem();
    __syncthreads();
    // X^T = Q^T P^{-1}
    issue([&] { mma_hilo(acc0, a_s0 - kHalf, a_s0, a_pi, a_pi + kHalf, false, false, 16, kIdesc); });
    if (tid >= 64) {
      float v[64];
      wait_mma();
      tmem_row64(acc0 + lane_off, v);
      tile_row_store(xt, i, v, 1.f);
      fence_proxy_async_smem();
      tc_fence_before();
      bar_named(2);
      // Q^T X (B = Q read from the Q^T tile K-major)
      issue([&] { mma_hilo(acc0, a_xt - kHalf, a_xt, a_s0, a_s0 + kHalf, false, false, 16, kIdesc); });
      wait_mma();
      tmem_row64(acc0 + lane_off, v);
#pragma unroll
      for (int c = 0; c < 16; ++c)
        *reinterpret_cast<float4 *>(stage + i * 64 + ((c ^ (i & 15)) << 2)) =
            make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
      tc_fence_before();
    }
    __syncthreads();
    if (tid < 64) {
      // S = R - Q^T X and S^{-1} by the sweep; S^{-1} replaces the staging
      // (every thread has read its part before the sweep's first barrier)
      Sweep<64> X;
#pragma unroll
      for (int a = 0; a < Sweep<64>::R; ++a)
#pragma unroll
        for (int b = 0; b <= a; ++b) {
          const int r = rg + kSweepGrid * a, c = cg + kSweepGrid * b;
          X.at(a, b) = Af[(64 + r) * 128 + 64 + c] + (r == c ? 1.f : 0.f) -
                       stage[r * 64 + (((c >> 2) ^ (r & 15)) << 2) + (c & 3)];
        }
      ok = X.run(cbuf, rg, cg, [] { bar_named(1); }) && ok;
      store_swept(X, s0, rg, cg);
      fence_proxy_async_smem();
      if (!ok && tid == 0) report_frame_failure(info, frame_base + f);
    }
    __syncthreads();
    issue([&] {
      // Y = X S^{-1}: A = X, the X^T tile read MN-major as the second 64-row
      // block (lanes 64-127) of a descriptor that starts one tile earlier
      mma_hilo(acc0, a_xt - kTile, a_xt + kHalf - kTile, a_s0, a_s0 + kHalf, true, false, kTile, kIdescAmn);
      // Y^T = S^{-1} X^T: B = X^T read MN-major
      mma_hilo(acc1, a_s0 - kHalf, a_s0, a_xt, a_xt + kHalf, false, true, 16, kIdescBmn);
    });
    if (tid >= 64) {
      float v[64];
      wait_mma();
      tmem_row64(acc0 + lane_off, v);  // row i of Y
      // top-right block: -Y
      if (img) img_row_store(img, 1, i, v, -1.f);
      if (Wf) w_row_store(Wf, 1, i, v, -1.f);
      // bottom-right block: row i of the S^{-1} tile; the image copies it chunk
      // by chunk (row 64 + i of the image has the same swizzle as row i of the tile)
      if (img) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint32_t o = (uint32_t)i * 128u + (uint32_t)c * 16u;
          uint8_t *dst = img + kImgRegion + (64 + i) * 128 + c * 16;
          *reinterpret_cast<uint4 *>(dst) = *reinterpret_cast<const uint4 *>(s0 + o);
          *reinterpret_cast<uint4 *>(dst + kImgHalf) = *reinterpret_cast<const uint4 *>(s0 + kHalf + o);
        }
      }
      if (Wf) {
        float u[64];
        tile_row_add(s0, i, u, false);
        w_row_store(Wf, 1, 64 + i, u, 1.f);
      }
      tile_row_store(s0, i, v, 1.f);  // the Y tile, A of the last product
      tmem_row64(acc1 + lane_off, v);  // row i of Y^T
      // bottom-left block: -Y^T
      if (img) img_row_store(img, 0, 64 + i, v, -1.f);
      if (Wf) w_row_store(Wf, 0, 64 + i, v, -1.f);
      fence_proxy_async_smem();
      tc_fence_before();
      bar_named(2);
      // Y X^T
      issue([&] { mma_hilo(acc0, a_s0 - kHalf, a_s0, a_xt, a_xt + kHalf, false, true, 16, kIdescBmn); });
      wait_mma();
      tmem_row64(acc0 + lane_off, v);
      // top-left block: P^{-1} + Y X^T, P^{-1} from its hi/lo tile
      tile_row_add(pi_t, i, v, true);
      if (img) img_row_store(img, 0, i, v, 1.f);
      if (Wf) w_row_store(Wf, 0, i, v, 1.f);
      tc_fence_before();
    }
    __syncthreads();
    if (*abort) break;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(acc0, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_invert_tc(const float *A, float *W, uint8_t *Wimg, int32_t *info, long long nframes,
                             cudaStream_t st, long long frame_base) {
  if (nframes <= 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(invert_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  // four CTAs per SM: 4 x 128 TMEM columns fill the SM's 512
  const long long cap = 4LL * device_sm_count();
  const long long grid = nframes < cap ? nframes : cap;
  invert_tc_kernel<<<(unsigned)grid, kThreads, kSmemBytes, st>>>(A, W, Wimg, info, nframes, frame_base);
  return cudaGetLastError();
}

}  // namespace vdn
