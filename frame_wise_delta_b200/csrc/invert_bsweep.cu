// W_t = (I + A_t)^{-1} for every frame (d = 128) by a blocked symmetric sweep:
// the matrix stays in tensor memory for the whole frame, the four 32 x 32
// pivot blocks are swept in registers by one warp each, and every block's
// rank-32 update of the rest of the matrix runs on the tensor cores.
// Paper: "Video DeltaNet: A Video-Native Hybrid Attention for Livestream
// Video Generation" (summary page), "Core method" (the closed form
// S_t = (Sbar_t + B_t)(I + A_t)^{-1}), "Method steps" step (3) (factor
// I + A_t per frame, independent of the state, all frames in parallel) and
// "Technical novelty" (the inverse produced directly by a Gauss-Jordan-type
// elimination in one kernel).
//
// This kernel serves the text state and the stage call vdn_frame_invert:
// every frame's whole inverse in one CTA, lower latency per frame than the
// block inverse (which needs its first half formed elsewhere) and fp16
// splits in every product. The fused frame path keeps the block inverse,
// whose first half (P^{-1}, X^T and the Schur complement) the Gram kernel's
// sweep pairs form beside the HBM stream.
//
// Sweeping the pivot block K (indices k0 .. k0 + 31) of a symmetric G maps
//   G_KK -> -G_KK^{-1},   G_iK -> G_iK G_KK^{-1} = c_i,   G_Kj -> c_j^T,
//   G_ij -> G_ij - c_i G_Kj                       (i, j outside K);
// after all four blocks G has become -G^{-1}. Per block:
//   1. every thread reads row i of the column block G_:K from TMEM and writes
//      it as an fp16 hi/lo operand row (tile GK, one of two buffers); warp K
//      (the lanes of the block's rows) sweeps G_KK in registers (spread over
//      the lanes as a 2-D grid, one pivot at a time with register shuffles),
//      giving Z = -G_KK^{-1}, writes G_KK^{-1} as the operand tile PI, and
//      -I as its rows of GK;
//   2. tensor cores: columns K of TMEM <- GK PI, which is c_i on every row i
//      outside K and -I G_KK^{-1} = Z on the rows of K;
//   3. every thread writes row i of -(columns K) as the update operand AU
//      (-c_i, and G_KK^{-1} on the rows of K); warp K zeroes its TMEM rows
//      outside the block;
//   4. tensor cores: the columns outside K accumulate AU GK^T: rows outside K
//      get -c_i G_Kj, rows K get G_KK^{-1} G_Kj (added to zero, so this part
//      carries no cancellation against the old G_Kj). The next block's
//      columns go first, with their own completion barrier, so that its sweep
//      starts while the rest of the update runs.
// Every product is a split-fp16 product (hi*hi + lo*hi + hi*lo) accumulated
// in fp32 in TMEM. A pivot that is not positive or not finite (G not positive
// definite) is reported in *info as 1 + the frame index.
//
// 128 threads per CTA, one frame at a time (persistent), four CTAs per SM
// (TMEM 4 x 128 columns). The frame's rows of A arrive by bulk copies of 32
// rows into two operand tiles, which are free between frames; since A is
// symmetric, thread i reads column i of each 32-row piece (a warp reads 128
// consecutive bytes) and stores it as 32 columns of its TMEM lane.
#include "common.cuh"
#include "internal.h"
#include "sweep.cuh"

namespace vdn {
namespace {

constexpr int kThreads = 128;
constexpr int kCtasPerSm = 4;
constexpr int kNb = 32;                          // pivot block
constexpr uint32_t kTile = 128 * 128;            // 128 rows of 128 B: fp16 hi (k < 32), lo (k >= 32)
constexpr uint32_t kOffGK0 = 0;                  // G_:K operand of even blocks; A piece buffer 0
constexpr uint32_t kOffGK1 = kTile;              // G_:K operand of odd blocks
constexpr uint32_t kOffAU = 2 * kTile;           // update operand; A piece buffer 1
constexpr uint32_t kOffPI = 3 * kTile;           // G_KK^{-1} operand, 32 rows; the sweep's layout exchange
constexpr uint32_t kOffBar = kOffPI + 32 * 128;  // c-MMA, first update part, load[2], drain, TMEM address, abort
constexpr size_t kSmemBytes = 1024 + kOffBar + 64;
constexpr uint32_t kPiece = 32 * 128 * 4;        // 32 rows of A, fp32
constexpr uint32_t kTmemCols = 128;

__device__ __forceinline__ void fail(volatile int *abort, int32_t *info) {
  *abort = 1;
  if (info) atomicExch(info, VDN_INFO_TIMEOUT);
}

// 32 lanes x 32 columns of 32-bit TMEM words from registers (thread l: row lane_base + l).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  uint32_t r[16];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
#pragma unroll
    for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(v[16 * h + e]);
    tmem_st16(taddr + 16 * h, r);
  }
}

// Row r of a hi/lo operand tile: 32 values, fp16 hi in logical chunks 0..3
// and lo in chunks 4..7 of the 128-byte swizzled row. The products of this
// kernel take fp16 splits (~2^-22 relative, against ~2^-17 for bf16): its
// rank-32 updates subtract terms much larger than the Schur complements they
// leave when I + A is ill-conditioned, and every value here is well inside
// the fp16 range (|G| <= 1 + U max beta, |G_KK^{-1}| <= 1).
__device__ __forceinline__ void operand_row(uint8_t *tile, int r, const float (&v)[32], float sign) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint4 h, l;
    split_f16x2(sign * v[8 * c + 0], sign * v[8 * c + 1], h.x, l.x);
    split_f16x2(sign * v[8 * c + 2], sign * v[8 * c + 3], h.y, l.y);
    split_f16x2(sign * v[8 * c + 4], sign * v[8 * c + 5], h.z, l.z);
    split_f16x2(sign * v[8 * c + 6], sign * v[8 * c + 7], h.w, l.w);
    uint8_t *row = tile + r * 128;
    *reinterpret_cast<uint4 *>(row + ((c ^ (r & 7)) << 4)) = h;
    *reinterpret_cast<uint4 *>(row + (((c + 4) ^ (r & 7)) << 4)) = l;
  }
}

// Symmetric sweep of the 32 x 32 positive definite pivot block by one warp,
// the block spread over the lanes as a 2-D grid so that every pivot needs
// only register shuffles: lane (a, b) = (lane & 7, lane >> 3) holds
// x[m][n] = G[a + 8m][b + 4n] (m < 4, n < 8). Sweeping pivot k maps
//   G[k][k] -> -1/G[k][k],  G[i][k] -> G[i][k]/G[k][k],  G[k][j] -> G[k][j]/G[k][k],
//   G[i][j] -> G[i][j] - G[i][k] G[k][j] / G[k][k];
// a lane fetches column k of its rows (4 shuffles), row k of its columns
// (8 shuffles) and the pivot (1), then updates its 32 values. Returns false
// if a pivot was not positive or not finite. On return x holds -G^{-1}.
struct Grid32 {
  float x[4][8];
};

__device__ __forceinline__ bool sweep32_grid(Grid32 &g, int lane) {
  const int a = lane & 7, b = lane >> 3;
  bool good = true;
#pragma unroll
  for (int k = 0; k < kNb; ++k) {
    const int km = k >> 3, kn = k >> 2;
    float c[4], r[8];
#pragma unroll
    for (int m = 0; m < 4; ++m) c[m] = __shfl_sync(0xffffffffu, g.x[m][kn], (k & 3) * 8 + a);  // G[a + 8m][k]
#pragma unroll
    for (int n = 0; n < 8; ++n) r[n] = __shfl_sync(0xffffffffu, g.x[km][n], b * 8 + (k & 7));  // G[k][b + 4n]
    const float piv = __shfl_sync(0xffffffffu, g.x[km][kn], (k & 3) * 8 + (k & 7));
    good = good && piv > 0.f && piv < INFINITY;
    const float rp = rcp_approx(piv);
    const bool row_k = a == (k & 7), col_k = b == (k & 3);
    // cr[m] = G[i][k] / piv; on row k, 1 - rp makes the update leave G[k][j] rp
    float cr[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) cr[m] = c[m] * rp;
    if (row_k) cr[km] = 1.f - rp;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const float2 nc = make_float2(-cr[m], -cr[m]);
#pragma unroll
      for (int n = 0; n < 8; n += 2) {
        const float2 y = __ffma2_rn(nc, make_float2(r[n], r[n + 1]), make_float2(g.x[m][n], g.x[m][n + 1]));
        g.x[m][n] = y.x;
        g.x[m][n + 1] = y.y;
      }
    }
    // column k: G[i][k] / piv, and -1/piv on the pivot itself
    if (col_k) {
#pragma unroll
      for (int m = 0; m < 4; ++m) g.x[m][kn] = cr[m];
      if (row_k) g.x[km][kn] = -rp;
    }
  }
  return good;
}

// Row layout (lane i: row i of the block, 32 values) to the grid layout and
// back, through 4 KB of shared memory (`t`: 32 rows of 32 floats, the
// 16-byte chunk c of row r stored at chunk c ^ (r & 7), so that the row
// stores and the grid accesses are both free of bank conflicts).
__device__ __forceinline__ void rows_to_grid(const float (&v)[32], Grid32 &g, float *t, int lane) {
#pragma unroll
  for (int c = 0; c < 8; ++c)
    *reinterpret_cast<float4 *>(t + lane * 32 + 4 * (c ^ (lane & 7))) =
        make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
  __syncwarp();
  const int a = lane & 7, b = lane >> 3;
#pragma unroll
  for (int m = 0; m < 4; ++m)
#pragma unroll
    for (int n = 0; n < 8; ++n) g.x[m][n] = t[(a + 8 * m) * 32 + 4 * (n ^ a) + b];
  __syncwarp();
}

__device__ __forceinline__ void grid_to_rows(const Grid32 &g, float (&v)[32], float *t, int lane) {
  const int a = lane & 7, b = lane >> 3;
#pragma unroll
  for (int m = 0; m < 4; ++m)
#pragma unroll
    for (int n = 0; n < 8; ++n) t[(a + 8 * m) * 32 + 4 * (n ^ a) + b] = g.x[m][n];
  __syncwarp();
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const float4 y = *reinterpret_cast<const float4 *>(t + lane * 32 + 4 * (c ^ (lane & 7)));
    v[4 * c] = y.x, v[4 * c + 1] = y.y, v[4 * c + 2] = y.z, v[4 * c + 3] = y.w;
  }
  __syncwarp();
}

// The six MMAs (3 hi/lo parts x 2 k-steps of 16) of a 32-deep split product
// D (+)= A B^T with A, B K-major hi/lo operand tiles.
__device__ __forceinline__ void mma_split32(uint32_t d, uint32_t a, uint32_t b, uint32_t idesc, bool accumulate) {
#pragma unroll
  for (int part = 0; part < 3; ++part) {
    const uint32_t ao = part == 1 ? 64u : 0u, bo = part == 2 ? 64u : 0u;
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      const uint64_t ad = smem_desc_sw128(a + ao + 32 * ks, 16, 1024);
      const uint64_t bd = smem_desc_sw128(b + bo + 32 * ks, 16, 1024);
      tc_mma_bf16(d, ad, bd, idesc, (accumulate || part > 0 || ks > 0) ? 1u : 0u);
    }
  }
}

__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    invert_bsweep_kernel(const float *__restrict__ A, float *__restrict__ W, uint8_t *__restrict__ Wimg,
                         int32_t *__restrict__ info, long long nframes, long long frame_base) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *gk0 = sm + kOffGK0, *au = sm + kOffAU, *pit = sm + kOffPI;
  float *xch = reinterpret_cast<float *>(pit);  // the sweep's exchange buffer (PI is written after it)
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + kOffBar);
  const uint32_t cbar = smem_u32(bars), pbar = cbar + 8, lbar = cbar + 16;  // load barriers: lbar + 8 b
  const uint32_t dbar = cbar + 32;                                           // drain at exit
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 5);
  volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int i = tid;  // matrix row = TMEM lane
  if (tid == 0) {
    mbar_init(cbar, 1);
    mbar_init(pbar, 1);
    mbar_init(lbar, 1);
    mbar_init(lbar + 8, 1);
    mbar_init(dbar, 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);  // this warp's lanes
  const uint32_t a_gk0 = smem_u32(gk0), a_au = smem_u32(au), a_pi = smem_u32(pit);

  // loads: piece p of frame f (rows 32p .. 32p + 31 of A) into tile buffer p & 1
  long long issued[2] = {0, 0}, landed[2] = {0, 0};
  auto issue_piece = [&](long long f, int p) {  // thread 0
    const int b = p & 1;
    mbar_arrive_expect_tx(lbar + 8 * b, kPiece);
    bulk_load(b ? a_au : a_gk0, A + f * (128LL * 128) + p * (32 * 128), kPiece, lbar + 8 * b);
    ++issued[b];
  };
  // every commit is waited on once, in order, by every thread
  uint32_t cph = 0, pph = 0;
  auto wait_bar = [&](uint32_t bar, uint32_t &ph) {
    bool ok = mbar_wait(bar, ph, abort);
    ph ^= 1u;
    ok = __syncthreads_and(ok) != 0;
    tc_fence_after();
    return ok;
  };

  bool ok = true;
  long long f = blockIdx.x;
  if (tid == 0 && f < nframes) {
    issue_piece(f, 0);
    issue_piece(f, 1);
  }
  for (; ok && f < nframes; f += gridDim.x) {
    const long long fn = f + gridDim.x;
    if (tid == 0 && fn < nframes) bulk_prefetch_l2(A + fn * (128LL * 128), 128 * 128 * 4);
    // ---- G = I + A into TMEM, 32 columns per piece
#pragma unroll 1
    for (int p = 0; p < 4; ++p) {
      const int b = p & 1;
      const bool got = mbar_wait(lbar + 8 * b, (uint32_t)(landed[b] & 1), abort);
      ++landed[b];
      const float *piece = reinterpret_cast<const float *>(b ? au : gk0);
      float v[32];
#pragma unroll
      for (int r = 0; r < 32; ++r) v[r] = piece[r * 128 + i] + (32 * p + r == i ? 1.f : 0.f);
      tmem_st32(trow + 32 * p, v);
      ok = __syncthreads_and(got && ok) != 0;  // every thread has read the buffer
      if (!ok) break;
      if (p < 2 && tid == 0) {
        fence_proxy_async_smem();
        issue_piece(f, p + 2);
      }
    }
    if (!ok) break;
    tmem_st_wait();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    bool good = true;
#pragma unroll 1
    for (int K = 0; K < 4; ++K) {
      const int k0 = kNb * K;
      const bool piv_warp = warp == K;
      // the block's GK buffer; the other one may still be read by the previous update
      uint8_t *gk = sm + ((K & 1) ? kOffGK1 : kOffGK0);
      const uint32_t a_gk = smem_u32(gk);
      // the block's columns are final once the previous block's first update part is done
      if (K > 0 && !wait_bar(pbar, pph)) {
        ok = false;
        break;
      }
      // 1. column block K as the GK operand; warp K sweeps the pivot block and
      //    writes G_KK^{-1} as the PI operand and -I as its rows of GK (so that
      //    step 2 leaves Z = -G_KK^{-1} on its block)
      {
        float v[32];
        tmem_ld32(trow + k0, v);
        if (piv_warp) {
          Grid32 gz;
          rows_to_grid(v, gz, xch, lane);
          good = sweep32_grid(gz, lane) && good;
          grid_to_rows(gz, v, xch, lane);  // v: row lane of Z = -G_KK^{-1}
          operand_row(pit, lane, v, -1.f);
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = e == lane ? -1.f : 0.f;
        }
        operand_row(gk, i, v, 1.f);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      // 2. columns K <- GK G_KK^{-1}: c_i on the rows outside K, Z on rows K
      if (tid == 0 && !*abort) {
        tc_fence_after();
        mma_split32(tmem + k0, a_gk, a_pi, idesc_f16_f32(128, 32, false, false), false);
        tc_commit(cbar);
      }
      // (this also means the previous block's update has completed: the MMAs
      // of one thread complete in order)
      if (!wait_bar(cbar, cph)) {
        ok = false;
        break;
      }
      // 3. the update operand: row i of -(columns K), i.e. -c_i, and -Z =
      //    G_KK^{-1} on the rows of K; warp K zeroes its rows outside the block
      {
        float c[32];
        tmem_ld32(trow + k0, c);
        operand_row(au, i, c, -1.f);
        if (piv_warp) {
#pragma unroll
          for (int e = 0; e < 32; ++e) c[e] = 0.f;
#pragma unroll
          for (int cb = 0; cb < 4; ++cb)
            if (cb != K) tmem_st32(trow + 32 * cb, c);
          tmem_st_wait();
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      // 4. columns outside K += AU GK^T: first the next block's columns (its
      //    sweep starts as soon as they are done), then the rest
      if (tid == 0 && !*abort) {
        tc_fence_after();
        if (K < 3) {
          mma_split32(tmem + k0 + kNb, a_au, a_gk + (k0 + kNb) * 128, idesc_f16_f32(128, kNb, false, false), true);
          tc_commit(pbar);
          if (k0 > 0) mma_split32(tmem, a_au, a_gk, idesc_f16_f32(128, k0, false, false), true);
          if (k0 + 2 * kNb < 128)
            mma_split32(tmem + k0 + 2 * kNb, a_au, a_gk + (k0 + 2 * kNb) * 128,
                        idesc_f16_f32(128, 128 - k0 - 2 * kNb, false, false), true);
        } else {
          mma_split32(tmem, a_au, a_gk, idesc_f16_f32(128, k0, false, false), true);
          tc_commit(cbar);
        }
      }
    }
    if (!ok) break;
    if (!wait_bar(cbar, cph)) {  // the last block's update
      ok = false;
      break;
    }
    // the operand tiles are free: the next frame's first pieces
    if (tid == 0 && fn < nframes) {
      fence_proxy_async_smem();
      issue_piece(fn, 0);
      issue_piece(fn, 1);
    }
    // ---- output: TMEM holds -W; row i of the image (hi/lo), W column i
    uint8_t *img = Wimg ? Wimg + f * (long long)kImgBytes : nullptr;
    float *Wf = W ? W + f * (128LL * 128) : nullptr;
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
      float v[32];
      tmem_ld32(trow + 32 * cc, v);
#pragma unroll
      for (int e = 0; e < 32; ++e) v[e] = -v[e];
      if (img) {
        uint8_t *base = img + (cc >> 1) * kImgRegion + i * 128;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 h, l;
          split_bf16x2(v[8 * q + 0], v[8 * q + 1], h.x, l.x);
          split_bf16x2(v[8 * q + 2], v[8 * q + 3], h.y, l.y);
          split_bf16x2(v[8 * q + 4], v[8 * q + 5], h.z, l.z);
          split_bf16x2(v[8 * q + 6], v[8 * q + 7], h.w, l.w);
          const uint32_t off = (uint32_t)(((4 * (cc & 1) + q) ^ (i & 7)) << 4);
          *reinterpret_cast<uint4 *>(base + off) = h;
          *reinterpret_cast<uint4 *>(base + kImgHalf + off) = l;
        }
      }
      if (Wf) {
#pragma unroll
        for (int e = 0; e < 32; ++e) Wf[(32 * cc + e) * 128 + i] = v[e];
      }
    }
    if (__any_sync(0xffffffffu, !good) && lane == 0) report_frame_failure(info, frame_base + f);
    tc_fence_before();
    __syncthreads();
  }
  if (!ok) fail(abort, info);
  // no copy may still be landing in shared memory and no MMA still writing
  // tensor memory when the CTA leaves (after a failed wait some may be)
  if (tid == 0) {
    volatile int never = 0;
    for (int b = 0; b < 2; ++b)
      for (long long n = landed[b]; n < issued[b]; ++n) mbar_wait(lbar + 8 * b, (uint32_t)(n & 1), &never);
    tc_commit(dbar);
    mbar_wait(dbar, 0, &never);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_invert_bsweep(const float *A, float *W, uint8_t *Wimg, int32_t *info, long long nframes,
                                 cudaStream_t st, long long frame_base) {
  if (nframes <= 0) return cudaSuccess;
  cudaError_t e =
      cudaFuncSetAttribute(invert_bsweep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const long long cap = (long long)kCtasPerSm * device_sm_count();
  const long long grid = nframes < cap ? nframes : cap;
  invert_bsweep_kernel<<<(unsigned)grid, kThreads, kSmemBytes, st>>>(A, W, Wimg, info, nframes, frame_base);
  return cudaGetLastError();
}

}  // namespace vdn
