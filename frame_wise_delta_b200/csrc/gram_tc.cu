// Frame statistics on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
// Paper: "Video DeltaNet: A Video-Native Hybrid Attention for Livestream
// Video Generation" (summary page), "Method steps" step (3):
//   A_t = K_t^T Diag(beta_t) K_t,   B_t = V_t^T Diag(beta_t) K_t   (bf16 in, fp32 out, d = 128).
//
// One MMA stream per frame computes D = K^T [K | V] (M = 128, N = 256,
// contraction over the frame's U tokens): columns 0..127 of D are A_t and
// columns 128..255 are B_t^T. Both operands come straight from the TMA
// tiles: a tile of 64 tokens x 128 channels is stored as 64-channel blocks,
// 128-byte swizzled, which is the MN-major canonical layout (token = K
// index, channel = M/N index). K-block stride 1024 B per 8 tokens, M/N-block
// stride 8 KB.
//
// With one gate per frame, beta_t scales the fp32 sums in the epilogue. With
// one gate per token ("Core method": beta_{t,u}), four more warps write a
// copy of each K tile with row u scaled by beta_{t,u}, split into bf16 hi and
// lo parts (hi + lo = beta k to ~2^-17), and two MMAs per step compute
// (Diag(beta) K)^T [K | V] instead.
//
// Persistent kernel, one CTA per SM, 6 warps (10 with per-token gates):
//   warp 0     : TMA producer (4 loads of 8 KB per 64-token stage)
//   warp 1     : TMEM allocator and single-thread MMA issuer
//   warps 2..5 : epilogue: TMEM -> registers -> fp32 stores
//   warps 6..9 : (per-token gates) the scaled K tile of each stage, or
//                (PSW) two pairs of sweep warps: each takes every other frame's
//                leading 64 x 64 block P of I + A_t, which the epilogue stages
//                in shared memory, sweeps it, and forms P^{-1}, X^T = Q^T P^{-1}
//                and the Schur complement S = R - Q^T X (schur.cuh) from the
//                rows 64..127 of A_t that the epilogue writes, so the CUDA-core
//                half of the block inverse runs beside the HBM-bound stream
//                instead of after it; rows 0..63 of A_t are then not written
//                (X^T and S take their place)
// TMEM holds two 256-column accumulators so a frame's epilogue overlaps the
// next frame's MMAs. Every wait is bounded (see common.cuh).
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "schur.cuh"
#include "sweep.cuh"

namespace vdn {
namespace {

constexpr int kD = 128;
constexpr int kUT = 64;                          // tokens per pipeline stage
constexpr int kStagesMax = 4;
constexpr int kBlockBytes = kUT * 128;           // one 64-channel block
constexpr uint32_t kTmemCols = 512;
constexpr int kPairs = 3;  // PSW: sweep pairs, each taking every kPairs-th frame
constexpr int kBarBytes = 8 * (3 * kStagesMax + 2 + 2 + 1 + 2 * kPairs);
// PSW: per sweep pair an fp32 staging of P (it then holds P^{-1}, then X^T)
// and one of Q^T, both in schur.cuh's layout, and the pair's exchange vector
constexpr int kPStage = kSchurBytes;
constexpr int kPTile = kSchurBytes;
constexpr int kPSmem = kPairs * (kPStage + kPTile + 2 * 64 * 4);
// per stage: the K and V blocks of channels 0..63 and 64..127 (+ the scaled
// K blocks: hi part of both, then lo part of both)
template <bool TOKB> constexpr int kStagesT = TOKB ? 3 : 4;
template <bool TOKB> constexpr int kStageBytesT = (TOKB ? 8 : 4) * kBlockBytes;
template <bool TOKB> constexpr int kThreadsT = TOKB ? 320 : 192;
template <bool TOKB, bool PSW>
constexpr size_t kSmemBytesT = 1024 + (size_t)kStagesT<TOKB> * kStageBytesT<TOKB> + (PSW ? kPSmem : 0) + kBarBytes + 16;

struct GramArgs {
  float *A;
  float *Bm;
  const float *beta;
  int32_t *info;
  long long nframes;
  int ntiles;
  int U;
  float *Pinv;            // PSW: [nframes] P^{-1} (64 x 64 fp32, schur.cuh layout)
  long long frame_base;   // PSW: frame index of frame 0 for *info
};

__device__ __forceinline__ void fail(volatile int *abort, int32_t *info) {
  *abort = 1;
  if (info) atomicExch(info, VDN_INFO_TIMEOUT);
}

template <bool TOKB, bool PSW>
__global__ void __launch_bounds__(TOKB ? 320 : PSW ? 192 + 64 * kPairs : 192, 1)
    gram_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   GramArgs p) {
  static_assert(!(TOKB && PSW), "one use of warps 6..9");
  constexpr int kStageBytes = kStageBytesT<TOKB>;
  constexpr int kStages = kStagesT<TOKB>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  uint8_t *stages = smem;
  uint8_t *pmem = smem + kStages * kStageBytes;  // PSW area
  float *pstage = reinterpret_cast<float *>(pmem);                               // [kPairs][16 KB] P
  uint8_t *ptile = pmem + kPairs * kPStage;                                      // [kPairs][16 KB] Q^T
  float *pcbuf = reinterpret_cast<float *>(pmem + kPairs * (kPStage + kPTile));  // [kPairs][2][64]
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kStages * kStageBytes + (PSW ? kPSmem : 0));
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(reinterpret_cast<uint8_t *>(bars) + kBarBytes);
  volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8 * kStages;
  const uint32_t tfull0 = empty0 + 8 * kStages;
  const uint32_t tempty0 = tfull0 + 16;
  const uint32_t drain = tempty0 + 16;
  const uint32_t scaled0 = drain + 8;  // per stage: the scaled K tile is written
  const uint32_t pready0 = scaled0 + 8 * kStagesMax;  // PSW, per pair: P staged (128 arrivals)
  const uint32_t pfree0 = pready0 + 8 * kPairs;       // PSW, per pair: stagings free (64 arrivals)

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8 * b, 1);
      mbar_init(tempty0 + 8 * b, 128);
    }
    mbar_init(drain, 1);
    if (TOKB)
      for (int s = 0; s < kStages; ++s) mbar_init(scaled0 + 8 * s, 128);
    if (PSW)
      for (int q = 0; q < kPairs; ++q) {
        mbar_init(pready0 + 8 * q, 128);
        mbar_init(pfree0 + 8 * q, 64);
      }
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
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int stage = 0;
      uint32_t phase = 0;
      int armed_parity[kStages];
      for (int s = 0; s < kStages; ++s) armed_parity[s] = -1;
      bool ok = true;
      for (long long f = blockIdx.x; ok && f < p.nframes; f += gridDim.x) {
        for (int j = 0; j < p.ntiles; ++j) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1, abort)) {
            fail(abort, p.info);
            ok = false;
            break;
          }
          const uint32_t dst = smem_u32(stages + stage * kStageBytes);
          const uint32_t fb = full0 + 8 * stage;
          mbar_arrive_expect_tx(fb, 4 * kBlockBytes);  // the four TMA blocks
          armed_parity[stage] = (int)phase;
          const int y = j * kUT, z = (int)f;
          tma_load_3d(dst + 0 * kBlockBytes, &tmK, fb, 0, y, z);
          tma_load_3d(dst + 1 * kBlockBytes, &tmK, fb, 64, y, z);
          tma_load_3d(dst + 2 * kBlockBytes, &tmV, fb, 0, y, z);
          tma_load_3d(dst + 3 * kBlockBytes, &tmV, fb, 64, y, z);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // Never leave with copies in flight: wait (bounded) for the last
      // arming of every stage to land.
      volatile int never = 0;
      for (int s = 0; s < kStages; ++s)
        if (armed_parity[s] >= 0) mbar_wait(full0 + 8 * s, (uint32_t)armed_parity[s], &never);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 256, true, true);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (long long f = blockIdx.x; ok && f < p.nframes; f += gridDim.x, ++it) {
        const int buf = it & 1;
        const uint32_t use = (uint32_t)(it >> 1);
        if (!mbar_wait(tempty0 + 8 * buf, (use & 1) ^ 1, abort)) {
          fail(abort, p.info);
          break;
        }
        tc_fence_after();
        const uint32_t dcol = tmem_base + (uint32_t)(buf * 256);
        for (int j = 0; j < p.ntiles; ++j) {
          if (!mbar_wait((TOKB ? scaled0 : full0) + 8 * stage, phase, abort)) {
            fail(abort, p.info);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t base = smem_u32(stages + stage * kStageBytes);
#pragma unroll
          for (int ks = 0; ks < kUT / 16; ++ks) {
            const uint64_t bdesc = smem_desc_sw128(base + ks * 2048, kBlockBytes, 1024);
            if (TOKB) {
              // (Diag(beta) K)^T as its hi and lo parts
#pragma unroll
              for (int part = 0; part < 2; ++part) {
                const uint32_t abase = base + (4 + 2 * part) * kBlockBytes;
                const uint64_t adesc = smem_desc_sw128(abase + ks * 2048, kBlockBytes, 1024);
                tc_mma_bf16(dcol, adesc, bdesc, idesc, (j > 0 || ks > 0 || part > 0) ? 1u : 0u);
              }
            } else {
              tc_mma_bf16(dcol, bdesc, bdesc, idesc, (j > 0 || ks > 0) ? 1u : 0u);
            }
          }
          tc_commit(empty0 + 8 * stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (ok) tc_commit(tfull0 + 8 * buf);
      }
      // Let every issued MMA finish before TMEM is released.
      tc_commit(drain);
      volatile int never = 0;
      mbar_wait(drain, 0, &never);
    }
  } else if (TOKB && warp >= 6) {
    // scaled copy of each K tile: row u (token j * 64 + u) times beta_{t,u},
    // split into bf16 hi and lo, at the same offsets (the swizzle permutes
    // 16-byte chunks inside a row, so a row is its 128-byte line)
    const int st_ = threadIdx.x - 192;         // 0..127
    const int blk = st_ >> 6, r = st_ & 63;    // one 128-byte row (token r) of one K block
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (long long f = blockIdx.x; ok && f < p.nframes; f += gridDim.x) {
      const float *bf = p.beta + f * (long long)p.U;
      for (int j = 0; j < p.ntiles; ++j) {
        const int u = j * kUT + r;
        const float b = u < p.U ? __ldg(bf + u) : 0.f;  // in flight during the wait
        if (!mbar_wait(full0 + 8 * stage, phase, abort)) {
          fail(abort, p.info);
          ok = false;
          break;
        }
        uint8_t *row = stages + stage * kStageBytes + blk * kBlockBytes + r * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          // rotate the chunk order by row so a warp's 16-byte accesses spread over the banks
          const int off = ((c + r) & 7) * 16;
          const uint4 x = *reinterpret_cast<const uint4 *>(row + off);
          const uint32_t w[4] = {x.x, x.y, x.z, x.w};
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            split_bf16x2(b * __uint_as_float(w[e] << 16), b * __uint_as_float(w[e] & 0xFFFF0000u), hi[e], lo[e]);
          *reinterpret_cast<uint4 *>(row + 4 * kBlockBytes + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4 *>(row + 6 * kBlockBytes + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
        fence_proxy_async_smem();
        mbar_arrive(scaled0 + 8 * stage);
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
  } else if (PSW && warp >= 6) {
    // sweep pair pq (warps 6 + 2 pq, 7 + 2 pq): every kPairs-th frame of this CTA
    const int pq = (warp - 6) >> 1;
    const int st = threadIdx.x - 192 - 64 * pq;  // 0..63
    const int rg = st / kSweepGrid, cg = st % kSweepGrid;
    const int nb = 3 + pq;  // the pair's named barrier
    float *ps = pstage + pq * (kPStage / 4);
    const float *qs = reinterpret_cast<const float *>(ptile + pq * kPTile);
    float(*cb)[64] = reinterpret_cast<float(*)[64]>(pcbuf + pq * 128);
    bool okw = true;
    int it = 0;
    for (long long f = blockIdx.x; f < p.nframes; f += gridDim.x, ++it) {
      if (it % kPairs != pq) continue;
      if (okw && !mbar_wait(pready0 + 8 * pq, (uint32_t)(it / kPairs) & 1, abort)) {
        fail(abort, p.info);
        okw = false;
      }
      Sweep<64> X;
#pragma unroll
      for (int a = 0; a < Sweep<64>::R; ++a)
#pragma unroll
        for (int b = 0; b <= a; ++b) X.at(a, b) = ps[swz64(rg + kSweepGrid * a, cg + kSweepGrid * b)];
      auto sync = [nb] { asm volatile("bar.sync %0, 64;" ::"r"(nb) : "memory"); };
      const bool ok = X.run(cb, rg, cg, sync);
      if (st == 0 && !ok) report_frame_failure(p.info, p.frame_base + f);
      // P^{-1}, then X^T, replace P in its staging; both stagings are
      // released to the epilogue (for the pair's next frame) at the end
      float *Af = p.A + f * (long long)(kD * kD);
      schur_prep(X, qs, Af + 64 * kD + 64, ps, p.Pinv + f * 64LL * 64, Af + kSchurXT, Af + kSchurS, st, sync);
      mbar_arrive(pfree0 + 8 * pq);
    }
    if (st == 0) bulk_wait_all();  // the P^{-1} and X^T copies have landed
  } else {
    // epilogue warps 2..5 -> TMEM sub-partitions 2, 3, 0, 1
    const int sub = warp & 3;
    const int row = sub * 32 + lane;
    int it = 0;
    for (long long f = blockIdx.x; f < p.nframes; f += gridDim.x, ++it) {
      const int buf = it & 1;
      const uint32_t use = (uint32_t)(it >> 1);
      const int pq = it % kPairs;  // PSW: the sweep pair of this frame
      const uint32_t puse = (uint32_t)(it / kPairs);
      float *ps = pstage + pq * (kPStage / 4);
      float *qs = reinterpret_cast<float *>(ptile + pq * kPTile);
      if (PSW && puse > 0) {
        // the pair is done with its stagings of kPairs frames ago
        if (!mbar_wait(pfree0 + 8 * pq, (puse - 1) & 1, abort)) fail(abort, p.info);
      }
      // every lane waits (acquire); the warp then agrees on the outcome so
      // that it enters the aligned TMEM loads together or not at all
      const bool ok = __all_sync(0xffffffffu, mbar_wait(tfull0 + 8 * buf, use & 1, abort));
      if (!ok) {
        fail(abort, p.info);
        break;
      }
      tc_fence_after();
      const float bt = TOKB ? 1.f : p.beta[f];
      float *Af = p.A + f * (long long)(kD * kD);
      float *Bf = p.Bm + f * (long long)(kD * kD);
#pragma unroll 1
      for (int cc = 0; cc < 8; ++cc) {
        float v[32];
        tmem_ld32(tmem_base + (uint32_t)(buf * 256 + cc * 32) + ((uint32_t)(sub * 32) << 16), v);
        // D[row][n]: n < 128 -> A[row][n] = A[n][row] (symmetric; written by
        // column so that a warp stores 32 consecutive floats); n >= 128 ->
        // B[n-128][row].
        float *dst = (cc < 4 ? Af + (cc * 32) * kD : Bf + ((cc - 4) * 32) * kD) + row;
        // PSW: P and Q^T are staged for the sweep pair instead of written;
        // of rows 64..127 only R (columns 64..127) is written, and the pair
        // puts X^T and S in rows 0..63
        if (!(PSW && (cc < 2 || (cc < 4 && row < 64)))) {
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) dst[jj * kD] = bt * v[jj];
        }
        if (PSW && cc < 2 && row < 64) {
          // P = I + A[0..63][0..63] for the sweep pair (A symmetric: row `row`)
#pragma unroll
          for (int c4 = 0; c4 < 8; ++c4) {
            const int c0 = cc * 32 + 4 * c4;
            *reinterpret_cast<float4 *>(ps + swz64(row, c0)) =
                make_float4(bt * v[4 * c4] + (row == c0 ? 1.f : 0.f), bt * v[4 * c4 + 1] + (row == c0 + 1 ? 1.f : 0.f),
                            bt * v[4 * c4 + 2] + (row == c0 + 2 ? 1.f : 0.f),
                            bt * v[4 * c4 + 3] + (row == c0 + 3 ? 1.f : 0.f));
          }
        }
        if (PSW && cc < 2 && row >= 64) {
          // Q^T: row row - 64, columns 32 cc .. + 31
#pragma unroll
          for (int c4 = 0; c4 < 8; ++c4)
            *reinterpret_cast<float4 *>(qs + swz64(row - 64, cc * 32 + 4 * c4)) =
                make_float4(bt * v[4 * c4], bt * v[4 * c4 + 1], bt * v[4 * c4 + 2], bt * v[4 * c4 + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(tempty0 + 8 * buf);
      if (PSW) mbar_arrive(pready0 + 8 * pq);
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

bool gram_tc_supported(int in_dtype, int D, int U) { return in_dtype == VDN_BF16 && D == 128 && U > 0; }

// 3-D tensor map over [frames][rows][128] bf16 with a (64 ch x box_rows x 1) box.
bool make_rows_map(CUtensorMap *m, const void *base, long long frames, int rows, int box_rows) {
  auto enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
  if (!enc) return false;
  cuuint64_t dims[3] = {128, (cuuint64_t)rows, (cuuint64_t)frames};
  cuuint64_t strides[2] = {128 * 2, (cuuint64_t)rows * 128 * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <bool TOKB, bool PSW>
cudaError_t launch_gram_t(const CUtensorMap &tmK, const CUtensorMap &tmV, const GramArgs &a, cudaStream_t st,
                          int spare_sms) {
  constexpr size_t smem = kSmemBytesT<TOKB, PSW>;
  cudaError_t e = cudaFuncSetAttribute(gram_tc_kernel<TOKB, PSW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  int sms = device_sm_count() - spare_sms;
  if (sms < 1) sms = 1;
  const long long grid = a.nframes < sms ? a.nframes : sms;
  gram_tc_kernel<TOKB, PSW><<<(unsigned)grid, TOKB ? 320 : PSW ? 192 + 64 * kPairs : 192, smem, st>>>(tmK, tmV, a);
  return cudaGetLastError();
}

cudaError_t launch_gram_tc(const void *K, const void *V, const float *beta, bool per_token, float *A,
                           float *Bm, long long nframes, int U, int32_t *info, cudaStream_t st, float *Pinv,
                           long long frame_base, int spare_sms) {
  if (nframes <= 0) return cudaSuccess;
  CUtensorMap tmK, tmV;
  if (!make_rows_map(&tmK, K, nframes, U, kUT) || !make_rows_map(&tmV, V, nframes, U, kUT))
    return cudaErrorInvalidValue;
  GramArgs a{A, Bm, beta, info, nframes, (U + kUT - 1) / kUT, U, Pinv, frame_base};
  if (per_token) {
    // the per-token stages use warps 6..9 and most of shared memory: P^{-1},
    // X^T and S then come from their own kernel
    cudaError_t e = launch_gram_t<true, false>(tmK, tmV, a, st, spare_sms);
    if (e != cudaSuccess || !Pinv) return e;
    return launch_schur_prep(A, Pinv, info, nframes, st, frame_base);
  }
  return Pinv ? launch_gram_t<false, true>(tmK, tmV, a, st, spare_sms)
              : launch_gram_t<false, false>(tmK, tmV, a, st, spare_sms);
}

}  // namespace vdn
