// C ABI of libvdn: host-side validation and dispatch of the VDA kernels.
// Every entry point checks its arguments before enqueuing anything, never
// allocates, and never synchronises. See include/vdn.h for the contract.
#include <stdarg.h>
#include <stdio.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace vdn {

void *tensor_map_encoder() {
  static std::once_flag once;
  static void *fn = nullptr;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = p;
  });
  return fn;
}

int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
    return 1;
  return n;
}

}  // namespace vdn

using namespace vdn;

namespace {

thread_local char g_err[512] = "";

vdn_status fail(vdn_status st, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

vdn_status cuda_fail(cudaError_t e, const char *where) {
  return fail(VDN_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

struct Geo {
  long long BH;
  int H, T, U, D, C, chunk, anchors, n_text, in_dtype, out_dtype, tokb, bridge;
  size_t in_elem, out_elem;
};

vdn_status check_shape(const vdn_shape *s, Geo *g) {
  if (!s) return fail(VDN_ERR_INVALID, "shape is NULL");
  if (s->B < 0 || s->H < 0 || s->T < 0 || s->U < 0 || s->n_text < 0)
    return fail(VDN_ERR_INVALID, "negative size (B=%d H=%d T=%d U=%d n_text=%d)", s->B, s->H, s->T,
                s->U, s->n_text);
  if (s->dk != s->dv) return fail(VDN_ERR_UNSUPPORTED, "dk (%d) != dv (%d)", s->dk, s->dv);
  if (s->dk != 16 && s->dk != 32 && s->dk != 64 && s->dk != 128)
    return fail(VDN_ERR_UNSUPPORTED, "d = %d not in {16, 32, 64, 128}", s->dk);
  if (s->chunk < 1 || s->chunk > 16) return fail(VDN_ERR_INVALID, "chunk = %d not in [1, 16]", s->chunk);
  if (s->anchors != 0 && s->anchors != 1) return fail(VDN_ERR_INVALID, "anchors must be 0 or 1");
  if (s->beta_per_token != 0 && s->beta_per_token != 1)
    return fail(VDN_ERR_INVALID, "beta_per_token must be 0 or 1");
  if (s->decay_bridge != 0 && s->decay_bridge != 1) return fail(VDN_ERR_INVALID, "decay_bridge must be 0 or 1");
  if ((s->in_dtype != VDN_F32 && s->in_dtype != VDN_BF16) ||
      (s->out_dtype != VDN_F32 && s->out_dtype != VDN_BF16))
    return fail(VDN_ERR_INVALID, "dtype must be VDN_F32 or VDN_BF16");
  g->BH = (long long)s->B * s->H;
  g->H = s->H;
  g->T = s->T;
  g->U = s->U;
  g->D = s->dk;
  g->chunk = s->chunk;
  g->C = (s->T + s->chunk - 1) / s->chunk;
  g->anchors = s->anchors ? 3 : 0;  // kernel mask: first and last frame
  g->n_text = s->n_text;
  g->in_dtype = s->in_dtype;
  g->out_dtype = s->out_dtype;
  g->tokb = s->beta_per_token;
  g->bridge = s->decay_bridge;
  g->in_elem = s->in_dtype == VDN_BF16 ? 2 : 4;
  g->out_elem = s->out_dtype == VDN_BF16 ? 2 : 4;
  if (g->BH * (long long)(g->T > 0 ? g->T : 1) > 0x7fffffffLL)
    return fail(VDN_ERR_UNSUPPORTED, "B*H*T = %lld exceeds 2^31-1", g->BH * g->T);
  if (g->C > 65535) return fail(VDN_ERR_UNSUPPORTED, "more than 65535 chunks");
  if ((double)g->BH * g->T * g->U * g->D > 4.0e18)
    return fail(VDN_ERR_UNSUPPORTED, "tensor too large");
  return VDN_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

vdn_status need(const void *p, const char *name, bool required) {
  if (!required) return VDN_OK;
  if (!p) return fail(VDN_ERR_INVALID, "%s is NULL", name);
  if (!aligned16(p)) return fail(VDN_ERR_INVALID, "%s is not 16-byte aligned", name);
  return VDN_OK;
}

#define VDN_TRY(x)                    \
  do {                                \
    vdn_status st_ = (x);             \
    if (st_ != VDN_OK) return st_;    \
  } while (0)

#define VDN_CUDA(x, where)                        \
  do {                                            \
    cudaError_t e_ = (x);                         \
    if (e_ != cudaSuccess) return cuda_fail(e_, where); \
  } while (0)

size_t align256(size_t n) { return (n + 255) & ~size_t(255); }


// ----------------------------------------------------------- stage calls
// Pinv (tensor path): also form each frame's P^{-1}, X^T and S for the block
// inverse (schur.cuh)
vdn_status run_grams(const Geo &g, const void *K, const void *V, const float *beta, float *A,
                     float *Bm, long long nframes, int U, int32_t *info, cudaStream_t st,
                     float *Pinv = nullptr, long long frame_base = 0, int spare_sms = 0) {
  if (nframes <= 0) return VDN_OK;
  const size_t bytes = (size_t)nframes * g.D * g.D * sizeof(float);
  if (U == 0) {
    VDN_CUDA(cudaMemsetAsync(A, 0, bytes, st), "memset A");
    VDN_CUDA(cudaMemsetAsync(Bm, 0, bytes, st), "memset Bm");
    if (Pinv) VDN_CUDA(launch_schur_prep(A, Pinv, info, nframes, st, frame_base), "Schur step");
    return VDN_OK;
  }
  if (gram_tc_supported(g.in_dtype, g.D, U)) {
    VDN_CUDA(launch_gram_tc(K, V, beta, g.tokb != 0, A, Bm, nframes, U, info, st, Pinv, frame_base, spare_sms),
             "gram_tc");
  } else {
    VDN_CUDA(launch_gram_simt(K, V, g.in_dtype, beta, g.tokb != 0, A, Bm, nframes, U, g.D, st),
             "gram_simt");
    if (Pinv) VDN_CUDA(launch_schur_prep(A, Pinv, info, nframes, st, frame_base), "Schur step");
  }
  return VDN_OK;
}

// og: the readout epilogue (step (5)), or nullptr
// F0: the forward state chunk 0 reads instead of F[0] (streaming), or nullptr
// alpha: the decay gates when the readout goes through the decay bridge
// (g.bridge), otherwise ignored.
// bridge_prev: with F0 and the bridge, the decay product that chunk 0's
// forward factor also carries (a stream segment), or nullptr.
vdn_status run_readout(const Geo &g, const void *Q, const float *F, const float *G, void *O,
                       int32_t *info, cudaStream_t st, const OutGate *og = nullptr,
                       const float *F0 = nullptr, const float *alpha = nullptr,
                       const float *bridge_prev = nullptr) {
  if (g.BH * g.T * g.U == 0) return VDN_OK;
  const float *bridge = g.bridge ? alpha : nullptr;
  const float *bprev = g.bridge ? bridge_prev : nullptr;
  if (readout_tc_supported(g.in_dtype, g.out_dtype, g.D, g.U)) {
    VDN_CUDA(launch_readout_tc(Q, F, G, O, g.BH, g.T, g.U, g.chunk, g.anchors, info, st, og, F0, bridge, bprev),
             "readout_tc");
  } else {
    VDN_CUDA(launch_readout_simt(Q, g.in_dtype, F, G, O, g.out_dtype, g.BH, g.T, g.U, g.chunk,
                                 g.anchors, g.D, st, og, F0, bridge, bprev),
             "readout_simt");
  }
  return VDN_OK;
}

// Validates a caller's vdn_out_gate (NULL allowed when `optional`) into *out.
vdn_status check_gate(const Geo &g, const vdn_out_gate *og, bool optional, OutGate *out, const OutGate **use) {
  *use = nullptr;
  if (!og) return optional ? VDN_OK : fail(VDN_ERR_INVALID, "og is NULL");
  const bool any = g.BH * g.T * g.U > 0;
  VDN_TRY(need(og->gate, "og->gate", any));
  VDN_TRY(need(og->norm_weight, "og->norm_weight", any));
  if (!(og->eps > 0.f) || !(og->eps < 3.0e38f)) return fail(VDN_ERR_INVALID, "og->eps must be positive and finite");
  *out = OutGate{og->gate, og->norm_weight, og->eps, g.H > 0 ? g.H : 1};
  *use = out;
  return VDN_OK;
}

bool tensor_path(const Geo &g) { return g.in_dtype == VDN_BF16 && g.out_dtype == VDN_BF16 && g.D == 128; }

size_t align256(size_t n);

// Scratch of the text state: Ax, Bx (fp32) and, on the tensor path, the W images.
struct TextLayout {
  size_t ax, bx, wimg, total;
};
TextLayout text_layout(const Geo &g) {
  TextLayout L{};
  const size_t dd = (size_t)g.D * g.D * sizeof(float);
  L.ax = 0;
  L.bx = align256(g.BH * dd);
  L.wimg = L.bx + align256(g.BH * dd);
  L.total = L.wimg + (tensor_path(g) ? align256((size_t)g.BH * kImgBytes) : 0);
  return L;
}

vdn_status run_text_state(const Geo &g, const void *Kx, const void *Vx, const float *beta_x,
                          float *S_T, char *ws, int32_t *info, cudaStream_t st) {
  if (g.BH == 0) return VDN_OK;
  if (g.n_text == 0) {
    VDN_CUDA(cudaMemsetAsync(S_T, 0, (size_t)g.BH * g.D * g.D * sizeof(float), st), "memset S_T");
    return VDN_OK;
  }
  const TextLayout L = text_layout(g);
  float *Ax = (float *)(ws + L.ax), *Bx = (float *)(ws + L.bx);
  VDN_TRY(run_grams(g, Kx, Vx, beta_x, Ax, Bx, g.BH, g.n_text, info, st));
  if (tensor_path(g)) {
    // S_T is the injection of one "frame" made of the text tokens: invert,
    // then one J-chain step (B_x W_x) on the tensor cores.
    uint8_t *Wimg = (uint8_t *)(ws + L.wimg);
    VDN_CUDA(launch_invert_bsweep(Ax, nullptr, Wimg, info, g.BH, st, 0), "text invert");
    VDN_CUDA(launch_compose_tc(Wimg, Bx, Ax, nullptr, S_T, nullptr, nullptr, nullptr, g.BH, 1, 1, 0,
                               /*ndirs=*/1, /*j_transposed=*/false, info, st),
             "text injection");
  } else {
    VDN_CUDA(launch_factor_simt(Ax, Bx, nullptr, nullptr, S_T, info, g.BH, 1, 0, g.D, st),
             "text factor");
  }
  return VDN_OK;
}

// One CTA waits on a barrier that nothing arrives at: the bounded wait gives
// up after its limit and the kernel reports the timeout in *info.
__global__ void wait_selftest_kernel(int32_t *info) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const bool ok = mbar_wait(smem_u32(&bar), 0, &abort);
  if (!__all_sync(0xffffffffu, ok) && threadIdx.x == 0) atomicExch(info, VDN_INFO_TIMEOUT);
}

}  // namespace

void vdn::set_last_error(const char *msg) { snprintf(g_err, sizeof(g_err), "%s", msg); }

vdn_status vdn::validate_shape(const vdn_shape *s) {
  Geo g;
  return check_shape(s, &g);
}

extern "C" {

const char *vdn_status_string(vdn_status st) {
  switch (st) {
    case VDN_OK: return "VDN_OK";
    case VDN_ERR_INVALID: return "VDN_ERR_INVALID";
    case VDN_ERR_UNSUPPORTED: return "VDN_ERR_UNSUPPORTED";
    case VDN_ERR_CUDA: return "VDN_ERR_CUDA";
    case VDN_ERR_NUMERIC: return "VDN_ERR_NUMERIC";
  }
  return "VDN_ERR_UNKNOWN";
}

const char *vdn_last_error(void) { return g_err; }

int32_t vdn_version(void) { return 100; }

vdn_status vdn_selftest_wait(int32_t *info, vdn_stream_t stream) {
  g_err[0] = 0;
  VDN_TRY(need(info, "info", true));
  cudaStream_t st = (cudaStream_t)stream;
  VDN_CUDA(cudaMemsetAsync(info, 0, sizeof(int32_t), st), "memset info");
  wait_selftest_kernel<<<1, 32, 0, st>>>(info);
  VDN_CUDA(cudaGetLastError(), "selftest wait");
  return VDN_OK;
}

vdn_status vdn_frame_grams(const vdn_shape *s, const void *K, const void *V, const float *beta,
                           float *A, float *Bm, int32_t *info, vdn_stream_t stream) {
  g_err[0] = 0;
  Geo g;
  VDN_TRY(check_shape(s, &g));
  const bool any = g.BH * g.T > 0;
  VDN_TRY(need(K, "K", any && g.U > 0));
  VDN_TRY(need(V, "V", any && g.U > 0));
  VDN_TRY(need(beta, "beta", any && g.U > 0));
  VDN_TRY(need(A, "A", any));
  VDN_TRY(need(Bm, "Bm", any));
  return run_grams(g, K, V, beta, A, Bm, g.BH * g.T, g.U, info, (cudaStream_t)stream);
}

vdn_status vdn_frame_factor(const vdn_shape *s, const float *A, const float *Bm, const float *alpha,
                            float *M, float *J, int32_t *info, vdn_stream_t stream) {
  g_err[0] = 0;
  Geo g;
  VDN_TRY(check_shape(s, &g));
  const bool any = g.BH * g.T > 0;
  VDN_TRY(need(A, "A", any));
  VDN_TRY(need(Bm, "Bm", any));
  VDN_TRY(need(alpha, "alpha", any));
  VDN_TRY(need(M, "M", any));
  VDN_TRY(need(J, "J", any));
  VDN_TRY(need(info, "info", true));
  cudaStream_t st = (cudaStream_t)stream;
  VDN_CUDA(cudaMemsetAsync(info, 0, sizeof(int32_t), st), "memset info");
  VDN_CUDA(launch_factor_simt(A, Bm, alpha, M, J, info, g.BH * g.T, g.T, g.anchors, g.D, st),
           "factor");
  return VDN_OK;
}

vdn_status vdn_chunk_compose(const vdn_shape *s, const float *M, const float *J, float *Mf,
                             float *Jf, float *Mb, float *Jb, vdn_stream_t stream) {
  g_err[0] = 0;
  Geo g;
  VDN_TRY(check_shape(s, &g));
  const bool any = g.BH * g.T > 0;
  VDN_TRY(need(M, "M", any));
  VDN_TRY(need(J, "J", any));
  VDN_TRY(need(Mf, "Mf", any));
  VDN_TRY(need(Jf, "Jf", any));
  VDN_TRY(need(Mb, "Mb", any));
  VDN_TRY(need(Jb, "Jb", any));
  VDN_CUDA(launch_compose_simt(M, J, Mf, Jf, Mb, Jb, g.BH, g.T, g.chunk, g.D, (cudaStream_t)stream),
           "compose");
  return VDN_OK;
}

static vdn_status scan_common(const vdn_shape *s, const float *Mf, const float *Jf, const float *Mb,
                              const float *Jb, const float *S_T, float *F, float *G, int mask,
                              vdn_stream_t stream) {
  g_err[0] = 0;
  Geo g;
  VDN_TRY(check_shape(s, &g));
  const bool any = g.BH > 0;
  const bool fw = mask & 1, bw = mask & 2;
  VDN_TRY(need(S_T, "S_T", any));
  VDN_TRY(need(Mf, "Mf", any && fw && g.C > 0));
  VDN_TRY(need(Jf, "Jf", any && fw && g.C > 0));
  VDN_TRY(need(F, "F", any && fw));
  VDN_TRY(need(Mb, "Mb", any && bw && g.C > 0));
  VDN_TRY(need(Jb, "Jb", any && bw && g.C > 0));
  VDN_TRY(need(G, "G", any && bw));
  VDN_CUDA(launch_scan_simt(Mf, Jf, Mb, Jb, S_T, F, G, g.BH, g.C, g.D, mask, (cudaStream_t)stream),
           "scan");
  return VDN_OK;
}

vdn_status vdn_scan_fwd(const vdn_shape *s, const float *Mf, const float *Jf, const float *S_T,
                        float *F, vdn_stream_t stream) {
  return scan_common(s, Mf, Jf, nullptr, nullptr, S_T, F, nullptr, 1, stream);
}

vdn_status vdn_scan_bwd(const vdn_shape *s, const float *Mb, const float *Jb, const float *S_T,
                        float *G, vdn_stream_t stream) {
  return scan_common(s, nullptr, nullptr, Mb, Jb, S_T, nullptr, G, 2, stream);
}

vdn_status vdn_scan_bidir(const vdn_shape *s, const float *Mf, const float *Jf, const float *Mb,
                          const float *Jb, const float *S_T, float *F, float *G,
                          vdn_stream_t stream) {
  return scan_common(s, Mf, Jf, Mb, Jb, S_T, F, G, 3, stream);
}

vdn_status vdn_chunk_readout(const vdn_shape *s, const void *Q, const float *F, const float *G,
                             void *O, int32_t *info, vdn_stream_t stream) {
  g_err[0] = 0;
  Geo g;
  VDN_TRY(check_shape(s, &g));
  const bool any = g.BH * g.T * g.U > 0;
  VDN_TRY(need(Q, "Q", any));
  VDN_TRY(need(F, "F", any));
  VDN_TRY(need(G, "G", any));
  VDN_TRY(need(O, "O", any));
  if (g.bridge) return fail(VDN_ERR_INVALID, "decay_bridge needs alpha: use vdn_chunk_readout_bridged");
  return run_readout(g, Q, F, G, O, info, (cudaStream_t)stream);
}

vdn_status vdn_chunk_readout_gated(const vdn_shape *s, const void *Q, const float *F, const float *G,
                                   const vdn_out_gate *og, void *O, int32_t *info, vdn_stream_t stream) {
  g_err[0] = 0;
  Geo g;
  VDN_TRY(check_shape(s, &g));
  const bool any = g.BH * g.T * g.U > 0;
  VDN_TRY(need(Q, "Q", any));
  VDN_TRY(need(F, "F", any));
  VDN_TRY(need(G, "G", any));
  VDN_TRY(need(O, "O", any));
  if (g.bridge) return fail(VDN_ERR_INVALID, "decay_bridge needs alpha: use vdn_chunk_readout_bridged");
  OutGate og_;
  const OutGate *use;
  VDN_TRY(check_gate(g, og, false, &og_, &use));
  return run_readout(g, Q, F, G, O, info, (cudaStream_t)stream, use);
}

vdn_status vdn_chunk_readout_bridged(const vdn_shape *s, const void *Q, const float *F, const float *G,
                                     const float *alpha, const vdn_out_gate *og, void *O, int32_t *info,
                                     vdn_stream_t stream) {
  g_err[0] = 0;
  Geo g;
  VDN_TRY(check_shape(s, &g));
  if (!g.bridge) return fail(VDN_ERR_INVALID, "vdn_chunk_readout_bridged needs shape.decay_bridge = 1");
  const bool any = g.BH * g.T * g.U > 0;
  VDN_TRY(need(Q, "Q", any));
  VDN_TRY(need(F, "F", any));
  VDN_TRY(need(G, "G", any));
  VDN_TRY(need(alpha, "alpha", any));
  VDN_TRY(need(O, "O", any));
  OutGate og_;
  const OutGate *use;
  VDN_TRY(check_gate(g, og, true, &og_, &use));
  return run_readout(g, Q, F, G, O, info, (cudaStream_t)stream, use, nullptr, alpha);
}

size_t vdn_text_state_workspace_bytes(const vdn_shape *s) {
  Geo g;
  if (check_shape(s, &g) != VDN_OK) return 0;
  return text_layout(g).total;
}

vdn_status vdn_text_state(const vdn_shape *s, const void *Kx, const void *Vx, const float *beta_x,
                          float *S_T, void *workspace, size_t workspace_bytes, int32_t *info,
                          vdn_stream_t stream) {
  g_err[0] = 0;
  Geo g;
  VDN_TRY(check_shape(s, &g));
  const bool any = g.BH > 0;
  VDN_TRY(need(Kx, "Kx", any && g.n_text > 0));
  VDN_TRY(need(Vx, "Vx", any && g.n_text > 0));
  VDN_TRY(need(beta_x, "beta_x", any && g.n_text > 0));
  VDN_TRY(need(S_T, "S_T", any));
  VDN_TRY(need(info, "info", true));
  const size_t ws = vdn_text_state_workspace_bytes(s);
  VDN_TRY(need(workspace, "workspace", any && ws > 0));
  if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(VDN_ERR_INVALID, "workspace is not 256-byte aligned");
  if (workspace_bytes < ws)
    return fail(VDN_ERR_INVALID, "workspace of %zu bytes < %zu required", workspace_bytes, ws);
  cudaStream_t st = (cudaStream_t)stream;
  VDN_CUDA(cudaMemsetAsync(info, 0, sizeof(int32_t), st), "memset info");
  return run_text_state(g, Kx, Vx, beta_x, S_T, (char *)workspace, info, st);
}

vdn_status vdn_frame_invert(const vdn_shape *s, const float *A, float *W, int32_t *info,
                            vdn_stream_t stream) {
  g_err[0] = 0;
  Geo g;
  VDN_TRY(check_shape(s, &g));
  const bool any = g.BH * g.T > 0;
  VDN_TRY(need(A, "A", any));
  VDN_TRY(need(W, "W", any));
  VDN_TRY(need(info, "info", true));
  cudaStream_t st = (cudaStream_t)stream;
  VDN_CUDA(cudaMemsetAsync(info, 0, sizeof(int32_t), st), "memset info");
  if (tensor_path(g))
    VDN_CUDA(launch_invert_bsweep(A, W, nullptr, info, g.BH * g.T, st, 0), "invert");
  else
    VDN_CUDA(launch_invert_simt(A, W, nullptr, info, g.BH * g.T, g.D, st), "invert");
  return VDN_OK;
}

namespace {
struct FwdLayout {
  size_t text, st, a, b, wimg, pinv, mf, jf, mb, jb, mimg, f, g, total;
};
FwdLayout fwd_layout(const Geo &g) {
  FwdLayout L{};
  const size_t dd = (size_t)g.D * g.D * sizeof(float);
  const bool tc = tensor_path(g);
  size_t off = 0;
  auto take = [&](size_t n) {
    size_t o = off;
    off += align256(n);
    return o;
  };
  L.text = take(text_layout(g).total);
  L.st = take(g.BH * dd);
  L.a = take(g.BH * g.T * dd);
  L.b = take(g.BH * g.T * dd);
  L.wimg = take(tc ? (size_t)g.BH * g.T * kImgBytes : 0);
  L.pinv = take(tc ? (size_t)g.BH * g.T * kPinvBytes : 0);
  L.mf = take(g.BH * g.C * dd);
  L.jf = take(g.BH * g.C * dd);
  L.mb = take(g.BH * g.C * dd);
  L.jb = take(g.BH * g.C * dd);
  L.mimg = take(tc ? (size_t)g.BH * 2 * g.C * kImgBytes : 0);
  L.f = take(g.BH * (g.C + 1) * dd);
  L.g = take(g.BH * (g.C + 1) * dd);
  L.total = off;
  return L;
}
}  // namespace

size_t vdn_forward_workspace_bytes(const vdn_shape *s) {
  Geo g;
  if (check_shape(s, &g) != VDN_OK) return 0;
  return fwd_layout(g).total;
}

vdn_status vdn_forward(const vdn_shape *s, const void *Q, const void *K, const void *V,
                       const float *beta, const float *alpha, const void *Kx, const void *Vx,
                       const float *beta_x, void *O, float *F, float *G, void *workspace,
                       size_t workspace_bytes, int32_t *info, const void *const *stage_events,
                       const vdn_out_gate *og, vdn_stream_t stream) {
  g_err[0] = 0;
  Geo g;
  VDN_TRY(check_shape(s, &g));
  const bool frames = g.BH * g.T > 0;
  VDN_TRY(need(Q, "Q", frames && g.U > 0));
  VDN_TRY(need(K, "K", frames && g.U > 0));
  VDN_TRY(need(V, "V", frames && g.U > 0));
  VDN_TRY(need(beta, "beta", frames && g.U > 0));
  VDN_TRY(need(alpha, "alpha", frames));
  VDN_TRY(need(Kx, "Kx", g.BH > 0 && g.n_text > 0));
  VDN_TRY(need(Vx, "Vx", g.BH > 0 && g.n_text > 0));
  VDN_TRY(need(beta_x, "beta_x", g.BH > 0 && g.n_text > 0));
  VDN_TRY(need(O, "O", frames && g.U > 0));
  if ((F && !aligned16(F)) || (G && !aligned16(G)))
    return fail(VDN_ERR_INVALID, "F/G not 16-byte aligned");
  VDN_TRY(need(info, "info", true));
  OutGate gate_;
  const OutGate *gate;
  VDN_TRY(check_gate(g, og, true, &gate_, &gate));
  const FwdLayout L = fwd_layout(g);
  VDN_TRY(need(workspace, "workspace", g.BH > 0));
  if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(VDN_ERR_INVALID, "workspace is not 256-byte aligned");
  if (workspace_bytes < L.total)
    return fail(VDN_ERR_INVALID, "workspace of %zu bytes < %zu required", workspace_bytes, L.total);

  cudaStream_t st = (cudaStream_t)stream;
  auto mark = [&](int i) -> vdn_status {
    if (stage_events && stage_events[i]) {
      VDN_CUDA(cudaEventRecord((cudaEvent_t)stage_events[i], st), "event record");
    }
    return VDN_OK;
  };
  VDN_TRY(mark(0));
  if (g.BH == 0) {
    for (int i = 1; i < 7; ++i) VDN_TRY(mark(i));
    return VDN_OK;
  }
  char *w = (char *)workspace;
  float *S_T = (float *)(w + L.st);
  float *A = (float *)(w + L.a), *Bm = (float *)(w + L.b);
  uint8_t *Wimg = (uint8_t *)(w + L.wimg), *Mimg = (uint8_t *)(w + L.mimg);
  float *Mf = (float *)(w + L.mf), *Jf = (float *)(w + L.jf);
  float *Mb = (float *)(w + L.mb), *Jb = (float *)(w + L.jb);
  float *Fo = F ? F : (float *)(w + L.f);
  float *Go = G ? G : (float *)(w + L.g);
  const bool tc = tensor_path(g);

  VDN_CUDA(cudaMemsetAsync(info, 0, sizeof(int32_t), st), "memset info");
  VDN_TRY(run_text_state(g, Kx, Vx, beta_x, S_T, w + L.text, info, st));
  VDN_TRY(mark(1));
  float *Pinv = tc ? (float *)(w + L.pinv) : nullptr;
  if (frames) VDN_TRY(run_grams(g, K, V, beta, A, Bm, g.BH * g.T, g.U, info, st, Pinv));
  VDN_TRY(mark(2));
  if (frames) {
    if (tc) {
      VDN_CUDA(launch_invert_tc(A, Pinv, nullptr, Wimg, info, g.BH * g.T, st, 0), "invert");
    } else {
      // M and J overwrite A and Bm in place (each element is read and
      // written by the same thread).
      VDN_CUDA(launch_factor_simt(A, Bm, alpha, A, Bm, info, g.BH * g.T, g.T, g.anchors, g.D, st),
               "factor");
    }
  }
  VDN_TRY(mark(3));
  if (frames) {
    if (tc) {
      // the fp32 Mc are not needed here: the scan reads their images
      VDN_CUDA(launch_compose_tc(Wimg, Bm, alpha, nullptr, Jf, nullptr, Jb, Mimg, g.BH, g.T, g.chunk,
                                 g.anchors, 2, true, info, st),
               "compose");
    } else {
      VDN_CUDA(launch_compose_simt(A, Bm, Mf, Jf, Mb, Jb, g.BH, g.T, g.chunk, g.D, st), "compose");
    }
  }
  VDN_TRY(mark(4));
  if (tc && frames) {
    VDN_CUDA(launch_scan_tc(Mimg, Jf, Jb, S_T, Fo, Go, g.BH, g.C, info, st), "scan");
  } else {
    VDN_CUDA(launch_scan_simt(Mf, Jf, Mb, Jb, S_T, Fo, Go, g.BH, g.C, g.D, 3, st), "scan");
  }
  VDN_TRY(mark(5));
  if (frames) VDN_TRY(run_readout(g, Q, Fo, Go, O, info, st, gate, nullptr, alpha));
  VDN_TRY(mark(6));
  return VDN_OK;
}

size_t vdn_stream_workspace_bytes(const vdn_shape *s) { return vdn_forward_workspace_bytes(s); }

}  // extern "C"

namespace {
// One stream segment; `bridged` reads through the decay bridge (shape flag
// decay_bridge), with alpha_prev ([BH, d] or NULL = ones) the decay product of
// the previous segment's last chunk and alpha_tail ([BH, d] or NULL) receiving
// this segment's.
vdn_status stream_segment(const vdn_shape *s, const void *Q, const void *K, const void *V, const float *beta,
                          const float *alpha, long long frame0, const float *S_prev, const float *S_in,
                          const float *alpha_prev, void *O, float *F, float *alpha_tail, void *workspace,
                          size_t workspace_bytes, int32_t *info, vdn_stream_t stream, bool bridged) {
  g_err[0] = 0;
  Geo g;
  VDN_TRY(check_shape(s, &g));
  if (frame0 < 0 || frame0 % g.chunk != 0)
    return fail(VDN_ERR_INVALID, "frame0 = %lld is not a non-negative multiple of chunk = %d", frame0, g.chunk);
  if (g.bridge && !bridged)
    return fail(VDN_ERR_UNSUPPORTED,
                "decay_bridge: a segment's first chunk needs the previous segment's decay product: use "
                "vdn_stream_segment_bridged");
  if (bridged && !g.bridge) return fail(VDN_ERR_INVALID, "vdn_stream_segment_bridged needs shape.decay_bridge = 1");
  // only the stream's first frame can be an anchor; there is no last one
  g.anchors = (s->anchors && frame0 == 0) ? 1 : 0;
  const bool frames = g.BH * g.T > 0;
  VDN_TRY(need(Q, "Q", frames && g.U > 0));
  VDN_TRY(need(K, "K", frames && g.U > 0));
  VDN_TRY(need(V, "V", frames && g.U > 0));
  VDN_TRY(need(beta, "beta", frames && g.U > 0));
  VDN_TRY(need(alpha, "alpha", frames));
  VDN_TRY(need(S_prev, "S_prev", g.BH > 0));
  VDN_TRY(need(S_in, "S_in", g.BH > 0));
  VDN_TRY(need(O, "O", frames && g.U > 0));
  VDN_TRY(need(F, "F", g.BH > 0));
  VDN_TRY(need(info, "info", true));
  if ((alpha_prev && !aligned16(alpha_prev)) || (alpha_tail && !aligned16(alpha_tail)))
    return fail(VDN_ERR_INVALID, "alpha_prev / alpha_tail not 16-byte aligned");
  const FwdLayout L = fwd_layout(g);
  VDN_TRY(need(workspace, "workspace", g.BH > 0));
  if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(VDN_ERR_INVALID, "workspace is not 256-byte aligned");
  if (workspace_bytes < L.total)
    return fail(VDN_ERR_INVALID, "workspace of %zu bytes < %zu required", workspace_bytes, L.total);
  if (g.BH == 0) return VDN_OK;
  cudaStream_t st = (cudaStream_t)stream;
  char *w = (char *)workspace;
  float *A = (float *)(w + L.a), *Bm = (float *)(w + L.b);
  uint8_t *Wimg = (uint8_t *)(w + L.wimg), *Mimg = (uint8_t *)(w + L.mimg);
  float *Mf = (float *)(w + L.mf), *Jf = (float *)(w + L.jf);
  float *Mb = (float *)(w + L.mb), *Jb = (float *)(w + L.jb);
  const bool tc = tensor_path(g);
  VDN_CUDA(cudaMemsetAsync(info, 0, sizeof(int32_t), st), "memset info");
  if (frames) {
    float *Pinv = tc ? (float *)(w + L.pinv) : nullptr;
    VDN_TRY(run_grams(g, K, V, beta, A, Bm, g.BH * g.T, g.U, info, st, Pinv));
    if (tc) {
      VDN_CUDA(launch_invert_tc(A, Pinv, nullptr, Wimg, info, g.BH * g.T, st, 0), "invert");
      VDN_CUDA(launch_compose_tc(Wimg, Bm, alpha, nullptr, Jf, nullptr, nullptr, Mimg, g.BH, g.T, g.chunk,
                                 g.anchors, 1, true, info, st),
               "compose");
      VDN_CUDA(launch_scan_tc(Mimg, Jf, nullptr, S_in, F, nullptr, g.BH, g.C, info, st, /*dir_mask=*/1,
                              /*init_scale=*/1.f),
               "scan");
    } else {
      VDN_CUDA(launch_factor_simt(A, Bm, alpha, A, Bm, info, g.BH * g.T, g.T, g.anchors, g.D, st), "factor");
      VDN_CUDA(launch_compose_simt(A, Bm, Mf, Jf, Mb, Jb, g.BH, g.T, g.chunk, g.D, st), "compose");
      VDN_CUDA(launch_scan_simt(Mf, Jf, nullptr, nullptr, S_in, F, nullptr, g.BH, g.C, g.D, 1, st, 1.f), "scan");
    }
    VDN_TRY(run_readout(g, Q, F, nullptr, O, info, st, nullptr, S_prev, alpha, alpha_prev));
  } else {
    VDN_CUDA(launch_scan_simt(nullptr, nullptr, nullptr, nullptr, S_in, F, nullptr, g.BH, 0, g.D, 1, st, 1.f),
             "scan");
  }
  if (bridged && alpha_tail)
    VDN_CUDA(launch_bridge_tail(alpha, alpha_tail, g.BH, g.T, g.chunk, g.anchors, g.D, st), "bridge tail");
  return VDN_OK;
}
}  // namespace

extern "C" {

vdn_status vdn_stream_segment(const vdn_shape *s, const void *Q, const void *K, const void *V,
                              const float *beta, const float *alpha, long long frame0, const float *S_prev,
                              const float *S_in, void *O, float *F, void *workspace, size_t workspace_bytes,
                              int32_t *info, vdn_stream_t stream) {
  return stream_segment(s, Q, K, V, beta, alpha, frame0, S_prev, S_in, nullptr, O, F, nullptr, workspace,
                        workspace_bytes, info, stream, false);
}

vdn_status vdn_stream_segment_bridged(const vdn_shape *s, const void *Q, const void *K, const void *V,
                                      const float *beta, const float *alpha, long long frame0,
                                      const float *S_prev, const float *S_in, const float *alpha_prev, void *O,
                                      float *F, float *alpha_tail, void *workspace, size_t workspace_bytes,
                                      int32_t *info, vdn_stream_t stream) {
  return stream_segment(s, Q, K, V, beta, alpha, frame0, S_prev, S_in, alpha_prev, O, F, alpha_tail, workspace,
                        workspace_bytes, info, stream, true);
}

vdn_status vdn_forward_pipelined(const vdn_shape *s, const void *Q, const void *K, const void *V,
                                 const float *beta, const float *alpha, const void *Kx,
                                 const void *Vx, const float *beta_x, void *O, float *F, float *G,
                                 void *workspace, size_t workspace_bytes, int32_t *info,
                                 int32_t groups, vdn_stream_t aux, const void *const *events,
                                 const vdn_out_gate *og, vdn_stream_t stream) {
  g_err[0] = 0;
  Geo g;
  VDN_TRY(check_shape(s, &g));
  if (!tensor_path(g))
    return fail(VDN_ERR_UNSUPPORTED, "the pipelined pass needs bf16 inputs and output and d = 128");
  if (groups < 1 || groups > 64) return fail(VDN_ERR_INVALID, "groups = %d not in [1, 64]", groups);
  if (!events) return fail(VDN_ERR_INVALID, "events is NULL");
  for (int i = 0; i < 8 + groups; ++i)
    if (!events[i]) return fail(VDN_ERR_INVALID, "events[%d] is NULL", i);
  const bool frames = g.BH * g.T > 0;
  VDN_TRY(need(Q, "Q", frames && g.U > 0));
  VDN_TRY(need(K, "K", frames && g.U > 0));
  VDN_TRY(need(V, "V", frames && g.U > 0));
  VDN_TRY(need(beta, "beta", frames && g.U > 0));
  VDN_TRY(need(alpha, "alpha", frames));
  VDN_TRY(need(Kx, "Kx", g.BH > 0 && g.n_text > 0));
  VDN_TRY(need(Vx, "Vx", g.BH > 0 && g.n_text > 0));
  VDN_TRY(need(beta_x, "beta_x", g.BH > 0 && g.n_text > 0));
  VDN_TRY(need(O, "O", frames && g.U > 0));
  if ((F && !aligned16(F)) || (G && !aligned16(G)))
    return fail(VDN_ERR_INVALID, "F/G not 16-byte aligned");
  VDN_TRY(need(info, "info", true));
  OutGate gate_;
  const OutGate *gate;
  VDN_TRY(check_gate(g, og, true, &gate_, &gate));
  const FwdLayout L = fwd_layout(g);
  VDN_TRY(need(workspace, "workspace", g.BH > 0));
  if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(VDN_ERR_INVALID, "workspace is not 256-byte aligned");
  if (workspace_bytes < L.total)
    return fail(VDN_ERR_INVALID, "workspace of %zu bytes < %zu required", workspace_bytes, L.total);

  cudaStream_t st = (cudaStream_t)stream, ax = (cudaStream_t)aux;
  auto ev = [&](int i) { return (cudaEvent_t)events[i]; };
  char *w = (char *)workspace;
  float *S_T = (float *)(w + L.st);
  float *A = (float *)(w + L.a), *Bm = (float *)(w + L.b);
  uint8_t *Wimg = (uint8_t *)(w + L.wimg), *Mimg = (uint8_t *)(w + L.mimg);
  float *Pinv = (float *)(w + L.pinv);
  float *Jf = (float *)(w + L.jf), *Jb = (float *)(w + L.jb);
  float *Fo = F ? F : (float *)(w + L.f);
  float *Go = G ? G : (float *)(w + L.g);
  const long long T = g.T, U = g.U, DD = (long long)g.D * g.D, D = g.D;
  const int G_ = (int)(groups < g.BH ? groups : (g.BH > 0 ? g.BH : 1));
  auto lo = [&](int gi) { return g.BH * gi / G_; };
  auto tok = [&](const void *p, long long b0) { return (const char *)p + b0 * T * U * D * g.in_elem; };

  VDN_CUDA(cudaMemsetAsync(info, 0, sizeof(int32_t), st), "memset info");
  VDN_CUDA(cudaEventRecord(ev(0), st), "event record");
  // the text state on the auxiliary stream, beside the first Grams
  VDN_CUDA(cudaStreamWaitEvent(ax, ev(0), 0), "stream wait");
  VDN_CUDA(cudaEventRecord(ev(1), ax), "event record");
  VDN_TRY(run_text_state(g, Kx, Vx, beta_x, S_T, w + L.text, info, ax));
  VDN_CUDA(cudaEventRecord(ev(2), ax), "event record");
  // the Grams of every group on the main stream (their kernel also forms the
  // block inverse's P^{-1}, X^T and S). Their persistent grid leaves some SMs
  // to the text state: its kernels need TMEM, which a Gram CTA takes whole.
  const int spare = g.n_text > 0 ? (int)(g.BH < device_sm_count() / 12 ? g.BH : device_sm_count() / 12) : 0;
  for (int gi = 0; gi < groups; ++gi) {
    const bool run = gi < G_ && frames;
    const long long b0 = run ? lo(gi) : 0, nbh = run ? lo(gi + 1) - b0 : 0;
    if (run)
      VDN_TRY(run_grams(g, tok(K, b0), tok(V, b0), beta + b0 * T * (g.tokb ? U : 1), A + b0 * T * DD,
                        Bm + b0 * T * DD, nbh * T, (int)U, info, st, Pinv + b0 * T * (kPinvBytes / 4), b0 * T, spare));
    VDN_CUDA(cudaEventRecord(ev(3 + gi), st), "event record");
  }
  // the rest of the inverse, the composition, the scans and the readout over
  // all pairs once the auxiliary stream (the text state) is done: these are
  // latency-bound chains whose time grows if they are split
  const int tail = 3 + groups;
  VDN_CUDA(cudaStreamWaitEvent(st, ev(2), 0), "stream wait");
  VDN_CUDA(cudaEventRecord(ev(tail), st), "event record");
  if (frames)
    VDN_CUDA(launch_invert_tc(A, Pinv, nullptr, Wimg, info, g.BH * g.T, st, 0), "invert");
  VDN_CUDA(cudaEventRecord(ev(tail + 1), st), "event record");
  if (frames)
    VDN_CUDA(launch_compose_tc(Wimg, Bm, alpha, nullptr, Jf, nullptr, Jb, Mimg, g.BH, g.T, g.chunk, g.anchors,
                               2, true, info, st),
             "compose");
  VDN_CUDA(cudaEventRecord(ev(tail + 2), st), "event record");
  if (frames)
    VDN_CUDA(launch_scan_tc(Mimg, Jf, Jb, S_T, Fo, Go, g.BH, g.C, info, st), "scan");
  else if (g.BH > 0)
    VDN_CUDA(launch_scan_simt(nullptr, nullptr, nullptr, nullptr, S_T, Fo, Go, g.BH, g.C, g.D, 3, st), "scan");
  VDN_CUDA(cudaEventRecord(ev(tail + 3), st), "event record");
  if (frames) VDN_TRY(run_readout(g, Q, Fo, Go, O, info, st, gate, nullptr, alpha));
  VDN_CUDA(cudaEventRecord(ev(tail + 4), st), "event record");
  return VDN_OK;
}

}  // extern "C"
