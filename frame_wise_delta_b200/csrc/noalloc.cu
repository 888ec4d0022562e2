// vdn_text_state_noalloc: the text-state computation of vdn_text_state
// without a caller workspace, for callers that cannot allocate device memory.
//
// Who needs it: callers that work under a fixed device-memory plan, such as a
// serving engine that reserves all of its memory at start-up and hands out no
// scratch afterwards, or a real-time loop that must not call cudaMalloc
// (which can synchronise the device and stall the other streams). They still
// pass their inputs and the output S_T; the two intermediate Gram matrices
// per (b, h) go to a fixed scratch array that this library holds in device
// memory instead.
//
// The scratch is a file-scope __device__ array of kScratchBytes (4 MiB). Every
// GPU that loads the library keeps it until the process exits. Host code must
// not pass the array's name to a kernel (on the host it only stands in for
// the symbol), so its device address is looked up with cudaGetSymbolAddress,
// with the device current, on the first call made on that device; make that
// first call before any stream capture. The address is kept per device
// together with the identity of the context it was looked up in: if that
// context has been destroyed and another created (cudaDeviceReset), the array
// was loaded again, possibly elsewhere, and the next call looks it up anew.
//
// All calls share the one array and it keeps the last call's contents.
// Nothing in it has to start at zero: the Gram kernels overwrite every element
// they later read. Calls whose kernels overlap on the GPU (other streams,
// other threads) race on the array and must be serialised by the caller.
#include <stdarg.h>
#include <stdio.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace {

constexpr size_t kScratchBytes = size_t(4) << 20;
constexpr size_t kScratchFloats = kScratchBytes / sizeof(float);
constexpr int kMaxDevices = 64;

__device__ __align__(256) float g_text_scratch[kScratchFloats];

// Report through vdn_last_error(), like every other entry point.
vdn_status fail(vdn_status st, const char *fmt, ...) {
  char msg[256];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(msg, sizeof(msg), fmt, ap);
  va_end(ap);
  vdn::set_last_error(msg);
  return st;
}

// Driver entry points for the identity of the current context (resolved once).
using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

void *driver_fn(const char *name) {
  void *p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return nullptr;
  return p;
}

// Unique id of the calling thread's current context, 0 if there is none (or
// the driver cannot tell): then nothing is cached.
unsigned long long current_context_id() {
  static std::once_flag once;
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  std::call_once(once, [] {
    get_current = reinterpret_cast<CtxGetCurrentFn>(driver_fn("cuCtxGetCurrent"));
    get_id = reinterpret_cast<CtxGetIdFn>(driver_fn("cuCtxGetId"));
  });
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of g_text_scratch on the current device, looked up once per
// device and context.
cudaError_t scratch_address(float **out) {
  static std::mutex mu;
  struct Slot {
    void *addr;
    unsigned long long ctx;
  };
  static Slot slot[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  const unsigned long long ctx = current_context_id();
  if (slot[dev].addr == nullptr || ctx == 0 || slot[dev].ctx != ctx) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_text_scratch);
    if (e != cudaSuccess) return e;
    // the lookup makes the device's primary context current if it was not yet
    slot[dev] = Slot{p, ctx != 0 ? ctx : current_context_id()};
  }
  *out = static_cast<float *>(slot[dev].addr);
  return cudaSuccess;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" vdn_status vdn_text_state_noalloc(const vdn_shape *s, const void *Kx, const void *Vx,
                                             const float *beta_x, float *S_T, int32_t *info,
                                             vdn_stream_t stream) {
  using namespace vdn;
  set_last_error("");
  // the same shape rules as vdn_text_state (and every other entry point)
  const vdn_status vs = validate_shape(s);
  if (vs != VDN_OK) return vs;
  const bool tokb = s->beta_per_token != 0;
  const long long BH = (long long)s->B * s->H;
  const int D = s->dk;
  const size_t per = (size_t)BH * D * D;  // floats of one Gram matrix set
  if (2 * per > kScratchFloats)
    return fail(VDN_ERR_UNSUPPORTED,
                "B*H*d*d = %zu floats needs %zu bytes of scratch; the fixed scratch holds %zu bytes "
                "(at most B*H*d*d = %zu)",
                per, 2 * per * sizeof(float), kScratchBytes, kScratchFloats / 2);
  if (BH > 0x7fffffffLL) return fail(VDN_ERR_UNSUPPORTED, "B*H too large");
  const bool any = BH > 0, text = any && s->n_text > 0;
  if (text && (!Kx || !Vx || !beta_x)) return fail(VDN_ERR_INVALID, "Kx, Vx and beta_x are required");
  if (any && !S_T) return fail(VDN_ERR_INVALID, "S_T is NULL");
  if (!info) return fail(VDN_ERR_INVALID, "info is NULL");
  if ((text && (!aligned16(Kx) || !aligned16(Vx) || !aligned16(beta_x))) || (S_T && !aligned16(S_T)))
    return fail(VDN_ERR_INVALID, "pointers must be 16-byte aligned");

  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(info, 0, sizeof(int32_t), st);
  if (e != cudaSuccess) return fail(VDN_ERR_CUDA, "memset info: %s", cudaGetErrorString(e));
  if (!any) return VDN_OK;
  if (s->n_text == 0) {
    e = cudaMemsetAsync(S_T, 0, per * sizeof(float), st);
    return e == cudaSuccess ? VDN_OK : fail(VDN_ERR_CUDA, "memset S_T: %s", cudaGetErrorString(e));
  }
  float *scratch = nullptr;
  e = scratch_address(&scratch);
  if (e != cudaSuccess) return fail(VDN_ERR_CUDA, "scratch address: %s", cudaGetErrorString(e));
  float *Ax = scratch;
  float *Bx = scratch + per;
  if (gram_tc_supported(s->in_dtype, D, s->n_text))
    e = launch_gram_tc(Kx, Vx, beta_x, tokb, Ax, Bx, BH, s->n_text, info, st);
  else
    e = launch_gram_simt(Kx, Vx, s->in_dtype, beta_x, tokb, Ax, Bx, BH, s->n_text, D, st);
  if (e != cudaSuccess) return fail(VDN_ERR_CUDA, "text gram: %s", cudaGetErrorString(e));
  e = launch_factor_simt(Ax, Bx, nullptr, nullptr, S_T, info, BH, 1, 0, D, st);
  if (e != cudaSuccess) return fail(VDN_ERR_CUDA, "text factor: %s", cudaGetErrorString(e));
  return VDN_OK;
}
