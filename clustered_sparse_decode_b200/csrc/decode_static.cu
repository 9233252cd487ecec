// mp_decode_static: the decode step without a caller-provided scratch buffer.
//
// Some callers cannot allocate device memory when they decode: a serving
// engine that hands all free device memory to its own KV-cache pool at
// start-up has none left to give, and on a latency-critical path cudaMalloc /
// cudaFree may synchronise the whole device.  This entry point runs the same
// decode kernels with their scratch in a fixed array that lives inside the
// library instead (MP_STATIC_SCRATCH_BYTES, held on every device that loads
// the library until the process exits).  It allocates nothing.
#include <cmath>
#include <mutex>

#include "mp_internal.cuh"

namespace mp {

mp_status decode_impl(const mp_index* idx, const void* Q, void* O, const mp_decode_params* prm, void* scratch,
                      size_t scratch_bytes, cudaStream_t st);
size_t decode_scratch_bytes(const mp_config& c, int slots, int coarse_slots);

// The scratch itself.  Its name in host code is only a host-side handle of the
// symbol, never a device address: the address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_decode_scratch[MP_STATIC_SCRATCH_BYTES];

// The array's device address belongs to the module loaded in one CUDA
// context: it is looked up again whenever the device's current context is not
// the one it was looked up in (after cudaDeviceReset, or when the caller made
// another driver-API context current).
constexpr int kMaxDevices = 64;
static std::mutex g_scratch_mu;
static void* g_scratch_addr[kMaxDevices];   // device address of g_decode_scratch, per device ...
static void* g_scratch_ctx[kMaxDevices];    // ... in this context

using CtxGetCurrent = int (*)(void**);       // cuCtxGetCurrent(CUcontext*) of the driver API
static CtxGetCurrent ctx_get_current() {
  static CtxGetCurrent fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrent>(p);
  });
  return fn;
}

// Device address of the scratch on the current device and context.
static mp_status scratch_address(int dev, void** out) {
  if (dev < 0 || dev >= kMaxDevices) return MP_EUNSUPPORTED;
  CtxGetCurrent get = ctx_get_current();
  void* ctx = nullptr;
  if (!get || get(&ctx) != 0) return MP_ECUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!ctx || !g_scratch_addr[dev] || g_scratch_ctx[dev] != ctx) {
    // the lookup also makes the runtime's context current if none was
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return MP_ECUDA;
    if (!ctx && (get(&ctx) != 0 || !ctx)) return MP_ECUDA;
    g_scratch_addr[dev] = p;
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_addr[dev];
  return MP_OK;
}

}  // namespace mp

using namespace mp;

extern "C" mp_status mp_decode_static(const mp_index* idx, const void* Q, void* O, const mp_decode_params* p,
                                      void* stream) {
  if (!idx || !idx->workspace || !Q || !O || !p) return MP_EINVAL;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MP_ECUDA;
  if (dev != idx->device) return MP_EINVAL;
  if (p->reserved != 0 || p->reserved2 != 0 || p->n_split < 0 || p->n_split > 64) return MP_EINVAL;
  if (p->n_phase_events < 0 || (p->n_phase_events > 0 && !p->phase_events)) return MP_EINVAL;
  if (!std::isfinite(p->scale)) return MP_EINVAL;
  if ((p->flags & ~MP_NO_APPROX) != 0) return MP_EINVAL;
  // the configuration's scratch must fit in the fixed array
  if (decode_scratch_bytes(idx->cfg, idx->slots, idx->coarse_slots) > (size_t)MP_STATIC_SCRATCH_BYTES)
    return MP_ENOSPC;
  void* scratch = nullptr;
  mp_status s = scratch_address(dev, &scratch);
  if (s != MP_OK) return s;
  // Every byte of the array that a decode step reads was written earlier in
  // the same step: the array needs no initialisation and no reset.
  return decode_impl(idx, Q, O, p, scratch, MP_STATIC_SCRATCH_BYTES, static_cast<cudaStream_t>(stream));
}
