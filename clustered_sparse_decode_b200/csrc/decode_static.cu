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

constexpr int kMaxDevices = 64;
static std::mutex g_scratch_mu;
static void* g_scratch_addr[kMaxDevices];   // device address of g_decode_scratch, per device

// Device address of the scratch on the current device; resolved on first use.
static mp_status scratch_address(int dev, void** out) {
  if (dev < 0 || dev >= kMaxDevices) return MP_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return MP_ECUDA;
    g_scratch_addr[dev] = p;
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
  // Apart from the ticket head (zero-initialised with the array and left zero
  // by every finished step), every byte a decode step reads was written
  // earlier in the same step.
  return decode_impl(idx, Q, O, p, scratch, MP_STATIC_SCRATCH_BYTES, static_cast<cudaStream_t>(stream));
}

extern "C" mp_status mp_decode_static_reset(void* stream) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MP_ECUDA;
  void* scratch = nullptr;
  mp_status s = scratch_address(dev, &scratch);
  if (s != MP_OK) return s;
  return cudaMemsetAsync(scratch, 0, kScratchTicketBytes, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MP_OK
                                                                                                        : MP_ECUDA;
}
