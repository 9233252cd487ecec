// Internal definitions shared by the library's translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "mpattn.h"

namespace mp {

// Byte offsets inside the index workspace (mp_index::layout).
enum Slot {
  S_KC = 0, S_VC, S_OFF, S_KP, S_VP, S_PERM, S_ASSIGN,   // the index proper
  S_KCC, S_VCC, S_COFF,                                  // levels == 2
  S_ERR,                                                 // device error word (int32)
  S_KCTMP, S_VCTMP,                                      // build scratch: centroid copies
  S_CASSIGN, S_CORDER, S_COFFTMP,                        // build scratch: coarse level
  S_BLKK, S_BLKV,                                        // update scratch: one block per unit
  S_MOVED,                                               // build scratch: per-block change counters
  S_COUNT
};

// Bits of the device error word.
enum DeviceError : int32_t {
  E_BAD_OFFSET = 1,     // a run offset or slot index outside the index
  E_BAD_LIST = 2,       // an internal run list inconsistent with its header
  E_TIMEOUT = 4,        // a bounded wait gave up
  E_CAPACITY = 8,       // a per-unit limit of a kernel was exceeded
};

constexpr int kWarp = 32;
constexpr unsigned kFull = 0xffffffffu;
constexpr float kLog2e = 1.4426950408889634f;

// Largest number of cluster slots per (batch, KV head) that one selection CTA
// holds in shared memory (keys, counts, rows: 12 bytes each).
constexpr int kMaxSlotsPerUnit = 16384;

template <typename T> struct DT;
template <> struct DT<float> { static constexpr int id = MP_F32; };
template <> struct DT<__nv_bfloat16> { static constexpr int id = MP_BF16; };

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Round an fp64 value to bf16, nearest-even, directly from fp64 (an fp32
// intermediate could round twice).  Written from the IEEE-754 formats: keep
// the sign, the 8-bit exponent range of fp32/bf16 and 7 stored fraction bits.
__device__ __forceinline__ __nv_bfloat16 bf16_rne_from_f64(double x) {
  uint64_t u = (uint64_t)__double_as_longlong(x);
  uint16_t sign = (uint16_t)((u >> 48) & 0x8000u);
  uint64_t mag = u & 0x7fffffffffffffffull;
  uint16_t out;
  if (mag > 0x7ff0000000000000ull) {                 // NaN
    out = sign | 0x7fc0u;
  } else {
    int e = (int)(mag >> 52) - 1023;                 // unbiased exponent
    if (e >= -126) {                                 // normal bf16 range (or overflow)
      // drop 45 fraction bits, ties to even; a carry may bump the exponent
      uint64_t lsb = (mag >> 45) & 1ull;
      uint64_t r = (mag + 0x0fffffffffffull + lsb) >> 45;   // sign-less, 18 bits: exp(11) + frac(7)
      int e2 = (int)(r >> 7) - 1023;
      if (e2 > 127) out = sign | 0x7f80u;            // overflow -> inf
      else out = sign | (uint16_t)(((e2 + 127) << 7) | (r & 0x7f));
    } else {                                         // bf16 subnormal or zero: multiples of 2^-133
      double a = fabs(x) * 0x1p133;                  // exact scaling by a power of two
      double q = rint(a);                            // nearest-even (default rounding mode)
      out = sign | (uint16_t)q;                      // q <= 128; 128 is the smallest normal
    }
  }
  return __ushort_as_bfloat16(out);
}

template <typename T> __device__ __forceinline__ T round_from_f64(double x);
template <> __device__ __forceinline__ float round_from_f64<float>(double x) { return __double2float_rn(x); }
template <> __device__ __forceinline__ __nv_bfloat16 round_from_f64<__nv_bfloat16>(double x) {
  return bf16_rne_from_f64(x);
}

// Order-preserving map of a float to uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t ordered_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
// the score of an ordered key (inverse of ordered_key)
__device__ __forceinline__ float key_score(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

__device__ __forceinline__ void set_error(int32_t* err, int32_t bit) {
  if (err) atomicOr(err, bit);
}

// Loads of DPL consecutive elements of a row (DPL * sizeof(T) bytes: 4, 8 or 16),
// through the read-only path, converted to fp32.
template <typename T, int DPL> struct RowChunk;
template <> struct RowChunk<__nv_bfloat16, 4> {
  uint2 raw;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) { raw = __ldg(reinterpret_cast<const uint2*>(p)); }
  __device__ __forceinline__ void zero() { raw = make_uint2(0u, 0u); }
  __device__ __forceinline__ float get(int i) const {
    uint32_t w = (i < 2) ? raw.x : raw.y;
    return __uint_as_float((i & 1) ? (w & 0xffff0000u) : (w << 16));
  }
};
template <> struct RowChunk<__nv_bfloat16, 2> {
  uint32_t raw;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) { raw = __ldg(reinterpret_cast<const uint32_t*>(p)); }
  __device__ __forceinline__ void zero() { raw = 0u; }
  __device__ __forceinline__ float get(int i) const {
    return __uint_as_float((i & 1) ? (raw & 0xffff0000u) : (raw << 16));
  }
};
template <> struct RowChunk<float, 4> {
  float4 raw;
  __device__ __forceinline__ void load(const float* p) { raw = __ldg(reinterpret_cast<const float4*>(p)); }
  __device__ __forceinline__ void zero() { raw = make_float4(0.f, 0.f, 0.f, 0.f); }
  __device__ __forceinline__ float get(int i) const {
    return i == 0 ? raw.x : i == 1 ? raw.y : i == 2 ? raw.z : raw.w;
  }
};
template <> struct RowChunk<float, 2> {
  float2 raw;
  __device__ __forceinline__ void load(const float* p) { raw = __ldg(reinterpret_cast<const float2*>(p)); }
  __device__ __forceinline__ void zero() { raw = make_float2(0.f, 0.f); }
  __device__ __forceinline__ float get(int i) const { return i == 0 ? raw.x : raw.y; }
};

}  // namespace mp

// Host-side helpers implemented in api.cu, used by the launchers.
namespace mp {
void* ws_ptr(const mp_index* idx, Slot s);
int elem_bytes(int dtype);
int32_t* err_word(const mp_index* idx);
}  // namespace mp
