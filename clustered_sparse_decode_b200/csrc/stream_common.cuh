// Device building blocks of the streaming decode kernels: PTX wrappers for
// mbarriers, TMA and cp.async, the swizzled shared-memory layouts that TMA
// tile and box loads write, and the per-warp online softmax over 16-row tiles
// on mma.sync (bf16 in, fp32 accumulate).
#pragma once

#include <cuda.h>

#include "mp_internal.cuh"

namespace mp {
namespace sc {

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ long long gtimer() {
  long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// 16 bytes global -> shared; valid == false writes 16 zero bytes and reads nothing
__device__ __forceinline__ void cp16(uint32_t dst, const void* src, bool valid) {
  const int sz = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(sz) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }
// an arrival on the mbarrier once this thread's earlier cp.async have landed
// (counted as one of the barrier's expected arrivals)
__device__ __forceinline__ void cp_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_init(uint32_t bar, int count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint32_t bar, uint32_t tx) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(tx) : "memory");
}
// `count` arrivals at once
__device__ __forceinline__ void mbar_arrive_cnt(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
// raise the phase's expected transaction bytes without arriving
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t tx) {
  asm volatile("mbarrier.expect_tx.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(tx) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(10000000u)   // suspend up to 10 ms until the phase completes
      : "memory");
  return ok != 0;
}
// Wait for the phase of `bar` with parity `parity`; gives up (false) once the
// global timer passes `deadline` (ns).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, long long deadline) {
  // the global timer is read once every 64 polls: a poll is cheap, a timer read is not
  for (uint32_t i = 1;; ++i) {
    if (mbar_try(bar, parity)) return true;
    if ((i & 63u) == 0u && gtimer() > deadline) return false;
  }
}
// one tile of a 2-D tensor map (columns x, rows y) into shared memory
__device__ __forceinline__ void tma_2d(uint32_t dst, const CUtensorMap* tm, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }
__device__ __forceinline__ void ldsm4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ void ldsm4t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr)
               : "memory");
}
// D[16x8] += A[16x16] B[16x8], bf16 in, fp32 accumulate
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// 2^x by the SFU (ex2.approx: a few ulp, subnormal results flushed to zero); 2^-inf = 0
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }
__device__ __forceinline__ uint32_t movtrans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

// ---------------------------------------------------------------------------
// Shared-memory layouts of a chunk's key (or value) rows
// ---------------------------------------------------------------------------
// Tile layout (TMA 2-D tiles of 64 columns x R rows, 128-byte swizzle, at a
// 1024-byte aligned destination): D/64 tiles of [R rows][128 bytes]; within a
// tile 16-byte chunk c of row r sits at (c ^ (r & 7)).  Offset of chunk c
// (0 .. D/8 - 1) of row r.
template <int R>
__device__ __forceinline__ uint32_t tswz(int r, int c) {
  return (uint32_t)((c >> 3) * (R * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}
// Box layout: 8-row boxes, box b at b * 32 D bytes holding its key rows, then
// its value rows, each as D/64 1024-byte atoms [8 rows][128 bytes] (128-byte
// swizzle): what one TMA load of an 8-row box of the key and the value store
// writes.  Offset of chunk c of row r from the key (or value) part.
template <int D>
__device__ __forceinline__ uint32_t bswz(int r, int c) {
  return (r >> 3) * (32 * D) + (c >> 3) * 1024 + (r & 7) * 128 + (((c & 7) ^ (r & 7)) << 4);
}
template <bool BOX, int D, int R>
__device__ __forceinline__ uint32_t lay(int r, int c) {
  if constexpr (BOX) return bswz<D>(r, c);
  else return tswz<R>(r, c);
}

// ---------------------------------------------------------------------------
// Per-warp online softmax over 16-row tiles
// ---------------------------------------------------------------------------
// The 16 keys of a tile are the M rows of mma.sync m16n8k16 and 8 "columns"
// of query heads the N columns: S^T = K Q^T.  With G <= 4 the columns 4..7
// repeat the heads of columns 0..3, so that every probability exists twice;
// the lanes holding columns 0..3 pass its bf16 value (hi) and the lanes
// holding 4..7 the bf16 rounding of the remainder (lo) into P.V, which
// therefore keeps ~16 significant bits of each weight in one mma per 16 value
// columns (G = 8: the hi and lo parts go through two mma into the same
// accumulator).  The transpose from the S^T accumulator layout to the
// B-operand layout of P.V (keys as K) is movmatrix.trans on the packed pairs.
//
// The running max is lazy: a tile whose logits exceed this lane's max by at
// most 2^8 is folded with the old max (weights up to 256); only otherwise do
// the lanes of a column agree on a new max and rescale.
template <int D, int G>
struct WarpSoftmax {
  static constexpr bool DUP = G <= 4;
  static constexpr float kLazy = 8.f;
  uint32_t qb[D / 16][2];      // B fragments of Q^T: [k-step][dims +0 | +8], column lane/4
  float acc[D / 16][4];        // numerator O^T: m-tile mt holds [d = 16 mt + lane/4 (+8)][column 2*(lane%4) (+1)]
  float m[2], l[2];            // running max (log2 units) and normaliser of this lane's two columns

  // the head of column 2 (lane % 4) + j, or -1 for an unused column
  __device__ static __forceinline__ int col_head(int lane, int j) {
    const int col = 2 * (lane & 3) + j;
    const int h = DUP ? (col & 3) : col;
    return h < G ? h : -1;
  }
  __device__ static __forceinline__ bool lo_cols(int lane) { return DUP && (lane & 3) >= 2; }
  // row of z[i][.] within the warp's 16
  __device__ static __forceinline__ int zrow(int lane, int i) { return (lane >> 2) + 8 * i; }

  __device__ __forceinline__ void reset() {
    m[0] = m[1] = -1e30f;
    l[0] = l[1] = 0.f;
#pragma unroll
    for (int n = 0; n < D / 16; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  }
  template <typename P>
  __device__ __forceinline__ void load_q(const P* q, int lane) {   // q: [G][D] bf16
    const int n = lane >> 2;
    const int h = DUP ? (n & 3) : n;
    const uint32_t* qs = reinterpret_cast<const uint32_t*>(q);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      qb[ks][0] = h < G ? qs[(h * D + ks * 16 + 2 * (lane & 3)) >> 1] : 0u;
      qb[ks][1] = h < G ? qs[(h * D + ks * 16 + 8 + 2 * (lane & 3)) >> 1] : 0u;
    }
  }
  // raw dot products of the tile's 16 keys with the columns: z[i][j] = key zrow(lane, i), column 2 (lane % 4) + j
  template <bool BOX, int R>
  __device__ __forceinline__ void qk(uint32_t kb, int r16, int lane, float (&z)[2][2]) const {
    float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};   // two accumulation chains
    const int row = r16 + (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t a0, a1, a2, a3;
      ldsm4(kb + lay<BOX, D, R>(row, 2 * ks + (lane >> 4)), a0, a1, a2, a3);
      if (ks & 1) mma16816(c1, a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
      else mma16816(c0, a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
    }
    z[0][0] = c0[0] + c1[0];
    z[0][1] = c0[1] + c1[1];
    z[1][0] = c0[2] + c1[2];
    z[1][1] = c0[3] + c1[3];
  }
  // Fold a tile with logits z (log2 units, -inf = no term) and weight sign into
  // the state: O^T += V^T P^T, the value rows' transpose as the A operand.
  template <bool BOX, int R>
  __device__ __forceinline__ void update(uint32_t vb, int r16, int lane, float (&z)[2][2], float sign) {
    const bool need = fmaxf(z[0][0], z[1][0]) > m[0] + kLazy || fmaxf(z[0][1], z[1][1]) > m[1] + kLazy;
    if (__any_sync(kFull, need)) {
      float t0 = fmaxf(z[0][0], z[1][0]), t1 = fmaxf(z[0][1], z[1][1]);
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        t0 = fmaxf(t0, __shfl_xor_sync(kFull, t0, o));
        t1 = fmaxf(t1, __shfl_xor_sync(kFull, t1, o));
      }
      const float n0 = fmaxf(m[0], t0), n1 = fmaxf(m[1], t1);
      const float a0 = ex2(m[0] - n0), a1 = ex2(m[1] - n1);
      m[0] = n0;
      m[1] = n1;
      l[0] *= a0;
      l[1] *= a1;
#pragma unroll
      for (int n = 0; n < D / 16; ++n) { acc[n][0] *= a0; acc[n][1] *= a1; acc[n][2] *= a0; acc[n][3] *= a1; }
    }
    float p[2][2];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 2; ++j) p[i][j] = sign * ex2(z[i][j] - m[j]);
    l[0] += p[0][0] + p[1][0];
    l[1] += p[0][1] + p[1][1];
    const uint32_t h0 = pack_bf16(p[0][0], p[0][1]);    // keys 0..7 of the tile (row lane/4)
    const uint32_t h1 = pack_bf16(p[1][0], p[1][1]);    // keys 8..15
    const uint32_t l0 = pack_bf16(p[0][0] - bf16_lo(h0), p[0][1] - bf16_hi(h0));
    const uint32_t l1 = pack_bf16(p[1][0] - bf16_lo(h1), p[1][1] - bf16_hi(h1));
    uint32_t b0, b1, c0 = 0u, c1 = 0u;
    if constexpr (DUP) {
      const bool lo = lo_cols(lane);
      b0 = movtrans(lo ? l0 : h0);
      b1 = movtrans(lo ? l1 : h1);
    } else {
      b0 = movtrans(h0);
      b1 = movtrans(h1);
      c0 = movtrans(l0);
      c1 = movtrans(l1);
    }
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      uint32_t v0, v1, v2, v3;
      ldsm4t(vb + lay<BOX, D, R>(r16 + (lane & 7) + 8 * (lane >> 4), 2 * mt + ((lane >> 3) & 1)), v0, v1, v2, v3);
      mma16816(acc[mt], v0, v1, v2, v3, b0, b1);
      if constexpr (!DUP) mma16816(acc[mt], v0, v1, v2, v3, c0, c1);
    }
  }
  // This warp's state as one partial: pm[G] (max, log2 units; -inf when the
  // normaliser is 0), pl[G] (normaliser), pacc[G][D] (numerator).  Generic
  // pointers: shared or global memory.
  __device__ __forceinline__ void store(float* pm, float* pl, float* pacc, int lane) const {
    float lt0 = l[0], lt1 = l[1];
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      lt0 += __shfl_xor_sync(kFull, lt0, o);
      lt1 += __shfl_xor_sync(kFull, lt1, o);
    }
    const bool wr = !lo_cols(lane);
    const int hd0 = col_head(lane, 0), hd1 = col_head(lane, 1), d0 = lane >> 2;
    if (wr && lane < 4) {
      if (hd0 >= 0) { pm[hd0] = lt0 != 0.f ? m[0] : -INFINITY; pl[hd0] = lt0; }
      if (hd1 >= 0) { pm[hd1] = lt1 != 0.f ? m[1] : -INFINITY; pl[hd1] = lt1; }
    }
    float* o0 = pacc + (hd0 < 0 ? 0 : hd0) * D + d0;
    float* o1 = pacc + (hd1 < 0 ? 0 : hd1) * D + d0;
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      float v[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[e] = acc[mt][e];
        if constexpr (DUP) v[e] += __shfl_xor_sync(kFull, acc[mt][e], 2);   // + the lo part of the same head
      }
      if (wr && hd0 >= 0) { o0[16 * mt] = v[0]; o0[16 * mt + 8] = v[2]; }
      if (wr && hd1 >= 0) { o1[16 * mt] = v[1]; o1[16 * mt + 8] = v[3]; }
    }
  }
};

}  // namespace sc
}  // namespace mp
