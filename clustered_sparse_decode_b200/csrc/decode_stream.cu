// Flat decode step for bf16 caches: a centroid pass and a value pass.
//
// "Multipole Attention for Efficient Long Context Reasoning" (arXiv abstract;
// atlas.scime summary, "Approach"): the query scores every key centroid, the
// best clusters up to a token budget are attended exactly, and every other
// cluster enters the same softmax as one term with logit score + ln(size) and
// its value centroid.
//
//   centroid pass  one CTA per 128 cluster slots of a (batch, KV head) unit:
//                  S[c][g] = scale * q_g . Kc_c for the G query heads (written
//                  to scratch) and one online-softmax partial over the centroid
//                  terms of ALL clusters of the range (logit S + ln n_c, value
//                  Vc_c).  The CTA that finishes a unit's last range runs the
//                  unit's budgeted selection and writes its value stream.
//   value pass     (programmatic dependent launch) CTAs over each unit's value
//                  stream: the exact rows (tokens of the selected clusters in
//                  slot order, then the un-clustered tail), then one row per
//                  selected cluster that SUBTRACTS its centroid term again, so
//                  that the centroid partials keep only the unselected
//                  clusters.  The CTA that finishes a unit's last range merges
//                  all partials of the unit into its output rows.
// The large centroid stream never waits for a selection.  Subtracting is safe
// in fp32: a selected centroid term n e^{q.Kc} is at most the exact mass of its
// cluster (Jensen, Kc being the member mean), so the cancellation error stays a
// few ulps of the final normaliser.
//
// Data movement: a centroid CTA loads its 128 contiguous Kc and Vc rows as TMA
// tiles (64 columns x 128 rows, 128-byte swizzle) at once; a value CTA's warps
// each gather their own 32 rows with cp.async (16-byte chunks, written in the
// same swizzled layout).  Three CTAs per SM keep ~200 KB of loads in flight
// without a software pipeline.  Compute: mma.sync m16n8k16 (bf16 in, fp32
// accumulate) with the G query heads as the M rows (G of 16 used) and 8 keys
// as the N columns; the probabilities enter P.V as a bf16 hi + lo pair, so the
// weights keep ~16 significant bits.  The contraction is small next to the
// bytes streamed: the tensor cores only keep the instructions per byte low.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdio>
#include <mutex>

#include "mp_internal.cuh"

namespace mp {
namespace stream {

constexpr int kW = 4;                         // warps per CTA
constexpr int kT = kW * kWarp;                // threads per CTA
constexpr int kRows = 128;                    // rows of a CTA's range (32 per warp)
constexpr int kTile = kRows * 128;            // one 64-column tile of the range (bytes)
constexpr int kMaxSpt = 32;                   // selection: slots per thread (slots <= 4096)
constexpr int kMaxItems = 64;                 // partials per unit and pass, each
constexpr int kMaxSlots = kMaxSpt * kT;

struct Args {
  CUtensorMap tmKc;            // Kc as [units*slots rows][D] bf16: 64 x 128 tiles, 128-byte swizzle
  CUtensorMap tmVc;
  const __nv_bfloat16* Q;      // [units*G][D]
  __nv_bfloat16* O;            // [units*G][D]
  const __nv_bfloat16* Vc;     // [units][slots][D]
  const __nv_bfloat16* Kp;     // [units][max_tokens][D]
  const __nv_bfloat16* Vp;
  const int32_t* off;          // [units][slots + 1]
  int units, slots, slots_active;
  int64_t max_tokens;
  int n_clustered, n_tail;
  float scale;                 // score scale, natural-log units
  int budget, approx;
  int NA, NB;                  // centroid / value CTAs per unit
  int capc;                    // selected-cluster capacity per unit
  float* S;                    // [units][slots][SG] scores (natural units), rows padded to 16 bytes
  int32_t* tok_src;            // [units][max_tokens] store row of each exact row of the value stream
  int32_t* sub_src;            // [units][capc] slot of each selected cluster (subtraction rows)
  float* sub_bias;             // [units][capc] log2 of its size
  int32_t* hdr;                // [units][2]: exact rows, subtraction rows
  float* pm;                   // [units][NA + NB][G] partial max (log2 units)
  float* pl;                   // [units][NA + NB][G] partial normaliser
  float* pacc;                 // [units][NA + NB][G][D] partial numerator
  int32_t* ctl;                // [u] centroid tickets; [U + u] value tickets
  uint8_t* sel_mask_out;       // optional [units][slots]
  float* scores_out;           // optional [units][slots]
  int32_t* err;
  long long timeout_ns;
};

template <int D, int G>
struct Geo {
  static constexpr int SG = (G + 3) / 4 * 4;           // floats per score row (16-byte multiple)
  static constexpr int CPR = D / 8;                    // 16-byte chunks per bf16 row
  static constexpr int AREA = kRows * D * 2;           // key (or value) rows: D/64 tiles
  static constexpr int OFF_V = AREA;
  static constexpr int OFF_AUX = 2 * AREA;             // offsets / row sources / biases (kRows + 4 ints)
  static constexpr int OFF_RED = OFF_AUX + (kRows + 4) * 4;
  static constexpr int OFF_BAR = OFF_RED + 64 * 4;
  static constexpr int SMEM = OFF_BAR + 16 + 1024;     // + alignment slack
  static constexpr int MERGE = kW * G * (D + 2) * 4;   // per-warp partials, in the key area at the end
  static_assert(D % 64 == 0, "rows are whole 64-column tiles");
  static_assert(kRows * SG * 4 <= AREA, "subtraction-row scores live in the key area");
  static_assert(MERGE <= AREA, "the merge buffer reuses the key area");
  static_assert(SMEM * 3 + 3 * 1024 <= 233472, "three CTAs per SM");
};

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
__device__ __forceinline__ void cp16(uint32_t dst, const void* src, bool valid) {
  const int sz = valid ? 16 : 0;   // 0: no global read, the 16 bytes are zero-filled
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(sz) : "memory");
}
__device__ __forceinline__ void cp_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }
__device__ __forceinline__ void mbar_init(uint32_t bar, int count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint32_t bar, uint32_t tx) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(tx) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// one 64-column x kRows-row tile of a 2-D tensor map into shared memory
__device__ __forceinline__ void tma_tile(uint32_t dst, const CUtensorMap* tm, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
// ticket: returns the old value; release orders this CTA's earlier writes (made
// visible to this thread by the preceding CTA barrier) before the increment,
// acquire orders the winner's later reads after it
__device__ __forceinline__ int ticket(int32_t* p) {
  int v;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;\n" : "=r"(v) : "l"(p) : "memory");
  return v;
}
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
// D[16x8] += A[16x16] B[16x8], bf16 in, fp32 accumulate.  Only rows 0..7 of A
// (the query heads) are non-zero, so only the two accumulators of those rows
// are kept; a1 = a3 = 0 and the row-8..15 accumulators are discarded.
__device__ __forceinline__ void mma16816(float& d0, float& d1, uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  [[maybe_unused]] float x2, x3;
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%11,%12,%13};\n"
      : "=f"(d0), "=f"(d1), "=f"(x2), "=f"(x3)
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1), "f"(d0), "f"(d1), "f"(0.f), "f"(0.f));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// Byte offset of 16-byte chunk c of row r inside a key or value area: the area
// holds D/64 tiles of [kRows rows][128 bytes]; within a tile the chunk index is
// XORed with the row's low 3 bits, which is the layout a TMA tile load with
// 128-byte swizzle writes to a 1024-byte aligned destination.
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return (uint32_t)((c >> 3) * kTile + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// ---------------------------------------------------------------------------
// Per-warp online softmax over 16-row tiles
// ---------------------------------------------------------------------------
template <int D, int G>
struct WarpSoftmax {
  uint32_t qa[D / 16][2];      // A fragments of the query heads (rows 0..7), k-steps of 16
  float acc[D / 8][2];         // numerator: head lane/4, columns n*8 + 2*(lane%4) + {0,1}
  float m, l;                  // running max (log2 units) and normaliser (this lane's share)

  __device__ __forceinline__ void reset() {
    m = -INFINITY;
    l = 0.f;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) acc[n][0] = acc[n][1] = 0.f;
  }
  __device__ __forceinline__ void load_q(const __nv_bfloat16* q, int lane) {
    const int hq = lane >> 2;
    const uint32_t* qs = reinterpret_cast<const uint32_t*>(q);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      qa[ks][0] = hq < G ? __ldg(qs + ((hq * D + ks * 16 + 2 * (lane & 3)) >> 1)) : 0u;
      qa[ks][1] = hq < G ? __ldg(qs + ((hq * D + ks * 16 + 8 + 2 * (lane & 3)) >> 1)) : 0u;
    }
  }
  // raw dot products q_g . k for the 16 rows of a tile (this lane: head lane/4, rows 2*(lane%4) + {0,1} + 8*nt)
  __device__ __forceinline__ void qk(uint32_t kb, int r16, int lane, float (&z)[2][2]) const {
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      float c0 = 0.f, c1 = 0.f, e0 = 0.f, e1 = 0.f;   // two accumulation chains
#pragma unroll
      for (int kc = 0; kc < D / 32; ++kc) {
        uint32_t b0, b1, b2, b3;
        ldsm4(kb + swz(r16 + nt * 8 + (lane & 7), 4 * kc + (lane >> 3)), b0, b1, b2, b3);
        mma16816(c0, c1, qa[2 * kc][0], qa[2 * kc][1], b0, b1);
        mma16816(e0, e1, qa[2 * kc + 1][0], qa[2 * kc + 1][1], b2, b3);
      }
      z[nt][0] = c0 + e0;
      z[nt][1] = c1 + e1;
    }
  }
  // fold a tile with logits z (log2 units, -inf = no term) and weight sign into the state
  __device__ __forceinline__ void update(uint32_t vb, int r16, int lane, float (&z)[2][2], float sign) {
    float mx = fmaxf(fmaxf(z[0][0], z[0][1]), fmaxf(z[1][0], z[1][1]));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
    const float mnew = fmaxf(m, mx);
    if (!__any_sync(kFull, mnew != -INFINITY)) return;
    float pr[2][2];
    float alpha = 1.f;
    if (mnew == -INFINITY) {
      pr[0][0] = pr[0][1] = pr[1][0] = pr[1][1] = 0.f;
    } else {
      alpha = exp2f(m - mnew);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int i = 0; i < 2; ++i) pr[nt][i] = sign * exp2f(z[nt][i] - mnew);
    }
    m = mnew;
    l = l * alpha + ((pr[0][0] + pr[0][1]) + (pr[1][0] + pr[1][1]));
    if (__any_sync(kFull, alpha != 1.f)) {
#pragma unroll
      for (int n = 0; n < D / 8; ++n) { acc[n][0] *= alpha; acc[n][1] *= alpha; }
    }
    const uint32_t h0 = pack_bf16(pr[0][0], pr[0][1]);
    const uint32_t h1 = pack_bf16(pr[1][0], pr[1][1]);
    const uint32_t l0 = pack_bf16(pr[0][0] - bf16_lo(h0), pr[0][1] - bf16_hi(h0));
    const uint32_t l1 = pack_bf16(pr[1][0] - bf16_lo(h1), pr[1][1] - bf16_hi(h1));
#pragma unroll
    for (int n2 = 0; n2 < D / 16; ++n2) {
      uint32_t v0, v1, v2, v3;
      ldsm4t(vb + swz(r16 + (lane & 7) + 8 * ((lane >> 3) & 1), 2 * n2 + (lane >> 4)), v0, v1, v2, v3);
      mma16816(acc[2 * n2][0], acc[2 * n2][1], h0, h1, v0, v1);
      mma16816(acc[2 * n2 + 1][0], acc[2 * n2 + 1][1], h0, h1, v2, v3);
      mma16816(acc[2 * n2][0], acc[2 * n2][1], l0, l1, v0, v1);
      mma16816(acc[2 * n2 + 1][0], acc[2 * n2 + 1][1], l0, l1, v2, v3);
    }
  }
};

// Merge the kW warps' states through shared memory (buf: MERGE bytes) and write
// the CTA's partial j of unit u.  Called by all threads; ends with a barrier.
template <int D, int G>
__device__ void write_partial(const Args& a, WarpSoftmax<D, G>& ws, float* buf, int u, int j) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, hq = lane >> 2;
  float* mbuf = buf;                 // [kW][G]
  float* lbuf = mbuf + kW * G;       // [kW][G]
  float* abuf = lbuf + kW * G;       // [kW][G][D]
  float lt = ws.l;
  lt += __shfl_xor_sync(kFull, lt, 1);
  lt += __shfl_xor_sync(kFull, lt, 2);
  if (hq < G) {
    if ((lane & 3) == 0) {
      mbuf[warp * G + hq] = ws.m;
      lbuf[warp * G + hq] = lt;
    }
#pragma unroll
    for (int n = 0; n < D / 8; ++n)
      *reinterpret_cast<float2*>(abuf + (size_t)(warp * G + hq) * D + n * 8 + 2 * (lane & 3)) =
          make_float2(ws.acc[n][0], ws.acc[n][1]);
  }
  __syncthreads();
  const size_t pbase = ((size_t)u * (a.NA + a.NB) + j) * G;
  for (int e = threadIdx.x; e < G * D / 4; e += kT) {
    const int g = (e * 4) / D, d = (e * 4) % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kW; ++w) M = fmaxf(M, mbuf[w * G + g]);
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < kW; ++w) {
      const float mw = mbuf[w * G + g];
      const float f = mw == -INFINITY ? 0.f : exp2f(mw - M);
      const float4 x = *reinterpret_cast<const float4*>(abuf + (size_t)(w * G + g) * D + d);
      o.x += f * x.x; o.y += f * x.y; o.z += f * x.z; o.w += f * x.w;
      L += f * lbuf[w * G + g];
    }
    *reinterpret_cast<float4*>(a.pacc + (pbase + g) * D + d) = o;
    if (d == 0) {
      a.pm[pbase + g] = M;
      a.pl[pbase + g] = L;
    }
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------
// Block-wide helpers (red: 64 ints)
// ---------------------------------------------------------------------------
__device__ __forceinline__ int bsum(int v, int* red, int& par) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  v = __reduce_add_sync(kFull, v);
  int* r = red + par * kW;
  if (lane == 0) r[warp] = v;
  __syncthreads();
  int t = 0;
#pragma unroll
  for (int i = 0; i < kW; ++i) t += r[i];
  par ^= 1;
  return t;
}

// exclusive scan of two ints over the threads in thread order; returns totals
__device__ __forceinline__ void bscan2(int a, int b, int& ea, int& eb, int& ta, int& tb, int* red) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int ia = a, ib = b;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int xa = __shfl_up_sync(kFull, ia, o), xb = __shfl_up_sync(kFull, ib, o);
    if (lane >= o) { ia += xa; ib += xb; }
  }
  int* r = red + 2 * kW;
  if (lane == 31) { r[warp] = ia; r[kW + warp] = ib; }
  __syncthreads();
  int pa = 0, pb = 0;
  ta = 0; tb = 0;
#pragma unroll
  for (int i = 0; i < kW; ++i) {
    if (i < warp) { pa += r[i]; pb += r[kW + i]; }
    ta += r[i]; tb += r[kW + i];
  }
  ea = pa + ia - a;
  eb = pb + ib - b;
  __syncthreads();   // r[] is reused by the next scan
}

// ---------------------------------------------------------------------------
// Selection of one unit (all threads of the CTA that finished the unit's last
// centroid range).  Token-budgeted: clusters by score descending, ties to the
// lower slot, shortest prefix whose token count reaches the budget (the
// crossing cluster whole); budget <= 0 selects nothing, a budget at or above
// all clustered tokens selects every non-empty cluster.  The threshold is
// found exactly by a bitwise search over the order-preserving uint32 image of
// the group scores: the largest key tau with W(key >= tau) >= budget.
// ---------------------------------------------------------------------------
template <int G, int SG>
__device__ void select_unit(const Args& a, int u, int* red) {
  const int tid = threadIdx.x;
  const int slots = a.slots;
  const int spt = (slots + kT - 1) / kT;
  const int s0 = tid * spt;
  const int32_t* offu = a.off + (size_t)u * (slots + 1);
  const float* Su = a.S + (size_t)u * slots * SG;
  int par = 0;

  uint32_t key[kMaxSpt];
  int w[kMaxSpt];
  int wsum = 0;
  // loads in batches of 8 slots, unconditional (clamped) so that they issue back to back
#pragma unroll
  for (int k0 = 0; k0 < kMaxSpt; k0 += 8) {
    if (k0 < spt) {
      int o[9];
      float4 sv[8][SG / 4];
#pragma unroll
      for (int k = 0; k <= 8; ++k) o[k] = __ldg(offu + min(s0 + k0 + k, slots));
#pragma unroll
      for (int k = 0; k < 8; ++k)
#pragma unroll
        for (int h = 0; h < SG / 4; ++h)
          sv[k][h] = __ldcg(reinterpret_cast<const float4*>(Su + (size_t)min(s0 + k0 + k, slots - 1) * SG) + h);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int c = s0 + k0 + k;
        const bool in = k0 + k < spt && c < slots;
        const int cnt = in ? o[k + 1] - o[k] : 0;
        float sh = -INFINITY;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float4 v4 = sv[k][g >> 2];
          const float x = (g & 3) == 0 ? v4.x : (g & 3) == 1 ? v4.y : (g & 3) == 2 ? v4.z : v4.w;
          sh = fmaxf(sh, x);
        }
        key[k0 + k] = cnt > 0 ? ordered_key(sh) : 0u;
        w[k0 + k] = cnt > 0 ? cnt : 0;
        wsum += w[k0 + k];
        if (in && a.scores_out) a.scores_out[(size_t)u * slots + c] = cnt > 0 ? sh : -INFINITY;
      }
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) { key[k0 + k] = 0u; w[k0 + k] = 0; }
    }
  }
  const int W = bsum(wsum, red, par);
  // mode 0: none, 1: all non-empty clusters, 2: threshold
  const int mode = (a.budget <= 0 || W == 0) ? 0 : (W <= a.budget ? 1 : 2);
  uint32_t tau = 0u;
  int need = 0;
  if (mode == 2) {
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = tau | (1u << bit);
      int part = 0;
#pragma unroll
      for (int k = 0; k < kMaxSpt; ++k) part += key[k] >= cand ? w[k] : 0;
      if (bsum(part, red, par) >= a.budget) tau = cand;
    }
    int above = 0;
#pragma unroll
    for (int k = 0; k < kMaxSpt; ++k) above += key[k] > tau ? w[k] : 0;
    need = a.budget - bsum(above, red, par);   // >= 1 tokens still to take among the ties at tau
  }
  int tw = 0;
  if (mode == 2) {
#pragma unroll
    for (int k = 0; k < kMaxSpt; ++k) tw += (key[k] == tau && w[k] > 0) ? w[k] : 0;
  }
  int tie_before, e2, t1, t2;
  bscan2(tw, 0, tie_before, e2, t1, t2, red);
  uint32_t selbits = 0u;
  int ntok = 0, nsel = 0;
#pragma unroll
  for (int k = 0; k < kMaxSpt; ++k) {
    if (w[k] > 0) {
      bool s = false;
      if (mode == 1) s = true;
      else if (mode == 2) {
        if (key[k] > tau) s = true;
        else if (key[k] == tau) { s = tie_before < need; tie_before += w[k]; }
      }
      if (s) { selbits |= 1u << k; ntok += w[k]; ++nsel; }
    }
  }
  int tok_base, sub_base, tok_total, sel_total;
  bscan2(ntok, nsel, tok_base, sub_base, tok_total, sel_total, red);

  int32_t* tsrc = a.tok_src + (size_t)u * a.max_tokens;
  int32_t* ssrc = a.sub_src + (size_t)u * a.capc;
  float* sbias = a.sub_bias + (size_t)u * a.capc;
#pragma unroll
  for (int k = 0; k < kMaxSpt; ++k) {
    const int c = s0 + k;
    if (k < spt && c < slots) {
      const bool s = (selbits >> k) & 1u;
      if (a.sel_mask_out) a.sel_mask_out[(size_t)u * slots + c] = s ? 1 : 0;
      if (s) {
        const int st = __ldg(offu + c);
        for (int i = 0; i < w[k]; ++i) tsrc[tok_base + i] = st + i;
        tok_base += w[k];
        ssrc[sub_base] = c;
        sbias[sub_base] = log2f((float)w[k]);
        ++sub_base;
      }
    }
  }
  for (int i = tid; i < a.n_tail; i += kT) tsrc[tok_total + i] = a.n_clustered + i;
  if (tid == 0) {
    a.hdr[2 * u] = tok_total + a.n_tail;
    a.hdr[2 * u + 1] = a.approx ? sel_total : 0;
  }
}

// ---------------------------------------------------------------------------
// Centroid pass: grid = units * NA CTAs, unit-major
// ---------------------------------------------------------------------------
template <int D, int G>
__global__ void __launch_bounds__(kT, 3) centroid_pass(const __grid_constant__ Args a) {
  using Gm = Geo<D, G>;
  constexpr int SG = Gm::SG;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // TMA tiles with 128-byte swizzle need 1024-byte aligned destinations
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(smem);
  int32_t* offs = reinterpret_cast<int32_t*>(smem + Gm::OFF_AUX);
  int* red = reinterpret_cast<int*>(smem + Gm::OFF_RED);
  const uint32_t bar = sb + Gm::OFF_BAR;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, hq = lane >> 2;
  const int u = blockIdx.x / a.NA, j = blockIdx.x - u * a.NA;
  const int p0 = j * kRows;
  const int cnt = max(0, min(kRows, a.slots_active - p0));

  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    if (cnt > 0) {
      const int y = u * a.slots + p0;
      mbar_arrive_tx(bar, (uint32_t)((a.approx ? 2 : 1) * Gm::AREA));
#pragma unroll
      for (int h = 0; h < D / 64; ++h) tma_tile(sb + h * kTile, &a.tmKc, 64 * h, y, bar);
      if (a.approx) {
#pragma unroll
        for (int h = 0; h < D / 64; ++h) tma_tile(sb + Gm::OFF_V + h * kTile, &a.tmVc, 64 * h, y, bar);
      }
    }
  }
  // cluster offsets of the rows (cnt + 1 values) and the query fragments, while the tiles land
  for (int i = threadIdx.x; i <= cnt; i += kT) offs[i] = __ldg(a.off + (size_t)u * (a.slots + 1) + p0 + i);
  WarpSoftmax<D, G> ws;
  ws.load_q(a.Q + (size_t)u * G * D, lane);
  ws.reset();
  __syncthreads();
  if (cnt > 0) {
    const long long t0 = gtimer();
    while (!mbar_try(bar, 0)) {
      if (gtimer() - t0 > a.timeout_ns) { set_error(a.err, E_TIMEOUT); break; }
    }
  }
  const float qk2 = a.scale * kLog2e;
  float* Srow = a.S + ((size_t)u * a.slots + p0) * SG;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int r16 = warp * 32 + t * 16;
    if (r16 >= cnt) break;
    float z[2][2];
    ws.qk(sb, r16, lane, z);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int r = r16 + nt * 8 + 2 * (lane & 3) + i;
        const float S = z[nt][i] * a.scale;
        if (hq < G && r < cnt) Srow[(size_t)r * SG + hq] = S;
        const int n = r < cnt ? offs[r + 1] - offs[r] : 0;
        z[nt][i] = (a.approx && n > 0 && hq < G) ? S * kLog2e + log2f((float)n) : -INFINITY;
      }
    (void)qk2;
    ws.update(sb + Gm::OFF_V, r16, lane, z, 1.f);
  }
  __syncthreads();   // the key area becomes the merge buffer
  write_partial<D, G>(a, ws, reinterpret_cast<float*>(smem), u, j);
  int* bc = red + 60;
  if (threadIdx.x == 0) bc[0] = ticket(a.ctl + u);
  __syncthreads();
  if (bc[0] == a.NA - 1) select_unit<G, SG>(a, u, red);
  // the value pass may start launching once every CTA got here (it waits for this grid's completion)
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

// ---------------------------------------------------------------------------
// Value pass: grid = units * NB CTAs, unit-major.  CTA j of a unit takes the
// 128-row chunks j, j + NB, ... of the unit's stream: ceil(n_tok / 128) chunks
// of exact rows, then ceil(n_sub / 128) chunks of subtraction rows.
// ---------------------------------------------------------------------------
template <int D, int G>
__global__ void __launch_bounds__(kT, 3) value_pass(const __grid_constant__ Args a) {
  using Gm = Geo<D, G>;
  constexpr int SG = Gm::SG;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(smem);
  int32_t* rows = reinterpret_cast<int32_t*>(smem + Gm::OFF_AUX);
  int* red = reinterpret_cast<int*>(smem + Gm::OFF_RED);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, hq = lane >> 2;
  const int u = blockIdx.x / a.NB, j = blockIdx.x - u * a.NB;
  const float qk2 = a.scale * kLog2e;

  WarpSoftmax<D, G> ws;
  ws.load_q(a.Q + (size_t)u * G * D, lane);   // the query is an input of the step, not of the centroid pass
  ws.reset();
  // everything below reads what the centroid pass wrote
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  const int n_tok = __ldcg(a.hdr + 2 * u), n_sub = __ldcg(a.hdr + 2 * u + 1);
  const int ct = (n_tok + kRows - 1) / kRows, cs = (n_sub + kRows - 1) / kRows;
  for (int ch = j; ch < ct + cs; ch += a.NB) {
    const bool tok = ch < ct;
    const int p0 = tok ? ch * kRows : (ch - ct) * kRows;
    const int cnt = min(kRows, (tok ? n_tok : n_sub) - p0);
    // this warp's 32 rows: sources (one per thread), then the copies, all warp-local
    const int r = threadIdx.x;
    int src = 0;
    if (r < cnt) {
      src = tok ? __ldcg(a.tok_src + (size_t)u * a.max_tokens + p0 + r) : __ldcg(a.sub_src + (size_t)u * a.capc + p0 + r);
      const int lim = tok ? (int)a.max_tokens : a.slots;
      if ((unsigned)src >= (unsigned)lim) {   // reported and replaced by row 0
        set_error(a.err, E_BAD_LIST);
        src = 0;
      }
    }
    rows[r] = src;
    float bias = 0.f;
    if (!tok && r < cnt) bias = __ldcg(a.sub_bias + (size_t)u * a.capc + p0 + r);
    __syncwarp();
    const int r32 = warp * 32;
    if (r32 < cnt) {
      const size_t ub = (size_t)u * (tok ? (size_t)a.max_tokens : (size_t)a.slots);
      const __nv_bfloat16* Kb = a.Kp + ub * D;
      const __nv_bfloat16* Vb = (tok ? a.Vp : a.Vc) + ub * D;
      constexpr int RPI = 32 / Gm::CPR;   // rows per warp instruction
      const int c = lane % Gm::CPR;
#pragma unroll 4
      for (int k = 0; k < 32 / RPI; ++k) {
        const int rr = r32 + k * RPI + lane / Gm::CPR;
        const bool v = rr < cnt;
        const size_t o = (size_t)rows[rr] * D + c * 8;
        if (tok) cp16(sb + swz(rr, c), v ? (const void*)(Kb + o) : (const void*)a.Kp, v);
        cp16(sb + Gm::OFF_V + swz(rr, c), v ? (const void*)(Vb + o) : (const void*)a.Vp, v);
      }
      if (!tok) {
        // the subtraction rows' scores, SG floats each, in the key area
        const float* Sb = a.S + (size_t)u * a.slots * SG;
        for (int i = lane; i < 32 * (SG / 4); i += kWarp) {
          const int rr = r32 + i / (SG / 4), cc = i % (SG / 4);
          cp16(sb + rr * SG * 4 + cc * 16, Sb + (size_t)rows[rr] * SG + cc * 4, rr < cnt);
        }
      }
      cp_wait_all();
      __syncwarp();
      const float* Ss = reinterpret_cast<const float*>(smem);
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int r16 = r32 + t * 16;
        if (r16 >= cnt) break;
        float z[2][2];
        if (tok) {
          ws.qk(sb, r16, lane, z);
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const int rr = r16 + nt * 8 + 2 * (lane & 3) + i;
              z[nt][i] = (hq < G && rr < cnt) ? z[nt][i] * qk2 : -INFINITY;
            }
        } else {
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const int rr = r16 + nt * 8 + 2 * (lane & 3) + i;
              const float b = __shfl_sync(kFull, bias, (rr - r32) & 31);
              z[nt][i] = (hq < G && rr < cnt) ? Ss[rr * SG + hq] * kLog2e + b : -INFINITY;
            }
        }
        ws.update(sb + Gm::OFF_V, r16, lane, z, tok ? 1.f : -1.f);
      }
    }
    __syncwarp();   // this warp's rows of the next chunk overwrite the same shared memory
  }
  __syncthreads();
  write_partial<D, G>(a, ws, reinterpret_cast<float*>(smem), u, a.NA + j);
  int* bc = red + 60;
  if (threadIdx.x == 0) bc[0] = ticket(a.ctl + a.units + u);
  __syncthreads();
  if (bc[0] != a.NB - 1) return;
  // last value CTA of the unit: merge all its partials into the output rows
  const int P = a.NA + a.NB;
  const size_t ubp = (size_t)u * P * G;
  for (int e = threadIdx.x; e < G * D / 4; e += kT) {
    const int g = (e * 4) / D, d = (e * 4) % D;
    float M = -INFINITY;
    for (int jj = 0; jj < P; ++jj) M = fmaxf(M, __ldcg(a.pm + ubp + (size_t)jj * G + g));
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    float L = 0.f;
#pragma unroll 8
    for (int jj = 0; jj < P; ++jj) {
      const float mj = __ldcg(a.pm + ubp + (size_t)jj * G + g);
      const float4 x = __ldcg(reinterpret_cast<const float4*>(a.pacc + (ubp + (size_t)jj * G + g) * D + d));
      const float lj = __ldcg(a.pl + ubp + (size_t)jj * G + g);
      const float f = mj == -INFINITY ? 0.f : exp2f(mj - M);
      o.x += f * x.x; o.y += f * x.y; o.z += f * x.z; o.w += f * x.w;
      L += f * lj;
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    __nv_bfloat16* out = a.O + ((size_t)u * G + g) * D + d;
    *reinterpret_cast<uint2*>(out) = make_uint2(pack_bf16(o.x * inv, o.y * inv), pack_bf16(o.z * inv, o.w * inv));
  }
}

}  // namespace stream

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
static inline size_t a256(size_t x) { return (x + 255) & ~(size_t)255; }

struct StreamLayout {
  int capc, SG;
  size_t o_S, o_tok, o_ssrc, o_sbias, o_hdr, o_pm, o_pl, o_pacc, o_ctl, ctl_bytes, bytes;
};

static StreamLayout stream_layout(const mp_config& c, int slots) {
  StreamLayout L{};
  const size_t U = (size_t)c.batch * c.kv_heads;
  const int G = c.q_heads / c.kv_heads, D = c.head_dim;
  const size_t P = 2 * stream::kMaxItems;
  L.SG = (G + 3) / 4 * 4;
  L.capc = ((slots + 3) & ~3) + 64;
  size_t cur = 0;
  L.o_S = cur; cur = a256(cur + U * slots * L.SG * 4);
  L.o_tok = cur; cur = a256(cur + U * (size_t)c.max_tokens * 4);
  L.o_ssrc = cur; cur = a256(cur + U * L.capc * 4);
  L.o_sbias = cur; cur = a256(cur + U * L.capc * 4);
  L.o_hdr = cur; cur = a256(cur + U * 2 * 4);
  L.o_pm = cur; cur = a256(cur + U * P * G * 4);
  L.o_pl = cur; cur = a256(cur + U * P * G * 4);
  L.o_pacc = cur; cur = a256(cur + U * P * G * D * 4);
  L.o_ctl = cur;                                      // ticket words, reset before every step
  L.ctl_bytes = 2 * U * 4;
  cur = a256(cur + L.ctl_bytes);
  L.bytes = cur;
  return L;
}

size_t stream_scratch_bytes(const mp_config& c, int slots) { return stream_layout(c, slots).bytes; }

bool stream_supported(const mp_config& c, int slots) {
  const int G = c.q_heads / c.kv_heads;
  return c.levels == 1 && c.dtype == MP_BF16 && (c.head_dim == 64 || c.head_dim == 128) &&
         (G == 1 || G == 2 || G == 4 || G == 8) && slots <= stream::kMaxSlots;
}

// cuTensorMapEncodeTiled from the driver, resolved once through the runtime
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// rows x D bf16 matrix, tiles of 64 columns x kRows rows, 128-byte swizzle
static bool encode_rows(CUtensorMap* tm, const void* base, uint64_t rows, int D) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  cuuint64_t gdim[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)stream::kRows};
  cuuint32_t estr[2] = {1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int G>
static cudaError_t launch_stream_t(const stream::Args& a, cudaStream_t st) {
  using Gm = stream::Geo<D, G>;
  auto k1 = stream::centroid_pass<D, G>;
  auto k2 = stream::value_pass<D, G>;
  cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, Gm::SMEM);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, Gm::SMEM);
  if (e != cudaSuccess) return e;
  k1<<<a.units * a.NA, stream::kT, Gm::SMEM, st>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // the value pass is launched as a programmatic dependent of the centroid pass:
  // its CTAs may become resident while the last centroid CTAs finish, and wait
  // (griddepcontrol.wait) for that grid's completion before reading its results
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(a.units * a.NB);
  cfg.blockDim = dim3(stream::kT);
  cfg.dynamicSmemBytes = Gm::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k2, a);
}

template <int D>
static cudaError_t launch_stream_d(int G, const stream::Args& a, cudaStream_t st) {
  switch (G) {
    case 1: return launch_stream_t<D, 1>(a, st);
    case 2: return launch_stream_t<D, 2>(a, st);
    case 4: return launch_stream_t<D, 4>(a, st);
    case 8: return launch_stream_t<D, 8>(a, st);
  }
  return cudaErrorInvalidValue;
}

// The flat bf16 decode step: a memset of the ticket words and two kernels.
mp_status stream_decode(const mp_index* idx, const void* Q, void* O, const mp_decode_params* prm, void* scratch,
                        size_t scratch_bytes, float scale, cudaStream_t st) {
  const mp_config& c = idx->cfg;
  StreamLayout L = stream_layout(c, idx->slots);
  if (scratch_bytes < L.bytes) return MP_ENOSPC;
  char* base = static_cast<char*>(scratch);
  const int U = c.batch * c.kv_heads, G = c.q_heads / c.kv_heads, D = c.head_dim;
  stream::Args a{};
  const void* Kc = ws_ptr(idx, S_KC);
  a.Vc = static_cast<const __nv_bfloat16*>(ws_ptr(idx, S_VC));
  if (!encode_rows(&a.tmKc, Kc, (uint64_t)U * idx->slots, D) ||
      !encode_rows(&a.tmVc, a.Vc, (uint64_t)U * idx->slots, D))
    return MP_ECUDA;
  a.Q = static_cast<const __nv_bfloat16*>(Q);
  a.O = static_cast<__nv_bfloat16*>(O);
  a.Kp = static_cast<const __nv_bfloat16*>(ws_ptr(idx, S_KP));
  a.Vp = static_cast<const __nv_bfloat16*>(ws_ptr(idx, S_VP));
  a.off = static_cast<const int32_t*>(ws_ptr(idx, S_OFF));
  a.units = U;
  a.slots = idx->slots;
  const int64_t blocks_used = (idx->n_clustered + c.block_tokens - 1) / c.block_tokens;
  a.slots_active = (int)std::min<int64_t>(idx->slots, blocks_used * idx->slots_per_block);
  a.max_tokens = c.max_tokens;
  a.n_clustered = (int)idx->n_clustered;
  a.n_tail = (int)(idx->n_tokens - idx->n_clustered);
  a.scale = scale;
  a.budget = prm->budget;
  a.approx = (prm->flags & MP_NO_APPROX) == 0;
  a.NA = std::max(1, std::min(stream::kMaxItems, (a.slots_active + stream::kRows - 1) / stream::kRows));
  if (prm->n_split > 0) {
    a.NB = std::min(prm->n_split, stream::kMaxItems);
  } else {
    // one 128-row chunk per value CTA for the expected stream length
    const int64_t est_tok = std::min<int64_t>(idx->n_tokens, (int64_t)std::max(prm->budget, 0) +
                                                                 8LL * c.tokens_per_centroid + a.n_tail);
    const int64_t est_chunks = (est_tok + stream::kRows - 1) / stream::kRows + 1;
    a.NB = (int)std::max<int64_t>(1, std::min<int64_t>(stream::kMaxItems, est_chunks));
  }
  a.capc = L.capc;
  a.S = reinterpret_cast<float*>(base + L.o_S);
  a.tok_src = reinterpret_cast<int32_t*>(base + L.o_tok);
  a.sub_src = reinterpret_cast<int32_t*>(base + L.o_ssrc);
  a.sub_bias = reinterpret_cast<float*>(base + L.o_sbias);
  a.hdr = reinterpret_cast<int32_t*>(base + L.o_hdr);
  a.pm = reinterpret_cast<float*>(base + L.o_pm);
  a.pl = reinterpret_cast<float*>(base + L.o_pl);
  a.pacc = reinterpret_cast<float*>(base + L.o_pacc);
  a.ctl = reinterpret_cast<int32_t*>(base + L.o_ctl);
  a.sel_mask_out = prm->sel_mask_out;
  a.scores_out = prm->scores_out;
  a.err = err_word(idx);
  a.timeout_ns = 2000000000LL;

  auto phase = [&](int i) {
    if (i < prm->n_phase_events && prm->phase_events[i])
      cudaEventRecord(static_cast<cudaEvent_t>(prm->phase_events[i]), st);
  };
  phase(0);
  if (cudaMemsetAsync(base + L.o_ctl, 0, L.ctl_bytes, st) != cudaSuccess) return MP_ECUDA;
  phase(1);
  cudaError_t e = D == 128 ? launch_stream_d<128>(G, a, st) : launch_stream_d<64>(G, a, st);
  phase(2);
  return e == cudaSuccess ? MP_OK : MP_ECUDA;
}

}  // namespace mp
