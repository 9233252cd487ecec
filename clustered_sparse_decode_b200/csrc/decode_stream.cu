// Flat decode step for bf16 caches: a centroid pass and a value pass, each a
// persistent kernel with one CTA per SM.
//
// "Multipole Attention for Efficient Long Context Reasoning" (arXiv abstract;
// atlas.scime summary, "Approach"): the query scores every key centroid, the
// best clusters up to a token budget are attended exactly, and every other
// cluster enters the same softmax as one term with logit score + ln(size) and
// its value centroid.
//
//   centroid pass  the (unit, 128-slot chunk) pairs of all (batch, KV head)
//                  units, split into equal contiguous shares per CTA.  Per
//                  chunk: S[c][g] = scale * q_g . Kc_c (written to scratch) and
//                  online-softmax state over the centroid terms of ALL its
//                  clusters (logit S + ln n_c, value Vc_c).  The CTA that
//                  finishes the last share of a unit runs the unit's budgeted
//                  selection and writes its value stream.
//   value pass     (programmatic dependent launch) the units' value streams,
//                  concatenated and split by bytes into equal shares per CTA:
//                  the exact rows (tokens of the selected clusters in slot
//                  order, then the un-clustered tail), then one row per
//                  selected cluster that SUBTRACTS its centroid term again, so
//                  that the centroid partials keep only the unselected
//                  clusters.  The CTA that finishes the last share of a unit
//                  merges all partials of the unit into its output rows.
// Subtracting is safe in fp32: a selected centroid term n e^{q.Kc} is at most
// the exact mass of its cluster (Jensen, Kc being the member mean), so the
// cancellation error stays a few ulps of the final normaliser.
//
// Data movement: the centroid pass has a producer warp that loads each chunk's
// contiguous Kc / Vc rows as TMA tiles (64 columns x 128 rows, 128-byte
// swizzle) into a ring of kNS chunks; in the value pass every warp gathers its
// own 16 rows of each chunk with cp.async (16-byte chunks, same swizzled
// layout), kNS - 1 chunks ahead of its compute.  Compute: eight warps, 16 rows
// of a chunk each, on the tensor cores with mma.sync m16n8k16 (bf16 in, fp32
// accumulate): the G query heads are the M rows (G of 16 used), 8 keys the N
// columns; the probabilities enter P.V as a bf16 hi + lo pair, so the weights
// keep ~16 significant bits.  The contraction is small next to the bytes
// streamed: the tensor cores only keep the instructions per byte low.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdio>
#include <mutex>

#include "mp_internal.cuh"

namespace mp {
namespace stream {

constexpr int kCW = 8;                        // compute warps per CTA
constexpr int kCT = kCW * kWarp;              // compute threads
constexpr int kRows = 128;                    // rows of a chunk (16 per compute warp)
constexpr int kTile = kRows * 128;            // one 64-column tile of a chunk (bytes)
constexpr int kNS = 3;                        // chunks in flight per CTA
constexpr int kMaxSpt = 16;                   // selection: slots per thread (slots <= 4096)
constexpr int kMaxSlots = kMaxSpt * kCT;
constexpr int kMaxUnits = 512;                // per-unit tables in shared memory
constexpr int kMaxGrid = 512;

struct Args {
  CUtensorMap tmKc;            // Kc as [units*slots rows][D] bf16: 64 x 128 tiles, 128-byte swizzle
  CUtensorMap tmVc;
  const __nv_bfloat16* Q;      // [units*G][D]
  __nv_bfloat16* O;            // [units*G][D]
  const __nv_bfloat16* Vc;     // [units][slots][D]
  const __nv_bfloat16* Kp;     // [units][max_tokens][D]
  const __nv_bfloat16* Vp;
  const int32_t* off;          // [units][slots + 1]
  int units, slots, slots_active, cpu;   // cpu: centroid chunks per unit (>= 1)
  int64_t max_tokens;
  int n_clustered, n_tail;
  float scale;                 // score scale, natural-log units
  int budget, approx;
  int capc;                    // selected-cluster capacity per unit
  float* S;                    // [units][slots][SG] scores (natural units), rows padded to 16 bytes
  int32_t* tok_src;            // [units][max_tokens] store row of each exact row of the value stream
  int32_t* sub_src;            // [units][capc] slot of each selected cluster (subtraction rows)
  float* sub_bias;             // [units][capc] log2 of its size
  int32_t* hdr;                // [units][2]: exact rows, subtraction rows
  float* pm;                   // [npart][G] partial max (log2 units)
  float* pl;                   // [npart][G] partial normaliser
  float* pacc;                 // [npart][G][D] partial numerator
  int part_v;                  // first partial of the value pass (the centroid pass uses [0, part_v));
                               // per (unit, share, warp): (first[u] + share index) * kCW + warp
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
  static constexpr int AREA = kRows * D * 2;           // key (or value) rows of a chunk: D/64 tiles
  static constexpr int SLOT = 2 * AREA;                // 1024-byte multiple
  static constexpr int QB = ((G * D * 2 + 127) / 128) * 128;
  static constexpr int OFF_AUX = kNS * SLOT;           // per slot: query rows, cluster offsets, meta
  static constexpr int AUX = QB + (kRows + 4) * 4 + 32;
  static constexpr int OFF_UNIT = OFF_AUX + kNS * AUX; // per unit and pass: first partial, number of shares
  static constexpr int OFF_WPRE = OFF_UNIT + kMaxUnits * 16;   // value pass: weight prefix over units
  static constexpr int OFF_HDR = (OFF_WPRE + (kMaxUnits + 1) * 8 + 15) / 16 * 16;   // value pass: stream lengths
  static constexpr int OFF_RED = OFF_HDR + kMaxUnits * 8;
  static constexpr int OFF_BAR = OFF_RED + 128 * 4;
  static constexpr int SMEM = OFF_BAR + 2 * kNS * 8 + 16 + 1024;   // + alignment slack
  static_assert(D % 64 == 0, "rows are whole 64-column tiles");
  static_assert(kRows * SG * 4 <= AREA, "subtraction-row scores live in the key area");
  static_assert(AUX % 16 == 0, "16-byte aligned side areas");
  static_assert(OFF_AUX % 1024 == 0 && OFF_UNIT % 16 == 0 && OFF_WPRE % 16 == 0 && OFF_HDR % 16 == 0 &&
                    OFF_RED % 16 == 0 && OFF_BAR % 16 == 0,
                "regions read with 16-byte vectors and mbarriers need 16-byte alignment");
  static_assert(SMEM <= 232448, "one CTA per SM");
};

struct ChunkMeta {
  int unit, p0, cnt, flags;    // flags: 1 first chunk of a share of the unit, 2 last
  int seg, pad0, pad1, pad2;   // seg: this CTA's share index within the unit
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
__device__ __forceinline__ void cp4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }
__device__ __forceinline__ void cp_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }
// the mbarrier's current phase also waits for this thread's earlier cp.async (not an expected arrival)
__device__ __forceinline__ void cp_arrive_inc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];\n" ::"r"(bar) : "memory");
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
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(10000000u)   // suspend up to 10 ms until the phase completes
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
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }
// ticket: returns the old value; release orders this CTA's earlier writes (made
// visible to this thread by the preceding CTA barrier) before the increment,
// acquire orders the winner's later reads after it
__device__ __forceinline__ int ticket(int32_t* p) {
  int v;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;\n" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// barrier of the compute warps only (the centroid pass's producer warp does not take part)
__device__ __forceinline__ void cbar() { asm volatile("bar.sync 1, %0;\n" ::"n"(kCT) : "memory"); }
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
// D[16x8] += A[16x16] B[16x8] with all four A registers and accumulators
__device__ __forceinline__ void mma16816_full(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
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

// Byte offset of 16-byte chunk c of row r inside a key or value area: the area
// holds D/64 tiles of [kRows rows][128 bytes]; within a tile the chunk index is
// XORed with the row's low 3 bits, which is the layout a TMA tile load with
// 128-byte swizzle writes to a 1024-byte aligned destination.
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return (uint32_t)((c >> 3) * kTile + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// ---------------------------------------------------------------------------
// Shares: N weighted positions split into `grid` contiguous shares
// ---------------------------------------------------------------------------
__host__ __device__ __forceinline__ long long share_lo(int c, long long N, int grid) {
  return (long long)c * N / grid;
}
// the CTA whose share holds position x (0 <= x < N): the largest c with share_lo(c) <= x
// (never an empty share: those have share_lo(c) == share_lo(c + 1))
__host__ __device__ __forceinline__ int share_owner(long long x, long long N, int grid) {
  return (int)(((x + 1) * grid - 1) / N);
}
// number of non-empty shares among [ca, cb)
__device__ __forceinline__ int shares_nonempty(int ca, int cb, long long N, int grid) {
  int n = 0;
  for (int c = ca; c < cb; ++c) n += share_lo(c + 1, N, grid) > share_lo(c, N, grid) ? 1 : 0;
  return n;
}
// the shares holding positions [xb, xe) (xe > xb): how many, and CTA c's index among them
__device__ __forceinline__ int shares_of(long long xb, long long xe, long long N, int grid) {
  const int c0 = share_owner(xb, N, grid), c1 = share_owner(xe - 1, N, grid);
  return 1 + shares_nonempty(c0 + 1, c1 + 1, N, grid);
}
__device__ __forceinline__ int share_index(int c, long long xb, long long N, int grid) {
  return shares_nonempty(share_owner(xb, N, grid), c, N, grid);
}
// Per unit: number of shares (partials of share s: (first + s) * kCW + warp) of the centroid pass (chunks [u * cpu, (u + 1) * cpu) of units * cpu) and, if
// wpre is given, of the value pass (weights [wpre[u], wpre[u + 1]) of wpre[units]).
__device__ void unit_tables(const Args& a, int grid, int* cfirst, int* cnsh, const long long* wpre, int* vfirst,
                            int* vnsh, int nthreads) {
  const long long NCH = (long long)a.units * a.cpu;
  for (int u = threadIdx.x; u < a.units; u += nthreads) {
    cnsh[u] = shares_of((long long)u * a.cpu, (long long)(u + 1) * a.cpu, NCH, grid);
    if (wpre) vnsh[u] = shares_of(wpre[u], wpre[u + 1], wpre[a.units], grid);
  }
  __syncwarp();
}

// ---------------------------------------------------------------------------
// Per-warp online softmax over 16-row tiles
// ---------------------------------------------------------------------------
template <int D, int G>
struct WarpSoftmax {
  uint32_t qa[D / 16][2];      // A fragments of the query heads (rows 0..7), k-steps of 16
  float acc[D / 16][4];        // numerator O^T: m-tile mt holds [d = 16 mt + lane/4 (+8)][head 2*(lane%4) (+1)]
  float m, l;                  // running max (log2 units) and normaliser share of head lane/4

  __device__ __forceinline__ void reset() {
    m = -INFINITY;
    l = 0.f;
#pragma unroll
    for (int n = 0; n < D / 16; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  }
  template <typename P>
  __device__ __forceinline__ void load_q(const P* q, int lane) {   // q: [G][D] bf16 (global or shared)
    const int hq = lane >> 2;
    const uint32_t* qs = reinterpret_cast<const uint32_t*>(q);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      qa[ks][0] = hq < G ? qs[(hq * D + ks * 16 + 2 * (lane & 3)) >> 1] : 0u;
      qa[ks][1] = hq < G ? qs[(hq * D + ks * 16 + 8 + 2 * (lane & 3)) >> 1] : 0u;
    }
  }
  // raw dot products q_g . k for the 16 rows of a tile (S = Q K^T with the heads as M rows;
  // this lane: head lane/4, rows 2*(lane%4) + {0,1} + 8*nt)
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
  // Fold a tile with logits z (log2 units, -inf = no term) and weight sign into
  // the state.  P.V is computed as O^T += V^T P^T: the value rows' transpose is
  // the A operand (m-tiles of 16 columns), and the probabilities, already in
  // the B-operand layout, enter as a bf16 hi + lo pair.
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
      alpha = ex2(m - mnew);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int i = 0; i < 2; ++i) pr[nt][i] = sign * ex2(z[nt][i] - mnew);
    }
    m = mnew;
    l = l * alpha + ((pr[0][0] + pr[0][1]) + (pr[1][0] + pr[1][1]));
    if (__any_sync(kFull, alpha != 1.f)) {
      // this lane's accumulators belong to heads 2*(lane%4) and 2*(lane%4) + 1
      const float a0 = __shfl_sync(kFull, alpha, 8 * (lane & 3));
      const float a1 = __shfl_sync(kFull, alpha, 8 * (lane & 3) + 4);
#pragma unroll
      for (int n = 0; n < D / 16; ++n) { acc[n][0] *= a0; acc[n][1] *= a1; acc[n][2] *= a0; acc[n][3] *= a1; }
    }
    const uint32_t h0 = pack_bf16(pr[0][0], pr[0][1]);
    const uint32_t h1 = pack_bf16(pr[1][0], pr[1][1]);
    const uint32_t l0 = pack_bf16(pr[0][0] - bf16_lo(h0), pr[0][1] - bf16_hi(h0));
    const uint32_t l1 = pack_bf16(pr[1][0] - bf16_lo(h1), pr[1][1] - bf16_hi(h1));
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      uint32_t v0, v1, v2, v3;
      ldsm4t(vb + swz(r16 + (lane & 7) + 8 * (lane >> 4), 2 * mt + ((lane >> 3) & 1)), v0, v1, v2, v3);
      mma16816_full(acc[mt], v0, v1, v2, v3, h0, h1);
      mma16816_full(acc[mt], v0, v1, v2, v3, l0, l1);
    }
  }
  // this warp's state as partial p: max and normaliser per head, numerator per head and column
  __device__ __forceinline__ void store(const Args& a, int p, int lane) const {
    const int hq = lane >> 2, h0 = 2 * (lane & 3), h1 = h0 + 1, d0 = lane >> 2;
    float lt = l;
    lt += __shfl_xor_sync(kFull, lt, 1);
    lt += __shfl_xor_sync(kFull, lt, 2);
    if (hq < G && (lane & 3) == 0) {
      a.pm[(size_t)p * G + hq] = m;
      a.pl[(size_t)p * G + hq] = lt;
    }
    float* o0 = a.pacc + ((size_t)p * G + h0) * D + d0;
    float* o1 = a.pacc + ((size_t)p * G + h1) * D + d0;
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      if (h0 < G) { o0[16 * mt] = acc[mt][0]; o0[16 * mt + 8] = acc[mt][2]; }
      if (h1 < G) { o1[16 * mt] = acc[mt][1]; o1[16 * mt + 8] = acc[mt][3]; }
    }
  }
};

// Merge the partials [p0, p0 + n0) and [p1, p1 + n1) of unit u into its output
// rows (compute threads; one thread per 4 columns of a head, online over the partials).
template <int D, int G>
__device__ void combine_unit(const Args& a, int u, int p0, int n0, int p1, int n1) {
  const int n = n0 + n1;
  for (int e = threadIdx.x; e < G * D / 4; e += kCT) {
    const int g = (e * 4) / D, d = (e * 4) % D;
    float M = -INFINITY, L = 0.f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j0 = 0; j0 < n; j0 += 16) {
      float mj[16], lj[16];
      float4 xj[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const int jj = min(j0 + k, n - 1);
        const size_t p = jj < n0 ? p0 + jj : p1 + jj - n0;
        mj[k] = j0 + k < n ? __ldcg(a.pm + p * G + g) : -INFINITY;
        lj[k] = __ldcg(a.pl + p * G + g);
        xj[k] = __ldcg(reinterpret_cast<const float4*>(a.pacc + (p * G + g) * D + d));
      }
      float Mn = M;
#pragma unroll
      for (int k = 0; k < 16; ++k) Mn = fmaxf(Mn, mj[k]);
      if (Mn == -INFINITY) continue;
      const float s0 = M == -INFINITY ? 0.f : ex2(M - Mn);
      o.x *= s0; o.y *= s0; o.z *= s0; o.w *= s0;
      L *= s0;
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const float f = mj[k] == -INFINITY ? 0.f : ex2(mj[k] - Mn);
        o.x += f * xj[k].x; o.y += f * xj[k].y; o.z += f * xj[k].z; o.w += f * xj[k].w;
        L += f * lj[k];
      }
      M = Mn;
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    __nv_bfloat16* out = a.O + ((size_t)u * G + g) * D + d;
    *reinterpret_cast<uint2*>(out) = make_uint2(pack_bf16(o.x * inv, o.y * inv), pack_bf16(o.z * inv, o.w * inv));
  }
}

// exclusive scan out[u] = base + sum(in[0..u)) for u < n <= 2 * kCT (compute threads; red: >= kCW ints)
template <typename T>
__device__ void scan_units(const T* in, T* out, int n, T base, T* red) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i0 = 2 * threadIdx.x;
  const T x0 = i0 < n ? in[i0] : T(0), x1 = i0 + 1 < n ? in[i0 + 1] : T(0);
  T v = x0 + x1, inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const T y = __shfl_up_sync(kFull, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) red[warp] = inc;
  cbar();
  T pre = base;
  for (int w = 0; w < warp; ++w) pre += red[w];
  const T ex = pre + inc - v;
  cbar();
  if (i0 < n) out[i0] = ex;
  if (i0 + 1 < n) out[i0 + 1] = ex + x0;
  cbar();
}

// ---------------------------------------------------------------------------
// Block-wide helpers for the compute threads (red: 64 ints)
// ---------------------------------------------------------------------------
__device__ __forceinline__ int csum(int v, int* red, int& par) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  v = __reduce_add_sync(kFull, v);
  int* r = red + par * kCW;
  if (lane == 0) r[warp] = v;
  cbar();
  int t = 0;
#pragma unroll
  for (int i = 0; i < kCW; ++i) t += r[i];
  par ^= 1;
  return t;
}

// exclusive scan of two ints over the compute threads in thread order; returns totals
__device__ __forceinline__ void cscan2(int a, int b, int& ea, int& eb, int& ta, int& tb, int* red) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int ia = a, ib = b;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int xa = __shfl_up_sync(kFull, ia, o), xb = __shfl_up_sync(kFull, ib, o);
    if (lane >= o) { ia += xa; ib += xb; }
  }
  int* r = red + 2 * kCW;
  if (lane == 31) { r[warp] = ia; r[kCW + warp] = ib; }
  cbar();
  int pa = 0, pb = 0;
  ta = 0; tb = 0;
#pragma unroll
  for (int i = 0; i < kCW; ++i) {
    if (i < warp) { pa += r[i]; pb += r[kCW + i]; }
    ta += r[i]; tb += r[kCW + i];
  }
  ea = pa + ia - a;
  eb = pb + ib - b;
  cbar();   // r[] is reused by the next scan
}

// ---------------------------------------------------------------------------
// Selection of one unit (the compute threads of the CTA that finished the
// unit's last centroid share).  Token-budgeted: clusters by score descending,
// ties to the lower slot, shortest prefix whose token count reaches the budget
// (the crossing cluster whole); budget <= 0 selects nothing, a budget at or
// above all clustered tokens selects every non-empty cluster.
// The threshold tau (the largest key with W(key >= tau) >= budget, keys being
// the order-preserving uint32 images of the group scores) is found exactly by
// a radix descent over the bits in which the candidates' keys differ: each
// level histograms the weights of the keys inside the current interval over
// 256 bins (shared-memory atomics), one warp finds the bin where the running
// weight from the top crosses the budget, and the interval narrows to it.
// hist: 256 ints of shared memory.
// ---------------------------------------------------------------------------
template <int G, int SG>
__device__ void select_unit(const Args& a, int u, int* red, int* hist) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int slots = a.slots;
  const int spt = (slots + kCT - 1) / kCT;
  const int s0 = tid * spt;
  const int32_t* offu = a.off + (size_t)u * (slots + 1);
  const float* Su = a.S + (size_t)u * slots * SG;

  uint32_t key[kMaxSpt];
  int w[kMaxSpt];
  int st0[kMaxSpt];
  int wsum = 0;
  uint32_t kmin = 0xffffffffu, kmax = 0u;
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
        st0[k0 + k] = o[k];
        wsum += w[k0 + k];
        if (cnt > 0) { kmin = min(kmin, key[k0 + k]); kmax = max(kmax, key[k0 + k]); }
        if (in && a.scores_out) a.scores_out[(size_t)u * slots + c] = cnt > 0 ? sh : -INFINITY;
      }
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) { key[k0 + k] = 0u; w[k0 + k] = 0; st0[k0 + k] = 0; }
    }
  }
  // total weight and key range of the candidates
  {
    const int ws_ = __reduce_add_sync(kFull, wsum);
    const uint32_t mn = __reduce_min_sync(kFull, kmin), mx = __reduce_max_sync(kFull, kmax);
    if (lane == 0) { red[warp] = ws_; red[kCW + warp] = (int)mn; red[2 * kCW + warp] = (int)mx; }
    cbar();
    wsum = 0; kmin = 0xffffffffu; kmax = 0u;
#pragma unroll
    for (int i = 0; i < kCW; ++i) {
      wsum += red[i];
      kmin = min(kmin, (uint32_t)red[kCW + i]);
      kmax = max(kmax, (uint32_t)red[2 * kCW + i]);
    }
    cbar();
  }
  const int W = wsum;
  // mode 0: none, 1: all non-empty clusters, 2: threshold
  const int mode = (a.budget <= 0 || W == 0) ? 0 : (W <= a.budget ? 1 : 2);
  uint32_t tau = 0u;
  int need = 0;
  if (mode == 2) {
    uint32_t lo = kmin;
    int nb = kmax == kmin ? 0 : 32 - __clz(kmax - kmin);   // the interval [lo, lo + 2^nb) holds all candidates
    int above = 0;                                          // weight of the keys above the interval
    while (nb > 0) {
      const int sh = max(nb - 8, 0);
      for (int i = tid; i < 256; i += kCT) hist[i] = 0;
      cbar();
      const unsigned long long hi_excl = (unsigned long long)lo + (1ull << nb);
#pragma unroll
      for (int k = 0; k < kMaxSpt; ++k)
        if (w[k] > 0 && key[k] >= lo && (unsigned long long)key[k] < hi_excl) atomicAdd(hist + ((key[k] - lo) >> sh), w[k]);
      cbar();
      if (warp == 0) {
        // lane l holds bins 8l .. 8l + 7; running weight from the top bin down
        int bl[8], ls = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) { bl[i] = hist[8 * lane + i]; ls += bl[i]; }
        int suf = ls;   // inclusive suffix over lanes l' >= l
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_down_sync(kFull, suf, o);
          if (lane + o < 32) suf += y;
        }
        int run = above + suf - ls;   // weight above this lane's bins
        int found = -1, ab = 0;
#pragma unroll
        for (int i = 7; i >= 0; --i) {
          if (found < 0 && run + bl[i] >= a.budget) { found = 8 * lane + i; ab = run; }
          run += bl[i];
        }
        const unsigned m = __ballot_sync(kFull, found >= 0);
        const int src = 31 - __clz(m);   // the highest lane with a crossing bin holds the answer
        const int fb = __shfl_sync(kFull, found, src), fa = __shfl_sync(kFull, ab, src);
        if (lane == 0) { red[0] = fb; red[1] = fa; }
      }
      cbar();
      const int b = red[0];
      above = red[1];
      lo += (uint32_t)b << sh;
      nb = sh;
      cbar();
    }
    tau = lo;
    need = a.budget - above;   // >= 1 tokens still to take among the ties at tau
  }
  int tw = 0;
  if (mode == 2) {
#pragma unroll
    for (int k = 0; k < kMaxSpt; ++k) tw += (key[k] == tau && w[k] > 0) ? w[k] : 0;
  }
  int tie_before, e2, t1, t2;
  cscan2(tw, 0, tie_before, e2, t1, t2, red);
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
  cscan2(ntok, nsel, tok_base, sub_base, tok_total, sel_total, red);

  int32_t* tsrc = a.tok_src + (size_t)u * a.max_tokens;
  int32_t* ssrc = a.sub_src + (size_t)u * a.capc;
  float* sbias = a.sub_bias + (size_t)u * a.capc;
  // this thread's selected clusters: mask, subtraction rows and their tokens.  One
  // compact loop (no unrolled copies of the store code): each warp walks its
  // lanes' selected clusters one at a time and stores each run coalesced.
  uint32_t selrem = selbits;
  if (a.sel_mask_out) {
    for (int k = 0; k < spt; ++k)
      if (s0 + k < slots) a.sel_mask_out[(size_t)u * slots + s0 + k] = (selbits >> k) & 1u;
  }
  int my_base = tok_base;
#pragma unroll 1
  for (;;) {
    // next selected cluster of this lane (if any), in slot order
    int k = selrem ? __ffs(selrem) - 1 : -1;
    int cnt = 0, st = 0;
    if (k >= 0) {
      selrem &= selrem - 1;
      st = __ldg(offu + s0 + k);
      cnt = __ldg(offu + s0 + k + 1) - st;
      ssrc[sub_base] = s0 + k;
      sbias[sub_base] = log2f((float)cnt);
      ++sub_base;
    }
    unsigned m = __ballot_sync(kFull, k >= 0);
    if (!m) break;
#pragma unroll 1
    while (m) {
      const int L = __ffs(m) - 1;
      m &= m - 1;
      const int sL = __shfl_sync(kFull, st, L), cL = __shfl_sync(kFull, cnt, L), bL = __shfl_sync(kFull, my_base, L);
      for (int i = lane; i < cL; i += kWarp) tsrc[bL + i] = sL + i;
    }
    my_base += cnt;
  }
  for (int i = tid; i < a.n_tail; i += kCT) tsrc[tok_total + i] = a.n_clustered + i;
  if (tid == 0) {
    a.hdr[2 * u] = tok_total + a.n_tail;
    a.hdr[2 * u + 1] = a.approx ? sel_total : 0;
  }
}

// ---------------------------------------------------------------------------
// Centroid pass: grid CTAs of kCT compute threads + one producer warp
// ---------------------------------------------------------------------------
template <int D, int G>
__global__ void __launch_bounds__(kCT + kWarp, 1) centroid_pass(const __grid_constant__ Args a) {
  using Gm = Geo<D, G>;
  constexpr int SG = Gm::SG;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // TMA tiles with 128-byte swizzle need 1024-byte aligned destinations
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(smem);
  int* first = reinterpret_cast<int*>(smem + Gm::OFF_UNIT);
  int* nsh = first + kMaxUnits;
  int* red = reinterpret_cast<int*>(smem + Gm::OFF_RED);
  const uint32_t full0 = sb + Gm::OFF_BAR, empty0 = full0 + kNS * 8;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, hq = lane >> 2;
  const long long NCH = (long long)a.units * a.cpu;
  const int c = blockIdx.x, grid = gridDim.x;
  const long long lo = share_lo(c, NCH, grid), hi = share_lo(c + 1, NCH, grid);
  const long long t_start = gtimer();
  auto aux = [&](int slot) { return smem + Gm::OFF_AUX + slot * Gm::AUX; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNS; ++i) {
      mbar_init(full0 + 8 * i, 1);           // the producer's arrival (+ TMA bytes, + tracked small copies)
      mbar_init(empty0 + 8 * i, kCW);        // one arrival per compute warp
    }
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  __syncthreads();

  if (warp == kCW) {
    // ======================= producer =======================
    for (long long x = lo; x < hi; ++x) {
      const int k = (int)(x - lo), slot = k % kNS;
      // wait until the compute warps released the slot (bounded)
      bool got = true;
      if (lane == 0) {
        while (!(got = mbar_try(empty0 + 8 * slot, ((k / kNS) & 1) ^ 1))) {
          if (gtimer() - t_start > a.timeout_ns) { set_error(a.err, E_TIMEOUT); break; }
        }
      }
      if (!__shfl_sync(kFull, got ? 1 : 0, 0)) break;
      const int u = (int)(x / a.cpu), j = (int)(x - (long long)u * a.cpu);
      const int p0 = j * kRows, cnt = max(0, min(kRows, a.slots_active - p0));
      unsigned char* ax = aux(slot);
      const uint32_t axs = smem_u32(ax);
      ChunkMeta* cm = reinterpret_cast<ChunkMeta*>(ax + Gm::QB + (kRows + 4) * 4);
      if (lane == 0) {
        const bool first_of_share = x == lo || j == 0;
        const bool last_of_share = x == hi - 1 || j == a.cpu - 1;
        const int seg = share_index(c, (long long)u * a.cpu, NCH, grid);
        *cm = ChunkMeta{u, p0, cnt, (first_of_share ? 1 : 0) | (last_of_share ? 2 : 0), seg, 0, 0, 0};
      }
      // small copies, tracked by the phase: the unit's query rows, the rows' cluster offsets
      const __nv_bfloat16* q = a.Q + (size_t)u * G * D;
      for (int i = lane; i < G * Gm::CPR; i += kWarp) cp16(axs + 16 * i, q + 8 * i, true);
      const int32_t* ob = a.off + (size_t)u * (a.slots + 1) + p0;
      for (int i = lane; i <= cnt; i += kWarp) cp4(axs + Gm::QB + 4 * i, ob + i);
      cp_arrive_inc(full0 + 8 * slot);
      __syncwarp();
      if (lane == 0) {
        const uint32_t dst = sb + slot * Gm::SLOT;
        if (cnt > 0) {
          fence_proxy_async();
          const int y = u * a.slots + p0;
          mbar_arrive_tx(full0 + 8 * slot, (uint32_t)((a.approx ? 2 : 1) * Gm::AREA));
#pragma unroll
          for (int h = 0; h < D / 64; ++h) tma_tile(dst + h * kTile, &a.tmKc, 64 * h, y, full0 + 8 * slot);
          if (a.approx) {
#pragma unroll
            for (int h = 0; h < D / 64; ++h) tma_tile(dst + Gm::AREA + h * kTile, &a.tmVc, 64 * h, y, full0 + 8 * slot);
          }
        } else {
          mbar_arrive(full0 + 8 * slot);
        }
      }
    }
    cp_wait_all();
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
    return;
  }

  // ======================= compute warps =======================
  unit_tables(a, grid, first, nsh, nullptr, nullptr, nullptr, kCT);
  cbar();
  scan_units<int>(nsh, first, a.units, 0, red + 64);
  WarpSoftmax<D, G> ws;
  ws.reset();
  int* bc = red + 120;
  for (long long x = lo; x < hi; ++x) {
    const int k = (int)(x - lo), slot = k % kNS;
    bool got = true;
    {
      while (!(got = mbar_try(full0 + 8 * slot, (k / kNS) & 1))) {
        if (gtimer() - t_start > 2 * a.timeout_ns) { set_error(a.err, E_TIMEOUT); break; }
      }
    }
    if (!got) break;
    const unsigned char* ax = aux(slot);
    const ChunkMeta cm = *reinterpret_cast<const ChunkMeta*>(ax + Gm::QB + (kRows + 4) * 4);
    const int32_t* offs = reinterpret_cast<const int32_t*>(ax + Gm::QB);
    const uint32_t dst = sb + slot * Gm::SLOT;
    const int u = cm.unit;
    if (cm.flags & 1) {
      ws.load_q(reinterpret_cast<const __nv_bfloat16*>(ax), lane);
      ws.reset();
    }
    const int r16 = warp * 16;
    if (r16 < cm.cnt) {
      float z[2][2];
      ws.qk(dst, r16, lane, z);
      float* Srow = a.S + ((size_t)u * a.slots + cm.p0) * SG;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int r = r16 + nt * 8 + 2 * (lane & 3) + i;
          const float S = z[nt][i] * a.scale;
          if (hq < G && r < cm.cnt) Srow[(size_t)r * SG + hq] = S;
          const int n = r < cm.cnt ? offs[r + 1] - offs[r] : 0;
          z[nt][i] = (a.approx && n > 0 && hq < G) ? S * kLog2e + log2f((float)n) : -INFINITY;
        }
      ws.update(dst + Gm::AREA, r16, lane, z, 1.f);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty0 + 8 * slot);
    if (cm.flags & 2) {
      // end of this CTA's share of unit u: the warps' partials, then the unit's ticket
      ws.store(a, (first[u] + cm.seg) * kCW + warp, lane);
      cbar();
      if (threadIdx.x == 0) bc[0] = ticket(a.ctl + u);
      cbar();
      const int t = bc[0];
      if (t == nsh[u] - 1) select_unit<G, SG>(a, u, red, reinterpret_cast<int*>(smem + Gm::OFF_WPRE));
      cbar();
    }
  }
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

// ---------------------------------------------------------------------------
// Value pass: grid CTAs of kCT threads, every warp its own copy pipeline
// ---------------------------------------------------------------------------
// Stream of unit u in weight units: 1 (a placeholder, so that every unit is in
// exactly one share even when it has no rows), 2 per exact row, 1 per
// subtraction row.  A row belongs to the share that holds its first weight.
struct VChunk {
  int unit, kind, p0, cnt;     // kind 0 exact rows, 1 subtraction rows, 2 empty (unit placeholder)
  int first, last, seg, pad;   // first / last chunk of this CTA's share of the unit; share index
};

// Cursor over this CTA's share of the concatenated streams (the same on every warp).
struct VCursor {
  long long pos, hi;           // weight position in [lo, hi)
  int u;                       // unit of pos
  bool started;                // a chunk of the current unit was already returned
};

template <int D, int G>
__global__ void __launch_bounds__(kCT, 1) value_pass(const __grid_constant__ Args a) {
  using Gm = Geo<D, G>;
  constexpr int SG = Gm::SG;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(smem);
  long long* wpre = reinterpret_cast<long long*>(smem + Gm::OFF_WPRE);          // [units + 1] weight prefix
  int* cfirst = reinterpret_cast<int*>(smem + Gm::OFF_UNIT);                    // centroid partial base per unit
  int* cnsh = cfirst + kMaxUnits;                                               // centroid shares per unit
  int* vfirst = cnsh + kMaxUnits;                                               // value partial base per unit
  int* vnsh = vfirst + kMaxUnits;                                               // value shares per unit
  int* lens = reinterpret_cast<int*>(smem + Gm::OFF_HDR);                       // [units][2]: exact / subtraction rows
  int* red = reinterpret_cast<int*>(smem + Gm::OFF_RED);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, hq = lane >> 2;
  const int c = blockIdx.x, grid = gridDim.x;
  const float qk2 = a.scale * kLog2e;

  // everything below reads what the centroid pass wrote
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  // per-unit weights and their prefix
  long long* wtmp = reinterpret_cast<long long*>(smem);   // the first slot is not in use yet
  for (int u = threadIdx.x; u <= a.units; u += kCT) {
    const int nt = u < a.units ? __ldcg(a.hdr + 2 * u) : 0, ns = u < a.units ? __ldcg(a.hdr + 2 * u + 1) : 0;
    if (u < a.units) { lens[2 * u] = nt; lens[2 * u + 1] = ns; }
    wtmp[u] = u < a.units ? 1 + 2LL * nt + ns : 0LL;
  }
  cbar();
  scan_units<long long>(wtmp, wpre, a.units + 1, 0LL, reinterpret_cast<long long*>(red + 64));
  const long long WT = wpre[a.units];
  unit_tables(a, grid, cfirst, cnsh, wpre, vfirst, vnsh, kCT);
  cbar();
  scan_units<int>(cnsh, cfirst, a.units, 0, red + 64);
  scan_units<int>(vnsh, vfirst, a.units, 0, red + 64);
  for (int u = threadIdx.x; u < a.units; u += kCT) vfirst[u] = a.part_v + vfirst[u] * kCW;
  cbar();

  const long long lo = share_lo(c, WT, grid), hi = share_lo(c + 1, WT, grid);
  // the unit holding lo
  int u0 = 0;
  {
    int l = 0, h = a.units - 1;
    while (l < h) { const int mid = (l + h + 1) >> 1; if (wpre[mid] <= lo) l = mid; else h = mid - 1; }
    u0 = l;
  }
  VCursor cur{lo, hi, u0, false};
  // next chunk of the share: rows of one unit and one kind, at most kRows
  auto next = [&](VChunk& ch) -> bool {
    while (cur.pos < cur.hi && cur.u < a.units) {
      const int u = cur.u;
      const long long ub = wpre[u], ue = wpre[u + 1];
      const int n_tok = lens[2 * u], n_sub = lens[2 * u + 1];
      const long long rel = cur.pos - ub, rel_end = (cur.hi < ue ? cur.hi : ue) - ub;
      ch.unit = u;
      ch.seg = share_index(c, ub, WT, grid);
      ch.first = !cur.started;
      // exact rows r with 1 + 2r in [rel, rel_end)
      const long long t_lo = rel <= 1 ? 0 : (rel - 1 + 1) / 2, t_hi = rel_end <= 1 ? 0 : (rel_end - 1 + 1) / 2;
      const long long tl = min((long long)n_tok, t_lo), th = min((long long)n_tok, t_hi);
      const long long s_lo = max(0LL, rel - 1 - 2LL * n_tok), s_hi = max(0LL, rel_end - 1 - 2LL * n_tok);
      const long long sl = min((long long)n_sub, s_lo), sh = min((long long)n_sub, s_hi);
      if (tl < th) {
        ch.kind = 0; ch.p0 = (int)tl; ch.cnt = (int)min((long long)kRows, th - tl);
        cur.pos = ub + 1 + 2LL * (tl + ch.cnt);                       // first weight after the chunk's rows
        if (cur.pos > ub + rel_end) cur.pos = ub + rel_end;
      } else if (sl < sh) {
        ch.kind = 1; ch.p0 = (int)sl; ch.cnt = (int)min((long long)kRows, sh - sl);
        cur.pos = ub + 1 + 2LL * n_tok + sl + ch.cnt;
        if (cur.pos > ub + rel_end) cur.pos = ub + rel_end;
      } else {
        // nothing left of this unit in the share (or only its placeholder)
        ch.kind = 2; ch.p0 = 0; ch.cnt = 0;
        cur.pos = ub + rel_end;
      }
      // is this the last chunk of the share of unit u?
      bool more = false;
      if (cur.pos < ub + rel_end) {
        const long long r2 = cur.pos - ub;
        const long long t2 = min((long long)n_tok, r2 <= 1 ? 0 : r2 / 2);
        const long long s2 = min((long long)n_sub, max(0LL, r2 - 1 - 2LL * n_tok));
        more = t2 < th || s2 < sh;
      }
      ch.last = !more;
      if (!more) {
        cur.pos = ub + rel_end;
        cur.u = u + 1;
        cur.started = false;
      } else {
        cur.started = true;
      }
      if (ch.kind == 2 && !ch.first) continue;   // a placeholder after rows of the unit adds nothing
      return true;
    }
    return false;
  };

  // per-warp copy pipeline: chunk i of the share in slot i % kNS; this warp owns rows [16w, 16w + 16)
  const int r16 = warp * 16;
  WarpSoftmax<D, G> ws;
  ws.reset();
  VChunk q[kNS];
  bool qv[kNS];
  int qsrc[kNS];
  float qbias[kNS];
  int* bc = red + 120;
  // load the row sources (lanes 0..15) and subtraction biases of a chunk
  auto load_src = [&](const VChunk& ch, int& src, float& bias) {
    src = 0;
    bias = 0.f;
    const int r = r16 + (lane & 15);
    if (ch.kind < 2 && lane < 16 && r < ch.cnt) {
      if (ch.kind == 0) {
        src = __ldcg(a.tok_src + (size_t)ch.unit * a.max_tokens + ch.p0 + r);
        if ((unsigned)src >= (unsigned)a.max_tokens) { set_error(a.err, E_BAD_LIST); src = 0; }
      } else {
        src = __ldcg(a.sub_src + (size_t)ch.unit * a.capc + ch.p0 + r);
        bias = __ldcg(a.sub_bias + (size_t)ch.unit * a.capc + ch.p0 + r);
        if ((unsigned)src >= (unsigned)a.slots) { set_error(a.err, E_BAD_LIST); src = 0; }
      }
    }
  };
  // copies of this warp's rows of chunk ch into slot s
  auto copy = [&](const VChunk& ch, int s, int src) {
    if (ch.kind < 2 && r16 < ch.cnt) {
      const uint32_t base = sb + s * Gm::SLOT;
      const bool tok = ch.kind == 0;
      const size_t ub = (size_t)ch.unit * (tok ? (size_t)a.max_tokens : (size_t)a.slots);
      const __nv_bfloat16* Kb = a.Kp + ub * D;
      const __nv_bfloat16* Vb = (tok ? a.Vp : a.Vc) + ub * D;
      constexpr int RPI = 32 / Gm::CPR;   // rows per warp instruction
      const int cc = lane % Gm::CPR;
#pragma unroll
      for (int k = 0; k < 16 / RPI; ++k) {
        const int rl = k * RPI + lane / Gm::CPR;     // row within the warp's 16
        const int rs = __shfl_sync(kFull, src, rl);
        const int r = r16 + rl;
        const bool v = r < ch.cnt;
        const size_t o = (size_t)rs * D + cc * 8;
        if (tok) cp16(base + swz(r, cc), v ? (const void*)(Kb + o) : (const void*)a.Kp, v);
        cp16(base + Gm::AREA + swz(r, cc), v ? (const void*)(Vb + o) : (const void*)a.Vp, v);
      }
      if (!tok) {
        // the subtraction rows' scores, SG floats each, in the key area
        const float* Sb = a.S + (size_t)ch.unit * a.slots * SG;
        for (int i = lane; i < 16 * (SG / 4); i += kWarp) {
          const int rl = i / (SG / 4), c4 = i % (SG / 4);
          const int rs = __shfl_sync(0xffffffffu >> (32 - min(32, 16 * (SG / 4))), src, rl);
          const int r = r16 + rl;
          cp16(base + r * SG * 4 + c4 * 16, Sb + (size_t)rs * SG + c4 * 4, r < ch.cnt);
        }
      }
    }
    cp_commit();
  };

  // prologue: kNS - 1 chunks in flight
#pragma unroll
  for (int i = 0; i < kNS; ++i) {
    qv[i] = next(q[i]);
    if (!qv[i]) q[i] = VChunk{0, 2, 0, 0, 0, 0, 0, 0};
    load_src(q[i], qsrc[i], qbias[i]);
  }
#pragma unroll
  for (int i = 0; i < kNS - 1; ++i) copy(q[i], i, qsrc[i]);
  int unit_q = -1;
  for (int i = 0; qv[i % kNS]; ++i) {
    const int s = i % kNS;
    // the chunk kNS - 1 ahead goes into the slot computed last iteration
    copy(q[(i + kNS - 1) % kNS], (i + kNS - 1) % kNS, qsrc[(i + kNS - 1) % kNS]);
    cp_wait<kNS - 1>();
    __syncwarp();
    const VChunk ch = q[s];
    const float bias = qbias[s];
    if (ch.first) {
      if (ch.unit != unit_q) {
        ws.load_q(a.Q + (size_t)ch.unit * G * D, lane);
        unit_q = ch.unit;
      }
      ws.reset();
    }
    if (ch.kind < 2 && r16 < ch.cnt) {
      const uint32_t base = sb + s * Gm::SLOT;
      float z[2][2];
      if (ch.kind == 0) {
        ws.qk(base, r16, lane, z);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int ii = 0; ii < 2; ++ii) {
            const int r = r16 + nt * 8 + 2 * (lane & 3) + ii;
            z[nt][ii] = (hq < G && r < ch.cnt) ? z[nt][ii] * qk2 : -INFINITY;
          }
      } else {
        const float* Ss = reinterpret_cast<const float*>(smem + s * Gm::SLOT);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int ii = 0; ii < 2; ++ii) {
            const int rl = nt * 8 + 2 * (lane & 3) + ii;
            const int r = r16 + rl;
            const float b = __shfl_sync(kFull, bias, rl);
            z[nt][ii] = (hq < G && r < ch.cnt) ? Ss[r * SG + hq] * kLog2e + b : -INFINITY;
          }
      }
      ws.update(base + Gm::AREA, r16, lane, z, ch.kind == 0 ? 1.f : -1.f);
    }
    __syncwarp();   // this slot is reused for the chunk kNS ahead
    // refill the descriptor ring: chunk i + kNS takes slot s
    const bool more = qv[s] ? next(q[s]) : false;
    const VChunk done = ch;
    qv[s] = more;
    if (!more) q[s] = VChunk{0, 2, 0, 0, 0, 0, 0, 0};
    load_src(q[s], qsrc[s], qbias[s]);
    if (done.last) {
      // end of this CTA's share of the unit: the warps' partials, then the unit's ticket
      ws.store(a, vfirst[done.unit] + done.seg * kCW + warp, lane);
      cbar();
      if (threadIdx.x == 0) bc[0] = ticket(a.ctl + a.units + done.unit);
      __syncthreads();
      if (bc[0] == vnsh[done.unit] - 1) {
        // last share of the unit: merge all its partials (centroid and value pass) into the output rows
        const int u = done.unit;
        combine_unit<D, G>(a, u, cfirst[u] * kCW, cnsh[u] * kCW, vfirst[u], vnsh[u] * kCW);
      }
      __syncthreads();
    }
  }
  cp_wait_all();
}

}  // namespace stream

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
static inline size_t a256(size_t x) { return (x + 255) & ~(size_t)255; }

struct StreamLayout {
  int capc, SG, npart;
  size_t o_S, o_tok, o_ssrc, o_sbias, o_hdr, o_pm, o_pl, o_pacc, o_ctl, ctl_bytes, bytes;
};

static StreamLayout stream_layout(const mp_config& c, int slots) {
  StreamLayout L{};
  const size_t U = (size_t)c.batch * c.kv_heads;
  const int G = c.q_heads / c.kv_heads, D = c.head_dim;
  // partials: per pass one per (unit, share, warp), at most (grid + units) * kCW
  L.npart = 2 * (stream::kMaxGrid + (int)U) * stream::kCW;
  L.SG = (G + 3) / 4 * 4;
  L.capc = ((slots + 3) & ~3) + 64;
  size_t cur = 0;
  L.o_S = cur; cur = a256(cur + U * slots * L.SG * 4);
  L.o_tok = cur; cur = a256(cur + U * (size_t)c.max_tokens * 4);
  L.o_ssrc = cur; cur = a256(cur + U * L.capc * 4);
  L.o_sbias = cur; cur = a256(cur + U * L.capc * 4);
  L.o_hdr = cur; cur = a256(cur + U * 2 * 4);
  L.o_pm = cur; cur = a256(cur + (size_t)L.npart * G * 4);
  L.o_pl = cur; cur = a256(cur + (size_t)L.npart * G * 4);
  L.o_pacc = cur; cur = a256(cur + (size_t)L.npart * G * D * 4);
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
         (G == 1 || G == 2 || G == 4 || G == 8) && slots <= stream::kMaxSlots &&
         c.batch * c.kv_heads < stream::kMaxUnits;
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
static cudaError_t launch_stream_t(const stream::Args& a, int grid, cudaStream_t st) {
  using Gm = stream::Geo<D, G>;
  auto k1 = stream::centroid_pass<D, G>;
  auto k2 = stream::value_pass<D, G>;
  cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, Gm::SMEM);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, Gm::SMEM);
  if (e != cudaSuccess) return e;
  k1<<<grid, stream::kCT + kWarp, Gm::SMEM, st>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // the value pass is launched as a programmatic dependent of the centroid pass:
  // its CTAs may start while the last centroid CTAs finish, and wait
  // (griddepcontrol.wait) for that grid's completion before reading its results
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(stream::kCT);
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
static cudaError_t launch_stream_d(int G, const stream::Args& a, int grid, cudaStream_t st) {
  switch (G) {
    case 1: return launch_stream_t<D, 1>(a, grid, st);
    case 2: return launch_stream_t<D, 2>(a, grid, st);
    case 4: return launch_stream_t<D, 4>(a, grid, st);
    case 8: return launch_stream_t<D, 8>(a, grid, st);
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
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return MP_ECUDA;
  // one CTA per SM; the caller's split count (n_split > 0) overrides it
  int grid = prm->n_split > 0 ? prm->n_split : sms;
  grid = std::max(1, std::min(grid, stream::kMaxGrid));
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
  a.cpu = std::max(1, (a.slots_active + stream::kRows - 1) / stream::kRows);
  a.max_tokens = c.max_tokens;
  a.n_clustered = (int)idx->n_clustered;
  a.n_tail = (int)(idx->n_tokens - idx->n_clustered);
  a.scale = scale;
  a.budget = prm->budget;
  a.approx = (prm->flags & MP_NO_APPROX) == 0;
  a.capc = L.capc;
  a.S = reinterpret_cast<float*>(base + L.o_S);
  a.tok_src = reinterpret_cast<int32_t*>(base + L.o_tok);
  a.sub_src = reinterpret_cast<int32_t*>(base + L.o_ssrc);
  a.sub_bias = reinterpret_cast<float*>(base + L.o_sbias);
  a.hdr = reinterpret_cast<int32_t*>(base + L.o_hdr);
  a.pm = reinterpret_cast<float*>(base + L.o_pm);
  a.pl = reinterpret_cast<float*>(base + L.o_pl);
  a.pacc = reinterpret_cast<float*>(base + L.o_pacc);
  a.part_v = L.npart / 2;
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
  cudaError_t e = D == 128 ? launch_stream_d<128>(G, a, grid, st) : launch_stream_d<64>(G, a, grid, st);
  phase(2);
  return e == cudaSuccess ? MP_OK : MP_ECUDA;
}

}  // namespace mp
