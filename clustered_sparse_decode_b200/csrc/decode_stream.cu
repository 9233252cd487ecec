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
  CUtensorMap tmKV;            // Kp and Vp as one map (columns, rows, [half,] key/value): 8-row boxes, 128-byte swizzle
  const __nv_bfloat16* Q;      // [units*G][D]
  __nv_bfloat16* O;            // [units*G][D]
  const __nv_bfloat16* Kc;     // [units][slots][D]
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
  float* shat;                 // [units][slots] group score (max over the group's heads) of each slot
  int32_t* boxes;              // [units][max_tokens] packed 8-row boxes of the exact rows (box_pack)
  int32_t* sub_src;            // [units][capc] slot of each selected cluster (subtraction rows)
  float* sub_bias;             // [units][capc] log2 of its size
  int32_t* hdr;                // [units][2]: boxes, subtraction rows
  float* pm;                   // [npart][G] partial max (log2 units)
  float* pl;                   // [npart][G] partial normaliser
  float* pacc;                 // [npart][G][D] partial numerator
  int part_v;                  // first partial of the value pass (the centroid pass uses [0, part_v));
                               // per (unit u, share c, warp): (c + u) * kCW + warp (unique: shares are
                               // contiguous, so the overlapping (c, u) pairs form a staircase)
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
  // centroid pass: query rows, cluster offsets, meta; value pass: meta, biases, row sources
  static constexpr int AUX_C = QB + (kRows + 4) * 4 + 32;
  static constexpr int AUX_V = 64 + 2 * kRows * 4;
  static constexpr int AUX = AUX_C > AUX_V ? AUX_C : AUX_V;
  static constexpr int OFF_UNIT = OFF_AUX + kNS * AUX; // per unit and pass: first partial, number of shares
  static constexpr int OFF_WPRE = OFF_UNIT + kMaxUnits * 16;   // value pass: weight prefix over units
  static constexpr int OFF_HDR = (OFF_WPRE + (kMaxUnits + 1) * 8 + 15) / 16 * 16;   // value pass: stream lengths
  static constexpr int OFF_RED = OFF_HDR + kMaxUnits * 8;
  static constexpr int OFF_SRC = OFF_RED + 128 * 4;    // value pass: the producer's ring of 3 chunks' sources
  static constexpr int OFF_BAR = OFF_SRC + 3 * 2 * kRows * 4;   // (also: kVP producers x 3 x 16 box entries)
  static constexpr int SMEM = OFF_BAR + 2 * kNS * 8 + 16 + 1024;   // + alignment slack
  static_assert(D % 64 == 0, "rows are whole 64-column tiles");
  static_assert(kRows * SG * 4 <= AREA, "subtraction-row scores live in the key area");
  static_assert(AUX % 16 == 0, "16-byte aligned side areas");
  static_assert(OFF_AUX % 1024 == 0 && OFF_UNIT % 16 == 0 && OFF_WPRE % 16 == 0 && OFF_HDR % 16 == 0 &&
                    OFF_RED % 16 == 0 && OFF_SRC % 16 == 0 && OFF_BAR % 16 == 0,
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
// one 8-row box of the key and value stores: a 4-D (d = 128: columns, rows, half,
// key/value) or 3-D (d = 64: columns, rows, key/value) tensor map, coordinates {0, y, 0[, 0]}
template <int D>
__device__ __forceinline__ void tma_box_t(uint32_t dst, const CUtensorMap* tm, int y, uint32_t bar) {
  if constexpr (D == 128) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %2, %2}], [%4];\n"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(tm)), "r"(0), "r"(y), "r"(bar)
        : "memory");
  } else {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %2}], [%4];\n"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(tm)), "r"(0), "r"(y), "r"(bar)
        : "memory");
  }
}
// bring [p, p + bytes) into L2 (bytes: a multiple of 16, p 16-byte aligned)
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  if (bytes) asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(p), "r"(bytes) : "memory");
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

// Box-major chunk layout of the value pass: 16 boxes of 8 rows, box b at
// b * 32 D bytes holding its key rows, then its value rows, each as D/64
// 1024-byte atoms [8 rows][128 bytes] (one per 64 columns, 128-byte swizzle):
// the layout one TMA load of an 8-row box of both the key and the value store
// writes.  Offset of 16-byte chunk c of row r from the key (or value) part.
template <int D>
__device__ __forceinline__ uint32_t bswz(int r, int c) {
  return (r >> 3) * (32 * D) + (c >> 3) * 1024 + (r & 7) * 128 + (((c & 7) ^ (r & 7)) << 4);
}
// offset of chunk c of row r in the layout of the pass (BOX: the value pass's boxes)
template <bool BOX, int D>
__device__ __forceinline__ uint32_t lay(int r, int c) {
  if constexpr (BOX) return bswz<D>(r, c);
  else return swz(r, c);
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
// the s-th of the shares holding positions from xb on (with N >= grid every
// share is non-empty; with N < grid every non-empty share holds one position)
__device__ __forceinline__ int nth_share(int s, long long xb, long long N, int grid) {
  return N >= grid ? share_owner(xb, N, grid) + s : share_owner(xb + s, N, grid);
}

// ---------------------------------------------------------------------------
// Per-warp online softmax over 16-row tiles
// ---------------------------------------------------------------------------
// The 16 keys of a tile are the M rows of mma.sync m16n8k16 and 8 "columns" of
// query heads the N columns: S^T = K Q^T.  With G <= 4 the columns 4..7 repeat
// the heads of columns 0..3, so that every probability exists twice; the lanes
// holding columns 0..3 pass its bf16 value (hi) and the lanes holding 4..7 the
// bf16 rounding of the remainder (lo) into P.V, which therefore keeps ~16
// significant bits of each weight in one mma per 16 value columns (G = 8: the
// hi and lo parts go through two mma into the same accumulator).  The
// transpose from the S^T accumulator layout to the B-operand layout of P.V
// (keys as K) is movmatrix.trans on the packed bf16 pairs.
//
// The running max is lazy: a tile whose logits exceed this lane's max by at
// most 2^8 is folded with the old max (weights up to 256); only otherwise do
// the lanes of a column agree on a new max and rescale.
__device__ __forceinline__ uint32_t movtrans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

template <int D, int G>
struct WarpSoftmax {
  static constexpr bool DUP = G <= 4;  // columns 4..7 repeat the heads of columns 0..3
  static constexpr float kLazy = 8.f;  // log2 of the largest weight folded without a new max
  uint32_t qb[D / 16][2];      // B fragments of Q^T: [k-step][dims +0 | +8], column lane/4
  float acc[D / 16][4];        // numerator O^T: m-tile mt holds [d = 16 mt + lane/4 (+8)][column 2*(lane%4) (+1)]
  float m[2], l[2];            // running max (log2 units) and normaliser of this lane's two columns

  // the head of column 2 (lane % 4) + j, or -1 for an unused column
  __device__ static __forceinline__ int col_head(int lane, int j) {
    const int col = 2 * (lane & 3) + j;
    const int h = DUP ? (col & 3) : col;
    return h < G ? h : -1;
  }
  // this lane's columns carry the lo parts (the repeated columns 4..7)
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
  __device__ __forceinline__ void load_q(const P* q, int lane) {   // q: [G][D] bf16 (global or shared)
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
  template <bool BOX = false>
  __device__ __forceinline__ void qk(uint32_t kb, int r16, int lane, float (&z)[2][2]) const {
    float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};   // two accumulation chains
    const int row = r16 + (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t a0, a1, a2, a3;
      ldsm4(kb + lay<BOX, D>(row, 2 * ks + (lane >> 4)), a0, a1, a2, a3);
      if (ks & 1) mma16816_full(c1, a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
      else mma16816_full(c0, a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
    }
    z[0][0] = c0[0] + c1[0];
    z[0][1] = c0[1] + c1[1];
    z[1][0] = c0[2] + c1[2];
    z[1][1] = c0[3] + c1[3];
  }
  // Fold a tile with logits z (log2 units, -inf = no term) and weight sign into
  // the state: O^T += V^T P^T, the value rows' transpose as the A operand.
  template <bool BOX = false>
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
      ldsm4t(vb + lay<BOX, D>(r16 + (lane & 7) + 8 * (lane >> 4), 2 * mt + ((lane >> 3) & 1)), v0, v1, v2, v3);
      mma16816_full(acc[mt], v0, v1, v2, v3, b0, b1);
      if constexpr (!DUP) mma16816_full(acc[mt], v0, v1, v2, v3, c0, c1);
    }
  }
  // this warp's state as partial p: max and normaliser per head, numerator per head and column
  __device__ __forceinline__ void store(const Args& a, int p, int lane) const {
    float lt0 = l[0], lt1 = l[1];
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      lt0 += __shfl_xor_sync(kFull, lt0, o);
      lt1 += __shfl_xor_sync(kFull, lt1, o);
    }
    const bool wr = !lo_cols(lane);
    const int hd0 = col_head(lane, 0), hd1 = col_head(lane, 1), d0 = lane >> 2;
    if (wr && lane < 4) {
      if (hd0 >= 0) { a.pm[(size_t)p * G + hd0] = lt0 != 0.f ? m[0] : -INFINITY; a.pl[(size_t)p * G + hd0] = lt0; }
      if (hd1 >= 0) { a.pm[(size_t)p * G + hd1] = lt1 != 0.f ? m[1] : -INFINITY; a.pl[(size_t)p * G + hd1] = lt1; }
    }
    float* o0 = a.pacc + ((size_t)p * G + (hd0 < 0 ? 0 : hd0)) * D + d0;
    float* o1 = a.pacc + ((size_t)p * G + (hd1 < 0 ? 0 : hd1)) * D + d0;
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

// Merge all partials of unit u into its output rows: kCW per share of the
// centroid pass (chunks [u cpu, (u + 1) cpu) of units cpu) and of the value
// pass (nvs shares from weight position vb of VN), share c's at (c + u) kCW.
// (compute threads; one thread per 4 columns of a head, online over the partials)
template <int D, int G>
__device__ void combine_unit(const Args& a, int u, int grid, long long vb, int nvs, long long VN) {
  constexpr int kCB = 8;                    // partials loaded per round
  const long long CN = (long long)a.units * a.cpu, cb = (long long)u * a.cpu;
  const int ncs = shares_of(cb, cb + a.cpu, CN, grid);
  const int n = (ncs + nvs) * kCW;
  // partial j: share j / kCW of the concatenated lists, warp j % kCW (the
  // shares of a list are consecutive CTAs unless the list has empty shares)
  const int cc0 = share_owner(cb, CN, grid), vc0 = share_owner(vb, VN, grid);
  const bool cseq = CN >= grid, vseq = VN >= grid;
  auto part = [&](int j) -> size_t {
    const int sh = j / kCW, w = j % kCW;
    if (sh < ncs) return (size_t)((cseq ? cc0 + sh : nth_share(sh, cb, CN, grid)) + u) * kCW + w;
    const int s2 = sh - ncs;
    return (size_t)a.part_v + (size_t)((vseq ? vc0 + s2 : nth_share(s2, vb, VN, grid)) + u) * kCW + w;
  };
  // SPLIT adjacent threads share an output group of 4 columns of a head: each
  // folds every SPLIT-th partial, then the states merge across the lanes
  constexpr int NE = G * D / 4;
  constexpr int SPLIT = NE >= kCT ? 1 : (kCT / NE >= 8 ? 8 : kCT / NE);
  const int part_i = threadIdx.x % SPLIT;
  for (int e = threadIdx.x / SPLIT; e < NE; e += kCT / SPLIT) {
    const int g = (e * 4) / D, d = (e * 4) % D;
    float M = -INFINITY, L = 0.f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j0 = part_i; j0 < n; j0 += kCB * SPLIT) {
      float mj[kCB], lj[kCB];
      float4 xj[kCB];
#pragma unroll
      for (int k = 0; k < kCB; ++k) {
        const int j = j0 + k * SPLIT;
        const size_t p = part(min(j, n - 1));
        mj[k] = j < n ? __ldcg(a.pm + p * G + g) : -INFINITY;
        lj[k] = __ldcg(a.pl + p * G + g);
        xj[k] = __ldcg(reinterpret_cast<const float4*>(a.pacc + (p * G + g) * D + d));
      }
      float Mn = M;
#pragma unroll
      for (int k = 0; k < kCB; ++k) Mn = fmaxf(Mn, mj[k]);
      if (Mn == -INFINITY) continue;
      const float s0 = M == -INFINITY ? 0.f : ex2(M - Mn);
      o.x *= s0; o.y *= s0; o.z *= s0; o.w *= s0;
      L *= s0;
#pragma unroll
      for (int k = 0; k < kCB; ++k) {
        const float f = mj[k] == -INFINITY ? 0.f : ex2(mj[k] - Mn);
        o.x += f * xj[k].x; o.y += f * xj[k].y; o.z += f * xj[k].z; o.w += f * xj[k].w;
        L += f * lj[k];
      }
      M = Mn;
    }
#pragma unroll
    for (int sft = 1; sft < SPLIT; sft <<= 1) {
      const float M2 = __shfl_xor_sync(kFull, M, sft), L2 = __shfl_xor_sync(kFull, L, sft);
      const float x2 = __shfl_xor_sync(kFull, o.x, sft), y2 = __shfl_xor_sync(kFull, o.y, sft);
      const float z2 = __shfl_xor_sync(kFull, o.z, sft), w2 = __shfl_xor_sync(kFull, o.w, sft);
      const float Mn = fmaxf(M, M2);
      const float f1 = M == -INFINITY ? 0.f : ex2(M - Mn), f2 = M2 == -INFINITY ? 0.f : ex2(M2 - Mn);
      o.x = o.x * f1 + x2 * f2; o.y = o.y * f1 + y2 * f2; o.z = o.z * f1 + z2 * f2; o.w = o.w * f1 + w2 * f2;
      L = L * f1 + L2 * f2;
      M = Mn;
    }
    if (part_i == 0) {
      const float inv = L > 0.f ? 1.f / L : 0.f;
      __nv_bfloat16* out = a.O + ((size_t)u * G + g) * D + d;
      *reinterpret_cast<uint2*>(out) = make_uint2(pack_bf16(o.x * inv, o.y * inv), pack_bf16(o.z * inv, o.w * inv));
    }
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
// An 8-row box of the store, packed: first row g (25 bits), valid rows [lo, hi)
// of the box (lo: 3 bits, hi - 1: 3 bits).  Box b of the run [st, st + cnt):
// rows st + 8b .. + 7, except a partial last box, which ends at the run's end
// (its first 8 - cnt % 8 rows repeat the previous box, or belong to the rows
// before the run, and are not valid); a run of fewer than 8 rows that starts
// within the first 8 rows takes rows 0..7 instead.  No box reaches past the
// run's end unless the run lies in rows 0..7, so with at least 8 rows held no
// box reads a row that was never written.
__device__ __forceinline__ int32_t box_entry(int st, int cnt, int b) {
  const int nb = (cnt + 7) >> 3, rem = cnt & 7;
  int g = st + 8 * b, lo = 0, hi = 8;
  if (b == nb - 1 && rem) {
    g = st + cnt - 8;
    lo = 8 - rem;
    if (g < 0) { g = 0; lo = st; hi = st + rem; }
  }
  return g | (lo << 25) | ((hi - 1) << 28);
}
__device__ __forceinline__ int box_row(int32_t e) { return e & ((1 << 25) - 1); }
__device__ __forceinline__ int box_lo(int32_t e) { return (e >> 25) & 7; }
__device__ __forceinline__ int box_hi(int32_t e) { return ((e >> 28) & 7) + 1; }

template <int kD, int G, int SG>
__device__ void select_unit(const Args& a, int u, int* red, int* hist) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int slots = a.slots;
  const int spt = (slots + kCT - 1) / kCT;
  const int s0 = tid * spt;
  const int32_t* offu = a.off + (size_t)u * (slots + 1);

  uint32_t key[kMaxSpt];
  int w[kMaxSpt];
  int st0[kMaxSpt];
  int wsum = 0;
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  // loads in batches of 8 slots, unconditional (clamped) so that they issue back to back
  const float* Hu = a.shat + (size_t)u * slots;
#pragma unroll
  for (int k0 = 0; k0 < kMaxSpt; k0 += 8) {
    if (k0 < spt) {
      int o[9];
      float sv[8];
#pragma unroll
      for (int k = 0; k <= 8; ++k) o[k] = __ldg(offu + min(s0 + k0 + k, slots));
#pragma unroll
      for (int k = 0; k < 8; ++k) sv[k] = __ldcg(Hu + min(s0 + k0 + k, slots - 1));
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int c = s0 + k0 + k;
        const bool in = k0 + k < spt && c < slots;
        const int cnt = in ? o[k + 1] - o[k] : 0;
        const float sh = sv[k];
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
  int need = 0, ntie = 0;
  bool resolved = false;
  int above = 0;                                            // weight of the keys above tau
  if (mode == 2) {
    // First try: 256 bins of equal width in score between the smallest and the
    // largest candidate score (the bin index is monotone in the score, so a
    // higher bin holds only higher keys); one warp finds the bin where the
    // weight from the top crosses the budget, and if at most 32 candidates fall
    // in it, sorts them by (key descending, slot ascending) and takes tau from
    // the running weight.  Otherwise the radix descent below decides.
    const float smin = key_score(kmin), smax = key_score(kmax);
    const float span = smax - smin, inv = 256.f / span;
    if (isfinite(smin) && isfinite(smax) && span > 0.f && isfinite(span) && isfinite(inv)) {
      auto fbin = [&](uint32_t kk) { return min(255, (int)((key_score(kk) - smin) * inv)); };
      int* lst = hist + 256;                                // [32][3] candidates of the crossing bin
      for (int i = tid; i < 256; i += kCT) hist[i] = 0;
      if (tid == 0) red[3] = 0;
      cbar();
#pragma unroll
      for (int k = 0; k < kMaxSpt; ++k)
        if (w[k] > 0) atomicAdd(hist + fbin(key[k]), w[k]);
      cbar();
      if (warp == 0) {
        int bl[8], ls = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) { bl[i] = hist[8 * lane + i]; ls += bl[i]; }
        int suf = ls;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_down_sync(kFull, suf, o);
          if (lane + o < 32) suf += y;
        }
        int run = suf - ls, found = -1, ab = 0;
#pragma unroll
        for (int i = 7; i >= 0; --i) {
          if (found < 0 && run + bl[i] >= a.budget) { found = 8 * lane + i; ab = run; }
          run += bl[i];
        }
        const unsigned m = __ballot_sync(kFull, found >= 0);
        const int src = 31 - __clz(m);
        const int fb = __shfl_sync(kFull, found, src), fa = __shfl_sync(kFull, ab, src);
        if (lane == 0) { red[0] = fb; red[1] = fa; }
      }
      cbar();
      const int fb = red[0], ab = red[1];
#pragma unroll
      for (int k = 0; k < kMaxSpt; ++k)
        if (w[k] > 0 && fbin(key[k]) == fb) {
          const int pos = atomicAdd(red + 3, 1);
          if (pos < 32) { lst[3 * pos] = (int)key[k]; lst[3 * pos + 1] = s0 + k; lst[3 * pos + 2] = w[k]; }
        }
      cbar();
      const int nc = red[3];
      if (nc <= 32) {
        if (warp == 0) {
          // lane l holds candidate l; empty lanes sort last with weight 0
          uint64_t v = lane < nc ? ((uint64_t)(uint32_t)lst[3 * lane] << 32) | (uint32_t)(0xffffffffu - (uint32_t)lst[3 * lane + 1])
                                 : 0ull;
          int wl = lane < nc ? lst[3 * lane + 2] : 0;
          // bitonic sort, descending
#pragma unroll
          for (int kk = 2; kk <= 32; kk <<= 1) {
#pragma unroll
            for (int jj = kk >> 1; jj > 0; jj >>= 1) {
              const uint64_t ov = __shfl_xor_sync(kFull, v, jj);
              const int ow = __shfl_xor_sync(kFull, wl, jj);
              const bool up = ((lane & kk) == 0) == ((lane & jj) == 0);   // this lane keeps the larger
              if (up ? ov > v : ov < v) { v = ov; wl = ow; }
            }
          }
          int inc = wl;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(kFull, inc, o);
            if (lane >= o) inc += y;
          }
          const unsigned cross = __ballot_sync(kFull, lane < nc && ab + inc >= a.budget);
          const uint32_t t = (uint32_t)(__shfl_sync(kFull, v, __ffs(cross) - 1) >> 32);
          const uint32_t kl = (uint32_t)(v >> 32);
          const int gt = __reduce_add_sync(kFull, lane < nc && kl > t ? wl : 0);
          const int nt = __popc(__ballot_sync(kFull, lane < nc && kl == t));
          if (lane == 0) { red[0] = (int)t; red[1] = ab + gt; red[2] = nt; }
        }
        cbar();
        tau = (uint32_t)red[0];
        above = red[1];
        ntie = red[2];
        resolved = true;
      }
      cbar();
    }
  }
  if (mode == 2 && !resolved) {
    // Radix descent over the interval [lo, lo + 2^nb) holding all candidates,
    // 8 bits a level: a 256-bin histogram of weights (and, on the last level,
    // where bins are single key values, of key counts), then warp 0 finds the
    // bin where the weight from the top crosses the budget.
    uint32_t lo = kmin;
    int nb = kmax == kmin ? 0 : 32 - __clz(kmax - kmin);
    above = 0;                                              // weight of the keys above the interval
    int* hcnt = hist + 256;
    ntie = -1;                                              // keys at tau: unknown unless a level ends on single keys
    while (nb > 0) {
      const int sh = max(nb - 8, 0);
      for (int i = tid; i < 256; i += kCT) { hist[i] = 0; hcnt[i] = 0; }
      cbar();
      const unsigned long long hi_excl = (unsigned long long)lo + (1ull << nb);
#pragma unroll
      for (int k = 0; k < kMaxSpt; ++k)
        if (w[k] > 0 && key[k] >= lo && (unsigned long long)key[k] < hi_excl) {
          const int bin = (int)((key[k] - lo) >> sh);
          atomicAdd(hist + bin, w[k]);
          if (sh == 0) atomicAdd(hcnt + bin, 1);
        }
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
        if (lane == 0) { red[0] = fb; red[1] = fa; red[2] = hcnt[fb]; }
      }
      cbar();
      const int b = red[0];
      above = red[1];
      if (sh == 0) ntie = red[2];     // the bins of this level were single key values
      lo += (uint32_t)b << sh;
      nb = sh;
      cbar();
    }
    tau = lo;
  }
  if (mode == 2) need = a.budget - above;   // >= 1 tokens still to take among the ties at tau
  int tw = 0;
  if (mode == 2) {
#pragma unroll
    for (int k = 0; k < kMaxSpt; ++k) tw += (key[k] == tau && w[k] > 0) ? w[k] : 0;
  }
  // the crossing cluster is taken whole; only several clusters at exactly tau
  // need their order (slot order: an exclusive scan of their weights)
  int tie_before = 0, e2, t1, t2;
  if (mode == 2 && ntie != 1) cscan2(tw, 0, tie_before, e2, t1, t2, red);
  uint32_t selbits = 0u;
  int nsel = 0;
#pragma unroll
  for (int k = 0; k < kMaxSpt; ++k) {
    if (w[k] > 0) {
      bool s = false;
      if (mode == 1) s = true;
      else if (mode == 2) {
        if (key[k] > tau) s = true;
        else if (key[k] == tau) { s = tie_before < need; tie_before += w[k]; }
      }
      if (s) { selbits |= 1u << k; ++nsel; }
    }
  }
  // the exact rows as 8-row boxes of the store: per selected cluster (slot order), then the tail
  int nbx = 0;
#pragma unroll
  for (int k = 0; k < kMaxSpt; ++k)
    if ((selbits >> k) & 1u) nbx += (w[k] + 7) >> 3;
  int box_base, sub_base, box_total, sel_total;
  cscan2(nbx, nsel, box_base, sub_base, box_total, sel_total, red);

  int32_t* bx = a.boxes + (size_t)u * a.max_tokens;
  int32_t* ssrc = a.sub_src + (size_t)u * a.capc;
  float* sbias = a.sub_bias + (size_t)u * a.capc;
  if (a.sel_mask_out) {
    for (int k = 0; k < spt; ++k)
      if (s0 + k < slots) a.sel_mask_out[(size_t)u * slots + s0 + k] = (selbits >> k) & 1u;
  }
  // one compact loop over this thread's selected clusters (offsets re-read: L1 hits)
  uint32_t selrem = selbits;
#pragma unroll 1
  while (selrem) {
    const int k = __ffs(selrem) - 1;
    selrem &= selrem - 1;
    const int st = __ldg(offu + s0 + k), cnt = __ldg(offu + s0 + k + 1) - st;
    const int nb = (cnt + 7) >> 3;
#pragma unroll 1
    for (int b = 0; b < nb; ++b) bx[box_base + b] = box_entry(st, cnt, b);
    box_base += nb;
    if (a.approx) {
      ssrc[sub_base] = s0 + k;
      sbias[sub_base] = log2f((float)cnt);
      ++sub_base;
    }
  }
  const int nbt = (a.n_tail + 7) >> 3;
  for (int b = tid; b < nbt; b += kCT) bx[box_total + b] = box_entry(a.n_clustered, a.n_tail, b);
  if (tid == 0) {
    a.hdr[2 * u] = box_total + nbt;
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
  int* red = reinterpret_cast<int*>(smem + Gm::OFF_RED);
  const uint32_t full0 = sb + Gm::OFF_BAR, empty0 = full0 + kNS * 8;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long NCH = (long long)a.units * a.cpu;
  const int c = blockIdx.x, grid = gridDim.x;
  const long long lo = share_lo(c, NCH, grid), hi = share_lo(c + 1, NCH, grid);
  const long long t_start = gtimer();
  auto aux = [&](int slot) { return smem + Gm::OFF_AUX + slot * Gm::AUX; };
  // value-pass tickets start at zero (the value pass reads them after this grid completes)
  if (c == 0)
    for (int u = threadIdx.x; u < a.units; u += blockDim.x) a.ctl[a.units + u] = 0;

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
      const bool wr = !WarpSoftmax<D, G>::lo_cols(lane);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int r = r16 + WarpSoftmax<D, G>::zrow(lane, i);
        const int n = r < cm.cnt ? offs[r + 1] - offs[r] : 0;
        const float lg = log2f((float)n);
        float gmax = -INFINITY;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int h = WarpSoftmax<D, G>::col_head(lane, j);
          const float S = z[i][j] * a.scale;
          if (wr && h >= 0 && r < cm.cnt) Srow[(size_t)r * SG + h] = S;
          if (wr && h >= 0) gmax = fmaxf(gmax, S);
          z[i][j] = (a.approx && n > 0 && h >= 0) ? S * kLog2e + lg : -INFINITY;
        }
        // the group score of the row: max over the four lanes holding its columns
        gmax = fmaxf(gmax, __shfl_xor_sync(kFull, gmax, 1));
        gmax = fmaxf(gmax, __shfl_xor_sync(kFull, gmax, 2));
        if ((lane & 3) == 0 && r < cm.cnt) a.shat[(size_t)u * a.slots + cm.p0 + r] = gmax;
      }
      // without centroid terms the value rows are not loaded: nothing to fold
      if (a.approx) ws.update(dst + Gm::AREA, r16, lane, z, 1.f);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty0 + 8 * slot);
    if (cm.flags & 2) {
      // end of this CTA's share of unit u: the warps' partials, then the unit's ticket
      ws.store(a, (c + u) * kCW + warp, lane);
      cbar();
      if (threadIdx.x == 0) bc[0] = ticket(a.ctl + u);
      cbar();
      const int t = bc[0];
      const int ncs = shares_of((long long)u * a.cpu, (long long)(u + 1) * a.cpu, NCH, grid);
      if ((t < 0 || t >= ncs) && threadIdx.x == 0) set_error(a.err, E_SCRATCH);
      if (t == ncs - 1)
        select_unit<D, G, SG>(a, u, red, reinterpret_cast<int*>(smem + Gm::OFF_WPRE));
      cbar();
    }
  }
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

// ---------------------------------------------------------------------------
// Value pass: grid CTAs of kCT compute threads + one producer warp
// ---------------------------------------------------------------------------
// Stream of unit u in weight units: 1 (a placeholder, so that every unit is in
// exactly one share even when it has no rows), kWB per 8-row box of exact rows,
// 1 per subtraction row.  A box or row belongs to the share that holds its first
// weight.  A chunk is up to kBoxes boxes, or up to kRows subtraction rows, of one unit.
constexpr int kWB = 16;
constexpr int kBoxes = kRows / 8;
// Producer warps of the value pass: one per ring slot.  Producer p fills chunks
// k = p (mod kVP), all in slot p, and so waits on the phases of slot p's empty
// barrier in order; with more producers than slots a producer could test the
// parity of a phase two completions ahead of the slot and pass its wait early.
constexpr int kVP = kNS;
static_assert(kVP <= kNS, "a producer's empty-barrier waits stay in phase order");

struct VChunk {
  int unit, kind, p0, cnt;     // kind 0 boxes, 1 subtraction rows, 2 empty (unit placeholder), 3 end of the share
  int first, last, seg, valid; // first / last chunk of this CTA's share of the unit; share index; 0: past the share
};


// What the producer tells the compute warps about the chunk in a slot (side area:
// this, then kRows biases, then kRows row sources).
struct VMeta {
  int unit, kind, cnt, flags;  // cnt: boxes loaded (an even number) or subtraction rows; flags 1 first, 2 last
  int seg, pad0, pad1, pad2;
  uint8_t lo[kBoxes], hi[kBoxes];   // valid rows [lo, hi) of each box
};
constexpr int kVMetaBytes = 64;
static_assert(sizeof(VMeta) <= kVMetaBytes, "value-pass meta");

template <int D, int G>
__global__ void __launch_bounds__(kCT + kVP * kWarp, 1) value_pass(const __grid_constant__ Args a) {
  using Gm = Geo<D, G>;
  constexpr int SG = Gm::SG;
  constexpr int kBoxB = 32 * D;        // one 8-row box: key rows, then value rows
  static_assert(kBoxes * kBoxB == Gm::SLOT, "a slot holds kBoxes boxes");
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(smem);
  long long* wpre = reinterpret_cast<long long*>(smem + Gm::OFF_WPRE);          // [units + 1] weight prefix
  int* lens = reinterpret_cast<int*>(smem + Gm::OFF_HDR);                       // [units][2]: boxes / subtraction rows
  int* red = reinterpret_cast<int*>(smem + Gm::OFF_RED);
  const uint32_t full0 = sb + Gm::OFF_BAR, empty0 = full0 + kNS * 8;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x, grid = gridDim.x;
  const float qk2 = a.scale * kLog2e;
  const long long t_start = gtimer();
  auto side = [&](int slot) { return smem + Gm::OFF_AUX + slot * Gm::AUX; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNS; ++i) {
      mbar_init(full0 + 8 * i, kWarp + 1);   // the producer lanes' copy-tracking arrivals + lane 0's (+ TMA bytes)
      mbar_init(empty0 + 8 * i, kCW);        // one arrival per compute warp
    }
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  // everything below reads what the centroid pass wrote
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  // the centroid pass is complete: its tickets go back to zero for the next step
  if (c == 0)
    for (int u = threadIdx.x; u < a.units; u += blockDim.x) a.ctl[u] = 0;
  if (warp < kCW) {
    // per-unit weights and their prefix
    long long* wtmp = reinterpret_cast<long long*>(smem);   // the first slot is not in use yet
    for (int u = threadIdx.x; u <= a.units; u += kCT) {
      const int nb = u < a.units ? __ldcg(a.hdr + 2 * u) : 0, ns = u < a.units ? __ldcg(a.hdr + 2 * u + 1) : 0;
      if (u < a.units) { lens[2 * u] = nb; lens[2 * u + 1] = ns; }
      wtmp[u] = u < a.units ? 1 + (long long)kWB * nb + ns : 0LL;
    }
    cbar();
    scan_units<long long>(wtmp, wpre, a.units + 1, 0LL, reinterpret_cast<long long*>(red + 64));
  }
  __syncthreads();
  const long long WT = wpre[a.units];
  const long long lo = share_lo(c, WT, grid), hi = share_lo(c + 1, WT, grid);

  if (warp >= kCW) {
    // ======================= producers =======================
    // kVP warps; chunk k of the share is produced by warp kCW + k % kVP, into slot
    // k % kNS = k % kVP (its own slot).  Every
    // producer walks the whole chunk sequence (cheap: the unit's spans are worked
    // out once per unit) and loads only its own chunks.
    const int pw = warp - kCW;
    int u = 0;
    {
      int l = 0, h = a.units - 1;
      while (l < h) { const int mid = (l + h + 1) >> 1; if (wpre[mid] <= lo) l = mid; else h = mid - 1; }
      u = l;
    }
    // this share's part of unit u: boxes [tl, th), subtraction rows [sl, sh), chunks, share index
    int tl = 0, th = 0, sl = 0, sh = 0, nbc = 0, nch = 0, seg = 0, ci = 0;
    auto span = [&]() {
      const long long ub = wpre[u], ue = wpre[u + 1];
      const int n_box = lens[2 * u], n_sub = lens[2 * u + 1];
      const long long rel = (lo > ub ? lo : ub) - ub, rel_end = (hi < ue ? hi : ue) - ub;
      // boxes b with first weight 1 + kWB b in [rel, rel_end); subtraction row s at weight 1 + kWB n_box + s
      const long long b_lo = rel <= 1 ? 0 : (rel - 1 + kWB - 1) / kWB;
      const long long b_hi = rel_end <= 1 ? 0 : (rel_end - 1 + kWB - 1) / kWB;
      tl = (int)min((long long)n_box, b_lo);
      th = (int)min((long long)n_box, b_hi);
      const long long sbase = 1 + (long long)kWB * n_box;
      sl = (int)min((long long)n_sub, max(0LL, rel - sbase));
      sh = (int)min((long long)n_sub, max(0LL, rel_end - sbase));
      nbc = (th - tl + kBoxes - 1) / kBoxes;
      nch = nbc + (sh - sl + kRows - 1) / kRows;
      if (nch == 0) nch = 1;                       // a share with none of the unit's rows still closes it
      seg = 0;
      ci = 0;
    };
    const bool any = lo < hi;
    if (any) span();
    // chunk descriptor at the cursor, then advance
    auto next = [&](VChunk& ch) {
      if (!any || u >= a.units || wpre[u] >= hi) { ch = VChunk{0, 3, 0, 0, 0, 0, 0, 0}; return; }
      ch.unit = u; ch.seg = seg; ch.first = ci == 0; ch.last = ci == nch - 1; ch.valid = 1;
      if (ci < nbc) { ch.kind = 0; ch.p0 = tl + ci * kBoxes; ch.cnt = min(kBoxes, th - ch.p0); }
      else if (tl + nbc * kBoxes < th || sl < sh) {
        const int j = ci - nbc;
        ch.kind = 1; ch.p0 = sl + j * kRows; ch.cnt = min(kRows, sh - ch.p0);
        if (ch.cnt <= 0) { ch.kind = 2; ch.p0 = 0; ch.cnt = 0; }
      } else { ch.kind = 2; ch.p0 = 0; ch.cnt = 0; }
      if (++ci == nch) {
        ++u;
        if (u < a.units && wpre[u] < hi) span();
      }
    };
    // this warp's chunks k = pw, pw + kVP, ...: box entries copied two own chunks ahead
    // into a ring of 3 (cp.async, one commit group per own chunk)
    int* pe = reinterpret_cast<int*>(smem + Gm::OFF_SRC) + pw * 3 * kBoxes;
    auto prefetch = [&](const VChunk& ch, int e) {
      if (ch.kind == 0 && lane < ch.cnt)
        cp4(smem_u32(pe + e * kBoxes + lane), a.boxes + (size_t)ch.unit * a.max_tokens + ch.p0 + lane);
      cp_commit();
    };
    // the next chunk of this warp (skipping the other producers' chunks).  The end
    // marker (kind 3, index K = the share's chunk count) is published by warp
    // K % kVP only (k = K); the other producers get k = -1 and stop without
    // touching the barriers, so that every arrival on a full barrier has landed
    // before the compute warps that wait on it can exit.
    int kc = 0;   // index of the chunk the cursor describes next
    auto next_own = [&](VChunk& ch, int& k) {
      for (;;) {
        VChunk t;
        next(t);
        const int kk = kc++;
        if (t.kind == 3) { ch = t; k = kk % kVP == pw ? kk : -1; return; }
        if (kk % kVP == pw) { ch = t; k = kk; return; }
      }
    };
    VChunk q0, q1, q2;
    int k0, k1, k2;
    next_own(q0, k0);
    prefetch(q0, 0);
    if (q0.kind != 3) next_own(q1, k1); else { q1 = q0; k1 = k0; }
    prefetch(q1, 1);
    for (int i = 0;; ++i) {
      if (k0 < 0) break;     // the end of the share, published by another producer
      const int k = k0, slot = k % kNS;
      const int* es = pe + (i % 3) * kBoxes;
      cp_wait<1>();          // this lane's copies of the chunk's entries have landed
      __syncwarp();          // ... and every lane's
      bool got = true;
      if (k >= kNS && lane == 0) {
        while (!(got = mbar_try(empty0 + 8 * slot, ((k / kNS) - 1) & 1))) {
          if (gtimer() - t_start > a.timeout_ns) { set_error(a.err, E_TIMEOUT); break; }
        }
      }
      if (!__shfl_sync(kFull, got ? 1 : 0, 0)) break;
      const VChunk ch = q0;
      unsigned char* sd = side(slot);
      VMeta* m = reinterpret_cast<VMeta*>(sd);
      float* sbias = reinterpret_cast<float*>(sd + kVMetaBytes);
      int* ssrc = reinterpret_cast<int*>(sd + kVMetaBytes + kRows * 4);
      const uint32_t dst = sb + slot * Gm::SLOT;
      int nload = 0;                 // boxes loaded: the chunk's, plus a masked copy of the last to an even count
      int32_t ent = 0;
      if (ch.kind == 0) {
        nload = (ch.cnt + 1) & ~1;
        ent = es[min(lane, ch.cnt - 1)];
        if ((unsigned)box_row(ent) + 8u > (unsigned)a.max_tokens) set_error(a.err, E_BAD_LIST);
        if (lane < kBoxes) {
          m->lo[lane] = lane < ch.cnt ? (uint8_t)box_lo(ent) : (uint8_t)0;
          m->hi[lane] = lane < ch.cnt ? (uint8_t)box_hi(ent) : (uint8_t)0;
        }
      } else if (ch.kind == 1) {
        // the subtraction rows' slots and biases (one chunk per unit: loaded here)
        for (int r = lane; r < kRows; r += kWarp) {
          int src = 0;
          float bias = 0.f;
          if (r < ch.cnt) {
            src = __ldcg(a.sub_src + (size_t)ch.unit * a.capc + ch.p0 + r);
            bias = __ldcg(a.sub_bias + (size_t)ch.unit * a.capc + ch.p0 + r);
          }
          if ((unsigned)src >= (unsigned)a.slots) { set_error(a.err, E_BAD_LIST); src = 0; }
          ssrc[r] = src;
          sbias[r] = bias;
        }
      }
      if (lane == 0) {
        m->unit = ch.unit; m->kind = ch.kind; m->cnt = ch.kind == 0 ? nload : ch.cnt;
        m->flags = (ch.first ? 1 : 0) | (ch.last ? 2 : 0);
        m->seg = ch.seg;
        if (nload > 0)
          asm volatile("mbarrier.expect_tx.shared::cta.b64 [%0], %1;\n" ::"r"(full0 + 8 * slot),
                       "r"((uint32_t)(nload * kBoxB))
                       : "memory");
      }
      __syncwarp();
      if (ch.kind == 0 && lane < nload) {
        // box lane: its 8 key rows and 8 value rows, all columns, in one load
        const int y = ch.unit * (int)a.max_tokens + box_row(ent);
        tma_box_t<D>(dst + lane * kBoxB, &a.tmKV, y, full0 + 8 * slot);
      } else if (ch.kind == 1) {
        // subtraction rows: value centroid rows and score rows; rows up to the 16-row tile end zero-filled
        const int rows = (ch.cnt + 15) & ~15;
        const __nv_bfloat16* Vb = a.Vc + (size_t)ch.unit * a.slots * D;
        const float* Sb = a.S + (size_t)ch.unit * a.slots * SG;
        constexpr int RPI = 32 / Gm::CPR;
        const int cc = lane % Gm::CPR;
        for (int r = lane / Gm::CPR; r < rows; r += RPI) {
          const bool v = r < ch.cnt;
          cp16(dst + kBoxB / 2 + bswz<D>(r, cc), Vb + (size_t)(v ? ssrc[r] : 0) * D + cc * 8, v);
        }
        for (int t = lane; t < ch.cnt * (SG / 4); t += kWarp) {
          const int r = t / (SG / 4), c4 = t % (SG / 4);
          cp16(dst + (r >> 3) * kBoxB + (r & 7) * SG * 4 + c4 * 16, Sb + (size_t)ssrc[r] * SG + c4 * 4, true);
        }
      }
      asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];\n" ::"r"(full0 + 8 * slot) : "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(full0 + 8 * slot);
      if (ch.kind == 3) break;
      // this warp's chunk after next: describe it and prefetch its entries
      if (q1.kind != 3) next_own(q2, k2); else { q2 = q1; k2 = k1; }
      prefetch(q2, (i + 2) % 3);
      q0 = q1; k0 = k1;
      q1 = q2; k1 = k2;
    }
    cp_wait_all();
    return;
  }

  // ======================= compute warps =======================
  const int r16 = warp * 16;
  WarpSoftmax<D, G> ws;
  ws.reset();
  int unit_q = -1;
  int* bc = red + 120;
  for (int k = 0;; ++k) {
    const int slot = k % kNS;
    bool got = true;
    while (!(got = mbar_try(full0 + 8 * slot, (k / kNS) & 1))) {
      if (gtimer() - t_start > 2 * a.timeout_ns) { set_error(a.err, E_TIMEOUT); break; }
    }
    if (!got) break;
    const unsigned char* sd = side(slot);
    const VMeta* m = reinterpret_cast<const VMeta*>(sd);
    const int kind = m->kind;
    if (kind == 3) break;
    const int u = m->unit, cnt = m->cnt, flags = m->flags;
    if (flags & 1) {
      if (u != unit_q) {
        ws.load_q(a.Q + (size_t)u * G * D, lane);
        unit_q = u;
      }
      ws.reset();
    }
    const uint32_t base = sb + slot * Gm::SLOT;
    if (kind == 0 && 2 * warp < cnt) {
      float z[2][2];
      ws.template qk<true>(base, r16, lane, z);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int bxi = 2 * warp + i;           // rows 8 i .. 8 i + 7 of this warp's tile are box bxi
        const int blo = m->lo[bxi], bhi = m->hi[bxi];
        const int rb = lane >> 2;               // row within the box
#pragma unroll
        for (int j = 0; j < 2; ++j)
          z[i][j] = (WarpSoftmax<D, G>::col_head(lane, j) >= 0 && rb >= blo && rb < bhi) ? z[i][j] * qk2 : -INFINITY;
      }
      ws.template update<true>(base + kBoxB / 2, r16, lane, z, 1.f);
    } else if (kind == 1 && r16 < cnt) {
      // the score rows of box b sit at the start of its key part
      const float* Ss = reinterpret_cast<const float*>(smem + slot * Gm::SLOT);
      const float* eb = reinterpret_cast<const float*>(sd + kVMetaBytes);
      float z[2][2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int r = r16 + WarpSoftmax<D, G>::zrow(lane, i);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int h = WarpSoftmax<D, G>::col_head(lane, j);
          z[i][j] = (h >= 0 && r < cnt) ? Ss[(r >> 3) * (kBoxB / 4) + (r & 7) * SG + h] * kLog2e + eb[r] : -INFINITY;
        }
      }
      ws.template update<true>(base + kBoxB / 2, r16, lane, z, -1.f);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty0 + 8 * slot);
    if (flags & 2) {
      // end of this CTA's share of the unit: the warps' partials, then the unit's ticket
      ws.store(a, a.part_v + (c + u) * kCW + warp, lane);
      cbar();
      if (threadIdx.x == 0) bc[0] = ticket(a.ctl + a.units + u);
      cbar();
      const int nvs = shares_of(wpre[u], wpre[u + 1], WT, grid);
      if ((bc[0] < 0 || bc[0] >= nvs) && threadIdx.x == 0) set_error(a.err, E_SCRATCH);
      if (bc[0] == nvs - 1) {
        // last share of the unit: merge all its partials (centroid and value pass) into the output rows;
        // every value share of the unit has taken its ticket, which goes back to zero
        combine_unit<D, G>(a, u, grid, wpre[u], nvs, WT);
        if (threadIdx.x == 0) a.ctl[a.units + u] = 0;
      }
      cbar();
    }
  }
}

}  // namespace stream

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
static inline size_t a256(size_t x) { return (x + 255) & ~(size_t)255; }

struct StreamLayout {
  int capc, SG, npart;
  size_t o_S, o_shat, o_tok, o_ssrc, o_sbias, o_hdr, o_pm, o_pl, o_pacc, o_ctl, ctl_bytes, bytes;
};

static StreamLayout stream_layout(const mp_config& c, int slots) {
  StreamLayout L{};
  const size_t U = (size_t)c.batch * c.kv_heads;
  const int G = c.q_heads / c.kv_heads, D = c.head_dim;
  // partials: per pass one per (unit, share, warp), at most (grid + units) * kCW
  L.npart = 2 * (stream::kMaxGrid + (int)U) * stream::kCW;
  L.SG = (G + 3) / 4 * 4;
  L.capc = ((slots + 3) & ~3) + 64;
  static_assert(2 * stream::kMaxUnits * 4 <= kScratchTicketBytes, "ticket words");
  L.o_ctl = 0;                                        // ticket words: zero between steps
  L.ctl_bytes = kScratchTicketBytes;
  size_t cur = kScratchTicketBytes;
  L.o_S = cur; cur = a256(cur + U * slots * L.SG * 4);
  L.o_shat = cur; cur = a256(cur + U * slots * 4);
  L.o_tok = cur; cur = a256(cur + U * (size_t)c.max_tokens * 4);
  L.o_ssrc = cur; cur = a256(cur + U * L.capc * 4);
  L.o_sbias = cur; cur = a256(cur + U * L.capc * 4);
  L.o_hdr = cur; cur = a256(cur + U * 2 * 4);
  L.o_pm = cur; cur = a256(cur + (size_t)L.npart * G * 4);
  L.o_pl = cur; cur = a256(cur + (size_t)L.npart * G * 4);
  L.o_pacc = cur; cur = a256(cur + (size_t)L.npart * G * D * 4);
  L.bytes = cur;
  return L;
}

size_t stream_scratch_bytes(const mp_config& c, int slots) { return stream_layout(c, slots).bytes; }

// The index shapes the two-pass kernels take: flat bf16, d 64 or 128, G in {1, 2, 4, 8},
// at most kMaxSlots slots and fewer than kMaxUnits units, store rows addressable by
// the tensor maps (int32 row coordinates, 25-bit box rows), and at least 8 tokens
// held (no 8-row box of the store reaches a row that was never written).
bool stream_supported(const mp_config& c, int slots, int64_t n_tokens) {
  const int G = c.q_heads / c.kv_heads;
  const int64_t U = (int64_t)c.batch * c.kv_heads;
  return c.levels == 1 && c.dtype == MP_BF16 && (c.head_dim == 64 || c.head_dim == 128) &&
         (G == 1 || G == 2 || G == 4 || G == 8) && slots <= stream::kMaxSlots && U < stream::kMaxUnits &&
         c.max_tokens <= (1 << 25) && U * c.max_tokens < (int64_t)INT32_MAX && n_tokens >= 8;
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

// rows x D bf16 matrix, boxes of 64 columns x box_rows rows, 128-byte swizzle
static bool encode_rows(CUtensorMap* tm, const void* base, uint64_t rows, int D, int box_rows) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  cuuint64_t gdim[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Kp and Vp ([rows][D] bf16 each, Vp after Kp) as one map whose outermost
// dimension steps from Kp to Vp: an 8-row box (boxDim {64, 8, [2,] 2}) lands as
// [key/value][64-column half][8 rows][128 bytes], 128-byte swizzle.  The map
// covers exactly the two stores, so no box reads outside them.
static bool encode_store_boxes(CUtensorMap* tm, const void* Kp, const void* Vp, uint64_t rows, int D) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  const intptr_t kv = reinterpret_cast<const char*>(Vp) - reinterpret_cast<const char*>(Kp);
  if (kv < (intptr_t)(rows * D * 2) || (kv & 15) != 0 || kv >= ((intptr_t)1 << 40)) return false;
  cuuint32_t estr[4] = {1, 1, 1, 1};
  if (D == 128) {
    cuuint64_t gdim[4] = {64, rows, 2, 2};
    cuuint64_t gstride[3] = {256, 128, (cuuint64_t)kv};
    cuuint32_t box[4] = {64, 8, 2, 2};
    return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(Kp), gdim, gstride, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  }
  cuuint64_t gdim[3] = {64, rows, 2};
  cuuint64_t gstride[2] = {128, (cuuint64_t)kv};
  cuuint32_t box[3] = {64, 8, 2};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(Kp), gdim, gstride, box, estr,
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
  cfg.blockDim = dim3(stream::kCT + stream::kVP * kWarp);
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

// The flat bf16 decode step: two kernels.  The centroid tickets at the head of
// the scratch are zero on entry; the value pass zeroes them again (after the
// centroid pass has completed), the centroid pass zeroes the value tickets at
// its start and each unit's combining CTA its own after the combine, so a
// finished step leaves the whole ticket head zero.
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
  a.Kc = static_cast<const __nv_bfloat16*>(Kc);
  a.Vc = static_cast<const __nv_bfloat16*>(ws_ptr(idx, S_VC));
  a.Kp = static_cast<const __nv_bfloat16*>(ws_ptr(idx, S_KP));
  a.Vp = static_cast<const __nv_bfloat16*>(ws_ptr(idx, S_VP));
  if (!encode_rows(&a.tmKc, Kc, (uint64_t)U * idx->slots, D, stream::kRows) ||
      !encode_rows(&a.tmVc, a.Vc, (uint64_t)U * idx->slots, D, stream::kRows) ||
      !encode_store_boxes(&a.tmKV, a.Kp, a.Vp, (uint64_t)U * c.max_tokens, D))
    return MP_ECUDA;
  a.Q = static_cast<const __nv_bfloat16*>(Q);
  a.O = static_cast<__nv_bfloat16*>(O);
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
  a.shat = reinterpret_cast<float*>(base + L.o_shat);
  a.boxes = reinterpret_cast<int32_t*>(base + L.o_tok);
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
  cudaError_t e = D == 128 ? launch_stream_d<128>(G, a, grid, st) : launch_stream_d<64>(G, a, grid, st);
  phase(1);
  if (e != cudaSuccess) {
    // a launch that did not happen may leave the centroid tickets taken
    cudaGetLastError();
    cudaMemsetAsync(base + L.o_ctl, 0, L.ctl_bytes, st);
    return MP_ECUDA;
  }
  return MP_OK;
}

}  // namespace mp
