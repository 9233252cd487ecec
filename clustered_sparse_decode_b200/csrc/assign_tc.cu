// k-means assignment on the tensor cores (tcgen05, accumulators in TMEM).
//
// "Multipole Attention for Efficient Long Context Reasoning" (arXiv abstract;
// atlas.scime summary, "Approach"): the keys of each block are clustered with
// k-means; the assignment step compares every key with every centroid of its
// block, assign[t] = argmin_c (|c|^2 - 2 k_t . c), ties to the lower slot.
// The dot products k_t . c are a dense bf16 GEMM of the block's keys
// [L x d] with its centroids [C x d]^T, accumulated in fp32.
//
// A CTA owns one (unit, block) and every NX-th 128-key tile of it.  Warp 8
// loads the block's centroids once and the key tiles double-buffered with TMA
// (64-column boxes, 128-byte swizzle: the canonical K-major layout of the UMMA
// shared-memory descriptors); one of its threads issues tcgen05.mma (M = 128
// keys, N <= 256 centroids, K = 16) into TMEM.  The 128 x 512 fp32 tile of a
// block with 512 centroids fills all 512 TMEM columns, as two N-halves with
// their own completion and release barriers, so that the epilogue of one half
// overlaps the MMAs of the other.  Warps 0-7 are the epilogue: warp w reads
// TMEM lanes 32 (w % 4) .. + 31 (one key per thread) of N-half w / 4 (or of
// every other 32-column chunk when one half holds all centroids) and keeps
// four interleaved running argmins of |c|^2 - 2 k.c in fp32; the candidates
// are merged by (distance, slot), which equals one scan in slot order with a
// strict < (the first slot attaining the minimum).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "mp_internal.cuh"

namespace mp {
namespace atc {

constexpr int kM = 128;          // keys per tile (UMMA M)
constexpr int kNH = 256;         // centroids per N-half (UMMA N <= 256)
constexpr int kMaxC = 2 * kNH;   // centroids per block handled here
constexpr int kEpiWarps = 8;
constexpr int kProducer = kEpiWarps;          // warp index of the TMA / MMA warp
constexpr int kThreads = (kEpiWarps + 1) * kWarp;

struct Args {
  CUtensorMap tmK;               // keys: [rows][D] bf16, boxes of 64 columns x kM rows
  CUtensorMap tmC;               // centroids: [units * slots][D] bf16, boxes of 64 columns x kNH rows
  const __nv_bfloat16* Kc;       // the same centroids, for the norms
  int32_t* assign;               // [units][max_tokens]
  int64_t max_tokens;
  int64_t src_unit_rows, src_row0;   // key row of token t of unit u: u * src_unit_rows + src_row0 + (t - blk0 * L_blk)
  int blk0, L_blk, T, C_blk, slots;
  int64_t n_total;
  int NX;                        // CTAs per (unit, block)
  int32_t* err;
  long long timeout_ns;
};

template <int D>
struct Geo {
  static constexpr int KT = D / 64;                 // 64-column tiles per row
  static constexpr int ATILE = kM * 128;            // one 64-column tile of a key tile
  static constexpr int BTILE = kNH * 128;           // one 64-column tile of an N-half
  static constexpr int OFF_B = 0;                   // [2 halves][KT][kNH rows][128 B]
  static constexpr int OFF_A = 2 * KT * BTILE;      // [2 buffers][KT][kM rows][128 B]
  static constexpr int OFF_CN = OFF_A + 2 * KT * ATILE;   // centroid norms, kMaxC floats (+inf past C)
  static constexpr int OFF_XD = OFF_CN + kMaxC * 4;       // [2][kM] distances of group 1
  static constexpr int OFF_XI = OFF_XD + 2 * kM * 4;      // [2][kM] slots of group 1
  static constexpr int OFF_BAR = OFF_XI + 2 * kM * 4;     // barriers, TMEM address
  static constexpr int USED = OFF_BAR + 128 + 1024;       // + alignment slack
  // one CTA per SM: a second one would wait in tcgen05.alloc for the columns
  static constexpr int SMEM = USED > 120 * 1024 ? USED : 120 * 1024;
  static_assert(SMEM <= 232448, "shared memory per CTA");
  static_assert(OFF_A % 1024 == 0 && ATILE % 1024 == 0 && BTILE % 1024 == 0, "swizzle atoms on 1024 B");
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
      : "r"(bar), "r"(parity), "r"(1000000u)
      : "memory");
  return ok != 0;
}
// Wait for the phase of the given parity; gives up (error word set, false) once
// the CTA has run for the time limit, so that every later wait fails at once.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, long long t0, long long limit, int32_t* err) {
  while (!mbar_try(bar, parity)) {
    if (gtimer() - t0 > limit) { set_error(err, E_TIMEOUT); return false; }
  }
  return true;
}
__device__ __forceinline__ void tma_tile(uint32_t dst, const CUtensorMap* tm, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
// UMMA shared-memory descriptor of a K-major operand in the 128-byte swizzled
// layout: rows of 128 bytes, 8-row groups 1024 bytes apart (stride byte offset),
// descriptor version 1, layout type 2 (SWIZZLE_128B).  A step of 16 elements
// along K inside the 128-byte row adds 32 bytes to the start address.
__device__ __forceinline__ uint64_t sdesc_k_sw128(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);          // start address
  d |= (uint64_t)1 << 16;                          // leading byte offset (fixed for swizzled K-major)
  d |= (uint64_t)(1024 >> 4) << 32;                // stride byte offset
  d |= (uint64_t)1 << 46;                          // descriptor version
  d |= (uint64_t)2 << 61;                          // SWIZZLE_128B
  return d;
}
// instruction descriptor of kind::f16: bf16 x bf16 -> fp32, both K-major, M = 128, N = n
__device__ __forceinline__ uint32_t idesc_bf16(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kM >> 4) << 24);
}
__device__ __forceinline__ void umma(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
      "l"(da), "l"(db), "r"(idesc), "r"(acc)
      : "memory");
}
// arrive on an mbarrier once all earlier tcgen05.mma of this thread have completed
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
// 32 consecutive TMEM columns of this thread's lane
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
// (d, i) before (bd, bi) in the order (distance, slot)
__device__ __forceinline__ bool before(float d, int i, float bd, int bi) { return d < bd || (d == bd && i < bi); }

// ---------------------------------------------------------------------------
// The kernel: grid (NX, blocks, units)
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kThreads, 1) assign_tc_kernel(const __grid_constant__ Args a) {
  using Gm = Geo<D>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(smem);
  float* cn = reinterpret_cast<float*>(smem + Gm::OFF_CN);
  float* xd = reinterpret_cast<float*>(smem + Gm::OFF_XD);
  int* xi = reinterpret_cast<int*>(smem + Gm::OFF_XI);
  const uint32_t bar0 = sb + Gm::OFF_BAR;
  // barriers: bfull, afull[2], aempty[2], done[2], tfree[2]; then the TMEM address
  const uint32_t bfull = bar0, afull = bar0 + 8, aempty = bar0 + 24, done = bar0 + 40, tfree = bar0 + 56;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Gm::OFF_BAR + 80);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int j = a.blk0 + blockIdx.y, unit = blockIdx.z;
  const int64_t s = (int64_t)j * a.L_blk;
  const int64_t rem = a.n_total - s;
  const int L = rem <= 0 ? 0 : (int)(rem < (int64_t)a.L_blk ? rem : (int64_t)a.L_blk);
  const int C = (L + a.T - 1) / a.T;
  const int ntiles = (L + kM - 1) / kM;
  const int nmine = (int)blockIdx.x < ntiles ? (ntiles - 1 - (int)blockIdx.x) / a.NX + 1 : 0;
  if (nmine == 0 || C == 0) return;                 // uniform over the CTA, before any barrier or TMEM use
  const int nh = (C + kNH - 1) / kNH;               // N-halves in use
  const long long t0 = gtimer();

  if (threadIdx.x == 0) {
    mbar_init(bfull, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(afull + 8 * i, 1);
      mbar_init(aempty + 8 * i, 1);
      mbar_init(done + 8 * i, 1);
    }
    // the epilogue warps that read a half release it: 4 warps each, or all 8 when one half holds every centroid
    mbar_init(tfree, nh == 2 ? kEpiWarps / 2 : kEpiWarps);
    mbar_init(tfree + 8, kEpiWarps / 2);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(tmem_slot)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  // centroid norms |c|^2 in fp32 from the stored (rounded) centroids, in element
  // order; +inf past the block's C, so that no padding column can win
  const __nv_bfloat16* Kcb = a.Kc + ((size_t)unit * a.slots + (size_t)j * a.C_blk) * D;
  for (int c = threadIdx.x; c < kMaxC; c += kThreads) {
    float sn = INFINITY;
    if (c < C) {
      sn = 0.f;
      const uint4* row = reinterpret_cast<const uint4*>(Kcb + (size_t)c * D);
#pragma unroll 4
      for (int q = 0; q < D / 8; ++q) {
        const uint4 v = __ldg(row + q);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float lo = __uint_as_float(w[i] << 16), hi = __uint_as_float(w[i] & 0xffff0000u);
          sn = fmaf(lo, lo, sn);
          sn = fmaf(hi, hi, sn);
        }
      }
    }
    cn[c] = sn;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kProducer) {
    // ================= TMA + MMA (one thread) =================
    if (lane == 0) {
      const int crow = unit * a.slots + j * a.C_blk;
      mbar_arrive_tx(bfull, (uint32_t)(nh * Gm::KT * Gm::BTILE));
      for (int h = 0; h < nh; ++h)
        for (int kt = 0; kt < Gm::KT; ++kt)
          tma_tile(sb + Gm::OFF_B + (h * Gm::KT + kt) * Gm::BTILE, &a.tmC, 64 * kt, crow + h * kNH, bfull);
      const int64_t krow0 = (int64_t)unit * a.src_unit_rows + a.src_row0 + (s - (int64_t)a.blk0 * a.L_blk);
      auto load_a = [&](int i) {   // the i-th tile of this CTA into buffer i % 2
        const int buf = i & 1;
        const int tile = (int)blockIdx.x + i * a.NX;
        mbar_arrive_tx(afull + 8 * buf, (uint32_t)(Gm::KT * Gm::ATILE));
        for (int kt = 0; kt < Gm::KT; ++kt)
          tma_tile(sb + Gm::OFF_A + (buf * Gm::KT + kt) * Gm::ATILE, &a.tmK, 64 * kt, (int)(krow0 + (int64_t)tile * kM),
                   afull + 8 * buf);
      };
      load_a(0);
      if (nmine > 1) load_a(1);
      bool ok = mbar_wait(bfull, 0, t0, a.timeout_ns, a.err);
      for (int i = 0; i < nmine && ok; ++i) {
        const int buf = i & 1;
        if (!(ok = mbar_wait(afull + 8 * buf, (i >> 1) & 1, t0, a.timeout_ns, a.err))) break;
        for (int h = 0; h < nh && ok; ++h) {
          if (i > 0 && !(ok = mbar_wait(tfree + 8 * h, (i - 1) & 1, t0, a.timeout_ns, a.err))) break;
          tc_fence_after();
          const int n = min(kNH, ((C - h * kNH) + 15) / 16 * 16);
          const uint32_t idesc = idesc_bf16(n);
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const int kt = ks >> 2, sub = ks & 3;
            const uint64_t da = sdesc_k_sw128(sb + Gm::OFF_A + (buf * Gm::KT + kt) * Gm::ATILE + sub * 32);
            const uint64_t db = sdesc_k_sw128(sb + Gm::OFF_B + (h * Gm::KT + kt) * Gm::BTILE + sub * 32);
            umma(tmem + (uint32_t)(h * kNH), da, db, idesc, ks > 0 ? 1u : 0u);
          }
          umma_commit(done + 8 * h);
        }
        if (!ok) break;
        umma_commit(aempty + 8 * buf);
        // the buffer of the previous tile takes the next tile once the previous tile's MMAs have read it
        if (i >= 1 && i + 1 < nmine) {
          if (!(ok = mbar_wait(aempty + 8 * ((i - 1) & 1), ((i - 1) >> 1) & 1, t0, a.timeout_ns, a.err))) break;
          load_a(i + 1);
        }
      }
      // the last two tiles' buffer releases: their MMAs have finished before the CTA ends
      for (int k = max(0, nmine - 2); k < nmine && ok; ++k)
        ok = mbar_wait(aempty + 8 * (k & 1), (k >> 1) & 1, t0, a.timeout_ns, a.err);
    }
  } else {
    // ================= epilogue =================
    const int grp = warp >> 2, quarter = warp & 3;
    const int h = nh == 2 ? grp : 0;
    const int cstep = nh == 2 ? 32 : 64;
    const int cbeg = nh == 2 ? h * kNH : 32 * grp;
    const int cend = min(C, (h + 1) * kNH);
    const uint32_t lane_base = tmem + ((uint32_t)(32 * quarter) << 16);
    bool ok = true;
    for (int i = 0; i < nmine; ++i) {
      float bd[4] = {INFINITY, INFINITY, INFINITY, INFINITY};
      int bi[4] = {0, 0, 0, 0};
      if (ok) ok = mbar_wait(done + 8 * h, i & 1, t0, a.timeout_ns, a.err);
      ok = __all_sync(kFull, ok);                   // the TMEM loads below are warp-collective
      if (ok) {
        tc_fence_after();
        for (int c0 = cbeg; c0 < cend; c0 += cstep) {
          float v[32];
          tmem_ld32(lane_base + (uint32_t)c0, v);
          const float4* cn4 = reinterpret_cast<const float4*>(cn + c0);
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            const float4 n4 = cn4[q4];
            const float nn[4] = {n4.x, n4.y, n4.z, n4.w};
#pragma unroll
            for (int r = 0; r < 4; ++r) {
              const float dd = fmaf(-2.f, v[4 * q4 + r], nn[r]);
              if (dd < bd[r]) { bd[r] = dd; bi[r] = c0 + 4 * q4 + r; }
            }
          }
        }
        tc_fence_before();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(tfree + 8 * h);
      float d = bd[0];
      int ix = bi[0];
#pragma unroll
      for (int r = 1; r < 4; ++r)
        if (before(bd[r], bi[r], d, ix)) { d = bd[r]; ix = bi[r]; }
      const int key = 32 * quarter + lane, xb = (i & 1) * kM;
      if (grp == 1) { xd[xb + key] = d; xi[xb + key] = ix; }
      asm volatile("bar.sync 1, %0;\n" ::"n"(kEpiWarps * kWarp) : "memory");
      if (grp == 0) {
        if (before(xd[xb + key], xi[xb + key], d, ix)) ix = xi[xb + key];
        const int t = ((int)blockIdx.x + i * a.NX) * kM + key;
        if (ok && t < L) a.assign[(size_t)unit * a.max_tokens + s + t] = j * a.C_blk + ix;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(512) : "memory");
  }
}

}  // namespace atc

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 atc_encoder() {
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

// 2-D map of a [rows][D] bf16 matrix, boxes of 64 columns x box_rows rows, 128-byte swizzle
static bool atc_encode(CUtensorMap* tm, const void* base, uint64_t rows, int D, int box_rows) {
  auto fn = atc_encoder();
  if (!fn) return false;
  cuuint64_t gdim[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Whether the tensor-core assignment takes this job: bf16 keys, d in {64, 128},
// at most 512 centroids per block, 16-byte aligned key and centroid bases and
// row indices inside the int32 range of the tensor maps.
bool assign_tc_supported(int dtype, int D, int C_blk, const void* srcK, const void* Kc, int64_t src_rows_total,
                         int64_t centroid_rows) {
  return dtype == MP_BF16 && (D == 64 || D == 128) && C_blk <= atc::kMaxC && C_blk > 0 &&
         ((uintptr_t)srcK & 15u) == 0 && ((uintptr_t)Kc & 15u) == 0 && src_rows_total < (int64_t)INT32_MAX - atc::kM &&
         centroid_rows < (int64_t)INT32_MAX - atc::kNH;
}

// One assignment step over the blocks [blk0, blk0 + nbj) of every unit.
cudaError_t launch_assign_tc(int D, const void* srcK, int64_t src_rows_total, int64_t src_unit_rows, int64_t src_row0,
                             const void* Kc, int units, int slots, int blk0, int nbj, int L_blk, int T, int C_blk,
                             int64_t n_total, int32_t* assign, int64_t max_tokens, int32_t* err, cudaStream_t st) {
  atc::Args a{};
  if (!atc_encode(&a.tmK, srcK, (uint64_t)src_rows_total, D, atc::kM) ||
      !atc_encode(&a.tmC, Kc, (uint64_t)units * slots, D, atc::kNH))
    return cudaErrorInvalidValue;
  a.Kc = static_cast<const __nv_bfloat16*>(Kc);
  a.assign = assign;
  a.max_tokens = max_tokens;
  a.src_unit_rows = src_unit_rows;
  a.src_row0 = src_row0;
  a.blk0 = blk0;
  a.L_blk = L_blk;
  a.T = T;
  a.C_blk = C_blk;
  a.slots = slots;
  a.n_total = n_total;
  a.err = err;
  a.timeout_ns = 2000000000LL;
  // CTAs per (unit, block): about 16 key tiles each, more while the grid is below one wave
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int ntiles = (L_blk + atc::kM - 1) / atc::kM;
  int nx = std::max(1, ntiles / 16);
  while (nx < ntiles && (int64_t)nx * nbj * units < sms) ++nx;
  a.NX = nx;
  cudaError_t e;
  if (D == 128) {
    auto k = atc::assign_tc_kernel<128>;
    if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, atc::Geo<128>::SMEM)) != cudaSuccess)
      return e;
    k<<<dim3(nx, nbj, units), atc::kThreads, atc::Geo<128>::SMEM, st>>>(a);
  } else {
    auto k = atc::assign_tc_kernel<64>;
    if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, atc::Geo<64>::SMEM)) != cudaSuccess)
      return e;
    k<<<dim3(nx, nbj, units), atc::kThreads, atc::Geo<64>::SMEM, st>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace mp
