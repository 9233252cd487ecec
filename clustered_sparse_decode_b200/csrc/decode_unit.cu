// Decode step for bf16 caches: one kernel in which each (batch, KV head) unit
// is decoded by one CTA, or by a cluster of k CTAs when there are few units
// (k = 2, 4 or 8 keeps the grid near one CTA per SM).  The same engine runs
// the dense baseline (every key attended exactly).
//
// "Multipole Attention for Efficient Long Context Reasoning" (arXiv abstract;
// atlas.scime summary, "Approach"): the query scores every key centroid, the
// best clusters up to a token budget are attended exactly, and every other
// cluster enters the same softmax as one term with logit score + ln(size) and
// its value centroid.
//
// Per unit, in one CTA (or cluster):
//   1. key centroids    128-row TMA tiles of Kc: scores S[c][g] = scale q_g.Kc_c
//                       (to the scratch, each read back by the thread that
//                       wrote it or after a block barrier) and group scores
//                       max_g S[c][g] (shared memory).
//   2. selection        token-budgeted over the group scores max_g S[c][g]
//                       (a cluster first gathers its CTAs' scores over
//                       distributed shared memory): clusters in descending
//                       score, ties to the lower slot, the crossing cluster
//                       whole.  Meanwhile the loaders already stream 3.: its
//                       loads do not depend on the selection.
//   3. value centroids  128-row TMA tiles of Vc: the centroid terms of the
//                       UNSELECTED non-empty clusters (logit S + ln n_c, value
//                       Vc_c) enter the online softmax; selected clusters are
//                       masked, so no term is ever added and taken out again.
//   4. exact rows       the selected clusters' runs of the cluster-ordered
//                       store, then the un-clustered tail, packed 64 rows to a
//                       chunk: the planner warp lists the rows in order, the
//                       loader warps gather them (keys and values, 16-byte
//                       cp.async into the swizzled 8-row box layout), so every
//                       selected row is read once and no row is padding.
//   5. combine          the eight warps' softmax states (and, in a cluster,
//                       the CTAs' states over distributed shared memory)
//                       merge into O.
//
// Warps: 8 compute warps in two groups of 4; group w computes the chunks
// k = w (mod 2) of a ring of 32 KB chunks (d = 128), on mma.sync (bf16 in, fp32
// accumulate); loader warp w fills the ring slots of group w's chunks; one
// planner warp turns the selection into the row list.  Every wait on the
// device is bounded (then an error bit is set and the kernel winds down).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "stream_common.cuh"

namespace mp {
namespace unit {
using namespace sc;

constexpr int kCW = 8;                         // compute warps (two groups of 4)
constexpr int kCT = kCW * kWarp;               // compute threads
constexpr int kGW = 4;                         // warps per compute group
constexpr int kLoaders = 4;                    // loader warps
constexpr int kThreads = kCT + (kLoaders + 1) * kWarp;   // + the loaders and the planner
constexpr int kRowCap = 1024;                  // planner -> loaders: row queue entries
constexpr int kRows = 128;                     // centroid rows per chunk (keys or values only)
constexpr int kDRows = 64;                     // dense chunks: key and value rows
constexpr int kChunkRows = 64;                 // exact rows (keys and values) per chunk, as 8-row boxes
constexpr int kBoxes = kChunkRows / 8;
constexpr int kMaxNS = 12;                     // ring slots at most
constexpr int kMinNS = 4;
constexpr int kMaxSpt = 16;                    // selection: slots per compute thread
constexpr int kMaxSlots = kMaxSpt * kCT;       // 4096
constexpr int kMaxCluster = 8;
constexpr int kFullCount = kWarp;              // arrivals completing a full slot: one per lane of its loader
constexpr int kSmemLimit = 232448;             // dynamic shared memory of one CTA per SM
constexpr int kBarC = 2;                       // named barrier: compute threads

enum Mode : int { M_FLAT = 0, M_DENSE = 1 };
enum ChunkKind : int { K_KC = 0, K_VC = 1, K_DENSE = 2 };

struct Args {
  CUtensorMap tmA;             // M_FLAT: Kc, M_DENSE: K, as [units*rows][D] bf16, 64-column tiles (128-byte swizzle)
  CUtensorMap tmB;             // M_FLAT: Vc, M_DENSE: V
  const char* Kp;              // M_FLAT: cluster-ordered key store [units * max_tokens][D] bf16
  const char* Vp;              // M_FLAT: value store, same layout
  const __nv_bfloat16* Q;      // [units][G][D]
  __nv_bfloat16* O;            // [units][G][D]
  const int32_t* off;          // M_FLAT: [units][slots + 1]
  float* S;                    // M_FLAT: scratch [units][slots][SG] per-head scores (natural-log units)
  uint8_t* sel_mask_out;       // optional [units][slots]
  float* scores_out;           // optional [units][slots]
  int32_t* err;
  int units, k;                // k: CTAs per unit (cluster size)
  int rows, rows_active;       // per unit: rows of the tile maps (slots | max_tokens) and rows to stream
  int max_tokens, n_clustered, n_tail;
  float scale;                 // score scale, natural-log units
  int budget, approx;
  long long timeout_ns;
  // shared-memory plan (byte offsets from the 1024-aligned base)
  int ns, o_meta, o_shat, o_offs, o_selm, o_wpre, o_q, o_red, o_bar, smem_bytes;
};

// What the producer tells the compute warps about the chunk in a ring slot.
struct Meta {                  // (tile chunks only; exact chunks need none)
  int kind, cnt, p0, pad;      // cnt: valid rows; p0: first row
};
constexpr int kMetaBytes = 16;
static_assert(sizeof(Meta) <= kMetaBytes, "meta");

// A ring slot holds kRows centroid rows, kChunkRows exact rows (keys and
// values, as 8-row boxes: [box][key/value][64-column half][8 rows][128 B]) or
// kDRows dense rows (keys and values): 256 D bytes.
template <int D>
struct Geo {
  static constexpr int SLOT = kRows * D * 2;
  static constexpr int BOXB = 32 * D;              // one 8-row box: key rows, then value rows
  static constexpr int DAREA = kDRows * D * 2;     // dense chunk: key rows, then value rows
  static_assert(kBoxes * BOXB == SLOT && 2 * DAREA == SLOT, "chunk kinds share the slot size");
};

__host__ __device__ inline int r16(int x) { return (x + 15) & ~15; }
__host__ __device__ inline int sg_of(int G) { return (G + 3) / 4 * 4; }

// Shared-memory plan: the ring takes what the unit's tables leave (host and device).
template <int D>
__host__ __device__ inline void plan(Args& a, int mode, int slots, int G) {
  const int sc = mode == M_FLAT ? (slots + 31) & ~31 : 0;
  int o = 0;
  const int meta = r16(kMaxNS * kMetaBytes);
  const int shat = sc * 4;
  const int offs = mode == M_FLAT ? r16((sc + 1) * 4) : 0;
  const int selm = mode == M_FLAT ? r16(sc / 8) : 0;
  const int wpre = mode == M_FLAT ? r16((sc / 32 + 1) * 4) : 0;
  const int q = mode == M_FLAT ? kRowCap * 4 + 128 : 0;
  const int red = mode == M_FLAT ? 1024 * 4 : 0;
  const int bar = 2 * kMaxNS * 8 + 32;
  const int fixed = meta + shat + offs + selm + wpre + q + red + bar;
  // An even number of slots: chunk k goes to slot k % ns and to compute group
  // k % 2, so every slot always serves the same group, which waits for that
  // slot's phases one after the other (a wait never runs two phases ahead of
  // the slot, where a parity test could not tell the phases apart).
  int ns = (kSmemLimit - 1024 - fixed) / Geo<D>::SLOT;
  ns = ns > kMaxNS ? kMaxNS : ns;
  ns &= ~1;
  a.ns = ns;
  o = ns * Geo<D>::SLOT;
  a.o_meta = o; o += meta;
  a.o_shat = o; o += shat;
  a.o_offs = o; o += offs;
  a.o_selm = o; o += selm;
  a.o_wpre = o; o += wpre;
  a.o_q = o; o += q;
  a.o_red = o; o += red;
  a.o_bar = o; o += bar;
  a.smem_bytes = o + 1024;     // + alignment slack
}

// ---------------------------------------------------------------------------
// Cluster helpers (distributed shared memory)
// ---------------------------------------------------------------------------
__device__ __forceinline__ int cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return (int)r;
}
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_sync() { cluster_arrive(); cluster_wait(); }
__device__ __forceinline__ uint32_t peer_addr(uint32_t local, int cta) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(cta));
  return r;
}
__device__ __forceinline__ uint32_t ld_peer_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ float4 ld_peer_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ void cbar() { asm volatile("bar.sync %0, %1;\n" ::"n"(kBarC), "n"(kCT) : "memory"); }
// shared-memory acquire load / release store of a flag (CTA scope)
__device__ __forceinline__ int ld_acquire(volatile int* p) {
  int v;
  asm volatile("ld.acquire.cta.shared.b32 %0, [%1];\n" : "=r"(v) : "r"(smem_u32(const_cast<int*>(p))) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(volatile int* p, int v) {
  asm volatile("st.release.cta.shared.b32 [%0], %1;\n" ::"r"(smem_u32(const_cast<int*>(p))), "r"(v) : "memory");
}
// named barrier `id` of n threads
__device__ __forceinline__ void named_bar(int id, int n) { asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(n) : "memory"); }

// ---------------------------------------------------------------------------
// Selection over the group scores (compute threads).  Token-budgeted:
// clusters by group score descending, ties to the lower slot, the shortest
// prefix whose token count reaches the budget (the crossing cluster whole);
// budget <= 0 selects nothing, a budget at or above all clustered tokens
// selects every non-empty cluster.  The threshold tau (the largest key with
// W(key >= tau) >= budget, keys being the order-preserving uint32 images of
// the group scores) is found first through 256 equal-width score bins (when at
// most 32 clusters fall into the crossing bin one warp sorts them), else by a
// radix descent over 256-bin histograms of the keys.  Every pass reads the
// scores and counts from shared memory in rolled loops: the selection runs
// once per step, so its code is kept small.  shat: [slots] group scores;
// writes the bitmask selm (complete after the final barrier).
// ---------------------------------------------------------------------------
// warp 0: the first of 256 bins (8 per lane, bin 8 l + i) from the top whose
// running weight, counted from `base` above, reaches the budget; the weight
// strictly above that bin.  Results in red[0], red[1].
__device__ __forceinline__ void crossing_bin(const int* hist, int base, int budget, int lane, int* red) {
  int bl[8], ls = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) { bl[i] = hist[8 * lane + i]; ls += bl[i]; }
  int suf = ls;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_down_sync(kFull, suf, o);
    if (lane + o < 32) suf += y;
  }
  int run = base + suf - ls, found = -1, ab = 0;
#pragma unroll
  for (int i = 7; i >= 0; --i) {
    if (found < 0 && run + bl[i] >= budget) { found = 8 * lane + i; ab = run; }
    run += bl[i];
  }
  const unsigned m = __ballot_sync(kFull, found >= 0);
  const int src = 31 - __clz(m);
  const int fb = __shfl_sync(kFull, found, src), fa = __shfl_sync(kFull, ab, src);
  if (lane == 0) { red[0] = fb; red[1] = fa; }
}

template <int G>
__device__ void select_smem(const Args& a, const float* shat, const int32_t* offs, uint32_t* selm, int* red,
                            int* hist, int u, bool write_out) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int slots = a.rows_active;
  // 1. total weight, smallest and largest key of the non-empty clusters
  int wsum = 0;
  uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll 1
  for (int c = tid; c < slots; c += kCT) {
    const int w = offs[c + 1] - offs[c];
    if (w > 0) {
      const uint32_t kk = ordered_key(shat[c]);
      wsum += w;
      kmin = min(kmin, kk);
      kmax = max(kmax, kk);
    }
  }
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
  const int mode = (a.budget <= 0 || W == 0) ? 0 : (W <= a.budget ? 1 : 2);   // none | all | threshold
  uint32_t tau = 0u;
  int ntie = 0, above = 0;
  bool resolved = false;
  if (mode == 2) {
    // 2a. 256 equal-width score bins; the crossing bin's clusters, if at most 32, sorted by one warp
    const float smin = key_score(kmin), smax = key_score(kmax);
    const float span = smax - smin, inv = 256.f / span;
    if (isfinite(smin) && isfinite(smax) && span > 0.f && isfinite(span) && isfinite(inv)) {
      auto fbin = [&](uint32_t kk) { return min(255, (int)((key_score(kk) - smin) * inv)); };
      int* lst = hist + 256;                                // [32][3] candidates of the crossing bin
      for (int i = tid; i < 256; i += kCT) hist[i] = 0;
      if (tid == 0) red[3] = 0;
      cbar();
#pragma unroll 1
      for (int c = tid; c < slots; c += kCT) {
        const int w = offs[c + 1] - offs[c];
        if (w > 0) atomicAdd(hist + fbin(ordered_key(shat[c])), w);
      }
      cbar();
      if (warp == 0) crossing_bin(hist, 0, a.budget, lane, red);
      cbar();
      const int fb = red[0], ab = red[1];
#pragma unroll 1
      for (int c = tid; c < slots; c += kCT) {
        const int w = offs[c + 1] - offs[c];
        if (w > 0) {
          const uint32_t kk = ordered_key(shat[c]);
          if (fbin(kk) == fb) {
            const int pos = atomicAdd(red + 3, 1);
            if (pos < 32) { lst[3 * pos] = (int)kk; lst[3 * pos + 1] = c; lst[3 * pos + 2] = w; }
          }
        }
      }
      cbar();
      const int nc = red[3];
      if (nc <= 32) {
        if (warp == 0) {
          // lane l holds candidate l (key, weight); the crossing key t is the
          // largest key whose candidates at or above it bring the running
          // weight ab + W(key >= t) to the budget
          const uint32_t kl = lane < nc ? (uint32_t)lst[3 * lane] : 0u;
          const int wl = lane < nc ? lst[3 * lane + 2] : 0;
          int wgt = 0, weq = 0;
#pragma unroll 1
          for (int j = 0; j < nc; ++j) {
            const uint32_t kj = (uint32_t)__shfl_sync(kFull, (int)kl, j);
            const int wj = __shfl_sync(kFull, wl, j);
            wgt += kj > kl ? wj : 0;
            weq += kj == kl ? wj : 0;
          }
          const bool reach = lane < nc && ab + wgt + weq >= a.budget;
          const uint32_t t = __reduce_max_sync(kFull, reach ? kl : 0u);
          const int tl = __ffs(__ballot_sync(kFull, reach && kl == t)) - 1;
          const int gt = __shfl_sync(kFull, wgt, tl);
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
    // 2b. radix descent over the keys in [kmin, kmax], 8 bits at a time
    uint32_t lo = kmin;
    int nb = kmax == kmin ? 0 : 32 - __clz(kmax - kmin);
    above = 0;
    int* hcnt = hist + 256;
    ntie = -1;
#pragma unroll 1
    while (nb > 0) {
      const int sh = max(nb - 8, 0);
      for (int i = tid; i < 256; i += kCT) { hist[i] = 0; hcnt[i] = 0; }
      cbar();
      const unsigned long long hi_excl = (unsigned long long)lo + (1ull << nb);
#pragma unroll 1
      for (int c = tid; c < slots; c += kCT) {
        const int w = offs[c + 1] - offs[c];
        if (w > 0) {
          const uint32_t kk = ordered_key(shat[c]);
          if (kk >= lo && (unsigned long long)kk < hi_excl) {
            const int bin = (int)((kk - lo) >> sh);
            atomicAdd(hist + bin, w);
            if (sh == 0) atomicAdd(hcnt + bin, 1);
          }
        }
      }
      cbar();
      if (warp == 0) {
        crossing_bin(hist, above, a.budget, lane, red);
        __syncwarp();
        if (lane == 0) red[2] = hcnt[red[0]];
      }
      cbar();
      const int bsel = red[0];
      above = red[1];
      if (sh == 0) ntie = red[2];
      lo += (uint32_t)bsel << sh;
      nb = sh;
      cbar();
    }
    tau = lo;
  }
  // 3. the selection bits: every cluster above tau, and the one at tau when
  // no other cluster ties with it (it is the crossing cluster: always taken)
#pragma unroll 1
  for (int base = warp * 32; base < slots; base += kCT) {
    const int c = base + lane;
    bool sel = false;
    if (c < slots && offs[c + 1] > offs[c]) {
      if (mode == 1) {
        sel = true;
      } else if (mode == 2) {
        const uint32_t kk = ordered_key(shat[c]);
        sel = kk > tau || (ntie == 1 && kk == tau);
      }
    }
    const unsigned bits = __ballot_sync(kFull, sel);
    if (lane == 0) selm[base >> 5] = bits;
  }
  cbar();
  if (mode == 2 && ntie != 1) {
    // several clusters exactly at tau: taken in slot order while the tokens
    // taken among them stay below budget - above (one warp; ties are rare)
    if (warp == 0) {
      const int need = a.budget - above;
      int taken = 0;
#pragma unroll 1
      for (int base = 0; base < slots && taken < need; base += 32) {
        const int c = base + lane;
        int tw = 0;
        if (c < slots) {
          const int w = offs[c + 1] - offs[c];
          if (w > 0 && ordered_key(shat[c]) == tau) tw = w;
        }
        int inc = tw;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(kFull, inc, o);
          if (lane >= o) inc += y;
        }
        const unsigned bits = __ballot_sync(kFull, tw > 0 && taken + inc - tw < need);
        if (lane == 0 && bits) selm[base >> 5] |= bits;
        taken += __shfl_sync(kFull, inc, 31);
      }
    }
    cbar();
  }
  if (write_out) {
#pragma unroll 1
    for (int c = tid; c < a.rows; c += kCT) {
      const bool in = c < slots && offs[c + 1] > offs[c];
      const bool sel = c < slots && ((selm[c >> 5] >> (c & 31)) & 1u);
      if (a.sel_mask_out) a.sel_mask_out[(size_t)u * a.rows + c] = sel ? 1 : 0;
      if (a.scores_out) a.scores_out[(size_t)u * a.rows + c] = in ? shat[c] : -INFINITY;
    }
  }
}

// The same selection with the slots held in registers: thread t owns the SPT
// consecutive slots [SPT t, SPT t + SPT) (16-byte loads of the group scores
// and offsets, once), and every pass works on those registers, so a pass costs
// a few instructions per slot instead of dependent shared-memory loads.  The
// selection bits of 32 slots are assembled from the owning threads' bits with
// shuffles.  SPT = 8 covers 2048 slots, 16 covers 4096.
template <int SPT>
__device__ void select_vec(const Args& a, const float* shat, const int32_t* offs, uint32_t* selm, int* red,
                           int* hist, int u, bool write_out) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int slots = a.rows_active;
  const int c0 = tid * SPT;
  uint32_t key[SPT];
  int w[SPT];
  {
    float sc[SPT];
    int of[SPT + 1];
    if (c0 + SPT <= slots) {
#pragma unroll
      for (int i = 0; i < SPT / 4; ++i) {
        const float4 s4 = reinterpret_cast<const float4*>(shat + c0)[i];
        const int4 o4 = reinterpret_cast<const int4*>(offs + c0)[i];
        sc[4 * i] = s4.x; sc[4 * i + 1] = s4.y; sc[4 * i + 2] = s4.z; sc[4 * i + 3] = s4.w;
        of[4 * i] = o4.x; of[4 * i + 1] = o4.y; of[4 * i + 2] = o4.z; of[4 * i + 3] = o4.w;
      }
      of[SPT] = offs[c0 + SPT];
    } else {
#pragma unroll
      for (int i = 0; i < SPT; ++i) {
        sc[i] = c0 + i < slots ? shat[c0 + i] : 0.f;
        of[i] = c0 + i <= slots ? offs[c0 + i] : 0;
      }
      of[SPT] = c0 + SPT <= slots ? offs[c0 + SPT] : 0;
    }
#pragma unroll
    for (int i = 0; i < SPT; ++i) {
      const int cnt = c0 + i < slots ? of[i + 1] - of[i] : 0;
      w[i] = cnt > 0 ? cnt : 0;
      key[i] = cnt > 0 ? ordered_key(sc[i]) : 0u;
    }
  }
  // 1. total weight, smallest and largest key of the non-empty clusters
  int wsum = 0;
  uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
  for (int i = 0; i < SPT; ++i)
    if (w[i] > 0) {
      wsum += w[i];
      kmin = min(kmin, key[i]);
      kmax = max(kmax, key[i]);
    }
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
  const int mode = (a.budget <= 0 || W == 0) ? 0 : (W <= a.budget ? 1 : 2);   // none | all | threshold
  uint32_t tau = 0u;
  int ntie = 0, above = 0;
  bool resolved = false;
  if (mode == 2) {
    // 2a. 256 equal-width score bins; the crossing bin's clusters, if at most 32, ranked by one warp
    const float smin = key_score(kmin), smax = key_score(kmax);
    const float span = smax - smin, inv = 256.f / span;
    if (isfinite(smin) && isfinite(smax) && span > 0.f && isfinite(span) && isfinite(inv)) {
      auto fbin = [&](uint32_t kk) { return min(255, (int)((key_score(kk) - smin) * inv)); };
      int* lst = hist + 256;                                // [32][3] candidates of the crossing bin
      for (int i = tid; i < 256; i += kCT) hist[i] = 0;
      if (tid == 0) red[3] = 0;
      cbar();
#pragma unroll
      for (int i = 0; i < SPT; ++i)
        if (w[i] > 0) atomicAdd(hist + fbin(key[i]), w[i]);
      cbar();
      if (warp == 0) crossing_bin(hist, 0, a.budget, lane, red);
      cbar();
      const int fb = red[0], ab = red[1];
#pragma unroll
      for (int i = 0; i < SPT; ++i)
        if (w[i] > 0 && fbin(key[i]) == fb) {
          const int pos = atomicAdd(red + 3, 1);
          if (pos < 32) { lst[3 * pos] = (int)key[i]; lst[3 * pos + 1] = c0 + i; lst[3 * pos + 2] = w[i]; }
        }
      cbar();
      const int nc = red[3];
      if (nc <= 32) {
        if (warp == 0) {
          // lane l holds candidate l (key, weight); the crossing key t is the
          // largest key whose candidates at or above it bring the running
          // weight ab + W(key >= t) to the budget
          const uint32_t kl = lane < nc ? (uint32_t)lst[3 * lane] : 0u;
          const int wl = lane < nc ? lst[3 * lane + 2] : 0;
          int wgt = 0, weq = 0;
#pragma unroll 1
          for (int j = 0; j < nc; ++j) {
            const uint32_t kj = (uint32_t)__shfl_sync(kFull, (int)kl, j);
            const int wj = __shfl_sync(kFull, wl, j);
            wgt += kj > kl ? wj : 0;
            weq += kj == kl ? wj : 0;
          }
          const bool reach = lane < nc && ab + wgt + weq >= a.budget;
          const uint32_t t = __reduce_max_sync(kFull, reach ? kl : 0u);
          const int tl = __ffs(__ballot_sync(kFull, reach && kl == t)) - 1;
          const int gt = __shfl_sync(kFull, wgt, tl);
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
    // 2b. radix descent over the keys in [kmin, kmax], 8 bits at a time
    uint32_t lo = kmin;
    int nb = kmax == kmin ? 0 : 32 - __clz(kmax - kmin);
    above = 0;
    int* hcnt = hist + 256;
    ntie = -1;
#pragma unroll 1
    while (nb > 0) {
      const int sh = max(nb - 8, 0);
      for (int i = tid; i < 256; i += kCT) { hist[i] = 0; hcnt[i] = 0; }
      cbar();
      const unsigned long long hi_excl = (unsigned long long)lo + (1ull << nb);
#pragma unroll
      for (int i = 0; i < SPT; ++i)
        if (w[i] > 0 && key[i] >= lo && (unsigned long long)key[i] < hi_excl) {
          const int bin = (int)((key[i] - lo) >> sh);
          atomicAdd(hist + bin, w[i]);
          if (sh == 0) atomicAdd(hcnt + bin, 1);
        }
      cbar();
      if (warp == 0) {
        crossing_bin(hist, above, a.budget, lane, red);
        __syncwarp();
        if (lane == 0) red[2] = hcnt[red[0]];
      }
      cbar();
      const int bsel = red[0];
      above = red[1];
      if (sh == 0) ntie = red[2];
      lo += (uint32_t)bsel << sh;
      nb = sh;
      cbar();
    }
    tau = lo;
  }
  // 3. the selection bits: every cluster above tau, and the one at tau when
  // no other cluster ties with it (it is the crossing cluster: always taken)
  {
    uint32_t mine = 0u;
#pragma unroll
    for (int i = 0; i < SPT; ++i) {
      bool sel = false;
      if (w[i] > 0) sel = mode == 1 || (mode == 2 && (key[i] > tau || (ntie == 1 && key[i] == tau)));
      mine |= sel ? (1u << i) : 0u;
    }
    constexpr int TPW = 32 / SPT;                        // threads per 32-slot word
    uint32_t word = mine << (SPT * (tid % TPW));
#pragma unroll
    for (int o = 1; o < TPW; o <<= 1) word |= __shfl_xor_sync(kFull, word, o);
    if (tid % TPW == 0 && c0 < slots) selm[c0 >> 5] = word;
  }
  cbar();
  if (mode == 2 && ntie != 1) {
    // several clusters exactly at tau: taken in slot order while the tokens
    // taken among them stay below budget - above (one warp; ties are rare)
    if (warp == 0) {
      const int need = a.budget - above;
      int taken = 0;
#pragma unroll 1
      for (int base = 0; base < slots && taken < need; base += 32) {
        const int c = base + lane;
        int tw = 0;
        if (c < slots) {
          const int ww = offs[c + 1] - offs[c];
          if (ww > 0 && ordered_key(shat[c]) == tau) tw = ww;
        }
        int inc = tw;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(kFull, inc, o);
          if (lane >= o) inc += y;
        }
        const unsigned bits = __ballot_sync(kFull, tw > 0 && taken + inc - tw < need);
        if (lane == 0 && bits) selm[base >> 5] |= bits;
        taken += __shfl_sync(kFull, inc, 31);
      }
    }
    cbar();
  }
  if (write_out) {
#pragma unroll 1
    for (int c = tid; c < a.rows; c += kCT) {
      const bool in = c < slots && offs[c + 1] > offs[c];
      const bool sel = c < slots && ((selm[c >> 5] >> (c & 31)) & 1u);
      if (a.sel_mask_out) a.sel_mask_out[(size_t)u * a.rows + c] = sel ? 1 : 0;
      if (a.scores_out) a.scores_out[(size_t)u * a.rows + c] = in ? shat[c] : -INFINITY;
    }
  }
}

// ---------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------
template <int D, int G, int MODE>
__global__ void __launch_bounds__(kThreads, 1) unit_decode(const __grid_constant__ Args a) {
  using Gm = Geo<D>;
  constexpr int SG = (G + 3) / 4 * 4;      // floats per score row (16-byte multiple)
  constexpr int CR = MODE == M_FLAT ? kRows : kDRows;   // rows per chunk of the first stream
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(smem);
  float* shat = reinterpret_cast<float*>(smem + a.o_shat);            // [rows] group scores max_g S
  int32_t* offs = reinterpret_cast<int32_t*>(smem + a.o_offs);        // [rows + 1] run offsets
  uint32_t* selm = reinterpret_cast<uint32_t*>(smem + a.o_selm);      // selection bitmask
  int32_t* wpre = reinterpret_cast<int32_t*>(smem + a.o_wpre);        // selected clusters before each word
  int* red = reinterpret_cast<int*>(smem + a.o_red);
  const uint32_t full0 = sb + a.o_bar, empty0 = full0 + kMaxNS * 8, selready = empty0 + kMaxNS * 8;
  auto meta = [&](int slot) { return reinterpret_cast<Meta*>(smem + a.o_meta + slot * kMetaBytes); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = a.k;
  const int rank = K > 1 ? cluster_rank() : 0;
  const int u = blockIdx.x / K;
  const int NS = a.ns;
  const long long deadline = gtimer() + a.timeout_ns;
  // this CTA's chunks [c_lo, c_hi) of the unit's first stream
  const int nch = (a.rows_active + CR - 1) / CR;
  const int c_lo = (int)((long long)rank * nch / K), c_hi = (int)((long long)(rank + 1) * nch / K);
  const int n1 = c_hi - c_lo;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(full0 + 8 * i, kFullCount);  // the loader's arrivals (+ the TMA bytes it announces)
      mbar_init(empty0 + 8 * i, kGW);        // one arrival per warp of the chunk's compute group
    }
    mbar_init(selready, 1);                  // the selection is in shared memory
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    if (MODE == M_FLAT) {
      volatile int* ctl = reinterpret_cast<volatile int*>(smem + a.o_q + kRowCap * 4);
      ctl[0] = 0;
      ctl[1] = -1;
      for (int i = 0; i < kLoaders; ++i) ctl[2 + i] = 0x3fffffff;   // loaders that gather no exact chunk
      ctl[2] = ctl[3] = 0;
      if (NS % 3 == 0) ctl[4] = 0;   // a third loader gathers when the ring is a multiple of 3
      for (int i = 0; i < kMaxNS; ++i) ctl[8 + i] = -1;   // gen[]: no exact chunk's slot handed over yet
    }
  }
  __syncthreads();
  if (MODE == M_FLAT && warp < kCW) {
    // the unit's run offsets (counts of every slot), for the centroid terms and the
    // selection: complete for every compute thread after the selection's first barrier
    const int32_t* ou = a.off + (size_t)u * (a.rows + 1);
    for (int i = threadIdx.x; i <= a.rows_active; i += kCT) offs[i] = __ldg(ou + i);
  }

  if (warp >= kCW) {
    // ======================== loaders and planner ========================
    // Loader 0 issues every TMA tile chunk (key centroids, or dense keys and
    // values; then value centroids).  The planner warp walks the selection in
    // slot order and lists the rows of the selected clusters' runs, then this
    // CTA's share of the un-clustered tail, in the row queue; the four loaders
    // gather them, 64 to an exact chunk, loader i the 16 rows from 16 i, as
    // 16-byte cp.async (keys and values) into the swizzled 8-row box layout.
    // Every wait is taken by all 32 lanes of a warp: a warp whose lane 0 alone
    // waits on an mbarrier (the other lanes parked at a later convergence
    // point) runs its following code several times slower.
    const int li = warp - kCW;               // 0..3: loader, 4: planner
    const int kx0 = MODE == M_FLAT && a.approx ? 2 * n1 : n1;   // first exact chunk
    int32_t* rowq = reinterpret_cast<int32_t*>(smem + a.o_q);
    volatile int* ctl = reinterpret_cast<volatile int*>(smem + a.o_q + kRowCap * 4);
    // ctl[0]: rows published, ctl[1]: all rows (-1 until known), ctl[2 + i]: loader i has
    // read every queue entry below 64 ctl[2 + i]
    if (K > 1 && MODE == M_FLAT) cluster_arrive();   // (1): nothing of these warps' is read by the peers
    bool ok = true;
    auto acquire = [&](int kk) -> bool {   // wait until the slot of chunk kk is free
      const bool got = kk < NS || mbar_wait(empty0 + 8 * (kk % NS), ((kk / NS) - 1) & 1, deadline);
      if (!got && lane == 0) set_error(a.err, E_TIMEOUT);
      return __all_sync(kFull, got);
    };
    if (li == 0) {
#pragma unroll 1
      for (int k = 0; k < kx0 && ok; ++k) {
        if (!(ok = acquire(k))) break;
        if (lane == 0) {
          const int slot = k % NS;
          Meta* m = meta(slot);
          const bool vc = k >= n1;
          const int p0 = (c_lo + (vc ? k - n1 : k)) * CR;
          m->kind = MODE == M_FLAT ? (vc ? K_VC : K_KC) : K_DENSE;
          m->cnt = min(CR, a.rows_active - p0);
          m->p0 = p0;
          const uint32_t dst = sb + slot * Gm::SLOT, bar = full0 + 8 * slot;
          const int y = u * a.rows + p0;
          mbar_expect_tx(bar, (uint32_t)Gm::SLOT);
          const CUtensorMap* tm = vc ? &a.tmB : &a.tmA;
#pragma unroll
          for (int h = 0; h < D / 64; ++h) tma_2d(dst + h * (CR * 128), tm, 64 * h, y, bar);
          if (MODE == M_DENSE) {
#pragma unroll
            for (int h = 0; h < D / 64; ++h) tma_2d(dst + Gm::DAREA + h * (CR * 128), &a.tmB, 64 * h, y, bar);
          }
          mbar_arrive_cnt(bar, kFullCount);
        }
        __syncwarp();
      }
    }
    if constexpr (MODE == M_FLAT) {
      if (li < kLoaders) {
        // ---------------- exact chunks ----------------
        // Exact chunk k is gathered whole by loader (k mod NS) mod nl: each slot
        // always takes the same loader, which waits for the slot's releases one
        // phase after the other (an empty barrier's parity test cannot tell
        // phases two apart).  The first NS exact chunks' slots last held tile
        // chunks: loader 0 follows those releases in order and hands each slot
        // over (gen[slot] = the chunk it is free for).
        const int nl = NS % 3 == 0 ? 3 : 2;    // loaders of exact chunks
        volatile int* gen = ctl + 8;
        // rows of exact chunk j: its count (0: past the rows; -1: timed out)
        auto chunk_rows = [&](int j) -> int {
#pragma unroll 1
          for (int spins = 0;; ++spins) {
            // acquire loads: the queue entries below the published count are visible after them
            const int total = __shfl_sync(kFull, ld_acquire(&ctl[1]), 0);
            const int avail = __shfl_sync(kFull, ld_acquire(&ctl[0]), 0);
            if (total >= 0) return max(0, min(kChunkRows, total - kChunkRows * j));
            if (avail >= kChunkRows * (j + 1)) return kChunkRows;
            if ((spins & 63) == 63 && __any_sync(kFull, gtimer() > deadline)) return -1;
            __nanosleep(64);
          }
        };
        auto gather = [&](int k, int j, int cnt) {
          const int r0 = lane < cnt ? rowq[(kChunkRows * j + lane) % kRowCap] : -1;
          const int r1 = lane + 32 < cnt ? rowq[(kChunkRows * j + 32 + lane) % kRowCap] : -1;
          const uint32_t dst = sb + (k % NS) * Gm::SLOT;
          if constexpr (D == 128) {
            // one row (keys and values, 2 x 256 B) per instruction: lane = kv:1 half:1 c16:3
            const int kv = lane >> 4, half = (lane >> 3) & 1, c16 = lane & 7;
            const char* g = (kv ? a.Vp : a.Kp) + half * 128 + c16 * 16;
            const uint32_t d0 = dst + kv * (Gm::BOXB / 2) + half * (Gm::BOXB / 4);
#pragma unroll 8
            for (int i = 0; i < kChunkRows; ++i) {
              const int rw = __shfl_sync(kFull, i < 32 ? r0 : r1, i & 31), rr = i & 7;
              cp16(d0 + (i >> 3) * Gm::BOXB + rr * 128 + ((c16 ^ rr) << 4), g + (size_t)max(rw, 0) * 256, rw >= 0);
            }
          } else {
            // two rows (keys and values, 2 x 128 B each) per instruction: lane = row:1 kv:1 c16:3
            const int sub = lane >> 4, kv = (lane >> 3) & 1, c16 = lane & 7;
            const char* g = (kv ? a.Vp : a.Kp) + c16 * 16;
            const uint32_t d0 = dst + kv * (Gm::BOXB / 2);
#pragma unroll 8
            for (int i2 = 0; i2 < kChunkRows; i2 += 2) {
              const int i = i2 + sub;
              const int rw = __shfl_sync(kFull, i2 < 32 ? r0 : r1, i & 31), rr = i & 7;
              cp16(d0 + (i >> 3) * Gm::BOXB + rr * 128 + ((c16 ^ rr) << 4), g + (size_t)max(rw, 0) * 128, rw >= 0);
            }
          }
          cp_arrive_noinc(full0 + 8 * (k % NS));   // one of the slot's 32 arrivals, once this lane's copies land
          // every copy above consumed its entry: the planner may reuse the chunk's entries
          __syncwarp();
          if (lane == 0) ctl[2 + li] = j + 1;
        };
        if (li < nl) {
          // loader 0: hand over the first NS exact slots, gathering its own among them
          if (li == 0) {
#pragma unroll 1
            for (int k = kx0; k < kx0 + NS && ok; ++k) {
              ok = acquire(k);
              __syncwarp();
              if (lane == 0) gen[k % NS] = ok ? k : -2;
              if (!ok || (k % NS) % nl != 0) continue;
              const int cnt = chunk_rows(k - kx0);
              if (cnt < 0) { ok = false; if (lane == 0) set_error(a.err, E_TIMEOUT); break; }
              if (cnt == 0) break;
              gather(k, k - kx0, cnt);
            }
          }
          // then every chunk of this loader's slots, in order
          const int k_first = li == 0 ? kx0 + NS : kx0;
#pragma unroll 1
          for (int k = k_first; ok; ++k) {
            if ((k % NS) % nl != li) continue;
            const int j = k - kx0;
            const int cnt = chunk_rows(j);
            if (cnt < 0) { ok = false; if (lane == 0) set_error(a.err, E_TIMEOUT); break; }
            if (cnt == 0) break;
            if (k >= kx0 + NS) {
              ok = acquire(k);
            } else {
#pragma unroll 1
              for (int spins = 0;; ++spins) {
                const int g = __shfl_sync(kFull, gen[k % NS], 0);
                if (g == k) break;
                if (g == -2 || ((spins & 63) == 63 && __any_sync(kFull, gtimer() > deadline))) { ok = false; break; }
                __nanosleep(32);
              }
              if (!ok && lane == 0) set_error(a.err, E_TIMEOUT);
            }
            if (!ok) break;
            gather(k, j, cnt);
          }
        }
        cp_wait_all();                         // this warp's copies have landed (also on an error path)
      } else {
        // ---------------- planner ----------------
        if (!__all_sync(kFull, mbar_wait(selready, 0, deadline))) {
          if (lane == 0) set_error(a.err, E_TIMEOUT);
          ok = false;
        }
        const int nw = (a.rows_active + 31) >> 5;
        int tot = 0;
#pragma unroll 1
        for (int w0 = 0; w0 < nw; w0 += 32) {   // per-word prefix of selected-cluster counts
          const int wi = w0 + lane;
          const int c = wi < nw ? __popc(selm[wi]) : 0;
          int inc = c;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(kFull, inc, o);
            if (lane >= o) inc += y;
          }
          if (wi < nw) wpre[wi] = tot + inc - c;
          tot += __shfl_sync(kFull, inc, 31);
        }
        __syncwarp();
        // this CTA's share: selected clusters of rank [r_lo, r_hi), tail rows [t_lo, t_hi)
        const int r_lo = (int)((long long)rank * tot / K), r_hi = (int)((long long)(rank + 1) * tot / K);
        const int t_lo = a.n_clustered + (int)((long long)rank * a.n_tail / K);
        const int t_hi = a.n_clustered + (int)((long long)(rank + 1) * a.n_tail / K);
        const int unit_row = u * a.max_tokens;
        int written = 0;
        bool tail_run = t_lo < t_hi;
#pragma unroll 1
        for (int rk = r_lo; ok && (rk < r_hi || tail_run);) {
          // up to 32 runs, one per lane: selected clusters located by rank, or the tail
          int st = 0, cnt = 0;
          if (rk < r_hi) {
            const int n = min(32, r_hi - rk);
            if (lane < n) {
              const int r = rk + lane;
              int lo = 0, hi = nw - 1;             // the word holding rank r: the last w with wpre[w] <= r
#pragma unroll 1
              while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (wpre[mid] <= r) lo = mid; else hi = mid - 1;
              }
              uint32_t word = selm[lo];
#pragma unroll 1
              for (int i = wpre[lo]; i < r && word; ++i) word &= word - 1;
              if (word == 0u) {
                set_error(a.err, E_BAD_LIST);
              } else {
                const int sl = (lo << 5) + __ffs(word) - 1;
                st = offs[sl];
                cnt = offs[sl + 1] - st;
                if (st < 0 || cnt < 1 || st + cnt > a.max_tokens) {
                  set_error(a.err, E_BAD_OFFSET);
                  cnt = 0;
                }
              }
            }
            rk += n;
          } else {
            if (lane == 0) { st = t_lo; cnt = t_hi - t_lo; }
            tail_run = false;
          }
          int incl = cnt;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl += y;
          }
          const int nrows = __shfl_sync(kFull, incl, 31);
#pragma unroll 1
          for (int b0 = 0; b0 < nrows; b0 += 32) {
            // room for 32 more entries: every loader has read the entries below 64 min(ctl[2 + i])
#pragma unroll 1
            for (int spins = 0;; ++spins) {
              int lo_j = ctl[2 + (lane & 3)];
              lo_j = min(lo_j, __shfl_xor_sync(kFull, lo_j, 1));
              lo_j = min(lo_j, __shfl_xor_sync(kFull, lo_j, 2));
              lo_j = __shfl_sync(kFull, lo_j, 0);
              if (written + b0 + 32 - kChunkRows * lo_j <= kRowCap) break;
              if ((spins & 63) == 63 && __any_sync(kFull, gtimer() > deadline)) { ok = false; break; }
              __nanosleep(64);
            }
            if (!ok) {
              if (lane == 0) set_error(a.err, E_TIMEOUT);
              break;
            }
            // entry b0 + lane lies in the run of the first lane whose inclusive count exceeds it
            const int q = b0 + lane;
            int lo = 0, hi = 31;
#pragma unroll
            for (int step = 0; step < 5; ++step) {
              const int mid = (lo + hi) >> 1;
              if (__shfl_sync(kFull, incl, mid) > q) hi = mid; else lo = mid + 1;
            }
            const int before = __shfl_sync(kFull, incl - cnt, lo);
            const int rs = __shfl_sync(kFull, st, lo);
            if (q < nrows) rowq[(written + q) % kRowCap] = unit_row + rs + (q - before);
            __syncwarp();
            if (lane == 0) st_release(&ctl[0], written + min(b0 + 32, nrows));
          }
          written += nrows;
        }
        __syncwarp();
        if (lane == 0) st_release(&ctl[1], ok ? written : 0);
      }
    }
    if (K > 1) {
      if (MODE == M_FLAT) cluster_wait();  // (1)
      cluster_sync();                      // (2) the CTA partials are complete
      cluster_sync();                      // (3) every CTA has read its peers' partials
    }
    return;
  }

  // ============================ compute warps ============================
  const int grp = warp / kGW, wg = warp % kGW;
  const float qk2 = a.scale * kLog2e;
  WarpSoftmax<D, G> ws;
  ws.reset();
  ws.load_q(a.Q + (size_t)u * G * D, lane);
  bool alive = true;
  auto wait_full = [&](int k) -> bool {
    if (mbar_wait(full0 + 8 * (k % NS), (k / NS) & 1, deadline)) return true;
    if (lane == 0) set_error(a.err, E_TIMEOUT);
    alive = false;
    return false;
  };
  // ---- first stream (this group's chunks k = grp, grp + 2, ...) ----
  for (int k = grp; k < n1 && alive; k += 2) {
    if (!wait_full(k)) break;
    const int slot = k % NS;
    const Meta* m = meta(slot);
    const int cnt = m->cnt, p0 = m->p0;
    const uint32_t dst = sb + slot * Gm::SLOT;
    if constexpr (MODE == M_FLAT) {
      // key centroids: 32 rows per warp, scores into shared memory
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int r16 = wg * 32 + t * 16;
        if (r16 < cnt) {
          float z[2][2];
          ws.template qk<false, kRows>(dst, r16, lane, z);
          const bool wr = !WarpSoftmax<D, G>::lo_cols(lane);
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int r = r16 + WarpSoftmax<D, G>::zrow(lane, i);
            float gmax = -INFINITY;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const int h = WarpSoftmax<D, G>::col_head(lane, j);
              const float sc = z[i][j] * a.scale;
              if (wr && h >= 0) {
                gmax = fmaxf(gmax, sc);
                if (r < cnt) a.S[((size_t)u * a.rows + p0 + r) * SG + h] = sc;
              }
            }
            // the group score of the row: max over the four lanes holding its columns
            gmax = fmaxf(gmax, __shfl_xor_sync(kFull, gmax, 1));
            gmax = fmaxf(gmax, __shfl_xor_sync(kFull, gmax, 2));
            if ((lane & 3) == 0 && r < cnt) shat[p0 + r] = gmax;
          }
        }
      }
    } else {
      // dense: 16 key and value rows per warp, every key exact
      const int r16 = wg * 16;
      if (r16 < cnt) {
        float z[2][2];
        ws.template qk<false, kDRows>(dst, r16, lane, z);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int r = r16 + WarpSoftmax<D, G>::zrow(lane, i);
#pragma unroll
          for (int j = 0; j < 2; ++j)
            z[i][j] = (WarpSoftmax<D, G>::col_head(lane, j) >= 0 && r < cnt) ? z[i][j] * qk2 : -INFINITY;
        }
        ws.template update<false, kDRows>(dst + Gm::DAREA, r16, lane, z, 1.f);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty0 + 8 * slot);
  }
  if constexpr (MODE == M_FLAT) {
    // ---- selection ----
    cbar();                                // this CTA's scores are in shared memory
    if (K > 1) {
      cluster_arrive();                    // (1) ... and every peer's
      cluster_wait();
      // the peers' group scores: slots [c_lo', c_hi') * kRows of CTA r'
      for (int r = 0; r < K; ++r) {
        if (r == rank) continue;
        const int lo = (int)((long long)r * nch / K) * kRows;
        const int hi = min(a.rows_active, (int)((long long)(r + 1) * nch / K) * kRows);
        const uint32_t base = peer_addr(smem_u32(shat), r);
        for (int i = lo + (int)threadIdx.x; i < hi; i += kCT) shat[i] = __uint_as_float(ld_peer_u32(base + 4u * i));
      }
      cbar();
    }
    if (a.rows_active <= 8 * kCT) select_vec<8>(a, shat, offs, selm, red, red + 256, u, rank == 0);
    else select_smem<G>(a, shat, offs, selm, red, red + 256, u, rank == 0);
    cbar();                                // every read of the group scores is done
    if (threadIdx.x == 0) mbar_arrive(selready);   // the loaders may pack the selected rows (over the group scores)
  }
  // ---- value centroids and exact rows ----
  // A value-centroid chunk's scores come from the scratch (written by the key
  // stream before the selection's barriers): each group loads them one of its
  // chunks ahead, so that the loads overlap the previous chunk.
  auto load_sv = [&](int kk, float (&sv)[2][2][2]) {
    if (!(MODE == M_FLAT && a.approx && kk < 2 * n1)) return;
    const int p0 = (c_lo + kk - n1) * kRows;
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int r = p0 + wg * 32 + t * 16 + WarpSoftmax<D, G>::zrow(lane, i);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int h = WarpSoftmax<D, G>::col_head(lane, j);
          sv[t][i][j] = (h >= 0 && r < a.rows_active) ? __ldcg(a.S + ((size_t)u * a.rows + r) * SG + h) : 0.f;
        }
      }
  };
  if constexpr (MODE == M_FLAT) {
    const int kx0 = a.approx ? 2 * n1 : n1;         // first exact chunk
    volatile int* ctl = reinterpret_cast<volatile int*>(smem + a.o_q + kRowCap * 4);
    float sv[2][2][2], svn[2][2][2];
    const int k2 = n1 + ((grp - n1) % 2 + 2) % 2;   // this group's first chunk of the second stream
    load_sv(k2, sv);
    for (int k = k2; alive; k += 2) {
      if (k >= kx0) {
        // exact chunk j exists once the planner has published a row of it; none is
        // left once all rows are known and they end before it
        const int j = k - kx0;
        int total = -1;
#pragma unroll 1
        for (int spins = 0;; ++spins) {
          total = ctl[1];
          if (total >= 0 || ctl[0] > kChunkRows * j) break;
          if ((spins & 63) == 63 && __any_sync(kFull, gtimer() > deadline)) {
            if (lane == 0) set_error(a.err, E_TIMEOUT);
            alive = false;
            break;
          }
          __nanosleep(64);
        }
        if (!alive || (total >= 0 && kChunkRows * j >= total)) break;
      }
      load_sv(k + 2, svn);
      if (!wait_full(k)) break;
      const int slot = k % NS;
      const uint32_t base = sb + slot * Gm::SLOT;
      if (k < kx0) {
        // value centroids of the unselected non-empty clusters: logit S + ln n
        const Meta* m = meta(slot);
        const int cnt = m->cnt, p0 = m->p0;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const int r16 = wg * 32 + t * 16;
          if (r16 < cnt) {
            float z[2][2];
            bool any = false;
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const int r = r16 + WarpSoftmax<D, G>::zrow(lane, i);
              const int s = p0 + r;
              const int n = r < cnt ? offs[s + 1] - offs[s] : 0;
              const bool take = n > 0 && !((selm[s >> 5] >> (s & 31)) & 1u);
              const float lg = log2f((float)n);
#pragma unroll
              for (int j = 0; j < 2; ++j) {
                const int h = WarpSoftmax<D, G>::col_head(lane, j);
                z[i][j] = (take && h >= 0) ? sv[t][i][j] * kLog2e + lg : -INFINITY;
                any |= take && h >= 0;
              }
            }
            if (__any_sync(kFull, any)) ws.template update<false, kRows>(base, r16, lane, z, 1.f);
          }
        }
      } else {
        // exact rows: 64 (the last chunk fewer, known from the row count by then)
        const int total = ctl[1];
        const int cnt = total >= 0 ? min(kChunkRows, total - kChunkRows * (k - kx0)) : kChunkRows;
        const int r16 = wg * 16;
        if (r16 < cnt) {
          float z[2][2];
          ws.template qk<true, kRows>(base, r16, lane, z);
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int r = r16 + 8 * i + (lane >> 2);   // rows 8 i .. 8 i + 7 of this warp's tile are box 2 wg + i
#pragma unroll
            for (int jj = 0; jj < 2; ++jj)
              z[i][jj] = (WarpSoftmax<D, G>::col_head(lane, jj) >= 0 && r < cnt) ? z[i][jj] * qk2 : -INFINITY;
          }
          ws.template update<true, kRows>(base + Gm::BOXB / 2, r16, lane, z, 1.f);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8 * slot);   // the loaders may refill the slot
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
          for (int jj = 0; jj < 2; ++jj) sv[t][i][jj] = svn[t][i][jj];
    }
  }
  // ---- combine ----
  cbar();                                  // every chunk is consumed: the ring is free
  float* pm = reinterpret_cast<float*>(smem);                 // [kCW][G]
  float* pl = pm + kCW * G;                                   // [kCW][G]
  float* pacc = pl + kCW * G;                                 // [kCW][G][D]
  float* cpart = pacc + kCW * G * D;                          // CTA partial: m[SG], l[SG], acc[G][D]
  ws.store(pm + warp * G, pl + warp * G, pacc + (size_t)warp * G * D, lane);
  cbar();
  constexpr int NE = G * D / 4;            // float4 groups of the output rows
  for (int e = threadIdx.x; e < NE; e += kCT) {
    const int g = (e * 4) / D, d = (e * 4) % D;
    float M = -INFINITY;
#pragma unroll
    for (int p = 0; p < kCW; ++p) M = fmaxf(M, pm[p * G + g]);
    float L = 0.f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    if (M != -INFINITY) {
#pragma unroll
      for (int p = 0; p < kCW; ++p) {
        const float mp_ = pm[p * G + g];
        const float f = mp_ == -INFINITY ? 0.f : ex2(mp_ - M);
        const float4 x = *reinterpret_cast<const float4*>(pacc + ((size_t)p * G + g) * D + d);
        o.x += f * x.x; o.y += f * x.y; o.z += f * x.z; o.w += f * x.w;
        L += f * pl[p * G + g];
      }
    }
    if (K == 1) {
      const float inv = L > 0.f ? 1.f / L : 0.f;
      __nv_bfloat16* out = a.O + ((size_t)u * G + g) * D + d;
      *reinterpret_cast<uint2*>(out) = make_uint2(pack_bf16(o.x * inv, o.y * inv), pack_bf16(o.z * inv, o.w * inv));
    } else {
      if (d == 0) { cpart[g] = M; cpart[SG + g] = L; }
      *reinterpret_cast<float4*>(cpart + 2 * SG + g * D + d) = o;
    }
  }
  if (K > 1) {
    cbar();
    cluster_sync();                        // (2) every CTA's partial is complete
    // this CTA writes the float4 groups [e_lo, e_hi) of the unit's output
    const int e_lo = rank * NE / K, e_hi = (rank + 1) * NE / K;
    const uint32_t cp_local = smem_u32(cpart);
    for (int e = e_lo + (int)threadIdx.x; e < e_hi; e += kCT) {
      const int g = (e * 4) / D, d = (e * 4) % D;
      float M = -INFINITY;
      for (int r = 0; r < K; ++r) M = fmaxf(M, __uint_as_float(ld_peer_u32(peer_addr(cp_local, r) + 4u * g)));
      float L = 0.f;
      float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
      if (M != -INFINITY) {
        for (int r = 0; r < K; ++r) {
          const uint32_t pb = peer_addr(cp_local, r);
          const float mr = __uint_as_float(ld_peer_u32(pb + 4u * g));
          if (mr == -INFINITY) continue;
          const float f = ex2(mr - M);
          const float lr = __uint_as_float(ld_peer_u32(pb + 4u * (SG + g)));
          const float4 x = ld_peer_f4(pb + 4u * (2 * SG + g * D + d));
          o.x += f * x.x; o.y += f * x.y; o.z += f * x.z; o.w += f * x.w;
          L += f * lr;
        }
      }
      const float inv = L > 0.f ? 1.f / L : 0.f;
      __nv_bfloat16* out = a.O + ((size_t)u * G + g) * D + d;
      *reinterpret_cast<uint2*>(out) = make_uint2(pack_bf16(o.x * inv, o.y * inv), pack_bf16(o.z * inv, o.w * inv));
    }
    cluster_sync();                        // (3) peers are done reading this CTA's partial
  }
}

}  // namespace unit

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
// Scratch of the unit kernel: the per-head scores [units][slots][SG] fp32
// (group scores, selection and partial states stay in shared memory).
size_t unit_scratch_bytes(const mp_config& c, int slots) {
  const size_t U = (size_t)c.batch * c.kv_heads;
  const int G = c.q_heads / c.kv_heads;
  return (U * slots * unit::sg_of(G) * 4 + 255) & ~(size_t)255;
}

static int unit_ring_slots(int D, int G, int mode, int slots) {
  unit::Args a{};
  if (D == 128) unit::plan<128>(a, mode, slots, G);
  else unit::plan<64>(a, mode, slots, G);
  return a.ns;
}

// The index shapes the unit kernel takes: flat bf16, d 64 or 128, G in {1, 2,
// 4, 8}, at most 4096 slots whose scores leave room for a ring of at least 4
// chunks in shared memory, store rows addressable by the tensor maps.
bool unit_supported(const mp_config& c, int slots) {
  const int G = c.q_heads / c.kv_heads;
  const int64_t U = (int64_t)c.batch * c.kv_heads;
  return c.levels == 1 && c.dtype == MP_BF16 && (c.head_dim == 64 || c.head_dim == 128) &&
         (G == 1 || G == 2 || G == 4 || G == 8) && slots <= unit::kMaxSlots &&
         U * c.max_tokens + 8 < (int64_t)INT32_MAX && U * slots < (int64_t)INT32_MAX &&
         U * unit::kMaxCluster < (int64_t)INT32_MAX &&
         unit_ring_slots(c.head_dim, G, unit::M_FLAT, slots) >= unit::kMinNS;
}

static PFN_cuTensorMapEncodeTiled_v12000 unit_encoder() {
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

// rows x D bf16 matrix, tiles of 64 columns x box_rows rows, 128-byte swizzle
static bool encode_tiles(CUtensorMap* tm, const void* base, uint64_t rows, int D, int box_rows) {
  auto fn = unit_encoder();
  if (!fn) return false;
  cuuint64_t gdim[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int G, int MODE>
static cudaError_t launch_unit_t(unit::Args& a, cudaStream_t st) {
  auto kern = unit::unit_decode<D, G, MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, a.smem_bytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)(a.units * a.k));
  cfg.blockDim = dim3(unit::kThreads);
  cfg.dynamicSmemBytes = a.smem_bytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = a.k;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.k > 1 ? 1 : 0;
  if (a.k > 1) {
    // the cluster must fit on the device with this kernel's shared memory
    int nclusters = 0;
    if (cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg) != cudaSuccess || nclusters < 1) {
      cudaGetLastError();
      a.k = 1;
      cfg.gridDim = dim3((unsigned)a.units);
      cfg.numAttrs = 0;
    }
  }
  return cudaLaunchKernelEx(&cfg, kern, (const unit::Args)a);
}

template <int D, int MODE>
static cudaError_t launch_unit_d(int G, unit::Args& a, cudaStream_t st) {
  switch (G) {
    case 1: return launch_unit_t<D, 1, MODE>(a, st);
    case 2: return launch_unit_t<D, 2, MODE>(a, st);
    case 4: return launch_unit_t<D, 4, MODE>(a, st);
    case 8: return launch_unit_t<D, 8, MODE>(a, st);
  }
  return cudaErrorInvalidValue;
}

template <int MODE>
static cudaError_t launch_unit(int D, int G, unit::Args& a, cudaStream_t st) {
  if (D == 128) {
    unit::plan<128>(a, MODE, a.rows, G);
    return launch_unit_d<128, MODE>(G, a, st);
  }
  unit::plan<64>(a, MODE, a.rows, G);
  return launch_unit_d<64, MODE>(G, a, st);
}

// CTAs per unit: clusters of k CTAs cover the SMs, each CTA with at least two
// chunks of the first stream; the caller's split count (n_split > 0) overrides it
static int cluster_size(int64_t units, int chunks, int n_split) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int k = 1;
  if (n_split > 0) {
    while (k * 2 <= std::min(n_split, unit::kMaxCluster)) k *= 2;
  } else {
    while (k * 2 <= unit::kMaxCluster && units * k * 2 <= sms && k * 2 * 2 <= chunks) k *= 2;
  }
  return k;
}

// One flat bf16 decode step with the unit kernel (one launch).
mp_status unit_decode(const mp_index* idx, const void* Q, void* O, const mp_decode_params* prm, void* scratch,
                      size_t scratch_bytes, float scale, cudaStream_t st) {
  const mp_config& c = idx->cfg;
  if (scratch_bytes < unit_scratch_bytes(c, idx->slots)) return MP_ENOSPC;
  const int U = c.batch * c.kv_heads, G = c.q_heads / c.kv_heads, D = c.head_dim;
  unit::Args a{};
  if (!encode_tiles(&a.tmA, ws_ptr(idx, S_KC), (uint64_t)U * idx->slots, D, unit::kRows) ||
      !encode_tiles(&a.tmB, ws_ptr(idx, S_VC), (uint64_t)U * idx->slots, D, unit::kRows))
    return MP_ECUDA;
  a.Kp = static_cast<const char*>(ws_ptr(idx, S_KP));
  a.Vp = static_cast<const char*>(ws_ptr(idx, S_VP));
  a.Q = static_cast<const __nv_bfloat16*>(Q);
  a.O = static_cast<__nv_bfloat16*>(O);
  a.off = static_cast<const int32_t*>(ws_ptr(idx, S_OFF));
  a.S = static_cast<float*>(scratch);
  a.sel_mask_out = prm->sel_mask_out;
  a.scores_out = prm->scores_out;
  a.err = err_word(idx);
  a.units = U;
  a.rows = idx->slots;
  const int64_t blocks_used = (idx->n_clustered + c.block_tokens - 1) / c.block_tokens;
  a.rows_active = (int)std::min<int64_t>(idx->slots, blocks_used * idx->slots_per_block);
  a.max_tokens = c.max_tokens;
  a.n_clustered = (int)idx->n_clustered;
  a.n_tail = (int)(idx->n_tokens - idx->n_clustered);
  a.scale = scale;
  a.budget = prm->budget;
  a.approx = (prm->flags & MP_NO_APPROX) == 0;
  a.timeout_ns = 2000000000LL;
  a.k = cluster_size(U, (a.rows_active + unit::kRows - 1) / unit::kRows, prm->n_split);

  auto phase = [&](int i) {
    if (i < prm->n_phase_events && prm->phase_events[i])
      cudaEventRecord(static_cast<cudaEvent_t>(prm->phase_events[i]), st);
  };
  phase(0);
  cudaError_t e = launch_unit<unit::M_FLAT>(D, G, a, st);
  phase(1);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return MP_ECUDA;
  }
  return MP_OK;
}

// Dense decode over a plain cache: every key of [0, n) of each head exact.
mp_status dense_decode_impl(const mp_config& c, const void* K, const void* V, int n, const void* Q, void* O,
                            float scale, cudaStream_t st) {
  const int U = c.batch * c.kv_heads, G = c.q_heads / c.kv_heads, D = c.head_dim;
  unit::Args a{};
  if (!encode_tiles(&a.tmA, K, (uint64_t)U * c.max_tokens, D, unit::kDRows) ||
      !encode_tiles(&a.tmB, V, (uint64_t)U * c.max_tokens, D, unit::kDRows))
    return MP_ECUDA;
  a.Q = static_cast<const __nv_bfloat16*>(Q);
  a.O = static_cast<__nv_bfloat16*>(O);
  a.units = U;
  a.rows = c.max_tokens;
  a.rows_active = n;
  a.max_tokens = c.max_tokens;
  a.scale = scale != 0.f ? scale : 1.0f / sqrtf((float)D);
  a.approx = 0;
  a.timeout_ns = 2000000000LL;
  a.k = cluster_size(U, (n + unit::kDRows - 1) / unit::kDRows, 0);
  cudaError_t e = launch_unit<unit::M_DENSE>(D, G, a, st);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return MP_ECUDA;
  }
  return MP_OK;
}

}  // namespace mp
