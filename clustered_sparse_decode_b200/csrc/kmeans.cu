// Blockwise Lloyd k-means over keys, the cluster-ordered KV store, the
// two-level hierarchy and the online block update.
//
// "Multipole Attention for Efficient Long Context Reasoning" (arXiv abstract:
// clustering groups semantically similar keys, and a fast cluster update
// re-clusters generated tokens; atlas.scime summary, "Approach": blockwise
// sliding-window online clustering, hierarchical variant).  Coleman Hooper's
// homepage (Squeezed Attention blurb): K-means over keys, one centroid per
// cluster.
//
// Per (batch, KV head, block) of L tokens with C = ceil(L/T) slots:
//   init (k-means++ / stride / given / warm)  ->  iters x { assign; sort; mean(K) }
//   -> [two levels: coarse k-means over fine centroids, reorder fine slots]
//   -> mean(V) -> permute K, V into the store.
// Decisions (nearest centroid) are taken on fp32 distances, ties to the lower
// slot; means are fp64 sums in token order, divided and rounded to the dtype
// once, so centroids are exactly the rounded member means.
#include <algorithm>

#include "mp_internal.cuh"

namespace mp {

// A launch over blocks [blk0, blk0 + gridDim.y) of every unit (gridDim.z).
struct BlockJob {
  const void* srcK;        // token rows of the clustered blocks
  const void* srcV;
  int64_t src_unit_rows;   // rows per unit in src
  int64_t src_row0;        // src row of token blk0 * L_blk
  int blk0;
  int64_t n_total;         // tokens of the index once this job is done (fixes each block's length)
  int L_blk, T, C_blk;
  int Tc, CC_blk;
  void* Kc; void* Vc; int32_t* off; int32_t* perm; int32_t* assign;
  void* Kp; void* Vp;
  void* Kcc; void* Vcc; int32_t* coff;
  void* kctmp; void* vctmp; int32_t* corder;
  int slots, coarse_slots;
  int64_t max_tokens;
  int iters;
  uint64_t seed;
  int32_t* err;
};

struct BlockGeo {
  int j, unit;
  int64_t s;    // first token id of the block
  int L, C;     // tokens, used slots
};

__device__ __forceinline__ BlockGeo block_geo(const BlockJob& b) {
  BlockGeo g;
  g.j = b.blk0 + blockIdx.y;
  g.unit = blockIdx.z;
  g.s = (int64_t)g.j * b.L_blk;
  int64_t rem = b.n_total - g.s;
  g.L = rem <= 0 ? 0 : (int)(rem < (int64_t)b.L_blk ? rem : (int64_t)b.L_blk);
  g.C = (g.L + b.T - 1) / b.T;
  return g;
}

// src row of token id t (a token of the launch's blocks)
__device__ __forceinline__ int64_t src_row(const BlockJob& b, int unit, int64_t t) {
  return (int64_t)unit * b.src_unit_rows + b.src_row0 + (t - (int64_t)b.blk0 * b.L_blk);
}

// ----------------------------------------------------------------------------
// splitmix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
// generators", OOPSLA 2014): state advances by the golden gamma, output is the
// two-multiply mix of the state.
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint64_t sm64_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}
__device__ __forceinline__ uint64_t sm64_out(uint64_t state, uint64_t k) {
  return sm64_mix(state + (k + 1) * 0x9E3779B97F4A7C15ull);
}
// uniform in [0, 1) for pick k of the stream of (unit, block, level)
__device__ __forceinline__ double stream_uniform(uint64_t seed, int unit, int block, int level, int k) {
  uint64_t ctr = (((uint64_t)unit << 20) + (uint64_t)block) * 2ull + (uint64_t)level;
  uint64_t key = sm64_out(seed, ctr);
  return (double)(sm64_out(key, (uint64_t)k) >> 11) * (1.0 / 9007199254740992.0);
}

// Block-wide exclusive scan of one double per thread (thread order).
template <int NT>
__device__ double block_scan_f64(double v, double* s_w, double* total) {
  const int lane = threadIdx.x % kWarp, warp = threadIdx.x / kWarp;
  double x = v;
#pragma unroll
  for (int o = 1; o < kWarp; o <<= 1) {
    double y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  if (lane == kWarp - 1) s_w[warp] = x;
  __syncthreads();
  if (warp == 0) {
    double w = lane < NT / kWarp ? s_w[lane] : 0.0;
#pragma unroll
    for (int o = 1; o < kWarp; o <<= 1) {
      double y = __shfl_up_sync(kFull, w, o);
      if (lane >= o) w += y;
    }
    if (lane < NT / kWarp) s_w[lane] = w;
  }
  __syncthreads();
  double before = (warp > 0 ? s_w[warp - 1] : 0.0) + (x - v);
  *total = s_w[NT / kWarp - 1];
  __syncthreads();
  return before;
}

template <int NT>
__device__ int block_scan_i32(int v, int* s_w, int* total) {
  const int lane = threadIdx.x % kWarp, warp = threadIdx.x / kWarp;
  int x = v;
#pragma unroll
  for (int o = 1; o < kWarp; o <<= 1) {
    int y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  if (lane == kWarp - 1) s_w[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < NT / kWarp ? s_w[lane] : 0;
#pragma unroll
    for (int o = 1; o < kWarp; o <<= 1) {
      int y = __shfl_up_sync(kFull, w, o);
      if (lane >= o) w += y;
    }
    if (lane < NT / kWarp) s_w[lane] = w;
  }
  __syncthreads();
  int before = (warp > 0 ? s_w[warp - 1] : 0) + x - v;
  *total = s_w[NT / kWarp - 1];
  __syncthreads();
  return before;
}

// ----------------------------------------------------------------------------
// k-means++ seeding (Arthur & Vassilvitskii, 2007).  One CTA per block.
// Pick 0 = floor(u0 * L); pick k = first point whose running sum of D^2 exceeds
// u_k * (sum of D^2), D^2 the squared distance to the nearest centre so far
// (fp64); if that sum is 0, pick 0 again.  Points are split into contiguous
// per-thread ranges, so the running sums follow point order.
// ----------------------------------------------------------------------------
constexpr int kPPThreads = 1024;

template <typename T, int D>
__global__ void __launch_bounds__(kPPThreads)
kmeanspp_kernel(BlockJob b) {
  extern __shared__ double s_d2[];            // [L_blk]
  __shared__ double s_c[D];
  __shared__ double s_w[kPPThreads / kWarp];
  __shared__ int s_pick;
  const BlockGeo g = block_geo(b);
  if (g.L == 0) return;
  const int tid = threadIdx.x, lane = tid % kWarp, warp = tid / kWarp;
  const T* src = reinterpret_cast<const T*>(b.srcK) + src_row(b, g.unit, g.s) * D;
  T* Kc = reinterpret_cast<T*>(b.Kc) + ((size_t)g.unit * b.slots + (size_t)g.j * b.C_blk) * D;
  const int per = (g.L + kPPThreads - 1) / kPPThreads;
  const int i0 = min(g.L, tid * per), i1 = min(g.L, i0 + per);
  constexpr int DPL = D / kWarp;

  double u0 = stream_uniform(b.seed, g.unit, g.j, 0, 0);
  int first = (int)floor(u0 * (double)g.L);
  first = min(first, g.L - 1);
  int pick = first;
  for (int k = 0; k < g.C; ++k) {
    if (tid < D) {
      T v = src[(size_t)pick * D + tid];
      Kc[(size_t)k * D + tid] = v;
      s_c[tid] = (double)to_f32(v);
    }
    __syncthreads();
    // D^2 update: each warp walks rows, lanes over dimensions
    for (int i = warp; i < g.L; i += kPPThreads / kWarp) {
      const T* x = src + (size_t)i * D + lane * DPL;
      double acc = 0.0;
#pragma unroll
      for (int e = 0; e < DPL; ++e) {
        double dd = (double)to_f32(x[e]) - s_c[lane * DPL + e];
        acc = fma(dd, dd, acc);
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
      if (lane == 0) s_d2[i] = (k == 0) ? acc : fmin(s_d2[i], acc);
    }
    __syncthreads();
    if (k + 1 == g.C) break;
    double mine = 0.0;
    for (int i = i0; i < i1; ++i) mine += s_d2[i];
    double tot;
    double before = block_scan_f64<kPPThreads>(mine, s_w, &tot);
    if (tid == 0) s_pick = g.L - 1;
    __syncthreads();
    int next = first;
    if (tot > 0.0) {
      const double thr = stream_uniform(b.seed, g.unit, g.j, 0, k + 1) * tot;
      double run = before;
      for (int i = i0; i < i1; ++i) {
        run += s_d2[i];
        if (run > thr) { atomicMin(&s_pick, i); break; }
      }
      __syncthreads();
      next = s_pick;
    }
    __syncthreads();
    pick = next;
  }
}

// The same seeding with far fewer key reads (Elkan, "Using the triangle
// inequality to accelerate k-means", ICML 2003).  Each point keeps its nearest
// centre a_i besides D_i^2.  When centre k is at least twice D_i away from
// c_{a_i}, |x_i - c_k| >= |c_k - c_{a_i}| - D_i >= D_i, so D_i cannot drop and
// row i is not read.  The test carries a relative margin of 1e-9, far above
// the fp64 rounding of the squared distances (about 130 ulp), so a skipped row
// is one whose recomputed D^2 would have lost the min: D^2 and the picks equal
// those of the full pass.  Per pick: centre-to-centre distances (thread per
// earlier centre), a compacted list of the rows left to recompute (thread per
// row, 16-byte loads), then the running sum in 32-row chunks per warp.
constexpr int kPPrThreads = 512;

template <typename T>
__device__ __forceinline__ void unpack16(const uint4& u, float* f);
template <>
__device__ __forceinline__ void unpack16<float>(const uint4& u, float* f) {
  f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y); f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
}
template <>
__device__ __forceinline__ void unpack16<__nv_bfloat16>(const uint4& u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// fp64 squared distance of one row (16-byte aligned) to the centre in s_c
template <typename T, int D, bool NC>
__device__ __forceinline__ double row_dist2(const T* x, const double* s_c) {
  constexpr int EPW = 16 / sizeof(T);
  constexpr int NB = (D / EPW) / 2 < 8 ? (D / EPW) / 2 : 8;   // 16-byte words in flight per thread
  const uint4* xv = reinterpret_cast<const uint4*>(x);
  double acc = 0.0;
#pragma unroll 1
  for (int w0 = 0; w0 < D / EPW; w0 += NB) {
    uint4 u[NB];
#pragma unroll
    for (int w = 0; w < NB; ++w) u[w] = NC ? __ldg(xv + w0 + w) : xv[w0 + w];
#pragma unroll
    for (int w = 0; w < NB; ++w) {
      float f[EPW];
      unpack16<T>(u[w], f);
#pragma unroll
      for (int e = 0; e < EPW; ++e) {
        const double dd = (double)f[e] - s_c[(w0 + w) * EPW + e];
        acc = fma(dd, dd, acc);
      }
    }
  }
  return acc;
}

size_t kmeanspp_pruned_smem(int L_blk, int C_blk) {
  return (size_t)L_blk * (sizeof(double) + 2 * sizeof(uint16_t)) + (size_t)C_blk * sizeof(double) + 16;
}

template <typename T, int D>
__global__ void __launch_bounds__(kPPrThreads, 2)
kmeanspp_pruned_kernel(BlockJob b) {
  constexpr int NT = kPPrThreads, NW = NT / kWarp;
  extern __shared__ double s_d2[];                                   // [L_blk] D^2
  double* s_cc = s_d2 + b.L_blk;                                     // [C_blk] |c_k - c_j|^2
  uint16_t* s_a = reinterpret_cast<uint16_t*>(s_cc + b.C_blk);      // [L_blk] nearest centre
  uint16_t* s_list = s_a + b.L_blk;                                  // [L_blk] rows to recompute
  __shared__ double s_c[D];
  __shared__ double s_w[NW];
  __shared__ int s_pick, s_n;
  const BlockGeo g = block_geo(b);
  if (g.L == 0) return;
  const int tid = threadIdx.x, lane = tid % kWarp, warp = tid / kWarp;
  const T* src = reinterpret_cast<const T*>(b.srcK) + src_row(b, g.unit, g.s) * D;
  T* Kc = reinterpret_cast<T*>(b.Kc) + ((size_t)g.unit * b.slots + (size_t)g.j * b.C_blk) * D;
  // each warp sums and searches a contiguous range of rows, in chunks of 32
  const int rpw = ((g.L + NW - 1) / NW + kWarp - 1) / kWarp * kWarp;
  const int wr0 = min(g.L, warp * rpw), wr1 = min(g.L, wr0 + rpw);

  double u0 = stream_uniform(b.seed, g.unit, g.j, 0, 0);
  int first = (int)floor(u0 * (double)g.L);
  first = min(first, g.L - 1);
  int pick = first;
  for (int k = 0; k < g.C; ++k) {
    if (tid < D) {
      T v = src[(size_t)pick * D + tid];
      Kc[(size_t)k * D + tid] = v;
      s_c[tid] = (double)to_f32(v);
    }
    if (tid == 0) s_n = 0;
    __syncthreads();
    // distances from centre k to the earlier centres (rows of Kc written by this CTA)
#pragma unroll 1
    for (int j = tid; j < k; j += NT) s_cc[j] = row_dist2<T, D, false>(Kc + (size_t)j * D, s_c);
    __syncthreads();
    // rows whose D^2 may drop
    for (int c0 = warp * kWarp; c0 < g.L; c0 += NT) {
      const int i = c0 + lane;
      bool need = false;
      if (i < g.L) need = (k == 0) || !(s_cc[s_a[i]] >= 4.0 * s_d2[i] * (1.0 + 1e-9));
      const unsigned m = __ballot_sync(kFull, need);
      if (m) {
        int base = 0;
        if (lane == 0) base = atomicAdd(&s_n, __popc(m));
        base = __shfl_sync(kFull, base, 0);
        if (need) s_list[base + __popc(m & ((1u << lane) - 1u))] = (uint16_t)i;
      }
    }
    __syncthreads();
    const int n_need = s_n;
#pragma unroll 1
    for (int q = tid; q < n_need; q += NT) {
      const int i = s_list[q];
      const double acc = row_dist2<T, D, true>(src + (size_t)i * D, s_c);
      if (k == 0 || acc < s_d2[i]) { s_d2[i] = acc; s_a[i] = (uint16_t)k; }
    }
    __syncthreads();
    if (k + 1 == g.C) break;
    double part = 0.0;
    for (int c0 = wr0; c0 < wr1; c0 += kWarp) part += (c0 + lane < wr1) ? s_d2[c0 + lane] : 0.0;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) part += __shfl_xor_sync(kFull, part, o);
    if (lane == 0) s_w[warp] = part;
    if (tid == 0) s_pick = g.L - 1;
    __syncthreads();
    double before = 0.0, tot = 0.0;
    for (int w = 0; w < NW; ++w) {
      const double v = s_w[w];
      if (w < warp) before += v;
      tot += v;
    }
    int next = first;
    if (tot > 0.0) {
      const double thr = stream_uniform(b.seed, g.unit, g.j, 0, k + 1) * tot;
      double run = before;
      for (int c0 = wr0; c0 < wr1; c0 += kWarp) {
        const int i = c0 + lane;
        double x = i < wr1 ? s_d2[i] : 0.0;
#pragma unroll
        for (int o = 1; o < kWarp; o <<= 1) {
          const double y = __shfl_up_sync(kFull, x, o);
          if (lane >= o) x += y;
        }
        const unsigned hit = __ballot_sync(kFull, i < wr1 && run + x > thr);
        if (hit) {
          if (lane == 0) atomicMin(&s_pick, c0 + __ffs(hit) - 1);
          break;
        }
        run += __shfl_sync(kFull, x, kWarp - 1);
      }
      __syncthreads();
      next = s_pick;
    }
    __syncthreads();
    pick = next;
  }
}

// Slots [c_from, C) of each block start at src tokens first + (k - c_from) * T
// (the stride initialisation, and the new slots of a warm start).
template <typename T, int D>
__global__ void seed_stride_kernel(BlockJob b, int c_from_tokens) {
  const BlockGeo g = block_geo(b);
  const int c_from = (c_from_tokens + b.T - 1) / b.T;  // slots of the tokens clustered before
  T* Kc = reinterpret_cast<T*>(b.Kc) + ((size_t)g.unit * b.slots + (size_t)g.j * b.C_blk) * D;
  const T* src = reinterpret_cast<const T*>(b.srcK) + src_row(b, g.unit, g.s) * D;
  for (int k = c_from + blockIdx.x; k < g.C; k += gridDim.x) {
    const int64_t t = c_from_tokens + (int64_t)(k - c_from) * b.T;
    for (int e = threadIdx.x; e < D; e += blockDim.x) Kc[(size_t)k * D + e] = src[t * D + e];
  }
}

// Slots [0, C) of each block from caller-given centroids [units][slots][D].
template <typename T, int D>
__global__ void seed_given_kernel(BlockJob b, const T* init) {
  const BlockGeo g = block_geo(b);
  const size_t base = ((size_t)g.unit * b.slots + (size_t)g.j * b.C_blk) * D;
  T* Kc = reinterpret_cast<T*>(b.Kc) + base;
  for (int k = blockIdx.x; k < g.C; k += gridDim.x)
    for (int e = threadIdx.x; e < D; e += blockDim.x) Kc[(size_t)k * D + e] = init[base + (size_t)k * D + e];
}

// ----------------------------------------------------------------------------
// Assignment (SIMT fp32): assign[t] = argmin_c (|c|^2 - 2 x_t . c), ties to the
// lower slot.  A CTA takes 64 tokens against all centroids of the block,
// streamed in tiles of 64; each thread owns a 4 x 4 register tile.
// ----------------------------------------------------------------------------
constexpr int kAT = 64;
constexpr int kALD = kAT + 4;   // padded rows: fewer bank conflicts when staging, 16-byte aligned float4 reads

template <typename T, int D>
__global__ void __launch_bounds__(256)
assign_simt_kernel(BlockJob b) {
  extern __shared__ float s_as[];              // [D][kALD] tokens, then [D][kALD] centroids, then [kAT] norms
  float* s_bs = s_as + D * kALD;
  float* s_cn = s_bs + D * kALD;
  const BlockGeo g = block_geo(b);
  const int i0 = blockIdx.x * kAT;
  if (i0 >= g.L) return;
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  const T* src = reinterpret_cast<const T*>(b.srcK);
  const T* Kc = reinterpret_cast<const T*>(b.Kc) + ((size_t)g.unit * b.slots + (size_t)g.j * b.C_blk) * D;
  for (int idx = tid; idx < kAT * D; idx += 256) {
    int t = idx / D, k = idx % D;
    float v = 0.f;
    if (i0 + t < g.L) v = to_f32(src[src_row(b, g.unit, g.s + i0 + t) * D + k]);
    s_as[k * kALD + t] = v;
  }
  float best[4];
  int besti[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) { best[i] = INFINITY; besti[i] = 0; }
  for (int c0 = 0; c0 < g.C; c0 += kAT) {
    __syncthreads();
    for (int idx = tid; idx < kAT * D; idx += 256) {
      int c = idx / D, k = idx % D;
      s_bs[k * kALD + c] = (c0 + c < g.C) ? to_f32(Kc[(size_t)(c0 + c) * D + k]) : 0.f;
    }
    __syncthreads();
    if (tid < kAT) {
      float sn = 0.f;
      for (int k = 0; k < D; ++k) sn = fmaf(s_bs[k * kALD + tid], s_bs[k * kALD + tid], sn);
      s_cn[tid] = sn;
    }
    __syncthreads();
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) acc[i][jj] = 0.f;
#pragma unroll 8
    for (int k = 0; k < D; ++k) {
      float4 av = *reinterpret_cast<const float4*>(s_as + k * kALD + ty * 4);
      float4 bv = *reinterpret_cast<const float4*>(s_bs + k * kALD + tx * 4);
      float a4[4] = {av.x, av.y, av.z, av.w}, b4[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) acc[i][jj] = fmaf(a4[i], b4[jj], acc[i][jj]);
    }
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int c = c0 + tx * 4 + jj;
      if (c < g.C) {
        const float cn = s_cn[tx * 4 + jj];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float dd = fmaf(-2.f, acc[i][jj], cn);
          if (dd < best[i]) { best[i] = dd; besti[i] = c; }
        }
      }
    }
  }
  // reduce over the 16 threads sharing these tokens (same half-warp)
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float bd = best[i];
    int bi = besti[i];
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) {
      float od = __shfl_xor_sync(kFull, bd, o);
      int oi = __shfl_xor_sync(kFull, bi, o);
      if (od < bd || (od == bd && oi < bi)) { bd = od; bi = oi; }
    }
    const int t = i0 + ty * 4 + i;
    if (tx == 0 && t < g.L) b.assign[(size_t)g.unit * b.max_tokens + g.s + t] = g.j * b.C_blk + bi;
  }
}

// ----------------------------------------------------------------------------
// Stable counting sort of a block's tokens by slot -> perm rows and offsets.
// Warp w owns a contiguous range of tokens; per-warp histograms give each warp
// its base per slot, and __match_any_sync ranks equal slots inside a step, so
// tokens of a slot keep their id order.
// ----------------------------------------------------------------------------
constexpr int kSortThreads = 1024;
constexpr int kSortWarps = kSortThreads / kWarp;

__global__ void __launch_bounds__(kSortThreads)
sort_kernel(BlockJob b) {
  extern __shared__ uint16_t s_hist[];                 // [kSortWarps][C_blk]
  int* s_tot = reinterpret_cast<int*>(s_hist + kSortWarps * ((b.C_blk + 1) & ~1));  // [C_blk]
  __shared__ int s_w[kSortWarps];
  const BlockGeo g = block_geo(b);
  if (g.L == 0) return;
  const int tid = threadIdx.x, lane = tid % kWarp, warp = tid / kWarp;
  const int Cb = b.C_blk;
  const int32_t* asg = b.assign + (size_t)g.unit * b.max_tokens + g.s;
  int32_t* perm = b.perm + (size_t)g.unit * b.max_tokens + g.s;
  int32_t* off = b.off + (size_t)g.unit * (b.slots + 1) + (size_t)g.j * Cb;
  const int tpw = (g.L + kSortWarps - 1) / kSortWarps;
  const int w0 = min(g.L, warp * tpw), w1 = min(g.L, w0 + tpw);
  for (int i = tid; i < kSortWarps * Cb; i += kSortThreads) s_hist[i] = 0;
  __syncthreads();
  uint16_t* h = s_hist + warp * Cb;
  const int cbase = g.j * Cb;
  for (int t0 = w0; t0 < w1; t0 += kWarp) {
    const int t = t0 + lane;
    const bool act = t < w1;
    int a = act ? asg[t] - cbase : 0;
    if (act && (a < 0 || a >= g.C)) { set_error(b.err, E_BAD_OFFSET); a = 0; }
    const unsigned am = __ballot_sync(kFull, act);
    if (act) {
      const unsigned peers = __match_any_sync(am, a);
      if (lane == __ffs(peers) - 1) h[a] = (uint16_t)(h[a] + __popc(peers));
    }
    __syncwarp();
  }
  __syncthreads();
  for (int c = tid; c < Cb; c += kSortThreads) {
    int run = 0;
    for (int w = 0; w < kSortWarps; ++w) {
      int v = s_hist[w * Cb + c];
      s_hist[w * Cb + c] = (uint16_t)run;
      run += v;
    }
    s_tot[c] = run;
  }
  __syncthreads();
  // exclusive scan of slot totals (each thread a contiguous range of slots)
  const int per = (Cb + kSortThreads - 1) / kSortThreads;
  const int c0 = min(Cb, tid * per), c1 = min(Cb, c0 + per);
  int mine = 0;
  for (int c = c0; c < c1; ++c) mine += s_tot[c];
  int total;
  int run = block_scan_i32<kSortThreads>(mine, s_w, &total);
  for (int c = c0; c < c1; ++c) { int v = s_tot[c]; s_tot[c] = run; run += v; }
  __syncthreads();
  for (int c = tid; c < Cb; c += kSortThreads) off[c] = (int32_t)(g.s + (c < g.C ? s_tot[c] : g.L));
  for (int t0 = w0; t0 < w1; t0 += kWarp) {
    const int t = t0 + lane;
    const bool act = t < w1;
    int a = act ? asg[t] - cbase : 0;
    if (act && (a < 0 || a >= g.C)) a = 0;
    const unsigned am = __ballot_sync(kFull, act);
    if (act) {
      const unsigned peers = __match_any_sync(am, a);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      const int pos = s_tot[a] + h[a] + rank;
      perm[pos] = (int32_t)(g.s + t);
      __syncwarp(am);
      if (lane == __ffs(peers) - 1) h[a] = (uint16_t)(h[a] + __popc(peers));
    }
    __syncwarp();
  }
}

// ----------------------------------------------------------------------------
// Member means: one warp per slot, fp64 sums over the members in store order
// (= token id order), one division, one rounding to the dtype.  Empty slots
// keep their key centroid; their value centroid is zero.
// ----------------------------------------------------------------------------
template <typename T, int D, bool VALUES>
__global__ void mean_kernel(BlockJob b) {
  constexpr int DPL = D / kWarp;
  const BlockGeo g = block_geo(b);
  const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
  const int c = blockIdx.x * (blockDim.x / kWarp) + warp;
  if (c >= g.C) return;
  const int32_t* off = b.off + (size_t)g.unit * (b.slots + 1) + (size_t)g.j * b.C_blk;
  const int32_t* perm = b.perm + (size_t)g.unit * b.max_tokens;
  const int a0 = off[c];
  const int a1 = (c + 1 < b.C_blk) ? off[c + 1] : (int)(g.s + g.L);
  T* out = reinterpret_cast<T*>(VALUES ? b.Vc : b.Kc) + ((size_t)g.unit * b.slots + (size_t)g.j * b.C_blk + c) * D;
  const T* src = reinterpret_cast<const T*>(VALUES ? b.srcV : b.srcK);
  if (a1 <= a0) {
    if (VALUES)
      for (int e = lane; e < D; e += kWarp) out[e] = from_f32<T>(0.f);
    return;
  }
  double acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] = 0.0;
  for (int p = a0; p < a1; ++p) {
    const int64_t id = perm[p];
    const T* x = src + src_row(b, g.unit, id) * D + lane * DPL;
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[e] += (double)to_f32(x[e]);
  }
  const double n = (double)(a1 - a0);
#pragma unroll
  for (int e = 0; e < DPL; ++e) out[lane * DPL + e] = round_from_f64<T>(acc[e] / n);
}

// Store rows [s, s + L): K, V rows of the tokens listed in perm.
template <typename T, int D>
__global__ void permute_kernel(BlockJob b) {
  const BlockGeo g = block_geo(b);
  const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
  const int r = blockIdx.x * (blockDim.x / kWarp) + warp;
  if (r >= g.L) return;
  const int64_t p = g.s + r;
  const int64_t id = b.perm[(size_t)g.unit * b.max_tokens + p];
  const int64_t sr = src_row(b, g.unit, id);
  const T* sk = reinterpret_cast<const T*>(b.srcK) + sr * D;
  const T* sv = reinterpret_cast<const T*>(b.srcV) + sr * D;
  T* dk = reinterpret_cast<T*>(b.Kp) + ((size_t)g.unit * b.max_tokens + p) * D;
  T* dv = reinterpret_cast<T*>(b.Vp) + ((size_t)g.unit * b.max_tokens + p) * D;
  for (int e = lane; e < D; e += kWarp) { dk[e] = sk[e]; dv[e] = sv[e]; }
}

// Store rows of one block back to token order (update staging).
template <typename T, int D>
__global__ void unpermute_kernel(BlockJob b, T* dstK, T* dstV) {
  const BlockGeo g = block_geo(b);
  const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
  const int r = blockIdx.x * (blockDim.x / kWarp) + warp;
  if (r >= g.L) return;
  const int64_t p = g.s + r;
  int64_t id = b.perm[(size_t)g.unit * b.max_tokens + p];
  if (id < g.s || id >= g.s + g.L) { set_error(b.err, E_BAD_OFFSET); return; }
  const T* sk = reinterpret_cast<const T*>(b.Kp) + ((size_t)g.unit * b.max_tokens + p) * D;
  const T* sv = reinterpret_cast<const T*>(b.Vp) + ((size_t)g.unit * b.max_tokens + p) * D;
  T* dk = dstK + ((size_t)g.unit * b.L_blk + (id - g.s)) * D;
  T* dv = dstV + ((size_t)g.unit * b.L_blk + (id - g.s)) * D;
  for (int e = lane; e < D; e += kWarp) { dk[e] = sk[e]; dv[e] = sv[e]; }
}

// ----------------------------------------------------------------------------
// Coarse level of one block (two-level index): count-weighted k-means over the
// block's fine centroids (weighted k-means++, then Lloyd with fp32 decisions
// and fp64 weighted means in slot order), the stable slot order by coarse
// cluster (corder: new local position of each fine slot) and coff.
// ----------------------------------------------------------------------------
constexpr int kCoarseThreads = 512;

template <typename T, int D>
__global__ void __launch_bounds__(kCoarseThreads)
coarse_kernel(BlockJob b) {
  constexpr int NW = kCoarseThreads / kWarp;
  constexpr int DPL = D / kWarp;
  constexpr int LD = D + 1;                            // padded centroid rows: lane k reads row k conflict-free
  extern __shared__ double s_cd2[];                   // [C_blk] D^2
  float* s_cent = reinterpret_cast<float*>(s_cd2 + b.C_blk);    // [CC_blk][LD]
  float* s_cnorm = s_cent + (size_t)b.CC_blk * LD;              // [CC_blk]
  float* s_f = s_cnorm + b.CC_blk;                              // [NW][D] staged fine centroid per warp
  int* s_wt = reinterpret_cast<int*>(s_f + NW * D);             // [C_blk]
  int* s_ca = s_wt + b.C_blk;                                   // [C_blk]
  int* s_cstart = s_ca + b.C_blk;                               // [CC_blk]
  __shared__ double s_w[NW];
  __shared__ int s_wi[NW];
  __shared__ int s_pick;
  const BlockGeo g = block_geo(b);
  if (g.L == 0) return;
  const int tid = threadIdx.x, lane = tid % kWarp, warp = tid / kWarp;
  const int C = g.C;
  const int CC = (g.L + b.Tc - 1) / b.Tc;
  const T* F = reinterpret_cast<const T*>(b.Kc) + ((size_t)g.unit * b.slots + (size_t)g.j * b.C_blk) * D;
  const int32_t* off = b.off + (size_t)g.unit * (b.slots + 1) + (size_t)g.j * b.C_blk;
  for (int c = tid; c < C; c += kCoarseThreads) {
    int a1 = (c + 1 < b.C_blk) ? off[c + 1] : (int)(g.s + g.L);
    s_wt[c] = a1 - off[c];
  }
  __syncthreads();
  const int per = (C + kCoarseThreads - 1) / kCoarseThreads;
  const int c0 = min(C, tid * per), c1 = min(C, c0 + per);

  // weighted k-means++: pick 0 by weight, then by weight * D^2
  int wmine = 0;
  for (int c = c0; c < c1; ++c) wmine += s_wt[c];
  int wtot;
  int wbefore = block_scan_i32<kCoarseThreads>(wmine, s_wi, &wtot);
  if (tid == 0) s_pick = C - 1;
  __syncthreads();
  {
    const double thr = stream_uniform(b.seed, g.unit, g.j, 1, 0) * (double)wtot;
    double run = (double)wbefore;
    for (int c = c0; c < c1; ++c) {
      run += (double)s_wt[c];
      if (run > thr) { atomicMin(&s_pick, c); break; }
    }
  }
  __syncthreads();
  const int first = s_pick;
  int pick = first;
  __syncthreads();
  for (int k = 0; k < CC; ++k) {
    for (int e = tid; e < D; e += kCoarseThreads) s_cent[(size_t)k * LD + e] = to_f32(F[(size_t)pick * D + e]);
    __syncthreads();
    for (int c = warp; c < C; c += NW) {
      double acc = 0.0;
#pragma unroll
      for (int e = 0; e < DPL; ++e) {
        double dd = (double)to_f32(F[(size_t)c * D + lane * DPL + e]) - (double)s_cent[(size_t)k * LD + lane * DPL + e];
        acc = fma(dd, dd, acc);
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
      if (lane == 0) s_cd2[c] = (k == 0) ? acc : fmin(s_cd2[c], acc);
    }
    __syncthreads();
    if (k + 1 == CC) break;
    double mine = 0.0;
    for (int c = c0; c < c1; ++c) mine += (double)s_wt[c] * s_cd2[c];
    double tot;
    double before = block_scan_f64<kCoarseThreads>(mine, s_w, &tot);
    if (tid == 0) s_pick = C - 1;
    __syncthreads();
    int next = first;
    if (tot > 0.0) {
      const double thr = stream_uniform(b.seed, g.unit, g.j, 1, k + 1) * tot;
      double run = before;
      for (int c = c0; c < c1; ++c) {
        run += (double)s_wt[c] * s_cd2[c];
        if (run > thr) { atomicMin(&s_pick, c); break; }
      }
      __syncthreads();
      next = s_pick;
    }
    __syncthreads();
    pick = next;
  }
  // Lloyd, count-weighted
  float* fw = s_f + warp * D;
  for (int it = 0; it < b.iters; ++it) {
    for (int k = tid; k < CC; k += kCoarseThreads) {
      float sn = 0.f;
      for (int e = 0; e < D; ++e) sn = fmaf(s_cent[(size_t)k * LD + e], s_cent[(size_t)k * LD + e], sn);
      s_cnorm[k] = sn;
    }
    __syncthreads();
    // nearest coarse centroid of each fine centroid: warp per fine slot, lanes over coarse slots
    for (int c = warp; c < C; c += NW) {
      for (int e = lane; e < D; e += kWarp) fw[e] = to_f32(F[(size_t)c * D + e]);
      __syncwarp();
      float bd = INFINITY;
      int bi = 0x7fffffff;
      for (int k = lane; k < CC; k += kWarp) {
        float dot = 0.f;
        for (int e = 0; e < D; ++e) dot = fmaf(fw[e], s_cent[(size_t)k * LD + e], dot);
        const float dd = fmaf(-2.f, dot, s_cnorm[k]);
        if (dd < bd) { bd = dd; bi = k; }
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) {
        const float od = __shfl_xor_sync(kFull, bd, o);
        const int oi = __shfl_xor_sync(kFull, bi, o);
        if (od < bd || (od == bd && oi < bi)) { bd = od; bi = oi; }
      }
      if (lane == 0) s_ca[c] = bi;
      __syncwarp();
    }
    __syncthreads();
    for (int k = warp; k < CC; k += NW) {
      double acc[DPL];
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[e] = 0.0;
      double sw = 0.0;
      for (int c = 0; c < C; ++c) {
        if (s_ca[c] != k || s_wt[c] == 0) continue;
        const double w = (double)s_wt[c];
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc[e] += w * (double)to_f32(F[(size_t)c * D + lane * DPL + e]);
        sw += w;
      }
      if (sw > 0.0) {
#pragma unroll
        for (int e = 0; e < DPL; ++e)
          s_cent[(size_t)k * LD + lane * DPL + e] = to_f32(round_from_f64<T>(acc[e] / sw));
      }
    }
    __syncthreads();
  }
  // stable order of fine slots by coarse cluster
  for (int k = tid; k < b.CC_blk; k += kCoarseThreads) s_cstart[k] = 0;
  __syncthreads();
  for (int c = tid; c < C; c += kCoarseThreads) atomicAdd(&s_cstart[s_ca[c]], 1);
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int k = 0; k < CC; ++k) { int v = s_cstart[k]; s_cstart[k] = run; run += v; }
  }
  __syncthreads();
  int32_t* corder = b.corder + (size_t)g.unit * b.slots + (size_t)g.j * b.C_blk;
  for (int c = tid; c < C; c += kCoarseThreads) {
    const int k = s_ca[c];
    int rank = 0;
    for (int c2 = 0; c2 < c; ++c2) rank += (s_ca[c2] == k);
    corder[c] = s_cstart[k] + rank;
  }
  int32_t* coff = b.coff + (size_t)g.unit * (b.coarse_slots + 1) + (size_t)g.j * b.CC_blk;
  for (int k = tid; k < b.CC_blk; k += kCoarseThreads)
    coff[k] = g.j * b.C_blk + (k < CC ? s_cstart[k] : C);
  T* Kcc = reinterpret_cast<T*>(b.Kcc) + ((size_t)g.unit * b.coarse_slots + (size_t)g.j * b.CC_blk) * D;
  for (int i = tid; i < b.CC_blk * D; i += kCoarseThreads) {
    const int k = i / D, e = i % D;
    Kcc[i] = from_f32<T>(k < CC ? s_cent[(size_t)k * LD + e] : 0.f);
  }
}

// Fine slots of a block move to their coarse-sorted position: centroids via
// the tmp copies, token assignments in place.
template <typename T, int D>
__global__ void remap_to_tmp_kernel(BlockJob b) {
  const BlockGeo g = block_geo(b);
  const size_t base = (size_t)g.unit * b.slots + (size_t)g.j * b.C_blk;
  const int32_t* corder = b.corder + base;
  for (int c = blockIdx.x; c < g.C; c += gridDim.x) {
    const size_t dst = (base + corder[c]) * D, srco = (base + c) * D;
    for (int e = threadIdx.x; e < D; e += blockDim.x) {
      reinterpret_cast<T*>(b.kctmp)[dst + e] = reinterpret_cast<const T*>(b.Kc)[srco + e];
    }
  }
}

template <typename T, int D>
__global__ void remap_back_kernel(BlockJob b) {
  const BlockGeo g = block_geo(b);
  const size_t base = (size_t)g.unit * b.slots + (size_t)g.j * b.C_blk;
  for (int c = blockIdx.x; c < g.C; c += gridDim.x)
    for (int e = threadIdx.x; e < D; e += blockDim.x)
      reinterpret_cast<T*>(b.Kc)[(base + c) * D + e] = reinterpret_cast<const T*>(b.kctmp)[(base + c) * D + e];
  // token assignments: old local slot -> new local slot
  const int32_t* corder = b.corder + base;
  int32_t* asg = b.assign + (size_t)g.unit * b.max_tokens + g.s;
  const int cb = g.j * b.C_blk;
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < g.L; t += gridDim.x * blockDim.x) {
    int a = asg[t] - cb;
    if (a < 0 || a >= g.C) { set_error(b.err, E_BAD_OFFSET); continue; }
    asg[t] = cb + corder[a];
  }
}

// Coarse centroids = means of their member tokens (store order of the new
// slot order); empty coarse clusters keep their Lloyd centroid, value 0.
template <typename T, int D>
__global__ void coarse_mean_kernel(BlockJob b) {
  constexpr int DPL = D / kWarp;
  const BlockGeo g = block_geo(b);
  const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
  const int k = blockIdx.x * (blockDim.x / kWarp) + warp;
  const int CC = (g.L + b.Tc - 1) / b.Tc;
  if (k >= CC) return;
  const int32_t* coff = b.coff + (size_t)g.unit * (b.coarse_slots + 1) + (size_t)g.j * b.CC_blk;
  const int32_t* off = b.off + (size_t)g.unit * (b.slots + 1);
  const int f0 = coff[k];
  const int f1 = (k + 1 < b.CC_blk) ? coff[k + 1] : g.j * b.C_blk + b.C_blk;
  const int blk_end_slot = g.j * b.C_blk + b.C_blk;
  const int r0 = (f0 < blk_end_slot) ? off[f0] : (int)(g.s + g.L);
  const int r1 = (f1 < blk_end_slot) ? off[f1] : (int)(g.s + g.L);
  const int32_t* perm = b.perm + (size_t)g.unit * b.max_tokens;
  T* Kcc = reinterpret_cast<T*>(b.Kcc) + ((size_t)g.unit * b.coarse_slots + (size_t)g.j * b.CC_blk + k) * D;
  T* Vcc = reinterpret_cast<T*>(b.Vcc) + ((size_t)g.unit * b.coarse_slots + (size_t)g.j * b.CC_blk + k) * D;
  if (r1 <= r0) {
    for (int e = lane; e < D; e += kWarp) Vcc[e] = from_f32<T>(0.f);
    return;
  }
  double ak[DPL], av[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) { ak[e] = 0.0; av[e] = 0.0; }
  for (int p = r0; p < r1; ++p) {
    const int64_t sr = src_row(b, g.unit, perm[p]);
    const T* xk = reinterpret_cast<const T*>(b.srcK) + sr * D + lane * DPL;
    const T* xv = reinterpret_cast<const T*>(b.srcV) + sr * D + lane * DPL;
#pragma unroll
    for (int e = 0; e < DPL; ++e) { ak[e] += (double)to_f32(xk[e]); av[e] += (double)to_f32(xv[e]); }
  }
  const double n = (double)(r1 - r0);
#pragma unroll
  for (int e = 0; e < DPL; ++e) {
    Kcc[lane * DPL + e] = round_from_f64<T>(ak[e] / n);
    Vcc[lane * DPL + e] = round_from_f64<T>(av[e] / n);
  }
}

// Index bookkeeping kernels.
__global__ void fill_i32_kernel(int32_t* p, size_t n, int32_t v) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) p[i] = v;
}

// off[unit][c] = value for c in [c_from, slots]; coff of blocks >= blk_from: first slot of the block.
__global__ void fill_tail_offsets_kernel(int32_t* off, int slots, int c_from, int32_t value, int32_t* coff,
                                         int coarse_slots, int cc_from, int CC_blk, int C_blk) {
  const int unit = blockIdx.y;
  for (int c = c_from + blockIdx.x * blockDim.x + threadIdx.x; c <= slots; c += gridDim.x * blockDim.x)
    off[(size_t)unit * (slots + 1) + c] = value;
  if (coff)
    for (int k = cc_from + blockIdx.x * blockDim.x + threadIdx.x; k <= coarse_slots; k += gridDim.x * blockDim.x)
      coff[(size_t)unit * (coarse_slots + 1) + k] = (k == coarse_slots) ? slots : (k / CC_blk) * C_blk;
}

// Appended rows of one unit (blockIdx.y): K, V rows [n0, n0 + n_new) of the
// store from the caller's [unit][n_new] rows, perm = own id, assign = -1.  W is
// the copy word (16 bytes when every address and row is 16-byte aligned).
template <typename W>
__global__ void append_kernel(const char* Kn, const char* Vn, char* Kp, char* Vp, size_t row_bytes, int64_t max_tokens,
                              int64_t n0, int n_new, int32_t* perm, int32_t* assign) {
  const int unit = blockIdx.y;
  const size_t words = (size_t)n_new * row_bytes / sizeof(W);
  const W* sk = reinterpret_cast<const W*>(Kn + (size_t)unit * n_new * row_bytes);
  const W* sv = reinterpret_cast<const W*>(Vn + (size_t)unit * n_new * row_bytes);
  W* dk = reinterpret_cast<W*>(Kp + ((size_t)unit * max_tokens + n0) * row_bytes);
  W* dv = reinterpret_cast<W*>(Vp + ((size_t)unit * max_tokens + n0) * row_bytes);
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < words; i += (size_t)gridDim.x * blockDim.x) {
    dk[i] = sk[i];
    dv[i] = sv[i];
  }
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_new; i += gridDim.x * blockDim.x) {
    perm[(size_t)unit * max_tokens + n0 + i] = (int32_t)(n0 + i);
    assign[(size_t)unit * max_tokens + n0 + i] = -1;
  }
}

// ----------------------------------------------------------------------------
// Host side
// ----------------------------------------------------------------------------
static BlockJob make_job(const mp_index* idx) {
  const mp_config& c = idx->cfg;
  BlockJob b{};
  b.L_blk = c.block_tokens;
  b.T = c.tokens_per_centroid;
  b.C_blk = idx->slots_per_block;
  b.Tc = c.levels == 2 ? c.coarse_tokens_per_centroid : 1;
  b.CC_blk = idx->coarse_per_block;
  b.Kc = ws_ptr(idx, S_KC); b.Vc = ws_ptr(idx, S_VC);
  b.off = static_cast<int32_t*>(ws_ptr(idx, S_OFF));
  b.perm = static_cast<int32_t*>(ws_ptr(idx, S_PERM));
  b.assign = static_cast<int32_t*>(ws_ptr(idx, S_ASSIGN));
  b.Kp = ws_ptr(idx, S_KP); b.Vp = ws_ptr(idx, S_VP);
  if (c.levels == 2) {
    b.Kcc = ws_ptr(idx, S_KCC); b.Vcc = ws_ptr(idx, S_VCC);
    b.coff = static_cast<int32_t*>(ws_ptr(idx, S_COFF));
    b.corder = static_cast<int32_t*>(ws_ptr(idx, S_CORDER));
  }
  b.kctmp = ws_ptr(idx, S_KCTMP);
  b.vctmp = ws_ptr(idx, S_VCTMP);
  b.slots = idx->slots;
  b.coarse_slots = idx->coarse_slots;
  b.max_tokens = c.max_tokens;
  b.iters = c.kmeans_iters;
  b.seed = c.seed;
  b.err = err_word(idx);
  return b;
}

// The tensor-core assignment (assign_tc.cu) for bf16 keys.
bool assign_tc_supported(int dtype, int D, int C_blk, const void* srcK, const void* Kc, int64_t src_rows_total,
                         int64_t centroid_rows);
cudaError_t launch_assign_tc(int D, const void* srcK, int64_t src_rows_total, int64_t src_unit_rows, int64_t src_row0,
                             const void* Kc, int units, int slots, int blk0, int nbj, int L_blk, int T, int C_blk,
                             int64_t n_total, int32_t* assign, int64_t max_tokens, int32_t* err, cudaStream_t st);

template <typename T, int D>
static cudaError_t run_lloyd(const BlockJob& b, int nbj, int units, int init_mode, int L_old_tokens,
                             const void* init, int levels, cudaStream_t st) {
  const dim3 gb(1, nbj, units);
  // 1. initial centroids
  if (init != nullptr) {
    seed_given_kernel<T, D><<<dim3(64, nbj, units), 128, 0, st>>>(b, static_cast<const T*>(init));
  } else if (init_mode == MP_INIT_KMEANSPP) {
    const size_t smem_p = kmeanspp_pruned_smem(b.L_blk, b.C_blk);
    if (smem_p <= 200 * 1024 && b.L_blk <= 65535 && b.C_blk <= 65535 && ((uintptr_t)b.srcK & 15u) == 0 &&
        ((uintptr_t)b.Kc & 15u) == 0) {
      cudaError_t e = cudaFuncSetAttribute(kmeanspp_pruned_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem_p);
      if (e != cudaSuccess) return e;
      kmeanspp_pruned_kernel<T, D><<<gb, kPPrThreads, smem_p, st>>>(b);
    } else {
      size_t smem = (size_t)b.L_blk * sizeof(double);
      cudaError_t e = cudaFuncSetAttribute(kmeanspp_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      kmeanspp_kernel<T, D><<<gb, kPPThreads, smem, st>>>(b);
    }
  } else {
    seed_stride_kernel<T, D><<<dim3(64, nbj, units), 128, 0, st>>>(b, L_old_tokens);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // 2. Lloyd iterations
  const size_t smem_a = (size_t)(2 * D * kALD + kAT) * sizeof(float);
  e = cudaFuncSetAttribute(assign_simt_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_a);
  if (e != cudaSuccess) return e;
  const size_t smem_s = (size_t)kSortWarps * ((b.C_blk + 1) & ~1) * sizeof(uint16_t) + (size_t)b.C_blk * sizeof(int);
  e = cudaFuncSetAttribute(sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_s);
  if (e != cudaSuccess) return e;
  const int tiles = (b.L_blk + kAT - 1) / kAT;
  const int mean_blocks = (b.C_blk + 7) / 8;
  const int64_t src_rows = (int64_t)units * b.src_unit_rows + b.src_row0;
  const bool tc = assign_tc_supported(DT<T>::id, D, b.C_blk, b.srcK, b.Kc, src_rows, (int64_t)units * b.slots);
  for (int it = 0; it < b.iters; ++it) {
    if (tc) {
      e = launch_assign_tc(D, b.srcK, src_rows, b.src_unit_rows, b.src_row0, b.Kc, units, b.slots, b.blk0, nbj,
                           b.L_blk, b.T, b.C_blk, b.n_total, b.assign, b.max_tokens, b.err, st);
      if (e != cudaSuccess) return e;
    } else {
      assign_simt_kernel<T, D><<<dim3(tiles, nbj, units), 256, smem_a, st>>>(b);
    }
    sort_kernel<<<gb, kSortThreads, smem_s, st>>>(b);
    mean_kernel<T, D, false><<<dim3(mean_blocks, nbj, units), 256, 0, st>>>(b);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // 3. coarse level
  if (levels == 2) {
    const size_t smem_c = (size_t)b.C_blk * sizeof(double) + (size_t)b.CC_blk * (D + 2) * sizeof(float) +
                          (size_t)(kCoarseThreads / kWarp) * D * sizeof(float) +
                          (size_t)(2 * b.C_blk + b.CC_blk) * sizeof(int);
    e = cudaFuncSetAttribute(coarse_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_c);
    if (e != cudaSuccess) return e;
    coarse_kernel<T, D><<<gb, kCoarseThreads, smem_c, st>>>(b);
    remap_to_tmp_kernel<T, D><<<dim3(64, nbj, units), 128, 0, st>>>(b);
    remap_back_kernel<T, D><<<dim3(64, nbj, units), 128, 0, st>>>(b);
    sort_kernel<<<gb, kSortThreads, smem_s, st>>>(b);
    coarse_mean_kernel<T, D><<<dim3((b.CC_blk + 7) / 8, nbj, units), 256, 0, st>>>(b);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // 4. value centroids and the store
  mean_kernel<T, D, true><<<dim3(mean_blocks, nbj, units), 256, 0, st>>>(b);
  permute_kernel<T, D><<<dim3((b.L_blk + 7) / 8, nbj, units), 256, 0, st>>>(b);
  return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t run_lloyd_any(const BlockJob& b, int nbj, int units, int init_mode, int L_old, const void* init,
                                 int levels, cudaStream_t st) {
  return run_lloyd<T, D>(b, nbj, units, init_mode, L_old, init, levels, st);
}

static cudaError_t dispatch_lloyd(int dtype, int D, const BlockJob& b, int nbj, int units, int init_mode, int L_old,
                                  const void* init, int levels, cudaStream_t st) {
  if (dtype == MP_BF16) {
    if (D == 128) return run_lloyd_any<__nv_bfloat16, 128>(b, nbj, units, init_mode, L_old, init, levels, st);
    if (D == 64) return run_lloyd_any<__nv_bfloat16, 64>(b, nbj, units, init_mode, L_old, init, levels, st);
  } else {
    if (D == 128) return run_lloyd_any<float, 128>(b, nbj, units, init_mode, L_old, init, levels, st);
    if (D == 64) return run_lloyd_any<float, 64>(b, nbj, units, init_mode, L_old, init, levels, st);
  }
  return cudaErrorInvalidValue;
}

static cudaError_t fill_tail_offsets(const mp_index* idx, int64_t n, int blocks_used, cudaStream_t st) {
  const int units = idx->cfg.batch * idx->cfg.kv_heads;
  int32_t* off = static_cast<int32_t*>(ws_ptr(idx, S_OFF));
  int32_t* coff = idx->cfg.levels == 2 ? static_cast<int32_t*>(ws_ptr(idx, S_COFF)) : nullptr;
  fill_tail_offsets_kernel<<<dim3(16, units), 256, 0, st>>>(off, idx->slots, blocks_used * idx->slots_per_block,
                                                           (int32_t)n, coff, idx->coarse_slots,
                                                           blocks_used * idx->coarse_per_block,
                                                           std::max(idx->coarse_per_block, 1), idx->slots_per_block);
  return cudaGetLastError();
}

mp_status build_impl(mp_index* idx, const void* K, const void* V, int32_t n, const void* init, cudaStream_t st) {
  const mp_config& c = idx->cfg;
  const int units = c.batch * c.kv_heads;
  const int es = elem_bytes(c.dtype);
  const size_t D = c.head_dim;
  cudaError_t e = cudaSuccess;
  // reset the index
  e = cudaMemsetAsync(ws_ptr(idx, S_KC), 0, (size_t)units * idx->slots * D * es, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws_ptr(idx, S_VC), 0, (size_t)units * idx->slots * D * es, st);
  if (e == cudaSuccess && c.levels == 2) {
    e = cudaMemsetAsync(ws_ptr(idx, S_KCC), 0, (size_t)units * idx->coarse_slots * D * es, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(ws_ptr(idx, S_VCC), 0, (size_t)units * idx->coarse_slots * D * es, st);
  }
  if (e != cudaSuccess) return MP_ECUDA;
  fill_i32_kernel<<<256, 256, 0, st>>>(static_cast<int32_t*>(ws_ptr(idx, S_PERM)), (size_t)units * c.max_tokens, -1);
  fill_i32_kernel<<<256, 256, 0, st>>>(static_cast<int32_t*>(ws_ptr(idx, S_ASSIGN)), (size_t)units * c.max_tokens, -1);
  const int nb = (n + c.block_tokens - 1) / c.block_tokens;
  e = fill_tail_offsets(idx, n, nb, st);
  if (e != cudaSuccess) return MP_ECUDA;
  idx->n_tokens = 0;
  idx->n_clustered = 0;
  if (n == 0) return MP_OK;
  BlockJob b = make_job(idx);
  b.srcK = K; b.srcV = V;
  b.src_unit_rows = n;
  b.src_row0 = 0;
  b.blk0 = 0;
  b.n_total = n;
  e = dispatch_lloyd(c.dtype, c.head_dim, b, nb, units, c.init, 0, init, c.levels, st);
  if (e != cudaSuccess) return MP_ECUDA;
  idx->n_tokens = n;
  idx->n_clustered = n;
  return MP_OK;
}

// One assignment step of every block of the index against its current
// centroids: the job of a build over the caller's keys, with the output rows
// [unit][n] of the caller's array.
template <typename T, int D>
static cudaError_t run_assign(const BlockJob& b, int nbj, int units, cudaStream_t st) {
  const int64_t src_rows = (int64_t)units * b.src_unit_rows + b.src_row0;
  if (assign_tc_supported(DT<T>::id, D, b.C_blk, b.srcK, b.Kc, src_rows, (int64_t)units * b.slots))
    return launch_assign_tc(D, b.srcK, src_rows, b.src_unit_rows, b.src_row0, b.Kc, units, b.slots, b.blk0, nbj,
                            b.L_blk, b.T, b.C_blk, b.n_total, b.assign, b.max_tokens, b.err, st);
  const size_t smem_a = (size_t)(2 * D * kALD + kAT) * sizeof(float);
  cudaError_t e =
      cudaFuncSetAttribute(assign_simt_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_a);
  if (e != cudaSuccess) return e;
  assign_simt_kernel<T, D><<<dim3((b.L_blk + kAT - 1) / kAT, nbj, units), 256, smem_a, st>>>(b);
  return cudaGetLastError();
}

mp_status assign_impl(const mp_index* idx, const void* K, int32_t n, int32_t* out, cudaStream_t st) {
  const mp_config& c = idx->cfg;
  if (n == 0) return MP_OK;
  const int units = c.batch * c.kv_heads;
  BlockJob b = make_job(idx);
  b.srcK = K;
  b.src_unit_rows = n;
  b.src_row0 = 0;
  b.blk0 = 0;
  b.n_total = n;
  b.assign = out;
  b.max_tokens = n;
  const int nb = (n + c.block_tokens - 1) / c.block_tokens;
  cudaError_t e = cudaErrorInvalidValue;
  if (c.dtype == MP_BF16) {
    if (c.head_dim == 128) e = run_assign<__nv_bfloat16, 128>(b, nb, units, st);
    else if (c.head_dim == 64) e = run_assign<__nv_bfloat16, 64>(b, nb, units, st);
  } else {
    if (c.head_dim == 128) e = run_assign<float, 128>(b, nb, units, st);
    else if (c.head_dim == 64) e = run_assign<float, 64>(b, nb, units, st);
  }
  return e == cudaSuccess ? MP_OK : MP_ECUDA;
}

template <typename T, int D>
static cudaError_t launch_unpermute(const BlockJob& b, int units, void* dk, void* dv, cudaStream_t st) {
  unpermute_kernel<T, D><<<dim3((b.L_blk + 7) / 8, 1, units), 256, 0, st>>>(b, static_cast<T*>(dk), static_cast<T*>(dv));
  return cudaGetLastError();
}

mp_status update_impl(mp_index* idx, const void* K_new, const void* V_new, int32_t n_new, int32_t* fired,
                      cudaStream_t st) {
  const mp_config& c = idx->cfg;
  const int units = c.batch * c.kv_heads;
  const int es = elem_bytes(c.dtype);
  const size_t row_bytes = (size_t)c.head_dim * es;
  const int64_t n0 = idx->n_tokens, nc = idx->n_clustered;
  if (fired) *fired = 0;
  cudaError_t e = cudaSuccess;
  if (n_new > 0) {
    // one launch per append: rows, perm and assign of the new tail
    char* Kp = static_cast<char*>(ws_ptr(idx, S_KP));
    char* Vp = static_cast<char*>(ws_ptr(idx, S_VP));
    int32_t* perm = static_cast<int32_t*>(ws_ptr(idx, S_PERM));
    int32_t* asg = static_cast<int32_t*>(ws_ptr(idx, S_ASSIGN));
    const bool v16 = (((uintptr_t)K_new | (uintptr_t)V_new | (uintptr_t)Kp | (uintptr_t)Vp | row_bytes) & 15u) == 0;
    const size_t words = (size_t)n_new * row_bytes / (v16 ? 16 : 2);
    const int gx = (int)std::min<size_t>(std::max<size_t>((words + 255) / 256, (size_t)(n_new + 255) / 256), 1024);
    const char* kn = static_cast<const char*>(K_new);
    const char* vn = static_cast<const char*>(V_new);
    if (v16)
      append_kernel<uint4><<<dim3(gx, units), 256, 0, st>>>(kn, vn, Kp, Vp, row_bytes, c.max_tokens, n0, n_new, perm, asg);
    else
      append_kernel<uint16_t><<<dim3(gx, units), 256, 0, st>>>(kn, vn, Kp, Vp, row_bytes, c.max_tokens, n0, n_new, perm,
                                                              asg);
    if (cudaGetLastError() != cudaSuccess) return MP_ECUDA;
  }
  const int64_t n1 = n0 + n_new;
  const int64_t Lb = c.block_tokens;
  const bool fire = (n1 - nc >= c.update_interval) || (n1 / Lb > nc / Lb);
  idx->n_tokens = n1;
  if (!fire) return MP_OK;
  void* bk = ws_ptr(idx, S_BLKK);
  void* bv = ws_ptr(idx, S_BLKV);
  for (int64_t j = nc / Lb; j < (n1 + Lb - 1) / Lb; ++j) {
    const int64_t s = j * Lb, eend = std::min(n1, s + Lb);
    const int L_old = (int)std::max<int64_t>(0, std::min(nc, eend) - s);
    BlockJob b = make_job(idx);
    b.srcK = bk; b.srcV = bv;
    b.src_unit_rows = Lb;
    b.src_row0 = 0;
    b.blk0 = (int)j;
    b.n_total = n1;
    if (c.dtype == MP_BF16) e = c.head_dim == 128 ? launch_unpermute<__nv_bfloat16, 128>(b, units, bk, bv, st)
                                                  : launch_unpermute<__nv_bfloat16, 64>(b, units, bk, bv, st);
    else e = c.head_dim == 128 ? launch_unpermute<float, 128>(b, units, bk, bv, st)
                               : launch_unpermute<float, 64>(b, units, bk, bv, st);
    if (e != cudaSuccess) return MP_ECUDA;
    e = dispatch_lloyd(c.dtype, c.head_dim, b, 1, units, MP_INIT_STRIDE, L_old, nullptr, c.levels, st);
    if (e != cudaSuccess) return MP_ECUDA;
  }
  e = fill_tail_offsets(idx, n1, (int)((n1 + Lb - 1) / Lb), st);
  if (e != cudaSuccess) return MP_ECUDA;
  idx->n_clustered = n1;
  if (fired) *fired = 1;
  return MP_OK;
}

}  // namespace mp
