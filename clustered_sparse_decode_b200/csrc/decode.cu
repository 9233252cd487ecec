// Multipole Attention decode step on sm_100a.
//
// "Multipole Attention for Efficient Long Context Reasoning" (arXiv abstract;
// atlas.scime summary, "Approach"): the query scores the key centroids; the
// top clusters up to a token budget are attended exactly; every other cluster
// contributes a count-weighted centroid term with its value centroid; both
// kinds of term share one softmax.
//
// Pipeline per call (every kernel works on all (batch, KV head) units):
//   1. pass     centroid rows (all clusters): group scores for the selection
//               and one online-softmax partial over ALL centroid terms;
//   2. select   budgeted top clusters -> run list of their tokens (+ tail),
//               and the list of selected centroid rows;
//   3. pass     exact terms over the gathered token runs, MINUS the centroid
//               terms of the selected clusters (so the centroid partial of
//               step 1 keeps only the unselected clusters);
//   4. combine  log-sum-exp merge of all partials, cast to the output dtype.
// The two-level variant runs pass/select once more at the coarse level.
//
// Every HBM byte of the method is read once: centroid keys AND values stream
// in step 1 before the selection is known (the subtraction in step 3 only
// re-reads the ~5% selected centroid rows), so the large sequential stream is
// not serialised behind the selection.  Subtracting is safe in fp32: each
// selected centroid term n*e^{q.Kc} is at most the exact mass of its cluster
// (Jensen, Kc being the member mean), so the cancellation error is a few fp32
// ulps of the final normaliser.
#include <algorithm>
#include <cstdio>
#include <cstring>

#include "mp_internal.cuh"

namespace mp {

// ----------------------------------------------------------------------------
// Run lists in the decode scratch
// ----------------------------------------------------------------------------
// A run list enumerates rows of a row array (centroid slots or store rows) as
// runs [start, start + len).  Per unit: hdr[0] = number of runs, hdr[1] = total
// rows; start[k]; pref[k] = rows before run k (pref[n_runs] = total).
struct RunList {
  int32_t* hdr;    // [units][2]
  int32_t* start;  // [units][cap]
  int32_t* pref;   // [units][cap + 1]
  int cap;
};

// Row kinds: where the bias (log2 of the cluster size) of a row comes from.
enum RowKind { ROW_TOKEN = 0, ROW_FINE = 1, ROW_COARSE = 2 };

struct PassList {
  const void* K;       // row array (Kp, Kc or Kcc), [units][unit_rows][D]
  const void* V;
  int64_t unit_rows;
  int kind;            // RowKind
  float sign;          // +1 add, -1 subtract
  int accumulate;      // 0: scores only (no softmax contribution)
  int implicit_n;      // > 0: the list is the single run [0, implicit_n)
  RunList rl;          // used when implicit_n == 0
  float* shat;         // optional: group score by list position, [units][shat_cap]
  int shat_cap;
};

struct PassArgs {
  PassList list[2];
  int n_lists;
  const void* Q;       // [B][H*G][D]
  const int32_t* off;  // [units][slots + 1]
  const int32_t* coff; // [units][coarse_slots + 1]
  int slots, coarse_slots;
  int64_t max_tokens;
  float scale;         // score scale (natural units)
  float* part_m;       // [units*G][P]
  float* part_l;
  float* part_acc;     // [units*G][P][D]
  int P, part_base;
  int32_t* err;
};

constexpr int kPassWarps = 8;
constexpr int kPassThreads = kPassWarps * kWarp;
constexpr int kChunk = 512;   // rows whose run mapping is staged in shared memory at a time

__device__ __forceinline__ int find_run(const int32_t* pref, int lo, int hi, int r) {
  // largest k in [lo, hi] with pref[k] <= r
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (__ldg(pref + mid) <= r) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ int row_count(int kind, const int32_t* off_u, const int32_t* coff_u, int row) {
  if (kind == ROW_FINE) return __ldg(off_u + row + 1) - __ldg(off_u + row);
  return __ldg(off_u + __ldg(coff_u + row + 1)) - __ldg(off_u + __ldg(coff_u + row));
}

// One pass over up to two row lists for every unit.  grid = (n_split, units).
// Each CTA takes the same fraction of every list; each warp consumes batches
// of R = 32/G rows: one lane slice of D/32 elements per row, the G dot
// products of a row reduced across the warp by one 31-shuffle butterfly that
// leaves (row = lane / G, head = lane % G) in each lane.
template <typename T, int D, int G>
__global__ void __launch_bounds__(kPassThreads)
pass_kernel(PassArgs a) {
  constexpr int DPL = D / kWarp;
  constexpr int R = kWarp / G;
  const int unit = blockIdx.y;
  const int split = blockIdx.x;
  const int nsplit = gridDim.x;
  const int warp = threadIdx.x / kWarp;
  const int lane = threadIdx.x % kWarp;
  const int Hq_unit = G;  // query heads of this unit

  __shared__ int s_phys[kChunk];
  __shared__ float s_bias[kChunk];
  __shared__ float s_p[kPassWarps][kWarp];
  __shared__ float s_m[kPassWarps][G];
  __shared__ float s_l[kPassWarps][G];
  __shared__ float s_acc[kPassWarps][G][D];

  // query slice of this lane, fp32
  const T* Q = reinterpret_cast<const T*>(a.Q) + (size_t)unit * Hq_unit * D;
  float q[G][DPL];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < DPL; ++e) q[g][e] = to_f32(Q[g * D + lane * DPL + e]);

  const float zscale = a.scale * kLog2e;   // logits in log2 units
  float m[G], l[G], acc[G][DPL];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY; l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[g][e] = 0.f;
  }
  const int32_t* off_u = a.off + (size_t)unit * (a.slots + 1);
  const int32_t* coff_u = a.coff ? a.coff + (size_t)unit * (a.coarse_slots + 1) : nullptr;

  for (int li = 0; li < a.n_lists; ++li) {
    const PassList& L = a.list[li];
    int total, nruns = 1;
    const int32_t *start = nullptr, *pref = nullptr;
    if (L.implicit_n > 0) {
      total = L.implicit_n;
    } else {
      nruns = L.rl.hdr[unit * 2 + 0];
      total = L.rl.hdr[unit * 2 + 1];
      start = L.rl.start + (size_t)unit * L.rl.cap;
      pref = L.rl.pref + (size_t)unit * (L.rl.cap + 1);
      if (nruns < 0 || nruns > L.rl.cap || total < 0) { set_error(a.err, E_BAD_LIST); total = 0; }
      if (nruns <= 0) total = 0;
    }
    if (L.shat && total > L.shat_cap) { set_error(a.err, E_BAD_LIST); total = L.shat_cap; }
    const int per = (total + nsplit - 1) / nsplit;
    const int r0 = min(total, split * per), r1 = min(total, r0 + per);
    const T* Kb = reinterpret_cast<const T*>(L.K) + (size_t)unit * L.unit_rows * D;
    const T* Vb = reinterpret_cast<const T*>(L.V) + (size_t)unit * L.unit_rows * D;
    const float sign = L.sign;
    const bool accum = L.accumulate != 0;

    for (int c0 = r0; c0 < r1; c0 += kChunk) {
      const int c1 = min(r1, c0 + kChunk);
      // stage the row map of [c0, c1): physical row and log2 weight
      int k0 = 0;
      if (L.implicit_n == 0) k0 = find_run(pref, 0, nruns - 1, c0);
      for (int r = c0 + threadIdx.x; r < c1; r += blockDim.x) {
        int phys;
        if (L.implicit_n > 0) {
          phys = r;
        } else {
          int k = find_run(pref, k0, min(nruns - 1, k0 + (r - c0)), r);
          phys = __ldg(start + k) + (r - __ldg(pref + k));
        }
        float bias = 0.f;
        if (phys < 0 || phys >= L.unit_rows) {
          set_error(a.err, E_BAD_OFFSET);
          phys = 0; bias = -INFINITY;
        } else if (L.kind != ROW_TOKEN) {
          int cnt = row_count(L.kind, off_u, coff_u, phys);
          bias = cnt > 0 ? log2f((float)cnt) : -INFINITY;
        }
        s_phys[r - c0] = phys;
        s_bias[r - c0] = bias;
      }
      __syncthreads();

      for (int bs = c0 + warp * R; bs < c1; bs += kPassWarps * R) {
        // loads: K and V slices of R rows (rows past c1 or with -inf weight: zeros)
        RowChunk<T, DPL> kr[R], vr[R];
        bool valid[R];
#pragma unroll
        for (int i = 0; i < R; ++i) {
          int r = bs + i;
          valid[i] = r < c1 && s_bias[min(r, c1 - 1) - c0] != -INFINITY;
          if (valid[i]) {
            size_t row = (size_t)s_phys[r - c0] * D + lane * DPL;
            kr[i].load(Kb + row);
            if (accum) vr[i].load(Vb + row); else vr[i].zero();
          } else {
            kr[i].zero(); vr[i].zero();
          }
        }
        // per-lane partial dot products p[i*G + g]
        float p[kWarp];
#pragma unroll
        for (int i = 0; i < R; ++i)
#pragma unroll
          for (int g = 0; g < G; ++g) {
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < DPL; ++e) s = fmaf(q[g][e], kr[i].get(e), s);
            p[i * G + g] = s;
          }
        // butterfly: lane ends with the full sum of entry j = lane
#pragma unroll
        for (int w = 16; w >= 1; w >>= 1) {
          const bool upper = (lane & w) != 0;
#pragma unroll
          for (int i = 0; i < w; ++i) {
            float send = upper ? p[i] : p[i + w];
            float keep = upper ? p[i + w] : p[i];
            p[i] = keep + __shfl_xor_sync(kFull, send, w);
          }
        }
        const int my_row = lane / G, my_g = lane % G;
        const int rr = bs + my_row;
        const bool my_valid = rr < c1 && s_bias[min(rr, c1 - 1) - c0] != -INFINITY;
        const float dot = p[0];
        if (L.shat) {
          float zn = dot * a.scale;
#pragma unroll
          for (int o = 1; o < G; o <<= 1) zn = fmaxf(zn, __shfl_xor_sync(kFull, zn, o));
          if (my_g == 0 && rr < c1)
            L.shat[(size_t)unit * L.shat_cap + rr] = my_valid ? zn : -INFINITY;
        }
        if (!accum) continue;
        float z = my_valid ? fmaf(dot, zscale, s_bias[rr - c0]) : -INFINITY;
        // batch max per head, broadcast to all lanes
        float mb = z;
#pragma unroll
        for (int o = G; o < kWarp; o <<= 1) mb = fmaxf(mb, __shfl_xor_sync(kFull, mb, o));
        float mnew[G];
#pragma unroll
        for (int g = 0; g < G; ++g) mnew[g] = fmaxf(m[g], __shfl_sync(kFull, mb, g));
        float pe = (z == -INFINITY) ? 0.f : sign * exp2f(z - mnew[my_g]);
        float lb = pe;
#pragma unroll
        for (int o = G; o < kWarp; o <<= 1) lb += __shfl_xor_sync(kFull, lb, o);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float alpha = (m[g] == mnew[g]) ? 1.f : exp2f(m[g] - mnew[g]);
          l[g] = fmaf(l[g], alpha, __shfl_sync(kFull, lb, g));
#pragma unroll
          for (int e = 0; e < DPL; ++e) acc[g][e] *= alpha;
          m[g] = mnew[g];
        }
        s_p[warp][lane] = pe;
        __syncwarp();
#pragma unroll
        for (int i = 0; i < R; ++i)
#pragma unroll
          for (int g = 0; g < G; ++g) {
            float w = s_p[warp][i * G + g];
#pragma unroll
            for (int e = 0; e < DPL; ++e) acc[g][e] = fmaf(w, vr[i].get(e), acc[g][e]);
          }
        __syncwarp();
      }
      __syncthreads();
    }
  }

  // merge the warps' states and write this CTA's partial
  if (lane < G) { s_m[warp][lane] = m[lane]; s_l[warp][lane] = l[lane]; }
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < DPL; ++e) s_acc[warp][g][lane * DPL + e] = acc[g][e];
  // lanes >= G also hold m and l replicated; lanes < G wrote them above
  __syncthreads();
  const int pidx = a.part_base + split;
  for (int t = threadIdx.x; t < G * D; t += blockDim.x) {
    const int g = t / D, dim = t % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kPassWarps; ++w) M = fmaxf(M, s_m[w][g]);
    float Lsum = 0.f, A = 0.f;
#pragma unroll
    for (int w = 0; w < kPassWarps; ++w) {
      float f = (s_m[w][g] == -INFINITY) ? 0.f : exp2f(s_m[w][g] - M);
      Lsum = fmaf(s_l[w][g], f, Lsum);
      A = fmaf(s_acc[w][g][dim], f, A);
    }
    const size_t row = (size_t)unit * G + g;
    a.part_acc[(row * a.P + pidx) * D + dim] = A;
    if (dim == 0) { a.part_m[row * a.P + pidx] = M; a.part_l[row * a.P + pidx] = Lsum; }
  }
}

// ----------------------------------------------------------------------------
// Budgeted selection
// ----------------------------------------------------------------------------
struct SelectArgs {
  int implicit_n;        // candidates: [0, implicit_n) or the run list `cand`
  RunList cand;
  const float* shat;     // group scores by candidate position, [units][shat_cap]
  int shat_cap;
  int kind;              // ROW_FINE (clusters -> token runs) or ROW_COARSE (coarse -> fine slot runs)
  const int32_t* off;
  const int32_t* coff;
  int slots, coarse_slots;
  int budget;
  RunList next;          // selected runs (+ tail run when tail_len > 0)
  int tail_start, tail_len;
  RunList sub;           // selected candidate rows as runs of length 1 (optional: hdr == nullptr)
  uint8_t* mask_out;     // optional [units][mask_stride]
  int mask_stride;
  float* scores_out;     // optional [units][mask_stride]: group score by candidate row
  int32_t* err;
};

constexpr int kSelThreads = 512;

template <int NT>
__device__ __forceinline__ int block_excl_scan(int v, int* s_warp, int* total) {
  // exclusive prefix of v over the CTA (thread order); *total = sum
  const int lane = threadIdx.x % kWarp, warp = threadIdx.x / kWarp;
  int x = v;
#pragma unroll
  for (int o = 1; o < kWarp; o <<= 1) {
    int y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  if (lane == kWarp - 1) s_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < NT / kWarp ? s_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < kWarp; o <<= 1) {
      int y = __shfl_up_sync(kFull, w, o);
      if (lane >= o) w += y;
    }
    if (lane < NT / kWarp) s_warp[lane] = w;   // inclusive over warps
  }
  __syncthreads();
  int before = (warp > 0 ? s_warp[warp - 1] : 0) + x - v;
  *total = s_warp[NT / kWarp - 1];
  __syncthreads();
  return before;
}

// One CTA per unit.  Ranks candidates by (group score desc, row asc) and takes
// the shortest prefix whose token count reaches the budget (crossing cluster
// whole; everything if the candidates hold <= budget tokens).  The threshold
// is found by a token-weighted radix select over order-preserving 32-bit keys
// (4 passes of 8 bits), equal keys are then ranked by row.
__global__ void __launch_bounds__(kSelThreads)
select_kernel(SelectArgs a) {
  extern __shared__ uint32_t s_dyn[];
  const int unit = blockIdx.x;
  const int tid = threadIdx.x;
  __shared__ int s_hist[256];
  __shared__ int s_warp[kSelThreads / kWarp];
  __shared__ int s_bcast[4];

  const int32_t* off_u = a.off + (size_t)unit * (a.slots + 1);
  const int32_t* coff_u = a.coff ? a.coff + (size_t)unit * (a.coarse_slots + 1) : nullptr;
  int n, nruns = 1;
  const int32_t *cstart = nullptr, *cpref = nullptr;
  if (a.implicit_n > 0) {
    n = a.implicit_n;
  } else {
    nruns = a.cand.hdr[unit * 2 + 0];
    n = a.cand.hdr[unit * 2 + 1];
    cstart = a.cand.start + (size_t)unit * a.cand.cap;
    cpref = a.cand.pref + (size_t)unit * (a.cand.cap + 1);
    if (nruns < 0 || nruns > a.cand.cap || n < 0 || n > a.shat_cap) {
      set_error(a.err, E_BAD_LIST); n = 0; nruns = 0;
    }
  }
  const int maxrow = a.kind == ROW_FINE ? a.slots : a.coarse_slots;
  uint32_t* s_key = s_dyn;                                   // [n]
  int* s_cnt = reinterpret_cast<int*>(s_dyn + a.shat_cap);   // [n], 0 = not a candidate
  int* s_row = s_cnt + a.shat_cap;                           // [n]

  // 1. candidates: row, count, key
  int my_total = 0;
  for (int pos = tid; pos < n; pos += kSelThreads) {
    int row;
    if (a.implicit_n > 0) {
      row = pos;
    } else {
      int k = find_run(cpref, 0, nruns - 1, pos);
      row = __ldg(cstart + k) + (pos - __ldg(cpref + k));
    }
    int cnt = 0;
    if (row < 0 || row >= maxrow) { set_error(a.err, E_BAD_OFFSET); row = 0; }
    else cnt = row_count(a.kind, off_u, coff_u, row);
    float sc = a.shat[(size_t)unit * a.shat_cap + pos];
    if (!(sc > -INFINITY)) cnt = 0;                          // -inf or NaN: not a candidate
    if (cnt < 0) { set_error(a.err, E_BAD_OFFSET); cnt = 0; }
    s_row[pos] = row;
    s_cnt[pos] = cnt;
    s_key[pos] = ordered_key(sc);
    my_total += cnt;
    if (a.scores_out) a.scores_out[(size_t)unit * a.mask_stride + row] = cnt > 0 ? sc : -INFINITY;
  }
  int total;
  block_excl_scan<kSelThreads>(my_total, s_warp, &total);

  // 2. threshold (key, row) of the crossing cluster
  const int need = a.budget;
  uint32_t thr_key = 0;
  int thr_pos = -1;   // selected: key > thr_key, or key == thr_key and pos <= thr_pos
  int mode;           // 0 none, 1 all, 2 threshold
  if (need <= 0) mode = 0;
  else if (total <= need) mode = 1;
  else mode = 2;
  bool resolved = false;
  if (mode == 2) {
    // First try: 256 bins of equal score width between the smallest and the
    // largest candidate score (monotone in the score, so the bin where the
    // weight from the top crosses the budget holds the crossing cluster); if
    // at most 32 candidates fall in it, one warp sorts them by (key
    // descending, position ascending) and the crossing one gives (thr_key,
    // thr_pos).  Otherwise the radix descent below decides.
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    for (int pos = tid; pos < n; pos += kSelThreads)
      if (s_cnt[pos] > 0) { kmin = min(kmin, s_key[pos]); kmax = max(kmax, s_key[pos]); }
    kmin = __reduce_min_sync(kFull, kmin);
    kmax = __reduce_max_sync(kFull, kmax);
    if (tid % kWarp == 0) { s_warp[tid / kWarp] = (int)kmin; s_hist[tid / kWarp] = (int)kmax; }
    __syncthreads();
    kmin = 0xffffffffu; kmax = 0u;
    for (int w = 0; w < kSelThreads / kWarp; ++w) {
      kmin = min(kmin, (uint32_t)s_warp[w]);
      kmax = max(kmax, (uint32_t)s_hist[w]);
    }
    __syncthreads();
    const float smin = key_score(kmin), smax = key_score(kmax);
    const float span = smax - smin, inv = 256.f / span;
    if (isfinite(smin) && isfinite(smax) && span > 0.f && isfinite(span) && isfinite(inv)) {
      auto fbin = [&](uint32_t k) { return min(255, (int)((key_score(k) - smin) * inv)); };
      if (tid < 256) s_hist[tid] = 0;
      if (tid == 0) s_bcast[3] = 0;
      __syncthreads();
      for (int pos = tid; pos < n; pos += kSelThreads)
        if (s_cnt[pos] > 0) atomicAdd(&s_hist[fbin(s_key[pos])], s_cnt[pos]);
      __syncthreads();
      int v = tid < 256 ? s_hist[255 - tid] : 0;
      int tot;
      int before = block_excl_scan<kSelThreads>(v, s_warp, &tot);
      if (tid < 256 && before < need && before + v >= need) {
        s_bcast[0] = 255 - tid;
        s_bcast[1] = before;
      }
      __syncthreads();
      const int fb = s_bcast[0], ab = s_bcast[1];
      int* lst = s_hist;                                   // [32][3]: the histogram is no longer needed
      __syncthreads();
      for (int pos = tid; pos < n; pos += kSelThreads)
        if (s_cnt[pos] > 0 && fbin(s_key[pos]) == fb) {
          const int q = atomicAdd(&s_bcast[3], 1);
          if (q < 32) { lst[3 * q] = (int)s_key[pos]; lst[3 * q + 1] = pos; lst[3 * q + 2] = s_cnt[pos]; }
        }
      __syncthreads();
      const int nc = s_bcast[3];
      if (nc <= 32) {
        if (tid < kWarp) {
          const int lane = tid;
          uint64_t key = lane < nc ? ((uint64_t)(uint32_t)lst[3 * lane] << 32) |
                                         (uint32_t)(0xffffffffu - (uint32_t)lst[3 * lane + 1])
                                   : 0ull;
          int wl = lane < nc ? lst[3 * lane + 2] : 0;
#pragma unroll
          for (int kk = 2; kk <= 32; kk <<= 1) {
#pragma unroll
            for (int jj = kk >> 1; jj > 0; jj >>= 1) {
              const uint64_t ok = __shfl_xor_sync(kFull, key, jj);
              const int ow = __shfl_xor_sync(kFull, wl, jj);
              const bool up = ((lane & kk) == 0) == ((lane & jj) == 0);   // this lane keeps the larger
              if (up ? ok > key : ok < key) { key = ok; wl = ow; }
            }
          }
          int inc = wl;
#pragma unroll
          for (int o = 1; o < kWarp; o <<= 1) {
            const int y = __shfl_up_sync(kFull, inc, o);
            if (lane >= o) inc += y;
          }
          const unsigned cross = __ballot_sync(kFull, lane < nc && ab + inc >= need);
          const uint64_t ck = __shfl_sync(kFull, key, __ffs(cross) - 1);
          if (lane == 0) {
            s_bcast[0] = (int)(uint32_t)(ck >> 32);
            s_bcast[2] = (int)(0xffffffffu - (uint32_t)ck);
          }
        }
        __syncthreads();
        thr_key = (uint32_t)s_bcast[0];
        thr_pos = s_bcast[2];
        resolved = true;
      }
      __syncthreads();
    }
  }
  if (mode == 2 && !resolved) {
    uint32_t prefix = 0, mask = 0;
    int committed = 0;
    for (int shift = 24; shift >= 0; shift -= 8) {
      if (tid < 256) s_hist[tid] = 0;
      __syncthreads();
      for (int pos = tid; pos < n; pos += kSelThreads) {
        int c = s_cnt[pos];
        uint32_t k = s_key[pos];
        if (c > 0 && (k & mask) == prefix) atomicAdd(&s_hist[(k >> shift) & 255u], c);
      }
      __syncthreads();
      // cumulative weight from the top bin down
      int v = tid < 256 ? s_hist[255 - tid] : 0;
      int tot;
      int before = block_excl_scan<kSelThreads>(v, s_warp, &tot);
      if (tid < 256 && committed + before < need && committed + before + v >= need) {
        s_bcast[0] = 255 - tid;
        s_bcast[1] = before;
      }
      __syncthreads();
      const int bin = s_bcast[0];
      committed += s_bcast[1];
      prefix |= (uint32_t)bin << shift;
      mask |= 255u << shift;
      __syncthreads();
    }
    thr_key = prefix;
    // equal keys, ranked by position (= ascending row)
    const int per = (n + kSelThreads - 1) / kSelThreads;
    const int p0 = min(n, tid * per), p1 = min(n, p0 + per);
    int mine = 0;
    for (int pos = p0; pos < p1; ++pos)
      if (s_cnt[pos] > 0 && s_key[pos] == thr_key) mine += s_cnt[pos];
    int tot;
    int before = block_excl_scan<kSelThreads>(mine, s_warp, &tot);
    if (tid == 0) s_bcast[2] = n;   // fallback (cannot happen with total > need)
    __syncthreads();
    int run = committed + before;
    for (int pos = p0; pos < p1; ++pos) {
      if (s_cnt[pos] > 0 && s_key[pos] == thr_key) {
        if (run < need && run + s_cnt[pos] >= need) s_bcast[2] = pos;
        run += s_cnt[pos];
      }
    }
    __syncthreads();
    thr_pos = s_bcast[2];
  }

  // 3. compaction in candidate order: selected runs, then the tail run
  const int per = (n + kSelThreads - 1) / kSelThreads;
  const int p0 = min(n, tid * per), p1 = min(n, p0 + per);
  auto is_sel = [&](int pos) -> bool {
    int c = s_cnt[pos];
    if (c <= 0 || mode == 0) return false;
    if (mode == 1) return true;
    uint32_t k = s_key[pos];
    return k > thr_key || (k == thr_key && pos <= thr_pos);
  };
  auto run_len = [&](int pos) -> int {
    if (a.kind == ROW_FINE) return s_cnt[pos];
    int r = s_row[pos];
    return __ldg(coff_u + r + 1) - __ldg(coff_u + r);
  };
  auto run_start = [&](int pos) -> int {
    int r = s_row[pos];
    return a.kind == ROW_FINE ? __ldg(off_u + r) : __ldg(coff_u + r);
  };
  int nsel_mine = 0, len_mine = 0;
  for (int pos = p0; pos < p1; ++pos)
    if (is_sel(pos)) { nsel_mine++; len_mine += run_len(pos); }
  int nsel_tot, len_tot;
  int k_before = block_excl_scan<kSelThreads>(nsel_mine, s_warp, &nsel_tot);
  int r_before = block_excl_scan<kSelThreads>(len_mine, s_warp, &len_tot);
  const int has_tail = a.tail_len > 0 ? 1 : 0;
  if (nsel_tot + has_tail > a.next.cap) {      // cannot happen for a valid index
    if (tid == 0) { set_error(a.err, E_CAPACITY); a.next.hdr[unit * 2] = 0; a.next.hdr[unit * 2 + 1] = 0; }
    if (a.sub.hdr && tid == 0) { a.sub.hdr[unit * 2] = 0; a.sub.hdr[unit * 2 + 1] = 0; }
    return;
  }
  int32_t* nst = a.next.start + (size_t)unit * a.next.cap;
  int32_t* npf = a.next.pref + (size_t)unit * (a.next.cap + 1);
  int32_t* sst = a.sub.hdr ? a.sub.start + (size_t)unit * a.sub.cap : nullptr;
  int32_t* spf = a.sub.hdr ? a.sub.pref + (size_t)unit * (a.sub.cap + 1) : nullptr;
  int k = k_before, rsum = r_before;
  for (int pos = p0; pos < p1; ++pos) {
    if (!is_sel(pos)) continue;
    nst[k] = run_start(pos);
    npf[k] = rsum;
    if (sst) { sst[k] = s_row[pos]; spf[k] = k; }
    if (a.mask_out) a.mask_out[(size_t)unit * a.mask_stride + s_row[pos]] = 1;
    rsum += run_len(pos);
    k++;
  }
  if (tid == 0) {
    if (has_tail) { nst[nsel_tot] = a.tail_start; npf[nsel_tot] = len_tot; }
    npf[nsel_tot + has_tail] = len_tot + (has_tail ? a.tail_len : 0);
    a.next.hdr[unit * 2 + 0] = nsel_tot + has_tail;
    a.next.hdr[unit * 2 + 1] = len_tot + (has_tail ? a.tail_len : 0);
    if (sst) {
      spf[nsel_tot] = nsel_tot;
      a.sub.hdr[unit * 2 + 0] = nsel_tot;
      a.sub.hdr[unit * 2 + 1] = nsel_tot;
    }
  }
}

// ----------------------------------------------------------------------------
// Combine
// ----------------------------------------------------------------------------
// P: partial stride of the layout; n_used: partials written by this call.
constexpr int kCombThreads = 512;
constexpr int kCombMaxParts = 128;   // >= the largest P: 32 centroid + 32 fine + 64 token splits

// One CTA per output row.  The partials' maxima and normalisers are read once
// into shared memory (one thread per partial); every partial's weight
// exp2(m_p - M) is computed there; then kCombThreads / D thread groups each
// sum a strided share of the partials' accumulators for every column, with
// independent loads, and the groups' sums are added in shared memory.
template <typename T, int D>
__global__ void __launch_bounds__(kCombThreads)
combine_kernel(const float* part_m, const float* part_l, const float* part_acc, int P,
                               int n_used, T* O) {
  constexpr int NG = kCombThreads / D;      // partial groups
  __shared__ float s_f[kCombMaxParts];
  __shared__ float s_red[kCombThreads / kWarp];
  __shared__ float s_acc[NG][D];
  const int row = blockIdx.x;   // unit * G + g == b * Hq + hq
  const int tid = threadIdx.x, lane = tid % kWarp, warp = tid / kWarp;
  const float* pm = part_m + (size_t)row * P;
  const float* pl = part_l + (size_t)row * P;
  const int n = min(n_used, kCombMaxParts);
  // 1. M = max over partials
  const float mp = tid < n ? pm[tid] : -INFINITY;
  float x = mp;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) x = fmaxf(x, __shfl_xor_sync(kFull, x, o));
  if (lane == 0) s_red[warp] = x;
  __syncthreads();
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < kCombThreads / kWarp; ++w) M = fmaxf(M, s_red[w]);
  __syncthreads();
  // 2. weights and the normaliser
  const float f = (tid < n && mp != -INFINITY) ? exp2f(mp - M) : 0.f;
  if (tid < n) s_f[tid] = f;
  float l = tid < n ? f * pl[tid] : 0.f;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) l += __shfl_xor_sync(kFull, l, o);
  if (lane == 0) s_red[warp] = l;
  __syncthreads();
  float Ls = 0.f;
#pragma unroll
  for (int w = 0; w < kCombThreads / kWarp; ++w) Ls += s_red[w];
  // 3. accumulators: group g sums partials g, g + NG, ...
  const int g = tid / D, dim = tid % D;
  const float* pa = part_acc + (size_t)row * P * D + dim;
  float A = 0.f;
#pragma unroll 4
  for (int p = g; p < n; p += NG) A = fmaf(pa[(size_t)p * D], s_f[p], A);
  s_acc[g][dim] = A;
  __syncthreads();
  if (tid < D) {
    float t = 0.f;
#pragma unroll
    for (int q = 0; q < NG; ++q) t += s_acc[q][tid];
    const float o = (M != -INFINITY && Ls > 0.f) ? t / Ls : 0.f;
    O[(size_t)row * D + tid] = from_f32<T>(o);
  }
}

__global__ void fill_f32(float* p, size_t n, float v) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) p[i] = v;
}

// ----------------------------------------------------------------------------
// Host side
// ----------------------------------------------------------------------------
static inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct DecodeLayout {
  int units, G, D;
  int nsplit_c, nsplit_f, nsplit_t_max, P;
  int cap_tok, cap_fine, cap_sub, cap_csub;
  size_t o_pm, o_pl, o_pa, o_shat, o_shatc;
  size_t o_tok[3], o_fine[3], o_sub[3], o_csub[3];
  size_t bytes;
};

constexpr int kMaxSplit = 64;
constexpr int kRowsPerCta = 256;

static void runlist_alloc(size_t& cur, int units, int cap, size_t o[3]) {
  o[0] = cur; cur = align256(cur + (size_t)units * 2 * 4);
  o[1] = cur; cur = align256(cur + (size_t)units * cap * 4);
  o[2] = cur; cur = align256(cur + (size_t)units * (cap + 1) * 4);
}

static DecodeLayout decode_layout(const mp_config& c, int slots, int coarse_slots) {
  DecodeLayout L{};
  L.units = c.batch * c.kv_heads;
  L.G = c.q_heads / c.kv_heads;
  L.D = c.head_dim;
  const int top = c.levels == 2 ? coarse_slots : slots;
  L.nsplit_c = std::max(1, std::min(32, (top + kRowsPerCta - 1) / kRowsPerCta));
  L.nsplit_f = c.levels == 2 ? 32 : 0;
  L.nsplit_t_max = kMaxSplit;
  L.P = L.nsplit_c + L.nsplit_f + L.nsplit_t_max;
  static_assert(32 + 32 + kMaxSplit <= kCombMaxParts, "combine holds every partial's weight");
  L.cap_tok = slots + 1;
  L.cap_fine = coarse_slots;
  L.cap_sub = slots;
  L.cap_csub = coarse_slots;
  size_t cur = 0;
  const size_t rows = (size_t)L.units * L.G;
  L.o_pm = cur; cur = align256(cur + rows * L.P * 4);
  L.o_pl = cur; cur = align256(cur + rows * L.P * 4);
  L.o_pa = cur; cur = align256(cur + rows * L.P * L.D * 4);
  L.o_shat = cur; cur = align256(cur + (size_t)L.units * slots * 4);
  L.o_shatc = cur; cur = align256(cur + (size_t)L.units * std::max(coarse_slots, 1) * 4);
  runlist_alloc(cur, L.units, L.cap_tok, L.o_tok);
  runlist_alloc(cur, L.units, std::max(L.cap_sub, 1), L.o_sub);
  if (c.levels == 2) {
    runlist_alloc(cur, L.units, L.cap_fine, L.o_fine);
    runlist_alloc(cur, L.units, L.cap_csub, L.o_csub);
  }
  L.bytes = cur;
  return L;
}

size_t unit_scratch_bytes(const mp_config& c, int slots);
bool unit_supported(const mp_config& c, int slots);
mp_status unit_decode(const mp_index* idx, const void* Q, void* O, const mp_decode_params* prm, void* scratch,
                      size_t scratch_bytes, float scale, cudaStream_t st);

// The decode path of an index places its scratch from the start of the
// buffer; after it, room for a device copy of Q when the caller's Q is
// page-locked host memory.
static size_t q_stage_offset(const mp_config& c, int slots, int coarse_slots) {
  if (unit_supported(c, slots)) return align256(unit_scratch_bytes(c, slots));
  return align256(decode_layout(c, slots, coarse_slots).bytes);
}
static size_t q_bytes(const mp_config& c) {
  return (size_t)c.batch * c.q_heads * c.head_dim * elem_bytes(c.dtype);
}
size_t decode_scratch_bytes(const mp_config& c, int slots, int coarse_slots) {
  return q_stage_offset(c, slots, coarse_slots) + align256(q_bytes(c));
}

// Q from page-locked host memory into the device: plain loads over the host link.
template <typename W>
__global__ void stage_q_kernel(const W* __restrict__ src, W* __restrict__ dst, size_t n) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    dst[i] = src[i];
}

// Where Q and O live: device (or managed) memory, or page-locked host memory
// that the device reaches through the unified address space.  Anything else
// (pageable host memory, unknown pointers) is refused.
static mp_status locate(const void* p, bool* host) {
  cudaPointerAttributes at{};
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return MP_EINVAL;
  }
  if (at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged) { *host = false; return MP_OK; }
  if (at.type == cudaMemoryTypeHost && at.devicePointer == p) { *host = true; return MP_OK; }
  return MP_EINVAL;
}

static RunList runlist_at(char* base, const size_t o[3], int cap) {
  RunList r;
  r.hdr = reinterpret_cast<int32_t*>(base + o[0]);
  r.start = reinterpret_cast<int32_t*>(base + o[1]);
  r.pref = reinterpret_cast<int32_t*>(base + o[2]);
  r.cap = cap;
  return r;
}

template <typename T, int D, int G>
static cudaError_t launch_pass(const PassArgs& a, int nsplit, int units, cudaStream_t st) {
  pass_kernel<T, D, G><<<dim3(nsplit, units), kPassThreads, 0, st>>>(a);
  return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t launch_pass_g(int G, const PassArgs& a, int nsplit, int units, cudaStream_t st) {
  switch (G) {
    case 1: return launch_pass<T, D, 1>(a, nsplit, units, st);
    case 2: return launch_pass<T, D, 2>(a, nsplit, units, st);
    case 4: return launch_pass<T, D, 4>(a, nsplit, units, st);
    case 8: return launch_pass<T, D, 8>(a, nsplit, units, st);
  }
  return cudaErrorInvalidValue;
}

static cudaError_t launch_pass_any(int dtype, int D, int G, const PassArgs& a, int nsplit, int units,
                                   cudaStream_t st) {
  if (dtype == MP_BF16) {
    if (D == 128) return launch_pass_g<__nv_bfloat16, 128>(G, a, nsplit, units, st);
    if (D == 64) return launch_pass_g<__nv_bfloat16, 64>(G, a, nsplit, units, st);
  } else {
    if (D == 128) return launch_pass_g<float, 128>(G, a, nsplit, units, st);
    if (D == 64) return launch_pass_g<float, 64>(G, a, nsplit, units, st);
  }
  return cudaErrorInvalidValue;
}

static cudaError_t launch_select(const SelectArgs& a, int units, cudaStream_t st) {
  // the 48 KB default limit covers static plus dynamic shared memory
  static size_t static_smem = [] {
    cudaFuncAttributes fa{};
    return cudaFuncGetAttributes(&fa, select_kernel) == cudaSuccess ? fa.sharedSizeBytes : (size_t)4096;
  }();
  size_t smem = (size_t)a.shat_cap * 12;
  if (smem + static_smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  select_kernel<<<units, kSelThreads, smem, st>>>(a);
  return cudaGetLastError();
}

static cudaError_t launch_combine(int dtype, int D, const float* pm, const float* pl, const float* pa, int P,
                                  int n_used, void* O, int rows, cudaStream_t st) {
  if (n_used > kCombMaxParts) return cudaErrorInvalidValue;
  if (dtype == MP_BF16) {
    if (D == 128) combine_kernel<__nv_bfloat16, 128><<<rows, kCombThreads, 0, st>>>(pm, pl, pa, P, n_used, (__nv_bfloat16*)O);
    else combine_kernel<__nv_bfloat16, 64><<<rows, kCombThreads, 0, st>>>(pm, pl, pa, P, n_used, (__nv_bfloat16*)O);
  } else {
    if (D == 128) combine_kernel<float, 128><<<rows, kCombThreads, 0, st>>>(pm, pl, pa, P, n_used, (float*)O);
    else combine_kernel<float, 64><<<rows, kCombThreads, 0, st>>>(pm, pl, pa, P, n_used, (float*)O);
  }
  return cudaGetLastError();
}

static void record_phase(const mp_decode_params* prm, int i, cudaStream_t st) {
  if (i < prm->n_phase_events && prm->phase_events[i])
    cudaEventRecord(static_cast<cudaEvent_t>(prm->phase_events[i]), st);
}

static mp_status decode_paths(const mp_index* idx, const void* Q, void* O, const mp_decode_params* prm,
                              void* scratch, size_t scratch_bytes, cudaStream_t st);

// Names of the intervals between the phase events of a decode of this index.
const char* decode_phase_names(const mp_index* idx) {
  const mp_config& c = idx->cfg;
  if (unit_supported(c, idx->slots)) return "decode";
  if (c.levels == 1) return "centroid pass|select|token pass|combine";
  return "coarse pass|coarse select|fine pass|fine select|token pass|combine";
}

mp_status decode_impl(const mp_index* idx, const void* Q, void* O, const mp_decode_params* prm,
                      void* scratch, size_t scratch_bytes, cudaStream_t st) {
  const mp_config& c = idx->cfg;
  bool q_host = false, o_host = false;
  if (locate(Q, &q_host) != MP_OK || locate(O, &o_host) != MP_OK) return MP_EINVAL;
  (void)o_host;   // the output is written in place either way (stores over the host link for host memory)
  if (q_host) {
    const size_t off = q_stage_offset(c, idx->slots, idx->coarse_slots), nb = q_bytes(c);
    if (scratch_bytes < off + nb) return MP_ENOSPC;
    void* qd = static_cast<char*>(scratch) + off;
    if (((uintptr_t)Q & 15u) == 0) {
      const size_t n = nb / 16;
      stage_q_kernel<uint4><<<(unsigned)std::min<size_t>((n + 255) / 256, 256), 256, 0, st>>>(
          static_cast<const uint4*>(Q), static_cast<uint4*>(qd), n);
    } else {
      const size_t n = nb / 2;
      stage_q_kernel<uint16_t><<<(unsigned)std::min<size_t>((n + 255) / 256, 256), 256, 0, st>>>(
          static_cast<const uint16_t*>(Q), static_cast<uint16_t*>(qd), n);
    }
    if (cudaGetLastError() != cudaSuccess) return MP_ECUDA;
    Q = qd;
  }
  return decode_paths(idx, Q, O, prm, scratch, scratch_bytes, st);
}

static mp_status decode_paths(const mp_index* idx, const void* Q, void* O, const mp_decode_params* prm,
                              void* scratch, size_t scratch_bytes, cudaStream_t st) {
  const mp_config& c = idx->cfg;
  // flat bf16 index: one kernel, one CTA (or CTA cluster) per unit (decode_unit.cu)
  if (unit_supported(c, idx->slots)) {
    const float sc = prm->scale != 0.f ? prm->scale : 1.0f / sqrtf((float)c.head_dim);
    return unit_decode(idx, Q, O, prm, scratch, scratch_bytes, sc, st);
  }
  DecodeLayout L = decode_layout(c, idx->slots, idx->coarse_slots);
  if (scratch_bytes < L.bytes) return MP_ENOSPC;
  char* base = static_cast<char*>(scratch);
  const int units = L.units, G = L.G, D = L.D;
  const int es = elem_bytes(c.dtype);
  const bool approx = (prm->flags & MP_NO_APPROX) == 0;
  const float scale = prm->scale != 0.f ? prm->scale : 1.0f / sqrtf((float)D);
  float* pm = reinterpret_cast<float*>(base + L.o_pm);
  float* pl = reinterpret_cast<float*>(base + L.o_pl);
  float* pa = reinterpret_cast<float*>(base + L.o_pa);
  float* shat = reinterpret_cast<float*>(base + L.o_shat);
  float* shatc = reinterpret_cast<float*>(base + L.o_shatc);
  RunList tok = runlist_at(base, L.o_tok, L.cap_tok);
  RunList sub = runlist_at(base, L.o_sub, std::max(L.cap_sub, 1));
  const int32_t* off = static_cast<const int32_t*>(ws_ptr(idx, S_OFF));
  const int32_t* coff = c.levels == 2 ? static_cast<const int32_t*>(ws_ptr(idx, S_COFF)) : nullptr;
  int32_t* err = err_word(idx);
  const int64_t n_clu = idx->n_clustered, n_tail = idx->n_tokens - idx->n_clustered;

  cudaError_t ce = cudaSuccess;
  if (prm->sel_mask_out) ce = cudaMemsetAsync(prm->sel_mask_out, 0, (size_t)units * idx->slots, st);
  if (ce == cudaSuccess && c.levels == 2 && prm->coarse_sel_mask_out)
    ce = cudaMemsetAsync(prm->coarse_sel_mask_out, 0, (size_t)units * idx->coarse_slots, st);
  if (ce == cudaSuccess && c.levels == 2 && prm->scores_out) {
    fill_f32<<<256, 256, 0, st>>>(prm->scores_out, (size_t)units * idx->slots, -INFINITY);
    ce = cudaGetLastError();
  }
  if (ce != cudaSuccess) return MP_ECUDA;

  // token-pass split: estimate of the rows it reads
  int64_t est = (int64_t)std::max(prm->budget, 0) + 8LL * c.tokens_per_centroid + n_tail;
  est = std::min<int64_t>(est, idx->n_tokens);
  int nsplit_t = prm->n_split > 0 ? prm->n_split : (int)std::max<int64_t>(1, (est + kRowsPerCta - 1) / kRowsPerCta);
  nsplit_t = std::min(nsplit_t, L.nsplit_t_max);

  PassArgs pa_args{};
  pa_args.Q = Q;
  pa_args.off = off;
  pa_args.coff = coff;
  pa_args.slots = idx->slots;
  pa_args.coarse_slots = idx->coarse_slots;
  pa_args.max_tokens = c.max_tokens;
  pa_args.scale = scale;
  pa_args.part_m = pm; pa_args.part_l = pl; pa_args.part_acc = pa;
  pa_args.P = L.P;
  pa_args.err = err;

  const void* Kc = ws_ptr(idx, S_KC);
  const void* Vc = ws_ptr(idx, S_VC);
  const void* Kp = ws_ptr(idx, S_KP);
  const void* Vp = ws_ptr(idx, S_VP);
  int part_used = 0;

  SelectArgs sa{};
  sa.off = off; sa.coff = coff; sa.slots = idx->slots; sa.coarse_slots = idx->coarse_slots; sa.err = err;

  int ev = 0;
  record_phase(prm, ev++, st);
  if (c.levels == 1) {
    // 1. all centroids
    PassArgs p1 = pa_args;
    p1.n_lists = 1;
    p1.list[0] = PassList{Kc, Vc, idx->slots, ROW_FINE, 1.f, approx ? 1 : 0, idx->slots, RunList{}, shat, idx->slots};
    p1.part_base = part_used;
    ce = launch_pass_any(c.dtype, D, G, p1, L.nsplit_c, units, st);
    part_used += L.nsplit_c;
    if (ce != cudaSuccess) return MP_ECUDA;
    record_phase(prm, ev++, st);
    // 2. select
    sa.implicit_n = idx->slots;
    sa.shat = shat; sa.shat_cap = idx->slots;
    sa.kind = ROW_FINE;
    sa.budget = prm->budget;
    sa.next = tok;
    sa.tail_start = (int)n_clu; sa.tail_len = (int)n_tail;
    sa.sub = approx ? sub : RunList{};
    sa.mask_out = prm->sel_mask_out; sa.mask_stride = idx->slots;
    sa.scores_out = prm->scores_out;
    ce = launch_select(sa, units, st);
    if (ce != cudaSuccess) return MP_ECUDA;
    record_phase(prm, ev++, st);
  } else {
    RunList fine = runlist_at(base, L.o_fine, L.cap_fine);
    RunList csub = runlist_at(base, L.o_csub, L.cap_csub);
    const void* Kcc = ws_ptr(idx, S_KCC);
    const void* Vcc = ws_ptr(idx, S_VCC);
    // 1. coarse centroids
    PassArgs p1 = pa_args;
    p1.n_lists = 1;
    p1.list[0] = PassList{Kcc, Vcc, idx->coarse_slots, ROW_COARSE, 1.f, approx ? 1 : 0, idx->coarse_slots,
                          RunList{}, shatc, idx->coarse_slots};
    p1.part_base = part_used;
    ce = launch_pass_any(c.dtype, D, G, p1, L.nsplit_c, units, st);
    part_used += L.nsplit_c;
    if (ce != cudaSuccess) return MP_ECUDA;
    record_phase(prm, ev++, st);
    // 2. coarse select -> fine candidate ranges
    SelectArgs s1 = sa;
    s1.implicit_n = idx->coarse_slots;
    s1.shat = shatc; s1.shat_cap = idx->coarse_slots;
    s1.kind = ROW_COARSE;
    s1.budget = prm->coarse_budget > 0 ? prm->coarse_budget : 8 * prm->budget;
    s1.next = fine;
    s1.tail_start = 0; s1.tail_len = 0;
    s1.sub = approx ? csub : RunList{};
    s1.mask_out = prm->coarse_sel_mask_out; s1.mask_stride = idx->coarse_slots;
    s1.scores_out = prm->coarse_scores_out;
    ce = launch_select(s1, units, st);
    if (ce != cudaSuccess) return MP_ECUDA;
    record_phase(prm, ev++, st);
    // 3. fine centroids under selected coarse clusters, minus the selected coarse terms
    PassArgs p2 = pa_args;
    p2.n_lists = approx ? 2 : 1;
    p2.list[0] = PassList{Kc, Vc, idx->slots, ROW_FINE, 1.f, approx ? 1 : 0, 0, fine, shat, idx->slots};
    p2.list[1] = PassList{Kcc, Vcc, idx->coarse_slots, ROW_COARSE, -1.f, 1, 0, csub, nullptr, 0};
    p2.part_base = part_used;
    ce = launch_pass_any(c.dtype, D, G, p2, L.nsplit_f, units, st);
    part_used += L.nsplit_f;
    if (ce != cudaSuccess) return MP_ECUDA;
    record_phase(prm, ev++, st);
    // 4. fine select -> token runs
    SelectArgs s2 = sa;
    s2.implicit_n = 0;
    s2.cand = fine;
    s2.shat = shat; s2.shat_cap = idx->slots;
    s2.kind = ROW_FINE;
    s2.budget = prm->budget;
    s2.next = tok;
    s2.tail_start = (int)n_clu; s2.tail_len = (int)n_tail;
    s2.sub = approx ? sub : RunList{};
    s2.mask_out = prm->sel_mask_out; s2.mask_stride = idx->slots;
    s2.scores_out = prm->scores_out;
    ce = launch_select(s2, units, st);
    if (ce != cudaSuccess) return MP_ECUDA;
    record_phase(prm, ev++, st);
  }
  // 5. exact tokens, minus the selected centroid terms
  PassArgs p3 = pa_args;
  p3.n_lists = approx ? 2 : 1;
  p3.list[0] = PassList{Kp, Vp, c.max_tokens, ROW_TOKEN, 1.f, 1, 0, tok, nullptr, 0};
  p3.list[1] = PassList{Kc, Vc, idx->slots, ROW_FINE, -1.f, 1, 0, sub, nullptr, 0};
  p3.part_base = part_used;
  ce = launch_pass_any(c.dtype, D, G, p3, nsplit_t, units, st);
  part_used += nsplit_t;
  if (ce != cudaSuccess) return MP_ECUDA;
  record_phase(prm, ev++, st);
  // 6. combine the partials written by this call
  ce = launch_combine(c.dtype, D, pm, pl, pa, L.P, part_used, O, units * G, st);
  record_phase(prm, ev++, st);
  (void)es;
  return ce == cudaSuccess ? MP_OK : MP_ECUDA;
}

}  // namespace mp
