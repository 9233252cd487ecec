/*
 * mpattn.h -- C ABI of the Multipole Attention decode library (sm_100a).
 *
 * The method ("Multipole Attention for Efficient Long Context Reasoning",
 * arXiv abstract; atlas.scime summary, "Approach"): keys of the KV cache are
 * grouped by k-means into clusters; at each decode step the query scores the
 * key centroids, the top clusters up to a token budget are attended exactly,
 * and every other cluster contributes one count-weighted centroid term with
 * its value centroid.  Clustering is blockwise and is refreshed online as
 * generated tokens arrive.
 *
 * Conventions for every entry point
 *  - All tensor arguments are DEVICE pointers on the current CUDA device,
 *    contiguous, row-major, in the index dtype (MP_F32: float, MP_BF16:
 *    bfloat16) unless stated otherwise.  Shapes use
 *      B  = batch, H = kv_heads, Hq = q_heads (Hq % H == 0, G = Hq / H;
 *           query head g belongs to KV head g / G),
 *      d  = head_dim (64 or 128).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  All device work is enqueued on it; no call synchronises the
 *    host except mp_check_device_error.
 *  - The library never allocates device memory.  The caller allocates the
 *    index workspace and the decode scratch (sizes from mp_workspace_size)
 *    and owns every buffer.  Inputs passed to a call must stay alive until the
 *    stream has executed the work of that call.
 *  - Arguments are validated on the host before anything is launched;
 *    invalid ones return MP_EINVAL (or MP_ENOSPC when a capacity would be
 *    exceeded) and leave the index unchanged.  A launch failure returns
 *    MP_ECUDA.  Kernels never trap: a data-dependent fault found on the device
 *    (e.g. corrupt offsets in an imported index) sets a device error word and
 *    skips the faulty access; mp_check_device_error reports it.  Its bits:
 *    1 a run offset or slot outside the index, 2 an inconsistent internal run
 *    list, 4 a bounded wait gave up, 8 a per-unit kernel limit exceeded.
 *  - An index is not thread-safe: one host thread, one stream at a time.
 */
#ifndef MPATTN_H
#define MPATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MP_OK = 0,
  MP_EINVAL = 1,         /* invalid argument or configuration */
  MP_ENOSPC = 2,         /* token capacity (max_tokens) or a buffer size exceeded */
  MP_ECUDA = 3,          /* a CUDA call or kernel launch failed */
  MP_EUNSUPPORTED = 4,   /* valid but not implemented (e.g. head_dim 96) */
  MP_EDEVICE = 5         /* the device error word was set (see mp_check_device_error) */
} mp_status;

typedef enum { MP_F32 = 0, MP_BF16 = 1 } mp_dtype;

/* Initial centroids of a from-scratch build. */
typedef enum {
  MP_INIT_KMEANSPP = 0,  /* seeded k-means++ (D^2 sampling) per block */
  MP_INIT_STRIDE = 1     /* slot k of a block starts at the key of the block's token k*T */
} mp_init;

/* Decode flags. */
#define MP_NO_APPROX 1u  /* drop the centroid terms of unselected clusters: exact attention
                            over the selected tokens only (the ablation of the atlas.scime
                            summary, "Measured effects": approximate vs omit unselected keys) */

/* Index configuration.  Clustering parameters follow the pages' base setting
 * (atlas.scime summary, "Measured effects": 1 centroid per 16 tokens, 8K-token
 * clustering blocks; "Approach": hierarchical variant, sliding-window update). */
typedef struct {
  int32_t batch, kv_heads, q_heads, head_dim;
  int32_t max_tokens;                 /* token capacity per sequence */
  int32_t tokens_per_centroid;        /* T: a block of L tokens gets ceil(L/T) clusters */
  int32_t block_tokens;               /* clustering block; blocks are aligned to position 0 */
  int32_t levels;                     /* 1 = flat, 2 = two-level (coarse over fine) */
  int32_t coarse_tokens_per_centroid; /* Tc (levels == 2): ceil(L/Tc) coarse clusters per block */
  int32_t kmeans_iters;               /* Lloyd iterations (>= 1) */
  int32_t update_interval;            /* re-cluster when the unclustered tail reaches this */
  int32_t dtype;                      /* mp_dtype of keys, values, queries, centroids, output */
  int32_t init;                       /* mp_init for mp_cluster_build */
  int32_t reserved;                   /* must be 0 */
  uint64_t seed;                      /* seed of the k-means++ streams */
} mp_config;

/* Host-side handle of an index living in a caller-owned device workspace.
 * Plain data: copy it freely, but keep one copy authoritative (the update
 * advances n_tokens / n_clustered).  Fields are read-only for callers. */
typedef struct {
  mp_config cfg;
  int64_t n_tokens;      /* tokens held (clustered + tail) */
  int64_t n_clustered;   /* tokens [0, n_clustered) are clustered; the rest is the tail */
  int32_t blocks_max;    /* ceil(max_tokens / block_tokens) */
  int32_t slots_per_block, slots;              /* ceil(block_tokens/T), blocks_max * that */
  int32_t coarse_per_block, coarse_slots;      /* levels == 2, else 0 */
  int32_t device;
  void* workspace;
  size_t workspace_bytes;
  uint64_t layout[24];   /* byte offsets of the arrays inside the workspace (private) */
} mp_index;

/* Device arrays of an index (mp_index_export / mp_index_import).
 *   Kc, Vc   [B, H, slots, d]       key / value centroids (dtype); slot s of
 *                                   block j is s = j*slots_per_block + local
 *   off      [B, H, slots + 1]      int32 run offsets: cluster s holds the
 *                                   store rows [off[s], off[s+1]); empty
 *                                   clusters have off[s] == off[s+1]
 *   Kp, Vp   [B, H, max_tokens, d]  cluster-ordered store: block j's tokens
 *                                   occupy rows [j*block_tokens, ...), each
 *                                   cluster contiguous, tokens in id order;
 *                                   rows [n_clustered, n_tokens) hold the tail
 *                                   in arrival order
 *   perm     [B, H, max_tokens]     int32 token id held by each store row
 *   assign   [B, H, max_tokens]     int32 cluster slot of each token id (-1: tail)
 *   Kcc, Vcc [B, H, coarse_slots, d]   levels == 2: coarse centroids (dtype)
 *   coff     [B, H, coarse_slots + 1]  levels == 2: coarse cluster c owns the
 *                                      fine slots [coff[c], coff[c+1]) */
typedef struct {
  void* Kc; void* Vc; int32_t* off;
  void* Kp; void* Vp; int32_t* perm; int32_t* assign;
  void* Kcc; void* Vcc; int32_t* coff;
} mp_index_view;

typedef struct {
  int32_t budget;           /* token budget of the (fine) selection; <= 0 selects nothing */
  int32_t coarse_budget;    /* levels == 2: token budget of the coarse selection; 0 => 8 * budget */
  float scale;              /* score scale; 0 => 1/sqrt(head_dim) */
  uint32_t flags;           /* MP_NO_APPROX */
  int32_t n_split;          /* work split of the token pass per KV head; 0 => automatic */
  int32_t reserved;         /* must be 0 */
  uint8_t* sel_mask_out;    /* optional [B, H, slots]: 1 where a fine cluster was selected */
  uint8_t* coarse_sel_mask_out; /* optional [B, H, coarse_slots] (levels == 2) */
  float* scores_out;        /* optional [B, H, slots]: group score max_g scale*q_g.Kc of every
                               scored non-empty fine cluster, -inf elsewhere */
  float* coarse_scores_out; /* optional [B, H, coarse_slots] (levels == 2) */
  void** phase_events;      /* optional: n_phase_events cudaEvent_t handles (created by the caller)
                               recorded on `stream` at the kernel boundaries of the step: the start,
                               then the end of each phase that mp_decode_phases names for the index
                               (extra handles are not touched) */
  int32_t n_phase_events;
  int32_t reserved2;        /* must be 0 */
} mp_decode_params;

/* Workspace sizes for `cfg`.  index_bytes: the index and the scratch its
 * build/update uses.  decode_scratch_bytes: scratch for one mp_decode call
 * (upper bound over all budgets and split counts).  Either pointer may be
 * NULL.  Returns MP_EINVAL for an invalid configuration. */
mp_status mp_workspace_size(const mp_config* cfg, size_t* index_bytes, size_t* decode_scratch_bytes);

/* Lay out an empty index (n_tokens = 0) in `d_workspace` (>= index_bytes,
 * 256-byte aligned) and zero it on `stream`.  Fills `*out`. */
mp_status mp_index_init(const mp_config* cfg, void* d_workspace, size_t bytes, mp_index* out,
                        void* stream);

/* Cluster tokens [0, n) of K, V ([B, H, n, d]) from scratch, replacing the
 * index content (pages: abstract, "clustering to group together semantically
 * similar key vectors"; atlas.scime summary, "Approach": blockwise).  Per
 * (batch, KV head, block): initial centroids (cfg.init, or `init_centroids`
 * [B, H, slots, d] in dtype if non-NULL), then kmeans_iters Lloyd iterations
 * (assign each key to the nearest centroid by squared L2 distance, fp32;
 * each centroid becomes the fp64 mean of its members rounded to dtype, empty
 * clusters keep theirs), value centroids = member means, and the
 * cluster-ordered store.  With levels == 2, each block's fine centroids are
 * then clustered by count-weighted k-means into ceil(L/Tc) coarse clusters
 * and the fine slots reordered by coarse cluster.  n == 0 empties the index.
 * MP_ENOSPC if n > max_tokens. */
mp_status mp_cluster_build(mp_index* idx, const void* K, const void* V, int32_t n,
                           const void* init_centroids, void* stream);

/* Append n_new generated tokens (K_new, V_new: [B, H, n_new, d]) to the
 * tail; then, if the tail holds at least update_interval tokens or reaches
 * the end of a block, re-cluster every block holding tail tokens over all its
 * tokens (pages: abstract, "fast cluster update"; atlas.scime summary,
 * "Approach": blockwise sliding-window online update).  Warm start: the
 * block's previous centroids keep their slots, new slots start at the keys
 * of the new tokens at stride T.  Full blocks are never touched again.
 * *reclustered (nullable) receives 1 if re-clustering ran.  MP_ENOSPC if
 * the capacity would be exceeded. */
mp_status mp_cluster_update(mp_index* idx, const void* K_new, const void* V_new, int32_t n_new,
                            int32_t* reclustered, void* stream);

/* One Lloyd assignment step against the index's current centroids (pages:
 * abstract, k-means clustering of the keys; atlas.scime summary, "Approach").
 * K: [B, H, n, d] device keys in dtype, the keys the index clusters, in token
 * order, with n == n_clustered (MP_EINVAL otherwise).  For every token t of
 * block j, assign_out[b, h, t] (device int32 [B, H, n], caller-owned) receives
 * the slot j * slots_per_block + c of its nearest centroid among the block's
 * ceil(L_j / T) centroids: argmin_c (|Kc_c|^2 - 2 k_t . Kc_c) in fp32, ties to
 * the lower slot; for bf16 the dot products run on the tensor cores with fp32
 * accumulation.  The index is not modified. */
mp_status mp_cluster_assign(const mp_index* idx, const void* K, int32_t n, int32_t* assign_out, void* stream);

/* One decode step (pages: abstract; atlas.scime summary, "Approach").
 * Q, O: [B, Hq, d].  Per KV head: score every non-empty cluster,
 * s[g,c] = scale * q_g . Kc_c, group score max_g s[g,c]; select clusters in
 * descending group score (ties: lower slot) until their token count reaches
 * the budget, the crossing cluster whole; then for each query head one
 * softmax over exact terms (every token of a selected cluster and every tail
 * token) and centroid terms (each unselected non-empty cluster, logit
 * s[g,c] + ln n_c, value Vc_c; dropped with MP_NO_APPROX).  With levels == 2
 * the coarse clusters are selected first (coarse_budget), fine clusters are
 * scored and selected only inside selected coarse clusters, and unselected
 * coarse clusters contribute coarse centroid terms.  Accumulation is fp32;
 * O is written in dtype.  `d_scratch` must hold decode_scratch_bytes.
 * Q and O are device memory, or page-locked host memory mapped into the
 * unified address space (cudaHostAlloc, cudaMallocHost; the benchmark's
 * host-buffer path): a host Q is copied into the scratch by a library kernel,
 * a host O is written in place over the host link, both within the stream
 * work of the call.  Any other pointer (pageable host memory) returns
 * MP_EINVAL before anything is launched.  The optional outputs in `params`
 * are device memory. */
mp_status mp_decode(const mp_index* idx, const void* Q, void* O, const mp_decode_params* params,
                    void* d_scratch, size_t scratch_bytes, void* stream);

/* Size of the library's own decode scratch used by mp_decode_static. */
#define MP_STATIC_SCRATCH_BYTES (32u << 20)

/* mp_decode for callers that cannot allocate device memory (no counterpart in
 * the paper: an interface addition).  A serving engine that gives all free
 * device memory to its own KV-cache pool at start-up has none left for the
 * decode scratch, and on a latency-critical path cudaMalloc / cudaFree may
 * synchronise the device.  Same arguments, semantics and results as
 * mp_decode, except that the scratch is a fixed array of
 * MP_STATIC_SCRATCH_BYTES (32 MiB) inside the library, which every device that
 * loads the library holds until the process exits.  It calls no allocator.
 *  - Returns MP_ENOSPC if the configuration's decode_scratch_bytes
 *    (mp_workspace_size) exceed MP_STATIC_SCRATCH_BYTES.
 *    A flat bf16 index needs the per-head centroid scores (B * Hkv * slots *
 *    4 * ceil(G / 4) * 4 bytes: 4 MiB at batch 16, 8 KV heads, 2048 slots,
 *    G = 4) plus room for a staged Q (B * Hq * d * 2 bytes: 128 KiB there),
 *    so flat bf16 configurations up to about 8 times that shape fit; fp32 and
 *    two-level indexes need the multi-kernel path's partials and run lists,
 *    which grow with batch x heads x slots.
 *  - The first call on each device, and the first after the device's current
 *    context changed (cudaDeviceReset, another driver-API context made
 *    current), looks up the array's device address (cudaGetSymbolAddress)
 *    with that device current; make that first call before any stream
 *    capture.
 *  - All calls on a device share the one array and it keeps the last call's
 *    contents; every call writes what it reads, so it needs no
 *    initialisation and no reset.  Calls that overlap on the GPU (other
 *    streams, other threads, other indices) race on it: order them, e.g. on
 *    one stream. */
mp_status mp_decode_static(const mp_index* idx, const void* Q, void* O, const mp_decode_params* params,
                           void* stream);

/* Device pointers of the index arrays (layouts above). */
mp_status mp_index_export(const mp_index* idx, mp_index_view* view);

/* Overwrite the index with arrays from `src` (device pointers with the
 * layouts above, e.g. a saved index) and set its token counts.  NULL
 * coarse pointers are allowed when levels == 1.  Enqueued on `stream`. */
mp_status mp_index_import(mp_index* idx, const mp_index_view* src, int64_t n_tokens,
                          int64_t n_clustered, void* stream);

/* Synchronise `stream`, read the device error word of the index and clear it.
 * Returns MP_OK, MP_EDEVICE (word was set; *code receives it, nullable) or
 * MP_ECUDA. */
mp_status mp_check_device_error(const mp_index* idx, int32_t* code, void* stream);

/* Dense decode: exact softmax attention of every query head over all n
 * cached keys of its KV head, no clustering.  It is the comparison point the
 * pages measure the method against (FlashDecoding; "Multipole Attention ...",
 * atlas.scime summary, "Key results" and "Experimental setup"), built here on
 * the same streaming engine as mp_decode.  `cfg` gives batch, kv_heads,
 * q_heads, head_dim, dtype and the row stride max_tokens (its clustering
 * fields are ignored).  K, V: device [B, H, max_tokens, d]; keys [0, n) of
 * each head are attended.  Q, O: device [B, Hq, d].  scale 0 => 1/sqrt(d).
 * Needs no scratch and allocates nothing.  bf16 only (MP_EUNSUPPORTED
 * otherwise); MP_EINVAL for n outside [0, max_tokens] or NULL pointers.  n = 0
 * writes O = 0. */
mp_status mp_dense_decode(const mp_config* cfg, const void* K, const void* V, int32_t n, const void* Q, void* O,
                          float scale, void* stream);

/* The phases of a decode step of this index, in order, separated by '|'
 * (e.g. "decode" for the one-kernel flat bf16 path): mp_decode records
 * phase_events[0] at the start and phase_events[i] at the end of phase i.
 * A static string; "" for a NULL index. */
const char* mp_decode_phases(const mp_index* idx);

/* Static description of a status code. */
const char* mp_status_str(mp_status s);

#ifdef __cplusplus
}
#endif
#endif /* MPATTN_H */
