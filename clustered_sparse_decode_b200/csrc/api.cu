// C ABI of the library: configuration checks, workspace layout, entry points.
#include <cmath>
#include <cstring>

#include "mp_internal.cuh"

namespace mp {

mp_status build_impl(mp_index* idx, const void* K, const void* V, int32_t n, const void* init, cudaStream_t st);
mp_status update_impl(mp_index* idx, const void* K_new, const void* V_new, int32_t n_new, int32_t* fired,
                      cudaStream_t st);
mp_status assign_impl(const mp_index* idx, const void* K, int32_t n, int32_t* out, cudaStream_t st);
const char* decode_phase_names(const mp_index* idx);
mp_status decode_impl(const mp_index* idx, const void* Q, void* O, const mp_decode_params* prm, void* scratch,
                      size_t scratch_bytes, cudaStream_t st);
size_t decode_scratch_bytes(const mp_config& c, int slots, int coarse_slots);
mp_status dense_decode_impl(const mp_config& c, const void* K, const void* V, int n, const void* Q, void* O,
                            float scale, cudaStream_t st);

int elem_bytes(int dtype) { return dtype == MP_BF16 ? 2 : 4; }

void* ws_ptr(const mp_index* idx, Slot s) {
  return static_cast<char*>(idx->workspace) + idx->layout[s];
}

int32_t* err_word(const mp_index* idx) { return static_cast<int32_t*>(ws_ptr(idx, S_ERR)); }

static inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct Geometry {
  int units, G, blocks_max, slots_per_block, slots, coarse_per_block, coarse_slots;
};

static mp_status check_config(const mp_config* c, Geometry* g) {
  if (!c) return MP_EINVAL;
  if (c->batch < 1 || c->kv_heads < 1 || c->q_heads < 1 || c->head_dim < 1) return MP_EINVAL;
  if (c->q_heads % c->kv_heads != 0) return MP_EINVAL;
  if (c->max_tokens < 1 || c->tokens_per_centroid < 1 || c->block_tokens < 1) return MP_EINVAL;
  if (c->block_tokens < c->tokens_per_centroid) return MP_EINVAL;
  if (c->levels != 1 && c->levels != 2) return MP_EINVAL;
  if (c->levels == 2 && c->coarse_tokens_per_centroid < 1) return MP_EINVAL;
  if (c->kmeans_iters < 1 || c->update_interval < 1) return MP_EINVAL;
  if (c->dtype != MP_F32 && c->dtype != MP_BF16) return MP_EINVAL;
  if (c->init != MP_INIT_KMEANSPP && c->init != MP_INIT_STRIDE) return MP_EINVAL;
  if (c->reserved != 0) return MP_EINVAL;
  const int G = c->q_heads / c->kv_heads;
  if (c->head_dim != 64 && c->head_dim != 128) return MP_EUNSUPPORTED;
  if (G != 1 && G != 2 && G != 4 && G != 8) return MP_EUNSUPPORTED;
  if (c->block_tokens > 16384) return MP_EUNSUPPORTED;          // k-means++ keeps a block's D^2 in shared memory
  const int64_t units = (int64_t)c->batch * c->kv_heads;
  if (units > 65535) return MP_EUNSUPPORTED;
  g->units = (int)units;
  g->G = G;
  g->blocks_max = (c->max_tokens + c->block_tokens - 1) / c->block_tokens;
  g->slots_per_block = (c->block_tokens + c->tokens_per_centroid - 1) / c->tokens_per_centroid;
  if (g->slots_per_block > 2048) return MP_EUNSUPPORTED;       // counting sort histograms in shared memory
  const int64_t slots = (int64_t)g->blocks_max * g->slots_per_block;
  if (slots > kMaxSlotsPerUnit) return MP_EUNSUPPORTED;
  g->slots = (int)slots;
  if (c->levels == 2) {
    g->coarse_per_block = (c->block_tokens + c->coarse_tokens_per_centroid - 1) / c->coarse_tokens_per_centroid;
    if (g->coarse_per_block > 256) return MP_EUNSUPPORTED;
    g->coarse_slots = g->blocks_max * g->coarse_per_block;
  } else {
    g->coarse_per_block = 0;
    g->coarse_slots = 0;
  }
  return MP_OK;
}

static size_t layout(const mp_config* c, const Geometry& g, uint64_t out[S_COUNT]) {
  const size_t es = elem_bytes(c->dtype), D = c->head_dim, U = g.units;
  size_t sz[S_COUNT] = {};
  sz[S_KC] = U * g.slots * D * es;
  sz[S_VC] = sz[S_KC];
  sz[S_OFF] = U * (g.slots + 1) * 4;
  sz[S_KP] = U * (size_t)c->max_tokens * D * es;
  sz[S_VP] = sz[S_KP];
  sz[S_PERM] = U * (size_t)c->max_tokens * 4;
  sz[S_ASSIGN] = sz[S_PERM];
  if (c->levels == 2) {
    sz[S_KCC] = U * g.coarse_slots * D * es;
    sz[S_VCC] = sz[S_KCC];
    sz[S_COFF] = U * (g.coarse_slots + 1) * 4;
    sz[S_CASSIGN] = U * g.slots * 4;
    sz[S_CORDER] = U * g.slots * 4;
    sz[S_COFFTMP] = 256;
  }
  sz[S_ERR] = 256;
  sz[S_KCTMP] = U * g.slots * D * es;
  sz[S_VCTMP] = 256;
  sz[S_BLKK] = U * (size_t)c->block_tokens * D * es;
  sz[S_BLKV] = sz[S_BLKK];
  sz[S_MOVED] = U * (size_t)g.blocks_max * 4;
  size_t cur = 0;
  for (int s = 0; s < S_COUNT; ++s) {
    if (out) out[s] = cur;
    cur = align256(cur + sz[s]);
  }
  return cur;
}

static mp_status check_index(const mp_index* idx) {
  if (!idx || !idx->workspace) return MP_EINVAL;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MP_ECUDA;
  if (dev != idx->device) return MP_EINVAL;
  return MP_OK;
}

}  // namespace mp

using namespace mp;

extern "C" {

mp_status mp_workspace_size(const mp_config* cfg, size_t* index_bytes, size_t* decode_scratch) {
  Geometry g;
  mp_status s = check_config(cfg, &g);
  if (s != MP_OK) return s;
  if (index_bytes) *index_bytes = layout(cfg, g, nullptr);
  if (decode_scratch) *decode_scratch = decode_scratch_bytes(*cfg, g.slots, g.coarse_slots);
  return MP_OK;
}

mp_status mp_index_init(const mp_config* cfg, void* d_workspace, size_t bytes, mp_index* out, void* stream) {
  Geometry g;
  mp_status s = check_config(cfg, &g);
  if (s != MP_OK) return s;
  if (!out || !d_workspace) return MP_EINVAL;
  if (reinterpret_cast<uintptr_t>(d_workspace) % 256 != 0) return MP_EINVAL;
  uint64_t lay[S_COUNT];
  const size_t need = layout(cfg, g, lay);
  if (bytes < need) return MP_ENOSPC;
  mp_index idx;
  std::memset(&idx, 0, sizeof(idx));
  idx.cfg = *cfg;
  idx.blocks_max = g.blocks_max;
  idx.slots_per_block = g.slots_per_block;
  idx.slots = g.slots;
  idx.coarse_per_block = g.coarse_per_block;
  idx.coarse_slots = g.coarse_slots;
  if (cudaGetDevice(&idx.device) != cudaSuccess) return MP_ECUDA;
  idx.workspace = d_workspace;
  idx.workspace_bytes = bytes;
  static_assert(S_COUNT <= 24, "layout table too small");
  for (int i = 0; i < S_COUNT; ++i) idx.layout[i] = lay[i];
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(d_workspace, 0, need, st) != cudaSuccess) return MP_ECUDA;
  // an empty index: every slot's run starts and ends at 0; coarse ranges at their block's first slot
  s = build_impl(&idx, nullptr, nullptr, 0, nullptr, st);
  if (s != MP_OK) return s;
  *out = idx;
  return MP_OK;
}

mp_status mp_cluster_build(mp_index* idx, const void* K, const void* V, int32_t n, const void* init_centroids,
                           void* stream) {
  mp_status s = check_index(idx);
  if (s != MP_OK) return s;
  if (n < 0) return MP_EINVAL;
  if (n > idx->cfg.max_tokens) return MP_ENOSPC;
  if (n > 0 && (!K || !V)) return MP_EINVAL;
  return build_impl(idx, K, V, n, init_centroids, static_cast<cudaStream_t>(stream));
}

mp_status mp_cluster_update(mp_index* idx, const void* K_new, const void* V_new, int32_t n_new, int32_t* reclustered,
                            void* stream) {
  mp_status s = check_index(idx);
  if (s != MP_OK) return s;
  if (n_new < 0) return MP_EINVAL;
  if (n_new > 0 && (!K_new || !V_new)) return MP_EINVAL;
  if (idx->n_tokens + n_new > idx->cfg.max_tokens) return MP_ENOSPC;
  return update_impl(idx, K_new, V_new, n_new, reclustered, static_cast<cudaStream_t>(stream));
}

mp_status mp_cluster_assign(const mp_index* idx, const void* K, int32_t n, int32_t* assign_out, void* stream) {
  mp_status s = check_index(idx);
  if (s != MP_OK) return s;
  if (n != idx->n_clustered || (n > 0 && (!K || !assign_out))) return MP_EINVAL;
  return assign_impl(idx, K, n, assign_out, static_cast<cudaStream_t>(stream));
}

mp_status mp_decode(const mp_index* idx, const void* Q, void* O, const mp_decode_params* p, void* d_scratch,
                    size_t scratch_bytes, void* stream) {
  mp_status s = check_index(idx);
  if (s != MP_OK) return s;
  if (!Q || !O || !p || !d_scratch) return MP_EINVAL;
  if (p->reserved != 0 || p->reserved2 != 0 || p->n_split < 0 || p->n_split > 64) return MP_EINVAL;
  if (p->n_phase_events < 0 || (p->n_phase_events > 0 && !p->phase_events)) return MP_EINVAL;
  if (!std::isfinite(p->scale)) return MP_EINVAL;
  if ((p->flags & ~MP_NO_APPROX) != 0) return MP_EINVAL;
  return decode_impl(idx, Q, O, p, d_scratch, scratch_bytes, static_cast<cudaStream_t>(stream));
}

mp_status mp_dense_decode(const mp_config* c, const void* K, const void* V, int32_t n, const void* Q, void* O,
                          float scale, void* stream) {
  if (!c || !K || !V || !Q || !O || !std::isfinite(scale)) return MP_EINVAL;
  if (c->batch < 1 || c->kv_heads < 1 || c->q_heads < 1 || c->q_heads % c->kv_heads != 0 || c->max_tokens < 1)
    return MP_EINVAL;
  if (n < 0 || n > c->max_tokens) return MP_EINVAL;
  if (c->dtype != MP_F32 && c->dtype != MP_BF16) return MP_EINVAL;
  const int G = c->q_heads / c->kv_heads;
  if (c->dtype != MP_BF16 || (c->head_dim != 64 && c->head_dim != 128) || (G != 1 && G != 2 && G != 4 && G != 8))
    return MP_EUNSUPPORTED;
  if ((int64_t)c->batch * c->kv_heads * c->max_tokens + 64 >= (int64_t)INT32_MAX) return MP_EUNSUPPORTED;
  return dense_decode_impl(*c, K, V, n, Q, O, scale, static_cast<cudaStream_t>(stream));
}

mp_status mp_index_export(const mp_index* idx, mp_index_view* v) {
  if (!idx || !idx->workspace || !v) return MP_EINVAL;
  v->Kc = ws_ptr(idx, S_KC);
  v->Vc = ws_ptr(idx, S_VC);
  v->off = static_cast<int32_t*>(ws_ptr(idx, S_OFF));
  v->Kp = ws_ptr(idx, S_KP);
  v->Vp = ws_ptr(idx, S_VP);
  v->perm = static_cast<int32_t*>(ws_ptr(idx, S_PERM));
  v->assign = static_cast<int32_t*>(ws_ptr(idx, S_ASSIGN));
  if (idx->cfg.levels == 2) {
    v->Kcc = ws_ptr(idx, S_KCC);
    v->Vcc = ws_ptr(idx, S_VCC);
    v->coff = static_cast<int32_t*>(ws_ptr(idx, S_COFF));
  } else {
    v->Kcc = v->Vcc = nullptr;
    v->coff = nullptr;
  }
  return MP_OK;
}

mp_status mp_index_import(mp_index* idx, const mp_index_view* src, int64_t n_tokens, int64_t n_clustered,
                          void* stream) {
  mp_status s = check_index(idx);
  if (s != MP_OK) return s;
  if (!src) return MP_EINVAL;
  if (n_clustered < 0 || n_clustered > n_tokens || n_tokens > idx->cfg.max_tokens) return MP_EINVAL;
  if (!src->Kc || !src->Vc || !src->off || !src->Kp || !src->Vp || !src->perm || !src->assign) return MP_EINVAL;
  const bool two = idx->cfg.levels == 2;
  if (two && (!src->Kcc || !src->Vcc || !src->coff)) return MP_EINVAL;
  const size_t es = elem_bytes(idx->cfg.dtype), D = idx->cfg.head_dim;
  const size_t U = (size_t)idx->cfg.batch * idx->cfg.kv_heads, n_max = idx->cfg.max_tokens;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  mp_index_view dst;
  mp_index_export(idx, &dst);
  struct Cp { void* d; const void* s; size_t n; } cps[] = {
      {dst.Kc, src->Kc, U * idx->slots * D * es},
      {dst.Vc, src->Vc, U * idx->slots * D * es},
      {dst.off, src->off, U * (idx->slots + 1) * 4},
      {dst.Kp, src->Kp, U * n_max * D * es},
      {dst.Vp, src->Vp, U * n_max * D * es},
      {dst.perm, src->perm, U * n_max * 4},
      {dst.assign, src->assign, U * n_max * 4},
      {two ? dst.Kcc : nullptr, src->Kcc, U * idx->coarse_slots * D * es},
      {two ? dst.Vcc : nullptr, src->Vcc, U * idx->coarse_slots * D * es},
      {two ? (void*)dst.coff : nullptr, src->coff, U * (idx->coarse_slots + 1) * 4},
  };
  for (const Cp& c : cps) {
    if (!c.d || c.n == 0) continue;
    if (cudaMemcpyAsync(c.d, c.s, c.n, cudaMemcpyDeviceToDevice, st) != cudaSuccess) return MP_ECUDA;
  }
  idx->n_tokens = n_tokens;
  idx->n_clustered = n_clustered;
  return MP_OK;
}

mp_status mp_check_device_error(const mp_index* idx, int32_t* code, void* stream) {
  mp_status s = check_index(idx);
  if (s != MP_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t h = 0;
  if (cudaMemcpyAsync(&h, err_word(idx), sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess) return MP_ECUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MP_ECUDA;
  if (code) *code = h;
  if (h != 0) {
    if (cudaMemsetAsync(err_word(idx), 0, sizeof(int32_t), st) != cudaSuccess) return MP_ECUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return MP_ECUDA;
    return MP_EDEVICE;
  }
  return MP_OK;
}

const char* mp_decode_phases(const mp_index* idx) {
  if (!idx) return "";
  return decode_phase_names(idx);
}

const char* mp_status_str(mp_status s) {
  switch (s) {
    case MP_OK: return "ok";
    case MP_EINVAL: return "invalid argument";
    case MP_ENOSPC: return "capacity or buffer size exceeded";
    case MP_ECUDA: return "CUDA error";
    case MP_EUNSUPPORTED: return "unsupported configuration";
    case MP_EDEVICE: return "device error word set";
  }
  return "unknown status";
}

}  // extern "C"
