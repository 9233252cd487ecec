"""Python binding of libmpattn: a multipole-attention KV index on one GPU.

Marshalling only: torch allocates the device memory and supplies the stream;
every step of clustering and decoding runs in the library's CUDA kernels.
There is no CPU fallback: without the built library every call raises.
"""
from __future__ import annotations

import ctypes
import math
from dataclasses import dataclass

import torch

from . import _lib as L

_DT = {"bf16": (L.MP_BF16, torch.bfloat16), "f32": (L.MP_F32, torch.float32)}


@dataclass
class Config:
    """Index configuration (see mp_config in include/mpattn.h)."""
    batch: int
    kv_heads: int
    q_heads: int
    head_dim: int
    max_tokens: int
    tokens_per_centroid: int = 16
    block_tokens: int = 8192
    levels: int = 1
    coarse_tokens_per_centroid: int = 128
    kmeans_iters: int = 10
    update_interval: int = 1024
    dtype: str = "bf16"
    init: str = "kmeans++"          # or "stride"
    seed: int = 0

    def to_c(self) -> L.MpConfig:
        c = L.MpConfig()
        for f in ("batch", "kv_heads", "q_heads", "head_dim", "max_tokens", "tokens_per_centroid",
                  "block_tokens", "levels", "coarse_tokens_per_centroid", "kmeans_iters", "update_interval"):
            setattr(c, f, int(getattr(self, f)))
        c.dtype = _DT[self.dtype][0]
        c.init = {"kmeans++": L.MP_INIT_KMEANSPP, "stride": L.MP_INIT_STRIDE}[self.init]
        c.reserved = 0
        c.seed = int(self.seed) & ((1 << 64) - 1)
        return c

    @property
    def torch_dtype(self):
        return _DT[self.dtype][1]


def workspace_size(cfg: Config):
    """(index_bytes, decode_scratch_bytes) for cfg."""
    lib = L.load()
    c = cfg.to_c()
    a, b = ctypes.c_size_t(), ctypes.c_size_t()
    L.check(lib.mp_workspace_size(ctypes.byref(c), ctypes.byref(a), ctypes.byref(b)), "mp_workspace_size")
    return a.value, b.value


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def dense_decode(cfg: Config, K, V, n, Q, out=None, scale=0.0, stream=None):
    """Exact attention of every query head over keys [0, n) of its KV head (mp_dense_decode).

    K, V: contiguous device tensors [B, Hkv, max_tokens, d]; Q: [B, Hq, d]; returns
    O [B, Hq, d].  The dense comparison point of the method, on the same engine.
    """
    lib = L.load()
    want = (cfg.batch, cfg.kv_heads, cfg.max_tokens, cfg.head_dim)
    for t in (K, V):
        if tuple(t.shape) != want or t.dtype != cfg.torch_dtype or not t.is_contiguous() or t.device.type != "cuda":
            raise ValueError(f"K and V must be contiguous {cfg.torch_dtype} device tensors of shape {want}")
    qw = (cfg.batch, cfg.q_heads, cfg.head_dim)
    if tuple(Q.shape) != qw or Q.dtype != cfg.torch_dtype or not Q.is_contiguous() or Q.device.type != "cuda":
        raise ValueError(f"Q must be a contiguous {cfg.torch_dtype} device tensor of shape {qw}")
    if out is None:
        out = torch.empty_like(Q)
    c = cfg.to_c()
    L.check(lib.mp_dense_decode(ctypes.byref(c), _ptr(K), _ptr(V), int(n), _ptr(Q), _ptr(out), float(scale),
                                _stream(stream)), "mp_dense_decode")
    return out


class MultipoleIndex:
    """Clustered KV cache of one attention layer: build, update, decode."""

    def __init__(self, cfg: Config, device=None, stream=None):
        self.lib = L.load()
        self.cfg = cfg
        self.device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        ib, sb = workspace_size(cfg)
        with torch.cuda.device(self.device):
            self.workspace = torch.empty(ib, dtype=torch.uint8, device=self.device)
            self.scratch_bytes = sb
            self._scratch = None     # allocated by the first decode() (decode_static() needs none)
            self.h = L.MpIndex()
            c = cfg.to_c()
            L.check(self.lib.mp_index_init(ctypes.byref(c), _ptr(self.workspace), ib, ctypes.byref(self.h),
                                           _stream(stream)), "mp_index_init")

    # ------------------------------------------------------------------ state
    @property
    def n_tokens(self):
        return self.h.n_tokens

    @property
    def n_clustered(self):
        return self.h.n_clustered

    @property
    def slots(self):
        return self.h.slots

    @property
    def coarse_slots(self):
        return self.h.coarse_slots

    def decode_phases(self):
        """Names of the intervals between the phase events that decode() records
        for this index, as the library reports them (mp_decode_phases)."""
        return self.lib.mp_decode_phases(ctypes.byref(self.h)).decode().split("|")

    def _check_kv(self, t, n):
        c = self.cfg
        want = (c.batch, c.kv_heads, n, c.head_dim)
        if tuple(t.shape) != want or t.dtype != c.torch_dtype or not t.is_contiguous() or t.device != self.device:
            raise ValueError(f"expected a contiguous {c.torch_dtype} tensor of shape {want} on {self.device}")

    def _check_q_out(self, Q, out):
        """Shape, dtype and memory checks of a decode's Q and O; allocates O if absent
        (pinned host memory for a host Q)."""
        c = self.cfg
        want = (c.batch, c.q_heads, c.head_dim)
        if tuple(Q.shape) != want or Q.dtype != c.torch_dtype or not Q.is_contiguous():
            raise ValueError(f"Q must be a contiguous {c.torch_dtype} tensor of shape {want}")
        if Q.device.type == "cpu" and not Q.is_pinned():
            raise ValueError("a host Q must be in page-locked memory (pin_memory())")
        if out is None:
            return torch.empty_like(Q, pin_memory=Q.device.type == "cpu")
        if (tuple(out.shape) != want or out.dtype != c.torch_dtype or not out.is_contiguous()
                or (out.device.type == "cpu" and not out.is_pinned())):
            raise ValueError(f"out must be a contiguous {c.torch_dtype} tensor of shape {want}, "
                             "on the device or in page-locked host memory")
        return out

    # ------------------------------------------------------------------ calls
    def build(self, K, V, init_centroids=None, stream=None):
        """Cluster K, V [B, Hkv, n, d] from scratch (mp_cluster_build)."""
        n = K.shape[2]
        self._check_kv(K, n)
        self._check_kv(V, n)
        if init_centroids is not None:
            c = self.cfg
            want = (c.batch, c.kv_heads, self.slots, c.head_dim)
            if tuple(init_centroids.shape) != want or init_centroids.dtype != c.torch_dtype:
                raise ValueError(f"init_centroids must be {want} {c.torch_dtype}")
            init_centroids = init_centroids.contiguous()
        L.check(self.lib.mp_cluster_build(ctypes.byref(self.h), _ptr(K), _ptr(V), int(n), _ptr(init_centroids),
                                          _stream(stream)), "mp_cluster_build")

    def update(self, K_new, V_new, stream=None):
        """Append generated tokens; returns True when blocks were re-clustered (mp_cluster_update)."""
        n = K_new.shape[2]
        self._check_kv(K_new, n)
        self._check_kv(V_new, n)
        fired = ctypes.c_int32(0)
        L.check(self.lib.mp_cluster_update(ctypes.byref(self.h), _ptr(K_new), _ptr(V_new), int(n),
                                           ctypes.byref(fired), _stream(stream)), "mp_cluster_update")
        return bool(fired.value)

    def assign(self, K, out=None, stream=None):
        """Nearest-centroid slot of every clustered key under the current centroids (mp_cluster_assign).

        K: the index's keys [B, Hkv, n_clustered, d] in token order; returns
        int32 [B, Hkv, n_clustered] global slots.
        """
        n = self.n_clustered
        self._check_kv(K, n)
        c = self.cfg
        want = (c.batch, c.kv_heads, n)
        if out is None:
            out = torch.empty(want, dtype=torch.int32, device=self.device)
        elif tuple(out.shape) != want or out.dtype != torch.int32 or not out.is_contiguous() or out.device != self.device:
            raise ValueError(f"out must be a contiguous int32 tensor of shape {want} on {self.device}")
        L.check(self.lib.mp_cluster_assign(ctypes.byref(self.h), _ptr(K), int(n), _ptr(out), _stream(stream)),
                "mp_cluster_assign")
        return out

    def decode(self, Q, budget, coarse_budget=0, scale=0.0, no_approx=False, n_split=0, out=None,
               sel_mask=None, coarse_sel_mask=None, scores=None, coarse_scores=None, phase_events=None,
               stream=None):
        """One decode step: O [B, Hq, d] for Q [B, Hq, d] (mp_decode).

        Q and out may be device tensors or page-locked (pinned) host tensors;
        a host Q is copied in by the library's kernel and a host out is written
        over the host link, within the call's stream work.

        Optional device outputs: sel_mask / coarse_sel_mask (uint8 [B, Hkv, slots]),
        scores / coarse_scores (float32 [B, Hkv, slots]).  phase_events: torch.cuda.Event
        objects (already recorded once) that the library records at its kernel boundaries.
        """
        out = self._check_q_out(Q, out)
        p = L.MpDecodeParams()
        p.budget = int(budget)
        p.coarse_budget = int(coarse_budget)
        p.scale = float(scale)
        p.flags = L.MP_NO_APPROX if no_approx else 0
        p.n_split = int(n_split)
        p.reserved = 0
        p.sel_mask_out = sel_mask.data_ptr() if sel_mask is not None else None
        p.coarse_sel_mask_out = coarse_sel_mask.data_ptr() if coarse_sel_mask is not None else None
        p.scores_out = scores.data_ptr() if scores is not None else None
        p.coarse_scores_out = coarse_scores.data_ptr() if coarse_scores is not None else None
        evs = None
        if phase_events:
            evs = (ctypes.c_void_p * len(phase_events))(*[e.cuda_event for e in phase_events])
            p.phase_events = ctypes.cast(evs, ctypes.c_void_p)
            p.n_phase_events = len(phase_events)
        p.reserved2 = 0
        L.check(self.lib.mp_decode(ctypes.byref(self.h), _ptr(Q), _ptr(out), ctypes.byref(p), _ptr(self.scratch),
                                   self.scratch.numel(), _stream(stream)), "mp_decode")
        return out

    def decode_static(self, Q, budget, coarse_budget=0, scale=0.0, no_approx=False, n_split=0, out=None,
                      stream=None):
        """decode() without the index's scratch tensor (mp_decode_static).

        For callers that cannot allocate device memory when they decode: the
        library's own fixed 32 MiB device array serves as scratch.  Calls that
        overlap on the GPU race on that array; the first call on a device should
        come before any stream capture.
        """
        out = self._check_q_out(Q, out)
        p = L.MpDecodeParams()
        p.budget = int(budget)
        p.coarse_budget = int(coarse_budget)
        p.scale = float(scale)
        p.flags = L.MP_NO_APPROX if no_approx else 0
        p.n_split = int(n_split)
        L.check(self.lib.mp_decode_static(ctypes.byref(self.h), _ptr(Q), _ptr(out), ctypes.byref(p),
                                          _stream(stream)), "mp_decode_static")
        return out

    def arrays(self):
        """Views (torch tensors) of the index arrays inside the workspace (mp_index_export)."""
        v = L.MpIndexView()
        L.check(self.lib.mp_index_export(ctypes.byref(self.h), ctypes.byref(v)), "mp_index_export")
        c = self.cfg
        U = (c.batch, c.kv_heads)
        base = self.workspace.data_ptr()
        dt = c.torch_dtype
        es = torch.tensor([], dtype=dt).element_size()

        def view(ptr, shape, dtype, esize):
            if not ptr:
                return None
            n = math.prod(shape)
            o = ptr - base
            return self.workspace[o:o + n * esize].view(dtype).view(shape)

        out = {
            "Kc": view(v.Kc, U + (self.slots, c.head_dim), dt, es),
            "Vc": view(v.Vc, U + (self.slots, c.head_dim), dt, es),
            "off": view(v.off, U + (self.slots + 1,), torch.int32, 4),
            "Kp": view(v.Kp, U + (c.max_tokens, c.head_dim), dt, es),
            "Vp": view(v.Vp, U + (c.max_tokens, c.head_dim), dt, es),
            "perm": view(v.perm, U + (c.max_tokens,), torch.int32, 4),
            "assign": view(v.assign, U + (c.max_tokens,), torch.int32, 4),
        }
        if c.levels == 2:
            out["Kcc"] = view(v.Kcc, U + (self.coarse_slots, c.head_dim), dt, es)
            out["Vcc"] = view(v.Vcc, U + (self.coarse_slots, c.head_dim), dt, es)
            out["coff"] = view(v.coff, U + (self.coarse_slots + 1,), torch.int32, 4)
        return out

    def load_arrays(self, arrays, n_tokens, n_clustered, stream=None):
        """Overwrite the index from device tensors with the layouts of arrays() (mp_index_import)."""
        v = L.MpIndexView()
        for k in ("Kc", "Vc", "off", "Kp", "Vp", "perm", "assign", "Kcc", "Vcc", "coff"):
            t = arrays.get(k)
            setattr(v, k, t.data_ptr() if t is not None else None)
        L.check(self.lib.mp_index_import(ctypes.byref(self.h), ctypes.byref(v), int(n_tokens), int(n_clustered),
                                         _stream(stream)), "mp_index_import")

    @property
    def scratch(self):
        """The decode scratch of mp_decode (device bytes), allocated on first use."""
        if self._scratch is None:
            with torch.cuda.device(self.device):
                self._scratch = torch.empty(self.scratch_bytes, dtype=torch.uint8, device=self.device)
        return self._scratch

    def check_device_error(self, stream=None):
        """Synchronise and return the device error word (0 = none); clears it."""
        code = ctypes.c_int32(0)
        st = self.lib.mp_check_device_error(ctypes.byref(self.h), ctypes.byref(code), _stream(stream))
        if st not in (L.MP_OK, L.MP_EDEVICE):
            L.check(st, "mp_check_device_error")
        return code.value
