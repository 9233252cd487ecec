"""Seeded synthetic GQA KV caches and decode queries.

This module only draws inputs.  It holds none of the attention or clustering
arithmetic and imports nothing else from this package, so the CUDA path and the
CPU checker can both take their inputs from it.

The caches stand in for the long-context reasoning workloads of "Multipole
Attention for Efficient Long Context Reasoning" (LongBench-V2, GSM-Infinite,
LongBench-V1 with Qwen3-8B; atlas.scime summary, "Experimental setup"), which
are not available here.  Keys come from a per-head Gaussian mixture, so that
keys really do form semantic clusters; values and queries are standard
normal.  Arrays are float32 holding values that are exact in the target dtype
(bf16 values are rounded to nearest-even once, here).
"""
from __future__ import annotations

import numpy as np

__all__ = ["to_bf16_exact", "mixture_keys", "make_cache", "make_queries", "component_assignment",
           "WORKLOADS", "workload"]


def to_bf16_exact(x):
    """float32 array -> float32 array of the nearest bf16 values (ties to even)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def _cast(x, dtype):
    x = np.asarray(x, dtype=np.float32)
    return to_bf16_exact(x) if dtype == "bf16" else x


def mixture_keys(rng, n, d, comps, sigma, radius, outliers, drift=None):
    """n keys of one head from a `comps`-component isotropic Gaussian mixture.

    radius=None: component means ~ N(0, 1) per channel.  radius=(lo, hi): means
    r_j * u_j with u_j uniform on the unit sphere and r_j ~ U(lo, hi).
    outliers=(k, s): k seeded channels of the head are multiplied by s.
    drift=(step, every, start): from token `start` on, after every `every`
    tokens all means move by a random direction of norm `step`.
    Returns (keys [n, d] float64, labels [n]).
    """
    if radius is None:
        mu = rng.standard_normal((comps, d))
    else:
        u = rng.standard_normal((comps, d))
        u /= np.linalg.norm(u, axis=1, keepdims=True)
        mu = u * rng.uniform(radius[0], radius[1], size=(comps, 1))
    labels = rng.integers(0, comps, size=n)
    noise = sigma * rng.standard_normal((n, d))
    if drift is None:
        keys = mu[labels] + noise
    else:
        step, every, start = drift
        keys = np.empty((n, d))
        keys[:start] = mu[labels[:start]] + noise[:start]
        for s in range(start, n, every):
            e = min(n, s + every)
            keys[s:e] = mu[labels[s:e]] + noise[s:e]
            dirs = rng.standard_normal((comps, d))
            dirs /= np.linalg.norm(dirs, axis=1, keepdims=True)
            mu = mu + step * dirs
    if outliers is not None:
        k, s = outliers
        ch = rng.choice(d, size=k, replace=False)
        keys[:, ch] *= s
    return keys, labels


def make_cache(B, Hkv, n, d, comps, sigma, radius=None, outliers=None, dtype="bf16", seed=0,
               drift=None):
    """K, V [B, Hkv, n, d] float32 (dtype-exact) and mixture labels [B, Hkv, n].

    Sequence b of the batch uses its own generator seeded with seed + b.
    """
    K = np.empty((B, Hkv, n, d), dtype=np.float32)
    V = np.empty((B, Hkv, n, d), dtype=np.float32)
    lab = np.empty((B, Hkv, n), dtype=np.int64)
    for b in range(B):
        rng = np.random.default_rng(seed + b)
        for h in range(Hkv):
            k, l = mixture_keys(rng, n, d, comps, sigma, radius, outliers, drift)
            K[b, h] = _cast(k, dtype)
            lab[b, h] = l
            V[b, h] = _cast(rng.standard_normal((n, d)), dtype)
    return K, V, lab


def make_queries(steps, B, Hq, d, dtype="bf16", seed=0, scale=1.0):
    """Decode queries [steps, B, Hq, d], N(0, scale^2) per element."""
    rng = np.random.default_rng(seed)
    return _cast(scale * rng.standard_normal((steps, B, Hq, d)), dtype)


def component_assignment(labels, n, L_blk, T):
    """A block-local cluster id per token taken from its mixture component.

    Block j (ceil(L_j/T) slots) maps component c to slot c mod ceil(L_j/T).
    Gives decode tests an index whose clusters are real mixture components
    without running k-means.
    """
    a = np.empty(labels.shape[:-1] + (n,), dtype=np.int64)
    for s in range(0, n, L_blk):
        e = min(n, s + L_blk)
        C = -(-(e - s) // T)
        a[..., s:e] = labels[..., s:e] % C
    return a


# Workloads: the five configurations the method is exercised on.  Sizes follow
# the pages' evaluation setting (8 KV / 32 query heads, head_dim 128, budgets
# 128 and 512 tokens, 1 centroid per 16 tokens, 8K-token blocks).
WORKLOADS = {
    "tiny_f32": dict(B=1, Hkv=1, Hq=4, d=64, n=2048, comps=64, sigma=0.3, radius=None, outliers=None,
                     dtype="f32", T=16, L_blk=2048, budget=128, iters=10, steps=1, seed=1000),
    "single_bf16": dict(B=1, Hkv=8, Hq=32, d=128, n=32768, comps=512, sigma=0.25, radius=(1.0, 4.0),
                        outliers=(4, 4.0), dtype="bf16", T=16, L_blk=8192, budget=128, iters=10,
                        steps=64, seed=2000),
    "batch16_32k_sparse95": dict(B=16, Hkv=8, Hq=32, d=128, n=32768, comps=512, sigma=0.25,
                                 radius=(1.0, 4.0), outliers=(4, 4.0), dtype="bf16", T=16,
                                 L_blk=8192, budget=1638, iters=10, steps=64, seed=3000),
    "batch4_32k_sparse95": dict(B=4, Hkv=8, Hq=32, d=128, n=32768, comps=512, sigma=0.25,
                                radius=(1.0, 4.0), outliers=(4, 4.0), dtype="bf16", T=16,
                                L_blk=8192, budget=1638, iters=10, steps=64, seed=3500),
    "hier_64k": dict(B=4, Hkv=8, Hq=32, d=128, n=65536, comps=512, sigma=0.25, radius=(1.0, 4.0),
                     outliers=(4, 4.0), dtype="bf16", T=16, L_blk=8192, budget=512, levels=2, Tc=128,
                     coarse_budget=4096, iters=10, steps=64, seed=4000),
    "online_16k_plus_16k": dict(B=8, Hkv=8, Hq=32, d=128, n=16384, n_gen=16384, comps=512, sigma=0.25,
                                radius=(1.0, 4.0), outliers=(4, 4.0), dtype="bf16", T=16, L_blk=8192,
                                budget=128, iters=10, update_interval=1024, drift=(0.01, 256, 16384),
                                steps=64, seed=5000),
}


def workload(name, **over):
    w = dict(WORKLOADS[name])
    w.update(over)
    return w
