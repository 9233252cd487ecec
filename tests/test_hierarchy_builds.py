"""NEXT-4: the top-down hierarchical build (fine k-means inside each coarse
cluster of a block's tokens) against R15's bottom-up build (coarse k-means
over the fine centroids), by the two-level decode's error against dense
attention at equal budgets on the same seeded cache.  CPU, oracle only.

The test checks what must hold for both builds (the error shrinks as the
budgets grow and vanishes when they cover every token) at a small size; with
MP_HIER_COMPARE_N set (e.g. 16384) and `-s` it prints the comparison table at
that size.
"""
import os

import numpy as np
import torch

from clustered_sparse_decode_b200 import synth
from oracle import multipole as mp


def _dense(Q, K, V, n, Hkv):
    q = torch.tensor(np.asarray(Q, dtype=np.float64))[:, :, None, :]
    G = q.shape[1] // Hkv
    k = torch.tensor(np.asarray(K[:, :, :n], dtype=np.float64)).repeat_interleave(G, dim=1)
    v = torch.tensor(np.asarray(V[:, :, :n], dtype=np.float64)).repeat_interleave(G, dim=1)
    return torch.nn.functional.scaled_dot_product_attention(q, k, v)[:, :, 0, :].numpy()


def compare(n, budgets, queries=8, d=64, Hkv=2, G=4, seed=40):
    """Mean relative L2 error of the two-level decode against dense attention,
    per build and per (budget, coarse budget)."""
    cfg = dict(B=1, Hkv=Hkv, Hq=G * Hkv, d=d, n_max=n, T=16, L_blk=min(n, 8192), levels=2, Tc=128, iters=5,
               update_interval=1024, dtype="f32", seed=seed)
    K, V, _ = synth.make_cache(1, Hkv, n, d, 256, 0.25, radius=(1.0, 4.0), dtype="f32", seed=seed)
    Qs = synth.make_queries(queries, 1, G * Hkv, d, "f32", seed=seed + 1)
    out = {}
    for build in ("bottom_up", "top_down"):
        idx = mp.build_index(K, V, n, cfg, hierarchy=build)
        for bud, cb in budgets:
            errs = []
            for q in Qs:
                ref = _dense(q, K, V, n, Hkv)
                O = mp.decode(idx, q, bud, coarse_budget=cb)
                errs.append(np.linalg.norm(O - ref, axis=-1) / np.linalg.norm(ref, axis=-1))
            out[(build, bud, cb)] = float(np.mean(errs))
    return out


def test_both_hierarchies_converge_to_dense_attention():
    n = 2048
    budgets = [(32, 256), (128, 1024), (n, n)]
    res = compare(n, budgets, queries=4)
    for build in ("bottom_up", "top_down"):
        e = [res[(build, b, c)] for b, c in budgets]
        assert e[0] >= e[1] - 1e-12 and e[2] < 1e-12, (build, e)
        assert e[0] < 0.5, (build, e)


def test_report_hierarchy_comparison():
    n = int(os.environ.get("MP_HIER_COMPARE_N", "0"))
    if not n:
        return
    budgets = [(128, 1024), (512, 4096), (1024, 8192)]
    res = compare(n, budgets)
    print(f"\nmean relative L2 error vs dense, n = {n} (2 KV x 4 query heads, d 64, T 16, Tc 128, 8 queries)")
    print("| budget / coarse budget | bottom-up (R15) | top-down (NEXT-4) |\n|---|---|---|")
    for b, c in budgets:
        print(f"| {b} / {c} | {res[('bottom_up', b, c)]:.4f} | {res[('top_down', b, c)]:.4f} |")
