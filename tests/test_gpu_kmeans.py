"""Clustering parity: the CUDA build/update (through the C ABI) against the fp64 oracle.

Assignments are decided on fp32 distances on both sides; a row whose two
nearest centroids lie closer than the fp32 error bound of the distance is a
tie and may go either way.  Where no tie occurred in a block's trajectory, the
whole index (centroids, offsets, permutation, store) must be bit-exact; past
the first tie only the iterations before it are compared exactly and the rest
through invariants that hold for any assignment.
"""
import numpy as np
import pytest
import torch

import helpers as H
from clustered_sparse_decode_b200 import MultipoleIndex, synth
from oracle import multipole as mp

pytestmark = pytest.mark.gpu


def tie_band(X, cents):
    """Per-row bound on the fp32 error of ||c||^2 - 2 x.c (d terms, relative error d * 2^-24)."""
    d = X.shape[1]
    return 4.0 * d * 2.0 ** -24 * (np.sum(X * X, axis=1) + np.max(np.sum(cents * cents, axis=1)))


def first_tie_iteration(hist, X, init):
    """Index of the first Lloyd iteration with a near-tie row (len(hist) if none)."""
    prev = init
    for t, h in enumerate(hist):
        if np.any(h["gap"] <= tie_band(X, prev)):
            return t
        prev = h["cents"]
    return len(hist)


def gpu_build(o, K, V, n, init=None, init_mode="kmeans++", iters=None):
    oo = dict(o)
    if iters is not None:
        oo["iters"] = iters
    g = MultipoleIndex(H.gcfg(oo, init=init_mode))
    g.build(H.tdev(K[:, :, :n], o["dtype"]), H.tdev(V[:, :, :n], o["dtype"]),
            init_centroids=None if init is None else H.tdev(init, o["dtype"]))
    torch.cuda.synchronize()
    assert g.check_device_error() == 0
    return g


def arrays_np(g):
    return {k: (H.to_np(v) if v.dtype in (torch.bfloat16, torch.float32) else v.cpu().numpy().astype(np.int64))
            for k, v in g.arrays().items()}


def assert_index_equal(ga, oidx, n, keys=("Kc", "Vc", "off", "Kp", "Vp", "perm", "assign")):
    for k in keys:
        a, b = ga[k], oidx[k]
        if k in ("Kp", "Vp", "perm", "assign"):
            a, b = a[:, :, :n], b[:, :, :n]
        np.testing.assert_array_equal(a, b, err_msg=k)


def check_invariants(o, ga, K, V, n):
    """Properties any valid index satisfies, whatever the trajectory."""
    B, Hk, T, Lb = o["B"], o["Hkv"], o["T"], o["L_blk"]
    for b in range(B):
        for h in range(Hk):
            perm = ga["perm"][b, h, :n]
            assert np.array_equal(np.sort(perm), np.arange(n))
            np.testing.assert_array_equal(ga["Kp"][b, h, :n], K[b, h, perm])
            np.testing.assert_array_equal(ga["Vp"][b, h, :n], V[b, h, perm])
            off = ga["off"][b, h]
            assert np.all(np.diff(off) >= 0) and off[-1] == n
            cnt = np.diff(off)
            for c in np.nonzero(cnt)[0]:
                ids = perm[off[c]:off[c + 1]]
                assert np.all(np.diff(ids) > 0)
                assert np.all(ga["assign"][b, h, ids] == c)
                mk = mp.round_to_dtype(K[b, h, ids].astype(np.float64).mean(0), o["dtype"])
                mv = mp.round_to_dtype(V[b, h, ids].astype(np.float64).mean(0), o["dtype"])
                # summation order can differ from a plain mean by fp64 rounding only
                assert np.abs(ga["Kc"][b, h, c] - mk).max() <= np.abs(mk).max() * 2 ** -7 + 1e-30
                assert np.abs(ga["Vc"][b, h, c] - mv).max() <= np.abs(mv).max() * 2 ** -7 + 1e-30


@pytest.mark.parametrize("init_mode", ["kmeans++", "stride"])
def test_tiny_f32_build_is_bit_exact(init_mode):
    """64-component mixture, one block of 2048 keys, 128 clusters, 10 Lloyd iterations."""
    w = synth.workload("tiny_f32")
    o = H.ocfg(B=1, Hkv=1, Hq=4, d=64, n_max=2048, T=16, L_blk=2048, dtype="f32", iters=10, seed=42)
    K, V, _ = synth.make_cache(1, 1, 2048, 64, w["comps"], w["sigma"], dtype="f32", seed=w["seed"])
    rec = {}
    oidx = mp.build_index(K, V, 2048, o, init_mode=init_mode, record=rec)
    g = gpu_build(o, K, V, 2048, init_mode=init_mode)
    ga = arrays_np(g)
    X = K[0, 0].astype(np.float64)
    C = 128
    u = mp.stream_uniforms(42, 0, 0, 0, C)
    init = X[mp.kmeanspp_pick(X, C, u)] if init_mode == "kmeans++" else X[16 * np.arange(C)]
    t_tie = first_tie_iteration(rec[(0, 0, 0)], X, init)
    assert t_tie == 10, "this seed has a near-tie; pick another"
    assert_index_equal(ga, oidx, 2048)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_each_lloyd_iteration_matches(dtype):
    """Builds with 1..6 iterations from the same given init, each against the oracle's trajectory."""
    o = H.ocfg(B=1, Hkv=2, Hq=8, d=128, n_max=5000, T=16, L_blk=2048, dtype=dtype, seed=3)
    K, V, lab = H.cache_for(o, 5000, comps=96, seed=21)
    n = 4500                                            # ragged last block
    g0 = MultipoleIndex(H.gcfg(o, init="stride"))
    init = np.zeros((1, 2, g0.slots, 128))
    rng = np.random.default_rng(0)
    for j in range(3):
        L = min(n, (j + 1) * 2048) - j * 2048
        C = -(-L // 16)
        for h in range(2):
            pick = rng.choice(L, size=C, replace=False)
            init[0, h, j * 128:j * 128 + C] = K[0, h, j * 2048 + pick]
    checked = 0
    for iters in range(1, 7):
        o_it = dict(o, iters=iters)
        rec = {}
        oidx = mp.build_index(K, V, n, o_it, init=init, record=rec)
        ga = arrays_np(gpu_build(o, K, V, n, init=init, iters=iters))
        for h in range(2):
            for j in range(3):
                s, e = j * 2048, min(n, (j + 1) * 2048)
                X = K[0, h, s:e].astype(np.float64)
                C = -(-(e - s) // 16)
                hist = rec[(0, h, j)]
                t_tie = first_tie_iteration(hist, X, init[0, h, j * 128:j * 128 + C])
                if t_tie < iters:
                    continue                             # trajectory may legitimately differ
                sl = slice(j * 128, (j + 1) * 128)
                np.testing.assert_array_equal(ga["Kc"][0, h, sl], oidx["Kc"][0, h, sl])
                np.testing.assert_array_equal(ga["Vc"][0, h, sl], oidx["Vc"][0, h, sl])
                np.testing.assert_array_equal(ga["off"][0, h, sl], oidx["off"][0, h, sl])
                np.testing.assert_array_equal(ga["perm"][0, h, s:e], oidx["perm"][0, h, s:e])
                np.testing.assert_array_equal(ga["assign"][0, h, s:e], oidx["assign"][0, h, s:e])
                np.testing.assert_array_equal(ga["Kp"][0, h, s:e], oidx["Kp"][0, h, s:e])
                checked += 1
        check_invariants(o, ga, K, V, n)
    assert checked >= 18 * 0.7


def test_kmeanspp_seeding_matches_oracle_picks():
    """iters = 1 builds start from k-means++ picks; the picks are integer decisions."""
    o = H.ocfg(B=2, Hkv=2, Hq=4, d=64, n_max=3000, T=16, L_blk=1024, dtype="bf16", iters=1, seed=77)
    K, V, _ = H.cache_for(o, 3000, comps=40, seed=5)
    rec = {}
    oidx = mp.build_index(K, V, 3000, o, record=rec)
    ga = arrays_np(gpu_build(o, K, V, 3000))
    for b in range(2):
        for h in range(2):
            for j in range(3):
                s, e = j * 1024, min(3000, (j + 1) * 1024)
                X = K[b, h, s:e].astype(np.float64)
                C = -(-(e - s) // 16)
                u = mp.stream_uniforms(77, b * 2 + h, j, 0, C)
                init = X[mp.kmeanspp_pick(X, C, u)]
                if first_tie_iteration(rec[(b, h, j)], X, init) < 1:
                    continue
                sl = slice(j * 64, j * 64 + C)
                np.testing.assert_array_equal(ga["Kc"][b, h, sl], oidx["Kc"][b, h, sl])
                np.testing.assert_array_equal(ga["perm"][b, h, s:e], oidx["perm"][b, h, s:e])


def test_hierarchical_build_is_bit_exact_without_ties():
    o = H.ocfg(B=1, Hkv=2, Hq=8, d=64, n_max=4096, T=16, L_blk=2048, levels=2, Tc=128, dtype="f32", iters=5,
               seed=9)
    K, V, _ = H.cache_for(o, 4096, comps=48, radius=None, sigma=0.3, seed=12)
    rec = {}
    oidx = mp.build_index(K, V, 4000, o, record=rec)
    ga = arrays_np(gpu_build(o, K, V, 4000))
    exact = 0
    for h in range(2):
        ok = True
        for j in range(2):
            s, e = j * 2048, min(4000, (j + 1) * 2048)
            X = K[0, h, s:e].astype(np.float64)
            C = -(-(e - s) // 16)
            u = mp.stream_uniforms(9, h, j, 0, C)
            init = X[mp.kmeanspp_pick(X, C, u)]
            if first_tie_iteration(rec[(0, h, j)], X, init) < 5:
                ok = False
            ch = rec[(0, h, j, "coarse")]
            if first_tie_iteration(ch["hist"], ch["points"], ch["points"][ch["picks"]]) < 5:
                ok = False
        if not ok:
            continue
        for k in ("Kc", "Vc", "off", "Kcc", "Vcc", "coff"):
            np.testing.assert_array_equal(ga[k][0, h], oidx[k][0, h], err_msg=k)
        for k in ("Kp", "Vp", "perm", "assign"):
            np.testing.assert_array_equal(ga[k][0, h, :4000], oidx[k][0, h, :4000], err_msg=k)
        exact += 1
    assert exact >= 1


def test_online_update_matches_oracle():
    """Prompt build, then appends that trigger warm-started re-clustering of the open block."""
    o = H.ocfg(B=1, Hkv=2, Hq=8, d=64, n_max=4096, T=16, L_blk=1024, update_interval=256, dtype="f32",
               iters=4, seed=13)
    K, V, _ = H.cache_for(o, 4096, comps=32, radius=None, sigma=0.3, seed=14)
    rec_b = {}
    oidx = mp.build_index(K, V, 1536, o, record=rec_b)
    g = gpu_build(o, K, V, 1536)
    pos = 1536
    fired_any = 0
    rec = []
    for step in [100, 200, 1, 300, 511, 700]:
        f_o = mp.cluster_update(oidx, K[:, :, pos:pos + step], V[:, :, pos:pos + step], record=rec)
        f_g = g.update(H.tdev(K[:, :, pos:pos + step], "f32"), H.tdev(V[:, :, pos:pos + step], "f32"))
        assert f_o == f_g
        fired_any += f_g
        pos += step
        assert g.n_tokens == oidx["n_tokens"] and g.n_clustered == oidx["n_clustered"]
    torch.cuda.synchronize()
    assert g.check_device_error() == 0
    assert fired_any >= 2
    ga = arrays_np(g)
    nc = oidx["n_clustered"]
    check_invariants(o, ga, K, V, nc)
    tied = set()
    for (b, h, j, X, ini, hist) in rec:
        if first_tie_iteration(hist, X, ini) < len(hist):
            tied.add(h)
    for (b, h, j), hist in rec_b.items():
        X = K[b, h, j * 1024:min(1536, (j + 1) * 1024)].astype(np.float64)
        C = -(-X.shape[0] // 16)
        init = X[mp.kmeanspp_pick(X, C, mp.stream_uniforms(13, h, j, 0, C))]
        if first_tie_iteration(hist, X, init) < len(hist):
            tied.add(h)
    for h in set(range(2)) - tied:
        for k in ("Kc", "Vc", "off"):
            np.testing.assert_array_equal(ga[k][0, h], oidx[k][0, h], err_msg=k)
        for k in ("Kp", "Vp", "perm", "assign"):
            np.testing.assert_array_equal(ga[k][0, h, :pos], oidx[k][0, h, :pos], err_msg=k)
    assert len(tied) < 2
    Q = synth.make_queries(1, 1, 8, 64, "f32", seed=4)[0]
    O_g = g.decode(H.tdev(Q, "f32"), 1 << 20)
    dense = mp.dense_attention(Q, K, V, pos, 2)
    assert np.abs(H.to_np(O_g) - dense).max() <= 1e-4
