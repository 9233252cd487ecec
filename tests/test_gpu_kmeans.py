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


# Unit roundoff of one fp32 accumulation step of the tensor cores (bf16 keys).
# Their fp32 adds are not specified as round-to-nearest; a step that truncates
# errs by up to 2^-23, and the bound takes a further factor of 2 for the
# alignment of the products inside one MMA.
U_TC = 2.0 ** -22


def tie_band(X, cents, d_terms=None, u_dot=2.0 ** -24):
    """Per-row fp32 error bound of the nearest-centroid decision.

    The kernel forms |c|^2 - 2 x.c with d-term fp32 dot products: the error of
    each distance is at most g (|c|^2 + 2 |x||c|) + u |dist|, g = d u' / (1 - d u'),
    u = 2^-24 and u' the unit of the dot products' accumulation (u for the
    fp32 SIMT path, U_TC for the tensor cores).  The oracle rounds its fp64
    distances to fp32 (error u |x - c|^2).  A row is a tie if its two nearest
    centroids are closer than the sum of these bounds for both of them.
    """
    u = 2.0 ** -24
    d = X.shape[1] if d_terms is None else d_terms
    g = d * u_dot / (1 - d * u_dot)
    cc = np.sum(cents * cents, axis=1)
    xx = np.sum(X * X, axis=1)
    dist = xx[:, None] + cc[None, :] - 2.0 * (X @ cents.T)
    top2 = np.argsort(dist, axis=1, kind="stable")[:, :2] if cents.shape[0] > 1 else np.zeros((X.shape[0], 1), int)
    nx = np.sqrt(xx)
    band = np.zeros(X.shape[0])
    for k in range(top2.shape[1]):
        c = top2[:, k]
        nc = np.sqrt(cc[c])
        kern = dist[np.arange(len(c)), c] - xx
        band += g * (cc[c] + 2 * nx * nc) + u * np.abs(kern) + u * np.abs(dist[np.arange(len(c)), c])
    return band


def band_for(X, cents):
    """tie_band of the path that assigns these keys: tensor cores for bf16, fp32 SIMT otherwise."""
    return tie_band(X, cents, u_dot=U_TC if X.dtype == np.float64 and _is_bf16(X) else 2.0 ** -24)


def _is_bf16(X):
    """True if every value of X is a bf16 number (the keys of a bf16 index)."""
    x = np.asarray(X, dtype=np.float32)
    return bool(np.all((x.view(np.uint32) & 0xFFFF) == 0))


def first_tie_iteration(hist, X, init):
    """Index of the first Lloyd iteration with a near-tie row (len(hist) if none)."""
    prev = init
    for t, h in enumerate(hist):
        if np.any(h["gap"] <= band_for(X, prev)):
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


def compare_trajectories(o, K, V, n, iters, init=None, init_mode="kmeans++"):
    """GPU builds with 1..iters Lloyd iterations against the oracle's, block by block.

    While a block's trajectories agree, every array of the block must be
    bit-exact.  A block may diverge only at an iteration where each differing
    assignment row is a tie under tie_band (both sides then hold the same
    centroids, so the band is well defined); from there on the block is
    checked through invariants only.  Returns (blocks, blocks in sync to the end).
    """
    B, Hk, Lb, T = o["B"], o["Hkv"], o["L_blk"], o["T"]
    nb = -(-n // Lb)
    C_blk = -(-Lb // T)
    in_sync = {(b, h, j): True for b in range(B) for h in range(Hk) for j in range(nb)}
    for k in range(1, iters + 1):
        ok = dict(o, iters=k)
        rec = {}
        oidx = mp.build_index(K, V, n, ok, init=init, init_mode=init_mode, record=rec)
        ga = arrays_np(gpu_build(o, K, V, n, init=init, init_mode=init_mode, iters=k))
        check_invariants(o, ga, K, V, n)
        for (b, h, j), sync in in_sync.items():
            if not sync:
                continue
            s0, e0 = j * Lb, min(n, (j + 1) * Lb)
            sl = slice(j * C_blk, (j + 1) * C_blk)
            hist = rec[(b, h, j)]
            diff = np.nonzero(ga["assign"][b, h, s0:e0] != oidx["assign"][b, h, s0:e0])[0]
            if diff.size == 0:
                for key in ("Kc", "Vc", "off"):
                    np.testing.assert_array_equal(ga[key][b, h, sl], oidx[key][b, h, sl], err_msg=f"{key} {(b, h, j, k)}")
                for key in ("perm", "Kp", "Vp"):
                    np.testing.assert_array_equal(ga[key][b, h, s0:e0], oidx[key][b, h, s0:e0],
                                                  err_msg=f"{key} {(b, h, j, k)}")
                continue
            X = K[b, h, s0:e0].astype(np.float64)
            prev = hist[k - 2]["cents"] if k >= 2 else None
            if prev is None:
                C = -(-(e0 - s0) // T)
                if init is not None:
                    prev = np.asarray(init[b, h, j * C_blk:j * C_blk + C], dtype=np.float64)
                elif init_mode == "kmeans++":
                    prev = X[mp.kmeanspp_pick(X, C, mp.stream_uniforms(o["seed"], b * Hk + h, j, 0, C))]
                else:
                    prev = X[T * np.arange(C)]
            band = band_for(X, prev)
            assert np.all(hist[k - 1]["gap"][diff] <= band[diff]), \
                f"block {(b, h, j)} iteration {k}: assignments differ outside the fp32 tie band"
            in_sync[(b, h, j)] = False
    return len(in_sync), sum(in_sync.values())


@pytest.mark.parametrize("init_mode", ["kmeans++", "stride"])
def test_tiny_f32_build_matches_oracle_trajectory(init_mode):
    """64-component mixture, one block of 2048 keys, 128 clusters, 10 Lloyd iterations."""
    w = synth.workload("tiny_f32")
    o = H.ocfg(B=1, Hkv=1, Hq=4, d=64, n_max=2048, T=16, L_blk=2048, dtype="f32", iters=10, seed=42)
    K, V, _ = synth.make_cache(1, 1, 2048, 64, w["comps"], w["sigma"], dtype="f32", seed=w["seed"])
    total, synced = compare_trajectories(o, K, V, 2048, 10, init_mode=init_mode)
    assert synced == total


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_lloyd_trajectories_from_a_given_init(dtype):
    """Given initial centroids; ragged last block; bf16 and fp32 keys."""
    o = H.ocfg(B=1, Hkv=2, Hq=8, d=128, n_max=5000, T=16, L_blk=2048, dtype=dtype, seed=3)
    K, V, lab = H.cache_for(o, 5000, comps=96, seed=21)
    n = 4500
    init = np.zeros((1, 2, 3 * 128, 128))
    rng = np.random.default_rng(0)
    for j in range(3):
        L = min(n, (j + 1) * 2048) - j * 2048
        C = -(-L // 16)
        for h in range(2):
            init[0, h, j * 128:j * 128 + C] = K[0, h, j * 2048 + rng.choice(L, size=C, replace=False)]
    total, synced = compare_trajectories(o, K, V, n, 6, init=init)
    assert synced >= total // 2


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


@pytest.mark.parametrize("aligned", [True, False])
def test_kmeanspp_seeding_on_8k_blocks(aligned):
    """512 picks over 8192 mixture keys (d 128): the seeding that skips rows
    by the triangle inequality (16-byte aligned keys) and the full-pass seeding
    (keys at an odd 2-byte offset) both give the oracle's picks, seen through
    the centroids after one Lloyd iteration."""
    o = H.ocfg(B=1, Hkv=2, Hq=8, d=128, n_max=8192, T=16, L_blk=8192, dtype="bf16", iters=1, seed=31)
    K, V, _ = H.cache_for(o, 8192, comps=512, outliers=(4, 4.0), seed=8)
    rec = {}
    oidx = mp.build_index(K, V, 8192, o, record=rec)
    g = MultipoleIndex(H.gcfg(o, init="kmeans++"))
    Kd, Vd = H.tdev(K, "bf16"), H.tdev(V, "bf16")
    if not aligned:
        buf = torch.empty(Kd.numel() + 1, dtype=torch.bfloat16, device="cuda")
        Kd = buf[1:].view(Kd.shape).copy_(Kd)
        assert Kd.data_ptr() % 16 != 0 and Kd.is_contiguous()
    g.build(Kd, Vd)
    torch.cuda.synchronize()
    assert g.check_device_error() == 0
    ga = arrays_np(g)
    for h in range(2):
        X = K[0, h].astype(np.float64)
        init = X[mp.kmeanspp_pick(X, 512, mp.stream_uniforms(31, h, 0, 0, 512))]
        # rows within the assignment's tie band may go either way; every other
        # row's slot, and the mean of every slot no such row touches, is exact
        tied = rec[(0, h, 0)][0]["gap"] <= band_for(X, init)
        assert tied.mean() < 0.01
        ag, ao = ga["assign"][0, h, :8192], oidx["assign"][0, h, :8192]
        np.testing.assert_array_equal(ag[~tied], ao[~tied])
        touched = np.zeros(512, dtype=bool)
        touched[ag[tied]] = True
        touched[ao[tied]] = True
        np.testing.assert_array_equal(ga["Kc"][0, h][~touched], oidx["Kc"][0, h][~touched])


def any_tie(hist, X, init):
    return first_tie_iteration(hist, X, init) < len(hist)


def test_hierarchical_build_matches_oracle():
    """Two levels, 1..4 iterations; a block may diverge only where its fine or coarse trajectory has a tie."""
    o = H.ocfg(B=1, Hkv=2, Hq=8, d=64, n_max=4096, T=16, L_blk=2048, levels=2, Tc=128, dtype="f32", seed=9)
    K, V, _ = H.cache_for(o, 4096, comps=48, radius=None, sigma=0.3, seed=12)
    n = 4000
    synced = {(h, j): True for h in range(2) for j in range(2)}
    for k in range(1, 5):
        rec = {}
        oidx = mp.build_index(K, V, n, dict(o, iters=k), record=rec)
        ga = arrays_np(gpu_build(o, K, V, n, iters=k))
        check_invariants(o, ga, K, V, n)
        for (h, j), ok in synced.items():
            if not ok:
                continue
            s0, e0 = j * 2048, min(n, (j + 1) * 2048)
            sl, csl = slice(j * 128, (j + 1) * 128), slice(j * 16, (j + 1) * 16)
            same = all(np.array_equal(ga[key][0, h, sl], oidx[key][0, h, sl]) for key in ("Kc", "Vc", "off")) and \
                all(np.array_equal(ga[key][0, h, csl], oidx[key][0, h, csl]) for key in ("Kcc", "Vcc", "coff")) and \
                all(np.array_equal(ga[key][0, h, s0:e0], oidx[key][0, h, s0:e0]) for key in ("perm", "Kp", "Vp"))
            if same:
                continue
            X = K[0, h, s0:e0].astype(np.float64)
            C = -(-(e0 - s0) // 16)
            init = X[mp.kmeanspp_pick(X, C, mp.stream_uniforms(9, h, j, 0, C))]
            ch = rec[(0, h, j, "coarse")]
            assert any_tie(rec[(0, h, j)], X, init) or any_tie(ch["hist"], ch["points"], ch["points"][ch["picks"]]), \
                f"block {(h, j)} differs at {k} iterations without a tie in its trajectory"
            synced[(h, j)] = False
    # the GPU-built index is a valid two-level index: dense attention when everything is selected
    g = gpu_build(o, K, V, n, iters=4)
    Q = synth.make_queries(1, 1, 8, 64, "f32", seed=5)[0]
    O = H.to_np(g.decode(H.tdev(Q, "f32"), 1 << 20, coarse_budget=1 << 20))
    assert np.abs(O - mp.dense_attention(Q, K, V, n, 2)).max() <= 1e-4
    ga = arrays_np(g)
    for h in range(2):
        coff, off = ga["coff"][0, h], ga["off"][0, h]
        assert np.all(np.diff(coff) >= 0) and coff[-1] == g.slots
        for cc in range(len(coff) - 1):                     # coarse centroid = mean of its tokens
            r0, r1 = off[coff[cc]], off[coff[cc + 1]]
            if r1 > r0:
                want = mp.round_to_dtype(ga["Kp"][0, h, r0:r1].mean(0), "f32")
                assert np.abs(ga["Kcc"][0, h, cc] - want).max() <= 1e-5 * (1 + np.abs(want).max())


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
        if any_tie(hist, X, ini):
            tied.add(h)
    for (b, h, j), hist in rec_b.items():
        X = K[b, h, j * 1024:min(1536, (j + 1) * 1024)].astype(np.float64)
        C = -(-X.shape[0] // 16)
        if any_tie(hist, X, X[mp.kmeanspp_pick(X, C, mp.stream_uniforms(13, h, j, 0, C))]):
            tied.add(h)
    for h in range(2):
        same = all(np.array_equal(ga[k][0, h], oidx[k][0, h]) for k in ("Kc", "Vc", "off")) and \
            all(np.array_equal(ga[k][0, h, :pos], oidx[k][0, h, :pos]) for k in ("Kp", "Vp", "perm", "assign"))
        assert same or h in tied, f"head {h} differs without a tie in its trajectory"
    Q = synth.make_queries(1, 1, 8, 64, "f32", seed=4)[0]
    O_g = g.decode(H.tdev(Q, "f32"), 1 << 20)
    dense = mp.dense_attention(Q, K, V, pos, 2)
    assert np.abs(H.to_np(O_g) - dense).max() <= 1e-4


# ----------------------------------------------------------------------------- one assignment step
def oracle_assign(o, Kc, K, n):
    """Oracle assignment of every key to its block's centroids: (slots, gap, band) per (b, h)."""
    Lb, T = o["L_blk"], o["T"]
    C_blk = -(-Lb // T)
    out = {}
    for b in range(o["B"]):
        for h in range(o["Hkv"]):
            a_all, gap_all, band_all = [], [], []
            for j in range(-(-n // Lb)):
                s0, e0 = j * Lb, min(n, (j + 1) * Lb)
                C = -(-(e0 - s0) // T)
                X = K[b, h, s0:e0].astype(np.float64)
                cents = Kc[b, h, j * C_blk:j * C_blk + C]
                a, gap = mp.assign_nearest(X, cents)
                a_all.append(a + j * C_blk)
                gap_all.append(gap)
                band_all.append(band_for(X, cents))
            out[(b, h)] = (np.concatenate(a_all), np.concatenate(gap_all), np.concatenate(band_all))
    return out


@pytest.mark.parametrize("dtype,d,L_blk,T,n", [
    ("bf16", 128, 8192, 16, 8192 + 3000),     # 512 centroids (two N-halves), then a ragged block of 188
    ("bf16", 128, 8192, 16, 8192 + 4200),     # ragged block of 263 centroids: a half of 7 centroids
    ("bf16", 64, 4096, 16, 2 * 4096 + 1000),  # 256 centroids: one half, chunks split over both warp groups
    ("bf16", 128, 2048, 8, 2048 + 77),        # 256 centroids; a last block of one tile with 10 centroids
    ("f32", 64, 2048, 16, 2048 + 500),        # fp32 keys: SIMT path
])
def test_assign_matches_oracle_except_ties(dtype, d, L_blk, T, n):
    """One assignment step against the index's own centroids: exact except fp32 ties."""
    o = H.ocfg(B=1, Hkv=2, Hq=4, d=d, n_max=n, T=T, L_blk=L_blk, dtype=dtype, iters=2, seed=5)
    K, V, _ = H.cache_for(o, n, comps=200, seed=8)
    g = gpu_build(o, K, V, n)
    Kd = H.tdev(K, dtype)
    a = g.assign(Kd).cpu().numpy().astype(np.int64)
    torch.cuda.synchronize()
    assert g.check_device_error() == 0
    Kc = H.to_np(g.arrays()["Kc"])
    want = oracle_assign(o, Kc, K, n)
    for (b, h), (ao, gap, band) in want.items():
        diff = np.nonzero(a[b, h] != ao)[0]
        assert np.all(gap[diff] <= band[diff]), f"unit {(b, h)}: {diff.size} rows differ outside the tie band"
        assert diff.size <= max(2, n // 1000)


@pytest.mark.parametrize("d,L_blk,n", [(128, 8192, 8192 + 2100), (64, 4096, 4096 + 600)])
def test_assign_duplicate_centroids_take_lower_slot(d, L_blk, n):
    """Bit-identical centroids give bit-identical distances: the lower slot must win.

    Duplicates are placed within one interleaved chain, across chains, across
    32-column chunks and across the two N-halves of a 512-centroid block; the
    keys are copies of centroids, so each key's nearest centroid is its own
    (distance 0) or an exact duplicate of it.
    """
    o = H.ocfg(B=1, Hkv=2, Hq=4, d=d, n_max=n, T=16, L_blk=L_blk, dtype="bf16", iters=1, seed=6)
    K, V, _ = H.cache_for(o, n, comps=100, seed=9)
    g = gpu_build(o, K, V, n)
    C_blk = L_blk // 16
    rng = np.random.default_rng(3)
    Kc = rng.standard_normal((1, 2, g.slots, d))
    Kc = np.asarray(torch.from_numpy(Kc).to(torch.bfloat16).float().numpy(), dtype=np.float64)
    pairs = [(0, 4), (1, 2), (3, 35), (40, 200), (7, 255), (8, 100)]
    if C_blk == 512:
        pairs += [(10, 256), (255, 256), (300, 301), (260, 511), (5, 500)]
    for j in range(-(-n // L_blk)):
        C = -(-(min(n, (j + 1) * L_blk) - j * L_blk) // 16)
        for p1, p2 in pairs:
            if p2 < C:
                Kc[:, :, j * C_blk + p2] = Kc[:, :, j * C_blk + p1]
    Kq = np.zeros((1, 2, n, d))
    for j in range(-(-n // L_blk)):
        s0, e0 = j * L_blk, min(n, (j + 1) * L_blk)
        C = -(-(e0 - s0) // 16)
        pick = rng.integers(0, C, size=e0 - s0)
        for p1, p2 in pairs:                    # every duplicate pair gets keys
            if p2 < C:
                pick[rng.integers(0, e0 - s0, size=4)] = p2
        Kq[:, :, s0:e0] = Kc[:, :, j * C_blk + pick]
    arr = g.arrays()
    arr["Kc"].copy_(H.tdev(Kc, "bf16"))
    a = g.assign(H.tdev(Kq, "bf16")).cpu().numpy().astype(np.int64)
    want = oracle_assign(o, Kc, Kq, n)
    for (b, h), (ao, _, _) in want.items():
        np.testing.assert_array_equal(a[b, h], ao)


def test_online_update_bf16_matches_oracle():
    """The online update with bf16 keys, d 128 and 4 query heads per KV head:
    re-clustering of the open 2048-token block assigns on the tensor cores from
    the update's block buffer.  One Lloyd iteration per (re-)clustering, and
    the whole index is compared after the build and after every update call:
    while a head's state equals the oracle's, both sides start each trigger
    from identical centroids, so the head may diverge only in rows inside the
    fp32 tie band of those centroids; from then on it is retired.  Decoding with
    every cluster selected is dense attention."""
    o = H.ocfg(B=1, Hkv=2, Hq=8, d=128, n_max=8192, T=16, L_blk=2048, update_interval=512, dtype="bf16",
               iters=1, seed=23)
    K, V, _ = H.cache_for(o, 8192, comps=128, outliers=(4, 4.0), seed=24)
    keys = ("Kc", "Vc", "off", "Kp", "Vp", "perm", "assign")

    def same_head(ga, h, n):
        return all(np.array_equal(ga[k][0, h], oidx[k][0, h]) for k in ("Kc", "Vc", "off")) and \
            all(np.array_equal(ga[k][0, h, :n], oidx[k][0, h, :n]) for k in ("Kp", "Vp", "perm", "assign"))

    def explained(ga, h, records, n):
        """Every differing assignment of head h lies in a block re-clustered now, inside the tie band."""
        diff = np.nonzero(ga["assign"][0, h, :n] != oidx["assign"][0, h, :n])[0]
        if diff.size == 0:
            return False
        for (b, hh, j, X, ini, hist) in records:
            if hh != h:
                continue
            rows = diff[(diff >= j * 2048) & (diff < j * 2048 + X.shape[0])] - j * 2048
            band = band_for(X, ini)
            if not np.all(hist[0]["gap"][rows] <= band[rows]):
                return False
            diff = np.setdiff1d(diff, rows + j * 2048)
        return diff.size == 0

    prompt = 3000
    rec_b = {}
    oidx = mp.build_index(K, V, prompt, o, record=rec_b)
    g = gpu_build(o, K, V, prompt)
    ga = arrays_np(g)
    live = set()
    for h in range(2):
        if same_head(ga, h, prompt):
            live.add(h)
        else:
            recs = []
            for j in range(2):
                X = K[0, h, j * 2048:min(prompt, (j + 1) * 2048)].astype(np.float64)
                C = -(-X.shape[0] // 16)
                recs.append((0, h, j, X, X[mp.kmeanspp_pick(X, C, mp.stream_uniforms(23, h, j, 0, C))],
                             rec_b[(0, h, j)]))
            assert explained(ga, h, recs, prompt), f"head {h} differs after the build outside the tie band"
    pos = prompt
    fired = compared = 0
    for step in [300, 212, 1, 1000, 600, 2000]:
        rec = []
        f_o = mp.cluster_update(oidx, K[:, :, pos:pos + step], V[:, :, pos:pos + step], record=rec)
        f_g = g.update(H.tdev(K[:, :, pos:pos + step], "bf16"), H.tdev(V[:, :, pos:pos + step], "bf16"))
        assert f_o == f_g
        fired += f_g
        pos += step
        assert g.n_tokens == oidx["n_tokens"] and g.n_clustered == oidx["n_clustered"]
        torch.cuda.synchronize()
        ga = arrays_np(g)
        for h in sorted(live):
            if same_head(ga, h, pos):
                compared += f_g
                continue
            assert f_g and explained(ga, h, rec, pos), f"head {h} differs after an update outside the tie band"
            live.discard(h)
    assert g.check_device_error() == 0
    assert fired >= 3
    assert compared >= 2, "fewer than two re-clusterings were compared bit for bit"
    check_invariants(o, ga, K, V, oidx["n_clustered"])
    Q = synth.make_queries(1, 1, 8, 128, "bf16", seed=4)[0]
    O_g = H.to_np(g.decode(H.tdev(Q, "bf16"), 1 << 20))
    assert np.abs(O_g - mp.dense_attention(Q, K, V, pos, 2)).max() <= H.TOL["bf16"]


def test_full_size_build_sampled_blocks():
    """The default bench workload's build at full size: batch 16 x 8 KV heads x
    32768 tokens, 4 blocks of 8192 keys per head, 512 centroids per block, 10
    Lloyd iterations from k-means++ seeds, bf16 keys (tensor-core assignment).
    Eight sampled (unit, block) pairs follow the oracle's trajectory: the GPU
    builds with 1 .. 10 iterations match it bit for bit (assignment,
    centroids, offsets) until an iteration in which every differing row lies
    inside the fp32 tie band of the centroids both sides then hold.  The
    sampled heads also satisfy the index invariants."""
    w = synth.workload("batch16_32k_sparse95")
    B, Hk, n, d, Lb, T = w["B"], w["Hkv"], w["n"], w["d"], w["L_blk"], w["T"]
    o = H.ocfg(B=B, Hkv=Hk, Hq=w["Hq"], d=d, n_max=n, T=T, L_blk=Lb, iters=w["iters"], dtype="bf16", seed=w["seed"])
    K, V, _ = synth.make_cache(B, Hk, n, d, w["comps"], w["sigma"], radius=w["radius"], outliers=w["outliers"],
                               dtype="bf16", seed=w["seed"])
    Kd, Vd = H.tdev(K, "bf16"), H.tdev(V, "bf16")
    C = Lb // T
    samples = [(0, 0, 0), (1, 3, 2), (5, 7, 1), (7, 2, 3), (9, 5, 0), (12, 1, 2), (14, 6, 3), (15, 4, 1)]
    traj = {}
    for (b, h, j) in samples:
        X = K[b, h, j * Lb:(j + 1) * Lb].astype(np.float64)
        init = X[mp.kmeanspp_pick(X, C, mp.stream_uniforms(w["seed"], b * Hk + h, j, 0, C))]
        _, _, hist = mp.lloyd(X, init, w["iters"], "bf16")
        traj[(b, h, j)] = (X, init, hist)
    following = set(samples)
    exact_to_end = 0
    for k in range(1, w["iters"] + 1):
        g = MultipoleIndex(H.gcfg(dict(o, iters=k)))
        g.build(Kd, Vd)
        torch.cuda.synchronize()
        assert g.check_device_error() == 0
        arr = g.arrays()
        for (b, h, j) in sorted(following):
            X, init, hist = traj[(b, h, j)]
            sl = slice(j * C, (j + 1) * C)
            a_g = arr["assign"][b, h, j * Lb:(j + 1) * Lb].cpu().numpy().astype(np.int64) - j * C
            a_o = hist[k - 1]["assign"]
            diff = np.nonzero(a_g != a_o)[0]
            if diff.size == 0:
                np.testing.assert_array_equal(H.to_np(arr["Kc"][b, h, sl]), hist[k - 1]["cents"],
                                              err_msg=f"Kc {(b, h, j, k)}")
                off = arr["off"][b, h, j * C:(j + 1) * C + 1].cpu().numpy().astype(np.int64)
                np.testing.assert_array_equal(np.diff(off), np.bincount(a_o, minlength=C), err_msg=f"off {(b, h, j, k)}")
                if k == w["iters"]:
                    exact_to_end += 1
                continue
            prev = hist[k - 2]["cents"] if k >= 2 else init
            band = band_for(X, prev)
            assert np.all(hist[k - 1]["gap"][diff] <= band[diff]), \
                f"block {(b, h, j)} iteration {k}: assignments differ outside the fp32 tie band"
            following.discard((b, h, j))
        if k == w["iters"]:
            ga = {key: arr[key][[s[0] for s in samples], [s[1] for s in samples]] for key in ("Kc", "Vc", "off", "Kp", "Vp", "perm", "assign")}
            ga = {key: (H.to_np(v) if v.dtype in (torch.bfloat16, torch.float32) else v.cpu().numpy().astype(np.int64))[:, None]
                  for key, v in ga.items()}
            Ks = np.stack([K[b, h] for (b, h, _) in samples])[:, None]
            Vs = np.stack([V[b, h] for (b, h, _) in samples])[:, None]
            check_invariants(dict(o, B=len(samples), Hkv=1), ga, Ks, Vs, n)
        del g, arr
    assert exact_to_end >= 1, "no sampled block stayed bit-exact through all iterations"
