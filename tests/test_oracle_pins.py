"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Closed forms (dense softmax attention through torch's fp64 SDPA), a hand-worked
example, brute force on tiny inputs, invariants of Lloyd's algorithm and of
the cluster-ordered store, and published splitmix64 outputs.  CPU only.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import brute
from clustered_sparse_decode_b200 import synth
from oracle import multipole as mp

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def ocfg(B=1, Hkv=1, Hq=4, d=16, n_max=256, T=4, L_blk=64, levels=1, Tc=16, iters=6,
         update_interval=32, dtype="f32", seed=5):
    return dict(B=B, Hkv=Hkv, Hq=Hq, d=d, n_max=n_max, T=T, L_blk=L_blk, levels=levels, Tc=Tc,
                iters=iters, update_interval=update_interval, dtype=dtype, seed=seed)


def cache(cfg, n, comps=8, sigma=0.3, seed=0, radius=None):
    K, V, lab = synth.make_cache(cfg["B"], cfg["Hkv"], n, cfg["d"], comps, sigma, radius=radius,
                                 dtype=cfg["dtype"], seed=seed)
    return K, V, lab


def sdpa(Q, K, V, n, Hkv, scale=None, mask=None):
    """Dense softmax attention via torch (fp64, CPU), GQA by repeating KV heads."""
    q = torch.tensor(np.asarray(Q, dtype=np.float64))[:, :, None, :]       # [B, Hq, 1, d]
    G = q.shape[1] // Hkv
    k = torch.tensor(np.asarray(K[:, :, :n], dtype=np.float64)).repeat_interleave(G, dim=1)
    v = torch.tensor(np.asarray(V[:, :, :n], dtype=np.float64)).repeat_interleave(G, dim=1)
    am = None if mask is None else torch.tensor(mask)[:, :, None, :]
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=am, scale=scale)
    return o[:, :, 0, :].numpy()


# --------------------------------------------------------------------------- RNG / rounding

def test_splitmix64_published_outputs():
    vals = [int(l) for l in open(os.path.join(GOLD, "splitmix64_seed1234567.txt")) if l.strip()
            and not l.startswith("#")]
    assert [mp.splitmix64_output(1234567, k) for k in range(len(vals))] == vals


def test_bf16_rounding_matches_torch_on_f32_inputs():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(20000) * 10 ** rng.uniform(-30, 30, 20000),
                        [0.0, 1.0, -1.0, 1.00390625, 1.01171875]]).astype(np.float32)
    want = torch.tensor(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(mp.round_to_dtype(x.astype(np.float64), "bf16"), want)


def test_bf16_rounding_from_f64_does_not_round_twice():
    # 1 + 2^-8 is the halfway point between bf16 neighbours 1 and 1 + 2^-7: ties to even -> 1.
    assert mp.round_to_dtype(np.array([1 + 2 ** -8]), "bf16")[0] == 1.0
    # a hair above halfway rounds up, even though an fp32 intermediate would first round to
    # the halfway value and then to even (down)
    assert mp.round_to_dtype(np.array([1 + 2 ** -8 + 2 ** -40]), "bf16")[0] == 1 + 2 ** -7
    assert mp.round_to_dtype(np.array([-(1 + 3 * 2 ** -8)]), "bf16")[0] == -(1 + 2 * 2 ** -7)
    assert mp.round_to_dtype(np.array([3.5e38]), "bf16")[0] == np.inf


# --------------------------------------------------------------------------- selection / assignment

@pytest.mark.parametrize("seed", range(20))
def test_selection_equals_brute_force(seed):
    rng = np.random.default_rng(seed)
    C = int(rng.integers(1, 40))
    scores = np.round(rng.standard_normal(C), 1)          # rounding forces exact ties
    counts = rng.integers(0, 6, size=C)
    for budget in [0, 1, 3, 7, 20, 1000]:
        sel, _ = mp.select_clusters(scores, counts, budget)
        assert list(sel) == brute.select(list(scores), list(counts), budget)


@pytest.mark.parametrize("seed", range(10))
def test_assignment_equals_brute_force(seed):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((30, 5))
    cents = rng.standard_normal((7, 5))
    cents[3] = cents[1]                                    # an exact tie: lower index wins
    a, _ = mp.assign_nearest(X, cents)
    assert list(a) == brute.assign(X.tolist(), cents.tolist())


@pytest.mark.parametrize("seed", range(6))
def test_kmeanspp_equals_brute_force(seed):
    rng = np.random.default_rng(seed)
    X = np.round(rng.standard_normal((40, 3)), 2)
    X[5] = X[9]                                            # duplicate points
    u = rng.uniform(size=12).tolist()
    assert mp.kmeanspp_pick(X, 12, u) == brute.kmeanspp(X.tolist(), 12, u)


# --------------------------------------------------------------------------- decode closed forms

def test_hand_worked_example():
    g = json.load(open(os.path.join(GOLD, "hand_worked_decode.json")))
    cfg = ocfg(d=2, Hq=1, n_max=6, T=2, L_blk=6)
    K = np.array(g["keys"], dtype=np.float32)[None, None]
    V = np.array(g["values"], dtype=np.float32)[None, None]
    a = np.array(g["assignment"])[None, None]
    idx = mp.index_from_assignment(K, V, 6, cfg, a)
    Q = np.array(g["query"], dtype=np.float32)[None, None]
    for case in g["cases"]:
        info = {}
        O = mp.decode(idx, Q, case["budget"], flags=mp.NO_APPROX if case["no_approx"] else 0,
                      scale=1.0, info=info)
        np.testing.assert_allclose(O[0, 0], case["expected"], rtol=1e-6)
        assert sorted(info[(0, 0)]["sel"].tolist()) == case["selected"]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("levels", [1, 2])
def test_budget_covering_everything_is_dense_attention(dtype, levels):
    """P1: budget >= n selects every cluster, so the step is dense softmax attention."""
    cfg = ocfg(B=2, Hkv=2, Hq=6, n_max=200, levels=levels, dtype=dtype)
    n = 200
    K, V, _ = cache(cfg, n)
    idx = mp.build_index(K, V, n, cfg)
    Q = synth.make_queries(1, 2, 6, cfg["d"], dtype, seed=3)[0]
    O = mp.decode(idx, Q, budget=n, coarse_budget=n)
    np.testing.assert_allclose(O, sdpa(Q, K, V, n, 2), atol=1e-12)


@pytest.mark.parametrize("budget", [1, 5, 40, 255])
def test_singleton_clusters_make_the_approximation_exact(budget):
    """P2: with one token per centroid, every centroid term equals its token's exact term."""
    cfg = ocfg(T=1, n_max=128, L_blk=64, iters=2)
    K, V, _ = cache(cfg, 128)
    idx = mp.build_index(K, V, 128, cfg)
    Q = synth.make_queries(1, 1, 4, cfg["d"], "f32", seed=4)[0]
    np.testing.assert_allclose(mp.decode(idx, Q, budget), sdpa(Q, K, V, 128, 1), atol=1e-6)


@pytest.mark.parametrize("budget", [0, 3, 17, 60])
def test_clusters_of_identical_keys_make_the_approximation_exact(budget):
    """P4: if all keys of a cluster coincide, n e^{q.Kc} Vc equals the sum of its exact terms."""
    cfg = ocfg(T=4, n_max=96, L_blk=96)
    rng = np.random.default_rng(1)
    protos = rng.standard_normal((24, cfg["d"])).astype(np.float32)
    a = rng.integers(0, 24, size=96)
    K = protos[a][None, None]
    V = rng.standard_normal((1, 1, 96, cfg["d"])).astype(np.float32)
    idx = mp.index_from_assignment(K, V, 96, cfg, a[None, None])
    Q = synth.make_queries(1, 1, 4, cfg["d"], "f32", seed=2)[0]
    np.testing.assert_allclose(mp.decode(idx, Q, budget), sdpa(Q, K, V, 96, 1), atol=1e-6)


def test_no_approx_is_dense_attention_over_the_selected_tokens():
    """P11: dropping centroid terms = softmax restricted to selected (and tail) tokens."""
    cfg = ocfg(B=1, Hkv=2, Hq=4, n_max=160)
    K, V, _ = cache(cfg, 160)
    idx = mp.build_index(K, V, 160, cfg)
    Q = synth.make_queries(1, 1, 4, cfg["d"], "f32", seed=9)[0]
    np.testing.assert_allclose(mp.decode(idx, Q, 160, flags=mp.NO_APPROX), sdpa(Q, K, V, 160, 2),
                               atol=1e-12)
    info = {}
    O = mp.decode(idx, Q, 25, flags=mp.NO_APPROX, info=info)
    mask = np.zeros((1, 4, 160), dtype=bool)
    for h in range(2):
        off = idx["off"][0, h]
        for c in info[(0, h)]["sel"]:
            ids = idx["perm"][0, h, off[c]:off[c + 1]]
            mask[0, 2 * h:2 * h + 2, ids] = True
    np.testing.assert_allclose(O, sdpa(Q, K, V, 160, 2, mask=mask), atol=1e-12)


def test_decode_equals_brute_force_on_tiny_index():
    cfg = ocfg(B=1, Hkv=1, Hq=2, d=6, n_max=40, T=4, L_blk=40)
    K, V, _ = cache(cfg, 40, comps=3)
    idx = mp.build_index(K, V, 40, cfg)
    Q = synth.make_queries(1, 1, 2, 6, "f32", seed=5)[0]
    scale = 1 / math.sqrt(6)
    off = idx["off"][0, 0]
    clusters = []
    for c in range(len(off) - 1):
        rows = range(off[c], off[c + 1])
        clusters.append(([idx["Kp"][0, 0, r].tolist() for r in rows], [idx["Vp"][0, 0, r].tolist() for r in rows],
                         idx["Kc"][0, 0, c].tolist(), idx["Vc"][0, 0, c].tolist()))
    counts = [len(c[0]) for c in clusters]
    for budget in [1, 6, 13, 40]:
        O = mp.decode(idx, Q, budget)
        S = [[scale * math.fsum(a * b for a, b in zip(Q[0, g], cl[2])) for cl in clusters] for g in range(2)]
        shat = [max(S[0][c], S[1][c]) for c in range(len(clusters))]
        sel = brute.select(shat, counts, budget)
        for g in range(2):
            want = brute.decode_one(Q[0, g].tolist(), scale, clusters, set(sel))
            np.testing.assert_allclose(O[0, g], want, atol=1e-12)


def test_large_logits_are_safe_and_select_the_top_term():
    """P12: q x 1e3 gives no overflow; dense result matches SDPA and is the top key's value."""
    cfg = ocfg(n_max=128)
    K, V, _ = cache(cfg, 128)
    idx = mp.build_index(K, V, 128, cfg)
    Q = synth.make_queries(1, 1, 4, cfg["d"], "f32", seed=1, scale=1e3)[0]
    O = mp.decode(idx, Q, 128)
    assert np.isfinite(O).all()
    ref = sdpa(Q, K, V, 128, 1)
    np.testing.assert_allclose(O, ref, atol=1e-9)
    z = (K[0, 0].astype(np.float64) @ Q[0].T.astype(np.float64)) / 4.0      # [n, G]
    top = np.argmax(z, axis=0)
    srt = np.sort(z, axis=0)
    for g in range(4):
        if srt[-1, g] - srt[-2, g] > 50:
            np.testing.assert_allclose(O[0, g], V[0, 0, top[g]], atol=1e-12)
    assert np.isfinite(mp.decode(idx, Q, 5)).all()


# --------------------------------------------------------------------------- clustering invariants

def test_lloyd_objective_never_increases_and_centroids_are_member_means():
    cfg = ocfg(d=8, n_max=512, T=8, L_blk=512, iters=8)
    K, V, _ = cache(cfg, 512, comps=20, sigma=0.5)
    rec = {}
    idx = mp.build_index(K, V, 512, cfg, record=rec)
    X = K[0, 0].astype(np.float64)
    hist = rec[(0, 0, 0)]
    obj = []
    for t, h in enumerate(hist):
        # objective of the assignment of iteration t against the centroids it produced
        obj.append(np.sum((X - h["cents"][h["assign"]]) ** 2))
    assert all(obj[i + 1] <= obj[i] * (1 + 1e-6) for i in range(len(obj) - 1))
    # each non-empty centroid is the member mean to within half an fp32 ulp (P3),
    # checked with torch's index_add (a different summation route)
    a = torch.tensor(hist[-1]["assign"])
    np.testing.assert_array_equal(idx["assign"][0, 0, :512], hist[-1]["assign"])
    sums = torch.zeros(64, 8, dtype=torch.float64).index_add_(0, a, torch.tensor(X))
    cnt = torch.bincount(a, minlength=64).double()
    nz = cnt > 0
    mean = (sums[nz] / cnt[nz, None]).numpy()
    Kc = idx["Kc"][0, 0, :64][nz.numpy()]
    assert np.all(np.abs(Kc - mean) <= 0.5 * np.spacing(np.abs(mean).astype(np.float32)) + 1e-300)


def test_well_separated_mixture_is_recovered():
    """P7: tight, far-apart components with init at the true means are found exactly."""
    rng = np.random.default_rng(3)
    C, d, L = 16, 12, 256
    mu = rng.standard_normal((C, d)) * 5
    lab = rng.integers(0, C, size=L)
    lab[:C] = np.arange(C)
    X = (mu[lab] + 0.01 * rng.standard_normal((L, d))).astype(np.float32).astype(np.float64)
    init = mp.round_to_dtype(mu, "f32")
    a, cents, _ = mp.lloyd(X, init, 5, "f32")
    np.testing.assert_array_equal(a, lab)
    np.testing.assert_allclose(cents, mu, atol=0.02)


@pytest.mark.parametrize("levels", [1, 2])
def test_store_is_a_permutation_with_cluster_runs(levels):
    """P8: the store holds every token once; run c holds exactly the tokens assigned to c."""
    cfg = ocfg(B=1, Hkv=2, n_max=300, L_blk=128, T=8, Tc=32, levels=levels)
    n = 300
    K, V, _ = cache(cfg, n)
    idx = mp.build_index(K, V, n, cfg)
    for h in range(2):
        perm = idx["perm"][0, h, :n]
        assert sorted(perm.tolist()) == list(range(n))
        np.testing.assert_array_equal(idx["Kp"][0, h, :n], K[0, h, perm])
        np.testing.assert_array_equal(idx["Vp"][0, h, :n], V[0, h, perm])
        off = idx["off"][0, h]
        assert np.all(np.diff(off) >= 0) and off[-1] == n
        for c in range(len(off) - 1):
            ids = perm[off[c]:off[c + 1]]
            np.testing.assert_array_equal(idx["assign"][0, h, ids], c)
            assert np.all(np.diff(ids) > 0)               # token order inside a run
        # blocks keep their tokens
        for j in range(3):
            s, e = j * 128, min(n, (j + 1) * 128)
            assert sorted(perm[s:e].tolist()) == list(range(s, e))
        if levels == 2:
            coff = idx["coff"][0, h]
            assert np.all(np.diff(coff) >= 0) and coff[-1] == len(off) - 1


def test_hierarchy_with_unbounded_coarse_budget_is_flat_decode():
    """P9: selecting every coarse cluster reduces the two-level step to the flat one."""
    cfg = ocfg(B=1, Hkv=2, Hq=4, n_max=256, L_blk=128, T=4, Tc=16, levels=2)
    K, V, _ = cache(cfg, 256)
    idx = mp.build_index(K, V, 256, cfg)
    flat = dict(idx)
    flat["cfg"] = dict(idx["cfg"], levels=1)
    Q = synth.make_queries(1, 1, 4, cfg["d"], "f32", seed=8)[0]
    for budget in [1, 10, 50]:
        np.testing.assert_allclose(mp.decode(idx, Q, budget, coarse_budget=256),
                                   mp.decode(flat, Q, budget), atol=1e-12)


def test_block_sized_updates_equal_a_fresh_stride_seeded_build():
    """P10: appending whole blocks triggers clustering from stride seeds, as a fresh build does."""
    cfg = ocfg(B=1, Hkv=2, n_max=256, L_blk=64, T=4, update_interval=32)
    K, V, _ = cache(cfg, 256)
    fresh = mp.build_index(K, V, 256, cfg, init_mode="stride")
    inc = mp.build_index(K, V, 0, cfg)
    for s in range(0, 256, 64):
        assert mp.cluster_update(inc, K[:, :, s:s + 64], V[:, :, s:s + 64])
    for key in ("Kc", "Vc", "off", "Kp", "Vp", "perm", "assign"):
        np.testing.assert_array_equal(inc[key], fresh[key])


def test_tail_tokens_are_attended_exactly():
    """R6: with budget >= clustered tokens, a step with an unclustered tail is dense attention."""
    cfg = ocfg(B=1, Hkv=1, n_max=256, L_blk=64, T=4, update_interval=48)
    K, V, _ = cache(cfg, 256)
    idx = mp.build_index(K, V, 128, cfg)
    assert not mp.cluster_update(idx, K[:, :, 128:150], V[:, :, 128:150])
    assert idx["n_clustered"] == 128 and idx["n_tokens"] == 150
    Q = synth.make_queries(1, 1, 4, cfg["d"], "f32", seed=6)[0]
    np.testing.assert_allclose(mp.decode(idx, Q, 128), sdpa(Q, K, V, 150, 1), atol=1e-12)
    # the update fires once the tail reaches the interval, re-clustering block 2 only
    frozen = idx["Kp"][0, 0, :128].copy()
    assert mp.cluster_update(idx, K[:, :, 150:180], V[:, :, 150:180])
    assert idx["n_clustered"] == 180
    np.testing.assert_array_equal(idx["Kp"][0, 0, :128], frozen)
    np.testing.assert_allclose(mp.decode(idx, Q, 180), sdpa(Q, K, V, 180, 1), atol=1e-12)


@pytest.mark.parametrize("budget,coarse_budget", [(1, 1), (5, 20), (30, 8), (96, 96)])
def test_hierarchy_with_identical_keys_per_coarse_cluster_is_exact(budget, coarse_budget):
    """P4 for two levels: coarse and fine centroid terms are exact when their keys coincide."""
    cfg = ocfg(T=4, Tc=8, n_max=96, L_blk=96, levels=2)
    rng = np.random.default_rng(7)
    protos = rng.standard_normal((12, cfg["d"])).astype(np.float32)
    p = rng.integers(0, 12, size=96)
    fine = 2 * p + rng.integers(0, 2, size=96)              # two fine clusters per prototype
    coarse = np.arange(24) // 2                              # fine slot -> its prototype
    K = protos[p][None, None]
    V = rng.standard_normal((1, 1, 96, cfg["d"])).astype(np.float32)
    idx = mp.index_from_assignment(K, V, 96, cfg, fine[None, None], coarse[None, None])
    Q = synth.make_queries(1, 1, 4, cfg["d"], "f32", seed=12)[0]
    info = {}
    O = mp.decode(idx, Q, budget, coarse_budget=coarse_budget, info=info)
    np.testing.assert_allclose(O, sdpa(Q, K, V, 96, 1), atol=1e-6)
    # and the coarse terms are really used: without them the result changes
    if len(info[(0, 0)]["csel"]) < 12:
        assert np.abs(mp.decode(idx, Q, budget, coarse_budget, flags=mp.NO_APPROX)
                      - O).max() > 1e-3


def test_coarse_centroids_are_means_of_their_tokens():
    cfg = ocfg(B=1, Hkv=1, n_max=256, L_blk=128, T=4, Tc=16, levels=2)
    K, V, _ = cache(cfg, 256)
    idx = mp.build_index(K, V, 256, cfg)
    off, coff = idx["off"][0, 0], idx["coff"][0, 0]
    for cc in range(len(coff) - 1):
        a0, a1 = off[coff[cc]], off[coff[cc + 1]]
        if a1 == a0:
            continue
        ids = idx["perm"][0, 0, a0:a1]
        mean_k = torch.tensor(K[0, 0, ids], dtype=torch.float64).mean(0).numpy()
        mean_v = torch.tensor(V[0, 0, ids], dtype=torch.float64).mean(0).numpy()
        tol = 0.5 * np.spacing(np.abs(mean_k).astype(np.float32))
        assert np.all(np.abs(idx["Kcc"][0, 0, cc] - mean_k) <= tol)
        tolv = 0.5 * np.spacing(np.abs(mean_v).astype(np.float32))
        assert np.all(np.abs(idx["Vcc"][0, 0, cc] - mean_v) <= tolv)


@pytest.mark.parametrize("levels", [1, 2])
def test_output_is_affine_in_the_values(levels):
    """Softmax weights sum to one and depend on keys only, and centroids are
    member means: values a*V + b give outputs a*O + b, selection unchanged, for
    every budget (exact and centroid terms, flat and two-level)."""
    cfg = ocfg(B=1, Hkv=2, Hq=4, n_max=256, L_blk=128, T=4, Tc=16, levels=levels)
    K, V, _ = cache(cfg, 256)
    a, b = 2.0, 0.5 * np.linspace(-1.0, 1.0, cfg["d"])
    V2 = a * V + b
    idx1 = mp.build_index(K, V, 256, cfg)
    idx2 = mp.build_index(K, V2, 256, cfg)
    Q = synth.make_queries(1, 1, 4, cfg["d"], "f32", seed=13)[0]
    for budget, cb in [(1, 8), (20, 40), (100, 120), (256, 256)]:
        i1, i2 = {}, {}
        O1 = mp.decode(idx1, Q, budget, coarse_budget=cb, info=i1)
        O2 = mp.decode(idx2, Q, budget, coarse_budget=cb, info=i2)
        for u in i1:
            np.testing.assert_array_equal(i1[u]["sel"], i2[u]["sel"])
        np.testing.assert_allclose(O2, a * O1 + b, atol=1e-6)


# --------------------------------------------------------------------------- online update, warm start (R14)

def _frac_rows(rows):
    from fractions import Fraction
    return np.array([[float(Fraction(x)) for x in r] for r in rows])


def _run_warm_start_case(block_init=None):
    """The hand-worked update of tests/golden/warm_start_update.json through the oracle."""
    g = json.load(open(os.path.join(GOLD, "warm_start_update.json")))
    c = g["config"]
    cfg = ocfg(B=c["B"], Hkv=c["Hkv"], Hq=c["Hq"], d=c["d"], n_max=c["n_max"], T=c["T"], L_blk=c["L_blk"],
               iters=c["iters"], update_interval=c["update_interval"], dtype=c["dtype"])
    K = np.array(g["keys"], dtype=np.float64)[None, None]
    V = np.array(g["values"], dtype=np.float64)[None, None]
    orig = mp._block_init
    if block_init is not None:
        mp._block_init = block_init
    try:
        idx = mp.build_index(K, V, 4, cfg, init_mode="stride")
        built = idx["Kc"][0, 0, :2].copy()
        rec = []
        fired = mp.cluster_update(idx, K[:, :, 4:], V[:, :, 4:], record=rec)
    finally:
        mp._block_init = orig
    return g["expected"], built, fired, rec, idx


def _matches_warm_start_golden(exp, built, fired, rec, idx):
    f32 = lambda a: np.asarray(a, dtype=np.float64).astype(np.float32)
    if not fired or len(rec) != 1:
        return False
    b, h, j, _, ini, hist = rec[0]
    return bool((b, h, j) == (0, 0, 0)
                and np.array_equal(f32(built), f32(_frac_rows(exp["build_Kc"])))
                and np.array_equal(f32(ini), f32(_frac_rows(exp["update_init"])))
                and np.array_equal(hist[0]["assign"], exp["update_assign"])
                and np.array_equal(f32(idx["Kc"][0, 0]), f32(_frac_rows(exp["Kc"])))
                and np.array_equal(f32(idx["Vc"][0, 0]), f32(_frac_rows(exp["Vc"])))
                and np.array_equal(idx["off"][0, 0], exp["off"])
                and np.array_equal(idx["perm"][0, 0], exp["perm"])
                and idx["n_clustered"] == 8)


def test_warm_start_update_matches_the_hand_worked_case():
    """R14 with a non-empty previous block: old centroids keep their slots, new
    slots start at the new tokens' keys at stride T (hand-worked golden)."""
    assert _matches_warm_start_golden(*_run_warm_start_case())


def _slip(kind):
    """A copy of the oracle's block init with one planted mistake in its warm start."""
    orig = mp._block_init

    def init(idx, b, h, j, X, L_old, init_mode, unit, init_given):
        if init_mode != "warm" or L_old == 0:
            return orig(idx, b, h, j, X, L_old, init_mode, unit, init_given)
        T = idx["cfg"]["T"]
        C, C_old = -(-X.shape[0] // T), -(-L_old // T)
        s0 = j * idx["geom"]["C_blk"]
        warm = idx["Kc"][b, h, s0:s0 + C_old].copy()
        if kind == "stride_from_block_start":
            return np.concatenate([warm, X[T * np.arange(C - C_old)]])
        if kind == "old_slots_reseeded":
            return X[T * np.arange(C)]
        if kind == "stride_one":
            return np.concatenate([warm, X[L_old + np.arange(C - C_old)]])
        if kind == "warm_after_new":
            return np.concatenate([X[L_old + T * np.arange(C - C_old)], warm])
        raise ValueError(kind)
    return init


@pytest.mark.parametrize("kind", ["stride_from_block_start", "old_slots_reseeded", "stride_one", "warm_after_new"])
def test_planted_warm_start_slips_fail_the_hand_worked_case(kind):
    """Each plausible mistake in the warm start, planted in the oracle, fails the golden case."""
    assert not _matches_warm_start_golden(*_run_warm_start_case(_slip(kind)))


# --------------------------------------------------------------------------- dense attention checker

@pytest.mark.parametrize("Hkv,Hq", [(2, 2), (2, 8), (3, 12)])
def test_dense_attention_equals_torch_sdpa(Hkv, Hq):
    """The dense checker (GQA: query head g reads KV head g // G) against torch's
    fp64 SDPA over the first n of more keys; keys, values and queries per head differ."""
    rng = np.random.default_rng(Hq)
    B, n_all, n, d = 2, 40, 33, 16
    K = rng.standard_normal((B, Hkv, n_all, d))
    V = rng.standard_normal((B, Hkv, n_all, d))
    Q = 2.0 * rng.standard_normal((B, Hq, d))
    np.testing.assert_allclose(mp.dense_attention(Q, K, V, n, Hkv), sdpa(Q, K, V, n, Hkv), atol=1e-12)
    np.testing.assert_allclose(mp.dense_attention(Q, K, V, n, Hkv, scale=0.3), sdpa(Q, K, V, n, Hkv, scale=0.3),
                               atol=1e-12)


# --------------------------------------------------------------------------- forced selections

@pytest.mark.parametrize("levels", [1, 2])
def test_forcing_the_natural_selection_changes_nothing(levels):
    """decode(force_sel=its own selection) is bit-identical, unit by unit."""
    cfg = ocfg(B=2, Hkv=2, Hq=4, n_max=256, L_blk=64, T=4, levels=levels, Tc=16)
    K, V, _ = cache(cfg, 256)
    idx = mp.build_index(K, V, 256, cfg)
    Q = synth.make_queries(1, 2, 4, cfg["d"], "f32", seed=3)[0]
    info = {}
    O = mp.decode(idx, Q, 30, coarse_budget=90, info=info)
    force = {u: {"sel": i["sel"], "csel": i.get("csel")} for u, i in info.items()}
    np.testing.assert_array_equal(mp.decode(idx, Q, 30, coarse_budget=90, force_sel=force), O)
    part = mp.decode(idx, Q, 30, coarse_budget=90, units=[(1, 0)])
    np.testing.assert_array_equal(part[1, 0:2], O[1, 0:2])
    assert not part[0].any() and not part[1, 2:].any()


def test_forcing_every_cluster_is_dense_and_forcing_none_is_all_centroids():
    """A forced set replaces only the selection: all clusters gives dense
    attention; no cluster gives the softmax over every centroid term."""
    cfg = ocfg(B=1, Hkv=1, Hq=4, n_max=128, L_blk=64, T=4)
    K, V, _ = cache(cfg, 128)
    idx = mp.build_index(K, V, 128, cfg)
    Q = synth.make_queries(1, 1, 4, cfg["d"], "f32", seed=4)[0]
    cnt = mp.counts_of(idx["off"][0, 0])
    nz = np.nonzero(cnt > 0)[0]
    O_all = mp.decode(idx, Q, 1, force_sel={(0, 0): {"sel": nz}})
    np.testing.assert_allclose(O_all, sdpa(Q, K, V, 128, 1), atol=1e-12)
    O_none = mp.decode(idx, Q, 1, force_sel={(0, 0): {"sel": np.zeros(0, dtype=np.int64)}})
    Kc, Vc = idx["Kc"][0, 0][nz], idx["Vc"][0, 0][nz]
    for g in range(4):
        z = (Kc @ Q[0, g]) / math.sqrt(cfg["d"]) + np.log(cnt[nz])
        p = np.exp(z - z.max())
        np.testing.assert_allclose(O_none[0, g], p @ Vc / p.sum(), atol=1e-12)


# --------------------------------------------------------------------------- per-query-head selection (NEXT-3)

def test_per_head_selection_equals_brute_force_on_tiny_index():
    """Each query head selects on its own scores (the other reading of R1):
    brute-force selection per head and the brute-force softmax of that head."""
    cfg = ocfg(B=1, Hkv=1, Hq=3, d=6, n_max=40, T=4, L_blk=40)
    K, V, _ = cache(cfg, 40, comps=3)
    idx = mp.build_index(K, V, 40, cfg)
    Q = synth.make_queries(1, 1, 3, 6, "f32", seed=9)[0]
    scale = 1 / math.sqrt(6)
    off = idx["off"][0, 0]
    clusters = []
    for c in range(len(off) - 1):
        rows = range(off[c], off[c + 1])
        clusters.append(([idx["Kp"][0, 0, r].tolist() for r in rows], [idx["Vp"][0, 0, r].tolist() for r in rows],
                         idx["Kc"][0, 0, c].tolist(), idx["Vc"][0, 0, c].tolist()))
    counts = [len(c[0]) for c in clusters]
    differs = False
    for budget in [1, 6, 13, 40]:
        O = mp.decode(idx, Q, budget, per_head=True)
        sels = []
        for g in range(3):
            S = [scale * math.fsum(a * b for a, b in zip(Q[0, g], cl[2])) for cl in clusters]
            sel = brute.select(S, counts, budget)
            sels.append(set(sel))
            want = brute.decode_one(Q[0, g].tolist(), scale, clusters, set(sel))
            np.testing.assert_allclose(O[0, g], want, atol=1e-12)
        differs |= len({frozenset(x) for x in sels}) > 1
    assert differs                    # the heads do select differently here


def test_per_head_selection_with_one_query_head_is_the_group_selection():
    cfg = ocfg(B=2, Hkv=2, Hq=2, n_max=256, L_blk=64, T=4)
    K, V, _ = cache(cfg, 256)
    idx = mp.build_index(K, V, 256, cfg)
    Q = synth.make_queries(1, 2, 2, cfg["d"], "f32", seed=4)[0]
    for budget in [0, 1, 30, 300]:
        np.testing.assert_array_equal(mp.decode(idx, Q, budget, per_head=True), mp.decode(idx, Q, budget))


def test_per_head_selection_with_identical_heads_is_the_group_selection():
    cfg = ocfg(B=1, Hkv=2, Hq=8, n_max=256, L_blk=64, T=4)
    K, V, _ = cache(cfg, 256, seed=2)
    idx = mp.build_index(K, V, 256, cfg)
    q = synth.make_queries(1, 1, 2, cfg["d"], "f32", seed=6)[0]
    Q = np.repeat(q, 4, axis=1)                     # the 4 query heads of each KV head are equal
    for budget in [1, 30, 100]:
        np.testing.assert_allclose(mp.decode(idx, Q, budget, per_head=True), mp.decode(idx, Q, budget), atol=1e-13)


def test_per_head_output_depends_on_its_own_query_only():
    """Changing the other query heads of the group leaves a head's output
    unchanged under per-head selection; under the group max it does not."""
    cfg = ocfg(B=1, Hkv=1, Hq=4, n_max=256, L_blk=64, T=4)
    K, V, _ = cache(cfg, 256, seed=3)
    idx = mp.build_index(K, V, 256, cfg)
    Q = synth.make_queries(2, 1, 4, cfg["d"], "f32", seed=8)
    Q2 = Q[0].copy()
    Q2[0, 1:] = Q[1][0, 1:] * 3.0                    # heads 1..3 replaced, head 0 kept
    a = mp.decode(idx, Q[0], 20, per_head=True)
    b = mp.decode(idx, Q2, 20, per_head=True)
    np.testing.assert_array_equal(a[0, 0], b[0, 0])
    assert not np.array_equal(mp.decode(idx, Q[0], 20)[0, 0], mp.decode(idx, Q2, 20)[0, 0])


def test_per_head_selection_with_the_whole_budget_is_dense_attention():
    cfg = ocfg(B=1, Hkv=2, Hq=4, n_max=256, L_blk=64, T=4)
    K, V, _ = cache(cfg, 200, seed=1)
    idx = mp.build_index(K, V, 200, cfg)
    Q = synth.make_queries(1, 1, 4, cfg["d"], "f32", seed=2)[0]
    np.testing.assert_allclose(mp.decode(idx, Q, 10 ** 6, per_head=True), sdpa(Q, K, V, 200, 2), atol=1e-12)


# --------------------------------------------------------------------------- top-down hierarchy (NEXT-4)

def test_fine_counts_share_the_block_by_size():
    assert list(mp.fine_counts_top_down([100, 0, 30, 5, 1], 34)) == [25, 0, 7, 1, 1]
    assert list(mp.fine_counts_top_down([10, 10, 10], 4)) == [2, 1, 1]        # remainder ties: lower index
    assert list(mp.fine_counts_top_down([3, 1], 10)) == [3, 1]               # never more clusters than tokens
    with pytest.raises(ValueError):
        mp.fine_counts_top_down([50, 1, 1, 1], 3)                              # a fine cluster for each coarse one
    f = mp.fine_counts_top_down([7, 9, 0, 40, 8], 16)
    assert f.sum() == 16 and f[2] == 0 and (f[[0, 1, 3, 4]] >= 1).all()


def test_top_down_index_nests_fine_clusters_in_coarse_clusters():
    """Every coarse cluster owns a contiguous fine-slot range and token range
    holding exactly its tokens; centroids are member means; the store is a
    permutation with cluster runs."""
    cfg = ocfg(B=1, Hkv=2, Hq=4, n_max=256, L_blk=128, T=4, Tc=16, levels=2)
    K, V, _ = cache(cfg, 256, seed=4)
    rec = {}
    idx = mp.build_index(K, V, 256, cfg, hierarchy="top_down", record=rec)
    g = idx["geom"]
    for h in range(2):
        np.testing.assert_array_equal(np.sort(idx["perm"][0, h, :256]), np.arange(256))
        off, coff = idx["off"][0, h], idx["coff"][0, h]
        for j in range(2):
            ca = rec[(0, h, j, "top_down")]["coarse_assign"]
            for cc in range(g["CC_blk"]):
                t0, t1 = off[coff[j * g["CC_blk"] + cc]], off[coff[j * g["CC_blk"] + cc + 1]]
                ids = np.sort(idx["perm"][0, h, t0:t1]) - 128 * j
                np.testing.assert_array_equal(ids, np.nonzero(ca == cc)[0])
                if t1 > t0:
                    np.testing.assert_allclose(idx["Kcc"][0, h, j * g["CC_blk"] + cc],
                                               K[0, h, 128 * j + ids].astype(np.float64).mean(axis=0), atol=1e-6)
            for s in range(j * g["C_blk"], (j + 1) * g["C_blk"]):
                if off[s + 1] > off[s]:
                    np.testing.assert_allclose(idx["Kc"][0, h, s], idx["Kp"][0, h, off[s]:off[s + 1]].mean(axis=0),
                                               atol=1e-6)
                    assert (idx["assign"][0, h, idx["perm"][0, h, off[s]:off[s + 1]]] == s).all()


def test_top_down_index_decodes_exactly_when_coarse_clusters_hold_identical_keys():
    cfg = ocfg(B=1, Hkv=1, Hq=4, n_max=128, L_blk=128, T=4, Tc=32, levels=2)
    rng = np.random.default_rng(11)
    protos = rng.standard_normal((4, cfg["d"])).astype(np.float32)
    K = protos[rng.integers(0, 4, size=128)][None, None]
    V = rng.standard_normal((1, 1, 128, cfg["d"])).astype(np.float32)
    idx = mp.build_index(K, V, 128, cfg, hierarchy="top_down")
    Q = synth.make_queries(1, 1, 4, cfg["d"], "f32", seed=2)[0]
    for budget, cb in [(1, 1), (8, 40), (30, 128)]:
        np.testing.assert_allclose(mp.decode(idx, Q, budget, coarse_budget=cb), sdpa(Q, K, V, 128, 1), atol=1e-6)


def test_top_down_with_unbounded_budgets_is_dense_and_with_unbounded_coarse_budget_is_flat():
    cfg = ocfg(B=1, Hkv=2, Hq=4, n_max=256, L_blk=128, T=4, Tc=16, levels=2)
    K, V, _ = cache(cfg, 256, seed=6)
    idx = mp.build_index(K, V, 256, cfg, hierarchy="top_down")
    Q = synth.make_queries(1, 1, 4, cfg["d"], "f32", seed=1)[0]
    np.testing.assert_allclose(mp.decode(idx, Q, 10 ** 6, coarse_budget=10 ** 6), sdpa(Q, K, V, 256, 2), atol=1e-12)
    flat = dict(idx)
    flat["cfg"] = dict(idx["cfg"], levels=1)
    for budget in [1, 10, 50]:
        np.testing.assert_allclose(mp.decode(idx, Q, budget, coarse_budget=256), mp.decode(flat, Q, budget),
                                   atol=1e-12)


# --------------------------------------------------------------------------- ragged lengths (NEXT-3)

@pytest.mark.parametrize("levels", [1, 2])
def test_ragged_lengths_equal_to_the_batch_length_are_the_plain_build(levels):
    cfg = ocfg(B=3, Hkv=2, Hq=4, n_max=256, L_blk=64, T=4, Tc=16, levels=levels)
    K, V, _ = cache(cfg, 200, seed=9)
    a = mp.build_index(K, V, 200, cfg)
    r = mp.build_index(K, V, [200, 200, 200], cfg)
    for key in ("Kc", "Vc", "off", "Kp", "Vp", "perm", "assign") + (("Kcc", "Vcc", "coff") if levels == 2 else ()):
        np.testing.assert_array_equal(r[key], a[key])
    Q = synth.make_queries(1, 3, 4, cfg["d"], "f32", seed=2)[0]
    np.testing.assert_array_equal(mp.decode(r, Q, 20, coarse_budget=60), mp.decode(a, Q, 20, coarse_budget=60))


@pytest.mark.parametrize("levels", [1, 2])
def test_ragged_batch_attends_each_sequence_to_its_own_tokens(levels):
    """With every token selected a ragged step is dense attention over each
    sequence's own first n_b tokens, and tokens past n_b change nothing."""
    lens = [37, 256, 129, 0]
    cfg = ocfg(B=4, Hkv=2, Hq=4, n_max=256, L_blk=64, T=4, Tc=16, levels=levels)
    K, V, _ = cache(cfg, 256, seed=13)
    idx = mp.build_index(K, V, lens, cfg)
    Q = synth.make_queries(1, 4, 4, cfg["d"], "f32", seed=5)[0]
    O = mp.decode(idx, Q, 10 ** 6, coarse_budget=10 ** 6)
    for b, nb in enumerate(lens):
        if nb == 0:
            assert not O[b].any()
            continue
        np.testing.assert_allclose(O[b:b + 1], sdpa(Q[b:b + 1], K[b:b + 1], V[b:b + 1], nb, 2), atol=1e-12)
    K2, V2 = K.copy(), V.copy()
    for b, nb in enumerate(lens):
        K2[b, :, nb:] *= -3.0
        V2[b, :, nb:] += 7.0
    idx2 = mp.build_index(K2, V2, lens, cfg)
    for budget in [5, 40]:
        np.testing.assert_array_equal(mp.decode(idx2, Q, budget, coarse_budget=4 * budget),
                                      mp.decode(idx, Q, budget, coarse_budget=4 * budget))


def test_ragged_index_refuses_the_update():
    cfg = ocfg(B=2, Hkv=1, Hq=4, n_max=256, L_blk=64, T=4)
    K, V, _ = cache(cfg, 128, seed=1)
    idx = mp.build_index(K, V, [100, 128], cfg)
    with pytest.raises(ValueError):
        mp.cluster_update(idx, K[:, :, :4], V[:, :, :4])
