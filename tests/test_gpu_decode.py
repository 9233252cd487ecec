"""Decode parity: the CUDA decode (through the C ABI) against the fp64 oracle.

The index is built by the oracle and uploaded with mp_index_import, so that
decode parity is checked independently of clustering parity.  Outputs are
compared element by element (max-abs 2e-2 for bf16 inputs, 1e-4 for fp32);
selected sets must match exactly unless a score tie within 1e-5 decides them.
"""
import ctypes

import numpy as np
import pytest
import torch

import helpers as H
from clustered_sparse_decode_b200 import MultipoleIndex, synth
from clustered_sparse_decode_b200 import _lib as L
from oracle import multipole as mp

pytestmark = pytest.mark.gpu


def run_decode(o, oidx, Q, budget, coarse_budget=0, no_approx=False, n_split=0, scale=None):
    gidx = MultipoleIndex(H.gcfg(o))
    H.upload_index(gidx, oidx)
    B, Hkv = o["B"], o["Hkv"]
    mask = torch.zeros((B, Hkv, gidx.slots), dtype=torch.uint8, device="cuda")
    scores = torch.empty((B, Hkv, gidx.slots), dtype=torch.float32, device="cuda")
    cmask = cscores = None
    if o["levels"] == 2:
        cmask = torch.zeros((B, Hkv, gidx.coarse_slots), dtype=torch.uint8, device="cuda")
        cscores = torch.empty((B, Hkv, gidx.coarse_slots), dtype=torch.float32, device="cuda")
    Qd = H.tdev(Q, o["dtype"])
    O = gidx.decode(Qd, budget, coarse_budget=coarse_budget, no_approx=no_approx, n_split=n_split,
                    scale=0.0 if scale is None else scale, sel_mask=mask, scores=scores,
                    coarse_sel_mask=cmask, coarse_scores=cscores)
    torch.cuda.synchronize()
    assert gidx.check_device_error() == 0
    info = {}

    def oracle(**kw):
        return mp.decode(oidx, Q, budget, coarse_budget=coarse_budget if coarse_budget > 0 else None,
                         flags=mp.NO_APPROX if no_approx else 0, scale=scale, **kw)
    O_ref = oracle(info=info)
    skipped = H.compare_decode(o, H.to_np(O), O_ref, info, mask.cpu().numpy(), scores.cpu().numpy(),
                               levels=o["levels"], gpu_cmask=None if cmask is None else cmask.cpu().numpy(),
                               redo=lambda fs, units: oracle(force_sel=fs, units=units))
    return skipped, H.to_np(O), O_ref


GEOMS = {
    # name: (oracle cfg kwargs, tokens)
    "f32_d64_g4": (dict(B=1, Hkv=1, Hq=4, d=64, n_max=2048, L_blk=2048, dtype="f32"), 2048),
    "bf16_d128_g4_ragged": (dict(B=2, Hkv=2, Hq=8, d=128, n_max=5000, L_blk=2048), 4999),
    "bf16_d128_g1": (dict(B=1, Hkv=3, Hq=3, d=128, n_max=3000, L_blk=1024), 3000),
    "bf16_d64_g2": (dict(B=2, Hkv=2, Hq=4, d=64, n_max=2500, L_blk=1024), 2400),
    "bf16_d128_g8": (dict(B=1, Hkv=2, Hq=16, d=128, n_max=2048, L_blk=2048), 2048),
    "f32_d128_g8": (dict(B=1, Hkv=1, Hq=8, d=128, n_max=1500, L_blk=1024, dtype="f32"), 1500),
}


@pytest.mark.parametrize("geom", list(GEOMS))
@pytest.mark.parametrize("budget", [0, 1, 100, 100000])
@pytest.mark.parametrize("no_approx", [False, True])
def test_decode_matches_oracle(geom, budget, no_approx):
    kw, n = GEOMS[geom]
    o = H.ocfg(**kw)
    K, V, lab = H.cache_for(o, n, comps=48, seed=11)
    oidx = H.component_index(o, K, V, lab, n)           # 48 components into up to 128 slots: empty clusters
    Q = synth.make_queries(1, o["B"], o["Hq"], o["d"], o["dtype"], seed=5)[0]
    skipped, _, _ = run_decode(o, oidx, Q, budget, no_approx=no_approx)
    assert skipped <= max(1, o["B"] * o["Hkv"] // 4)


@pytest.mark.parametrize("G,d", [(4, 128), (1, 128), (2, 64), (8, 128)])
@pytest.mark.parametrize("n_split", [1, 3, 17, 64])
def test_split_count_does_not_change_the_result(n_split, G, d):
    """CTAs per unit (a cluster of 1, 2 or 8 CTAs that exchange scores and
    partials over distributed shared memory) change neither the selection nor,
    beyond fp32 rounding, the output."""
    o = H.ocfg(B=2, Hkv=2, Hq=2 * G, d=d, n_max=4096, L_blk=2048)
    K, V, lab = H.cache_for(o, 4096, comps=128, seed=3)
    oidx = H.component_index(o, K, V, lab, 4096)
    Q = synth.make_queries(1, 2, 2 * G, d, "bf16", seed=8)[0]
    _, O1, ref = run_decode(o, oidx, Q, 700, n_split=n_split)
    _, O2, _ = run_decode(o, oidx, Q, 700, n_split=1)
    assert np.abs(O1 - O2).max() <= 4e-3


def test_kmeans_index_and_tail_tokens():
    """An oracle k-means index with an unclustered tail (attended exactly)."""
    o = H.ocfg(B=1, Hkv=2, Hq=8, d=64, n_max=4096, T=16, L_blk=1024, update_interval=512, dtype="f32", iters=4)
    K, V, _ = H.cache_for(o, 3000, comps=32, radius=None, sigma=0.3, seed=4)
    oidx = mp.build_index(K, V, 2500, o)
    assert not mp.cluster_update(oidx, K[:, :, 2500:2900], V[:, :, 2500:2900])
    assert oidx["n_tokens"] == 2900 and oidx["n_clustered"] == 2500
    Q = synth.make_queries(1, 1, 8, 64, "f32", seed=2)[0]
    for budget in (1, 64, 2500):
        run_decode(o, oidx, Q, budget)


def test_singleton_clusters_equal_dense_attention():
    o = H.ocfg(B=1, Hkv=1, Hq=4, d=128, n_max=512, T=1, L_blk=512, dtype="f32")
    K, V, lab = H.cache_for(o, 512, comps=16, seed=1)
    oidx = mp.index_from_assignment(K, V, 512, o, np.broadcast_to(np.arange(512), (1, 1, 512)))
    Q = synth.make_queries(1, 1, 4, 128, "f32", seed=1)[0]
    _, O, _ = run_decode(o, oidx, Q, 7)
    dense = mp.dense_attention(Q, K, V, 512, 1)
    assert np.abs(O - dense).max() <= 1e-4


def test_large_logits_stay_finite():
    o = H.ocfg(B=1, Hkv=2, Hq=8, d=128, n_max=2048, L_blk=2048)
    K, V, lab = H.cache_for(o, 2048, comps=64, seed=6)
    oidx = H.component_index(o, K, V, lab, 2048)
    Q = synth.make_queries(1, 1, 8, 128, "bf16", seed=7, scale=1e3)[0]
    for budget in (1, 200, 5000):
        _, O, _ = run_decode(o, oidx, Q, budget)
        assert np.isfinite(O).all()


@pytest.mark.parametrize("coarse_budget", [64, 600, 100000])
@pytest.mark.parametrize("budget", [1, 100, 100000])
@pytest.mark.parametrize("no_approx", [False, True])
def test_hierarchical_decode_matches_oracle(coarse_budget, budget, no_approx):
    o = H.ocfg(B=2, Hkv=2, Hq=8, d=128, n_max=6000, T=16, L_blk=2048, levels=2, Tc=128)
    K, V, lab = H.cache_for(o, 5500, comps=96, seed=9)
    oidx = H.component_index(o, K, V, lab, 5500)
    Q = synth.make_queries(1, 2, 8, 128, "bf16", seed=3)[0]
    run_decode(o, oidx, Q, budget, coarse_budget=coarse_budget, no_approx=no_approx)


@pytest.mark.parametrize("levels,dt", [(1, "f32"), (2, "bf16"), (1, "bf16")])
def test_4096_slot_units_decode(levels, dt):
    """One unit of 64K tokens at 16 tokens per centroid: 4096 slots.  The fp32
    flat index runs the multi-kernel path (its selection keys fill the 48 KB
    default shared-memory window exactly), the hierarchical index the
    two-level path, and the bf16 flat index the one-kernel decode with its
    largest unit (a ring of 4 slots, the shared-memory selection for more
    than 2048 slots)."""
    o = H.ocfg(B=1, Hkv=1, Hq=4, d=128, n_max=65536, T=16, L_blk=8192, levels=levels, Tc=128, dtype=dt)
    K, V, lab = H.cache_for(o, 65536, comps=512, seed=21)
    oidx = H.component_index(o, K, V, lab, 65536)
    Q = synth.make_queries(1, 1, 4, 128, dt, seed=4)[0]
    run_decode(o, oidx, Q, 512, coarse_budget=4096 if levels == 2 else 0)


def brute_selection(score, count, budget):
    """Clusters by score descending (ties: lower slot), shortest prefix whose
    token count reaches the budget; every non-empty cluster if it never does."""
    order = sorted(np.nonzero(count > 0)[0].tolist(), key=lambda c: (-score[c], c))
    sel, tot = set(), 0
    for c in order:
        if budget <= 0 or tot >= budget:
            break
        sel.add(c)
        tot += int(count[c])
    return sel


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("budget", [1, 100, 1124, 3000, 4096, 5000])
def test_selection_with_exact_score_ties(budget, dtype):
    """The selection as a function of the scores it reports: groups of 64 and of
    4 clusters with identical keys (exact score ties at the crossing, more and
    fewer candidates than one warp resolves) and one unit of distinct keys;
    bf16 runs the one-kernel unit decode, fp32 the multi-kernel path."""
    o = H.ocfg(B=1, Hkv=3, Hq=12, d=128, n_max=4096, T=16, L_blk=4096, dtype=dtype)
    rng = np.random.default_rng(12)
    K = np.empty((1, 3, 4096, 128), dtype=np.float32)
    for h, grp in enumerate((64, 4, 1)):
        base = synth._cast(rng.standard_normal((256 // grp, 128)), dtype)
        K[0, h] = np.repeat(base, 16 * grp, axis=0)
    V = synth._cast(rng.standard_normal((1, 3, 4096, 128)), dtype)
    a = np.broadcast_to(np.arange(4096) // 16, (1, 3, 4096))
    oidx = mp.index_from_assignment(K, V, 4096, o, a)
    gidx = MultipoleIndex(H.gcfg(o))
    H.upload_index(gidx, oidx)
    mask = torch.zeros((1, 3, gidx.slots), dtype=torch.uint8, device="cuda")
    scores = torch.empty((1, 3, gidx.slots), dtype=torch.float32, device="cuda")
    Q = synth.make_queries(1, 1, 12, 128, dtype, seed=6)[0]
    gidx.decode(H.tdev(Q, dtype), budget, sel_mask=mask, scores=scores)
    torch.cuda.synchronize()
    assert gidx.check_device_error() == 0
    count = np.diff(oidx["off"][0], axis=-1)
    for h in range(3):
        want = brute_selection(scores[0, h].cpu().numpy(), count[h], budget)
        got = set(np.nonzero(mask[0, h].cpu().numpy())[0].tolist())
        assert got == want, f"unit {h}"


@pytest.mark.parametrize("dtype,levels", [("bf16", 1), ("f32", 1), ("bf16", 2)])
def test_host_buffers_give_the_device_result(dtype, levels):
    """Q and O in pinned host memory (Q staged by the library's kernel, O written
    over the host link) give the bits of the device-buffer call; pageable host
    memory is refused before anything is launched."""
    o = H.ocfg(B=2, Hkv=2, Hq=8, d=128, n_max=4096, T=16, L_blk=2048, levels=levels, Tc=128, dtype=dtype, seed=2)
    K, V, lab = H.cache_for(o, 4000, comps=64, seed=4)
    oidx = H.component_index(o, K, V, lab, 4000)
    gidx = MultipoleIndex(H.gcfg(o))
    H.upload_index(gidx, oidx)
    Q = H.tdev(synth.make_queries(1, 2, 8, 128, dtype, seed=9)[0], dtype)
    ref = gidx.decode(Q, 300, coarse_budget=1200)
    Qh = Q.cpu().pin_memory()
    Oh = gidx.decode(Qh, 300, coarse_budget=1200)
    torch.cuda.synchronize()
    assert Oh.device.type == "cpu" and Oh.is_pinned()
    assert torch.equal(Oh, ref.cpu())
    # mixed: host Q into a device O, device Q into a host O
    Od = torch.empty_like(Q)
    gidx.decode(Qh, 300, coarse_budget=1200, out=Od)
    Oh2 = torch.empty_like(Qh).pin_memory()
    gidx.decode(Q, 300, coarse_budget=1200, out=Oh2)
    torch.cuda.synchronize()
    assert torch.equal(Od, ref) and torch.equal(Oh2, ref.cpu())
    assert gidx.check_device_error() == 0
    # pageable host memory: refused by the library itself
    Qp = Q.cpu()
    p = L.MpDecodeParams()
    p.budget = 300
    st = gidx.lib.mp_decode(ctypes.byref(gidx.h), ctypes.c_void_p(Qp.data_ptr()), ctypes.c_void_p(Od.data_ptr()),
                            ctypes.byref(p), ctypes.c_void_p(gidx.scratch.data_ptr()), gidx.scratch.numel(),
                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == L.MP_EINVAL


def test_full_size_bench_launch_sampled_units():
    """The default bench workload at full size (batch 16, 8 KV / 32 query
    heads, 32768 tokens, 2048 slots per head, budget 1638, bf16) in the bench's
    launch configuration (one CTA per SM over all 128 units).  The index holds
    8 distinct oracle-built heads (mixture components as clusters), tiled over
    the 128 units; every unit gets its own queries; 8 units spread over the
    grid's shares are checked against the oracle (selection and outputs)."""
    w = synth.workload("batch16_32k_sparse95")
    B, Hkv, Hq, d, n = w["B"], w["Hkv"], w["Hq"], w["d"], w["n"]
    G = Hq // Hkv
    o1 = H.ocfg(B=1, Hkv=1, Hq=G, d=d, n_max=n, T=w["T"], L_blk=w["L_blk"])
    heads = []
    for s in range(8):
        K, V, lab = synth.make_cache(1, 1, n, d, w["comps"], w["sigma"], radius=w["radius"], outliers=w["outliers"],
                                     dtype="bf16", seed=w["seed"] + 17 * s)
        heads.append(H.component_index(o1, K, V, lab, n))
    src = torch.arange(B * Hkv) % 8
    arr = {}
    for k in ("Kc", "Vc", "Kp", "Vp"):
        t = torch.stack([torch.from_numpy(np.asarray(h[k][0, 0], dtype=np.float32)) for h in heads])
        arr[k] = t[src].reshape(B, Hkv, *t.shape[1:]).to(torch.bfloat16).cuda()
    for k in ("off", "perm", "assign"):
        t = torch.stack([torch.from_numpy(h[k][0, 0].astype(np.int32)) for h in heads])
        arr[k] = t[src].reshape(B, Hkv, *t.shape[1:]).cuda()
    cfg = H.gcfg(H.ocfg(B=B, Hkv=Hkv, Hq=Hq, d=d, n_max=n, T=w["T"], L_blk=w["L_blk"]))
    gidx = MultipoleIndex(cfg)
    gidx.load_arrays(arr, n, n)
    assert gidx.decode_phases() == ["decode"]
    Q = synth.make_queries(1, B, Hq, d, "bf16", seed=71)[0]
    mask = torch.zeros((B, Hkv, gidx.slots), dtype=torch.uint8, device="cuda")
    scores = torch.empty((B, Hkv, gidx.slots), dtype=torch.float32, device="cuda")
    O = H.to_np(gidx.decode(H.tdev(Q, "bf16"), w["budget"], sel_mask=mask, scores=scores))
    torch.cuda.synchronize()
    assert gidx.check_device_error() == 0
    mask, scores = mask.cpu().numpy(), scores.cpu().numpy()
    skipped = 0
    for u in (0, 17, 38, 55, 73, 90, 111, 127):
        b, h = divmod(u, Hkv)
        info = {}
        Qu = Q[b:b + 1, h * G:(h + 1) * G]
        O_ref = mp.decode(heads[u % 8], Qu, w["budget"], info=info)
        skipped += H.compare_decode(o1, O[b:b + 1, h * G:(h + 1) * G], O_ref, info, mask[b:b + 1, h:h + 1],
                                    scores[b:b + 1, h:h + 1],
                                    redo=lambda fs, units, hd=heads[u % 8], q=Qu: mp.decode(hd, q, w["budget"],
                                                                                           force_sel=fs, units=units))
    assert skipped <= 2


@pytest.mark.parametrize("n", [0, 5, 8, 500])
def test_unclustered_indices(n):
    """Indices holding only a tail (appended tokens below the update interval):
    empty (O = 0), 5, 8 and 500 tokens (a tail only, no cluster: the unit
    decode's exact stream alone, a partial chunk for 5 and 8).  Every token is
    attended exactly: the oracle's decode of its own appended index."""
    o = H.ocfg(B=2, Hkv=2, Hq=8, d=128, n_max=4096, T=16, L_blk=2048, update_interval=1024)
    K, V, _ = H.cache_for(o, max(n, 1), comps=8, seed=30 + n)
    oidx = mp.empty_index(o)
    gidx = MultipoleIndex(H.gcfg(o))
    if n > 0:
        assert not mp.cluster_update(oidx, K[:, :, :n], V[:, :, :n])
        assert not gidx.update(H.tdev(K[:, :, :n], "bf16"), H.tdev(V[:, :, :n], "bf16"))
    assert gidx.n_tokens == n and gidx.n_clustered == 0
    Q = synth.make_queries(1, 2, 8, 128, "bf16", seed=n)[0]
    for budget in (0, 16):
        O = H.to_np(gidx.decode(H.tdev(Q, "bf16"), budget))
        torch.cuda.synchronize()
        assert gidx.check_device_error() == 0
        O_ref = mp.decode(oidx, Q, budget)
        assert np.abs(O - O_ref).max() <= H.TOL["bf16"]
        if n == 0:
            assert not O.any()
