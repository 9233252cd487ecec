"""Shared helpers for the GPU parity tests: oracle <-> device marshalling and comparisons."""
import numpy as np
import torch

from clustered_sparse_decode_b200 import synth
from oracle import multipole as mp

TOL = {"bf16": 2e-2, "f32": 1e-4}          # decode output max-abs tolerance per input dtype
SCORE_TIE = 1e-5                            # selection ties: scores closer than this may swap


def ocfg(B, Hkv, Hq, d, n_max, T=16, L_blk=8192, levels=1, Tc=128, iters=10, update_interval=1024,
         dtype="bf16", seed=0):
    return dict(B=B, Hkv=Hkv, Hq=Hq, d=d, n_max=n_max, T=T, L_blk=L_blk, levels=levels, Tc=Tc, iters=iters,
                update_interval=update_interval, dtype=dtype, seed=seed)


def gcfg(o, init="kmeans++"):
    from clustered_sparse_decode_b200 import Config
    return Config(batch=o["B"], kv_heads=o["Hkv"], q_heads=o["Hq"], head_dim=o["d"], max_tokens=o["n_max"],
                  tokens_per_centroid=o["T"], block_tokens=o["L_blk"], levels=o["levels"],
                  coarse_tokens_per_centroid=o["Tc"], kmeans_iters=o["iters"],
                  update_interval=o["update_interval"], dtype=o["dtype"], init=init, seed=o["seed"])


def tdev(x, dtype, device="cuda"):
    """numpy (dtype-exact values) -> device tensor of the torch dtype."""
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device=device).to(tdt)


def upload_index(gidx, oidx):
    """Copy an oracle-built index into a device index (mp_index_import)."""
    dt = oidx["cfg"]["dtype"]
    arr = {}
    for k in ("Kc", "Vc", "Kp", "Vp", "Kcc", "Vcc"):
        if k in oidx:
            arr[k] = tdev(oidx[k], dt)
    for k in ("off", "perm", "assign", "coff"):
        if k in oidx:
            arr[k] = torch.from_numpy(oidx[k].astype(np.int32)).cuda()
    gidx.load_arrays(arr, oidx["n_tokens"], oidx["n_clustered"])
    torch.cuda.synchronize()
    return arr


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def unit_margin(info_u, key="shat", sel="sel", ranked="ranked"):
    """Score gap that decides the selected set of one unit (inf if order does not matter)."""
    s, r = info_u[sel], info_u[ranked]
    if s.size == 0 or s.size == r.size:
        return np.inf
    sh = info_u[key]
    return float(sh[s].min() - sh[r[s.size:]].max())


def compare_decode(o, O_gpu, O_ref, info, gpu_mask, gpu_scores, levels=1, gpu_cmask=None, tol=None, redo=None):
    """Element-wise decode parity for every unit.

    Where no score gap within SCORE_TIE decides a unit's selection, the GPU's
    selected set must equal the oracle's and the outputs must match.  Where such
    a tie decides it, the sets may differ only in clusters inside the tie band,
    and the GPU's outputs are compared with the oracle's decode of the GPU's own
    set: ``redo(force_sel, units)`` is the oracle decode with that selection
    forced.  Returns the number of units whose selection a tie decided.
    """
    B, H, G = o["B"], o["Hkv"], o["Hq"] // o["Hkv"]
    tol = TOL[o["dtype"]] if tol is None else tol
    tied = 0
    for b in range(B):
        for h in range(H):
            iu = info[(b, h)]
            margin = unit_margin(iu)
            cmargin = unit_margin(iu, key="chat", sel="csel", ranked="cranked") if levels == 2 else np.inf
            sel_ref = np.zeros(gpu_mask.shape[-1], dtype=bool)
            sel_ref[iu["sel"]] = True
            sel_gpu = gpu_mask[b, h].astype(bool)
            # scores of scored clusters agree to fp32 rounding
            fin = np.isfinite(iu["shat"])
            np.testing.assert_array_equal(np.isfinite(gpu_scores[b, h]), fin)
            np.testing.assert_allclose(gpu_scores[b, h][fin], iu["shat"][fin], rtol=1e-5, atol=1e-5)
            rows = slice(h * G, (h + 1) * G)
            if min(margin, cmargin) > SCORE_TIE:
                assert np.array_equal(sel_gpu, sel_ref), f"selection differs at unit {(b, h)}"
                if levels == 2:
                    cref = np.zeros(gpu_cmask.shape[-1], dtype=bool)
                    cref[iu["csel"]] = True
                    assert np.array_equal(gpu_cmask[b, h].astype(bool), cref)
                ref = O_ref[b, rows]
            else:
                tied += 1
                forced = {"sel": np.nonzero(sel_gpu)[0]}
                same_coarse = True
                if levels == 2:
                    csel_gpu = gpu_cmask[b, h].astype(bool)
                    cref = np.zeros(csel_gpu.size, dtype=bool)
                    cref[iu["csel"]] = True
                    cdiff = np.nonzero(csel_gpu != cref)[0]
                    cthr = iu["chat"][iu["csel"]].min() if iu["csel"].size else np.inf
                    assert np.all(np.abs(iu["chat"][cdiff] - cthr) <= 4 * SCORE_TIE), \
                        f"coarse selection differs beyond a tie at unit {(b, h)}"
                    forced["csel"] = np.nonzero(csel_gpu)[0]
                    same_coarse = cdiff.size == 0
                if same_coarse:
                    diff = np.nonzero(sel_gpu != sel_ref)[0]
                    thr = iu["shat"][iu["sel"]].min() if iu["sel"].size else np.inf
                    assert np.all(np.abs(iu["shat"][diff] - thr) <= 4 * SCORE_TIE), \
                        f"selection differs beyond a tie at unit {(b, h)}"
                assert redo is not None, "a tie-decided unit needs the oracle decode of the GPU's set"
                ref = redo({(b, h): forced}, [(b, h)])[b, rows]
            err = np.abs(O_gpu[b, rows] - ref).max()
            assert err <= tol, f"unit {(b, h)}: max-abs {err:.3g} > {tol}"
    return tied


def cache_for(o, n, comps=64, sigma=0.25, radius=(1.0, 4.0), outliers=None, seed=0):
    K, V, lab = synth.make_cache(o["B"], o["Hkv"], n, o["d"], comps, sigma, radius=radius, outliers=outliers,
                                 dtype=o["dtype"], seed=seed)
    return K, V, lab


def component_index(o, K, V, lab, n):
    a = synth.component_assignment(lab, n, o["L_blk"], o["T"])
    ca = None
    if o["levels"] == 2:
        g = mp.geometry(o)
        ca = np.zeros((o["B"], o["Hkv"], g["C_max"]), dtype=np.int64)
        for j in range(-(-n // o["L_blk"])):
            L = min(n, (j + 1) * o["L_blk"]) - j * o["L_blk"]
            C, CC = -(-L // o["T"]), -(-L // o["Tc"])
            ca[:, :, j * g["C_blk"]:j * g["C_blk"] + C] = (np.arange(C) * CC) // C
    return mp.index_from_assignment(K, V, n, o, a, ca)
