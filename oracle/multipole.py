"""Reference oracle for Multipole Attention decode and its k-means key index.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this module.  The product path
(the CUDA library and its Python binding) never calls it, and it shares no code
with them: no kernels, headers, helpers, tables or constants.

Plain, slow and meant to be read against the method's statement.  Arithmetic is
fp64 unless a step's precision is fixed below.  Sources, by page and section:

* "Multipole Attention for Efficient Long Context Reasoning", arXiv abstract:
  keys are clustered by semantic similarity; the centroids identify the
  important keys, exact attention is computed for those, and the remaining
  keys are approximated through the centroids; a fast cluster update
  re-clusters newly generated tokens.
* Same paper, atlas.scime summary, "Approach": centroid attention scores select
  keys for exact attention and, with value centroids, approximate the
  contribution of unselected clusters; a hierarchical variant; a blockwise
  sliding-window online clustering update.
* Same summary, "Key results" / "Measured effects": token budgets (128, 512);
  approximating unselected keys versus omitting them (the ``no_approx``
  ablation); 1 centroid per 16 tokens and 8K-token clustering blocks as the
  base setting of the ablations.
* Coleman Hooper's homepage, Squeezed Attention blurb: K-means over keys, one
  centroid per cluster, the query compared with key centroids.

Readings where the pages are silent (each restated where it is used):

* R1  GQA: one selection per KV head, on the max over its query heads of the
      centroid score; approximation terms use each query head's own score.
* R2  budget: clusters in descending score order (ties: lower cluster index)
      until the cumulative token count reaches the budget; the crossing cluster
      is included whole; if all clusters hold <= budget tokens, all are taken.
* R4  score scale 1/sqrt(d).
* R5  empty clusters: weight 0, never selected, Lloyd keeps their old centroid.
* R6  tokens not yet clustered (the online tail) are attended exactly and do
      not count against the budget.
* R7  blocks are aligned to position 0; a block of L tokens has ceil(L/T)
      cluster slots; slot numbering is global per head (block j owns slots
      [j*C_blk, (j+1)*C_blk)).
* R8  centroids are stored rounded (round-to-nearest-even) to the key dtype.
* R9  a fixed number of Lloyd iterations; the index keeps the last
      assignment and the means computed from it.
* R11 the KV store is a permuted copy in which each cluster is a contiguous
      run, clusters of a block in slot order, tokens of a cluster in id order.
* R12 k-means++ randomness: splitmix64 (Steele, Lea & Flood, 2014) streams.
* R13 the online update re-clusters only blocks that hold tail tokens.
* R14 update init: a block's previous centroids keep their slots; new slots
      are seeded with the keys of the new tokens at stride T, counted from the
      first new token.  The pages fix no update initialisation; this reading
      is pinned by a hand-worked update of a non-empty block (old slots kept,
      new seeds at the new tokens) and by the block-sized case (equal to a
      fresh stride-seeded build).
* R15 hierarchy: coarse clusters are a count-weighted k-means over a block's
      fine centroids, ceil(L/Tc) of them; fine slots are reordered so every
      coarse cluster owns a contiguous range of fine slots (and of tokens);
      coarse centroids are the means of their member tokens.
* R16 hierarchical decode: coarse selection with its own token budget, then
      fine selection among the fine clusters of the selected coarse clusters.
"""
from __future__ import annotations

import math

import numpy as np

# ----------------------------------------------------------------------------
# dtypes and rounding
# ----------------------------------------------------------------------------

F32 = "f32"
BF16 = "bf16"
NO_APPROX = 1  # decode flag: drop the centroid terms of unselected clusters


def round_to_dtype(x, dtype):
    """Round fp64 values to the storage dtype, round-to-nearest-even (R8).

    bf16 keeps 8 significant bits and fp32's exponent range.  The rounding is
    done directly from fp64 (no fp32 intermediate, which could round twice):
    scale each value by its bf16 unit in the last place, round half to even,
    and scale back.
    """
    x = np.asarray(x, dtype=np.float64)
    if dtype == F32:
        return x.astype(np.float32).astype(np.float64)
    if dtype != BF16:
        raise ValueError(dtype)
    out = np.zeros_like(x)
    nz = (x != 0) & np.isfinite(x)
    _, e = np.frexp(x[nz])                      # x = m * 2**e, 0.5 <= |m| < 1
    e = np.maximum(e, -125)                     # bf16 subnormal spacing 2**-133
    ulp = np.ldexp(1.0, e - 8)                  # 8 significant bits
    r = np.round(x[nz] / ulp) * ulp             # np.round: half to even
    r[np.abs(r) > 3.3895313892515355e38] = np.inf * np.sign(r[np.abs(r) > 3.3895313892515355e38])
    out[nz] = r
    out[~np.isfinite(x)] = x[~np.isfinite(x)]
    return out


# ----------------------------------------------------------------------------
# splitmix64 random streams (R12)
# ----------------------------------------------------------------------------

_GAMMA = 0x9E3779B97F4A7C15
_M64 = (1 << 64) - 1


def splitmix64_mix(z):
    """The splitmix64 output function (Steele, Lea & Flood, OOPSLA 2014)."""
    z &= _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def splitmix64_output(state, k):
    """k-th output (k = 0, 1, ...) of a splitmix64 generator seeded with state."""
    return splitmix64_mix(state + (k + 1) * _GAMMA)


def stream_uniforms(seed, unit, block, level, count):
    """Uniforms in [0, 1) for the k-means++ picks of one (unit, block, level).

    The stream key is output number ((unit * 2**20 + block) * 2 + level) of a
    splitmix64 generator seeded with ``seed``; the uniforms are the top 53 bits
    of the successive outputs of a generator seeded with that key.
    """
    ctr = ((unit << 20) + block) * 2 + level
    key = splitmix64_output(seed & _M64, ctr)
    return [(splitmix64_output(key, k) >> 11) * (1.0 / (1 << 53)) for k in range(count)]


# ----------------------------------------------------------------------------
# k-means (Lloyd) over keys
# ----------------------------------------------------------------------------

def kmeanspp_pick(X, C, u, w=None):
    """k-means++ seeding (Arthur & Vassilvitskii, 2007), weighted if w is given.

    Pick 0: the first index whose running sum of weights exceeds u[0] * total
    (unweighted: floor(u[0] * L)).  Pick k >= 1: the first index whose running
    sum of w * D^2 exceeds u[k] * total, where D^2 is the squared distance to
    the nearest centre picked so far (fp64).  If that total is 0 (every
    weighted point already coincides with a centre), pick 0 is repeated.
    Returns the list of picked row indices.
    """
    L = X.shape[0]
    if w is None:
        w = np.ones(L)
    csum = np.cumsum(w)
    first = int(np.searchsorted(csum, u[0] * csum[-1], side="right"))
    first = min(first, L - 1)
    picks = [first]
    d2 = np.sum((X - X[first]) ** 2, axis=1)
    for k in range(1, C):
        wd = w * d2
        cs = np.cumsum(wd)
        tot = cs[-1]
        if tot > 0:
            i = int(np.searchsorted(cs, u[k] * tot, side="right"))
            i = min(i, L - 1)
        else:
            i = first
        picks.append(i)
        d2 = np.minimum(d2, np.sum((X - X[i]) ** 2, axis=1))
    return picks


def assign_nearest(X, cents):
    """Nearest centroid for each row: argmin_c ||x - c||^2.

    Distances are formed in fp64 and the decision is taken on their fp32
    roundings (the precision the match criterion fixes for assignments); ties
    go to the lower index.  Also returns, per row, the fp64 gap between the
    two smallest distances, so callers can tell near-ties apart.
    """
    xx = np.sum(X * X, axis=1)[:, None]
    cc = np.sum(cents * cents, axis=1)[None, :]
    dist = xx + cc - 2.0 * (X @ cents.T)
    a = np.argmin(dist.astype(np.float32), axis=1)
    if cents.shape[0] > 1:
        part = np.partition(dist, 1, axis=1)
        gap = part[:, 1] - part[:, 0]
    else:
        gap = np.full(X.shape[0], np.inf)
    return a.astype(np.int64), gap


def lloyd(X, init, iters, dtype, w=None):
    """``iters`` Lloyd iterations from ``init`` (R9).

    Each iteration assigns every row to its nearest centroid, then replaces each
    centroid by the (w-weighted) mean of its members, rounded to ``dtype``
    (R8); a centroid with no (weighted) members keeps its value (R5).
    Returns (assignment, centroids, history) where history[t] holds the
    assignment of iteration t, the centroids after it, and the smallest gap
    seen in its assignment step.
    """
    cents = np.array(init, dtype=np.float64, copy=True)
    C = cents.shape[0]
    if w is None:
        w = np.ones(X.shape[0])
    hist = []
    a = None
    for _ in range(iters):
        a, gap = assign_nearest(X, cents)
        sw = np.bincount(a, weights=w, minlength=C)
        sums = np.zeros_like(cents)
        np.add.at(sums, a, X * w[:, None])
        new = cents.copy()
        nz = sw > 0
        new[nz] = round_to_dtype(sums[nz] / sw[nz, None], dtype)
        cents = new
        hist.append({"assign": a.copy(), "cents": cents.copy(),
                     "min_gap": float(gap.min()) if gap.size else np.inf, "gap": gap})
    return a, cents, hist


def member_means(Y, a, C, dtype, empty=None):
    """Per-cluster mean of rows Y (fp64, rounded to dtype); empty -> ``empty`` row or 0."""
    cnt = np.bincount(a, minlength=C).astype(np.float64)
    sums = np.zeros((C, Y.shape[1]))
    np.add.at(sums, a, Y)
    out = np.zeros((C, Y.shape[1])) if empty is None else np.array(empty, dtype=np.float64, copy=True)
    nz = cnt > 0
    out[nz] = round_to_dtype(sums[nz] / cnt[nz, None], dtype)
    return out


# ----------------------------------------------------------------------------
# index layout
# ----------------------------------------------------------------------------

def geometry(cfg):
    """Derived sizes (R7): blocks, fine and coarse slots per block and per head."""
    T, Lb, n_max = cfg["T"], cfg["L_blk"], cfg["n_max"]
    NB = -(-n_max // Lb)
    C_blk = -(-Lb // T)
    Tc = cfg.get("Tc", 128)
    CC_blk = -(-Lb // Tc)
    return {"NB": NB, "C_blk": C_blk, "C_max": NB * C_blk, "CC_blk": CC_blk, "CC_max": NB * CC_blk}


def empty_index(cfg):
    g = geometry(cfg)
    B, H, d, n_max = cfg["B"], cfg["Hkv"], cfg["d"], cfg["n_max"]
    idx = {
        "cfg": dict(cfg), "geom": g, "n_tokens": 0, "n_clustered": 0,
        "Kc": np.zeros((B, H, g["C_max"], d)), "Vc": np.zeros((B, H, g["C_max"], d)),
        "off": np.zeros((B, H, g["C_max"] + 1), dtype=np.int64),
        "Kp": np.zeros((B, H, n_max, d)), "Vp": np.zeros((B, H, n_max, d)),
        "perm": np.full((B, H, n_max), -1, dtype=np.int64),
        "assign": np.full((B, H, n_max), -1, dtype=np.int64),
    }
    if cfg.get("levels", 1) == 2:
        idx["Kcc"] = np.zeros((B, H, g["CC_max"], d))
        idx["Vcc"] = np.zeros((B, H, g["CC_max"], d))
        idx["coff"] = np.zeros((B, H, g["CC_max"] + 1), dtype=np.int64)
    return idx


def counts_of(off):
    """Cluster sizes from the run offsets: n_c = off[c+1] - off[c]."""
    return np.diff(off)


def _store_block(idx, b, h, j, Xk, Xv, a, cents, tok0):
    """Write one block's clusters: centroids, runs in the store, offsets (R11)."""
    cfg, g = idx["cfg"], idx["geom"]
    dtype = cfg["dtype"]
    C_blk = g["C_blk"]
    L = Xk.shape[0]
    C = cents.shape[0]
    s0 = j * C_blk
    idx["Kc"][b, h, s0:s0 + C_blk] = 0.0
    idx["Vc"][b, h, s0:s0 + C_blk] = 0.0
    idx["Kc"][b, h, s0:s0 + C] = cents
    idx["Vc"][b, h, s0:s0 + C] = member_means(Xv, a, C, dtype)
    order = np.argsort(a, kind="stable")          # by cluster, then token id
    cnt = np.bincount(a, minlength=C)
    starts = tok0 + np.concatenate([[0], np.cumsum(cnt)[:-1]])
    idx["off"][b, h, s0:s0 + C] = starts
    idx["off"][b, h, s0 + C:s0 + C_blk] = tok0 + L
    idx["Kp"][b, h, tok0:tok0 + L] = Xk[order]
    idx["Vp"][b, h, tok0:tok0 + L] = Xv[order]
    idx["perm"][b, h, tok0:tok0 + L] = tok0 + order
    idx["assign"][b, h, tok0:tok0 + L] = s0 + a


def seq_counts(idx, b):
    """(n_clustered, n_tokens) of batch element b: the index's counts, or its
    per-sequence lengths (NEXT-3: a ragged batch, every token clustered)."""
    if "seq_lens" in idx:
        nb = int(idx["seq_lens"][b])
        return nb, nb
    return idx["n_clustered"], idx["n_tokens"]


def _finish_offsets(idx):
    """Slots of blocks past the clustered range start (and end) at n_clustered
    (per batch element when the index holds per-sequence lengths)."""
    g = idx["geom"]
    for b in range(idx["cfg"]["B"]):
        nc = seq_counts(idx, b)[0]
        nb_used = -(-nc // idx["cfg"]["L_blk"])
        idx["off"][b, :, nb_used * g["C_blk"]:] = nc
        if "coff" in idx:
            # an absent block's fine slots (all empty) form its first coarse range
            for j in range(nb_used, g["NB"]):
                idx["coff"][b, :, j * g["CC_blk"]:(j + 1) * g["CC_blk"]] = j * g["C_blk"]
            idx["coff"][b, :, g["CC_max"]] = g["C_max"]


def _coarse_block(idx, b, h, j, L, tok0, unit):
    """Two-level hierarchy for one clustered block (R15).

    Count-weighted k-means over the block's fine centroids, then reorder the
    fine slots (and their token runs) by coarse cluster, stably.
    """
    cfg, g = idx["cfg"], idx["geom"]
    dtype, T, Tc = cfg["dtype"], cfg["T"], cfg["Tc"]
    C_blk, CC_blk = g["C_blk"], g["CC_blk"]
    C = -(-L // T)
    CC = -(-L // Tc)
    s0, t0 = j * C_blk, j * CC_blk
    F = idx["Kc"][b, h, s0:s0 + C].copy()
    off = idx["off"][b, h, s0:s0 + C + 1].copy()
    off[C] = tok0 + L
    w = np.diff(off).astype(np.float64)
    u = stream_uniforms(cfg["seed"], unit, j, 1, CC)
    picks = kmeanspp_pick(F, CC, u, w=w)
    ca, ccent, chist = lloyd(F, F[picks], cfg["iters"], dtype, w=w)
    # coarse centroids: means of the member tokens' keys and values
    ids = idx["perm"][b, h, tok0:tok0 + L]                      # token id by store position
    tok_coarse = ca[idx["assign"][b, h, ids] - s0]
    Kst = idx["Kp"][b, h, tok0:tok0 + L]
    Vst = idx["Vp"][b, h, tok0:tok0 + L]
    Kcc = member_means(Kst, tok_coarse, CC, dtype, empty=ccent)
    Vcc = member_means(Vst, tok_coarse, CC, dtype)
    # stable reorder of fine slots by coarse cluster
    fo = np.argsort(ca, kind="stable")                           # new slot r <- old slot fo[r]
    newpos = np.empty(C, dtype=np.int64)
    newpos[fo] = np.arange(C)
    Kc_old = idx["Kc"][b, h, s0:s0 + C].copy()
    Vc_old = idx["Vc"][b, h, s0:s0 + C].copy()
    idx["Kc"][b, h, s0:s0 + C] = Kc_old[fo]
    idx["Vc"][b, h, s0:s0 + C] = Vc_old[fo]
    runs = [(off[c], off[c + 1]) for c in range(C)]
    seg_K, seg_V, seg_P = [], [], []
    starts = []
    pos = tok0
    for r in range(C):
        a0, a1 = runs[fo[r]]
        starts.append(pos)
        pos += a1 - a0
        seg_K.append(idx["Kp"][b, h, a0:a1].copy())
        seg_V.append(idx["Vp"][b, h, a0:a1].copy())
        seg_P.append(idx["perm"][b, h, a0:a1].copy())
        idx["assign"][b, h, idx["perm"][b, h, a0:a1]] = s0 + r
    idx["Kp"][b, h, tok0:tok0 + L] = np.concatenate(seg_K)
    idx["Vp"][b, h, tok0:tok0 + L] = np.concatenate(seg_V)
    idx["perm"][b, h, tok0:tok0 + L] = np.concatenate(seg_P)
    idx["off"][b, h, s0:s0 + C] = starts
    ccnt = np.bincount(ca, minlength=CC)                          # fine slots per coarse
    idx["Kcc"][b, h, t0:t0 + CC_blk] = 0.0
    idx["Vcc"][b, h, t0:t0 + CC_blk] = 0.0
    idx["Kcc"][b, h, t0:t0 + CC] = Kcc
    idx["Vcc"][b, h, t0:t0 + CC] = Vcc
    idx["coff"][b, h, t0:t0 + CC] = s0 + np.concatenate([[0], np.cumsum(ccnt)[:-1]])
    idx["coff"][b, h, t0 + CC:t0 + CC_blk] = s0 + C
    return {"coarse_assign": ca, "fine_order": fo, "hist": chist, "points": F, "picks": picks}


def fine_counts_top_down(sizes, C):
    """Fine clusters per coarse cluster for the top-down hierarchy (NEXT-4).

    The block's C fine clusters are shared out in proportion to the coarse
    clusters' token counts (largest remainder, ties to the lower coarse
    cluster), every non-empty coarse cluster getting at least one and at most
    its token count; empty coarse clusters get none.
    """
    sizes = np.asarray(sizes, dtype=np.int64)
    L = int(sizes.sum())
    f = np.zeros(sizes.size, dtype=np.int64)
    if L == 0:
        return f
    if int((sizes > 0).sum()) > C:
        raise ValueError("more non-empty coarse clusters than fine clusters (tokens per coarse centroid < T)")
    quota = C * sizes / L
    f = np.where(sizes > 0, np.maximum(1, np.floor(quota).astype(np.int64)), 0)
    f = np.minimum(f, sizes)
    rem = quota - np.floor(quota)
    while f.sum() < C:
        room = (sizes > 0) & (f < sizes)
        if not room.any():
            break
        cand = np.nonzero(room)[0]
        c = cand[np.lexsort((cand, -rem[cand]))[0]]    # largest remainder, then lower index
        f[c] += 1
        rem[c] = -1.0
        if (rem[room] < 0).all():
            rem = np.where(room, quota - np.floor(quota), rem)
    while f.sum() > C:
        big = np.nonzero(f > 1)[0]
        c = big[np.lexsort((big, -f[big]))[0]]          # the largest share, then lower index
        f[c] -= 1
    return f


def _top_down_block(idx, b, h, j, Xk, Xv, tok0, unit):
    """Two-level hierarchy for one block, top down (NEXT-4, the other reading
    of the hierarchical variant): coarse k-means over the block's tokens, then
    fine k-means inside each coarse cluster, the block's fine clusters shared
    out by ``fine_counts_top_down``.  Fine slots are laid out by coarse
    cluster (so each coarse cluster covers a contiguous fine range and token
    range, as in the bottom-up build); centroids are member means."""
    cfg, g = idx["cfg"], idx["geom"]
    dtype, T, Tc = cfg["dtype"], cfg["T"], cfg["Tc"]
    C_blk, CC_blk = g["C_blk"], g["CC_blk"]
    L = Xk.shape[0]
    C = -(-L // T)
    CC = -(-L // Tc)
    s0, t0 = j * C_blk, j * CC_blk
    u = stream_uniforms(cfg["seed"], unit, j, 1, CC)
    picks = kmeanspp_pick(Xk, CC, u)
    ca, ccent, chist = lloyd(Xk, Xk[picks], cfg["iters"], dtype)
    sizes = np.bincount(ca, minlength=CC)
    f = fine_counts_top_down(sizes, C)
    Kc = np.zeros((C_blk, Xk.shape[1]))
    Vc = np.zeros((C_blk, Xk.shape[1]))
    fine = np.empty(L, dtype=np.int64)                 # block-local fine slot of every token
    slot = 0
    coff = np.zeros(CC_blk, dtype=np.int64)
    for cc in range(CC):
        coff[cc] = slot
        if f[cc] == 0:
            continue
        members = np.nonzero(ca == cc)[0]              # token order
        X = Xk[members]
        # the coarse cluster's own k-means++ stream: the block's level-0 stream key
        # re-keyed by the coarse index (a generator seeded with seed + cc + 1)
        uf = stream_uniforms((cfg["seed"] + cc + 1) & _M64, unit, j, 0, int(f[cc]))
        fp = kmeanspp_pick(X, int(f[cc]), uf)
        fa, fcent, _ = lloyd(X, X[fp], cfg["iters"], dtype)
        fine[members] = slot + fa
        Kc[slot:slot + f[cc]] = fcent
        Vc[slot:slot + f[cc]] = member_means(Xv[members], fa, int(f[cc]), dtype)
        slot += int(f[cc])
    coff[CC:] = slot
    # the store: tokens by fine slot (slots already grouped by coarse cluster), then token id
    order = np.argsort(fine, kind="stable")
    cnt = np.bincount(fine, minlength=C_blk)
    starts = tok0 + np.concatenate([[0], np.cumsum(cnt)[:-1]])
    idx["Kc"][b, h, s0:s0 + C_blk] = Kc
    idx["Vc"][b, h, s0:s0 + C_blk] = Vc
    idx["off"][b, h, s0:s0 + C_blk] = starts
    idx["Kp"][b, h, tok0:tok0 + L] = Xk[order]
    idx["Vp"][b, h, tok0:tok0 + L] = Xv[order]
    idx["perm"][b, h, tok0:tok0 + L] = tok0 + order
    idx["assign"][b, h, tok0:tok0 + L] = s0 + fine
    idx["Kcc"][b, h, t0:t0 + CC_blk] = 0.0
    idx["Vcc"][b, h, t0:t0 + CC_blk] = 0.0
    idx["Kcc"][b, h, t0:t0 + CC] = member_means(Xk, ca, CC, dtype, empty=ccent)
    idx["Vcc"][b, h, t0:t0 + CC] = member_means(Xv, ca, CC, dtype)
    idx["coff"][b, h, t0:t0 + CC_blk] = s0 + coff
    return {"coarse_assign": ca, "fine_counts": f, "hist": chist}


def _block_init(idx, b, h, j, X, L_old, init_mode, unit, init_given):
    """Initial centroids of one block: k-means++ (R12), given, or warm/stride (R14)."""
    cfg, g = idx["cfg"], idx["geom"]
    T = cfg["T"]
    L = X.shape[0]
    C = -(-L // T)
    s0 = j * g["C_blk"]
    if init_given is not None:
        return np.array(init_given[s0:s0 + C], dtype=np.float64)
    if init_mode == "kmeans++":
        u = stream_uniforms(cfg["seed"], unit, j, 0, C)
        return X[kmeanspp_pick(X, C, u)]
    # warm start: previous centroids keep their slots, new slots at stride T
    C_old = -(-L_old // T)
    warm = idx["Kc"][b, h, s0:s0 + C_old].copy()
    new = X[L_old + T * np.arange(C - C_old)]
    return np.concatenate([warm, new], axis=0)


def _cluster_block(idx, b, h, j, Xk, Xv, init):
    """Lloyd over one block and write it to the index."""
    cfg = idx["cfg"]
    tok0 = j * cfg["L_blk"]
    a, cents, hist = lloyd(Xk, init, cfg["iters"], cfg["dtype"])
    _store_block(idx, b, h, j, Xk, Xv, a, cents, tok0)
    return hist


def build_index(K, V, n, cfg, init=None, init_mode="kmeans++", record=None, hierarchy="bottom_up"):
    """Cluster the first n tokens of every (batch, KV head) from scratch.

    K, V: [B, Hkv, >=n, d] arrays whose values are exact in ``cfg['dtype']``.
    ``init``: optional [B, Hkv, C_max, d] initial centroids (dtype values).
    ``init_mode``: "kmeans++" (default) or "stride" (slot k of a block starts
    at the key of the block's token k*T).  ``record``: optional dict that
    receives the per-block Lloyd histories keyed by (b, h, j).
    ``hierarchy`` (two levels only): "bottom_up" (R15: coarse k-means over the
    fine centroids) or "top_down" (NEXT-4: fine k-means inside each coarse
    cluster of the block's tokens).
    ``n`` may be a sequence of B lengths (NEXT-3, a ragged batch): batch
    element b clusters its first n[b] tokens, blocks aligned to 0 as always,
    and its decode attends to those tokens only.
    """
    idx = empty_index(cfg)
    ragged = not np.isscalar(n)
    if ragged:
        lens = np.asarray(n, dtype=np.int64)
        if lens.shape != (cfg["B"],) or (lens < 0).any() or (lens > cfg["n_max"]).any():
            raise ValueError("per-sequence lengths: B values in [0, n_max]")
        idx["seq_lens"] = lens
        n = int(lens.max())
    n_of = (lambda b: int(idx["seq_lens"][b])) if ragged else (lambda b: n)
    if hierarchy == "top_down":
        if cfg.get("levels", 1) != 2 or init is not None or init_mode != "kmeans++":
            raise ValueError("the top-down hierarchy is a two-level k-means++ build")
        B, H, Lb = cfg["B"], cfg["Hkv"], cfg["L_blk"]
        for b in range(B):
            for h in range(H):
                for j in range(-(-n_of(b) // Lb)):
                    s, e = j * Lb, min(n_of(b), (j + 1) * Lb)
                    rec = _top_down_block(idx, b, h, j, np.asarray(K[b, h, s:e], dtype=np.float64),
                                          np.asarray(V[b, h, s:e], dtype=np.float64), s, b * H + h)
                    if record is not None:
                        record[(b, h, j, "top_down")] = rec
        idx["n_tokens"] = n
        idx["n_clustered"] = n
        _finish_offsets(idx)
        return idx
    B, H = cfg["B"], cfg["Hkv"]
    Lb = cfg["L_blk"]
    for b in range(B):
        for h in range(H):
            unit = b * H + h
            for j in range(-(-n_of(b) // Lb)):
                s, e = j * Lb, min(n_of(b), (j + 1) * Lb)
                Xk = np.asarray(K[b, h, s:e], dtype=np.float64)
                Xv = np.asarray(V[b, h, s:e], dtype=np.float64)
                mode = "kmeans++" if init_mode == "kmeans++" else "stride"
                ini = _block_init(idx, b, h, j, Xk, 0, mode, unit, None if init is None else init[b, h])
                hist = _cluster_block(idx, b, h, j, Xk, Xv, ini)
                if record is not None:
                    record[(b, h, j)] = hist
    idx["n_tokens"] = n
    idx["n_clustered"] = n
    _finish_offsets(idx)
    if cfg.get("levels", 1) == 2:
        for b in range(B):
            for h in range(H):
                for j in range(-(-n_of(b) // Lb)):
                    s, e = j * Lb, min(n_of(b), (j + 1) * Lb)
                    ch = _coarse_block(idx, b, h, j, e - s, s, b * H + h)
                    if record is not None:
                        record[(b, h, j, "coarse")] = ch
        _finish_offsets(idx)
    return idx


def index_from_assignment(K, V, n, cfg, assign, coarse_assign=None):
    """Build the store from a given per-token assignment (no Lloyd).

    ``assign``: [B, Hkv, n] block-local cluster ids in [0, ceil(L_j/T)).
    Centroids are the rounded member means (R8); empty slots get zero
    centroids.  ``coarse_assign`` (levels == 2): [B, Hkv, C_max] coarse ids of
    the fine slots, block-local, in [0, ceil(L_j/Tc)).
    Used to give decode tests an index without running k-means.
    """
    idx = empty_index(cfg)
    B, H = cfg["B"], cfg["Hkv"]
    Lb, T, dtype = cfg["L_blk"], cfg["T"], cfg["dtype"]
    g = idx["geom"]
    nb = -(-n // Lb)
    for b in range(B):
        for h in range(H):
            for j in range(nb):
                s, e = j * Lb, min(n, (j + 1) * Lb)
                Xk = np.asarray(K[b, h, s:e], dtype=np.float64)
                Xv = np.asarray(V[b, h, s:e], dtype=np.float64)
                C = -(-(e - s) // T)
                a = np.asarray(assign[b, h, s:e], dtype=np.int64)
                cents = member_means(Xk, a, C, dtype)
                _store_block(idx, b, h, j, Xk, Xv, a, cents, s)
    idx["n_tokens"] = n
    idx["n_clustered"] = n
    _finish_offsets(idx)
    if cfg.get("levels", 1) == 2:
        C_blk, CC_blk, Tc = g["C_blk"], g["CC_blk"], cfg["Tc"]
        for b in range(B):
            for h in range(H):
                for j in range(nb):
                    s, e = j * Lb, min(n, (j + 1) * Lb)
                    L = e - s
                    C, CC = -(-L // T), -(-L // Tc)
                    s0, t0 = j * C_blk, j * CC_blk
                    ca = np.asarray(coarse_assign[b, h, s0:s0 + C], dtype=np.int64)
                    _reorder_by_coarse(idx, b, h, j, s, L, C, CC, ca)
        _finish_offsets(idx)
    return idx


def _reorder_by_coarse(idx, b, h, j, tok0, L, C, CC, ca):
    """Coarse level from a given fine->coarse assignment (token-mean centroids)."""
    cfg, g = idx["cfg"], idx["geom"]
    dtype = cfg["dtype"]
    s0, t0 = j * g["C_blk"], j * g["CC_blk"]
    off = idx["off"][b, h, s0:s0 + C + 1].copy()
    off[C] = tok0 + L
    ids = idx["perm"][b, h, tok0:tok0 + L]
    tok_coarse = ca[idx["assign"][b, h, ids] - s0]
    Kcc = member_means(idx["Kp"][b, h, tok0:tok0 + L], tok_coarse, CC, dtype)
    Vcc = member_means(idx["Vp"][b, h, tok0:tok0 + L], tok_coarse, CC, dtype)
    fo = np.argsort(ca, kind="stable")
    Kc_old = idx["Kc"][b, h, s0:s0 + C].copy()
    Vc_old = idx["Vc"][b, h, s0:s0 + C].copy()
    idx["Kc"][b, h, s0:s0 + C] = Kc_old[fo]
    idx["Vc"][b, h, s0:s0 + C] = Vc_old[fo]
    seg = {k: [] for k in ("Kp", "Vp", "perm")}
    starts, pos = [], tok0
    for r in range(C):
        a0, a1 = off[fo[r]], off[fo[r] + 1]
        starts.append(pos)
        pos += a1 - a0
        for k in seg:
            seg[k].append(idx[k][b, h, a0:a1].copy())
        idx["assign"][b, h, idx["perm"][b, h, a0:a1]] = s0 + r
    for k in seg:
        idx[k][b, h, tok0:tok0 + L] = np.concatenate(seg[k])
    idx["off"][b, h, s0:s0 + C] = starts
    ccnt = np.bincount(ca, minlength=CC)
    CC_blk = g["CC_blk"]
    idx["Kcc"][b, h, t0:t0 + CC_blk] = 0.0
    idx["Vcc"][b, h, t0:t0 + CC_blk] = 0.0
    idx["Kcc"][b, h, t0:t0 + CC] = Kcc
    idx["Vcc"][b, h, t0:t0 + CC] = Vcc
    idx["coff"][b, h, t0:t0 + CC] = s0 + np.concatenate([[0], np.cumsum(ccnt)[:-1]])
    idx["coff"][b, h, t0 + CC:t0 + CC_blk] = s0 + C


# ----------------------------------------------------------------------------
# online update (R13, R14)
# ----------------------------------------------------------------------------

def block_tokens_in_order(idx, b, h, j, n_upto):
    """Keys/values of block j's tokens [j*L_blk, n_upto) in token-id order."""
    Lb = idx["cfg"]["L_blk"]
    s, e = j * Lb, n_upto
    pos = np.arange(s, e)
    ids = idx["perm"][b, h, s:e]
    inv = np.empty(e - s, dtype=np.int64)
    inv[ids - s] = pos
    return idx["Kp"][b, h, inv], idx["Vp"][b, h, inv]


def cluster_update(idx, K_new, V_new, record=None):
    """Append generated tokens; re-cluster the blocks holding tail tokens on a trigger.

    The trigger (R13): the tail (tokens not yet clustered) holds at least
    ``update_interval`` tokens, or it reaches the end of a block.  Each block
    holding tail tokens is re-clustered over all its tokens with the warm start
    of R14.  Returns True if a trigger fired.  ``record`` (optional list)
    receives (b, h, j, keys, init, Lloyd history) per re-clustered block.
    """
    cfg = idx["cfg"]
    if "seq_lens" in idx:
        raise ValueError("the update appends the same number of tokens to every sequence: not ragged")
    B, H = cfg["B"], cfg["Hkv"]
    Lb = cfg["L_blk"]
    n0 = idx["n_tokens"]
    m = K_new.shape[2]
    if n0 + m > cfg["n_max"]:
        raise ValueError("capacity exceeded")
    pos = np.arange(n0, n0 + m)
    idx["Kp"][:, :, n0:n0 + m] = K_new
    idx["Vp"][:, :, n0:n0 + m] = V_new
    idx["perm"][:, :, n0:n0 + m] = pos
    idx["assign"][:, :, n0:n0 + m] = -1
    idx["n_tokens"] = n1 = n0 + m
    nc = idx["n_clustered"]
    fire = (n1 - nc >= cfg["update_interval"]) or (n1 // Lb > nc // Lb)
    if not fire:
        return False
    for b in range(B):
        for h in range(H):
            unit = b * H + h
            for j in range(nc // Lb, -(-n1 // Lb)):
                s, e = j * Lb, min(n1, (j + 1) * Lb)
                L_old = max(0, min(nc, e) - s)
                Xk, Xv = block_tokens_in_order(idx, b, h, j, e)
                ini = _block_init(idx, b, h, j, Xk, L_old, "warm", unit, None)
                hist = _cluster_block(idx, b, h, j, Xk, Xv, ini)
                if record is not None:
                    record.append((b, h, j, Xk, ini, hist))
                if cfg.get("levels", 1) == 2:
                    _coarse_block(idx, b, h, j, e - s, s, unit)
    idx["n_clustered"] = n1
    _finish_offsets(idx)
    return True


# ----------------------------------------------------------------------------
# decode
# ----------------------------------------------------------------------------

def select_clusters(shat, counts, budget):
    """Token-budgeted selection (R2).

    Candidates are clusters with count > 0.  Order them by score descending,
    ties to the lower index; take the shortest prefix whose token count reaches
    ``budget`` (the crossing cluster whole).  budget <= 0 selects nothing; if
    all candidates together hold <= budget tokens, all are selected.
    Returns (selected ids in rank order, ranked candidate ids).
    """
    cand = np.nonzero(counts > 0)[0]
    order = cand[np.lexsort((cand, -shat[cand]))]
    if budget <= 0 or order.size == 0:
        return order[:0], order
    cum = np.cumsum(counts[order])
    if cum[-1] <= budget:
        return order, order
    k = int(np.searchsorted(cum, budget, side="left"))
    return order[:k + 1], order


def _softmax_terms(z, vals):
    """sum(exp(z - m) * v) / sum(exp(z - m)) over the given terms (fp64)."""
    if z.size == 0:
        return np.zeros(vals.shape[1])
    m = np.max(z)
    p = np.exp(z - m)
    return (p[:, None] * vals).sum(axis=0) / p.sum()


def _scores(q, cents, scale):
    return scale * (q @ cents.T)          # [G, C]


def decode(idx, Q, budget, coarse_budget=None, flags=0, scale=None, info=None, force_sel=None,
           units=None, per_head=False):
    """One decode step for every (batch, query head).  Returns O [B, Hq, d] (fp64).

    Flat index (levels == 1), per KV head h and its query heads g (R1):
      S[g, c] = scale * q_g . Kc_c; score(c) = max_g S[g, c]; select (R2);
      o_g = softmax-weighted sum over
        exact terms  (logit scale * q_g . k_i, value v_i) for every token i of a
                     selected cluster and every tail token (R6), and
        centroid terms (logit S[g, c] + ln n_c, value Vc_c) for every unselected
                     non-empty cluster (dropped with NO_APPROX).
    Two-level index (levels == 2, R16): the same, with coarse selection first,
    fine scores and selection only among fine clusters of selected coarse
    clusters, and coarse centroid terms for unselected coarse clusters.
    ``info`` (dict, optional) receives per-unit selections and scores.

    ``force_sel`` (dict, optional): (b, h) -> {"sel": fine cluster ids[,
    "csel": coarse cluster ids]} replaces the selection step of that unit by the
    given sets; every other step is unchanged.  Where a score tie (R3) lets more
    than one set be correct, this gives the output that belongs to a particular
    one of them.  ``units`` (optional): the (b, h) pairs to compute; the output
    rows of the other units are left zero.

    ``per_head`` (flat index only): the other reading of R1 left open by the
    pages — every query head g selects on its own scores S[g, c] instead of the
    group max, with the same token budget, and its softmax takes exact terms
    for its own selected clusters (and the tail) and centroid terms for its own
    unselected clusters.  A KV head then reads the union of its query heads'
    selections.  ``info`` receives the per-head sets as ``sel_heads``.
    """
    cfg = idx["cfg"]
    B, H, Hq, d = cfg["B"], cfg["Hkv"], cfg["Hq"], cfg["d"]
    G = Hq // H
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if coarse_budget is None:
        coarse_budget = 8 * budget
    if per_head and (cfg.get("levels", 1) != 1 or force_sel is not None):
        raise ValueError("per_head selection is defined for flat indices without forced sets")
    O = np.zeros((B, Hq, d))
    todo = None if units is None else {tuple(u) for u in units}
    for b in range(B):
        for h in range(H):
            if todo is not None and (b, h) not in todo:
                continue
            forced = None if force_sel is None else force_sel.get((b, h))
            nc, nt = seq_counts(idx, b)
            q = np.asarray(Q[b, h * G:(h + 1) * G], dtype=np.float64)
            off = idx["off"][b, h]
            cnt = counts_of(off)
            Kc, Vc = idx["Kc"][b, h], idx["Vc"][b, h]
            Kp, Vp = idx["Kp"][b, h], idx["Vp"][b, h]
            S = _scores(q, Kc, scale)
            shat = np.where(cnt > 0, S.max(axis=0), -np.inf)
            unit_info = {}
            if per_head:
                sel_heads = []
                for gi in range(G):
                    sel_g, _ = select_clusters(np.where(cnt > 0, S[gi], -np.inf), cnt, budget)
                    approx_g = np.setdiff1d(np.nonzero(cnt > 0)[0], sel_g)
                    tok = [np.arange(off[c], off[c + 1]) for c in sel_g] + [np.arange(nc, nt)]
                    tok = np.concatenate(tok).astype(np.int64)
                    z = [scale * (Kp[tok] @ q[gi])]
                    vals = [Vp[tok]]
                    if not (flags & NO_APPROX):
                        z.append(S[gi, approx_g] + np.log(cnt[approx_g]))
                        vals.append(Vc[approx_g])
                    O[b, h * G + gi] = _softmax_terms(np.concatenate(z), np.concatenate(vals, axis=0))
                    sel_heads.append(sel_g)
                if info is not None:
                    info[(b, h)] = {"sel_heads": sel_heads, "S": S}
                continue
            if cfg.get("levels", 1) == 1:
                sel, ranked = select_clusters(shat, cnt, budget)
                if forced is not None:
                    sel = np.asarray(forced["sel"], dtype=np.int64)
                approx = np.setdiff1d(np.nonzero(cnt > 0)[0], sel)
                coarse_terms = np.zeros(0, dtype=np.int64)
                unit_info.update(sel=sel, ranked=ranked, shat=shat)
            else:
                coff = idx["coff"][b, h]
                ccnt = off[coff[1:]] - off[coff[:-1]]
                Kcc, Vcc = idx["Kcc"][b, h], idx["Vcc"][b, h]
                Sc = _scores(q, Kcc, scale)
                chat = np.where(ccnt > 0, Sc.max(axis=0), -np.inf)
                csel, cranked = select_clusters(chat, ccnt, coarse_budget)
                if forced is not None:
                    csel = np.asarray(forced["csel"], dtype=np.int64)
                fine_cand = np.zeros(cnt.size, dtype=bool)
                for cc in csel:
                    fine_cand[coff[cc]:coff[cc + 1]] = True
                shat_f = np.where(fine_cand & (cnt > 0), shat, -np.inf)
                cnt_f = np.where(fine_cand, cnt, 0)
                sel, ranked = select_clusters(shat_f, cnt_f, budget)
                if forced is not None:
                    sel = np.asarray(forced["sel"], dtype=np.int64)
                approx = np.setdiff1d(np.nonzero(cnt_f > 0)[0], sel)
                coarse_terms = np.setdiff1d(np.nonzero(ccnt > 0)[0], csel)
                unit_info.update(sel=sel, ranked=ranked, shat=shat_f, csel=csel,
                                 cranked=cranked, chat=chat)
            tok = [np.arange(off[c], off[c + 1]) for c in sel] + [np.arange(nc, nt)]
            tok = np.concatenate(tok).astype(np.int64)
            for gi in range(G):
                z = [scale * (Kp[tok] @ q[gi])]
                vals = [Vp[tok]]
                if not (flags & NO_APPROX):
                    z.append(S[gi, approx] + np.log(cnt[approx]))
                    vals.append(Vc[approx])
                    if coarse_terms.size:
                        z.append(Sc[gi, coarse_terms] + np.log(ccnt[coarse_terms]))
                        vals.append(Vcc[coarse_terms])
                O[b, h * G + gi] = _softmax_terms(np.concatenate(z), np.concatenate(vals, axis=0))
            if info is not None:
                info[(b, h)] = unit_info
    return O


def dense_attention(Q, K, V, n, Hkv, scale=None):
    """Plain softmax attention of each query head over the first n keys of its KV head."""
    B, Hq, d = Q.shape
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    O = np.zeros((B, Hq, d))
    for b in range(B):
        for hq in range(Hq):
            h = hq // G
            z = scale * (np.asarray(K[b, h, :n], dtype=np.float64) @ np.asarray(Q[b, hq], dtype=np.float64))
            O[b, hq] = _softmax_terms(z, np.asarray(V[b, h, :n], dtype=np.float64))
    return O
