"""Brute-force restatements for tiny inputs (pure Python loops, math.fsum).

Independent of the oracle's vectorised code: every quantity is enumerated one
term at a time.  Used only to pin the oracle on tiny cases.
"""
import math


def select(scores, counts, budget):
    """Rank candidates (count > 0) by (-score, index); take clusters until the count reaches budget."""
    cand = [c for c in range(len(scores)) if counts[c] > 0]
    ranked = sorted(cand, key=lambda c: (-scores[c], c))
    if budget <= 0:
        return []
    total = sum(counts[c] for c in ranked)
    if total <= budget:
        return ranked
    out, acc = [], 0
    for c in ranked:
        out.append(c)
        acc += counts[c]
        if acc >= budget:
            break
    return out


def sqdist(x, c):
    return math.fsum((a - b) * (a - b) for a, b in zip(x, c))


def assign(X, cents):
    out = []
    for x in X:
        best, bi = None, -1
        for i, c in enumerate(cents):
            dd = sqdist(x, c)
            if best is None or dd < best:
                best, bi = dd, i
        out.append(bi)
    return out


def kmeanspp(X, C, u):
    """k-means++ picks: first floor(u0*L); then the first index whose running D^2 sum exceeds u*total."""
    L = len(X)
    first = min(int(math.floor(u[0] * L)), L - 1)
    picks = [first]
    for k in range(1, C):
        d2 = [min(sqdist(x, X[p]) for p in picks) for x in X]
        tot = 0.0
        run = []
        for v in d2:
            tot += v
            run.append(tot)
        if tot <= 0:
            picks.append(first)
            continue
        thr = u[k] * tot
        pick = L - 1
        for i, r in enumerate(run):
            if r > thr:
                pick = i
                break
        picks.append(pick)
    return picks


def decode_one(q, scale, clusters, selected, tail=(), no_approx=False):
    """One query head.  clusters: list of (keys, values, centroid_key, centroid_value).

    Terms: every token of a selected cluster and every tail token (exact), and
    count * exp(score) with the value centroid for every other non-empty cluster.
    Weights are exp of logits shifted by the largest logit.
    """
    terms = []
    for ci, (keys, vals, kc, vc) in enumerate(clusters):
        if not keys:
            continue
        if ci in selected:
            for k, v in zip(keys, vals):
                terms.append((scale * math.fsum(a * b for a, b in zip(q, k)), v))
        elif not no_approx:
            s = scale * math.fsum(a * b for a, b in zip(q, kc))
            terms.append((s + math.log(len(keys)), vc))
    for k, v in tail:
        terms.append((scale * math.fsum(a * b for a, b in zip(q, k)), v))
    d = len(q)
    if not terms:
        return [0.0] * d
    m = max(z for z, _ in terms)
    w = [math.exp(z - m) for z, _ in terms]
    den = math.fsum(w)
    return [math.fsum(wi * v[j] for wi, (_, v) in zip(w, terms)) / den for j in range(d)]
