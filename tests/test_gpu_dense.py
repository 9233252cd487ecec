"""The dense decode baseline (mp_dense_decode) against the oracle's dense attention.

mp_dense_decode attends every query head to all n cached keys of its KV head
(exact softmax attention, no clustering): the comparison point for the
method's speed, which the pages quote against FlashDecoding ("Multipole
Attention ...", atlas.scime summary, "Key results" and "Experimental setup").
The oracle's dense_attention is pinned to torch's fp64 SDPA in
test_oracle_pins.py.  Outputs are compared element by element at the bf16
tolerance, max-abs 2e-2.
"""
import ctypes

import numpy as np
import pytest
import torch

import helpers as H
from clustered_sparse_decode_b200 import Config, dense_decode, synth
from clustered_sparse_decode_b200 import _lib as L
from oracle import multipole as mp

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,Hkv,G,d,n_max,n", [
    (2, 2, 4, 128, 5000, 4999),      # ragged: not a multiple of the 64-row tile
    (1, 3, 1, 128, 3000, 3000),
    (2, 2, 2, 64, 2500, 2400),
    (1, 2, 8, 128, 2048, 2048),
    (1, 1, 4, 128, 200, 37),         # fewer rows than one tile
])
def test_dense_decode_matches_oracle(B, Hkv, G, d, n_max, n):
    o = H.ocfg(B=B, Hkv=Hkv, Hq=G * Hkv, d=d, n_max=n_max)
    K, V, _ = H.cache_for(o, n_max, comps=32, seed=n)
    Q = synth.make_queries(1, B, G * Hkv, d, "bf16", seed=n + 1)[0]
    cfg = H.gcfg(o)
    O = H.to_np(dense_decode(cfg, H.tdev(K, "bf16"), H.tdev(V, "bf16"), n, H.tdev(Q, "bf16")))
    torch.cuda.synchronize()
    ref = mp.dense_attention(Q, K, V, n, Hkv)
    assert np.abs(O - ref).max() <= H.TOL["bf16"]


@pytest.mark.parametrize("qscale", [4.0, 1e3])
def test_dense_decode_sharp_softmax(qscale):
    """Queries scaled x4 (a sharp softmax) and x1000 (one key takes all the
    weight): finite, and within the tolerance of the oracle."""
    o = H.ocfg(B=1, Hkv=2, Hq=8, d=128, n_max=4096)
    K, V, _ = H.cache_for(o, 4096, comps=16, seed=5)
    Q = synth.make_queries(1, 1, 8, 128, "bf16", seed=6, scale=qscale)[0]
    O = H.to_np(dense_decode(H.gcfg(o), H.tdev(K, "bf16"), H.tdev(V, "bf16"), 4096, H.tdev(Q, "bf16")))
    torch.cuda.synchronize()
    assert np.isfinite(O).all()
    assert np.abs(O - mp.dense_attention(Q, K, V, 4096, 2)).max() <= H.TOL["bf16"]


def test_dense_decode_refuses_bad_arguments():
    lib = L.load()
    cfg = H.gcfg(H.ocfg(B=1, Hkv=1, Hq=4, d=128, n_max=128)).to_c()
    K = torch.zeros((1, 1, 128, 128), dtype=torch.bfloat16, device="cuda")
    Q = torch.zeros((1, 4, 128), dtype=torch.bfloat16, device="cuda")
    O = torch.empty_like(Q)
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    assert lib.mp_dense_decode(ctypes.byref(cfg), p(K), p(K), 129, p(Q), p(O), ctypes.c_float(0.0), st) == L.MP_EINVAL
    assert lib.mp_dense_decode(ctypes.byref(cfg), None, p(K), 64, p(Q), p(O), ctypes.c_float(0.0), st) == L.MP_EINVAL
    f32 = H.gcfg(H.ocfg(B=1, Hkv=1, Hq=4, d=128, n_max=128, dtype="f32")).to_c()
    assert lib.mp_dense_decode(ctypes.byref(f32), p(K), p(K), 64, p(Q), p(O), ctypes.c_float(0.0), st) == \
        L.MP_EUNSUPPORTED
