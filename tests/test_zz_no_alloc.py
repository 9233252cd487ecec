"""mp_decode_static: the decode step for callers that cannot allocate device memory.

A serving engine that hands all free device memory to its own KV-cache pool,
or code on a latency-critical path where cudaMalloc may synchronise the device,
cannot provide the decode scratch buffer that mp_decode takes.  mp_decode_static
uses a fixed 32 MiB array inside the library instead.  These tests call it
through the C ABI and check it against mp_decode on two calls in a row.
"""
import ctypes

import pytest
import torch

import helpers as H
from clustered_sparse_decode_b200 import Config, MpError, MultipoleIndex, synth
from clustered_sparse_decode_b200 import _lib as L

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,levels", [("bf16", 1), ("f32", 2)])
def test_static_scratch_decode_matches_decode(dtype, levels):
    o = H.ocfg(B=2, Hkv=2, Hq=8, d=128, n_max=4096, T=16, L_blk=2048, levels=levels, Tc=128, iters=3,
               dtype=dtype, seed=5)
    K, V, _ = H.cache_for(o, 4096, comps=64, seed=2)
    idx = MultipoleIndex(H.gcfg(o))
    idx.build(H.tdev(K, dtype), H.tdev(V, dtype))
    Qs = synth.make_queries(2, 2, 8, 128, dtype, seed=3)
    for call in range(2):                       # two calls in a row share the library's array
        Q = H.tdev(Qs[call], dtype)
        ref = idx.decode(Q, 300, coarse_budget=1500)
        got = idx.decode_static(Q, 300, coarse_budget=1500)
        torch.cuda.synchronize()
        err = (got.float() - ref.float()).abs().max().item()
        assert err <= H.TOL[dtype], f"call {call}: max-abs {err}"
    assert idx.check_device_error() == 0


def test_static_scratch_rejects_configurations_that_do_not_fit():
    # an fp32 index decodes on the multi-kernel path, whose partials grow with batch x heads
    cfg = Config(batch=32, kv_heads=8, q_heads=64, head_dim=128, max_tokens=256, block_tokens=256,
                 kmeans_iters=1, dtype="f32")
    _, scratch = __import__("clustered_sparse_decode_b200").workspace_size(cfg)
    assert scratch > L.MP_STATIC_SCRATCH_BYTES
    idx = MultipoleIndex(cfg)
    Q = torch.zeros((32, 64, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(MpError) as e:
        idx.decode_static(Q, 16)
    assert e.value.status == L.MP_ENOSPC
    # the regular entry point still works for it
    idx.decode(Q, 16)
    torch.cuda.synchronize()


def test_one_scratch_serves_indices_of_different_shapes():
    """The library's array serves, in turn, flat bf16 indices of 4 and 16
    units and a multi-kernel (fp32) index, many steps each, whatever the
    previous call left in it (no error bit, results equal to mp_decode's)."""
    shapes = [("bf16", 2, 2), ("bf16", 4, 4), ("f32", 2, 2)]
    runs = []
    for s, (dtype, B, Hkv) in enumerate(shapes):
        o = H.ocfg(B=B, Hkv=Hkv, Hq=4 * Hkv, d=128, n_max=4096, T=16, L_blk=2048, iters=2, dtype=dtype, seed=s)
        K, V, _ = H.cache_for(o, 3000 + 100 * s, comps=48, seed=s)
        idx = MultipoleIndex(H.gcfg(o))
        idx.build(H.tdev(K[:, :, :3000 + 100 * s], dtype), H.tdev(V[:, :, :3000 + 100 * s], dtype))
        Q = H.tdev(synth.make_queries(1, B, 4 * Hkv, 128, dtype, seed=s)[0], dtype)
        runs.append((idx, Q, idx.decode(Q, 200).clone()))
    for rep in range(5):
        for idx, Q, ref in runs[::-1] if rep % 2 else runs:
            got = idx.decode_static(Q, 200)
            torch.cuda.synchronize()
            assert torch.equal(got, ref)
    for idx, _, _ in runs:
        assert idx.check_device_error() == 0
