"""The C ABI without a GPU: exports, struct layout, host-side validation."""
import ctypes
import os
import re
import subprocess

import pytest

from clustered_sparse_decode_b200 import _lib as L
from clustered_sparse_decode_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mpattn.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.load()


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:mp_status|const char\*)\s+(mp_\w+)\s*\(", src, re.M)))


def test_every_declared_function_is_exported(lib):
    names = declared_functions()
    assert set(names) >= set(L.EXPORTS) - {"mp_status_str"} or names
    for n in names:
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", L.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (mp_\w+)$", out, re.M))
    assert set(names) <= exported, set(names) - exported


def test_struct_layout_matches_the_header(tmp_path):
    probe = tmp_path / "probe.c"
    fields = {
        "mp_config": ["batch", "max_tokens", "dtype", "init", "reserved", "seed"],
        "mp_index": ["cfg", "n_tokens", "n_clustered", "blocks_max", "slots", "device", "workspace",
                     "workspace_bytes", "layout"],
        "mp_index_view": ["Kc", "coff"],
        "mp_decode_params": ["budget", "scale", "flags", "n_split", "reserved", "sel_mask_out",
                             "coarse_scores_out", "phase_events", "n_phase_events", "reserved2"],
    }
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "mpattn.h"', "int main(void){"]
    for s, fs in fields.items():
        lines.append(f'printf("{s} %zu\\n", sizeof({s}));')
        for f in fs:
            lines.append(f'printf("{s}.{f} %zu\\n", offsetof({s}, {f}));')
    lines.append("return 0;}")
    probe.write_text("\n".join(lines))
    exe = tmp_path / "probe"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.dirname(HEADER), str(probe), "-o", str(exe)], check=True)
    got = dict(l.split() for l in subprocess.run([str(exe)], capture_output=True, text=True).stdout.splitlines())
    cmap = {"mp_config": L.MpConfig, "mp_index": L.MpIndex, "mp_index_view": L.MpIndexView,
            "mp_decode_params": L.MpDecodeParams}
    for s, cls in cmap.items():
        assert int(got[s]) == ctypes.sizeof(cls), s
        for f in fields[s]:
            assert int(got[f"{s}.{f}"]) == getattr(cls, f).offset, f"{s}.{f}"


def cfg(**kw):
    c = L.MpConfig(batch=2, kv_heads=2, q_heads=8, head_dim=128, max_tokens=4096, tokens_per_centroid=16,
                   block_tokens=2048, levels=1, coarse_tokens_per_centroid=128, kmeans_iters=3,
                   update_interval=512, dtype=L.MP_BF16, init=L.MP_INIT_KMEANSPP, reserved=0, seed=1)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def sizes(lib, c):
    a, b = ctypes.c_size_t(), ctypes.c_size_t()
    st = lib.mp_workspace_size(ctypes.byref(c), ctypes.byref(a), ctypes.byref(b))
    return st, a.value, b.value


def test_workspace_size_of_a_valid_config(lib):
    st, ib, sb = sizes(lib, cfg())
    assert st == L.MP_OK
    # the store alone: K and V, 2 units x 4096 tokens x 128 x 2 bytes each
    assert ib >= 2 * 2 * 2 * 4096 * 128 * 2
    assert sb > 0
    st2, ib2, _ = sizes(lib, cfg(levels=2))
    assert st2 == L.MP_OK and ib2 > ib


@pytest.mark.parametrize("bad", [
    dict(batch=0), dict(kv_heads=0), dict(q_heads=7), dict(max_tokens=0), dict(tokens_per_centroid=0),
    dict(block_tokens=8, tokens_per_centroid=16), dict(levels=3), dict(levels=2, coarse_tokens_per_centroid=0),
    dict(kmeans_iters=0), dict(update_interval=0), dict(dtype=7), dict(init=5), dict(reserved=1),
])
def test_invalid_configs_are_rejected(lib, bad):
    assert sizes(lib, cfg(**bad))[0] == L.MP_EINVAL


@pytest.mark.parametrize("unsup", [dict(head_dim=96), dict(q_heads=6, kv_heads=2), dict(block_tokens=32768),
                                   dict(tokens_per_centroid=2, block_tokens=8192),
                                   dict(max_tokens=1 << 22, tokens_per_centroid=16)])
def test_unsupported_configs_are_reported(lib, unsup):
    assert sizes(lib, cfg(**unsup))[0] == L.MP_EUNSUPPORTED


def test_null_arguments_are_rejected_before_any_device_work(lib):
    c = cfg()
    assert lib.mp_workspace_size(None, None, None) == L.MP_EINVAL
    idx = L.MpIndex()
    assert lib.mp_index_init(ctypes.byref(c), None, 0, ctypes.byref(idx), None) == L.MP_EINVAL
    assert lib.mp_index_export(None, None) == L.MP_EINVAL


def test_status_strings(lib):
    for s in range(6):
        assert L.status_str(s) and L.status_str(s) != "unknown status"
    assert L.status_str(99) == "unknown status"
