"""Refusals on the host, before any device work: capacity overflow of a
build or an update (MP_ENOSPC) and malformed decode buffers.  The index is
left as it was."""
import pytest
import torch

import helpers as H
from clustered_sparse_decode_b200 import MpError, MultipoleIndex
from clustered_sparse_decode_b200 import _lib as L

pytestmark = pytest.mark.gpu


def test_capacity_overflow_is_refused_and_leaves_the_index_unchanged():
    o = H.ocfg(B=1, Hkv=1, Hq=4, d=64, n_max=64, T=16, L_blk=64, dtype="f32")
    g = MultipoleIndex(H.gcfg(o))
    over = torch.zeros((1, 1, 65, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(MpError) as e:
        g.build(over, over)
    assert e.value.status == L.MP_ENOSPC
    with pytest.raises(MpError) as e:
        g.update(over, over)
    assert e.value.status == L.MP_ENOSPC
    assert g.n_tokens == 0 and g.n_clustered == 0
    fit = torch.zeros((1, 1, 40, 64), dtype=torch.float32, device="cuda")
    g.update(fit, fit)
    with pytest.raises(MpError) as e:
        g.update(fit, fit)                       # 80 > 64
    assert e.value.status == L.MP_ENOSPC
    assert g.n_tokens == 40
    assert g.check_device_error() == 0


def test_malformed_decode_buffers_are_refused():
    o = H.ocfg(B=1, Hkv=1, Hq=4, d=64, n_max=64, T=16, L_blk=64, dtype="f32")
    g = MultipoleIndex(H.gcfg(o))
    Q = torch.zeros((1, 4, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(ValueError):
        g.decode(Q[:, :3], 8)                    # wrong shape
    with pytest.raises(ValueError):
        g.decode(Q.to(torch.bfloat16), 8)        # wrong dtype
    with pytest.raises(ValueError):
        g.decode(Q.cpu(), 8)                     # pageable host memory
    with pytest.raises(ValueError):
        g.decode(Q, 8, out=torch.zeros((1, 4, 32), dtype=torch.float32, device="cuda"))
