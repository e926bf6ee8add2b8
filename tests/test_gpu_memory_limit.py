"""Device-memory cap of a handle: a call whose buffers would grow past it fails
with MUON_ERR_OOM before launching anything (W and B keep their bits), and the
handle works normally once the cap allows the call.  This injects an allocation
failure on the host side, without any device fault."""
import numpy as np
import pytest
import torch

import muon_newton_schulz_04_b200 as mb
from muon_newton_schulz_04_b200 import build as mbuild

pytestmark = pytest.mark.gpu

SHAPES = [(1024, 768), (768, 1024), (512, 512)]


@pytest.fixture(scope="module", autouse=True)
def built():
    mbuild.build()


def _state(seed):
    rng = np.random.default_rng(seed)
    W = [torch.from_numpy((0.02 * rng.standard_normal(s)).astype(np.float32)).cuda() for s in SHAPES]
    G = [torch.from_numpy(rng.standard_normal(s).astype(np.float32)).to(torch.bfloat16).cuda() for s in SHAPES]
    B = [torch.from_numpy((0.1 * rng.standard_normal(s)).astype(np.float32)).cuda() for s in SHAPES]
    return W, G, B


def _groups(W, G, B):
    return [mb.Group(W=[W[i]], G=[G[i]], B=[B[i]]) for i in range(len(SHAPES))]


@pytest.mark.parametrize("precision", [mb.PREC_BF16, mb.PREC_FP32_DEBUG])
def test_memory_limit_rejects_then_recovers(precision):
    cfg = mb.config(precision=precision, weight_decay=0.1)
    W, G, B = _state(11)
    W0 = [x.clone() for x in W]
    B0 = [x.clone() for x in B]
    opt = mb.Muon(cfg)
    assert opt.memory_held() == 0
    opt.set_memory_limit(1 << 20)                   # far below the workspace these shapes need
    with pytest.raises(mb.MuonError) as ei:
        opt.step(_groups(W, G, B))
    assert ei.value.status == mb.MUON_ERR_OOM
    assert "memory limit" in str(ei.value)
    torch.cuda.synchronize()
    assert opt.memory_held() == 0
    for a, b in zip(W, W0):
        assert torch.equal(a, b)
    for a, b in zip(B, B0):
        assert torch.equal(a, b)
    # no cap: the same handle runs the step, with the bits of an uncapped handle
    opt.set_memory_limit(0)
    opt.step(_groups(W, G, B))
    opt.sync()
    held = opt.memory_held()
    assert held > (1 << 20)
    ref = mb.Muon(cfg)
    W2, G2, B2 = _state(11)
    ref.step(_groups(W2, G2, B2))
    ref.sync()
    for a, b in zip(W + B, W2 + B2):
        assert torch.equal(a, b)
    # a cap equal to what the handle holds admits further calls of the same shapes
    opt.set_memory_limit(held)
    opt.step(_groups(W, G, B))
    opt.sync()
    assert opt.memory_held() == held
    opt.close()
    ref.close()
