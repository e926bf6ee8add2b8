"""The weight update fused into the last update GEMM's epilogue (MUON_FUSED_APPLY=1).

By default the bf16 path applies W <- decay*W - lr*s*O with the apply kernel after
the last update GEMM; the fused form does the same arithmetic on the same stored
pair O = hi + lo inside that GEMM's epilogue.  Both must give bitwise the same W (and
the same copied-out O for orthogonalize), and the fused form must pass the oracle
parity on its own.  The switch is read when a handle builds its plan, so each case
here uses fresh handles."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
import muon_newton_schulz_04_b200 as mb
from muon_newton_schulz_04_b200 import build as mbuild

from parity import StepParity, TOL_O, grad_tensor, make_groups, rel_fro

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    mbuild.build()


def _step_weights(w, fused, monkeypatch, steps=2, cfg=None):
    monkeypatch.setenv("MUON_FUSED_APPLY", "1" if fused else "0")
    opt = mb.Muon(cfg or mb.config(weight_decay=w.weight_decay))
    W = [torch.from_numpy(x).cuda() for x in wl.weights(w)]
    B = [torch.zeros_like(x) for x in W]
    for t in range(steps):
        G = [grad_tensor(g, w.grad_dtype) for g in wl.grads(w, t)]
        opt.step(make_groups(w, W, G, B))
    opt.sync()
    opt.close()
    return [x.cpu() for x in W]


@pytest.mark.parametrize("key", ["gpt2_small", "square4096"])
def test_fused_and_standalone_apply_give_the_same_weights(key, monkeypatch):
    w = wl.get(key)
    a = _step_weights(w, True, monkeypatch)
    b = _step_weights(w, False, monkeypatch)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_fused_apply_gpt2_small_three_steps_parity(monkeypatch):
    monkeypatch.setenv("MUON_FUSED_APPLY", "1")
    StepParity(wl.get(2), mb.PREC_BF16).run().assert_ok()


def test_fused_apply_match_rms_and_weight_decay(monkeypatch):
    monkeypatch.setenv("MUON_FUSED_APPLY", "1")
    cfg = dict(scale_mode=mb.SCALE_MATCH_RMS, rms_target=0.2, weight_decay=0.1)
    StepParity(wl.get(2), mb.PREC_BF16, cfg_overrides=cfg, steps=1).run(
        scale_fn=lambda r, c: oracle.shape_scale(r, c, oracle.SCALE_MATCH_RMS, 0.2)).assert_ok()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_fused_copy_out_matches_standalone_and_oracle(dtype, monkeypatch):
    rng = np.random.default_rng(11)
    shapes = [(256, 512, 2), (512, 256, 1), (320, 776, 1), (1000, 37, 1)]
    Ms = [[torch.from_numpy(rng.standard_normal((r, c)).astype(np.float32)).to(dtype).cuda() for _ in range(k)]
          for (r, c, k) in shapes]
    outs = []
    for fused in (True, False):
        monkeypatch.setenv("MUON_FUSED_APPLY", "1" if fused else "0")
        opt = mb.Muon(mb.config())
        Os = [[torch.empty(r, c, device="cuda") for _ in range(k)] for (r, c, k) in shapes]
        opt.orthogonalize(list(zip(Ms, Os)))
        opt.sync()
        opt.close()
        outs.append(Os)
    for g in range(len(shapes)):
        for M, Of, Os in zip(Ms[g], outs[0][g], outs[1][g]):
            assert torch.equal(Of, Os)
            ref = oracle.newton_schulz(M.float().cpu().numpy().astype(np.float64), eps=1e-7)
            assert rel_fro(Of.cpu().numpy().astype(np.float64), ref) <= TOL_O[mb.PREC_BF16]


@pytest.mark.parametrize("fused", [False, True])
def test_one_cta_kernel_whole_step_parity(fused, monkeypatch):
    """The selectable one-CTA GEMM kernel (MUON_GEMM_PAIR=0) through a whole step:
    GPT-2-small (all 72 matrices) against the oracle, with the apply kernel and with
    its own fused weight update."""
    monkeypatch.setenv("MUON_GEMM_PAIR", "0")
    monkeypatch.setenv("MUON_FUSED_APPLY", "1" if fused else "0")
    StepParity(wl.get(2), mb.PREC_BF16, steps=1).run().assert_ok()

