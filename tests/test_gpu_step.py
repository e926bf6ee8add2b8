"""End-to-end parity of muon_step against the fp64 oracle on the five workloads.

Workloads 1-3 are checked on every matrix for 3 consecutive steps; the two
large ones at full size for 1 step, on the oracle's parity subset (the GPU runs
every matrix of the workload in the same grouped launches the benchmark times)."""
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


@pytest.mark.parametrize("precision", [mb.PREC_BF16, mb.PREC_FP32_DEBUG])
def test_tiny_three_steps(precision):
    StepParity(wl.get(1), precision).run().assert_ok()


def test_gpt2_small_three_steps_bf16():
    sp = StepParity(wl.get(2), mb.PREC_BF16).run().assert_ok()
    print("gpt2_small worst", sp.worst())


def test_gpt2_small_one_step_fp32_debug():
    StepParity(wl.get(2), mb.PREC_FP32_DEBUG, subset=[0, 4, 5], steps=1).run().assert_ok()


def test_square4096_three_steps_bf16():
    sp = StepParity(wl.get(3), mb.PREC_BF16).run().assert_ok()
    print("square4096 worst", sp.worst())


@pytest.mark.slow
def test_gpt2_xl_full_size_subset():
    w = wl.get(4)
    sp = StepParity(w, mb.PREC_BF16, subset=wl.parity_subset(w), steps=1).run().assert_ok()
    print("gpt2_xl worst", sp.worst())


@pytest.mark.slow
def test_moe_sweep_full_size_subset():
    w = wl.get(5)
    sp = StepParity(w, mb.PREC_BF16, subset=wl.parity_subset(w), steps=1).run().assert_ok()
    print("moe_sweep worst", sp.worst())


def test_match_rms_and_custom_scale():
    w = wl.get(1)
    cfg = dict(scale_mode=mb.SCALE_MATCH_RMS, rms_target=0.2)
    StepParity(w, mb.PREC_BF16, cfg_overrides=cfg).run(
        scale_fn=lambda r, c: oracle.shape_scale(r, c, oracle.SCALE_MATCH_RMS, 0.2)).assert_ok()


def test_step_is_deterministic():
    w = wl.get(2)
    outs = []
    for _ in range(2):
        opt = mb.Muon(mb.config())
        W = [torch.from_numpy(x).cuda() for x in wl.weights(w)]
        B = [torch.zeros_like(x) for x in W]
        G = [grad_tensor(g, w.grad_dtype) for g in wl.grads(w, 0)]
        opt.step(make_groups(w, W, G, B))
        opt.sync()
        outs.append(torch.cat([x.flatten() for x in W]).cpu())
        opt.close()
    assert torch.equal(outs[0], outs[1])


def test_step_host_matches_device_step():
    w = wl.get(2)
    G = wl.grads(w, 0)
    W0 = wl.weights(w)
    opt = mb.Muon(mb.config())
    Wd = [torch.from_numpy(x).cuda() for x in W0]
    Bd = [torch.zeros_like(x) for x in Wd]
    Gd = [grad_tensor(g, w.grad_dtype) for g in G]
    opt.step(make_groups(w, Wd, Gd, Bd))
    opt.sync()
    Wh = [torch.from_numpy(x.copy()).pin_memory() for x in W0]
    Bh = [torch.zeros_like(x).pin_memory() for x in Wh]
    Gh = [grad_tensor(g, w.grad_dtype, device="cpu").pin_memory() for g in G]
    opt.step_host(make_groups(w, Wh, Gh, Bh))
    opt.sync()
    for a, b in zip(Wd, Wh):
        assert torch.equal(a.cpu(), b)
    for a, b in zip(Bd, Bh):
        assert torch.equal(a.cpu(), b)
    opt.close()


def test_last_norms_are_frobenius_norms_of_direction():
    w = wl.get(2)
    opt = mb.Muon(mb.config())
    W = [torch.from_numpy(x).cuda() for x in wl.weights(w)]
    B = [torch.zeros_like(x) for x in W]
    G = wl.grads(w, 0)
    opt.step(make_groups(w, W, [grad_tensor(g, w.grad_dtype) for g in G], B))
    norms = opt.last_norms()
    order = [k for (_, _, idx) in w.groups() for k in idx]
    for pos, k in enumerate(order):
        U = oracle.nesterov_direction(wl.widen(G[k], w.grad_dtype), wl.widen(G[k], w.grad_dtype), 0.95, True)
        assert abs(norms[pos] - np.linalg.norm(U)) <= 1e-6 * np.linalg.norm(U)
    opt.close()
