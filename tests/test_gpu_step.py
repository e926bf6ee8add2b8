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


def test_square4096_one_step_fp32_debug():
    StepParity(wl.get(3), mb.PREC_FP32_DEBUG, steps=1).run().assert_ok()


@pytest.mark.slow
def test_gpt2_xl_full_size_subset():
    """Two consecutive steps: B stays within 1e-6 across steps (it does not depend on O)."""
    w = wl.get(4)
    sp = StepParity(w, mb.PREC_BF16, subset=wl.parity_subset(w), steps=2).run().assert_ok()
    print("gpt2_xl worst", sp.worst())


@pytest.mark.slow
def test_moe_sweep_full_size_subset():
    w = wl.get(5)
    sp = StepParity(w, mb.PREC_BF16, subset=wl.parity_subset(w), steps=2).run().assert_ok()
    print("moe_sweep worst", sp.worst())


@pytest.mark.slow
@pytest.mark.parametrize("index", [4, 5])
def test_large_workloads_fp32_debug_subset(index):
    """The fp32 debug path (<= 1e-4) at full size; the oracle checks the parity subset."""
    w = wl.get(index)
    sp = StepParity(w, mb.PREC_FP32_DEBUG, subset=wl.parity_subset(w), steps=1).run().assert_ok()
    print(w.key, "fp32 debug worst", sp.worst())


def _match_rms(rms_target):
    return lambda r, c: oracle.shape_scale(r, c, oracle.SCALE_MATCH_RMS, rms_target)


def test_gpt2_small_match_rms_and_weight_decay_three_steps():
    """The per-shape scale matters where shapes differ: 768x768 and 3072x768 matrices
    get different s; with decoupled weight decay on every matrix, 3 steps."""
    w = wl.get(2)
    cfg = dict(scale_mode=mb.SCALE_MATCH_RMS, rms_target=0.2, weight_decay=0.1)
    sp = StepParity(w, mb.PREC_BF16, cfg_overrides=cfg).run(scale_fn=_match_rms(0.2)).assert_ok()
    print("gpt2_small MATCH_RMS + wd worst", sp.worst())


@pytest.mark.slow
def test_gpt2_xl_match_rms_and_weight_decay_subset():
    w = wl.get(4)
    cfg = dict(scale_mode=mb.SCALE_MATCH_RMS, rms_target=0.2, weight_decay=0.05)
    StepParity(w, mb.PREC_BF16, subset=wl.parity_subset(w), steps=1, cfg_overrides=cfg).run(
        scale_fn=_match_rms(0.2)).assert_ok()


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


def test_update_rms_export():
    """muon_last_update_rms: lr * s * RMS(O) per matrix, against the GPU's own O (fp64
    sum of the same values, 1e-5) and the oracle's O (the 3e-2 Frobenius bound on O
    bounds the RMS difference too), with MATCH_RMS so that s differs per shape."""
    w = wl.get(2)
    rms_target = 0.2
    opt = mb.Muon(mb.config(scale_mode=mb.SCALE_MATCH_RMS, rms_target=rms_target))
    W0 = wl.weights(w)
    W = [torch.from_numpy(x).cuda() for x in W0]
    B = [torch.zeros_like(x) for x in W]
    G = wl.grads(w, 0)
    opt.step(make_groups(w, W, [grad_tensor(g, w.grad_dtype) for g in G], B))
    rms = opt.last_update_rms()
    order = [(gi, j, k) for gi, (_, _, idx) in enumerate(w.groups()) for j, k in enumerate(idx)]
    assert len(rms) == w.count
    for pos, (gi, j, k) in enumerate(order):
        spec = w.matrices[k]
        s = oracle.shape_scale(spec.rows, spec.cols, oracle.SCALE_MATCH_RMS, rms_target)
        O = torch.empty(spec.rows, spec.cols, device="cuda")
        opt.last_update(gi, j, O)
        torch.cuda.synchronize()
        O = O.cpu().numpy().astype(np.float64)
        own = 0.02 * s * float(np.sqrt(np.mean(O * O)))
        assert abs(rms[pos] - own) <= 1e-5 * own, (k, rms[pos], own)
        if k in (0, 4, 5):
            res = oracle.muon_step(W0[k].astype(np.float64), wl.widen(G[k], w.grad_dtype), np.zeros(W0[k].shape),
                                   lr=0.02, momentum=0.95, scale=s)
            ref = 0.02 * s * float(np.sqrt(np.mean(res["O"] ** 2)))
            assert abs(rms[pos] - ref) <= 3e-2 * ref, (k, rms[pos], ref)
    opt.close()
