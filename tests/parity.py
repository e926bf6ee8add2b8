"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and the fp64 oracle on the same seeded inputs, and compare them with the
tolerances the method's precision allows:

  momentum B          <= 1e-6 relative per element, denominator |mu B_old| + |G|
  update O (bf16)     <= 3e-2 relative Frobenius per matrix
  update O (fp32 dbg) <= 1e-4 relative Frobenius per matrix
  apply W             <= 1e-6 relative per element, denominator |W_old| + lr |s O|,
                      with the GPU's own O fed to the oracle's update formula
  W after k steps     ||W_gpu - W_orc||_F <= sum_t lr s tol_O ||O_t||_F + 1e-6 ||W||_F
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence

import numpy as np
import torch

import oracle
import workloads as wl
import muon_newton_schulz_04_b200 as mb

TOL_B = 1e-6
TOL_APPLY = 1e-6
TOL_O = {mb.PREC_BF16: 3e-2, mb.PREC_FP32_DEBUG: 1e-4}


def grad_tensor(g: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    if dtype == wl.BF16:
        return torch.from_numpy(np.ascontiguousarray(g).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(g, dtype=np.float32)).to(device)


def rel_fro(a: np.ndarray, b: np.ndarray) -> float:
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def make_groups(w: wl.Workload, W: List[torch.Tensor], G: List[torch.Tensor], B: List[torch.Tensor], scale=1.0):
    groups = []
    for (r, c, idx) in w.groups():
        groups.append(mb.Group(W=[W[k] for k in idx], G=[G[k] for k in idx], B=[B[k] for k in idx], scale=scale))
    return groups


def group_index(w: wl.Workload):
    """matrix index -> (group, index in group)."""
    out = {}
    for gi, (r, c, idx) in enumerate(w.groups()):
        for j, k in enumerate(idx):
            out[k] = (gi, j)
    return out


class StepParity:
    """Runs `steps` Muon steps of a workload on the GPU and on the oracle and
    records, per step and per checked matrix, the errors against the tolerances."""

    def __init__(self, w: wl.Workload, precision: int = mb.PREC_BF16, subset: Optional[Sequence[int]] = None,
                 steps: Optional[int] = None, cfg_overrides: Optional[dict] = None):
        self.w = w
        self.precision = precision
        self.subset = list(range(w.count)) if subset is None else list(subset)
        self.steps = w.steps if steps is None else steps
        kw = dict(lr=w.lr, momentum=w.momentum, nesterov=int(w.nesterov), weight_decay=w.weight_decay,
                  ns_steps=w.ns_steps, eps=w.eps, precision=precision)
        kw.update(cfg_overrides or {})
        self.cfg = mb.config(**kw)
        self.hp = dict(lr=float(self.cfg.lr), momentum=float(self.cfg.momentum), nesterov=bool(self.cfg.nesterov),
                       weight_decay=float(self.cfg.weight_decay), ns_steps=int(self.cfg.ns_steps),
                       coeffs=(float(self.cfg.ns_a), float(self.cfg.ns_b), float(self.cfg.ns_c)),
                       eps=float(self.cfg.eps))
        self.report: List[Dict] = []

    def run(self, scale_fn=None) -> "StepParity":
        w = self.w
        opt = mb.Muon(self.cfg)
        W0 = wl.weights(w)
        Wd = [torch.from_numpy(x).cuda() for x in W0]
        Bd = [torch.zeros_like(x) for x in Wd]
        idx = group_index(w)
        W_orc = {k: W0[k].astype(np.float64) for k in self.subset}
        B_orc = {k: np.zeros_like(W_orc[k]) for k in self.subset}
        W_gpu_prev = {k: W0[k].astype(np.float64) for k in self.subset}
        wbound = {k: 0.0 for k in self.subset}
        tol_o = TOL_O[self.precision]
        for t in range(self.steps):
            G = wl.grads(w, t)
            Gd = [grad_tensor(g, w.grad_dtype) for g in G]
            opt.step(make_groups(w, Wd, Gd, Bd))
            opt.sync()
            for k in self.subset:
                spec = w.matrices[k]
                s = 1.0 if scale_fn is None else scale_fn(spec.rows, spec.cols)
                g64 = wl.widen(G[k], w.grad_dtype)
                res = oracle.muon_step(W_orc[k], g64, B_orc[k], scale=s, **self.hp)
                O_gpu = torch.empty(spec.rows, spec.cols, dtype=torch.float32, device="cuda")
                opt.last_update(*idx[k], O_gpu)
                torch.cuda.synchronize()
                O_gpu = O_gpu.cpu().numpy().astype(np.float64)
                B_gpu = Bd[k].cpu().numpy().astype(np.float64)
                W_gpu = Wd[k].cpu().numpy().astype(np.float64)
                denB = np.abs(self.hp["momentum"] * B_orc[k]) + np.abs(g64)
                errB = float(np.max(np.abs(B_gpu - res["B"]) / np.maximum(denB, 1e-30)))
                errO = rel_fro(O_gpu, res["O"])
                W_apply = oracle.apply_update(W_gpu_prev[k], O_gpu, self.hp["lr"], self.hp["weight_decay"], s)
                denW = np.abs(W_gpu_prev[k]) + self.hp["lr"] * abs(s) * np.abs(O_gpu)
                errA = float(np.max(np.abs(W_gpu - W_apply) / np.maximum(denW, 1e-30)))
                wbound[k] += self.hp["lr"] * abs(s) * tol_o * float(np.linalg.norm(res["O"]))
                errW = float(np.linalg.norm(W_gpu - res["W"]))
                boundW = wbound[k] + 1e-6 * float(np.linalg.norm(res["W"]))
                self.report.append(dict(step=t, mat=k, errB=errB, errO=errO, errA=errA, errW=errW, boundW=boundW,
                                        finite=bool(np.isfinite(O_gpu).all())))
                W_orc[k], B_orc[k] = res["W"], res["B"]
                W_gpu_prev[k] = W_gpu
        opt.close()
        return self

    def worst(self) -> Dict[str, float]:
        return dict(errB=max(r["errB"] for r in self.report), errO=max(r["errO"] for r in self.report),
                    errA=max(r["errA"] for r in self.report),
                    errW_over_bound=max(r["errW"] / r["boundW"] for r in self.report))

    def assert_ok(self):
        tol_o = TOL_O[self.precision]
        for r in self.report:
            assert r["finite"], r
            assert r["errB"] <= TOL_B, r
            assert r["errO"] <= tol_o, r
            assert r["errA"] <= TOL_APPLY, r
            assert r["errW"] <= r["boundW"], r
        return self
