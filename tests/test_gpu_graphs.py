"""CUDA graphs: muon_step replays its captured launch sequence, and a caller may
capture muon_step inside a graph of its own.  Both must give the same bits as
direct launches."""
import os

import numpy as np
import pytest
import torch

import workloads as wl
import muon_newton_schulz_04_b200 as mb
from muon_newton_schulz_04_b200 import build as mbuild

from parity import grad_tensor, make_groups

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    mbuild.build()


def _handle(graphs: bool):
    old = os.environ.get("MUON_GRAPHS")
    os.environ["MUON_GRAPHS"] = "1" if graphs else "0"
    try:
        return mb.Muon(mb.config())
    finally:
        if old is None:
            os.environ.pop("MUON_GRAPHS", None)
        else:
            os.environ["MUON_GRAPHS"] = old


def _run(w, graphs: bool, steps: int = 3):
    opt = _handle(graphs)
    W = [torch.from_numpy(x).cuda() for x in wl.weights(w)]
    B = [torch.zeros_like(x) for x in W]
    G = [grad_tensor(g, w.grad_dtype) for g in wl.grads(w, 0)]
    for t in range(steps):
        for dst, g in zip(G, wl.grads(w, t)):          # same buffers: the graph is replayed
            dst.copy_(grad_tensor(g, w.grad_dtype))
        opt.step(make_groups(w, W, G, B))
    opt.sync()
    out = torch.cat([x.flatten() for x in W] + [x.flatten() for x in B]).cpu()
    opt.close()
    return out


@pytest.mark.parametrize("key", ["tiny", "gpt2_small"])
def test_graph_replay_matches_direct_launches(key):
    w = wl.get(key)
    assert torch.equal(_run(w, True), _run(w, False))


def test_step_inside_a_caller_graph():
    w = wl.get("tiny")
    G0 = [grad_tensor(g, w.grad_dtype) for g in wl.grads(w, 0)]

    def fresh():
        W = [torch.from_numpy(x).cuda() for x in wl.weights(w)]
        return W, [torch.zeros_like(x) for x in W], [g.clone() for g in G0]

    # direct: three steps on the same gradient
    opt = mb.Muon(mb.config())
    W1, B1, G1 = fresh()
    for _ in range(3):
        opt.step(make_groups(w, W1, G1, B1))
    opt.sync()
    # captured by the caller after one eager step (the first call allocates the workspace)
    W2, B2, G2 = fresh()
    opt2 = mb.Muon(mb.config())
    opt2.step(make_groups(w, W2, G2, B2))
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            opt2.step(make_groups(w, W2, G2, B2))
    torch.cuda.current_stream().wait_stream(s)
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([x.flatten() for x in W1]), torch.cat([x.flatten() for x in W2]))
    assert torch.equal(torch.cat([x.flatten() for x in B1]), torch.cat([x.flatten() for x in B2]))
    opt.close()
    opt2.close()
