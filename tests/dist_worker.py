"""Worker of the gloo tests of the matrix-sharded step (CPU, no GPU).

The CUDA step cannot run on the CPU, so the rank's local step is the fp64 oracle
applied to its own matrices; what is under test is the host logic around it:
ownership, packing, the all-gather and unpacking."""
import os

import numpy as np
import torch
import torch.distributed as dist

import oracle
from muon_newton_schulz_04_b200.distributed import ShardedMuon

SHAPES = [(16, 24), (24, 16), (8, 8), (32, 12), (12, 32), (16, 16), (40, 8)]
HP = dict(lr=0.02, momentum=0.95, nesterov=True, weight_decay=0.1, eps=1e-7)


def oracle_step(W, G, B):
    for w, g, b in zip(W, G, B):
        res = oracle.muon_step(w.double().numpy(), g.double().numpy(), b.double().numpy(), **HP)
        w.copy_(torch.from_numpy(res["W"]).float())
        b.copy_(torch.from_numpy(res["B"]).float())


def inputs(step):
    rng = np.random.default_rng(100 + step)
    return [torch.from_numpy(rng.standard_normal(s).astype(np.float32)) for s in SHAPES]


def initial_weights():
    rng = np.random.default_rng(7)
    return [torch.from_numpy((0.02 * rng.standard_normal(s)).astype(np.float32)) for s in SHAPES]


def reference(steps):
    W = initial_weights()
    B = [torch.zeros_like(w) for w in W]
    for t in range(steps):
        oracle_step(W, inputs(t), B)
    return W


def run(rank, world, port, steps, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        opt = ShardedMuon(SHAPES, local_step=oracle_step)
        W = initial_weights()
        B = opt.new_momentum(W)
        for t in range(steps):
            opt.step(W, inputs(t), B)
        torch.save({"W": W, "own": opt.own, "parts": opt.parts}, os.path.join(out_dir, f"rank{rank}.pt"))
    finally:
        dist.destroy_process_group()
