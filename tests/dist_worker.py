"""Workers of the gloo tests of the sharded steps (CPU, no GPU).

The CUDA step cannot run on the CPU, so each rank's per-matrix work is the fp64
oracle; what is under test is the host logic around it: ownership or row
slices, packing, the all-gathers and unpacking."""
import os

import numpy as np
import torch
import torch.distributed as dist

import oracle
from muon_newton_schulz_04_b200.distributed import ShardedMuon, Zero1Muon

SHAPES = [(16, 24), (24, 16), (8, 8), (32, 12), (12, 32), (16, 16), (40, 8), (5, 7)]
HP = dict(lr=0.02, momentum=0.95, nesterov=True, weight_decay=0.1, eps=1e-7)


def _momentum(g, b):
    B_new = oracle.momentum_accumulate(b.double().numpy(), g.double().numpy(), HP["momentum"])
    return B_new, oracle.nesterov_direction(g.double().numpy(), B_new, HP["momentum"], HP["nesterov"])


def oracle_direction(G, B, O):
    """Momentum and the orthogonalised direction of whole matrices; O in O's dtype."""
    for g, b, o in zip(G, B, O):
        B_new, U = _momentum(g, b)
        b.copy_(torch.from_numpy(B_new).float())
        o.copy_(torch.from_numpy(oracle.newton_schulz(U, eps=HP["eps"])).to(o.dtype))


def oracle_apply(W, O):
    for w, o in zip(W, O):
        w.copy_(torch.from_numpy(oracle.apply_update(w.double().numpy(), o.double().numpy(), HP["lr"],
                                                     HP["weight_decay"], 1.0)).float())


def oracle_momentum(G, B, U):
    """Momentum of row slices; U keeps the fp64 direction."""
    for g, b, u in zip(G, B, U):
        B_new, Ud = _momentum(g, b)
        b.copy_(torch.from_numpy(B_new).float())
        u.copy_(torch.from_numpy(Ud))


def oracle_ortho(U, O):
    for u, o in zip(U, O):
        o.copy_(torch.from_numpy(oracle.newton_schulz(u.double().numpy(), eps=HP["eps"])))


def inputs(step):
    rng = np.random.default_rng(100 + step)
    return [torch.from_numpy(rng.standard_normal(s).astype(np.float32)) for s in SHAPES]


def initial_weights():
    rng = np.random.default_rng(7)
    return [torch.from_numpy((0.02 * rng.standard_normal(s)).astype(np.float32)) for s in SHAPES]


def reference(steps, payload_dtype=None):
    """One process, every matrix: the oracle step (payload_dtype None), or the
    direction rounded to payload_dtype and then applied."""
    W = initial_weights()
    B = [torch.zeros_like(w) for w in W]
    for t in range(steps):
        G = inputs(t)
        if payload_dtype is None:
            for k in range(len(W)):
                res = oracle.muon_step(W[k].double().numpy(), G[k].double().numpy(), B[k].double().numpy(), **HP)
                W[k] = torch.from_numpy(res["W"]).float()
                B[k] = torch.from_numpy(res["B"]).float()
        else:
            O = [torch.empty(s, dtype=payload_dtype) for s in SHAPES]
            oracle_direction(G, B, O)
            oracle_apply(W, O)
    return W


def run(rank, world, port, steps, out_dir, variant):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        if variant == "sharded":
            opt = ShardedMuon(SHAPES, direction_fn=oracle_direction, apply_fn=oracle_apply)
            own = opt.own
        else:
            opt = Zero1Muon(SHAPES, momentum_fn=oracle_momentum, ortho_fn=oracle_ortho, apply_fn=oracle_apply,
                            u_dtype=torch.float64)
            own = [opt.slices[k][rank] for k in range(len(SHAPES))]
        W = initial_weights()
        B = opt.new_momentum(W)
        for t in range(steps):
            opt.step(W, inputs(t), B)
        torch.save({"W": W, "B": B, "own": own}, os.path.join(out_dir, f"rank{rank}.pt"))
    finally:
        dist.destroy_process_group()
