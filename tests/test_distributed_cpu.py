"""Host logic of the matrix-sharded step on CPU: LPT ownership, and gloo runs at
world sizes 2 and 3 whose ranks end with identical weights equal to a
single-process run."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as tmp

from muon_newton_schulz_04_b200.distributed import lpt_partition, ns_flops, row_slices

import oracle

import dist_worker


def test_lpt_partition_covers_and_balances():
    rng = np.random.default_rng(0)
    costs = list(rng.uniform(1, 100, size=57))
    for world in (1, 2, 3, 8):
        parts = lpt_partition(costs, world)
        flat = sorted(i for p in parts for i in p)
        assert flat == list(range(len(costs)))
        loads = [sum(costs[i] for i in p) for p in parts]
        # LPT bound: max load <= 4/3 of the optimum <= 4/3 max(mean, largest)
        assert max(loads) <= 4.0 / 3.0 * max(sum(costs) / world, max(costs)) + 1e-9
    assert lpt_partition([5.0, 5.0], 2) == [[0], [1]]
    assert lpt_partition([], 3) == [[], [], []]


def test_gpt2_xl_shapes_split_evenly_over_8_ranks():
    shapes = ([(1600, 1600)] * 4 + [(6400, 1600), (1600, 6400)]) * 48
    costs = [ns_flops(r, c) for (r, c) in shapes]
    loads = [sum(costs[i] for i in p) for p in lpt_partition(costs, 8)]
    assert max(loads) / min(loads) < 1.02


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_row_slices_cover_rows():
    for rows in (1, 2, 5, 40, 1600):
        for world in (1, 2, 3, 8):
            sl = row_slices(rows, world)
            assert sl[0][0] == 0 and sl[-1][1] == rows and len(sl) == world
            assert all(a[1] == b[0] for a, b in zip(sl, sl[1:]))
            sizes = [b - a for a, b in sl]
            assert max(sizes) - min(sizes) <= 1


def _spawn(tmp_path, world, steps, variant):
    tmp.spawn(dist_worker.run, args=(world, _free_port(), steps, str(tmp_path), variant), nprocs=world, join=True)
    return [torch.load(tmp_path / f"rank{r}.pt") for r in range(world)]


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world", [2, 3, 8])
def test_sharded_step_gloo(tmp_path, world):
    """Whole-matrix ownership with the bf16 direction payload: every rank ends with
    the weights of a one-process run that applies the same bf16 directions.  World 3
    gives shards of unequal element counts (the packed buffer is padded); world 8 one
    matrix per rank."""
    steps = 2
    outs = _spawn(tmp_path, world, steps, "sharded")
    ref = dist_worker.reference(steps, payload_dtype=torch.bfloat16)
    assert sorted(i for o in outs for i in o["own"]) == list(range(len(dist_worker.SHAPES)))
    assert all(o["own"] for o in outs)
    for o in outs:
        for w, wr in zip(o["W"], ref):
            assert torch.equal(w, wr)


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world", [2, 3, 8])
def test_zero1_step_gloo(tmp_path, world):
    """Row-sliced momentum (ZeRO-1 Distributed Muon): gather the direction rows,
    orthogonalise full matrices, update own rows, gather W.  Every rank ends with
    the weights of the one-process oracle step, bitwise, and its momentum rows are
    that run's momentum rows.  World 3 splits 8-row and 5-row matrices unevenly;
    world 8 leaves three ranks with no rows of the 5-row matrix."""
    steps = 2
    outs = _spawn(tmp_path, world, steps, "zero1")
    W_ref = dist_worker.initial_weights()
    B_ref = [torch.zeros_like(w) for w in W_ref]
    for t in range(steps):
        G = dist_worker.inputs(t)
        for k in range(len(W_ref)):
            res = oracle.muon_step(W_ref[k].double().numpy(), G[k].double().numpy(), B_ref[k].double().numpy(),
                                   **dist_worker.HP)
            W_ref[k] = torch.from_numpy(res["W"]).float()
            B_ref[k] = torch.from_numpy(res["B"]).float()
    for r, o in enumerate(outs):
        for k, (w, wr) in enumerate(zip(o["W"], W_ref)):
            assert torch.equal(w, wr), (r, k)
            r0, r1 = o["own"][k]
            assert torch.equal(o["B"][k], B_ref[k][r0:r1])
