"""Host logic of the matrix-sharded step on CPU: LPT ownership, and gloo runs at
world sizes 2 and 3 whose ranks end with identical weights equal to a
single-process run."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as tmp

from muon_newton_schulz_04_b200.distributed import lpt_partition, ns_flops

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


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world", [2, 3])
def test_sharded_step_gloo(tmp_path, world):
    """World 3 gives shards of unequal element counts (the packed buffer is padded
    to the largest)."""
    steps = 2
    tmp.spawn(dist_worker.run, args=(world, _free_port(), steps, str(tmp_path)), nprocs=world, join=True)
    ref = dist_worker.reference(steps)
    outs = [torch.load(tmp_path / f"rank{r}.pt") for r in range(world)]
    assert sorted(i for o in outs for i in o["own"]) == list(range(len(dist_worker.SHAPES)))
    assert all(o["own"] for o in outs)
    for o in outs:
        for w, wr in zip(o["W"], ref):
            assert torch.equal(w, wr)
