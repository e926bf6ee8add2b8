"""The seeded input generators: shapes, determinism, bf16 rounding, structure."""
import numpy as np
import pytest
import torch

import workloads as wl


def test_workload_shapes_and_counts():
    assert wl.get(1).count == 1 and (wl.get(1).matrices[0].rows, wl.get(1).matrices[0].cols) == (256, 512)
    assert wl.get(2).count == 72 and wl.get(2).elements == 84_934_656
    assert wl.get(3).count == 1 and wl.get(3).weight_decay == 0.1
    assert wl.get(4).count == 288 and wl.get(4).elements == 1_474_560_000
    assert wl.get(5).count == 131
    assert [len(g[2]) for g in wl.get(5).groups()] == [64, 64, 1, 1, 1]
    # nominal NS FLOPs 5(4 m^2 n + 2 m^3)
    assert abs(wl.get(3).ns_flops_nominal() - 5 * 6 * 4096 ** 3) < 1
    assert abs(wl.get(2).ns_flops_nominal() / 1e12 - 1.63) < 0.01
    assert abs(wl.get(4).ns_flops_nominal() / 1e12 - 59.0) < 0.1


def test_bf16_rounding_matches_torch():
    x = np.random.default_rng(0).standard_normal(100_000).astype(np.float32) * 37
    x[:4] = [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -0.0, 65504.0]       # ties and specials
    ours = wl.fp32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = wl.bf16_bits_to_fp32(ours)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_draws_are_deterministic_and_step_dependent():
    w = wl.get(2)
    a = wl.grad(w, 0, 5)
    assert np.array_equal(a, wl.grad(w, 0, 5))
    assert not np.array_equal(a, wl.grad(w, 1, 5))
    assert not np.array_equal(a, wl.grad(w, 0, 6))
    assert a.dtype == np.uint16 and a.shape == (768, 3072)
    assert np.array_equal(wl.weight(w, 3), wl.weight(w, 3))
    assert wl.grad(wl.get(1), 0, 0).dtype == np.float32


def test_lowrank_structure():
    w = wl.get(2)
    g = wl.widen(wl.grad(w, 0, 0), wl.BF16)
    s = np.linalg.svd(g, compute_uv=False)
    assert abs(np.linalg.norm(g) / 768 - 1.0) < 0.05      # Frobenius ~ sqrt(r c)
    assert s[0] / s[100] > 100                              # sigma_i ~ i^-1.5


def test_heavy_rows_structure():
    w = wl.get(5)
    g = wl.widen(wl.grad(w, 0, 64), wl.BF16)                 # 1408 x 2048
    rn = np.linalg.norm(g, axis=1) / np.sqrt(g.shape[1])
    assert int(np.sum(rn > 10)) == int(np.ceil(0.01 * 1408))


def test_parity_subsets():
    assert wl.parity_subset(wl.get(4)) == list(range(6)) + list(range(282, 288))
    assert len(wl.parity_subset(wl.get(5))) == 11
