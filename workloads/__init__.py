"""Seeded synthetic inputs for the Muon step: shapes, hyperparameters and data.

This module is shared by the fp64 oracle tests, the CUDA parity tests and the
benchmark.  It holds no part of the Muon arithmetic (no momentum, no
normalisation, no Newton-Schulz, no update); it only draws the tensors a
training loop would hand to the optimizer, with the shapes and value structure
of the five workloads:

  1. one 256x512 fp32 gradient, i.i.d. N(0,1)               ("tiny")
  2. GPT-2-small hidden matrices, 12 layers x {Q,K,V,O 768x768, fc 3072x768,
     proj 768x3072}, bf16 gradients U diag(sigma) V^T + 0.01 noise,
     sigma_i ~ i^-1.5                                        ("gpt2_small")
  3. one 4096x4096 bf16 gradient, sigma_i ~ i^-1, weight decay 0.1
                                                             ("square4096")
  4. GPT-2-XL hidden matrices, 48 layers x {Q,K,V,O 1600x1600, 6400x1600,
     1600x6400}, bf16 N(0,1)/sqrt(fan_in) + rank-8 spike     ("gpt2_xl")
  5. MoE experts 64x 2048x1408 + 64x 1408x2048 and single 8192x2048,
     2048x8192, 16384x4096; N(0,1) with 1% of rows x20     ("moe_sweep")

Every draw is seeded: gradient of matrix k at optimizer step t of workload w
uses SeedSequence([1234 + 1000*w + t, k, 1]); the initial weight of matrix k
uses SeedSequence([1234 + 1000*w, k, 2]).  Weights are N(0, 0.02^2) fp32 and
the momentum buffer starts at zero (the caller's job, as in any optimizer).

bf16 tensors are carried as numpy uint16 bit patterns (round-to-nearest-even
from fp32), so that the oracle can widen the exact stored values to fp64 and
the GPU side can view the same bytes as torch.bfloat16.
"""
from __future__ import annotations

import dataclasses
import math
from concurrent.futures import ThreadPoolExecutor
from typing import List, Optional, Sequence, Tuple

import numpy as np

BF16 = "bf16"
FP32 = "fp32"


@dataclasses.dataclass(frozen=True)
class MatrixSpec:
    rows: int
    cols: int
    name: str


@dataclasses.dataclass(frozen=True)
class Workload:
    index: int              # 1..5
    key: str
    description: str
    matrices: Tuple[MatrixSpec, ...]
    grad_dtype: str         # BF16 or FP32
    grad_kind: str          # "iid", "lowrank", "spike", "heavy_rows"
    lr: float = 0.02
    momentum: float = 0.95
    nesterov: bool = True
    weight_decay: float = 0.0
    ns_steps: int = 5
    eps: float = 1e-7
    steps: int = 3          # consecutive optimizer steps in the parity run

    @property
    def count(self) -> int:
        return len(self.matrices)

    @property
    def elements(self) -> int:
        return sum(s.rows * s.cols for s in self.matrices)

    def groups(self) -> List[Tuple[int, int, List[int]]]:
        """Same-shape matrices grouped, in first-appearance order: (rows, cols, indices)."""
        order: List[Tuple[int, int]] = []
        members = {}
        for k, s in enumerate(self.matrices):
            key = (s.rows, s.cols)
            if key not in members:
                members[key] = []
                order.append(key)
            members[key].append(k)
        return [(r, c, members[(r, c)]) for (r, c) in order]

    def ns_flops_nominal(self) -> float:
        """5 x (4 m^2 n + 2 m^3) per matrix, m = min(r,c), n = max(r,c)."""
        tot = 0.0
        for s in self.matrices:
            m, n = min(s.rows, s.cols), max(s.rows, s.cols)
            tot += self.ns_steps * (4.0 * m * m * n + 2.0 * m ** 3)
        return tot

    def ns_flops_symmetric(self) -> float:
        """FLOPs when the two symmetric products are computed on one triangle."""
        tot = 0.0
        for s in self.matrices:
            m, n = min(s.rows, s.cols), max(s.rows, s.cols)
            tot += self.ns_steps * (3.0 * m * m * n + 1.0 * m ** 3)
        return tot


def _gpt2_small() -> Tuple[MatrixSpec, ...]:
    out = []
    for layer in range(12):
        for nm in ("q", "k", "v", "o"):
            out.append(MatrixSpec(768, 768, f"h{layer}.attn.{nm}"))
        out.append(MatrixSpec(3072, 768, f"h{layer}.mlp.fc"))
        out.append(MatrixSpec(768, 3072, f"h{layer}.mlp.proj"))
    return tuple(out)


def _gpt2_xl() -> Tuple[MatrixSpec, ...]:
    out = []
    for layer in range(48):
        for nm in ("q", "k", "v", "o"):
            out.append(MatrixSpec(1600, 1600, f"h{layer}.attn.{nm}"))
        out.append(MatrixSpec(6400, 1600, f"h{layer}.mlp.fc"))
        out.append(MatrixSpec(1600, 6400, f"h{layer}.mlp.proj"))
    return tuple(out)


def _moe_sweep() -> Tuple[MatrixSpec, ...]:
    out = [MatrixSpec(2048, 1408, f"expert{e}.up") for e in range(64)]
    out += [MatrixSpec(1408, 2048, f"expert{e}.down") for e in range(64)]
    out += [MatrixSpec(8192, 2048, "tall8192x2048"),
            MatrixSpec(2048, 8192, "wide2048x8192"),
            MatrixSpec(16384, 4096, "tall16384x4096")]
    return tuple(out)


WORKLOADS = {
    1: Workload(1, "tiny", "single 256x512 fp32 gradient, i.i.d. N(0,1)",
                (MatrixSpec(256, 512, "w"),), FP32, "iid"),
    2: Workload(2, "gpt2_small", "GPT-2-small hidden matrices (72), ill-conditioned bf16 gradients",
                _gpt2_small(), BF16, "lowrank"),
    3: Workload(3, "square4096", "single 4096x4096 bf16 gradient, power-law spectrum, weight decay 0.1",
                (MatrixSpec(4096, 4096, "w"),), BF16, "powerlaw", weight_decay=0.1),
    4: Workload(4, "gpt2_xl", "GPT-2-XL hidden matrices (288), N(0,1)/sqrt(fan_in) + rank-8 spike",
                _gpt2_xl(), BF16, "spike"),
    5: Workload(5, "moe_sweep", "MoE experts 64x2048x1408 + 64x1408x2048 + 3 aspect-sweep singles",
                _moe_sweep(), BF16, "heavy_rows"),
}
BY_KEY = {w.key: w for w in WORKLOADS.values()}


def get(w) -> Workload:
    if isinstance(w, Workload):
        return w
    if isinstance(w, str):
        return BY_KEY[w]
    return WORKLOADS[int(w)]


# --------------------------------------------------------------------------- bf16 bits

def fp32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_fp32(u: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 exactly."""
    return (np.ascontiguousarray(u, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def widen(g: np.ndarray, dtype: str) -> np.ndarray:
    """Exact fp64 value of a stored gradient (bf16 bits or fp32)."""
    if dtype == BF16:
        return bf16_bits_to_fp32(g).astype(np.float64)
    return np.asarray(g, dtype=np.float32).astype(np.float64)


# --------------------------------------------------------------------------- draws

def _rng(w: int, step: int, k: int, stream: int) -> np.random.Generator:
    base = 1234 + 1000 * w + (step if stream == 1 else 0)
    return np.random.default_rng(np.random.SeedSequence([base, k, stream]))


def _haar_columns(rng: np.random.Generator, n: int, k: int) -> np.ndarray:
    """n x k matrix with orthonormal columns, Haar-distributed (QR with sign fix)."""
    q, r = np.linalg.qr(rng.standard_normal((n, k)))
    return q * np.sign(np.diag(r))[None, :]


def grad_fp32(wl: Workload, step: int, k: int) -> np.ndarray:
    """The fp32 value of gradient k at `step` before storage rounding."""
    spec = wl.matrices[k]
    r, c = spec.rows, spec.cols
    rng = _rng(wl.index, step, k, 1)
    if wl.grad_kind == "iid":
        return rng.standard_normal((r, c), dtype=np.float32)
    if wl.grad_kind in ("lowrank", "powerlaw"):
        m = min(r, c)
        expo = 1.5 if wl.grad_kind == "lowrank" else 1.0
        sigma = np.arange(1, m + 1, dtype=np.float64) ** (-expo)
        # Frobenius norm sqrt(r*c): the size of a unit-variance r x c matrix
        sigma *= math.sqrt(r * c) / np.linalg.norm(sigma)
        u = _haar_columns(rng, r, m)
        v = _haar_columns(rng, c, m)
        g = (u * sigma[None, :]) @ v.T
        if wl.grad_kind == "lowrank":
            g += 0.01 * rng.standard_normal((r, c))
        return g.astype(np.float32)
    if wl.grad_kind == "spike":
        g = rng.standard_normal((r, c), dtype=np.float32) * np.float32(1.0 / math.sqrt(c))
        sigma_edge = (math.sqrt(r) + math.sqrt(c)) / math.sqrt(c)
        u = _haar_columns(rng, r, 8)
        v = _haar_columns(rng, c, 8)
        g += ((10.0 * sigma_edge) * (u @ v.T)).astype(np.float32)
        return g
    if wl.grad_kind == "heavy_rows":
        g = rng.standard_normal((r, c), dtype=np.float32)
        heavy = rng.choice(r, size=int(math.ceil(0.01 * r)), replace=False)
        g[heavy, :] *= np.float32(20.0)
        return g
    raise ValueError(wl.grad_kind)


def grad(wl: Workload, step: int, k: int) -> np.ndarray:
    """Stored gradient: uint16 bf16 bits (bf16 workloads) or fp32 array."""
    g = grad_fp32(wl, step, k)
    return fp32_to_bf16_bits(g) if wl.grad_dtype == BF16 else g


def weight(wl: Workload, k: int) -> np.ndarray:
    spec = wl.matrices[k]
    rng = _rng(wl.index, 0, k, 2)
    return (0.02 * rng.standard_normal((spec.rows, spec.cols), dtype=np.float32)).astype(np.float32)


def _map(fn, items: Sequence[int], threads: Optional[int]):
    if threads == 1 or len(items) <= 1:
        return [fn(i) for i in items]
    with ThreadPoolExecutor(max_workers=threads or 8) as ex:
        return list(ex.map(fn, items))


def grads(wl: Workload, step: int, indices: Optional[Sequence[int]] = None, threads: Optional[int] = None):
    idx = list(range(wl.count)) if indices is None else list(indices)
    if threads is None and wl.grad_kind in ("lowrank", "powerlaw"):
        threads = 1          # QR-bound draws: the BLAS threads already use every core
    return _map(lambda k: grad(wl, step, k), idx, threads)


def weights(wl: Workload, indices: Optional[Sequence[int]] = None, threads: Optional[int] = None):
    idx = list(range(wl.count)) if indices is None else list(indices)
    return _map(lambda k: weight(wl, k), idx, threads)


def parity_subset(wl: Workload) -> List[int]:
    """Matrices the fp64 oracle checks at full size.

    Workloads 1-3: all.  GPT-2-XL: layers 0 and 47 (12 matrices).
    MoE sweep: experts 0-3 of each orientation and the three singles.
    """
    if wl.index in (1, 2, 3):
        return list(range(wl.count))
    if wl.index == 4:
        return list(range(0, 6)) + list(range(6 * 47, 6 * 48))
    if wl.index == 5:
        return [0, 1, 2, 3, 64, 65, 66, 67, 128, 129, 130]
    raise ValueError(wl.index)


def random_orthogonal(n: int, seed: int) -> np.ndarray:
    """Haar n x n orthogonal matrix (for invariance tests)."""
    return _haar_columns(np.random.default_rng(seed), n, n)


# --------------------------------------------------------------------------- on-device draws (benchmark)

def _torch_seed(w: int, step: int, k: int, stream: int) -> int:
    base = 1234 + 1000 * w + (step if stream == 1 else 0)
    return (base * 1_000_003 + k) * 4 + stream


def device_tensors(wl: Workload, step: int, device, dtype_grad: bool = True):
    """The workload's gradients at `step` and initial weights drawn on a CUDA device
    with torch's generator: the same recipe as grad_fp32 / weight (shapes, value
    distribution, spectrum, spike, heavy rows), a different random stream.  For the
    benchmark's large workloads, whose numpy draws take tens of seconds; parity tests
    use the numpy draws above.  Returns (weights fp32, gradients bf16 or fp32)."""
    import torch
    gen = torch.Generator(device=device)

    def randn(shape, seed):
        gen.manual_seed(seed)
        return torch.randn(shape, generator=gen, device=device, dtype=torch.float32)

    def haar(n, k, seed):
        q, r = torch.linalg.qr(randn((n, k), seed))
        return q * torch.sign(torch.diagonal(r))[None, :]

    Ws, Gs = [], []
    for k, spec in enumerate(wl.matrices):
        r, c = spec.rows, spec.cols
        Ws.append(0.02 * randn((r, c), _torch_seed(wl.index, 0, k, 2)))
        s1 = _torch_seed(wl.index, step, k, 1)
        if wl.grad_kind == "iid":
            g = randn((r, c), s1)
        elif wl.grad_kind in ("lowrank", "powerlaw"):
            m = min(r, c)
            expo = 1.5 if wl.grad_kind == "lowrank" else 1.0
            sigma = torch.arange(1, m + 1, device=device, dtype=torch.float32) ** (-expo)
            sigma *= math.sqrt(r * c) / torch.linalg.vector_norm(sigma)
            g = (haar(r, m, s1) * sigma[None, :]) @ haar(c, m, s1 + 1).T
            if wl.grad_kind == "lowrank":
                g += 0.01 * randn((r, c), s1 + 2)
        elif wl.grad_kind == "spike":
            sigma_edge = (math.sqrt(r) + math.sqrt(c)) / math.sqrt(c)
            g = randn((r, c), s1) * (1.0 / math.sqrt(c))
            g += (10.0 * sigma_edge) * (haar(r, 8, s1 + 1) @ haar(c, 8, s1 + 2).T)
        elif wl.grad_kind == "heavy_rows":
            g = randn((r, c), s1)
            gen.manual_seed(s1 + 1)
            heavy = torch.randperm(r, generator=gen, device=device)[: int(math.ceil(0.01 * r))]
            g[heavy, :] *= 20.0
        else:
            raise ValueError(wl.grad_kind)
        Gs.append(g.to(torch.bfloat16) if (dtype_grad and wl.grad_dtype == BF16) else g)
    return Ws, Gs
