"""Per-kernel parity on the GPU: the three Newton-Schulz GEMMs (tensor-core bf16
path and fp32 debug path) through muon_ns_phase_run, each against the oracle's
piece of eq. 4 (gram, poly_matrix, ns_update) on the same bf16 inputs widened
exactly to fp64.  Sizes span several 128x256 tiles with ragged tails."""
import os

import numpy as np
import pytest
import torch

import oracle
import muon_newton_schulz_04_b200 as mb
from muon_newton_schulz_04_b200 import build as mbuild

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", params=["pair", "pair-split", "single"])
def opt(request):
    """Handles on the two-CTA GEMM kernel (default), the two-CTA kernel with the last
    round of tiles split over all clusters, and the one-CTA kernel."""
    mbuild.build()
    env = {"pair": ("1", "0"), "pair-split": ("1", "1"), "single": ("0", "0")}[request.param]
    old = {k: os.environ.get(k) for k in ("MUON_GEMM_PAIR", "MUON_GEMM_SPLIT")}
    os.environ["MUON_GEMM_PAIR"], os.environ["MUON_GEMM_SPLIT"] = env
    o = mb.Muon(mb.config())
    yield o
    o.close()
    for k, v in old.items():
        if v is None:
            os.environ.pop(k, None)
        else:
            os.environ[k] = v


def bf16(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).cuda()


def f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


# (2048, 2560): 80 update tiles on 74 clusters -> the tail round runs as 128-column halves;
# (3328, 3328): 91 Gram / polynomial tiles -> the same for the symmetric products.
SHAPES = [(128, 256, 1), (320, 776, 3), (384, 384, 2), (136, 1032, 1), (8, 64, 2), (520, 264, 1), (1024, 1536, 1),
          (2048, 2560, 1), (3328, 3328, 1)]


@pytest.mark.parametrize("m,n,count", SHAPES)
def test_gram_bf16(opt, m, n, count):
    rng = np.random.default_rng(m * 7 + n)
    X = bf16(rng.standard_normal((count, m, n)) / np.sqrt(n))
    out = torch.full((count, m, m), float("nan"), dtype=torch.bfloat16, device="cuda")
    alpha = 0.75
    opt.ns_phase(mb.NS_GRAM, mb.PREC_BF16, m, n, count, alpha, 0.0, x_op=X, out=out)
    opt.sync()
    Xh, A = f64(X), f64(out)
    for z in range(count):
        ref = alpha * oracle.gram(Xh[z])
        bound = 2.0 ** -8 * np.abs(ref) + 1e-5 * alpha * (np.abs(Xh[z]) @ np.abs(Xh[z]).T)
        assert np.all(np.abs(A[z] - ref) <= bound + 1e-30), float(np.max(np.abs(A[z] - ref) - bound))
        assert np.array_equal(A[z], A[z].T)          # mirrored: exactly symmetric


@pytest.mark.parametrize("m,n,count", SHAPES)
def test_poly_bf16(opt, m, n, count):
    rng = np.random.default_rng(m + 3 * n)
    S = rng.standard_normal((count, m, m)) / np.sqrt(m)
    S = S + np.transpose(S, (0, 2, 1))
    A = bf16(S)
    out = torch.full((count, m, m), float("nan"), dtype=torch.bfloat16, device="cuda")
    a, b, c = oracle.NS_COEFFS
    opt.ns_phase(mb.NS_POLY, mb.PREC_BF16, m, m, count, c, b, a_in=A, out=out)
    opt.sync()
    Ah, P = f64(A), f64(out)
    for z in range(count):
        ref = oracle.poly_matrix(Ah[z], b, c)
        bound = 2.0 ** -8 * np.abs(ref) + 1e-5 * (abs(b) * np.abs(Ah[z]) + abs(c) * np.abs(Ah[z]) @ np.abs(Ah[z]))
        assert np.all(np.abs(P[z] - ref) <= bound + 1e-30), float(np.max(np.abs(P[z] - ref) - bound))
        assert np.array_equal(P[z], P[z].T)


@pytest.mark.parametrize("m,n,count", SHAPES)
def test_update_bf16(opt, m, n, count):
    """X' = alpha P X + a X with X = hi + lo (bf16 pair): the product reads hi, the
    a X term reads hi + lo; the result comes back as a bf16 pair as well."""
    rng = np.random.default_rng(m + 5 * n)
    P = bf16(rng.standard_normal((count, m, m)) / np.sqrt(m))
    X = torch.from_numpy(rng.standard_normal((count, m, n)).astype(np.float32)).cuda()
    hi = X.to(torch.bfloat16)
    lo = (X - hi.float()).to(torch.bfloat16)
    out = torch.full((count, m, n), float("nan"), dtype=torch.bfloat16, device="cuda")
    out_lo = torch.full((count, m, n), float("nan"), dtype=torch.bfloat16, device="cuda")
    a = oracle.NS_COEFFS[0]
    alpha = 1.25
    opt.ns_phase(mb.NS_UPDATE, mb.PREC_BF16, m, n, count, alpha, a, x_op=hi, a_in=P, x_master=lo, out=out,
                 out_op=out_lo)
    opt.sync()
    Ph, Hh, Lh = f64(P), f64(hi), f64(lo)
    O = f64(out) + f64(out_lo)
    for z in range(count):
        ref = oracle.ns_update(Ph[z], Hh[z], 0.0) * alpha + a * (Hh[z] + Lh[z])
        bound = 1e-5 * (abs(alpha) * np.abs(Ph[z]) @ np.abs(Hh[z]) + abs(a) * np.abs(Hh[z] + Lh[z])) \
            + 2.0 ** -15 * np.abs(ref)
        assert np.all(np.abs(O[z] - ref) <= bound), float(np.max(np.abs(O[z] - ref) - bound))
    # the high part is the bf16 rounding of the result: the low part is at most half an ulp
    h = f64(out)
    nz = h != 0
    ulp = 2.0 ** (np.floor(np.log2(np.abs(h[nz]))) - 7)
    assert np.all(np.abs(f64(out_lo)[nz]) <= 0.5 * ulp * (1 + 1e-6))


@pytest.mark.parametrize("m,n,count", [(64, 96, 2), (200, 136, 1), (37, 1000, 1)])
def test_phases_fp32_debug(opt, m, n, count):
    rng = np.random.default_rng(m * n)
    X = torch.from_numpy(rng.standard_normal((count, m, n)).astype(np.float32)).cuda()
    A = torch.empty(count, m, m, device="cuda")
    opt.ns_phase(mb.NS_GRAM, mb.PREC_FP32_DEBUG, m, n, count, 0.5, 0.0, x_op=X, out=A)
    P = torch.empty(count, m, m, device="cuda")
    a, b, c = oracle.NS_COEFFS
    opt.ns_phase(mb.NS_POLY, mb.PREC_FP32_DEBUG, m, m, count, c, b, a_in=A, out=P)
    Y = torch.empty(count, m, n, device="cuda")
    opt.ns_phase(mb.NS_UPDATE, mb.PREC_FP32_DEBUG, m, n, count, 1.0, a, x_op=X, a_in=P, x_master=X, out=Y)
    opt.sync()
    Xh = X.cpu().numpy().astype(np.float64)
    for z in range(count):
        Aref = 0.5 * oracle.gram(Xh[z])
        assert np.max(np.abs(A[z].cpu().numpy() - Aref)) <= 1e-5 * np.max(np.abs(Aref)) * np.sqrt(n)
        Pref = oracle.poly_matrix(A[z].cpu().numpy().astype(np.float64), b, c)
        assert np.max(np.abs(P[z].cpu().numpy() - Pref)) <= 1e-5 * np.max(np.abs(Pref)) * np.sqrt(m)
        Yref = oracle.ns_update(P[z].cpu().numpy().astype(np.float64), Xh[z], a)
        assert np.max(np.abs(Y[z].cpu().numpy() - Yref)) <= 1e-5 * np.max(np.abs(Yref)) * np.sqrt(m)


def test_phase_argument_errors(opt):
    X = torch.zeros(1, 12, 16, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(1, 12, 12, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mb.MuonError) as e:
        opt.ns_phase(mb.NS_GRAM, mb.PREC_BF16, 12, 16, 1, 1.0, 0.0, x_op=X, out=out)   # m % 8 != 0
    assert e.value.status == mb.MUON_ERR_UNSUPPORTED
    with pytest.raises(mb.MuonError) as e:
        opt.ns_phase(mb.NS_GRAM, mb.PREC_BF16, 16, 16, 1, 1.0, 0.0, x_op=None, out=out)
    assert e.value.status == mb.MUON_ERR_INVALID
    with pytest.raises(mb.MuonError) as e:
        opt.ns_phase(7, mb.PREC_BF16, 16, 16, 1, 1.0, 0.0, x_op=X, out=out)
    assert e.value.status == mb.MUON_ERR_INVALID
