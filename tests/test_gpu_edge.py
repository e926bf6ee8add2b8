"""Edge cases of the CUDA path: degenerate inputs, ragged and odd shapes, the
scalar (unaligned) path, NaN isolation between matrices of one launch,
orthogonalisation alone, and argument errors through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import muon_newton_schulz_04_b200 as mb
from muon_newton_schulz_04_b200 import build as mbuild

from parity import TOL_O, rel_fro

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    mbuild.build()


def _step_one(shapes, cfg, grads, weights, dtype=torch.float32):
    """One step over single-matrix groups; returns (W, B, O) as fp64 numpy lists."""
    opt = mb.Muon(cfg)
    W = [torch.from_numpy(w.astype(np.float32)).cuda() for w in weights]
    B = [torch.zeros_like(x) for x in W]
    G = [torch.from_numpy(g.astype(np.float32)).to(dtype).cuda() for g in grads]
    opt.step([mb.Group(W=[W[i]], G=[G[i]], B=[B[i]]) for i in range(len(shapes))])
    O = []
    for i, (r, c) in enumerate(shapes):
        o = torch.empty(r, c, device="cuda")
        opt.last_update(i, 0, o)
        O.append(o)
    opt.sync()
    out = ([x.cpu().numpy().astype(np.float64) for x in W], [x.cpu().numpy().astype(np.float64) for x in B],
           [x.cpu().numpy().astype(np.float64) for x in O])
    opt.close()
    return out


@pytest.mark.parametrize("precision", [mb.PREC_BF16, mb.PREC_FP32_DEBUG])
def test_rank_deficient_gradients(precision):
    """The method's degenerate inputs: Newton-Schulz maps zero singular values to
    zero, so a rank-r gradient (here rank 1, 5 and 64) gives a rank-r direction, and
    zero rows of G give zero rows of O.

    In finite precision the iteration amplifies whatever rounding leaves in the null
    space: p(s) ~ a s for small s, so a component entering at iteration j grows by
    a^(5-j+1) and the sum over the five iterations is at most sum_j a^j ~ 580
    (a = 3.4445).  fp32 GEMMs at K <= 1024 leave ~ sqrt(K) 2^-24 ~ 2e-6 of ||X|| per
    iteration, hence a null-space part up to ~1.2e-3 of ||O|| in the fp32 debug path
    (2e-3 below); the bf16-pair iterate (~2^-17 per element) gives ~1e-2, under the
    bf16 tolerance.  So: the part of O in G's column space matches the oracle within
    the path's tolerance, the rest stays under that bound, and the zero rows are zero
    exactly (every product that forms them is a product with zero)."""
    rng = np.random.default_rng(21)
    cases = [((512, 256), 1), ((256, 768), 5), ((1024, 384), 64), ((300, 300), None)]
    shapes = [sh for sh, _ in cases]
    G = []
    for (r, c), k in cases:
        if k is None:
            g = rng.standard_normal((r, c)).astype(np.float32)
            g[::7][:40] = 0.0                                  # 40 zero rows, spread out
        else:
            g = (rng.standard_normal((r, k)) @ rng.standard_normal((k, c))).astype(np.float32)
        G.append(g)
    W0 = [0.02 * rng.standard_normal(sh) for sh in shapes]
    W, B, O = _step_one(shapes, mb.config(precision=precision), G, W0)
    tol = TOL_O[precision]
    null_tol = tol if precision == mb.PREC_BF16 else 2e-3
    for i, ((r, c), k) in enumerate(cases):
        res = oracle.muon_step(W0[i].astype(np.float32).astype(np.float64), G[i].astype(np.float64),
                               np.zeros((r, c)), lr=0.02, momentum=0.95, nesterov=True, eps=1e-7)
        assert np.array_equal(B[i], G[i].astype(np.float64))        # first step from B = 0: B = G exactly
        if k is None:
            zero = np.all(G[i] == 0.0, axis=1)
            assert zero.sum() == 40
            assert np.all(O[i][zero] == 0.0)
            assert rel_fro(O[i], res["O"]) <= tol, (r, c, rel_fro(O[i], res["O"]))
            continue
        Ur = np.linalg.svd(G[i].astype(np.float64), full_matrices=False)[0][:, :k]
        inside = Ur @ (Ur.T @ O[i])
        assert rel_fro(inside, Ur @ (Ur.T @ res["O"])) <= tol, (r, c, k, rel_fro(inside, Ur @ (Ur.T @ res["O"])))
        null = np.linalg.norm(O[i] - inside) / np.linalg.norm(O[i])
        assert null <= null_tol, (r, c, k, null)


CUBIC = (1.5, -0.5, 0.0)      # the classical cubic Newton-Schulz step X <- 1.5X - 0.5XX^TX


@pytest.mark.parametrize("ns_steps,coeffs,precision", [
    (1, None, mb.PREC_BF16), (2, None, mb.PREC_BF16), (3, None, mb.PREC_BF16), (4, None, mb.PREC_BF16),
    (6, None, mb.PREC_BF16), (2, None, mb.PREC_FP32_DEBUG), (4, CUBIC, mb.PREC_BF16), (3, CUBIC, mb.PREC_FP32_DEBUG)])
def test_iteration_count_and_coefficients(ns_steps, coeffs, precision):
    """Other iteration counts (odd and even: the final iterate sits in either buffer of
    the ping-pong pair) and other coefficients (the cubic step, c = 0) against the
    oracle run with the same settings, on a wide, a tall (transposed) and a ragged
    matrix in one grouped call; W from the GPU's O by the oracle's update formula."""
    rng = np.random.default_rng(31 + ns_steps)
    shapes = [(256, 512), (640, 384), (520, 264)]
    G = [rng.standard_normal(sh).astype(np.float32) for sh in shapes]
    W0 = [0.02 * rng.standard_normal(sh) for sh in shapes]
    kw = dict(ns_steps=ns_steps, precision=precision, weight_decay=0.1)
    if coeffs is not None:
        kw.update(ns_a=coeffs[0], ns_b=coeffs[1], ns_c=coeffs[2])
    W, B, O = _step_one(shapes, mb.config(**kw), G, W0)
    for i, sh in enumerate(shapes):
        w0 = W0[i].astype(np.float32).astype(np.float64)
        res = oracle.muon_step(w0, G[i].astype(np.float64), np.zeros(sh), lr=0.02, momentum=0.95, nesterov=True,
                               weight_decay=0.1, ns_steps=ns_steps, eps=1e-7,
                               coeffs=coeffs if coeffs is not None else oracle.NS_COEFFS)
        assert rel_fro(O[i], res["O"]) <= TOL_O[precision], (sh, rel_fro(O[i], res["O"]))
        assert np.array_equal(B[i], G[i].astype(np.float64))
        Wexp = oracle.apply_update(w0, O[i], 0.02, 0.1, 1.0)
        assert np.max(np.abs(W[i] - Wexp) / (np.abs(w0) + 0.02 * np.abs(O[i]) + 1e-30)) <= 1e-6


ODD = [(37, 1000), (1000, 37), (1, 64), (64, 1), (1, 1), (129, 257), (300, 129), (8, 8),
       (1001, 72), (130, 8)]          # tall with 8-aligned columns: vector transpose, ragged rows


@pytest.mark.parametrize("precision,gdtype", [(mb.PREC_BF16, torch.float32), (mb.PREC_FP32_DEBUG, torch.float32),
                                              (mb.PREC_BF16, torch.bfloat16)])
def test_odd_shapes_one_call(precision, gdtype):
    rng = np.random.default_rng(5)
    G = [rng.standard_normal(s).astype(np.float32) for s in ODD]
    # the oracle sees the gradient the kernel reads: bf16-rounded when G is bf16
    G = [torch.from_numpy(g).to(gdtype).float().numpy() for g in G]
    W0 = [0.02 * rng.standard_normal(s) for s in ODD]
    cfg = mb.config(precision=precision, weight_decay=0.1)
    W, B, O = _step_one(ODD, cfg, G, W0, dtype=gdtype)
    for i, s in enumerate(ODD):
        res = oracle.muon_step(W0[i].astype(np.float32).astype(np.float64), G[i].astype(np.float64),
                               np.zeros(s), lr=0.02, momentum=0.95, nesterov=True, weight_decay=0.1, eps=1e-7)
        assert rel_fro(O[i], res["O"]) <= TOL_O[precision], (s, rel_fro(O[i], res["O"]))
        assert np.max(np.abs(B[i] - res["B"]) / (np.abs(G[i]) + 1e-30)) <= 1e-6


def test_zero_gradient_gives_pure_decay():
    s = [(64, 128), (256, 96)]
    W0 = [np.ones(x) * 0.5 for x in s]
    W, B, O = _step_one(s, mb.config(weight_decay=0.1), [np.zeros(x) for x in s], W0)
    for i in range(2):
        assert np.all(O[i] == 0.0) and np.all(B[i] == 0.0)
        assert np.allclose(W[i], np.float32(0.5) * np.float32(1 - np.float32(0.02) * np.float32(0.1)), rtol=1e-6)


@pytest.mark.parametrize("precision,tol", [(mb.PREC_FP32_DEBUG, 1e-6), (mb.PREC_BF16, 3e-5)])
def test_zero_ns_steps_is_normalised_direction(precision, tol):
    """ns_steps = 0 leaves O = U / (||U|| + eps).  The bf16 path stores the iterate as
    a bf16 pair hi + lo (about 16 significant bits), hence its looser bound."""
    rng = np.random.default_rng(6)
    s = [(96, 200), (200, 96)]
    G = [rng.standard_normal(x).astype(np.float32) for x in s]
    W, B, O = _step_one(s, mb.config(ns_steps=0, precision=precision), G, [np.zeros(x) for x in s])
    for i in range(2):
        U = 1.95 * G[i].astype(np.float64)
        assert rel_fro(O[i], U / (np.linalg.norm(U) + 1e-7)) <= tol


@pytest.mark.parametrize("mu,nesterov", [(0.0, 1), (0.9, 0)])
def test_momentum_variants(mu, nesterov):
    rng = np.random.default_rng(7)
    s = [(128, 384)]
    G = [rng.standard_normal(s[0]).astype(np.float32)]
    W, B, O = _step_one(s, mb.config(momentum=mu, nesterov=nesterov), G, [np.zeros(s[0])])
    res = oracle.muon_step(np.zeros(s[0]), G[0].astype(np.float64), np.zeros(s[0]), lr=0.02, momentum=mu,
                           nesterov=bool(nesterov), eps=1e-7)
    assert np.array_equal(B[0], G[0].astype(np.float64))     # B = mu*0 + G exactly
    assert rel_fro(O[0], res["O"]) <= 3e-2


def test_unaligned_views_take_the_scalar_path():
    rng = np.random.default_rng(8)
    r, c = 96, 160
    big = torch.zeros(r * c + 1, device="cuda")
    W = big[1:].view(r, c)                        # 4-byte aligned, not 16
    W.copy_(torch.from_numpy(0.02 * rng.standard_normal((r, c)).astype(np.float32)))
    W0 = W.cpu().numpy().astype(np.float64)
    gbig = torch.zeros(r * c + 2, dtype=torch.bfloat16, device="cuda")
    G = gbig[2:].view(r, c)                       # 4-byte aligned bf16
    G.copy_(torch.from_numpy(rng.standard_normal((r, c)).astype(np.float32)).to(torch.bfloat16))
    bbig = torch.zeros(r * c + 3, device="cuda")
    B = bbig[3:].view(r, c)
    opt = mb.Muon(mb.config())
    opt.step([mb.Group(W=[W], G=[G], B=[B])])
    opt.sync()
    res = oracle.muon_step(W0, G.float().cpu().numpy().astype(np.float64), np.zeros((r, c)), lr=0.02, momentum=0.95,
                           nesterov=True, eps=1e-7)
    assert rel_fro(W.cpu().numpy().astype(np.float64) - W0, res["W"] - W0) <= 3e-2
    assert float(big[0]) == 0.0 and float(bbig[:3].abs().sum()) == 0.0       # nothing written outside the views
    opt.close()


def test_nan_stays_in_its_matrix():
    rng = np.random.default_rng(9)
    s = [(128, 256), (128, 256), (128, 256)]
    G = [rng.standard_normal(x).astype(np.float32) for x in s]
    W0 = [0.02 * rng.standard_normal(x) for x in s]
    clean = _step_one(s, mb.config(), G, W0)
    Gn = [g.copy() for g in G]
    Gn[1][5, 7] = np.nan
    opt = mb.Muon(mb.config())
    W = [torch.from_numpy(w.astype(np.float32)).cuda() for w in W0]
    B = [torch.zeros_like(x) for x in W]
    Gd = [torch.from_numpy(g).cuda() for g in Gn]
    opt.step([mb.Group(W=W, G=Gd, B=B)])                 # one group of three matrices
    opt.sync()
    assert torch.isnan(W[1]).all()
    for i in (0, 2):
        assert np.array_equal(W[i].cpu().numpy().astype(np.float64), clean[0][i])
    opt.close()


@pytest.mark.parametrize("precision", [mb.PREC_BF16, mb.PREC_FP32_DEBUG])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_orthogonalize_matches_oracle(precision, dtype):
    rng = np.random.default_rng(10)
    shapes = [(256, 512, 2), (512, 256, 1), (320, 776, 1), (1000, 37, 1)]
    opt = mb.Muon(mb.config(precision=precision))
    Ms, Os = [], []
    for (r, c, k) in shapes:
        Ms.append([torch.from_numpy(rng.standard_normal((r, c)).astype(np.float32)).to(dtype).cuda() for _ in range(k)])
        Os.append([torch.empty(r, c, device="cuda") for _ in range(k)])
    opt.orthogonalize(list(zip(Ms, Os)))
    opt.sync()
    for g in range(len(shapes)):
        for M, O in zip(Ms[g], Os[g]):
            ref = oracle.newton_schulz(M.float().cpu().numpy().astype(np.float64), eps=1e-7)
            assert rel_fro(O.cpu().numpy().astype(np.float64), ref) <= TOL_O[precision]
    opt.close()


def test_step_argument_errors():
    opt = mb.Muon(mb.config())
    W = torch.zeros(8, 8, device="cuda")
    with pytest.raises(TypeError):
        opt.step([mb.Group(W=[W], G=[torch.zeros(8, 8, dtype=torch.float16, device="cuda")], B=[W])])
    with pytest.raises(ValueError):
        opt.step([mb.Group(W=[W], G=[torch.zeros(8, 9, device="cuda")], B=[W])])
    G8 = torch.zeros(8, 8, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mb.MuonError) as e:                  # B is W: refused before any launch
        opt.step([mb.Group(W=[W], G=[G8], B=[W])])
    assert e.value.status == mb.MUON_ERR_INVALID
    bad = mb.config()
    bad.momentum = 2.0
    with pytest.raises(mb.MuonError) as e:
        opt.set_config(bad)
    assert e.value.status == mb.MUON_ERR_INVALID
    opt.close()
