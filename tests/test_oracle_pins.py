"""Pins of the fp64 oracle to facts outside itself (CPU only).

Each check uses a route independent of the code under test: the printed
coefficients, exact rational arithmetic, a brute-force Jacobi SVD (itself
checked against LAPACK), orthogonal invariances of the definition, and closed
forms of the momentum recursion.  The mutation tests at the end plant
plausible mistakes in a copy of the oracle and show that a pin catches each.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import muon_oracle as mo
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def p_scalar(s, coeffs=oracle.NS_COEFFS):
    a, b, c = coeffs
    return a * s + b * s ** 3 + c * s ** 5


def p_iter(s, k, coeffs=oracle.NS_COEFFS):
    for _ in range(k):
        s = p_scalar(s, coeffs)
    return s


def closed_form_ns(M, steps=5, eps=0.0, coeffs=oracle.NS_COEFFS):
    """U p^steps(S/(||M||_F+eps)) V^T from the brute-force Jacobi SVD."""
    U, S, Vt = oracle.jacobi_svd(M)
    nrm = math.sqrt(float(np.sum(np.asarray(M, dtype=np.float64) ** 2))) + eps
    return (U * p_iter(S / nrm, steps, coeffs)[None, :]) @ Vt


def rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


# ----------------------------------------------------------------------------- golden

def test_coefficients_match_printed_values():
    g = json.load(open(os.path.join(GOLDEN, "ns_coefficients.json")))
    assert oracle.NS_COEFFS == (g["a"], g["b"], g["c"])
    assert oracle.NS_STEPS == g["steps"]


# ----------------------------------------------------------------------------- Jacobi SVD

@pytest.mark.parametrize("shape,rank", [((4, 7), None), ((16, 16), None), ((9, 5), None),
                                        ((12, 12), 5), ((3, 40), None), ((64, 128), None)])
def test_jacobi_svd_against_lapack(shape, rank):
    rng = np.random.default_rng(7)
    M = rng.standard_normal(shape)
    if rank is not None:
        M = rng.standard_normal((shape[0], rank)) @ rng.standard_normal((rank, shape[1]))
    U, S, Vt = oracle.jacobi_svd(M)
    assert np.allclose((U * S) @ Vt, M, atol=1e-12 * np.abs(M).max())
    assert np.allclose(S, np.linalg.svd(M, compute_uv=False), atol=1e-12 * S.max())
    k = min(shape) if rank is None else rank
    assert np.allclose(Vt[:k] @ Vt[:k].T, np.eye(k), atol=1e-12)
    assert np.allclose(U[:, :k].T @ U[:, :k], np.eye(k), atol=1e-12)


# ----------------------------------------------------------------------------- NS closed form

@pytest.mark.parametrize("shape", [(4, 7), (16, 16), (9, 5), (33, 20), (7, 64), (64, 128)])
def test_newton_schulz_equals_polynomial_of_singular_values(shape):
    rng = np.random.default_rng(sum(shape))
    M = rng.standard_normal(shape)
    O = oracle.newton_schulz(M, eps=0.0)
    assert O.shape == M.shape
    assert rel(O, closed_form_ns(M)) < 1e-10


def test_newton_schulz_rank_deficient_closed_form():
    rng = np.random.default_rng(3)
    M = rng.standard_normal((12, 5)) @ rng.standard_normal((5, 20))
    O = oracle.newton_schulz(M, eps=0.0)
    assert rel(O, closed_form_ns(M)) < 1e-10
    s = np.linalg.svd(O, compute_uv=False)
    assert np.all(s[5:] < 1e-10 * s[0])          # zero singular values stay zero (p(0) = 0)


@pytest.mark.parametrize("steps,coeffs", [(1, oracle.NS_COEFFS), (3, oracle.NS_COEFFS), (6, oracle.NS_COEFFS),
                                          (4, (1.5, -0.5, 0.0)), (2, (2.0, -1.5, 0.5))])
def test_other_steps_and_coefficients_follow_the_closed_form(steps, coeffs):
    """The iteration count and (a, b, c) are parameters of one polynomial map,
    U p^steps(S / ||M||_F) V^T with p(s) = a s + b s^3 + c s^5: for the quintic of
    section 4 at other counts and for other coefficients (the classical cubic step
    (1.5, -0.5, 0)).  muon_step passes both on: its first step from B = 0 orthogonalises
    the Nesterov direction U = G + mu G."""
    rng = np.random.default_rng(steps)
    M = rng.standard_normal((24, 40))
    assert rel(oracle.newton_schulz(M, steps=steps, coeffs=coeffs, eps=0.0), closed_form_ns(M, steps, 0.0, coeffs)) < 1e-10
    G = rng.standard_normal((40, 24))
    res = oracle.muon_step(np.zeros((40, 24)), G, np.zeros((40, 24)), lr=0.02, momentum=0.9, nesterov=True,
                           ns_steps=steps, coeffs=coeffs, eps=0.0)
    assert rel(res["O"], closed_form_ns(G + 0.9 * G, steps, 0.0, coeffs)) < 1e-10


def test_newton_schulz_eps_enters_as_norm_plus_eps():
    M = np.random.default_rng(5).standard_normal((6, 10)) * 1e-6
    eps = 1e-7
    assert rel(oracle.newton_schulz(M, eps=eps), closed_form_ns(M, eps=eps)) < 1e-10


@pytest.mark.parametrize("steps", [1, 2, 5])
def test_diagonal_input_exact_rational(steps):
    """X = [diag(d) 0]: every step acts on d entrywise; compare with exact Fractions."""
    d = [Fraction(3, 1), Fraction(1, 2), Fraction(1, 7), Fraction(2, 1), Fraction(1, 100)]
    m, n = len(d), 8
    X = np.zeros((m, n))
    X[np.arange(m), np.arange(m)] = [float(v) for v in d]
    a, b, c = (Fraction(str(v)) for v in oracle.NS_COEFFS)
    nrm = math.sqrt(float(sum(v * v for v in d)))
    out = oracle.newton_schulz(X, steps=steps, eps=0.0)
    for i, v in enumerate(d):
        s = Fraction(float(v) / nrm)          # the normalised entry, one rounding
        for _ in range(steps):
            s = a * s + b * s ** 3 + c * s ** 5
        assert abs(out[i, i] - float(s)) <= 1e-13 * max(1.0, abs(float(s)))
    off = out.copy()
    off[np.arange(m), np.arange(m)] = 0
    assert np.abs(off).max() == 0.0


def test_single_iteration_matches_quintic_definition():
    """One step equals aX + b(XX^T)X + c(XX^T)^2 X with the powers written out."""
    X = np.random.default_rng(11).standard_normal((5, 9))
    a, b, c = oracle.NS_COEFFS
    S = X @ X.T
    want = a * X + b * (S @ X) + c * (S @ (S @ X))
    assert rel(oracle.ns_iteration(X), want) < 1e-13
    # and its pieces
    assert np.allclose(oracle.gram(X), S)
    assert np.allclose(oracle.poly_matrix(S, b, c), b * S + c * (S @ S))
    assert np.allclose(oracle.ns_update(oracle.poly_matrix(S, b, c), X, a), want)


# ----------------------------------------------------------------------------- invariances

def test_orthogonal_equivariance():
    rng = np.random.default_rng(21)
    M = rng.standard_normal((10, 14))
    Q = workloads.random_orthogonal(10, 1)
    R = workloads.random_orthogonal(14, 2)
    assert rel(oracle.newton_schulz(Q @ M @ R, eps=0.0), Q @ oracle.newton_schulz(M, eps=0.0) @ R) < 1e-11


def test_transpose_equivariance_and_orientation():
    M = np.random.default_rng(22).standard_normal((13, 6))
    assert rel(oracle.newton_schulz(M.T), oracle.newton_schulz(M).T) < 1e-13
    X, t = oracle.orient(M)
    assert t and X.shape == (6, 13)
    X, t = oracle.orient(M.T)
    assert not t and X.shape == (6, 13)
    X, t = oracle.orient(np.zeros((4, 4)))
    assert not t


def test_scale_invariance_and_zero():
    M = np.random.default_rng(23).standard_normal((8, 12))
    assert rel(oracle.newton_schulz(37.5 * M, eps=0.0), oracle.newton_schulz(M, eps=0.0)) < 1e-12
    assert np.array_equal(oracle.newton_schulz(np.zeros((5, 9))), np.zeros((5, 9)))


def test_output_band_is_polynomial_image():
    """Singular values of the output lie in p^5's image of the normalised spectrum."""
    rng = np.random.default_rng(24)
    M = rng.standard_normal((20, 30))
    s = np.linalg.svd(M, compute_uv=False)
    s = s / np.linalg.norm(s)
    grid = np.linspace(s.min(), s.max(), 20001)
    img = p_iter(grid, 5)
    so = np.linalg.svd(oracle.newton_schulz(M, eps=0.0), compute_uv=False)
    assert so.min() >= img.min() - 1e-9 and so.max() <= img.max() + 1e-9
    # p(1) = a + b + c = 0.701: the iteration does not converge to the polar factor
    assert abs(p_scalar(1.0) - 0.701) < 1e-12


# ----------------------------------------------------------------------------- momentum / apply

def test_momentum_closed_form_exact():
    rng = np.random.default_rng(31)
    mu = 0.5                                     # exact in binary
    Gs = [rng.integers(-8, 9, size=(3, 4)).astype(np.float64) for _ in range(4)]
    B = np.zeros((3, 4))
    for k, G in enumerate(Gs):
        B = oracle.momentum_accumulate(B, G, mu)
        want = sum(mu ** (k - j) * Gs[j] for j in range(k + 1))
        assert np.array_equal(B, want)
        assert np.array_equal(oracle.nesterov_direction(G, B, mu, True), G + mu * want)
        assert np.array_equal(oracle.nesterov_direction(G, B, mu, False), want)


def test_zero_momentum_reduces_to_gradient():
    G = np.random.default_rng(32).standard_normal((4, 6))
    B = oracle.momentum_accumulate(np.random.default_rng(1).standard_normal((4, 6)), G, 0.0)
    assert np.array_equal(B, G)
    assert np.array_equal(oracle.nesterov_direction(G, B, 0.0, True), G)


def test_apply_update_exact():
    W = np.array([[1.0, -2.0], [0.5, 4.0]])
    O = np.array([[0.25, 1.0], [-1.0, 0.0]])
    assert np.array_equal(oracle.apply_update(W, O, 0.5), W - 0.5 * O)          # eq. (3)
    got = oracle.apply_update(W, O, 0.5, weight_decay=0.25, scale=2.0)
    assert np.array_equal(got, W - 0.125 * W - 1.0 * O)


def test_match_rms_scale_gives_target_rms():
    for r, c in [(64, 256), (256, 64), (100, 100)]:
        Q = np.linalg.qr(np.random.default_rng(r + c).standard_normal((max(r, c), min(r, c))))[0]
        O = Q if r >= c else Q.T                                # exactly semi-orthogonal
        s = oracle.shape_scale(r, c, oracle.SCALE_MATCH_RMS, rms_target=0.2)
        assert abs(np.sqrt(np.mean((s * O) ** 2)) - 0.2) < 1e-12
    assert oracle.shape_scale(3, 5) == 1.0
    assert oracle.shape_scale(3, 5, oracle.SCALE_CUSTOM, custom=0.7) == 0.7


def test_three_steps_against_closed_form_chain():
    """muon_steps equals: momentum sums, SVD closed form of NS, explicit update formula."""
    rng = np.random.default_rng(41)
    W0 = rng.standard_normal((6, 9)) * 0.02
    Gs = [rng.standard_normal((6, 9)) for _ in range(3)]
    lr, mu, wd, eps = 0.02, 0.95, 0.1, 1e-7
    res = oracle.muon_steps(W0, Gs, lr=lr, momentum=mu, nesterov=True, weight_decay=wd, eps=eps)
    W = W0.copy()
    for k in range(3):
        Bk = sum(mu ** (k - j) * Gs[j] for j in range(k + 1))
        Uk = Gs[k] + mu * Bk
        Ok = closed_form_ns(Uk, eps=eps)
        W = W - lr * wd * W - lr * Ok
        assert rel(res[k]["B"], Bk) < 1e-14
        assert rel(res[k]["O"], Ok) < 1e-10
        assert rel(res[k]["W"], W) < 1e-12


# ----------------------------------------------------------------------------- mutations

def _chain_error(shape=(6, 9)):
    """Largest relative gap between oracle.muon_steps (through the module's own
    globals, so monkeypatched steps take effect) and the closed-form chain."""
    rng = np.random.default_rng(61)
    W0 = rng.standard_normal(shape) * 0.02
    Gs = [rng.standard_normal(shape) for _ in range(3)]
    lr, mu, wd = 0.02, 0.95, 0.1
    res = mo.muon_steps(W0, Gs, lr=lr, momentum=mu, nesterov=True, weight_decay=wd, eps=0.0)
    W, err = W0.copy(), 0.0
    for k in range(3):
        Bk = sum(mu ** (k - j) * Gs[j] for j in range(k + 1))
        Ok = closed_form_ns(Gs[k] + mu * Bk)
        W = W - lr * wd * W - lr * Ok
        for e in (rel(res[k]["B"], Bk), rel(res[k]["O"], Ok), rel(res[k]["W"], W)):
            err = max(err, e if np.isfinite(e) else np.inf)
    return err


@pytest.mark.filterwarnings("ignore::RuntimeWarning")
def test_chain_is_clean_without_mutation():
    assert _chain_error() < 1e-10
    assert _chain_error((8, 8)) < 1e-10


def _it_drop_c(X, coeffs=oracle.NS_COEFFS):
    a, b, c = coeffs
    A = X @ X.T
    return a * X + (b * A) @ X


def _it_sign_b(X, coeffs=oracle.NS_COEFFS):
    a, b, c = coeffs
    A = X @ X.T
    return a * X + (-b * A + c * A @ A) @ X


def _it_no_a(X, coeffs=oracle.NS_COEFFS):
    a, b, c = coeffs
    A = X @ X.T
    return X + (b * A + c * A @ A) @ X


def _it_right_multiply(X, coeffs=oracle.NS_COEFFS):
    a, b, c = coeffs              # P applied on the wrong side (conformable when square)
    A = X @ X.T
    return a * X + X @ (b * A + c * A @ A)


def _it_transposed_gram_operand(X, coeffs=oracle.NS_COEFFS):
    a, b, c = coeffs              # A = X X (not X X^T), conformable when square
    A = X @ X
    return a * X + (b * A + c * A @ A) @ X


@pytest.mark.parametrize("fn,shape", [(_it_drop_c, (6, 9)), (_it_sign_b, (6, 9)), (_it_no_a, (6, 9)),
                                      (_it_right_multiply, (8, 8)),
                                      (_it_transposed_gram_operand, (8, 8))])
def test_pins_catch_planted_iteration_mistakes(fn, shape, monkeypatch):
    monkeypatch.setattr(mo, "ns_iteration", fn)
    assert _chain_error(shape) > 1e-3


@pytest.mark.parametrize("name,fn", [
    ("momentum_accumulate", lambda B, G, mu: mu * B + (1 - mu) * G),           # dampening
    ("momentum_accumulate", lambda B, G, mu: B + mu * G),                      # swapped roles
    ("nesterov_direction", lambda G, B, mu, nesterov: B.copy()),               # Nesterov dropped
    ("nesterov_direction", lambda G, B, mu, nesterov: G + mu * G),             # stale buffer
    ("frobenius_normalize", lambda X, eps=0.0: X),                             # no normalisation
    ("frobenius_normalize", lambda X, eps=0.0: X / np.abs(X).max()),           # wrong norm
    ("apply_update", lambda W, O, lr, weight_decay=0.0, scale=1.0:
        (W - lr * scale * O) * (1 - lr * weight_decay)),                       # decay on new W
    ("apply_update", lambda W, O, lr, weight_decay=0.0, scale=1.0:
        W - lr * weight_decay * W + lr * scale * O),                           # sign
])
@pytest.mark.filterwarnings("ignore::RuntimeWarning")
def test_pins_catch_planted_step_mistakes(name, fn, monkeypatch):
    monkeypatch.setattr(mo, name, fn)
    assert _chain_error() > 1e-6


# ----------------------------------------------------------------------------- QK-Clip

def _head_max_logits(Wq, Wk, Xin, head_dim):
    """Per-head maximum of q.k over all query/key token pairs of the input batch."""
    q = Xin @ Wq.T
    k = Xin @ Wk.T
    out = []
    for h in range(Wq.shape[0] // head_dim):
        sl = slice(h * head_dim, (h + 1) * head_dim)
        out.append(float(np.max(q[:, sl] @ k[:, sl].T)))
    return out


def test_qk_clip_caps_each_head_at_tau():
    rng = np.random.default_rng(71)
    heads, hd, d = 4, 8, 32
    Wq = rng.standard_normal((heads * hd, d))
    Wk = rng.standard_normal((heads * hd, d))
    Xin = rng.standard_normal((10, d))
    S = _head_max_logits(Wq, Wk, Xin, hd)
    tau = float(np.median(S))
    Wq2, Wk2 = oracle.qk_clip(Wq, Wk, S, tau, hd)
    S2 = _head_max_logits(Wq2, Wk2, Xin, hd)
    for s, s2 in zip(S, S2):
        assert abs(s2 - min(s, tau)) <= 1e-9 * abs(s)
    # heads at or below tau are bit-for-bit untouched
    for h, s in enumerate(S):
        if s <= tau:
            assert np.array_equal(Wq2[h * hd:(h + 1) * hd], Wq[h * hd:(h + 1) * hd])


def test_qk_clip_pin_catches_unsplit_scale(monkeypatch):
    """Scaling only W_q by gamma (not sqrt(gamma) on both) also caps the logits, but the
    pages' reading splits it: check the factor on each side."""
    rng = np.random.default_rng(72)
    Wq = rng.standard_normal((8, 4))
    Wk = rng.standard_normal((8, 4))
    Wq2, Wk2 = oracle.qk_clip(Wq, Wk, [4.0, 1.0], 1.0, 4)
    assert np.allclose(Wq2[:4], 0.5 * Wq[:4]) and np.allclose(Wk2[:4], 0.5 * Wk[:4])
    assert np.array_equal(Wq2[4:], Wq[4:]) and np.array_equal(Wk2[4:], Wk[4:])
