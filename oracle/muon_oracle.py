"""fp64 CPU oracle of one Muon optimizer step.  TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline / reference
leg may import this module.  The CUDA library never calls it and shares no code
with it: this file uses numpy only, with one library matrix product per step
of the method and no blocking, fusion or reordering beyond what the method
states.

Source of every step: the page "Muon: An optimizer for hidden layers in neural
networks" (papers.chlience.com synthesis note), section 4 "Muon 的算法定义",
equations (1)-(5) in the order printed there, plus its section "关键实验/定理",
result 2 (Moonlight: decoupled weight decay, per-shape update scale), and the
sina.com.hk news page "爆肝一篇博客拿下OpenAI offer…", the paragraph that says
Muon runs SGD-momentum, then Newton-Schulz on each update matrix, then applies
it.  Where the pages are silent the reading taken is stated beside the code.

Notation: W (r x c, PyTorch Linear layout), gradient G, momentum buffer B,
update direction U, oriented iterate X (m x n, m = min(r,c)), output O.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

# section 4, eq. (5): the tuned quintic coefficients
NS_COEFFS: Tuple[float, float, float] = (3.4445, -4.7750, 2.0315)
# section 4, closing paragraph: five iterations in practice
NS_STEPS: int = 5
# Not on the pages: the epsilon added to the Frobenius norm (reading: X/(||X||_F + eps)).
DEFAULT_EPS: float = 1e-7

SCALE_NONE = 0
SCALE_MATCH_RMS = 1
SCALE_CUSTOM = 2


def momentum_accumulate(B_prev: np.ndarray, G: np.ndarray, mu: float) -> np.ndarray:
    """B_t = mu * B_{t-1} + G_t  (section 4, eq. (1)); no (1 - mu) dampening is written."""
    return mu * np.asarray(B_prev, dtype=np.float64) + np.asarray(G, dtype=np.float64)


def nesterov_direction(G: np.ndarray, B_t: np.ndarray, mu: float, nesterov: bool) -> np.ndarray:
    """The matrix handed to the orthogonalisation.

    Section 4 says implementations usually take a Nesterov-style momentum and
    prints no formula; the reading taken is U = G_t + mu * B_t with the freshly
    updated B_t.  Without Nesterov the direction is B_t itself (eq. (1))."""
    G = np.asarray(G, dtype=np.float64)
    B_t = np.asarray(B_t, dtype=np.float64)
    return G + mu * B_t if nesterov else B_t.copy()


def orient(M: np.ndarray) -> Tuple[np.ndarray, bool]:
    """Smaller-Gram orientation (section 4, closing paragraph): transpose when rows > cols,
    so that X is m x n with m <= n and X X^T is the m x m Gram matrix."""
    if M.shape[0] > M.shape[1]:
        return M.T, True
    return M, False


def frobenius_normalize(X: np.ndarray, eps: float = DEFAULT_EPS) -> np.ndarray:
    """X / (||X||_F + eps) (section 4, closing paragraph: the input is first scaled by its
    Frobenius norm; eps is this library's reading, the pages give none)."""
    return X / (math.sqrt(float(np.sum(X * X))) + eps)


def gram(X: np.ndarray) -> np.ndarray:
    """A = X X^T, the Gram matrix inside eq. (4)."""
    return X @ X.T


def poly_matrix(A: np.ndarray, b: float, c: float) -> np.ndarray:
    """P = b A + c A^2, so that b(XX^T)X + c(XX^T)^2 X = P X (eq. (4), grouped)."""
    return b * A + c * (A @ A)


def ns_update(P: np.ndarray, X: np.ndarray, a: float) -> np.ndarray:
    """X <- a X + P X, the remaining terms of eq. (4)."""
    return a * X + P @ X


def ns_iteration(X: np.ndarray, coeffs: Sequence[float] = NS_COEFFS) -> np.ndarray:
    """One quintic Newton-Schulz step X <- aX + b(XX^T)X + c(XX^T)^2 X (section 4, eq. (4))."""
    a, b, c = coeffs
    A = gram(X)
    P = poly_matrix(A, b, c)
    return ns_update(P, X, a)


def newton_schulz(M: np.ndarray, steps: int = NS_STEPS, coeffs: Sequence[float] = NS_COEFFS,
                  eps: float = DEFAULT_EPS) -> np.ndarray:
    """Approximate orthogonalisation of M (section 4, eqs. (2), (4), (5)).

    Orient to the smaller Gram, normalise by the Frobenius norm, run `steps`
    quintic iterations, orient back.  The result approximates the polar factor
    U V^T of eq. (2) only loosely: it is U p^steps(S / ||M||_F) V^T, with
    p(s) = a s + b s^3 + c s^5."""
    X, transposed = orient(np.asarray(M, dtype=np.float64))
    X = frobenius_normalize(X, eps)
    for _ in range(steps):
        X = ns_iteration(X, coeffs)
    return X.T if transposed else X


def shape_scale(rows: int, cols: int, mode: int = SCALE_NONE, rms_target: float = 0.2,
                custom: float = 1.0) -> float:
    """Per-shape multiplier of the update (section "关键实验/定理", result 2: Moonlight's
    per-parameter update scale for a shape-independent update RMS).  The pages give
    no formula.  Reading: a full-rank semi-orthogonal r x c matrix has RMS
    1/sqrt(max(r,c)), so MATCH_RMS uses rms_target * sqrt(max(r,c))."""
    if mode == SCALE_NONE:
        return 1.0
    if mode == SCALE_MATCH_RMS:
        return rms_target * math.sqrt(max(rows, cols))
    if mode == SCALE_CUSTOM:
        return float(custom)
    raise ValueError(mode)


def apply_update(W: np.ndarray, O: np.ndarray, lr: float, weight_decay: float = 0.0,
                 scale: float = 1.0) -> np.ndarray:
    """W_{t+1} = W_t - lr * O_t (section 4, eq. (3)) with decoupled weight decay
    (result 2, Moonlight: AdamW-style).  Reading: W - lr*wd*W - lr*scale*O with the
    old W on the right-hand side; wd = 0 and scale = 1 give eq. (3) exactly."""
    W = np.asarray(W, dtype=np.float64)
    return W - lr * weight_decay * W - lr * scale * np.asarray(O, dtype=np.float64)


def muon_step(W: np.ndarray, G: np.ndarray, B: np.ndarray, *, lr: float, momentum: float,
              nesterov: bool = True, weight_decay: float = 0.0, ns_steps: int = NS_STEPS,
              coeffs: Sequence[float] = NS_COEFFS, eps: float = DEFAULT_EPS,
              scale: float = 1.0) -> Dict[str, np.ndarray]:
    """One Muon step for one matrix, every intermediate returned (fp64).

    Order of section 4: momentum (eq. 1) -> Nesterov direction -> orient,
    normalise, Newton-Schulz (eqs. 4, 5) -> update (eq. 3, with result 2's
    weight decay and scale)."""
    B_new = momentum_accumulate(B, G, momentum)
    U = nesterov_direction(G, B_new, momentum, nesterov)
    X, transposed = orient(U)
    norm = math.sqrt(float(np.sum(X * X)))
    O = newton_schulz(U, ns_steps, coeffs, eps)
    W_new = apply_update(W, O, lr, weight_decay, scale)
    return {"W": W_new, "B": B_new, "U": U, "O": O, "norm": np.float64(norm),
            "transposed": np.bool_(transposed)}


def muon_steps(W0: np.ndarray, grads: Sequence[np.ndarray], **hp) -> List[Dict[str, np.ndarray]]:
    """Consecutive Muon steps from B = 0; returns the per-step results."""
    W = np.asarray(W0, dtype=np.float64)
    B = np.zeros_like(W)
    out = []
    for G in grads:
        res = muon_step(W, G, B, **hp)
        W, B = res["W"], res["B"]
        out.append(res)
    return out


def qk_clip(Wq: np.ndarray, Wk: np.ndarray, max_logits: Sequence[float], tau: float,
            head_dim: int) -> Tuple[np.ndarray, np.ndarray]:
    """QK-Clip of MuonClip (section "关键实验/定理", result 3: after the Muon step the
    query and key projections of each attention head are rescaled according to that
    head's maximum attention logit).  The page gives no formula.  Reading: with
    gamma_h = min(1, tau / S_h) for the head's maximum logit S_h, the rows of head h
    (rows h*head_dim .. (h+1)*head_dim - 1 of W_q and of W_k, PyTorch Linear layout)
    are multiplied by sqrt(gamma_h), so every logit q.k of the head is multiplied
    by gamma_h and the head's maximum logit becomes min(S_h, tau)."""
    Wq = np.asarray(Wq, dtype=np.float64).copy()
    Wk = np.asarray(Wk, dtype=np.float64).copy()
    for h, s in enumerate(max_logits):
        gamma = min(1.0, tau / float(s)) if s > 0 else 1.0
        f = math.sqrt(gamma)
        Wq[h * head_dim:(h + 1) * head_dim, :] *= f
        Wk[h * head_dim:(h + 1) * head_dim, :] *= f
    return Wq, Wk
