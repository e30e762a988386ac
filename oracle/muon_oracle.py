"""Float64 CPU oracle for the Muon optimizer step on 2-D weight matrices.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py`` (its ``cpu_baseline`` leg and its ``--impl reference`` arm) may
import or run anything in this package.  The CUDA library and its Python
binding never import it, and it imports nothing from them: the two sides share
no code.  Inputs reach it as plain float64 NumPy arrays (the exact values the
GPU sees, widened from their storage type).

What the pages fix, and what they leave open
--------------------------------------------
* "开发者千美元训3.8B模型 击败GPT-2" (aiproducthub, little-lm 3.8B news flash),
  影响 paragraph: the hybrid optimizer applies Newton-Schulz orthogonalisation
  to the matrix parameters and AdamW to the rest.
* "把 GPT-2 的训练租金估算从 4.3 万美元压到 40 美元 ..." (magicnetworld), the
  glossary table, row "Muon": an orthogonalised-momentum optimizer for matrix
  parameters.
* "Karpathy 只花 $72 就訓練出 GPT-2" (gu-log), section
  "那些讓 600 倍加速成為可能的技術", and linkstar.cloud article 169, section
  "删不掉"的优化器: the optimizer could not be removed from the recipe.

None of the pages prints a formula, a coefficient, a step count, a scale or a
dtype.  This oracle therefore takes the plainest reading of "orthogonalised
momentum by Newton-Schulz" that the rest of the material supports, one step at
a time, in this order:

  1. momentum as a lerp          M1 = beta*M + (1 - beta)*G
  2. Nesterov blend              U  = (1 - beta)*G + beta*M1   (else U = M1)
  3. orientation                 X  = U, or U^T when rows > cols (so that the
                                 Gram matrix is the small side)
  4. Frobenius normalisation     X  = X / (||X||_F + eps)
  5. k Newton-Schulz steps       A = X X^T;  B = b*A + c*A A;  X = a*X + B X
  6. orientation back            O  = X, or X^T when rows > cols
  7. parameter write             W1 = (1 - lr*wd)*W - lr*sqrt(max(1, rows/cols))*O

Every reading (the lerp form of the momentum, the Nesterov form, eps added to
the norm rather than to its square, weight decay applied to the pre-update W,
the scale taken on the caller's own rows/cols) is listed with its reason in the
repository's design notes.  A library matmul (``numpy.matmul`` in float64)
serves as the one primitive; nothing is blocked, fused or reordered.

Parity pins (tests/test_oracle.py, all CPU):
  * momentum_lerp / nesterov_blend / frobenius_normalize / parameter_write:
    hand-computed worked examples in tests/golden/, special cases
    (beta = 0, beta = 1, G = M), the textbook Frobenius norm of a 3-4-5 vector;
    a zero direction with eps = 0 leaves exactly (1 - lr wd) W.
  * newton_schulz: the cubic (1.5, -0.5, 0) converges to the SVD polar factor
    U V^T; for any (a, b, c) the result equals U diag(phi^k(s_i / (||X||+eps))) V^T
    with phi(x) = a x + b x^3 + c x^5 iterated as a scalar; odd symmetry,
    transpose symmetry, scale invariance, orthogonal equivariance, fixed points
    of orthonormal inputs; a hand-derived 2x2 diagonal example.
  * the matmul primitive against a brute-force triple loop.
  * adamw_step: a hand-derived first step, the closed form for a constant gradient
    (bias-corrected moments equal g and g^2 at every step), the beta = 0 special case.
No function here is unpinned.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

# Coefficient triples for the Newton-Schulz polynomial phi(x) = a x + b x^3 + c x^5.
# QUINTIC is the widely used fast-converging set; CUBIC is the classical iteration,
# which converges to the polar factor of the input.
QUINTIC = (3.4445, -4.7750, 2.0315)
CUBIC = (1.5, -0.5, 0.0)


@dataclass(frozen=True)
class Hyper:
    """Hyper-parameters of one Muon step (plain values, no defaults hidden elsewhere)."""

    lr: float = 0.02
    beta: float = 0.95
    weight_decay: float = 0.0
    eps: float = 1e-7
    nesterov: bool = True
    ns_steps: int = 5
    abc: tuple = QUINTIC


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def momentum_lerp(M, G, beta: float) -> np.ndarray:
    """Step 1, momentum as a lerp of the buffer toward the gradient: beta*M + (1-beta)*G.

    The pages call Muon an orthogonalised *momentum* optimizer (magicnetworld,
    glossary table, row "Muon") but give no update rule; the lerp form is the
    reading taken here.
    """
    M, G = _f64(M), _f64(G)
    return beta * M + (1.0 - beta) * G


def nesterov_blend(G, M1, beta: float, nesterov: bool) -> np.ndarray:
    """Step 2, the direction handed to the orthogonaliser.

    With Nesterov look-ahead it is the lerp of the gradient toward the *updated*
    buffer, (1-beta)*G + beta*M1; without it, the updated buffer itself.
    """
    G, M1 = _f64(G), _f64(M1)
    if nesterov:
        return (1.0 - beta) * G + beta * M1
    return M1.copy()


def frobenius_norm(X) -> float:
    """sqrt of the sum of squares of all entries."""
    X = _f64(X)
    return math.sqrt(float(np.sum(X * X)))


def frobenius_normalize(X, eps: float) -> np.ndarray:
    """Step 4: X / (||X||_F + eps).  eps is added to the norm, not to its square.

    The all-zero matrix has no direction.  For every eps > 0 it normalises to the zero
    matrix (0 / eps), and with eps = 0 it takes that same value, its limit as eps -> 0+,
    instead of 0 / 0: a matrix whose momentum direction is exactly zero gets a zero update,
    so only the weight decay acts on it.
    """
    X = _f64(X)
    d = frobenius_norm(X) + eps
    if d == 0.0:
        return np.zeros_like(X)
    return X / d


def ns_iteration(X, a: float, b: float, c: float) -> np.ndarray:
    """One Newton-Schulz step on a wide (or square) X: A = X X^T, B = b A + c A A, X' = a X + B X.

    Written for X with rows <= cols so that A is the small (rows x rows) Gram matrix.
    """
    X = _f64(X)
    A = X @ X.T
    B = b * A + c * (A @ A)
    return a * X + B @ X


def newton_schulz(U, steps: int, abc=QUINTIC, eps: float = 1e-7) -> np.ndarray:
    """Steps 3-6: orient, normalise, iterate ``steps`` times, orient back.

    Tall inputs (rows > cols) are transposed first so the Gram matrix is
    min(rows, cols) square; square inputs are not transposed.
    """
    U = _f64(U)
    if U.ndim != 2:
        raise ValueError("newton_schulz expects a 2-D matrix")
    a, b, c = abc
    tall = U.shape[0] > U.shape[1]
    X = U.T if tall else U
    X = frobenius_normalize(X, eps)
    for _ in range(steps):
        X = ns_iteration(X, a, b, c)
    return X.T if tall else X


def shape_scale(rows: int, cols: int) -> float:
    """sqrt(max(1, rows/cols)) on the caller's own orientation of the matrix."""
    return math.sqrt(max(1.0, rows / cols))


def parameter_write(W, O, lr: float, weight_decay: float) -> np.ndarray:
    """Step 7: decoupled weight decay on the pre-update W, then the scaled orthogonal step."""
    W, O = _f64(W), _f64(O)
    rows, cols = W.shape
    return (1.0 - lr * weight_decay) * W - lr * shape_scale(rows, cols) * O


def muon_step(W, G, M, hp: Hyper):
    """One Muon step for one matrix.  Returns (W1, M1, O), all float64."""
    W, G, M = _f64(W), _f64(G), _f64(M)
    if not (W.shape == G.shape == M.shape) or W.ndim != 2:
        raise ValueError("W, G, M must be 2-D and of one shape")
    M1 = momentum_lerp(M, G, hp.beta)
    U = nesterov_blend(G, M1, hp.beta, hp.nesterov)
    O = newton_schulz(U, hp.ns_steps, hp.abc, hp.eps)
    W1 = parameter_write(W, O, hp.lr, hp.weight_decay)
    return W1, M1, O


def muon_step_set(Ws, Gs, Ms, hp: Hyper):
    """The step over a parameter set: each matrix independently, in order."""
    out = [muon_step(W, G, M, hp) for W, G, M in zip(Ws, Gs, Ms)]
    return [o[0] for o in out], [o[1] for o in out], [o[2] for o in out]


# ---------------------------------------------------------------------------
# AdamW for the parameters that are not matrices.
# ---------------------------------------------------------------------------

def adamw_step(p, g, m, v, step: int, lr: float, beta1: float, beta2: float, eps: float,
               weight_decay: float):
    """One AdamW step (returns p1, m1, v1 as float64).

    The hybrid recipe hands every parameter that is not a 2-D matrix to AdamW
    ("开发者千美元训3.8B模型 击败GPT-2", aiproducthub, 影响 paragraph).  The pages
    give no formula; this is the plainest reading, the decoupled-weight-decay Adam
    with bias correction, in its usual order:
      m1 = beta1 m + (1 - beta1) g;  v1 = beta2 v + (1 - beta2) g^2
      mh = m1 / (1 - beta1^t);       vh = v1 / (1 - beta2^t)      (t = step >= 1)
      p1 = (1 - lr wd) p - lr mh / (sqrt(vh) + eps)
    """
    p, g, m, v = _f64(p), _f64(g), _f64(m), _f64(v)
    if step < 1:
        raise ValueError("step counts from 1")
    m1 = beta1 * m + (1.0 - beta1) * g
    v1 = beta2 * v + (1.0 - beta2) * g * g
    mh = m1 / (1.0 - beta1 ** step)
    vh = v1 / (1.0 - beta2 ** step)
    p1 = (1.0 - lr * weight_decay) * p - lr * mh / (np.sqrt(vh) + eps)
    return p1, m1, v1


# ---------------------------------------------------------------------------
# Plain definitions the iteration is pinned against (used by tests only).
# ---------------------------------------------------------------------------

def polar_factor(X) -> np.ndarray:
    """U V^T from the thin SVD X = U S V^T: the orthogonal factor of the polar decomposition."""
    U, _, Vt = np.linalg.svd(_f64(X), full_matrices=False)
    return U @ Vt


def scalar_map(x, steps: int, abc=QUINTIC):
    """phi iterated ``steps`` times on scalars, phi(x) = a x + b x^3 + c x^5."""
    a, b, c = abc
    x = _f64(x)
    for _ in range(steps):
        x = a * x + b * x ** 3 + c * x ** 5
    return x


def spectral_newton_schulz(U, steps: int, abc=QUINTIC, eps: float = 1e-7) -> np.ndarray:
    """What the iteration must equal: singular vectors kept, singular values mapped by phi^k.

    With X = P diag(s) Q^T, ||X||_F = sqrt(sum s^2), the k-step result is
    P diag(phi^k(s / (||X||_F + eps))) Q^T.  Computed from the SVD, not by matmul iteration.
    """
    P, s, Qt = np.linalg.svd(_f64(U), full_matrices=False)
    x = s / (math.sqrt(float(np.sum(s * s))) + eps)
    return (P * scalar_map(x, steps, abc)) @ Qt


def ns_flops(rows: int, cols: int, steps: int) -> int:
    """Algorithmic flops of the iteration (2 per multiply-add, symmetric products counted once).

    Per step with m = min, n = max: m*m*n (Gram, half of 2 m^2 n) + m^3 (A A, half of
    2 m^3) + 2 m^2 n (B X).
    """
    m, n = min(rows, cols), max(rows, cols)
    return steps * (3 * m * m * n + m ** 3)
