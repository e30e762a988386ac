"""Pins for the float64 oracle: each check comes from somewhere other than the oracle itself.

Sources of truth used here: hand-derived worked examples (tests/golden/hand_examples.json),
the SVD polar factor (LAPACK), the spectral characterisation of the iteration (singular
vectors kept, singular values mapped by the scalar polynomial), textbook special cases and
a brute-force triple-loop matmul.  The last test plants mistakes in a copy of the
iteration and checks that these pins catch every one of them.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle as O

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")))


def rel(a, b):
    return np.linalg.norm(np.asarray(a) - np.asarray(b)) / max(np.linalg.norm(np.asarray(b)), 1e-300)


def orthogonal(rng, n):
    q, r = np.linalg.qr(rng.standard_normal((n, n)))
    return q * np.sign(np.diag(r))


def with_singular_values(rng, rows, cols, s):
    k = min(rows, cols)
    P = orthogonal(rng, rows)[:, :k]
    Q = orthogonal(rng, cols)[:, :k]
    return (P * s) @ Q.T


# ---------------------------------------------------------------- primitive

def test_matmul_primitive_matches_triple_loop():
    rng = np.random.default_rng(1)
    A = rng.standard_normal((8, 12))
    B = rng.standard_normal((12, 8))
    C = np.zeros((8, 8))
    for i in range(8):
        for j in range(8):
            s = 0.0
            for k in range(12):
                s += A[i, k] * B[k, j]
            C[i, j] = s
    assert np.max(np.abs(C - A @ B)) < 1e-13


def test_gram_step_matches_triple_loop():
    # The Gram and B X products of one step, written as loops over a 4x6 matrix.
    rng = np.random.default_rng(2)
    X = rng.standard_normal((4, 6))
    a, b, c = O.QUINTIC
    A = [[sum(X[i, k] * X[j, k] for k in range(6)) for j in range(4)] for i in range(4)]
    AA = [[sum(A[i][k] * A[k][j] for k in range(4)) for j in range(4)] for i in range(4)]
    Bm = [[b * A[i][j] + c * AA[i][j] for j in range(4)] for i in range(4)]
    Xn = [[a * X[i, j] + sum(Bm[i][k] * X[k, j] for k in range(4)) for j in range(6)] for i in range(4)]
    assert rel(O.ns_iteration(X, a, b, c), np.array(Xn)) < 1e-14


# ---------------------------------------------------------------- worked examples

def test_momentum_worked_example():
    g = GOLD["momentum"]
    M1 = O.momentum_lerp(np.array([[g["M"]]]), np.array([[g["G"]]]), g["beta"])
    assert abs(M1[0, 0] - g["M1"]) < 1e-15
    U = O.nesterov_blend(np.array([[g["G"]]]), M1, g["beta"], True)
    assert abs(U[0, 0] - g["U_nesterov"]) < 1e-15
    U = O.nesterov_blend(np.array([[g["G"]]]), M1, g["beta"], False)
    assert abs(U[0, 0] - g["U_plain"]) < 1e-15


def test_frobenius_worked_example():
    g = GOLD["frobenius"]
    assert O.frobenius_norm(np.array(g["X"])) == g["norm"]
    assert np.allclose(O.frobenius_normalize(np.array(g["X"]), 0.0), g["normalized"], atol=1e-15)


@pytest.mark.parametrize("key,abc,k", [("cubic_k1", O.CUBIC, 1), ("cubic_k2", O.CUBIC, 2), ("quintic_k1", O.QUINTIC, 1)])
def test_ns_diagonal_worked_example(key, abc, k):
    g = GOLD["ns_diagonal"]
    out = O.newton_schulz(np.array(g["U"]), k, abc, g["eps"])
    assert np.max(np.abs(out - np.array(g[key]))) < 1e-14


def test_ns_tall_worked_example():
    g = GOLD["ns_tall"]
    out = O.newton_schulz(np.array(g["U"]), 1, O.CUBIC, g["eps"])
    assert out.shape == (3, 2)
    assert np.max(np.abs(out - np.array(g["cubic_k1"]))) < 1e-14


def test_parameter_write_worked_example():
    g = GOLD["write"]
    assert abs(O.shape_scale(3, 2) - g["scale"]) < 1e-15
    W1 = O.parameter_write(np.array(g["W"]), np.array(g["O"]), g["lr"], g["weight_decay"])
    assert np.max(np.abs(W1 - np.array(g["W1"]))) < 1e-10


def test_muon_step_worked_example():
    # W = 0, M = 0, G = diag(3, 4)/c: U is a positive multiple of diag(3, 4), so with eps = 0
    # the orthogonalised direction is the cubic_k1 diagonal, whatever beta is.
    g = GOLD["ns_diagonal"]
    G = np.array(g["U"]) / 7.0
    hp = O.Hyper(lr=0.5, beta=0.9, weight_decay=0.0, eps=0.0, nesterov=True, ns_steps=1, abc=O.CUBIC)
    W1, M1, Oo = O.muon_step(np.zeros((2, 2)), G, np.zeros((2, 2)), hp)
    assert np.max(np.abs(M1 - 0.1 * G)) < 1e-16
    assert np.max(np.abs(Oo - np.array(g["cubic_k1"]))) < 1e-14
    assert np.max(np.abs(W1 + 0.5 * np.array(g["cubic_k1"]))) < 1e-14


def test_quintic_constants():
    g = GOLD["quintic_constants"]
    assert abs(O.scalar_map(1.0, 1) - g["phi_at_1"]) < 1e-12
    xs = np.linspace(0.0, 1.0, 200001)
    ys = O.scalar_map(xs, 1)
    assert abs(xs[np.argmax(ys)] - g["argmax_on_unit_interval"]) < 1e-4
    assert abs(ys.max() - g["max_on_unit_interval"]) < 1e-5


# ---------------------------------------------------------------- special cases

def test_momentum_special_cases():
    rng = np.random.default_rng(3)
    G, M = rng.standard_normal((5, 7)), rng.standard_normal((5, 7))
    # beta = 0: no memory, the direction is the gradient
    M1 = O.momentum_lerp(M, G, 0.0)
    assert np.array_equal(M1, G)
    assert np.array_equal(O.nesterov_blend(G, M1, 0.0, True), G)
    # beta = 1: the buffer never moves
    M1 = O.momentum_lerp(M, G, 1.0)
    assert np.array_equal(M1, M)
    assert np.array_equal(O.nesterov_blend(G, M1, 1.0, True), M)
    # G = M: a fixed point of the lerp, and of the blend
    M1 = O.momentum_lerp(M, M, 0.95)
    assert np.max(np.abs(M1 - M)) < 1e-15
    assert np.max(np.abs(O.nesterov_blend(M, M1, 0.95, True) - M)) < 1e-15


def test_norm_against_lapack():
    rng = np.random.default_rng(4)
    X = rng.standard_normal((33, 17))
    assert abs(O.frobenius_norm(X) - np.linalg.norm(X, "fro")) < 1e-12
    assert abs(O.frobenius_norm(X) - math.sqrt(np.sum(np.linalg.svd(X, compute_uv=False) ** 2))) < 1e-12


def test_shape_scale():
    assert O.shape_scale(1536, 1536) == 1.0
    assert O.shape_scale(1536, 6144) == 1.0
    assert abs(O.shape_scale(6144, 1536) - 2.0) < 1e-15
    assert abs(O.shape_scale(3072, 1024) - math.sqrt(3.0)) < 1e-15
    assert abs(O.shape_scale(12288, 3072) - 2.0) < 1e-15


# ---------------------------------------------------------------- iteration vs plain definitions

@pytest.mark.parametrize("shape", [(32, 48), (48, 32), (40, 40)])
def test_cubic_converges_to_polar_factor(shape):
    rng = np.random.default_rng(5)
    s = np.linspace(0.1, 1.0, min(shape))
    X = with_singular_values(rng, *shape, s)
    out = O.newton_schulz(X, 40, O.CUBIC, 0.0)
    assert rel(out, O.polar_factor(X)) < 1e-12


def test_cubic_polar_on_gaussian_256():
    # The 256x256 N(0,1) matrix from seed 0: sigma_min / ||X||_F is small, so the step count
    # is chosen from it: log(0.5/s_min)/log(1.5) steps to reach the quadratic basin, plus 8.
    X = np.random.default_rng(0).standard_normal((256, 256))
    s = np.linalg.svd(X, compute_uv=False)
    smin = s[-1] / math.sqrt(np.sum(s * s))
    k = math.ceil(math.log(0.5 / smin) / math.log(1.5)) + 8
    out = O.newton_schulz(X, k, O.CUBIC, 0.0)
    assert rel(out, O.polar_factor(X)) < 1e-10, k


@pytest.mark.parametrize("shape", [(24, 40), (40, 24), (30, 30)])
@pytest.mark.parametrize("k", [1, 2, 5])
@pytest.mark.parametrize("abc", [O.QUINTIC, O.CUBIC, (2.0, -1.5, 0.5)])
def test_iteration_equals_spectral_map(shape, k, abc):
    rng = np.random.default_rng(6)
    X = rng.standard_normal(shape)
    out = O.newton_schulz(X, k, abc, 1e-7)
    assert rel(out, O.spectral_newton_schulz(X, k, abc, 1e-7)) < 1e-12


def test_spectral_map_ill_conditioned():
    # singular values spanning 1e-6 .. 1, as in the conditioning stress set
    rng = np.random.default_rng(7)
    s = np.exp(rng.uniform(np.log(1e-6), 0.0, 48))
    X = with_singular_values(rng, 48, 96, s)
    for k in (5, 10):
        assert rel(O.newton_schulz(X, k), O.spectral_newton_schulz(X, k)) < 1e-11


# ---------------------------------------------------------------- invariants

def test_invariants():
    rng = np.random.default_rng(8)
    X = rng.standard_normal((20, 36))
    base = O.newton_schulz(X, 5)
    # transpose symmetry: the tall path is the wide path transposed, exactly
    assert np.array_equal(O.newton_schulz(X.T, 5), base.T)
    # odd polynomial
    assert np.array_equal(O.newton_schulz(-X, 5), -base)
    # scale invariance (exact with eps = 0, up to rounding)
    b0 = O.newton_schulz(X, 5, eps=0.0)
    assert rel(O.newton_schulz(123.0 * X, 5, eps=0.0), b0) < 1e-13
    # orthogonal equivariance
    P, Q = orthogonal(rng, 20), orthogonal(rng, 36)
    assert rel(O.newton_schulz(P @ X @ Q, 5), P @ base @ Q) < 1e-12


def test_orthonormal_rows_fixed_points():
    rng = np.random.default_rng(9)
    Q = orthogonal(rng, 40)[:16, :]  # 16x40, orthonormal rows
    # the bare cubic step keeps Q where it is
    assert np.max(np.abs(O.ns_iteration(Q, *O.CUBIC) - Q)) < 1e-14
    # with normalisation the result is a scalar multiple of Q: phi^k(1/(sqrt(r)+eps)) Q
    eps = 1e-7
    for abc in (O.CUBIC, O.QUINTIC):
        for k in (1, 5, 30):
            scale = O.scalar_map(1.0 / (math.sqrt(16) + eps), k, abc)
            assert rel(O.newton_schulz(Q, k, abc, eps), scale * Q) < 1e-13
    # for the cubic the scalar goes to 1
    assert abs(O.scalar_map(1.0 / (4 + eps), 40, O.CUBIC) - 1.0) < 1e-12


def test_zero_input_stays_finite():
    # eps keeps the normalisation finite; the zero matrix maps to zero
    out = O.newton_schulz(np.zeros((8, 16)), 5)
    assert np.array_equal(out, np.zeros((8, 16)))


def _zero_direction_pin_holds():
    # A matrix whose gradient and momentum are both zero has U = 0.  With eps = 0 the
    # normalisation would be 0 / 0; the zero matrix is taken as its own direction (the value it
    # has for every eps > 0), so O = 0 and the step leaves exactly (1 - lr wd) W.  With the
    # default eps the same holds without any special case.
    rng = np.random.default_rng(41)
    W = rng.standard_normal((6, 10))
    z = np.zeros_like(W)
    ok = True
    for eps in (0.0, 1e-7):
        hp = O.Hyper(lr=0.05, beta=0.9, weight_decay=0.3, eps=eps, nesterov=True, ns_steps=5)
        with np.errstate(invalid="ignore", divide="ignore"):
            W1, M1, O1 = O.muon_step(W, z, z, hp)
        ok = ok and np.array_equal(O1, z) and np.array_equal(M1, z)
        ok = ok and np.max(np.abs(W1 - (1.0 - 0.05 * 0.3) * W)) == 0.0
    return bool(ok)


def test_zero_direction_with_zero_eps(monkeypatch):
    import oracle.muon_oracle as mo

    assert _zero_direction_pin_holds()
    # a non-zero matrix with eps = 0 is normalised by its norm alone
    X = np.array([[3.0, 4.0]])
    assert np.array_equal(O.frobenius_normalize(X, 0.0), np.array([[0.6, 0.8]]))
    # the unguarded division (0 / 0) turns the zero direction into NaN and fails the pin
    monkeypatch.setattr(mo, "frobenius_normalize", lambda X, eps: X / (mo.frobenius_norm(X) + eps))
    assert not _zero_direction_pin_holds()


def test_ns_flops_counts():
    # square: 3 m^3 + m^3 per step; wide m x n: 3 m^2 n + m^3
    assert O.ns_flops(1536, 1536, 1) == 4 * 1536 ** 3
    assert O.ns_flops(6144, 1536, 5) == 5 * (3 * 1536 * 1536 * 6144 + 1536 ** 3)


# ---------------------------------------------------------------- planted mistakes

def _mutants():
    a, b, c = O.QUINTIC

    def drop_c(X):
        A = X @ X.T
        return a * X + (b * A) @ X

    def wrong_gram(X):
        # the Gram of the other side, still multiplied from the left (square inputs only)
        A = X.T @ X
        B = b * A + c * (A @ A)
        return a * X + B @ X

    def wrong_sign(X):
        A = X @ X.T
        B = b * A - c * (A @ A)
        return a * X + B @ X

    def transposed_update(X):
        A = X @ X.T
        B = b * A + c * (A @ A)
        return a * X + (B @ X) @ np.eye(X.shape[1])[::-1]

    return [drop_c, wrong_gram, wrong_sign, transposed_update]


@pytest.mark.parametrize("mutant", _mutants(), ids=lambda f: f.__name__)
def test_pins_catch_planted_mistakes(mutant, monkeypatch):
    """Each plausible slip in the iteration must fail the spectral pin."""
    import oracle.muon_oracle as mo

    rng = np.random.default_rng(10)
    X = rng.standard_normal((30, 30))
    good = mo.newton_schulz(X, 3)
    monkeypatch.setattr(mo, "ns_iteration", lambda Y, a, b, c: mutant(Y))
    bad = mo.newton_schulz(X, 3)
    assert rel(good, O.spectral_newton_schulz(X, 3)) < 1e-12
    assert rel(bad, O.spectral_newton_schulz(X, 3)) > 1e-3


# ---------------------------------------------------------------- AdamW (the non-matrix half)

def test_adamw_first_step_worked_example():
    # t = 1, m = v = 0: m1 = 0.1 g, v1 = 0.001 g^2, corrected to g and g^2, so with eps = 0
    # the step is lr * sign(g); p = 1, g = 2, lr = 0.1 -> 0.9; with wd = 0.5 -> 0.95 - 0.1
    p1, m1, v1 = O.adamw_step(np.array([1.0]), np.array([2.0]), np.zeros(1), np.zeros(1), 1,
                              lr=0.1, beta1=0.9, beta2=0.999, eps=0.0, weight_decay=0.0)
    assert abs(m1[0] - 0.2) < 1e-15 and abs(v1[0] - 0.004) < 1e-15
    assert abs(p1[0] - 0.9) < 1e-14
    p1, _, _ = O.adamw_step(np.array([1.0]), np.array([2.0]), np.zeros(1), np.zeros(1), 1,
                            lr=0.1, beta1=0.9, beta2=0.999, eps=0.0, weight_decay=0.5)
    assert abs(p1[0] - 0.85) < 1e-14


def test_adamw_constant_gradient_closed_form():
    # with a constant gradient the bias-corrected moments are exactly g and g^2 at every step,
    # so T steps move p by T * lr * g / (|g| + eps)
    rng = np.random.default_rng(20)
    g = rng.standard_normal(50)
    p0 = rng.standard_normal(50)
    p, m, v = p0.copy(), np.zeros(50), np.zeros(50)
    for t in range(1, 8):
        p, m, v = O.adamw_step(p, g, m, v, t, lr=1e-2, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.0)
    assert np.max(np.abs(p - (p0 - 7 * 1e-2 * g / (np.abs(g) + 1e-8)))) < 1e-12


def test_adamw_zero_betas():
    # beta1 = beta2 = 0: no memory, the step is lr * g / (|g| + eps) whatever m and v held
    rng = np.random.default_rng(21)
    p, g, m, v = (rng.standard_normal(30) for _ in range(4))
    v = np.abs(v)
    p1, m1, v1 = O.adamw_step(p, g, m, v, 3, lr=0.05, beta1=0.0, beta2=0.0, eps=1e-6, weight_decay=0.0)
    assert np.array_equal(m1, g) and np.array_equal(v1, g * g)
    assert np.max(np.abs(p1 - (p - 0.05 * g / (np.abs(g) + 1e-6)))) < 1e-15


def test_adamw_pin_catches_missing_bias_correction():
    rng = np.random.default_rng(22)
    g = rng.standard_normal(10)
    m1 = 0.1 * g
    v1 = 0.05 * g * g
    wrong = -1e-2 * m1 / (np.sqrt(v1) + 1e-8)  # the step without bias correction
    right = O.adamw_step(np.zeros(10), g, np.zeros(10), np.zeros(10), 1, lr=1e-2, beta1=0.9, beta2=0.95,
                         eps=1e-8, weight_decay=0.0)[0]
    assert np.max(np.abs(right - wrong)) > 1e-3


def _step_orientation_pin_holds():
    # Stepping the transposed matrix gives the transposed M1 and direction O exactly; only the
    # shape scale changes, since it is taken on the caller's own orientation:
    # (W1 - (1 - lr wd) W) / (-lr sqrt(max(1, r/c))) = O for either orientation.
    rng = np.random.default_rng(31)
    r, c = 24, 10  # tall: the oracle orthogonalises its transpose and transposes back
    W, G, M = (rng.standard_normal((r, c)) for _ in range(3))
    hp = O.Hyper(lr=0.05, beta=0.9, weight_decay=0.2, eps=1e-7, nesterov=True, ns_steps=4)
    W1, M1, O1 = O.muon_step(W, G, M, hp)
    W1t, M1t, O1t = O.muon_step(W.T, G.T, M.T, hp)
    decay = 1.0 - hp.lr * hp.weight_decay
    d = (W1 - decay * W) / (-hp.lr * np.sqrt(r / c))
    dt = (W1t - decay * W.T) / (-hp.lr * 1.0)
    return (np.array_equal(M1t, M1.T) and np.array_equal(O1t, O1.T) and rel(d, O1) < 1e-13
            and rel(dt, O1t) < 1e-13)


def test_full_step_transpose_equivariance():
    assert _step_orientation_pin_holds()
    rng = np.random.default_rng(31)
    r, c = 24, 10
    W, G, M = (rng.standard_normal((r, c)) for _ in range(3))
    # the direction of a tall matrix has orthonormal-ish columns: O^T O near I after enough steps
    hp_many = O.Hyper(lr=0.05, beta=0.9, weight_decay=0.0, eps=1e-7, nesterov=True, ns_steps=60, abc=O.CUBIC)
    _, _, Oc = O.muon_step(W, G, M, hp_many)
    assert rel(Oc.T @ Oc, np.eye(c)) < 1e-6


def test_full_step_without_nesterov_orthogonalises_the_momentum():
    rng = np.random.default_rng(32)
    W, G, M = (rng.standard_normal((6, 9)) for _ in range(3))
    hp = O.Hyper(lr=0.1, beta=0.8, weight_decay=0.0, eps=1e-7, nesterov=False, ns_steps=3)
    _, M1, O1 = O.muon_step(W, G, M, hp)
    # without the Nesterov blend the direction is NS(M1), not NS((1 - beta) G + beta M1)
    assert rel(O1, O.newton_schulz(M1, 3)) < 1e-14
    hp_n = O.Hyper(lr=0.1, beta=0.8, weight_decay=0.0, eps=1e-7, nesterov=True, ns_steps=3)
    _, _, On = O.muon_step(W, G, M, hp_n)
    assert rel(On, O1) > 1e-3


def test_step_pin_catches_planted_mistakes(monkeypatch):
    import math

    import oracle.muon_oracle as mo

    assert _step_orientation_pin_holds()
    # the shape scale taken on the oriented (min x max) shape instead of the caller's
    with monkeypatch.context() as mp:
        mp.setattr(mo, "shape_scale", lambda r, c: math.sqrt(max(r, c) / min(r, c)))
        assert not _step_orientation_pin_holds()
    # weight decay applied after the update instead of to the pre-update W
    with monkeypatch.context() as mp:
        mp.setattr(mo, "parameter_write",
                   lambda W, Ov, lr, wd: (1.0 - lr * wd) * (W - lr * mo.shape_scale(*W.shape) * Ov))
        assert not _step_orientation_pin_holds()


def test_adamw_weight_decay_is_decoupled(monkeypatch):
    # g = 0 with fresh moments: m1 = v1 = 0, so the Adam update is exactly 0 and only the decoupled
    # decay acts, p1 = (1 - lr wd) p.  Adding wd p to the gradient instead (Adam with L2) would
    # move the moments and fail this.
    import oracle.muon_oracle as mo

    p = np.array([1.5, -2.0, 0.25, 3.0])
    z = np.zeros_like(p)
    p1, m1, v1 = O.adamw_step(p, z, z, z, 1, lr=0.01, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1)
    assert np.array_equal(m1, z) and np.array_equal(v1, z)
    assert np.max(np.abs(p1 - (1.0 - 0.01 * 0.1) * p)) < 1e-16

    def l2_in_gradient(p, g, m, v, step, lr, beta1, beta2, eps, weight_decay):
        g = g + weight_decay * p
        m1 = beta1 * m + (1 - beta1) * g
        v1 = beta2 * v + (1 - beta2) * g * g
        mh, vh = m1 / (1 - beta1 ** step), v1 / (1 - beta2 ** step)
        return p - lr * mh / (np.sqrt(vh) + eps), m1, v1

    monkeypatch.setattr(mo, "adamw_step", l2_in_gradient)
    q1, _, _ = mo.adamw_step(p, z, z, z, 1, lr=0.01, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1)
    assert np.max(np.abs(q1 - (1.0 - 0.01 * 0.1) * p)) > 1e-3
