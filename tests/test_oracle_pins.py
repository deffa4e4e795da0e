"""Pins of the fp64 oracle to what the pages and the mathematics fix (CPU only).

Every function of the oracle is checked against something other than itself:
printed worked examples (tests/golden), closed forms, special cases that reduce to
round-to-nearest, brute force, and independent least-squares solves on the token
matrices.
"""

import numpy as np
import pytest

import oracle as O


def sse(X, cand, w):
    """||X (cand - w)||^2 summed over samples, as in the pages' two self-checks."""
    d = np.asarray(cand, float) - np.asarray(w, float)
    return float(np.sum((np.asarray(X) @ d) ** 2))


# ------------------------------------------------------------------ two-weight example

def test_two_weight_example_gram_and_inverse(golden):
    g = golden("two_weight_example.txt")
    H = O.gram(g["X"])
    np.testing.assert_allclose(H, g["H"], atol=1e-12)
    np.testing.assert_allclose(np.linalg.inv(H), g["P"], atol=1e-12)


def test_two_weight_example_first_step_and_final(golden):
    g = golden("two_weight_example.txt")
    H, w = g["H"], g["w"]
    s = np.array([g["scale"]])
    bits = int(g["bits"])
    codes, W_hat, loss, trace = O.obq_sweep(H, w[None, :], s, bits, return_trace=True)
    np.testing.assert_allclose(trace[0][0] - w, g["first_step_delta"], atol=1e-12)
    np.testing.assert_allclose(trace[0][0], g["trace_after_step0"], atol=1e-12)
    assert sse(g["X"], trace[0][0], w) == pytest.approx(g["sse_after_step0"], abs=1e-12)
    np.testing.assert_array_equal(W_hat[0], g["final"])
    np.testing.assert_array_equal(codes[0], g["final_codes"])
    assert sse(g["X"], W_hat[0], w) == pytest.approx(g["sse_final"], abs=1e-12)
    rtn = O.dequantize(O.quantize_codes(w, s[0], bits), s[0], bits)
    np.testing.assert_array_equal(rtn, g["rtn"])
    assert sse(g["X"], rtn, w) == pytest.approx(g["sse_rtn"], abs=1e-12)
    assert np.mean((rtn - w) ** 2) == pytest.approx(g["weight_mse_rtn"], abs=1e-12)
    assert np.mean((W_hat[0] - w) ** 2) == pytest.approx(g["weight_mse_final"], abs=1e-12)
    # the per-step increase r^2 / (2 P_qq) sums to the final output error
    assert loss[0] == pytest.approx(g["sse_final"], abs=1e-12)


def test_two_weight_example_row_form(golden):
    g = golden("two_weight_example.txt")
    U = O.upper_factor(g["H"])
    np.testing.assert_allclose(U.T @ U, g["P"], atol=1e-12)
    assert U[1, 1] ** 2 == pytest.approx(g["U11_squared"], abs=1e-12)
    assert abs(U[1, 1] ** 2 - g["P"][1, 1]) > 0.1
    codes, W_hat, _ = O.row_form_sweep(U, g["w"][None, :], np.array([g["scale"]]),
                                       int(g["bits"]), blocksize=2)
    np.testing.assert_allclose(W_hat[0], g["final"], atol=1e-12)


# ------------------------------------------------------------------ three-weight example

def test_three_weight_counterexample(golden):
    g = golden("three_weight_counterexample.txt")
    H = O.gram(g["X"])
    np.testing.assert_allclose(H, g["H"], atol=1e-12)
    np.testing.assert_allclose(np.linalg.inv(H), g["P"], atol=1e-12)
    np.testing.assert_allclose(O.upper_factor(H), g["U"], atol=1e-12)
    w, s, bits = g["w"], np.array([g["scale"]]), int(g["bits"])
    for mode in ("schur", "direct"):
        codes, W_hat, loss, trace = O.obq_sweep(H, w[None, :], s, bits, mode=mode,
                                                return_trace=True)
        np.testing.assert_allclose(trace[0][0], g["trace_after_step0"], atol=1e-12)
        np.testing.assert_allclose(trace[1][0], g["trace_after_step1"], atol=1e-12)
        np.testing.assert_allclose(W_hat[0], g["final"], atol=1e-12)
        assert sse(g["X"], W_hat[0], w) == pytest.approx(g["sse_sequential"], abs=1e-12)
    for B in (1, 2, 3):
        _, W_row, _ = O.row_form_sweep(g["U"], w[None, :], s, bits, blocksize=B)
        np.testing.assert_allclose(W_row[0], g["final"], atol=1e-12)
    rtn = O.dequantize(O.quantize_codes(w, s[0], bits), s[0], bits)
    assert sse(g["X"], rtn, w) == pytest.approx(g["sse_rtn"], abs=1e-12)
    best, arg = O.brute_force_best(H, w, range(-8, 8))
    assert best == pytest.approx(g["sse_global_best"], abs=1e-12)
    assert arg == [tuple(g["global_best"])]
    assert len(list(range(-8, 8))) ** 3 == g["grid_points"]


# ------------------------------------------------------------------ damping

def test_rank_one_needs_damping(golden):
    g = golden("rank_one_damping.txt")
    H = O.gram(np.atleast_2d(g["X"]))
    assert np.linalg.matrix_rank(H) == 1
    H0, dead0 = O.dead_and_damp(H, g["percdamp_singular"])
    assert not dead0.any()
    assert not O.is_positive_definite(H0)
    H1, _ = O.dead_and_damp(H, g["percdamp_default"])
    assert O.is_positive_definite(H1)
    # the increment is percdamp * mean(diag H)
    np.testing.assert_allclose(np.diag(H1) - np.diag(H), 0.01 * np.mean(np.diag(H)))
    with pytest.raises(np.linalg.LinAlgError):
        O.solve_layer(H, np.array([[0.3, -0.2]]), 4, percdamp=0.0)


def test_damping_scales_with_H_and_dead_fix():
    rng = np.random.default_rng(0)
    X = rng.standard_normal((50, 6))
    X[:, 2] = 0.0                                  # coordinate 2 never excited
    H = O.gram(X)
    Hd, dead = O.dead_and_damp(H, 0.01)
    assert dead.tolist() == [False, False, True, False, False, False]
    H_fix = H.copy()
    H_fix[2, 2] = 1.0
    np.testing.assert_allclose(np.diag(Hd), np.diag(H_fix) + 0.01 * np.mean(np.diag(H_fix)))
    # a positive scale of H scales the damped live diagonal by the same factor
    Hd3, _ = O.dead_and_damp(3.0 * H, 0.01)
    live = ~dead
    H_fix3 = 3.0 * H
    H_fix3[2, 2] = 1.0
    np.testing.assert_allclose(np.diag(Hd3)[live],
                               3.0 * np.diag(H)[live] + 0.01 * np.mean(np.diag(H_fix3)))
    # dead weights are zeroed and end on code z (value 0)
    W = rng.standard_normal((4, 6)) * 0.02
    out = O.solve_layer(H, W, 3, percdamp=0.01)
    assert np.all(out["W_hat"][:, 2] == 0.0)
    assert np.all(out["codes"][:, 2] == 4)


# ------------------------------------------------------------------ grid and rounding

@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_symmetric_grid(bits):
    rng = np.random.default_rng(bits)
    W = rng.standard_normal((16, 40))
    s, z = O.symmetric_scale(W, bits)
    assert z == 2 ** (bits - 1)
    c = O.quantize_codes(W, s[:, None], bits)
    assert c.min() >= 0 and c.max() <= 2 ** bits - 1
    q = O.dequantize(c, s[:, None], bits)
    lv = q / s[:, None]
    np.testing.assert_allclose(lv, np.round(lv), atol=1e-12)
    lv = np.round(lv)
    assert lv.min() >= -2 ** (bits - 1) and lv.max() <= 2 ** (bits - 1) - 1
    # a channel whose scale is exact puts -amax and +amax on the grid edges:
    # -amax / s = -(2^b - 1) / 2 is a tie that goes to the even level -2^(b-1)
    amax = (2 ** bits - 1) / 2.0
    s1, _ = O.symmetric_scale(np.array([[-amax, 0.25, amax]]), bits)
    assert s1[0] == 1.0
    edge = O.quantize_codes(np.array([-amax, amax]), s1[0], bits)
    np.testing.assert_array_equal(edge, [0, 2 ** bits - 1])


def test_round_half_to_even():
    # ties go to the even neighbour ("最近偶数舍入")
    w = np.array([0.5, 1.5, 2.5, -0.5, -1.5, 0.49, 0.51])
    c = O.quantize_codes(w, 1.0, 4) - 8
    np.testing.assert_array_equal(c, [0, 2, 2, 0, -2, 0, 1])
    assert O.symmetric_scale(np.zeros((1, 3)), 4)[0][0] == 1.0


# ------------------------------------------------------------------ forms agree

def _random_problem(K, N, seed, M=None):
    rng = np.random.default_rng(seed)
    M = M or 3 * K
    X = rng.standard_normal((M, K)) @ rng.standard_normal((K, K)) / np.sqrt(K)
    H = O.gram(X)
    Hd, _ = O.dead_and_damp(H, 0.01)
    W = rng.standard_normal((N, K)) * 0.02
    return X, H, Hd, W


@pytest.mark.parametrize("K,seed", [(3, 1), (7, 2), (12, 3), (16, 4)])
def test_direct_schur_and_row_forms_agree(K, seed):
    X, H, Hd, W = _random_problem(K, 9, seed)
    s, _ = O.symmetric_scale(W, 3)
    c_dir, w_dir, l_dir = O.obq_sweep(Hd, W, s, 3, mode="direct")
    c_sch, w_sch, l_sch = O.obq_sweep(Hd, W, s, 3, mode="schur")
    np.testing.assert_array_equal(c_dir, c_sch)
    np.testing.assert_allclose(w_dir, w_sch, atol=1e-12)
    np.testing.assert_allclose(l_dir, l_sch, rtol=1e-10)
    U = O.upper_factor(Hd)
    for B in (1, 2, 4, 8, K):
        c_row, w_row, E = O.row_form_sweep(U, W, s, 3, B)
        np.testing.assert_array_equal(c_row, c_sch)
        np.testing.assert_allclose(w_row, w_sch, atol=1e-12)
        # per-channel loss: sum r^2/(2 P_qq) = 1/2 sum E^2
        np.testing.assert_allclose(0.5 * np.sum(E ** 2, axis=1), l_sch, rtol=1e-9)


@pytest.mark.parametrize("K", [4, 9, 16])
def test_U_diagonal_is_free_set_pivot(K):
    _, _, Hd, _ = _random_problem(K, 1, 10 + K)
    U = O.upper_factor(Hd)
    assert np.allclose(np.tril(U, -1), 0.0)
    for j in range(K):
        P_F = np.linalg.inv(Hd[j:, j:])
        assert U[j, j] ** 2 == pytest.approx(P_F[0, 0], rel=1e-10)


@pytest.mark.parametrize("K,t", [(9, 4), (16, 1), (16, 15)])
def test_U_trailing_block_is_factor_of_trailing_block(K, t):
    # H_d = V V^T with V = U^-1 upper, so the trailing principal block of H_d only sees
    # the trailing block of V: U[T, T] is the factor of H_d[T, T] alone (the property
    # the full-size GPU tests sample), and U H_d U^T = I on every row pair
    _, _, Hd, _ = _random_problem(K, 1, 40 + K + t)
    U = O.upper_factor(Hd)
    T = slice(K - t, K)
    np.testing.assert_allclose(U[T, T], O.upper_factor(Hd[T, T]), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(U @ Hd @ U.T, np.eye(K), atol=1e-10)
    # a transposed factor fails the identity, and the other upper factor of H_d^-1
    # (R^-1 with R^T R = H_d, so R^-1 R^-T = H_d^-1) fails the trailing-block property
    assert not np.allclose(U.T @ Hd @ U, np.eye(K), atol=1e-6)
    Rinv = np.linalg.inv(np.linalg.cholesky(Hd).T)
    np.testing.assert_allclose(Rinv @ Rinv.T, np.linalg.inv(Hd), atol=1e-10)
    assert not np.allclose(Rinv[T, T], O.upper_factor(Hd[T, T]), atol=1e-6)


def test_damped_diagonal_is_dead_and_damp_diagonal():
    _, _, Hd, _ = _random_problem(12, 1, 77)
    H = Hd.copy()
    H[3, :] = 0.0
    H[:, 3] = 0.0
    full, dead = O.dead_and_damp(H, 0.05)
    d, dead_d = O.damped_diagonal(np.diag(H), 0.05)
    np.testing.assert_array_equal(dead, dead_d)
    np.testing.assert_array_equal(np.diag(full), d)
    # dead entry: 1 plus the damping of a mean that includes that 1
    assert d[3] == pytest.approx(1.0 + 0.05 * (np.trace(H) + 1.0) / 12, rel=1e-14)


def test_objective_identities():
    X, H, Hd, W = _random_problem(10, 5, 7, M=200)
    s, _ = O.symmetric_scale(W, 2)
    # undamped: the increase per step sums to the output error ||X Δ||^2
    codes, W_hat, loss = O.obq_sweep(H, W, s, 2)
    out_err = np.sum((X @ (W_hat - W).T) ** 2, axis=0)
    np.testing.assert_allclose(loss, out_err, rtol=1e-9)
    assert O.layer_error(H, W, W_hat) == pytest.approx(out_err.sum(), rel=1e-10)
    # damped: 1/2 Δ^T H_d Δ = 1/2 sum E^2
    U = O.upper_factor(Hd)
    _, W_d, E = O.row_form_sweep(U, W, s, 2, 4)
    D = W_d - W
    np.testing.assert_allclose(0.5 * np.sum((D @ Hd) * D, axis=1),
                               0.5 * np.sum(E ** 2, axis=1), rtol=1e-9)


# ------------------------------------------------------------------ special cases

def test_identity_hessian_is_rtn():
    rng = np.random.default_rng(3)
    W = rng.standard_normal((6, 20)) * 0.02
    s, _ = O.symmetric_scale(W, 3)
    codes, W_hat, _ = O.obq_sweep(2.0 * np.eye(20), W, s, 3)
    np.testing.assert_array_equal(codes, O.quantize_codes(W, s[:, None], 3))
    c1, _, _ = O.obq_sweep(np.array([[3.7]]), W[:, :1], s, 3)
    np.testing.assert_array_equal(c1, O.quantize_codes(W[:, :1], s[:, None], 3))


def test_scaled_hessian_same_codes_and_permutation_equivariance():
    X, H, Hd, W = _random_problem(12, 8, 11)
    s, _ = O.symmetric_scale(W, 4)
    c0, w0, _ = O.obq_sweep(Hd, W, s, 4)
    c1, w1, _ = O.obq_sweep(37.0 * Hd, W, s, 4)
    np.testing.assert_array_equal(c0, c1)
    np.testing.assert_allclose(w0, w1, atol=1e-12)
    perm = np.random.default_rng(1).permutation(8)
    c2, w2, _ = O.obq_sweep(Hd, W[perm], s[perm], 4)
    np.testing.assert_array_equal(c2, c0[perm])


def test_sequential_never_beats_brute_force():
    for seed in range(5):
        X, H, Hd, W = _random_problem(3, 1, 100 + seed)
        w = W[0] / 0.02 * 1.3
        codes, W_hat, _ = O.obq_sweep(H, w[None, :], np.array([1.0]), 4)
        best, _ = O.brute_force_best(H, w, range(-8, 8))
        assert O.layer_error(H, w[None, :], W_hat) >= best - 1e-12


# ------------------------------------------------------------------ weighted / grouped Gram

def test_weighted_gram_equals_repeated_tokens():
    rng = np.random.default_rng(5)
    X = rng.standard_normal((30, 7))
    reps = rng.integers(0, 4, size=30)
    np.testing.assert_allclose(O.gram(X, reps.astype(float)), O.gram(np.repeat(X, reps, 0)),
                               atol=1e-10)
    np.testing.assert_allclose(O.gram(X, np.ones(30)), O.gram(X), atol=1e-12)


def test_grouped_solve_is_independent_groups():
    rng = np.random.default_rng(8)
    X = rng.standard_normal((120, 10))
    W = rng.standard_normal((8, 10)) * 0.02
    Hs = np.stack([O.gram(X, rng.random(120) * 2) for _ in range(4)])
    out = O.solve_layer(Hs, W, 3, groups=4)
    for g in range(4):
        ref = O.solve_layer(Hs[g], W[2 * g:2 * g + 2], 3, scales=out["scales"][2 * g:2 * g + 2])
        np.testing.assert_array_equal(out["codes"][2 * g:2 * g + 2], ref["codes"])
    same = O.solve_layer(np.stack([O.gram(X)] * 2), W, 3, groups=2)
    plain = O.solve_layer(O.gram(X), W, 3)
    np.testing.assert_array_equal(same["codes"], plain["codes"])


# ------------------------------------------------------------------ GPTAQ

def _gptaq_problem(K, M, seed, noise=0.1):
    rng = np.random.default_rng(seed)
    X_fp = rng.standard_normal((M, K)) @ (np.eye(K) + 0.3 * rng.standard_normal((K, K)) / np.sqrt(K))
    X_q = X_fp + noise * rng.standard_normal((M, K))
    return X_fp, X_q


def test_gptaq_first_step_is_least_squares_on_tokens():
    """Step 0's residual term equals the least-squares fit of the free columns of the
    quantised stream to neuron 0's share of r1 = w (X~ - X), solved on the token
    matrices directly (no H, no C)."""
    K, M = 6, 80
    X_fp, X_q = _gptaq_problem(K, M, 21)
    H = O.gram(X_q)
    C = O.cross_gram(X_q, X_fp)
    w = np.array([[0.31, -0.12, 0.05, 0.2, -0.07, 0.11]])
    s = np.array([1.0])
    _, _, _, tr_aq = O.obq_sweep(H, w, s, 4, C=C, return_trace=True)
    _, _, _, tr_q = O.obq_sweep(H, w, s, 4, return_trace=True)
    extra = tr_aq[0][0, 1:] - tr_q[0][0, 1:]
    dX = X_fp - X_q
    v, *_ = np.linalg.lstsq(X_q[:, 1:], dX[:, 0] * w[0, 0], rcond=None)
    np.testing.assert_allclose(extra, v, rtol=1e-9, atol=1e-12)


def test_gptaq_zero_residual_is_gptq_and_p1_matches_explicit():
    K, M = 14, 90
    X_fp, X_q = _gptaq_problem(K, M, 5)
    H = O.gram(X_q)
    Hd, _ = O.dead_and_damp(H, 0.01)
    W = np.random.default_rng(2).standard_normal((7, K)) * 0.02
    s, _ = O.symmetric_scale(W, 2)
    c_q, w_q, _ = O.obq_sweep(Hd, W, s, 2)
    c0, w0, _ = O.obq_sweep(Hd, W, s, 2, C=O.cross_gram(X_q, X_q))
    np.testing.assert_array_equal(c0, c_q)
    np.testing.assert_allclose(w0, w_q, atol=1e-12)
    C = O.cross_gram(X_q, X_fp)
    c_aq, w_aq, _ = O.obq_sweep(Hd, W, s, 2, C=C)
    U = O.upper_factor(Hd)
    P1 = O.gptaq_p1(C, U)
    assert np.allclose(np.tril(P1), 0.0)
    for q in range(K - 1):
        row = C[q, q + 1:] @ np.linalg.inv(Hd[q + 1:, q + 1:])
        np.testing.assert_allclose(P1[q, q + 1:], row, rtol=1e-8, atol=1e-12)
    for B in (1, 3, 8, K):
        c_row, w_row, _ = O.row_form_sweep(U, W, s, 2, B, P1=P1)
        np.testing.assert_array_equal(c_row, c_aq)
        np.testing.assert_allclose(w_row, w_aq, atol=1e-12)
    # the asymmetric term moves the free weights for a non-trivial residual
    _, _, _, tr_aq = O.obq_sweep(Hd, W, s, 2, C=C, return_trace=True)
    _, _, _, tr_q = O.obq_sweep(Hd, W, s, 2, return_trace=True)
    assert not np.allclose(tr_aq[0], tr_q[0])


def test_gptaq_inclusive_mask_would_differ():
    """An inclusive mask adds a diagonal term; the strict reading is the only one
    equal to the explicit free-set update."""
    K = 8
    X_fp, X_q = _gptaq_problem(K, 40, 9)
    Hd, _ = O.dead_and_damp(O.gram(X_q), 0.01)
    C = O.cross_gram(X_q, X_fp)
    U = O.upper_factor(Hd)
    inclusive = np.triu(C @ U.T) @ U
    assert not np.allclose(inclusive, O.gptaq_p1(C, U))


# ------------------------------------------------------------------ replay protocol

def test_replay_counts_flips_without_cascade():
    X, H, Hd, W = _random_problem(16, 6, 31)
    s, _ = O.symmetric_scale(W, 3)
    U = O.upper_factor(Hd)
    codes, W_hat, _ = O.row_form_sweep(U, W, s, 3, 16)
    rep = O.replay_row_form(U, W, s, 3, codes)
    assert rep["tie_flips"] == 0 and rep["mismatches"] == 0
    np.testing.assert_array_equal(rep["codes"], codes)
    # plant one wrong decision in an oracle run; the run continues consistently
    # from it (as another implementation would), and the replay of that run counts
    # exactly one mismatch
    bad = codes.copy()
    bad[2, 5] = bad[2, 5] + 1 if bad[2, 5] < 7 else bad[2, 5] - 1
    planted = O.replay_row_form(U, W, s, 3, np.where(np.arange(16) == 5, bad, -1))
    other = planted["codes"]
    assert other[2, 5] == bad[2, 5]
    rep = O.replay_row_form(U, W, s, 3, other)
    assert rep["mismatches"] == 1 and rep["tie_flips"] == 0
    np.testing.assert_array_equal(rep["codes"], other)


# ------------------------------------------------------------ input groups and act-order

def _problem(K, N, seed, M=None):
    rng = np.random.default_rng(seed)
    M = M or 4 * K
    X = rng.standard_normal((M, K)) @ rng.standard_normal((K, K)) * 0.5
    W = rng.standard_normal((N, K)) * 0.1
    Hd, _ = O.dead_and_damp(O.gram(X), 0.01)
    return Hd, W


def test_act_order_example():
    # diagonal (1, 3, 3, 2): 3 before 3 by index, then 2, then 1
    H = np.diag([1.0, 3.0, 3.0, 2.0])
    np.testing.assert_array_equal(O.act_order(H), [1, 2, 3, 0])
    # a dead coordinate (zero diagonal) comes last
    np.testing.assert_array_equal(O.act_order(np.diag([0.0, 5.0, 1.0])), [1, 2, 0])


def test_one_group_is_per_channel_gptq():
    # a single group spanning every coordinate, natural order: the per-channel sweep
    Hd, W = _problem(12, 5, 1)
    s, _ = O.symmetric_scale(W, 3)
    c0, W0, l0 = O.obq_sweep(Hd, W, s, 3)
    r = O.obq_sweep_grouped(Hd, W, 3, groupsize=12)
    np.testing.assert_array_equal(r["codes"], c0)
    np.testing.assert_allclose(r["W_hat"], W0, atol=1e-12)
    np.testing.assert_allclose(r["scales"][:, 0], s, rtol=1e-15)
    np.testing.assert_allclose(r["loss"], l0, rtol=1e-12)


@pytest.mark.parametrize("static", [False, True])
def test_diagonal_hessian_is_group_rtn(static):
    # no coupling between coordinates: every coordinate is rounded with its group's
    # scale taken from W as given (nothing is compensated before a group is entered)
    rng = np.random.default_rng(2)
    K, N, G, bits = 16, 6, 4, 2
    Hd = np.diag(rng.uniform(0.5, 2.0, K))
    W = rng.standard_normal((N, K))
    perm = O.act_order(Hd)
    r = O.obq_sweep_grouped(Hd, W, bits, G, static=static, perm=perm)
    expect = np.zeros((N, K))
    for g in range(K // G):
        cols = (np.arange(g * G, (g + 1) * G) if static else perm[g * G:(g + 1) * G])
        amax = np.max(np.abs(W[:, cols]), axis=1)
        s = 2 * amax / (2 ** bits - 1)
        expect[:, cols] = np.clip(np.rint(W[:, cols] / s[:, None]) + 2 ** (bits - 1), 0, 2 ** bits - 1)
    np.testing.assert_array_equal(r["codes"], expect)
    z = 2 ** (bits - 1)
    np.testing.assert_allclose(r["W_hat"], r["scales"][np.arange(N)[:, None], r["g_idx"][None, :]]
                               * (r["codes"] - z), atol=1e-15)


def test_sorted_diagonal_act_order_is_natural_order():
    Hd, W = _problem(10, 4, 3)
    order = np.argsort(-np.diag(Hd), kind="stable")
    Hs = Hd[np.ix_(order, order)]
    Ws = W[:, order]
    assert np.all(np.diff(np.diag(Hs)) <= 0)
    a = O.obq_sweep_grouped(Hs, Ws, 3, 5, perm=O.act_order(Hs))
    b = O.obq_sweep_grouped(Hs, Ws, 3, 5)
    np.testing.assert_array_equal(a["codes"], b["codes"])
    np.testing.assert_allclose(a["W_hat"], b["W_hat"], atol=1e-12)


@pytest.mark.parametrize("static", [False])
def test_act_order_is_permutation_equivariant(static):
    # relabelling the input coordinates does not change what act-order computes with
    # re-estimated groups (static groups are tied to the original column labels)
    Hd, W = _problem(12, 5, 4)
    rng = np.random.default_rng(5)
    Q = rng.permutation(12)
    Hq, Wq = Hd[np.ix_(Q, Q)], W[:, Q]
    G = 4
    a = O.obq_sweep_grouped(Hd, W, 3, G, static=static, perm=O.act_order(Hd))
    b = O.obq_sweep_grouped(Hq, Wq, 3, G, static=static, perm=O.act_order(Hq))
    np.testing.assert_array_equal(b["codes"], a["codes"][:, Q])
    np.testing.assert_allclose(b["W_hat"], a["W_hat"][:, Q], atol=1e-12)
    if not static:   # dynamic groups follow the processing order, itself equivariant
        np.testing.assert_allclose(b["scales"], a["scales"], rtol=1e-12)


@pytest.mark.parametrize("static", [False, True])
def test_grouped_row_form_matches_explicit(static):
    # the Cholesky row form with U of the reordered H_d reproduces the explicit
    # Schur-updated sweep, group scales included
    Hd, W = _problem(16, 6, 6)
    perm = O.act_order(Hd)
    G = 8
    r = O.obq_sweep_grouped(Hd, W, 3, G, static=static, perm=perm)
    U = O.upper_factor(Hd[np.ix_(perm, perm)])
    rep = O.replay_row_form_grouped(U, W, 3, G, r["codes"], static=static, perm=perm)
    assert rep["mismatches"] == 0 and rep["tie_flips"] == 0
    np.testing.assert_allclose(rep["W_hat"], r["W_hat"], atol=1e-9)
    np.testing.assert_allclose(rep["scales"], r["scales"], rtol=1e-9)
    np.testing.assert_array_equal(rep["g_idx"], r["g_idx"])


def test_reestimated_groups_see_compensation():
    # the first group's scale is the same either way; a later group's re-estimated
    # scale is taken from compensated weights and differs from the static one
    Hd, W = _problem(12, 5, 7)
    a = O.obq_sweep_grouped(Hd, W, 2, 4, static=False)
    b = O.obq_sweep_grouped(Hd, W, 2, 4, static=True)
    np.testing.assert_allclose(a["scales"][:, 0], b["scales"][:, 0], rtol=1e-15)
    assert np.max(np.abs(a["scales"][:, 1:] - b["scales"][:, 1:])) > 1e-6


# ------------------------------------------------------------------ compensation-aware error

def _collapsed(U):
    """I - diag(U)^-1 U: what [(H U^T) ⊙ M] U reduces to when U^T U = (H + λI)^-1
    (H U^T = U^-1 - λ U^T, and the strict upper part of U^T is zero), worked by hand."""
    return np.eye(U.shape[0]) - U / np.diag(U)[:, None]


def test_cae_p2_closed_form():
    K, M = 12, 60
    X_fp, X_q = _gptaq_problem(K, M, 31)
    X_q[:, 4] = 0.0                        # a dead input coordinate
    H = O.gram(X_q)
    Hd, dead = O.dead_and_damp(H, 0.05)
    assert dead[4]
    C = O.cross_gram(X_q, X_fp)
    assert np.abs(C[4]).max() > 0          # the dead row still carries cross terms
    U = O.upper_factor(Hd)
    np.testing.assert_allclose(O.cae_p2(H, C, U), O.gptaq_p1(C, U) + _collapsed(U), atol=1e-10)
    np.testing.assert_allclose(O.cae_p2(H, None, U), _collapsed(U), atol=1e-10)
    # the strict mask leaves a zero diagonal: coordinate q's own row term never moves q
    assert np.allclose(np.tril(O.cae_p2(H, C, U)), 0.0)


def test_cae_second_step_is_least_squares_on_tokens():
    """Step 0 owes nothing to r2 (w^(0) and w^(0) agree); at step 1 the term equals
    the least-squares fit of the quantised stream's free columns to coordinate 1's
    share of r2 = (w^(0) - w^(1)) X~, solved on the token matrices (no H, no C)."""
    K, M = 6, 80
    X_fp, X_q = _gptaq_problem(K, M, 23)
    H = O.gram(X_q)
    C = O.cross_gram(X_q, X_fp)
    w = np.array([[0.31, -0.12, 0.05, 0.2, -0.07, 0.11]])
    s = np.array([1.0])
    _, _, _, tr_cae = O.obq_sweep(H, w, s, 4, C=C, cae_H=H, return_trace=True)
    _, _, _, tr_aq = O.obq_sweep(H, w, s, 4, C=C, return_trace=True)
    np.testing.assert_array_equal(tr_cae[0], tr_aq[0])
    drift = w[0, 1] - tr_aq[0][0, 1]
    assert abs(drift) > 1e-3
    extra = tr_cae[1][0, 2:] - tr_aq[1][0, 2:]
    v, *_ = np.linalg.lstsq(X_q[:, 2:], X_fp[:, 1] * drift, rcond=None)
    np.testing.assert_allclose(extra, v, rtol=1e-9, atol=1e-12)


def test_cae_three_weight_hand_trace(golden):
    """The printed three-weight problem with the compensation-aware term, worked by
    hand: step 0 is unchanged, [0, -0.6, 0.2]; at step 1 coordinate 1 has drifted by
    w^(0)_1 - w_1 = 0.2 and P2[1, 2] = H[1, 2] / H[2, 2] = 2/3 adds 2/15 to the 7/15
    of plain GPTQ, giving [0, -1, 0.6]; step 2 rounds 0.6 to 1."""
    g = golden("three_weight_counterexample.txt")
    H = O.gram(g["X"])
    w, s, bits = g["w"], np.array([g["scale"]]), int(g["bits"])
    for mode in ("schur", "direct"):
        _, W_hat, _, tr = O.obq_sweep(H, w[None, :], s, bits, mode=mode, cae_H=H,
                                      return_trace=True)
        np.testing.assert_allclose(tr[0][0], [0.0, -0.6, 0.2], atol=1e-12)
        np.testing.assert_allclose(tr[1][0], [0.0, -1.0, 0.6], atol=1e-12)
        np.testing.assert_allclose(W_hat[0], [0.0, -1.0, 1.0], atol=1e-12)
    P2 = O.cae_p2(H, None, g["U"])
    assert P2[1, 2] == pytest.approx(2.0 / 3.0, abs=1e-12)
    for B in (1, 2, 3):
        _, W_row, _ = O.row_form_sweep(g["U"], w[None, :], s, bits, B, P2=P2)
        np.testing.assert_allclose(W_row[0], [0.0, -1.0, 1.0], atol=1e-12)


@pytest.mark.parametrize("with_c", [False, True])
def test_cae_row_form_matches_explicit(with_c):
    K, M = 14, 90
    X_fp, X_q = _gptaq_problem(K, M, 7)
    H = O.gram(X_q)
    Hd, _ = O.dead_and_damp(H, 0.01)
    C = O.cross_gram(X_q, X_fp) if with_c else None
    W = np.random.default_rng(3).standard_normal((7, K)) * 0.02
    s, _ = O.symmetric_scale(W, 2)
    c_ex, w_ex, _, tr = O.obq_sweep(Hd, W, s, 2, C=C, cae_H=H, return_trace=True)
    c_dir, w_dir, _ = O.obq_sweep(Hd, W, s, 2, C=C, cae_H=H, mode="direct")
    np.testing.assert_array_equal(c_dir, c_ex)
    np.testing.assert_allclose(w_dir, w_ex, atol=1e-12)
    U = O.upper_factor(Hd)
    P1 = O.gptaq_p1(C, U) if with_c else None
    P2 = O.cae_p2(H, C, U)
    for B in (1, 3, 8, K):
        c_row, w_row, _ = O.row_form_sweep(U, W, s, 2, B, P1=P1, P2=P2)
        np.testing.assert_array_equal(c_row, c_ex)
        np.testing.assert_allclose(w_row, w_ex, atol=1e-12)
    rep = O.replay_row_form(U, W, s, 2, c_ex, P1=P1, P2=P2)
    assert rep["mismatches"] == 0 and rep["tie_flips"] == 0
    np.testing.assert_allclose(rep["W_hat"], w_ex, atol=1e-12)
    # the term moves the free weights once compensation has moved a coordinate
    _, _, _, tr_plain = O.obq_sweep(Hd, W, s, 2, C=C, return_trace=True)
    assert not np.allclose(tr[1], tr_plain[1])


def test_cae_collapsed_sweep_matches_row_form():
    """With P2 = P1 + I - diag(U)^-1 U the two row terms merge with the GPTQ step into
    one propagated error E'_j = (w^(0)_j - q_j) / U_jj and a P1 row scaled by w^(0)_j
    (algebra; the form a lazy-block implementation can use without P2). Written out
    here, separately from the oracle, and compared with its row form."""
    K, M = 16, 100
    X_fp, X_q = _gptaq_problem(K, M, 11)
    H = O.gram(X_q)
    Hd, _ = O.dead_and_damp(H, 0.01)
    C = O.cross_gram(X_q, X_fp)
    U = O.upper_factor(Hd)
    P1 = O.gptaq_p1(C, U)
    W0 = np.random.default_rng(5).standard_normal((5, K)) * 0.02
    s, _ = O.symmetric_scale(W0, 3)
    c_ref, w_ref, _ = O.row_form_sweep(U, W0, s, 3, 4, P1=P1, P2=O.cae_p2(H, C, U))
    W = W0.copy()
    z = 4
    for j in range(K):
        c = np.clip(np.rint(W[:, j] / s) + z, 0, 7)
        q = s * (c - z)
        e = (W0[:, j] - q) / U[j, j]
        W[:, j + 1:] += -np.outer(e, U[j, j + 1:]) + np.outer(W0[:, j], P1[j, j + 1:])
        W[:, j] = q
        np.testing.assert_array_equal(c, c_ref[:, j])
    np.testing.assert_allclose(W, w_ref, atol=1e-12)


def test_cae_special_cases_reduce_to_rtn():
    # a diagonal Hessian compensates nothing, so no coordinate drifts and the term is
    # void; a single coordinate has nothing after it
    rng = np.random.default_rng(9)
    K = 10
    H = np.diag(rng.uniform(0.5, 2.0, K))
    W = rng.standard_normal((6, K)) * 0.02
    s, _ = O.symmetric_scale(W, 3)
    c, W_hat, _ = O.obq_sweep(H, W, s, 3, cae_H=H)
    np.testing.assert_array_equal(c, O.quantize_codes(W, s[:, None], 3))
    np.testing.assert_allclose(O.cae_p2(H, None, O.upper_factor(H)), 0.0, atol=1e-15)
    c1, _, _ = O.obq_sweep(np.array([[2.0]]), W[:, :1], s, 3, cae_H=np.array([[2.0]]))
    np.testing.assert_array_equal(c1, O.quantize_codes(W[:, :1], s[:, None], 3))


def test_cae_grouped_row_form_matches_explicit():
    K, M = 16, 90
    X_fp, X_q = _gptaq_problem(K, M, 13)
    H = O.gram(X_q)
    Hd, _ = O.dead_and_damp(H, 0.01)
    C = O.cross_gram(X_q, X_fp)
    W = np.random.default_rng(4).standard_normal((6, K)) * 0.02
    perm = O.act_order(H)
    r = O.obq_sweep_grouped(Hd, W, 3, 8, perm=perm, C=C, cae_H=H)
    ix = np.ix_(perm, perm)
    U = O.upper_factor(Hd[ix])
    rep = O.replay_row_form_grouped(U, W, 3, 8, r["codes"], perm=perm,
                                    P1=O.gptaq_p1(C[ix], U), P2=O.cae_p2(H[ix], C[ix], U))
    assert rep["mismatches"] == 0 and rep["tie_flips"] == 0
    np.testing.assert_allclose(rep["W_hat"], r["W_hat"], atol=1e-9)
    plain = O.obq_sweep_grouped(Hd, W, 3, 8, perm=perm, C=C)
    assert not np.allclose(plain["W_hat"], r["W_hat"]) or not np.array_equal(plain["codes"], r["codes"])


# ------------------------------------------------------------------ packed storage

@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("K", [1, 31, 32, 33, 100])
def test_pack_is_the_little_endian_bit_stream(bits, K):
    # independent statement of the layout: the row's words read as one little-endian
    # integer equal sum_k c_k 2^(b k) (Python integers, no bit loop over words)
    rng = np.random.default_rng(bits * 100 + K)
    c = rng.integers(0, 2 ** bits, size=(5, K))
    words = O.pack_codes(c, bits)
    assert words.dtype == np.uint32 and words.shape == (5, (K * bits + 31) // 32)
    for n in range(5):
        as_int = int.from_bytes(words[n].astype("<u4").tobytes(), "little")
        assert as_int == sum(int(v) << (bits * k) for k, v in enumerate(c[n]))
    np.testing.assert_array_equal(O.unpack_codes(words, bits, K), c)


def test_pack_whole_code_widths_match_byte_views():
    # 8-bit codes: the words' bytes are the codes; 4-bit: byte j = c[2j] | c[2j+1] << 4;
    # 2-bit: byte j = c[4j] | c[4j+1] << 2 | c[4j+2] << 4 | c[4j+3] << 6
    rng = np.random.default_rng(1)
    c8 = rng.integers(0, 256, size=(3, 64))
    np.testing.assert_array_equal(O.pack_codes(c8, 8).view(np.uint8), c8.astype(np.uint8))
    c4 = rng.integers(0, 16, size=(3, 64))
    np.testing.assert_array_equal(O.pack_codes(c4, 4).view(np.uint8),
                                  (c4[:, 0::2] | (c4[:, 1::2] << 4)).astype(np.uint8))
    c2 = rng.integers(0, 4, size=(3, 64))
    np.testing.assert_array_equal(
        O.pack_codes(c2, 2).view(np.uint8),
        (c2[:, 0::4] | (c2[:, 1::4] << 2) | (c2[:, 2::4] << 4) | (c2[:, 3::4] << 6)).astype(np.uint8))


def test_pack_three_bit_straddle_by_hand():
    # 3-bit codes 0..7 repeated: code 10 (value 2 = 0b010) sits at bits 30..32, so
    # word 0 ends with bits 30, 31 = 0, 1 and word 1 starts with bit 0 = 0; code 21
    # (value 5 = 0b101) sits at bits 63..65: word 1's top bit 1, word 2's bits 0, 1 = 0, 1
    c = (np.arange(32) % 8)[None, :]
    w = O.pack_codes(c, 3)
    assert w.shape == (1, 3)
    assert (int(w[0, 0]) >> 30) == 0b10
    assert int(w[0, 1]) & 1 == 0
    assert (int(w[0, 1]) >> 31) == 1
    assert int(w[0, 2]) & 0b11 == 0b10
    # the first ten codes fill word 0's low 30 bits
    assert int(w[0, 0]) & ((1 << 30) - 1) == sum(k % 8 << (3 * k) for k in range(10))


# ------------------------------------------------------------------ first-order term (reading)

def _fo_problem(K, N, seed):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((4 * K, K)) @ (np.eye(K) + 0.3 * rng.standard_normal((K, K)) / np.sqrt(K))
    Hd, _ = O.dead_and_damp(O.gram(X), 0.01)
    W = 0.02 * rng.standard_normal((N, K))
    G = 0.5 * rng.standard_normal((N, K))
    return Hd, W, G


def test_first_order_zero_gradient_is_gptq():
    Hd, W, _ = _fo_problem(12, 6, 1)
    c, w, s = O.first_order_obq_sweep(Hd, W, np.zeros_like(W), 0.7, 3)
    s0, _ = O.symmetric_scale(W, 3)
    c0, w0, _ = O.obq_sweep(Hd, W, s0, 3)
    np.testing.assert_array_equal(c, c0)
    np.testing.assert_allclose(w, w0, atol=1e-12)


def test_first_order_is_gptq_from_the_shifted_start():
    # the quadratic model's sequential minimisers equal GPTQ's row form started at
    # w0 - beta H^-1 g (solved per step vs Cholesky rows and lazy blocks)
    Hd, W, G = _fo_problem(14, 7, 2)
    for beta in (0.3, 1.0):
        c, w, s = O.first_order_obq_sweep(Hd, W, G, beta, 3)
        Ws, _ = O.first_order_shift(Hd, W, G, beta)
        np.testing.assert_allclose(s, O.symmetric_scale(Ws, 3)[0], rtol=1e-12)
        for B in (1, 4, 14):
            c_row, w_row, _ = O.row_form_sweep(O.upper_factor(Hd), Ws, s, 3, B)
            np.testing.assert_array_equal(c_row, c)
            np.testing.assert_allclose(w_row, w, atol=1e-10)


def test_first_order_follow_equals_row_form_replay_from_the_shifted_start():
    # the explicit first-order sweep's tie-follow mode against replay_row_form (its own
    # pins) from the shifted start, with planted disagreements: a near tie whose other
    # code is adopted as a tie flip, and a code two steps away adopted as a mismatch
    Hd, W, G = _fo_problem(16, 9, 5)
    beta = 0.8
    c, w, s = O.first_order_obq_sweep(Hd, W, G, beta, 3)
    Ws, _ = O.first_order_shift(Hd, W, G, beta)
    U = O.upper_factor(Hd)
    # follow its own codes: nothing to count, the same result
    c2, w2, s2, st = O.first_order_obq_sweep(Hd, W, G, beta, 3, follow=c)
    assert st["tie_flips"] == 0 and st["mismatches"] == 0
    np.testing.assert_array_equal(c2, c)
    np.testing.assert_allclose(w2, w, atol=1e-12)
    follow = c.copy()
    follow[2, 5] = c[2, 5] + 2 if c[2, 5] <= 5 else c[2, 5] - 2
    follow[6, 11] = c[6, 11] + 1 if c[6, 11] < 7 else c[6, 11] - 1
    for band in (1e-4, 0.6):     # 0.6: every one-apart difference counts as a tie
        c3, w3, _, st3 = O.first_order_obq_sweep(Hd, W, G, beta, 3, follow=follow, band=band)
        rep = O.replay_row_form(U, Ws, s, 3, follow, band=band)
        np.testing.assert_array_equal(c3, rep["codes"])
        np.testing.assert_allclose(w3, rep["W_hat"], atol=1e-10)
        assert st3["tie_flips"] == rep["tie_flips"] and st3["mismatches"] == rep["mismatches"]
        assert c3[2, 5] == follow[2, 5] and c3[6, 11] == follow[6, 11]
        assert st3["mismatches"] >= 1


def test_first_order_diagonal_hessian_is_rtn_of_the_newton_point():
    rng = np.random.default_rng(3)
    K, N = 9, 5
    h = rng.uniform(0.5, 2.0, K)
    W = 0.02 * rng.standard_normal((N, K))
    G = 0.01 * rng.standard_normal((N, K))
    c, w, s = O.first_order_obq_sweep(np.diag(h), W, G, 0.6, 4)
    target = W - 0.6 * G / h
    np.testing.assert_array_equal(c, O.quantize_codes(target, s[:, None], 4))


def test_first_order_gamma_and_trust_region():
    Hd, W, G = _fo_problem(10, 4, 4)
    _, gamma = O.first_order_shift(Hd, W, G, 1.0)
    assert gamma == pytest.approx(sum(G[n] @ np.linalg.inv(Hd) @ G[n] for n in range(4)), rel=1e-12)
    # the factor meets the bound with equality below 1, is 1 when the bound allows it,
    # and 0 when alpha is 0
    for alpha, lq in ((0.1, 0.05 * gamma), (2.0, 0.4 * gamma), (0.0, gamma)):
        b = O.trust_region_beta(alpha, lq, gamma)
        assert 0.0 <= b <= 1.0
        lhs = (b - b * b / 2) * gamma
        if b < 1.0:
            assert lhs == pytest.approx(alpha * lq, rel=1e-12, abs=1e-300)
        else:
            assert lhs <= alpha * lq + 1e-15
    assert O.trust_region_beta(1.0, 1.0, 0.0) == 1.0


def test_planted_mistakes_still_apply():
    # tests/oracle_mutations.py plants each mistake by replacing a line of the oracle; a
    # change to the oracle's text must keep every planted mistake applicable (the full
    # check, which runs these pins once per mistake, is run by hand)
    import importlib.util
    import os
    here = os.path.dirname(os.path.abspath(__file__))
    spec = importlib.util.spec_from_file_location("oracle_mutations",
                                                  os.path.join(here, "oracle_mutations.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    src = open(os.path.join(os.path.dirname(here), "oracle", "gptq_oracle.py"),
               encoding="utf-8").read()
    assert len(mod.MUTATIONS) >= 50
    for name, old, new in mod.MUTATIONS:
        assert old in src and new != old, name
