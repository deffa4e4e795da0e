"""fp64 reference of the GPTQ per-layer solve and its GPTAQ / grouped extensions.

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the library.

Sources (cited by title and section):
  [GPTQ blog]  "GPTQ：量化一个权重之后怎样补偿输出误差" (charlestar.github.io),
               sections "Calibration 让量化看见输入方向", "两个权重怎样互相补偿",
               "一次约束补偿的公式从哪里来", "为什么 Cholesky Factor 不能当作原始逆矩阵",
               "GPTQ 怎样把逐个补偿变成可扩展算法", "Damping 与两个不同的分组参数",
               "局部连续最优为什么不保证最终优于 RTN", "落在格点上与真正存成低位权重是两步".
  [ResComp]    "Rethinking Residual Errors in Compensation-based LLM Quantization"
               (papernotes.org), "关键设计" items 1-3 (column objective, residual split,
               neuron decomposition with P1/P2).
  [GPTAQ]      "GPTAQ: Efficient Finetuning-Free Quantization for Asymmetric
               Calibration" (Paper-Notes), "关键设计" (asymmetric objective, OBC
               closed form, channel parallelism).
  [G2PTQ]      "G²PTQ: Improving LLM Post-Training Quantization with Generalized
               Gradient Compensation" (agihunt.info summary): output-channel groups
               sharing one Hessian per group.

Layout. The blog writes X (M tokens x K inputs), W (K x N), Y = XW. Here weights are
stored as nn.Linear does, W[n][k] (N x K): row n is the blog's column w of output
channel n. Every function takes and returns float64 numpy arrays.
"""

from __future__ import annotations

import itertools

import numpy as np


# --------------------------------------------------------------------------------------
# Statistics: Gram / Hessian
# --------------------------------------------------------------------------------------

def gram(X, s=None):
    """H = 2 X^T diag(s) X.

    [GPTQ blog] "Calibration 让量化看见输入方向": the layer objective ||X(w_hat - w)||^2 has
    Hessian 2X^T X, one K x K matrix shared by every output channel and accumulated
    batch by batch. The factor 2 is fixed by the two-weight example of
    "两个权重怎样互相补偿" (X = [[1, .5], [0, sqrt(3)/2]] gives H = [[2, 1], [1, 2]]).
    [G2PTQ] groups of output channels each carry their own Hessian; with a per-token
    weight s_m the group Hessian is 2 sum_m s_m x_m x_m^T.
    """
    X = np.asarray(X, dtype=np.float64)
    if s is None:
        return 2.0 * (X.T @ X)
    s = np.asarray(s, dtype=np.float64)
    return 2.0 * (X.T @ (X * s[:, None]))


def cross_gram(X_quant, X_fp):
    """C = 2 dX^T X with dX = X_fp - X_quant (tokens x inputs).

    [ResComp] item 2 splits the residual as r1 = w (X~ - X) with X~ the
    full-precision stream and X the quantised stream; item 3 precomputes the
    cross statistic dX X^T (their row convention) from dX = X~ - X. In the K x N
    convention that statistic is dX^T X; it carries the same factor 2 as H so that
    the GPTAQ update below needs no extra constant.
    """
    Xq = np.asarray(X_quant, dtype=np.float64)
    dX = np.asarray(X_fp, dtype=np.float64) - Xq
    return 2.0 * (dX.T @ Xq)


# --------------------------------------------------------------------------------------
# Dead coordinates and damping
# --------------------------------------------------------------------------------------

def dead_and_damp(H, percdamp):
    """Dead-coordinate fix, then damping. Returns (H_d, dead mask).

    [GPTQ blog] "Damping 与两个不同的分组参数": a coordinate whose Hessian diagonal is
    zero is "dead": its diagonal is adjusted and its weights are zeroed. Then the
    diagonal increment percdamp * mean(diag H) (default ratio 0.01) is added.
    Reading: the dead diagonal is set to 1 and the fix comes before the damping, so
    the mean includes those 1s. (With a Gram H the dead row and column are zero, so
    the value chosen does not change the solve.)
    """
    H = np.array(H, dtype=np.float64, copy=True)
    d, dead = damped_diagonal(np.diag(H), percdamp)
    H[np.diag_indices(H.shape[0])] = d
    return H, dead


def damped_diagonal(diag, percdamp):
    """The diagonal of H_d from the diagonal of H alone (dead_and_damp touches nothing
    else): dead entries set to 1, then percdamp times the mean of the result added to
    every entry. Returns (diagonal, dead mask)."""
    d = np.array(diag, dtype=np.float64, copy=True)
    dead = d == 0.0
    d[dead] = 1.0
    return d + percdamp * np.mean(d), dead


def is_positive_definite(H):
    """True when every Cholesky pivot of H is clearly positive.

    [GPTQ blog] "Damping 与两个不同的分组参数": with only the input [1, 1] observed,
    X^T X has rank 1 and cannot be inverted; the damping term makes it PD. The
    blog's self-check ("用标准库核对二维补偿") refuses a non-PD Hessian instead of
    repairing it. Reading: a pivot d_j is "clearly positive" when it exceeds the
    Cholesky backward-error size K * eps * H_jj (eps = 2^-52 here); an exactly
    singular H whose rounded pivot lands at +1e-16 is then refused too.
    """
    H = np.asarray(H, dtype=np.float64)
    K = H.shape[0]
    try:
        L = np.linalg.cholesky(H)
    except np.linalg.LinAlgError:
        return False
    pivots = np.diag(L) ** 2
    return bool(np.all(pivots > K * np.finfo(np.float64).eps * np.diag(H)))


# --------------------------------------------------------------------------------------
# Quantisation grid
# --------------------------------------------------------------------------------------

def symmetric_scale(W, bits):
    """Per-output-channel symmetric scale s_n and the zero point z.

    [G2PTQ] weights use symmetric per-channel quantisation; [GPTQ blog]
    "两个权重怎样互相补偿" fixes, for 4 bits, the grid {-8..7} written as unsigned codes
    0..15 with zero point 8. Reading (the formula is not printed): the min-max
    symmetric scale s = 2 * max_k |W[n, k]| / (2^b - 1), zero point z = 2^(b-1), so
    the representable set is s * {-2^(b-1) .. 2^(b-1) - 1}. An all-zero channel takes
    s = 1 (any positive value reconstructs it exactly).
    """
    W = np.asarray(W, dtype=np.float64)
    amax = np.max(np.abs(W), axis=1)
    s = 2.0 * amax / (2 ** bits - 1)
    s[amax == 0.0] = 1.0
    return s, 2 ** (bits - 1)


def quantize_codes(w, s, bits):
    """Integer codes c = clamp(round_half_even(w / s) + z, 0, 2^b - 1).

    [GPTQ blog] "两个权重怎样互相补偿": nearest grid point with ties to even ("最近偶数舍入");
    codes are unsigned 0..2^b-1 around the zero point z = 2^(b-1).
    """
    z = 2 ** (bits - 1)
    c = np.rint(np.asarray(w, dtype=np.float64) / s) + z
    return np.clip(c, 0, 2 ** bits - 1)


def dequantize(c, s, bits):
    """Reconstruction s (c - z).

    [GPTQ blog] "落在格点上与真正存成低位权重是两步": the quantiser returns the
    reconstructed value s(q - z) in floating point; codes are a separate artefact.
    """
    return np.asarray(s, dtype=np.float64) * (np.asarray(c, dtype=np.float64) - 2 ** (bits - 1))


# --------------------------------------------------------------------------------------
# The sweep in explicit OBQ form (no Cholesky, no lazy batching)
# --------------------------------------------------------------------------------------

def obq_sweep(H_d, W, s, bits, mode="schur", C=None, return_trace=False, steps=None,
              cae_H=None):
    """Quantise coordinates 0..K-1 in order, compensating the free set each step.

    [GPTQ blog] "一次约束补偿的公式从哪里来": with free set F and P_F = (H[F, F])^-1, fixing
    coordinate q at its grid value Q(w_q) with r = w_q - Q(w_q) moves the free
    coordinates by delta_F = -r P_F[:, q] / (P_F)_qq (this includes q itself, which
    lands exactly on Q(w_q)); the objective rises by r^2 / (2 (P_F)_qq).
    "为什么 Cholesky Factor 不能当作原始逆矩阵": after q is fixed the next free-set
    inverse is the Schur update P_F - P_F[:, q] P_F[q, :] / (P_F)_qq, not a
    sub-block of the original inverse.
    "GPTQ 怎样把逐个补偿变成可扩展算法": all output channels use the same order.

    mode "schur" carries P by the Schur update; mode "direct" re-inverts H_d[F, F]
    at every step (small K only).

    C (optional) adds the GPTAQ residual term ([GPTAQ] "非对称校准目标" and
    "基于最优脑压缩的闭式解"; [ResComp] item 2, Δw = ... + r X^T H^-1_{-q} with
    r1 = w^(q)(X~ - X)). By the neuron decomposition of [ResComp] item 3 the part of
    r1 owed to coordinate q is applied at q's step, restricted to the coordinates
    still free after q (F' = F minus q):
        w_F' += w_q^pre * C[q, F'] (H_d[F', F'])^-1,
    with w_q^pre the value of coordinate q at its step, before rounding (reading;
    r1 is written with the current weights w^(q)). The single-step form is pinned by
    an independent least-squares solve on the token matrices; which w multiplies
    the row is a reading no printed value pins.

    cae_H (optional) adds the compensation-aware error term of [ResComp] items 1-3:
    the objective keeps the fixed target w^(0) X~, the residual gains
    r2 = (w^(0) - w^(q)) X~, and by the same neuron decomposition the part owed to
    coordinate q is applied at q's step:
        w_F' += (w_q^(0) - w_q^pre) * (X~X^T)[q, F'] (H_d[F', F'])^-1,
    with X~X^T = XX^T + dX X^T, i.e. cae_H + C in the factor-2 convention (cae_H the
    undamped Gram 2 X^T X, C = 0 when absent). Readings: w^(0) is the weight vector
    the sweep starts from (after dead coordinates are zeroed), and w_q^pre the value
    of coordinate q at its step, before rounding.

    Returns (codes, W_hat, loss) with loss[n] = sum_q r^2 / (2 (P_F)_qq), and the
    per-step weights when return_trace. `steps` stops after the first `steps`
    coordinates (a prefix of the same sweep; used to time a bounded sample).
    """
    H_d = np.asarray(H_d, dtype=np.float64)
    W = np.array(W, dtype=np.float64, copy=True)
    W0 = W.copy()
    N, K = W.shape
    if cae_H is not None:
        Xt = np.asarray(cae_H, dtype=np.float64) + (0.0 if C is None else np.asarray(C, dtype=np.float64))
    s = np.asarray(s, dtype=np.float64)
    codes = np.zeros((N, K))
    loss = np.zeros(N)
    trace = []
    P = np.linalg.inv(H_d) if mode == "schur" else None
    for q in range(K if steps is None else min(steps, K)):
        if mode == "direct":
            P = np.linalg.inv(H_d[q:, q:])
        # P is the inverse over F = {q, ..., K-1}; local index 0 is coordinate q.
        w_pre = W[:, q].copy()
        c = quantize_codes(w_pre, s, bits)
        target = dequantize(c, s, bits)
        r = w_pre - target
        p_qq = P[0, 0]
        W[:, q:] -= np.outer(r / p_qq, P[:, 0])
        W[:, q] = target                      # fixed exactly, not compensated twice
        loss += r * r / (2.0 * p_qq)
        codes[:, q] = c
        if q + 1 < K:
            P_next = P[1:, 1:] - np.outer(P[1:, 0], P[0, 1:]) / p_qq
            if C is not None:
                W[:, q + 1:] += np.outer(w_pre, C[q, q + 1:] @ P_next)
            if cae_H is not None:
                W[:, q + 1:] += np.outer(W0[:, q] - w_pre, Xt[q, q + 1:] @ P_next)
            P = P_next
        if return_trace:
            trace.append(W.copy())
    if return_trace:
        return codes, W, loss, trace
    return codes, W, loss


# --------------------------------------------------------------------------------------
# Cholesky row form (used for comparison with the GPU's factor and for replay)
# --------------------------------------------------------------------------------------

def upper_factor(H_d):
    """U upper triangular with U^T U = H_d^-1.

    [GPTQ blog] "为什么 Cholesky Factor 不能当作原始逆矩阵": GPTQ reads the inverse through
    an upper triangular U with U^T U = H^-1; row q of U carries the free-set
    inverse at q's step, (P_F)_qq = U_qq^2. Built here from the library inverse and
    Cholesky routines.
    """
    P = np.linalg.inv(np.asarray(H_d, dtype=np.float64))
    P = 0.5 * (P + P.T)
    return np.linalg.cholesky(P).T


def gptaq_p1(C, U):
    """P1 = [(C U^T) ⊙ M] U with M the strict upper mask (column index > row index).

    [ResComp] item 3: P1 = [(dX X^T L) ⊙ M_U] L^T with H^-1 = L L^T. In the K x N
    convention L = U^T. Reading: M_U is strict. Row q then equals
    C[q, F'] (H[F', F'])^-1 over the coordinates after q, the explicit GPTAQ term of
    obq_sweep (pinned by comparing the two).
    """
    C = np.asarray(C, dtype=np.float64)
    U = np.asarray(U, dtype=np.float64)
    T = C @ U.T
    T = np.triu(T, k=1)
    return T @ U


def cae_p2(H, C, U):
    """P2 = [((H + C) U^T) ⊙ M] U, M the strict upper mask as in gptaq_p1.

    [ResComp] item 3: P2 = [(X~X^T L) ⊙ M_U] L^T with X~X^T = XX^T + dX X^T reused from
    the quantities already at hand; in the factor-2 convention X~X^T is H + C with H
    the undamped Gram and C the cross statistic (None: no asymmetric stream, X~ = X).
    Row q is (H + C)[q, F'] (H_d[F', F'])^-1 over the coordinates after q, the
    explicit compensation-aware term of obq_sweep.
    """
    A = np.asarray(H, dtype=np.float64)
    if C is not None:
        A = A + np.asarray(C, dtype=np.float64)
    U = np.asarray(U, dtype=np.float64)
    return np.triu(A @ U.T, k=1) @ U


def row_form_sweep(U, W, s, bits, blocksize, P1=None, P2=None):
    """GPTQ sweep with U rows and lazy blocks of `blocksize` coordinates.

    [GPTQ blog] "为什么 Cholesky Factor 不能当作原始逆矩阵" and "GPTQ 怎样把逐个补偿变成可扩展算法":
    inside a block, E_j = (w_j - Q(w_j)) / U_jj and W_k -= U_jk E_j for the block's
    later k at once; at the block end the far coordinates get the bulk update
    W_far -= U[blk, far]^T E_blk. The blocking changes only the order of the work.
    With P1, [ResComp] item 3's extra row term w_j^pre * P1[j, k] is added the same
    way (immediately inside the block, in bulk for the far coordinates); with P2, the
    compensation-aware row term (w_j^(0) - w_j^pre) * P2[j, k] likewise, w^(0) being
    the weights the sweep starts from.

    Returns (codes, W_hat, E) with E[n, j] the normalised errors.
    """
    U = np.asarray(U, dtype=np.float64)
    W = np.array(W, dtype=np.float64, copy=True)
    W0 = W.copy()
    N, K = W.shape
    codes = np.zeros((N, K))
    E = np.zeros((N, K))
    for i0 in range(0, K, blocksize):
        i1 = min(i0 + blocksize, K)
        W_pre = np.zeros((N, i1 - i0))
        for j in range(i0, i1):
            w = W[:, j].copy()
            W_pre[:, j - i0] = w
            c = quantize_codes(w, s, bits)
            target = dequantize(c, s, bits)
            e = (w - target) / U[j, j]
            W[:, j:i1] -= np.outer(e, U[j, j:i1])
            if P1 is not None:
                W[:, j + 1:i1] += np.outer(w, P1[j, j + 1:i1])
            if P2 is not None:
                W[:, j + 1:i1] += np.outer(W0[:, j] - w, P2[j, j + 1:i1])
            W[:, j] = target
            codes[:, j] = c
            E[:, j] = e
        if i1 < K:
            W[:, i1:] -= E[:, i0:i1] @ U[i0:i1, i1:]
            if P1 is not None:
                W[:, i1:] += W_pre @ P1[i0:i1, i1:]
            if P2 is not None:
                W[:, i1:] += (W0[:, i0:i1] - W_pre) @ P2[i0:i1, i1:]
    return codes, W, E


def replay_row_form(U, W, s, bits, codes_gpu, P1=None, band=1e-4, P2=None):
    """Tie-follow replay of the unbatched row-form sweep against another run's codes.

    At each (j, n) the oracle takes its own fp64 decision. Where the other run's
    code differs, the step counts as a tie flip when the codes differ by one and
    |frac(w / s) - 0.5| < band, else as a mismatch; in both cases the oracle then
    continues with the other run's code, so one decision never cascades. A
    negative entry in codes_gpu means "no decision given": the oracle keeps its own.
    P1 and P2 add the row terms of row_form_sweep.

    Returns dict(codes, W_hat, tie_flips, mismatches, worst_tie_distance, loss) with
    loss[n] = 1/2 sum_j E_j^2 along the replayed trajectory.
    """
    U = np.asarray(U, dtype=np.float64)
    W = np.array(W, dtype=np.float64, copy=True)
    W0 = W.copy()
    s = np.asarray(s, dtype=np.float64)
    G = np.asarray(codes_gpu, dtype=np.float64)
    N, K = W.shape
    z = 2 ** (bits - 1)
    codes = np.zeros((N, K))
    tie_flips = 0
    mismatches = 0
    worst = 0.0
    loss = np.zeros(N)
    for j in range(K):
        w = W[:, j].copy()
        c = quantize_codes(w, s, bits)
        diff = (c != G[:, j]) & (G[:, j] >= 0)
        if np.any(diff):
            ratio = w[diff] / s[diff]
            frac_dist = np.abs(np.abs(ratio - np.floor(ratio)) - 0.5)
            one_apart = np.abs(c[diff] - G[diff, j]) == 1
            # clamped codes at the grid edge are never near a tie
            tie = one_apart & (frac_dist < band)
            tie_flips += int(np.count_nonzero(tie))
            mismatches += int(np.count_nonzero(~tie))
            if np.any(tie):
                worst = max(worst, float(np.max(frac_dist[tie])))
            c = np.where(diff, G[:, j], c)
        target = s * (c - z)
        e = (w - target) / U[j, j]
        loss += 0.5 * e * e
        W[:, j:] -= np.outer(e, U[j, j:])
        if P1 is not None and j + 1 < K:
            W[:, j + 1:] += np.outer(w, P1[j, j + 1:])
        if P2 is not None and j + 1 < K:
            W[:, j + 1:] += np.outer(W0[:, j] - w, P2[j, j + 1:])
        W[:, j] = target
        codes[:, j] = c
    return dict(codes=codes, W_hat=W, tie_flips=tie_flips, mismatches=mismatches,
                worst_tie_distance=worst, loss=loss)


# --------------------------------------------------------------------------------------
# Objective and whole-layer driver
# --------------------------------------------------------------------------------------

def layer_error(H, W, W_hat):
    """sum_n 1/2 (w_hat_n - w_n)^T H (w_hat_n - w_n) = ||X (W_hat - W)^T||_F^2 for H = 2X^T X.

    [GPTQ blog] "Calibration 让量化看见输入方向": the layer reconstruction objective; with
    H = 2X^T X one half of the quadratic form is the squared output error.
    """
    D = np.asarray(W_hat, dtype=np.float64) - np.asarray(W, dtype=np.float64)
    return 0.5 * float(np.sum((D @ np.asarray(H, dtype=np.float64)) * D))


def solve_layer(H, W, bits, percdamp=0.01, groups=1, C=None, scales=None, mode="schur",
                cae=False):
    """Whole per-layer solve: dead fix, damping, scale, dead zeroing, sweep.

    H is (K, K) for groups == 1 or (g, K, K); output channels are split into g
    contiguous groups of N / g, group i solved with H[i] ([G2PTQ] GuidedQuant-style
    groups with one shared Hessian per group). The scale comes from W as given,
    before dead coordinates are zeroed (reading). cae adds the compensation-aware
    term of obq_sweep with each group's H as given. Returns dict(codes, W_hat,
    scales, loss, dead).
    """
    W = np.asarray(W, dtype=np.float64)
    N, K = W.shape
    Hs = np.asarray(H, dtype=np.float64).reshape(groups, K, K)
    if scales is None:
        s, _ = symmetric_scale(W, bits)
    else:
        s = np.asarray(scales, dtype=np.float64)
    per = N // groups
    codes = np.zeros((N, K))
    W_hat = np.zeros((N, K))
    loss = np.zeros(N)
    deads = np.zeros((groups, K), dtype=bool)
    for g in range(groups):
        H_d, dead = dead_and_damp(Hs[g], percdamp)
        if not is_positive_definite(H_d):
            raise np.linalg.LinAlgError("damped Hessian is not positive definite")
        rows = slice(g * per, (g + 1) * per)
        Wg = W[rows].copy()
        Wg[:, dead] = 0.0
        c, wh, l = obq_sweep(H_d, Wg, s[rows], bits, mode=mode, C=C,
                             cae_H=Hs[g] if cae else None)
        codes[rows], W_hat[rows], loss[rows] = c, wh, l
        deads[g] = dead
    return dict(codes=codes, W_hat=W_hat, scales=s, loss=loss, dead=deads)


def brute_force_best(H, w, grid):
    """Exhaustive minimiser of 1/2 (v - w)^T H (v - w) over v in grid^K (tiny K only).

    [GPTQ blog] "局部连续最优为什么不保证最终优于 RTN": the sequential result is compared with
    the best of all 16^3 grid vectors. Returns (best value, list of minimisers).
    """
    H = np.asarray(H, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    best = np.inf
    arg = []
    for v in itertools.product(grid, repeat=len(w)):
        d = np.asarray(v, dtype=np.float64) - w
        val = 0.5 * float(d @ H @ d)
        if val < best - 1e-12:
            best, arg = val, [tuple(v)]
        elif abs(val - best) <= 1e-12:
            arg.append(tuple(v))
    return best, arg


# --------------------------------------------------------------------------------------
# Input-dimension groups and act-order
# --------------------------------------------------------------------------------------

def act_order(H):
    """Processing order of the input coordinates: decreasing Hessian diagonal.

    [GPTQ blog] "Damping 与两个不同的分组参数": act-order reorders the input coordinates
    by the Hessian diagonal from large to small; it is an ordering heuristic, and the
    coordinates are restored afterwards. Reading: ties keep the lower index first;
    the diagonal is the one given (the accumulated H, before the dead fix and the
    damping, so dead coordinates come last).
    """
    d = np.diag(np.asarray(H, dtype=np.float64))
    return np.array(sorted(range(len(d)), key=lambda k: (-d[k], k)), dtype=np.int64)


def static_group_scales(W, bits, groupsize):
    """Scales of fixed ("static") groups: for channel n and original group g, the
    symmetric scale of W[n, gG:(g+1)G] as given.

    [GPTQ blog] "Damping 与两个不同的分组参数": the group parameters can be re-estimated
    during compensation or fixed beforehand as static groups. Reading: fixed groups
    are the original columns [gG, (g+1)G) and take the min-max symmetric scale of
    symmetric_scale on them.
    """
    W = np.asarray(W, dtype=np.float64)
    N, K = W.shape
    ng = (K + groupsize - 1) // groupsize
    S = np.zeros((N, ng))
    for g in range(ng):
        S[:, g], _ = symmetric_scale(W[:, g * groupsize:(g + 1) * groupsize], bits)
    return S


def obq_sweep_grouped(H_d, W, bits, groupsize, static=False, perm=None, C=None, cae_H=None):
    """The explicit OBQ sweep of obq_sweep with input-dimension groups and an order.

    [GPTQ blog] "Damping 与两个不同的分组参数": blocksize organises the computation,
    groupsize changes the representation: each output channel has one scale per
    group of input coordinates. Readings:
      - processing order `perm` (identity when None): coordinate perm[q] is fixed at
        step q, with H_d and W taken in that order;
      - re-estimated groups (static=False): the groups are processing positions
        [gG, (g+1)G); when the sweep enters group g, s[n, g] is the symmetric scale of
        channel n's current (already compensated) weights on the group's coordinates;
      - static groups (static=True): s from static_group_scales on W as given, and
        coordinate k uses its original group k // G at whatever step it is fixed;
      - afterwards codes and weights are restored to the original coordinate order,
        with g_idx[k] the group whose scale reconstructs coordinate k.
    C (optional) is the GPTAQ cross statistic and cae_H (optional) the undamped Gram
    of the compensation-aware term (both as in obq_sweep), in the original order.

    Returns dict(codes, W_hat, scales, g_idx, loss), all in the original order.
    """
    H_d = np.asarray(H_d, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    N, K = W.shape
    order = np.arange(K) if perm is None else np.asarray(perm)
    G = groupsize
    ng = (K + G - 1) // G
    Hp = H_d[np.ix_(order, order)]
    Wp = W[:, order].copy()
    Cp = None if C is None else np.asarray(C, dtype=np.float64)[np.ix_(order, order)]
    Xt = None
    if cae_H is not None:
        Xt = np.asarray(cae_H, dtype=np.float64)[np.ix_(order, order)]
        if Cp is not None:
            Xt = Xt + Cp
    W0p = Wp.copy()
    S_static = static_group_scales(W, bits, G) if static else None
    scales = S_static.copy() if static else np.zeros((N, ng))
    codes_p = np.zeros((N, K))
    loss = np.zeros(N)
    P = np.linalg.inv(Hp)
    for q in range(K):
        if static:
            s = S_static[:, order[q] // G]
        else:
            if q % G == 0:
                scales[:, q // G], _ = symmetric_scale(Wp[:, q:q + G], bits)
            s = scales[:, q // G]
        w_pre = Wp[:, q].copy()
        c = quantize_codes(w_pre, s, bits)
        target = dequantize(c, s, bits)
        r = w_pre - target
        p_qq = P[0, 0]
        Wp[:, q:] -= np.outer(r / p_qq, P[:, 0])
        Wp[:, q] = target
        loss += r * r / (2.0 * p_qq)
        codes_p[:, q] = c
        if q + 1 < K:
            P_next = P[1:, 1:] - np.outer(P[1:, 0], P[0, 1:]) / p_qq
            if Cp is not None:
                Wp[:, q + 1:] += np.outer(w_pre, Cp[q, q + 1:] @ P_next)
            if Xt is not None:
                Wp[:, q + 1:] += np.outer(W0p[:, q] - w_pre, Xt[q, q + 1:] @ P_next)
            P = P_next
    codes = np.zeros((N, K))
    W_hat = np.zeros((N, K))
    codes[:, order] = codes_p
    W_hat[:, order] = Wp
    inv = np.empty(K, dtype=np.int64)
    inv[order] = np.arange(K)
    g_idx = (np.arange(K) // G) if static else (inv // G)
    return dict(codes=codes, W_hat=W_hat, scales=scales, g_idx=g_idx, loss=loss)


def replay_row_form_grouped(U, W, bits, groupsize, codes_gpu, static=False, perm=None,
                            static_scales=None, band=1e-4, P1=None, P2=None):
    """Tie-follow replay (as replay_row_form) of the row-form sweep with groups and an
    order, against another run's codes given in the original order.

    U is the factor of H_d in processing order (U^T U = (H_d[perm][:, perm])^-1). The
    scales follow obq_sweep_grouped's rules along the replayed trajectory (static
    scales may be passed in, e.g. the other run's, to replay its decisions exactly).
    P1 and P2, in processing order, add the row terms of row_form_sweep.
    Returns dict(codes, W_hat, scales, g_idx, tie_flips, mismatches) in the original
    order.
    """
    U = np.asarray(U, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    N, K = W.shape
    order = np.arange(K) if perm is None else np.asarray(perm)
    G = groupsize
    ng = (K + G - 1) // G
    Wp = W[:, order].copy()
    W0p = Wp.copy()
    Gc = np.asarray(codes_gpu, dtype=np.float64)[:, order]
    if static:
        S = static_group_scales(W, bits, G) if static_scales is None else np.asarray(static_scales, dtype=np.float64)
    else:
        S = np.zeros((N, ng))
    z = 2 ** (bits - 1)
    codes_p = np.zeros((N, K))
    tie_flips = mismatches = 0
    for j in range(K):
        if static:
            s = S[:, order[j] // G]
        else:
            if j % G == 0:
                S[:, j // G], _ = symmetric_scale(Wp[:, j:j + G], bits)
            s = S[:, j // G]
        w = Wp[:, j].copy()
        c = quantize_codes(w, s, bits)
        diff = c != Gc[:, j]
        if np.any(diff):
            ratio = w[diff] / s[diff]
            frac_dist = np.abs(np.abs(ratio - np.floor(ratio)) - 0.5)
            tie = (np.abs(c[diff] - Gc[diff, j]) == 1) & (frac_dist < band)
            tie_flips += int(np.count_nonzero(tie))
            mismatches += int(np.count_nonzero(~tie))
            c = np.where(diff, Gc[:, j], c)
        target = s * (c - z)
        e = (w - target) / U[j, j]
        Wp[:, j:] -= np.outer(e, U[j, j:])
        if P1 is not None and j + 1 < K:
            Wp[:, j + 1:] += np.outer(w, P1[j, j + 1:])
        if P2 is not None and j + 1 < K:
            Wp[:, j + 1:] += np.outer(W0p[:, j] - w, P2[j, j + 1:])
        Wp[:, j] = target
        codes_p[:, j] = c
    codes = np.zeros((N, K))
    W_hat = np.zeros((N, K))
    codes[:, order] = codes_p
    W_hat[:, order] = Wp
    inv = np.empty(K, dtype=np.int64)
    inv[order] = np.arange(K)
    g_idx = (np.arange(K) // G) if static else (inv // G)
    return dict(codes=codes, W_hat=W_hat, scales=S, g_idx=g_idx, tie_flips=tie_flips,
                mismatches=mismatches)


# --------------------------------------------------------------------------------------
# Storage: codes packed into 32-bit words
# --------------------------------------------------------------------------------------

def pack_codes(codes, bits):
    """Each channel's codes as one little-endian bit stream in 32-bit words.

    [GPTQ blog] "落在格点上与真正存成低位权重是两步": landing on the grid is not yet
    low-bit storage; the integer codes must be packed into wider containers (the
    3-bit codes into an integer buffer), with scale, zero point and layout kept
    beside them. The pages fix no layout. Reading: per output channel n, code k takes
    bits [b k, b k + b) of the channel's stream (least significant bit first), and
    stream bit t is bit t mod 32 of word t // 32; a row has ceil(K b / 32) words and
    the unused high bits of its last word are zero. For b = 2, 4, 8 this puts 32 / b
    whole codes in each word; for b = 3, 32 codes fill 3 words and some straddle two.

    codes: (N, K) integers in [0, 2^b). Returns (N, ceil(K b / 32)) uint32.
    """
    c = np.asarray(codes).astype(np.int64)
    N, K = c.shape
    nw = (K * bits + 31) // 32
    words = np.zeros((N, nw), dtype=np.uint64)
    for k in range(K):
        for i in range(bits):
            t = k * bits + i
            bit = ((c[:, k] >> i) & 1).astype(np.uint64)
            words[:, t // 32] |= bit << np.uint64(t % 32)
    return words.astype(np.uint32)


def unpack_codes(words, bits, K):
    """Inverse of pack_codes: (N, ceil(K b / 32)) uint32 -> (N, K) codes."""
    w = np.asarray(words).astype(np.uint64)
    N = w.shape[0]
    c = np.zeros((N, K), dtype=np.int64)
    for k in range(K):
        for i in range(bits):
            t = k * bits + i
            bit = (w[:, t // 32] >> np.uint64(t % 32)) & np.uint64(1)
            c[:, k] |= bit.astype(np.int64) << i
    return c


# --------------------------------------------------------------------------------------
# First-order (gradient) term with a trust-region step
# --------------------------------------------------------------------------------------

def first_order_obq_sweep(H_d, W, G, beta, bits, follow=None, band=1e-4):
    """Sequential OBQ on the quadratic model with a first-order term, explicit form.

    [G2PTQ] summary: the compensation keeps GPTQ's second-order update and adds the
    first-order term from an exact gradient G of the block objective, scaled by a
    trust-region factor beta in [0, 1]. The pages give no formula. Reading: per output
    channel the objective around the given weights w0 is the quadratic model
        L(w) = beta g^T (w - w0) + 1/2 (w - w0)^T H_d (w - w0),
    and OBQ keeps every free coordinate at the model's minimiser given the fixed ones:
    before step 0 all coordinates are free, so they start at w0 - beta H_d^-1 g; at
    step q coordinate q is rounded on the grid of the weights being quantised (scale
    from that starting point, as GPTQ takes it from the weights it is given) and fixed,
    and the coordinates after q move to
        x = w0_F - (H_d[F, F])^-1 (beta g_F + H_d[F, fixed] (w_fixed - w0_fixed)),
    solved directly at every step (no Cholesky form, no lazy batching). With g = 0 this
    is obq_sweep. PARITY UNPINNED against the pages: no formula or value is printed;
    the pins are internal (reduction to GPTQ, the shifted-start identity, closed forms).

    follow (optional): another run's codes, followed as replay_row_form does. Where
    they differ from this sweep's decision the step counts as a tie flip when the
    codes differ by one and |frac(w / s) - 0.5| < band, else as a mismatch, and the
    sweep continues with the other run's code, so one decision never cascades.

    Returns (codes, W_hat, scales), and with `follow` a fourth item
    dict(tie_flips, mismatches, worst_tie_distance).
    """
    H_d = np.asarray(H_d, dtype=np.float64)
    W0 = np.asarray(W, dtype=np.float64)
    G = np.asarray(G, dtype=np.float64)
    N, K = W0.shape
    w = W0 - beta * np.linalg.solve(H_d, G.T).T
    s, _ = symmetric_scale(w, bits)
    codes = np.zeros((N, K))
    stats = dict(tie_flips=0, mismatches=0, worst_tie_distance=0.0)
    Fw = None if follow is None else np.asarray(follow, dtype=np.float64)
    for q in range(K):
        c = quantize_codes(w[:, q], s, bits)
        if Fw is not None:
            diff = c != Fw[:, q]
            if np.any(diff):
                ratio = w[diff, q] / s[diff]
                frac_dist = np.abs(np.abs(ratio - np.floor(ratio)) - 0.5)
                tie = (np.abs(c[diff] - Fw[diff, q]) == 1) & (frac_dist < band)
                stats["tie_flips"] += int(np.count_nonzero(tie))
                stats["mismatches"] += int(np.count_nonzero(~tie))
                if np.any(tie):
                    stats["worst_tie_distance"] = max(stats["worst_tie_distance"],
                                                      float(np.max(frac_dist[tie])))
                c = np.where(diff, Fw[:, q], c)
        w[:, q] = dequantize(c, s, bits)
        codes[:, q] = c
        if q + 1 < K:
            F = slice(q + 1, K)
            fx = slice(0, q + 1)
            rhs = beta * G[:, F].T + H_d[F, fx] @ (w[:, fx] - W0[:, fx]).T
            w[:, F] = W0[:, F] - np.linalg.solve(H_d[F, F], rhs).T
    if Fw is not None:
        return codes, w, s, stats
    return codes, w, s


def first_order_shift(H_d, W, G, beta):
    """w0 - beta H_d^-1 g per channel (the starting point of first_order_obq_sweep), and
    gamma = sum_n g_n H_d^-1 g_n^T, the curvature-weighted size of the gradient: the
    model's loss change along the step is -(beta - beta^2 / 2) gamma."""
    H_d = np.asarray(H_d, dtype=np.float64)
    G = np.asarray(G, dtype=np.float64)
    Z = np.linalg.solve(H_d, G.T).T
    return np.asarray(W, dtype=np.float64) - beta * Z, float(np.sum(G * Z))


def trust_region_beta(alpha, loss_gptq, gamma):
    """Largest beta in [0, 1] whose first-order loss change stays within alpha times the
    GPTQ term's loss: (beta - beta^2 / 2) gamma <= alpha * loss_gptq.

    [G2PTQ] summary: beta scales the first-order step so that the loss change it causes
    does not exceed alpha times that of the GPTQ term (alpha searched per block on
    [0, 3]). Reading: both changes are the quadratic model's, the first-order one along
    the step -beta H^-1 g, the GPTQ one the sweep's loss (1/2 sum E^2)."""
    if gamma <= 0.0:
        return 1.0
    x = alpha * loss_gptq / gamma
    if x >= 0.5:
        return 1.0
    return 1.0 - np.sqrt(1.0 - 2.0 * x)
