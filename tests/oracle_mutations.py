"""Planted-mistake check of the oracle's pins (CPU; run by hand, not collected by pytest).

    python tests/oracle_mutations.py

Each entry plants one plausible mistake in a copy of oracle/gptq_oracle.py (a dropped
factor, a wrong sign, a transposed operand, an inclusive mask, a skipped term, a wrong
rounding or layout rule) and runs tests/test_oracle_pins.py against the copy. Every
mistake must make at least one pin fail; the script prints the pin that caught it and
exits non-zero if a mistake survives or no longer applies to the source.
"""

import os
import shutil
import subprocess
import sys
import tempfile

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

MUTATIONS = [
    ("gram factor 2 dropped", "        return 2.0 * (X.T @ X)\n", "        return 1.0 * (X.T @ X)\n"),
    ("weighted gram ignores s", "    return 2.0 * (X.T @ (X * s[:, None]))", "    return 2.0 * (X.T @ X)"),
    ("cross gram sign", "    dX = np.asarray(X_fp, dtype=np.float64) - Xq", "    dX = Xq - np.asarray(X_fp, dtype=np.float64)"),
    ("cross gram transposed", "    return 2.0 * (dX.T @ Xq)", "    return 2.0 * (Xq.T @ dX)"),
    ("dead diag value", "    d[dead] = 1.0\n    return d + percdamp", "    d[dead] = 0.5\n    return d + percdamp"),
    ("damping mean excludes dead", "    return d + percdamp * np.mean(d), dead", "    return d + percdamp * np.mean(d[~dead]) if (~dead).any() else d, dead"),
    ("damping not scaled by mean", "    return d + percdamp * np.mean(d), dead", "    return d + percdamp, dead"),
    ("PD threshold dropped", "    return bool(np.all(pivots > K * np.finfo(np.float64).eps * np.diag(H)))", "    return bool(np.all(pivots > 0))"),
    ("scale uses 2^b", "    s = 2.0 * amax / (2 ** bits - 1)", "    s = 2.0 * amax / (2 ** bits)"),
    ("scale uses 2^(b-1)-1", "    s = 2.0 * amax / (2 ** bits - 1)", "    s = amax / (2 ** (bits - 1) - 1)"),
    ("zero channel scale 0", "    s[amax == 0.0] = 1.0", "    s[amax == 0.0] = 1e-30"),
    ("rounding half up", "    c = np.rint(np.asarray(w, dtype=np.float64) / s) + z", "    c = np.floor(np.asarray(w, dtype=np.float64) / s + 0.5) + z"),
    ("no clamp", "    return np.clip(c, 0, 2 ** bits - 1)", "    return c"),
    ("clamp one short", "    return np.clip(c, 0, 2 ** bits - 1)", "    return np.clip(c, 1, 2 ** bits - 1)"),
    ("dequant zero point", "    return np.asarray(s, dtype=np.float64) * (np.asarray(c, dtype=np.float64) - 2 ** (bits - 1))", "    return np.asarray(s, dtype=np.float64) * (np.asarray(c, dtype=np.float64) - 2 ** (bits - 1) + 1)"),
    ("obq update sign", "        W[:, q:] -= np.outer(r / p_qq, P[:, 0])", "        W[:, q:] += np.outer(r / p_qq, P[:, 0])"),
    ("obq uses row of P", "        W[:, q:] -= np.outer(r / p_qq, P[:, 0])", "        W[:, q:] -= np.outer(r, P[:, 0])"),
    ("obq loss factor", "        loss += r * r / (2.0 * p_qq)", "        loss += r * r / p_qq"),
    ("schur update sign", "            P_next = P[1:, 1:] - np.outer(P[1:, 0], P[0, 1:]) / p_qq", "            P_next = P[1:, 1:] + np.outer(P[1:, 0], P[0, 1:]) / p_qq"),
    ("schur skipped (sub-block of inverse)", "            P_next = P[1:, 1:] - np.outer(P[1:, 0], P[0, 1:]) / p_qq", "            P_next = P[1:, 1:]"),
    ("gptaq term sign", "                W[:, q + 1:] += np.outer(w_pre, C[q, q + 1:] @ P_next)", "                W[:, q + 1:] -= np.outer(w_pre, C[q, q + 1:] @ P_next)"),
    ("gptaq term uses rounded w", "                W[:, q + 1:] += np.outer(w_pre, C[q, q + 1:] @ P_next)", "                W[:, q + 1:] += np.outer(target, C[q, q + 1:] @ P_next)"),
    ("gptaq term transposed C", "                W[:, q + 1:] += np.outer(w_pre, C[q, q + 1:] @ P_next)", "                W[:, q + 1:] += np.outer(w_pre, C[q + 1:, q] @ P_next)"),
    ("upper factor transposed", "    return np.linalg.cholesky(P).T", "    return np.linalg.cholesky(P)"),
    ("upper factor of H not H^-1", "    P = np.linalg.inv(np.asarray(H_d, dtype=np.float64))\n    P = 0.5 * (P + P.T)\n    return np.linalg.cholesky(P).T", "    P = np.asarray(H_d, dtype=np.float64)\n    return np.linalg.inv(np.linalg.cholesky(P))"),
    ("p1 inclusive mask", "    T = np.triu(T, k=1)\n    return T @ U", "    T = np.triu(T, k=0)\n    return T @ U"),
    ("p1 C^T", "    T = C @ U.T\n    T = np.triu(T, k=1)\n    return T @ U", "    T = C.T @ U.T\n    T = np.triu(T, k=1)\n    return T @ U"),
    ("row form E not normalised", "            e = (w - target) / U[j, j]\n            W[:, j:i1] -= np.outer(e, U[j, j:i1])\n            if P1 is not None:\n                W[:, j + 1:i1] += np.outer(w, P1[j, j + 1:i1])", "            e = (w - target)\n            W[:, j:i1] -= np.outer(e, U[j, j:i1])\n            if P1 is not None:\n                W[:, j + 1:i1] += np.outer(w, P1[j, j + 1:i1])"),
    ("row form far update transposed", "            W[:, i1:] -= E[:, i0:i1] @ U[i0:i1, i1:]", "            W[:, i1:] -= E[:, i0:i1] @ U[i1:, i0:i1].T"),
    ("row form far update skipped", "            W[:, i1:] -= E[:, i0:i1] @ U[i0:i1, i1:]", "            pass"),
    ("row form far P1 skipped", "            if P1 is not None:\n                W[:, i1:] += W_pre @ P1[i0:i1, i1:]", "            if P1 is not None:\n                pass"),
    ("layer error factor", "    return 0.5 * float(np.sum((D @ np.asarray(H, dtype=np.float64)) * D))", "    return float(np.sum((D @ np.asarray(H, dtype=np.float64)) * D))"),
    ("act order ascending", "key=lambda k: (-d[k], k)", "key=lambda k: (d[k], k)"),
    ("act order ties high index first", "key=lambda k: (-d[k], k)", "key=lambda k: (-d[k], -k)"),
    ("static scales on processing order", "            s = S_static[:, order[q] // G]", "            s = S_static[:, q // G]"),
    ("regroup scale from starting weights", "                scales[:, q // G], _ = symmetric_scale(Wp[:, q:q + G], bits)", "                scales[:, q // G], _ = symmetric_scale(W[:, order][:, q:q + G], bits)"),
    ("grouped g_idx not inverted", "    g_idx = (np.arange(K) // G) if static else (inv // G)\n    return dict(codes=codes, W_hat=W_hat, scales=scales, g_idx=g_idx, loss=loss)", "    g_idx = (np.arange(K) // G) if static else (order // G)\n    return dict(codes=codes, W_hat=W_hat, scales=scales, g_idx=g_idx, loss=loss)"),
    ("grouped codes not restored", "    codes[:, order] = codes_p\n    W_hat[:, order] = Wp\n    inv = np.empty(K, dtype=np.int64)\n    inv[order] = np.arange(K)\n    g_idx = (np.arange(K) // G) if static else (inv // G)\n    return dict(codes=codes, W_hat=W_hat, scales=scales", "    codes[:, :] = codes_p\n    W_hat[:, order] = Wp\n    inv = np.empty(K, dtype=np.int64)\n    inv[order] = np.arange(K)\n    g_idx = (np.arange(K) // G) if static else (inv // G)\n    return dict(codes=codes, W_hat=W_hat, scales=scales"),
    ("replay tie band ignored", "            tie = one_apart & (frac_dist < band)", "            tie = one_apart"),
    ("replay does not follow", "            c = np.where(diff, G[:, j], c)\n        target = s * (c - z)\n        e = (w - target) / U[j, j]\n        loss", "            pass\n        target = s * (c - z)\n        e = (w - target) / U[j, j]\n        loss"),
    ("pack bit order reversed", "            words[:, t // 32] |= bit << np.uint64(t % 32)", "            words[:, t // 32] |= bit << np.uint64(31 - t % 32)"),
    ("pack code bits reversed", "            bit = ((c[:, k] >> i) & 1).astype(np.uint64)", "            bit = ((c[:, k] >> (bits - 1 - i)) & 1).astype(np.uint64)"),
    ("first order shift sign", "    return np.asarray(W, dtype=np.float64) - beta * Z, float(np.sum(G * Z))", "    return np.asarray(W, dtype=np.float64) + beta * Z, float(np.sum(G * Z))"),
    ("first order gamma without H^-1", "    return np.asarray(W, dtype=np.float64) - beta * Z, float(np.sum(G * Z))", "    return np.asarray(W, dtype=np.float64) - beta * Z, float(np.sum(G * G))"),
    ("first order sweep drops beta in re-solve", "            rhs = beta * G[:, F].T + H_d[F, fx] @ (w[:, fx] - W0[:, fx]).T", "            rhs = G[:, F].T + H_d[F, fx] @ (w[:, fx] - W0[:, fx]).T"),
    ("first order replay does not follow", "                c = np.where(diff, Fw[:, q], c)\n        w[:, q] = dequantize(c, s, bits)", "                pass\n        w[:, q] = dequantize(c, s, bits)"),
    ("first order replay tie band ignored", "                tie = (np.abs(c[diff] - Fw[diff, q]) == 1) & (frac_dist < band)", "                tie = np.abs(c[diff] - Fw[diff, q]) == 1"),
    ("first order sweep scale from W0", "    w = W0 - beta * np.linalg.solve(H_d, G.T).T\n    s, _ = symmetric_scale(w, bits)\n", "    w = W0 - beta * np.linalg.solve(H_d, G.T).T\n    s, _ = symmetric_scale(W0, bits)\n"),
    ("trust region root sign", "    return 1.0 - np.sqrt(1.0 - 2.0 * x)", "    return 1.0 + np.sqrt(1.0 - 2.0 * x) if x < 0 else 1.0 - np.sqrt(1.0 - x)"),
    ("cae p2 without C", "        A = A + np.asarray(C, dtype=np.float64)\n", "        A = A\n"),
    ("cae p2 inclusive mask", "    return np.triu(A @ U.T, k=1) @ U", "    return np.triu(A @ U.T, k=0) @ U"),
    ("cae explicit uses current w", "                W[:, q + 1:] += np.outer(W0[:, q] - w_pre, Xt[q, q + 1:] @ P_next)", "                W[:, q + 1:] += np.outer(W0[:, q] - target, Xt[q, q + 1:] @ P_next)"),
]


def run_one(workdir, old, new):
    case = os.path.join(workdir, "case")
    if os.path.exists(case):
        shutil.rmtree(case)
    os.makedirs(case)
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(case, "oracle"),
                    ignore=shutil.ignore_patterns("__pycache__"))
    shutil.copytree(HERE, os.path.join(case, "tests"),
                    ignore=shutil.ignore_patterns("__pycache__", ".mut*"))
    path = os.path.join(case, "oracle", "gptq_oracle.py")
    src = open(path, encoding="utf-8").read()
    if old not in src:
        return "not applied"
    with open(path, "w", encoding="utf-8") as f:
        f.write(src.replace(old, new))
    # the copy is its own pytest root, so the repository's pytest.ini and conftest stay out
    # of it and the pins import the mutated oracle; the pin that checks the planted
    # mistakes still apply to the oracle's text is left out, since the copy's text is
    # changed on purpose
    with open(os.path.join(case, "pytest.ini"), "w", encoding="utf-8") as f:
        f.write("[pytest]\n")
    r = subprocess.run([sys.executable, "-m", "pytest", "tests/test_oracle_pins.py", "-x", "-q",
                        "-p", "no:cacheprovider", "--rootdir", case, "--deselect",
                        "tests/test_oracle_pins.py::test_planted_mistakes_still_apply"],
                       cwd=case, capture_output=True, text=True, timeout=600)
    if r.returncode == 0:
        return "survived"
    failed = [ln for ln in r.stdout.splitlines() if ln.startswith("FAILED")]
    return "caught by " + (failed[0].split("::")[1].split(" ")[0] if failed else "an error")


def main():
    bad = 0
    with tempfile.TemporaryDirectory(prefix=".mut", dir=HERE) as workdir:
        for name, old, new in MUTATIONS:
            verdict = run_one(workdir, old, new)
            bad += not verdict.startswith("caught")
            print(f"{name:42s} {verdict}", flush=True)
    print(f"{len(MUTATIONS) - bad} of {len(MUTATIONS)} planted mistakes caught")
    return 1 if bad else 0


if __name__ == "__main__":
    sys.exit(main())
