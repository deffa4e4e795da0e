"""GPU path vs the fp64 oracle on the same seeded inputs (calls go through the C ABI).

Sizes span several tiles and ragged tails; the pages' worked examples run through
the GPU path too. Full-size cases live in test_gpu_fullsize.py.
"""

import numpy as np
import pytest
import torch

import oracle as O
import post_weight_quantization_solve_b200 as gq
from post_weight_quantization_solve_b200 import synth
from post_weight_quantization_solve_b200.build import build

from gpu_util import (CODE_SAME, TOL_H, TOL_P1, TOL_RECON, TOL_U, check_codes_by_replay, dev,
                      gpu_hessian, own_decisions_same, rel_max, solve_on_gpu)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    gq.load_library()


def _np(t):
    return t.double().cpu().numpy()


def _full_check(wl, chunks, W, groups=1, weights=None, gptaq_fp=None, label=""):
    """Gram -> prepare -> (residual) -> quantize on the GPU; every stage vs the oracle."""
    K, N = wl.K, wl.N
    d = dev()
    H = gpu_hessian(chunks, K, g=groups, weights=weights)
    H_gpu = _np(H).reshape(groups, K, K)
    X = np.concatenate([_np(c) for c in chunks])
    for g in range(groups):
        s = None if weights is None else np.concatenate([_np(w[g]) for w in weights])
        assert rel_max(H_gpu[g], O.gram(X, s)) <= TOL_H, f"{label} H group {g}"
    C_gpu = None
    C_dev = None
    if gptaq_fp is not None:
        C_dev = torch.zeros(K, K, device=d)
        for xf, xq in zip(gptaq_fp, chunks):
            gq.gptaq_accumulate_cross(C_dev, xf.to(d).contiguous(), xq.to(d).contiguous())
        C_gpu = _np(C_dev)
        Xf = np.concatenate([_np(c) for c in gptaq_fp])
        C_ora = O.cross_gram(X, Xf)
        assert rel_max(C_gpu, C_ora) <= TOL_H, f"{label} C"
    out = solve_on_gpu(H, W, wl.bits, wl.blocksize, wl.percdamp, groups=groups, P1_from_C=C_dev)
    W64 = _np(W)
    s_ora, _ = O.symmetric_scale(W64, wl.bits)
    np.testing.assert_allclose(out["scales"], s_ora, rtol=2e-7)
    per = N // groups
    for g in range(groups):
        rows = slice(g * per, (g + 1) * per)
        Hd, dead = O.dead_and_damp(H_gpu[g], wl.percdamp)
        np.testing.assert_array_equal(out["dead"][g], dead)
        U_ora = O.upper_factor(Hd)
        assert rel_max(out["U"].reshape(groups, K, K)[g], U_ora) <= TOL_U, f"{label} U group {g}"
        P1 = None
        if C_gpu is not None:
            P1 = O.gptaq_p1(C_gpu, U_ora)
            assert rel_max(out["P1"], P1) <= TOL_P1, f"{label} P1"
        Wg = W64[rows].copy()
        Wg[:, dead] = 0.0
        rep, _ = check_codes_by_replay(U_ora, Wg, out["scales"][rows], wl.bits,
                                       out["codes"][rows], P1=P1)
        same = own_decisions_same(rep, Wg.size)
        assert rep["mismatches"] == 0, f"{label}: {rep['mismatches']} codes differ outside ties"
        assert same >= CODE_SAME, f"{label}: identical codes {same}"
        # all outputs on the grid: W_hat = s (c - z) exactly (fp32 write-back)
        z = 2 ** (wl.bits - 1)
        expect = (out["scales"][rows, None].astype(np.float32) *
                  (out["codes"][rows] - z).astype(np.float32))
        np.testing.assert_array_equal(out["W_hat"][rows].astype(np.float32)
                                      if W.dtype == torch.float32 else out["W_hat"][rows],
                                      expect if W.dtype == torch.float32 else
                                      torch.tensor(expect).bfloat16().double().numpy())
        assert out["codes"][rows].min() >= 0 and out["codes"][rows].max() <= 2 ** wl.bits - 1
        # independent runs: output error of the GPU result vs the oracle's own solve
        Hx = O.gram(X, None if weights is None else
                    np.concatenate([_np(w[g]) for w in weights]))
        Hd_x, dead_x = O.dead_and_damp(Hx, wl.percdamp)
        W_ora_in = W64[rows].copy()
        W_ora_in[:, dead_x] = 0.0
        _, W_ora, _ = O.row_form_sweep(O.upper_factor(Hd_x), W_ora_in, s_ora[rows], wl.bits,
                                       wl.blocksize,
                                       P1=None if C_gpu is None else
                                       O.gptaq_p1(O.cross_gram(X, np.concatenate(
                                           [_np(c) for c in gptaq_fp])), O.upper_factor(Hd_x)))
        W_gpu_hat = O.dequantize(out["codes"][rows], out["scales"][rows, None], wl.bits)
        e_gpu = O.layer_error(Hx, W64[rows], W_gpu_hat)
        e_ora = O.layer_error(Hx, W64[rows], W_ora)
        assert abs(e_gpu - e_ora) <= TOL_RECON * e_ora, f"{label}: {e_gpu} vs {e_ora}"
        # loss = 1/2 sum E^2 along the trajectory; for plain GPTQ it also equals the
        # damped objective 1/2 D^T H_d D of the result
        np.testing.assert_allclose(out["loss"][rows], rep["loss"], rtol=1e-3, atol=1e-12)
        if C_gpu is None:
            D = W_gpu_hat - Wg
            np.testing.assert_allclose(out["loss"][rows], 0.5 * np.sum((D @ Hd) * D, axis=1),
                                       rtol=2e-3, atol=1e-12)
    return out


def test_tiny_workload_fp32():
    wl = synth.WORKLOADS["tiny"]
    _full_check(wl, [synth.tokens_chunk(wl, 0)], synth.weights(wl), label="tiny")


@pytest.mark.parametrize("K,N,M,B,bits", [(384, 300, 3001, 128, 3), (200, 130, 1500, 32, 4),
                                          (136, 70, 777, 16, 2), (256, 129, 2048, 64, 8)])
def test_ragged_bf16(K, N, M, B, bits):
    wl = synth.WORKLOADS["mlp_up"].scaled(K=K, N=N, M=M, blocksize=B, bits=bits, chunk=1024)
    chunks = [synth.tokens_chunk(wl, c) for c in range(synth.num_chunks(wl))]
    _full_check(wl, chunks, synth.weights(wl), label=f"ragged {K}x{N}")


@pytest.mark.parametrize("form", ["0", "1", "2", "3"])
def test_every_sweep_form(form, monkeypatch):
    # one thread, four lanes or two lanes per channel, or the tensor-core sweep (one
    # launch per super-block, near updates in TMEM): each form on its own, on ragged
    # blocks, plain and GPTAQ
    monkeypatch.setenv("GPTQ_SWEEP_FORM", form)
    wl = synth.WORKLOADS["mlp_up"].scaled(K=392, N=200, M=2000, blocksize=128, bits=3,
                                         chunk=1024)
    chunks = [synth.tokens_chunk(wl, c) for c in range(synth.num_chunks(wl))]
    _full_check(wl, chunks, synth.weights(wl), label=f"form {form}")
    wl = synth.WORKLOADS["gptaq"].scaled(K=256, N=136, M=2048, chunk=1024)
    n = synth.num_chunks(wl)
    xq = [synth.tokens_chunk(wl, c) for c in range(n)]
    xf = [synth.fp_tokens_chunk(wl, c) for c in range(n)]
    _full_check(wl, xq, synth.weights(wl), gptaq_fp=xf, label=f"gptaq form {form}")


def test_rotated_qproj_small():
    wl = synth.WORKLOADS["q_proj"].scaled(K=256, N=256, M=4096)
    _full_check(wl, [synth.tokens_chunk(wl, 0)], synth.weights(wl), label="q_proj")


def test_gptaq_small():
    wl = synth.WORKLOADS["gptaq"].scaled(K=256, N=192, M=4096, chunk=2048)
    n = synth.num_chunks(wl)
    xq = [synth.tokens_chunk(wl, c) for c in range(n)]
    xf = [synth.fp_tokens_chunk(wl, c) for c in range(n)]
    _full_check(wl, xq, synth.weights(wl), gptaq_fp=xf, label="gptaq")


def test_grouped_small():
    wl = synth.WORKLOADS["grouped70b"].scaled(K=320, N=256, M=3000, chunk=1500)
    n = synth.num_chunks(wl)
    chunks = [synth.tokens_chunk(wl, c) for c in range(n)]
    wts = [synth.token_weights_chunk(wl, c) for c in range(n)]
    _full_check(wl, chunks, synth.weights(wl), groups=4, weights=wts, label="grouped")


@pytest.mark.parametrize("K,M", [(64, 1000), (200, 333), (384, 4097)])
def test_weighted_and_cross_gram_ragged(K, M):
    """The tensor-core transform Gram on ragged shapes (partial tiles, token counts
    that are not a multiple of the 32-token step)."""
    d = dev()
    g = 3
    gen = torch.Generator(device="cpu").manual_seed(K + M)
    Xf = torch.randn(M, K, generator=gen).bfloat16()
    Xq = (Xf.float() + 0.05 * torch.randn(M, K, generator=gen)).bfloat16()
    w = torch.rand(g, M, generator=gen) * 2
    H = torch.zeros(g, K, K, device=d)
    gq.gptq_accumulate_hessian(H, Xq.to(d), w.to(d))
    C = torch.zeros(K, K, device=d)
    gq.gptaq_accumulate_cross(C, Xf.to(d), Xq.to(d))
    torch.cuda.synchronize()
    Xq64, Xf64 = _np(Xq), _np(Xf)
    for gi in range(g):
        assert rel_max(_np(H[gi]), O.gram(Xq64, _np(w[gi]))) <= TOL_H
    assert rel_max(_np(C), O.cross_gram(Xq64, Xf64)) <= TOL_H


def test_dead_coordinates():
    wl = synth.WORKLOADS["mlp_up"].scaled(K=144, N=96, M=1000, blocksize=32, bits=3)
    X = synth.tokens_chunk(wl, 0).clone()
    X[:, [0, 7, 64, 143]] = 0
    out = _full_check(wl, [X], synth.weights(wl), label="dead")
    assert out["dead"][0][[0, 7, 64, 143]].all() and out["dead"][0].sum() == 4
    assert np.all(out["W_hat"][:, [0, 7, 64, 143]] == 0)


def _example_on_gpu(H, w, bits=4):
    d = dev()
    Ht = torch.tensor(H, dtype=torch.float32, device=d)
    W = torch.tensor(np.asarray(w)[None, :], dtype=torch.float32, device=d)
    out = solve_on_gpu(Ht, W, bits, 16, 0.0, scales_in=torch.ones(1, device=d))
    return out


def test_pages_two_weight_example_on_gpu(golden):
    g = golden("two_weight_example.txt")
    out = _example_on_gpu(g["H"], g["w"])
    np.testing.assert_array_equal(out["codes"][0], g["final_codes"])
    np.testing.assert_array_equal(out["W_hat"][0], g["final"])
    assert out["U"][1, 1] ** 2 == pytest.approx(g["U11_squared"], rel=1e-6)
    assert out["loss"][0] == pytest.approx(g["sse_final"], rel=1e-6)


def test_pages_three_weight_example_on_gpu(golden):
    g = golden("three_weight_counterexample.txt")
    out = _example_on_gpu(g["H"], g["w"])
    np.testing.assert_array_equal(out["W_hat"][0], g["final"])
    np.testing.assert_allclose(out["U"], g["U"], atol=1e-6)


def test_status_errors_on_gpu(golden):
    d = dev()
    g = golden("rank_one_damping.txt")
    H1 = torch.tensor(O.gram(np.atleast_2d(g["X"])), dtype=torch.float32, device=d)
    st = gq.gptq_prepare(H1.clone(), g["percdamp_singular"])
    assert int(st.item()) == gq.GPTQ_ERR_NOT_PD
    st = gq.gptq_prepare(H1.clone(), g["percdamp_default"])
    assert int(st.item()) == gq.GPTQ_OK
    Hn = torch.eye(32, device=d) * 2
    Hn[3, 5] = float("nan")
    assert int(gq.gptq_prepare(Hn, 0.01).item()) == gq.GPTQ_ERR_NONFINITE
    # a failed prepare makes the following quantize skip (status propagates)
    W = torch.randn(8, 32, device=d)
    Hb = torch.eye(32, device=d) * 2
    Hb[4, 4] = -1.0
    st = gq.gptq_prepare(Hb, 0.0)
    codes, st = gq.gptq_quantize_layer(W, Hb, 4, 16, status=st)
    assert int(st.item()) == gq.GPTQ_ERR_NOT_PD
    Wn = torch.randn(8, 32, device=d)
    Wn[2, 2] = float("inf")
    Hok = torch.eye(32, device=d) * 2
    st = gq.gptq_prepare(Hok, 0.01)
    codes, st = gq.gptq_quantize_layer(Wn, Hok, 4, 16, status=st)
    assert int(st.item()) == gq.GPTQ_ERR_NONFINITE
    with pytest.raises(gq.GPTQError):
        gq.raise_on_status(st)


def test_identity_hessian_is_rtn_on_gpu():
    d = dev()
    K, N = 160, 64
    H = torch.eye(K, device=d) * 2.0
    W = torch.randn(N, K, device=d, generator=torch.Generator(device=d).manual_seed(3)) * 0.02
    out = solve_on_gpu(H, W, 3, 32, 0.0)
    # with H = 2I there is no compensation: the replay (U = I / sqrt 2) is RTN, and
    # the only allowed differences are exact ties such as -amax / s = -3.5
    rep, _ = check_codes_by_replay(np.eye(K) / np.sqrt(2.0), _np(W), out["scales"], 3,
                                   out["codes"])
    assert rep["mismatches"] == 0
    assert own_decisions_same(rep, N * K) >= CODE_SAME
    s, _ = O.symmetric_scale(_np(W), 3)
    np.testing.assert_array_equal(rep["codes"], out["codes"])
    assert np.abs(O.quantize_codes(_np(W), s[:, None], 3) - out["codes"]).max() <= 1


def test_empty_chunk_is_noop():
    d = dev()
    H = torch.ones(16, 16, device=d)
    gq.gptq_accumulate_hessian(H, torch.zeros(0, 16, dtype=torch.bfloat16, device=d))
    assert torch.all(H == 1)


@pytest.mark.parametrize("K,M", [(256, 1000), (392, 3000), (1024, 70000)])
def test_gram_cta_pair_matches_single_cta(K, M, monkeypatch):
    # the CTA-pair Gram (256 x 256 tiles over two SMs) and the single-CTA Gram agree
    # with each other and with the fp64 Gram, ragged tiles and token parts included
    d = dev()
    g = torch.Generator(device=d).manual_seed(K + M)
    X = torch.randn(M, K, device=d, generator=g).to(torch.bfloat16)
    out = {}
    for pair in ("1", "0"):
        monkeypatch.setenv("GPTQ_GRAM_PAIR", pair)
        H = torch.zeros(K, K, device=d)
        st = gq.new_status(d)
        gq.gptq_accumulate_hessian(H, X, status=st)
        gq.raise_on_status(st, "gram")
        out[pair] = _np(H)
    ref = O.gram(_np(X))
    for H in out.values():
        assert rel_max(H, ref) <= TOL_H
        assert np.abs(H - H.T).max() <= 1e-6 * np.abs(ref).max()
    assert rel_max(out["1"], out["0"]) <= 1e-6


@pytest.mark.parametrize("form", ["blk", "pairs", "single"])
@pytest.mark.parametrize("K,g", [(128, 1), (200, 1), (392, 2), (1000, 1)])
def test_every_diagonal_factor_form(form, K, g, monkeypatch):
    # the blocked diagonal factor (16-pivot sub-blocks) and the per-pivot kernels (two
    # pivots or one per block barrier): U against the oracle's factor of the same damped
    # H, with a short first block (K not a multiple of 128), two Hessians and a dead
    # coordinate
    monkeypatch.setenv("GPTQ_DIAG", form)
    d = dev()
    gen = torch.Generator(device=d).manual_seed(K + 7 * g)
    Hs = []
    for _ in range(g):
        X = torch.randn(3 * K, K, device=d, generator=gen) @ (
            torch.eye(K, device=d) + 0.3 * torch.randn(K, K, device=d, generator=gen) / K ** 0.5)
        X[:, K // 3] = 0.0                       # a dead coordinate
        Hs.append(2.0 * X.T @ X)
    H = torch.stack(Hs) if g > 1 else Hs[0]
    H_in = H.double().cpu().numpy().reshape(g, K, K)
    U = H.clone()
    st = gq.gptq_prepare(U, 0.01)
    gq.raise_on_status(st, f"prepare {form}")
    torch.cuda.synchronize()
    U_gpu = U.double().cpu().numpy().reshape(g, K, K)
    for gi in range(g):
        Hd, dead = O.dead_and_damp(H_in[gi], 0.01)
        assert dead[K // 3]
        assert rel_max(U_gpu[gi], O.upper_factor(Hd)) <= TOL_U, (form, gi)
        assert np.all(np.tril(U_gpu[gi], -1) == 0.0)
