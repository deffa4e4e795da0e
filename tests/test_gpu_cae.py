"""Compensation-aware error term on the GPU vs the fp64 oracle (C ABI calls).

The library applies the term in its merged form (the propagated error is measured
from the starting weights, and P1 is scaled by them); the oracle states it as the
pages do, with P2 = [((H + C) U^T) ⊙ M] U formed explicitly and the row
(w^(0)_j - w_j) P2[j, k] added at each step. The parity protocol is the plain
sweep's: the oracle factors the GPU's damped Hessian, replays with tie-following
against the GPU's codes, and every output sits exactly on its grid.
"""

import numpy as np
import pytest
import torch

import oracle as O
import post_weight_quantization_solve_b200 as gq
from post_weight_quantization_solve_b200.build import build

from gpu_util import CODE_SAME, TIE_BAND, TOL_P1, TOL_RECON, TOL_U, dev, rel_max, solve_on_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    gq.load_library()


def _np(t):
    return t.double().cpu().numpy()


def _streams(K, M, seed, dead_cols=()):
    """Seeded full-precision and quantised token streams (bf16) and their statistics."""
    d = dev()
    g = torch.Generator(device=d).manual_seed(seed)
    A = torch.randn(K, K, device=d, generator=g) / K ** 0.5
    Xf = torch.randn(M, K, device=d, generator=g) @ A
    Xq = (Xf + 0.05 * Xf.pow(2).mean().sqrt() * torch.randn(M, K, device=d, generator=g))
    Xf, Xq = Xf.to(torch.bfloat16), Xq.to(torch.bfloat16)
    for c in dead_cols:
        Xq[:, c] = 0
    H = torch.zeros(K, K, device=d)
    gq.gptq_accumulate_hessian(H, Xq.contiguous())
    C = torch.zeros(K, K, device=d)
    gq.gptaq_accumulate_cross(C, Xf.contiguous(), Xq.contiguous())
    return H, C, Xf, Xq, g


def _check(K, N, bits, B, seed, gptaq, wdtype=torch.bfloat16, dead_cols=(), sample=None):
    d = dev()
    H, C, Xf, Xq, g = _streams(K, 4 * K, seed, dead_cols)
    W = (0.02 * torch.randn(N, K, device=d, generator=g)).to(wdtype)
    U = H.clone()
    dead = torch.empty(1, K, dtype=torch.uint8, device=d)
    st = gq.gptq_prepare(U, 0.01, dead_out=dead)
    P1 = None
    if gptaq:
        P1 = torch.empty(K, K, device=d)
        gq.gptaq_residual(P1, C, U)
    Wq = W.clone()
    scales = torch.empty(N, device=d)
    loss = torch.empty(N, device=d)
    codes, st = gq.gptq_quantize_layer(Wq, U, bits, B, P1=P1, dead=dead, scales_out=scales,
                                       loss=loss, write_back=True, status=st, cae=True)
    gq.raise_on_status(st, "cae solve")
    plain, st2 = gq.gptq_quantize_layer(W.clone(), U, bits, B, P1=P1, dead=dead)
    gq.raise_on_status(st2, "plain solve")
    torch.cuda.synchronize()

    H64 = _np(H)
    Hd, dead_o = O.dead_and_damp(H64, 0.01)
    np.testing.assert_array_equal(dead.cpu().numpy()[0].astype(bool), dead_o)
    U_ora = O.upper_factor(Hd)
    assert rel_max(_np(U), U_ora) <= TOL_U
    C64 = _np(C) if gptaq else None
    P1_ora = O.gptaq_p1(C64, U_ora) if gptaq else None
    if gptaq:
        assert rel_max(_np(P1), P1_ora) <= TOL_P1
    P2_ora = O.cae_p2(H64, C64, U_ora)
    W64 = _np(W)
    Wz = W64.copy()
    Wz[:, dead_o] = 0.0
    c_gpu = codes.cpu().numpy().astype(np.float64)
    s_gpu = _np(scales)
    rows = np.arange(N) if sample is None else np.sort(
        np.random.default_rng(seed).choice(N, sample, replace=False))
    rep = O.replay_row_form(U_ora, Wz[rows], s_gpu[rows], bits, c_gpu[rows], P1=P1_ora,
                            P2=P2_ora, band=TIE_BAND)
    assert rep["mismatches"] == 0, rep["mismatches"]
    assert 1.0 - rep["tie_flips"] / c_gpu[rows].size >= CODE_SAME
    np.testing.assert_allclose(_np(loss)[rows], rep["loss"], rtol=1e-3, atol=1e-12)
    # on the grid, in the weights' dtype
    z = 2 ** (bits - 1)
    expect = torch.tensor(s_gpu[:, None].astype(np.float32) *
                          (codes.cpu().numpy().astype(np.float32) - z)).to(W.dtype)
    assert torch.equal(Wq.cpu(), expect)
    # the term is active: it changes decisions against the same call without it
    assert (codes != plain).sum().item() > 0
    # independent runs: the output error of the GPU result is that of the oracle's own
    # solve on the fp64 statistics of the same tokens
    Xq64, Xf64 = _np(Xq), _np(Xf)
    Hx = O.gram(Xq64)
    Hd_x, dead_x = O.dead_and_damp(Hx, 0.01)
    Cx = O.cross_gram(Xq64, Xf64) if gptaq else None
    U_x = O.upper_factor(Hd_x)
    Wx = W64[rows].copy()
    Wx[:, dead_x] = 0.0
    s_ora, _ = O.symmetric_scale(W64[rows], bits)
    _, W_ora, _ = O.row_form_sweep(U_x, Wx, s_ora, bits, B,
                                   P1=O.gptaq_p1(Cx, U_x) if gptaq else None,
                                   P2=O.cae_p2(Hx, Cx, U_x))
    W_gpu_hat = O.dequantize(c_gpu[rows], s_gpu[rows, None], bits)
    e_gpu = O.layer_error(Hx, W64[rows], W_gpu_hat)
    e_ora = O.layer_error(Hx, W64[rows], W_ora)
    assert abs(e_gpu - e_ora) <= TOL_RECON * e_ora, (e_gpu, e_ora)


@pytest.mark.parametrize("gptaq", [False, True])
def test_cae_lanes_sweep(gptaq):
    # few channels: four lanes per channel; K spans several blocks and a ragged tail
    _check(392, 200, 3, 128, seed=11 + gptaq, gptaq=gptaq)


def test_cae_small_blocks_fp32_dead():
    _check(200, 72, 4, 32, seed=5, gptaq=True, wdtype=torch.float32, dead_cols=(3, 150))


@pytest.mark.parametrize("form", [None, "0"])
@pytest.mark.parametrize("gptaq,K", [(False, 256), (True, 640)])
def test_cae_many_channels(gptaq, K, form, monkeypatch):
    # many channels: two lanes per channel by default, or one thread per channel
    # (checked on a sample of channels)
    if form is not None:
        monkeypatch.setenv("GPTQ_SWEEP_FORM", form)
    _check(K, 9600, 2, 128, seed=31 + gptaq, gptaq=gptaq, sample=96)


def test_cae_crosses_super_blocks():
    # K past one 512-coordinate super-block: near and far lazy updates carry E'
    _check(1096, 160, 3, 128, seed=17, gptaq=True, sample=40)


def test_cae_three_weight_example_on_gpu(golden):
    g = golden("three_weight_counterexample.txt")
    d = dev()
    Ht = torch.tensor(g["H"], dtype=torch.float32, device=d)
    W = torch.tensor(np.asarray(g["w"])[None, :], dtype=torch.float32, device=d)
    out = solve_on_gpu(Ht, W, 4, 16, 0.0, scales_in=torch.ones(1, device=d), cae=True)
    # worked by hand from the pages' update (the oracle pin of the same trace)
    np.testing.assert_array_equal(out["W_hat"][0], [0.0, -1.0, 1.0])


@pytest.mark.parametrize("G,static", [(64, False), (128, True)])
def test_cae_grouped_act_order(G, static):
    d = dev()
    K, N, bits, B = 384, 96, 3, 128
    H, C, _, _, g = _streams(K, 4 * K, 40 + G + static, dead_cols=(9,))
    W = (0.02 * torch.randn(N, K, device=d, generator=g)).to(torch.bfloat16)
    perm = gq.gptq_act_order(H)
    Hp = gq.gptq_permute_hessian(H, perm)
    Cp = gq.gptq_permute_hessian(C, perm)
    H_in = _np(Hp)
    dead = torch.empty(K, dtype=torch.uint8, device=d)
    st = gq.gptq_prepare(Hp, 0.01, dead_out=dead)
    P1 = torch.empty(K, K, device=d)
    gq.gptaq_residual(P1, Cp, Hp)
    Wq = W.clone()
    codes, scales, g_idx, st = gq.gptq_quantize_layer_grouped(
        Wq, Hp, bits, B, G, static_groups=static, perm=perm, P1=P1, dead=dead,
        write_back=True, status=st, cae=True)
    gq.raise_on_status(st, "grouped cae")
    torch.cuda.synchronize()
    order = perm.cpu().numpy()
    Hd, dead_o = O.dead_and_damp(H_in, 0.01)
    U_ora = O.upper_factor(Hd)
    assert rel_max(_np(Hp), U_ora) <= TOL_U
    C64 = _np(Cp)
    W64 = _np(W)
    dead_orig = np.zeros(K, bool)
    dead_orig[order[dead_o]] = True
    Wz = W64.copy()
    Wz[:, dead_orig] = 0.0
    c_gpu = codes.cpu().numpy().astype(np.float64)
    rep = O.replay_row_form_grouped(
        U_ora, Wz, bits, G, c_gpu, static=static, perm=order,
        static_scales=O.static_group_scales(W64, bits, G) if static else None,
        P1=O.gptaq_p1(C64, U_ora), P2=O.cae_p2(H_in, C64, U_ora))
    assert rep["mismatches"] == 0, rep["mismatches"]
    assert 1.0 - rep["tie_flips"] / c_gpu.size >= CODE_SAME
    np.testing.assert_array_equal(g_idx.cpu().numpy(), rep["g_idx"])
    # re-estimated scales are maxima of compensated weights, so they carry the
    # trajectory's error, which U's own tolerance bounds
    np.testing.assert_allclose(_np(scales), rep["scales"], rtol=TOL_U)
    z = 2 ** (bits - 1)
    gi = g_idx.cpu().numpy()
    expect = torch.tensor((scales.cpu().numpy()[:, gi].astype(np.float32) *
                           (codes.cpu().numpy().astype(np.float32) - z))).to(W.dtype)
    assert torch.equal(Wq.cpu(), expect)
