"""First-order (gradient) term on the GPU vs the fp64 oracle (C ABI calls).

The library applies the term as a shifted start W - beta G H^-1 (through U; tf32x3
tensor-core products for K a multiple of 32 from 256, the fp32 SIMT GEMM otherwise) and then
runs the ordinary sweep on the shifted fp32 weights. Here:
  - the shift and gamma against the same factor in fp64 (the kernel's own error), and
    against the fp64 solve within a first-order perturbation bound derived per case from
    U's measured error and the case's own G and H_d (no fixed widening);
  - the codes of the whole GPU path (shift, then sweep) against the oracle's explicit
    per-step first-order sweep from its own fp64 start, by tie-follow;
  - the sweep on the GPU's shifted weights by the row-form replay.
The reading itself is unpinned against the pages (they print no formula).
"""

import numpy as np
import pytest
import torch

import oracle as O
import post_weight_quantization_solve_b200 as gq
from post_weight_quantization_solve_b200.build import build

from gpu_util import CODE_SAME, TIE_BAND, TOL_P1, TOL_U, dev, rel_max

pytestmark = pytest.mark.gpu

# the two chained tf32x3 products against the same operands in fp64: the bound of P1,
# which the residual computes by the same two-product route
TOL_KERNEL = TOL_P1


def shift_bound(U_gpu, U_ora, Hd, G):
    """First-order perturbation bounds of the shift d = -beta G M (M = H_d^-1 = U^T U) and
    of gamma = sum_n g_n M g_n^T when M is formed from the GPU's U instead of the exact
    factor. With eps = ||U_gpu - U_ora||_2 / ||U_ora||_2,
        ||U_gpu^T U_gpu - M||_2 <= (2 eps + eps^2) ||M||_2,
    so ||delta d||_F <= (2 eps + eps^2) ||M||_2 beta ||G||_F and
    |delta gamma| <= (2 eps + eps^2) ||M||_2 ||G||_F^2. Relative to the exact values:
        d:     (2 eps + eps^2) * ||G||_F ||M||_2 / ||G M||_F      (<= (2 eps + eps^2) kappa(H_d))
        gamma: (2 eps + eps^2) * ||G||_F^2 ||M||_2 / gamma.
    Returns (eps, rel_d, rel_gamma)."""
    eps = np.linalg.norm(U_gpu - U_ora, 2) / np.linalg.norm(U_ora, 2)
    M = np.linalg.inv(Hd)
    m2 = np.linalg.norm(M, 2)
    gf = np.linalg.norm(G)
    amp = 2 * eps + eps * eps
    gamma = float(np.sum((G @ M) * G))
    return eps, amp * gf * m2 / np.linalg.norm(G @ M), amp * gf * gf * m2 / gamma


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    gq.load_library()


def _np(t):
    return t.double().cpu().numpy()


def _setup(K, N, seed, gdtype):
    d = dev()
    g = torch.Generator(device=d).manual_seed(seed)
    X = (torch.randn(4 * K, K, device=d, generator=g) @
         (torch.randn(K, K, device=d, generator=g) / K ** 0.5)).to(torch.bfloat16)
    H = torch.zeros(K, K, device=d)
    gq.gptq_accumulate_hessian(H, X.contiguous())
    H_in = _np(H)
    U = H.clone()
    st = gq.gptq_prepare(U, 0.01)
    W = (0.02 * torch.randn(N, K, device=d, generator=g))
    G = (0.05 * torch.randn(N, K, device=d, generator=g)).to(gdtype)
    return H_in, U, W, G, st


@pytest.mark.parametrize("K,N,gdtype,beta", [(392, 200, torch.float32, 0.6),
                                             (256, 96, torch.bfloat16, 1.0),
                                             (136, 40, torch.float32, 0.0),
                                             (1024, 300, torch.bfloat16, 0.4)])
def test_shift_and_gamma_match_oracle(K, N, gdtype, beta):
    H_in, U, W, G, st = _setup(K, N, K + N, gdtype)
    Ws = W.clone()
    gamma = torch.zeros(1, dtype=torch.float64, device=dev())
    gq.gptq_first_order_shift(Ws, U, G, beta, gamma=gamma, status=st)
    gq.raise_on_status(st, "shift")
    Hd, _ = O.dead_and_damp(H_in, 0.01)
    W_ora, gamma_ora = O.first_order_shift(Hd, _np(W), _np(G), beta)
    if beta == 0.0:
        assert torch.equal(Ws, W)
        return
    # the kernel: the step against the same factor in fp64, beta G (U^T U) and |G U^T|^2
    U64, G64 = _np(U), _np(G)
    T64 = G64 @ U64.T
    d_gpu, d_same = _np(Ws) - _np(W), -beta * T64 @ U64
    gamma_same = float(np.sum(T64 * T64))
    assert rel_max(d_gpu, d_same) <= TOL_KERNEL
    kern_f = np.linalg.norm(d_gpu - d_same) / np.linalg.norm(d_same)
    assert kern_f <= TOL_KERNEL
    assert gamma.item() == pytest.approx(gamma_same, rel=TOL_KERNEL)
    # end to end against the fp64 solve: U itself within its tolerance, and the shift and
    # gamma within the perturbation that U's measured error allows (shift_bound) plus the
    # kernel's own error on top
    U_ora = O.upper_factor(Hd)
    assert rel_max(U64, U_ora) <= TOL_U
    eps, rel_d, rel_g = shift_bound(U64, U_ora, Hd, G64)
    d_ora = W_ora - _np(W)
    bound_d = kern_f * (1 + rel_d) + rel_d
    assert np.linalg.norm(d_gpu - d_ora) / np.linalg.norm(d_ora) <= bound_d, (eps, rel_d)
    kern_g = abs(gamma.item() - gamma_same) / gamma_same
    assert abs(gamma.item() - gamma_ora) / gamma_ora <= kern_g * (1 + rel_g) + rel_g, (eps, rel_g)


@pytest.mark.parametrize("K,N,bs,gdtype,beta", [(256, 96, 128, torch.float32, 0.7),
                                                (192, 130, 32, torch.bfloat16, 1.0),
                                                (256, 64, 64, torch.bfloat16, 0.35)])
def test_first_order_codes_match_explicit_oracle_sweep(K, N, bs, gdtype, beta):
    # the whole GPU path (tf32x3 shift for K = 256, the SIMT shift for K = 192, then the
    # sweep) against the oracle's explicit per-step solve of the quadratic model from its
    # own fp64 start and scales (the oracle factors nothing: H_d^-1 g and the re-solves
    # are np.linalg.solve on the GPU's Gram, upcast)
    H_in, U, W, G, st = _setup(K, N, 31 + K + N, gdtype)
    Hd, _ = O.dead_and_damp(H_in, 0.01)
    Ws = W.clone()
    gq.gptq_first_order_shift(Ws, U, G, beta, status=st)
    scales = torch.empty(N, device=dev())
    Wq = Ws.clone()
    codes, st = gq.gptq_quantize_layer(Wq, U, 3, bs, scales_out=scales, write_back=True, status=st)
    gq.raise_on_status(st, "first-order solve")
    torch.cuda.synchronize()
    c_gpu = codes.cpu().numpy().astype(np.float64)
    c_ora, w_ora, s_ora, stats = O.first_order_obq_sweep(Hd, _np(W), _np(G), beta, 3,
                                                         follow=c_gpu, band=TIE_BAND)
    assert stats["mismatches"] == 0, stats
    assert 1.0 - stats["tie_flips"] / c_gpu.size >= CODE_SAME
    # scales: |amax(a) - amax(b)| <= max |a - b| per channel, plus fp32 rounding
    Ws_ora, _ = O.first_order_shift(Hd, _np(W), _np(G), beta)
    amax = np.abs(Ws_ora).max(axis=1)
    rtol = np.abs(_np(Ws) - Ws_ora).max(axis=1) / amax + 4 * 2.0 ** -24
    assert np.all(np.abs(_np(scales) - s_ora) <= rtol * s_ora)
    # write-back on the GPU's grid with the followed codes
    z = 4.0
    np.testing.assert_array_equal(_np(Wq), (_np(scales)[:, None] * (c_gpu - z)).astype(np.float32))


@pytest.mark.parametrize("K,N,sample", [(392, 200, None), (256, 9600, 64)])
def test_shifted_sweep_matches_oracle_replay(K, N, sample):
    # lanes and thread sweeps on the shifted fp32 weights
    H_in, U, W, G, st = _setup(K, N, 7 + K, torch.float32)
    Hd, _ = O.dead_and_damp(H_in, 0.01)
    gamma = torch.zeros(1, dtype=torch.float64, device=dev())
    Ws = W.clone()
    gq.gptq_first_order_shift(Ws, U, G, 0.8, gamma=gamma, status=st)
    Wq = Ws.clone()
    scales = torch.empty(N, device=dev())
    loss = torch.empty(N, device=dev())
    codes, st = gq.gptq_quantize_layer(Wq, U, 3, 128, scales_out=scales, loss=loss,
                                       write_back=True, status=st)
    gq.raise_on_status(st, "first-order solve")
    torch.cuda.synchronize()
    U_ora = O.upper_factor(Hd)
    rows = np.arange(N) if sample is None else np.sort(np.random.default_rng(K).choice(N, sample, replace=False))
    Ws64 = _np(Ws)[rows]
    s_gpu = _np(scales)[rows]
    np.testing.assert_allclose(s_gpu, O.symmetric_scale(Ws64, 3)[0], rtol=2e-7)
    c_gpu = codes.cpu().numpy().astype(np.float64)[rows]
    rep = O.replay_row_form(U_ora, Ws64, s_gpu, 3, c_gpu, band=TIE_BAND)
    assert rep["mismatches"] == 0, rep["mismatches"]
    assert 1.0 - rep["tie_flips"] / c_gpu.size >= CODE_SAME
    np.testing.assert_allclose(_np(loss)[rows], rep["loss"], rtol=1e-3, atol=1e-12)
    # the trust-region factor from this solve's own loss and gamma stays in [0, 1]
    b = gq.gptq_trust_region_beta(1.0, float(loss.sum().item()), gamma.item())
    assert 0.0 <= b <= 1.0
    assert b == pytest.approx(O.trust_region_beta(1.0, float(loss.sum().item()), gamma.item()),
                              rel=1e-6, abs=1e-7)
