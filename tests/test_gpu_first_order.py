"""First-order (gradient) term on the GPU vs the fp64 oracle (C ABI calls).

The library applies the term as a shifted start W - beta G H^-1 (through U; tf32x3
tensor-core products for K a multiple of 32 from 256, the fp32 SIMT GEMM otherwise) and then
runs the ordinary sweep on the shifted fp32 weights; the oracle's explicit per-step
form equals that reading by its CPU pins. Here: the shift and gamma against the fp64
solve, then the sweep on the shifted weights by tie-follow replay. The reading itself
is unpinned against the pages (they print no formula).
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
    assert rel_max(_np(Ws) - _np(W), -beta * T64 @ U64) <= TOL_KERNEL
    assert gamma.item() == pytest.approx(float(np.sum(T64 * T64)), rel=TOL_KERNEL)
    # end to end against the fp64 solve: the step applies U twice, so its bound is U's
    # tolerance amplified by the conditioning of H (checked here with a 10x margin)
    assert rel_max(_np(Ws) - _np(W), W_ora - _np(W)) <= 10 * TOL_U
    assert gamma.item() == pytest.approx(gamma_ora, rel=10 * TOL_U)


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
