"""Input-dimension groups and act-order on the GPU vs the fp64 oracle (C ABI calls).

The act-order permutation and the reordered Hessian are integer / copy work and must
match bit for bit. The quantisation follows the parity protocol of the plain sweep:
the oracle factors the GPU's (reordered, damped) Hessian, replays the sweep with
tie-following against the GPU's codes (re-estimated group scales recomputed along
that trajectory), and the outputs must sit exactly on each coordinate's group grid.
"""

import numpy as np
import pytest
import torch

import oracle as O
import post_weight_quantization_solve_b200 as gq
from post_weight_quantization_solve_b200.build import build

from gpu_util import CODE_SAME, TOL_U, dev, rel_max

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    gq.load_library()


def _np(t):
    return t.double().cpu().numpy()


def _problem(K, N, M, seed, wdtype=torch.bfloat16, dead_cols=()):
    d = dev()
    g = torch.Generator(device=d).manual_seed(seed)
    A = torch.randn(K, K, device=d, generator=g) / K ** 0.5
    X = (torch.randn(M, K, device=d, generator=g) @ A).to(torch.bfloat16)
    for c in dead_cols:
        X[:, c] = 0
    H = torch.zeros(K, K, device=d)
    gq.gptq_accumulate_hessian(H, X.contiguous())
    W = (0.02 * torch.randn(N, K, device=d, generator=g)).to(wdtype)
    return H, W


def test_act_order_and_permutation_exact():
    d = dev()
    K = 296      # bf16 token rows need K % 8 == 0; not a multiple of the tile sizes
    H, _ = _problem(K, 8, 2048, 1, dead_cols=(7, 123))
    # a tie on the diagonal
    H[5, 5] = H[17, 17]
    perm = gq.gptq_act_order(H)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(perm.cpu().numpy(), O.act_order(_np(H)))
    Hp = gq.gptq_permute_hessian(H, perm)
    p = perm.long()
    assert torch.equal(Hp, H[p][:, p])


def _run(K, N, bits, blocksize, G, static, act, seed, wdtype=torch.bfloat16, dead_cols=(),
         sample=None):
    H, W = _problem(K, N, 4 * K, seed, wdtype, dead_cols)
    perm = gq.gptq_act_order(H) if act else None
    Hp = gq.gptq_permute_hessian(H, perm) if act else H.clone()
    H_in = _np(Hp)
    dead = torch.empty(K, dtype=torch.uint8, device=H.device)
    st = gq.gptq_prepare(Hp, 0.01, dead_out=dead)
    gq.raise_on_status(st, "prepare")
    Wq = W.clone()
    codes, scales, g_idx, st = gq.gptq_quantize_layer_grouped(
        Wq, Hp, bits, blocksize, G, static_groups=static, perm=perm, dead=dead, write_back=True)
    gq.raise_on_status(st, "quantize")
    torch.cuda.synchronize()
    order = None if perm is None else perm.cpu().numpy()
    Hd, dead_ora = O.dead_and_damp(H_in, 0.01)
    np.testing.assert_array_equal(dead.cpu().numpy().astype(bool), dead_ora)
    U_ora = O.upper_factor(Hd)
    assert rel_max(_np(Hp), U_ora) <= TOL_U
    W64 = _np(W)
    # dead coordinates (processing positions) are zeroed before the sweep
    dead_orig = np.zeros(K, bool)
    dead_orig[(order if order is not None else np.arange(K))[dead_ora]] = True
    W64z = W64.copy()
    W64z[:, dead_orig] = 0.0
    c_gpu = codes.cpu().numpy().astype(np.float64)
    rows = np.arange(N) if sample is None else np.sort(np.random.default_rng(seed).choice(N, sample, replace=False))
    s_gpu = _np(scales)
    rep = O.replay_row_form_grouped(U_ora, W64z[rows], bits, G, c_gpu[rows], static=static,
                                    perm=order,
                                    static_scales=(O.static_group_scales(W64, bits, G)[rows]
                                                   if static else None))
    assert rep["mismatches"] == 0, rep["mismatches"]
    same = 1.0 - rep["tie_flips"] / c_gpu[rows].size
    assert same >= CODE_SAME
    np.testing.assert_array_equal(g_idx.cpu().numpy(), rep["g_idx"])
    # re-estimated scales are maxima of compensated weights, so they carry the
    # trajectory's error, which U's own tolerance bounds
    np.testing.assert_allclose(s_gpu[rows], rep["scales"], rtol=TOL_U)
    # reconstruction on each coordinate's group grid, in the weights' dtype
    z = 2 ** (bits - 1)
    gi = g_idx.cpu().numpy()
    expect = torch.tensor((scales.cpu().numpy()[:, gi].astype(np.float32) *
                           (codes.cpu().numpy().astype(np.float32) - z))).to(W.dtype)
    assert torch.equal(Wq.cpu(), expect)


@pytest.mark.parametrize("G,static,act", [(32, False, False), (64, False, True),
                                          (128, False, True), (128, True, True),
                                          (64, True, False), (32, True, True)])
def test_grouped_sweep_matches_oracle(G, static, act):
    _run(384, 96, 3, 128, G, static, act, seed=G + 7 * static + 3 * act)


def test_grouped_ragged_and_dead_fp32():
    # K not a multiple of the group or block size, two dead coordinates, fp32 weights
    _run(200, 40, 4, 64, 32, False, True, seed=21, wdtype=torch.float32, dead_cols=(3, 150))


def test_grouped_wide_layer_thread_sweep():
    # N large enough for the one-thread-per-channel sweep
    _run(256, 10240, 3, 128, 128, False, True, seed=5, sample=64)


@pytest.mark.slow
def test_grouped_q_proj_size():
    _run(4096, 4096, 3, 128, 128, False, True, seed=9, sample=24)
