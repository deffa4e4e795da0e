"""The synthetic inputs follow their stated recipes (CPU, small sizes of each workload).

These inputs stand in for the pages' calibration data, so their statistics are checked:
the Student-t stream's variance and tails, the rotated stream's orthogonal rotation that
leaves the layer's outputs unchanged and spreads the outlier channels, the asymmetric
streams' noise level, the group weights' mean, the weights' spread, and that any chunk of
a long stream can be regenerated on its own.
"""

import numpy as np
import pytest
import torch

from post_weight_quantization_solve_b200 import synth


def _small(name, **kw):
    base = dict(K=256, N=64, M=16384, chunk=4096)
    base.update(kw)
    return synth.WORKLOADS[name].scaled(**base)


def test_student_t_stream_unit_variance_heavy_tails():
    wl = _small("mlp_up")
    X = torch.cat([synth.tokens_chunk(wl, c) for c in range(synth.num_chunks(wl))]).double()
    assert X.dtype == torch.float64 and X.shape == (wl.M, wl.K)
    assert float(X.var()) == pytest.approx(1.0, rel=0.1)
    # t with 4 degrees of freedom: far heavier tails than a normal sample of this size
    kurt = float(((X - X.mean()) ** 4).mean() / X.var() ** 2)
    assert kurt > 4.5
    assert float(X.abs().max()) > 8.0


def test_rotation_is_orthogonal_and_keeps_the_layer():
    wl = _small("q_proj", N=32)
    R = synth._rotation(wl, "cpu").double()
    np.testing.assert_allclose((R @ R.T).numpy(), np.eye(wl.K), atol=1e-12)
    # X and W are rotated alike, so X W^T is the unrotated layer's output
    g = synth.generator(wl.seed, synth.T_X, 0)
    X0 = torch.randn(512, wl.K, generator=g)
    X0[:, synth._outlier_channels(wl, "cpu")] *= 20.0
    Xr = synth.tokens_chunk(wl, 0, rows=512).double()
    np.testing.assert_allclose(Xr.numpy(), (X0.double() @ R).numpy(), rtol=1e-2, atol=0.05)
    W0 = torch.randn(wl.N, wl.K, generator=synth.generator(wl.seed, synth.T_W, 0)) * wl.w_sigma
    Wr = synth.weights(wl).double()
    out_rot = (Xr @ Wr.T).numpy()
    out_ref = (X0.double() @ W0.double().T).numpy()
    assert np.abs(out_rot - out_ref).max() <= 0.02 * np.abs(out_ref).max()


def test_outlier_channels_are_spread_by_the_rotation():
    wl = _small("q_proj")
    idx = synth._outlier_channels(wl, "cpu")
    assert len(set(idx.tolist())) == wl.outliers == 16
    Xr = synth.tokens_chunk(wl, 0).double()
    col_rms = Xr.pow(2).mean(0).sqrt()
    # before the rotation 16 channels carry 20x the rms; after it every coordinate
    # carries about the same energy
    assert float(col_rms.max() / col_rms.min()) < 1.5
    expect = np.sqrt((wl.K - 16 + 16 * 400) / wl.K)
    assert float(col_rms.mean()) == pytest.approx(expect, rel=0.05)


def test_asymmetric_streams_noise_level():
    wl = _small("gptaq")
    n = synth.num_chunks(wl)
    Xf = torch.cat([synth.fp_tokens_chunk(wl, c) for c in range(n)]).double()
    Xq = torch.cat([synth.tokens_chunk(wl, c) for c in range(n)]).double()
    rms = float(Xf.pow(2).mean().sqrt())
    assert synth.fp_stream_rms(wl) == pytest.approx(rms, rel=1e-6)
    D = Xq - Xf
    assert float(D.pow(2).mean().sqrt()) == pytest.approx(0.05 * rms, rel=0.1)
    assert float(D.mean()) == pytest.approx(0.0, abs=2e-3)


def test_group_weights_have_mean_one_over_the_stream():
    wl = _small("grouped70b", N=64)
    n = synth.num_chunks(wl)
    S = torch.cat([synth.token_weights_chunk(wl, c) for c in range(n)], dim=1).double()
    assert S.shape == (wl.groups, wl.M)
    assert float(S.min()) >= 0.0
    np.testing.assert_allclose(S.mean(1).numpy(), np.ones(wl.groups), rtol=1e-5)
    # squared normals: variance 2 after normalising the mean to one
    assert float(S.var(1).mean()) == pytest.approx(2.0, rel=0.15)


@pytest.mark.parametrize("name", ["mlp_up", "gptaq", "grouped70b", "tiny"])
def test_weights_spread_and_dtype(name):
    wl = synth.WORKLOADS[name].scaled(K=128, N=256, M=2048, chunk=1024)
    W = synth.weights(wl)
    assert W.shape == (wl.N, wl.K) and W.dtype == wl.xdtype
    assert float(W.double().std()) == pytest.approx(wl.w_sigma, rel=0.05)


def test_chunks_regenerate_on_their_own_and_the_last_is_ragged():
    wl = _small("mlp_up", M=10000)
    assert synth.num_chunks(wl) == 3
    a = synth.tokens_chunk(wl, 1)
    b = synth.tokens_chunk(wl, 1)
    assert torch.equal(a, b)
    assert not torch.equal(a, synth.tokens_chunk(wl, 0))
    assert synth.tokens_chunk(wl, 2).shape == (10000 - 2 * 4096, wl.K)


def test_correlated_stream_covariance():
    wl = synth.WORKLOADS["tiny"].scaled(M=65536, chunk=65536)
    X = synth.tokens_chunk(wl, 0).double()
    A = torch.randn(wl.K, wl.K, generator=synth.generator(wl.seed, synth.T_MIX, 0),
                    dtype=torch.float64) / wl.K ** 0.5
    cov = (X.T @ X / X.shape[0]).numpy()
    ref = (A.T @ A).numpy()
    assert np.abs(cov - ref).max() <= 0.05 * np.abs(ref).max()
