"""Shared pieces of the GPU parity tests: run the C-ABI path, compare with the oracle."""

import numpy as np
import torch

import oracle as O
import post_weight_quantization_solve_b200 as gq

# Tolerances: H, U, P1 within 1e-4 max-norm relative error (fp32 accumulation against
# fp64); codes identical on >= 99.9 % of entries with every difference a near tie
# (|frac - 1/2| < 1e-4, followed by the oracle's replay); output error within 1e-3
# relative of the oracle's own solve.
TOL_H = 1e-4
TOL_U = 1e-4
TOL_P1 = 1e-4
CODE_SAME = 0.999
TIE_BAND = 1e-4
TOL_RECON = 1e-3


def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda:0")


def rel_max(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-300))


def gpu_hessian(chunks, K, g=1, weights=None, device=None):
    """Accumulate H over a list of token chunks through the C ABI."""
    device = device or dev()
    H = torch.zeros((g, K, K) if g > 1 else (K, K), device=device)
    for i, X in enumerate(chunks):
        w = None if weights is None else weights[i].to(device).contiguous()
        gq.gptq_accumulate_hessian(H, X.to(device).contiguous(), w)
    return H


def solve_on_gpu(H, W, bits, blocksize, percdamp, groups=1, P1_from_C=None, scales_in=None,
                 write_back=True, cae=False):
    """prepare + (residual) + quantize on the device; returns host numpy results."""
    d = H.device
    K = H.shape[-1]
    N = W.shape[0]
    U = H.clone()
    dead = torch.zeros((groups, K), dtype=torch.uint8, device=d)
    status = gq.gptq_prepare(U, percdamp, dead_out=dead)
    P1 = None
    if P1_from_C is not None:
        P1 = torch.empty(K, K, device=d)
        gq.gptaq_residual(P1, P1_from_C, U)
    Wd = W.to(d).clone()
    scales = torch.empty(N, device=d)
    loss = torch.empty(N, device=d)
    codes, status = gq.gptq_quantize_layer(
        Wd, U, bits, blocksize, groups=groups, P1=P1, dead=dead, scales_in=scales_in,
        scales_out=scales, loss=loss, write_back=write_back, status=status, cae=cae)
    gq.raise_on_status(status, "solve")
    torch.cuda.synchronize()
    return dict(U=U.double().cpu().numpy(), codes=codes.cpu().numpy().astype(np.float64),
                W_hat=Wd.double().cpu().numpy(), scales=scales.double().cpu().numpy(),
                loss=loss.double().cpu().numpy(), dead=dead.cpu().numpy().astype(bool),
                P1=None if P1 is None else P1.double().cpu().numpy())


def check_codes_by_replay(U_ora, W_in, scales, bits, codes_gpu, P1=None, rows=None):
    """Tie-follow replay (oracle decisions vs the GPU's). Returns the replay dict."""
    W_in = np.asarray(W_in, dtype=np.float64)
    if rows is not None:
        W_in, scales, codes_gpu = W_in[rows], scales[rows], codes_gpu[rows]
    rep = O.replay_row_form(U_ora, W_in, scales, bits, codes_gpu, P1=P1, band=TIE_BAND)
    same = float(np.mean(rep["codes"] == codes_gpu))  # replay adopts GPU codes: compare own
    return rep, same


def own_decisions_same(rep, total):
    """Fraction of entries where the oracle's own decision equalled the GPU's."""
    return 1.0 - (rep["tie_flips"] + rep["mismatches"]) / total
