"""gptq_prepare_noalloc: the prepare step for callers that cannot allocate device
memory when they need the factor (a host application that owns every device
allocation and gives plug-ins no workspace, or a path that must not take the
device-wide synchronisation of cudaMalloc / cudaFree).

It runs the same kernels as gptq_prepare with the library's fixed scratch array,
so its U must match gptq_prepare's. The array keeps the previous call's contents;
several calls in a row, of different sizes, check that nothing stale leaks into
the next result. This file is collected last on purpose.
"""

import ctypes

import pytest
import torch

import post_weight_quantization_solve_b200 as gq
from post_weight_quantization_solve_b200 import synth
from post_weight_quantization_solve_b200.build import build

from gpu_util import TOL_U, dev, rel_max

pytestmark = pytest.mark.gpu


def _hessian(K, seed, d, g=1):
    Hs = []
    for gi in range(g):
        wl = synth.WORKLOADS["mlp_up"].scaled(K=K, N=8, M=3 * K, seed=seed + 101 * gi)
        X = synth.tokens_chunk(wl, 0, d).float()
        Hs.append(2.0 * (X.T @ X))          # test input only
    return Hs[0] if g == 1 else torch.stack(Hs)


def _noalloc(lib, H, percdamp, dead, status):
    g = 1 if H.dim() == 2 else H.shape[0]
    return lib.gptq_prepare_noalloc(ctypes.c_void_p(H.data_ptr()), H.shape[-1], g,
                                    ctypes.c_float(percdamp), ctypes.c_void_p(dead.data_ptr()),
                                    ctypes.c_void_p(status.data_ptr()),
                                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


# Sizes in an order that would expose stale scratch from the call before: the SIMT path
# (K = 1000, 4096) and the tensor-core path, where the array also holds the tf32 pairs
# and the lookahead's panel buffers (K = 512 and 896 with one Hessian, K = 512 with two).
CASES = [(1000, 1, 11), (512, 1, 14), (4096, 1, 12), (896, 1, 15), (512, 2, 16), (1000, 1, 13),
         (512, 1, 17)]


def test_noalloc_prepare_matches_workspace_prepare():
    build()
    lib = gq.load_library()
    d = dev()
    for K, g, seed in CASES:
        H = _hessian(K, seed, d, g)
        U_ref = H.clone()
        dead_ref = torch.empty((g, K) if g > 1 else (K,), dtype=torch.uint8, device=d)
        st_ref = gq.gptq_prepare(U_ref, 0.01, dead_out=dead_ref)
        U_new = H.clone()
        dead_new = torch.full_like(dead_ref, 7)
        st_new = torch.zeros(1, dtype=torch.int32, device=d)
        assert _noalloc(lib, U_new, 0.01, dead_new, st_new) == gq.GPTQ_OK
        torch.cuda.synchronize()
        assert int(st_ref.item()) == gq.GPTQ_OK and int(st_new.item()) == gq.GPTQ_OK
        assert rel_max(U_new.double().cpu().numpy(), U_ref.double().cpu().numpy()) <= TOL_U, (K, g)
        assert torch.equal(dead_new, dead_ref)


def test_noalloc_prepare_rejects_sizes_beyond_its_scratch():
    lib = gq.load_library()
    d = dev()
    H = torch.zeros(4, device=d)     # never read: the call is refused on the host
    st = torch.zeros(1, dtype=torch.int32, device=d)
    assert lib.gptq_prepare_noalloc(ctypes.c_void_p(H.data_ptr()), 4097, 1, ctypes.c_float(0.01),
                                    None, ctypes.c_void_p(st.data_ptr()), None) == gq.GPTQ_ERR_ARG
    assert lib.gptq_prepare_noalloc(ctypes.c_void_p(H.data_ptr()), 2048, 5, ctypes.c_float(0.01),
                                    None, ctypes.c_void_p(st.data_ptr()), None) == gq.GPTQ_ERR_ARG
    torch.cuda.synchronize()
    assert int(st.item()) == 0
