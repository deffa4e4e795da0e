"""GPTQ-family per-layer solve on B200 (sm_100a): thin binding over libgptq.so.

Each function here has the name of a C entry point of include/gptq.h and only
marshals arguments: torch tensors supply device memory and the CUDA stream, every
step of the solve runs in the library's kernels. There is no fallback: when the
library is missing, every call raises.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgptq.so")

GPTQ_OK, GPTQ_ERR_ARG, GPTQ_ERR_NOT_PD, GPTQ_ERR_NONFINITE = 0, 1, 2, 3
GPTQ_ERR_CUDA, GPTQ_ERR_TIMEOUT, GPTQ_ERR_WORKSPACE = 4, 5, 6
GPTQ_BF16, GPTQ_F32 = 0, 1
GPTQ_OP_PREPARE, GPTQ_OP_RESIDUAL, GPTQ_OP_QUANTIZE, GPTQ_OP_QUANTIZE_GROUPED = 0, 1, 2, 3
GPTQ_OP_FIRST_ORDER = 4
GPTQ_WS_CAE = 0x100

EXPORTS = ("gptq_accumulate_hessian", "gptaq_accumulate_cross", "gptq_prepare",
           "gptq_prepare_noalloc",
           "gptaq_residual", "gptq_quantize_layer", "gptq_act_order", "gptq_permute_hessian",
           "gptq_quantize_layer_grouped", "gptq_pack_codes", "gptq_unpack_codes",
           "gptq_first_order_shift", "gptq_trust_region_beta", "gptq_selftest_timeout",
           "gptq_workspace_size",
           "gptq_kernel_launches", "gptq_status_string")

_lib = None


class GPTQError(RuntimeError):
    def __init__(self, code, where=""):
        self.code = int(code)
        super().__init__(f"{where}: {gptq_status_string(code)} (status {self.code})")


def load_library():
    """Load libgptq.so from the package directory (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m post_weight_quantization_solve_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, I64, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    sig = {
        "gptq_accumulate_hessian": [P, I, I, P, I, I64, I64, P, I64, P, P],
        "gptaq_accumulate_cross": [P, I, P, P, I, I64, I64, P, P],
        "gptq_prepare": [P, I, I, F, P, P, SZ, P, P],
        "gptq_prepare_noalloc": [P, I, I, F, P, P, P],
        "gptaq_residual": [P, P, P, I, P, SZ, P],
        "gptq_quantize_layer": [P, I, I, I, P, I, I, I, P, I, P, P, P, P, P, I, P, SZ, P, P],
        "gptq_act_order": [P, I, P, P],
        "gptq_permute_hessian": [P, P, I, P, P],
        "gptq_quantize_layer_grouped": [P, I, I, I, P, I, I, I, I, P, P, I, P, P, P, P, P, I, P,
                                        SZ, P, P],
        "gptq_pack_codes": [P, I, I, I64, I, P, I64, P],
        "gptq_unpack_codes": [P, I, I, I64, I, P, I64, P],
        "gptq_first_order_shift": [P, I, I, P, P, I, F, P, P, SZ, P, P],
        "gptq_trust_region_beta": [F, ctypes.c_double, ctypes.c_double],
        "gptq_selftest_timeout": [P, P],
        "gptq_workspace_size": [I, I, I, I, I],
        "gptq_status_string": [I],
        "gptq_kernel_launches": [],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    lib.gptq_workspace_size.restype = ctypes.c_size_t
    lib.gptq_trust_region_beta.restype = ctypes.c_float
    lib.gptq_status_string.restype = ctypes.c_char_p
    lib.gptq_kernel_launches.restype = ctypes.c_ulonglong
    _lib = lib
    return lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return GPTQ_BF16
    if t.dtype == torch.float32:
        return GPTQ_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _check(code, where):
    if code != GPTQ_OK:
        raise GPTQError(code, where)


def _workspace(nbytes, device, workspace):
    if workspace is not None:
        return workspace
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


def new_status(device="cuda"):
    """A zeroed device status word."""
    return torch.zeros(1, dtype=torch.int32, device=device)


def raise_on_status(status, where="gptq"):
    """Synchronise with the status word's device and raise if a kernel failed."""
    code = int(status.item())
    _check(code, where)


def gptq_status_string(code):
    return load_library().gptq_status_string(int(code)).decode()


def gptq_kernel_launches():
    """Kernels enqueued through the library by this process so far."""
    return int(load_library().gptq_kernel_launches())


def gptq_workspace_size(op, K, N=0, g=1, blocksize=0):
    return int(load_library().gptq_workspace_size(op, K, N, g, blocksize))


def gptq_accumulate_hessian(H, X, w=None, status=None, stream=None):
    """H[g] += 2 X^T diag(w[g]) X (see include/gptq.h). H: (K,K) or (g,K,K) fp32."""
    lib = load_library()
    K = H.shape[-1]
    g = 1 if H.dim() == 2 else H.shape[0]
    M = X.shape[0]
    ldw = 0 if w is None else w.stride(0) if w.dim() == 2 else w.shape[-1]
    code = lib.gptq_accumulate_hessian(_ptr(H), K, g, _ptr(X), _dtype_code(X), M, X.stride(0),
                                       _ptr(w), ldw, _ptr(status), _stream(stream))
    _check(code, "gptq_accumulate_hessian")


def gptaq_accumulate_cross(C, X_fp, X_q, status=None, stream=None):
    """C += 2 (X_fp - X_q)^T X_q (see include/gptq.h)."""
    lib = load_library()
    if X_fp.stride(0) != X_q.stride(0) or X_fp.dtype != X_q.dtype or X_fp.shape != X_q.shape:
        raise ValueError("X_fp and X_q must share shape, dtype and row stride")
    code = lib.gptaq_accumulate_cross(_ptr(C), C.shape[-1], _ptr(X_fp), _ptr(X_q),
                                      _dtype_code(X_q), X_q.shape[0], X_q.stride(0),
                                      _ptr(status), _stream(stream))
    _check(code, "gptaq_accumulate_cross")


def gptq_prepare(H, percdamp=0.01, dead_out=None, workspace=None, status=None, stream=None):
    """In place: dead fix, damping, H -> U. Returns the status tensor (not synchronised)."""
    lib = load_library()
    K = H.shape[-1]
    g = 1 if H.dim() == 2 else H.shape[0]
    status = new_status(H.device) if status is None else status
    ws = _workspace(gptq_workspace_size(GPTQ_OP_PREPARE, K, 0, g, 0), H.device, workspace)
    code = lib.gptq_prepare(_ptr(H), K, g, float(percdamp), _ptr(dead_out), _ptr(ws),
                            ws.numel() * ws.element_size(), _ptr(status), _stream(stream))
    _check(code, "gptq_prepare")
    return status


def gptq_prepare_noalloc(H, percdamp=0.01, dead_out=None, status=None, stream=None):
    """gptq_prepare with the library's fixed device scratch instead of a workspace
    (no allocation anywhere on this path). Returns the status tensor."""
    lib = load_library()
    K = H.shape[-1]
    g = 1 if H.dim() == 2 else H.shape[0]
    if status is None:
        raise ValueError("gptq_prepare_noalloc needs a caller-provided status word")
    code = lib.gptq_prepare_noalloc(_ptr(H), K, g, float(percdamp), _ptr(dead_out),
                                    _ptr(status), _stream(stream))
    _check(code, "gptq_prepare_noalloc")
    return status


def gptaq_residual(P1, C, U, workspace=None, stream=None):
    """P1 = [(C U^T) ⊙ strict-upper] U (see include/gptq.h)."""
    lib = load_library()
    K = U.shape[-1]
    ws = _workspace(gptq_workspace_size(GPTQ_OP_RESIDUAL, K, 0, 1, 0), U.device, workspace)
    code = lib.gptaq_residual(_ptr(P1), _ptr(C), _ptr(U), K, _ptr(ws),
                              ws.numel() * ws.element_size(), _stream(stream))
    _check(code, "gptaq_residual")


def gptq_quantize_layer(W, U, bits, blocksize=128, groups=1, P1=None, dead=None, scales_in=None,
                        scales_out=None, codes=None, loss=None, write_back=False,
                        workspace=None, status=None, stream=None, cae=False):
    """The shared-order sweep (cae: with the compensation-aware error term).
    Returns (codes, status); see include/gptq.h."""
    lib = load_library()
    N, K = W.shape
    if codes is None:
        codes = torch.empty(N, K, dtype=torch.uint8, device=W.device)
    status = new_status(W.device) if status is None else status
    op = GPTQ_OP_QUANTIZE | (GPTQ_WS_CAE if cae else 0)
    ws = _workspace(gptq_workspace_size(op, K, N, groups, blocksize), W.device, workspace)
    code = lib.gptq_quantize_layer(_ptr(W), _dtype_code(W), N, K, _ptr(U), groups, bits,
                                   blocksize, _ptr(P1), int(bool(cae)), _ptr(dead), _ptr(scales_in),
                                   _ptr(scales_out), _ptr(codes), _ptr(loss), int(write_back),
                                   _ptr(ws), ws.numel() * ws.element_size(), _ptr(status),
                                   _stream(stream))
    _check(code, "gptq_quantize_layer")
    return codes, status


def gptq_act_order(H, perm=None, stream=None):
    """The act-order processing order of H's input coordinates (int32 [K])."""
    lib = load_library()
    K = H.shape[-1]
    if perm is None:
        perm = torch.empty(K, dtype=torch.int32, device=H.device)
    _check(lib.gptq_act_order(_ptr(H), K, _ptr(perm), _stream(stream)), "gptq_act_order")
    return perm


def gptq_permute_hessian(H, perm, out=None, stream=None):
    """out = H[perm][:, perm] (a new K x K tensor unless `out` is given)."""
    lib = load_library()
    K = H.shape[-1]
    if out is None:
        out = torch.empty_like(H)
    _check(lib.gptq_permute_hessian(_ptr(out), _ptr(H), K, _ptr(perm), _stream(stream)),
           "gptq_permute_hessian")
    return out


def gptq_quantize_layer_grouped(W, U, bits, blocksize=128, groupsize=128, static_groups=False,
                                perm=None, P1=None, dead=None, scales_out=None, g_idx=None,
                                codes=None, loss=None, write_back=False, workspace=None,
                                status=None, stream=None, cae=False):
    """The sweep with input-dimension groups and an optional processing order.
    Returns (codes, scales [N][ceil(K / groupsize)], g_idx [K], status); see include/gptq.h."""
    lib = load_library()
    N, K = W.shape
    if codes is None:
        codes = torch.empty(N, K, dtype=torch.uint8, device=W.device)
    if scales_out is None:
        shape = (N, (K + groupsize - 1) // groupsize) if groupsize else (N,)
        scales_out = torch.empty(shape, dtype=torch.float32, device=W.device)
    if g_idx is None:
        g_idx = torch.empty(K, dtype=torch.int32, device=W.device)
    status = new_status(W.device) if status is None else status
    op = GPTQ_OP_QUANTIZE_GROUPED | (GPTQ_WS_CAE if cae else 0)
    ws = _workspace(gptq_workspace_size(op, K, N, 1, blocksize), W.device, workspace)
    code = lib.gptq_quantize_layer_grouped(_ptr(W), _dtype_code(W), N, K, _ptr(U), bits, blocksize,
                                           groupsize, int(bool(static_groups)), _ptr(perm),
                                           _ptr(P1), int(bool(cae)), _ptr(dead), _ptr(scales_out),
                                           _ptr(g_idx),
                                           _ptr(codes), _ptr(loss), int(write_back), _ptr(ws),
                                           ws.numel() * ws.element_size(), _ptr(status),
                                           _stream(stream))
    _check(code, "gptq_quantize_layer_grouped")
    return codes, scales_out, g_idx, status


def gptq_pack_codes(codes, bits, words=None, stream=None):
    """codes uint8 [N][K] -> words int32 [N][ceil(K bits / 32)] holding the uint32 bit
    patterns of include/gptq.h's layout (view them with .view(torch.uint32))."""
    lib = load_library()
    N, K = codes.shape
    nw = (K * bits + 31) // 32
    if words is None:
        words = torch.empty(N, nw, dtype=torch.int32, device=codes.device)
    _check(lib.gptq_pack_codes(_ptr(codes), N, K, codes.stride(0), bits, _ptr(words),
                               words.stride(0), _stream(stream)), "gptq_pack_codes")
    return words


def gptq_unpack_codes(words, bits, K, codes=None, stream=None):
    """The inverse of gptq_pack_codes: words [N][>= ceil(K bits / 32)] -> uint8 [N][K]."""
    lib = load_library()
    N = words.shape[0]
    if codes is None:
        codes = torch.empty(N, K, dtype=torch.uint8, device=words.device)
    _check(lib.gptq_unpack_codes(_ptr(words), N, K, words.stride(0), bits, _ptr(codes),
                                 codes.stride(0), _stream(stream)), "gptq_unpack_codes")
    return codes


def gptq_first_order_shift(W, U, G, beta, gamma=None, workspace=None, status=None, stream=None):
    """W (fp32 [N][K]) <- W - beta G H^-1 in place; gamma (float64 [1]) gets
    sum_n g_n H^-1 g_n^T when given. Returns status; see include/gptq.h."""
    lib = load_library()
    if W.dtype != torch.float32:
        raise TypeError("gptq_first_order_shift shifts an fp32 copy of the weights")
    N, K = W.shape
    status = new_status(W.device) if status is None else status
    ws = _workspace(gptq_workspace_size(GPTQ_OP_FIRST_ORDER, K, N, 1, 0), W.device, workspace)
    code = lib.gptq_first_order_shift(_ptr(W), N, K, _ptr(U), _ptr(G), _dtype_code(G),
                                      ctypes.c_float(beta), _ptr(gamma), _ptr(ws),
                                      ws.numel() * ws.element_size(), _ptr(status),
                                      _stream(stream))
    _check(code, "gptq_first_order_shift")
    return status


def gptq_trust_region_beta(alpha, loss_gptq, gamma):
    """Host: the largest beta in [0, 1] with (beta - beta^2/2) gamma <= alpha loss_gptq."""
    return float(load_library().gptq_trust_region_beta(ctypes.c_float(alpha),
                                                        ctypes.c_double(loss_gptq),
                                                        ctypes.c_double(gamma)))


def gptq_selftest_timeout(status=None, stream=None):
    """Run the library's bounded-wait failure path once (about a second): the returned
    status word ends up holding GPTQ_ERR_TIMEOUT; see include/gptq.h."""
    lib = load_library()
    dev = torch.device("cuda", torch.cuda.current_device())
    status = new_status(dev) if status is None else status
    _check(lib.gptq_selftest_timeout(_ptr(status), _stream(stream)), "gptq_selftest_timeout")
    return status
