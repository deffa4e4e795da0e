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
# GPTQ_LIBRARY selects another build of the library (the index-checking
# libgptq_dbg.so of `build --debug-bounds`); by default the package's libgptq.so
LIB_PATH = os.environ.get("GPTQ_LIBRARY") or os.path.join(_HERE, "libgptq.so")

GPTQ_OK, GPTQ_ERR_ARG, GPTQ_ERR_NOT_PD, GPTQ_ERR_NONFINITE = 0, 1, 2, 3
GPTQ_ERR_CUDA, GPTQ_ERR_TIMEOUT, GPTQ_ERR_WORKSPACE, GPTQ_ERR_BOUNDS = 4, 5, 6, 7
GPTQ_BF16, GPTQ_F32 = 0, 1
GPTQ_OP_PREPARE, GPTQ_OP_RESIDUAL, GPTQ_OP_QUANTIZE, GPTQ_OP_QUANTIZE_GROUPED = 0, 1, 2, 3
GPTQ_OP_FIRST_ORDER = 4
GPTQ_WS_CAE = 0x100
GPTQ_PROF_SWEEP, GPTQ_PROF_UPDATE, GPTQ_PROF_DIAG, GPTQ_PROF_TC32, GPTQ_PROF_SPLIT = 0, 1, 2, 3, 4

EXPORTS = ("gptq_accumulate_hessian", "gptaq_accumulate_cross", "gptq_prepare",
           "gptq_prepare_noalloc",
           "gptaq_residual", "gptq_quantize_layer", "gptq_act_order", "gptq_permute_hessian",
           "gptq_quantize_layer_grouped", "gptq_pack_codes", "gptq_unpack_codes",
           "gptq_first_order_shift", "gptq_trust_region_beta", "gptq_selftest_timeout",
           "gptq_workspace_size",
           "gptq_kernel_launches", "gptq_status_string", "gptq_profile_enable",
           "gptq_profile_read", "gptq_profile_timeline", "gptq_chain_latency",
           "gptq_bounds_report", "gptq_bounds_selftest")

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
        "gptq_profile_enable": [I],
        "gptq_profile_read": [I, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int)],
        "gptq_bounds_report": [ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int),
                               ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int64), I],
        "gptq_bounds_selftest": [P, P],
        "gptq_profile_timeline": [I, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int),
                                  ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double),
                                  ctypes.POINTER(ctypes.c_int)],
        "gptq_chain_latency": [P, I, P],
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


def _device(t, name):
    """The CUDA device of the call's main tensor (every other tensor must be on it)."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor"
                         + (f" (got {t.device})" if isinstance(t, torch.Tensor) else ""))
    return t.device


def _ptr(t, dev=None, name="tensor", rows=False):
    """Device pointer of `t` for the C ABI, after the layout checks the ABI relies on:
    a CUDA tensor on the call's device, dense (or, with rows=True, rows that may be
    padded but whose elements are contiguous). A host pointer would reach the kernels
    otherwise."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor"
                         + (f" (got {t.device})" if isinstance(t, torch.Tensor) else ""))
    if dev is not None and t.device != dev:
        raise ValueError(f"{name} is on {t.device}, the call runs on {dev}")
    _check_layout(t, name, rows)
    return ctypes.c_void_p(t.data_ptr())


def _check_layout(t, name, rows=False):
    """Dense, or (rows=True) contiguous within each row with any row pitch."""
    if rows:
        if t.dim() >= 1 and t.numel() > 1 and t.shape[-1] > 1 and t.stride(-1) != 1:
            raise ValueError(f"{name}: the elements of a row must be contiguous")
    elif not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _stream(stream, dev=None):
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    elif dev is not None and stream.device != dev:
        raise ValueError(f"the stream is on {stream.device}, the call runs on {dev}")
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
    dev = _device(H, "H")
    K = H.shape[-1]
    g = 1 if H.dim() == 2 else H.shape[0]
    M = X.shape[0]
    ldw = 0 if w is None else w.stride(0) if w.dim() == 2 else w.shape[-1]
    args = (_ptr(H, dev, "H"), K, g, _ptr(X, dev, "X", rows=True), _dtype_code(X), M,
            X.stride(0), _ptr(w, dev, "w", rows=True), ldw, _ptr(status, dev, "status"),
            _stream(stream, dev))
    with torch.cuda.device(dev):
        code = lib.gptq_accumulate_hessian(*args)
    _check(code, "gptq_accumulate_hessian")


def gptaq_accumulate_cross(C, X_fp, X_q, status=None, stream=None):
    """C += 2 (X_fp - X_q)^T X_q (see include/gptq.h)."""
    lib = load_library()
    if X_fp.stride(0) != X_q.stride(0) or X_fp.dtype != X_q.dtype or X_fp.shape != X_q.shape:
        raise ValueError("X_fp and X_q must share shape, dtype and row stride")
    dev = _device(C, "C")
    args = (_ptr(C, dev, "C"), C.shape[-1], _ptr(X_fp, dev, "X_fp", rows=True),
            _ptr(X_q, dev, "X_q", rows=True), _dtype_code(X_q), X_q.shape[0], X_q.stride(0),
            _ptr(status, dev, "status"), _stream(stream, dev))
    with torch.cuda.device(dev):
        code = lib.gptaq_accumulate_cross(*args)
    _check(code, "gptaq_accumulate_cross")


def gptq_prepare(H, percdamp=0.01, dead_out=None, workspace=None, status=None, stream=None):
    """In place: dead fix, damping, H -> U. Returns the status tensor (not synchronised)."""
    lib = load_library()
    dev = _device(H, "H")
    K = H.shape[-1]
    g = 1 if H.dim() == 2 else H.shape[0]
    status = new_status(dev) if status is None else status
    ws = _workspace(gptq_workspace_size(GPTQ_OP_PREPARE, K, 0, g, 0), dev, workspace)
    args = (_ptr(H, dev, "H"), K, g, float(percdamp), _ptr(dead_out, dev, "dead_out"),
            _ptr(ws, dev, "workspace"), ws.numel() * ws.element_size(),
            _ptr(status, dev, "status"), _stream(stream, dev))
    with torch.cuda.device(dev):
        code = lib.gptq_prepare(*args)
    _check(code, "gptq_prepare")
    return status


def gptq_prepare_noalloc(H, percdamp=0.01, dead_out=None, status=None, stream=None):
    """gptq_prepare with the library's fixed device scratch instead of a workspace
    (no allocation anywhere on this path). Returns the status tensor."""
    lib = load_library()
    dev = _device(H, "H")
    K = H.shape[-1]
    g = 1 if H.dim() == 2 else H.shape[0]
    if status is None:
        raise ValueError("gptq_prepare_noalloc needs a caller-provided status word")
    args = (_ptr(H, dev, "H"), K, g, float(percdamp), _ptr(dead_out, dev, "dead_out"),
            _ptr(status, dev, "status"), _stream(stream, dev))
    with torch.cuda.device(dev):
        code = lib.gptq_prepare_noalloc(*args)
    _check(code, "gptq_prepare_noalloc")
    return status


def gptaq_residual(P1, C, U, workspace=None, stream=None):
    """P1 = [(C U^T) ⊙ strict-upper] U (see include/gptq.h)."""
    lib = load_library()
    dev = _device(U, "U")
    K = U.shape[-1]
    ws = _workspace(gptq_workspace_size(GPTQ_OP_RESIDUAL, K, 0, 1, 0), dev, workspace)
    args = (_ptr(P1, dev, "P1"), _ptr(C, dev, "C"), _ptr(U, dev, "U"), K,
            _ptr(ws, dev, "workspace"), ws.numel() * ws.element_size(), _stream(stream, dev))
    with torch.cuda.device(dev):
        code = lib.gptaq_residual(*args)
    _check(code, "gptaq_residual")


def gptq_quantize_layer(W, U, bits, blocksize=128, groups=1, P1=None, dead=None, scales_in=None,
                        scales_out=None, codes=None, loss=None, write_back=False,
                        workspace=None, status=None, stream=None, cae=False):
    """The shared-order sweep (cae: with the compensation-aware error term).
    Returns (codes, status); see include/gptq.h."""
    lib = load_library()
    dev = _device(W, "W")
    N, K = W.shape
    if codes is None:
        codes = torch.empty(N, K, dtype=torch.uint8, device=dev)
    status = new_status(dev) if status is None else status
    op = GPTQ_OP_QUANTIZE | (GPTQ_WS_CAE if cae else 0)
    ws = _workspace(gptq_workspace_size(op, K, N, groups, blocksize), dev, workspace)
    args = (_ptr(W, dev, "W"), _dtype_code(W), N, K, _ptr(U, dev, "U"), groups, bits, blocksize,
            _ptr(P1, dev, "P1"), int(bool(cae)), _ptr(dead, dev, "dead"),
            _ptr(scales_in, dev, "scales_in"), _ptr(scales_out, dev, "scales_out"),
            _ptr(codes, dev, "codes"), _ptr(loss, dev, "loss"), int(write_back),
            _ptr(ws, dev, "workspace"), ws.numel() * ws.element_size(),
            _ptr(status, dev, "status"), _stream(stream, dev))
    with torch.cuda.device(dev):
        code = lib.gptq_quantize_layer(*args)
    _check(code, "gptq_quantize_layer")
    return codes, status


def gptq_act_order(H, perm=None, stream=None):
    """The act-order processing order of H's input coordinates (int32 [K])."""
    lib = load_library()
    dev = _device(H, "H")
    K = H.shape[-1]
    if perm is None:
        perm = torch.empty(K, dtype=torch.int32, device=dev)
    args = (_ptr(H, dev, "H"), K, _ptr(perm, dev, "perm"), _stream(stream, dev))
    with torch.cuda.device(dev):
        code = lib.gptq_act_order(*args)
    _check(code, "gptq_act_order")
    return perm


def gptq_permute_hessian(H, perm, out=None, stream=None):
    """out = H[perm][:, perm] (a new K x K tensor unless `out` is given)."""
    lib = load_library()
    dev = _device(H, "H")
    K = H.shape[-1]
    if out is None:
        out = torch.empty_like(H, memory_format=torch.contiguous_format)
    args = (_ptr(out, dev, "out"), _ptr(H, dev, "H"), K, _ptr(perm, dev, "perm"),
            _stream(stream, dev))
    with torch.cuda.device(dev):
        code = lib.gptq_permute_hessian(*args)
    _check(code, "gptq_permute_hessian")
    return out


def gptq_quantize_layer_grouped(W, U, bits, blocksize=128, groupsize=128, static_groups=False,
                                perm=None, P1=None, dead=None, scales_out=None, g_idx=None,
                                codes=None, loss=None, write_back=False, workspace=None,
                                status=None, stream=None, cae=False):
    """The sweep with input-dimension groups and an optional processing order.
    Returns (codes, scales [N][ceil(K / groupsize)], g_idx [K], status); see include/gptq.h."""
    lib = load_library()
    dev = _device(W, "W")
    N, K = W.shape
    if codes is None:
        codes = torch.empty(N, K, dtype=torch.uint8, device=dev)
    if scales_out is None:
        shape = (N, (K + groupsize - 1) // groupsize) if groupsize else (N,)
        scales_out = torch.empty(shape, dtype=torch.float32, device=dev)
    if g_idx is None:
        g_idx = torch.empty(K, dtype=torch.int32, device=dev)
    status = new_status(dev) if status is None else status
    op = GPTQ_OP_QUANTIZE_GROUPED | (GPTQ_WS_CAE if cae else 0)
    ws = _workspace(gptq_workspace_size(op, K, N, 1, blocksize), dev, workspace)
    args = (_ptr(W, dev, "W"), _dtype_code(W), N, K, _ptr(U, dev, "U"), bits, blocksize,
            groupsize, int(bool(static_groups)), _ptr(perm, dev, "perm"), _ptr(P1, dev, "P1"),
            int(bool(cae)), _ptr(dead, dev, "dead"), _ptr(scales_out, dev, "scales_out"),
            _ptr(g_idx, dev, "g_idx"), _ptr(codes, dev, "codes"), _ptr(loss, dev, "loss"),
            int(write_back), _ptr(ws, dev, "workspace"), ws.numel() * ws.element_size(),
            _ptr(status, dev, "status"), _stream(stream, dev))
    with torch.cuda.device(dev):
        code = lib.gptq_quantize_layer_grouped(*args)
    _check(code, "gptq_quantize_layer_grouped")
    return codes, scales_out, g_idx, status


def gptq_pack_codes(codes, bits, words=None, stream=None):
    """codes uint8 [N][K] -> words int32 [N][ceil(K bits / 32)] holding the uint32 bit
    patterns of include/gptq.h's layout (view them with .view(torch.uint32))."""
    lib = load_library()
    dev = _device(codes, "codes")
    N, K = codes.shape
    nw = (K * bits + 31) // 32
    if words is None:
        words = torch.empty(N, nw, dtype=torch.int32, device=dev)
    args = (_ptr(codes, dev, "codes", rows=True), N, K, codes.stride(0), bits,
            _ptr(words, dev, "words", rows=True), words.stride(0), _stream(stream, dev))
    with torch.cuda.device(dev):
        code = lib.gptq_pack_codes(*args)
    _check(code, "gptq_pack_codes")
    return words


def gptq_unpack_codes(words, bits, K, codes=None, stream=None):
    """The inverse of gptq_pack_codes: words [N][>= ceil(K bits / 32)] -> uint8 [N][K]."""
    lib = load_library()
    dev = _device(words, "words")
    N = words.shape[0]
    if codes is None:
        codes = torch.empty(N, K, dtype=torch.uint8, device=dev)
    args = (_ptr(words, dev, "words", rows=True), N, K, words.stride(0), bits,
            _ptr(codes, dev, "codes", rows=True), codes.stride(0), _stream(stream, dev))
    with torch.cuda.device(dev):
        code = lib.gptq_unpack_codes(*args)
    _check(code, "gptq_unpack_codes")
    return codes


def gptq_first_order_shift(W, U, G, beta, gamma=None, workspace=None, status=None, stream=None):
    """W (fp32 [N][K]) <- W - beta G H^-1 in place; gamma (float64 [1]) gets
    sum_n g_n H^-1 g_n^T when given. Returns status; see include/gptq.h."""
    lib = load_library()
    dev = _device(W, "W")
    if W.dtype != torch.float32:
        raise TypeError("gptq_first_order_shift shifts an fp32 copy of the weights")
    N, K = W.shape
    status = new_status(dev) if status is None else status
    ws = _workspace(gptq_workspace_size(GPTQ_OP_FIRST_ORDER, K, N, 1, 0), dev, workspace)
    args = (_ptr(W, dev, "W"), N, K, _ptr(U, dev, "U"), _ptr(G, dev, "G"), _dtype_code(G),
            ctypes.c_float(beta), _ptr(gamma, dev, "gamma"), _ptr(ws, dev, "workspace"),
            ws.numel() * ws.element_size(), _ptr(status, dev, "status"), _stream(stream, dev))
    with torch.cuda.device(dev):
        code = lib.gptq_first_order_shift(*args)
    _check(code, "gptq_first_order_shift")
    return status


def gptq_trust_region_beta(alpha, loss_gptq, gamma):
    """Host: the largest beta in [0, 1] with (beta - beta^2/2) gamma <= alpha loss_gptq."""
    return float(load_library().gptq_trust_region_beta(ctypes.c_float(alpha),
                                                        ctypes.c_double(loss_gptq),
                                                        ctypes.c_double(gamma)))


def gptq_profile_enable(on):
    """Start (True) or stop (False) a kernel-timing window (see include/gptq.h)."""
    _check(load_library().gptq_profile_enable(1 if on else 0), "gptq_profile_enable")


def gptq_profile_read(kind):
    """(summed ms, launches) of one kernel class in the current timing window."""
    ms, n = ctypes.c_double(0.0), ctypes.c_int(0)
    _check(load_library().gptq_profile_read(int(kind), ctypes.byref(ms), ctypes.byref(n)),
           "gptq_profile_read")
    return ms.value, n.value


def gptq_profile_timeline(max_records=4096):
    """The timing window's records in launch order: a list of (kind, lane, begin_ms,
    end_ms), lane numbering the streams in order of first use, times from the first
    record's begin (see include/gptq.h)."""
    n = max(0, int(max_records))
    kind, lane = (ctypes.c_int * max(n, 1))(), (ctypes.c_int * max(n, 1))()
    t0, t1 = (ctypes.c_double * max(n, 1))(), (ctypes.c_double * max(n, 1))()
    count = ctypes.c_int(0)
    _check(load_library().gptq_profile_timeline(n, kind, lane, t0, t1, ctypes.byref(count)),
           "gptq_profile_timeline")
    return [(kind[i], lane[i], t0[i], t1[i]) for i in range(min(n, count.value))]


def gptq_chain_latency(out, steps=65536, stream=None):
    """One thread times `steps` steps of the sweep's dependent chain: out (3 float32 on
    the device) receives SM cycles per step, ns per step and a keep-alive value. Returns
    `out` (not synchronised)."""
    lib = load_library()
    dev = _device(out, "out")
    args = (_ptr(out, dev, "out"), int(steps), _stream(stream, dev))
    with torch.cuda.device(dev):
        code = lib.gptq_chain_latency(*args)
    _check(code, "gptq_chain_latency")
    return out


def gptq_bounds_report(reset=False):
    """Records of the index-checking build: (enabled, failed checks, first site, first
    index); enabled is False for the normal build (see include/gptq.h)."""
    en, cnt, site = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    idx = ctypes.c_int64(0)
    _check(load_library().gptq_bounds_report(ctypes.byref(en), ctypes.byref(cnt), ctypes.byref(site),
                                             ctypes.byref(idx), 1 if reset else 0),
           "gptq_bounds_report")
    return bool(en.value), cnt.value, site.value, idx.value


def gptq_bounds_selftest(status=None, stream=None):
    """Index-checking build only: one check that always fails (no access), so the
    returned status word ends up holding GPTQ_ERR_BOUNDS."""
    lib = load_library()
    dev = status.device if status is not None else torch.device("cuda", torch.cuda.current_device())
    status = new_status(dev) if status is None else status
    args = (_ptr(status, dev, "status"), _stream(stream, dev))
    with torch.cuda.device(dev):
        code = lib.gptq_bounds_selftest(*args)
    _check(code, "gptq_bounds_selftest")
    return status


def gptq_selftest_timeout(status=None, stream=None):
    """Run the library's bounded-wait failure path once (about a second): the returned
    status word ends up holding GPTQ_ERR_TIMEOUT; see include/gptq.h."""
    lib = load_library()
    dev = status.device if status is not None else torch.device("cuda", torch.cuda.current_device())
    status = new_status(dev) if status is None else status
    args = (_ptr(status, dev, "status"), _stream(stream, dev))
    with torch.cuda.device(dev):
        code = lib.gptq_selftest_timeout(*args)
    _check(code, "gptq_selftest_timeout")
    return status
