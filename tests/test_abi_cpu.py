"""The C-ABI library loads on a machine without a GPU, exports every entry point
that include/gptq.h declares, and rejects bad arguments on the host before any
device work (no compute call is made here)."""

import ctypes
import os
import re

import pytest
import torch

import post_weight_quantization_solve_b200 as gq
from post_weight_quantization_solve_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return gq.load_library()


def header_entry_points():
    text = open(os.path.join(ROOT, "include", "gptq.h"), encoding="utf-8").read()
    return re.findall(r"GPTQ_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


def test_exports_every_declared_symbol(lib):
    names = header_entry_points()
    assert set(names) == set(gq.EXPORTS)
    for name in names:
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code in range(8):
        assert gq.gptq_status_string(code) not in ("", "unknown status")
    assert gq.gptq_status_string(99) == "unknown status"


def test_workspace_sizes(lib):
    p1 = gq.gptq_workspace_size(gq.GPTQ_OP_PREPARE, 4096, 0, 1, 0)
    p4 = gq.gptq_workspace_size(gq.GPTQ_OP_PREPARE, 4096, 0, 4, 0)
    assert p1 > 4096 * 4 and p4 > p1
    q = gq.gptq_workspace_size(gq.GPTQ_OP_QUANTIZE, 4096, 14336, 1, 128)
    assert q >= 4096 * 14336 * 4
    assert gq.gptq_workspace_size(gq.GPTQ_OP_RESIDUAL, 512, 0, 1, 0) >= 512 * 512 * 4
    assert gq.gptq_workspace_size(7, 128, 1, 1, 1) == 0
    # the compensation-aware term adds one fp32 copy of W; the flag fits only the sweeps
    qc = gq.gptq_workspace_size(gq.GPTQ_OP_QUANTIZE | gq.GPTQ_WS_CAE, 4096, 14336, 1, 128)
    assert qc >= q + 4096 * 14336 * 4
    qg = gq.gptq_workspace_size(gq.GPTQ_OP_QUANTIZE_GROUPED, 4096, 14336, 1, 128)
    assert gq.gptq_workspace_size(gq.GPTQ_OP_QUANTIZE_GROUPED | gq.GPTQ_WS_CAE, 4096, 14336, 1,
                                  128) >= qg + 4096 * 14336 * 4
    assert gq.gptq_workspace_size(gq.GPTQ_OP_PREPARE | gq.GPTQ_WS_CAE, 4096, 0, 1, 0) == 0
    assert gq.gptq_workspace_size(gq.GPTQ_OP_PREPARE, 0, 0, 1, 0) == 0


def test_host_argument_checks(lib):
    P = ctypes.c_void_p
    fake = P(1 << 20)   # never dereferenced: every call below fails its host checks
    ws = P(1 << 21)
    # quantize: bits, blocksize, groups, NULL pointers, GPTAQ with groups
    assert lib.gptq_quantize_layer(fake, 0, 8, 16, fake, 1, 5, 128, None, 0, None, None, None,
                                   fake, None, 0, ws, 1 << 30, fake, None) == gq.GPTQ_ERR_ARG
    assert lib.gptq_quantize_layer(fake, 0, 8, 16, fake, 1, 4, 256, None, 0, None, None, None,
                                   fake, None, 0, ws, 1 << 30, fake, None) == gq.GPTQ_ERR_ARG
    assert lib.gptq_quantize_layer(fake, 0, 9, 16, fake, 2, 4, 128, None, 0, None, None, None,
                                   fake, None, 0, ws, 1 << 30, fake, None) == gq.GPTQ_ERR_ARG
    assert lib.gptq_quantize_layer(fake, 0, 8, 16, fake, 2, 4, 128, fake, 0, None, None, None,
                                   fake, None, 0, ws, 1 << 30, fake, None) == gq.GPTQ_ERR_ARG
    assert lib.gptq_quantize_layer(fake, 0, 8, 16, fake, 1, 4, 128, None, 0, None, None, None,
                                   None, None, 0, ws, 1 << 30, fake, None) == gq.GPTQ_ERR_ARG
    assert lib.gptq_quantize_layer(fake, 0, 8, 16, fake, 1, 4, 128, None, 0, None, None, None,
                                   fake, None, 0, ws, 16, fake, None) == gq.GPTQ_ERR_WORKSPACE
    assert lib.gptq_quantize_layer(fake, 0, 8, 16, fake, 1, 4, 128, None, 0, None, None, None,
                                   fake, None, 0, P((1 << 21) + 8), 1 << 30, fake,
                                   None) == gq.GPTQ_ERR_WORKSPACE
    # cae: only 0 or 1, and its workspace includes the copy of W
    assert lib.gptq_quantize_layer(fake, 0, 8, 16, fake, 1, 4, 128, None, 2, None, None, None,
                                   fake, None, 0, ws, 1 << 30, fake, None) == gq.GPTQ_ERR_ARG
    plain = gq.gptq_workspace_size(gq.GPTQ_OP_QUANTIZE, 16, 8, 1, 128)
    assert lib.gptq_quantize_layer(fake, 0, 8, 16, fake, 1, 4, 128, None, 1, None, None, None,
                                   fake, None, 0, ws, plain, fake, None) == gq.GPTQ_ERR_WORKSPACE
    assert lib.gptq_quantize_layer_grouped(fake, 0, 8, 16, fake, 4, 128, 32, 0, None, None, 3,
                                           None, None, None, fake, None, 0, ws, 1 << 30, fake,
                                           None) == gq.GPTQ_ERR_ARG
    # timing diagnostics: an empty window reads zero; bad kinds and chain lengths refused
    assert lib.gptq_profile_enable(1) == gq.GPTQ_OK
    ms, cnt = ctypes.c_double(-1.0), ctypes.c_int(-1)
    assert lib.gptq_profile_read(gq.GPTQ_PROF_UPDATE, ctypes.byref(ms), ctypes.byref(cnt)) == gq.GPTQ_OK
    assert ms.value == 0.0 and cnt.value == 0
    assert lib.gptq_profile_read(5, ctypes.byref(ms), ctypes.byref(cnt)) == gq.GPTQ_ERR_ARG
    assert lib.gptq_profile_read(0, None, ctypes.byref(cnt)) == gq.GPTQ_ERR_ARG
    ki, la = (ctypes.c_int * 2)(), (ctypes.c_int * 2)()
    t0, t1 = (ctypes.c_double * 2)(), (ctypes.c_double * 2)()
    assert lib.gptq_profile_timeline(2, ki, la, t0, t1, ctypes.byref(cnt)) == gq.GPTQ_OK
    assert cnt.value == 0
    assert lib.gptq_profile_timeline(-1, ki, la, t0, t1, ctypes.byref(cnt)) == gq.GPTQ_ERR_ARG
    assert lib.gptq_profile_timeline(2, ki, la, t0, None, ctypes.byref(cnt)) == gq.GPTQ_ERR_ARG
    assert lib.gptq_profile_enable(0) == gq.GPTQ_OK
    assert lib.gptq_chain_latency(fake, 12, None) == gq.GPTQ_ERR_ARG
    # index-check records: the normal build has none and no self-test
    en, cnt, site, idx = ctypes.c_int(-1), ctypes.c_int(-1), ctypes.c_int(-1), ctypes.c_int64(-1)
    assert lib.gptq_bounds_report(ctypes.byref(en), ctypes.byref(cnt), ctypes.byref(site),
                                  ctypes.byref(idx), 1) == gq.GPTQ_OK
    assert (en.value, cnt.value, site.value, idx.value) == (0, 0, 0, 0)
    assert lib.gptq_bounds_report(None, ctypes.byref(cnt), ctypes.byref(site), ctypes.byref(idx),
                                  0) == gq.GPTQ_ERR_ARG
    assert lib.gptq_bounds_selftest(fake, None) == gq.GPTQ_ERR_ARG
    assert lib.gptq_bounds_selftest(None, None) == gq.GPTQ_ERR_ARG
    assert lib.gptq_chain_latency(None, 64, None) == gq.GPTQ_ERR_ARG
    # pack / unpack: bits, strides, NULL pointers; N == 0 does nothing
    assert lib.gptq_pack_codes(fake, 4, 64, 64, 5, fake, 64, None) == gq.GPTQ_ERR_ARG
    assert lib.gptq_pack_codes(fake, 4, 64, 63, 4, fake, 8, None) == gq.GPTQ_ERR_ARG
    assert lib.gptq_pack_codes(fake, 4, 64, 64, 3, fake, 5, None) == gq.GPTQ_ERR_ARG
    assert lib.gptq_pack_codes(None, 4, 64, 64, 3, fake, 6, None) == gq.GPTQ_ERR_ARG
    assert lib.gptq_unpack_codes(fake, 4, 64, 1, 2, fake, 64, None) == gq.GPTQ_ERR_ARG
    assert lib.gptq_pack_codes(fake, 0, 64, 64, 3, fake, 6, None) == gq.GPTQ_OK
    assert lib.gptq_unpack_codes(fake, 0, 64, 6, 3, fake, 64, None) == gq.GPTQ_OK
    # first-order shift: beta in [0, 1], dtype, workspace
    assert lib.gptq_first_order_shift(fake, 8, 16, fake, fake, 0, ctypes.c_float(1.5), None, ws,
                                      1 << 30, fake, None) == gq.GPTQ_ERR_ARG
    assert lib.gptq_first_order_shift(fake, 8, 16, fake, fake, 7, ctypes.c_float(0.5), None, ws,
                                      1 << 30, fake, None) == gq.GPTQ_ERR_ARG
    assert lib.gptq_first_order_shift(fake, 8, 16, fake, fake, 0, ctypes.c_float(0.5), None, ws,
                                      64, fake, None) == gq.GPTQ_ERR_WORKSPACE
    # prepare: negative damping, missing status, small workspace
    assert lib.gptq_prepare(fake, 16, 1, ctypes.c_float(-0.1), None, ws, 1 << 30, fake,
                            None) == gq.GPTQ_ERR_ARG
    assert lib.gptq_prepare(fake, 16, 1, ctypes.c_float(0.01), None, ws, 1 << 30, None,
                            None) == gq.GPTQ_ERR_ARG
    assert lib.gptq_prepare(fake, 4096, 1, ctypes.c_float(0.01), None, ws, 64, fake,
                            None) == gq.GPTQ_ERR_WORKSPACE
    # Hessian: bf16 needs K % 8 == 0 and 16-byte aligned rows; g > 1 needs weights
    assert lib.gptq_accumulate_hessian(fake, 12, 1, fake, gq.GPTQ_BF16, 10, 12, None, 0,
                                       None, None) == gq.GPTQ_ERR_ARG
    assert lib.gptq_accumulate_hessian(fake, 16, 1, fake, gq.GPTQ_BF16, 10, 20, None, 0,
                                       None, None) == gq.GPTQ_ERR_ARG
    assert lib.gptq_accumulate_hessian(fake, 16, 2, fake, gq.GPTQ_BF16, 10, 16, None, 0,
                                       None, None) == gq.GPTQ_ERR_ARG
    assert lib.gptq_accumulate_hessian(fake, 16, 1, fake, 7, 10, 16, None, 0,
                                       None, None) == gq.GPTQ_ERR_ARG
    # M == 0 is a no-op that succeeds without touching the device
    assert lib.gptq_accumulate_hessian(fake, 16, 1, fake, gq.GPTQ_BF16, 0, 16, None, 0,
                                       None, None) == gq.GPTQ_OK
    assert lib.gptaq_accumulate_cross(fake, 16, fake, fake, gq.GPTQ_BF16, 0, 16,
                                      None, None) == gq.GPTQ_OK
    assert lib.gptaq_residual(fake, fake, fake, 16, ws, 8, None) == gq.GPTQ_ERR_WORKSPACE


def test_checking_build_exports_the_same_entry_points(lib):
    # the GPTQ_DEBUG_BOUNDS variant builds and loads beside the normal library, with the
    # same C ABI (it differs only inside the kernels)
    from post_weight_quantization_solve_b200.build import LIB_DBG

    dbg = ctypes.CDLL(build(debug_bounds=True))
    assert os.path.samefile(LIB_DBG, dbg._name)
    for name in header_entry_points():
        assert hasattr(dbg, name), name


def test_product_path_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(gq, "_lib", None)
    monkeypatch.setattr(gq, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        gq.load_library()


def test_trust_region_beta_matches_the_oracle(lib):
    import oracle as O
    for alpha, lq, gamma in ((0.1, 0.3, 2.0), (2.0, 1.0, 1.0), (0.0, 1.0, 5.0), (1.0, 1.0, 0.0),
                             (0.7, 1e-3, 40.0)):
        assert gq.gptq_trust_region_beta(alpha, lq, gamma) == pytest.approx(
            O.trust_region_beta(alpha, lq, gamma), rel=1e-6, abs=1e-7)


C_CONSUMER = r"""
#include <stdio.h>
#include <string.h>
#include "gptq.h"

int main(void) {
    void *fake = (void *)(size_t)(1u << 20);
    int32_t *status = (int32_t *)fake;
    size_t ws = gptq_workspace_size(GPTQ_OP_QUANTIZE, 4096, 14336, 1, 128);
    size_t wsc = gptq_workspace_size(GPTQ_OP_QUANTIZE | GPTQ_WS_CAE, 4096, 14336, 1, 128);
    gptq_status bad_bits = gptq_quantize_layer(fake, GPTQ_BF16, 8, 16, (const float *)fake, 1, 5,
                                               128, NULL, 0, NULL, NULL, NULL, (uint8_t *)fake,
                                               NULL, 0, fake, (size_t)1 << 30, status, NULL);
    gptq_status empty = gptq_pack_codes((const uint8_t *)fake, 0, 64, 64, 3, (uint32_t *)fake,
                                        6, NULL);
    float beta = gptq_trust_region_beta(2.0f, 1.0f, 1.0f);
    printf("%zu %zu %d %d %.6f %s\n", ws, wsc, (int)bad_bits, (int)empty, beta,
           gptq_status_string(GPTQ_ERR_NOT_PD));
    return 0;
}
"""


def test_header_is_plain_c_and_the_library_links(lib, tmp_path):
    # a C99 consumer: the header compiles as C with warnings as errors, the program links
    # against the in-tree library and makes host-only calls through the ABI
    src = tmp_path / "consumer.c"
    src.write_text(C_CONSUMER)
    exe = tmp_path / "consumer"
    libdir = os.path.dirname(gq.LIB_PATH)
    import subprocess
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                         "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                         "-L", libdir, "-l:" + os.path.basename(gq.LIB_PATH),
                         "-Wl,-rpath," + libdir], capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stderr
    ws, wsc, bad_bits, empty, beta, *msg = run.stdout.split()
    assert int(ws) == gq.gptq_workspace_size(gq.GPTQ_OP_QUANTIZE, 4096, 14336, 1, 128)
    assert int(wsc) >= int(ws) + 4096 * 14336 * 4
    assert int(bad_bits) == gq.GPTQ_ERR_ARG and int(empty) == gq.GPTQ_OK
    assert float(beta) == pytest.approx(gq.gptq_trust_region_beta(2.0, 1.0, 1.0), rel=1e-6)
    assert " ".join(msg) == gq.gptq_status_string(gq.GPTQ_ERR_NOT_PD)


def test_binding_refuses_host_tensors(lib):
    # a host pointer must never reach a kernel: every call checks its tensors first
    W = torch.zeros(8, 16)
    H = torch.eye(16)
    X = torch.zeros(32, 16, dtype=torch.bfloat16)
    codes = torch.zeros(8, 16, dtype=torch.uint8)
    calls = [
        lambda: gq.gptq_accumulate_hessian(H, X),
        lambda: gq.gptaq_accumulate_cross(H, X, X),
        lambda: gq.gptq_prepare(H),
        lambda: gq.gptq_prepare_noalloc(H, status=torch.zeros(1, dtype=torch.int32)),
        lambda: gq.gptaq_residual(H, H, H),
        lambda: gq.gptq_quantize_layer(W, H, 4, 16),
        lambda: gq.gptq_act_order(H),
        lambda: gq.gptq_permute_hessian(H, torch.arange(16, dtype=torch.int32)),
        lambda: gq.gptq_quantize_layer_grouped(W, H, 4, 16, 16),
        lambda: gq.gptq_pack_codes(codes, 4),
        lambda: gq.gptq_unpack_codes(torch.zeros(8, 2, dtype=torch.int32), 4, 16),
        lambda: gq.gptq_first_order_shift(W, H, W, 0.5),
    ]
    for call in calls:
        with pytest.raises(ValueError, match="must be a CUDA tensor"):
            call()


def test_binding_layout_rules():
    A = torch.zeros(6, 8)
    gq._check_layout(A, "A")
    gq._check_layout(A[1:4], "A")                      # a block of whole rows is dense
    with pytest.raises(ValueError, match="contiguous"):
        gq._check_layout(A[:, 1:5], "A")               # padded rows: not dense
    gq._check_layout(A[:, 1:5], "A", rows=True)        # but fine where a pitch is passed
    with pytest.raises(ValueError, match="row must be contiguous"):
        gq._check_layout(A.t(), "A", rows=True)        # a transposed view is refused
    with pytest.raises(ValueError, match="contiguous"):
        gq._check_layout(A.t(), "A")
    gq._check_layout(torch.zeros(0, 8).t(), "A", rows=True)
    gq._check_layout(torch.zeros(5, 1)[::2], "A", rows=True)


def test_every_wrapper_matches_its_c_signature(lib, monkeypatch):
    # each wrapper's argument list against the ctypes signature of its entry point: the
    # count, and every value convertible to its declared type (a fake library records the
    # calls; the device checks are bypassed so that host tensors stand in for device ones)
    import contextlib

    calls = {}

    class FakeLib:
        def __getattr__(self, name):
            real = getattr(lib, name)

            def fn(*args):
                assert len(args) == len(real.argtypes), (name, len(args), len(real.argtypes))
                for a, t in zip(args, real.argtypes):
                    t.from_param(a)
                calls[name] = args
                return 0
            return fn

    monkeypatch.setattr(gq, "_lib", FakeLib())
    monkeypatch.setattr(gq, "_device", lambda t, name: t.device)
    monkeypatch.setattr(gq, "_stream", lambda stream, dev=None: ctypes.c_void_p(0))

    def host_ptr(t, dev=None, name="tensor", rows=False):
        if t is None:
            return None
        gq._check_layout(t, name, rows)
        return ctypes.c_void_p(t.data_ptr())
    monkeypatch.setattr(gq, "_ptr", host_ptr)
    monkeypatch.setattr(torch.cuda, "device", lambda d: contextlib.nullcontext())
    real_ws = lib.gptq_workspace_size
    monkeypatch.setattr(gq, "gptq_workspace_size", lambda *a: int(real_ws(*a)))

    K, N = 32, 8
    H = torch.eye(K)
    W = torch.zeros(N, K)
    X = torch.zeros(64, K, dtype=torch.bfloat16)
    st = torch.zeros(1, dtype=torch.int32)
    gq.gptq_accumulate_hessian(H, X, status=st)
    gq.gptq_accumulate_hessian(torch.zeros(2, K, K), X, torch.ones(2, 64), status=st)
    gq.gptaq_accumulate_cross(H, X, X, status=st)
    gq.gptq_prepare(H, 0.01, dead_out=torch.zeros(K, dtype=torch.uint8), status=st)
    gq.gptq_prepare_noalloc(H, 0.01, status=st)
    gq.gptaq_residual(torch.zeros(K, K), H, H)
    gq.gptq_quantize_layer(W, H, 3, 16, P1=H, dead=torch.zeros(K, dtype=torch.uint8),
                           scales_out=torch.zeros(N), loss=torch.zeros(N), write_back=True,
                           status=st, cae=True)
    perm = gq.gptq_act_order(H)
    gq.gptq_permute_hessian(H, perm)
    gq.gptq_quantize_layer_grouped(W, H, 3, 16, 16, static_groups=True, perm=perm, P1=H,
                                   status=st, cae=True)
    words = gq.gptq_pack_codes(torch.zeros(N, K, dtype=torch.uint8), 3)
    gq.gptq_unpack_codes(words, 3, K)
    gq.gptq_first_order_shift(W, H, W, 0.5, gamma=torch.zeros(1, dtype=torch.float64),
                              status=st)
    gq.gptq_selftest_timeout(status=st)
    gq.gptq_chain_latency(torch.zeros(3), steps=64)
    gq.gptq_profile_enable(True)
    gq.gptq_profile_read(gq.GPTQ_PROF_SWEEP)
    gq.gptq_profile_timeline(8)
    gq.gptq_bounds_report(reset=True)
    gq.gptq_bounds_selftest(status=st)
    assert set(calls) == set(gq.EXPORTS) - {"gptq_trust_region_beta", "gptq_workspace_size",
                                            "gptq_kernel_launches", "gptq_status_string"}
    # the workspace sizes passed are the ones the library asks for
    assert calls["gptq_quantize_layer"][17] >= int(real_ws(gq.GPTQ_OP_QUANTIZE | gq.GPTQ_WS_CAE,
                                                           K, N, 1, 16))


@pytest.mark.parametrize("op", [0, 1, 2, 3, 4, 2 | 0x100, 3 | 0x100])
def test_workspace_sizes_grow_and_stay_aligned(lib, op):
    # sizes are multiples of 256 bytes, never shrink as the layer grows on the
    # tensor-core paths (K a multiple of 32; other K take the smaller SIMT workspaces),
    # and do not overflow at the largest such K the ABI accepts
    prev = 0
    for K in (128, 256, 1024, 4096, 14336, 28672, 65504):
        size = gq.gptq_workspace_size(op, K, 4096, 1, 128)
        assert size % 256 == 0, (op, K, size)
        assert size >= prev, (op, K, size, prev)
        prev = size
    assert prev >= 4 * 65504 * (65504 if op in (0, 1) else 4096)
    assert gq.gptq_workspace_size(op, 65535, 4096, 1, 128) % 256 == 0
    sizes_n = [gq.gptq_workspace_size(op, 4096, N, 1, 128) for N in (1, 100, 4096, 65535)]
    assert sizes_n == sorted(sizes_n)
    if op == 0:   # prepare: one more group never costs less
        assert gq.gptq_workspace_size(0, 4096, 0, 4, 0) > gq.gptq_workspace_size(0, 4096, 0, 2, 0)
