"""Packed code storage on the GPU vs the oracle's packing (bit for bit; C ABI calls)."""

import numpy as np
import pytest
import torch

import oracle as O
import post_weight_quantization_solve_b200 as gq
from post_weight_quantization_solve_b200.build import build

from gpu_util import dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    gq.load_library()


def _words(t):
    return t.cpu().numpy().view(np.uint32)


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("N,K", [(1, 1), (3, 31), (5, 33), (7, 200), (130, 1000)])
def test_pack_matches_oracle(bits, N, K):
    g = torch.Generator(device=dev()).manual_seed(bits * 1000 + K)
    codes = torch.randint(0, 2 ** bits, (N, K), generator=g, device=dev(), dtype=torch.uint8)
    words = gq.gptq_pack_codes(codes, bits)
    back = gq.gptq_unpack_codes(words, bits, K)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(_words(words), O.pack_codes(codes.cpu().numpy(), bits))
    assert torch.equal(back, codes)


def test_pack_strided_rows_and_untouched_tail():
    # row pitches larger than the rows (unaligned for the code side); words past each
    # row's ceil(K b / 32) keep their contents
    d = dev()
    N, K, bits = 9, 77, 3
    base = torch.randint(0, 8, (N, K + 5), device=d, dtype=torch.uint8)
    codes = base[:, 2:K + 2]
    nw = (K * bits + 31) // 32
    words = torch.full((N, nw + 3), -1, dtype=torch.int32, device=d)
    gq.gptq_pack_codes(codes, bits, words=words)
    out = torch.zeros(N, K + 9, dtype=torch.uint8, device=d)
    gq.gptq_unpack_codes(words, bits, K, codes=out[:, 1:K + 1])
    torch.cuda.synchronize()
    np.testing.assert_array_equal(_words(words)[:, :nw], O.pack_codes(codes.cpu().numpy(), bits))
    assert (_words(words)[:, nw:] == 0xFFFFFFFF).all()
    assert torch.equal(out[:, 1:K + 1], codes)
    assert (out[:, 0] == 0).all() and (out[:, K + 1:] == 0).all()


def test_pack_only_low_bits_are_read():
    d = dev()
    codes = torch.randint(0, 256, (4, 64), device=d, dtype=torch.uint8)
    words = gq.gptq_pack_codes(codes, 2)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(_words(words), O.pack_codes(codes.cpu().numpy() & 3, 2))


def test_packed_grouped_act_order_reconstructs_write_back():
    # storage round trip of a real solve: unpacked codes with scales[:, g_idx] give the
    # written-back weights, coordinates in the original order
    d = dev()
    K, N, bits, G = 256, 48, 3, 64
    g = torch.Generator(device=d).manual_seed(3)
    X = (torch.randn(4 * K, K, device=d, generator=g) @
         (torch.randn(K, K, device=d, generator=g) / K ** 0.5)).to(torch.bfloat16)
    H = torch.zeros(K, K, device=d)
    gq.gptq_accumulate_hessian(H, X)
    W = (0.02 * torch.randn(N, K, device=d, generator=g)).to(torch.bfloat16)
    perm = gq.gptq_act_order(H)
    Hp = gq.gptq_permute_hessian(H, perm)
    st = gq.gptq_prepare(Hp, 0.01)
    codes, scales, g_idx, st = gq.gptq_quantize_layer_grouped(W, Hp, bits, 128, G, perm=perm,
                                                              write_back=True, status=st)
    gq.raise_on_status(st, "solve")
    words = gq.gptq_pack_codes(codes, bits)
    c = gq.gptq_unpack_codes(words, bits, K).float()
    W_rec = (scales[:, g_idx.long()] * (c - 2 ** (bits - 1))).to(torch.bfloat16)
    torch.cuda.synchronize()
    assert torch.equal(W_rec, W)


def test_pack_headline_layer_size():
    d = dev()
    N, K, bits = 14336, 4096, 3
    g = torch.Generator(device=d).manual_seed(7)
    codes = torch.randint(0, 8, (N, K), generator=g, device=d, dtype=torch.uint8)
    words = gq.gptq_pack_codes(codes, bits)
    back = gq.gptq_unpack_codes(words, bits, K)
    torch.cuda.synchronize()
    assert torch.equal(back, codes)
    rows = np.random.default_rng(0).choice(N, 8, replace=False)
    np.testing.assert_array_equal(_words(words)[rows],
                                  O.pack_codes(codes.cpu().numpy()[rows], bits))
