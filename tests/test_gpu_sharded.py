"""The token-sharded layer through the library, on one GPU (C ABI calls).

[GPTQ blog] "Calibration 让量化看见输入方向": H is a sum over token batches, so each rank
can accumulate its own chunks and one all-reduce adds the partial sums;
"GPTQ 怎样把逐个补偿变成可扩展算法": given the shared factor every output channel is
quantised on its own, so each rank solves a slice of the channels. Here the ranks of
bench.py --shard tokens run one after the other in one process (no collective: the
partial statistics are added as the all-reduce would add them) with the same helpers
(sharded.chunk_range, channel_range, channel_segments):
  - the summed partial Grams equal the one-pass Gram and the oracle's Gram;
  - every rank's channel segments, each quantised with its output group's factor,
    assemble to codes and scales bit-identical to the whole-layer call on that H.
"""

import numpy as np
import pytest
import torch

import oracle as O
import post_weight_quantization_solve_b200 as gq
from post_weight_quantization_solve_b200 import sharded, synth
from post_weight_quantization_solve_b200.build import build

from gpu_util import TOL_H, dev, rel_max

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    gq.load_library()


@pytest.mark.parametrize("world,groups", [(2, 1), (3, 1), (3, 4)])
def test_token_sharded_layer_matches_single_call(world, groups):
    d = dev()
    if groups == 1:
        wl = synth.WORKLOADS["mlp_up"].scaled(K=512, N=392, M=5000, bits=3, chunk=1024)
    else:
        wl = synth.WORKLOADS["grouped70b"].scaled(K=256, N=512, M=5000, chunk=1024)
    K, N, g = wl.K, wl.N, groups
    nch = synth.num_chunks(wl)
    chunks = [synth.tokens_chunk(wl, c, d) for c in range(nch)]
    wts = [synth.token_weights_chunk(wl, c, d) for c in range(nch)] if g > 1 else None
    shape = (g, K, K) if g > 1 else (K, K)

    # one pass over the whole stream
    H_one = torch.zeros(shape, device=d)
    for c in range(nch):
        gq.gptq_accumulate_hessian(H_one, chunks[c], None if wts is None else wts[c])
    # per rank: its contiguous chunks into a partial statistic; then the sum
    H = torch.zeros(shape, device=d)
    for r in range(world):
        c0, c1 = sharded.chunk_range(nch, r, world)
        Hr = torch.zeros(shape, device=d)
        for c in range(c0, c1):
            gq.gptq_accumulate_hessian(Hr, chunks[c], None if wts is None else wts[c])
        H += Hr
    torch.cuda.synchronize()
    X = torch.cat([c.double().cpu() for c in chunks]).numpy()
    for gi in range(g):
        Hg = H[gi] if g > 1 else H
        s = None if wts is None else torch.cat([w[gi].double().cpu() for w in wts]).numpy()
        assert rel_max(Hg.double().cpu().numpy(), O.gram(X, s)) <= TOL_H
        assert rel_max(Hg.double().cpu().numpy(), (H_one[gi] if g > 1 else H_one).double().cpu().numpy()) <= TOL_H

    # the factor, replicated on every rank in bench.py
    U = H.clone()
    st = gq.gptq_prepare(U, wl.percdamp)
    W = synth.weights(wl, d)
    codes_all = torch.empty(N, K, dtype=torch.uint8, device=d)
    scales_all = torch.empty(N, device=d)
    gq.gptq_quantize_layer(W.clone(), U, wl.bits, wl.blocksize, groups=g, codes=codes_all,
                           scales_out=scales_all, status=st)
    # per rank: its channels, split at the output-group boundaries
    codes_parts, scales_parts = [], []
    for r in range(world):
        n0, n1 = sharded.channel_range(N, r, world)
        cr = torch.empty(n1 - n0, K, dtype=torch.uint8, device=d)
        sr = torch.empty(n1 - n0, device=d)
        for gi, a, b in sharded.channel_segments(n0, n1, N, g):
            gq.gptq_quantize_layer(W[a:b].clone(), U[gi] if g > 1 else U, wl.bits, wl.blocksize,
                                   codes=cr[a - n0:b - n0], scales_out=sr[a - n0:b - n0], status=st)
        codes_parts.append(cr)
        scales_parts.append(sr)
    gq.raise_on_status(st, "sharded solve")
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(codes_parts), codes_all)
    assert torch.equal(torch.cat(scales_parts), scales_all)
