"""Failure path and resume on the GPU (no fault, trap or hang is ever caused).

- The bounded-wait failure path: a wait that nothing releases runs out after its budget,
  the status word reports GPTQ_ERR_TIMEOUT, later calls given that word skip their work,
  and the context stays usable.
- Checkpoint / resume: the accumulation state is the caller's H; saved to the host after
  some chunks and restored, it continues to the same result.
"""

import numpy as np
import pytest
import torch

import oracle as O
import post_weight_quantization_solve_b200 as gq
from post_weight_quantization_solve_b200 import synth
from post_weight_quantization_solve_b200.build import build

from gpu_util import TOL_H, dev, rel_max

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    gq.load_library()


def test_bounded_wait_times_out_and_context_survives():
    d = dev()
    st = gq.gptq_selftest_timeout()
    torch.cuda.synchronize()
    assert int(st.item()) == gq.GPTQ_ERR_TIMEOUT
    # a failed status word makes later kernels skip their work
    K = 256
    H = torch.eye(K, device=d) * 3.0
    gq.gptq_prepare(H, 0.01, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == gq.GPTQ_ERR_TIMEOUT
    assert torch.equal(H, torch.eye(K, device=d) * 3.0)
    # the context is intact: a fresh solve works
    X = torch.randn(4096, K, device=d).to(torch.bfloat16)
    H2 = torch.zeros(K, K, device=d)
    st2 = gq.new_status(d)
    gq.gptq_accumulate_hessian(H2, X, status=st2)
    gq.raise_on_status(st2, "after timeout")
    assert rel_max(H2.double().cpu().numpy(), O.gram(X.double().cpu().numpy())) <= TOL_H


def test_hessian_checkpoint_and_resume():
    d = dev()
    wl = synth.WORKLOADS["mlp_up"].scaled(K=512, N=64, M=6 * 4096, chunk=4096)
    chunks = [synth.tokens_chunk(wl, c, d) for c in range(synth.num_chunks(wl))]
    K = wl.K
    full = torch.zeros(K, K, device=d)
    for x in chunks:
        gq.gptq_accumulate_hessian(full, x)
    part = torch.zeros(K, K, device=d)
    for x in chunks[:3]:
        gq.gptq_accumulate_hessian(part, x)
    saved = part.cpu().clone()                 # checkpoint to the host
    del part
    resumed = saved.to(d)                      # restore and continue
    for x in chunks[3:]:
        gq.gptq_accumulate_hessian(resumed, x)
    torch.cuda.synchronize()
    # the same sums in another order of fp32 reductions
    assert rel_max(resumed.double().cpu().numpy(), full.double().cpu().numpy()) <= 1e-6
    X = np.concatenate([x.double().cpu().numpy() for x in chunks])
    assert rel_max(resumed.double().cpu().numpy(), O.gram(X)) <= TOL_H
