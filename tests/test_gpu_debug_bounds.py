"""The index-checking build of the library (GPTQ_DEBUG_BOUNDS, libgptq_dbg.so).

Its kernels check tile origins, TMA box coordinates and computed output offsets
before each access; a failed check records the site and index, stores
GPTQ_ERR_BOUNDS in the status word and skips the access (no trap, no fault). Two
runs in child processes that load that build (GPTQ_LIBRARY):
  - the self-test: one check that always fails is recorded, the status word says so,
    a reset clears the record, and a clean solve afterwards records nothing;
  - the parity suites (every per-kernel and end-to-end comparison with the oracle at
    ragged and tile-spanning sizes), each test failing if any check failed during it.
"""

import os
import re
import subprocess
import sys

import pytest

from post_weight_quantization_solve_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = pytest.mark.gpu

SUITES = ["tests/test_gpu_parity.py", "tests/test_gpu_cae.py", "tests/test_gpu_grouped_input.py",
          "tests/test_gpu_first_order.py", "tests/test_gpu_pack.py", "tests/test_gpu_sharded.py",
          "tests/test_zz_no_alloc.py"]

SELFTEST = r"""
import torch
import post_weight_quantization_solve_b200 as gq
from post_weight_quantization_solve_b200 import synth

gq.load_library()
assert gq.gptq_bounds_report(reset=True) == (True, 0, 0, 0)
d = torch.device("cuda:0")
st = gq.new_status(d)
gq.gptq_bounds_selftest(status=st)
torch.cuda.synchronize()
assert int(st.item()) == gq.GPTQ_ERR_BOUNDS, int(st.item())
enabled, count, site, index = gq.gptq_bounds_report(reset=True)
assert (enabled, count, site, index) == (True, 1, 1, -1), (enabled, count, site, index)
assert gq.gptq_bounds_report() == (True, 0, 0, 0)
# a clean solve (Gram, factor, sweep and updates at a ragged size) records nothing
wl = synth.WORKLOADS["mlp_up"].scaled(K=392, N=300, M=3000, bits=3, chunk=1024)
H = torch.zeros(wl.K, wl.K, device=d)
st = gq.new_status(d)
for c in range(synth.num_chunks(wl)):
    gq.gptq_accumulate_hessian(H, synth.tokens_chunk(wl, c, d), status=st)
gq.gptq_prepare(H, wl.percdamp, status=st)
gq.gptq_quantize_layer(synth.weights(wl, d), H, wl.bits, wl.blocksize, status=st)
torch.cuda.synchronize()
assert int(st.item()) == 0, int(st.item())
assert gq.gptq_bounds_report(reset=True) == (True, 0, 0, 0)
print("index-check self-test ok")
"""


def _child(args, timeout):
    env = dict(os.environ, GPTQ_LIBRARY=build(debug_bounds=True))
    return subprocess.run([sys.executable, *args], cwd=ROOT, env=env, capture_output=True,
                          text=True, timeout=timeout)


def test_checking_build_records_a_failed_check():
    r = _child(["-c", SELFTEST], 600)
    assert r.returncode == 0, (r.stdout + r.stderr)[-4000:]
    assert "self-test ok" in r.stdout


def test_parity_suites_pass_with_no_failed_check():
    r = _child(["-m", "pytest", *SUITES, "-m", "gpu", "-x", "-q", "-p", "no:cacheprovider",
                "--basetemp", os.path.join(ROOT, "_build", "pytest-tmp-dbg")], 2400)
    assert r.returncode == 0, (r.stdout + r.stderr)[-4000:]
    passed = re.search(r"(\d+) passed", r.stdout)
    assert passed and int(passed.group(1)) >= 90, r.stdout[-2000:]
