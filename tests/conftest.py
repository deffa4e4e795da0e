import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


@pytest.hookimpl(tryfirst=True)
def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workloads")
    # scratch files of the tests (tmp_path) stay inside the repository, in a build folder
    if not config.option.basetemp:
        os.makedirs(os.path.join(ROOT, "_build"), exist_ok=True)
        config.option.basetemp = os.path.join(ROOT, "_build", "pytest-tmp")


@pytest.fixture(autouse=True)
def _index_check_records(request):
    """Under the index-checking build (GPTQ_LIBRARY=.../libgptq_dbg.so), a GPU test
    fails if any kernel check failed during it (the access was skipped, so the test's
    own comparisons may still have passed)."""
    yield
    if not os.environ.get("GPTQ_LIBRARY") or request.node.get_closest_marker("gpu") is None:
        return
    import post_weight_quantization_solve_b200 as gq

    if gq._lib is None:
        return
    enabled, count, site, index = gq.gptq_bounds_report(reset=True)
    assert not enabled or count == 0, f"{count} failed index checks, first at site {site}, index {index}"


def load_golden(name):
    """Parse a `key = values` fixture; `;` separates matrix rows."""
    out = {}
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = (p.strip() for p in line.split("=", 1))
            rows = [r.split() for r in val.split(";")]
            arr = np.array([[float(x) for x in r] for r in rows])
            out[key] = arr[0] if arr.shape[0] == 1 else arr
            if out[key].size == 1:
                out[key] = float(out[key].reshape(-1)[0])
    return out


@pytest.fixture
def golden():
    return load_golden
