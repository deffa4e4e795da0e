"""The multi-rank split of one layer on CPU: two gloo ranks (no GPU).

Each rank accumulates its share of the token chunks into a partial Gram, one all-reduce
sums them, and each rank solves its slice of output channels; the assembled result must
equal the single-process solve. The per-rank arithmetic is the fp64 oracle here (these
tests check the split and the collectives, the GPU tests check the kernels); the
collectives are the same helpers bench.py uses over NCCL.
"""

import os
import socket
import traceback

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
from post_weight_quantization_solve_b200 import sharded


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run(world, fn, *args, timeout_s=60):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_entry, args=(r, world, port, fn, args, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(world):
        r, res = q.get(timeout=timeout_s)
        out[r] = res
    for p in procs:
        p.join(timeout=timeout_s)
    return out


def _entry(rank, world, port, fn, args, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    try:
        import datetime
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=20))
        try:
            res = fn(rank, world, *args)
        finally:
            dist.destroy_process_group()
        q.put((rank, ("ok", res)))
    except Exception:
        q.put((rank, ("error", traceback.format_exc())))


# ------------------------------------------------------------------ host arithmetic

@pytest.mark.parametrize("n,world", [(32, 2), (7, 3), (2, 4), (0, 2), (14336, 8)])
def test_ranges_partition(n, world):
    seen = []
    for r in range(world):
        a, b = sharded.chunk_range(n, r, world)
        assert 0 <= a <= b <= n and b - a in (n // world, n // world + 1)
        seen.extend(range(a, b))
    assert seen == list(range(n))


@pytest.mark.parametrize("N,groups,world", [(12, 1, 2), (12, 4, 5), (8192, 4, 8), (10, 2, 3)])
def test_channel_segments_follow_groups(N, groups, world):
    per = N // groups
    covered = []
    for r in range(world):
        n0, n1 = sharded.channel_range(N, r, world)
        for gi, a, b in sharded.channel_segments(n0, n1, N, groups):
            assert gi * per <= a < b <= (gi + 1) * per
            covered.extend(range(a, b))
    assert covered == list(range(N))
    with pytest.raises(ValueError):
        sharded.channel_segments(0, 5, 10, 3)


# ------------------------------------------------------------------ collectives

def _rank_solve(rank, world, X, W, bits, chunk, groups, weights):
    """One rank: partial Gram of its chunks, all-reduce, solve its channel slice."""
    M, K = X.shape
    nch = (M + chunk - 1) // chunk
    c0, c1 = sharded.chunk_range(nch, rank, world)
    rows = slice(c0 * chunk, min(M, c1 * chunk))
    H = torch.zeros(groups, K, K, dtype=torch.float64)
    for gi in range(groups):
        if rows.stop > rows.start:
            s = None if weights is None else weights[gi][rows]
            H[gi] = torch.from_numpy(O.gram(X[rows], s))
    sharded.allreduce_statistics(H)
    N = W.shape[0]
    n0, n1 = sharded.channel_range(N, rank, world)
    codes = torch.zeros(n1 - n0, K, dtype=torch.float64)
    for gi, a, b in sharded.channel_segments(n0, n1, N, groups):
        r = O.solve_layer(H[gi].numpy(), W[a:b], bits)
        codes[a - n0:b - n0] = torch.from_numpy(r["codes"])
    full = sharded.all_gather_rows(codes, N)
    t = torch.tensor([float(rank), 2.0 * rank], dtype=torch.float64)
    sharded.max_over_ranks(t)
    return H.numpy(), full.numpy(), t.numpy()


@pytest.mark.parametrize("groups,world", [(1, 2), (2, 2), (2, 3)])
def test_token_sharded_layer_equals_single_process(groups, world):
    # with 3 ranks the token counts differ (the last of the 6 chunks is ragged), the 10
    # channels split 3/3/4, and rank 1's channels straddle the two 5-channel groups
    rng = np.random.default_rng(3 + groups + world)
    M, K, N, chunk, bits = 700, 24, 10, 128, 3
    X = rng.standard_normal((M, K)) @ (np.eye(K) + 0.2 * rng.standard_normal((K, K)))
    W = 0.02 * rng.standard_normal((N, K))
    weights = None if groups == 1 else [rng.uniform(0.5, 2.0, M) for _ in range(groups)]
    out = _run(world, _rank_solve, X, W, bits, chunk, groups, weights)
    for r in range(world):
        assert out[r][0] == "ok", out[r][1]
    H0, codes0, t0 = out[0][1]
    for gi in range(groups):
        ref = O.gram(X, None if weights is None else weights[gi])
        np.testing.assert_allclose(H0[gi], ref, rtol=1e-12, atol=1e-9)
    per = N // groups
    expect = np.zeros((N, K))
    for gi in range(groups):
        expect[gi * per:(gi + 1) * per] = O.solve_layer(
            O.gram(X, None if weights is None else weights[gi]), W[gi * per:(gi + 1) * per],
            bits)["codes"]
    for r in range(world):
        Hr, codes_r, t_r = out[r][1]
        np.testing.assert_array_equal(Hr, H0)      # every rank holds the same statistic
        np.testing.assert_array_equal(codes_r, expect)
        np.testing.assert_array_equal(t_r, [world - 1.0, 2.0 * (world - 1)])


def _rank_leaves(rank, world):
    """Rank 1 leaves before the all-reduce; rank 0's collective must end with an error
    (not hang) within the process group's timeout."""
    if rank == 1:
        return "left"
    H = torch.ones(4, 4, dtype=torch.float64)
    try:
        sharded.allreduce_statistics(H)
    except Exception as e:       # gloo reports the lost peer or the timeout
        return f"error: {type(e).__name__}"
    return "completed"


def test_lost_rank_fails_the_collective():
    out = _run(2, _rank_leaves, timeout_s=90)
    assert out[1] == ("ok", "left")
    status, msg = out[0]
    assert (status == "ok" and msg.startswith("error")) or status == "error", out[0]
