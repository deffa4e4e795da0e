#!/usr/bin/env python3
"""Benchmark of the GPTQ per-layer solve on B200.

One step = the whole per-layer path on one layer's calibration batch, inputs
resident in HBM:
  Gram over the full token stream (32 x 65,536-token chunks of
  gptq_accumulate_hessian) -> gptq_prepare -> gptq_quantize_layer.
Workload (default): LLaMA-3-8B up_proj shapes, K=4096 inputs, N=14336 outputs,
2,097,152 Student-t bf16 tokens, 3-bit symmetric per-channel, blocksize 128,
percdamp 0.01. value = weights quantized per second of the whole step (K*N per
step); the breakdown reports the layer solve (prepare + quantize) and the Gram.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

For N > 1 each rank solves its own independent layer (weak scaling, no
collective on the data path); timing is the max over ranks. With --shard tokens the
N ranks solve ONE layer instead (strong scaling): each accumulates its share of the
token chunks, one NCCL all-reduce sums H (and C), every rank factors H, and each
quantises its slice of the output channels.
--impl reference times the fp64 CPU oracle on a bounded sample of the same job.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GPTQ layer-solve ms & weights quantized/s (4096×14336, W3); % of TC/HBM roofline"

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch of the dominant
# kernel, from an ncu capture of the same 65,536-token launch. Set to None whenever
# k_gram_tc2 changes until it is captured again.
GRAM_TRAFFIC_BYTES = 1.568243e9 + 0.498444e9
GRAM_TRAFFIC_SOURCE = ("ncu dram__bytes_read.sum + dram__bytes_write.sum of one k_gram_tc2 launch "
                       "(65,536 tokens, K=4096), profiles/gram_tc2_mlp_up_w3_chunk65536.md")
UNIT = "weights/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="mlp_up_w3")
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-seconds", type=float, default=12.0)
    ap.add_argument("--shard", choices=["layers", "tokens"], default="layers",
                    help="N > 1: independent layers per rank, or one layer token-sharded")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch the step's kernels one by one instead of replaying CUDA graphs")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override the stream length (small profiling cases only)")
    return ap.parse_args()


# ----------------------------------------------------------------------------- clocks

CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    """nvidia-smi sampled every 200 ms while the timed region runs."""

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.lines = []
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={CLOCK_FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.gpu_id)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def gpu_smi_id(torch, dev):
    try:
        p = torch.cuda.get_device_properties(dev)
        return f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
    except Exception:
        return dev.index or 0


# ----------------------------------------------------------------------------- CPU oracle sample

def oracle_sample(wl, budget_s):
    """Time the fp64 oracle on a bounded sample of the job; scale to the full job.

    Sample: the Gram of 4,096 tokens (scaled by tokens), the damping + PD check +
    inverse at full K, and the explicit-OBQ sweep over a prefix of the coordinates
    for 8 and 64 channels (scaled by operation counts: the Schur update costs
    (K-j)^2 per step, the channel update N (K-j) per step)."""
    import numpy as np
    import torch

    import oracle as O
    from post_weight_quantization_solve_b200 import synth

    K, N, M = wl.K, wl.N, wl.M
    m_s = 4096
    X = synth.tokens_chunk(wl, 0, "cpu", rows=m_s).double().numpy()
    W = synth.weights(wl, "cpu").double().numpy()
    t = time.perf_counter()
    H = O.gram(X)
    t_gram = (time.perf_counter() - t) * (M / m_s)
    t = time.perf_counter()
    Hd, _ = O.dead_and_damp(H, wl.percdamp)
    O.is_positive_definite(Hd)
    t_prep = time.perf_counter() - t
    t = time.perf_counter()
    np.linalg.inv(Hd)                      # the sweep's one-off inverse (counted in prepare)
    t_inv = time.perf_counter() - t
    t_prep += t_inv
    s, _ = O.symmetric_scale(W, wl.bits)

    def prefix(nch, q):
        t0 = time.perf_counter()
        O.obq_sweep(Hd, W[:nch], s[:nch], wl.bits, steps=q)
        return max(time.perf_counter() - t0 - t_inv, 1e-6)

    probe = 32
    t_probe = prefix(64, probe)
    q = int(max(probe, min(K, probe * (0.4 * budget_s) / t_probe)))
    t_a = prefix(8, q)
    t_b = prefix(64, q)
    j = np.arange(K, dtype=np.float64)
    S_all, S_pre = np.sum((K - j) ** 2), np.sum((K - j[:q]) ** 2)
    L_all, L_pre = np.sum(K - j), np.sum(K - j[:q])
    c_ch = max(t_b - t_a, 0.0) / 56.0
    t_schur = max(t_a - 8 * c_ch, 1e-9)
    t_sweep = t_schur * S_all / S_pre + c_ch * N * L_all / L_pre
    total = t_gram + t_prep + t_sweep
    cores = oracle_threads(torch)
    return {
        "seconds_per_step": total,
        "value": K * N / total,
        "cores": cores,
        "sample": (f"oracle fp64: Gram of {m_s} tokens x{M // m_s} by tokens; damping+PD check+"
                   f"inverse at K={K}; explicit-OBQ sweep, first {q} of {K} coordinates for 8 and "
                   f"64 channels, scaled by (K-j)^2 Schur and N(K-j) channel operation counts "
                   f"(extrapolated)"),
        "parts_s": {"gram": t_gram, "prepare": t_prep, "sweep": t_sweep},
        "measured_s": time_sum(t_gram * m_s / M, t_prep, t_probe, t_a, t_b, 3 * t_inv),
    }


def time_sum(*a):
    return round(sum(a), 2)


def oracle_threads(torch):
    """Threads the oracle's arithmetic runs on: numpy's BLAS pool (its matmuls and
    inverses), else torch's intra-op pool."""
    try:
        import numpy  # noqa: F401  (loads the BLAS the oracle uses)
        import threadpoolctl
        pools = [i["num_threads"] for i in threadpoolctl.threadpool_info()
                 if i.get("user_api") == "blas"]
        if pools:
            return max(pools)
    except Exception:
        pass
    return torch.get_num_threads()


def host_cpu():
    """Model name of the host CPU and its logical core count."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_model": model, "nproc": os.cpu_count()}


def cpu_baseline_entry(cb, value):
    """The JSON line's cpu_baseline object for one oracle sample."""
    return {"value": value, "unit": UNIT, "cores": cb["cores"], "kind": "oracle",
            "sample": cb["sample"], **host_cpu(),
            "stage_seconds": {k: round(v, 3) for k, v in cb["parts_s"].items()},
            "measured_seconds": cb["measured_s"]}


def workload_desc(wl, num_chunks):
    """The workload string of the JSON line's config (both arms)."""
    return (f"{wl.name}: K={wl.K} N={wl.N} tokens={wl.M} (chunks {num_chunks}x{wl.chunk}) "
            f"W{wl.bits} blocksize {wl.blocksize} percdamp {wl.percdamp} groups {wl.groups}"
            + (" gptaq" if wl.gptaq else "") + (" cae" if wl.cae else "")
            + (f" groupsize {wl.groupsize}" if wl.groupsize else "")
            + (" act-order" if wl.act_order else "")
            + (f" first-order beta {wl.first_order}" if wl.first_order else ""))


# ----------------------------------------------------------------------------- ours

def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist

    import post_weight_quantization_solve_b200 as gq
    from post_weight_quantization_solve_b200 import sharded, synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    gq.load_library()
    base = synth.WORKLOADS[args.workload]
    tokens_sharded = args.shard == "tokens" and world > 1
    # independent layers: one layer per rank; token-sharded: the same layer on every rank
    wl = base.scaled(name=base.name, seed=base.seed + (0 if tokens_sharded else 1000 * rank))
    if args.tokens:
        wl = wl.scaled(name=base.name + f"_tokens{args.tokens}", M=args.tokens)
    K, N, M, ch = wl.K, wl.N, wl.M, wl.chunk
    nch = synth.num_chunks(wl)
    # this rank's token chunks and output channels (everything when not token-sharded)
    c0, c1 = sharded.chunk_range(nch, rank, world) if tokens_sharded else (0, nch)
    n0, n1 = sharded.channel_range(N, rank, world) if tokens_sharded else (0, N)
    Ml = min(M, c1 * ch) - c0 * ch     # tokens held by this rank

    g = wl.groups
    X = torch.empty(max(Ml, 0), K, dtype=wl.xdtype, device=dev)
    for c in range(c0, c1):
        X[(c - c0) * ch:(c - c0 + 1) * ch] = synth.tokens_chunk(wl, c, dev)
    Xf = None
    if wl.gptaq:                       # full-precision stream of the asymmetric calibration
        Xf = torch.empty(max(Ml, 0), K, dtype=wl.xdtype, device=dev)
        for c in range(c0, c1):
            Xf[(c - c0) * ch:(c - c0 + 1) * ch] = synth.fp_tokens_chunk(wl, c, dev)
    TW = None
    if g > 1:                          # per-token group weights [g][M]
        TW = torch.empty(g, max(Ml, 0), device=dev)
        for c in range(c0, c1):
            TW[:, (c - c0) * ch:(c - c0 + 1) * ch] = synth.token_weights_chunk(wl, c, dev)
    W = synth.weights(wl, dev)[n0:n1].contiguous()
    Nl = n1 - n0
    H = torch.empty((g, K, K) if g > 1 else (K, K), device=dev)
    C = torch.empty(K, K, device=dev) if wl.gptaq else None
    P1 = torch.empty(K, K, device=dev) if wl.gptaq else None
    codes = torch.empty(Nl, K, dtype=torch.uint8, device=dev)
    grouped = wl.groupsize > 0 or wl.act_order
    if grouped and g > 1:
        raise SystemExit("input groups / act-order take one Hessian (groups == 1)")
    scales = (torch.empty(Nl, (K + wl.groupsize - 1) // wl.groupsize, device=dev) if wl.groupsize
              else torch.empty(Nl, device=dev))
    # first-order term: the sweep quantises an fp32 copy shifted by -beta G H^-1
    Gd = W32 = gamma = ws_f = None
    if wl.first_order:
        if grouped or g > 1 or wl.gptaq or tokens_sharded:
            raise SystemExit("the first-order workload is plain per-channel GPTQ on one layer")
        Gd = synth.gradient(wl, dev)[n0:n1].contiguous()
        W32 = torch.empty(Nl, K, device=dev)
        gamma = torch.zeros(1, dtype=torch.float64, device=dev)
        ws_f = torch.empty(gq.gptq_workspace_size(gq.GPTQ_OP_FIRST_ORDER, K, Nl, 1, 0),
                           dtype=torch.uint8, device=dev)
    g_idx = torch.empty(K, dtype=torch.int32, device=dev) if grouped else None
    perm = torch.empty(K, dtype=torch.int32, device=dev) if wl.act_order else None
    Hp = torch.empty(K, K, device=dev) if wl.act_order else None
    status = gq.new_status(dev)
    ws_p = torch.empty(gq.gptq_workspace_size(gq.GPTQ_OP_PREPARE, K, 0, g, 0), dtype=torch.uint8,
                       device=dev)
    op_q = ((gq.GPTQ_OP_QUANTIZE_GROUPED if grouped else gq.GPTQ_OP_QUANTIZE) |
            (gq.GPTQ_WS_CAE if wl.cae else 0))
    ws_q = torch.empty(gq.gptq_workspace_size(op_q, K, max(Nl, 1), 1 if tokens_sharded else g,
                                              wl.blocksize), dtype=torch.uint8, device=dev)
    segments = sharded.channel_segments(n0, n1, N, g)
    Cp = torch.empty(K, K, device=dev) if (wl.act_order and wl.gptaq) else None
    ws_r = (torch.empty(gq.gptq_workspace_size(gq.GPTQ_OP_RESIDUAL, K, 0, 1, 0), dtype=torch.uint8,
                        device=dev) if wl.gptaq else None)
    # the step runs on its own stream, so that its three phases can be captured as CUDA
    # graphs (every kernel still runs at every replay; graphs only remove launch gaps)
    stream = torch.cuda.Stream(dev)
    use_graph = not args.no_graph and not tokens_sharded
    gram_ev = []
    Hs = Hp if perm is not None else H
    Cs = Cp if (perm is not None and C is not None) else C

    def gram_part(record=None):
        H.zero_()
        if C is not None:
            C.zero_()
        for c in range(c1 - c0):
            if record is not None:
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
            w = None if TW is None else TW[:, c * ch:(c + 1) * ch]
            gq.gptq_accumulate_hessian(H, X[c * ch:(c + 1) * ch], w, status=status, stream=stream)
            if record is not None:
                b.record(stream)
                record.append((a, b))
            if C is not None:
                gq.gptaq_accumulate_cross(C, Xf[c * ch:(c + 1) * ch], X[c * ch:(c + 1) * ch],
                                          status=status, stream=stream)
        if tokens_sharded:              # the solve's one exchange: sum the partial statistics
            sharded.allreduce_statistics(H, C)

    def prepare_part():
        if perm is not None:            # act-order: solve in the reordered coordinates
            gq.gptq_act_order(H, perm=perm, stream=stream)
            gq.gptq_permute_hessian(H, perm, out=Hp, stream=stream)
            if C is not None:
                gq.gptq_permute_hessian(C, perm, out=Cp, stream=stream)
        gq.gptq_prepare(Hs, wl.percdamp, workspace=ws_p, status=status, stream=stream)
        if P1 is not None:
            gq.gptaq_residual(P1, Cs, Hs, workspace=ws_r, stream=stream)

    def quantize_part():
        if Nl == 0:
            pass
        elif grouped:
            gq.gptq_quantize_layer_grouped(W, Hs, wl.bits, wl.blocksize, wl.groupsize,
                                           static_groups=wl.static_groups, perm=perm, P1=P1,
                                           scales_out=scales, g_idx=g_idx, codes=codes,
                                           workspace=ws_q, status=status, stream=stream,
                                           cae=wl.cae)
        elif wl.first_order:
            W32.copy_(W)
            gq.gptq_first_order_shift(W32, Hs, Gd, wl.first_order, gamma=gamma, workspace=ws_f,
                                      status=status, stream=stream)
            gq.gptq_quantize_layer(W32, Hs, wl.bits, wl.blocksize, scales_out=scales, codes=codes,
                                   workspace=ws_q, status=status, stream=stream)
        elif not tokens_sharded:
            gq.gptq_quantize_layer(W, Hs, wl.bits, wl.blocksize, groups=g, P1=P1,
                                   scales_out=scales, codes=codes, workspace=ws_q, status=status,
                                   stream=stream, cae=wl.cae)
        else:                           # this rank's channels, segment by output group
            for gi, a, b in segments:
                gq.gptq_quantize_layer(W[a - n0:b - n0], Hs[gi] if g > 1 else Hs, wl.bits,
                                       wl.blocksize, P1=P1, scales_out=scales[a - n0:b - n0],
                                       codes=codes[a - n0:b - n0], workspace=ws_q,
                                       status=status, stream=stream, cae=wl.cae)

    parts = (gram_part, prepare_part, quantize_part)
    graphs = None

    def step(record=None):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        with torch.cuda.stream(stream):
            ev[0].record(stream)
            for i in range(3):
                if graphs is not None:
                    graphs[i].replay()
                elif i == 0:
                    gram_part(record)
                else:
                    parts[i]()
                ev[i + 1].record(stream)
        return ev

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    gq.raise_on_status(status, "warmup")
    graph_note = "off"
    graph_launches = 0
    if use_graph:
        try:
            l0 = gq.gptq_kernel_launches()
            cap = []
            for fn in parts:
                cap.append(torch.cuda.CUDAGraph())
                with torch.cuda.graph(cap[-1], stream=stream):
                    fn()
            graph_launches = gq.gptq_kernel_launches() - l0   # library kernels in one step
            graphs, cap = cap, None
            step()                      # one replay before timing
            torch.cuda.synchronize()
            gq.raise_on_status(status, "graph replay")
            graph_note = "on (Gram, prepare and quantize phases each replayed as a CUDA graph)"
        except Exception as e:          # report it and time the eager launches instead
            graphs = cap = None
            graph_note = f"capture failed, eager launches: {type(e).__name__}: {e}"[:200]
            torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()

    launches0 = gq.gptq_kernel_launches()
    evs = []
    with ClockSampler(gpu_smi_id(torch, dev)) as clk:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(args.steps):
            evs.append(step(gram_ev))
        t1.record(stream)
        torch.cuda.synchronize()
    # library kernels launched in the timed steps: counted at launch, or, for graph
    # replays, the kernels captured into one step's graphs times the steps
    launches = (gq.gptq_kernel_launches() - launches0) + (graph_launches * args.steps
                                                          if graphs is not None else 0)
    # release the graphs now: with the token-sharded Gram they hold NCCL calls, and a
    # graph holding NCCL work must be gone before the process group is destroyed
    graphs = None
    if world > 1:
        dist.barrier()
    gq.raise_on_status(status, "timed steps")
    total_ms = t0.elapsed_time(t1)
    parts_ms = np.array([[e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2]),
                          e[2].elapsed_time(e[3])] for e in evs])
    # per Gram launch: events around each launch when eager, the phase over its launches
    # when replayed as a graph (inter-launch gaps included)
    gram_launch_ms = (float(np.mean([a.elapsed_time(b) for a, b in gram_ev])) if gram_ev
                      else float(parts_ms[:, 0].mean()) / max(c1 - c0, 1))

    stats = torch.tensor([total_ms, *parts_ms.mean(0).tolist(), gram_launch_ms],
                         dtype=torch.float64, device=dev)
    sharded.max_over_ranks(stats)     # the slowest rank decides
    total_ms, gram_ms, prep_ms, quant_ms, gram_launch_ms = stats.tolist()
    ms_per_step = total_ms / args.steps

    # storage: the step's codes packed to low-bit words (outside the timed steps)
    words = gq.gptq_pack_codes(codes, wl.bits, stream=stream)
    pk0, pk1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    pk0.record(stream)
    for _ in range(10):
        gq.gptq_pack_codes(codes, wl.bits, words=words, stream=stream)
    pk1.record(stream)
    torch.cuda.synchronize()
    pack_ms = pk0.elapsed_time(pk1) / 10
    pack_bytes = Nl * K + words.numel() * 4

    # one eager solve with the library's kernel timing on (outside the timed steps): the
    # per-class kernel times of prepare + quantize, and the sweep's dependent-chain latency
    solve_prof = None
    if not tokens_sharded and Nl > 0:
        with torch.cuda.stream(stream):
            gram_part()
        torch.cuda.synchronize()
        gq.gptq_profile_enable(True)
        with torch.cuda.stream(stream):
            pe0, pe1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            pe0.record(stream)
            prepare_part()
            quantize_part()
            pe1.record(stream)
        torch.cuda.synchronize()
        solve_prof = {k: gq.gptq_profile_read(v) for k, v in
                      (("sweep", gq.GPTQ_PROF_SWEEP), ("update", gq.GPTQ_PROF_UPDATE),
                       ("diag", gq.GPTQ_PROF_DIAG), ("tc32", gq.GPTQ_PROF_TC32))}
        gq.gptq_profile_enable(False)
        solve_prof["eager_ms"] = pe0.elapsed_time(pe1)
        out = gq.gptq_chain_latency(torch.zeros(3, device=dev), steps=1 << 16, stream=stream)
        torch.cuda.synchronize()
        solve_prof["chain"] = (float(out[0].item()), float(out[1].item()))
        gq.raise_on_status(status, "profiled solve")

    e2e = None
    # through the public API with host buffers: the plain per-channel workloads
    if (not args.no_e2e and g == 1 and not wl.gptaq and not tokens_sharded and not grouped
            and not wl.cae and not wl.first_order):
        e2e = run_e2e(args, wl, X, W, dev, gq, torch, dist, world)

    if rank != 0:
        return None
    clocks = clk.summary()
    # symmetric Gram work per 65,536-token chunk (per group for weighted Hessians)
    flops_launch = float(ch) * K * (K + 1) * g
    peaks = load_peaks()
    # the dominant kernel is the tcgen05 Gram; it is timed inside a seconds-long step, so it
    # is compared with the sustained bf16 peak (fallback 1400 TFLOP/s when no measurement)
    peak = peaks.get("bf16_tflops_sustained") or 1400.0
    achieved = flops_launch / (gram_launch_ms * 1e-3) / 1e12
    roofline = {"kernel": ("k_gram_tc2 (CTA pairs)" if g == 1 and K >= 256 else
                           "k_gram_tc" if g == 1 else "k_gram_x_tc (weighted)") +
                          " (gptq_accumulate_hessian, tcgen05)", "bound": "tensor",
                "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4),
                "traffic": GRAM_TRAFFIC_BYTES if (g == 1 and args.workload == "mlp_up_w3") else None,
                "traffic_source": GRAM_TRAFFIC_SOURCE,
                "peak_source": ("MEASURED_PEAKS.json bf16_tflops_sustained (of measured)"
                                if peaks.get("bf16_tflops_sustained") else "fallback 1.4 PFLOP/s"),
                "per_launch": f"{ch} tokens x K(K+1) = {flops_launch:.3e} FLOP (symmetric count)",
                "ms_per_launch": round(gram_launch_ms, 4)}
    weights = K * N * (1 if tokens_sharded else world)
    solve = solve_summary(wl, solve_prof, prep_ms, quant_ms, peaks, wl.groupsize > 0)
    line = {
        "metric": METRIC, "value": weights / (ms_per_step * 1e-3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "strong" if tokens_sharded else "weak",
        "vs_baseline": None, "dtype": "bf16->f32",
        "data": f"synthetic ({wl.stream} bf16 tokens, N(0,{wl.w_sigma}^2) bf16 weights)",
        "config": {"workload": workload_desc(wl, nch),
                   "l2": f"inputs larger than L2 (X {Ml * K * 2 / 1e9:.1f} GB per rank)",
                   "cuda_graphs": graph_note,
                   "parallelism": (f"{world} ranks on one layer: token-sharded Gram, NCCL "
                                   "all-reduce of H, channel-sliced quantisation"
                                   if tokens_sharded else f"{world} independent layers")},
        "breakdown": {"gram_ms": gram_ms, "prepare_ms": prep_ms, "quantize_ms": quant_ms,
                      "layer_solve_ms": prep_ms + quant_ms,
                      "solve_weights_per_s": K * N / ((prep_ms + quant_ms) * 1e-3),
                      "gram_tflops_symmetric": M * K * (K + 1) * g / (gram_ms * 1e-3) / 1e12,
                      "gram_includes_cross": bool(wl.gptaq),
                      "gram_includes_allreduce": tokens_sharded,
                      "quantize_includes_first_order_shift": bool(wl.first_order),
                      "prepare_includes_residual": bool(wl.gptaq)},
        "roofline": roofline,
        "solve": solve,
        "pack": {"kernel": "k_pack (gptq_pack_codes)", "ms": round(pack_ms, 4),
                 "bytes": pack_bytes, "gbs": round(pack_bytes / (pack_ms * 1e-3) / 1e9, 1),
                 "frac_of_hbm": (round(pack_bytes / (pack_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)
                                 if peaks.get("hbm_gbs") else None),
                 "note": "codes N x K bytes in + packed words out, 10 launches after the timed "
                         "steps, not part of the step; issued back to back from Python, so the "
                         "host's launch rate can bound this figure (the kernel alone: "
                         "profiles/pack_mlp_up_w3_N14336_K4096.md)"},
        "gpu_launches": int(launches),
        "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"],
                   "reasons": clocks["reasons"]},
        "measured_peaks": {k: peaks.get(k) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")},
    }
    if e2e:
        line["e2e"] = e2e
    if world == 1 and not args.no_cpu_baseline:
        cb = oracle_sample(wl, args.cpu_sample_seconds)
        line["cpu_baseline"] = cpu_baseline_entry(cb, cb["value"])
    return line


def solve_summary(wl, prof, prep_ms, quant_ms, peaks, input_groups):
    """The layer solve (prepare + quantize on a resident H: the headline of the metric)
    with its rooflines, from the timed steps and one profiled eager solve."""
    K, N = wl.K, wl.N
    ms = prep_ms + quant_ms
    hbm = peaks.get("hbm_gbs") or 6650.0
    tflops = peaks.get("bf16_tflops_sustained") or 1400.0
    # algorithmic HBM bytes per weight of the solve: W in (bf16), one code byte out, and
    # U (fp32 K x K) read once, amortised over the N channels
    bpw = 2.0 + 1.0 + 4.0 * K / N
    out = {"what": "layer solve: gptq_prepare + gptq_quantize_layer on a resident H (CUDA-graph "
                   "replay, timed steps)",
           "ms": ms, "weights_per_s": K * N / (ms * 1e-3),
           "hbm_roofline": {"bytes_per_weight": round(bpw, 4),
                            "peak_weights_per_s": hbm * 1e9 / bpw,
                            "frac": round(K * N / (ms * 1e-3) / (hbm * 1e9 / bpw), 6),
                            "peak_gbs": hbm, "peak_source": "MEASURED_PEAKS.json hbm_gbs (of measured)"
                            if peaks.get("hbm_gbs") else "fallback"}}
    if not prof:
        return out
    sweep_ms, sweep_n = prof["sweep"]
    upd_ms, upd_n = prof["update"]
    cyc, ns = prof["chain"]
    tc_sweep = (K % 4 == 0 and not input_groups and
                os.environ.get("GPTQ_SWEEP_FORM", "3") not in ("0", "1", "2"))
    S = (256 if wl.gptaq else 512) if tc_sweep else 512
    # sweep: bytes it must move (fp32 working weights in, codes out, E as a bf16 pair out;
    # the starting weights in for CAE, the GPTAQ V pair out) against its dependent chain
    sweep_bytes = N * K * (4 + 1 + 4 + (4 if wl.cae else 0) + (4 if wl.gptaq else 0))
    chain_ms = K * ns * 1e-6
    out["sweep"] = {
        "kernel": ("k_sweep_tc (tensor-core near updates in TMEM)" if tc_sweep
                   else "k_sweep_thread / k_sweep_lanes"),
        "ms": round(sweep_ms, 4), "launches": sweep_n,
        "chain_ns_per_step": round(ns, 3), "chain_cycles_per_step": round(cyc, 2),
        "chain_bound_ms": round(chain_ms, 4),
        "frac_of_chain_bound": round(chain_ms / sweep_ms, 4) if sweep_ms else None,
        "bound": "latency (K dependent rounding steps per channel)",
        "hbm_bytes": sweep_bytes,
        "hbm_frac": round(sweep_bytes / (sweep_ms * 1e-3) / (hbm * 1e9), 4) if sweep_ms else None}
    # far updates: every super-block's E (and GPTAQ's V) against the coordinates after it
    useful = 0.0
    for sb0 in range(0, K, S):
        sb1 = min(K, sb0 + S)
        useful += 2.0 * N * (sb1 - sb0) * (K - sb1) * (2 if wl.gptaq else 1)
    if not tc_sweep:     # the SIMT sweeps leave the near updates to the same kernel
        B = wl.blocksize
        for sb0 in range(0, K, 512):
            sb1 = min(K, sb0 + 512)
            for i0 in range(sb0, sb1, B):
                i1 = min(i0 + B, sb1)
                useful += 2.0 * N * (i1 - i0) * (sb1 - i1) * (2 if wl.gptaq else 1)
    ach = useful / (upd_ms * 1e-3) / 1e12 if upd_ms else None
    out["update"] = {
        "kernel": "k_update_tc (bf16x3: three MMAs per product)", "ms": round(upd_ms, 4),
        "launches": upd_n, "useful_flop": useful,
        "achieved_tflops_useful": round(ach, 1) if ach else None,
        "peak_tflops": tflops, "frac_of_sustained": round(ach / tflops, 4) if ach else None,
        "split_ceiling": "1/3 of peak in useful FLOP (each product is three bf16 MMAs)",
        "frac_of_split_ceiling": round(3 * ach / tflops, 4) if ach else None}
    out["prepare_kernels"] = {"diag_ms": round(prof["diag"][0], 4), "diag_launches": prof["diag"][1],
                              "tc32_ms": round(prof["tc32"][0], 4), "tc32_launches": prof["tc32"][1]}
    out["profiled_eager_solve_ms"] = round(prof["eager_ms"], 4)
    out["timing"] = ("sweep / update / factor kernels: CUDA events around each launch on its "
                     "stream in one eager solve after the timed steps (gptq_profile_*); chain: "
                     "gptq_chain_latency, one thread, 65536 dependent steps")
    return out


def run_e2e(args, wl, X, W, dev, gq, torch, dist, world):
    """Same step through the public API with host buffers: every step copies the
    token stream and W from pinned host memory and reads codes + scales back."""
    K, N, M, ch = wl.K, wl.N, wl.M, wl.chunk
    nch = (M + ch - 1) // ch
    Xh = torch.empty(M, K, dtype=X.dtype, pin_memory=True)
    Xh.copy_(X)
    Wh = W.cpu().pin_memory()
    codes_h = torch.empty(N, K, dtype=torch.uint8, pin_memory=True)
    scales_h = torch.empty(N, dtype=torch.float32, pin_memory=True)
    bufs = [torch.empty(ch, K, dtype=X.dtype, device=dev) for _ in range(2)]
    Wd = torch.empty_like(W)
    H = torch.empty(K, K, device=dev)
    codes = torch.empty(N, K, dtype=torch.uint8, device=dev)
    scales = torch.empty(N, device=dev)
    status = gq.new_status(dev)
    ws_p = torch.empty(gq.gptq_workspace_size(gq.GPTQ_OP_PREPARE, K, 0, 1, 0), dtype=torch.uint8,
                       device=dev)
    ws_q = torch.empty(gq.gptq_workspace_size(gq.GPTQ_OP_QUANTIZE, K, N, 1, wl.blocksize),
                       dtype=torch.uint8, device=dev)
    comp = torch.cuda.current_stream(dev)
    copy = torch.cuda.Stream(dev)

    def step():
        H.zero_()
        done = [torch.cuda.Event() for _ in range(2)]
        ready = [torch.cuda.Event() for _ in range(nch)]
        copy.wait_stream(comp)
        for c in range(nch):
            b = bufs[c % 2]
            if c >= 2:
                copy.wait_event(done[c % 2])
            rows = min(ch, M - c * ch)
            with torch.cuda.stream(copy):
                b[:rows].copy_(Xh[c * ch:c * ch + rows], non_blocking=True)
                if c == 0:
                    Wd.copy_(Wh, non_blocking=True)
            ready[c].record(copy)
            comp.wait_event(ready[c])
            gq.gptq_accumulate_hessian(H, b[:rows], stream=comp)
            done[c % 2].record(comp)
        gq.gptq_prepare(H, wl.percdamp, workspace=ws_p, status=status, stream=comp)
        gq.gptq_quantize_layer(Wd, H, wl.bits, wl.blocksize, scales_out=scales, codes=codes,
                               workspace=ws_q, status=status, stream=comp)
        codes_h.copy_(codes, non_blocking=True)
        scales_h.copy_(scales, non_blocking=True)

    step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(comp)
    for _ in range(args.e2e_steps):
        step()
    t1.record(comp)
    torch.cuda.synchronize()
    gq.raise_on_status(status, "e2e")
    ms = torch.tensor([t0.elapsed_time(t1) / args.e2e_steps], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(ms, op=dist.ReduceOp.MAX)
    ms = float(ms.item())
    h2d = Xh.numel() * Xh.element_size() + Wh.numel() * Wh.element_size()
    d2h = codes_h.numel() + scales_h.numel() * 4
    return {"value": K * N * world / (ms * 1e-3), "unit": UNIT, "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            # the copies bound this step: the rate the host-to-device stream achieved
            "h2d_gbs": h2d / (ms * 1e-3) / 1e9,
            "note": "token stream + W from pinned host each step (copy stream, double-buffered), "
                    "codes + scales back; bound by the host-to-device copy of the stream"}


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f)
    except OSError:
        return {}


# ----------------------------------------------------------------------------- reference arm

def run_reference(args, rank, world):
    from post_weight_quantization_solve_b200 import synth

    if rank != 0:
        return None
    wl = synth.WORKLOADS[args.workload]
    budget = max(2.0, min(args.cpu_sample_seconds, 150.0 / max(args.steps + args.warmup, 1)))
    for _ in range(args.warmup):
        oracle_sample(wl, budget)
    runs = [oracle_sample(wl, budget) for _ in range(args.steps)]
    sec = statistics.mean(r["seconds_per_step"] for r in runs)
    value = wl.K * wl.N / sec
    cb = runs[-1]
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (same recipe, CPU generator)",
        "config": {"workload": workload_desc(wl, synth.num_chunks(wl)),
                   "parallelism": "rank 0 only: the fp64 CPU oracle on a bounded sample, scaled "
                                  "to the whole job"},
        "cpu_baseline": cpu_baseline_entry(cb, value),
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", args.gpus if args.gpus == 1 else 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
    else:
        import datetime

        import torch
        import torch.distributed as dist

        if world > 1:
            torch.cuda.set_device(local_rank)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        try:
            line = run_ours(args, rank, world, local_rank)
        finally:
            if world > 1:
                dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
