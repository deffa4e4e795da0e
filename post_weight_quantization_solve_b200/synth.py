"""Seeded synthetic calibration inputs shaped like the LLaMA-3 layer workloads.

This module only draws random numbers and lays them out; it holds none of the
solve's arithmetic, so both the fp64 oracle and the CUDA path can be fed from it.
Every tensor is drawn from a torch generator keyed by (workload seed, tensor id,
chunk index), so any 65,536-token chunk of a long stream can be regenerated on its
own. CPU and CUDA generators give different streams: a test draws once and hands
the same bytes to both sides.

Workloads (sizes from the pages: 1024 calibration sequences of 2048 tokens,
LLaMA-3 8B / 70B layer widths):
  tiny       K=128,  N=256,   2,048 fp32 tokens X = Z A (correlated columns)
  q_proj     K=N=4096,        262,144 bf16 tokens, 16 outlier channels x20, then a
             random-sign Hadamard rotation applied to X and W alike
  mlp_up     K=4096, N=14336, 2,097,152 bf16 Student-t(4)/sqrt(2) tokens
  mlp_down   K=14336, N=4096, same stream recipe
  gptaq      K=N=4096, 262,144 tokens: full-precision stream X~ ~ N(0,1) bf16 and
             quantised stream X = bf16(X~ + D), D ~ N(0, (0.05 rms(X~))^2)
  grouped70b K=28672, N=8192, 262,144 bf16 N(0,1) tokens, g=4 per-token weights
             s_g = z^2 / mean(z^2)
"""

from __future__ import annotations

from dataclasses import dataclass, field

import torch

CHUNK_TOKENS = 65536

# tensor ids inside a workload
T_X, T_W, T_MIX, T_OUTLIER, T_SIGNS, T_NOISE, T_TOKW, T_CHI, T_GRAD = range(9)


def generator(seed: int, tensor_id: int, chunk: int = 0, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + tensor_id) * 1_000_033 + chunk)
    return g


@dataclass
class Workload:
    name: str
    K: int
    N: int
    M: int
    bits: int
    blocksize: int
    percdamp: float
    seed: int
    xdtype: torch.dtype
    groups: int = 1
    gptaq: bool = False
    stream: str = "normal"        # normal | correlated | student_t | rotated
    w_sigma: float = 0.02
    outliers: int = 0
    chunk: int = CHUNK_TOKENS
    groupsize: int = 0            # input-dimension groups (0: per-channel scales)
    act_order: bool = False
    static_groups: bool = False
    cae: bool = False             # compensation-aware error term
    first_order: float = 0.0      # beta of the first-order (gradient) term; 0: none
    extra: dict = field(default_factory=dict)

    def scaled(self, K=None, N=None, M=None, name=None, **kw):
        """Same recipe at other sizes (parity cases the oracle finishes in seconds)."""
        d = dict(self.__dict__)
        d.update(K=K or self.K, N=N or self.N, M=M or self.M, name=name or self.name + "_small")
        d.update(kw)
        return Workload(**d)


WORKLOADS = {
    "tiny": Workload("tiny", 128, 256, 2048, 4, 32, 0.01, 0, torch.float32, stream="correlated"),
    "q_proj": Workload("q_proj", 4096, 4096, 262144, 3, 128, 0.01, 1, torch.bfloat16,
                       stream="rotated", outliers=16),
    "mlp_up": Workload("mlp_up", 4096, 14336, 2097152, 2, 128, 0.01, 2, torch.bfloat16,
                       stream="student_t"),
    "mlp_down": Workload("mlp_down", 14336, 4096, 2097152, 2, 128, 0.01, 2, torch.bfloat16,
                         stream="student_t"),
    "gptaq": Workload("gptaq", 4096, 4096, 262144, 2, 128, 0.01, 3, torch.bfloat16,
                      gptaq=True),
    "grouped70b": Workload("grouped70b", 28672, 8192, 262144, 4, 128, 0.01, 4, torch.bfloat16,
                           groups=4, w_sigma=0.01),
}
# the headline solve: up_proj shapes at 3 bits
WORKLOADS["mlp_up_w3"] = WORKLOADS["mlp_up"].scaled(name="mlp_up_w3", bits=3)
# the same layer with 128-wide input groups (re-estimated) and act-order
WORKLOADS["mlp_up_w3_g128"] = WORKLOADS["mlp_up"].scaled(name="mlp_up_w3_g128", bits=3,
                                                         groupsize=128, act_order=True)
# the asymmetric-calibration layer with the compensation-aware error term as well
WORKLOADS["gptaq_cae"] = WORKLOADS["gptaq"].scaled(name="gptaq_cae", cae=True)
# the headline layer with a first-order term (synthetic gradient, beta 0.5)
WORKLOADS["mlp_up_w3_fo"] = WORKLOADS["mlp_up"].scaled(name="mlp_up_w3_fo", bits=3,
                                                       first_order=0.5)


def hadamard(K: int, device="cpu") -> torch.Tensor:
    """Sylvester Hadamard matrix of order K (a power of two), entries +-1."""
    assert K & (K - 1) == 0
    Hm = torch.ones(1, 1, device=device)
    while Hm.shape[0] < K:
        Hm = torch.cat([torch.cat([Hm, Hm], 1), torch.cat([Hm, -Hm], 1)], 0)
    return Hm


def _rotation(wl: Workload, device) -> torch.Tensor:
    signs = torch.randint(0, 2, (wl.K,), generator=generator(wl.seed, T_SIGNS, 0, device),
                          device=device).float() * 2 - 1
    return (signs[:, None] * hadamard(wl.K, device)) / (wl.K ** 0.5)


def _outlier_channels(wl: Workload, device) -> torch.Tensor:
    perm = torch.randperm(wl.K, generator=generator(wl.seed, T_OUTLIER, 0, device), device=device)
    return perm[: wl.outliers]


def tokens_chunk(wl: Workload, chunk: int, device="cpu", rows=None) -> torch.Tensor:
    """Chunk `chunk` of the calibration stream X (rows x K, the workload's dtype).

    For the GPTAQ workload this is the quantised stream X; see fp_tokens_chunk."""
    m0 = chunk * wl.chunk
    rows = rows if rows is not None else min(wl.chunk, wl.M - m0)
    g = generator(wl.seed, T_X, chunk, device)
    if wl.stream == "correlated":
        Z = torch.randn(rows, wl.K, generator=g, device=device, dtype=torch.float64)
        A = torch.randn(wl.K, wl.K, generator=generator(wl.seed, T_MIX, 0, device), device=device,
                        dtype=torch.float64) / (wl.K ** 0.5)
        return (Z @ A).to(wl.xdtype)
    if wl.stream == "student_t":
        z = torch.randn(rows, wl.K, generator=g, device=device)
        # chi-square with 4 degrees of freedom = sum of two exponentials of mean 2
        gc = generator(wl.seed, T_CHI, chunk, device)
        u = torch.rand(2, rows, wl.K, generator=gc, device=device).clamp_min_(1e-30)
        chi4 = -2.0 * torch.log(u).sum(0)
        t = z / torch.sqrt(chi4 / 4.0)
        return (t / (2.0 ** 0.5)).to(wl.xdtype)      # Var t_4 = 2
    if wl.stream == "rotated":
        X0 = torch.randn(rows, wl.K, generator=g, device=device)
        X0[:, _outlier_channels(wl, device)] *= 20.0
        return (X0 @ _rotation(wl, device)).to(wl.xdtype)
    if wl.gptaq:
        Xfp = fp_tokens_chunk(wl, chunk, device, rows)
        rms = fp_stream_rms(wl, device)
        D = torch.randn(rows, wl.K, generator=generator(wl.seed, T_NOISE, chunk, device),
                        device=device) * (0.05 * rms)
        return (Xfp.float() + D).to(wl.xdtype)
    return torch.randn(rows, wl.K, generator=g, device=device).to(wl.xdtype)


def fp_tokens_chunk(wl: Workload, chunk: int, device="cpu", rows=None) -> torch.Tensor:
    """GPTAQ full-precision stream X~ (N(0,1), the workload's dtype)."""
    m0 = chunk * wl.chunk
    rows = rows if rows is not None else min(wl.chunk, wl.M - m0)
    g = generator(wl.seed, T_X, chunk, device)
    return torch.randn(rows, wl.K, generator=g, device=device).to(wl.xdtype)


_RMS_CACHE: dict = {}


def fp_stream_rms(wl: Workload, device="cpu") -> float:
    """Global scalar rms of X~ over the whole stream."""
    key = (wl.name, wl.seed, wl.M, wl.K, wl.chunk, str(device))
    if key not in _RMS_CACHE:
        acc, cnt = 0.0, 0
        for c in range(num_chunks(wl)):
            x = fp_tokens_chunk(wl, c, device).float()
            acc += float((x * x).sum())
            cnt += x.numel()
        _RMS_CACHE[key] = (acc / cnt) ** 0.5
    return _RMS_CACHE[key]


def num_chunks(wl: Workload) -> int:
    return (wl.M + wl.chunk - 1) // wl.chunk


def token_weights_chunk(wl: Workload, chunk: int, device="cpu", rows=None) -> torch.Tensor:
    """Per-token group weights s[g][rows] (fp32): z^2 normalised to mean 1 per group.

    The normaliser is the mean over the whole stream, drawn chunk by chunk."""
    m0 = chunk * wl.chunk
    rows = rows if rows is not None else min(wl.chunk, wl.M - m0)
    z = torch.randn(wl.groups, rows, generator=generator(wl.seed, T_TOKW, chunk, device),
                    device=device)
    return (z * z) / _token_weight_mean(wl, device)[:, None]


_TW_CACHE: dict = {}


def _token_weight_mean(wl: Workload, device) -> torch.Tensor:
    key = (wl.name, wl.seed, wl.M, wl.groups, wl.chunk, str(device))
    if key not in _TW_CACHE:
        acc = torch.zeros(wl.groups, device=device, dtype=torch.float64)
        for c in range(num_chunks(wl)):
            rows = min(wl.chunk, wl.M - c * wl.chunk)
            z = torch.randn(wl.groups, rows, generator=generator(wl.seed, T_TOKW, c, device),
                            device=device)
            acc += (z * z).double().sum(1)
        _TW_CACHE[key] = (acc / wl.M).float()
    return _TW_CACHE[key]


def weights(wl: Workload, device="cpu") -> torch.Tensor:
    """Layer weights W[N][K] (nn.Linear order), N(0, sigma^2), rotated like X for
    the rotated stream; stored in the stream's dtype."""
    W = torch.randn(wl.N, wl.K, generator=generator(wl.seed, T_W, 0, device), device=device)
    W = W * wl.w_sigma
    if wl.stream == "rotated":
        W = W @ _rotation(wl, device)
    return W.to(wl.xdtype)


def gradient(wl: Workload, device="cpu") -> torch.Tensor:
    """A synthetic gradient of the block objective w.r.t. W[N][K] for the first-order
    term, fp32 (the gradient comes from backprop, which the solve does not run). Like
    H = 2 X^T X it grows with the token count: for unit-variance tokens H's diagonal is
    about 2M, so g ~ N(0, (0.1 w_sigma 2M)^2) makes the Newton step H^-1 g about a tenth
    of the weights' spread."""
    g = torch.randn(wl.N, wl.K, generator=generator(wl.seed, T_GRAD, 0, device), device=device)
    return g * (0.1 * wl.w_sigma * 2.0 * wl.M)
