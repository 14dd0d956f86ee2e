"""Seeded synthetic workloads for the HSA operator.

This module only draws random tensors; it holds none of HSA's arithmetic, so both the CUDA path and
the CPU oracle can be fed from it. Every tensor is bf16, drawn from a ``torch.Generator`` seeded per
workload, on the device the caller names.

Workload recipes (shapes follow the benchmark workloads of the operator):
  * ``iid``        Q, K, V, L ~ N(0, 1).
  * ``chunk_mean`` Q, K, V ~ N(0, 1); each landmark is the fp32 mean of its chunk's 64 keys plus
                   N(0, 0.1^2) noise (standard deviation 0.1), rounded to bf16, so that retrieval
                   scores carry structure.
  * decode         q, K/V cache and landmark cache ~ N(0, 1); in every sequence one chunk index is
                   drawn uniformly among the complete chunks and, for every head, that chunk's
                   landmark is set to bf16(3 * q): a planted "needle" shaped like the explainer's
                   single-needle retrieval probe (synthetic; no evaluation-suite item is used).
"""
from dataclasses import dataclass, field

import torch

BF16 = torch.bfloat16


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str                 # "forward" | "decode" | "backward"
    B: int
    H: int
    D: int
    topk: int
    seed: int
    T: int = 0                # prefill / backward sequence length
    cache_len: int = 0        # decode: tokens in every sequence's cache
    landmarks: str = "iid"    # "iid" | "chunk_mean"
    noise_std: float = 0.1
    chunk: int = 64
    extra: dict = field(default_factory=dict)


WORKLOADS = {
    w.name: w
    for w in (
        Workload("fwd_t4k_h4_d64_k8", "forward", B=1, H=4, D=64, topk=8, T=4096, seed=1001),
        Workload("fwd_t32k_h8_d128_k16", "forward", B=2, H=8, D=128, topk=16, T=32768,
                 landmarks="chunk_mean", seed=1002),
        Workload("decode_1m_b16_h8_d128_k16", "decode", B=16, H=8, D=128, topk=16, cache_len=1 << 20,
                 seed=1003),
        Workload("decode_16m_b1_h8_d128_k32", "decode", B=1, H=8, D=128, topk=32, cache_len=1 << 24,
                 seed=1004),
        Workload("fwdbwd_t64k_h8_d128_k16", "backward", B=1, H=8, D=128, topk=16, T=65536, seed=1005),
    )
}


def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(shape, g, device):
    return torch.randn(shape, generator=g, device=device, dtype=BF16)


def forward_inputs(B, H, T, D, seed, chunk=64, landmarks="iid", noise_std=0.1, device="cpu"):
    """Q, K, V [B, H, T, D] and L [B, H, T // chunk, D], all bf16."""
    g = _gen(seed, device)
    Q = _randn((B, H, T, D), g, device)
    K = _randn((B, H, T, D), g, device)
    V = _randn((B, H, T, D), g, device)
    N = T // chunk
    if landmarks == "iid":
        L = _randn((B, H, N, D), g, device)
    elif landmarks == "chunk_mean":
        mean = K[:, :, : N * chunk].float().reshape(B, H, N, chunk, D).mean(dim=3)
        noise = torch.randn((B, H, N, D), generator=g, device=device, dtype=torch.float32) * noise_std
        L = (mean + noise).to(BF16)
    else:
        raise ValueError(f"unknown landmark recipe {landmarks!r}")
    return Q, K, V, L


def upstream_grad(B, H, T, D, seed, device="cpu"):
    """dO [B, H, T, D] bf16 ~ N(0, 1), from its own stream (seed + 7919)."""
    return _randn((B, H, T, D), _gen(seed + 7919, device), device)


def decode_inputs(B, H, cache_len, D, seed, chunk=64, needle=True, Tmax=None, device="cpu"):
    """q [B,H,D]; Kc, Vc [B,H,Tmax,D]; Lc [B,H,Tmax//chunk,D]; cache_len [B] int64; needle [B] int64.

    ``cache_len`` may be an int (same length for every sequence) or a list of B ints.
    """
    lens = [int(cache_len)] * B if isinstance(cache_len, int) else [int(x) for x in cache_len]
    if Tmax is None:
        Tmax = max(lens)
    g = _gen(seed, device)
    q = _randn((B, H, D), g, device)
    Kc = _randn((B, H, Tmax, D), g, device)
    Vc = _randn((B, H, Tmax, D), g, device)
    Nmax = Tmax // chunk
    Lc = _randn((B, H, Nmax, D), g, device)
    needle_pos = torch.full((B,), -1, dtype=torch.int64)
    if needle:
        gcpu = _gen(seed + 104729, "cpu")
        for b in range(B):
            n = lens[b] // chunk
            if n > 0:
                c = int(torch.randint(0, n, (1,), generator=gcpu).item())
                needle_pos[b] = c
                Lc[b, :, c, :] = (3.0 * q[b].float()).to(BF16)
    lens_t = torch.tensor(lens, dtype=torch.int64, device=device)
    return q, Kc, Vc, Lc, lens_t, needle_pos


def workload_inputs(w: Workload, device="cpu"):
    """Inputs of a named workload (forward/backward: Q, K, V, L[, dO]; decode: see decode_inputs)."""
    if w.kind == "forward":
        return forward_inputs(w.B, w.H, w.T, w.D, w.seed, w.chunk, w.landmarks, w.noise_std, device)
    if w.kind == "backward":
        Q, K, V, L = forward_inputs(w.B, w.H, w.T, w.D, w.seed, w.chunk, w.landmarks, w.noise_std, device)
        return Q, K, V, L, upstream_grad(w.B, w.H, w.T, w.D, w.seed, device)
    if w.kind == "decode":
        return decode_inputs(w.B, w.H, w.cache_len, w.D, w.seed, w.chunk, True, device=device)
    raise ValueError(w.kind)
