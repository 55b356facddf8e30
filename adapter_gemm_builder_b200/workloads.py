"""Seeded synthetic workloads for the multi-tenant LoRA path.

This module only draws random inputs and stores them in their storage types
(bf16 bit patterns as uint16, int32 ids). It holds none of the method's
arithmetic, so both the CUDA path's tests/benchmark and the CPU oracle take
their inputs from here.

Shapes follow the pages' workloads: Llama-2 projection shapes (GD2O page;
7B q_proj 4096x4096, 7B MLP up_proj 4096x11008, 13B o_proj 5120x5120,
70B-like up_proj 8192x28672), decode batches and Punica's adapter popularity
settings (Punica README: "Distinct", "Identical", "Uniform", "Skewed";
Skewed is drawn from a finite Zipf law).

Distributions: x ~ N(0,1); A ~ N(0, 1/h_in); B ~ N(0, 1/r_i); W ~ N(0, 1/K);
a stand-in for the base output y_in ~ N(0,1); every value rounded to bf16
(round-to-nearest-even, by torch's CPU conversion). Adapter padding beyond an
adapter's rank (A columns, B rows) is filled with ``pad_value`` bits (NaN by
default, so any read of it shows up in the result).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

BF16_NAN = 0x7FC0


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 array -> bf16 bit patterns (uint16), round to nearest even (torch CPU)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def normal_bf16(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return to_bf16_bits(a)


def zipf_ids(rng: np.random.Generator, n: int, n_adapters: int, s: float = 1.1) -> np.ndarray:
    """Finite Zipf law over 0..n_adapters-1: P(k) proportional to (k+1)^-s,
    sampled by inverting the cumulative distribution."""
    w = np.arange(1, n_adapters + 1, dtype=np.float64) ** (-s)
    cdf = np.cumsum(w / w.sum())
    cdf[-1] = 1.0
    u = rng.random(n)
    return np.searchsorted(cdf, u, side="right").astype(np.int32)


def make_ids(kind: str, rng: np.random.Generator, T: int, n_adapters: int,
             none_frac: float = 0.0) -> np.ndarray:
    """Per-token adapter ids for one batch.

    kind: "distinct" (token t -> adapter t, needs T <= n_adapters),
    "identical" (all adapter 0), "uniform", "zipf" (Zipf s=1.1),
    "sorted_zipf" (zipf then sorted). A fraction ``none_frac`` of tokens,
    drawn independently, is set to -1 (no adapter)."""
    if kind == "distinct":
        ids = rng.permutation(T).astype(np.int32) % max(n_adapters, 1)
    elif kind == "identical":
        ids = np.zeros(T, np.int32)
    elif kind == "uniform":
        ids = rng.integers(0, n_adapters, size=T, dtype=np.int32)
    elif kind == "zipf":
        ids = zipf_ids(rng, T, n_adapters)
    elif kind == "sorted_zipf":
        ids = np.sort(zipf_ids(rng, T, n_adapters))
    else:
        raise ValueError(kind)
    if none_frac > 0:
        ids = np.where(rng.random(T) < none_frac, -1, ids).astype(np.int32)
    return ids.astype(np.int32)


@dataclass
class LoraProblem:
    """One multi-tenant LoRA layer call (possibly several projections at once).

    x: bf16 [n_slices, T, h_in]; A: bf16 [n_slices, n_adapters, h_in, r_max];
    B: bf16 [n_slices, n_adapters, r_max, h_out]; y_in: bf16 [n_slices, T, h_out];
    ids: int32 [T]; ranks: int32 [n_adapters]; scales: fp32 [n_adapters];
    W: bf16 [n_slices, h_out, h_in] or None."""
    name: str
    x: np.ndarray
    A: np.ndarray
    B: np.ndarray
    ids: np.ndarray
    ranks: np.ndarray
    scales: np.ndarray
    y_in: np.ndarray
    W: np.ndarray | None = None
    meta: dict = field(default_factory=dict)

    @property
    def n_slices(self): return self.x.shape[0]
    @property
    def T(self): return self.x.shape[1]
    @property
    def h_in(self): return self.x.shape[2]
    @property
    def h_out(self): return self.B.shape[3]
    @property
    def n_adapters(self): return self.A.shape[1]
    @property
    def r_max(self): return self.A.shape[3]


def make_lora_problem(name: str, seed: int, T: int, n_adapters: int, h_in: int, h_out: int,
                      r_max: int, ids: np.ndarray | None = None, ids_kind: str = "uniform",
                      none_frac: float = 0.0, ranks: np.ndarray | None = None,
                      rank_choices=None, scale: float = 2.0, n_slices: int = 1,
                      with_W: bool = False, pad_value: int = BF16_NAN,
                      shared_x_slices: int = 1) -> LoraProblem:
    """Draw one problem. ``shared_x_slices`` > 1 makes the first that many
    slices use the same x (q/k/v projections of one hidden state)."""
    rng = np.random.default_rng(seed)
    if ids is None:
        ids = make_ids(ids_kind, rng, T, n_adapters, none_frac)
    ids = np.asarray(ids, np.int32)
    if ranks is None:
        if rank_choices is not None:
            ranks = rng.choice(np.asarray(rank_choices, np.int32), size=n_adapters).astype(np.int32)
        else:
            ranks = np.full(n_adapters, r_max, np.int32)
    ranks = np.asarray(ranks, np.int32)
    scales = np.full(n_adapters, scale, np.float32)
    xs = []
    for s in range(n_slices):
        if s > 0 and s < shared_x_slices:
            xs.append(xs[0])
        else:
            xs.append(normal_bf16(rng, (T, h_in)))
    x = np.stack(xs)
    A = np.full((n_slices, n_adapters, h_in, r_max), pad_value, np.uint16)
    B = np.full((n_slices, n_adapters, r_max, h_out), pad_value, np.uint16)
    for s in range(n_slices):
        for a in range(n_adapters):
            r = int(ranks[a])
            A[s, a, :, :r] = normal_bf16(rng, (h_in, r), std=1.0 / np.sqrt(h_in))
            B[s, a, :r, :] = normal_bf16(rng, (r, h_out), std=1.0 / np.sqrt(r))
    y_in = np.stack([normal_bf16(rng, (T, h_out)) for _ in range(n_slices)])
    W = None
    if with_W:
        W = np.stack([normal_bf16(rng, (h_out, h_in), std=1.0 / np.sqrt(h_in))
                      for _ in range(n_slices)])
    return LoraProblem(name, x, A, B, ids, ranks, scales, y_in, W,
                       meta=dict(seed=seed, ids_kind=ids_kind, none_frac=none_frac))


# --------------------------------------------------------------------------
# The named workloads (sizes and ids as stated for each).
# --------------------------------------------------------------------------

def sgmv_tiny(seed: int = 0) -> LoraProblem:
    """64 tokens in 4 contiguous segments of 16, 4 adapters, h_in=h_out=1024, r=16, s=2."""
    ids = np.repeat(np.arange(4, dtype=np.int32), 16)
    return make_lora_problem("sgmv_tiny", seed, T=64, n_adapters=4, h_in=1024, h_out=1024,
                             r_max=16, ids=ids, with_W=True)


def bgmv_decode(seed: int = 1, ids_kind: str = "distinct") -> LoraProblem:
    """36 decode tokens: 32 each with its own adapter (32 adapters) plus four
    with id -1, shuffled; h_in=h_out=4096 (Llama-2-7B q_proj), r=16, s=2.
    ids_kind="identical" gives Punica's Identical setting on the same shapes."""
    rng = np.random.default_rng(seed + 1000)
    if ids_kind == "distinct":
        ids = rng.permutation(np.concatenate([np.arange(32), np.full(4, -1)])).astype(np.int32)
    elif ids_kind == "identical":
        ids = np.zeros(36, np.int32)
    else:
        raise ValueError(ids_kind)
    return make_lora_problem("bgmv_decode", seed, T=36, n_adapters=32, h_in=4096, h_out=4096,
                             r_max=16, ids=ids)


def sgmv_prefill_lengths(seed: int = 2) -> np.ndarray:
    rng = np.random.default_rng(seed + 2000)
    return rng.integers(64, 512, size=8, endpoint=True).astype(np.int32)


def sgmv_prefill(seed: int = 2, lengths: np.ndarray | None = None) -> LoraProblem:
    """8 adapters, segment lengths uniform in [64, 512] (seeded), tokens sorted by
    adapter; h_in=4096, h_out=11008 (Llama-2-7B MLP up_proj), r=64, s=2."""
    if lengths is None:
        lengths = sgmv_prefill_lengths(seed)
    ids = np.repeat(np.arange(len(lengths), dtype=np.int32), lengths)
    return make_lora_problem("sgmv_prefill", seed, T=int(ids.shape[0]), n_adapters=len(lengths),
                             h_in=4096, h_out=11008, r_max=64, ids=ids)


def many_tenants(seed: int = 4, T: int = 512, n_adapters: int = 256, h: int = 5120,
                 ids_kind: str = "zipf") -> LoraProblem:
    """512 decode tokens, 256 adapters with ranks from {8,16,32,64}, Zipf(1.1)
    ids with 5% at -1, h_in=h_out=5120 (Llama-2-13B o_proj), pool padded to
    r_max=64, four projections (q/k/v/o) in one call; q/k/v share x."""
    return make_lora_problem("many_tenants", seed, T=T, n_adapters=n_adapters, h_in=h, h_out=h,
                             r_max=64, ids_kind=ids_kind, none_frac=0.05,
                             rank_choices=(8, 16, 32, 64), n_slices=4, shared_x_slices=3)


@dataclass
class Fp8Problem:
    """FP8 base GEMM + LoRA epilogue: x bf16 [M, K]; W bf16 [N, K] (quantised
    per output channel by whoever consumes it); a LoRA pool with r=16."""
    name: str
    x: np.ndarray
    W: np.ndarray
    A: np.ndarray
    B: np.ndarray
    ids: np.ndarray
    ranks: np.ndarray
    scales: np.ndarray
    meta: dict = field(default_factory=dict)

    @property
    def M(self): return self.x.shape[0]
    @property
    def K(self): return self.x.shape[1]
    @property
    def N(self): return self.W.shape[0]


def fp8_problem(M: int, K: int = 8192, N: int = 28672, n_adapters: int = 16, r: int = 16,
                seed: int = 3, ids_kind: str = "zipf", none_frac: float = 0.0,
                rank_choices=None, pad_value: int = BF16_NAN, W: np.ndarray | None = None
                ) -> Fp8Problem:
    """M decode tokens, K=8192, N=28672 (Llama-2-70B-like up_proj), 16 adapters
    of rank 16, Zipf(1.1) ids, s=2. W ~ N(0, 1/K) in bf16 before quantisation."""
    rng = np.random.default_rng(seed)
    ids = make_ids(ids_kind, rng, M, n_adapters, none_frac)
    x = normal_bf16(rng, (M, K))
    if rank_choices is not None:
        ranks = rng.choice(np.asarray(rank_choices, np.int32), size=n_adapters).astype(np.int32)
    else:
        ranks = np.full(n_adapters, r, np.int32)
    A = np.full((n_adapters, K, r), pad_value, np.uint16)
    B = np.full((n_adapters, r, N), pad_value, np.uint16)
    for a in range(n_adapters):
        ra = int(ranks[a])
        A[a, :, :ra] = normal_bf16(rng, (K, ra), std=1.0 / np.sqrt(K))
        B[a, :ra, :] = normal_bf16(rng, (ra, N), std=1.0 / np.sqrt(ra))
    if W is None:
        W = weight_bf16(N, K, seed=seed + 7000)
    scales = np.full(n_adapters, 2.0, np.float32)
    return Fp8Problem(f"fp8_gemm_lora_M{M}", x, W, A, B, ids, ranks, scales,
                      meta=dict(seed=seed))


def weight_bf16(N: int, K: int, seed: int) -> np.ndarray:
    """Base weight W [N, K] ~ N(0, 1/K), bf16 bits; drawn in row blocks to bound memory."""
    rng = np.random.default_rng(seed)
    out = np.empty((N, K), np.uint16)
    step = max(1, (1 << 24) // K)
    for n0 in range(0, N, step):
        n1 = min(N, n0 + step)
        out[n0:n1] = normal_bf16(rng, (n1 - n0, K), std=1.0 / np.sqrt(K))
    return out
