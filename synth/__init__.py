"""Seeded synthetic inputs for the MXFP8 routed-experts MLP.

This module holds no part of the method's arithmetic: it only draws random
numbers and builds routings.  Both the CPU oracle and the CUDA path read the
same arrays from here.

Workloads (shapes and distributions follow the routed-experts MLP of the
torchtitan "fully-fused grouped-GEMM MXFP8 plan" page, section "What it adds",
and the SwiGLU-boundary page, section "Summary"):

* ``tiny``      E=4, D=F=256, 512 tokens, top-2 uniform, pad 128
* ``swiglu``    h13 [16384, 2*4096] ~N(0,1) with 1 % outliers x100
* ``cast``      x [8192, 7168] ~N(0,1) (the A2E transport payload)
* ``dsv3_16b``  E=64, D=2048, F=1408, 8192 tokens, top-6, Zipf(1.1), pad 256,
                two experts never routed
* ``dsv3``      E=256, D=7168, F=2048, 16384 tokens, top-8, Zipf(1.0), pad 256,
                0.1 % activation outliers x50, weights ~N(0, 0.006)

Routing recipe: each token draws ``top_k`` distinct experts without
replacement from the popularity vector; per-expert counts are padded up to
``pad_multiple`` (a zero count stays zero); offsets are the exclusive prefix
sum; token rows are gathered expert-major (tokens in ascending order inside a
segment) and pad rows are zero.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch


@dataclasses.dataclass
class Routing:
    """Expert-major padded layout of routed token rows."""

    counts: np.ndarray        # [E] real rows per expert
    padded: np.ndarray        # [E] padded rows per expert
    offsets: np.ndarray       # [E+1] int32 exclusive prefix sum of ``padded``
    src_token: np.ndarray     # [M] source token of each row, -1 for pad rows
    M: int                    # rows of the buffer (= offsets[-1])
    R: int                    # real rows (tokens * top_k)
    topk: np.ndarray | None = None   # [T, k] drawn expert ids (None for explicit counts)


@dataclasses.dataclass
class Spec:
    name: str
    E: int
    D: int
    F: int
    tokens: int
    top_k: int
    pad: int
    zipf_s: float | None      # None = uniform popularity
    zero_experts: int         # experts forced to popularity 0
    w_std: float
    x_outlier_frac: float = 0.0
    x_outlier_mul: float = 1.0
    dy_std: float = 1e-2


SPECS = {
    "tiny": Spec("tiny", 4, 256, 256, 512, 2, 128, None, 0, 0.02),
    "dsv3_16b": Spec("dsv3_16b", 64, 2048, 1408, 8192, 6, 256, 1.1, 2, 0.02),
    "dsv3": Spec("dsv3", 256, 7168, 2048, 16384, 8, 256, 1.0, 0, 0.006,
                 x_outlier_frac=1e-3, x_outlier_mul=50.0),
    # 16 experts of the DSv3-scale layer (same D, F, routing law, padding and
    # per-expert load): a few GB on the device, for profiling its kernels
    "dsv3_slice": Spec("dsv3_slice", 16, 7168, 2048, 1024, 8, 256, 1.0, 0, 0.006,
                       x_outlier_frac=1e-3, x_outlier_mul=50.0),
}


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def to_bf16(a: np.ndarray) -> torch.Tensor:
    """float32 numpy array -> bf16 torch tensor (CPU)."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def popularity(spec: Spec, g: np.random.Generator) -> np.ndarray:
    E = spec.E
    if spec.zipf_s is None:
        p = np.ones(E)
    else:
        perm = g.permutation(E)
        rank = np.empty(E)
        rank[perm] = np.arange(1, E + 1)
        p = rank ** (-spec.zipf_s)
    if spec.zero_experts:
        zero = g.choice(E, size=spec.zero_experts, replace=False)
        p[zero] = 0.0
    return p / p.sum()


def make_routing(spec: Spec, seed: int = 0, counts_override=None) -> Routing:
    """Draw a routing and lay it out expert-major with padding."""
    g = rng(seed)
    E, T, k = spec.E, spec.tokens, spec.top_k
    if counts_override is not None:
        # explicit per-expert real counts (tests of edge cases); tokens are
        # assigned round-robin so that every row has a source token.
        counts = np.asarray(counts_override, dtype=np.int64)
        choice = None
        lists = []
        t = 0
        for e in range(E):
            lists.append(np.arange(t, t + counts[e]) % max(T, 1))
            t += counts[e]
    else:
        p = popularity(spec, g)
        # top-k distinct experts per token: Gumbel-top-k == sampling without
        # replacement proportionally to p.
        with np.errstate(divide="ignore"):
            logp = np.log(p)
        gumbel = g.gumbel(size=(T, E))
        keys = logp[None, :] + gumbel
        choice = np.argsort(-keys, axis=1)[:, :k]          # [T, k]
        tok = np.repeat(np.arange(T), k)
        exp = choice.reshape(-1)
        order = np.lexsort((tok, exp))                      # expert-major, token order inside
        tok, exp = tok[order], exp[order]
        counts = np.bincount(exp, minlength=E).astype(np.int64)
        lists = np.split(tok, np.cumsum(counts)[:-1])
    pad = spec.pad
    padded = ((counts + pad - 1) // pad) * pad
    offsets = np.zeros(E + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(padded)
    M = int(offsets[-1])
    src = -np.ones(M, dtype=np.int64)
    for e in range(E):
        o = offsets[e]
        src[o:o + counts[e]] = lists[e]
    return Routing(counts=counts, padded=padded, offsets=offsets, src_token=src,
                   M=M, R=int(counts.sum()),
                   topk=None if choice is None else choice.astype(np.int32))


def normal(g: np.random.Generator, shape, std=1.0, outlier_frac=0.0, outlier_mul=1.0):
    a = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    if outlier_frac > 0:
        n = a.size
        k = int(round(n * outlier_frac))
        idx = g.choice(n, size=k, replace=False)
        a.reshape(-1)[idx] *= np.float32(outlier_mul)
    return a


@dataclasses.dataclass
class MoEInputs:
    spec: Spec
    routing: Routing
    x: torch.Tensor          # [M, D] bf16, pad rows zero
    w13: torch.Tensor        # [E, 2F, D] bf16, rows 0..F-1 gate (w1), F..2F-1 up (w3)
    w2: torch.Tensor         # [E, D, F] bf16
    dy: torch.Tensor         # [M, D] bf16, pad rows zero
    x_tok: torch.Tensor | None = None   # [tokens, D] bf16 token rows before routing (device draw only)


def make_moe_inputs(spec: Spec | str, seed: int = 0, counts_override=None,
                    with_dy: bool = True) -> MoEInputs:
    """Token activations, weights and upstream gradient for one MoE layer (CPU)."""
    if isinstance(spec, str):
        spec = SPECS[spec]
    routing = make_routing(spec, seed, counts_override)
    g = rng(seed + 1)
    tok = normal(g, (spec.tokens, spec.D), 1.0, spec.x_outlier_frac, spec.x_outlier_mul)
    x = np.zeros((routing.M, spec.D), dtype=np.float32)
    real = routing.src_token >= 0
    x[real] = tok[routing.src_token[real]]
    w13 = normal(g, (spec.E, 2 * spec.F, spec.D), spec.w_std)
    w2 = normal(g, (spec.E, spec.D, spec.F), spec.w_std)
    dy = np.zeros((routing.M, spec.D), dtype=np.float32)
    if with_dy:
        dy[real] = normal(g, (int(real.sum()), spec.D), spec.dy_std)
    return MoEInputs(spec, routing, to_bf16(x), to_bf16(w13), to_bf16(w2), to_bf16(dy))


def router_weights(T: int, k: int, seed: int = 0) -> np.ndarray:
    """[T, k] float32 combine weights: a softmax over k N(0,1) logits per token."""
    g = rng(seed + 7)
    z = g.standard_normal(size=(T, k))
    w = np.exp(z - z.max(axis=1, keepdims=True))
    return (w / w.sum(axis=1, keepdims=True)).astype(np.float32)


def topk_ids(T: int, k: int, E: int, seed: int = 0, zipf_s: float | None = None) -> np.ndarray:
    """[T, k] int32 distinct expert ids per token (uniform or Zipf popularity)."""
    spec = Spec("route", E, 32, 32, T, k, 32, zipf_s, 0, 1.0)
    g = rng(seed)
    p = popularity(spec, g)
    with np.errstate(divide="ignore"):
        keys = np.log(p)[None, :] + g.gumbel(size=(T, E))
    return np.argsort(-keys, axis=1)[:, :k].astype(np.int32)


def make_swiglu_input(rows: int = 16384, F: int = 4096, seed: int = 0) -> torch.Tensor:
    """h13 [rows, 2F] bf16 ~N(0,1) with 1 % of elements scaled by 100."""
    g = rng(seed)
    return to_bf16(normal(g, (rows, 2 * F), 1.0, 0.01, 100.0))


def make_cast_input(rows: int = 8192, cols: int = 7168, seed: int = 0) -> torch.Tensor:
    """Transport payload x [rows, cols] bf16 ~N(0,1)."""
    g = rng(seed)
    return to_bf16(normal(g, (rows, cols)))


def device_moe_inputs(spec: Spec | str, seed: int = 0, device="cuda"):
    """Full-size inputs drawn on the device with a seeded torch generator.

    Used where the host draw would be slow (the E=256, D=7168 layer holds
    11 G weight elements).  The routing itself is still drawn on the host.
    """
    if isinstance(spec, str):
        spec = SPECS[spec]
    routing = make_routing(spec, seed)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed + 1)
    D, F, E = spec.D, spec.F, spec.E
    tok = torch.randn(spec.tokens, D, generator=gen, device=device, dtype=torch.float32)
    if spec.x_outlier_frac > 0:
        n = tok.numel()
        k = int(round(n * spec.x_outlier_frac))
        idx = torch.randperm(n, generator=gen, device=device)[:k]
        tok.view(-1)[idx] *= spec.x_outlier_mul
    src = torch.from_numpy(routing.src_token).to(device)
    real = src >= 0
    x = torch.zeros(routing.M, D, device=device, dtype=torch.bfloat16)
    x_tok = tok.to(torch.bfloat16)
    x[real] = x_tok[src[real]]
    del tok
    w13 = torch.empty(E, 2 * F, D, device=device, dtype=torch.bfloat16)
    w2 = torch.empty(E, D, F, device=device, dtype=torch.bfloat16)
    for e in range(E):   # per expert, to bound the fp32 temporary
        w13[e] = (torch.randn(2 * F, D, generator=gen, device=device) * spec.w_std).to(torch.bfloat16)
        w2[e] = (torch.randn(D, F, generator=gen, device=device) * spec.w_std).to(torch.bfloat16)
    dy = torch.zeros(routing.M, D, device=device, dtype=torch.bfloat16)
    nreal = int(real.sum())
    dy[real] = (torch.randn(nreal, D, generator=gen, device=device) * spec.dy_std).to(torch.bfloat16)
    return MoEInputs(spec, routing, x, w13, w2, dy, x_tok)
