"""Seeded synthetic Q/K/V for the ISA forward pass.

This module is the one piece shared by the CPU oracle side and the CUDA side
of the tests and the bench: it draws the inputs, rounds them to bfloat16 and
hands out the same bits to both.  It holds none of the method's arithmetic
(no pooling, no scores, no selection) -- only random numbers and shapes.

Shapes follow the workloads of "LIVEditor-14B: Lightning Unified Video Editing
via In-Context Sparse Attention" (paper.rainbus.top summary, Fig. 2 latency
sweep at 23768 tokens and 4K-131K tokens; techwalker.com retelling, Fig. 2 at
131072 tokens / head dim 128; model card, 65K tokens).  The pages measure on
Wan-2.2 video latents that are not available here, so a clustered generator
stands in for them: tokens of one 64-token cluster share a centroid, with a
per-cluster noise level, so that in-block variance (the quantity the Taylor
error is said to grow with) varies across blocks.

Layout: every tensor is [B, H, L, D] with L = L_src + L_ctx, the context
tokens appended after the source tokens.  bfloat16 values travel as numpy
uint16 bit patterns (``*_bits``); ``bf16_to_f64`` turns them into the exact
float64 values the oracle works on.

Random streams: each (tensor, batch*H + head) pair draws from its own
``numpy.random.PCG64`` seeded with the entropy list ``[seed, stream, bh]``,
stream 0/1/2 = Q/K/V, 3 = per-cluster noise level, 4 = per-head Q temperature,
5 = the upstream gradient dout of the backward (standard normal per element).
A head can therefore be regenerated on its own, which is how the tests fetch
oracle inputs for sampled heads of the large workloads.
"""
from __future__ import annotations

import concurrent.futures as _cf
import dataclasses
import math
import os
from typing import Dict, List, Optional, Tuple

import numpy as np

CLUSTER = 64          # tokens per generator cluster, also when the block is 32
CTX_CENTROID_SCALE = 0.5


@dataclasses.dataclass(frozen=True)
class Workload:
    """One ISA forward problem: shapes, ratios and the input recipe."""
    name: str
    B: int
    H: int
    D: int
    L_src: int
    L_ctx: int
    block: int = 64
    alpha_s: float = 0.125
    alpha_f: float = 0.5
    alpha_ns: float = 0.0625
    kind: str = "clustered"     # "iid" or "clustered"
    seed: int = 0

    @property
    def L(self) -> int:
        return self.L_src + self.L_ctx

    @property
    def BH(self) -> int:
        return self.B * self.H

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def named_workloads() -> Dict[str, Workload]:
    """The five workload families of the ISA forward benchmark.

    tiny     : i.i.d. N(0,1), B=1 H=2 D=64, 1024 + 1024 tokens, b=64.
    mid      : clustered, B=1 H=8 D=128, 11884 + 11884 tokens (23768, the
               Fig. 2 length), b=64.
    dit14b   : clustered, B=2 (a CFG pair) H=40 D=128, 16384 + 16384 tokens.
    long65k  : clustered, B=1 H=40 D=128, 32768 + 32768 tokens, b=64 (the
               b=32 and alpha_f variants are built with ``replace``).
    sweep*   : clustered, B=1 H=40, total length 4096..131072 split evenly;
               at 131072 tokens, D=128 also the ratio grid alpha_s in
               {0.0625, 0.125, 0.25} x alpha_ns in {0.03125, 0.0625, 0.125}.
    """
    w = {
        "tiny": Workload("tiny", 1, 2, 64, 1024, 1024, kind="iid", seed=0),
        "mid": Workload("mid", 1, 8, 128, 11884, 11884, seed=1000),
        "dit14b": Workload("dit14b", 2, 40, 128, 16384, 16384, seed=2000),
        "long65k": Workload("long65k", 1, 40, 128, 32768, 32768, seed=3000),
        "long65k_b32": Workload("long65k_b32", 1, 40, 128, 32768, 32768, block=32, seed=3001),
        "long65k_af025": Workload("long65k_af025", 1, 40, 128, 32768, 32768, alpha_f=0.25, seed=3002),
        "long65k_af075": Workload("long65k_af075", 1, 40, 128, 32768, 32768, alpha_f=0.75, seed=3003),
    }
    point = 0
    for D in (64, 128):
        for total in (4096, 16384, 65536, 131072):
            name = f"sweep_L{total}_D{D}"
            w[name] = Workload(name, 1, 40, D, total // 2, total // 2, seed=4000 + point)
            point += 1
    # the ratio grid at 131072 tokens, D=128: alpha_s in {0.0625, 0.125, 0.25}
    # x alpha_ns in {0.03125, 0.0625, 0.125} (the centre point is
    # sweep_L131072_D128); the points on the centre's row and column first,
    # then the four corners
    for tag, kw in (("as0625", dict(alpha_s=0.0625)), ("as25", dict(alpha_s=0.25)),
                    ("ans03125", dict(alpha_ns=0.03125)), ("ans125", dict(alpha_ns=0.125)),
                    ("as0625_ans03125", dict(alpha_s=0.0625, alpha_ns=0.03125)),
                    ("as0625_ans125", dict(alpha_s=0.0625, alpha_ns=0.125)),
                    ("as25_ans03125", dict(alpha_s=0.25, alpha_ns=0.03125)),
                    ("as25_ans125", dict(alpha_s=0.25, alpha_ns=0.125))):
        name = f"sweep_L131072_D128_{tag}"
        w[name] = Workload(name, 1, 40, 128, 65536, 65536, seed=4000 + point, **kw)
        point += 1
    return w


# ----------------------------------------------------------------------------
# bfloat16 bit handling (round to nearest even; inputs are finite)
# ----------------------------------------------------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return bf16_to_f32(bits).astype(np.float64)


# ----------------------------------------------------------------------------
# generators
# ----------------------------------------------------------------------------

def _rng(seed: int, stream: int, bh: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([int(seed), int(stream), int(bh)]))


def _cluster_ids(L_src: int, L_ctx: int) -> Tuple[np.ndarray, np.ndarray, int]:
    """Cluster index of every token and whether it is a context token.

    Clusters are laid out per segment: source tokens [0, L_src) form
    ceil(L_src/64) clusters, context tokens form ceil(L_ctx/64) more, each
    segment's last cluster possibly short.
    """
    n_src = -(-L_src // CLUSTER)
    n_ctx = -(-L_ctx // CLUSTER)
    src = np.arange(L_src) // CLUSTER
    ctx = n_src + np.arange(L_ctx) // CLUSTER
    cid = np.concatenate([src, ctx])
    is_ctx = np.concatenate([np.zeros(L_src, bool), np.ones(L_ctx, bool)])
    return cid, is_ctx, n_src + n_ctx


def head_f32(w: Workload, bh: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """float32 Q, K, V of one head (index bh = b*H + h), before bf16 rounding."""
    L, D = w.L, w.D
    if w.kind == "iid":
        return tuple(_rng(w.seed, s, bh).standard_normal((L, D), dtype=np.float32) for s in range(3))
    if w.kind != "clustered":
        raise ValueError(f"unknown generator kind {w.kind!r}")
    cid, is_ctx, n_clusters = _cluster_ids(w.L_src, w.L_ctx)
    sigma = _rng(w.seed, 3, bh).uniform(0.05, 1.0, size=n_clusters).astype(np.float32)
    tau = np.float32(_rng(w.seed, 4, bh).uniform(0.5, 2.0))
    cscale = np.where(is_ctx, np.float32(CTX_CENTROID_SCALE), np.float32(1.0)).astype(np.float32)
    out = []
    for s in range(3):
        g = _rng(w.seed, s, bh)
        centroids = g.standard_normal((n_clusters, D), dtype=np.float32)
        noise = g.standard_normal((L, D), dtype=np.float32)
        x = centroids[cid] * cscale[:, None] + sigma[cid][:, None] * noise
        if s == 0:
            x = x * tau
        out.append(x.astype(np.float32))
    return tuple(out)


def head_bits(w: Workload, bh: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """bf16 bit patterns of Q, K, V of one head, each [L, D] uint16."""
    return tuple(f32_to_bf16_bits(x) for x in head_f32(w, bh))


def generate_bits(w: Workload, heads: Optional[List[int]] = None,
                  threads: Optional[int] = None) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """bf16 bits of Q, K, V.

    With ``heads=None`` returns full [B, H, L, D] uint16 arrays; otherwise
    [len(heads), L, D] arrays for the listed bh indices.  Heads are drawn in
    parallel threads (numpy releases the GIL while drawing).
    """
    hs = list(range(w.BH)) if heads is None else list(heads)
    shape = (len(hs), w.L, w.D)
    q = np.empty(shape, np.uint16)
    k = np.empty(shape, np.uint16)
    v = np.empty(shape, np.uint16)

    def one(i: int) -> None:
        q[i], k[i], v[i] = head_bits(w, hs[i])

    nthreads = threads or min(len(hs), max(1, os.cpu_count() or 1))
    if nthreads <= 1 or len(hs) <= 1:
        for i in range(len(hs)):
            one(i)
    else:
        with _cf.ThreadPoolExecutor(nthreads) as ex:
            list(ex.map(one, range(len(hs))))
    if heads is None:
        return tuple(a.reshape(w.B, w.H, w.L, w.D) for a in (q, k, v))
    return q, k, v


def dout_head_bits(w: Workload, bh: int) -> np.ndarray:
    """bf16 bits of the upstream gradient dout [L, D] of head bh: independent
    standard normal values (the loss is sum(dout * out))."""
    g = _rng(w.seed, 5, bh)
    return f32_to_bf16_bits(g.standard_normal((w.L, w.D), dtype=np.float32))


def generate_dout_bits(w: Workload, heads: Optional[List[int]] = None, threads: Optional[int] = None) -> np.ndarray:
    """dout bits, [B, H, L, D] (heads=None) or [len(heads), L, D]."""
    hs = list(range(w.BH)) if heads is None else list(heads)
    out = np.empty((len(hs), w.L, w.D), np.uint16)
    with _cf.ThreadPoolExecutor(max_workers=max(1, min(len(hs), threads or os.cpu_count() or 1))) as ex:
        for i, x in zip(range(len(hs)), ex.map(lambda h: dout_head_bits(w, h), hs)):
            out[i] = x
    return out.reshape(w.B, w.H, w.L, w.D) if heads is None else out


def sample_blocks(w: Workload, n_heads: int, n_blocks: int, seed: int = 7) -> List[Tuple[int, int]]:
    """Seeded sample of (bh, query-block) pairs for spot checks at full size."""
    T = -(-w.L_src // w.block) + -(-w.L_ctx // w.block)
    g = np.random.Generator(np.random.PCG64([seed, w.BH, T]))
    heads = sorted(g.choice(w.BH, size=min(n_heads, w.BH), replace=False).tolist())
    out = []
    for bh in heads:
        for blk in sorted(g.choice(T, size=min(n_blocks, T), replace=False).tolist()):
            out.append((bh, blk))
    return out


def flops_dense(w: Workload) -> float:
    """Dense attention work, 4*D*L*L per head (QK^T and PV, 2 flops per MAC)."""
    return 4.0 * w.D * w.L * w.L * w.BH


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


__all__ = [
    "Workload", "named_workloads", "f32_to_bf16_bits", "bf16_to_f32", "bf16_to_f64",
    "head_f32", "head_bits", "generate_bits", "dout_head_bits", "generate_dout_bits", "sample_blocks",
    "flops_dense", "ceil_div",
    "CLUSTER",
]
