"""Multi-GPU ISA: one process per GPU, heads split across ranks.

ISA is independent per (batch, head): planning, selection, split and
attention never mix heads (summary card, "Method steps in detail": every
step is per head).  So

* head sharding needs no data-path collective: rank r runs the whole path on
  its contiguous slice of the B*H heads (`head_range`, `isa_attention_heads`);
* inputs that arrive sharded along the sequence (rank r holds tokens
  [r*L/N, (r+1)*L/N) of every head, as sequence-parallel training lays them
  out) are first regrouped by one all-to-all into full sequences of H/N heads
  per rank, and the output is sent back the same way (`seq_to_heads`,
  `heads_to_seq`, `isa_attention_seq_sharded`).  The all-to-all runs through
  torch.distributed (NCCL over NVLink on GPUs; gloo in the CPU tests); the
  pages do not say how the method composes with sequence parallelism, this is
  the standard regrouping.

The per-head computation is a parameter (`compute(q, k, v, B, H) -> out`) so
that the data movement can be tested on any backend; it defaults to the CUDA
path (`isa_attention`).
"""
from __future__ import annotations

from typing import Callable, Optional, Tuple

import torch
import torch.distributed as dist

Compute = Callable[[torch.Tensor, torch.Tensor, torch.Tensor, int, int], torch.Tensor]


def head_range(n_heads: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous, balanced slice [lo, hi) of n_heads for `rank` of `world`
    (the first n_heads % world ranks take one head more)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"bad rank {rank} of world {world}")
    base, extra = divmod(n_heads, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def _cuda_compute(p_template, rope_base: Optional[float] = None) -> Compute:
    from . import isa_attention, make_params

    def run(q, k, v, B, H):
        p = make_params(B, H, p_template.D, p_template.L_src, p_template.L_ctx, p_template.block,
                        p_template.alpha_s, p_template.alpha_f, p_template.alpha_ns, p_template.scale)
        return isa_attention(q, k, v, p, rope_base=rope_base)
    return run


def isa_attention_heads(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, p, rank: int, world: int,
                        compute: Optional[Compute] = None) -> Tuple[torch.Tensor, Tuple[int, int]]:
    """Head-sharded ISA on full [B, H, L, D] inputs: this rank's heads only.
    Returns (out [n_local, L, D], (lo, hi)) for the flattened heads
    lo..hi-1 of B*H; no communication."""
    B, H, L, D = q.shape
    lo, hi = head_range(B * H, rank, world)
    run = compute or _cuda_compute(p)
    if hi == lo:
        return q.new_empty((0, L, D)), (lo, hi)
    sl = lambda t: t.reshape(B * H, L, D)[lo:hi].unsqueeze(0).contiguous()
    out = run(sl(q), sl(k), sl(v), 1, hi - lo)
    return out.reshape(hi - lo, L, D), (lo, hi)


def seq_to_heads(x: torch.Tensor, group=None) -> torch.Tensor:
    """[B, H, L/N, D] (this rank's sequence chunk of every head) ->
    [B, H/N, L, D] (full sequences of this rank's H/N heads)."""
    world = dist.get_world_size(group)
    B, H, Lc, D = x.shape
    if H % world:
        raise ValueError(f"H={H} is not divisible by the world size {world}")
    send = x.reshape(B, world, H // world, Lc, D).permute(1, 0, 2, 3, 4).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)          # recv[i] = chunk i of my heads
    return recv.permute(1, 2, 0, 3, 4).reshape(B, H // world, world * Lc, D).contiguous()


def heads_to_seq(y: torch.Tensor, group=None) -> torch.Tensor:
    """Inverse of `seq_to_heads`: [B, H/N, L, D] -> [B, H, L/N, D]."""
    world = dist.get_world_size(group)
    B, Hl, L, D = y.shape
    if L % world:
        raise ValueError(f"L={L} is not divisible by the world size {world}")
    Lc = L // world
    send = y.reshape(B, Hl, world, Lc, D).permute(2, 0, 1, 3, 4).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)          # recv[i] = my chunk of rank i's heads
    return recv.permute(1, 0, 2, 3, 4).reshape(B, world * Hl, Lc, D).contiguous()


def isa_attention_seq_sharded(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, p, group=None,
                              compute: Optional[Compute] = None, rope_base: Optional[float] = None) -> torch.Tensor:
    """ISA on sequence-sharded inputs [B, H, L/N, D] (rank r holds tokens
    [r*L/N, (r+1)*L/N) of every head, L = p.L_src + p.L_ctx): all-to-all to
    full sequences of H/N heads, ISA per head (after the decoupled RoPE when
    `rope_base` is given, which needs the full sequence's positions), and
    all-to-all back.  Returns this rank's [B, H, L/N, D] output chunk."""
    B, H, Lc, D = q.shape
    world = dist.get_world_size(group)
    if world * Lc != p.L_src + p.L_ctx:
        raise ValueError("sequence chunks do not add up to L_src + L_ctx")
    qh, kh, vh = (seq_to_heads(t, group) for t in (q, k, v))
    run = compute or _cuda_compute(p, rope_base)
    out = run(qh, kh, vh, B, H // world)
    return heads_to_seq(out.reshape(B, H // world, world * Lc, D), group)
