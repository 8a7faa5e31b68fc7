"""One rank of the multi-process CPU tests of block_sparse_attention_coarse_b200.shard.

Run as `python tests/shard_worker.py RANK WORLD PORT OUTDIR`.  Joins a gloo
process group on 127.0.0.1, builds the same seeded inputs on every rank and
runs (1) the sequence<->head all-to-all round trip, (2) sequence-sharded
ISA, without and with the decoupled RoPE, and (3) head-sharded ISA, with
the fp64 oracle as the per-head computation; writes this rank's results to
OUTDIR/rank{RANK}.npz.
"""
import datetime
import os
import sys

import numpy as np
import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle as O  # noqa: E402
from block_sparse_attention_coarse_b200 import shard  # noqa: E402

B, H, D, L_SRC, L_CTX, BLOCK = 1, 4, 16, 40, 24, 8


def inputs():
    g = np.random.default_rng(123)
    L = L_SRC + L_CTX
    return [torch.from_numpy(g.normal(size=(B, H, L, D))) for _ in range(3)]


def oracle_compute(rope_base=None):
    """Per-head computation for the sharding helpers: the oracle's forward,
    after its decoupled RoPE of Q and K when rope_base is given."""
    p = O.Params(D=D, L_src=L_SRC, L_ctx=L_CTX, block=BLOCK, alpha_s=0.5, alpha_f=0.5, alpha_ns=0.25)

    def run(q, k, v, b, h):
        q, k, v = (t.numpy().reshape(b, h, -1, D) for t in (q, k, v))
        if rope_base is not None:
            q, k = O.rope_decoupled(q, L_SRC, L_CTX, rope_base), O.rope_decoupled(k, L_SRC, L_CTX, rope_base)
        out, _, _ = O.isa_forward(q, k, v, p)
        return torch.from_numpy(out)
    return run


class _P:
    """Shape parameters the sharding helpers read (the CUDA Params carries the same fields)."""
    D, L_src, L_ctx, block, alpha_s, alpha_f, alpha_ns, scale = D, L_SRC, L_CTX, BLOCK, 0.5, 0.5, 0.25, 0.0


def main():
    rank, world, port, outdir = int(sys.argv[1]), int(sys.argv[2]), sys.argv[3], sys.argv[4]
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    q, k, v = inputs()
    L = L_SRC + L_CTX
    Lc = L // world
    chunk = lambda t: t[:, :, rank * Lc:(rank + 1) * Lc].contiguous()
    # (1) round trip and layout of the regrouping
    heads = shard.seq_to_heads(chunk(q))
    back = shard.heads_to_seq(heads)
    # (2) sequence-sharded ISA
    out_seq = shard.isa_attention_seq_sharded(chunk(q), chunk(k), chunk(v), _P, compute=oracle_compute())
    out_rope = shard.isa_attention_seq_sharded(chunk(q), chunk(k), chunk(v), _P, compute=oracle_compute(500.0))
    # (3) head-sharded ISA on full inputs
    out_heads, (lo, hi) = shard.isa_attention_heads(q, k, v, _P, rank, world, compute=oracle_compute())
    np.savez(os.path.join(outdir, f"rank{rank}.npz"), heads=heads.numpy(), back=back.numpy(),
             out_seq=out_seq.numpy(), out_rope=out_rope.numpy(), out_heads=out_heads.numpy(), lo=lo, hi=hi)
    dist.barrier()
    dist.destroy_process_group()


if __name__ == "__main__":
    main()
