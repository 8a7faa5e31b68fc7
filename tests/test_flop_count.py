"""The executed-work count behind the bench's TFLOP/s (`bench.executed_flops`).

Convention (the ISA forward metric): 4*D FLOPs per (valid query token, key
column) pair, where an exactly attended key token is one column and a pooled
block is one column, plus 2*T*T*D per head for the coarse scores.  Checked
against a block-by-block loop over oracle plans with partial blocks, and
against the closed form at the bench shape, where every block is full so
the count does not depend on which blocks the plan chose."""
import numpy as np
import torch

import block_sparse_attention_coarse_b200 as isa
from bench import executed_flops
import oracle as O
from parity import oracle_params
from workloads import Workload, bf16_to_f64, generate_bits


def fake_view(plans, n_exact):
    """The plan-view fields executed_flops reads, from oracle plans."""
    pl0 = plans[0]
    return {"T_src": pl0.T_src, "T": pl0.T, "T_kv": len(pl0.kept), "n_exact": n_exact,
            "kept": torch.tensor(np.stack([p.kept for p in plans])),
            "sharp_ids": torch.tensor(np.stack([p.sharp for p in plans])),
            "flat_ids": torch.tensor(np.stack([p.flat for p in plans])),
            "exact": torch.tensor(np.stack([p.exact for p in plans]))}


def block_loop_count(plans, D):
    total = 0
    for pl in plans:
        n = pl.counts
        flat_pos = {int(b): r for r, b in enumerate(pl.flat)}
        for i in range(pl.T):
            if i in flat_pos:
                ex = pl.kept[pl.exact[flat_pos[i]]]
                cols = sum(int(n[j]) for j in ex) + (len(pl.kept) - len(ex))
            else:
                cols = sum(int(n[j]) for j in pl.kept)
            total += 4 * D * int(n[i]) * cols
        total += 2 * pl.T * pl.T * D
    return total


def test_count_matches_a_block_loop_with_partial_blocks():
    w = Workload("flops", 1, 3, 64, 300, 170, block=32, alpha_s=0.4, alpha_f=0.5, alpha_ns=0.3, seed=21)
    qb, kb, vb = (x.reshape(w.BH, w.L, w.D) for x in generate_bits(w))
    op = oracle_params(w)
    plans = [O.plan_head(bf16_to_f64(qb[h]), bf16_to_f64(kb[h]), bf16_to_f64(vb[h]), op) for h in range(w.BH)]
    assert any(c != w.block for c in plans[0].counts)
    p = isa.make_params(w.B, w.H, w.D, w.L_src, w.L_ctx, w.block, w.alpha_s, w.alpha_f, w.alpha_ns)
    got = executed_flops(p, fake_view(plans, plans[0].exact.shape[1]))
    assert got == float(block_loop_count(plans, w.D))


def test_count_at_the_bench_shape_is_the_closed_form():
    """B=2, H=40, 16384 + 16384 tokens, D=128, b=64: T = 512 blocks, 288
    kept, 256 sharp and 256 flat blocks, 18 exact blocks per flat block.
    Per head: sharp 256*64 * 288*64 pairs, flat 256*64 * (18*64 + 270)
    pairs, times 4*128, plus 2*512^2*128."""
    rng = np.random.default_rng(5)
    plans = []
    for _ in range(80):
        kept = np.concatenate([np.arange(256), 256 + np.sort(rng.choice(256, 32, replace=False))])
        perm = rng.permutation(512)
        sharp, flat = np.sort(perm[:256]), np.sort(perm[256:])
        exact = np.stack([np.sort(rng.choice(288, 18, replace=False)) for _ in range(256)])
        plans.append(O.HeadPlan(np.arange(512) * 64, np.full(512, 64), 256, 256, None, None, None, None, None,
                                None, kept, None, sharp, flat, exact))
    p = isa.make_params(2, 40, 128, 16384, 16384)
    per_head = (256 * 64 * 288 * 64 + 256 * 64 * (18 * 64 + 270)) * 4 * 128 + 2 * 512 * 512 * 128
    assert executed_flops(p, fake_view(plans, 18)) == float(80 * per_head) == 13.32916256768e12
