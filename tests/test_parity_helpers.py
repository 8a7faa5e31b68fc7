"""The comparison helpers of the GPU parity tests (tests/parity.py) reject
what they must.  A helper that always agreed would make every GPU parity
test pass, so each rule is checked here on the CPU with planted
disagreements: a chosen set beyond the margin, wrong counts, a moved
context block, perturbed pooled means, a swapped sharp/flat pair, an exact
bitmap that disagrees with its list, and an output error in a sampled row."""
import numpy as np

import oracle as O
from parity import (MARGIN_EXACT, block_rows, check_head_plan, compare_outputs, energy_from_oracle,
                    oracle_params, plan_from_gpu, topk_agrees)
from workloads import Workload, bf16_to_f64, generate_bits


def test_topk_agrees_margin_rule():
    s = [5.0, 4.0, 3.0, 2.0, 1.0]
    assert topk_agrees(s, 2, [1, 0], 0.1) == (True, 0)
    assert not topk_agrees(s, 2, [0, 2], 0.1)[0]          # 4.0 is clearly in, 3.0 clearly out
    assert not topk_agrees(s, 2, [0], 0.1)[0]             # wrong count
    assert not topk_agrees(s, 2, [0, 0], 0.1)[0]          # duplicate
    assert not topk_agrees(s, 2, [0, 5], 0.1)[0]          # out of range
    assert topk_agrees(s, 0, [], 0.1) == (True, 0)
    assert topk_agrees(s, 5, [4, 3, 2, 1, 0], 0.1) == (True, 0)
    # a near tie at the boundary: either side is valid within the margin
    t = [5.0, 3.0005, 3.0, 1.0]
    assert topk_agrees(t, 2, [0, 2], 1e-3) == (True, 1)
    assert not topk_agrees(t, 2, [0, 2], 1e-4)[0]
    assert not topk_agrees(t, 2, [0, 3], 1e-3)[0]


def plan_and_view():
    w = Workload("helpers", 1, 1, 64, 300, 200, block=32, alpha_s=0.5, alpha_f=0.5, alpha_ns=0.25, seed=12)
    qb, kb, vb = (x.reshape(w.L, w.D) for x in generate_bits(w))
    pl = O.plan_head(bf16_to_f64(qb), bf16_to_f64(kb), bf16_to_f64(vb), oracle_params(w))
    words = (len(pl.kept) + 31) // 32
    bits = np.zeros((len(pl.flat), words), np.int64)
    for r, row in enumerate(pl.exact):
        for x in row:
            bits[r, x // 32] |= 1 << (x % 32)
    view = {"Qc": pl.Qc[None].copy(), "Kc": pl.Kc[None].copy(), "Vc": pl.Vc[None].copy(), "imp": pl.imp[None].copy(),
            "ctx_sel": pl.ctx_sel[None].copy(), "kept": pl.kept[None].copy(),
            "energy": energy_from_oracle(pl)[None].copy(), "sharp_ids": pl.sharp[None].copy(),
            "flat_ids": pl.flat[None].copy(), "exact": pl.exact[None].copy(), "exact_bits": bits[None]}
    return pl, view


def test_check_head_plan_accepts_the_oracle_plan():
    pl, view = plan_and_view()
    r = check_head_plan(pl, view, 0)
    assert not r.errors and r.ctx_equal and not r.split_moved and not r.exact_moved


def test_check_head_plan_rejects_planted_disagreements():
    pl, base = plan_and_view()

    def errors_after(change):
        view = {k: v.copy() for k, v in base.items()}
        change(view)
        return check_head_plan(pl, view, 0).errors

    # the lowest-importance context block in place of the highest
    lo, hi = int(np.argmin(pl.imp)), int(np.argmax(pl.imp))

    def move_ctx(v):
        sel = sorted((set(pl.ctx_sel.tolist()) - {hi}) | {lo})
        v["ctx_sel"][0] = sel
        v["kept"][0] = np.concatenate([np.arange(pl.T_src), pl.T_src + np.array(sel)])
    assert any("ctx_sel" in e for e in errors_after(move_ctx))

    def nudge_qc(v):
        v["Qc"][0][3, 5] += 1e-2
    assert any("Qc" in e for e in errors_after(nudge_qc))

    # the sharpest block declared flat and the flattest declared sharp
    E = energy_from_oracle(pl)
    top, bottom = int(np.argmax(E)), int(np.argmin(E))

    def swap_split(v):
        v["sharp_ids"][0] = sorted((set(pl.sharp.tolist()) - {top}) | {bottom})
        v["flat_ids"][0] = sorted((set(pl.flat.tolist()) - {bottom}) | {top})
    assert any("sharp set" in e for e in errors_after(swap_split))

    def flip_bit(v):
        v["exact_bits"][0][0, 0] ^= 1
    assert any("bitmap" in e for e in errors_after(flip_bit))

    # a flat row's exact list with its best block replaced by its worst
    row = pl.S[pl.flat[0], pl.kept]
    best, worst = int(np.argmax(row)), int(np.argmin(row))
    assert row[best] - row[worst] > 10 * MARGIN_EXACT

    def worst_exact(v):
        v["exact"][0][0] = sorted((set(pl.exact[0].tolist()) - {best}) | {worst})
    assert any("exact list" in e for e in errors_after(worst_exact))


def test_compare_outputs_reads_only_the_listed_rows():
    pl, _ = plan_and_view()
    ref = np.zeros((500, 4))
    got = np.zeros((500, 4), np.float32)
    rows = block_rows(pl, [1])
    assert rows.tolist() == list(range(32, 64))
    got[40, 2] = 0.5
    got[100, 0] = 9.0                      # outside the listed rows
    mx, mean = compare_outputs(got, ref, rows)
    assert mx == 0.5 and abs(mean - 0.5 / (32 * 4)) < 1e-12
    assert compare_outputs(got, ref, np.zeros(0, np.int64)) == (0.0, 0.0)


def view_of(pl):
    """A one-head plan view (host arrays) holding an oracle plan's index sets."""
    words = (len(pl.kept) + 31) // 32
    bits = np.zeros((len(pl.flat), words), np.int64)
    for r, row in enumerate(pl.exact):
        for x in row:
            bits[r, x // 32] |= 1 << (x % 32)
    return {"Qc": pl.Qc[None].copy(), "Kc": pl.Kc[None].copy(), "Vc": pl.Vc[None].copy(), "imp": pl.imp[None].copy(),
            "ctx_sel": pl.ctx_sel[None].copy(), "kept": pl.kept[None].copy(),
            "energy": energy_from_oracle(pl)[None].copy(), "sharp_ids": pl.sharp[None].copy(),
            "flat_ids": pl.flat[None].copy(), "exact": pl.exact[None].copy(), "exact_bits": bits[None]}


def test_plan_from_gpu_round_trips_the_oracle_plan():
    """Injecting a plan's own index sets gives back the same plan, and the
    same output; also with no flat block (alpha_f = 0) and with no exact
    block (alpha_ns = 0)."""
    for a_f, a_ns in ((0.5, 0.25), (0.0, 0.25), (1.0, 0.0)):
        w = Workload("inject", 1, 1, 64, 300, 200, block=32, alpha_s=0.5, alpha_f=a_f, alpha_ns=a_ns, seed=12)
        qb, kb, vb = (bf16_to_f64(x.reshape(w.L, w.D)) for x in generate_bits(w))
        op = oracle_params(w)
        pl = O.plan_head(qb, kb, vb, op)
        view = view_of(pl)
        r = check_head_plan(pl, view, 0)
        assert not r.errors and r.ctx_equal and not r.split_moved and not r.exact_moved
        got = plan_from_gpu(pl, view, 0)
        for name in ("ctx_sel", "kept", "sharp", "flat", "exact"):
            assert np.array_equal(getattr(got, name), getattr(pl, name)), (a_f, a_ns, name)
        o1, l1 = O.forward_head(qb, kb, vb, pl, op)
        o2, l2 = O.forward_head(qb, kb, vb, got, op)
        assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_plan_from_gpu_uses_the_gpu_choice():
    """A within-margin exact-list swap in the CUDA plan: the check accepts it
    and records the block as moved, and the injected plan carries the CUDA
    choice, so the oracle's output for that block changes with it."""
    w = Workload("inject2", 1, 1, 64, 300, 200, block=32, alpha_s=0.5, alpha_f=0.5, alpha_ns=0.25, seed=12)
    qb, kb, vb = (bf16_to_f64(x.reshape(w.L, w.D)) for x in generate_bits(w))
    op = oracle_params(w)
    pl = O.plan_head(qb, kb, vb, op)
    # move the first flat block's k-th exact block to the (k+1)-th, as a
    # margin-sized fp32 disagreement would; widen the margin to accept it
    b0 = int(pl.flat[0])
    row = pl.S[b0, pl.kept]
    order = np.lexsort((np.arange(len(row)), -row))
    k = pl.exact.shape[1]
    swapped = sorted((set(pl.exact[0].tolist()) - {int(order[k - 1])}) | {int(order[k])})
    view = view_of(pl)
    view["exact"][0][0] = swapped
    view["exact_bits"][0][0] = 0
    for x in swapped:
        view["exact_bits"][0][0, x // 32] |= 1 << (x % 32)
    import parity
    old = parity.MARGIN_EXACT
    parity.MARGIN_EXACT = float(row[order[k - 1]] - row[order[k]]) + 1e-9
    try:
        r = check_head_plan(pl, view, 0)
    finally:
        parity.MARGIN_EXACT = old
    assert not r.errors and r.exact_moved == [b0]
    got = plan_from_gpu(pl, view, 0)
    assert got.exact[0].tolist() == swapped
    o_ref, _ = O.forward_head(qb, kb, vb, pl, op, blocks=[b0])
    o_got, _ = O.forward_head(qb, kb, vb, got, op, blocks=[b0])
    rows = block_rows(pl, [b0])
    assert not np.array_equal(o_ref[rows], o_got[rows])
