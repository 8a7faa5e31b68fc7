"""The comparison helpers of the GPU parity tests (tests/parity.py) reject
what they must.  A helper that always agreed would make every GPU parity
test pass, so each rule is checked here on the CPU with planted
disagreements: a chosen set beyond the margin, wrong counts, a moved
context block, perturbed pooled means, a swapped sharp/flat pair, an exact
bitmap that disagrees with its list, and an output error in a sampled row."""
import numpy as np

import oracle as O
from parity import (MARGIN_EXACT, block_rows, check_head_plan, compare_outputs, energy_from_oracle,
                    oracle_params, topk_agrees)
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
