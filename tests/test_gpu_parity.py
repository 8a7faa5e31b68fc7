"""GPU parity of the CUDA path (through the C-ABI) against the fp64 oracle.

Every case draws seeded inputs from `workloads`, runs isa_plan / isa_forward
/ isa_dense on the GPU and compares with the oracle on the same bf16 values:
  * plan index sets: bit-exact outside the margins of tests/parity.py;
  * outputs: max-abs <= 2e-2 and mean-abs <= 2e-3 (bf16 inputs, fp32
    accumulation, bf16 output), on every compared row;
  * lse (natural-log softmax normaliser): abs <= 2e-2.
Small cases are compared in full; the full-size workloads on a seeded sample
of heads and query blocks.  Where the CUDA plan differs from the oracle's
inside the margins, the oracle runs on the CUDA plan's (validated) index
sets, so no sampled block or head is left out of the output comparison.
"""
import numpy as np
import pytest
import torch

import oracle as O
from parity import (OUT_MAX_ABS, OUT_MEAN_ABS, check_case, check_head_plan, oracle_params, params_of,
                    plan_view_host, run_isa, to_torch_bf16)
from workloads import Workload, bf16_to_f64, generate_bits, named_workloads, sample_blocks

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def isa():
    from block_sparse_attention_coarse_b200 import build
    build.build()
    import block_sparse_attention_coarse_b200 as I
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return I


# ---------------------------------------------------------------------------
# planning only (no tensor-core kernel involved)
# ---------------------------------------------------------------------------

def test_plan_tiny_matches_oracle(isa):
    w = named_workloads()["tiny"]
    qb, kb, vb = generate_bits(w)
    q, k, v = (to_torch_bf16(x) for x in (qb, kb, vb))
    p = params_of(isa, w)
    ws = isa.plan(q, k, v, p)
    torch.cuda.synchronize()
    view = plan_view_host(isa.plan_view(p, ws))
    op = oracle_params(w)
    for h in range(w.BH):
        pl = O.plan_head(bf16_to_f64(qb.reshape(w.BH, w.L, w.D)[h]), bf16_to_f64(kb.reshape(w.BH, w.L, w.D)[h]),
                         bf16_to_f64(vb.reshape(w.BH, w.L, w.D)[h]), op)
        r = check_head_plan(pl, view, h)
        assert not r.errors, r.errors[:5]


@pytest.mark.parametrize("L_src,L_ctx,b,D", [(300, 150, 64, 128), (333, 97, 32, 64), (64, 20, 32, 128)])
def test_plan_ragged_matches_oracle(isa, L_src, L_ctx, b, D):
    w = Workload("ragged", 1, 3, D, L_src, L_ctx, block=b, alpha_s=0.3, alpha_f=0.5, alpha_ns=0.2, seed=77)
    qb, kb, vb = generate_bits(w)
    q, k, v = (to_torch_bf16(x) for x in (qb, kb, vb))
    p = params_of(isa, w)
    ws = isa.plan(q, k, v, p)
    torch.cuda.synchronize()
    view = plan_view_host(isa.plan_view(p, ws))
    op = oracle_params(w)
    for h in range(w.BH):
        pl = O.plan_head(*(bf16_to_f64(x.reshape(w.BH, w.L, w.D)[h]) for x in (qb, kb, vb)), op)
        r = check_head_plan(pl, view, h)
        assert not r.errors, r.errors[:5]
        # bf16 pooled keys/values of the kept blocks, zero padding
        Kp = view["Kp"][h]
        assert np.abs(Kp[:len(pl.kept)] - pl.Kc[pl.kept]).max() <= 2 ** -8 * max(1, np.abs(pl.Kc).max())
        assert np.all(Kp[len(pl.kept):] == 0)


# ---------------------------------------------------------------------------
# dense kernel
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("L_src,L_ctx,D", [(128, 128, 128), (200, 77, 64), (1000, 536, 128)])
def test_dense_matches_oracle(isa, L_src, L_ctx, D):
    w = Workload("dense", 1, 2, D, L_src, L_ctx, kind="iid", seed=5)
    qb, kb, vb = generate_bits(w)
    q, k, v = (to_torch_bf16(x) for x in (qb, kb, vb))
    p = params_of(isa, w)
    lse = torch.empty(w.B, w.H, w.L, dtype=torch.float32, device="cuda")
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    out = isa.dense(q, k, v, p, lse=lse, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    out = out.float().cpu().numpy().reshape(w.BH, w.L, w.D)
    lse = lse.cpu().numpy().reshape(w.BH, w.L)
    for h in range(w.BH):
        ref, ref_lse = O.dense_attention(*(bf16_to_f64(x.reshape(w.BH, w.L, w.D)[h]) for x in (qb, kb, vb)),
                                         1 / np.sqrt(D))
        d = np.abs(out[h] - ref)
        assert d.max() <= OUT_MAX_ABS and d.mean() <= OUT_MEAN_ABS, (d.max(), d.mean())
        assert np.abs(lse[h] - ref_lse).max() <= 2e-2


# ---------------------------------------------------------------------------
# ISA forward, small cases in full
# ---------------------------------------------------------------------------

def test_forward_tiny(isa):
    check_case(isa, named_workloads()["tiny"])


SMALL = [
    # name, B, H, D, L_src, L_ctx, b, alpha_s, alpha_f, alpha_ns
    ("ragged128", 1, 2, 128, 300, 150, 64, 0.125, 0.5, 0.0625),
    ("ragged64_b32", 1, 2, 64, 333, 97, 32, 0.3, 0.5, 0.2),
    ("no_pruning_all_sharp", 1, 2, 128, 256, 192, 64, 1.0, 0.0, 0.5),
    ("all_flat_pooled_only", 1, 2, 128, 400, 300, 64, 0.5, 1.0, 0.0),
    ("alpha_ns_one", 1, 2, 64, 256, 256, 64, 0.25, 0.5, 1.0),
    ("single_ctx_block", 2, 2, 128, 512, 20, 64, 0.125, 0.5, 0.0625),
    ("b32_d128", 1, 3, 128, 1024, 1024, 32, 0.125, 0.5, 0.0625),
    ("odd_counts", 1, 1, 64, 700, 650, 64, 0.2, 0.37, 0.11),
    # the degenerate minimum: one source and one context token, so two
    # one-token blocks and two rows in all (fewer than one TMA box); one
    # block flat with one exact block, the other sharp
    ("one_token_each", 1, 1, 64, 1, 1, 64, 0.125, 0.5, 0.0625),
    ("one_token_each_d128_b32", 1, 1, 128, 1, 1, 32, 1.0, 0.5, 0.5),
]


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_forward_small_cases(isa, case):
    name, B, H, D, Ls, Lc, b, a_s, a_f, a_ns = case
    check_case(isa, Workload(name, B, H, D, Ls, Lc, block=b, alpha_s=a_s, alpha_f=a_f, alpha_ns=a_ns, seed=31))


def test_no_pruning_equals_dense(isa):
    """alpha_s = 1, alpha_f = 0 reduces ISA to dense attention: the two CUDA
    paths must agree with each other as well as with the oracle."""
    w = Workload("np", 1, 2, 128, 384, 256, alpha_s=1.0, alpha_f=0.0, seed=9)
    bits, out, _, _ = run_isa(isa, w)
    q, k, v = (to_torch_bf16(x) for x in bits)
    d = isa.dense(q, k, v, params_of(isa, w)).float().view(w.BH, w.L, w.D)
    assert float((d - out.float()).abs().max()) <= 1e-2


def test_forward_is_deterministic(isa):
    w = Workload("det", 1, 2, 128, 512, 512, seed=3)
    qb, kb, vb = generate_bits(w)
    q, k, v = (to_torch_bf16(x) for x in (qb, kb, vb))
    p = params_of(isa, w)
    ws = isa.plan(q, k, v, p)
    a = isa.forward(q, k, v, ws, p).clone()
    b = isa.forward(q, k, v, ws, p)
    ws2 = isa.plan(q, k, v, p)
    c = isa.forward(q, k, v, ws2, p)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(a, c)


# ---------------------------------------------------------------------------
# full-size workloads, sampled: every named workload of the benchmark
# ---------------------------------------------------------------------------

def full_size_sample(w: Workload):
    """(heads, query blocks per head) compared at full size: every head of
    the 8-head workload, otherwise a seeded sample of heads (two at 131072
    tokens, where one head's oracle plan already takes a few seconds)."""
    if w.BH <= 8:
        return list(range(w.BH)), 10
    n_heads = 2 if w.L >= 131072 else 3
    return sorted({bh for bh, _ in sample_blocks(w, n_heads, 1)}), 6


FULL_SIZE = [n for n in named_workloads() if n != "tiny"]


@pytest.mark.parametrize("name", FULL_SIZE)
def test_forward_full_size(isa, name):
    """Each workload of the benchmark at its full size, in the launch the
    bench times (all B*H heads in one plan and one forward): mid (23768
    tokens, partial last blocks), dit14b (B=2, H=40, 32768 tokens), 65536
    tokens at b=64 and b=32 and with alpha_f 0.25 / 0.75, the length sweep
    4096..131072 at D=64 and D=128, and the alpha_s x alpha_ns grid at
    131072 tokens.  Plans of the sampled heads are checked under the margin
    rules; the outputs and lse of sampled query blocks element by element."""
    w = named_workloads()[name]
    heads, per_head = full_size_sample(w)
    check_case(isa, w, heads=heads, blocks_per_head=per_head)


def test_dense_dit14b_full_size_sampled_rows(isa):
    """isa_dense at the benchmarked size against the oracle's dense attention
    on a seeded sample of rows of a few heads."""
    w = named_workloads()["dit14b"]
    qb, kb, vb = generate_bits(w)
    q, k, v = (to_torch_bf16(x) for x in (qb, kb, vb))
    p = params_of(isa, w)
    lse = torch.empty(w.B, w.H, w.L, dtype=torch.float32, device="cuda")
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    out = isa.dense(q, k, v, p, lse=lse, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    out = out.float().cpu().numpy().reshape(w.BH, w.L, w.D)
    lse = lse.cpu().numpy().reshape(w.BH, w.L)
    g = np.random.default_rng(77)
    for h in sorted(g.choice(w.BH, size=3, replace=False).tolist()):
        rows = np.sort(g.choice(w.L, size=256, replace=False))
        ref, ref_lse = O.dense_attention(*(bf16_to_f64(x.reshape(w.BH, w.L, w.D)[h]) for x in (qb, kb, vb)),
                                         1 / np.sqrt(w.D), rows=rows)
        d = np.abs(out[h][rows] - ref)
        assert d.max() <= OUT_MAX_ABS and d.mean() <= OUT_MEAN_ABS, (h, d.max(), d.mean())
        assert np.abs(lse[h][rows] - ref_lse).max() <= 2e-2


# ---------------------------------------------------------------------------
# bounded waits
# ---------------------------------------------------------------------------

def test_timeout_path_reports_status_and_context_survives(isa):
    """Fault injection makes the attention kernel wait on a barrier nothing
    arrives on; the wait must run out, raise the status word and return, and
    the next normal launch must still be correct."""
    w = Workload("to", 1, 1, 64, 128, 128, kind="iid", seed=1)
    qb, kb, vb = generate_bits(w)
    q, k, v = (to_torch_bf16(x) for x in (qb, kb, vb))
    p = params_of(isa, w)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    isa.set_wait_timeout_ns(2_000_000)
    isa.set_fault_injection(1)
    try:
        isa.dense(q, k, v, p, status=status)
        torch.cuda.synchronize()
    finally:
        isa.set_fault_injection(0)
        isa.set_wait_timeout_ns(0)
    assert int(status.item()) == isa.ISA_ERR_DEVICE_TIMEOUT
    out = isa.dense(q, k, v, p, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref, _ = O.dense_attention(*(bf16_to_f64(x.reshape(w.L, w.D)) for x in (qb, kb, vb)), 1 / 8.0)
    assert np.abs(out.float().cpu().numpy().reshape(w.L, w.D) - ref).max() <= OUT_MAX_ABS
