"""GPU parity of isa_backward (gradients of the sparse attention with the
plan held fixed) against the fp64 oracle's backward.

The pages state that ISA has a forward and a backward implementation and is
trained end to end (paper.rainbus.top summary card, "Core method" and
innovation (c)); the oracle's backward is pinned by finite differences and
autograd special cases in test_oracle_backward.py.

Tolerance, from the arithmetic of the CUDA path (u = 2^-9, the bf16 unit
roundoff): P and dS are rounded to bf16 before their tensor-core products,
Delta = rowsum(dout * out) is formed from the bf16 forward output, and dq,
dk, dv are rounded to bf16 once; every sum is fp32.  Each gradient element
is then within a few u of the sum of the magnitudes of its terms, and since
the logit gradients of a row add up to zero (cancellation) that sum is
bounded by the tensor's scale rather than by the element.  Per head and
gradient:  max |gpu - ref| <= 16u max|ref|  and  mean |gpu - ref| <= 4u rms(ref).
Where the GPU plan differs from the oracle's inside the planning margins
(both are then valid plans), the oracle's backward runs on the GPU's
validated index sets, so every head is compared.
"""
import numpy as np
import pytest
import torch

import oracle as O
from parity import check_head_plan, oracle_params, plan_from_gpu, plan_view_host, to_torch_bf16
from workloads import Workload, bf16_to_f64, dout_head_bits, generate_bits, generate_dout_bits, head_bits, \
    named_workloads

pytestmark = pytest.mark.gpu

U = 2.0 ** -9
MAX_REL = 16 * U      # of max|ref|
MEAN_REL = 4 * U      # of rms(ref)


@pytest.fixture(scope="module")
def isa():
    from block_sparse_attention_coarse_b200 import build
    build.build()
    import block_sparse_attention_coarse_b200 as I
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return I


def run_gpu(isa, w: Workload, qb, kb, vb, db):
    q, k, v, do = (to_torch_bf16(x) for x in (qb, kb, vb, db))
    p = isa.make_params(w.B, w.H, w.D, w.L_src, w.L_ctx, w.block, w.alpha_s, w.alpha_f, w.alpha_ns)
    ws = isa.plan(q, k, v, p)
    lse = torch.empty(w.B, w.H, w.L, dtype=torch.float32, device="cuda")
    out = isa.forward(q, k, v, ws, p, lse=lse)
    dq, dk, dv = isa.backward(q, k, v, ws, p, out, lse, do)
    torch.cuda.synchronize()
    view = plan_view_host(isa.plan_view(p, ws))
    assert int(view["status"][0]) == 0
    grads = [x.float().cpu().numpy().reshape(w.BH, w.L, w.D) for x in (dq, dk, dv)]
    return grads, view


def gpu_plan(pl, view, h):
    """The oracle plan with the GPU's index sets, once they pass the margin
    rules (where the two plans differ only between near-equal scores, both
    are valid and the gradients are compared for the GPU's choice)."""
    r = check_head_plan(pl, view, h)
    assert not r.errors, (h, r.errors[:5])
    return plan_from_gpu(pl, view, h)


def assert_grads_close(got, ref, what):
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        assert not np.isnan(g).any(), (what, name)
        e = np.abs(g - r)
        assert e.max() <= MAX_REL * np.abs(r).max(), (what, name, float(e.max()), float(np.abs(r).max()))
        assert e.mean() <= MEAN_REL * np.sqrt((r ** 2).mean()), (what, name, float(e.mean()))


CASES = [
    # name, B, H, D, L_src, L_ctx, b, alpha_s, alpha_f, alpha_ns
    ("b64", 1, 2, 128, 520, 300, 64, 0.25, 0.5, 0.1),
    ("b32", 1, 2, 128, 333, 200, 32, 0.25, 0.5, 0.2),
    ("d64_b64", 1, 2, 64, 700, 333, 64, 0.5, 0.5, 0.1),
    ("d64_b32", 1, 2, 64, 300, 77, 32, 0.3, 0.6, 0.15),
    ("no_flat", 1, 2, 128, 600, 200, 64, 0.25, 0.0, 0.1),
    ("dense_equivalent", 1, 2, 128, 400, 300, 64, 1.0, 0.0, 0.1),
    ("all_flat_all_pooled", 1, 2, 128, 500, 260, 64, 0.5, 1.0, 0.0),
    ("alpha_ns_one", 1, 2, 128, 500, 260, 64, 0.5, 0.7, 1.0),
    ("batch2_default_ratios", 2, 2, 128, 1100, 900, 64, 0.125, 0.5, 0.0625),
    ("one_ctx_block", 1, 2, 64, 257, 1, 32, 0.5, 0.5, 0.3),
    ("one_block_per_segment", 1, 3, 128, 40, 24, 64, 1.0, 0.5, 0.5),
]


@pytest.mark.parametrize("name,B,H,D,Ls,Lc,b,a_s,a_f,a_ns", CASES)
def test_backward_matches_oracle(isa, name, B, H, D, Ls, Lc, b, a_s, a_f, a_ns):
    """Every element of dq, dk, dv of every head (several tiles, ragged
    segment tails, both block sizes and head dims, the degenerate ratios)."""
    w = Workload(name, B, H, D, Ls, Lc, block=b, alpha_s=a_s, alpha_f=a_f, alpha_ns=a_ns, seed=81)
    qb, kb, vb = generate_bits(w)
    db = generate_dout_bits(w)
    (gq, gk, gv), view = run_gpu(isa, w, qb, kb, vb, db)
    op = oracle_params(w)
    for h in range(w.BH):
        qh, kh, vh, dh = (bf16_to_f64(x.reshape(w.BH, w.L, w.D)[h]) for x in (qb, kb, vb, db))
        pl = gpu_plan(O.plan_head(qh, kh, vh, op), view, h)
        ref = O.backward_head(qh, kh, vh, pl, op, dh)
        assert_grads_close((gq[h], gk[h], gv[h]), ref, (name, h))
        # context blocks the pre-selection dropped get exactly zero
        dropped = [c for c in range(pl.T_ctx) if c not in set(pl.ctx_sel.tolist())]
        for c in dropped:
            rows = slice(Ls + c * b, min(Ls + (c + 1) * b, w.L))
            assert not gk[h][rows].any() and not gv[h][rows].any()


def test_autograd_function_gradients(isa):
    """IsaAttention.apply under torch.autograd gives the same gradients as
    calling plan / forward / backward directly."""
    w = Workload("autograd", 1, 2, 128, 300, 200, block=64, alpha_s=0.5, alpha_f=0.5, alpha_ns=0.2, seed=82)
    qb, kb, vb = generate_bits(w)
    db = generate_dout_bits(w)
    (gq, gk, gv), _ = run_gpu(isa, w, qb, kb, vb, db)
    q, k, v = (to_torch_bf16(x).requires_grad_(True) for x in (qb, kb, vb))
    p = isa.make_params(w.B, w.H, w.D, w.L_src, w.L_ctx, w.block, w.alpha_s, w.alpha_f, w.alpha_ns)
    out = isa.IsaAttention.apply(q, k, v, p, 0.0)
    out.backward(to_torch_bf16(db))
    torch.cuda.synchronize()
    for g, t in ((gq, q), (gk, k), (gv, v)):
        assert np.array_equal(g, t.grad.float().cpu().numpy().reshape(w.BH, w.L, w.D))


def test_backward_full_size(isa):
    """The bench shape (B=2, H=40, 16384 + 16384 tokens, D=128, b=64):
    every element of dq, dk, dv of one head against the oracle, and for all
    80 heads the sums every softmax attention obeys (each row's weights add
    up to one and its logit gradients to zero): sum_t dv_t = sum_r dout_r and
    sum_t dk_t = 0, to the rounding of the bf16 terms."""
    w = named_workloads()["dit14b"]
    qb, kb, vb = generate_bits(w)
    db = generate_dout_bits(w)
    (gq, gk, gv), view = run_gpu(isa, w, qb, kb, vb, db)
    for g in (gq, gk, gv):
        assert not np.isnan(g).any()
    dsum = bf16_to_f64(db.reshape(w.BH, w.L, w.D)).sum(axis=1)
    for h in range(w.BH):
        sv = gv[h].astype(np.float64).sum(axis=0)
        sk = gk[h].astype(np.float64).sum(axis=0)
        scale_v = np.abs(gv[h]).astype(np.float64).sum(axis=0)
        scale_k = np.abs(gk[h]).astype(np.float64).sum(axis=0)
        assert np.all(np.abs(sv - dsum[h]) <= 4 * U * scale_v + 1e-3), h
        assert np.all(np.abs(sk) <= 4 * U * scale_k + 1e-3), h
    h = 11
    op = oracle_params(w)
    q, k, v = (bf16_to_f64(x) for x in head_bits(w, h))
    dh = bf16_to_f64(dout_head_bits(w, h))
    pl = gpu_plan(O.plan_head(q, k, v, op), view, h)
    ref = O.backward_head(q, k, v, pl, op, dh)
    assert_grads_close((gq[h], gk[h], gv[h]), ref, ("dit14b", h))


def test_backward_rejects_missing_lse(isa):
    w = Workload("lse", 1, 1, 64, 128, 64, seed=83)
    qb, kb, vb = generate_bits(w)
    q, k, v = (to_torch_bf16(x) for x in (qb, kb, vb))
    p = isa.make_params(w.B, w.H, w.D, w.L_src, w.L_ctx)
    ws = isa.plan(q, k, v, p)
    out = isa.forward(q, k, v, ws, p)
    with pytest.raises(isa.IsaError):
        isa.backward(q, k, v, ws, p, out, torch.empty(1, 1, w.L, dtype=torch.float16, device="cuda"), out)


def test_backward_timeout_path_reports_status_and_context_survives(isa):
    """Fault injection makes both backward kernels' MMA warps wait on a
    barrier nothing arrives on: every wait must run out, the plan's status
    word must read ISA_ERR_DEVICE_TIMEOUT, and after a new plan the next
    backward must be correct."""
    w = Workload("bto", 1, 2, 64, 256, 128, block=64, alpha_s=0.5, alpha_f=0.5, alpha_ns=0.25, seed=84)
    qb, kb, vb = generate_bits(w)
    db = generate_dout_bits(w)
    q, k, v, do = (to_torch_bf16(x) for x in (qb, kb, vb, db))
    p = isa.make_params(w.B, w.H, w.D, w.L_src, w.L_ctx, w.block, w.alpha_s, w.alpha_f, w.alpha_ns)
    ws = isa.plan(q, k, v, p)
    lse = torch.empty(w.B, w.H, w.L, dtype=torch.float32, device="cuda")
    out = isa.forward(q, k, v, ws, p, lse=lse)
    torch.cuda.synchronize()
    assert int(isa.plan_view(p, ws)["status"].item()) == 0
    isa.set_wait_timeout_ns(2_000_000)
    isa.set_fault_injection(1)
    try:
        isa.backward(q, k, v, ws, p, out, lse, do)
        torch.cuda.synchronize()
    finally:
        isa.set_fault_injection(0)
        isa.set_wait_timeout_ns(0)
    assert int(isa.plan_view(p, ws)["status"].item()) == isa.ISA_ERR_DEVICE_TIMEOUT
    # a new plan clears the status word; the normal path is intact
    (gq, gk, gv), view = run_gpu(isa, w, qb, kb, vb, db)
    op = oracle_params(w)
    for h in range(w.BH):
        qh, kh, vh, dh = (bf16_to_f64(x.reshape(w.BH, w.L, w.D)[h]) for x in (qb, kb, vb, db))
        pl = gpu_plan(O.plan_head(qh, kh, vh, op), view, h)
        assert_grads_close((gq[h], gk[h], gv[h]), O.backward_head(qh, kh, vh, pl, op, dh), ("bto", h))


@pytest.mark.parametrize("name", ["long65k_b32", "sweep_L131072_D64"])
def test_backward_long_sequences(isa, name):
    """65536 tokens with b=32 (T = 2048 blocks) and 131072 tokens with D=64:
    for every head the gradient sums of any softmax attention (sum_t dv_t =
    sum_r dout_r, sum_t dk_t = 0); for two heads the dq rows of sampled sharp
    and flat blocks against the oracle (a block's dq rows need only that
    block's row of the backward)."""
    w = named_workloads()[name]
    qb, kb, vb = generate_bits(w)
    db = generate_dout_bits(w)
    (gq, gk, gv), view = run_gpu(isa, w, qb, kb, vb, db)
    dsum = bf16_to_f64(db.reshape(w.BH, w.L, w.D)).sum(axis=1)
    for h in range(w.BH):
        for g in (gq[h], gk[h], gv[h]):
            assert not np.isnan(g).any(), h
        sv = gv[h].astype(np.float64).sum(axis=0)
        sk = gk[h].astype(np.float64).sum(axis=0)
        assert np.all(np.abs(sv - dsum[h]) <= 4 * U * np.abs(gv[h]).astype(np.float64).sum(axis=0) + 1e-3), h
        assert np.all(np.abs(sk) <= 4 * U * np.abs(gk[h]).astype(np.float64).sum(axis=0) + 1e-3), h
    op = oracle_params(w)
    for h in (0, 23, 37):
        q, k, v = (bf16_to_f64(x) for x in head_bits(w, h))
        dh = bf16_to_f64(dout_head_bits(w, h))
        pl = gpu_plan(O.plan_head(q, k, v, op), view, h)
        blocks = [int(pl.sharp[0]), int(pl.sharp[-1]), int(pl.flat[0]), int(pl.flat[len(pl.flat) // 2])]
        ref_dq, _, _ = O.backward_head(q, k, v, pl, op, dh, blocks=blocks)
        rows = np.concatenate([np.arange(pl.starts[i], pl.starts[i] + pl.counts[i]) for i in blocks])
        e = np.abs(gq[h][rows] - ref_dq[rows])
        r = ref_dq[rows]
        assert e.max() <= MAX_REL * np.abs(r).max() and e.mean() <= MEAN_REL * np.sqrt((r ** 2).mean()), (name, h)
