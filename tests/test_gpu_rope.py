"""GPU parity of isa_rope (decoupled RoPE of Q and K) against the fp64 oracle.

  * Rotated values: the kernel computes in fp32 from the bf16 inputs with an
    fp64 table of angles and rounds once to bf16, the oracle in fp64; every
    element must agree within two bf16 half-ulps of the oracle's value
    (|gpu - ref| <= 2^-8 |ref| + 1e-6).
  * In place and out of place give identical bits.
  * isa_plan_rope (the rotation inside the pooling pass) equals isa_rope then
    isa_plan bit for bit: rotated q, k and every plan array.
  * End to end: rope -> isa_plan -> isa_forward (and isa_plan_rope ->
    isa_forward) on the GPU against the oracle's
    rope (rounded once to bf16, the precision the GPU hands on) -> plan ->
    forward.  The two sides plan from rotations rounded independently (a few
    elements one bf16 ulp apart), so value checks allow one rounding of the
    inputs and index sets that differ beyond the margins are counted (at most
    5 %); every block's output is compared with the oracle run on the GPU's
    plan, within the tolerances of the other parity tests.
"""
import numpy as np
import pytest
import torch

import oracle as O
from parity import (OUT_MAX_ABS, OUT_MEAN_ABS, block_rows, check_head_plan, compare_outputs, oracle_params,
                    plan_from_gpu, plan_view_host, to_torch_bf16)
from workloads import Workload, bf16_to_f64, f32_to_bf16_bits, generate_bits, named_workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def isa():
    from block_sparse_attention_coarse_b200 import build
    build.build()
    import block_sparse_attention_coarse_b200 as I
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return I


def params_of(isa, w: Workload):
    return isa.make_params(w.B, w.H, w.D, w.L_src, w.L_ctx, w.block, w.alpha_s, w.alpha_f, w.alpha_ns)


def bits_of(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def assert_rotation_close(gpu_bits: np.ndarray, ref: np.ndarray):
    g = bf16_to_f64(gpu_bits)
    d = np.abs(g - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 1e-6
    assert np.all(d <= bound), (float((d - bound).max()), int((d > bound).sum()))


@pytest.mark.parametrize("B,H,D,L_src,L_ctx,base", [(1, 2, 64, 300, 77, 10000.0), (2, 3, 128, 512, 512, 10000.0),
                                                      (1, 1, 128, 1000, 24, 500.0), (1, 2, 64, 64, 1, 1e6)])
def test_rope_matches_oracle(isa, B, H, D, L_src, L_ctx, base):
    w = Workload("rope", B, H, D, L_src, L_ctx, seed=61)
    qb, kb, _ = generate_bits(w)
    q, k = to_torch_bf16(qb), to_torch_bf16(kb)
    p = params_of(isa, w)
    qr, kr = isa.rope(q, k, p, base)
    torch.cuda.synchronize()
    for src_bits, out in ((qb, qr), (kb, kr)):
        x = bf16_to_f64(src_bits).reshape(B * H, w.L, D)
        ref = O.rope_decoupled(x, L_src, L_ctx, base)
        assert_rotation_close(bits_of(out).reshape(B * H, w.L, D), ref)


def test_rope_in_place_equals_out_of_place(isa):
    w = Workload("rope_ip", 1, 2, 128, 700, 333, seed=62)
    qb, kb, _ = generate_bits(w)
    q, k = to_torch_bf16(qb), to_torch_bf16(kb)
    p = params_of(isa, w)
    qr, kr = isa.rope(q, k, p)
    q2, k2 = q.clone(), k.clone()
    isa.rope(q2, k2, p, inplace=True)
    torch.cuda.synchronize()
    assert torch.equal(qr, q2) and torch.equal(kr, k2)
    assert not torch.equal(qr, q)


def test_rope_full_size_sampled_heads(isa):
    """The bench shape (B=2, H=40, 16384 + 16384 tokens, D=128): every
    element of two heads against the oracle."""
    w = named_workloads()["dit14b"]
    qb, kb, _ = generate_bits(w)
    q, k = to_torch_bf16(qb), to_torch_bf16(kb)
    p = params_of(isa, w)
    qr, kr = isa.rope(q, k, p)
    torch.cuda.synchronize()
    for src_bits, out in ((qb, qr), (kb, kr)):
        x = src_bits.reshape(w.BH, w.L, w.D)
        g = bits_of(out).reshape(w.BH, w.L, w.D)
        for h in (3, 57):
            ref = O.rope_decoupled(bf16_to_f64(x[h]), w.L_src, w.L_ctx)
            assert_rotation_close(g[h], ref)


def assert_plans_equal(isa, p, ws_a, ws_b):
    va, vb = isa.plan_view(p, ws_a), isa.plan_view(p, ws_b)
    for name, a in va.items():
        if isinstance(a, torch.Tensor):
            assert torch.equal(a, vb[name]), name


@pytest.mark.parametrize("B,H,D,L_src,L_ctx,b,base", [(1, 2, 128, 520, 300, 64, 10000.0),
                                                        (2, 2, 64, 333, 97, 32, 500.0),
                                                        (1, 3, 128, 1000, 1, 64, 1e6)])
def test_plan_rope_equals_rope_then_plan(isa, B, H, D, L_src, L_ctx, b, base):
    """isa_plan_rope (the rotation folded into the pooling pass) gives bit
    for bit the rotated q, k and the plan of isa_rope followed by isa_plan,
    out of place and in place, and so the same forward output."""
    w = Workload("plan_rope", B, H, D, L_src, L_ctx, block=b, alpha_s=0.25, alpha_f=0.5, alpha_ns=0.2, seed=64)
    qb, kb, vb = generate_bits(w)
    q, k, v = (to_torch_bf16(x) for x in (qb, kb, vb))
    p = params_of(isa, w)
    qr, kr = isa.rope(q, k, p, base)
    ws_sep = isa.plan(qr, kr, v, p)
    ws_fused, qf, kf = isa.plan_rope(q, k, v, p, base)
    q2, k2 = q.clone(), k.clone()
    ws_ip, q2r, k2r = isa.plan_rope(q2, k2, v, p, base, inplace=True)
    torch.cuda.synchronize()
    assert torch.equal(qf, qr) and torch.equal(kf, kr)
    assert q2r.data_ptr() == q2.data_ptr() and torch.equal(q2, qr) and torch.equal(k2, kr)
    assert torch.equal(q, to_torch_bf16(qb)) and torch.equal(k, to_torch_bf16(kb))   # inputs untouched
    assert_plans_equal(isa, p, ws_sep, ws_fused)
    assert_plans_equal(isa, p, ws_sep, ws_ip)
    assert int(isa.plan_view(p, ws_fused)["status"].item()) == 0
    assert torch.equal(isa.forward(qr, kr, v, ws_sep, p), isa.forward(qf, kf, v, ws_fused, p))


def test_plan_rope_equals_rope_then_plan_full_size(isa):
    """The same bit-equality on every head of the bench shape (B=2, H=40,
    16384 + 16384 tokens, D=128)."""
    w = named_workloads()["dit14b"]
    q, k, v = (to_torch_bf16(x) for x in generate_bits(w))
    p = params_of(isa, w)
    qr, kr = isa.rope(q, k, p)
    ws_sep = isa.plan(qr, kr, v, p)
    ws_fused, qf, kf = isa.plan_rope(q, k, v, p)
    torch.cuda.synchronize()
    assert torch.equal(qf, qr) and torch.equal(kf, kr)
    assert_plans_equal(isa, p, ws_sep, ws_fused)


@pytest.mark.parametrize("fused", [True, False], ids=["plan_rope", "rope_then_plan"])
@pytest.mark.parametrize("name,B,H,D,Ls,Lc,b", [("rope_e2e", 1, 2, 128, 520, 300, 64),
                                                ("rope_e2e_b32", 1, 2, 64, 333, 200, 32)])
def test_isa_with_rope_end_to_end(isa, name, B, H, D, Ls, Lc, b, fused):
    w = Workload(name, B, H, D, Ls, Lc, block=b, alpha_s=0.25, alpha_f=0.5, alpha_ns=0.2, seed=63)
    qb, kb, vb = generate_bits(w)
    q, k, v = (to_torch_bf16(x) for x in (qb, kb, vb))
    p = params_of(isa, w)
    lse = torch.empty(B, H, w.L, dtype=torch.float32, device="cuda")
    if fused:
        ws, qr, kr = isa.plan_rope(q, k, v, p)
    else:
        qr, kr = isa.rope(q, k, p)
        ws = isa.plan(qr, kr, v, p)
    out = isa.forward(qr, kr, v, ws, p, lse=lse)
    torch.cuda.synchronize()
    view = plan_view_host(isa.plan_view(p, ws))
    assert int(view["status"][0]) == 0
    out = out.float().cpu().numpy().reshape(w.BH, w.L, D)
    lse = lse.cpu().numpy().reshape(w.BH, w.L)
    op = oracle_params(w)
    n_sets = n_outside = 0
    for h in range(w.BH):
        # oracle side: its own rotation of the bf16 inputs, rounded once to bf16
        qo = O.rope_decoupled(bf16_to_f64(qb.reshape(w.BH, w.L, D)[h]), Ls, Lc)
        ko = O.rope_decoupled(bf16_to_f64(kb.reshape(w.BH, w.L, D)[h]), Ls, Lc)
        qo, ko = bf16_to_f64(f32_to_bf16_bits(qo)), bf16_to_f64(f32_to_bf16_bits(ko))
        vo = bf16_to_f64(vb.reshape(w.BH, w.L, D)[h])
        pl = O.plan_head(qo, ko, vo, op)
        r = check_head_plan(pl, view, h, inputs_equal=False)
        assert not r.errors, (h, r.errors[:5])
        # the plans came from inputs one bf16 rounding apart, so an index set
        # may differ beyond the margin where scores are that close: count such
        # sets, then compare every block with the oracle run on the GPU's plan
        n_outside += len(r.outside_margin)
        n_sets += 1 + (pl.T > len(pl.sharp)) + len(pl.flat)
        ref, ref_lse = O.forward_head(qo, ko, vo, plan_from_gpu(pl, view, h), op)
        rows = block_rows(pl, range(pl.T))
        mx, mean = compare_outputs(out[h], ref, rows)
        assert mx <= OUT_MAX_ABS and mean <= OUT_MEAN_ABS, (h, mx, mean)
        assert np.abs(lse[h][rows] - ref_lse[rows]).max() <= 2e-2
    assert n_outside <= 0.05 * max(n_sets, 1), (n_outside, n_sets)
