"""GPU parity of the gamma * O_coarse residual (isa_coarse_residual and its
backward) against the fp64 oracle (coarse_residual, coarse_residual_backward;
summary card step (6), reading in the oracle).

Tolerance from the arithmetic: the CUDA path works in fp32 on the plan's fp32
pooled means (which differ from the oracle's fp64 means by fp32 rounding) and
rounds each result to bf16 once (out += residual; dq, dk, dv += gradient), so
every element lies within 2^-8 of its own magnitude plus 2^-12 of the
tensor's largest value (sums of T terms in fp32); dgamma (an fp32 sum of
B*H*L*D products) within 1e-4 relative.
"""
import numpy as np
import pytest
import torch

import oracle as O
from parity import oracle_params, to_torch_bf16
from workloads import Workload, bf16_to_f64, generate_bits, generate_dout_bits, head_bits, named_workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def isa():
    from block_sparse_attention_coarse_b200 import build
    build.build()
    import block_sparse_attention_coarse_b200 as I
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return I


def assert_close(got, ref, what):
    e = np.abs(got - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 2.0 ** -12 * np.abs(ref).max()
    assert np.all(e <= bound), (what, float((e - bound).max()), int((e > bound).sum()))


# the last one has 1100 pooled blocks in its head: 17 full 64-block tiles
# and a ragged one, on both sides of the kernels' tile loops
CASES = [("d128_b64", 1, 2, 128, 520, 300, 64, 0.7), ("d128_b32", 1, 2, 128, 333, 200, 32, -1.5),
         ("d64_b64", 2, 1, 64, 700, 333, 64, 0.25), ("d64_b32_one_ctx_token", 1, 2, 64, 257, 1, 32, 2.0),
         ("d128_b32_1100_blocks", 1, 1, 128, 17600, 17600, 32, 0.5)]


@pytest.mark.parametrize("name,B,H,D,Ls,Lc,b,gamma", CASES)
def test_residual_forward_and_backward(isa, name, B, H, D, Ls, Lc, b, gamma):
    w = Workload(name, B, H, D, Ls, Lc, block=b, seed=91)
    qb, kb, vb = generate_bits(w)
    db = generate_dout_bits(w)
    q, k, v, do = (to_torch_bf16(x) for x in (qb, kb, vb, db))
    p = isa.make_params(w.B, w.H, w.D, w.L_src, w.L_ctx, w.block)
    ws = isa.plan(q, k, v, p)
    # forward on a non-zero output: out + gamma * O_coarse
    base = to_torch_bf16(db)
    out = isa.coarse_residual(base.clone(), ws, p, gamma)
    zq, zk, zv = (torch.zeros_like(q) for _ in range(3))
    dgamma = torch.zeros(w.B * w.H, dtype=torch.float32, device="cuda")
    isa.coarse_residual_backward(ws, p, gamma, do, zq, zk, zv, dgamma)
    torch.cuda.synchronize()
    op = oracle_params(w)
    got_out = out.float().cpu().numpy().reshape(w.BH, w.L, w.D)
    grads = [t.float().cpu().numpy().reshape(w.BH, w.L, w.D) for t in (zq, zk, zv)]
    dg = dgamma.cpu().numpy()
    for h in range(w.BH):
        qh, kh, vh, dh = (bf16_to_f64(x.reshape(w.BH, w.L, w.D)[h]) for x in (qb, kb, vb, db))
        pl = O.plan_head(qh, kh, vh, op)
        assert_close(got_out[h], dh + O.coarse_residual(pl, op, gamma), (name, h, "out"))
        rq, rk, rv, rg = O.coarse_residual_backward(pl, op, gamma, dh)
        for nm, g, r in zip(("dq", "dk", "dv"), grads, (rq, rk, rv)):
            assert_close(g[h], r, (name, h, nm))
        assert abs(dg[h] - rg) <= 1e-4 * max(1.0, abs(rg)), (name, h, dg[h], rg)


def test_autograd_with_residual(isa):
    """IsaAttention with gamma != 0 equals the sparse forward plus the
    residual, and its gradients equal backward + the residual's backward."""
    w = Workload("ag_res", 1, 2, 128, 300, 200, block=64, alpha_s=0.5, alpha_f=0.5, alpha_ns=0.2, seed=92)
    qb, kb, vb = generate_bits(w)
    db = generate_dout_bits(w)
    p = isa.make_params(w.B, w.H, w.D, w.L_src, w.L_ctx, w.block, w.alpha_s, w.alpha_f, w.alpha_ns)
    q, k, v, do = (to_torch_bf16(x) for x in (qb, kb, vb, db))
    ws = isa.plan(q, k, v, p)
    lse = torch.empty(w.B, w.H, w.L, dtype=torch.float32, device="cuda")
    out = isa.forward(q, k, v, ws, p, lse=lse)
    ref_out = isa.coarse_residual(out.clone(), ws, p, 0.5)
    dq, dk, dv = isa.backward(q, k, v, ws, p, out, lse, do)
    isa.coarse_residual_backward(ws, p, 0.5, do, dq, dk, dv)
    qa, ka, va = (t.clone().requires_grad_(True) for t in (q, k, v))
    got = isa.IsaAttention.apply(qa, ka, va, p, 0.5)
    got.backward(do)
    torch.cuda.synchronize()
    assert torch.equal(got, ref_out)
    for a, b in ((qa.grad, dq), (ka.grad, dk), (va.grad, dv)):
        assert torch.equal(a, b)


def test_residual_full_size_sampled_heads(isa):
    """The bench shape (B=2, H=40, 16384 + 16384 tokens, D=128): every output
    element of two heads."""
    w = named_workloads()["dit14b"]
    qb, kb, vb = generate_bits(w)
    q, k, v = (to_torch_bf16(x) for x in (qb, kb, vb))
    p = isa.make_params(w.B, w.H, w.D, w.L_src, w.L_ctx, w.block)
    ws = isa.plan(q, k, v, p)
    out = isa.coarse_residual(torch.zeros_like(q), ws, p, 1.0)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy().reshape(w.BH, w.L, w.D)
    op = oracle_params(w)
    for h in (5, 66):
        qh, kh, vh = (bf16_to_f64(x) for x in head_bits(w, h))
        assert_close(got[h], O.coarse_residual(O.plan_head(qh, kh, vh, op), op, 1.0), ("dit14b", h))


def test_residual_backward_full_size_sampled_heads(isa):
    """The bench shape: every element of dq, dk, dv and dgamma of two heads."""
    w = named_workloads()["dit14b"]
    qb, kb, vb = generate_bits(w)
    q, k, v = (to_torch_bf16(x) for x in (qb, kb, vb))
    do = to_torch_bf16(generate_dout_bits(w))
    p = isa.make_params(w.B, w.H, w.D, w.L_src, w.L_ctx, w.block)
    ws = isa.plan(q, k, v, p)
    zq, zk, zv = (torch.zeros_like(q) for _ in range(3))
    dgamma = torch.zeros(w.BH, dtype=torch.float32, device="cuda")
    isa.coarse_residual_backward(ws, p, 0.75, do, zq, zk, zv, dgamma)
    torch.cuda.synchronize()
    op = oracle_params(w)
    dob = generate_dout_bits(w, heads=[7, 48])
    for idx, h in enumerate((7, 48)):
        qh, kh, vh = (bf16_to_f64(x) for x in head_bits(w, h))
        pl = O.plan_head(qh, kh, vh, op)
        rq, rk, rv, rg = O.coarse_residual_backward(pl, op, 0.75, bf16_to_f64(dob[idx]))
        for nm, t, r in (("dq", zq, rq), ("dk", zk, rk), ("dv", zv, rv)):
            assert_close(t.reshape(w.BH, w.L, w.D)[h].float().cpu().numpy(), r, ("dit14b", h, nm))
        assert abs(float(dgamma[h]) - rg) <= 1e-4 * max(1.0, abs(rg))
