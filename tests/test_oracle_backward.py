"""Pins of the oracle's backward (gradients of the ISA output with the plan
held fixed) against what the mathematics fixes.

The LIVEditor pages state that the method has a backward implementation and
is trained end to end (paper.rainbus.top summary card, "Core method" and
innovation (c); techwalker.com retelling, section on training) but print no
gradient formulas.  Each check below gets its expectation without the
oracle's backward arithmetic:
  * central finite differences of the oracle forward (itself pinned by the
    forward tests), with the plan's index sets held fixed and the pooled
    means recomputed from the perturbed inputs;
  * torch autograd of plain softmax attention in the special cases where
    ISA reduces to it (alpha_s = 1 and alpha_f = 0; alpha_ns = 1);
  * the zero in-block key variance case, where the Taylor path is exact;
  * sums that hold for any softmax attention: every row's weights add up to
    one and every row's logit gradients add up to zero.
"""
import dataclasses
import math

import numpy as np
import pytest
import torch

import oracle as O
from test_oracle import brute_block_of, brute_kept, brute_pool, kept_token_mask, rand_qkv


def loss_fixed_plan(q, k, v, plan, p, dout):
    """sum(dout * out) with the plan's choices fixed and the pooled means
    taken from the given k, v."""
    Kc, _ = brute_pool(k, p.L_src, p.L_ctx, p.block)
    Vc, _ = brute_pool(v, p.L_src, p.L_ctx, p.block)
    out, _ = O.forward_head(q, k, v, dataclasses.replace(plan, Kc=Kc, Vc=Vc), p)
    return float((dout * out).sum())


def central_differences(q, k, v, plan, p, dout, h=1e-5):
    grads = []
    for which in range(3):
        xs = [q.copy(), k.copy(), v.copy()]
        g = np.zeros_like(xs[which])
        for idx in np.ndindex(*g.shape):
            x0 = xs[which][idx]
            xs[which][idx] = x0 + h
            fp = loss_fixed_plan(*xs, plan, p, dout)
            xs[which][idx] = x0 - h
            fm = loss_fixed_plan(*xs, plan, p, dout)
            xs[which][idx] = x0
            g[idx] = (fp - fm) / (2 * h)
        grads.append(g)
    return grads


def autograd_attention(q, k, v, dout, s, col_mask=None):
    """(dq, dk, dv) of softmax(s q k^T) v restricted to the columns in
    col_mask, by torch autograd in fp64."""
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    logits = s * tq @ tk.T
    if col_mask is not None:
        logits = logits.masked_fill(~torch.tensor(col_mask)[None, :], float("-inf"))
    out = torch.softmax(logits, dim=1) @ tv
    (out * torch.tensor(dout)).sum().backward()
    return tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


@pytest.mark.parametrize("L_src,L_ctx,b,D,ratios,seed", [
    (22, 13, 8, 6, (0.5, 0.5, 0.34), 3),
    (30, 17, 8, 4, (0.5, 0.6, 0.2), 8),
])
def test_backward_matches_central_differences(L_src, L_ctx, b, D, ratios, seed):
    """Every element of dq, dk and dv against central differences of the
    forward (partial blocks in both segments, sharp and flat blocks, pooled
    columns of partial blocks)."""
    rng = np.random.default_rng(seed)
    q, k, v = rand_qkv(rng, L_src + L_ctx, D)
    dout = rng.standard_normal((L_src + L_ctx, D))
    a_s, a_f, a_ns = ratios
    p = O.Params(D=D, L_src=L_src, L_ctx=L_ctx, block=b, alpha_s=a_s, alpha_f=a_f, alpha_ns=a_ns)
    plan = O.plan_head(q, k, v, p)
    # the case must exercise both paths and a pooled partial block
    assert len(plan.sharp) > 0 and len(plan.flat) > 0
    partial = {j for j in plan.kept if plan.counts[j] < b}
    pooled_partial = any(j not in set(plan.kept[plan.exact[r]].tolist()) for r in range(len(plan.flat))
                         for j in partial)
    assert pooled_partial
    dq, dk, dv = O.backward_head(q, k, v, plan, p, dout)
    fq, fk, fv = central_differences(q, k, v, plan, p, dout)
    for got, ref in ((dq, fq), (dk, fk), (dv, fv)):
        np.testing.assert_allclose(got, ref, rtol=1e-6, atol=1e-7)


@pytest.mark.parametrize("L_src,L_ctx,b,D", [(48, 40, 16, 8), (37, 21, 8, 4)])
def test_no_pruning_no_flat_is_full_attention_gradient(L_src, L_ctx, b, D):
    """alpha_s = 1, alpha_f = 0: plain softmax attention, so the gradients
    are autograd's."""
    rng = np.random.default_rng(31)
    q, k, v = rand_qkv(rng, L_src + L_ctx, D)
    dout = rng.standard_normal(q.shape)
    p = O.Params(D=D, L_src=L_src, L_ctx=L_ctx, block=b, alpha_s=1.0, alpha_f=0.0, alpha_ns=0.3)
    got = O.isa_backward(q, k, v, dout, p)
    ref = autograd_attention(q, k, v, dout, 1 / math.sqrt(D))
    for g, r in zip(got, ref):
        np.testing.assert_allclose(g, r, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("alpha_f", [0.5, 1.0])
def test_alpha_ns_one_is_exact_attention_gradient_over_kept(alpha_f):
    """alpha_ns = 1: exact attention over the kept tokens; tokens of context
    blocks that were not selected get zero gradient."""
    L_src, L_ctx, b, D = 50, 45, 8, 6
    rng = np.random.default_rng(5)
    q, k, v = rand_qkv(rng, L_src + L_ctx, D)
    dout = rng.standard_normal(q.shape)
    s = 1 / math.sqrt(D)
    p = O.Params(D=D, L_src=L_src, L_ctx=L_ctx, block=b, alpha_s=0.3, alpha_f=alpha_f, alpha_ns=1.0)
    mask = kept_token_mask(brute_kept(q, k, L_src, L_ctx, b, 0.3, s), L_src, L_ctx, b)
    assert not mask.all()
    got = O.isa_backward(q, k, v, dout, p)
    ref = autograd_attention(q, k, v, dout, s, mask)
    for g, r in zip(got, ref):
        np.testing.assert_allclose(g, r, rtol=1e-11, atol=1e-12)
    assert np.all(got[1][~mask] == 0) and np.all(got[2][~mask] == 0)


@pytest.mark.parametrize("ratios", [(0.125, 0.5, 0.0625), (0.5, 1.0, 0.0), (0.25, 0.75, 0.2)])
def test_identical_keys_taylor_gradients(ratios):
    """Zero in-block key variance: the Taylor output equals exact attention
    over the kept tokens as a function of q and v, so dq and dv are exact
    attention's.  As a function of the keys the pooled column only sees the
    block mean, so per block the sum of dk equals exact attention's."""
    L_src, L_ctx, b, D = 64, 40, 8, 5
    rng = np.random.default_rng(17)
    q, k, v = rand_qkv(rng, L_src + L_ctx, D)
    dout = rng.standard_normal(q.shape)
    T_src = -(-L_src // b)
    for t in range(L_src + L_ctx):
        j = brute_block_of(t, L_src, b)
        k[t] = k[j * b if t < L_src else L_src + (j - T_src) * b]
    a_s, a_f, a_ns = ratios
    s = 1 / math.sqrt(D)
    p = O.Params(D=D, L_src=L_src, L_ctx=L_ctx, block=b, alpha_s=a_s, alpha_f=a_f, alpha_ns=a_ns)
    mask = kept_token_mask(brute_kept(q, k, L_src, L_ctx, b, a_s, s), L_src, L_ctx, b)
    dq, dk, dv = O.isa_backward(q, k, v, dout, p)
    rq, rk, rv = autograd_attention(q, k, v, dout, s, mask)
    np.testing.assert_allclose(dq, rq, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(dv, rv, rtol=1e-10, atol=1e-11)
    blocks = np.array([brute_block_of(t, L_src, b) for t in range(L_src + L_ctx)])
    for j in range(blocks.max() + 1):
        np.testing.assert_allclose(dk[blocks == j].sum(axis=0), rk[blocks == j].sum(axis=0), rtol=1e-10, atol=1e-11)


@pytest.mark.parametrize("ratios", [(0.125, 0.5, 0.0625), (0.4, 0.8, 0.25), (1.0, 1.0, 0.0)])
def test_gradient_sums(ratios):
    """Every output row is a convex combination of value columns and a
    pooled column's gradient is spread over its tokens with weights 1/n_j
    summing to one, so sum_t dv_t = sum_r dout_r; the logit gradients of a
    row add up to zero, so sum_t dk_t = 0."""
    L_src, L_ctx, b, D = 70, 51, 8, 7
    rng = np.random.default_rng(41)
    q, k, v = rand_qkv(rng, L_src + L_ctx, D)
    dout = rng.standard_normal(q.shape)
    a_s, a_f, a_ns = ratios
    p = O.Params(D=D, L_src=L_src, L_ctx=L_ctx, block=b, alpha_s=a_s, alpha_f=a_f, alpha_ns=a_ns)
    dq, dk, dv = O.isa_backward(q, k, v, dout, p)
    np.testing.assert_allclose(dv.sum(axis=0), dout.sum(axis=0), rtol=1e-12, atol=1e-11)
    np.testing.assert_allclose(dk.sum(axis=0), 0.0, atol=1e-11)


def test_batched_backward_is_per_head():
    """[B, H, L, D] inputs: each head planned and differentiated on its own."""
    L_src, L_ctx, b, D = 24, 16, 8, 4
    rng = np.random.default_rng(2)
    x = [rng.standard_normal((2, 3, L_src + L_ctx, D)) for _ in range(4)]
    p = O.Params(D=D, L_src=L_src, L_ctx=L_ctx, block=b, alpha_s=0.5, alpha_f=0.5, alpha_ns=0.25)
    got = O.isa_backward(*x, p)
    for bb in range(2):
        for h in range(3):
            qh, kh, vh, dh = (t[bb, h] for t in x)
            ref = O.backward_head(qh, kh, vh, O.plan_head(qh, kh, vh, p), p, dh)
            for g, r in zip(got, ref):
                assert np.array_equal(g[bb, h], r)
