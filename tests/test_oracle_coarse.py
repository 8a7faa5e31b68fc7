"""Pins of the oracle's gamma * O_coarse residual (paper.rainbus.top summary
card, "Method steps in detail" step (6): a low-frequency residual
gamma * O_coarse added to the scattered output; O_coarse read as the output
of the block-level pooling attention of "Block-sparse attention and pooling
attention", softmax(Qc Kc^T / sqrt(D)) Vc over all blocks, broadcast to each
token of its query block).

Expectations come from loops over tokens and blocks written here, from the
one-token-block case (where the pooled attention is plain attention, pinned
by the forward tests), and from central finite differences.
"""
import math

import numpy as np
import pytest

import oracle as O
from test_oracle import brute_attention, brute_block_of, brute_pool, rand_qkv


def brute_residual(q, k, v, L_src, L_ctx, b, s, gamma):
    Qc, n = brute_pool(q, L_src, L_ctx, b)
    Kc, _ = brute_pool(k, L_src, L_ctx, b)
    Vc, _ = brute_pool(v, L_src, L_ctx, b)
    T = len(n)
    oc = np.zeros_like(Qc)
    for i in range(T):
        logits = [s * float(np.dot(Qc[i], Kc[j])) for j in range(T)]
        m = max(logits)
        w = [math.exp(x - m) for x in logits]
        oc[i] = sum(wj * Vc[j] for wj, j in zip(w, range(T))) / sum(w)
    res = np.zeros_like(q)
    for t in range(L_src + L_ctx):
        res[t] = gamma * oc[brute_block_of(t, L_src, b)]
    return res


@pytest.mark.parametrize("L_src,L_ctx,b,D,gamma", [(48, 40, 16, 8, 0.7), (37, 21, 8, 4, -1.3), (64, 1, 32, 6, 2.0)])
def test_residual_matches_block_loop(L_src, L_ctx, b, D, gamma):
    rng = np.random.default_rng(3)
    q, k, v = rand_qkv(rng, L_src + L_ctx, D)
    p = O.Params(D=D, L_src=L_src, L_ctx=L_ctx, block=b)
    plan = O.plan_head(q, k, v, p)
    got = O.coarse_residual(plan, p, gamma)
    np.testing.assert_allclose(got, brute_residual(q, k, v, L_src, L_ctx, b, 1 / math.sqrt(D), gamma),
                               rtol=1e-12, atol=1e-12)


def test_one_token_blocks_give_dense_attention():
    """b = 1: the pooled means are the tokens, so O_coarse is plain softmax
    attention over all tokens."""
    L_src, L_ctx, D = 13, 9, 5
    rng = np.random.default_rng(4)
    q, k, v = rand_qkv(rng, L_src + L_ctx, D)
    p = O.Params(D=D, L_src=L_src, L_ctx=L_ctx, block=1)
    got = O.coarse_residual(O.plan_head(q, k, v, p), p, 1.0)
    ref, _ = brute_attention(q, k, v, 1 / math.sqrt(D))
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_gamma_zero_is_no_residual():
    rng = np.random.default_rng(5)
    q, k, v = rand_qkv(rng, 40, 4)
    p = O.Params(D=4, L_src=24, L_ctx=16, block=8)
    plan = O.plan_head(q, k, v, p)
    assert not O.coarse_residual(plan, p, 0.0).any()
    dq, dk, dv, dg = O.coarse_residual_backward(plan, p, 0.0, rng.standard_normal((40, 4)))
    assert not (dq.any() or dk.any() or dv.any())
    assert dg != 0.0


@pytest.mark.parametrize("L_src,L_ctx,b,D,gamma", [(22, 13, 8, 4, 0.9), (30, 17, 16, 3, -0.6)])
def test_residual_backward_matches_central_differences(L_src, L_ctx, b, D, gamma):
    rng = np.random.default_rng(6)
    q, k, v = rand_qkv(rng, L_src + L_ctx, D)
    dout = rng.standard_normal(q.shape)
    p = O.Params(D=D, L_src=L_src, L_ctx=L_ctx, block=b)

    def loss(qq, kk, vv, g):
        return float((dout * O.coarse_residual(O.plan_head(qq, kk, vv, p), p, g)).sum())

    dq, dk, dv, dg = O.coarse_residual_backward(O.plan_head(q, k, v, p), p, gamma, dout)
    h = 1e-6
    for which, got in ((0, dq), (1, dk), (2, dv)):
        xs = [q.copy(), k.copy(), v.copy()]
        for idx in np.ndindex(*got.shape):
            x0 = xs[which][idx]
            xs[which][idx] = x0 + h
            fp = loss(*xs, gamma)
            xs[which][idx] = x0 - h
            fm = loss(*xs, gamma)
            xs[which][idx] = x0
            assert abs((fp - fm) / (2 * h) - got[idx]) <= 1e-6 * max(1.0, abs(got[idx])), (which, idx)
    assert abs((loss(q, k, v, gamma + h) - loss(q, k, v, gamma - h)) / (2 * h) - dg) <= 1e-6 * max(1.0, abs(dg))


def test_residual_invariant_to_permutation_within_blocks():
    L_src, L_ctx, b, D = 40, 27, 8, 6
    rng = np.random.default_rng(8)
    q, k, v = rand_qkv(rng, L_src + L_ctx, D)
    p = O.Params(D=D, L_src=L_src, L_ctx=L_ctx, block=b)
    perm = np.arange(L_src + L_ctx)
    for s0 in list(range(0, L_src, b)) + list(range(L_src, L_src + L_ctx, b)):
        e = min(s0 + b, L_src if s0 < L_src else L_src + L_ctx)
        perm[s0:e] = rng.permutation(np.arange(s0, e))
    a = O.coarse_residual(O.plan_head(q, k, v, p), p, 0.5)
    c = O.coarse_residual(O.plan_head(q[perm], k[perm], v[perm], p), p, 0.5)
    np.testing.assert_allclose(a, c, rtol=1e-12, atol=1e-13)
