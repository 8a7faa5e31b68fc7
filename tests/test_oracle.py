"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these checks calls back into the oracle to produce its expectation:
each uses a hand-worked fixture, a brute-force restatement on tiny inputs, a
closed form of a special case, or an invariant.  Source of the method:
"LIVEditor-14B: Lightning Unified Video Editing via In-Context Sparse
Attention", paper.rainbus.top summary card, "Method steps in detail" steps
(1)-(5), "0th-order Taylor approximate attention", "Core method"; the
techwalker.com retelling, sections 3-5 and 9.
"""
import math
import os

import numpy as np
import pytest

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------
# independent brute-force helpers (loops over tokens, no oracle code)
# ----------------------------------------------------------------------------

def brute_block_of(t, L_src, b):
    if t < L_src:
        return t // b
    T_src = -(-L_src // b)
    return T_src + (t - L_src) // b


def brute_pool(X, L_src, L_ctx, b):
    T = -(-L_src // b) + -(-L_ctx // b)
    acc = np.zeros((T, X.shape[1]))
    cnt = np.zeros(T)
    for t in range(L_src + L_ctx):
        j = brute_block_of(t, L_src, b)
        acc[j] += X[t]
        cnt[j] += 1
    return acc / cnt[:, None], cnt


def brute_topk(scores, k):
    idx = sorted(range(len(scores)), key=lambda i: (-scores[i], i))[:k]
    return sorted(idx)


def brute_kept(q, k, L_src, L_ctx, b, alpha_s, s):
    """Context pre-selection restated: importance of context block c is the
    sum over source query blocks i of s * Qc_i . Kc_(T_src+c)."""
    Qc, _ = brute_pool(q, L_src, L_ctx, b)
    Kc, _ = brute_pool(k, L_src, L_ctx, b)
    T_src = -(-L_src // b)
    T_ctx = -(-L_ctx // b)
    imp = []
    for c in range(T_ctx):
        tot = 0.0
        for i in range(T_src):
            tot += s * float(np.dot(Qc[i], Kc[T_src + c]))
        imp.append(tot)
    K_sel = min(max(math.ceil(np.float32(alpha_s) * T_ctx), 1), T_ctx)
    sel = brute_topk(imp, K_sel)
    return list(range(T_src)) + [T_src + c for c in sel]


def kept_token_mask(kept, L_src, L_ctx, b):
    return np.array([brute_block_of(t, L_src, b) in set(kept) for t in range(L_src + L_ctx)])


def brute_attention(q, k, v, s, col_mask=None):
    """Row-by-row softmax attention."""
    L = q.shape[0]
    out = np.zeros((L, v.shape[1]))
    lse = np.zeros(L)
    for t in range(L):
        logits = np.array([s * float(np.dot(q[t], k[u])) for u in range(k.shape[0])])
        if col_mask is not None:
            logits = np.where(col_mask, logits, -np.inf)
        m = logits.max()
        w = np.exp(logits - m)
        out[t] = (w[:, None] * v).sum(axis=0) / w.sum()
        lse[t] = m + math.log(w.sum())
    return out, lse


def rand_qkv(rng, L, D, scale=1.0):
    return [rng.standard_normal((L, D)) * scale for _ in range(3)]


# ----------------------------------------------------------------------------
# the hand-worked fixture
# ----------------------------------------------------------------------------

def load_golden(name):
    env = {"e": math.e, "exp": math.exp, "log": math.log, "__builtins__": {}}
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, expr = line.split("=", 1)
            vals[key.strip()] = eval(expr, env)  # fixture is committed text with plain arithmetic
    return vals


def test_hand_example_every_step():
    g = load_golden("hand_example.txt")
    q, k, v = (np.array(g[n], float) for n in ("q", "k", "v"))
    p = O.Params(D=g["D"], L_src=g["L_src"], L_ctx=g["L_ctx"], block=g["block"],
                 alpha_s=g["alpha_s"], alpha_f=g["alpha_f"], alpha_ns=g["alpha_ns"], scale=g["scale"])
    pl = O.plan_head(q, k, v, p)
    np.testing.assert_array_equal(pl.counts, g["counts"])
    np.testing.assert_allclose(pl.Qc, g["Qc"], atol=1e-15)
    np.testing.assert_allclose(pl.Kc, g["Kc"], atol=1e-15)
    np.testing.assert_allclose(pl.Vc, g["Vc"], atol=1e-15)
    np.testing.assert_allclose(pl.S, g["S"], atol=1e-15)
    np.testing.assert_allclose(pl.imp, g["imp"], atol=1e-15)
    assert pl.ctx_sel.tolist() == g["ctx_sel"]
    assert pl.kept.tolist() == g["kept"]
    T = len(g["E"])
    np.testing.assert_allclose(pl.M, np.array(g["E"]) / T - 1.0 / T ** 2, rtol=1e-12, atol=1e-15)
    assert pl.sharp.tolist() == g["sharp"]
    assert pl.flat.tolist() == g["flat"]
    assert pl.exact.tolist() == g["exact"]
    out, lse = O.forward_head(q, k, v, pl, p)
    np.testing.assert_allclose(out, g["out"], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(lse, g["lse"], rtol=1e-13, atol=1e-13)


# ----------------------------------------------------------------------------
# step (1): blocks and pooling
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("L_src,L_ctx,b", [(64, 64, 16), (70, 33, 16), (5, 3, 4), (1, 1, 32), (100, 7, 32)])
def test_pool_matches_token_loop(L_src, L_ctx, b):
    rng = np.random.default_rng(L_src * 1000 + L_ctx)
    X = rng.standard_normal((L_src + L_ctx, 6))
    starts, counts, T_src, T_ctx = O.segment_blocks(L_src, L_ctx, b)
    ref, cnt = brute_pool(X, L_src, L_ctx, b)
    np.testing.assert_array_equal(counts, cnt)
    assert T_src == -(-L_src // b) and T_ctx == -(-L_ctx // b)
    np.testing.assert_allclose(O.pool(X, starts, counts), ref, rtol=1e-13, atol=1e-14)
    # no block mixes source and context tokens
    for j in range(T_src + T_ctx):
        toks = range(starts[j], starts[j] + counts[j])
        assert len({t < L_src for t in toks}) == 1


# ----------------------------------------------------------------------------
# selection rules
# ----------------------------------------------------------------------------

def test_topk_ties_lower_index():
    rng = np.random.default_rng(3)
    for trial in range(200):
        n = int(rng.integers(1, 40))
        scores = rng.integers(0, 5, size=n).astype(float)     # many ties
        k = int(rng.integers(0, n + 1))
        assert O.topk_lower_index(scores, k).tolist() == brute_topk(scores.tolist(), k)


def test_split_order_and_ties():
    M = np.array([0.3, 0.1, 0.3, 0.2, 0.1, 0.5])
    # sharpness order (descending, lower index first on ties): 5, 0, 2, 3, 1, 4
    sharp, flat = O.split_sharp_flat(M, 3)
    assert sharp.tolist() == [0, 2, 5] and flat.tolist() == [1, 3, 4]
    sharp, flat = O.split_sharp_flat(M, 2)
    assert sharp.tolist() == [0, 2, 3, 5] and flat.tolist() == [1, 4]
    sharp, flat = O.split_sharp_flat(M, 5)
    assert sharp.tolist() == [5] and flat.tolist() == [0, 1, 2, 3, 4]
    sharp, flat = O.split_sharp_flat(M, 0)
    assert flat.tolist() == [] and len(sharp) == 6
    # the boundary inside a tie: of two equal M, the lower block is the sharper
    sharp, flat = O.split_sharp_flat(M, 4)
    assert sharp.tolist() == [0, 5] and flat.tolist() == [1, 2, 3, 4]
    sharp, flat = O.split_sharp_flat(M, 1)
    assert sharp.tolist() == [0, 1, 2, 3, 5] and flat.tolist() == [4]


def test_counts_follow_ratios():
    assert O.n_select(0.125, 256) == 32 and O.n_select(0.125, 186) == 24   # ceil(23.25)
    assert O.n_select(1e-9, 10) == 1 and O.n_select(1.0, 10) == 10
    assert O.n_flat_blocks(0.5, 512) == 256 and O.n_flat_blocks(0.5, 33) == 16
    assert O.n_exact_blocks(0.0625, 288) == 18 and O.n_exact_blocks(0.0625, 210) == 14
    assert O.n_exact_blocks(0.0, 288) == 0 and O.n_exact_blocks(1.0, 288) == 288


def test_default_ratios_are_the_pages_settings():
    """The summary card's "Core method" section states the defaults as
    sparsity rates: the context pre-selection removes 87.5 % of the context
    blocks, half of the query blocks take the Taylor path, and the Taylor
    path is 93.75 % sparse (the techwalker.com retelling, section 9, gives
    alpha_ns = 0.0625); step (1) blocks 64 tokens."""
    p = O.Params(D=64, L_src=1, L_ctx=1)
    assert (1.0 - p.alpha_s, p.alpha_f, 1.0 - p.alpha_ns, p.block) == (0.875, 0.5, 0.9375, 64)


def test_exact_share_counts_the_kept_blocks():
    """alpha_ns is a share of the KV blocks the flat path sees, the kept ones
    (techwalker.com retelling, section 9: alpha_ns = 0.0625 sends 6.25 % of
    the KV blocks to the exact path and the rest to the Taylor path; the KV
    set there is the one left after the context pre-selection).  16 + 16
    tokens in blocks of 2:
    T_src = T_ctx = 8, alpha_s = 0.25 keeps 2 context blocks, so T_kv = 10
    and alpha_ns = 0.25 gives ceil(2.5) = 3 exact blocks per flat block (a
    share of all 16 blocks would give 4).  Exact and pooled blocks split the
    kept set."""
    p = O.Params(L_src=16, L_ctx=16, D=4, block=2, alpha_s=0.25, alpha_f=0.5, alpha_ns=0.25)
    rng = np.random.default_rng(7)
    q, k, v = (rng.standard_normal((32, 4)) for _ in range(3))
    pl = O.plan_head(q, k, v, p)
    assert len(pl.kept) == 10 and len(pl.flat) == 8
    assert pl.exact.shape == (8, 3)
    for row in pl.exact:
        assert len(set(row.tolist())) == 3 and all(0 <= x < 10 for x in row)


# ----------------------------------------------------------------------------
# special cases with closed forms
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("L_src,L_ctx,b,D", [(48, 40, 16, 8), (37, 21, 8, 4)])
def test_no_pruning_no_flat_is_full_attention(L_src, L_ctx, b, D):
    """alpha_s = 1 and alpha_f = 0: every context block kept, every query
    block sharp -> plain softmax attention over all tokens."""
    rng = np.random.default_rng(11)
    q, k, v = rand_qkv(rng, L_src + L_ctx, D)
    p = O.Params(D=D, L_src=L_src, L_ctx=L_ctx, block=b, alpha_s=1.0, alpha_f=0.0, alpha_ns=0.3)
    out, lse, _ = O.isa_forward(q, k, v, p)
    ref, ref_lse = brute_attention(q, k, v, 1 / math.sqrt(D))
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)
    ref2, _ = O.dense_attention(q, k, v, 1 / math.sqrt(D))
    np.testing.assert_allclose(ref2, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("alpha_f", [0.5, 1.0])
def test_alpha_ns_one_is_exact_over_kept(alpha_f):
    """alpha_ns = 1: every kept block of a flat block is exact, so the output
    is exact attention over the kept tokens for every query."""
    L_src, L_ctx, b, D = 50, 45, 8, 6
    rng = np.random.default_rng(5)
    q, k, v = rand_qkv(rng, L_src + L_ctx, D)
    s = 1 / math.sqrt(D)
    p = O.Params(D=D, L_src=L_src, L_ctx=L_ctx, block=b, alpha_s=0.3, alpha_f=alpha_f, alpha_ns=1.0)
    out, lse, plans = O.isa_forward(q, k, v, p)
    kept = brute_kept(q, k, L_src, L_ctx, b, 0.3, s)
    assert plans[0].kept.tolist() == kept
    ref, ref_lse = brute_attention(q, k, v, s, kept_token_mask(kept, L_src, L_ctx, b))
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("ratios", [(0.125, 0.5, 0.0625), (0.5, 1.0, 0.0), (0.25, 0.75, 0.2)])
def test_identical_keys_make_taylor_exact(ratios):
    """Zero in-block key variance (the exact case of the Taylor bound):
    exp(s q.k_t) = exp(s q.Kc) for every token of a block, so the n_j-weighted
    pooled term equals the block's exact contribution and the output is exact
    attention over the kept tokens, whatever the ratios."""
    L_src, L_ctx, b, D = 64, 40, 8, 5
    rng = np.random.default_rng(17)
    q, k, v = rand_qkv(rng, L_src + L_ctx, D)
    for t in range(L_src + L_ctx):
        j = brute_block_of(t, L_src, b)
        first = j * b if t < L_src else L_src + (j - (-(-L_src // b))) * b
        k[t] = k[first]
    a_s, a_f, a_ns = ratios
    s = 1 / math.sqrt(D)
    p = O.Params(D=D, L_src=L_src, L_ctx=L_ctx, block=b, alpha_s=a_s, alpha_f=a_f, alpha_ns=a_ns)
    out, lse, _ = O.isa_forward(q, k, v, p)
    kept = brute_kept(q, k, L_src, L_ctx, b, a_s, s)
    ref, ref_lse = brute_attention(q, k, v, s, kept_token_mask(kept, L_src, L_ctx, b))
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-11, atol=1e-11)


def test_all_flat_no_exact_is_block_pooled_attention():
    """alpha_f = 1, alpha_ns = 0: every query token attends to the kept
    blocks' pooled keys with logits s q.Kc_j + ln n_j and pooled values."""
    L_src, L_ctx, b, D = 45, 30, 8, 4
    rng = np.random.default_rng(23)
    q, k, v = rand_qkv(rng, L_src + L_ctx, D)
    s = 1 / math.sqrt(D)
    p = O.Params(D=D, L_src=L_src, L_ctx=L_ctx, block=b, alpha_s=0.4, alpha_f=1.0, alpha_ns=0.0)
    out, lse, _ = O.isa_forward(q, k, v, p)
    kept = brute_kept(q, k, L_src, L_ctx, b, 0.4, s)
    Kc, n = brute_pool(k, L_src, L_ctx, b)
    Vc, _ = brute_pool(v, L_src, L_ctx, b)
    for t in range(L_src + L_ctx):
        w = np.array([n[j] * math.exp(s * float(np.dot(q[t], Kc[j]))) for j in kept])
        ref = (w[:, None] * Vc[kept]).sum(axis=0) / w.sum()
        np.testing.assert_allclose(out[t], ref, rtol=1e-12, atol=1e-12)
        assert abs(lse[t] - math.log(w.sum())) < 1e-12


# ----------------------------------------------------------------------------
# invariants
# ----------------------------------------------------------------------------

def test_permutation_within_blocks():
    """Permuting tokens inside blocks leaves pooled means, and so every index
    set, unchanged; outputs follow the permutation of the query tokens."""
    L_src, L_ctx, b, D = 40, 27, 8, 6
    rng = np.random.default_rng(29)
    q, k, v = rand_qkv(rng, L_src + L_ctx, D)
    p = O.Params(D=D, L_src=L_src, L_ctx=L_ctx, block=b, alpha_s=0.4, alpha_f=0.5, alpha_ns=0.25)
    out, _, pl = O.isa_forward(q, k, v, p)
    perm = np.arange(L_src + L_ctx)
    starts, counts, _, _ = O.segment_blocks(L_src, L_ctx, b)
    for s0, n in zip(starts, counts):
        perm[s0:s0 + n] = s0 + rng.permutation(n)
    out2, _, pl2 = O.isa_forward(q[perm], k[perm], v[perm], p)
    for a, c in [(pl[0].ctx_sel, pl2[0].ctx_sel), (pl[0].sharp, pl2[0].sharp),
                 (pl[0].flat, pl2[0].flat), (pl[0].exact, pl2[0].exact)]:
        assert np.array_equal(a, c)
    np.testing.assert_allclose(out2, out[perm], rtol=1e-11, atol=1e-12)


def test_variance_identity_and_temperature():
    """M_i = E_i/T - 1/T^2 with E_i = sum_j p_ij^2 (population variance of a
    probability vector), and sharpening the queries by tau > 1 raises every
    E_i (d/dtau sum p^2 = 2 Cov_p(p, x) >= 0 for comonotone p and x)."""
    L_src, L_ctx, b, D = 64, 64, 8, 8
    rng = np.random.default_rng(31)
    q, k, v = rand_qkv(rng, L_src + L_ctx, D)
    p = O.Params(D=D, L_src=L_src, L_ctx=L_ctx, block=b)
    pl = O.plan_head(q, k, v, p)
    T = pl.T
    P = np.exp(pl.S - pl.S.max(axis=1, keepdims=True))
    P /= P.sum(axis=1, keepdims=True)
    E = (P ** 2).sum(axis=1)
    np.testing.assert_allclose(pl.M, E / T - 1.0 / T ** 2, rtol=1e-10, atol=1e-16)
    pl2 = O.plan_head(q * 1.5, k, v, p)
    P2 = np.exp(pl2.S - pl2.S.max(axis=1, keepdims=True))
    P2 /= P2.sum(axis=1, keepdims=True)
    assert np.all((P2 ** 2).sum(axis=1) > E)
    assert np.all(pl2.M > pl.M)


def test_sharpness_readings():
    """The source-columns / no-softmax reading of step (3) is the plain
    variance of S's source columns; 'kept' uses only the kept columns."""
    L_src, L_ctx, b, D = 32, 32, 8, 4
    rng = np.random.default_rng(37)
    q, k, v = rand_qkv(rng, L_src + L_ctx, D)
    p = O.Params(D=D, L_src=L_src, L_ctx=L_ctx, block=b, sharp_cols="src", sharp_softmax=False)
    pl = O.plan_head(q, k, v, p)
    T_src = pl.T_src
    for i in range(pl.T):
        row = pl.S[i, :T_src]
        mean = sum(row) / len(row)
        assert abs(pl.M[i] - sum((x - mean) ** 2 for x in row) / len(row)) < 1e-12
    p3 = O.Params(D=D, L_src=L_src, L_ctx=L_ctx, block=b, ns_base="all", alpha_ns=0.25)
    pl3 = O.plan_head(q, k, v, p3)
    assert pl3.exact.shape[1] == math.ceil(0.25 * pl3.T)


# ----------------------------------------------------------------------------
# Taylor error behaviour (statistical, tiny inputs)
# ----------------------------------------------------------------------------

def clustered(rng, L_src, L_ctx, D, b, sigma):
    L = L_src + L_ctx
    out = []
    blocks = [brute_block_of(t, L_src, b) for t in range(L)]
    T = max(blocks) + 1
    for _ in range(3):
        c = rng.standard_normal((T, D))
        out.append(np.array([c[blocks[t]] + sigma * rng.standard_normal(D) for t in range(L)]))
    return out


def taylor_error(q, k, v, p):
    """Per-row error of ISA against exact attention over the same kept tokens."""
    out, _, plans = O.isa_forward(q, k, v, p)
    kept = plans[0].kept
    mask = np.isin([brute_block_of(t, p.L_src, p.block) for t in range(p.L)], kept)
    ref, _ = brute_attention(q, k, v, p.s, mask)
    return np.abs(out - ref).max(axis=1), plans[0]


def test_taylor_error_grows_with_in_block_variance():
    L_src, L_ctx, b, D = 96, 64, 16, 8
    means = []
    for sigma in (0.05, 0.3, 1.0):
        errs = []
        for seed in range(3):
            rng = np.random.default_rng(100 + seed)
            q, k, v = clustered(rng, L_src, L_ctx, D, b, sigma)
            p = O.Params(D=D, L_src=L_src, L_ctx=L_ctx, block=b, alpha_s=0.5, alpha_f=1.0, alpha_ns=0.0)
            e, _ = taylor_error(q, k, v, p)
            errs.append(e.mean())
        means.append(float(np.mean(errs)))
    assert means[0] < means[1] < means[2], means
    assert means[0] < 0.05 * means[2]


def test_taylor_error_correlates_with_sharpness():
    """Fig. 6 of the paper (as described on the summary card): the Taylor
    error of a block grows with its sharpness M_i.  Checked as a positive
    Spearman rank correlation over blocks of several random heads."""
    L_src, L_ctx, b, D = 128, 64, 16, 8
    Ms, Es = [], []
    for seed in range(6):
        rng = np.random.default_rng(200 + seed)
        q, k, v = clustered(rng, L_src, L_ctx, D, b, 0.5)
        q = q * rng.uniform(0.5, 2.0)
        p = O.Params(D=D, L_src=L_src, L_ctx=L_ctx, block=b, alpha_s=0.5, alpha_f=1.0, alpha_ns=0.0)
        e, pl = taylor_error(q, k, v, p)
        for i in range(pl.T):
            rows = slice(pl.starts[i], pl.starts[i] + pl.counts[i])
            Ms.append(pl.M[i])
            Es.append(e[rows].mean())
    rm = np.argsort(np.argsort(Ms))
    re_ = np.argsort(np.argsort(Es))
    rho = np.corrcoef(rm, re_)[0, 1]
    assert rho > 0.3, rho


def test_flat_path_is_convex_combination():
    """Each flat output is a weighted average of exact values and pooled
    values, so it lies inside the per-dimension range of V."""
    L_src, L_ctx, b, D = 64, 64, 8, 4
    rng = np.random.default_rng(41)
    q, k, v = rand_qkv(rng, L_src + L_ctx, D, 2.0)
    p = O.Params(D=D, L_src=L_src, L_ctx=L_ctx, block=b, alpha_f=1.0, alpha_ns=0.1)
    out, _, _ = O.isa_forward(q, k, v, p)
    assert np.all(out <= v.max(axis=0) + 1e-12) and np.all(out >= v.min(axis=0) - 1e-12)


# ---------------------------------------------------------------------------
# decoupled RoPE
# ---------------------------------------------------------------------------

def test_rope_position_zero_is_identity_in_both_segments():
    rng = np.random.default_rng(5)
    x = rng.normal(size=(9 + 6, 16))
    y = O.rope_decoupled(x, 9, 6)
    assert np.array_equal(y[0], x[0]) and np.array_equal(y[9], x[9])
    assert not np.allclose(y[1], x[1])


def test_rope_preserves_each_pair_norm():
    rng = np.random.default_rng(6)
    x = rng.normal(size=(3, 40, 32))
    y = O.rope_decoupled(x, 25, 15)
    nx = np.hypot(x[..., 0::2], x[..., 1::2])
    ny = np.hypot(y[..., 0::2], y[..., 1::2])
    assert np.abs(nx - ny).max() < 1e-12


def test_rope_scores_depend_only_on_the_position_offset():
    """Rotations compose: <R(m) q, R(n) k> is a function of n - m.  The same q
    and k placed at (m, n) and at (m + s, n + s) give the same score."""
    rng = np.random.default_rng(7)
    D, L = 16, 50
    q0, k0 = rng.normal(size=D), rng.normal(size=D)
    for m, n, s in ((2, 9, 13), (0, 31, 7), (20, 3, 25)):
        x = np.zeros((2, L, D))
        x[0, m], x[1, n] = q0, k0
        x[0, m + s], x[1, n + s] = q0, k0
        y = O.rope_decoupled(x, L, 0)
        a = y[0, m] @ y[1, n]
        b = y[0, m + s] @ y[1, n + s]
        assert abs(a - b) < 1e-10, (m, n, s, a, b)


def test_rope_context_positions_restart_at_zero():
    """A context token at segment position j is rotated exactly like a source
    token at position j (not L_src + j)."""
    rng = np.random.default_rng(8)
    L_src, L_ctx, D = 30, 12, 8
    x = rng.normal(size=(L_src + L_ctx, D))
    x[L_src:] = x[:L_ctx]
    y = O.rope_decoupled(x, L_src, L_ctx)
    assert np.abs(y[L_src:] - y[:L_ctx]).max() < 1e-15


def test_rope_rotation_angle_per_position_step():
    """Measured with atan2: pair i = components (2i, 2i+1) turns
    counter-clockwise by base^(-2i/D) radians per position step."""
    D, L, base = 8, 6, 10000.0
    x = np.zeros((L, D))
    x[:, 0::2] = 1.0                  # every pair starts on the positive first axis
    y = O.rope_decoupled(x, L, 0, base)
    for i in range(D // 2):
        ang = np.arctan2(y[:, 2 * i + 1], y[:, 2 * i])
        step = np.angle(np.exp(1j * np.diff(ang)))
        assert np.allclose(step, base ** (-2.0 * i / D), atol=1e-12), (i, step)
