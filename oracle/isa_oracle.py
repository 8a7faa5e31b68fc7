"""Plain fp64 CPU oracle of the In-context Sparse Attention (ISA) forward pass.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code,
table or helper with the CUDA library and imports nothing from it.

Source: "LIVEditor-14B: Lightning Unified Video Editing via In-Context Sparse
Attention" (arXiv:2605.04569) as described on
  [R] paper.rainbus.top summary card, sections "Block-sparse attention and
      pooling attention" (块稀疏注意力与 Pooling Attention), "0th-order Taylor
      approximate attention" (0 阶 Taylor 近似注意力), "Core method" (核心方法)
      and "Method steps in detail" (方法步骤详情, steps (1)-(6));
  [T] techwalker.com retelling, sections 4 (the ISA workflow), 5 (block-wise
      0th-order Taylor sparse attention) and 9 (hyper-parameters).

The oracle follows the steps in the order of [R] "Method steps in detail":
  (1) blocking, mean pooling, coarse scores S = Qc Kc^T / sqrt(D)
  (2) context importance (source rows x context columns of S, summed over the
      query dimension) and TopK pre-selection of alpha_s * ceil(L_ctx/b)
      context blocks; kept KV = source KV + selected context KV
  (3) block sharpness M_i, sort descending, the top (1 - alpha_f) share of
      query blocks is "sharp", the rest "flat"
  (4) sharp blocks: exact softmax attention over the kept KV
  (5) flat blocks: for each flat block the alpha_ns share of kept KV blocks
      with the highest coarse score is attended exactly; every other kept
      block contributes exp(q Kc_j^T / sqrt(D)) * Vc_j weighted by its token
      count; one softmax normaliser over both parts
  (6) outputs return to token order; the gamma * O_coarse residual is a
      separate add-on (``coarse_residual``, reading above its definition).
The backward (``backward_head``, ``isa_backward``) differentiates steps
(4)-(6) with the plan held fixed; see the note above ``backward_head``.

Readings of points the pages leave open (every one is switchable where a
second reading is plausible; the defaults are the ones the CUDA path uses):
  * Blocking is per segment: source tokens [0, L_src) and context tokens
    [L_src, L) are cut into blocks of b separately, only each segment's last
    block may be partial, and padding never enters a sum ([R] step (2) counts
    context blocks as ceil(L_ctx/b)).
  * b is a parameter; b=64 is [R] step (1), b=32 is [T] section 5.
  * Sharpness is the population variance of softmax(row i of S) over all T
    block columns (``sharp_cols="all"``, ``sharp_softmax=True``), following
    [R] "Core method"; [R] step (3) writes the variance of the source columns
    of S without a softmax (``sharp_cols="src"``, ``sharp_softmax=False``).
  * Ties: TopK keeps the lower index on equal scores; in the sharpness order
    the lower block index counts as sharper.
  * alpha_f is the share of query blocks on the Taylor path ([R] step (3):
    the top 1 - alpha_f by sharpness stay exact).  [R]'s Fig. 8 caption and
    limitations paragraph and [T] section 9 describe a lower alpha_f as
    sending more blocks to the approximation, the other direction; at the
    default 0.5 both readings give the same split.
  * A flat block's exact blocks are the kept blocks with the largest coarse
    score in its row of S ([R] step (5) names no rule; [T] section 5 lets the
    coarse relevance map decide).
  * alpha_ns counts blocks of the kept KV (``ns_base="kept"``), following [T]
    section 9 (6.25% of KV blocks exact, 93.75% approximated); [R] step (5)
    says "total block count" (``ns_base="all"``: ceil(alpha_ns * T)).
  * The token-count weight n_j of a pooled block multiplies both the
    numerator and the softmax normaliser ([R] step (5) shows it on V_c only;
    without it in the normaliser the result is not a weighted average and the
    zero-in-block-variance case would not be exact).
  * The Taylor part uses each query token, not the pooled query.
  * Context blocks that are not selected take part in neither path.
  * Counts: K_sel = clamp(ceil(alpha_s*T_ctx), 1, T_ctx);
    n_flat = floor(alpha_f*T); n_exact = min(ceil(alpha_ns*T_kv), T_kv),
    each ratio first rounded to float32 (the C interface carries float32).
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence, Tuple

import numpy as np


# ----------------------------------------------------------------------------
# parameters and readings
# ----------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Params:
    D: int
    L_src: int
    L_ctx: int
    block: int = 64
    alpha_s: float = 0.125
    alpha_f: float = 0.5
    alpha_ns: float = 0.0625
    scale: Optional[float] = None           # default 1/sqrt(D)
    sharp_cols: str = "all"                 # "all" | "src" | "kept"
    sharp_softmax: bool = True
    ns_base: str = "kept"                   # "kept" | "all"

    @property
    def L(self) -> int:
        return self.L_src + self.L_ctx

    @property
    def s(self) -> float:
        return 1.0 / math.sqrt(self.D) if self.scale is None else float(self.scale)


def _f32(x: float) -> float:
    return float(np.float32(x))


def n_select(alpha_s: float, T_ctx: int) -> int:
    """Number of kept context blocks, alpha_s * ceil(L_ctx/b) ([R] step (2))."""
    return int(min(max(math.ceil(_f32(alpha_s) * T_ctx), 1), T_ctx))


def n_flat_blocks(alpha_f: float, T: int) -> int:
    """Number of flat query blocks, the alpha_f share ([R] step (3))."""
    return int(min(max(math.floor(_f32(alpha_f) * T), 0), T))


def n_exact_blocks(alpha_ns: float, base: int) -> int:
    """Number of exactly attended KV blocks per flat block ([R] step (5))."""
    return int(min(max(math.ceil(_f32(alpha_ns) * base), 0), base))


# ----------------------------------------------------------------------------
# step (1): blocks, pooling, coarse scores
# ----------------------------------------------------------------------------

def segment_blocks(L_src: int, L_ctx: int, b: int) -> Tuple[np.ndarray, np.ndarray, int, int]:
    """Token start and token count of every block, source blocks first.

    Returns (start[T], count[T], T_src, T_ctx).
    """
    T_src = -(-L_src // b)
    T_ctx = -(-L_ctx // b)
    starts, counts = [], []
    for j in range(T_src):
        starts.append(j * b)
        counts.append(min(b, L_src - j * b))
    for c in range(T_ctx):
        starts.append(L_src + c * b)
        counts.append(min(b, L_ctx - c * b))
    return np.array(starts, np.int64), np.array(counts, np.int64), T_src, T_ctx


def pool(X: np.ndarray, starts: np.ndarray, counts: np.ndarray) -> np.ndarray:
    """Mean of the valid tokens of every block: Xc[j] = (1/n_j) sum_t X[t]."""
    out = np.empty((len(starts), X.shape[1]), np.float64)
    for j, (s0, n) in enumerate(zip(starts, counts)):
        out[j] = X[s0:s0 + n].astype(np.float64).sum(axis=0) / float(n)
    return out


def coarse_scores(Qc: np.ndarray, Kc: np.ndarray, s: float) -> np.ndarray:
    """S_coarse = Qc Kc^T * s, rows = query blocks, columns = key blocks."""
    return (Qc @ Kc.T) * s


# ----------------------------------------------------------------------------
# step (2): context importance and TopK pre-selection
# ----------------------------------------------------------------------------

def context_importance(S: np.ndarray, T_src: int) -> np.ndarray:
    """Sum over the source query rows of the source-row x context-column region."""
    return S[:T_src, T_src:].sum(axis=0)


def topk_lower_index(scores: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest scores, ties broken toward the lower index,
    returned in ascending index order."""
    order = np.lexsort((np.arange(len(scores)), -np.asarray(scores, np.float64)))
    return np.sort(order[:k])


# ----------------------------------------------------------------------------
# step (3): sharpness and the sharp/flat split
# ----------------------------------------------------------------------------

def softmax_rows(S: np.ndarray) -> np.ndarray:
    m = S.max(axis=1, keepdims=True)
    e = np.exp(S - m)
    return e / e.sum(axis=1, keepdims=True)


def sharpness(S: np.ndarray, T_src: int, kept: np.ndarray, cols: str = "all",
              use_softmax: bool = True) -> np.ndarray:
    """Block sharpness M_i: population variance of (softmaxed) row i of S."""
    if cols == "all":
        X = S
    elif cols == "src":
        X = S[:, :T_src]
    elif cols == "kept":
        X = S[:, kept]
    else:
        raise ValueError(cols)
    P = softmax_rows(X) if use_softmax else X
    return P.var(axis=1)


def split_sharp_flat(M: np.ndarray, n_flat: int) -> Tuple[np.ndarray, np.ndarray]:
    """Sort blocks by M descending (lower index first on ties); the first
    T - n_flat are sharp, the remaining n_flat are flat.  Both lists are
    returned in ascending block order."""
    T = len(M)
    order = np.lexsort((np.arange(T), -np.asarray(M, np.float64)))
    sharp = np.sort(order[:T - n_flat])
    flat = np.sort(order[T - n_flat:])
    return sharp, flat


# ----------------------------------------------------------------------------
# the plan of one head
# ----------------------------------------------------------------------------

@dataclasses.dataclass
class HeadPlan:
    starts: np.ndarray        # [T] token start of each block
    counts: np.ndarray        # [T] valid tokens of each block (n_j)
    T_src: int
    T_ctx: int
    Qc: np.ndarray
    Kc: np.ndarray
    Vc: np.ndarray
    S: np.ndarray             # [T, T]
    imp: np.ndarray           # [T_ctx]
    ctx_sel: np.ndarray       # [K_sel] selected context block indices (0-based within context), ascending
    kept: np.ndarray          # [T_kv] kept block ids (source blocks, then selected context blocks)
    M: np.ndarray             # [T] sharpness
    sharp: np.ndarray         # ascending block ids
    flat: np.ndarray          # ascending block ids
    exact: np.ndarray         # [n_flat, n_exact] positions in `kept` (ascending per row)

    @property
    def T(self) -> int:
        return self.T_src + self.T_ctx


def plan_head(q: np.ndarray, k: np.ndarray, v: np.ndarray, p: Params) -> HeadPlan:
    """Steps (1)-(3) and the exact-block choice of step (5) for one head.

    q, k, v: [L, D] arrays of the (bf16-exact) input values.
    """
    starts, counts, T_src, T_ctx = segment_blocks(p.L_src, p.L_ctx, p.block)
    T = T_src + T_ctx
    # (1)
    Qc, Kc, Vc = pool(q, starts, counts), pool(k, starts, counts), pool(v, starts, counts)
    S = coarse_scores(Qc, Kc, p.s)
    # (2)
    imp = context_importance(S, T_src)
    ctx_sel = topk_lower_index(imp, n_select(p.alpha_s, T_ctx))
    kept = np.concatenate([np.arange(T_src), T_src + ctx_sel]).astype(np.int64)
    # (3)
    M = sharpness(S, T_src, kept, p.sharp_cols, p.sharp_softmax)
    sharp, flat = split_sharp_flat(M, n_flat_blocks(p.alpha_f, T))
    # (5) exact-block lists, by coarse score over the kept blocks
    base = len(kept) if p.ns_base == "kept" else T
    n_ex = min(n_exact_blocks(p.alpha_ns, base), len(kept))
    exact = np.zeros((len(flat), n_ex), np.int64)
    for r, i in enumerate(flat):
        exact[r] = topk_lower_index(S[i, kept], n_ex)
    return HeadPlan(starts, counts, T_src, T_ctx, Qc, Kc, Vc, S, imp, ctx_sel, kept, M,
                    sharp, flat, exact)


# ----------------------------------------------------------------------------
# steps (4)-(6): attention
# ----------------------------------------------------------------------------

def _kept_tokens(plan: HeadPlan, blocks: Sequence[int]) -> np.ndarray:
    if len(blocks) == 0:
        return np.zeros(0, np.int64)
    return np.concatenate([np.arange(plan.starts[j], plan.starts[j] + plan.counts[j]) for j in blocks])


def _weighted_average(logits: np.ndarray, values: np.ndarray, log_weights: np.ndarray):
    """Rows of softmax(logits + log_weights) @ values, and log of the normaliser."""
    z = logits + log_weights[None, :]
    m = z.max(axis=1, keepdims=True)
    e = np.exp(z - m)
    den = e.sum(axis=1, keepdims=True)
    return (e @ values) / den, (m + np.log(den))[:, 0]


def sharp_block(q, k, v, plan: HeadPlan, i: int, s: float):
    """Step (4): exact softmax attention of block i's query tokens over every
    token of the kept KV blocks."""
    rows = np.arange(plan.starts[i], plan.starts[i] + plan.counts[i])
    cols = _kept_tokens(plan, plan.kept)
    logits = (q[rows] @ k[cols].T) * s
    return rows, *_weighted_average(logits, v[cols], np.zeros(len(cols)))


def flat_block(q, k, v, plan: HeadPlan, i: int, exact_pos: np.ndarray, s: float):
    """Step (5): exact terms for the chosen kept blocks, count-weighted pooled
    terms exp(s q . Kc_j) * n_j for every other kept block, one normaliser."""
    rows = np.arange(plan.starts[i], plan.starts[i] + plan.counts[i])
    ex_blocks = plan.kept[exact_pos]
    pooled_blocks = np.array([j for j in plan.kept if j not in set(ex_blocks.tolist())], np.int64)
    tok = _kept_tokens(plan, ex_blocks)
    logits_t = (q[rows] @ k[tok].T) * s
    logits_p = (q[rows] @ plan.Kc[pooled_blocks].T) * s if len(pooled_blocks) else np.zeros((len(rows), 0))
    logits = np.concatenate([logits_t, logits_p], axis=1)
    values = np.concatenate([v[tok].astype(np.float64), plan.Vc[pooled_blocks]], axis=0)
    logw = np.concatenate([np.zeros(len(tok)), np.log(plan.counts[pooled_blocks].astype(np.float64))])
    return rows, *_weighted_average(logits, values, logw)


def forward_head(q, k, v, plan: HeadPlan, p: Params, blocks: Optional[Sequence[int]] = None):
    """Output rows (and natural-log softmax normalisers) of one head.

    ``blocks`` restricts the work to a subset of query blocks; rows of other
    blocks are returned as NaN.  Returns (out [L, D], lse [L]).
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    out = np.full((p.L, p.D), np.nan)
    lse = np.full(p.L, np.nan)
    todo = range(plan.T) if blocks is None else blocks
    flat_pos = {int(b): r for r, b in enumerate(plan.flat)}
    for i in todo:
        i = int(i)
        if i in flat_pos:
            rows, o, l = flat_block(q, k, v, plan, i, plan.exact[flat_pos[i]], p.s)
        else:
            rows, o, l = sharp_block(q, k, v, plan, i, p.s)
        out[rows] = o
        lse[rows] = l
    return out, lse


def dense_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, s: float, rows=None):
    """Full softmax attention over all L tokens (what ISA approximates)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    r = np.arange(q.shape[0]) if rows is None else np.asarray(rows)
    logits = (q[r] @ k.T) * s
    o, l = _weighted_average(logits, v, np.zeros(k.shape[0]))
    return o, l


def isa_forward(q: np.ndarray, k: np.ndarray, v: np.ndarray, p: Params):
    """Whole forward over [B, H, L, D] (or [L, D]) fp64 inputs.

    Returns (out, lse, plans) with plans a flat list over the B*H heads.
    """
    q = np.asarray(q, np.float64)
    single = q.ndim == 2
    if single:
        q, k, v = q[None], np.asarray(k)[None], np.asarray(v)[None]
    lead = q.shape[:-2]
    qf = q.reshape(-1, p.L, p.D)
    kf = np.asarray(k, np.float64).reshape(-1, p.L, p.D)
    vf = np.asarray(v, np.float64).reshape(-1, p.L, p.D)
    outs, lses, plans = [], [], []
    for h in range(qf.shape[0]):
        pl = plan_head(qf[h], kf[h], vf[h], p)
        o, l = forward_head(qf[h], kf[h], vf[h], pl, p)
        outs.append(o)
        lses.append(l)
        plans.append(pl)
    out = np.stack(outs).reshape(*lead, p.L, p.D)
    lse = np.stack(lses).reshape(*lead, p.L)
    if single:
        out, lse = out[0], lse[0]
    return out, lse, plans


# ----------------------------------------------------------------------------
# decoupled rotary position embedding (applied to Q and K before step (1))
# ----------------------------------------------------------------------------

def rope_decoupled(x: np.ndarray, L_src: int, L_ctx: int, base: float = 10000.0) -> np.ndarray:
    """Rotary position embedding with per-segment positions ([T] "Decoupled
    RoPE": the reference video's positions restart at 0 instead of continuing
    after the source video; [R] innovation (d): source and context each encode
    positions from 0).

    x: [..., L, D] with L = L_src + L_ctx.  Token l has position l in the
    source segment and l - L_src in the context segment.  Reading of what the
    pages leave open: one-dimensional RoPE over the token index, frequencies
    theta_i = base^(-2i/D) for i = 0..D/2-1, pair i = components (2i, 2i+1)
    rotated by the angle position * theta_i:
        y[2i]   = x[2i] cos(a) - x[2i+1] sin(a)
        y[2i+1] = x[2i] sin(a) + x[2i+1] cos(a).
    fp64 throughout.
    """
    x = np.asarray(x, np.float64)
    L, D = x.shape[-2], x.shape[-1]
    assert L == L_src + L_ctx and D % 2 == 0
    pos = np.concatenate([np.arange(L_src), np.arange(L_ctx)]).astype(np.float64)
    theta = base ** (-2.0 * np.arange(D // 2) / D)
    ang = pos[:, None] * theta[None, :]                     # [L, D/2]
    c, s = np.cos(ang), np.sin(ang)
    xe, xo = x[..., 0::2], x[..., 1::2]
    y = np.empty_like(x)
    y[..., 0::2] = xe * c - xo * s
    y[..., 1::2] = xe * s + xo * c
    return y


# ----------------------------------------------------------------------------
# backward of steps (4)-(6)
# ----------------------------------------------------------------------------
# [R] "Core method" and innovation (c), [T] "Decoupled RoPE" paragraph: the
# method has a forward and a backward implementation and is trained end to
# end.  The pages give no backward formulas; the reading here is the plain
# one: the gradient of the step (4)-(6) output with respect to Q, K and V
# with the plan held fixed.  The plan's choices (kept context blocks, the
# sharp/flat split, the exact lists) are piecewise constant in the inputs and
# carry no gradient; the pooled key/value means of the flat path are
# functions of K and V (Kc_j = mean of the keys of block j), so their
# gradient reaches every token of block j divided by n_j.  The count weight
# n_j is a constant.

def _weighted_average_grad(logits: np.ndarray, values: np.ndarray, log_weights: np.ndarray,
                           dout: np.ndarray):
    """Gradients of rows o = softmax(logits + log_weights) @ values.

    Returns (dlogits, dvalues): with P the softmax and dP = dout values^T,
    dlogits = P * (dP - rowsum(dout * o)) and dvalues = P^T dout.
    """
    z = logits + log_weights[None, :]
    e = np.exp(z - z.max(axis=1, keepdims=True))
    P = e / e.sum(axis=1, keepdims=True)
    o = P @ values
    dP = dout @ values.T
    delta = (dout * o).sum(axis=1, keepdims=True)
    return P * (dP - delta), P.T @ dout


def backward_head(q, k, v, plan: HeadPlan, p: Params, dout, blocks: Optional[Sequence[int]] = None):
    """(dq, dk, dv) [L, D] of one head for the loss sum(dout * out).

    Same columns per query block as ``forward_head``: a sharp block sees
    every token of the kept blocks; a flat block sees the tokens of its exact
    blocks and one pooled column (Kc_j, Vc_j, log-weight ln n_j) per other
    kept block.  The gradients of the pooled columns are gathered per block
    and spread over the block's tokens with weight 1/n_j at the end.
    ``blocks`` restricts the sum to those query blocks (their dq rows are
    then complete; dk, dv hold only their share).
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    dout = np.asarray(dout, np.float64)
    s = p.s
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dKc, dVc = np.zeros((plan.T, p.D)), np.zeros((plan.T, p.D))
    todo = range(plan.T) if blocks is None else blocks
    flat_pos = {int(b): r for r, b in enumerate(plan.flat)}
    for i in todo:
        i = int(i)
        rows = np.arange(plan.starts[i], plan.starts[i] + plan.counts[i])
        if i not in flat_pos:
            cols = _kept_tokens(plan, plan.kept)
            dz, dvals = _weighted_average_grad((q[rows] @ k[cols].T) * s, v[cols], np.zeros(len(cols)), dout[rows])
            dq[rows] += s * (dz @ k[cols])
            dk[cols] += s * (dz.T @ q[rows])
            dv[cols] += dvals
            continue
        ex_blocks = plan.kept[plan.exact[flat_pos[i]]]
        pooled = np.array([j for j in plan.kept if j not in set(ex_blocks.tolist())], np.int64)
        tok = _kept_tokens(plan, ex_blocks)
        nt = len(tok)
        logits = np.concatenate([q[rows] @ k[tok].T, q[rows] @ plan.Kc[pooled].T], axis=1) * s
        values = np.concatenate([v[tok], plan.Vc[pooled]], axis=0)
        logw = np.concatenate([np.zeros(nt), np.log(plan.counts[pooled].astype(np.float64))])
        dz, dvals = _weighted_average_grad(logits, values, logw, dout[rows])
        dq[rows] += s * (dz[:, :nt] @ k[tok] + dz[:, nt:] @ plan.Kc[pooled])
        dk[tok] += s * (dz[:, :nt].T @ q[rows])
        dv[tok] += dvals[:nt]
        dKc[pooled] += s * (dz[:, nt:].T @ q[rows])
        dVc[pooled] += dvals[nt:]
    # Kc_j = (1/n_j) * sum of the keys of block j (and Vc_j likewise)
    for j in range(plan.T):
        t = slice(plan.starts[j], plan.starts[j] + plan.counts[j])
        dk[t] += dKc[j] / plan.counts[j]
        dv[t] += dVc[j] / plan.counts[j]
    return dq, dk, dv


def isa_backward(q, k, v, dout, p: Params):
    """Backward over [B, H, L, D] (or [L, D]) fp64 inputs: plans each head
    from (q, k, v) as ``isa_forward`` does and returns (dq, dk, dv)."""
    q = np.asarray(q, np.float64)
    single = q.ndim == 2
    if single:
        q, k, v, dout = q[None], np.asarray(k)[None], np.asarray(v)[None], np.asarray(dout)[None]
    lead = q.shape[:-2]
    flat = [np.asarray(x, np.float64).reshape(-1, p.L, p.D) for x in (q, k, v, dout)]
    grads = [[], [], []]
    for h in range(flat[0].shape[0]):
        qh, kh, vh, dh = (x[h] for x in flat)
        g = backward_head(qh, kh, vh, plan_head(qh, kh, vh, p), p, dh)
        for a, b in zip(grads, g):
            a.append(b)
    out = [np.stack(g).reshape(*lead, p.L, p.D) for g in grads]
    if single:
        out = [x[0] for x in out]
    return tuple(out)


# ----------------------------------------------------------------------------
# step (6): gamma * O_coarse low-frequency residual
# ----------------------------------------------------------------------------
# [R] step (6) adds gamma * O_coarse to the scattered output as a
# low-frequency residual without defining either.  Reading: O_coarse is the
# output of the block-level (pooling) attention the method already computes
# in step (1) -- [R] "Block-sparse attention and pooling attention":
# attention at low resolution on the pooled means -- i.e. row i of
# softmax(S) Vc over all T blocks, with S = Qc Kc^T * s the coarse scores;
# every token of query block i receives gamma * O_coarse_i.  gamma is a
# scalar the caller supplies (a learned weight in training).

def coarse_output(plan: HeadPlan) -> np.ndarray:
    """O_coarse [T, D]: softmax over all T blocks of each row of the coarse
    scores, times the pooled values."""
    return softmax_rows(plan.S) @ plan.Vc


def coarse_residual(plan: HeadPlan, p: Params, gamma: float) -> np.ndarray:
    """gamma * O_coarse of each token's block, [L, D]."""
    oc = coarse_output(plan)
    res = np.zeros((p.L, p.D))
    for i in range(plan.T):
        res[plan.starts[i]:plan.starts[i] + plan.counts[i]] = gamma * oc[i]
    return res


def coarse_residual_backward(plan: HeadPlan, p: Params, gamma: float, dout):
    """Gradients of sum(dout * coarse_residual) with respect to q, k, v
    ([L, D] each, through the pooled means: 1/n_j per token of block j) and
    to gamma.  O = P Vc with P = softmax(S), S = s Qc Kc^T."""
    dout = np.asarray(dout, np.float64)
    T = plan.T
    P = softmax_rows(plan.S)
    oc = P @ plan.Vc
    dO = np.zeros((T, p.D))
    for i in range(T):
        dO[i] = dout[plan.starts[i]:plan.starts[i] + plan.counts[i]].sum(axis=0)
    dgamma = float((dO * oc).sum())
    dO *= gamma
    dP = dO @ plan.Vc.T
    dS = P * (dP - (dO * oc).sum(axis=1, keepdims=True))
    dQc = p.s * (dS @ plan.Kc)
    dKc = p.s * (dS.T @ plan.Qc)
    dVc = P.T @ dO
    dq, dk, dv = (np.zeros((p.L, p.D)) for _ in range(3))
    for j in range(T):
        t = slice(plan.starts[j], plan.starts[j] + plan.counts[j])
        dq[t] += dQc[j] / plan.counts[j]
        dk[t] += dKc[j] / plan.counts[j]
        dv[t] += dVc[j] / plan.counts[j]
    return dq, dk, dv, dgamma
