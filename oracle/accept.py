"""Lossless acceptance of k drafted tokens, the correction draw and the bonus draw, float64.

Test infrastructure (CPU oracle): never imported by the product path.

The rule (the pages cite Leviathan et al., "Fast Inference from Transformers via
Speculative Decoding", for it -- Google blog translation, section "how speculative
decoding works"; Gemma 4 MTP serving guide, section 1 -- and state its property: rejected
tokens are replaced by a token the target generates itself, so the output is
distributionally identical to decoding without a drafter -- "Gemma 4 MTP: drafter drafts,
target verifies", section "basic structure of speculative decoding"):

  target logits z [B, k+1, V], draft logits y [B, k, V], drafts d [B, k].
  p_i = softmax(z[i-1] / T), q_i = softmax(y[i-1] / T) for i = 1..k; p_{k+1} from z[k].
  For i = 1..k: accept d_i iff u_i < p_i(d_i) / q_i(d_i), u_i uniform in [0, 1); stop at
  the first rejection (serving guide, section 4: from the first rejected token on the
  rest of the draft is discarded and the target generates the token itself).
  Rejected at i: emit x ~ norm(max(0, p_i - q_i)) (p_i itself when that is all zero).
  All k accepted: emit the bonus token x ~ p_{k+1} (GeekNews summary, section "how MTP
  works": when the target agrees with the drafts it accepts them and adds one token).
  Outputs: a = accepted count, tokens [d_1 .. d_a, x, -1 ...] of length k+1.

  T = 0 (greedy): accept d_i iff d_i == argmax z[i-1]; emit argmax z[a]; the lowest id
  wins ties.

Readings of points the pages leave open:
  * q(d) = 0 accepts iff p(d) > 0 (the ratio is +inf).
  * Categorical draws are exponential races taken in two levels.  The row's tokens fall in
    groups of GROUP = 512 consecutive ids (the last group ragged).  Level 1 races the groups:
    g* = argmax_g ln W_g - ln E_g over W_g > 0, W_g the sum of the group's weights and
    E_g = -ln(1 - V_g), V_g the group's Philox uniform (philox.group_uniform_rows).  Level 2
    races the tokens of g*: x = argmax ln w_v - ln E_v over w_v > 0, E_v from the per-token
    Philox uniform V_v of the draw's row and purpose.  Lowest index wins ties at both levels.
    An exponential race is an exact categorical draw needing no normalisation, and so is the
    pair: P(g*) = W_g* / W and P(x | g*) = w_x / W_g*.
  * Margins (decisions a float32 implementation may take differently): an acceptance
    with |u - p/q| < MARGIN; a race whose winner's lowest possible key does not beat every
    other competitor's highest possible key by MARGIN, at either level, the key bounds taking
    each weight as w +- REL_P * (p + q) (the float32 error of p - q) and ln E, z / T to within
    ABS_KEY (a group's sums of the token bounds, its key error the largest of its weighted
    tokens'); a greedy argmax whose top two logits differ by less than MARGIN * max(1, |top|).
"""
from __future__ import annotations

import numpy as np

from .philox import accept_uniform, group_uniform_rows, token_uniform_at

GROUP = 512            # tokens per group of the two-level race
MARGIN = 1e-4          # spec margin on |u - p/q|; reused for draws and argmaxes
REL_P = 1e-5           # assumed float32 relative error bound on a probability p_v or q_v
ABS_KEY = 1e-5         # assumed float32 absolute error bound on ln E_v and z_v / T

PURPOSE_ACCEPT = 0
PURPOSE_TARGET = 1
PURPOSE_DRAFTER = 2


def softmax(x: np.ndarray) -> np.ndarray:
    x = np.asarray(x, np.float64)
    m = x.max(axis=-1, keepdims=True)
    e = np.exp(x - m)
    return e / e.sum(axis=-1, keepdims=True)


def race(w: np.ndarray, V: np.ndarray):
    """Exponential race per row: returns (winner ids, ln-keys g)."""
    E = -np.log1p(-V)
    with np.errstate(divide="ignore"):
        g = np.log(w) - np.log(E)
    g = np.where(w > 0, g, -np.inf)
    return np.argmax(g, axis=-1), g


def _race_margin(g_lo: np.ndarray, g_hi: np.ndarray, x: np.ndarray) -> np.ndarray:
    """True where the winner x might lose: its lowest possible key is not MARGIN above the
    highest possible key of every other token."""
    R = g_lo.shape[0]
    hi = g_hi.copy()
    hi[np.arange(R), x] = -np.inf
    return hi.max(axis=-1) > g_lo[np.arange(R), x] - MARGIN


def _group_sum(a: np.ndarray, n_groups: int, reduce=np.sum) -> np.ndarray:
    R, V = a.shape
    pad = np.zeros((R, n_groups * GROUP - V))
    return reduce(np.concatenate([a, pad], axis=1).reshape(R, n_groups, GROUP), axis=-1)


def two_level_race(w, w_lo, w_hi, key_err, seed: int, step: int, rows, purpose: int):
    """Two-level exponential race per row of the weights w [R, V] (bounds w_lo, w_hi and the
    per-token key error key_err for the margin).  Returns (winner ids, margin flags)."""
    w, w_lo, w_hi, key_err = (np.asarray(a, np.float64) for a in (w, w_lo, w_hi, key_err))
    R, V = w.shape
    NG = (V + GROUP - 1) // GROUP
    rows = np.asarray(rows)
    # level 1: the groups
    W, W_lo, W_hi = (_group_sum(a, NG) for a in (w, w_lo, w_hi))
    kerr = _group_sum(np.where(w_hi > 0, key_err, 0.0), NG, np.max)
    lnEg = np.log(-np.log1p(-group_uniform_rows(seed, step, rows, purpose, NG)))
    with np.errstate(divide="ignore", invalid="ignore"):
        G = np.where(W > 0, np.log(W) - lnEg, -np.inf)
        G_hi = np.where(W_hi > 0, np.log(W_hi) - lnEg + kerr, -np.inf)
        G_lo = np.where(W_lo > 0, np.log(W_lo) - lnEg - kerr, -np.inf)
    gs = np.argmax(G, axis=-1)
    margin = _race_margin(G_lo, G_hi, gs)
    # level 2: the tokens of the winning group (ids past the vocabulary carry weight 0)
    ids = gs[:, None] * GROUP + np.arange(min(GROUP, V))[None, :]
    live = ids < V
    idc = np.minimum(ids, V - 1)
    take = lambda a: np.where(live, np.take_along_axis(a, idc, axis=1), 0.0)
    wg, wg_lo, wg_hi, kg = take(w), take(w_lo), take(w_hi), take(key_err)
    lnE = np.log(-np.log1p(-token_uniform_at(seed, step, rows, purpose, ids)))
    with np.errstate(divide="ignore", invalid="ignore"):
        g = np.where(wg > 0, np.log(wg) - lnE, -np.inf)
        g_hi = np.where(wg_hi > 0, np.log(wg_hi) - lnE + kg, -np.inf)
        g_lo = np.where(wg_lo > 0, np.log(wg_lo) - lnE - kg, -np.inf)
    j = np.argmax(g, axis=-1)
    margin |= _race_margin(g_lo, g_hi, j)
    return gs * GROUP + j, margin


def greedy_gap(z: np.ndarray) -> np.ndarray:
    """(top1 - top2) / max(1, |top1|) over the last axis."""
    part = np.partition(z, -2, axis=-1)
    t1, t2 = part[..., -1], part[..., -2]
    return (t1 - t2) / np.maximum(1.0, np.abs(t1))


def accept(z, y, drafts, temperature: float, seed: int, step: int,
           purpose: int = PURPOSE_TARGET):
    """Apply the rule to a batch.  z [B, k+1, V], y [B, k, V] (unused when k = 0 or T = 0),
    drafts [B, k].  Returns dict(n_accepted [B], out_tokens [B, k+1], margin [B] bool)."""
    z = np.asarray(z, np.float64)
    B, n_q, V = z.shape
    k = n_q - 1
    drafts = np.asarray(drafts, np.int64).reshape(B, k)
    n_acc = np.zeros(B, np.int64)
    margin = np.zeros(B, bool)
    bidx = np.arange(B)

    if temperature == 0.0:
        am = np.argmax(z, axis=-1)
        gap = greedy_gap(z)
        active = np.ones(B, bool)
        for i in range(1, k + 1):
            margin |= active & (gap[:, i - 1] < MARGIN)
            ok = active & (drafts[:, i - 1] == am[:, i - 1])
            n_acc += ok
            active = ok
        margin |= gap[bidx, n_acc] < MARGIN
        x = am[bidx, n_acc]
    else:
        T = float(temperature)
        p = softmax(z / T)
        q = softmax(np.asarray(y, np.float64) / T) if k > 0 else None
        rows = bidx * n_q
        active = np.ones(B, bool)
        for i in range(1, k + 1):
            d = drafts[:, i - 1]
            pd = p[bidx, i - 1, d]
            qd = q[bidx, i - 1, d]
            with np.errstate(divide="ignore", invalid="ignore"):
                ratio = np.where(qd > 0, pd / qd, np.where(pd > 0, np.inf, 0.0))
            u = accept_uniform(seed, step, rows + i - 1)
            margin |= active & (np.abs(u - ratio) < MARGIN)
            active = active & (u < ratio)
            n_acc += active
        pa = p[bidx, n_acc]
        za = z[bidx, n_acc] / T
        if k > 0:
            qa = q[bidx, np.minimum(n_acc, k - 1)]
            resid = np.maximum(0.0, pa - qa)
            bonus = n_acc == k
            empty = resid.sum(axis=-1) == 0.0
            use_p = (bonus | empty)[:, None]
            w = np.where(use_p, pa, resid)
            slack = REL_P * (pa + qa)
            w_hi = np.where(use_p, pa, resid + slack)
            w_lo = np.where(use_p, pa, np.maximum(resid - slack, 0.0))
            key_err = np.where(use_p, ABS_KEY * (1.0 + np.abs(za)), ABS_KEY)
        else:
            w = w_hi = w_lo = pa
            key_err = ABS_KEY * (1.0 + np.abs(za))
        # a token of weight exactly 0 (a -inf logit, or an empty residual entry) cannot win
        # on either side: its key bound is -inf (its key error term may be infinite there,
        # and -inf + inf would be NaN and hide the row's other competitors from the check)
        key_err = np.where(w_hi > 0, np.broadcast_to(key_err, w.shape), 0.0)
        x, m = two_level_race(w, w_lo, w_hi, key_err, seed, step, rows + n_acc, purpose)
        margin |= m

    out = np.full((B, n_q), -1, np.int64)
    for b in range(B):
        a = int(n_acc[b])
        out[b, :a] = drafts[b, :a]
        out[b, a] = x[b]
    return dict(n_accepted=n_acc, out_tokens=out, margin=margin)
