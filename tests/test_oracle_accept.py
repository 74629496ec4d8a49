"""Pins of the oracle's acceptance rule.

* Brute-force enumeration of every outcome of one verify step on a tiny vocabulary, with
  p_i and q_i depending on the drafted prefix, written here independently of the oracle.
  The enumeration itself is checked against the lossless property the pages state (the
  first emitted token is distributed as p_1, the first two as p_1 * p_2), then the
  oracle's Philox-driven outcome frequencies are chi-square tested against it
  (10^6 trials).
* Closed forms: acceptance probability of a draft = sum_v min(p, q) = 1 - TV(p, q).
* Special cases: T = 0 greedy rule; q(d) = 0; p = q (every draft accepted); empty
  residual falls back to p; k = 0 is a plain draw.
"""
import itertools

import numpy as np
import pytest
from scipy import stats

from oracle import accept as ACC


def _tables(seed, V, k, sharp=1.0):
    """Prefix-dependent distributions p_i(.|d_<i), i = 1..k+1 and q_i(.|d_<i), i = 1..k."""
    rng = np.random.default_rng(seed)
    P, Q = {}, {}
    for i in range(1, k + 2):
        for pre in itertools.product(range(V), repeat=i - 1):
            zp = rng.standard_normal(V) * sharp
            P[pre] = np.exp(zp) / np.exp(zp).sum()
            if i <= k:
                zq = zp + rng.standard_normal(V) * 1.2
                Q[pre] = np.exp(zq) / np.exp(zq).sum()
    return P, Q


def _enumerate(P, Q, V, k):
    """Exact probability of every outcome (a, d_1..d_a, x) of one verify step."""
    out = {}

    def walk(pre, mass):
        j = len(pre)
        p, q = P[pre], (Q[pre] if j < k else None)
        if j == k:  # all accepted: bonus from p_{k+1}
            for x in range(V):
                out[(j, pre, x)] = out.get((j, pre, x), 0.0) + mass * p[x]
            return
        alpha = np.minimum(1.0, p / q)
        for x in range(V):  # rejection at position j+1: sum_d q(d)(1-alpha(d)) * w(x)/sum w
            w = np.maximum(0.0, p - q)
            rej = np.sum(q * (1 - alpha))
            if rej > 0:
                out[(j, pre, x)] = out.get((j, pre, x), 0.0) + mass * rej * w[x] / w.sum()
        for d in range(V):  # accept d_{j+1}
            walk(pre + (d,), mass * q[d] * alpha[d])

    walk((), 1.0)
    return out


@pytest.mark.parametrize("V,k", [(4, 1), (4, 3), (8, 2)])
def test_enumeration_is_lossless(V, k):
    P, Q = _tables(V * 10 + k, V, k)
    E = _enumerate(P, Q, V, k)
    assert abs(sum(E.values()) - 1.0) < 1e-12
    first = np.zeros(V)
    for (a, pre, x), pr in E.items():
        first[pre[0] if a >= 1 else x] += pr
    np.testing.assert_allclose(first, P[()], rtol=0, atol=1e-12)
    # joint of the first two emitted tokens; a step that emits one token is continued by
    # a step whose first token is ~ p_2(.|e1) (the single-token identity above)
    two = np.zeros((V, V))
    for (a, pre, x), pr in E.items():
        seq = list(pre) + [x]
        if len(seq) >= 2:
            two[seq[0], seq[1]] += pr
        else:
            two[seq[0]] += pr * P[(seq[0],)]
    ref = P[()][:, None] * np.stack([P[(v,)] for v in range(V)])
    np.testing.assert_allclose(two, ref, rtol=0, atol=1e-12)


def _sample_drafts(rng, Q, V, k, n):
    d = np.zeros((n, k), np.int64)
    for i in range(k):
        for pre in itertools.product(range(V), repeat=i):
            sel = np.all(d[:, :i] == np.array(pre, np.int64), axis=1) if i else np.ones(n, bool)
            m = int(sel.sum())
            if m:
                d[sel, i] = rng.choice(V, size=m, p=Q[pre])
    return d


def _logits_for(P, Q, drafts, V, k, T):
    n = drafts.shape[0]
    z = np.zeros((n, k + 1, V))
    y = np.zeros((n, k, V))
    for i in range(k + 1):
        for pre in itertools.product(range(V), repeat=i):
            sel = np.all(drafts[:, :i] == np.array(pre, np.int64), axis=1) if i else np.ones(n, bool)
            z[sel, i] = T * np.log(P[pre])
            if i < k:
                y[sel, i] = T * np.log(Q[pre])
    return z, y


@pytest.mark.parametrize("V,k,T", [(8, 2, 1.0), (4, 3, 0.7)])
def test_oracle_frequencies_match_enumeration(V, k, T):
    P, Q = _tables(V * 10 + k, V, k)
    E = _enumerate(P, Q, V, k)
    keys = sorted(E)
    index = {key: i for i, key in enumerate(keys)}
    counts = np.zeros(len(keys))
    first = np.zeros(V)
    n_total, chunk = 1_000_000, 250_000
    rng = np.random.default_rng(123)
    for c in range(n_total // chunk):
        drafts = _sample_drafts(rng, Q, V, k, chunk)
        z, y = _logits_for(P, Q, drafts, V, k, T)
        r = ACC.accept(z, y, drafts, T, seed=77, step=c)
        a, toks = r["n_accepted"], r["out_tokens"]
        for b in range(chunk):
            ab = int(a[b])
            counts[index[(ab, tuple(int(t) for t in toks[b, :ab]), int(toks[b, ab]))]] += 1
        np.add.at(first, toks[:, 0], 1)
    expect = np.array([E[key] for key in keys]) * n_total
    big = expect >= 5
    obs = np.append(counts[big], counts[~big].sum())
    exp = np.append(expect[big], expect[~big].sum())
    if exp[-1] == 0:
        obs, exp = obs[:-1], exp[:-1]
    assert stats.chisquare(obs, exp).pvalue > 0.01
    # the pages' guarantee: the first emitted token follows p_1
    assert stats.chisquare(first, P[()] * n_total).pvalue > 0.01


def test_acceptance_rate_closed_form():
    V, n = 8, 400_000
    rng = np.random.default_rng(3)
    p = rng.dirichlet(np.ones(V))
    q = rng.dirichlet(np.ones(V))
    drafts = rng.choice(V, size=(n, 1), p=q)
    z = np.broadcast_to(np.log(p), (n, 2, V))
    y = np.broadcast_to(np.log(q), (n, 1, V))
    r = ACC.accept(z, y, drafts, 1.0, seed=5, step=0)
    rate = r["n_accepted"].mean()
    alpha = np.minimum(p, q).sum()
    assert abs(alpha - (1 - 0.5 * np.abs(p - q).sum())) < 1e-15
    assert abs(rate - alpha) < 4 * np.sqrt(alpha * (1 - alpha) / n)


def test_greedy_rule():
    z = np.array([[[0, 5, 1, 5], [2, 0, 0, 1], [0, 0, 3, 0]],     # argmax ties -> id 1
                  [[9, 0, 0, 0], [0, 7, 0, 0], [0, 0, 0, 4]]], float)
    drafts = np.array([[1, 0], [0, 1]])
    r = ACC.accept(z, None, drafts, 0.0, seed=0, step=0)
    assert r["n_accepted"].tolist() == [2, 2]
    assert r["out_tokens"].tolist() == [[1, 0, 2], [0, 1, 3]]
    r = ACC.accept(z, None, np.array([[3, 0], [0, 2]]), 0.0, seed=0, step=0)
    assert r["n_accepted"].tolist() == [0, 1]
    assert r["out_tokens"].tolist() == [[1, -1, -1], [0, 1, -1]]
    assert bool(r["margin"][0])  # row 0 of sequence 0 has a tie at the top


def test_identical_distributions_accept_everything():
    V, n = 16, 2000
    rng = np.random.default_rng(4)
    z = rng.standard_normal((n, 3, V))
    drafts = rng.integers(0, V, (n, 2))
    r = ACC.accept(z, z[:, :2], drafts, 1.0, seed=1, step=2)
    assert np.all(r["n_accepted"] == 2)
    assert np.all(r["out_tokens"][:, :2] == drafts)


def test_zero_draft_probability_and_empty_residual():
    # q(d) = 0 with p(d) > 0 accepts; a rejected row with p == q falls back to p
    z = np.log(np.array([[[0.5, 0.5, 0.0001], [0.2, 0.3, 0.5]]]))
    y = np.array([[[0.0, 0.0, -np.inf]]])
    r = ACC.accept(z, y, np.array([[2]]), 1.0, seed=3, step=0)
    assert r["n_accepted"][0] == 1
    # p = q everywhere except the drafted token has q > p -> residual on others only
    V, n = 6, 20000
    p = np.full(V, 1 / V)
    q = p.copy()
    q[0] += 0.1
    q[1:] -= 0.1 / 5
    z = np.broadcast_to(np.log(p), (n, 2, V))
    y = np.broadcast_to(np.log(q), (n, 1, V))
    r = ACC.accept(z, y, np.zeros((n, 1), np.int64), 1.0, seed=9, step=0)
    rej = r["n_accepted"] == 0
    assert rej.sum() > 0
    assert np.all(r["out_tokens"][rej, 0] != 0)


def test_k0_is_a_plain_draw_from_p():
    V, n = 5, 200_000
    p = np.array([0.1, 0.2, 0.3, 0.05, 0.35])
    z = np.broadcast_to(np.log(p), (n, 1, V))
    r = ACC.accept(z, None, np.zeros((n, 0), np.int64), 1.0, seed=2, step=9,
                   purpose=ACC.PURPOSE_DRAFTER)
    assert np.all(r["n_accepted"] == 0)
    counts = np.bincount(r["out_tokens"][:, 0], minlength=V)
    assert stats.chisquare(counts, p * n).pvalue > 0.01


def test_race_picks_unique_positive_weight_and_prefers_lower_id_on_ties():
    w = np.array([[0.0, 0.0, 3.0, 0.0], [1.0, 1.0, 0.0, 0.0]])
    V = np.array([[0.5, 0.5, 0.9, 0.1], [0.25, 0.25, 0.1, 0.1]])
    x, g = ACC.race(w, V)
    assert x.tolist() == [2, 0]


def test_masked_tokens_do_not_hide_a_near_tie():
    """A plain draw over a row whose other tokens are masked (-inf logits), with the two live
    tokens' logits set so that their race keys differ by 1e-5 (flagged) or by 2 (not
    flagged).  Zero-weight tokens have key -inf; an infinite key error on them must not turn
    the row's competitor bound into NaN."""
    from oracle.philox import token_uniform_rows
    V, seed, step = 16, 5, 9
    live = (3, 11)
    u = token_uniform_rows(seed, step, [0], ACC.PURPOSE_DRAFTER, V)[0]
    lnE = np.log(-np.log1p(-u))
    for gap, want in ((1e-5, True), (2.0, False)):
        z = np.full((1, 1, V), -np.inf)
        z[0, 0, live[0]] = 0.3
        z[0, 0, live[1]] = 0.3 + (lnE[live[1]] - lnE[live[0]]) + gap  # key difference = gap
        r = ACC.accept(z, None, np.zeros((1, 0), np.int64), 1.0, seed=seed, step=step,
                       purpose=ACC.PURPOSE_DRAFTER)
        assert bool(r["margin"][0]) is want, gap
        assert r["out_tokens"][0, 0] == live[1]


def _ratio_row(r, V=4):
    """log p for a row with p(0) = r * q(0) under a uniform q over V tokens: token 0 gets r / V,
    token 1 almost all the rest, the others a negligible 1e-12 each (so a residual draw after
    a rejection at token 0 has a single token of clearly positive weight)."""
    p = np.full(V, 1e-12)
    p[0] = r / V
    p[1] = 1.0 - p[0] - (V - 2) * 1e-12
    return np.log(p)


def test_acceptance_margin_is_the_absolute_gap_between_u_and_the_ratio():
    """The spec margin: a decision with |u - p(d)/q(d)| < 1e-4 is flagged, one 2e-4 away
    is not, on either side of u; the gap is absolute (a sequence whose u is small has a
    relative gap far above 1e-4 but is still flagged); u is the uniform of the decision's own
    row b * (k + 1) + i - 1, so a near-tie built on that row's u is seen only by that row."""
    from oracle.philox import accept_uniform
    seed, step, V, B = 13, 4, 4, 64
    u = accept_uniform(seed, step, np.arange(B) * 2)
    small = int(np.argmin(u))
    assert u[small] < 0.05
    cases = {small: (5e-5, True)}
    others = [b for b in range(B) if b != small and 0.05 < u[b] < 0.95][:4]
    for b, delta in zip(others, (5e-5, -5e-5, 2e-4, -2e-4)):
        cases[b] = (delta, abs(delta) < 1e-4)
    bs = sorted(cases)
    z = np.empty((B, 2, V))
    z[:, 0] = _ratio_row(2.0)       # sequences not under test: ratio 2, always accepted
    z[:, 1] = [0.0, -50.0, -50.0, -50.0]   # bonus row: one token dominates the draw
    for b in bs:
        z[b, 0] = _ratio_row(u[b] + cases[b][0])
    y = np.zeros((B, 1, V))         # q uniform: q(0) = 1/4
    r = ACC.accept(z, y, np.zeros((B, 1), np.int64), 1.0, seed=seed, step=step)
    for b in bs:
        delta, want = cases[b]
        assert bool(r["margin"][b]) is want, (b, u[b], delta)
        assert r["n_accepted"][b] == (1 if delta > 0 else 0)
    rest = [b for b in range(B) if b not in cases]
    assert not r["margin"][rest].any()


def test_acceptance_margin_ignores_decisions_never_taken():
    """k = 2: a near-tie at draft 2 is flagged when draft 1 was accepted, and not flagged when
    draft 1 was rejected (draft 2 is then never tested)."""
    from oracle.philox import accept_uniform
    seed, step, V, B = 21, 7, 4, 32
    u = accept_uniform(seed, step, np.arange(B * 3)).reshape(B, 3)
    bs = [b for b in range(B) if 0.05 < u[b, 0] < 0.95 and 0.05 < u[b, 1] < 0.95][:2]
    assert len(bs) == 2
    z = np.empty((B, 3, V))
    z[:, 0] = _ratio_row(2.0)
    z[:, 1] = _ratio_row(2.0)
    z[:, 2] = [0.0, -50.0, -50.0, -50.0]
    acc_b, rej_b = bs
    z[acc_b, 0] = _ratio_row(2.0)                   # draft 1 accepted (|u - 2| > 1)
    z[rej_b, 0] = _ratio_row(u[rej_b, 0] / 2)       # draft 1 rejected, far from the margin
    for b in bs:
        z[b, 1] = _ratio_row(u[b, 1] + 5e-5)        # near-tie at draft 2 (row b * 3 + 1)
    y = np.zeros((B, 2, V))
    r = ACC.accept(z, y, np.zeros((B, 2), np.int64), 1.0, seed=seed, step=step)
    assert r["n_accepted"][rej_b] == 0 and not r["margin"][rej_b]
    assert r["n_accepted"][acc_b] == 2 and r["margin"][acc_b]
    assert r["out_tokens"][rej_b, 0] == 1          # the residual's only positive token


def test_two_level_draw_is_exact_over_several_groups():
    """A plain draw over 700 tokens: two groups of the two-level race (512 and a ragged 188),
    the second holding most of the mass.  The Philox-driven frequencies of 60 000 draws (one
    logit row each) follow p: a group weight that dropped a term, a wrong group boundary or a
    lost ragged tail would bias whole groups."""
    V, n = 700, 60_000
    rng = np.random.default_rng(7)
    logp = rng.standard_normal(V) * 0.5
    logp[512:] += 1.5                      # group 1 (188 tokens) carries about 60 % of p
    p = np.exp(logp) / np.exp(logp).sum()
    assert 0.5 < p[512:].sum() < 0.8
    z = np.broadcast_to(logp, (n, 1, V))
    r = ACC.accept(z, None, np.zeros((n, 0), np.int64), 1.0, seed=11, step=3,
                   purpose=ACC.PURPOSE_DRAFTER)
    counts = np.bincount(r["out_tokens"][:, 0], minlength=V)
    assert stats.chisquare(counts, p * n).pvalue > 0.01
    # the group split alone: group 1's share is binomial around its mass
    share = counts[512:].sum() / n
    assert abs(share - p[512:].sum()) < 4 * np.sqrt(p[512:].sum() * (1 - p[512:].sum()) / n)


def test_residual_draw_over_several_groups_follows_the_residual():
    """k = 1 over 1100 tokens (groups of 512, 512, 76): among the rejected sequences the
    emitted token follows norm(max(0, p - q)), whose mass sits in different groups than p's."""
    V, n = 1100, 40_000
    rng = np.random.default_rng(3)
    zp = rng.standard_normal(V)
    zq = zp.copy()
    zq[:600] += 1.0                        # q over-weights the first groups: residual elsewhere
    p = np.exp(zp) / np.exp(zp).sum()
    q = np.exp(zq) / np.exp(zq).sum()
    resid = np.maximum(0.0, p - q)
    resid /= resid.sum()
    z = np.empty((n, 2, V))
    z[:, 0] = zp
    z[:, 1] = zp
    y = np.broadcast_to(zq, (n, 1, V))
    drafts = rng.choice(V, size=(n, 1), p=q)
    r = ACC.accept(z, y, drafts, 1.0, seed=23, step=1)
    rej = r["n_accepted"] == 0
    assert rej.sum() > 5000
    counts = np.bincount(r["out_tokens"][rej, 0], minlength=V)
    exp = resid * rej.sum()
    big = exp >= 5
    obs = np.append(counts[big], counts[~big].sum())
    ex = np.append(exp[big], exp[~big].sum())
    assert stats.chisquare(obs, ex).pvalue > 0.01


def test_group_level_near_tie_is_flagged():
    """Two groups of equal-weight tokens whose level-1 keys differ by 1e-5 (flagged) or by 2
    (not flagged); the winning group is the one with the larger key either way."""
    from oracle.philox import group_uniform_rows
    V, seed, step = 1024, 5, 9
    ug = group_uniform_rows(seed, step, [0], ACC.PURPOSE_DRAFTER, 2)[0]
    lnEg = np.log(-np.log1p(-ug))
    for gap, want in ((1e-5, True), (2.0, False)):
        # ln W_1 - lnE_1 = ln W_0 - lnE_0 + gap, tokens equal inside each group
        lnW0 = 0.0
        lnW1 = lnW0 + lnEg[1] - lnEg[0] + gap
        z = np.empty((1, 1, V))
        z[0, 0, :512] = lnW0 - np.log(512)
        z[0, 0, 512:] = lnW1 - np.log(512)
        r = ACC.accept(z, None, np.zeros((1, 0), np.int64), 1.0, seed=seed, step=step,
                       purpose=ACC.PURPOSE_DRAFTER)
        assert 512 <= r["out_tokens"][0, 0] < 1024
        if want:
            assert r["margin"][0]
        else:
            # not flagged by level 1; level 2 over 512 equal weights rarely ties within 1e-4
            G = np.log(np.exp(z[0, 0]).reshape(2, 512).sum(-1)) - lnEg
            assert G[1] - G[0] > 1.9
            assert not r["margin"][0]
