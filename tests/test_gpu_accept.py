"""GPU parity of sd_accept against the float64 oracle on identical float32 inputs.

Integer outputs must match bit for bit, except sequences the oracle flags as within the
spec margin (|u - p/q| < 1e-4, or a draw / argmax whose best keys are that close);
those are counted and checked for validity only.  The GPU's own margin flags follow the same
error model: every sequence whose GPU outcome differs from the oracle's must be flagged by
both, and the two sets of flags may differ only on decisions at the edge of the margin.
"""
import itertools
import json
import os

import numpy as np
import pytest
import torch
from scipy import stats

import synthetic as S
import verify_step_b200 as sd
from oracle import accept as OACC
from tests.gpu_util import DEV, status_ok, to_dev, workspace

pytestmark = pytest.mark.gpu

NOISE = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "draft_noise.json")))


def gpu_accept(z, y, drafts, T, seed, step, purpose=1):
    B, n_q, V = z.shape
    k = n_q - 1
    desc = sd.AcceptDesc(batch=B, k=k, vocab=V, temperature=float(T), seed=seed, step=step,
                         purpose=purpose)
    n_acc = torch.full((B,), -9, dtype=torch.int32, device=DEV)
    out = torch.full((B, n_q), -9, dtype=torch.int32, device=DEV)
    flags = torch.full((B,), -9, dtype=torch.int32, device=DEV)
    ws = workspace(sd.sd_accept_workspace_size(desc))
    sd.sd_accept(desc, to_dev(z), to_dev(y) if (y is not None and k > 0) else None,
                 to_dev(drafts) if k > 0 else None, n_acc, out, flags, ws)
    torch.cuda.synchronize()
    return n_acc.cpu().numpy(), out.cpu().numpy(), flags.cpu().numpy()


def draw_drafts(y, T, seed, step):
    """Drafts drawn from q = softmax(y / T) by the oracle's own draw (drafter purpose)."""
    B, k, V = y.shape
    d = np.zeros((B, k), np.int64)
    for i in range(k):
        if T == 0:
            d[:, i] = np.argmax(y[:, i].numpy(), axis=-1)
        else:
            r = OACC.accept(y[:, i:i + 1].numpy(), None, np.zeros((B, 0)), T, seed=seed,
                            step=step * 64 + i, purpose=OACC.PURPOSE_DRAFTER)
            d[:, i] = r["out_tokens"][:, 0]
    return torch.from_numpy(d.astype(np.int32))


def compare(z, y, drafts, T, seed, step, purpose=1, max_flag_frac=0.05):
    n_acc, out, gflags = gpu_accept(z, y, drafts, T, seed, step, purpose)
    ref = OACC.accept(z.double().numpy(), None if y is None else y.double().numpy(),
                      drafts.numpy(), T, seed=seed, step=step, purpose=purpose)
    ok = ~ref["margin"]
    assert np.array_equal(n_acc[ok], ref["n_accepted"][ok])
    assert np.array_equal(out[ok], ref["out_tokens"][ok])
    # flagged sequences: outputs still well formed
    B, n_q = out.shape
    for b in np.nonzero(~ok)[0]:
        a = n_acc[b]
        assert 0 <= a < n_q and np.all(out[b, :a] == drafts[b, :a].numpy())
        assert 0 <= out[b, a] < z.shape[-1] and np.all(out[b, a + 1:] == -1)
    assert (~ok).sum() <= max(1, max_flag_frac * len(ok))
    assert np.all((gflags == 0) | (gflags == 1))
    # the GPU flags every sequence it decided differently from the exact rule
    differ = (n_acc != ref["n_accepted"]) | np.any(out != ref["out_tokens"], axis=1)
    assert np.all(gflags[differ] == 1), np.nonzero(differ & (gflags == 0))[0][:10]
    # and its flags agree with the oracle's except at the edge of the margin
    disagree = int(((gflags == 1) != ref["margin"]).sum())
    assert disagree <= max(1, int(1e-3 * len(ok))), (disagree, int(ref["margin"].sum()),
                                                      int(gflags.sum()))
    assert status_ok()
    return n_acc, out, ref


def tuned_inputs(seed, B, k, V=262144):
    z = S.make_logits(seed, B * (k + 1), V).reshape(B, k + 1, V)
    sig = [NOISE["sigma_pos0"]] + [NOISE["sigma_later"]] * (k - 1)
    y = torch.stack([S.perturb(seed * 100 + i, z[:, i], sig[i]) for i in range(k)], dim=1)
    return z, y


@pytest.mark.parametrize("k", [1, 2, 4, 6])
def test_full_vocab_sampling(k):
    """B8, V262144, T=1, draft logits tuned to the serving guide's acceptance."""
    z, y = tuned_inputs(100 + k, 8, k)
    drafts = draw_drafts(y, 1.0, seed=5, step=k)
    compare(z, y, drafts, 1.0, seed=11, step=k)


def test_full_vocab_temperature_and_batch64():
    z, y = tuned_inputs(7, 64, 2)
    drafts = draw_drafts(y, 0.7, seed=6, step=1)
    compare(z, y, drafts, 0.7, seed=12, step=3)


def test_full_vocab_greedy():
    z, y = tuned_inputs(8, 16, 3)
    drafts = draw_drafts(y, 0, seed=0, step=0)
    drafts[::2, 0] = torch.from_numpy(np.argmax(z[::2, 0].numpy(), axis=-1).astype(np.int32))
    n_acc, _, _ = compare(z, None, drafts, 0.0, seed=0, step=0)


def test_drafter_draw_with_masked_logits():
    """k = 0 (the drafter sampling its own token, purpose 2) on clustered-style logits that
    are -inf outside a subset of tokens."""
    B, V = 8, 262144
    z = S.make_logits(9, B, V)
    mask = torch.from_numpy(np.random.default_rng(1).random((B, V)) < 0.03)
    z = torch.where(mask, z, torch.full_like(z, float("-inf"))).reshape(B, 1, V)
    n_acc, out, _ = compare(z, None, torch.zeros(B, 0, dtype=torch.int32), 1.0, seed=3, step=2,
                            purpose=2)
    assert np.all(mask.numpy()[np.arange(B), out[:, 0]])


def test_small_vocab_exact_many_sequences():
    """V=8, k=3, 100000 sequences: every unflagged output equals the oracle."""
    B, k, V = 100_000, 3, 8
    z = S.make_logits(21, B * (k + 1), V, std=1.5).reshape(B, k + 1, V)
    y = torch.stack([S.perturb(22 + i, z[:, i], 1.0) for i in range(k)], dim=1)
    drafts = draw_drafts(y, 1.0, seed=1, step=0)
    compare(z, y, drafts, 1.0, seed=99, step=4, max_flag_frac=0.01)


def _tables(seed, V, k):
    rng = np.random.default_rng(seed)
    P, Q = {}, {}
    for i in range(1, k + 2):
        for pre in itertools.product(range(V), repeat=i - 1):
            zp = rng.standard_normal(V)
            P[pre] = np.exp(zp) / np.exp(zp).sum()
            if i <= k:
                zq = zp + rng.standard_normal(V) * 1.2
                Q[pre] = np.exp(zq) / np.exp(zq).sum()
    return P, Q


def test_gpu_reproduces_target_distribution():
    """The pages' guarantee on the GPU: with 10^6 sequences the first emitted token follows
    p_1 and the first two follow p_1 * p_2 (chi-square, p > 0.01)."""
    V, k, n = 8, 2, 1_000_000
    P, Q = _tables(5, V, k)
    rng = np.random.default_rng(2)
    d = np.zeros((n, k), np.int64)
    d[:, 0] = rng.choice(V, n, p=Q[()])
    for v in range(V):
        s = d[:, 0] == v
        d[s, 1] = rng.choice(V, int(s.sum()), p=Q[(v,)])
    z = np.zeros((n, k + 1, V), np.float32)
    y = np.zeros((n, k, V), np.float32)
    z[:, 0] = np.log(P[()])
    y[:, 0] = np.log(Q[()])
    for v in range(V):
        s = d[:, 0] == v
        z[s, 1] = np.log(P[(v,)])
        y[s, 1] = np.log(Q[(v,)])
        for u in range(V):
            s2 = s & (d[:, 1] == u)
            z[s2, 2] = np.log(P[(v, u)])
    n_acc, out, _ = gpu_accept(torch.from_numpy(z), torch.from_numpy(y),
                               torch.from_numpy(d.astype(np.int32)), 1.0, seed=17, step=0)
    first = np.bincount(out[:, 0], minlength=V)
    assert stats.chisquare(first, P[()] * n).pvalue > 0.01
    # two-token joint over the sequences that emitted >= 2 tokens, compared with the
    # probability of that event per pair: P(e1, e2, a >= 1)
    two = np.zeros((V, V))
    sel = n_acc >= 1
    np.add.at(two, (out[sel, 0], out[sel, 1]), 1)
    exp = np.zeros((V, V))
    for v in range(V):
        alpha = min(1.0, P[()][v] / Q[()][v])
        exp[v] = Q[()][v] * alpha * P[(v,)]  # d1 = v accepted; next token ~ p_2(.|v) exactly
    exp = exp / exp.sum() * two.sum()
    assert stats.chisquare(two.ravel(), exp.ravel()).pvalue > 0.01


def test_step_read_from_device_word():
    """step_ptr set: the counter uses *step_ptr + step (what a graph-replayed loop relies on)."""
    z, y = tuned_inputs(41, 8, 2)
    drafts = draw_drafts(y, 1.0, seed=2, step=9)
    B, n_q, V = z.shape
    counter = torch.tensor([123456], dtype=torch.int64, device=DEV)
    desc = sd.AcceptDesc(batch=B, k=2, vocab=V, temperature=1.0, seed=77, step=1000,
                         purpose=1, step_ptr=counter.data_ptr())
    n_acc = torch.empty(B, dtype=torch.int32, device=DEV)
    out = torch.empty((B, n_q), dtype=torch.int32, device=DEV)
    ws = workspace(sd.sd_accept_workspace_size(desc))
    sd.sd_accept(desc, to_dev(z), to_dev(y), to_dev(drafts), n_acc, out, None, ws)
    torch.cuda.synchronize()
    ref = OACC.accept(z.double().numpy(), y.double().numpy(), drafts.numpy(), 1.0, seed=77,
                      step=123456 + 1000)
    ok = ~ref["margin"]
    assert np.array_equal(n_acc.cpu().numpy()[ok], ref["n_accepted"][ok])
    assert np.array_equal(out.cpu().numpy()[ok], ref["out_tokens"][ok])


def test_plain_draw_dense_rows_twice_on_one_workspace():
    """k = 0 at T = 0.7 on dense rows (every token can win), B = 64: the draw takes no row
    statistics; a second call on the same workspace reuses the per-sequence tickets."""
    B, V = 64, 65536
    z = S.make_logits(12, B, V).reshape(B, 1, V)
    desc = sd.AcceptDesc(batch=B, k=0, vocab=V, temperature=0.7, seed=5, step=3, purpose=2)
    ws = workspace(sd.sd_accept_workspace_size(desc))
    for step in (3, 4):
        desc.step = step
        n_acc = torch.full((B,), -9, dtype=torch.int32, device=DEV)
        out = torch.full((B, 1), -9, dtype=torch.int32, device=DEV)
        sd.sd_accept(desc, to_dev(z), None, None, n_acc, out, None, ws)
        torch.cuda.synchronize()
        ref = OACC.accept(z.double().numpy(), None, np.zeros((B, 0), np.int64), 0.7, seed=5,
                          step=step, purpose=2)
        ok = ~ref["margin"]
        assert (~ok).sum() <= 1
        assert np.array_equal(n_acc.cpu().numpy(), np.zeros(B, np.int32))
        assert np.array_equal(out.cpu().numpy()[ok], ref["out_tokens"][ok])
    assert status_ok()


def _ratio_row(r, V):
    """log p with p(0) = r * q(0) for a uniform q over V tokens (token 1 takes the rest)."""
    p = np.full(V, 1e-12)
    p[0] = r / V
    p[1] = 1.0 - p[0] - (V - 2) * 1e-12
    return np.log(p)


def test_margin_flags_on_constructed_near_ties():
    """Acceptance tests placed 5e-5 and 2e-4 from the row's uniform (either side), and a
    plain draw whose two live tokens' race keys differ by 1e-5 or by 2: the GPU's margin flags
    equal the oracle's, and the unflagged outcomes are the oracle's."""
    from oracle.philox import accept_uniform, token_uniform_rows
    seed, step, V, B = 13, 4, 16, 64
    u = accept_uniform(seed, step, np.arange(B) * 2)
    bs = [b for b in range(B) if 0.05 < u[b] < 0.95][:4]
    z = np.empty((B, 2, V))
    z[:, 0] = _ratio_row(2.0, V)
    z[:, 1] = -50.0
    z[:, 1, 0] = 0.0
    for b, delta in zip(bs, (5e-5, -5e-5, 2e-4, -2e-4)):
        z[b, 0] = _ratio_row((u[b] + delta) * 1.0, V)
    y = np.zeros((B, 1, V))
    zt = torch.from_numpy(z.astype(np.float32))
    yt = torch.from_numpy(y.astype(np.float32))
    drafts = torch.zeros((B, 1), dtype=torch.int32)
    n_acc, out, gflags = gpu_accept(zt, yt, drafts, 1.0, seed, step)
    ref = OACC.accept(zt.double().numpy(), yt.double().numpy(), drafts.numpy(), 1.0, seed=seed,
                      step=step)
    assert ref["margin"][bs].tolist() == [True, True, False, False]
    assert gflags.tolist() == ref["margin"].astype(int).tolist()
    ok = ~ref["margin"]
    assert np.array_equal(n_acc[ok], ref["n_accepted"][ok])
    assert np.array_equal(out[ok], ref["out_tokens"][ok])
    # plain draw over two live tokens
    Vd, seed_d, step_d = 16, 5, 9
    uu = token_uniform_rows(seed_d, step_d, [0, 1], OACC.PURPOSE_DRAFTER, Vd)
    lnE = np.log(-np.log1p(-uu))
    live = (3, 11)
    zd = np.full((2, 1, Vd), -np.inf, np.float32)
    for b, gap in enumerate((1e-5, 2.0)):
        zd[b, 0, live[0]] = 0.3
        zd[b, 0, live[1]] = 0.3 + (lnE[b, live[1]] - lnE[b, live[0]]) + gap
    zdt = torch.from_numpy(zd)
    n_acc, out, gflags = gpu_accept(zdt, None, torch.zeros((2, 0), dtype=torch.int32), 1.0,
                                    seed_d, step_d, purpose=2)
    ref = OACC.accept(zdt.double().numpy(), None, np.zeros((2, 0), np.int64), 1.0, seed=seed_d,
                      step=step_d, purpose=OACC.PURPOSE_DRAFTER)
    assert ref["margin"].tolist() == [True, False]
    assert gflags.tolist() == [1, 0]
    assert out[1, 0] == ref["out_tokens"][1, 0] == live[1]
    assert status_ok()


def test_two_level_draw_over_several_groups_follows_p():
    """Plain draws over 1300 tokens (groups of 512, 512 and a ragged 276, the last carrying
    most of the mass): 200 000 GPU draws follow p (chi-square), and the first 2000 equal the
    oracle's outside the margin."""
    V, n = 1300, 200_000
    rng = np.random.default_rng(31)
    logp = rng.standard_normal(V) * 0.5
    logp[1024:] += 1.2
    p = np.exp(logp) / np.exp(logp).sum()
    z = torch.from_numpy(np.broadcast_to(logp.astype(np.float32), (n, 1, V)).copy())
    n_acc, out, flags = gpu_accept(z, None, torch.zeros(n, 0, dtype=torch.int32), 1.0, seed=9,
                                   step=2, purpose=2)
    counts = np.bincount(out[:, 0], minlength=V)
    assert stats.chisquare(counts, p * n).pvalue > 0.01
    m = 2000
    ref = OACC.accept(z[:m].double().numpy(), None, np.zeros((m, 0), np.int64), 1.0, seed=9,
                      step=2, purpose=2)
    ok = ~ref["margin"]
    assert np.array_equal(out[:m][ok], ref["out_tokens"][ok])
    differ = out[:m, 0] != ref["out_tokens"][:, 0]
    assert np.all(flags[:m][differ] == 1)
    assert status_ok()


def test_residual_draw_over_several_groups_follows_the_residual():
    """k = 1 over 1100 tokens (groups 512, 512, 76) with q heavier than p on the first 600
    tokens: among the rejected sequences the GPU's emitted token follows norm(max(0, p - q))."""
    V, n = 1100, 200_000
    rng = np.random.default_rng(4)
    zp = rng.standard_normal(V).astype(np.float32)
    zq = zp.copy()
    zq[:600] += 1.0
    p = np.exp(zp.astype(np.float64)) / np.exp(zp.astype(np.float64)).sum()
    q = np.exp(zq.astype(np.float64)) / np.exp(zq.astype(np.float64)).sum()
    resid = np.maximum(0.0, p - q)
    resid /= resid.sum()
    z = torch.from_numpy(np.broadcast_to(np.stack([zp, zp]), (n, 2, V)).copy())
    y = torch.from_numpy(np.broadcast_to(zq, (n, 1, V)).copy())
    drafts = torch.from_numpy(rng.choice(V, size=(n, 1), p=q).astype(np.int32))
    n_acc, out, _ = gpu_accept(z, y, drafts, 1.0, seed=23, step=5)
    rej = n_acc == 0
    assert rej.sum() > 30_000
    counts = np.bincount(out[rej, 0], minlength=V)
    exp = resid * rej.sum()
    big = exp >= 5
    obs = np.append(counts[big], counts[~big].sum())
    ex = np.append(exp[big], exp[~big].sum())
    assert stats.chisquare(obs, ex).pvalue > 0.01
    assert status_ok()


def test_group_level_near_tie_is_flagged_on_the_gpu():
    """Two groups of equal-weight tokens whose level-1 keys differ by 1e-5 (both sides flag
    it) or by 2 (neither does); the token comes from the winning group either way."""
    from oracle.philox import group_uniform_rows
    V, seed, step = 1024, 5, 9
    ug = group_uniform_rows(seed, step, [0], OACC.PURPOSE_DRAFTER, 2)[0]
    lnEg = np.log(-np.log1p(-ug))
    for gap, want in ((1e-5, 1), (2.0, 0)):
        lnW1 = lnEg[1] - lnEg[0] + gap
        z = np.empty((1, 1, V), np.float32)
        z[0, 0, :512] = -np.log(512)
        z[0, 0, 512:] = lnW1 - np.log(512)
        n_acc, out, flags = gpu_accept(torch.from_numpy(z), None,
                                       torch.zeros(1, 0, dtype=torch.int32), 1.0, seed=seed,
                                       step=step, purpose=2)
        ref = OACC.accept(z.astype(np.float64), None, np.zeros((1, 0), np.int64), 1.0,
                          seed=seed, step=step, purpose=2)
        assert int(flags[0]) == want == int(ref["margin"][0])
        if not want:
            assert out[0, 0] == ref["out_tokens"][0, 0]
        assert 0 <= out[0, 0] < V
    assert status_ok()
