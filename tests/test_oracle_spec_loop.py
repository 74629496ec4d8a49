"""End-to-end pins of the oracle's verify step on a toy autoregressive target.

The pages' checklist asks to confirm on dozens of samples that speculative output is
identical to plain decoding ("Gemma 4 MTP: drafter drafts, target verifies", section
"operations checklist").  At temperature 0 that is an exact statement: the tokens a
speculative loop emits must equal greedy autoregressive decoding token for token.

The toy target: token x has query/key/value embeddings Eq[x] [h_q, D], Ek[x], Ev[x]
[h_kv, D]; one causal (optionally sliding) GQA attention layer; logits = W . flatten(o).
The autoregressive reference below is written independently of the oracle (dense arrays,
recomputed from scratch each step).  The speculative loop composes the oracle's
verify_attention, lm_head, accept and commit over a shuffled paged cache.
"""
import numpy as np
import pytest

from oracle import accept as ACC
from oracle import attention as A
from oracle import commit as C
from oracle import lm_head as H

BS = 4


class Toy:
    def __init__(self, seed, V=40, hq=4, hkv=2, D=8, window=0):
        rng = np.random.default_rng(seed)
        self.V, self.hq, self.hkv, self.D, self.window = V, hq, hkv, D, window
        self.Eq = rng.standard_normal((V, hq, D))
        self.Ek = rng.standard_normal((V, hkv, D))
        self.Ev = rng.standard_normal((V, hkv, D))
        self.W = rng.standard_normal((V, hq * D)) * 2.0
        self.scale = 1.0 / np.sqrt(D)

    def logits_ar(self, toks):
        """Next-token logits after the sequence ``toks`` (dense, from scratch)."""
        t = len(toks) - 1
        lo = max(0, t - self.window + 1) if self.window > 0 else 0
        o = np.zeros((self.hq, self.D))
        G = self.hq // self.hkv
        for h in range(self.hq):
            s = np.array([self.Eq[toks[t], h] @ self.Ek[toks[p], h // G]
                          for p in range(lo, t + 1)]) * self.scale
            w = np.exp(s - s.max())
            w /= w.sum()
            o[h] = sum(w[i] * self.Ev[toks[lo + i], h // G] for i in range(len(w)))
        return self.W @ o.ravel()


def greedy(toy, prompt, n):
    toks = list(prompt)
    for _ in range(n):
        toks.append(int(np.argmax(toy.logits_ar(toks))))
    return toks[len(prompt):]


def speculative(toy, prompt, n, k, drafter_noise, seed, temperature=0.0):
    rng = np.random.default_rng(seed)
    cap = len(prompt) + n + k + 2
    nblk = (cap + BS - 1) // BS
    table = rng.permutation(nblk)[None, :]
    kc = np.full((nblk, toy.hkv, BS, toy.D), np.nan)
    vc = np.full_like(kc, np.nan)
    # prefill positions 0..len(prompt)-2; the last prompt token is verified with the drafts
    L = len(prompt) - 1
    pre = np.array(prompt[:L])
    if L:
        kc, vc = A.append_kv(kc, vc, toy.Ek[pre][None], toy.Ev[pre][None], table,
                             np.array([0]), BS)
    toks = list(prompt)
    ctx = np.array([L])
    step = 0
    while len(toks) - len(prompt) < n:
        # drafter: noisy copy of the target, greedy
        drafts, seq = [], list(toks)
        for _ in range(k):
            yl = toy.logits_ar(seq) + rng.standard_normal(toy.V) * drafter_noise
            d = int(np.argmax(yl))
            drafts.append(d)
            seq.append(d)
        vt = np.array([toks[-1]] + drafts)
        q, kn, vn = toy.Eq[vt][None], toy.Ek[vt][None], toy.Ev[vt][None]
        o = A.verify_attention(q, kn, vn, kc, vc, table, ctx, toy.window, toy.scale, BS)
        z = H.lm_head(o[0].reshape(k + 1, -1), toy.W)[None]
        r = ACC.accept(z, None, np.array([drafts]), temperature, seed=seed, step=step)
        kc, vc = A.append_kv(kc, vc, kn, vn, table, ctx, BS)
        c = C.commit(ctx, r["n_accepted"], table, BS, k + 1)
        # roll back: poison what was not committed
        for (_, p, s) in c["rolled_back"]:
            kc[s // BS, :, s % BS] = np.nan
            vc[s // BS, :, s % BS] = np.nan
        a = int(r["n_accepted"][0])
        toks += [int(t) for t in r["out_tokens"][0, :a + 1]]
        ctx = c["ctx_len"]
        assert ctx[0] == len(toks) - 1
        step += 1
    return toks[len(prompt):len(prompt) + n]


@pytest.mark.parametrize("seed", range(24))
def test_greedy_equality(seed):
    window = [0, 5][seed % 2]
    k = 1 + seed % 4
    toy = Toy(seed, window=window)
    rng = np.random.default_rng(1000 + seed)
    prompt = list(rng.integers(0, toy.V, size=int(rng.integers(1, 7))))
    n = 14
    ref = greedy(toy, prompt, n)
    out = speculative(toy, prompt, n, k, drafter_noise=[0.0, 1.0, 3.0][seed % 3], seed=seed)
    assert out == ref


def test_perfect_drafter_accepts_everything():
    toy = Toy(99)
    prompt = [3, 1, 4]
    ref = greedy(toy, prompt, 12)
    out = speculative(toy, prompt, 12, 3, drafter_noise=0.0, seed=5)
    assert out == ref
