"""Pins of the oracle's commit / rollback."""
import numpy as np

from oracle import attention as A
from oracle import commit as C

BS = 4


def test_closed_form_on_contiguous_table():
    B, mb, n_q = 3, 8, 4
    table = np.arange(B * mb).reshape(B, mb)
    L = np.array([0, 5, 17])
    a = np.array([3, 0, 2])
    hidden = np.arange(B * n_q * 2).reshape(B, n_q, 2)
    r = C.commit(L, a, table, BS, n_q, hidden)
    assert r["ctx_len"].tolist() == [4, 6, 20]
    # contiguous table: slot of position p of sequence b is b*mb*BS + p
    for b in range(B):
        exp = [b * mb * BS + L[b] + j if j <= a[b] else -1 for j in range(n_q)]
        assert r["committed_slots"][b].tolist() == exp
    assert r["next_hidden"].tolist() == [hidden[0, 3].tolist(), hidden[1, 0].tolist(),
                                         hidden[2, 2].tolist()]
    assert sorted(p for (b, p, s) in r["rolled_back"] if b == 1) == [6, 7, 8]
    assert len(r["rolled_back"]) == (n_q - 1 - a).sum()


def test_rollback_then_reverify_equals_rebuilt_cache():
    """After committing a prefix, the next verify step reads the same keys as a cache
    built from scratch with only the committed tokens."""
    rng = np.random.default_rng(0)
    hkv, hq, D, n_q = 2, 4, 8, 4
    L0 = 6
    n_tok = L0 + 2 * n_q + 2
    Kseq = rng.standard_normal((n_tok, hkv, D))
    Vseq = rng.standard_normal((n_tok, hkv, D))
    nblk = (n_tok + BS - 1) // BS + 1
    table = rng.permutation(nblk)[None]
    kc = rng.standard_normal((nblk, hkv, BS, D))
    vc = rng.standard_normal((nblk, hkv, BS, D))
    kc, vc = A.append_kv(kc, vc, Kseq[None, :L0], Vseq[None, :L0], table, np.array([0]), BS)
    # verify n_q positions with junk rows past the accepted prefix
    kn = Kseq[None, L0:L0 + n_q].copy()
    vn = Vseq[None, L0:L0 + n_q].copy()
    a = 1
    kn[0, a + 1:] = 1e3
    vn[0, a + 1:] = -1e3
    kc, vc = A.append_kv(kc, vc, kn, vn, table, np.array([L0]), BS)
    r = C.commit(np.array([L0]), np.array([a]), table, BS, n_q)
    L1 = r["ctx_len"]
    assert L1[0] == L0 + a + 1
    q = rng.standard_normal((1, n_q, hq, D))
    kn2, vn2 = Kseq[None, L1[0]:L1[0] + n_q], Vseq[None, L1[0]:L1[0] + n_q]
    out = A.verify_attention(q, kn2, vn2, kc, vc, table, L1, 0, 0.3, BS)
    # rebuilt: fresh cache holding only the committed tokens
    kc2 = np.zeros_like(kc)
    vc2 = np.zeros_like(vc)
    kc2, vc2 = A.append_kv(kc2, vc2, Kseq[None, :L1[0]], Vseq[None, :L1[0]], table,
                           np.array([0]), BS)
    ref = A.verify_attention(q, kn2, vn2, kc2, vc2, table, L1, 0, 0.3, BS)
    np.testing.assert_array_equal(out, ref)
