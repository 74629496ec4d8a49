"""Pins of the oracle's verify attention and drafter cross-attention.

Each pin checks the oracle against something other than its own formula: closed forms
(one key, identical keys), invariants (sliding == global when the window covers
everything, paging-order independence, k+1 queries == k+1 single decodes), and torch's
scaled_dot_product_attention (a library routine) in float64 with an explicit mask.
"""
import numpy as np
import pytest
import torch

from oracle import attention as A

BS = 4


def _setup(seed, B, L, n_q, hq, hkv, D, shuffle=False, extra=2):
    rng = np.random.default_rng(seed)
    need = (np.asarray(L) + n_q + extra + BS - 1) // BS
    mb = int(need.max())
    total = int(need.sum())
    ids = rng.permutation(total) if shuffle else np.arange(total)
    table = np.full((B, mb), -1, np.int64)
    o = 0
    for b in range(B):
        table[b, :need[b]] = ids[o:o + need[b]]
        o += need[b]
    kc = rng.standard_normal((total, hkv, BS, D))
    vc = rng.standard_normal((total, hkv, BS, D))
    q = rng.standard_normal((B, n_q, hq, D))
    kn = rng.standard_normal((B, n_q, hkv, D))
    vn = rng.standard_normal((B, n_q, hkv, D))
    return q, kn, vn, kc, vc, table, np.asarray(L, np.int64)


def _dense_seq(kc, vc, kn, vn, table, L, b):
    """Keys/values of sequence b in position order [L+n_q, hkv, D] after the append."""
    n_q = kn.shape[1]
    pos = np.arange(L[b] + n_q)
    K = np.empty((len(pos), kc.shape[1], kc.shape[3]))
    V = np.empty_like(K)
    for p in pos:
        if p < L[b]:
            K[p] = kc[table[b, p // BS], :, p % BS]
            V[p] = vc[table[b, p // BS], :, p % BS]
        else:
            K[p] = kn[b, p - L[b]]
            V[p] = vn[b, p - L[b]]
    return K, V


def _sdpa(q, K, V, mask, scale):
    """torch SDPA in float64; q [hq, nq, D], K/V [hkv, nk, D], GQA via enable_gqa."""
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(K)[None], torch.from_numpy(V)[None],
        attn_mask=torch.from_numpy(mask)[None, None], scale=scale, enable_gqa=True)[0].numpy()


def test_single_key_gives_value():
    # L = 0, one query: it sees only its own appended key
    q, kn, vn, kc, vc, table, L = _setup(0, 1, [0], 1, 4, 2, 8)
    out = A.verify_attention(q, kn, vn, kc, vc, table, L, 0, 0.3, BS)
    for h in range(4):
        np.testing.assert_allclose(out[0, 0, h], vn[0, 0, h // 2], rtol=0, atol=1e-15)


def test_identical_keys_give_mean_of_values():
    q, kn, vn, kc, vc, table, L = _setup(1, 1, [9], 1, 2, 1, 8)
    kc[:] = 0.7
    kn[:] = 0.7
    out = A.verify_attention(q, kn, vn, kc, vc, table, L, 0, 0.5, BS)
    K, V = _dense_seq(kc, vc, kn, vn, table, L, 0)
    np.testing.assert_allclose(out[0, 0, 0], V[:, 0].mean(axis=0), rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("window", [0, 3, 7])
def test_matches_torch_sdpa_with_mask(window):
    B, n_q, hq, hkv, D = 3, 4, 8, 2, 16
    L = [5, 13, 1]
    q, kn, vn, kc, vc, table, L = _setup(2, B, L, n_q, hq, hkv, D, shuffle=True)
    scale = 1.0 / np.sqrt(D)
    out = A.verify_attention(q, kn, vn, kc, vc, table, L, window, scale, BS)
    for b in range(B):
        K, V = _dense_seq(kc, vc, kn, vn, table, L, b)
        t = L[b] + np.arange(n_q)[:, None]
        p = np.arange(K.shape[0])[None, :]
        mask = p <= t
        if window > 0:
            mask &= p > t - window
        ref = _sdpa(q[b].transpose(1, 0, 2), K.transpose(1, 0, 2), V.transpose(1, 0, 2),
                    mask, scale)
        np.testing.assert_allclose(out[b], ref.transpose(1, 0, 2), rtol=1e-12, atol=1e-12)


def test_window_covering_everything_equals_global():
    q, kn, vn, kc, vc, table, L = _setup(3, 2, [6, 11], 3, 4, 4, 8)
    g = A.verify_attention(q, kn, vn, kc, vc, table, L, 0, 0.4, BS)
    s = A.verify_attention(q, kn, vn, kc, vc, table, L, 100, 0.4, BS)
    np.testing.assert_array_equal(g, s)


def test_shuffled_paging_equals_contiguous():
    a = _setup(4, 2, [7, 10], 3, 4, 2, 8, shuffle=False)
    q, kn, vn, kc, vc, table, L = a
    ref = A.verify_attention(q, kn, vn, kc, vc, table, L, 5, 0.4, BS)
    # move every physical block to a new random location
    perm = np.random.default_rng(9).permutation(kc.shape[0])
    kc2 = np.empty_like(kc)
    vc2 = np.empty_like(vc)
    kc2[perm] = kc
    vc2[perm] = vc
    table2 = np.where(table >= 0, perm[np.maximum(table, 0)], -1)
    out = A.verify_attention(q, kn, vn, kc2, vc2, table2, L, 5, 0.4, BS)
    np.testing.assert_array_equal(out, ref)


def test_k_plus_one_queries_equal_sequential_single_decodes():
    """Verifying n_q positions at once equals n_q one-query steps that each append one
    row: pins the causal mask (query j sees the new keys 0..j, not j+1..)."""
    n_q = 4
    q, kn, vn, kc, vc, table, L = _setup(5, 2, [6, 9], n_q, 4, 2, 8)
    once = A.verify_attention(q, kn, vn, kc, vc, table, L, 6, 0.35, BS)
    kc2, vc2, L2 = kc.copy(), vc.copy(), L.copy()
    for j in range(n_q):
        o = A.verify_attention(q[:, j:j + 1], kn[:, j:j + 1], vn[:, j:j + 1], kc2, vc2,
                               table, L2, 6, 0.35, BS)
        np.testing.assert_allclose(o[:, 0], once[:, j], rtol=1e-13, atol=1e-13)
        kc2, vc2 = A.append_kv(kc2, vc2, kn[:, j:j + 1], vn[:, j:j + 1], table, L2, BS)
        L2 = L2 + 1


def test_append_places_rows_at_their_slots():
    q, kn, vn, kc, vc, table, L = _setup(6, 2, [3, 8], 3, 2, 1, 4, shuffle=True)
    kc2, vc2 = A.append_kv(kc, vc, kn, vn, table, L, BS)
    for b in range(2):
        K, V = _dense_seq(kc2, vc2, kn * 0, vn * 0, table, L + 3, b)
        np.testing.assert_array_equal(K[L[b]:L[b] + 3], kn[b])
        np.testing.assert_array_equal(V[L[b]:L[b] + 3], vn[b])
    # nothing else changed
    changed = np.argwhere(np.any(kc2 != kc, axis=(1, 3)))
    assert len(changed) == 6


@pytest.mark.parametrize("window", [0, 4])
def test_draft_xattn_matches_sdpa_on_committed_keys(window):
    B, hq, hkv, D = 3, 4, 2, 8
    q, kn, vn, kc, vc, table, L = _setup(7, B, [9, 12, 5], 1, hq, hkv, D)
    q_pos = np.array([9, 10, 30])  # beyond, inside and far beyond the committed range
    out = A.draft_attention(q, kc, vc, table, L, q_pos, window, 0.3, BS)
    for b in range(B):
        K, V = _dense_seq(kc, vc, kn[:, :0], vn[:, :0], table, L, b)
        p = np.arange(L[b])[None, :]
        mask = p <= q_pos[b]
        if window > 0:
            mask &= p > q_pos[b] - window
        if not mask.any():
            np.testing.assert_array_equal(out[b, 0], 0.0)
            continue
        ref = _sdpa(q[b].transpose(1, 0, 2), K.transpose(1, 0, 2), V.transpose(1, 0, 2),
                    mask, 0.3)
        np.testing.assert_allclose(out[b], ref.transpose(1, 0, 2), rtol=1e-12, atol=1e-12)


def test_draft_xattn_empty_range_is_zero():
    q, kn, vn, kc, vc, table, L = _setup(8, 1, [0], 1, 2, 1, 4)
    out = A.draft_attention(q, kc, vc, table, L, np.array([0]), 0, 0.5, BS)
    np.testing.assert_array_equal(out, 0.0)


def test_draft_xattn_reads_only_committed_keys():
    """Poisoning everything past L_b does not change the drafter's output."""
    q, kn, vn, kc, vc, table, L = _setup(9, 2, [7, 5], 1, 2, 1, 4)
    ref = A.draft_attention(q, kc, vc, table, L, np.array([20, 20]), 0, 0.5, BS)
    kc2, vc2 = kc.copy(), vc.copy()
    for b in range(2):
        for p in range(L[b], table.shape[1] * BS):
            if table[b, p // BS] >= 0:
                kc2[table[b, p // BS], :, p % BS] = np.nan
                vc2[table[b, p // BS], :, p % BS] = np.nan
    out = A.draft_attention(q, kc2, vc2, table, L, np.array([20, 20]), 0, 0.5, BS)
    np.testing.assert_array_equal(out, ref)
