"""Pins of the oracle's multi-layer target verify (oracle/target.py): closed forms, causality,
equality with position-by-position decoding, the window limit and the layer order."""
import math

import numpy as np

from oracle import attention as A
from oracle import drafter as DR
from oracle import target as T


def _layer(rng, d, hq, hkv, D, F, W=0, scale=0.5):
    return dict(head_dim=D, window=W, g_attn=1 + 0.1 * rng.standard_normal(d),
                Wq=scale * rng.standard_normal((hq * D, d)),
                Wk=scale * rng.standard_normal((hkv * D, d)),
                Wv=scale * rng.standard_normal((hkv * D, d)),
                Wo=scale * rng.standard_normal((d, hq * D)), g_mlp=1 + 0.1 * rng.standard_normal(d),
                Wg=scale * rng.standard_normal((F, d)), Wu=scale * rng.standard_normal((F, d)),
                Wd=scale * rng.standard_normal((d, F)))


def _cache(rng, B, L, hkv, D, bs=4, extra=4):
    nblk = int(sum((l + extra + bs - 1) // bs for l in L))
    perm = rng.permutation(nblk)
    mb = max((l + extra + bs - 1) // bs for l in L)
    table = np.full((B, mb), -1, np.int64)
    i = 0
    for b, l in enumerate(L):
        for j in range((l + extra + bs - 1) // bs):
            table[b, j] = perm[i]
            i += 1
    return dict(k=rng.standard_normal((nblk, hkv, bs, D)), v=rng.standard_normal((nblk, hkv, bs, D)),
                table=table, block_size=bs)


def test_layer_on_an_empty_context_attends_to_its_own_row():
    """L = 0 and one position: the only key is the position's own, so every head of kv group g
    outputs v_new[g] = (W_v rmsnorm(x))[g]; with the MLP off the layer adds W_o of those."""
    rng = np.random.default_rng(0)
    d, hq, hkv, D = 8, 4, 2, 3
    lw = _layer(rng, d, hq, hkv, D, 5)
    lw["Wd"][:] = 0
    cache = _cache(rng, 2, [0, 0], hkv, D)
    x = rng.standard_normal((2, d))
    out, o, kn, vn = T.target_layer(x, lw, cache, np.array([0, 0]), 1, hq, hkv, D, 0)
    v = DR.rmsnorm(x, lw["g_attn"]) @ lw["Wv"].T
    for b in range(2):
        cat = np.concatenate([v[b, (h // (hq // hkv)) * D:(h // (hq // hkv) + 1) * D]
                              for h in range(hq)])
        np.testing.assert_allclose(o[b], cat, rtol=1e-12)
        np.testing.assert_allclose(out[b], x[b] + lw["Wo"] @ cat, rtol=1e-12)


def test_layer_without_output_projections_is_the_identity():
    rng = np.random.default_rng(1)
    lw = _layer(rng, 8, 2, 1, 4, 6)
    lw["Wo"][:] = 0
    lw["Wd"][:] = 0
    cache = _cache(rng, 1, [5], 1, 4)
    x = rng.standard_normal((3, 8))
    out = T.target_layer(x, lw, cache, np.array([5]), 3, 2, 1, 4, 0)[0]
    np.testing.assert_array_equal(out, x)


def test_position_j_does_not_see_later_positions():
    """Changing the input row of the last position leaves the earlier positions' outputs as
    they were (the causal mask over the new positions)."""
    rng = np.random.default_rng(2)
    d, hq, hkv, D, n_q = 8, 4, 2, 4, 3
    lw = _layer(rng, d, hq, hkv, D, 6)
    cache = _cache(rng, 2, [6, 9], hkv, D)
    x = rng.standard_normal((2 * n_q, d))
    y = x.copy()
    y[[2, 5]] += rng.standard_normal((2, d))
    a = T.target_layer(x, lw, cache, np.array([6, 9]), n_q, hq, hkv, D, 0)[0]
    b = T.target_layer(y, lw, cache, np.array([6, 9]), n_q, hq, hkv, D, 0)[0]
    keep = [0, 1, 3, 4]
    np.testing.assert_array_equal(a[keep], b[keep])
    assert np.abs(a[[2, 5]] - b[[2, 5]]).max() > 1e-3


def test_k_plus_one_positions_equal_position_by_position_decoding():
    """The k+1 positions in one pass give what k+1 one-position passes give, each appending its
    own key and value before the next one runs (window and global layers)."""
    rng = np.random.default_rng(3)
    d, hq, hkv, D, n_q, bs = 8, 4, 2, 4, 3, 4
    for W in (0, 4):
        lw = _layer(rng, d, hq, hkv, D, 6, W=W)
        L = np.array([5, 2])
        cache = _cache(rng, 2, L, hkv, D, bs=bs)
        x = rng.standard_normal((2 * n_q, d))
        joint = T.target_layer(x, lw, cache, L, n_q, hq, hkv, D, W)[0]
        kc, vc = cache["k"].copy(), cache["v"].copy()
        for j in range(n_q):
            rows = [b * n_q + j for b in range(2)]
            c = dict(k=kc, v=vc, table=cache["table"], block_size=bs)
            step, _, kn, vn = T.target_layer(x[rows], lw, c, L + j, 1, hq, hkv, D, W)
            np.testing.assert_allclose(step, joint[rows], rtol=1e-10, atol=1e-12)
            kc, vc = A.append_kv(kc, vc, kn, vn, cache["table"], L + j, bs)


def test_window_wider_than_the_context_is_global():
    rng = np.random.default_rng(4)
    d, hq, hkv, D, n_q = 8, 2, 1, 4, 3
    lw = _layer(rng, d, hq, hkv, D, 6)
    L = np.array([7])
    cache = _cache(rng, 1, L, hkv, D)
    x = rng.standard_normal((n_q, d))
    g = T.target_layer(x, lw, cache, L, n_q, hq, hkv, D, 0)[0]
    w = T.target_layer(x, lw, cache, L, n_q, hq, hkv, D, int(L[0]) + n_q)[0]
    np.testing.assert_array_equal(g, w)
    narrow = T.target_layer(x, lw, cache, L, n_q, hq, hkv, D, 2)[0]
    assert np.abs(narrow - g).max() > 1e-3


def test_verify_layers_runs_the_layers_in_order_on_their_own_caches():
    rng = np.random.default_rng(5)
    d, hq, hkv, n_q = 8, 2, 1, 2
    layers = [_layer(rng, d, hq, hkv, 4, 6, W=3), _layer(rng, d, hq, hkv, 8, 6)]
    L = np.array([4, 6])
    caches = [_cache(rng, 2, L, hkv, 4), _cache(rng, 2, L, hkv, 8)]
    x0 = rng.standard_normal((2 * n_q, d))
    out = T.verify_layers(x0, layers, caches, L, n_q, hq, hkv)
    x = x0
    for i, (lw, c) in enumerate(zip(layers, caches)):
        x, o, kn, vn = T.target_layer(x, lw, c, L, n_q, hq, hkv, lw["head_dim"], lw["window"])
        np.testing.assert_array_equal(out["x"][i], x)
        np.testing.assert_array_equal(out["o"][i], o)


def test_attention_scale_is_one_over_root_head_dim():
    """Scaling W_q by sqrt(D) and the head dim's scale cancel: the layer equals one whose
    scores are computed with scale 1 on the scaled queries (checked through the attention
    oracle directly)."""
    rng = np.random.default_rng(6)
    d, hq, hkv, D, n_q = 8, 2, 1, 4, 2
    lw = _layer(rng, d, hq, hkv, D, 6)
    L = np.array([5])
    cache = _cache(rng, 1, L, hkv, D)
    x = rng.standard_normal((n_q, d))
    _, o, kn, vn = T.target_layer(x, lw, cache, L, n_q, hq, hkv, D, 0)
    q = (DR.rmsnorm(x, lw["g_attn"]) @ lw["Wq"].T).reshape(1, n_q, hq, D) / math.sqrt(D)
    ref = A.verify_attention(q, kn, vn, cache["k"], cache["v"], cache["table"], L, 0, 1.0,
                             cache["block_size"])
    np.testing.assert_allclose(o, ref.reshape(n_q, hq * D), rtol=1e-12)
