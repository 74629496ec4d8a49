"""Pins of the oracle's drafter dense layers (oracle/drafter.py) against closed forms,
invariants, a library routine and brute force on tiny inputs."""
import math

import numpy as np
import pytest
from scipy.special import erf

from oracle import attention as A
from oracle import drafter as DR


# ----------------------------------------------------------------------------- RMSNorm

def test_rmsnorm_of_a_constant_row_is_the_gain_times_its_sign():
    g = np.array([0.5, -2.0, 3.0, 1.0])
    for c in (4.0, -0.25):
        out = DR.rmsnorm(np.full((1, 4), c), g)
        want = np.sign(c) * g * abs(c) / math.sqrt(c * c + DR.RMS_EPS)
        np.testing.assert_allclose(out[0], want, rtol=1e-15)


def test_rmsnorm_output_has_unit_mean_square_and_ignores_scale():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((6, 64)) * 3.0
    out = DR.rmsnorm(x, np.ones(64))
    ms = np.mean(x * x, axis=1)
    np.testing.assert_allclose(np.mean(out * out, axis=1), ms / (ms + DR.RMS_EPS), rtol=1e-12)
    np.testing.assert_allclose(DR.rmsnorm(7.5 * x, np.ones(64)), out, rtol=1e-6)


def test_rmsnorm_is_per_row_and_per_column_gain():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((3, 8))
    g = rng.standard_normal(8)
    rows = np.stack([DR.rmsnorm(x[i:i + 1], g)[0] for i in range(3)])
    np.testing.assert_allclose(DR.rmsnorm(x, g), rows, rtol=1e-15)
    np.testing.assert_allclose(DR.rmsnorm(x, g), DR.rmsnorm(x, np.ones(8)) * g, rtol=1e-15)


# ----------------------------------------------------------------------------- GELU

def test_gelu_tanh_is_close_to_the_erf_gelu():
    """The tanh form approximates z * Phi(z) to a few 1e-4 over the real line."""
    z = np.linspace(-8, 8, 4001)
    exact = 0.5 * z * (1 + erf(z / math.sqrt(2)))
    assert np.max(np.abs(DR.gelu_tanh(z) - exact)) < 1e-3


def test_gelu_tanh_odd_part_and_limits():
    """gelu(z) - gelu(-z) = z exactly for the tanh form; gelu(0) = 0; identity far right,
    zero far left."""
    z = np.linspace(-5, 5, 101)
    np.testing.assert_allclose(DR.gelu_tanh(z) - DR.gelu_tanh(-z), z, atol=1e-15)
    assert DR.gelu_tanh(0.0) == 0.0
    assert DR.gelu_tanh(12.0) == pytest.approx(12.0, abs=1e-12)
    assert abs(DR.gelu_tanh(-12.0)) < 1e-12


# ----------------------------------------------------------------------------- linear

def test_linear_matches_brute_force_loops():
    rng = np.random.default_rng(2)
    x, W = rng.standard_normal((3, 5)), rng.standard_normal((4, 5))
    want = [[sum(x[r, c] * W[i, c] for c in range(5)) for i in range(4)] for r in range(3)]
    np.testing.assert_allclose(DR.linear(x, W), np.array(want), rtol=1e-14)


def test_linear_one_entry_picks_one_input_column():
    """W[i, c] = 1 alone makes output column i equal input column c: catches a transpose."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal((4, 7))
    W = np.zeros((5, 7))
    W[2, 6] = 1.0
    y = DR.linear(x, W)
    np.testing.assert_array_equal(y[:, 2], x[:, 6])
    assert not y[:, [0, 1, 3, 4]].any()


def test_geglu_gate_and_up_roles():
    """A large positive gate passes the up projection through times the gate value; a zero
    gate gives zero whatever the up projection: catches swapped gate and up."""
    rng = np.random.default_rng(4)
    m = rng.standard_normal((3, 6))
    Wu = rng.standard_normal((2, 6))
    Wg = np.zeros((2, 6))
    Wg[:, 0] = 1.0
    m[:, 0] = 20.0                      # gate value 20 for every row and feature
    np.testing.assert_allclose(DR.geglu(m, Wg, Wu), 20.0 * (m @ Wu.T), rtol=1e-12)
    assert not DR.geglu(m, np.zeros((2, 6)), Wu).any()
    assert np.any(DR.geglu(m, Wu, Wg) != DR.geglu(m, Wg, Wu))


# ----------------------------------------------------------------------------- one layer

def _layer(rng, d, hq, D, F, scale=1.0):
    return dict(g_attn=1 + 0.1 * rng.standard_normal(d), Wq=scale * rng.standard_normal((hq * D, d)),
                Wo=scale * rng.standard_normal((d, hq * D)), g_mlp=1 + 0.1 * rng.standard_normal(d),
                Wg=scale * rng.standard_normal((F, d)), Wu=scale * rng.standard_normal((F, d)),
                Wd=scale * rng.standard_normal((d, F)))


def test_layer_without_output_projections_is_the_identity():
    rng = np.random.default_rng(5)
    lw = _layer(rng, 8, 2, 4, 6)
    lw["Wo"][:] = 0
    lw["Wd"][:] = 0
    x = rng.standard_normal((3, 8))
    np.testing.assert_array_equal(DR.drafter_layer(x, lw, lambda q: q), x)


def test_layer_attention_branch_with_one_key_is_the_value_row():
    """With one committed key, softmax weights are 1: every head of kv group g outputs V_0[g],
    whatever the query.  The attention branch is then W_o . concat_h V_0[h // G]; the MLP is
    switched off.  Catches the head order of the concatenation and the GQA map."""
    rng = np.random.default_rng(6)
    d, hq, hkv, D, bs = 8, 4, 2, 3, 4
    lw = _layer(rng, d, hq, D, 5)
    lw["Wd"][:] = 0
    kc = rng.standard_normal((2, hkv, bs, D))
    vc = rng.standard_normal((2, hkv, bs, D))
    table = np.array([[1], [0]], np.int32)
    ctx = np.array([1, 1], np.int32)
    cache = dict(k=kc, v=vc, table=table, block_size=bs)
    x = rng.standard_normal((2, d))
    out = DR.drafter_layer(x, lw, DR.cross_attend(cache, hq, D, 0, ctx, 0))
    for b in range(2):
        blk = table[b, 0]
        o = np.concatenate([vc[blk, h // (hq // hkv), 0] for h in range(hq)])
        np.testing.assert_allclose(out[b], x[b] + lw["Wo"] @ o, rtol=1e-12)


def test_layer_mlp_input_is_normalised():
    """The MLP branch reads rmsnorm(x): scaling x leaves it unchanged (attention off)."""
    rng = np.random.default_rng(7)
    lw = _layer(rng, 8, 2, 4, 6)
    lw["Wo"][:] = 0
    x = rng.standard_normal((2, 8))
    d1 = DR.drafter_layer(x, lw, lambda q: q) - x
    d2 = DR.drafter_layer(9.0 * x, lw, lambda q: q) - 9.0 * x
    # equal up to the eps inside the norm (relative 1e-6 on its input); without the norm
    # the branch would change by an order of magnitude
    np.testing.assert_allclose(d1, d2, rtol=1e-4)


def test_layer_attention_query_is_normalised_and_projected():
    """The callback receives W_q . rmsnorm(x, g_attn) (checked with a recording callback)."""
    rng = np.random.default_rng(8)
    lw = _layer(rng, 8, 2, 4, 6)
    x = rng.standard_normal((2, 8))
    seen = []
    DR.drafter_layer(x, lw, lambda q: seen.append(q) or np.zeros_like(q))
    g = lw["g_attn"]
    want = [[sum(lw["Wq"][i, c] * x[r, c] / math.sqrt(np.mean(x[r] ** 2) + DR.RMS_EPS) * g[c]
                 for c in range(8)) for i in range(8)] for r in range(2)]
    np.testing.assert_allclose(seen[0], np.array(want), rtol=1e-12)


# ----------------------------------------------------------------------------- one link

def _weights(rng, d, dt, de, V, hq, Ds, F):
    return dict(E=rng.standard_normal((V, de)), W_in=rng.standard_normal((d, dt + de)),
                layers=[_layer(rng, d, hq, D, F, 0.3) for D in Ds], g_final=np.ones(d),
                W_back=rng.standard_normal((dt, d)))


def test_input_projection_gathers_the_token_embedding():
    """W_in = [0 | I] makes x_in the embedding row of each token; [I | 0] the activation."""
    rng = np.random.default_rng(9)
    d, dt, V = 4, 6, 10
    w = _weights(rng, d, dt, d, V, 1, [2], 3)
    w["layers"] = []
    tokens = np.array([7, 0, 9])
    h = rng.standard_normal((3, dt))
    w["W_in"] = np.concatenate([np.zeros((d, dt)), np.eye(d)], axis=1)
    np.testing.assert_array_equal(DR.drafter_step(h, tokens, w, [])["x_in"], w["E"][tokens])
    w["W_in"] = np.concatenate([np.eye(d, dt), np.zeros((d, d))], axis=1)
    np.testing.assert_array_equal(DR.drafter_step(h, tokens, w, [])["x_in"], h[:, :d])


def test_output_row_and_back_projection():
    rng = np.random.default_rng(10)
    d, dt, V = 4, 6, 10
    w = _weights(rng, d, dt, 3, V, 1, [2], 3)
    w["layers"] = []
    w["g_final"] = rng.standard_normal(d)
    h = rng.standard_normal((2, dt))
    out = DR.drafter_step(h, [1, 2], w, [])
    np.testing.assert_allclose(out["h"], DR.rmsnorm(out["x_in"], w["g_final"]), rtol=1e-15)
    np.testing.assert_allclose(out["h_back"], out["h"] @ w["W_back"].T, rtol=1e-14)
    assert "h_back" not in DR.drafter_step(h, [1, 2], w, [], back=False)


def test_link_runs_the_layers_in_order():
    """Each entry of x is the previous one passed through its own layer and callback."""
    rng = np.random.default_rng(11)
    d, dt = 6, 5
    w = _weights(rng, d, dt, 4, 12, 2, [3, 3, 3, 2], 4)
    calls = []

    def mk(i, D):
        def att(q):
            calls.append(i)
            return np.tanh(q) * (i + 1)
        return att

    atts = [mk(i, D) for i, D in enumerate([3, 3, 3, 2])]
    out = DR.drafter_step(rng.standard_normal((2, dt)), [3, 4], w, atts)
    assert calls == [0, 1, 2, 3]
    x = out["x_in"]
    for i, lw in enumerate(w["layers"]):
        x = DR.drafter_layer(x, lw, atts[i])
        np.testing.assert_array_equal(out["x"][i], x)


def test_cross_attend_callback_matches_the_attention_oracle():
    """The callback places the query at ctx_len + j and reads the committed keys only."""
    rng = np.random.default_rng(12)
    B, hq, hkv, D, bs = 2, 4, 2, 8, 4
    ctx = np.array([5, 9], np.int32)
    kc = rng.standard_normal((8, hkv, bs, D))
    vc = rng.standard_normal((8, hkv, bs, D))
    table = np.array([[3, 0, 5, 6], [1, 2, 4, 7]], np.int32)
    cache = dict(k=kc, v=vc, table=table, block_size=bs)
    q = rng.standard_normal((B, hq * D))
    for j, W in ((0, 0), (1, 3)):
        got = DR.cross_attend(cache, hq, D, W, ctx, j)(q)
        want = A.draft_attention(q.reshape(B, 1, hq, D), kc, vc, table, ctx, ctx + j, W,
                                 1 / math.sqrt(D), bs).reshape(B, hq * D)
        np.testing.assert_array_equal(got, want)
