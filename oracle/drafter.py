"""Drafter dense layers around the drafter's cross-attention, in float64.

Test infrastructure (CPU oracle): never imported by the product path.

What is computed:

* "Gemma 4 MTP: drafter drafts, target verifies", section "drafter internal architecture":
  the drafter owns a token embedder, runs a block of 4 transformer layers (3 sliding-window
  layers and 1 global layer) whose attention reads the target's KV cache, and is fed the
  target's last-layer activation from the previous step together with the drafter
  embedding of the last token; it proposes its k tokens one after another.
* Gemma 4 MTP serving guide, section 4 (execution flow at k = 2): the drafter predicts the
  candidates t+1 and t+2 as a chain, on the shared embedding and the shared KV cache.

Readings where the pages leave the step open (each is the plainest one the rest supports):

* "activation + embedding": the target activation h (target width) and the embedding row e
  (drafter width) are concatenated and projected to the drafter width, x = W_in [h ; e].
* every layer is a pre-norm block with RMSNorm (gain vector, eps 1e-6) and a gated MLP whose
  activation is the tanh form of GELU:
      x += W_o . xattn(W_q . rmsnorm(x, g_attn))
      m  = rmsnorm(x, g_mlp)
      x += W_d . (gelu(W_g . m) * (W_u . m))
* layer order: the three sliding layers, then the global one; a sliding layer reads the
  target's sliding-layer cache and the global layer its global-layer cache; the query of
  chain link j sits at position ctx_len + j.
* the drafter's output row is rmsnorm(x, g_final), the input of its LM head; the next link of
  the chain takes W_back . (that row), a row of target width, in place of the target
  activation.

Functions
  rmsnorm, gelu_tanh, linear, geglu      the dense pieces
  drafter_layer                          one pre-norm block around a cross-attention callback
  drafter_step                           one link of the chain (input projection, 4 layers,
                                         output norm, back projection)
"""
from __future__ import annotations

import math

import numpy as np

from . import attention as A

RMS_EPS = 1e-6


def rmsnorm(x, gain, eps: float = RMS_EPS):
    """x / sqrt(mean(x^2) + eps) * gain over the last axis (float64)."""
    x = np.asarray(x, np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(gain, np.float64)


def gelu_tanh(z):
    """GELU in its tanh form: z/2 * (1 + tanh(sqrt(2/pi) * (z + 0.044715 z^3)))."""
    z = np.asarray(z, np.float64)
    return 0.5 * z * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (z + 0.044715 * z ** 3)))


def linear(x, W):
    """y[r, i] = sum_c x[r, c] W[i, c]  (W stored as [out, in], float64)."""
    return np.asarray(x, np.float64) @ np.asarray(W, np.float64).T


def geglu(m, Wg, Wu):
    """gelu(W_g m) * (W_u m), row by row."""
    return gelu_tanh(linear(m, Wg)) * linear(m, Wu)


def drafter_layer(x, lw, attend):
    """One pre-norm block.  lw holds g_attn, Wq, Wo, g_mlp, Wg, Wu, Wd (float64-able arrays);
    attend(q) maps the projected queries [B, h_q * D] to the attention output [B, h_q * D]."""
    x = np.asarray(x, np.float64)
    q = linear(rmsnorm(x, lw["g_attn"]), lw["Wq"])
    x = x + linear(attend(q), lw["Wo"])
    m = rmsnorm(x, lw["g_mlp"])
    return x + linear(geglu(m, lw["Wg"], lw["Wu"]), lw["Wd"])


def cross_attend(cache, h_q, head_dim, window, ctx_len, j):
    """The attention callback of a drafter layer on one target cache: the query of sequence b
    sits at ctx_len[b] + j and reads that cache's committed keys (oracle.attention)."""
    def attend(q):
        B = q.shape[0]
        qv = q.reshape(B, 1, h_q, head_dim)
        q_pos = np.asarray(ctx_len, np.int64) + j
        o = A.draft_attention(qv, cache["k"], cache["v"], cache["table"], ctx_len, q_pos,
                              window, 1.0 / math.sqrt(head_dim), cache["block_size"])
        return o.reshape(B, h_q * head_dim)
    return attend


def drafter_step(h_prev, tokens, wts, attends, back: bool = True):
    """One link of the drafter chain.

    h_prev  [B, d_target]   target activation (link 0) or the previous link's back projection
    tokens  [B]             last token of each sequence (ids into wts["E"])
    wts     E [V, d_e], W_in [d, d_target + d_e], layers (4 dicts, see drafter_layer),
            g_final [d], W_back [d_target, d]
    attends one attention callback per layer
    Returns x_in, x (after each layer), h (the output row) and, if back, h_back."""
    E = np.asarray(wts["E"])
    e = np.asarray(E[np.asarray(tokens, np.int64)], np.float64)
    x = linear(np.concatenate([np.asarray(h_prev, np.float64), e], axis=1), wts["W_in"])
    out = {"x_in": x, "x": []}
    for lw, attend in zip(wts["layers"], attends):
        x = drafter_layer(x, lw, attend)
        out["x"].append(x)
    h = rmsnorm(x, wts["g_final"])
    out["h"] = h
    if back:
        out["h_back"] = linear(h, wts["W_back"])
    return out
