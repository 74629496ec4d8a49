"""Multi-layer target verify (the target's layers over the k+1 verified positions), in float64.

Test infrastructure (CPU oracle): never imported by the product path.

What is computed:

* "Gemma 4 MTP: drafter drafts, target verifies", section "drafter internal architecture": the
  target checks the k drafted tokens and one more position in one forward pass; Gemma 4 MTP
  serving guide, section 4 (execution flow): the target runs the whole draft sequence through
  one forward pass and compares it with its own distribution; the same guide, section 7: the
  target mixes sliding-window layers (head_dim 256) with global layers (head_dim 512).
* Each layer's attention is the verify attention of oracle.attention: the k+1 new positions
  append their keys and values to the layer's paged cache and attend causally (within the
  window for a sliding layer).

Readings where the pages leave the step open (the same block as the drafter's layers):

* pre-norm blocks with RMSNorm (gain, eps 1e-6) and a gated tanh-GELU MLP:
      a = rmsnorm(x, g_attn);  q = W_q a,  k_new = W_k a,  v_new = W_v a
      x += W_o . verify_attention(q, k_new, v_new)        (keys and values appended)
      m = rmsnorm(x, g_mlp);   x += W_d . (gelu(W_g m) * (W_u m))
* no soft-capping and no query/key norm (the pages name neither); the layer input x is the
  residual stream of the k+1 positions of every sequence (row b (k+1) + j).

Functions
  target_layer     one layer: projections, verify attention with the append, MLP
  verify_layers    the layers in order, each over its own cache
"""
from __future__ import annotations

import math

import numpy as np

from . import attention as A
from .drafter import geglu, linear, rmsnorm


def target_layer(x, lw, cache, ctx_len, n_q, h_q, h_kv, head_dim, window):
    """One layer over rows x [B * n_q, d].  cache: dict(k, v, table, block_size) of this layer
    (float64-indexable); returns (x_out, attention output [B*n_q, h_q*D], k_new, v_new) and the
    cache contents after the append (k, v)."""
    x = np.asarray(x, np.float64)
    B = x.shape[0] // n_q
    a = rmsnorm(x, lw["g_attn"])
    q = linear(a, lw["Wq"]).reshape(B, n_q, h_q, head_dim)
    k_new = linear(a, lw["Wk"]).reshape(B, n_q, h_kv, head_dim)
    v_new = linear(a, lw["Wv"]).reshape(B, n_q, h_kv, head_dim)
    o = A.verify_attention(q, k_new, v_new, cache["k"], cache["v"], cache["table"], ctx_len,
                           window, 1.0 / math.sqrt(head_dim), cache["block_size"])
    o = o.reshape(B * n_q, h_q * head_dim)
    x = x + linear(o, lw["Wo"])
    m = rmsnorm(x, lw["g_mlp"])
    x = x + linear(geglu(m, lw["Wg"], lw["Wu"]), lw["Wd"])
    return x, o, k_new, v_new


def verify_layers(x0, layers, caches, ctx_len, n_q, h_q, h_kv):
    """The layers in order.  layers[i] holds the weights and ``head_dim``, ``window`` of layer
    i; caches[i] its cache.  Returns the residual stream after each layer and each layer's
    attention output and new rows."""
    x = np.asarray(x0, np.float64)
    out = {"x": [], "o": [], "k_new": [], "v_new": []}
    for lw, cache in zip(layers, caches):
        x, o, kn, vn = target_layer(x, lw, cache, ctx_len, n_q, h_q, h_kv, lw["head_dim"],
                                    lw["window"])
        out["x"].append(x)
        out["o"].append(o)
        out["k_new"].append(kn)
        out["v_new"].append(vn)
    return out
