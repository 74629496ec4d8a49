"""Verify attention and drafter cross-attention over a paged KV cache, in float64.

Test infrastructure (CPU oracle): never imported by the product path.

What is computed (plain definition):

* Verify attention -- "Gemma 4 MTP: drafter drafts, target verifies", section "drafter
  internal architecture": the target checks k drafts plus one position, k+1 positions, in
  one forward pass; Gemma 4 MTP serving guide, section 4 "execution flow": the target
  compares the whole draft sequence with its own distribution in one forward pass.
  For sequence b with committed length L_b the n_q = k+1 new positions L_b .. L_b+k are
  appended to the cache; query j sits at absolute position t = L_b + j and attends
  causally to keys p in [lo, t], lo = max(0, t - W + 1) for a sliding layer of window W
  (W keys including its own position) and lo = 0 for a global layer.  Query head h
  reads kv head floor(h / G), G = h_q / h_kv.  out = softmax(scale * q.K^T) . V.
* Drafter cross-attention -- same page, section "drafter internal architecture" (each
  drafter layer attends directly into the target's KV cache); Google blog as summarised
  by GeekNews, section "MTP drafter internal optimisations" (the drafter shares the
  target's KV cache): one query at logical position q_pos[b] attends the committed keys
  p in [lo, min(q_pos, L_b - 1)], lo relative to q_pos as above; nothing is written.
  An empty key range gives a zero output.

Cache layout: [num_blocks, h_kv, block_size, D]; logical position p of sequence b lives in
physical block block_table[b, p // bs] at row p % bs.
"""
from __future__ import annotations

import numpy as np


def key_range(t: int, window: int, last: int):
    """Positions a query at absolute position t may read, capped at ``last``."""
    lo = max(0, t - window + 1) if window > 0 else 0
    return lo, min(t, last)


def gather_rows(cache: np.ndarray, block_table: np.ndarray, b: int, g: int,
                positions: np.ndarray, block_size: int) -> np.ndarray:
    """Rows [len(positions), D] of kv head g of sequence b from a paged cache."""
    blk = block_table[b, positions // block_size]
    return cache[blk, g, positions % block_size]


def softmax_attend(qv: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """softmax(scale * K.q) . V for one query vector, float64."""
    if K.shape[0] == 0:
        return np.zeros(V.shape[1], np.float64)
    s = scale * (K @ qv)
    s = s - s.max()
    w = np.exp(s)
    w = w / w.sum()
    return w @ V


def verify_attention_one(b, j, h, q, k_new, v_new, k_cache, v_cache, block_table, ctx_len,
                         window, scale, block_size):
    """Output of query j, head h of sequence b (the cache holds keys before L_b; keys of
    the new positions come from k_new / v_new, which is what appending them gives)."""
    G = q.shape[2] // k_cache.shape[1]
    g = h // G
    L = int(ctx_len[b])
    t = L + j
    lo, hi = key_range(t, window, t)
    old = np.arange(lo, min(hi + 1, L))
    new = np.arange(max(lo, L), hi + 1) - L
    K = np.concatenate([gather_rows(k_cache, block_table, b, g, old, block_size),
                        k_new[b, new, g]], axis=0)
    V = np.concatenate([gather_rows(v_cache, block_table, b, g, old, block_size),
                        v_new[b, new, g]], axis=0)
    return softmax_attend(q[b, j, h], K, V, scale)


def verify_attention(q, k_new, v_new, k_cache, v_cache, block_table, ctx_len, window, scale,
                     block_size):
    """All outputs [B, n_q, h_q, D] (float64)."""
    B, n_q, hq, D = q.shape
    out = np.zeros((B, n_q, hq, D), np.float64)
    for b in range(B):
        for j in range(n_q):
            for h in range(hq):
                out[b, j, h] = verify_attention_one(b, j, h, q, k_new, v_new, k_cache,
                                                    v_cache, block_table, ctx_len, window,
                                                    scale, block_size)
    return out


def append_kv(k_cache, v_cache, k_new, v_new, block_table, ctx_len, block_size):
    """Cache contents after appending the new rows at positions L_b .. L_b+n_q-1."""
    kc, vc = k_cache.copy(), v_cache.copy()
    B, n_q = k_new.shape[:2]
    for b in range(B):
        for j in range(n_q):
            p = int(ctx_len[b]) + j
            blk = block_table[b, p // block_size]
            kc[blk, :, p % block_size] = k_new[b, j]
            vc[blk, :, p % block_size] = v_new[b, j]
    return kc, vc


def draft_attention_one(b, h, q, k_cache, v_cache, block_table, ctx_len, q_pos, window, scale,
                        block_size):
    """Drafter cross-attention output of head h of sequence b (q: [B, 1, h_q, D])."""
    G = q.shape[2] // k_cache.shape[1]
    g = h // G
    L = int(ctx_len[b])
    lo, hi = key_range(int(q_pos[b]), window, L - 1)
    pos = np.arange(lo, hi + 1)
    K = gather_rows(k_cache, block_table, b, g, pos, block_size)
    V = gather_rows(v_cache, block_table, b, g, pos, block_size)
    return softmax_attend(q[b, 0, h], K, V, scale)


def draft_attention(q, k_cache, v_cache, block_table, ctx_len, q_pos, window, scale,
                    block_size):
    B, _, hq, D = q.shape
    out = np.zeros((B, 1, hq, D), np.float64)
    for b in range(B):
        for h in range(hq):
            out[b, 0, h] = draft_attention_one(b, h, q, k_cache, v_cache, block_table,
                                               ctx_len, q_pos, window, scale, block_size)
    return out
