"""LM-head projection, dense and clustered, in float64.

Test infrastructure (CPU oracle): never imported by the product path.

* Dense: logits[m, v] = sum_i h[m, i] * W[v, i] over the full 262144-token vocabulary
  (Gemma 4 MTP serving guide, section 1: 256k vocabulary; the target's p must come from the
  full projection for the acceptance rule to stay lossless).  Written as a library matmul
  in float64; ``cols`` restricts the output to a subset of vocabulary rows (each logit is
  still one dot product, nothing is reordered).
* Clustered (drafter side) -- Google blog as summarised by GeekNews, section "MTP drafter
  internal optimisations", and the serving guide, section 1: the edge drafters group the
  vocabulary into clusters so the 256k-vocabulary logit projection costs less.  The pages
  give no algorithm; this build's reading is one flat level: score every cluster centroid
  (score_c = h . C_c), keep the top_c clusters per row (higher score first, equal scores
  ordered by lower cluster id), give exact logits h . W_v for the tokens of the kept
  clusters and -inf to every other token.  Weights are stored cluster-major,
  w_cm[c, i] = W[cluster_tokens[c, i]].
"""
from __future__ import annotations

import numpy as np


def lm_head(h: np.ndarray, W: np.ndarray, cols=None) -> np.ndarray:
    """Dense logits [M, V] (or [M, len(cols)]) in float64."""
    Wc = W if cols is None else W[np.asarray(cols)]
    return np.asarray(h, np.float64) @ np.asarray(Wc, np.float64).T


def cluster_scores(h: np.ndarray, centroids: np.ndarray) -> np.ndarray:
    return np.asarray(h, np.float64) @ np.asarray(centroids, np.float64).T


def top_clusters(scores: np.ndarray, top_c: int):
    """Per row: the top_c cluster ids (returned in ascending id order) and the gap between
    the top_c-th and (top_c+1)-th scores (inf when every cluster is kept)."""
    M, C = scores.shape
    sel = np.zeros((M, top_c), np.int64)
    gap = np.full(M, np.inf)
    ids = np.arange(C)
    for m in range(M):
        order = np.lexsort((ids, -scores[m]))  # score descending, then id ascending
        sel[m] = np.sort(order[:top_c])
        if top_c < C:
            gap[m] = scores[m, order[top_c - 1]] - scores[m, order[top_c]]
    return sel, gap


def clustered_lm_head(h, centroids, w_cm, cluster_tokens, top_c: int):
    """Returns (logits [M, V] float64 with -inf outside kept clusters, sel [M, top_c],
    selection-boundary score gap [M])."""
    h = np.asarray(h, np.float64)
    C, cs, d = w_cm.shape
    V = C * cs
    scores = cluster_scores(h, centroids)
    sel, gap = top_clusters(scores, top_c)
    logits = np.full((h.shape[0], V), -np.inf)
    for m in range(h.shape[0]):
        for c in sel[m]:
            logits[m, cluster_tokens[c]] = np.asarray(w_cm[c], np.float64) @ h[m]
    return logits, sel, gap
