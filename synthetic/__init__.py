"""Seeded synthetic inputs for the speculative-decoding verify step.

This module is shared by the tests, the benchmark and the CPU oracle's callers.  It holds
none of the method's arithmetic: only seeded random numbers, round-to-nearest-even bf16
rounding (done by torch's dtype conversion), and the bookkeeping of a paged KV cache (which
physical block holds which logical block of which sequence).

Workload shapes follow the five verify-step configurations the pages' setting implies
(Gemma 4 MTP serving guide, section 7 recipe: max context 16384, local head_dim 256 / global
head_dim 512; Google blog "MTP drafter internals": 262144-token vocabulary):

  tiny_fp32   B1  L256      k2  4q/1kv  D64  global           d256  V1024   fp32
  edge        B1  L4096     k2  8q/2kv  D256 window 512       d2560 V262144 bf16
  global      B8  L16384    k1..6 16q/4kv D512 global          d5376 V262144 bf16
  drafter     B8  L16384    chained k4, 3 x (D256 W512) + 1 x D512, hidden 1024,
              clustered head 1024 clusters x 256 tokens, top 32
  serving     B64 L~U[1024,16384] k2 16q/4kv D256 W512 and D512, shuffled blocks, d5376

Generation is chunked: chunk i of a tensor drawn with seed s comes from PCG64 seeded with
[s, i], so the values do not depend on the number of threads used.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np
import torch

CHUNK = 1 << 22  # elements per independently seeded chunk
_THREADS = max(1, min(16, os.cpu_count() or 1))


# ----------------------------------------------------------------------------- primitives

def normal(seed: int, shape, std: float = 1.0) -> np.ndarray:
    """float32 array of iid N(0, std^2) values, deterministic in (seed, shape)."""
    shape = tuple(int(s) for s in (shape if hasattr(shape, "__len__") else (shape,)))
    n = int(np.prod(shape)) if shape else 1
    out = np.empty(n, np.float32)
    nch = (n + CHUNK - 1) // CHUNK

    def fill(i):
        rng = np.random.default_rng([int(seed) & 0xFFFFFFFF, i])
        rng.standard_normal(out=out[i * CHUNK:(i + 1) * CHUNK], dtype=np.float32)

    if nch <= 1:
        if n:
            fill(0)
    else:
        with ThreadPoolExecutor(_THREADS) as ex:
            list(ex.map(fill, range(nch)))
    if std != 1.0:
        out *= np.float32(std)
    return out.reshape(shape)


def bf16(x: np.ndarray) -> torch.Tensor:
    """Round a float32 array to bf16 (round to nearest even); CPU tensor."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


def as_f64(t) -> np.ndarray:
    """Exact float64 copy of a bf16/fp32 tensor or array (bf16 -> fp64 is exact)."""
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu").to(torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def ctx_lengths(seed: int, batch: int, lo: int, hi: int) -> np.ndarray:
    """Committed context lengths uniform on the integers [lo, hi] (inclusive)."""
    rng = np.random.default_rng([seed & 0xFFFFFFFF, 0xC7])
    return rng.integers(lo, hi + 1, size=batch).astype(np.int32)


def block_table(seed: int, ctx_len: np.ndarray, reserve: int, bs: int,
                shuffle: bool, max_blocks: int | None = None):
    """Paged-cache block table for sequences of committed length ctx_len.

    Each sequence gets physical blocks for its logical blocks 0..ceil((L_b+reserve)/bs)-1
    (``reserve`` positions past the context: the k+1 verify positions plus room to grow).
    Blocks are numbered contiguously per sequence, or taken from a seeded random
    permutation of the pool when ``shuffle``.  Unused table entries hold -1.
    Returns (table [B, max_blocks] int32, num_blocks).
    """
    ctx_len = np.asarray(ctx_len, np.int64)
    need = (ctx_len + reserve + bs - 1) // bs
    mb = int(need.max()) if max_blocks is None else int(max_blocks)
    if (need > mb).any():
        raise ValueError("max_blocks too small for ctx_len + reserve")
    total = int(need.sum())
    ids = np.arange(total, dtype=np.int64)
    if shuffle:
        rng = np.random.default_rng([seed & 0xFFFFFFFF, 0xB10C])
        ids = rng.permutation(total)
    table = np.full((len(ctx_len), mb), -1, np.int32)
    o = 0
    for b, n in enumerate(need):
        table[b, :n] = ids[o:o + n]
        o += int(n)
    return table, total


def window_block_table(seed: int, ctx_len: np.ndarray, reserve: int, bs: int, window: int,
                       shuffle: bool, max_blocks: int):
    """Block table of a sliding-window layer: only blocks that can hold a key inside the
    window of some query position in [L_b, L_b+reserve) are materialised; earlier entries
    alias the sequence's first materialised block (they are never read)."""
    ctx_len = np.asarray(ctx_len, np.int64)
    first = np.maximum(0, ctx_len - window + 1) // bs
    last = (ctx_len + reserve - 1) // bs
    need = last - first + 1
    total = int(need.sum())
    ids = np.arange(total, dtype=np.int64)
    if shuffle:
        rng = np.random.default_rng([seed & 0xFFFFFFFF, 0x5EED])
        ids = rng.permutation(total)
    table = np.full((len(ctx_len), max_blocks), -1, np.int32)
    o = 0
    for b in range(len(ctx_len)):
        n = int(need[b])
        if last[b] >= max_blocks:
            raise ValueError("max_blocks too small")
        table[b, first[b]:last[b] + 1] = ids[o:o + n]
        table[b, :first[b]] = ids[o]
        o += n
    return table, total


# ----------------------------------------------------------------------------- workloads

@dataclass
class AttnLayer:
    """One attention layer of the target cache: head_dim D, window (0 = global)."""
    head_dim: int
    window: int = 0


@dataclass
class Workload:
    name: str
    batch: int
    ctx: int | tuple            # int, or (lo, hi) for ragged uniform lengths
    k: int
    h_q: int
    h_kv: int
    layers: list                # list[AttnLayer]
    d_model: int
    vocab: int
    dtype: str = "bf16"         # "bf16" or "f32"
    block_size: int = 16
    shuffle: bool = False
    temperature: float = 1.0
    qkv_std: str = "rsqrt_d"    # "unit" or "rsqrt_d" (N(0,1)/sqrt(head_dim))
    drafter_hidden: int = 0
    n_clusters: int = 0
    cluster_size: int = 0
    top_c: int = 0
    draft_layers: list = field(default_factory=list)
    seed: int = 0


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", 1, 256, 2, 4, 1, [AttnLayer(64)], 256, 1024,
                          dtype="f32", qkv_std="unit", seed=1),
    "edge": Workload("edge", 1, 4096, 2, 8, 2, [AttnLayer(256, 512)], 2560, 262144, seed=2),
    "global": Workload("global", 8, 16384, 2, 16, 4, [AttnLayer(512)], 5376, 262144, seed=3),
    "drafter": Workload("drafter", 8, 16384, 4, 16, 4, [AttnLayer(256, 512), AttnLayer(512)],
                        1024, 262144, drafter_hidden=1024, n_clusters=1024, cluster_size=256,
                        top_c=32, draft_layers=[0, 0, 0, 1], seed=4),
    "serving": Workload("serving", 64, (1024, 16384), 2, 16, 4,
                        [AttnLayer(256, 512), AttnLayer(512)], 5376, 262144, shuffle=True,
                        seed=5),
}


def qkv_std(w: Workload, head_dim: int) -> float:
    return 1.0 if w.qkv_std == "unit" else 1.0 / math.sqrt(head_dim)


def contexts(w: Workload) -> np.ndarray:
    if isinstance(w.ctx, tuple):
        return ctx_lengths(w.seed, w.batch, w.ctx[0], w.ctx[1])
    return np.full(w.batch, int(w.ctx), np.int32)


def make_cache(w: Workload, layer: int, ctx_len: np.ndarray, reserve: int,
               max_blocks: int | None = None, seed_offset: int = 0):
    """Paged K/V cache of one layer filled with seeded values at every slot.

    Returns dict(table, num_blocks, k_cache, v_cache) with caches shaped
    [num_blocks, h_kv, block_size, head_dim] in the workload dtype (CPU tensors).
    """
    lay = w.layers[layer]
    bs = w.block_size
    if max_blocks is None:
        max_blocks = int(((np.asarray(ctx_len, np.int64) + reserve + bs - 1) // bs).max())
    if lay.window > 0:
        table, nb = window_block_table(w.seed + 17 * layer, ctx_len, reserve, bs, lay.window,
                                       w.shuffle, max_blocks)
    else:
        table, nb = block_table(w.seed + 17 * layer, ctx_len, reserve, bs, w.shuffle,
                                max_blocks)
    shape = (nb, w.h_kv, bs, lay.head_dim)
    std = qkv_std(w, lay.head_dim)
    s = 1000 * w.seed + 100 * layer + seed_offset
    kc = normal(s + 1, shape, std)
    vc = normal(s + 2, shape, std)
    if w.dtype == "bf16":
        kc, vc = bf16(kc), bf16(vc)
    else:
        kc, vc = torch.from_numpy(kc), torch.from_numpy(vc)
    return dict(table=torch.from_numpy(table), num_blocks=nb, k_cache=kc, v_cache=vc,
                max_blocks=max_blocks)


def make_step_qkv(w: Workload, layer: int, n_q: int, step: int = 0):
    """Queries and the new keys/values of the n_q verify positions of one layer."""
    lay = w.layers[layer]
    std = qkv_std(w, lay.head_dim)
    s = 1000 * w.seed + 100 * layer + 10 * (step + 1)
    q = normal(s + 3, (w.batch, n_q, w.h_q, lay.head_dim), std)
    kn = normal(s + 4, (w.batch, n_q, w.h_kv, lay.head_dim), std)
    vn = normal(s + 5, (w.batch, n_q, w.h_kv, lay.head_dim), std)
    cv = bf16 if w.dtype == "bf16" else torch.from_numpy
    return dict(q=cv(q), k_new=cv(kn), v_new=cv(vn))


def make_lm_head(w: Workload, d: int | None = None, seed_offset: int = 0):
    """Dense LM-head weights W [vocab, d] ~ N(0, 1/d)."""
    d = w.d_model if d is None else d
    W = normal(1000 * w.seed + 7 + seed_offset, (w.vocab, d), 1.0 / math.sqrt(d))
    return bf16(W) if w.dtype == "bf16" else torch.from_numpy(W)


def make_hidden(w: Workload, m: int, d: int | None = None, step: int = 0, std: float = 1.0):
    d = w.d_model if d is None else d
    h = normal(1000 * w.seed + 8 + 31 * step, (m, d), std)
    return bf16(h) if w.dtype == "bf16" else torch.from_numpy(h)


def make_clustered_head(w: Workload, seed_offset: int = 0):
    """Synthetic clustered LM head of the drafter.

    Tokens are assigned to clusters by a seeded random permutation (cluster c holds tokens
    perm[c*cs:(c+1)*cs]); weights are stored cluster-major W_cm [C, cs, d] ~ N(0, 1/d) in
    bf16; each centroid is the mean of its member rows (the bf16 values), rounded to bf16.
    """
    C, cs, d = w.n_clusters, w.cluster_size, w.drafter_hidden
    assert C * cs == w.vocab
    rng = np.random.default_rng([w.seed + seed_offset, 0xC1])
    perm = rng.permutation(w.vocab).astype(np.int32).reshape(C, cs)
    Wcm = bf16(normal(1000 * w.seed + 9 + seed_offset, (C, cs, d), 1.0 / math.sqrt(d)))
    cent = bf16(Wcm.to(torch.float32).mean(dim=1).numpy())
    return dict(cluster_tokens=torch.from_numpy(perm), w_cm=Wcm, centroids=cent)


def make_logits(seed: int, rows: int, vocab: int, std: float = 1.0) -> torch.Tensor:
    """Synthetic target logits: iid N(0, std^2) per token (the distribution of h.W^T with
    h ~ N(0,1) and W ~ N(0,1/d)), fp32."""
    return torch.from_numpy(normal(seed, (rows, vocab), std))


def perturb(seed: int, z: torch.Tensor, sigma: float) -> torch.Tensor:
    """Draft logits y = z + N(0, sigma^2) noise (fp32)."""
    return z + torch.from_numpy(normal(seed, tuple(z.shape), sigma))


# ----------------------------------------------------------------------------- drafter layers

DRAFTER_FF = 4096  # gated-MLP width of the synthetic drafter layers (4 x the hidden width)


def make_drafter_weights(seed: int, d: int, d_target: int, vocab: int, h_q: int, head_dims,
                         ff: int = DRAFTER_FF):
    """Synthetic drafter weights (CPU tensors): embedding E [vocab, d], input projection
    W_in [d, d_target + d], per layer RMSNorm gains (float32, 1 + N(0, 0.1^2)) and bf16
    projections Wq [h_q D, d], Wo [d, h_q D], Wg, Wu [ff, d], Wd [d, ff] (each ~ N(0, 1/fan_in)),
    the output gain g_final and the back projection W_back [d_target, d]."""
    s = 50000 + 1000 * int(seed)
    out = {"E": bf16(normal(s, (vocab, d))),
           "W_in": bf16(normal(s + 1, (d, d_target + d), 1 / math.sqrt(d_target + d))),
           "g_final": torch.from_numpy(1 + normal(s + 2, (d,), 0.1)),
           "W_back": bf16(normal(s + 3, (d_target, d), 1 / math.sqrt(d))),
           "layers": []}
    for i, D in enumerate(head_dims):
        t = s + 10 * (i + 1)
        out["layers"].append({
            "g_attn": torch.from_numpy(1 + normal(t, (d,), 0.1)),
            "Wq": bf16(normal(t + 1, (h_q * D, d), 1 / math.sqrt(d))),
            "Wo": bf16(normal(t + 2, (d, h_q * D), 1 / math.sqrt(h_q * D))),
            "g_mlp": torch.from_numpy(1 + normal(t + 3, (d,), 0.1)),
            "Wg": bf16(normal(t + 4, (ff, d), 1 / math.sqrt(d))),
            "Wu": bf16(normal(t + 5, (ff, d), 1 / math.sqrt(d))),
            "Wd": bf16(normal(t + 6, (d, ff), 1 / math.sqrt(ff))),
        })
    return out



def make_target_weights(seed: int, d: int, ff: int, h_q: int, h_kv: int, layers):
    """Synthetic target layers (CPU tensors) for the multi-layer verify: per layer (head_dim D,
    window W) RMSNorm gains (float32, 1 + N(0, 0.1^2)) and bf16 projections Wq [h_q D, d],
    Wk, Wv [h_kv D, d], Wo [d, h_q D], Wg, Wu [ff, d], Wd [d, ff], each ~ N(0, 1/fan_in)."""
    out = []
    for i, (D, W) in enumerate(layers):
        t = 70000 + 1000 * int(seed) + 10 * i
        out.append({
            "head_dim": int(D), "window": int(W),
            "g_attn": torch.from_numpy(1 + normal(t, (d,), 0.1)),
            "Wq": bf16(normal(t + 1, (h_q * D, d), 1 / math.sqrt(d))),
            "Wk": bf16(normal(t + 2, (h_kv * D, d), 1 / math.sqrt(d))),
            "Wv": bf16(normal(t + 3, (h_kv * D, d), 1 / math.sqrt(d))),
            "Wo": bf16(normal(t + 4, (d, h_q * D), 1 / math.sqrt(h_q * D))),
            "g_mlp": torch.from_numpy(1 + normal(t + 5, (d,), 0.1)),
            "Wg": bf16(normal(t + 6, (ff, d), 1 / math.sqrt(d))),
            "Wu": bf16(normal(t + 7, (ff, d), 1 / math.sqrt(d))),
            "Wd": bf16(normal(t + 8, (d, ff), 1 / math.sqrt(ff))),
        })
    return out
