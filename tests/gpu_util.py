"""Helpers shared by the GPU parity tests (not a test module)."""
from __future__ import annotations

import math

import numpy as np
import torch

import synthetic as S
import verify_step_b200 as sd

DEV = "cuda"


class F64View:
    """Read-only float64 view of a CPU torch tensor: indexing converts only what it touches,
    so the oracle can sample a multi-GB bf16 cache without a full float64 copy."""

    def __init__(self, t: torch.Tensor):
        self.t = t
        self.shape = tuple(t.shape)

    def __getitem__(self, idx):
        if not isinstance(idx, tuple):
            idx = (idx,)
        idx = tuple(torch.as_tensor(np.asarray(i, np.int64)) if isinstance(i, (np.ndarray, list))
                    else i for i in idx)
        return self.t[idx].to(torch.float64).numpy()


def rel_err(x, y) -> float:
    """max over rows of ||x - y||_inf / ||y||_inf (last axis = row)."""
    x = np.asarray(x, np.float64)
    y = np.asarray(y, np.float64)
    x = x.reshape(-1, x.shape[-1])
    y = y.reshape(-1, y.shape[-1])
    num = np.abs(x - y).max(axis=-1)
    den = np.maximum(np.abs(y).max(axis=-1), 1e-30)
    return float((num / den).max())


def attn_desc(B, n_q, hq, hkv, D, bs, mbps, nblocks, window, dtype=sd.SD_BF16, scale=None):
    return sd.AttnDesc(batch=B, n_q=n_q, h_q=hq, h_kv=hkv, head_dim=D, block_size=bs,
                       max_blocks_per_seq=mbps, num_blocks=nblocks, window=window,
                       scale=float(scale if scale is not None else 1.0 / math.sqrt(D)),
                       dtype=dtype)


def workspace(nbytes: int) -> torch.Tensor:
    """Scratch buffer filled with 0xFF bytes (NaN as float32), so a kernel that reads a
    workspace slot it never wrote produces NaN instead of a stale but plausible value."""
    return torch.full((max(int(nbytes), 16),), 255, dtype=torch.uint8, device=DEV)


def to_dev(t: torch.Tensor) -> torch.Tensor:
    return t.contiguous().to(DEV)


def small_paged(seed, L, n_q, hkv, D, bs, dtype="bf16", shuffle=True, window=0, reserve=None):
    """Seeded paged cache for a handful of sequences (host tensors)."""
    L = np.asarray(L, np.int32)
    reserve = n_q + 3 if reserve is None else reserve
    table, nb = S.block_table(seed, L, reserve, bs, shuffle)
    std = 1.0 / math.sqrt(D)
    kc = S.normal(seed * 10 + 1, (nb, hkv, bs, D), std)
    vc = S.normal(seed * 10 + 2, (nb, hkv, bs, D), std)
    cv = S.bf16 if dtype == "bf16" else torch.from_numpy
    return dict(table=torch.from_numpy(table), nb=nb, kc=cv(kc), vc=cv(vc),
                L=torch.from_numpy(L), mbps=table.shape[1])


def qkv(seed, B, n_q, hq, hkv, D, dtype="bf16"):
    std = 1.0 / math.sqrt(D)
    cv = S.bf16 if dtype == "bf16" else torch.from_numpy
    return (cv(S.normal(seed * 10 + 3, (B, n_q, hq, D), std)),
            cv(S.normal(seed * 10 + 4, (B, n_q, hkv, D), std)),
            cv(S.normal(seed * 10 + 5, (B, n_q, hkv, D), std)))


def status_ok():
    st = sd.sd_device_status_read()
    sd.sd_device_status_clear()
    return st == 0
