"""Philox4x32-10 counter-based generator and the uniforms the verify step draws from it.

Test infrastructure (CPU oracle): never imported by the product path.

The generator is written from its published definition: J. K. Salmon, M. A. Moraes,
R. O. Dror, D. E. Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3", SC'11, section on
the Philox family (4x32 variant, 10 rounds).  One round maps the counter (c0, c1, c2, c3)
and key (k0, k1) to (hi(M1*c2) ^ c1 ^ k0, lo(M1*c2), hi(M0*c0) ^ c3 ^ k1, lo(M0*c0)), then
bumps the key by the Weyl constants.  Arrays are numpy uint64 holding 32-bit values (a
32x32-bit product fits exactly in 64 bits).

Uniforms used by the acceptance rule (the pages state no generator; this build's reading):
  key     = (seed & 0xffffffff, seed >> 32)
  counter = (c0, r, step & 0xffffffff, purpose)   r = b*(k+1) + i is the logit row
  acceptance uniform of row r:   c0 = 0, purpose 0, u = (word0 >> 8) * 2^-24  in [0, 1)
  token uniform of token v on row r for a draw with purpose P (1 = target, 2 = drafter):
      c0 = v >> 1, x = (word[2(v&1)+1] << 32) | word[2(v&1)]  (64 bits)
      V  = m * 2^(-24-n) with n = clz64(x), m = top 24 bits of x << n   (V in (0, 1)),
      V  = 0 when x = 0.
  V keeps 24 significant bits at every scale, so it is exactly representable in float32
  and float64 and both sides of a parity test see the same number.
  group uniform of token group g (tokens 512 g .. 512 g + 511) on row r for a draw with
  purpose P: the token uniform's construction with purpose P + 16 and g in place of v.
"""
from __future__ import annotations

import numpy as np

M0 = np.uint64(0xD2511F53)
M1 = np.uint64(0xCD9E8D57)
W0 = np.uint64(0x9E3779B9)
W1 = np.uint64(0xBB67AE85)
MASK = np.uint64(0xFFFFFFFF)
S32 = np.uint64(32)


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Ten Philox4x32 rounds on broadcastable uint64 arrays of 32-bit values."""
    c0, c1, c2, c3, k0, k1 = (np.asarray(x, dtype=np.uint64) & MASK
                              for x in (c0, c1, c2, c3, k0, k1))
    for _ in range(10):
        p0 = M0 * c0
        p1 = M1 * c2
        hi0, lo0 = p0 >> S32, p0 & MASK
        hi1, lo1 = p1 >> S32, p1 & MASK
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
        k0 = (k0 + W0) & MASK
        k1 = (k1 + W1) & MASK
    return c0, c1, c2, c3


def _key(seed: int):
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    return np.uint64(seed & 0xFFFFFFFF), np.uint64(seed >> 32)


def accept_uniform(seed: int, step: int, rows) -> np.ndarray:
    """Acceptance uniforms u in [0, 1) for logit rows ``rows`` (float64, exact)."""
    k0, k1 = _key(seed)
    rows = np.asarray(rows, dtype=np.uint64)
    w0, _, _, _ = philox4x32_10(0, rows, int(step) & 0xFFFFFFFF, 0, k0, k1)
    return (w0 >> np.uint64(8)).astype(np.float64) * 2.0 ** -24


def _float_uniform(x: np.ndarray) -> np.ndarray:
    """V = m * 2^(-24-n): 24 leading bits of the 64-bit word x scaled into (0, 1)."""
    x = np.asarray(x, dtype=np.uint64)
    out = np.zeros(x.shape, np.float64)
    nz = x != 0
    xs = x[nz]
    # count leading zeros of a 64-bit word
    n = np.zeros(xs.shape, np.int64)
    v = xs.copy()
    for sh in (32, 16, 8, 4, 2, 1):
        top = v >> np.uint64(64 - sh)
        z = top == 0
        n[z] += sh
        v[z] = v[z] << np.uint64(sh)
    m = (v >> np.uint64(40)).astype(np.float64)          # in [2^23, 2^24)
    out[nz] = np.ldexp(m, (-24 - n).astype(np.int64))
    return out


def token_uniform(seed: int, step: int, row: int, purpose: int, vocab_ids) -> np.ndarray:
    """Token uniforms V_v in (0, 1) for tokens ``vocab_ids`` of logit row ``row``."""
    k0, k1 = _key(seed)
    v = np.asarray(vocab_ids, dtype=np.uint64)
    ws = philox4x32_10(v >> np.uint64(1), int(row), int(step) & 0xFFFFFFFF, int(purpose),
                       k0, k1)
    odd = (v & np.uint64(1)).astype(bool)
    lo = np.where(odd, ws[2], ws[0])
    hi = np.where(odd, ws[3], ws[1])
    return _float_uniform((hi << S32) | lo)


def token_uniform_at(seed: int, step: int, rows, purpose: int, ids) -> np.ndarray:
    """Token uniforms of tokens ``ids`` [R, n] on rows ``rows`` [R]: shape [R, n]."""
    k0, k1 = _key(seed)
    rows = np.asarray(rows, dtype=np.uint64)[:, None]
    v = np.asarray(ids, dtype=np.uint64)
    ws = philox4x32_10(v >> np.uint64(1), rows, int(step) & 0xFFFFFFFF, int(purpose), k0, k1)
    odd = np.broadcast_to((v & np.uint64(1)).astype(bool), ws[0].shape)
    lo = np.where(odd, ws[2], ws[0])
    hi = np.where(odd, ws[3], ws[1])
    return _float_uniform((hi << S32) | lo)


def token_uniform_rows(seed: int, step: int, rows, purpose: int, vocab: int) -> np.ndarray:
    """Token uniforms for several rows at once: shape [len(rows), vocab]."""
    k0, k1 = _key(seed)
    rows = np.asarray(rows, dtype=np.uint64)[:, None]
    v = np.arange(vocab, dtype=np.uint64)[None, :]
    ws = philox4x32_10(v >> np.uint64(1), rows, int(step) & 0xFFFFFFFF, int(purpose), k0, k1)
    odd = np.broadcast_to((v & np.uint64(1)).astype(bool), ws[0].shape)
    lo = np.where(odd, ws[2], ws[0])
    hi = np.where(odd, ws[3], ws[1])
    return _float_uniform((hi << S32) | lo)


GROUP_PURPOSE_OFFSET = 16


def group_uniform_rows(seed: int, step: int, rows, purpose: int, n_groups: int) -> np.ndarray:
    """Uniforms of the token groups of a two-level draw, shape [len(rows), n_groups]."""
    return token_uniform_rows(seed, step, rows, int(purpose) + GROUP_PURPOSE_OFFSET, n_groups)
