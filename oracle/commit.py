"""Commit of the accepted prefix and rollback of the rejected positions.

Test infrastructure (CPU oracle): never imported by the product path.

"Gemma 4 MTP: drafter drafts, target verifies", section "basic structure of speculative
decoding": when a draft is wrong only the prefix up to that position is kept and the
drafter restarts; Gemma 4 MTP serving guide, section 4: drafts after the first rejected
token are discarded.  Section "drafter internal architecture" of the first page: the
drafter's next input is the target's last-layer activation.

With a_b accepted drafts the verify step wrote K/V for positions L_b .. L_b+k; the ones
at L_b .. L_b+a_b (the last committed token and the accepted drafts) are kept, so the new
committed length is L_b + a_b + 1 and positions L_b+a_b+1 .. L_b+k are rolled back (the
emitted correction / bonus token has no K/V yet; the next verify step writes it).
committed_slots[b, j] = physical slot of position L_b + j for j <= a_b, else -1, with
slot = block_table[b, p // bs] * bs + p % bs.  next_hidden[b] = hidden[b, a_b], the
activation at the last kept position.
"""
from __future__ import annotations

import numpy as np


def commit(ctx_len, n_accepted, block_table, block_size: int, n_q: int, hidden=None):
    ctx_len = np.asarray(ctx_len, np.int64)
    a = np.asarray(n_accepted, np.int64)
    B = ctx_len.shape[0]
    new_len = ctx_len + a + 1
    slots = np.full((B, n_q), -1, np.int64)
    rolled = []
    for b in range(B):
        for j in range(n_q):
            p = int(ctx_len[b]) + j
            s = int(block_table[b, p // block_size]) * block_size + p % block_size
            if j <= a[b]:
                slots[b, j] = s
            else:
                rolled.append((b, p, s))
    out = dict(ctx_len=new_len, committed_slots=slots, rolled_back=rolled)
    if hidden is not None:
        hidden = np.asarray(hidden)
        out["next_hidden"] = hidden[np.arange(B), a]
    return out
