"""sd_accept_noalloc: acceptance without a caller-provided workspace.

Some callers cannot allocate device memory for scratch (a serving loop that must not call
cudaMalloc, or a framework that only lends its input and output buffers).  For them the library
has sd_accept_noalloc, which keeps its scratch in a fixed array inside the library.  This test
calls it through the C ABI several times in a row with different shapes (so each call finds
the array holding another call's leftovers at other offsets) and checks each result against
sd_accept run with an ordinary workspace; it also checks that a request larger than the fixed
array is refused before anything runs.  It sits in a file of its own that pytest collects last.
"""
import ctypes
import json
import os

import numpy as np
import pytest
import torch

import synthetic as S
import verify_step_b200 as sd

pytestmark = pytest.mark.gpu

DEV = "cuda"
NOISE = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "draft_noise.json")))


def _inputs(seed, B, k, V):
    z = S.make_logits(seed, B * (k + 1), V)
    if k == 0:
        return z.to(DEV), None, None
    y = torch.stack([S.perturb(seed * 10 + i, z.reshape(B, k + 1, V)[:, i],
                               NOISE["sigma_pos0"] if i == 0 else NOISE["sigma_later"])
                     for i in range(k)], dim=1)
    drafts = torch.from_numpy(np.argmax(y.numpy(), axis=-1).astype(np.int32))
    return z.to(DEV), y.contiguous().to(DEV), drafts.to(DEV)


def _outputs(B, n_q):
    return (torch.full((B,), -9, dtype=torch.int32, device=DEV),
            torch.full((B, n_q), -9, dtype=torch.int32, device=DEV),
            torch.full((B,), -9, dtype=torch.int32, device=DEV))


def _check(call, B, k, V, T, seed, step, purpose=1):
    z, y, drafts = _inputs(seed, B, k, V)
    desc = sd.AcceptDesc(batch=B, k=k, vocab=V, temperature=T, seed=11, step=step,
                         purpose=purpose)
    ref = _outputs(B, k + 1)
    ws = torch.full((max(16, sd.sd_accept_workspace_size(desc)),), 0xFF, dtype=torch.uint8,
                    device=DEV)
    sd.sd_accept(desc, z, y if k > 0 else None, drafts if k > 0 else None, *ref, ws)
    got = _outputs(B, k + 1)
    sd.sd_accept_noalloc(desc, z, y if k > 0 else None, drafts if k > 0 else None, *got)
    torch.cuda.synchronize()
    for r, g in zip(ref, got):
        assert torch.equal(r, g), f"call {call}"
    assert sd.sd_device_status_read() == 0


def test_noalloc_matches_workspace_version_twice():
    V = 262144
    _check(0, 8, 2, V, 1.0, 5, 3)
    _check(1, 8, 2, V, 0.7, 6, 4)


def test_noalloc_other_shapes_in_a_row():
    """A plain draw (k = 0, T = 0.7) at B = 64, then a greedy call (T = 0), then the k = 2
    sampling call again: each finds the previous call's statistics, candidates and tickets at
    other offsets of the shared array."""
    V = 262144
    _check(0, 64, 0, V, 0.7, 7, 5, purpose=2)
    _check(1, 16, 3, V, 0.0, 8, 6)
    _check(2, 8, 2, V, 1.0, 9, 7)


def test_noalloc_refuses_requests_beyond_its_scratch():
    V, k = 262144, 6
    desc = sd.AcceptDesc(batch=283, k=k, vocab=V, temperature=1.0, seed=0, step=0, purpose=1)
    assert sd.sd_accept_workspace_size(desc) > (4 << 20)
    desc.batch = 282
    assert sd.sd_accept_workspace_size(desc) <= (4 << 20)
    desc.batch = 283
    # nothing is dereferenced or launched: null data pointers are fine for the size check
    st = sd.lib().sd_accept_noalloc(ctypes.byref(desc), None, None, None, None, None, None,
                                    None)
    assert st == sd.SD_ERR_WORKSPACE
