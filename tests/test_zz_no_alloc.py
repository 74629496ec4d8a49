"""sd_accept_noalloc: acceptance without a caller-provided workspace.

Some callers cannot allocate device memory for scratch (a serving loop that must not call
cudaMalloc, or a framework that only lends its input and output buffers).  For them the library
has sd_accept_noalloc, which keeps its scratch in a fixed array inside the library.  This test
calls it through the C ABI twice in a row and checks each result against sd_accept run with an
ordinary workspace; it also checks that a request larger than the fixed array is refused
before anything runs.  It sits in a file of its own that pytest collects last.
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
    y = torch.stack([S.perturb(seed * 10 + i, z.reshape(B, k + 1, V)[:, i],
                               NOISE["sigma_pos0"] if i == 0 else NOISE["sigma_later"])
                     for i in range(k)], dim=1)
    drafts = torch.from_numpy(np.argmax(y.numpy(), axis=-1).astype(np.int32))
    return z.to(DEV), y.contiguous().to(DEV), drafts.to(DEV)


def _outputs(B, n_q):
    return (torch.full((B,), -9, dtype=torch.int32, device=DEV),
            torch.full((B, n_q), -9, dtype=torch.int32, device=DEV),
            torch.full((B,), -9, dtype=torch.int32, device=DEV))


def test_noalloc_matches_workspace_version_twice():
    B, k, V = 8, 2, 262144
    for call, (seed, step, T) in enumerate(((5, 3, 1.0), (6, 4, 0.7))):
        z, y, drafts = _inputs(seed, B, k, V)
        desc = sd.AcceptDesc(batch=B, k=k, vocab=V, temperature=T, seed=11, step=step,
                             purpose=1)
        ref = _outputs(B, k + 1)
        ws = torch.empty(sd.sd_accept_workspace_size(desc), dtype=torch.uint8, device=DEV)
        sd.sd_accept(desc, z, y, drafts, *ref, ws)
        got = _outputs(B, k + 1)
        sd.sd_accept_noalloc(desc, z, y, drafts, *got)
        torch.cuda.synchronize()
        for r, g in zip(ref, got):
            assert torch.equal(r, g), f"call {call}"
        assert sd.sd_device_status_read() == 0


def test_noalloc_refuses_requests_beyond_its_scratch():
    V, k = 262144, 6
    desc = sd.AcceptDesc(batch=627, k=k, vocab=V, temperature=1.0, seed=0, step=0, purpose=1)
    assert sd.sd_accept_workspace_size(desc) > (4 << 20)
    # nothing is dereferenced or launched: null data pointers are fine for the size check
    st = sd.lib().sd_accept_noalloc(ctypes.byref(desc), None, None, None, None, None, None,
                                    None)
    assert st == sd.SD_ERR_WORKSPACE
