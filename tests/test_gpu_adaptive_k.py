"""Adaptive k closed on the GPU: the accepted counts of sd_accept drive the controller.

Gemma 4 MTP serving guide, sections 2 and 6 and its closing checklist: raise k while the mean
accepted length per step (MAL) still improves, hold it where it stops, and cut to one draft when
position 1 collapses.  Each window here is 4000 sequences of one verify step: target logits
z ~ N(0, 1) per token, draft logits y = z + noise with the tuned standard deviations (1.446 at
draft 1, 1.318 after it: closed-form acceptance 0.47, then 0.51), drafts drawn from q by the
drafter's own plain draw (sd_accept, k = 0, purpose 2), then sd_accept on (z, y, drafts).  Only
the accepted counts the GPU returns reach the controller.
"""
import json
import os

import numpy as np
import pytest
import torch

import verify_step_b200 as sd
from tests.gpu_util import DEV, status_ok
from verify_step_b200.adaptive_k import AdaptiveK

pytestmark = pytest.mark.gpu

NOISE = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "draft_noise.json")))
V = 32768          # the acceptance of the tuned noise is 0.469 / 0.507 at this vocabulary
WINDOW = 4000
B = 500            # sequences per call


def window_counts(k, sigmas, gen, window_index):
    n_acc = torch.empty(B, dtype=torch.int32, device=DEV)
    out = torch.empty((B, k + 1), dtype=torch.int32, device=DEV)
    flags = torch.empty(B, dtype=torch.int32, device=DEV)
    draw_acc = torch.empty(B * k, dtype=torch.int32, device=DEV)
    drafts = torch.empty((B, k), dtype=torch.int32, device=DEV)
    counts = []
    for call in range(WINDOW // B):
        step = window_index * 64 + call
        z = torch.randn((B, k + 1, V), generator=gen, device=DEV)
        y = torch.stack([z[:, i] + sigmas[min(i, len(sigmas) - 1)] *
                         torch.randn((B, V), generator=gen, device=DEV) for i in range(k)],
                        dim=1).contiguous()
        dd = sd.AcceptDesc(batch=B * k, k=0, vocab=V, temperature=1.0, seed=3, step=step,
                           purpose=2)
        ws = torch.empty(max(sd.sd_accept_workspace_size(dd), 256), dtype=torch.uint8,
                         device=DEV)
        sd.sd_accept(dd, y, None, None, draw_acc, drafts, None, ws)
        desc = sd.AcceptDesc(batch=B, k=k, vocab=V, temperature=1.0, seed=5, step=step,
                             purpose=1)
        ws2 = torch.empty(sd.sd_accept_workspace_size(desc), dtype=torch.uint8, device=DEV)
        sd.sd_accept(desc, z, y, drafts, n_acc, out, flags, ws2)
        counts.append(n_acc.cpu().numpy().copy())
    assert status_ok()
    return np.concatenate(counts)


def test_adaptive_k_settles_at_two_and_cuts_on_a_position_one_collapse():
    gen = torch.Generator(device=DEV)
    gen.manual_seed(2024)
    ctrl = AdaptiveK(k_init=1, k_max=4, window=WINDOW)
    tuned = (NOISE["sigma_pos0"], NOISE["sigma_later"])
    ks, mals = [], {}
    for w in range(5):
        k = ctrl.k
        d = ctrl.observe(window_counts(k, tuned, gen, w))
        assert d is not None
        ks.append(k)
        mals[k] = d.telemetry["mal"]
    # explore 1 -> 2 -> 3, then hold at 2 (k = 3 gains less than 10 % over k = 2)
    assert ks == [1, 2, 3, 2, 2], (ks, mals)
    assert ctrl.phase == "hold" and ctrl.k == 2
    # the guide's measured MAL at k = 1 and 2 (1.45, 1.71); closed form 1.47, 1.71
    assert abs(mals[1] - 1.47) < 0.05 and abs(mals[2] - 1.71) < 0.06, mals
    # position 1 collapses (its noise raised: conditional acceptance about 0.21): cut to one
    d = ctrl.observe(window_counts(2, (NOISE["sigma_pos0"], 2.5), gen, 10))
    r = d.telemetry["position_rates"]
    assert r[0] >= 0.35 and r[1] < 0.15, r
    assert d.k == 1 and ctrl.k == 1
