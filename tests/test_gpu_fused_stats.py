"""Softmax partials produced by the kernels that write the logits (the dense head's epilogue and
the drafter's plain draw) and consumed by the acceptance in place of its statistics pass.

The merged partials of a row must give its log-sum-exp at temperature T (checked against the
float64 oracle of the row), and an acceptance fed with them must return what the oracle
returns (the same bar as every acceptance test).
"""
import math

import numpy as np
import pytest
import torch

import synthetic as S
import verify_step_b200 as sd
from oracle import accept as OACC
from oracle import lm_head as OH
from tests.gpu_util import DEV, F64View, rel_err, status_ok, to_dev, workspace

pytestmark = pytest.mark.gpu


def merged_lse(parts):
    """log sum exp of a row from its (max, sum exp(x - max)) slots (float64)."""
    p = parts.double().numpy()
    m, s = p[..., 0], p[..., 1]
    top = np.max(np.where(s > 0, m, -np.inf), axis=-1, keepdims=True)
    return top[..., 0] + np.log(np.sum(np.where(s > 0, s * np.exp(m - top), 0.0), axis=-1))


def lse(x):
    x = np.asarray(x, np.float64)
    top = np.max(x, axis=-1, keepdims=True)
    return top[..., 0] + np.log(np.sum(np.exp(x - top), axis=-1))


@pytest.mark.parametrize("m,T", [(24, 1.0), (5, 0.7), (64, 1.3)])
def test_head_partials_give_the_row_log_sum_exp(m, T):
    d, V = 512, 65536 + 200  # a ragged last vocabulary tile
    W = S.bf16(S.normal(51, (V, d), 1 / math.sqrt(d)))
    h = S.bf16(S.normal(52, (m, d)))
    desc = sd.HeadDesc(m=m, d=d, vocab=V, dtype=sd.SD_BF16, stats_temperature=T)
    slots = sd.sd_lm_head_stats_slots(desc)
    assert slots > 0
    parts = torch.full((m, slots, 2), float("nan"), dtype=torch.float32, device=DEV)
    desc.row_stats = parts.data_ptr()
    logits = torch.empty((m, V), dtype=torch.float32, device=DEV)
    sd.sd_lm_head(desc, to_dev(h), to_dev(W), logits)
    torch.cuda.synchronize()
    ref = OH.lm_head(h.double().numpy(), W.double().numpy())
    assert rel_err(logits.cpu().numpy(), ref) <= 1e-5
    got = merged_lse(parts.cpu())
    want = lse(ref / T)
    assert np.max(np.abs(got - want)) <= 1e-5 * np.maximum(1.0, np.abs(want)).max()
    assert status_ok()


def test_head_partials_refused_where_unsupported():
    desc = sd.HeadDesc(m=65, d=512, vocab=4096, dtype=sd.SD_BF16, stats_temperature=1.0)
    assert sd.sd_lm_head_stats_slots(desc) == 0
    desc.row_stats = 16  # any non-null address: refused before a launch
    with pytest.raises(sd.SdError):
        sd.sd_lm_head(desc, torch.zeros((65, 512), dtype=torch.bfloat16, device=DEV),
                      torch.zeros((4096, 512), dtype=torch.bfloat16, device=DEV),
                      torch.zeros((65, 4096), dtype=torch.float32, device=DEV))


@pytest.mark.parametrize("masked", [False, True])
def test_plain_draw_partials_give_the_row_log_sum_exp(masked):
    B, V, T = 8, 262144, 0.8
    z = S.make_logits(61, B, V)
    if masked:
        keep = torch.from_numpy(np.random.default_rng(6).random((B, V)) < 0.03)
        z = torch.where(keep, z, torch.full_like(z, float("-inf")))
    desc = sd.AcceptDesc(batch=B, k=0, vocab=V, temperature=T, seed=4, step=7, purpose=2)
    slots = sd.sd_accept_stats_slots(desc)
    assert slots > 0
    parts = torch.full((B, slots, 2), float("nan"), dtype=torch.float32, device=DEV)
    desc.stats_out = parts.data_ptr()
    n_acc = torch.empty(B, dtype=torch.int32, device=DEV)
    out = torch.empty((B, 1), dtype=torch.int32, device=DEV)
    ws = workspace(sd.sd_accept_workspace_size(desc))
    sd.sd_accept(desc, to_dev(z.reshape(B, 1, V)), None, None, n_acc, out, None, ws)
    torch.cuda.synchronize()
    got = merged_lse(parts.cpu())
    want = lse(z.double().numpy() / T)
    assert np.max(np.abs(got - want)) <= 1e-5 * np.maximum(1.0, np.abs(want)).max()
    # the draw itself is unchanged by producing the partials
    ref = OACC.accept(z.reshape(B, 1, V).double().numpy(), None, np.zeros((B, 0), np.int64), T,
                      seed=4, step=7, purpose=2)
    ok = ~ref["margin"]
    assert np.array_equal(out.cpu().numpy()[ok], ref["out_tokens"][ok])
    assert status_ok()


def host_parts(rows, T, slots=3):
    """Exact partials of each row split into `slots` contiguous pieces (float64 -> float32)."""
    x = rows.double().numpy() / T
    pieces = np.array_split(x, slots, axis=-1)
    out = np.zeros(x.shape[:-1] + (slots, 2), np.float32)
    for s, piece in enumerate(pieces):
        m = piece.max(axis=-1)
        out[..., s, 0] = m
        out[..., s, 1] = np.exp(piece - m[..., None]).sum(axis=-1)
    return torch.from_numpy(out)


@pytest.mark.parametrize("which", ["target", "draft", "both"])
def test_accept_with_producer_partials_matches_the_oracle(which):
    B, k, V, T = 8, 2, 262144, 1.0
    z = S.make_logits(71, B * (k + 1), V).reshape(B, k + 1, V)
    y = torch.stack([S.perturb(720 + i, z[:, i], 1.4) for i in range(k)], dim=1)
    drafts = torch.from_numpy(np.stack([
        OACC.accept(y[:, i:i + 1].numpy(), None, np.zeros((B, 0)), T, seed=3, step=64 + i,
                    purpose=OACC.PURPOSE_DRAFTER)["out_tokens"][:, 0] for i in range(k)],
        axis=1).astype(np.int32))
    desc = sd.AcceptDesc(batch=B, k=k, vocab=V, temperature=T, seed=9, step=5, purpose=1)
    keep = []
    if which in ("target", "both"):
        tp = to_dev(host_parts(z.reshape(B * (k + 1), V), T))
        desc.target_stats, desc.target_stats_slots = tp.data_ptr(), 3
        keep.append(tp)
    if which in ("draft", "both"):
        dp = to_dev(host_parts(y.reshape(B * k, V), T, slots=5))
        desc.draft_stats, desc.draft_stats_slots = dp.data_ptr(), 5
        keep.append(dp)
    n_acc = torch.full((B,), -9, dtype=torch.int32, device=DEV)
    out = torch.full((B, k + 1), -9, dtype=torch.int32, device=DEV)
    ws = workspace(sd.sd_accept_workspace_size(desc))
    sd.sd_accept(desc, to_dev(z), to_dev(y), to_dev(drafts), n_acc, out, None, ws)
    torch.cuda.synchronize()
    ref = OACC.accept(z.double().numpy(), y.double().numpy(), drafts.numpy(), T, seed=9, step=5)
    ok = ~ref["margin"]
    assert (~ok).sum() <= 1
    assert np.array_equal(n_acc.cpu().numpy()[ok], ref["n_accepted"][ok])
    assert np.array_equal(out.cpu().numpy()[ok], ref["out_tokens"][ok])
    assert status_ok()


def test_chain_head_and_drafter_partials_feed_the_verify():
    """Drafter plain draws write their rows' partials into the draft-statistics buffer, the
    dense head writes the target rows' partials, and the verify's acceptance reads both."""
    B, k, d, V, T = 8, 2, 512, 65536, 1.0
    W = S.bf16(S.normal(81, (V, d), 1 / math.sqrt(d)))
    h = S.bf16(S.normal(82, (B * (k + 1), d)))
    y = torch.stack([S.make_logits(83 + i, B, V, std=1.3) for i in range(k)], dim=1)  # [B,k,V]
    y_dev = to_dev(y.contiguous())
    drafts = torch.zeros((B, k), dtype=torch.int32, device=DEV)
    n_acc = torch.empty(B, dtype=torch.int32, device=DEV)
    ws = workspace(1 << 24)
    probe = sd.AcceptDesc(batch=B, k=0, vocab=V, temperature=T, purpose=2)
    dslots = sd.sd_accept_stats_slots(probe)
    dparts = torch.full((B * k, dslots, 2), float("nan"), dtype=torch.float32, device=DEV)
    for j in range(k):
        ad = sd.AcceptDesc(batch=B, k=0, vocab=V, temperature=T, seed=11, step=100 + j,
                           purpose=2, ld_target=k * V, ld_out=k,
                           stats_out=dparts.data_ptr() + j * dslots * 8, ld_stats_out=k * dslots)
        sd.sd_accept(ad, y_dev.data_ptr() + j * V * 4, None, None, n_acc,
                     drafts.data_ptr() + j * 4, None, ws)
    hd = sd.HeadDesc(m=B * (k + 1), d=d, vocab=V, dtype=sd.SD_BF16, stats_temperature=T)
    tslots = sd.sd_lm_head_stats_slots(hd)
    tparts = torch.full((B * (k + 1), tslots, 2), float("nan"), dtype=torch.float32, device=DEV)
    hd.row_stats = tparts.data_ptr()
    z = torch.empty((B * (k + 1), V), dtype=torch.float32, device=DEV)
    sd.sd_lm_head(hd, to_dev(h), to_dev(W), z)
    desc = sd.AcceptDesc(batch=B, k=k, vocab=V, temperature=T, seed=12, step=3, purpose=1,
                         target_stats=tparts.data_ptr(), target_stats_slots=tslots,
                         draft_stats=dparts.data_ptr(), draft_stats_slots=dslots)
    out = torch.empty((B, k + 1), dtype=torch.int32, device=DEV)
    sd.sd_accept(desc, z, y_dev, drafts, n_acc, out, None, ws)
    torch.cuda.synchronize()
    zc = z.cpu().reshape(B, k + 1, V)
    ref = OACC.accept(zc.double().numpy(), y.double().numpy(), drafts.cpu().numpy(), T, seed=12,
                      step=3)
    ok = ~ref["margin"]
    assert (~ok).sum() <= 1
    assert np.array_equal(n_acc.cpu().numpy()[ok], ref["n_accepted"][ok])
    assert np.array_equal(out.cpu().numpy()[ok], ref["out_tokens"][ok])
    assert status_ok()
