"""GPU parity of sd_verify_attn / sd_draft_xattn against the float64 oracle.

Tolerance (the benchmark spec): per-row max-abs error / max-abs reference <= 2e-2 for bf16 outputs,
<= 1e-5 for float32 outputs.  The cache append is a byte copy: bit-exact.
"""
import math

import numpy as np
import pytest
import torch

import synthetic as S
import verify_step_b200 as sd
from oracle import attention as OA
from tests.gpu_util import (DEV, F64View, attn_desc, qkv, rel_err, small_paged, status_ok,
                            to_dev, workspace)

pytestmark = pytest.mark.gpu

BF16_TOL = 2e-2
F32_TOL = 1e-5


def run_verify(desc, q, kn, vn, kc, vc, table, L):
    kc_d, vc_d = to_dev(kc), to_dev(vc)
    out = torch.empty(q.shape, dtype=q.dtype, device=DEV)
    ws = workspace(sd.sd_verify_attn_workspace_size(desc))
    sd.sd_verify_attn(desc, to_dev(q), to_dev(kn), to_dev(vn), kc_d, vc_d, to_dev(table),
                      to_dev(L), out, ws)
    torch.cuda.synchronize()
    return out.cpu(), kc_d.cpu(), vc_d.cpu()


def oracle_verify(q, kn, vn, kc, vc, table, L, window, scale, bs):
    f = lambda t: t.to(torch.float64).numpy()
    return OA.verify_attention(f(q), f(kn), f(vn), f(kc), f(vc), table.numpy(), L.numpy(),
                               window, scale, bs)


def check_append(kc_out, vc_out, kn, vn, table, L, bs):
    for b in range(kn.shape[0]):
        for j in range(kn.shape[1]):
            p = int(L[b]) + j
            blk = int(table[b, p // bs])
            assert torch.equal(kc_out[blk, :, p % bs], kn[b, j])
            assert torch.equal(vc_out[blk, :, p % bs], vn[b, j])


def test_tiny_fp32_config():
    """The tiny float32 configuration: B1, L256, k2, 4q/1kv, D64, global."""
    w = S.WORKLOADS["tiny_fp32"]
    L = S.contexts(w)
    c = S.make_cache(w, 0, L, reserve=w.k + 1)
    s = S.make_step_qkv(w, 0, w.k + 1)
    desc = attn_desc(1, 3, 4, 1, 64, 16, c["max_blocks"], c["num_blocks"], 0, sd.SD_F32)
    Lt = torch.from_numpy(L)
    out, kco, vco = run_verify(desc, s["q"], s["k_new"], s["v_new"], c["k_cache"],
                               c["v_cache"], c["table"], Lt)
    ref = oracle_verify(s["q"], s["k_new"], s["v_new"], c["k_cache"], c["v_cache"],
                        c["table"], Lt, 0, desc.scale, 16)
    assert rel_err(out.numpy(), ref) <= F32_TOL
    check_append(kco, vco, s["k_new"], s["v_new"], c["table"], Lt, 16)
    assert status_ok()


CASES = [
    # (seed, L list, n_q, hq, hkv, D, bs, window)
    (1, [37, 100, 5], 3, 8, 2, 64, 16, 0),
    (2, [37, 100, 5], 1, 8, 2, 128, 32, 24),
    (3, [300, 17], 7, 16, 4, 256, 16, 0),
    (4, [300, 17], 3, 8, 2, 256, 16, 40),
    (5, [129, 64, 250, 1], 3, 16, 4, 512, 16, 0),
    (6, [129, 64], 2, 16, 4, 512, 16, 33),
    (7, [90], 5, 8, 1, 512, 16, 0),
    (8, [0, 3], 4, 4, 4, 256, 16, 0),
    (9, [200, 31], 3, 32, 2, 128, 16, 16),  # 48 rows: three 16-row tiles
    (10, [64, 70], 8, 32, 4, 256, 16, 0),    # 64 rows
    (13, [300, 17, 1000], 7, 16, 4, 512, 16, 0),  # 28 rows at D 512
    (14, [90, 260], 8, 16, 2, 512, 16, 0),        # 64 rows at D 512
    (15, [500, 40], 8, 16, 4, 512, 32, 100),      # 32 rows at D 512, sliding window
    (16, [20000], 1, 8, 1, 64, 16, 0),   # one item over every CTA: more than 512 partials
    (17, [9000], 2, 8, 2, 128, 16, 0),   # a few items, hundreds of partials each
]


@pytest.mark.parametrize("case", CASES, ids=[str(c[0]) for c in CASES])
def test_verify_bf16_small(case):
    seed, L, n_q, hq, hkv, D, bs, window = case
    B = len(L)
    c = small_paged(seed, L, n_q, hkv, D, bs, window=window)
    q, kn, vn = qkv(seed, B, n_q, hq, hkv, D)
    desc = attn_desc(B, n_q, hq, hkv, D, bs, c["mbps"], c["nb"], window)
    out, kco, vco = run_verify(desc, q, kn, vn, c["kc"], c["vc"], c["table"], c["L"])
    ref = oracle_verify(q, kn, vn, c["kc"], c["vc"], c["table"], c["L"], window, desc.scale, bs)
    assert rel_err(out.float().numpy(), ref) <= BF16_TOL
    check_append(kco, vco, kn, vn, c["table"], c["L"], bs)
    assert status_ok()


def test_verify_split_across_ctas():
    """Long contexts: every item is split over several persistent CTAs and merged by the
    combine kernel."""
    seed, L, n_q, hq, hkv, D, bs = 11, [5000, 4000], 3, 16, 4, 512, 16
    c = small_paged(seed, L, n_q, hkv, D, bs)
    q, kn, vn = qkv(seed, 2, n_q, hq, hkv, D)
    desc = attn_desc(2, n_q, hq, hkv, D, bs, c["mbps"], c["nb"], 0)
    out, _, _ = run_verify(desc, q, kn, vn, c["kc"], c["vc"], c["table"], c["L"])
    ref = oracle_verify(q, kn, vn, c["kc"], c["vc"], c["table"], c["L"], 0, desc.scale, bs)
    assert rel_err(out.float().numpy(), ref) <= BF16_TOL
    assert status_ok()


def test_verify_ignores_nan_in_unread_slots():
    """Rolled-back / never-written slots in a tile may hold NaN: the output must not see it."""
    seed, L, n_q, hq, hkv, D, bs = 12, [21, 40], 3, 8, 2, 256, 16
    c = small_paged(seed, L, n_q, hkv, D, bs, reserve=30)
    kc, vc = c["kc"].clone(), c["vc"].clone()
    for b in range(2):
        for p in range(L[b] + n_q, L[b] + 30):
            blk = int(c["table"][b, p // bs])
            kc[blk, :, p % bs] = float("nan")
            vc[blk, :, p % bs] = float("nan")
    q, kn, vn = qkv(seed, 2, n_q, hq, hkv, D)
    desc = attn_desc(2, n_q, hq, hkv, D, bs, c["mbps"], c["nb"], 0)
    out, _, _ = run_verify(desc, q, kn, vn, kc, vc, c["table"], c["L"])
    assert torch.isfinite(out.float()).all()
    ref = oracle_verify(q, kn, vn, c["kc"], c["vc"], c["table"], c["L"], 0, desc.scale, bs)
    assert rel_err(out.float().numpy(), ref) <= BF16_TOL


# Sliding windows of at most 2048 keys run on the cluster kernel (one cluster of CTAs per
# (sequence, kv head), partials merged in distributed shared memory); longer windows on the
# persistent split-KV kernel.  Cases cover two 16-row tiles, head dims 64..512, a single
# sequence (largest clusters), a batch too large for clusters (one CTA per item), tile rings
# that wrap (more tiles per CTA than stages) and a window past the cluster limit.
WINDOW_CASES = [
    # (seed, L list, n_q, hq, hkv, D, bs, window)
    (31, [700, 20, 513], 7, 16, 4, 256, 16, 100),   # 28 rows
    (32, [1000], 3, 8, 2, 64, 16, 300),             # B1: clusters of 8
    (33, [2500, 2200, 3000], 1, 16, 4, 512, 32, 2048),  # 129 tiles per item: the ring wraps
    (34, [600] * 40, 3, 8, 2, 128, 16, 512),        # 80 items: one CTA each, ring wraps
    (35, [5000, 4100], 3, 16, 4, 256, 16, 3000),    # past the cluster limit: split-KV kernel
    (36, [8, 1, 40], 2, 8, 2, 256, 16, 512),        # window longer than every context
]


@pytest.mark.parametrize("case", WINDOW_CASES, ids=[str(c[0]) for c in WINDOW_CASES])
def test_verify_window(case):
    seed, L, n_q, hq, hkv, D, bs, window = case
    B = len(L)
    c = small_paged(seed, L, n_q, hkv, D, bs, window=window)
    q, kn, vn = qkv(seed, B, n_q, hq, hkv, D)
    desc = attn_desc(B, n_q, hq, hkv, D, bs, c["mbps"], c["nb"], window)
    out, kco, vco = run_verify(desc, q, kn, vn, c["kc"], c["vc"], c["table"], c["L"])
    ref = oracle_verify(q, kn, vn, c["kc"], c["vc"], c["table"], c["L"], window, desc.scale, bs)
    assert rel_err(out.float().numpy(), ref) <= BF16_TOL
    check_append(kco, vco, kn, vn, c["table"], c["L"], bs)
    assert status_ok()


def test_window_ignores_nan_outside_the_window():
    """Slots older than the window and slots past the new rows may hold NaN."""
    seed, L, n_q, hq, hkv, D, bs, window = 37, [300, 90], 3, 16, 4, 256, 16, 64
    c = small_paged(seed, L, n_q, hkv, D, bs, reserve=30)
    kc, vc = c["kc"].clone(), c["vc"].clone()
    for b in range(2):
        old = range(0, max(0, L[b] + 1 - window))
        new = range(L[b] + n_q, L[b] + 30)
        for p in list(old) + list(new):
            blk = int(c["table"][b, p // bs])
            kc[blk, :, p % bs] = float("nan")
            vc[blk, :, p % bs] = float("nan")
    q, kn, vn = qkv(seed, 2, n_q, hq, hkv, D)
    desc = attn_desc(2, n_q, hq, hkv, D, bs, c["mbps"], c["nb"], window)
    out, _, _ = run_verify(desc, q, kn, vn, kc, vc, c["table"], c["L"])
    assert torch.isfinite(out.float()).all()
    ref = oracle_verify(q, kn, vn, c["kc"], c["vc"], c["table"], c["L"], window, desc.scale, bs)
    assert rel_err(out.float().numpy(), ref) <= BF16_TOL
    assert status_ok()


@pytest.mark.parametrize("window", [0, 64])
def test_out_of_range_block_is_flagged(window):
    """A block-table entry outside [0, num_blocks) inside the key range: the tile is skipped
    (never copied) and the device status reports SD_ERR_DEVICE."""
    seed, L, n_q, hq, hkv, D, bs = 38, [100, 50], 3, 8, 2, 256, 16
    c = small_paged(seed, L, n_q, hkv, D, bs)
    table = c["table"].clone()
    table[0, 5] = c["nb"] + 7  # positions 80..95 of sequence 0: inside both key ranges
    q, kn, vn = qkv(seed, 2, n_q, hq, hkv, D)
    desc = attn_desc(2, n_q, hq, hkv, D, bs, c["mbps"], c["nb"], window)
    out, _, _ = run_verify(desc, q, kn, vn, c["kc"], c["vc"], table, c["L"])
    assert sd.sd_device_status_read() == sd.SD_ERR_DEVICE
    sd.sd_device_status_clear()
    # the other sequence is untouched by the bad entry
    ref = oracle_verify(q, kn, vn, c["kc"], c["vc"], c["table"], c["L"], window, desc.scale, bs)
    assert rel_err(out[1].float().numpy(), ref[1]) <= BF16_TOL


DRAFT_CASES = [
    (21, [37, 100, 5], [40, 99, 0], 8, 2, 256, 16, 24),
    (22, [300, 17], [299, 500], 16, 4, 512, 16, 0),
    (23, [64, 0, 9], [63, 5, 2], 16, 4, 256, 16, 512),
    (24, [20000], [19999], 8, 1, 64, 16, 0),   # one item over every CTA: over 512 partials
    (25, [9000], [8999], 8, 2, 512, 16, 0),    # B 1 at D 512: hundreds of partials per item
]


@pytest.mark.parametrize("case", DRAFT_CASES, ids=[str(c[0]) for c in DRAFT_CASES])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_draft_xattn(case, dtype):
    seed, L, qpos, hq, hkv, D, bs, window = case
    B = len(L)
    c = small_paged(seed, L, 1, hkv, D, bs, dtype=dtype, window=window)
    q, _, _ = qkv(seed, B, 1, hq, hkv, D, dtype=dtype)
    desc = attn_desc(B, 1, hq, hkv, D, bs, c["mbps"], c["nb"], window,
                     sd.SD_BF16 if dtype == "bf16" else sd.SD_F32)
    qp = torch.tensor(qpos, dtype=torch.int32)
    out = torch.empty(q.shape, dtype=q.dtype, device=DEV)
    ws = workspace(sd.sd_draft_xattn_workspace_size(desc))
    kc_d, vc_d = to_dev(c["kc"]), to_dev(c["vc"])
    sd.sd_draft_xattn(desc, to_dev(q), kc_d, vc_d, to_dev(c["table"]), to_dev(c["L"]),
                      to_dev(qp), out, ws)
    torch.cuda.synchronize()
    assert torch.equal(kc_d.cpu(), c["kc"])  # read-only
    f = lambda t: t.to(torch.float64).numpy()
    ref = OA.draft_attention(f(q), f(c["kc"]), f(c["vc"]), c["table"].numpy(), c["L"].numpy(),
                             qp.numpy(), window, desc.scale, bs)
    tol = BF16_TOL if dtype == "bf16" else F32_TOL
    got = out.cpu().float().numpy()
    for b in range(B):
        if np.abs(ref[b]).max() == 0:
            assert np.all(got[b] == 0)
        else:
            assert rel_err(got[b], ref[b]) <= tol
    assert status_ok()


def _sampled_check(w, layer, n_q, L, cache, step, samples, seed):
    """Full-size verify on workload ``w``: all appended rows bit-exact, sampled outputs vs
    the oracle computed one by one (samples=None: every (sequence, position, head) row)."""
    lay = w.layers[layer]
    s = S.make_step_qkv(w, layer, n_q, step)
    B = w.batch
    desc = attn_desc(B, n_q, w.h_q, w.h_kv, lay.head_dim, w.block_size, cache["max_blocks"],
                     cache["num_blocks"], lay.window)
    Lt = torch.from_numpy(np.asarray(L, np.int32))
    out, kco, vco = run_verify(desc, s["q"], s["k_new"], s["v_new"], cache["k_cache"],
                               cache["v_cache"], cache["table"], Lt)
    check_append(kco, vco, s["k_new"], s["v_new"], cache["table"], Lt, w.block_size)
    rng = np.random.default_rng(seed)
    f = lambda t: t.to(torch.float64).numpy()
    q64, kn64, vn64 = f(s["q"]), f(s["k_new"]), f(s["v_new"])
    kc64, vc64 = F64View(cache["k_cache"]), F64View(cache["v_cache"])
    table = cache["table"].numpy()
    worst = 0.0
    if samples is None:
        picks = [(b, j, h) for b in range(B) for j in range(n_q) for h in range(w.h_q)]
    else:
        picks = [(int(rng.integers(B)), int(rng.integers(n_q)), int(rng.integers(w.h_q)))
                 for _ in range(samples)]
    for b, j, h in picks:
        ref = OA.verify_attention_one(b, j, h, q64, kn64, vn64, kc64, vc64, table, L,
                                      lay.window, desc.scale, w.block_size)
        worst = max(worst, rel_err(out[b, j, h].float().numpy()[None], ref[None]))
    assert worst <= BF16_TOL
    assert status_ok()
    return out


@pytest.mark.parametrize("k", [1, 2, 4, 6])
def test_global_config_full_size(k):
    """B8, L16384, D512, 16q/4kv, block 16, k swept: sampled outputs vs the oracle."""
    w = S.WORKLOADS["global"]
    L = S.contexts(w)
    cache = S.make_cache(w, 0, L, reserve=8)
    _sampled_check(w, 0, k + 1, L, cache, step=k, samples=24, seed=k)


def test_edge_config_full():
    """B1, L4096, sliding window 512, D256, 8q/2kv, k2: all 24 output rows vs the oracle."""
    w = S.WORKLOADS["edge"]
    L = S.contexts(w)
    cache = S.make_cache(w, 0, L, reserve=3)
    _sampled_check(w, 0, 3, L, cache, step=0, samples=None, seed=5)


@pytest.mark.parametrize("layer", [0, 1])
def test_serving_config_full_size(layer):
    """B64, ragged L in [1024, 16384], shuffled blocks, sliding D256 and global D512."""
    w = S.WORKLOADS["serving"]
    L = S.contexts(w)
    cache = S.make_cache(w, layer, L, reserve=3)
    _sampled_check(w, layer, 3, L, cache, step=0, samples=24, seed=layer)


def test_drafter_config_full_size():
    """Drafter cross-attention on the B8 x L16384 shared cache (sliding D256 W512 and global
    D512 layers), query positions inside the committed range."""
    w = S.WORKLOADS["drafter"]
    L = S.contexts(w)
    rng = np.random.default_rng(4)
    for layer in (0, 1):
        lay = w.layers[layer]
        cache = S.make_cache(w, layer, L, reserve=w.k + 1)
        q = S.bf16(S.normal(77 + layer, (w.batch, 1, w.h_q, lay.head_dim),
                            1 / math.sqrt(lay.head_dim)))
        qp = torch.from_numpy((L - 1).astype(np.int32))
        desc = attn_desc(w.batch, 1, w.h_q, w.h_kv, lay.head_dim, w.block_size,
                         cache["max_blocks"], cache["num_blocks"], lay.window)
        out = torch.empty(q.shape, dtype=q.dtype, device=DEV)
        ws = workspace(sd.sd_draft_xattn_workspace_size(desc))
        sd.sd_draft_xattn(desc, to_dev(q), to_dev(cache["k_cache"]), to_dev(cache["v_cache"]),
                          to_dev(cache["table"]), to_dev(torch.from_numpy(L)), to_dev(qp), out, ws)
        torch.cuda.synchronize()
        q64 = q.to(torch.float64).numpy()
        for _ in range(12):
            b, h = int(rng.integers(w.batch)), int(rng.integers(w.h_q))
            ref = OA.draft_attention_one(b, h, q64, F64View(cache["k_cache"]),
                                         F64View(cache["v_cache"]), cache["table"].numpy(), L,
                                         qp.numpy(), lay.window, desc.scale, w.block_size)
            assert rel_err(out[b, 0, h].cpu().float().numpy()[None], ref[None]) <= BF16_TOL
    assert status_ok()


def test_draft_xattn_position_from_context_length():
    """q_pos == NULL: the query sits at ctx_len + q_offset (a drafter chain step)."""
    seed, L, hq, hkv, D, bs, window = 24, [300, 40, 77], 16, 4, 256, 16, 64
    B = len(L)
    c = small_paged(seed, L, 1, hkv, D, bs)
    q, _, _ = qkv(seed, B, 1, hq, hkv, D)
    kc_d, vc_d, tab, Ld = to_dev(c["kc"]), to_dev(c["vc"]), to_dev(c["table"]), to_dev(c["L"])
    for j in (0, 1, 3):
        desc = attn_desc(B, 1, hq, hkv, D, bs, c["mbps"], c["nb"], window)
        desc.q_offset = j
        ws = workspace(sd.sd_draft_xattn_workspace_size(desc))
        out_a = torch.empty(q.shape, dtype=q.dtype, device=DEV)
        out_b = torch.empty(q.shape, dtype=q.dtype, device=DEV)
        sd.sd_draft_xattn(desc, to_dev(q), kc_d, vc_d, tab, Ld, None, out_a, ws)
        qp = to_dev(c["L"] + j)
        sd.sd_draft_xattn(desc, to_dev(q), kc_d, vc_d, tab, Ld, qp, out_b, ws)
        torch.cuda.synchronize()
        assert torch.equal(out_a, out_b)
        f = lambda t: t.to(torch.float64).numpy()
        ref = OA.draft_attention(f(q), f(c["kc"]), f(c["vc"]), c["table"].numpy(),
                                 c["L"].numpy(), (c["L"] + j).numpy(), window, desc.scale, bs)
        assert rel_err(out_a.cpu().float().numpy(), ref) <= BF16_TOL
    assert status_ok()
