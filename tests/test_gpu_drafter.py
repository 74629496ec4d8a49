"""Drafter dense layers on the GPU (sd_linear and one drafter link) against the float64 oracle.

Tolerance (the bf16 bar of the attention tests): per-row max-abs error / max-abs reference
<= 2e-2 wherever a bf16 rounding sits on the path (a normalised or float32 input row rounded to
bf16 for the tensor cores, a bf16 output); <= 1e-5 for float32 outputs of bf16-exact inputs,
where only the float32 summation order differs from the oracle.
"""
import math

import numpy as np
import pytest
import torch

import synthetic as S
import verify_step_b200 as sd
from oracle import drafter as DR
from tests.gpu_util import DEV, F64View, attn_desc, rel_err, small_paged, status_ok, to_dev
from verify_step_b200 import drafter as VD

pytestmark = pytest.mark.gpu

BF16_TOL, F32_TOL = 2e-2, 1e-5


def f64(t):
    return t.detach().cpu().double().numpy()


# (m, n, k, x_dtype, norm, epilogue, out_dtype, k_gather)
LINEAR_CASES = [
    (8, 8192, 1024, "f32", True, "store", "bf16", 0),     # W_q of the global layer
    (8, 1024, 8192, "bf16", False, "add", "f32", 0),      # W_o of the global layer
    (8, 8192, 1024, "f32", True, "geglu", "bf16", 0),     # gate and up rows
    (8, 1024, 4096, "bf16", False, "add", "f32", 0),      # W_d
    (8, 1024, 6400, "bf16", False, "store", "f32", 1024),  # W_in with the embedding gather
    (8, 5376, 1024, "f32", True, "store", "bf16", 0),     # W_back (with the normalised copy)
    (5, 48, 96, "f32", True, "store", "f32", 0),          # ragged: a half row block, 3 chunks
    (3, 48, 64, "f32", True, "geglu", "bf16", 0),         # gated, half row block
    (1, 16, 32, "bf16", False, "store", "f32", 0),        # the smallest shape
    (24, 1024, 8192, "bf16", False, "add", "f32", 0),     # three token groups
    (64, 2048, 6400, "f32", True, "store", "bf16", 0),    # 64 rows: several staged pieces
    (33, 160, 2048, "bf16", False, "store", "f32", 2048),  # every column gathered
    (12, 1024, 2048, "f32", True, "store", "bf16", 0),    # two token groups (B 4, k 2)
    (16, 512, 4096, "bf16", False, "add", "f32", 0),      # two full token groups
    (24, 2048, 1024, "f32", True, "geglu", "bf16", 0),    # three groups, gated (B 8, k 2)
    # the target's projections at d 5376, MLP 21504 (B 8, k 2: 24 rows)
    (24, 8192, 5376, "f32", True, "store", "bf16", 0),    # W_q of a global layer
    (24, 1024, 5376, "f32", True, "store", "bf16", 0),    # W_k of a sliding layer
    (24, 5376, 8192, "bf16", False, "add", "f32", 0),     # W_o of a global layer
    (24, 43008, 5376, "f32", True, "geglu", "bf16", 0),   # gate and up rows of the MLP
    (24, 5376, 21504, "bf16", False, "add", "f32", 0),    # W_d of the MLP
    (48, 4096, 5376, "f32", True, "store", "f32", 0),     # B 8, k 5: 48 rows
]


def run_linear(m, n, k, x_dtype, norm, epi, out_dtype, k_gather, seed=0, bad_token=False):
    rng = np.random.default_rng(seed)
    k_x = k - k_gather
    xs = S.normal(100 + seed, (m, max(k_x, 1)), 1.0)
    x = S.bf16(xs) if x_dtype == "bf16" else torch.from_numpy(xs)
    W = S.bf16(S.normal(200 + seed, (n, k), 1 / math.sqrt(k)))
    gain = torch.from_numpy(1 + S.normal(300 + seed, (k,), 0.1)) if norm else None
    V = 1000
    table = S.bf16(S.normal(400 + seed, (V, k_gather), 1.0)) if k_gather else None
    toks = torch.from_numpy(rng.integers(0, V, (m, 3)).astype(np.int32))
    sel = torch.from_numpy(rng.integers(0, 3, m).astype(np.int32))
    if bad_token:
        toks[0, sel[0]] = V + 5
    # oracle input rows
    parts = []
    if k_x:
        parts.append(f64(x))
    if k_gather:
        ids = toks.numpy()[np.arange(m), sel.numpy()]
        e = np.zeros((m, k_gather))
        ok = (ids >= 0) & (ids < V)
        e[ok] = f64(table)[ids[ok]]
        parts.append(e)
    xr = np.concatenate(parts, axis=1)
    if norm:
        xr = DR.rmsnorm(xr, f64(gain))
    out_cols = n // 2 if epi == "geglu" else n
    out_t = torch.float32 if out_dtype == "f32" else torch.bfloat16
    out0 = torch.from_numpy(S.normal(500 + seed, (m, out_cols), 1.0)) if epi == "add" else None
    if epi == "geglu":
        Wg, Wu = W[: n // 2], W[n // 2:]
        ref = DR.geglu(xr, f64(Wg), f64(Wu))
        W_dev = to_dev(VD.gate_up_blocks(Wg, Wu))
    else:
        ref = DR.linear(xr, f64(W))
        W_dev = to_dev(W)
        if epi == "add":
            ref = f64(out0) + ref
    desc = sd.LinearDesc(m=m, n=n, k=k, x_dtype=sd.SD_BF16 if x_dtype == "bf16" else sd.SD_F32,
                         ld_x=max(k_x, 4) if k_x else 0, k_gather=k_gather, ld_table=k_gather,
                         table_rows=V, ld_tokens=3, norm_eps=DR.RMS_EPS,
                         epilogue={"store": sd.SD_EPI_STORE, "add": sd.SD_EPI_ADD,
                                   "geglu": sd.SD_EPI_GEGLU}[epi],
                         out_dtype=sd.SD_BF16 if out_dtype == "bf16" else sd.SD_F32,
                         ld_out=out_cols)
    keep = []
    if norm:
        g_dev = to_dev(gain)
        keep.append(g_dev)
        desc.norm_gain = g_dev.data_ptr()
        normed = torch.full((m, k), float("nan"), dtype=torch.bfloat16, device=DEV)
        desc.norm_out, desc.ld_norm_out = normed.data_ptr(), k
    outs = []
    # a NaN-filled workspace: a read of a slot the call did not write fails the comparison
    ws = torch.full((max(256, sd.sd_linear_workspace_size(desc)) // 4,), float("nan"),
                    dtype=torch.float32, device=DEV)
    for _ in range(2):  # twice: the result must not depend on the launch
        out = to_dev(out0) if epi == "add" else torch.full((m, out_cols), float("nan"),
                                                            dtype=out_t, device=DEV)
        sd.sd_linear(desc, to_dev(x) if k_x else None, W_dev, out,
                     table=to_dev(table) if k_gather else None,
                     tokens=to_dev(toks) if k_gather else None,
                     token_sel=to_dev(sel) if k_gather else None, ws=ws)
        torch.cuda.synchronize()
        outs.append(out.cpu())
    assert torch.equal(outs[0], outs[1])
    res = dict(got=f64(outs[0]), ref=ref)
    if norm:
        res["normed"] = f64(normed)
        res["normed_ref"] = xr
    return res


@pytest.mark.parametrize("case", LINEAR_CASES, ids=lambda c: "-".join(map(str, c)))
def test_linear_matches_the_oracle(case):
    m, n, k, x_dtype, norm, epi, out_dtype, k_gather = case
    r = run_linear(*case)
    exact_operand = not norm and x_dtype == "bf16"
    tol = F32_TOL if (out_dtype == "f32" and exact_operand) else BF16_TOL
    assert rel_err(r["got"], r["ref"]) <= tol
    if norm:
        assert rel_err(r["normed"], r["normed_ref"]) <= BF16_TOL
    assert status_ok()


def test_linear_token_out_of_range_reads_zeros_and_is_recorded():
    r = run_linear(4, 64, 128, "bf16", False, "store", "f32", 64, seed=3, bad_token=True)
    assert rel_err(r["got"], r["ref"]) <= F32_TOL  # the oracle used a zero row there
    assert sd.sd_device_status_read() == sd.SD_ERR_DEVICE
    sd.sd_device_status_clear()


def test_linear_unsupported_shapes_refused():
    desc = sd.LinearDesc(m=65, n=32, k=64, x_dtype=sd.SD_F32, ld_x=64, epilogue=sd.SD_EPI_STORE,
                         out_dtype=sd.SD_F32, ld_out=32)
    x = torch.zeros((65, 64), device=DEV)
    W = torch.zeros((32, 64), dtype=torch.bfloat16, device=DEV)
    out = torch.zeros((65, 32), device=DEV)
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device=DEV)
    with pytest.raises(sd.SdError):
        sd.sd_linear(desc, x, W, out, ws=ws)
    # a workspace smaller than sd_linear_workspace_size is refused before any launch
    desc.m = 8
    need = sd.sd_linear_workspace_size(desc)
    assert need > 0
    with pytest.raises(sd.SdError) as e:
        sd.sd_linear(desc, x, W, out, ws=ws[: need - 256])
    assert e.value.status == sd.SD_ERR_WORKSPACE


# ----------------------------------------------------------------------------- one link

def make_link_case(B=8, seed=7):
    hq, hkv, bs = 16, 4, 16
    d, dt, F, V = 1024, 5376, S.DRAFTER_FF, 4096
    dims = (256, 256, 256, 512)
    L = np.random.default_rng(seed).integers(600, 2000, B).astype(np.int32)
    caches = {D: small_paged(seed * 3 + D, L, 1, hkv, D, bs, reserve=8) for D in (256, 512)}
    host = S.make_drafter_weights(seed, d, dt, V, hq, dims, F)
    return dict(B=B, hq=hq, hkv=hkv, bs=bs, d=d, dt=dt, F=F, V=V, dims=dims, L=L,
                caches=caches, host=host)


def oracle_links(c, h0, tok0, tok1):
    wts = {k: f64(c["host"][k]) for k in ("E", "W_in", "g_final", "W_back")}
    wts["layers"] = [{k: f64(v) for k, v in lw.items()} for lw in c["host"]["layers"]]
    cache = {D: dict(k=F64View(p["kc"]), v=F64View(p["vc"]), table=p["table"].numpy(),
                     block_size=c["bs"]) for D, p in c["caches"].items()}
    outs, h_prev = [], f64(h0)
    for j, tokens in enumerate((tok0, tok1)):
        atts = [DR.cross_attend(cache[D], c["hq"], D, 512 if D == 256 else 0, c["L"], j)
                for D in c["dims"]]
        o = DR.drafter_step(h_prev, tokens, wts, atts)
        outs.append(o)
        h_prev = o["h_back"]
    return outs


def test_two_link_chain_matches_the_oracle():
    c = make_link_case()
    B, d, dt = c["B"], c["d"], c["dt"]
    shape = VD.DrafterShape(batch=B, d=d, d_target=dt, ff=c["F"], h_q=c["hq"],
                            head_dims=c["dims"], vocab=c["V"])
    wts = VD.device_weights(c["host"])
    buf = VD.buffers(shape)
    dev_cache = {D: dict(kc=to_dev(p["kc"]), vc=to_dev(p["vc"]), table=to_dev(p["table"]),
                         nb=p["nb"], mbps=p["mbps"]) for D, p in c["caches"].items()}
    ctx = to_dev(torch.from_numpy(c["L"]))
    ws = torch.empty(1 << 26, dtype=torch.uint8, device=DEV)
    rng = np.random.default_rng(11)
    h0 = S.bf16(S.normal(12, (B, dt), 1.0))
    out_tokens = torch.from_numpy(rng.integers(0, c["V"], (B, 3)).astype(np.int32))
    n_acc = torch.from_numpy(rng.integers(0, 3, B).astype(np.int32))
    drafts = torch.from_numpy(rng.integers(0, c["V"], (B, 2)).astype(np.int32))
    tok0 = out_tokens.numpy()[np.arange(B), n_acc.numpy()]
    tok1 = drafts.numpy()[:, 0]
    ref = oracle_links(c, h0, tok0, tok1)

    def attend_for(j, record):
        def attend(i, q, o):
            D = c["dims"][i]
            p = dev_cache[D]
            desc = attn_desc(B, 1, c["hq"], c["hkv"], D, c["bs"], p["mbps"], p["nb"],
                             512 if D == 256 else 0)
            desc.q_offset = j
            sd.sd_draft_xattn(desc, q, p["kc"], p["vc"], p["table"], ctx, None, o, ws)
            record.append(None)
        return attend

    got = []
    h_prev = to_dev(h0)
    tokens_dev = [(to_dev(out_tokens), 3, to_dev(n_acc)), (to_dev(drafts), 2, None)]
    for j in range(2):
        calls = []
        toks, ld, sel = tokens_dev[j]
        VD.link(shape, wts, buf, h_prev, toks, ld, attend_for(j, calls), token_sel=sel)
        torch.cuda.synchronize()
        assert len(calls) == 4
        got.append(dict(x=f64(buf["x"]), h=f64(buf["h"]), h_back=f64(buf["h_back"])))
        h_prev = buf["h_back"].clone()
    for j in range(2):
        assert rel_err(got[j]["x"], ref[j]["x"][-1]) <= BF16_TOL, j
        assert rel_err(got[j]["h"], ref[j]["h"]) <= BF16_TOL, j
        assert rel_err(got[j]["h_back"], ref[j]["h_back"]) <= BF16_TOL, j
    assert status_ok()
