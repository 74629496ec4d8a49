"""Multi-layer target verify on the GPU (sd_linear projections around sd_verify_attn, one
sliding and one global layer) against the float64 oracle.

Tolerance: the bf16 bar of the attention tests, per-row max-abs error / max-abs reference
<= 2e-2 (bf16 roundings sit on the path: normalised rows, queries, keys, values, attention
outputs and the MLP activation).  The appended cache rows are the kernel's own k and v
projections, copied bit for bit.
"""
import numpy as np
import pytest
import torch

import synthetic as S
import verify_step_b200 as sd
from oracle import target as OT
from tests.gpu_util import DEV, F64View, attn_desc, rel_err, small_paged, status_ok, to_dev
from tests.gpu_util import workspace
from verify_step_b200 import target as VT

pytestmark = pytest.mark.gpu

BF16_TOL = 2e-2


def f64(t):
    return t.detach().cpu().double().numpy()


@pytest.mark.parametrize("B,k,d,ff", [(8, 2, 2048, 4096), (4, 1, 2048, 4096),
                                      (8, 2, 5376, 21504)],
                         ids=["b8k2-d2048", "b4k1-d2048", "b8k2-d5376-full-width"])
def test_two_layer_verify_matches_the_oracle(B, k, d, ff):
    """The last case is the benchmark's own width: d 5376, MLP 21504 (gate and up rows
    n 43008, W_d k 21504)."""
    n_q, hq, hkv, bs = k + 1, 16, 4, 16
    layers = ((256, 512), (512, 0))
    rng = np.random.default_rng(100 + B)
    L = rng.integers(300, 1200, B).astype(np.int32)
    host = S.make_target_weights(B + k, d, ff, hq, hkv, layers)
    caches_h = [small_paged(40 + 7 * i + B, L, n_q, hkv, D, bs) for i, (D, _) in
                enumerate(layers)]
    x0 = torch.from_numpy(S.normal(91 + B, (B * n_q, d), 1.0))
    shape = VT.TargetShape(batch=B, n_q=n_q, d=d, ff=ff, h_q=hq, h_kv=hkv, layers=layers)
    wts = VT.device_weights(host)
    buf = VT.buffers(shape)
    buf["x"].copy_(x0.to(DEV))
    caches = []
    for (D, W), c in zip(layers, caches_h):
        caches.append(dict(desc=attn_desc(B, n_q, hq, hkv, D, bs, c["mbps"], c["nb"], W),
                           k=to_dev(c["kc"]), v=to_dev(c["vc"]), table=to_dev(c["table"])))
    ctx = to_dev(torch.from_numpy(L))
    ws = workspace(max(sd.sd_verify_attn_workspace_size(c["desc"]) for c in caches))
    VT.verify_layers(shape, wts, buf, caches, ctx, ws)
    torch.cuda.synchronize()

    lw = []
    for L_h, (D, W) in zip(host, layers):
        e = {kk: f64(v) for kk, v in L_h.items() if isinstance(v, torch.Tensor)}
        e.update(head_dim=D, window=W, Wg=f64(L_h["Wg"]), Wu=f64(L_h["Wu"]))
        lw.append(e)
    oc = [dict(k=F64View(c["kc"]), v=F64View(c["vc"]), table=c["table"].numpy(),
               block_size=bs) for c in caches_h]
    ref = OT.verify_layers(f64(x0), lw, oc, L, n_q, hq, hkv)

    assert rel_err(f64(buf["x"]), ref["x"][-1]) <= BF16_TOL
    for i, (D, _) in enumerate(layers):
        assert rel_err(f64(buf["o"][i]), ref["o"][i]) <= BF16_TOL, i
        kn = f64(buf["k"][i]).reshape(B, n_q, hkv, D)
        assert rel_err(kn, ref["k_new"][i]) <= BF16_TOL, i
        # the appended rows are the kernel's own k and v projections, bit for bit
        kc, vc = caches[i]["k"].cpu(), caches[i]["v"].cpu()
        table = caches_h[i]["table"].numpy()
        kb = buf["k"][i].cpu().view(B, n_q, hkv, D)
        vb = buf["v"][i].cpu().view(B, n_q, hkv, D)
        for b in range(B):
            for j in range(n_q):
                pos = int(L[b]) + j
                blk = table[b, pos // bs]
                assert torch.equal(kc[blk, :, pos % bs], kb[b, j])
                assert torch.equal(vc[blk, :, pos % bs], vb[b, j])
    assert torch.equal(ctx.cpu(), torch.from_numpy(L))  # the verify does not commit
    assert status_ok()
