"""GPU parity of sd_lm_head (dense tcgen05 path, float32 path, clustered two-stage head)."""
import math

import numpy as np
import pytest
import torch

import synthetic as S
import verify_step_b200 as sd
from oracle import lm_head as OH
from tests.gpu_util import DEV, F64View, rel_err, status_ok, to_dev, workspace

pytestmark = pytest.mark.gpu

F32_OUT_TOL = 1e-5  # float32 logits vs the float64 oracle


def head_desc(m, d, V, dtype=sd.SD_BF16, ld=0, C=0, cs=0, top_c=0):
    return sd.HeadDesc(m=m, d=d, vocab=V, ld_logits=ld, n_clusters=C, cluster_size=cs,
                       top_c=top_c, dtype=dtype)


def run_dense(h, W, ld=0):
    m, d = h.shape
    V = W.shape[0]
    desc = head_desc(m, d, V, sd.SD_BF16 if h.dtype == torch.bfloat16 else sd.SD_F32, ld)
    ldv = ld or V
    logits = torch.full((m, ldv), float("nan"), dtype=torch.float32, device=DEV)
    sd.sd_lm_head(desc, to_dev(h), to_dev(W), logits)
    torch.cuda.synchronize()
    return logits.cpu()


def test_tiny_fp32_config():
    w = S.WORKLOADS["tiny_fp32"]
    h = S.make_hidden(w, 3)
    W = S.make_lm_head(w)
    out = run_dense(h, W)
    ref = OH.lm_head(h.double().numpy(), W.double().numpy())
    assert rel_err(out.numpy(), ref) <= F32_OUT_TOL


@pytest.mark.parametrize("m,d,V", [(1, 64, 128), (3, 2560, 4096), (24, 128, 1000),
                                   (40, 320, 2176), (56, 192, 3000), (100, 64, 640),
                                   (192, 256, 1536), (300, 128, 1024)])
def test_dense_bf16_shapes(m, d, V):
    h = S.bf16(S.normal(m * 7 + d, (m, d)))
    W = S.bf16(S.normal(V + d, (V, d), 1 / math.sqrt(d)))
    out = run_dense(h, W)
    ref = OH.lm_head(h.double().numpy(), W.double().numpy())
    assert rel_err(out.numpy(), ref) <= F32_OUT_TOL
    assert status_ok()


def test_dense_bf16_row_stride():
    """ld_logits > vocab: rows land at their stride, the padding is untouched."""
    m, d, V, ld = 5, 128, 512, 700
    h = S.bf16(S.normal(1, (m, d)))
    W = S.bf16(S.normal(2, (V, d), 1 / math.sqrt(d)))
    out = run_dense(h, W, ld=ld)
    assert torch.isnan(out[:, V:]).all()
    ref = OH.lm_head(h.double().numpy(), W.double().numpy())
    assert rel_err(out[:, :V].numpy(), ref) <= F32_OUT_TOL


@pytest.mark.parametrize("name,m", [("global", 24), ("serving", 192), ("edge", 3),
                                    ("global", 56)])
def test_full_vocab_sampled(name, m):
    """Full-size heads (d 5376 or 2560, V 262144): sampled vocabulary rows vs the oracle."""
    w = S.WORKLOADS[name]
    W = S.make_lm_head(w)
    h = S.make_hidden(w, m)
    out = run_dense(h, W)
    assert torch.isfinite(out).all()
    rng = np.random.default_rng(m)
    cols = np.sort(rng.choice(w.vocab, size=3000, replace=False))
    cols[-1] = w.vocab - 1
    ref = OH.lm_head(h.double().numpy(), F64View(W), cols)
    assert rel_err(out[:, cols].numpy(), ref) <= F32_OUT_TOL
    assert status_ok()


def _run_clustered(h, cl, top_c):
    C, cs, d = cl["w_cm"].shape
    m = h.shape[0]
    desc = head_desc(m, d, C * cs, C=C, cs=cs, top_c=top_c)
    logits = torch.empty((m, C * cs), dtype=torch.float32, device=DEV)
    sel = torch.full((m, top_c), -7, dtype=torch.int32, device=DEV)
    ws = workspace(sd.sd_lm_head_workspace_size(desc))
    sd.sd_lm_head(desc, to_dev(h), to_dev(cl["w_cm"]), logits, centroids=to_dev(cl["centroids"]),
                  cluster_tokens=to_dev(cl["cluster_tokens"]), sel_clusters=sel, ws=ws)
    torch.cuda.synchronize()
    return logits.cpu(), sel.cpu()


def _check_clustered(h, cl, top_c, gap_tol=1e-5):
    logits, sel = _run_clustered(h, cl, top_c)
    ref, ref_sel, gap = OH.clustered_lm_head(h.double().numpy(),
                                             cl["centroids"].double().numpy(),
                                             F64View(cl["w_cm"]), cl["cluster_tokens"].numpy(),
                                             top_c)
    scores = OH.cluster_scores(h.double().numpy(), cl["centroids"].double().numpy())
    n_near = 0
    for r in range(h.shape[0]):
        if gap[r] < gap_tol * max(1.0, abs(scores[r].max())):
            n_near += 1  # near-tie at the selection boundary: check validity only
            got = set(sel[r].tolist())
            assert len(got) == top_c and all(0 <= c < cl["w_cm"].shape[0] for c in got)
            continue
        assert sel[r].tolist() == ref_sel[r].tolist()
        fin = np.isfinite(ref[r])
        assert np.array_equal(np.isfinite(logits[r].numpy()), fin)
        assert np.all(logits[r].numpy()[~fin] == -np.inf)
        assert rel_err(logits[r].numpy()[fin][None], ref[r][fin][None]) <= F32_OUT_TOL
    return n_near


def test_clustered_small():
    w = S.Workload("c", 4, 0, 0, 4, 1, [], 128, 64 * 16, n_clusters=64, cluster_size=16,
                   drafter_hidden=128, seed=31)
    cl = S.make_clustered_head(w)
    h = S.bf16(S.normal(5, (5, 128)))
    assert _check_clustered(h, cl, 5) <= 1
    assert status_ok()


def test_clustered_keep_all_equals_dense():
    w = S.Workload("c", 4, 0, 0, 4, 1, [], 64, 32 * 8, n_clusters=32, cluster_size=8,
                   drafter_hidden=64, seed=32)
    cl = S.make_clustered_head(w)
    h = S.bf16(S.normal(6, (3, 64)))
    logits, sel = _run_clustered(h, cl, 32)
    assert sel.tolist() == [list(range(32))] * 3
    W = torch.empty(256, 64, dtype=torch.bfloat16)
    W[cl["cluster_tokens"].reshape(-1).long()] = cl["w_cm"].reshape(-1, 64)
    dense = run_dense(h, W)
    assert rel_err(logits.numpy(), dense.numpy()) <= 1e-6


def test_drafter_clustered_config():
    """1024 clusters x 256 tokens, d 1024, top 32, 8 rows (the drafter's head)."""
    w = S.WORKLOADS["drafter"]
    cl = S.make_clustered_head(w)
    h = S.make_hidden(w, w.batch, d=w.drafter_hidden)
    assert _check_clustered(h, cl, w.top_c) <= 2
    assert status_ok()


@pytest.mark.parametrize("C,cs,top_c", [(300, 3, 17), (4096, 2, 64), (8192, 1, 5), (200, 32, 7)])
def test_clustered_cluster_counts(C, cs, top_c):
    """Cluster counts that are not multiples of the selection block, up to the 8192 limit;
    cluster sizes that take the per-warp gather (not a multiple of 16) and the staged one."""
    w = S.Workload("c", 4, 0, 0, 4, 1, [], 64, C * cs, n_clusters=C, cluster_size=cs,
                   drafter_hidden=64, seed=33)
    cl = S.make_clustered_head(w)
    h = S.bf16(S.normal(7, (6, 64)))
    assert _check_clustered(h, cl, top_c) <= 1
    assert status_ok()


def test_clustered_exact_ties_go_to_lower_ids():
    """Equal scores at the selection boundary: the lower cluster ids are kept.  Centroids are
    +v for a scattered set of 100 clusters and -v elsewhere, so every row's scores take two
    bit-identical values and the kept set is the 40 lowest ids of the +v set."""
    C, cs, d, top_c = 512, 2, 64, 40
    w = S.Workload("c", 4, 0, 0, 4, 1, [], d, C * cs, n_clusters=C, cluster_size=cs,
                   drafter_hidden=d, seed=34)
    cl = S.make_clustered_head(w)
    rng = np.random.default_rng(34)
    plus = np.sort(rng.choice(C, size=100, replace=False))
    v = S.bf16(S.normal(8, (1, d)))[0]
    cent = (-v).repeat(C, 1)
    cent[torch.from_numpy(plus).long()] = v
    cl["centroids"] = cent.contiguous()
    h = v.float().repeat(3, 1)
    h[1] *= 2.0
    h = h.to(torch.bfloat16)
    _, sel = _run_clustered(h, cl, top_c)
    assert sel.tolist() == [plus[:top_c].tolist()] * 3
    assert status_ok()
