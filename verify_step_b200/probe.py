"""Times single entry-point calls on synthetic inputs of a given shape (CUDA events, inputs
rotated over more than L2 where they are large), for micro-benchmarks and profiler captures.

    python -m verify_step_b200.probe accept --batch 8 --k 2 [--vocab 262144] [--temperature 1]
    python -m verify_step_b200.probe linear --m 24 --n 43008 --kdim 5376 [--epilogue geglu]
                                            [--x f32|bf16] [--norm] [--out f32|bf16]
    python -m verify_step_b200.probe head --m 24 --d 5376 --vocab 65536
    python -m verify_step_b200.probe head --m 8 --d 1024 --clusters 1024 [--top-c 32]
    python -m verify_step_b200.probe attn --batch 2 --ctx 16384 --head-dim 512 --k 2 [--draft]

--reps 1 --warmup 1 runs the call twice (one warm-up), eagerly, for a profiler capture; more
repetitions are timed as replays of a CUDA graph holding them.  Inputs are
random (torch on the device); nothing is checked here: the tests hold the parity checks.
Prints one line per shape: microseconds per call and the weight / logit / KV stream rate.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import sys


def _events(torch):
    return torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)


def _time(torch, fn, reps, warmup):
    """Microseconds per call.  With more than one repetition the calls are captured once in a
    CUDA graph and the graph is replayed, so that host launch overhead does not set the time of
    short calls; with one (a profiler capture) they run eagerly."""
    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize()
    e0, e1 = _events(torch)
    if reps <= 1:
        e0.record()
        for i in range(reps):
            fn(warmup + i)
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / max(reps, 1) * 1e3
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(reps):
            fn(warmup + i)
    g.replay()
    torch.cuda.synchronize()
    replays = 3
    e0.record()
    for _ in range(replays):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / (replays * reps) * 1e3


def run_accept(a, torch, sd):
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    noise = json.load(open(os.path.join(root, "tests", "golden", "draft_noise.json")))
    B, k, V, T = a.batch, a.k, a.vocab, a.temperature
    g = torch.Generator(device="cuda")
    g.manual_seed(1)
    z = torch.randn((B, k + 1, V), generator=g, device="cuda")
    y = drafts = None
    if k > 0:
        sig = [noise["sigma_pos0"]] + [noise["sigma_later"]] * (k - 1)
        y = torch.stack([z[:, i] + sig[i] * torch.randn((B, V), generator=g, device="cuda")
                         for i in range(k)], 1).contiguous()
        drafts = torch.argmax(y, dim=-1).to(torch.int32).contiguous()
    desc = sd.AcceptDesc(batch=B, k=k, vocab=V, temperature=T, seed=1, step=0,
                         purpose=1 if k else 2)
    ws = torch.empty(max(256, sd.sd_accept_workspace_size(desc)), dtype=torch.uint8,
                     device="cuda")
    n_acc = torch.empty(B, dtype=torch.int32, device="cuda")
    out = torch.empty((B, k + 1), dtype=torch.int32, device="cuda")
    flags = torch.empty(B, dtype=torch.int32, device="cuda")

    def call(i):
        desc.step = i
        sd.sd_accept(desc, z, y, drafts, n_acc, out, flags, ws)

    us = _time(torch, call, a.reps, a.warmup)
    mb = (B * (k + 1) + (B * k if T > 0 else 0)) * V * 4 / 1e6
    print(f"accept B{B} k{k} V{V} T{T}: {us:.1f} us ({mb:.1f} MB of logit rows)")


def run_linear(a, torch, sd):
    m, n, k = a.m, a.n, a.kdim
    epi = {"store": sd.SD_EPI_STORE, "add": sd.SD_EPI_ADD, "geglu": sd.SD_EPI_GEGLU}[a.epilogue]
    x = torch.randn(m, k, device="cuda", dtype=torch.float32 if a.x == "f32" else torch.bfloat16)
    oc = n // 2 if epi == sd.SD_EPI_GEGLU else n
    out_f32 = a.out == "f32" and epi != sd.SD_EPI_GEGLU
    out = torch.zeros(m, oc, device="cuda", dtype=torch.float32 if out_f32 else torch.bfloat16)
    gain = torch.ones(k, device="cuda")
    desc = sd.LinearDesc(m=m, n=n, k=k, x_dtype=sd.SD_F32 if a.x == "f32" else sd.SD_BF16,
                         ld_x=k, norm_eps=1e-6, epilogue=epi,
                         out_dtype=sd.SD_F32 if out_f32 else sd.SD_BF16, ld_out=oc)
    if a.norm:
        desc.norm_gain = gain.data_ptr()
    ws = torch.empty(max(256, sd.sd_linear_workspace_size(desc)), dtype=torch.uint8,
                     device="cuda")
    copies = 1 if a.reps <= 1 else max(2, int(300e6 // (n * k * 2)) + 1)
    Ws = [(torch.randn(n, k, device="cuda") / math.sqrt(k)).to(torch.bfloat16)
          for _ in range(copies)]
    us = _time(torch, lambda i: sd.sd_linear(desc, x, Ws[i % copies], out, ws=ws), a.reps,
               a.warmup)
    print(f"linear m{m} n{n} k{k} {a.epilogue}: {us:.1f} us, "
          f"{n * k * 2 / (us * 1e3):.0f} GB/s of weights")


def run_head_clustered(a, torch, sd):
    """The clustered head: centroid scores, top-c selection, exact logits of the kept clusters
    (cluster-major weights; random cluster membership, as the benchmark's drafter head)."""
    m, d, V, C = a.m, a.d, a.vocab, a.clusters
    cs = V // C
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    h = torch.randn(m, d, device="cuda", generator=g).to(torch.bfloat16)
    w_cm = (torch.randn(C, cs, d, device="cuda", generator=g) / math.sqrt(d)).to(torch.bfloat16)
    cent = w_cm.float().mean(dim=1).to(torch.bfloat16)
    tokens = torch.randperm(V, device="cuda", generator=g).to(torch.int32).reshape(C, cs)
    out = torch.empty(m, V, device="cuda")
    sel = torch.empty(m, a.top_c, dtype=torch.int32, device="cuda")
    desc = sd.HeadDesc(m=m, d=d, vocab=V, n_clusters=C, cluster_size=cs, top_c=a.top_c,
                       dtype=sd.SD_BF16)
    ws = torch.empty(max(256, sd.sd_lm_head_workspace_size(desc)), dtype=torch.uint8,
                     device="cuda")
    us = _time(torch, lambda i: sd.sd_lm_head(desc, h, w_cm, out, centroids=cent,
                                              cluster_tokens=tokens, sel_clusters=sel, ws=ws),
               a.reps, a.warmup)
    gb = (C * d * 2 + m * a.top_c * cs * d * 2 + m * V * 4) / 1e9
    print(f"clustered head m{m} d{d} V{V} C{C} top{a.top_c}: {us:.1f} us, "
          f"{gb / (us * 1e-6):.0f} GB/s (centroids, kept clusters' weights, logit rows)")


def run_head(a, torch, sd):
    if a.clusters:
        return run_head_clustered(a, torch, sd)
    m, d, V = a.m, a.d, a.vocab
    h = torch.randn(m, d, device="cuda").to(torch.bfloat16)
    copies = 1 if a.reps <= 1 else max(2, int(300e6 // (V * d * 2)) + 1)
    Ws = [(torch.randn(V, d, device="cuda") / math.sqrt(d)).to(torch.bfloat16)
          for _ in range(copies)]
    out = torch.empty(m, V, device="cuda")
    desc = sd.HeadDesc(m=m, d=d, vocab=V, dtype=sd.SD_BF16)
    us = _time(torch, lambda i: sd.sd_lm_head(desc, h, Ws[i % copies], out), a.reps, a.warmup)
    gb = (V * d * 2 + m * d * 2 + m * V * 4) / 1e9
    print(f"head m{m} d{d} V{V}: {us:.1f} us, {gb / (us * 1e-6):.0f} GB/s")


def run_attn(a, torch, sd):
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import synthetic as S
    D, W = a.head_dim, a.window
    w = S.Workload("probe", a.batch, a.ctx, a.k, 16, 4, [S.AttnLayer(D, W)], 5376, 262144,
                   seed=3)
    L = S.contexts(w)
    c = S.make_cache(w, 0, L, reserve=8 + a.reps + a.warmup)
    s = S.make_step_qkv(w, 0, a.k + 1)
    g = lambda t: t.contiguous().to("cuda")
    desc = sd.AttnDesc(batch=a.batch, n_q=a.k + 1, h_q=16, h_kv=4, head_dim=D, block_size=16,
                       max_blocks_per_seq=c["max_blocks"], num_blocks=c["num_blocks"],
                       window=W, scale=1 / math.sqrt(D), dtype=sd.SD_BF16)
    kc, vc, tab, ctx = g(c["k_cache"]), g(c["v_cache"]), g(c["table"]), g(torch.from_numpy(L))
    q, kn, vn = g(s["q"]), g(s["k_new"]), g(s["v_new"])
    if a.draft:  # the drafter's read-only cross-attention: one query per sequence at L - 1
        desc.n_q = 1
        q = q[:, :1].contiguous()
        out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(max(256, sd.sd_draft_xattn_workspace_size(desc)), dtype=torch.uint8,
                         device="cuda")
        qpos = (ctx - 1).to(torch.int32)
        us = _time(torch, lambda i: sd.sd_draft_xattn(desc, q, kc, vc, tab, ctx, qpos, out, ws),
                   a.reps, a.warmup)
        keys = L if W == 0 else [min(int(x), W) for x in L]
    else:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(max(256, sd.sd_verify_attn_workspace_size(desc)), dtype=torch.uint8,
                         device="cuda")
        us = _time(torch, lambda i: sd.sd_verify_attn(desc, q, kn, vn, kc, vc, tab, ctx, out,
                                                      ws), a.reps, a.warmup)
        keys = (L + a.k + 1) if W == 0 else [min(int(x) + a.k + 1, W + a.k) for x in L]
    gb = sum(int(x) for x in keys) * 4 * D * 2 * 2 / 1e9
    print(f"{'xattn' if a.draft else 'attn'} B{a.batch} ctx{a.ctx} D{D} W{W} k{a.k}: "
          f"{us:.1f} us, {gb / (us * 1e-6):.0f} GB/s of K/V")


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("what", choices=["accept", "linear", "head", "attn"])
    ap.add_argument("--batch", type=int, default=8)
    ap.add_argument("--k", type=int, default=2)
    ap.add_argument("--vocab", type=int, default=262144)
    ap.add_argument("--temperature", type=float, default=1.0)
    ap.add_argument("--m", type=int, default=24)
    ap.add_argument("--n", type=int, default=8192)
    ap.add_argument("--kdim", type=int, default=5376, help="linear: columns of W")
    ap.add_argument("--d", type=int, default=5376)
    ap.add_argument("--epilogue", choices=["store", "add", "geglu"], default="store")
    ap.add_argument("--x", choices=["f32", "bf16"], default="f32")
    ap.add_argument("--out", choices=["f32", "bf16"], default="bf16")
    ap.add_argument("--norm", action="store_true")
    ap.add_argument("--ctx", type=int, default=16384)
    ap.add_argument("--head-dim", type=int, default=512)
    ap.add_argument("--window", type=int, default=0)
    ap.add_argument("--draft", action="store_true", help="attn: the drafter cross-attention")
    ap.add_argument("--clusters", type=int, default=0, help="head: clustered head with C clusters")
    ap.add_argument("--top-c", type=int, default=32)
    ap.add_argument("--reps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    a = ap.parse_args(argv)
    import torch

    import verify_step_b200 as sd
    sd.lib()
    {"accept": run_accept, "linear": run_linear, "head": run_head, "attn": run_attn}[a.what](
        a, torch, sd)
    status = sd.sd_device_status_read()
    if status != 0:
        raise SystemExit(f"device status {status}")


if __name__ == "__main__":
    main()
