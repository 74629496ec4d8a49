#!/usr/bin/env python
"""Benchmark of the speculative-decoding verify step on B200.

One step is one pass of the whole hot path for a batch of B = 8 sequences with 16384 committed
tokens and k = 2 drafts (the global-layer verify configuration at its reference point, with
the drafter's pass over the same shared cache):

  drafter chain, j = 0..k-1:   3 x sd_draft_xattn (sliding, D256, W512) + 1 x sd_draft_xattn
                               (global, D512) on the target cache, the clustered LM head
                               (1024 clusters x 256 tokens, d 1024, top 32) and the drafter's
                               own draw (sd_accept, k = 0, purpose 2)
  verify:                      sd_verify_attn on the global (D512) and sliding (D256, W512)
                               layers (k+1 = 3 positions, 16q/4kv, block 16), the dense LM head
                               (d 5376, V 262144), sd_accept (T = 1), sd_commit

The metric is verified positions per second, B * (k+1) per step, over the whole job.
Inputs are synthetic and resident in HBM; every step reads ~6 GB, far more than the 126 MB L2,
so no L2 flush is needed between steps.  Contexts grow by the accepted length each step.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--k K] [--batch B] [--ctx L]   (other points of the workload range)

N > 1 (under torch.distributed.run): independent replicas, one batch per GPU, no collective
on the data path (weak scaling); time = max over ranks.
--impl reference times the CPU oracle (float64, host cores) on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "spec_step_b8_ctx16384_k2"  # the default configuration


def workload_name(batch, ctx, k, drafter_layers=False, target_layers=False):
    return (f"spec_step_b{batch}_ctx{ctx}_k{k}" + ("_drafter_layers" if drafter_layers else "") +
            ("_target_layers" if target_layers else ""))
METRIC = "verified tokens/s per verify step (B,k,ctx); HBM GB/s as % of B200 peak"
UNIT = "verified tokens/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--k", type=int, default=2)
    ap.add_argument("--batch", type=int, default=8)
    ap.add_argument("--ctx", type=int, default=16384)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--drafter-layers", action="store_true",
                    help="run the drafter's dense layers (input projection, 4 x (W_q, W_o, "
                         "gated MLP, W_d), output projection) around its cross-attention, so "
                         "the chain is driven by the committed hidden row and tokens")
    ap.add_argument("--target-layers", action="store_true",
                    help="verify through two target layers with their own projections (a "
                         "sliding and a global layer: q/k/v/o and a gated MLP 21504 wide at "
                         "d 5376) instead of the two attention calls on given q, k, v")
    return ap.parse_args()


# kernel group -> the CUDA source whose ncu counters a committed profile summary holds
GROUP_SOURCE = {"head_dense": "lm_head.cu", "head_clustered": "lm_head.cu",
                "verify_global": "attention.cu", "verify_sliding": "attention.cu",
                "xattn_global": "attention.cu", "xattn_sliding": "attention.cu",
                "accept": "accept.cu", "accept_draft": "accept.cu", "commit": "commit.cu",
                "drafter_dense": "linear.cu", "target_dense": "linear.cu"}


def source_hash(name):
    import hashlib
    h = hashlib.sha256()
    for f in (name, "common.cuh", "philox.cuh"):
        path = os.path.join(ROOT, "verify_step_b200", "csrc", f)
        if os.path.exists(path):
            h.update(open(path, "rb").read())
    return h.hexdigest()[:16]


def dram_traffic(group, workload=WORKLOAD):
    """DRAM bytes per launch of a kernel group from the committed ncu summary, or None when
    the summary is missing or the kernel source changed since its counters were taken."""
    path = os.path.join(ROOT, "profiles", "dram_traffic_%s.json" % workload)
    try:
        d = json.load(open(path))
        e = d["groups"][group]
        if e["source_sha"] != source_hash(GROUP_SOURCE[group]):
            return None
        return int(e["dram_bytes_per_launch"])
    except Exception:
        return None


def rank_seed(rank):
    """Seed of a rank's synthetic inputs: every rank verifies its own batch of sequences."""
    return 100 + 7 * rank


def max_over_ranks(x, world, device):
    """A per-rank time maximised over the ranks (the identity at one rank)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world, batch, n_q, steps, ms):
    """Verified tokens per second of the whole job: each of the world ranks verifies batch x n_q
    tokens per step, all within ms (the slowest rank's time)."""
    return world * batch * n_q * steps / (ms / 1e3)


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


# --------------------------------------------------------------------------------- workload

class SpecStep:
    """Device buffers, descriptors and the call sequence of one speculative step."""

    def __init__(self, k=2, B=8, L=16384, reserve=600, rank=0, dev="cuda", dense=False,
                 target=False):
        import numpy as np
        import torch

        import synthetic as S
        import verify_step_b200 as sd
        self.sd, self.np, self.torch = sd, np, torch
        self.k, self.B, self.n_q = k, B, k + 1
        self.dev = dev
        self.dense = dense
        self.target = target
        self.hq, self.hkv, self.bs = 16, 4, 16
        self.V, self.d, self.dh = 262144, 5376, 1024
        self.C, self.cs, self.top_c = 1024, 256, 32
        seed = rank_seed(rank)
        wg = S.Workload("g", B, L, k, 16, 4, [S.AttnLayer(512), S.AttnLayer(256, 512)],
                        self.d, self.V, seed=seed, n_clusters=self.C, cluster_size=self.cs,
                        drafter_hidden=self.dh, top_c=self.top_c)
        self.w = wg
        self.L0 = S.contexts(wg)
        self.host = {}
        g = lambda t: t.contiguous().to(dev)
        mb = int((self.L0.max() + reserve + self.bs - 1) // self.bs)
        # target cache: layer 0 global D512, layer 1 sliding D256 W512
        self.cache = []
        for layer in (0, 1):
            c = S.make_cache(wg, layer, self.L0, reserve=reserve, max_blocks=mb)
            self.host[f"cache{layer}"] = c
            self.cache.append(dict(k=g(c["k_cache"]), v=g(c["v_cache"]), table=g(c["table"]),
                                   nb=c["num_blocks"], mb=c["max_blocks"]))
        self.ctx = g(torch.from_numpy(self.L0))
        self.ctx0 = self.ctx.clone()
        # per-step inputs (reused every step; copied from pinned host memory in the e2e leg)
        inp = {}
        for layer in ((0, 1) if not target else ()):
            s = S.make_step_qkv(wg, layer, self.n_q)
            inp[f"q{layer}"], inp[f"kn{layer}"], inp[f"vn{layer}"] = s["q"], s["k_new"], s["v_new"]
        if target:
            # input rows of the k+1 positions (the residual stream entering the first layer)
            inp["x0"] = torch.from_numpy(S.normal(seed * 41 + 5, (B * self.n_q, self.d)))
        inp["hidden"] = S.make_hidden(wg, B * self.n_q)
        for j in range(0 if dense else k):
            for layer, D in ((0, 512), (1, 256)):
                n = 1 if layer == 0 else 3
                inp[f"dq{j}_{layer}"] = S.bf16(S.normal(seed * 31 + 10 * j + layer,
                                                        (n, B, 1, self.hq, D), 1 / math.sqrt(D)))
            inp[f"dh{j}"] = S.bf16(S.normal(seed * 37 + j, (B, self.dh)))
        self.host_inputs = inp
        # all per-step inputs live in one device buffer (256-byte aligned views) ordered by
        # the phase that first reads them (drafter step 0, drafter step 1, ..., verify), so the
        # end-to-end leg moves each phase's inputs with one host-to-device copy
        phases = [[] if dense else [f"dq{j}_0", f"dq{j}_1", f"dh{j}"] for j in range(k)]
        phases.append([kk for kk in inp if not kk.startswith("dq") and not kk.startswith("dh")])
        offs, total, self.phase_ranges = {}, 0, []
        for keys in phases:
            start = total
            for kk in keys:
                v = inp[kk]
                offs[kk] = total
                total += (v.numel() * v.element_size() + 255) // 256 * 256
            self.phase_ranges.append((start, total))
        self.input_buf = torch.empty(total, dtype=torch.uint8, device=dev)
        self.input_offs = offs
        self.inputs = {}
        for kk, v in inp.items():
            n = v.numel() * v.element_size()
            view = self.input_buf[offs[kk]:offs[kk] + n].view(v.dtype).view(v.shape)
            view.copy_(v.contiguous().to(dev))
            self.inputs[kk] = view
        self.W = g(S.make_lm_head(wg))
        self.host["W"] = None  # regenerated on demand for the CPU baseline
        cl = S.make_clustered_head(wg)
        self.host["cl"] = cl
        self.cl = {kk: g(v) for kk, v in cl.items()}
        # outputs and scratch
        f32, i32 = torch.float32, torch.int32
        self.attn_out = [torch.empty((B, self.n_q, self.hq, D), dtype=torch.bfloat16, device=dev)
                         for D in (512, 256)]
        self.xout = [torch.empty((B, 1, self.hq, D), dtype=torch.bfloat16, device=dev)
                     for D in (512, 256)]
        self.draft_logits = torch.empty((B, k, self.V), dtype=f32, device=dev)
        self.target_logits = torch.empty((B * self.n_q, self.V), dtype=f32, device=dev)
        self.sel = torch.empty((B, self.top_c), dtype=i32, device=dev)
        self.drafts = torch.zeros((B, k), dtype=i32, device=dev)
        # the step's results, read back to the host as one block: n_accepted then out_tokens
        self.results = torch.zeros(B * (1 + self.n_q), dtype=i32, device=dev)
        self.n_acc = self.results[:B]
        self.out_tokens = self.results[B:].view(B, self.n_q)
        self.margin = torch.zeros(B, dtype=i32, device=dev)
        self.dtok = torch.zeros((B, 1), dtype=i32, device=dev)
        self.slots = torch.zeros((B, self.n_q), dtype=i32, device=dev)
        self.next_hidden = g(S.make_hidden(wg, B, step=97))
        if dense:
            # the drafter's dense layers: link 0 reads the committed hidden row and the last
            # emitted token of the previous step, link j > 0 the back projection of link j-1
            # and draft j-1
            from verify_step_b200 import drafter as VD
            self.VD = VD
            self.dshape = VD.DrafterShape(batch=B, d=self.dh, d_target=self.d,
                                          ff=S.DRAFTER_FF, h_q=self.hq,
                                          head_dims=(256, 256, 256, 512), vocab=self.V)
            self.dwts = VD.device_weights(S.make_drafter_weights(
                seed, self.dh, self.d, self.V, self.hq, self.dshape.head_dims), dev)
            self.dbuf = VD.buffers(self.dshape, dev)
        if target:
            # two target layers over the bench's caches: the sliding one, then the global one
            from verify_step_b200 import target as VT
            self.VT = VT
            self.tshape = VT.TargetShape(batch=B, n_q=self.n_q, d=self.d, ff=4 * self.d,
                                         h_q=self.hq, h_kv=self.hkv,
                                         layers=((256, 512), (512, 0)))
            self.twts = VT.device_weights(S.make_target_weights(
                seed, self.d, 4 * self.d, self.hq, self.hkv, self.tshape.layers), dev)
            self.tbuf = VT.buffers(self.tshape, dev)
        # descriptors
        self.vdesc = [self._adesc(0, self.n_q), self._adesc(1, self.n_q)]
        self.xdesc = [[self._adesc(layer, 1, q_offset=j) for layer in (0, 1)] for j in range(k)]
        self.hdesc_dense = sd.HeadDesc(m=B * self.n_q, d=self.d, vocab=self.V, dtype=sd.SD_BF16)
        self.hdesc_cl = sd.HeadDesc(m=B, d=self.dh, vocab=self.V, ld_logits=k * self.V,
                                    n_clusters=self.C, cluster_size=self.cs, top_c=self.top_c,
                                    dtype=sd.SD_BF16)
        # step counter on the device: the acceptance draws of step s use counter value s (the
        # drafter's chain step j adds (j+1) << 28 to keep its uniforms apart); sd_commit
        # advances it, so a step captured once in a CUDA graph draws fresh numbers each replay
        self.step_dev = torch.zeros(1, dtype=torch.int64, device=dev)
        sp = self.step_dev.data_ptr()
        self.adesc_draft = [sd.AcceptDesc(batch=B, k=0, vocab=self.V, temperature=1.0, seed=7,
                                          step=(j + 1) << 28, purpose=2, ld_target=k * self.V,
                                          ld_out=k, step_ptr=sp)
                            for j in range(k)]
        self.adesc = sd.AcceptDesc(batch=B, k=k, vocab=self.V, temperature=1.0, seed=7, step=0,
                                   purpose=1, step_ptr=sp)
        self.cdesc = sd.CommitDesc(batch=B, k=k, block_size=self.bs,
                                   max_blocks_per_seq=self.cache[0]["mb"],
                                   num_blocks=self.cache[0]["nb"], d=self.d,
                                   hidden_dtype=sd.SD_BF16, step_ptr=sp)
        wsz = max([sd.sd_verify_attn_workspace_size(x) for x in self.vdesc] +
                  [sd.sd_draft_xattn_workspace_size(x) for row in self.xdesc for x in row] +
                  [sd.sd_lm_head_workspace_size(self.hdesc_cl),
                   sd.sd_accept_workspace_size(self.adesc)] +
                  [sd.sd_accept_workspace_size(x) for x in self.adesc_draft])
        self.ws = torch.empty(wsz, dtype=torch.uint8, device=dev)
        torch.cuda.synchronize()

    def _adesc(self, layer, n_q, q_offset=0):
        D, W = (512, 0) if layer == 0 else (256, 512)
        c = self.cache[layer]
        return self.sd.AttnDesc(batch=self.B, n_q=n_q, h_q=self.hq, h_kv=self.hkv, head_dim=D,
                                block_size=self.bs, max_blocks_per_seq=c["mb"],
                                num_blocks=c["nb"], window=W, scale=1 / math.sqrt(D),
                                dtype=self.sd.SD_BF16, q_offset=q_offset)

    # kernels launched per call (bf16 paths)
    # kernels per call of each group on this workload (the step graph's kernel nodes are
    # counted directly where the CUDA runtime allows; this is the fallback)
    LAUNCHES = dict(xattn_sliding=1, xattn_global=2, verify_sliding=1, verify_global=3,
                    head_dense=1, head_clustered=3, accept_draft=1, accept=2, commit=1,
                    drafter_dense=1, target_dense=1)

    def launches_per_step(self):
        L = self.LAUNCHES
        dense = self.VD.LAUNCHES_PER_LINK * L["drafter_dense"] if self.dense else 0
        return (self.k * (3 * L["xattn_sliding"] + L["xattn_global"] + L["head_clustered"] +
                          L["accept_draft"] + dense) +
                (2 * self.VT.LINEAR_CALLS_PER_LAYER * L["target_dense"] if self.target else 0) +
                L["verify_global"] + L["verify_sliding"] + L["head_dense"] + L["accept"] +
                L["commit"])

    def run(self, ev=None, before_phase=None):
        """Issue one step on the current stream.  ev (used while capturing a CUDA graph) maps a
        kernel group to a list that receives (start, end) events recorded as graph nodes
        around each call of that group.  before_phase(j) is called before drafter step j
        (j < k) and before the verify (j = k)."""
        sd, I = self.sd, self.inputs

        def timed(name, fn):
            if ev is None or name not in ev:
                fn()
                return
            a, b = new_event(), new_event()
            record_external(a)
            fn()
            record_external(b)
            ev[name].append((a, b))

        c0, c1 = self.cache
        for j in range(self.k):
            if before_phase is not None:
                before_phase(j)
            xd0, xd1 = self.xdesc[j]
            if self.dense:
                self._dense_link(j, timed)
            else:
                for r in range(3):
                    timed("xattn_sliding", lambda: sd.sd_draft_xattn(
                        xd1, I[f"dq{j}_1"][r], c1["k"], c1["v"], c1["table"], self.ctx, None,
                        self.xout[1], self.ws))
                timed("xattn_global", lambda: sd.sd_draft_xattn(
                    xd0, I[f"dq{j}_0"][0], c0["k"], c0["v"], c0["table"], self.ctx, None,
                    self.xout[0], self.ws))
            timed("head_clustered", lambda: self._clustered(j))
            ad = self.adesc_draft[j]
            timed("accept_draft", lambda: sd.sd_accept(
                ad, self._row_ptr(self.draft_logits, j), None, None, self.n_acc,
                self._col_ptr(self.drafts, j), None, self.ws))
        if before_phase is not None:
            before_phase(self.k)
        if self.target:
            self._target_layers(timed)
        else:
            timed("verify_global", lambda: sd.sd_verify_attn(
                self.vdesc[0], I["q0"], I["kn0"], I["vn0"], c0["k"], c0["v"], c0["table"],
                self.ctx, self.attn_out[0], self.ws))
            timed("verify_sliding", lambda: sd.sd_verify_attn(
                self.vdesc[1], I["q1"], I["kn1"], I["vn1"], c1["k"], c1["v"], c1["table"],
                self.ctx, self.attn_out[1], self.ws))
        timed("head_dense", lambda: sd.sd_lm_head(self.hdesc_dense, I["hidden"], self.W,
                                                  self.target_logits))
        timed("accept", lambda: sd.sd_accept(self.adesc, self.target_logits, self.draft_logits,
                                             self.drafts, self.n_acc, self.out_tokens,
                                             self.margin, self.ws))
        timed("commit", lambda: sd.sd_commit(self.cdesc, c0["table"], self.ctx, self.n_acc,
                                             self.slots, I["hidden"], self.next_hidden))

    def _dense_link(self, j, timed):
        sd = self.sd
        c0, c1 = self.cache
        xd0, xd1 = self.xdesc[j]

        def attend(i, q, o):
            if i < 3:  # sliding layers first, the global layer last
                timed("xattn_sliding", lambda: sd.sd_draft_xattn(
                    xd1, q, c1["k"], c1["v"], c1["table"], self.ctx, None, o, self.ws))
            else:
                timed("xattn_global", lambda: sd.sd_draft_xattn(
                    xd0, q, c0["k"], c0["v"], c0["table"], self.ctx, None, o, self.ws))

        if j == 0:
            h_prev, toks, ld, sel = self.next_hidden, self.out_tokens, self.n_q, self.n_acc
        else:
            h_prev, toks, ld, sel = self.dbuf["h_back"], self._col_ptr(self.drafts, j - 1), \
                self.k, None
        self.VD.link(self.dshape, self.dwts, self.dbuf, h_prev, toks, ld, attend,
                     token_sel=sel, wrap=lambda fn: timed("drafter_dense", fn))

    def _target_layers(self, timed):
        c0, c1 = self.cache
        caches = [dict(desc=self.vdesc[1], k=c1["k"], v=c1["v"], table=c1["table"]),
                  dict(desc=self.vdesc[0], k=c0["k"], v=c0["v"], table=c0["table"])]
        self.tbuf["x"].copy_(self.inputs["x0"])
        names = iter(["verify_sliding", "verify_global"])

        def wrap(kind, fn):
            timed(next(names) if kind == "attn" else "target_dense", fn)

        self.VT.verify_layers(self.tshape, self.twts, self.tbuf, caches, self.ctx, self.ws,
                              wrap=wrap)

    def _row_ptr(self, t, j):
        return t.data_ptr() + j * self.V * t.element_size()

    def _col_ptr(self, t, j):
        return t.data_ptr() + j * t.element_size()

    def _clustered(self, j):
        # logits of draft step j go to row b*k + j of draft_logits (ld_logits = k * V)
        hidden = self.dbuf["h"] if self.dense else self.inputs[f"dh{j}"]
        self.sd.sd_lm_head(self.hdesc_cl, hidden, self.cl["w_cm"],
                           self._row_ptr(self.draft_logits, j),
                           centroids=self.cl["centroids"],
                           cluster_tokens=self.cl["cluster_tokens"], sel_clusters=self.sel,
                           ws=self.ws)

    # --------------------------------------------------------------- algorithmic bytes
    def bytes_per_call(self, L):
        """Algorithmic HBM bytes of one call of each kernel group at committed lengths L."""
        np = self.np
        B, hkv, n_q, hq = self.B, self.hkv, self.n_q, self.hq
        L = np.asarray(L, np.int64)
        out = {}
        # verify: K and V of every key read once per (sequence, kv head), new rows written,
        # queries read, outputs written
        for name, D, W in (("verify_global", 512, 0), ("verify_sliding", 256, 512)):
            keys = (L + n_q) if W == 0 else np.minimum(L + n_q, W + n_q - 1)
            out[name] = int(keys.sum() * hkv * D * 2 * 2 + B * n_q * hkv * D * 2 * 2 * 2 +
                            2 * B * n_q * hq * D * 2)
        for name, D, W in (("xattn_global", 512, 0), ("xattn_sliding", 256, 512)):
            # chain step j queries position L + j: the committed keys in its window
            keys = L if W == 0 else np.mean([np.minimum(L, W - 1 - j) for j in range(self.k)],
                                            axis=0)
            out[name] = int(keys.sum() * hkv * D * 2 * 2 + 2 * B * hq * D * 2)
        out["head_dense"] = int(self.V * self.d * 2 + B * n_q * self.d * 2 +
                                B * n_q * self.V * 4)
        out["head_clustered"] = int(self.C * self.dh * 2 + B * self.dh * 2 +
                                    B * self.top_c * self.cs * self.dh * 2 + B * self.V * 4)
        out["accept"] = int((B * n_q + B * self.k) * self.V * 4)
        out["accept_draft"] = int(B * self.V * 4)
        out["commit"] = int(B * (n_q * 4 * 2 + self.d * 2 * 2))
        if self.dense:
            out["drafter_dense"] = int(self.VD.hbm_bytes_per_link(self.dshape) /
                                       self.VD.LAUNCHES_PER_LINK)
        if self.target:
            out["target_dense"] = int(self._target_dense_bytes() /
                                      (2 * self.VT.LINEAR_CALLS_PER_LAYER))
        return out

    def _target_dense_bytes(self):
        """Algorithmic HBM bytes of the target layers' projections per step: every weight
        once, the input rows read and the outputs written (the residual read and written)."""
        t = self.tshape
        m, d, F = t.batch * t.n_q, t.d, t.ff
        total = 0
        for D, _ in t.layers:
            nq, nkv = t.h_q * D, t.h_kv * D
            total += (nq + 2 * nkv) * d * 2 + 3 * m * d * 4 + m * (nq + 2 * nkv) * 2
            total += d * nq * 2 + m * nq * 2 + 2 * m * d * 4
            total += 2 * F * d * 2 + m * d * 4 + m * F * 2
            total += d * F * 2 + m * F * 2 + 2 * m * d * 4
        return total

    def calls_per_step(self):
        out = dict(xattn_sliding=3 * self.k, xattn_global=self.k, head_clustered=self.k,
                   accept_draft=self.k, verify_global=1, verify_sliding=1, head_dense=1,
                   accept=1, commit=1)
        if self.dense:
            out["drafter_dense"] = self.VD.LAUNCHES_PER_LINK * self.k
        if self.target:
            out["target_dense"] = 2 * self.VT.LINEAR_CALLS_PER_LAYER
        return out

    def reset(self):
        self.ctx.copy_(self.ctx0)

    def capture(self, ev=None):
        torch = self.torch
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.run(ev)
        return g

    def capture_e2e(self, pinned, res_h):
        """The step with its host transfers as graph nodes: the first drafter step's inputs
        are copied on the step's stream before it starts; the later phases' inputs are copied
        on a second stream meanwhile, each phase waiting only for its own block; the results
        are copied back to pinned host memory at the end."""
        torch = self.torch
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        with torch.cuda.graph(g):
            cur = torch.cuda.current_stream()
            s0, e0 = self.phase_ranges[0]
            self.input_buf[s0:e0].copy_(pinned[s0:e0], non_blocking=True)
            fork = torch.cuda.Event()
            fork.record(cur)
            side.wait_event(fork)
            ready = []
            with torch.cuda.stream(side):
                for s, e in self.phase_ranges[1:]:
                    self.input_buf[s:e].copy_(pinned[s:e], non_blocking=True)
                    ev = torch.cuda.Event()
                    ev.record(side)
                    ready.append(ev)

            def before_phase(j):
                if j >= 1:
                    cur.wait_event(ready[j - 1])

            self.run(before_phase=before_phase)
            res_h.copy_(self.results, non_blocking=True)
        return g


def new_event():
    """A timing event whose CUDA handle exists (torch creates it lazily on first record)."""
    import torch
    e = torch.cuda.Event(enable_timing=True)
    e.record()
    return e


def graph_kernel_nodes(graph):
    """Kernel nodes in a captured torch CUDA graph (None if the runtime cannot say)."""
    try:
        from cuda.bindings import runtime as cudart
        g = cudart.cudaGraph_t(graph.raw_cuda_graph())
        err, _, n = cudart.cudaGraphGetNodes(g, 0)
        if err != cudart.cudaError_t.cudaSuccess:
            return None
        err, nodes, n = cudart.cudaGraphGetNodes(g, n)
        if err != cudart.cudaError_t.cudaSuccess:
            return None
        kinds = [cudart.cudaGraphNodeGetType(nd) for nd in nodes]
        return sum(1 for e, t in kinds if e == cudart.cudaError_t.cudaSuccess and
                   t == cudart.cudaGraphNodeType.cudaGraphNodeTypeKernel)
    except Exception:
        return None


def record_external(ev):
    """Record ``ev`` on the current stream as an event node of the graph being captured
    (cudaEventRecordExternal), so every replay re-records it."""
    import torch
    from cuda.bindings import runtime as cudart
    err, = cudart.cudaEventRecordWithFlags(
        cudart.cudaEvent_t(ev.cuda_event),
        cudart.cudaStream_t(torch.cuda.current_stream().cuda_stream),
        cudart.cudaEventRecordExternal)
    if err != cudart.cudaError_t.cudaSuccess:
        raise RuntimeError(f"cudaEventRecordWithFlags: {err}")


# --------------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, dev_index):
        self.proc = None
        self.err = None
        try:
            import torch
            props = torch.cuda.get_device_properties(dev_index)
            bus = getattr(props, "pci_bus_id", None)
            dom = getattr(props, "pci_domain_id", 0)
            dvc = getattr(props, "pci_device_id", 0)
            sel = ["-i", "%08X:%02X:%02X.0" % (dom, bus, dvc)] if bus is not None else []
            self.cmd = ["nvidia-smi", *sel, "--query-gpu=timestamp," + self.FIELDS,
                        "--format=csv,noheader,nounits", "-lms", "20"]
            self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE,
                                         stderr=subprocess.PIPE, text=True)
        except Exception as e:  # no nvidia-smi: report why
            self.err = repr(e)

    def stop(self):
        if self.proc is None:
            return {"error": self.err}
        self.proc.terminate()
        try:
            out, errout = self.proc.communicate(timeout=10)
        except Exception:
            self.proc.kill()
            return {"error": "nvidia-smi did not stop"}
        rows = []
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]),
                                 power=float(parts[3]) if parts[3] not in ("[N/A]", "") else 0.0,
                                 active=parts[4], hw=parts[5], hwt=parts[6], swt=parts[7],
                                 pcap=parts[8]))
            except ValueError:
                continue
        if not rows:
            return {"error": "no samples", "cmd": " ".join(self.cmd),
                    "stdout": out.strip().splitlines()[:3], "stderr": errout.strip()[:300]}
        load = [r for r in rows if r["power"] > 300] or rows
        reasons = set()
        for r in load:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in load),
                "sm_max_mhz": max(r["smax"] for r in rows), "reasons": sorted(reasons),
                "samples": len(load), "power_w_max": max(r["power"] for r in rows),
                "window": "warm-up, timed, per-kernel and end-to-end passes (samples above "
                          "300 W taken as under load)"}


# --------------------------------------------------------------------------------- oracle

def oracle_sample(step_obj, seqs, s):
    """The CPU oracle on sequences ``seqs`` of the batch: the full step for them (drafter
    chain, verify on both layers, dense LM head over the full vocabulary, acceptance,
    commit).  Returns the number of verified positions."""
    import numpy as np
    import torch

    import synthetic as S
    from oracle import accept as OACC
    from oracle import attention as OA
    from oracle import commit as OC
    from oracle import lm_head as OH

    class F64:
        def __init__(self, t):
            self.t = t
            self.shape = tuple(t.shape)

        def __getitem__(self, idx):
            idx = idx if isinstance(idx, tuple) else (idx,)
            idx = tuple(torch.as_tensor(np.asarray(i, np.int64)) if isinstance(i, np.ndarray)
                        else i for i in idx)
            return self.t[idx].to(torch.float64).numpy()

    from oracle import drafter as OD
    from oracle import target as OT

    st = step_obj
    dense, target = getattr(st, "dense", False), getattr(st, "target", False)
    if st.host.get("W") is None:
        st.host["W"] = S.make_lm_head(st.w)
    k, n_q, B = st.k, st.n_q, st.B
    hi = st.host_inputs
    f = lambda t: t.to(torch.float64).numpy()
    L = st.L0.copy()
    c0, c1 = st.host["cache0"], st.host["cache1"]
    cl = st.host["cl"]
    seqs = list(seqs)
    m = len(seqs)
    drafts = np.zeros((m, k), np.int64)
    draft_logits = np.zeros((m, k, st.V))
    ocache = {D: dict(k=F64(c["k_cache"]), v=F64(c["v_cache"]), table=c["table"].numpy()[seqs],
                      block_size=st.bs) for D, c in ((512, c0), (256, c1))}
    if dense:
        h_prev = f(st.host["h0"])[seqs]
        tokens = np.zeros(m, np.int64)
    for j in range(k):
        if dense:
            # the drafter's dense layers around its four cross-attentions (sequences seqs)
            atts = [OD.cross_attend(ocache[D], st.hq, D, 512 if D == 256 else 0, L[seqs], j)
                    for D in (256, 256, 256, 512)]
            link = OD.drafter_step(h_prev, tokens, st.host["drafter"], atts)
            hj, h_prev = link["h"], link["h_back"]
        else:
            for layer, cache, D, W, n in ((1, c1, 256, 512, 3), (0, c0, 512, 0, 1)):
                q = f(hi[f"dq{j}_{layer}"])
                for r in range(n):
                    for b in seqs:
                        for h in range(st.hq):
                            OA.draft_attention_one(b, h, q[r], F64(cache["k_cache"]),
                                                   F64(cache["v_cache"]),
                                                   cache["table"].numpy(), L, L + j, W,
                                                   1 / math.sqrt(D), st.bs)
            hj = f(hi[f"dh{j}"])[seqs]
        lg, _, _ = OH.clustered_lm_head(hj, f(cl["centroids"]),
                                        F64(cl["w_cm"]), cl["cluster_tokens"].numpy(), st.top_c)
        draft_logits[:, j] = lg
        r = OACC.accept(lg[:, None, :], None, np.zeros((m, 0)), 1.0, seed=7,
                        step=((j + 1) << 28) + s, purpose=OACC.PURPOSE_DRAFTER)
        drafts[:, j] = r["out_tokens"][:, 0]
        tokens = drafts[:, j]
    rows = np.concatenate([np.arange(b * n_q, (b + 1) * n_q) for b in seqs])
    if target:
        # the target's two layers with their own projections (sliding, then global)
        OT.verify_layers(f(hi["x0"])[rows], st.host["target"], [ocache[256], ocache[512]],
                         L[seqs], n_q, st.hq, st.hkv)
    else:
        for layer, cache, D, W in ((0, c0, 512, 0), (1, c1, 256, 512)):
            q, kn, vn = f(hi[f"q{layer}"]), f(hi[f"kn{layer}"]), f(hi[f"vn{layer}"])
            for b in seqs:
                for j in range(n_q):
                    for h in range(st.hq):
                        OA.verify_attention_one(b, j, h, q, kn, vn, F64(cache["k_cache"]),
                                                F64(cache["v_cache"]), cache["table"].numpy(),
                                                L, W, 1 / math.sqrt(D), st.bs)
    h = f(hi["hidden"])[rows]
    Wv = F64(st.host["W"])
    z = np.empty((len(rows), st.V))
    chunk = 16384
    for v0 in range(0, st.V, chunk):
        z[:, v0:v0 + chunk] = OH.lm_head(h, Wv, np.arange(v0, min(st.V, v0 + chunk)))
    z = z.astype(np.float32).astype(np.float64).reshape(m, n_q, st.V)
    r = OACC.accept(z, draft_logits, drafts, 1.0, seed=7, step=s)
    OC.commit(L[seqs], r["n_accepted"], c0["table"].numpy()[seqs], st.bs, n_q,
              f(hi["hidden"]).reshape(B, n_q, -1)[seqs])
    return m * n_q


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


# --------------------------------------------------------------------------------- main

def main():
    a = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if a.impl == "reference":
        return run_reference(a, rank, world)

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    from verify_step_b200 import build as B
    if rank == 0 or world == 1:
        B.build()
    if world > 1:
        dist.barrier()
    import verify_step_b200 as sd
    sd.lib()

    # every pass below runs a.steps steps (warm-up, timed, per-kernel, e2e): reserve the blocks
    reserve = (a.warmup + 4 * a.steps + 8) * (a.k + 1) + 64
    st = SpecStep(k=a.k, B=a.batch, L=a.ctx, reserve=reserve, rank=rank,
                  dense=a.drafter_layers, target=a.target_layers)
    wname = workload_name(st.B, a.ctx, st.k, a.drafter_layers, a.target_layers)
    L_start = st.L0.copy()
    clock = ClockSampler(local)
    for _ in range(a.warmup):
        st.run()
    torch.cuda.synchronize()
    sd.sd_device_status_clear()
    graph = st.capture()
    kernels_per_step = graph_kernel_nodes(graph)
    if kernels_per_step is None:
        kernels_per_step = st.launches_per_step()
    graph.replay()
    torch.cuda.synchronize()
    ctx_a = st.ctx.cpu().numpy()

    # ---- timed region: exactly K steps, one graph replay each
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(a.steps):
        graph.replay()
    t1.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ctx_b = st.ctx.cpu().numpy()
    ms = max_over_ranks(t0.elapsed_time(t1), world, "cuda")
    ms_step = ms / a.steps
    value = whole_job_rate(world, st.B, st.n_q, a.steps, ms)

    # ---- per-kernel device times: the same step captured with event nodes around each call,
    # replayed K times (synchronised per replay to read the events)
    groups = list(st.calls_per_step())
    ev = {g: [] for g in groups}
    graph_ev = st.capture(ev)
    sums = {g: 0.0 for g in groups}
    ctx_c = st.ctx.cpu().numpy()
    for _ in range(a.steps):
        graph_ev.replay()
        torch.cuda.synchronize()
        for g in groups:
            sums[g] += sum(x.elapsed_time(y) for x, y in ev[g])
    ctx_d = st.ctx.cpu().numpy()
    kern_ms = {g: sums[g] / (a.steps * len(ev[g])) if ev[g] else 0.0 for g in groups}
    nbytes = st.bytes_per_call((ctx_c + ctx_d) / 2.0)
    hbm, tfl, src = peaks()
    cps = st.calls_per_step()
    per_kernel = {g: {"ms": round(kern_ms[g], 4), "calls_per_step": cps[g],
                      "bytes_per_call": nbytes[g],
                      "GBps": round(nbytes[g] / (kern_ms[g] * 1e6), 1) if kern_ms[g] else None,
                      "frac_hbm": round(nbytes[g] / (kern_ms[g] * 1e6) / hbm, 3)
                      if kern_ms[g] else None}
                  for g in groups}
    busy_ms = sum(kern_ms[g] * cps[g] for g in groups)
    dom = max(groups, key=lambda g: kern_ms[g] * cps[g])

    def roof(g):
        ach = nbytes[g] / (kern_ms[g] * 1e6)
        return {"kernel": g, "bound": "hbm", "achieved": round(ach, 1), "peak": hbm,
                "unit": "GB/s", "frac": round(ach / hbm, 4),
                "traffic": dram_traffic(g, wname),
                "peak_source": src, "bytes_per_launch": nbytes[g],
                "ms_per_launch": round(kern_ms[g], 4)}
    # telemetry of the acceptance rule on these (random) weights
    mean_acc = float(((ctx_b - ctx_a) - a.steps).sum()) / max(1, a.steps * st.B)

    # ---- end-to-end: every step copies its inputs from pinned host memory, replays the step
    # and reads the accepted counts and tokens back to the host
    e2e = None
    graph_e2e = None
    if not a.no_e2e:
        pinned = torch.empty(st.input_buf.numel(), dtype=torch.uint8).pin_memory()
        for kk, v in st.host_inputs.items():
            n = v.numel() * v.element_size()
            pinned[st.input_offs[kk]:st.input_offs[kk] + n].view(v.dtype).copy_(
                v.contiguous().view(-1))
        res_h = torch.empty(st.results.numel(), dtype=torch.int32).pin_memory()
        h2d = sum(v.numel() * v.element_size() for v in st.host_inputs.values())
        d2h = res_h.numel() * 4
        if world > 1:
            dist.barrier()
        graph_e2e = st.capture_e2e(pinned, res_h)
        graph_e2e.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(a.steps):
            graph_e2e.replay()
            torch.cuda.current_stream().synchronize()
        e1.record()
        torch.cuda.synchronize()
        ems = max_over_ranks(e0.elapsed_time(e1), world, "cuda")
        e2e = {"value": round(whole_job_rate(world, st.B, st.n_q, a.steps, ems), 1), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": round(ems / a.steps, 4),
               "path": "public C ABI calls and the step's host transfers captured once in a "
                       "CUDA graph; per step: H2D of the step inputs from pinned memory in one "
                       "block per phase (drafter step 0 first; drafter step 1 and the verify "
                       "inputs on a second stream while the drafter runs), the kernels, one "
                       "D2H of n_accepted and out_tokens, stream synchronise"}
    clocks = clock.stop()
    status = sd.sd_device_status_read()
    del graph, graph_ev, graph_e2e

    cpu = None
    if (rank == 0 and world == 1 and not a.no_cpu_baseline and not a.drafter_layers and
            not a.target_layers):
        t = time.perf_counter()
        nv = oracle_sample(st, [0], 0)
        dt = time.perf_counter() - t
        cpu = {"value": round(nv / dt, 4), "unit": UNIT, "cores": blas_threads(),
               "kind": "oracle",
               "sample": "sequence 0 of the batch: full step (drafter chain, verify on both "
                         "layers, dense LM head over all 262144 tokens, acceptance, commit) "
                         "in float64 on the host; %.1f s for %d verified positions" % (dt, nv)}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": wname, "batch": st.B, "ctx": a.ctx,
                   "k": st.k,
                   "heads": "16q/4kv", "layers": "global D512 + sliding D256 W512",
                   "lm_head": "d5376 x V262144", "drafter": "2-step chain, 4 cross-attn "
                   "layers, clustered head 1024x256 top-32 d1024", "block_size": 16,
                   "parallelism": "replicas" if world > 1 else "single",
                   "l2": "inputs larger than L2 (~6 GB read per step)",
                   "ctx_growth": "contexts advance by the accepted length each step",
                   **({"drafter_layers": "per link: W_in [1024 x (5376+1024)] on the committed "
                       "hidden row and the embedding of the last token, 4 x (RMSNorm, W_q, "
                       "cross-attention, W_o, RMSNorm, gated GELU MLP 4096, W_d), RMSNorm, "
                       "W_back [5376 x 1024]; synthetic weights"} if a.drafter_layers else {}),
                   **({"target_layers": "verify through 2 target layers (sliding D256 W512, "
                       "then global D512), each RMSNorm, W_q/W_k/W_v, verify attention, W_o, "
                       "RMSNorm, gated GELU MLP 21504, W_d at d 5376; synthetic weights; the "
                       "dense head still reads the given hidden rows"} if a.target_layers
                      else {})},
        "gpu_launches": kernels_per_step * a.steps,
        "roofline": roof(dom),
        "roofline_attention": roof("verify_global"),
        "roofline_lm_head": roof("head_dense"),
        "kernels": per_kernel,
        "kernel_busy_ms_per_step": round(busy_ms, 4),
        "clocks": clocks,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "mean_accepted": round(mean_acc, 4),
        "device_status": status,
    }
    print(json.dumps(line))


def run_reference(a, rank, world):
    """The CPU oracle, as it stands, on the host cores: each step is a bounded sample (one
    sequence of the batch, the full step for it)."""
    if rank != 0:
        return
    import torch  # noqa: F401
    os.environ.setdefault("CUDA_VISIBLE_DEVICES", "")
    st = HostOnlyStep(a.k, a.batch, a.ctx, dense=a.drafter_layers, target=a.target_layers)
    for s in range(a.warmup):
        oracle_sample(st, [s % st.B], s)
    t = time.perf_counter()
    nv = 0
    for s in range(a.steps):
        nv += oracle_sample(st, [s % st.B], a.warmup + s)
    dt = time.perf_counter() - t
    value = nv / dt
    line = {"metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(dt / a.steps * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": workload_name(a.batch, a.ctx, a.k, a.drafter_layers,
                                                 a.target_layers), "batch": a.batch,
                       "ctx": a.ctx, "k": a.k},
            "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": blas_threads(),
                             "kind": "oracle",
                             "sample": "per step one sequence of the batch (round robin): the "
                                       "full step for it in float64 on the host"},
            "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


class HostOnlyStep:
    """The workload's host tensors only (for the CPU oracle arm)."""

    def __init__(self, k, B, L, reserve=64, dense=False, target=False):
        import torch

        import synthetic as S
        self.dense, self.target = dense, target
        self.k, self.B, self.n_q = k, B, k + 1
        self.hq, self.hkv, self.bs = 16, 4, 16
        self.V, self.d, self.dh = 262144, 5376, 1024
        self.C, self.cs, self.top_c = 1024, 256, 32
        seed = 100
        self.w = S.Workload("g", B, L, k, 16, 4, [S.AttnLayer(512), S.AttnLayer(256, 512)],
                            self.d, self.V, seed=seed, n_clusters=self.C, cluster_size=self.cs,
                            drafter_hidden=self.dh, top_c=self.top_c)
        self.L0 = S.contexts(self.w)
        mb = int((self.L0.max() + reserve + self.bs - 1) // self.bs)
        self.host = {f"cache{layer}": S.make_cache(self.w, layer, self.L0, reserve=reserve,
                                                   max_blocks=mb) for layer in (0, 1)}
        inp = {}
        for layer in (0, 1):
            s = S.make_step_qkv(self.w, layer, self.n_q)
            inp[f"q{layer}"], inp[f"kn{layer}"], inp[f"vn{layer}"] = s["q"], s["k_new"], s["v_new"]
        inp["hidden"] = S.make_hidden(self.w, B * self.n_q)
        for j in range(k):
            for layer, D in ((0, 512), (1, 256)):
                n = 1 if layer == 0 else 3
                inp[f"dq{j}_{layer}"] = S.bf16(S.normal(seed * 31 + 10 * j + layer,
                                                        (n, B, 1, self.hq, D), 1 / math.sqrt(D)))
            inp[f"dh{j}"] = S.bf16(S.normal(seed * 37 + j, (B, self.dh)))
        self.host_inputs = inp
        self.host["cl"] = S.make_clustered_head(self.w)
        self.host["W"] = None
        f32 = lambda t: t.float().numpy()  # bf16 -> float32 is exact
        if dense:
            dw = S.make_drafter_weights(seed, self.dh, self.d, self.V, self.hq,
                                        (256, 256, 256, 512))
            self.host["drafter"] = {
                "E": f32(dw["E"]), "W_in": f32(dw["W_in"]), "g_final": f32(dw["g_final"]),
                "W_back": f32(dw["W_back"]),
                "layers": [{kk: f32(v) for kk, v in lw.items()} for lw in dw["layers"]]}
            self.host["h0"] = S.make_hidden(self.w, B, step=97)
        if target:
            tw = S.make_target_weights(seed, self.d, 4 * self.d, self.hq, self.hkv,
                                       ((256, 512), (512, 0)))
            self.host["target"] = [{kk: (f32(v) if hasattr(v, "float") else v)
                                    for kk, v in lw.items()} for lw in tw]
            inp["x0"] = torch.from_numpy(S.normal(seed * 41 + 5, (B * self.n_q, self.d)))


if __name__ == "__main__":
    main()
