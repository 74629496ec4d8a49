#!/usr/bin/env python
"""Benchmark of the speculative-decoding verify step on B200.

The default workload (``spec_step``) is one pass of the whole hot path for a batch of B = 8
sequences with 16384 committed tokens and k = 2 drafts -- the global-layer verify
configuration at its reference point, with the drafter's pass over the same shared cache:

  drafter chain, j = 0..k-1:   3 x sd_draft_xattn (sliding, D256, W512) + 1 x sd_draft_xattn
                               (global, D512) on the target cache, the clustered LM head
                               (1024 clusters x 256 tokens, d 1024, top 32) and the drafter's
                               own draw of draft j (sd_accept, k = 0, purpose 2)
  verify:                      sd_verify_attn on the global (D512) and sliding (D256, W512)
                               layers (k+1 = 3 positions, 16q/4kv, block 16), the dense LM head
                               (d 5376, V 262144), sd_accept (T = 1), sd_commit

The draft distribution q that the drafter samples from and the acceptance tests against is, by
default, the target's own logits perturbed by the tuned noise of the synthetic recipe (standard
deviation 1.446 at draft 1 and 1.318 after it, which makes the closed-form acceptance 0.47 and
then 0.51, the serving guide's measured per-position rates).  Random drafter weights give a q
unrelated to p, which rejects almost every draft; the drafter's kernels still run at full size
and their logits are written, but the draws read the tuned q (``--random-q`` draws from the
drafter's clustered logits instead).  The tuned q is device-resident, like the weights: it
stands in for the drafter's device output.

Other workloads (``--workload``), one JSON line each: ``tiny_fp32`` (B 1, ctx 256, fp32,
d 256, V 1024), ``edge`` (B 1, ctx 4096, sliding D256 W512, d 2560), ``global`` (B 8, ctx 16384,
global D512 only, k swept by --k), ``drafter`` (the 4-layer drafter pass with its dense layers
chained for 4 drafts; drafted tokens/s) and ``serving`` (B 64, ragged contexts in
[1024, 16384], shuffled block tables, a sliding and a global layer).  Workloads without a
drafter pass draw their k drafts from q in one sd_accept call (k = 0, purpose 2) each step.

The metric is verified positions per second, B * (k+1) per step, over the whole job.
Inputs are synthetic and resident in HBM; the large workloads read far more than the 126 MB L2
per step, so no L2 flush is needed between steps (the line says which).  Contexts grow by the
accepted length each step.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload NAME] [--k K] [--batch B] [--ctx L]

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
from dataclasses import dataclass, field, replace

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "verified tokens/s per verify step (B,k,ctx); HBM GB/s as % of B200 peak"
UNIT = "verified tokens/s"
NOISE_FILE = os.path.join(ROOT, "tests", "golden", "draft_noise.json")


# --------------------------------------------------------------------------------- workloads

@dataclass
class Cfg:
    """One benchmark workload."""
    kind: str                      # workload family (see WORKLOADS)
    B: int
    L: object                      # committed context: int, or (lo, hi) ragged
    k: int                         # drafts per sequence
    verify_layers: tuple           # ((head_dim, window), ...) of the verify
    hq: int = 16
    hkv: int = 4
    d: int = 5376                  # target width (dense head input)
    V: int = 262144
    dtype: str = "bf16"
    shuffle: bool = False
    chain: int = 0                 # drafter chain links per step (0: no drafter pass)
    xlayers: tuple = ()            # drafter layers' cache ((D, W), ...)
    dh: int = 1024                 # drafter width
    C: int = 1024
    cs: int = 256
    top_c: int = 32
    drafter_dense: bool = False    # the drafter's projections around its cross-attention
    target_layers: bool = False    # verify through two target layers with their projections
    q_mode: str = "tuned"          # "tuned": q = softmax((z + noise) / T); "drafter": its logits
    sigmas: tuple = ()             # noise std of draft position 0, 1, ...
    T: float = 1.0
    verify: bool = True
    seed_base: int = 100

    @property
    def n_q(self):
        return self.k + 1

    @property
    def cache_layers(self):
        """Distinct (D, W) layers of the target cache, in first-use order."""
        out = []
        for lay in tuple(self.verify_layers) + tuple(self.xlayers):
            if lay not in out:
                out.append(lay)
        return out

    def name(self):
        ctx = self.L if isinstance(self.L, int) else "%d-%d" % tuple(self.L)
        base = {"spec_step": "spec_step", "tiny_fp32": "tiny_fp32", "edge": "edge_verify",
                "global": "global_verify", "drafter": "drafter_pass",
                "serving": "serving_verify"}[self.kind]
        n = f"{base}_b{self.B}_ctx{ctx}_k{self.k}"
        if self.drafter_dense and self.kind == "spec_step":
            n += "_drafter_layers"
        if self.target_layers:
            n += "_target_layers"
        if self.kind in ("spec_step",) and self.q_mode == "drafter":
            n += "_random_q"
        return n

    @property
    def unit(self):
        return UNIT if self.verify else "drafted tokens/s"


def _sigmas(k):
    try:
        d = json.load(open(NOISE_FILE))
        s0, s1 = float(d["sigma_pos0"]), float(d["sigma_later"])
    except Exception:
        s0, s1 = 1.4458, 1.3183
    return tuple([s0] + [s1] * max(0, k - 1))


def make_cfg(a) -> Cfg:
    """The workload named by --workload, with --k / --batch / --ctx applied where they fit."""
    kind = a.workload
    SL, GL = (256, 512), (512, 0)
    if kind == "spec_step":
        k = a.k
        c = Cfg("spec_step", a.batch, a.ctx, k, (GL, SL), chain=k, xlayers=(SL, SL, SL, GL),
                drafter_dense=a.drafter_layers, target_layers=a.target_layers,
                q_mode="drafter" if a.random_q else "tuned", sigmas=_sigmas(k))
    elif kind == "tiny_fp32":
        # configuration 1: draft q = softmax(z + N(0, 1.5)) (1.5 a variance)
        c = Cfg("tiny_fp32", 1, 256, 2, ((64, 0),), hq=4, hkv=1, d=256, V=1024, dtype="f32",
                sigmas=(math.sqrt(1.5),) * 2, seed_base=1)
    elif kind == "edge":
        c = Cfg("edge", 1, 4096, 2, (SL,), hq=8, hkv=2, d=2560, sigmas=_sigmas(2), seed_base=2)
    elif kind == "global":
        c = Cfg("global", 8, 16384, a.k, (GL,), sigmas=_sigmas(a.k), seed_base=3)
    elif kind == "drafter":
        c = Cfg("drafter", 8, 16384, 4, (), chain=4, xlayers=(SL, SL, SL, GL),
                drafter_dense=True, q_mode="drafter", verify=False, seed_base=4)
    elif kind == "serving":
        c = Cfg("serving", 64, (1024, 16384), 2, (SL, GL), shuffle=True, sigmas=_sigmas(2),
                seed_base=5)
    else:
        raise SystemExit(f"unknown workload {kind}")
    return c


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="spec_step",
                    choices=["spec_step", "tiny_fp32", "edge", "global", "drafter", "serving"])
    ap.add_argument("--k", type=int, default=2, help="drafts (spec_step, global)")
    ap.add_argument("--batch", type=int, default=8, help="sequences (spec_step)")
    ap.add_argument("--ctx", type=int, default=16384, help="committed tokens (spec_step)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--telemetry-steps", type=int, default=64,
                    help="untimed steps after the timed region whose acceptance outcomes are "
                         "read back for the telemetry")
    ap.add_argument("--random-q", action="store_true",
                    help="spec_step: draw and accept against the drafter's clustered logits "
                         "(random weights) instead of the tuned q")
    ap.add_argument("--drafter-layers", action="store_true",
                    help="spec_step: run the drafter's dense layers (input projection, 4 x "
                         "(W_q, W_o, gated MLP, W_d), output projection) around its "
                         "cross-attention, so the chain is driven by the committed hidden row "
                         "and tokens")
    ap.add_argument("--target-layers", action="store_true",
                    help="spec_step: verify through two target layers with their own "
                         "projections (a sliding and a global layer: q/k/v/o and a gated MLP "
                         "21504 wide at d 5376) instead of the two attention calls on given "
                         "q, k, v")
    return ap.parse_args(argv)


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


def dram_traffic(group, workload):
    """DRAM bytes per launch of a kernel group from the committed ncu summary, with the source
    hash it was taken at, or (None, None) when the summary is missing or the kernel source
    changed since its counters were taken."""
    path = os.path.join(ROOT, "profiles", "dram_traffic_%s.json" % workload)
    try:
        d = json.load(open(path))
        e = d["groups"][group]
        sha = source_hash(GROUP_SOURCE[group])
        if e["source_sha"] != sha:
            return None, None
        return int(e["dram_bytes_per_launch"]), sha
    except Exception:
        return None, None


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


# --------------------------------------------------------------------------------- the step

class SpecStep:
    """Host inputs, device buffers, descriptors and the call sequence of one step of a
    workload.  dev=None builds the host side only (the CPU oracle arm)."""

    def __init__(self, cfg: Cfg, reserve=600, rank=0, dev="cuda"):
        import numpy as np
        import torch

        import synthetic as S
        self.cfg, self.np, self.torch, self.S = cfg, np, torch, S
        self.dev = dev
        c = cfg
        self.k, self.B, self.n_q = c.k, c.B, c.n_q
        self.hq, self.hkv, self.bs = c.hq, c.hkv, 16
        self.V, self.d, self.dh = c.V, c.d, c.dh
        self.C, self.cs, self.top_c = c.C, c.cs, c.top_c
        self.dense, self.target = c.drafter_dense, c.target_layers
        self.f32 = c.dtype == "f32"
        seed = c.seed_base + 7 * rank if c.kind == "spec_step" else c.seed_base + 1000 * rank
        self.seed = seed
        lay = [S.AttnLayer(D, W) for D, W in c.cache_layers]
        wg = S.Workload(c.kind, c.B, c.L, c.k, c.hq, c.hkv, lay, c.d, c.V, dtype=c.dtype,
                        shuffle=c.shuffle, seed=seed, n_clusters=c.C, cluster_size=c.cs,
                        drafter_hidden=c.dh, top_c=c.top_c)
        self.w = wg
        self.L0 = S.contexts(wg)
        self.li = {lw: i for i, lw in enumerate(c.cache_layers)}
        mb = int((self.L0.max() + reserve + self.bs - 1) // self.bs)
        self.host = {"caches": [S.make_cache(wg, i, self.L0, reserve=reserve, max_blocks=mb)
                                for i in range(len(c.cache_layers))]}
        # per-step inputs (copied from pinned host memory in the end-to-end leg)
        inp = {}
        if c.verify and not c.target_layers:
            for D, W in c.verify_layers:
                i = self.li[(D, W)]
                s = S.make_step_qkv(wg, i, self.n_q)
                inp[f"q{i}"], inp[f"kn{i}"], inp[f"vn{i}"] = s["q"], s["k_new"], s["v_new"]
        if c.verify and c.target_layers:
            # input rows of the k+1 positions (the residual stream entering the first layer)
            inp["x0"] = torch.from_numpy(S.normal(seed * 41 + 5, (c.B * self.n_q, c.d)))
        if c.verify:
            inp["hidden"] = S.make_hidden(wg, c.B * self.n_q)
        for j in range(0 if c.drafter_dense else c.chain):
            for i, (D, W) in enumerate(c.xlayers):
                inp[f"dq{j}_{i}"] = S.bf16(S.normal(seed * 31 + 10 * j + i, (c.B, 1, c.hq, D),
                                                    1 / math.sqrt(D)))
            inp[f"dh{j}"] = S.bf16(S.normal(seed * 37 + j, (c.B, c.dh)))
        if c.drafter_dense and not c.verify:
            # the drafter pass alone: the target's last activation and the last token enter
            # from the host every step
            inp["h0"] = S.make_hidden(wg, c.B, step=97)
            inp["tok0"] = torch.from_numpy(
                np.random.default_rng([seed, 0x70]).integers(0, c.V, c.B).astype(np.int32))
        self.host_inputs = inp
        # phases: drafter link j reads its own block, the verify the last one
        self.phases = [[kk for kk in inp if kk.startswith((f"dq{j}_", f"dh{j}")) or
                        (j == 0 and kk in ("h0", "tok0"))] for j in range(c.chain)]
        if c.verify:
            self.phases.append([kk for kk in inp if not kk.startswith(("dq", "dh"))])
        self.host["W"] = None  # regenerated on demand for the CPU oracle
        if c.chain > 0:
            self.host["cl"] = S.make_clustered_head(wg)
        if c.drafter_dense:
            self.host["drafter_w"] = S.make_drafter_weights(
                seed, c.dh, c.d, c.V, c.hq, tuple(D for D, _ in c.xlayers))
            self.host["h0"] = S.make_hidden(wg, c.B, step=97)
        if c.target_layers:
            self.host["target_w"] = S.make_target_weights(
                seed, c.d, 4 * c.d, c.hq, c.hkv, ((256, 512), (512, 0)))
        if dev is not None:
            self._device(reserve)

    # ------------------------------------------------------------------ device side
    def _device(self, reserve):
        np, torch, S, c = self.np, self.torch, self.S, self.cfg
        import verify_step_b200 as sd
        self.sd = sd
        dev, B, k = self.dev, self.B, self.k
        g = lambda t: t.contiguous().to(dev)
        sdt = sd.SD_F32 if self.f32 else sd.SD_BF16
        self.sdt = sdt
        self.cache = [dict(k=g(h["k_cache"]), v=g(h["v_cache"]), table=g(h["table"]),
                           nb=h["num_blocks"], mb=h["max_blocks"]) for h in self.host["caches"]]
        self.ctx = g(torch.from_numpy(self.L0))
        self.ctx0 = self.ctx.clone()
        # all per-step inputs in one device buffer (256-byte aligned views), ordered by phase
        offs, total, self.phase_ranges = {}, 0, []
        for keys in self.phases:
            start = total
            for kk in keys:
                v = self.host_inputs[kk]
                offs[kk] = total
                total += (v.numel() * v.element_size() + 255) // 256 * 256
            self.phase_ranges.append((start, total))
        self.input_buf = torch.empty(max(total, 256), dtype=torch.uint8, device=dev)
        self.input_offs = offs
        self.inputs = {}
        for kk, v in self.host_inputs.items():
            n = v.numel() * v.element_size()
            view = self.input_buf[offs[kk]:offs[kk] + n].view(v.dtype).view(v.shape)
            view.copy_(v.contiguous().to(dev))
            self.inputs[kk] = view
        f32, i32 = torch.float32, torch.int32
        if c.verify:
            self.W = g(S.make_lm_head(self.w))
            self.attn_out = {lw: torch.empty((B, self.n_q, self.hq, lw[0]),
                                             dtype=torch.float32 if self.f32 else torch.bfloat16,
                                             device=dev) for lw in c.verify_layers}
            self.target_logits = torch.empty((B * self.n_q, self.V), dtype=f32, device=dev)
        if c.chain > 0:
            self.cl = {kk: g(v) for kk, v in self.host["cl"].items()}
            self.xout = {lw: torch.empty((B, 1, self.hq, lw[0]), dtype=torch.bfloat16,
                                         device=dev) for lw in set(c.xlayers)}
            self.draft_logits = torch.empty((B, c.chain, self.V), dtype=f32, device=dev)
            self.sel = torch.empty((B, self.top_c), dtype=i32, device=dev)
        self.drafts = torch.zeros((B, max(k, c.chain)), dtype=i32, device=dev)
        # the step's results, read back to the host as one block: n_accepted then out_tokens
        self.results = torch.zeros(B * (1 + self.n_q), dtype=i32, device=dev)
        self.n_acc = self.results[:B]
        self.out_tokens = self.results[B:].view(B, self.n_q)
        self.margin = torch.zeros(B, dtype=i32, device=dev)
        hid_dt = torch.float32 if self.f32 else torch.bfloat16
        self.next_hidden = torch.zeros((B, self.d), dtype=hid_dt, device=dev)
        if c.drafter_dense:
            from verify_step_b200 import drafter as VD
            self.VD = VD
            self.dshape = VD.DrafterShape(batch=B, d=self.dh, d_target=self.d,
                                          ff=S.DRAFTER_FF, h_q=self.hq,
                                          head_dims=tuple(D for D, _ in c.xlayers),
                                          vocab=self.V)
            self.dwts = VD.device_weights(self.host["drafter_w"], dev)
            self.dbuf = VD.buffers(self.dshape, dev)
            self.next_hidden.copy_(g(self.host["h0"]))
        if c.target_layers:
            from verify_step_b200 import target as VT
            self.VT = VT
            self.tshape = VT.TargetShape(batch=B, n_q=self.n_q, d=self.d, ff=4 * self.d,
                                         h_q=self.hq, h_kv=self.hkv,
                                         layers=((256, 512), (512, 0)))
            self.twts = VT.device_weights(self.host["target_w"], dev)
            self.tbuf = VT.buffers(self.tshape, dev)
        # descriptors
        self.vdesc = {lw: self._adesc(lw, self.n_q) for lw in c.verify_layers}
        if c.target_layers:
            for lw in ((256, 512), (512, 0)):
                self.vdesc[lw] = self._adesc(lw, self.n_q)
        self.xdesc = [{lw: self._adesc(lw, 1, q_offset=j) for lw in set(c.xlayers)}
                      for j in range(c.chain)]
        if c.verify:
            self.hdesc_dense = sd.HeadDesc(m=B * self.n_q, d=self.d, vocab=self.V, dtype=sdt)
        if c.chain > 0:
            self.hdesc_cl = sd.HeadDesc(m=B, d=self.dh, vocab=self.V, ld_logits=c.chain * self.V,
                                        n_clusters=self.C, cluster_size=self.cs,
                                        top_c=self.top_c, dtype=sd.SD_BF16)
        # step counter on the device: the acceptance draws of step s use counter value s (the
        # drafter's chain step j adds (j+1) << 28 to keep its uniforms apart); sd_commit
        # advances it, so a step captured once in a CUDA graph draws fresh numbers each replay
        self.step_dev = torch.zeros(1, dtype=torch.int64, device=dev)
        sp = self.step_dev.data_ptr()
        qrows = c.chain if c.q_mode == "drafter" else k
        self.adesc_draft = [sd.AcceptDesc(batch=B, k=0, vocab=self.V, temperature=c.T, seed=7,
                                          step=(j + 1) << 28, purpose=2,
                                          ld_target=qrows * self.V, ld_out=self.drafts.shape[1],
                                          step_ptr=sp)
                            for j in range(c.chain)]
        # workloads without a drafter pass draw all k drafts from q in one call
        self.adesc_draws = sd.AcceptDesc(batch=B * k, k=0, vocab=self.V, temperature=c.T, seed=7,
                                         step=1 << 28, purpose=2, step_ptr=sp)
        if c.verify:
            self.adesc = sd.AcceptDesc(batch=B, k=k, vocab=self.V, temperature=c.T, seed=7,
                                       step=0, purpose=1, ld_draft=self.V,
                                       ld_out=self.n_q, step_ptr=sp)
            cc = self.cache[self.commit_layer()]
            self.cdesc = sd.CommitDesc(batch=B, k=k, block_size=self.bs,
                                       max_blocks_per_seq=cc["mb"], num_blocks=cc["nb"], d=self.d,
                                       hidden_dtype=sdt, step_ptr=sp)
            self.ctable = self.cache[self.commit_layer()]["table"]
        wsz = [sd.sd_verify_attn_workspace_size(x) for x in self.vdesc.values()]
        wsz += [sd.sd_draft_xattn_workspace_size(x) for row in self.xdesc for x in row.values()]
        if c.chain > 0:
            wsz.append(sd.sd_lm_head_workspace_size(self.hdesc_cl))
        wsz += [sd.sd_accept_workspace_size(x) for x in self.adesc_draft]
        if c.verify:
            wsz += [sd.sd_accept_workspace_size(self.adesc),
                    sd.sd_accept_workspace_size(self.adesc_draws)]
        self.ws = torch.empty(max([256] + wsz), dtype=torch.uint8, device=dev)
        # the draft distribution: the tuned noise on the target's own logits (the hidden rows,
        # hence the logits, are the same every step)
        if c.q_mode == "tuned" and c.verify:
            sd.sd_lm_head(self.hdesc_dense, self.inputs["hidden"], self.W, self.target_logits)
            torch.cuda.synchronize()
            z = self.target_logits.view(B, self.n_q, self.V)[:, :k].cpu()
            self.q_tuned = g(z + self.tuned_noise(range(B)))
            self.host["z_gpu"] = z
        torch.cuda.synchronize()

    def commit_layer(self):
        """Cache layer whose block table gives the committed slots: the first global layer."""
        for i, (D, W) in enumerate(self.cfg.cache_layers):
            if W == 0:
                return i
        return 0

    def tuned_noise(self, seqs):
        """Noise of the tuned draft logits, [len(seqs), k, V] float32 (position i has standard
        deviation sigmas[i]); the same values for the GPU and the oracle arm."""
        np, torch, S, c = self.np, self.torch, self.S, self.cfg
        out = np.empty((len(seqs), self.k, self.V), np.float32)
        for n, b in enumerate(seqs):
            for i in range(self.k):
                out[n, i] = S.normal(self.seed * 53 + 1000 * b + i, (self.V,), c.sigmas[i])
        return torch.from_numpy(out)

    def _adesc(self, lw, n_q, q_offset=0):
        D, W = lw
        c = self.cache[self.li[lw]]
        return self.sd.AttnDesc(batch=self.B, n_q=n_q, h_q=self.hq, h_kv=self.hkv, head_dim=D,
                                block_size=self.bs, max_blocks_per_seq=c["mb"],
                                num_blocks=c["nb"], window=W, scale=1 / math.sqrt(D),
                                dtype=self.sdt, q_offset=q_offset)

    @staticmethod
    def group(kind, lw):
        return f"{kind}_{'global' if lw[1] == 0 else 'sliding'}"

    # kernels per call of each group (fallback when the graph's kernel nodes cannot be counted)
    LAUNCHES = dict(xattn_sliding=1, xattn_global=2, verify_sliding=1, verify_global=3,
                    head_dense=1, head_clustered=3, accept_draft=2, accept=2, commit=1,
                    drafter_dense=1, target_dense=1)

    def launches_per_step(self):
        return sum(self.LAUNCHES[g] * n for g, n in self.calls_per_step().items())

    def q_source(self):
        return self.q_tuned if self.cfg.q_mode == "tuned" else self.draft_logits

    def run(self, ev=None, before_phase=None):
        """Issue one step on the current stream.  ev (used while capturing a CUDA graph) maps a
        kernel group to a list that receives (start, end) events recorded as graph nodes
        around each call of that group.  before_phase(j) is called before drafter link j
        (j < chain) and before the verify (j = chain)."""
        sd, I, c = self.sd, self.inputs, self.cfg

        def timed(name, fn):
            if ev is None or name not in ev:
                fn()
                return
            a, b = new_event(), new_event()
            record_external(a)
            fn()
            record_external(b)
            ev[name].append((a, b))

        for j in range(c.chain):
            if before_phase is not None:
                before_phase(j)
            if self.dense:
                self._dense_link(j, timed)
            else:
                for i, lw in enumerate(c.xlayers):
                    cc = self.cache[self.li[lw]]
                    timed(self.group("xattn", lw), lambda i=i, lw=lw, cc=cc: sd.sd_draft_xattn(
                        self.xdesc[j][lw], I[f"dq{j}_{i}"], cc["k"], cc["v"], cc["table"],
                        self.ctx, None, self.xout[lw], self.ws))
            timed("head_clustered", lambda: self._clustered(j))
            ad = self.adesc_draft[j]
            timed("accept_draft", lambda: sd.sd_accept(
                ad, self._row_ptr(self.q_source(), j), None, None, self.n_acc,
                self._col_ptr(self.drafts, j), None, self.ws))
        if not c.verify:
            return
        if before_phase is not None:
            before_phase(c.chain)
        if c.chain == 0:
            timed("accept_draft", lambda: sd.sd_accept(
                self.adesc_draws, self.q_tuned, None, None, self.n_acc, self.drafts, None,
                self.ws))
        if self.target:
            self._target_layers(timed)
        else:
            for lw in c.verify_layers:
                i, cc = self.li[lw], self.cache[self.li[lw]]
                timed(self.group("verify", lw), lambda i=i, lw=lw, cc=cc: sd.sd_verify_attn(
                    self.vdesc[lw], I[f"q{i}"], I[f"kn{i}"], I[f"vn{i}"], cc["k"], cc["v"],
                    cc["table"], self.ctx, self.attn_out[lw], self.ws))
        timed("head_dense", lambda: sd.sd_lm_head(self.hdesc_dense, I["hidden"], self.W,
                                                  self.target_logits))
        timed("accept", lambda: sd.sd_accept(self.adesc, self.target_logits, self.q_source(),
                                             self.drafts, self.n_acc, self.out_tokens,
                                             self.margin, self.ws))
        timed("commit", lambda: sd.sd_commit(self.cdesc, self.ctable, self.ctx, self.n_acc,
                                             self.slots_buf(), I["hidden"], self.next_hidden))

    def slots_buf(self):
        if not hasattr(self, "_slots"):
            self._slots = self.torch.zeros((self.B, self.n_q), dtype=self.torch.int32,
                                           device=self.dev)
        return self._slots

    def _dense_link(self, j, timed):
        sd, c = self.sd, self.cfg

        def attend(i, q, o):
            lw = c.xlayers[i]
            cc = self.cache[self.li[lw]]
            timed(self.group("xattn", lw), lambda: sd.sd_draft_xattn(
                self.xdesc[j][lw], q, cc["k"], cc["v"], cc["table"], self.ctx, None, o,
                self.ws))

        if j == 0:
            if c.verify:  # the committed hidden row and the last emitted token of the last step
                h_prev, toks, ld, sel = self.next_hidden, self.out_tokens, self.n_q, self.n_acc
            else:         # drafter pass alone: the row and token copied in for this step
                h_prev, toks, ld, sel = self.inputs["h0"], self.inputs["tok0"], 1, None
        else:
            h_prev, toks, ld, sel = (self.dbuf["h_back"], self._col_ptr(self.drafts, j - 1),
                                     self.drafts.shape[1], None)
        self.VD.link(self.dshape, self.dwts, self.dbuf, h_prev, toks, ld, attend,
                     token_sel=sel, wrap=lambda fn: timed("drafter_dense", fn))

    def _target_layers(self, timed):
        caches = []
        for lw in ((256, 512), (512, 0)):
            cc = self.cache[self.li[lw]]
            caches.append(dict(desc=self.vdesc[lw], k=cc["k"], v=cc["v"], table=cc["table"]))
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
        # logits of chain link j go to row b*chain + j of draft_logits (ld_logits = chain * V)
        hidden = self.dbuf["h"] if self.dense else self.inputs[f"dh{j}"]
        self.sd.sd_lm_head(self.hdesc_cl, hidden, self.cl["w_cm"],
                           self._row_ptr(self.draft_logits, j),
                           centroids=self.cl["centroids"],
                           cluster_tokens=self.cl["cluster_tokens"], sel_clusters=self.sel,
                           ws=self.ws)

    # --------------------------------------------------------------- algorithmic bytes
    def bytes_per_call(self, L):
        """Algorithmic HBM bytes of one call of each kernel group at committed lengths L."""
        np, c = self.np, self.cfg
        B, hkv, n_q, hq = self.B, self.hkv, self.n_q, self.hq
        es = 4 if self.f32 else 2
        L = np.asarray(L, np.float64)
        out = {}
        verify_layers = (((256, 512), (512, 0)) if self.target else c.verify_layers) \
            if c.verify else ()
        for lw in verify_layers:
            D, W = lw
            # K and V of every key read once per (sequence, kv head), new rows written,
            # queries read, outputs written
            keys = (L + n_q) if W == 0 else np.minimum(L + n_q, W + n_q - 1)
            out[self.group("verify", lw)] = int(keys.sum() * hkv * D * es * 2 +
                                                B * n_q * hkv * D * es * 2 * 2 +
                                                2 * B * n_q * hq * D * es)
        for lw in set(c.xlayers):
            D, W = lw
            # chain link j queries position L + j: the committed keys in its window
            keys = L if W == 0 else np.mean([np.minimum(L, W - 1 - j) for j in range(c.chain)],
                                            axis=0)
            out[self.group("xattn", lw)] = int(keys.sum() * hkv * D * 2 * 2 +
                                               2 * B * hq * D * 2)
        if c.verify:
            out["head_dense"] = int(self.V * self.d * es + B * n_q * self.d * es +
                                    B * n_q * self.V * 4)
            out["accept"] = int((B * n_q + B * self.k) * self.V * 4)
            out["commit"] = int(B * (n_q * 4 * 2 + self.d * es * 2))
        if c.chain > 0:
            out["head_clustered"] = int(self.C * self.dh * 2 + B * self.dh * 2 +
                                        B * self.top_c * self.cs * self.dh * 2 +
                                        B * self.V * 4)
            out["accept_draft"] = int(B * self.V * 4)
        elif c.verify:
            out["accept_draft"] = int(B * self.k * self.V * 4)
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
        c = self.cfg
        out = {}
        for lw in c.xlayers:
            g = self.group("xattn", lw)
            out[g] = out.get(g, 0) + c.chain
        if c.chain > 0:
            out["head_clustered"] = c.chain
            out["accept_draft"] = c.chain
        if c.verify:
            if c.chain == 0:
                out["accept_draft"] = 1
            layers = ((256, 512), (512, 0)) if self.target else c.verify_layers
            for lw in layers:
                g = self.group("verify", lw)
                out[g] = out.get(g, 0) + 1
            out.update(head_dense=1, accept=1, commit=1)
        if self.dense:
            out["drafter_dense"] = self.VD.LAUNCHES_PER_LINK * c.chain
        if self.target:
            out["target_dense"] = 2 * self.VT.LINEAR_CALLS_PER_LAYER
        return out

    def positions_per_step(self):
        """Verified positions (or drafted tokens for the drafter pass alone) per step."""
        return self.B * (self.n_q if self.cfg.verify else self.cfg.chain)

    def input_bytes(self):
        return sum(v.numel() * v.element_size() for v in self.host_inputs.values())

    def reset(self):
        self.ctx.copy_(self.ctx0)

    def capture(self, ev=None):
        torch = self.torch
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.run(ev)
        return g

    def capture_e2e(self, pinned, res_h):
        """The step with its host transfers as graph nodes: the first phase's inputs are copied
        on the step's stream before it starts; the later phases' inputs are copied on a second
        stream meanwhile, each phase waiting only for its own block; the results are copied
        back to pinned host memory at the end."""
        torch = self.torch
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        with torch.cuda.graph(g):
            cur = torch.cuda.current_stream()
            s0, e0 = self.phase_ranges[0]
            if e0 > s0:
                self.input_buf[s0:e0].copy_(pinned[s0:e0], non_blocking=True)
            fork = torch.cuda.Event()
            fork.record(cur)
            side.wait_event(fork)
            ready = []
            with torch.cuda.stream(side):
                for s, e in self.phase_ranges[1:]:
                    if e > s:
                        self.input_buf[s:e].copy_(pinned[s:e], non_blocking=True)
                    ev = torch.cuda.Event()
                    ev.record(side)
                    ready.append(ev)

            def before_phase(j):
                if j >= 1:
                    cur.wait_event(ready[j - 1])

            self.run(before_phase=before_phase)
            if not ready:  # a single phase: nothing else to wait for
                cur.wait_event(fork)
            else:
                cur.wait_event(ready[-1])
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

def oracle_sample(st, seqs, s):
    """The CPU oracle on sequences ``seqs`` of the batch: the full step of the workload for
    them (drafter chain, verify on every layer, dense LM head over the full vocabulary,
    acceptance, commit).  Returns the number of verified positions (drafted tokens for the
    drafter pass alone)."""
    import numpy as np
    import torch

    import synthetic as S
    from oracle import accept as OACC
    from oracle import attention as OA
    from oracle import commit as OC
    from oracle import drafter as OD
    from oracle import lm_head as OH
    from oracle import target as OT

    class F64:
        def __init__(self, t):
            self.t = t
            self.shape = tuple(t.shape)

        def __getitem__(self, idx):
            idx = idx if isinstance(idx, tuple) else (idx,)
            idx = tuple(torch.as_tensor(np.asarray(i, np.int64)) if isinstance(i, np.ndarray)
                        else i for i in idx)
            return self.t[idx].to(torch.float64).numpy()

    c = st.cfg
    k, n_q, B, V = st.k, st.n_q, st.B, st.V
    hi = st.host_inputs
    f = lambda t: t.to(torch.float64).numpy()
    f32 = lambda t: t.float().numpy()
    L = st.L0.copy()
    seqs = list(seqs)
    m = len(seqs)
    caches = {lw: st.host["caches"][st.li[lw]] for lw in c.cache_layers}
    ocache = {lw: dict(k=F64(h["k_cache"]), v=F64(h["v_cache"]), table=h["table"].numpy()[seqs],
                       block_size=st.bs) for lw, h in caches.items()}
    rows = np.concatenate([np.arange(b * n_q, (b + 1) * n_q) for b in seqs]) if c.verify \
        else np.zeros(0, np.int64)
    z = None
    if c.verify:
        if st.host.get("W") is None:
            st.host["W"] = S.make_lm_head(st.w)
        h = f(hi["hidden"])[rows]
        Wv = F64(st.host["W"])
        z = np.empty((len(rows), V))
        chunk = 16384
        for v0 in range(0, V, chunk):
            z[:, v0:v0 + chunk] = OH.lm_head(h, Wv, np.arange(v0, min(V, v0 + chunk)))
        z = z.astype(np.float32).astype(np.float64).reshape(m, n_q, V)
    q_tuned = None
    if c.q_mode == "tuned" and c.verify:
        q_tuned = (z[:, :k].astype(np.float32) + st.tuned_noise(seqs).numpy()).astype(np.float64)
    drafts = np.zeros((m, max(k, c.chain)), np.int64)
    draft_logits = np.zeros((m, c.chain, V))
    if c.drafter_dense:
        dw = st.host["drafter_w"]
        wts = {"E": f32(dw["E"]), "W_in": f32(dw["W_in"]), "g_final": f32(dw["g_final"]),
               "W_back": f32(dw["W_back"]),
               "layers": [{kk: f32(v) for kk, v in lw.items()} for lw in dw["layers"]]}
        if c.verify:
            h_prev = f(st.host["h0"])[seqs]
            tokens = np.zeros(m, np.int64)
        else:
            h_prev = f(hi["h0"])[seqs]
            tokens = hi["tok0"].numpy()[seqs].astype(np.int64)
    for j in range(c.chain):
        if c.drafter_dense:
            atts = [OD.cross_attend(ocache[lw], st.hq, lw[0], lw[1], L[seqs], j)
                    for lw in c.xlayers]
            link = OD.drafter_step(h_prev, tokens, wts, atts)
            hj, h_prev = link["h"], link["h_back"]
        else:
            for i, (D, W) in enumerate(c.xlayers):
                cache = caches[(D, W)]
                q = f(hi[f"dq{j}_{i}"])
                for b in seqs:
                    for hh in range(st.hq):
                        OA.draft_attention_one(b, hh, q, F64(cache["k_cache"]),
                                               F64(cache["v_cache"]), cache["table"].numpy(),
                                               L, L + j, W, 1 / math.sqrt(D), st.bs)
            hj = f(hi[f"dh{j}"])[seqs]
        cl = st.host["cl"]
        lg, _, _ = OH.clustered_lm_head(hj, f(cl["centroids"]), F64(cl["w_cm"]),
                                        cl["cluster_tokens"].numpy(), st.top_c)
        draft_logits[:, j] = lg
        qj = q_tuned[:, j] if q_tuned is not None else lg
        r = OACC.accept(qj[:, None, :], None, np.zeros((m, 0)), c.T, seed=7,
                        step=((j + 1) << 28) + s, purpose=OACC.PURPOSE_DRAFTER)
        drafts[:, j] = r["out_tokens"][:, 0]
        tokens = drafts[:, j]
    if not c.verify:
        return m * c.chain
    if c.chain == 0:  # the k drafts drawn from q in one call (rows b * k + i)
        r = OACC.accept(q_tuned.reshape(m * k, 1, V), None, np.zeros((m * k, 0)), c.T, seed=7,
                        step=(1 << 28) + s, purpose=OACC.PURPOSE_DRAFTER)
        drafts[:, :k] = r["out_tokens"][:, 0].reshape(m, k)
    if c.target_layers:
        OT.verify_layers(f(hi["x0"])[rows], st.host["target_w_f32"] if "target_w_f32" in st.host
                         else _target_f32(st), [ocache[(256, 512)], ocache[(512, 0)]],
                         L[seqs], n_q, st.hq, st.hkv)
    else:
        for lw in c.verify_layers:
            D, W = lw
            i = st.li[lw]
            cache = caches[lw]
            q, kn, vn = f(hi[f"q{i}"]), f(hi[f"kn{i}"]), f(hi[f"vn{i}"])
            for b in seqs:
                for j in range(n_q):
                    for hh in range(st.hq):
                        OA.verify_attention_one(b, j, hh, q, kn, vn, F64(cache["k_cache"]),
                                                F64(cache["v_cache"]), cache["table"].numpy(),
                                                L, W, 1 / math.sqrt(D), st.bs)
    y = q_tuned if q_tuned is not None else draft_logits
    r = OACC.accept(z, y, drafts[:, :k], c.T, seed=7, step=s)
    OC.commit(L[seqs], r["n_accepted"], caches[c.cache_layers[0]]["table"].numpy()[seqs], st.bs,
              n_q, f(hi["hidden"]).reshape(B, n_q, -1)[seqs])
    return m * n_q


def _target_f32(st):
    tw = st.host["target_w"]
    st.host["target_w_f32"] = [{kk: (v.float().numpy() if hasattr(v, "float") else v)
                                for kk, v in lw.items()} for lw in tw]
    return st.host["target_w_f32"]


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


# --------------------------------------------------------------------------------- main

def config_line(st, a, world):
    c = st.cfg
    desc = {
        "spec_step": "drafter chain (4 cross-attention layers, clustered head 1024x256 top-32 "
                     "d1024, draw) per draft + verify on a global D512 and a sliding D256 W512 "
                     "layer, dense head d5376 x V262144, acceptance T=1, commit",
        "tiny_fp32": "fp32: global D64 4q/1kv verify, dense head d256 x V1024, drafts drawn "
                     "from q, acceptance T=1, commit",
        "edge": "sliding D256 W512 8q/2kv verify, dense head d2560 x V262144, drafts drawn from "
                "q, acceptance T=1, commit",
        "global": "global D512 16q/4kv verify, dense head d5376 x V262144, drafts drawn from "
                  "q, acceptance T=1, commit",
        "drafter": "drafter pass alone: 4 links, each W_in, 4 x (RMSNorm, W_q, cross-attention "
                   "into the target cache (3 sliding D256 W512, 1 global D512), W_o, gated "
                   "MLP 4096, W_d), W_back, clustered head 1024x256 top-32, draw",
        "serving": "ragged contexts U[1024,16384], shuffled block tables, sliding D256 W512 "
                   "and global D512 verify, dense head d5376 x V262144, drafts drawn from q, "
                   "acceptance T=1, commit and rollback",
    }[c.kind]
    big = c.kind != "tiny_fp32" and c.kind != "edge"
    out = {"workload": c.name(), "batch": c.B, "ctx": c.L if isinstance(c.L, int) else list(c.L),
           "k": c.k, "heads": f"{c.hq}q/{c.hkv}kv", "block_size": 16, "step": desc,
           "parallelism": "replicas" if world > 1 else "single",
           "l2": "inputs larger than L2 (GBs read per step)" if big else
                 "inputs smaller than L2, not flushed: the step reads its weights once "
                 "(tiny/edge workloads are latency-bound)",
           "shuffled_block_tables": c.shuffle}
    if c.verify:
        out["draft_q"] = ("tuned noise on the target's logits, std " +
                          "/".join("%.3f" % s for s in c.sigmas) + " per draft position "
                          "(closed-form acceptance 0.47, then 0.51); device-resident")\
            if c.q_mode == "tuned" else "the drafter's clustered-head logits (random weights)"
        out["ctx_growth"] = "contexts advance by the accepted length each step"
    if c.drafter_dense and c.kind == "spec_step":
        out["drafter_layers"] = ("per link: W_in [1024 x (5376+1024)] on the committed hidden "
                                 "row and the embedding of the last token, 4 x (RMSNorm, W_q, "
                                 "cross-attention, W_o, RMSNorm, gated GELU MLP 4096, W_d), "
                                 "RMSNorm, W_back [5376 x 1024]; synthetic weights")
    if c.target_layers:
        out["target_layers"] = ("verify through 2 target layers (sliding D256 W512, then global "
                                "D512), each RMSNorm, W_q/W_k/W_v, verify attention, W_o, "
                                "RMSNorm, gated GELU MLP 21504, W_d at d 5376; synthetic "
                                "weights; the dense head still reads the given hidden rows")
    return out


def telemetry(st, graph, steps):
    """Acceptance outcomes of ``steps`` untimed replays, read back after each: realised
    acceptance per position (cumulative P(a >= i)), mean accepted length (MAL = 1 + E[a]),
    overall acceptance E[a] / k and the count of margin-flagged sequences."""
    import numpy as np
    torch = st.torch
    acc = []
    flags = 0
    for _ in range(steps):
        graph.replay()
        torch.cuda.synchronize()
        acc.append(st.n_acc.cpu().numpy().copy())
        flags += int(st.margin.cpu().numpy().sum())
    a = np.concatenate(acc).astype(np.float64)
    k = st.k
    return {"sequences": int(a.size),
            "accept_cumulative": [round(float((a >= i).mean()), 4) for i in range(1, k + 1)],
            "mal": round(1.0 + float(a.mean()), 4),
            "acceptance_overall": round(float(a.mean()) / k, 4) if k else None,
            "margin_flagged": flags,
            "window": f"{steps} untimed steps after the timed region, n_accepted and "
                      "margin_flags read back after each"}


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

    cfg = make_cfg(a)
    # every pass below runs a.steps steps (warm-up, timed, per-kernel, e2e, telemetry): reserve
    # the blocks the contexts grow into
    reserve = (a.warmup + 4 * a.steps + a.telemetry_steps + 8) * (cfg.k + 1) + 64
    st = SpecStep(cfg, reserve=reserve, rank=rank)
    wname = cfg.name()
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
    per_step = st.positions_per_step()
    value = world * per_step * a.steps / (ms / 1e3)

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
        if g not in kern_ms or not kern_ms[g]:
            return None
        ach = nbytes[g] / (kern_ms[g] * 1e6)
        traffic, sha = dram_traffic(g, wname)
        return {"kernel": g, "bound": "hbm", "achieved": round(ach, 1), "peak": hbm,
                "unit": "GB/s", "frac": round(ach / hbm, 4), "traffic": traffic,
                "traffic_source": (f"committed ncu summary profiles/dram_traffic_{wname}.json, "
                                   f"kernel source sha {sha}") if traffic else None,
                "peak_source": src, "bytes_per_launch": nbytes[g],
                "ms_per_launch": round(kern_ms[g], 4)}

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
        h2d = st.input_bytes()
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
        e2e = {"value": round(world * per_step * a.steps / (ems / 1e3), 1), "unit": cfg.unit,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": round(ems / a.steps, 4),
               "path": "public C ABI calls and the step's host transfers captured once in a "
                       "CUDA graph; per step: H2D of the step inputs from pinned memory in one "
                       "block per phase (later phases on a second stream while the earlier "
                       "ones run), the kernels, one D2H of n_accepted and out_tokens, stream "
                       "synchronise"}
    # ---- acceptance telemetry (untimed)
    tele = None
    if cfg.verify and a.telemetry_steps > 0:
        tele = telemetry(st, graph, a.telemetry_steps)
        tele["emitted_tokens_per_s"] = round(world * st.B * tele["mal"] / (ms_step / 1e3), 1)
    clocks = clock.stop()
    status = sd.sd_device_status_read()
    del graph, graph_ev, graph_e2e

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        t = time.perf_counter()
        nv = oracle_sample(st, [0], 0)
        dt = time.perf_counter() - t
        cpu = {"value": round(nv / dt, 4), "unit": cfg.unit, "cores": blas_threads(),
               "kind": "oracle",
               "sample": "sequence 0 of the batch: the workload's full step for it in float64 "
                         "on the host; %.1f s for %d %s" %
                         (dt, nv, "verified positions" if cfg.verify else "drafted tokens")}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": cfg.unit, "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32" if cfg.dtype == "f32" else "bf16", "data": "synthetic",
        "config": config_line(st, a, world),
        "gpu_launches": kernels_per_step * a.steps,
        "roofline": roof(dom),
        "roofline_attention": roof("verify_global") or roof("verify_sliding")
        or roof("xattn_global"),
        "roofline_lm_head": roof("head_dense"),
        "kernels": per_kernel,
        "kernel_busy_ms_per_step": round(busy_ms, 4),
        "kernel_times_note": "per-kernel times come from a second capture of the step with an "
                             "event node around every call; those nodes add time, so the sum "
                             "exceeds ms_per_step and the per-kernel fractions read slightly low",
        "clocks": clocks,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "telemetry": tele,
        "mean_accepted": round(float(((ctx_b - ctx_a) - a.steps).sum()) /
                               max(1, a.steps * st.B), 4) if cfg.verify else None,
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
    cfg = make_cfg(a)
    st = SpecStep(cfg, reserve=64, dev=None)
    for s in range(a.warmup):
        oracle_sample(st, [s % st.B], s)
    t = time.perf_counter()
    nv = 0
    for s in range(a.steps):
        nv += oracle_sample(st, [s % st.B], a.warmup + s)
    dt = time.perf_counter() - t
    value = nv / dt
    line = {"metric": METRIC, "value": round(value, 4), "unit": cfg.unit, "n_gpus": world,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(dt / a.steps * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": cfg.name(), "batch": cfg.B,
                       "ctx": cfg.L if isinstance(cfg.L, int) else list(cfg.L), "k": cfg.k},
            "cpu_baseline": {"value": round(value, 4), "unit": cfg.unit, "cores": blas_threads(),
                             "kind": "oracle",
                             "sample": "per step one sequence of the batch (round robin): the "
                                       "workload's full step for it in float64 on the host"},
            "e2e": {"value": round(value, 4), "unit": cfg.unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


if __name__ == "__main__":
    main()
