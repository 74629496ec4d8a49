"""The target's layers over the k+1 verified positions, as a sequence of library calls.

"Gemma 4 MTP: drafter drafts, target verifies", section "drafter internal architecture": the
target checks the k drafts plus one position in one forward pass; Gemma 4 MTP serving guide,
section 7: its layers mix sliding-window (head_dim 256) and global (head_dim 512) attention.
This module only marshals arguments: every step is an ``sd_linear`` or ``sd_verify_attn`` call
of the CUDA library (no arithmetic here).

Per layer, over the residual stream x [B (k+1), d] (f32, updated in place):

  sd_linear       q = W_q a, k_new = W_k a, v_new = W_v a,  a = rmsnorm(x, g_attn)   (bf16)
  sd_verify_attn  o = attention of the k+1 positions; k_new, v_new appended to the cache
  sd_linear       x += W_o o
                  u = gelu(W_g m) * (W_u m),  m = rmsnorm(x, g_mlp)                   (bf16)
                  x += W_d u
"""
from __future__ import annotations

from dataclasses import dataclass

from . import (SD_BF16, SD_EPI_ADD, SD_EPI_GEGLU, SD_EPI_STORE, SD_F32, sd_linear,
               sd_verify_attn)
from .drafter import gate_up_blocks, linear_desc, workspace_bytes


@dataclass
class TargetShape:
    batch: int
    n_q: int          # k + 1 verified positions per sequence
    d: int            # model width
    ff: int           # gated-MLP width
    h_q: int
    h_kv: int
    layers: tuple     # ((head_dim, window), ...), window 0 for a global layer


def device_weights(host, dev="cuda"):
    """Device copies of per-layer weight dicts (g_attn, Wq, Wk, Wv, Wo, g_mlp, Wg, Wu, Wd) with
    the gate and up rows fused by gate_up_blocks."""
    g = lambda t: t.contiguous().to(dev)
    return [{"g_attn": g(L["g_attn"]), "Wq": g(L["Wq"]), "Wk": g(L["Wk"]), "Wv": g(L["Wv"]),
             "Wo": g(L["Wo"]), "g_mlp": g(L["g_mlp"]),
             "Wgu": g(gate_up_blocks(L["Wg"], L["Wu"])), "Wd": g(L["Wd"])} for L in host]


def call_shapes(shape: TargetShape):
    """(m, n, k) of every layer's sd_linear calls."""
    m, d, F = shape.batch * shape.n_q, shape.d, shape.ff
    out = []
    for D, _ in shape.layers:
        nq, nkv = shape.h_q * D, shape.h_kv * D
        out += [(m, nq, d), (m, nkv, d), (m, d, nq), (m, 2 * F, d), (m, d, F)]
    return out


def buffers(shape: TargetShape, dev="cuda"):
    """The residual stream, per-layer activation buffers and the sd_linear workspace."""
    import torch
    m = shape.batch * shape.n_q
    bf = torch.bfloat16
    mk = lambda n: torch.empty((m, n), dtype=bf, device=dev)
    return {"ws": torch.empty(max(256, workspace_bytes(call_shapes(shape))), dtype=torch.uint8,
                              device=dev),
            "x": torch.empty((m, shape.d), dtype=torch.float32, device=dev),
            "q": [mk(shape.h_q * D) for D, _ in shape.layers],
            "k": [mk(shape.h_kv * D) for D, _ in shape.layers],
            "v": [mk(shape.h_kv * D) for D, _ in shape.layers],
            "o": [mk(shape.h_q * D) for D, _ in shape.layers],
            "u": mk(shape.ff)}


def verify_layers(shape: TargetShape, wts, buf, caches, ctx_len, ws, stream=None, wrap=None):
    """Run every layer on buf["x"] (the caller fills it with the k+1 positions' input rows).

    caches[i]: dict(desc=AttnDesc with n_q = shape.n_q, k=k_cache, v=v_cache, table=block
    table) of layer i; ctx_len int32 [B] (not advanced: sd_commit does that); ws the attention
    workspace.  wrap(kind, fn) optionally runs each call (kind "linear" or "attn")."""
    m, d, F = shape.batch * shape.n_q, shape.d, shape.ff
    x = buf["x"]
    call = wrap if wrap is not None else (lambda kind, fn: fn())
    lws = buf.get("ws")

    def sd_linear_ws(*args, **kw):
        return sd_linear(*args, ws=lws, **kw)

    desc = linear_desc
    for i, (L, (D, _W)) in enumerate(zip(wts, shape.layers)):
        nq, nkv = shape.h_q * D, shape.h_kv * D
        q, kn, vn, o = buf["q"][i], buf["k"][i], buf["v"][i], buf["o"][i]
        gain = L["g_attn"].data_ptr()
        # each call's arguments are bound when its closure is made, so a wrap that defers the
        # call still issues this layer's projection
        for W, out, n in ((L["Wq"], q, nq), (L["Wk"], kn, nkv), (L["Wv"], vn, nkv)):
            call("linear", lambda W=W, out=out, n=n, gain=gain: sd_linear_ws(
                desc(m, n, d, SD_F32, d, SD_EPI_STORE, SD_BF16, n, norm_gain=gain), x, W, out,
                stream=stream))
        c = caches[i]
        call("attn", lambda c=c, q=q, kn=kn, vn=vn, o=o: sd_verify_attn(
            c["desc"], q, kn, vn, c["k"], c["v"], c["table"], ctx_len, o, ws, stream=stream))
        call("linear", lambda L=L, o=o, nq=nq: sd_linear_ws(
            desc(m, d, nq, SD_BF16, nq, SD_EPI_ADD, SD_F32, d), o, L["Wo"], x, stream=stream))
        call("linear", lambda L=L: sd_linear_ws(
            desc(m, 2 * F, d, SD_F32, d, SD_EPI_GEGLU, SD_BF16, F,
                 norm_gain=L["g_mlp"].data_ptr()), x, L["Wgu"], buf["u"], stream=stream))
        call("linear", lambda L=L: sd_linear_ws(desc(m, d, F, SD_BF16, F, SD_EPI_ADD, SD_F32, d),
                                             buf["u"], L["Wd"], x, stream=stream))


LINEAR_CALLS_PER_LAYER = 6
