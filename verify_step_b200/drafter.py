"""One link of the drafter chain as a sequence of library calls.

"Gemma 4 MTP: drafter drafts, target verifies", section "drafter internal architecture": the
drafter projects the target's last-layer activation together with its own embedding of the last
token, runs 4 transformer layers (3 sliding-window, 1 global) whose attention reads the target's
KV cache, and hands its output row to its LM head; Gemma 4 MTP serving guide, section 4: the
links form a chain.  This module only marshals arguments: every step is an ``sd_linear`` or
``sd_draft_xattn`` call of the CUDA library (no arithmetic here).

Per link (B token rows, drafter width d, target width d_t):

  sd_linear  x      = W_in [h_prev ; E[token]]                      (f32 residual stream)
  per layer  q      = W_q rmsnorm(x, g_attn)                        (bf16)
             o      = sd_draft_xattn(q)                             (caller's callback)
             x     += W_o o
             u      = gelu(W_g m) * (W_u m),  m = rmsnorm(x, g_mlp)  (bf16, gated epilogue)
             x     += W_d u
  sd_linear  h      = rmsnorm(x, g_final)  (the LM head's input, written by the prologue)
             h_back = W_back h                                      (next link's activation)
"""
from __future__ import annotations

from dataclasses import dataclass

from . import (SD_BF16, SD_EPI_ADD, SD_EPI_GEGLU, SD_EPI_STORE, SD_F32, LinearDesc,
               sd_linear, sd_linear_workspace_size)

RMS_EPS = 1e-6


@dataclass
class DrafterShape:
    batch: int
    d: int            # drafter width
    d_target: int     # target width (the activation fed to the first link)
    ff: int           # gated-MLP width
    h_q: int
    head_dims: tuple  # per layer, e.g. (256, 256, 256, 512)
    vocab: int        # rows of the embedding table


def gate_up_blocks(Wg, Wu):
    """The row layout sd_linear's gated epilogue reads (torch tensors [ff, d] -> [2 ff, d]):
    blocks of 16 rows, the 8 gate rows of features 8t .. 8t+7 followed by their 8 up rows.
    A pure reordering of rows."""
    import torch
    ff, d = Wg.shape
    if tuple(Wu.shape) != (ff, d) or ff % 8:
        raise ValueError("gate and up weights must both be [ff, d] with ff a multiple of 8")
    return torch.stack([Wg.reshape(ff // 8, 8, d), Wu.reshape(ff // 8, 8, d)],
                       dim=1).reshape(2 * ff, d).contiguous()


def device_weights(host, dev="cuda"):
    """Device copies of a weight dict (E, W_in, g_final, W_back and per layer g_attn, Wq, Wo,
    g_mlp, Wg, Wu, Wd) with each layer's gate and up rows fused by gate_up_blocks."""
    g = lambda t: t.contiguous().to(dev)
    out = {k: g(host[k]) for k in ("E", "W_in", "g_final", "W_back")}
    out["layers"] = [{"g_attn": g(L["g_attn"]), "Wq": g(L["Wq"]), "Wo": g(L["Wo"]),
                      "g_mlp": g(L["g_mlp"]), "Wgu": g(gate_up_blocks(L["Wg"], L["Wu"])),
                      "Wd": g(L["Wd"])} for L in host["layers"]]
    return out


def call_shapes(shape: DrafterShape):
    """(m, n, k) of the link's sd_linear calls."""
    B, d, dt, F = shape.batch, shape.d, shape.d_target, shape.ff
    out = [(B, d, dt + d)]
    for D in shape.head_dims:
        n = shape.h_q * D
        out += [(B, n, d), (B, d, n), (B, 2 * F, d), (B, d, F)]
    out.append((B, dt, d))
    return out


def workspace_bytes(shapes):
    """The largest sd_linear workspace over calls of the given (m, n, k) shapes."""
    return max(sd_linear_workspace_size(LinearDesc(m=m, n=n, k=k)) for m, n, k in shapes)


def buffers(shape: DrafterShape, dev="cuda"):
    """Activation buffers of one link (reused by every link) and the sd_linear workspace."""
    import torch
    B = shape.batch
    bf, f32 = torch.bfloat16, torch.float32
    return {"ws": torch.empty(max(256, workspace_bytes(call_shapes(shape))), dtype=torch.uint8,
                              device=dev),
            "x": torch.empty((B, shape.d), dtype=f32, device=dev),
            "q": [torch.empty((B, shape.h_q * D), dtype=bf, device=dev) for D in shape.head_dims],
            "o": [torch.empty((B, shape.h_q * D), dtype=bf, device=dev) for D in shape.head_dims],
            "u": torch.empty((B, shape.ff), dtype=bf, device=dev),
            "h": torch.empty((B, shape.d), dtype=bf, device=dev),
            "h_back": torch.empty((B, shape.d_target), dtype=bf, device=dev)}


def linear_desc(m, n, k, x_dtype, ld_x, epilogue, out_dtype, ld_out, **kw):
    """An sd_linear descriptor with the RMSNorm epsilon of these layers."""
    return LinearDesc(m=m, n=n, k=k, x_dtype=x_dtype, ld_x=ld_x, epilogue=epilogue,
                      out_dtype=out_dtype, ld_out=ld_out, norm_eps=RMS_EPS, **kw)


def link(shape: DrafterShape, wts, buf, h_prev, tokens, ld_tokens, attend, token_sel=None,
         stream=None, wrap=None):
    """Issue one link on the stream.

    h_prev     bf16 [B, d_target] (device tensor or address)
    tokens     int32 token ids; row r reads tokens[r * ld_tokens + (token_sel[r] or 0)]
    attend(i, q, o)  issues layer i's cross-attention from q into o (sd_draft_xattn)
    wrap(fn)   optional: runs fn, which issues one sd_linear call (e.g. between timing events)
    Results: buf["h"] (the LM head's input) and buf["h_back"] (the next link's activation)."""
    B, d, dt, F = shape.batch, shape.d, shape.d_target, shape.ff
    x = buf["x"]
    call = wrap if wrap is not None else (lambda fn: fn())
    ws = buf.get("ws")

    def sd_linear_ws(*args, **kw):
        return sd_linear(*args, ws=ws, **kw)

    desc = linear_desc
    call(lambda: sd_linear_ws(
        desc(B, d, dt + d, SD_BF16, dt, SD_EPI_STORE, SD_F32, d, k_gather=d, ld_table=d,
             table_rows=shape.vocab, ld_tokens=ld_tokens),
        h_prev, wts["W_in"], x, table=wts["E"], tokens=tokens, token_sel=token_sel,
        stream=stream))
    # each call's arguments are bound when its closure is made, so a wrap that defers the call
    # still issues this layer's projection
    for i, (L, D) in enumerate(zip(wts["layers"], shape.head_dims)):
        n = shape.h_q * D
        q, o = buf["q"][i], buf["o"][i]
        call(lambda L=L, n=n, q=q: sd_linear_ws(desc(B, n, d, SD_F32, d, SD_EPI_STORE, SD_BF16, n,
                                                  norm_gain=L["g_attn"].data_ptr()),
                                             x, L["Wq"], q, stream=stream))
        attend(i, q, o)
        call(lambda L=L, n=n, o=o: sd_linear_ws(desc(B, d, n, SD_BF16, n, SD_EPI_ADD, SD_F32, d),
                                             o, L["Wo"], x, stream=stream))
        call(lambda L=L: sd_linear_ws(desc(B, 2 * F, d, SD_F32, d, SD_EPI_GEGLU, SD_BF16, F,
                                        norm_gain=L["g_mlp"].data_ptr()),
                                   x, L["Wgu"], buf["u"], stream=stream))
        call(lambda L=L: sd_linear_ws(desc(B, d, F, SD_BF16, F, SD_EPI_ADD, SD_F32, d), buf["u"],
                                   L["Wd"], x, stream=stream))
    call(lambda: sd_linear_ws(desc(B, dt, d, SD_F32, d, SD_EPI_STORE, SD_BF16, dt,
                                norm_gain=wts["g_final"].data_ptr(),
                                norm_out=buf["h"].data_ptr(), ld_norm_out=d),
                           x, wts["W_back"], buf["h_back"], stream=stream))


def hbm_bytes_per_link(shape: DrafterShape):
    """Algorithmic HBM bytes of the link's sd_linear calls: every weight once, the input rows
    read, the outputs written (the residual stream read and written by the adding calls)."""
    B, d, dt, F = shape.batch, shape.d, shape.d_target, shape.ff
    total = d * (dt + d) * 2 + B * (dt * 2 + d * 2) + B * d * 4          # W_in
    for D in shape.head_dims:
        n = shape.h_q * D
        total += n * d * 2 + B * d * 4 + B * n * 2                       # W_q
        total += d * n * 2 + B * n * 2 + 2 * B * d * 4                   # W_o (+= x)
        total += 2 * F * d * 2 + B * d * 4 + B * F * 2                   # gate and up
        total += d * F * 2 + B * F * 2 + 2 * B * d * 4                   # W_d (+= x)
    total += dt * d * 2 + B * d * 4 + B * dt * 2 + B * d * 2             # W_back, h
    return total


LAUNCHES_PER_LINK = 2 + 4 * 4  # input and output projections + 4 per layer (attention apart)
