"""B200-native speculative-decoding verify step: Python binding of include/sd_verify.h.

Argument marshalling only.  Every step of the path runs in the CUDA kernels of
libsdverify.so (built in-tree by ``python -m verify_step_b200.build``); torch supplies device
memory and streams.  There is no fallback: if the library is missing or a call fails, the
binding raises.

Functions carry the C names (sd_verify_attn, sd_draft_xattn, sd_lm_head, sd_accept,
sd_commit, sd_linear and the *_workspace_size / status helpers).  Tensors are passed as torch CUDA
tensors (their data_ptr is used; they must be contiguous), descriptors as the ctypes
structures below, ``stream`` as a torch.cuda.Stream (default: the current stream).
"""
from __future__ import annotations

import ctypes
import os

from .telemetry import acceptance_telemetry  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsdverify.so")

SD_OK, SD_ERR_INVALID_ARG, SD_ERR_UNSUPPORTED, SD_ERR_WORKSPACE = 0, 1, 2, 3
SD_ERR_CUDA, SD_ERR_TIMEOUT, SD_ERR_DEVICE = 4, 5, 6
SD_F32, SD_BF16 = 0, 1


class SdError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {status_string(status)} (status {status})")


class AttnDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("n_q", ctypes.c_int), ("h_q", ctypes.c_int),
                ("h_kv", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("block_size", ctypes.c_int), ("max_blocks_per_seq", ctypes.c_int),
                ("num_blocks", ctypes.c_int), ("window", ctypes.c_int),
                ("scale", ctypes.c_float), ("dtype", ctypes.c_int),
                ("q_offset", ctypes.c_int)]


class HeadDesc(ctypes.Structure):
    _fields_ = [("m", ctypes.c_int), ("d", ctypes.c_int), ("vocab", ctypes.c_int),
                ("ld_logits", ctypes.c_int), ("n_clusters", ctypes.c_int),
                ("cluster_size", ctypes.c_int), ("top_c", ctypes.c_int),
                ("dtype", ctypes.c_int)]


class AcceptDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("k", ctypes.c_int), ("vocab", ctypes.c_int),
                ("temperature", ctypes.c_float), ("seed", ctypes.c_uint64),
                ("step", ctypes.c_uint64), ("purpose", ctypes.c_int),
                ("ld_target", ctypes.c_int), ("ld_draft", ctypes.c_int),
                ("ld_out", ctypes.c_int), ("step_ptr", ctypes.c_void_p)]


class PoisonCache(ctypes.Structure):
    _fields_ = [("cache", ctypes.c_void_p), ("h_kv", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("dtype", ctypes.c_int)]


class CommitDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("k", ctypes.c_int), ("block_size", ctypes.c_int),
                ("max_blocks_per_seq", ctypes.c_int), ("num_blocks", ctypes.c_int),
                ("d", ctypes.c_int), ("hidden_dtype", ctypes.c_int),
                ("n_poison", ctypes.c_int), ("poison", ctypes.POINTER(PoisonCache)),
                ("step_ptr", ctypes.c_void_p)]


SD_EPI_STORE, SD_EPI_ADD, SD_EPI_GEGLU = 0, 1, 2


class LinearDesc(ctypes.Structure):
    _fields_ = [("m", ctypes.c_int), ("n", ctypes.c_int), ("k", ctypes.c_int),
                ("x_dtype", ctypes.c_int), ("ld_x", ctypes.c_int64), ("k_gather", ctypes.c_int),
                ("ld_table", ctypes.c_int64), ("table_rows", ctypes.c_int64),
                ("ld_tokens", ctypes.c_int64), ("norm_gain", ctypes.c_void_p),
                ("norm_eps", ctypes.c_float), ("epilogue", ctypes.c_int),
                ("out_dtype", ctypes.c_int), ("ld_out", ctypes.c_int64),
                ("norm_out", ctypes.c_void_p), ("ld_norm_out", ctypes.c_int64),
                ("ws", ctypes.c_void_p), ("ws_bytes", ctypes.c_size_t)]


_lib = None

_P = ctypes.c_void_p
_SIGS = {
    "sd_verify_attn_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(AttnDesc)]),
    "sd_verify_attn": (ctypes.c_int, [ctypes.POINTER(AttnDesc), _P, _P, _P, _P, _P, _P, _P, _P,
                                      _P, ctypes.c_size_t, _P]),
    "sd_draft_xattn_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(AttnDesc)]),
    "sd_draft_xattn": (ctypes.c_int, [ctypes.POINTER(AttnDesc), _P, _P, _P, _P, _P, _P, _P, _P,
                                      ctypes.c_size_t, _P]),
    "sd_lm_head_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(HeadDesc)]),
    "sd_lm_head": (ctypes.c_int, [ctypes.POINTER(HeadDesc), _P, _P, _P, _P, _P, _P, _P,
                                  ctypes.c_size_t, _P]),
    "sd_accept_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(AcceptDesc)]),
    "sd_accept": (ctypes.c_int, [ctypes.POINTER(AcceptDesc), _P, _P, _P, _P, _P, _P, _P,
                                 ctypes.c_size_t, _P]),
    "sd_accept_noalloc": (ctypes.c_int, [ctypes.POINTER(AcceptDesc), _P, _P, _P, _P, _P, _P,
                                         _P]),
    "sd_commit": (ctypes.c_int, [ctypes.POINTER(CommitDesc), _P, _P, _P, _P, _P, _P, _P]),
    "sd_linear_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(LinearDesc)]),
    "sd_linear": (ctypes.c_int, [ctypes.POINTER(LinearDesc), _P, _P, _P, _P, _P, _P, _P]),
    "sd_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "sd_device_status_read": (ctypes.c_int, [ctypes.POINTER(ctypes.c_int), _P]),
    "sd_device_status_clear": (ctypes.c_int, [_P]),
    "sd_selftest_bounded_wait": (ctypes.c_int, [_P]),
    "sd_version": (ctypes.c_int, []),
}


def lib() -> ctypes.CDLL:
    """The loaded CUDA library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m verify_step_b200.build` (no fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def exported_symbols():
    return list(_SIGS)


def status_string(status: int) -> str:
    return lib().sd_status_string(int(status)).decode()


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("tensor arguments must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor arguments must be contiguous")
    return t.data_ptr()


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _nbytes(t):
    return 0 if t is None else t.numel() * t.element_size()


def _check(fn, status):
    if status != SD_OK:
        raise SdError(fn, status)


def sd_verify_attn_workspace_size(desc: AttnDesc) -> int:
    return lib().sd_verify_attn_workspace_size(ctypes.byref(desc))


def sd_draft_xattn_workspace_size(desc: AttnDesc) -> int:
    return lib().sd_draft_xattn_workspace_size(ctypes.byref(desc))


def sd_lm_head_workspace_size(desc: HeadDesc) -> int:
    return lib().sd_lm_head_workspace_size(ctypes.byref(desc))


def sd_accept_workspace_size(desc: AcceptDesc) -> int:
    return lib().sd_accept_workspace_size(ctypes.byref(desc))


def sd_verify_attn(desc, q, k_new, v_new, k_cache, v_cache, block_table, ctx_len, out, ws,
                   stream=None):
    _check("sd_verify_attn", lib().sd_verify_attn(
        ctypes.byref(desc), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
        _ptr(block_table), _ptr(ctx_len), _ptr(out), _ptr(ws), _nbytes(ws), _stream(stream)))


def sd_draft_xattn(desc, q, k_cache, v_cache, block_table, ctx_len, q_pos, out, ws,
                   stream=None):
    _check("sd_draft_xattn", lib().sd_draft_xattn(
        ctypes.byref(desc), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
        _ptr(ctx_len), _ptr(q_pos), _ptr(out), _ptr(ws), _nbytes(ws), _stream(stream)))


def sd_lm_head(desc, h, w, logits, centroids=None, cluster_tokens=None, sel_clusters=None,
               ws=None, stream=None):
    _check("sd_lm_head", lib().sd_lm_head(
        ctypes.byref(desc), _ptr(h), _ptr(w), _ptr(centroids), _ptr(cluster_tokens),
        _ptr(logits), _ptr(sel_clusters), _ptr(ws), _nbytes(ws), _stream(stream)))


def sd_accept(desc, target_logits, draft_logits, draft_tokens, n_accepted, out_tokens,
              margin_flags, ws, stream=None):
    _check("sd_accept", lib().sd_accept(
        ctypes.byref(desc), _ptr(target_logits), _ptr(draft_logits), _ptr(draft_tokens),
        _ptr(n_accepted), _ptr(out_tokens), _ptr(margin_flags), _ptr(ws), _nbytes(ws),
        _stream(stream)))


def sd_accept_noalloc(desc, target_logits, draft_logits, draft_tokens, n_accepted, out_tokens,
                      margin_flags, stream=None):
    """sd_accept without a caller workspace: the library's fixed scratch array is used (see
    include/sd_verify.h for its size limit and the rule that overlapping calls race)."""
    _check("sd_accept_noalloc", lib().sd_accept_noalloc(
        ctypes.byref(desc), _ptr(target_logits), _ptr(draft_logits), _ptr(draft_tokens),
        _ptr(n_accepted), _ptr(out_tokens), _ptr(margin_flags), _stream(stream)))


def sd_commit(desc, block_table, ctx_len, n_accepted, committed_slots, hidden=None,
              next_hidden=None, stream=None):
    _check("sd_commit", lib().sd_commit(
        ctypes.byref(desc), _ptr(block_table), _ptr(ctx_len), _ptr(n_accepted),
        _ptr(committed_slots), _ptr(hidden), _ptr(next_hidden), _stream(stream)))


def sd_linear_workspace_size(desc: LinearDesc) -> int:
    return lib().sd_linear_workspace_size(ctypes.byref(desc))


def sd_linear(desc, x, w, out, table=None, tokens=None, token_sel=None, stream=None, ws=None):
    """One projection; ``ws`` (a device tensor or address), when given, is set as the
    descriptor's workspace (its size in bytes from the tensor)."""
    if ws is not None:
        desc.ws = _ptr(ws)
        desc.ws_bytes = ws.numel() * ws.element_size() if hasattr(ws, "numel") else desc.ws_bytes
    _check("sd_linear", lib().sd_linear(
        ctypes.byref(desc), _ptr(x), _ptr(w), _ptr(out), _ptr(table), _ptr(tokens),
        _ptr(token_sel), _stream(stream)))


def sd_device_status_read(stream=None) -> int:
    v = ctypes.c_int(0)
    _check("sd_device_status_read", lib().sd_device_status_read(ctypes.byref(v),
                                                                _stream(stream)))
    return v.value


def sd_device_status_clear(stream=None):
    _check("sd_device_status_clear", lib().sd_device_status_clear(_stream(stream)))


def sd_selftest_bounded_wait(stream=None):
    _check("sd_selftest_bounded_wait", lib().sd_selftest_bounded_wait(_stream(stream)))


def sd_version() -> int:
    return lib().sd_version()


def poison_list(caches):
    """ctypes array of PoisonCache for sd_commit from (tensor, h_kv, head_dim, dtype) tuples."""
    arr = (PoisonCache * len(caches))()
    for i, (t, h_kv, hd, dt) in enumerate(caches):
        arr[i] = PoisonCache(_ptr(t), h_kv, hd, dt)
    return arr
