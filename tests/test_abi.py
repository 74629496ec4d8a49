"""The C ABI: the library builds, loads and exports every entry point the header declares;
host-side validation rejects bad descriptors before any device work (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import pytest

import verify_step_b200 as sd
from verify_step_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return sd.lib()


def declared_functions():
    names = set()
    inc = os.path.join(ROOT, "include")
    for f in os.listdir(inc):
        if f.endswith(".h"):
            text = open(os.path.join(inc, f)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(sd_\w+)\s*\(", text))
    return sorted(names)


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert "sd_verify_attn" in names and "sd_commit" in names and len(names) >= 13
    out = subprocess.run(["nm", "-D", "--defined-only", sd.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    # the binding covers every entry point
    assert set(names) <= set(sd.exported_symbols())


def test_status_strings(lib):
    assert sd.status_string(0) == "ok"
    assert "workspace" in sd.status_string(3)
    assert sd.sd_version() >= 100


def test_validation_rejects_bad_descriptors(lib):
    L = lib
    # null descriptor
    assert L.sd_verify_attn(None, *([None] * 8), None, 0, None) == sd.SD_ERR_INVALID_ARG
    # h_q not a multiple of h_kv
    d = sd.AttnDesc(batch=1, n_q=3, h_q=5, h_kv=2, head_dim=256, block_size=16,
                    max_blocks_per_seq=4, num_blocks=4, window=0, scale=0.1, dtype=sd.SD_BF16)
    assert L.sd_verify_attn(ctypes.byref(d), *([None] * 8), None, 0, None) == sd.SD_ERR_INVALID_ARG
    # unsupported head_dim for bf16
    d.h_q, d.head_dim = 4, 96
    assert L.sd_verify_attn(ctypes.byref(d), *([None] * 8), None, 0, None) == sd.SD_ERR_UNSUPPORTED
    # drafter needs n_q == 1
    d.head_dim = 256
    assert L.sd_draft_xattn(ctypes.byref(d), *([None] * 7), None, 0, None) == sd.SD_ERR_INVALID_ARG
    # block size must be a multiple of 16 for bf16
    d.n_q, d.block_size = 1, 8
    assert L.sd_draft_xattn(ctypes.byref(d), *([None] * 7), None, 0, None) == sd.SD_ERR_UNSUPPORTED
    # too many rows per kv head
    d.block_size, d.h_q, d.h_kv, d.n_q = 16, 32, 1, 3
    assert L.sd_verify_attn(ctypes.byref(d), *([None] * 8), None, 0, None) == sd.SD_ERR_UNSUPPORTED
    # LM head: d not a multiple of 64 in bf16; clustered sizes inconsistent
    h = sd.HeadDesc(m=4, d=100, vocab=1024, ld_logits=0, n_clusters=0, cluster_size=0, top_c=0,
                    dtype=sd.SD_BF16)
    assert L.sd_lm_head(ctypes.byref(h), *([None] * 6), None, 0, None) == sd.SD_ERR_UNSUPPORTED
    h.d, h.top_c, h.n_clusters, h.cluster_size = 128, 4, 10, 100
    assert L.sd_lm_head(ctypes.byref(h), *([None] * 6), None, 0, None) == sd.SD_ERR_INVALID_ARG
    h.ld_logits, h.top_c = 10, 0
    assert L.sd_lm_head(ctypes.byref(h), *([None] * 6), None, 0, None) == sd.SD_ERR_INVALID_ARG
    # accept: k out of range, bad purpose, negative temperature, ragged vocab
    a = sd.AcceptDesc(batch=2, k=16, vocab=1024, temperature=1.0, seed=0, step=0, purpose=1)
    assert L.sd_accept(ctypes.byref(a), *([None] * 6), None, 0, None) == sd.SD_ERR_INVALID_ARG
    a.k, a.purpose = 2, 0
    assert L.sd_accept(ctypes.byref(a), *([None] * 6), None, 0, None) == sd.SD_ERR_INVALID_ARG
    a.purpose, a.temperature = 1, -1.0
    assert L.sd_accept(ctypes.byref(a), *([None] * 6), None, 0, None) == sd.SD_ERR_INVALID_ARG
    a.temperature, a.vocab = 1.0, 1001
    assert L.sd_accept(ctypes.byref(a), *([None] * 6), None, 0, None) == sd.SD_ERR_UNSUPPORTED
    # accept workspace grows with batch and vocabulary
    a.vocab = 262144
    w1 = L.sd_accept_workspace_size(ctypes.byref(a))
    a.batch = 64
    assert L.sd_accept_workspace_size(ctypes.byref(a)) > w1 > 0
    # commit: null pointers, too many poison caches
    c = sd.CommitDesc(batch=2, k=2, block_size=16, max_blocks_per_seq=4, num_blocks=8)
    assert L.sd_commit(ctypes.byref(c), *([None] * 6), None) == sd.SD_ERR_INVALID_ARG
    assert L.sd_commit(None, *([None] * 6), None) == sd.SD_ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors(lib):
    import torch
    d = sd.HeadDesc(m=1, d=64, vocab=64, dtype=sd.SD_F32)
    with pytest.raises(ValueError):
        sd._ptr(torch.zeros(4))
    with pytest.raises(ValueError):
        sd._ptr(torch.zeros(4, 4).t())
    assert d.m == 1


def test_linear_validation(lib):
    L = lib
    A = 4096  # any 16-byte aligned non-null address: every case below is refused before a launch
    assert L.sd_linear(None, None, None, None, None, None, None, None) == sd.SD_ERR_INVALID_ARG
    d = sd.LinearDesc(m=0, n=32, k=64, x_dtype=sd.SD_BF16, ld_x=64, epilogue=sd.SD_EPI_STORE,
                      out_dtype=sd.SD_F32, ld_out=32)
    # an empty batch launches nothing
    assert L.sd_linear(ctypes.byref(d), None, None, None, None, None, None, None) == sd.SD_OK
    d.m = 8
    assert L.sd_linear(ctypes.byref(d), None, A, A, None, None, None, None) == sd.SD_ERR_INVALID_ARG
    for field, value, want in (("m", 65, sd.SD_ERR_UNSUPPORTED), ("n", 40, sd.SD_ERR_UNSUPPORTED),
                               ("k", 48, sd.SD_ERR_UNSUPPORTED), ("ld_x", 62, sd.SD_ERR_INVALID_ARG),
                               ("ld_out", 16, sd.SD_ERR_INVALID_ARG),
                               ("x_dtype", 7, sd.SD_ERR_INVALID_ARG)):
        e = sd.LinearDesc.from_buffer_copy(d)
        setattr(e, field, value)
        if field == "k":
            e.ld_x = 48
        assert L.sd_linear(ctypes.byref(e), A, A, A, None, None, None, None) == want, field
    # misaligned x or W
    assert L.sd_linear(ctypes.byref(d), A + 8, A, A, None, None, None, None) == sd.SD_ERR_INVALID_ARG
    assert L.sd_linear(ctypes.byref(d), A, A + 2, A, None, None, None, None) == sd.SD_ERR_INVALID_ARG
    # epilogue / output type pairs
    e = sd.LinearDesc.from_buffer_copy(d)
    e.epilogue, e.out_dtype = sd.SD_EPI_ADD, sd.SD_BF16
    assert L.sd_linear(ctypes.byref(e), A, A, A, None, None, None, None) == sd.SD_ERR_INVALID_ARG
    e.epilogue, e.out_dtype = sd.SD_EPI_GEGLU, sd.SD_F32
    assert L.sd_linear(ctypes.byref(e), A, A, A, None, None, None, None) == sd.SD_ERR_INVALID_ARG
    # normalised copy without a gain; gather without a table
    e = sd.LinearDesc.from_buffer_copy(d)
    e.norm_out, e.ld_norm_out = A, 64
    assert L.sd_linear(ctypes.byref(e), A, A, A, None, None, None, None) == sd.SD_ERR_INVALID_ARG
    e = sd.LinearDesc.from_buffer_copy(d)
    e.k_gather, e.ld_x, e.ld_table, e.table_rows = 32, 32, 32, 100
    assert L.sd_linear(ctypes.byref(e), A, A, A, None, A, None, None) == sd.SD_ERR_INVALID_ARG
    e.k_gather = 12
    assert L.sd_linear(ctypes.byref(e), A, A, A, A, A, None, None) == sd.SD_ERR_UNSUPPORTED


def test_descriptor_layouts_match_the_header(tmp_path):
    """The ctypes descriptors have the C structs' size and field offsets (gcc on the header)."""
    structs = {"sd_attn_desc": sd.AttnDesc, "sd_head_desc": sd.HeadDesc,
               "sd_accept_desc": sd.AcceptDesc, "sd_commit_desc": sd.CommitDesc,
               "sd_poison_cache": sd.PoisonCache, "sd_linear_desc": sd.LinearDesc}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "sd_verify.h"',
             'int main(void) {']
    for cname, py in structs.items():
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for fname, _ in py._fields_:
            lines.append(f'  printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    lines += ['  return 0;', '}']
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                   check=True)
    got = {}
    for line in subprocess.run([str(exe)], capture_output=True, text=True,
                               check=True).stdout.splitlines():
        cname, fname, v = line.split()
        got[(cname, fname)] = int(v)
    for cname, py in structs.items():
        assert got[(cname, "size")] == ctypes.sizeof(py), cname
        for fname, _ in py._fields_:
            assert got[(cname, fname)] == getattr(py, fname).offset, (cname, fname)
