"""Host logic of the drafter link (no GPU): the gate/up row layout and the sequence of library
calls one link issues, with the library call replaced by a recorder."""
import pytest
import torch

import verify_step_b200 as sd
from verify_step_b200 import drafter as VD


def test_gate_up_blocks_layout():
    ff, d = 24, 3
    Wg = torch.arange(ff * d, dtype=torch.float32).reshape(ff, d)
    Wu = -Wg - 1
    W = VD.gate_up_blocks(Wg, Wu)
    assert W.shape == (2 * ff, d)
    for t in range(ff // 8):
        for i in range(8):
            assert torch.equal(W[16 * t + i], Wg[8 * t + i])
            assert torch.equal(W[16 * t + 8 + i], Wu[8 * t + i])
    with pytest.raises(ValueError):
        VD.gate_up_blocks(Wg[:12], Wu[:12])


class _T:
    """Stand-in for a device tensor: only data_ptr is read by the link."""
    def __init__(self, addr):
        self.addr = addr

    def data_ptr(self):
        return self.addr


def test_link_call_sequence(monkeypatch):
    calls = []
    monkeypatch.setattr(VD, "sd_linear", lambda desc, x, w, out, **kw: calls.append(
        (sd.LinearDesc.from_buffer_copy(desc), x, w, out, kw)))
    shape = VD.DrafterShape(batch=8, d=1024, d_target=5376, ff=4096, h_q=16,
                            head_dims=(256, 256, 256, 512), vocab=262144)
    n = iter(range(1000, 10 ** 6, 16))
    wts = {k: _T(next(n)) for k in ("E", "W_in", "g_final", "W_back")}
    wts["layers"] = [{k: _T(next(n)) for k in ("g_attn", "Wq", "Wo", "g_mlp", "Wgu", "Wd")}
                     for _ in range(4)]
    buf = {"x": _T(1), "u": _T(2), "h": _T(3), "h_back": _T(4),
           "q": [_T(10 + i) for i in range(4)], "o": [_T(20 + i) for i in range(4)]}
    att = []
    VD.link(shape, wts, buf, "h_prev", "toks", 3, lambda i, q, o: att.append((i, q, o)),
            token_sel="sel")
    assert len(calls) == VD.LAUNCHES_PER_LINK == 18
    assert [a[0] for a in att] == [0, 1, 2, 3]
    first = calls[0][0]
    assert (first.m, first.n, first.k, first.k_gather, first.ld_x) == (8, 1024, 6400, 1024, 5376)
    assert first.table_rows == 262144 and first.ld_tokens == 3 and calls[0][4]["token_sel"] == "sel"
    for i, D in enumerate(shape.head_dims):
        q, o, gu, dn = calls[1 + 4 * i: 5 + 4 * i]
        assert (q[0].n, q[0].k, q[0].epilogue, q[0].norm_gain) == (16 * D, 1024, sd.SD_EPI_STORE,
                                                                   wts["layers"][i]["g_attn"].addr)
        assert q[3] is buf["q"][i] and att[i][1] is buf["q"][i] and o[1] is buf["o"][i]
        assert (o[0].n, o[0].k, o[0].epilogue, o[0].out_dtype) == (1024, 16 * D, sd.SD_EPI_ADD,
                                                                   sd.SD_F32)
        assert (gu[0].n, gu[0].epilogue, gu[0].ld_out) == (8192, sd.SD_EPI_GEGLU, 4096)
        assert (dn[0].n, dn[0].k, dn[0].epilogue) == (1024, 4096, sd.SD_EPI_ADD)
        assert o[3] is buf["x"] and dn[3] is buf["x"]
    last = calls[-1][0]
    assert (last.n, last.k, last.norm_out, last.ld_norm_out) == (5376, 1024, 3, 1024)
    assert calls[-1][3] is buf["h_back"]
