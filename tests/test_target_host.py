"""Host logic of the multi-layer verify (no GPU): the calls one layer issues, with the library
calls replaced by recorders."""
import verify_step_b200 as sd
from verify_step_b200 import target as VT


class _T:
    def __init__(self, addr):
        self.addr = addr

    def data_ptr(self):
        return self.addr


def test_layer_call_sequence(monkeypatch):
    calls = []
    monkeypatch.setattr(VT, "sd_linear", lambda desc, x, w, out, **kw: calls.append(
        ("linear", sd.LinearDesc.from_buffer_copy(desc), x, w, out)))
    monkeypatch.setattr(VT, "sd_verify_attn", lambda desc, q, kn, vn, kc, vc, t, ctx, o, ws, **kw:
                        calls.append(("attn", desc, q, kn, vn, kc, vc, t, ctx, o, ws)))
    shape = VT.TargetShape(batch=8, n_q=3, d=5376, ff=21504, h_q=16, h_kv=4,
                           layers=((256, 512), (512, 0)))
    n = iter(range(1000, 10 ** 6, 16))
    wts = [{kk: _T(next(n)) for kk in ("g_attn", "Wq", "Wk", "Wv", "Wo", "g_mlp", "Wgu", "Wd")}
           for _ in range(2)]
    buf = {"x": _T(1), "u": _T(2)}
    for kk in ("q", "k", "v", "o"):
        buf[kk] = [_T(10 * (ord(kk)) + i) for i in range(2)]
    caches = [dict(desc=f"desc{i}", k=f"kc{i}", v=f"vc{i}", table=f"t{i}") for i in range(2)]
    VT.verify_layers(shape, wts, buf, caches, "ctx", "ws")
    assert len(calls) == 2 * (VT.LINEAR_CALLS_PER_LAYER + 1)
    for i, (D, _) in enumerate(shape.layers):
        seq = calls[7 * i: 7 * i + 7]
        assert [c[0] for c in seq] == ["linear"] * 3 + ["attn"] + ["linear"] * 3
        q, k, v = seq[0][1], seq[1][1], seq[2][1]
        assert (q.m, q.n, q.k, q.norm_gain) == (24, 16 * D, 5376, wts[i]["g_attn"].addr)
        assert (k.n, v.n) == (4 * D, 4 * D) and k.norm_gain == v.norm_gain == q.norm_gain
        assert seq[0][4] is buf["q"][i] and seq[1][4] is buf["k"][i] and seq[2][4] is buf["v"][i]
        a = seq[3]
        assert a[1] == f"desc{i}" and a[2] is buf["q"][i] and a[3] is buf["k"][i]
        assert a[4] is buf["v"][i] and a[5:9] == (f"kc{i}", f"vc{i}", f"t{i}", "ctx")
        assert a[9] is buf["o"][i] and a[10] == "ws"
        o, gu, dn = seq[4][1], seq[5][1], seq[6][1]
        assert (o.n, o.k, o.epilogue) == (5376, 16 * D, sd.SD_EPI_ADD) and seq[4][4] is buf["x"]
        assert (gu.n, gu.epilogue, gu.ld_out, gu.norm_gain) == (43008, sd.SD_EPI_GEGLU, 21504,
                                                                 wts[i]["g_mlp"].addr)
        assert (dn.n, dn.k, dn.epilogue) == (5376, 21504, sd.SD_EPI_ADD)
