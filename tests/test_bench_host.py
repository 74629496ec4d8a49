"""The benchmark's workload table and its CPU oracle arm (no GPU).

Each workload must carry the shapes of its configuration (batch, context, drafts, layers,
width, vocabulary, precision); the tiny float32 one is small enough to run the oracle arm here.
"""
import json

import pytest

import bench


def cfg(*argv):
    return bench.make_cfg(bench.parse(list(argv)))


def test_workloads_carry_their_configuration():
    c = cfg()
    assert (c.kind, c.B, c.L, c.k, c.chain, c.d, c.V) == ("spec_step", 8, 16384, 2, 2, 5376,
                                                          262144)
    assert c.verify_layers == ((512, 0), (256, 512)) and c.q_mode == "tuned"
    assert len(c.sigmas) == 2 and c.sigmas[0] > c.sigmas[1] > 1.0
    c = cfg("--workload", "tiny_fp32")
    assert (c.B, c.L, c.k, c.hq, c.hkv, c.d, c.V, c.dtype) == (1, 256, 2, 4, 1, 256, 1024, "f32")
    assert c.verify_layers == ((64, 0),) and c.sigmas == (1.5 ** 0.5,) * 2
    c = cfg("--workload", "edge")
    assert (c.B, c.L, c.hq, c.hkv, c.d) == (1, 4096, 8, 2, 2560)
    assert c.verify_layers == ((256, 512),)
    c = cfg("--workload", "global", "--k", "6")
    assert (c.B, c.L, c.k, c.verify_layers, c.chain) == (8, 16384, 6, ((512, 0),), 0)
    assert len(c.sigmas) == 6
    c = cfg("--workload", "drafter")
    assert (c.chain, c.verify, c.drafter_dense, c.q_mode) == (4, False, True, "drafter")
    assert c.xlayers == ((256, 512),) * 3 + ((512, 0),) and c.unit == "drafted tokens/s"
    c = cfg("--workload", "serving")
    assert (c.B, c.L, c.k, c.shuffle) == (64, (1024, 16384), 2, True)
    assert set(c.verify_layers) == {(256, 512), (512, 0)}
    names = {cfg("--workload", w).name() for w in
             ("spec_step", "tiny_fp32", "edge", "global", "drafter", "serving")}
    assert len(names) == 6


def test_tiny_workload_reference_arm(capsys):
    args = bench.parse(["--impl", "reference", "--workload", "tiny_fp32", "--steps", "2",
                        "--warmup", "0"])
    bench.run_reference(args, 0, 1)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["config"]["workload"] == "tiny_fp32_b1_ctx256_k2"
    assert line["dtype"] == "f64" and line["e2e"]["h2d_bytes_per_step"] == 0
