"""Host logic of bench.py, on the CPU: the reference arm's JSON contract on the smallest
workload, the quantizer selection and its rejections, and the algorithmic counts the
rooflines divide by."""
import argparse
import importlib.util
import json
import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    return b


def args(**kw):
    base = dict(gpus=1, steps=1, warmup=0, impl="reference", workload="tiny_nvfp4", e2e_steps=1,
                no_cpu_baseline=True, block=0, mode="", fmt="", scale_fmt="", x_rows=0,
                serial=False)
    base.update(kw)
    return argparse.Namespace(**base)


def test_reference_arm_line(tmp_path):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny_nvfp4", "--steps", "2", "--warmup", "1"],
                         cwd=ROOT, capture_output=True, text=True, timeout=600,
                         env=dict(os.environ, CUDA_VISIBLE_DEVICES=""))
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "dtype", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["steps"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    assert "tiny_nvfp4" in line["config"]["workload"]


def test_quantizer_selection(bench):
    from block_scaled_weight_b200 import synth
    q = bench.quantizer_for(synth.WORKLOADS["nvfp4_full_calib"], args())
    assert q == bench.HEADLINE_Q
    q = bench.quantizer_for(synth.WORKLOADS["e4m3_tiles"], args(mode="gptq"))
    assert (q.fmt, q.block, q.mode) == ("e4m3", 64, "gptq")
    assert bench.full_gptq(bench.quantizer_for(synth.WORKLOADS["nvfp4_full_calib"],
                                               args(mode="gptq-ord")))
    with pytest.raises(SystemExit):
        bench.quantizer_for(synth.WORKLOADS["int8_e4m3scale"], args(mode="gptq"))
    with pytest.raises(SystemExit):
        bench.quantizer_for(synth.WORKLOADS["e4m3_tiles"], args(mode="gptq-ord"))


def test_algorithmic_counts(bench):
    # the search: C candidates x 6 (+4); 126 E4M3 scales, 255 on the 8-bit grids
    assert bench.ops_per_weight("nvfp4", "hopt", -1) == 126 * 6 + 4
    assert bench.ops_per_weight("nvfp4", "sse", -1) == 126 * 5 + 4
    assert bench.ops_per_weight("nvfp4", "hopt", -1, "ue4m4") == 255 * 6 + 4
    assert bench.ops_per_weight("int8", "hopt", 8) == 17 * 6 + 4
    assert bench.ops_per_weight("e4m3", "hopt", -1) == 64 * 6 + 4
    assert bench.ops_per_weight("nvfp4", "bhopt", -1, "e4m3", 16) == 126 * 20 + 4
    # GPTQ sweep: the search + 6 + (k/2)(1 + 1/B) updates received
    q = bench.Quantizer("nvfp4", 16, "gptq", -1, "e4m3")
    assert bench.sweep_ops_per_weight(q, 9728) == 760 + 6 + 4864 * (1 + 1 / 16)
    # our launches per GPTQ step on the 9728-wide workload: 820, 824 ordered (the Hessian is
    # three of them: the tensor-core product, the last wave's chunk sums, the transpose)
    assert bench.gptq_launches(9728, False) == 820
    assert bench.gptq_launches(9728, True) == 824
    assert bench.code_bytes("nvfp4", 16) == 0.5 + 1 / 16
    assert bench.code_bytes("e4m3", 64) == 1 + 4 / 4096


def test_workload_descriptions(bench):
    """The config line says which GPTQ runs: the full-Hessian one (sequential or ordered) on
    the 4-bit blocks, the tile one on E4M3."""
    from block_scaled_weight_b200 import synth
    full = synth.WORKLOADS["nvfp4_full_calib"]
    for mode, kind in (("gptq", "sequential"), ("gptq-ord", "ordered")):
        d = bench.workload_desc(full, bench.quantizer_for(full, args(mode=mode)))
        assert f"{kind} GPTQ over the full input dimension" in d and "H = X^T X / R" in d
        assert "64x64 tiles" not in d
    tiles = synth.WORKLOADS["e4m3_tiles"]
    d = bench.workload_desc(tiles, bench.quantizer_for(tiles, args(mode="gptq")))
    assert "e4m3 64x64 tiles" in d and "GPTQ sweep" in d
    d = bench.workload_desc(full, bench.quantizer_for(full, args()))
    assert "GPTQ" not in d and "hopt" in d



@pytest.mark.parametrize("mode,kind", [("gptq", "sequential"), ("gptq-ord", "ordered")])
def test_reference_arm_gptq_line(mode, kind):
    """The reference arm times the oracle's full-Hessian GPTQ (h, H, factor, [order], sweep)
    on the smallest workload and prints the same contract line."""
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny_nvfp4", "--mode", mode, "--steps", "1",
                          "--warmup", "0"], cwd=ROOT, capture_output=True, text=True,
                         timeout=600, env=dict(os.environ, CUDA_VISIBLE_DEVICES=""))
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "G weights/s"
    assert f"{kind} GPTQ over the full input dimension" in line["config"]["workload"]
    assert line["cpu_baseline"]["kind"] == "oracle"
