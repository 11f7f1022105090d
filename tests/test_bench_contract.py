"""The benchmark's JSON line on CPU: the reference arm (the oracle on the
host cores) prints the contract's keys for a small workload, and the GPU arm
without a GPU fails loudly instead of falling back."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(*args, timeout=300):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, capture_output=True,
                          text=True, timeout=timeout)


def test_reference_arm_line_has_the_contract_keys():
    r = _bench("--impl", "reference", "--workload", "tiny_lsh", "--steps", "1", "--warmup", "1")
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["n_gpus"] == 1 and line["steps"] == 1
    assert line["config"]["workload"] == "tiny_lsh"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["value"] > 0 and line["e2e"]["value"] == line["value"]


def test_gpu_arm_without_a_gpu_fails_loudly():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    r = _bench("--workload", "tiny_lsh", "--steps", "1", "--warmup", "1", "--no-cpu-baseline")
    assert r.returncode != 0
    assert r.stdout.strip() == "" or "value" not in r.stdout


def test_roofline_arithmetic():
    """The byte counts behind the reported fractions: the 512K layer's
    algorithmic bytes, the norm-weighted and paged retrieval bytes, and the
    encode roofline of each hash family."""
    sys.path.insert(0, ROOT)
    import bench
    import synth
    w = synth.WORKLOADS["qwen7b_512k"]
    C = w.N - w.n_sink - w.n_local
    assert w.candidates() == C
    kv = w.B * w.Hkv * (w.top_k + w.n_sink + w.n_local) * 128 * 2 * 2
    assert w.algorithmic_bytes() >= w.B * w.Hkv * C * 16 + kv
    sv = synth.WORKLOADS["signvq"]
    r = bench.normw_roofline(sv, 1, 0.1, 0.2, 6548.8, "measured")
    assert r["bytes_per_launch"] == 16 * 8 * 65536 * (16 + 2)
    assert r["frac"] == pytest.approx(r["bytes_per_launch"] / 1e-4 / 1e9 / 6548.8)
    he = synth.WORKLOADS["hashevict_lsh"]
    r = bench.paged_roofline(he, 2, 0.1, 0.3, 256, 6548.8, "measured")
    assert r["bytes_per_launch"] == 8 * 8 * (32768 - 4 - 64) * 8
    assert r["launch_us"] == pytest.approx(50.0) and r["step_us_per_layer"] == pytest.approx(150.0)
    assert r["step_frac"] == pytest.approx(he.algorithmic_bytes() / 150e-6 / 1e9 / 6548.8)
    e = bench.encode_roofline(he, 1, 1.0)
    assert e["bound"] == "hbm" and e["gbs"] == pytest.approx(8 * 8 * 32768 * (256 + 8) / 1e-3 / 1e9)
    e = bench.encode_roofline(synth.WORKLOADS["spotlight_mlp"], 1, 1.0)
    assert e["bound"] == "tensor" and e["unit"] == "TFLOP/s"


def test_traffic_records_follow_their_sources(tmp_path, monkeypatch):
    """A recorded DRAM byte count is reported only while every source file of
    the kernel is unchanged: the committed records match the sources, and a
    one-byte change to any listed file voids the record."""
    sys.path.insert(0, ROOT)
    import bench
    csrc = os.path.join(ROOT, "hash_sparse_kv_b200", "csrc")
    fused = os.path.join(csrc, "retrieve.cu")
    normw = [os.path.join(csrc, f) for f in ("normw.cu", "normw_select.cuh")]
    assert bench.traffic_record(fused, "qwen7b_512k") is not None
    assert bench.traffic_record(normw, "signvq") is not None
    # a copy of the sources with one byte changed in the second file
    copies = []
    for i, f in enumerate(normw):
        dst = tmp_path / os.path.basename(f)
        data = open(f, "rb").read()
        dst.write_bytes(data + (b" " if i == 1 else b""))
        copies.append(str(dst))
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "dram_traffic.json").write_bytes(
        open(os.path.join(ROOT, "profiles", "dram_traffic.json"), "rb").read())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_record(copies, "signvq") is None
    assert bench.source_digest(copies) != bench.source_digest(normw)
