"""Host logic behind the bench line's `traffic` and roofline fields (no GPU): the source hash that
keeps a DRAM-traffic record valid, the record lookup, and the compulsory-byte count."""
import json
import os
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _tree(tmp_path):
    """A copy of the CUDA sources and the traffic records under a scratch root."""
    csrc = tmp_path / "exact_io_aware_43_b200" / "csrc"
    shutil.copytree(os.path.join(ROOT, "exact_io_aware_43_b200", "csrc"), csrc)
    prof = tmp_path / "profiles"
    prof.mkdir()
    shutil.copy(os.path.join(ROOT, "profiles", "dram_traffic.json"), prof / "dram_traffic.json")
    return csrc, prof


def test_source_hash_ignores_comments_and_whitespace_only(tmp_path, monkeypatch):
    csrc, _ = _tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.csrc_code_hash()
    f = csrc / "merge.cuh"
    src = f.read_text()
    f.write_text("// a new comment line\n/* and a block\n   comment */\n" + src.replace("\n", "\n\n", 3))
    assert bench.csrc_code_hash() == h0
    f.write_text(src.replace("namespace fattn {", "namespace fattn { ;", 1))  # a change to the code
    assert bench.csrc_code_hash() != h0


def test_traffic_record_lookup_follows_the_source_hash(tmp_path, monkeypatch):
    csrc, prof = _tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    recs = json.loads((prof / "dram_traffic.json").read_text())["records"]
    h = bench.csrc_code_hash()
    for r in recs:
        r["csrc_sha256"] = h
    (prof / "dram_traffic.json").write_text(json.dumps({"records": recs}))
    r0 = recs[0]
    assert bench.kernel_traffic(r0["kernel"], r0["workload"]) == r0["bytes_per_launch"]
    # another workload of the same kernel has no record
    other = dict(r0["workload"], N=r0["workload"].get("N", 0) + 128)
    assert bench.kernel_traffic(r0["kernel"], other) is None
    # a code change makes every record stale
    f = csrc / "merge.cuh"
    f.write_text(f.read_text().replace("namespace fattn {", "namespace fattn { ;", 1))
    assert bench.kernel_traffic(r0["kernel"], r0["workload"]) is None


def test_compulsory_bytes_by_hand():
    # forward: Q, K, V read and O written in bf16, L in fp32
    B, H, N, d = 2, 16, 8192, 128
    t = B * H * N * d * 2
    assert bench.pass_bytes(B, H, H, N, d, True) == 4 * t + B * H * N * 4
    # backward: Q, dO, K, V, L, D read; dQ, dK, dV written
    assert bench.pass_bytes(B, H, H, N, d, False) == 7 * t + 2 * B * H * N * 4
    # grouped heads: K, V (and dK, dV) have H_kv heads
    kv = B * 2 * N * d * 2
    assert bench.pass_bytes(B, H, 2, N, d, True) == 2 * t + 2 * kv + B * H * N * 4


def test_binding_roof_is_the_longer_ideal_time():
    peaks = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6500.0}
    # long causal backward: 1.374e12 FLOP against 0.6 GB -> tensor bound
    r = bench.binding_roofline(1.374e12, 600_000_000, 1.4, peaks, "measured")
    assert r["bound"] == "tensor" and r["other_roof"]["bound"] == "hbm"
    assert abs(r["achieved"] - 1.374e12 / 1.4e-3 / 1e12) < 1e-9
    assert abs(r["frac"] - r["achieved"] / 1600.0) < 1e-12
    assert abs(r["frac_of_sustained"] - r["achieved"] / 1400.0) < 1e-12
    # a short sequence: little work per byte -> HBM bound, with its algorithmic bytes
    r = bench.binding_roofline(1.0e10, 200_000_000, 0.05, peaks, "measured")
    assert r["bound"] == "hbm" and r["algorithmic_bytes"] == 200_000_000
    assert abs(r["achieved"] - 200_000_000 / 0.05e-3 / 1e9) < 1e-6
    assert r["other_roof"]["bound"] == "tensor"
    # the crossover: equal ideal times pick the tensor roof
    r = bench.binding_roofline(1600e12 * 1e-3, int(6500e9 * 1e-3), 2.0, peaks, "x")
    assert r["bound"] == "tensor"
