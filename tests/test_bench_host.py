"""bench.py's host-side helpers on CPU: the roofline denominators (measured
peaks, else the stated fallback), the weak-scaling config, and the DRAM traffic
figure, which is reported only while the GEMM source matches the capture."""
import hashlib
import json
import os

import pytest

import bench


def test_peaks_measured_and_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.peaks()[3] == "fallback"
    (tmp_path / "MEASURED_PEAKS.json").write_text(
        json.dumps({"hbm_gbs": 6543.0, "bf16_tflops": 1617.4, "bf16_tflops_sustained": 1373.0}))
    hbm, bf16, sus, src = bench.peaks()
    assert (hbm, bf16, sus, src) == (6543.0, 1617.4, 1373.0, "measured")


def test_config_is_weak_scaling():
    for world in (1, 2, 8):
        c = bench.config(world)
        assert c["global_batch"] == 2048 * world
        assert c["parallelism"] == f"dp{world}"
        assert (c["tokens_per_gpu"], c["linears"], c["r"]) == (2048, 7, 16)


def test_measured_step_flops_match_the_workload():
    """The layer's FLOP count per step: sum over the seven linears of
    4 M N K + 6 M r (K + N) (7,041.2 GFLOP at 2048 tokens, r = 16)."""
    from synthetic import inputs as S
    w = S.WORKLOADS["c4"]
    tot = sum(bench._lin_flops(w.M, l.N, l.K, w.r) for l in w.linears)
    assert abs(tot / 1e9 - 7041.2) < 0.1


def _fake_tree(tmp_path, src: bytes, recorded_sha: str):
    csrc = tmp_path / "bit_nf4_quantized_10_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "gemm.cu").write_bytes(src)
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic.json").write_text(json.dumps(
        {"qlora_gemm_kernel": {bench.WORKLOAD: {"dram_bytes_per_launch": 45117440, "gemm_cu_sha256": recorded_sha}}}))


def test_gemm_traffic_only_for_the_captured_source(tmp_path, monkeypatch):
    src = b"// kernel source\n"
    _fake_tree(tmp_path, src, hashlib.sha256(src).hexdigest())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.gemm_traffic() == 45117440.0
    (tmp_path / "bit_nf4_quantized_10_b200" / "csrc" / "gemm.cu").write_bytes(src + b"// changed\n")
    assert bench.gemm_traffic() is None


def test_gemm_traffic_missing_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.gemm_traffic() is None


@pytest.mark.skipif(not os.path.exists(os.path.join(bench.ROOT, "profiles", "traffic.json")), reason="no capture")
def test_committed_traffic_record_is_well_formed():
    for d in json.load(open(os.path.join(bench.ROOT, "profiles", "traffic.json")))["qlora_gemm_kernel"].values():
        assert d["dram_bytes_per_launch"] > 0 and len(d["gemm_cu_sha256"]) == 64
