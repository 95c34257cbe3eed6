"""Host-side helpers of bench.py (CPU): the algorithmic FLOP counts behind
the roofline line, the ncu traffic lookup that must only answer for the
grouped-GEMM source it was captured on, and the peak denominators."""
import os
import re

import bench
import synth


def test_gemm_flops_are_the_algorithmic_counts():
    c = synth.CONFIGS["bf16_n4096_d2048_e8_k2_f8192_swiglu"]
    f1, f2 = bench.gemm_flops(c, c.N * c.K)
    assert f1 == 2.0 * 8192 * 2048 * 2 * 8192 and f2 == 2.0 * 8192 * 8192 * 2048
    assert f1 == 549755813888.0                       # the bench line's per-launch figure
    c = synth.CONFIGS["e4m3_n8192_h7168_e256_k8_n2048_gmm"]
    f1, f2 = bench.gemm_flops(c, c.N * c.K)
    assert f1 == 2.0 * 65536 * 7168 * 2048 and f2 == 0.0
    c = synth.CONFIGS["fp32_n256_d256_e8_k2_f1024_relu"]
    f1, f2 = bench.gemm_flops(c, c.N * c.K)
    assert f1 == f2 == 2.0 * 512 * 256 * 1024


def test_replica_throughput_counts_every_rank():
    assert bench.replica_throughput(4096, 10, 1, 8.0) == 4096 * 10 / 8e-3
    assert bench.replica_throughput(4096, 10, 4, 8.0) == 4 * 4096 * 10 / 8e-3


def test_profiled_traffic_follows_the_kernel_source_hash(tmp_path, monkeypatch):
    """A committed summary whose hash matches the current GEMM source gives
    its bytes; any other hash (the kernel changed since) gives None."""
    h = bench.kernel_source_hash()
    assert re.fullmatch(r"[0-9a-f]{16}", h)
    prof = os.path.join(bench.ROOT, "profiles",
                        "ffn1_swiglu_tc_bf16_n16384_d2048_e128_k8_f768_swiglu_zipf.md")
    text = open(prof).read()
    committed = re.search(r"kernel_source_sha256_16: ([0-9a-f]+)", text).group(1)
    value = bench.profiled_traffic("bf16_n16384_d2048_e128_k8_f768_swiglu_zipf", "ffn1_swiglu_tc")
    if committed == h:
        assert value == float(re.search(r"dram_bytes_per_launch: ([0-9]+)", text).group(1))
    else:
        assert value is None
    # a copy of the tree's profiles with a stale hash answers None
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "k_w.md").write_text(
        "kernel_source_sha256_16: 0000000000000000\ndram_bytes_per_launch: 123\n")
    (tmp_path / "profiles" / "k_v.md").write_text(
        f"kernel_source_sha256_16: {h}\ndram_bytes_per_launch: 456\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: h)
    assert bench.profiled_traffic("w", "k") is None
    assert bench.profiled_traffic("v", "k") == 456.0
    assert bench.profiled_traffic("missing", "k") is None


def test_peaks_are_the_measured_file_when_present():
    peaks, src = bench.load_peaks()
    assert src in ("measured", "fallback")
    for key in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained"):
        assert peaks[key] > 0
