"""Host arithmetic of bench.py (CPU): the roofline units, the traffic records and
the kernel-source key they depend on."""
import hashlib
import os

import numpy as np
import pytest

import bench
import workloads


def test_algorithmic_work_counts_active_experts_only():
    cfg = workloads.config_by_name("decode_t64_h6144_i2048_e256_k8")
    counts = np.zeros(cfg.E, dtype=np.int64)
    counts[:226] = 1
    g1, g2, active = bench.algorithmic_work(cfg, counts)
    assert active == 226
    T, H, I, k = cfg.T, cfg.H, cfg.I, cfg.k
    A = T * k
    # packed INT4 (half a byte per weight) plus one bf16 scale per 128-group
    per_expert_13 = 2 * I * H // 2 + 2 * I * (H // 128) * 2
    per_expert_2 = H * I // 2 + H * (I // 128) * 2
    assert per_expert_13 + per_expert_2 == 18_874_368 + 589_824   # the layer's 19.46 MB/expert
    assert g1["bytes"] - 226 * per_expert_13 == T * H + T * 4 + A * I * 4 + A * 4 + A * 8
    assert g2["bytes"] - 226 * per_expert_2 == A * I + A * 4 + A * H * 4
    assert g1["flops"] == 2 * A * 2 * I * H and g2["flops"] == 2 * A * H * I


def test_algorithmic_work_channel_variant_and_shared_expert():
    cfg = workloads.config_by_name("prefill_t16384_outlier_h6144_i2048_e256_k8")
    counts = np.ones(cfg.E, dtype=np.int64)
    g1, _, _ = bench.algorithmic_work(cfg, counts, "channel-int8")
    g1w, _, _ = bench.algorithmic_work(cfg, counts, "w4a8")
    # per-channel: a scale and a nibble sum per row instead of a scale per group
    diff = cfg.E * 2 * cfg.I * ((cfg.H // 128) * 2 - (2 + 4))
    assert g1w["bytes"] - g1["bytes"] == diff
    s1, s2 = bench.shared_work(cfg)
    T, H, I = cfg.T, cfg.H, cfg.I
    assert s1["flops"] == 4 * T * I * H and s2["flops"] == 2 * T * H * I
    assert s1["bytes"] > 2 * I * H and s2["bytes"] > H * I       # E4M3 weights, 1 B each


def test_recorded_traffic_is_keyed_by_the_kernel_source(tmp_path, monkeypatch):
    sid = bench.kernel_source_id()
    path = os.path.join(bench.ROOT, "w4a8_quantized_moe_b200", "csrc", "grouped_gemm.cu")
    data = open(path, "rb").read()
    assert sid == hashlib.sha1(b"blob %d\0" % len(data) + data).hexdigest()   # git's blob id
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "dram_traffic.txt").write_text(
        "# comment\n"
        f"wl grouped_gemm_gate_up 123 {sid}\n"
        f"wl:channel-int8 grouped_gemm_gate_up 456 {sid}\n"
        "old grouped_gemm_gate_up 789 0000000000000000000000000000000000000000\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_id", lambda: sid)
    assert bench.recorded_traffic("wl", "grouped_gemm_gate_up") == 123
    assert bench.recorded_traffic("wl:channel-int8", "grouped_gemm_gate_up") == 456
    assert bench.recorded_traffic("wl", "grouped_gemm_down") is None
    assert bench.recorded_traffic("old", "grouped_gemm_gate_up") is None   # stale source


def test_committed_traffic_records_name_known_workloads():
    names = {c.name for c in workloads.CONFIGS}
    for ln in open(os.path.join(bench.ROOT, "profiles", "dram_traffic.txt")):
        if ln.startswith("#") or not ln.strip():
            continue
        wl, kernel, nbytes, sid = ln.split()
        assert wl.split(":")[0] in names
        assert kernel in ("grouped_gemm_gate_up", "grouped_gemm_down")
        assert int(nbytes) > 0 and len(sid) == 40


def test_layer_work_is_the_survey_decode_formula():
    # whole-layer bytes: active experts' weights and scales, hidden in, logits
    # in, output out, h (float32, written and read) and its codes, Y (float32,
    # written and read); FLOPs 6 A H I
    cfg = workloads.config_by_name("decode_t64_h6144_i2048_e256_k8")
    counts = np.zeros(cfg.E, dtype=np.int64)
    counts[:226] = 2
    w = bench.layer_work(cfg, counts)
    T, H, I, E, k = cfg.T, cfg.H, cfg.I, cfg.E, cfg.k
    A = T * k
    assert w["bytes"] == (226 * (18_874_368 + 589_824) + T * H * 2 + T * E * 4 + T * H * 2
                          + A * I * 9 + A * H * 8)
    assert w["flops"] == 6 * A * H * I


def test_roofline_uses_burst_fp8_for_prefill_and_hbm_for_decode():
    pk = dict(hbm=6000.0, bf16=1600.0, bf16_sus=1400.0, src="test")
    r = bench.roofline(dict(bytes=6e9, flops=3.2e12), 1.0, False, pk, "k", None)
    assert r["bound"] == "hbm" and r["achieved"] == pytest.approx(6000.0)
    assert r["frac"] == pytest.approx(1.0) and r["kernel"] == "k" and r["traffic"] is None
    r = bench.roofline(dict(bytes=6e9, flops=3.2e12), 1.0, True, pk)
    assert r["bound"] == "tensor" and r["peak"] == 3200.0          # 2 x the burst bf16 rate
    assert r["achieved"] == pytest.approx(3200.0) and r["frac"] == pytest.approx(1.0)
    assert r["frac_of_sustained"] == pytest.approx(3200.0 / 2800.0)
    assert "kernel" not in r


def test_segment_histogram_bins_every_expert_once():
    counts = np.array([0, 0, 1, 8, 9, 32, 33, 128, 129, 512, 513, 2048, 2049, 60000])
    h = bench.segment_histogram(counts)
    assert sum(h["bins"].values()) == len(counts) == h["experts"]
    assert h["bins"] == {"0": 2, "1-8": 2, "9-32": 2, "33-128": 2, "129-512": 2,
                         "513-2048": 2, ">=2049": 2}
    assert h["active"] == 12 and h["max"] == 60000


def test_shared_fused_rule_and_launch_counts(monkeypatch):
    """The bench's account of where the shared expert's GEMMs run follows the
    library's rule: decode-sized batches (T k <= 32 E) without split tiling, the
    default decode shapes, W4A8_SHARED_FUSED not 0; then a step launches the
    routed kernels plus the tables and two quantisers, else also the two GEMMs."""
    import w4a8_quantized_moe_b200 as w4
    monkeypatch.delenv("W4A8_SHARED_FUSED", raising=False)
    monkeypatch.delenv("W4A8_GEMM_DECODE_SHAPE", raising=False)
    decode = workloads.CONFIGS[1]                         # T=64, E=256, k=8
    prefill = workloads.CONFIGS[3]
    assert bench.shared_fused(w4, decode, "w4a8+shared")
    assert not bench.shared_fused(w4, decode, "w4a8")
    assert not bench.shared_fused(w4, prefill, "w4a8+shared")
    assert bench.step_launches(w4, decode, "w4a8") == bench.KERNELS_PER_STEP
    assert bench.step_launches(w4, decode, "w4a8+shared") == \
        bench.KERNELS_PER_STEP + bench.SHARED_KERNELS_PER_STEP - 2
    assert bench.step_launches(w4, prefill, "w4a8+shared") == \
        w4.w4a8_moe_forward_launches(prefill.T, prefill.E, prefill.k) + bench.SHARED_KERNELS_PER_STEP
    monkeypatch.setenv("W4A8_SHARED_FUSED", "0")
    assert not bench.shared_fused(w4, decode, "w4a8+shared")
    monkeypatch.setenv("W4A8_SHARED_FUSED", "1")
    monkeypatch.setenv("W4A8_GEMM_DECODE_SHAPE", "3")
    assert not bench.shared_fused(w4, decode, "w4a8+shared")
