"""Host logic of bench.py, on the CPU: the launch count it claims, the traffic
figure it takes from the committed ncu record (and drops once the kernel code
changes), the peak denominators, the clock-sample parser that decides whether
a run is kept, and the oracle arm (`--impl reference`) end to end."""
import json
import os
import re
import shutil

import pytest

import bench
import bit_fp8_attention_smooth_b200 as vc
from bit_fp8_attention_smooth_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("iters", [1, 2, 10])
def test_launches_per_step_by_mode(iters):
    import dataclasses

    base = vc.Params(C=16, iters=iters, block=128)
    # C <= 64, the fused pass: init, km_pass and km_refine a pass, km_finalize
    # between passes, scan and scatter once, then K/V block quantisation
    assert bench.launches_per_step(base) == 1 + 2 * iters + (iters - 1) + 2 + 2 + 2
    assert bench.launches_per_step(dataclasses.replace(base, C=64)) == bench.launches_per_step(base)
    # C > 64: init, 4 a pass (assign, refine, scan, scatter), update and
    # finalize between passes, then K/V block quantisation
    big = dataclasses.replace(base, C=256)
    assert bench.launches_per_step(big) == 1 + 4 * iters + 2 * (iters - 1) + 2 + 2

    assert bench.launches_per_step(dataclasses.replace(base, smooth=0)) == 3 + 2
    assert bench.launches_per_step(dataclasses.replace(base, smooth=2)) == 2 + 2


def _fake_root(tmp_path, per_head=1000):
    csrc = tmp_path / "bit_fp8_attention_smooth_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in ("vc_attn.cu", "vc_device.cuh"):
        shutil.copy(os.path.join(ROOT, "bit_fp8_attention_smooth_b200", "csrc", name), csrc / name)
    (tmp_path / "profiles").mkdir()
    return csrc


def _write_profile(tmp_path, code_hash, per_head, kernel="vc_attn_kernel"):
    (tmp_path / "profiles" / "attn_traffic.json").write_text(json.dumps(
        {kernel: {"sources_sha256_16": code_hash, "dram_bytes_per_head": per_head}}))


def test_traffic_follows_the_kernel_code(tmp_path, monkeypatch):
    csrc = _fake_root(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.kernel_code_hash()
    assert h == bench.kernel_code_hash() and re.fullmatch(r"[0-9a-f]{16}", h)
    _write_profile(tmp_path, h, 1234)
    assert bench.attn_traffic_bytes(40) == 1234 * 40
    # comments and blank lines do not change the hash
    src = csrc / "vc_attn.cu"
    src.write_text("// a new comment\n\n" + src.read_text().replace("\n", "  // trailing\n", 1))
    assert bench.kernel_code_hash() == h
    assert bench.attn_traffic_bytes(8) == 1234 * 8
    # a code change does: the counters no longer apply
    src.write_text(src.read_text() + "\nstatic int changed_code = 1;\n")
    assert bench.kernel_code_hash() != h
    assert bench.attn_traffic_bytes(40) is None


def test_traffic_without_a_profile_is_null(tmp_path, monkeypatch):
    _fake_root(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.attn_traffic_bytes(40) is None
    (tmp_path / "profiles" / "attn_traffic.json").write_text("{}")
    assert bench.attn_traffic_bytes(40) is None
    (tmp_path / "profiles" / "attn_traffic.json").write_text("not json")
    assert bench.attn_traffic_bytes(40) is None
    # a record of another kernel does not apply
    _write_profile(tmp_path, bench.kernel_code_hash(), 99, kernel="vc_attn4_kernel")
    assert bench.attn_traffic_bytes(40) is None
    assert bench.attn_traffic_bytes(40, "vc_attn4_kernel") == 99 * 40


def test_traffic_applies_only_to_the_captured_shape(tmp_path, monkeypatch):
    _fake_root(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "profiles" / "attn_traffic.json").write_text(json.dumps({"vc_attn_kernel": {
        "sources_sha256_16": bench.kernel_code_hash(), "dram_bytes_per_head": 77, "N": 32768, "d": 128,
        "block": 128}}))
    assert bench.attn_traffic_bytes(40, "vc_attn_kernel", 32768, 128, 128) == 77 * 40
    assert bench.attn_traffic_bytes(40, "vc_attn_kernel", 75600, 128, 128) is None
    assert bench.attn_traffic_bytes(2, "vc_attn_kernel", 32768, 64, 128) is None
    assert bench.attn_traffic_bytes(40, "vc_attn_kernel", 32768, 128, 64) is None


def test_committed_traffic_records_are_well_formed():
    path = os.path.join(ROOT, "profiles", "attn_traffic.json")
    if not os.path.exists(path):
        pytest.skip("no traffic record committed")
    recs = json.load(open(path))
    for kernel, rec in recs.items():
        assert re.fullmatch(r"[0-9a-f]{16}", rec["sources_sha256_16"]), kernel
        # at least the fp8 Q and K and the V residual of one head are read
        assert int(rec["dram_bytes_per_head"]) >= 2 * 32768 * 128, kernel


def test_peaks_measured_and_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    p = bench.load_peaks()
    assert p["source"] == "fallback" and p["hbm_gbs"] == 6650.0 and p["bf16"] == 1590.0
    (tmp_path / "MEASURED_PEAKS.json").write_text(
        '{"hbm_gbs": 6538.0, "bf16_tflops": 1606.0, "bf16_tflops_sustained": 1384.2}')
    p = bench.load_peaks()
    assert p == dict(hbm_gbs=6538.0, bf16=1606.0, bf16_sustained=1384.2, source="measured")


def _sampler(lines):
    c = bench.ClockSampler(0)
    c.lines = lines
    return c


def test_clock_summary_median_and_reasons():
    idle = "Not Active"
    lines = [
        f"0, 1335, 1965, 950.1, 0x0000000000000004, {idle}, {idle}, {idle}, Active",
        f"0, 1965, 1965, 400.0, 0x0000000000000000, {idle}, {idle}, {idle}, {idle}",
        f"0, 1500, 1965, 990.0, 0x0000000000000004, {idle}, {idle}, {idle}, Active",
        "garbage line",
        "0, [N/A], 1965, 1.0, 0x0, x, x, x, x",
    ]
    s = _sampler(lines).summary()
    assert s == {"sm_mhz": 1500.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}


def test_clock_summary_flags_slowdowns():
    idle = "Not Active"
    s = _sampler([f"0, 900, 1965, 700, 0x8, Active, {idle}, Active, {idle}"]).summary()
    assert s["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]


def test_clock_summary_without_samples_is_null():
    assert _sampler([]).summary() is None


def test_config_names_the_workload_and_its_l2_rule():
    w = synth.WORKLOADS["mid_32k_d128"]
    c = bench.config_of(w, True)
    assert c["v_smooth"] is True and bench.config_of(w, False)["v_smooth"] is False
    assert c["workload"] == w.name and (c["B"], c["H"], c["N"], c["d"]) == (w.B, w.H, w.N, w.d)
    assert c["residual"] == "e4m3"
    gb = float(re.search(r"inputs ([0-9.]+) GB", c["l2"]).group(1))
    assert gb * 1e9 > 126e6
    assert bench.config_of(synth.WORKLOADS["nvfp4_32k_d128"], True)["residual"].startswith("nvfp4")
    # a parity-size case is named as one, not passed off as L2-exceeding
    assert "fit in the 126 MB L2" in bench.config_of(synth.WORKLOADS["tiny_1k_d64"], True)["l2"]


def _run_reference(env_extra):
    import json
    import subprocess
    import sys

    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    env.update(env_extra)
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0",
                        "--ref-rows", "16"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [line for line in r.stdout.splitlines() if line.startswith("{")]
    return [json.loads(line) for line in lines]


def test_reference_arm_prints_one_contract_line():
    """The oracle arm on the host: one JSON line with the contract's keys,
    its own e2e (no transfers) and a cpu_baseline describing the run."""
    (line,) = _run_reference({})
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "TFLOPS"
    assert line["metric"] == bench.METRIC and line["higher_is_better"] is True and line["n_gpus"] == 1
    assert line["config"] == bench.config_of(synth.WORKLOADS["mid_32k_d128"], True)
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    assert cb["cpu_model"]
    # ms_per_step is the measured sample; the full-workload time is an extrapolation beside it
    samp = line["sample_s"]["prep"] + line["sample_s"]["rows"]
    assert line["ms_per_step"] >= 0.9 * samp * 1e3
    assert line["extrapolated_step_s"] == pytest.approx(line["extrapolated_head_s"] * 40)
    assert line["value"] == pytest.approx(40 * 4.0 * 32768 ** 2 * 128 / line["extrapolated_step_s"] / 1e12)
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOPS", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_do_no_work():
    assert _run_reference({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}) == []


def test_prep_roofline_against_the_workload_arithmetic():
    """The compulsory prep bytes and k-means flops of the 40-head 32K
    workload: 25.43 MB and 5.37 GFLOP a head (1.017 GB and 215 GFLOP in all).
    At the measured peaks the two floors nearly coincide (about 0.156 ms)."""
    w = synth.WORKLOADS["mid_32k_d128"]
    peaks = dict(hbm_gbs=6538.0, bf16=1606.0, bf16_sustained=1384.2)
    r = bench.prep_roofline(w, 3.45, peaks, timed_s=5.0)
    per_head = 4 * 32768 * 128 + 2 * 32768 * 128 + 4 * 32768 + 4 * 256 * 128 + 4 * 256 + 4 * 128
    assert r["bytes"] == 40 * per_head and abs(r["bytes"] / 1e9 - 1.017) < 0.001
    assert r["flops"] == 2.0 * 32768 * 64 * 128 * 10 * 40 and abs(r["flops"] / 1e9 - 214.7) < 0.1
    t_bytes, t_flops = r["bytes"] / 6538e9, r["flops"] / 1384.2e12
    assert r["floor_ms"] == pytest.approx(max(t_bytes, t_flops) * 1e3)
    assert r["frac"] == pytest.approx(r["floor_ms"] / 3.45) and 0 < r["frac"] < 1
    assert r["achieved_gbs"] == pytest.approx(r["bytes"] / 3.45e-3 / 1e9)
    # the 4-bit workload writes half the residual bytes plus one scale byte per 16
    w4 = synth.WORKLOADS["nvfp4_32k_d128"]
    r4 = bench.prep_roofline(w4, 2.0, peaks, timed_s=5.0)
    per_head4 = per_head - 32768 * 128 // 2 + 256 * 128 * 8
    assert r4["bytes"] == 24 * per_head4
    # without a sustained figure the burst one is used
    assert bench.prep_roofline(w, 3.45, dict(hbm_gbs=6538.0, bf16=1606.0, bf16_sustained=None),
                               timed_s=5.0)["peak_bf16_tflops"] == 1606.0
    # and so it is for a timed region under two seconds
    assert bench.prep_roofline(w, 3.45, peaks, timed_s=0.3)["peak_bf16_tflops"] == 1606.0


def test_tensor_peak_by_timed_region():
    peaks = dict(hbm_gbs=6538.0, bf16=1606.0, bf16_sustained=1384.2)
    assert bench.tensor_peak(peaks, 0.35) == (1606.0, "burst")
    assert bench.tensor_peak(peaks, 3.0) == (1384.2, "sustained")
    assert bench.tensor_peak(dict(peaks, bf16_sustained=None), 3.0) == (1606.0, "burst")
