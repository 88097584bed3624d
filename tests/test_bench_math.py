"""The bench's roofline arithmetic on made-up numbers (no GPU): which bound applies,
which peak a power-capped run is held to, and the fractions it reports."""
import bench

PEAKS = (1600.0, 1400.0, 6400.0, "measured")   # bf16 burst / sustained TFLOP/s, HBM GB/s


def test_tensor_bound_kernel_at_burst_clocks():
    # 2 TFLOP over 2.5 GB: 800 FLOP/B, above the 250 FLOP/B ridge
    r = bench.roofline_record(2.0e12, 2.5e9, [1.25, 1.25], {"reasons": [], "sm_mhz": 1965, "sm_max_mhz": 1965},
                              False, PEAKS)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["peak"] == 1600.0
    assert abs(r["achieved"] - 1600.0) < 1e-9 and abs(r["frac"] - 1.0) < 1e-12
    assert abs(r["frac_of_sustained"] - 1600.0 / 1400.0) < 1e-12
    assert r["launches_timed"] == 2 and r["avg_ms"] == 1.25
    # beside the measured peak, the nominal dense one (2.25 PFLOP/s bf16)
    assert r["nominal_peak"] == 2250.0 and abs(r["frac_of_nominal"] - 1600.0 / 2250.0) < 1e-12


def test_power_capped_run_keeps_the_burst_peak_and_is_flagged():
    clk = {"reasons": ["sw_power_cap"], "sm_mhz": 1965, "sm_max_mhz": 1965}
    r = bench.roofline_record(2.0e12, 2.5e9, [1.25], clk, False, PEAKS)
    assert r["peak"] == 1600.0 and "burst" in r["peak_kind"] and r["power_capped"]
    assert abs(r["frac_of_sustained"] - 1600.0 / 1400.0) < 1e-12
    # a clock stuck well below its maximum counts as capped as well
    assert bench.power_capped({"reasons": [], "sm_mhz": 1500, "sm_max_mhz": 1965})
    assert not bench.power_capped({"reasons": [], "sm_mhz": 1900, "sm_max_mhz": 1965})
    # with per-sample counts, one capped sample among many in the window is not a cap
    one = {"reasons": ["sw_power_cap"], "sw_power_cap_samples": 1, "samples_in_window": 40,
           "sm_mhz": 1965, "sm_max_mhz": 1965}
    assert not bench.power_capped(one)
    assert bench.power_capped({**one, "sw_power_cap_samples": 12})


def test_e4m3_kernel_takes_twice_the_bf16_peak():
    r = bench.roofline_record(4.0e12, 2.5e9, [1.25], None, True, PEAKS)
    assert r["peak"] == 3200.0 and "x2" in r["peak_kind"]
    assert r["nominal_peak"] == 4500.0 and abs(r["frac_of_nominal"] - 3200.0 / 4500.0) < 1e-12


def test_decode_kernel_is_hbm_bound():
    # 60 GFLOP over 7.7 GB: 7.8 FLOP/B, far below the ridge
    r = bench.roofline_record(6.0e10, 7.7e9, [1.2], None, False, PEAKS)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] == 6400.0
    assert abs(r["achieved"] - 7.7e9 / 1.2e-3 / 1e9) < 1e-6
    assert abs(r["frac"] - r["achieved"] / 6400.0) < 1e-12
    assert r["nominal_peak"] == 8000.0 and abs(r["frac_of_nominal"] - r["achieved"] / 8000.0) < 1e-12


def test_no_launches_gives_no_fraction():
    r = bench.roofline_record(6.0e10, 7.7e9, [], None, False, PEAKS)
    assert r["achieved"] is None and r["frac"] is None and r["launches_timed"] == 0
    assert r["frac_of_nominal"] is None


def test_gate_up_kernel_sources_follow_the_library_rule():
    from mixture_experts_ffn_08_b200 import workloads as W
    assert bench.gateup_sources(W.MIXTRAL_PREFILL) == bench.DUAL_GEMM_SOURCES
    assert bench.gateup_sources(W.DSV3_PREFILL) == bench.DUAL_GEMM_SOURCES
    assert bench.gateup_sources(W.DSV3_DECODE) == bench.GEMM_SOURCES
    assert bench.gateup_sources(W.SKEWED_FP8) == bench.FP8_GEMM_SOURCES
    assert bench.gateup_sources(W.FP4["dsv3_prefill_fp4"]) == bench.FP8_GEMM_SOURCES
    assert bench.gateup_sources(W.FP4["dsv3_decode_fp4"]) == bench.FP8_GEMM_SOURCES


def test_profiled_traffic_only_for_the_kernel_it_covers(tmp_path, monkeypatch):
    (tmp_path / "profiles").mkdir()
    pkg = tmp_path / "mixture_experts_ffn_08_b200" / "csrc"
    pkg.mkdir(parents=True)
    for f in ("a.cuh", "b.cu"):
        (pkg / f).write_text(f"// {f}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    sha = bench.sources_sha256(["csrc/a.cuh", "csrc/b.cu"])
    (tmp_path / "profiles" / "gateup_swiglu_w.md").write_text(
        f"traffic_bytes_per_launch: 1234\nkernel_sources: csrc/a.cuh, csrc/b.cu\nkernel_source_sha256: {sha}\n")
    (tmp_path / "profiles" / "gateup_swiglu_big.md").write_text(
        f"traffic_per_algorithmic_byte: 1.25\nscaled_from: small case\n"
        f"kernel_sources: csrc/a.cuh, csrc/b.cu\nkernel_source_sha256: {sha}\n")
    assert bench._profiled_traffic("w", ("csrc/a.cuh", "csrc/b.cu"))[0] == 1234
    t, src = bench._profiled_traffic("big", ("csrc/a.cuh", "csrc/b.cu"), 1000)
    assert t == 1250 and "small case" in src
    assert bench._profiled_traffic("w", ("csrc/a.cuh",))[0] is None          # another kernel runs now
    (pkg / "b.cu").write_text("// changed\n")
    assert bench._profiled_traffic("w", ("csrc/a.cuh", "csrc/b.cu"))[0] is None  # sources changed
    assert bench._profiled_traffic("none", ("csrc/a.cuh",))[0] is None


def _smi_line(ts, sm, reason_cap="Not Active", smax=1965):
    # ClockSampler.FIELDS order: timestamp, index, clocks.sm, clocks.max.sm, power.draw,
    # reasons.active, hw_slowdown, hw_thermal_slowdown, sw_thermal_slowdown, sw_power_cap
    return f"{ts}, 0, {sm}, {smax}, 900.5, 0x0000000000000004, Not Active, Not Active, Not Active, {reason_cap}"


def test_clock_summary_uses_the_samples_inside_the_timed_window():
    from datetime import datetime
    t = lambda s: datetime.strptime(s, "%Y/%m/%d %H:%M:%S.%f").timestamp()
    lines = [_smi_line("2026/12/02 10:00:00.000", 1965),                      # idle, before
             _smi_line("2026/12/02 10:00:00.250", 1372, "Active"),            # timed region
             _smi_line("2026/12/02 10:00:00.300", 1380, "Active"),
             _smi_line("2026/12/02 10:00:00.350", 1390, "Active"),
             _smi_line("2026/12/02 10:00:00.700", 1965),                      # idle, after
             "garbage line"]
    win = (t("2026/12/02 10:00:00.200"), t("2026/12/02 10:00:00.400"))
    c = bench.summarize_clock_rows(lines, win)
    assert c["sm_mhz"] == 1380 and c["sm_max_mhz"] == 1965 and c["reasons"] == ["sw_power_cap"]
    assert c["samples"] == 5 and c["samples_in_window"] == 3 and c["sw_power_cap_samples"] == 3
    assert bench.power_capped(c)
    # a region shorter than the sampling interval: all samples, flagged as such
    short = (t("2026/12/02 10:00:00.400"), t("2026/12/02 10:00:00.450"))
    c = bench.summarize_clock_rows(lines, short)
    assert c["samples_in_window"] == 0 and c["samples"] == 5 and c["sm_mhz"] == 1390
    assert bench.summarize_clock_rows([], None)["sm_mhz"] is None


def test_steps_fill_the_target_time():
    assert bench._steps_for(7.5, 20) == 40          # 300 ms / 7.5 ms
    assert bench._steps_for(100.0, 20) == 20        # never below the asked steps
    assert bench._steps_for(0.01, 20) == 1000       # capped
    assert bench._steps_for(0.01, 2000) == 2000


def test_cpu_sample_sizes():
    from mixture_experts_ffn_08_b200 import workloads as W
    assert bench._cpu_sample_tokens(W.TINY) == 64                  # whole batch
    assert bench._cpu_sample_tokens(W.MIXTRAL_PREFILL) == 2838     # 2e12 / (6*2*4096*14336), floored
    assert bench._cpu_sample_tokens(W.DSV3_DECODE) == 128
    n = bench._cpu_sample_tokens(W.DSV3_PREFILL)
    assert 2000 < n < 3000


def test_host_weights_load_time_is_kept_apart_and_cache_is_bounded():
    import torch
    from mixture_experts_ffn_08_b200 import workloads as W
    wl = W.Workload("hw", T=4, H=128, I=128, E=4, K=2)
    d = {n: torch.randn(wl.E, 128, 128).to(torch.bfloat16) for n in ("w_gate", "w_up", "w_down")}
    hw = bench.HostWeights(wl, d, cap_bytes=2 * bench._expert_f64_bytes(wl))
    for e in (0, 1, 2, 0):
        g, u, dn = hw(e)
        assert g.dtype.name == "float64" and (g == d["w_gate"][e].double().numpy()).all()
    assert len(hw.cache) <= 2 and hw.load_s > 0


def test_default_line_carries_every_workload_and_the_micro_record(monkeypatch, capsys):
    """run_ours on one GPU: the headline record, one record per other workload (the e2m1
    decode layer without a CPU baseline) and the GroupedTopK micro record, in one line.
    measure() and the micro benchmark are stubbed, so this runs without a GPU."""
    import argparse
    import json
    calls = []

    def fake_measure(wl, steps, warmup, world=1, rank=0, local=0, cpu=True, adapt_steps=False):
        calls.append((wl.name, cpu, adapt_steps))
        return {"workload": wl.name, "value": 1.0, "unit": "tokens/s", "ms_per_step": 1.0, "steps": steps,
                "dtype": "bf16", "roofline": {}, "cpu_baseline": {"value": 1.0} if cpu else None}

    monkeypatch.setattr(bench, "measure", fake_measure)
    monkeypatch.setattr(bench, "micro_grouped_topk_record", lambda steps, warmup: {"value": 6.3, "unit": "us/call"})
    monkeypatch.setattr(bench.torch.cuda, "set_device", lambda d: None)
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    args = argparse.Namespace(workload="dsv3_prefill", steps=5, warmup=3, no_cpu_baseline=False, no_configs=False,
                              fused_combine=False, block_m=0, masked_cap=0)
    bench.run_ours(args)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["config"]["workload"] == "dsv3_prefill"
    assert set(line["configs"]) == {"tiny", "mixtral_prefill", "dsv3_decode", "skewed_fp8", "dsv3_decode_fp4"}
    assert line["configs"]["dsv3_decode_fp4"]["cpu_baseline"] is None
    assert all(line["configs"][n]["cpu_baseline"] is not None for n in ("tiny", "mixtral_prefill", "dsv3_decode",
                                                                       "skewed_fp8"))
    assert line["micro"]["grouped_topk"]["unit"] == "us/call"
    assert calls[0] == ("dsv3_prefill", True, False)
    assert all(adapt for _, _, adapt in calls[1:])


def test_host_cpu_reports_a_model_and_a_count():
    model, n = bench.host_cpu()
    assert isinstance(model, str) and model and isinstance(n, int) and n >= 1


def test_reference_arm_runs_the_oracle_on_the_host(monkeypatch, capsys):
    """bench.py --impl reference on the tiny workload: the fp64 oracle alone, one JSON line
    with impl, the CPU baseline (model, cores) and an end-to-end figure equal to the value."""
    import argparse
    import json
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    monkeypatch.setattr(bench, "REFERENCE_BUDGET_S", 2.0)
    bench.run_reference(argparse.Namespace(workload="tiny", steps=3, warmup=3))
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["dtype"] == "f64" and line["steps"] == 3
    assert line["value"] > 0 and line["e2e"]["value"] == line["value"]
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["cpu_baseline"]["cpu_model"]
    assert line["config"]["workload"].startswith("tiny")
    per_token = 2 * 256 * 8 + 2 * 6 * 256 * 128   # router + K=2 routed SwiGLU FFNs of the tiny layer
    assert abs(line["cpu_baseline"]["gflops"] - line["value"] * per_token / 1e9) < 1e-9 * line["value"]


def test_cpu_baseline_record_on_host_inputs():
    """The oracle's CPU baseline of the tiny layer from host-resident inputs: tokens/s, the
    GFLOP/s they imply, the cores used and the host CPU."""
    from mixture_experts_ffn_08_b200 import inputs, workloads as W
    d = inputs.make_inputs(W.TINY, seed=0, device="cpu")
    r = bench.cpu_baseline_record(W.TINY, d)
    assert r["kind"] == "oracle" and r["value"] > 0 and r["cores"] >= 1 and r["cpu_model"]
    assert abs(r["gflops"] - r["value"] * bench.oracle_flops_per_token(W.TINY) / 1e9) < 1e-9 * r["value"]
    assert bench.oracle_flops_per_token(W.DSV3_PREFILL) == 2 * 7168 * 256 + 8 * 6 * 7168 * 2048 + 6 * 7168 * 2048
