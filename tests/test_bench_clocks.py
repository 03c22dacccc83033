"""bench.py's clock sampler against a fake NVML (no GPU needed): the median SM
clock, the maximum and the clock-event reasons seen while it runs."""
import sys
import time
import types


def _fake_nvml(clocks, reasons):
    m = types.ModuleType("pynvml")
    m.NVML_CLOCK_SM = 1
    m.nvmlClocksEventReasonSwPowerCap = 0x4
    m.nvmlClocksEventReasonHwSlowdown = 0x8
    m.nvmlClocksEventReasonSwThermalSlowdown = 0x20
    m.nvmlClocksEventReasonHwThermalSlowdown = 0x40
    state = {"i": 0}
    m.nvmlInit = lambda: None
    m.nvmlDeviceGetHandleByIndex = lambda i: ("dev", i)
    m.nvmlDeviceGetHandleByUUID = lambda u: ("dev", u)
    m.nvmlDeviceGetMaxClockInfo = lambda h, kind: 1965

    def clock(h, kind):
        state["i"] += 1
        return clocks[(state["i"] - 1) % len(clocks)]
    m.nvmlDeviceGetClockInfo = clock
    m.nvmlDeviceGetCurrentClocksEventReasons = lambda h: reasons
    return m


def test_nvml_sampler_reports_median_and_reasons(monkeypatch):
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml([1800, 1900, 1700], 0x4 | 0x1))
    import bench
    c = bench.Clocks("0")
    c.start()
    time.sleep(0.1)
    r = c.stop()
    assert r["samples"] >= 3
    assert r["sm_mhz"] in (1700, 1800, 1900)
    assert r["sm_max_mhz"] == 1965
    assert r["reasons"] == ["sw_power_cap"]       # bit 0x1 (idle) is not a reason we report


def test_throttle_reasons_are_named():
    import bench
    assert set(bench.Clocks.NAMES) == {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                                       "sw_power_cap"}


def test_work_unit_and_traffic_ratio_of_each_gemm():
    """The tensor-core work unit bench.py attributes to each GEMM (it keys the
    ncu traffic ratio): on the bf16 bench workload GEMM1 takes the tokens-as-N
    kernel and GEMM2 the 256 x 512 pair tiles; E4M3 and small batches take
    single-CTA 128-row units; a forced kernel choice wins."""
    import bench
    from shared_routed_expert_b200 import synth
    bf16, fp8, dec = (synth.CONFIGS[n] for n in ("prefill_bf16", "prefill_fp8", "decode_bf16"))
    assert bench.unit_rows(bf16, "auto", "gemm1_tc") == "swap"
    assert bench.unit_rows(bf16, "auto", "gemm2_tc") == "pair256x512"
    assert bench.unit_rows(fp8, "auto", "gemm1_tc") == 128
    assert bench.unit_rows(dec, "auto", "gemm1_tc") == 128
    assert bench.unit_rows(bf16, "tcgen05_wide", "gemm1_tc") == "pair256x512"
    assert bench.unit_rows(bf16, "tcgen05_m256", "gemm2_tc") == 256
    r = bench.PROFILED_TRAFFIC_RATIO
    assert r[("gemm1_tc", "bf16", "swap")] == 1.007 and r[("gemm2_tc", "bf16", "pair256x512")] == 0.967


def test_cpu_baseline_times_the_oracle_and_small_batches_on_one_core():
    """The CPU baseline runs the oracle on a token sample with all host cores;
    batches of <= 64 tokens are also timed on one core."""
    import bench
    from shared_routed_expert_b200 import synth
    cfg = synth.CONFIGS["tiny_fp32"]
    r = bench.cpu_baseline(cfg, synth.make_inputs(cfg), seconds=0.2)
    assert r["kind"] == "oracle" and r["unit"] == "tokens/s" and r["value"] > 0 and r["cores"] >= 1
    assert r["single_thread"]["cores"] == 1 and r["single_thread"]["value"] > 0


def test_roofline_of_gemm1_on_the_bf16_bench_workload():
    """bench.py's roofline entry for GEMM1 of prefill_bf16 against the closed
    forms: FLOPs 2 R 2I H, bytes = the touched experts' gate/up weights + the
    gathered rows in + h out; with the measured peaks the launch sits on the HBM
    side of the ridge (bytes / 6544 GB/s > FLOPs / sustained bf16 peak)."""
    import numpy as np
    import bench
    from shared_routed_expert_b200 import synth
    cfg = synth.CONFIGS["prefill_bf16"]
    R, H, I, E = cfg.rows, cfg.H, cfg.I, cfg.n_experts
    counts = np.full(E, R // E)
    fl, nb = bench.algorithmic(cfg, "gemm1_tc", counts)
    assert fl == 2 * R * 2 * I * H
    assert nb == E * 2 * I * H * 2 + R * H * 2 + R * I * 2
    pk = {"hbm_gbs": 6544.0, "bf16_tflops": 1414.4, "source": "measured"}
    ms = 1.0
    r = bench.roofline_of(cfg, "gemm1_tc", ms, counts, pk, "auto")
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] == 6544.0
    assert abs(r["achieved"] - nb / 1e-3 / 1e9) < 1e-6 * r["achieved"]
    assert abs(r["frac"] - r["achieved"] / 6544.0) < 1e-12
    assert r["traffic"] == int(1.007 * nb)                    # the tokens-as-N capture's ratio
    assert abs(r["tensor_frac"] - fl / 1e-3 / 1e12 / 1414.4) < 1e-9


def test_every_timed_kernel_has_algorithmic_bytes():
    """Each kernel the bench times gets the bytes it must move at least once,
    so that no roofline entry is left without its numerator."""
    import numpy as np
    import bench
    from shared_routed_expert_b200 import synth
    for name in ("prefill_bf16", "prefill_fp8", "decode_bf16"):
        cfg = synth.CONFIGS[name]
        counts = np.full(cfg.n_experts, cfg.rows // cfg.n_experts)
        for k in bench.KERNELS:
            if k.endswith("_simt") and cfg.w_dtype != "f32":
                continue
            fl, nb = bench.algorithmic(cfg, k, counts)
            assert nb is not None and nb > 0, (name, k)


def test_gather_bytes_leave_out_the_shared_rows():
    """The fused layer's gather copies only the routed rows (the shared
    expert's rows are x itself, read by GEMM1): prefill_bf16 reads x once
    (4096 x 5120 x 2 B) and writes 32768 routed rows of 10240 B = 377.5 MB; the
    unfused layer has no shared rows in its grouped pass and copies all R."""
    import bench
    from shared_routed_expert_b200 import synth
    cfg = synth.CONFIGS["prefill_bf16"]
    _, nb = bench.algorithmic(cfg, "gather", None)
    assert nb == 4096 * 5120 * 2 + 32768 * 5120 * 2 == 377_487_360
    _, nb_u = bench.algorithmic(cfg, "gather", None, fused=False)
    assert nb_u == 4096 * 5120 * 2 + cfg.rows * 5120 * 2
    # E4M3 layers gather token by token from bf16 x: x read once (2 B per
    # element), the codes of every token and of the 32768 routed rows written
    # (1 B per element) with one fp32 scale per row
    c8 = synth.CONFIGS["skewed_fp8"]
    _, nb8 = bench.algorithmic(c8, "gather", None)
    assert nb8 == 4096 * 5120 * 2 + (4096 + 32768) * (5120 + 4)


def test_unmeasured_figures_print_as_null(capsys):
    import json

    import bench
    bench.emit({"value": 1.5, "unfused": {"ms_per_step": float("nan"), "x": [float("inf"), 2]}})
    out = capsys.readouterr().out
    assert json.loads(out) == {"value": 1.5, "unfused": {"ms_per_step": None, "x": [None, 2]}}
    assert "NaN" not in out and "Infinity" not in out


def test_route_path_and_its_dims_follow_the_library_rule():
    """bench.py charges the routing kernels by the same rule the library uses:
    prefill batches (T > 256, bf16 activations, renormalised, 32..256 routed
    experts, K <= 16) take the tensor-core routing, decode and fp32 layers the
    fixed-order router; NP pads the experts to 32, KS slices H (<= H/256)."""
    import bench
    from shared_routed_expert_b200 import synth
    C = synth.CONFIGS
    assert bench.route_tc_path(C["prefill_bf16"]) and bench.route_tc_path(C["prefill_fp8"])
    assert bench.route_tc_path(C["skewed_fp8"])
    assert not bench.route_tc_path(C["decode_bf16"]) and not bench.route_tc_path(C["tiny_fp32"])
    assert not bench.route_tc_path(synth.variant(C["prefill_bf16"], renormalize=False))
    assert not bench.route_tc_path(synth.variant(C["prefill_bf16"], n_routed=16, top_k=4))
    assert bench.route_tc_dims(C["prefill_bf16"]) == (160, 4)
    assert bench.route_tc_dims(synth.variant(C["prefill_bf16"], H=512, n_routed=40)) == (64, 2)
    assert bench.route_tc_dims(synth.variant(C["prefill_bf16"], H=768, n_routed=33)) == (64, 2)
    assert bench.route_tc_dims(synth.variant(C["prefill_bf16"], H=256, n_routed=256)) == (256, 1)
