"""The N>1 host path of bench.py: replicas report the max of their timings and the
job throughput counts every replica's work.  Two gloo ranks on CPU."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    ms = [10.0 + rank, 50.0 - 10 * rank]          # rank 0: (10, 50); rank 1: (11, 40)
    got = bench.max_over_ranks(ms, world, "cpu")
    out[rank] = got
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == [11.0, 50.0] and out[1] == [11.0, 50.0]


def test_job_throughput_counts_all_replicas():
    import bench
    assert bench.job_tflops(1e12, 1, 10, 1000.0) == pytest.approx(10.0)
    assert bench.job_tflops(1e12, 4, 10, 1000.0) == pytest.approx(40.0)
    assert bench.max_over_ranks([3.0, 4.0], 1) == [3.0, 4.0]


def test_clock_summary_decodes_reasons():
    """The clock record: median SM clock under load and the reasons seen, decoded from
    the NVML bit mask (a fake NVML module; nothing is queried)."""
    import types

    import bench
    fake = types.SimpleNamespace(nvmlClocksEventReasonHwSlowdown=0x8,
                                 nvmlClocksEventReasonHwThermalSlowdown=0x40,
                                 nvmlClocksEventReasonSwThermalSlowdown=0x20,
                                 nvmlClocksEventReasonSwPowerCap=0x4)
    c = bench.ClockSampler("cpu")
    assert c.summary()["reasons"] == ["unsampled"]
    c.nvml, c.max_mhz = fake, 1965
    c.samples = [(1900, 0), (1950, 0x4), (1800, 0x4 | 0x1), (1965, 0)]
    s = c.summary()
    assert s["sm_mhz"] == 1925 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]
    c.samples.append((1200, 0x40))
    assert bench.ClockSampler.summary(c)["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    c.samples = [(1965, 0), (1965, 0x80), (1965, 0)]
    assert c.summary()["reasons"] == ["hw_power_brake_slowdown"]


def test_clock_sampler_keeps_only_the_timed_region(monkeypatch):
    """The sampler's thread has taken a sample before the region starts, and only the
    samples taken between entering and leaving the region are summarised (a fake NVML
    whose clock reads 1000 MHz until the region starts, 1965 MHz inside it)."""
    import time
    import types
    import bench
    state = {"inside": False}
    fake = types.SimpleNamespace(
        NVML_CLOCK_SM=0, nvmlClocksEventReasonSwPowerCap=0x4,
        nvmlDeviceGetClockInfo=lambda h, c: 1965 if state["inside"] else 1000,
        nvmlDeviceGetCurrentClocksEventReasons=lambda h: 0x4 if state["inside"] else 0x40,
        nvmlShutdown=lambda: None)

    def fake_open(self):
        self.nvml, self.handle, self.max_mhz = fake, object(), 1965
        time.sleep(0.02)  # a slow NVML start

    monkeypatch.setattr(bench.ClockSampler, "_open", fake_open)
    with bench.ClockSampler("cpu") as c:
        assert c.raw, "no sample before the region"
        state["inside"] = True
        time.sleep(0.1)
    s = c.summary()
    assert s["samples"] >= 3
    assert s["sm_mhz"] == 1965 and s["reasons"] == ["sw_power_cap"]


def test_hw_fp4_peak_uses_the_sampled_clock():
    """The GEMM roofline's peak: 32768 FP4 FLOP per SM per cycle on 148 SMs at the
    median clock of the timed region, falling back to the maximum clock (then 1965
    MHz) when nothing was sampled."""
    import bench
    peak, mhz = bench.hw_fp4_peak({"sm_mhz": 1965.0, "sm_max_mhz": 1965})
    assert mhz == 1965.0 and abs(peak - 32768 * 148 * 1965e6 / 1e12) < 0.1
    peak, mhz = bench.hw_fp4_peak({"sm_mhz": 1500.0, "sm_max_mhz": 1965})
    assert mhz == 1500.0 and abs(peak - 32768 * 148 * 1500e6 / 1e12) < 0.1
    assert bench.hw_fp4_peak({"sm_mhz": None, "sm_max_mhz": 1800})[1] == 1800
    assert bench.hw_fp4_peak(None)[1] == 1965


def test_grouped_roofline_bytes_and_flops():
    """The MoE grouped GEMMs' roofline: the up projection (K 4096 -> N 1536) and the
    down projection (K 1536 -> N 4096) over 65536 routed rows move 578.8 MB and
    820.0 MB (codes, scales, bf16 output) and each does 824.6 GFLOP."""
    import types

    import bench
    step = types.SimpleNamespace(routed=65536)
    pk = {"hbm_gbs": 6550.4, "source": "measured"}
    r = bench.grouped_roofline([0.1, 0.2, 0.1, 0.2], 2, step, pk, 9529.6)
    assert r["up"]["algorithmic_bytes"] == 578813952
    assert r["down"]["algorithmic_bytes"] == 819986432
    up_roof = max(2 * 65536 * 1536 * 4096 / 9529.6e12, 578813952 / 6550.4e9) * 1e6
    assert abs(r["up"]["roofline_us"] - round(up_roof, 1)) < 0.11
    assert abs(r["up"]["frac"] - up_roof / 100.0) < 1e-4


def test_both_arms_report_the_same_config():
    """The reference arm's line carries the workload `config` of the measured arm,
    built by the same function (routed rows: every token goes to TOPK experts)."""
    import inspect
    import bench
    c = bench.bench_config(2)
    assert c["parallelism"] == "replicas x2"
    assert c["moe"]["routed_rows"] == bench.MOE_TOKENS * bench.TOPK
    assert "bench_config(world)" in inspect.getsource(bench.run_reference)
    assert "bench_config(world)" in inspect.getsource(bench.main)
