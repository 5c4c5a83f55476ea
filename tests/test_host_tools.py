"""Host tools behind the committed measurements (no GPU): the ncu launch-list
summary and the nvidia-smi clock sampler that decides whether a bench run is
kept (throttle reasons, median SM clock under load)."""
import csv

import os
import sys

sys.path.insert(0, os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "benchmarks"))
import ncu_summary  # noqa: E402


def _launch_csv(path, launches):
    with open(path, "w", newline="") as f:
        w = csv.writer(f)
        w.writerow(["==PROF== Connected to process 1"])
        w.writerow(["ID", "Kernel Name", "Metric Name", "Metric Unit", "Metric Value"])
        for i, (name, unit, value) in enumerate(launches):
            w.writerow([i, name, "gpu__time_duration.sum", unit, value])


def test_ncu_summary_takes_the_last_complete_step_and_groups_kernels(tmp_path):
    p = tmp_path / "launches.csv"
    _launch_csv(p, [
        ("dash::rows::rope_table_kernel(float2 *, long, int, double)", "us", "9"),  # an earlier step
        ("dash::attn::attn_kernel<128, 0>(...)", "ms", "50"),
        ("dash::rows::rope_table_kernel(float2 *, long, int, double)", "us", "10"),  # last step starts
        ("void dash::gemm::gemm_pair_kernel<3, 0>(...)", "ms", "3"),
        ("void dash::attn::attn_kernel<128, 0>(...)", "us", "2,000"),
        ("void dash::attn::attn_kernel<128, 1>(...)", "ns", "1000000"),
        ("void dash::rows::rmsnorm_kernel<0>(...)", "us", "500"),
        ("dash::rows::rope_table_kernel(float2 *, long, int, double)", "us", "11"),  # a step cut short
        ("void dash::attn::attn_kernel<128, 0>(...)", "ms", "7"),
    ])
    lines = ncu_summary.summarise(str(p)).splitlines()
    rows = {ln[:34].strip(): ln[34:].split() for ln in lines[1:]}
    assert rows["attention"] == ["2", "3.000", "46.1%"]       # (2 + 1) ms of 6.51; the 50 ms launch is not in the step
    assert rows["gemm_gate_up_swiglu"] == ["1", "3.000", "46.1%"]
    assert rows["rmsnorm"][:2] == ["1", "0.500"]
    assert rows["rope_table"][:2] == ["1", "0.010"]
    assert rows["total (one step)"] == ["5", "6.510"]
    # rows are ordered by time, largest first
    shares = [float(ln.split()[-1].rstrip("%")) for ln in lines[1:-1]]
    assert shares == sorted(shares, reverse=True)


def test_ncu_summary_names_unknown_kernels():
    assert ncu_summary.short("void some_library_kernel<float>(int)") == "other: void some_library_kernel<float>"
    assert ncu_summary.short("void dash::rows::move_rows_kernel<true>(...)") == "scatter"


class _DoneProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def test_clock_sampler_reports_median_clock_and_active_reasons(tmp_path):
    import bench
    path = tmp_path / "clocks.csv"
    path.write_text(
        "0, 1400, 1965, 990.1, 0x4, Not Active, Not Active, Not Active, Active\n"
        "0, 1300, 1965, 998.0, 0x4, Not Active, Not Active, Not Active, Active\n"
        "0, 1500, 1965, 970.5, 0x0, Not Active, Not Active, Not Active, Not Active\n"
        "garbled line\n")
    s = bench.ClockSampler(0)
    s.proc, s.path = _DoneProc(), str(path)
    r = s.stop()
    assert r == {"sm_mhz": 1400.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    assert not path.exists()


def test_clock_sampler_without_nvidia_smi_reports_nothing():
    import bench
    s = bench.ClockSampler(0)
    assert s.stop() is None
