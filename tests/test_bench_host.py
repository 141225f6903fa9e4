"""Host-side pieces of bench.py that decide what a bench line reports: the
algorithmic byte counts behind the roofline, the committed ncu traffic record
(used only while the kernel source is unchanged), and the clock record that
rejects throttled runs.  No GPU needed."""
import os
import sys

import pytest

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_gateup_bytes_counts_codes_scales_x_and_h():
    wl = synth.workload("olmoe_like")          # H 2048, I 1024, k 8, MXFP4 (group 32)
    per_expert = 2 * 1024 * 2048 // 2 + 2 * 1024 * 2048 // 32   # codes + E8M0 scales of gate and up
    want = 64 * per_expert + 32 * 2048 * 2 + 32 * 8 * 1024 * 2
    assert bench.gateup_bytes(wl, 64, 32) == want == 143261696


def test_layer_bytes_adds_router_shared_expert_and_io():
    wl = synth.workload("deepseek_v4_flash_like")
    got = bench.layer_bytes(wl, 10, 4)
    want = (10 * wl.expert_bytes() + wl.n_experts * wl.hidden * 4 + 4 * wl.hidden * 6
            + 3 * wl.shared_inter * wl.hidden * 2)
    assert got == want


def test_traffic_record_only_for_the_profiled_source(tmp_path):
    """A summary's DRAM bytes count only while the kernel source it was taken
    on is unchanged (its sha256 is recorded in the summary)."""
    import hashlib
    src = tmp_path / "k.cu"
    src.write_bytes(b"// kernel source\n")
    h = hashlib.sha256(src.read_bytes()).hexdigest()
    summ = tmp_path / "summary.md"
    summ.write_text(f"- dram_bytes_per_launch: 149500000\n- kernel_source_sha256: `{h}`\n")
    assert bench.traffic_record(str(summ), str(src)) == 149500000.0
    src.write_bytes(b"// kernel source\n// changed\n")
    assert bench.traffic_record(str(summ), str(src)) is None
    assert bench.traffic_record(str(tmp_path / "no_such_summary.md"), str(src)) is None


class _FakeSmi:
    def __init__(self, out):
        self.out = out

    def terminate(self):
        pass

    def communicate(self, timeout=None):
        return self.out, ""


@pytest.mark.parametrize("rows,reasons", [
    (["0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active"] * 3, []),
    (["0, 1965, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
      "0, 1830, 1965, 999.0, 0x4, Not Active, Not Active, Not Active, Active"], ["sw_power_cap"]),
    (["0, 1200, 1965, 600.0, 0x8, Active, Not Active, Not Active, Not Active"], ["hw_slowdown"]),
])
def test_clock_record_reports_median_and_throttle_reasons(rows, reasons):
    cs = bench.ClockSampler(None)
    cs.proc = _FakeSmi("\n".join(rows + ["garbage line"]) + "\n")
    rec = cs.stop()
    assert rec["samples"] == len(rows)
    assert rec["reasons"] == reasons
    assert rec["sm_max_mhz"] == 1965.0
    sm = sorted(float(r.split(",")[1]) for r in rows)
    assert rec["sm_mhz"] == (sm[len(sm) // 2] if len(sm) % 2 else (sm[len(sm) // 2 - 1] + sm[len(sm) // 2]) / 2)


def test_clock_record_without_nvidia_smi():
    rec = bench.ClockSampler(None).stop()
    assert rec["samples"] == 0 and rec["reasons"] == ["nvidia-smi unavailable"]


def test_binding_roof_takes_the_slowest_resource_plus_serial_stages():
    wl = synth.workload("qwen3_8_flash_next_like")
    T, act = 8192, 500
    miss = 450 * 7077900
    r = bench.binding_roof(wl, T, act, miss, 50.0, 6500.0, 1400.0, 1.5, 80.0)
    assert r["binding"] == "pcie"
    assert r["t_pcie_ms"] == pytest.approx(miss / 50e9 * 1e3)
    assert r["t_hbm_ms"] == pytest.approx(bench.layer_bytes(wl, act, T) / 6500e9 * 1e3)
    flops = 6.0 * T * 10 * 4096 * 1024 + 6.0 * T * 4096 * 1024
    assert r["t_tc_ms"] == pytest.approx(flops / 1400e12 * 1e3)
    assert r["tau_ms"] == pytest.approx(r["t_pcie_ms"] + 1.5)
    assert r["frac_of_tau"] == pytest.approx(r["tau_ms"] / 80.0)
    # all resident: nothing staged, the tensor work binds
    r = bench.binding_roof(wl, T, act, 0, 50.0, 6500.0, 1400.0, 1.5, 3.0)
    assert r["binding"] == "tc" and r["t_pcie_ms"] == 0.0


def test_default_workload_is_the_largest_single_gpu_layer():
    a = bench.parse([])
    wl = synth.workload(a.workload)
    assert a.workload == "qwen3_8_flash_next_like" and a.tokens == wl.prefill_tokens == 8192
    assert a.slots == "workload" and a.numerics == "exact" and a.warmup >= 3
    sizes = {n: w.n_experts * w.expert_bytes() for n, w in synth.WORKLOADS.items()}
    assert max(sizes, key=sizes.get) == a.workload


class _FakeNvml:
    """Stands in for pynvml: two 64-bit affinity words for the GPU."""

    def __init__(self, words, fail=False):
        self.words, self.fail = words, fail

    def nvmlInit(self):
        if self.fail:
            raise RuntimeError("no driver")

    def nvmlDeviceGetHandleByIndex(self, i):
        return ("index", i)

    def nvmlDeviceGetCpuAffinity(self, h, n):
        return self.words[:n] + [0] * max(0, n - len(self.words))


def test_gpu_local_cpus_intersects_nvml_affinity_with_allowed_cpus():
    allowed = os.sched_getaffinity(0)
    # every allowed CPU below 128 marked local, plus one that is not allowed
    words = [0, 0]
    for c in allowed:
        if c < 128:
            words[c // 64] |= 1 << (c % 64)
    extra = next((c for c in range(128) if c not in allowed), None)
    if extra is not None:
        words[extra // 64] |= 1 << (extra % 64)
    got = bench.gpu_local_cpus(None, 0, nvml=_FakeNvml(words))
    want = {c for c in allowed if c < 128}
    assert got == (want or None)


def test_gpu_local_cpus_gives_none_without_nvml_or_overlap():
    assert bench.gpu_local_cpus(None, 0, nvml=_FakeNvml([0, 0], fail=True)) is None
    assert bench.gpu_local_cpus(None, 0, nvml=_FakeNvml([0, 0])) is None
