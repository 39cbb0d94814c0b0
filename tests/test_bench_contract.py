"""The JSON line `bench.py` prints, checked on the CPU: `main()` runs with its GPU timing
legs replaced by fixed numbers, so the assembly of the line (keys, units, derived values,
the warm-up floor, the nested roofline / e2e / cpu_baseline / clocks objects) is tested
without a device. The timing legs themselves run only on a GPU."""

import json
import os

import pytest
import torch

import bench

STEPS = 10
BYTES_PER_STEP = 5.0e9
MS_PER_STEP = 1.0


def _fake_time_ours(w, steps, warmup, device, dist, e2e=True, clocks=True, local_rank=0):
    res = {"ms_total": MS_PER_STEP * steps, "bytes": BYTES_PER_STEP * steps, "launches": 5 * steps,
           "seq_tokens": 1000 * steps, "kernel_ms_mean": 0.9, "kernel_bytes_mean": BYTES_PER_STEP,
           "clocks": {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 3} if clocks else None,
           "num_cow": 0, "prefix_report": None}
    if e2e:
        res["e2e"] = {"ms_total": 1.1 * steps, "bytes": BYTES_PER_STEP * steps, "h2d": 7, "d2h": 3,
                      "steps": steps}
    return res


def _fake_time_extend(name, steps, warmup, device, subset=0):
    return {"workload": name, "ms_per_call": 0.4, "kv_gbs": 6000.0, "tflops": 700.0, "query_rows": 16,
            "kv_bytes": 1, "flops": 1}


@pytest.fixture
def line(monkeypatch, capsys):
    monkeypatch.setattr(bench, "time_ours", _fake_time_ours)
    monkeypatch.setattr(bench, "time_extend", _fake_time_extend)
    monkeypatch.setattr(bench, "cpu_baseline_obj",
                        lambda w, budget, subset=0: {"value": 0.07, "unit": "GB/s", "cores": 1,
                                                     "kind": "oracle", "sample": "fixed"})
    monkeypatch.setattr(torch.cuda, "is_available", lambda: True)
    monkeypatch.setattr(torch.cuda, "set_device", lambda d: None)
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.main(["--steps", str(STEPS), "--warmup", "1", "--also", "long_fp8,prefill_8x2k,spec4_mix"]) == 0
    out = [l for l in capsys.readouterr().out.splitlines() if l.strip()]
    assert len(out) == 1, "exactly one JSON line"
    return json.loads(out[0])


def test_top_level_keys_and_values(line):
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e",
              "gpu_launches", "clocks"):
        assert k in line, k
    assert line["metric"] == bench.METRIC and line["unit"] == "GB/s"
    assert line["n_gpus"] == 1 and line["steps"] == STEPS
    assert line["warmup"] == 3                                   # raised to the floor of 3
    assert line["higher_is_better"] is True and line["scaling"] == "weak" and line["vs_baseline"] is None
    assert line["data"] == "synthetic" and line["dtype"] == "bf16"
    assert line["config"]["workload"] == "llama13b_mix"
    assert line["value"] == pytest.approx(BYTES_PER_STEP / (MS_PER_STEP / 1e3) / 1e9)
    assert line["ms_per_step"] == pytest.approx(MS_PER_STEP)
    assert line["gpu_launches"] == 5 * STEPS


def test_nested_objects(line):
    r = line["roofline"]
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in r, k
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(BYTES_PER_STEP / 0.9e-3 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"])
    hbm, src = bench.peaks()                      # the measured copy bandwidth, else the fallback
    assert r["peak"] == pytest.approx(hbm) and r["peak_source"].startswith(src)
    e = line["e2e"]
    assert e["unit"] == "GB/s" and e["h2d_bytes_per_step"] == 7 and e["d2h_bytes_per_step"] == 3
    assert e["value"] == pytest.approx(BYTES_PER_STEP / 1.1e-3 / 1e9)
    c = line["cpu_baseline"]
    assert {"value", "unit", "cores", "kind", "sample"} <= set(c) and c["kind"] == "oracle"
    assert {"sm_mhz", "sm_max_mhz", "reasons"} <= set(line["clocks"])
    names = [x["workload"] for x in line["extend"]]
    assert names == ["prefill_8x2k", "spec4_mix"]
    pre, spec = line["extend"]
    assert pre["roofline"]["bound"] == "tensor" and pre["roofline"]["unit"] == "TFLOP/s"
    assert pre["roofline"]["peak"] == pytest.approx(bench.bf16_peak()[0])
    assert spec["roofline"]["bound"] == "hbm" and spec["roofline"]["frac"] == pytest.approx(6000.0 / r["peak"])
    assert [x["workload"] for x in line["also"]] == ["long_fp8"]


def test_clock_samples_inside_the_timed_window(tmp_path, monkeypatch):
    """ClockSampler.stop: median SM clock, max clock and active throttle reasons of the
    samples inside the timed window only (nvidia-smi replaced by a prepared CSV)."""
    import datetime
    monkeypatch.setenv("PA_CLOCKS_DIR", str(tmp_path))
    s = bench.ClockSampler(0)
    t0 = datetime.datetime(2026, 1, 1, 12, 0, 0)

    def row(dt, clk, reasons=("Not Active",) * 4):
        ts = (t0 + datetime.timedelta(seconds=dt)).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        return f"{ts}, 0, {clk}, 1965, 900.0, 0x0, " + ", ".join(reasons) + "\n"
    with open(s.path, "w") as f:
        f.write(row(0.0, 1200))                                           # before the window
        f.write(row(1.0, 1965))
        f.write(row(1.1, 1950, ("Not Active", "Not Active", "Not Active", "Active")))
        f.write(row(1.2, 1965))
        f.write("garbage line\n")
        f.write(row(3.0, 800, ("Active", "Not Active", "Not Active", "Not Active")))  # after it

    class FakeProc:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0

        def kill(self):
            pass
    s.proc, s.f = FakeProc(), open(tmp_path / "unused.csv", "w")
    w0 = (t0 + datetime.timedelta(seconds=0.9)).timestamp()
    w1 = (t0 + datetime.timedelta(seconds=1.3)).timestamp()
    c = s.stop((w0, w1))
    assert c["samples"] == 3 and c["sm_mhz"] == 1965.0 and c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"]


def test_nvml_clock_samples_inside_the_timed_window(tmp_path):
    """NvmlClockSampler.stop: the same summary from the NVML child's CSV lines (wall
    time, SM clock, max clock, power, four reason bits), inside the window only."""
    class FakeProps:
        uuid, pci_domain_id, pci_bus_id, pci_device_id = "abc", 0, 0x1b, 0

    s = bench.NvmlClockSampler.__new__(bench.NvmlClockSampler)
    s.interval, s.path, s.uuid, s.bus = 0.002, str(tmp_path / "n.csv"), FakeProps.uuid, "x"
    with open(s.path, "w") as f:
        f.write("ready\n")
        f.write("99.000,1200,1965,300.0,0,0,0,0\n")                       # before the window
        for k, clk in enumerate((1965, 1950, 1965, 1965)):
            f.write(f"{100.0 + 0.002 * k:.6f},{clk},1965,950.0,0,0,0,{1 if k == 1 else 0}\n")
        f.write("bad,line\n")
        f.write("200.000,800,1965,100.0,1,0,0,0\n")                        # after it

    class FakeProc:
        def poll(self):
            return 0
    s.proc, s.f = FakeProc(), open(tmp_path / "unused.csv", "w")
    c = s.stop((99.5, 101.0))
    assert c["samples"] == 4 and c["sm_mhz"] == 1965.0 and c["sm_max_mhz"] == 1965.0 and c["sm_mhz_min"] == 1950
    assert c["reasons"] == ["sw_power_cap"] and c["power_w_median"] == 950.0


def test_traffic_is_reported_only_for_the_captured_kernel_source(tmp_path, monkeypatch):
    import json as _json
    import shutil
    rec = _json.load(open(os.path.join(bench.ROOT, "profiles", "partition_kernel_traffic.json")))
    ratio = rec["traffic_per_algorithmic_byte"]["llama13b_mix"]
    assert bench.kernel_traffic("llama13b_mix", 1.0e9) == pytest.approx(ratio * 1.0e9)
    assert bench.kernel_traffic("tiny", 1.0e9) is None                 # no capture for it
    # a copy of the tree: host code outside the partition kernel may change (the figure
    # stays); one byte more inside the kernel's source drops it
    for d in ("profiles", os.path.join("paged_kv_cache_436_b200", "csrc")):
        shutil.copytree(os.path.join(bench.ROOT, d), tmp_path / d)
    path = tmp_path / "paged_kv_cache_436_b200" / "csrc" / "pa_decode.cu"
    with open(path, "a") as f:
        f.write("\n// host code after the kernels\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.kernel_traffic("llama13b_mix", 1.0e9) == pytest.approx(ratio * 1.0e9)
    src = path.read_text()
    i = src.index("// partition kernel")
    path.write_text(src[:i] + "// partition kernel \n" + src[i + len("// partition kernel"):])
    assert bench.kernel_traffic("llama13b_mix", 1.0e9) is None
