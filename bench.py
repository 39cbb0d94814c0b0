"""Benchmark of the paged-KV-cache decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload llama13b_mix|long_fp8|...] [--also long_fp8] [--no-e2e]

A step is one pass of the whole hot path over the batch: host block bookkeeping
(C++), one metadata upload, block-table patch, copy-on-write block copies, the
KV-cache write of every sequence's new token, and paged decode attention (plan,
partition kernel, log-sum-exp merge). Each sequence appends one token per step,
so contexts grow by one token per step, as in serving.

Metric: KV-read GB/s = the bytes a decode step must move at minimum (every
context token's K and V row once per kv head, q, out, block-table entries,
context lengths) / device time of the whole step; also sequence-tokens/s
(context tokens attended per second). The KV read per step (10.5 GB for the 13B
mix, 2.1 GB for the 32K fp8 case) is far larger than the 126 MB L2, so no flush
is needed between steps.

N > 1 (torchrun): replicas. Each rank runs the same workload on its own GPU with
no collective on the data path (sequences are independent); the step time is the
max over ranks and `value` is the sum of all ranks' bytes over that time.

--impl reference times the float64 CPU oracle (the correctness reference) on a
bounded sample of the same workload, on the host's cores, on rank 0 only.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode attention KV-read GB/s (% of B200 HBM peak); seq-tokens/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0   # burst dense bf16 figure of the same earlier measurement


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_traffic(workload: str, bytes_per_launch: float):
    """DRAM bytes per partition-kernel launch, scaled from the committed ncu capture's
    traffic / algorithmic-byte ratio; None when the kernel source changed since."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "partition_kernel_traffic.json")) as f:
            rec = json.load(f)
        csrc = os.path.join(ROOT, "paged_kv_cache_436_b200", "csrc")
        with open(os.path.join(csrc, "pa_decode.cu")) as f:
            dec = f.read()
        with open(os.path.join(csrc, "pa_device.cuh")) as f:
            dev = f.read()
        # the partition kernel's own source (from its banner to the merge kernel's) and the
        # device helpers it uses: host code around it may change without a recapture
        a, b = dec.index("// partition kernel"), dec.index("// log-sum-exp merge of partitions")
        h = hashlib.sha256()
        h.update(dec[a:b].encode())
        h.update(dev.encode())
        if h.hexdigest() != rec["source_sha256"]:
            return None
        base = workload.split("[")[0]
        return rec["traffic_per_algorithmic_byte"][base] * bytes_per_launch
    except (OSError, KeyError, ValueError):
        return None


def decode_bytes(lens, hkv, hq, d, kv_bytes, q_bytes, bs) -> int:
    """Algorithmic bytes of one decode step: K and V of every context token once per
    kv head, q in, out back, the block-table entries read, the context lengths."""
    lens = np.asarray(lens, dtype=np.int64)
    kv = int(2 * lens.sum() * hkv * d * kv_bytes)
    s = len(lens)
    return kv + 2 * s * hq * d * q_bytes + int(4 * ((lens + bs - 1) // bs).sum()) + 4 * s


# ---------------------------------------------------------------------------
# distributed plumbing (replicas: only timing is reduced across ranks)
# ---------------------------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, backend):
    if world <= 1:
        return None
    import datetime
    import torch.distributed as dist
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def reduce_max(x: float, dist, device=None) -> float:
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(x: float, dist, device=None) -> float:
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(dist, device=None):
    if dist is not None:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        # the raw samples (the JSON line carries their summary); PA_CLOCKS_DIR keeps them elsewhere
        import tempfile
        out_dir = os.environ.get("PA_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out_dir, f"pa_clocks_gpu{gpu_index}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self, window=None):
        """Median SM clock, max clock and throttle reasons of the samples taken inside
        `window` = (t_start, t_end) host wall-clock seconds (all samples if None)."""
        import datetime
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                clk, cmax = float(parts[2]), float(parts[3])
            except ValueError:
                continue
            if window is not None and not (window[0] - 0.05 <= ts <= window[1] + 0.05):
                continue
            sm.append(clk)
            smax.append(cmax)
            for n, v in zip(names, parts[6:10]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# Reads the SM clock, its maximum, the power draw and the clock-event reasons every
# `interval` seconds through NVML (read-only queries) and prints one CSV line per
# sample with its wall-clock time; the device is found by the UUID or PCI bus id the
# parent passes (CUDA and NVML number devices differently).
_NVML_LOOP = r"""
import sys, time, pynvml as N
uuid, bus, interval = sys.argv[1], sys.argv[2], float(sys.argv[3])
N.nvmlInit()
h = None
for cand in (uuid, "GPU-" + uuid):
    try:
        h = N.nvmlDeviceGetHandleByUUID(cand); break
    except Exception:
        pass
if h is None:
    h = N.nvmlDeviceGetHandleByPciBusId(bus)
cmax = N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM)
bits = (N.nvmlClocksEventReasonHwSlowdown, N.nvmlClocksEventReasonHwThermalSlowdown,
        N.nvmlClocksEventReasonSwThermalSlowdown, N.nvmlClocksEventReasonSwPowerCap)
print("ready", flush=True)
while True:
    t = time.time()
    clk = N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM)
    r = N.nvmlDeviceGetCurrentClocksEventReasons(h)
    pw = N.nvmlDeviceGetPowerUsage(h) / 1000.0
    print("%.6f,%d,%d,%.1f,%s" % (t, clk, cmax, pw, ",".join("1" if r & b else "0" for b in bits)), flush=True)
    time.sleep(max(0.0, interval - (time.time() - t)))
"""


class NvmlClockSampler:
    """Clock record of the timed region sampled every 2 ms through NVML in a child
    process (no GIL shared with the timing loop): a region of a few tens of
    milliseconds still gets a dozen samples. Same summary as ClockSampler.stop."""

    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, device, interval=0.002):
        import tempfile
        import torch
        props = torch.cuda.get_device_properties(device)
        self.uuid = str(props.uuid)
        self.bus = "%08X:%02X:%02X.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
        self.interval = interval
        out_dir = os.environ.get("PA_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out_dir, f"pa_clocks_nvml_{os.getpid()}.csv")
        self.proc = None

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen([sys.executable, "-c", _NVML_LOOP, self.uuid, self.bus, str(self.interval)],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
            t0 = time.time()
            while time.time() - t0 < 30:             # until the first sample is written
                time.sleep(0.05)
                if self.proc.poll() is not None:
                    raise RuntimeError("NVML sampler exited")
                with open(self.path) as g:
                    if len(g.read().splitlines()) >= 2:
                        return True
            raise RuntimeError("NVML sampler gave no sample")
        except Exception:
            self.stop_proc()
            self.proc = None
            return False

    def stop_proc(self):
        if self.proc is not None and self.proc.poll() is None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        try:
            self.f.close()
        except Exception:
            pass

    def stop(self, window=None):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        time.sleep(0.01)
        self.stop_proc()
        sm, smax, pw, reasons = [], [], [], set()
        for line in open(self.path):
            parts = line.strip().split(",")
            if len(parts) != 8:
                continue
            try:
                ts, clk, cmax, p = float(parts[0]), float(parts[1]), float(parts[2]), float(parts[3])
            except ValueError:
                continue
            if window is not None and not (window[0] <= ts <= window[1]):
                continue
            sm.append(clk)
            smax.append(cmax)
            pw.append(p)
            for n, v in zip(self.NAMES, parts[4:8]):
                if v == "1":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm), "sm_mhz_min": min(sm), "power_w_median": statistics.median(pw),
                "source": "NVML every %g ms in the timed region" % (self.interval * 1e3)}


def clock_sampler(device, local_rank):
    """NVML sampling when it works, else nvidia-smi at 100 ms."""
    s = NvmlClockSampler(device)
    if s.start():
        return s
    s = ClockSampler(local_rank)
    s.start()
    return s


# ---------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------

def build_engine(w, growth, device):
    """Engine for workload `w` with room for `growth` more tokens per sequence; the
    cache is filled with seeded N(0,1) draws on the device; every sequence holds its
    history (L - 1 tokens), so the timed steps append from position L - 1."""
    import torch
    import synthetic
    from paged_kv_cache_436_b200.engine import DecodeEngine
    w = synthetic.grown(w, growth)
    eng = DecodeEngine(num_seqs=w.num_seqs, num_q_heads=w.num_q_heads, num_kv_heads=w.num_kv_heads,
                       head_dim=w.head_dim, block_size=w.block_size, kv_dtype=w.kv_dtype, q_dtype=w.q_dtype,
                       num_blocks=w.num_blocks, initial_order=w.initial_order,
                       max_blocks_per_seq=w.max_blocks_per_seq(growth),
                       max_context_len=w.max_context_len + growth, scale=w.scale, device=device)
    if w.kv_dtype == "e4m3":
        kc, ks = synthetic.normal_e4m3_codes(tuple(eng.k_cache.shape), w.seed * 10 + 1, device)
        eng.k_cache.copy_(kc)
        del kc
        vc, vs = synthetic.normal_e4m3_codes(tuple(eng.v_cache.shape), w.seed * 10 + 2, device)
        eng.v_cache.copy_(vc)
        del vc
        eng.cache.desc.k_scale, eng.cache.desc.v_scale = ks, vs
    else:
        synthetic.fill_normal_(eng.k_cache, w.kv_dtype, w.seed * 10 + 1)
        synthetic.fill_normal_(eng.v_cache, w.kv_dtype, w.seed * 10 + 2)
    if getattr(w, "beam_width", 0):
        # each request's prompt is written once; its other beams fork it
        W = w.beam_width
        for r in range(w.num_seqs // W):
            eng.extend(r * W, w.context_lens[r * W] - 1)
            for j in range(1, W):
                eng.fork(r * W, r * W + j)
    elif w.prefix_len:
        # requests admitted through the prefix cache: all carry the same history, so
        # every request after the first reuses its full blocks and allocates only its
        # partial block and private tokens (the step appends each request's last token)
        import paged_kv_cache_436_b200 as pa
        rng = np.random.default_rng(w.seed + 5)
        hist = rng.integers(0, 32000, size=w.prefix_len).tolist()
        cache = pa.PrefixCache(w.block_size)
        t0 = time.perf_counter()
        for s, priv in enumerate(w.private_lens):
            prompt = hist + rng.integers(0, 32000, size=priv - 1).tolist()
            n = cache.match(eng.pool, prompt, eng.bt_host[s])
            eng.lens[s] = n * w.block_size
            eng.extend(s, len(prompt) - n * w.block_size)
            cache.insert(eng.pool, prompt, eng.bt_host[s])
        eng.prefix_report = {"host_us_per_request": (time.perf_counter() - t0) / w.num_seqs * 1e6,
                             "kv_blocks_held": w.num_blocks - eng.pool.num_free(),
                             "kv_blocks_without_prefix_cache": int(sum(-(-(w.prefix_len + p - 1) // w.block_size)
                                                                       for p in w.private_lens)),
                             "cached_blocks": len(cache)}
        eng.prefix_cache = cache
    else:
        for s, L in enumerate(w.context_lens):
            eng.extend(s, L - 1)
    eng.upload_tables()
    torch.cuda.synchronize(device)
    return eng


class StepRunner:
    """Runs engine steps with events around the partition kernel (decode stage 1)."""

    def __init__(self, eng, w, n_inputs, device):
        import torch
        import synthetic
        import paged_kv_cache_436_b200 as pa
        self.pa, self.torch = pa, torch
        self.eng, self.w, self.device = eng, w, device
        self.inputs = []
        for i in range(n_inputs):
            q, k, v = synthetic.step_inputs(w, i, device=device)
            self.inputs.append((q, k, v))
        self.out = torch.empty_like(self.inputs[0][0])
        self.stream = torch.cuda.current_stream(device)
        self.kv_bytes = 1 if w.kv_dtype == "e4m3" else 2
        self.q_bytes = 2

    def step(self, i, ev_pair=None):
        """One native engine step on device-resident inputs; CUDA events around the
        partition kernel. Beam workloads re-select their beams first (host reorder +
        table upload). Returns (decode bytes, kernel launches)."""
        q, k, v = self.inputs[i % len(self.inputs)]
        width = getattr(self.w, "beam_width", 0)
        if width:
            import synthetic
            self.eng.reorder(synthetic.beam_parents(self.w.num_seqs // width, width, i, self.w.seed))
        self.eng.step(q, k, v, self.out, events=ev_pair)
        nbytes = decode_bytes(self.eng.lens, self.w.num_kv_heads, self.w.num_q_heads, self.w.head_dim,
                              self.kv_bytes, self.q_bytes, self.w.block_size)
        return nbytes, self.eng.last_step()[2]


def time_ours(w, steps, warmup, device, dist, e2e=True, clocks=True, local_rank=0):
    import torch
    n_e2e = steps if e2e else 0
    growth = warmup + steps + (warmup + n_e2e if e2e else 0) + 2
    eng = build_engine(w, growth, device)
    run = StepRunner(eng, w, 4, device)
    for i in range(warmup):
        run.step(i)
    torch.cuda.synchronize(device)
    barrier(dist, device)
    sampler = clock_sampler(device, local_rank) if clocks else None
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in kev:            # torch creates the CUDA events at their first record
        a.record()
        b.record()
    torch.cuda.synchronize(device)
    barrier(dist, device)
    total_bytes, launches, lens_sum, kbytes = 0, 0, 0, []
    wall0 = time.time()
    t0.record()
    for i in range(steps):
        nb, nl = run.step(i, kev[i])
        total_bytes += nb
        launches += nl
        lens_sum += int(eng.lens.sum())
        kbytes.append(nb)
    t1.record()
    torch.cuda.synchronize(device)
    wall1 = time.time()
    clk = sampler.stop((wall0, wall1)) if sampler else None
    ms = t0.elapsed_time(t1)
    kernel_ms = [a.elapsed_time(b) for a, b in kev]
    ms_max = reduce_max(ms, dist, device)
    res = {"ms_total": ms_max, "bytes": total_bytes, "launches": launches, "seq_tokens": lens_sum,
           "kernel_ms_mean": float(np.mean(kernel_ms)), "kernel_bytes_mean": float(np.mean(kbytes)),
           "clocks": clk, "num_cow": eng.last_step()[0],
           "prefix_report": getattr(eng, "prefix_report", None)}
    if e2e:
        # the same steps through the host-buffer API: pinned inputs copied in and the
        # output copied out every step, overlapped with the kernels of adjacent steps
        from paged_kv_cache_436_b200.engine import HostPipeline
        q0, k0, v0 = run.inputs[0]
        hq, hk, hv = q0.cpu().pin_memory(), k0.cpu().pin_memory(), v0.cpu().pin_memory()
        hout = [torch.empty_like(run.out, device="cpu").pin_memory() for _ in range(2)]
        pipe = HostPipeline(eng)
        for i in range(warmup):
            pipe.submit(hq, hk, hv, hout[i & 1])
        pipe.sync()
        barrier(dist, device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        eb = 0
        e0.record(pipe.compute)
        pipe.h2d.wait_event(e0)
        for i in range(n_e2e):
            pipe.submit(hq, hk, hv, hout[i & 1])
            eb += decode_bytes(eng.lens, w.num_kv_heads, w.num_q_heads, w.head_dim, run.kv_bytes,
                               run.q_bytes, w.block_size)
        e1.record(pipe.d2h)
        pipe.sync()
        ems = reduce_max(e0.elapsed_time(e1), dist, device)
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv)) + eng.meta_bytes
        d2h = hout[0].numel() * hout[0].element_size()
        res["e2e"] = {"ms_total": ems, "bytes": eb, "h2d": h2d, "d2h": d2h, "steps": n_e2e}
    del eng, run
    torch.cuda.empty_cache()
    return res


def time_extend(name, steps, warmup, device, subset=0):
    """pa_extend alone (the tensor-core multi-query kernel and its merge), timed with
    CUDA events: `spec4_mix` = 4 draft tokens per sequence over the 13B mix contexts
    (speculative verification; HBM-bound), `prefill_8x2k` = 8 whole 2048-token prompts
    (prefill from an empty context; compute-bound)."""
    import torch
    import synthetic
    import paged_kv_cache_436_b200 as pa
    if name in ("spec4_mix", "spec4_long_fp8"):   # 4 draft tokens over the 13B mix / the 32K E4M3 cache
        base = synthetic.make("llama13b_mix" if name == "spec4_mix" else "long_fp8")
        w, qlen = (synthetic.subset(base, subset) if subset else base), 4
    elif name == "prefill_gqa_8x2k":   # Llama-3-8B attention shapes: 32 q heads over 8 kv heads
        w = synthetic.custom(8, 32, 8, 128, 16, "bf16", "bf16", [2048] * 8, 4372, pool_factor=1.05)
        qlen = 2048
    else:
        w = synthetic.custom(8, 32, 32, 128, 16, "bf16", "bf16", [2048] * 8, 4371, pool_factor=1.05)
        qlen = 2048
    eng = build_engine(w, 1, device)                            # every sequence holds L - 1 tokens
    for s in range(w.num_seqs):
        eng.extend(s, 1)                                        # ... and now all L
    eng.upload_tables()
    qlens = [min(qlen, L) for L in w.context_lens]
    qs = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    T = int(qs[-1])
    q = synthetic.normal_values((T, w.num_q_heads, w.head_dim), w.q_dtype, w.seed + 11, device)
    out = torch.empty_like(q)
    ws = torch.empty(pa.extend_workspace_size(w.num_seqs, T, w.num_q_heads, w.head_dim, eng.max_context_len),
                     dtype=torch.uint8, device=device)
    qs_dev = torch.from_numpy(qs).to(device)

    def call():
        pa.extend(q, eng.cache, qs_dev, eng.bt_dev, eng.lens_dev, eng.max_context_len, w.scale, out, ws)

    def timed(fn):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            fn()
        e1.record()
        torch.cuda.synchronize(device)
        return e0.elapsed_time(e1) / steps

    ms = timed(call)
    prefill = None
    if name.startswith("prefill"):
        # the whole prefill step: the prompts' K / V into the cache plus the attention, as
        # one fused pa_prefill and as pa_reshape_and_cache followed by pa_extend
        k_new = synthetic.normal_values((T, w.num_kv_heads, w.head_dim), w.kv_dtype, w.seed + 12, device)
        v_new = synthetic.normal_values((T, w.num_kv_heads, w.head_dim), w.kv_dtype, w.seed + 13, device)
        BS = w.block_size
        slots = np.concatenate([eng.bt_host[s, np.arange(L) // BS].astype(np.int64) * BS + np.arange(L) % BS
                                for s, L in enumerate(w.context_lens)])
        slots_dev = torch.from_numpy(slots).to(device)

        def fused():
            pa.prefill(q, k_new, v_new, eng.cache, qs_dev, eng.bt_dev, eng.lens_dev, eng.max_context_len, w.scale,
                       out, ws)

        def two_pass():
            pa.reshape_and_cache(k_new, v_new, slots_dev, eng.cache)
            call()

        prefill = {"fused_ms": timed(fused), "reshape_then_extend_ms": timed(two_pass)}
    lens = np.asarray(w.context_lens, dtype=np.int64)
    kvb = 1 if w.kv_dtype == "e4m3" else 2
    kv_bytes = int(2 * lens.sum() * w.num_kv_heads * w.head_dim * kvb) + 2 * T * w.num_q_heads * w.head_dim * 2
    flops = 0
    for L, Qn in zip(lens, qlens):
        pos = L - Qn + np.arange(Qn, dtype=np.int64)
        flops += int(4 * w.num_q_heads * w.head_dim * (pos + 1).sum())
    del eng
    torch.cuda.empty_cache()
    res = {"workload": name, "ms_per_call": ms, "kv_gbs": kv_bytes / (ms / 1e3) / 1e9,
           "tflops": flops / (ms / 1e3) / 1e12, "query_rows": T, "kv_bytes": kv_bytes, "flops": flops}
    if prefill is not None:
        prefill["fused_tflops"] = flops / (prefill["fused_ms"] / 1e3) / 1e12
        prefill["note"] = ("whole prefill step = the prompts' K/V written to the cache + attention; "
                           "ms_per_call / tflops above time the attention alone (pa_extend)")
        res["prefill_step"] = prefill
    return res


# ---------------------------------------------------------------------------
# the oracle on the host cores (cpu_baseline and --impl reference)
# ---------------------------------------------------------------------------

def _sample_item(w, s):
    """Blocks of sequence s for the oracle, drawn on the host from a per-sequence seed
    (the same in every process), laid out 0..n-1."""
    import synthetic
    L = w.context_lens[s]
    nbk = -(-L // w.block_size)
    shape = (nbk, w.num_kv_heads, w.block_size, w.head_dim)
    seed = w.seed * 7919 + 2 * s
    if w.kv_dtype == "e4m3":
        rng = np.random.default_rng(seed)
        kc = rng.integers(0, 0x7E, size=shape, dtype=np.uint8)
        vc = rng.integers(0, 0x7E, size=shape, dtype=np.uint8)
        ks = vs = 6.0 / 448
    else:
        kc = synthetic.normal_codes(shape, w.kv_dtype, seed + 1).numpy().view(np.uint16)
        vc = synthetic.normal_codes(shape, w.kv_dtype, seed + 2).numpy().view(np.uint16)
        ks = vs = 1.0
    return (s, L, kc, vc, ks, vs, np.arange(nbk, dtype=np.int64)[None, :])


def _oracle_q(w):
    import synthetic
    return synthetic.normal_codes((w.num_seqs, w.num_q_heads, w.head_dim), w.q_dtype, w.seed + 9).numpy().view(
        np.uint16)


def _seq_bytes(w, s):
    kvb = 1 if w.kv_dtype == "e4m3" else 2
    return decode_bytes([w.context_lens[s]], w.num_kv_heads, w.num_q_heads, w.head_dim, kvb, 2, w.block_size)


def _seq_order(w):
    return [int(s) for s in np.random.default_rng(w.seed + 7).permutation(w.num_seqs)]


def oracle_sample_inputs(w, budget_s):
    """A bounded sample of the workload for the float64 oracle: whole sequences (all
    heads) in a seeded order, added one at a time until the oracle has spent about
    `budget_s` seconds of CPU time on them."""
    q = _oracle_q(w)
    items, spent = [], 0.0
    for s in _seq_order(w):
        item = _sample_item(w, s)
        spent += oracle_run(w, q, [item])[2]
        items.append(item)
        if spent >= budget_s:
            break
    return q, items


def oracle_run(w, q, items):
    """One pass of the oracle over the sample; returns (bytes, tokens, cpu seconds)."""
    from threadpoolctl import threadpool_limits
    from oracle import attention as oatt
    nbytes, ntok = 0, 0
    with threadpool_limits(limits=1):
        t0 = time.process_time()
        for s, L, kc, vc, ks, vs, bt in items:
            oatt.paged_decode(q[s:s + 1], w.q_dtype, kc, vc, w.kv_dtype, ks, vs, bt, [L], w.scale)
            nbytes += _seq_bytes(w, s)
            ntok += L
        dt = time.process_time() - t0
    return nbytes, ntok, dt


def sample_text(w, items, seconds, passes=1):
    lens = [it[1] for it in items]
    return (f"float64 numpy oracle on 1 thread (BLAS limited to 1): {len(items)} whole sequences of the "
            f"{w.name} workload (context lengths {min(lens)}..{max(lens)}, all {w.num_q_heads} q heads), "
            f"{passes} pass(es), {seconds:.1f} s of CPU time")


def _workload_by_name(name, subset):
    import synthetic
    w = synthetic.make(name)
    return synthetic.subset(w, subset) if subset else w


def _pool_worker(name, subset, seqs, conn):
    """One oracle process of the all-cores baseline (started with spawn, BLAS limited to
    one thread): draws its sequences, then runs one timed pass per "run" command."""
    for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ[var] = "1"
    sys.path.insert(0, ROOT)
    w = _workload_by_name(name, subset)
    q = _oracle_q(w)
    items = [_sample_item(w, s) for s in seqs]
    conn.send("ready")
    while conn.recv() == "run":
        t0 = time.perf_counter()
        nb, nt, _ = oracle_run(w, q, items)
        conn.send((nb, nt, time.perf_counter() - t0))
    conn.close()


class OraclePool:
    """The float64 oracle on `workers` processes at once (one per host core), each over
    its share of a sample of whole sequences (longest-first onto the least-loaded
    process). A pass starts every process together; its time is the slowest process's."""

    def __init__(self, w, workers, budget_s, rate_1t, subset=0):
        import multiprocessing as mp
        self.w = w
        self.workers = max(1, int(workers))
        # whole sequences in the seeded order while the estimated single-thread time of
        # the sample stays within budget_s on every process
        quota = budget_s * rate_1t * self.workers
        chosen, tot = [], 0
        for s in _seq_order(w):
            b = _seq_bytes(w, s)
            if chosen and tot + b > quota:
                break
            chosen.append(s)
            tot += b
        loads = [0] * self.workers
        shares = [[] for _ in range(self.workers)]
        for s in sorted(chosen, key=lambda x: -_seq_bytes(w, x)):
            k = min(range(self.workers), key=lambda i: loads[i])
            shares[k].append(s)
            loads[k] += _seq_bytes(w, s)
        self.seqs = chosen
        ctx = mp.get_context("spawn")
        self.conns, self.procs = [], []
        for share in shares:
            if not share:
                continue
            a, b = ctx.Pipe()
            p = ctx.Process(target=_pool_worker, args=(w.name, subset, share, b), daemon=True)
            p.start()
            self.conns.append(a)
            self.procs.append(p)
        for c in self.conns:
            assert c.recv() == "ready"

    def run(self):
        for c in self.conns:
            c.send("run")
        res = [c.recv() for c in self.conns]
        return sum(r[0] for r in res), sum(r[1] for r in res), max(r[2] for r in res)

    def close(self):
        for c in self.conns:
            c.send("stop")
        for p in self.procs:
            p.join(timeout=30)

    def describe(self, seconds, passes):
        lens = [self.w.context_lens[s] for s in self.seqs]
        whole = len(self.seqs) == self.w.num_seqs
        return (f"float64 numpy oracle on {len(self.procs)} processes (one per host core, BLAS limited to 1 "
                f"thread each, started together): {'the whole' if whole else 'a sample of the'} "
                f"{self.w.name} workload, {len(self.seqs)} whole sequences (context lengths "
                f"{min(lens)}..{max(lens)}, all {self.w.num_q_heads} q heads), {passes} pass(es), "
                f"{seconds:.1f} s of wall time")


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline_obj(w, budget, subset=0):
    """The oracle on every host core (the headline figure) and on one thread (a second field)."""
    q, items = oracle_sample_inputs(w, budget)
    nb, nt, dt = oracle_run(w, q, items)
    one = {"value": nb / dt / 1e9, "unit": "GB/s", "cores": 1, "seq_tokens_per_s": nt / dt,
           "sample": sample_text(w, items, dt)}
    pool = OraclePool(w, host_cores(), budget, nb / dt, subset)
    try:
        pb, pt, pdt = pool.run()
        text = pool.describe(pdt, 1)
        cores = len(pool.procs)
    finally:
        pool.close()
    return {"value": pb / pdt / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "seq_tokens_per_s": pt / pdt, "sample": text, "single_thread": one}


def reference_arm(w, args):
    """--impl reference: the oracle on every host core, each step one pass over a bounded
    sample (all processes at once; the step time is the slowest process's)."""
    per_step = max(0.2, min(2.0, 120.0 / (args.steps + args.warmup)))
    q, items = oracle_sample_inputs(w, min(per_step, 1.0))
    nb, _, dt = oracle_run(w, q, items)
    pool = OraclePool(w, host_cores(), per_step, nb / dt, args.subset)
    try:
        for _ in range(args.warmup):
            pool.run()
        tb, tt, ts = 0, 0, 0.0
        for _ in range(args.steps):
            b, t, d = pool.run()
            tb, tt, ts = tb + b, tt + t, ts + d
        text = pool.describe(ts, args.steps) + "; ms_per_step is the time of one pass over this sample"
        cores = len(pool.procs)
    finally:
        pool.close()
    gbs = tb / ts / 1e9
    return {"metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ts / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": workload_config(w, 1), "seq_tokens_per_s": tt / ts,
            "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": text},
            "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------------------

def workload_config(w, n_gpus):
    return {"workload": w.name, "num_seqs": w.num_seqs, "num_q_heads": w.num_q_heads,
            "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim, "block_size": w.block_size,
            "kv_dtype": w.kv_dtype, "q_dtype": w.q_dtype, "sum_context_tokens": int(sum(w.context_lens)),
            "max_context_len": int(max(w.context_lens)), "partition_tokens": 512,
            "l2": "no flush: KV read per step far above the 126 MB L2",
            "parallelism": f"replicas{n_gpus}" if n_gpus > 1 else "single GPU"}


EXTEND_WORKLOADS = ("spec4_mix", "spec4_long_fp8", "prefill_8x2k", "prefill_gqa_8x2k")


def bf16_peak():
    """Dense bf16 TFLOP/s: the measured burst figure, else the earlier measurement."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def extend_roofline(e, hbm_peak):
    spec = e["workload"].startswith("spec")
    tensor_peak, tensor_src = bf16_peak()
    r = {"bound": "hbm" if spec else "tensor", "achieved": e["kv_gbs"] if spec else e["tflops"],
         "peak": hbm_peak if spec else tensor_peak, "unit": "GB/s" if spec else "TFLOP/s"}
    if not spec and tensor_src != "measured":
        r["peak_source"] = tensor_src
    r["frac"] = r["achieved"] / r["peak"]
    return r


def extend_only(args, world, rank, local):
    """`--workload spec4_mix|prefill_8x2k`: pa_extend alone on one GPU (a profiling and
    tuning entry; the default line reports these under "extend")."""
    import torch
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the product path has no CPU fallback)")
    import paged_kv_cache_436_b200 as pa
    pa.lib()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    e = time_extend(args.workload, args.steps, args.warmup, device, subset=args.subset)
    peak, _ = peaks()
    e["roofline"] = extend_roofline(e, peak)
    if rank == 0:
        print(json.dumps(e))
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llama13b_mix")
    ap.add_argument("--also", default="long_fp8,prefill_8x2k,spec4_mix,spec4_long_fp8",
                    help="further workloads reported in the same line ('' = none)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle's cpu_baseline leg")
    ap.add_argument("--subset", type=int, default=0,
                    help="only the first N sequences (a smaller case of the same shapes, for profiling)")
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)

    import synthetic
    world, rank, local = dist_env()
    if args.workload in EXTEND_WORKLOADS:
        return extend_only(args, world, rank, local)
    w = synthetic.make(args.workload)
    if args.subset:
        w = synthetic.subset(w, args.subset)

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(reference_arm(w, args)))
        return 0

    import torch
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the product path has no CPU fallback)")
    import paged_kv_cache_436_b200 as pa
    pa.lib()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist = init_dist(world, "nccl")
    try:
        res = time_ours(w, args.steps, args.warmup, device, dist, e2e=not args.no_e2e,
                        clocks=True, local_rank=local)
        also = []
        extend_entries = []
        for name in [a for a in args.also.split(",") if a]:
            if name in EXTEND_WORKLOADS:
                extend_entries.append(time_extend(name, max(3, args.steps // 5), args.warmup, device))
                continue
            if name == "beam5":
                wa = synthetic.beam_workload()
            elif name == "gqa_noshare":
                # the GQA-prefix shapes with every sequence holding its own blocks
                g = synthetic.make("gqa_prefix")
                wa = synthetic.custom(g.num_seqs, g.num_q_heads, g.num_kv_heads, g.head_dim, g.block_size,
                                      g.kv_dtype, g.q_dtype, g.context_lens, g.seed, pool_factor=1.1,
                                      scale=g.scale)
                wa.name = "gqa_noshare"
            else:
                wa = synthetic.make(name)
            if args.subset:
                wa = synthetic.subset(wa, max(1, args.subset * wa.num_seqs // 256))
            also.append((wa, time_ours(wa, args.steps, args.warmup, device, dist, e2e=False, clocks=False,
                                       local_rank=local)))
        peak, peak_src = peaks()
        all_bytes = reduce_sum(res["bytes"], dist, device)
        value = all_bytes / (res["ms_total"] / 1e3) / 1e9
        tokens = reduce_sum(res["seq_tokens"], dist, device) / (res["ms_total"] / 1e3)
        kern_gbs = res["kernel_bytes_mean"] / (res["kernel_ms_mean"] / 1e3) / 1e9
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": res["ms_total"] / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w.kv_dtype, "data": "synthetic",
            "config": workload_config(w, world),
            "seq_tokens_per_s": tokens,
            "pct_of_hbm": {"measured_copy": value / world / peak, "nominal_8tbs": value / world / NOMINAL_HBM_GBS},
            "roofline": {"bound": "hbm", "kernel": "partition_kernel (pa_decode stage 1)",
                         "achieved": kern_gbs, "peak": peak, "unit": "GB/s", "frac": kern_gbs / peak,
                         "peak_source": peak_src + " HBM copy bandwidth (MEASURED_PEAKS hbm_gbs)",
                         "frac_of_nominal_8tbs": kern_gbs / NOMINAL_HBM_GBS,
                         "bytes_per_launch": res["kernel_bytes_mean"], "ms_per_launch": res["kernel_ms_mean"],
                         "traffic": kernel_traffic(w.name, res["kernel_bytes_mean"])},
            "gpu_launches": res["launches"],
            "clocks": res["clocks"],
        }
        if "e2e" in res:
            e = res["e2e"]
            line["e2e"] = {"value": reduce_sum(e["bytes"], dist, device) / (e["ms_total"] / 1e3) / 1e9,
                           "unit": "GB/s", "h2d_bytes_per_step": e["h2d"], "d2h_bytes_per_step": e["d2h"],
                           "ms_per_step": e["ms_total"] / e["steps"]}
        for wa, ra in also:
            kg = ra["kernel_bytes_mean"] / (ra["kernel_ms_mean"] / 1e3) / 1e9
            entry = {"workload": wa.name,
                     "value": reduce_sum(ra["bytes"], dist, device) / (ra["ms_total"] / 1e3) / 1e9,
                     "unit": "GB/s", "ms_per_step": ra["ms_total"] / args.steps,
                     "seq_tokens_per_s": reduce_sum(ra["seq_tokens"], dist, device) / (ra["ms_total"] / 1e3),
                     "roofline": {"bound": "hbm", "achieved": kg, "peak": peak, "unit": "GB/s",
                                  "frac": kg / peak, "ms_per_launch": ra["kernel_ms_mean"],
                                  "traffic": kernel_traffic(wa.name, ra["kernel_bytes_mean"])}}
            if getattr(wa, "beam_width", 0):
                entry["note"] = ("logical bytes: each beam's whole context is counted; the beams of a "
                                 "request share their prompt blocks")
                entry["copy_on_write_pairs_last_step"] = ra["num_cow"]
            if wa.prefix_len:
                entry["note"] = ("logical bytes: the shared prefix is counted once per sequence; "
                                 "it is read from HBM about once and from L2 after that")
                entry["prefix_cache"] = ra.get("prefix_report")
            line.setdefault("also", []).append(entry)
        for e in extend_entries:
            e["roofline"] = extend_roofline(e, peak)
            line.setdefault("extend", []).append(e)
        if rank == 0 and world == 1 and not args.no_cpu:
            line["cpu_baseline"] = cpu_baseline_obj(w, args.cpu_budget, args.subset)
        if rank == 0:
            print(json.dumps(line))
    finally:
        if dist is not None:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
