"""CPU tests of bench.py's host logic: byte accounting, the max-over-ranks timing
reduction across 2 gloo ranks (replicas), and isolation of the product path from
the oracle."""

import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synthetic  # noqa: E402
from oracle import accounting  # noqa: E402


@pytest.mark.parametrize("name", synthetic.NAMES)
def test_decode_bytes_match_oracle_accounting(name):
    w = synthetic.make(name)
    kvb = 1 if w.kv_dtype == "e4m3" else 2
    got = bench.decode_bytes(w.context_lens, w.num_kv_heads, w.num_q_heads, w.head_dim, kvb, 2, w.block_size)
    want = accounting.decode_bytes(w.context_lens, w.num_kv_heads, w.num_q_heads, w.head_dim, kvb, 2,
                                   w.block_size)
    assert got == want


def test_workload_sizes_match_the_recipes():
    w = synthetic.make("llama13b_mix")
    lens = np.array(w.context_lens)
    assert (((lens >= 128) & (lens < 144)).sum(), ((lens >= 1024) & (lens < 1040)).sum(),
            ((lens >= 8192) & (lens < 8208)).sum()) == (128, 77, 51)
    gb = bench.decode_bytes(lens, 40, 40, 128, 2, 2, 16) / 1e9
    assert 10.4 < gb < 10.7
    w5 = synthetic.make("long_fp8")
    assert abs(bench.decode_bytes(w5.context_lens, 32, 32, 128, 1, 2, 32) / 1e9 - 2.147) < 0.01
    w4 = synthetic.make("gqa_prefix")
    assert all(1001 <= L <= 1256 for L in w4.context_lens) and w4.num_q_heads // w4.num_kv_heads == 4


_RANK_SCRIPT = r"""
import os, sys
sys.path.insert(0, {root!r})
import torch.distributed as dist
import bench
world, rank, local = bench.dist_env()
d = bench.init_dist(world, "gloo")
mx = bench.reduce_max(10.0 + rank, d)
sm = bench.reduce_sum(1.5 * (rank + 1), d)
bench.barrier(d)
print(f"rank{{rank}} max={{mx}} sum={{sm}}")
dist.destroy_process_group()
"""


def test_replica_timing_reduction_over_two_gloo_ranks(tmp_path):
    script = tmp_path / "ranks.py"
    script.write_text(_RANK_SCRIPT.format(root=ROOT))
    env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT="29533", WORLD_SIZE="2")
    procs = []
    for r in range(2):
        e = dict(env, RANK=str(r), LOCAL_RANK=str(r))
        procs.append(subprocess.Popen([sys.executable, str(script)], env=e, stdout=subprocess.PIPE,
                                      stderr=subprocess.STDOUT, text=True))
    outs = [p.communicate(timeout=120)[0] for p in procs]
    assert all(p.returncode == 0 for p in procs), outs
    for r, o in enumerate(outs):
        assert f"rank{r} max=11.0 sum=4.5" in o, o


def test_product_path_does_not_import_the_oracle():
    code = ("import sys; sys.path.insert(0, %r); import bench, paged_kv_cache_436_b200, "
            "paged_kv_cache_436_b200.engine; print(any(m == 'oracle' or m.startswith('oracle.') "
            "for m in sys.modules))" % ROOT)
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == "False"


def test_reference_arm_runs_on_cpu():
    """--impl reference: the oracle on a bounded sample, one JSON line."""
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny", "--steps", "3", "--warmup", "3"],
                         capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    import json
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_cpu_baseline_on_every_core_and_on_one_thread():
    """cpu_baseline: the oracle on one process per host core (spawned, one BLAS thread
    each, a pass timed by its slowest process) with the one-thread figure beside it."""
    import bench
    w = synthetic.make("tiny")
    c = bench.cpu_baseline_obj(w, 0.2)
    assert c["kind"] == "oracle" and c["unit"] == "GB/s" and c["value"] > 0
    assert 1 <= c["cores"] <= bench.host_cores() and c["cores"] <= w.num_seqs
    assert "processes" in c["sample"] and "the whole tiny workload" in c["sample"]
    one = c["single_thread"]
    assert one["cores"] == 1 and one["value"] > 0 and "1 thread" in one["sample"]


def test_reference_arm_other_ranks_exit_without_work():
    """Under torchrun only rank 0 runs the oracle and prints; rank 1 exits 0 silently."""
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                          "--steps", "3", "--warmup", "3"], capture_output=True, text=True, timeout=120, env=env)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == ""


def test_workloads_and_inputs_are_reproducible():
    """Every input is seeded: building a workload or drawing its inputs twice gives the
    same bits, and different steps or seeds give different draws."""
    import numpy as np
    import torch
    for name in synthetic.NAMES:
        a, b = synthetic.make(name), synthetic.make(name)
        assert list(a.context_lens) == list(b.context_lens), name
        assert list(a.initial_order) == list(b.initial_order), name
    w = synthetic.make("tiny")
    q0, k0, v0 = synthetic.step_inputs(w, 0)
    q1, k1, v1 = synthetic.step_inputs(w, 0)
    assert all(torch.equal(x.view(torch.int16), y.view(torch.int16)) for x, y in ((q0, q1), (k0, k1), (v0, v1)))
    q2, _, _ = synthetic.step_inputs(w, 1)
    assert not torch.equal(q0.view(torch.int16), q2.view(torch.int16))
    c1 = synthetic.normal_e4m3_codes((4, 64), 5)
    c2 = synthetic.normal_e4m3_codes((4, 64), 5)
    assert torch.equal(c1[0], c2[0]) and c1[1] == c2[1]
    assert np.array_equal(synthetic.beam_parents(4, 5, 3, 9), synthetic.beam_parents(4, 5, 3, 9))
