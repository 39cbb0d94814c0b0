"""Parity at the benchmark's full sizes, in the launch configuration the benchmark
times (the same engine step), checked on sampled (sequence, head) outputs the
oracle computes one by one; block tables and the touched cache blocks are
compared exactly."""

import numpy as np
import pytest

import synthetic
from tests.gpu_cases import run_decode_step

pytestmark = pytest.mark.gpu


def test_llama13b_mix_full_size_sampled():
    w = synthetic.make("llama13b_mix")
    lens = np.array(w.context_lens)
    pick = []
    for lo, hi in ((0, 200), (1000, 1100), (8000, 9000)):
        idx = np.nonzero((lens >= lo) & (lens < hi))[0]
        pick += idx[[0, -1]].tolist()
    pick += [int(np.argmax(lens)), int(np.argmin(lens)), w.num_seqs - 1]
    run_decode_step(w, sample_heads=[0, 13, 27, 39], sample_seqs=sorted(set(pick)))


def test_long_fp8_full_size_sampled():
    w = synthetic.make("long_fp8")
    run_decode_step(w, sample_heads=[0, 11, 22, 31], sample_seqs=[0, 3, 7])
