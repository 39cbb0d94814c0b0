"""Parity at the benchmark's full sizes, in the launch configuration the benchmark
times (the same engine step): EVERY (sequence, q head) output row of the 13B mix
(256 sequences x 40 heads) and of the 32K FP8 case (8 x 32 heads) against the float64
oracle, which runs on all host cores (one spawned process per core, sequences shared
out longest first). The whole cache after the step is compared bit for bit, and every
cache byte past the contexts is NaN before the step."""

import pytest

import synthetic
from tests.gpu_cases import run_decode_step_all_rows

pytestmark = pytest.mark.gpu


def test_llama13b_mix_every_row():
    run_decode_step_all_rows(synthetic.make("llama13b_mix"))


def test_long_fp8_every_row():
    run_decode_step_all_rows(synthetic.make("long_fp8"))
