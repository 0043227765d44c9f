"""The step's algorithmic byte count that bench.py divides by (host only).

The count is the denominator of the reported roofline fraction, so it is
checked here against an explicit tally for the two headline shapes.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from diffusion_decoding_step_b200 import workload as wl  # noqa: E402


def test_llada_dual_step_bytes():
    w = wl.WORKLOADS["llada8b_dual"]
    L, d, R, keys = 32, 4096, 32, 512
    weights = L * (12288 * d * 2 + d * d * 2) + 126464 * d * 2
    kv_read = L * 32 * keys * 128 * 2 * 2
    # per layer: q,k,v written; xb read; q read + out written + out read; x r/w + xb w
    acts = L * (R * 12288 * 2 + R * d * 2 + R * d * 2 * 3 + R * d * 10) + R * d * 2 + R * d * 6
    assert bench.step_algorithmic_bytes(w, w.prompt_len) == weights + kv_read + acts
    assert 5.6e9 < bench.step_algorithmic_bytes(w, w.prompt_len) < 5.8e9


def test_dream_prefix_keys_grow_with_the_block():
    w = wl.WORKLOADS["dream7b_prefix"]
    assert bench.step_key_counts(w, 512) == [544]
    assert bench.step_key_counts(w, 992) == [1024]
    assert bench.step_algorithmic_bytes(w, 992) > bench.step_algorithmic_bytes(w, 512)


def test_pruned_suffix_keys_are_window_plus_trailing():
    w = wl.WORKLOADS["qwen7b_long_pruned"]
    s = w.prompt_len
    assert bench.step_key_counts(w, s) == [s + w.block + w.window + 1] * w.batch
    last = w.seq_len - w.block
    assert bench.step_key_counts(w, last) == [w.seq_len] * w.batch


@pytest.mark.parametrize("name", list(wl.WORKLOADS))
def test_bytes_positive_for_every_workload(name):
    w = wl.WORKLOADS[name]
    assert bench.step_algorithmic_bytes(w, w.prompt_len) > 0
