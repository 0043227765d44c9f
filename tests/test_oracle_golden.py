"""The fp64 oracle against its stored free-running decodes of the tiny
workload (tests/golden/oracle_tiny_decode.json, written from the oracle
itself by tests/golden/make_oracle_tiny.py).

This is a regression pin of the oracle. The other pins check it against
closed forms and invariants; this one fails on any change that moves a
token, a commit or a step count, or a confidence by more than 1e-9 relative.
"""
import importlib.util
import json
import os

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
_spec = importlib.util.spec_from_file_location(
    "make_oracle_tiny", os.path.join(HERE, "golden", "make_oracle_tiny.py"))
gen = importlib.util.module_from_spec(_spec)
_spec.loader.exec_module(gen)

with open(gen.OUT) as f:
    GOLDEN = json.load(f)


@pytest.mark.parametrize("key", sorted(GOLDEN))
def test_oracle_reproduces_its_stored_decode(key):
    name, kind = key.split(":")
    got = gen.record(gen.VARIANTS[name], mirror=(kind == "mirror"))
    want = GOLDEN[key]
    assert got["steps_per_block"] == want["steps_per_block"]
    assert got["tokens"] == want["tokens"]
    assert len(got["steps"]) == len(want["steps"])
    for g, w in zip(got["steps"], want["steps"]):
        assert (g["block"], g["commit"], g["tok"]) == (w["block"], w["commit"], w["tok"])
        assert [c is None for c in g["conf"]] == [c is None for c in w["conf"]]
        for a, b in zip(g["conf"], w["conf"]):
            if b is not None:
                assert a == pytest.approx(b, rel=1e-9, abs=0.0)


def test_a_planted_oracle_mistake_is_caught(monkeypatch):
    """Scaling the attention queries by 1.001 inside the oracle moves the
    stored confidences by far more than the pin's tolerance."""
    from oracle import dllm_oracle as O
    real = O.attention
    monkeypatch.setattr(O, "attention", lambda q, k, v, *a, **kw: real(q * 1.001, k, v, *a, **kw))
    got = gen.record(gen.VARIANTS["tiny_prefix"], mirror=False)
    want = GOLDEN["tiny_prefix:exact"]
    worst = 0.0
    for g, w in zip(got["steps"], want["steps"]):
        for a, b in zip(g["conf"], w["conf"]):
            if a is not None and b is not None:
                worst = max(worst, abs(a - b) / abs(b))
    assert worst > 1e-6 or got["tokens"] != want["tokens"]
