"""The DLLM_DEBUG build (libdllm_debug.so) on the GPU.

Its kernels range-check the row positions they read from device memory (the
per-sequence block starts of dllm_decode_all) and record DLLM_DEVICE_INDEX
instead of making an out-of-range access.  On valid decodes the checks must
stay silent and change nothing: every token equals the product build's.
Each build runs in a child process, since a process loads one library.
"""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CASES = ["batch_mid_dual", "qwen_mid_pruned"]


def decode_with(lib_path):
    """Child: lockstep and per-sequence decodes of CASES with one library."""
    from diffusion_decoding_step_b200 import abi
    abi.LIB_PATH = lib_path
    import torch

    from diffusion_decoding_step_b200 import workload as wl
    from diffusion_decoding_step_b200.runtime import Decoder
    from tests.test_gpu_decode import PER_SEQ
    out = {}
    for name in CASES:
        w = PER_SEQ[name]
        weights = wl.make_weights(w, device="cuda")
        tokens, masked = wl.make_tokens(w)
        plants = wl.make_plants(w, weights.w_lm)
        dec = Decoder(w, weights, tokens, masked, wl.seq_starts(w), plants)
        dec.generate()
        torch.cuda.synchronize()
        lock = dec.tokens.cpu().tolist()
        dec.reset()
        dec.generate_per_sequence()
        torch.cuda.synchronize()
        out[name] = {"lockstep": lock, "per_seq": dec.tokens.cpu().tolist(),
                     "left": int(dec.masked.sum().item()), "status": dec.device_status()}
        abi.dllm_graph_cache_clear()
    print(json.dumps(out))


def _run(lib_path):
    code = ("import sys; sys.path.insert(0, %r); import tests.test_gpu_debug_build as t; "
            "t.decode_with(%r)" % (ROOT, lib_path))
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


@pytest.mark.gpu
def test_debug_build_is_silent_and_matches_the_product_build():
    from diffusion_decoding_step_b200 import build
    prod = _run(build.build())
    dbg = _run(build.build(debug=True))
    for name in CASES:
        assert prod[name]["status"] == 0 and dbg[name]["status"] == 0, name
        assert prod[name]["left"] == 0 and dbg[name]["left"] == 0, name
        assert dbg[name]["lockstep"] == prod[name]["lockstep"], name
        assert dbg[name]["per_seq"] == prod[name]["per_seq"], name
