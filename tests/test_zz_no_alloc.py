"""The allocation-free LM-head entry point agrees with the workspace one (B200 only).

dllm_lmhead_confidence_noalloc exists for callers that cannot give the
library device memory: an allocator that owns the whole device pool and
forbids cudaMalloc on the request path, or a binding that can pass tensors
but no workspace.  Its scratch is a fixed array inside the library, so two
calls in a row must still each give the same confidences, tokens and gaps as
dllm_lmhead_confidence with a caller workspace.  This file is collected last
and is self-contained, so it runs alone or after the rest of the suite.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from diffusion_decoding_step_b200 import workload as wl
from diffusion_decoding_step_b200.runtime import make_config, workspace_bytes
from tests.gpu_util import ensure_lib, ptr, stream

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _inputs(R, d, V, seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    W = (torch.randn(V, d, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    t = torch.randint(0, V, (R,), generator=g, device=DEV)
    a = torch.rand(R, generator=g, device=DEV) * 20
    rows = W[t].float()
    h = a[:, None] * rows / (rows * rows).sum(1, keepdim=True)
    h = (h + torch.randn(R, d, generator=g, device=DEV) / (0.02 * d ** 0.5)).to(torch.bfloat16)
    return W, h


def _outputs(R):
    return (torch.full((R,), -1.0, device=DEV), torch.full((R,), -1, dtype=torch.int32, device=DEV),
            torch.full((R,), -1.0, device=DEV))


# (rows, hidden, vocab, seed), called in a row: 200 rows over four reduce
# CTAs, then 32; then the largest row count the scratch holds on the
# LLaDA-8B-shaped LM head and the Dream-7B-shaped one (the widest per-row
# statistic extents of the benchmark shapes).
CALLS = ((200, 1024, 32768, 11), (32, 1024, 32768, 12), (256, 4096, 126464, 13),
         (32, 3584, 152064, 14))


def test_noalloc_lmhead_matches_workspace_entry_point_on_calls_in_a_row():
    abi = ensure_lib()
    for call, (R, d, V, seed) in enumerate(CALLS):
        w = wl.Workload("t", batch=4, n_layers=1, hidden=d, n_q_heads=d // 128,
                        n_kv_heads=d // 128, head_dim=128, vocab=V, prompt_len=0, gen_len=64,
                        block=64)
        cfg = make_config(w)
        n = workspace_bytes(w)
        ws = torch.empty(n, dtype=torch.uint8, device=DEV)
        abi.check(abi.dllm_workspace_init(C.byref(cfg), ptr(ws), n, stream()), "ws init")
        W, h = _inputs(R, d, V, seed)
        wc = abi.dllm_weights(ptr(W), ptr(W), ptr(W), ptr(W))
        ref = _outputs(R)
        abi.check(abi.dllm_lmhead_confidence(C.byref(cfg), C.byref(wc), ptr(h), R, ptr(ref[0]),
                                             ptr(ref[1]), ptr(ref[2]), ptr(ws), n, stream()),
                  "lmhead")
        got = _outputs(R)
        abi.check(abi.dllm_lmhead_confidence_noalloc(C.byref(cfg), C.byref(wc), ptr(h), R,
                                                     ptr(got[0]), ptr(got[1]), ptr(got[2]),
                                                     stream()), "lmhead noalloc")
        torch.cuda.synchronize()
        c0, t0, g0 = (x.cpu().numpy() for x in ref)
        c1, t1, g1 = (x.cpu().numpy() for x in got)
        # no wait gave up: a call whose device wait gives up reports NaN / -1
        assert np.isfinite(c1).all() and (t1 >= 0).all(), f"call {call}: invalid outputs"
        assert np.abs(c1 - c0).max() <= 2e-3, f"call {call}: confidence differs"
        assert np.array_equal(t1, t0), f"call {call}: argmax differs"
        assert np.abs(g1 - g0).max() <= 1e-3, f"call {call}: gap differs"
        assert (c1 > 0).all() and (c1 <= 1.0 + 1e-6).all()
        del W, h, ws
        torch.cuda.empty_cache()


def test_noalloc_lmhead_rejects_rows_beyond_its_scratch():
    abi = ensure_lib()
    w = wl.Workload("t", batch=8, n_layers=1, hidden=256, n_q_heads=2, n_kv_heads=2, head_dim=128,
                    vocab=1024, prompt_len=0, gen_len=64, block=64)
    cfg = make_config(w)
    W = torch.zeros(1024, 256, dtype=torch.bfloat16, device=DEV)
    h = torch.zeros(512, 256, dtype=torch.bfloat16, device=DEV)
    out = _outputs(512)
    wc = abi.dllm_weights(ptr(W), ptr(W), ptr(W), ptr(W))
    st = abi.dllm_lmhead_confidence_noalloc(C.byref(cfg), C.byref(wc), ptr(h), 257, ptr(out[0]),
                                            ptr(out[1]), ptr(out[2]), stream())
    assert st == abi.DLLM_ERR_UNSUPPORTED
