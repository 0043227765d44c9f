"""Checkpoint and resume of a decode (GPU).

All decode state lives in caller-owned buffers: tokens, the mask and the K/V
caches.  The workspace carries nothing from one block to the next in lockstep
decoding.  So a decoder rebuilt from a host copy of those buffers, taken
between blocks, finishes a generation exactly like an uninterrupted run.
"""
import pytest
import torch

from diffusion_decoding_step_b200.runtime import Decoder
from tests.gpu_util import ensure_lib
from tests.oracle_inputs import Case
from tests.test_gpu_decode import MID, make_decoder

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["batch_mid_dual", "qwen_mid_pruned", "dream_mid_prefix"])
def test_decode_resumes_from_state_saved_between_blocks(name):
    """All decode state lives in caller-owned buffers (tokens, mask, K/V
    caches): a decoder rebuilt from a host copy taken between blocks finishes
    the generation with the tokens of an uninterrupted run."""
    case = Case(MID[name])
    w = case.w
    dec = make_decoder(case)
    dec.generate()
    torch.cuda.synchronize()
    want = dec.tokens.cpu().clone()
    dec.reset()
    dec.prefill()
    blocks = list(range(w.prompt_len, w.seq_len, w.block))
    half = len(blocks) // 2
    for s in blocks[:half]:
        dec.decode_block(s)
    torch.cuda.synchronize()
    saved = [t.cpu().clone() for t in (dec.tokens, dec.masked, dec.k_cache, dec.v_cache)]
    del dec
    abi = ensure_lib()
    abi.dllm_graph_cache_clear()  # cached graphs reference the freed buffers
    dec2 = Decoder(w, case.weights, saved[0], saved[1], case.starts, case.plants)
    dec2.k_cache.copy_(saved[2])
    dec2.v_cache.copy_(saved[3])
    for s in blocks[half:]:
        dec2.decode_block(s)
    torch.cuda.synchronize()
    assert dec2.device_status() == 0
    assert not dec2.masked.any()
    assert torch.equal(dec2.tokens.cpu(), want)
