"""Step-level and whole-decode parity of the CUDA path with the oracle (B200 only)."""
import ctypes as C
import os

import numpy as np
import pytest
import torch

from oracle import dllm_oracle as O
from diffusion_decoding_step_b200 import workload as wl
from diffusion_decoding_step_b200.runtime import Decoder
from tests.gpu_util import ensure_lib
from tests.lockstep import lockstep, compare_step, state_from_gpu
from tests.oracle_inputs import Case

pytestmark = pytest.mark.gpu

TINY = wl.WORKLOADS["tiny"]

# Mid-size variants of the workload shapes: every mode, GQA + RoPE, ragged
# batches and the pruned suffix, with sizes the oracle finishes in seconds.
MID = {
    "tiny_prefix": TINY,
    "tiny_nocache": TINY.replace(mode=wl.MODE_NONE),
    "llada_mid_dual": wl.Workload("llada_mid_dual", batch=1, n_layers=2, hidden=512,
                                  n_q_heads=4, n_kv_heads=4, head_dim=128, vocab=8192,
                                  prompt_len=64, gen_len=64, block=32, mode=wl.MODE_DUAL),
    "dream_mid_prefix": wl.Workload("dream_mid_prefix", batch=1, n_layers=2, hidden=896,
                                    n_q_heads=7, n_kv_heads=1, head_dim=128, vocab=8192,
                                    prompt_len=96, gen_len=64, block=32, mode=wl.MODE_PREFIX,
                                    rope_theta=1e6),
    "batch_mid_dual": wl.Workload("batch_mid_dual", batch=3, n_layers=2, hidden=256,
                                  n_q_heads=2, n_kv_heads=2, head_dim=128, vocab=4096,
                                  prompt_len=100, prompt_len_min=60, gen_len=64, block=32,
                                  mode=wl.MODE_DUAL),
    "qwen_mid_pruned": wl.Workload("qwen_mid_pruned", batch=2, n_layers=2, hidden=512,
                                   n_q_heads=4, n_kv_heads=2, head_dim=128, vocab=4096,
                                   prompt_len=200, gen_len=128, block=32,
                                   mode=wl.MODE_DUAL_PRUNED, window=16, rope_theta=1e4),
}


def make_decoder(case: Case) -> Decoder:
    ensure_lib()
    return Decoder(case.w, case.weights, case.tokens, case.masked, case.starts, case.plants)


@pytest.mark.parametrize("name", list(MID))
def test_lockstep_decode(name):
    case = Case(MID[name])
    dec = make_decoder(case)
    rep = lockstep(dec, case)
    assert rep.steps >= (case.w.gen_len // case.w.block)
    assert rep.flagged_mismatch <= max(2, rep.rows // 50)
    assert not dec.masked.any()


@pytest.mark.parametrize("name", ["llada_mid_dual", "dream_mid_prefix", "qwen_mid_pruned"])
def test_lockstep_decode_layer_stack(name):
    """The persistent layer-stack kernel (one launch for all layers of a step
    or refresh; off by default) in lockstep with the oracle."""
    from diffusion_decoding_step_b200 import abi
    case = Case(MID[name])
    dec = make_decoder(case)
    info = (C.c_int32 * 8)()
    abi.check(abi.dllm_layer_stack_plan(dec.cfg_p, case.w.prompt_len, info), "plan")
    assert info[0] == 1 and info[7] == 1
    abi.check(abi.dllm_set_layer_stack(1, 16), "layer stack on")
    try:
        rep = lockstep(dec, case)
    finally:
        abi.check(abi.dllm_set_layer_stack(0, 16), "layer stack off")
    assert rep.steps >= (case.w.gen_len // case.w.block)
    assert rep.flagged_mismatch <= max(2, rep.rows // 50)
    assert not dec.masked.any()


def settled_before_first_flag(tr, B):
    """Positions the oracle's free-running decode commits before its first
    flagged decision that can change the state, with their tokens.  A state
    change needs a commit: a row whose commit decision is flagged, or a
    committed row whose argmax is flagged.  (A row with a flagged argmax that
    is not committed, and whose commit decision is not flagged, changes
    nothing on either side.)  Up to that step the GPU takes the same path, so
    it must commit the same tokens there (a committed token is never revised);
    rows committed at that step count too when they are not flagged."""
    out = {}
    for s, r in tr.steps:
        flag = r.amb_tok | r.amb_commit
        for bi in range(r.commit.shape[0]):
            for i in np.where(r.commit[bi] & ~flag[bi])[0]:
                out[(bi, s + int(i))] = int(r.tok[bi, i])
        if (r.amb_commit | (r.amb_tok & r.commit)).any():
            break
    return out


def state_flags(tr):
    """Flagged decisions of a decode that can change its state."""
    return sum(int((r.amb_commit | (r.amb_tok & r.commit)).sum()) for _, r in tr.steps)


# A plant draw of the tiny workload whose free-running oracle decode raises no
# ambiguity flag anywhere (found by searching draws 2..80), with several
# commits per step in most blocks.
FLAG_FREE_PLANT_SEED = 35


@pytest.mark.parametrize("mode", [wl.MODE_PREFIX, wl.MODE_NONE])
def test_tiny_free_running_decode_equals_oracle_bit_exact(mode):
    """Whole generations decoded by the GPU on its own equal the oracle's
    bit for bit: tokens and steps per block (no flagged row to excuse)."""
    case = Case(TINY.replace(mode=mode), plant_seed=FLAG_FREE_PLANT_SEED)
    tr = case.decode()
    flags = sum(int((r.amb_tok | r.amb_commit).sum()) for _, r in tr.steps)
    assert flags == 0
    assert sum(tr.steps_per_block) < TINY.gen_len  # parallel commits happen
    dec = make_decoder(case)
    steps = dec.generate()
    torch.cuda.synchronize()
    assert dec.device_status() == 0
    assert not dec.masked.any()
    assert np.array_equal(dec.tokens.cpu().numpy(), tr.tokens)
    assert steps == tr.steps_per_block


EARLY_EXIT_CASES = {
    # (workload, plant scale or None for the workload's draw, plant seed)
    "prefix": (TINY.replace(commit_mode=wl.COMMIT_EARLY_EXIT, exit_tau=0.5), None, 35),
    "nocache": (TINY.replace(commit_mode=wl.COMMIT_EARLY_EXIT, exit_tau=0.3,
                             mode=wl.MODE_NONE), None, 35),
    "converged": (TINY.replace(commit_mode=wl.COMMIT_EARLY_EXIT, exit_tau=0.5), 8.0, None),
}


@pytest.mark.parametrize("name", list(EARLY_EXIT_CASES))
def test_early_exit_generation_equals_oracle_bit_exact(name):
    """The early-exit commit rule (converged rows commit above exit_tau) on
    the GPU, whole generations against a flag-free oracle decode: tokens and
    steps per block bit for bit.  'converged' plants confidences between
    exit_tau and tau, where every block takes exactly two steps."""
    w, a, seed = EARLY_EXIT_CASES[name]
    case = Case(w, a_override=a, noise=a is None, plant_seed=seed)
    tr = case.decode()
    assert state_flags(tr) == 0
    if name == "converged":
        assert tr.steps_per_block == [2] * (w.gen_len // w.block)
    dec = make_decoder(case)
    steps = dec.generate()
    torch.cuda.synchronize()
    assert dec.device_status() == 0
    assert np.array_equal(dec.tokens.cpu().numpy(), tr.tokens)
    assert steps == tr.steps_per_block
    # a second generation from the reset state restarts the rule at the first
    # block (the saved argmax of an earlier generation is not reused)
    dec.reset()
    assert dec.generate() == tr.steps_per_block
    assert np.array_equal(dec.tokens.cpu().numpy(), tr.tokens)


@pytest.mark.parametrize("name", ["llada_mid_dual", "dream_mid_prefix", "qwen_mid_pruned"])
def test_lockstep_decode_early_exit(name):
    case = Case(MID[name].replace(commit_mode=wl.COMMIT_EARLY_EXIT, exit_tau=0.5))
    dec = make_decoder(case)
    rep = lockstep(dec, case)
    assert rep.steps >= (case.w.gen_len // case.w.block)
    assert rep.flagged_mismatch <= max(2, rep.rows // 50)
    assert not dec.masked.any()


def test_tiny_free_running_decode_matches_oracle_up_to_first_flag():
    """The default plant draw flags rows (8 over the generation), so the two
    decodes may part at the first flagged step; every position settled before
    it must carry the oracle's token, and the prompt is untouched."""
    case = Case(TINY)
    tr = case.decode()
    settled = settled_before_first_flag(tr, TINY.block)
    assert len(settled) >= 5  # the first flag comes at the sixth step of the first block
    dec = make_decoder(case)
    dec.generate()
    torch.cuda.synchronize()
    got = dec.tokens.cpu().numpy()
    assert not dec.masked.any()
    assert np.array_equal(got[:, :TINY.prompt_len], tr.tokens[:, :TINY.prompt_len])
    bad = [(k, v, int(got[k])) for k, v in settled.items() if int(got[k]) != v]
    assert not bad, f"settled positions differ (position, oracle, gpu): {bad[:8]}"


def test_decode_block_equals_step_by_step():
    w = MID["llada_mid_dual"]
    case = Case(w)
    a = make_decoder(case)
    b = make_decoder(case)
    a.prefill()
    b.prefill()
    s = w.prompt_len
    n = a.decode_block(s)
    m = 0
    while b.masked[:, s:s + w.block].any():
        b.step(s)
        m += 1
    b.refresh(s)
    torch.cuda.synchronize()
    assert n == m
    assert torch.equal(a.tokens, b.tokens)
    assert torch.equal(a.k_cache, b.k_cache)


def test_tau_above_one_commits_one_row_per_step():
    w = MID["llada_mid_dual"].replace(tau=1.5, gen_len=32)
    case = Case(w)
    dec = make_decoder(case)
    dec.prefill()
    n = dec.decode_block(w.prompt_len)
    assert n == w.block
    assert not dec.masked.any()


def test_tiny_tau_commits_whole_block_in_one_step():
    w = MID["llada_mid_dual"].replace(tau=1e-9, gen_len=32)
    case = Case(w)
    dec = make_decoder(case)
    dec.prefill()
    assert dec.decode_block(w.prompt_len) == 1


# ---------------------------------------------------------------- full-size steps
FULL = ["llada8b_dual", "dream7b_prefix"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_first_steps_lockstep(name):
    """Full-size shapes: prefill on the GPU, then the first two steps of the
    first block checked row by row against the oracle on the GPU's state."""
    w = wl.WORKLOADS[name]
    ensure_lib()
    case = Case(w, device="cuda")
    dec = make_decoder(case)
    dec.prefill()
    torch.cuda.synchronize()
    assert dec.device_status() == 0
    bad = [l for l in range(w.n_layers)
           if not (bool(torch.isfinite(dec.k_cache[l]).all())
                   and bool(torch.isfinite(dec.v_cache[l]).all()))]
    assert not bad, f"non-finite cache after prefill in layers {bad[:8]}"
    # layer-0 keys of sampled prompt positions depend only on their embedding
    D, Hq, Hkv = w.head_dim, w.n_q_heads, w.n_kv_heads
    Wk = case.weights.wqkv[0, Hq * D:(Hq + Hkv) * D].double().cpu().numpy()
    for p in (0, 17, w.prompt_len - 1):
        tok = int(case.tokens[0, p])
        e = case.weights.w_lm[tok].double().cpu().numpy()
        k = ((O.round_bf16(e) @ Wk.T) * O.inv_rms(e)).reshape(Hkv, D)
        if w.rope_theta > 0:
            k = O.rope(k[:, None, :], np.array([p]), w.rope_theta)[:, 0, :]
        got = dec.k_cache[0, 0, :, p].double().cpu().numpy()
        np.testing.assert_allclose(got, O.round_bf16(k), rtol=2 ** -7, atol=1e-5)
    from tests.lockstep import Report
    rep = Report()
    for _ in range(2):
        compare_step(dec, case, w.prompt_len, rep, check_kv=False)
    assert rep.steps == 2


@pytest.mark.skipif(os.environ.get("DLLM_FULL_PARITY") != "1",
                    reason="opt-in (DLLM_FULL_PARITY=1): about half an hour of oracle time")
@pytest.mark.parametrize("name,blocks", [("llada8b_dual", None), ("dream7b_prefix", 2)])
def test_full_size_generation_lockstep(name, blocks):
    """Whole LLaDA-8B-shaped generation (8 blocks, every step and refresh) and
    the first two blocks of the Dream-7B-shaped one, in lockstep with the
    oracle in the launch configuration bench.py times: confidences within
    2e-3, tokens and commits bit-exact outside flagged rows, the block's
    keys/values after every step and refresh within rel-L2 5e-3, prefill of
    layer 0 within rel-L2 5e-3 and of all layers within 1e-2 (both sides run
    the prefill free through every layer)."""
    from tests.lockstep import lockstep_incremental
    w = wl.WORKLOADS[name]
    ensure_lib()
    case = Case(w, device="cuda")
    dec = make_decoder(case)
    rep = lockstep_incremental(dec, case, max_blocks=blocks, log=lambda m: print(m, flush=True))
    print(f"{name}: {rep}")
    assert rep.steps >= (blocks or w.gen_len // w.block)
    assert rep.flagged_mismatch <= max(2, rep.rows // 50)
    if blocks is None:
        assert not dec.masked.any()


# ---------------------------------------------------------------- full-size batches
BATCHED = ["llada8b_dual_b16", "qwen7b_long_pruned"]


@pytest.mark.parametrize("name", BATCHED)
def test_full_size_batched_step_sampled_sequences(name):
    """Batched full-size shapes (16 ragged LLaDA-8B-shaped sequences with
    DualCache; 4 long Qwen-shaped sequences with the pruned suffix): prefill,
    then one step of the first block on the GPU, the first and the last
    sequence recomputed alone by the oracle from the GPU's state."""
    from tests.lockstep import Report, compare_step_sampled
    w = wl.WORKLOADS[name]
    ensure_lib()
    case = Case(w, device="cuda")
    dec = make_decoder(case)
    dec.prefill()
    torch.cuda.synchronize()
    assert dec.device_status() == 0
    for l in (0, w.n_layers - 1):
        assert bool(torch.isfinite(dec.k_cache[l]).all())
        assert bool(torch.isfinite(dec.v_cache[l]).all())
    rep = Report()
    compare_step_sampled(dec, case, w.prompt_len, [0, w.batch - 1], rep)
    assert rep.steps == 1 and rep.rows > 0
    # every sequence committed at least one row and nothing outside the block
    commit = dec.step_outputs()[3].cpu().numpy()
    assert (commit.sum(1) >= 1).all()
    masked = dec.masked.cpu().numpy()
    assert masked[:, w.prompt_len + w.block:].all()



# ---------------------------------------------------------------- fixed-budget commits
TOPK = {
    "tiny_prefix_topk": TINY.replace(commit_mode=wl.COMMIT_TOPK, steps_per_block=3),
    "llada_mid_dual_topk": MID["llada_mid_dual"].replace(commit_mode=wl.COMMIT_TOPK,
                                                         steps_per_block=5),
}


@pytest.mark.parametrize("name", list(TOPK))
def test_lockstep_decode_topk(name):
    """The fixed-budget rule in lockstep with the oracle; every block takes
    exactly steps_per_block steps."""
    w = TOPK[name]
    case = Case(w)
    dec = make_decoder(case)
    rep = lockstep(dec, case)
    assert rep.steps == (w.gen_len // w.block) * w.steps_per_block
    assert rep.flagged_mismatch <= max(2, rep.rows // 50)
    assert not dec.masked.any()


def test_decode_block_topk_takes_the_step_budget():
    w = TOPK["llada_mid_dual_topk"]
    case = Case(w)
    dec = make_decoder(case)
    steps = dec.generate()
    torch.cuda.synchronize()
    assert steps == [w.steps_per_block] * (w.gen_len // w.block)
    assert not dec.masked.any()



# ---------------------------------------------------------------- prefix cache, suffix as queries
SUFQ = {
    "tiny_suffixq": TINY.replace(mode=wl.MODE_PREFIX_SUFFIXQ),
    "dream_mid_suffixq": MID["dream_mid_prefix"].replace(mode=wl.MODE_PREFIX_SUFFIXQ),
}


@pytest.mark.parametrize("name", list(SUFQ))
def test_lockstep_decode_suffix_queries(name):
    """Every step runs the block and the whole suffix through the layers
    (GQA and RoPE in the mid-size case), in lockstep with the oracle."""
    case = Case(SUFQ[name])
    dec = make_decoder(case)
    rep = lockstep(dec, case)
    assert rep.steps >= (case.w.gen_len // case.w.block)
    assert rep.flagged_mismatch <= max(2, rep.rows // 50)
    assert not dec.masked.any()


# ---------------------------------------------------------------- step cap
CAPPED = {
    "tiny_prefix_cap2": TINY.replace(steps_per_block=2),
    "llada_mid_dual_cap3": MID["llada_mid_dual"].replace(steps_per_block=3),
}


@pytest.mark.parametrize("name", list(CAPPED))
def test_lockstep_decode_step_cap(name):
    """Threshold rule with a per-block step cap, in lockstep with the oracle:
    the capping step commits every row still masked."""
    w = CAPPED[name]
    case = Case(w)
    dec = make_decoder(case)
    rep = lockstep(dec, case)
    assert rep.steps <= (w.gen_len // w.block) * w.steps_per_block
    assert rep.flagged_mismatch <= max(2, rep.rows // 50)
    assert not dec.masked.any()


def test_decode_block_respects_the_step_cap_across_generations():
    w = CAPPED["llada_mid_dual_cap3"]
    case = Case(w)
    dec = make_decoder(case)
    for _ in range(2):   # the per-sequence step counters restart with every block
        dec.reset()
        steps = dec.generate()
        torch.cuda.synchronize()
        assert all(1 <= n <= w.steps_per_block for n in steps)
        assert not dec.masked.any()


# ---------------------------------------------------------------- per-sequence blocks
PER_SEQ = {
    "batch_mid_dual": MID["batch_mid_dual"],
    "qwen_mid_pruned": MID["qwen_mid_pruned"],
    "tiny_prefix": TINY,
    "batch_mid_dual_topk": MID["batch_mid_dual"].replace(commit_mode=wl.COMMIT_TOPK,
                                                         steps_per_block=4),
    "batch_mid_dual_cap": MID["batch_mid_dual"].replace(steps_per_block=3),
    "batch_mid_dual_exit": MID["batch_mid_dual"].replace(commit_mode=wl.COMMIT_EARLY_EXIT,
                                                         exit_tau=0.5),
}


@pytest.mark.parametrize("name", list(PER_SEQ))
def test_per_sequence_blocks_reproduce_lockstep_tokens(name):
    """Sequences never interact, so decoding each at its own block must give
    bit-identical tokens to the batch moving block by block in lockstep (whose
    parity with the oracle the lockstep tests establish)."""
    w = PER_SEQ[name]
    case = Case(w)
    dec = make_decoder(case)
    steps = dec.generate()
    torch.cuda.synchronize()
    want = dec.tokens.cpu().numpy().copy()
    assert not dec.masked.any()
    dec.reset()
    passes = dec.generate_per_sequence()
    torch.cuda.synchronize()
    assert dec.device_status() == 0
    assert not dec.masked.any()
    assert np.array_equal(dec.tokens.cpu().numpy(), want)
    # a sequence takes its blocks' steps plus one refresh pass per block; the
    # batch finishes with the slowest sequence, never later than lockstep
    assert passes <= sum(steps) + len(steps)


@pytest.mark.parametrize("name", list(PER_SEQ))
def test_per_sequence_blocks_match_the_oracle_decoding_each_sequence_alone(name):
    """dllm_decode_all against the oracle: every sequence is decoded alone by
    the oracle (batch 1, its own prompt start), blocks left to right, with the
    step counters of the commit rule restarting per block.  Every position the
    oracle settles before its first flagged decision carries the oracle's
    token, and a sequence whose oracle decode raises no flag equals it bit for
    bit."""
    import dataclasses
    w = PER_SEQ[name]
    case = Case(w)
    dec = make_decoder(case)
    dec.generate_per_sequence()
    torch.cuda.synchronize()
    assert dec.device_status() == 0
    assert not dec.masked.any()
    got = dec.tokens.cpu().numpy()
    cfg1 = dataclasses.replace(case.cfg, batch=1)
    compared, whole = 0, 0
    for bi in range(w.batch):
        tr = O.decode(cfg1, case.W, case.tokens[bi:bi + 1].numpy(),
                      case.masked[bi:bi + 1].numpy().astype(bool),
                      case.starts[bi:bi + 1].numpy(), case.plants64[bi:bi + 1])
        if state_flags(tr) == 0:
            assert np.array_equal(got[bi], tr.tokens[0]), f"sequence {bi} differs"
            whole += 1
            compared += w.gen_len
            continue
        settled = settled_before_first_flag(tr, w.block)
        bad = [(p, v, int(got[bi, p])) for (_, p), v in settled.items() if int(got[bi, p]) != v]
        assert not bad, f"sequence {bi}: settled positions differ (position, oracle, gpu): {bad[:8]}"
        compared += len(settled)
    assert compared >= w.batch * min(4, w.block)
    print(f"{name}: {compared} positions compared, {whole} of {w.batch} sequences whole")


def test_per_sequence_blocks_reject_unsupported_caches():
    abi = ensure_lib()
    for w in (TINY.replace(mode=wl.MODE_NONE), TINY.replace(mode=wl.MODE_PREFIX_SUFFIXQ)):
        case = Case(w)
        dec = make_decoder(case)
        n = C.c_int32(0)
        st = abi.dllm_decode_all(dec.cfg_p, C.byref(dec.weights_c), C.byref(dec.state_c),
                                 C.byref(n), C.c_void_p(dec.ws.data_ptr()), dec.ws_bytes,
                                 dec._sh)
        assert st == abi.DLLM_ERR_UNSUPPORTED


# ---------------------------------------------------------------- per-sequence thresholds
def test_per_sequence_tau_in_lockstep_with_the_oracle():
    """Each sequence commits against its own threshold, read from device
    memory every step (here fixed per sequence; a policy may change them)."""
    from tests.lockstep import Report, compare_step_sampled
    w = MID["batch_mid_dual"]
    taus = [0.5, 0.9, 1.5]
    case = Case(w)
    dec = make_decoder(case)
    dec.set_tau(taus)
    dec.prefill()
    rep = Report()
    for s in range(w.prompt_len, w.seq_len, w.block):
        n = 0
        while dec.masked[:, s:s + w.block].any():
            compare_step_sampled(dec, case, s, list(range(w.batch)), rep, taus=taus,
                                 step_in_block=n)
            n += 1
            assert n <= w.block
        dec.refresh(s)
    torch.cuda.synchronize()
    assert dec.device_status() == 0 and not dec.masked.any()
    assert rep.flagged_mismatch <= max(2, rep.rows // 50)


def test_tau_array_changes_between_steps():
    """The graphs read the thresholds from device memory: changing them
    between steps takes effect without rebuilding anything."""
    w = MID["batch_mid_dual"]
    case = Case(w)
    dec = make_decoder(case)
    dec.set_tau([2.0] * w.batch)          # one commit per sequence per step
    dec.prefill()
    s = w.prompt_len
    dec.step(s)
    c1 = dec.step_outputs()[3].cpu().numpy().sum(1)
    dec.tau_seq.fill_(-1.0)               # now every masked row clears it
    dec.step(s)
    torch.cuda.synchronize()
    c2 = dec.step_outputs()[3].cpu().numpy().sum(1)
    assert (c1 <= 1).all()
    assert (dec.masked[:, s:s + w.block].cpu().numpy() == 0).all()
    assert (c2 >= 1).all()

