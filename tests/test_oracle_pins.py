"""Pins of the fp64 oracle against facts it does not compute itself.

Each test ties one oracle function to a closed form, a library routine, an
invariant the pages state, or a special case that reduces to one, so that a
dropped term, a wrong sign, a wrong index or a transposed operand fails here.
"""
import numpy as np
import pytest
import scipy.special
import torch

from oracle import dllm_oracle as O
from diffusion_decoding_step_b200 import workload as wl
from tests.oracle_inputs import Case, oracle_config

RNG = np.random.default_rng(1234)


# ---------------------------------------------------------------- rounding
def test_round_bf16_matches_torch():
    x = np.concatenate([RNG.standard_normal(20000) * 10.0 ** RNG.integers(-8, 8, 20000),
                        [0.0, -0.0, 1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 65504.0]])
    ref = torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.round_bf16(x), ref)


def test_round_bf16_ties_to_even():
    # 1 + 2^-8 lies halfway between bf16 neighbours 1 and 1 + 2^-7 -> even (1.0)
    assert O.round_bf16(1.0 + 2.0 ** -8) == 1.0
    # 1 + 3*2^-8 lies halfway between 1 + 2^-7 and 1 + 2^-6 -> even mantissa
    assert O.round_bf16(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6


# ---------------------------------------------------------------- rms norm
def test_inv_rms_closed_form_and_scale_invariance():
    x = np.array([[3.0, 4.0], [0.0, 0.0]])
    r = O.inv_rms(x)
    assert abs(r[0] - 1.0 / np.sqrt(12.5 + 1e-6)) < 1e-15
    assert abs(r[1] - 1.0 / np.sqrt(1e-6)) < 1e-6
    y = RNG.standard_normal((4, 64)) * 5
    for c in (0.25, 3.0, 1e3):
        np.testing.assert_allclose((c * y) * O.inv_rms(c * y)[:, None], y * O.inv_rms(y)[:, None],
                                   rtol=1e-6)
    z = y * O.inv_rms(y)[:, None]
    np.testing.assert_allclose((z * z).mean(axis=1), 1.0, rtol=1e-6)


def test_deep_stack_stays_finite():
    # 24 layers of d = 512 with N(0, 0.02^2) weights: without the
    # normalisation the residual would grow by ~1.3x per layer
    w = TINY.replace(n_layers=24, hidden=512, n_q_heads=4, n_kv_heads=4, head_dim=128,
                     gen_len=8, weight_f32=False, mode=wl.MODE_DUAL)
    tr = Case(w).decode(max_steps=1)
    r = tr.steps[0][1]
    assert np.isfinite(r.hidden).all()
    assert np.abs(r.hidden).max() < 1e3
    assert (r.conf[0] > 0.5).any() and (r.conf[0] < 0.1).any()


# ---------------------------------------------------------------- rope
def test_rope_position_zero_is_identity():
    x = RNG.standard_normal((5, 3, 16))
    np.testing.assert_array_equal(O.rope(x, np.zeros(3), 1e6), x)


def test_rope_d2_is_complex_rotation():
    # D = 2: inv_freq = 1, so the pair (x1, x2) is the complex number x1 + i x2
    # multiplied by exp(i * pos).
    x = RNG.standard_normal((7, 2))
    pos = np.arange(7) * 0.37
    z = (x[:, 0] + 1j * x[:, 1]) * np.exp(1j * pos)
    out = O.rope(x, pos, 10000.0)
    np.testing.assert_allclose(out[:, 0], z.real, atol=1e-14)
    np.testing.assert_allclose(out[:, 1], z.imag, atol=1e-14)


def test_rope_scores_depend_on_relative_position_only():
    D = 32
    q = RNG.standard_normal((1, D))
    k = RNG.standard_normal((1, D))
    for theta in (1e4, 1e6):
        base = (O.rope(q, np.array([11.0]), theta) @ O.rope(k, np.array([4.0]), theta).T)[0, 0]
        shifted = (O.rope(q, np.array([511.0]), theta)
                   @ O.rope(k, np.array([504.0]), theta).T)[0, 0]
        assert abs(base - shifted) < 1e-10
        # and it is not the unrotated product (the rotation does something)
        assert abs(base - (q @ k.T)[0, 0]) > 1e-6


def test_rope_frequency_of_last_pair():
    # pair i = D/2 - 1 rotates by pos * theta^(-(D-2)/D)
    D, theta, pos = 8, 100.0, 3.0
    x = np.zeros((1, D))
    x[0, D // 2 - 1] = 1.0
    out = O.rope(x, np.array([pos]), theta)
    ang = pos * theta ** (-(D - 2) / D)
    assert abs(out[0, D // 2 - 1] - np.cos(ang)) < 1e-14
    assert abs(out[0, D - 1] - np.sin(ang)) < 1e-14


# ---------------------------------------------------------------- attention
def test_attention_closed_form_weights():
    # keys built so that q.k_i / sqrt(D) = log w_i: softmax weights are w / sum(w)
    D = 16
    q = RNG.standard_normal((1, D))
    w = np.array([1.0, 2.0, 3.0, 10.0])
    k = (np.sqrt(D) * np.log(w))[:, None] * q / (q @ q.T)
    v = RNG.standard_normal((4, D))
    o = O.attention(q, k, v)
    np.testing.assert_allclose(o[0], (w / w.sum()) @ v, rtol=1e-12, atol=1e-12)


def test_attention_single_key_returns_value():
    q = RNG.standard_normal((3, 8))
    k = RNG.standard_normal((1, 8))
    v = RNG.standard_normal((1, 8))
    np.testing.assert_allclose(O.attention(q, k, v), np.repeat(v, 3, 0), atol=1e-15)


def test_attention_equal_scores_give_mean():
    q = np.zeros((2, 8))
    k = RNG.standard_normal((5, 8))
    v = RNG.standard_normal((5, 8))
    np.testing.assert_allclose(O.attention(q, k, v), np.repeat(v.mean(0, keepdims=True), 2, 0),
                               atol=1e-15)


def test_attention_key_order_irrelevant_and_rows_independent():
    q = RNG.standard_normal((4, 8))
    k = RNG.standard_normal((9, 8))
    v = RNG.standard_normal((9, 8))
    perm = RNG.permutation(9)
    o = O.attention(q, k, v)
    np.testing.assert_allclose(O.attention(q, k[perm], v[perm]), o, atol=1e-14)
    np.testing.assert_allclose(O.attention(q[2:3], k, v), o[2:3], atol=1e-15)


def test_attention_scale_is_inverse_sqrt_d():
    # two keys with q.k difference delta: weight ratio exp(delta / sqrt(D))
    D = 64
    q = np.zeros((1, D)); q[0, 0] = 1.0
    k = np.zeros((2, D)); k[1, 0] = 3.0
    v = np.array([[0.0] * D, [1.0] * D])
    p1 = 1.0 / (1.0 + np.exp(-3.0 / 8.0))
    np.testing.assert_allclose(O.attention(q, k, v)[0], np.full(D, p1), rtol=1e-13)


# ---------------------------------------------------------------- LM head
def test_lm_head_identity_closed_form():
    # w_lm = I  -> logits = h;  h = (0, ln 2, ln 5) -> conf = 5/8, tok = 2, gap = ln 5 - ln 2
    h = np.array([[0.0, np.log(2.0), np.log(5.0)]])
    c, t, g = O.lm_head_confidence(h, np.eye(3))
    assert abs(c[0] - 5.0 / 8.0) < 1e-15 and t[0] == 2
    assert abs(g[0] - (np.log(5.0) - np.log(2.0))) < 1e-15


def test_lm_head_matches_scipy_softmax_and_logsumexp():
    h = RNG.standard_normal((6, 32)) * 3
    w = RNG.standard_normal((500, 32)) * 0.3
    c, t, g = O.lm_head_confidence(h, w)
    logits = h @ w.T
    p = scipy.special.softmax(logits, axis=1)
    np.testing.assert_allclose(p.sum(1), 1.0, atol=1e-12)
    np.testing.assert_allclose(c, p.max(1), rtol=1e-12)
    np.testing.assert_allclose(c, np.exp(logits.max(1) - scipy.special.logsumexp(logits, axis=1)),
                               rtol=1e-12)
    assert np.all(t == np.argmax(p, axis=1))
    srt = np.sort(logits, axis=1)
    np.testing.assert_allclose(g, srt[:, -1] - srt[:, -2], atol=1e-12)
    assert np.all((c > 0) & (c <= 1) & (c >= 1.0 / 500 - 1e-15))


def test_lm_head_ties_lowest_id_and_zero_gap():
    w = np.eye(4)
    h = np.array([[1.0, 3.0, 3.0, 0.0]])
    c, t, g = O.lm_head_confidence(h, w)
    assert t[0] == 1 and g[0] == 0.0


def test_lm_head_uniform_logits_conf_is_one_over_v():
    c, t, g = O.lm_head_confidence(np.zeros((1, 4)), RNG.standard_normal((37, 4)))
    assert abs(c[0] - 1.0 / 37) < 1e-15 and t[0] == 0


# ---------------------------------------------------------------- commit
def test_commit_threshold_strict_and_forced():
    conf = np.array([0.95, 0.9, 0.2, 0.99, 0.5])
    masked = np.array([True, True, True, False, True])
    c = O.threshold_commit(conf, masked, 0.9)
    assert c.tolist() == [True, False, False, False, False]      # 0.9 does not clear 0.9
    c = O.threshold_commit(np.array([0.1, 0.3, 0.3, 0.2]), np.ones(4, bool), 0.9)
    assert c.tolist() == [False, True, False, False]              # forced, lowest position on tie


def test_commit_tau_above_one_commits_exactly_one():
    for _ in range(50):
        conf = RNG.uniform(0, 1, 16)
        masked = RNG.uniform(size=16) < 0.6
        masked[RNG.integers(16)] = True
        c = O.threshold_commit(conf, masked, 1.5)
        assert c.sum() == 1 and masked[c].all()
        assert np.argmax(np.where(masked, conf, -1)) == np.where(c)[0][0]


def test_commit_tiny_tau_commits_all_masked():
    conf = RNG.uniform(1e-3, 1, 16)
    masked = RNG.uniform(size=16) < 0.5
    masked[0] = True
    c = O.threshold_commit(conf, masked, 1e-6)
    assert np.array_equal(c, masked)


def test_commit_nothing_masked_commits_nothing():
    assert not O.threshold_commit(np.ones(4), np.zeros(4, bool), 0.9).any()


# ---------------------------------------------------------------- key sets
def test_key_positions_modes():
    S, B, W = 100, 8, 5
    assert O.key_positions(O.MODE_PREFIX, 40, B, S, W, 0).tolist() == list(range(48))
    assert O.key_positions(O.MODE_NONE, 40, B, S, W, 3).tolist() == list(range(3, 48))
    assert O.key_positions(O.MODE_DUAL, 40, B, S, W, 2).tolist() == list(range(2, 100))
    assert O.key_positions(O.MODE_DUAL_PRUNED, 40, B, S, W, 0).tolist() == \
        list(range(53)) + [99]
    # window reaching the trailing position: not duplicated
    assert O.key_positions(O.MODE_DUAL_PRUNED, 88, B, S, W, 0).tolist() == list(range(100))
    # window clipped at S
    assert O.key_positions(O.MODE_DUAL_PRUNED, 90, B, S, 50, 0).tolist() == list(range(100))
    # last block: empty suffix
    assert O.key_positions(O.MODE_DUAL_PRUNED, 92, B, S, W, 0).tolist() == list(range(100))


def test_pruned_with_large_window_equals_dual():
    for s in range(0, 96, 8):
        np.testing.assert_array_equal(O.key_positions(O.MODE_DUAL_PRUNED, s, 8, 96, 96, 4),
                                      O.key_positions(O.MODE_DUAL, s, 8, 96, 96, 4))


# ---------------------------------------------------------------- whole decode
TINY = wl.WORKLOADS["tiny"]


@pytest.fixture(scope="module")
def tiny_prefix():
    return Case(TINY)


def test_tiny_decode_invariants(tiny_prefix):
    case = tiny_prefix
    tr = case.decode()
    B = TINY.block
    assert not (tr.tokens[:, TINY.prompt_len:] < 0).any()
    # never re-masked; committed tokens never change; every block commits B rows
    seen_tok = {}
    per_block = {}
    for s, r in tr.steps:
        per_block[s] = per_block.get(s, 0) + int(r.commit.sum())
        for (bi, i) in zip(*np.where(r.commit)):
            key = (bi, s + i)
            assert key not in seen_tok
            seen_tok[key] = r.tok[bi, i]
        conf = r.conf[~np.isnan(r.conf)]
        assert np.all((conf > 0) & (conf <= 1))
    assert all(v == B for v in per_block.values())
    for (bi, p), t in seen_tok.items():
        assert tr.tokens[bi, p] == t
    assert np.array_equal(tr.tokens[:, :TINY.prompt_len], case.tokens.numpy()[:, :TINY.prompt_len])
    # prompt and step counts: each step commits >= 1
    assert all(1 <= n <= B for n in tr.steps_per_block)


def test_tiny_confidence_spread(tiny_prefix):
    # the planted states spread confidences from ~1/V to ~1 and some clear tau
    tr = tiny_prefix.decode()
    c = np.concatenate([r.conf[~np.isnan(r.conf)] for _, r in tr.steps])
    assert c.min() < 0.05 and c.max() > 0.95
    assert (c > TINY.tau).sum() >= 3


def test_prefix_cache_equals_no_cache_at_one_layer():
    # one layer: keys/values of settled positions depend only on their
    # embedding, so the cached decode must reproduce the full recompute.
    a = Case(TINY.replace(mode=wl.MODE_PREFIX)).decode()
    b = Case(TINY.replace(mode=wl.MODE_NONE)).decode()
    assert np.array_equal(a.tokens, b.tokens)
    assert a.steps_per_block == b.steps_per_block
    for (sa, ra), (sb, rb) in zip(a.steps, b.steps):
        assert sa == sb
        np.testing.assert_allclose(ra.conf, rb.conf, atol=1e-12, equal_nan=True)
        assert np.array_equal(ra.commit, rb.commit)


def test_dual_step_equals_fresh_full_forward_at_one_layer():
    # DualCache, first step of block 0: the cache from prefill must give the
    # same block output as a forward over the whole sequence built from scratch
    w = TINY.replace(mode=wl.MODE_DUAL)
    case = Case(w)
    cfg, W = case.cfg, case.W
    st = O.new_state(cfg, case.tokens.numpy(), case.masked.numpy().astype(bool),
                     case.starts.numpy())
    O.prefill(cfg, W, st)
    s = w.prompt_len
    r = O.decode_step(cfg, W, st, case.plants64, s, apply=False)
    S = w.seq_len
    x0 = W.embed(case.tokens.numpy()[:, :S])       # masked positions hold mask_id
    shape = (cfg.n_layers, 1, cfg.n_kv_heads, S, cfg.head_dim)
    kc, vc = np.zeros(shape), np.zeros(shape)
    x = O.forward_rows(cfg, W, x0, np.arange(S), [np.arange(S)], kc, vc, np.zeros(1, int), True)
    np.testing.assert_allclose(r.hidden, x[:, s:s + w.block], rtol=0, atol=1e-9)


def test_tau_above_one_takes_block_steps_in_confidence_order():
    w = TINY.replace(tau=1.5, gen_len=16)
    tr = Case(w).decode()
    assert tr.steps_per_block == [w.block] * (w.gen_len // w.block)
    for s, r in tr.steps:
        assert r.commit.sum() == 1
        m = ~np.isnan(r.conf[0])
        best = np.where(m)[0][np.argmax(r.conf[0][m])]
        assert r.commit[0, best]


def test_tau_below_one_over_v_takes_one_step_per_block():
    w = TINY.replace(tau=0.5 / TINY.vocab)
    tr = Case(w).decode()
    assert tr.steps_per_block == [1] * (w.gen_len // w.block)


def test_strong_plant_decodes_planted_token():
    # a = 50 and no noise: the target logit dominates, token = t
    w = TINY.replace(plant_a_max=50.0)
    case = Case(w, a_override=50.0, noise=False)
    r = case.decode(max_steps=1).steps[0][1]
    assert np.array_equal(r.tok[0], case.plants.t.numpy()[0, :w.block])


def test_gqa_equals_mha_with_repeated_kv_heads():
    # GQA with g = Hq/Hkv must equal MHA whose k/v weights repeat each kv head g times
    w = TINY.replace(n_q_heads=4, n_kv_heads=2, gen_len=8, rope_theta=1e4)
    case = Case(w)
    D, Hq, Hkv = w.head_dim, w.n_q_heads, w.n_kv_heads
    g = Hq // Hkv
    wq = case.weights.wqkv[:, :Hq * D]
    wk = case.weights.wqkv[:, Hq * D:(Hq + Hkv) * D].reshape(w.n_layers, Hkv, D, w.hidden)
    wv = case.weights.wqkv[:, (Hq + Hkv) * D:].reshape(w.n_layers, Hkv, D, w.hidden)
    wk_r = wk.repeat_interleave(g, dim=1).reshape(w.n_layers, Hq * D, w.hidden)
    wv_r = wv.repeat_interleave(g, dim=1).reshape(w.n_layers, Hq * D, w.hidden)
    mha_w = w.replace(n_kv_heads=Hq)
    mha = Case(mha_w)
    mha.weights.wqkv = torch.cat([wq, wk_r, wv_r], dim=1)
    mha.weights.wo = case.weights.wo
    mha.weights.w_lm = case.weights.w_lm
    from tests.oracle_inputs import oracle_weights
    mha.W = oracle_weights(mha.weights)
    mha.plants64 = case.plants64
    a, b = case.decode(), mha.decode()
    assert np.array_equal(a.tokens, b.tokens)
    for (_, ra), (_, rb) in zip(a.steps, b.steps):
        np.testing.assert_allclose(ra.conf, rb.conf, atol=1e-12, equal_nan=True)


def test_batch_sequences_independent_with_left_padding():
    # two sequences with different prompt lengths, left-padded to the longest:
    # each must decode exactly as it does alone without padding (RoPE on)
    w = TINY.replace(batch=3, prompt_len=64, prompt_len_min=40, rope_theta=1e4,
                     mode=wl.MODE_DUAL, gen_len=16)
    case = Case(w)
    tr = case.decode()
    starts = case.starts.numpy()
    assert len(set(starts.tolist())) > 1
    for bi in range(w.batch):
        st = int(starts[bi])
        wa = w.replace(batch=1, prompt_len=w.prompt_len - st, prompt_len_min=None)
        alone = Case(wa)
        alone.tokens = case.tokens[bi:bi + 1, st:].clone()
        alone.masked = case.masked[bi:bi + 1, st:].clone()
        alone.starts = torch.zeros(1, dtype=torch.int32)
        alone.plants64 = alone.plants64 * 0 + case.plants64[bi:bi + 1]
        ta = alone.decode()
        np.testing.assert_array_equal(ta.tokens[0], tr.tokens[bi, st:])


def test_pruned_large_window_decode_equals_dual():
    w = TINY.replace(mode=wl.MODE_DUAL, gen_len=24)
    a = Case(w).decode()
    b = Case(w.replace(mode=wl.MODE_DUAL_PRUNED, window=w.gen_len)).decode()
    assert np.array_equal(a.tokens, b.tokens)
    for (_, ra), (_, rb) in zip(a.steps, b.steps):
        np.testing.assert_allclose(ra.conf, rb.conf, atol=1e-12, equal_nan=True)


def test_pruned_small_window_differs_from_dual():
    # the pruned key set is really smaller: confidences change
    w = TINY.replace(mode=wl.MODE_DUAL, gen_len=32)
    a = Case(w).decode(max_steps=1)
    b = Case(w.replace(mode=wl.MODE_DUAL_PRUNED, window=4)).decode(max_steps=1)
    assert np.abs(np.nan_to_num(a.steps[0][1].conf) - np.nan_to_num(b.steps[0][1].conf)).max() > 1e-9


def test_refresh_writes_committed_block_kv():
    # after a block is done, its cache rows are the keys/values of its
    # committed tokens (one layer: k = Wk E[token], rounded to bf16)
    w = TINY.replace(mode=wl.MODE_PREFIX, gen_len=8)
    case = Case(w)
    cfg, W = case.cfg, case.W
    st = O.new_state(cfg, case.tokens.numpy(), case.masked.numpy().astype(bool),
                     case.starts.numpy())
    O.prefill(cfg, W, st)
    s = w.prompt_len
    while st.masked[:, s:s + w.block].any():
        O.decode_step(cfg, W, st, case.plants64, s)
    O.refresh_block(cfg, W, st, s)
    D, Hq, Hkv = w.head_dim, w.n_q_heads, w.n_kv_heads
    e = W.embed(st.tokens[0, s:s + w.block])
    scale = 1.0 / np.sqrt((e * e).mean(axis=1) + 1e-6)
    k = (O.round_bf16(e) @ W.wqkv(0)[Hq * D:(Hq + Hkv) * D].T) * scale[:, None]
    want = O.round_bf16(k.reshape(w.block, Hkv, D).transpose(1, 0, 2))
    np.testing.assert_array_equal(st.kcache[0, 0][:, s:s + w.block], want)


# ---------------------------------------------------------------- fixed-budget (top-k) commit
def _schedule(B, S):
    ks, m = [], B
    while m:
        k = O.topk_budget(B, S, m)
        ks.append(k)
        m -= k
    return ks


def test_topk_budget_spreads_the_block_over_the_steps():
    assert _schedule(32, 5) == [7, 7, 6, 6, 6]
    assert _schedule(32, 8) == [4] * 8
    assert _schedule(32, 32) == [1] * 32
    assert _schedule(32, 1) == [32]
    assert _schedule(8, 3) == [3, 3, 2]
    for B in (8, 32, 64):
        for S in range(1, B + 1):
            ks = _schedule(B, S)
            assert len(ks) == S and sum(ks) == B and max(ks) - min(ks) <= 1


def test_topk_commit_picks_the_most_confident_rows_lowest_position_first():
    rng = np.random.default_rng(7)
    for _ in range(200):
        B = int(rng.integers(1, 65))
        conf = np.round(rng.random(B), 1)            # coarse values: many ties
        masked = rng.random(B) < 0.7
        if not masked.any():
            continue
        k = int(rng.integers(1, masked.sum() + 1))
        c = O.topk_commit(conf, masked, k)
        assert c.sum() == k and not (c & ~masked).any()
        # every committed row beats every masked row left out, (conf, -position) lexicographic
        for i in np.where(c)[0]:
            for j in np.where(masked & ~c)[0]:
                assert conf[i] > conf[j] or (conf[i] == conf[j] and i < j)


def test_topk_with_one_row_per_step_equals_tau_above_one():
    w1 = TINY.replace(commit_mode=wl.COMMIT_TOPK, steps_per_block=TINY.block, gen_len=16)
    w2 = TINY.replace(tau=1.5, gen_len=16)
    t1, t2 = Case(w1).decode(), Case(w2).decode()
    assert np.array_equal(t1.tokens, t2.tokens)
    assert t1.steps_per_block == t2.steps_per_block == [TINY.block] * 2


def test_topk_decode_takes_exactly_the_step_budget():
    w = TINY.replace(commit_mode=wl.COMMIT_TOPK, steps_per_block=3, gen_len=16)
    tr = Case(w).decode()
    assert tr.steps_per_block == [3, 3]
    per_step = [int(r.commit.sum()) for _, r in tr.steps]
    assert per_step == [3, 3, 2, 3, 3, 2]
    assert not (tr.tokens[:, w.prompt_len:] < 0).any()


def test_topk_single_step_commits_the_whole_block():
    w = TINY.replace(commit_mode=wl.COMMIT_TOPK, steps_per_block=1, gen_len=16)
    tr = Case(w).decode()
    assert tr.steps_per_block == [1, 1]


# ---------------------------------------------------------------- prefix cache, suffix as queries
def test_suffix_query_mode_keys_are_the_whole_valid_range():
    for start in (0, 3):
        np.testing.assert_array_equal(
            O.key_positions(O.MODE_PREFIX_SUFFIXQ, 72, 8, 96, 0, start), np.arange(start, 96))


def test_suffix_query_step_equals_dual_step_at_one_layer():
    # with one layer a key/value depends only on its own embedding, so the
    # suffix keys the step recomputes equal the ones DualCache's prefill cached:
    # the block rows see identical keys and values
    w4 = TINY.replace(mode=wl.MODE_PREFIX_SUFFIXQ)
    w2 = TINY.replace(mode=wl.MODE_DUAL)
    r = {}
    for w in (w4, w2):
        case = Case(w)
        cfg, W = case.cfg, case.W
        st = O.new_state(cfg, case.tokens.numpy(), case.masked.numpy().astype(bool),
                         case.starts.numpy())
        O.prefill(cfg, W, st)
        r[w.mode] = O.decode_step(cfg, W, st, case.plants64, w.prompt_len, apply=False)
    np.testing.assert_allclose(r[4].hidden, r[2].hidden, rtol=0, atol=1e-12)
    assert np.array_equal(r[4].tok, r[2].tok)
    np.testing.assert_allclose(r[4].conf, r[2].conf, rtol=0, atol=1e-12)


def test_suffix_query_mode_differs_from_dual_with_two_layers():
    # from the second layer on, the recomputed suffix states attend to the
    # current block, so the two readings part
    w4 = TINY.replace(mode=wl.MODE_PREFIX_SUFFIXQ, n_layers=2)
    w2 = TINY.replace(mode=wl.MODE_DUAL, n_layers=2)
    h = {}
    for w in (w4, w2):
        case = Case(w)
        cfg, W = case.cfg, case.W
        st = O.new_state(cfg, case.tokens.numpy(), case.masked.numpy().astype(bool),
                         case.starts.numpy())
        O.prefill(cfg, W, st)
        h[w.mode] = O.decode_step(cfg, W, st, case.plants64, w.prompt_len, apply=False).hidden
    assert np.abs(h[4] - h[2]).max() > 1e-6


def test_suffix_query_decode_invariants():
    w = TINY.replace(mode=wl.MODE_PREFIX_SUFFIXQ, gen_len=16)
    tr = Case(w).decode()
    assert all(1 <= n <= w.block for n in tr.steps_per_block)
    assert not (tr.tokens[:, w.prompt_len:] < 0).any()
    for s, r in tr.steps:
        conf = r.conf[~np.isnan(r.conf)]
        assert np.all((conf > 0) & (conf <= 1))


# ---------------------------------------------------------------- step cap on the threshold rule
def test_step_cap_of_one_commits_each_block_in_one_step():
    w = TINY.replace(steps_per_block=1, gen_len=16)
    tr = Case(w).decode()
    assert tr.steps_per_block == [1, 1]
    for _, r in tr.steps:
        assert r.commit.sum() == w.block


def test_step_cap_at_block_size_changes_nothing():
    w = TINY.replace(gen_len=16)
    t0 = Case(w).decode()
    t1 = Case(w.replace(steps_per_block=w.block)).decode()
    assert np.array_equal(t0.tokens, t1.tokens)
    assert t0.steps_per_block == t1.steps_per_block


def test_step_cap_of_two_finishes_every_block_by_its_second_step():
    w = TINY.replace(steps_per_block=2, gen_len=16)
    tr = Case(w).decode()
    assert all(n <= 2 for n in tr.steps_per_block)
    for s, r in tr.steps:
        m = ~np.isnan(r.conf[0])
        if r.commit[0][m].all() and m.sum() > 1:
            break
    else:
        raise AssertionError("no step committed a whole multi-row remainder")


# ---------------------------------------------------------------- block state
def test_block_state_done_and_refresh_rule():
    m = np.array([True, False, True])
    assert O.block_state(m, np.zeros(3, bool), 96) == (True, 96)      # this commit finished it
    assert O.block_state(np.zeros(3, bool), np.zeros(3, bool), 96) == (True, -1)  # already done
    assert O.block_state(m, np.array([False, False, True]), 96) == (False, -1)


def test_block_state_over_a_decode_with_tau_above_one():
    # one commit per step: the block is done, and due for its refresh, at
    # exactly its B-th step and at no other
    w = TINY.replace(tau=1.5)
    case = Case(w)
    tr = case.decode()
    B = w.block
    masked = case.masked.numpy().astype(bool).copy()
    k = 0
    for s, r in tr.steps:
        before = masked[0, s:s + B].copy()
        masked[0, s:s + B] &= ~r.commit[0]
        done, refresh = O.block_state(before, masked[0, s:s + B], s)
        k = k + 1 if k < B else 1
        assert done == (k == B) and refresh == (s if k == B else -1)


# ---------------------------------------------------------------- early exit
def test_early_exit_commit_cases():
    tau, ex = 0.9, 0.5
    conf = np.array([0.60, 0.60, 0.95, 0.40, 0.70, 0.55])
    tok = np.array([3, 4, 5, 6, 7, 8])
    prev = np.array([3, 9, 1, 6, -1, 8])      # rows 0, 3, 5 repeat; row 4 has no previous
    masked = np.array([True, True, True, True, True, False])
    c = O.early_exit_commit(conf, tok, prev, masked, tau, ex)
    # 0: repeats and clears exit_tau; 1: changed; 2: clears tau; 3: repeats but
    # below exit_tau; 4: no previous step; 5: not masked
    assert c.tolist() == [True, False, True, False, False, False]
    # the most confident masked row commits even when nothing else does
    c = O.early_exit_commit(np.array([0.3, 0.4]), np.array([1, 2]), np.array([-1, -1]),
                            np.ones(2, bool), tau, ex)
    assert c.tolist() == [False, True]
    # exit_tau at tau: the plain threshold rule
    for _ in range(50):
        conf = RNG.uniform(0, 1, 12)
        tok = RNG.integers(0, 3, 12)
        prev = RNG.integers(-1, 3, 12)
        masked = RNG.uniform(size=12) < 0.8
        masked[0] = True
        np.testing.assert_array_equal(O.early_exit_commit(conf, tok, prev, masked, tau, tau),
                                      O.threshold_commit(conf, masked, tau))


def test_early_exit_finishes_converged_blocks_in_two_steps():
    # planted confidences between exit_tau and tau, argmax fixed by the plant:
    # the threshold rule commits one forced row per step (B steps per block);
    # with the early exit every other row has repeated its argmax by the
    # second step and commits there
    base = TINY.replace(tau=0.9)
    thr = Case(base, a_override=8.0, noise=False).decode()
    assert thr.steps_per_block == [base.block] * (base.gen_len // base.block)
    ex = base.replace(commit_mode=wl.COMMIT_EARLY_EXIT, exit_tau=0.5)
    tr = Case(ex, a_override=8.0, noise=False).decode()
    assert tr.steps_per_block == [2] * (base.gen_len // base.block)
    # converged rows commit the token they repeated: the same sequence
    np.testing.assert_array_equal(tr.tokens, thr.tokens)


def test_early_exit_at_or_above_tau_is_the_threshold_decode():
    base = TINY
    thr = Case(base).decode()
    ex = Case(base.replace(commit_mode=wl.COMMIT_EARLY_EXIT, exit_tau=base.tau)).decode()
    assert ex.steps_per_block == thr.steps_per_block
    np.testing.assert_array_equal(ex.tokens, thr.tokens)


def test_early_exit_decode_invariants():
    w = TINY.replace(commit_mode=wl.COMMIT_EARLY_EXIT, exit_tau=0.3)
    tr = Case(w).decode()
    B = w.block
    assert not (tr.tokens == -1).any()
    prev_block, prev = None, None
    for s, r in tr.steps:
        if s != prev_block:
            prev_block, prev = s, None
        m = ~np.isnan(r.conf[0])
        c = r.commit[0]
        assert c.any() and not (c & ~m).any()
        # every committed row cleared tau, repeated its argmax above exit_tau,
        # or is the forced pick
        best = int(np.argmax(np.where(m, r.conf[0], -np.inf)))
        for i in np.where(c)[0]:
            rep_ = prev is not None and prev[i] == r.tok[0, i]
            assert r.conf[0, i] > w.tau or (rep_ and r.conf[0, i] > w.exit_tau) or i == best
        prev = r.tok[0].copy()
    assert all(1 <= n <= B for n in tr.steps_per_block)
