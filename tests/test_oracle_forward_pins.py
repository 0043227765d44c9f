"""Brute-force pins of the oracle's layer stack, LM-head input and ambiguity flags.

The layer composition of ``forward_rows`` (RMS-normalised projection input,
rotary embedding, non-causal attention over the key set, output projection
added to the residual) and the LM-head input of ``lm_input`` are recomputed
here with explicit scalar Python loops over hand-sized shapes (hidden 8, one
or two query heads), without numpy linear algebra.  Each test also computes
the plausible mistakes (no residual, the norm applied after the residual
add, no 1/sqrt(D), a transposed W_o, the wrong GQA map, RoPE at the wrong
position, no RMS scale on the LM-head input) and checks that every one of them
is far from the oracle, so that the pin would catch it.

``ambiguity_flags`` decides which GPU decisions the lockstep tests excuse;
its three bands and a row outside all of them are checked on hand-built
confidence / gap vectors.
"""
import math

import numpy as np
import pytest

from oracle import dllm_oracle as O

EPS = O.RMS_EPS


# ---------------------------------------------------------------- brute force
def _matvec(W, x):
    """W [n][m] (nested lists) times x [m]."""
    return [sum(W[i][k] * x[k] for k in range(len(x))) for i in range(len(W))]


def _rope_vec(v, pos, theta):
    """Rotate-half rotary embedding of one head vector at one position."""
    D = len(v)
    half = D // 2
    out = list(v)
    for i in range(half):
        ang = pos * theta ** (-2.0 * i / D)
        c, s = math.cos(ang), math.sin(ang)
        out[i] = v[i] * c - v[i + half] * s
        out[i + half] = v[i + half] * c + v[i] * s
    return out


def _softmax_attn(q, ks, vs):
    D = len(q)
    sc = [sum(q[j] * k[j] for j in range(D)) / math.sqrt(D) for k in ks]
    m = max(sc)
    e = [math.exp(x - m) for x in sc]
    z = sum(e)
    return [sum(e[i] * vs[i][j] for i in range(len(ks))) / z for j in range(D)]


def brute_forward(x0, rows, keys, kcache, vcache, wqkv, wo, Hq, Hkv, D, theta, start,
                  mistake=None):
    """Layer stack of one sequence with scalar loops.

    x0 [n][d] inputs of query rows at positions ``rows``; keys: key positions;
    kcache/vcache [L][Hkv][S][D] hold the keys/values of positions that are not
    query rows (the rows' own are written here, layer by layer).  Per layer:
    r = 1/sqrt(mean(x^2) + eps); q, k, v = r * (W_qkv x); RoPE at position
    p - start on q and k; o_h = softmax(q_h . K / sqrt(D)) V with kv head
    h // (Hq / Hkv); x <- x + W_o [o_0 ... o_{Hq-1}].  ``mistake`` names one
    plausible slip to reproduce instead.
    """
    L = len(wqkv)
    g = Hq // Hkv
    x = [list(r) for r in x0]
    kc = [[[list(kcache[l][h][p]) for p in range(len(kcache[l][h]))] for h in range(Hkv)]
          for l in range(L)]
    vc = [[[list(vcache[l][h][p]) for p in range(len(vcache[l][h]))] for h in range(Hkv)]
          for l in range(L)]
    for l in range(L):
        W = wqkv[l]
        qs, ks_new, vs_new = [], [], []
        for i, xi in enumerate(x):
            d = len(xi)
            r = 1.0 / math.sqrt(sum(t * t for t in xi) / d + EPS)
            y = [r * t for t in _matvec(W, xi)]
            q = [y[h * D:(h + 1) * D] for h in range(Hq)]
            k = [y[(Hq + h) * D:(Hq + h + 1) * D] for h in range(Hkv)]
            v = [y[(Hq + Hkv + h) * D:(Hq + Hkv + h + 1) * D] for h in range(Hkv)]
            if theta > 0:
                pos = rows[i] - (0 if mistake == "rope_absolute" else start)
                q = [_rope_vec(t, pos, theta) for t in q]
                k = [_rope_vec(t, pos, theta) for t in k]
            qs.append(q)
            ks_new.append(k)
            vs_new.append(v)
        for i, p in enumerate(rows):
            for h in range(Hkv):
                kc[l][h][p] = ks_new[i][h]
                vc[l][h][p] = vs_new[i][h]
        new_x = []
        for i, xi in enumerate(x):
            o = []
            for h in range(Hq):
                kvh = (h % Hkv) if mistake == "gqa_modulo" else h // g
                qv = qs[i][h]
                if mistake == "no_scale":
                    qv = [t * math.sqrt(D) for t in qv]
                o += _softmax_attn(qv, [kc[l][kvh][p] for p in keys],
                                   [vc[l][kvh][p] for p in keys])
            if mistake == "wo_transposed":
                Wo = [[wo[l][j][i2] for j in range(len(wo[l]))] for i2 in range(len(wo[l][0]))]
            else:
                Wo = wo[l]
            add = _matvec(Wo, o)
            if mistake == "no_residual":
                new_x.append(add)
            elif mistake == "post_norm":
                z = [xi[j] + add[j] for j in range(len(xi))]
                r = 1.0 / math.sqrt(sum(t * t for t in z) / len(z) + EPS)
                new_x.append([r * t for t in z])
            else:
                new_x.append([xi[j] + add[j] for j in range(len(xi))])
        x = new_x
    return x, kc, vc


# ---------------------------------------------------------------- cases
def _case(L, Hq, Hkv, D, d, theta, n_rows=3, S=7, start=1, seed=0):
    """Hand-sized inputs: weights and inputs of mixed signs and magnitudes
    (entries of order 0.3, so that attention weights are far from uniform)."""
    rng = np.random.default_rng(seed)
    wqkv = rng.standard_normal((L, (Hq + 2 * Hkv) * D, d)) * 0.6
    wo = rng.standard_normal((L, d, Hq * D)) * 0.5
    x0 = rng.standard_normal((1, n_rows, d)) * 1.5
    kc = rng.standard_normal((L, 1, Hkv, S, D))
    vc = rng.standard_normal((L, 1, Hkv, S, D))
    rows = np.arange(S - n_rows - 1, S - 1)           # a block with one position after it
    keys = np.arange(start, S)                         # prefix, block and suffix
    cfg = O.Config(batch=1, n_layers=L, hidden=d, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=D,
                   vocab=16, prompt_len=int(rows[0]), gen_len=S - int(rows[0]),
                   block=n_rows, tau=0.9, mode=O.MODE_DUAL, window=0, rope_theta=theta,
                   mask_id=15)
    W = O.Weights(lambda l: wqkv[l], lambda l: wo[l], rng.standard_normal((16, d)))
    return cfg, W, wqkv, wo, x0, kc, vc, rows, keys, start


def _oracle(cfg, W, x0, kc, vc, rows, keys, start):
    kco, vco = kc.copy(), vc.copy()
    x = O.forward_rows(cfg, W, x0, rows, [keys], kco, vco, np.array([start]), mirror=False)
    return x[0], kco, vco


def _brute(args, mistake=None):
    cfg, W, wqkv, wo, x0, kc, vc, rows, keys, start = args
    x, kb, vb = brute_forward(x0[0].tolist(), [int(p) for p in rows], [int(p) for p in keys],
                              kc[:, 0].tolist(), vc[:, 0].tolist(), wqkv.tolist(), wo.tolist(),
                              cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.rope_theta, start,
                              mistake)
    return np.array(x), np.array(kb), np.array(vb)


SHAPES = {
    "one_layer_one_head": dict(L=1, Hq=1, Hkv=1, D=8, d=8, theta=0.0),
    "two_layers_rope": dict(L=2, Hq=1, Hkv=1, D=8, d=8, theta=10.0),
    "two_layers_gqa": dict(L=2, Hq=2, Hkv=1, D=4, d=8, theta=0.0),
    "three_layers_gqa_rope": dict(L=3, Hq=4, Hkv=2, D=4, d=8, theta=100.0),
}


@pytest.mark.parametrize("name", list(SHAPES))
def test_forward_rows_equals_scalar_loop_stack(name):
    args = _case(**SHAPES[name], seed=len(name))
    cfg, W, wqkv, wo, x0, kc, vc, rows, keys, start = args
    xo, ko, vo = _oracle(cfg, W, x0, kc, vc, rows, keys, start)
    xb, kb, vb = _brute(args)
    np.testing.assert_allclose(xo, xb, rtol=1e-12, atol=1e-12)
    # every layer's keys/values of the query rows, and untouched cache rows
    np.testing.assert_allclose(ko[:, 0], kb, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(vo[:, 0], vb, rtol=1e-12, atol=1e-12)


MISTAKES = {
    "no_residual": SHAPES["two_layers_rope"],
    "post_norm": SHAPES["two_layers_rope"],
    "no_scale": SHAPES["one_layer_one_head"],
    "wo_transposed": SHAPES["two_layers_rope"],
    "gqa_modulo": SHAPES["three_layers_gqa_rope"],
    "rope_absolute": SHAPES["two_layers_rope"],
}


@pytest.mark.parametrize("mistake", list(MISTAKES))
def test_each_plausible_slip_moves_the_stack_far_from_the_oracle(mistake):
    args = _case(**MISTAKES[mistake], seed=len(mistake))
    cfg, W, wqkv, wo, x0, kc, vc, rows, keys, start = args
    xo, _, _ = _oracle(cfg, W, x0, kc, vc, rows, keys, start)
    xb, _, _ = _brute(args, mistake)
    assert np.abs(xo - xb).max() > 1e-3, f"{mistake} would not be caught"


def test_oracle_stack_is_not_the_embedding_alone():
    # the layers change the residual by an O(1) amount on these inputs, so a
    # stack that skipped them would fail the equality pins above
    args = _case(**SHAPES["two_layers_rope"], seed=3)
    cfg, W, wqkv, wo, x0, kc, vc, rows, keys, start = args
    xo, _, _ = _oracle(cfg, W, x0, kc, vc, rows, keys, start)
    assert np.abs(xo - x0[0]).max() > 0.1


# ---------------------------------------------------------------- LM-head input
def _brute_lm_input(x, plants, masked, rms=True):
    out = []
    for i, xi in enumerate(x):
        d = len(xi)
        r = 1.0 / math.sqrt(sum(t * t for t in xi) / d + EPS) if rms else 1.0
        out.append([r * xi[j] + (plants[i][j] if masked[i] else 0.0) for j in range(d)])
    return out


def test_lm_input_is_normalised_residual_plus_plant_where_masked():
    rng = np.random.default_rng(7)
    B, d, P = 5, 8, 10
    cfg = O.Config(batch=1, n_layers=1, hidden=d, n_q_heads=1, n_kv_heads=1, head_dim=8,
                   vocab=16, prompt_len=P, gen_len=2 * B, block=B, tau=0.9, mode=O.MODE_DUAL,
                   window=0, rope_theta=0.0, mask_id=15)
    x = rng.standard_normal((1, B, d)) * 7.0          # far from unit RMS
    plants = rng.standard_normal((1, 2 * B, d))
    masked = np.array([[True, False, True, True, False]])
    s = P + B                                          # the second block: plants [B, 2B)
    got = O.lm_input(cfg, x, plants, masked, s, mirror=False)[0]
    want = _brute_lm_input(x[0].tolist(), plants[0, B:2 * B].tolist(), masked[0].tolist())
    np.testing.assert_allclose(got, np.array(want), rtol=1e-13, atol=1e-13)
    # mistakes the pin catches: no RMS scale, the first block's plants
    no_rms = _brute_lm_input(x[0].tolist(), plants[0, B:2 * B].tolist(), masked[0].tolist(),
                             rms=False)
    assert np.abs(got - np.array(no_rms)).max() > 1.0
    wrong_block = _brute_lm_input(x[0].tolist(), plants[0, :B].tolist(), masked[0].tolist())
    assert np.abs(got - np.array(wrong_block)).max() > 0.1
    # unmasked rows carry no plant: unit RMS exactly
    for i in np.where(~masked[0])[0]:
        assert abs(float(np.mean(got[i] ** 2)) - 1.0) < 1e-5


# ---------------------------------------------------------------- ambiguity flags
TAU = 0.9


def _flags(conf, gap, masked):
    return O.ambiguity_flags(np.array(conf, dtype=np.float64), np.array(gap, dtype=np.float64),
                             np.array(masked, dtype=bool), TAU)


def test_flag_band_i_top2_logit_gap():
    conf = [0.30, 0.40, 0.50, 0.60]
    gap = [0.005, 0.0099, 0.0101, 0.5]
    amb_tok, amb_commit = _flags(conf, gap, [True, True, True, True])
    assert amb_tok.tolist() == [True, True, False, False]
    assert not amb_commit.any()
    # an unmasked row is never flagged, whatever its gap
    amb_tok, _ = _flags(conf, gap, [False, True, True, True])
    assert amb_tok.tolist() == [False, True, False, False]


def test_flag_band_ii_conf_near_threshold():
    conf = [TAU - 0.0015, TAU + 0.0019, TAU + 0.0021, TAU - 0.0030, 0.95]
    gap = [1.0] * 5
    amb_tok, amb_commit = _flags(conf, gap, [True] * 5)
    assert not amb_tok.any()
    assert amb_commit.tolist() == [True, True, False, False, False]


def test_flag_band_iii_forced_pick_between_close_leaders():
    # nothing clears tau: every masked row within 2e-3 of the leader (0.5015)
    # may take the forced pick instead of it; 0.4985 is 3e-3 below the leader
    amb_tok, amb_commit = _flags([0.5000, 0.5015, 0.20, 0.4985, 0.5001], [1.0] * 5, [True] * 5)
    assert amb_commit.tolist() == [True, True, False, False, True]
    # leaders 1e-2 apart: the forced pick is unambiguous
    _, amb_commit = _flags([0.50, 0.51, 0.20], [1.0] * 3, [True] * 3)
    assert not amb_commit.any()
    # the leader clears tau by more than the band: every row above tau commits
    # anyway, so closeness of the top two does not matter
    _, amb_commit = _flags([0.95, 0.9495, 0.20], [1.0] * 3, [True] * 3)
    assert not amb_commit.any()
    # a masked row close to an UNmasked one is not a forced-pick tie
    _, amb_commit = _flags([0.5000, 0.5010, 0.20], [1.0] * 3, [True, False, True])
    assert not amb_commit.any()


def test_rows_outside_every_band_are_never_flagged():
    rng = np.random.default_rng(5)
    for _ in range(200):
        n = int(rng.integers(2, 12))
        # well-separated confidences away from tau, large gaps
        base = rng.permutation(np.linspace(0.05, 0.85, 40))[:n]
        conf = np.where(rng.random(n) < 0.3, np.clip(base + 0.12, 0.0, 0.99), base)
        conf = np.where(np.abs(conf - TAU) < 0.01, conf - 0.02, conf)
        srt = np.sort(conf)
        if n > 1 and np.diff(srt).min() < 0.005:
            continue
        gap = rng.uniform(0.02, 5.0, n)
        masked = rng.random(n) < 0.8
        amb_tok, amb_commit = _flags(conf, gap, masked)
        assert not amb_tok.any() and not amb_commit.any()
