"""Plain fp64 CPU oracle of the masked-diffusion block-decode step.

TEST INFRASTRUCTURE.  Only the test suite, the package smoke check and the
benchmark's CPU-baseline leg may import this module.  It shares no code with
the CUDA library and imports nothing from it.

What it computes (sources, by page title and section):

* Fast-dLLM README ("Fast-dLLM", project table, row "Key Techniques"):
  v1 decodes with "KV Cache + Parallel Decoding" on Dream/LLaDA backbones.
* "Fast-dLLM: Four Acceleration Tracks ...", section "The v1 Mechanism":
  every masked position of the block is evaluated in parallel, the ones whose
  confidence exceeds the threshold are committed, a committed token is never
  revised, and a key/value cache keeps the attention state of settled
  positions so that it is not recomputed.
* Same page, section "Fast-dLLM v1 Versus a Standard Diffusion Sampler":
  the cache plus the threshold, on top of a block schedule.
* Fast-dLLM README, "Quick Start": the knobs gen_length, block_size,
  threshold=0.9, use_cache, alg=confidence_threshold.
* Streaming-dLLM README, figure "Illustration of approximated suffix
  pruning": the suffix is cut to a sliding window right after the block plus
  the trailing position.

The pages give no formulas.  Where they are silent this module takes the
plainest reading that the rest supports:
textbook scaled-dot-product softmax attention with scale 1/sqrt(D) and
contiguous GQA groups; rotate-half rotary embedding; confidence = the largest
softmax probability over the whole vocabulary; argmax ties go to the lowest
id; the threshold test is strict ``conf > tau``; at least the single most
confident masked row commits each step (lowest position on ties); the key set
per cache mode is given by :func:`key_positions`.

Layer stack.  The backbones the workloads are shaped like (LLaDA-8B,
Dream-7B / Qwen2.5-7B) are pre-norm transformers; with the MLP replaced by identity each layer is
    x <- x + Wo . attention(q, k, v),   (q, k, v) = W_qkv . x / rms(x)
with a weightless RMSNorm (eps 1e-6), and the LM head reads the final
RMSNorm of the residual.  Without the norms, random N(0, 0.02^2) weights at
d = 4096 have operator norm ~1.3 and the residual overflows within ~24
layers.  A masked row's layer-0 input is the embedding of the mask token;
its planted hidden state is added to the LM-head input (final normalised
hidden state), which keeps the planted confidence spread at any depth.

Precision.  Everything is float64.  With ``mirror=True`` values are rounded at
the points where the CUDA path stores them: the projection input (bf16), q/k/v
after RoPE (bf16), the attention output (bf16), the residual stream after each
layer (fp32) and the LM-head input (bf16).  Logits are never rounded.
"""
from __future__ import annotations

import dataclasses
from typing import Callable, Optional, Sequence

import numpy as np

MODE_NONE, MODE_PREFIX, MODE_DUAL, MODE_DUAL_PRUNED = 0, 1, 2, 3
MODE_PREFIX_SUFFIXQ = 4   # prefix cache; block and suffix recomputed as queries every step
COMMIT_THRESHOLD, COMMIT_TOPK, COMMIT_EARLY_EXIT = 0, 1, 2

AMBIG_GAP = 1e-2     # top-2 logit gap below which an argmax is ambiguous
AMBIG_CONF = 2e-3    # |conf - tau| (or forced-pick conf difference) band


# --------------------------------------------------------------------------
# Rounding helpers
# --------------------------------------------------------------------------
def round_bf16(x) -> np.ndarray:
    """Round to the nearest bfloat16 (ties to even), returned as float64.

    The value is first rounded to float32, then its 16 low bits are rounded
    away with round-half-to-even on the bit pattern.
    """
    x32 = np.asarray(x, dtype=np.float64).astype(np.float32)
    bits = x32.view(np.uint32).astype(np.uint64)
    lsb = (bits >> np.uint64(16)) & np.uint64(1)
    bits = (bits + np.uint64(0x7FFF) + lsb) & np.uint64(0xFFFF0000)
    return bits.astype(np.uint32).view(np.float32).astype(np.float64)


def round_f32(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


RMS_EPS = 1e-6


def inv_rms(x: np.ndarray) -> np.ndarray:
    """1 / sqrt(mean(x^2) + eps) over the last axis (weightless RMSNorm scale)."""
    return 1.0 / np.sqrt(np.mean(x * x, axis=-1) + RMS_EPS)


# --------------------------------------------------------------------------
# Building blocks
# --------------------------------------------------------------------------
def rope(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotary position embedding, rotate-half form, on the last axis.

    ``x`` is [..., n, D] and ``pos`` is [n].  Dimension i < D/2 is paired with
    i + D/2 and rotated by angle pos * theta^(-2i/D).
    """
    D = x.shape[-1]
    half = D // 2
    inv_freq = theta ** (-(2.0 * np.arange(half, dtype=np.float64)) / D)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * inv_freq[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """Non-causal scaled-dot-product attention of one head.

    q [n, D], k [m, D], v [m, D] -> o [n, D];  o = softmax(q k^T / sqrt(D)) v.
    """
    D = q.shape[-1]
    s = (q @ k.T) / np.sqrt(D)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=1, keepdims=True)
    return p @ v


def key_positions(mode: int, s: int, B: int, S: int, window: int, start: int) -> np.ndarray:
    """Key positions a block row attends to, for a block at [s, s+B).

    start is the sequence's first valid position (left padding before it).
      NONE / PREFIX : prefix and block, [start, s+B)
      DUAL          : prefix, block and the whole suffix, [start, S)
      DUAL_PRUNED   : prefix, block, the window [s+B, min(s+B+window, S)) and
                      the trailing position S-1 (once) when the suffix is not
                      empty.
      PREFIX_SUFFIXQ: prefix, block and suffix, [start, S); the suffix keys
                      are recomputed by the step itself (its rows are queries)
    """
    end = s + B
    if mode in (MODE_NONE, MODE_PREFIX):
        return np.arange(start, end)
    if mode in (MODE_DUAL, MODE_PREFIX_SUFFIXQ):
        return np.arange(start, S)
    if mode == MODE_DUAL_PRUNED:
        wend = min(end + window, S)
        pos = list(range(start, wend))
        if end < S and S - 1 >= wend:
            pos.append(S - 1)
        return np.asarray(pos, dtype=np.int64)
    raise ValueError(f"unknown mode {mode}")


def lm_head_confidence(h: np.ndarray, w_lm: np.ndarray):
    """Max-softmax confidence, argmax token and top-2 logit gap of each row.

    h [n, d], w_lm [V, d].  logits = h w_lm^T;  m = max logit;
    conf = 1 / sum_v exp(logit_v - m);  tok = lowest id with logit == m;
    gap = m - (second largest logit, counting a tied maximum).
    """
    logits = h @ w_lm.T
    tok = np.argmax(logits, axis=1)                 # first occurrence
    m = logits[np.arange(len(tok)), tok]
    conf = 1.0 / np.exp(logits - m[:, None]).sum(axis=1)
    if logits.shape[1] > 1:
        top2 = np.partition(logits, -2, axis=1)[:, -2]
    else:
        top2 = np.full_like(m, -np.inf)
    return conf, tok.astype(np.int64), m - top2


def threshold_commit(conf: np.ndarray, masked: np.ndarray, tau: float) -> np.ndarray:
    """Rows of one block to commit this step.

    conf [B] (any value where not masked), masked [B] bool.  A masked row
    commits if conf > tau; the masked row of largest conf (lowest position on
    equal conf) always commits.  Returns a bool [B].
    """
    commit = masked & (conf > tau)
    if masked.any():
        cand = np.where(masked, conf, -np.inf)
        best = int(np.argmax(cand))                 # first occurrence = lowest position
        commit[best] = True
    return commit


def block_state(masked_before: np.ndarray, masked_after: np.ndarray, s: int):
    """One sequence's block after a commit: (done, refresh).

    done: no row of the block is left masked.  refresh: the block start s when
    this commit finished the block (some row was masked before it), else -1;
    a finished block's keys/values are then recomputed from its committed
    tokens, since the cache keeps the attention state of settled positions
    ("Fast-dLLM: Four Acceleration Tracks ...", section "The v1 Mechanism").
    """
    done = not bool(np.asarray(masked_after).any())
    return done, (int(s) if done and bool(np.asarray(masked_before).any()) else -1)


def topk_budget(block: int, steps_per_block: int, n_masked: int) -> int:
    """Rows a fixed-budget step commits (the low-confidence-remasking sampler).

    Fast-dLLM's README sets the sampler's total steps (--steps) next to the
    block length, and the Fast-dLLM overview page contrasts the cache plus
    threshold with a standard diffusion sampler.  Plainest reading of that
    sampler: a block of B masked positions is decoded in exactly S =
    steps_per_block steps; step j (0-based) commits floor(B/S) rows, plus one
    more while j < B mod S.  j is recovered from the rows already committed,
    c = B - n_masked.  Never more than n_masked.
    """
    base, rem = divmod(block, steps_per_block)
    c = block - n_masked
    if c < rem * (base + 1):
        j = c // (base + 1)
    else:
        j = rem + (c - rem * (base + 1)) // max(base, 1)
    k = base + (1 if j < rem else 0)
    return int(min(max(k, 1), n_masked))


def topk_commit(conf: np.ndarray, masked: np.ndarray, k: int) -> np.ndarray:
    """The k masked rows of highest confidence (lower position first on
    equal confidence).  Returns a bool [B]."""
    commit = np.zeros(masked.shape, dtype=bool)
    idx = np.where(masked)[0]
    order = sorted(idx, key=lambda i: (-conf[i], i))
    commit[order[:k]] = True
    return commit


def topk_ambiguity(conf, masked, k):
    """Top-k commit: the rows within AMBIG_CONF of the k-th / (k+1)-th
    boundary may land on either side of it."""
    amb = np.zeros(masked.shape, dtype=bool)
    idx = np.where(masked)[0]
    if 0 < k < len(idx):
        c = np.sort(conf[idx])[::-1]
        lo, hi = c[k], c[k - 1]
        if hi - lo < AMBIG_CONF:
            amb[idx[np.abs(conf[idx] - 0.5 * (hi + lo)) <= 0.5 * (hi - lo) + AMBIG_CONF]] = True
    return amb


def early_exit_commit(conf: np.ndarray, tok: np.ndarray, prev_tok: np.ndarray,
                      masked: np.ndarray, tau: float, exit_tau: float) -> np.ndarray:
    """Threshold commit with an early exit for converged rows.

    Streaming-dLLM's abstract (listing page, third abstract) names a dynamic,
    confidence-aware strategy with an early exit that skips the remaining
    iterations of converged tokens, without a formula.  Reading: a masked row
    has converged when its argmax equals its argmax at the previous step of
    the same block (prev_tok; -1 where there is none, as at a block's first
    step); a converged row commits once its confidence exceeds exit_tau, a
    bound at or below tau, instead of tau.  Rows with conf > tau commit as in
    the plain rule, and the most confident masked row always commits (lowest
    position on ties).  exit_tau >= tau gives the plain threshold rule.
    Returns a bool [B].
    """
    stable = masked & (prev_tok >= 0) & (tok == prev_tok)
    commit = masked & ((conf > tau) | (stable & (conf > exit_tau)))
    if masked.any():
        cand = np.where(masked, conf, -np.inf)
        commit[int(np.argmax(cand))] = True
    return commit


def early_exit_ambiguity(conf, gap, tok, prev_tok, masked, tau, exit_tau):
    """Flags of the early-exit rule: the threshold rule's bands, rows whose
    confidence is within 2e-3 of exit_tau while their argmax repeats, and rows
    whose argmax itself is ambiguous (top-2 gap < 1e-2) while their confidence
    could clear exit_tau, since their 'repeats' test may go either way."""
    amb_tok, amb_commit = ambiguity_flags(conf, gap, masked, tau)
    has_prev = masked & (prev_tok >= 0)
    stable = has_prev & (tok == prev_tok)
    amb_commit = (amb_commit | (stable & (np.abs(conf - exit_tau) < AMBIG_CONF))
                  | (has_prev & (gap < AMBIG_GAP) & (conf > exit_tau - AMBIG_CONF)))
    return amb_tok, amb_commit


def capped(cfg, step_in_block: int) -> bool:
    """Threshold rule with a step cap (steps_per_block > 0): the Fast-dLLM
    README's evaluation knobs bound the sampler's steps (diffusion_steps) next
    to the threshold; plainest reading: the step that reaches the cap commits
    every row still masked, so a block never takes more steps than that."""
    return (cfg.commit_mode in (COMMIT_THRESHOLD, COMMIT_EARLY_EXIT) and cfg.steps_per_block > 0
            and step_in_block + 1 >= cfg.steps_per_block)


def ambiguity_flags(conf, gap, masked, tau):
    """Rows whose outcome a correct implementation may decide either way.

    (i) argmax: top-2 logit gap < 1e-2; (ii) threshold: |conf - tau| < 2e-3;
    (iii) forced pick: the two most confident masked rows are within 2e-3 and
    the leader does not clear tau by more than 2e-3.
    """
    amb_tok = masked & (gap < AMBIG_GAP)
    amb_commit = masked & (np.abs(conf - tau) < AMBIG_CONF)
    idx = np.where(masked)[0]
    if len(idx) >= 2:
        c = conf[idx]
        order = np.argsort(-c, kind="stable")
        c0, c1 = c[order[0]], c[order[1]]
        if c0 - c1 < AMBIG_CONF and c0 <= tau + AMBIG_CONF:
            close = idx[np.abs(c - c0) < AMBIG_CONF]
            amb_commit[close] = True
    return amb_tok, amb_commit


# --------------------------------------------------------------------------
# Model
# --------------------------------------------------------------------------
@dataclasses.dataclass
class Config:
    batch: int
    n_layers: int
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    vocab: int
    prompt_len: int
    gen_len: int
    block: int
    tau: float
    mode: int
    window: int
    rope_theta: float
    mask_id: int
    commit_mode: int = COMMIT_THRESHOLD
    steps_per_block: int = 0
    exit_tau: float = 1.0   # COMMIT_EARLY_EXIT: confidence bound of converged rows

    @property
    def seq_len(self):
        return self.prompt_len + self.gen_len


class Weights:
    """fp64 view of the weights, fetched one layer at a time.

    ``wqkv(l)`` [(Hq+2Hkv)D, d], ``wo(l)`` [d, Hq D], ``w_lm()`` [V, d];
    the embedding is tied to w_lm.
    """

    def __init__(self, wqkv: Callable[[int], np.ndarray], wo: Callable[[int], np.ndarray],
                 w_lm: np.ndarray):
        self._wqkv, self._wo, self._w_lm = wqkv, wo, w_lm

    def wqkv(self, layer):
        return np.asarray(self._wqkv(layer), dtype=np.float64)

    def wo(self, layer):
        return np.asarray(self._wo(layer), dtype=np.float64)

    def w_lm(self):
        return self._w_lm

    def embed(self, ids):
        return self._w_lm[np.asarray(ids, dtype=np.int64)]


def forward_rows(cfg: Config, W: Weights, x0: np.ndarray, rows: np.ndarray,
                 keys: Sequence[np.ndarray], kcache: np.ndarray, vcache: np.ndarray,
                 starts: np.ndarray, mirror: bool) -> np.ndarray:
    """Run the layer stack for query rows at positions ``rows`` of every sequence.

    x0 [b, n, d] is the layer-0 input.  Per layer: project the RMS-normalised
    residual to q/k/v (rotary embedding at position p - start on q and k when
    rope_theta > 0), write this layer's k/v of the rows into the caches
    ([L, b, Hkv, S, D]), attend every row to the key positions keys[b], add
    the output projection to the residual.  Returns the final residual
    [b, n, d].  (The projection input is bf16(x) scaled by 1/rms(x) after the
    product, the order in which the CUDA path rounds.)
    """
    b, n, d = x0.shape
    Hq, Hkv, D = cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim
    g = Hq // Hkv
    x = round_f32(x0) if mirror else x0.copy()
    for layer in range(cfg.n_layers):
        xin = round_bf16(x) if mirror else x
        qkv = (xin @ W.wqkv(layer).T) * inv_rms(x)[..., None]   # [b, n, (Hq+2Hkv)D]
        q = qkv[..., :Hq * D].reshape(b, n, Hq, D).transpose(0, 2, 1, 3)
        k = qkv[..., Hq * D:(Hq + Hkv) * D].reshape(b, n, Hkv, D).transpose(0, 2, 1, 3)
        v = qkv[..., (Hq + Hkv) * D:].reshape(b, n, Hkv, D).transpose(0, 2, 1, 3)
        if cfg.rope_theta > 0:
            for bi in range(b):
                pos = rows - starts[bi]
                q[bi] = rope(q[bi], pos, cfg.rope_theta)
                k[bi] = rope(k[bi], pos, cfg.rope_theta)
        if mirror:
            q, k, v = round_bf16(q), round_bf16(k), round_bf16(v)
        kcache[layer][:, :, rows, :] = k
        vcache[layer][:, :, rows, :] = v
        o = np.empty((b, n, Hq, D))
        for bi in range(b):
            kp = keys[bi]
            for h in range(Hq):
                kvh = h // g
                o[bi, :, h, :] = attention(q[bi, h], kcache[layer][bi, kvh][kp],
                                           vcache[layer][bi, kvh][kp])
        if mirror:
            o = round_bf16(o)
        x = x + o.reshape(b, n, Hq * D) @ W.wo(layer).T
        if mirror:
            x = round_f32(x)
    return x


@dataclasses.dataclass
class State:
    """Decode state: tokens [b,S], masked [b,S] bool, caches [L,b,Hkv,S,D]."""
    tokens: np.ndarray
    masked: np.ndarray
    kcache: np.ndarray
    vcache: np.ndarray
    starts: np.ndarray


def new_state(cfg: Config, tokens, masked, starts) -> State:
    S = cfg.seq_len
    shape = (cfg.n_layers, cfg.batch, cfg.n_kv_heads, S, cfg.head_dim)
    return State(np.array(tokens, dtype=np.int64), np.array(masked, dtype=bool),
                 np.zeros(shape), np.zeros(shape), np.asarray(starts, dtype=np.int64))


def prefill(cfg: Config, W: Weights, st: State, mirror: bool = True) -> None:
    """Fill the caches before decoding.

    PREFIX: the prompt attends to itself.  DUAL / DUAL_PRUNED: prompt and all
    masked generated positions (input E[mask_id]) attend to the whole
    sequence, so the suffix cache holds mask-token keys/values.  NONE: nothing.
    Rows before a sequence's start are computed but never read.
    """
    if cfg.mode == MODE_NONE:
        return
    S = cfg.seq_len
    end = cfg.prompt_len if cfg.mode in (MODE_PREFIX, MODE_PREFIX_SUFFIXQ) else S
    rows = np.arange(0, end)
    x0 = W.embed(input_ids(cfg, st, 0, end))
    keys = [np.arange(st.starts[bi], end) for bi in range(cfg.batch)]
    forward_rows(cfg, W, x0, rows, keys, st.kcache, st.vcache, st.starts, mirror)


def input_ids(cfg: Config, st: State, lo: int, hi: int) -> np.ndarray:
    """Token ids fed to the embedding for positions [lo, hi): mask_id where masked."""
    return np.where(st.masked[:, lo:hi], cfg.mask_id, st.tokens[:, lo:hi])


def lm_input(cfg: Config, x: np.ndarray, plants: np.ndarray, masked: np.ndarray, s: int,
             mirror: bool) -> np.ndarray:
    """LM-head input of the block rows: RMSNorm(x) plus the plant where masked."""
    gi = s - cfg.prompt_len
    pl = plants[:, gi:gi + cfg.block, :]
    h = x * inv_rms(x)[..., None] + np.where(masked[..., None], pl, 0.0)
    return round_bf16(h) if mirror else h


@dataclasses.dataclass
class StepResult:
    conf: np.ndarray        # [b, B]   (nan where not masked)
    tok: np.ndarray         # [b, B]   (-1 where not masked)
    gap: np.ndarray         # [b, B]
    commit: np.ndarray      # [b, B] bool
    amb_tok: np.ndarray     # [b, B] bool
    amb_commit: np.ndarray  # [b, B] bool
    hidden: np.ndarray      # [b, B, d] final residual of the block rows


def decode_step(cfg: Config, W: Weights, st: State, plants: np.ndarray, s: int,
                mirror: bool = True, apply: bool = True, step_in_block: int = 0,
                prev_tok: Optional[np.ndarray] = None) -> StepResult:
    """One denoising step of the block at [s, s+B).

    prev_tok [b, B]: the argmax of each row at the previous step of this block
    (-1 where there is none), read by the early-exit rule only.

    The block rows run through every layer (their keys/values overwrite the
    cache at [s, s+B)), the LM head scores the masked rows, and the commit
    rule (threshold, or the fixed top-k budget) commits rows: tokens take the
    argmax, the mask bit goes to 0.
    Without a cache (MODE_NONE) all positions [start, s+B) are recomputed.
    """
    B, b = cfg.block, cfg.batch
    if cfg.mode == MODE_PREFIX_SUFFIXQ:
        # Fast-dLLM's prefix cache read with the suffix as queries: the block
        # and every later position run through the layers each step against
        # [start, S); only the prompt's keys/values come from the cache
        S = cfg.seq_len
        rows = np.arange(s, S)
        x0 = W.embed(input_ids(cfg, st, s, S))
        keys = [np.arange(st.starts[bi], S) for bi in range(b)]
        x = forward_rows(cfg, W, x0, rows, keys, st.kcache, st.vcache, st.starts, mirror)[:, :B]
    elif cfg.mode == MODE_NONE:
        rows = np.arange(0, s + B)
        x0 = W.embed(input_ids(cfg, st, 0, s + B))
        keys = [np.arange(st.starts[bi], s + B) for bi in range(b)]
        shape = (cfg.n_layers, b, cfg.n_kv_heads, cfg.seq_len, cfg.head_dim)
        kc, vc = np.zeros(shape), np.zeros(shape)
        x = forward_rows(cfg, W, x0, rows, keys, kc, vc, st.starts, mirror)[:, s:s + B]
    else:
        rows = np.arange(s, s + B)
        x0 = W.embed(input_ids(cfg, st, s, s + B))
        keys = [key_positions(cfg.mode, s, B, cfg.seq_len, cfg.window, st.starts[bi])
                for bi in range(b)]
        x = forward_rows(cfg, W, x0, rows, keys, st.kcache, st.vcache, st.starts, mirror)
    h = lm_input(cfg, x, plants, st.masked[:, s:s + B], s, mirror)
    conf = np.full((b, B), np.nan)
    tok = np.full((b, B), -1, dtype=np.int64)
    gap = np.full((b, B), np.inf)
    commit = np.zeros((b, B), dtype=bool)
    amb_tok = np.zeros((b, B), dtype=bool)
    amb_commit = np.zeros((b, B), dtype=bool)
    for bi in range(b):
        m = st.masked[bi, s:s + B].copy()
        if m.any():
            c, t, gp = lm_head_confidence(h[bi][m], W.w_lm())
            conf[bi, m], tok[bi, m], gap[bi, m] = c, t, gp
            cm = np.where(m, conf[bi], 0.0)
            if cfg.commit_mode == COMMIT_TOPK:
                k = topk_budget(B, cfg.steps_per_block, int(m.sum()))
                commit[bi] = topk_commit(cm, m, k)
                amb_tok[bi] = m & (gap[bi] < AMBIG_GAP)
                amb_commit[bi] = topk_ambiguity(cm, m, k)
            elif capped(cfg, step_in_block):
                commit[bi] = m.copy()   # the step budget is spent: every masked row commits
                amb_tok[bi] = m & (gap[bi] < AMBIG_GAP)
            elif cfg.commit_mode == COMMIT_EARLY_EXIT:
                pt = (np.full(B, -1, dtype=np.int64) if prev_tok is None
                      else np.asarray(prev_tok[bi], dtype=np.int64))
                commit[bi] = early_exit_commit(cm, tok[bi], pt, m, cfg.tau, cfg.exit_tau)
                amb_tok[bi], amb_commit[bi] = early_exit_ambiguity(cm, gap[bi], tok[bi], pt, m,
                                                                   cfg.tau, cfg.exit_tau)
            else:
                commit[bi] = threshold_commit(cm, m, cfg.tau)
                amb_tok[bi], amb_commit[bi] = ambiguity_flags(cm, gap[bi], m, cfg.tau)
        if apply:
            idx = np.where(commit[bi])[0]
            st.tokens[bi, s + idx] = tok[bi, idx]
            st.masked[bi, s + idx] = False
    return StepResult(conf, tok, gap, commit, amb_tok, amb_commit, x)


def refresh_block(cfg: Config, W: Weights, st: State, s: int, mirror: bool = True) -> None:
    """Recompute the keys/values of a finished block from its committed tokens.

    The block rows (input E[token]) run through every layer against the same
    key set as a decode step; no LM head.  Only the block's cache slots change.
    """
    if cfg.mode == MODE_NONE:
        return
    B = cfg.block
    rows = np.arange(s, s + B)
    x0 = W.embed(st.tokens[:, s:s + B])
    keys = [key_positions(cfg.mode, s, B, cfg.seq_len, cfg.window, st.starts[bi])
            for bi in range(cfg.batch)]
    forward_rows(cfg, W, x0, rows, keys, st.kcache, st.vcache, st.starts, mirror)


@dataclasses.dataclass
class DecodeTrace:
    tokens: np.ndarray
    steps_per_block: list
    steps: list             # list of (block_start, StepResult)


def decode(cfg: Config, W: Weights, tokens, masked, starts, plants,
           mirror: bool = True, max_steps: Optional[int] = None) -> DecodeTrace:
    """Whole generation: prefill, then block by block until no masked rows.

    Blocks advance together across the batch; a finished sequence idles until
    every sequence's block is done, then the block is refreshed.
    """
    st = new_state(cfg, tokens, masked, starts)
    prefill(cfg, W, st, mirror)
    B = cfg.block
    steps_per_block, trace = [], []
    for s in range(cfg.prompt_len, cfg.seq_len, B):
        n = 0
        prev = np.full((cfg.batch, B), -1, dtype=np.int64)   # argmax at the previous step
        while st.masked[:, s:s + B].any():
            if max_steps is not None and n >= max_steps:
                break
            r = decode_step(cfg, W, st, plants, s, mirror, step_in_block=n, prev_tok=prev)
            trace.append((s, r))
            prev = r.tok.copy()
            n += 1
        steps_per_block.append(n)
        refresh_block(cfg, W, st, s, mirror)
    return DecodeTrace(st.tokens.copy(), steps_per_block, trace)
