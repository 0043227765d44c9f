"""Seeded synthetic workloads for the block-decode step.

This module only draws random numbers and lays them out.  It holds none of
the decode method's arithmetic, so both the CUDA path and the CPU oracle can
take their inputs from it.

Shapes follow the decode setups the pages use: LLaDA-8B-like and
Dream-7B / Qwen2.5-7B-like backbones with gen length 256/512, block 32 and
tau 0.9 (Fast-dLLM README, "Quick Start"; Streaming-dLLM README, result
tables), plus a tiny single-layer case and a long-context case with a pruned
suffix window (Streaming-dLLM README, figure "approximated suffix pruning").
No benchmark item, prompt or trained weight is used: token ids are uniform
random and weights are N(0, 0.02^2).

Planted hidden states.  A masked block row's LM-head input gets the offset
``h = a * W_lm[t] / ||W_lm[t]||^2 + n`` with ``n ~ N(0, (sigma_w sqrt(d))^-2 I)``
added to its final normalised hidden state (its layer-0 input is the mask
token's embedding, like any masked position).
This puts the target logit at about ``a`` above logits that are N(0, 1), so
confidences spread from ~1/V to ~1 as ``a`` goes from 0 to its maximum.
``t``, ``a`` and ``n`` are drawn once per (sequence, generated position).

Seeds: weights 0, prompts 1, plants 2, prompt lengths 3.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

MODE_NONE, MODE_PREFIX, MODE_DUAL, MODE_DUAL_PRUNED = 0, 1, 2, 3
MODE_PREFIX_SUFFIXQ = 4    # prefix cache, block and suffix recomputed as queries each step
# conf > tau; a fixed top-k budget per step; conf > tau or, for a row whose
# argmax repeats from the previous step of the block, conf > exit_tau
COMMIT_THRESHOLD, COMMIT_TOPK, COMMIT_EARLY_EXIT = 0, 1, 2
MODE_NAMES = {MODE_NONE: "none", MODE_PREFIX: "prefix", MODE_DUAL: "dual",
              MODE_DUAL_PRUNED: "dual_pruned", MODE_PREFIX_SUFFIXQ: "prefix_suffixq"}

SIGMA_W = 0.02
SEED_WEIGHTS, SEED_PROMPTS, SEED_PLANTS, SEED_LENGTHS = 0, 1, 2, 3


@dataclasses.dataclass
class Workload:
    """Shape and policy of one decode workload (sizes only, no data)."""
    name: str
    batch: int
    n_layers: int
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    vocab: int
    prompt_len: int            # longest prompt; shorter prompts are left-padded to it
    gen_len: int
    block: int
    tau: float = 0.9
    mode: int = MODE_DUAL
    window: int = 0            # suffix window for MODE_DUAL_PRUNED
    rope_theta: float = 0.0    # 0 = no rotary embedding
    mask_id: int = -1          # -1 = vocab - 1
    weight_f32: bool = False   # fp32 weights (tiny case) instead of bf16
    plant_a_max: float = 20.0
    prompt_len_min: Optional[int] = None  # ragged prompts: U[min, prompt_len]
    commit_mode: int = COMMIT_THRESHOLD
    steps_per_block: int = 0   # COMMIT_TOPK: a block is decoded in exactly this many steps
    exit_tau: float = 1.0      # COMMIT_EARLY_EXIT: confidence bound of rows whose argmax repeats

    def __post_init__(self):
        if self.mask_id < 0:
            self.mask_id = self.vocab - 1

    @property
    def seq_len(self) -> int:
        return self.prompt_len + self.gen_len

    @property
    def qkv_rows(self) -> int:
        return (self.n_q_heads + 2 * self.n_kv_heads) * self.head_dim

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workload shapes.  Index 1 is the LLaDA-8B-shaped DualCache step.
WORKLOADS = {
    "tiny": Workload("tiny", batch=1, n_layers=1, hidden=128, n_q_heads=4, n_kv_heads=4,
                     head_dim=32, vocab=1024, prompt_len=64, gen_len=32, block=8,
                     mode=MODE_PREFIX, weight_f32=True, plant_a_max=12.0, mask_id=1023),
    "llada8b_dual": Workload("llada8b_dual", batch=1, n_layers=32, hidden=4096, n_q_heads=32,
                             n_kv_heads=32, head_dim=128, vocab=126464, prompt_len=256,
                             gen_len=256, block=32, mode=MODE_DUAL),
    "dream7b_prefix": Workload("dream7b_prefix", batch=1, n_layers=28, hidden=3584, n_q_heads=28,
                               n_kv_heads=4, head_dim=128, vocab=152064, prompt_len=512,
                               gen_len=512, block=32, mode=MODE_PREFIX, rope_theta=1e6),
    "llada8b_dual_b16": Workload("llada8b_dual_b16", batch=16, n_layers=32, hidden=4096,
                                 n_q_heads=32, n_kv_heads=32, head_dim=128, vocab=126464,
                                 prompt_len=1024, prompt_len_min=512, gen_len=256, block=32,
                                 mode=MODE_DUAL),
    "qwen7b_long_pruned": Workload("qwen7b_long_pruned", batch=4, n_layers=28, hidden=3584,
                                   n_q_heads=28, n_kv_heads=4, head_dim=128, vocab=152064,
                                   prompt_len=8192, gen_len=1024, block=64,
                                   mode=MODE_DUAL_PRUNED, window=64, rope_theta=1e6),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def prompt_lengths(w: Workload) -> torch.Tensor:
    """Per-sequence prompt lengths (int64, CPU)."""
    if w.prompt_len_min is None:
        return torch.full((w.batch,), w.prompt_len, dtype=torch.int64)
    g = _gen(SEED_LENGTHS, "cpu")
    return torch.randint(w.prompt_len_min, w.prompt_len + 1, (w.batch,), generator=g)


def seq_starts(w: Workload) -> torch.Tensor:
    """First valid position of each sequence (left padding), int32 CPU."""
    return (w.prompt_len - prompt_lengths(w)).to(torch.int32)


def make_tokens(w: Workload) -> tuple[torch.Tensor, torch.Tensor]:
    """Initial token ids int32 [b][S] and mask bitmap uint8 [b][S] (CPU).

    Prompt ids are uniform over the vocabulary; generated positions hold
    mask_id and are marked masked; left padding holds 0 and is not masked.
    """
    S = w.seq_len
    g = _gen(SEED_PROMPTS, "cpu")
    ids = torch.randint(0, w.vocab, (w.batch, w.prompt_len), generator=g, dtype=torch.int64)
    tokens = torch.zeros((w.batch, S), dtype=torch.int32)
    masked = torch.zeros((w.batch, S), dtype=torch.uint8)
    starts = seq_starts(w)
    for b in range(w.batch):
        st = int(starts[b])
        tokens[b, st:w.prompt_len] = ids[b, st:].to(torch.int32)
    tokens[:, w.prompt_len:] = w.mask_id
    masked[:, w.prompt_len:] = 1
    return tokens, masked


@dataclasses.dataclass
class Weights:
    """Model weights in the library's layout.

    wqkv [L][(Hq+2Hkv)*D][d]  rows: q heads, then k heads, then v heads
    wo   [L][d][Hq*D]
    w_lm [V][d]               the embedding is tied to it
    """
    wqkv: torch.Tensor
    wo: torch.Tensor
    w_lm: torch.Tensor


def make_weights(w: Workload, device="cpu", layers: Optional[int] = None) -> Weights:
    """N(0, 0.02^2) weights; bf16 unless ``w.weight_f32``.  Drawn layer by layer."""
    L = w.n_layers if layers is None else layers
    g = _gen(SEED_WEIGHTS, device)
    dt = torch.float32 if w.weight_f32 else torch.bfloat16
    wqkv = torch.empty((L, w.qkv_rows, w.hidden), dtype=dt, device=device)
    wo = torch.empty((L, w.hidden, w.n_q_heads * w.head_dim), dtype=dt, device=device)
    for layer in range(L):
        wqkv[layer] = (torch.randn(wqkv.shape[1:], generator=g, device=device) * SIGMA_W).to(dt)
        wo[layer] = (torch.randn(wo.shape[1:], generator=g, device=device) * SIGMA_W).to(dt)
    w_lm = torch.empty((w.vocab, w.hidden), dtype=dt, device=device)
    chunk = 8192
    for v0 in range(0, w.vocab, chunk):
        v1 = min(w.vocab, v0 + chunk)
        w_lm[v0:v1] = (torch.randn((v1 - v0, w.hidden), generator=g, device=device)
                       * SIGMA_W).to(dt)
    return Weights(wqkv, wo, w_lm)


@dataclasses.dataclass
class Plants:
    """Planted LM-head input offsets of generated positions (added to the final
    normalised hidden state of a masked row).

    h [b][G][d] bf16 and the draws behind it: target t [b][G] and scale a [b][G].
    """
    h: torch.Tensor
    t: torch.Tensor
    a: torch.Tensor


def make_plants(w: Workload, w_lm: torch.Tensor, a_override: Optional[float] = None,
                noise: bool = True, seed: Optional[int] = None) -> Plants:
    """Draw the planted hidden states on ``w_lm``'s device (seed: another draw
    of the same distribution; default SEED_PLANTS)."""
    dev = w_lm.device
    g = _gen(SEED_PLANTS if seed is None else seed, dev)
    G = w.gen_len
    t = torch.randint(0, w.vocab, (w.batch, G), generator=g, device=dev)
    a = torch.rand((w.batch, G), generator=g, device=dev, dtype=torch.float32) * w.plant_a_max
    if a_override is not None:
        a = torch.full_like(a, float(a_override))
    n = torch.randn((w.batch, G, w.hidden), generator=g, device=dev, dtype=torch.float32)
    sigma_n = 1.0 / (SIGMA_W * (w.hidden ** 0.5))
    rows = w_lm[t.reshape(-1)].float().reshape(w.batch, G, w.hidden)
    sq = (rows * rows).sum(-1, keepdim=True)
    h = a.unsqueeze(-1) * rows / sq
    if noise:
        h = h + n * sigma_n
    return Plants(h.to(torch.bfloat16), t.to(torch.int32), a)
