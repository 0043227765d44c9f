"""Turn a seeded workload into the oracle's fp64 inputs (test helper)."""
from __future__ import annotations

import numpy as np
import torch

from oracle import dllm_oracle as O
from diffusion_decoding_step_b200 import workload as wl


def oracle_config(w: wl.Workload) -> O.Config:
    return O.Config(batch=w.batch, n_layers=w.n_layers, hidden=w.hidden,
                    n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, head_dim=w.head_dim,
                    vocab=w.vocab, prompt_len=w.prompt_len, gen_len=w.gen_len,
                    block=w.block, tau=w.tau, mode=w.mode, window=w.window,
                    rope_theta=w.rope_theta, mask_id=w.mask_id, commit_mode=w.commit_mode,
                    steps_per_block=w.steps_per_block, exit_tau=w.exit_tau)


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def oracle_weights(W: wl.Weights) -> O.Weights:
    """fp64 weights; per-layer matrices are converted when the oracle asks."""
    return O.Weights(lambda l: to64(W.wqkv[l]), lambda l: to64(W.wo[l]), to64(W.w_lm))


class Case:
    """All inputs of one workload on the CPU, plus the oracle's views of them."""

    def __init__(self, w: wl.Workload, device="cpu", a_override=None, noise=True,
                 plant_seed=None):
        self.w = w
        self.weights = wl.make_weights(w, device=device)
        self.tokens, self.masked = wl.make_tokens(w)
        self.starts = wl.seq_starts(w)
        self.plants = wl.make_plants(w, self.weights.w_lm, a_override=a_override, noise=noise,
                                     seed=plant_seed)
        self.cfg = oracle_config(w)
        self.W = oracle_weights(self.weights)
        self.plants64 = to64(self.plants.h)

    def decode(self, mirror=True, **kw):
        return O.decode(self.cfg, self.W, self.tokens.numpy(), self.masked.numpy().astype(bool),
                        self.starts.numpy(), self.plants64, mirror=mirror, **kw)
