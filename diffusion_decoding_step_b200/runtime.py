"""Device buffers for one decode workload, held in torch tensors, driven
through the C ABI.  PyTorch only allocates memory and provides the stream;
all arithmetic of the path runs in libdllm.so.
"""
from __future__ import annotations

import ctypes as C
from typing import Optional

import torch

from . import abi
from .workload import Workload, Weights, Plants


def make_config(w: Workload) -> abi.dllm_config:
    return abi.dllm_config(
        batch=w.batch, n_layers=w.n_layers, hidden=w.hidden, n_q_heads=w.n_q_heads,
        n_kv_heads=w.n_kv_heads, head_dim=w.head_dim, vocab=w.vocab, prompt_len=w.prompt_len,
        gen_len=w.gen_len, block=w.block, window=w.window, mask_id=w.mask_id, tau=w.tau,
        rope_theta=w.rope_theta, mode=w.mode,
        weight_format=abi.DLLM_W_F32_SPLIT if w.weight_f32 else abi.DLLM_W_BF16,
        commit_mode=w.commit_mode, steps_per_block=w.steps_per_block, exit_tau=w.exit_tau)


def workspace_bytes(w: Workload) -> int:
    n = C.c_size_t(0)
    abi.check(abi.dllm_workspace_size(C.byref(make_config(w)), C.byref(n)), "workspace_size")
    return int(n.value)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else C.c_void_p(t.data_ptr())


class Decoder:
    """All device state of one workload: weights, tokens/mask, caches, workspace."""

    def __init__(self, w: Workload, weights: Weights, tokens: torch.Tensor, masked: torch.Tensor,
                 seq_start: torch.Tensor, plants: Plants, device: str = "cuda"):
        self.w = w
        self.device = torch.device(device)
        self.cfg = make_config(w)
        self.stream = torch.cuda.current_stream(self.device)
        sh = self._sh = C.c_void_p(self.stream.cuda_stream)
        dev = self.device
        if w.weight_f32:
            self.embed = weights.w_lm.to(dev, torch.float32).contiguous()
            self.wqkv = self._split(weights.wqkv)
            self.wo = self._split(weights.wo)
            self.w_lm = self._split(weights.w_lm)
        else:
            self.wqkv = weights.wqkv.to(dev, torch.bfloat16).contiguous()
            self.wo = weights.wo.to(dev, torch.bfloat16).contiguous()
            self.w_lm = weights.w_lm.to(dev, torch.bfloat16).contiguous()
            self.embed = self.w_lm
        self.weights_c = abi.dllm_weights(_ptr(self.wqkv), _ptr(self.wo), _ptr(self.w_lm),
                                          _ptr(self.embed))
        self.tokens0 = tokens.to(dev, torch.int32).contiguous()
        self.masked0 = masked.to(dev, torch.uint8).contiguous()
        self.tokens = self.tokens0.clone()
        self.masked = self.masked0.clone()
        self.seq_start = seq_start.to(dev, torch.int32).contiguous()
        self.plants = plants.h.to(dev, torch.bfloat16).contiguous()
        cache_shape = (w.n_layers, w.batch, w.n_kv_heads, w.seq_len, w.head_dim)
        self.k_cache = torch.zeros(cache_shape, dtype=torch.bfloat16, device=dev)
        self.v_cache = torch.zeros(cache_shape, dtype=torch.bfloat16, device=dev)
        self.state_c = abi.dllm_state(_ptr(self.tokens), _ptr(self.masked), _ptr(self.seq_start),
                                      _ptr(self.k_cache), _ptr(self.v_cache), _ptr(self.plants))
        self.tau_seq = None
        self.ws_bytes = workspace_bytes(w)
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=dev)
        abi.check(abi.dllm_workspace_init(C.byref(self.cfg), _ptr(self.ws), self.ws_bytes, sh),
                  "workspace_init")

    def _split(self, t: torch.Tensor) -> torch.Tensor:
        src = t.to(self.device, torch.float32).contiguous()
        rows = src.numel() // src.shape[-1]
        cols = src.shape[-1]
        dst = torch.empty(src.shape[:-1] + (2 * cols,), dtype=torch.bfloat16, device=self.device)
        abi.check(abi.dllm_split_f32_weights(_ptr(src), _ptr(dst), rows, cols, self._sh), "split")
        return dst

    # ------------------------------------------------------------------ calls
    @property
    def cfg_p(self):
        return C.byref(self.cfg)

    def reset(self):
        self.tokens.copy_(self.tokens0)
        self.masked.copy_(self.masked0)

    def set_tau(self, tau) -> None:
        """Per-sequence thresholds (a list of b floats), or None for the
        configuration's single tau.  The steps read them from device memory."""
        if tau is None:
            self.tau_seq = None
            self.state_c.tau = None
        else:
            vals = [float(t) for t in tau]
            if len(vals) != self.w.batch:
                raise ValueError(f"set_tau: {len(vals)} thresholds for {self.w.batch} sequences")
            self.tau_seq = torch.tensor(vals, dtype=torch.float32, device=self.device)
            self.state_c.tau = _ptr(self.tau_seq)

    def prefill(self):
        abi.check(abi.dllm_prefill(self.cfg_p, C.byref(self.weights_c), C.byref(self.state_c),
                                   _ptr(self.ws), self.ws_bytes, self._sh), "prefill")

    def step(self, block_start: int):
        abi.check(abi.dllm_decode_step(self.cfg_p, C.byref(self.weights_c),
                                       C.byref(self.state_c), block_start, _ptr(self.ws),
                                       self.ws_bytes, self._sh), "decode_step")

    def refresh(self, block_start: int):
        abi.check(abi.dllm_kv_cache_refresh(self.cfg_p, C.byref(self.weights_c),
                                            C.byref(self.state_c), block_start, _ptr(self.ws),
                                            self.ws_bytes, self._sh), "refresh")

    def decode_block(self, block_start: int, max_steps: int = 0) -> int:
        n = C.c_int32(0)
        abi.check(abi.dllm_decode_block(self.cfg_p, C.byref(self.weights_c),
                                        C.byref(self.state_c), block_start, max_steps,
                                        C.byref(n), _ptr(self.ws), self.ws_bytes, self._sh),
                  "decode_block")
        return int(n.value)

    def generate(self) -> list:
        """Prefill, then every block to completion; returns steps per block."""
        self.prefill()
        steps = []
        for s in range(self.w.prompt_len, self.w.seq_len, self.w.block):
            steps.append(self.decode_block(s))
        return steps

    def generate_per_sequence(self) -> int:
        """Prefill, then every sequence decoded at its own block position
        (dllm_decode_all); returns the number of passes."""
        self.prefill()
        return self.decode_all()

    def decode_all(self) -> int:
        """Every sequence decoded at its own block position, after a prefill;
        returns the number of passes."""
        n = C.c_int32(0)
        abi.check(abi.dllm_decode_all(self.cfg_p, C.byref(self.weights_c), C.byref(self.state_c),
                                      C.byref(n), _ptr(self.ws), self.ws_bytes, self._sh),
                  "decode_all")
        return int(n.value)

    def _outputs(self):
        ptrs = [C.c_void_p() for _ in range(6)]
        abi.check(abi.dllm_step_outputs(self.cfg_p, _ptr(self.ws), self.ws_bytes,
                                        *[C.byref(p) for p in ptrs]), "step_outputs")
        return [p.value - self.ws.data_ptr() for p in ptrs]

    def step_outputs(self):
        """(conf, tok, gap, commit) of the last step, each [b][B], as views."""
        n = self.w.batch * self.w.block
        out = []
        for off, dt, size in zip(self._outputs()[:4],
                                 (torch.float32, torch.int32, torch.float32, torch.uint8),
                                 (4, 4, 4, 1)):
            out.append(self.ws[off:off + n * size].view(dt).view(self.w.batch, self.w.block))
        return tuple(out)

    def block_state(self):
        """(block_done, refresh_list) of the last step's commit, each [b] int32
        views: 1 when the sequence's block has no masked row left, and the
        block start whose keys/values the commit made due for a refresh (-1:
        none)."""
        b = self.w.batch
        return tuple(self.ws[off:off + 4 * b].view(torch.int32) for off in self._outputs()[4:])

    def device_status(self) -> int:
        code = C.c_int32(0)
        abi.check(abi.dllm_device_status(_ptr(self.ws), C.byref(code), self._sh), "status")
        return int(code.value)
