"""Per-CTA phase trace of the projection GEMMs in one decode step (a profiling
tool; needs a B200).

The tool copies the CUDA sources into a temporary directory and inserts
`globaltimer` stamps into gemm_kernel there. It builds that copy as a separate
library, runs one denoising step of a workload, and prints the mean per-CTA
time between phases. The phases are:
- the programmatic-dependency wait;
- the first MMA and the last one;
- the accumulator being ready;
- the split-K sends, the receive and the partial sums;
- the epilogue and the kernel's end.

The Q/K/V projection, the O-projection and the LM head are each reported as a
mean over the layers. The library the package loads is not touched.

    python -m diffusion_decoding_step_b200.phase_trace llada8b_dual

Each stamp is one 64-bit global store from one designated thread.
"""
from __future__ import annotations

import ctypes as C
import os
import shutil
import subprocess
import sys
import tempfile

import numpy as np

from . import build as _build

SLOTS, CTAS, PHASES = 256, 320, 16
# phase index -> name; 14 holds the launch's split count instead of a time
NAMES = {0: "start", 1: "dep", 2: "mma0", 3: "last_mma", 4: "acc", 5: "sync", 6: "sent",
         7: "recv", 8: "summed", 9: "epilogue", 10: "cluster_end", 11: "launched",
         12: "cl_wait", 13: "arrived", 15: "end"}

_STAMP = ('#define TS(k) do { unsigned long long t_; asm volatile("mov.u64 %0, %%globaltimer;" '
          ': "=l"(t_)); g_gt[p.trace_slot & 255][blockIdx.x < 320 ? blockIdx.x : 319][k] = t_; '
          '} while (0)\n')

# (anchor, replacement) pairs; each anchor must occur exactly once
_GEMM = [
    ("namespace dllm {\n\ntemplate <int NT, int EPI>\nstruct GemmCfg",
     "namespace dllm {\n__device__ unsigned long long g_gt[256][320][16];\nstatic int g_gslot = 0;\n"
     'extern "C" int dllm_gt_read(unsigned long long* h) '
     "{ return (int)cudaMemcpyFromSymbol(h, g_gt, sizeof(g_gt)); }\n"
     'extern "C" int dllm_gt_reset() { static unsigned long long z[256 * 320 * 16]; '
     "return (int)cudaMemcpyToSymbol(g_gt, z, sizeof(z)); }\n"
     'extern "C" int dllm_gt_slot() { return g_gslot; }\n' + _STAMP +
     "\ntemplate <int NT, int EPI>\nstruct GemmCfg"),
    ("  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;\n  // Split K is reduced",
     "  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;\n"
     "  if (threadIdx.x == 0) { TS(0); "
     "g_gt[p.trace_slot & 255][blockIdx.x < 320 ? blockIdx.x : 319][14] = p.splits; }\n"
     "  // Split K is reduced"),
    ("      grid_dep_wait();\n      mbar_arrive(dep_bar);",
     "      grid_dep_wait();\n      TS(1);\n      mbar_arrive(dep_bar);"),
    ("          tc_fence_after();\n          const uint32_t wa = smem_u32(w_st + s * C::kWBytes);",
     "          tc_fence_after();\n          if (it == 0) TS(2);\n"
     "          const uint32_t wa = smem_u32(w_st + s * C::kWBytes);"),
    ("        if (!ok) break;\n        umma_commit(&tfull[acc]);",
     "        if (!ok) break;\n        umma_commit(&tfull[acc]);\n        TS(3);"),
    ("      if (named_bar_or(1, 128, bad)) {\n        flags[0] = 1;\n        break;\n      }\n"
     "      tc_fence_after();",
     "      if (named_bar_or(1, 128, bad)) {\n        flags[0] = 1;\n        break;\n      }\n"
     "      if (et == 0) TS(4);\n      tc_fence_after();"),
    ("  __syncthreads();\n  // Every mainloop of this CTA is done",
     "  __syncthreads();\n  if (threadIdx.x == 0) TS(5);\n  // Every mainloop of this CTA is done"),
    ("  grid_dep_launch();\n  if constexpr (kClusterSplit) {\n    if (p.splits > 1) {",
     "  grid_dep_launch();\n  if (threadIdx.x == 64) TS(11);\n"
     "  if constexpr (kClusterSplit) {\n    if (p.splits > 1) {"),
    ("      cluster_wait();\n      if (p.recv_in_ring) {",
     "      cluster_wait();\n      if (threadIdx.x == 64) TS(12);\n      if (p.recv_in_ring) {"),
    ("      if (epi && rank < NT / 16) {\n        const bool got = mbar_wait_cluster(red_bar, 0, "
     "p.status);\n        cluster_arrive_relaxed();",
     "      if (epi && et == 0) TS(6);\n      if (epi && rank < NT / 16) {\n"
     "        const bool got = mbar_wait_cluster(red_bar, 0, p.status);\n"
     "        if (et == 0) TS(7);\n        cluster_arrive_relaxed();\n        if (et == 0) TS(13);"),
    ("            epi_chunk<NT, kEpi>(p, m, n, q * 16, wl, et, v, xpre[lq], stage, run);\n"
     "          }",
     "            if (et == 0) TS(8);\n"
     "            epi_chunk<NT, kEpi>(p, m, n, q * 16, wl, et, v, xpre[lq], stage, run);\n"
     "            if (et == 0) TS(9);\n          }"),
    ("      } else {\n        cluster_arrive_relaxed();\n      }\n      cluster_wait();\n    }\n  }",
     "      } else {\n        cluster_arrive_relaxed();\n      }\n      cluster_wait();\n"
     "      if (threadIdx.x == 0) TS(10);\n    }\n  }"),
    ("    tmem_dealloc(*tmem_slot, C::kTmemCols);\n  }\n}",
     "    tmem_dealloc(*tmem_slot, C::kTmemCols);\n    if (lane == 0) TS(15);\n  }\n}"),
    ("cudaError_t launch_gemm(int epi, int nt, const CUtensorMap& wmap, const CUtensorMap& xmap,\n"
     "                        const GemmParams& p, int grid, bool pdl, cudaStream_t s) {\n"
     "  switch (epi) {",
     "cudaError_t launch_gemm(int epi, int nt, const CUtensorMap& wmap, const CUtensorMap& xmap,\n"
     "                        const GemmParams& p0, int grid, bool pdl, cudaStream_t s) {\n"
     "  GemmParams p = p0;\n  p.trace_slot = g_gslot++;\n  switch (epi) {"),
]
_KERNELS = [("  L2Prefetch pf;\n};\n\nstruct AttnParams {",
             "  L2Prefetch pf;\n  int trace_slot;\n};\n\nstruct AttnParams {")]


def _patch(path: str, pairs) -> None:
    with open(path) as f:
        s = f.read()
    for a, b in pairs:
        if s.count(a) != 1:
            raise RuntimeError(f"{os.path.basename(path)}: anchor not found once: {a[:60]!r}")
        s = s.replace(a, b)
    with open(path, "w") as f:
        f.write(s)


def build_traced(out_dir: str) -> str:
    """Build the stamped copy of the library into out_dir; returns its path."""
    src = os.path.join(out_dir, "src")
    csrc = os.path.join(src, "diffusion_decoding_step_b200", "csrc")
    os.makedirs(csrc)
    os.makedirs(os.path.join(src, "include"))
    for f in os.listdir(_build.CSRC):
        shutil.copy(os.path.join(_build.CSRC, f), csrc)
    shutil.copy(os.path.join(_build.HERE, "..", "include", "dllm.h"), os.path.join(src, "include"))
    _patch(os.path.join(csrc, "kernels.cuh"), _KERNELS)
    _patch(os.path.join(csrc, "gemm.cu"), _GEMM)
    lib = os.path.join(out_dir, "libdllm_phase_trace.so")
    cmd = [_build.nvcc(), *_build.FLAGS] + [os.path.join(csrc, f) for f in _build.SOURCES]
    subprocess.run(cmd + ["-o", lib], check=True)
    return lib


def _summarise(t: np.ndarray, kinds: list, s0: int) -> dict:
    """Per kind: mean over its launches of per-CTA phase gaps (µs)."""
    out: dict = {}
    for i, kind in enumerate(kinds):
        a = t[(s0 + i) % SLOTS]
        a = a[a[:, 0] > 0]
        us = lambda x, y: (a[:, y] - a[:, x]) / 1e3  # noqa: E731
        rows = {"CTAs": float(a.shape[0]),
                "dep -> first MMA (last CTA)": (a[:, 2].max() - a[:, 1].max()) / 1e3,
                "first MMA -> last MMA (grid)": (a[:, 3].max() - a[:, 2].min()) / 1e3,
                "last-MMA spread over CTAs": (a[:, 3].max() - a[:, 3].min()) / 1e3,
                "last MMA -> accumulator ready": us(3, 4).mean(),
                "accumulator -> tail start": us(4, 5).mean(),
                "last MMA -> kernel end (grid)": (a[:, 15].max() - a[:, 3].max()) / 1e3}
        if (a[:, 6] > 0).all():
            rows["tail start -> sends issued"] = us(5, 6).mean()
            sp = int(a[0, 14])
            waits = []
            for c in range(0, a.shape[0], max(sp, 1)):
                cl = a[c:c + sp]
                owners = cl[cl[:, 7] > 0]
                waits += list((owners[:, 7] - cl[:, 6].max()) / 1e3)
            own = a[a[:, 7] > 0]
            rows["split count"] = float(sp)
            if waits:
                rows["last peer's send -> received"] = float(np.mean(waits))
                rows["received -> partials summed"] = float(((own[:, 8] - own[:, 7]) / 1e3).mean())
                rows["partials summed -> epilogue done"] = float(
                    ((own[:, 9] - own[:, 8]) / 1e3).mean())
        for k, v in rows.items():
            out.setdefault(kind, {}).setdefault(k, []).append(float(v))
    return {k: {r: float(np.mean(v[1:-1] if len(v) > 3 else v)) for r, v in d.items()}
            for k, d in out.items()}


def run(workload: str) -> dict:
    import torch

    from . import abi
    from . import workload as wl
    tmp = tempfile.mkdtemp(prefix="dllm_phase_trace_")
    try:
        abi.LIB_PATH = build_traced(tmp)
        lib = abi.lib()
        from .runtime import Decoder
        w = wl.WORKLOADS[workload]
        weights = wl.make_weights(w, device="cuda")
        tokens, masked = wl.make_tokens(w)
        dec = Decoder(w, weights, tokens, masked, wl.seq_starts(w),
                      wl.make_plants(w, weights.w_lm))
        dec.prefill()
        torch.cuda.synchronize()
        s0 = lib.dllm_gt_slot()
        for _ in range(3):
            dec.step(w.prompt_len)
        torch.cuda.synchronize()
        buf = np.zeros(SLOTS * CTAS * PHASES, dtype=np.uint64)
        lib.dllm_gt_reset()
        dec.step(w.prompt_len)
        torch.cuda.synchronize()
        lib.dllm_gt_read(C.c_void_p(buf.ctypes.data))
        if dec.device_status() != 0:
            raise RuntimeError("device status word set during the traced step")
        kinds = [k for _ in range(w.n_layers) for k in ("qkv_proj", "o_proj")] + ["lm_head"]
        return _summarise(buf.reshape(SLOTS, CTAS, PHASES).astype(np.float64), kinds, s0)
    finally:
        shutil.rmtree(tmp, ignore_errors=True)


def main() -> None:
    name = sys.argv[1] if len(sys.argv) > 1 else "llada8b_dual"
    for kind, rows in run(name).items():
        print(f"{name} {kind}")
        for k, v in rows.items():
            print(f"  {k:36s} {v:9.2f}")


if __name__ == "__main__":
    main()
