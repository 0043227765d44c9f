"""The C-ABI library loads and exports what include/dllm.h declares (no GPU).

Only host-side entry points that launch nothing are called here: the
workspace-size query and argument validation.
"""
import ctypes as C
import os
import re

import pytest

from diffusion_decoding_step_b200 import abi, build
from diffusion_decoding_step_b200 import workload as wl
from diffusion_decoding_step_b200.runtime import make_config

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return abi.lib()


def header_functions():
    text = open(os.path.join(ROOT, "include", "dllm.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dllm_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = header_functions()
    for must in ("dllm_block_attn", "dllm_lmhead_confidence", "dllm_threshold_commit",
                 "dllm_kv_cache_refresh", "dllm_decode_block"):
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    for name in header_functions():
        assert hasattr(lib, name), name
        assert name in abi.SIGNATURES, f"binding lacks {name}"


def test_debug_build_exports_every_declared_symbol():
    """The DLLM_DEBUG build (range checks of device-side row positions) is the
    same library: it builds and exports the whole ABI."""
    dbg = C.CDLL(build.build(debug=True))
    for name in header_functions():
        assert hasattr(dbg, name), name


def test_status_bits_match_the_header():
    text = open(os.path.join(ROOT, "include", "dllm.h")).read()
    bits = dict(re.findall(r"#define (DLLM_DEVICE_[A-Z_]+) (\d+)", text))
    assert set(bits) == {"DLLM_DEVICE_TIMEOUT", "DLLM_DEVICE_BAD_TOKEN", "DLLM_DEVICE_INDEX"}
    for name, value in bits.items():
        assert getattr(abi, name) == int(value), name
    assert len({int(v) for v in bits.values()}) == len(bits)  # distinct bits


@pytest.mark.parametrize("name", list(wl.WORKLOADS))
def test_workspace_size_for_every_workload(lib, name):
    n = C.c_size_t(0)
    assert abi.dllm_workspace_size(C.byref(make_config(wl.WORKLOADS[name])), C.byref(n)) == 0
    assert n.value > 0 and n.value % 256 == 0


def _status(w: wl.Workload):
    n = C.c_size_t(0)
    return abi.dllm_workspace_size(C.byref(make_config(w)), C.byref(n))


def test_rejects_bad_configs(lib):
    base = wl.WORKLOADS["tiny"]
    assert _status(base) == abi.DLLM_OK
    assert _status(base.replace(head_dim=64)) == abi.DLLM_ERR_UNSUPPORTED
    assert _status(base.replace(n_kv_heads=3)) == abi.DLLM_ERR_INVALID
    assert _status(base.replace(gen_len=30)) == abi.DLLM_ERR_INVALID
    assert _status(base.replace(hidden=96)) == abi.DLLM_ERR_UNSUPPORTED
    assert _status(base.replace(block=128, gen_len=128)) == abi.DLLM_ERR_UNSUPPORTED
    assert _status(base.replace(vocab=1000, mask_id=5)) == abi.DLLM_ERR_UNSUPPORTED
    assert _status(base.replace(mask_id=2000)) == abi.DLLM_ERR_INVALID
    assert abi.dllm_workspace_size(None, None) == abi.DLLM_ERR_INVALID
    # rope_theta and tau
    assert _status(base.replace(rope_theta=float("nan"))) == abi.DLLM_ERR_INVALID
    assert _status(base.replace(rope_theta=float("inf"))) == abi.DLLM_ERR_INVALID
    assert _status(base.replace(rope_theta=-1.0)) == abi.DLLM_ERR_INVALID
    assert _status(base.replace(tau=float("nan"))) == abi.DLLM_ERR_INVALID
    assert _status(base.replace(tau=float("inf"))) == abi.DLLM_OK   # forced commits only
    # sizes whose positions or 32-bit row offsets would overflow
    assert _status(base.replace(prompt_len=2 ** 31 - 64)) == abi.DLLM_ERR_UNSUPPORTED
    assert _status(base.replace(prompt_len=2 ** 24)) == abi.DLLM_ERR_UNSUPPORTED
    llada = wl.WORKLOADS["llada8b_dual"]
    assert _status(llada.replace(batch=1024, prompt_len=65536 - 256)) \
        == abi.DLLM_ERR_UNSUPPORTED                                      # L*b*Hkv*S >= 2^31
    assert _status(llada.replace(batch=1024, prompt_len=1024)) == abi.DLLM_OK


def test_commit_mode_validation(lib):
    base = wl.WORKLOADS["tiny"]
    topk = base.replace(commit_mode=wl.COMMIT_TOPK)
    assert _status(topk.replace(steps_per_block=1)) == abi.DLLM_OK
    assert _status(topk.replace(steps_per_block=base.block)) == abi.DLLM_OK
    assert _status(topk.replace(steps_per_block=0)) == abi.DLLM_ERR_INVALID
    assert _status(topk.replace(steps_per_block=base.block + 1)) == abi.DLLM_ERR_INVALID
    ex = base.replace(commit_mode=wl.COMMIT_EARLY_EXIT)
    assert _status(ex.replace(exit_tau=0.5)) == abi.DLLM_OK
    assert _status(ex.replace(exit_tau=0.0)) == abi.DLLM_OK
    assert _status(ex.replace(exit_tau=-0.1)) == abi.DLLM_ERR_INVALID
    assert _status(ex.replace(exit_tau=float("nan"))) == abi.DLLM_ERR_INVALID
    assert _status(ex.replace(exit_tau=float("inf"))) == abi.DLLM_ERR_INVALID
    assert _status(base.replace(commit_mode=3)) == abi.DLLM_ERR_INVALID
    # the threshold rule ignores steps_per_block
    assert _status(base.replace(steps_per_block=-3)) == abi.DLLM_OK


def test_null_pointers_rejected_before_launch(lib):
    cfg = make_config(wl.WORKLOADS["tiny"])
    n = C.c_size_t(0)
    abi.dllm_workspace_size(C.byref(cfg), C.byref(n))
    # null workspace / weights / state: rejected by validation, nothing launched
    assert abi.dllm_decode_step(C.byref(cfg), None, None, 64, None, n.value, None) \
        == abi.DLLM_ERR_INVALID
    assert abi.dllm_workspace_init(C.byref(cfg), None, n.value, None) == abi.DLLM_ERR_INVALID
    assert abi.dllm_threshold_commit(C.byref(cfg), 64, None, None, None, None, None, None,
                                     None, None, None) == abi.DLLM_ERR_INVALID
    import torch
    if torch.cuda.is_available():   # the checks below pass dummy device pointers
        return
    # misaligned workspace pointer
    assert abi.dllm_workspace_init(C.byref(cfg), C.c_void_p(0x1008), n.value, None) \
        == abi.DLLM_ERR_INVALID
    # too-small workspace
    assert abi.dllm_workspace_init(C.byref(cfg), C.c_void_p(0x100000), 256, None) \
        == abi.DLLM_ERR_WORKSPACE


def test_status_strings(lib):
    assert abi.dllm_status_string(0) == b"ok"
    assert b"workspace" in abi.dllm_status_string(abi.DLLM_ERR_WORKSPACE)


def test_range_arguments_cannot_wrap(lib):
    """Row and block ranges are checked in 64-bit before anything touches the
    device: int32 arguments near 2^31 that would wrap an int32 sum are
    rejected.  Every call here must fail validation, so the dummy pointers
    are never used (no call in this test may pass it)."""
    import torch
    if torch.cuda.is_available():   # a regression would launch on the dummy pointers
        pytest.skip("dummy device pointers: runs only where no GPU is visible")
    w = wl.WORKLOADS["llada8b_dual"]           # P 256, B 32, S 512
    cfg = C.byref(make_config(w))
    n = C.c_size_t(0)
    assert abi.dllm_workspace_size(cfg, C.byref(n)) == abi.DLLM_OK
    d = C.c_void_p(1 << 20)                    # aligned, never dereferenced
    weights = C.byref(abi.dllm_weights(d, d, d, d))
    state = C.byref(abi.dllm_state(d, d, d, d, d, d, None))
    big = 2 ** 31 - 32                         # (big - P) % B == 0; big + B wraps
    bad = abi.DLLM_ERR_INVALID
    assert abi.dllm_decode_step(cfg, weights, state, big, d, n.value, None) == bad
    assert abi.dllm_kv_cache_refresh(cfg, weights, state, big, d, n.value, None) == bad
    steps = C.c_int32(0)
    assert abi.dllm_decode_block(cfg, weights, state, big, 0, C.byref(steps), d, n.value,
                                 None) == bad
    assert abi.dllm_threshold_commit(cfg, big, d, d, d, d, None, None, None, None, None) == bad
    assert abi.dllm_embed_rows(cfg, weights, state, big, 64, d, d, None, None) == bad
    assert abi.dllm_final_norm(cfg, d, big, 64, 256, d, d, d, None) == bad
    assert abi.dllm_final_norm(cfg, d, 0, 512, big, d, d, d, None) == bad
    assert abi.dllm_qkv_proj(cfg, weights, 0, d, None, big, 64, d, d, d, d, d, n.value,
                             None) == bad
    assert abi.dllm_o_proj(cfg, weights, 0, d, big, 64, d, d, None, d, n.value, None) == bad
    assert abi.dllm_qkv_proj(cfg, weights, 0, d, None, 0, 2 ** 31 - 1, d, d, d, d, d, n.value,
                             None) == bad


def test_layer_stack_plan_partitions_every_weight_block():
    """Host plan of the persistent layer-stack kernel: for the workload shapes
    it serves and for ragged mid-size ones, every 64-wide k-block of every
    weight tile belongs to exactly one CTA share, and the attention units fit
    one per CTA.  Shapes outside its scope report that they do not qualify."""
    from diffusion_decoding_step_b200 import workload as wl
    from diffusion_decoding_step_b200.runtime import make_config
    shapes = [wl.WORKLOADS["llada8b_dual"], wl.WORKLOADS["dream7b_prefix"]]
    for hidden, hq, hkv in ((512, 4, 4), (896, 7, 1), (1280, 10, 2), (3584, 28, 4),
                            (4096, 32, 8), (384, 3, 1), (8192, 64, 8)):
        shapes.append(wl.Workload("s", batch=1, n_layers=2, hidden=hidden, n_q_heads=hq,
                                  n_kv_heads=hkv, head_dim=128, vocab=8192, prompt_len=96,
                                  gen_len=64, block=32, mode=wl.MODE_DUAL))
    for w in shapes:
        cfg = make_config(w)
        for blk in range(w.prompt_len, w.seq_len, w.block):
            info = (C.c_int32 * 8)()
            assert abi.dllm_layer_stack_plan(C.byref(cfg), blk, info) == abi.DLLM_OK
            assert info[0] == 1, (w.hidden, blk)
            assert info[7] == 1, (w.hidden, blk)
            assert 1 <= info[2] <= 148 and 1 <= info[3] <= 148
            assert info[6] <= 148 and info[4] in (1, 2, 4, 8, 16)
    for name in ("tiny", "llada8b_dual_b16", "qwen7b_long_pruned"):
        w = wl.WORKLOADS[name]
        info = (C.c_int32 * 8)()
        assert abi.dllm_layer_stack_plan(C.byref(make_config(w)), w.prompt_len, info) == abi.DLLM_OK
        assert info[0] == 0


def _attn_plan(w, block_start):
    info = (C.c_int32 * 8)()
    st = abi.dllm_attention_plan(C.byref(make_config(w)), block_start, info)
    return st, list(info)


def _cdiv(a, b):
    return -(-a // b)


def test_attention_plan_invariants():
    """Host plan of the block attention: the row tiles cover the GQA group's
    query rows with none empty, the key chunks cover the key-tile bound
    (seven chunks run as eight, the last empty), the cluster stays within the
    merge buffer's limit, 32-row tiles only with head_dim 128, and row tiles
    that already fill the SMs keep one chunk."""
    shapes = list(wl.WORKLOADS.values())
    for mode in (wl.MODE_NONE, wl.MODE_PREFIX, wl.MODE_DUAL, wl.MODE_DUAL_PRUNED,
                 wl.MODE_PREFIX_SUFFIXQ):
        shapes.append(wl.WORKLOADS["dream7b_prefix"].replace(mode=mode, window=64))
        shapes.append(wl.WORKLOADS["tiny"].replace(mode=mode, window=8))
    for w in shapes:
        g = w.n_q_heads // w.n_kv_heads
        starts = list(range(w.prompt_len, w.seq_len, w.block))
        if w.mode != wl.MODE_NONE:
            starts.append(-1)
        for blk in starts:
            st, info = _attn_plan(w, blk)
            assert st == abi.DLLM_OK, (w.name, blk)
            rows_per_tile, row_tiles, chunks, tpc, ctas, ntb, threads, stages = info
            if blk < 0:
                n_rows = w.prompt_len if w.mode in (wl.MODE_PREFIX, wl.MODE_PREFIX_SUFFIXQ) \
                    else w.seq_len
            elif w.mode == wl.MODE_NONE:
                n_rows = blk + w.block
            elif w.mode == wl.MODE_PREFIX_SUFFIXQ:
                n_rows = w.seq_len - blk
            else:
                n_rows = w.block
            gr = g * n_rows
            assert rows_per_tile in (32, 128)
            assert rows_per_tile == 128 or w.head_dim == 128
            assert rows_per_tile * row_tiles >= gr > rows_per_tile * (row_tiles - 1)
            assert threads == (128 if rows_per_tile == 32 else 256)
            assert chunks * tpc >= ntb >= 1
            assert chunks == _cdiv(ntb, tpc) or (_cdiv(ntb, tpc) == 7 and chunks == 8)
            assert chunks <= (8 if w.head_dim == 128 else 6)
            assert stages == (1 if tpc <= 1 else 2)
            assert ctas == w.batch * w.n_kv_heads * row_tiles * chunks
            if w.batch * w.n_kv_heads * row_tiles >= 148:
                assert chunks == 1


def test_attention_plan_of_the_workload_shapes():
    """The plans the design notes measure: LLaDA-8B's one-head groups take
    32-row tiles in 4 key chunks; Dream-7B's 224-row groups 7 such tiles per
    kv head with 3 chunks of 2 key tiles at the first block (84 CTAs, leaving
    SMs for the O-projection); the long-context Qwen shape 128-row tiles in 2
    chunks (one wave); the 16-sequence batch one chunk; prefills 128-row
    tiles."""
    W = wl.WORKLOADS
    assert _attn_plan(W["llada8b_dual"], 256)[1][:5] == [32, 1, 4, 1, 128]
    assert _attn_plan(W["dream7b_prefix"], 512)[1][:5] == [32, 7, 3, 2, 84]
    assert _attn_plan(W["dream7b_prefix"], 992)[1][:4] == [32, 7, 4, 2]
    q = _attn_plan(W["qwen7b_long_pruned"], 8192)[1]
    assert q[:3] == [128, 4, 2] and q[4] == 128
    assert _attn_plan(W["llada8b_dual_b16"], 1024)[1][:5] == [32, 1, 1, 10, 512]
    assert _attn_plan(W["llada8b_dual"], -1)[1][:4] == [128, 4, 1, 4]
    assert _attn_plan(W["tiny"], 64)[1][0] == 128                 # head_dim 32
    # not a block of the generation; a prefill of a cache mode without one
    assert _attn_plan(W["llada8b_dual"], 257)[0] == abi.DLLM_ERR_INVALID
    assert _attn_plan(W["llada8b_dual"].replace(mode=wl.MODE_NONE), -1)[0] == abi.DLLM_ERR_INVALID
