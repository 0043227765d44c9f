"""Lockstep comparison of the CUDA decode with the oracle (test helper).

Every step the oracle starts from the GPU's current state (tokens, mask and
bf16 caches) and recomputes the step; the GPU then runs the same step.
Confidences must agree within 2e-3, argmax tokens and commit decisions
exactly, except at rows the oracle flags as ambiguous, where the GPU's choice
is kept (it is the state the next step starts from) and counted.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

from oracle import dllm_oracle as O
from tests.gpu_util import f64, rel_l2

CONF_TOL = 2e-3


@dataclasses.dataclass
class Report:
    steps: int = 0
    rows: int = 0
    flagged: int = 0
    flagged_mismatch: int = 0
    max_conf_err: float = 0.0
    max_kv_rel: float = 0.0


def state_from_gpu(dec, layers=None) -> O.State:
    L = dec.w.n_layers if layers is None else layers
    return O.State(tokens=dec.tokens.cpu().numpy().astype(np.int64),
                   masked=dec.masked.cpu().numpy().astype(bool),
                   kcache=f64(dec.k_cache[:L]), vcache=f64(dec.v_cache[:L]),
                   starts=dec.seq_start.cpu().numpy().astype(np.int64))


def compare_step(dec, case, s: int, rep: Report, check_kv: bool = True,
                 step_in_block: int = 0, prev_tok=None):
    """One step compared; returns the GPU's argmax of the rows masked before
    the step (-1 elsewhere), the previous-step argmax of the early-exit rule."""
    cfg, W = case.cfg, case.W
    st = state_from_gpu(dec)
    r = O.decode_step(cfg, W, st, case.plants64, s, apply=False, step_in_block=step_in_block,
                      prev_tok=prev_tok)
    dec.step(s)
    torch.cuda.synchronize()
    assert dec.device_status() == 0
    conf, tok, gap, commit = (t.cpu().numpy() for t in dec.step_outputs())
    B = cfg.block
    check_block_state(dec, st.masked, s, B)
    for bi in range(cfg.batch):
        m = ~np.isnan(r.conf[bi])
        if not m.any():
            assert not commit[bi].any()
            continue
        rep.rows += int(m.sum())
        err = np.abs(conf[bi][m] - r.conf[bi][m])
        rep.max_conf_err = max(rep.max_conf_err, float(err.max()))
        assert err.max() <= CONF_TOL, f"conf error {err.max()} at block {s}"
        flag = r.amb_tok[bi] | r.amb_commit[bi]
        rep.flagged += int(flag.sum())
        tok_bad = m & (tok[bi] != r.tok[bi])
        com_bad = commit[bi].astype(bool) != r.commit[bi]
        bad = tok_bad | com_bad
        assert not (bad & ~flag).any(), (
            f"block {s} seq {bi}: unflagged mismatch rows {np.where(bad & ~flag)[0]} "
            f"gpu tok {tok[bi][bad]} oracle {r.tok[bi][bad]} gpu conf {conf[bi][bad]} "
            f"oracle conf {r.conf[bi][bad]}")
        rep.flagged_mismatch += int(bad.sum())
        # the state update matches the step's own commit decisions
        committed = commit[bi].astype(bool)
        assert not (committed & ~m).any()
        toks = dec.tokens[bi, s:s + B].cpu().numpy()
        assert np.array_equal(toks[committed], tok[bi][committed])
        assert not dec.masked[bi, s:s + B].cpu().numpy()[committed].any()
    if check_kv and cfg.mode != O.MODE_NONE:
        got = f64(dec.k_cache[:, :, :, s:s + B])
        rep.max_kv_rel = max(rep.max_kv_rel, rel_l2(got, st.kcache[:, :, :, s:s + B]))
        assert rel_l2(got, st.kcache[:, :, :, s:s + B]) <= 5e-3
        got = f64(dec.v_cache[:, :, :, s:s + B])
        assert rel_l2(got, st.vcache[:, :, :, s:s + B]) <= 5e-3
    rep.steps += 1
    return np.where(st.masked[:, s:s + B], tok, -1).astype(np.int64)


def check_block_state(dec, masked_before, s: int, B: int) -> None:
    """The commit step's block-done flags and refresh list are exactly the
    oracle's rule applied to the mask before and after the GPU's own commit."""
    done, refresh = (t.cpu().numpy() for t in dec.block_state())
    after = dec.masked.cpu().numpy().astype(bool)
    for bi in range(dec.w.batch):
        d_ref, r_ref = O.block_state(masked_before[bi, s:s + B], after[bi, s:s + B], s)
        assert int(done[bi]) == int(d_ref) and int(refresh[bi]) == r_ref, (s, bi)


def compare_refresh(dec, case, s: int) -> None:
    cfg, W = case.cfg, case.W
    if cfg.mode == O.MODE_NONE:
        return
    st = state_from_gpu(dec)
    O.refresh_block(cfg, W, st, s)
    dec.refresh(s)
    torch.cuda.synchronize()
    B = cfg.block
    for cache, ref in ((dec.k_cache, st.kcache), (dec.v_cache, st.vcache)):
        assert rel_l2(f64(cache[:, :, :, s:s + B]), ref[:, :, :, s:s + B]) <= 5e-3


def compare_prefill(dec, case) -> None:
    cfg, W = case.cfg, case.W
    dec.prefill()
    torch.cuda.synchronize()
    if cfg.mode == O.MODE_NONE:
        return
    st = state_from_gpu(dec)
    st.kcache[:] = 0
    st.vcache[:] = 0
    O.prefill(cfg, W, st)
    end = cfg.prompt_len if cfg.mode == O.MODE_PREFIX else cfg.seq_len
    for bi in range(cfg.batch):
        a = int(st.starts[bi])
        for cache, ref in ((dec.k_cache, st.kcache), (dec.v_cache, st.vcache)):
            got = f64(cache[:, bi, :, a:end])
            assert rel_l2(got, ref[:, bi, :, a:end]) <= 5e-3


def lockstep(dec, case, max_blocks: int | None = None, max_steps: int | None = None) -> Report:
    rep = Report()
    compare_prefill(dec, case)
    cfg = case.cfg
    blocks = list(range(cfg.prompt_len, cfg.seq_len, cfg.block))
    if max_blocks is not None:
        blocks = blocks[:max_blocks]
    for s in blocks:
        n = 0
        prev = None
        while dec.masked[:, s:s + cfg.block].any():
            if max_steps is not None and n >= max_steps:
                break
            prev = compare_step(dec, case, s, rep, step_in_block=n, prev_tok=prev)
            n += 1
            assert n <= cfg.block
        compare_refresh(dec, case, s)
    return rep


def compare_step_sampled(dec, case, s: int, seqs, rep: Report, taus=None,
                         step_in_block: int = 0) -> None:
    """One GPU step of the whole batch, checked on the sequences `seqs` only:
    the oracle recomputes each of them alone from its GPU state (sequences of
    a batch are independent, which the oracle's own pins establish).  taus:
    per-sequence thresholds, when the GPU runs with them."""
    refs = {}
    for bi in seqs:
        cfg1 = dataclasses.replace(case.cfg, batch=1,
                                   **({} if taus is None else {"tau": float(taus[bi])}))
        st = O.State(tokens=dec.tokens[bi:bi + 1].cpu().numpy().astype(np.int64),
                     masked=dec.masked[bi:bi + 1].cpu().numpy().astype(bool),
                     kcache=f64(dec.k_cache[:, bi:bi + 1]), vcache=f64(dec.v_cache[:, bi:bi + 1]),
                     starts=dec.seq_start[bi:bi + 1].cpu().numpy().astype(np.int64))
        refs[bi] = O.decode_step(cfg1, case.W, st, case.plants64[bi:bi + 1], s, apply=False,
                                 step_in_block=step_in_block)
        del st
    dec.step(s)
    torch.cuda.synchronize()
    assert dec.device_status() == 0
    conf, tok, gap, commit = (t.cpu().numpy() for t in dec.step_outputs())
    for bi, r in refs.items():
        m = ~np.isnan(r.conf[0])
        if not m.any():  # this sequence's block is already done
            assert not commit[bi].any()
            continue
        rep.rows += int(m.sum())
        err = np.abs(conf[bi][m] - r.conf[0][m])
        rep.max_conf_err = max(rep.max_conf_err, float(err.max()))
        assert err.max() <= CONF_TOL, f"seq {bi}: conf error {err.max()}"
        flag = r.amb_tok[0] | r.amb_commit[0]
        rep.flagged += int(flag.sum())
        bad = (m & (tok[bi] != r.tok[0])) | (commit[bi].astype(bool) != r.commit[0])
        assert not (bad & ~flag).any(), f"seq {bi}: unflagged mismatch rows {np.where(bad & ~flag)[0]}"
        rep.flagged_mismatch += int(bad.sum())
    rep.steps += 1


def lockstep_incremental(dec, case, max_blocks=None, log=None) -> Report:
    """lockstep() for full-size workloads: the oracle's copy of the state is
    kept on the host and only what a GPU step or refresh writes (the block's
    cache slots, tokens and mask) is copied back, instead of the whole caches
    every step.  Prefill, every step and every refresh are compared exactly as
    lockstep() does; the block's keys/values are compared after each step."""
    import time
    rep = Report()
    cfg, W, B = case.cfg, case.W, case.cfg.block
    dec.prefill()
    torch.cuda.synchronize()
    assert dec.device_status() == 0
    st = state_from_gpu(dec)
    end = cfg.prompt_len if cfg.mode == O.MODE_PREFIX else cfg.seq_len
    ref = O.new_state(cfg, st.tokens, st.masked, st.starts)
    O.prefill(cfg, W, ref)
    # Both prefills run free through every layer: unlike a step or a refresh,
    # the keys the attention reads are each side's own, so the two sides'
    # bf16 roundings decorrelate with depth.  Layer 0 (same inputs up to
    # rounding) keeps 5e-3; all layers together get 1e-2, about 1.3 bf16 ulps
    # of relative spacing (2^-7).  On the 32-layer shape the per-layer rel-L2
    # rises from 1e-4 at layer 0 to 5.7e-3 at layer 31.
    for bi in range(cfg.batch):
        a = int(st.starts[bi])
        for got, want in ((st.kcache, ref.kcache), (st.vcache, ref.vcache)):
            assert rel_l2(got[0, bi, :, a:end], want[0, bi, :, a:end]) <= 5e-3
            assert rel_l2(got[:, bi, :, a:end], want[:, bi, :, a:end]) <= 1e-2
    del ref
    blocks = list(range(cfg.prompt_len, cfg.seq_len, B))[:max_blocks]
    t0 = time.time()
    for s in blocks:
        n = 0
        prev = None
        while st.masked[:, s:s + B].any():
            r = O.decode_step(cfg, W, st, case.plants64, s, apply=False, step_in_block=n,
                              prev_tok=prev)
            dec.step(s)
            torch.cuda.synchronize()
            assert dec.device_status() == 0
            conf, tok, gap, commit = (t.cpu().numpy() for t in dec.step_outputs())
            check_block_state(dec, st.masked, s, B)
            for bi in range(cfg.batch):
                m = ~np.isnan(r.conf[bi])
                if not m.any():
                    assert not commit[bi].any()
                    continue
                rep.rows += int(m.sum())
                err = np.abs(conf[bi][m] - r.conf[bi][m])
                rep.max_conf_err = max(rep.max_conf_err, float(err.max()))
                assert err.max() <= CONF_TOL, f"conf error {err.max()} at block {s}"
                flag = r.amb_tok[bi] | r.amb_commit[bi]
                rep.flagged += int(flag.sum())
                bad = (m & (tok[bi] != r.tok[bi])) | (commit[bi].astype(bool) != r.commit[bi])
                assert not (bad & ~flag).any(), (
                    f"block {s} seq {bi}: unflagged mismatch rows {np.where(bad & ~flag)[0]}")
                rep.flagged_mismatch += int(bad.sum())
            # the oracle wrote its own keys/values of the block rows into st:
            # compare, then continue from what the GPU wrote
            got_k = f64(dec.k_cache[:, :, :, s:s + B])
            got_v = f64(dec.v_cache[:, :, :, s:s + B])
            kr = rel_l2(got_k, st.kcache[:, :, :, s:s + B])
            rep.max_kv_rel = max(rep.max_kv_rel, kr)
            assert kr <= 5e-3
            assert rel_l2(got_v, st.vcache[:, :, :, s:s + B]) <= 5e-3
            st.kcache[:, :, :, s:s + B] = got_k
            st.vcache[:, :, :, s:s + B] = got_v
            prev = np.where(st.masked[:, s:s + B], tok, -1).astype(np.int64)
            st.tokens = dec.tokens.cpu().numpy().astype(np.int64)
            st.masked = dec.masked.cpu().numpy().astype(bool)
            rep.steps += 1
            n += 1
            assert n <= B
        O.refresh_block(cfg, W, st, s)
        dec.refresh(s)
        torch.cuda.synchronize()
        got_k = f64(dec.k_cache[:, :, :, s:s + B])
        got_v = f64(dec.v_cache[:, :, :, s:s + B])
        assert rel_l2(got_k, st.kcache[:, :, :, s:s + B]) <= 5e-3
        assert rel_l2(got_v, st.vcache[:, :, :, s:s + B]) <= 5e-3
        st.kcache[:, :, :, s:s + B] = got_k
        st.vcache[:, :, :, s:s + B] = got_v
        if log:
            log(f"block {s}: {n} steps, {rep.steps} steps so far, flagged {rep.flagged}, "
                f"flagged mismatches {rep.flagged_mismatch}, max conf err {rep.max_conf_err:.2e}, "
                f"max kv rel {rep.max_kv_rel:.2e}, {time.time() - t0:.0f} s")
    return rep
