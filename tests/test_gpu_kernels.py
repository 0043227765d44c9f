"""Per-kernel parity of the CUDA path against the fp64 oracle (B200 only).

Each test feeds the same seeded bf16 inputs to one C-ABI entry point and to
the oracle function that defines it, and compares element by element with the
tolerances of the decode step: bf16 attention output rel-L2 <= 5e-3 and
max-abs <= 1e-2; confidence abs <= 2e-3; argmax ids, commit masks and token
updates bit-exact except rows the oracle flags as ambiguous.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from oracle import dllm_oracle as O
from diffusion_decoding_step_b200 import workload as wl
from diffusion_decoding_step_b200.runtime import make_config, workspace_bytes
from tests.gpu_util import ensure_lib, ptr, stream, f64, bf16_ulp_close, rel_l2

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _ws(w):
    abi = ensure_lib()
    cfg = make_config(w)
    n = workspace_bytes(w)
    ws = torch.empty(n, dtype=torch.uint8, device=DEV)
    abi.check(abi.dllm_workspace_init(C.byref(cfg), ptr(ws), n, stream()), "ws init")
    return abi, cfg, ws, n


def _gen(seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    return g


def _weights_c(abi, wqkv=None, wo=None, w_lm=None, embed=None):
    return abi.dllm_weights(ptr(wqkv), ptr(wo), ptr(w_lm), ptr(embed if embed is not None else w_lm))


# ---------------------------------------------------------------- LM head
LM_CASES = [  # (rows, hidden, vocab, batch, block)
    (8, 128, 1024, 1, 8),
    (32, 512, 8192, 1, 32),
    (50, 256, 4096, 1, 64),
    (200, 256, 2048, 4, 64),
    (512, 512, 4096, 16, 32),
    (32, 4096, 126464, 1, 32),
    (512, 512, 65536, 16, 32),      # several tiles per CTA at 256 rows
    (128, 1024, 32768, 4, 32),      # several tiles per CTA at 128 rows
]


@pytest.mark.parametrize("R,d,V,b,B", LM_CASES)
def test_lmhead_confidence_matches_oracle(R, d, V, b, B):
    w = wl.Workload("t", batch=b, n_layers=1, hidden=d, n_q_heads=1, n_kv_heads=1, head_dim=128,
                    vocab=V, prompt_len=0, gen_len=B, block=B)
    abi, cfg, ws, n = _ws(w)
    g = _gen(R + d + V)
    W = (torch.randn(V, d, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    t = torch.randint(0, V, (R,), generator=g, device=DEV)
    a = torch.rand(R, generator=g, device=DEV) * 20
    rows = W[t].float()
    h = a[:, None] * rows / (rows * rows).sum(1, keepdim=True)
    h = h + torch.randn(R, d, generator=g, device=DEV) / (0.02 * d ** 0.5)
    h[0] = 0.0  # uniform logits: conf = 1/V, token 0
    h = h.to(torch.bfloat16)
    conf = torch.empty(R, dtype=torch.float32, device=DEV)
    tok = torch.empty(R, dtype=torch.int32, device=DEV)
    gap = torch.empty(R, dtype=torch.float32, device=DEV)
    wc = _weights_c(abi, w_lm=W)
    abi.check(abi.dllm_lmhead_confidence(C.byref(cfg), C.byref(wc), ptr(h), R, ptr(conf),
                                         ptr(tok), ptr(gap), ptr(ws), n, stream()), "lmhead")
    torch.cuda.synchronize()
    c_ref, t_ref, g_ref = O.lm_head_confidence(f64(h), f64(W))
    c, tk, gp = f64(conf), tok.cpu().numpy(), f64(gap)
    assert np.abs(c - c_ref).max() <= 2e-3
    sure = g_ref >= O.AMBIG_GAP
    assert np.array_equal(tk[sure], t_ref[sure])
    assert np.abs(gp[sure] - g_ref[sure]).max() < 1e-3
    assert tk[0] == 0 and abs(c[0] - 1.0 / V) < 1e-6
    assert (c > 0).all() and (c <= 1.0 + 1e-6).all()


# ---------------------------------------------------------------- QKV projection
QKV_CASES = [  # (hidden, Hq, Hkv, D, batch, n_rows, row0, theta, S)
    (128, 4, 4, 32, 1, 8, 64, 0.0, 96),
    (512, 4, 4, 128, 1, 32, 256, 0.0, 512),
    (896, 7, 1, 128, 2, 32, 512, 1e6, 1024),
    (4096, 32, 32, 128, 1, 32, 256, 0.0, 512),
    (3584, 28, 4, 128, 1, 32, 512, 1e6, 1024),
    (512, 4, 2, 128, 2, 300, 0, 1e4, 300),
    (4096, 32, 32, 128, 1, 512, 0, 0.0, 512),   # prefill shape: 256-row tiles, split K
    (4096, 32, 32, 128, 1, 128, 0, 0.0, 512),   # 128-row tiles, several per CTA
    (4096, 32, 32, 128, 1, 64, 0, 0.0, 512),
]


def _qkv_case(d, Hq, Hkv, D, b, nr, row0, theta, S, f32=False, seed=0, norm=True):
    w = wl.Workload("t", batch=b, n_layers=2, hidden=d, n_q_heads=Hq, n_kv_heads=Hkv,
                    head_dim=D, vocab=1024, prompt_len=S - 32, gen_len=32, block=32,
                    rope_theta=theta, weight_f32=f32)
    abi, cfg, ws, n = _ws(w)
    g = _gen(seed + d + nr)
    rows = w.qkv_rows
    Wf = torch.randn(2, rows, d, generator=g, device=DEV) * 0.02
    xf = torch.randn(b * nr, d, generator=g, device=DEV) * 3
    x = xf.to(torch.bfloat16)
    sumsq = (xf * xf).reshape(b * nr, d // 128, 128).sum(-1).contiguous() if norm else None
    starts = torch.randint(0, 5, (b,), generator=g, device=DEV).to(torch.int32)
    if f32:
        Wk = torch.empty(2, rows, 2 * d, dtype=torch.bfloat16, device=DEV)
        abi.check(abi.dllm_split_f32_weights(ptr(Wf.contiguous()), ptr(Wk), 2 * rows, d,
                                             stream()), "split")
        Wref = f64(Wf)
    else:
        Wk = Wf.to(torch.bfloat16)
        Wref = f64(Wk)
    q = torch.zeros(b, Hq, nr, D, dtype=torch.bfloat16, device=DEV)
    kc = torch.zeros(2, b, Hkv, S, D, dtype=torch.bfloat16, device=DEV)
    vc = torch.zeros_like(kc)
    wc = _weights_c(abi, wqkv=Wk, wo=Wk, w_lm=Wk)
    layer = 1
    abi.check(abi.dllm_qkv_proj(C.byref(cfg), C.byref(wc), layer, ptr(x), ptr(sumsq), row0, nr,
                                ptr(starts), ptr(q), ptr(kc), ptr(vc), ptr(ws), n, stream()),
              "qkv")
    torch.cuda.synchronize()
    X = f64(x).reshape(b, nr, d)
    qkv = X @ Wref[layer].T
    if norm:
        qkv = qkv * O.inv_rms(f64(xf).reshape(b, nr, d))[..., None]
    qr = qkv[..., :Hq * D].reshape(b, nr, Hq, D).transpose(0, 2, 1, 3)
    kr = qkv[..., Hq * D:(Hq + Hkv) * D].reshape(b, nr, Hkv, D).transpose(0, 2, 1, 3)
    vr = qkv[..., (Hq + Hkv) * D:].reshape(b, nr, Hkv, D).transpose(0, 2, 1, 3)
    if theta > 0:
        st = starts.cpu().numpy()
        for bi in range(b):
            pos = np.maximum(np.arange(row0, row0 + nr) - st[bi], 0)
            qr[bi] = O.rope(qr[bi], pos, theta)
            kr[bi] = O.rope(kr[bi], pos, theta)
    return (f64(q), qr, f64(kc[layer, :, :, row0:row0 + nr]), kr,
            f64(vc[layer, :, :, row0:row0 + nr]), vr, kc, vc, row0, nr)


def _acc_atol(ref):
    # fp32 accumulation over K terms leaves an absolute error of a few 1e-6 of
    # the output scale; values that cancel to near zero can round to another
    # bf16 neighbour for that reason alone
    return 1e-5 * max(1.0, float(np.sqrt(np.mean(ref * ref))))


@pytest.mark.parametrize("case", QKV_CASES)
def test_qkv_projection_rope_and_cache_write(case):
    q, qr, k, kr, v, vr, kc, vc, row0, nr = _qkv_case(*case)
    for gpu, ref in ((q, qr), (k, kr), (v, vr)):
        bf16_ulp_close(gpu, O.round_bf16(ref), ulps=1.0, atol=_acc_atol(ref))
    # nothing outside the rows was written
    assert float(kc[1, :, :, :row0].abs().sum()) == 0.0
    assert float(vc[1, :, :, row0 + nr:].abs().sum()) == 0.0
    assert float(kc[0].abs().sum()) == 0.0


def test_qkv_projection_without_row_scale():
    q, qr, k, kr, v, vr, *_ = _qkv_case(512, 4, 4, 128, 1, 32, 256, 0.0, 512, norm=False)
    for gpu, ref in ((q, qr), (k, kr), (v, vr)):
        bf16_ulp_close(gpu, O.round_bf16(ref), ulps=1.0, atol=_acc_atol(ref))


def test_qkv_projection_f32_split_weights():
    q, qr, k, kr, v, vr, *_ = _qkv_case(128, 4, 4, 32, 1, 8, 64, 0.0, 96, f32=True)
    for gpu, ref in ((q, qr), (k, kr), (v, vr)):
        bf16_ulp_close(gpu, O.round_bf16(ref), ulps=1.0, atol=_acc_atol(ref))


# ---------------------------------------------------------------- O projection
OPROJ_CASES = [  # (hidden, Hq, D, batch, n_rows, block_start)
    (128, 4, 32, 1, 8, 64),
    (4096, 32, 128, 1, 32, 256),
    (3584, 28, 128, 1, 32, 512),
    (512, 4, 128, 2, 96, 32),
    (512, 8, 128, 16, 32, 0),
    (4096, 32, 128, 1, 512, 0),
    (4096, 32, 128, 1, 128, 0),
    (4096, 32, 128, 2, 32, 256),   # 64-row tiles, K split over a 3-CTA cluster
    (1024, 8, 128, 1, 48, 64),     # ragged 64-row tile, 3-CTA cluster
    (8192, 64, 128, 1, 32, 0),     # 2-CTA cluster
]


@pytest.mark.parametrize("d,Hq,D,b,nr,blk", OPROJ_CASES)
def test_output_projection_residual(d, Hq, D, b, nr, blk):
    w = wl.Workload("t", batch=b, n_layers=2, hidden=d, n_q_heads=Hq, n_kv_heads=Hq, head_dim=D,
                    vocab=1024, prompt_len=max(blk, 32), gen_len=max(32, -(-nr // 32) * 32),
                    block=32)
    abi, cfg, ws, n = _ws(w)
    g = _gen(d + nr)
    Wo = (torch.randn(2, d, Hq * D, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    attn = torch.randn(b * nr, Hq * D, generator=g, device=DEV).to(torch.bfloat16)
    x = torch.randn(b * nr, d, generator=g, device=DEV)
    x0 = x.clone()
    xb = torch.zeros(b * nr, d, dtype=torch.bfloat16, device=DEV)
    sumsq = torch.full((b * nr, d // 128), -1.0, device=DEV)
    wc = _weights_c(abi, wqkv=Wo, wo=Wo, w_lm=Wo)
    row0 = blk
    abi.check(abi.dllm_o_proj(C.byref(cfg), C.byref(wc), 1, ptr(attn), row0, nr, ptr(x), ptr(xb),
                              ptr(sumsq), ptr(ws), n, stream()), "oproj")
    torch.cuda.synchronize()
    ref = f64(x0) + f64(attn) @ f64(Wo[1]).T
    got = f64(x)
    assert np.abs(got - ref).max() <= 1e-4 * (1 + np.abs(ref).max())
    bf16_ulp_close(f64(xb), O.round_bf16(got), ulps=0.0, atol=0.0)
    want = (got * got).reshape(b * nr, d // 128, 128).sum(-1)
    np.testing.assert_allclose(f64(sumsq), want, rtol=1e-5)


# ---------------------------------------------------------------- embed / final norm
@pytest.mark.parametrize("f32", [False, True])
def test_embed_rows_mask_token_and_sumsq(f32):
    w = wl.WORKLOADS["tiny"].replace(weight_f32=f32, batch=2, hidden=256, n_q_heads=8)
    abi = ensure_lib()
    cfg = make_config(w)
    g = _gen(7)
    E = torch.randn(w.vocab, w.hidden, generator=g, device=DEV) * 0.5
    if not f32:
        E = E.to(torch.bfloat16)
    S = w.seq_len
    tokens = torch.randint(0, w.vocab, (w.batch, S), generator=g, device=DEV).to(torch.int32)
    masked = (torch.rand(w.batch, S, generator=g, device=DEV) < 0.3).to(torch.uint8)
    row0, nr = 10, 70
    x = torch.empty(w.batch * nr, w.hidden, device=DEV)
    xb = torch.empty(w.batch * nr, w.hidden, dtype=torch.bfloat16, device=DEV)
    sumsq = torch.full((w.batch * nr, w.hidden // 128), -1.0, device=DEV)
    wc = _weights_c(abi, w_lm=E, embed=E)
    st = abi.dllm_state(ptr(tokens), ptr(masked), None, None, None, None)
    abi.check(abi.dllm_embed_rows(C.byref(cfg), C.byref(wc), C.byref(st), row0, nr, ptr(x),
                                  ptr(xb), ptr(sumsq), stream()), "embed")
    torch.cuda.synchronize()
    ids = torch.where(masked[:, row0:row0 + nr].bool(), w.mask_id, tokens[:, row0:row0 + nr])
    want = f64(E[ids.long()].float()).reshape(w.batch * nr, w.hidden)
    np.testing.assert_array_equal(f64(x), want)
    np.testing.assert_array_equal(f64(xb), O.round_bf16(want))
    ss = f64(sumsq)
    np.testing.assert_allclose(ss[:, 0], (want * want).sum(1), rtol=1e-5)
    assert (ss[:, 1:] == 0).all()


@pytest.mark.parametrize("mode,b,B", [(wl.MODE_DUAL, 1, 32), (wl.MODE_DUAL, 3, 64),
                                      (wl.MODE_NONE, 2, 8)])
def test_final_norm_adds_plants_of_masked_rows(mode, b, B):
    w = wl.Workload("t", batch=b, n_layers=1, hidden=512, n_q_heads=4, n_kv_heads=4,
                    head_dim=128, vocab=1024, prompt_len=64, gen_len=2 * B, block=B, mode=mode)
    abi = ensure_lib()
    cfg = make_config(w)
    g = _gen(b * B)
    blk = w.prompt_len + B
    row0, nr = (0, blk + B) if mode == wl.MODE_NONE else (blk, B)
    x = torch.randn(b * nr, w.hidden, generator=g, device=DEV) * 4
    masked = (torch.rand(b, w.seq_len, generator=g, device=DEV) < 0.5).to(torch.uint8)
    plants = torch.randn(b, w.gen_len, w.hidden, generator=g, device=DEV).to(torch.bfloat16)
    h = torch.empty(b, B, w.hidden, dtype=torch.bfloat16, device=DEV)
    abi.check(abi.dllm_final_norm(C.byref(cfg), ptr(x), row0, nr, blk, ptr(masked), ptr(plants),
                                  ptr(h), stream()), "final_norm")
    torch.cuda.synchronize()
    X = f64(x).reshape(b, nr, w.hidden)[:, blk - row0:blk - row0 + B]
    m = masked[:, blk:blk + B].cpu().numpy().astype(bool)
    pl = f64(plants)[:, blk - w.prompt_len:blk - w.prompt_len + B]
    want = X * O.inv_rms(X)[..., None] + np.where(m[..., None], pl, 0.0)
    bf16_ulp_close(f64(h), O.round_bf16(want), ulps=1.0, atol=1e-6)


# ---------------------------------------------------------------- attention
ATTN_CASES = [  # (Hq, Hkv, D, batch, n_rows, S, segs per sequence, layer)
    (32, 32, 128, 1, 32, 512, [[(0, 512), (0, 0)]], 0),
    (28, 4, 128, 1, 32, 1024, [[(0, 576), (0, 0)]], 1),
    (2, 2, 128, 2, 5, 300, [[(3, 250), (299, 1)], [(0, 77), (0, 0)]], 0),
    (4, 4, 32, 1, 8, 96, [[(0, 72), (0, 0)]], 0),
    (4, 4, 32, 1, 1, 96, [[(40, 1), (0, 0)]], 0),
    (28, 4, 128, 1, 64, 2300, [[(0, 2200), (2299, 1)]], 0),
    (8, 8, 128, 3, 32, 1280, [[(300, 980), (0, 0)], [(0, 1280), (0, 0)], [(512, 768), (0, 0)]], 1),
    (4, 2, 128, 1, 700, 700, [[(0, 700), (0, 0)]], 0),
    (32, 32, 128, 1, 512, 512, [[(0, 512), (0, 0)]], 1),   # prefill shape
    (28, 4, 128, 1, 32, 640, [[(0, 544), (639, 1)]], 0),   # 32-row tiles: 7 per kv head, 3 chunks
    (28, 4, 128, 1, 32, 1024, [[(5, 539), (0, 0)]], 1),    # 32-row tiles, 3 chunks of 3 tiles
    (8, 8, 32, 1, 16, 640, [[(0, 600), (0, 0)]], 0),       # head_dim 32, 6 chunks
    (28, 4, 128, 1, 32, 896, [[(0, 880), (895, 1)]], 0),   # 32-row tiles, 4 chunks
    (28, 4, 128, 1, 32, 768, [[(3, 700), (0, 0)]], 1),     # 32-row tiles, 4 chunks
    # 128-row tiles (groups of 448 rows)
    (28, 4, 128, 1, 64, 640, [[(0, 544), (639, 1)]], 0),   # 6 key chunks
    (28, 4, 128, 1, 64, 896, [[(0, 880), (895, 1)]], 0),   # 8 key chunks
    (28, 4, 128, 1, 64, 768, [[(3, 700), (0, 0)]], 1),     # 7 tiles: 8 chunks, the last empty
    # one 32-row tile per kv head
    (4, 4, 128, 1, 8, 768, [[(3, 700), (0, 0)]], 0),       # 7 tiles: 8 chunks, the last empty
    (4, 4, 128, 1, 8, 640, [[(0, 544), (639, 1)]], 1),     # 6 key chunks
    (4, 4, 128, 1, 1, 96, [[(0, 96), (0, 0)]], 0),         # one row, two tiles in one CTA
    (1, 1, 128, 1, 16, 64, [[(0, 64), (0, 0)]], 1),        # one tile, no chunks
    (16, 2, 128, 2, 4, 200, [[(0, 150), (199, 1)], [(20, 100), (0, 0)]], 0),  # GQA, 32 rows
]


@pytest.mark.parametrize("Hq,Hkv,D,b,nr,S,segs,layer", ATTN_CASES)
def test_block_attention_matches_oracle(Hq, Hkv, D, b, nr, S, segs, layer):
    w = wl.Workload("t", batch=b, n_layers=2, hidden=max(128, Hq * D), n_q_heads=Hq,
                    n_kv_heads=Hkv, head_dim=D, vocab=1024, prompt_len=S - 32, gen_len=32,
                    block=32)
    abi, cfg, ws, n = _ws(w)
    g = _gen(Hq * S + nr)
    q = torch.randn(b, Hq, nr, D, generator=g, device=DEV).to(torch.bfloat16)
    kc = torch.randn(2, b, Hkv, S, D, generator=g, device=DEV).to(torch.bfloat16)
    vc = torch.randn(2, b, Hkv, S, D, generator=g, device=DEV).to(torch.bfloat16)
    sg = torch.tensor([[v for seg in s for v in seg] for s in segs], dtype=torch.int32, device=DEV)
    out = torch.zeros(b * nr, Hq * D, dtype=torch.bfloat16, device=DEV)
    abi.check(abi.dllm_block_attn(C.byref(cfg), layer, nr, ptr(q), ptr(kc), ptr(vc), ptr(sg),
                                  ptr(out), ptr(ws), n, stream()), "attn")
    torch.cuda.synchronize()
    Q, K, V = f64(q), f64(kc[layer]), f64(vc[layer])
    ref = np.zeros((b, nr, Hq, D))
    gsz = Hq // Hkv
    for bi in range(b):
        keys = np.concatenate([np.arange(s0, s0 + ln) for s0, ln in segs[bi]]).astype(int)
        for h in range(Hq):
            ref[bi, :, h] = O.attention(Q[bi, h], K[bi, h // gsz][keys], V[bi, h // gsz][keys])
    got = f64(out).reshape(b, nr, Hq, D)
    assert rel_l2(got, ref) <= 5e-3
    assert np.abs(got - ref).max() <= 1e-2


# ---------------------------------------------------------------- commit
@pytest.mark.parametrize("b,B,tau", [(1, 8, 0.9), (1, 32, 0.9), (16, 32, 0.9), (4, 64, 0.5),
                                     (3, 32, 1.5), (2, 32, 1e-6)])
def test_threshold_commit_bit_exact(b, B, tau):
    w = wl.Workload("t", batch=b, n_layers=1, hidden=128, n_q_heads=4, n_kv_heads=4,
                    head_dim=32, vocab=1024, prompt_len=64, gen_len=2 * B, block=B, tau=tau)
    abi = ensure_lib()
    cfg = make_config(w)
    rng = np.random.default_rng(b * 100 + B)
    S = w.seq_len
    s = w.prompt_len + B
    conf = rng.uniform(0, 1, (b, B)).astype(np.float32)
    conf[0, :3] = 0.95
    conf[0, 3] = np.float32(tau) if tau < 1 else 0.5     # exactly tau: does not clear it
    if B > 8:
        conf[-1, 5] = conf[-1, 6] = 0.99999               # equal confidences
    masked = np.zeros((b, S), dtype=np.uint8)
    masked[:, s:s + B] = rng.uniform(size=(b, B)) < 0.7
    masked[0, s:s + B] = 1
    if b > 1:
        masked[1, s:s + B] = 0                             # a finished sequence
    tok = rng.integers(0, 1024, (b, B)).astype(np.int32)
    tokens = rng.integers(0, 1024, (b, S)).astype(np.int32)
    t_tokens = torch.tensor(tokens, device=DEV)
    t_masked = torch.tensor(masked, device=DEV)
    commit = torch.zeros(b, B, dtype=torch.uint8, device=DEV)
    remaining = torch.zeros(b, dtype=torch.int32, device=DEV)
    t_conf = torch.tensor(conf, device=DEV)
    t_tok = torch.tensor(tok, device=DEV)
    done = torch.full((b,), 7, dtype=torch.int32, device=DEV)
    refresh = torch.full((b,), 7, dtype=torch.int32, device=DEV)
    abi.check(abi.dllm_threshold_commit(C.byref(cfg), s, ptr(t_conf), ptr(t_tok), ptr(t_tokens),
                                        ptr(t_masked), ptr(commit), ptr(remaining), ptr(done),
                                        ptr(refresh), stream()),
              "commit")
    torch.cuda.synchronize()
    for bi in range(b):
        m = masked[bi, s:s + B].astype(bool)
        c_ref = O.threshold_commit(conf[bi].astype(np.float64), m, tau)
        assert np.array_equal(commit[bi].cpu().numpy().astype(bool), c_ref)
        want_tok = tokens[bi].copy()
        want_tok[s:s + B][c_ref] = tok[bi][c_ref]
        want_mask = masked[bi].copy()
        want_mask[s:s + B][c_ref] = 0
        assert np.array_equal(t_tokens[bi].cpu().numpy(), want_tok)
        assert np.array_equal(t_masked[bi].cpu().numpy(), want_mask)
        assert int(remaining[bi]) == int(m.sum() - c_ref.sum())
        d_ref, r_ref = O.block_state(m, m & ~c_ref, s)
        assert int(done[bi]) == int(d_ref) and int(refresh[bi]) == r_ref, f"seq {bi}"


@pytest.mark.parametrize("b,B,spb,done", [(1, 8, 3, 0), (1, 32, 5, 14), (16, 32, 8, 0),
                                          (4, 64, 7, 19), (3, 32, 32, 31), (2, 32, 1, 0)])
def test_topk_commit_bit_exact(b, B, spb, done):
    """Fixed-budget rule: every sequence commits its step's share of the
    block (from the rows it has committed so far), by confidence, lower
    position first on ties."""
    w = wl.Workload("t", batch=b, n_layers=1, hidden=128, n_q_heads=4, n_kv_heads=4,
                    head_dim=32, vocab=1024, prompt_len=64, gen_len=2 * B, block=B,
                    commit_mode=wl.COMMIT_TOPK, steps_per_block=spb)
    abi = ensure_lib()
    cfg = make_config(w)
    rng = np.random.default_rng(b * 1000 + B + spb)
    S = w.seq_len
    s = w.prompt_len + B
    conf = np.round(rng.uniform(0, 1, (b, B)), 2).astype(np.float32)   # many ties
    masked = np.zeros((b, S), dtype=np.uint8)
    for bi in range(b):
        left = rng.permutation(B)[:B - done] if bi % 2 == 0 else rng.permutation(B)[:max(1, B - done - bi)]
        masked[bi, s + left] = 1
    tok = rng.integers(0, 1024, (b, B)).astype(np.int32)
    tokens = rng.integers(0, 1024, (b, S)).astype(np.int32)
    t_tokens = torch.tensor(tokens, device=DEV)
    t_masked = torch.tensor(masked, device=DEV)
    commit = torch.zeros(b, B, dtype=torch.uint8, device=DEV)
    remaining = torch.zeros(b, dtype=torch.int32, device=DEV)
    t_conf = torch.tensor(conf, device=DEV)
    t_tok = torch.tensor(tok, device=DEV)
    done = torch.full((b,), 7, dtype=torch.int32, device=DEV)
    refresh = torch.full((b,), 7, dtype=torch.int32, device=DEV)
    abi.check(abi.dllm_threshold_commit(C.byref(cfg), s, ptr(t_conf), ptr(t_tok), ptr(t_tokens),
                                        ptr(t_masked), ptr(commit), ptr(remaining), ptr(done),
                                        ptr(refresh), stream()),
              "commit")
    torch.cuda.synchronize()
    for bi in range(b):
        m = masked[bi, s:s + B].astype(bool)
        k = O.topk_budget(B, spb, int(m.sum()))
        c_ref = O.topk_commit(conf[bi].astype(np.float64), m, k)
        assert np.array_equal(commit[bi].cpu().numpy().astype(bool), c_ref), f"seq {bi}"
        want_tok = tokens[bi].copy()
        want_tok[s:s + B][c_ref] = tok[bi][c_ref]
        assert np.array_equal(t_tokens[bi].cpu().numpy(), want_tok)
        assert int(remaining[bi]) == int(m.sum() - c_ref.sum())
        d_ref, r_ref = O.block_state(m, m & ~c_ref, s)
        assert int(done[bi]) == int(d_ref) and int(refresh[bi]) == r_ref, f"seq {bi}"
