"""Property test of the C ABI's host-side validation (no GPU).

Random configurations, many of them nonsense, go to dllm_workspace_size,
which validates a configuration exactly as every launching entry point does
and launches nothing.  It must answer with a defined status and never crash.
A configuration it accepts must get a finite, aligned workspace size that
does not shrink when the batch grows.
"""
import ctypes as C

from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

from diffusion_decoding_step_b200 import abi, build

build.build()
_lib = abi.lib()

EDGE = [-(2 ** 31), -1, 0, 1, 2, 3, 7, 8, 31, 32, 33, 64, 127, 128, 129, 1024, 4096,
        2 ** 16, 2 ** 20, 2 ** 31 - 1]
small = st.one_of(st.sampled_from(EDGE), st.integers(-4, 300))
dims = st.one_of(st.sampled_from([32, 64, 96, 128, 256, 512, 3584, 4096] + EDGE),
                 st.integers(-8, 9000))


@st.composite
def configs(draw):
    return abi.dllm_config(
        batch=draw(small), n_layers=draw(small), hidden=draw(dims), n_q_heads=draw(small),
        n_kv_heads=draw(small), head_dim=draw(st.sampled_from([32, 64, 128] + EDGE)),
        vocab=draw(st.one_of(st.sampled_from([1024, 4096, 126464, 152064] + EDGE),
                             st.integers(-8, 200000))),
        prompt_len=draw(dims), gen_len=draw(dims), block=draw(small), window=draw(small),
        mask_id=draw(st.one_of(st.sampled_from(EDGE), st.integers(-2, 200000))),
        tau=draw(st.floats(allow_nan=True, allow_infinity=True, width=32)),
        rope_theta=draw(st.floats(allow_nan=True, allow_infinity=True, width=32)),
        mode=draw(st.integers(-2, 6)), weight_format=draw(st.integers(-1, 3)),
        commit_mode=draw(st.integers(-1, 3)), steps_per_block=draw(small))


FIELDS = [f for f, _ in abi.dllm_config._fields_]


@st.composite
def perturbed(draw):
    """A valid workload's configuration with one to three fields replaced."""
    from diffusion_decoding_step_b200 import workload as wl
    from diffusion_decoding_step_b200.runtime import make_config
    cfg = make_config(draw(st.sampled_from(list(wl.WORKLOADS.values()))))
    for field in draw(st.lists(st.sampled_from(FIELDS), min_size=1, max_size=3, unique=True)):
        cur = getattr(cfg, field)
        if isinstance(cur, float):
            val = draw(st.floats(allow_nan=True, allow_infinity=True, width=32))
        else:
            val = draw(st.one_of(st.sampled_from(EDGE), st.integers(-2, 2 * max(abs(cur), 2)),
                                 st.sampled_from([cur // 2, cur * 2, cur + 1, cur - 1])))
        setattr(cfg, field, max(-(2 ** 31), min(2 ** 31 - 1, val)) if isinstance(val, int)
                else val)
    return cfg


def _stack_rows(cfg):
    """Whether any block of the configuration runs as one layer-stack launch."""
    info = (C.c_int32 * 8)()
    for blk in range(max(cfg.prompt_len, 0), cfg.prompt_len + cfg.gen_len,
                     max(cfg.block, 1)):
        if abi.dllm_layer_stack_plan(C.byref(cfg), blk, info) == abi.DLLM_OK and info[0]:
            return True
    return False


def _size(cfg):
    n = C.c_size_t(0)
    return abi.dllm_workspace_size(C.byref(cfg), C.byref(n)), n.value


@settings(max_examples=3000, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(st.one_of(configs(), perturbed()))
def test_workspace_query_answers_every_configuration(cfg):
    status, n = _size(cfg)
    assert status in (abi.DLLM_OK, abi.DLLM_ERR_INVALID, abi.DLLM_ERR_UNSUPPORTED)
    if status != abi.DLLM_OK:
        return
    assert 0 < n < (1 << 44) and n % 256 == 0   # under 16 TiB: no wrapped arithmetic
    bigger = abi.dllm_config.from_buffer_copy(cfg)
    bigger.batch = cfg.batch + 1
    s2, n2 = _size(bigger)
    # the layer-stack kernel's scratch is reserved only for shapes it runs
    # (at most 64 activation rows), so compare sizes on the same path
    if s2 == abi.DLLM_OK and _stack_rows(cfg) == _stack_rows(bigger):
        assert n2 >= n
