"""C-ABI checks that need no GPU: the library loads, exports every function
include/tp.h declares, and rejects bad arguments on the host before any launch.

Every call here either fails validation or has T = 0, so no kernel is ever
launched (the fake pointers below are never dereferenced)."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

from megatron_tensor_transformer_gemm_b200 import tp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tp.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"TP_API\s+[\w\s\*]+?\b(tp_\w+)\s*\(", src)))


def test_header_declares_the_layer_and_collective_calls():
    names = declared_functions()
    for must in ["tp_plan_create", "tp_column_fwd", "tp_row_fwd_partial", "tp_reduce_partials",
                 "tp_reduce_scatter_seq", "tp_all_gather_seq", "tp_row_bwd", "tp_column_bwd",
                 "tp_reduce_scatter_seq_bwd", "tp_all_gather_seq_bwd"]:
        assert must in names


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) >= 25
    out = subprocess.run(["nm", "-D", "--defined-only", tp.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\sT\s(tp_\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        assert hasattr(tp.lib, n)


def _create(h, f, H, p, dtype=1, act=1, partial=None):
    ptr = ctypes.c_void_p()
    st = tp.lib.tp_plan_create(h, f, H, p, dtype, act, dtype if partial is None else partial,
                               ctypes.byref(ptr))
    return st, ptr


@pytest.mark.parametrize("args,status,needle", [
    ((4096, 11008, 32, 0), 1, "p = 0"),
    ((4096, 11008, 32, 17), 1, "p = 17"),
    ((4100, 11008, 32, 8), 2, "hidden"),
    ((4096, 11008, 20, 8), 2, "heads = 20"),      # the 20-heads-on-TP8 case of the walkthrough §6.1
    ((4096, 11010, 32, 8), 2, "ffn"),
    ((4096, 11008, 48, 8), 2, "hidden = 4096 is not divisible by heads = 48"),
    ((0, 11008, 32, 8), 1, "hidden"),
])
def test_plan_create_divisibility(args, status, needle):
    st, ptr = _create(*args)
    assert st == status
    assert not ptr.value
    assert needle in tp.last_error()


def test_plan_partial_dtype():
    """Partials are stored in the plan dtype or in fp32; fp32 plans take fp32."""
    st, ptr = _create(4096, 11008, 32, 8, dtype=1, partial=0)   # bf16 plan, fp32 partials
    assert st == 0 and ptr.value
    tp.lib.tp_plan_destroy(ptr)
    st, ptr = _create(4096, 11008, 32, 8, dtype=0, partial=1)   # fp32 plan, bf16 partials
    assert st == 4 and not ptr.value
    assert "partial dtype" in tp.last_error()
    st, ptr = _create(4096, 11008, 32, 8, dtype=1, partial=7)
    assert st == 4 and not ptr.value
    p = tp.Plan(4096, 11008, 32, 8, "bf16", "swiglu", partial_dtype="f32")
    assert "partials=f32" in p.describe()
    assert p.partial_torch_dtype == torch.float32


def test_plan_describe_prints_shard_shapes():
    p = tp.Plan(4096, 11008, 32, 8, "bf16", "swiglu")
    d = p.describe()
    assert "[2752, 4096] = [G_i; U_i]" in d
    assert "W2_i: [4096, 1376]" in d
    assert "4 heads x 128" in d


FAKE = 0x10000  # 16-byte aligned, never dereferenced (every call below stops before launch)


def _arr(vals):
    return (ctypes.c_void_p * len(vals))(*vals)


@pytest.fixture()
def plan():
    p = tp.Plan(256, 512, 4, 2, "bf16", "gelu")
    yield p
    p.close()


def test_column_fwd_rejects_null_and_misaligned(plan):
    L, h = tp.lib, plan.handle
    W = _arr([FAKE, FAKE])
    H = _arr([FAKE, FAKE])
    assert L.tp_column_fwd(h, 0, 64, None, W, None, None, H, None) == 1           # X NULL
    assert "X is NULL" in tp.last_error()
    assert L.tp_column_fwd(h, 0, 64, FAKE + 2, W, None, None, H, None) == 3      # misaligned X
    assert L.tp_column_fwd(h, 0, 64, FAKE, _arr([FAKE, 0]), None, None, H, None) == 1
    assert "W[1] is NULL" in tp.last_error()
    assert L.tp_column_fwd(h, 0, 64, FAKE, W, None, None, _arr([FAKE, FAKE + 8]), None) == 3
    assert L.tp_column_fwd(h, 0, -1, FAKE, W, None, None, H, None) == 1           # negative T
    assert L.tp_column_fwd(h, 1, 64, FAKE, W, None, _arr([FAKE, FAKE]), H, None) == 1  # Z with no activation
    assert L.tp_column_fwd(h, 2, 64, FAKE, W, None, None, H, None) == 1           # outproj is not column
    assert L.tp_column_fwd(None, 0, 64, FAKE, W, None, None, H, None) == 1


def test_zero_tokens_is_a_no_op(plan):
    L, h = tp.lib, plan.handle
    W = _arr([FAKE, FAKE])
    assert L.tp_column_fwd(h, 0, 0, FAKE, W, None, None, _arr([FAKE, FAKE]), None) == 0
    assert L.tp_row_fwd_partial(h, 0, 0, W, W, W, None) == 0
    assert L.tp_reduce_partials(h, 0, 2, W, None, None, FAKE, None) == 0
    assert L.tp_all_gather_seq(h, 0, 2, W, FAKE, None) == 0
    assert L.tp_row_bwd(h, 0, 0, FAKE, W, W, W, W, None, None, None) == 0
    assert L.tp_column_bwd(h, 0, 0, FAKE, W, W, None, None, None, None) == 0


def test_reduce_and_sequence_calls_validate(plan):
    L, h = tp.lib, plan.handle
    P = _arr([FAKE, FAKE])
    assert L.tp_reduce_partials(h, 64, 0, P, None, None, FAKE, None) == 1          # n = 0
    assert L.tp_reduce_partials(h, 64, 17, P, None, None, FAKE, None) == 1         # n > max
    assert L.tp_reduce_partials(h, 64, 2, P, FAKE + 4, None, FAKE, None) == 3      # bias misaligned
    assert L.tp_reduce_scatter_seq(h, 63, 2, P, None, None, P, None) == 2          # T % n
    assert "not divisible" in tp.last_error()
    assert L.tp_all_gather_seq(h, 63, 2, P, FAKE, None) == 2
    assert L.tp_all_gather_seq(h, 64, 2, _arr([FAKE, 0]), FAKE, None) == 1


def test_row_width_must_be_16_bytes():
    p = tp.Plan(256, 24, 0, 2, "bf16", "gelu")  # ffn/p = 12 bf16 = 24 bytes per row
    W = _arr([FAKE, FAKE])
    assert tp.lib.tp_column_fwd(p.handle, 0, 64, FAKE, W, None, None, W, None) == 3
    assert "16 bytes" in tp.last_error()


def test_plan_without_attention_rejects_attention_calls():
    p = tp.Plan(256, 512, 0, 2, "bf16", "gelu")
    A = _arr([FAKE, FAKE])
    assert tp.lib.tp_attention_fwd(p.handle, 2, 64, A, A, None, None) == 1
    assert tp.lib.tp_column_fwd(p.handle, 1, 64, FAKE, A, None, None, A, None) == 1


def test_swiglu_rejects_column_bias():
    p = tp.Plan(256, 512, 0, 2, "bf16", "swiglu")
    A = _arr([FAKE, FAKE])
    assert tp.lib.tp_column_fwd(p.handle, 0, 64, FAKE, A, A, None, A, None) == 1
    assert "SwiGLU" in tp.last_error()


def test_device_status_without_a_device_is_a_host_error():
    """With no usable GPU the status read fails on the host (TP_ERR_NO_DEVICE or
    TP_ERR_CUDA), never with one of the device-reported codes."""
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    st = tp.lib.tp_get_device_status(None, None)
    assert st in (6, 8)
    with pytest.raises(tp.TPError):
        tp.device_status()


def test_selftest_wait_limit_is_validated_before_launch():
    assert tp.lib.tp_selftest_wait_timeout(0, None, None) == 1
    assert tp.lib.tp_selftest_wait_timeout(2_000_000_000, None, None) == 1
    assert "limit_ns" in tp.last_error()
    assert tp.lib.tp_selftest_wait_timeout(1000, FAKE + 2, None) == 3


def test_status_strings():
    for i, name in enumerate(tp.STATUS):
        assert tp.lib.tp_status_string(i).decode() == name


def test_binding_raises_tperror():
    with pytest.raises(tp.TPError) as e:
        tp.Plan(4096, 11008, 20, 8)
    assert e.value.status_name == "TP_ERR_DIVISIBILITY"


def test_vocab_padding_on_the_plan():
    p = tp.Plan(4096, 0, 0, 8, "bf16", "none")
    assert p.set_vocab(32000) == 32000
    assert p.set_vocab(32001) == 32064
    assert "vocab 32001 padded to 32064" in p.describe()
    q = tp.Plan(384, 0, 0, 3, "bf16", "none")
    assert q.set_vocab(100) == 120
    with pytest.raises(tp.TPError):
        q.set_vocab(0)


@pytest.mark.parametrize("dtype,hidden", [("bf16", 1004), ("bf16", 16392), ("f32", 16384)])
def test_layernorm_row_limits(dtype, hidden):
    """LayerNorm rows: hidden a multiple of 8 and at most 16384 bf16 / 8192 fp32
    columns; anything else is TP_ERR_UNSUPPORTED before any launch."""
    p = tp.Plan(hidden, 0, 0, 1, dtype, "none")
    try:
        L, h = tp.lib, p.handle
        assert L.tp_layernorm_fwd(h, 4, FAKE, FAKE, FAKE, FAKE, None, None, None) == 5
        assert L.tp_layernorm_all_gather_seq(h, 4, 1, _arr([FAKE]), FAKE, FAKE, FAKE, None, None, None) == 5
    finally:
        p.close()


def test_peer_calls_validate_before_any_launch(plan):
    """The peer-memory steps check the group, the sizes and the pointers on
    the host (no device needed for these errors)."""
    L, h = tp.lib, plan.handle
    W = _arr([FAKE, FAKE])
    ok = tp.peer_group(2, 1, 64 * 256, [FAKE, FAKE + 4096], [FAKE + 256, FAKE + 8192])
    assert L.tp_peer_reduce(None, 64, 256, None, None, 1, _arr([FAKE]), 1, None) == 1
    bad = tp.peer_group(2, 2, 64 * 256, [FAKE, FAKE], [FAKE, FAKE])      # rank outside [0, world)
    assert L.tp_peer_reduce(ctypes.byref(bad), 64, 256, None, None, 1, _arr([FAKE]), 1, None) == 1
    bad = tp.peer_group(2, 0, 64 * 256, [FAKE, 0], [FAKE, FAKE])         # a NULL flag pointer
    assert L.tp_peer_wait(ctypes.byref(bad), 1, None) == 1
    bad = tp.peer_group(2, 0, 64 * 256, [FAKE, FAKE + 8], [FAKE, FAKE])  # misaligned flags
    assert L.tp_peer_wait(ctypes.byref(bad), 1, None) == 3
    assert L.tp_peer_reduce(ctypes.byref(ok), 63, 256, None, None, 1, _arr([FAKE]), 1, None) == 2   # T % world
    assert L.tp_peer_reduce(ctypes.byref(ok), 128, 256, None, None, 1, _arr([FAKE]), 1, None) == 1  # capacity
    assert "exceeds the receive buffers" in tp.last_error()
    assert L.tp_peer_reduce(ctypes.byref(ok), 64, 100, None, None, 1, _arr([FAKE]), 1, None) == 3   # hidden % 8
    assert L.tp_peer_reduce(ctypes.byref(ok), 64, 256, None, None, 0, _arr([FAKE]), 1, None) == 1   # n_out
    assert L.tp_peer_reduce(ctypes.byref(ok), 64, 256, FAKE + 2, None, 1, _arr([FAKE]), 1, None) == 3
    assert L.tp_row_fwd_push_peer(h, 0, 63, W, W, ctypes.byref(ok), 1, None) == 2
    assert L.tp_row_fwd_push_peer(h, 0, 64, W, W, None, 1, None) == 1
    assert L.tp_column_bwd_push_peer(h, 0, 128, FAKE, W, W, None, None, ctypes.byref(ok), 1, None) == 1
    f32 = tp.Plan(256, 512, 0, 2, "f32", "gelu")
    try:
        assert L.tp_row_fwd_push_peer(f32.handle, 0, 64, W, W, ctypes.byref(ok), 1, None) == 4
    finally:
        f32.close()
    assert L.tp_peer_set_wait_limit(-5) == 1
    assert L.tp_peer_set_wait_limit(61 * 10**9) == 1
    assert L.tp_peer_set_wait_limit(0) == 0
    with pytest.raises(ValueError):
        tp.peer_open(b"short")
    assert L.tp_peer_alloc(0, ctypes.byref(ctypes.c_void_p()), ctypes.create_string_buffer(64)) == 1


def test_peer_all_gather_calls_validate(plan):
    L, h = tp.lib, plan.handle
    ok = tp.peer_group(2, 0, 64 * 256, [FAKE, FAKE + 4096], [FAKE + 256, FAKE + 8192])
    assert L.tp_all_gather_push_peer(None, 8, 256, FAKE, _arr([FAKE, FAKE]), 1, None) == 1
    assert L.tp_all_gather_push_peer(ctypes.byref(ok), 8, 100, FAKE, _arr([FAKE, FAKE]), 1, None) == 3
    assert L.tp_all_gather_push_peer(ctypes.byref(ok), 8, 256, FAKE, _arr([FAKE, 0]), 1, None) == 1
    assert L.tp_all_gather_push_peer(ctypes.byref(ok), -1, 256, FAKE, _arr([FAKE, FAKE]), 1, None) == 1
    assert L.tp_layernorm_all_gather_push_peer(h, ctypes.byref(ok), 8, FAKE, FAKE, FAKE,
                                               _arr([FAKE, FAKE + 2]), None, None, 1, None) == 3
    assert L.tp_layernorm_all_gather_push_peer(h, None, 8, FAKE, FAKE, FAKE,
                                               _arr([FAKE, FAKE]), None, None, 1, None) == 1


def test_wgrad_grouping_calls_validate(plan):
    L = tp.lib
    assert L.tp_set_wgrad_grouping(None, 1) == 1
    assert L.tp_flush_wgrad(None) == 1
    assert L.tp_set_wgrad_grouping(plan.handle, 1) == 0
    assert L.tp_flush_wgrad(plan.handle) == 0          # nothing waits: no device call
    assert L.tp_set_wgrad_grouping(plan.handle, 0) == 0


def test_static_column_sum_validates_before_any_device_call():
    """The allocation-free column sum rejects bad arguments on the host, and
    column counts beyond its fixed scratch (512 Ki floats) with a clear error."""
    f = tp.lib.tp_column_sum_static
    assert f(4, 8, 7, FAKE, FAKE, 0, None) == 4                 # unknown dtype
    assert f(-1, 8, 1, FAKE, FAKE, 0, None) == 1                # rows < 0
    assert f(4, 0, 1, FAKE, FAKE, 0, None) == 1                 # cols = 0
    assert f(4, 524288 + 8, 1, FAKE, FAKE, 0, None) == 5        # beyond the static scratch
    assert "524288" in tp.last_error()
    assert f(4, 8, 1, None, FAKE, 0, None) == 1                 # x NULL with rows > 0
    assert f(4, 8, 1, FAKE, None, 0, None) == 1                 # out NULL
    assert f(4, 8, 1, FAKE + 2, FAKE, 0, None) == 3             # x not 16-byte aligned
    assert f(4, 12, 1, FAKE, FAKE, 0, None) == 3                # a bf16 row of 24 bytes
    if not torch.cuda.is_available():
        # valid arguments reach the device lookup, which fails on the host
        assert f(4, 8, 1, FAKE, FAKE, 0, None) in (6, 8)
