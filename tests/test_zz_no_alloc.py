"""tp_column_sum_static: column sums for callers that cannot call cudaMalloc
(for instance a framework whose caching allocator owns the device memory, or a
latency-sensitive loop that must not take cudaMalloc's implicit device
synchronisation). Its scratch is a fixed device array inside libtp.so, so it
allocates nothing. This file is collected last on purpose.

The new call is checked through the C ABI against the existing tp_column_sum
(which uses a plan's cudaMalloc'd workspace) on two calls in a row, so the
second call also shows that nothing left in the shared scratch by the first
leaks into its result."""

import pytest
import torch

import oracle as O
from gpu_helpers import assert_bitexact, assert_close, host

pytestmark = pytest.mark.gpu

TOL = 1e-4  # the column-sum tolerance used elsewhere in the suite (fp32 sums)


def _lib():
    from megatron_tensor_transformer_gemm_b200 import tp
    return tp


def _static(tp, rows, cols, x, out, accumulate=0):
    dt = tp.TP_BF16 if x.dtype == torch.bfloat16 else tp.TP_F32
    st = torch.cuda.current_stream().cuda_stream
    return tp.lib.tp_column_sum_static(rows, cols, dt, x.data_ptr(), out.data_ptr(), accumulate, st)


@pytest.mark.parametrize("rows,cols,dtype", [(32768, 4096, torch.bfloat16), (1000, 136, torch.float32),
                                             (5, 8192, torch.bfloat16)])
def test_static_scratch_column_sum_matches_workspace_version(rows, cols, dtype):
    tp = _lib()
    g = torch.Generator().manual_seed(rows + cols)
    plan = tp.Plan(cols, 0, 0, 1, "bf16" if dtype == torch.bfloat16 else "f32", "none")
    for call in range(2):
        if call == 0:
            x = torch.randint(-4, 5, (rows, cols), generator=g).to(dtype).cuda()
        else:
            x = torch.randn(rows, cols, generator=g).to(dtype).cuda()
        want = torch.empty(cols, dtype=torch.float32, device="cuda")
        got = torch.full((cols,), float("nan"), dtype=torch.float32, device="cuda")
        plan.column_sum(rows, cols, x, want)
        assert _static(tp, rows, cols, x, got) == 0, tp.last_error()
        assert_close(got[None, :], host(want)[None, :], TOL, f"call {call}")
        if call == 0:  # integer values: every sum is exact, so both agree with the definition bit for bit
            assert_bitexact(got, O.bias_grad(O.f64(x)), "static column sum")
        # accumulate mode adds to the existing contents
        assert _static(tp, rows, cols, x, got, accumulate=1) == 0, tp.last_error()
        assert_close(got[None, :], 2 * host(want)[None, :], TOL, f"call {call} accumulate")


def test_static_scratch_rejects_too_many_columns():
    tp = _lib()
    x = torch.zeros(8, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(8, dtype=torch.float32, device="cuda")
    cols = 512 * 1024 + 8
    assert tp.lib.tp_column_sum_static(1, cols, tp.TP_BF16, x.data_ptr(), out.data_ptr(), 0, None) == 5
    assert "static scratch" in tp.last_error()


def test_static_scratch_allocates_nothing_after_the_first_call():
    """After one warm-up call per shape (the first call on a device may load
    the library's module, which reserves the array), repeated calls leave the
    device's free memory unchanged: every input is allocated beforehand and no
    plan call runs inside the window."""
    tp = _lib()
    big = torch.ones(32768, 4096, dtype=torch.bfloat16, device="cuda")
    wide_cols = 512 * 1024  # the static scratch's limit: a single row split
    wide = torch.ones(8, wide_cols, dtype=torch.float32, device="cuda")
    out_big = torch.empty(4096, dtype=torch.float32, device="cuda")
    out_wide = torch.empty(wide_cols, dtype=torch.float32, device="cuda")
    calls = [(32768, 4096, big, out_big), (8, wide_cols, wide, out_wide), (0, 4096, big, out_big)]
    for rows, cols, x, out in calls:
        assert _static(tp, rows, cols, x, out) == 0, tp.last_error()
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        for rows, cols, x, out in calls[:2]:
            assert _static(tp, rows, cols, x, out) == 0, tp.last_error()
    torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info()[0]
    assert free1 == free0, f"free device memory changed by {free0 - free1} bytes"
    # the values are still the column sums (every sum of ones is exact)
    assert torch.equal(out_big, torch.full_like(out_big, 32768.0))
    assert torch.equal(out_wide, torch.full_like(out_wide, 8.0))
