"""GPU parity of the HBM kernels: sharding copies, reduce of the partials,
reduce-scatter / all-gather along the sequence, column sums, LayerNorm.
Integer-valued inputs make every sum exact, so those comparisons are bit for bit."""
import numpy as np
import pytest
import torch

import oracle as O
import tp_synth
from gpu_helpers import TOL_BF16, TOL_F32, assert_bitexact, assert_close, dev, host

pytestmark = pytest.mark.gpu


def _tp():
    from megatron_tensor_transformer_gemm_b200 import tp
    return tp


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("p", [1, 2, 3, 8, 16])
@pytest.mark.parametrize("T,h", [(1000, 136), (64, 4096), (1, 8)])
def test_reduce_partials_bitexact(dtype, p, T, h):
    tp = _tp()
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    if h * (2 if dtype == "bf16" else 4) % 16:
        pytest.skip("row not 16-byte aligned")
    P, b, r = tp_synth.draw_partials(p, T, h, tdt, seed=p, integer_valued=True, residual=True)
    plan = tp.Plan(h, 0, 0, 1, dtype, "none")
    Pd = [dev(x) for x in P]
    Y = torch.empty(T, h, dtype=tdt, device="cuda")
    plan.reduce_partials(T, Pd, dev(b), dev(r), Y)
    assert_bitexact(Y, O.reduce_partials([O.f64(x) for x in P], O.f64(b), O.f64(r)), "reduce")
    # no bias, no residual
    plan.reduce_partials(T, Pd, None, None, Y)
    assert_bitexact(Y, O.reduce_partials([O.f64(x) for x in P]), "reduce/no-bias")


@pytest.mark.parametrize("p", [2, 8])
def test_reduce_partials_random_within_tolerance(p):
    tp = _tp()
    T, h = 777, 512
    P, b, _ = tp_synth.draw_partials(p, T, h, torch.bfloat16, seed=3)
    plan = tp.Plan(h, 0, 0, 1, "bf16", "none")
    Y = torch.empty(T, h, dtype=torch.bfloat16, device="cuda")
    plan.reduce_partials(T, [dev(x) for x in P], dev(b), None, Y)
    assert_close(Y, O.reduce_partials([O.f64(x) for x in P], O.f64(b)), TOL_BF16, "reduce")


def test_bias_added_once_on_gpu():
    tp = _tp()
    p, T, h = 8, 32, 64
    P, b, _ = tp_synth.draw_partials(p, T, h, torch.bfloat16, integer_valued=True)
    plan = tp.Plan(h, 0, 0, 1, "bf16", "none")
    Y = torch.empty(T, h, dtype=torch.bfloat16, device="cuda")
    plan.reduce_partials(T, [dev(x) for x in P], dev(b), None, Y)
    once = host(Y)
    Pf = [O.f64(x) for x in P]
    assert np.array_equal(O.reduce_partials([x + O.f64(b)[None, :] for x in Pf]) - once,
                          np.broadcast_to((p - 1) * O.f64(b), once.shape))


@pytest.mark.parametrize("n", [1, 2, 4, 8])
def test_reduce_scatter_and_all_gather_bitexact(n):
    tp = _tp()
    T, h = 96 * n, 264
    P, b, r = tp_synth.draw_partials(n, T, h, torch.bfloat16, seed=n, integer_valued=True, residual=True)
    plan = tp.Plan(h, 0, 0, 1, "bf16", "none")
    Pd = [dev(x) for x in P]
    t = T // n
    r_seq = [dev(r[j * t:(j + 1) * t]) for j in range(n)]
    Y_seq = [torch.empty(t, h, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    plan.reduce_scatter_seq(T, Pd, dev(b), r_seq, Y_seq)
    ref = O.reduce_scatter_seq([O.f64(x) for x in P], O.f64(b), [O.f64(r[j * t:(j + 1) * t]) for j in range(n)])
    for j in range(n):
        assert_bitexact(Y_seq[j], ref[j], f"RS shard {j}")
    full = torch.empty(T, h, dtype=torch.bfloat16, device="cuda")
    plan.all_gather_seq(T, Y_seq, full)
    assert_bitexact(full, O.all_gather_seq(ref), "AG")
    # AG(RS(P)) == AR(P) on the device, bit for bit
    plan.reduce_scatter_seq(T, Pd, dev(b), None, Y_seq)
    plan.all_gather_seq(T, Y_seq, full)
    Y = torch.empty(T, h, dtype=torch.bfloat16, device="cuda")
    plan.reduce_partials(T, Pd, dev(b), None, Y)
    assert torch.equal(full, Y)
    # the backward aliases
    plan.reduce_scatter_seq_bwd(T, Y_seq, full)
    assert torch.equal(full, Y)
    plan.all_gather_seq_bwd(T, Pd, Y_seq)
    ref2 = O.reduce_scatter_seq([O.f64(x) for x in P])
    for j in range(n):
        assert_bitexact(Y_seq[j], ref2[j], f"AG-bwd shard {j}")


@pytest.mark.parametrize("act", ["gelu", "swiglu"])
@pytest.mark.parametrize("p", [1, 2, 4, 8])
def test_shard_unshard_mlp_bitexact(act, p):
    tp = _tp()
    h, f = 64, 8 * 24
    inp = tp_synth.draw_mlp(4, h, f, act, torch.bfloat16, seed=p, bias=(act == "gelu"))
    plan = tp.Plan(h, f, 0, p, "bf16", act)
    W1, W2 = dev(inp.W1), dev(inp.W2)
    n1 = (2 if act == "swiglu" else 1) * f // p
    W1s = [torch.empty(n1, h, dtype=torch.bfloat16, device="cuda") for _ in range(p)]
    W2s = [torch.empty(h, f // p, dtype=torch.bfloat16, device="cuda") for _ in range(p)]
    plan.shard_column("mlp", W1, W1s)
    plan.shard_row("mlp", W2, W2s)
    w1 = O.f64(inp.W1)
    for i in range(p):
        ref = O.shard_gate_up(w1, p, i) if act == "swiglu" else O.shard_rows(w1, p, i)
        assert_bitexact(W1s[i], ref, f"column shard {i}")
        assert_bitexact(W2s[i], O.shard_cols(O.f64(inp.W2), p, i), f"row shard {i}")
    back1, back2 = torch.zeros_like(W1), torch.zeros_like(W2)
    plan.unshard_column("mlp", W1s, back1)
    plan.unshard_row("mlp", W2s, back2)
    assert torch.equal(back1, W1) and torch.equal(back2, W2)
    if act == "gelu":
        bs = [torch.empty(n1, dtype=torch.bfloat16, device="cuda") for _ in range(p)]
        plan.shard_column_bias("mlp", dev(inp.b1), bs)
        for i in range(p):
            assert_bitexact(bs[i], O.shard_vec(O.f64(inp.b1), p, i), "bias shard")


@pytest.mark.parametrize("p", [1, 2, 4, 8])
def test_shard_qkv_by_heads_bitexact(p):
    tp = _tp()
    h, H = 128, 8
    a = tp_synth.draw_attn_block(1, 4, h, torch.bfloat16, bias=True)
    plan = tp.Plan(h, 0, H, p, "bf16", "none")
    Ws = [torch.empty(3 * h // p, h, dtype=torch.bfloat16, device="cuda") for _ in range(p)]
    bs = [torch.empty(3 * h // p, dtype=torch.bfloat16, device="cuda") for _ in range(p)]
    plan.shard_column("qkv", dev(a.Wqkv), Ws)
    plan.shard_column_bias("qkv", dev(a.bqkv), bs)
    Wo = [torch.empty(h, h // p, dtype=torch.bfloat16, device="cuda") for _ in range(p)]
    plan.shard_row("outproj", dev(a.Wo), Wo)
    for i in range(p):
        assert_bitexact(Ws[i], O.shard_qkv(O.f64(a.Wqkv), H, p, i), "qkv shard")
        assert_bitexact(bs[i], O.shard_qkv_vec(O.f64(a.bqkv), H, p, i), "qkv bias shard")
        assert_bitexact(Wo[i], O.shard_cols(O.f64(a.Wo), p, i), "out-proj shard")


@pytest.mark.parametrize("rows,cols", [(5000, 4096), (37, 136), (1, 8), (0, 64)])
def test_column_sum(rows, cols):
    tp = _tp()
    g = torch.Generator().manual_seed(rows)
    x = torch.randint(-4, 5, (rows, cols), generator=g).to(torch.bfloat16)
    plan = tp.Plan(cols, 0, 0, 1, "bf16", "none")
    out = torch.full((cols,), 7.0, dtype=torch.float32, device="cuda")
    plan.column_sum(rows, cols, dev(x), out)
    assert_bitexact(out, O.bias_grad(O.f64(x)), "column sum")  # integer sums are exact
    plan.column_sum(rows, cols, dev(x), out, accumulate=True)
    assert_bitexact(out, 2 * O.bias_grad(O.f64(x)), "column sum accumulate")


def test_column_sum_one_launch_rearms_its_counters():
    """The single-launch column sum counts each column slab's finished blocks
    on the plan's counters, and the last block sets its counter back: many
    sums of changing shapes on one plan (eager and replayed from a CUDA graph)
    must each be exact. Integer inputs make every order give the same sum."""
    tp = _tp()
    plan = tp.Plan(8, 0, 0, 1, "bf16", "none")
    shapes = [(4096, 512), (37, 8), (4096, 1536), (1000, 136), (64, 4096), (5000, 2048)]
    for rep in range(3):
        for rows, cols in shapes:
            g = torch.Generator().manual_seed(rows * 7 + cols + rep)
            x = torch.randint(-4, 5, (rows, cols), generator=g).to(torch.bfloat16)
            out = torch.empty(cols, dtype=torch.float32, device="cuda")
            plan.column_sum(rows, cols, dev(x), out)
            assert_bitexact(out, O.bias_grad(O.f64(x)), f"column sum {rows}x{cols} rep {rep}")
    rows, cols = 4096, 1536
    g = torch.Generator().manual_seed(99)
    x = dev(torch.randint(-4, 5, (rows, cols), generator=g).to(torch.bfloat16))
    out = torch.zeros(cols, dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        plan.column_sum(rows, cols, x, out, stream=s)  # first use on this stream, before capture
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=s):
            plan.column_sum(rows, cols, x, out, accumulate=True, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(4):
        gr.replay()
    torch.cuda.synchronize()
    assert_bitexact(out, 5 * O.bias_grad(O.f64(host(x))), "column sum replayed")
    # fp32 inputs take the same kernel
    xf = torch.randint(-9, 10, (3000, 264), generator=g).to(torch.float32)
    plan32 = tp.Plan(8, 0, 0, 1, "f32", "none")
    outf = torch.empty(264, dtype=torch.float32, device="cuda")
    plan32.column_sum(3000, 264, dev(xf), outf)
    assert_bitexact(outf, O.bias_grad(O.f64(xf)), "column sum fp32")


@pytest.mark.parametrize("h", [512, 4096, 8192, 136, 16384])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_layernorm_fwd_bwd(h, dtype):
    """Rows up to 16384 bf16 / 8192 fp32 columns take the one-pass staged
    backward; fp32 rows of 136 columns and below still fit it too."""
    if dtype == "f32" and h > 8192:
        pytest.skip("fp32 LayerNorm rows are limited to 8192 columns")
    tp = _tp()
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    tol = TOL_BF16 if dtype == "bf16" else TOL_F32
    rows = 300
    g = torch.Generator().manual_seed(h)
    x = (torch.randn(rows, h, generator=g) * 2 + 0.5).to(tdt)
    gamma = (1 + 0.1 * torch.randn(h, generator=g)).to(tdt)
    beta = (0.1 * torch.randn(h, generator=g)).to(tdt)
    dy = torch.randn(rows, h, generator=g).to(tdt)
    plan = tp.Plan(h, 0, 0, 1, dtype, "none")
    y = torch.empty(rows, h, dtype=tdt, device="cuda")
    mean = torch.empty(rows, dtype=torch.float32, device="cuda")
    rstd = torch.empty(rows, dtype=torch.float32, device="cuda")
    plan.layernorm_fwd(rows, dev(x), dev(gamma), dev(beta), y, mean, rstd)
    ry, rm, rr = O.layernorm_fwd(O.f64(x), O.f64(gamma), O.f64(beta))
    assert_close(y, ry, tol, "LN fwd")
    np.testing.assert_allclose(host(mean), rm, rtol=1e-5, atol=1e-5)
    np.testing.assert_allclose(host(rstd), rr, rtol=1e-4)
    dx = torch.empty_like(y)
    dg = torch.empty(h, dtype=torch.float32, device="cuda")
    db = torch.empty(h, dtype=torch.float32, device="cuda")
    plan.layernorm_bwd(rows, dev(x), dev(gamma), dev(dy), mean, rstd, dx, dg, db)
    rdx, rdg, rdb = O.layernorm_bwd(O.f64(x), O.f64(gamma), O.f64(dy), rm, rr)
    assert_close(dx, rdx, tol, "LN dx")
    assert_close(dg[None, :], rdg[None, :], 1e-3, "LN dgamma")
    assert_close(db[None, :], rdb[None, :], 1e-3, "LN dbeta")
    # accumulate: a second call adds the same parameter gradients
    plan.layernorm_bwd(rows, dev(x), dev(gamma), dev(dy), mean, rstd, dx, dg, db, accumulate=True)
    assert_close(dg[None, :], 2 * rdg[None, :], 1e-3, "LN dgamma accumulated")
    assert_close(db[None, :], 2 * rdb[None, :], 1e-3, "LN dbeta accumulated")
    # the residual branch's gradient added in the same launch, also in place (dres is dx)
    dres = torch.randn(rows, h, generator=g).to(tdt)
    plan.layernorm_bwd(rows, dev(x), dev(gamma), dev(dy), mean, rstd, dx, dg, db, dres=dev(dres))
    assert_close(dx, rdx + O.f64(dres), tol, "LN dx + dres")
    inplace = dev(dres)
    plan.layernorm_bwd(rows, dev(x), dev(gamma), dev(dy), mean, rstd, inplace, dg, db, dres=inplace)
    assert_close(inplace, rdx + O.f64(dres), tol, "LN dx + dres in place")


@pytest.mark.parametrize("n", [1, 4, 8])
def test_layernorm_all_gather_equals_gather_of_layernorm(n):
    tp = _tp()
    h, t = 1024, 40
    T = n * t
    g = torch.Generator().manual_seed(n)
    xs = [torch.randn(t, h, generator=g).to(torch.bfloat16) for _ in range(n)]
    gamma = (1 + 0.1 * torch.randn(h, generator=g)).to(torch.bfloat16)
    beta = (0.1 * torch.randn(h, generator=g)).to(torch.bfloat16)
    plan = tp.Plan(h, 0, 0, 1, "bf16", "none")
    Y = torch.empty(T, h, dtype=torch.bfloat16, device="cuda")
    mean = torch.empty(T, dtype=torch.float32, device="cuda")
    rstd = torch.empty(T, dtype=torch.float32, device="cuda")
    plan.layernorm_all_gather_seq(T, [dev(x) for x in xs], dev(gamma), dev(beta), Y, mean, rstd)
    # the fused kernel equals LN per shard followed by the gather, bit for bit
    parts = []
    for x in xs:
        y = torch.empty(t, h, dtype=torch.bfloat16, device="cuda")
        plan.layernorm_fwd(t, dev(x), dev(gamma), dev(beta), y)
        parts.append(y)
    full = torch.empty_like(Y)
    plan.all_gather_seq(T, parts, full)
    assert torch.equal(full, Y)
    ref = O.all_gather_seq([O.layernorm_fwd(O.f64(x), O.f64(gamma), O.f64(beta))[0] for x in xs])
    assert_close(Y, ref, TOL_BF16, "LN+AG")


def test_device_status_is_clean():
    tp = _tp()
    assert tp.device_status() == "TP_OK"


@pytest.mark.parametrize("p", [2, 8, 16])
@pytest.mark.parametrize("T,h", [(1000, 136), (33, 4096)])
def test_fp32_partials_reduce_bitexact(p, T, h):
    """A bf16 plan with fp32 partials: integer-valued partials (exact in both
    types) sum bit for bit, with the bias once and the residual, and the
    sequence reduce-scatter scatters the same rows."""
    tp = _tp()
    P, b, r = tp_synth.draw_partials(p, T, h, torch.float32, seed=p, integer_valued=True, residual=True)
    plan = tp.Plan(h, 0, 0, 1, "bf16", "none", partial_dtype="f32")
    Pd = [dev(x) for x in P]
    Y = torch.empty(T, h, dtype=torch.bfloat16, device="cuda")
    plan.reduce_partials(T, Pd, dev(b.bfloat16()), dev(r.bfloat16()), Y)
    ref = O.reduce_partials([O.f64(x) for x in P], O.f64(b), O.f64(r))
    assert np.abs(ref).max() < 256  # every value exact in bf16
    assert_bitexact(Y, ref, "reduce, fp32 partials")
    if T % p == 0:
        t = T // p
        outs = [torch.empty(t, h, dtype=torch.bfloat16, device="cuda") for _ in range(p)]
        plan.reduce_scatter_seq(T, Pd, dev(b.bfloat16()), None, outs)
        refs = O.reduce_scatter_seq([O.f64(x) for x in P], O.f64(b))
        for j in range(p):
            assert_bitexact(outs[j], refs[j], f"RS shard {j}, fp32 partials")


def test_fp32_partials_row_layer_against_oracle_and_bf16_partials():
    """Row GEMM partials stored in fp32 (the plan's partial dtype) and summed:
    within tolerance of the oracle, the partials themselves within the fp32
    bound, and the summed output measurably closer to the oracle than with
    bf16 partials (only the final rounding remains: RMS error about 1/sqrt(2)
    of the bf16-partials path, where each partial is rounded once more)."""
    tp = _tp()
    T, h, f, p = 512, 1024, 4096, 8
    g = torch.Generator().manual_seed(41)
    fp = f // p
    Hs = [torch.randn(T, fp, generator=g).to(torch.bfloat16) for _ in range(p)]
    W2 = (torch.randn(h, f, generator=g) * 0.02).to(torch.bfloat16)
    b2 = (torch.rand(h, generator=g) * 0.2 - 0.1).to(torch.bfloat16)
    W2f = O.f64(W2)
    parts = [O.row_partial(O.f64(Hs[i]), O.shard_cols(W2f, p, i)) for i in range(p)]
    ref = O.reduce_partials(parts, O.f64(b2))
    rms = {}
    for pd in ("bf16", "f32"):
        plan = tp.Plan(h, f, 0, p, "bf16", "gelu", partial_dtype=pd)
        Ws = [torch.empty(h, fp, dtype=torch.bfloat16, device="cuda") for _ in range(p)]
        plan.shard_row("mlp", dev(W2), Ws)
        P = [torch.empty(T, h, dtype=plan.partial_torch_dtype, device="cuda") for _ in range(p)]
        plan.row_fwd_partial("mlp", T, [dev(x) for x in Hs], Ws, P)
        if pd == "f32":
            for i in range(p):
                assert_close(P[i], parts[i], TOL_F32, f"fp32 partial {i}")
        Y = torch.empty(T, h, dtype=torch.bfloat16, device="cuda")
        plan.reduce_partials(T, P, dev(b2), None, Y)
        assert_close(Y, ref, TOL_BF16, f"Y ({pd} partials)")
        d = host(Y) - ref
        rms[pd] = float(np.sqrt((d * d).mean() / (ref * ref).mean()))
    assert rms["f32"] < 0.85 * rms["bf16"], rms


def test_fp32_partials_column_backward_dx():
    """dX partials of the column backward in fp32, reduce-scattered along the
    sequence into bf16 shards, against the oracle."""
    tp = _tp()
    T, h, f, p = 256, 512, 1024, 4
    g = torch.Generator().manual_seed(43)
    n = f // p
    W1 = (torch.randn(f, h, generator=g) * 0.05).to(torch.bfloat16)
    dZs = [torch.randn(T, n, generator=g).to(torch.bfloat16) for _ in range(p)]
    plan = tp.Plan(h, f, 0, p, "bf16", "gelu", partial_dtype="f32")
    Ws = [torch.empty(n, h, dtype=torch.bfloat16, device="cuda") for _ in range(p)]
    plan.shard_column("mlp", dev(W1), Ws)
    dXp = [torch.empty(T, h, dtype=torch.float32, device="cuda") for _ in range(p)]
    plan.column_bwd("mlp", T, None, [dev(z) for z in dZs], Ws, None, None, dXp)
    W1f = O.f64(W1)
    parts = [O.column_bwd_shard(np.zeros((T, h)), O.f64(dZs[i]), O.shard_rows(W1f, p, i))[2]
             for i in range(p)]
    for i in range(p):
        assert_close(dXp[i], parts[i], TOL_F32, f"fp32 dX partial {i}")
    t = T // p
    outs = [torch.empty(t, h, dtype=torch.bfloat16, device="cuda") for _ in range(p)]
    plan.all_gather_seq_bwd(T, dXp, outs)
    refs = O.reduce_scatter_seq(parts)
    for j in range(p):
        assert_close(outs[j], refs[j], TOL_BF16, f"dX RS shard {j}")


def test_bounded_wait_times_out_and_reports():
    """The device-side failure path: a kernel whose bounded wait (1 ms here)
    never sees its arrival gives up, returns, and the status word reads
    TP_ERR_TIMEOUT once; the next read is clean and the context still works."""
    tp = _tp()
    assert tp.device_status() == "TP_OK"
    flag = torch.zeros(4, dtype=torch.int32, device="cuda")
    tp.selftest_wait_timeout(1_000_000, flag)
    assert tp.device_status() == "TP_ERR_TIMEOUT"
    assert int(flag[0]) == 1
    assert tp.device_status() == "TP_OK"
    # the context is intact: an ordinary call still runs and is correct
    P, b, _ = tp_synth.draw_partials(2, 16, 64, torch.bfloat16, integer_valued=True)
    plan = tp.Plan(64, 0, 0, 1, "bf16", "none")
    Y = torch.empty(16, 64, dtype=torch.bfloat16, device="cuda")
    plan.reduce_partials(16, [dev(x) for x in P], dev(b), None, Y)
    assert_bitexact(Y, O.reduce_partials([O.f64(x) for x in P], O.f64(b)), "reduce after a timeout")
    assert tp.device_status(plan=plan) == "TP_OK"


@pytest.mark.parametrize("n,t,h", [(8, 600, 1032), (3, 1000, 4096), (2, 64, 8192)])
def test_all_gather_large_shards_bitexact(n, t, h):
    """The sequence all-gather of shards of 1 MB and more (600 rows x 2064
    bytes, 1000 x 8192 bytes, exactly 1 MB) is copied bit for bit."""
    tp = _tp()
    g = torch.Generator().manual_seed(n * t + h)
    xs = [torch.randn(t, h, generator=g).to(torch.bfloat16) for _ in range(n)]
    plan = tp.Plan(h, 0, 0, 1, "bf16", "none")
    out = torch.full((n * t, h), float("nan"), dtype=torch.bfloat16, device="cuda")
    plan.all_gather_seq(n * t, [dev(x) for x in xs], out)
    assert torch.equal(out.cpu(), torch.cat(xs, 0))
    assert tp.device_status() == "TP_OK"
