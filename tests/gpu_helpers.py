"""Helpers shared by the GPU parity tests (device copies, tolerances)."""
import numpy as np
import torch

import oracle as O

TOL_BF16 = 2e-2   # max over rows of (max |gpu - oracle|) / (max |oracle|), bf16 storage
TOL_F32 = 1e-4    # same metric for fp32 plans


def dev(t):
    return None if t is None else t.to("cuda").contiguous()


def host(t):
    torch.cuda.synchronize()
    return O.f64(t)


def assert_close(got, ref, tol, what=""):
    err = O.max_row_rel_err(host(got) if isinstance(got, torch.Tensor) else got, ref)
    assert err <= tol, f"{what}: max row-normalised error {err:.3e} > {tol:.1e}"
    return err


def assert_bitexact(got, ref, what=""):
    g = host(got) if isinstance(got, torch.Tensor) else got
    assert g.shape == ref.shape, (g.shape, ref.shape)
    bad = np.argwhere(g != ref)
    assert bad.size == 0, f"{what}: {len(bad)} mismatches, first at {bad[0]}: {g[tuple(bad[0])]} vs {ref[tuple(bad[0])]}"
