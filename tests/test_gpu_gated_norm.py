"""GPU parity of kda_gated_rmsnorm (the output gate: grouped RMS norm times act(z)) against the fp64
oracle on the same input bits."""
import numpy as np
import pytest
import torch

import oracle
from tests.kda_testutil import np64

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = {"bf16": 1e-2, "f32": 2e-6}   # max-abs error / max |y| (bf16 output: one rounding, 2^-8)


def kda():
    import gated_delta_rule_83_b200 as m
    return m


def case(dtype, rows, d, seed):
    g = torch.Generator().manual_seed(seed)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    o = (torch.randn(rows, d, generator=g) * 3.0).to(dt)
    z = torch.randn(rows, d, generator=g).to(dt)
    w = torch.rand(d, generator=g) + 0.5
    return o, z, w


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("group", [0, 8, 32, 64])
@pytest.mark.parametrize("gate", ["none", "sigmoid"])
def test_gated_rmsnorm_matches_oracle(dtype, d, group, gate):
    m = kda()
    o, z, w = case(dtype, 1000, d, seed=d + group)
    use_w = group in (0, 32)
    y = m.gated_rmsnorm(o.to(DEV), z.to(DEV), weight=w.to(DEV) if use_w else None, group=group, gate=gate)
    m.check()
    ref = oracle.gated_rmsnorm(np64(o), np64(z), weight=w.numpy() if use_w else None,
                               group=None if group == 0 else group, eps=1e-6, gate=gate)
    err = np.max(np.abs(np64(y) - ref)) / np.max(np.abs(ref))
    assert err <= TOL[dtype], f"error {err:.3e}"


@pytest.mark.parametrize("rows", [1, 3, 37])
def test_gated_rmsnorm_ragged_rows_and_in_place(rows):
    m = kda()
    o, z, w = case("bf16", rows, 128, seed=rows)
    ref = oracle.gated_rmsnorm(np64(o), np64(z), weight=w.numpy(), gate="sigmoid")
    od = o.to(DEV)
    guard = torch.full((64,), 7, dtype=torch.bfloat16, device=DEV)
    buf = torch.cat([od.reshape(-1), guard])           # canary right after the last row
    y = m.gated_rmsnorm(buf[:rows * 128].view(rows, 128), z.to(DEV), weight=w.to(DEV), gate="sigmoid",
                        out=buf[:rows * 128].view(rows, 128))
    m.check()
    err = np.max(np.abs(np64(y) - ref)) / np.max(np.abs(ref))
    assert err <= TOL["bf16"]
    assert torch.all(buf[rows * 128:] == 7)            # nothing written past the rows


def test_gated_rmsnorm_after_prefill_layout():
    """Applied to a [B, T, H, dv] prefill output with a gate of the same layout."""
    m = kda()
    o, z, _ = case("bf16", 2 * 70 * 3, 128, seed=5)
    o4, z4 = o.view(2, 70, 3, 128), z.view(2, 70, 3, 128)
    y = m.gated_rmsnorm(o4.to(DEV), z4.to(DEV), gate="sigmoid")
    m.check()
    assert y.shape == o4.shape
    ref = oracle.gated_rmsnorm(np64(o4), np64(z4), gate="sigmoid")
    assert np.max(np.abs(np64(y) - ref)) / np.max(np.abs(ref)) <= TOL["bf16"]
