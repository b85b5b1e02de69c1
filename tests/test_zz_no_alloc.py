"""kda_chunk_fwd_noalloc: the prefill for callers that cannot allocate device memory (a host whose
memory is reserved up front by its own pool, a plugin hook that may not call cudaMalloc, a fixed
memory budget).  It runs on the library's built-in static scratch instead of a caller workspace.

This file is collected last on purpose (pytest orders files by name), so a run that stops at the
first failure has already run every other test.  It must pass in a fresh process and after the
other tests: the scratch address is looked up on the device current at each call.
"""
import ctypes

import pytest
import torch

from gated_delta_rule_83_b200 import synth
from tests.kda_testutil import TOL, np64, oracle_prefill, out_err, state_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _lib():
    from gated_delta_rule_83_b200 import kda
    return kda.load_library()


def _noalloc(lib, d, out, sf, cu=None):
    B, T, H, dk = d["q"].shape
    dv = d["v"].shape[-1]
    N = B if cu is None else cu.numel() - 1
    dt = 0 if d["q"].dtype == torch.bfloat16 else 1
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    return lib.kda_chunk_fwd_noalloc(p(d["q"]), p(d["k"]), p(d["v"]), p(d["log_alpha"]), p(d["beta"]), p(d["S0"]),
                                     p(cu), N, p(out), p(sf), B, T, H, dk, dv, dt,
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


CASES = [("bf16", 128, 128, 300, None), ("f32", 64, 64, 130, None), ("bf16", 128, 128, None, [1, 64, 65, 130])]


@pytest.mark.parametrize("dtype,dk,dv,T,lengths", CASES)
def test_noalloc_matches_workspace_entry_point(dtype, dk, dv, T, lengths):
    """Same kernels on the same inputs: the C entry point's results equal the workspace entry
    point's bit for bit, on two calls in a row (the second reuses the scratch the first left)."""
    import gated_delta_rule_83_b200 as kda
    lib = _lib()
    w = synth.Workload("noalloc", "prefill", 2, 0, 2, dk, dv, dtype, 99, s0_std=0.2)
    inp = synth.prefill_inputs(w, device=DEV, T=T, lengths=lengths)
    cu = inp["cu_seqlens"]
    ref_out, ref_S = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], S0=inp["S0"],
                                   cu_seqlens=cu)
    kda.check()
    for call in range(2):
        out = torch.full_like(ref_out, float("nan"))
        sf = torch.full_like(ref_S, float("nan"))
        assert _noalloc(lib, inp, out, sf, cu) == 0
        kda.check()
        assert torch.equal(out, ref_out), f"call {call}: output differs from kda_chunk_fwd"
        assert torch.equal(sf, ref_S), f"call {call}: final state differs from kda_chunk_fwd"


@pytest.mark.parametrize("dtype,dk,dv,T,lengths", CASES[::2])
def test_noalloc_against_oracle(dtype, dk, dv, T, lengths):
    """The binding (kda.chunk_fwd_noalloc) against the fp64 oracle at the operator's tolerances."""
    import gated_delta_rule_83_b200 as kda
    w = synth.Workload("noalloc", "prefill", 2, 0, 2, dk, dv, dtype, 98, s0_std=0.2)
    inp = synth.prefill_inputs(w, T=T, lengths=lengths)
    d = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    out = torch.empty(d["v"].shape, dtype=d["q"].dtype, device=DEV)
    sf = torch.empty_like(d["S0"])
    for _ in range(2):
        kda.chunk_fwd_noalloc(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], out, sf,
                              cu_seqlens=d["cu_seqlens"])
        kda.check()
        o_ref, s_ref = oracle_prefill(inp)
        tol_o, tol_s = TOL[dtype]
        assert out_err(np64(out), o_ref) <= tol_o
        assert state_err(np64(sf), s_ref) <= tol_s


def test_noalloc_binding_rejects_bf16_gates_on_gpu():
    import gated_delta_rule_83_b200 as kda
    w = synth.Workload("noalloc", "prefill", 1, 128, 2, 128, 128, "bf16", 97, s0_std=0.2)
    d = synth.prefill_inputs(w, device=DEV)
    out = torch.empty(d["v"].shape, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(TypeError):
        kda.chunk_fwd_noalloc(d["q"], d["k"], d["v"], d["log_alpha"].to(torch.bfloat16), d["beta"], d["S0"], out,
                              None)


def test_noalloc_rejects_problems_beyond_its_scratch():
    import gated_delta_rule_83_b200 as kda
    lib = _lib()
    limit = kda.kda.NOALLOC_SCRATCH_BYTES
    T = 1 << 16
    assert kda.workspace_size(1, T, 32, 128, 128) > limit
    fake = ctypes.c_void_p(0x100000)  # rejected on the host before anything is launched
    rc = lib.kda_chunk_fwd_noalloc(fake, fake, fake, fake, fake, None, None, 0, fake, None, 1, T, 32, 128, 128, 0,
                                   None)
    assert rc == 5  # KDA_ERR_WORKSPACE
