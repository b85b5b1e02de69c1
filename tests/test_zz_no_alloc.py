"""kda_chunk_fwd_noalloc: the prefill for callers that cannot allocate device memory (a host whose
memory is reserved up front by its own pool, a plugin hook that may not call cudaMalloc, a fixed
memory budget).  It runs on the library's built-in static scratch instead of a caller workspace.

This file is collected last on purpose (pytest orders files by name), so a run that stops at the
first failure has already run every other test.  It must pass in a fresh process and after the
other tests: the scratch lookup happens on the first call on the device.
"""
import ctypes

import pytest
import torch

from gated_delta_rule_83_b200 import synth
from tests.kda_testutil import TOL, np64, out_err, state_err

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


@pytest.mark.parametrize("dtype,dk,dv,T,lengths", [("bf16", 128, 128, 300, None), ("f32", 64, 64, 130, None),
                                                   ("bf16", 128, 128, None, [1, 64, 65, 130])])
def test_noalloc_matches_workspace_entry_point(dtype, dk, dv, T, lengths):
    import gated_delta_rule_83_b200 as kda
    lib = _lib()
    w = synth.Workload("noalloc", "prefill", 2, 0, 2, dk, dv, dtype, 99, s0_std=0.2)
    inp = synth.prefill_inputs(w, device=DEV, T=T, lengths=lengths)
    cu = inp["cu_seqlens"]
    ref_out, ref_S = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], S0=inp["S0"],
                                   cu_seqlens=cu)
    kda.check()
    tol_o, tol_s = TOL[dtype]
    for call in range(2):  # two calls in a row share (and reuse) the built-in scratch
        out = torch.full_like(ref_out, float("nan"))
        sf = torch.full_like(ref_S, float("nan"))
        assert _noalloc(lib, inp, out, sf, cu) == 0
        kda.check()
        assert out_err(np64(out), np64(ref_out)) <= tol_o, f"call {call}: output differs"
        assert state_err(np64(sf), np64(ref_S)) <= tol_s, f"call {call}: final state differs"


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
