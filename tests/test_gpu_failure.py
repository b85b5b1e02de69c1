"""Failure detection without a GPU fault: a bounded device wait that gives up reports
KDA_ERR_TIMEOUT through the device error word, and the context stays usable afterwards."""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    import gated_delta_rule_83_b200 as kda
    from gated_delta_rule_83_b200 import synth
    lib = kda.load_library()
    kda.check()  # start from a clean error word
    assert lib.kda_selftest_timeout(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0
    with pytest.raises(kda.KdaError) as ei:
        kda.check()
    assert ei.value.code == 4  # KDA_ERR_TIMEOUT
    kda.check()  # cleared
    # the context still runs the operator correctly afterwards
    w = synth.Workload("t", "prefill", 1, 0, 2, 128, 128, "bf16", 3, s0_std=0.1)
    inp = synth.prefill_inputs(w, T=70, device="cuda")
    out, sf = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], S0=inp["S0"])
    kda.check()
    assert torch.isfinite(out.float()).all() and torch.isfinite(sf).all()
