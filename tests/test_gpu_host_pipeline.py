"""GPU parity of the host-pipelined prefill (``kda_chunk_fwd_host``): host inputs and outputs,
segments of the token axis copied in, computed and copied out on overlapping streams.  Segments
start on chunk boundaries and the state is carried on the device, so the results must equal, bit
for bit, one device call on the whole input; they are also checked against the fp64 oracle."""
import pytest
import torch

from gated_delta_rule_83_b200 import synth
from tests.kda_testutil import TOL, np64, oracle_prefill, out_err, state_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def kda():
    import gated_delta_rule_83_b200 as m
    return m


def pinned(inp):
    return {k_: (v_.contiguous().pin_memory() if isinstance(v_, torch.Tensor) else v_) for k_, v_ in inp.items()}


def device_call(inp, prologue=0):
    m = kda()
    d = {k_: (v_.to(DEV) if isinstance(v_, torch.Tensor) else v_) for k_, v_ in inp.items()}
    out, sf = m.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=d["S0"], prologue=prologue)
    m.check()
    return out.cpu(), sf.cpu()


@pytest.mark.parametrize("dtype,d,B,T,seg", [("bf16", 128, 2, 300, 128), ("f32", 64, 1, 200, 64),
                                              ("bf16", 128, 1, 100, 4096), ("bf16", 64, 3, 256, 64),
                                              ("f32", 128, 2, 130, 128)])
def test_host_pipeline_equals_device_call(dtype, d, B, T, seg):
    m = kda()
    w = synth.Workload("host", "prefill", B, T, 2, d, d, dtype, 51, s0_std=0.5)
    inp = synth.prefill_inputs(w)
    h = pinned(inp)
    out, sf = m.chunk_fwd_host(h["q"], h["k"], h["v"], h["log_alpha"], h["beta"], S0=h["S0"], segment_tokens=seg)
    m.check()
    o_dev, s_dev = device_call(inp)
    assert torch.equal(out, o_dev) and torch.equal(sf, s_dev)
    o_ref, s_ref = oracle_prefill(inp)
    assert out_err(np64(out), o_ref) <= TOL[dtype][0]
    assert state_err(np64(sf), s_ref) <= TOL[dtype][1]


def test_host_pipeline_with_options():
    """Grouped q/k heads, the full input prologue and bf16 gates pass through unchanged."""
    m = kda()
    g = torch.Generator().manual_seed(52)
    B, T, H, Hk, d = 2, 200, 4, 2, 128
    inp = dict(q=(torch.randn(B, T, Hk, d, generator=g) * 3).to(torch.bfloat16),
               k=(torch.randn(B, T, Hk, d, generator=g) * 0.2).to(torch.bfloat16),
               v=torch.randn(B, T, H, d, generator=g).to(torch.bfloat16),
               log_alpha=(torch.randn(B, T, H, d, generator=g) + 3).to(torch.bfloat16),
               beta=torch.randn(B, T, H, generator=g), S0=torch.randn(B, H, d, d, generator=g) * 0.3,
               cu_seqlens=None)
    h = pinned(inp)
    out, sf = m.chunk_fwd_host(h["q"], h["k"], h["v"], h["log_alpha"], h["beta"], S0=h["S0"], prologue=7,
                               segment_tokens=64)
    m.check()
    o_dev, s_dev = device_call(inp, prologue=7)
    assert torch.equal(out, o_dev) and torch.equal(sf, s_dev)


def test_host_pipeline_without_state_buffers():
    m = kda()
    w = synth.Workload("host0", "prefill", 1, 192, 2, 128, 128, "bf16", 53)
    inp = synth.prefill_inputs(w)
    h = pinned(inp)
    out, sf = m.chunk_fwd_host(h["q"], h["k"], h["v"], h["log_alpha"], h["beta"], S0=None,
                               output_final_state=False, segment_tokens=64)
    m.check()
    assert sf is None
    o_dev, _ = device_call(inp)
    assert torch.equal(out, o_dev)


def test_host_pipeline_reuses_and_releases_its_streams():
    """Calls on one stream reuse the cached copy streams and events; on a second stream they get
    their own; after release_host_resources() a call creates them again.  Every result stays
    bit-identical to the device call."""
    m = kda()
    w = synth.Workload("host_r", "prefill", 1, 320, 2, 128, 128, "bf16", 54, s0_std=0.2)
    inp = synth.prefill_inputs(w)
    h = pinned(inp)
    o_dev, s_dev = device_call(inp)
    side = torch.cuda.Stream()
    for stream in (None, None, side, None):
        out, sf = m.chunk_fwd_host(h["q"], h["k"], h["v"], h["log_alpha"], h["beta"], S0=h["S0"],
                                   segment_tokens=64, stream=stream)
        m.check()
        assert torch.equal(out, o_dev) and torch.equal(sf, s_dev)
    m.release_host_resources()
    out, sf = m.chunk_fwd_host(h["q"], h["k"], h["v"], h["log_alpha"], h["beta"], S0=h["S0"], segment_tokens=128)
    m.check()
    assert torch.equal(out, o_dev) and torch.equal(sf, s_dev)
    m.release_host_resources()
