"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every function that
include/kda.h declares, and rejects bad arguments before launching anything."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from gated_delta_rule_83_b200 import build, kda
    build.build()
    return kda.load_library()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "kda.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(kda_\w+)\s*\(", src, flags=re.M)))


def test_options_struct_matches_header():
    """kda_options in the binding has the header's field order and size (8 ints)."""
    from gated_delta_rule_83_b200.kda import KdaOptions
    src = open(os.path.join(ROOT, "include", "kda.h")).read()
    body = re.search(r"typedef struct \{(.*?)\} kda_options;", src, flags=re.S).group(1)
    names = re.findall(r"(\w+)(?:\[\d+\])?;", body)
    assert names == [f[0] for f in KdaOptions._fields_]
    assert ctypes.sizeof(KdaOptions) == 32


def test_output_gate_struct_matches_header():
    """kda_output_gate in the binding has the header's field order and size (2 pointers, 6 ints)."""
    from gated_delta_rule_83_b200.kda import KdaOutputGate
    src = open(os.path.join(ROOT, "include", "kda.h")).read()
    body = re.search(r"typedef struct \{([^}]*)\} kda_output_gate;", src).group(1)
    names = re.findall(r"\**(\w+)(?:\[\d+\])?;", body)
    assert names == [f[0] for f in KdaOutputGate._fields_]
    assert ctypes.sizeof(KdaOutputGate) == 40


def test_header_declares_entry_points():
    names = declared_functions()
    for required in ("kda_chunk_fwd", "kda_decode_step", "kda_chunk_fwd_workspace_size", "kda_check",
                     "kda_status_string", "kda_version"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"libkda.so does not export {name}"


def test_binding_covers_the_abi():
    from gated_delta_rule_83_b200 import kda
    assert set(declared_functions()) <= set(kda.ABI)


def test_status_strings(lib):
    for code, name in [(0, b"KDA_OK"), (1, b"KDA_ERR_INVALID_ARG"), (2, b"KDA_ERR_UNSUPPORTED"),
                       (5, b"KDA_ERR_WORKSPACE"), (6, b"KDA_ERR_BAD_SEQLENS")]:
        assert lib.kda_status_string(code) == name
    assert lib.kda_status_string(99) == b"KDA_ERR_UNKNOWN"
    assert b"sm_100a" in lib.kda_version()


def _ws(lib, *args):
    n = ctypes.c_size_t(0)
    rc = lib.kda_chunk_fwd_workspace_size(*args, ctypes.byref(n))
    return rc, n.value


def test_workspace_size_rules(lib):
    rc, n = _ws(lib, 1, 32768, 32, 128, 128, 0, 0, 0)
    assert rc == 0 and n > 0
    rc2, n2 = _ws(lib, 1, 65536, 32, 128, 128, 1, 8, 0)   # varlen: bound grows with num_seqs
    assert rc2 == 0 and n2 >= 2 * n - 4096
    assert _ws(lib, 1, 256, 2, 96, 64, 0, 0, 0)[0] == 2    # dk unsupported
    assert _ws(lib, 2, 256, 2, 64, 64, 1, 2, 0)[0] == 1    # varlen needs B == 1
    assert _ws(lib, 1, -1, 2, 64, 64, 0, 0, 0)[0] == 1
    assert _ws(lib, 1, 256, 2, 64, 64, 0, 0, 7)[0] == 1    # bad dtype
    assert _ws(lib, 1, 0, 2, 64, 64, 0, 0, 1)[0] == 0      # T = 0 is valid


def test_chunk_fwd_rejects_before_launch(lib):
    fake = 0x100000  # never dereferenced: every call below fails validation first
    # null inputs
    rc = lib.kda_chunk_fwd(None, None, None, None, None, None, None, 0, None, None, 1, 64, 2, 64, 64, 1,
                           fake, 1 << 30, None)
    assert rc == 1
    # misaligned pointer
    rc = lib.kda_chunk_fwd(fake + 2, fake, fake, fake, fake, None, None, 0, fake, None, 1, 64, 2, 64, 64, 1,
                           fake, 1 << 30, None)
    assert rc == 1
    # workspace missing / too small / misaligned
    args = (fake, fake, fake, fake, fake, None, None, 0, fake, None, 1, 64, 2, 64, 64, 1)
    assert lib.kda_chunk_fwd(*args, None, 1 << 30, None) == 5
    assert lib.kda_chunk_fwd(*args, fake, 16, None) == 5
    assert lib.kda_chunk_fwd(*args, fake + 16, 1 << 30, None) == 5
    # unsupported head dims
    assert lib.kda_chunk_fwd(fake, fake, fake, fake, fake, None, None, 0, fake, None, 1, 64, 2, 32, 64, 1,
                             fake, 1 << 30, None) == 2


def test_decode_rejects_before_launch(lib):
    fake = 0x100000
    assert lib.kda_decode_step(None, fake, fake, fake, fake, fake, fake, 4, 2, 64, 64, 0, None) == 1
    assert lib.kda_decode_step(fake, fake, fake, fake, fake, fake, fake, 4, 2, 48, 64, 0, None) == 2
    assert lib.kda_decode_step(fake, fake, fake, fake, fake, fake + 4, fake, 4, 2, 64, 64, 0, None) == 1
    assert lib.kda_decode_step(fake, fake, fake, fake, fake, fake, fake, 4, 2, 64, 64, 3, None) == 1
    # N = 0 is a no-op that touches nothing
    assert lib.kda_decode_step(None, None, None, None, None, None, None, 0, 2, 64, 64, 0, None) == 0


def test_options_are_validated_before_launch(lib):
    """kda_options: num_qk_heads must divide H and the reserved words must be zero; a NULL or
    zeroed options struct behaves like the plain entry point (here: the same argument errors)."""
    from gated_delta_rule_83_b200.kda import KdaOptions
    fake = 0x100000  # never dereferenced
    args = (fake, fake, fake, fake, fake, None, None, 0, fake, None, 1, 64, 6, 64, 64, 1)
    bad_group = KdaOptions(num_qk_heads=4)          # 6 % 4 != 0
    assert lib.kda_chunk_fwd_ex(*args, ctypes.byref(bad_group), fake, 1 << 30, None) == 1
    neg = KdaOptions(num_qk_heads=-2)
    assert lib.kda_chunk_fwd_ex(*args, ctypes.byref(neg), fake, 1 << 30, None) == 1
    res = KdaOptions(num_qk_heads=3)
    res.reserved[2] = 1
    assert lib.kda_chunk_fwd_ex(*args, ctypes.byref(res), fake, 1 << 30, None) == 1
    unknown = KdaOptions(prologue=16)               # not a KDA_PROLOGUE_* bit
    assert lib.kda_chunk_fwd_ex(*args, ctypes.byref(unknown), fake, 1 << 30, None) == 1
    ok_group = KdaOptions(num_qk_heads=3, prologue=15)
    # a valid group with a missing workspace fails only on the workspace, like kda_chunk_fwd
    assert lib.kda_chunk_fwd_ex(*args, ctypes.byref(ok_group), None, 1 << 30, None) == 5
    assert lib.kda_chunk_fwd_ex(*args, None, None, 1 << 30, None) == 5
    dargs = (fake, fake, fake, fake, fake, fake, fake, 4, 6, 64, 64, 0)
    assert lib.kda_decode_step_ex(*dargs, ctypes.byref(bad_group), None) == 1
    assert lib.kda_decode_step_ex(*dargs[:6], fake + 4, *dargs[7:], ctypes.byref(ok_group), None) == 1  # misaligned out
    assert lib.kda_decode_step_ex(None, None, None, None, None, None, None, 0, 6, 64, 64, 0,
                                  ctypes.byref(ok_group), None) == 0  # N = 0: no-op


def test_gated_rmsnorm_rejects_before_launch(lib):
    fake = 0x100000
    c = ctypes.c_float
    assert lib.kda_gated_rmsnorm(fake, fake, None, fake, 10, 96, 0, c(1e-6), 0, 0, None) == 2      # d
    assert lib.kda_gated_rmsnorm(fake, fake, None, fake, 10, 128, 24, c(1e-6), 0, 0, None) == 1    # group
    assert lib.kda_gated_rmsnorm(fake, fake, None, fake, 10, 64, 128, c(1e-6), 0, 0, None) == 1    # group > d
    assert lib.kda_gated_rmsnorm(fake, fake, None, fake, 10, 128, 0, c(0.0), 0, 0, None) == 1      # eps
    assert lib.kda_gated_rmsnorm(fake, fake, None, fake, 10, 128, 0, c(1e-6), 5, 0, None) == 1     # act
    assert lib.kda_gated_rmsnorm(fake + 8, fake, None, fake, 10, 128, 0, c(1e-6), 0, 0, None) == 1  # aligned
    assert lib.kda_gated_rmsnorm(None, None, None, None, 0, 128, 0, c(1e-6), 0, 0, None) == 0      # rows = 0


def test_gated_prefill_rejects_before_launch(lib):
    """kda_chunk_fwd_gated checks every gate field before anything else is launched; a NULL gate is
    kda_chunk_fwd_ex (here: the same workspace error)."""
    from gated_delta_rule_83_b200.kda import KdaOutputGate
    fake = 0x100000  # never dereferenced
    args = (fake, fake, fake, fake, fake, None, None, 0, fake, None, 1, 64, 2, 128, 128, 0, None)

    def rc(**kw):
        g = KdaOutputGate(z=kw.pop("z", fake), weight=kw.pop("weight", None), group=kw.pop("group", 0),
                          eps=kw.pop("eps", 1e-6), act=kw.pop("act", 1))
        for i, r in enumerate(kw.pop("reserved", ())):
            g.reserved[i] = r
        return lib.kda_chunk_fwd_gated(*args, ctypes.byref(g), None, 1 << 30, None)

    assert rc(group=24) == 1          # not a power of two
    assert rc(group=256) == 1         # more than dv
    assert rc(group=4) == 1           # fewer than 8
    assert rc(eps=0.0) == 1
    assert rc(eps=-1.0) == 1
    assert rc(act=2) == 1
    assert rc(z=None) == 1            # tokens but no gate input
    assert rc(z=fake + 8) == 1        # misaligned
    assert rc(weight=fake + 4) == 1   # misaligned
    assert rc(reserved=(0, 1)) == 1
    assert rc(group=8) == 5           # a valid gate fails only on the missing workspace
    assert rc(group=128, act=0) == 5
    assert lib.kda_chunk_fwd_gated(*args, None, None, 1 << 30, None) == 5


def test_missing_library_fails_loudly(tmp_path):
    from gated_delta_rule_83_b200 import kda
    with pytest.raises(ImportError):
        kda.load_library(str(tmp_path / "libkda.so"))


def test_synth_distributions():
    """The seeded generator matches the documented distributions (host-side, small sizes)."""
    import numpy as np
    import torch
    from gated_delta_rule_83_b200 import synth
    w = synth.WORKLOADS["prefill_32k"]
    inp = synth.prefill_inputs(w, T=512, H=4)
    k = inp["k"].float()
    assert torch.allclose(k.norm(dim=-1), torch.ones(()), atol=1e-2)
    la = inp["log_alpha"].double()
    assert float(la.max()) < 0 and abs(float(la.mean()) - (-0.07)) < 0.03
    b = inp["beta"]
    assert 0 < float(b.min()) and float(b.max()) < 1 and abs(float(b.mean()) - 0.5) < 0.05
    assert abs(float(inp["S0"].std()) - 0.02) < 0.002
    lens = synth.varlen_lengths(2)
    assert len(lens) == 8 and sum(lens) == 65536 and all(1024 <= x <= 16384 for x in lens)
    assert lens == synth.varlen_lengths(2)
    # same seed -> same bits
    inp2 = synth.prefill_inputs(w, T=512, H=4)
    assert torch.equal(inp["q"], inp2["q"]) and torch.equal(inp["log_alpha"], inp2["log_alpha"])


def test_host_pipeline_rejects_before_launch(lib):
    """kda_chunk_fwd_host validates the segment length and the workspace before any CUDA call."""
    fake = 0x100000
    n = ctypes.c_size_t(0)
    assert lib.kda_chunk_fwd_host_workspace_size(1, 1000, 2, 128, 128, 0, None, 100, ctypes.byref(n)) == 1
    assert lib.kda_chunk_fwd_host_workspace_size(1, 0, 2, 128, 128, 0, None, 128, ctypes.byref(n)) == 1
    assert lib.kda_chunk_fwd_host_workspace_size(1, 1000, 2, 128, 128, 0, None, 128, ctypes.byref(n)) == 0
    assert n.value > 0
    args = (fake, fake, fake, fake, fake, None, fake, None, 1, 1000, 2, 128, 128, 0, None)
    assert lib.kda_chunk_fwd_host(*args, 96, fake, 1 << 40, None) == 1         # segment not a multiple of 64
    assert lib.kda_chunk_fwd_host(*args, 128, None, 1 << 40, None) == 5        # no workspace
    assert lib.kda_chunk_fwd_host(*args, 128, fake, 16, None) == 5             # workspace too small



def test_backward_rejects_before_launch(lib):
    """kda_chunk_bwd validates options, shapes, pointers and the workspace before any CUDA call."""
    from gated_delta_rule_83_b200.kda import KdaOptions
    fake = 0x100000
    n = ctypes.c_size_t(0)
    assert lib.kda_chunk_bwd_workspace_size(1, 256, 4, 128, 128, 0, 0, 0, None, ctypes.byref(n)) == 0
    plain = n.value
    grouped = KdaOptions(num_qk_heads=2)
    assert lib.kda_chunk_bwd_workspace_size(1, 256, 4, 128, 128, 0, 0, 0, ctypes.byref(grouped), ctypes.byref(n)) == 0
    assert n.value > plain                                     # per-value-head dq/dk buffers
    assert lib.kda_chunk_bwd_workspace_size(1, 256, 4, 96, 128, 0, 0, 0, None, ctypes.byref(n)) == 2  # dk
    bad = KdaOptions(num_qk_heads=3)                           # 4 % 3 != 0
    base = (fake, fake, fake, fake, fake, None, None, 0, fake, None, fake, fake, fake, fake, fake, None,
            1, 256, 4, 128, 128, 0)
    assert lib.kda_chunk_bwd(*base, ctypes.byref(bad), fake, 1 << 40, None) == 1
    assert lib.kda_chunk_bwd(*base, None, None, 1 << 40, None) == 5          # no workspace
    assert lib.kda_chunk_bwd(*base, None, fake, 16, None) == 5                # workspace too small
    mis = list(base)
    mis[8] = fake + 4                                                         # misaligned dout
    assert lib.kda_chunk_bwd(*mis, None, fake, 1 << 40, None) == 1
    nul = list(base)
    nul[10] = None                                                            # no dq
    assert lib.kda_chunk_bwd(*nul, None, fake, 1 << 40, None) == 1


def _noalloc_inputs(B=1, T=100, H=2, d=128, dtype=None):
    import torch
    dt = dtype or torch.bfloat16
    z = lambda *s, t=dt: torch.zeros(*s, dtype=t)
    return dict(q=z(B, T, H, d), k=z(B, T, H, d), v=z(B, T, H, d), log_alpha=z(B, T, H, d, t=torch.float32),
                beta=z(B, T, H, t=torch.float32), S0=z(B, H, d, d, t=torch.float32), out=z(B, T, H, d),
                S_final=z(B, H, d, d, t=torch.float32))


@pytest.mark.parametrize("field,bad,exc", [
    ("log_alpha", "bf16", TypeError),      # the entry point reads float gates: bf16 would overrun
    ("beta", "bf16", TypeError),
    ("S0", "bf16", TypeError),
    ("S_final", "f64", TypeError),
    ("k", "f32", TypeError),               # q/k/v/out share one dtype
    ("out", "f32", TypeError),
    ("k", "shape", ValueError),
    ("v", "shape", ValueError),
    ("log_alpha", "shape", ValueError),
    ("beta", "shape", ValueError),
    ("S0", "shape", ValueError),
    ("out", "shape", ValueError),
    ("S_final", "shape", ValueError),
    ("out", None, TypeError),              # out is required
    ("q", "cpu", ValueError),              # well-formed but not on a GPU
])
def test_noalloc_binding_rejects_bad_arguments(field, bad, exc):
    """chunk_fwd_noalloc checks dtypes and shapes before placement and before touching the
    library, so every malformed call raises here without a GPU (and without a launch on one)."""
    import torch
    import gated_delta_rule_83_b200 as m
    a = _noalloc_inputs()
    t = a[field]
    if bad == "bf16":
        a[field] = t.to(torch.bfloat16)
    elif bad == "f32":
        a[field] = t.float()
    elif bad == "f64":
        a[field] = t.double()
    elif bad == "shape":
        a[field] = t[..., :-1] if t.dim() > 1 else t[:-1]
    elif bad is None:
        a[field] = None
    with pytest.raises(exc):
        m.chunk_fwd_noalloc(a["q"], a["k"], a["v"], a["log_alpha"], a["beta"], a["S0"], a["out"], a["S_final"])


def test_noalloc_scratch_limit_boundary(lib):
    """The built-in scratch (KDA_NOALLOC_SCRATCH_BYTES) holds 25 chunks of 32 heads at bf16, d = 128:
    1,600 tokens fit, 1,664 are rejected on the host with KDA_ERR_WORKSPACE."""
    from gated_delta_rule_83_b200 import kda
    limit = kda.NOALLOC_SCRATCH_BYTES
    assert _ws(lib, 1, 1600, 32, 128, 128, 0, 0, 0)[1] <= limit
    assert _ws(lib, 1, 1664, 32, 128, 128, 0, 0, 0)[1] > limit
    fake = ctypes.c_void_p(0x100000)  # never dereferenced: the size check comes first
    rc = lib.kda_chunk_fwd_noalloc(fake, fake, fake, fake, fake, None, None, 0, fake, None, 1, 1664, 32, 128, 128, 0,
                                   None)
    assert rc == 5
