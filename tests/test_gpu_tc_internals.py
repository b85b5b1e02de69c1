"""White-box check of the tensor-core prefill's phase A: the bf16 operand images it leaves in the
workspace (swizzled shared-memory layout) are decoded here and compared with an fp64 numpy
evaluation of their definitions -- W = T (k e^g), Uv = T v, Q' = q e^g - P W, O0 = P Uv,
Kd = k e^{g_last - g} and e^{g_last}, with T = (I + A)^{-1} diag(beta).  Pinpoints a wrong
descriptor or layout to one product."""
import numpy as np
import pytest
import torch

from gated_delta_rule_83_b200 import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"

SLOT = dict(W=0, Q=16384, Kd=32768, Uv=49152, O0=65536, gam=81920, bytes=82432)


def sw128_off(r, c, R):
    return (c >> 6) * R * 128 + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + ((c & 7) << 1)


def decode_tile(buf, base, R, C):
    out = np.zeros((R, C), np.float32)
    raw = buf[base:base + R * C * 2]
    for r in range(R):
        for c in range(C):
            o = sw128_off(r, c, R)
            b = int(raw[o]) | (int(raw[o + 1]) << 8)
            out[r, c] = np.frombuffer(np.uint32(b << 16).tobytes(), np.float32)[0]
    return out


def bf16_to_f32(u8):
    u16 = u8.view(np.uint16).astype(np.uint32) << 16
    return u16.view(np.float32)


def expected_chunk(inp, t0, L, h):
    k = inp["k"][0, t0:t0 + L, h].double().numpy()
    q = inp["q"][0, t0:t0 + L, h].double().numpy()
    v = inp["v"][0, t0:t0 + L, h].double().numpy()
    la = inp["log_alpha"][0, t0:t0 + L, h].double().numpy()
    b = inp["beta"][0, t0:t0 + L, h].double().numpy()
    g = np.cumsum(la, axis=0)
    E = np.exp(g[:, None, :] - g[None, :, :])                    # [r, i, c]
    A = np.einsum("rc,ic,ric->ri", k, k, E) * b[:, None]
    A = np.tril(A, -1)
    P = np.tril(np.einsum("rc,ic,ric->ri", q, k, E))
    T = np.linalg.solve(np.eye(L) + A, np.diag(b))
    W = T @ (k * np.exp(g))
    Uv = T @ v
    Qg = q * np.exp(g)
    Kd = k * np.exp(g[-1] - g)
    return dict(W=W, Uv=Uv, Qp=Qg - P @ W, O0=P @ Uv, Kd=Kd, gam=np.exp(g[-1]))


def rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


def test_phase_a_images():
    import gated_delta_rule_83_b200 as kda
    w = synth.Workload("wb", "prefill", 1, 0, 2, 128, 128, "bf16", 21, s0_std=0.1)
    T = 100   # chunk 0 full, chunk 1 ragged (36 rows)
    inp = synth.prefill_inputs(w, T=T)
    d = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    nbytes = kda.workspace_size(1, T, 2, 128, 128)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=DEV)
    kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=d["S0"], workspace=ws)
    kda.check()
    buf = ws.cpu().numpy()
    H = 2
    slots0 = 256 + 256   # header + chunk table and sequence order (2N+1 ints rounded to 256 B)
    for j, (t0, L) in enumerate([(0, 64), (64, 36)]):
        for h in range(H):
            base = slots0 + (j * H + h) * SLOT["bytes"]
            ex = expected_chunk(inp, t0, L, h)
            Wg = decode_tile(buf, base + SLOT["W"], 64, 128)[:L]
            Qp = decode_tile(buf, base + SLOT["Q"], 64, 128)[:L]
            Kd = decode_tile(buf, base + SLOT["Kd"], 64, 128)[:L]
            Uv = decode_tile(buf, base + SLOT["Uv"], 64, 128)[:L]
            O0 = decode_tile(buf, base + SLOT["O0"], 64, 128)[:L]
            gam = buf[base + SLOT["gam"]:base + SLOT["gam"] + 512].copy().view(np.float32)
            errs = dict(Qp=rel(Qp, ex["Qp"]), Kd=rel(Kd, ex["Kd"]), W=rel(Wg, ex["W"]), Uv=rel(Uv, ex["Uv"]),
                        O0=rel(O0, ex["O0"]), gam=rel(gam, ex["gam"]))
            for name, e in errs.items():
                assert e < 2e-2, f"chunk {j} head {h}: {name} error {e:.3e} (all: {errs})"
