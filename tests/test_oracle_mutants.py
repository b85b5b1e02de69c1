"""The pins must reject plausible mistakes.  Each case plants one mistake in a private copy of
the oracle's C source (on the CPU), builds it, and checks that at least one pin fails."""
import os
import subprocess

import pytest

import oracle as oracle_mod
from tests import test_oracle_bwd as bwd_pins
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle_mod.__file__), "kda_oracle.c")

# (name, exact text in kda_oracle.c, replacement)
MUTANTS = [
    ("seq: beta dropped from the correction",
     "S[(size_t)c * dv + j] += -b * kc * w[j] + b * kc * (double)vt[j];",
     "S[(size_t)c * dv + j] += -kc * w[j] + b * kc * (double)vt[j];"),
    ("seq: correction sign flipped",
     "S[(size_t)c * dv + j] += -b * kc * w[j] + b * kc * (double)vt[j];",
     "S[(size_t)c * dv + j] += b * kc * w[j] + b * kc * (double)vt[j];"),
    ("seq: no decay",
     "for (int j = 0; j < dv; ++j) S[(size_t)c * dv + j] *= a;\n        }\n        /* w = k^T S'",
     "for (int j = 0; j < dv; ++j) S[(size_t)c * dv + j] *= 1.0;\n        }\n        /* w = k^T S'"),
    ("seq: readout with k instead of q",
     "const double qc = (double)qt[c];\n                for (int j = 0; j < dv; ++j) o[j] += qc * S",
     "const double qc = (double)kt[c];\n                for (int j = 0; j < dv; ++j) o[j] += qc * S"),
    ("chunked: A loses its first sub-diagonal",
     "if (i < r)\n                    for (int c = 0; c < dk; ++c)\n                        acc += (double)J->k",
     "if (i + 1 < r)\n                    for (int c = 0; c < dk; ++c)\n                        acc += (double)J->k"),
    ("chunked: A gate exponent sign flipped",
     "exp(g[(size_t)r * dk + c] - g[(size_t)i * dk + c]);\n                A[",
     "exp(g[(size_t)i * dk + c] - g[(size_t)r * dk + c]);\n                A["),
    ("chunked: chunk-end decay inverted",
     "exp(glast[c] - g[(size_t)i * dk + c])",
     "exp(g[(size_t)i * dk + c] - glast[c])"),
    ("chunked: P excludes the diagonal",
     "for (int i = 0; i <= r; ++i) {\n                    double p = 0.0;",
     "for (int i = 0; i < r; ++i) {\n                    double p = 0.0;"),
    ("grouped: value head h reads q/k head h % Hk",
     "#define QKIDX(J, t, h, c) IDX3(t, (h) / ((J)->H / (J)->Hk), c, (J)->Hk, (J)->dk)",
     "#define QKIDX(J, t, h, c) IDX3(t, (h) % (J)->Hk, c, (J)->Hk, (J)->dk)"),
    ("bwd: dM loses the k dw^T term",
     "const double dm = G[(size_t)c * dv + j] + (double)kt[c] * (-b * du[j]);",
     "const double dm = G[(size_t)c * dv + j];"),
    ("bwd: dv without beta",
     "dvt[j] = b * acc;",
     "dvt[j] = acc;"),
    ("bwd: carried cotangent not decayed",
     "G[(size_t)c * dv + j] = a * dm;",
     "G[(size_t)c * dv + j] = dm;"),
    ("bwd: dq from the state before the step",
     "acc += St[(size_t)c * dv + j] * dot[j];",
     "acc += Sp[(size_t)c * dv + j] * dot[j];"),
    ("bwd: dk misses the M dw term",
     "dkt[c] = acc + acc2;",
     "dkt[c] = acc;"),
    ("bwd: recomputed segment starts one step late",
     "memcpy(seg, ck + (size_t)s * sz, sizeof(double) * sz);\n        for (int64_t t = ts; t < e; ++t) {",
     "memcpy(seg, ck + (size_t)s * sz, sizeof(double) * sz);\n        for (int64_t t = ts + 1; t < e; ++t) {"),
    ("decode: output from the decayed (pre-update) state",
     "for (int c = 0; c < dk; ++c)\n            for (int j = 0; j < dv; ++j) Sp[(size_t)c * dv + j] += (double)kp[c] * (b * d[j]);\n        if (out)",
     "if (out)"),
]


def _pins():
    return [
        lambda o: pins.test_hand_worked_example(o),
        lambda o: pins.test_beta_zero_closed_form(o, "seq"),
        lambda o: pins.test_beta_zero_closed_form(o, "chunked16"),
        lambda o: pins.test_orthonormal_write_retrieve(o, "seq"),
        lambda o: pins.test_orthonormal_write_retrieve(o, "chunked"),
        lambda o: pins.test_bruteforce_vs_seq(o, 5),
        lambda o: pins.test_chunked_vs_seq(o, 16),
        lambda o: pins.test_decode_equals_prefill(o),
        lambda o: pins.test_per_step_invariant(o),
        lambda o: pins.test_grouped_heads_equal_repeated_qk(o, "seq"),
        lambda o: bwd_pins.test_bwd_matches_finite_differences(o),
        lambda o: bwd_pins.test_bwd_single_step_closed_form(o),
    ]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_reject_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique/present: {name}"
    mut = tmp_path / "kda_oracle_mutant.c"
    mut.write_text(src.replace(old, new))
    lib = tmp_path / "libkda_oracle_mutant.so"
    subprocess.run(["gcc", "-O1", "-fPIC", "-shared", "-std=c11", "-o", str(lib), str(mut), "-lm", "-lpthread"],
                   check=True)
    oracle_mod.use_library(str(lib))
    try:
        failed = 0
        for pin in _pins():
            try:
                pin(oracle_mod)
            except AssertionError:
                failed += 1
        assert failed > 0, f"no pin rejected the mutant '{name}'"
    finally:
        oracle_mod.use_library(None)
