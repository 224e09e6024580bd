"""Plant plausible mistakes in a copy of the oracle (CPU only) and check that
the pins catch every one of them: a dropped term, a wrong scale, sign or
index, a transposed operand, a wrong head mapping or layout."""
import os
import shutil
import subprocess

import pytest

import oracle
import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "moda_oracle.c")

# (name, text in the oracle, planted replacement)
MUTANTS = [
    ("seq_scale_dropped", "row[j] = scale * dot(", "row[j] = dot("),
    ("depth_scale_dropped", "row[n_seq + l] = scale * dot(", "row[n_seq + l] = dot("),
    ("depth_of_previous_token", "kd_off(b, hk, t, l0, Hk, T, L, d) : NULL;\n                const double* vd",
     "kd_off(b, hk, t > 0 ? t - 1 : 0, l0, Hk, T, L, d) : NULL;\n                const double* vd"),
    ("gqa_head_tiled", "const int hk = h / G;   /* [GQA] */", "const int hk = h % Hk;"),
    ("depth_value_dropped", "o[c] += w * Vdep[", "o[c] += 0.0 * Vdep["),
    ("lse_without_max", "*lse = m + log(Z);", "*lse = log(Z);"),
    ("bwd_ds_sign", "const double ds = p * (dot(go, v, d) - Dr[r]);\n                        for (int c = 0; c < d; ++c) dq",
     "const double ds = p * (dot(go, v, d) + Dr[r]);\n                        for (int c = 0; c < d; ++c) dq"),
    ("bwd_dkd_unscaled", "dKd[o + c] += scale * ds * q[c];", "dKd[o + c] += ds * q[c];"),
    ("bwd_dv_uses_ds", "dv[c] += p * go[c];", "dv[c] += ds * go[c];"),
    ("bwd_dk_diagonal_dropped", "for (int t = causal ? j : 0; t < T; ++t)",
     "for (int t = causal ? j + 1 : 0; t < T; ++t)"),
    ("bwd_dq_transposed_operand", "dq[c] += scale * ds * k[c];", "dq[c] += scale * ds * q[c];"),
    ("noncausal_ignored", "{ return causal ? t + 1 : T; }", "{ return t + 1; }"),
    ("depth_window_ignored", "{ return (window > 0 && window < L) ? L - window : 0; }", "{ return 0; }"),
    ("repack_layer_major_kept", "const size_t o = (((size_t)b * Hk + hk) * T + t) * L + l;",
     "const size_t o = (((size_t)b * Hk + hk) * L + l) * T + t;"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(tmp_path, name, old, new):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation anchor for {name} not unique"
    src = tmp_path / "mutant.c"
    src.write_text(text.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", str(src), "-o", str(so), "-lm"])
    lib = oracle.load_library(str(so))
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(lib)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake {name}"


# The exact worked example alone decides every mutant of the default
# (causal, full-depth) operator; the modes and the repack have their own pins.
WORKED_EXAMPLE_CATCHES = [m for m in MUTANTS if m[0] not in
                          ("noncausal_ignored", "depth_window_ignored", "repack_layer_major_kept")]


@pytest.mark.parametrize("name,old,new", WORKED_EXAMPLE_CATCHES, ids=[m[0] for m in WORKED_EXAMPLE_CATCHES])
def test_worked_example_alone_catches(tmp_path, name, old, new):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    src = tmp_path / "mutant.c"
    src.write_text(open(SRC).read().replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", str(src), "-o", str(so), "-lm"])
    lib = oracle.load_library(str(so))
    with pytest.raises(AssertionError):
        oracle_pins.pin_worked_example(lib)
