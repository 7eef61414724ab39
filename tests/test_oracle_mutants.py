"""The pins must catch plausible mistakes in the oracle.

Each case plants one mistake in a copy of gdn_oracle.c (on the CPU, in a
temporary directory), loads the mutant in place of the real oracle and runs
every pin of test_oracle_pins.py against it.  At least one pin must fail.
"""
import ctypes
import inspect
import os
import subprocess

import pytest

from oracle import oracle as O
import tests.test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(O.__file__), "gdn_oracle.c")

# (name, original text, mutated text)
MUTANTS = [
    ("decay_after_read",  # the read uses the undecayed state
     "  for (size_t x = 0; x < (size_t)dk * dv; ++x) S[x] *= alpha;\n  for (int j = 0; j < dv; ++j) kv[j] = 0.0;\n  for (int i = 0; i < dk; ++i)\n    for (int j = 0; j < dv; ++j) kv[j] += S[(size_t)i * dv + j] * k[i];\n",
     "  for (int j = 0; j < dv; ++j) kv[j] = 0.0;\n  for (int i = 0; i < dk; ++i)\n    for (int j = 0; j < dv; ++j) kv[j] += S[(size_t)i * dv + j] * k[i];\n  for (size_t x = 0; x < (size_t)dk * dv; ++x) S[x] *= alpha;\n"),
    ("readout_transposed",  # o_i = sum_j S_ij q_j on a square state
     "    for (int j = 0; j < dv; ++j) o[j] += S[(size_t)i * dv + j] * q[i];",
     "    for (int j = 0; j < dv; ++j) o[j] += S[(size_t)j * dv + i] * q[j < dk ? j : 0];"),
    ("beta_dropped",
     "kv[j] = beta * (v[j] - kv[j]);", "kv[j] = (v[j] - kv[j]);"),
    ("delta_sign",
     "kv[j] = beta * (v[j] - kv[j]);", "kv[j] = beta * (v[j] + kv[j]);"),
    ("readout_before_write",  # o uses S' instead of S_t
     "  for (int j = 0; j < dv; ++j) kv[j] = beta * (v[j] - kv[j]);\n  for (int i = 0; i < dk; ++i)\n    for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] += k[i] * kv[j];\n  for (int j = 0; j < dv; ++j) o[j] = 0.0;\n  for (int i = 0; i < dk; ++i)\n    for (int j = 0; j < dv; ++j) o[j] += S[(size_t)i * dv + j] * q[i];\n",
     "  for (int j = 0; j < dv; ++j) kv[j] = beta * (v[j] - kv[j]);\n  for (int j = 0; j < dv; ++j) o[j] = 0.0;\n  for (int i = 0; i < dk; ++i)\n    for (int j = 0; j < dv; ++j) o[j] += S[(size_t)i * dv + j] * q[i];\n  for (int i = 0; i < dk; ++i)\n    for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] += k[i] * kv[j];\n"),
    ("gate_sign", "*g = -exp(A_log) * softplus(a + dt_bias);",
     "*g = exp(A_log) * softplus(a + dt_bias);"),
    ("gate_no_exp", "*g = -exp(A_log) * softplus(a + dt_bias);",
     "*g = -A_log * softplus(a + dt_bias);"),
    ("softplus_threshold", "  if (x > 0.0) return x + log1p(exp(-x));",
     "  if (x > 20.0) return x;\n  if (x > 0.0) return x + log1p(exp(-x));"),
    ("beta_sigmoid_sign", "static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }",
     "static double sigmoid(double x) { return 1.0 / (1.0 + exp(x)); }"),
    ("norm_no_eps", "double inv = 1.0 / sqrt(ss + 1e-6);", "double inv = 1.0 / sqrt(ss);"),
    ("scale_on_k", "load_vec(k, in_f64, (row * Hk + hk) * dk, dk, l2norm, 1.0, kt);",
     "load_vec(k, in_f64, (row * Hk + hk) * dk, dk, l2norm, scale, kt);"),
    ("gqa_modulo", "hk = hv / group;\n    double* S", "hk = hv % Hk;\n    double* S"),
    ("conv_taps_reversed",
     "    double acc = ld(conv_w, in_f64, (size_t)c * 4 + 0) * cs[c * 3 + 0] +",
     "    double acc = ld(conv_w, in_f64, (size_t)c * 4 + 3) * cs[c * 3 + 0] +"),
    ("conv_no_shift", "    cs[c * 3 + 0] = cs[c * 3 + 1];\n", "\n"),
    ("conv_prefill_shared_window",  # every sequence of the batch reads one window
     "                     conv_state + (size_t)b * Cc * 3, y + ((size_t)b * T + t) * Cc);",
     "                     conv_state, y + ((size_t)b * T + t) * Cc);"),
    ("conv_prefill_time_major",  # x read as [T, B, Cc]
     "      conv_silu_step(x, ((size_t)b * T + t) * Cc, conv_w, in_f64, Cc,",
     "      conv_silu_step(x, ((size_t)t * B + b) * Cc, conv_w, in_f64, Cc,"),
    ("bwd_read_term_dropped",  # dS' misses k dkv^T
     "            dSp[(size_t)i * dv + j] = dS[(size_t)i * dv + j] + kt[i] * dkv[j];",
     "            dSp[(size_t)i * dv + j] = dS[(size_t)i * dv + j];"),
    ("bwd_decay_missing", "          dS[x] = alpha * dSp[x];", "          dS[x] = dSp[x];"),
    ("bwd_dbeta_sign", "          dbeta += dd[j] * (vt[j] - kv[j]);",
     "          dbeta += dd[j] * (kv[j] - vt[j]);"),
    ("bwd_norm_projection_dropped",
     "  for (int i = 0; i < n; ++i) gx[i] += scale * (gy[i] / nrm - x[i] * xg / (nrm * nrm * nrm));",
     "  for (int i = 0; i < n; ++i) gx[i] += scale * (gy[i] / nrm);"),
    ("bwd2_erase_read_dropped",  # dS_bar misses e dr^T
     "              dS[(size_t)i * dv + j] += et[i] * drr[j];      /* dS_bar */",
     "              dS[(size_t)i * dv + j] += 0.0 * drr[j];      /* dS_bar */"),
    ("bwd2_decay_missing", "              dS[(size_t)i * dv + j] *= dec[i];",
     "              dS[(size_t)i * dv + j] *= 1.0;"),
    ("bwd2_erase_gate_path_dropped", "            gk[i] += de[i] * bg[i];", "            gk[i] += 0.0;"),
    ("kda_decay_dropped",  # the projection applied to S instead of D S
     "        for (int j = 0; j < dv; ++j) DS[(size_t)i * dv + j] = dec[i] * S[(size_t)i * dv + j];",
     "        for (int j = 0; j < dv; ++j) DS[(size_t)i * dv + j] = S[(size_t)i * dv + j];"),
    ("kda_write_unscaled", "          double acc = beta * kt[i] * vt[j];",
     "          double acc = kt[i] * vt[j];"),
    ("rmsnorm_mean_as_sum",  # the sum of squares not divided by d_v
     "    const double inv = 1.0 / sqrt(ss / dv + eps);",
     "    const double inv = 1.0 / sqrt(ss + eps);"),
    ("rmsnorm_eps_outside",
     "    const double inv = 1.0 / sqrt(ss / dv + eps);",
     "    const double inv = 1.0 / (sqrt(ss / dv) + eps);"),
    ("rmsnorm_gate_sigmoid",  # sigmoid(z) in place of SiLU(z)
     " * (zj * sigmoid(zj));", " * (sigmoid(zj));"),
    ("rmsnorm_weight_dropped",
     "ld(o, in_f64, (size_t)n * dv + j) * inv * ld(weight, in_f64, (size_t)j) * (zj * sigmoid(zj));",
     "ld(o, in_f64, (size_t)n * dv + j) * inv * (zj * sigmoid(zj));"),
    ("gdn2_decay_value_side",
     "        for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= dec[i];",
     "        for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= dec[j < dk ? j : 0];"),
    ("gdn2_erase_unscaled", "        et[i] = bi_ * kt[i];", "        et[i] = kt[i];"),
    ("gdn2_write_ungated", "        zt[j] = wj * vt[j];", "        zt[j] = vt[j];"),
]

PIN_TESTS = [(n, f) for n, f in inspect.getmembers(pins, inspect.isfunction)
             if n.startswith("test_")]


def _build_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    mutated = src.replace(old, new)
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"lib{name}.so"
    c.write_text(mutated)
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-w", "-o",
                    str(so), str(c), "-lm"], check=True)
    return str(so)


def _run_pins_against(lib_path):
    """Run every pin with the oracle's library swapped for lib_path; count failures."""
    real = O._load()
    mutant = ctypes.CDLL(lib_path)
    for fname in ("oracle_gdn_fwd", "oracle_gate_prep", "oracle_conv_step",
                  "oracle_conv_prefill", "oracle_rmsnorm_gated", "oracle_kda_fwd",
                  "oracle_gdn_bwd", "oracle_gdn2_bwd",
                  "oracle_gdn_decode_step",
                  "oracle_gdn2_fwd"):
        getattr(mutant, fname).argtypes = getattr(real, fname).argtypes
        getattr(mutant, fname).restype = ctypes.c_int
    mutant.oracle_max_threads.restype = ctypes.c_int
    failed = []
    O._lib = mutant
    try:
        for n, f in PIN_TESTS:
            params = inspect.signature(f).parameters
            marks = getattr(f, "pytestmark", [])
            argsets = [{}]
            for m in marks:
                if m.name == "parametrize":
                    names = [s.strip() for s in m.args[0].split(",")]
                    argsets = [dict(zip(names, v if isinstance(v, tuple) else (v,)))
                               for v in m.args[1]]
            assert all(set(a) == set(params) for a in argsets), n
            for a in argsets:
                try:
                    f(**a)
                except Exception:  # noqa: BLE001 - any failure counts as caught
                    failed.append(n)
                    break
    finally:
        O._lib = real
    return failed


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, old, new):
    lib = _build_mutant(tmp_path, name, old, new)
    failed = _run_pins_against(lib)
    assert failed, f"no pin caught the planted mistake '{name}'"


def test_unmutated_copy_passes_all_pins(tmp_path):
    lib = _build_mutant(tmp_path, "identity", "#include <math.h>", "#include <math.h>")
    assert _run_pins_against(lib) == []
