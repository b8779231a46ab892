"""The oracle's pins must catch plausible mistakes.

Each case copies one oracle source (``oracle/attention_oracle.c`` or
``oracle/fp8_oracle.c``), plants one mistake (a dropped term, a wrong sign or
index, a swapped operand, a misplaced mask boundary, a wrong rounding rule),
compiles it with the other source unchanged on the CPU and runs the matching
pin file (``tests/test_oracle_pins.py``, the backward or the FP8 pins) against
it.  The pins pass on the real oracle (that file's own run) and must fail on
every mutant.  Mistakes are chosen so that every memory access stays in
bounds.
"""
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "attention_oracle.c")
FP8_SRC = os.path.join(ROOT, "oracle", "fp8_oracle.c")

PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")
BACKWARD_PINS = os.path.join(ROOT, "tests", "test_oracle_backward_pins.py")
FP8_PINS = os.path.join(ROOT, "tests", "test_oracle_fp8_pins.py")
DECODE_PINS = os.path.join(ROOT, "tests", "test_oracle_decode_pins.py")
SPARSE_PINS = os.path.join(ROOT, "tests", "test_oracle_sparse_pins.py")

MUTANTS = {
    "mask_hides_diagonal": ("return causal ? (i + 1) : N;",
                            "return causal ? (i > 0 ? i : 1) : N;"),
    "mask_leaks_next_key": ("return causal ? (i + 1) : N;",
                            "return causal ? (i + 1 < N ? i + 2 : N) : N;"),
    "no_max_subtraction": ("double e = exp(s[j] - m);", "double e = exp(s[j]);"),
    "lse_drops_max": ("*lse = m + log(l);", "*lse = log(l);"),
    "no_normalisation": ("for (int64_t t = 0; t < d; ++t) o[t] /= l;", ""),
    "scale_dropped": ("s[j] = scale * acc;", "s[j] = acc;"),
    "scale_squared": ("s[j] = scale * acc;", "s[j] = scale * scale * acc;"),
    "keys_replaced_by_values": ("acc += qi[t] * Kh[j * d + t];",
                                "acc += qi[t] * Vh[j * d + t];"),
    "values_reversed": ("o[t] += e * V[j * d + t];",
                        "o[t] += e * V[(n - 1 - j) * d + t];"),
    "max_sign_flipped": ("if (s[j] > m) m = s[j];",
                         "if (-s[j] > m) m = -s[j];"),
    "sum_sign_flipped": ("l += e;", "l -= e;"),
}

# planted mistakes in the backward pass; each must fail a backward pin
BACKWARD_MUTANTS = {
    "bwd_D_unweighted": ("Di += pr[j] * acc;", "Di += acc;"),
    "bwd_dS_sign": ("const double dsij = pr[j] * (dp[j] - Di);",
                    "const double dsij = pr[j] * (Di - dp[j]);"),
    "bwd_dK_no_scale": ("dK[j * d + t] += scale * dsij * qi[t];",
                        "dK[j * d + t] += dsij * qi[t];"),
    "bwd_dV_uses_dP": ("dV[j * d + t] += pr[j] * doi[t];",
                       "dV[j * d + t] += dp[j] * doi[t];"),
    "bwd_dQ_uses_V": ("dQ[i * d + t] += scale * dsij * K[j * d + t];",
                      "dQ[i * d + t] += scale * dsij * V[j * d + t];"),
    "bwd_mask_leak": ("const int64_t n = visible_keys(i, N, causal);\n    const double *qi = Q + i * d, *doi",
                      "const int64_t n = causal ? (i + 1 < N ? i + 2 : N) : N;\n    const double *qi = Q + i * d, *doi"),
}

# planted mistakes in the FP8 oracle; each must fail an FP8 pin
FP8_MUTANTS = {
    "fp8_ties_away_from_even": ("else pick = (lo & 1) ? hi : lo;",
                                "else pick = hi;"),
    "fp8_subnormal_scale": ("v = ldexp((double)man, -9);",
                            "v = ldexp((double)man, -10);"),
    "fp8_signs_ignored": ("acc += x[a] * (double)s[a] * hadamard_entry(a, t);",
                          "acc += x[a] * hadamard_entry(a, t);"),
    "fp8_hadamard_or": ("(popcount_u32((uint32_t)(a & t)) & 1)",
                        "(popcount_u32((uint32_t)(a | t)) & 1)"),
    "fp8_scale_half_range": ("while (ldexp(amax, e) > E4M3_MAX) --e;",
                             "while (ldexp(amax, e) > E4M3_MAX / 2) --e;"),
    "fp8_no_probability_offset": ("const double p = offset * exp(s[c - k0] - m);",
                                  "const double p = exp(s[c - k0] - m);"),
    "fp8_offset_ignores_threshold": ("const double offset = exp2(8.0 - tau);",
                                     "const double offset = 256.0;"),
    "fp8_base_ignores_threshold": ("if (gap > tau) {", "if (gap > 0.0) {"),
    "fp8_base_never_moves": ("if (gap > tau) {", "if (gap > tau + 8.0) {"),
    "fp8_lse_offset_fixed": ("*lse = m + log(l) - (8.0 - tau) * ln2;",
                             "*lse = m + log(l) - 8.0 * ln2;"),
    "fp8_sum_of_rounded_p": ("      l += p;\n",
                             "      l += oracle_e4m3_decode(oracle_e4m3_encode((float)p));\n"),
    "fp8_no_output_rescale": ("for (int64_t t = 0; t < d; ++t) acc[t] *= alpha;", ""),
    "fp8_mask_leak": ("const int64_t kend = causal ? i + 1 : N;",
                      "const int64_t kend = causal ? (i + 2 < N ? i + 2 : N) : N;"),
    "fp8_first_q_scale_only": ("q_scale[bh * qblocks + i / q_block]",
                               "q_scale[bh * qblocks]"),
}

# planted mistakes in the decode oracle; each must fail a decode pin
DECODE_MUTANTS = {
    "decode_top_left_mask": ("return causal ? (Nk - Nq + i + 1) : Nk;",
                             "return causal ? (i + 1) : Nk;"),
    "decode_mask_one_short": ("return causal ? (Nk - Nq + i + 1) : Nk;",
                              "return causal ? (Nk - Nq + i) : Nk;"),
    "decode_keys_stride_q": ("const double *Kh = K + bh * Nk * d, *Vh = V + bh * Nk * d;\n      const double *qi = Q + r * d;\n      const int64_t n = decode_visible_keys",
                             "const double *Kh = K + bh * Nq * d, *Vh = V + bh * Nk * d;\n      const double *qi = Q + r * d;\n      const int64_t n = decode_visible_keys"),
    "decode_rows_values_from_keys": ("for (int64_t t = 0; t < d; ++t) vv[j * d + t] = bf16_bits_to_double(Vh[j * d + t]);",
                                     "for (int64_t t = 0; t < d; ++t) vv[j * d + t] = bf16_bits_to_double(Kh[j * d + t]);"),
}

# planted mistakes in the block-sparse oracle; each must fail a sparse pin
SPARSE_MUTANTS = {
    "sparse_mask_transposed": (
        "if (mrow[j / 128] == 0) continue;",
        "if (mask[(mask_per_head ? bh * T * T : 0) + (j / 128) * T + i / 128] == 0) continue;"),
    "sparse_heads_share_first_mask": (
        "const uint8_t *mrow = mask + (mask_per_head ? bh * T * T : 0) + (i / 128) * T;",
        "const uint8_t *mrow = mask + (i / 128) * T;"),
    "sparse_blocks_of_64_keys": (
        "if (mrow[j / 128] == 0) continue;",
        "if (mrow[j / 64 < T ? j / 64 : T - 1] == 0) continue;"),
    "sparse_empty_row_not_special": (
        "      if (n == 0) {\n        for (int64_t t = 0; t < d; ++t) O_out[a * d + t] = 0.0;",
        "      if (n < 0) {\n        for (int64_t t = 0; t < d; ++t) O_out[a * d + t] = 0.0;"),
    "sparse_causal_ignored": (
        "const int64_t jend = visible_keys(i, N, causal);\n      for (int64_t j = 0; j < jend; ++j) {\n        if (mrow",
        "const int64_t jend = N;\n      for (int64_t j = 0; j < jend; ++j) {\n        if (mrow"),
}


def _build_mutant(name, tmpdir):
    if name in FP8_MUTANTS:
        old, new = FP8_MUTANTS[name]
        target, other = FP8_SRC, SRC
    else:
        old, new = {**MUTANTS, **BACKWARD_MUTANTS, **DECODE_MUTANTS, **SPARSE_MUTANTS}[name]
        target, other = SRC, FP8_SRC
    src = open(target).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    path_c = os.path.join(tmpdir, f"{name}.c")
    path_so = os.path.join(tmpdir, f"{name}.so")
    with open(path_c, "w") as f:
        f.write(src.replace(old, new))
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                    path_c, other, "-o", path_so, "-lm"], check=True)
    return path_so


def _run_against(mutants, pin_file, tmp):
    procs = {}
    for name in mutants:
        so = _build_mutant(name, tmp)
        env = dict(os.environ, ORACLE_LIBRARY=so)
        procs[name] = subprocess.Popen(
            [sys.executable, "-m", "pytest", "-q", "-x", "-p",
             "no:cacheprovider", pin_file],
            cwd=ROOT, env=env, stdout=subprocess.PIPE,
            stderr=subprocess.STDOUT)
    survivors = []
    for name, p in procs.items():
        p.communicate(timeout=600)
        if p.returncode == 0:
            survivors.append(name)
    return survivors


def test_every_planted_mistake_fails_a_pin():
    with tempfile.TemporaryDirectory() as tmp:
        survivors = _run_against(MUTANTS, PINS, tmp)
        assert not survivors, f"pins did not catch: {survivors}"


def test_every_planted_backward_mistake_fails_a_backward_pin():
    with tempfile.TemporaryDirectory() as tmp:
        survivors = _run_against(BACKWARD_MUTANTS, BACKWARD_PINS, tmp)
        assert not survivors, f"backward pins did not catch: {survivors}"


def test_every_planted_fp8_mistake_fails_an_fp8_pin():
    with tempfile.TemporaryDirectory() as tmp:
        survivors = _run_against(FP8_MUTANTS, FP8_PINS, tmp)
        assert not survivors, f"FP8 pins did not catch: {survivors}"


def test_every_planted_decode_mistake_fails_a_decode_pin():
    with tempfile.TemporaryDirectory() as tmp:
        survivors = _run_against(DECODE_MUTANTS, DECODE_PINS, tmp)
        assert not survivors, f"decode pins did not catch: {survivors}"


def test_every_planted_sparse_mistake_fails_a_sparse_pin():
    with tempfile.TemporaryDirectory() as tmp:
        survivors = _run_against(SPARSE_MUTANTS, SPARSE_PINS, tmp)
        assert not survivors, f"block-sparse pins did not catch: {survivors}"
