"""Each plausible mistake planted in a copy of the oracle must be caught by a pin.

The copy is the oracle's own C source with one textual change, compiled to a temporary
library on the CPU; the real oracle is not touched.  Every mutant keeps all memory
accesses in bounds for the shapes the pins use (square-safe index swaps are avoided).
"""
import os
import subprocess

import pytest

import oracle
import pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "nq_oracle.c")

MUTANTS = {
    "drop_s2": ("orc_f16_to_double(s2[j]) * orc_bf16_to_double(x[b * n + j]);\n\n    /* step 2",
                "orc_bf16_to_double(x[b * n + j]);\n\n    /* step 2"),
    "drop_s1": ("y[b * m + i] = si * acc;", "y[b * m + i] = acc;"),
    "sign_flip": ("& 1u) ? +1 : -1;", "& 1u) ? -1 : +1;"),
    "msb_first": ("(word >> (col % 32))", "(word >> (31 - col % 32))"),
    "pack_zero_as_minus": ("signs[row * cols + col] >= 0", "signs[row * cols + col] > 0"),
    "t_skips_last": ("acc += orc_sign_at(Vpk, wpr_v, k, j) * xs[b * n + j];",
                     "if (j + 1 < n) acc += orc_sign_at(Vpk, wpr_v, k, j) * xs[b * n + j];"),
    "bpw_no_scales": ("+ 16.0 * (double)(m + n)", "+ 0.0 * (double)(m + n)"),
    "f16_bias": ("expo - 15 - 10", "expo - 16 - 10"),
    "bf16_subnormal": ("-126 - 7", "-127 - 7"),
    "t_wrong_token": ("orc_sign_at(Vpk, wpr_v, k, j) * xs[b * n + j];", "orc_sign_at(Vpk, wpr_v, k, j) * xs[j];"),
    "y_wrong_t_index": ("acc += orc_sign_at(Upk, wpr_u, i, k) * t[b * r + k];",
                        "acc += orc_sign_at(Upk, wpr_u, i, k) * t[b * r + (k + 1) % r];"),
    "bf16_truncates": ("double q = rint(ldexp(a, 7 - E));", "double q = floor(ldexp(a, 7 - E));"),
    "bf16_no_carry": ("if (q >= 256.0) {", "if (q > 256.0) {"),
    "bf16_subnormal_quantum": ("if (E < -126) E = -126;", "if (E < -127) E = -127;"),
    "rms_sum_not_mean": ("sqrt(acc / (double)cols)", "sqrt(acc)"),
    "rms_no_sqrt": ("double rms = sqrt(acc / (double)cols);", "double rms = acc / (double)cols;"),
    "bwd_drop_s1": ("g[b * m + i] = orc_f16_to_double(s1[i]) * orc_bf16_to_double(dy[b * m + i]);",
                    "g[b * m + i] = orc_bf16_to_double(dy[b * m + i]);"),
    "bwd_s1_for_s2": ("double sj = orc_f16_to_double(s2[j]);", "double sj = orc_f16_to_double(s1[j % m]);"),
    "bwd_u_from_v": ("acc += orc_sign_at(Upk, wpr_u, i, k) * g[b * m + i];",
                     "acc += orc_sign_at(Upk, wpr_u, i % m, (k + i) % r) * g[b * m + i];"),
    "bwd_dx_wrong_u": ("acc += orc_sign_at(Vpk, wpr_v, k, j) * u[b * r + k];",
                       "acc += orc_sign_at(Vpk, wpr_v, k, j) * u[k];"),
    "scales_ds1_uses_s1": ("ds1[i] += orc_bf16_to_double(dy[b * m + i]) * z;",
                           "ds1[i] += orc_f16_to_double(s1[i]) * orc_bf16_to_double(dy[b * m + i]) * z;"),
    "scales_ds2_from_t": ("for (int64_t k = 0; k < r; ++k) w += orc_sign_at(Vpk, wpr_v, k, j) * u[b * r + k];",
                          "for (int64_t k = 0; k < r; ++k) w += orc_sign_at(Vpk, wpr_v, k, j) * t[b * r + k];"),
    "scales_u_no_s1": ("au += orc_sign_at(Upk, wpr_u, i, k) * (orc_f16_to_double(s1[i]) * orc_bf16_to_double(dy[b * m + i]));",
                       "au += orc_sign_at(Upk, wpr_u, i, k) * orc_bf16_to_double(dy[b * m + i]);"),
    "factors_dU_no_s1": ("dU[i * r + k] = si * acc;", "dU[i * r + k] = acc;"),
    "factors_dV_uses_t": ("for (int64_t b = 0; b < batch; ++b) acc += orc_bf16_to_double(x[b * n + j]) * u[b * r + k];",
                          "for (int64_t b = 0; b < batch; ++b) acc += orc_bf16_to_double(x[b * n + j]) * t[b * r + k];"),
    "envelope_first_term_only": ("for (int64_t q = 1; q < l && st == ORC_OK; ++q) {",
                                 "for (int64_t q = 1; q < 1 && st == ORC_OK; ++q) {"),
    "envelope_b_of_first_term": ("a + q * m, b + q * n, m, n, r, batch, term", "a + q * m, b, m, n, r, batch, term"),
    "envelope_a_of_first_term": ("a + q * m, b + q * n, m, n, r, batch, term", "a, b + q * n, m, n, r, batch, term"),
    "envelope_subtracts": ("y[e] += term[e];", "y[e] -= term[e];"),
    "envelope_bpw_one_pair": ("16.0 * (double)l * (double)(m + n)", "16.0 * (double)(m + n)"),
    "transpose_msb": ("out[j * wpr_out + i / 32] |= 1u << (i % 32);", "out[j * wpr_out + i / 32] |= 1u << (31 - i % 32);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    before, after = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(before) == 1, f"mutation site for {name} not unique"
    mutated = tmp_path / "mut.c"
    mutated.write_text(src.replace(before, after))
    lib = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O1", "-fPIC", "-shared", "-std=c11", "-o", str(lib), str(mutated), "-lm"])
    o = oracle.Oracle(str(lib))
    failures = []
    for pin in pins.ALL_PINS:
        try:
            pin(o)
        except (AssertionError, ValueError):
            failures.append(pin.__name__)
    assert failures, f"mutant {name} passed every pin"


# Wiring mistakes planted in a copy of the oracle's Python chain composition.
CHAIN_MUTANTS = {
    "o_reads_h": ('out["o"] = self.lowrank_linear_fwd(out["x_o"], *w["o"])',
                  'out["o"] = self.lowrank_linear_fwd(h_bits, *w["o"])'),
    "down_reads_gate": ('out["x_down"] = self.round_to_bf16(out["up"])',
                        'out["x_down"] = self.round_to_bf16(out["gate"])'),
    "next_from_o": ('out["h_next"] = self.rms_normalize_bf16(out["down"])',
                    'out["h_next"] = self.rms_normalize_bf16(out["o"])'),
}


@pytest.mark.parametrize("name", sorted(CHAIN_MUTANTS))
def test_chain_mutant_is_caught(name):
    import types

    before, after = CHAIN_MUTANTS[name]
    path = os.path.join(os.path.dirname(oracle.__file__), "__init__.py")
    src = open(path).read()
    assert src.count(before) == 1, f"mutation site for {name} not unique"
    mod = types.ModuleType("oracle_mutant")
    mod.__file__ = path
    exec(compile(src.replace(before, after), "oracle_mutant", "exec"), mod.__dict__)
    o = mod.Oracle(oracle.build())
    with pytest.raises(AssertionError):
        pins.pin_chain_block(o)
