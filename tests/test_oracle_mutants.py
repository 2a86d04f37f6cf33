"""Plant plausible mistakes in a copy of the oracle and check that the pins
catch every one of them (CPU only).

Each mutant is one textual edit of ``oracle/sfn_oracle.c`` (a flipped tie
rule, a dropped term, a wrong sign, a transposed operand, a wrong index...),
compiled into a temporary library.  Every edit keeps all memory accesses in
bounds.  The committed oracle itself is never modified.
"""
import os
import subprocess

import pytest

import oracle
import oracle_pins

MUTANTS = {
    "tie_to_higher_index": ("&& i < j)) ++rank", "&& i > j)) ++rank"),
    "keep_k_plus_one": ("if (rank < k)", "if (rank <= k)"),
    "smallest_instead_of_largest": ("return a > b;", "return a < b;"),
    "nan_ranks_first": ("if (isnan(a)) return 0;", "if (isnan(a)) return 1;"),
    "wrong_bit": ("word |= (uint64_t)1 << j;", "word |= (uint64_t)1 << (j ^ 1);"),
    "sigmoid_sign": ("return 1.0 / (1.0 + exp(-z));", "return 1.0 / (1.0 + exp(z));"),
    "dropped_sigmoid": ("double a = sfn_oracle_sigmoid(logits[t * d_i + j]) * g * u;",
                        "double a = g * u;"),
    "up_replaced_by_gate": ("double a = sfn_oracle_sigmoid(logits[t * d_i + j]) * g * u;",
                            "double a = sfn_oracle_sigmoid(logits[t * d_i + j]) * g * g;"),
    "B_transposed": ("ld(B, B_dt, (int64_t)j * r + m)", "ld(B, B_dt, (int64_t)m * d_i + j)"),
    "Wd_transposed": ("yt[n] += a * ld(Wd, Wd_dt, (int64_t)j * d + n);",
                      "yt[n] += a * ld(Wd, Wd_dt, (int64_t)n * d_i + j);"),
    "predictor_token0_only": ("ld(A, A_dt, (int64_t)m * d + n) * ld(x, x_dt, t * d + n);",
                              "ld(A, A_dt, (int64_t)m * d + n) * ld(x, x_dt, n);"),
    "predictor_skips_last_rank": ("for (int m = 0; m < r; ++m) s += ld(B",
                                  "for (int m = 0; m < r - 1; ++m) s += ld(B"),
    "dense4x_amplitude_signed": ("amp[j] = fabs(act[j]);", "amp[j] = act[j];"),
    "dense4x_gate_not_silu": ("act[j] = g * sfn_oracle_sigmoid(g) * u;",
                              "act[j] = sfn_oracle_sigmoid(g) * u;"),
    "bwd_surrogate_dropped": ("(mj * s * (1.0 - s) + s * sur)", "(mj * s * (1.0 - s))"),
    "bwd_surrogate_unscaled": ("sur = sz * (1.0 - sz) / temp;", "sur = sz * (1.0 - sz);"),
    "bwd_threshold_is_kth": ("tau[b] = (k < bank) ? 0.5 * (pk + pk1) : NAN;",
                             "tau[b] = (k < bank) ? pk : NAN;"),
    "bwd_du_uses_u": ("du[j] = da * mj * s * g;", "du[j] = da * mj * s * u;"),
    "bwd_sigmoid_derivative_dropped": ("(mj * s * (1.0 - s) + s * sur)", "(mj * s + s * sur)"),
    "bwd_dx_without_predictor": ("for (int m = 0; m < r; ++m) acc += dh[m] * ld(A",
                                 "for (int m = 0; m < 0; ++m) acc += dh[m] * ld(A"),
    "bwd_dA_without_x": ("dA[(int64_t)m * d + n] += acc * ld(x, x_dt, t * d + n);",
                         "dA[(int64_t)m * d + n] += acc;"),
}


@pytest.fixture(scope="module")
def source():
    return open(os.path.join(os.path.dirname(oracle.__file__), "sfn_oracle.c")).read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, source, tmp_path, monkeypatch):
    old, new = MUTANTS[name]
    assert source.count(old) == 1, f"mutation site for {name} not unique"
    src = tmp_path / f"mutant_{name}.c"
    src.write_text(source.replace(old, new))
    so = tmp_path / f"libmutant_{name}.so"
    subprocess.run(["gcc", "-O1", "-std=c99", "-fopenmp", "-fPIC", "-shared", "-o", str(so),
                    str(src), "-lm"], check=True)
    monkeypatch.setattr(oracle, "_lib", oracle._open(str(so)))
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin()
        except AssertionError:
            caught.append(pin.__name__)
            break
    assert caught, f"mutant {name} passed every pin"
