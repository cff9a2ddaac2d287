"""Plant plausible mistakes in copies of the oracle and check the pins catch them.

Each mutant edits one expression of oracle/engram_oracle.c (a dropped term, a
wrong sign, a swapped operand, a signed remainder, ...), is compiled on the CPU
into a temporary library, and must fail at least one pin of oracle_pins.  The
committed oracle itself is never modified.
"""
import os
import subprocess

import pytest

import oracle
import oracle_pins

MUTANTS = {
    "hash_add_instead_of_xor": ("h ^= (uint64_t)tok", "h += (uint64_t)tok"),
    "hash_pad_off_by_one": ("(s - i >= 0) ?", "(s - i > 0) ?"),
    "hash_signed_remainder": ("(int64_t)(h % P)", "((int64_t)h % (int64_t)P)"),
    "hash_multiplier_order": ("multipliers[(int64_t)l * n_max + i]",
                              "multipliers[(int64_t)l * n_max + (ngram_n[l] - 1 - i)]"),
    "gather_wrong_table_offset": ("acc += table_sizes[q];", "acc += table_sizes[0];"),
    "gather_bwd_overwrites": ("dst[c] += src[c];", "dst[c] = src[c];"),
    "gather_bwd_wrong_row": ("int64_t r = first_row[q] + idx[t * ntab + q];",
                             "int64_t r = idx[t * ntab + q];"),
    "fwd_wrong_weight_on_k": ("double b = k[j] * rk * we[j];\n        dot",
                              "double b = k[j] * rk * wh[j];\n        dot"),
    "fwd_eps_dropped": ("ss / (double)H + eps", "ss / (double)H"),
    "fwd_signed_sqrt_sign_lost": ("if (s < 0) return -sqrt(-s);", "if (s < 0) return sqrt(-s);"),
    "fwd_scalar_outside_sqrt": ("sigmoid(signed_sqrt(dot * scalar))",
                                "sigmoid(signed_sqrt(dot) * scalar)"),
    "fwd_sigmoid_sign": ("1.0 / (1.0 + exp(-u))", "1.0 / (1.0 + exp(u))"),
    "bwd_rms_term_dropped": (" - rx * rx * rx * xt[j] * cx / (double)H", ""),
    "bwd_clamp_dropped": ("sqrt(abs_s > 1e-6 ? abs_s : 1e-6)", "sqrt(abs_s)"),
    "bwd_sigmoid_derivative": ("dgate * gate * (1.0 - gate)", "dgate * gate"),
    "bwd_dwh_wrong_factor": ("sh[j - j0] += (ddot * b) * xj * rx;",
                             "sh[j - j0] += (ddot * a) * xj * rx;"),
    "bwd_dk_wrong_weight": ("dk[t * H + j] = rk * we[j] * db", "dk[t * H + j] = rk * wh[j] * db"),
    "bwd_dv_gate_dropped": ("dv[t * H + j] = gate * gt[j];", "dv[t * H + j] = gt[j];"),
    "bwd_residual_dropped": ("dx[t * H + j] = gt[j] + rx", "dx[t * H + j] = rx"),
    "bwd_dgate_wrong_operand": ("dgate += gt[j] * vt[j];", "dgate += gt[j] * xt[j];"),
}


def _build_mutant(tmp_path, name, old, new):
    with open(oracle.SOURCE) as f:
        src = f.read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    path = os.path.join(tmp_path, f"{name}.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    lib = os.path.join(tmp_path, f"lib{name}.so")
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-fopenmp", "-ffp-contract=off",
                    "-shared", "-o", lib, path, "-lm"], check=True)
    return oracle.Oracle(lib)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    old, new = MUTANTS[name]
    o = _build_mutant(str(tmp_path), name, old, new)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(o)
        except Exception:  # a failed comparison or a rejected (invalid) result
            caught.append(pin.__name__)
    assert caught, f"no pin catches mutant {name}"
