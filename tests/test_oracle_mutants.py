"""The oracle's pins catch planted mistakes.  Each case compiles a copy of oracle.c with one
plausible error (a dropped term or factor, a wrong sign, a transposed or off-by-one index, a
missing bias correction) and runs the pin checks of test_oracle.py against it: at least one
must fail.  The mistakes live only in these temporary copies, on the CPU."""
import os
import subprocess

import pytest

import oracle
import test_oracle as T

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

MUTANTS = {
    "dB_scale_dropped": ("dB[i][c * r + k] = s * acc;", "dB[i][c * r + k] = acc;"),
    "G_scale_dropped": ("    return s * acc;\n}", "    return acc;\n}"),
    "lora_sign_flipped": ("Y_out[q * d_out + c] = base + s * lora;", "Y_out[q * d_out + c] = base - s * lora;"),
    "dX_base_dropped": ("dX_out[q * d_in + j] = base + lora;", "dX_out[q * d_in + j] = lora;"),
    "segment_boundary_off_by_one": ("if (t >= off[i] && t < off[i + 1]) return i;",
                                    "if (t >= off[i] && t <= off[i + 1]) return i;"),
    "dA_stored_transposed": ("dA[i][(int64_t)k * d_in + j] = acc;", "dA[i][j * r + k] = acc;"),
    "H_uses_wrong_factor_row": ("ld(Ai, dtype, (int64_t)k * d_in + j);", "ld(Ai, dtype, j);"),
    "adamw_bias_correction_dropped": ("p[e] = p[e] - (lr / bc1) * m[e] / denom;", "p[e] = p[e] - lr * m[e] / denom;"),
    "adamw_decay_coupled": ("p[e] = p[e] * (1.0 - lr * weight_decay);", "p[e] = p[e] * (1.0 - weight_decay);"),
    # column-subset mode: the q-th requested column stored at position q instead of its own index
    "dB_column_subset_stored_by_position": ("dB[i][c * r + k] = s * acc;", "dB[i][q * r + k] = s * acc;"),
    "dA_column_subset_stored_by_position": ("dA[i][(int64_t)k * d_in + j] = acc;",
                                            "dA[i][(int64_t)k * d_in + q] = acc;"),
    "dA_column_subset_reads_position": ("acc += ld(X, dtype, (t0 + u) * d_in + j) * G[u * r + k];",
                                        "acc += ld(X, dtype, (t0 + u) * d_in + q) * G[u * r + k];"),
}

PINS = [
    ("merged_weight_fp32", lambda: T.test_forward_and_input_grad_match_merged_weight(1, "fp32")),
    ("hand_derived", T.test_hand_derived_integer_example),
    ("B_zero", lambda: T.test_B_zero_gives_base_exactly_and_zero_dA("fp32")),
    ("rank1", T.test_rank1_outer_product_closed_forms),
    ("linear_in_scale", T.test_linear_in_scale),
    ("finite_differences", T.test_gradients_match_central_finite_differences),
    ("segment_signature", T.test_segment_signature_exact),
    ("column_subset_fp32", lambda: T.test_column_subset_api_matches_full_columns("fp32")),
    ("column_subset_bf16", lambda: T.test_column_subset_api_matches_full_columns("bf16")),
    ("adamw_torch", lambda: T.test_adamw_matches_torch_adamw_in_float64(T.ADAMW_CASES[0])),
    ("adamw_first_step", T.test_adamw_first_step_closed_form),
    ("adamw_zero_grad", T.test_adamw_zero_gradient_is_pure_decay),
]


def _build(tmp_path, name, src):
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"{name}.so"
    c.write_text(src)
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c11", str(c), "-o", str(so), "-lm"],
                   check=True)
    return str(so)


def _failures(path):
    failed = []
    with oracle.use_library(path):
        for name, pin in PINS:
            try:
                pin()
            except AssertionError:
                failed.append(name)
    return failed


def test_unmutated_copy_passes_every_pin(tmp_path):
    assert _failures(_build(tmp_path, "clean", open(SRC).read())) == []


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_planted_mistake_is_caught(mutant, tmp_path):
    old, new = MUTANTS[mutant]
    src = open(SRC).read()
    assert src.count(old) == 1, mutant
    failed = _failures(_build(tmp_path, mutant, src.replace(old, new)))
    assert failed, f"{mutant} passed every pin"
