"""Do the pins catch plausible mistakes?  Plant one mistake at a time in a
copy of the oracle's C source, on the CPU, and check that some pin fails.

Each mutant is compiled from a temporary copy of oracle/zero_oracle.c with
one textual change (a wrong sign, a dropped term, a swapped operand, a
missing bias correction, a reversed or shortened rank order, truncation
instead of round-to-nearest-even, a lost offset, a weaker overflow test),
loaded in place of the real oracle library, and run through the pins of the
other test files until one of them fails.  A mutant that survives every pin
fails this test.  The real oracle is untouched.
"""
import os
import subprocess
import tempfile

import pytest

import oracle
import test_oracle_adam as A
import test_oracle_clip as C
import test_oracle_formats as F
import test_oracle_layout as LY
import test_oracle_reduce as R
import test_oracle_stages as S

SRC = os.path.join(os.path.dirname(oracle.__file__), "zero_oracle.c")

# (name, text to find, replacement); every occurrence is replaced
MUTANTS = [
    ("update sign", "fmaf(-lr, u, master[j] * decay)", "fmaf(lr, u, master[j] * decay)"),
    ("epsilon dropped", "fmaf(sqrtf(vn), rsbc2, eps)", "(sqrtf(vn) * rsbc2)"),
    ("beta1 and beta2 swapped in m", "fmaf(b1, m[j], omb1 * g)", "fmaf(b2, m[j], omb1 * g)"),
    ("v uses g instead of g^2", "(omb2 * g) * g", "(omb2 * g)"),
    ("no bias correction of m", "c[7] = (float)(1.0 / (1.0 - pow((double)beta1, (double)t)));", "c[7] = 1.0f;"),
    ("no bias correction of v", "c[8] = (float)(1.0 / sqrt(1.0 - pow((double)beta2, (double)t)));", "c[8] = 1.0f;"),
    ("weight decay not applied", "master[j] * decay)", "master[j])"),
    ("sum instead of mean", "c[4] = (float)(1.0 / (divisor * (double)loss_scale));",
     "c[4] = (float)(1.0 / ((double)loss_scale));"),
    ("replica 0 dropped", "float acc = to_f32(G[0][begin + j], dtype);", "float acc = 0.0f;"),
    ("rank order reversed",
     "float acc = to_f32(G[0][begin + j], dtype);\n        for (int32_t k = 1; k < N; ++k) acc = acc + to_f32(G[k][begin + j], dtype);",
     "float acc = to_f32(G[N - 1][begin + j], dtype);\n        for (int32_t k = N - 2; k >= 0; --k) acc = acc + to_f32(G[k][begin + j], dtype);"),
    ("truncation instead of rounding", "if (rem > half || (rem == half && (q & 1u))) q += 1u;", "(void)half;"),
    ("ties away from zero", "(rem == half && (q & 1u))", "(rem == half)"),
    ("gather ignores the shard offset", "shards[r][offset + j]", "shards[r][j]"),
    ("overflow test misses NaN", "if (!isfinite(s[j])) any = 1;", "if (isinf(s[j])) any = 1;"),
    ("norm squares the scaled sum", "float g = s[j] * inv;\n        acc += (double)g * (double)g;",
     "float g = s[j];\n        acc += (double)g * (double)g;"),
    ("clip factor not clamped", "return coef < 1.0 ? (float)coef : 1.0f;", "return (float)coef;"),
    ("reduced gradient not unscaled", "g[j] = s[j] * inv;", "g[j] = s[j];"),
]

# cheap pins first; each entry is (label, callable)
PINS = [
    ("formats ties", F.test_f32_to_f16_ties_to_even),
    ("formats f16 numpy", F.test_f32_to_f16_rne_matches_numpy),
    ("formats bf16 torch", F.test_f32_to_bf16_rne_matches_torch),
    ("reduce single replica", R.test_single_replica_is_exact_conversion),
    ("reduce integers", R.test_integer_gradients_sum_exactly),
    ("reduce order", R.test_rank_order_is_left_to_right),
    ("reduce error bound", R.test_reduce_within_fp32_error_bound_of_exact_sum),
    ("nan flag", R.test_nan_alone_sets_the_flag),
    ("flag f16", lambda: R.test_overflow_flag(oracle.F16)),
    ("sqnorm", R.test_grad_sqnorm_matches_fp64_sum),
    ("unscale exact", lambda: R.test_unscale_by_power_of_two_is_exact(8, 65536.0)),
    ("gather offset", LY.test_allgather_with_offset_brute_force),
    ("adam constants", A.test_constants_are_rounded_from_double),
    ("adam step-1 closed form", lambda: A.test_step1_closed_form(0.0)),
    ("adam step-1 closed form wd", lambda: A.test_step1_closed_form(0.01)),
    ("adam zero lr", A.test_zero_lr_changes_no_weight),
    ("adam zero grad", A.test_zero_gradient_keeps_moments_and_decays_weights),
    ("adam constant gradient", A.test_constant_gradient_gives_constant_update),
    ("adam fp64 textbook", A.test_fp64_textbook_brute_force),
    ("adam torch", lambda: A.test_matches_torch_adamw_cpu(0.01)),
    ("clip closed form", lambda: C.test_coefficient_closed_form(0.25, 1.0)),
    ("clip torch", C.test_matches_torch_clip_then_adamw),
    ("stages", lambda: S.test_stages_equal_plain_dp_bit_exact(4, [10_007], 0, oracle.F16)),
]


def _build_mutant(src_text: str, workdir: str) -> str:
    c = os.path.join(workdir, "mutant.c")
    so = os.path.join(workdir, "mutant.so")
    with open(c, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", *oracle.CFLAGS, "-o", so, c, "-lm"])
    return so


@pytest.mark.parametrize("name,find,repl", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_every_mutant_is_caught(name, find, repl):
    with open(SRC) as f:
        text = f.read()
    assert find in text, f"mutation target not found: {find!r}"
    mutated = text.replace(find, repl)
    with tempfile.TemporaryDirectory() as d:
        lib = oracle.load_library(_build_mutant(mutated, d))
        saved = oracle._lib
        oracle._lib = lib
        caught_by = None
        try:
            for label, pin in PINS:
                try:
                    pin()
                except AssertionError:
                    caught_by = label
                    break
        finally:
            oracle._lib = saved
    assert caught_by is not None, f"no pin catches the mutant '{name}'"


def test_the_unmutated_oracle_passes_every_pin():
    for label, pin in PINS:
        pin()
