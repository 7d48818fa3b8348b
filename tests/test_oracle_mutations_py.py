"""Do the pins catch plausible mistakes in the oracle's Python parts?

The layout, the loss-scale rule, the accounting and the stage drivers are
plain Python in oracle/__init__.py.  Each mutant here rewrites one function
(or the StageRun class) from its own source with one textual change (a
bucket boundary off by one, padding truncated instead of rounded up, the
alignment unit dropped, the growth test off by one, the scale floor lost,
gradients counted as replicated in Stage 2, Stage 3 without its second
gather, a reduce-scatter or an optimizer slice at the wrong partition, t not
advancing), installs it in place of the original on the oracle module, and
runs the pins until one fails.  A mutant that survives every pin fails this
test.  The original is restored afterwards; nothing on disk changes.
"""
import inspect

import pytest

import oracle
import test_oracle_accounting as AC
import test_oracle_layout as LY
import test_oracle_stages as S

MUTANTS = [
    ("partition_layout", "bucket boundary off by one", "cur_n + n > bucket_elems", "cur_n + n >= bucket_elems"),
    ("partition_layout", "padding truncated", "pad = -(-off // unit) * unit", "pad = (off // unit) * unit"),
    ("partition_layout", "alignment unit dropped", "unit = world * align_elems", "unit = world"),
    ("loss_scale_update", "growth test off by one", "if good_steps >= growth_interval:",
     "if good_steps > growth_interval:"),
    ("loss_scale_update", "scale floor lost", "return max(scale / 2.0, min_scale), 0", "return scale / 2.0, 0"),
    ("model_state_bytes", "Stage 2 gradients counted as replicated", "g = full if stage < 2 else part",
     "g = full if stage < 1 else part"),
    ("comm_elements", "Stage 3 without its second gather", "return ag + ag + rs", "return ag + rs"),
    ("StageRun", "reduce-scatter of the wrong partition", "reduce(grads[b], self.gdtype, r * P, P)",
     "reduce(grads[b], self.gdtype, 0, P)"),
    ("StageRun", "Stage 1 updates the wrong slice", "s[r * P:(r + 1) * P]", "s[0:P]"),
    ("StageRun", "t does not advance", "sc.t = t", "sc.t = sc.t"),
]

PINS = [                                    # cheapest first
    ("layout invariants", lambda: LY.test_layout_invariants_small(3, 1000, 2)),
    ("layout invariants, one bucket", lambda: LY.test_layout_invariants_small(5, 0, 1)),
    ("odd flat padding", LY.test_odd_flat_model_padding),
    ("bucket filled to capacity", LY.test_bucket_filled_exactly_to_capacity),
    ("loss-scale rule", S.test_loss_scale_rule),
    ("memory formulas", lambda: AC.test_memory_formulas_exact_when_N_divides_psi(8)),
    ("communication", lambda: AC.test_communication_volumes(8)),
    ("stages equal DP", lambda: S.test_stages_equal_plain_dp_bit_exact(3, [5, 1000, 17, 333, 2, 4096], 1500,
                                                                       oracle.F16)),
    ("overflow skip and t", S.test_overflow_skips_update_and_halves_scale),
    ("6.7b units", LY.test_gpt_6p7b_units),
    ("gpt2 buckets", LY.test_gpt2_tensor_list_and_buckets),
]


def _install(name, find, repl):
    src = inspect.getsource(getattr(oracle, name))
    assert find in src, f"mutation target not found in {name}: {find!r}"
    ns = dict(vars(oracle))
    exec(compile(src.replace(find, repl), f"<mutant of {name}>", "exec"), ns)
    return ns[name]


@pytest.mark.parametrize("name,label,find,repl", MUTANTS, ids=[m[1] for m in MUTANTS])
def test_every_python_mutant_is_caught(name, label, find, repl):
    original = getattr(oracle, name)
    mutant = _install(name, find, repl)
    caught_by = None
    setattr(oracle, name, mutant)
    try:
        for pin_label, pin in PINS:
            try:
                pin()
            except (AssertionError, ZeroDivisionError, ValueError, FloatingPointError):
                caught_by = pin_label
                break
    finally:
        setattr(oracle, name, original)
    assert caught_by is not None, f"no pin catches the mutant '{label}'"


def test_the_unmutated_python_oracle_passes_every_pin():
    for _, pin in PINS:
        pin()
