"""Mutation check of the oracle pins (CPU only).

Each case plants one plausible mistake in a temporary copy of oracle/ssd_oracle.c,
builds it, routes the oracle to it and runs the pins of test_oracle_pins.py.  The
pins must reject every mutant: at least one of them has to fail.  The real oracle
source is never modified.
"""
import os
import subprocess

import pytest

import oracle.native as native
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(native.__file__), "ssd_oracle.c")

# (name, original text, planted mistake)
MUTANTS = [
    ("drop_D_skip", "yt[p] = acc + skip * xt[p];", "yt[p] = acc;"),
    ("positive_A", "const double A = -exp(A_log[h]);", "const double A = exp(A_log[h]);"),
    ("exclusive_diagonal",
     "row[n] = a * row[n] + dt * xt[p] * Bt[n];\n                        acc += row[n] * Ct[n];",
     "acc += row[n] * Ct[n];\n                        row[n] = a * row[n] + dt * xt[p] * Bt[n];"),
    ("swap_B_C", "const double *Bt = Bm + (bt * G + g) * N;", "const double *Bt = Cm + (bt * G + g) * N;"),
    ("no_dt_on_input", "row[n] = a * row[n] + dt * xt[p] * Bt[n];", "row[n] = a * row[n] + xt[p] * Bt[n];"),
    ("bias_after_softplus", "return clip(sp(dt_raw + bias), dt_min, dt_max);",
     "return clip(sp(dt_raw) + bias, dt_min, dt_max);"),
    ("no_clip", "return clip(sp(dt_raw + bias), dt_min, dt_max);", "return sp(dt_raw + bias);"),
    ("interleaved_groups", "const int g = h / heads_per_group;\n            const double A",
     "const int g = h % G;\n            const double A"),
    ("decay_without_dt", "const double a = exp(dt * A);", "const double a = exp(A);"),
    ("h0_ignored", "st[i] = h0 ? h0[((size_t)b * H + h) * P * N + i] : 0.0;", "st[i] = 0.0;"),
    ("conv_window_reversed",
     "if (s >= 0) acc += w[(size_t)c * K + k] * xBC[((size_t)b * L + s) * Cc + c];",
     "if (s >= 0) acc += w[(size_t)c * K + (K - 1 - k)] * xBC[((size_t)b * L + s) * Cc + c];"),
    ("conv_no_bias", "double acc = bias ? bias[c] : 0.0;", "double acc = 0.0;"),
    ("decode_roll_before_use",
     "const double v = (k < K - 1) ? cs[k] : newest;",
     "const double v = (k < K - 2) ? cs[k + 1] : newest;"),
    ("decode_drop_D", "y_t[((size_t)b * H + h) * P + p] = acc + (D ? D[h] : 0.0) * xp;",
     "y_t[((size_t)b * H + h) * P + p] = acc;"),
    ("decode_state_not_decayed", "row[n] = a * row[n] + dt * xp * Bs[g * N + n];",
     "row[n] = row[n] + dt * xp * Bs[g * N + n];"),
]

PIN_TESTS = [
    (pins.test_sequential_equals_chunked, {"chunk": 4, "unclipped": False}),
    (pins.test_sequential_equals_chunked, {"chunk": 16, "unclipped": True}),
    (pins.test_sequential_equals_dense, {"h0": True}),
    (pins.test_no_decay_is_causal_linear_attention, {}),
    (pins.test_geometric_series_scalar_state, {}),
    (pins.test_impulse_response_decay_indexing, {}),
    (pins.test_full_decay_keeps_only_current_token, {}),
    (pins.test_single_token_with_initial_state, {}),
    (pins.test_hand_worked_three_tokens, {}),
    (pins.test_split_resume_equals_one_pass, {}),
    (pins.test_head_to_group_mapping, {}),
    (pins.test_dt_softplus_and_clip, {}),
    (pins.test_causal_conv_matches_library_convolution, {}),
    (pins.test_prefill_then_decode_equals_recompute, {"G": 2}),
]


def _build_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique/absent"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / f"{name}.so"
    subprocess.run(["gcc", "-O1", "-fopenmp", "-shared", "-fPIC", "-o", str(so), str(path), "-lm"],
                   check=True)
    return str(so)


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_reject_mutant(tmp_path, name, old, new):
    so = _build_mutant(tmp_path, name, old, new)
    caught = []
    with native.use_library(so):
        for fn, kw in PIN_TESTS:
            try:
                fn(**kw)
            except Exception:            # a failed assertion or a numerical blow-up
                caught.append(fn.__name__)
    assert caught, f"no pin caught the planted mistake {name}"
