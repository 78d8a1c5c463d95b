"""Pins of the fp64 gated RMS norm (oracle/block.py) and a mutation check of those pins.

The norm is y * SiLU(z), RMS-normalised per token over groups of consecutive channels,
then scaled per channel.  The pages fix only that its variance is taken in float32 or
better (article "Mamba-2状态空间模型的编译器优先实现" (bqwf.cn) §4.1); the rest is the
Mamba-2 block's norm.  Each pin checks the oracle against something other than its own
formula: a library routine (scipy's logistic function), a hand-worked case, a closed form
for a constant group, or an invariant (unit RMS, scale invariance, oddness, group
independence, a zero gate).  Every planted slip below fails at least one pin.
"""
import importlib.util
import math
import os

import numpy as np
import pytest
from scipy.special import expit

import oracle.block as block

BLOCK_SRC = os.path.join(os.path.dirname(block.__file__), "block.py")


def _rng(seed):
    return np.random.default_rng(seed)


# ---- the pins, each taking the module under test -------------------------------------
def pin_silu_matches_scipy(m):
    z = np.linspace(-30.0, 30.0, 601)
    np.testing.assert_allclose(m.silu(z), z * expit(z), rtol=1e-14, atol=1e-300)


def pin_hand_worked(m):
    # y = (3, 4), z = 60: SiLU(60) = 60 to 1e-24, so g = (180, 240), mean g^2 = 45000,
    # rms = 212.132..., out = (180, 240) / rms = (0.848528..., 1.131370...) for eps = 0.
    out = m.gated_rmsnorm(np.array([[3.0, 4.0]]), np.array([[60.0, 60.0]]), np.array([1.0, 2.0]), eps=0.0)
    rms = math.sqrt((180.0 ** 2 + 240.0 ** 2) / 2.0)
    np.testing.assert_allclose(out, [[180.0 / rms, 2.0 * 240.0 / rms]], rtol=1e-14)


def pin_zero_gate_gives_zero(m):
    r = _rng(1)
    y = r.standard_normal((3, 16))
    z = r.standard_normal((3, 16))
    z[:, ::2] = 0.0  # SiLU(0) = 0: those channels are exactly 0 whatever y is
    out = m.gated_rmsnorm(y, z, np.ones(16), eps=1e-6)
    assert np.all(out[:, ::2] == 0.0)
    assert np.all(out[:, 1::2] != 0.0)


def pin_unit_rms_per_group(m):
    r = _rng(2)
    C, G = 24, 3
    y = r.standard_normal((5, C))
    z = r.standard_normal((5, C))
    w = r.uniform(0.5, 2.0, C)
    out = m.gated_rmsnorm(y, z, w, eps=0.0, n_groups=G)
    ms = np.mean((out / w).reshape(5, G, C // G) ** 2, axis=-1)
    np.testing.assert_allclose(ms, 1.0, rtol=1e-13)


def pin_constant_group_closed_form(m):
    # a group whose gated values all equal c: out = w c / sqrt(c^2 + eps)
    c_y, z0, eps = 0.7, 1.3, 0.25
    c = c_y * z0 / (1.0 + math.exp(-z0))
    y = np.full((1, 8), c_y)
    z = np.full((1, 8), z0)
    w = np.arange(1.0, 9.0)
    out = m.gated_rmsnorm(y, z, w, eps=eps)
    np.testing.assert_allclose(out[0], w * c / math.sqrt(c * c + eps), rtol=1e-14)


def pin_scale_invariance_and_oddness(m):
    r = _rng(3)
    y = r.standard_normal((4, 32))
    z = r.standard_normal((4, 32))
    w = r.standard_normal(32)
    base = m.gated_rmsnorm(y, z, w, eps=0.0, n_groups=2)
    np.testing.assert_allclose(m.gated_rmsnorm(7.5 * y, z, w, eps=0.0, n_groups=2), base, rtol=1e-13)
    np.testing.assert_allclose(m.gated_rmsnorm(-y, z, w, eps=0.0, n_groups=2), -base, rtol=1e-13)


def pin_groups_are_independent(m):
    r = _rng(4)
    y = r.standard_normal((2, 32))
    z = r.standard_normal((2, 32))
    w = np.ones(32)
    a = m.gated_rmsnorm(y, z, w, eps=1e-5, n_groups=4)
    y2 = y.copy()
    y2[:, :8] *= 3.0  # group 0 only
    b = m.gated_rmsnorm(y2, z, w, eps=1e-5, n_groups=4)
    np.testing.assert_array_equal(a[:, 8:], b[:, 8:])
    one = m.gated_rmsnorm(y2, z, w, eps=1e-5, n_groups=1)  # one group: every channel moves
    assert np.all(np.abs(one[:, 8:] - m.gated_rmsnorm(y, z, w, eps=1e-5, n_groups=1)[:, 8:]) > 0)


def pin_weight_per_channel(m):
    r = _rng(5)
    y = r.standard_normal((3, 12))
    z = r.standard_normal((3, 12))
    w = r.uniform(0.1, 3.0, 12)
    perm = r.permutation(12)
    out = m.gated_rmsnorm(y, z, w, eps=1e-3)
    # one group: permuting the channels of y, z and w permutes the output
    np.testing.assert_allclose(m.gated_rmsnorm(y[:, perm], z[:, perm], w[perm], eps=1e-3), out[:, perm],
                               rtol=1e-13)
    np.testing.assert_allclose(out / w, m.gated_rmsnorm(y, z, np.ones(12), eps=1e-3), rtol=1e-13)


PINS = [pin_silu_matches_scipy, pin_hand_worked, pin_zero_gate_gives_zero, pin_unit_rms_per_group,
        pin_constant_group_closed_form, pin_scale_invariance_and_oddness, pin_groups_are_independent,
        pin_weight_per_channel]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_norm_pin(pin):
    pin(block)


# ---- mutation check: plausible slips planted in a temporary copy of oracle/block.py ----
MUTANTS = [
    ("no_gate", "g = y * silu(z)", "g = y"),
    ("sigmoid_gate", "g = y * silu(z)", "g = y / (1.0 + np.exp(-z))"),
    ("silu_wrong_sign", "return z / (1.0 + np.exp(-z))", "return z / (1.0 + np.exp(z))"),
    ("eps_outside_sqrt", "normed = grouped / np.sqrt(ms + eps)", "normed = grouped / (np.sqrt(ms) + eps)"),
    ("no_sqrt", "normed = grouped / np.sqrt(ms + eps)", "normed = grouped / (ms + eps)"),
    ("sum_not_mean", "ms = np.mean(grouped * grouped, axis=-1, keepdims=True)",
     "ms = np.sum(grouped * grouped, axis=-1, keepdims=True)"),
    ("whole_row_not_groups", "ms = np.mean(grouped * grouped, axis=-1, keepdims=True)",
     "ms = np.mean(grouped * grouped, axis=(-2, -1), keepdims=True)"),
    ("interleaved_groups", "grouped = g.reshape(g.shape[:-1] + (n_groups, C // n_groups))",
     "grouped = g.reshape(g.shape[:-1] + (C // n_groups, n_groups))"),
    ("weight_inside_norm", "g = y * silu(z)", "g = y * silu(z) * w"),
    ("weight_dropped", "return normed.reshape(g.shape) * w", "return normed.reshape(g.shape)"),
]


def _load_mutant(tmp_path, old, new):
    src = open(BLOCK_SRC).read()
    assert src.count(old) == 1, old
    path = tmp_path / "block_mutant.py"
    path.write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location("block_mutant", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_norm_pins_reject_mutant(tmp_path, name, old, new):
    mod = _load_mutant(tmp_path, old, new)
    failed = []
    for pin in PINS:
        try:
            with np.errstate(all="ignore"):
                pin(mod)
        except (AssertionError, ValueError, FloatingPointError):
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passes every pin"
