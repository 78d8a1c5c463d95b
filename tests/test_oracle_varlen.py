"""Pins of the varlen oracle (oracle/varlen.py): packed sequences of different lengths.

Each pin checks it against something other than its own loop: the batched C recurrence
(equal lengths are a plain batch), chaining through states (a sequence cut in two and resumed
from the first part's final state is the whole sequence), and isolation (nothing of one
sequence reaches another; an empty sequence hands its initial state straight through).
Source: the article "Mamba-2状态空间模型的编译器优先实现" (bqwf.cn) §1.1 (the state is passed
along one sequence).
"""
import numpy as np
import pytest

import oracle
import ssd_synth as S
from conftest import f64


def _packed(T, H=4, P=8, G=2, N=8, seed=0, h0_rows=None):
    inp = f64(S.prefill_inputs(1, T, H, P, G, N, dtype="f32", seed=seed))
    h0 = None
    if h0_rows:
        h0 = np.random.default_rng(seed + 1).standard_normal((h0_rows, H, P, N)) * 0.3
    return inp, h0


def _run(inp, cu, h0):
    return oracle.ssd_scan_varlen(inp["x"][0], inp["dt"][0], inp["A_log"], inp["Bm"][0], inp["Cm"][0], cu,
                                  D=inp["D"], dt_bias=inp["dt_bias"], dt_min=inp["dt_min"],
                                  dt_max=inp["dt_max"], h0=h0)


def test_equal_lengths_equal_the_batched_recurrence():
    n, L = 3, 37
    inp, h0 = _packed(n * L, seed=1, h0_rows=n)
    y, hf = _run(inp, [0, L, 2 * L, 3 * L], h0)
    H, P = inp["x"].shape[-2:]
    G, N = inp["Bm"].shape[-2:]
    yb, hb = oracle.ssd_scan_sequential(inp["x"][0].reshape(n, L, H, P), inp["dt"][0].reshape(n, L, H),
                                        inp["A_log"], inp["Bm"][0].reshape(n, L, G, N),
                                        inp["Cm"][0].reshape(n, L, G, N), inp["D"], inp["dt_bias"],
                                        inp["dt_min"], inp["dt_max"], h0)
    np.testing.assert_allclose(y, yb.reshape(n * L, H, P), rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(hf, hb, rtol=1e-13, atol=1e-13)


def test_sequences_do_not_leak():
    cu = [0, 5, 5, 40, 41, 90]
    inp, h0 = _packed(90, seed=2, h0_rows=5)
    y, hf = _run(inp, cu, h0)
    inp2 = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in inp.items()}
    inp2["x"] = inp["x"].copy()
    inp2["x"][0, 5:40] *= -2.0  # sequence 2 only
    y2, hf2 = _run(inp2, cu, h0)
    np.testing.assert_array_equal(y2[:5], y[:5])
    np.testing.assert_array_equal(y2[40:], y[40:])
    np.testing.assert_array_equal(hf2[[0, 1, 3, 4]], hf[[0, 1, 3, 4]])
    assert not np.allclose(y2[5:40], y[5:40])


def test_empty_sequence_passes_its_state_through():
    inp, h0 = _packed(20, seed=3, h0_rows=3)
    y, hf = _run(inp, [0, 10, 10, 20], h0)
    np.testing.assert_array_equal(hf[1], h0[1])


def test_cut_and_resume_equals_one_sequence():
    inp, h0 = _packed(60, seed=4, h0_rows=1)
    y_one, hf_one = _run(inp, [0, 60], h0)
    y_a, hf_a = _run({**inp, "x": inp["x"][:, :23], "dt": inp["dt"][:, :23], "Bm": inp["Bm"][:, :23],
                      "Cm": inp["Cm"][:, :23]}, [0, 23], h0)
    y_b, hf_b = _run({**inp, "x": inp["x"][:, 23:], "dt": inp["dt"][:, 23:], "Bm": inp["Bm"][:, 23:],
                      "Cm": inp["Cm"][:, 23:]}, [0, 37], hf_a)
    np.testing.assert_allclose(np.concatenate([y_a, y_b]), y_one, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(hf_b, hf_one, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("cu", [[1, 10], [0, 5, 3, 10], [0, 9]])
def test_bad_cu_seqlens_rejected(cu):
    inp, _ = _packed(10, seed=5)
    with pytest.raises(ValueError):
        _run(inp, cu, None)


# ---- mutation check: slips planted in a temporary copy of oracle/varlen.py ----
import importlib.util  # noqa: E402
import os  # noqa: E402

import oracle.varlen as varlen_mod  # noqa: E402

VARLEN_SRC = os.path.join(os.path.dirname(varlen_mod.__file__), "varlen.py")
MUTANTS = [
    ("h0_of_first_sequence", "h0_i = None if h0 is None else np.asarray(h0, dtype=np.float64)[i:i + 1]",
     "h0_i = None if h0 is None else np.asarray(h0, dtype=np.float64)[0:1]"),
    ("state_carried_across", "h0_i = None if h0 is None else np.asarray(h0, dtype=np.float64)[i:i + 1]",
     "h0_i = (None if h0 is None else np.asarray(h0, dtype=np.float64)[i:i + 1]) if i == 0 else hf[i - 1:i]"),
    ("empty_sequence_zero_state", "hf[i] = hi[0]", "hf[i] = hi[0] if b > a else 0.0"),
]
PINS = [test_equal_lengths_equal_the_batched_recurrence, test_sequences_do_not_leak,
        test_empty_sequence_passes_its_state_through, test_cut_and_resume_equals_one_sequence]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_varlen_pins_reject_mutant(tmp_path, monkeypatch, name, old, new):
    src = open(VARLEN_SRC).read()
    assert src.count(old) == 1, old
    src = src.replace(old, new).replace("from .native import", "from oracle.native import")
    path = tmp_path / "varlen_mutant.py"
    path.write_text(src)
    spec = importlib.util.spec_from_file_location("varlen_mutant", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    monkeypatch.setattr(oracle, "ssd_scan_varlen", mod.ssd_scan_varlen)
    failed = []
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passes every pin"
