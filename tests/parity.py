"""Helpers shared by the GPU parity tests: moving seeded inputs to the device and the
elementwise tolerance rule |got - ref| <= atol + rtol * |ref|.

Tolerances (written here once, used by every parity test):
  float32 storage:  rtol 1e-4, atol 1e-5 on y and on the state.
  bf16 storage:     y      rtol 2e-2, atol 2e-2 * RMS(ref)   (y crosses zero, so an absolute
                                                               floor scaled to the data is needed)
                    state  rtol 1e-3, atol 1e-3 * RMS(ref)
  gated norm output ("norm"): float32 rtol 1e-4, atol 1e-6; bf16 rtol 5e-3, atol 1e-6 * RMS(ref).
                    The bf16 bound is the output's own rounding (unit roundoff 2^-8 = 3.9e-3)
                    plus the fp32 sum of squares over at most 32768 channels (<= 1e-3 relative
                    in the worst case, far less in practice); the inputs are exact on both sides.
"""
import numpy as np
import torch

TOL = {
    ("f32", "y"): (1e-4, 1e-5, None),
    ("f32", "h"): (1e-4, 1e-5, None),
    ("bf16", "y"): (2e-2, None, 2e-2),
    ("bf16", "h"): (1e-3, None, 1e-3),
    ("f32", "norm"): (1e-4, 1e-6, None),
    ("bf16", "norm"): (5e-3, None, 1e-6),
}


def dev(a, device="cuda"):
    """A storage array from ssd_synth (float32, or uint16 bf16 bits) -> torch tensor."""
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(a).to(device)


def host64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def check_close(got, ref, dtype, kind, what=""):
    rtol, atol_abs, atol_rms = TOL[(dtype, kind)]
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    if ref.size == 0:
        return 0.0
    atol = atol_abs if atol_abs is not None else atol_rms * float(np.sqrt(np.mean(ref ** 2)))
    err = np.abs(got - ref)
    bound = atol + rtol * np.abs(ref)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    worst = float(np.max(err / bound))
    if worst > 1.0:
        i = np.unravel_index(np.argmax(err / bound), ref.shape)
        n_bad = int(np.sum(err > bound))
        raise AssertionError(f"{what}: {n_bad}/{ref.size} elements out of tolerance; worst at {i}: "
                             f"got {got[i]!r} ref {ref[i]!r} (err/bound {worst:.3g})")
    return worst
