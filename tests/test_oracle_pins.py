"""Pins of the fp64 oracle to facts fixed by the pages and by mathematics.

Each test checks the oracle against something other than itself: a closed form, an
independent algorithm (the chunked and dense forms of the SSD duality), a library
routine (np.convolve, scipy's logistic function, math.log1p), an invariant the pages
state (the cached state is constant-size; prefill then cached decode equals full
recomputation), or a hand-worked case.  The set is chosen so that a plausible slip in
the oracle (a dropped term, a flipped sign, an off-by-one in the decay, B and C
swapped, the wrong group for a head, a reversed conv window) fails at least one test;
tests/test_oracle_mutants.py plants such slips and checks exactly that.

Sources: "Compiler-First State Space Duality and Portable O(1) Autoregressive Caching
for Inference" (abstract; decode independent of sequence length, checkpoint parity)
and the article "Mamba-2状态空间模型的编译器优先实现" (bqwf.cn) §1.1 (chunked SSD,
decay mask), §2.1 (constant-size state, conv window), §2.2 (cache update), §5.1
(cached O(1) decode against O(L^2) recomputation).
"""
import math

import numpy as np
import pytest
from scipy.special import expit

import oracle
import ssd_synth as S
from conftest import f64, oracle_args

TIGHT = 1e-11


def rel(a, b):
    a, b = np.asarray(a), np.asarray(b)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def small_inputs(Bsz=2, L=37, H=4, P=8, G=2, N=6, seed=5, h0=True, bias=True, unclipped=False):
    inp = S.prefill_inputs(Bsz, L, H, P, G, N, dtype="f32", seed=seed, h0=h0,
                           dt_bias_zero=not bias, unclipped=unclipped)
    return f64(inp)


# ---------------------------------------------------------------------------------
# cross-form agreement (the SSD duality: recurrence == chunked == quadratic)
# ---------------------------------------------------------------------------------
@pytest.mark.parametrize("chunk", [1, 4, 16, 64])
@pytest.mark.parametrize("unclipped", [False, True])
def test_sequential_equals_chunked(chunk, unclipped):
    f = small_inputs(L=53, unclipped=unclipped)
    y1, h1 = oracle.ssd_scan_sequential(*oracle_args(f))
    y2, h2 = oracle.ssd_chunked(*oracle_args(f), chunk=chunk)
    assert rel(y2, y1) < TIGHT and rel(h2, h1) < TIGHT


@pytest.mark.parametrize("h0", [False, True])
def test_sequential_equals_dense(h0):
    f = small_inputs(L=29, h0=h0)
    y1, h1 = oracle.ssd_scan_sequential(*oracle_args(f))
    y3, h3 = oracle.ssd_dense(*oracle_args(f))
    assert rel(y3, y1) < TIGHT and rel(h3, h1) < TIGHT


def test_chunked_workload_shape_ragged():
    # chunk 256 over a length that leaves a ragged tail, bigger state dims
    f = small_inputs(Bsz=1, L=300, H=2, P=16, G=1, N=32, seed=11)
    y1, h1 = oracle.ssd_scan_sequential(*oracle_args(f))
    y2, h2 = oracle.ssd_chunked(*oracle_args(f), chunk=256)
    assert rel(y2, y1) < TIGHT and rel(h2, h1) < TIGHT


# ---------------------------------------------------------------------------------
# closed forms and special cases
# ---------------------------------------------------------------------------------
def test_no_decay_is_causal_linear_attention():
    # A_log -> -inf gives A = 0, a_t = 1: the state is a running sum.
    f = small_inputs(h0=False)
    f["A_log"] = np.full_like(f["A_log"], -1e4)
    y, hf = oracle.ssd_scan_sequential(*oracle_args(f))
    dt, _ = oracle.discretise(f["dt"], f["A_log"], f["dt_bias"], f["dt_min"], f["dt_max"])
    H, G = f["x"].shape[2], f["Bm"].shape[2]
    Bh = np.repeat(f["Bm"], H // G, axis=2)
    Ch = np.repeat(f["Cm"], H // G, axis=2)
    contrib = np.einsum("blhp,blhn->blhpn", f["x"] * dt[..., None], Bh)
    run = np.cumsum(contrib, axis=1)                      # h_t = sum_{s<=t} dt x B^T
    want = np.einsum("blhpn,blhn->blhp", run, Ch) + f["D"][None, None, :, None] * f["x"]
    assert rel(y, want) < TIGHT and rel(hf, run[:, -1]) < TIGHT


def test_geometric_series_scalar_state():
    # P = N = 1, constant dt, A, B, C, x: h_t = dt x b (1 - a^(t+1)) / (1 - a)
    L, dt, A_log, b, c, xv, Dv = 40, 0.05, math.log(3.0), 0.7, -1.3, 0.9, 0.25
    z = math.log(math.expm1(dt))                  # softplus^-1 so that dt is exact
    a = math.exp(dt * -3.0)
    x = np.full((1, L, 1, 1), xv)
    y, hf = oracle.ssd_scan_sequential(x, np.full((1, L, 1), z), np.array([A_log]),
                                       np.full((1, L, 1, 1), b), np.full((1, L, 1, 1), c),
                                       np.array([Dv]), None, 0.0, float("inf"), None)
    t = np.arange(L)
    h = dt * xv * b * (1 - a ** (t + 1)) / (1 - a)
    assert rel(y[0, :, 0, 0], c * h + Dv * xv) < 1e-12
    assert abs(hf[0, 0, 0, 0] - h[-1]) < 1e-12 * abs(h[-1])


def test_impulse_response_decay_indexing():
    # x nonzero only at s0: y_t = dt_s0 (C_t . B_s0) x_s0 prod_{k=s0+1..t} a_k for t >= s0
    rng = np.random.default_rng(3)
    L, P, N, s0 = 24, 3, 5, 7
    f = small_inputs(Bsz=1, L=L, H=1, P=P, G=1, N=N, h0=False, unclipped=True)
    f["x"][:] = 0.0
    f["x"][0, s0, 0] = rng.standard_normal(P)
    f["D"][:] = 0.0
    y, _ = oracle.ssd_scan_sequential(*oracle_args(f))
    dt, dA = oracle.discretise(f["dt"], f["A_log"], f["dt_bias"], f["dt_min"], f["dt_max"])
    Bs0 = f["Bm"][0, s0, 0]
    for t in range(L):
        if t < s0:
            want = np.zeros(P)
        else:
            decay = math.prod(math.exp(dA[0, k, 0]) for k in range(s0 + 1, t + 1))
            want = dt[0, s0, 0] * float(f["Cm"][0, t, 0] @ Bs0) * decay * f["x"][0, s0, 0]
        np.testing.assert_allclose(y[0, t, 0], want, rtol=1e-12, atol=1e-15)


def test_full_decay_keeps_only_current_token():
    # dt*|A| huge: a_t = 0, so y_t = dt_t (C_t . B_t) x_t + D x_t and h_T = dt x_T B_T^T
    f = small_inputs(h0=True)
    f["A_log"] = np.full_like(f["A_log"], 60.0)
    f["dt_min"] = 1e-3
    y, hf = oracle.ssd_scan_sequential(*oracle_args(f))
    dt, _ = oracle.discretise(f["dt"], f["A_log"], f["dt_bias"], f["dt_min"], f["dt_max"])
    H, G = f["x"].shape[2], f["Bm"].shape[2]
    Bh = np.repeat(f["Bm"], H // G, axis=2)
    Ch = np.repeat(f["Cm"], H // G, axis=2)
    cb = np.einsum("blhn,blhn->blh", Ch, Bh)
    want = (dt * cb)[..., None] * f["x"] + f["D"][None, None, :, None] * f["x"]
    assert rel(y, want) < TIGHT
    last = np.einsum("bhp,bhn->bhpn", f["x"][:, -1] * dt[:, -1, :, None], Bh[:, -1])
    assert rel(hf, last) < TIGHT


def test_single_token_with_initial_state():
    f = small_inputs(L=1, h0=True)
    y, hf = oracle.ssd_scan_sequential(*oracle_args(f))
    dt, dA = oracle.discretise(f["dt"], f["A_log"], f["dt_bias"], f["dt_min"], f["dt_max"])
    H, G = f["x"].shape[2], f["Bm"].shape[2]
    B0 = np.repeat(f["Bm"], H // G, axis=2)[:, 0]       # [B,H,N]
    C0 = np.repeat(f["Cm"], H // G, axis=2)[:, 0]
    x0 = f["x"][:, 0]                                    # [B,H,P]
    a = np.exp(dA[:, 0])                                 # [B,H]
    want_h = a[..., None, None] * f["h0"] + dt[:, 0, :, None, None] * x0[..., None] * B0[:, :, None, :]
    want_y = np.einsum("bhpn,bhn->bhp", want_h, C0) + f["D"][None, :, None] * x0
    assert rel(hf, want_h) < TIGHT and rel(y[:, 0], want_y) < TIGHT


def test_hand_worked_three_tokens():
    # P = N = 1, dt clipped to exactly 0.5, A = -2 so a = e^-1; B = 1, C = 2, D = 0.5,
    # x = (1, 2, -1), h0 = 0.3.  By hand, with e = exp(-1):
    #   h1 = 0.3e + 0.5        y1 = 2 h1 + 0.5
    #   h2 = e h1 + 1.0        y2 = 2 h2 + 1.0
    #   h3 = e h2 - 0.5        y3 = 2 h3 - 0.5
    e = math.exp(-1.0)
    h1 = 0.3 * e + 0.5
    h2 = e * h1 + 1.0
    h3 = e * h2 - 0.5
    want = [2 * h1 + 0.5, 2 * h2 + 1.0, 2 * h3 - 0.5]
    y, hf = oracle.ssd_scan_sequential(
        np.array([1.0, 2.0, -1.0]).reshape(1, 3, 1, 1), np.zeros((1, 3, 1)),
        np.array([math.log(2.0)]), np.ones((1, 3, 1, 1)), np.full((1, 3, 1, 1), 2.0),
        np.array([0.5]), None, 0.5, 0.5, np.full((1, 1, 1, 1), 0.3))
    np.testing.assert_allclose(y.ravel(), want, rtol=1e-14)
    assert abs(hf.item() - h3) < 1e-14


# ---------------------------------------------------------------------------------
# invariants
# ---------------------------------------------------------------------------------
def test_linearity_in_x_and_h0():
    f = small_inputs(h0=False)
    g = small_inputs(h0=False, seed=9)
    y1, _ = oracle.ssd_scan_sequential(*oracle_args(f))
    f2 = dict(f)
    f2["x"] = g["x"]
    y2, _ = oracle.ssd_scan_sequential(*oracle_args(f2))
    f3 = dict(f)
    f3["x"] = f["x"] - 2.5 * g["x"]
    y3, _ = oracle.ssd_scan_sequential(*oracle_args(f3))
    assert rel(y3, y1 - 2.5 * y2) < TIGHT
    # with x = 0 the output is linear in h0
    h = small_inputs(h0=True)
    h["x"] = np.zeros_like(h["x"])
    ya, ha = oracle.ssd_scan_sequential(*oracle_args(h))
    h["h0"] = -3.0 * h["h0"]
    yb, hb = oracle.ssd_scan_sequential(*oracle_args(h))
    assert rel(yb, -3.0 * ya) < TIGHT and rel(hb, -3.0 * ha) < TIGHT


def test_split_resume_equals_one_pass():
    f = small_inputs(L=61, h0=True)
    y, hf = oracle.ssd_scan_sequential(*oracle_args(f))
    cut = 23
    a = dict(f)
    b = dict(f)
    for k in ("x", "dt", "Bm", "Cm"):
        a[k] = f[k][:, :cut]
        b[k] = f[k][:, cut:]
    ya, ha = oracle.ssd_scan_sequential(*oracle_args(a))
    b["h0"] = ha
    yb, hb = oracle.ssd_scan_sequential(*oracle_args(b))
    assert rel(np.concatenate([ya, yb], axis=1), y) < TIGHT and rel(hb, hf) < TIGHT


def test_state_size_independent_of_length():
    for L in (1, 7, 300):
        f = small_inputs(Bsz=1, L=L, H=2, P=4, G=1, N=3)
        _, hf = oracle.ssd_scan_sequential(*oracle_args(f))
        assert hf.shape == (1, 2, 4, 3)


def test_head_to_group_mapping():
    f = small_inputs(Bsz=1, L=19, H=4, P=3, G=2, N=4, h0=False)
    f["Bm"][:, :, 1] = 0.0                   # group 1 (heads 2, 3) gets no input
    y, hf = oracle.ssd_scan_sequential(*oracle_args(f))
    skip = f["D"][None, None, :, None] * f["x"]
    assert rel(y[:, :, 2:], skip[:, :, 2:]) < TIGHT
    assert np.all(hf[:, 2:] == 0.0)
    assert np.max(np.abs(y[:, :, :2] - skip[:, :, :2])) > 1e-3


# ---------------------------------------------------------------------------------
# discretisation
# ---------------------------------------------------------------------------------
def test_dt_softplus_and_clip():
    assert oracle.dt_value(0.0, 0.0, 0.0, 10.0) == pytest.approx(math.log(2.0), rel=1e-15)
    for z in (-7.0, -1.2, 0.3, 4.0, 25.0):
        assert oracle.dt_value(z, 0.0, 0.0, 1e9) == pytest.approx(math.log1p(math.exp(z)),
                                                                  rel=1e-14)
    assert oracle.dt_value(800.0, 0.0, 0.0, 1e9) == pytest.approx(800.0, rel=1e-15)
    assert oracle.dt_value(5.0, 0.0, 1e-3, 0.1) == 0.1
    assert oracle.dt_value(-30.0, 0.0, 1e-3, 0.1) == 1e-3
    # the bias is added before the softplus
    assert oracle.dt_value(-2.5, 0.7, 0.0, 1e9) == oracle.dt_value(-1.8, 0.0, 0.0, 1e9)
    np.testing.assert_allclose(oracle.softplus(np.array([-3.0, 0.0, 2.0])),
                               np.log1p(np.exp([-3.0, 0.0, 2.0])), rtol=1e-15)


# ---------------------------------------------------------------------------------
# conv window and cached decode
# ---------------------------------------------------------------------------------
def test_causal_conv_matches_library_convolution():
    rng = np.random.default_rng(1)
    Bsz, L, Cc, K = 2, 11, 5, 4
    xbc = rng.standard_normal((Bsz, L, Cc))
    w = rng.standard_normal((Cc, K))
    bias = rng.standard_normal(Cc)
    out, cs = oracle.causal_conv1d(xbc, w, bias)
    for b in range(Bsz):
        for c in range(Cc):
            pre = np.convolve(xbc[b, :, c], w[c, ::-1])[:L] + bias[c]
            np.testing.assert_allclose(out[b, :, c], pre * expit(pre), rtol=1e-13, atol=1e-15)
            np.testing.assert_array_equal(cs[b, c], xbc[b, L - (K - 1):, c])
    # a sequence shorter than the window leaves zeros in the oldest slots
    _, cs2 = oracle.causal_conv1d(xbc[:, :2], w, bias)
    np.testing.assert_array_equal(cs2[:, :, 0], 0.0)
    np.testing.assert_array_equal(cs2[:, :, 1:], np.transpose(xbc[:, :2], (0, 2, 1)))


def _block_reference(xbc, dt_raw, prm, H, P, G, N):
    """Full recompute: conv over the whole raw sequence, split, SSD recurrence."""
    u, _ = oracle.causal_conv1d(xbc, prm["conv_w"], prm["conv_b"])
    Bsz, L, _ = xbc.shape
    x = u[..., :H * P].reshape(Bsz, L, H, P)
    Bm = u[..., H * P:H * P + G * N].reshape(Bsz, L, G, N)
    Cm = u[..., H * P + G * N:].reshape(Bsz, L, G, N)
    return oracle.ssd_scan_sequential(x, dt_raw, prm["A_log"], Bm, Cm, prm["D"],
                                      prm["dt_bias"], prm["dt_min"], prm["dt_max"], None)


@pytest.mark.parametrize("G", [1, 2])
def test_prefill_then_decode_equals_recompute(G):
    # [blog §5.1]: cached decode (O(1) per token) must reproduce the O(L^2) recompute.
    H, P, N, K, Bsz, L, k = 4, 4, 6, 4, 2, 13, 5
    prm = f64(S.decode_params(H, P, G, N, K, seed=7))
    seq = S.raw_xbc_sequence(Bsz, L + k, H, P, G, N, dtype="f32", seed=8)
    xbc, dt_raw = seq["xBC"][1], seq["dt"][1]
    y_full, h_full = _block_reference(xbc, dt_raw, prm, H, P, G, N)
    # prefill the first L tokens, keep the caches
    u, conv_state = oracle.causal_conv1d(xbc[:, :L], prm["conv_w"], prm["conv_b"])
    x = u[..., :H * P].reshape(Bsz, L, H, P)
    Bm = u[..., H * P:H * P + G * N].reshape(Bsz, L, G, N)
    Cm = u[..., H * P + G * N:].reshape(Bsz, L, G, N)
    _, ssm = oracle.ssd_scan_sequential(x, dt_raw[:, :L], prm["A_log"], Bm, Cm, prm["D"],
                                        prm["dt_bias"], prm["dt_min"], prm["dt_max"], None)
    for j in range(k):
        t = L + j
        y_t, ssm, conv_state = oracle.decode_step(
            ssm, conv_state, xbc[:, t], dt_raw[:, t], prm["A_log"], prm["D"], prm["dt_bias"],
            prm["dt_min"], prm["dt_max"], prm["conv_w"], prm["conv_b"], H, P, G, N)
        assert rel(y_t, y_full[:, t]) < TIGHT
        np.testing.assert_array_equal(conv_state, np.transpose(xbc[:, t - K + 2:t + 1], (0, 2, 1)))
    assert rel(ssm, h_full) < TIGHT
