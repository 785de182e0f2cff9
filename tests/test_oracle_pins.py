"""Pins for the fp64 oracle: checks against things other than the oracle itself.

Each test ties one oracle function to a hand-derived value, a closed form, a
library routine computing the same quantity by a different method, or an
invariant the operator must satisfy (recurrence = convolution, impulse
response = filter, prompt state + decode = full convolution, linearity, shift
invariance).  A dropped term, a wrong sign, a conjugated pole, an off-by-one
filter index or a wrong channel->head map fails at least one of them.
"""
import cmath
import json
import os

import numpy as np
import pytest

GOLD = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")


def _cplx(a):
    a = np.asarray(a, dtype=np.float64)
    return a[..., 0] + 1j * a[..., 1]


def _rand_params(rng, H, d, rmin=0.3, rmax=0.95):
    mag = rng.uniform(rmin, rmax, size=(H, d))
    arg = rng.uniform(0, np.pi, size=(H, d))
    lam = mag * np.exp(1j * arg)
    R = (rng.normal(size=(H, d)) + 1j * rng.normal(size=(H, d))) / np.sqrt(2 * d)
    D = rng.normal(size=H)
    return lam, R, D


def _rand_act(rng, B, L, Dch):
    return [rng.normal(size=(B, L, Dch)) for _ in range(3)]


# ---------------------------------------------------------------- golden values
def test_golden_real_pole(oracle):
    g = json.load(open(GOLD))["real_pole"]
    lam, R, D = _cplx(g["lam"]), _cplx(g["R"]), np.array(g["Dskip"])
    h = oracle.filter_from_modes(lam, R, D, 4)
    np.testing.assert_array_equal(h[0], g["h"])
    k = np.array(g["k"]).reshape(1, 3, 1)
    v = np.array(g["v"]).reshape(1, 3, 1)
    q = np.array(g["q"]).reshape(1, 3, 1)
    y = oracle.conv_direct(q, k, v, h[:, :3], H=1)
    np.testing.assert_array_equal(y.ravel(), g["y"])
    s = oracle.prompt_state(k, v, lam, H=1)
    assert s.shape == (1, 1, 1)
    assert s[0, 0, 0] == complex(*g["state"])
    yr, sr = oracle.recurrent(q, k, v, lam, R, D, H=1)
    np.testing.assert_array_equal(yr.ravel(), g["y"])
    assert sr[0, 0, 0] == complex(*g["state"])
    dd = g["decode"]
    y1, s1 = oracle.decode_step(np.full((1, 1), dd["q"]), np.full((1, 1), dd["k"]),
                                np.full((1, 1), dd["v"]), lam, R, D, 1, s)
    assert y1[0, 0] == dd["y"]
    assert s1[0, 0, 0] == complex(*dd["state"])


def test_golden_imaginary_pole(oracle):
    g = json.load(open(GOLD))["imaginary_pole"]
    lam, D = _cplx(g["lam"]), np.array(g["Dskip"])
    h1 = oracle.filter_from_modes(lam, _cplx(g["R_one"]), D, 6)
    np.testing.assert_array_equal(h1[0], g["h_R_one"])
    hi = oracle.filter_from_modes(lam, _cplx(g["R_i"]), D, 6)
    np.testing.assert_array_equal(hi[0], g["h_R_i"])


def test_golden_decode_complex_state(oracle):
    g = json.load(open(GOLD))["decode_complex_state"]
    lam, R, D = _cplx(g["lam"]), _cplx(g["R"]), np.array(g["Dskip"])
    s0 = np.array([[[complex(*g["state"])]]])
    y, s = oracle.decode_step(np.full((1, 1), g["q"]), np.full((1, 1), g["k"]),
                              np.full((1, 1), g["v"]), lam, R, D, 1, s0)
    assert y[0, 0] == g["y"]
    assert s[0, 0, 0] == complex(*g["new_state"])


def test_golden_two_heads(oracle):
    g = json.load(open(GOLD))["two_heads"]
    lam, R, D = _cplx(g["lam"]), _cplx(g["R"]), np.array(g["Dskip"])
    v = np.array(g["v_rows"], dtype=np.float64)[None]
    k = np.ones_like(v)
    q = np.ones_like(v)
    h = oracle.filter_from_modes(lam, R, D, 3)
    y = oracle.conv_direct(q, k, v, h, H=2)
    np.testing.assert_array_equal(y[0], np.array(g["y_rows"], dtype=np.float64))
    yr, _ = oracle.recurrent(q, k, v, lam, R, D, H=2)
    np.testing.assert_array_equal(yr[0], np.array(g["y_rows"], dtype=np.float64))


# ---------------------------------------------------------------- closed forms
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_single_pole_closed_forms(oracle, seed):
    """d = 1: h_j = Re(R lam^(j-1)); step response and all-ones state are geometric sums."""
    rng = np.random.default_rng(seed)
    lam = 0.97 * np.exp(1j * rng.uniform(0, np.pi))
    R = complex(rng.normal(), rng.normal())
    D = rng.normal()
    L = 300
    h = oracle.filter_from_modes(np.array([[lam]]), np.array([[R]]), np.array([D]), L)[0]
    assert h[0] == D
    ref = np.array([(R * cmath.exp((j - 1) * cmath.log(lam))).real for j in range(1, L)])
    np.testing.assert_allclose(h[1:], ref, rtol=0, atol=1e-12)
    # step response  sum_{j=1}^{t} h_j = Re(R (1 - lam^t) / (1 - lam))
    t = np.arange(1, L)
    closed = (R * (1 - lam ** t) / (1 - lam)).real
    np.testing.assert_allclose(np.cumsum(h[1:]), closed, rtol=0, atol=1e-11)
    # state after an all-ones prompt: s = (1 - lam^L) / (1 - lam)
    ones = np.ones((1, L, 1))
    s = oracle.prompt_state(ones, ones, np.array([[lam]]), H=1)[0, 0, 0]
    assert abs(s - (1 - lam ** L) / (1 - lam)) < 1e-11
    # the recurrence from zero leaves the same state
    _, sr = oracle.recurrent(ones, ones, ones, np.array([[lam]]), np.array([[R]]),
                             np.array([D]), H=1)
    assert abs(sr[0, 0, 0] - (1 - lam ** L) / (1 - lam)) < 1e-11


def test_zero_pole_two_tap(oracle):
    """lam = 0: filter [Dskip, Re sum R, 0, ...]; y_t = q_t (Dskip u_t + Re(sum R) u_{t-1})."""
    rng = np.random.default_rng(7)
    d, L = 3, 20
    R = rng.normal(size=(1, d)) + 1j * rng.normal(size=(1, d))
    D = np.array([rng.normal()])
    lam = np.zeros((1, d), dtype=complex)
    h = oracle.filter_from_modes(lam, R, D, L)[0]
    assert h[0] == D[0]
    assert abs(h[1] - R.sum().real) < 1e-15
    assert np.all(h[2:] == 0.0)
    q, k, v = _rand_act(rng, 1, L, 1)
    u = (k * v)[0, :, 0]
    expect = q[0, :, 0] * (D[0] * u + R.sum().real * np.concatenate([[0.0], u[:-1]]))
    y, _ = oracle.recurrent(q, k, v, lam, R, D, H=1)
    np.testing.assert_allclose(y[0, :, 0], expect, rtol=0, atol=1e-12)
    yd = oracle.conv_direct(q, k, v, h[None], H=1)
    np.testing.assert_allclose(yd[0, :, 0], expect, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- library routines
def test_conv_matches_numpy_convolve(oracle):
    rng = np.random.default_rng(3)
    B, L, Dch, H, d = 2, 37, 6, 3, 4
    lam, R, D = _rand_params(rng, H, d)
    q, k, v = _rand_act(rng, B, L, Dch)
    h = oracle.filter_from_modes(lam, R, D, L)
    y = oracle.conv_direct(q, k, v, h, H=H)
    ch = Dch // H
    for b in range(B):
        for c in range(Dch):
            z = np.convolve(h[c // ch], k[b, :, c] * v[b, :, c])[:L]
            np.testing.assert_allclose(y[b, :, c], q[b, :, c] * z, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("L,N", [(5, 16), (64, 128), (100, 256)])
def test_spectrum_matches_numpy_rfft(oracle, L, N):
    rng = np.random.default_rng(L)
    h = rng.normal(size=(2, L))
    spec = oracle.spectrum(h, N)
    ref = np.fft.rfft(np.pad(h, ((0, 0), (0, N - L))), axis=1)
    np.testing.assert_allclose(spec, ref, rtol=0, atol=1e-10 * np.abs(ref).max())
    bins = [0, 1, N // 4, N // 2 - 1, N // 2]
    np.testing.assert_allclose(oracle.spectrum(h, N, bins=bins), ref[:, bins],
                               rtol=0, atol=1e-10 * np.abs(ref).max())


def test_filter_matches_matrix_power_form(oracle):
    """h_j = Re(R^T diag(lam)^(j-1) 1): the same filter via numpy.linalg.matrix_power."""
    rng = np.random.default_rng(11)
    H, d, L = 2, 5, 40
    lam, R, D = _rand_params(rng, H, d)
    h = oracle.filter_from_modes(lam, R, D, L)
    for hd in range(H):
        A = np.diag(lam[hd])
        for j in range(1, L):
            ref = (R[hd] @ np.linalg.matrix_power(A, j - 1) @ np.ones(d)).real
            assert abs(h[hd, j] - ref) < 1e-12
        assert h[hd, 0] == D[hd]


# ---------------------------------------------------------------- invariants
@pytest.mark.parametrize("B,L,Dch,H,d", [(1, 50, 4, 2, 3), (2, 129, 6, 3, 8), (1, 300, 2, 1, 16)])
def test_recurrence_equals_direct_convolution(oracle, B, L, Dch, H, d):
    rng = np.random.default_rng(B * 1000 + L)
    lam, R, D = _rand_params(rng, H, d)
    q, k, v = _rand_act(rng, B, L, Dch)
    h = oracle.filter_from_modes(lam, R, D, L)
    yd = oracle.conv_direct(q, k, v, h, H=H)
    yr, s = oracle.recurrent(q, k, v, lam, R, D, H=H)
    assert np.abs(yd - yr).max() <= 1e-10 * np.abs(yd).max()
    s2 = oracle.prompt_state(k, v, lam, H=H)
    assert np.abs(s - s2).max() <= 1e-10 * np.abs(s2).max()


def test_impulse_response_is_filter(oracle):
    rng = np.random.default_rng(5)
    H, d, L, Dch = 3, 6, 64, 6
    lam, R, D = _rand_params(rng, H, d)
    h = oracle.filter_from_modes(lam, R, D, L)
    k = np.zeros((1, L, Dch)); k[0, 0, :] = 1.0
    v = np.ones((1, L, Dch)); q = np.ones((1, L, Dch))
    yr, _ = oracle.recurrent(q, k, v, lam, R, D, H=H)
    yd = oracle.conv_direct(q, k, v, h, H=H)
    for c in range(Dch):
        np.testing.assert_allclose(yr[0, :, c], h[c // (Dch // H)], rtol=0, atol=1e-13)
        np.testing.assert_array_equal(yd[0, :, c], h[c // (Dch // H)])


@pytest.mark.parametrize("L,T", [(1, 5), (40, 17), (128, 64)])
def test_prompt_state_then_decode_equals_full_convolution(oracle, L, T):
    rng = np.random.default_rng(L + T)
    B, Dch, H, d = 2, 4, 2, 5
    lam, R, D = _rand_params(rng, H, d)
    q, k, v = _rand_act(rng, B, L + T, Dch)
    h = oracle.filter_from_modes(lam, R, D, L + T)
    y_full = oracle.conv_direct(q, k, v, h, H=H)
    s = oracle.prompt_state(k[:, :L], v[:, :L], lam, H=H)
    ys = []
    for t in range(L, L + T):
        yt, s = oracle.decode_step(q[:, t], k[:, t], v[:, t], lam, R, D, H, s)
        ys.append(yt)
    y_dec = np.stack(ys, axis=1)
    err = np.abs(y_dec - y_full[:, L:]).max()
    assert err <= 1e-11 * np.abs(y_full).max()


def test_linearity_and_shift_invariance_brute_force(oracle):
    rng = np.random.default_rng(9)
    H, d, L, Dch = 1, 2, 8, 1
    lam, R, D = _rand_params(rng, H, d)
    h = oracle.filter_from_modes(lam, R, D, L)
    ones = np.ones((1, L, Dch))
    # brute-force Toeplitz: column j of the operator is the response to e_j
    T = np.zeros((L, L))
    for j in range(L):
        e = np.zeros((1, L, Dch)); e[0, j, 0] = 1.0
        T[:, j] = oracle.conv_direct(ones, e, ones, h, H=1)[0, :, 0]
    for i in range(L):
        for j in range(L):
            assert T[i, j] == (h[0, i - j] if i >= j else 0.0)
    a, b = rng.normal(size=(1, L, Dch)), rng.normal(size=(1, L, Dch))
    ya = oracle.conv_direct(ones, a, ones, h, H=1)
    yb = oracle.conv_direct(ones, b, ones, h, H=1)
    yab = oracle.conv_direct(ones, 2.0 * a - 3.0 * b, ones, h, H=1)
    np.testing.assert_allclose(yab, 2.0 * ya - 3.0 * yb, rtol=0, atol=1e-12)


def test_gates_enter_as_products(oracle):
    """q gates the output, k and v gate the input symmetrically (u = k*v)."""
    rng = np.random.default_rng(21)
    lam, R, D = _rand_params(rng, 1, 3)
    q, k, v = _rand_act(rng, 1, 20, 2)
    h = oracle.filter_from_modes(lam, R, D, 20)
    y1 = oracle.conv_direct(q, k, v, h, H=1)
    y2 = oracle.conv_direct(q, v, k, h, H=1)
    np.testing.assert_allclose(y1, y2, rtol=1e-14, atol=0)
    y3 = oracle.conv_direct(2 * q, k, v, h, H=1)
    np.testing.assert_allclose(y3, 2 * y1, rtol=1e-14, atol=0)


def test_workload_generator_is_deterministic_and_distributed():
    """The seeded generator reproduces itself and matches the stated distributions."""
    from distilled_ssm_decode_b200 import workloads as W
    w = W.WORKLOADS["mid_bf16"]
    p1, p2 = W.params(w), W.params(w)
    np.testing.assert_array_equal(p1.lam, p2.lam)
    mag = np.abs(p1.lam)
    assert mag.min() >= w.rmin - 1e-6 and mag.max() <= w.rmax + 1e-6
    assert np.angle(p1.lam).min() >= -1e-6 and np.angle(p1.lam).max() <= np.pi + 1e-6
    q, k, v = W.prefill_inputs(w, B=1, L=64, Dch=32)
    assert q.dtype == w.torch_dtype and q.shape == (1, 64, 32)
    q2, _, _ = W.prefill_inputs(w, B=1, L=64, Dch=32)
    assert (q.float() == q2.float()).all()
    a = W.decode_inputs(w, step=3, B=2, Dch=16)[0]
    b = W.decode_inputs(w, step=3, B=2, Dch=16)[0]
    c = W.decode_inputs(w, step=4, B=2, Dch=16)[0]
    assert (a.float() == b.float()).all() and not (a.float() == c.float()).all()


# ---------------------------------------------------------------- modal truncation
def test_truncation_selection_hand_example(oracle):
    """Scores |R|/(1-|lambda|) worked by hand: lambda = [1/2, 9/10, 0, i/2], R = [1, 1/10, 1/2, 3]
    give 2, 1, 1/2, 6, so the ranking is modes 3, 0, 1, 2; kept modes come out in index order."""
    lam = np.array([[0.5, 0.9, 0.0, 0.5j]])
    R = np.array([[1.0, 0.1, 0.5, 3.0]], dtype=complex)
    expect = {0: [], 1: [3], 2: [0, 3], 3: [0, 1, 3], 4: [0, 1, 2, 3]}
    dropped_scores = {0: 9.5, 1: 3.5, 2: 1.5, 3: 0.5, 4: 0.0}
    for k, ids in expect.items():
        kept, lo, ro, b, e1, e2 = oracle.modal_truncate(lam, R, k, J=4000)
        assert kept[0].tolist() == ids
        assert np.array_equal(lo[0], lam[0, ids]) and np.array_equal(ro[0], R[0, ids])
        assert b[0] == pytest.approx(dropped_scores[k], rel=1e-15)
    # equal scores: the lower index wins
    kept, *_ = oracle.modal_truncate(np.array([[0.5, 0.5]]), np.array([[1.0, -1.0]], dtype=complex), 1)
    assert kept[0].tolist() == [0]


@pytest.mark.parametrize("lam,R", [(0.8, 1.5), (0.6 * cmath.exp(1j), 0.3 - 0.7j), (-0.95j, 2j), (0.0, 1.0)])
def test_truncation_single_mode_closed_form(oracle, lam, R):
    """Dropping the only mode leaves dh_j = Re(R lambda^(j-1)).  Closed forms of its norms:
    sum_j dh_j^2 = Re(R^2 / (1 - lambda^2)) / 2 + |R|^2 / (1 - |lambda|^2) / 2 (from
    Re(z)^2 = (z^2 + 2|z|^2 + conj(z)^2) / 4 and geometric series), and for a positive real pole
    and residue sum_j |dh_j| = R / (1 - lambda), which the bound then equals."""
    lam_a, R_a = np.array([[lam]], dtype=complex), np.array([[R]], dtype=complex)
    kept, lo, ro, b, e1, e2 = oracle.modal_truncate(lam_a, R_a, 0, J=5000)
    l2sq = (R * R / (1 - lam * lam)).real / 2 + abs(R) ** 2 / (1 - abs(lam) ** 2) / 2
    assert e2[0] ** 2 == pytest.approx(l2sq, rel=1e-12)
    assert b[0] == pytest.approx(abs(R) / (1 - abs(lam)), rel=1e-15)
    assert e1[0] <= b[0] * (1 + 1e-12)
    if isinstance(lam, float) and lam > 0:
        assert e1[0] == pytest.approx(R / (1 - lam), rel=1e-12)


@pytest.mark.parametrize("seed", [0, 1])
def test_truncation_splits_the_filter(oracle, seed):
    """Kept modes' filter + dropped modes' filter = the full filter (brute force), the direct l1/l2
    errors are the norms of that difference, and the l1 error never exceeds the bound."""
    rng = np.random.default_rng(seed)
    H, d, J = 3, 9, 3000
    lam, R, D = _rand_params(rng, H, d, rmin=0.2, rmax=0.97)
    h = oracle.filter_from_modes(lam, R, D, J + 1)
    for k in (0, 3, 8, 9):
        kept, lo, ro, b, e1, e2 = oracle.modal_truncate(lam, R, k, J=J)
        hk = oracle.filter_from_modes(lo, ro, D, J + 1) if k else np.tile(D[:, None], (1, J + 1)) * np.eye(1, J + 1)
        dh = (h - hk)[:, 1:]
        assert np.allclose(np.abs(dh).sum(1), e1, rtol=1e-10, atol=1e-14)
        assert np.allclose(np.sqrt((dh ** 2).sum(1)), e2, rtol=1e-10, atol=1e-14)
        assert np.all(e1 <= b * (1 + 1e-12))
        assert np.array_equal(hk[:, 0], D)
        if k == d:
            assert np.all(e2 == 0) and np.all(b == 0)
