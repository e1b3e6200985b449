"""Pins of the oracle's Bi-WKV and gate against closed forms, hand-expanded
sums, invariants and the pages' second (RNN) form.

Sources: "Vision-RWKV Backbone", Linear Complexity Bidirectional Attention,
eq. 5 (summation form), eq. 6-7 (RNN form with hidden states a, b, c, d);
Overall Architecture, eq. 2 (sigma(R) (.) wkv).
"""
import numpy as np
import pytest

from linear_complexity_vision_b200 import synth


def _rand(B, T, C, seed=0, kscale=1.0, wlo=-3, whi=3):
    rng = np.random.default_rng(seed)
    k = kscale * rng.standard_normal((B, T, C))
    v = rng.standard_normal((B, T, C))
    w = rng.uniform(wlo, whi, C)
    u = rng.normal(0, 0.5, C)
    return k, v, w, u


def _col(a):
    return np.asarray(a, dtype=np.float64).reshape(1, -1, 1)


def test_T1_returns_v(oracle_mod):
    k, v, w, u = _rand(3, 1, 5)
    np.testing.assert_allclose(oracle_mod.biwkv_direct(k, v, w, u), v, rtol=4e-16)
    np.testing.assert_allclose(oracle_mod.biwkv_rnn(k, v, w, u), v, rtol=1e-15)


def test_T2_closed_form(oracle_mod):
    # neighbours at distance 1 carry no decay: exponent -(1-1)/T*w = 0
    k0, k1, v0, v1, w, u = 0.3, -1.2, 2.0, -0.7, 1.7, 0.4
    out = oracle_mod.biwkv_direct(_col([k0, k1]), _col([v0, v1]), [w], [u])[0, :, 0]
    e = np.exp
    want0 = (e(k1) * v1 + e(u + k0) * v0) / (e(k1) + e(u + k0))
    want1 = (e(k0) * v0 + e(u + k1) * v1) / (e(k0) + e(u + k1))
    np.testing.assert_allclose(out, [want0, want1], rtol=1e-14)


def test_T3_hand_expanded(oracle_mod):
    k = [0.5, -0.25, 1.5]
    v = [1.0, -2.0, 3.0]
    w, u = 2.4, -0.3
    e = np.exp
    # T = 3: distance 2 decays by exp(-(2-1)/3 * w); the diagonal uses e^{u+k}
    wts = [
        [e(u + k[0]), e(k[1]), e(-w / 3 + k[2])],
        [e(k[0]), e(u + k[1]), e(k[2])],
        [e(-w / 3 + k[0]), e(k[1]), e(u + k[2])],
    ]
    want = [sum(a * b for a, b in zip(row, v)) / sum(row) for row in wts]
    out = oracle_mod.biwkv_direct(_col(k), _col(v), [w], [u])[0, :, 0]
    np.testing.assert_allclose(out, want, rtol=1e-14)
    np.testing.assert_allclose(oracle_mod.biwkv_rnn(_col(k), _col(v), [w], [u])[0, :, 0],
                               want, rtol=1e-13)


def test_T4_hand_expanded_negative_decay(oracle_mod):
    k = [0.1, 0.9, -0.4, 0.2]
    v = [-1.0, 0.5, 2.5, -3.0]
    w, u = -1.6, 0.8  # negative w: far tokens weigh more (flexible decay)
    e = np.exp
    q = w / 4
    wts = [
        [e(u + k[0]), e(k[1]), e(-q + k[2]), e(-2 * q + k[3])],
        [e(k[0]), e(u + k[1]), e(k[2]), e(-q + k[3])],
        [e(-q + k[0]), e(k[1]), e(u + k[2]), e(k[3])],
        [e(-2 * q + k[0]), e(-q + k[1]), e(k[2]), e(u + k[3])],
    ]
    want = [sum(a * b for a, b in zip(row, v)) / sum(row) for row in wts]
    out = oracle_mod.biwkv_direct(_col(k), _col(v), [w], [u])[0, :, 0]
    np.testing.assert_allclose(out, want, rtol=1e-14)
    for f in (oracle_mod.biwkv_rnn, oracle_mod.biwkv_rnn_literal):
        np.testing.assert_allclose(f(_col(k), _col(v), [w], [u])[0, :, 0], want,
                                   rtol=1e-13)


def test_constant_v_and_convexity(oracle_mod):
    k, v, w, u = _rand(2, 37, 6, seed=1, kscale=2.0, wlo=-8, whi=8)
    c = np.full_like(v, -1.25)
    np.testing.assert_allclose(oracle_mod.biwkv_direct(k, c, w, u), c, rtol=1e-14)
    out = oracle_mod.biwkv_direct(k, v, w, u)
    # a weighted mean stays within the range of its column
    assert np.all(out <= v.max(axis=1, keepdims=True) + 1e-12)
    assert np.all(out >= v.min(axis=1, keepdims=True) - 1e-12)


def test_affine_in_v_and_shift_invariant_in_k(oracle_mod):
    k, v, w, u = _rand(2, 29, 5, seed=2)
    base = oracle_mod.biwkv_direct(k, v, w, u)
    np.testing.assert_allclose(oracle_mod.biwkv_direct(k, 3.0 * v - 0.5, w, u),
                               3.0 * base - 0.5, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(oracle_mod.biwkv_direct(k + 80.0, v, w, u), base,
                               rtol=1e-12, atol=1e-12)


def test_reversal_symmetry(oracle_mod):
    k, v, w, u = _rand(2, 33, 4, seed=3)
    out = oracle_mod.biwkv_direct(k, v, w, u)
    rev = oracle_mod.biwkv_direct(k[:, ::-1], v[:, ::-1], w, u)
    np.testing.assert_allclose(rev[:, ::-1], out, rtol=1e-13)


def test_w0_u0_is_softmax_average(oracle_mod):
    k, v, _, _ = _rand(2, 21, 3, seed=4)
    C = k.shape[2]
    out = oracle_mod.biwkv_direct(k, v, np.zeros(C), np.zeros(C))
    p = np.exp(k - k.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    want = (p * v).sum(axis=1, keepdims=True)
    np.testing.assert_allclose(out, np.broadcast_to(want, out.shape), rtol=1e-13)


def test_w0_with_bonus_closed_form(oracle_mod):
    k, v, _, u = _rand(1, 17, 4, seed=5)
    C = k.shape[2]
    out = oracle_mod.biwkv_direct(k, v, np.zeros(C), u)
    ek = np.exp(k)
    S = (ek * v).sum(axis=1, keepdims=True)
    Z = ek.sum(axis=1, keepdims=True)
    eu = np.exp(u + k)
    want = (S - ek * v + eu * v) / (Z - ek + eu)
    np.testing.assert_allclose(out, want, rtol=1e-13)


def test_large_positive_w_leaves_three_taps(oracle_mod):
    T = 9
    k, v, _, u = _rand(1, T, 3, seed=6)
    C = k.shape[2]
    w = np.full(C, 60.0 * T)  # exp(-(d-1)*60) for d >= 2: below 1e-26
    out = oracle_mod.biwkv_direct(k, v, w, u)
    e = np.exp
    for c in range(C):
        for t in range(T):
            num = e(u[c] + k[0, t, c]) * v[0, t, c]
            den = e(u[c] + k[0, t, c])
            for i in (t - 1, t + 1):
                if 0 <= i < T:
                    num += e(k[0, i, c]) * v[0, i, c]
                    den += e(k[0, i, c])
            assert out[0, t, c] == pytest.approx(num / den, rel=1e-14, abs=1e-15)


def test_large_bonus_returns_v(oracle_mod):
    k, v, w, _ = _rand(1, 23, 3, seed=7)
    out = oracle_mod.biwkv_direct(k, v, w, np.full(3, 200.0))
    np.testing.assert_allclose(out, v, rtol=4e-16, atol=0)


@pytest.mark.parametrize("T,kscale,wlo,whi", [(5, 1.0, -3, 3), (64, 2.0, -8, 8),
                                               (196, 1.0, -5, 5)])
def test_direct_equals_rnn(oracle_mod, T, kscale, wlo, whi):
    k, v, w, u = _rand(2, T, 6, seed=T, kscale=kscale, wlo=wlo, whi=whi)
    d = oracle_mod.biwkv_direct(k, v, w, u)
    np.testing.assert_allclose(oracle_mod.biwkv_rnn(k, v, w, u), d, rtol=1e-11, atol=1e-12)
    if T <= 64:
        np.testing.assert_allclose(oracle_mod.biwkv_rnn_literal(k, v, w, u), d,
                                   rtol=1e-8, atol=1e-9)


def test_points_match_full(oracle_mod):
    k, v, w, u = _rand(3, 40, 7, seed=8)
    full = oracle_mod.biwkv_direct(k, v, w, u)
    idx = np.array([0, 5, 17, full.size - 1, 3 * 40 * 7 // 2])
    np.testing.assert_array_equal(oracle_mod.biwkv_points(k, v, w, u, idx),
                                  full.reshape(-1)[idx])


def test_gate_endpoints(oracle_mod):
    rng = np.random.default_rng(9)
    wkv = rng.standard_normal(100)
    np.testing.assert_allclose(oracle_mod.gate(np.zeros(100), wkv), wkv / 2, rtol=1e-15)
    np.testing.assert_allclose(oracle_mod.gate(np.full(100, 50.0), wkv), wkv, rtol=1e-15)
    np.testing.assert_allclose(oracle_mod.gate(np.full(100, -800.0), wkv), 0.0, atol=0)
    r = rng.standard_normal(100)
    # sigma(r) + sigma(-r) = 1
    np.testing.assert_allclose(oracle_mod.gate(r, wkv) + oracle_mod.gate(-r, wkv), wkv,
                               rtol=1e-14, atol=1e-15)


def test_spatial_core_composition(oracle_mod):
    wl = synth.workload(3, B=2, H=5, W=6, C=16)
    inp = wl.generate()
    out = oracle_mod.spatial_core(inp["r"], inp["k"], inp["v"], inp["w"], inp["u"],
                                  wl.H, wl.W, 1, 0.25, inp["mu_r"], inp["mu_k"], inp["mu_v"])
    rnn = oracle_mod.spatial_core(inp["r"], inp["k"], inp["v"], inp["w"], inp["u"],
                                  wl.H, wl.W, 1, 0.25, inp["mu_r"], inp["mu_k"], inp["mu_v"],
                                  method="rnn")
    np.testing.assert_allclose(out, rnn, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("qshift_on,gate_on", [(True, True), (True, False), (False, True)])
def test_spatial_core_points_match_full(oracle_mod, qshift_on, gate_on):
    wl = synth.workload(3, B=2, H=6, W=7, C=20)
    inp = wl.generate()
    r, k, v = inp["r"], inp["k"], inp["v"]
    args = (wl.H, wl.W, 1, 0.25, inp["mu_r"], inp["mu_k"], inp["mu_v"])
    if gate_on:
        full = oracle_mod.spatial_core(r, k, v, inp["w"], inp["u"], *args, qshift_on=qshift_on)
    else:
        ks = oracle_mod.qshift(k, wl.H, wl.W, 1, 0.25, inp["mu_k"])
        vs = oracle_mod.qshift(v, wl.H, wl.W, 1, 0.25, inp["mu_v"])
        full = oracle_mod.biwkv_direct(ks, vs, inp["w"], inp["u"])
    idx = np.arange(0, full.size, 7)
    pts = oracle_mod.spatial_core_points(r, k, v, inp["w"], inp["u"], wl.H, wl.W, idx, 1, 0.25,
                                         inp["mu_r"], inp["mu_k"], inp["mu_v"],
                                         qshift_on=qshift_on, gate_on=gate_on)
    np.testing.assert_allclose(pts, full.reshape(-1)[idx], rtol=1e-13, atol=1e-14)
