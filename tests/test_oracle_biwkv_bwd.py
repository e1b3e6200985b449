"""Pins of the oracle's Bi-WKV backward pass (derivatives of eq. 5 of
"Vision-RWKV Backbone", Linear Complexity Bidirectional Attention).

The pages put the backward formulas in an appendix they do not reproduce, so
the oracle writes out the chain rule of eq. 5.  These tests tie it to
something other than itself:
  - central finite differences of the forward oracle (eq. 5 summed directly,
    itself pinned by hand-worked values) for every gradient;
  - invariants of eq. 5: adding a constant to every k of a column leaves wkv
    unchanged (sum_i dL/dk_i = 0); wkv_t is a weighted mean of v
    (sum_i dwkv_t/dv_i = 1); with T = 2 every off-diagonal distance is 1, so w
    drops out (dL/dw = 0); with T = 1, wkv = v;
  - the per-column routine agrees with the whole-tensor one.
"""
import numpy as np
import pytest


def _loss(oracle, k, v, w, u, g):
    return float(np.sum(g * oracle.biwkv_direct(k, v, w, u)))


def _inputs(seed, B=2, T=7, C=3, wscale=2.0):
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((B, T, C))
    v = rng.standard_normal((B, T, C))
    g = rng.standard_normal((B, T, C))
    w = rng.uniform(-wscale, wscale, C)
    u = rng.standard_normal(C)
    return k, v, w, u, g


@pytest.mark.parametrize("seed,T", [(0, 7), (1, 12), (2, 3)])
def test_gradients_match_finite_differences(oracle_mod, seed, T):
    k, v, w, u, g = _inputs(seed, T=T)
    gk, gv, gw, gu = oracle_mod.biwkv_bwd(k, v, w, u, g)
    h = 1e-6
    B, _, C = k.shape
    for name, arr, grad in (("k", k, gk), ("v", v, gv)):
        fd = np.empty_like(arr)
        for idx in np.ndindex(arr.shape):
            a0 = arr[idx]
            arr[idx] = a0 + h
            lp = _loss(oracle_mod, k, v, w, u, g)
            arr[idx] = a0 - h
            lm = _loss(oracle_mod, k, v, w, u, g)
            arr[idx] = a0
            fd[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(grad, fd, rtol=1e-6, atol=1e-8, err_msg=name)
    # w and u are shared by the batch: the oracle reports per-batch parts
    for name, vec, grad in (("w", w, gw), ("u", u, gu)):
        for c in range(C):
            c0 = vec[c]
            vec[c] = c0 + h
            lp = _loss(oracle_mod, k, v, w, u, g)
            vec[c] = c0 - h
            lm = _loss(oracle_mod, k, v, w, u, g)
            vec[c] = c0
            np.testing.assert_allclose(grad[:, c].sum(), (lp - lm) / (2 * h), rtol=1e-6,
                                       atol=1e-8, err_msg=f"{name}[{c}]")


def test_per_batch_parts_of_w_and_u(oracle_mod):
    # perturbing w[c] only through batch element b: the gradient of batch b's
    # own loss is the b-th part
    k, v, w, u, g = _inputs(3)
    _, _, gw, gu = oracle_mod.biwkv_bwd(k, v, w, u, g)
    h = 1e-6
    for b in range(k.shape[0]):
        sl = slice(b, b + 1)
        for c in range(k.shape[2]):
            for vec, grad in ((w, gw), (u, gu)):
                c0 = vec[c]
                vec[c] = c0 + h
                lp = _loss(oracle_mod, k[sl], v[sl], w, u, g[sl])
                vec[c] = c0 - h
                lm = _loss(oracle_mod, k[sl], v[sl], w, u, g[sl])
                vec[c] = c0
                np.testing.assert_allclose(grad[b, c], (lp - lm) / (2 * h), rtol=1e-6, atol=1e-8)


def test_k_gradient_sums_to_zero(oracle_mod):
    k, v, w, u, g = _inputs(4, B=3, T=40, C=5, wscale=8.0)
    gk, _, _, _ = oracle_mod.biwkv_bwd(k, v, w, u, g)
    scale = np.abs(gk).sum(axis=1)
    assert np.all(np.abs(gk.sum(axis=1)) <= 1e-12 * np.maximum(scale, 1.0))


def test_v_gradient_of_one_output_sums_to_one(oracle_mod):
    k, v, w, u, _ = _inputs(5, B=1, T=9, C=2)
    for t in range(9):
        g = np.zeros_like(k)
        g[0, t, :] = 1.0
        _, gv, _, _ = oracle_mod.biwkv_bwd(k, v, w, u, g)
        np.testing.assert_allclose(gv.sum(axis=1), 1.0, rtol=1e-13)
        assert np.all(gv >= 0.0)


def test_two_tokens_w_drops_out(oracle_mod):
    k, v, w, u, g = _inputs(6, T=2)
    _, _, gw, _ = oracle_mod.biwkv_bwd(k, v, w, u, g)
    assert np.all(gw == 0.0)


def test_single_token(oracle_mod):
    k, v, w, u, g = _inputs(7, T=1)
    gk, gv, gw, gu = oracle_mod.biwkv_bwd(k, v, w, u, g)
    # y = e^{u+k} v / e^{u+k} = v up to one rounding, so v - y ~ 1e-16
    np.testing.assert_allclose(gk, 0.0, atol=1e-14)
    np.testing.assert_allclose(gu, 0.0, atol=1e-14)
    assert np.all(gw == 0.0)
    np.testing.assert_allclose(gv, g, rtol=1e-15)


def test_columns_match_full(oracle_mod):
    k, v, w, u, g = _inputs(8, B=2, T=30, C=4)
    gk, gv, gw, gu = oracle_mod.biwkv_bwd(k, v, w, u, g)
    cols = np.array([0, 3, 5, 6])
    ck, cv, cw, cu = oracle_mod.biwkv_bwd_columns(k, v, w, u, g, cols)
    C = k.shape[2]
    for j, col in enumerate(cols):
        b, c = divmod(int(col), C)
        np.testing.assert_array_equal(ck[j], gk[b, :, c])
        np.testing.assert_array_equal(cv[j], gv[b, :, c])
        assert cw[j] == gw[b, c] and cu[j] == gu[b, c]


def test_shift_of_k_leaves_gradients(oracle_mod):
    # the max-of-k renormalisation must not change any gradient
    k, v, w, u, g = _inputs(9, T=20)
    a = oracle_mod.biwkv_bwd(k, v, w, u, g)
    b = oracle_mod.biwkv_bwd(k + 50.0, v, w, u, g)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, rtol=1e-9, atol=1e-12)
