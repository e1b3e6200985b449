"""A float64 model of the decomposition the fused forward kernel uses for eq. 5
of "Vision-RWKV Backbone" (Linear Complexity Bidirectional Attention),
checked against the oracle's direct summation of eq. 5.

The model follows the kernel's structure, not its code: a column of T tokens
splits into CTAs of 512 tokens, a CTA into warps of 8 chunks of KL tokens,
a chunk into KL/8 sub-chunks of 8 tokens.  The kernel runs KL = 16 (4 warps)
and KL = 8 (8 warps); KL = 32 is a candidate for fewer instructions per
element.
- Each sub-chunk sums relative to its own maximum of k.
- Going up, the chunk fold, the warp scan, the CTA scan and the cross-CTA
  exchange rescale by 2^(M_lower - M_upper) <= 1 and decay by a^distance.
- At the output, each token combines its sub-chunk's local sums with the
  carries from the left and the right.

What this pins (independently of CUDA): the fold
F = sum_h a^{8(KH-1-h)} e_h F_h and G = sum_h a^{8h} e_h G_h (KL = 16:
F = a^8 e0 F0 + e1 F1, G = e0 G0 + a^8 e1 G1), the carries each sub-chunk
takes from the others, the distances behind every decay power, and the
choice of references that keeps every scale factor <= 1 (k shifted by +80
and spreads of k across CTAs).
"""
import numpy as np
import pytest

SUB, CPW, TC = 8, 8, 512   # sub-chunk (the TMA element stride), chunks per warp, tokens per CTA


def _exp(x):
    with np.errstate(over="ignore", under="ignore"):
        return np.exp(x)


def model_column(k, v, w, u, KL=16):
    """wkv of one (b, c) column by the kernel's decomposition with chunks of
    KL tokens (8 and 16 are the kernel's two shapes; 32 a candidate).  Carries
    that cross the padding past T may overflow (as in the kernel, they only
    reach tokens past T, which are dropped); the tests compare real tokens."""
    with np.errstate(over="ignore", invalid="ignore"):
        return _model_column(k, v, w, u, KL)


def _model_column(k, v, w, u, KL):
    T = k.shape[0]
    KH = KL // SUB                   # sub-chunks per chunk
    NW = TC // (KL * CPW)            # warps per CTA
    lam = w / T
    cap = 126.0 * np.log(2.0)  # the kernel caps decay exponents at 2^126

    def ap(L):
        """a^L with a = e^(-w/T), capped like the kernel's powers: spans past
        the sequence end then multiply zero sums instead of overflowing."""
        return np.exp(np.minimum(-lam * np.asarray(L, dtype=np.float64), cap))
    eu = np.exp(u)
    ncl = -(-T // TC)
    Tp = ncl * TC
    kk = np.full(Tp, -np.inf)
    vv = np.zeros(Tp)
    kk[:T], vv[:T] = k, v
    nsub = Tp // SUB
    ks, vs = kk.reshape(nsub, SUB), vv.reshape(nsub, SUB)

    # sub-chunks: own maximum, p, local two-sided sums, totals
    Mh = ks.max(axis=1)                                  # -inf for an empty sub-chunk
    ref = np.where(np.isfinite(Mh), Mh, 0.0)
    p = _exp(ks - ref[:, None])
    pv = p * vs
    i = np.arange(SUB)
    dist = i[:, None] - i[None, :]                       # t - j
    fwd = np.where(dist > 0, ap(np.maximum(dist - 1.0, 0.0)), 0.0)    # j < t
    bwd = np.where(dist < 0, ap(np.maximum(-dist - 1.0, 0.0)), 0.0)   # j > t
    n = pv @ (fwd + bwd).T + eu * pv
    dd = p @ (fwd + bwd).T + eu * p
    F = np.stack([pv @ ap(SUB - 1 - i), p @ ap(SUB - 1 - i)], -1)   # to the sub-chunk's end
    G = np.stack([pv @ ap(i), p @ ap(i)], -1)                       # from its start

    # chunks of KH sub-chunks and the warp maximum
    nch = nsub // KH
    MhK = Mh.reshape(nch, KH)
    Mw = MhK.reshape(-1, CPW, KH).max(axis=(1, 2))       # per warp
    mref = np.where(np.isfinite(Mw), Mw, 0.0)
    e = _exp(MhK - np.repeat(mref, CPW)[:, None])        # 2^(M_h - M_warp), 0 if empty
    Fs = e[..., None] * F.reshape(nch, KH, 2)            # sub-chunk totals, warp reference
    Gs = e[..., None] * G.reshape(nch, KH, 2)
    h_ = np.arange(KH)
    Fc = np.einsum("h,chx->cx", ap(SUB * (KH - 1 - h_)), Fs)   # the chunk fold
    Gc = np.einsum("h,chx->cx", ap(SUB * h_), Gs)

    # warp scans over 8 chunks (decay a^KL per chunk)
    nw = nch // CPW
    Fw, Gw = Fc.reshape(nw, CPW, 2), Gc.reshape(nw, CPW, 2)
    X, Y = np.zeros_like(Fw), np.zeros_like(Gw)
    FI, GI = np.zeros_like(Fw), np.zeros_like(Gw)
    for wi in range(nw):
        acc = np.zeros(2)
        for q in range(CPW):
            X[wi, q] = acc
            acc = ap(KL) * acc + Fw[wi, q]
            FI[wi, q] = acc
        acc = np.zeros(2)
        for q in reversed(range(CPW)):
            Y[wi, q] = acc
            acc = ap(KL) * acc + Gw[wi, q]
            GI[wi, q] = acc

    # CTA scans over the warps (decay a^(KL CPW) per warp), rescaled to the CTA maximum
    MwN = Mw.reshape(ncl, NW)
    Mcta = MwN.max(axis=1)
    ws = _exp(MwN - Mcta[:, None])
    fagg = ws[..., None] * FI.reshape(ncl, NW, CPW, 2)[:, :, -1]
    gagg = ws[..., None] * GI.reshape(ncl, NW, CPW, 2)[:, :, 0]
    XW, YW = np.zeros_like(fagg), np.zeros_like(gagg)
    own_F, own_G = np.zeros((ncl, 2)), np.zeros((ncl, 2))
    for r in range(ncl):
        acc = np.zeros(2)
        for wi in range(NW):
            XW[r, wi] = acc
            acc = ap(KL * CPW) * acc + fagg[r, wi]
        own_F[r] = acc
        acc = np.zeros(2)
        for wi in reversed(range(NW)):
            YW[r, wi] = acc
            acc = ap(KL * CPW) * acc + gagg[r, wi]
        own_G[r] = acc

    # exchange across the column's CTAs (decay a^512 per CTA), common reference
    Mc = Mcta.max()
    sc = _exp(Mcta - Mc)
    Af, Bb = np.zeros((ncl, 2)), np.zeros((ncl, 2))
    acc = np.zeros(2)
    for r in range(ncl):
        Af[r] = acc
        acc = ap(TC) * acc + sc[r] * own_F[r]
    acc = np.zeros(2)
    for r in reversed(range(ncl)):
        Bb[r] = acc
        acc = ap(TC) * acc + sc[r] * own_G[r]

    # outputs: each sub-chunk's carries take the totals of the other sub-chunks
    out = np.empty(Tp)
    pw = ap(i)
    for r in range(ncl):
        for wi in range(NW):
            W_ = r * NW + wi
            slw = sc[r] * ws[r, wi]
            for cq in range(CPW):
                qc = wi * CPW + cq                       # chunk within the CTA
                ch = W_ * CPW + cq                       # chunk within the column
                slF, slB = sc[r] * ap(KL * cq), sc[r] * ap(KL * (CPW - 1 - cq))
                kf, kb = ap(KL * qc), ap(KL * (TC // KL - 1 - qc))
                As = slw * X[W_, cq] + slF * XW[r, wi] + kf * Af[r]
                Be = slw * Y[W_, cq] + slB * YW[r, wi] + kb * Bb[r]
                for h in range(KH):
                    Ah = ap(SUB * h) * As
                    for hh in range(h):
                        Ah = Ah + slw * ap(SUB * (h - 1 - hh)) * Fs[ch, hh]
                    Bh = ap(SUB * (KH - 1 - h)) * Be
                    for hh in range(h + 1, KH):
                        Bh = Bh + slw * ap(SUB * (hh - h - 1)) * Gs[ch, hh]
                    sh = slw * e[ch, h]
                    s = KH * ch + h
                    num = sh * n[s] + pw * Ah[0] + pw[::-1] * Bh[0]
                    den = sh * dd[s] + pw * Ah[1] + pw[::-1] * Bh[1]
                    out[s * SUB:(s + 1) * SUB] = num / den
    return out[:T]


@pytest.mark.parametrize("KL", [8, 16, 32])
@pytest.mark.parametrize("T", [1, 7, 33, 512, 513, 1000, 2048, 4096])
@pytest.mark.parametrize("w", [-8.0, -0.5, 0.0, 3.0, 8.0])
def test_model_equals_eq5(oracle_mod, T, w, KL):
    rng = np.random.default_rng(T * 31 + int(w * 10) + 1000)
    k = rng.normal(0.0, 2.0, T)
    v = rng.normal(0.0, 1.0, T)
    u = 0.7
    got = model_column(k, v, w, u, KL)
    want = oracle_mod.biwkv_direct(k[None, :, None], v[None, :, None], np.array([w]),
                                   np.array([u]))[0, :, 0]
    scale = np.abs(v).max()
    assert np.max(np.abs(got - want)) <= 1e-11 * scale


def test_model_handles_k_spread_across_ctas(oracle_mod):
    # maxima that differ by ~30 between CTAs and sub-chunks: every scale
    # factor stays <= 1 and nothing overflows
    T = 2048
    rng = np.random.default_rng(7)
    k = rng.normal(0.0, 1.0, T) + np.repeat([0.0, 30.0, -10.0, 20.0], T // 4)
    v = rng.normal(0.0, 1.0, T)
    got = model_column(k, v, 2.0, 0.3)
    want = oracle_mod.biwkv_direct(k[None, :, None], v[None, :, None], np.array([2.0]),
                                   np.array([0.3]))[0, :, 0]
    assert np.all(np.isfinite(got))
    assert np.max(np.abs(got - want)) <= 1e-10


def test_model_shift_invariance_in_k():
    T = 1500
    rng = np.random.default_rng(3)
    k, v = rng.normal(0.0, 1.0, T), rng.normal(0.0, 1.0, T)
    a = model_column(k, v, -3.0, 0.5)
    b = model_column(k + 80.0, v, -3.0, 0.5)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)
