"""A float64 model of the decomposition the 16-channel slab forward kernel
uses for eq. 5 of "Vision-RWKV Backbone" (Linear Complexity Bidirectional
Attention), checked against the oracle's direct summation of eq. 5.

The model follows the kernel's structure, not its code:
- a column of T tokens (T a multiple of 16) splits into CTAs of 512 tokens,
  a CTA into 32 chunks of 16 tokens, a chunk into two sub-chunks of 8;
- every p of a CTA is taken relative to the CTA's maximum of k;
- each sub-chunk's forward total (referenced to its last token) and
  backward total (referenced to its first) come from Horner sums; a chunk's
  totals are F = a^8 F0 + F1 and G = G0 + a^8 G1;
- the 32 chunk totals are scanned (decay a^16 per chunk), giving exclusive
  carries into each chunk;
- across CTAs every record is rescaled to the column maximum, scanned with
  decay a^512 per CTA, and the carry into the CTA is lifted into its frame by
  2^min(M_col - M_cta, 64) (base 2) and decayed to each chunk;
- per sub-chunk, a forward walk from the carry and a backward walk finish
  num and den.

What this pins independently of CUDA: the sub-chunk and chunk totals'
reference tokens, the carries each sub-chunk takes, every decay distance,
the column rescaling and the capped lift into the CTA frame (k spreads
across CTAs and k + 80).
"""
import numpy as np
import pytest

L, S, NCH = 16, 8, 32   # tokens per chunk, per sub-chunk; chunks per CTA
TC = L * NCH
CAP = 64.0              # exponent cap (base 2) of the lift into the CTA frame


def model_column(k, v, w, u):
    T = k.shape[0]
    assert T % L == 0
    with np.errstate(over="ignore", under="ignore", invalid="ignore"):
        return _model(k, v, w, u)


def _model(k, v, w, u):
    T = k.shape[0]
    lam = w / T                       # a = e^{-lam}
    ln2 = np.log(2.0)

    def ap(n):
        # decay powers a^n, exponent capped like the kernel's 2^126
        return np.exp(np.minimum(-lam * np.asarray(n, dtype=np.float64), 126.0 * ln2))
    a = ap(1)
    eu = np.exp(u)
    ncl = -(-T // TC)
    Tp = ncl * TC
    kk = np.full(Tp, -np.inf)
    vv = np.zeros(Tp)
    kk[:T], vv[:T] = k, v
    out = np.zeros(Tp)
    recs = []  # per CTA: (M, Fcta, Gcta) with F, G = (num, den)
    cta_state = []
    for r in range(ncl):
        kc, vc = kk[r * TC:(r + 1) * TC], vv[r * TC:(r + 1) * TC]
        M = np.max(kc)
        p = np.exp(kc - M) if np.isfinite(M) else np.zeros(TC)
        pv = p * vc
        # sub-chunk totals (Horner)
        nsub = TC // S
        Fs = np.zeros((nsub, 2))
        Gs = np.zeros((nsub, 2))
        for h in range(nsub):
            fa = fc = ga = gc = 0.0
            for i in range(S):
                t = h * S + i
                fa, fc = a * fa + pv[t], a * fc + p[t]
            for i in reversed(range(S)):
                t = h * S + i
                ga, gc = a * ga + pv[t], a * gc + p[t]
            Fs[h] = fa, fc
            Gs[h] = ga, gc
        a8 = ap(S)
        F = np.array([a8 * Fs[2 * q] + Fs[2 * q + 1] for q in range(NCH)])
        G = np.array([Gs[2 * q] + a8 * Gs[2 * q + 1] for q in range(NCH)])
        # inclusive scans over chunks (decay a^16 per chunk)
        Fi, Gi = F.copy(), G.copy()
        for q in range(1, NCH):
            Fi[q] = F[q] + ap(L) * Fi[q - 1]
        for q in range(NCH - 2, -1, -1):
            Gi[q] = G[q] + ap(L) * Gi[q + 1]
        cF = np.vstack([np.zeros(2), Fi[:-1]])
        cG = np.vstack([Gi[1:], np.zeros(2)])
        recs.append((M * np.log2(np.e), Fi[-1], Gi[0]))
        cta_state.append((p, pv, Fs, Gs, cF, cG, M * np.log2(np.e)))
    # column: rescale to the column maximum (base 2), scan across CTAs
    Mcol = max(m for m, _, _ in recs)
    PF = [f * (2.0 ** (m - Mcol) if np.isfinite(m) else 0.0) for m, f, _ in recs]
    PG = [g * (2.0 ** (m - Mcol) if np.isfinite(m) else 0.0) for m, _, g in recs]
    for rr in range(1, ncl):
        PF[rr] = PF[rr] + ap(TC) * PF[rr - 1]
    for rr in range(ncl - 2, -1, -1):
        PG[rr] = PG[rr] + ap(TC) * PG[rr + 1]
    for r in range(ncl):
        p, pv, Fs, Gs, cF, cG, Mown = cta_state[r]
        colF = PF[r - 1] if r > 0 else np.zeros(2)
        colG = PG[r + 1] if r + 1 < ncl else np.zeros(2)
        up = 2.0 ** min(Mcol - Mown, CAP) if np.isfinite(Mown) else 0.0
        colF, colG = colF * up, colG * up
        a8 = ap(S)
        for q in range(NCH):
            cFq = cF[q] + ap(L * q) * colF
            cGq = cG[q] + ap(L * (NCH - 1 - q)) * colG
            A = [cFq, a8 * cFq + Fs[2 * q]]
            B = [a8 * cGq + Gs[2 * q + 1], cGq]
            for h in range(2):
                An, Ad = A[h]
                Y, Z = np.zeros(S), np.zeros(S)
                for i in range(S):
                    t = q * L + h * S + i
                    Y[i], Z[i] = eu * pv[t] + An, eu * p[t] + Ad
                    An, Ad = a * An + pv[t], a * Ad + p[t]
                Bn, Bd = B[h]
                for i in reversed(range(S)):
                    t = q * L + h * S + i
                    out[r * TC + t] = (Y[i] + Bn) / (Z[i] + Bd)
                    Bn, Bd = a * Bn + pv[t], a * Bd + p[t]
    return out[:T]


def _direct(oracle_mod, k, v, w, u):
    T = k.shape[0]
    y = oracle_mod.biwkv_direct(k.reshape(1, T, 1), v.reshape(1, T, 1),
                                np.array([w]), np.array([u]))
    return y.reshape(T)


@pytest.mark.parametrize("T", [16, 32, 512, 528, 1024, 2048 + 16, 4096])
@pytest.mark.parametrize("w", [-8.0, -0.7, 0.0, 3.0, 8.0])
def test_model_matches_eq5(oracle_mod, T, w):
    rng = np.random.default_rng(T * 7 + int(w * 10) + 100)
    k = rng.normal(0, 2, T)
    v = rng.normal(0, 1, T)
    u = 0.6
    got = model_column(k, v, w, u)
    want = _direct(oracle_mod, k, v, w, u)
    np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)


def test_model_k_spread_across_ctas_and_shift(oracle_mod):
    # CTA maxima differ by ~30 (natural units): the lift into each CTA's
    # frame stays below the cap and the result is exact; adding 80 to every k
    # changes nothing
    T = 4096
    rng = np.random.default_rng(5)
    k = rng.normal(0, 1, T) + np.repeat(np.linspace(-15, 15, 8), 512)
    v = rng.normal(0, 1, T)
    for w in (-5.0, 2.0):
        want = _direct(oracle_mod, k, v, w, 0.3)
        np.testing.assert_allclose(model_column(k, v, w, 0.3), want, rtol=1e-9, atol=1e-12)
        np.testing.assert_allclose(model_column(k + 80.0, v, w, 0.3), want, rtol=1e-9, atol=1e-12)


def test_model_capped_lift_keeps_dominant_carries(oracle_mod):
    # one CTA's k far above the rest (beyond the cap): the others' outputs are
    # ruled by the carries from it; the capped lift leaves them exact to the
    # relative weight of their own terms (below 2^-20 here)
    T = 2048
    rng = np.random.default_rng(9)
    k = rng.normal(0, 1, T)
    k[512:1024] += 60.0   # 60 / ln 2 = 86.6 > 64 in base 2
    v = rng.normal(0, 1, T)
    want = _direct(oracle_mod, k, v, 1.0, 0.2)
    got = model_column(k, v, 1.0, 0.2)
    assert np.all(np.isfinite(got))
    np.testing.assert_allclose(got, want, rtol=1e-6, atol=1e-9)
