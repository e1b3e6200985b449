"""A float64 model of the decomposition the Bi-WKV backward kernel uses (the
chain rule of eq. 5 of "Vision-RWKV Backbone", Linear Complexity
Bidirectional Attention), checked against the oracle's backward, itself
pinned by finite differences of eq. 5.

The model follows the kernel's structure, not its code: CTAs of 512 tokens,
8 warps of 8 chunks of 8 tokens each.
- Pass 1: each thread walks its 8 tokens to the (A, H) aggregates of p v and
  p.  The aggregates are scanned across the warp's chunks and the CTA's
  warps, relative to the CTA maximum of k.  They are then folded across the
  column's CTAs in the frame of the column maximum.
- The final walks give N, D and H(pv), H(p) per token, hence y, q = g / D,
  r = q y and the dw, du terms.
- Pass 2 scans q and r the same way and gives dv and dk.
Every decay distance and the rescaling between frames are pinned here,
independently of CUDA.
"""
import numpy as np
import pytest

L, CPW, NW = 8, 8, 8      # tokens per thread, chunks per warp, warps per CTA
TC = L * CPW * NW          # 512 tokens per CTA


def _walk_fwd(x, a):
    """(A, H) of a segment walked left to right: A = sum a^{n-1-j} x_j,
    H = sum (n-1-j) a^{n-1-j} x_j."""
    A = np.zeros_like(x[0])
    H = np.zeros_like(x[0])
    for xi in x:
        H = a * (H + A)
        A = a * A + xi
    return A, H


def _cross(left, aL, Ln, right):
    A1, H1 = left
    A2, H2 = right
    return aL * A1 + A2, aL * (H1 + Ln * A1) + H2


def _scan(aggs, ap, Ln):
    """Exclusive and inclusive scans of (A, H) aggregates of segments of Ln
    tokens each, left to right (ap(L) = a^L)."""
    zero = (np.zeros_like(aggs[0][0]), np.zeros_like(aggs[0][1]))
    excl, incl, acc = [], [], zero
    for g in aggs:
        excl.append(acc)
        acc = _cross(acc, ap(Ln), Ln, g)
        incl.append(acc)
    return excl, incl


def model_bwd(k, v, g, w, u):
    """dk, dv, dw, du of one (b, c) column by the kernel's decomposition.
    Sums carried across the padding past T may overflow (as in the kernel,
    they reach only padding tokens, which take no part)."""
    with np.errstate(over="ignore", invalid="ignore"):
        return _model_bwd(k, v, g, w, u)


def _model_bwd(k, v, g, w, u):
    T = len(k)
    a, eu = np.exp(-w / T), np.exp(u)
    cap = 126.0 * np.log(2.0)

    def ap(Ln):
        """a^Ln with the kernel's cap of 2^126 on decay powers"""
        return np.exp(min(-w / T * Ln, cap))
    ncl = -(-T // TC)
    Tp = ncl * TC
    real = np.arange(Tp) < T
    kk = np.where(real, np.pad(k, (0, Tp - T)), -np.inf)
    vv = np.pad(v, (0, Tp - T))
    gg = np.pad(g, (0, Tp - T))

    # pass 1: p relative to each CTA's maximum; per-thread segment aggregates
    kc = kk.reshape(ncl, TC)
    Mcta = kc.max(axis=1)
    p = np.exp(kc - Mcta[:, None]).reshape(-1)
    x1 = np.stack([p * vv, p], -1)                       # (p v, p) per token
    nthr = Tp // L
    seg = x1.reshape(nthr, L, 2)
    lf = [_walk_fwd(seg[t], a) for t in range(nthr)]             # forward aggregates
    lb = [_walk_fwd(seg[t][::-1], a) for t in range(nthr)]       # backward aggregates

    def carries(agg_f, agg_b, own_frame_scale):
        """Exclusive forward and backward carries into every thread's chunk,
        in each CTA's frame, then folded across CTAs into the column frame.
        Returns per-thread (KF, KB) in the column frame."""
        KF, KB = [None] * nthr, [None] * nthr
        ctaF, ctaB = [], []
        per_thr_f, per_thr_b = [None] * nthr, [None] * nthr
        for r in range(ncl):
            warps_f, warps_b = [], []
            for wi in range(NW):
                t0 = r * CPW * NW + wi * CPW
                ex_f, in_f = _scan([agg_f[t] for t in range(t0, t0 + CPW)], ap, L)
                ex_b, in_b = _scan([agg_b[t] for t in reversed(range(t0, t0 + CPW))], ap, L)
                for c in range(CPW):
                    per_thr_f[t0 + c] = ex_f[c]
                    per_thr_b[t0 + CPW - 1 - c] = ex_b[c]
                warps_f.append(in_f[-1])
                warps_b.append(in_b[-1])
            exw_f, inw_f = _scan(warps_f, ap, L * CPW)
            exw_b, inw_b = _scan(warps_b[::-1], ap, L * CPW)
            for wi in range(NW):
                t0 = r * CPW * NW + wi * CPW
                for c in range(CPW):
                    t = t0 + c
                    # chunk carry = warp carry carried over the chunks before it
                    KF[t] = _cross(exw_f[wi], ap(L * c), L * c, per_thr_f[t])
                    KB[t] = _cross(exw_b[NW - 1 - wi], ap(L * (CPW - 1 - c)), L * (CPW - 1 - c),
                                   per_thr_b[t])
            ctaF.append(inw_f[-1])
            ctaB.append(inw_b[-1])
        # fold across CTAs in the column frame
        sc = own_frame_scale
        out_f, out_b = [None] * nthr, [None] * nthr
        for r in range(ncl):
            kin_f = (np.zeros(ctaF[0][0].shape), np.zeros(ctaF[0][0].shape))
            for rr in range(r):
                kin_f = _cross(kin_f, ap(TC), TC, (sc[rr] * ctaF[rr][0], sc[rr] * ctaF[rr][1]))
            kin_b = (np.zeros(ctaB[0][0].shape), np.zeros(ctaB[0][0].shape))
            for rr in reversed(range(r + 1, ncl)):
                kin_b = _cross(kin_b, ap(TC), TC, (sc[rr] * ctaB[rr][0], sc[rr] * ctaB[rr][1]))
            for t in range(r * CPW * NW, (r + 1) * CPW * NW):
                wi, c = (t // CPW) % NW, t % CPW
                d_f = L * (CPW * wi + c)                 # CTA start -> chunk start
                d_b = L * (CPW * (NW - 1 - wi) + CPW - 1 - c)
                out_f[t] = _cross(kin_f, ap(d_f), d_f, (sc[r] * KF[t][0], sc[r] * KF[t][1]))
                out_b[t] = _cross(kin_b, ap(d_b), d_b, (sc[r] * KB[t][0], sc[r] * KB[t][1]))
        return out_f, out_b

    Mc = Mcta.max()
    sc = np.exp(Mcta - Mc)
    KF, KB = carries(lf, lb, sc)

    # per-token pass-1 results in the column frame
    pc = p * np.repeat(sc, TC)
    q = np.zeros(Tp)
    rr_ = np.zeros(Tp)
    gw = gu = 0.0
    for t in range(nthr):
        A_f, H_f = KF[t]
        fw = []
        for i in range(L):                               # sums over tokens before i
            fw.append((A_f.copy(), H_f.copy()))
            x = np.array([pc[t * L + i] * vv[t * L + i], pc[t * L + i]])
            H_f = a * (H_f + A_f)
            A_f = a * A_f + x
        A_b, H_b = KB[t]
        for i in reversed(range(L)):                     # sums over tokens after i
            j = t * L + i
            x = np.array([pc[j] * vv[j], pc[j]])
            N = fw[i][0][0] + A_b[0] + eu * x[0]
            D = fw[i][0][1] + A_b[1] + eu * x[1]
            HN, HD = fw[i][1][0] + H_b[0], fw[i][1][1] + H_b[1]
            if real[j]:
                q[j] = gg[j] / D
                rr_[j] = q[j] * N / D
                gw += q[j] * HN - rr_[j] * HD
                gu += eu * pc[j] * (q[j] * vv[j] - rr_[j])
            H_b = a * (H_b + A_b)
            A_b = a * A_b + x

    # pass 2: sums of q and r (the H parts are not needed)
    x2 = np.stack([q, rr_], -1).reshape(nthr, L, 2)
    lf2 = [_walk_fwd(x2[t], a) for t in range(nthr)]
    lb2 = [_walk_fwd(x2[t][::-1], a) for t in range(nthr)]
    QF, QB = carries(lf2, lb2, np.ones(ncl))
    dv = np.zeros(Tp)
    dk = np.zeros(Tp)
    for t in range(nthr):
        Af = QF[t][0].copy()
        fq = []
        for i in range(L):
            fq.append(Af.copy())
            Af = a * Af + np.array([q[t * L + i], rr_[t * L + i]])
        Ab = QB[t][0].copy()
        for i in reversed(range(L)):
            j = t * L + i
            Sq = eu * q[j] + fq[i][0] + Ab[0]
            Sr = eu * rr_[j] + fq[i][1] + Ab[1]
            dv[j] = pc[j] * Sq
            dk[j] = vv[j] * dv[j] - pc[j] * Sr
            Ab = a * Ab + np.array([q[j], rr_[j]])
    return dk[:T], dv[:T], -gw / T, gu


@pytest.mark.parametrize("T", [1, 9, 64, 513, 1100])
@pytest.mark.parametrize("w", [-5.0, 0.0, 4.0])
def test_bwd_model_equals_oracle(oracle_mod, T, w):
    rng = np.random.default_rng(T * 7 + int(w) + 100)
    k = rng.normal(0.0, 1.5, T)
    v = rng.normal(0.0, 1.0, T)
    g = rng.normal(0.0, 1.0, T)
    u = -0.4
    dk, dv, dw, du = model_bwd(k, v, g, w, u)
    ok, ov, ow, ou = oracle_mod.biwkv_bwd(k[None, :, None], v[None, :, None], np.array([w]),
                                          np.array([u]), g[None, :, None])
    np.testing.assert_allclose(dv, ov[0, :, 0], rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dk, ok[0, :, 0], rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dw, ow[0, 0], rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(du, ou[0, 0], rtol=1e-9, atol=1e-11)
