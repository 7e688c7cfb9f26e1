"""Why the plan keeps the fp64 draft map (DraftAttention2 Eq. 3, Sec. 3.1): an fp32
screen with fp64 certification only saves work for the rows whose pairs all lie
outside the uncertainty band of the two cuts.  With the standard a-priori bound
of an fp32 dot product (gamma_d * sum |q_c k_c|) carried through the softmax,
that band covers nearly every row of a draft map; only the errors actually seen
(a band no screen can prove) would leave most rows certified.

Seeded Wan2.1-1.3B-shaped inputs, first two heads, the oracle's fp64 draft map.
"""
import numpy as np

from oracle import oracle
from video_dit_sparse_da2_b200.inputs import BY_NAME, workload_qkv


def test_fp32_screen_band_covers_nearly_every_row():
    w = BY_NAME["wan2.1-1.3b-480p"]
    q, k, v = (t[:, :2] for t in workload_qkv(w))
    desc = oracle.prepare(q, k, v, w.F, w.Hv, w.Wv).desc   # avg Q, max Q, avg K, max K
    A64 = oracle.draft(desc, w.lam)[0]
    H, R, _ = A64.shape
    d = desc.shape[-1]
    rd = np.float32(1.0 / np.sqrt(d))
    u = 2.0 ** -24
    gam = d * u / (1 - d * u)
    RR = R * R
    cuts = (RR * w.bp8 // 10000, RR * (w.bp8 + w.bp4) // 10000)

    def softmax32(L):
        m = L.max(axis=1, keepdims=True)
        e = np.exp(L - m, dtype=np.float32)
        return e / e.sum(axis=1, dtype=np.float32, keepdims=True)

    rows_seen = rows_proven = 0
    for h in range(H):
        Qa, Qm, Ka, Km = (desc[i, 0, h].astype(np.float32) for i in range(4))
        A32 = (np.float32(w.lam) * softmax32((Qm @ Km.T) * rd)
               + np.float32(1 - w.lam) * softmax32((Qa @ Ka.T) * rd)).astype(np.float64)
        err = np.abs(A32 - A64[h])
        seen = err.max()

        def rel_bound(Qx, Kx):
            EL = gam * (np.abs(Qx.astype(np.float64)) @ np.abs(Kx.astype(np.float64)).T) * float(rd)
            # shift by the row maximum (two logit errors), exp, normalizing sum
            return 4 * EL.max() + (R + 4) * u

        eps = max(rel_bound(Qa, Ka), rel_bound(Qm, Km))
        # the a-priori bound holds on these maps (entries above fp32's exp range)
        # and lies far above the errors actually seen
        big = A64[h] > 1e-30
        assert np.all(err[big] <= eps * A64[h][big])
        assert eps > 100 * (err[big] / A64[h][big]).max()
        flat = np.sort(A64[h].ravel())[::-1]
        band_seen = np.zeros(R, bool)
        band_proven = np.zeros(R, bool)
        for C in cuts:
            thr = flat[C - 1]
            band_seen |= (np.abs(A32 - thr) <= seen).any(axis=1)
            band_proven |= (np.abs(A32 - thr) <= eps * thr + seen).any(axis=1)
        rows_seen += int(band_seen.sum())
        rows_proven += int(band_proven.sum())
    total = H * R
    assert rows_proven >= 0.9 * total   # a sound screen recomputes nearly every row in fp64
    assert rows_seen <= 0.25 * total    # only an unprovable band would certify most rows


def test_fp32_softmax_screen_over_fp64_logits_certifies_most_rows():
    # Keep the logits as defined (fp64); take the row softmax and the mixture in
    # fp32 with pairwise sums.  The a-priori relative bound is then
    # (2 |t|max + 2 ceil(log2 R) + 14) u (shifted-logit rounding and exp, the
    # sum's terms and its pairwise additions, division, mixture; doubled), and only
    # a few rows hold a pair inside a cut's band.
    w = BY_NAME["wan2.1-1.3b-480p"]
    q, k, v = (t[:, :2] for t in workload_qkv(w))
    desc = oracle.prepare(q, k, v, w.F, w.Hv, w.Wv).desc
    A64 = oracle.draft(desc, w.lam)[0]
    H, R, _ = A64.shape
    rd = 1.0 / np.sqrt(desc.shape[-1])
    u = 2.0 ** -24
    RR = R * R
    cuts = (RR * w.bp8 // 10000, RR * (w.bp8 + w.bp4) // 10000)

    def softmax32(L64):
        t = (L64 - L64.max(axis=1, keepdims=True)).astype(np.float32)
        e = np.exp(t, dtype=np.float32)
        return e / e.sum(axis=1, dtype=np.float32, keepdims=True)

    rows = 0
    for h in range(H):
        Qa, Qm, Ka, Km = (desc[i, 0, h] for i in range(4))
        La, Lm = (Qa @ Ka.T) * rd, (Qm @ Km.T) * rd
        A32 = (np.float32(w.lam) * softmax32(Lm) + np.float32(1 - w.lam) * softmax32(La)).astype(np.float64)
        tmax = max(np.abs(L - L.max(axis=1, keepdims=True)).max() for L in (La, Lm))
        eps = (2 * tmax + 2 * np.ceil(np.log2(R)) + 14) * u
        big = A64[h] > 1e-30
        assert np.all(np.abs(A32 - A64[h])[big] <= eps * A64[h][big])
        flat = np.sort(A64[h].ravel())[::-1]
        band = np.zeros(R, bool)
        for C in cuts:
            thr = flat[C - 1]
            band |= (np.abs(A32 - thr) <= eps * thr).any(axis=1)
        rows += int(band.sum())
    assert rows <= 0.05 * H * R
