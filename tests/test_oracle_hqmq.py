"""Pins for the oracle's HQMQ codec ["Hurwitz Quaternion Multiplicative
Quantization for KV Cache Compression", 1-3]: the primary codebook is the
binary tetrahedral group (closed under the Hamilton product, 60 degrees
apart), codeword selection is the largest inner product over all 24 x 1024
products by brute force in fp64 (numpy's own quaternion product), the
coverage is as fine as the page's O((24 S)^(-1/3)) suggests, Med3x keeps
the largest blocks above three medians, radii are within half a step, and
the pool stores exactly what the row encoder produced.  No GPU."""
import itertools

import numpy as np
import pytest

import oracle as O
import workloads as W


def hamilton(a, b):
    a0, a1, a2, a3 = np.moveaxis(np.asarray(a, np.float64), -1, 0)
    b0, b1, b2, b3 = np.moveaxis(np.asarray(b, np.float64), -1, 0)
    return np.stack([a0 * b0 - a1 * b1 - a2 * b2 - a3 * b3,
                     a0 * b1 + a1 * b0 + a2 * b3 - a3 * b2,
                     a0 * b2 - a1 * b3 + a2 * b0 + a3 * b1,
                     a0 * b3 + a1 * b2 - a2 * b1 + a3 * b0], axis=-1)


P = np.stack([O.hqmq_unit(p) for p in range(24)]).astype(np.float64)


def test_primary_codebook_is_the_binary_tetrahedral_group():
    assert len({tuple(q) for q in P}) == 24
    assert np.allclose(np.linalg.norm(P, axis=1), 1.0)
    assert any(np.array_equal(q, [1, 0, 0, 0]) for q in P)
    for a, b in itertools.product(P, P):  # closed under the product
        ab = hamilton(a, b)
        assert np.min(np.abs(P - ab).sum(axis=1)) < 1e-12
    G = P @ P.T
    off = G[~np.eye(24, dtype=bool)]
    assert set(np.round(off, 12).tolist()) <= {-1.0, -0.5, 0.0, 0.5}  # at least 60 degrees apart
    assert np.isclose(off.max(), 0.5)


def test_secondary_codebooks_are_unit_and_seeded():
    S = O.hqmq_codebook(5, 0, 0)
    assert S.shape == (O.HQMQ_NS, 4) and np.allclose(np.linalg.norm(S, axis=1), 1.0, atol=3e-7)
    assert np.array_equal(S, O.hqmq_codebook(5, 0, 0))
    assert not np.array_equal(S, O.hqmq_codebook(5, 0, 1)) and not np.array_equal(S, O.hqmq_codebook(5, 1, 0))
    assert not np.array_equal(S, O.hqmq_codebook(6, 0, 0))
    # roughly uniform on the sphere: the mean is near 0
    assert np.abs(S.mean(axis=0)).max() < 0.06


def test_codeword_is_the_largest_inner_product_by_brute_force():
    S = O.hqmq_codebook(11, 2, 1).astype(np.float64)
    C = hamilton(P[:, None, :], S[None, :, :])  # [24, NS, 4]: q_p q_s
    rng = np.random.default_rng(0)
    u = rng.standard_normal((300, 4))
    u = (u / np.linalg.norm(u, axis=1, keepdims=True)).astype(np.float32)
    idx = O.hqmq_encode_dirs(u, S.astype(np.float32))
    ip = np.einsum('nc,psc->nps', u.astype(np.float64), C)  # [n, 24, NS]
    best = ip.reshape(300, -1).max(axis=1)
    got = ip[np.arange(300), idx % 24, idx // 24]
    assert np.all(got >= best - 2e-6), (got - best).min()
    # coverage: O((24 S)^-1/3); with 24 x 1024 codewords directions are close
    assert got.mean() > 0.995 and got.min() > 0.98


def _row_case(seed, heavy=False):
    rng = np.random.default_rng(seed)
    y = rng.standard_normal((64, 128)).astype(np.float32)
    if heavy:  # a few blocks 20-200x longer, as in outlier-heavy models
        for r in range(64):
            for b in rng.choice(32, size=rng.integers(0, 4), replace=False):
                y[r, 4 * b:4 * b + 4] *= rng.uniform(20, 200)
    return y


@pytest.mark.parametrize("heavy", [False, True])
def test_row_codec_med3x_and_radius(heavy):
    y = _row_case(1 + heavy, heavy)
    S = O.hqmq_codebook(3, 0, 0)
    field, step, mask, outl = O.hqmq_quantize_rows(y, S)
    for r in range(y.shape[0]):
        rad = np.sqrt((y[r].reshape(32, 4).astype(np.float64) ** 2).sum(axis=1))
        tau = 3 * np.sort(rad)[15]
        above = np.nonzero(rad > tau * (1 + 1e-6))[0]
        flagged = [b for b in range(32) if (mask[r] >> b) & 1]
        assert len(flagged) == min(2, len(above))
        if flagged:  # the largest ones
            assert set(flagged) == set(above[np.argsort(-rad[above])][:len(flagged)])
            for k, b in enumerate(sorted(flagged)):
                assert np.array_equal(outl[r, k], y[r, 4 * b:4 * b + 4].astype(np.float16).view(np.uint16))
        st = float(np.array(step[r], np.uint16).view(np.float16))
        assert st >= tau / 31 * (1 - 1e-6) and st <= tau / 31 * (1 + 2e-3) + 1e-30
        rc = field[r] >> 15
        assert np.all(rc <= 31)
        for b in range(32):
            if b in flagged:
                continue
            if rad[b] <= tau:
                assert abs(rc[b] * st - rad[b]) <= st / 2 * (1 + 1e-5) + 1e-12
            else:
                assert rc[b] == 31  # beyond the outlier slots: clipped


def test_pool_round_trip_and_reconstruction():
    wl = W.scaled(W.hqmq(), [40])
    pages = W.page_table(wl)[0]
    cfg = O.make_config(wl.Hq, wl.Hkv, wl.d, O.HQMQ, O.HQMQ, 4, 4, rotation_seed=wl.rotation_seed,
                        num_pages=pages.num_pages)
    pool = O.new_pool(cfg)
    k, v = W.prefix_kv(wl, 0)
    sl = pages.slots(0, 0, 40)
    rc, yrot = O.append(cfg, pool, k, v, sl, want_rotated=True)
    assert rc == 0
    kd, vd = O.dequant(cfg, pool, sl)
    for kvh in range(wl.Hkv):
        for tensor in (0, 1):
            S = O.hqmq_codebook(wl.rotation_seed, kvh, tensor)
            y = yrot[:, kvh, tensor]
            f, st, m, ol = O.hqmq_quantize_rows(y, S)
            for t in range(40):
                f2, st2, m2, ol2 = O.hqmq_read_row(cfg, pool, int(sl[t]), kvh, tensor)
                assert np.array_equal(f2, f[t]) and st2 == st[t] and m2 == m[t] and np.array_equal(ol2, ol[t])
            rec = (kd if tensor == 0 else vd)[:, kvh]
            # blockwise: the reconstruction is (code x step) times a unit codeword, or the fp16 outlier
            err = np.linalg.norm((y - rec).reshape(40, 32, 4), axis=2)
            rad = np.linalg.norm(y.reshape(40, 32, 4).astype(np.float64), axis=2)
            assert np.all(err <= 0.25 * rad + 0.6 * (st.astype(np.uint16).view(np.float16).astype(np.float64)[:, None]) + 1e-3)
    # relative reconstruction error of the whole cache is small (~5 bits per element)
    yk = yrot[:, :, 0].reshape(40, -1)
    assert np.linalg.norm(yk - kd.reshape(40, -1)) / np.linalg.norm(yk) < 0.15


def test_tie_rules_of_the_codeword_choice():
    """Exact ties, built with a codebook of identical entries: the first s
    wins; an axis unit wins a tie against a half unit; the first component
    wins among equal |w_i|."""
    S = np.tile(np.array([1.0, 0.0, 0.0, 0.0], np.float32), (O.HQMQ_NS, 1))
    h = np.float32(1.0) / np.sqrt(np.float32(2.0))
    u = np.array([[h, h, 0, 0],        # max |w_i| = half-sum exactly: axis unit p = 0
                  [0, -h, h, 0],       # axis -i (p = 3) beats +j on the component tie
                  [0.5, -0.5, 0.5, 0.5],  # a half unit exactly: p = 8 + 2 = 10
                  [0, 0, 0, -1]], np.float32)  # -k: p = 7
    idx = O.hqmq_encode_dirs(u, S)
    assert idx.tolist() == [0, 3, 10, 7]  # every s ties: s = 0


def test_tie_rules_of_med3x():
    """A block exactly at tau = 3 x median is not an outlier (strictly
    greater); among equal radii above tau the lowest blocks are kept."""
    y = np.zeros((1, 128), np.float32)
    y[0, 0::4] = 1.0                   # every block radius 1: median 1, tau 3
    y[0, 4 * 2] = 3.0                  # exactly tau: coded, not kept
    for b in (5, 9, 20):
        y[0, 4 * b] = 5.0              # three equal radii above tau: blocks 5, 9 kept
    S = O.hqmq_codebook(1, 0, 0)
    field, step, mask, outl = O.hqmq_quantize_rows(y, S)
    assert int(mask[0]) == (1 << 5) | (1 << 9)
    assert np.all(np.asarray(outl[0]).view(np.float16).astype(np.float32)[:, 0] == 5.0)
    st = float(np.array(step[0], np.uint16).view(np.float16))
    q = np.float32(3.0) / np.float32(31.0)       # the step: fp16 rounded up of tau / 31
    up = np.float16(q) if float(np.float16(q)) >= q else np.nextafter(np.float16(q), np.float16(np.inf))
    assert st == float(up)
    assert (int(field[0, 20]) >> 15) == 31   # the third one: clipped radius
    assert (int(field[0, 2]) >> 15) == int(np.rint(3.0 / st))
    # one block above tau and one exactly at it: only the first is kept
    y2 = np.zeros((1, 128), np.float32)
    y2[0, 0::4] = 1.0
    y2[0, 4 * 2], y2[0, 4 * 7] = 3.0, 5.0
    assert int(O.hqmq_quantize_rows(y2, S)[2][0]) == 1 << 7


def test_covering_rate_of_the_product_codebook():
    """The page's Proposition 3.1: the product codebook of 24 Hurwitz units
    and S random unit quaternions covers S^3 at the rate O((24 S)^(-1/3)).
    With the first S of a generated codebook (S = 32 .. 1024), the mean angle
    from a random direction to its nearest codeword falls with slope -1/3 in
    log-log."""
    rng = np.random.default_rng(0)
    u = rng.standard_normal((3000, 4))
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    S = O.hqmq_codebook(3, 0, 0).astype(np.float64)
    xs, ys = [], []
    for n in (32, 64, 128, 256, 512, 1024):
        C = hamilton(P[:, None, :], S[None, :n, :]).reshape(-1, 4)
        theta = np.arccos(np.clip(np.max(u @ C.T, axis=1), -1, 1))
        xs.append(np.log(24 * n))
        ys.append(np.log(theta.mean()))
    slope = np.polyfit(xs, ys, 1)[0]
    assert -0.38 < slope < -0.29, slope
