"""OSCAR's bit-reversal permutation P_br ("OSCAR", 2.2(a): R = U H P_br;
without the data-derived U, the rotate = 2 option: sign flips, Hadamard,
then the bit reversal of the channel index).  Pins of the oracle's rotation
against the dense matrices, its inverse and dot products, the reversal table
written out for d = 8, and a decode invariance: with 2-bit groups of the
whole row a channel permutation changes no group, so the decode output is
the same as without it.  Also the measurement of what P_br changes in the
reconstruction error.  No GPU."""
import math

import numpy as np
import pytest
import scipy.linalg

import oracle as O
import workloads as W


def _bitrev(d):
    b = d.bit_length() - 1
    return np.array([int(format(i, f"0{b}b")[::-1], 2) for i in range(d)])


def _mse(fmt, group, clip, y):
    code, sh, zh, _, _ = O.quantize_rows(fmt, group, clip, y)
    s = np.repeat(np.asarray(sh, np.uint16).view(np.float16).astype(np.float64), group, axis=1)
    z = np.repeat(np.asarray(zh, np.uint16).view(np.float16).astype(np.float64), group, axis=1)
    return float(((code * s + z - y.astype(np.float64)) ** 2).mean())


def _rows(wl, tensor, n):
    k, v = W.prefix_kv(W.scaled(wl, [n]), 0)
    x = (k if tensor == 0 else v).reshape(-1, wl.d)
    return O.rotate_f32(x.astype(np.float32), wl.rotation_seed)


def test_bit_reversal_changes_int4_groups_negligibly_and_int2_rows_not_at_all():
    br = _bitrev(128)
    assert sorted(br.tolist()) == list(range(128)) and np.array_equal(br[br], np.arange(128))
    for tensor in (0, 1):
        y = _rows(W.llama(), tensor, 256)
        a, b = _mse(O.INT4_ASYM, 32, 1.0, y), _mse(O.INT4_ASYM, 32, 1.0, y[:, br])
        assert abs(b - a) / a < 0.01, (a, b)
    y = _rows(W.int2(), 0, 256)
    a, b = _mse(O.INT2_ASYM, 128, 0.9, y), _mse(O.INT2_ASYM, 128, 0.9, y[:, br])
    assert abs(b - a) <= 1e-12 * a


def test_reversal_table_for_eight_channels():
    # 3-bit indices reversed: 000 000, 001 100, 010 010, 011 110, ...
    assert _bitrev(8).tolist() == [0, 4, 2, 6, 1, 5, 3, 7]


@pytest.mark.parametrize("d", [8, 64, 128])
def test_rotate2_is_the_dense_hadamard_then_bit_reversal(d):
    seed = 0x2B
    s = O.signs(seed, d).astype(np.float64)
    R1 = scipy.linalg.hadamard(d).astype(np.float64) @ np.diag(s) / math.sqrt(d)
    P = np.zeros((d, d))
    P[np.arange(d), _bitrev(d)] = 1.0  # (P t)_j = t_br(j)
    R2 = P @ R1
    X = np.random.default_rng(4).standard_normal((7, d))
    got = O.rotate_f64(X, seed, rotate=2)
    assert np.allclose(got, X @ R2.T, rtol=0, atol=1e-12)
    assert np.allclose(O.inv_rotate_f64(got, seed, rotate=2), X, rtol=0, atol=1e-12)
    assert np.allclose(R2 @ R2.T, np.eye(d), atol=1e-12)
    q, k = X[0], X[1]
    assert abs(got[0] @ got[1] - q @ k) <= 1e-12 * (abs(q @ k) + 1)


@pytest.mark.parametrize("d", [8, 64, 128])
def test_bit_reversal_commutes_with_the_sylvester_hadamard(d):
    """H[i][j] = (-1)^popcount(i & j) and br permutes the bits of i and j
    alike, so H[br(i)][br(j)] = H[i][j]: P_br H = H P_br.  Which side of H
    the permutation stands on changes no value, only the fp32 rounding
    order; the rotate = 2 output is also H applied to the bit-reversed
    signed input."""
    br = _bitrev(d)
    H = scipy.linalg.hadamard(d)
    assert np.array_equal(H[np.ix_(br, br)], H)
    seed = 0x51
    s = O.signs(seed, d).astype(np.float64)
    X = np.random.default_rng(6).standard_normal((5, d))
    want = ((X * s)[:, br] @ H.T.astype(np.float64)) / math.sqrt(d)
    assert np.allclose(O.rotate_f64(X, seed, rotate=2), want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("d", [64, 128])
def test_rotate2_f32_is_the_f32_rotation_reordered_bit_for_bit(d):
    x = np.random.default_rng(5).standard_normal((40, d)).astype(np.float16).astype(np.float32)
    a = O.rotate_f32(x, 9, rotate=1)
    b = O.rotate_f32(x, 9, rotate=2)
    assert np.array_equal(b.view(np.uint32), a[:, _bitrev(d)].view(np.uint32))


def _int2_cache(rotate):
    wl = W.scaled(W.int2(B=2), [300, 77])
    pages = W.page_table(wl)[0]
    cfg = O.make_config(wl.Hq, wl.Hkv, wl.d, wl.k_fmt, wl.v_fmt, wl.k_group, wl.v_group, wl.clip, 0x77,
                        rotate=rotate, num_pages=pages.num_pages)
    pool = O.new_pool(cfg)
    for b in range(wl.B):
        k, v = W.prefix_kv(wl, b)
        assert O.append(cfg, pool, k, v, pages.slots(b, 0, wl.ctx[b])) == 0
    return wl, cfg, pool, pages


def test_rotate2_decode_equals_rotate1_for_whole_row_groups():
    wl, c1, p1, pages = _int2_cache(1)
    _, c2, p2, _ = _int2_cache(2)
    br = _bitrev(wl.d)
    slots = pages.slots(0, 0, wl.ctx[0])
    K1, V1 = O.dequant(c1, p1, slots)
    K2, V2 = O.dequant(c2, p2, slots)
    # the same codes, scales and zeros, stored in the reversed channel order
    assert np.array_equal(K2, K1[:, :, br]) and np.array_equal(V2, V1[:, :, br])
    q = W.queries(wl, 0)
    o1 = O.decode(c1, p1, q, pages.block_table, wl.ctx)
    o2 = O.decode(c2, p2, q, pages.block_table, wl.ctx)
    assert np.allclose(o1, o2, rtol=0, atol=1e-12)
