"""The measurement behind leaving out OSCAR's bit-reversal permutation P_br
("OSCAR", 2.2: R = U H P_br; without the data-derived U): permuting the
rotated coordinates by bit reversal only changes which coordinates share a
quantisation group.  With the oracle's codec on the llama and int2 recipes
the reconstruction error moves by well under 1% for int4 g32, and not at
all for 2-bit groups of the whole row.  No GPU."""
import numpy as np

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
