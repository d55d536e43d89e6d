"""Pins for the CPU oracle: each test checks the oracle against something other
than itself -- numpy's float16 conversion, a published generator output, the
textbook Sylvester Hadamard matrix (scipy), dense numpy softmax attention,
brute force over all quantisation levels, closed forms and invariants, and a
hand-derived byte-layout fixture.  No GPU."""
import math
import os

import numpy as np
import pytest
import scipy.linalg

import oracle as O
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- fp16 --------

def _fp16_grid_neighbourhood():
    """fp32 values at, between and just around every finite fp16 value."""
    h = np.arange(0x0000, 0x7C00, dtype=np.uint32).astype(np.uint16)
    f = h.view(np.float16).astype(np.float64)
    nxt = np.append(f[1:], 65536.0)
    mid = (f + nxt) / 2.0  # exact midpoints (fit in fp32)
    mid32 = mid.astype(np.float32)
    cand = [f.astype(np.float32), mid32, np.nextafter(mid32, np.float32(np.inf)),
            np.nextafter(mid32, np.float32(0)), np.nextafter(f.astype(np.float32), np.float32(np.inf))]
    x = np.concatenate(cand)
    return np.concatenate([x, -x])


def test_f2h_rn_matches_numpy_on_grid_and_midpoints():
    x = _fp16_grid_neighbourhood()
    want = x.astype(np.float16).view(np.uint16)
    got = O.f2h_rn(x)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"{bad.size} mismatches, first x={x[bad[0]]!r} got={got[bad[0]]:#x} want={want[bad[0]]:#x}"


def test_f2h_rn_matches_numpy_random_bits():
    rng = np.random.default_rng(7)
    bits = rng.integers(0, 2**32, size=4_000_000, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[np.isfinite(x)]
    want = x.astype(np.float16).view(np.uint16)
    got = O.f2h_rn(x)
    assert np.array_equal(got, want)


def test_f2h_ru_is_least_fp16_not_below():
    x = _fp16_grid_neighbourhood()
    x = x[np.abs(x) <= 65504.0]
    h = O.f2h_ru(x)
    v = h.view(np.float16).astype(np.float64)
    assert np.all(v >= x.astype(np.float64))
    # the next fp16 toward -inf must be below x
    below = np.nextafter(h.view(np.float16), np.float16(-np.inf)).astype(np.float64)
    assert np.all(below < x.astype(np.float64))


def test_h2f_matches_numpy_all_patterns():
    h = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    want = h.view(np.float16).astype(np.float32)
    got = O.h2f(h)
    fin = np.isfinite(want)
    assert np.array_equal(got[fin].view(np.uint32), want[fin].view(np.uint32))
    assert np.array_equal(np.isnan(got), np.isnan(want))


# ----------------------------------------------------------- signs, c_d -------

def _golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def test_splitmix64_known_answer():
    for seed, idx, out in _golden_lines("splitmix64.txt"):
        assert O.splitmix64_output(int(seed), int(idx)) == int(out, 16)


def test_signs_are_pm1_and_balanced():
    s = O.signs(12345, 1 << 14)
    assert set(np.unique(s)) == {-1.0, 1.0}
    frac = float(np.mean(s > 0))
    assert abs(frac - 0.5) < 4 * 0.5 / math.sqrt(s.size)
    # different seeds give different vectors; the prefix does not depend on d
    assert not np.array_equal(O.signs(1, 128), O.signs(2, 128))
    assert np.array_equal(O.signs(9, 64), O.signs(9, 128)[:64])


def test_rotation_scale_bits():
    for d, bits in _golden_lines("rotation_scale.txt"):
        assert int(O.rot_scale_f32(int(d)).view(np.uint32)) == int(bits, 16)


# ------------------------------------------------------------- rotation -------

@pytest.mark.parametrize("d", [64, 128])
def test_rotation_equals_dense_sylvester_hadamard(d):
    seed = 77
    s = O.signs(seed, d).astype(np.float64)
    R = scipy.linalg.hadamard(d).astype(np.float64) @ np.diag(s) / math.sqrt(d)
    X = np.random.default_rng(0).standard_normal((9, d))
    got = O.rotate_f64(X, seed)
    assert np.allclose(got, X @ R.T, rtol=0, atol=1e-12)
    # inverse is R^T
    assert np.allclose(O.inv_rotate_f64(got, seed), X, rtol=0, atol=1e-12)
    assert np.allclose(O.inv_rotate_f64(X, seed), X @ R, rtol=0, atol=1e-12)


@pytest.mark.parametrize("d", [64, 128])
def test_rotation_orthonormal_and_preserves_dot(d):
    seed = 3
    R = O.rotate_f64(np.eye(d), seed)  # row i = R e_i = column i of R
    assert np.allclose(R @ R.T, np.eye(d), atol=1e-12)
    rng = np.random.default_rng(1)
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    assert abs(O.rotate_f64(q, seed) @ O.rotate_f64(k, seed) - q @ k) <= 1e-12 * (abs(q @ k) + 1)


@pytest.mark.parametrize("d", [64, 128])
def test_rotation_f32_close_to_f64_and_round_trip(d):
    seed = 11
    x = np.random.default_rng(2).standard_normal((50, d)).astype(np.float16).astype(np.float32)
    y32 = O.rotate_f32(x, seed)
    y64 = O.rotate_f64(x.astype(np.float64), seed)
    assert np.max(np.abs(y32 - y64)) <= 1e-6 * np.max(np.abs(y64))
    back = O.inv_rotate_f64(y32.astype(np.float64), seed)
    assert np.max(np.abs(back - x)) <= 1e-6 * np.max(np.abs(x))


def test_rotation_off_is_identity():
    x = np.random.default_rng(3).standard_normal((4, 64)).astype(np.float32)
    assert np.array_equal(O.rotate_f32(x, 5, rotate=0), x)


# ---------------------------------------------------------------- codec -------

def _rows(n, d, seed=0, outliers=True):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, d))
    if outliers:
        x[:, rng.choice(d, 3, replace=False)] *= 20
    return O.rotate_f32(x.astype(np.float16).astype(np.float32), 99)


FMTS = [(O.INT4_ASYM, 32, 1.0), (O.INT2_ASYM, 128, 0.9), (O.INT2_ASYM, 128, 1.0), (O.INT8_SYM, 128, 1.0),
        (O.INT4_ASYM, 64, 1.0)]


def _levels(fmt):
    return np.arange(-127, 128) if fmt == O.INT8_SYM else np.arange(0, 1 << (4 if fmt == O.INT4_ASYM else 2))


def _dequant_f64(fmt, group, code, sh, zh):
    n, d = code.shape
    s = sh.view(np.float16).astype(np.float64)
    if fmt == O.INT8_SYM:
        return code * s[:, :1]
    z = zh.view(np.float16).astype(np.float64)
    g = np.arange(d) // group
    return code * s[:, g] + z[:, g]


@pytest.mark.parametrize("fmt,group,clip", FMTS)
def test_codes_are_nearest_level_brute_force(fmt, group, clip):
    y = _rows(200, 128, seed=fmt * 10 + group)
    code, sh, zh, _, _ = O.quantize_rows(fmt, group, clip, y)
    n, d = y.shape
    s = sh.view(np.float16).astype(np.float64)
    z = np.zeros_like(s) if fmt == O.INT8_SYM else zh.view(np.float16).astype(np.float64)
    gi = np.zeros(d, int) if fmt == O.INT8_SYM else np.arange(d) // group
    lv = _levels(fmt)
    cand = lv[None, None, :] * s[:, gi][:, :, None] + z[:, gi][:, :, None]  # [n, d, L]
    dist = np.abs(y.astype(np.float64)[:, :, None] - cand)
    best = dist.min(axis=2)
    mine = np.abs(y.astype(np.float64) - _dequant_f64(fmt, group, code, sh, zh))
    tol = 1e-6 * s[:, gi] + 1e-30
    assert np.all(mine <= best + tol)


@pytest.mark.parametrize("fmt,group,clip", [f for f in FMTS if f[0] != O.INT8_SYM])
def test_asym_scale_zero_and_half_step_bound(fmt, group, clip):
    y = _rows(300, 128, seed=5)
    code, sh, zh, _, _ = O.quantize_rows(fmt, group, clip, y)
    qmax = (1 << (4 if fmt == O.INT4_ASYM else 2)) - 1
    yg = y.reshape(300, -1, group).astype(np.float32)
    lo = yg.min(axis=2) * np.float32(clip)
    hi = yg.max(axis=2) * np.float32(clip)
    # zero is the (clipped) minimum rounded to fp16; scale the step (hi-lo)/qmax
    assert np.array_equal(zh, lo.astype(np.float16).view(np.uint16))
    assert np.array_equal(sh, ((hi - lo) / np.float32(qmax)).astype(np.float16).view(np.uint16))
    # inside the representable range the error is at most half a step
    s = sh.view(np.float16).astype(np.float64)
    z = zh.view(np.float16).astype(np.float64)
    yhat = _dequant_f64(fmt, group, code, sh, zh).reshape(300, -1, group)
    inside = (yg >= z[:, :, None]) & (yg <= z[:, :, None] + qmax * s[:, :, None])
    err = np.abs(yg - yhat)
    half = np.broadcast_to(s[:, :, None] / 2 * (1 + 1e-6), err.shape)
    assert np.all(err[inside] <= half[inside])
    if clip == 1.0:
        # unclipped: the group minimum lands on code 0 and the maximum on qmax
        cg = code.reshape(300, -1, group)
        assert np.all(np.take_along_axis(cg, yg.argmin(axis=2)[:, :, None], 2) == 0)
        assert np.all(np.take_along_axis(cg, yg.argmax(axis=2)[:, :, None], 2) == qmax)
    else:
        # clipped: values beyond the clipped range saturate
        cg = code.reshape(300, -1, group)
        assert np.all(cg[yg > hi[:, :, None] + s[:, :, None]] == qmax)


def test_int8_is_textbook_absmax_with_round_up_scale():
    y = _rows(300, 128, seed=6)
    code, sh, _, _, _ = O.quantize_rows(O.INT8_SYM, 128, 1.0, y)
    a = np.abs(y).max(axis=1)
    s = sh[:, 0].view(np.float16).astype(np.float64)
    # round-up scale: the least fp16 not below absmax/127 (fp32 quotient)
    q = (a / np.float32(127)).astype(np.float64)
    assert np.all(s >= q)
    assert np.all(np.nextafter(sh[:, 0].view(np.float16), np.float16(-np.inf)).astype(np.float64) < q)
    # codes: round(y / scale), never clipped, and the absmax element hits +-127
    want = np.rint(y.astype(np.float64) / s[:, None])
    assert np.max(np.abs(code - want)) <= 1  # ties of the fp32 reciprocal path aside
    assert np.array_equal(np.abs(code).max(axis=1), np.full(300, 127))
    assert np.all(np.abs(y - code * s[:, None]) <= s[:, None] / 2 * (1 + 1e-6))


def test_descriptors_are_max_errors():
    y = _rows(64, 128, seed=8)
    for fmt, group, clip in FMTS:
        code, sh, zh, em, am = O.quantize_rows(fmt, group, clip, y)
        yhat = _dequant_f64(fmt, group, code, sh, zh)
        assert np.allclose(em, np.abs(y - yhat).max(axis=1), rtol=1e-6, atol=1e-7)
        assert np.array_equal(am, np.abs(y).max(axis=1))


def test_rotation_helps_outlier_rows():
    """[SRFT]/[OSCAR]: spreading outlier energy before low-bit rounding lowers
    the reconstruction error of rows with outlier channels."""
    rng = np.random.default_rng(4)
    x = rng.standard_normal((400, 128))
    x[:, [5, 40, 77, 100]] *= 15
    x = x.astype(np.float16).astype(np.float32)
    for fmt, group, clip in [(O.INT4_ASYM, 32, 1.0), (O.INT2_ASYM, 128, 1.0)]:
        errs = []
        for rot in (0, 1):
            y = O.rotate_f32(x, 21, rotate=rot)
            code, sh, zh, _, _ = O.quantize_rows(fmt, group, clip, y)
            xr = O.inv_rotate_f64(_dequant_f64(fmt, group, code, sh, zh), 21, rotate=rot)
            errs.append(np.mean((xr - x) ** 2))
        assert errs[1] < errs[0]


# ---------------------------------------------------------------- layout ------

def _parse_layout():
    cases, cur = [], None
    for ln in _golden_lines("layout_d64.txt"):
        if ln[0] == "case":
            cur = dict(name=ln[1], k_fmt=int(ln[2]), v_fmt=int(ln[3]), k_group=int(ln[4]), v_group=int(ln[5]),
                       pool=int(ln[6]), bytes=[])
            cases.append(cur)
        elif ln[0] in ("k", "v"):
            cur[ln[0]] = np.array([float(t) for t in ln[1:]], np.float16)
        elif ln[0] == "bytes":
            cur["bytes"].append((int(ln[1]), bytes.fromhex(ln[2])))
    return cases


@pytest.mark.parametrize("case", _parse_layout(), ids=lambda c: c["name"])
def test_layout_matches_hand_derived_bytes(case):
    cfg = O.make_config(2, 1, 64, case["k_fmt"], case["v_fmt"], case["k_group"], case["v_group"], rotate=0,
                        num_pages=2)
    assert O.pool_bytes(cfg) == case["pool"]
    pool = O.new_pool(cfg)
    rc = O.append(cfg, pool, case["k"][None, None, :], case["v"][None, None, :], np.array([17], np.int32))
    assert rc == 0
    want = np.zeros_like(pool)
    for off, b in case["bytes"]:
        want[off:off + len(b)] = np.frombuffer(b, np.uint8)
    diff = np.nonzero(pool != want)[0]
    assert diff.size == 0, f"first differing byte at {diff[0]}: {pool[diff[0]]:#x} vs {want[diff[0]]:#x}"


@pytest.mark.parametrize("fmt,group", [(O.INT4_ASYM, 32), (O.INT2_ASYM, 128), (O.INT8_SYM, 128)])
def test_pack_unpack_every_code_every_position(fmt, group):
    """Store rows whose codes cycle through every level at every channel
    position (rotation off, crafted values), read them back unchanged."""
    d = 128
    L = _levels(fmt)
    nl = len(L)
    rows = []
    for shift in range(nl):
        c = L[(np.arange(d) + shift) % nl]
        if fmt == O.INT8_SYM:
            c[0] = 127  # pin absmax to 127 so the scale is exactly 1
        else:
            c[0::group] = L[0]
            c[1::group] = L[-1]  # every group spans all levels -> scale 1, zero 0
        rows.append(c)
    rows = np.array(rows, np.float64)
    n = rows.shape[0]
    cfg = O.make_config(4, 1, d, fmt, fmt, group, group, rotate=0, num_pages=(n + 15) // 16)
    pool = O.new_pool(cfg)
    slots = np.random.default_rng(0).permutation(n).astype(np.int32)
    x = rows.astype(np.float16)[:, None, :]
    assert O.append(cfg, pool, x, x, slots) == 0
    for i in range(n):
        for tensor in (0, 1):
            code, _, _ = O.read_row(cfg, pool, int(slots[i]), 0, tensor)
            assert np.array_equal(code, rows[i].astype(np.int16))


def test_append_skips_negative_slots_and_rejects_overflow():
    cfg = O.make_config(8, 2, 64, num_pages=1)
    pool = O.new_pool(cfg)
    x = np.ones((2, 2, 64), np.float16)
    assert O.append(cfg, pool, x, x, np.array([-1, -1], np.int32)) == 0
    assert not pool.any()
    assert O.append(cfg, pool, x, x, np.array([16, 3], np.int32)) == -1  # 16 is past one page


# ------------------------------------------------------------- attention ------

def _small_cache(wl, T, seed_rot=0x5EED, extra=0):
    wl = W.scaled(wl, T)
    pages = W.page_table(wl, extra_tokens=extra)[0]
    cfg = O.make_config(wl.Hq, wl.Hkv, wl.d, wl.k_fmt, wl.v_fmt, wl.k_group, wl.v_group, wl.clip, seed_rot,
                        num_pages=pages.num_pages, bound_block_tokens=wl.bound_block)
    pool = O.new_pool(cfg)
    kv = []
    for b in range(wl.B):
        k, v = W.prefix_kv(wl, b)
        assert O.append(cfg, pool, k, v, pages.slots(b, 0, wl.ctx[b])) == 0
        kv.append((k, v))
    return wl, cfg, pool, pages, kv


def test_decode_equals_dense_numpy_attention():
    wl, cfg, pool, pages, _ = _small_cache(W.paged(B=3), [37, 16, 70])
    q = W.queries(wl, 0)
    out = O.decode(cfg, pool, q, pages.block_table, wl.ctx)
    d, g = wl.d, wl.g
    Hs = scipy.linalg.hadamard(d) / math.sqrt(d)
    s = O.signs(cfg.rotation_seed, d).astype(np.float64)
    R = Hs @ np.diag(s)
    for b in range(wl.B):
        slots = pages.slots(b, 0, wl.ctx[b])
        K, V = O.dequant(cfg, pool, slots)  # rotated domain [T, Hkv, d]
        for h in range(wl.Hq):
            qr = R @ q[b, h].astype(np.float64)
            sc = K[:, h // g, :] @ qr / math.sqrt(d)
            p = np.exp(sc - sc.max())
            p /= p.sum()
            o = R.T @ (p @ V[:, h // g, :])
            assert np.allclose(out[b, h], o, rtol=0, atol=1e-12)


def test_decode_constant_keys_gives_mean_value():
    wl = W.scaled(W.tiny(), 48)
    pages = W.page_table(wl)[0]
    cfg = O.make_config(wl.Hq, wl.Hkv, wl.d, num_pages=pages.num_pages)
    pool = O.new_pool(cfg)
    k, v = W.prefix_kv(wl, 0)
    k[:] = k[0]  # every key identical -> uniform softmax
    O.append(cfg, pool, k, v, pages.slots(0, 0, 48))
    out = O.decode(cfg, pool, W.queries(wl, 0), pages.block_table, wl.ctx)
    _, V = O.dequant(cfg, pool, pages.slots(0, 0, 48))
    for h in range(wl.Hq):
        want = O.inv_rotate_f64(V[:, h // wl.g, :].mean(axis=0), cfg.rotation_seed)
        assert np.allclose(out[0, h], want, rtol=0, atol=1e-12)


def test_decode_single_key_returns_its_value_and_empty_is_zero():
    wl = W.scaled(W.tiny(), 1)
    pages = W.page_table(wl)[0]
    cfg = O.make_config(wl.Hq, wl.Hkv, wl.d, num_pages=pages.num_pages)
    pool = O.new_pool(cfg)
    k, v = W.prefix_kv(wl, 0)
    O.append(cfg, pool, k, v, pages.slots(0, 0, 1))
    q = W.queries(wl, 0)
    out = O.decode(cfg, pool, q, pages.block_table, [1])
    _, V = O.dequant(cfg, pool, pages.slots(0, 0, 1))
    for h in range(wl.Hq):
        assert np.allclose(out[0, h], O.inv_rotate_f64(V[0, h // wl.g], cfg.rotation_seed), atol=1e-12)
    assert not O.decode(cfg, pool, q, pages.block_table, [0]).any()


def test_split_k_merge_equals_single_pass():
    wl, cfg, pool, pages, _ = _small_cache(W.llama(), 300)
    q = W.queries(wl, 1)
    ref = O.decode(cfg, pool, q, pages.block_table, wl.ctx, n_split=1)
    for ns in (2, 7, 300):
        got = O.decode(cfg, pool, q, pages.block_table, wl.ctx, n_split=ns)
        assert np.allclose(got, ref, rtol=0, atol=1e-12)


def test_page_permutation_invariance():
    wl, cfg, pool, pages, _ = _small_cache(W.tiny(), 100)
    q = W.queries(wl, 0)
    ref = O.decode(cfg, pool, q, pages.block_table, wl.ctx)
    # move every page to a new physical index and permute the table to match
    n = cfg.num_pages
    perm = np.random.default_rng(5).permutation(n)
    pb = O.page_bytes(cfg)
    pool2 = pool.copy()
    for old in range(n):
        new = perm[old]
        pool2[256 + new * pb:256 + (new + 1) * pb] = pool[256 + old * pb:256 + (old + 1) * pb]
    bt2 = perm[pages.block_table].astype(np.int32)
    assert np.allclose(O.decode(cfg, pool2, q, bt2, wl.ctx), ref, rtol=0, atol=0)


def test_rotation_lowers_attention_error_vs_fp16():
    """Quality (reported, not a parity bar): [SRFT]/[OSCAR] claim the rotation
    is what keeps low-bit attention usable with outlier channels; int4 g32
    attention error against unquantised fp16 attention must be lower with the
    rotation than without it."""
    errs = []
    for rot in (0, 1):
        wl = W.scaled(W.llama(), 512)
        pages = W.page_table(wl)[0]
        cfg = O.make_config(wl.Hq, wl.Hkv, wl.d, rotate=rot, num_pages=pages.num_pages)
        pool = O.new_pool(cfg)
        k, v = W.prefix_kv(wl, 0)
        sl = pages.slots(0, 0, 512)
        O.append(cfg, pool, k, v, sl)
        q = W.queries(wl, 0)
        out = O.decode(cfg, pool, q, pages.block_table, wl.ctx)
        ks = np.zeros((cfg.num_pages * 16, wl.Hkv, wl.d), np.float16)
        vs = np.zeros_like(ks)
        ks[sl], vs[sl] = k, v
        ref = O.decode_fp16(cfg, ks, vs, q, pages.block_table, wl.ctx)
        errs.append(np.linalg.norm(out - ref) / np.linalg.norm(ref))
    assert errs[1] < errs[0]


# ------------------------------------------------------------- certified ------

def _cert_case(T=700, frac=0.05):
    wl = W.scaled(W.certified(), T)
    pages = W.page_table(wl)[0]
    cfg = O.make_config(wl.Hq, wl.Hkv, wl.d, wl.k_fmt, wl.v_fmt, wl.k_group, wl.v_group, num_pages=pages.num_pages,
                        bound_block_tokens=wl.bound_block)
    pool = O.new_pool(cfg)
    k, v = W.prefix_kv(wl, 0)
    sl = pages.slots(0, 0, T)
    assert O.append(cfg, pool, k, v, sl) == 0
    ks = np.zeros((cfg.num_pages * 16, wl.Hkv, wl.d), np.float16)
    vs = np.zeros_like(ks)
    ks[sl], vs[sl] = k, v
    return wl, cfg, pool, pages, ks, vs


def test_promote_count():
    assert O.promote_count(0.01, 1024) == 11
    assert O.promote_count(0.01, 100) == 1
    assert O.promote_count(1.0, 37) == 37
    assert O.promote_count(0.0, 37) == 0


def test_certified_bound_is_rigorous_and_limits_hold():
    wl, cfg, pool, pages, ks, vs = _cert_case()
    q = W.queries(wl, 0)
    bt, ctx = pages.block_table, wl.ctx
    quant = O.decode(cfg, pool, q, bt, ctx)
    exact = O.decode_fp16(cfg, ks, vs, q, bt, ctx)
    out0, _, _, bsum = O.decode_certified(cfg, pool, ks, vs, q, bt, ctx, 0.0)
    assert np.allclose(out0, quant, rtol=0, atol=1e-12)  # 0% promotion = quantised attention
    out1, prom1, _, _ = O.decode_certified(cfg, pool, ks, vs, q, bt, ctx, 1.0)
    assert np.allclose(out1, exact, rtol=0, atol=1e-10)  # 100% = fp16 attention
    assert sorted(prom1[0, 0].tolist()) == list(range((ctx[0] + 127) // 128))
    # rigour: the summed bound covers the error of the rotated output (inf-norm)
    err_rot = np.abs(O.rotate_f64(quant - exact, cfg.rotation_seed)).max(axis=2)
    assert np.all(bsum[0] >= err_rot[0] * (1 - 1e-9))


def test_certified_promotes_top_scores_and_reduces_error():
    wl, cfg, pool, pages, ks, vs = _cert_case(T=1000, frac=0.2)
    q = W.queries(wl, 2)
    bt, ctx = pages.block_table, wl.ctx
    out, prom, scores, _ = O.decode_certified(cfg, pool, ks, vs, q, bt, ctx, 0.25)
    nb = (ctx[0] + 127) // 128
    k = O.promote_count(0.25, nb)
    exact = O.decode_fp16(cfg, ks, vs, q, bt, ctx)
    quant = O.decode(cfg, pool, q, bt, ctx)
    for kvh in range(wl.Hkv):
        sel = prom[0, kvh, :k]
        order = sorted(range(nb), key=lambda b: (-scores[0, kvh, b], b))[:k]
        assert sel.tolist() == order
    assert np.linalg.norm(out - exact) <= np.linalg.norm(quant - exact)


def test_certified_forced_selection():
    """Forcing the oracle's own top-k reproduces its output exactly; forcing
    every block gives fp16 attention; forcing none gives quantised attention."""
    wl, cfg, pool, pages, ks, vs = _cert_case(T=900)
    q = W.queries(wl, 1)
    bt, ctx = pages.block_table, wl.ctx
    nb = (ctx[0] + 127) // 128
    out, prom, _, _ = O.decode_certified(cfg, pool, ks, vs, q, bt, ctx, 0.3)
    out_f, prom_f, _, _ = O.decode_certified(cfg, pool, ks, vs, q, bt, ctx, 0.3, forced=prom)
    assert np.array_equal(out, out_f) and np.array_equal(prom, prom_f)
    every = np.tile(np.arange(nb, dtype=np.int32), (1, wl.Hkv, 1))
    out_all, _, _, _ = O.decode_certified(cfg, pool, ks, vs, q, bt, ctx, 0.0, forced=every)
    assert np.allclose(out_all, O.decode_fp16(cfg, ks, vs, q, bt, ctx), rtol=0, atol=1e-10)
    none = np.full((1, wl.Hkv, 3), -1, np.int32)
    out_none, _, _, _ = O.decode_certified(cfg, pool, ks, vs, q, bt, ctx, 0.5, forced=none)
    assert np.allclose(out_none, O.decode(cfg, pool, q, bt, ctx), rtol=0, atol=1e-12)
