"""Pins for the oracle's certified ladder ["Runtime-Certified Bounded-Error
Quantized Attention", Methodology 3: adaptive Top-K, ranking-consistency
check, four-rung fallback ladder].  Each test checks the oracle against
something other than its own formulas: closed-form block masses of a cache
whose keys quantise without loss, the limits (nothing promoted = quantised
attention, everything promoted = fp16 attention), the measured error of the
mixed output (the certified bound must cover it, with the key or the value
term isolated), a tier-2 store tampered with on purpose (the ranking check
must catch it), and monotonicity of every threshold.  No GPU."""
import numpy as np
import pytest

import oracle as O
import workloads as W

OFF = dict(tau_cov=0.0, max_frac=1.0, key_tol=np.inf, v_tol=np.inf, rank_tol=np.inf, cert_tol=np.inf,
           layer_frac=1.0)


def _case(wl, rotate=1, k_rows=None, v_rows=None):
    pages = W.page_table(wl)[0]
    cfg = O.make_config(wl.Hq, wl.Hkv, wl.d, wl.k_fmt, wl.v_fmt, wl.k_group, wl.v_group, wl.clip,
                        wl.rotation_seed, rotate=rotate, num_pages=pages.num_pages,
                        bound_block_tokens=wl.bound_block)
    pool = O.new_pool(cfg)
    ks = np.zeros((cfg.num_pages * 16, wl.Hkv, wl.d), np.float16)
    vs = np.zeros_like(ks)
    for b in range(wl.B):
        k, v = W.prefix_kv(wl, b)
        if k_rows is not None:
            k = k_rows[b]
        if v_rows is not None:
            v = v_rows[b]
        sl = pages.slots(b, 0, wl.ctx[b])
        assert O.append(cfg, pool, k, v, sl) == 0
        ks[sl], vs[sl] = k, v
    return cfg, pool, pages, ks, vs


def _run(wl, cfg, pool, pages, ks, vs, q, **pol):
    p = dict(OFF)
    p.update(pol)
    return O.decode_ladder(cfg, pool, ks, vs, q, pages.block_table, wl.ctx, p)


def _err_rot(cfg, a, b):
    return np.abs(O.rotate_f64(a - b, cfg.rotation_seed, cfg.rotate)).max(axis=-1)


def test_ladder_off_is_quantised_attention_with_the_plain_bound():
    wl = W.scaled(W.ladder(), [900, 300])
    cfg, pool, pages, ks, vs = _case(wl)
    q = W.queries(wl, 0)
    r = _run(wl, cfg, pool, pages, ks, vs, q)
    quant = O.decode(cfg, pool, q, pages.block_table, wl.ctx)
    assert np.allclose(r["out"], quant, rtol=0, atol=1e-12)
    assert np.all(r["k_star"] == 0) and np.all(r["flags"] == 0) and np.all(r["status"] == 0)
    _, _, _, bsum = O.decode_certified(cfg, pool, ks, vs, q, pages.block_table, wl.ctx, 0.0)
    assert np.allclose(r["bound"], bsum, rtol=1e-12, atol=0)
    exact = O.decode_fp16(cfg, ks, vs, q, pages.block_table, wl.ctx)
    assert np.all(r["bound"] >= _err_rot(cfg, quant, exact) * (1 - 1e-9))


def test_ladder_everything_exact_is_fp16_attention_with_zero_bound():
    wl = W.scaled(W.ladder(), [700])
    cfg, pool, pages, ks, vs = _case(wl)
    q = W.queries(wl, 1)
    r = _run(wl, cfg, pool, pages, ks, vs, q, tau_cov=1.0, v_tol=0.0)
    nb = (700 + 127) // 128
    assert np.all(r["k_star"] == nb) and np.all(r["flags"][0, :, :nb] == 3)
    exact = O.decode_fp16(cfg, ks, vs, q, pages.block_table, wl.ctx)
    assert np.allclose(r["mixed"], exact, rtol=0, atol=1e-10)
    assert np.all(np.abs(r["bound"]) <= 1e-12) and np.all(r["err"] <= 1e-10)


def _lossless_keys(wl, amp_exp):
    """Keys a_t * e_0 with a_t = 127 * 2^-m: int8 per-token scaling stores them
    without loss (scale = 2^-m exactly, code 127), so with the rotation off the
    quantised and exact scores agree and block masses have a closed form."""
    T = wl.ctx[0]
    k = np.zeros((T, wl.Hkv, wl.d), np.float16)
    a = (127.0 * 2.0 ** -np.asarray(amp_exp, np.float64))  # per token
    k[:, :, 0] = a[:, None]
    return [k]


def test_ladder_coverage_and_ranking_closed_form():
    wl = W.scaled(W.ladder(), [1000])  # 8 blocks, the last one 104 tokens
    block_m = [3, 1, 4, 0, 5, 2, 6, 1]  # block j's keys: 127 * 2^-m
    m = np.repeat(block_m, 128)[:1000]
    cfg, pool, pages, ks, vs = _case(wl, rotate=0, k_rows=_lossless_keys(wl, m))
    q = np.zeros((1, wl.Hq, wl.d), np.float16)
    q[0, :, 0] = 0.25  # score of a token: 0.25 * a / sqrt(128)
    s = 0.25 * 127.0 * 2.0 ** -np.asarray(block_m, np.float64) / np.sqrt(128.0)
    n = np.array([128] * 7 + [104], np.float64)
    w = n * np.exp(s - s.max())
    P = w / w.sum()
    order = sorted(range(8), key=lambda j: (-P[j], j))
    cum = np.concatenate([[0.0], np.cumsum(P[order])])
    for tau in (0.3, 0.5, 0.8, 0.95, 0.999):
        r = _run(wl, cfg, pool, pages, ks, vs, q, tau_cov=tau, key_tol=1e-12)
        kc = int(np.argmax(cum >= tau))
        assert np.all(r["k_cov"] == kc), (tau, r["k_cov"], kc)
        assert np.all(r["k_key"] == 0) and np.all(r["ekey"] <= 1e-13)  # lossless keys: Delta = 0, no key term
        assert np.all(r["k_star"] == kc)
        assert np.allclose(r["rscore"][0, 0], P, rtol=1e-12, atol=0)
        assert np.allclose(r["cov"][0, 0], cum, rtol=1e-12, atol=1e-15)
        for kvh in range(wl.Hkv):
            assert sorted(np.nonzero(r["flags"][0, kvh] & 1)[0].tolist()) == sorted(order[:kc])
        assert np.all(r["status"] & O.LADDER_RANK_FAIL == 0)  # exact = quantised masses: consistent at rho=0


def test_ladder_equal_masses_rank_the_lower_block_first():
    wl = W.scaled(W.ladder(), [1024])
    cfg, pool, pages, ks, vs = _case(wl, rotate=0, k_rows=_lossless_keys(wl, np.zeros(1024)))
    q = np.zeros((1, wl.Hq, wl.d), np.float16)  # all scores 0: every block 1/8 of the mass
    r = _run(wl, cfg, pool, pages, ks, vs, q, tau_cov=0.6)
    assert np.all(r["k_cov"] == 5)
    assert np.all(r["flags"][0, :, :5] & 1 == 1) and np.all(r["flags"][0, :, 5:] & 1 == 0)


def _independent_err(cfg, pages, wl, ks, vs, q, mixed):
    exact = O.decode_fp16(cfg, ks, vs, q, pages.block_table, wl.ctx)
    return _err_rot(cfg, mixed, exact)


def _random_flags(rng, shape, nb, p_key, p_val):
    f = np.zeros(shape, np.uint8)
    f[..., :nb] = (rng.random(f[..., :nb].shape) < p_key) | ((rng.random(f[..., :nb].shape) < p_val) << 1)
    return f


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_bound_covers_the_error_value_term_alone(seed):
    """Keys without loss (rotation off, int8 of a*e_0): the key term vanishes
    and the bound is the value term alone; it must still cover the error."""
    wl = W.scaled(W.ladder(), [1000])
    rng = np.random.default_rng(seed)
    m = np.repeat(rng.integers(0, 6, size=8), 128)[:1000]
    cfg, pool, pages, ks, vs = _case(wl, rotate=0, k_rows=_lossless_keys(wl, m))
    q = (rng.standard_normal((1, wl.Hq, wl.d)) * 2.0).astype(np.float16)
    ff = _random_flags(rng, (1, wl.Hkv, 8), 8, 0.5, 0.4)
    r = O.decode_ladder(cfg, pool, ks, vs, q, pages.block_table, wl.ctx, dict(OFF), forced_flags=ff)
    err = _independent_err(cfg, pages, wl, ks, vs, q, r["mixed"])
    assert np.all(err > 0)
    assert np.all(r["bound"] >= err * (1 - 1e-9)), (r["bound"], err)
    allv = ff | 2
    r2 = O.decode_ladder(cfg, pool, ks, vs, q, pages.block_table, wl.ctx, dict(OFF), forced_flags=allv)
    assert np.all(np.abs(r2["bound"]) <= 1e-12)  # nothing left to bound
    assert np.all(_independent_err(cfg, pages, wl, ks, vs, q, r2["mixed"]) <= 1e-12)


@pytest.mark.parametrize("seed", [0, 1])
def test_bound_covers_the_error_key_term_alone(seed):
    """Every value exact, random key promotion: the bound is the key term
    alone and must cover the error of the mixed output."""
    wl = W.scaled(W.certified(), [1100])
    cfg, pool, pages, ks, vs = _case(wl)
    rng = np.random.default_rng(seed)
    q = W.queries(wl, seed)
    ff = _random_flags(rng, (1, wl.Hkv, 9), 9, 0.4, 1.0)
    r = O.decode_ladder(cfg, pool, ks, vs, q, pages.block_table, wl.ctx, dict(OFF), forced_flags=ff)
    err = _independent_err(cfg, pages, wl, ks, vs, q, r["mixed"])
    assert np.all(err > 0) and np.all(r["bound"] >= err * (1 - 1e-9))


@pytest.mark.parametrize("name,wl", [
    ("needle", W.scaled(W.ladder(), [1500, 260])),
    ("llama-int4k", W.scaled(W.certified(), [800, 1300])),
    ("gqa8", W.scaled(W.certified(), [600])),
])
def test_bound_covers_the_error_random_promotion(name, wl):
    import dataclasses
    if name == "llama-int4k":
        wl = dataclasses.replace(wl, k_fmt=O.INT4_ASYM, k_group=32)
    if name == "gqa8":
        wl = dataclasses.replace(wl, Hq=64)
    cfg, pool, pages, ks, vs = _case(wl)
    rng = np.random.default_rng(7)
    nb = (max(wl.ctx) + 127) // 128
    for trial in range(3):
        q = W.queries(wl, trial)
        ff = _random_flags(rng, (wl.B, wl.Hkv, nb), nb, 0.3, 0.3)
        r = O.decode_ladder(cfg, pool, ks, vs, q, pages.block_table, wl.ctx, dict(OFF), forced_flags=ff)
        err = _independent_err(cfg, pages, wl, ks, vs, q, r["mixed"])
        assert np.all(r["bound"] >= err * (1 - 1e-9))


def test_curves_are_monotone_and_decisions_follow_them():
    wl = W.scaled(W.ladder(), [2000])
    cfg, pool, pages, ks, vs = _case(wl)
    q = W.queries(wl, 3)
    nb = 16
    for key_tol, tau in ((0.05, 0.9), (0.01, 0.995), (1e-3, 0.5)):
        r = _run(wl, cfg, pool, pages, ks, vs, q, tau_cov=tau, key_tol=key_tol)
        for kvh in range(wl.Hkv):
            cov, ek = r["cov"][0, kvh], r["ekey"][0, kvh]
            assert np.all(np.diff(cov) >= -1e-15) and abs(cov[nb] - 1.0) < 1e-12 and cov[0] == 0.0
            assert np.all(np.diff(ek) <= 1e-15) and ek[nb] <= 1e-12
            kc = int(np.argmax(cov >= tau))
            kk = int(np.argmax(ek <= key_tol))
            assert r["k_cov"][0, kvh] == kc and r["k_key"][0, kvh] == kk
            assert r["k_star"][0, kvh] == max(kc, kk)
            order = sorted(range(nb), key=lambda j: (-r["rscore"][0, kvh, j], j))
            keys = set(np.nonzero(r["flags"][0, kvh] & 1)[0].tolist())
            assert keys == set(order[:max(kc, kk)])
            expanded = bool(r["status"][0, kvh * wl.g] & O.LADDER_EXPANDED)
            assert expanded == (kk > kc)


def test_value_rung_thresholds_are_nested():
    wl = W.scaled(W.ladder(), [1500])
    cfg, pool, pages, ks, vs = _case(wl)
    q = W.queries(wl, 0)
    prev = None
    for v_tol in (0.0, 1e-5, 1e-4, 1e-3, 1e-2, np.inf):
        r = _run(wl, cfg, pool, pages, ks, vs, q, v_tol=v_tol)
        vset = (r["flags"] >> 1) & 1
        if v_tol == 0.0:
            assert np.all(vset[..., :12] == 1)  # every block has a value error and some mass
        if v_tol == np.inf:
            assert not vset.any()
        if prev is not None:
            assert np.all(vset <= prev)  # a higher threshold promotes a subset
        has = vset.any(axis=2)
        assert np.array_equal(has, (r["status"][:, ::wl.g] & O.LADDER_VALUES) != 0)
        prev = vset


def test_budget_caps_the_promoted_keys():
    wl = W.scaled(W.ladder(), [3000])
    cfg, pool, pages, ks, vs = _case(wl)
    q = W.queries(wl, 0)
    nb = (3000 + 127) // 128
    full = _run(wl, cfg, pool, pages, ks, vs, q, tau_cov=0.999, key_tol=1e-4)
    cap = _run(wl, cfg, pool, pages, ks, vs, q, tau_cov=0.999, key_tol=1e-4, max_frac=0.1)
    kc = O.promote_count(0.1, nb)
    for kvh in range(wl.Hkv):
        want = max(full["k_cov"][0, kvh], full["k_key"][0, kvh])
        assert full["k_star"][0, kvh] == want
        assert cap["k_star"][0, kvh] == min(want, kc)
        capped = bool(cap["status"][0, kvh * wl.g] & O.LADDER_CAPPED)
        assert capped == (want > kc)
        order = sorted(range(nb), key=lambda j: (-cap["rscore"][0, kvh, j], j))
        assert set(np.nonzero(cap["flags"][0, kvh] & 1)[0].tolist()) == set(order[:min(want, kc)])


def _closed_form_case():
    wl = W.scaled(W.ladder(), [1000])
    block_m = [3, 1, 4, 0, 5, 2, 6, 1]
    m = np.repeat(block_m, 128)[:1000]
    cfg, pool, pages, ks, vs = _case(wl, rotate=0, k_rows=_lossless_keys(wl, m))
    q = np.zeros((1, wl.Hq, wl.d), np.float16)
    q[0, :, 0] = 0.25
    return wl, cfg, pool, pages, ks, vs, q


def test_ranking_check_catches_a_tampered_tier2_store():
    """Swap the tier-2 key rows of blocks 0 and 4 (the cache keeps the true
    ones): the exact masses of those blocks trade places while the quantised
    ranking does not, which is the silent distortion the check exists for.
    The check must fail at rho = 0, pass with a slack larger than the swap's
    mass ratio, and the failing heads must come back as fp16 attention over
    the (tampered) tier-2 rows."""
    wl, cfg, pool, pages, ks, vs, q = _closed_form_case()
    sl0, sl4 = pages.slots(0, 0, 128), pages.slots(0, 512, 640)
    bad = ks.copy()
    bad[sl0], bad[sl4] = ks[sl4], ks[sl0]
    clean = _run(wl, cfg, pool, pages, ks, vs, q, tau_cov=1.0, rank_tol=0.0)
    assert np.all(clean["status"] & O.LADDER_RANK_FAIL == 0)
    r = _run(wl, cfg, pool, pages, bad, vs, q, tau_cov=1.0, rank_tol=0.0)
    assert np.all(r["status"] & O.LADDER_RANK_FAIL) and np.all(r["status"] & O.LADDER_HEAD_DENSE)
    dense = O.decode_fp16(cfg, bad, vs, q, pages.block_table, wl.ctx)
    assert np.allclose(r["out"], dense, rtol=0, atol=1e-12)
    s = 0.25 * 127.0 * 2.0 ** -np.array([3.0, 5.0]) / np.sqrt(128.0)
    ratio = np.exp(s[0] - s[1])  # exact mass of block 4 over block 0 after the swap
    loose = _run(wl, cfg, pool, pages, bad, vs, q, tau_cov=1.0, rank_tol=ratio * 1.001 - 1.0)
    assert np.all(loose["status"] & O.LADDER_RANK_FAIL == 0)
    tight = _run(wl, cfg, pool, pages, bad, vs, q, tau_cov=1.0, rank_tol=ratio * 0.999 - 1.0)
    assert np.all(tight["status"] & O.LADDER_RANK_FAIL)
    # the margin is that ratio (the swap is the only inversion); with the true
    # store every promoted block keeps its place
    assert np.allclose(r["rank_margin"], ratio - 1.0, rtol=1e-12, atol=0)
    assert np.all(clean["rank_margin"] == 0.0)
    # outside the promoted set the check sees nothing: promote only block 3 (the heaviest)
    one = _run(wl, cfg, pool, pages, bad, vs, q, tau_cov=0.01, rank_tol=0.0)
    assert np.all(one["k_star"] == 1) and np.all(one["status"] & O.LADDER_RANK_FAIL == 0)


def test_head_and_layer_fallbacks():
    wl = W.scaled(W.ladder(), [1200, 700])
    cfg, pool, pages, ks, vs = _case(wl)
    q = W.queries(wl, 2)
    dense = O.decode_fp16(cfg, ks, vs, q, pages.block_table, wl.ctx)
    base = _run(wl, cfg, pool, pages, ks, vs, q, tau_cov=0.9)
    assert not np.any(base["status"] & (O.LADDER_HEAD_DENSE | O.LADDER_LAYER_DENSE))
    assert np.allclose(base["out"], base["mixed"], rtol=0, atol=0)
    assert np.allclose(base["dense"], dense, rtol=0, atol=0)
    tol = float(np.median(base["bound"]))
    nfail = int((base["bound"] > tol).sum())
    frac = nfail / base["bound"].size
    for layer_frac, layer in ((min(1.0, frac + 0.1), False), (max(0.0, frac - 0.1), True)):
        r = _run(wl, cfg, pool, pages, ks, vs, q, tau_cov=0.9, cert_tol=tol, layer_frac=layer_frac)
        fell = base["bound"] > tol
        assert np.array_equal((r["status"] & O.LADDER_BOUND_FAIL) != 0, fell)
        assert np.array_equal((r["status"] & O.LADDER_HEAD_DENSE) != 0, fell)
        assert np.all(((r["status"] & O.LADDER_LAYER_DENSE) != 0) == layer)
        use_dense = fell | layer
        assert np.allclose(r["out"][use_dense], dense[use_dense], rtol=0, atol=0)
        assert np.allclose(r["out"][~use_dense], base["mixed"][~use_dense], rtol=0, atol=0)
    every = _run(wl, cfg, pool, pages, ks, vs, q, tau_cov=0.9, cert_tol=0.0)
    assert np.allclose(every["out"], dense, rtol=0, atol=0)


def test_forcing_the_oracles_own_decisions_reproduces_it():
    wl = W.scaled(W.ladder(), [1800])
    cfg, pool, pages, ks, vs = _case(wl)
    q = W.queries(wl, 4)
    pol = dict(OFF, tau_cov=0.995, key_tol=0.02, v_tol=1e-3, rank_tol=0.05, cert_tol=5e-3, layer_frac=0.9)
    r = O.decode_ladder(cfg, pool, ks, vs, q, pages.block_table, wl.ctx, pol)
    fb = ((r["status"] & (O.LADDER_HEAD_DENSE | O.LADDER_LAYER_DENSE)) != 0).astype(np.int32)
    f = O.decode_ladder(cfg, pool, ks, vs, q, pages.block_table, wl.ctx, pol, forced_flags=r["flags"],
                        forced_fallback=fb)
    for key in ("out", "mixed", "bound", "flags", "k_star"):
        assert np.array_equal(r[key], f[key]), key


def test_key_and_value_promotion_of_one_set_equals_the_fixed_fraction_mode():
    wl = W.scaled(W.certified(), [1400])
    cfg, pool, pages, ks, vs = _case(wl)
    q = W.queries(wl, 1)
    out, prom, _, _ = O.decode_certified(cfg, pool, ks, vs, q, pages.block_table, wl.ctx, 0.3)
    nb = (1400 + 127) // 128
    ff = np.zeros((1, wl.Hkv, nb), np.uint8)
    for kvh in range(wl.Hkv):
        ff[0, kvh, prom[0, kvh][prom[0, kvh] >= 0]] = 3
    r = O.decode_ladder(cfg, pool, ks, vs, q, pages.block_table, wl.ctx, dict(OFF), forced_flags=ff)
    assert np.allclose(r["mixed"], out, rtol=0, atol=1e-12)


def test_empty_sequence_and_ragged_tail():
    wl = W.scaled(W.ladder(), [0, 333])
    cfg, pool, pages, ks, vs = _case(wl)
    q = W.queries(wl, 0)
    r = _run(wl, cfg, pool, pages, ks, vs, q, tau_cov=0.995, v_tol=1e-3, cert_tol=1e-2)
    assert np.all(r["out"][0] == 0) and np.all(r["status"][0] == 0) and np.all(r["bound"][0] == 0)
    assert np.all(r["k_star"][0] == 0) and not r["flags"][0].any()
    assert np.all(r["k_star"][1] >= 1) and not r["flags"][1, :, 3:].any()
    err = _independent_err(cfg, pages, wl, ks, vs, q, r["mixed"])
    assert np.all(r["bound"] >= err * (1 - 1e-9) - 1e-12)  # all three blocks exact here: both ~1e-15


def test_coverage_must_hold_for_every_head_of_the_group():
    """Two heads per group pulling opposite ways (closed form): even heads
    favour the large-amplitude blocks, odd heads the small ones.  Ranking is
    by the larger of the two masses and K_cov must reach tau for both."""
    wl = W.scaled(W.ladder(), [1024])
    block_m = [0, 6, 1, 5, 2, 4, 3, 3]
    m = np.repeat(block_m, 128)
    cfg, pool, pages, ks, vs = _case(wl, rotate=0, k_rows=_lossless_keys(wl, m))
    q = np.zeros((1, wl.Hq, wl.d), np.float16)
    q[0, 0::2, 0] = 0.5
    q[0, 1::2, 0] = -0.5
    a = 127.0 * 2.0 ** -np.asarray(block_m, np.float64)
    P = []
    for x in (0.5, -0.5):
        s = x * a / np.sqrt(128.0)
        w = np.exp(s - s.max())
        P.append(w / w.sum())
    P = np.array(P)  # [2 heads, 8 blocks]
    r_score = P.max(axis=0)
    order = sorted(range(8), key=lambda j: (-r_score[j], j))
    cum = np.cumsum(P[:, order], axis=1)
    for tau in (0.5, 0.7, 0.9, 0.99):
        want = int(np.argmax(np.all(cum >= tau, axis=0))) + 1
        r = _run(wl, cfg, pool, pages, ks, vs, q, tau_cov=tau)
        assert np.all(r["k_cov"] == want), (tau, r["k_cov"][0], want)
        head0_only = int(np.argmax(cum[0] >= tau)) + 1
        if tau == 0.9:
            assert want != head0_only  # the case separates "every head" from "the first head"


def test_blocks_without_value_error_are_never_value_promoted():
    """Values on the int4 grid (each group holds 0 and 15, rotation off) are
    stored without loss: eta = 0, so even v_tol = 0 leaves such blocks
    alone, while every lossy block is promoted."""
    wl = W.scaled(W.ladder(), [512])  # 4 blocks
    rng = np.random.default_rng(3)
    v = rng.normal(0, 0.5, size=(512, wl.Hkv, wl.d)).astype(np.float16)
    grid = rng.integers(0, 16, size=(128, wl.Hkv, wl.d)).astype(np.float16)
    grid[:, :, ::32] = 0.0
    grid[:, :, 1::32] = 15.0
    v[128:256] = grid  # block 1 is lossless
    cfg, pool, pages, ks, vs = _case(wl, rotate=0, v_rows=[v])
    q = W.queries(wl, 0)
    r = _run(wl, cfg, pool, pages, ks, vs, q, v_tol=0.0)
    vset = (r["flags"][0] >> 1) & 1
    assert np.all(vset[:, 1] == 0) and np.all(vset[:, [0, 2, 3]] == 1)


def test_layer_fallback_needs_strictly_more_than_the_fraction():
    wl = W.scaled(W.ladder(), [1200, 700])  # 64 heads in the call
    cfg, pool, pages, ks, vs = _case(wl)
    q = W.queries(wl, 2)
    base = _run(wl, cfg, pool, pages, ks, vs, q, tau_cov=0.9)
    tol = float(np.sort(base["bound"].ravel())[-9])  # exactly 8 heads above it
    assert int((base["bound"] > tol).sum()) == 8
    at = _run(wl, cfg, pool, pages, ks, vs, q, tau_cov=0.9, cert_tol=tol, layer_frac=8 / 64)
    assert not np.any(at["status"] & O.LADDER_LAYER_DENSE)
    below = _run(wl, cfg, pool, pages, ks, vs, q, tau_cov=0.9, cert_tol=tol, layer_frac=7 / 64)
    assert np.all(below["status"] & O.LADDER_LAYER_DENSE)
