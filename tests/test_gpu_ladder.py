"""GPU parity of the certified ladder ["Runtime-Certified Bounded-Error
Quantized Attention", Methodology 3] against the oracle, through
kvq_decode_certified.

  decisions -> key/value flags, K*, fallback and status bits equal the
               oracle's; where fp32 and fp64 legitimately part, the
               difference must be a near-tie (a ranking score within a
               relative 1e-4 of the boundary block's, a coverage or key-term
               value within 1e-4 of its threshold, a bound or ranking margin
               within 1e-3 of its tolerance), and the outputs are then checked
               against the oracle run on the GPU's decisions;
  output    -> max-abs <= 2e-3 and rel-L2 <= 1e-3 against the oracle's fp64
               output (mixed, or fp16 attention for heads that fell back);
  bound     -> within a relative 2e-3 (+1e-6) of the oracle's.
The tier-2 rows live in pinned host memory unless a test says otherwise.
"""
import dataclasses

import numpy as np
import pytest

import oracle as O
import workloads as W
from _cases import TOL_MAX_ABS, TOL_REL_L2, attn_errors, build_pair

pytestmark = pytest.mark.gpu

NEAR = 1e-4
OFF = dict(tau_cov=0.0, max_frac=1.0, key_tol=np.inf, v_tol=np.inf, rank_tol=np.inf, cert_tol=np.inf,
           layer_frac=1.0)
DENSE = O.LADDER_HEAD_DENSE | O.LADDER_LAYER_DENSE


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import quantized_kv_cache_16_b200 as K
    K.lib()


def _tier2(pair, pinned=True, swap=None):
    """Exact fp16 rows by slot (host arrays for the oracle; pinned or device
    tensors for the GPU).  swap=(b, t0, t1, n): exchange the key rows of
    tokens [t0, t0+n) and [t1, t1+n) of sequence b in the store only."""
    import torch
    wl = pair.wl
    ks = np.zeros((pair.pages.num_pages * 16, wl.Hkv, wl.d), np.float16)
    vs = np.zeros_like(ks)
    for b in range(wl.B):
        sl = pair.pages.slots(b, 0, wl.ctx[b])
        ks[sl], vs[sl] = pair.kv[b]
    if swap is not None:
        b, t0, t1, n = swap
        s0, s1 = pair.pages.slots(b, t0, t0 + n), pair.pages.slots(b, t1, t1 + n)
        ks[s0], ks[s1] = ks[s1].copy(), ks[s0].copy()
    if pinned:
        kt, vt = torch.from_numpy(ks).pin_memory(), torch.from_numpy(vs).pin_memory()
    else:
        kt, vt = torch.from_numpy(ks).cuda(), torch.from_numpy(vs).cuda()
    return ks, vs, kt, vt


def _gpu(pair, pol, kt, vt, q):
    import torch
    out, rep = pair.cache.decode_ladder(torch.from_numpy(q).cuda(), pair.block_table(), pair.ctx(), kt, vt,
                                        report=True, **pol)
    assert pair.cache.sync_status() == 0
    return out.cpu().numpy(), {k: v.cpu().numpy() for k, v in rep.items()}


def _eta(pair):
    """Largest value error of every bound block [B, Hkv, nb] from the oracle
    pool's descriptors."""
    wl, cfg = pair.wl, pair.ocfg
    blk = wl.bound_block
    nbm = max(1, (max(wl.ctx) + blk - 1) // blk)
    desc = pair.opool[O.desc_offset(cfg):].view(np.float32).reshape(cfg.num_pages, wl.Hkv, 4)
    eta = np.zeros((wl.B, wl.Hkv, nbm))
    for b in range(wl.B):
        for p in range((wl.ctx[b] + 15) // 16):
            eta[b, :, p * 16 // blk] = np.maximum(eta[b, :, p * 16 // blk], desc[pair.pages.block_table[b, p], :, 1])
    return eta


def _first(mask):
    idx = np.nonzero(mask)[0]
    return int(idx[0]) if idx.size else len(mask) - 1


def _check_flags(pair, pol, o, rep):
    """Accept the GPU's flags where they equal the oracle's, or differ only
    on near-ties; returns True if they differ anywhere."""
    wl = pair.wl
    blk = wl.bound_block
    eta = _eta(pair)
    differ = False
    for b in range(wl.B):
        nb = (wl.ctx[b] + blk - 1) // blk
        for kvh in range(wl.Hkv):
            gf, of = rep["flags"][b, kvh, :nb], o["flags"][b, kvh, :nb]
            assert np.all(rep["flags"][b, kvh, nb:] == 0)
            gk = np.nonzero(gf & 1)[0]
            assert len(gk) == rep["k_star"][b, kvh]
            if np.array_equal(gf, of):
                continue
            differ = True
            rs = o["rscore"][b, kvh, :nb]
            kg = len(gk)
            if kg:  # a top-kg set by the oracle's ranking, up to near-ties
                lo = rs[gk].min()
                assert np.all(np.delete(rs, gk) <= lo * (1 + NEAR)), (b, kvh)
            ko = int(o["k_star"][b, kvh])
            if kg != ko:  # the count must sit at a near-tie of a threshold
                cov, ek = o["cov"][b, kvh, :nb + 1], o["ekey"][b, kvh, :nb + 1]
                cap = O.promote_count(float(np.float32(pol["max_frac"])), nb)
                tau, kt = pol["tau_cov"], pol["key_tol"]
                kc_lo = 0 if tau <= 0 else _first(cov >= tau * (1 - NEAR))
                kc_hi = 0 if tau <= 0 else _first(cov >= tau * (1 + NEAR)) if tau * (1 + NEAR) <= 1 else nb
                kk_lo = _first(ek <= kt * (1 + NEAR) + 1e-6)
                kk_hi = _first(ek <= max(kt * (1 - NEAR) - 1e-6, 0.0)) if np.isfinite(kt) else 0
                lo_k, hi_k = min(cap, max(kc_lo, kk_lo)), min(cap, max(kc_hi, kk_hi))
                assert lo_k <= kg <= hi_k, (b, kvh, kg, ko, lo_k, hi_k)
            gv, ov = (gf >> 1) & 1, (of >> 1) & 1
            for x in np.nonzero(gv != ov)[0]:
                w = rs[x] * eta[b, kvh, x]
                assert abs(w - pol["v_tol"]) <= NEAR * pol["v_tol"] + 1e-9, (b, kvh, x, w)
    return differ


def _check(pair, pol, step=0, pinned=True, swap=None, q=None):
    pol = dict(OFF, **pol)
    wl = pair.wl
    ks, vs, kt, vt = _tier2(pair, pinned, swap)
    q = W.queries(wl, step) if q is None else q
    got, rep = _gpu(pair, pol, kt, vt, q)
    nbc = rep["flags"].shape[2]
    bt, ctx = pair.pages.block_table, wl.ctx
    o = O.decode_ladder(pair.ocfg, pair.opool, ks, vs, q, bt, ctx, pol, max_blocks=nbc)
    forced_flags = rep["flags"] if _check_flags(pair, pol, o, rep) else None
    if forced_flags is not None:
        o = O.decode_ladder(pair.ocfg, pair.opool, ks, vs, q, bt, ctx, pol, max_blocks=nbc, forced_flags=forced_flags)
    # fallback decisions: equal, or near-ties of the bound / the ranking margin
    gst, ost = rep["status"], o["status"]
    g_rank, o_rank = (gst & O.LADDER_RANK_FAIL) != 0, (ost & O.LADDER_RANK_FAIL) != 0
    g_bnd, o_bnd = (gst & O.LADDER_BOUND_FAIL) != 0, (ost & O.LADDER_BOUND_FAIL) != 0
    for i in zip(*np.nonzero(g_rank != o_rank)):
        assert abs(o["rank_margin"][i] - pol["rank_tol"]) <= 1e-3 * (1 + pol["rank_tol"]), (i, o["rank_margin"][i])
    for i in zip(*np.nonzero(g_bnd != o_bnd)):
        assert abs(o["bound"][i] - pol["cert_tol"]) <= 1e-3 * pol["cert_tol"] + 1e-6, (i, o["bound"][i])
    g_dense = (gst & DENSE) != 0
    if forced_flags is not None or not np.array_equal(g_dense, (ost & DENSE) != 0):
        o = O.decode_ladder(pair.ocfg, pair.opool, ks, vs, q, bt, ctx, pol, max_blocks=nbc,
                            forced_flags=rep["flags"], forced_fallback=g_dense.astype(np.int32))
    else:
        assert np.array_equal(gst, ost)
        assert np.array_equal(rep["k_star"], o["k_star"])
    bnd_err = np.abs(rep["bound"] - o["bound"])
    assert np.all(bnd_err <= 2e-3 * np.abs(o["bound"]) + 1e-6), float(bnd_err.max())
    max_abs, rel = attn_errors(got, o["out"])
    assert max_abs <= TOL_MAX_ABS and rel <= TOL_REL_L2, f"max_abs={max_abs:.3e} rel={rel:.3e}"
    return got, rep, o


CASES = [
    ("needle-T2000", W.scaled(W.ladder(), [2000]),
     dict(tau_cov=0.995, key_tol=0.02, v_tol=1e-3, rank_tol=0.05, cert_tol=5e-3, layer_frac=0.9)),
    ("needle-B4-empty-ragged-capped", W.scaled(W.ladder(), [0, 700, 1500, 129]),
     dict(tau_cov=0.99, max_frac=0.5, key_tol=0.05, v_tol=2e-3, rank_tol=0.1, cert_tol=1e-2)),
    ("diffuse-T2500-capped", W.scaled(W.certified(), [2500]), dict(tau_cov=0.9, max_frac=0.25, rank_tol=0.1)),
    ("int4k-gqa8-B2", dataclasses.replace(W.scaled(W.ladder(), [900, 333]), k_fmt=O.INT4_ASYM, k_group=32, Hq=64,
                                          bound_block=64),
     dict(tau_cov=0.99, key_tol=0.05, v_tol=1e-3, rank_tol=0.1, cert_tol=2e-2)),
    ("d64-int4k-block32", dataclasses.replace(W.scaled(W.ladder(), [1000]), d=64, Hq=8, Hkv=2, k_fmt=O.INT4_ASYM,
                                              k_group=32, bound_block=32),
     dict(tau_cov=0.99, key_tol=0.01, v_tol=1e-3, rank_tol=0.05, cert_tol=1e-2)),
]


@pytest.mark.parametrize("name,wl,pol", CASES, ids=[c[0] for c in CASES])
def test_ladder_matches_oracle(name, wl, pol):
    _check(build_pair(wl), pol)


def test_ladder_many_blocks_sorted_in_shared_memory():
    """1250 bound blocks of 16 tokens and K* near a thousand: the selection
    sorts more keys than its registers hold, and so does the ranking check
    wherever K* exceeds 1024."""
    wl = dataclasses.replace(W.scaled(W.certified(), [20000]), bound_block=16)
    _, rep, _ = _check(build_pair(wl), dict(tau_cov=0.9, v_tol=1e-4, rank_tol=0.2))
    assert rep["k_star"].max() > 1024


def test_ladder_tier2_on_the_device():
    _check(build_pair(W.scaled(W.ladder(), [1200])), dict(tau_cov=0.995, v_tol=1e-3, rank_tol=0.05, cert_tol=5e-3),
           pinned=False)


def test_ladder_off_is_the_quantised_decode_bit_for_bit():
    import torch
    pair = build_pair(W.scaled(W.ladder(), [1500, 64]))
    ks, vs, kt, vt = _tier2(pair)
    q = W.queries(pair.wl, 0)
    got, rep = _gpu(pair, OFF, kt, vt, q)
    plain = pair.cache.decode(torch.from_numpy(q).cuda(), pair.block_table(), pair.ctx()).cpu().numpy()
    assert np.array_equal(got, plain)
    assert np.all(rep["k_star"] == 0) and not rep["flags"].any() and np.all(rep["status"] == 0)
    o = O.decode_ladder(pair.ocfg, pair.opool, ks, vs, q, pair.pages.block_table, pair.wl.ctx, OFF)
    assert np.all(np.abs(rep["bound"] - o["bound"]) <= 2e-3 * o["bound"] + 1e-6)


def test_ladder_everything_exact_is_fp16_attention():
    pair = build_pair(W.scaled(W.ladder(), [1100, 300]))
    ks, vs, kt, vt = _tier2(pair)
    q = W.queries(pair.wl, 1)
    got, rep = _gpu(pair, dict(OFF, tau_cov=1.0, v_tol=0.0), kt, vt, q)
    exact = O.decode_fp16(pair.ocfg, ks, vs, q, pair.pages.block_table, pair.wl.ctx)
    max_abs, rel = attn_errors(got, exact)
    assert max_abs <= TOL_MAX_ABS and rel <= TOL_REL_L2
    assert np.all(rep["bound"] == 0.0)


def test_ranking_check_catches_a_tampered_tier2_store():
    """Swap the tier-2 keys of two hot spans (a needle and the recent window)
    in the store only: the exact masses of their blocks trade places, the
    check fails and those heads come back as fp16 attention over the store."""
    wl = W.scaled(W.ladder(), [2048])
    pair = build_pair(wl)
    pos, _ = W.hot_tokens(wl, 0)
    needle = int(pos[(pos >= 256) & (pos < 2048 - 384)][0]) // 128 * 128
    swap = (0, needle, 2048 - 128, 128)
    _, rep, o = _check(pair, dict(tau_cov=0.995, rank_tol=0.05), swap=swap)
    assert np.any(rep["status"] & O.LADDER_RANK_FAIL)
    assert np.array_equal((rep["status"] & O.LADDER_HEAD_DENSE) != 0, (rep["status"] & O.LADDER_RANK_FAIL) != 0)


def test_layer_fallback_recomputes_every_head():
    pair = build_pair(W.scaled(W.ladder(), [1500, 900]))
    ks, vs, kt, vt = _tier2(pair)
    q = W.queries(pair.wl, 2)
    o = O.decode_ladder(pair.ocfg, pair.opool, ks, vs, q, pair.pages.block_table, pair.wl.ctx,
                        dict(OFF, tau_cov=0.99))
    bs = np.sort(o["bound"].ravel())[::-1]
    n = next(k for k in range(4, 40) if bs[k - 1] > bs[k] * 1.02)  # n heads above the cut, no near-tie
    tol = float(np.sqrt(bs[n - 1] * bs[n]))
    _, rep, _ = _check(pair, dict(tau_cov=0.99, cert_tol=tol, layer_frac=(n - 1) / 64), q=q)
    assert np.all(rep["status"] & O.LADDER_LAYER_DENSE)
    _, rep, _ = _check(pair, dict(tau_cov=0.99, cert_tol=tol, layer_frac=n / 64), q=q)
    assert not np.any(rep["status"] & O.LADDER_LAYER_DENSE)
    assert int(((rep["status"] & O.LADDER_HEAD_DENSE) != 0).sum()) == n


def test_ladder_repeated_calls_reuse_the_workspace():
    """Counters return to zero: two calls in a row agree bit for bit, and a
    call that falls back everywhere leaves the next one unaffected."""
    pair = build_pair(W.scaled(W.ladder(), [2500]))
    ks, vs, kt, vt = _tier2(pair)
    q = W.queries(pair.wl, 3)
    pol = dict(OFF, tau_cov=0.995, v_tol=1e-3, rank_tol=0.05, cert_tol=5e-3)
    a, ra = _gpu(pair, pol, kt, vt, q)
    _gpu(pair, dict(pol, cert_tol=0.0), kt, vt, q)
    b, rb = _gpu(pair, pol, kt, vt, q)
    assert np.array_equal(a, b)
    for k in ra:
        assert np.array_equal(ra[k], rb[k]), k


@pytest.mark.slow
def test_ladder_full_size():
    """Batch 1, context 131072, int8 keys / int4 values, 128-token blocks,
    attention concentrated on a sink, six needles and the recent window."""
    _check(build_pair(W.ladder()), dict(tau_cov=0.995, max_frac=0.05, key_tol=0.02, v_tol=1e-3, rank_tol=0.05,
                                        cert_tol=5e-3, layer_frac=0.5))


def test_ladder_rejects_bad_arguments():
    import torch
    import quantized_kv_cache_16_b200 as K
    pair = build_pair(W.scaled(W.ladder(), [300]))
    ks, vs, kt, vt = _tier2(pair)
    q = torch.from_numpy(W.queries(pair.wl, 0)).cuda()
    bt, ctx = pair.block_table(), pair.ctx()
    for bad in (dict(tau_cov=1.5), dict(tau_cov=float("nan")), dict(max_frac=-0.1), dict(key_tol=-1.0),
                dict(v_tol=float("nan")), dict(rank_tol=-0.5), dict(cert_tol=-1e-3), dict(layer_frac=2.0)):
        with pytest.raises(K.KvqError) as e:
            pair.cache.decode_ladder(q, bt, ctx, kt, vt, **bad)
        assert e.value.status == K.KVQ_ERR_INVALID_ARG, bad
    with pytest.raises(K.KvqError) as e:  # pageable host memory is not device-accessible
        pair.cache.decode_ladder(q, bt, ctx, torch.from_numpy(ks), vt)
    assert e.value.status == K.KVQ_ERR_INVALID_ARG
    plain = build_pair(W.scaled(W.llama(), [300]))  # no bound blocks
    with pytest.raises(K.KvqError) as e:
        plain.cache.decode_ladder(torch.from_numpy(W.queries(plain.wl, 0)).cuda(), plain.block_table(), plain.ctx(),
                                  kt, vt)
    assert e.value.status == K.KVQ_ERR_INVALID_ARG
    ws = pair.cache.workspace_for(1, bt.shape[1])
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    small = K.kvq_ladder_report(0, torch.zeros(1, 8, 1, dtype=torch.uint8, device="cuda").data_ptr(), 1, 0, 0)
    with pytest.raises(K.KvqError) as e:  # fewer flag columns than blocks
        K.kvq_decode_certified(pair.cache.handle, q, bt, bt.shape[1], ctx, 1, 0.0, kt, vt,
                               K.kvq_ladder(0.9, 1, float("inf"), float("inf"), float("inf"), float("inf"), 1),
                               ws, ws.numel(), out, small)
    assert e.value.status == K.KVQ_ERR_INVALID_ARG
    assert pair.cache.sync_status() == 0
