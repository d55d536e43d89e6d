"""GPU parity of the certified decode mode ["Runtime-Certified Bounded-Error
Quantized Attention", Methodology 1-3] against the oracle.

  selection -> the promoted blocks (rank order) equal the oracle's; where
               they differ, every difference is a near-tie (scores within a
               relative 1e-4 of each other) and the output is then compared
               with the oracle run on the GPU's selection;
  output    -> max-abs <= 2e-3 and rel-L2 <= 1e-3 against the oracle's fp64
               certified output (promoted blocks exact, the rest dequantised);
  limits    -> 0% promotion is the plain quantised decode, bit for bit;
               100% promotion is fp16 attention.
The exact (tier-2) rows live in pinned host memory, as the pages place them.
"""
import numpy as np
import pytest

import oracle as O
import workloads as W
from _cases import TOL_MAX_ABS, TOL_REL_L2, attn_errors, build_pair

pytestmark = pytest.mark.gpu

NEAR_TIE = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import quantized_kv_cache_16_b200 as K
    K.lib()


def _tier2(pair, pinned=True):
    """Exact fp16 rows by slot: host arrays for the oracle, pinned (or
    device) tensors for the GPU."""
    import torch
    wl = pair.wl
    ks = np.zeros((pair.pages.num_pages * 16, wl.Hkv, wl.d), np.float16)
    vs = np.zeros_like(ks)
    for b in range(wl.B):
        sl = pair.pages.slots(b, 0, wl.ctx[b])
        ks[sl], vs[sl] = pair.kv[b]
    if pinned:
        kt, vt = torch.from_numpy(ks).pin_memory(), torch.from_numpy(vs).pin_memory()
    else:
        kt, vt = torch.from_numpy(ks).cuda(), torch.from_numpy(vs).cuda()
    return ks, vs, kt, vt


def _kmax(wl, frac, max_pages):
    return O.promote_count(float(np.float32(frac)), (max_pages * 16 + wl.bound_block - 1) // wl.bound_block)


def _run(pair, frac, step=0, pinned=True):
    import torch
    wl = pair.wl
    ks, vs, kt, vt = _tier2(pair, pinned)
    q = W.queries(wl, step)
    bt = pair.block_table()
    kmax = _kmax(wl, frac, bt.shape[1])
    prom = torch.full((wl.B, wl.Hkv, max(kmax, 1)), -7, dtype=torch.int32, device="cuda")
    out = pair.cache.decode_certified(torch.from_numpy(q).cuda(), bt, pair.ctx(), kt, vt, frac,
                                      promoted_out=prom if kmax else None)
    assert pair.cache.sync_status() == 0
    return out.cpu().numpy(), prom.cpu().numpy()[:, :, :kmax], (ks, vs, q, kmax)


def _check(pair, frac, step=0, pinned=True):
    wl = pair.wl
    got, gprom, (ks, vs, q, kmax) = _run(pair, frac, step, pinned)
    f32 = float(np.float32(frac))
    want, oprom, scores, _ = O.decode_certified(pair.ocfg, pair.opool, ks, vs, q, pair.pages.block_table,
                                                wl.ctx, f32)
    forced = False
    for b in range(wl.B):
        nb = (wl.ctx[b] + wl.bound_block - 1) // wl.bound_block
        k = O.promote_count(f32, nb)
        for kvh in range(wl.Hkv):
            g_sel, o_sel = gprom[b, kvh], oprom[b, kvh]
            assert np.all(g_sel[k:] == -1) and np.all(o_sel[k:kmax] == -1)
            if np.array_equal(g_sel[:k], o_sel[:k]):
                continue
            sc = scores[b, kvh, :nb]
            kth = np.sort(sc)[::-1][k - 1]
            assert len(set(g_sel[:k].tolist())) == k and all(0 <= x < nb for x in g_sel[:k])
            for x in g_sel[:k]:  # every GPU pick is within a near-tie of the k-th score
                assert sc[x] >= kth * (1 - NEAR_TIE), (b, kvh, x, sc[x], kth)
            for x, y in zip(g_sel[:k - 1], g_sel[1:k]):  # rank order, up to near-ties
                assert sc[x] >= sc[y] * (1 - NEAR_TIE)
            forced = True
    if forced:
        want, _, _, _ = O.decode_certified(pair.ocfg, pair.opool, ks, vs, q, pair.pages.block_table, wl.ctx, f32,
                                           forced=gprom)
    max_abs, rel = attn_errors(got, want)
    assert max_abs <= TOL_MAX_ABS and rel <= TOL_REL_L2, f"max_abs={max_abs:.3e} rel={rel:.3e}"
    return got, want


CASES = [
    ("T2000-f0.25", W.scaled(W.certified(), [2000]), 0.25),
    ("T1000-ragged-f0.2", W.scaled(W.certified(), [1000]), 0.2),
    ("B3-mixed-f0.01", W.scaled(W.certified(), [700, 1500, 129]), 0.01),
    ("B2-f0.5", W.scaled(W.certified(), [3000, 64]), 0.5),
]


@pytest.mark.parametrize("name,wl,frac", CASES, ids=[c[0] for c in CASES])
def test_certified_matches_oracle(name, wl, frac):
    _check(build_pair(wl), frac)


def test_certified_many_blocks_sorted_in_shared_memory():
    """1250 bound blocks of 16 tokens: more than the selection's register sort
    holds, so the shared-memory sort runs."""
    import dataclasses
    wl = dataclasses.replace(W.scaled(W.certified(), [20000]), bound_block=16)
    _check(build_pair(wl), 0.01)


def test_certified_tier2_on_the_device():
    _check(build_pair(W.scaled(W.certified(), [1200])), 0.3, pinned=False)


def test_certified_int4_keys_and_gqa8():
    import dataclasses
    wl = dataclasses.replace(W.scaled(W.certified(), [900, 333]), k_fmt=O.INT4_ASYM, k_group=32, Hq=64,
                             bound_block=64)
    _check(build_pair(wl), 0.2)


def test_certified_limits():
    """0% promotion is the plain quantised decode, bit for bit; 100% is fp16
    attention."""
    import torch
    wl = W.scaled(W.certified(), [1500, 200])
    pair = build_pair(wl)
    got0, prom0, _ = _run(pair, 0.0)
    q = torch.from_numpy(W.queries(wl, 0)).cuda()
    plain = pair.cache.decode(q, pair.block_table(), pair.ctx()).cpu().numpy()
    assert prom0.size == 0 and np.array_equal(got0, plain)
    got1, prom1, (ks, vs, qn, kmax) = _run(pair, 1.0)
    exact = O.decode_fp16(pair.ocfg, ks, vs, qn, pair.pages.block_table, wl.ctx)
    max_abs, rel = attn_errors(got1, exact)
    assert max_abs <= TOL_MAX_ABS and rel <= TOL_REL_L2, f"max_abs={max_abs:.3e} rel={rel:.3e}"
    for b in range(wl.B):
        nb = (wl.ctx[b] + 127) // 128
        for kvh in range(wl.Hkv):
            assert sorted(prom1[b, kvh, :nb].tolist()) == list(range(nb))


def test_certified_repeated_calls_reuse_the_workspace():
    """The promote counters return to zero: two calls in a row agree."""
    pair = build_pair(W.scaled(W.certified(), [2500]))
    a, pa, _ = _run(pair, 0.1, step=3)
    b, pb, _ = _run(pair, 0.1, step=3)
    assert np.array_equal(a, b) and np.array_equal(pa, pb)


@pytest.mark.slow
def test_certified_full_size():
    """Batch 1, context 131072, int8 keys / int4 values, 128-token blocks,
    top 1% promoted from pinned host memory."""
    _check(build_pair(W.certified()), 0.01)


def test_certified_rejects_bad_arguments():
    import torch
    import quantized_kv_cache_16_b200 as K
    wl = W.scaled(W.certified(), [300])
    pair = build_pair(wl)
    ks, vs, kt, vt = _tier2(pair)
    q = torch.from_numpy(W.queries(wl, 0)).cuda()
    bt, ctx = pair.block_table(), pair.ctx()
    with pytest.raises(K.KvqError) as e:
        pair.cache.decode_certified(q, bt, ctx, kt, vt, 1.5)
    assert e.value.status == K.KVQ_ERR_INVALID_ARG
    unpinned = torch.from_numpy(ks)  # pageable host memory: not device-accessible
    with pytest.raises(K.KvqError) as e:
        pair.cache.decode_certified(q, bt, ctx, unpinned, vt, 0.5)
    assert e.value.status == K.KVQ_ERR_INVALID_ARG
    plain = build_pair(W.scaled(W.llama(), [300]))  # no bound blocks
    with pytest.raises(K.KvqError) as e:
        plain.cache.decode_certified(torch.from_numpy(W.queries(plain.wl, 0)).cuda(), plain.block_table(),
                                     plain.ctx(), kt, vt, 0.5)
    assert e.value.status == K.KVQ_ERR_INVALID_ARG
