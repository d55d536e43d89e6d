"""GPU parity of the NVFP4 codec ["Search Your Block Floating Point Scales!",
NVFP4 and ScaleSearch]: the pool the append kernel writes (e2m1 codes and
E4M3 scale bytes, with and without ScaleSearch, rotation on and off, values
across the E4M3 range) is bit-exact against the oracle; decode attention
over the codes (hardware fp4/fp8 conversions feeding the tensor cores)
meets the attention tolerance against the oracle's fp64 attention, for
every GQA group size and for ragged and empty sequences; the calls NVFP4
does not serve refuse it."""
import dataclasses

import numpy as np
import pytest

import oracle as O
import workloads as W
from _cases import TOL_MAX_ABS, TOL_REL_L2, attn_errors, build_pair

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import quantized_kv_cache_16_b200 as K
    K.lib()


def _bytes_equal(pair):
    gpu = pair.cache.pool.cpu().numpy()
    diff = np.nonzero(gpu[256:] != pair.opool[256:])[0]
    assert diff.size == 0, f"{diff.size} bytes differ, first at pool offset {256 + diff[0]}"


def _wide_rows(wl, seed):
    """Rows whose blocks span the E4M3 scale range: each token-head row
    scaled by 2^u, u uniform in [-14, 11] (block scales from subnormal to
    the saturated 448)."""
    rng = np.random.default_rng(seed)
    out = []
    for b in range(wl.B):
        kv = []
        for _ in range(2):
            x = rng.standard_normal((wl.ctx[b], wl.Hkv, wl.d)) * np.exp2(rng.uniform(-14, 11, (wl.ctx[b], wl.Hkv, 1)))
            kv.append(np.clip(x, -60000, 60000).astype(np.float16))
        out.append(tuple(kv))
    return out


NV = W.nvfp4()
CASES = [
    ("search-B2", W.scaled(NV, [37, 300]), None),
    ("default-B2", dataclasses.replace(W.scaled(NV, [37, 300]), scale_search=0), None),
    ("search-unrotated", dataclasses.replace(W.scaled(NV, [90]), rotate=0), None),
    ("laplace-outliers", dataclasses.replace(W.scaled(NV, [200]), dist="laplace", Hq=8, Hkv=2), None),
    ("wide-range", dataclasses.replace(W.scaled(NV, [64, 96]), Hq=8, Hkv=2, rotate=0), "wide"),
    ("gqa1", dataclasses.replace(W.scaled(NV, [90]), Hq=4, Hkv=4), None),
    ("gqa2", dataclasses.replace(W.scaled(NV, [70]), Hq=8, Hkv=4), None),
    ("gqa8", dataclasses.replace(W.scaled(NV, [130]), Hq=16, Hkv=2), None),
    ("ragged-B4", dataclasses.replace(W.scaled(NV, [0, 1, 17, 33]), Hq=8, Hkv=2), None),
]


@pytest.mark.parametrize("name,wl,rows", CASES, ids=[c[0] for c in CASES])
def test_append_bit_exact_and_decode(name, wl, rows):
    import torch
    kv = _wide_rows(wl, 13) if rows == "wide" else None
    pair = build_pair(wl, kv_rows=kv)
    _bytes_equal(pair)
    q = W.queries(wl, 0)
    got = pair.cache.decode(torch.from_numpy(q).cuda(), pair.block_table(), pair.ctx()).cpu().numpy()
    want = O.decode(pair.ocfg, pair.opool, q, pair.pages.block_table, wl.ctx)
    if rows == "wide":  # tolerance relative to each head's output scale
        scale = np.maximum(np.abs(want).max(axis=2, keepdims=True), 1e-30)
        got, want = got / scale, want / scale
    max_abs, rel = attn_errors(got, want)
    assert max_abs <= TOL_MAX_ABS and rel <= TOL_REL_L2, f"max_abs={max_abs:.3e} rel={rel:.3e}"
    for b, T in enumerate(wl.ctx):
        if T == 0:
            assert np.all(got[b] == 0.0)
    assert pair.cache.sync_status() == 0


def test_token_by_token_appends():
    import torch
    wl = dataclasses.replace(W.scaled(NV, [24]), Hq=8, Hkv=2)
    pair = build_pair(wl, extra_tokens=6)
    for step in range(6):
        kn, vn = W.step_kv(wl, step)
        slot = pair.pages.slots(0, wl.ctx[0] + step, wl.ctx[0] + step + 1)
        pair.cache.append(torch.from_numpy(kn).cuda(), torch.from_numpy(vn).cuda(), torch.from_numpy(slot).cuda())
        assert O.append(pair.ocfg, pair.opool, kn, vn, slot) == 0
    torch.cuda.synchronize()
    _bytes_equal(pair)


def test_bad_and_skipped_slots():
    import torch
    import quantized_kv_cache_16_b200 as K
    wl = dataclasses.replace(W.scaled(NV, [16]), Hq=8, Hkv=2)
    pair = build_pair(wl)
    before = pair.cache.pool.cpu().numpy().copy()
    k, v = W.step_kv(wl, 0)
    n_slots = pair.pages.num_pages * 16
    for bad, status in ((-1, K.KVQ_OK), (n_slots, K.KVQ_ERR_OUT_OF_RANGE)):
        pair.cache.append(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda(),
                          torch.tensor([bad], dtype=torch.int32, device="cuda"))
        assert pair.cache.sync_status() == status
        assert np.array_equal(pair.cache.pool.cpu().numpy()[256:], before[256:])


def test_calls_nvfp4_does_not_serve():
    """With ScaleSearch the fused step refuses the cache (its append codes
    with the default scales); the integer read-back refuses NVFP4."""
    import torch
    import quantized_kv_cache_16_b200 as K
    wl = dataclasses.replace(W.scaled(NV, [32]), Hq=8, Hkv=2)
    pair = build_pair(wl, extra_tokens=1, oracle=False)
    q = torch.from_numpy(W.queries(wl, 0)).cuda()
    kn, vn = (torch.from_numpy(x).cuda() for x in W.step_kv(wl, 0))
    slot = torch.tensor([pair.pages.slot(0, 32)], dtype=torch.int32, device="cuda")
    with pytest.raises(K.KvqError) as e:
        pair.cache.step(kn, vn, slot, q, pair.block_table(), pair.ctx(1))
    assert e.value.status == K.KVQ_ERR_UNSUPPORTED
    with pytest.raises(K.KvqError) as e:
        pair.cache.dequant(torch.tensor(pair.pages.slots(0, 0, 4)).cuda())
    assert e.value.status == K.KVQ_ERR_UNSUPPORTED


@pytest.mark.slow
def test_full_size_bit_exact_and_decode():
    """The benchmark's workload (32768 tokens, 8 kv heads, GQA 4, ScaleSearch):
    the whole pool bit-exact and the attention within tolerance."""
    import torch
    wl = NV
    pair = build_pair(wl)
    _bytes_equal(pair)
    q = W.queries(wl, 0)
    got = pair.cache.decode(torch.from_numpy(q).cuda(), pair.block_table(), pair.ctx()).cpu().numpy()
    want = O.decode(pair.ocfg, pair.opool, q, pair.pages.block_table, wl.ctx)
    max_abs, rel = attn_errors(got, want)
    assert max_abs <= TOL_MAX_ABS and rel <= TOL_REL_L2, f"max_abs={max_abs:.3e} rel={rel:.3e}"
    assert pair.cache.sync_status() == 0


@pytest.mark.parametrize("rotate", [1, 0])
def test_decode_step_fuses_append_and_decode(rotate):
    """Without ScaleSearch, kvq_decode_step on an NVFP4 cache stores exactly
    the bytes kvq_append (and the oracle) stores and returns exactly what
    kvq_append followed by kvq_decode_attn returns."""
    import torch
    wl = dataclasses.replace(W.scaled(NV, [300, 31, 16]), scale_search=0, rotate=rotate)
    fused = build_pair(wl, extra_tokens=2)
    split = build_pair(wl, extra_tokens=2, oracle=False)
    for step in range(2):
        k, v = W.step_kv(wl, step)
        slots = np.array([fused.pages.slot(b, wl.ctx[b] + step) for b in range(wl.B)], np.int32)
        q = torch.from_numpy(W.queries(wl, step)).cuda()
        kd, vd, sd = torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda(), torch.from_numpy(slots).cuda()
        out_f = fused.cache.step(kd, vd, sd, q, fused.block_table(), fused.ctx(step + 1))
        split.cache.append(kd, vd, sd)
        out_s = split.cache.decode(q, split.block_table(), split.ctx(step + 1))
        assert O.append(fused.ocfg, fused.opool, k, v, slots) == 0
        assert fused.cache.sync_status() == 0
        _bytes_equal(fused)
        assert np.array_equal(out_f.cpu().numpy(), out_s.cpu().numpy())
        want = O.decode(fused.ocfg, fused.opool, W.queries(wl, step), fused.pages.block_table,
                        [t + step + 1 for t in wl.ctx])
        max_abs, rel = attn_errors(out_f.cpu().numpy(), want)
        assert max_abs <= TOL_MAX_ABS and rel <= TOL_REL_L2, f"max_abs={max_abs:.3e} rel={rel:.3e}"
