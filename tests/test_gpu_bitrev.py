"""OSCAR's bit-reversal permutation P_br on the GPU ("OSCAR", 2.2(a):
R = U H_Had P_br without the data-derived U; config rotate = 2): the bulk
append's pool bytes equal the oracle's, the decode, the fused decode step
and the certified call match the oracle's attention over the same cache,
for int4 g32, int8 K / int4 V and 2-bit rows at head_dim 128 and int4 at
head_dim 64.  The codecs that own their rotation (HQMQ, NVFP4) refuse the
option."""
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
    K.lib()  # fails loudly if the library is missing


CASES = [
    ("tiny-d64", W.tiny()),
    ("llama-1000", W.scaled(W.llama(), 1000)),
    ("paged-B3", W.scaled(W.paged(), [37, 300, 16])),
    ("int8k-700", W.scaled(W.certified(), 700)),
    ("int2-B2", W.scaled(W.int2(), [1000, 333])),
]


@pytest.mark.parametrize("name,wl", CASES, ids=[c[0] for c in CASES])
def test_append_and_decode_with_bit_reversal(name, wl):
    import torch
    pair = build_pair(wl, rotate=2)
    gpu = pair.cache.pool.cpu().numpy()
    diff = np.nonzero(gpu[256:] != pair.opool[256:])[0]
    assert diff.size == 0, f"{diff.size} bytes differ, first at pool offset {256 + diff[0]}"
    q = W.queries(wl, 0)
    out = pair.cache.decode(torch.from_numpy(q).cuda(), pair.block_table(), pair.ctx())
    want = O.decode(pair.ocfg, pair.opool, q, pair.pages.block_table, wl.ctx)
    max_abs, rel = attn_errors(out.float().cpu().numpy(), want)
    assert max_abs <= TOL_MAX_ABS and rel <= TOL_REL_L2, f"max_abs={max_abs:.3e} rel={rel:.3e}"
    assert pair.cache.sync_status() == 0


def _exact_attention(wl, k, v, q):
    """fp64 softmax attention of one sequence over its unquantised rows
    (kv head h // (Hq / Hkv), scale 1 / sqrt(d))."""
    g = wl.Hq // wl.Hkv
    out = np.zeros((1, wl.Hq, wl.d))
    for h in range(wl.Hq):
        s = k[:, h // g].astype(np.float64) @ q[0, h].astype(np.float64) / np.sqrt(wl.d)
        p = np.exp(s - s.max())
        out[0, h] = (p / p.sum()) @ v[:, h // g].astype(np.float64)
    return out


def test_bit_reversal_changes_the_stored_order_not_the_error():
    """The same rows under rotate = 1 and rotate = 2: different bytes (the
    channels of a row are stored in another order, so the int4 groups hold
    other coordinates), and an attention error against the exact fp64
    attention of the same size (the oracle gives rel-L2 0.273 and 0.217 on
    this case: the int4 error on these outlier-heavy rows is large, the two
    groupings differ in it by chance, not by design)."""
    import torch
    wl = W.scaled(W.llama(), 600)
    a, b = build_pair(wl, rotate=1, oracle=False), build_pair(wl, rotate=2, oracle=False)
    assert not np.array_equal(a.cache.pool.cpu().numpy()[256:], b.cache.pool.cpu().numpy()[256:])
    q = W.queries(wl, 0)
    ex = _exact_attention(wl, *a.kv[0], q)
    qd = torch.from_numpy(q).cuda()
    ea = attn_errors(a.cache.decode(qd, a.block_table(), a.ctx()).cpu().numpy(), ex)[1]
    eb = attn_errors(b.cache.decode(qd, b.block_table(), b.ctx()).cpu().numpy(), ex)[1]
    assert 0 < eb <= 1.25 * ea and ea < 0.4, (ea, eb)


STEP_CASES = [
    ("llama-ragged", W.scaled(W.llama(), [1000, 31, 16])),
    ("int2-B2", W.scaled(W.int2(), [301, 64])),
]


@pytest.mark.parametrize("name,wl", STEP_CASES, ids=[c[0] for c in STEP_CASES])
def test_decode_step_with_bit_reversal(name, wl):
    """kvq_decode_step codes the new token's rows with P_br too: the pool
    bytes equal the oracle's append, the output matches its attention."""
    import torch
    pair = build_pair(wl, extra_tokens=2, rotate=2)
    for step in range(2):
        k, v = W.step_kv(wl, step)
        slots = np.array([pair.pages.slot(b, wl.ctx[b] + step) for b in range(wl.B)], np.int32)
        q = W.queries(wl, step)
        out = pair.cache.step(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda(), torch.from_numpy(slots).cuda(),
                              torch.from_numpy(q).cuda(), pair.block_table(), pair.ctx(step + 1))
        assert O.append(pair.ocfg, pair.opool, k, v, slots) == 0
        assert pair.cache.sync_status() == 0
        assert np.array_equal(pair.cache.pool.cpu().numpy()[256:], pair.opool[256:])
        want = O.decode(pair.ocfg, pair.opool, q, pair.pages.block_table, [t + step + 1 for t in wl.ctx])
        max_abs, rel = attn_errors(out.cpu().numpy(), want)
        assert max_abs <= TOL_MAX_ABS and rel <= TOL_REL_L2, f"max_abs={max_abs:.3e} rel={rel:.3e}"


def test_certified_call_with_bit_reversal():
    """Certified mode (1% of the blocks promoted from pinned fp16 rows): the
    rotated query and the inverse rotation of the dequantised sums carry
    P_br; the selection and the output match the oracle's (the certified
    tests' own check)."""
    from test_gpu_certified import _check
    _check(build_pair(W.scaled(W.certified(), 2000), rotate=2), 0.01)


def test_ladder_with_bit_reversal():
    """The certified ladder (coverage, key-error growth, value promotion,
    ranking check, fallbacks) over a bit-reversed cache: flags, K*, bounds
    and output as the ladder tests check them."""
    from test_gpu_ladder import _check as ladder_check
    ladder_check(build_pair(W.scaled(W.ladder(), [2000, 300]), rotate=2),
                 dict(tau_cov=0.995, key_tol=0.02, v_tol=1e-3, rank_tol=0.05, cert_tol=5e-3))


def test_windows_with_bit_reversal():
    """fp16 sink and recent windows over a bit-reversed 2-bit cache: the
    window rows enter through the same rotated query."""
    from test_gpu_windows import _run as windows_run
    got, want, _ = windows_run(build_pair(W.scaled(W.int2(), [3000, 777]), rotate=2), 16, 500)
    max_abs, rel = attn_errors(got, want)
    assert max_abs <= TOL_MAX_ABS and rel <= TOL_REL_L2, f"max_abs={max_abs:.3e} rel={rel:.3e}"


def test_codecs_with_their_own_rotation_refuse_bit_reversal():
    import quantized_kv_cache_16_b200 as K
    for fmt, group in ((K.KVQ_NVFP4, 16), (K.KVQ_HQMQ, 4)):
        with pytest.raises(K.KvqError):
            K.Cache(K.make_config(32, 8, 128, fmt, fmt, group, group, rotate=2, num_pages=4))
