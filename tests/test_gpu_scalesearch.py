"""GPU parity of ScaleSearch ["Search Your Block Floating Point Scales!",
ScaleSearch] in the append kernel: with the search on, pool bytes (codes,
the searched scales, zeros, descriptors) are bit-exact against the oracle,
including a row built so that two candidates tie exactly; decoding a
searched cache meets the usual attention tolerance; the fused decode step
refuses such a cache."""
import dataclasses

import numpy as np
import pytest

import oracle as O
import workloads as W
from _cases import TOL_MAX_ABS, TOL_REL_L2, attn_errors, build_pair
from test_oracle_scalesearch import tie_row

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import quantized_kv_cache_16_b200 as K
    K.lib()


def _ss(wl):
    return dataclasses.replace(wl, scale_search=1)


CASES = [
    ("tiny", _ss(W.tiny())),
    ("llama-1000", _ss(W.scaled(W.llama(), 1000))),
    ("paged-B3-ragged", _ss(W.scaled(W.paged(), [37, 300, 17]))),
    ("int8k-2000", _ss(W.scaled(W.certified(), 2000))),
    ("int2-B2", _ss(W.scaled(W.int2(), [3000, 777]))),
]


def _bytes_equal(pair):
    gpu = pair.cache.pool.cpu().numpy()
    diff = np.nonzero(gpu[256:] != pair.opool[256:])[0]
    assert diff.size == 0, f"{diff.size} bytes differ, first at pool offset {256 + diff[0]}"


@pytest.mark.parametrize("name,wl", CASES, ids=[c[0] for c in CASES])
def test_searched_append_bit_exact_and_decodes(name, wl):
    import torch
    pair = build_pair(wl)
    _bytes_equal(pair)
    # the search moved some scales: the pool differs from the plain codec's
    plain = build_pair(dataclasses.replace(wl, scale_search=0), oracle=False)
    assert not np.array_equal(plain.cache.pool.cpu().numpy()[256:], pair.opool[256:])
    q = W.queries(wl, 0)
    got = pair.cache.decode(torch.from_numpy(q).cuda(), pair.block_table(), pair.ctx()).cpu().numpy()
    want = O.decode(pair.ocfg, pair.opool, q, pair.pages.block_table, wl.ctx)
    max_abs, rel = attn_errors(got, want)
    assert max_abs <= TOL_MAX_ABS and rel <= TOL_REL_L2, f"max_abs={max_abs:.3e} rel={rel:.3e}"
    assert pair.cache.sync_status() == 0


def test_exact_tie_keeps_the_default_scale():
    """Rotation off, every row of every head the tie row: the stored scales
    must be the default 0x2C00, not its tied neighbour."""
    wl = dataclasses.replace(W.tiny(), ctx=[32], scale_search=1)
    row = tie_row()[0].astype(np.float16)
    k = np.tile(row, (32, wl.Hkv, 1))
    pair = build_pair(wl, rotate=0, kv_rows=[(k, k.copy())])
    _bytes_equal(pair)
    c, meta_s, _ = O.read_row(pair.ocfg, pair.opool, int(pair.pages.slots(0, 0, 1)[0]), 0, 0)
    assert np.all(np.asarray(meta_s) == 0x2C00)


@pytest.mark.slow
def test_searched_bulk_prefill_full_size():
    """The 2-bit bulk prefill (65536 tokens x 8 kv heads, clip 0.9) with the
    search on, as the benchmark's append leg runs it."""
    wl = _ss(W.scaled(W.int2(), [65536]))
    _bytes_equal(build_pair(wl))


def test_fused_step_refuses_a_searched_cache():
    import torch
    import quantized_kv_cache_16_b200 as K
    wl = _ss(W.scaled(W.llama(), 100))
    pair = build_pair(wl, extra_tokens=1, oracle=False)
    kn, vn = (torch.from_numpy(x).cuda() for x in W.step_kv(wl, 0))
    slot = torch.tensor([pair.pages.slot(0, 100)], dtype=torch.int32, device="cuda")
    with pytest.raises(K.KvqError) as e:
        pair.cache.step(kn, vn, slot, torch.from_numpy(W.queries(wl, 0)).cuda(), pair.block_table(), pair.ctx(1))
    assert e.value.status == K.KVQ_ERR_UNSUPPORTED
