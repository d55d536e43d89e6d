"""GPU parity of the decode with 16-bit sink and recent windows ["OSCAR",
2.2b] against the oracle: max-abs <= 2e-3 and rel-L2 <= 1e-3, with the
windows' limits (empty = the quantised decode bit for bit; covering every
token = fp16 attention), ragged and overlapping windows, a ring that has
wrapped, and a workspace shared with the certified calls."""
import numpy as np
import pytest

import oracle as O
import workloads as W
from _cases import TOL_MAX_ABS, TOL_REL_L2, attn_errors, build_pair
from test_oracle_windows import window_store

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import quantized_kv_cache_16_b200 as K
    K.lib()


def _run(pair, sink, recent, step=0, device=True):
    import torch
    wl = pair.wl
    wk, wv = window_store(wl, pair.kv, sink, recent)
    q = W.queries(wl, step)
    if device:
        kt, vt = torch.from_numpy(wk).cuda(), torch.from_numpy(wv).cuda()
    else:
        kt, vt = torch.from_numpy(wk).pin_memory(), torch.from_numpy(wv).pin_memory()
    got = pair.cache.decode_windows(torch.from_numpy(q).cuda(), pair.block_table(), pair.ctx(), kt, vt, sink,
                                    recent).cpu().numpy()
    assert pair.cache.sync_status() == 0
    want = O.decode_windows(pair.ocfg, pair.opool, wk, wv, sink, recent, q, pair.pages.block_table, wl.ctx)
    return got, want, q


CASES = [
    ("llama-4000-s64-r512", W.scaled(W.llama(), [4000]), 64, 512),
    ("paged-B4-s16-r100", W.scaled(W.paged(), [37, 700, 16, 1500]), 16, 100),
    ("int8k-2000-s128-r256", W.scaled(W.certified(), [2000]), 128, 256),
    ("int2-B2-s4-r1000", W.scaled(W.int2(), [3000, 777]), 4, 1000),
    ("tiny-overlap", W.tiny(), 100, 200),
]


@pytest.mark.parametrize("name,wl,sink,recent", CASES, ids=[c[0] for c in CASES])
def test_windows_match_oracle(name, wl, sink, recent):
    got, want, _ = _run(build_pair(wl), sink, recent)
    max_abs, rel = attn_errors(got, want)
    assert max_abs <= TOL_MAX_ABS and rel <= TOL_REL_L2, f"max_abs={max_abs:.3e} rel={rel:.3e}"


def test_window_store_in_pinned_host_memory():
    got, want, _ = _run(build_pair(W.scaled(W.llama(), [2500])), 32, 256, device=False)
    max_abs, rel = attn_errors(got, want)
    assert max_abs <= TOL_MAX_ABS and rel <= TOL_REL_L2


def test_empty_windows_are_the_quantised_decode_and_full_ones_fp16():
    import torch
    wl = W.scaled(W.llama(), [1200, 300])
    pair = build_pair(wl)
    got, _, q = _run(pair, 0, 0)
    plain = pair.cache.decode(torch.from_numpy(q).cuda(), pair.block_table(), pair.ctx()).cpu().numpy()
    assert np.array_equal(got, plain)
    ks = np.zeros((pair.pages.num_pages * 16, wl.Hkv, wl.d), np.float16)
    vs = np.zeros_like(ks)
    for b in range(wl.B):
        sl = pair.pages.slots(b, 0, wl.ctx[b])
        ks[sl], vs[sl] = pair.kv[b]
    got, _, q = _run(pair, 0, 1200)
    exact = O.decode_fp16(pair.ocfg, ks, vs, q, pair.pages.block_table, wl.ctx)
    max_abs, rel = attn_errors(got, exact)
    assert max_abs <= TOL_MAX_ABS and rel <= TOL_REL_L2


def test_workspace_shared_with_certified_calls():
    """Window, certified and window calls in a row on one workspace agree with
    the oracle each time (each kind leaves its own counters zero)."""
    import torch
    wl = W.scaled(W.certified(), [1500])
    pair = build_pair(wl)
    ks = np.zeros((pair.pages.num_pages * 16, wl.Hkv, wl.d), np.float16)
    vs = np.zeros_like(ks)
    sl = pair.pages.slots(0, 0, 1500)
    ks[sl], vs[sl] = pair.kv[0]
    a, want, q = _run(pair, 64, 256)
    pair.cache.decode_certified(torch.from_numpy(q).cuda(), pair.block_table(), pair.ctx(),
                                torch.from_numpy(ks).cuda(), torch.from_numpy(vs).cuda(), 0.3)
    pair.cache.decode_ladder(torch.from_numpy(q).cuda(), pair.block_table(), pair.ctx(),
                             torch.from_numpy(ks).cuda(), torch.from_numpy(vs).cuda(), cert_tol=0.0)
    b, _, _ = _run(pair, 64, 256)
    assert np.array_equal(a, b)
    max_abs, rel = attn_errors(b, want)
    assert max_abs <= TOL_MAX_ABS and rel <= TOL_REL_L2


def test_windows_reject_bad_arguments():
    import torch
    import quantized_kv_cache_16_b200 as K
    pair = build_pair(W.scaled(W.llama(), [300]), oracle=False)
    q = torch.from_numpy(W.queries(pair.wl, 0)).cuda()
    wk = torch.zeros((1, 8, 8, 128), dtype=torch.float16)  # pageable host memory
    with pytest.raises(K.KvqError) as e:
        pair.cache.decode_windows(q, pair.block_table(), pair.ctx(), wk, wk, 4, 4)
    assert e.value.status == K.KVQ_ERR_INVALID_ARG
    with pytest.raises(K.KvqError) as e:
        pair.cache.decode_windows(q, pair.block_table(), pair.ctx(), wk.cuda(), wk.cuda(), -1, 4)
    assert e.value.status == K.KVQ_ERR_INVALID_ARG
