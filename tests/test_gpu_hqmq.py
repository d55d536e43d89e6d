"""GPU parity of the HQMQ codec ["Hurwitz Quaternion Multiplicative
Quantization for KV Cache Compression", 1-3]: the pool the append kernels
write (codebooks, 20-bit fields, radius steps, Med3x outlier masks and fp16
outlier slots) is bit-exact against the oracle, through both append paths (a
warp per row for bulk appends, the CTA per row for few-token appends), with
and without the rotation and on outlier-heavy rows; decode attention over the
codes meets the attention tolerance against the oracle's fp64 attention over
its own dequantised rows, for every GQA group size and for ragged and empty
sequences; the calls HQMQ does not serve refuse it."""
import concurrent.futures as cf
import dataclasses
import os

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


def _heavy_rows(wl, seed):
    """Raw K/V with a few blocks per row 20-200x longer (outlier-heavy models):
    rows with more than two such blocks clip the rest at the radius limit."""
    rng = np.random.default_rng(seed)
    rows = []
    for b in range(wl.B):
        kv = []
        for t in range(2):
            x = rng.standard_normal((wl.ctx[b], wl.Hkv, wl.d))
            for n in range(wl.ctx[b]):
                for h in range(wl.Hkv):
                    for blk in rng.choice(wl.d // 4, size=rng.integers(0, 4), replace=False):
                        x[n, h, 4 * blk:4 * blk + 4] *= rng.uniform(20, 200)
            kv.append(x.astype(np.float16))
        rows.append(tuple(kv))
    return rows


HQ = W.hqmq()
CASES = [
    # B=2: 37 tokens (592 rows: the CTA-per-row path), 300 (4800 rows: warp per row)
    ("llama-B2", W.scaled(HQ, [37, 300]), None),
    ("llama-B2-rotated", dataclasses.replace(W.scaled(HQ, [37, 300]), rotate=1), None),
    ("heavy-B2", dataclasses.replace(W.scaled(HQ, [40, 200]), Hkv=2, Hq=8), "heavy"),
    ("gqa1", dataclasses.replace(W.scaled(HQ, [90]), Hq=4, Hkv=4), None),
    ("gqa2", dataclasses.replace(W.scaled(HQ, [70]), Hq=8, Hkv=4), None),
    ("gqa8", dataclasses.replace(W.scaled(HQ, [130]), Hq=16, Hkv=2), None),
    ("ragged-B4", dataclasses.replace(W.scaled(HQ, [0, 1, 17, 33]), Hq=8, Hkv=2), None),
]


@pytest.mark.parametrize("name,wl,rows", CASES, ids=[c[0] for c in CASES])
def test_append_bit_exact_and_decode(name, wl, rows):
    import torch
    kv = _heavy_rows(wl, 11) if rows == "heavy" else None
    pair = build_pair(wl, kv_rows=kv)
    _bytes_equal(pair)
    q = W.queries(wl, 0)
    got = pair.cache.decode(torch.from_numpy(q).cuda(), pair.block_table(), pair.ctx()).cpu().numpy()
    want = O.decode(pair.ocfg, pair.opool, q, pair.pages.block_table, wl.ctx)
    max_abs, rel = attn_errors(got, want)
    assert max_abs <= TOL_MAX_ABS and rel <= TOL_REL_L2, f"max_abs={max_abs:.3e} rel={rel:.3e}"
    for b, T in enumerate(wl.ctx):
        if T == 0:
            assert np.all(got[b] == 0.0)
    assert pair.cache.sync_status() == 0
    if rows == "heavy":  # the outlier path ran: some rows keep fp16 blocks
        masks = [O.hqmq_read_row(pair.ocfg, pair.opool, int(s), 0, 0)[2] for s in pair.pages.slots(1, 0, 50)]
        assert any(m != 0 for m in masks)


def test_token_by_token_appends_match_one_bulk_append():
    """Decode-step appends (one token per call: the CTA shares each row) write
    the same bytes as the oracle's append of the same tokens."""
    import torch
    wl = dataclasses.replace(W.scaled(HQ, [24]), Hq=8, Hkv=2)
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
    wl = dataclasses.replace(W.scaled(HQ, [16]), Hq=8, Hkv=2)
    pair = build_pair(wl)
    before = pair.cache.pool.cpu().numpy().copy()
    k, v = W.step_kv(wl, 0)
    n_slots = pair.pages.num_pages * 16
    for bad, status in ((-1, K.KVQ_OK), (n_slots, K.KVQ_ERR_OUT_OF_RANGE)):
        pair.cache.append(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda(),
                          torch.tensor([bad], dtype=torch.int32, device="cuda"))
        assert pair.cache.sync_status() == status
        assert np.array_equal(pair.cache.pool.cpu().numpy()[256:], before[256:])


def test_calls_hqmq_does_not_serve():
    import torch
    import quantized_kv_cache_16_b200 as K
    wl = dataclasses.replace(W.scaled(HQ, [32]), Hq=8, Hkv=2)
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


def _oracle_head_cache(wl, kvh, pages, k, v, threads):
    """Oracle cache of kv head `kvh` alone (a one-head config codes a head's
    rows exactly as the full config does: the sign vector and the codebook
    of head 0 / tensor t are the same draws), appended by `threads` threads
    over disjoint token ranges (the C call releases the GIL)."""
    ocfg = O.make_config(wl.g, 1, wl.d, O.HQMQ, O.HQMQ, 4, 4, rotation_seed=wl.rotation_seed,
                         rotate=wl.rotate, num_pages=pages.num_pages)
    assert kvh == 0
    opool = O.new_pool(ocfg)
    T = k.shape[0]
    cuts = np.linspace(0, T, threads + 1).astype(int)
    kh, vh = np.ascontiguousarray(k[:, kvh:kvh + 1]), np.ascontiguousarray(v[:, kvh:kvh + 1])
    slots = pages.slots(0, 0, T)

    def part(i):
        a, b = cuts[i], cuts[i + 1]
        return O.append(ocfg, opool, kh[a:b], vh[a:b], slots[a:b])

    with cf.ThreadPoolExecutor(threads) as ex:
        assert all(rc == 0 for rc in ex.map(part, range(threads)))
    return ocfg, opool


@pytest.mark.slow
def test_full_size_sampled_rows_and_head0_attention():
    """The benchmark's workload (32768 tokens, 8 kv heads, GQA 4): 64 sampled
    tokens' rows of every head bit-exact; the attention of kv head 0's four
    query heads over the whole context against the oracle."""
    import torch
    wl = HQ
    pair = build_pair(wl, oracle=False)
    gpu = pair.cache.pool.cpu().numpy()
    k, v = pair.kv[0]
    T = wl.ctx[0]
    rng = np.random.default_rng(3)
    idx = np.sort(rng.choice(T, size=64, replace=False))
    idx[0], idx[-1] = 0, T - 1
    ocfg = pair.ocfg
    opool = O.new_pool(ocfg)
    slots = pair.pages.slots(0, 0, T)
    assert O.append(ocfg, opool, k[idx], v[idx], slots[idx]) == 0
    for s in slots[idx]:
        for h in range(wl.Hkv):
            for t in range(2):
                assert O.hqmq_read_row(ocfg, gpu, int(s), h, t)[0].tolist() == \
                    O.hqmq_read_row(ocfg, opool, int(s), h, t)[0].tolist()
                a = O.hqmq_read_row(ocfg, gpu, int(s), h, t)[1:]
                b = O.hqmq_read_row(ocfg, opool, int(s), h, t)[1:]
                assert a[0] == b[0] and a[1] == b[1] and np.array_equal(a[2], b[2])
    # kv head 0 over the whole context
    q = W.queries(wl, 0)
    got = pair.cache.decode(torch.from_numpy(q).cuda(), pair.block_table(), pair.ctx()).cpu().numpy()
    hcfg, hpool = _oracle_head_cache(wl, 0, pair.pages, k, v, threads=max(1, min(32, os.cpu_count() or 1)))
    want = O.decode(hcfg, hpool, q[:, :wl.g], pair.pages.block_table, wl.ctx)
    max_abs, rel = attn_errors(got[:, :wl.g], want)
    assert max_abs <= TOL_MAX_ABS and rel <= TOL_REL_L2, f"max_abs={max_abs:.3e} rel={rel:.3e}"
    assert pair.cache.sync_status() == 0
