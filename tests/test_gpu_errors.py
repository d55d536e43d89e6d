"""Error behaviour through the C ABI: host-side argument checks return a
status and launch nothing; conditions only the device sees (slot or page
outside the pool, a context longer than the block table) are recorded in the
pool's status word and reported by kvq_sync_status.  Nothing here faults the
GPU: every bad index is one the kernels check before touching memory."""
import numpy as np
import pytest

import quantized_kv_cache_16_b200 as K
import workloads as W
from _cases import build_pair

pytestmark = pytest.mark.gpu


def _torch():
    import torch
    assert torch.cuda.is_available()
    return torch


def test_create_rejects_bad_pools():
    torch = _torch()
    cfg = K.make_config(32, 8, 128, num_pages=4)
    need = K.kvq_pool_bytes(cfg)
    small = torch.empty(need - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(K.KvqError) as e:
        K.kvq_create_cache(cfg, small)
    assert e.value.status == K.KVQ_ERR_CAPACITY
    host = torch.empty(need, dtype=torch.uint8)
    with pytest.raises(K.KvqError) as e:
        K.kvq_create_cache(cfg, host)
    assert e.value.status == K.KVQ_ERR_INVALID_ARG
    big = torch.empty(need + 512, dtype=torch.uint8, device="cuda")
    with pytest.raises(K.KvqError) as e:
        K.kvq_create_cache(cfg, big[8:], need)  # not 256-byte aligned
    assert e.value.status == K.KVQ_ERR_INVALID_ARG


def test_append_checks_arguments_and_slots():
    torch = _torch()
    c = K.Cache(K.make_config(8, 2, 64, num_pages=2))
    k = torch.randn(3, 2, 64, device="cuda").half()
    with pytest.raises(K.KvqError):
        K.kvq_append(c.handle, None, k, torch.zeros(3, dtype=torch.int32, device="cuda"))
    with pytest.raises(K.KvqError):  # misaligned k
        K.kvq_append(c.handle, k.view(-1)[1:], k, torch.zeros(3, dtype=torch.int32, device="cuda"), n_tok=1)
    # slot 32 is past the 2-page pool: recorded, the other tokens land
    slots = torch.tensor([0, 32, -1], dtype=torch.int32, device="cuda")
    c.append(k, k, slots)
    assert c.sync_status() == K.KVQ_ERR_OUT_OF_RANGE
    assert c.sync_status() == K.KVQ_OK  # read-and-clear
    assert c.pool[256:].any()


def test_decode_checks_arguments_and_indices():
    torch = _torch()
    wl = W.scaled(W.llama(), [40])
    pair = build_pair(wl, oracle=False)
    c = pair.cache
    q = torch.from_numpy(W.queries(wl, 0)).cuda()
    bt = pair.block_table()
    ctx = pair.ctx()
    ws_need = K.kvq_decode_workspace_bytes(c.handle, 1, bt.shape[1])
    ws = torch.zeros(ws_need, dtype=torch.uint8, device="cuda")
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    with pytest.raises(K.KvqError) as e:
        K.kvq_decode_attn(c.handle, q, bt, bt.shape[1], ctx, 1, 0.0, None, ws, ws_need - 256, out)
    assert e.value.status == K.KVQ_ERR_CAPACITY
    with pytest.raises(K.KvqError) as e:
        K.kvq_decode_attn(c.handle, None, bt, bt.shape[1], ctx, 1, 0.0, None, ws, ws_need, out)
    assert e.value.status == K.KVQ_ERR_INVALID_ARG
    # a page id outside the pool: recorded, that page is skipped
    bad = bt.clone()
    bad[0, 1] = 10_000
    K.kvq_decode_attn(c.handle, q, bad, bt.shape[1], ctx, 1, 0.0, None, ws, ws_need, out)
    assert c.sync_status() == K.KVQ_ERR_OUT_OF_RANGE
    # a context longer than the block table allows: recorded and clamped
    long_ctx = torch.tensor([bt.shape[1] * 16 + 5], dtype=torch.int32, device="cuda")
    K.kvq_decode_attn(c.handle, q, bt, bt.shape[1], long_ctx, 1, 0.0, None, ws, ws_need, out)
    assert c.sync_status() == K.KVQ_ERR_OUT_OF_RANGE
    # and the next plain call is clean and finite
    K.kvq_decode_attn(c.handle, q, bt, bt.shape[1], ctx, 1, 0.0, None, ws, ws_need, out)
    assert c.sync_status() == K.KVQ_OK
    assert torch.isfinite(out).all()


def test_timeout_path_reports_and_recovers():
    """The bounded-wait path, driven by the library's test hook (no copy is
    made to stall): every warp's first page wait counts as expired, the warp
    waits out the copies it started and attends nothing, and the call leaves
    KVQ_ERR_TIMEOUT for kvq_sync_status.  With the hook off, the next call on
    the same cache is the oracle's attention again."""
    torch = _torch()
    from _cases import TOL_MAX_ABS, TOL_REL_L2, attn_errors
    import oracle as O
    wl = W.scaled(W.llama(), [1000])
    pair = build_pair(wl)
    c = pair.cache
    qn = W.queries(wl, 0)
    q = torch.from_numpy(qn).cuda()
    bt = pair.block_table()
    ctx = pair.ctx()
    ws_need = K.kvq_decode_workspace_bytes(c.handle, 1, bt.shape[1])
    ws = torch.zeros(ws_need, dtype=torch.uint8, device="cuda")
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    with pytest.raises(K.KvqError):
        K.kvq_debug_expire_first_wait(c.handle, 3)
    K.kvq_debug_expire_first_wait(c.handle, 1)
    try:
        K.kvq_decode_attn(c.handle, q, bt, bt.shape[1], ctx, 1, 0.0, None, ws, ws_need, out)
        assert c.sync_status() == K.KVQ_ERR_TIMEOUT
    finally:
        K.kvq_debug_expire_first_wait(c.handle, 0)
    K.kvq_decode_attn(c.handle, q, bt, bt.shape[1], ctx, 1, 0.0, None, ws, ws_need, out)
    assert c.sync_status() == K.KVQ_OK
    want = O.decode(pair.ocfg, pair.opool, qn, pair.pages.block_table, wl.ctx)
    max_abs, rel = attn_errors(out.cpu().numpy(), want)
    assert max_abs <= TOL_MAX_ABS and rel <= TOL_REL_L2, (max_abs, rel)


def test_wrong_block_table_guesses_are_redone():
    """A decode CTA may start while the previous kernel is still running and
    reads the block table early to start its first page copies; with the
    test hook's mode 2 every such guess counts as wrong, so each warp waits
    its early copies out and copies the pages again.  The result is still
    the oracle's attention, for a single sequence and a ragged batch."""
    torch = _torch()
    from _cases import TOL_MAX_ABS, TOL_REL_L2, attn_errors
    import oracle as O
    for ctx in ([1000], [700, 31, 16]):
        wl = W.scaled(W.llama(), ctx)
        pair = build_pair(wl)
        c = pair.cache
        qn = W.queries(wl, 0)
        q = torch.from_numpy(qn).cuda()
        bt = pair.block_table()
        K.kvq_debug_expire_first_wait(c.handle, 2)
        try:
            out = c.decode(q, bt, pair.ctx())
            assert c.sync_status() == K.KVQ_OK
        finally:
            K.kvq_debug_expire_first_wait(c.handle, 0)
        want = O.decode(pair.ocfg, pair.opool, qn, pair.pages.block_table, wl.ctx)
        max_abs, rel = attn_errors(out.cpu().numpy(), want)
        assert max_abs <= TOL_MAX_ABS and rel <= TOL_REL_L2, (ctx, max_abs, rel)
