"""kvq_decode_attn_static: decode attention for callers that cannot allocate
device memory (an engine that has reserved the whole GPU for its own pools,
or that must not allocate while serving).  It uses a fixed array inside the
library instead of a caller-provided workspace.  This file is collected last
so that a run stopping at the first failure has already run every other test;
it passes on its own in a fresh process and after the other tests."""
import numpy as np
import pytest

import quantized_kv_cache_16_b200 as K
import workloads as W
from _cases import TOL_MAX_ABS, TOL_REL_L2, attn_errors, build_pair

pytestmark = pytest.mark.gpu


def test_static_decode_matches_workspace_decode_twice():
    import torch
    assert torch.cuda.is_available()
    wl = W.scaled(W.paged(), [1000, 37, 300])
    pair = build_pair(wl, oracle=False)
    c = pair.cache
    bt, ctx = pair.block_table(), pair.ctx()
    batch, max_pages = bt.shape
    for step in range(2):  # two calls in a row through the same static array
        q = torch.from_numpy(W.queries(wl, step)).cuda()
        want = c.decode(q, bt, ctx)
        got = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
        K.kvq_decode_attn_static(c.handle, q, bt, max_pages, ctx, batch, 0.0, got)
        torch.cuda.synchronize()
        assert c.sync_status() == K.KVQ_OK
        max_abs, rel = attn_errors(got.cpu().numpy(), want.cpu().numpy().astype(np.float64))
        assert max_abs <= TOL_MAX_ABS and rel <= TOL_REL_L2, f"max_abs={max_abs:.3e} rel={rel:.3e}"


def test_static_decode_refuses_a_workspace_over_its_limit():
    import torch
    wl = W.scaled(W.llama(), [64])
    pair = build_pair(wl, oracle=False)
    c = pair.cache
    q = torch.from_numpy(W.queries(wl, 0)).cuda()
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    batch = 4096  # a block table this wide needs far more than 4 MiB of splits
    bt = torch.zeros((batch, 64), dtype=torch.int32, device="cuda")
    assert K.kvq_decode_workspace_bytes(c.handle, batch, 64) > (4 << 20)
    with pytest.raises(K.KvqError) as e:
        K.kvq_decode_attn_static(c.handle, q, bt, 64, torch.zeros(batch, dtype=torch.int32, device="cuda"), batch,
                                 0.0, out)
    assert e.value.status == K.KVQ_ERR_CAPACITY
