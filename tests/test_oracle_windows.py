"""Pins for the oracle's decode with 16-bit sink and recent windows ["OSCAR",
2.2b: sink and recent tokens at full precision, the middle history low-bit]:
empty windows are the quantised decode, windows over every token are fp16
attention, and block-aligned windows equal the certified decode with those
blocks forced exact (a separate code path that reads slot-indexed rows, so
the window store's ring indexing is checked against it).  No GPU."""
import numpy as np
import pytest

import oracle as O
import workloads as W


def _case(T, B=1):
    wl = W.scaled(W.certified(), [T] * B if isinstance(T, int) else T)
    pages = W.page_table(wl)[0]
    cfg = O.make_config(wl.Hq, wl.Hkv, wl.d, wl.k_fmt, wl.v_fmt, wl.k_group, wl.v_group, num_pages=pages.num_pages,
                        bound_block_tokens=wl.bound_block)
    pool = O.new_pool(cfg)
    ks = np.zeros((cfg.num_pages * 16, wl.Hkv, wl.d), np.float16)
    vs = np.zeros_like(ks)
    kv = []
    for b in range(wl.B):
        k, v = W.prefix_kv(wl, b)
        sl = pages.slots(b, 0, wl.ctx[b])
        if len(sl):
            assert O.append(cfg, pool, k, v, sl) == 0
            ks[sl], vs[sl] = k, v
        kv.append((k, v))
    return wl, cfg, pool, pages, ks, vs, kv


def window_store(wl, kv, sink, recent):
    """The compact store: row t for t < sink, row sink + t % recent for the
    last `recent` tokens (older ring contents are whatever was there)."""
    W_ = sink + recent
    wk = np.zeros((wl.B, max(W_, 1), wl.Hkv, wl.d), np.float16)
    wv = np.zeros_like(wk)
    for b, (k, v) in enumerate(kv):
        T = wl.ctx[b]
        for t in range(min(sink, T)):
            wk[b, t], wv[b, t] = k[t], v[t]
        if recent:
            for t in range(max(0, T - recent), T):
                wk[b, sink + t % recent], wv[b, sink + t % recent] = k[t], v[t]
    return wk, wv


def test_empty_windows_are_the_quantised_decode():
    wl, cfg, pool, pages, ks, vs, kv = _case(700)
    q = W.queries(wl, 0)
    wk, wv = window_store(wl, kv, 0, 0)
    out = O.decode_windows(cfg, pool, wk, wv, 0, 0, q, pages.block_table, wl.ctx)
    assert np.allclose(out, O.decode(cfg, pool, q, pages.block_table, wl.ctx), rtol=0, atol=1e-12)


@pytest.mark.parametrize("sink,recent", [(1000, 0), (0, 1000), (300, 400), (128, 256)])
def test_windows_over_every_token_are_fp16_attention(sink, recent):
    wl, cfg, pool, pages, ks, vs, kv = _case([700, 333])
    q = W.queries(wl, 1)
    if sink + recent < 700:
        wl.ctx = [min(t, sink + recent) for t in wl.ctx]  # a context the windows cover
    wk, wv = window_store(wl, kv, sink, recent)
    out = O.decode_windows(cfg, pool, wk, wv, sink, recent, q, pages.block_table, wl.ctx)
    assert np.allclose(out, O.decode_fp16(cfg, ks, vs, q, pages.block_table, wl.ctx), rtol=0, atol=1e-10)


@pytest.mark.parametrize("T,sink,recent", [(1024, 128, 256), (1152, 256, 128), (1280, 128, 512), (1000, 128, 104)])
def test_block_aligned_windows_equal_the_forced_certified_decode(T, sink, recent):
    wl, cfg, pool, pages, ks, vs, kv = _case(T)
    q = W.queries(wl, 2)
    wk, wv = window_store(wl, kv, sink, recent)
    out = O.decode_windows(cfg, pool, wk, wv, sink, recent, q, pages.block_table, wl.ctx)
    nb = (T + 127) // 128
    # blocks whose every token lies in a window (T, sink and recent multiples of 128 at the ends)
    first = [b for b in range(nb) if (b + 1) * 128 <= sink]
    last = [b for b in range(nb) if b * 128 >= T - recent]
    blocks = sorted(set(first + last))
    covered = set()
    for b in blocks:
        covered.update(range(b * 128, min((b + 1) * 128, T)))
    exact_tokens = set(range(min(sink, T))) | set(range(max(0, T - recent), T))
    assert covered == exact_tokens  # the cases are block-aligned
    forced = np.full((1, wl.Hkv, len(blocks)), -1, np.int32)
    forced[0, :, :] = blocks
    want, _, _, _ = O.decode_certified(cfg, pool, ks, vs, q, pages.block_table, wl.ctx, 0.0, forced=forced)
    assert np.allclose(out, want, rtol=0, atol=1e-12)


def test_windows_help_and_empty_sequences_are_zero():
    wl, cfg, pool, pages, ks, vs, kv = _case([0, 900])
    q = W.queries(wl, 3)
    wk, wv = window_store(wl, kv, 64, 128)
    out = O.decode_windows(cfg, pool, wk, wv, 64, 128, q, pages.block_table, wl.ctx)
    assert np.all(out[0] == 0)
    exact = O.decode_fp16(cfg, ks, vs, q, pages.block_table, wl.ctx)
    quant = O.decode(cfg, pool, q, pages.block_table, wl.ctx)
    assert np.linalg.norm(out[1] - exact[1]) < np.linalg.norm(quant[1] - exact[1])
