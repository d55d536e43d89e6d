"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the
same seeded inputs.

  append  -> pool bytes (codes, scales, zeros, descriptors) bit-exact;
  dequant -> kvq_dequant_debug values equal fp32(oracle fp64 dequant), codes equal;
  decode  -> max |gpu - oracle| <= 2e-3 and rel-L2 <= 1e-3 against the
             oracle's fp64 attention over the same dequantised cache.

Sizes span several pages, several splits and a ragged tail; the full-size
workloads run in the launch configuration the benchmark uses.
"""
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


def _decode_check(pair, step=0, extra=0, softmax_scale=0.0):
    import torch
    wl = pair.wl
    q = W.queries(wl, step)
    out = pair.cache.decode(torch.from_numpy(q).cuda(), pair.block_table(), pair.ctx(extra),
                            softmax_scale=softmax_scale)
    got = out.float().cpu().numpy()
    ctx = [t + extra for t in wl.ctx]
    want = O.decode(pair.ocfg, pair.opool, q, pair.pages.block_table, ctx, scale=softmax_scale)
    max_abs, rel = attn_errors(got, want)
    assert max_abs <= TOL_MAX_ABS and rel <= TOL_REL_L2, f"max_abs={max_abs:.3e} rel={rel:.3e}"
    assert pair.cache.sync_status() == 0
    return got, want


SMALL = [
    ("tiny", W.tiny()),
    ("llama-1000", W.scaled(W.llama(), 1000)),
    ("llama-ragged", W.scaled(W.llama(), 17)),
    ("paged-B5", W.scaled(W.paged(), [37, 300, 16, 1, 513])),
    ("int8k-2000", W.scaled(W.certified(), 2000)),
    ("int2-B2", W.scaled(W.int2(), [3000, 777])),
]


@pytest.mark.parametrize("name,wl", SMALL, ids=[s[0] for s in SMALL])
def test_append_bytes_bit_exact(name, wl):
    pair = build_pair(wl)
    gpu = pair.cache.pool.cpu().numpy()
    assert gpu.shape == pair.opool.shape
    diff = np.nonzero(gpu[256:] != pair.opool[256:])[0]
    assert diff.size == 0, f"{diff.size} bytes differ, first at pool offset {256 + diff[0]}"


@pytest.mark.parametrize("name,wl", SMALL, ids=[s[0] for s in SMALL])
def test_dequant_debug_matches_oracle(name, wl):
    import torch
    pair = build_pair(wl)
    slots = np.concatenate([pair.pages.slots(b, 0, wl.ctx[b]) for b in range(wl.B)])
    pick = np.random.default_rng(0).choice(slots, size=min(200, len(slots)), replace=False).astype(np.int32)
    k, v, codes, meta = pair.cache.dequant(torch.from_numpy(pick).cuda())
    ko, vo = O.dequant(pair.ocfg, pair.opool, pick)
    assert np.array_equal(k.cpu().numpy(), ko.astype(np.float32))
    assert np.array_equal(v.cpu().numpy(), vo.astype(np.float32))
    codes = codes.cpu().numpy()
    for i, s in enumerate(pick[:20]):
        for kvh in range(wl.Hkv):
            for t in range(2):
                c, _, _ = O.read_row(pair.ocfg, pair.opool, int(s), kvh, t)
                fmt = wl.v_fmt if t else wl.k_fmt
                want = c.astype(np.int64) & (0xFF if fmt == O.INT8_SYM else 0xF if fmt == O.INT4_ASYM else 0x3)
                assert np.array_equal(codes[i, kvh, t].astype(np.int64), want)


@pytest.mark.parametrize("name,wl", SMALL, ids=[s[0] for s in SMALL])
def test_decode_matches_oracle(name, wl):
    pair = build_pair(wl)
    _decode_check(pair)


def test_decode_edge_lengths():
    """Empty context (zero output), one token, exactly one page, page + 1."""
    wl = W.scaled(W.llama(), [0, 1, 16, 17])
    pair = build_pair(wl)
    got, _ = _decode_check(pair)
    assert not got[0].any()


@pytest.mark.parametrize("hq,hkv", [(8, 8), (16, 8), (64, 8), (6, 2)])
def test_decode_gqa_group_sizes(hq, hkv):
    import dataclasses
    wl = dataclasses.replace(W.scaled(W.llama(), [700, 45]), Hq=hq, Hkv=hkv)
    _decode_check(build_pair(wl))


def test_decode_without_rotation_and_explicit_scale():
    wl = W.scaled(W.llama(), [900])
    pair = build_pair(wl, rotate=0)
    gpu = pair.cache.pool.cpu().numpy()
    assert np.array_equal(gpu[256:], pair.opool[256:])
    _decode_check(pair, softmax_scale=0.05)


def test_decode_steps_append_then_attend():
    """The decode step of the benchmark: append one token per sequence, then
    attend over the grown context, several steps in a row, with the workspace
    reused (its counters must come back to zero after every call)."""
    import torch
    wl = W.scaled(W.paged(), [100, 31, 260], steps=3)
    pair = build_pair(wl, extra_tokens=wl.steps)
    for step in range(wl.steps):
        k, v = W.step_kv(wl, step)
        slots = np.array([pair.pages.slot(b, wl.ctx[b] + step) for b in range(wl.B)], np.int32)
        pair.cache.append(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda(), torch.from_numpy(slots).cuda())
        assert O.append(pair.ocfg, pair.opool, k, v, slots) == 0
        got1, _ = _decode_check(pair, step=step, extra=step + 1)
        got2, _ = _decode_check(pair, step=step, extra=step + 1)
        assert np.array_equal(got1, got2)
    gpu = pair.cache.pool.cpu().numpy()
    assert np.array_equal(gpu[256:], pair.opool[256:])


FULL = [
    ("tiny-d64-T256", W.tiny),
    ("llama3-8b-layer-T32768", lambda: W.scaled(W.llama(), 32768)),
    ("paged-B16", W.paged),
    ("int8k-int4v-T131072", lambda: W.scaled(W.certified(), 131072)),
    ("int2-B4-T65536", W.int2),
]


@pytest.mark.parametrize("name,make", FULL, ids=[f[0] for f in FULL])
def test_full_size_workloads(name, make):
    """Full sizes: pool bytes bit-exact, every output row within tolerance."""
    wl = make()
    pair = build_pair(wl)
    gpu = pair.cache.pool.cpu().numpy()
    diff = np.nonzero(gpu[256:] != pair.opool[256:])[0]
    assert diff.size == 0, f"{diff.size} bytes differ, first at {256 + diff[0]}"
    _decode_check(pair)


STEP_CASES = [
    ("tiny", W.scaled(W.tiny(), [255])),
    ("llama-ragged", W.scaled(W.llama(), [1000, 31, 16])),
    ("int8k-descriptors", W.scaled(W.certified(), [700])),
    ("int2-B2", W.scaled(W.int2(), [301, 64])),
]


@pytest.mark.parametrize("name,wl", STEP_CASES, ids=[s[0] for s in STEP_CASES])
def test_decode_step_fuses_append_and_decode(name, wl):
    """kvq_decode_step stores exactly the bytes kvq_append stores and returns
    exactly what kvq_append followed by kvq_decode_attn returns."""
    import torch
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
        gpu = fused.cache.pool.cpu().numpy()
        assert np.array_equal(gpu[256:], fused.opool[256:])
        assert np.array_equal(out_f.cpu().numpy(), out_s.cpu().numpy())
        want = O.decode(fused.ocfg, fused.opool, W.queries(wl, step), fused.pages.block_table,
                        [t + step + 1 for t in wl.ctx])
        max_abs, rel = attn_errors(out_f.cpu().numpy(), want)
        assert max_abs <= TOL_MAX_ABS and rel <= TOL_REL_L2, f"max_abs={max_abs:.3e} rel={rel:.3e}"


def test_decode_step_rejects_a_slot_off_the_last_position():
    import torch
    wl = W.scaled(W.llama(), [40])
    pair = build_pair(wl, extra_tokens=1)
    before = pair.cache.pool.cpu().numpy().copy()
    k, v = W.step_kv(wl, 0)
    bad = np.array([pair.pages.slot(0, 3)], np.int32)  # not position 40
    pair.cache.step(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda(), torch.from_numpy(bad).cuda(),
                    torch.from_numpy(W.queries(wl, 0)).cuda(), pair.block_table(), pair.ctx(1))
    assert pair.cache.sync_status() == 4  # KVQ_ERR_OUT_OF_RANGE
    assert np.array_equal(pair.cache.pool.cpu().numpy()[256:], before[256:])


def _host_record(cache, wl, step, slots, ctx):
    """The pinned host record of kvq_decode_step_host (q, k_new, v_new, slots,
    ctx lengths, sections 16-byte aligned)."""
    import torch
    import quantized_kv_cache_16_b200 as K
    k, v = W.step_kv(wl, step)
    q = W.queries(wl, step)
    up = lambda n: (n + 15) // 16 * 16
    parts = [q.view(np.uint8).ravel(), k.view(np.uint8).ravel(), v.view(np.uint8).ravel(),
             np.asarray(slots, np.int32).view(np.uint8), np.asarray(ctx, np.int32).view(np.uint8)]
    rec = np.zeros(K.kvq_step_record_bytes(cache.handle, wl.B), np.uint8)
    off = 0
    for a in parts:
        rec[off:off + a.size] = a
        off += up(a.size)
    assert off == rec.size
    return torch.from_numpy(rec).pin_memory()


def _record_of(cache, q, k, v, slots, ctx):
    """kvq_decode_step_host's pinned record of explicit arrays (sections
    16-byte aligned: q, k_new, v_new, slots, ctx lengths)."""
    import torch
    import quantized_kv_cache_16_b200 as K
    up = lambda n: (n + 15) // 16 * 16
    parts = [q.view(np.uint8).ravel(), k.view(np.uint8).ravel(), v.view(np.uint8).ravel(),
             np.asarray(slots, np.int32).view(np.uint8), np.asarray(ctx, np.int32).view(np.uint8)]
    rec = np.zeros(K.kvq_step_record_bytes(cache.handle, q.shape[0]), np.uint8)
    off = 0
    for a in parts:
        rec[off:off + a.size] = a
        off += up(a.size)
    assert off == rec.size
    return torch.from_numpy(rec).pin_memory()


def test_decode_step_host_back_to_back():
    """Six kvq_decode_step_host calls issued with no synchronisation between
    them, each with its own pinned record and output: the record copy of a
    step runs on the library's copy stream while the previous step's kernel
    may still read the other buffer half.  In mid-run the device record
    buffer changes (step 2) and so does the batch, hence the record size
    (step 4): both must wait for the two halves still in use.  After one
    synchronisation every step's output and the final pool bytes equal those
    of kvq_decode_step run one step at a time on device copies."""
    import torch
    import quantized_kv_cache_16_b200 as K
    wl = W.scaled(W.llama(), [700, 45, 16])
    host = build_pair(wl, extra_tokens=8, oracle=False)
    devp = build_pair(wl, extra_tokens=8, oracle=False)
    P = host.pages.block_table.shape[1]
    ws = host.cache.workspace_for(wl.B, P)
    d_recs = [torch.empty(2 * K.kvq_step_record_bytes(host.cache.handle, wl.B), dtype=torch.uint8, device="cuda")
              for _ in range(2)]
    plan = [(0, 3), (0, 3), (1, 3), (1, 3), (1, 2), (1, 2)]  # (device record buffer, batch) of each step
    pos = list(wl.ctx)
    rng = np.random.default_rng(11)
    bt_h = host.block_table()
    steps = []
    for step, (buf, B) in enumerate(plan):
        q = rng.standard_normal((B, wl.Hq, wl.d)).astype(np.float16)
        k = rng.standard_normal((B, wl.Hkv, wl.d)).astype(np.float16)
        v = (0.5 * rng.standard_normal((B, wl.Hkv, wl.d))).astype(np.float16)
        slots = np.array([host.pages.slot(b, pos[b]) for b in range(B)], np.int32)
        ctx = np.array([pos[b] + 1 for b in range(B)], np.int32)
        for b in range(B):
            pos[b] += 1
        h_in = _record_of(host.cache, q, k, v, slots, ctx)
        h_out = torch.full((B, wl.Hq, wl.d), float("nan"), dtype=torch.float32).pin_memory()
        K.kvq_decode_step_host(host.cache.handle, h_in, d_recs[buf], bt_h[:B], P, B, 0.0, ws, ws.numel(), h_out)
        steps.append((q, k, v, slots, ctx, B, h_in, h_out))
    torch.cuda.synchronize()
    bt_d = devp.block_table()
    for step, (q, k, v, slots, ctx, B, _, h_out) in enumerate(steps):
        want = devp.cache.step(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda(), torch.from_numpy(slots).cuda(),
                               torch.from_numpy(q).cuda(), bt_d[:B], torch.from_numpy(ctx).cuda())
        torch.cuda.synchronize()
        assert np.array_equal(h_out.numpy(), want.cpu().numpy()), f"step {step}"
    assert np.array_equal(host.cache.pool.cpu().numpy()[256:], devp.cache.pool.cpu().numpy()[256:])
    assert host.cache.sync_status() == 0 and devp.cache.sync_status() == 0


def test_decode_step_host_many_steps_unsynchronised():
    """Forty kvq_decode_step_host calls in one layout with no
    synchronisation between them: the record copies and the kernels meet
    only through the library's ready and consumed flags, so the copy of step
    n must wait for the kernel of step n - 1 to start (its half's last reader
    done) whether or not the host already sees the mark.  Every step's output
    and the final pool bytes equal those of kvq_decode_step run one step at
    a time on device copies."""
    import torch
    import quantized_kv_cache_16_b200 as K
    n_steps = 40
    wl = W.scaled(W.llama(), [900, 60, 17])
    host = build_pair(wl, extra_tokens=n_steps, oracle=False)
    devp = build_pair(wl, extra_tokens=n_steps, oracle=False)
    P = host.pages.block_table.shape[1]
    ws = host.cache.workspace_for(wl.B, P)
    d_rec = torch.empty(2 * K.kvq_step_record_bytes(host.cache.handle, wl.B), dtype=torch.uint8, device="cuda")
    pos = list(wl.ctx)
    rng = np.random.default_rng(12)
    bt_h = host.block_table()
    steps = []
    for step in range(n_steps):
        q = rng.standard_normal((wl.B, wl.Hq, wl.d)).astype(np.float16)
        k = rng.standard_normal((wl.B, wl.Hkv, wl.d)).astype(np.float16)
        v = (0.5 * rng.standard_normal((wl.B, wl.Hkv, wl.d))).astype(np.float16)
        slots = np.array([host.pages.slot(b, pos[b]) for b in range(wl.B)], np.int32)
        ctx = np.array([pos[b] + 1 for b in range(wl.B)], np.int32)
        for b in range(wl.B):
            pos[b] += 1
        h_in = _record_of(host.cache, q, k, v, slots, ctx)
        h_out = torch.full((wl.B, wl.Hq, wl.d), float("nan"), dtype=torch.float32).pin_memory()
        K.kvq_decode_step_host(host.cache.handle, h_in, d_rec, bt_h, P, wl.B, 0.0, ws, ws.numel(), h_out)
        steps.append((q, k, v, slots, ctx, h_in, h_out))
    torch.cuda.synchronize()
    bt_d = devp.block_table()
    for step, (q, k, v, slots, ctx, _, h_out) in enumerate(steps):
        want = devp.cache.step(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda(), torch.from_numpy(slots).cuda(),
                               torch.from_numpy(q).cuda(), bt_d, torch.from_numpy(ctx).cuda())
        torch.cuda.synchronize()
        assert np.array_equal(h_out.numpy(), want.cpu().numpy()), f"step {step}"
    assert np.array_equal(host.cache.pool.cpu().numpy()[256:], devp.cache.pool.cpu().numpy()[256:])
    assert host.cache.sync_status() == 0 and devp.cache.sync_status() == 0


def test_decode_step_host_equals_the_device_step():
    """kvq_decode_step_host (the pinned host record copied in on the
    library's copy stream into alternating buffers, the kernel writing the
    pinned host output through its device mapping) stores the same bytes and
    returns the same output as kvq_decode_step on device copies of the same
    inputs, over steps that use both buffers; pageable host memory is
    refused."""
    import torch
    import quantized_kv_cache_16_b200 as K
    wl = W.scaled(W.llama(), [1000, 31, 16])
    host = build_pair(wl, extra_tokens=3, oracle=False)
    devp = build_pair(wl, extra_tokens=3, oracle=False)
    ws = host.cache.workspace_for(wl.B, host.pages.block_table.shape[1])
    h_out = torch.empty((wl.B, wl.Hq, wl.d), dtype=torch.float32).pin_memory()
    d_rec = torch.empty(2 * K.kvq_step_record_bytes(host.cache.handle, wl.B), dtype=torch.uint8, device="cuda")
    for step in range(3):
        slots = np.array([host.pages.slot(b, wl.ctx[b] + step) for b in range(wl.B)], np.int32)
        ctx = [t + step + 1 for t in wl.ctx]
        h_in = _host_record(host.cache, wl, step, slots, ctx)
        K.kvq_decode_step_host(host.cache.handle, h_in, d_rec, host.block_table(), host.pages.block_table.shape[1],
                               wl.B, 0.0, ws, ws.numel(), h_out)
        torch.cuda.synchronize()
        k, v = W.step_kv(wl, step)
        want = devp.cache.step(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda(),
                               torch.from_numpy(slots).cuda(), torch.from_numpy(W.queries(wl, step)).cuda(),
                               devp.block_table(), devp.ctx(step + 1))
        assert np.array_equal(h_out.numpy(), want.cpu().numpy())
        assert np.array_equal(host.cache.pool.cpu().numpy()[256:], devp.cache.pool.cpu().numpy()[256:])
    assert host.cache.sync_status() == 0
    pageable = torch.zeros_like(h_out)
    with pytest.raises(K.KvqError) as e:
        K.kvq_decode_step_host(host.cache.handle, h_in, d_rec, host.block_table(), host.pages.block_table.shape[1],
                               wl.B, 0.0, ws, ws.numel(), pageable)
    assert e.value.status == K.KVQ_ERR_INVALID_ARG
