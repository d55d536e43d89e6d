"""Seeded synthetic inputs shaped like the pages' long-context workloads.

This module holds none of the method's arithmetic: it only draws random fp16
K/V rows and queries, picks context lengths, and lays out shuffled 16-token
page tables.  Both the CUDA path (tests, bench) and the CPU oracle consume the
arrays it returns.  The pages measure on models and datasets that are not
available here; these recipes stand in for them (Llama-3-8B head geometry,
32K-128K contexts, outlier channels that the rotation is meant to spread).

Recipes (numpy ``default_rng``; every stream is keyed by (seed, stream id)):
  tiny        B=1, Hq=8, Hkv=2, d=64, T=256; K,V ~ N(0,1) with 2 outlier
              channels per kv head (x20) in both K and V; int4 g32 K and V.
  llama       B=1, Hq=32, Hkv=8, d=128, T=32768; K ~ N(0,1) with 4 fixed
              outlier channels per kv head (x15); V ~ N(0, 0.5^2); int4 g32.
  paged       B=16, 32/8, d=128, T_b ~ U[1024, 8192]; llama's distributions;
              int4 g32; pages shuffled in the block table.
  certified   B=1, 32/8, d=128, T=131072; llama's distributions; K int8
              symmetric per token-head, V int4 g32; 128-token bound blocks;
              top 1% of blocks promoted from the fp16 copy.
  ladder      certified's geometry and formats with concentrated attention
              (a stand-in for the needle-retrieval workloads the pages
              measure): llama's K/V, plus per kv head a seeded unit direction
              u; the keys of "hot" tokens -- the first 16 (sink), six needle
              spans of 64 tokens at seeded positions, the last 128 -- get
              a*u added with a ~ U[10, 14] (then rounded to fp16); queries are
              N(0,1) + 14*u of their kv head.
  hqmq        llama's geometry, distributions and context with the HQMQ codec
              for K and V.
  nvfp4       llama's geometry, distributions and context, rotated, NVFP4 K and
              V with ScaleSearch on the E4M3 scales.
  int2        prefill of 65536 tokens x 8 kv heads x d=128 per sequence, K and
              V ~ Laplace(0,1) with 1% of elements x30; 2-bit g128, clip 0.9;
              decode B=4, Hq=32, T=65536 (four independent prefills).
  q           ~ N(0,1), drawn anew for every step (ladder: plus its pull).
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field

import numpy as np

INT4_ASYM, INT8_SYM, INT2_ASYM, HQMQ_FMT, NVFP4_FMT = 0, 1, 2, 3, 4
PAGE_TOKENS = 16

# stream ids
_S_K, _S_V, _S_Q, _S_LEN, _S_PERM, _S_OUT, _S_NEWK, _S_NEWV, _S_DIR, _S_HOT = range(10)

NEEDLES, NEEDLE_LEN, SINK_LEN, RECENT_LEN, QUERY_PULL = 6, 64, 16, 128, 14.0


@dataclass
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    ctx: list  # per-sequence prefix length
    k_fmt: int = INT4_ASYM
    v_fmt: int = INT4_ASYM
    k_group: int = 32
    v_group: int = 32
    clip: float = 1.0
    bound_block: int = 0
    promote_frac: float = 0.0
    scale_search: int = 0  # 1: the codec searches each scale (ScaleSearch)
    dist: str = "llama"  # tiny | llama | laplace | needle
    seed: int = 0
    rotation_seed: int = 0x5EED
    steps: int = 1  # decode steps (each appends one token per sequence first)
    rotate: int = 1  # 1: sign + Hadamard rotation before coding; 0: the raw rows
    description: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def g(self) -> int:
        return self.Hq // self.Hkv


def tiny() -> Workload:
    return Workload("tiny-d64-T256", 1, 8, 2, 64, [256], dist="tiny", seed=0, steps=1,
                    description="batch 1, 8/2 heads, head_dim 64, context 256, int4 g32, one decode step")


def llama(T: int = 32768, steps: int = 100) -> Workload:
    return Workload(f"llama3-8b-layer-T{T}", 1, 32, 8, 128, [T], dist="llama", seed=1, steps=steps,
                    description="batch 1, 32/8 heads, head_dim 128, int4 g32 K and V, rotated; each step "
                                "appends 1 token then decodes")


def paged(B: int = 16, lo: int = 1024, hi: int = 8192, seed: int = 2) -> Workload:
    rng = np.random.default_rng([seed, _S_LEN])
    ctx = [int(t) for t in rng.integers(lo, hi + 1, size=B)]
    return Workload(f"paged-B{B}-U[{lo},{hi}]", B, 32, 8, 128, ctx, dist="llama", seed=seed, steps=1,
                    description="batch 16, 32/8 heads, head_dim 128, lengths uniform in [1024,8192], shuffled "
                                "16-token pages, int4 g32; append 1 token per sequence then decode")


def certified(T: int = 131072) -> Workload:
    return Workload(f"int8k-int4v-certified-T{T}", 1, 32, 8, 128, [T], k_fmt=INT8_SYM, k_group=128,
                    bound_block=128, promote_frac=0.01, dist="llama", seed=3, steps=1,
                    description="batch 1, 32/8 heads, head_dim 128, K int8 symmetric per token-head, V int4 g32, "
                                "128-token bound blocks, top 1% promoted from pinned fp16")


def ladder(T: int = 131072) -> Workload:
    return Workload(f"int8k-int4v-ladder-T{T}", 1, 32, 8, 128, [T], k_fmt=INT8_SYM, k_group=128,
                    bound_block=128, dist="needle", seed=5, steps=1,
                    description="batch 1, 32/8 heads, head_dim 128, K int8 symmetric per token-head, V int4 g32, "
                                "128-token bound blocks, attention concentrated on a sink, six needles and the "
                                "recent window; adaptive certified ladder over pinned fp16")


def hqmq(T: int = 32768) -> Workload:
    return Workload(f"hqmq-llama3-8b-layer-T{T}", 1, 32, 8, 128, [T], k_fmt=HQMQ_FMT, v_fmt=HQMQ_FMT, k_group=4,
                    v_group=4, dist="llama", seed=6, steps=1, rotate=0,
                    description="batch 1, 32/8 heads, head_dim 128, llama's K/V (outlier key channels x15), HQMQ K "
                                "and V of the raw rows (4-element quaternion blocks, 24 x 1024 codewords, 5-bit "
                                "radii, Med3x fp16 outliers)")


def nvfp4(T: int = 32768, search: int = 1) -> Workload:
    return Workload(f"nvfp4-llama3-8b-layer-T{T}", 1, 32, 8, 128, [T], k_fmt=NVFP4_FMT, v_fmt=NVFP4_FMT, k_group=16,
                    v_group=16, dist="llama", seed=7, steps=1, scale_search=search,
                    description="batch 1, 32/8 heads, head_dim 128, llama's K/V, rotated, NVFP4 K and V (e2m1 codes, "
                                "an E4M3 scale per 16 elements, ScaleSearch on the scales)")


def int2(B: int = 4, T: int = 65536) -> Workload:
    return Workload(f"int2-g128-clip0.9-B{B}-T{T}", B, 32, 8, 128, [T] * B, k_fmt=INT2_ASYM, v_fmt=INT2_ASYM,
                    k_group=128, v_group=128, clip=0.9, dist="laplace", seed=4, steps=1,
                    description="prefill 65536 x 8 x 128 Laplace(0,1) with 1% outliers x30 per sequence, 2-bit "
                                "g128 clip 0.9; decode batch 4, 32 q heads, context 65536")


ALL = {"tiny": tiny, "llama": llama, "paged": paged, "certified": certified, "ladder": ladder, "int2": int2,
       "hqmq": hqmq, "nvfp4": nvfp4}


def scaled(wl: Workload, ctx, steps: int = 1) -> Workload:
    """Same recipe with other context lengths (for parity runs the oracle
    finishes in seconds)."""
    ctx = list(ctx) if not isinstance(ctx, int) else [ctx] * wl.B
    return dataclasses.replace(wl, ctx=ctx, B=len(ctx), steps=steps, name=f"{wl.name}@{ctx[:4]}")


# --- random draws -------------------------------------------------------------

def _outlier_channels(wl: Workload, n: int) -> np.ndarray:
    rng = np.random.default_rng([wl.seed, _S_OUT])
    return np.stack([rng.choice(wl.d, size=n, replace=False) for _ in range(wl.Hkv)])  # [Hkv, n]


def _rows(wl: Workload, b: int, stream: int, n: int, t0: int, tensor: int) -> np.ndarray:
    """n token rows [n, Hkv, d] fp16 of tensor (0 = K, 1 = V) for sequence b,
    starting at token t0.  Draws are keyed by (seed, stream, b, t0) so the
    prefix and the appended tokens are independent streams."""
    rng = np.random.default_rng([wl.seed, stream, b, t0])
    shape = (n, wl.Hkv, wl.d)
    if wl.dist == "laplace":
        x = rng.laplace(0.0, 1.0, size=shape)
        mask = rng.random(size=shape) < 0.01
        x[mask] *= 30.0
    elif wl.dist == "tiny":
        x = rng.standard_normal(size=shape)
        ch = _outlier_channels(wl, 2)
        for h in range(wl.Hkv):
            x[:, h, ch[h]] *= 20.0
    else:  # llama (and the needle recipe's base rows)
        if tensor == 0:
            x = rng.standard_normal(size=shape)
            ch = _outlier_channels(wl, 4)
            for h in range(wl.Hkv):
                x[:, h, ch[h]] *= 15.0
        else:
            x = rng.normal(0.0, 0.5, size=shape)
    return x.astype(np.float16)


def needle_directions(wl: Workload) -> np.ndarray:
    """Unit directions u [Hkv, d] (float64) of the needle recipe."""
    rng = np.random.default_rng([wl.seed, _S_DIR])
    u = rng.standard_normal(size=(wl.Hkv, wl.d))
    return u / np.linalg.norm(u, axis=1, keepdims=True)


def hot_tokens(wl: Workload, b: int):
    """(positions int64 [n], amplitudes float64 [n]) of sequence b's hot
    tokens in the needle recipe: sink, needle spans, recent window (clipped to
    the prefix; overlaps keep one entry)."""
    T = wl.ctx[b]
    rng = np.random.default_rng([wl.seed, _S_HOT, b])
    starts = rng.integers(0, max(1, T - NEEDLE_LEN), size=NEEDLES)
    pos = [np.arange(0, min(SINK_LEN, T)), np.arange(max(0, T - RECENT_LEN), T)]
    pos += [np.arange(s, min(s + NEEDLE_LEN, T)) for s in starts]
    pos = np.unique(np.concatenate(pos)).astype(np.int64)
    amp = rng.uniform(10.0, 14.0, size=pos.shape[0])
    return pos, amp


def prefix_kv(wl: Workload, b: int):
    """fp16 K, V [ctx_b, Hkv, d] of sequence b's prefix."""
    T = wl.ctx[b]
    k, v = _rows(wl, b, _S_K, T, 0, 0), _rows(wl, b, _S_V, T, 0, 1)
    if wl.dist == "needle" and T > 0:
        pos, amp = hot_tokens(wl, b)
        u = needle_directions(wl)
        k[pos] = (k[pos].astype(np.float64) + amp[:, None, None] * u[None]).astype(np.float16)
    return k, v


def step_kv(wl: Workload, step: int):
    """fp16 K, V [B, Hkv, d]: the token each sequence appends at `step`."""
    k = np.stack([_rows(wl, b, _S_NEWK, 1, wl.ctx[b] + step, 0)[0] for b in range(wl.B)])
    v = np.stack([_rows(wl, b, _S_NEWV, 1, wl.ctx[b] + step, 1)[0] for b in range(wl.B)])
    return k, v


def queries(wl: Workload, step: int) -> np.ndarray:
    rng = np.random.default_rng([wl.seed, _S_Q, step])
    q = rng.standard_normal(size=(wl.B, wl.Hq, wl.d))
    if wl.dist == "needle":
        q = q + QUERY_PULL * np.repeat(needle_directions(wl), wl.g, axis=0)[None]
    return q.astype(np.float16)


# --- page tables --------------------------------------------------------------

@dataclass
class Pages:
    num_pages: int
    block_table: np.ndarray  # int32 [B, max_pages]
    capacity: list  # tokens each sequence may hold

    def slot(self, b: int, t: int) -> int:
        return int(self.block_table[b, t // PAGE_TOKENS]) * PAGE_TOKENS + t % PAGE_TOKENS

    def slots(self, b: int, t0: int, t1: int) -> np.ndarray:
        t = np.arange(t0, t1)
        return (self.block_table[b, t // PAGE_TOKENS] * PAGE_TOKENS + t % PAGE_TOKENS).astype(np.int32)


def page_table(wl: Workload, extra_tokens: int = 0, copies: int = 1, shuffle: bool = True,
               spare_pages: int = 0) -> list:
    """Shuffled 16-token page tables for `copies` independent caches of the
    workload inside one pool: returns [Pages] (one per copy), all sharing one
    num_pages.  Every sequence gets room for ctx_b + extra_tokens tokens."""
    need = [(t + extra_tokens + PAGE_TOKENS - 1) // PAGE_TOKENS for t in wl.ctx]
    per_copy = sum(need)
    total = per_copy * copies + spare_pages
    rng = np.random.default_rng([wl.seed, _S_PERM])
    perm = rng.permutation(total).astype(np.int32) if shuffle else np.arange(total, dtype=np.int32)
    max_pages = max(need) if need else 1
    out = []
    pos = 0
    for _ in range(copies):
        bt = np.zeros((wl.B, max_pages), np.int32)
        for b, n in enumerate(need):
            bt[b, :n] = perm[pos:pos + n]
            pos += n
        out.append(Pages(total, bt, [n * PAGE_TOKENS for n in need]))
    return out


# --- device-side draws for timing runs --------------------------------------

def prefix_kv_device(wl: Workload, b: int, device):
    """fp16 K, V [ctx_b, Hkv, d] of sequence b drawn on the device with the
    same recipe as prefix_kv (same distributions and outlier channels, a
    torch generator instead of numpy's streams, so not the same numbers).
    For timing runs whose inputs are too large to draw on the host quickly;
    parity tests use prefix_kv."""
    import torch
    T = wl.ctx[b]
    shape = (T, wl.Hkv, wl.d)
    out = []
    for tensor, stream in ((0, _S_K), (1, _S_V)):
        gen = torch.Generator(device=device)
        gen.manual_seed((wl.seed * 1000003 + stream * 1009 + b) & 0x7FFFFFFFFFFFFFFF)
        if wl.dist == "laplace":
            u = torch.rand(shape, generator=gen, device=device, dtype=torch.float32) - 0.5
            x = -torch.sign(u) * torch.log1p(-2.0 * u.abs())
            mask = torch.rand(shape, generator=gen, device=device) < 0.01
            x = torch.where(mask, x * 30.0, x)
        elif wl.dist == "tiny" or tensor == 0:
            x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
            n, factor = (2, 20.0) if wl.dist == "tiny" else (4, 15.0)
            ch = torch.from_numpy(_outlier_channels(wl, n)).to(device)
            for h in range(wl.Hkv):
                x[:, h, ch[h]] *= factor
        else:
            x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * 0.5
        out.append(x.to(torch.float16))
    if wl.dist == "needle" and T > 0:
        pos, amp = hot_tokens(wl, b)
        u = torch.from_numpy(needle_directions(wl)).to(device)
        p = torch.from_numpy(pos).to(device)
        a = torch.from_numpy(amp).to(device)
        out[0][p] = (out[0][p].double() + a[:, None, None] * u[None]).to(torch.float16)
    return out[0], out[1]
