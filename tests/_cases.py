"""Shared set-up for the GPU parity tests: build the same cache twice, once
through the C ABI on the GPU and once with the CPU oracle, from one seeded
workload.  Inputs come only from `workloads`; expected values only from
`oracle`."""
from __future__ import annotations

import dataclasses

import numpy as np

import oracle as O
import workloads as W

TOL_MAX_ABS = 2e-3  # attention vs the oracle's fp64 attention (same dequantised cache)
TOL_REL_L2 = 1e-3


def configs(wl: W.Workload, num_pages: int, rotate=None):
    rotate = wl.rotate if rotate is None else rotate
    import quantized_kv_cache_16_b200 as K
    kw = dict(num_q_heads=wl.Hq, num_kv_heads=wl.Hkv, head_dim=wl.d, k_fmt=wl.k_fmt, v_fmt=wl.v_fmt,
              k_group=wl.k_group, v_group=wl.v_group, clip_ratio=wl.clip, rotation_seed=wl.rotation_seed,
              rotate=rotate, num_pages=num_pages, bound_block_tokens=wl.bound_block, scale_search=wl.scale_search)
    return K.make_config(**kw), O.make_config(**kw)


@dataclasses.dataclass
class Pair:
    wl: W.Workload
    pages: W.Pages
    cache: object  # quantized_kv_cache_16_b200.Cache
    ocfg: O.Config
    opool: np.ndarray
    kv: list  # per-sequence fp16 prefix (k, v)

    def block_table(self):
        import torch
        return torch.from_numpy(self.pages.block_table).cuda()

    def ctx(self, extra=0):
        import torch
        return torch.tensor([t + extra for t in self.wl.ctx], dtype=torch.int32, device="cuda")


def build_pair(wl: W.Workload, extra_tokens: int = 0, rotate=None, oracle: bool = True, kv_rows=None) -> Pair:
    import torch
    import quantized_kv_cache_16_b200 as K
    pages = W.page_table(wl, extra_tokens=extra_tokens)[0]
    kcfg, ocfg = configs(wl, pages.num_pages, rotate)
    cache = K.Cache(kcfg)
    opool = O.new_pool(ocfg) if oracle else None
    kv = []
    for b in range(wl.B):
        k, v = W.prefix_kv(wl, b) if kv_rows is None else kv_rows[b]
        slots = pages.slots(b, 0, wl.ctx[b])
        if len(slots):
            cache.append(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda(), torch.from_numpy(slots).cuda())
            if oracle:
                assert O.append(ocfg, opool, k, v, slots) == 0
        kv.append((k, v))
    torch.cuda.synchronize()
    return Pair(wl, pages, cache, ocfg, opool, kv)


def attn_errors(got: np.ndarray, want: np.ndarray):
    err = got.astype(np.float64) - want
    max_abs = float(np.max(np.abs(err))) if err.size else 0.0
    den = float(np.linalg.norm(want))
    rel = float(np.linalg.norm(err)) / den if den > 0 else float(np.linalg.norm(err))
    return max_abs, rel
