"""Thin Python binding over libkvq.so, the C ABI declared in include/kvq.h.

Every function here has the name of the C entry point it calls and only
marshals arguments (torch tensors -> device pointers, the current torch stream
-> cudaStream_t).  All arithmetic runs in the CUDA kernels of the library;
there is no CPU or PyTorch fallback: if the library is missing, loading fails
with an error that says how to build it.

PyTorch is used only for device memory and streams (see ``Cache``).
"""
from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkvq.so")

KVQ_OK, KVQ_ERR_INVALID_ARG, KVQ_ERR_UNSUPPORTED, KVQ_ERR_CAPACITY = 0, 1, 2, 3
KVQ_ERR_OUT_OF_RANGE, KVQ_ERR_CUDA, KVQ_ERR_TIMEOUT = 4, 5, 6
KVQ_INT4_ASYM, KVQ_INT8_SYM, KVQ_INT2_ASYM, KVQ_HQMQ, KVQ_NVFP4 = 0, 1, 2, 3, 4
PAGE_TOKENS = 16

# Every symbol include/kvq.h declares (checked by the ABI test).
EXPORTS = (
    "kvq_pool_bytes", "kvq_create_cache", "kvq_destroy_cache", "kvq_append", "kvq_reset_pages",
    "kvq_decode_workspace_bytes", "kvq_decode_attn", "kvq_decode_certified", "kvq_decode_windows",
    "kvq_decode_windows_workspace_bytes", "kvq_decode_step", "kvq_step_record_bytes", "kvq_decode_step_host",
    "kvq_decode_attn_static", "kvq_dequant_debug", "kvq_debug_expire_first_wait", "kvq_sync_status",
    "kvq_status_string",
)


class KvqError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {kvq_status_string(status)} (status {status})")
        self.status = status


class kvq_config(C.Structure):
    _fields_ = [
        ("num_q_heads", C.c_int32), ("num_kv_heads", C.c_int32), ("head_dim", C.c_int32),
        ("k_fmt", C.c_int32), ("v_fmt", C.c_int32), ("k_group", C.c_int32), ("v_group", C.c_int32),
        ("clip_ratio", C.c_float), ("rotation_seed", C.c_uint64), ("rotate", C.c_int32),
        ("page_tokens", C.c_int32), ("num_pages", C.c_int32), ("bound_block_tokens", C.c_int32),
        ("scale_search", C.c_int32),
    ]


class kvq_tier2(C.Structure):
    _fields_ = [("k_host", C.c_void_p), ("v_host", C.c_void_p), ("promote_frac", C.c_float)]


class kvq_ladder(C.Structure):
    _fields_ = [(n, C.c_float) for n in ("tau_cov", "max_frac", "key_tol", "v_tol", "rank_tol", "cert_tol",
                                          "layer_frac")]


class kvq_ladder_report(C.Structure):
    _fields_ = [("k_star", C.c_void_p), ("block_flags", C.c_void_p), ("flags_cols", C.c_int32),
                ("bound", C.c_void_p), ("status", C.c_void_p)]


KVQ_LADDER_EXPANDED, KVQ_LADDER_CAPPED, KVQ_LADDER_VALUES = 1, 2, 4
KVQ_LADDER_RANK_FAIL, KVQ_LADDER_BOUND_FAIL, KVQ_LADDER_HEAD_DENSE, KVQ_LADDER_LAYER_DENSE = 8, 16, 32, 64

_lib = None


def lib() -> C.CDLL:
    """Load libkvq.so (built by __graft_entry__.build() or
    ``python -m quantized_kv_cache_16_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: the CUDA library has not been built "
                              "(run `python -m quantized_kv_cache_16_b200.build`)")
        L = C.CDLL(LIB_PATH)
        P, i32, sz = C.c_void_p, C.c_int32, C.c_size_t
        cfgp = C.POINTER(kvq_config)
        sig = {
            "kvq_pool_bytes": (sz, [cfgp]),
            "kvq_create_cache": (i32, [cfgp, P, sz, C.POINTER(C.c_void_p)]),
            "kvq_destroy_cache": (i32, [P]),
            "kvq_append": (i32, [P, P, P, P, i32, P]),
            "kvq_reset_pages": (i32, [P, P, i32, P]),
            "kvq_decode_workspace_bytes": (sz, [P, i32, i32]),
            "kvq_decode_attn": (i32, [P, P, P, i32, P, i32, C.c_float, C.POINTER(kvq_tier2), P, sz, P, P, P]),
            "kvq_decode_certified": (i32, [P, P, P, i32, P, i32, C.c_float, P, P, C.POINTER(kvq_ladder), P, sz,
                                           P, C.POINTER(kvq_ladder_report), P]),
            "kvq_decode_windows": (i32, [P, P, P, i32, P, i32, C.c_float, P, P, i32, i32, P, sz, P, P]),
            "kvq_decode_windows_workspace_bytes": (sz, [P, i32, i32]),
            "kvq_decode_step": (i32, [P, P, P, P, P, P, i32, P, i32, C.c_float, P, sz, P, P]),
            "kvq_step_record_bytes": (sz, [P, i32]),
            "kvq_decode_step_host": (i32, [P, P, P, P, i32, i32, C.c_float, P, sz, P, P]),
            "kvq_decode_attn_static": (i32, [P, P, P, i32, P, i32, C.c_float, P, P]),
            "kvq_dequant_debug": (i32, [P, P, i32, P, P, P, P, P]),
            "kvq_debug_expire_first_wait": (i32, [P, i32]),
            "kvq_sync_status": (i32, [P]),
            "kvq_status_string": (C.c_char_p, [i32]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return C.c_void_p(x)
    return C.c_void_p(x.data_ptr())


def _stream(s):
    if s is None:
        import torch
        return C.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(s, int):
        return C.c_void_p(s)
    return C.c_void_p(s.cuda_stream)


def _check(fn, status):
    if status != KVQ_OK:
        raise KvqError(fn, status)


def make_config(num_q_heads, num_kv_heads, head_dim, k_fmt=KVQ_INT4_ASYM, v_fmt=KVQ_INT4_ASYM, k_group=32,
                v_group=32, clip_ratio=1.0, rotation_seed=0, rotate=1, num_pages=1, bound_block_tokens=0,
                scale_search=0):
    return kvq_config(num_q_heads, num_kv_heads, head_dim, k_fmt, v_fmt, k_group, v_group, clip_ratio,
                      rotation_seed, rotate, PAGE_TOKENS, num_pages, bound_block_tokens, scale_search)


# ------------------------------------------------------------ C entry points --

def kvq_pool_bytes(cfg: kvq_config) -> int:
    return int(lib().kvq_pool_bytes(C.byref(cfg)))


def kvq_create_cache(cfg: kvq_config, pool, pool_bytes: int | None = None) -> C.c_void_p:
    h = C.c_void_p()
    nbytes = pool.numel() * pool.element_size() if pool_bytes is None else pool_bytes
    _check("kvq_create_cache", lib().kvq_create_cache(C.byref(cfg), _ptr(pool), nbytes, C.byref(h)))
    return h


def kvq_destroy_cache(cache) -> None:
    _check("kvq_destroy_cache", lib().kvq_destroy_cache(cache))


def kvq_append(cache, k, v, slot_mapping, n_tok: int | None = None, stream=None) -> None:
    n = slot_mapping.shape[0] if n_tok is None else n_tok
    _check("kvq_append", lib().kvq_append(cache, _ptr(k), _ptr(v), _ptr(slot_mapping), n, _stream(stream)))


def kvq_reset_pages(cache, page_ids, n: int | None = None, stream=None) -> None:
    n = page_ids.shape[0] if n is None else n
    _check("kvq_reset_pages", lib().kvq_reset_pages(cache, _ptr(page_ids), n, _stream(stream)))


def kvq_decode_workspace_bytes(cache, batch: int, max_pages_per_seq: int) -> int:
    return int(lib().kvq_decode_workspace_bytes(cache, batch, max_pages_per_seq))


def kvq_decode_attn(cache, q, block_table, max_pages_per_seq: int, ctx_lens, batch: int, softmax_scale: float,
                    tier2, workspace, ws_bytes: int, out, promoted_out=None, stream=None) -> None:
    t2 = C.byref(tier2) if tier2 is not None else None
    _check("kvq_decode_attn",
           lib().kvq_decode_attn(cache, _ptr(q), _ptr(block_table), max_pages_per_seq, _ptr(ctx_lens), batch,
                                 softmax_scale, t2, _ptr(workspace), ws_bytes, _ptr(out), _ptr(promoted_out),
                                 _stream(stream)))


def kvq_decode_certified(cache, q, block_table, max_pages_per_seq: int, ctx_lens, batch: int,
                         softmax_scale: float, k_tier2, v_tier2, policy: kvq_ladder, workspace, ws_bytes: int, out,
                         report: kvq_ladder_report | None = None, stream=None) -> None:
    rep = C.byref(report) if report is not None else None
    _check("kvq_decode_certified",
           lib().kvq_decode_certified(cache, _ptr(q), _ptr(block_table), max_pages_per_seq, _ptr(ctx_lens), batch,
                                      softmax_scale, _ptr(k_tier2), _ptr(v_tier2), C.byref(policy), _ptr(workspace),
                                      ws_bytes, _ptr(out), rep, _stream(stream)))


def kvq_decode_windows_workspace_bytes(cache, batch: int, max_pages_per_seq: int) -> int:
    return int(lib().kvq_decode_windows_workspace_bytes(cache, batch, max_pages_per_seq))


def kvq_decode_windows(cache, q, block_table, max_pages_per_seq: int, ctx_lens, batch: int, softmax_scale: float,
                       k_win, v_win, sink: int, recent: int, workspace, ws_bytes: int, out, stream=None) -> None:
    _check("kvq_decode_windows",
           lib().kvq_decode_windows(cache, _ptr(q), _ptr(block_table), max_pages_per_seq, _ptr(ctx_lens), batch,
                                    softmax_scale, _ptr(k_win), _ptr(v_win), sink, recent, _ptr(workspace), ws_bytes,
                                    _ptr(out), _stream(stream)))


def kvq_decode_step(cache, k_new, v_new, slot_mapping, q, block_table, max_pages_per_seq: int, ctx_lens,
                    batch: int, softmax_scale: float, workspace, ws_bytes: int, out, stream=None) -> None:
    _check("kvq_decode_step",
           lib().kvq_decode_step(cache, _ptr(k_new), _ptr(v_new), _ptr(slot_mapping), _ptr(q), _ptr(block_table),
                                 max_pages_per_seq, _ptr(ctx_lens), batch, softmax_scale, _ptr(workspace), ws_bytes,
                                 _ptr(out), _stream(stream)))


def kvq_step_record_bytes(cache, batch: int) -> int:
    return int(lib().kvq_step_record_bytes(cache, batch))


def kvq_decode_step_host(cache, host_in, dev_rec, block_table, max_pages_per_seq: int, batch: int,
                         softmax_scale: float, workspace, ws_bytes: int, host_out, stream=None) -> None:
    """host_in / host_out: pinned host tensors (or addresses); the record
    layout is kvq_step_record_bytes' (q, k_new, v_new, slots, ctx_lens);
    dev_rec: a device buffer of that size."""
    _check("kvq_decode_step_host",
           lib().kvq_decode_step_host(cache, _ptr(host_in), _ptr(dev_rec), _ptr(block_table), max_pages_per_seq,
                                      batch, softmax_scale, _ptr(workspace), ws_bytes, _ptr(host_out),
                                      _stream(stream)))


def kvq_decode_attn_static(cache, q, block_table, max_pages_per_seq: int, ctx_lens, batch: int,
                           softmax_scale: float, out, stream=None) -> None:
    _check("kvq_decode_attn_static",
           lib().kvq_decode_attn_static(cache, _ptr(q), _ptr(block_table), max_pages_per_seq, _ptr(ctx_lens),
                                        batch, softmax_scale, _ptr(out), _stream(stream)))


def kvq_dequant_debug(cache, slots, n: int | None = None, k_out=None, v_out=None, codes_out=None, meta_out=None,
                      stream=None) -> None:
    n = slots.shape[0] if n is None else n
    _check("kvq_dequant_debug", lib().kvq_dequant_debug(cache, _ptr(slots), n, _ptr(k_out), _ptr(v_out),
                                                        _ptr(codes_out), _ptr(meta_out), _stream(stream)))


def kvq_debug_expire_first_wait(cache, on: int) -> None:
    _check("kvq_debug_expire_first_wait", lib().kvq_debug_expire_first_wait(cache, int(on)))


def kvq_sync_status(cache) -> int:
    return int(lib().kvq_sync_status(cache))


def kvq_status_string(status: int) -> str:
    return lib().kvq_status_string(status).decode()


# ------------------------------------------------- torch-owned device memory --

class Cache:
    """A cache whose pool is a torch uint8 tensor on the current CUDA device.

    Holds the pool, the handle and a decode workspace (grown on demand,
    zero-filled once, reused by later calls on the same stream).
    """

    def __init__(self, cfg: kvq_config, device=None):
        import torch
        self.cfg = cfg
        nbytes = kvq_pool_bytes(cfg)
        if nbytes == 0:
            raise KvqError("kvq_pool_bytes", KVQ_ERR_INVALID_ARG)
        self.pool = torch.empty(nbytes, dtype=torch.uint8, device=device or "cuda")
        self.handle = kvq_create_cache(cfg, self.pool)
        self.workspace = None

    def close(self):
        if self.handle is not None:
            kvq_destroy_cache(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def append(self, k, v, slot_mapping, stream=None):
        kvq_append(self.handle, k, v, slot_mapping, stream=stream)

    def workspace_for(self, batch: int, max_pages: int):
        import torch
        need = max(kvq_decode_workspace_bytes(self.handle, batch, max_pages),
                   kvq_decode_windows_workspace_bytes(self.handle, batch, max_pages))
        if self.workspace is None or self.workspace.numel() < need:
            self.workspace = torch.zeros(max(need, 256), dtype=torch.uint8, device=self.pool.device)
        return self.workspace

    def decode(self, q, block_table, ctx_lens, out=None, softmax_scale: float = 0.0, tier2=None,
               promoted_out=None, stream=None):
        import torch
        batch, max_pages = block_table.shape
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        ws = self.workspace_for(batch, max_pages)
        kvq_decode_attn(self.handle, q, block_table, max_pages, ctx_lens, batch, softmax_scale, tier2, ws,
                        ws.numel(), out, promoted_out, stream)
        return out

    def decode_certified(self, q, block_table, ctx_lens, k_tier2, v_tier2, promote_frac: float,
                         promoted_out=None, out=None, softmax_scale: float = 0.0, stream=None):
        """Certified decode: k_tier2 / v_tier2 are the exact fp16 rows
        [num_pages*16, Hkv, d] by slot, in pinned host memory (or on the
        device); promoted_out (optional) int32 [B, Hkv, kmax] on the device."""
        t2 = kvq_tier2(k_tier2.data_ptr(), v_tier2.data_ptr(), promote_frac)
        return self.decode(q, block_table, ctx_lens, out, softmax_scale, t2, promoted_out, stream)

    def decode_ladder(self, q, block_table, ctx_lens, k_tier2, v_tier2, tau_cov: float = 0.995,
                      max_frac: float = 1.0, key_tol: float = float("inf"), v_tol: float = float("inf"),
                      rank_tol: float = float("inf"), cert_tol: float = float("inf"), layer_frac: float = 1.0,
                      out=None, report: bool = False, softmax_scale: float = 0.0, stream=None):
        """Certified decode with the adaptive ladder (kvq_decode_certified).
        Returns out, or (out, dict of device tensors k_star [B,Hkv],
        flags [B,Hkv,nb], bound [B,Hq], status [B,Hq]) with report=True."""
        import torch
        batch, max_pages = block_table.shape
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        ws = self.workspace_for(batch, max_pages)
        pol = kvq_ladder(tau_cov, max_frac, key_tol, v_tol, rank_tol, cert_tol, layer_frac)
        rep, rd = None, None
        if report:
            blk = self.cfg.bound_block_tokens
            nb = max(1, (max_pages * PAGE_TOKENS + blk - 1) // blk)
            dev = q.device
            hkv, hq = self.cfg.num_kv_heads, self.cfg.num_q_heads
            rd = {"k_star": torch.full((batch, hkv), -1, dtype=torch.int32, device=dev),
                  "flags": torch.full((batch, hkv, nb), 255, dtype=torch.uint8, device=dev),
                  "bound": torch.full((batch, hq), -1.0, dtype=torch.float32, device=dev),
                  "status": torch.full((batch, hq), -1, dtype=torch.int32, device=dev)}
            rep = kvq_ladder_report(rd["k_star"].data_ptr(), rd["flags"].data_ptr(), nb, rd["bound"].data_ptr(),
                                    rd["status"].data_ptr())
        kvq_decode_certified(self.handle, q, block_table, max_pages, ctx_lens, batch, softmax_scale, k_tier2,
                             v_tier2, pol, ws, ws.numel(), out, rep, stream)
        return (out, rd) if report else out

    def decode_windows(self, q, block_table, ctx_lens, k_win, v_win, sink: int, recent: int, out=None,
                       softmax_scale: float = 0.0, stream=None):
        """Decode with each sequence's first `sink` and last `recent` tokens
        at fp16 from the window store k_win / v_win [B, sink + recent, Hkv, d]
        (row t for t < sink, row sink + t % recent for recent tokens)."""
        import torch
        batch, max_pages = block_table.shape
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        ws = self.workspace_for(batch, max_pages)
        kvq_decode_windows(self.handle, q, block_table, max_pages, ctx_lens, batch, softmax_scale, k_win, v_win, sink,
                           recent, ws, ws.numel(), out, stream)
        return out

    def step(self, k_new, v_new, slot_mapping, q, block_table, ctx_lens, out=None, softmax_scale: float = 0.0,
             stream=None):
        """Append one token per sequence and decode, in one launch."""
        import torch
        batch, max_pages = block_table.shape
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        ws = self.workspace_for(batch, max_pages)
        kvq_decode_step(self.handle, k_new, v_new, slot_mapping, q, block_table, max_pages, ctx_lens, batch,
                        softmax_scale, ws, ws.numel(), out, stream)
        return out

    def dequant(self, slots):
        import torch
        n = slots.shape[0]
        hkv, d = self.cfg.num_kv_heads, self.cfg.head_dim
        dev = self.pool.device
        k = torch.empty(n, hkv, d, dtype=torch.float32, device=dev)
        v = torch.empty_like(k)
        codes = torch.empty(n, hkv, 2, d, dtype=torch.uint8, device=dev)
        meta = torch.empty(n, hkv, 2, 8, dtype=torch.int16, device=dev)
        kvq_dequant_debug(self.handle, slots, n, k, v, codes, meta)
        return k, v, codes, meta

    def sync_status(self) -> int:
        return kvq_sync_status(self.handle)
