"""CPU oracle for the low-bit KV cache -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  The product path (``quantized_kv_cache_16_b200``)
never imports it, and this package never imports the product.

The arithmetic lives in ``kvq_oracle.c`` (plain C99, fp32 codec with every
operation rounded separately, fp64 attention).  This module only compiles that
file with gcc (``-O2 -ffp-contract=off``, no fast-math) and marshals numpy
arrays to it through ctypes.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvq_oracle.c")
_LIB = os.path.join(_HERE, "_liboracle.so")

INT4_ASYM, INT8_SYM, INT2_ASYM, HQMQ, NVFP4 = 0, 1, 2, 3, 4
HQMQ_NS, HQMQ_NO = 1024, 2
PAGE_TOKENS = 16


def build(force: bool = False) -> str:
    """Compile the oracle into oracle/_liboracle.so (if missing or stale)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(
            ["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
             "-Wall", "-o", tmp, _SRC, "-lm"],
            check=True,
        )
        os.replace(tmp, _LIB)
    return _LIB


class Config(C.Structure):
    """Mirror of the oracle's own config struct (field order matters)."""

    _fields_ = [
        ("num_q_heads", C.c_int32),
        ("num_kv_heads", C.c_int32),
        ("head_dim", C.c_int32),
        ("k_fmt", C.c_int32),
        ("v_fmt", C.c_int32),
        ("k_group", C.c_int32),
        ("v_group", C.c_int32),
        ("clip_ratio", C.c_float),
        ("rotation_seed", C.c_uint64),
        ("rotate", C.c_int32),
        ("page_tokens", C.c_int32),
        ("num_pages", C.c_int32),
        ("bound_block_tokens", C.c_int32),
        ("scale_search", C.c_int32),
    ]


class Ladder(C.Structure):
    """Mirror of the oracle's ladder policy."""

    _fields_ = [(n, C.c_double) for n in ("tau_cov", "max_frac", "key_tol", "v_tol", "rank_tol", "cert_tol",
                                           "layer_frac")]


class LadderOut(C.Structure):
    """Mirror of the oracle's ladder output pointers."""

    _fields_ = [("out", C.c_void_p), ("mixed", C.c_void_p), ("dense", C.c_void_p), ("err", C.c_void_p),
                ("bound", C.c_void_p), ("status", C.c_void_p), ("k_star", C.c_void_p), ("k_cov", C.c_void_p),
                ("k_key", C.c_void_p), ("flags", C.c_void_p), ("rscore", C.c_void_p), ("cov", C.c_void_p),
                ("ekey", C.c_void_p), ("max_blocks", C.c_int32), ("rank_margin", C.c_void_p)]


LADDER_EXPANDED, LADDER_CAPPED, LADDER_VALUES = 1, 2, 4
LADDER_RANK_FAIL, LADDER_BOUND_FAIL, LADDER_HEAD_DENSE, LADDER_LAYER_DENSE = 8, 16, 32, 64


def make_config(num_q_heads, num_kv_heads, head_dim, k_fmt=INT4_ASYM, v_fmt=INT4_ASYM, k_group=32, v_group=32,
                clip_ratio=1.0, rotation_seed=0, rotate=1, num_pages=1, bound_block_tokens=0,
                scale_search=0) -> Config:
    return Config(num_q_heads, num_kv_heads, head_dim, k_fmt, v_fmt, k_group, v_group, clip_ratio,
                  rotation_seed, rotate, PAGE_TOKENS, num_pages, bound_block_tokens, scale_search)


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = C.CDLL(build())
        P = C.c_void_p
        i32, u64, f64, sz = C.c_int32, C.c_uint64, C.c_double, C.c_size_t
        cfgp = C.POINTER(Config)
        sig = {
            "kvqo_h2f": (C.c_float, [C.c_uint16]),
            "kvqo_f2h_rn": (C.c_uint16, [C.c_float]),
            "kvqo_f2h_ru": (C.c_uint16, [C.c_float]),
            "kvqo_f2h_rn_n": (None, [P, P, sz]),
            "kvqo_f2h_ru_n": (None, [P, P, sz]),
            "kvqo_h2f_n": (None, [P, P, sz]),
            "kvqo_splitmix64_output": (u64, [u64, i32]),
            "kvqo_signs": (None, [u64, i32, P]),
            "kvqo_rot_scale_f32": (C.c_float, [i32]),
            "kvqo_rotate_f32": (None, [P, P, i32, i32, P]),
            "kvqo_rotate_f64": (None, [P, P, i32, i32, P]),
            "kvqo_inv_rotate_f64": (None, [P, P, i32, i32, P]),
            "kvqo_quantize_rows": (None, [i32, i32, C.c_float, P, i32, i32, P, P, P, P, P, i32]),
            "kvqo_config_ok": (i32, [cfgp]),
            "kvqo_page_bytes": (sz, [cfgp]),
            "kvqo_desc_offset": (sz, [cfgp]),
            "kvqo_pool_bytes": (sz, [cfgp]),
            "kvqo_read_row": (None, [cfgp, P, i32, i32, i32, P, P, P]),
            "kvqo_dequant_row": (None, [cfgp, P, i32, i32, i32, P]),
            "kvqo_append": (i32, [cfgp, P, P, P, P, i32, P]),
            "kvqo_dequant": (None, [cfgp, P, P, i32, P, P]),
            "kvqo_attend": (None, [P, P, P, i32, i32, f64, i32, P]),
            "kvqo_decode": (i32, [cfgp, P, P, P, i32, P, i32, f64, i32, P, P]),
            "kvqo_decode_fp16": (i32, [cfgp, P, P, P, P, i32, P, i32, f64, P, P]),
            "kvqo_promote_count": (i32, [f64, i32]),
            "kvqo_decode_certified": (i32, [cfgp, P, P, P, P, P, i32, P, i32, f64, f64, P, P, P, i32, P, i32, P, P]),
            "kvqo_init_pool": (None, [cfgp, P]),
            "kvqo_hqmq_table_offset": (sz, [cfgp]),
            "kvqo_hqmq_unit": (None, [i32, P]),
            "kvqo_hqmq_codebook": (None, [u64, i32, i32, P]),
            "kvqo_hqmq_quantize_rows": (None, [P, i32, i32, P, P, P, P, P]),
            "kvqo_hqmq_encode_dirs": (None, [P, i32, P, P]),
            "kvqo_hqmq_read_row": (None, [cfgp, P, i32, i32, i32, P, P, P, P]),
            "kvqo_e4m3_value": (f64, [C.c_uint8]),
            "kvqo_e4m3_rn_sat_n": (None, [P, P, sz]),
            "kvqo_e2m1_rn_n": (None, [P, P, sz]),
            "kvqo_nvfp4_quantize_rows": (None, [P, i32, i32, i32, P, P]),
            "kvqo_nvfp4_read_row": (None, [cfgp, P, i32, i32, i32, P, P]),
            "kvqo_decode_windows": (i32, [cfgp, P, P, P, i32, i32, P, P, i32, P, i32, f64, P]),
            "kvqo_decode_ladder": (i32, [cfgp, P, P, P, P, P, i32, P, i32, f64, C.POINTER(Ladder), P, P,
                                         C.POINTER(LadderOut)]),
            "kvqo_set_threads": (i32, [i32]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        L.kvqo_set_threads(1)  # one thread unless a caller asks for more
        _lib = L
    return _lib


def set_threads(n: int) -> int:
    """Threads of the decode's (sequence, kv head) loop (timing only: the
    results do not depend on it); returns the count in effect."""
    return int(lib().kvqo_set_threads(int(n)))


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# --- scalar / array primitives ------------------------------------------------

def f2h_rn(x) -> np.ndarray:
    x = _c(x, np.float32)
    h = np.empty(x.shape, np.uint16)
    lib().kvqo_f2h_rn_n(_p(x), _p(h), x.size)
    return h


def f2h_ru(x) -> np.ndarray:
    x = _c(x, np.float32)
    h = np.empty(x.shape, np.uint16)
    lib().kvqo_f2h_ru_n(_p(x), _p(h), x.size)
    return h


def h2f(h) -> np.ndarray:
    h = _c(h, np.uint16)
    x = np.empty(h.shape, np.float32)
    lib().kvqo_h2f_n(_p(h), _p(x), h.size)
    return x


def splitmix64_output(seed: int, index: int) -> int:
    return int(lib().kvqo_splitmix64_output(seed, index))


def signs(seed: int, d: int) -> np.ndarray:
    s = np.empty(d, np.float32)
    lib().kvqo_signs(seed, d, _p(s))
    return s


def rot_scale_f32(d: int) -> np.float32:
    return np.float32(lib().kvqo_rot_scale_f32(d))


def rotate_f32(x, seed: int, rotate: int = 1) -> np.ndarray:
    """fp32 codec rotation of rows x[..., d] (butterfly order of the codec)."""
    x = _c(x, np.float32)
    d = x.shape[-1]
    s = signs(seed, d)
    flat = x.reshape(-1, d)
    y = np.empty_like(flat)
    for r in range(flat.shape[0]):
        lib().kvqo_rotate_f32(_p(flat[r]), _p(s), d, rotate, _p(y[r]))
    return y.reshape(x.shape)


def _rot64(fn, x, seed, rotate):
    x = _c(x, np.float64)
    d = x.shape[-1]
    s = signs(seed, d)
    flat = x.reshape(-1, d)
    y = np.empty_like(flat)
    for r in range(flat.shape[0]):
        fn(_p(flat[r]), _p(s), d, rotate, _p(y[r]))
    return y.reshape(x.shape)


def rotate_f64(x, seed: int, rotate: int = 1) -> np.ndarray:
    return _rot64(lib().kvqo_rotate_f64, x, seed, rotate)


def inv_rotate_f64(x, seed: int, rotate: int = 1) -> np.ndarray:
    return _rot64(lib().kvqo_inv_rotate_f64, x, seed, rotate)


def quantize_rows(fmt: int, group: int, clip: float, y, search: int = 0):
    """Quantise rotated fp32 rows y[n, d]; returns codes, scales, zeros (fp16
    bits), max |y - yhat| and max |y| per row.  search=1: ScaleSearch."""
    y = _c(y, np.float32)
    n, d = y.shape
    ng = 1 if fmt == INT8_SYM else d // group
    code = np.empty((n, d), np.int16)
    sh = np.empty((n, ng), np.uint16)
    zh = np.empty((n, ng), np.uint16)
    em = np.empty(n, np.float32)
    am = np.empty(n, np.float32)
    lib().kvqo_quantize_rows(fmt, group, clip, _p(y), n, d, _p(code), _p(sh), _p(zh), _p(em), _p(am), search)
    return code, sh, zh, em, am


# --- cache-level entry points -------------------------------------------------

def pool_bytes(cfg: Config) -> int:
    return int(lib().kvqo_pool_bytes(C.byref(cfg)))


def page_bytes(cfg: Config) -> int:
    return int(lib().kvqo_page_bytes(C.byref(cfg)))


def desc_offset(cfg: Config) -> int:
    return int(lib().kvqo_desc_offset(C.byref(cfg)))


def config_ok(cfg: Config) -> bool:
    return bool(lib().kvqo_config_ok(C.byref(cfg)))


def new_pool(cfg: Config) -> np.ndarray:
    """A zeroed pool of the config's size (with the HQMQ codebooks written,
    as kvq_create_cache does)."""
    pool = np.zeros(pool_bytes(cfg), np.uint8)
    lib().kvqo_init_pool(C.byref(cfg), _p(pool))
    return pool


def append(cfg: Config, pool: np.ndarray, k, v, slot_mapping, want_rotated: bool = False):
    """Quantise-on-append of fp16 k, v [n_tok, Hkv, d] into the pool image."""
    k = _c(k, np.float16).view(np.uint16)
    v = _c(v, np.float16).view(np.uint16)
    slots = _c(slot_mapping, np.int32)
    n = slots.shape[0]
    y = np.empty((n, cfg.num_kv_heads, 2, cfg.head_dim), np.float32) if want_rotated else None
    rc = lib().kvqo_append(C.byref(cfg), _p(pool), _p(k), _p(v), _p(slots), n, _p(y))
    return (rc, y) if want_rotated else rc


def read_row(cfg: Config, pool: np.ndarray, slot: int, kvh: int, tensor: int):
    d = cfg.head_dim
    code = np.empty(d, np.int16)
    sh = np.empty(d, np.uint16)
    zh = np.empty(d, np.uint16)
    lib().kvqo_read_row(C.byref(cfg), _p(pool), slot, kvh, tensor, _p(code), _p(sh), _p(zh))
    fmt, grp = (cfg.v_fmt, cfg.v_group) if tensor else (cfg.k_fmt, cfg.k_group)
    ng = 1 if fmt == INT8_SYM else d // grp
    return code, sh[:ng].copy(), zh[:ng].copy()


def dequant(cfg: Config, pool: np.ndarray, slots):
    slots = _c(slots, np.int32)
    n = slots.shape[0]
    k = np.empty((n, cfg.num_kv_heads, cfg.head_dim), np.float64)
    v = np.empty_like(k)
    lib().kvqo_dequant(C.byref(cfg), _p(pool), _p(slots), n, _p(k), _p(v))
    return k, v


def attend(qr, K, V, scale: float, n_split: int = 1) -> np.ndarray:
    qr, K, V = _c(qr, np.float64), _c(K, np.float64), _c(V, np.float64)
    T, d = K.shape
    o = np.empty(d, np.float64)
    lib().kvqo_attend(_p(qr), _p(K), _p(V), T, d, scale, n_split, _p(o))
    return o


def decode(cfg: Config, pool: np.ndarray, q, block_table, ctx_lens, scale: float = 0.0, n_split: int = 1,
           sel=None) -> np.ndarray:
    q = _c(q, np.float16).view(np.uint16)
    bt = _c(block_table, np.int32)
    cl = _c(ctx_lens, np.int32)
    B = cl.shape[0]
    sel = None if sel is None else _c(sel, np.int32)
    out = np.zeros((B, cfg.num_q_heads, cfg.head_dim), np.float64)
    rc = lib().kvqo_decode(C.byref(cfg), _p(pool), _p(q), _p(bt), bt.shape[1], _p(cl), B, scale, n_split,
                           _p(sel), _p(out))
    if rc != 0:
        raise ValueError(f"oracle decode rejected its arguments (rc={rc})")
    return out


def decode_fp16(cfg: Config, k_slots, v_slots, q, block_table, ctx_lens, scale: float = 0.0, sel=None):
    k = _c(k_slots, np.float16).view(np.uint16)
    v = _c(v_slots, np.float16).view(np.uint16)
    q = _c(q, np.float16).view(np.uint16)
    bt = _c(block_table, np.int32)
    cl = _c(ctx_lens, np.int32)
    B = cl.shape[0]
    sel = None if sel is None else _c(sel, np.int32)
    out = np.zeros((B, cfg.num_q_heads, cfg.head_dim), np.float64)
    rc = lib().kvqo_decode_fp16(C.byref(cfg), _p(k), _p(v), _p(q), _p(bt), bt.shape[1], _p(cl), B, scale,
                                _p(sel), _p(out))
    if rc != 0:
        raise ValueError(f"oracle fp16 decode rejected its arguments (rc={rc})")
    return out


def promote_count(frac: float, n_blocks: int) -> int:
    return int(lib().kvqo_promote_count(frac, n_blocks))


def decode_certified(cfg: Config, pool: np.ndarray, k_slots, v_slots, q, block_table, ctx_lens, frac: float,
                     scale: float = 0.0, sel=None, forced=None):
    """Returns (out [B,Hq,d], promoted [B,Hkv,kmax], scores [B,Hkv,nblk_max],
    bound_sums [B,Hq]).  forced [B,Hkv,kmax] (-1 padded): promote exactly
    these blocks instead of the top scores."""
    k = _c(k_slots, np.float16).view(np.uint16)
    v = _c(v_slots, np.float16).view(np.uint16)
    q = _c(q, np.float16).view(np.uint16)
    bt = _c(block_table, np.int32)
    cl = _c(ctx_lens, np.int32)
    B = cl.shape[0]
    blk = cfg.bound_block_tokens
    nbmax = max(1, int((int(cl.max()) + blk - 1) // blk)) if B else 1
    kmax = max(1, promote_count(frac, nbmax))
    sel = None if sel is None else _c(sel, np.int32)
    if forced is not None:
        forced = _c(forced, np.int32)
        kmax = forced.shape[2]
        assert forced.shape == (B, cfg.num_kv_heads, kmax)
    out = np.zeros((B, cfg.num_q_heads, cfg.head_dim), np.float64)
    prom = np.full((B, cfg.num_kv_heads, kmax), -1, np.int32)
    scores = np.zeros((B, cfg.num_kv_heads, nbmax), np.float64)
    bsum = np.zeros((B, cfg.num_q_heads), np.float64)
    rc = lib().kvqo_decode_certified(C.byref(cfg), _p(pool), _p(k), _p(v), _p(q), _p(bt), bt.shape[1], _p(cl), B,
                                     scale, frac, _p(sel), _p(out), _p(prom), kmax, _p(scores), nbmax, _p(bsum),
                                     _p(forced))
    if rc != 0:
        raise ValueError(f"oracle certified decode rejected its arguments (rc={rc})")
    return out, prom, scores, bsum


def decode_ladder(cfg: Config, pool: np.ndarray, k_slots, v_slots, q, block_table, ctx_lens, policy: dict,
                  scale: float = 0.0, max_blocks: int = 0, forced_flags=None, forced_fallback=None) -> dict:
    """Certified decode with the adaptive ladder.  policy: tau_cov, max_frac,
    key_tol, v_tol, rank_tol, cert_tol, layer_frac (missing entries: the rung
    is off -- tau 0, budget 1, tolerances inf, layer_frac 1).  Returns a dict
    of numpy arrays: out, mixed, dense [B,Hq,d]; err, bound, status [B,Hq];
    k_star, k_cov, k_key [B,Hkv]; flags, rscore [B,Hkv,max_blocks]; cov, ekey
    [B,Hkv,max_blocks+1]; rank_margin [B,Hq]."""
    k = _c(k_slots, np.float16).view(np.uint16)
    v = _c(v_slots, np.float16).view(np.uint16)
    q = _c(q, np.float16).view(np.uint16)
    bt = _c(block_table, np.int32)
    cl = _c(ctx_lens, np.int32)
    B, hq, hkv, d = cl.shape[0], cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim
    blk = cfg.bound_block_tokens
    mb = max_blocks or max(1, int((int(cl.max()) + blk - 1) // blk) if B else 1)
    pol = dict(tau_cov=0.0, max_frac=1.0, key_tol=np.inf, v_tol=np.inf, rank_tol=np.inf, cert_tol=np.inf,
               layer_frac=1.0)
    pol.update(policy)
    r = {
        "out": np.zeros((B, hq, d)), "mixed": np.zeros((B, hq, d)), "dense": np.zeros((B, hq, d)),
        "err": np.zeros((B, hq)), "bound": np.zeros((B, hq)), "status": np.zeros((B, hq), np.int32),
        "k_star": np.zeros((B, hkv), np.int32), "k_cov": np.zeros((B, hkv), np.int32),
        "k_key": np.zeros((B, hkv), np.int32), "flags": np.zeros((B, hkv, mb), np.uint8),
        "rscore": np.zeros((B, hkv, mb)), "cov": np.zeros((B, hkv, mb + 1)), "ekey": np.zeros((B, hkv, mb + 1)),
        "rank_margin": np.zeros((B, hq)),
    }
    o = LadderOut(*[r[n].ctypes.data for n in ("out", "mixed", "dense", "err", "bound", "status", "k_star", "k_cov",
                                                "k_key", "flags", "rscore", "cov", "ekey")], mb,
                  r["rank_margin"].ctypes.data)
    ff = None if forced_flags is None else _c(forced_flags, np.uint8)
    if ff is not None:
        assert ff.shape == (B, hkv, mb)
    fb = None if forced_fallback is None else _c(forced_fallback, np.int32)
    if fb is not None:
        assert fb.shape == (B, hq)
    lp = Ladder(**{f[0]: float(pol[f[0]]) for f in Ladder._fields_})
    rc = lib().kvqo_decode_ladder(C.byref(cfg), _p(pool), _p(k), _p(v), _p(q), _p(bt), bt.shape[1], _p(cl), B,
                                  scale, C.byref(lp), _p(ff), _p(fb), C.byref(o))
    if rc != 0:
        raise ValueError(f"oracle ladder decode rejected its arguments (rc={rc})")
    return r


def decode_windows(cfg: Config, pool: np.ndarray, win_k, win_v, sink: int, recent: int, q, block_table, ctx_lens,
                   scale: float = 0.0) -> np.ndarray:
    """Decode with each sequence's first `sink` and last `recent` tokens exact
    (fp16 rows from the window store win_k/win_v [B, sink + recent, Hkv, d]:
    row t for t < sink, row sink + t % recent for recent tokens)."""
    wk = _c(win_k, np.float16).view(np.uint16)
    wv = _c(win_v, np.float16).view(np.uint16)
    q = _c(q, np.float16).view(np.uint16)
    bt = _c(block_table, np.int32)
    cl = _c(ctx_lens, np.int32)
    B = cl.shape[0]
    out = np.zeros((B, cfg.num_q_heads, cfg.head_dim), np.float64)
    rc = lib().kvqo_decode_windows(C.byref(cfg), _p(pool), _p(wk), _p(wv), sink, recent, _p(q), _p(bt), bt.shape[1],
                                   _p(cl), B, scale, _p(out))
    if rc != 0:
        raise ValueError(f"oracle window decode rejected its arguments (rc={rc})")
    return out


# --- HQMQ ([HQMQ] Hurwitz quaternion multiplicative quantisation) ------------

def hqmq_unit(p: int) -> np.ndarray:
    q = np.zeros(4, np.float32)
    lib().kvqo_hqmq_unit(p, _p(q))
    return q


def hqmq_codebook(seed: int, kvh: int, tensor: int) -> np.ndarray:
    S = np.zeros((HQMQ_NS, 4), np.float32)
    lib().kvqo_hqmq_codebook(seed, kvh, tensor, _p(S))
    return S


def hqmq_quantize_rows(y, S):
    """Encode rotated rows y [n, d]: fields [n, d/4] (15-bit index, 5-bit radius
    code), step (fp16 bits) [n], outlier mask [n], outlier slots [n, NO, 4]."""
    y = _c(y, np.float32)
    S = _c(S, np.float32)
    n, d = y.shape
    field = np.zeros((n, d // 4), np.uint32)
    step = np.zeros(n, np.uint16)
    mask = np.zeros(n, np.uint32)
    outl = np.zeros((n, HQMQ_NO, 4), np.uint16)
    lib().kvqo_hqmq_quantize_rows(_p(y), n, d, _p(S), _p(field), _p(step), _p(mask), _p(outl))
    return field, step, mask, outl


def hqmq_encode_dirs(u, S) -> np.ndarray:
    u = _c(u, np.float32)
    S = _c(S, np.float32)
    idx = np.zeros(u.shape[0], np.int32)
    lib().kvqo_hqmq_encode_dirs(_p(u), u.shape[0], _p(S), _p(idx))
    return idx


def e4m3_value(b: int) -> float:
    """Value of an E4M3 byte (NaN for S.1111.111)."""
    return float(lib().kvqo_e4m3_value(int(b) & 0xFF))


def e4m3_rn(x) -> np.ndarray:
    """Non-negative fp32 values to E4M3 bytes (nearest, ties to even, saturating at 448)."""
    x = _c(np.atleast_1d(x), np.float32)
    out = np.zeros(x.shape, np.uint8)
    lib().kvqo_e4m3_rn_sat_n(_p(x), _p(out), x.size)
    return out


def e2m1_rn(v) -> np.ndarray:
    """fp32 values to 4-bit e2m1 codes (nearest, ties to the even magnitude, saturating at 6)."""
    v = _c(np.atleast_1d(v), np.float32)
    out = np.zeros(v.shape, np.uint8)
    lib().kvqo_e2m1_rn_n(_p(v), _p(out), v.size)
    return out


def nvfp4_quantize_rows(y, search: int = 0):
    """NVFP4 codes [n, d] (uint8, one per element) and E4M3 scale bytes [n, d/16]
    of fp32 rows [n, d] (the codec the append applies)."""
    y = _c(y, np.float32)
    n, d = y.shape
    code = np.zeros((n, d), np.uint8)
    scale = np.zeros((n, d // 16), np.uint8)
    lib().kvqo_nvfp4_quantize_rows(_p(y), n, d, int(search), _p(code), _p(scale))
    return code, scale


def nvfp4_read_row(cfg: Config, pool: np.ndarray, slot: int, kvh: int, tensor: int):
    d = cfg.head_dim
    code = np.zeros(d, np.uint8)
    scale = np.zeros(d // 16, np.uint8)
    lib().kvqo_nvfp4_read_row(C.byref(cfg), _p(pool), slot, kvh, tensor, _p(code), _p(scale))
    return code, scale


def hqmq_read_row(cfg: Config, pool: np.ndarray, slot: int, kvh: int, tensor: int):
    d = cfg.head_dim
    field = np.zeros(d // 4, np.uint32)
    step = np.zeros(1, np.uint16)
    mask = np.zeros(1, np.uint32)
    outl = np.zeros((HQMQ_NO, 4), np.uint16)
    lib().kvqo_hqmq_read_row(C.byref(cfg), _p(pool), slot, kvh, tensor, _p(field), _p(step), _p(mask), _p(outl))
    return field, int(step[0]), int(mask[0]), outl
