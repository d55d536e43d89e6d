#!/usr/bin/env python
"""Benchmark of the low-bit KV-cache hot path on B200.

One step = quantise-on-append of one new token (K and V, 8 kv heads) plus
split-K decode attention of the 32 query heads over the grown context:
Llama-3-8B-shaped layer, batch 1, head_dim 128, int4 group-32 K and V with the
sign + Hadamard rotation, 16-token shuffled pages, context 32769..32868 (the
workload's 100-step window, replayed).  The step sequence is captured in a
CUDA graph; consecutive steps rotate over enough cache copies that the cache
they read is not resident in L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  value = decode KV bytes per step (packed codes
+ scales/zeros of every context token) / step time, whole job.  Under torchrun
every rank runs an independent replica (no collective on the data path;
"scaling": "weak"); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import ctypes as C
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "int4-KV decode attn: KV-bytes GB/s as % of HBM peak; µs/step; append GB/s"
NOMINAL_HBM_GBS = 8000.0


# DRAM bytes (read + write) per launch of the dominant kernel, as an ncu
# capture of the decode kernel at this workload counted them
# (dram__bytes_read.sum + dram__bytes_write.sum).  Reported as
# roofline.traffic only while the decode kernel's sources hash to the digest
# they had when the counters were taken; null otherwise.
PROFILED_DECODE = {"sources_sha256": "626c094f50917150a990ae7d752084cea4bba58f6ee155bac8bdcc98e96b37b0",
                   "dram_bytes_per_launch": 42160768}
DECODE_SOURCES = ("kvq_decode.cu", "kvq_internal.cuh", "kvq_warp.cuh")


def decode_sources_digest() -> str:
    import hashlib
    h = hashlib.sha256()
    for name in DECODE_SOURCES:
        with open(os.path.join(ROOT, "quantized_kv_cache_16_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def profiled_traffic():
    if PROFILED_DECODE["sources_sha256"] and PROFILED_DECODE["sources_sha256"] == decode_sources_digest():
        return PROFILED_DECODE["dram_bytes_per_launch"]
    return None


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-steps", type=int, default=4, help="oracle steps in the CPU baseline sample")
    ap.add_argument("--no-extras", action="store_true", help="skip e2e, append and CPU legs")
    ap.add_argument("--leg", choices=["paged", "certified", "ladder", "windows", "hqmq", "nvfp4", "contexts", "append",
                                      "e2e", "bitrev"],
                    help="run only this leg (one GPU, --steps calls) and print its JSON")
    ap.add_argument("--ctx", type=int, default=0, help="context length of --leg (default: its workload's)")
    return ap.parse_args()


# ------------------------------------------------------------------ plumbing --

class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        self.device = "cpu"

    def init(self, backend):
        if self.world > 1:
            import datetime
            import torch.distributed as td
            td.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = True
            self.device = "cuda" if backend == "nccl" else "cpu"

    def barrier(self):
        if self.pg:
            import torch.distributed as td
            td.barrier()

    def max(self, x: float) -> float:
        if not self.pg:
            return x
        import torch
        import torch.distributed as td
        t = torch.tensor([x], dtype=torch.float64, device=self.device)
        td.all_reduce(t, op=td.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            import torch.distributed as td
            td.destroy_process_group()


class Cudart:
    """cudaEventRecordWithFlags(..., cudaEventRecordExternal) so that event
    nodes captured in a graph stay observable timestamps."""

    def __init__(self):
        import torch  # noqa: F401  (loads libcudart into the process)
        lib = None
        for name in ("libcudart.so.12", "libcudart.so"):
            try:
                lib = C.CDLL(name)
                break
            except OSError:
                continue
        if lib is None:
            import glob
            import nvidia.cuda_runtime as rt
            lib = C.CDLL(glob.glob(os.path.join(os.path.dirname(rt.__file__), "lib", "libcudart.so*"))[0])
        self.lib = lib

    def event(self):
        ev = C.c_void_p()
        assert self.lib.cudaEventCreate(C.byref(ev)) == 0
        return ev

    def record_external(self, ev, stream):
        rc = self.lib.cudaEventRecordWithFlags(ev, C.c_void_p(stream), 1)
        assert rc == 0, f"cudaEventRecordWithFlags returned {rc}"

    def record(self, ev, stream):
        rc = self.lib.cudaEventRecord(ev, C.c_void_p(stream))
        assert rc == 0, f"cudaEventRecord returned {rc}"

    def elapsed_ms(self, a, b) -> float:
        ms = C.c_float()
        assert self.lib.cudaEventElapsedTime(C.byref(ms), a, b) == 0
        return ms.value

    def destroy(self, ev):
        self.lib.cudaEventDestroy(ev)

    def graph_upload(self, graph, stream):
        """cudaGraphUpload of a captured torch graph: its first launch then
        does not pay the upload of the executable graph to the device."""
        rc = self.lib.cudaGraphUpload(C.c_void_p(graph.raw_cuda_graph_exec()), C.c_void_p(stream))
        assert rc == 0, f"cudaGraphUpload returned {rc}"


class ClockSampler(threading.Thread):
    """Polls NVML (SM clock, clock-event reasons) every ~2 ms."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting", 0x10: "sync_boost"}

    def __init__(self, index):
        super().__init__(daemon=True)
        self.samples = []
        self.stop_flag = False
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            self.reasons_fn = fn
            self.ok = True
        except Exception as e:  # no NVML: report that, do not guess
            self.err = repr(e)

    def run(self):
        while self.ok and not self.stop_flag:
            try:
                t = time.perf_counter()
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = self.reasons_fn(self.h)
                self.samples.append((t, mhz, rs))
            except Exception:
                pass
            time.sleep(0.002)

    def wait_samples(self, n, limit_s=3.0):
        t = time.perf_counter()
        while self.ok and len(self.samples) < n and time.perf_counter() - t < limit_s:
            time.sleep(0.001)

    def wait_after(self, t1, limit_s=1.0):
        t = time.perf_counter()
        while self.ok and not any(s[0] > t1 for s in self.samples[-3:]) and time.perf_counter() - t < limit_s:
            time.sleep(0.001)

    def summary(self, t0, t1):
        if not self.ok:
            return {"error": getattr(self, "err", "nvml unavailable")}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        window = "timed region"
        if not inside:  # region shorter than one poll: the samples just before and after it
            before = [s for s in self.samples if s[0] < t0][-1:]
            after = [s for s in self.samples if s[0] > t1][:1]
            inside = before + after
            window = "samples just before and after a timed region shorter than the poll period"
        reasons = set()
        for _, _, rs in inside:
            for bit, name in self.REASONS.items():
                if rs & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s[1] for s in inside) if inside else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(inside), "window": window}


# ----------------------------------------------------------- the workload ---

def workload_name(T: int, window: int) -> str:
    return (f"llama3-8b layer decode step: B=1, Hq=32, Hkv=8, d=128, int4 g32 K/V, sign+Hadamard rotation, "
            f"16-token shuffled pages, context {T + 1}..{T + window} (append 1 token + decode per step)")


def kv_bytes_per_token(d: int, hkv: int) -> int:
    # int4 g32: d/2 code bytes + (d/32) x (scale, zero) fp16, for K and for V
    return hkv * 2 * (d // 2 + (d // 32) * 4)


class Workload:
    """Llama-3-8B layer decode steps over C rotating cache copies."""

    def __init__(self, dist: Dist, T: int = 0, window: int = 100, rotate: int = 1):
        import numpy as np
        import torch

        import quantized_kv_cache_16_b200 as K
        import workloads as W

        self.K, self.W = K, W
        self.wl = wl = W.llama() if not T else W.llama(T=T, steps=window)
        self.T, self.window = wl.ctx[0], wl.steps
        dev = torch.device("cuda", torch.cuda.current_device())
        props = torch.cuda.get_device_properties(dev)
        l2 = int(getattr(props, "L2_cache_size", 126 << 20))
        cache_bytes = (self.T + self.window) * kv_bytes_per_token(wl.d, wl.Hkv)
        self.copies = max(2, math.ceil(3 * l2 / cache_bytes))
        self.l2 = l2
        tabs = W.page_table(wl, extra_tokens=self.window, copies=self.copies)
        self.tabs = tabs
        kw = dict(num_q_heads=wl.Hq, num_kv_heads=wl.Hkv, head_dim=wl.d, k_fmt=wl.k_fmt, v_fmt=wl.v_fmt,
                  k_group=wl.k_group, v_group=wl.v_group, clip_ratio=wl.clip, rotation_seed=wl.rotation_seed,
                  rotate=rotate, num_pages=tabs[0].num_pages)
        self.cfg_kw = kw
        self.cache = K.Cache(K.make_config(**kw))
        if T:  # other contexts (timing only): the prefix is drawn on the device
            kd, vd = W.prefix_kv_device(wl, 0, dev)
        else:
            k, v = W.prefix_kv(wl, 0)
            kd, vd = torch.from_numpy(k).to(dev), torch.from_numpy(v).to(dev)
        for c in range(self.copies):  # same prefix values, distinct memory per copy
            self.cache.append(kd, vd, torch.from_numpy(tabs[c].slots(0, 0, self.T)).to(dev))
        del kd, vd
        nk, nv, qs = [], [], []
        for u in range(self.window):
            a, b = W.step_kv(wl, u)
            nk.append(a)
            nv.append(b)
            qs.append(W.queries(wl, u))
        self.h_newk, self.h_newv, self.h_q = np.stack(nk), np.stack(nv), np.stack(qs)
        self.newk = torch.from_numpy(self.h_newk).to(dev)  # [window, 1, Hkv, d]
        self.newv = torch.from_numpy(self.h_newv).to(dev)
        self.q = torch.from_numpy(self.h_q).to(dev)        # [window, 1, Hq, d]
        self.h_slots = np.array([[tabs[c].slot(0, self.T + u) for u in range(self.window)]
                                 for c in range(self.copies)], np.int32)
        self.slots = torch.from_numpy(self.h_slots).to(dev)  # [C, window]
        self.h_ctx = np.arange(self.T + 1, self.T + self.window + 1, dtype=np.int32)
        self.ctx = torch.from_numpy(self.h_ctx).to(dev)  # [window]
        self.bt = torch.stack([torch.from_numpy(t.block_table) for t in tabs]).to(dev)  # [C, 1, P]
        self.max_pages = self.bt.shape[2]
        self.ws = self.cache.workspace_for(1, self.max_pages)
        self.out = torch.empty(1, wl.Hq, wl.d, dtype=torch.float32, device=dev)
        torch.cuda.synchronize()

    def step_index(self, s):
        return s % self.copies, (s // self.copies) % self.window

    def kv_bytes(self, s):
        _, u = self.step_index(s)
        return int(self.h_ctx[u]) * kv_bytes_per_token(self.wl.d, self.wl.Hkv)

    def decode_algorithmic_bytes(self, s):
        _, u = self.step_index(s)
        wl = self.wl
        ctx = int(self.h_ctx[u])
        qo = wl.B * wl.Hq * wl.d * (2 + 4)  # fp16 q in, fp32 out
        return self.kv_bytes(s) + qo + 4 * ((ctx + 15) // 16) + 4

    def launch_step(self, s, stream, rt=None, evs=None):
        """One step through the public API: kvq_decode_step appends the new
        token and attends over the grown context in one launch."""
        K = self.K
        c, u = self.step_index(s)
        if rt is not None:
            rt.record_external(evs[0], stream.cuda_stream)
        K.kvq_decode_step(self.cache.handle, self.newk[u], self.newv[u], self.slots[c, u:u + 1], self.q[u],
                          self.bt[c], self.max_pages, self.ctx[u:u + 1], 1, 0.0, self.ws, self.ws.numel(), self.out,
                          stream)
        if rt is not None:
            rt.record_external(evs[1], stream.cuda_stream)


def run_ours(args, dist: Dist):
    import numpy as np
    import torch

    torch.cuda.set_device(dist.local)
    dist.init("nccl")
    wk = Workload(dist)
    rt = Cudart()
    stream = torch.cuda.Stream()
    K = args.steps

    def capture(n, with_events):
        g = torch.cuda.CUDAGraph()
        evs = [(rt.event(), rt.event()) for _ in range(n)] if with_events else None
        with torch.cuda.stream(stream):
            for s in range(3):  # first-use configuration outside the capture
                wk.launch_step(s, stream)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=stream):
            for s in range(n):
                wk.launch_step(s, stream, rt if with_events else None, evs[s] if with_events else None)
        return g, evs

    g_warm, _ = capture(max(args.warmup, 3), False)
    g_timed, _ = capture(K, False)
    sampler = ClockSampler(dist.local)
    sampler.start()
    sampler.wait_samples(2)  # polling before the timed region starts
    for _ in range(2):
        g_warm.replay()
    # the timed graph goes to the device before timing (uploaded at its first
    # launch otherwise: ~1.6 us a step of the first replay at 2000 steps)
    rt.graph_upload(g_timed, stream.cuda_stream)
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = rt.event(), rt.event()
    t0 = time.perf_counter()
    rt.record(e0, stream.cuda_stream)
    with torch.cuda.stream(stream):
        g_timed.replay()
    rt.record(e1, stream.cuda_stream)
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    sampler.wait_after(t1)  # one sample on each side of a region shorter than the poll period
    dist.barrier()
    sampler.stop_flag = True
    elapsed_ms = rt.elapsed_ms(e0, e1)
    elapsed_ms = dist.max(elapsed_ms)
    clocks = sampler.summary(t0, t1)

    bytes_rank = sum(wk.kv_bytes(s) for s in range(K))
    value = bytes_rank * dist.world / (elapsed_ms * 1e-3) / 1e9
    peak, peak_kind = measured_peaks()
    alg = statistics.mean(wk.decode_algorithmic_bytes(s) for s in range(K))
    # the timed region is K launches of the one fused kernel back to back:
    # its average launch duration is the region's time over K (the graph's
    # launch gaps included, so this slightly understates the kernel)
    dec_mean = elapsed_ms / K
    achieved = alg / (dec_mean * 1e-3) / 1e9
    result = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": dist.world, "steps": K,
        "warmup": max(args.warmup, 3), "ms_per_step": elapsed_ms / K, "us_per_step": 1e3 * elapsed_ms / K,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int4 codes; f16 mma with f32 accumulate", "data": "synthetic",
        "config": {"workload": workload_name(wk.T, wk.window),
                   "global_batch": dist.world, "seq_len": wk.T, "parallelism": f"replicas x{dist.world}",
                   "l2_policy": f"{wk.copies} rotating cache copies ({wk.copies * (wk.T + wk.window) * kv_bytes_per_token(128, 8) / 1e6:.0f} MB) > 3x L2 ({wk.l2 / 1e6:.0f} MB)",
                   "cuda_graph": True},
        "pct_hbm_peak": value / dist.world / peak, "peak_gbs": peak, "peak_kind": peak_kind,
        "pct_hbm_nominal_8tbs": value / dist.world / NOMINAL_HBM_GBS,
        "roofline": {"bound": "hbm", "kernel": "decode_kernel<128,int4,int4> (fused append + decode step)",
                     "achieved": round(achieved, 1), "duration": "timed region / launches",
                     "peak": peak, "unit": "GB/s", "frac": achieved / peak, "traffic": profiled_traffic(),
                     "bytes_per_launch": alg, "launch_us": dec_mean * 1e3,
                     "note": f"peak of {peak_kind}"},
        "gpu_launches": K,
        "clocks": clocks,
    }
    if not args.no_extras:
        result["e2e"] = e2e_leg(wk, K, stream, dist)
        result["append"] = append_leg()
        result["paged"] = paged_leg(min(K, 200))
        result["certified"] = certified_leg(min(K, 200))
        result["ladder"] = ladder_leg(min(K, 100))
        result["windows"] = windows_leg(min(K, 200))
        result["hqmq"] = hqmq_leg(min(K, 200))
        result["nvfp4"] = nvfp4_leg(min(K, 200))
        result["contexts"] = contexts_leg(min(K, 200))
        result["bitrev"] = bitrev_leg(min(K, 200))
    if dist.rank == 0:
        if not args.no_extras:
            result["cpu_baseline"] = cpu_leg(wk, args.cpu_steps)
        print(json.dumps(result), flush=True)
    del g_warm, g_timed
    dist.close()


def e2e_leg(wk: Workload, K: int, stream, dist: Dist):
    """The same steps through the public C ABI with host buffers: one
    kvq_decode_step_host call a step enqueues the copy of that step's pinned
    host record (q, the new token's k and v, its slot and the context length)
    to the device (on the library's copy stream, overlapping the previous
    step's kernel) and the fused append + decode, whose kernel writes the
    output to pinned host memory through its device mapping.  The call's
    arguments are marshalled once, before the timed region."""
    import ctypes as C

    import numpy as np
    import torch
    Kb = wk.K
    dev = wk.q.device
    handle = wk.cache.handle
    rec = Kb.kvq_step_record_bytes(handle, 1)
    nq, nk = wk.q[0].numel() * 2, wk.newk[0].numel() * 2
    off_k = (nq + 15) // 16 * 16
    off_v = off_k + (nk + 15) // 16 * 16
    off_s = off_v + (nk + 15) // 16 * 16
    off_c = off_s + 16
    assert rec == off_c + 16
    h_in = np.zeros((wk.copies, wk.window, rec), np.uint8)
    for c in range(wk.copies):
        for u in range(wk.window):
            h_in[c, u, :nq] = wk.h_q[u].reshape(-1).view(np.uint8)
            h_in[c, u, off_k:off_k + nk] = wk.h_newk[u].reshape(-1).view(np.uint8)
            h_in[c, u, off_v:off_v + nk] = wk.h_newv[u].reshape(-1).view(np.uint8)
            h_in[c, u, off_s:off_s + 4] = np.array([wk.h_slots[c, u]], np.int32).view(np.uint8)
            h_in[c, u, off_c:off_c + 4] = np.array([wk.h_ctx[u]], np.int32).view(np.uint8)
    h_in = torch.from_numpy(h_in).pin_memory()
    h_out = torch.empty((wk.window,) + tuple(wk.out.shape), dtype=torch.float32).pin_memory()
    d_rec = torch.empty(2 * rec, dtype=torch.uint8, device=dev)  # two records, used alternately
    fn = Kb.lib().kvq_decode_step_host
    st = C.c_void_p(stream.cuda_stream)
    args = {}
    for c in range(wk.copies):
        for u in range(wk.window):
            args[(c, u)] = (handle, C.c_void_p(h_in[c, u].data_ptr()), C.c_void_p(d_rec.data_ptr()),
                            C.c_void_p(wk.bt[c].data_ptr()), wk.max_pages, 1, C.c_float(0.0),
                            C.c_void_p(wk.ws.data_ptr()), wk.ws.numel(), C.c_void_p(h_out[u].data_ptr()), st)

    def step(s):
        rc = fn(*args[wk.step_index(s)])
        if rc != 0:
            raise Kb.KvqError("kvq_decode_step_host", rc)

    for s in range(20):
        step(s)
    torch.cuda.synchronize()
    dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    t0 = time.perf_counter()
    for s in range(K):
        step(s)
    t_host = time.perf_counter() - t0
    e1.record(stream)
    torch.cuda.synchronize()
    ms = dist.max(e0.elapsed_time(e1))
    h2d = rec
    d2h = wk.out.numel() * 4
    bytes_rank = sum(wk.kv_bytes(s) for s in range(K))
    return {"value": round(bytes_rank * dist.world / (ms * 1e-3) / 1e9, 1), "unit": "GB/s",
            "us_per_step": 1e3 * ms / K, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "host_us_per_step": round(1e6 * t_host / K, 2),
            "how": "one kvq_decode_step_host call per step: the step's pinned host record (q, k, v, slot, ctx) "
                   "copied to the device on the library's copy stream (overlapping the previous step's kernel), "
                   "the fused append + decode, whose kernel writes the output to pinned host memory through its "
                   "device mapping, inside the event-timed region"}


def append_leg():
    """Bulk quantise-on-append: one 65536-token prefill of K and V (8 kv
    heads x 128, Laplace(0,1) with 1% outliers x30) to 2-bit g128, clip 0.9;
    then the same with ScaleSearch of every scale (nine candidates a group)."""
    import numpy as np
    import torch

    import quantized_kv_cache_16_b200 as K
    import workloads as W
    wl = W.int2(B=1)
    T = wl.ctx[0]
    pages = W.page_table(wl)[0]
    k, v = W.prefix_kv(wl, 0)
    kd, vd = torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda()
    slots = torch.from_numpy(pages.slots(0, 0, T)).cuda()
    in_bytes = 2 * T * wl.Hkv * wl.d * 2
    out_bytes = 2 * T * wl.Hkv * (wl.d // 4 + 4)
    peak, kind = measured_peaks()
    res = {}
    for search in (0, 1):
        cfg = K.make_config(wl.Hq, wl.Hkv, wl.d, wl.k_fmt, wl.v_fmt, wl.k_group, wl.v_group, wl.clip,
                            wl.rotation_seed, num_pages=pages.num_pages, scale_search=search)
        cache = K.Cache(cfg)
        for _ in range(3):
            cache.append(kd, vd, slots)
        torch.cuda.synchronize()
        reps = 20
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for a, b in evs:
            a.record()
            cache.append(kd, vd, slots)
            b.record()
        torch.cuda.synchronize()
        res[search] = statistics.mean(a.elapsed_time(b) for a, b in evs) * 1e3
        del cache
    gbs = (in_bytes + out_bytes) / (res[0] * 1e-6) / 1e9
    gbs_s = (in_bytes + out_bytes) / (res[1] * 1e-6) / 1e9
    return {"workload": "prefill append 65536 x 8 x 128 K and V, 2-bit g128 clip 0.9, rotated",
            "GB/s": round(gbs, 1), "us": res[0], "bytes": in_bytes + out_bytes, "pct_hbm_peak": gbs / peak,
            "peak_kind": kind, "inputs_exceed_l2": True,
            "scale_search": {"GB/s": round(gbs_s, 1), "us": res[1], "pct_hbm_peak": gbs_s / peak}}


def _tier2_cache(wl, copies: int):
    """A certified-mode cache of `copies` independent copies of sequence 0 of
    `wl` (drawn on the device), with the exact fp16 rows in pinned host memory
    as tier 2."""
    import torch

    import quantized_kv_cache_16_b200 as K
    import workloads as W
    T = wl.ctx[0]
    dev = torch.device("cuda", torch.cuda.current_device())
    tabs = W.page_table(wl, copies=copies)
    cfg = K.make_config(wl.Hq, wl.Hkv, wl.d, wl.k_fmt, wl.v_fmt, wl.k_group, wl.v_group, wl.clip, wl.rotation_seed,
                        num_pages=tabs[0].num_pages, bound_block_tokens=wl.bound_block)
    cache = K.Cache(cfg)
    kd, vd = W.prefix_kv_device(wl, 0, dev)
    rows = tabs[0].num_pages * 16
    k2 = torch.empty((rows, wl.Hkv, wl.d), dtype=torch.float16).pin_memory()
    v2 = torch.empty_like(k2).pin_memory()
    kh, vh = kd.cpu(), vd.cpu()
    for c in range(copies):
        sl = torch.from_numpy(tabs[c].slots(0, 0, T)).long()
        cache.append(kd, vd, sl.int().to(dev))
        k2[sl], v2[sl] = kh, vh
    del kd, vd, kh, vh
    bts = [torch.from_numpy(t.block_table).to(dev) for t in tabs]
    ctx = torch.tensor([T], dtype=torch.int32, device=dev)
    return cache, k2, v2, bts, ctx


def _graph_time(call, steps: int, stream) -> float:
    """Mean microseconds of call(s) for s in range(steps), replayed as one
    CUDA graph after four eager warm-up calls and one warm-up replay."""
    import torch
    with torch.cuda.stream(stream):
        for s in range(4):
            call(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
        for s in range(steps):
            call(s)
    g.replay()
    torch.cuda.synchronize()
    rt = Cudart()
    e0, e1 = rt.event(), rt.event()
    rt.record(e0, stream.cuda_stream)
    with torch.cuda.stream(stream):
        g.replay()
    rt.record(e1, stream.cuda_stream)
    torch.cuda.synchronize()
    us = rt.elapsed_ms(e0, e1) * 1e3 / steps
    del g
    return us


def certified_leg(steps: int, T: int = 0):
    """Certified decode at its own configuration: batch 1, context 131072,
    int8 K / int4 g32 V, 128-token bound blocks, top 1% of each kv head's
    blocks promoted from exact fp16 rows in pinned host memory.  Calls (four
    launches each) replayed in a CUDA graph over two cache copies (440 MB >
    3x L2) and timed as a whole, beside the plain quantised decode of the
    same cache."""
    import torch

    import quantized_kv_cache_16_b200 as K
    import workloads as W
    wl = W.certified(T) if T else W.certified()
    T, frac, copies = wl.ctx[0], 0.01, 2
    dev = torch.device("cuda", torch.cuda.current_device())
    cache, k2, v2, bts, ctx = _tier2_cache(wl, copies)
    nq = 8
    gen = torch.Generator(device=dev)
    gen.manual_seed(wl.seed)
    qs = torch.randn((nq, 1, wl.Hq, wl.d), generator=gen, device=dev).half()
    max_pages = bts[0].shape[1]
    ws = cache.workspace_for(1, max_pages)
    out = torch.empty((1, wl.Hq, wl.d), dtype=torch.float32, device=dev)
    nb = (T + wl.bound_block - 1) // wl.bound_block
    kmax = math.ceil(frac * nb - 1e-9)
    prom = torch.empty((1, wl.Hkv, kmax), dtype=torch.int32, device=dev)
    t2 = K.kvq_tier2(k2.data_ptr(), v2.data_ptr(), frac)
    stream = torch.cuda.Stream()

    def caller(tier2):
        def call(s):
            K.kvq_decode_attn(cache.handle, qs[s % nq], bts[s % copies], max_pages, ctx, 1, 0.0, tier2, ws,
                              ws.numel(), out, prom if tier2 is not None else None, stream)
        return call

    res = {name: _graph_time(caller(tier2), steps, stream) for name, tier2 in (("quantised_only", None),
                                                                                ("certified", t2))}
    assert cache.sync_status() == 0
    hbm = T * wl.Hkv * (wl.d + 2 + wl.d // 2 + 4 * (wl.d // 32))
    link = wl.Hkv * kmax * wl.bound_block * wl.d * 2 * 2
    peak, kind = measured_peaks()
    return {"workload": f"certified decode: B=1, 32/8 heads, d=128, context {T}, int8 K / int4 g32 V, "
                        "128-token bound blocks, top 1% promoted from pinned host fp16 rows",
            "us": round(res["certified"], 2), "quantised_only_us": round(res["quantised_only"], 2),
            "overhead_x": round(res["certified"] / res["quantised_only"], 2),
            "hbm_bytes": hbm, "host_link_bytes": link, "promoted_blocks_per_kv_head": kmax,
            "quantised_only_GB/s": round(hbm / (res["quantised_only"] * 1e-6) / 1e9, 1),
            "quantised_only_pct_hbm_peak": hbm / (res["quantised_only"] * 1e-6) / 1e9 / peak, "peak_kind": kind,
            "l2_policy": "2 cache copies (440 MB) alternate", "steps": steps}


def paged_leg(steps: int, T: int = 0):
    """Batched paged decode: batch 16, 32/8 heads, d=128, int4 g32 rotated,
    context lengths uniform in [1024, 8192] from the seed, 16-token pages
    shuffled in the block table.  Each step appends one token per sequence
    and attends (kvq_decode_step, one launch); steps replayed in a CUDA graph
    that rotates over enough cache copies to exceed 3x L2."""
    import torch

    import quantized_kv_cache_16_b200 as K
    import workloads as W
    wl = W.paged()
    window = 16
    dev = torch.device("cuda", torch.cuda.current_device())
    l2 = int(getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 126 << 20))
    per_copy = sum(wl.ctx) * kv_bytes_per_token(wl.d, wl.Hkv)
    copies = max(2, math.ceil(3 * l2 / per_copy))
    tabs = W.page_table(wl, extra_tokens=window, copies=copies)
    cfg = K.make_config(wl.Hq, wl.Hkv, wl.d, wl.k_fmt, wl.v_fmt, wl.k_group, wl.v_group, wl.clip, wl.rotation_seed,
                        num_pages=tabs[0].num_pages)
    cache = K.Cache(cfg)
    for b in range(wl.B):
        kd, vd = W.prefix_kv_device(wl, b, dev)
        for c in range(copies):
            cache.append(kd, vd, torch.from_numpy(tabs[c].slots(b, 0, wl.ctx[b])).to(dev))
        del kd, vd
    gen = torch.Generator(device=dev)
    gen.manual_seed(wl.seed)
    newk = torch.randn((window, wl.B, wl.Hkv, wl.d), generator=gen, device=dev).half()
    newv = (0.5 * torch.randn((window, wl.B, wl.Hkv, wl.d), generator=gen, device=dev)).half()
    qs = torch.randn((window, wl.B, wl.Hq, wl.d), generator=gen, device=dev).half()
    slots = torch.tensor([[[tabs[c].slot(b, wl.ctx[b] + u) for b in range(wl.B)] for u in range(window)]
                          for c in range(copies)], dtype=torch.int32, device=dev)  # [C, window, B]
    ctxs = torch.tensor([[t + u + 1 for t in wl.ctx] for u in range(window)], dtype=torch.int32, device=dev)
    bts = [torch.from_numpy(t.block_table).to(dev) for t in tabs]
    max_pages = bts[0].shape[1]
    ws = cache.workspace_for(wl.B, max_pages)
    out = torch.empty((wl.B, wl.Hq, wl.d), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream()
    n = (steps // (copies * window) + 1) * copies * window  # whole passes over (copy, step)

    def step(s):
        c, u = s % copies, (s // copies) % window
        K.kvq_decode_step(cache.handle, newk[u], newv[u], slots[c, u], qs[u], bts[c], max_pages, ctxs[u], wl.B, 0.0,
                          ws, ws.numel(), out, stream)

    us = _graph_time(step, n, stream)
    assert cache.sync_status() == 0
    mean_ctx = sum(wl.ctx) + wl.B * (window + 1) / 2
    kv = mean_ctx * kv_bytes_per_token(wl.d, wl.Hkv)
    alg = kv + wl.B * wl.Hq * wl.d * (2 + 4) + 4 * sum((t + window + 15) // 16 for t in wl.ctx) + \
        wl.B * wl.Hkv * wl.d * 2 * 2
    peak, kind = measured_peaks()
    gbs = alg / (us * 1e-6) / 1e9
    return {"workload": f"batched paged decode step: B={wl.B}, 32/8 heads, d=128, int4 g32 rotated, context "
                        f"lengths U[1024, 8192] (sum {sum(wl.ctx)}), shuffled 16-token pages, append 1 token per "
                        f"sequence + decode (one launch)",
            "us_per_step": round(us, 2), "kv_bytes_per_step": int(kv), "algorithmic_bytes_per_step": int(alg),
            "gbs": round(gbs, 1), "pct_hbm_peak": gbs / peak, "peak_kind": kind,
            "pct_hbm_nominal_8tbs": gbs / NOMINAL_HBM_GBS, "steps": n,
            "l2_policy": f"{copies} rotating cache copies ({copies * per_copy / 1e6:.0f} MB) > 3x L2"}


def windows_leg(steps: int, T: int = 0, sink: int = 128, recent: int = 1024):
    """Decode with fp16 sink and recent windows over the 2-bit cache (batch 4,
    32/8 heads, context 65536, 2-bit g128 clip 0.9): the first 128 and the
    last 1024 tokens of each sequence from a device window store, the rest
    quantised; CUDA graph over two cache copies, beside the plain quantised
    decode of the same cache."""
    import torch

    import quantized_kv_cache_16_b200 as K
    import workloads as W
    wl = W.int2() if not T else W.int2(T=T)
    copies = 2
    dev = torch.device("cuda", torch.cuda.current_device())
    tabs = W.page_table(wl, copies=copies)
    cfg = K.make_config(wl.Hq, wl.Hkv, wl.d, wl.k_fmt, wl.v_fmt, wl.k_group, wl.v_group, wl.clip, wl.rotation_seed,
                        num_pages=tabs[0].num_pages)
    cache = K.Cache(cfg)
    Wn = sink + recent
    wk = torch.empty((wl.B, Wn, wl.Hkv, wl.d), dtype=torch.float16, device=dev)
    wv = torch.empty_like(wk)
    for b in range(wl.B):
        kd, vd = W.prefix_kv_device(wl, b, dev)
        Tb = wl.ctx[b]
        for c in range(copies):
            cache.append(kd, vd, torch.from_numpy(tabs[c].slots(b, 0, Tb)).to(dev))
        wk[b, :sink], wv[b, :sink] = kd[:sink], vd[:sink]
        pos = torch.arange(Tb - recent, Tb, device=dev)
        wk[b, sink + pos % recent], wv[b, sink + pos % recent] = kd[pos], vd[pos]
        del kd, vd
    gen = torch.Generator(device=dev)
    gen.manual_seed(wl.seed)
    nq = 8
    qs = torch.randn((nq, wl.B, wl.Hq, wl.d), generator=gen, device=dev).half()
    bts = [torch.from_numpy(t.block_table).to(dev) for t in tabs]
    max_pages = bts[0].shape[1]
    ctx = torch.tensor(wl.ctx, dtype=torch.int32, device=dev)
    ws = cache.workspace_for(wl.B, max_pages)
    out = torch.empty((wl.B, wl.Hq, wl.d), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream()

    def quant(s):
        K.kvq_decode_attn(cache.handle, qs[s % nq], bts[s % copies], max_pages, ctx, wl.B, 0.0, None, ws, ws.numel(),
                          out, None, stream)

    def win(s):
        K.kvq_decode_windows(cache.handle, qs[s % nq], bts[s % copies], max_pages, ctx, wl.B, 0.0, wk, wv, sink,
                             recent, ws, ws.numel(), out, stream)

    q_us = _graph_time(quant, steps, stream)
    w_us = _graph_time(win, steps, stream)
    assert cache.sync_status() == 0
    kv_bytes = sum(wl.ctx) * wl.Hkv * 2 * (wl.d // 4 + 4)
    win_bytes = wl.B * Wn * wl.Hkv * wl.d * 2 * 2
    return {"workload": f"2-bit g128 cache, B={wl.B}, 32/8 heads, d=128, context {wl.ctx[0]}, fp16 sink {sink} + "
                        f"recent {recent} tokens per sequence from a device store",
            "us": round(w_us, 2), "quantised_only_us": round(q_us, 2), "overhead_x": round(w_us / q_us, 3),
            "cache_bytes": kv_bytes, "window_bytes": win_bytes, "steps": steps}


CONTEXTS = (4096, 8192, 16384, 32768, 65536, 131072, 262144)


def contexts_leg(steps: int, T: int = 0):
    """The headline decode step (batch 1, int4 g32, append + decode, rotating
    cache copies > 3x L2) at contexts from 4K to 256K tokens, and a least
    squares fit of step time = fixed + bytes / stream bandwidth over them: the
    fixed part is what a step costs whatever the context (launch, prologue,
    the two merges), the bandwidth is the page stream's."""
    import numpy as np
    import torch
    stream = torch.cuda.Stream()
    peak, peak_kind = measured_peaks()
    rows = []
    for ctx in ((T,) if T else CONTEXTS):
        wk = Workload(Dist(), T=ctx, window=16)
        us = _graph_time(lambda s: wk.launch_step(s, stream), steps, stream)
        assert wk.cache.sync_status() == 0
        alg = statistics.mean(wk.decode_algorithmic_bytes(s) for s in range(steps))
        rows.append({"context": ctx + 1, "us": round(us, 2), "bytes": int(alg), "gbs": round(alg / us / 1e3, 1),
                     "frac": round(alg / us / 1e3 / peak, 4), "copies": wk.copies})
        del wk
        torch.cuda.empty_cache()
    out = {"workload": "llama3-8b layer decode step (B=1, 32/8 heads, d=128, int4 g32, append 1 token + decode) "
                       "at each context; cache copies rotate over > 3x L2",
           "peak_gbs": peak, "peak_kind": peak_kind, "points": rows, "steps": steps}
    if len(rows) >= 3:
        x = np.array([r["bytes"] for r in rows], float)
        y = np.array([r["us"] for r in rows], float)
        slope, fixed = np.polyfit(x, y, 1)
        out["fit"] = {"fixed_us": round(float(fixed), 2), "stream_gbs": round(1e-3 / float(slope), 1),
                      "stream_frac": round(1e-3 / float(slope) / peak, 4),
                      "model": "us = fixed_us + bytes / stream_gbs"}
    return out


def bitrev_leg(steps: int, T: int = 0):
    """The headline decode step with the sign + Hadamard rotation (rotate 1)
    and with OSCAR's bit-reversal permutation after it (rotate 2), on the
    same rows and the same rotating cache copies: what the permutation costs
    the append and the decode."""
    import torch
    stream = torch.cuda.Stream()
    peak, peak_kind = measured_peaks()
    rows = []
    for rot in (1, 2):
        wk = Workload(Dist(), T=T, window=100, rotate=rot)
        us = _graph_time(lambda s: wk.launch_step(s, stream), steps, stream)
        assert wk.cache.sync_status() == 0
        alg = statistics.mean(wk.decode_algorithmic_bytes(s) for s in range(steps))
        rows.append({"rotate": rot, "context": wk.T + 1, "us": round(us, 2), "gbs": round(alg / us / 1e3, 1),
                     "frac": round(alg / us / 1e3 / peak, 4)})
        del wk
        torch.cuda.empty_cache()
    return {"workload": "llama3-8b layer decode step (B=1, 32/8 heads, d=128, int4 g32, append 1 token + decode), "
                        "rotate 1 (signs + Hadamard) vs rotate 2 (then bit reversal); cache copies rotate over > 3x L2",
            "peak_gbs": peak, "peak_kind": peak_kind, "points": rows, "steps": steps}


def nvfp4_leg(steps: int, T: int = 0):
    """The NVFP4 codec at Llama-3-8B layer shape (batch 1, 32/8 heads,
    d=128, context 32768, rotated, ScaleSearch on the E4M3 scales): the bulk
    append of the whole context and a one-token append timed with events;
    the decode replayed in a CUDA graph over four cache copies (151 MB, above
    L2), beside the same decode of a cache without ScaleSearch and that
    cache's fused append + decode step (kvq_decode_step, one launch)."""
    import torch

    import quantized_kv_cache_16_b200 as K
    import workloads as W
    wl = W.nvfp4(T) if T else W.nvfp4()
    T, copies = wl.ctx[0], 4
    dev = torch.device("cuda", torch.cuda.current_device())
    tabs = W.page_table(wl, copies=copies, extra_tokens=8)
    rt = Cudart()
    stream = torch.cuda.Stream()
    e0, e1 = rt.event(), rt.event()
    kd, vd = W.prefix_kv_device(wl, 0, dev)
    res = {}
    for search in (1, 0):
        cfg = K.make_config(wl.Hq, wl.Hkv, wl.d, wl.k_fmt, wl.v_fmt, wl.k_group, wl.v_group, wl.clip,
                            wl.rotation_seed, rotate=wl.rotate, num_pages=tabs[0].num_pages, scale_search=search)
        cache = K.Cache(cfg)
        bulk_ms = []
        for c in range(copies):
            sl = torch.from_numpy(tabs[c].slots(0, 0, T)).to(dev)
            rt.record(e0, stream.cuda_stream)
            with torch.cuda.stream(stream):
                cache.append(kd, vd, sl, stream=stream)
            rt.record(e1, stream.cuda_stream)
            torch.cuda.synchronize()
            bulk_ms.append(rt.elapsed_ms(e0, e1))
        kn, vn = (torch.from_numpy(x).to(dev) for x in W.step_kv(wl, 0))
        tok_slots = [torch.from_numpy(tabs[0].slots(0, T + i, T + i + 1)).to(dev) for i in range(8)]
        with torch.cuda.stream(stream):
            for i in range(3):
                cache.append(kn, vn, tok_slots[i], stream=stream)
        torch.cuda.synchronize()
        rt.record(e0, stream.cuda_stream)
        with torch.cuda.stream(stream):
            for i in range(50):
                cache.append(kn, vn, tok_slots[i % 8], stream=stream)
        rt.record(e1, stream.cuda_stream)
        torch.cuda.synchronize()
        tok_us = rt.elapsed_ms(e0, e1) * 1e3 / 50
        gen = torch.Generator(device=dev)
        gen.manual_seed(wl.seed)
        nq = 8
        qs = torch.randn((nq, wl.B, wl.Hq, wl.d), generator=gen, device=dev).half()
        bts = [torch.from_numpy(t.block_table).to(dev) for t in tabs]
        max_pages = bts[0].shape[1]
        ctx = torch.tensor(wl.ctx, dtype=torch.int32, device=dev)
        ws = cache.workspace_for(wl.B, max_pages)
        out = torch.empty((wl.B, wl.Hq, wl.d), dtype=torch.float32, device=dev)

        def dec(s):
            K.kvq_decode_attn(cache.handle, qs[s % nq], bts[s % copies], max_pages, ctx, wl.B, 0.0, None, ws,
                              ws.numel(), out, None, stream)

        d_us = _graph_time(dec, steps, stream)
        step_us = None
        if not search:  # the fused append + decode step (default scales): the token at position T
            ctx1 = torch.tensor([T + 1], dtype=torch.int32, device=dev)
            st_slots = [torch.from_numpy(t.slots(0, T, T + 1)).to(dev) for t in tabs]

            def step(s):
                K.kvq_decode_step(cache.handle, kn, vn, st_slots[s % copies], qs[s % nq], bts[s % copies], max_pages,
                                  ctx1, wl.B, 0.0, ws, ws.numel(), out, stream)

            step_us = _graph_time(step, steps, stream)
        assert cache.sync_status() == 0
        res[search] = (min(bulk_ms), tok_us, d_us, step_us)
        del cache
    del kd, vd
    row_bytes = wl.d // 2 + wl.d // 16  # e2m1 codes + E4M3 scales
    kv_bytes = T * wl.Hkv * 2 * row_bytes
    rows = 2 * T * wl.Hkv
    peak, kind = measured_peaks()
    bulk, tok_us, d_us, _ = res[1]
    return {"workload": f"NVFP4 K/V, B=1, 32/8 heads, d=128, context {T}, rotated, ScaleSearch on",
            "decode_us": round(d_us, 2), "decode_gbs": round(kv_bytes / d_us / 1e3, 1),
            "decode_pct_hbm_peak": kv_bytes / d_us / 1e3 / peak, "peak_kind": kind, "cache_bytes": kv_bytes,
            "bits_per_element": row_bytes * 8 / wl.d, "bulk_append_ms": round(bulk, 3),
            "bulk_append_rows_per_s": round(rows / bulk * 1e3, 1), "token_append_us": round(tok_us, 2),
            "no_search": {"bulk_append_ms": round(res[0][0], 3), "token_append_us": round(res[0][1], 2),
                          "decode_us": round(res[0][2], 2), "fused_step_us": round(res[0][3], 2)},
            "steps": steps}


def hqmq_leg(steps: int, T: int = 0):
    """The HQMQ codec at Llama-3-8B layer shape (batch 1, 32/8 heads, d=128,
    context 32768, K and V coded from the raw rows): the bulk append of the
    whole context and a one-token append (8 kv heads, the CTA per row), timed
    with events; the decode replayed in a CUDA graph over four cache copies
    (218 MB, above L2)."""
    import torch

    import quantized_kv_cache_16_b200 as K
    import workloads as W
    wl = W.hqmq(T) if T else W.hqmq()
    T, copies = wl.ctx[0], 4
    dev = torch.device("cuda", torch.cuda.current_device())
    tabs = W.page_table(wl, copies=copies, extra_tokens=8)
    cfg = K.make_config(wl.Hq, wl.Hkv, wl.d, wl.k_fmt, wl.v_fmt, wl.k_group, wl.v_group, wl.clip, wl.rotation_seed,
                        rotate=wl.rotate, num_pages=tabs[0].num_pages)
    cache = K.Cache(cfg)
    kd, vd = W.prefix_kv_device(wl, 0, dev)
    rt = Cudart()
    stream = torch.cuda.Stream()
    slots = [torch.from_numpy(t.slots(0, 0, T)).to(dev) for t in tabs]
    e0, e1 = rt.event(), rt.event()
    bulk_ms = []
    for c in range(copies):
        rt.record(e0, stream.cuda_stream)
        with torch.cuda.stream(stream):
            cache.append(kd, vd, slots[c], stream=stream)
        rt.record(e1, stream.cuda_stream)
        torch.cuda.synchronize()
        bulk_ms.append(rt.elapsed_ms(e0, e1))
    del kd, vd
    # one token (all kv heads) per call, into spare slots of copy 0
    kn, vn = (torch.from_numpy(x).to(dev) for x in W.step_kv(wl, 0))
    tok_slots = [torch.from_numpy(tabs[0].slots(0, T + i, T + i + 1)).to(dev) for i in range(8)]
    with torch.cuda.stream(stream):
        for i in range(3):
            cache.append(kn, vn, tok_slots[i], stream=stream)
    torch.cuda.synchronize()
    n_tok_calls = 50
    rt.record(e0, stream.cuda_stream)
    with torch.cuda.stream(stream):
        for i in range(n_tok_calls):
            cache.append(kn, vn, tok_slots[i % 8], stream=stream)
    rt.record(e1, stream.cuda_stream)
    torch.cuda.synchronize()
    tok_us = rt.elapsed_ms(e0, e1) * 1e3 / n_tok_calls
    gen = torch.Generator(device=dev)
    gen.manual_seed(wl.seed)
    nq = 8
    qs = torch.randn((nq, wl.B, wl.Hq, wl.d), generator=gen, device=dev).half()
    bts = [torch.from_numpy(t.block_table).to(dev) for t in tabs]
    max_pages = bts[0].shape[1]
    ctx = torch.tensor(wl.ctx, dtype=torch.int32, device=dev)
    ws = cache.workspace_for(wl.B, max_pages)
    out = torch.empty((wl.B, wl.Hq, wl.d), dtype=torch.float32, device=dev)

    def dec(s):
        K.kvq_decode_attn(cache.handle, qs[s % nq], bts[s % copies], max_pages, ctx, wl.B, 0.0, None, ws, ws.numel(),
                          out, None, stream)

    d_us = _graph_time(dec, steps, stream)
    assert cache.sync_status() == 0
    row_bytes = wl.d * 5 // 8 + 24  # 20-bit fields + step, mask and two fp16 outlier blocks
    kv_bytes = T * wl.Hkv * 2 * row_bytes
    rows = 2 * T * wl.Hkv
    bulk = min(bulk_ms)
    return {"workload": f"HQMQ K/V, B=1, 32/8 heads, d=128, context {T}, raw rows (no rotation)",
            "decode_us": round(d_us, 2), "decode_gbs": round(kv_bytes / d_us / 1e3, 1), "cache_bytes": kv_bytes,
            "bits_per_element": row_bytes * 8 / wl.d, "bulk_append_ms": round(bulk, 3),
            "bulk_append_rows_per_s": round(rows / bulk * 1e3, 1), "token_append_us": round(tok_us, 2),
            "steps": steps}


LADDER_POLICY = dict(tau_cov=0.995, max_frac=0.05, key_tol=0.02, v_tol=1e-3, rank_tol=0.05, cert_tol=0.02,
                     layer_frac=0.5)


def ladder_leg(steps: int, T: int = 0):
    """Certified decode with the adaptive ladder (kvq_decode_certified, six
    launches) at context 131072 on the needle workload (attention
    concentrated on a sink, six needles and the recent window), replayed in
    a CUDA graph over two cache copies; beside it the quantised decode of the
    same cache, and the whole-call fp16 fallback (rung 4, every head
    recomputed from pinned host rows) timed eagerly over a few calls."""
    import numpy as np
    import torch

    import quantized_kv_cache_16_b200 as K
    import workloads as W
    wl = W.ladder(T) if T else W.ladder()
    T, copies = wl.ctx[0], 2
    dev = torch.device("cuda", torch.cuda.current_device())
    cache, k2, v2, bts, ctx = _tier2_cache(wl, copies)
    nq = 8
    qs = torch.from_numpy(np.stack([W.queries(wl, s) for s in range(nq)])).to(dev)
    max_pages = bts[0].shape[1]
    ws = cache.workspace_for(1, max_pages)
    out = torch.empty((1, wl.Hq, wl.d), dtype=torch.float32, device=dev)
    nb = (T + wl.bound_block - 1) // wl.bound_block
    rep_t = {"k_star": torch.zeros((1, wl.Hkv), dtype=torch.int32, device=dev),
             "flags": torch.zeros((1, wl.Hkv, nb), dtype=torch.uint8, device=dev),
             "bound": torch.zeros((1, wl.Hq), dtype=torch.float32, device=dev),
             "status": torch.zeros((1, wl.Hq), dtype=torch.int32, device=dev)}
    rep = K.kvq_ladder_report(rep_t["k_star"].data_ptr(), rep_t["flags"].data_ptr(), nb, rep_t["bound"].data_ptr(),
                              rep_t["status"].data_ptr())
    stream = torch.cuda.Stream()

    def caller(pol):
        names = ("tau_cov", "max_frac", "key_tol", "v_tol", "rank_tol", "cert_tol", "layer_frac")
        lp = None if pol is None else K.kvq_ladder(*[pol[n] for n in names])

        def call(s):
            if pol is None:
                K.kvq_decode_attn(cache.handle, qs[s % nq], bts[s % copies], max_pages, ctx, 1, 0.0, None, ws,
                                  ws.numel(), out, None, stream)
            else:
                K.kvq_decode_certified(cache.handle, qs[s % nq], bts[s % copies], max_pages, ctx, 1, 0.0, k2, v2, lp,
                                       ws, ws.numel(), out, rep, stream)
        return call

    quant_us = _graph_time(caller(None), steps, stream)
    ladder_us = _graph_time(caller(LADDER_POLICY), steps, stream)
    # rungs 1-2 alone: no ranking check, no bound fallback
    rungs12_us = _graph_time(caller(dict(LADDER_POLICY, rank_tol=math.inf, cert_tol=math.inf)), steps, stream)
    # what the ladder did on each of the nq queries
    kstar, nval, dense = [], [], []
    for s in range(nq):
        caller(LADDER_POLICY)(s)
        torch.cuda.synchronize()
        fl = rep_t["flags"].cpu().numpy()
        kstar.append(rep_t["k_star"].cpu().numpy().mean())
        nval.append(((fl >> 1) & 1).sum(axis=2).mean())
        dense.append(int(((rep_t["status"].cpu().numpy() & K.KVQ_LADDER_HEAD_DENSE) != 0).sum()))
    # rung 4: every head recomputed from the host rows
    layer_pol = dict(LADDER_POLICY, cert_tol=0.0)
    call = caller(layer_pol)
    with torch.cuda.stream(stream):
        call(0)
    torch.cuda.synchronize()
    rt = Cudart()
    e0, e1 = rt.event(), rt.event()
    n_layer = 3
    rt.record(e0, stream.cuda_stream)
    for s in range(n_layer):
        call(s)
    rt.record(e1, stream.cuda_stream)
    torch.cuda.synchronize()
    layer_us = rt.elapsed_ms(e0, e1) * 1e3 / n_layer
    assert int((rep_t["status"].cpu().numpy() & K.KVQ_LADDER_LAYER_DENSE != 0).sum()) == wl.Hq
    assert cache.sync_status() == 0
    row = wl.bound_block * wl.d * 2
    link = int(round((np.mean(kstar) + np.mean(nval)) * wl.Hkv * row))
    return {"workload": f"certified ladder: B=1, 32/8 heads, d=128, context {T}, int8 K / int4 g32 V, 128-token "
                        "blocks, needle attention (sink, six needles, recent window); pinned host fp16 tier 2",
            "policy": LADDER_POLICY, "us": round(ladder_us, 2), "quantised_only_us": round(quant_us, 2),
            "overhead_x": round(ladder_us / quant_us, 2), "no_fallback_us": round(rungs12_us, 2),
            "no_fallback_overhead_x": round(rungs12_us / quant_us, 2),
            "mean_key_blocks_per_kv_head": round(float(np.mean(kstar)), 2),
            "mean_value_blocks_per_kv_head": round(float(np.mean(nval)), 2),
            "mean_heads_dense": round(float(np.mean(dense)), 2), "host_link_bytes": link,
            "layer_fallback_us": round(layer_us, 1), "layer_fallback_host_bytes": T * wl.Hkv * wl.d * 2 * 2,
            "steps": steps, "queries": nq}


def host_cpu():
    """The host's logical CPU count and model name (from /proc/cpuinfo)."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return os.cpu_count() or 1, model


def cpu_leg(wk: Workload, n_steps: int):
    """The CPU oracle on a bounded sample of the same steps: one thread, then
    its (sequence, kv head) loop on all cores (OpenMP)."""
    import oracle as O
    wl = wk.wl
    ocfg = O.make_config(**wk.cfg_kw)
    pool = O.new_pool(ocfg)
    k, v = wk.W.prefix_kv(wl, 0)
    O.append(ocfg, pool, k, v, wk.tabs[0].slots(0, 0, wk.T))
    nproc, model = host_cpu()

    def timed(threads, steps, first):
        used = O.set_threads(threads)
        times, nbytes = [], 0
        for u in range(first, first + steps):
            t = time.perf_counter()
            O.append(ocfg, pool, wk.h_newk[u], wk.h_newv[u], wk.h_slots[0, u:u + 1])
            O.decode(ocfg, pool, wk.h_q[u], wk.tabs[0].block_table, [int(wk.h_ctx[u])])
            times.append(time.perf_counter() - t)
            nbytes += int(wk.h_ctx[u]) * kv_bytes_per_token(wl.d, wl.Hkv)
        return nbytes, sum(times), min(used, wl.B * wl.Hkv)

    nb1, sec1, _ = timed(1, n_steps, 0)
    nbn, secn, used = timed(nproc, 2 * n_steps, n_steps)
    O.set_threads(1)
    return {"value": round(nb1 / sec1 / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "us_per_step": 1e6 * sec1 / n_steps, "host": {"nproc": nproc, "cpu_model": model},
            "sample": f"{n_steps} of the window's steps (append 1 token + fp64 decode over the full context), "
                      f"C oracle -O2 single thread, {sec1:.1f} s",
            "all_cores": {"value": round(nbn / secn / 1e9, 4), "unit": "GB/s", "cores": used,
                          "us_per_step": 1e6 * secn / (2 * n_steps),
                          "sample": f"the next {2 * n_steps} steps, OpenMP over the (sequence, kv head) pairs: "
                                    f"{used} threads busy of {nproc} ({wl.B * wl.Hkv} pairs), {secn:.1f} s"}}


def run_reference(args, dist: Dist):
    """Reference arm: the CPU oracle timed on the host on the same workload."""
    if dist.rank != 0:
        return
    import numpy as np

    import oracle as O
    import workloads as W
    wl = W.llama()
    T = wl.ctx[0]
    tab = W.page_table(wl, extra_tokens=wl.steps)[0]
    ocfg = O.make_config(wl.Hq, wl.Hkv, wl.d, wl.k_fmt, wl.v_fmt, wl.k_group, wl.v_group, wl.clip,
                         wl.rotation_seed, num_pages=tab.num_pages)
    pool = O.new_pool(ocfg)
    k, v = W.prefix_kv(wl, 0)
    O.append(ocfg, pool, k, v, tab.slots(0, 0, T))
    per_tok = kv_bytes_per_token(wl.d, wl.Hkv)

    def step(u):
        nk, nv = W.step_kv(wl, u)
        O.append(ocfg, pool, nk, nv, np.array([tab.slot(0, T + u)], np.int32))
        O.decode(ocfg, pool, W.queries(wl, u), tab.block_table, [T + u + 1])
        return (T + u + 1) * per_tok

    # the oracle takes seconds per step: a bounded sample of the K steps, its
    # (sequence, kv head) loop spread over the host's cores
    nproc, model = host_cpu()
    used = min(O.set_threads(nproc), wl.B * wl.Hkv)
    n_w = min(args.warmup, 1)
    n_t = max(1, min(args.steps, 8))
    for u in range(n_w):
        step(u)
    t = time.perf_counter()
    nbytes = sum(step(u % wl.steps) for u in range(n_t))
    sec = time.perf_counter() - t
    val = nbytes / sec / 1e9
    sample = (f"{n_t} steps of the 100-step window (append 1 token + fp64 decode), C oracle -O2, OpenMP over "
              f"the {wl.B * wl.Hkv} (sequence, kv head) pairs on {used} of {nproc} threads ({model}), {sec:.1f} s")
    line = {"impl": "reference", "metric": METRIC, "value": round(val, 4), "unit": "GB/s", "n_gpus": dist.world,
            "steps": n_t, "warmup": n_w, "ms_per_step": 1e3 * sec / n_t, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32 codec / f64 attention", "data": "synthetic",
            "config": {"workload": workload_name(T, wl.steps), "global_batch": dist.world, "seq_len": T,
                       "parallelism": f"host CPU oracle, {used} threads"},
            "cpu_baseline": {"value": round(val, 4), "unit": "GB/s", "cores": used, "kind": "oracle",
                             "sample": sample, "host": {"nproc": nproc, "cpu_model": model}},
            "e2e": {"value": round(val, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    dist = Dist()
    if args.leg:
        import torch
        torch.cuda.set_device(0)
        leg = {"paged": paged_leg, "certified": certified_leg, "ladder": ladder_leg, "windows": windows_leg, "hqmq": hqmq_leg,
               "nvfp4": nvfp4_leg, "contexts": contexts_leg, "bitrev": bitrev_leg, "append": lambda steps, ctx: append_leg(),
               "e2e": lambda steps, ctx: e2e_leg(Workload(dist), steps, torch.cuda.Stream(), dist)}[args.leg]
        print(json.dumps(leg(args.steps, args.ctx)), flush=True)
        return
    if args.impl == "reference":
        run_reference(args, dist)
    else:
        run_ours(args, dist)


if __name__ == "__main__":
    main()
