#!/usr/bin/env python3
"""Decode-attention throughput on B200: one JSON line on rank 0.

A step is one decode step of one layer for the whole batch: for the c4a
layer (the default workload) dsv4kv_index_topk followed by
dsv4kv_sparse_decode; for the c128a layer dsv4kv_dense_decode.  The caches
are resident in HBM (a KV cache is state, not a per-step input); the steps
cycle through enough cache replicas that the bytes read between two reads of
one replica exceed twice the L2, so every step streams from DRAM.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun every rank runs its own batch (weak scaling, no collective on
the data path); the time is the max over ranks.  `--impl reference` times the
float64 CPU oracle on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attn steps/s per layer type; HBM GB/s vs ~8 TB/s peak, 1 B200"
WORKLOADS = {
    # name: (kind, batch, t, heads, main_fmt, index_fmt)
    "c4a_b32": ("c4a", 32, 131072, 64, 0, 0),
    "c128a_b8": ("c128a", 8, 131072, 64, 0, 0),
    "c128a_b32": ("c128a", 32, 131072, 64, 0, 0),
    "q_c4a_fp8": ("c4a", 64, 262144, 64, 1, 2),
    "q_c4a_fp4": ("c4a", 64, 262144, 64, 2, 2),
    "q_c128a_fp8": ("c128a", 64, 262144, 64, 1, 0),
    "q_c128a_fp4": ("c128a", 64, 262144, 64, 2, 0),
    "q_c4a_fp8rope": ("c4a", 64, 262144, 64, 3, 2),
    "q_c128a_fp8rope": ("c128a", 64, 262144, 64, 3, 0),
    # a CSA2 Reindex layer: top-512 re-indexed inside the 2048-entry pool a Full
    # layer built (the pool size is a reading; the pages give none)
    "c4a_b32_reindex": ("c4a", 32, 131072, 64, 0, 0, 2048),
    # one c4a layer of the 61-layer stack on its own (one 1M-token sequence)
    "c4a_b1_t1m": ("c4a", 1, 1 << 20, 64, 0, 0),
    "c128a_b1_t1m": ("c128a", 1, 1 << 20, 64, 0, 0),
    # paged caches of a ragged batch: every sequence has its own length (uniform in
    # [t/2, t], seeded), its caches in 256-row pages of shared pools, pages shuffled
    "c4a_b32_paged": ("c4a", 32, 131072, 64, 0, 0, 0, "paged"),
}
FMT_NAME = {0: "bf16", 1: "fp8", 2: "fp4", 3: "fp8+bf16rope"}
L2_BYTES = 126 * 2 ** 20
# DRAM bytes (read + write) per launch of the dominant kernel, from one ncu
# capture of that kernel in this workload (profiles/ holds the summary and the
# command); cleared whenever the kernel changes
TRAFFIC = {("c4a_b32", "index_score_stream<bf16>"): 274427392}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d.get("bf16_tflops", 1671.7)), "measured"
    return 6650.0, 1590.0, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    def __init__(self, dev_index: int, period_s: float = 0.01):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period, self._stop, self._t = period_s, threading.Event(), None
        try:
            import pynvml as N
            N.nvmlInit()
            self.N, self.h = N, N.nvmlDeviceGetHandleByIndex(dev_index)
            self.max_mhz = N.nvmlDeviceGetMaxClockInfo(self.h, N.NVML_CLOCK_SM)
        except Exception:
            self.N = None

    _NAMES = {0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
              0x80: "hw_power_brake_slowdown", 0x4: "sw_power_cap", 0x1: "gpu_idle", 0x2: "applications_clocks_setting"}

    def _sample(self):
        N = self.N
        self.samples.append(N.nvmlDeviceGetClockInfo(self.h, N.NVML_CLOCK_SM))
        try:
            r = N.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            r = N.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        for bit, name in self._NAMES.items():
            if r & bit and name != "gpu_idle":
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def __enter__(self):
        if self.N:
            self._sample()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self.N:
            self._stop.set()
            self._t.join()
            self._sample()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------ our arm
ROW_BYTES = {0: 1024, 1: 516, 2: 288, 3: 580}  # one 512-channel cache row: bf16, fp8 + scale, fp4 + scales,
                                              # fp8 body + bf16 rotary channels + scale
KEY_BYTES = {0: 256, 2: 72}               # one 128-channel indexer key: bf16, fp4 + scales


def step_bytes(kind, batch, t, main_fmt, index_fmt, k=512, window=128, pool=0):
    """Algorithmic bytes one step reads from one cache replica: indexer keys
    (c4a; only the pool's keys for a Reindex layer) + the attended rows.
    Queries and outputs are excluded."""
    n = (t - window) // (4 if kind == "c4a" else 128)
    rows = (k + window) if kind == "c4a" else (n + window)
    b = batch * rows * ROW_BYTES[main_fmt]
    if kind == "c4a":
        b += batch * (pool if pool else n) * KEY_BYTES[index_fmt]
    return b


def replicas_for(kind, batch, t, main_fmt, index_fmt, at_least, pool=0, l2_factor=4):
    """Cache replicas the timed steps cycle through: together they hold at
    least `l2_factor` times the L2 (4 for every timed run), so every step
    streams its rows from DRAM."""
    per = step_bytes(kind, batch, t, main_fmt, index_fmt, pool=pool)
    return max(at_least, -(-l2_factor * L2_BYTES // per))


PAGE_ROWS = 256


def torch_empty_like(t):
    import torch
    return torch.empty_like(t)


def ragged_lengths(batch, t, seed):
    """Per-sequence query positions of the ragged workloads: uniform in [t/2, t]."""
    rng = np.random.default_rng(seed)
    return rng.integers(t // 2, t + 1, size=batch).astype(np.int64)


class PagedLayer:
    """A c4a layer over paged caches of a ragged batch (R replicas of pools and
    shuffled block tables): one step is dsv4kv_index_topk_paged +
    dsv4kv_sparse_decode_paged."""

    def __init__(self, batch, t, heads, seed, replicas, layer_id=0):
        import torch
        import compressed_sparse_kv_b200 as K
        import datagen.gpu as G
        from datagen import workloads as WL
        self.K, self.torch = K, torch
        self.kind, self.batch, self.t, self.heads = "c4a", batch, t, heads
        self.main_fmt, self.index_fmt, self.pool = 0, 0, 0
        self.window, self.k = 128, 512
        self.t_host = ragged_lengths(batch, t, seed)
        self.t_max = int(t)
        self.n_seq = np.maximum(0, (self.t_host - self.window) // 4)
        self.n = int(self.n_seq.max())
        dev = "cuda"
        rng = np.random.default_rng(seed + 1)

        def tables(counts, most):
            # `most`: the rows a sequence of length t_max may have (the table's row pitch covers them)
            need = (counts + PAGE_ROWS - 1) // PAGE_ROWS
            perm = rng.permutation(int(need.sum())).astype(np.int32)
            tab = np.full((batch, max(1, (most + PAGE_ROWS - 1) // PAGE_ROWS)), -1, np.int32)
            o = 0
            for b, m in enumerate(need):
                tab[b, :m] = perm[o:o + m]
                o += m
            return torch.from_numpy(tab).to(dev), int(need.sum())

        w_seq = np.minimum(self.t_host, self.window)
        self.reps = []
        for r in range(replicas):
            keys = WL.keys_for(seed, 1000 * r + layer_id)
            n_most = max(0, (self.t_max - self.window) // 4)
            ct, cp = tables(self.n_seq, n_most)
            kt, kp = tables(self.n_seq, n_most)
            wt, wp = tables(w_seq, self.window)
            comp = G.normal_bf16_(torch.empty(cp * PAGE_ROWS, 512, dtype=torch.bfloat16, device=dev), keys["comp"])
            win = G.normal_bf16_(torch.empty(wp * PAGE_ROWS, 512, dtype=torch.bfloat16, device=dev), keys["win"])
            kidx = G.int_bf16_(torch.empty(kp * PAGE_ROWS, 128, dtype=torch.bfloat16, device=dev), keys["kidx"])
            self.reps.append({"comp": K.PagedCache(0, comp, ct, PAGE_ROWS), "win": K.PagedCache(0, win, wt, PAGE_ROWS),
                              "kidx": K.PagedCache(0, kidx, kt, PAGE_ROWS, dim=128)})
        keys = WL.keys_for(seed, layer_id)
        self.t_seq = torch.from_numpy(self.t_host).to(dev)
        self.q = G.normal_bf16_(torch.empty(batch, heads, 512, dtype=torch.bfloat16, device=dev), keys["q"])
        self.qidx = G.int_bf16_(torch.empty(batch, 128, dtype=torch.bfloat16, device=dev), keys["qidx"])
        self.idx = torch.empty(batch, self.k, dtype=torch.int32, device=dev)
        self.cnt = torch.empty(batch, dtype=torch.int32, device=dev)
        self.out = torch.empty(batch, heads, 512, dtype=torch.bfloat16, device=dev)
        self.ws_idx = K.new_workspace(K.lib().dsv4kv_index_topk_paged_workspace_bytes(batch, self.t_max, 128, 4, 512))
        self.ws_dec = K.new_workspace(K.lib().dsv4kv_sparse_decode_paged_workspace_bytes(batch, heads, 512, 512, 128))
        torch.cuda.synchronize()

    def twin(self):
        """The same layer (same caches) with its own per-step buffers and workspaces."""
        import copy
        t = copy.copy(self)
        t.idx, t.cnt, t.out = torch_empty_like(self.idx), torch_empty_like(self.cnt), torch_empty_like(self.out)
        t.ws_idx, t.ws_dec = self.K.new_workspace(self.ws_idx.numel()), self.K.new_workspace(self.ws_dec.numel())
        return t

    def alg_bytes(self):
        sel = np.minimum(self.n_seq, self.k)
        win = np.minimum(self.t_host, self.window)
        return int((self.n_seq * KEY_BYTES[0]).sum() + ((sel + win) * ROW_BYTES[0]).sum())

    def index_bytes(self):
        return int((self.n_seq * KEY_BYTES[0]).sum()) + self.batch * 256

    def flops(self):
        return int(((np.minimum(self.n_seq, self.k) + np.minimum(self.t_host, self.window)) * 4 * self.heads * 512).sum())

    def launches_per_step(self):
        return 4

    def index(self, r, qidx=None):
        self.K.index_topk_paged(self.qidx if qidx is None else qidx, self.reps[r]["kidx"], self.t_seq, self.t_max,
                                self.k, idx_out=self.idx, count_out=self.cnt, ws=self.ws_idx)

    def index_score(self, r):
        self.index(r)

    def index_select(self):
        pass

    def decode(self, r, q=None, out=None):
        rep = self.reps[r]
        self.K.sparse_decode_paged(self.q if q is None else q, rep["comp"], rep["win"], self.idx, self.t_seq,
                                   self.t_max, out=self.out if out is None else out, ws=self.ws_dec)

    def step(self, r):
        self.index(r)
        self.decode(r)


class Layer:
    """One layer's resident caches (R replicas) and per-step buffers on the GPU."""

    def __init__(self, kind, batch, t, heads, seed, replicas, main_fmt=0, index_fmt=0, layer_id=0, shared=None,
                 pool=0):
        import torch
        import compressed_sparse_kv_b200 as K
        import datagen.gpu as G
        from datagen import workloads as WL
        self.K, self.torch = K, torch
        self.kind, self.batch, self.t, self.heads = kind, batch, t, heads
        self.main_fmt, self.index_fmt = main_fmt, index_fmt
        self.window, self.k = 128, 512
        self.pool = pool  # > 0: a Reindex layer over a pool of this many entries
        stride = 4 if kind == "c4a" else 128
        self.n = (t - self.window) // stride
        dev = "cuda"

        def rows(key, count):
            x = G.normal_bf16_(torch.empty(batch, count, 512, dtype=torch.bfloat16, device=dev), key)
            if main_fmt == 0:
                return K.Cache(0, x)
            codes, scales = K.quantize(x, main_fmt)
            del x
            return K.Cache(main_fmt, codes, scales)

        self.reps = []
        for r in range(replicas):
            keys = WL.keys_for(seed, 1000 * r + layer_id)
            rep = {"comp": rows(keys["comp"], self.n), "win": rows(keys["win"], self.window)}
            if kind == "c4a":
                if index_fmt == 0:
                    kt = G.int_bf16_(torch.empty(batch, self.n, 128, dtype=torch.bfloat16, device=dev), keys["kidx"])
                    rep["kidx"] = K.Cache(0, kt, None, 128)
                else:
                    codes = torch.empty(batch, self.n, 64, dtype=torch.uint8, device=dev)
                    scales = torch.empty(batch, self.n, 8, dtype=torch.uint8, device=dev)
                    G.fp4_index_keys_(codes, scales, keys["kidx_fp4"])
                    rep["kidx"] = K.Cache(2, codes, scales, 128)
            self.reps.append(rep)
        if pool:
            # the pool: the top-`pool` entries of each replica's keys under another
            # layer's query (the Full layer of the group), built once
            qf = G.int_bf16_(torch.empty(batch, 128, dtype=torch.bfloat16, device=dev),
                             WL.keys_for(seed, 5000 + layer_id)["qidx"])
            for rep in self.reps:
                rep["pool"], _ = K.index_topk(qf, rep["kidx"], self.n, pool)
            self.ws_pool = K.new_workspace(16)
        keys = WL.keys_for(seed, layer_id)
        self.q = G.normal_bf16_(torch.empty(batch, heads, 512, dtype=torch.bfloat16, device=dev), keys["q"])
        # the inputs are generated on the current stream; the timed work runs on its own stream
        self.qidx = G.int_bf16_(torch.empty(batch, 128, dtype=torch.bfloat16, device=dev), keys["qidx"])
        sh = shared if shared is not None else {}
        self.idx = sh.setdefault("idx", torch.empty(batch, self.k, dtype=torch.int32, device=dev))
        self.cnt = sh.setdefault("cnt", torch.empty(batch, dtype=torch.int32, device=dev))
        self.out = torch.empty(batch, heads, 512, dtype=torch.bfloat16, device=dev)
        if kind == "c4a":
            need_i = K.index_topk_workspace_bytes(batch, self.n, self.k)
            need_d = K.sparse_decode_workspace_bytes(batch, heads, self.k, self.window)
            if "ws_idx" not in sh or sh["ws_idx"].numel() < need_i:
                sh["ws_idx"] = K.new_workspace(need_i)
            self.ws_idx = sh["ws_idx"]
        else:
            need_d = K.dense_decode_workspace_bytes(batch, heads, self.n, self.window)
        if "ws_dec" not in sh or sh["ws_dec"].numel() < need_d:
            sh["ws_dec"] = K.new_workspace(need_d)
        self.ws_dec = sh["ws_dec"]
        torch.cuda.synchronize()  # inputs and zeroed workspaces are complete before any other stream uses them

    def twin(self):
        """The same layer (same caches) with its own per-step buffers and workspaces."""
        import copy
        t = copy.copy(self)
        t.idx, t.cnt, t.out = torch_empty_like(self.idx), torch_empty_like(self.cnt), torch_empty_like(self.out)
        t.ws_dec = self.K.new_workspace(self.ws_dec.numel())
        if self.kind == "c4a":
            t.ws_idx = self.K.new_workspace(self.ws_idx.numel())
        if self.pool:
            t.ws_pool = self.K.new_workspace(self.ws_pool.numel())
        return t

    # algorithmic bytes of one step: indexer keys + rows read (queries/outputs excluded)
    def alg_bytes(self):
        return step_bytes(self.kind, self.batch, self.t, self.main_fmt, self.index_fmt, self.k, self.window, self.pool)

    def index_bytes(self):
        return self.batch * (self.pool or self.n) * KEY_BYTES[self.index_fmt] + self.batch * 256

    def flops(self):
        rows = (self.k + self.window) if self.kind == "c4a" else (self.n + self.window)
        return self.batch * rows * 4 * self.heads * 512

    def launches_per_step(self):
        if self.kind != "c4a":
            return 2
        return 3 if self.pool else 4

    def index(self, r, qidx=None):
        qidx = self.qidx if qidx is None else qidx
        if self.pool:
            self.K.index_topk_pool(qidx, self.reps[r]["kidx"], self.n, self.reps[r]["pool"], self.k,
                                   idx_out=self.idx, count_out=self.cnt, ws=self.ws_pool)
            return
        self.K.index_topk(qidx, self.reps[r]["kidx"], self.n, self.k, idx_out=self.idx, count_out=self.cnt,
                          ws=self.ws_idx)

    # the same call in its two steps (dsv4kv_index_score; dsv4kv_index_select);
    # a Reindex layer's one call (dsv4kv_index_topk_pool) stands in the first
    def index_score(self, r):
        if self.pool:
            self.K.index_topk_pool(self.qidx, self.reps[r]["kidx"], self.n, self.reps[r]["pool"], self.k,
                                   idx_out=self.idx, count_out=self.cnt, ws=self.ws_pool)
            return
        self.K.index_score(self.qidx, self.reps[r]["kidx"], self.n, self.k, self.ws_idx)

    def index_select(self):
        if self.pool:
            return
        self.K.index_select(self.batch, self.n, self.k, self.idx, self.cnt, self.ws_idx)

    def decode(self, r, q=None, out=None):
        rep = self.reps[r]
        K = self.K
        q = self.q if q is None else q
        out = self.out if out is None else out
        if self.kind == "c4a":
            K.sparse_decode(q, rep["comp"], rep["win"], self.idx, self.n, self.window, self.t, out=out, ws=self.ws_dec)
        else:
            K.dense_decode(q, rep["comp"], rep["win"], self.n, self.window, self.t, out=out, ws=self.ws_dec)

    def step(self, r):
        if self.kind == "c4a":
            self.index(r)
        self.decode(r)


def time_stack(steps, warmup, seed, dist_max):
    """The 61-layer stack at t = 2^20, B = 1 (layer l: c128a if l is even,
    c4a if odd), one decode step = every layer once, captured as one graph."""
    import torch
    from datagen import workloads as WL
    shared = {}
    layers = [Layer(WL.stack_layer_kind(l), 1, 1 << 20, 64, seed, 1, layer_id=l, shared=shared)
              for l in range(WL.STACK_LAYERS)]
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        for _ in range(max(warmup, 1)):
            for L in layers:
                L.step(0)
    stream.synchronize()
    ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2 * len(layers) + 1)]

    def capture(events):
        # events: event nodes around every layer's calls (each one costs the
        # programmatic-launch overlap at its boundary), for the per-call times
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            if events:
                ev[0].record(stream)
            for i, L in enumerate(layers):
                if L.kind == "c4a":
                    L.index(0)
                if events:
                    ev[2 * i + 1].record(stream)
                L.decode(0)
                if events:
                    ev[2 * i + 2].record(stream)
        return g

    g = capture(False)       # the timed step
    g_inst = capture(True)   # the same step with event nodes, for the breakdown
    with torch.cuda.stream(stream):
        for _ in range(3):
            g.replay()
        g_inst.replay()
    stream.synchronize()
    # one instrumented replay for the per-call breakdown
    inst_start, inst_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        inst_start.record(stream)
        g_inst.replay()
        inst_stop.record(stream)
    stream.synchronize()
    inst_ms = inst_start.elapsed_time(inst_stop)
    idx_ms = sum(ev[2 * i].elapsed_time(ev[2 * i + 1]) for i, L in enumerate(layers) if L.kind == "c4a")
    c4a_dec = sum(ev[2 * i + 1].elapsed_time(ev[2 * i + 2]) for i, L in enumerate(layers) if L.kind == "c4a")
    c128a_ms = sum(ev[2 * i].elapsed_time(ev[2 * i + 2]) for i, L in enumerate(layers) if L.kind == "c128a")
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist_barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        start.record(stream)
        for _ in range(steps):
            g.replay()
        stop.record(stream)
    stop.synchronize()
    ms = dist_max(start.elapsed_time(stop)) / steps
    alg = sum(L.alg_bytes() for L in layers)
    n4 = sum(1 for L in layers if L.kind == "c4a")
    res = {"workload": "61-layer stack decode step B=1 t=1048576 H=64 (30 c4a + 31 c128a), bf16, one CUDA graph",
           "steps_per_s": round(1e3 / ms, 2), "ms_per_step": round(ms, 4), "alg_bytes_per_step": alg,
           "hbm_gbs": round(alg / (ms * 1e-3) / 1e9, 1),
           "c4a_layer_us": round((idx_ms + c4a_dec) / n4 * 1e3, 2),
           "c4a_index_us": round(idx_ms / n4 * 1e3, 2),
           "c128a_layer_us": round(c128a_ms / (len(layers) - n4) * 1e3, 2),
           "breakdown_note": "per-layer times from a replay with event nodes between the calls "
                             f"({round(inst_ms, 4)} ms per step); the timed step has none",
           "launches_per_step": sum(L.launches_per_step() for L in layers)}
    del g, g_inst, layers
    torch.cuda.empty_cache()
    return res


def time_bulk(seed):
    """Bulk throughput of the c4a / c128a compressors and the fp8 / fp4 quantiser;
    per-token time of the incremental cache maintenance."""
    import torch
    import compressed_sparse_kv_b200 as K
    import datagen as D
    import datagen.gpu as G
    out = {}
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    raw = G.normal_bf16_(torch.empty(8, 131072, 512, dtype=torch.bfloat16, device="cuda"), D.stream_key(seed, D.TID_RAW_S))
    for kind, st, k in (("c4a", 4, 8), ("c128a", 128, 128)):
        w = torch.from_numpy(D.compress_weights(seed, 0, k, 512)).cuda()
        n = K.compress_entries(131072, 128, st)
        o = torch.empty(8, n, 512, dtype=torch.bfloat16, device="cuda")
        for _ in range(3):
            K.compress(raw, w, st, 128, out=o)
        s.record()
        for _ in range(10):
            K.compress(raw, w, st, 128, out=o)
        e.record()
        e.synchronize()
        ms = s.elapsed_time(e) / 10
        byts = raw.numel() * 2 + o.numel() * 2
        out[f"compress_{kind}"] = {"workload": f"B=8 t=131072 -> {n} entries, bf16 out", "us": round(ms * 1e3, 1),
                                   "gbs": round(byts / (ms * 1e-3) / 1e9, 1)}
    x = raw.view(-1, 512)[: 64 * 2175]
    for fmt, name, rb in ((1, "fp8", 516), (2, "fp4", 288)):
        codes, scales = K.quantize(x, fmt)
        s.record()
        for _ in range(10):
            K.quantize(x, fmt, codes, scales)
        e.record()
        e.synchronize()
        ms = s.elapsed_time(e) / 10
        byts = x.shape[0] * (1024 + rb)
        out[f"quantize_{name}"] = {"workload": f"{x.shape[0]} rows x 512 bf16", "us": round(ms * 1e3, 1),
                                   "gbs": round(byts / (ms * 1e-3) / 1e9, 1)}
    # incremental maintenance (dsv4kv_append) per decoded token at t = 131072:
    # B = 32 for c4a (an entry every 4 tokens), B = 8 for c128a (every 128);
    # the mean over a run of consecutive tokens, one CUDA graph
    for kind, st, k, bsz in (("c4a", 4, 8, 32), ("c128a", 128, 128, 8)):
        w = torch.from_numpy(D.compress_weights(seed, 0, k, 512)).cuda()
        ring = torch.zeros(bsz, 128 + k, 512, dtype=torch.bfloat16, device="cuda")
        win = torch.zeros(bsz, 128, 512, dtype=torch.bfloat16, device="cuda")
        comp = torch.zeros(bsz, K.compress_entries(131072 + 256, 128, st) + 1, 512, dtype=torch.bfloat16, device="cuda")
        x = raw[:, 0].repeat(bsz // 8, 1).contiguous()  # [bsz][512] states
        t0, steps = 131072, 256
        stream = torch.cuda.Stream()
        with torch.cuda.stream(stream):
            for i in range(steps):
                K.append(x, w, t0 + i, st, 128, ring, win, comp)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(steps):
                K.append(x, w, t0 + i, st, 128, ring, win, comp)
        with torch.cuda.stream(stream):
            g.replay()
            s.record(stream)
            g.replay()
            e.record(stream)
        e.synchronize()
        emits = sum(1 for i in range(steps) if (t0 + i + 1 - 128) % st == 0)
        out[f"append_{kind}"] = {"workload": f"B={bsz}, {steps} consecutive tokens from t={t0} ({emits} entries emitted)",
                                 "us_per_token": round(s.elapsed_time(e) * 1e3 / steps, 2)}
        del g
    del raw
    torch.cuda.empty_cache()
    return out


def time_layer(layer, steps, warmup, dist_max, dev_index, sample_clocks):
    """Device time of exactly `steps` steps.  All steps (replicas alternating)
    are captured into one CUDA graph and timed with events on the launching
    stream around its replay.  A second graph of the same steps with event
    nodes between the calls (which cost the programmatic-launch overlap at
    each event) gives the per-call device times."""
    torch = layer.torch
    R = len(layer.reps)
    stream = torch.cuda.Stream()
    # one full cycle over the replicas first, so no replica is still in L2
    # from its creation; every graph then continues the cycle where the
    # previous one stopped
    n_eager = max(warmup, R)
    with torch.cuda.stream(stream):
        for i in range(n_eager):
            layer.step(i % R)
    stream.synchronize()
    # external=True: records inside the capture become event nodes of the graph
    ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)] for _ in range(steps)]

    def capture(first, n_steps, events):
        # events: step start | after index_score | after index_select | after decode
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(n_steps):
                r = (first + i) % R
                if events:
                    events[i][0].record(stream)
                if layer.kind == "c4a":
                    layer.index_score(r)
                if events:
                    events[i][1].record(stream)
                if layer.kind == "c4a":
                    layer.index_select()
                if events:
                    events[i][2].record(stream)
                layer.decode(r)
                if events:
                    events[i][3].record(stream)
        return g

    n_warm = max(warmup, 1)
    g_warm = capture(n_eager, n_warm, None)
    g_main = capture(n_eager + n_warm, steps, None)
    g_inst = capture(n_eager + n_warm + steps, steps, ev)
    # every graph is launched once before it is timed (its first launch also
    # uploads it to the device, a one-time cost of some milliseconds)
    with torch.cuda.stream(stream):
        g_warm.replay()
        g_main.replay()
        g_inst.replay()
        g_warm.replay()
    stream.synchronize()
    dist_barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(dev_index) if sample_clocks else None
    if sampler:
        sampler.__enter__()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record(stream)
        g_main.replay()
        stop.record(stream)
    torch.cuda.synchronize()
    if sampler:
        sampler.__exit__()
    dist_barrier()
    total_ms = start.elapsed_time(stop)
    # four more timed replays of the same graph (not part of `value`): their
    # median with the first is reported beside it
    reps_ms = [total_ms]
    for _ in range(4):
        with torch.cuda.stream(stream):
            start.record(stream)
            g_main.replay()
            stop.record(stream)
        stop.synchronize()
        reps_ms.append(start.elapsed_time(stop))
    with torch.cuda.stream(stream):
        g_inst.replay()
    torch.cuda.synchronize()
    score_ms = [e[0].elapsed_time(e[1]) for e in ev] if layer.kind == "c4a" else [0.0]
    select_ms = [e[1].elapsed_time(e[2]) for e in ev] if layer.kind == "c4a" else [0.0]
    dec_ms = [e[2].elapsed_time(e[3]) for e in ev]
    total_ms = dist_max(total_ms)
    del g_warm, g_main, g_inst
    return {"total_ms": total_ms, "median5_ms": float(np.median(reps_ms)),
            "score_ms": float(np.mean(score_ms)), "select_ms": float(np.mean(select_ms)),
            "index_ms": float(np.mean(score_ms) + np.mean(select_ms)), "decode_ms": float(np.mean(dec_ms)),
            "clocks": sampler.summary() if sampler else None}


def time_e2e(layer, steps):
    """Same steps through the public API with host buffers: every step copies
    its queries (and, for c4a, its indexer query) from pinned host memory to
    the device, makes the library calls and copies its output back to pinned
    host memory, all inside the timed region.

    The steps run as a three-stage pipeline over three streams (upload,
    compute, download), in chunks of C steps with two sets of C device and
    pinned host buffers: the uploads of chunk c (one copy per step) overlap
    the calls of chunk c-1, every step's download follows its calls, and
    events order every reuse of a buffer.  The compute stream waits on the
    other streams once per chunk: a cross-stream dependency in front of a
    step's first kernel costs the programmatic-launch overlap with the
    previous step's last kernel.  The whole pipeline of `steps` steps
    (copies, calls and event dependencies) is captured once into one CUDA
    graph and replayed, the way a serving loop launches its decode
    iterations without a host round trip per kernel.  The eager figure issues
    the same copies and calls from Python step by step.  Returns (graph ms,
    eager ms, H2D bytes per step, D2H bytes per step)."""
    torch = layer.torch
    R = len(layer.reps)
    C = 3                                                  # steps per chunk
    NB = 2 * C                                             # buffer sets: two chunks' worth
    lanes = [layer.twin() for _ in range(NB)]             # own output buffers and workspaces per set
    q_host = [layer.q.cpu().pin_memory() for _ in range(NB)]
    qi_host = [layer.qidx.cpu().pin_memory() for _ in range(NB)]
    out_host = [torch.empty(layer.out.shape, dtype=layer.out.dtype).pin_memory() for _ in range(NB)]
    q_dev = [torch.empty_like(layer.q) for _ in range(NB)]
    qi_dev = [torch.empty_like(layer.qidx) for _ in range(NB)]
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]       # per chunk parity: the chunk's inputs are up
    ev_comp = [torch.cuda.Event() for _ in range(2)]     # the chunk's calls are done (its inputs read)
    ev_out = [torch.cuda.Event() for _ in range(2)]      # the chunk's outputs are down
    ev_step = [torch.cuda.Event() for _ in range(NB)]    # one step's calls are done

    def calls(j, r):
        L = lanes[j]
        if L.kind == "c4a":
            L.index(r, qidx=qi_dev[j])
        L.decode(r, q=q_dev[j])

    for j in range(NB):
        for r in range(R):
            with torch.cuda.stream(s_comp):
                calls(j, r)                            # every buffer and kernel set up before capture
    torch.cuda.synchronize()

    def pipeline(head):
        """Issues the steps; `head` is the stream they start after (and end on)."""
        fork = torch.cuda.Event()
        fork.record(head)
        for s in (s_in, s_comp, s_out):
            s.wait_event(fork)
        for c in range((steps + C - 1) // C):
            cp = c % 2
            chunk = range(c * C, min(steps, (c + 1) * C))
            if c >= 2:
                s_in.wait_event(ev_comp[cp])           # chunk c - 2's calls have read these input sets
            with torch.cuda.stream(s_in):
                for i in chunk:
                    j = cp * C + i % C
                    q_dev[j].copy_(q_host[j], non_blocking=True)
                    if layer.kind == "c4a":
                        qi_dev[j].copy_(qi_host[j], non_blocking=True)
            ev_in[cp].record(s_in)
            s_comp.wait_event(ev_in[cp])
            if c >= 2:
                s_comp.wait_event(ev_out[cp])          # chunk c - 2's outputs have left these sets
            for i in chunk:
                j, r = cp * C + i % C, i % R
                with torch.cuda.stream(s_comp):
                    calls(j, r)
                ev_step[j].record(s_comp)
                s_out.wait_event(ev_step[j])
                with torch.cuda.stream(s_out):
                    out_host[j].copy_(lanes[j].out, non_blocking=True)
            ev_comp[cp].record(s_comp)
            ev_out[cp].record(s_out)
        for s in (s_in, s_comp, s_out):                # join every stream back into the head
            e = torch.cuda.Event()
            e.record(s)
            head.wait_event(e)

    head = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=head):
        pipeline(head)
    torch.cuda.synchronize()

    def timed(fn):
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        start.record(head)
        fn()
        stop.record(head)
        stop.synchronize()
        return start.elapsed_time(stop)

    def replay():
        with torch.cuda.stream(head):
            g.replay()

    # warm-up: the first launch uploads the graph, and the first passes of the
    # copies over fresh pinned buffers run measurably slower (92-100 us per
    # c4a B=32 step against 85 us from the fourth pass on)
    for _ in range(4):
        replay()
    torch.cuda.synchronize()
    eager_ms = timed(lambda: pipeline(head))
    graph_ms = sorted(timed(replay) for _ in range(3))[1]  # median of three passes
    del g
    h2d = layer.q.numel() * 2 + (layer.qidx.numel() * 2 if layer.kind == "c4a" else 0)
    return graph_ms, eager_ms, h2d, layer.out.numel() * 2


# ------------------------------------------------------------------ oracle arm
class OracleStep:
    """The float64 oracle on one layer step of a workload, sequence by
    sequence, with every input generated before any timing: the queries,
    window rows and indexer keys of each sequence, and the compressed rows
    the step reads (all of them for c128a; for c4a the rows its top-k picks,
    found by one untimed top-k, as a resident cache would hold them).  A
    timed sequence runs the oracle's top-k over all its keys, gathers the
    selected rows and runs its attention."""

    def __init__(self, kind, batch, t, heads, seqs, seed=7, t_seq=None):
        import datagen as D
        from datagen import workloads as WL
        from oracle import formats as OF
        from oracle import indexer as OI
        self.kind, self.batch, self.heads, self.window, self.k = kind, batch, heads, 128, 512
        self.seqs = list(seqs)
        stride = 4 if kind == "c4a" else 128
        keys = WL.keys_for(seed, 0)
        self.inp = {}
        for b in self.seqs:
            tb = int(t if t_seq is None else t_seq[b])
            n = max(0, (tb - self.window) // stride)
            w = min(tb, self.window)
            q = OF.bf16_bits_to_f64(D.rows_normal_bf16(keys["q"], np.arange(b * heads, (b + 1) * heads), 512))
            win = OF.bf16_bits_to_f64(D.rows_normal_bf16(keys["win"], np.arange(b * 128, b * 128 + w), 512))
            e = {"t": tb, "q": q, "win": win}
            if kind == "c4a":
                kr = OF.bf16_bits_to_f64(D.rows_int_bf16(keys["kidx"], np.arange(b * n, (b + 1) * n), 128))
                qi = OF.bf16_bits_to_f64(D.rows_int_bf16(keys["qidx"], np.array([b]), 128)[0])
                idx, cnt = OI.index_topk(qi, kr, self.k)
                sel = idx[:cnt].astype(np.int64)
                e.update(keys=kr, qidx=qi, sel=sel,
                         rows=OF.bf16_bits_to_f64(D.rows_normal_bf16(keys["comp"], b * n + sel, 512)))
            else:
                e["comp"] = OF.bf16_bits_to_f64(D.rows_normal_bf16(keys["comp"], np.arange(b * n, (b + 1) * n), 512))
            self.inp[b] = e

    def run(self, b):
        from oracle import attention as OA
        from oracle import indexer as OI
        e = self.inp[b]
        if self.kind == "c4a":
            idx, cnt = OI.index_topk(e["qidx"], e["keys"], self.k)
            rows = e["rows"][np.searchsorted(e["sel"], idx[:cnt])]          # the selected rows of the cache
            return OA.shared_kv_decode(e["q"], np.concatenate([rows, e["win"]]), 512 ** -0.5, e["t"])
        return OA.dense_decode(e["q"][None], e["comp"][None], e["win"][None], e["t"], 512 ** -0.5)[0]


def oracle_per_seq(kind, batch, t, heads, budget_s=12.0, t_seq=None):
    """(seconds per sequence, sequences timed) of the oracle: the first
    sequences of the batch, each once, until the budget is used."""
    first = OracleStep(kind, batch, t, heads, [0], t_seq=t_seq)
    t0 = time.perf_counter()
    first.run(0)
    one = time.perf_counter() - t0
    m = int(max(1, min(batch, budget_s / max(one, 1e-6))))
    st = OracleStep(kind, batch, t, heads, range(m), t_seq=t_seq)
    t0 = time.perf_counter()
    for b in range(m):
        st.run(b)
    return (time.perf_counter() - t0) / m, m


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([i.get("num_threads", 1) for i in info] or [1])
    except Exception:
        return 1


def cpu_baseline(kind, batch, t, heads, budget_s, t_seq=None):
    """The oracle on the host: with all the BLAS threads it starts with, and
    again limited to one thread."""
    per_seq, m = oracle_per_seq(kind, batch, t, heads, budget_s, t_seq)
    out = {"value": 1.0 / (per_seq * batch), "unit": "steps/s", "cores": blas_threads(), "kind": "oracle",
           "sample": f"{m} of the {batch} sequences of one step (float64 NumPy oracle, inputs generated before "
                     f"timing), scaled to the whole step"}
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            per1, m1 = oracle_per_seq(kind, batch, t, heads, budget_s / 2, t_seq)
        out["value_1core"] = 1.0 / (per1 * batch)
        out["sample_1core"] = f"{m1} sequences, one BLAS thread"
    except ImportError:
        pass
    return out


def reference_arm(args, kind, batch, t, heads, config, wl_name, t_seq=None, budget_s=150.0):
    """--impl reference: the oracle times `warmup` untimed and `steps` timed
    steps on the host cores.  A step is the whole batch when all the steps
    fit the budget; otherwise each step is a sample of S sequences (the next
    S of the batch, cycling), and value counts whole steps (S / batch each)."""
    probe = OracleStep(kind, batch, t, heads, [0], t_seq=t_seq)
    t0 = time.perf_counter()
    probe.run(0)
    per_seq = time.perf_counter() - t0
    total = args.steps + args.warmup
    S = batch if total * batch * per_seq <= budget_s else int(max(1, budget_s / (total * per_seq)))
    seqs = sorted({(i * S + j) % batch for i in range(total) for j in range(S)})
    st = OracleStep(kind, batch, t, heads, seqs, t_seq=t_seq)

    def one_step(i):
        for j in range(S):
            st.run((i * S + j) % batch)

    for i in range(args.warmup):
        one_step(i)
    t0 = time.perf_counter()
    for i in range(args.warmup, total):
        one_step(i)
    el = time.perf_counter() - t0
    v = args.steps * S / batch / el
    sample = (f"whole steps ({batch} sequences each)" if S == batch else
              f"each step {S} of the {batch} sequences (cycling through the batch), counted as {S}/{batch} of a step")
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "steps/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el * 1e3 / args.steps,
            "sequences_per_step": S, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic", "config": config,
            "cpu_baseline": {"value": v, "unit": "steps/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": sample + "; float64 NumPy oracle, inputs generated before timing"},
            "e2e": {"value": v, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------------ distributed plumbing
_dist = {"on": False}


def dist_init():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws > 1:
        import datetime
        import torch
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        _dist.update(on=True, rank=dist.get_rank(), world=ws, local=int(os.environ.get("LOCAL_RANK", "0")))
    else:
        _dist.update(on=False, rank=0, world=1, local=0)
    return _dist


def dist_barrier():
    if _dist["on"]:
        import torch.distributed as dist
        dist.barrier()


def dist_max(x: float) -> float:
    if not _dist["on"]:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="c4a_b32")
    ap.add_argument("--secondary", default="c128a_b8,c128a_b32,q_c4a_fp8,q_c4a_fp4,q_c128a_fp8,q_c128a_fp4,"
                                           "q_c4a_fp8rope,q_c128a_fp8rope,c4a_b32_reindex,c4a_b32_paged",
                    help="extra per-layer-type workloads (comma list, 'none' = none)")
    ap.add_argument("--no-stack", action="store_true", help="skip the 61-layer stack step")
    ap.add_argument("--no-bulk", action="store_true", help="skip compressor/quantiser throughput")
    ap.add_argument("--stack-only", action="store_true",
                    help="time only the 61-layer stack step (--steps replays) and print its figures")
    ap.add_argument("--replicas", type=int, default=2, help="minimum cache replicas (raised until they hold 4x L2)")
    ap.add_argument("--l2-factor", type=int, default=4,
                    help="replicas hold at least this many L2 sizes (0 only for small profiling runs)")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    d = dist_init()
    kind, batch, t, heads, mfmt, ifmt = WORKLOADS[args.workload][:6]
    pool = WORKLOADS[args.workload][6] if len(WORKLOADS[args.workload]) > 6 else 0
    paged = len(WORKLOADS[args.workload]) > 7 and WORKLOADS[args.workload][7] == "paged"

    def wl_desc(kind, batch, t, heads, mfmt, ifmt, pool=0):
        idx = f", {FMT_NAME[ifmt]} indexer" if kind == "c4a" else ""
        if pool:
            idx += f", Reindex layer (top-512 inside a {pool}-entry pool)"
        return f"{kind} layer decode B={batch} t={t} H={heads} k=512 W=128 {FMT_NAME[mfmt]} main cache{idx}"

    wl_name = wl_desc(kind, batch, t, heads, mfmt, ifmt, pool)

    # the workload's cache replicas and bytes per step, from the shapes alone, so
    # that both arms print the same config
    seed = 1234 + d["rank"]
    if paged:
        reps = replicas_for(kind, batch, t // 2, mfmt, ifmt, args.replicas, 0, args.l2_factor)
        t_seq = ragged_lengths(batch, t, seed)
        n_seq = np.maximum(0, (t_seq - 128) // 4)
        alg = int((n_seq * KEY_BYTES[0]).sum() + ((np.minimum(n_seq, 512) + np.minimum(t_seq, 128)) * ROW_BYTES[0]).sum())
        wl_name = (f"c4a layer decode, paged caches ({PAGE_ROWS}-row pages, shuffled), ragged B={batch}: t_b uniform "
                   f"in [{t // 2}, {t}], H={heads} k=512 W=128 bf16")
    else:
        reps = replicas_for(kind, batch, t, mfmt, ifmt, args.replicas, pool, args.l2_factor)
        t_seq = None
        alg = step_bytes(kind, batch, t, mfmt, ifmt, pool=pool)
    config = {"workload": wl_name, "batch_per_gpu": batch, "context": t, "heads": heads,
              "parallelism": f"dp{d['world']}",
              "l2": f"inputs larger than L2: {reps} cache replicas cycle, {alg / 1e6:.0f} MB read per step, "
                    f"{reps * alg / 1e6:.0f} MB in all (>= 4 x the 126 MB L2)"}

    if args.impl == "reference":
        if d["rank"] != 0:
            return
        print(json.dumps(reference_arm(args, kind, batch, t, heads, config, wl_name, t_seq)), flush=True)
        return

    import torch
    import compressed_sparse_kv_b200 as K
    K.lib()
    torch.cuda.set_device(d["local"])
    if args.stack_only:
        st = time_stack(args.steps, args.warmup, seed + 7, dist_max)
        if d["rank"] == 0:
            print(json.dumps({"stack": st}), flush=True)
        return
    hbm_peak, tf_peak, peak_src = measured_peaks()
    if paged:
        layer = PagedLayer(batch, t, heads, seed, reps)
    else:
        layer = Layer(kind, batch, t, heads, seed, reps, mfmt, ifmt, pool=pool)
    assert layer.alg_bytes() == alg
    res = time_layer(layer, args.steps, args.warmup, dist_max, d["local"], sample_clocks=(d["rank"] == 0))
    ms = res["total_ms"] / args.steps
    steps_per_s = d["world"] * 1e3 / ms            # whole job: every rank ran `steps` steps
    e2e_ms, e2e_eager_ms, h2d, d2h = time_e2e(layer, args.steps)
    e2e_ms, e2e_eager_ms = dist_max(e2e_ms), dist_max(e2e_eager_ms)
    e2e_v = d["world"] * args.steps * 1e3 / e2e_ms
    e2e_eager_v = d["world"] * args.steps * 1e3 / e2e_eager_ms

    # roofline of the dominant kernel: the indexer score kernel for c4a (one
    # launch per dsv4kv_index_score call), the dense decode call for c128a
    if kind == "c4a":
        dom_bytes, dom_ms = layer.index_bytes(), res["score_ms"]
        dom_name = ("index_pool_select" if pool else "index_score_paged + index_select" if paged
                    else "index_score_stream<bf16>" if ifmt == 0 else "index_score_stream<fp4>")
    else:
        dom_bytes, dom_ms, dom_name = alg, res["decode_ms"], "dsv4kv_dense_decode (decode_kernel + decode_combine)"
    achieved = dom_bytes / (dom_ms * 1e-3) / 1e9
    roof = {"bound": "hbm", "kernel": dom_name, "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
            "frac": round(achieved / hbm_peak, 4), "peak_source": peak_src,
            "traffic": TRAFFIC.get((args.workload, dom_name)),
            "bytes_per_launch": dom_bytes, "avg_launch_ms": round(dom_ms, 5)}

    per_type = {kind: {"workload": wl_name, "steps_per_s": round(steps_per_s, 1),
                       "tokens_per_s": round(steps_per_s * batch, 1),
                       "hbm_gbs": round(alg / (ms * 1e-3) / 1e9, 1),
                       "frac_of_peak_hbm": round(alg / (ms * 1e-3) / 1e9 / hbm_peak, 4),
                       "frac_of_8tbs": round(alg / (ms * 1e-3) / 8e12, 4),
                       "index_ms": round(res["index_ms"], 5), "score_ms": round(res["score_ms"], 5),
                       "select_ms": round(res["select_ms"], 5), "decode_ms": round(res["decode_ms"], 5),
                       "median_of_5_ms_per_step": round(dist_max(res["median5_ms"]) / args.steps, 5)}}
    for name in [s for s in args.secondary.split(",") if s and s not in ("none", args.workload)]:
        spec = WORKLOADS[name]
        pool2 = spec[6] if len(spec) > 6 else 0
        paged2 = len(spec) > 7 and spec[7] == "paged"
        if paged2:
            # every length is >= t/2, so replicas sized at t/2 hold >= 4 x L2
            r2n = replicas_for(spec[0], spec[1], spec[2] // 2, spec[4], spec[5], 2)
            L2 = PagedLayer(spec[1], spec[2], spec[3], seed + 99, r2n)
        else:
            r2n = replicas_for(spec[0], spec[1], spec[2], spec[4], spec[5], 2, pool2)
            L2 = Layer(*spec[:4], seed + 99, r2n, spec[4], spec[5], pool=pool2)
        r2 = time_layer(L2, args.steps, args.warmup, dist_max, d["local"], sample_clocks=False)
        ms2 = r2["total_ms"] / args.steps
        a2 = L2.alg_bytes()
        desc2 = wl_desc(*spec[:7])
        if paged2:
            desc2 = (f"c4a layer decode, paged caches ({PAGE_ROWS}-row pages, shuffled), ragged B={spec[1]}: t_b "
                     f"uniform in [{spec[2] // 2}, {spec[2]}] (mean {L2.t_host.mean():.0f}), H={spec[3]} k=512 "
                     f"W=128 bf16")
        per_type[name] = {"workload": desc2, "steps_per_s": round(d["world"] * 1e3 / ms2, 1),
                          "us_per_step": round(ms2 * 1e3, 2), "cache_replicas": r2n,
                          "hbm_gbs": round(a2 / (ms2 * 1e-3) / 1e9, 1),
                          "frac_of_peak_hbm": round(a2 / (ms2 * 1e-3) / 1e9 / hbm_peak, 4),
                          "tflops": round(L2.flops() / (ms2 * 1e-3) / 1e12, 1),
                          "frac_of_peak_bf16": round(L2.flops() / (ms2 * 1e-3) / 1e12 / tf_peak, 4)}
        if spec[0] == "c4a":
            per_type[name]["index_us"] = round(r2["index_ms"] * 1e3, 2)
            per_type[name]["score_us"] = round(r2["score_ms"] * 1e3, 2)
            per_type[name]["select_us"] = round(r2["select_ms"] * 1e3, 2)
            per_type[name]["decode_us"] = round(r2["decode_ms"] * 1e3, 2)
        del L2
        torch.cuda.empty_cache()
    stack = None if args.no_stack else time_stack(max(10, args.steps // 20), args.warmup, seed + 7, dist_max)
    bulk = None if args.no_bulk else time_bulk(seed + 11)

    line = {"metric": METRIC, "value": round(steps_per_s, 2), "unit": "steps/s", "n_gpus": d["world"],
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": FMT_NAME[mfmt], "data": "synthetic",
            "config": config,
            "hbm_gbs": round(alg / (ms * 1e-3) / 1e9, 1), "alg_bytes_per_step": alg,
            "per_layer_type": per_type, "roofline": roof,
            "e2e": {"value": round(e2e_v, 2), "unit": "steps/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "eager_value": round(e2e_eager_v, 2),
                    "method": "public API (the layer's index and decode calls) on pinned host buffers; per "
                              "step an H2D of the queries and a D2H of the outputs, pipelined over upload / "
                              "compute / download streams with three buffer sets; the whole pipeline of the "
                              "timed steps (copies, calls, event dependencies) captured as one CUDA graph and "
                              "replayed (eager_value: the same copies and calls issued from Python step by "
                              "step)"},
            "gpu_launches": layer.launches_per_step() * args.steps,
            "clocks": res["clocks"]}
    if stack:
        line["stack"] = stack
    if bulk:
        line["bulk"] = bulk
    if d["rank"] == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(kind, batch, t, heads, args.cpu_budget, t_seq)
    if d["rank"] == 0:
        print(json.dumps(line), flush=True)
    if _dist["on"]:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
