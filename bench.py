#!/usr/bin/env python
"""Benchmark of the block-sparse attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the workload's hot path over one batch of synthetic,
seeded input already resident in HBM:
  gist_prefill_32k   layout build + forward    (default; N=32768, 32q/8kv heads)
  gzip_8k            mask build + forward      (batch 8, N=8192, b=64)
  gzip_64k_fwdbwd    mask build + forward + backward (batch 2, N=65536, b=128)
  gist_decode_128k   one decode step           (16 seqs, 131072-token caches)
  gist_prefill_32k_fwdbwd  layout build + forward + backward on the 32K gist inputs
  gist_coarse_20k    coarse (segment-wise) layout build + forward: 16 segments
                     of 1024 raw tokens + 256 gists (20480 positions, 32q/8kv)
  gist_coarse_20k_fwdbwd   the same with the backward
  gist_hier_decode_128k    gist-of-gist decode step over the decode cache shape
                     (128 level-2 gists, top-8 groups, top-64 chunks)
  gzip_flags_128m    on-device literal flags over 2048 rows of 64 KiB (b=128)
Prefill/backward workloads report visited-tile TFLOP/s (every visited block
pair counted as a full b x b tile: 4*d*b^2 forward, 10*d*b^2 backward; gist
layouts count their tile-list sub-blocks, 128 or 32 columns wide), and beside
it the same step counted by exact (query, key) edges (4*d per edge forward,
10*d backward); the decode workloads report algorithmic HBM GB/s. Inputs are larger than the
126 MB L2, so no flush is needed between steps. Under torchrun each rank runs
its own independent copy of the workload (weak scaling, no collective on the
data path); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import sa_workloads as W  # noqa: E402

METRIC = "visited-tile attn TFLOP/s & % bf16 tensor peak; gist-decode HBM GB/s"


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], "measured"
    return 6650.0, 1590.0, "fallback"


# --------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event reasons sampled during the timed region: NVML
    polled every 10 ms from a thread (the timed region of a fast workload is
    tens of milliseconds), else nvidia-smi every 200 ms. start() returns once
    the first sample is in, so sampling covers the whole region. Reads only."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))

    def __init__(self, index: int):
        self.index, self.proc, self.lines = index, None, []
        self.nvml, self.samples, self.stop_ev = None, [], threading.Event()

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.nvml = (pynvml, h)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            threading.Thread(target=self._poll, daemon=True).start()
            t0 = time.time()
            while not self.samples and time.time() - t0 < 2.0:
                time.sleep(0.002)
            return
        except Exception:
            self.nvml = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._read, daemon=True).start()
            t0 = time.time()
            while not self.lines and time.time() - t0 < 3.0:
                time.sleep(0.01)
        except OSError:
            self.proc = None

    def _poll(self):
        nv, h = self.nvml
        while not self.stop_ev.is_set():
            try:
                sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                rs = int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))
                self.samples.append((sm, rs))
            except Exception:
                return
            time.sleep(0.01)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.nvml is not None:
            self.stop_ev.set()
            time.sleep(0.02)
            if not self.samples:
                return None
            sm = [x[0] for x in self.samples]
            reasons = sorted({n for _, rs in self.samples for n, bit in self.REASONS if rs & bit})
            return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                    "samples": len(sm), "source": "nvml, 10 ms"}
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        self.proc.wait(timeout=5)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvidia-smi, 200 ms"}


# ------------------------------------------------------------- workloads


# the kernels whose DRAM traffic profiles/traffic.json records, and their sources; the
# backward is reported as one unit: row prep, the query-major dQ pass and the
# key-major dK/dV pass
KERNEL_SOURCES = {"fwd_tc_kernel": ["attn_fwd_sm100.cu"],
                  "backward": ["attn_bwd_sm100.cu", "attn_dq_sm100.cu"],
                  "decode_tc_kernel": ["decode_sm100.cu"],
                  "hier decode (6 CUDA-core passes)": ["decode.cu"],
                  "decode_tc_kernel (gist of gists)": ["decode_sm100.cu"],
                  "deflate_size_kernel + literal_flags_kernel": ["compress.cu"]}


def kernel_digest(kernel):
    """SHA-256 (16 hex digits) of a kernel's .cu file and the shared headers."""
    import hashlib
    csrc = os.path.join(ROOT, "content_adaptive_block_sa_b200", "csrc")
    m = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel] + ["sm100.cuh", "attn_mask.cuh", "sa_common.cuh"]:
        with open(os.path.join(csrc, f), "rb") as fh:
            m.update(fh.read())
    return m.hexdigest()[:16]


def recorded_traffic(workload, kernel):
    """DRAM bytes per full-size launch from profiles/traffic.json, or None when
    no row exists or the kernel's sources changed since the counters were taken
    (a stale row is reported as null until a new capture replaces it)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if kernel not in KERNEL_SOURCES or not os.path.exists(path):
        return None
    for row in json.load(open(path))["rows"]:
        if row["workload"] == workload and row["kernel"] == kernel:
            return int(row["traffic"]) if row["source"] == kernel_digest(kernel) else None
    return None


def io_bytes(wl):
    """Bytes a step copies host -> device and device -> host."""
    ins, outs = wl.io_tensors()
    nb = lambda t: t.numel() * t.element_size()
    return sum(nb(h) for h, _ in ins), sum(nb(o) for o in outs)


def e2e_run(wl, torch, steps):
    """`steps` end-to-end steps through the public API, each copying its inputs
    from pinned host memory and reading its results back, pipelined on three
    streams with two staging sets: while step i computes, step i+1's inputs
    come in and step i-1's results go out (PCIe both ways at once). Inputs land
    in a staging buffer and are copied on the device into the workload's
    tensors, results are copied out to a staging buffer before the next step
    overwrites them. Steps that move under 16 MB run the copies in line on the
    compute stream. Returns the elapsed ms of all steps (CUDA events)."""
    ins, outs = wl.io_tensors()
    cur = torch.cuda.current_stream()
    if sum(io_bytes(wl)) < (16 << 20):
        # a few KB per step (a decode token): staging would only add copies
        host_out = [o.new_empty(o.shape, device="cpu").pin_memory() for o in outs]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(cur)
        for _ in range(steps):
            for h, d in ins:
                d.copy_(h, non_blocking=True)
            wl.step()
            for o, h in zip(outs, host_out):
                h.copy_(o, non_blocking=True)
        t1.record(cur)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)
    sh, sd = torch.cuda.Stream(), torch.cuda.Stream()
    stg_in = [[d.new_empty(d.shape) for _, d in ins] for _ in range(2)]
    stg_out = [[o.new_empty(o.shape) for o in outs] for _ in range(2)]
    host_out = [[o.new_empty(o.shape, device="cpu").pin_memory() for o in outs] for _ in range(2)]
    in_free, out_free, h2d_done = [None, None], [None, None], [None, None]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def h2d(i):
        b = i & 1
        with torch.cuda.stream(sh):
            if in_free[b] is not None:
                sh.wait_event(in_free[b])
            for (h, _), st in zip(ins, stg_in[b]):
                st.copy_(h, non_blocking=True)
            h2d_done[b] = torch.cuda.Event()
            h2d_done[b].record(sh)

    t0.record(cur)
    sh.wait_stream(cur)
    sd.wait_stream(cur)
    h2d(0)
    for i in range(steps):
        b = i & 1
        if i + 1 < steps:
            h2d(i + 1)
        cur.wait_event(h2d_done[b])
        for (_, d), st in zip(ins, stg_in[b]):
            d.copy_(st, non_blocking=True)
        in_free[b] = torch.cuda.Event()
        in_free[b].record(cur)
        wl.step()
        if out_free[b] is not None:
            cur.wait_event(out_free[b])
        for o, st in zip(outs, stg_out[b]):
            st.copy_(o, non_blocking=True)
        done = torch.cuda.Event()
        done.record(cur)
        with torch.cuda.stream(sd):
            sd.wait_event(done)
            for st, h in zip(stg_out[b], host_out[b]):
                h.copy_(st, non_blocking=True)
            out_free[b] = torch.cuda.Event()
            out_free[b].record(sd)
    cur.wait_stream(sh)
    cur.wait_stream(sd)
    t1.record(cur)
    torch.cuda.synchronize()
    return t0.elapsed_time(t1)


class GzipWorkload:
    def __init__(self, sa, torch, w, backward, device_flags=False):
        self.sa, self.torch, self.backward = sa, torch, backward
        self.w = w
        Bt, N, H, d, b = w["batch"], w["seq_len"], w["heads"], w["head_dim"], w["block"]
        # a1 on the device: every step computes the flags from the raw bytes
        # (sa_literal_flags_device) instead of taking host-made flags
        self.device_flags = device_flags
        if device_flags:
            if w.get("flags_from") == "bernoulli":
                raise ValueError("this workload draws its flags; it has no bytes to compress")
            raw = np.stack([np.frombuffer(W.workload_bytes(w, i), np.uint8) for i in range(Bt)])
            self.h_bytes = torch.from_numpy(raw).pin_memory()
            self.x = self.h_bytes.cuda()
            self.sizes = torch.empty(Bt, N // b, dtype=torch.int32, device="cuda")
            flags = np.zeros((Bt, N // b), np.uint8)
        elif w.get("flags_from") == "bernoulli":
            flags = W.bernoulli_flags(w)
        else:
            flags = np.stack([sa.literal_flags(W.workload_bytes(w, i), b) for i in range(Bt)])
        self.h_flags = torch.from_numpy(flags).pin_memory()
        mk = lambda t: torch.from_numpy(np.stack([W.qkv(w, t, i) for i in range(Bt)])).to(torch.bfloat16)
        self.h_in = {t: mk(t).pin_memory() for t in (["q", "k", "v"] + (["do"] if backward else []))}
        dev = {t: x.cuda() for t, x in self.h_in.items()}
        self.q, self.k, self.v = dev["q"], dev["k"], dev["v"]
        self.do = dev.get("do")
        self.flags = self.h_flags.cuda()
        self.md = sa.gzip_mask(Bt, N, b, w["window"], H)
        self.lists = sa.BlockLists(self.md)
        self.build_ws = sa._workspace(256, "cuda")
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty(Bt, H, N, dtype=torch.float32, device="cuda")
        self.ad = sa.attn_desc(self.q, self.k, self.v, self.o)
        self.fws = sa.forward_workspace(self.ad, self.md)
        if backward:
            self.dq = torch.empty(self.q.shape, dtype=torch.float32, device="cuda")
            self.dk = torch.empty_like(self.dq)
            self.dv = torch.empty_like(self.dq)
            self.bws = sa.backward_workspace(self.ad, self.md)
        self.step()
        torch.cuda.synchronize()
        # visited block pairs per (batch, class) from the lists just built
        B = N // b
        rp = self.lists.row_ptr.cpu().numpy().reshape(Bt * 3, B + 1)
        nnz = rp[:, -1] - rp[:, 0]
        cls = [0] * (H // 2) + [1] * (H // 4) + [2] * (H - H // 2 - H // 4)
        pairs = sum(int(nnz[bt * 3 + c]) for bt in range(Bt) for c in cls)
        self.pairs = pairs
        self.flops_fwd = 4.0 * d * b * b * pairs
        self.flops = self.flops_fwd * (1 + (2.5 if backward else 0))
        # exact token edges: every list row holds its diagonal block, whose
        # b(b+1)/2 causal pairs replace the b*b of a full tile
        diag = Bt * H * B
        self.exact_fwd = 4.0 * d * (b * b * (pairs - diag) + diag * b * (b + 1) // 2)
        self.exact = self.exact_fwd * (1 + (2.5 if backward else 0))
        # builder + forward (+ the pairing pre-pass for 64-token blocks) (+ backward:
        # row prep, query-major dQ pass, key-major dK/dV pass)
        self.kernels_per_step = 2 + (1 if b == 64 else 0) + (3 if backward else 0) + \
            (2 if device_flags else 0)
        self.kernel = "fwd_tc_kernel"
        self.unit = "TFLOP/s"

    def fwd_only(self):
        self.sa.sa_forward(self.ad, self.md, self.q, self.k, self.v, self.lists, self.o, self.lse,
                           self.fws)

    def step(self, ev=None):
        sa = self.sa
        if self.device_flags:
            sa.literal_flags_device(self.x, self.w["block"], sizes=self.sizes, flags=self.flags)
        sa.sa_build_block_mask(self.md, self.flags, self.lists, self.build_ws)
        if ev is not None:
            ev[0].record()
        self.fwd_only()
        if ev is not None:
            ev[1].record()
        if self.backward:
            sa.sa_backward(self.ad, self.md, self.q, self.k, self.v, self.o, self.lse, self.do,
                           self.lists, self.dq, self.dk, self.dv, self.bws)
            if ev is not None:
                ev[2].record()

    def io_tensors(self):
        """(host input, device input) pairs a step copies in, and the device
        results it reads back."""
        ins = [(h, getattr(self, t)) for t, h in self.h_in.items()]
        ins.append((self.h_bytes, self.x) if self.device_flags else (self.h_flags, self.flags))
        return ins, [self.o, self.lse] + ([self.dq, self.dk, self.dv] if self.backward else [])

    def cpu_baseline(self, heads=None):
        """The oracle on batch row 0, one head of each class (whole heads)."""
        from oracle import attention as A
        from oracle import gzip_mask as G
        w, b = self.w, self.w["block"]
        flags = G.literal_flags(W.workload_bytes(w, 0), b) if w.get("flags_from") != "bernoulli" \
            else W.bernoulli_flags(w)[0]
        masks = G.block_masks(flags, w["window"])
        H = w["heads"]
        heads = [0, H // 2, H - 1] if heads is None else heads
        cls = G.head_classes(H)
        N = w["seq_len"]
        R = min(N, max(b, 2048 // b * b))  # the last R query rows (whole blocks)
        rows = np.arange(N - R, N)
        data = {h: [W.qkv(w, t, 0, head=h) for t in ("q", "k", "v", "do")] for h in heads}
        t0 = time.perf_counter()
        flops = exact = 0.0
        for h in heads:
            bm = masks[cls[h]]
            q, k, v, do = data[h]
            mask = lambda r: G.token_mask(bm, b, rows=rows[r])
            if self.backward:
                A.backward(q[rows], k, v, do[rows], mask)
            else:
                A.forward(q[rows], k, v, mask)
            pairs = int(bm[(N - R) // b:].sum())
            per = (4.0 + (10.0 if self.backward else 0.0)) * w["head_dim"]
            flops += per * b * b * pairs
            exact += per * (b * b * (pairs - R // b) + (R // b) * b * (b + 1) // 2)
        dt = time.perf_counter() - t0
        return flops / dt / 1e12, (f"batch row 0, heads {heads} (one per class), last {R} query "
                                   "rows each, fp64"), dt, exact / dt / 1e12


class GistWorkload(GzipWorkload):
    def __init__(self, sa, torch, w, backward=False):
        self.sa, self.torch, self.backward = sa, torch, backward
        self.w = w
        self.device_flags = False  # the gist layout has no a1 step
        N, H, Hkv, d = w["seq_len"], w["heads"], w["kv_heads"], w["head_dim"]
        self.h_in = {t: torch.from_numpy(W.qkv(w, t, 0)[None]).to(torch.bfloat16).pin_memory()
                     for t in ("q", "k", "v") + (("do",) if backward else ())}
        self.q, self.k, self.v = (self.h_in[t].cuda() for t in ("q", "k", "v"))
        self.do = self.h_in["do"].cuda() if backward else None
        self.md = sa.gist_mask(N, H, w["sinks"], w["ratio"], w["window"], gist_tail=w["gist_tail"],
                               segment=w.get("gist_segment", 0))
        self.lists = sa.BlockLists(self.md)
        self.flags = None
        self.h_flags = torch.zeros(1, dtype=torch.uint8)
        self.build_ws = sa._workspace(256, "cuda")
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty(1, H, N, dtype=torch.float32, device="cuda")
        self.ad = sa.attn_desc(self.q, self.k, self.v, self.o)
        self.fws = sa.forward_workspace(self.ad, self.md)
        if backward:
            self.dq = torch.empty(self.q.shape, dtype=torch.float32, device="cuda")
            self.dk = torch.empty(self.k.shape, dtype=torch.float32, device="cuda")
            self.dv = torch.empty_like(self.dk)
            self.bws = sa.backward_workspace(self.ad, self.md)
        self.step()
        torch.cuda.synchronize()
        T = (N + 127) // 128
        rp = self.lists.tile_row_ptr.cpu().numpy()
        kinds = self.lists.tile_kind.cpu().numpy()[: rp[-1]]
        width = np.where(kinds == 2, w["gist_tail"], 128)
        self.flops_fwd = 4.0 * d * H * 128 * float(width.sum())
        self.flops = self.flops_fwd * (1 + (2.5 if backward else 0))
        self.exact_fwd = 4.0 * d * H * float(gist_visible_pairs(w))
        self.exact = self.exact_fwd * (1 + (2.5 if backward else 0))
        # builder (4 launches) + sink/gist gather + near-tile masks + forward (+ backward:
        # row prep, the three gist pre-passes, dQ pass, dK/dV pass, far scatter)
        self.kernels_per_step = 7 + (7 if backward else 0)
        self.kernel = "fwd_tc_kernel"
        self.unit = "TFLOP/s"

    def io_tensors(self):
        ins = [(h, getattr(self, t)) for t, h in self.h_in.items()]
        return ins, [self.o, self.lse] + ([self.dq, self.dk, self.dv] if self.backward else [])

    def cpu_baseline(self):
        from oracle import attention as A
        from oracle import gist as Gi
        w = self.w
        N, L = w["seq_len"], w.get("gist_segment", 0)
        if L:  # coarse layout: segments of L raw tokens, then L / ratio gists
            g = Gi.coarse_gist_flags(N, w["sinks"], L, w["ratio"])
            seg = Gi.segment_ids(N, w["sinks"], L, w["ratio"])
            vis_rows = lambda r: Gi.coarse_visibility(g, seg, w["sinks"], rows=r)
        else:
            g = Gi.gist_flags(N, w["sinks"], w["ratio"])
            vis_rows = lambda r: Gi.visibility(g, w["sinks"], w["window"], rows=r)
        perm = Gi.shift_permutation(g, 128)
        inv = np.empty_like(perm)
        inv[perm] = np.arange(N)
        rows = np.arange(N - 2048, N)  # the last 2048 logical query rows of head 0
        q = W.qkv(w, "q", 0, head=0)[inv]
        k = W.qkv(w, "k", 0, head=0)[inv]
        v = W.qkv(w, "v", 0, head=0)[inv]
        mask = lambda r: vis_rows(rows[r])
        t0 = time.perf_counter()
        if self.backward:
            do = W.qkv(w, "do", 0, head=0)[inv]
            A.backward(q[rows], k, v, do[rows], mask)
        else:
            A.forward(q[rows], k, v, mask)
        dt = time.perf_counter() - t0
        # the GPU leg's two counts for those rows (the last 16 tiles hold exactly
        # the last 2048 logical positions: the shift stays inside a tile):
        # tile-list sub-blocks, and exact visible pairs
        T = N // 128
        _, _, kinds = Gi.tile_lists(lambda r: vis_rows(perm[r])[:, perm], 128, w["gist_tail"], N=N,
                                    query_tiles=range(T - 16, T))
        width = float(np.where(kinds == Gi.TAIL, w["gist_tail"], 128).sum())
        n_vis = int(vis_rows(rows).sum())
        per = (4.0 + (10.0 if self.backward else 0.0)) * w["head_dim"]
        return per * 128 * width / dt / 1e12, \
            "head 0, last 2048 query rows, fp64", dt, per * n_vis / dt / 1e12


def gist_visible_pairs(w):
    """Visible (query, key) pairs of one head of a gist layout, counted from
    its rule: key j <= query i is seen when j is a sink or a gist, or lies in
    i's window (fine layout: i - j < window) or segment (coarse layout)."""
    N, S, r = w["seq_len"], w["sinks"], w["ratio"]
    p = np.arange(N, dtype=np.int64)
    L = w.get("gist_segment", 0)
    if L:
        period = L + L // r
        gist = (p >= S) & ((p - S) % period >= L)
    else:
        gist = (p >= S) & ((p - S) % (r + 1) == r)
    pref = np.concatenate([[0], np.cumsum((p < S) | gist)])  # sinks + gists below x
    if L:
        start = np.where(p < S, 0, S + (p - S) // period * period)  # own segment's first position
        near = p - start + 1
        return int((near + np.where(p < S, 0, pref[start])).sum())
    Wn = w["window"]
    return int((np.minimum(Wn, p + 1) + pref[np.maximum(0, p - Wn + 1)]).sum())


def repeat_for(budget_s, fn):
    """Calls fn until budget_s seconds have passed (at least once): (calls, seconds)."""
    n, t0 = 0, time.perf_counter()
    while True:
        fn()
        n += 1
        dt = time.perf_counter() - t0
        if dt >= budget_s:
            return n, dt


# decode chunk selection rules (sa_select_rule)
SELECT_RULES = {"sum_logits": 0, "sum_probs": 1, "top_p": 2, "per_head": 3}


class DecodeWorkload:
    def __init__(self, sa, torch, w):
        self.sa, self.torch = sa, torch
        self.w = w
        n, Hkv, L, d, G = w["n_seq"], w["kv_heads"], w["cache_len"], w["head_dim"], w["n_gists"]
        self.kc = torch.empty(n, Hkv, L, d, dtype=torch.bfloat16, device="cuda")
        self.vc = torch.empty_like(self.kc)
        from concurrent.futures import ThreadPoolExecutor

        def one(i):
            s, g = divmod(i, Hkv)
            return i, W.decode_raw(w, s, g, "k"), W.decode_raw(w, s, g, "v")

        with ThreadPoolExecutor(8) as ex:
            for i, rk, rv in ex.map(one, range(n * Hkv)):
                s, g = divmod(i, Hkv)
                self.kc[s, g] = torch.from_numpy(rk).to("cuda", torch.bfloat16)
                self.vc[s, g] = torch.from_numpy(rv).to("cuda", torch.bfloat16)
        bf = lambda a: torch.from_numpy(a).to(torch.bfloat16)
        self.h_q = bf(W.decode_query(w)).pin_memory()
        self.h_gk = bf(np.stack([W.decode_gists(w, s, "k") for s in range(n)])).pin_memory()
        self.h_gv = bf(np.stack([W.decode_gists(w, s, "v") for s in range(n)])).pin_memory()
        self.q, self.gk, self.gv = self.h_q.cuda(), self.h_gk.cuda(), self.h_gv.cuda()
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty(n, w["heads"], dtype=torch.float32, device="cuda")
        rule = SELECT_RULES[w.get("select", "sum_logits")]
        rows = w["heads"] if rule == 3 else Hkv  # per-head rule: one selection per query head
        self.sel = torch.empty(n, rows, w["top_k"], dtype=torch.int32, device="cuda")
        self.dd = sa.decode_desc(self.q, self.gk, self.kc, self.o, w["chunk"], w["top_k"], w["window"],
                                 select_rule=rule, top_p=w.get("top_p", 1.0))
        self.ws = sa.decode_workspace(self.dd)
        self.step()
        torch.cuda.synchronize()
        # algorithmic bytes: every gist, each distinct unfolded chunk of a KV
        # group once (the union over its heads under the per-head rule) and the
        # window, K and V in bf16
        sel = self.sel.cpu().numpy().reshape(n, Hkv, -1)
        n_chunks = sum(len(np.unique(sel[s_, g_][sel[s_, g_] >= 0])) for s_ in range(n) for g_ in range(Hkv))
        kv_rows = n * Hkv * (G + w["window"]) + n_chunks * w["chunk"]
        self.bytes = float(kv_rows * d * 2 * 2 + 2 * self.q.numel() * 2 + self.lse.numel() * 4
                           + self.sel.numel() * 4)
        # one tensor-core kernel for these shapes, else the four CUDA-core passes
        c = w["chunk"]
        tc = 8 <= c <= 128 and 128 % c == 0 and 128 <= G <= 8192 and L >= 128
        self.kernels_per_step = 1 if tc else 4
        self.kernel = "decode_tc_kernel" if tc else "decode (4 CUDA-core passes)"
        self.unit = "GB/s"

    def step(self, ev=None):
        if ev is not None:
            ev[0].record()
        self.sa.sa_gist_decode(self.dd, self.q, self.gk, self.gv, self.kc, self.vc, self.sel, self.o,
                               self.lse, self.ws)
        if ev is not None:
            ev[1].record()

    def io_tensors(self):
        # a decode step's input is the new token's query; the caches are resident
        return [(self.h_q, self.q)], [self.o, self.lse, self.sel]

    def cpu_baseline(self, budget_s=10.0):
        from oracle import decode as D
        w = self.w
        q = W.decode_query(w)[0]
        gk, gv = W.decode_gists(w, 0, "k"), W.decode_gists(w, 0, "v")
        rk = [W.decode_raw(w, 0, g, "k") for g in range(w["kv_heads"])]
        rv = [W.decode_raw(w, 0, g, "v") for g in range(w["kv_heads"])]
        raw_k, raw_v = (lambda g: rk[g]), (lambda g: rv[g])
        rule = SELECT_RULES[w.get("select", "sum_logits")]
        out = {}

        def one():
            out["sel"] = D.decode_one(q, gk, gv, raw_k, raw_v, w["chunk"], w["window"], w["top_k"],
                                      rule=rule, top_p=w.get("top_p", 1.0))[0]
        n, dt = repeat_for(budget_s, one)
        sel = out["sel"].reshape(w["kv_heads"], -1)  # the group's rows (one per head: per-head rule)
        n_chunks = sum(len(np.unique(r_[r_ >= 0])) for r_ in sel)
        rows = w["kv_heads"] * (w["n_gists"] + w["window"]) + n_chunks * w["chunk"]
        return n * rows * w["head_dim"] * 2 * 2 / dt / 1e9, \
            f"sequence 0 decoded {n} times, all kv heads (raw cache generation excluded), fp64", dt


class HierDecodeWorkload(DecodeWorkload):
    """Gist-of-gist decode: level-2 gists, the kept groups' level-1 gists, the
    unfolded chunks and the window (one tensor-core kernel)."""

    def __init__(self, sa, torch, w):
        self.sa, self.torch = sa, torch
        self.w = w
        n, Hkv, L, d = w["n_seq"], w["kv_heads"], w["cache_len"], w["head_dim"]
        self.kc = torch.empty(n, Hkv, L, d, dtype=torch.bfloat16, device="cuda")
        self.vc = torch.empty_like(self.kc)
        from concurrent.futures import ThreadPoolExecutor

        def one(i):
            s, g = divmod(i, Hkv)
            return i, W.decode_raw(w, s, g, "k"), W.decode_raw(w, s, g, "v")

        with ThreadPoolExecutor(8) as ex:
            for i, rk, rv in ex.map(one, range(n * Hkv)):
                s, g = divmod(i, Hkv)
                self.kc[s, g] = torch.from_numpy(rk).to("cuda", torch.bfloat16)
                self.vc[s, g] = torch.from_numpy(rv).to("cuda", torch.bfloat16)
        bf = lambda a: torch.from_numpy(a).to(torch.bfloat16)
        self.h_q = bf(W.decode_query(w)).pin_memory()
        self.q = self.h_q.cuda()
        self.g2k, self.g2v, self.gk, self.gv = (
            bf(np.stack([fn(w, s, kv) for s in range(n)])).cuda()
            for fn, kv in ((W.decode_gists2, "k"), (W.decode_gists2, "v"),
                           (W.decode_gists, "k"), (W.decode_gists, "v")))
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty(n, w["heads"], dtype=torch.float32, device="cuda")
        self.sel2 = torch.empty(n, Hkv, w["top_k2"], dtype=torch.int32, device="cuda")
        self.sel = torch.empty(n, Hkv, w["top_k"], dtype=torch.int32, device="cuda")
        self.hd = sa.hier_decode_desc(self.q, self.g2k, self.gk, self.kc, self.o, w["chunk"],
                                      w["fanout"], w["top_k2"], w["top_k"], w["window"])
        self.ws = sa.hier_decode_workspace(self.hd)
        self.step()
        torch.cuda.synchronize()
        # algorithmic bytes: every level-2 gist, the kept groups' level-1 gists,
        # the unfolded chunks and the window, K and V in bf16
        n2 = w["n_gists"] // w["fanout"]
        kept = int((self.sel2.cpu() >= 0).sum()) * w["fanout"]
        chunks = int((self.sel.cpu() >= 0).sum()) * w["chunk"]
        rows = n * Hkv * (n2 + w["window"]) + kept + chunks
        self.bytes = float(rows * d * 2 * 2 + 2 * self.q.numel() * 2 + self.lse.numel() * 4
                           + (self.sel.numel() + self.sel2.numel()) * 4)
        # one tensor-core kernel for these shapes (both selections inside it),
        # else the six CUDA-core passes
        c, fo, n2 = w["chunk"], w["fanout"], w["n_gists"] // w["fanout"]
        tc = (8 <= c <= 128 and 128 % c == 0 and 8 <= fo <= 128 and 128 % fo == 0
              and 128 <= n2 <= 8192 and L >= 128)
        self.kernels_per_step = 1 if tc else 6
        self.kernel = "decode_tc_kernel (gist of gists)" if tc else "hier decode (6 CUDA-core passes)"
        self.unit = "GB/s"

    def step(self, ev=None):
        if ev is not None:
            ev[0].record()
        self.sa.sa_gist_hier_decode(self.hd, self.q, self.g2k, self.g2v, self.gk, self.gv, self.kc,
                                    self.vc, self.sel2, self.sel, self.o, self.lse, self.ws)
        if ev is not None:
            ev[1].record()

    def io_tensors(self):
        return [(self.h_q, self.q)], [self.o, self.lse, self.sel2, self.sel]

    def cpu_baseline(self, budget_s=10.0):
        from oracle import decode as D
        w = self.w
        q = W.decode_query(w)[0]
        g2k, g2v = W.decode_gists2(w, 0, "k"), W.decode_gists2(w, 0, "v")
        gk, gv = W.decode_gists(w, 0, "k"), W.decode_gists(w, 0, "v")
        rk = [W.decode_raw(w, 0, g, "k") for g in range(w["kv_heads"])]
        rv = [W.decode_raw(w, 0, g, "v") for g in range(w["kv_heads"])]
        out = {}

        def one():
            out["sel"] = D.hier_decode_one(q, g2k, g2v, gk, gv, rk, rv, w["chunk"], w["fanout"],
                                           w["top_k2"], w["top_k"], w["window"])[:2]
        n, dt = repeat_for(budget_s, one)
        sel2, sel1 = out["sel"]
        n2 = w["n_gists"] // w["fanout"]
        rows = (w["kv_heads"] * (n2 + w["window"]) + int((sel2 >= 0).sum()) * w["fanout"]
                + int((sel1 >= 0).sum()) * w["chunk"])
        return n * rows * w["head_dim"] * 2 * 2 / dt / 1e9, \
            f"sequence 0 decoded {n} times, all kv heads (raw cache generation excluded), fp64", dt


class FlagsWorkload:
    """On-device literal flags (each block's DEFLATE size, the smallest of a
    fixed, dynamic or stored block, then the mean rule) over rows of bytes
    already in HBM."""

    def __init__(self, sa, torch, w):
        self.sa, self.torch, self.w = sa, torch, w
        src = W.WORKLOADS[w["rows_from"]]
        rows = [np.frombuffer(W.workload_bytes(src, i % src["batch"]), np.uint8)
                for i in range(src["batch"])]
        x = np.stack([rows[i % len(rows)] for i in range(w["batch"])])
        self.h_x = torch.from_numpy(x).pin_memory()
        self.x = self.h_x.cuda()
        self.step()
        torch.cuda.synchronize()
        self.bytes = float(self.x.numel() + 2 * self.flags.numel() + 4 * self.sizes.numel())
        self.kernels_per_step = 2
        self.kernel = "deflate_size_kernel + literal_flags_kernel"
        self.unit = "GB/s"

    def step(self, ev=None):
        if ev is not None:
            ev[0].record()
        self.sizes, self.flags = self.sa.literal_flags_device(self.x, self.w["block"])
        if ev is not None:
            ev[1].record()

    def io_tensors(self):
        return [(self.h_x, self.x)], [self.flags]

    def cpu_baseline(self, budget_s=10.0):
        from oracle import deflate_size as F
        src = W.WORKLOADS[self.w["rows_from"]]
        rows = [W.workload_bytes(src, i) for i in range(src["batch"])]
        chunks = [r[i:i + 8192] for r in rows for i in range(0, len(r), 8192)]  # 64 blocks each
        k = [0]

        def one():
            F.block_sizes(chunks[k[0] % len(chunks)], self.w["block"])
            k[0] += 1
        n, dt = repeat_for(budget_s, one)
        return n * 8192 / dt / 1e9, f"{n} successive 8 KiB pieces of the rows (64 blocks each), pure Python", dt


SMALL = {"gzip_8k": dict(batch=8), "gzip_64k_fwdbwd": dict(batch=1, heads=4, kv_heads=4),
         "gist_prefill_32k": dict(heads=8, kv_heads=2), "gist_decode_128k": dict(n_seq=4),
         "gist_coarse_20k": dict(heads=8, kv_heads=2), "gist_hier_decode_128k": dict(n_seq=4),
         "gzip_flags_128m": dict(batch=1024)}
# workloads that run another one's inputs with the backward added
FWDBWD_OF = {"gist_prefill_32k_fwdbwd": "gist_prefill_32k",
             "gist_coarse_20k_fwdbwd": "gist_coarse_20k"}


def workload_params(name, rank, size):
    name = FWDBWD_OF.get(name, name)
    w = dict(W.WORKLOADS[name])
    if size == "small":
        w.update(SMALL[name])
    if rank:
        w["index"] = w["index"] + 1000 * rank  # an independent copy per rank
    return w


def make(sa, torch, name, rank, size="full", select=None, device_flags=False):
    w = workload_params(name, rank, size)
    if select is not None:
        w["select"], w["top_p"] = select, 0.9  # top-p keeps 90% of the probability
    if w["kind"] == "gzip":
        return GzipWorkload(sa, torch, w, name.endswith("fwdbwd"), device_flags)
    if device_flags:
        raise ValueError("--flags-on-device applies to the gzip workloads")
    if w["kind"] == "gist":
        return GistWorkload(sa, torch, w, name.endswith("fwdbwd"))
    if w["kind"] == "hier":
        return HierDecodeWorkload(sa, torch, w)
    if w["kind"] == "flags":
        return FlagsWorkload(sa, torch, w)
    return DecodeWorkload(sa, torch, w)


# ----------------------------------------------------------------- ranks
def rank_barrier(world: int) -> None:
    """Barrier across ranks (no-op on one process)."""
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def rank_max(x: float, world: int, device: str = "cuda") -> float:
    """Max of a per-rank number over all ranks (the timing reduction only)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank: float, world: int, ms_per_step: float, scale: float) -> float:
    """Whole-job throughput: every rank's units over the slowest rank's time."""
    return units_per_rank * world / (ms_per_step * 1e-3) / scale


# ----------------------------------------------------------------- main
def run_reference(args):
    """The oracle on the host cores, on a bounded sample of the workload."""
    import torch

    class Stub:
        pass
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    torch.set_num_threads(len(os.sched_getaffinity(0)))
    wl = Stub()
    wl.w = dict(W.WORKLOADS[FWDBWD_OF.get(args.workload, args.workload)])
    wl.backward = args.workload.endswith("fwdbwd")
    if args.select is not None:
        wl.w["select"], wl.w["top_p"] = args.select, 0.9
    cls = {"gzip": GzipWorkload, "gist": GistWorkload, "decode": DecodeWorkload,
           "hier": HierDecodeWorkload, "flags": FlagsWorkload}
    fn = cls[wl.w["kind"]].cpu_baseline
    vals = []
    H = wl.w.get("heads", 1)
    for i in range(args.warmup + args.steps):
        if wl.w["kind"] == "gzip":
            # one head per step, cycling through the three classes
            res = fn(wl, heads=[(0, H // 2, H - 1)[i % 3]])
            sample = res[1].replace("heads", "one head per step cycling local/literal/hybrid:", 1)
        elif wl.w["kind"] in ("decode", "hier", "flags"):
            # each step a bounded sample: the whole run stays within a few minutes
            res = fn(wl, budget_s=max(0.2, min(10.0, 120.0 / (args.steps + args.warmup))))
            sample = res[1]
        else:
            res = fn(wl)
            sample = res[1]
        if i >= args.warmup:
            vals.append((res[0], res[2], res[3] if len(res) > 3 else None))
    value = float(np.mean([v[0] for v in vals]))
    exact = None if vals[0][2] is None else float(np.mean([v[2] for v in vals]))
    unit = "GB/s" if wl.w["kind"] in ("decode", "hier", "flags") else "TFLOP/s"
    cores = len(os.sched_getaffinity(0))
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": float(np.mean([v[1] for v in vals]) * 1e3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "u8" if wl.w["kind"] == "flags" else "f64",
        "data": "synthetic",
        "config": {"workload": args.workload, **({"select": args.select} if args.select else {})},
        "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle",
                         "sample": sample, **({"exact_edges_value": exact} if exact else {})},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="gist_prefill_32k",
                    choices=["gzip_8k", "gzip_64k_fwdbwd", "gist_prefill_32k", "gist_decode_128k",
                             "gist_prefill_32k_fwdbwd", "gist_coarse_20k", "gist_coarse_20k_fwdbwd",
                             "gist_hier_decode_128k", "gzip_flags_128m"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--size", default="full", choices=["full", "small"],
                    help="small: fewer heads/sequences (inputs still larger than L2), for profiling")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--select", default=None, choices=list(SELECT_RULES),
                    help="gist_decode_128k: chunk selection rule (default sum_logits; top_p at p = 0.9)")
    ap.add_argument("--flags-on-device", action="store_true",
                    help="gzip_64k_fwdbwd: each step computes the literal flags from the raw bytes "
                         "on the GPU (DEFLATE size estimate) instead of taking host zlib flags")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    import content_adaptive_block_sa_b200 as sa
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))

    barrier = lambda: rank_barrier(world)
    max_over_ranks = lambda x: rank_max(x, world, "cuda")

    wl = make(sa, torch, args.workload, rank, args.size, args.select, args.flags_on_device)
    for _ in range(args.warmup):
        wl.step()
    torch.cuda.synchronize()

    # ---- device-timed region: K steps, inputs resident
    # per step: before the timed kernel, after it (and after the backward)
    fwd_ev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3))
              for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(args.steps):
        wl.step(fwd_ev[i])
    t1.record()
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    ms = max_over_ranks(t0.elapsed_time(t1)) / args.steps
    kern_ms = max_over_ranks(float(np.mean([e[0].elapsed_time(e[1]) for e in fwd_ev])))
    bwd_ms = (max_over_ranks(float(np.mean([e[1].elapsed_time(e[2]) for e in fwd_ev])))
              if getattr(wl, "backward", False) else None)

    # ---- end-to-end through the public API with host buffers
    e2e_run(wl, torch, 2)
    barrier()
    e2e_ms = max_over_ranks(e2e_run(wl, torch, args.steps)) / args.steps
    barrier()
    h2d, d2h = io_bytes(wl)

    hbm, bf16, src = peaks()
    if wl.unit == "GB/s":
        units = wl.bytes
        value = weak_scaling_value(units, world, ms, 1e9)
        e2e_value = weak_scaling_value(units, world, e2e_ms, 1e9)
        ach = wl.bytes / (kern_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                "traffic": None, "peak_source": src, "kernel": wl.kernel}
    else:
        value = weak_scaling_value(wl.flops, world, ms, 1e12)
        e2e_value = weak_scaling_value(wl.flops, world, e2e_ms, 1e12)
        value_exact = weak_scaling_value(wl.exact, world, ms, 1e12)
        fwd_ach = wl.flops_fwd / (kern_ms * 1e-3) / 1e12
        if bwd_ms is not None and bwd_ms > kern_ms:  # the backward dominates the step
            ach = (wl.flops - wl.flops_fwd) / (bwd_ms * 1e-3) / 1e12
            ach_exact = (wl.exact - wl.exact_fwd) / (bwd_ms * 1e-3) / 1e12
            kname = "backward"
        else:
            ach, kname = fwd_ach, wl.kernel
            ach_exact = wl.exact_fwd / (kern_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": bf16, "unit": "TFLOP/s",
                "frac": ach / bf16, "traffic": None, "peak_source": src, "kernel": kname,
                "exact_tflops": ach_exact, "exact_frac": ach_exact / bf16}
        if bwd_ms is not None:
            roof["forward_tflops"] = fwd_ach
            roof["backward_ms"] = bwd_ms
    # (the recorded rows are the default selection rule's, at full size)
    roof["traffic"] = recorded_traffic(args.workload if args.size == "full" and not args.select else "",
                                       roof["kernel"])
    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return
    line = {
        "metric": METRIC, "value": value, "unit": wl.unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": {"fp32": "fp32", "bf16": "bf16"}.get(wl.w.get("dtype"), "u8"),
        "data": "synthetic (seeded generators in sa_workloads)",
        "config": {"workload": args.workload, **({"select": args.select} if args.select else {}),
                   **({"a1": "literal flags computed on the device each step"}
                      if args.flags_on_device else {}),
                   "l2": "inputs larger than L2, no flush",
                   "parallelism": f"independent replica per rank x{world}"},
        "roofline": roof, "clocks": clk,
        "e2e": {"value": e2e_value, "unit": wl.unit, "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h)},
        "gpu_launches": int(wl.kernels_per_step * args.steps),
        "kernel_ms": kern_ms,
    }
    if wl.unit == "TFLOP/s":
        # the same step counted by exact (query, key) edges instead of visited tiles
        line["value_exact_edges"] = value_exact
    if world == 1 and not args.no_cpu_baseline:
        torch.set_num_threads(len(os.sched_getaffinity(0)))
        res = wl.cpu_baseline()
        line["cpu_baseline"] = {"value": res[0], "unit": wl.unit, "cores": len(os.sched_getaffinity(0)),
                                "kind": "oracle", "sample": res[1], "seconds": res[2]}
        if len(res) > 3:
            line["cpu_baseline"]["exact_edges_value"] = res[3]
    print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
