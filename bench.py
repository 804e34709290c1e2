#!/usr/bin/env python
"""Benchmark of the OLMo 3 hybrid sliding-window attention hot path on B200.

One step = one pass of every hot-path step over one batch of synthetic input:
layer types (host), QK-norm + RoPE, KV-cache append, attention (prefill or
decode) for each layer of the workload.  Default workload: the 7B prefill
(B=1, T=8192, H=G=32, d=128, one sliding layer and one full layer), followed by
one decode token per layer so that decode runs in every step too.

Prints ONE JSON line (rank 0).  Time is measured with CUDA events on the
stream the kernels run on, bracketed by a barrier and device synchronisation,
as the max over ranks.  With several GPUs every rank runs an independent
replica (the path has no data-path exchange): scaling is weak.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload 7b-prefill|32b-prefill|7b-decode|32b-decode|ragged-7b-decode|
                              7b-prefill-chunked|32b-prefill-chunked|7b-qkv-proj|32b-qkv-proj|
                              7b-out-proj|32b-out-proj]

The chunked workloads feed the prefill prompt through the chunked-prefill call
(--chunk tokens at a time); the projection workloads time the attention block's
fused QKV projection (+ QK-norm + RoPE) and output side (W_o + reordered norm +
residual) over the prefill workloads' tokens.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "decode attn HBM GB/s & tok/s; prefill TFLOP/s (band), % of B200 roofline"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PROFILES = os.path.join(ROOT, "profiles")
CSRC = os.path.join(ROOT, "hybrid_sliding_window_olmo3_b200", "csrc")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="7b-prefill",
                    choices=["7b-prefill", "32b-prefill", "7b-decode", "32b-decode", "ragged-7b-decode",
                             "7b-prefill-chunked", "32b-prefill-chunked", "7b-out-proj", "32b-out-proj",
                             "7b-qkv-proj", "32b-qkv-proj"])
    ap.add_argument("--chunk", type=int, default=2048, help="prompt chunk of the *-prefill-chunked workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--batch", type=int, default=0, help="override B of a decode workload (small profiling captures)")
    ap.add_argument("--shared-caches", action="store_true",
                    help="decode: one cache per layer type even when per-layer caches would fit")
    return ap.parse_args()


# --------------------------------------------------------------------------
# algorithmic work (closed forms of the mask's row counts min(t + 1, window))
# --------------------------------------------------------------------------
def band_pairs(T: int, window: int, full: bool) -> int:
    if full or window >= T:
        return T * (T + 1) // 2
    return window * (window + 1) // 2 + (T - window) * window


def prefill_flops(B, T, H, d, window, full) -> int:
    return 4 * d * H * B * band_pairs(T, window, full)


def load_peaks():
    if os.path.exists(PEAKS_FILE):
        with open(PEAKS_FILE) as f:
            return json.load(f), "measured"
    return FALLBACK_PEAKS, "fallback"


def traffic_from_profile(kernel_file: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernel source changed since the counters were taken."""
    path = os.path.join(PROFILES, f"{kernel_file[:-3]}_{workload}.md")
    if not os.path.exists(path):
        return None
    txt = open(path).read()
    m_sha = re.search(r"source_sha256:\s*([0-9a-f]{64})", txt)
    m_tr = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    if not m_sha or not m_tr:
        return None
    src = open(os.path.join(CSRC, kernel_file), "rb").read()
    if hashlib.sha256(src).hexdigest() != m_sha.group(1):
        return None
    return float(m_tr.group(1))


# --------------------------------------------------------------------------
# clocks during the timed region
# --------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        if self.proc is None:
            return None
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1].split()[0]))
                mx = float(parts[2].split()[0])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------
# workloads
# --------------------------------------------------------------------------
class PrefillStep:
    """Prefill of T tokens on one sliding and one full layer, then one decode
    token per layer, through the C ABI.  With chunk > 0 the prompt goes in
    pieces of `chunk` tokens through the chunked-prefill entry point (each piece
    attends over the cache the earlier pieces filled)."""

    def __init__(self, name, dev, stream, chunk=0):
        from hybrid_sliding_window_olmo3_b200 import olmo3 as L
        from hybrid_sliding_window_olmo3_b200 import workloads as WL
        self.L = L
        wl = WL.WORKLOADS[name]
        sh = wl.shape
        self.wl, self.sh, self.dev, self.stream = wl, sh, dev, stream
        B, T, H, G, d, W = wl.B, wl.T, sh.H, sh.G, sh.d, sh.window
        self.B, self.T, self.chunk = B, T, chunk
        types = L.layer_types(sh.n_layers)
        self.layers = []
        for li in wl.layers:
            typ = types[li]
            q, k, v, gq, gk = WL.qkv_bf16(B, T, H, G, d, wl.seed, layer=li)
            g = torch.Generator().manual_seed(wl.seed * 7 + li)
            q1 = torch.randn(B, 1, H, d, generator=g).to(torch.bfloat16)
            k1 = torch.randn(B, 1, G, d, generator=g).to(torch.bfloat16)
            v1 = torch.randn(B, 1, G, d, generator=g).to(torch.bfloat16)
            host = dict(q=q, k=k, v=v, gq=gq, gk=gk, q1=q1, k1=k1, v1=v1)
            lay = dict(typ=typ, host={n: t.pin_memory() for n, t in host.items()})
            lay.update({n: t.to(dev) for n, t in host.items()})
            lay["cache"] = L.KVCache(typ, B, G, d, W, capacity=T + 1, device=dev)
            lay["qh"] = torch.empty(B, T, H, d, dtype=torch.bfloat16, device=dev)
            lay["kh"] = torch.empty(B, T, G, d, dtype=torch.bfloat16, device=dev)
            lay["out"] = torch.empty(B, T, H, d, dtype=torch.bfloat16, device=dev)
            lay["qh1"] = torch.empty(B, 1, H, d, dtype=torch.bfloat16, device=dev)
            lay["kh1"] = torch.empty(B, 1, G, d, dtype=torch.bfloat16, device=dev)
            lay["out1"] = torch.empty(B, H, d, dtype=torch.bfloat16, device=dev)
            n_ws = L.attn_decode_workspace_size(B, H, G, d, T + 1, typ, W)
            lay["ws"] = torch.empty(max(n_ws // 4, 4), dtype=torch.float32, device=dev)
            if chunk:
                n_cw = L.attn_prefill_chunk_workspace_size(B, chunk, G, d, typ, W)
                lay["cws"] = torch.empty(max(n_cw, 16), dtype=torch.uint8, device=dev)
                lay["chunks"] = []
                for c0 in range(0, T, chunk):
                    c1 = min(T, c0 + chunk)
                    lay["chunks"].append(dict(
                        c0=c0, q=lay["q"][:, c0:c1].contiguous(), k=lay["k"][:, c0:c1].contiguous(),
                        v=lay["v"][:, c0:c1].contiguous(),
                        qh=torch.empty(B, c1 - c0, H, d, dtype=torch.bfloat16, device=dev),
                        kh=torch.empty(B, c1 - c0, G, d, dtype=torch.bfloat16, device=dev),
                        out=torch.empty(B, c1 - c0, H, d, dtype=torch.bfloat16, device=dev),
                        pos=torch.full((B,), c0, dtype=torch.int32, device=dev)))
            lay["flops"] = prefill_flops(B, T, H, d, W, typ == L.FULL)
            self.layers.append(lay)
        self.pos0 = torch.zeros(B, dtype=torch.int32, device=dev)
        self.posT = torch.full((B,), T, dtype=torch.int32, device=dev)
        self.kvlen = torch.full((B,), T + 1, dtype=torch.int32, device=dev)
        self.flops_per_step = sum(x["flops"] for x in self.layers)
        n_chunks = len(self.layers[0].get("chunks", [])) if chunk else 0
        # one-shot: qknorm, append, prefill, qknorm, append, decode + combine per layer;
        # chunked: per chunk qknorm + chunk call (gather, prefill, append on sliding layers;
        # append, prefill on full layers), then the decode token
        self.launches_per_step = (7 * len(self.layers) if not chunk else
                                  sum(n_chunks * (1 + (3 if x["typ"] == L.SLIDING else 2)) + 4 for x in self.layers))
        self.unit = "TFLOP/s"
        self.h2d = sum(t.numel() * t.element_size() for lay in self.layers for n, t in lay["host"].items())
        self.d2h = sum(lay["out"].numel() * 2 + lay["out1"].numel() * 2 for lay in self.layers)
        self.config = {
            "workload": f"OLMo 3 {sh.name[6:]} prefill attention: B={B}, T={T}, H={H}, G={G}, d={d}, window {W}, "
                        f"layers {list(wl.layers)} (types {[x['typ'] for x in self.layers]}, 0=sliding 1=full), "
                        + (f"prompt in chunks of {chunk} tokens through the chunked-prefill call, " if chunk else "")
                        + "then one decode token per layer",
            "global_batch": B, "seq_len": T,
            "l2": f"inputs larger than L2 ({self.h2d / 2**20:.0f} MiB read per step)",
            "parallelism": "replicas",
        }
        self.kernel_file, self.kernel_name = "attn_prefill.cu", "attn_prefill_kernel"
        self.ev = []

    def step(self, timed_kernel=False, host_io=False):
        L, s = self.L, self.stream
        for lay in self.layers:
            if host_io:
                for n in ("q", "k", "v", "gq", "gk", "q1", "k1", "v1"):
                    lay[n].copy_(lay["host"][n], non_blocking=True)
            if self.chunk:
                if timed_kernel:
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record(s)
                for ch in lay["chunks"]:
                    L.qknorm_rope(ch["q"], ch["k"], lay["gq"], lay["gk"], ch["pos"], q_out=ch["qh"], k_out=ch["kh"],
                                  stream=s)
                    L.attn_prefill_chunk(ch["qh"], ch["kh"], ch["v"], lay["cache"], ch["pos"], out=ch["out"],
                                         workspace=lay["cws"], stream=s)
                if timed_kernel:
                    e1.record(s)
                    self.ev.append((e0, e1, lay["flops"]))
            else:
                L.qknorm_rope(lay["q"], lay["k"], lay["gq"], lay["gk"], self.pos0, q_out=lay["qh"],
                              k_out=lay["kh"], stream=s)
                L.kv_append(lay["cache"], lay["kh"], lay["v"], self.pos0, stream=s)
                if timed_kernel:
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record(s)
                L.attn_prefill(lay["qh"], lay["kh"], lay["v"], lay["typ"], self.sh.window, out=lay["out"], stream=s)
                if timed_kernel:
                    e1.record(s)
                    self.ev.append((e0, e1, lay["flops"]))
            L.qknorm_rope(lay["q1"], lay["k1"], lay["gq"], lay["gk"], self.posT, q_out=lay["qh1"],
                          k_out=lay["kh1"], stream=s)
            L.kv_append(lay["cache"], lay["kh1"], lay["v1"], self.posT, stream=s)
            L.attn_decode(lay["qh1"][:, 0], lay["cache"], self.kvlen, self.T + 1, out=lay["out1"],
                          workspace=lay["ws"], stream=s)
            if host_io:
                lay.setdefault("out_h", torch.empty_like(lay["out"], device="cpu").pin_memory())
                lay.setdefault("out1_h", torch.empty_like(lay["out1"], device="cpu").pin_memory())
                lay["out_h"].copy_(lay["out"], non_blocking=True)
                lay["out1_h"].copy_(lay["out1"], non_blocking=True)

    def work_per_step(self):
        return self.flops_per_step / 1e12  # TFLOP

    def kernel_roofline(self, peaks):
        tot_ms = sum(e0.elapsed_time(e1) for e0, e1, _ in self.ev)
        tot_fl = sum(f for _, _, f in self.ev)
        achieved = tot_fl / (tot_ms * 1e-3) / 1e12
        peak = peaks["bf16_tflops"]
        return {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4), "peak_kind": "measured burst cuBLAS bf16"
                if peaks is not FALLBACK_PEAKS else "fallback burst",
                "kernel": self.kernel_name if not self.chunk else
                "qknorm_rope + attn_prefill_chunk over all chunks of a layer", "launches": len(self.ev),
                "avg_launch_ms": round(tot_ms / max(len(self.ev), 1), 4)}

    def cpu_baseline(self, seconds, rows_per_block=16):
        """The oracle on a bounded sample: QK-norm+RoPE and attention of blocks of
        query rows of every layer, until `seconds` have passed."""
        import oracle.olmo3_oracle as O
        L = self.L
        sh, T = self.sh, self.T
        rng = np.random.default_rng(0)
        data = []
        for lay in self.layers:
            h = lay["host"]
            data.append((lay["typ"], h["q"].float().numpy(), h["k"].float().numpy(), h["v"].float().numpy(),
                         h["gq"].numpy(), h["gk"].numpy()))
        done_fl, t0, blocks = 0, time.perf_counter(), 0
        pos = np.arange(T)[None, :]
        while time.perf_counter() - t0 < seconds:
            for typ, q, k, v, gq, gk in data:
                r0 = int(rng.integers(0, T - rows_per_block))
                rows = np.arange(r0, r0 + rows_per_block)
                lo = 0 if typ == L.FULL else max(0, r0 - sh.window + 1)
                hi = r0 + rows_per_block
                qh, _ = O.qk_norm_rope(q[:, rows], k[:, rows], gq, gk, pos[:, rows], sh.eps, sh.theta)
                _, kh = O.qk_norm_rope(q[:, lo:hi], k[:, lo:hi], gq, gk, pos[:, lo:hi], sh.eps, sh.theta)
                O.attend(qh, pos[:, rows], kh, pos[:, lo:hi], v[:, lo:hi],
                         O.FULL if typ == L.FULL else O.SLIDING, sh.window)
                n_pairs = sum(min(t + 1, T if typ == L.FULL else sh.window) for t in rows)
                done_fl += 4 * sh.d * sh.H * n_pairs
                blocks += 1
        el = time.perf_counter() - t0
        return {"value": done_fl / el / 1e12, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
                "sample": f"{blocks} blocks of {rows_per_block} query rows x {sh.H} heads (QK-norm+RoPE of the "
                          f"rows and their band of keys, then band attention), alternating the layers, "
                          f"{el:.1f} s; numpy einsum, single thread"}


class DecodeStep:
    """One decode token per sequence through every layer of the model pattern."""

    def __init__(self, name, dev, stream, batch=0, shared=False):
        from hybrid_sliding_window_olmo3_b200 import olmo3 as L
        from hybrid_sliding_window_olmo3_b200 import workloads as WL
        self.L = L
        wl = WL.WORKLOADS[name]
        sh = wl.shape
        self.wl, self.sh, self.dev, self.stream = wl, sh, dev, stream
        B, H, G, d, W = (batch or wl.B), sh.H, sh.G, sh.d, sh.window
        self.B = B
        if wl.ragged:
            lens = WL.ragged_lengths(B, wl.seed)
        else:
            lens = np.full(B, wl.context, dtype=np.int64)
        self.lens = lens
        # cache room for the positions of the warm-up, timed and end-to-end steps
        self.extra = int(os.environ.get("OLMO3_BENCH_DECODE_ROOM", "1024"))
        self.types = L.layer_types(sh.n_layers)
        cap_full = int(lens.max()) + self.extra
        per_layer = {L.SLIDING: B * W * G * d * 4, L.FULL: B * cap_full * G * d * 4}
        need = sum(per_layer[t] for t in self.types)
        free = torch.cuda.mem_get_info(dev)[0]
        self.shared = shared or need > 0.8 * free
        caches = {}

        def make(typ, key):
            cap = W if typ == L.SLIDING else cap_full
            c = L.KVCache(typ, B, G, d, W, capacity=cap, device=dev,
                          k=WL.randn_bf16((B * cap, G, d), wl.seed * 100 + key, dev),
                          v=WL.randn_bf16((B * cap, G, d), wl.seed * 100 + key + 50, dev))
            return c
        self.caches = []
        for li, typ in enumerate(self.types):
            key = typ if self.shared else li
            if key not in caches:
                caches[key] = make(typ, key)
            self.caches.append(caches[key])
        g = torch.Generator().manual_seed(wl.seed)
        self.q = torch.randn(B, 1, H, d, generator=g).to(torch.bfloat16).to(dev)
        self.k = torch.randn(B, 1, G, d, generator=g).to(torch.bfloat16).to(dev)
        self.v = torch.randn(B, 1, G, d, generator=g).to(torch.bfloat16).to(dev)
        self.gq = (torch.rand(H * d, generator=g) + 0.5).to(dev)
        self.gk = (torch.rand(G * d, generator=g) + 0.5).to(dev)
        self.host = {n: getattr(self, n).cpu().pin_memory() for n in ("q", "k", "v", "gq", "gk")}
        self.qh = torch.empty(B, 1, H, d, dtype=torch.bfloat16, device=dev)
        self.kh = torch.empty(B, 1, G, d, dtype=torch.bfloat16, device=dev)
        self.out = torch.empty(B, H, d, dtype=torch.bfloat16, device=dev)
        self.out_h = torch.empty(B, H, d, dtype=torch.bfloat16).pin_memory()
        self.pos0 = torch.from_numpy((lens - 1).astype(np.int32)).to(dev)  # each step first advances it
        self.pos = self.pos0.clone()                                          # position of the new token
        self.kvlen = self.pos + 1
        self.g_step = self.g_attn = None
        self.max_len = int(lens.max()) + self.extra
        ws = max(L.attn_decode_workspace_size(B, H, G, d, self.max_len, t, W) for t in (0, 1))
        self.ws = torch.empty(max(ws // 4, 4), dtype=torch.float32, device=dev)
        self.launches_per_step = 5 * len(self.types)
        self.unit = "GB/s"
        self.h2d = sum(t.numel() * t.element_size() for t in self.host.values())
        self.d2h = self.out.numel() * 2
        self.step_idx = 0
        self.ev = []
        self.kernel_file = "attn_decode.cu"
        self.kernel_name = "attn_decode_gqa_kernel" if H > G else "attn_decode_split_kernel"
        self.config = {
            "workload": f"OLMo 3 {sh.name[6:]} decode: {sh.n_layers}-layer pattern, B={B}, "
                        + (f"ragged contexts U[1,65536] (seeded)" if wl.ragged else f"context {wl.context}")
                        + f", H={H}, G={G}, d={d}, window {W}",
            "global_batch": B, "seq_len": int(lens.max()),
            "caches": "one cache per layer type (capacity rule)" if self.shared else "one cache per layer",
            "l2": "inputs larger than L2 (every cache buffer >= 128 MiB, read once per layer)",
            "parallelism": "replicas",
        }

    def _bytes(self, step_idx):
        """K+V bytes of the valid cache entries read by one step (all layers)."""
        sh, W = self.sh, self.sh.window
        L_ = self.lens + step_idx + 1
        row = sh.G * sh.d * 2 * 2
        per = {0: int(np.minimum(L_, W).sum()) * row, 1: int(L_.sum()) * row}
        return sum(per[t] for t in self.types)

    # The decode step is captured in a CUDA graph: a sliding layer of the 32B moves only
    # 134 MB (~20 us of HBM time), less than the host needs to issue its four launches.
    def _body(self):
        """One decode token per sequence through every layer (captured into a graph)."""
        L = self.L
        self.pos.add_(1)
        self.kvlen.copy_(self.pos + 1)
        for li, typ in enumerate(self.types):
            c = self.caches[li]
            L.qknorm_rope(self.q, self.k, self.gq, self.gk, self.pos, q_out=self.qh, k_out=self.kh)
            L.kv_append(c, self.kh, self.v, self.pos)
            L.attn_decode(self.qh[:, 0], c, self.kvlen, self.max_len, out=self.out, workspace=self.ws)

    def _attn_only(self):
        """The decode attention launches of every layer back to back (kernel timing)."""
        for li in range(len(self.types)):
            self.L.attn_decode(self.qh[:, 0], self.caches[li], self.kvlen, self.max_len, out=self.out,
                               workspace=self.ws)

    def _capture(self):
        side = torch.cuda.Stream(self.dev)
        side.wait_stream(torch.cuda.current_stream(self.dev))
        with torch.cuda.stream(side):  # first calls outside capture (one-time kernel attributes)
            self._body()
            self._attn_only()
        torch.cuda.current_stream(self.dev).wait_stream(side)
        torch.cuda.synchronize(self.dev)
        self.pos.copy_(self.pos0)
        self.g_step, self.g_attn = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.g_step):
            self._body()
        with torch.cuda.graph(self.g_attn):
            self._attn_only()
        self.pos.copy_(self.pos0)
        torch.cuda.synchronize(self.dev)

    def step(self, timed_kernel=False, host_io=False):
        if self.g_step is None:
            self._capture()
        if host_io:
            for n in ("q", "k", "v", "gq", "gk"):
                getattr(self, n).copy_(self.host[n], non_blocking=True)
        self.g_step.replay()
        if host_io:
            self.out_h.copy_(self.out, non_blocking=True)
        self.step_idx += 1

    def time_kernel(self, reps):
        """Average duration of the decode attention launches (split + combine), from graph replays."""
        s = torch.cuda.current_stream(self.dev)
        self.g_attn.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for _ in range(reps):
            self.g_attn.replay()
        e1.record(s)
        torch.cuda.synchronize(self.dev)
        n = reps * len(self.types)
        row = self.sh.G * self.sh.d * 4
        Ls = self.lens + self.step_idx  # kv_len after step_idx steps
        per_layer = {0: int(np.minimum(Ls, self.sh.window).sum()) * row, 1: int(Ls.sum()) * row}
        b = reps * sum(per_layer[t] for t in self.types)
        self.ev = [(e0, e1, b, n)]

    def work_per_step(self):
        return self._bytes(self.step_idx) / 1e9  # GB (uses the upcoming step's lengths)

    def kernel_roofline(self, peaks):
        e0, e1, tot_b, n = self.ev[0]
        tot_ms = e0.elapsed_time(e1)
        achieved = tot_b / (tot_ms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "peak_kind": "measured copy" if peaks is not FALLBACK_PEAKS
                else "fallback", "kernel": self.kernel_name + " (+ combine)", "launches": n,
                "avg_launch_ms": round(tot_ms / max(n, 1), 4),
                "timing": "graph of the decode launches of all layers, back to back"}

    def cpu_baseline(self, seconds):
        """The oracle on a bounded sample: QK-norm+RoPE of the new token, its
        cache of one sliding and one full layer, and decode attention, for the
        first and last sequence, until `seconds` of oracle time have passed."""
        import oracle.olmo3_oracle as O
        L = self.L
        sh = self.sh
        q, k = self.host["q"].float().numpy(), self.host["k"].float().numpy()
        gq, gk = self.host["gq"].numpy(), self.host["gk"].numpy()
        done, el, n_calls = 0, 0.0, 0
        while el < seconds:
            for typ in (L.SLIDING, L.FULL):
                c = self.caches[self.types.index(typ)]
                ot = O.SLIDING if typ == L.SLIDING else O.FULL
                for b in (0, self.B - 1):
                    n = int(self.lens[b]) + 1
                    cap = c.capacity
                    first = max(0, n - cap) if typ == L.SLIDING else 0
                    idx = torch.tensor([b * cap + (p % cap if typ == L.SLIDING else p) for p in range(first, n - 1)],
                                       dtype=torch.int64, device=c.k.device)
                    kk = c.k[idx].float().cpu().numpy()
                    vv = c.v[idx].float().cpu().numpy()
                    t1 = time.perf_counter()
                    qh, kh = O.qk_norm_rope(q[b:b + 1], k[b:b + 1], gq, gk, np.array([[n - 1]]), sh.eps, sh.theta)
                    oc = O.KVCache(ot, cap, sh.G, sh.d)
                    oc.append(range(first, n - 1), kk, vv)
                    oc.append([n - 1], kh[0], self.host["v"][b].float().numpy())
                    O.decode_attention(qh[:, 0], [oc], [n - 1], ot, sh.window)
                    el += time.perf_counter() - t1
                    done += (n - first) * sh.G * sh.d * 4
                    n_calls += 1
        return {"value": done / el / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
                "sample": f"{n_calls} decode calls (QK-norm+RoPE, cache fill, attention; sequences 0 and B-1, "
                          f"one sliding and one full layer), {el:.1f} s of oracle time; numpy, single thread"}


class OutProjStep:
    """The attention block's output side for a whole prompt: h = x + RMSNorm(attn W_o^T) * gain
    (one persistent tcgen05 GEMM whose epilogue applies the row norm and the residual)."""

    def __init__(self, name, dev, stream):
        from hybrid_sliding_window_olmo3_b200 import olmo3 as L
        from hybrid_sliding_window_olmo3_b200 import workloads as WL
        self.L = L
        wl = WL.WORKLOADS[name.replace("out-proj", "prefill")]
        sh = wl.shape
        self.sh, self.dev, self.stream = sh, dev, stream
        M, K = wl.B * wl.T, sh.H * sh.d
        D = {"olmo3-7b": 4096, "olmo3-32b": 5120}[sh.name]
        self.M, self.D, self.K = M, D, K
        host = dict(attn=WL.randn_bf16((M, K), wl.seed + 11), x=WL.randn_bf16((M, D), wl.seed + 12),
                    w=(WL.randn_bf16((D, K), wl.seed + 13).float() / K ** 0.5).to(torch.bfloat16),
                    g=torch.rand(D, generator=torch.Generator().manual_seed(wl.seed)) + 0.5)
        self.host = {n: t.pin_memory() for n, t in host.items()}
        for n, t in host.items():
            setattr(self, n, t.to(dev))
        self.h = torch.empty(M, D, dtype=torch.bfloat16, device=dev)
        self.h_host = torch.empty(M, D, dtype=torch.bfloat16).pin_memory()
        self.ws = torch.empty(L.out_proj_workspace_size(M, D), dtype=torch.uint8, device=dev)
        self.flops = 2 * M * D * K
        self.unit = "TFLOP/s"
        self.launches_per_step = 1  # the GEMM (plus a memset of the row sums and counters)
        self.h2d = sum(t.numel() * t.element_size() for t in self.host.values())
        self.d2h = M * D * 2
        self.ev = []
        self.kernel_file, self.kernel_name = "proj_gemm.cu", "proj_gemm_kernel<PostNormEpilogue>"
        self.config = {"workload": f"OLMo 3 {sh.name[6:]} attention output side: h = x + RMSNorm(attn W_o^T), "
                                   f"M={M} tokens, K={K}, D={D}, bf16",
                       "global_batch": wl.B, "seq_len": wl.T, "l2": "inputs larger than L2", "parallelism": "replicas"}

    def step(self, timed_kernel=False, host_io=False):
        s = self.stream
        if host_io:
            for n in ("attn", "x", "w", "g"):
                getattr(self, n).copy_(self.host[n], non_blocking=True)
        if timed_kernel:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s)
        self.L.out_proj_postnorm_residual(self.attn, self.w, self.g, self.x, h_out=self.h, workspace=self.ws,
                                          stream=s)
        if timed_kernel:
            e1.record(s)
            self.ev.append((e0, e1, self.flops))
        if host_io:
            self.h_host.copy_(self.h, non_blocking=True)

    def work_per_step(self):
        return self.flops / 1e12

    def kernel_roofline(self, peaks):
        tot_ms = sum(e0.elapsed_time(e1) for e0, e1, _ in self.ev)
        achieved = sum(f for _, _, f in self.ev) / (tot_ms * 1e-3) / 1e12
        peak = peaks["bf16_tflops"]
        return {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4), "peak_kind": "measured burst cuBLAS bf16",
                "kernel": self.kernel_name, "launches": len(self.ev),
                "avg_launch_ms": round(tot_ms / max(len(self.ev), 1), 4)}

    def cpu_baseline(self, seconds):
        import oracle.olmo3_oracle as O
        a, w, x, g = (self.host[n].float().numpy() for n in ("attn", "w", "x", "g"))
        done, el, rows = 0, 0.0, 0
        rng = np.random.default_rng(0)
        while el < seconds:
            r = rng.integers(0, self.M, 8)
            t0 = time.perf_counter()
            O.out_proj_postnorm_residual(x[r], a[r], w, g)
            el += time.perf_counter() - t0
            done += 2 * 8 * self.D * self.K
            rows += 8
        try:
            from threadpoolctl import threadpool_info
            cores = max([i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"] or [1])
        except Exception:  # noqa: BLE001 - reporting only
            cores = len(os.sched_getaffinity(0))
        return {"value": done / el / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                "sample": f"{rows} rows (fp64 matmul with W_o, norm, residual), {el:.1f} s; numpy (BLAS threads)"}


class QkvProjStep(OutProjStep):
    """The attention block's input side for a whole prompt: [q|k|v] = x W_qkv^T, then QK-norm
    + RoPE on q and k (one persistent tcgen05 GEMM with the norm and rotation in its epilogue)."""

    def __init__(self, name, dev, stream):
        from hybrid_sliding_window_olmo3_b200 import olmo3 as L
        from hybrid_sliding_window_olmo3_b200 import workloads as WL
        self.L = L
        wl = WL.WORKLOADS[name.replace("qkv-proj", "prefill")]
        sh = wl.shape
        self.sh, self.dev, self.stream, self.wl = sh, dev, stream, wl
        D = {"olmo3-7b": 4096, "olmo3-32b": 5120}[sh.name]
        M, N = wl.B * wl.T, (sh.H + 2 * sh.G) * sh.d
        self.M, self.D, self.K, self.N = M, N, D, N
        host = dict(x=WL.randn_bf16((wl.B, wl.T, D), wl.seed + 21),
                    w=(WL.randn_bf16((N, D), wl.seed + 22).float() / D ** 0.5).to(torch.bfloat16),
                    gq=torch.rand(sh.H * sh.d, generator=torch.Generator().manual_seed(wl.seed + 23)) + 0.5,
                    gk=torch.rand(sh.G * sh.d, generator=torch.Generator().manual_seed(wl.seed + 24)) + 0.5,
                    pos=torch.zeros(wl.B, dtype=torch.int32))
        self.host = {n: t.pin_memory() for n, t in host.items()}
        for n, t in host.items():
            setattr(self, n, t.to(dev))
        B, T = wl.B, wl.T
        self.outs = (torch.empty(B, T, sh.H, sh.d, dtype=torch.bfloat16, device=dev),
                     torch.empty(B, T, sh.G, sh.d, dtype=torch.bfloat16, device=dev),
                     torch.empty(B, T, sh.G, sh.d, dtype=torch.bfloat16, device=dev))
        self.outs_host = tuple(torch.empty(o.shape, dtype=torch.bfloat16).pin_memory() for o in self.outs)
        self.ws = torch.empty(L.qkv_proj_workspace_size(M), dtype=torch.uint8, device=dev)
        self.flops = 2 * M * N * D
        self.unit = "TFLOP/s"
        self.launches_per_step = 1  # the GEMM (plus a memset of the row sums and counters)
        self.h2d = sum(t.numel() * t.element_size() for t in self.host.values())
        self.d2h = M * N * 2
        self.ev = []
        self.kernel_file, self.kernel_name = "proj_gemm.cu", "proj_gemm_kernel<QkvEpilogue<128>>"
        self.config = {"workload": f"OLMo 3 {sh.name[6:]} attention input side: [q|k|v] = x W_qkv^T + QK-norm + "
                                   f"RoPE, M={M} tokens, D={D}, N={N} (H={sh.H}, G={sh.G}, d={sh.d}), bf16",
                       "global_batch": wl.B, "seq_len": wl.T, "l2": "inputs larger than L2", "parallelism": "replicas"}

    def step(self, timed_kernel=False, host_io=False):
        s, sh = self.stream, self.sh
        if host_io:
            for n in ("x", "w", "gq", "gk", "pos"):
                getattr(self, n).copy_(self.host[n], non_blocking=True)
        if timed_kernel:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s)
        q, k, v = self.outs
        self.L.qkv_proj_qknorm_rope(self.x, self.w, self.gq, self.gk, self.pos, sh.H, sh.G, sh.d, theta=sh.theta,
                                    q_out=q, k_out=k, v_out=v, workspace=self.ws, stream=s)
        if timed_kernel:
            e1.record(s)
            self.ev.append((e0, e1, self.flops))
        if host_io:
            for o, h in zip(self.outs, self.outs_host):
                h.copy_(o, non_blocking=True)

    def cpu_baseline(self, seconds):
        import oracle.olmo3_oracle as O
        sh = self.sh
        x, w, gq, gk = (self.host[n].float().numpy() for n in ("x", "w", "gq", "gk"))
        x = x.reshape(self.M, self.K)
        done, el, rows = 0, 0.0, 0
        rng = np.random.default_rng(0)
        while el < seconds:
            r = rng.integers(0, self.M, 8)
            pos = (r % self.wl.T)[None]
            t0 = time.perf_counter()
            O.qkv_projection(x[r][None], w, gq, gk, pos, sh.H, sh.G, sh.d, theta=sh.theta)
            el += time.perf_counter() - t0
            done += 2 * 8 * self.N * self.K
            rows += 8
        try:
            from threadpoolctl import threadpool_info
            cores = max([i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"] or [1])
        except Exception:  # noqa: BLE001 - reporting only
            cores = len(os.sched_getaffinity(0))
        return {"value": done / el / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                "sample": f"{rows} rows (fp64 matmul with W_qkv, QK-norm, RoPE), {el:.1f} s; numpy (BLAS threads)"}


def make_workload(name, dev, stream, batch=0, shared=False, chunk=0):
    if name.endswith("qkv-proj"):
        return QkvProjStep(name, dev, stream)
    if name.endswith("out-proj"):
        return OutProjStep(name, dev, stream)
    if name.endswith("prefill"):
        return PrefillStep(name, dev, stream)
    if name.endswith("prefill-chunked"):
        return PrefillStep(name[:-len("-chunked")], dev, stream, chunk=chunk)
    return DecodeStep(name, dev, stream, batch, shared)


# --------------------------------------------------------------------------
def reduce_over_ranks(dist, dev, ms, work, ms_e2e, work_e2e):
    """Replicas only: the step time is the slowest rank's, the work is the sum of
    all ranks' (value = total work / max time).  Returns (ms_max, work_sum,
    ms_e2e_max, work_e2e_sum); without a process group the rank's own figures."""
    if dist is None:
        return ms, work, ms_e2e, work_e2e
    t = torch.tensor([ms, work, ms_e2e, work_e2e], dtype=torch.float64, device=dev)
    tmax, tsum = t.clone(), t.clone()
    dist.all_reduce(tmax, op=dist.ReduceOp.MAX)
    dist.all_reduce(tsum, op=dist.ReduceOp.SUM)
    return tmax[0].item(), tsum[1].item(), tmax[2].item(), tsum[3].item()


def run_ours(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    stream = torch.cuda.current_stream(dev)
    wk = make_workload(args.workload, dev, stream, args.batch, args.shared_caches, args.chunk)
    peaks, peak_src = load_peaks()

    def barrier():
        torch.cuda.synchronize(dev)
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    work = 0.0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:  # started before the warm-up so that it is sampling when timing begins
        for _ in range(args.warmup):
            wk.step()
        barrier()
        e0.record(stream)
        for _ in range(args.steps):
            work += wk.work_per_step()
            wk.step(timed_kernel=True)
        e1.record(stream)
        barrier()
    ms = e0.elapsed_time(e1)
    if hasattr(wk, "time_kernel"):
        wk.time_kernel(max(3, min(args.steps, 50)))
    roof = wk.kernel_roofline(peaks)

    e2e = None
    if not args.no_e2e:
        for _ in range(2):
            wk.step(host_io=True)
        barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        work_e = 0.0
        f0.record(stream)
        for _ in range(args.steps):
            work_e += wk.work_per_step()
            wk.step(host_io=True)
        f1.record(stream)
        barrier()
        ms_e = f0.elapsed_time(f1)
        e2e = (work_e, ms_e)

    ms_max, work_tot, ms_e_max, work_e_tot = reduce_over_ranks(
        dist, dev, ms, work, e2e[1] if e2e else 0.0, e2e[0] if e2e else 0.0)

    if rank == 0:
        scale = 1.0  # TFLOP per ms*1e-3 -> TFLOP/s ; GB per s -> GB/s
        value = work_tot / (ms_max * 1e-3) * scale
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": wk.unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_max / args.steps, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": wk.config, "impl": "ours",
            "gpu_launches": wk.launches_per_step * args.steps,
            "roofline": None, "clocks": clk.summary(), "peaks_source": peak_src,
        }
        roof["traffic"] = traffic_from_profile(wk.kernel_file, args.workload)
        line["roofline"] = roof
        if args.workload.endswith("decode"):
            line["tok_per_s"] = round(wk.B * world * args.steps / (ms_max * 1e-3), 1)
        if e2e:
            line["e2e"] = {"value": round(work_e_tot / (ms_e_max * 1e-3), 2), "unit": wk.unit,
                           "h2d_bytes_per_step": wk.h2d, "d2h_bytes_per_step": wk.d2h}
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = wk.cpu_baseline(args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def run_reference(args):
    """The oracle as it stands, on the host cores, on bounded samples of the
    same workload: rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    dev = torch.device("cuda", 0) if torch.cuda.is_available() else None
    if dev is None:
        print(json.dumps({"impl": "reference", "unavailable": "the sampled workload is generated on a CUDA device"}))
        return
    wk = make_workload(args.workload, dev, torch.cuda.current_stream(dev), args.batch, args.shared_caches,
                       args.chunk)
    per = []
    for i in range(args.warmup + args.steps):
        cb = wk.cpu_baseline(max(2.0, min(8.0, 150.0 / (args.warmup + args.steps))))
        if i >= args.warmup:
            per.append(cb)
    value = statistics.median(c["value"] for c in per)
    cb = dict(per[-1])
    cb["value"] = value
    line = {"metric": METRIC, "value": value, "unit": wk.unit, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": wk.config, "impl": "reference",
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": wk.unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    os.environ.setdefault("OLMO3_BENCH_DECODE_ROOM", str(args.warmup + 2 * args.steps + 64))
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
