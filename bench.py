"""CSA2 decode benchmark on B200: queries/s and HBM GB/s of the whole hot path.

One step = one pass of the CSA2 path over one batch of synthetic, seeded inputs:
FP4 quantize-on-write of the new entries, indexer scoring + exact Top-K (and the candidate
pool / Reindex / Reuse layers the workload has), then the fused gather + dequant + sparse /
sliding-window attention of every layer. Everything runs in libcsa2's kernels.

Default workload: Full-mode decode, batch 32, 65,536-token context at compression ratio 2
(32,768 compressed entries per sequence), FP8 indexer keys with 64 heads, Top-512, 64 query
heads of 512 channels, 128-row FP8 window.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference] [--workload NAME]

For N > 1 bench.py starts N ranks itself (torch.distributed.run on 127.0.0.1) unless it
already runs under a launcher: every rank runs its own batch (weak scaling, no collective on
the data path); the time is the max over ranks.
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from fp4_compressed_sparse_quantize_b200 import csa2, synth  # noqa: E402

DEFAULT_WORKLOAD = "decode_full_b32_ctx64k_r2"
# reported beside the default line: the rest of the 64K-1M decode range and the prefill chunk
EXTRA_DECODE = ("decode_group4_b64_ctx256k", "decode_pool_reindex_b4_ctx1m",
                "decode_full_b32_ctx64k_r2_key68")
EXTRA_PREFILL = "prefill_b2_t4k_ctx128k_r2"
L2_FLUSH_BYTES = 256 << 20
SCAN_KERNEL_SRC = os.path.join(ROOT, "fp4_compressed_sparse_quantize_b200", "csrc", "indexer.cu")

# DRAM traffic of one indexer-scan launch, from `ncu --metrics dram__bytes_read.sum,
# dram__bytes_write.sum` (summary in profiles/), valid only for the indexer.cu it was taken
# on: {workload: (sha1 of indexer.cu, bytes per launch)}.
# device buffer sets of the end-to-end pipeline (step inputs and outputs)
E2E_SETS = 3

SCAN_TRAFFIC = {
    "decode_full_b32_ctx64k_r2": ("000c6d6bf38b6d6fecd39db36f22a85ceb28acdd",
                                  134714368 + 3515904),
}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ---- clocks sampler ------------------------------------------------------------------------

class Clocks:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
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
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---- workload ----------------------------------------------------------------------------

class Decode:
    """Device-resident state of one decode workload plus its per-step inputs."""

    def __init__(self, w, seed, dev):
        self.w = w
        self.dev = dev
        self.seed = seed
        B, N, cap = w.B, w.N, w.cap
        self.tau = 1.0 / math.sqrt(synth.D_MAIN)
        # layers' query-side inputs; planted keys follow the layers' indexer queries
        self.layers = [synth.layer_inputs(w, li, seed, dev) for li in range(len(w.layers))]
        dirs = None
        if w.planted:
            dirs = synth.planted_direction([L["q_I"] for L, m in zip(self.layers, w.layers)
                                            if m in ("full", "reindex")])
        self.k_I, self.planted = synth.indexer_keys(w, seed, dev, planted_dirs=dirs)
        if w.key_format == "fp4":
            # compact 68-byte keys, written by the library's key quantiser
            kb = self.k_I
            self.k_I = csa2.Fp4Keys(B, cap, device=dev)
            csa2.quantize_keys_fp4(kb, torch.zeros(B, dtype=torch.int32, device=dev), self.k_I)
            del kb
        # FP4 cache built once by the library's own quantize-on-write
        self.codes = torch.zeros((B, cap, 256), dtype=torch.uint8, device=dev)
        self.scales = torch.zeros((B, cap, 32), dtype=torch.uint8, device=dev)
        chunk = max(1, (1 << 28) // (cap * 1024))
        for b0 in range(0, B, chunk):
            b1 = min(B, b0 + chunk)
            src = torch.empty((b1 - b0, cap, synth.D_MAIN), dtype=torch.bfloat16, device=dev)
            for b in range(b0, b1):
                src[b - b0] = _main_rows(w, seed, b, dev)
            csa2.quantize_kv(src, torch.zeros(b1 - b0, dtype=torch.int32, device=dev),
                             self.codes[b0:b1], self.scales[b0:b1])
            del src
        self.n_vis = synth.decode_positions(w, dev)
        self.dst = (self.n_vis - 1).contiguous()
        # the newest entry is re-quantised every step from its bf16 row
        self.kv_new = torch.stack([_main_rows(w, seed, b, dev)[N - 1:N] for b in range(B)])
        self.idx = [torch.empty((B, 1, w.K), dtype=torch.int32, device=dev) for _ in w.layers]
        self.out = [torch.empty((B, w.H, synth.D_MAIN), dtype=torch.float32, device=dev)
                    for _ in w.layers]
        self.pool = None
        if w.pool:
            self.pool = torch.empty((B, 1, synth.POOL_BLOCKS * synth.POOL_BLOCK),
                                    dtype=torch.int32, device=dev)
        P = synth.POOL_BLOCKS * synth.POOL_BLOCK
        ws_i = max(csa2.workspace_bytes(0, B, 1, w.H_I, cap, w.K,
                                        synth.POOL_BLOCKS if w.pool else 0),
                   csa2.workspace_bytes(0, B, 1, w.H_I, P, w.K))
        self.ws_idx = csa2.new_workspace(ws_i)
        self.ws_attn = csa2.new_workspace(csa2.workspace_bytes(1, B, 1, w.H, cap, w.K))
        torch.cuda.synchronize()

    def step(self, scan_events=None, attn_events=None, stream=None):
        """One decode step. scan_events: (start, stop) around the first Full layer's indexer
        scan; attn_events: one (start, stop) pair per layer around its attention call (both
        become external event nodes when the step is captured into a graph)."""
        w = self.w
        csa2.quantize_kv(self.kv_new, self.dst, self.codes, self.scales,
                         status=self.ws_idx[:4].view(torch.int32), stream=stream)
        cur = None
        for li, mode in enumerate(w.layers):
            L = self.layers[li]
            if mode == "full":
                if scan_events is not None:
                    csa2.set_stage_events(*scan_events)
                    scan_events = None
                csa2.index_score_topk("full", L["q_I"], L["w"], self.k_I, w.K, self.idx[li],
                                      self.ws_idx, n_vis0=self.n_vis, pool_out=self.pool,
                                      pool_blocks=synth.POOL_BLOCKS if w.pool else 0,
                                      stream=stream)
                cur = self.idx[li]
            elif mode == "reindex":
                csa2.index_score_topk("reindex", L["q_I"], L["w"], self.k_I, w.K, self.idx[li],
                                      self.ws_idx, n_vis0=self.n_vis, pool_in=self.pool,
                                      stream=stream)
                cur = self.idx[li]
            else:
                csa2.index_score_topk("reuse", L["q_I"], L["w"], self.k_I, w.K, cur,
                                      self.ws_idx, n_vis0=self.n_vis, stream=stream)
            if attn_events is not None:
                csa2.record_event(attn_events[li][0], stream)
            csa2.sparse_attn_decode(mode, L["q"], self.codes, self.scales, cur.view(w.B, w.K),
                                    L["swa"], self.out[li], self.ws_attn, scale=self.tau,
                                    stream=stream)
            if attn_events is not None:
                csa2.record_event(attn_events[li][1], stream)

    def launches_per_step(self):
        """Kernels of this library per step (memsets excluded)."""
        n = 1  # quantize
        for m in self.w.layers:
            if m == "full":
                n += 3 + (1 if self.w.pool else 0)   # prep, scan, Top-K (+ pool Top-K)
            elif m == "reindex":
                n += 3
            n += csa2.sparse_attn_decode_launches(self.w.B, self.w.K, synth.WINDOW)
        return n

    def step_inputs(self):
        """Per-step host->device inputs: every layer's queries and window rows, the new row."""
        t = [self.kv_new]
        for L in self.layers:
            t += [L["q_I"], L["w"], L["q"], L["swa"]]
        return t

    def step_outputs(self):
        return self.out

    def set_io(self, ins, outs):
        """Point the step at another set of per-step inputs and outputs (the order of
        step_inputs / step_outputs)."""
        self.kv_new = ins[0]
        for li, L in enumerate(self.layers):
            L["q_I"], L["w"], L["q"], L["swa"] = ins[1 + 4 * li:5 + 4 * li]
        self.out = list(outs)

    def algorithmic_bytes(self):
        w = self.w
        B, N, K, H, W = w.B, w.N, w.K, w.H, synth.WINDOW
        ek = 2 if w.idx_dtype == "bf16" else 1
        kb = 68 if w.key_format == "fp4" else 128 * ek      # indexer-key bytes per entry
        tot = B * (512 * 2 + 288)                         # quantize-on-write
        scan = 0
        for m in w.layers:
            if m in ("full", "reindex"):
                rows = N if m == "full" else synth.POOL_BLOCKS * synth.POOL_BLOCK
                b = B * (rows * kb + w.H_I * 128 * ek + w.H_I * 4 + K * 4)
                if m == "full":
                    scan = B * (N * kb + w.H_I * 128 * ek + w.H_I * 4)
                if m == "reindex":
                    b += B * rows * 4
                if m == "full" and w.pool:
                    b += B * synth.POOL_BLOCKS * synth.POOL_BLOCK * 4
                tot += b
            tot += B * (K * 4 + K * 288 + W * 512 + H * 512 * 2 + H * 512 * 4)
        return tot, scan

    def attention_bytes(self):
        """Algorithmic bytes of every layer's decode attention in one step: per query the
        K indices, the K gathered FP4 entries (288 B), the W window rows (512 B E4M3), the bf16
        query and the fp32 output."""
        w = self.w
        per_q = w.K * 4 + w.K * 288 + synth.WINDOW * 512 + w.H * 512 * 2 + w.H * 512 * 4
        return len(w.layers) * w.B * per_q


def packed_like(tensors, device):
    """One uint8 buffer (pinned when on the host) holding room for every tensor at a
    256-byte aligned offset, and a view of it per tensor with the tensor's shape and dtype."""
    offs, o = [], 0
    for t in tensors:
        offs.append(o)
        o = (o + t.numel() * t.element_size() + 255) // 256 * 256
    host = str(device) == "cpu"
    buf = torch.empty(o, dtype=torch.uint8, device=device, pin_memory=host)
    views = [buf[a:a + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
             for a, t in zip(offs, tensors)]
    return buf, views


def flush_l2(buf, k):
    """Evict L2 between timed steps: write a buffer twice the size of L2, then read it back
    so that the dirty lines are written to HBM here and not during the next step."""
    buf.fill_(k & 0xFF)
    torch.sum(buf.view(torch.int64))


def capture_steps(state, events, attn_events, stream):
    """One CUDA graph per timed step: the step's library calls, with that step's scan events
    and per-layer attention events recorded inside (as external event nodes)."""
    graphs = []
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        state.step()                      # warm the side stream
    stream.wait_stream(side)
    torch.cuda.synchronize()
    for ev, aev in zip(events, attn_events):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            state.step(scan_events=ev, attn_events=aev, stream=side)
        graphs.append(g)
    torch.cuda.synchronize()
    return graphs


def capture_plain(state, stream):
    """One CUDA graph of a whole step with no events inside: the graph the step time is
    taken on, so that no event node sits between two kernels that could overlap."""
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        state.step()
    stream.wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        state.step(stream=side)
    torch.cuda.synchronize()
    return g


def _event_pair():
    pair = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    return pair


def timed_decode(state, steps, warmup, stream, local, eager=False, pg=None):
    """Warm up, then time `steps` decode steps (one graph replay each, L2 flushed between
    them outside the events). The step times come from a graph with no event inside; then
    `steps` more replays of graphs with events around the scan and each layer's attention
    give the kernel times. Returns a dict of the device-timed figures (milliseconds) and the
    clocks seen over both passes."""
    w = state.w
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=stream.device)
    for _ in range(max(3, warmup)):
        state.step()
    torch.cuda.synchronize()
    assert csa2.read_device_status(state.ws_idx) == 0, "device status set during warm-up"
    assert csa2.read_device_status(state.ws_attn) == 0
    ev = [_event_pair() for _ in range(steps)]
    sev = [_event_pair() for _ in range(steps)]
    aev = [[_event_pair() for _ in w.layers] for _ in range(steps)]
    for pair in sev + [p for step in aev for p in step]:   # events exist once recorded
        pair[0].record(stream)
        pair[1].record(stream)
    # Each timed step is one CUDA-graph replay of the whole step (captured once per step so
    # that every replay records its own events): launches reach the GPU back to back.
    graphs = capture_steps(state, sev, aev, stream) if not eager else None
    plain = capture_plain(state, stream) if not eager else None
    # every graph is launched once before the timed replays (a graph's first launch also
    # uploads it); these warm replays record the events again in the timed pass below
    for g in (graphs or []) + ([plain] if plain else []):
        g.replay()
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    clocks = Clocks(local)
    clocks.start()
    for k in range(steps):
        flush_l2(flush, k)                      # evict L2 between steps (outside the events)
        ev[k][0].record(stream)
        if plain:
            plain.replay()
        else:
            state.step()
        ev[k][1].record(stream)
    for k in range(steps):                      # kernel times: events inside the step
        flush_l2(flush, k)
        if graphs:
            graphs[k].replay()
        else:
            state.step(scan_events=sev[k], attn_events=aev[k])
    torch.cuda.synchronize()
    clk = clocks.stop()
    if pg:
        pg.barrier()
    del graphs, plain, flush
    step_ms = [a.elapsed_time(b) for a, b in ev]
    has_scan = any(m == "full" for m in w.layers)
    scan_ms = [a.elapsed_time(b) for a, b in sev] if has_scan else [0.0]
    attn_ms = [sum(a.elapsed_time(b) for a, b in step) for step in aev]
    return {"step_ms": step_ms, "scan_ms": scan_ms, "attn_ms": attn_ms, "clocks": clk}


def decode_summary(state, tm, peak):
    """Per-workload figures of a timed_decode run: queries/s, the step's HBM rate and the
    rooflines of the indexer scan (the dominant kernel) and of the decode attention (row
    staging + attention kernels, every layer), each as algorithmic bytes over device time."""
    w = state.w
    steps = len(tm["step_ms"])
    per_step = sum(tm["step_ms"]) / steps
    alg, scan_bytes = state.algorithmic_bytes()
    scan_avg = sum(tm["scan_ms"]) / len(tm["scan_ms"])
    attn_avg = sum(tm["attn_ms"]) / steps
    ab = state.attention_bytes()
    out = {"queries_per_s": w.B / (per_step / 1e3), "ms_per_step": per_step,
           "hbm_gbs_step": alg / (per_step / 1e3) / 1e9,
           "step_roofline_frac": alg / (per_step / 1e3) / 1e9 / peak,
           "attention": {"bound": "hbm", "bytes_per_step": ab, "avg_ms_per_step": attn_avg,
                         "achieved": ab / (attn_avg / 1e3) / 1e9, "peak": peak, "unit": "GB/s",
                         "frac": ab / (attn_avg / 1e3) / 1e9 / peak}}
    if scan_bytes:
        out["scan"] = {"bound": "hbm", "bytes_per_launch": scan_bytes, "avg_launch_ms": scan_avg,
                       "achieved": scan_bytes / (scan_avg / 1e3) / 1e9, "peak": peak,
                       "unit": "GB/s", "frac": scan_bytes / (scan_avg / 1e3) / 1e9 / peak}
    return out


def extra_decode(name, args, dev, local):
    """A shorter timed run of another decode workload (its own state, freed afterwards)."""
    w = synth.WORKLOADS[name]
    state = Decode(w, args.seed, dev)
    tm = timed_decode(state, args.extra_steps, 3, torch.cuda.current_stream(dev), local)
    peak, _ = peaks()
    out = decode_summary(state, tm, peak)
    out.update({"steps": args.extra_steps, "batch": w.B, "context_tokens": w.ctx,
                "compressed_entries": w.N, "layers": list(w.layers), "clocks": tm["clocks"],
                "device_status": [csa2.read_device_status(state.ws_idx),
                                  csa2.read_device_status(state.ws_attn)]})
    del state
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def max_over_ranks(ms, pg, dev):
    """Device-timed milliseconds of this rank -> the slowest rank's (every rank gets it)."""
    if pg is None:
        return float(ms)
    t = torch.tensor([float(ms)], dtype=torch.float64, device=dev)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def job_throughput(batch_per_rank, world, steps, total_ms):
    """Whole-job queries/s: every rank's queries over the slowest rank's time."""
    return batch_per_rank * world * steps / (total_ms / 1e3)


def rank_seed(seed, rank):
    """Each rank draws its own independent batch."""
    return seed + 7919 * rank


class Prefill:
    """Device-resident state of the chunked-prefill workload plus its per-step inputs."""

    def __init__(self, w, seed, dev):
        self.w = w
        self.dev = dev
        self.seed = seed
        B, T, cap, K = w.B, w.T, w.cap, w.K
        self.tau = 1.0 / math.sqrt(synth.D_MAIN)
        self.L = synth.layer_inputs(w, 0, seed, dev)
        self.k_I, _ = synth.indexer_keys(w, seed, dev)
        self.n_old = w.ctx // w.ratio
        self.codes = torch.zeros((B, cap, 256), dtype=torch.uint8, device=dev)
        self.scales = torch.zeros((B, cap, 32), dtype=torch.uint8, device=dev)
        src = torch.stack([_main_rows(w, seed, b, dev) for b in range(B)])
        csa2.quantize_kv(src[:, :self.n_old], torch.zeros(B, dtype=torch.int32, device=dev),
                         self.codes, self.scales)
        self.kv_new = src[:, self.n_old:].contiguous()
        del src
        self.dst = torch.full((B,), self.n_old, dtype=torch.int32, device=dev)
        self.q_pos0 = synth.prefill_positions(w, dev)
        self.idx = torch.empty((B, T, K), dtype=torch.int32, device=dev)
        self.out = torch.empty((B, T, w.H, synth.D_MAIN), dtype=torch.float32, device=dev)
        self.ws = csa2.new_workspace(csa2.workspace_bytes(0, B, T, w.H_I, cap, K))
        self.wsa = csa2.new_workspace(csa2.workspace_bytes(2, B, T, w.H, cap, K))
        torch.cuda.synchronize()

    def step(self, scan_events=None, attn_events=None, stream=None):
        w = self.w
        csa2.quantize_kv(self.kv_new, self.dst, self.codes, self.scales,
                         status=self.ws[:4].view(torch.int32), stream=stream)
        if scan_events is not None:
            csa2.set_stage_events(*scan_events)
        csa2.index_score_topk("full", self.L["q_I"], self.L["w"], self.k_I, w.K, self.idx,
                              self.ws, q_pos0=self.q_pos0, ratio=w.ratio, stream=stream)
        if attn_events is not None:
            attn_events[0].record(stream or torch.cuda.current_stream())
        csa2.sparse_attn_prefill(self.L["q"], self.codes, self.scales, self.idx, self.L["swa"],
                                 self.out, self.wsa, synth.WINDOW, q_pos0=self.q_pos0,
                                 scale=self.tau, stream=stream)
        if attn_events is not None:
            attn_events[1].record(stream or torch.cuda.current_stream())

    def flops(self):
        """Algorithmic FLOPs of one step: the indexer over every causally visible
        (token, entry) pair and the attention (S and P x V) over K + W rows per token."""
        w = self.w
        vis = sum((w.ctx + t + 1) // w.ratio for t in range(w.T))
        scan = w.B * vis * w.H_I * synth.D_IDX * 2
        attn = w.B * w.T * w.H * (w.K + synth.WINDOW) * synth.D_MAIN * 2 * 2
        return scan, attn


def measure_prefill(w, seed, steps, warmup, dev):
    """Time `steps` chunked-prefill steps with the scan and attention events inside; returns
    the tokens/s and the tensor-roofline figures of the indexer scan and the attention."""
    state = Prefill(w, seed, dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(max(3, warmup)):
        state.step()
    torch.cuda.synchronize()
    assert csa2.read_device_status(state.ws) == 0 and csa2.read_device_status(state.wsa) == 0
    mk = lambda: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    ev = [mk() for _ in range(steps)]
    sev = [mk() for _ in range(steps)]
    aev = [mk() for _ in range(steps)]
    for pair in sev + aev:
        pair[0].record(stream)
        pair[1].record(stream)
    torch.cuda.synchronize()
    clocks = Clocks(local_rank())
    clocks.start()
    for k in range(steps):
        ev[k][0].record(stream)
        state.step(scan_events=sev[k], attn_events=aev[k])
        ev[k][1].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    st = [csa2.read_device_status(state.ws), csa2.read_device_status(state.wsa)]
    total_ms = sum(a.elapsed_time(b) for a, b in ev)
    scan_ms = sum(a.elapsed_time(b) for a, b in sev) / steps
    attn_ms = sum(a.elapsed_time(b) for a, b in aev) / steps
    scan_f, attn_f = state.flops()
    bf16, bf16_src = measured_bf16_tflops()
    tokens = w.B * w.T * steps
    del state
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return {"tokens_per_s": tokens / (total_ms / 1e3), "ms_per_step": total_ms / steps,
            "scan": {"kernel": "csa2 indexer scan (tcgen05 kind::f8f6f4)", "bound": "tensor",
                     "achieved": scan_f / (scan_ms / 1e3) / 1e12, "peak": 2 * bf16,
                     "unit": "TFLOP/s", "frac": scan_f / (scan_ms / 1e3) / 1e12 / (2 * bf16),
                     "peak_source": bf16_src + " bf16 burst x 2 (FP8/bf16 nominal ratio)",
                     "flops_per_launch": scan_f, "avg_launch_ms": scan_ms},
            "attention": {"kernel": "csa2 prefill attention (tcgen05 kind::f16)",
                          "bound": "tensor", "achieved": attn_f / (attn_ms / 1e3) / 1e12,
                          "peak": bf16, "unit": "TFLOP/s",
                          "frac": attn_f / (attn_ms / 1e3) / 1e12 / bf16,
                          "peak_source": bf16_src + " bf16 burst",
                          "flops_per_call": attn_f, "avg_call_ms": attn_ms},
            "clocks": clk, "device_status": st, "steps": steps}


COMPRESS_CASES = (("compress_prefill_b2_n2048_r2", 2, 2048, 2, 67584),
                  ("compress_decode_b32_n1_r2", 32, 1, 2, 32768))


def measure_compress(name, B, n_new, r, cap, seed, steps, dev):
    """Device time of csa2_compress_kv (compressor + indexer-K projection + FP4 write) on
    synthetic source tokens, each launch in a graph between two event nodes, L2 flushed
    between launches (outside the events). Roofline:
    HBM bytes = the source latents and logits read + the FP4 entry (288 B) and E4M3 key
    (128 B) written per entry + the projection matrix (128 KiB) once."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    n_tok = r * n_new
    Cs = torch.randn((B, n_tok, 512), generator=g).to(torch.bfloat16).to(dev)
    Zs = (torch.randn((B, n_tok, 512), generator=g) * 2).to(torch.bfloat16).to(dev)
    W = (torch.randn((128, 512), generator=g) * 0.06).to(torch.bfloat16).to(dev)
    dst = torch.full((B,), cap - n_new, dtype=torch.int32, device=dev)
    codes = torch.zeros((B, cap, 256), dtype=torch.uint8, device=dev)
    scales = torch.zeros((B, cap, 32), dtype=torch.uint8, device=dev)
    keys = torch.zeros((B, cap, 128), dtype=torch.float8_e4m3fn, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(3):
        csa2.compress_kv(Cs, Zs, r, W, dst, codes, scales, keys, status=st)
    ev = [_event_pair() for _ in range(steps)]
    for pair in ev:                             # events exist once recorded
        pair[0].record(stream)
        pair[1].record(stream)
    # one graph per launch with its events inside (external event nodes): the host's
    # marshalling and tensor-map encoding stay out of the timed interval
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    torch.cuda.synchronize()
    graphs = []
    for e0, e1 in ev:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            csa2.record_event(e0, side)
            csa2.compress_kv(Cs, Zs, r, W, dst, codes, scales, keys, status=st, stream=side)
            csa2.record_event(e1, side)
        graphs.append(g)
    for g in graphs:                            # first launch (upload) outside the timing
        g.replay()
    torch.cuda.synchronize()
    for k in range(steps):
        flush_l2(flush, k)
        graphs[k].replay()
    torch.cuda.synchronize()
    del graphs
    ms = sum(a.elapsed_time(b) for a, b in ev) / steps
    entries = B * n_new
    nbytes = entries * (2 * r * 512 * 2 + 288 + 128) + 128 * 512 * 2
    peak, _src = peaks()
    out = {"kernel": "csa2 compressor + indexer-K projection (tcgen05) + FP4 write",
           "entries": entries, "ratio": r, "bound": "hbm", "bytes_per_launch": nbytes,
           "avg_launch_ms": ms, "achieved": nbytes / (ms / 1e3) / 1e9, "peak": peak,
           "unit": "GB/s", "frac": nbytes / (ms / 1e3) / 1e9 / peak,
           "device_status": int(st.item())}
    del Cs, Zs, codes, scales, keys, flush
    torch.cuda.empty_cache()
    return out


def prefill_main(args, w, dev, rank, world):
    m = measure_prefill(w, rank_seed(args.seed, rank), args.steps, args.warmup, dev)
    line = {
        "metric": "CSA2 chunked prefill tokens/s (FP8 indexer + sparse attention), 1 B200",
        "value": m["tokens_per_s"] * world, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup),
        "ms_per_step": m["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3 indexer / fp16 attention (fp32 accumulate)",
        "data": "synthetic",
        "config": {"workload": w.name, "batch": w.B, "new_tokens": w.T, "cached_tokens": w.ctx,
                   "ratio": w.ratio, "topk": w.K, "indexer_heads": w.H_I, "query_heads": w.H,
                   "window": synth.WINDOW, "l2": "inputs larger than L2"},
        "roofline": m["scan"],
        "attention": m["attention"],
        "gpu_launches": 5 * args.steps,   # quantize, prep, scan, Top-K, attention
        "clocks": m["clocks"],
        "device_status": m["device_status"],
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


CP_WORKLOAD = "decode_pool_reindex_b4_ctx1m"


def cp_main(args, dev, rank, world, local):
    """Context-parallel Full layer of the 1M-context workload (--cp): every rank holds one
    contiguous shard of every sequence's entries (indexer keys and FP4 main KV); the layer's
    selection (scan, candidate pool, Top-512) and its attention run through cp.select and
    cp.attend, whose exchanges are NCCL all-gathers of the shard selections and of the
    attention partials. Strong scaling: the same B queries whatever the rank count."""
    import socket
    import torch.distributed as dist
    from fp4_compressed_sparse_quantize_b200 import cp
    if not dist.is_initialized():          # one rank: a one-rank NCCL group
        sk = socket.socket()
        sk.bind(("127.0.0.1", 0))
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", str(sk.getsockname()[1]))
        sk.close()
        import datetime
        dist.init_process_group("nccl", rank=0, world_size=1, device_id=dev,
                                timeout=datetime.timedelta(seconds=120))
    w = synth.WORKLOADS[CP_WORKLOAD]
    B, cap, K = w.B, w.cap, w.K
    seed = args.seed                        # one batch: the same inputs on every rank
    lo, hi = cp.shards(cap, world)[rank]
    L = synth.layer_inputs(w, 0, seed, dev)
    dirs = synth.planted_direction([L["q_I"]]) if w.planted else None
    k_full, _ = synth.indexer_keys(w, seed, dev, planted_dirs=dirs)
    k_shard = k_full[:, lo:hi].contiguous()
    del k_full
    codes = torch.zeros((B, hi - lo, 256), dtype=torch.uint8, device=dev)
    scales = torch.zeros((B, hi - lo, 32), dtype=torch.uint8, device=dev)
    for b in range(B):
        src = _main_rows(w, seed, b, dev)[lo:hi].contiguous()
        csa2.quantize_kv(src[None], torch.zeros(1, dtype=torch.int32, device=dev),
                         codes[b:b + 1], scales[b:b + 1])
        del src
    n_vis = synth.decode_positions(w, dev)
    ws_i = csa2.new_workspace(csa2.workspace_bytes(0, B, 1, w.H_I, hi - lo, K, synth.POOL_BLOCKS))
    ws_a = csa2.new_workspace(csa2.workspace_bytes(1, B, 1, w.H, hi - lo, K))
    out = torch.empty((B, w.H, synth.D_MAIN), dtype=torch.float32, device=dev)
    tau = 1.0 / math.sqrt(synth.D_MAIN)
    swa = L["swa"] if rank == 0 else None
    torch.cuda.empty_cache()

    def step():
        idx, _pool = cp.select(L["q_I"], L["w"], k_shard, n_vis, lo, K, ws_i,
                               pool_blocks=synth.POOL_BLOCKS)
        cp.attend("full", L["q"], codes, scales, idx.view(B, K), lo, swa, out, ws_a, scale=tau)

    stream = torch.cuda.current_stream(dev)
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    dist.barrier()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    clocks = Clocks(local)
    clocks.start()
    for k in range(args.steps):
        ev[k][0].record(stream)
        step()
        ev[k][1].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    total = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), dist, dev)
    st = [csa2.read_device_status(ws_i), csa2.read_device_status(ws_a)]
    ms = total / args.steps
    # per step: prep, scan, Top-K, pool Top-K; candidates, merge (x2), pool candidates, pool
    # expansion; local indices, the attention's launches, the partials' merge
    launches = 4 + 5 + 1 + csa2.sparse_attn_decode_launches(B, K, synth.WINDOW) + 1
    exch = world * B * (K * 8 + synth.POOL_BLOCKS * 8 + w.H * (synth.D_MAIN + 2) * 4)
    line = {
        "metric": "CSA2 context-parallel Full layer (scan + pool + Top-512 + attention) "
                  "queries/s at 1M ctx",
        "value": B / (ms / 1e3), "unit": "queries/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": ms, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "e4m3/fp4/fp16 (fp32 accumulate)",
        "data": "synthetic",
        "config": {"workload": CP_WORKLOAD + " (Full layer)", "batch": B,
                   "compressed_entries": cap, "shard_entries": hi - lo,
                   "parallelism": f"cp{world} (entries sharded; NCCL all-gather of selections "
                                  "and attention partials)",
                   "launch": "eager (NCCL collectives between the library calls)",
                   "l2": "not flushed: each step streams the shard's indexer keys"},
        "exchange_bytes_per_step": exch,
        "gpu_launches": launches * args.steps,
        "clocks": clk, "device_status": st,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    dist.barrier()
    dist.destroy_process_group()


def local_rank():
    return int(os.environ.get("LOCAL_RANK", "0"))


def measured_bf16_tflops():
    """(dense bf16 TFLOP/s, source): the burst figure of MEASURED_PEAKS.json, else the
    pool's earlier burst measurement."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


def _main_rows(w, seed, b, dev):
    """bf16 [cap, 512] main-KV source rows of sequence b (drawn per sequence, exactly as
    synth.main_kv_source draws them)."""
    g = synth._gen(seed, 1, b, dev)
    x = torch.randn((w.cap, synth.D_MAIN), generator=g, device=dev, dtype=torch.float32)
    if w.lognormal_channels:
        s = torch.exp(torch.randn((synth.D_MAIN,), generator=synth._gen(seed, 2, b, dev),
                                  device=dev, dtype=torch.float32))
        x = x * s
    return x.to(torch.bfloat16)


# ---- CPU baseline / reference arm (the oracle as it stands) --------------------------------------

def decode_config(w, world, eager):
    return {"workload": w.name, "batch_per_gpu": w.B, "context_tokens": w.ctx,
            "launch": "eager" if eager else "cuda graph replay per step",
            "ratio": w.ratio, "compressed_entries": w.N, "topk": w.K,
            "indexer_heads": w.H_I, "indexer_dtype": w.idx_dtype, "query_heads": w.H,
            "window": synth.WINDOW, "layers": list(w.layers),
            "parallelism": f"dp{world} (independent batches)",
            "l2": "flushed between steps (256 MiB write + read, outside the timed events)"}


class RefInputs:
    """The seeded inputs of a decode workload without any library work (reference arm)."""

    def __init__(self, w, seed, dev):
        self.w, self.seed, self.dev = w, seed, dev
        self.tau = 1.0 / math.sqrt(synth.D_MAIN)
        self.layers = [synth.layer_inputs(w, li, seed, dev) for li in range(len(w.layers))]
        dirs = None
        if w.planted:
            dirs = synth.planted_direction([L["q_I"] for L, m in zip(self.layers, w.layers)
                                            if m in ("full", "reindex")])
        self.k_I, _ = synth.indexer_keys(w, seed, dev, planted_dirs=dirs)


def oracle_queries(state, budget_s):
    """Run the oracle over whole decode queries of this workload until ~budget_s of CPU work;
    returns (queries done, seconds, cores)."""
    sys.path.insert(0, ROOT)
    from oracle import oracle as O
    w = state.w
    ek = O.BF16 if w.idx_dtype == "bf16" else O.E4M3
    done, t_total = 0, 0.0
    b = 0
    while t_total < budget_s and b < w.B:
        # inputs of sequence b (copied out of device memory before the clock starts)
        fp4 = w.key_format == "fp4"
        if fp4:
            k_codes = state.k_I.codes[b, :w.N].cpu().numpy()
            k_scales = state.k_I.scales[b, :w.N].cpu().numpy()
        else:
            k_raw = state.k_I[b, :w.N].contiguous().cpu().view(torch.uint8 if ek == O.E4M3 else torch.int16).numpy()
            if ek == O.BF16:
                k_raw = k_raw.view(np.uint16)
        src = _main_rows(w, state.seed, b, state.dev)[: w.N].cpu().view(torch.int16).numpy().view(np.uint16)
        lay = []
        for L in state.layers:
            qi = L["q_I"][b, 0].contiguous().cpu().view(torch.uint8 if ek == O.E4M3 else torch.int16).numpy()
            if ek == O.BF16:
                qi = qi.view(np.uint16)
            lay.append((qi, L["w"][b, 0].cpu().numpy(), L["q"][b].cpu().view(torch.int16).numpy().view(np.uint16),
                        L["swa"][b].cpu().view(torch.uint8).numpy()))
        t0 = time.perf_counter()
        O.quantize_entries(src[w.N - 1:w.N])              # quantize-on-write of the new entry
        cur = None
        pool = None
        for (qi, wt, qb, swa), mode in zip(lay, w.layers):
            if mode == "full":
                s = (O.index_scores_fp4key(qi, wt, k_codes, k_scales) if fp4
                     else O.index_scores(qi, wt, k_raw, ek))
                cur = O.topk(s, w.K)
                if w.pool:
                    pool = O.pool(s, synth.POOL_BLOCKS)
            elif mode == "reindex":
                ids = pool[pool >= 0]
                s = O.index_scores(qi, wt, k_raw, ek, rows=ids)
                cur = O.topk(s, w.K, ids)
            sel = [int(i) for i in cur if i >= 0]
            c, sc = O.quantize_entries(src[sel])
            rows = np.concatenate([O.dequant_entries(c, sc),
                                   O.e4m3_array_to_f64(swa).reshape(-1, 512)])
            O.attention(O.bf16_array_to_f64(qb).reshape(-1, 512), rows, state.tau)
        t_total += time.perf_counter() - t0
        done += 1
        b += 1
    return done, t_total, O.num_threads()


# ---- launcher ---------------------------------------------------------------------------------

def _free_port():
    import socket
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        return so.getsockname()[1]


def spawn_ranks(n, argv, timeout_s=3600):
    """Re-run this script with the same arguments as n ranks of one node
    (torch.distributed.run on 127.0.0.1); returns the launcher's exit status."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr=127.0.0.1",
           f"--master-port={_free_port()}", os.path.abspath(__file__)] + list(argv)
    try:
        return subprocess.run(cmd, timeout=timeout_s).returncode
    except subprocess.TimeoutExpired:
        return 124


# ---- main -------------------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="csa2", choices=["csa2", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--seed", type=int, default=1234)
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the shorter runs of the other workloads (256K, 1M, prefill)")
    ap.add_argument("--extra-steps", type=int, default=10)
    ap.add_argument("--cp", action="store_true",
                    help="context-parallel Full layer of the 1M-context workload over the ranks")
    ap.add_argument("--eager", action="store_true",
                    help="launch every call from Python instead of replaying CUDA graphs")
    ap.add_argument("--compress-only", action="store_true",
                    help="time only the KV compressor cases (one GPU; one JSON line each)")
    args = ap.parse_args()

    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        # not under a launcher: start one rank per GPU on this node and wait for them
        sys.exit(spawn_ranks(args.gpus, sys.argv[1:]))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        sys.exit(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}")
    if args.impl == "reference":
        return reference_arm(args, rank, world, local)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if args.compress_only:
        if world != 1:
            sys.exit("bench.py: --compress-only runs on one GPU")
        for name, B, n_new, r, cap in COMPRESS_CASES:
            m = measure_compress(name, B, n_new, r, cap, args.seed, args.steps, dev)
            print(json.dumps({"workload": name, **m}), flush=True)
        return
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist
    if args.cp:
        return cp_main(args, dev, rank, world, local)
    w = synth.WORKLOADS[args.workload]
    if w.kind == "prefill":
        prefill_main(args, w, dev, rank, world)
        if pg:
            pg.barrier()
            pg.destroy_process_group()
        return
    state = Decode(w, rank_seed(args.seed, rank), dev)
    stream = torch.cuda.current_stream(dev)
    tm = timed_decode(state, args.steps, args.warmup, stream, local, args.eager, pg)
    step_ms, scan_ms, attn_ms, clk = tm["step_ms"], tm["scan_ms"], tm["attn_ms"], tm["clocks"]
    total_ms = max_over_ranks(sum(step_ms), pg, dev)

    # end-to-end: host inputs -> device -> step -> host output, through the public API.
    # Steps are pipelined as a serving loop would run them: E2E_SETS sets of device inputs
    # and outputs, so that the host->device copies of the next steps and the device->host
    # copies of the previous ones (copy streams) overlap step k (compute stream). Every step copies all of its
    # inputs in and its outputs back. L2 is not flushed inside this continuous region: each
    # step streams the 134 MB indexer-key cache (evict-first), more than the 126 MB L2.
    # Every step's inputs travel in one host->device copy and its outputs in one
    # device->host copy: the tensors of a step are packed at 256-byte aligned offsets of one
    # pinned host buffer and one device buffer (the library calls get views of it). Several
    # copies of a few KB to 2 MB each ran at 13 GB/s on this PCIe link, one 4.5 MB copy at 50.
    ins0 = state.step_inputs()
    outs0 = state.step_outputs()
    h_inbuf, h_in = packed_like(ins0, "cpu")
    for h, x in zip(h_in, ins0):
        h.copy_(x)
    h_outbuf, _ = packed_like(outs0, "cpu")
    bi, bo = h_inbuf.numel(), h_outbuf.numel()
    io = []
    for _ in range(E2E_SETS):
        d_inbuf, d_in = packed_like(ins0, dev)
        d_outbuf, d_out = packed_like(outs0, dev)
        for d, x in zip(d_in, ins0):
            d.copy_(x)
        io.append((d_inbuf, d_in, d_outbuf, d_out))
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    g_io = []
    if not args.eager:
        side = torch.cuda.Stream()
        for _bi, ins, _bo, outs in io:
            state.set_io(ins, outs)
            side.wait_stream(stream)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=side):
                state.step(stream=side)
            g_io.append(g)
        torch.cuda.synchronize()
    ev = lambda: torch.cuda.Event(enable_timing=False)
    loaded, consumed, drained = [[ev() for _ in range(E2E_SETS)] for _ in range(3)]

    def pipelined(n):
        for k in range(n):
            s_ = k % E2E_SETS
            inbuf, ins, outbuf, outs = io[s_]
            with torch.cuda.stream(h2d):
                if k >= E2E_SETS:
                    h2d.wait_event(consumed[s_])      # the last step on set s_ no longer reads it
                inbuf.copy_(h_inbuf, non_blocking=True)
                loaded[s_].record(h2d)
            stream.wait_event(loaded[s_])
            if k >= E2E_SETS:
                stream.wait_event(drained[s_])        # that step's outputs are on the host
            if g_io:
                with torch.cuda.stream(stream):
                    g_io[s_].replay()
            else:
                state.set_io(ins, outs)
                state.step(stream=stream)
            consumed[s_].record(stream)
            with torch.cuda.stream(d2h):
                d2h.wait_event(consumed[s_])
                h_outbuf.copy_(outbuf, non_blocking=True)
                drained[s_].record(d2h)

    pipelined(E2E_SETS)                               # warm the copy streams
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(h2d)
    pipelined(args.steps)
    d2h.wait_stream(h2d)
    d2h.wait_stream(stream)
    e1.record(d2h)
    torch.cuda.synchronize()
    state.set_io(ins0, outs0)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), pg, dev)
    st_i = csa2.read_device_status(state.ws_idx)
    st_a = csa2.read_device_status(state.ws_attn)

    # other workloads of the metric's 64K-1M range (and the prefill chunk): one GPU only
    extra = {}
    if world == 1 and not args.no_extra:
        state_keep = state
        for name in EXTRA_DECODE:
            if name != args.workload:
                extra[name] = extra_decode(name, args, dev, local)
        pw = synth.WORKLOADS[EXTRA_PREFILL]
        extra[EXTRA_PREFILL] = measure_prefill(pw, args.seed, args.extra_steps, 3, dev)
        for name, B, n_new, r, cap in COMPRESS_CASES:
            extra[name] = measure_compress(name, B, n_new, r, cap, args.seed, args.extra_steps,
                                           dev)
        state = state_keep

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n, secs, cores = oracle_queries(state, args.cpu_budget)
        cpu = {"value": n / secs, "unit": "queries/s", "cores": cores, "kind": "oracle",
               "sample": f"{n} whole decode queries (sequences 0..{n - 1}) of the same workload, "
                         f"{secs:.1f} s of oracle time"}

    if rank == 0:
        alg_bytes, scan_bytes = state.algorithmic_bytes()
        per_step_ms = total_ms / args.steps
        queries = w.B * world * args.steps
        value = job_throughput(w.B, world, args.steps, total_ms)
        peak, src = peaks()
        scan_avg = sum(scan_ms) / len(scan_ms)
        achieved = scan_bytes / (scan_avg / 1e3) / 1e9
        sha = hashlib.sha1(open(SCAN_KERNEL_SRC, "rb").read()).hexdigest()
        tr = SCAN_TRAFFIC.get(args.workload)
        traffic = tr[1] if tr and tr[0] == sha else None
        line = {
            "metric": "CSA2 decode queries/s & HBM GB/s at 64K-1M ctx (frac of roofline), 1 B200",
            "value": value, "unit": "queries/s", "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": per_step_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "e4m3/fp4/fp16 (fp32 accumulate)", "data": "synthetic",
            "config": decode_config(w, world, args.eager),
            "hbm_gbs_step": alg_bytes / (per_step_ms / 1e3) / 1e9,
            "roofline": {"kernel": "csa2 indexer scan (tcgen05, FP8 keys)", "bound": "hbm",
                         "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_source": src,
                         "frac_of_8TBs": achieved / 8000.0,
                         "bytes_per_launch": scan_bytes, "avg_launch_ms": scan_avg,
                         "traffic": traffic},
            "step_roofline_frac": (alg_bytes / (per_step_ms / 1e3) / 1e9) / peak,
            "attention_roofline": decode_summary(state, tm, peak)["attention"],
            "e2e": {"value": queries / (e2e_ms / 1e3), "unit": "queries/s",
                    "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo,
                    "schedule": "pipelined: step k+1's inputs in and step k-1's outputs out "
                                "on copy streams while step k runs (three device buffer sets); "
                                "one packed copy each way per step"},
            "gpu_launches": state.launches_per_step() * args.steps,
            "clocks": clk,
            "device_status": [st_i, st_a],
            "cpu_baseline": cpu,
            "workloads": extra,
        }
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


def reference_arm(args, rank, world, local):
    """The oracle, as it stands, timed on the host cores: rank 0 only."""
    if rank != 0:
        return
    # a launcher's one-thread-per-rank default must not starve the only working rank: the
    # oracle's parallel loops take every host core
    if world > 1:
        from oracle import oracle as O
        O.set_num_threads(os.cpu_count() or 1)
    w = synth.WORKLOADS[args.workload]
    dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    if dev.type == "cuda":
        torch.cuda.set_device(local)
    state = RefInputs(w, args.seed, dev)
    # each step is a bounded sample: whole queries until ~budget/steps seconds
    per = max(1.0, args.cpu_budget / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_queries(state, per)
    n_tot, s_tot, cores = 0, 0.0, 1
    for _ in range(args.steps):
        n, s, cores = oracle_queries(state, per)
        n_tot += n
        s_tot += s
    value = n_tot / s_tot
    line = {"impl": "reference",
            "metric": "CSA2 decode queries/s & HBM GB/s at 64K-1M ctx (frac of roofline), 1 B200",
            "value": value, "unit": "queries/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * s_tot / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": decode_config(w, world, args.eager),
            "cpu_baseline": {"value": value, "unit": "queries/s", "cores": cores,
                             "kind": "oracle",
                             "sample": f"{n_tot} whole decode queries over {args.steps} steps"},
            "e2e": {"value": value, "unit": "queries/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
