#!/usr/bin/env python
"""Benchmark of the quantized-KV decode hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--precision K8V4]
    python bench.py --impl reference ...      # the CPU oracle on host cores

One step = one decode step of the workload: every sequence gains one token;
for each layer the new token's K / V are quantised into the paged cache and
the query attends to the whole cache.  For quantized caches that is one
kvq_decode_append_attn launch per layer (append, split-KV attention and the
log-sum-exp combine in one kernel); fp16 caches (and --separate) call
kvq_append then kvq_decode_attn.  Metric: algorithmic KV bytes moved per
second (cache codes + scales read by decode, fp16 q / out, the appended
token's fp16 read and quantised write), and decode tokens/s = batch / step.
By default one step is captured in a CUDA graph after the warm-up and every
timed step replays it (the same token re-appended at the same position, the
same length attended); --eager makes the API calls directly each step.

The default run (no --workload) also measures, as compact "extra" records with
their own clocks, the 70B-shaped single-sequence decode (K8V4 and FP16) and
the ragged chunked prefill (prefill TFLOP/s and append GB/s).

Multi-GPU (torchrun): every rank holds an independent replica of the workload
(sequences are independent, so the batch shards with no collective); value =
bytes of all ranks / the slowest rank's time ("weak" scaling).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "K8V4 decode-attention KV GB/s (fraction of HBM peak) and decode tokens/s"
DEFAULT_WORKLOAD = "llama3-8b-b32-32k"
L2_BYTES = 126 * 1024 * 1024
PROFILE_DIR = os.path.join(ROOT, "profiles")


# --------------------------------------------------------------------------- helpers
def tok_bytes(bits: int, D: int) -> int:
    """Stored bytes of one token's K or V row of one head (codes + scales)."""
    return 2 * D if bits == 16 else (D // 32) * (34 if bits == 8 else 18)


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "source": "fallback"}


KERNEL_SOURCES = {
    "decode_split": ("decode_kernel.cuh", "decode_launch.cuh", "decode.cu", "decode_common.cuh", "sm100_util.cuh"),
    "decode_q": ("decode_q.cuh", "decode_launch.cuh", "decode.cu", "decode_common.cuh", "sm100_util.cuh",
                 "quant_block.cuh"),
    "decode_tc": ("decode_tc.cu", "decode.cu", "decode_common.cuh", "sm100_util.cuh", "tcgen05_util.cuh"),
    "append": ("append.cu", "quant_block.cuh", "kvq_internal.cuh"),
}


def kernel_source_sha(kernel: str = "decode_split") -> str:
    """Hash of one decode kernel's sources: ncu traffic figures are valid only for this hash."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "asymmetric_quantized_kv_kvq_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str, precision: str, kernel: str = "decode_split"):
    """DRAM bytes per launch of the decode kernel from the committed ncu summary
    of this workload, if it was captured on the current kernel source."""
    path = os.path.join(PROFILE_DIR, f"{kernel}_{precision.lower()}_{workload}.txt")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip()
    if vals.get("kernel_source_sha") != kernel_source_sha(kernel):
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clocks, power and throttle reasons sampled every 100 ms (the four named reasons and
    the whole active-reason mask, whose other bits are decoded by name)."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap,clocks_event_reasons.active")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    MASK_NAMES = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
                  0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
                  0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.samples = []
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == 8:
                self.samples.append(parts)

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        sm = [float(s[0]) for s in self.samples if s[0].replace(".", "").isdigit()]
        mx = [float(s[1]) for s in self.samples if s[1].replace(".", "").isdigit()]
        reasons = {self.NAMES[i] for s in self.samples for i in range(4) if s[3 + i] == "Active"}
        mask = 0
        for smp in self.samples:
            try:
                mask |= int(smp[7], 16)
            except ValueError:
                pass
        reasons |= {name for bit, name in self.MASK_NAMES.items() if mask & bit and bit != 0x1}
        pw = []
        for smp in self.samples:
            try:
                pw.append(float(smp[2]))
            except ValueError:
                pass
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(self.samples),
                "power_w": round(statistics.median(pw), 1) if pw else None, "reasons_mask": hex(mask)}


# --------------------------------------------------------------------------- decode workload
class DecodeRun:
    """A resident cache of the workload plus one decode step's inputs."""

    def __init__(self, wl, kb: int, vb: int, capacity_extra: int, device, decode_tc: bool = False,
                 separate: bool = False, layer_batched: bool = False):
        import torch
        from asymmetric_quantized_kv_kvq_b200 import kvq
        from asymmetric_quantized_kv_kvq_b200.inputs import gen_kv, gen_q, GEN_CHUNK
        self.wl, self.kb, self.vb, self.dev = wl, kb, vb, device
        L, B, H, D, T = wl.n_layers, wl.batch, wl.n_kv_heads, wl.head_dim, wl.cached
        P = 256
        cap = T + capacity_extra
        self.cache = kvq.Cache(L, H, D, kb, vb, max_seqs=B, max_tokens=B * (-(-cap // P)) * P, max_seq_tokens=cap,
                               decode_tc=decode_tc)
        self.ids = list(range(B))
        # fill: chunk by chunk, every layer (the order a model's prefill writes the cache)
        for c in range(-(-T // GEN_CHUNK)):
            n = min(GEN_CHUNK, T - c * GEN_CHUNK)
            self.cache.extend(self.ids, [n] * B)
            for layer in range(L):
                ks, vs = [], []
                for b in self.ids:
                    k, v = gen_kv(wl, layer, b, c * GEN_CHUNK, n, device=device)
                    ks.append(k)
                    vs.append(v)
                self.cache.append(layer, self.ids, [n] * B, torch.cat(ks), torch.cat(vs))
                del ks, vs
        torch.cuda.synchronize()
        # one decode step's inputs (same values every step), stacked over the layers: q / out
        # [L, B, Hq, D], new K / V [L, B, H, D]; the per-layer lists are views of them
        ks, vs, qs = [], [], []
        for layer in range(L):
            k1, v1 = zip(*[gen_kv(wl, layer, b, T, 1, device=device) for b in self.ids])
            ks.append(torch.cat(k1))
            vs.append(torch.cat(v1))
            qs.append(gen_q(wl, layer, 0, device=device))
        self.k_all, self.v_all, self.q_all = torch.stack(ks), torch.stack(vs), torch.stack(qs)
        self.out_all = torch.empty_like(self.q_all)
        del ks, vs, qs
        self.k_new, self.v_new = list(self.k_all.unbind(0)), list(self.v_all.unbind(0))
        self.q, self.out = list(self.q_all.unbind(0)), list(self.out_all.unbind(0))
        # layer-batched: one kvq_decode_attn_layers call per step, one launch per run of up to
        # KVQ_MAX_BATCH // B layers
        self.batched = layer_batched
        self.runs = -(-L // max(1, 256 // B)) if layer_batched else L
        ws = self.cache.decode_layers_workspace_size(L, B, wl.n_q_heads) if layer_batched else \
            self.cache.decode_workspace_size(B, wl.n_q_heads)
        self.ws = torch.empty(ws, dtype=torch.uint8, device=device)
        self.ones = [1] * B
        self.ev = None
        # one launch per layer (append fused into the decode kernel) for quantized caches on CUDA cores
        self.fused = kb != 16 and not decode_tc and not separate

    def lengths(self):
        return [self.cache.length(b) for b in self.ids]

    def step_bytes(self, lens) -> tuple:
        """(decode bytes, append bytes) of one step whose sequences end at `lens`."""
        wl = self.wl
        H, D, L, Hq = wl.n_kv_heads, wl.head_dim, wl.n_layers, wl.n_q_heads
        per_tok = H * (tok_bytes(self.kb, D) + tok_bytes(self.vb, D))
        dec = sum(lens) * per_tok + 2 * len(lens) * Hq * D * 2
        app = len(lens) * (H * D * 2 * 2 + per_tok)
        return L * dec, L * app

    def launches_per_step(self, lens_before) -> int:
        pt = 1 if any(n % 256 == 0 for n in lens_before) else 0
        if self.fused:
            return pt + self.runs                        # one decode kernel (append + split + combine)
        combine = 0 if (self.kb != 16 and not self.cache_tc) else 1
        return pt + self.runs * (2 + combine)           # append, decode[, combine]

    @property
    def cache_tc(self) -> bool:
        return self.cache.cfg.flags & 2 != 0 and self.kb == 8 and self.wl.head_dim == 128

    def step(self, record=None):
        self.cache.extend(self.ids, self.ones)
        if self.batched:
            if record is not None:
                record[0][0].record()
            self.cache.decode_layers(0, self.ids, self.q_all, self.k_all, self.v_all, out=self.out_all,
                                     workspace=self.ws)
            if record is not None:
                record[0][1].record()
            return
        for layer in range(self.wl.n_layers):
            if self.fused:
                if record is not None:
                    record[layer][0].record()
                self.cache.decode_append(layer, self.ids, self.q[layer], self.k_new[layer], self.v_new[layer],
                                         out=self.out[layer], workspace=self.ws)
            else:
                self.cache.append(layer, self.ids, self.ones, self.k_new[layer], self.v_new[layer])
                if record is not None:
                    record[layer][0].record()
                self.cache.decode(layer, self.ids, self.q[layer], out=self.out[layer], workspace=self.ws)
            if record is not None:
                record[layer][1].record()


def run_decode_bench(args, wl, kb, vb, rank, world) -> dict:
    import torch
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    extra = args.warmup + 2 * args.steps + 8
    t0 = time.time()
    run = DecodeRun(wl, kb, vb, extra, dev, decode_tc=args.decode_tc, separate=args.separate,
                    layer_batched=getattr(args, "layer_batched", False))
    setup_s = time.time() - t0
    L = wl.n_layers
    lens0 = run.lengths()
    total_kv = sum(lens0) * wl.n_kv_heads * (tok_bytes(kb, wl.head_dim) + tok_bytes(vb, wl.head_dim)) * L
    flush = total_kv < 2 * L2_BYTES
    scratch = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if flush else None

    for _ in range(args.warmup):
        run.step()
    run.cache.check()
    graph, graph_lens, launch_mode = None, None, "eager (--eager)"
    if not args.eager:
        graph, graph_lens, launch_mode = capture_step(run, run.step)
    barrier(world)
    torch.cuda.synchronize()

    # ---- timed region: K steps, CUDA events on the launching stream.  With a captured graph every
    #      step is one replay of the same decode step (append of one token per sequence + decode, all
    #      layers): the token is re-appended at the same position and attended over the same length.
    # event pairs of an eager step: one per layer's call, or one around the layer-batched call
    n_ev = 1 if run.batched else L
    ev = [[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)] for _ in range(n_ev)]
    dec_ms, step_ms, dec_bytes, app_bytes, launches = [], [], 0, 0, 0
    gpu_id = gpu_uuid(dev)
    with ClockSampler(gpu_id) as clk:
        for _ in range(args.steps):
            if flush:
                scratch.zero_()
            lens_before = graph_lens if graph is not None else run.lengths()
            s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0.record()
            if graph is not None:
                graph.replay()
            else:
                run.step(record=ev)
            s1.record()
            torch.cuda.synchronize()
            step_ms.append(s0.elapsed_time(s1))
            if graph is None:
                dec_ms.extend(e0.elapsed_time(e1) for e0, e1 in ev)
            d, a = run.step_bytes([n + 1 for n in lens_before])
            dec_bytes += d
            app_bytes += a
            launches += run.launches_per_step(lens_before)
    in_step_bytes = (dec_bytes + (app_bytes if run.fused else 0)) / args.steps
    if graph is not None:
        # per-layer decode durations inside a step: one eager step with events (outside the timed region)
        lens_e = run.lengths()
        if flush:
            scratch.zero_()
        run.step(record=ev)
        torch.cuda.synchronize()
        dec_ms.extend(e0.elapsed_time(e1) for e0, e1 in ev)
        d_e, a_e = run.step_bytes([n + 1 for n in lens_e])
        in_step_bytes = d_e + (a_e if run.fused else 0)
    # ---- kernel duration: every layer's decode call once more (or the layer-batched call 8 times),
    #      back to back on the stream behind a short device-side sleep, so that host work between
    #      calls (binding, plan) never leaves the GPU idle inside the events
    lens_k = run.lengths()
    kd, ka = run.step_bytes(lens_k)
    kern_bytes = (kd + (ka if run.fused else 0)) / n_ev
    reps = 8 if run.batched else max(L, 8)
    kern_ms = []
    for _ in range(2):
        torch.cuda.synchronize()
        if hasattr(torch.cuda, "_sleep"):
            torch.cuda._sleep(4_000_000)
        k0, k1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        k0.record()
        for i in range(reps):
            lay = i % L
            if run.batched:      # fused: re-appends the last token at the same position
                run.cache.decode_layers(0, run.ids, run.q_all, run.k_all if run.fused else None,
                                        run.v_all if run.fused else None, out=run.out_all, workspace=run.ws)
            elif run.fused:        # re-appends the last token at the same position, as a replayed step does
                run.cache.decode_append(lay, run.ids, run.q[lay], run.k_new[lay], run.v_new[lay], out=run.out[lay],
                                        workspace=run.ws)
            else:
                run.cache.decode(lay, run.ids, run.q[lay], out=run.out[lay], workspace=run.ws)
        k1.record()
        torch.cuda.synchronize()
        kern_ms.append(k0.elapsed_time(k1) / reps)
    barrier(world)
    torch.cuda.synchronize()
    run.cache.check()

    local_ms = sum(step_ms)
    max_ms = all_reduce_max(local_ms, world, dev)
    tot_bytes = all_reduce_sum(float(dec_bytes + app_bytes), world, dev)
    tot_tokens = all_reduce_sum(float(wl.batch * args.steps), world, dev)
    res = {
        "ms_per_step": max_ms / args.steps,
        "value": tot_bytes / (max_ms * 1e-3) / 1e9,
        "decode_tokens_per_s": tot_tokens / (max_ms * 1e-3),
        "dec_bytes_per_launch": in_step_bytes / n_ev,
        "launch_mode": launch_mode,
        "dec_ms_per_launch": statistics.mean(dec_ms),
        "kern_bytes_per_launch": kern_bytes,
        "kern_ms_per_launch": min(kern_ms),
        "launches": launches,
        "clocks": clk.summary(),
        "flush": flush,
        "setup_s": setup_s,
        "fused": run.fused,
        "step_only_decode": run.fused and graph is not None,
        "batched": run.batched,
        "runs": run.runs,
        "step_bytes": (dec_bytes + app_bytes) / args.steps,
    }

    # ---- content dedup pass (kvq_cache_dedup) over the resident cache: every full page is hashed on
    #      the GPU (the contents differ, so nothing is merged); CUDA events around the call
    if getattr(args, "dedup_probe", False):
        P = 256
        full = sum(n // P for n in run.lengths())
        page_bytes = wl.n_kv_heads * P * (tok_bytes(kb, wl.head_dim) + tok_bytes(vb, wl.head_dim)) * L
        torch.cuda.synchronize()
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        d0.record()
        freed = run.cache.dedup()
        d1.record()
        torch.cuda.synchronize()
        ms = d0.elapsed_time(d1)
        res["dedup"] = {"metric": "content-hash dedup pass GB/s (kvq_cache_dedup over the resident cache)",
                        "value": full * page_bytes / (ms * 1e-3) / 1e9, "unit": "GB/s", "ms": ms,
                        "pages_hashed": full, "bytes_hashed": full * page_bytes, "pages_freed": freed,
                        "timing": "CUDA events around one kvq_cache_dedup call (hash kernels, read-back of the "
                                  "hashes per 1024 pages, host grouping)"}
        run.cache.check()

    # ---- end to end through the public API with host buffers: replaying the captured step (the
    #      default launch mode) and, beside it, calling the API eagerly every step
    if not args.no_e2e:
        res["e2e"] = run_e2e(run, args, world, dev, eager=args.eager)
        if not args.eager:
            res["e2e_eager"] = run_e2e(run, args, world, dev, eager=True)
    del graph
    run.cache.close()
    return res


def capture_step(run, body):
    """Capture `body` (one decode step through the public API) into a CUDA graph.
    Returns (graph, lengths before the captured step, launch-mode note); on a
    capture error, (None, None, the reason) and the caller steps eagerly."""
    import torch
    lens = run.lengths()
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            body()
        torch.cuda.synchronize()
        for _ in range(2):          # upload + warm replays, untimed
            g.replay()
        torch.cuda.synchronize()
        return g, lens, "CUDA graph of one decode step (all layers), replayed"
    except Exception as e:  # noqa: BLE001 -- reported in the JSON line
        torch.cuda.synchronize()
        return None, None, f"eager (graph capture failed: {type(e).__name__}: {str(e)[:120]})"


def run_e2e(run, args, world, dev, eager: bool) -> dict:
    """Same step, but every step copies its inputs (q, new K / V for all layers)
    from pinned host memory and reads all outputs back to pinned host memory
    (one copy per tensor, all layers at once);
    the step is a replayed graph of the copies + calls, or (eager) the host
    calls themselves, binding and validation included."""
    import torch
    # every layer's inputs and outputs sit in one pinned host buffer each ([L, B, ...], the layout of
    # the device tensors), so a step moves them with three host-to-device copies and one back
    hq = run.q_all.cpu().pin_memory()
    hk = run.k_all.cpu().pin_memory()
    hv = run.v_all.cpu().pin_memory()
    ho = torch.empty(run.out_all.shape, dtype=run.out_all.dtype, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
    d2h = ho.numel() * ho.element_size()

    def body():
        run.q_all.copy_(hq, non_blocking=True)
        run.k_all.copy_(hk, non_blocking=True)
        run.v_all.copy_(hv, non_blocking=True)
        run.step()
        ho.copy_(run.out_all, non_blocking=True)

    for _ in range(2):
        body()
    graph, graph_lens = None, None
    if not eager:
        graph, graph_lens, _ = capture_step(run, body)
    barrier(world)
    torch.cuda.synchronize()
    nbytes, ms = 0, 0.0
    for _ in range(args.steps):
        lens_before = graph_lens if graph is not None else run.lengths()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record()
        if graph is not None:
            graph.replay()
        else:
            body()
        s1.record()
        torch.cuda.synchronize()
        ms += s0.elapsed_time(s1)
        d, a = run.step_bytes([n + 1 for n in lens_before])
        nbytes += d + a
    barrier(world)
    max_ms = all_reduce_max(ms, world, dev)
    tot = all_reduce_sum(float(nbytes), world, dev)
    del graph
    return {"value": tot / (max_ms * 1e-3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "launch": "eager API calls" if eager else "replayed CUDA graph"}


PREFILL_METRIC = "K8V4 chunked-prefill TFLOP/s (causal FLOPs) and quantise-on-append GB/s"


class PrefillRun:
    """Ragged sequences with cached prefixes; one step appends a chunk to every
    sequence (quantise-on-append) and runs causal prefill of the chunk over
    cache + chunk, then rewinds the sequences to their prefixes."""

    def __init__(self, wl, kb: int, vb: int, device):
        import torch
        from asymmetric_quantized_kv_kvq_b200 import kvq
        from asymmetric_quantized_kv_kvq_b200.inputs import gen_kv, gen_q_chunk, cached_lengths, GEN_CHUNK
        self.wl, self.kb, self.vb, self.dev = wl, kb, vb, device
        H, D, C = wl.n_kv_heads, wl.head_dim, wl.chunk
        self.T = cached_lengths(wl)
        n = len(self.T)
        self.ids = list(range(n))
        P = 256
        cap = sum(-(-(t + C) // P) * P for t in self.T)
        self.cache = kvq.Cache(wl.n_layers, H, D, kb, vb, max_seqs=n, max_tokens=cap, max_seq_tokens=max(self.T) + C)
        for b, t in enumerate(self.T):
            for c in range(-(-t // GEN_CHUNK)):
                m = min(GEN_CHUNK, t - c * GEN_CHUNK)
                self.cache.extend([b], [m])
                for layer in range(wl.n_layers):
                    k, v = gen_kv(wl, layer, b, c * GEN_CHUNK, m, device=device)
                    self.cache.append(layer, [b], [m], k, v)
        kv = [gen_kv(wl, 0, b, t, C, device=device) for b, t in enumerate(self.T)]
        self.k_new = torch.cat([k for k, _ in kv]).contiguous()
        self.v_new = torch.cat([v for _, v in kv]).contiguous()
        self.q = torch.cat([gen_q_chunk(wl, 0, b, C, device=device) for b in self.ids]).contiguous()
        self.out = torch.empty_like(self.q)
        self.chunks = [C] * n
        self.cache.extend(self.ids, self.chunks)
        self.ws = torch.empty(self.cache.prefill_workspace_size(self.ids, self.chunks, wl.n_q_heads),
                              dtype=torch.uint8, device=device)
        for b, t in enumerate(self.T):
            self.cache.truncate(b, t)
        torch.cuda.synchronize()

    def flops(self) -> float:
        wl, C = self.wl, self.wl.chunk
        return 4.0 * wl.n_q_heads * wl.head_dim * sum(C * t + C * (C + 1) / 2 for t in self.T)

    def append_bytes(self) -> int:
        wl = self.wl
        D = wl.head_dim
        per_tok = wl.n_kv_heads * (2 * D * 2 + tok_bytes(self.kb, D) + tok_bytes(self.vb, D))
        return len(self.T) * wl.chunk * per_tok

    def step(self, ev=None):
        self.cache.extend(self.ids, self.chunks)
        if ev is not None:
            ev[0].record()
        self.cache.append(0, self.ids, self.chunks, self.k_new, self.v_new)
        if ev is not None:
            ev[1].record()
        self.cache.prefill(0, self.ids, self.chunks, self.q, out=self.out, workspace=self.ws)
        if ev is not None:
            ev[2].record()
        for b, t in enumerate(self.T):
            self.cache.truncate(b, t)


def run_prefill_bench(args, wl, kb, vb, rank, world) -> dict:
    import torch
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    t0 = time.time()
    run = PrefillRun(wl, kb, vb, dev)
    setup_s = time.time() - t0
    for _ in range(args.warmup):
        run.step()
    run.cache.check()
    barrier(world)
    torch.cuda.synchronize()
    app_ms, pre_ms, step_ms = [], [], []
    with ClockSampler(gpu_uuid(dev)) as clk:
        for _ in range(args.steps):
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            run.step(ev)
            torch.cuda.synchronize()
            app_ms.append(ev[0].elapsed_time(ev[1]))
            pre_ms.append(ev[1].elapsed_time(ev[2]))
            step_ms.append(ev[0].elapsed_time(ev[2]))
    # ---- append kernel duration: the chunk's append repeated back to back (same positions) behind a
    #      short device sleep, so that the binding's host work stays out of the events
    run.cache.extend(run.ids, run.chunks)
    torch.cuda.synchronize()
    if hasattr(torch.cuda, "_sleep"):
        torch.cuda._sleep(4_000_000)
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 8
    a0.record()
    for _ in range(reps):
        run.cache.append(0, run.ids, run.chunks, run.k_new, run.v_new)
    a1.record()
    torch.cuda.synchronize()
    app_kernel_ms = a0.elapsed_time(a1) / reps
    for bi, t in enumerate(run.T):
        run.cache.truncate(bi, t)
    barrier(world)
    torch.cuda.synchronize()
    run.cache.check()
    local = sum(step_ms)
    max_ms = all_reduce_max(local, world, dev)
    flops = all_reduce_sum(run.flops() * args.steps, world, dev)
    res = {"ms_per_step": max_ms / args.steps, "value": flops / (max_ms * 1e-3) / 1e12,
           "prefill_ms": statistics.mean(pre_ms), "append_ms": statistics.mean(app_ms),
           "prefill_tflops": run.flops() / (statistics.mean(pre_ms) * 1e-3) / 1e12,
           "append_gbs": run.append_bytes() / (app_kernel_ms * 1e-3) / 1e9, "append_kernel_ms": app_kernel_ms,
           "append_gbs_in_step": run.append_bytes() / (statistics.mean(app_ms) * 1e-3) / 1e9,
           "clocks": clk.summary(), "setup_s": setup_s, "launches": args.steps * 4,
           "cached": run.T, "flops_per_step": run.flops()}
    if not args.no_e2e:
        hq, hk, hv = (t.cpu().pin_memory() for t in (run.q, run.k_new, run.v_new))
        ho = torch.empty(run.out.shape, dtype=run.out.dtype, pin_memory=True)
        barrier(world)
        torch.cuda.synchronize()
        ms = 0.0
        for _ in range(args.steps):
            s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0.record()
            run.q.copy_(hq, non_blocking=True)
            run.k_new.copy_(hk, non_blocking=True)
            run.v_new.copy_(hv, non_blocking=True)
            run.step()
            ho.copy_(run.out, non_blocking=True)
            s1.record()
            torch.cuda.synchronize()
            ms += s0.elapsed_time(s1)
        max_e = all_reduce_max(ms, world, dev)
        res["e2e"] = {"value": flops / (max_e * 1e-3) / 1e12, "unit": "TFLOP/s",
                      "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in (hq, hk, hv)),
                      "d2h_bytes_per_step": ho.numel() * ho.element_size()}
    run.cache.close()
    return res


def oracle_prefill_rows(wl, kb, vb, budget_s: float) -> dict:
    """CPU baseline for prefill: the oracle's causal attention for chunk rows of
    one (sequence, KV head) slice (dequantise + attention in float64), timed
    over as many rows as fit in the budget; scaled to FLOP/s."""
    import numpy as np
    import oracle
    from asymmetric_quantized_kv_kvq_b200.inputs import gen_kv, gen_q_chunk, cached_lengths
    T = cached_lengths(wl)[0]
    C = wl.chunk
    k, v = gen_kv(wl, 0, 0, 0, T + C)
    kc, ks = oracle.quantize_kv(k.numpy(), kb)
    vc, vs = oracle.quantize_kv(v.numpy(), vb)
    q = gen_q_chunk(wl, 0, 0, C).numpy()
    rows, secs, flops = 0, 0.0, 0.0
    t0 = time.perf_counter()
    kh = oracle.dequantize_kv(kc, ks, kb)
    vh = oracle.dequantize_kv(vc, vs, vb)
    secs += time.perf_counter() - t0
    while secs < budget_s or rows == 0:
        r = (rows * 997) % C
        t0 = time.perf_counter()
        oracle.attention_prefill(q, kh, vh, T, rows=[r])
        secs += time.perf_counter() - t0
        flops += 4.0 * wl.n_q_heads * wl.head_dim * (T + r + 1)
        rows += 1
    return {"value": flops / secs / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{rows} chunk rows (all {wl.n_q_heads} q heads) of sequence 0 (cached {T}, chunk {C}): "
                      f"dequantise + causal attention in float64 NumPy, {secs:.1f} s"}


# --------------------------------------------------------------------------- distributed plumbing
def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _all_reduce(x: float, world: int, dev, op):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=op)
    return float(t.item())


def all_reduce_max(x, world, dev):
    import torch.distributed as dist
    return _all_reduce(x, world, dev, dist.ReduceOp.MAX) if world > 1 else x


def all_reduce_sum(x, world, dev):
    import torch.distributed as dist
    return _all_reduce(x, world, dev, dist.ReduceOp.SUM) if world > 1 else x


def gpu_uuid(dev) -> str:
    import torch
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return "0"


# --------------------------------------------------------------------------- CPU oracle leg
def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return 1


def prepare_oracle_slice(wl, kb, vb, layer=0, seq=0):
    """Stored form of one (layer, sequence) slice of the decode workload and its
    query, prepared (untimed) by the oracle's own quantiser."""
    import oracle
    from asymmetric_quantized_kv_kvq_b200.inputs import gen_kv, gen_q
    k, v = gen_kv(wl, layer, seq, 0, wl.cached)
    kc, ks = oracle.quantize_kv(k.numpy(), kb)
    vc, vs = oracle.quantize_kv(v.numpy(), vb)
    return kc, ks, vc, vs, gen_q(wl, layer, 0)[seq].numpy()


def time_oracle_slice(sl, kb, vb) -> float:
    """One decode step of the oracle on a slice: read the stored cache
    (dequantise codes + scales to float64) and attend with every query head."""
    import oracle
    kc, ks, vc, vs, q = sl
    t0 = time.perf_counter()
    kh = oracle.dequantize_kv(kc, ks, kb)
    vh = oracle.dequantize_kv(vc, vs, vb)
    oracle.attention_decode(q, kh, vh)
    return time.perf_counter() - t0


def slice_bytes(wl, kb, vb) -> int:
    D = wl.head_dim
    return wl.cached * wl.n_kv_heads * (tok_bytes(kb, D) + tok_bytes(vb, D)) + 2 * wl.n_q_heads * D * 2


def oracle_decode_slices(wl, kb, vb, budget_s: float) -> dict:
    """CPU baseline: the oracle timed on repeated decode steps of one
    (layer, sequence) slice until `budget_s` seconds of work are done."""
    sl = prepare_oracle_slice(wl, kb, vb)
    done, secs = 0, 0.0
    while secs < budget_s or done == 0:
        secs += time_oracle_slice(sl, kb, vb)
        done += 1
    return {"value": done * slice_bytes(wl, kb, vb) / secs / 1e9, "unit": "GB/s", "cores": blas_threads(),
            "kind": "oracle",
            "sample": f"{done} decode steps of one (layer, sequence) slice: {wl.cached} tokens x "
                      f"{wl.n_kv_heads} KV heads x {wl.group} q heads, dequantise + attention in float64 "
                      f"NumPy ({secs:.1f} s)"}


# --------------------------------------------------------------------------- main
def parse():
    from asymmetric_quantized_kv_kvq_b200.inputs import WORKLOADS
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=list(WORKLOADS), default=None,
                    help=f"default {DEFAULT_WORKLOAD} (plus the extra records)")
    ap.add_argument("--precision", default=None, help="K8V4, K8V8, K4V4, K4V8 or FP16 (default: first of the workload)")
    ap.add_argument("--layers", type=int, default=0, help="override the workload's layer count (profiling)")
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch (profiling)")
    ap.add_argument("--cached", type=int, default=0, help="override the cached tokens per sequence (profiling)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the CPU-oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--eager", action="store_true",
                    help="launch every decode step through the API calls directly instead of replaying a "
                         "CUDA graph of one captured step")
    ap.add_argument("--separate", action="store_true",
                    help="quantized caches: kvq_append + kvq_decode_attn per layer instead of the fused "
                         "kvq_decode_append_attn launch")
    ap.add_argument("--dedup-probe", action="store_true",
                    help="time one kvq_cache_dedup pass over the resident cache (on by default for the default run)")
    ap.add_argument("--no-extras", action="store_true",
                    help="default run: skip the 70B-shaped decode and the prefill sub-records")
    ap.add_argument("--layer-batched", action="store_true",
                    help="decode: one kvq_decode_attn_layers call per step (one launch per run of layers) "
                         "instead of one call per layer")
    ap.add_argument("--decode-tc", action="store_true",
                    help="decode on the tensor-core kernel (cache flag KVQ_CACHE_DECODE_TENSOR_CORES) "
                         "instead of the default CUDA-core kernel")
    a = ap.parse_args()
    if a.warmup < 3 and a.impl == "ours":
        ap.error("--warmup must be >= 3")
    return a


def config_of(wl, precision, world, flush) -> dict:
    return {"workload": wl.name, "precision": precision, "layers": wl.n_layers, "q_heads": wl.n_q_heads,
            "kv_heads": wl.n_kv_heads, "head_dim": wl.head_dim, "batch": wl.batch, "cached_tokens": wl.cached,
            "page_tokens": 256, "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "flushed between steps (2x L2 write)" if flush else "inputs larger than L2 (no flush)"}


def main():
    args = parse()
    from asymmetric_quantized_kv_kvq_b200.inputs import WORKLOADS, parse_precision
    default_run = args.workload is None
    args.workload = args.workload or DEFAULT_WORKLOAD
    args.dedup_probe = (default_run and not args.no_extras) or args.dedup_probe
    wl = WORKLOADS[args.workload]
    if args.layers or args.batch or args.cached:
        import dataclasses
        wl = dataclasses.replace(wl, n_layers=args.layers or wl.n_layers, batch=args.batch or wl.batch,
                                 cached=args.cached or wl.cached)
    precision = (args.precision or wl.precisions[0]).upper()
    kb, vb = parse_precision(precision)
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))

    if args.impl == "reference":
        if rank != 0:
            return
        if wl.chunk:
            r = oracle_prefill_rows(wl, kb, vb, budget_s=0.0)
            vals = [oracle_prefill_rows(wl, kb, vb, budget_s=1.0) for _ in range(args.steps)]
            val = statistics.mean(v["value"] for v in vals)
            line = {"metric": PREFILL_METRIC, "value": val, "unit": "TFLOP/s", "impl": "reference", "n_gpus": world, "device": "host cores (oracle)",
                    "steps": args.steps, "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True,
                    "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                    "config": {"workload": wl.name, "precision": precision},
                    "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                                     "sample": r["sample"]},
                    "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
            print(json.dumps(line), flush=True)
            return
        sl = prepare_oracle_slice(wl, kb, vb)
        times = [time_oracle_slice(sl, kb, vb) for _ in range(args.warmup + args.steps)][args.warmup:]
        secs = sum(times)
        val = args.steps * slice_bytes(wl, kb, vb) / secs / 1e9
        line = {"metric": METRIC, "value": val, "unit": "GB/s", "impl": "reference", "n_gpus": world, "device": "host cores (oracle)",
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": config_of(wl, precision, 1, False),
                "cpu_baseline": {"value": val, "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
                                 "sample": f"each step: one (layer, sequence) slice of {wl.cached} tokens, "
                                           f"dequantise + attention in float64 NumPy"},
                "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    import torch
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    from asymmetric_quantized_kv_kvq_b200 import build as kbuild
    if rank == 0:
        kbuild.build()
    barrier(world)

    if wl.chunk:
        prefill_main(args, wl, precision, kb, vb, rank, world)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    res = run_decode_bench(args, wl, kb, vb, rank, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_decode_slices(wl, kb, vb, args.cpu_seconds)
    extras = []
    if default_run and world == 1 and not args.no_extras:
        extras = run_extras(args)
    if rank == 0:
        line = decode_line(args, wl, precision, kb, vb, res, world)
        line["cpu_baseline"] = None if cpu is None else {k: cpu[k] for k in ("value", "unit", "cores", "kind",
                                                                             "sample")}
        if extras:
            line["extra"] = extras
        if "dedup" in res:
            line["dedup"] = res["dedup"]
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def decode_line(args, wl, precision, kb, vb, res, world) -> dict:
    """The JSON line of a decode run.  The roofline's dominant kernel is the decode
    kernel; for the fused one-launch step the replayed step is nothing but those
    launches, so its bytes / the step's own CUDA-event time is the kernel's
    achieved bandwidth (same basis as ms_per_step)."""
    peaks = measured_peaks()
    L = wl.n_layers
    isolated = res["kern_bytes_per_launch"] / (res["kern_ms_per_launch"] * 1e-3) / 1e9
    in_step = res["dec_bytes_per_launch"] / (res["dec_ms_per_launch"] * 1e-3) / 1e9
    tc = args.decode_tc and kb == 8 and vb in (4, 8) and wl.head_dim == 128
    R = res["runs"]                                   # launches of one step's decode (layers, or layer runs)
    per = "per run of layers" if res["batched"] else "per layer"
    if res["step_only_decode"]:
        achieved = res["value"]
        ms_launch = res["ms_per_step"] / R
        timing = (f"CUDA events around each replayed step = {R} back-to-back decode launches (one {per}, "
                  f"append and combine fused); ms_per_launch = ms_per_step / {R}")
        kernel = "decode_q_kernel (append + split-KV + combine)"
        bytes_launch = res["step_bytes"] / R
    else:
        achieved = isolated
        ms_launch = res["kern_ms_per_launch"]
        timing = ("CUDA events around 8 back-to-back layer-batched decode calls" if res["batched"] else
                  f"CUDA events around {max(L, 8)} back-to-back decode calls (one per layer)") + \
            " queued behind a device sleep; best of 2"
        if tc:
            kernel = "decode_tc_kernel + lse_combine_kernel"
        elif kb == 16:
            kernel = "decode_split_kernel + lse_combine_kernel"
        else:
            kernel = "decode_q_kernel (split-KV + combine)"
        bytes_launch = res["kern_bytes_per_launch"]
    traffic_kernel = "decode_tc" if tc else ("decode_split" if kb == 16 else "decode_q")
    line = {
        "metric": METRIC, "value": res["value"], "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": res["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": dict(config_of(wl, precision, world, res["flush"]),
                       decode_kernel="tensor cores (opt-in)" if tc else "CUDA cores",
                       step_launch=res["launch_mode"] + ("; one fused append+decode launch " + per
                                                         if res["fused"] else "") +
                       (f"; layer-batched (kvq_decode_attn_layers): {R} launch(es) for {L} layers"
                        if res["batched"] else "")),
        "decode_tokens_per_s": res["decode_tokens_per_s"],
        "roofline": {"bound": "hbm", "kernel": kernel, "achieved": achieved, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"], "peak_source": peaks["source"],
                     "frac_of_8tbs_nominal": achieved / 8000.0, "bytes_per_launch": bytes_launch,
                     "ms_per_launch": ms_launch, "timing": timing,
                     "achieved_isolated": isolated, "achieved_in_eager_step": in_step,
                     "traffic": ncu_traffic(wl.name, precision, traffic_kernel)},
        "cpu_baseline": None,
        "e2e": res.get("e2e"),
        "e2e_eager": res.get("e2e_eager"),
        "clocks": res["clocks"],
        "gpu_launches": res["launches"],
    }
    return line


def run_extras(args) -> list:
    """Compact records of the other gate workloads, measured in the same run: the
    70B-shaped 128K-token decode and the 22-layer TinyLlama-shaped 8K decode in K8V4
    and FP16 (per-layer calls and the layer-batched call), and the ragged chunked prefill."""
    import argparse as _ap
    import torch
    from asymmetric_quantized_kv_kvq_b200.inputs import WORKLOADS, parse_precision
    out = []
    sub = _ap.Namespace(**vars(args))
    # timed regions of a few hundred ms each, so that the clock sampler (100 ms) sees several samples
    sub.steps, sub.warmup, sub.no_e2e, sub.decode_tc, sub.separate = 20, 3, True, False, False
    sub.dedup_probe = False
    # per-layer calls (a model's step: each layer's query needs the previous layer's output), then
    # the layer-batched call (kvq_decode_attn_layers, every layer's query known at once)
    for name, prec, batched in (("llama70b-b1-128k", "K8V4", False), ("llama70b-b1-128k", "FP16", False),
                                ("llama70b-b1-128k", "K8V4", True), ("llama70b-b1-128k", "FP16", True),
                                ("tinyllama-22l-8k", "K8V4", False), ("tinyllama-22l-8k", "FP16", False),
                                ("tinyllama-22l-8k", "K8V4", True), ("tinyllama-22l-8k", "FP16", True)):
        wl = WORKLOADS[name]
        kb, vb = parse_precision(prec)
        sub.layer_batched = batched
        torch.cuda.empty_cache()
        r = run_decode_bench(sub, wl, kb, vb, 0, 1)
        line = decode_line(sub, wl, prec, kb, vb, r, 1)
        out.append({"workload": name, "precision": prec, "layer_batched": batched, "metric": "decode KV GB/s",
                    "value": r["value"], "unit": "GB/s", "ms_per_step": r["ms_per_step"], "steps": sub.steps,
                    "decode_tokens_per_s": r["decode_tokens_per_s"],
                    "roofline_frac": line["roofline"]["frac"], "kernel": line["roofline"]["kernel"],
                    "step_launch": line["config"]["step_launch"], "gpu_launches": r["launches"],
                    "l2": line["config"]["l2"], "clocks": r["clocks"]})
    sub.layer_batched = False
    wl = WORKLOADS["prefill-16x4096"]
    kb, vb = parse_precision("K8V4")
    torch.cuda.empty_cache()
    sub.steps = 10
    r = run_prefill_bench(sub, wl, kb, vb, 0, 1)
    peak = measured_tensor_peak()
    out.append({"workload": wl.name, "precision": "K8V4", "metric": PREFILL_METRIC, "value": r["value"],
                "unit": "TFLOP/s", "ms_per_step": r["ms_per_step"], "steps": sub.steps,
                "prefill_tflops": r["prefill_tflops"], "prefill_frac": r["prefill_tflops"] / peak["value"],
                "append_gbs": r["append_gbs"], "append_frac": r["append_gbs"] / measured_peaks()["hbm_gbs"],
                "gpu_launches": r["launches"], "clocks": r["clocks"]})
    return out


def prefill_main(args, wl, precision, kb, vb, rank, world):
    res = run_prefill_bench(args, wl, kb, vb, rank, world)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_prefill_rows(wl, kb, vb, args.cpu_seconds)
    if rank != 0:
        return
    peak = measured_tensor_peak()
    line = {
        "metric": PREFILL_METRIC, "value": res["value"], "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": res["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16 MMA, f32 accumulate", "data": "synthetic",
        "config": {"workload": wl.name, "precision": precision, "layers": wl.n_layers, "q_heads": wl.n_q_heads,
                   "kv_heads": wl.n_kv_heads, "head_dim": wl.head_dim, "sequences": wl.batch, "chunk": wl.chunk,
                   "cached_tokens": res["cached"], "page_tokens": 256,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "inputs larger than L2 (no flush)"},
        "prefill_tflops": res["prefill_tflops"], "append_gbs": res["append_gbs"],
        "prefill_ms": res["prefill_ms"], "append_ms": res["append_ms"],
        "append_roofline": {"bound": "hbm", "kernel": "append_kernel", "achieved": res["append_gbs"],
                            "peak": measured_peaks()["hbm_gbs"], "unit": "GB/s",
                            "frac": res["append_gbs"] / measured_peaks()["hbm_gbs"],
                            "ms_per_launch": res["append_kernel_ms"],
                            "timing": "CUDA events around 8 back-to-back appends of the chunk queued behind a "
                                      "device sleep",
                            "achieved_in_step": res["append_gbs_in_step"],
                            "traffic": ncu_traffic(wl.name, precision, "append")},
        "roofline": {"bound": "tensor", "kernel": "dequant_tiles_kernel + prefill_attn_kernel",
                     "achieved": res["prefill_tflops"], "peak": peak["value"], "unit": "TFLOP/s",
                     "frac": res["prefill_tflops"] / peak["value"], "peak_source": peak["source"],
                     "flops_per_launch": res["flops_per_step"], "traffic": None},
        "cpu_baseline": cpu, "e2e": res.get("e2e"), "clocks": res["clocks"], "gpu_launches": res["launches"],
    }
    print(json.dumps(line), flush=True)


def measured_tensor_peak() -> dict:
    """Dense fp16 / bf16 tensor peak (same rate on B200): the sustained figure,
    since one prefill launch runs tens of milliseconds of tensor work."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"value": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured bf16 dense, sustained (fp16 runs at the same rate)"}
    return {"value": 1400.0, "source": "fallback sustained"}


if __name__ == "__main__":
    main()
