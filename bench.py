#!/usr/bin/env python
"""Benchmark of the block-sparse KV attention hot path on B200.

Workload: the 48-chunk sweep at its headline point, chunk 48 (batch 1,
24 heads, head_dim 128, bf16; chunks of T=4, H=30, W=52 latent tokens =
49 blocks, 32 pad rows; 2303 history blocks; top-64 per query block plus the
49 own-chunk blocks = 113 selected blocks; geometric prior g ~ Beta(0.5, 2)
with 30% zeros, lambda = 2, g_ref = 0.2).  The cache of the 47 earlier
chunks is built before timing.

One step = one pass of the whole path over chunk 48:
  bsa_tokens_to_blocks_mean (Q and its block means) -> bsa_route_qmean,
  with bsa_kv_append (K, V) on a forked stream beside the route ->
  bsa_attn -> bsa_blocks_to_tokens (O)
and the chunk's blocks are rewritten in place every step.

Printed JSON line (rank 0):
  value         selected attention FLOPs / step time (TFLOP/s), whole job
  attn          bsa_attn alone: ms per call and TFLOP/s
  roofline      bsa_attn against the measured dense bf16 peak
  e2e           same metric with host inputs/outputs copied inside the step
  cpu_baseline  the fp64 oracle on a bounded sample (rank 0, N = 1)

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Multi-GPU (torchrun): every rank runs an independent problem of the same
size (its own heads of another layer) - weak scaling, no collective on the
data path; the time reported is the max over ranks.
"""
from __future__ import annotations

import argparse
import ctypes
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

CONFIG_KEY = 4
CHUNK = 48
BLK = 128
METRIC = "bsa_attn selected-block TFLOP/s at chunk 48 (48-chunk sweep), 1 B200"
L2_FLUSH_BYTES = 256 << 20
KERNELS_PER_STEP = 6  # append (fused), Q to blocks + means, score_means, topk, attn, O to tokens
# The step's attention kernel as ncu names it (block-order output, D = 128).
ATTN_KERNEL = "bsa_attn_kernel<128, false>"


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--chunk", type=int, default=CHUNK)
    ap.add_argument("--sweep", default="all",
                    help="chunks of the 48-chunk sweep at which sparse and dense bsa_attn are "
                         "timed (after the timed steps, each on the cache as it stood after "
                         "that chunk's append): 'all' (every chunk), a comma list, or '' to "
                         "skip; chunk 48 itself is the timed workload")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-config measurements (configs 1, 2, 3 and 5)")
    ap.add_argument("--no-oracle-ops", action="store_true",
                    help="skip the per-op, per-config oracle timings")
    return ap.parse_args()


def measured_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from profiles/traffic.json (one ncu
    capture of this workload), or None when the kernel's sources changed
    since the capture or there is no capture."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            entry = json.load(f)[kernel]
        h = hashlib.sha256()
        for rel in entry["files"]:
            with open(os.path.join(ROOT, rel), "rb") as f:
                h.update(f.read())
        if h.hexdigest()[:16] != entry["sources"]:
            return None
        return int(entry["read"]) + int(entry["write"])
    except (OSError, KeyError, ValueError):
        return None


def append_traffic():
    """DRAM bytes of one append (the fused gather + pooling launch), or None
    unless the capture matches the current sources."""
    return measured_traffic("append_gather_kernel<16>")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------

def dist_setup(n_gpus):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        pg = dist
    return rank, world, local, pg


def max_over_ranks(x: float, pg, device) -> float:
    if pg is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def barrier(pg, device):
    if pg is not None:
        if device.type == "cuda":
            pg.barrier(device_ids=[device.index])
        else:
            pg.barrier()


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.samples = []
        self.nvml_samples = []
        self.proc = None
        self.nvml_stop = threading.Event()
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            sel = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            return
        # NVML read every 10 ms, so a timed region of a fraction of a second
        # still gets many samples (read-only queries).
        try:
            import pynvml
            pynvml.nvmlInit()
            handle = pynvml.nvmlDeviceGetHandleByUUID(sel)
            self.nvml_thread = threading.Thread(target=self._poll_nvml, args=(pynvml, handle),
                                                daemon=True)
            self.nvml_thread.start()
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", sel, "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def _poll_nvml(self, nv, handle):
        try:
            mx = nv.nvmlDeviceGetMaxClockInfo(handle, nv.NVML_CLOCK_SM)
            bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
            while not self.nvml_stop.is_set():
                mhz = nv.nvmlDeviceGetClockInfo(handle, nv.NVML_CLOCK_SM)
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(handle)
                self.nvml_samples.append((time.time(), float(mhz), float(mx),
                                          {k for k, b in bits.items() if r & b}))
                time.sleep(0.01)
        except Exception:
            pass

    def stop(self):
        self.nvml_stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0, t1):
        rows = [s for (t, s) in self.samples if t0 <= t <= t1]
        if not rows:  # short region: take the samples nearest to it
            rows = [s for (t, s) in self.samples if t0 - 0.3 <= t <= t1 + 0.3]
        mhz, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            parts = [p.strip() for p in r.split(",")]
            if len(parts) < 9:
                continue
            try:
                mhz.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        n_smi = len(mhz)
        nv = [x for x in self.nvml_samples if t0 <= x[0] <= t1]
        for _, m, m_max, rs in nv:
            mhz.append(m)
            mx = mx if mx is not None else m_max
            reasons |= rs
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": mx,
                "sm_mhz_range": [min(mhz), max(mhz)] if mhz else None,
                "reasons": sorted(reasons), "samples": len(mhz),
                "sources": f"nvidia-smi -lms 100: {n_smi}, NVML every 10 ms: {len(nv)}"}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

_flush_bufs = {}


def l2_flush(device=None):
    """Write a buffer larger than L2 (kept per device)."""
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    buf = _flush_bufs.get(device)
    if buf is None:
        buf = _flush_bufs[device] = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    buf.zero_()


def _external_event_record():
    """cudaEventRecordWithFlags from the CUDA runtime torch has loaded, or
    None.  With cudaEventRecordExternal (1) an event recorded during stream
    capture becomes an event-record node of the graph."""
    try:
        lib = ctypes.CDLL("libcudart.so.12")
        f = lib.cudaEventRecordWithFlags
    except (OSError, AttributeError):
        return None
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_uint]
    f.restype = ctypes.c_int
    return f


def _cuda_ok(status: int):
    if status != 0:
        raise RuntimeError(f"cudaEventRecordWithFlags failed ({status})")


def capture(fn):
    """fn's launches as a CUDA graph.  The library's calls take the current
    stream and neither allocate nor synchronise when given their outputs and
    workspace, so they capture as they are; replaying the graph runs the same
    kernels on the same buffers without the per-call host marshalling."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def _time_call(fn, reps=3):
    """Median CUDA-event time (ms) of fn() over `reps` calls: fn is run once,
    captured as a CUDA graph, and each timed replay follows an L2 flush, so
    the GPU is busy while the host records the events."""
    fn()
    g = capture(fn)
    ts = []
    for _ in range(reps):
        l2_flush()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    del g
    return sorted(ts)[len(ts) // 2]


def sweep_point(bsa, w, cache, q_tok, c, own_first, nbc, device):
    """bsa_attn of chunk c with its routed top-K and with every cache block
    selected (dense): the per-chunk comparison of the 48-chunk sweep."""
    T, H, W = w.grid
    n_hist = own_first
    q_blk = bsa.bsa_tokens_to_blocks(q_tok, T, H, W)
    g = synth.prior(w, c, nbc, n_hist) if n_hist > 0 else None
    g = torch.from_numpy(g).to(device) if g is not None else None
    q_valid = cache.block_valid[own_first:own_first + nbc].clone()
    idx, cnt = bsa.bsa_route(q_blk, cache, n_hist, own_first, nbc, w.top_k[0], g=g, lam=w.lam,
                             g_ref=w.g_ref, sm_scale=w.sm_scale, q_valid=q_valid)
    n_all = cache.n_blocks
    idx_d = torch.arange(n_all, dtype=torch.int32, device=device).expand(
        w.B, w.Hh, nbc, n_all).contiguous()
    cnt_d = torch.full((w.B, w.Hh, nbc), n_all, dtype=torch.int32, device=device)
    o = torch.empty_like(q_blk)
    lse = torch.empty((w.B, w.Hh, nbc * BLK), dtype=torch.float32, device=device)
    sp = _time_call(lambda: bsa.bsa_attn(q_blk, cache, idx, cnt, q_valid=q_valid,
                                         sm_scale=w.sm_scale, o=o, lse=lse))
    dn = _time_call(lambda: bsa.bsa_attn(q_blk, cache, idx_d, cnt_d, q_valid=q_valid,
                                         sm_scale=w.sm_scale, o=o, lse=lse))
    bsa.raise_on_device_error(device)
    sel = int(cnt[0, 0, 0].item())
    return {"chunk": c, "selected_blocks": sel, "all_blocks": n_all,
            "sparse_ms": round(sp, 4), "dense_ms": round(dn, 4), "speedup": round(dn / sp, 2)}


# Every synthetic config measured op by op at 1 GPU: (config, top-K).  The
# dense-equivalence config runs once with every history block selected
# (top-K 256 = all 256 history blocks) and once with top-32.
CONFIG_RUNS = ((1, 3), (2, 16), (3, 50), (5, 256), (5, 32))


def _frac(x, peak):
    return round(x / peak, 4) if peak else None


def config_point(key: int, top_k: int, device, peaks: dict, reps: int = 5) -> dict:
    """One synthetic config, op by op: the cache of its history is built
    (appended chunks, or blocks written directly and pooled), then the query
    chunk's append (rewritten in place), Q reordering, route (from the
    pooled-key cache) and attention are each captured as a CUDA graph and
    timed after an L2 flush (median of ``reps``).  Each op is reported with
    its algorithmic bytes or selected FLOPs and its roofline fraction."""
    import block_sparse_kv_bsa_b200 as bsa
    w = synth.CONFIGS[key]
    T, H, W = w.grid
    nbc = w.blocks_per_chunk
    n_hist = w.n_hist
    cache = bsa.KVCache(w.B, w.Hh, w.D, n_hist + nbc, device=device, pooled_keys=True)
    if w.hist_direct:
        kd, vd = synth.direct_blocks(w, w.hist_direct, device=device)
        cache.k[:, :, :w.hist_direct] = kd
        cache.v[:, :, :w.hist_direct] = vd
        cache.block_valid[:w.hist_direct] = BLK
        cache.n_blocks = w.hist_direct
        bsa.bsa_kv_pool_means(cache, 0, w.hist_direct)
        del kd, vd
    for c in range(1, w.hist_chunks + 1):
        t = synth.chunk_tokens(w, c, device=device, want=("k", "v"))
        bsa.bsa_kv_append(cache, t["k"], t["v"], T, H, W)
    qc = w.hist_chunks + 1 if w.hist_direct == 0 else 1
    t = synth.chunk_tokens(w, qc, device=device)
    own_first = cache.n_blocks
    bsa.bsa_kv_append(cache, t["k"], t["v"], T, H, W)
    q_tok, k_tok, v_tok = t["q"], t["k"], t["v"]
    g = synth.prior(w, qc, nbc, n_hist) if n_hist > 0 else None
    g = torch.from_numpy(g).to(device) if g is not None else None
    q_valid = cache.block_valid[own_first:own_first + nbc].clone()
    q_blk = torch.empty((w.B, w.Hh, nbc * BLK, w.D), dtype=torch.bfloat16, device=device)
    q_mean = torch.empty((w.B, w.Hh, nbc, w.D), dtype=torch.float32, device=device)
    bsa.bsa_tokens_to_blocks_mean(q_tok, T, H, W, out=q_blk, mean=q_mean)
    max_sel = bsa.route_max_sel(top_k, n_hist, nbc)
    idx = torch.empty((w.B, w.Hh, nbc, max_sel), dtype=torch.int32, device=device)
    cnt = torch.empty((w.B, w.Hh, nbc), dtype=torch.int32, device=device)
    ws = torch.empty(max(bsa.bsa_route_workspace_size(w.B, w.Hh, w.D, nbc, n_hist), 256),
                     dtype=torch.uint8, device=device)
    o = torch.empty_like(q_blk)
    lse = torch.empty((w.B, w.Hh, nbc * BLK), dtype=torch.float32, device=device)

    def append():
        cache.n_blocks = own_first
        bsa.bsa_kv_append(cache, k_tok, v_tok, T, H, W)

    def route():
        bsa.bsa_route_qmean(q_mean, cache, n_hist, own_first, nbc, top_k, g=g, lam=w.lam,
                            g_ref=w.g_ref, sm_scale=w.sm_scale, max_sel=max_sel, idx=idx,
                            cnt=cnt, workspace=ws)

    def attn():
        bsa.bsa_attn(q_blk, cache, idx, cnt, q_valid=q_valid, sm_scale=w.sm_scale, o=o, lse=lse)

    route()
    attn()
    bsa.raise_on_device_error(device)
    t_app = _time_call(append, reps)
    t_q = _time_call(lambda: bsa.bsa_tokens_to_blocks_mean(q_tok, T, H, W, out=q_blk,
                                                           mean=q_mean), reps)
    t_route = _time_call(route, reps)
    t_attn = _time_call(attn, reps)
    bsa.raise_on_device_error(device)
    sel = cnt.to(torch.float64)
    flops = float(sel.sum().item()) * 4.0 * BLK * BLK * w.D
    tok_b = w.B * w.tokens * w.Hh * w.D * 2
    blk_b = w.B * w.Hh * nbc * BLK * w.D * 2
    app_b = 2 * (tok_b + blk_b) + w.B * w.Hh * nbc * w.D * 4
    qm_b = w.B * w.Hh * nbc * w.D * 4
    q_b = tok_b + blk_b + qm_b
    route_b = (qm_b + w.B * w.Hh * n_hist * w.D * 4 + (0 if g is None else g.numel() * 4)
               + 2 * w.B * w.Hh * nbc * n_hist * 4 + (idx.numel() + cnt.numel()) * 4)
    hbm, tc = peaks["hbm_gbs"], peaks["bf16_tflops"]

    def gbs(b, ms):
        return round(b / (ms * 1e-3) / 1e9, 1)
    out = {
        "config": key, "name": w.name, "top_k": top_k,
        "shape": f"B{w.B} Hh{w.Hh} D{w.D}, chunk {T}x{H}x{W} ({nbc} blocks), "
                 f"{n_hist} history blocks" + (", prior" if g is not None else ""),
        "selected_blocks_per_query_block": {"min": int(sel.min().item()),
                                            "max": int(sel.max().item())},
        "attn": {"ms_per_call": round(t_attn, 4),
                 "tflops": round(flops / (t_attn * 1e-3) / 1e12, 2),
                 "frac_of_bf16_peak": _frac(flops / (t_attn * 1e-3) / 1e12, tc),
                 "selected_tflop_per_call": round(flops / 1e12, 5)},
        "route": {"ms_per_call": round(t_route, 4), "gbs": gbs(route_b, t_route),
                  "frac_of_hbm": _frac(route_b / (t_route * 1e-3) / 1e9, hbm),
                  "bytes_per_call": int(route_b), "keys": "pooled-key cache"},
        "append": {"ms_per_call": round(t_app, 4), "gbs": gbs(app_b, t_app),
                   "frac_of_hbm": _frac(app_b / (t_app * 1e-3) / 1e9, hbm),
                   "bytes_per_call": int(app_b)},
        "q_to_blocks": {"ms_per_call": round(t_q, 4), "gbs": gbs(q_b, t_q),
                        "frac_of_hbm": _frac(q_b / (t_q * 1e-3) / 1e9, hbm),
                        "bytes_per_call": int(q_b)},
    }
    if key == 5 and top_k >= n_hist:
        out["note"] = "every history block selected: dense attention over the cache"
    del cache
    return out


class State:
    """Device-resident inputs and preallocated outputs of one rank's problem."""

    def __init__(self, w, chunk, device, seed_rank=0, sweep_chunks=()):
        import block_sparse_kv_bsa_b200 as bsa
        self.bsa = bsa
        self.w = w
        T, H, W = w.grid
        self.grid = (T, H, W)
        nbc = w.blocks_per_chunk
        self.n_own = nbc
        self.n_hist = nbc * (chunk - 1)
        self.device = device
        # The pooled-key cache: bsa_kv_append writes each block's key mean, and
        # bsa_route scores from those instead of re-reading the history keys.
        self.cache = bsa.KVCache(w.B, w.Hh, w.D, self.n_hist + nbc, device=device,
                                 pooled_keys=True)
        # A different rank solves a different, equally sized problem.
        wr = w if seed_rank == 0 else synth.Workload(**{**w.__dict__, "key": w.key + 100 * seed_rank})
        self.wr = wr
        self.sweep = []
        self.sweep_pending = []     # (chunk, its first block): timed by run_sweep
        for c in range(1, chunk):
            t = synth.chunk_tokens(wr, c, device=device, want=("k", "v"))
            first = self.cache.n_blocks
            bsa.bsa_kv_append(self.cache, t["k"], t["v"], T, H, W)
            if c in sweep_chunks:
                self.sweep_pending.append((c, first))
        self.own_first = self.cache.n_blocks
        t = synth.chunk_tokens(wr, chunk, device=device)
        self.k_tok, self.v_tok, self.q_tok = t["k"], t["v"], t["q"]
        g = synth.prior(wr, chunk, nbc, self.n_hist)
        self.g = torch.from_numpy(g).to(device) if g is not None else None
        self.q_blk = torch.empty((w.B, w.Hh, nbc * BLK, w.D), dtype=torch.bfloat16, device=device)
        self.q_mean = torch.empty((w.B, w.Hh, nbc, w.D), dtype=torch.float32, device=device)
        self.max_sel = bsa.route_max_sel(w.top_k[0], self.n_hist, nbc)
        self.idx = torch.empty((w.B, w.Hh, nbc, self.max_sel), dtype=torch.int32, device=device)
        self.cnt = torch.empty((w.B, w.Hh, nbc), dtype=torch.int32, device=device)
        ws = bsa.bsa_route_workspace_size(w.B, w.Hh, w.D, nbc, self.n_hist)
        self.ws = torch.empty(max(ws, 256), dtype=torch.uint8, device=device)
        self.o_blk = torch.empty_like(self.q_blk)
        self.lse = torch.empty((w.B, w.Hh, nbc * BLK), dtype=torch.float32, device=device)
        self.o_tok = torch.empty_like(self.q_tok)
        self.side = torch.cuda.Stream(device)
        self.step_graph = None
        bsa.bsa_kv_append(self.cache, self.k_tok, self.v_tok, T, H, W)
        torch.cuda.synchronize(device)
        self.q_valid = self.cache.block_valid[self.own_first:self.own_first + nbc].clone()

    def calls(self):
        """The five library calls of one step, in order, as (name, fn): the
        query chunk is reordered and pooled in one pass, the route scores
        from those means (so the query blocks are read once), and O goes
        back to raster token order after the attention.  (bsa_attn_tokens,
        which writes O in token order from the attention epilogue, measured
        slower at chunk 48: 1.016 ms against 0.967 + 0.020 ms.)"""
        bsa, w = self.bsa, self.w
        T, H, W = self.grid

        def append():
            self.cache.n_blocks = self.own_first   # the chunk's blocks are rewritten in place
            bsa.bsa_kv_append(self.cache, self.k_tok, self.v_tok, T, H, W)
        return [
            ("append", append),
            ("q_to_blocks", lambda: bsa.bsa_tokens_to_blocks_mean(
                self.q_tok, T, H, W, out=self.q_blk, mean=self.q_mean)),
            ("route", lambda: bsa.bsa_route_qmean(
                self.q_mean, self.cache, self.n_hist, self.own_first, self.n_own, w.top_k[0],
                g=self.g, lam=w.lam, g_ref=w.g_ref, sm_scale=w.sm_scale, max_sel=self.max_sel,
                idx=self.idx, cnt=self.cnt, workspace=self.ws)),
            ("attn", lambda: bsa.bsa_attn(self.q_blk, self.cache, self.idx, self.cnt,
                                          q_valid=self.q_valid, sm_scale=w.sm_scale,
                                          o=self.o_blk, lse=self.lse)),
            ("o_to_tokens", lambda: bsa.bsa_blocks_to_tokens(self.o_blk, T, H, W,
                                                             out=self.o_tok)),
        ]

    def run_sweep(self):
        """The sweep points of the chunks before the timed one, each on the
        cache as it stood after that chunk's append (a prefix of the final
        cache: later appends write only later blocks), with that chunk's
        query tokens drawn again from their seed.  Run after the timed
        steps, so that the dense calls (up to 18 ms each) do not heat the GPU
        just before them."""
        nbc = self.n_own
        T, H, W = self.grid
        saved = self.cache.n_blocks
        try:
            for c, first in self.sweep_pending:
                self.cache.n_blocks = first + nbc
                q = synth.chunk_tokens(self.wr, c, device=self.device, want=("q",))["q"]
                self.sweep.append(sweep_point(self.bsa, self.wr, self.cache, q, c, first, nbc,
                                              self.device))
        finally:
            self.cache.n_blocks = saved
        self.sweep_pending = []

    def step(self, record=None):
        """One pass of the whole path through the library's calls.

        The append of the chunk's K/V and the route do not depend on each
        other (the route reads only the history's pooled keys and valid
        counts, the append writes only the chunk's own blocks), so the
        append runs on a side stream while the route runs: the HBM-bound
        append fills the time of the latency-bound route kernels (started
        together with the HBM-bound Q reordering instead, the two streams
        only slowed each other).  The attention waits for both.
        ``record(i, stream)`` marks the event points 0..6: start, Q
        reordered, append done (side stream), routed, joined, attention
        done, O reordered."""
        main = torch.cuda.current_stream(self.device)
        calls = dict(self.calls())
        mark = record if record is not None else (lambda i, stream: None)
        mark(0, main)
        calls["q_to_blocks"]()
        mark(1, main)
        self.side.wait_stream(main)
        with torch.cuda.stream(self.side):
            calls["append"]()
            mark(2, self.side)
        calls["route"]()
        mark(3, main)
        main.wait_stream(self.side)
        mark(4, main)
        calls["attn"]()
        mark(5, main)
        calls["o_to_tokens"]()
        mark(6, main)

    # (name, first event, last event) of each timed span of a step
    SPANS = (("q_to_blocks", 0, 1), ("append", 1, 2), ("route", 1, 3), ("attn", 4, 5),
             ("o_to_tokens", 5, 6), ("step", 0, 6))
    N_EVENTS = 7

    def capture(self):
        """The step as one CUDA graph (the side stream's fork and join become
        graph edges) with event-record nodes (cudaEventRecordExternal) at the
        step's event points.  The node events are rewritten by every replay,
        so each step is read back before the next.  Fallback (runtime entry
        point not found): the graph without event nodes, with events
        recorded around the replay only (per-call times then come from
        isolated per-call graphs)."""
        self.call_names = [name for name, _ in self.calls()]
        self.step_graph = None
        self.node_events = [torch.cuda.Event(enable_timing=True) for _ in range(self.N_EVENTS)]
        for e in self.node_events:
            e.record()                   # creates the events before the capture
        torch.cuda.synchronize(self.device)
        record = _external_event_record()
        if record is not None:
            def mark(i, stream):
                _cuda_ok(record(self.node_events[i].cuda_event, stream.cuda_stream, 1))
            self.step_graph = capture(lambda: self.step(mark))
            self.node_timing = True
        else:
            self.step_graph = capture(self.step)
            self.node_timing = False
        self.timing = ("one CUDA graph per step (append on a forked stream, overlapping the "
                       "route), event-record nodes at the step's event points"
                       if self.node_timing else
                       "one CUDA graph per step (append on a forked stream), events around "
                       "the replay")

    def replay(self):
        """One step from the captured graph; then self.read_times() gives the
        span times (ms) of SPANS, after the step has completed."""
        if self.node_timing:
            self.step_graph.replay()
            return
        ev = self.node_events
        ev[0].record()
        self.step_graph.replay()
        ev[-1].record()

    def read_times(self):
        ev = self.node_events
        if not self.node_timing:
            return {"step": ev[0].elapsed_time(ev[-1])}
        return {name: ev[a].elapsed_time(ev[b]) for name, a, b in self.SPANS}

    def isolated_ms(self, reps: int = 10) -> dict:
        """Each call of the step timed on its own (a CUDA graph of the call,
        replayed after an L2 flush, median of ``reps``): the per-call
        figures behind the HBM fractions, free of the overlap inside a step."""
        return {name: _time_call(fn, reps) for name, fn in self.calls()}

    def release_graphs(self):
        self.step_graph = None

    def route_bytes(self, from_means: bool = True) -> float:
        """Algorithmic bytes of the route.  From means (bsa_route_qmean on the
        pooled-key cache): the query means and the history key means read.
        Streaming (bsa_route on the query blocks, no pooled-key cache): the
        query blocks and every history key block read.  Both: g read, model
        scores written and read back by top-K, idx/cnt written."""
        w = self.w
        if from_means:
            q = w.B * w.Hh * self.n_own * w.D * 4
            k = w.B * w.Hh * self.n_hist * w.D * 4
        else:
            q = w.B * w.Hh * self.n_own * BLK * w.D * 2
            k = w.B * w.Hh * self.n_hist * BLK * w.D * 2
        g = 0 if self.g is None else self.g.numel() * 4
        s = 2 * w.B * w.Hh * self.n_own * self.n_hist * 4
        idx = (self.idx.numel() + self.cnt.numel()) * 4
        return float(q + k + g + s + idx)

    def append_bytes(self) -> float:
        """K and V tokens read, the chunk's cache blocks written, and the
        chunk's key means written."""
        w = self.w
        tok = w.B * w.tokens * w.Hh * w.D * 2
        blk = w.B * w.Hh * self.n_own * BLK * w.D * 2
        means = w.B * w.Hh * self.n_own * w.D * 4
        return float(2 * (tok + blk) + means)

    def velox_point(self, reps: int = 10) -> dict:
        """The page's own route at this chunk (Velox constants; synthetic
        coverage and prior), timed, and bsa_attn timed on those routes.  The
        route takes the query means of the step's Q reordering, as the step's
        own route does (bsa_route_velox_qmean)."""
        w, bsa = self.w, self.bsa
        cov = torch.from_numpy(synth.coverage(w, CHUNK, self.n_own)).to(self.device)
        kw = dict(g=self.g, coverage=cov, lam=w.lam, g_ref=w.g_ref, sm_scale=w.sm_scale,
                  tau=0.1, eta_cov=0.9, k_cov=80, k_unc=150, mass=0.9,
                  prev_first=self.own_first - self.n_own, n_prev=self.n_own, window_half=13,
                  q_mean=self.q_mean, workspace=self.ws)
        idx, cnt = bsa.bsa_route_velox(None, self.cache, self.n_hist, self.own_first,
                                       self.n_own, **kw)
        o = torch.empty_like(self.q_blk)
        lse = torch.empty(self.q_blk.shape[:3], dtype=torch.float32, device=self.device)
        rt = _time_call(lambda: bsa.bsa_route_velox(None, self.cache, self.n_hist,
                                                    self.own_first, self.n_own, idx=idx,
                                                    cnt=cnt, **kw), reps)
        at = _time_call(lambda: bsa.bsa_attn(self.q_blk, self.cache, idx, cnt,
                                             q_valid=self.q_valid, sm_scale=w.sm_scale, o=o,
                                             lse=lse), reps)
        bsa.raise_on_device_error(self.device)
        c = cnt.to(torch.float64)
        flops = float(c.sum().item()) * 4.0 * BLK * BLK * w.D
        return {"route_ms": round(rt, 4), "attn_ms": round(at, 4),
                "attn_tflops": round(flops / (at * 1e-3) / 1e12, 1),
                "blocks_per_query_block": {"mean": round(float(c.mean().item()), 1),
                                           "min": int(c.min().item()),
                                           "max": int(c.max().item())},
                "covered_query_blocks": int((cov >= 0.9).sum().item()),
                "query_means": "from the step's Q reordering (bsa_route_velox_qmean)",
                "constants": "tau 0.1, g_ref 0.2, lambda 2, eta_cov 0.9, K_cov 80, "
                             "K_unc 150, mass 0.9, window +/-13 in the previous chunk"}

    def geometry_point(self, reps: int = 20) -> dict:
        """The geometric prior computed on the GPU (bsa_geometry_prior: slab
        boxes, separating-axis test, 8^3 grid IoU, coverage) from seeded
        synthetic slabs of this chunk's history, timed; then the page's route
        from that g and coverage, and bsa_attn on those routes."""
        w, bsa = self.w, self.bsa
        sc = synth.slab_scene(w.grid, self.n_hist // self.n_own, self.n_own,
                              seed=1000 * w.key + 800 + CHUNK)

        def dev(x, dtype):
            return torch.from_numpy(np.ascontiguousarray(x)[None]).to(self.device, dtype)
        t = {k: dev(getattr(sc, k), torch.float32) for k in ("cams", "h_rect", "q_rect", "tok_uvd")}
        t.update({k: dev(getattr(sc, k), torch.int32) for k in ("h_cam", "q_cam", "tok_cam")})

        def call():
            return bsa.bsa_geometry_prior(t["cams"], sc.intr, t["h_cam"], t["h_rect"], t["q_cam"],
                                          t["q_rect"], t["tok_cam"], t["tok_uvd"],
                                          q_valid=self.q_valid, grid_n=8)
        g, cov = call()
        gt = _time_call(call, reps)
        kw = dict(g=g, coverage=cov, lam=w.lam, g_ref=w.g_ref, sm_scale=w.sm_scale, tau=0.1,
                  eta_cov=0.9, k_cov=80, k_unc=150, mass=0.9,
                  prev_first=self.own_first - self.n_own, n_prev=self.n_own, window_half=13,
                  q_mean=self.q_mean, workspace=self.ws)
        idx, cnt = bsa.bsa_route_velox(None, self.cache, self.n_hist, self.own_first,
                                       self.n_own, **kw)
        o = torch.empty_like(self.q_blk)
        lse = torch.empty(self.q_blk.shape[:3], dtype=torch.float32, device=self.device)
        rt = _time_call(lambda: bsa.bsa_route_velox(None, self.cache, self.n_hist,
                                                    self.own_first, self.n_own, idx=idx,
                                                    cnt=cnt, **kw), 10)
        at = _time_call(lambda: bsa.bsa_attn(self.q_blk, self.cache, idx, cnt,
                                             q_valid=self.q_valid, sm_scale=w.sm_scale, o=o,
                                             lse=lse), 10)
        bsa.raise_on_device_error(self.device)
        c = cnt.to(torch.float64)
        n_slab_pairs = int((t["q_cam"] >= 0).sum().item()) * int((t["h_cam"] >= 0).sum().item())
        return {"prior_ms": round(gt, 4),
                "slab_box_pairs": n_slab_pairs,
                "token_slab_tests": int((t["tok_cam"] >= 0).sum().item()) *
                int((t["h_cam"] >= 0).sum().item()),
                "g_nonzero_frac": round(float((g > 0).double().mean().item()), 4),
                "coverage_mean": round(float(cov.double().mean().item()), 4),
                "route_ms": round(rt, 4), "attn_ms": round(at, 4),
                "blocks_per_query_block": {"mean": round(float(c.mean().item()), 1),
                                           "min": int(c.min().item()),
                                           "max": int(c.max().item())},
                "scene": "seeded synthetic slabs: camera trajectory, wall at z=14, "
                         "foreground objects; grid 8^3"}

    def route_stream_ms(self, reps: int = 20) -> float:
        """bsa_route timed without the pooled-key cache, i.e. streaming every
        history key block (L2 flushed before each call)."""
        w, bsa = self.w, self.bsa
        saved = self.cache.kmean
        self.cache.kmean = None
        try:
            return _time_call(lambda: bsa.bsa_route(
                self.q_blk, self.cache, self.n_hist, self.own_first, self.n_own, w.top_k[0],
                g=self.g, lam=w.lam, g_ref=w.g_ref, sm_scale=w.sm_scale, q_valid=self.q_valid,
                max_sel=self.max_sel, idx=self.idx, cnt=self.cnt, workspace=self.ws), reps)
        finally:
            self.cache.kmean = saved

    def selected_flops(self) -> float:
        c = self.cnt.to(torch.float64).sum().item()
        return c * 4.0 * BLK * BLK * self.w.D


def append_entry(st, ms: float, in_step_ms, peaks: dict, traffic) -> dict:
    """The append's figures: algorithmic bytes over its isolated time, and,
    beside them, the DRAM bytes one ncu capture measured over the same time.
    Part of the append's writes are still in L2 when it ends (they reach
    DRAM during the next kernels), so the DRAM figure is the lower one."""
    b = st.append_bytes()
    out = {"ms_per_call": round(ms, 4),
           "in_step_ms": round(in_step_ms, 4) if in_step_ms is not None else None,
           "gbs": round(b / (ms * 1e-3) / 1e9, 1),
           "frac_of_hbm": round(b / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
           "bytes_per_call": int(b), "traffic": traffic}
    if traffic:
        out["dram_gbs"] = round(traffic / (ms * 1e-3) / 1e9, 1)
        out["dram_frac_of_hbm"] = round(traffic / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)
        out["dram_note"] = ("traffic = DRAM bytes of one ncu capture; writes still in L2 at "
                            "the kernel's end are not in it")
    return out


def run_ours(args, rank, world, local, pg):
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    w = synth.CONFIGS[CONFIG_KEY]
    sweep = set()
    if rank == 0 and args.sweep.strip() == "all":
        sweep = set(range(1, args.chunk))
    elif rank == 0:
        sweep = {int(x) for x in args.sweep.split(",") if x.strip()}
    st = State(w, args.chunk, device, seed_rank=rank, sweep_chunks=sweep)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    _flush_bufs[device] = flush            # the same buffer for the per-call timings

    # Warm-up through the library's calls; then each call is captured as a
    # CUDA graph, and the graphs are warmed up too.
    warm = max(args.warmup, 3)
    for _ in range(warm):
        st.step()
    st.bsa.raise_on_device_error(device)
    flops = st.selected_flops()
    st.capture()
    for _ in range(warm):
        flush.zero_()
        st.replay()
        torch.cuda.synchronize(device)
        st.read_times()
    st.bsa.raise_on_device_error(device)

    clocks = ClockSampler(device) if rank == 0 else None
    time.sleep(0.25)
    barrier(pg, device)
    torch.cuda.synchronize(device)
    t_wall0 = time.time()
    torch.cuda.nvtx.range_push("timed")
    step_times = []
    for _ in range(args.steps):
        flush.zero_()  # L2 flush between steps, outside the timed events
        st.replay()
        torch.cuda.synchronize(device)   # the step's events are read before the next replay
        step_times.append(st.read_times())
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize(device)
    barrier(pg, device)
    t_wall1 = time.time()
    st.bsa.raise_on_device_error(device)
    per_step = [t["step"] for t in step_times]
    total_ms = max_over_ranks(sum(per_step), pg, device)
    st.release_graphs()
    # Each call alone (its own graph, L2 flushed): the figures behind the
    # per-call HBM fractions, since inside a step the append overlaps the
    # Q reorder and the route.
    isolated = {k: max_over_ranks(v, pg, device) for k, v in st.isolated_ms().items()}
    # Span times from the timed region itself (event nodes of the step graph);
    # the attention span has the GPU to itself.
    phase_ms = {name: sum(t[name] for t in step_times) / args.steps
                for name, _, _ in st.SPANS if name in step_times[0]}
    phase_ms = {k: max_over_ranks(v, pg, device) for k, v in phase_ms.items()}
    attn_avg = phase_ms.get("attn", isolated["attn"])
    spread = sorted(per_step)
    step_spread = {"min": round(spread[0], 4), "median": round(spread[len(spread) // 2], 4),
                   "max": round(spread[-1], 4)}
    clock_info = None
    if clocks is not None:
        time.sleep(0.3)
        clocks.stop()
        clock_info = clocks.summary(t_wall0, t_wall1)

    route_stream = st.route_stream_ms()
    velox = st.velox_point() if rank == 0 else None
    geometry = st.geometry_point() if rank == 0 else None
    if rank == 0 and st.sweep is not None and args.sweep:
        st.run_sweep()
        st.sweep.append(sweep_point(st.bsa, w, st.cache, st.q_tok, args.chunk, st.own_first,
                                    st.n_own, device))
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(st, args, device, pg, flops)
    per_config = None
    if rank == 0 and not args.no_configs:
        per_config = [config_point(k, kk, device, load_peaks()) for k, kk in CONFIG_RUNS]

    ms_per_step = total_ms / args.steps
    value = flops * world / (ms_per_step * 1e-3) / 1e12
    peaks = load_peaks()
    attn_tflops = flops / (attn_avg * 1e-3) / 1e12
    out = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": max(args.warmup, 3),
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; N(0,1) Q/K/V with per-tile N(0,0.5^2) offsets on Q/K; "
                "g ~ Beta(0.5,2) with 30% zeros)",
        "config": {"workload": "48-chunk sweep, chunk 48: B1 Hh24 D128, chunk 4x30x52 "
                               "(49 blocks), 2303 history blocks, top-64 + own chunk, prior",
                   "chunk": args.chunk, "global_batch": w.B * world, "heads": w.Hh,
                   "head_dim": w.D, "selected_blocks_per_query_block": st.max_sel,
                   "parallelism": f"independent problem per rank x{world}",
                   "l2": "flushed between steps (256 MB write outside the timed events); "
                         "step inputs also exceed L2"},
        "attn": {"ms_per_call": round(attn_avg, 4), "tflops": round(attn_tflops, 2),
                 "selected_tflop_per_call": round(flops / 1e12, 4)},
        "phases_ms": {k: round(v, 4) for k, v in phase_ms.items()},
        "phases_note": "spans inside the timed steps: append runs on a forked stream while "
                       "the route runs, so those two overlap; q_to_blocks, attn and "
                       "o_to_tokens have the GPU to themselves",
        "isolated_ms": {k: round(v, 4) for k, v in isolated.items()},
        "step_ms_spread": step_spread,
        "timing": st.timing + "; each step read back before the next",
        "route": {"ms_per_call": round(isolated["route"], 4),
                  "in_step_ms": round(phase_ms["route"], 4) if "route" in phase_ms else None,
                  "keys": "pooled-key cache (means written by bsa_kv_append)",
                  "gbs": round(st.route_bytes() / (isolated["route"] * 1e-3) / 1e9, 1),
                  "bytes_per_call": int(st.route_bytes())},
        "route_stream": {"ms_per_call": round(route_stream, 4),
                         "keys": "history keys streamed from the cache (no pooled-key cache)",
                         "gbs": round(st.route_bytes(False) / (route_stream * 1e-3) / 1e9, 1),
                         "frac_of_hbm": round(st.route_bytes(False) / (route_stream * 1e-3) / 1e9
                                              / peaks["hbm_gbs"], 4),
                         "bytes_per_call": int(st.route_bytes(False)),
                         "pool_score_traffic": (measured_traffic("pool_score_kernel<16>")
                                                if args.chunk == CHUNK else None)},
        "append": append_entry(st, isolated["append"], phase_ms.get("append"), peaks,
                               append_traffic() if args.chunk == CHUNK else None),
        "roofline": {"bound": "tensor", "achieved": round(attn_tflops, 2),
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(attn_tflops / peaks["bf16_tflops"], 4),
                     "peak_source": f"{peaks['source']} burst dense bf16 (cuBLAS)",
                     "kernel": ATTN_KERNEL,
                     "traffic": (measured_traffic(ATTN_KERNEL)
                                 if args.chunk == CHUNK else None)},
        "e2e": e2e,
        "gpu_launches": KERNELS_PER_STEP * args.steps,
        "sweep": st.sweep,
        "per_config": per_config,
        "velox_route": velox,
        "geometry_prior": geometry,
        "clocks": clock_info,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        base = oracle_sample_base(args.chunk, range(2))
        out["cpu_baseline"] = cpu_baseline(args.chunk, args.cpu_seconds, base=base)
        if not args.no_oracle_ops and args.chunk == CHUNK:
            out["cpu_baseline"]["per_op"] = oracle_per_config(base)
    if pg is not None:
        pg.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


def run_e2e(st, args, device, pg, flops):
    """The step with host inputs and outputs: every step copies its chunk's K,
    V, Q tokens and prior from pinned host memory and reads O and LSE back.
    As in a serving loop, the upload of step i+1 runs on a copy stream while
    step i computes (two device input sets, ordered by events); all copies of
    every step are inside the timed region."""
    k_h = st.k_tok.cpu().pin_memory()
    v_h = st.v_tok.cpu().pin_memory()
    q_h = st.q_tok.cpu().pin_memory()
    g_h = st.g.cpu().pin_memory() if st.g is not None else None
    o_h = torch.empty(st.o_tok.shape, dtype=st.o_tok.dtype).pin_memory()
    l_h = torch.empty(st.lse.shape, dtype=st.lse.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (k_h, v_h, q_h) + ((g_h,) if g_h is not None else ()))
    d2h = o_h.numel() * o_h.element_size() + l_h.numel() * l_h.element_size()
    steps = max(3, min(args.steps, 50))
    sets = [(st.k_tok, st.v_tok, st.q_tok, st.g),
            (torch.empty_like(st.k_tok), torch.empty_like(st.v_tok), torch.empty_like(st.q_tok),
             None if st.g is None else torch.empty_like(st.g))]
    copy_stream = torch.cuda.Stream(device)
    comp = torch.cuda.current_stream(device)
    uploaded = [torch.cuda.Event(), torch.cuda.Event()]
    consumed = [torch.cuda.Event(), torch.cuda.Event()]

    def upload(i):
        k, v, q, g = sets[i % 2]
        with torch.cuda.stream(copy_stream):
            copy_stream.wait_event(consumed[i % 2])
            k.copy_(k_h, non_blocking=True)
            v.copy_(v_h, non_blocking=True)
            q.copy_(q_h, non_blocking=True)
            if g is not None:
                g.copy_(g_h, non_blocking=True)
            uploaded[i % 2].record(copy_stream)

    def compute(i):
        k, v, q, g = sets[i % 2]
        comp.wait_event(uploaded[i % 2])
        st.k_tok, st.v_tok, st.q_tok, st.g = k, v, q, g
        st.step()
        consumed[i % 2].record(comp)
        o_h.copy_(st.o_tok, non_blocking=True)
        l_h.copy_(st.lse, non_blocking=True)

    for i in range(2):
        consumed[i].record(comp)
    upload(0)
    for i in range(3):          # warm-up
        upload(i + 1)
        compute(i)
    torch.cuda.synchronize(device)
    barrier(pg, device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    base = 3
    for i in range(base, base + steps):
        upload(i + 1)
        compute(i)
    comp.wait_stream(copy_stream)
    e1.record(comp)
    torch.cuda.synchronize(device)
    st.k_tok, st.v_tok, st.q_tok, st.g = sets[0]
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, pg, device)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    return {"value": round(flops * world / (ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 4), "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "steps": steps,
            "overlap": "upload of step i+1 on a copy stream during step i"}


# ---------------------------------------------------------------------------
# the oracle, timed on the host cores
# ---------------------------------------------------------------------------

def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def oracle_sample_step(inputs, n_items):
    """The oracle's whole path for one head of chunk 48: Gilbert scatter of the
    head's K/V/Q, pooling and fused top-K routing of its 49 query blocks, and
    attention of the first ``n_items`` query blocks.  Returns the selected
    attention FLOPs done."""
    import oracle
    T, H, W = inputs["grid"]
    D = inputs["D"]
    kb = oracle.tokens_to_blocks(inputs["k_tok"], T, H, W)
    vb = oracle.tokens_to_blocks(inputs["v_tok"], T, H, W)
    qb = oracle.tokens_to_blocks(inputs["q_tok"], T, H, W)
    n_hist = inputs["n_hist"]
    kc = np.concatenate([inputs["k_hist"], kb], axis=2)
    vc = np.concatenate([inputs["v_hist"], vb], axis=2)
    valid = inputs["valid"]
    nb = kb.shape[2]
    q_blk = qb.reshape(1, 1, nb * BLK, D)
    idx, _ = oracle.route(q_blk, kc, valid, n_hist, n_hist, nb, inputs["g"], 2.0, 0.2,
                          1.0 / math.sqrt(D), inputs["top_k"])
    flops = 0.0
    for j in range(n_items):
        sel = idx[0][0][j]
        oracle.attn_block(q_blk, kc, vc, valid, int(valid[n_hist + j]), 0, 0, j, sel,
                          1.0 / math.sqrt(D))
        flops += len(sel) * 4.0 * BLK * BLK * D
    return flops


def oracle_sample_base(chunk: int, heads) -> dict:
    """Inputs of the oracle's timed sample for ``heads`` of chunk ``chunk``,
    made on the host from the seeded generators alone: every chunk's tokens
    from ``synth`` (drawn by the CPU generator, so the values differ from
    the device-drawn ones while shapes and distributions are the same), the
    prior from ``synth.prior`` and the valid-row counts from the oracle.
    Nothing here comes from the CUDA path."""
    import oracle
    w = synth.CONFIGS[CONFIG_KEY]
    T, H, W = w.grid
    nbc = w.blocks_per_chunk
    hs = list(heads)
    hist = []
    for c in range(1, chunk):
        t = synth.chunk_tokens(w, c, device="cpu", want=("k", "v"))
        hist.append((t["k"][:, :, hs].clone(), t["v"][:, :, hs].clone()))
    cur = synth.chunk_tokens(w, chunk, device="cpu")
    n_hist = nbc * (chunk - 1)
    valid = np.tile(np.asarray(oracle.block_valid_for(T, H, W), dtype=np.int64), chunk)
    return {"w": w, "hist": hist, "n_hist": n_hist, "valid": valid,
            "cur": {n: cur[n][:, :, hs].clone() for n in ("q", "k", "v")},
            "g": synth.prior(w, chunk, nbc, n_hist) if n_hist > 0 else None}


def oracle_inputs(base: dict, i: int) -> dict:
    """fp64 inputs of the i-th sampled head: its history blocks, scattered by
    the oracle's own Gilbert order (before the timing), and its current-chunk
    tokens (scattered inside the timed step)."""
    import oracle
    w = base["w"]
    T, H, W = w.grid

    def hist_blocks(which):
        parts = [oracle.tokens_to_blocks(kv[which][:, :, i:i + 1].double().numpy(), T, H, W)
                 for kv in base["hist"]]
        if not parts:
            return np.zeros((w.B, 1, 0, BLK, w.D))
        return np.concatenate(parts, axis=2)
    return {
        "grid": w.grid, "D": w.D, "n_hist": base["n_hist"], "top_k": w.top_k[0],
        "k_tok": base["cur"]["k"][:, :, i:i + 1].double().numpy(),
        "v_tok": base["cur"]["v"][:, :, i:i + 1].double().numpy(),
        "q_tok": base["cur"]["q"][:, :, i:i + 1].double().numpy(),
        "k_hist": hist_blocks(0), "v_hist": hist_blocks(1),
        "valid": base["valid"], "g": base["g"],
    }


def cpu_baseline(chunk: int, seconds: float, n_heads: int = 2, base=None):
    """Oracle throughput on whole heads of the chunk (scatter, route of all
    query blocks, attention of all of them), cycling over ``n_heads`` heads
    until about ``seconds`` of timed work."""
    w = synth.CONFIGS[CONFIG_KEY]
    if base is None:
        base = oracle_sample_base(chunk, range(n_heads))
    inputs = [oracle_inputs(base, i) for i in range(n_heads)]
    flops, dt, steps = 0.0, 0.0, 0
    while dt < seconds:
        t0 = time.perf_counter()
        flops += oracle_sample_step(inputs[steps % n_heads], w.blocks_per_chunk)
        dt += time.perf_counter() - t0
        steps += 1
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": host_cores(),
            "kind": "oracle", "seconds": round(dt, 2),
            "sample": f"fp64 numpy oracle, {steps} whole heads of chunk {chunk} (heads "
                      f"0-{n_heads - 1} in turn, of {w.Hh}): Gilbert scatter of K/V/Q, route of "
                      f"all {w.blocks_per_chunk} query blocks, attention of all of them; "
                      f"inputs drawn on the host from the seeded generators"}


def _oracle_case(w, chunk: int, hist_kv, cur: dict) -> dict:
    """fp64 inputs of head (0, 0) of a config for the oracle's per-op timing:
    the history blocks (the oracle's own Gilbert scatter of the seeded
    history tokens, or the blocks written directly), the query chunk's raster
    tokens, the valid-row counts and the prior.  Made on the host from the
    seeded generators; nothing comes from the CUDA path."""
    import oracle
    T, H, W = w.grid
    nbc = w.blocks_per_chunk

    def head(x):
        return x[:1, :, :1].double().numpy()
    parts_k, parts_v = [], []
    valid = []
    if w.hist_direct:
        kd, vd = synth.direct_blocks(w, w.hist_direct, device="cpu")
        parts_k.append(kd[:1, :1].double().numpy())
        parts_v.append(vd[:1, :1].double().numpy())
        valid.append(np.full(w.hist_direct, BLK, dtype=np.int64))
    per = np.asarray(oracle.block_valid_for(T, H, W), dtype=np.int64)
    for k, v in hist_kv:
        parts_k.append(oracle.tokens_to_blocks(head(k), T, H, W))
        parts_v.append(oracle.tokens_to_blocks(head(v), T, H, W))
        valid.append(per)
    valid.append(per)
    n_hist = sum(x.shape[2] for x in parts_k)
    g = synth.prior(w, chunk, nbc, n_hist) if n_hist > 0 else None
    return {"w": w, "grid": (T, H, W), "n_hist": n_hist,
            "k_hist": np.concatenate(parts_k, axis=2) if parts_k else
            np.zeros((1, 1, 0, BLK, w.D)),
            "v_hist": np.concatenate(parts_v, axis=2) if parts_v else
            np.zeros((1, 1, 0, BLK, w.D)),
            "valid": np.concatenate(valid), "g": None if g is None else g[:1],
            "q_tok": head(cur["q"]), "k_tok": head(cur["k"]), "v_tok": head(cur["v"])}


def _timed(fn, min_s: float = 0.2, max_reps: int = 3):
    """Median wall time (s) of fn() over 1..max_reps runs (stops after min_s)."""
    ts = []
    while len(ts) < max_reps and (not ts or sum(ts) < min_s):
        t0 = time.perf_counter()
        fn()
        ts.append(time.perf_counter() - t0)
    return sorted(ts)[len(ts) // 2]


def oracle_op_times(case: dict, top_k: int, attn_items: int = 2) -> dict:
    """The oracle, as it stands, timed op by op on head (0, 0) of a config,
    each op scaled to a full call of the config by its unit count: the
    append by the (batch, head) pairs, the route likewise, the attention by
    the (batch, head, query block) items."""
    import oracle
    w = case["w"]
    T, H, W = case["grid"]
    nbc = w.blocks_per_chunk
    n_hist = case["n_hist"]
    sm = w.sm_scale
    t_app = _timed(lambda: (oracle.tokens_to_blocks(case["k_tok"], T, H, W),
                            oracle.tokens_to_blocks(case["v_tok"], T, H, W)))
    kb = oracle.tokens_to_blocks(case["k_tok"], T, H, W)
    vb = oracle.tokens_to_blocks(case["v_tok"], T, H, W)
    qb = oracle.tokens_to_blocks(case["q_tok"], T, H, W).reshape(1, 1, nbc * BLK, w.D)
    kc = np.concatenate([case["k_hist"], kb], axis=2)
    vc = np.concatenate([case["v_hist"], vb], axis=2)
    valid = case["valid"]
    res = {}

    def rt():
        res["idx"], _ = oracle.route(qb, kc, valid, n_hist, n_hist, nbc, case["g"], w.lam,
                                     w.g_ref, sm, top_k)
    t_route = _timed(rt)
    sel = res["idx"][0][0]
    m = min(attn_items, nbc)

    def at():
        for j in range(m):
            oracle.attn_block(qb, kc, vc, valid, int(valid[n_hist + j]), 0, 0, j, sel[j], sm)
    t_attn = _timed(at) / m
    pairs = w.B * w.Hh
    return {"append_ms": round(1e3 * t_app * pairs, 2),
            "route_ms": round(1e3 * t_route * pairs, 2),
            "attn_ms": round(1e3 * t_attn * pairs * nbc, 2),
            "sample": f"head (0, 0): append and route of the whole head, attention of "
                      f"{m} query block(s); scaled by {pairs} (batch, head) pairs and "
                      f"{pairs * nbc} attention items"}


def oracle_per_config(base48: dict) -> dict:
    """Per-op oracle timings for every config run and for the 48-chunk
    sweep at chunks 1, 12, 24 and 48 (the history of the sweep is shared
    with the whole-path CPU baseline's)."""
    out = {"cores": host_cores(), "kind": "oracle", "configs": [], "sweep_chunks": []}
    done = {}
    for key, top_k in CONFIG_RUNS:
        w = synth.CONFIGS[key]
        if key not in done:
            hist = [tuple(synth.chunk_tokens(w, c, device="cpu", want=("k", "v"))[n]
                          for n in ("k", "v")) for c in range(1, w.hist_chunks + 1)]
            qc = w.hist_chunks + 1 if w.hist_direct == 0 else 1
            done[key] = _oracle_case(w, qc, hist, synth.chunk_tokens(w, qc, device="cpu"))
        out["configs"].append({"config": key, "top_k": top_k,
                               **oracle_op_times(done[key], top_k)})
    w4 = synth.CONFIGS[CONFIG_KEY]
    for c in (1, 12, 24, 48):
        if c == 48:
            cur = {n: base48["cur"][n] for n in ("q", "k", "v")}
        else:
            t = synth.chunk_tokens(w4, c, device="cpu", want=("q",))
            cur = {"q": t["q"][:, :, :1], "k": base48["hist"][c - 1][0],
                   "v": base48["hist"][c - 1][1]}
        case = _oracle_case(w4, c, base48["hist"][:c - 1], cur)
        out["sweep_chunks"].append({"chunk": c, "top_k": w4.top_k[0],
                                    **oracle_op_times(case, w4.top_k[0])})
    return out


def run_reference(args, rank, world):
    """Reference arm: the oracle, as it stands, on the host cores."""
    if rank != 0:
        return
    inputs = oracle_inputs(oracle_sample_base(args.chunk, [0]), 0)
    n_items = 2
    for _ in range(max(args.warmup, 3)):
        oracle_sample_step(inputs, 1)
    times, flops = [], 0.0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        flops = oracle_sample_step(inputs, n_items)
        times.append(time.perf_counter() - t0)
    ms = 1e3 * sum(times) / len(times)
    value = flops / (ms * 1e-3) / 1e12
    sample = (f"fp64 numpy oracle per step: head 0 of chunk {args.chunk}, Gilbert scatter, "
              f"route of 49 query blocks, attention of {n_items} query blocks; inputs drawn "
              f"on the host from the seeded generators")
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
           "n_gpus": world, "steps": args.steps, "warmup": max(args.warmup, 3),
           "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
           "config": {"workload": "48-chunk sweep, chunk 48 (bounded oracle sample per step)",
                      "chunk": args.chunk},
           "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": host_cores(),
                            "kind": "oracle", "sample": sample},
           "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        run_reference(args, rank, world)
        return
    rank, world, local, pg = dist_setup(args.gpus)
    run_ours(args, rank, world, local, pg)


if __name__ == "__main__":
    main()
