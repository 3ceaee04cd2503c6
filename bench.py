"""Benchmark of the quantized paged KV cache on B200.

One step = one decode token through the attention cache of every layer of a
Qwen3-32B-shaped model at 16K context: for each of 64 layers, the new
token's K/V (8 kv heads x 128, bf16) is quantize-appended into that layer's
packed k4v2_g128 pool, then decode attention runs for 64 query heads over the
16384 cached tokens.  The 64 layers' pools (13.6 MB each, 872 MB together)
are separate buffers, so every step reads the whole cache from HBM (inputs
larger than L2, no flush needed).  A step is captured once in a CUDA graph and
replayed.

Printed (rank 0, one JSON line): decode tokens/s of the whole job; the decode
kernel's effective HBM GB/s on packed-cache bytes against the measured copy
bandwidth; quantize GB/s of a 16 x 16384-token prefill append; an end-to-end
figure with pinned host copies inside the timed region; and the CPU oracle's
throughput on a bounded sample.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kvq|reference]
                    [--profile qwen3-32b-16k|qwen3-32b-16k-window|batched|long|mixed|prefill-quantize]

--profile times the decode kernel alone on one workload (or, with
prefill-quantize, the bulk write path on 3 x 16384 fresh tokens) and prints
its per-launch time; it is the command the ncu summaries are taken with.

For N > 1 (torchrun), every rank runs an independent replica (the path has
no cross-GPU step); the timing is the max over ranks and the value sums all
ranks' tokens.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "decode attention tokens/s and effective HBM GB/s (% of roofline), quantize GB/s"
SEG = 1664
BYTES_PER_TOKEN_HEAD = 104


# DRAM bytes (read + write) of one decode launch on the Qwen3-32B layer
# workload, from `ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum`
# (cache control on: every replay starts cold, as every launch of the step
# does), with the SHA-256 of the kernel code it was taken on (decode_code_sha256:
# comments stripped).  Reported as roofline.traffic only while the code still
# has that hash.
DECODE_TRAFFIC = {"sha256": "c4f33186e28d0459040e0ea253d5f85cc3abae1990a281bb1dbc0e466415e57e",
                  "bytes": 13764352}


def decode_code_sha256():
    """SHA-256 of the decode kernel source with // comments and blank lines
    removed (a comment edit does not change the kernel)."""
    import hashlib
    import re
    path = os.path.join(ROOT, "bit_kv_cache_18_b200", "csrc", "kvq_decode.cu")
    with open(path) as f:
        lines = [re.sub(r"\s*//.*$", "", ln).rstrip() for ln in f]
    return hashlib.sha256("\n".join(ln for ln in lines if ln).encode()).hexdigest()


def decode_traffic():
    return DECODE_TRAFFIC["bytes"] if decode_code_sha256() == DECODE_TRAFFIC["sha256"] else None


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# --------------------------------------------------------------------------- ranks

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, backend):
    if world <= 1:
        return None
    import datetime
    import torch.distributed as dist
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def aggregate(dist, local_ms: float, local_units: float, device=None):
    """Max of the elapsed time and sum of the work over ranks."""
    if dist is None:
        return local_ms, local_units
    import torch
    t = torch.tensor([local_ms], dtype=torch.float64, device=device)
    u = torch.tensor([local_units], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t[0]), float(u[0])


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock and clock-event reasons sampled while a timed region runs.

    Reads NVML from a background thread every ~2 ms (read-only queries; the
    timed regions here last tens of milliseconds, too short for
    nvidia-smi's 200 ms loop), falling back to `nvidia-smi -lms 200` into a
    temporary file.  The samples are written as CSV to `log_path` when one is
    given (bench.py --clock-log)."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4), ("hw_power_brake_slowdown", 0x80))

    def __init__(self, index: int, uuid: str | None = None, period_s: float = 0.002, log_path: str | None = None):
        self.index = index
        self.uuid = uuid
        self.period = period_s
        self.rows = []  # (t, sm_mhz, max_mhz, power_w, reasons bitmask)
        self.proc = None
        self.thread = None
        self.nvml = None
        self.log_path = log_path
        self.path = None  # nvidia-smi fallback output (a temporary file)

    def _poll(self):
        nv, h = self.nvml, self.handle
        max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        while not self.stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
            except Exception:  # noqa: BLE001 - a failed read ends sampling, not the bench
                break
            self.rows.append((time.perf_counter(), sm, max_mhz, pw, rs))
            self.stop.wait(self.period)

    def __enter__(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            # by UUID: NVML enumerates every GPU of the machine, CUDA only the visible ones
            self.handle = (pynvml.nvmlDeviceGetHandleByUUID(self.uuid) if self.uuid
                           else pynvml.nvmlDeviceGetHandleByIndex(self.index))
            self.stop = threading.Event()
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            deadline = time.perf_counter() + 2.0
            while not self.rows and time.perf_counter() < deadline:
                time.sleep(0.001)
            return self
        except Exception:  # noqa: BLE001
            self.nvml = None
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(prefix="kvq_clocks_", suffix=".csv")
            self.f = os.fdopen(fd, "w")
            fields = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={fields}", "--format=csv,noheader,nounits",
                                          "-i", str(self.index), "-lms", "200"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
            self.nvml.nvmlShutdown()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()
            with open(self.path) as f:
                for line in f:
                    p = [x.strip() for x in line.split(",")]
                    if len(p) >= 4 and p[0].replace(".", "").isdigit():
                        rs = int(p[3], 16) if p[3].lower().startswith("0x") else 0
                        self.rows.append((0.0, float(p[0]), float(p[1]), float(p[2] or 0), rs))
            os.unlink(self.path)
        if self.log_path:
            try:
                with open(self.log_path, "w") as f:
                    f.write("t_s,sm_mhz,max_sm_mhz,power_w,reasons_hex\n")
                    for t, sm, mx, pw, rs in self.rows:
                        f.write(f"{t:.4f},{sm},{mx},{pw:.1f},{int(rs):#x}\n")
            except OSError:
                pass

    def summary(self):
        if not self.rows:
            return None
        sm = [r[1] for r in self.rows]
        mask = 0
        for r in self.rows:
            mask |= int(r[4])
        return {"sm_mhz": statistics.median(sm), "sm_min_mhz": min(sm), "sm_max_mhz": float(self.rows[0][2]),
                "reasons": [n for n, bit in self.REASONS if mask & bit], "samples": len(self.rows),
                "source": "nvml" if self.thread is not None else "nvidia-smi"}


def device_uuid(torch, dev):
    try:
        return "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:  # noqa: BLE001
        return None


# --------------------------------------------------------------------------- the step

class QwenStep:
    """64 layers of a Qwen3-32B-shaped attention cache at 16K context, batch 1."""

    layers = 64
    batch = 1
    hq = 64
    hkv = 8
    context = 16384
    win_sink = 4
    win_recent = 128

    def __init__(self, kvq, torch, dev, seed=0):
        self.kvq, self.torch, self.dev = kvq, torch, dev
        wl = synth.qwen3_32b_layer(seed, self.context)
        self.wl = wl
        self.nblocks = wl.num_blocks
        T = wl.total_tokens
        slots = wl.slots()
        # layer 0's cache from the seeded workload; the other layers get copies
        # of its bytes in their own buffers (identical work, distinct addresses)
        k = torch.from_numpy(wl.kv_rows(synth.TID_K, 0, T).view(np.int16)).to(dev).view(torch.bfloat16)
        v = torch.from_numpy(wl.kv_rows(synth.TID_V, 0, T).view(np.int16)).to(dev).view(torch.bfloat16)
        pool0 = kvq.new_pool(self.nblocks, self.hkv, device=dev)
        kvq.kvq_quantize_append(pool0, self.nblocks, self.hkv, k.reshape(T, -1), v.reshape(T, -1),
                                torch.from_numpy(slots).to(dev))
        # a bf16 window of the 4 sink and 128 most recent tokens, each layer its own
        idx = np.concatenate([np.arange(self.win_sink), np.arange(T - self.win_recent, T)]).astype(np.int64)
        ti = torch.from_numpy(idx).to(dev)
        win0 = kvq.new_window(1, self.hkv, self.win_sink, self.win_recent, device=dev)
        kvq.kvq_window_append(win0, self.win_sink, self.win_recent, k.reshape(T, -1)[ti].contiguous(),
                              v.reshape(T, -1)[ti].contiguous(), torch.zeros(len(idx), dtype=torch.int32, device=dev),
                              ti.to(torch.int32))
        torch.cuda.synchronize()
        del k, v
        self.wins = [win0] + [win0.clone() for _ in range(self.layers - 1)]
        self.pools = [pool0] + [pool0.clone() for _ in range(self.layers - 1)]
        self.bt = torch.from_numpy(wl.block_table).to(dev)
        self.lens = torch.from_numpy(wl.seq_lens).to(dev)
        # per-layer new token K/V and query (bf16), and outputs
        nk = synth.kv(seed, synth.TID_NEWK, 0, self.layers, self.hkv, 128, 3, 10.0, 30.0, synth.BF16)
        nv = synth.kv(seed, synth.TID_NEWV, 0, self.layers, self.hkv, 128, 3, 10.0, 30.0, synth.BF16)
        qq = synth.normal(seed, synth.TID_Q, self.layers * self.hq * 128, synth.BF16)
        self.h_in = torch.empty(self.layers * (2 * self.hkv + self.hq) * 128, dtype=torch.bfloat16).pin_memory()
        hv = self.h_in.view(torch.int16).numpy()
        n_kv = self.layers * self.hkv * 128
        hv[:n_kv] = nk.reshape(-1).view(np.int16)
        hv[n_kv:2 * n_kv] = nv.reshape(-1).view(np.int16)
        hv[2 * n_kv:] = qq.view(np.int16)
        self.d_in = self.h_in.to(dev)
        self.new_k = self.d_in[:n_kv].view(self.layers, 1, self.hkv * 128)
        self.new_v = self.d_in[n_kv:2 * n_kv].view(self.layers, 1, self.hkv * 128)
        self.q = self.d_in[2 * n_kv:].view(self.layers, self.batch, self.hq, 128)
        self.out = torch.empty((self.layers, self.batch, self.hq, 128), dtype=torch.bfloat16, device=dev)
        self.h_out = torch.empty(self.out.shape, dtype=torch.bfloat16).pin_memory()
        self.ws = kvq.new_workspace(self.nblocks, self.hkv, self.batch, self.hq, self.context, device=dev)
        self.copy_stream = torch.cuda.Stream(device=dev)
        self.wws = kvq.new_window_workspace(self.nblocks, self.hkv, self.batch, self.hq, self.context, device=dev)

    @property
    def packed_bytes_per_decode(self):
        return self.context * self.hkv * BYTES_PER_TOKEN_HEAD

    def launches_per_step(self):
        return self.layers

    def step(self, decode_only=False):
        """One token through all layers: per layer one fused launch that
        quantize-appends the new token's K/V at position 16383 and runs decode
        attention over the 16384 cached tokens (decode_only: the decode
        kernel alone, for its roofline)."""
        kvq = self.kvq
        for l in range(self.layers):
            if decode_only:
                kvq.kvq_decode_attention(self.pools[l], self.nblocks, self.hkv, self.q[l], self.bt, self.lens,
                                         self.context, self.out[l], self.ws)
            else:
                kvq.kvq_append_decode_attention(self.pools[l], self.nblocks, self.hkv, self.new_k[l], self.new_v[l],
                                                self.q[l], self.bt, self.lens, self.context, self.out[l], self.ws)

    def step_window(self):
        """The decode of every layer with its bf16 window of sink and recent
        tokens (one launch per layer; the window's rows stand in for the
        pool's at those positions)."""
        kvq = self.kvq
        for l in range(self.layers):
            kvq.kvq_decode_attention_window(self.pools[l], self.nblocks, self.hkv, self.wins[l], self.win_sink,
                                            self.win_recent, self.q[l], self.bt, self.lens, self.context, self.out[l],
                                            self.wws)

    def step_e2e(self, chunk=16):
        """The step with its host copies, in chunks of `chunk` layers on a
        copy stream: a chunk's inputs come in before its first layer runs and
        its outputs go back once its last layer is done, so the copies of the
        other chunks overlap the compute; every byte still crosses every
        step."""
        assert self.layers % chunk == 0
        torch, kvq = self.torch, self.kvq
        s = torch.cuda.current_stream()
        c = self.copy_stream
        n_kv = self.layers * self.hkv * 128
        nq = self.hq * 128
        h, d = self.h_in, self.d_in
        c.wait_stream(s)
        ins = []
        with torch.cuda.stream(c):
            for l0 in range(0, self.layers, chunk):
                l1 = l0 + chunk
                kv0, kv1 = l0 * self.hkv * 128, l1 * self.hkv * 128
                d[kv0:kv1].copy_(h[kv0:kv1], non_blocking=True)
                d[n_kv + kv0:n_kv + kv1].copy_(h[n_kv + kv0:n_kv + kv1], non_blocking=True)
                d[2 * n_kv + l0 * nq:2 * n_kv + l1 * nq].copy_(h[2 * n_kv + l0 * nq:2 * n_kv + l1 * nq],
                                                               non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(c)
                ins.append(ev)
        for l in range(self.layers):
            if l % chunk == 0:
                s.wait_event(ins[l // chunk])
            kvq.kvq_append_decode_attention(self.pools[l], self.nblocks, self.hkv, self.new_k[l], self.new_v[l],
                                            self.q[l], self.bt, self.lens, self.context, self.out[l], self.ws)
            if l % chunk == chunk - 1:
                done = torch.cuda.Event()
                done.record(s)
                c.wait_event(done)
                with torch.cuda.stream(c):
                    self.h_out[l + 1 - chunk:l + 1].copy_(self.out[l + 1 - chunk:l + 1], non_blocking=True)
        s.wait_stream(c)

    def tokens_per_step(self):
        return self.batch


def graph_of(torch, fn):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()  # warm (attribute caches, first-launch setup) outside capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def time_replays(torch, g, n, barrier=None, pre=None, post=None):
    """Device time (ms) of n replays of g, events on the replay stream."""
    if barrier:
        barrier()
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(n):
        if pre:
            pre()
        g.replay()
        if post:
            post()
    e1.record(s)
    torch.cuda.synchronize()
    if barrier:
        barrier()
    return e0.elapsed_time(e1)


def seg_bytes(preset):
    """Bytes of one (block, kv head) segment: 16 rows of K and V codes + 4 x 16 fp16."""
    return 16 * 128 * (preset[0] + preset[1]) // 8 + 128


def prefill_quantize_gbs(kvq, torch, dev, seed=0, seqs=16, tokens=16384, reps=10, preset=(4, 2)):
    """Quantize-append of 16 x 16384 fresh tokens, 8 kv heads, bf16."""
    hkv = 8
    T = seqs * tokens
    nblocks = T // 16
    # inputs: one seeded sequence's worth, repeated (the kernel's work does not
    # depend on the values); slots: a seeded permutation of the pool
    base = synth.kv(seed, synth.TID_K, 0, tokens, hkv, 128, 3, 10.0, 30.0, synth.BF16)
    kb = torch.from_numpy(base.view(np.int16)).to(dev).view(torch.bfloat16).reshape(tokens, -1)
    k = kb.repeat(seqs, 1)
    v = torch.roll(k, 1, 0).contiguous()
    perm = synth.permutation(seed, synth.TID_PERM, nblocks).astype(np.int64)
    slots = (perm[np.arange(T) // 16] * 16 + np.arange(T) % 16).astype(np.int32)
    sl = torch.from_numpy(slots).to(dev)
    pool = kvq.new_pool(nblocks, hkv, device=dev, preset=preset)
    kvq.kvq_quantize_append(pool, nblocks, hkv, k, v, sl, preset=preset)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        kvq.kvq_quantize_append(pool, nblocks, hkv, k, v, sl, preset=preset)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    nbytes = T * hkv * (2 * 128 * 2 + seg_bytes(preset) // 16) + T * 4
    status = kvq.kvq_last_device_status()
    del k, v, pool, kb
    return {"us": ms * 1e3, "gbs": nbytes / (ms * 1e-3) / 1e9, "bytes": nbytes, "status": status}


def seeded_pool(kvq, torch, dev, wl, preset=(4, 2)):
    """A pool for workload wl filled from its seeded stream: the first
    min(16384, total) tokens are quantized through the library and their
    segments repeated over the rest of the pool (the same value distribution,
    hence the same running-max behaviour, without generating gigabytes of
    K/V on the host)."""
    T0 = min(16384, wl.total_tokens)
    nb0 = (T0 + 15) // 16
    k = torch.from_numpy(wl.kv_rows(synth.TID_K, 0, T0).view(np.int16)).to(dev).view(torch.bfloat16)
    v = torch.from_numpy(wl.kv_rows(synth.TID_V, 0, T0).view(np.int16)).to(dev).view(torch.bfloat16)
    base = kvq.new_pool(nb0, wl.hkv, device=dev, preset=preset)
    kvq.kvq_quantize_append(base, nb0, wl.hkv, k.reshape(T0, -1), v.reshape(T0, -1),
                            torch.arange(T0, dtype=torch.int32, device=dev), preset=preset)
    del k, v
    pool = kvq.new_pool(wl.num_blocks, wl.hkv, device=dev, preset=preset)
    seg = pool.view(wl.num_blocks, -1)
    b0 = base.view(nb0, -1)
    for s0 in range(0, wl.num_blocks, nb0):
        n = min(nb0, wl.num_blocks - s0)
        seg[s0:s0 + n].copy_(b0[:n])
    del base
    return pool


def time_decode_workload(kvq, torch, dev, wl, preset=(4, 2), reps=10, fused=False):
    """Decode launches (or, fused=True, the one-step append + decode launch
    with each sequence's new token) on a seeded pool of workload wl; CUDA
    events on the launching stream around `reps` launches after 3 warm-ups.
    Every workload's pool is larger than L2 except where noted by the caller.
    Returns µs per launch and GB/s on packed-cache bytes."""
    pool = seeded_pool(kvq, torch, dev, wl, preset)
    q = torch.from_numpy(wl.query().view(np.int16)).to(dev).view(torch.bfloat16)
    bt = torch.from_numpy(wl.block_table).to(dev)
    lens = torch.from_numpy(wl.seq_lens).to(dev)
    msl = int(wl.seq_lens.max())
    out = torch.empty((wl.batch, wl.hq, 128), dtype=torch.bfloat16, device=dev)
    ws = kvq.new_workspace(wl.num_blocks, wl.hkv, wl.batch, wl.hq, msl, device=dev, preset=preset)
    if fused:
        kn = torch.from_numpy(wl.kv_rows(synth.TID_NEWK, 0, wl.batch).view(np.int16)).to(dev).view(torch.bfloat16)
        vn = torch.from_numpy(wl.kv_rows(synth.TID_NEWV, 0, wl.batch).view(np.int16)).to(dev).view(torch.bfloat16)
        kn, vn = kn.reshape(wl.batch, -1), vn.reshape(wl.batch, -1)

    def launch():
        if fused:
            kvq.kvq_append_decode_attention(pool, wl.num_blocks, wl.hkv, kn, vn, q, bt, lens, msl, out, ws,
                                            preset=preset)
        else:
            kvq.kvq_decode_attention(pool, wl.num_blocks, wl.hkv, q, bt, lens, msl, out, ws, preset=preset)

    for _ in range(3):
        launch()
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(reps):
        launch()
    e1.record(s)
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / reps
    nbytes = int(wl.seq_lens.astype(np.int64).sum()) * wl.hkv * seg_bytes(preset) // 16
    status = kvq.kvq_last_device_status()
    del pool, ws
    peak = measured_peaks()[0]
    gbs = nbytes / (us * 1e-6) / 1e9
    return {"us": us, "bytes": nbytes, "gbs": gbs, "frac": gbs / peak, "frac_of_8000": gbs / 8000.0,
            "query_tokens_per_s": wl.batch / (us * 1e-6),
            "context_tokens_per_s": float(wl.seq_lens.astype(np.int64).sum()) / (us * 1e-6), "status": status}


def preset_decode_gbs(kvq, torch, dev, preset, batch=32, context=8192, reps=10):
    """Decode of batch x context tokens (64/8 heads) on a seeded pool of the
    preset (larger than L2); µs per launch and GB/s on packed bytes."""
    return time_decode_workload(kvq, torch, dev, synth.mixed_decode(0, batch=batch, context=context), preset, reps)


def workload_suite(kvq, torch, dev, reps=10):
    """The other decode workloads, each on its own seeded pool (all larger
    than L2): batched ragged 32 x U[4096, 16384]; Llama-3.1-70B-shaped 8 x
    131072; the mixed step (64 x 8192, the new token of every sequence
    appended and read in one fused launch), plus its decode alone."""
    res = {}
    for key, wl, fused in (("batched_32x_u4096_16384", synth.batched(0), False),
                           ("long_8x131072", synth.long_context(0), False),
                           ("mixed_step_64x8192", synth.mixed_decode(0), True),
                           ("mixed_decode_64x8192", synth.mixed_decode(0), False)):
        r = time_decode_workload(kvq, torch, dev, wl, reps=reps, fused=fused)
        r["launch"] = ("fused 1-token append + decode" if fused else "decode")
        res[key] = r
    return res


def dense_error_sample(kvq, torch, dev, seed=0, kv_head=0):
    """Max abs error of the GPU read path against unquantized attention on the
    raw bf16 K/V (the oracle's dense attention in double), for the query heads
    of one kv head of the Qwen3-32B-shaped layer: the error quantisation adds.
    Reported, not gated (the pages give no number for it)."""
    import oracle
    wl = synth.qwen3_32b_layer(seed)
    T = wl.total_tokens
    k = wl.kv_rows(synth.TID_K, 0, T)
    v = wl.kv_rows(synth.TID_V, 0, T)
    kd = torch.from_numpy(k.view(np.int16)).to(dev).view(torch.bfloat16).reshape(T, -1)
    vd = torch.from_numpy(v.view(np.int16)).to(dev).view(torch.bfloat16).reshape(T, -1)
    pool = kvq.new_pool(wl.num_blocks, wl.hkv, device=dev)
    kvq.kvq_quantize_append(pool, wl.num_blocks, wl.hkv, kd, vd, torch.from_numpy(wl.slots()).to(dev))
    q = wl.query()
    out = torch.empty((wl.batch, wl.hq, 128), dtype=torch.float32, device=dev)
    ws = kvq.new_workspace(wl.num_blocks, wl.hkv, wl.batch, wl.hq, T, device=dev)
    kvq.kvq_decode_attention(pool, wl.num_blocks, wl.hkv, torch.from_numpy(q.view(np.int16)).to(dev)
                             .view(torch.bfloat16), torch.from_numpy(wl.block_table).to(dev),
                             torch.from_numpy(wl.seq_lens).to(dev), T, out, ws)
    got = out.cpu().numpy().astype(np.float64)
    G = wl.hq // wl.hkv
    # tokens in the order of the sequence (the slots follow it)
    err, ref_max = 0.0, 0.0
    for j in range(kv_head * G, (kv_head + 1) * G):
        ref = oracle.attention_dense(k, v, wl.dtype, q[0, j], wl.dtype, wl.hq, j)
        err = max(err, float(np.max(np.abs(got[0, j] - ref))))
        ref_max = max(ref_max, float(np.max(np.abs(ref))))
    del pool, ws, kd, vd
    return {"max_abs_err": err, "max_abs_output": ref_max, "query_heads": G, "tokens": T,
            "against": "unquantized attention in double on the raw bf16 K/V (oracle)", "gated": False}


# --------------------------------------------------------------------------- CPU oracle

class OracleSample:
    """The oracle, as it stands, on a bounded sample of one step: the 1-token
    write plus the decode of one kv head (8 query heads over 16384 tokens) of
    one layer.  A step is 64 layers x 8 kv heads of such units.  The cache
    state it reads is written by the oracle itself, once, untimed.

    unit() runs one such unit on one thread.  unit_mt(n) runs n units at once
    on n threads (the oracle's own std::thread split over (sequence, kv head)
    pairs: the sample's one kv head is read by n batch rows), which is how
    the oracle uses all the host's cores."""

    desc = ("oracle 1-token write + decode of 1 kv head (8 query heads x 16384 tokens) of 1 layer, single "
            "thread; one step = 64 layers x 8 kv heads of these units")

    def __init__(self, seed=0):
        import oracle
        self.oracle = oracle
        wl = synth.qwen3_32b_layer(seed, QwenStep.context)
        T = wl.total_tokens
        self.wl = wl
        self.k = np.ascontiguousarray(wl.kv_rows(synth.TID_K, 0, T)[:, :1])
        self.v = np.ascontiguousarray(wl.kv_rows(synth.TID_V, 0, T)[:, :1])
        self.g = oracle.geom(num_blocks=wl.num_blocks, num_kv_heads=1)
        self.pool = oracle.new_pool(self.g)
        self.slots = wl.slots()
        assert oracle.quantize_append(self.g, self.pool, self.k, self.v, wl.dtype, self.slots) == 0
        self.q = np.ascontiguousarray(wl.query()[:, :8])

    def unit(self) -> float:
        o, wl = self.oracle, self.wl
        t0 = time.perf_counter()
        assert o.quantize_append(self.g, self.pool, self.k[-1:], self.v[-1:], wl.dtype, self.slots[-1:]) == 0
        o.decode_attention(self.g, self.pool, self.q, wl.dtype, wl.block_table, wl.seq_lens, nthreads=1)
        return time.perf_counter() - t0

    def unit_mt(self, n: int) -> float:
        """Seconds per unit when n units run at once on n threads."""
        o, wl = self.oracle, self.wl
        q = np.ascontiguousarray(np.repeat(self.q, n, axis=0))
        bt = np.ascontiguousarray(np.repeat(wl.block_table, n, axis=0))
        lens = np.ascontiguousarray(np.repeat(wl.seq_lens, n))
        t0 = time.perf_counter()
        assert o.quantize_append(self.g, self.pool, self.k[-1:], self.v[-1:], wl.dtype, self.slots[-1:]) == 0
        o.decode_attention(self.g, self.pool, q, wl.dtype, bt, lens, nthreads=n)
        return (time.perf_counter() - t0) / n


def host_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# --------------------------------------------------------------------------- profile mode

PROFILE_WORKLOADS = {
    "qwen3-32b-16k": lambda: synth.qwen3_32b_layer(0),
    "qwen3-32b-16k-window": lambda: synth.qwen3_32b_layer(0),
    "batched": lambda: synth.batched(0),
    "long": lambda: synth.long_context(0),
    "mixed": lambda: synth.mixed_decode(0),
}


def profile_decode(args):
    """Decode launches alone on one workload, for ncu captures and sweeps.

    The pool is filled from the seeded workload: the first min(16384, total)
    tokens are quantized through the library and their segments repeated over
    the rest of the pool (same value distribution, no host-side generation of
    gigabytes).  Prints one JSON line with the per-launch device time."""
    import torch
    import bit_kv_cache_18_b200 as kvq
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    wl = PROFILE_WORKLOADS[args.profile]()
    pool = seeded_pool(kvq, torch, dev, wl)
    q = torch.from_numpy(wl.query().view(np.int16)).to(dev).view(torch.bfloat16)
    bt = torch.from_numpy(wl.block_table).to(dev)
    lens = torch.from_numpy(wl.seq_lens).to(dev)
    msl = int(wl.seq_lens.max())
    out = torch.empty((wl.batch, wl.hq, 128), dtype=torch.bfloat16, device=dev)
    ws = kvq.new_workspace(wl.num_blocks, wl.hkv, wl.batch, wl.hq, msl, device=dev)

    def launch():
        kvq.kvq_decode_attention(pool, wl.num_blocks, wl.hkv, q, bt, lens, msl, out, ws)

    if args.profile.endswith("-window"):
        # the same layer with a bf16 window of 4 sink and 128 recent tokens,
        # from the workload's own rows (one sequence: positions = rows)
        sink, recent = QwenStep.win_sink, QwenStep.win_recent
        T = wl.total_tokens
        idx = np.concatenate([np.arange(sink), np.arange(T - recent, T)])
        kw = torch.from_numpy(wl.kv_rows(synth.TID_K, 0, T)[idx].view(np.int16)).to(dev).view(torch.bfloat16)
        vw = torch.from_numpy(wl.kv_rows(synth.TID_V, 0, T)[idx].view(np.int16)).to(dev).view(torch.bfloat16)
        win = kvq.new_window(1, wl.hkv, sink, recent, device=dev)
        kvq.kvq_window_append(win, sink, recent, kw.reshape(len(idx), -1), vw.reshape(len(idx), -1),
                              torch.zeros(len(idx), dtype=torch.int32, device=dev),
                              torch.from_numpy(idx.astype(np.int32)).to(dev))
        wws = kvq.new_window_workspace(wl.num_blocks, wl.hkv, wl.batch, wl.hq, msl, device=dev)

        def launch():  # noqa: F811
            kvq.kvq_decode_attention_window(pool, wl.num_blocks, wl.hkv, win, sink, recent, q, bt, lens, msl, out,
                                            wws)

    for _ in range(args.warmup):
        launch()
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(args.steps):
        launch()
    e1.record(s)
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / args.steps
    nbytes = wl.total_tokens * wl.hkv * BYTES_PER_TOKEN_HEAD
    peak, kind = measured_peaks()
    gbs = nbytes / (us * 1e-6) / 1e9
    print(json.dumps({"profile": args.profile, "launches": args.steps, "us_per_launch": us,
                      "bytes_per_launch": nbytes, "gbs": gbs, "frac": gbs / peak, "peak_kind": kind,
                      "device_status": kvq.kvq_last_device_status()}))
    return 0


# --------------------------------------------------------------------------- main

def run_reference(args, world, rank):
    """The reference arm: the CPU oracle timed on the machine's host cores."""
    if rank != 0:
        return 0
    units_per_step = QwenStep.layers * QwenStep.hkv
    sample = OracleSample()
    n = host_threads()
    for _ in range(args.warmup):
        sample.unit_mt(n)
    samples = [sample.unit_mt(n) for _ in range(args.steps)]
    per_unit = sum(samples) / len(samples)
    desc = (f"oracle 1-token write + decode of 1 kv head (8 query heads x 16384 tokens) of 1 layer per unit, "
            f"{n} units at once on {n} threads; one step = 64 layers x 8 kv heads of these units; each timed "
            f"step runs one such batch of units, {args.steps} steps")
    step_s = per_unit * units_per_step
    value = QwenStep.batch / step_s
    single = 1.0 / (sample.unit() * units_per_step)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "qwen3-32b-16k-64layers", "batch": 1, "num_q_heads": 64, "num_kv_heads": 8,
                       "head_dim": 128, "context": 16384, "layers": 64, "block_size": 16},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": n, "kind": "oracle",
                             "sample": desc},
            "cpu_baseline_single_thread": {"value": single, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                           "sample": sample.desc + "; one unit"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-suite", action="store_true",
                    help="skip the other workloads (batched, long, mixed step), the presets and the error sample")
    ap.add_argument("--clock-log", default=None, help="write the clock samples of the timed region here (CSV)")
    ap.add_argument("--profile", choices=sorted(PROFILE_WORKLOADS) + ["prefill-quantize"], default=None,
                    help="time decode launches alone on one workload, or the bulk quantize-append "
                         "(1 GPU; for ncu captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.profile == "prefill-quantize":
        import torch
        import bit_kv_cache_18_b200 as kvq
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        r = prefill_quantize_gbs(kvq, torch, dev, seqs=3, reps=args.steps)
        peak, kind = measured_peaks()
        print(json.dumps({"profile": args.profile, "launches": args.steps, "us_per_launch": r["us"],
                          "bytes_per_launch": r["bytes"], "gbs": r["gbs"], "frac": r["gbs"] / peak,
                          "peak_kind": kind, "device_status": r["status"]}))
        return 0
    if args.profile:
        return profile_decode(args)
    world, rank, local = dist_env()
    if args.impl == "reference":
        return run_reference(args, world, rank)

    import torch
    import bit_kv_cache_18_b200 as kvq
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    dist = init_dist(world, "nccl")
    barrier = (lambda: dist.barrier(device_ids=[local])) if dist else None

    stepper = QwenStep(kvq, torch, dev)
    g_step = graph_of(torch, stepper.step)
    g_dec = graph_of(torch, lambda: stepper.step(decode_only=True))
    for _ in range(args.warmup):
        g_step.replay()
    torch.cuda.synchronize()
    if kvq.kvq_last_device_status() != 0:
        raise RuntimeError("device status set during warm-up")

    # timed region: K steps
    with ClockSampler(local, device_uuid(torch, dev), log_path=args.clock_log) as clocks:
        ms = time_replays(torch, g_step, args.steps, barrier)
    ms_max, tokens = aggregate(dist, ms, args.steps * stepper.tokens_per_step(), dev)
    value = tokens / (ms_max * 1e-3)
    ms_per_step = ms_max / args.steps

    # decode kernel alone (roofline): the same 64 launches without the appends
    for _ in range(3):
        g_dec.replay()
    dec_reps = max(args.steps, 10)
    dms = time_replays(torch, g_dec, dec_reps) / (dec_reps * stepper.layers)
    achieved = stepper.packed_bytes_per_decode / (dms * 1e-3) / 1e9
    peak, peak_kind = measured_peaks()
    # the same decode with a bf16 window of sink and recent tokens
    g_win = graph_of(torch, stepper.step_window)
    for _ in range(3):
        g_win.replay()
    wms = time_replays(torch, g_win, dec_reps) / (dec_reps * stepper.layers)

    # end to end: pinned host inputs in, outputs back, every step (a step's
    # copies go in chunks of 16 layers beside its compute)
    g_e2e = graph_of(torch, stepper.step_e2e)
    for _ in range(3):
        g_e2e.replay()
    e2e_ms = time_replays(torch, g_e2e, args.steps, barrier)
    e2e_ms_max, e2e_tokens = aggregate(dist, e2e_ms, args.steps * stepper.tokens_per_step(), dev)

    quant = prefill_quantize_gbs(kvq, torch, dev)
    presets, suite, dense = {}, None, None
    if not args.no_suite:
        # the other configurations, each on a seeded pool larger than L2
        suite = workload_suite(kvq, torch, dev)
        # every preset on the same shapes: decode of 32 x 8192 tokens on a
        # seeded pool and the prefill append of 4 x 16384 tokens (the default
        # preset included, for comparison)
        for pr in kvq.PRESETS:
            dq = preset_decode_gbs(kvq, torch, dev, pr)
            pq = prefill_quantize_gbs(kvq, torch, dev, seqs=4, reps=5, preset=pr)
            presets[f"kvarn_k{pr[0]}v{pr[1]}_g128"] = {
                "segment_bytes": seg_bytes(pr),
                "decode_32x8192": {"us": dq["us"], "gbs": dq["gbs"], "frac": dq["frac"]},
                "quantize_4x16384": {"us": pq["us"], "gbs": pq["gbs"], "frac": pq["gbs"] / measured_peaks()[0]},
                "device_status": dq["status"] or pq["status"]}
        if rank == 0:
            dense = dense_error_sample(kvq, torch, dev)
    status = kvq.kvq_last_device_status()

    cpu = cpu_mt = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sample = OracleSample()
        per_unit = sum(sample.unit() for _ in range(3)) / 3
        cpu_value = 1.0 / (per_unit * stepper.layers * stepper.hkv)
        cpu = {"value": cpu_value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
               "sample": sample.desc + "; mean of 3 units"}
        n = host_threads()
        per_unit_mt = sample.unit_mt(n)
        cpu_mt = {"value": 1.0 / (per_unit_mt * stepper.layers * stepper.hkv), "unit": "tokens/s", "cores": n,
                  "kind": "oracle",
                  "sample": f"{n} such units at once on {n} threads (the oracle's std::thread split), one run"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": "qwen3-32b-16k-64layers", "batch": 1, "num_q_heads": 64, "num_kv_heads": 8,
                       "head_dim": 128, "context": 16384, "layers": 64, "block_size": 16,
                       "cache": "kvarn_k4v2_g128", "step": "per layer: one fused launch (1-token quantize-append + decode attention)",
                       "q_dtype": "bf16", "kv_in_dtype": "bf16", "out_dtype": "bf16",
                       "l2": "inputs larger than L2: 64 distinct 13.6 MB pools (872 MB) per step",
                       "parallelism": f"replicas x{world}"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": decode_traffic(),
                         "kernel": "decode", "peak_kind": peak_kind,
                         "us_per_launch": dms * 1e3, "bytes_per_launch": stepper.packed_bytes_per_decode,
                         "frac_of_8000": achieved / 8000.0},
            "decode": {"us_per_layer": dms * 1e3, "effective_gbs": achieved,
                       "layer_tokens_per_s": stepper.batch / (dms * 1e-3),
                       "context_tokens_per_s": stepper.context * stepper.batch / (dms * 1e-3)},
            "window": {"workload": "the decode graph with a bf16 window of 4 sink and 128 recent tokens per layer",
                       "sink": stepper.win_sink, "recent": stepper.win_recent, "us_per_layer": wms * 1e3,
                       "decode_us_per_layer": dms * 1e3},
            "quantize": {"workload": "prefill append 16 x 16384 tokens, 8 kv heads, bf16", "us": quant["us"],
                         "gbs": quant["gbs"], "bytes": quant["bytes"], "frac": quant["gbs"] / peak},
            "presets": presets,
            "workloads": suite,
            "error_vs_unquantized": dense,
            "e2e": {"value": e2e_tokens / (e2e_ms_max * 1e-3), "unit": "tokens/s",
                    "h2d_bytes_per_step": stepper.h_in.numel() * 2, "d2h_bytes_per_step": stepper.h_out.numel() * 2},
            "gpu_launches": stepper.launches_per_step() * args.steps,
            "clocks": clocks.summary(),
            "device_status": status,
        }
        if cpu:
            line["cpu_baseline"] = cpu
        if cpu_mt:
            line["cpu_baseline_mt"] = cpu_mt
        print(json.dumps(line))
    if dist:
        del g_step, g_dec, g_win, g_e2e
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
