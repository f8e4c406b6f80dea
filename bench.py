#!/usr/bin/env python
"""Benchmark of the rotated INT2 KV-cache hot path on B200.

One step = rotate-quantize-append of the step's new token(s) + decode
attention of one query per head over the packed cache (the whole hot path).
The default workload is the largest single-GPU one, "ragged": a serving
batch of B=64 sequences with context lengths drawn uniformly from [1024,
65536] (seeded; 6.5 GB of packed cache read per step), 32 heads (MHA),
head_dim 128, dense per-head rotations, INT2 group 32 with fp16 scale/zero;
each step appends one token per sequence, then decodes one query per head.
Beside it: the single-layer llama7b step (B=1, 32 heads, context 32768),
the bulk appends (the ragged workload's 4 x 32768-token prefill among
them), the decode of every workload, the extensions, and the CPU oracle on a
bounded sample.  Inputs are seeded synthetic tensors (workloads.py).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...      # the CPU oracle as reference arm
    torchrun --nproc-per-node N bench.py --gpus N ...

Timing: exactly K steps run back to back on the launching stream between
one pair of CUDA events, with a barrier + synchronize on both sides; the
max over ranks is reported.  The steps are replayed from CUDA graphs (whole
rounds over the layers plus one graph of the remainder, with their
programmatic dependent launches), as a serving loop would run them, so the
host's launch cost stays out of the device time; `e2e` still drives every
step through the public API.  L2 (126 MB) must not serve the cache across
steps: a cache larger than 3x L2 (ragged: 12.9 GB allocated) is read
afresh by every step; a smaller one is replicated into independent layers
(distinct memory, same contents, like the layers of a model) that the steps
cycle through, so every step reads a cache that at least 3x L2 of other
cache traffic has passed through L2 since its last use.  Each step appends
at the same position (its own row of pre-append lengths), so the context is
the same for every step.  A cache too small for 64 layers to cover that
falls back to flushing L2 between steps (256 MB written, then 256 MB read,
so L2 holds clean lines) with each step bracketed by its own events.  The
isolated-step latency (flush, then one step between its own events) is
reported beside the throughput.  With N GPUs every rank serves its own
independent batch (weak scaling, no collective on the data path).

Prints one JSON line (rank 0).
"""
import argparse
import datetime
import hashlib
import json
import os
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "INT2-KV decode attention tokens/s and packed-KV GB/s (% of HBM peak), 1 B200"
KERNELS_PER_STEP = 4      # append (with the length update), query preparation, decode split, merge
FLUSH_BYTES = 256 << 20
L2_BYTES = 126 << 20      # B200 L2
MAX_LAYERS = 64


class L2Flush:
    """Evicts the cache's data from L2: write one buffer larger than L2,
    then read another, so L2 ends up holding clean lines."""

    def __init__(self, device):
        self.w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
        self.r = torch.ones(FLUSH_BYTES // 4, dtype=torch.int32, device=device)

    def __call__(self, k):
        self.w.fill_(k & 0xff)
        self.r.sum()


# --- distributed plumbing (also exercised by tests/test_bench_dist.py on CPU) ----------------

def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), \
        int(os.environ.get("LOCAL_RANK", 0))


def init_dist(backend, world):
    if world <= 1:
        return False
    import torch.distributed as dist
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return True


def barrier(enabled, device=None):
    if enabled:
        import torch.distributed as dist
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(x, enabled, device):
    """Max of a float over all ranks (identity when not distributed)."""
    if not enabled:
        return float(x)
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_workload(w, rank):
    """Each rank serves its own batch: same shapes, its own seed."""
    import dataclasses
    return dataclasses.replace(w, seed=w.seed + 7919 * rank)


# --- clocks -------------------------------------------------------------------------------------

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x20: "sync_boost", 0x40: "sw_thermal_slowdown",
               0x80: "hw_thermal_slowdown", 0x100: "hw_power_brake_slowdown",
               0x200: "display_clock_setting"}

    def __init__(self, index, period=0.002):
        self.samples, self.reasons, self.ok = [], set(), False
        self.period, self.stop_flag = period, threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report that instead of numbers
            self.err = str(e)

    def _run(self):
        nv = self.nv
        get_r = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self.stop_flag.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = get_r(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit and bit != 0x1:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self.stop_flag.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.err}
        return {"sm_mhz": float(np.median(self.samples)) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# --- helpers ------------------------------------------------------------------------------------

def measured_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    except Exception:
        return 6650.0, "fallback (6.65 TB/s, earlier measurement on this pool)"


def kernel_source_sha():
    h = hashlib.sha256()
    for f in ("kvq_decode.cu", "kvq_internal.cuh"):
        with open(os.path.join(ROOT, "rotated_int2_kv_head_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload, kv_bytes=None):
    """dram bytes per launch of the split kernel from the committed ncu
    summary, if it was taken on the current kernel source; else None.  A
    summary taken on a smaller case of the workload (its
    algorithmic_bytes_per_launch below kv_bytes) is scaled to a full launch
    by the ratio of algorithmic bytes (the units processed)."""
    p = os.path.join(ROOT, "profiles", "decode_split_%s.txt" % workload)
    if not os.path.exists(p):
        return None
    vals = {}
    for line in open(p):
        if ":" in line:
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip().split()[0] if v.strip() else ""
    if vals.get("source_sha256") != kernel_source_sha():
        return None
    try:
        dram = float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None
    try:
        alg = float(vals["algorithmic_bytes_per_launch"])
    except (KeyError, ValueError):
        alg = None
    if kv_bytes is not None and alg:
        dram *= kv_bytes / alg
    return dram


def packed_kv_bytes(w, lens):
    """Algorithmic cache bytes one decode reads: 96 per token-head (codes 64,
    scale/zero 32), 512 per fp16 sink token-head."""
    tot = 0
    for L in lens:
        s = min(w.sink, int(L))
        tot += w.Hkv * ((int(L) - s) * 96 + s * 512)
    return tot


# --- the CUDA arm ---------------------------------------------------------------------------------

def layers_for(cache_bytes):
    """How many independent layers to cycle so that, with no flush, each step
    reads a cache that the steps since its last use have pushed out of L2
    (at least 3x L2 of other cache traffic in between); 0 = too small for
    that, flush L2 between steps instead."""
    if cache_bytes >= 3 * L2_BYTES:
        return 1
    n = -(-3 * L2_BYTES // cache_bytes) + 1
    return n if n <= MAX_LAYERS else 0


def host_ahead(seconds):
    """Hold the current stream for about `seconds` (torch's spin kernel,
    counted in SM cycles at the maximum clock) so that the host can queue
    the work that follows before the device reaches it."""
    torch.cuda._sleep(int(seconds * 2.0e9))


class Step:
    """One pass of the hot path: append the step's new tokens to one layer's
    cache, then decode over it.  With n_layers > 1 the layers are
    independent copies (cache, rotations: same contents, distinct memory)
    used round robin, like the layers of a model; the new K/V rows and the
    queries are shared.  Sequence lengths come from a caller-provided row
    holding the pre-append lengths, so every step runs at the same context
    without a reset kernel."""

    def __init__(self, w, device, n_layers=1):
        import rotated_int2_kv_head_b200 as kvq
        self.kvq, self.w, self.dev = kvq, w, device
        lens = w.seq_lens()
        self.L = int(lens.max())
        self.T = w.append_T
        self.cap = ((self.L + 15) // 16) * 16
        Rk, Rv, perm = W.rotations(w)
        self.rot_np = (Rk, Rv, perm)
        Rk = torch.from_numpy(Rk).to(device) if Rk is not None else None
        Rv = torch.from_numpy(Rv).to(device) if Rv is not None else None
        perm = torch.from_numpy(perm).to(device) if perm is not None else None
        cache = kvq.KVCache(w.B, w.Hkv, self.cap, w.sink, device=device)
        self.len_base = torch.from_numpy(lens.astype(np.int32)).to(device) - self.T
        # prefill [0, L - T) on the GPU, in chunks, all sequences together
        pre = self.L - self.T
        fill = torch.zeros(w.B, dtype=torch.int32, device=device)
        for t0 in range(0, pre, 2048):
            t1 = min(pre, t0 + 2048)
            K, V = W.kv_batch(w, t0, t1, device)
            kvq.kvq_rotate_quantize_append(K, V, w.mode, Rk, Rv, perm, cache, fill)
        torch.cuda.synchronize(device)
        if kvq.kvq_get_status(cache) != 0:
            raise RuntimeError("cache fill flagged device status %d" % kvq.kvq_get_status(cache))
        self.layers = [(cache, Rk, Rv, perm)]
        for _ in range(1, n_layers):
            c2 = kvq.KVCache(w.B, w.Hkv, self.cap, w.sink, device=device)
            c2.blocks.copy_(cache.blocks)
            if cache.k_sink is not None:
                c2.k_sink.copy_(cache.k_sink)
                c2.v_sink.copy_(cache.v_sink)
            self.layers.append((c2, *(None if x is None else x.clone() for x in (Rk, Rv, perm))))
        # the step's inputs (new K and V rows, queries) share one device
        # buffer, so the end-to-end run moves them with a single copy
        Kn, Vn = W.kv_batch(w, pre, self.L, device)
        Qn = W.queries(w, device)
        nk, nq = Kn.numel(), Qn.numel()
        self.inbuf = torch.empty(2 * nk + nq, dtype=torch.float16, device=device)
        self.Knew = self.inbuf[:nk].view(Kn.shape)
        self.Vnew = self.inbuf[nk:2 * nk].view(Vn.shape)
        self.Q = self.inbuf[2 * nk:].view(Qn.shape)
        self.Knew.copy_(Kn)
        self.Vnew.copy_(Vn)
        self.Q.copy_(Qn)
        self.out = torch.empty_like(self.Q)
        self.ws = kvq.decode_workspace(w.B, w.Hq, w.Hkv, self.L, device=device)
        torch.cuda.synchronize(device)
        self.cache_bytes = cache.blocks.numel()

    def lengths(self, n):
        """n rows of pre-append sequence lengths, one per step."""
        return self.len_base.repeat(n, 1).contiguous()

    def run(self, k, seq_lens, split_events=None):
        kvq, w = self.kvq, self.w
        cache, Rk, Rv, perm = self.layers[k % len(self.layers)]
        if split_events is not None:
            kvq.kvq_rotate_quantize_append(self.Knew, self.Vnew, w.mode, Rk, Rv, perm, cache,
                                           seq_lens)
            kvq.kvq_decode_attention_timed(self.Q, cache, w.mode, Rk, Rv, perm, seq_lens, w.sink,
                                           self.L, self.ws, self.out, *split_events)
        else:          # the serving step's one call: append, then decode
            kvq.kvq_append_decode(self.Knew, self.Vnew, self.Q, cache, w.mode, Rk, Rv, perm,
                                  seq_lens, self.L, self.ws, self.out)

    def status(self):
        return max(self.kvq.kvq_get_status(c[0]) for c in self.layers)


def append_rates(device, peak, reps=5):
    """Throughput of the append alone (rotate + quantize + pack + store) on the
    bulk appends of the workload set: the llama7b prefill (B=1, 32768 tokens,
    32 heads, dense), the ragged workload's prefill (B=4, 32768 tokens, 32
    heads, dense), the hadamard workload's step append (B=16, 128 tokens,
    32 heads, permutation + FWHT) and a chunked-prefill append of the same
    size with a dense rotation.  Bytes = fp16 K
    and V read (512 B per token-head) + packed codes and metadata written
    (96 B) + the rotations read once; L2 flushed before each timed call."""
    import rotated_int2_kv_head_b200 as kvq
    flush = L2Flush(device)
    out = {}
    w0 = W.WORKLOADS["ragged"]
    wl = W.WORKLOADS["llama7b"]
    cases = [("llama7b prefill", W.custom(name="llama7b_prefill", seed=wl.seed + 1, B=1, Hq=32,
                                          Hkv=32, mode=0, k_outliers=8, context=wl.context),
              wl.context),
             ("ragged prefill", W.custom(name="ragged_prefill", seed=w0.seed + 1, B=w0.extra["prefill_B"],
                                         Hq=32, Hkv=32, mode=0, k_outliers=8,
                                         context=w0.extra["prefill_T"]), w0.extra["prefill_T"]),
             ("hadamard step append", W.WORKLOADS["hadamard"], W.WORKLOADS["hadamard"].append_T),
             ("dense chunk append", W.custom(name="dense_chunk", seed=wl.seed + 2, B=16, Hq=32, Hkv=32,
                                             mode=0, k_outliers=8, context=128), 128)]
    for name, w, T in cases:
        Rk, Rv, perm = W.rotations(w)
        rk = torch.from_numpy(Rk).to(device) if Rk is not None else None
        rv = torch.from_numpy(Rv).to(device) if Rv is not None else None
        pm = torch.from_numpy(perm).to(device) if perm is not None else None
        K, V = W.kv_batch(w, 0, T, device)
        cache = kvq.KVCache(w.B, w.Hkv, ((T + 15) // 16) * 16, w.sink, device=device)
        sl = torch.zeros(w.B, dtype=torch.int32, device=device)
        ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
        ms = []
        for k in range(reps + 2):
            sl.zero_()
            flush(k)
            host_ahead(300e-6)
            ev[0].record()
            kvq.kvq_rotate_quantize_append(K, V, w.mode, rk, rv, pm, cache, sl)
            ev[1].record()
            torch.cuda.synchronize(device)
            if k >= 2:
                ms.append(ev[0].elapsed_time(ev[1]))
        if kvq.kvq_get_status(cache) != 0:
            raise RuntimeError("append status %d" % kvq.kvq_get_status(cache))
        nbytes = T * w.B * w.Hkv * (512 + 96) + (2 * w.Hkv * 128 * 128 * 4 if w.mode == 0 else 0)
        t = float(np.median(ms)) * 1e-3
        out[name] = {"B": w.B, "T": T, "Hkv": w.Hkv, "rotation": "dense" if w.mode == 0 else "perm+fwht",
                     "ms": t * 1e3, "GB_per_s": nbytes / t / 1e9, "frac_of_hbm_peak": nbytes / t / 1e9 / peak,
                     "bytes": nbytes}
        del K, V, cache
        if nbytes < 3 * L2_BYTES:
            out[name].update(append_back_to_back(w, T, nbytes, rk, rv, pm, device, peak))
    return out


def append_back_to_back(w, T, nbytes, rk, rv, pm, device, peak, calls=40):
    """An append small enough for L2 timed as a serving loop runs it: `calls`
    appends back to back between one pair of events (no flush, no host gap),
    cycling over independent input sets and caches (distinct memory, at least
    3x L2 of traffic between two uses of one set), each append at the next
    position of its cache."""
    import rotated_int2_kv_head_b200 as kvq
    nset = -(-3 * L2_BYTES // nbytes) + 1
    per = -(-calls // nset)
    sets = []
    for i in range(nset):
        K, V = W.kv_batch(w, i * T, (i + 1) * T, device)
        cache = kvq.KVCache(w.B, w.Hkv, T * per, w.sink, device=device)
        sets.append((K, V, cache, torch.zeros(w.B, dtype=torch.int32, device=device)))
    ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))

    def run():
        for _, _, _, sl in sets:
            sl.zero_()
        host_ahead(500e-6)
        ev[0].record()
        for k in range(calls):
            K, V, cache, sl = sets[k % nset]
            kvq.kvq_rotate_quantize_append(K, V, w.mode, rk, rv, pm, cache, sl)
        ev[1].record()
        torch.cuda.synchronize(device)
        return ev[0].elapsed_time(ev[1]) * 1e-3 / calls

    run()                                   # warm-up
    t = sorted(run() for _ in range(3))[1]
    if max(kvq.kvq_get_status(c) for _, _, c, _ in sets) != 0:
        raise RuntimeError("append status (back to back)")
    del sets
    torch.cuda.empty_cache()
    return {"back_to_back_us": t * 1e6, "back_to_back_frac_of_hbm_peak": nbytes / t / 1e9 / peak,
            "back_to_back_how": "%d appends between one event pair over %d independent input sets "
                                "and caches, no flush; median of 3" % (calls, nset)}


def extension_rates(device, reps=50):
    """Decode-only timings (L2 flushed before each call, events around it) of
    the serving extensions on the llama7b cache (B=1, 32 heads, context
    32768): the plain decode, the same cache paged through a random block
    table (one pool block per 16 tokens x all heads), and q_len = 4 new
    tokens per sequence (each attending causally)."""
    import rotated_int2_kv_head_b200 as kvq
    step = Step(W.WORKLOADS["llama7b"], device, 1)
    w = step.w
    cache, Rk, Rv, perm = step.layers[0]
    L = step.L
    lens = step.len_base + step.T
    nblk = step.cap // 16
    flush = L2Flush(device)
    ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))

    def timed(fn):
        ms = []
        for k in range(reps + 3):
            flush(k)
            host_ahead(300e-6)
            ev[0].record()
            fn()
            ev[1].record()
            torch.cuda.synchronize(device)
            if k >= 3:
                ms.append(ev[0].elapsed_time(ev[1]))
        return float(np.median(ms))

    out = torch.empty_like(step.Q)
    plain = timed(lambda: kvq.kvq_decode_attention(step.Q, cache, w.mode, Rk, Rv, perm, lens, w.sink,
                                                   L, step.ws, out))
    num_blocks = w.B * nblk + 64
    g = torch.Generator().manual_seed(11)
    table = torch.randperm(num_blocks, generator=g)[:w.B * nblk].view(w.B, nblk).to(torch.int32)
    table = table.to(device)
    paged = kvq.PagedKVCache(w.B, w.Hkv, step.cap, num_blocks, table, w.sink, device=device)
    paged.block_view()[table.long()] = cache.block_view().permute(0, 2, 1, 3)
    if w.sink:
        paged.k_sink.copy_(cache.k_sink)
        paged.v_sink.copy_(cache.v_sink)
    out_p = torch.empty_like(step.Q)
    paged_ms = timed(lambda: kvq.kvq_decode_attention(step.Q, paged, w.mode, Rk, Rv, perm, lens,
                                                      w.sink, L, step.ws, out_p))
    same = bool(torch.equal(out, out_p))
    res = {"how": "decode only, L2 flushed before each call, median of %d" % reps,
           "plain_decode_ms": plain,
           "paged_decode_ms": paged_ms, "paged_output_bit_identical": same}
    q_len = 4
    if (w.Hq // w.Hkv) * q_len <= 8:
        Qm = torch.randn((w.B, w.Hq, q_len, 128), generator=torch.Generator().manual_seed(12)
                         ).to(torch.float16).to(device)
        wsm = kvq.decode_workspace(w.B, w.Hq * q_len, w.Hkv, L, device=device)
        outm = torch.empty_like(Qm)
        res["multi_query_q_len"] = q_len
        res["multi_query_decode_ms"] = timed(lambda: kvq.kvq_decode_attention_ex(
            Qm, cache, w.mode, Rk, Rv, perm, lens, w.sink, L, wsm, outm))
    if max(kvq.kvq_get_status(cache), kvq.kvq_get_status(paged)) != 0:
        raise RuntimeError("device status after the extension timings")
    return res


def sink_rates(device, reps=30):
    """Identified sinks on their full-size workload (gqa_sinks_identified:
    B=8, 32 query heads over 8 KV heads, context 131072, 4 fp16 rows per
    sequence): the same tokens appended into a cache with identified sinks
    (kvq_identify_sinks before each append) and into one with the 4 leading
    positions as sinks; decode-only times of both (L2 flushed before each
    call) and the time of the identification kernel for one decode step
    (T=1) and for a 32768-token prefill chunk."""
    import rotated_int2_kv_head_b200 as kvq
    w = W.WORKLOADS["gqa_sinks_identified"]
    L = int(w.context)
    cap = L
    Rk, Rv, _ = W.rotations(w)
    rk = torch.from_numpy(Rk).to(device)
    rv = torch.from_numpy(Rv).to(device)
    ident = kvq.KVCache(w.B, w.Hkv, cap, w.sink, device=device, identified_sinks=True)
    lead = kvq.KVCache(w.B, w.Hkv, cap, w.sink, device=device)
    sl_i = torch.zeros(w.B, dtype=torch.int32, device=device)
    sl_l = torch.zeros_like(sl_i)
    chunk = 8192
    for t0 in range(0, L, chunk):
        t1 = min(L, t0 + chunk)
        K, V = W.kv_batch(w, t0, t1, device)
        act = torch.from_numpy(np.stack([W.activations(w, b, t0, t1) for b in range(w.B)])).to(device)
        kvq.kvq_identify_sinks(act, W.MASSIVE_TAU, ident, sl_i)
        kvq.kvq_rotate_quantize_append(K, V, w.mode, rk, rv, None, ident, sl_i)
        kvq.kvq_rotate_quantize_append(K, V, w.mode, rk, rv, None, lead, sl_l)
    torch.cuda.synchronize(device)
    Q = W.queries(w, device)
    ws = kvq.decode_workspace(w.B, w.Hq, w.Hkv, L, device=device)
    flush = L2Flush(device)
    ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))

    def timed(fn, n=reps):
        ms = []
        for k in range(n + 3):
            flush(k)
            host_ahead(300e-6)
            ev[0].record()
            fn()
            ev[1].record()
            torch.cuda.synchronize(device)
            if k >= 3:
                ms.append(ev[0].elapsed_time(ev[1]))
        return float(np.median(ms))

    out_i = torch.empty_like(Q)
    out_l = torch.empty_like(Q)
    dec_i = timed(lambda: kvq.kvq_decode_attention(Q, ident, w.mode, rk, rv, None, sl_i, w.sink, L,
                                                   ws, out_i))
    dec_l = timed(lambda: kvq.kvq_decode_attention(Q, lead, w.mode, rk, rv, None, sl_l, w.sink, L,
                                                   ws, out_l))
    # identification alone, on a scratch copy of the sink list (the
    # lengths are set so that every sequence has room for the tokens)
    probe = kvq.KVCache(w.B, w.Hkv, 32768 + 16, w.sink, device=device, identified_sinks=True)
    sl0 = torch.zeros(w.B, dtype=torch.int32, device=device)
    a1 = torch.from_numpy(np.stack([W.activations(w, b, 5, 6) for b in range(w.B)])).to(device)
    aP = torch.from_numpy(np.stack([W.activations(w, b, 0, 32768) for b in range(w.B)])).to(device)

    def ident_once(a):
        probe.sink_count.zero_()
        kvq.kvq_identify_sinks(a, W.MASSIVE_TAU, probe, sl0)

    id_step = timed(lambda: ident_once(a1))
    id_pre = timed(lambda: ident_once(aP))
    counts = ident.sink_count.cpu().tolist()
    if max(kvq.kvq_get_status(ident), kvq.kvq_get_status(lead)) != 0:
        raise RuntimeError("device status after the identified-sink timings")
    if not bool(torch.isfinite(out_i.float()).all()):
        raise RuntimeError("non-finite decode output with identified sinks")
    kv_bytes = w.B * w.Hkv * L * 96
    return {"workload": "gqa_sinks_identified", "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv,
            "context": L, "sink_rows": w.sink, "sinks_per_sequence": counts,
            "how": "decode only / identification only, L2 flushed before each call, "
                   "median of %d; includes a sink-count reset memset in the identification "
                   "timings" % reps,
            "decode_identified_ms": dec_i, "decode_leading_ms": dec_l,
            "decode_identified_packed_kv_gbs": kv_bytes / (dec_i * 1e-3) / 1e9,
            "identify_step_ms": id_step, "identify_prefill_32768_ms": id_pre}


def decode_rates(device, peak, reps=20):
    """Decode alone on every workload of workloads.py at its full size (the
    cache filled through the library's append, L2 flushed before each timed
    call, median of `reps`): tokens/s = B / t, context tokens/s = sum of
    L_b * Hkv / t, packed-KV GB/s (96 B per cached token-head, 512 B per fp16
    sink token-head) and its fraction of the HBM peak, and a total-bytes rate
    that adds the rotations (dense: 2 * Hkv * 64 KB; FWHT: the permutations),
    Q and the output."""
    import rotated_int2_kv_head_b200 as kvq
    flush = L2Flush(device)
    ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    res = {"how": "decode only, cache filled first, L2 flushed before each call, median of %d; "
                  "back_to_back_*: 40 decodes between one event pair over independent copies of "
                  "the cache (no flush, no host gap), median of 3" % reps}
    # the floor of the isolated timing itself: the same flush, spin and event
    # pair around one trivial kernel (torch's spin of ~0 cycles)
    fl = []
    for k in range(reps + 3):
        flush(k)
        host_ahead(300e-6)
        ev[0].record()
        torch.cuda._sleep(1)
        ev[1].record()
        torch.cuda.synchronize(device)
        if k >= 3:
            fl.append(ev[0].elapsed_time(ev[1]))
    res["event_pair_floor_us"] = float(np.median(fl)) * 1e3
    for name in ("tiny", "llama7b", "hadamard", "gqa_sinks", "gqa8", "ragged"):
        w = W.WORKLOADS[name]
        lens_np = w.seq_lens().astype(np.int32)
        L = int(lens_np.max())
        cap = ((L + 15) // 16) * 16
        Rk, Rv, perm = W.rotations(w)
        rk = torch.from_numpy(Rk).to(device) if Rk is not None else None
        rv = torch.from_numpy(Rv).to(device) if Rv is not None else None
        pm = torch.from_numpy(perm).to(device) if perm is not None else None
        cache = kvq.KVCache(w.B, w.Hkv, cap, w.sink, device=device)
        fill = torch.zeros(w.B, dtype=torch.int32, device=device)
        for t0 in range(0, L, 4096):
            K, V = W.kv_batch(w, t0, min(L, t0 + 4096), device)
            kvq.kvq_rotate_quantize_append(K, V, w.mode, rk, rv, pm, cache, fill)
            del K, V
        lens = torch.from_numpy(lens_np).to(device)
        Q = W.queries(w, device)
        ws = kvq.decode_workspace(w.B, w.Hq, w.Hkv, L, device=device)
        out = torch.empty_like(Q)
        ms = []
        for k in range(reps + 3):
            flush(k)
            host_ahead(300e-6)
            ev[0].record()
            kvq.kvq_decode_attention(Q, cache, w.mode, rk, rv, pm, lens, w.sink, L, ws, out)
            ev[1].record()
            torch.cuda.synchronize(device)
            if k >= 3:
                ms.append(ev[0].elapsed_time(ev[1]))
        if kvq.kvq_get_status(cache) != 0 or not bool(torch.isfinite(out.float()).all()):
            raise RuntimeError("decode timings on %s: bad status or output" % name)
        t = float(np.median(ms)) * 1e-3
        kv = packed_kv_bytes(w, lens_np)
        rot = 2 * w.Hkv * 128 * 128 * 4 if w.mode == 0 else 2 * w.Hkv * 128 * 4
        total = kv + rot + 2 * Q.numel() * 2
        res[name] = {"B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "context_max": L,
                     "rotation": "dense" if w.mode == 0 else "perm+fwht", "sink_fp16": w.sink,
                     "decode_us": t * 1e6, "tokens_per_s": w.B / t,
                     "context_tokens_per_s": float(lens_np.astype(np.int64).sum()) * w.Hkv / t,
                     "packed_kv_bytes": kv, "packed_kv_gbs": kv / t / 1e9,
                     "frac_of_hbm_peak": kv / t / 1e9 / peak, "total_bytes_gbs": total / t / 1e9}
        n_layers = layers_for(cache.blocks.numel())
        if n_layers == 0:
            # too small to cycle out of L2: one distinct copy per call, L2 flushed
            # once before each timed run, so every call still reads a cold cache
            n_layers = -40
        tb = decode_back_to_back(w, cache, Q, rk, rv, pm, lens, L, ws, out, n_layers, device,
                                 flush=flush if n_layers < 0 else None)
        res[name].update({"back_to_back_us": tb * 1e6,
                          "back_to_back_frac_of_hbm_peak": kv / tb / 1e9 / peak,
                          "back_to_back_layers": abs(n_layers)})
        del cache, ws
        torch.cuda.empty_cache()
    return res


def decode_back_to_back(w, cache, Q, rk, rv, pm, lens, L, ws, out, n_layers, device, calls=40,
                        flush=None):
    """Decode as a serving loop runs it: `calls` decodes back to back between
    one pair of events (no host gap), cycling over n_layers independent
    copies of the cache (at least 3x L2 of other cache traffic between two
    uses of one copy).  A cache too small for that passes n_layers = -calls
    and an L2 flush: one copy per call, L2 flushed once before each run
    (outside the events).  Median of 3 runs, seconds per decode."""
    import rotated_int2_kv_head_b200 as kvq
    n_layers = abs(n_layers)
    layers = [cache]
    for _ in range(1, n_layers):
        c2 = kvq.KVCache(w.B, w.Hkv, cache.capacity, w.sink, device=device)
        c2.blocks.copy_(cache.blocks)
        if cache.k_sink is not None:
            c2.k_sink.copy_(cache.k_sink)
            c2.v_sink.copy_(cache.v_sink)
        layers.append(c2)
    ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))

    def run():
        if flush is not None:
            flush(0)
        host_ahead(500e-6)
        ev[0].record()
        for k in range(calls):
            kvq.kvq_decode_attention(Q, layers[k % n_layers], w.mode, rk, rv, pm, lens, w.sink, L,
                                     ws, out)
        ev[1].record()
        torch.cuda.synchronize(device)
        return ev[0].elapsed_time(ev[1]) * 1e-3 / calls

    run()                                   # warm-up
    t = sorted(run() for _ in range(3))[1]
    if max(kvq.kvq_get_status(c) for c in layers) != 0:
        raise RuntimeError("decode status (back to back)")
    del layers
    return t


def prerope_rates(device, reps=20):
    """Pre-RoPE grouped-head key rotation on the llama7b shape (B=1, 32
    heads, context 32768): the 32768-token prefill appended through
    kvq_prerope_append, then decode-only timings (L2 flushed before each
    call) for group sizes 1 and 4, beside the post-RoPE FWHT decode of the
    same tokens.  The decode is bound by its instruction stream (a 128*gh
    point FWHT, the permutation scatter and RoPE per cached token), so its
    roofline is reported as packed-KV bytes / time for comparison only."""
    import rotated_int2_kv_head_b200 as kvq
    w = W.custom(name="llama7b_prerope", seed=1002, B=1, Hq=32, Hkv=32, mode=1, context=32768,
                 k_outliers=8)
    L = 32768
    flush = L2Flush(device)
    ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))

    def timed(fn, n=reps):
        ms = []
        for k in range(n + 3):
            flush(k)
            host_ahead(300e-6)
            ev[0].record()
            fn()
            ev[1].record()
            torch.cuda.synchronize(device)
            if k >= 3:
                ms.append(ev[0].elapsed_time(ev[1]))
        return float(np.median(ms))

    K, V = W.kv_batch(w, 0, L, device)
    Q = W.queries(w, device)
    lens = torch.full((1,), L, dtype=torch.int32, device=device)
    res = {"workload": "llama7b shape, pre-RoPE keys", "B": 1, "Hq": 32, "Hkv": 32, "context": L,
           "how": "L2 flushed before each call, median of %d" % reps}
    for gh in (1, 4):
        perm = torch.from_numpy(W.prerope_perm(w, gh)).to(device)
        cache = kvq.KVCache(1, 32, L, device=device)
        sl = torch.zeros(1, dtype=torch.int32, device=device)

        def app():
            sl.zero_()
            kvq.kvq_prerope_append(K, V, gh, perm, cache, sl)

        app_ms = timed(app, 5)
        ws = kvq.prerope_workspace(1, 32, 32, gh, L, device=device)
        out = torch.empty_like(Q)
        dec_ms = timed(lambda: kvq.kvq_prerope_decode(Q, cache, gh, perm, 10000.0, lens, L, ws, out))
        if kvq.kvq_get_status(cache) != 0 or not bool(torch.isfinite(out.float()).all()):
            raise RuntimeError("pre-RoPE timings: bad status or output")
        res["gh%d" % gh] = {"prefill_append_ms": app_ms, "decode_ms": dec_ms,
                            "decode_packed_kv_gbs": 32 * L * 96 / (dec_ms * 1e-3) / 1e9}
    # the post-RoPE FWHT decode over the same tokens, for comparison
    Rk = Rv = None
    perm1 = torch.from_numpy(W.rotations(w)[2]).to(device)
    cache = kvq.KVCache(1, 32, L, device=device)
    sl = torch.zeros(1, dtype=torch.int32, device=device)
    kvq.kvq_rotate_quantize_append(K, V, 1, Rk, Rv, perm1, cache, sl)
    ws = kvq.decode_workspace(1, 32, 32, L, device=device)
    out = torch.empty_like(Q)
    res["post_rope_fwht_decode_ms"] = timed(lambda: kvq.kvq_decode_attention(
        Q, cache, 1, Rk, Rv, perm1, lens, 0, L, ws, out))
    return res


def sample_sequence(lens):
    """The sequence whose length is the batch median (the lower middle one
    for an even batch; the first of equal lengths): the CPU oracle's sample
    of a ragged batch."""
    order = np.argsort(np.asarray(lens), kind="stable")
    return int(order[(len(order) - 1) // 2])


def sample_scale(w, lens, b, heads):
    """Factor from the oracle's sample (KV heads 0..heads-1 of sequence b) to
    the whole step: decode work grows with the context, so the factor is the
    batch's context token-heads over the sample's, sum_b' L_b' * Hkv /
    (L_b * heads); for a uniform batch it is B * Hkv / heads."""
    lens = np.asarray(lens, np.int64)
    return float(lens.sum()) * w.Hkv / (float(lens[b]) * heads)


class OracleSample:
    """The CPU oracle holding one sequence's cache for the first `heads` KV
    heads, filled to the step's pre-append length, ready to run the step's
    append of T tokens and its decode; rows drawn on `device` (the very
    tensors the GPU arm used, when given that arm's Step)."""

    def __init__(self, w, b, heads, device, step=None):
        from oracle import oracle as orc
        self.orc, self.w, self.b, self.heads = orc, w, b, heads
        lens = w.seq_lens()
        self.L, T = int(lens[b]), w.append_T
        self.pre = self.L - T
        Rk, Rv, perm = W.rotations(w)
        self.rk = Rk[:heads] if Rk is not None else None
        self.rv = Rv[:heads] if Rv is not None else None
        self.pm = perm[:, :heads] if perm is not None else None
        self.oc = orc.Cache(1, heads, ((self.L + 15) // 16) * 16, w.sink)
        self.sl = np.zeros(1, np.int32)
        for t0 in range(0, self.pre, 4096):
            t1 = min(self.pre, t0 + 4096)
            K, V = W.kv_batch(w, t0, t1, device, bs=[b])
            orc.append(self.oc, W.f16_bits(K[:, :, :heads]), W.f16_bits(V[:, :, :heads]), w.mode,
                       self.rk, self.rv, self.pm, self.sl)
        if step is not None:
            Kn, Vn, Q = step.Knew[b:b + 1], step.Vnew[b:b + 1], step.Q[b:b + 1]
        else:
            Kn, Vn = W.kv_batch(w, self.pre, self.L, device, bs=[b])
            Q = W.queries(w, device)[b:b + 1]
        self.Kn = W.f16_bits(Kn[:, :, :heads])
        self.Vn = W.f16_bits(Vn[:, :, :heads])
        self.Q = W.f16_bits(Q[:, :heads * w.G])
        self.cores = len(os.sched_getaffinity(0))

    def step(self):
        """The step's append of T tokens at the pre-append length, then the
        decode over the sample's context (OpenMP over the cores)."""
        self.sl[0] = self.pre
        self.orc.append(self.oc, self.Kn, self.Vn, self.w.mode, self.rk, self.rv, self.pm, self.sl)
        self.orc.decode(self.oc, self.Q, self.w.mode, self.rk, self.rv, self.pm, self.sl,
                        n_threads=self.cores)

    def describe(self, n, el, scale):
        return ("sequence %d (context %d, the batch median), KV heads 0..%d of %d: append %d "
                "token(s) + decode, %d sample steps in %.2f s; per-step time scaled by %.1f "
                "(the batch's context token-heads over the sample's)"
                % (self.b, self.L, self.heads - 1, self.w.Hkv, self.w.append_T, n, el, scale))


def cpu_baseline(w, step, device, heads=2, min_seconds=5.0):
    """The CPU oracle, as it stands, on a bounded sample of the same workload
    (the first `heads` KV heads of the batch's median-length sequence; its
    rows drawn on `device`, or the GPU arm's own step inputs when `step` is
    given), timed for append + decode and scaled to the whole step by
    sample_scale."""
    lens = w.seq_lens()
    b = sample_sequence(lens)
    heads = min(heads, w.Hkv)
    smp = OracleSample(w, b, heads, device, step)
    n, t_start = 0, time.perf_counter()
    while True:
        smp.step()
        n += 1
        el = time.perf_counter() - t_start
        if el >= min_seconds or n >= 1000:
            break
    scale = sample_scale(w, lens, b, heads)
    per_step = el / n * scale
    return {"value": w.B / per_step, "unit": "tokens/s", "cores": smp.cores, "kind": "oracle",
            "sample": smp.describe(n, el, scale)}


def graph_plan(K, n_layers, per_graph_target=40):
    """Exactly K steps as CUDA-graph replays: (per_graph, full, remainder) =
    `full` replays of a graph of per_graph steps (whole rounds over the
    layers) and, if remainder > 0, one replay of a graph of the remaining
    steps."""
    per_graph = n_layers * max(1, per_graph_target // n_layers)
    return per_graph, K // per_graph, K % per_graph


def measure_step(w, dev, K, warmup, dist_on, local, e2e=True):
    """Times K steps (append + decode) of workload w on device dev: the
    throughput loop (graph replay over independent layers, or flushed
    single steps for caches too small for layers), the split kernel alone by
    library events, the isolated flushed step, and (e2e) the host-buffer
    step through kvq_append_decode_host.  Returns a dict of raw timings."""
    import rotated_int2_kv_head_b200 as kvq
    lens = w.seq_lens()
    cap = ((int(lens.max()) + 15) // 16) * 16
    n_layers = layers_for(w.B * w.Hkv * (cap // 16) * 1536)
    step = Step(w, dev, max(1, n_layers))
    flush = L2Flush(dev) if n_layers == 0 else None

    def steps(n, sl, timed=None, split_events=None):
        """n steps; with `timed`, one event pair around all of them (layers
        mode) or around each (flush mode, the flush outside the events)."""
        ms = 0.0
        if flush is None and timed is not None:
            timed[0].record()
        for k in range(n):
            if flush is not None:
                flush(k)
                if timed is not None:
                    timed[0].record()
            step.run(k, sl[k], None if split_events is None else split_events[k])
            if flush is not None and timed is not None:
                timed[1].record()
                torch.cuda.synchronize(dev)
                ms += timed[0].elapsed_time(timed[1])
        if flush is None and timed is not None:
            timed[1].record()
            torch.cuda.synchronize(dev)
            ms = timed[0].elapsed_time(timed[1])
        return ms

    steps(warmup, step.lengths(warmup))
    torch.cuda.synchronize(dev)
    ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    graphs = []
    per_graph = 0
    if flush is None:
        # Layers mode: the steps are replayed from CUDA graphs, as a serving
        # loop would, so the host's per-call launch cost (about 33 us per
        # step through the Python binding) stays out of the device timing.
        # A graph = a copy that resets its rows of pre-append lengths, then
        # its steps' kernels with their programmatic dependent launches;
        # exactly K steps run: `full` graphs of per_graph steps, then one of
        # the remainder.
        per_graph, full, rem = graph_plan(K, len(step.layers))
        side = torch.cuda.Stream(dev)
        for n_g, reps in ((per_graph, full), (rem, 1)):
            if n_g == 0 or reps == 0:
                continue
            sl_g = step.lengths(n_g)
            sl_init = sl_g.clone()
            side.wait_stream(torch.cuda.current_stream(dev))
            with torch.cuda.stream(side):
                for k in range(n_g):
                    step.run(k, sl_g[k])
            torch.cuda.current_stream(dev).wait_stream(side)
            torch.cuda.synchronize(dev)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                sl_g.copy_(sl_init)
                for k in range(n_g):
                    step.run(k, sl_g[k])
            graphs.append((g, reps, sl_g, sl_init))
        for _ in range(max(1, -(-warmup // max(1, per_graph)))):
            graphs[0][0].replay()
        torch.cuda.synchronize(dev)
    sl = step.lengths(K) if not graphs else None
    with ClockSampler(local) as clk:
        barrier(dist_on, dev)
        torch.cuda.synchronize(dev)
        if not graphs:
            total_ms = steps(K, sl, ev)
        else:
            ev[0].record()
            for g, reps, _, _ in graphs:
                for _ in range(reps):
                    g.replay()
            ev[1].record()
            torch.cuda.synchronize(dev)
            total_ms = ev[0].elapsed_time(ev[1])
        torch.cuda.synchronize(dev)
        barrier(dist_on, dev)
    steps_run = K
    total_ms = max_over_ranks(total_ms, dist_on, dev)
    del graphs

    # the streaming kernel alone, timed live by events the library records
    # around it (a separate loop: events between kernels stop the
    # programmatic overlap of the steps above)
    n_split = min(K, 100)
    split_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(n_split)]
    for pair in split_ev:          # create the underlying events before handing them to C
        for e in pair:
            e.record()
    sl_split = step.lengths(n_split)
    torch.cuda.synchronize(dev)
    # The host takes about as long to submit a step as the device takes to
    # run a small one, so a kernel could wait on its own submission between
    # the events.  torch's spin kernel (a fixed cycle count) at the head of
    # the stream lets the host queue every step before the first one runs.
    host_ahead(n_split * 80e-6 + 2e-3)
    steps(n_split, sl_split, None, split_ev)
    torch.cuda.synchronize(dev)
    split_ms = [x.elapsed_time(y) for x, y in split_ev]

    # one step at a time after an L2 flush, each bracketed by its own events
    # (the latency of an isolated step, for reference)
    n_iso = min(K, 50)
    iso_flush = flush or L2Flush(dev)
    sl_iso = step.lengths(n_iso)
    iso_ms = []
    for k in range(n_iso):
        iso_flush(k)
        host_ahead(300e-6)
        ev[0].record()
        step.run(k, sl_iso[k])
        ev[1].record()
        torch.cuda.synchronize(dev)
        iso_ms.append(ev[0].elapsed_time(ev[1]))
    del iso_flush
    if step.status() != 0:
        raise RuntimeError("device status %d after timed steps" % step.status())
    res = {"step": step, "n_layers": n_layers, "total_ms": total_ms, "steps": steps_run,
           "per_graph": per_graph, "split_ms": split_ms, "iso_ms": iso_ms,
           "clocks": clk.summary()}
    if not e2e:
        return res

    # end to end through the C-ABI call with host buffers: one
    # kvq_append_decode_host per step copies the step's new K/V rows and
    # queries in from pinned memory, appends, decodes and copies the output
    # back; the host then waits for the stream.  The inputs are views of one
    # pinned buffer, back to back, so the call moves them with a single copy.
    hIn = step.inbuf.cpu().pin_memory()
    nk = step.Knew.numel()
    hK = hIn[:nk].view(step.Knew.shape)
    hV = hIn[nk:2 * nk].view(step.Vnew.shape)
    hQ = hIn[2 * nk:].view(step.Q.shape)
    hO = torch.empty(step.out.shape, dtype=step.out.dtype).pin_memory()
    wsh = kvq.step_workspace(w.B, step.T, w.Hq, w.Hkv, step.L, device=dev)
    n_e2e = min(K, 200)
    sl_e2e = step.lengths(n_e2e + 3)
    # one prepared host step per layer (arguments checked once, as a serving
    # loop would hold them); each call names its own row of lengths
    plans = [kvq.HostStep(hK, hV, hQ, cache, w.mode, Rk, Rv, perm, sl_e2e[0], step.L, wsh, hO)
             for cache, Rk, Rv, perm in step.layers]
    e2e_s = 0.0
    for k in range(n_e2e + 3):
        if flush is not None:
            flush(k)
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        plans[k % len(plans)].run(sl_e2e[k])
        torch.cuda.synchronize(dev)
        if k >= 3:
            e2e_s += time.perf_counter() - t0
    e2e_s = max_over_ranks(e2e_s, dist_on, dev)
    if not torch.equal(hO.to(dev), step.out):      # the same step as the device-timed one
        raise RuntimeError("host-buffer step output differs from the device step")
    res.update(e2e_s=e2e_s, n_e2e=n_e2e, h2d=(hK.numel() + hV.numel() + hQ.numel()) * 2,
               d2h=hO.numel() * 2)
    return res


def l2_note(m):
    step, n_layers = m["step"], m["n_layers"]
    if n_layers == 0:
        return "flushed between steps (256 MB write, then 256 MB read); steps timed one by one"
    if n_layers > 1:
        note = ("inputs larger than L2: %d independent layers (%.1f MB of cache each) cycled, so "
                "each step reads a cache %d other steps (%.0f MB) after its last use; steps back "
                "to back" % (n_layers, step.cache_bytes / 1e6, n_layers - 1,
                             (n_layers - 1) * step.cache_bytes / 1e6))
    else:
        note = ("inputs larger than L2 (one %.0f MB cache, %.0f MB of it read per step); steps "
                "back to back" % (step.cache_bytes / 1e6, packed_kv_bytes(step.w, step.w.seq_lens())
                                  / 1e6))
    return note + "; timed steps replayed from CUDA graphs of %d steps (+ one of the remainder)" \
        % m["per_graph"]


def split_roofline(w, m, peak, peak_src, workload):
    kv_bytes = packed_kv_bytes(w, w.seq_lens())
    split_mean_s = float(np.mean(m["split_ms"])) * 1e-3
    achieved = kv_bytes / split_mean_s / 1e9
    return {"bound": "hbm", "kernel": "decode_split_kernel (streams the packed cache)",
            "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
            "traffic": profiled_traffic(workload, kv_bytes),
            "algorithmic_bytes_per_launch": kv_bytes, "kernel_ms_mean": split_mean_s * 1e3,
            "peak_source": peak_src,
            "timing": "CUDA events the library records around the kernel, %d eager steps "
                      "queued behind a spin kernel (no host gap inside the events)"
                      % len(m["split_ms"])}


def run_cuda(args):
    rank, world, local = dist_env()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    dist_on = init_dist("nccl", world)
    from rotated_int2_kv_head_b200 import build as kbuild
    kbuild.build()
    w = rank_workload(W.WORKLOADS[args.workload], rank)
    lens = w.seq_lens()
    K = args.steps
    m = measure_step(w, dev, K, args.warmup, dist_on, local)
    step = m["step"]

    if rank != 0:
        if dist_on:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    peak, peak_src = measured_peak()
    kv_bytes = packed_kv_bytes(w, lens)
    ms_per_step = m["total_ms"] / K
    tokens = w.B * world
    line = {
        "metric": METRIC,
        "value": tokens * K / (m["total_ms"] * 1e-3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": m["steps"],
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int2 codes + fp16 scale/zero, fp32 accumulate",
        "data": "synthetic (seeded; workloads.py)",
        "config": {"workload": args.workload, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "head_dim": 128,
                   "context": int(lens.max()) if w.ragged is None else
                   "ragged U[%d, %d] (sum %d)" % (w.ragged[0], w.ragged[1], int(lens.sum())),
                   "append_T": w.append_T,
                   "rotation": "dense" if w.mode == 0 else "perm+fwht", "sink_fp16": w.sink,
                   "group": 32, "l2": l2_note(m), "layers": max(1, m["n_layers"]),
                   "parallelism": "replicas: one independent batch per GPU"},
        "packed_kv_gbs": kv_bytes / (ms_per_step * 1e-3) / 1e9,
        "packed_kv_bytes_per_step": kv_bytes,
        "context_tokens_per_s": float(lens.astype(np.int64).sum()) * w.Hkv * world
        / (ms_per_step * 1e-3),
        "roofline": split_roofline(w, m, peak, peak_src, args.workload),
        "e2e": {"value": tokens * m["n_e2e"] / m["e2e_s"], "unit": "tokens/s",
                "h2d_bytes_per_step": m["h2d"], "d2h_bytes_per_step": m["d2h"],
                "how": "wall clock per step: one kvq_append_decode_host call through a prepared "
                       "HostStep (pinned H2D of the new K/V/Q, append, decode, D2H of the "
                       "output), then a stream synchronise"},
        "isolated_step": {"ms": float(np.median(m["iso_ms"])), "how": "median of %d steps, each "
                          "after an L2 flush and bracketed by its own events, queued behind a "
                          "spin kernel" % len(m["iso_ms"])},
        "gpu_launches": KERNELS_PER_STEP * K,
        "clocks": m["clocks"],
    }
    del m, step
    torch.cuda.empty_cache()
    if world == 1 and not args.no_extras and args.workload != "llama7b":
        # the single-layer 32-head decode step (B=1, context 32768) as an extra
        wl = W.WORKLOADS["llama7b"]
        ml = measure_step(wl, dev, min(K, 400), args.warmup, False, local, e2e=True)
        msl = ml["total_ms"] / ml["steps"]
        line["llama7b_step"] = {
            "tokens_per_s": wl.B * ml["steps"] / (ml["total_ms"] * 1e-3), "ms_per_step": msl,
            "steps": ml["steps"], "l2": l2_note(ml),
            "roofline": split_roofline(wl, ml, peak, peak_src, "llama7b"),
            "e2e_tokens_per_s": wl.B * ml["n_e2e"] / ml["e2e_s"],
            "isolated_step_ms": float(np.median(ml["iso_ms"]))}
        del ml
        torch.cuda.empty_cache()
    if world == 1 and not args.no_append:
        line["append"] = append_rates(dev, peak)
    if world == 1 and not args.no_extensions:
        line["extensions"] = extension_rates(dev)
        line["extensions"]["identified_sinks"] = sink_rates(dev)
        line["extensions"]["pre_rope"] = prerope_rates(dev)
    if world == 1 and not args.no_workloads:
        line["workloads"] = decode_rates(dev, peak)
    if world == 1 and not args.no_cpu_baseline:
        sw = rank_workload(W.WORKLOADS[args.workload], rank)
        line["cpu_baseline"] = cpu_baseline(sw, None, "cpu")
    print(json.dumps(line), flush=True)
    if dist_on:
        import torch.distributed as dist
        dist.destroy_process_group()


# --- the reference arm: the CPU oracle ----------------------------------------------------------

def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    w = W.WORKLOADS[args.workload]
    lens = w.seq_lens()
    b = sample_sequence(lens)
    heads = 1
    smp = OracleSample(w, b, heads, "cpu")
    for _ in range(args.warmup):
        smp.step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        smp.step()
    el = time.perf_counter() - t0
    scale = sample_scale(w, lens, b, heads)
    ms_sample = el / args.steps * 1e3
    value = w.B / (ms_sample * 1e-3 * scale)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup,
        # the time each sample step actually took; the whole-batch step would
        # take sample_scale times as long (the value is computed from that)
        "ms_per_step": ms_sample, "sample_scale": scale,
        "ms_per_step_scaled_estimate": ms_sample * scale,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64 (fp32 quantizer)", "data": "synthetic (seeded; workloads.py)",
        "config": {"workload": args.workload, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "head_dim": 128,
                   "context": int(lens.max()) if w.ragged is None else
                   "ragged U[%d, %d] (sum %d)" % (w.ragged[0], w.ragged[1], int(lens.sum())),
                   "append_T": w.append_T,
                   "rotation": "dense" if w.mode == 0 else "perm+fwht",
                   "sink_fp16": w.sink, "group": 32},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": smp.cores, "kind": "oracle",
                         "sample": smp.describe(args.steps, el, scale)},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["kvq", "reference"], default="kvq")
    ap.add_argument("--workload", default="ragged", choices=sorted(W.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-append", action="store_true", help="skip the bulk-append rates")
    ap.add_argument("--no-extensions", action="store_true",
                    help="skip the extension timings (paged, multi-query, identified sinks, pre-RoPE)")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the decode timings of every workload at full size")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the llama7b step measured beside a ragged headline")
    ap.add_argument("--extension", choices=["pre_rope", "identified_sinks", "workloads"],
                    default=None,
                    help="time one extension alone and print its JSON")
    ap.add_argument("--append-only", action="store_true",
                    help="only the bulk-append rates (one GPU), as one JSON line")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.steps < 1:
        ap.error("--steps must be >= 1")
    if args.impl == "reference":
        run_reference(args)
    elif args.append_only:
        torch.cuda.set_device(0)
        from rotated_int2_kv_head_b200 import build as kbuild
        kbuild.build()
        peak, src = measured_peak()
        print(json.dumps({"append": append_rates(torch.device("cuda", 0), peak), "peak_gbs": peak,
                          "peak_source": src}), flush=True)
    elif args.extension:
        # one extension's timings alone (the same functions the full run
        # reports under "extensions")
        torch.cuda.set_device(0)
        from rotated_int2_kv_head_b200 import build as kbuild
        kbuild.build()
        dev = torch.device("cuda", 0)
        if args.extension == "workloads":
            print(json.dumps({"workloads": decode_rates(dev, measured_peak()[0])}), flush=True)
        else:
            fn = {"pre_rope": prerope_rates, "identified_sinks": sink_rates}[args.extension]
            print(json.dumps({args.extension: fn(dev)}), flush=True)
    else:
        run_cuda(args)


if __name__ == "__main__":
    main()
