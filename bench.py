"""Benchmark: one decode step of packed-KV attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kvq|reference]

Workload (the decode GQA configuration): batch 32, H_q 32, H_kv 8, d_h 128,
context 4096 for every sequence, 4-bit codes in groups of 32 with float32
scales, bf16 Q and O.  One step is one pass of the whole hot path for a
decode step:

  1. append -- kvq_pack re-packs the K group that holds the new token
     (tokens 4064..4095) from a float32 recent-token window, and packs the
     new token's V row (token 4095), and
  2. attend -- kvq_attend over the whole 4096-token packed cache.

Two independent packed caches (2 x 168 MB, more than the 126 MB L2) are used
in turn so no step reads the previous step's cache from L2.

Prints one JSON line (rank 0).  ``value`` is algorithmic bytes per step
(packed codes + scales of every valid token + Q + O for the attend, float32
window in + codes/scales out for the append) over the device time per step,
summed over all ranks and divided by the max over ranks.

``--impl reference`` times the CPU oracle instead (NumPy, on this host's
cores), on a bounded sample of the same workload, and reports the same
metric.

Studies of the kvq arm (not the headline): ``--workload`` long_context or
chunk, ``--bits 8``, ``--group 8``, ``--window W`` (the last W tokens of each
sequence kept unquantized, kvq_attend_window) and ``--causal`` (the chunk's
rows are each sequence's last positions, kvq_attend_causal).  ``e2e`` goes
through the Python API with every step's inputs copied in from pinned host
memory and its output read back, the copies on a second stream so that the
next step's inputs arrive while a step computes.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "4-bit packed-KV attention: achieved HBM GB/s (% of 8 TB/s), µs per decode step"
WORKLOAD = "decode_gqa"
SEED = 0


# ---------------------------------------------------------------------------
# ranks: the batch is sharded, one independent batch per rank (no collective
# on the data path); the timing is the max over ranks
# ---------------------------------------------------------------------------

def rank_seed(rank: int) -> int:
    """Seed of rank `rank`'s batch: every rank attends its own sequences."""
    return SEED + rank


def max_over_ranks(values, world: int, device=None):
    """Element-wise max over the ranks of a list of floats (all_reduce MAX of
    the process group in use: NCCL on GPUs, gloo on CPU)."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def whole_job_rate(units_per_rank: float, world: int, ms_per_step: float) -> float:
    """Units all ranks processed per second, timed by the slowest rank."""
    return world * units_per_rank / (ms_per_step * 1e-3)


# ---------------------------------------------------------------------------
# byte accounting
# ---------------------------------------------------------------------------

def attend_bytes(B, H_q, H_kv, D, lengths, bits=4, group=32, q_bytes=2, o_bytes=2, lq=1):
    """Algorithmic bytes of one attend: codes + scales of every valid token of
    every (b, h_kv), plus Q and O.  K scales count per started group of g
    tokens (a K group's scale row is read whole), V scales per token."""
    dp = -(-D // group) * group
    total = 0
    for n in lengths:
        n = int(n)
        k_codes = n * D * bits // 8
        v_codes = n * dp * bits // 8
        k_scales = -(-n // group) * D * 4
        v_scales = n * (dp // group) * 4
        total += H_kv * (k_codes + v_codes + k_scales + v_scales)
    total += B * H_q * lq * D * (q_bytes + o_bytes)
    return total


def append_bytes(B, H_kv, D, k_tokens, v_tokens=1, bits=4, group=32, in_bytes=4):
    """Bytes of the decode-step append: the K tail group (k_tokens float32
    rows in, their codes and the group's scale row out) and the new V rows
    (v_tokens float32 rows in, codes and scales out)."""
    dp = -(-D // group) * group
    k = k_tokens * D * in_bytes + k_tokens * D * bits // 8 + -(-k_tokens // group) * D * 4
    v = v_tokens * D * in_bytes + v_tokens * dp * bits // 8 + v_tokens * (dp // group) * 4
    return B * H_kv * (k + v)


# ---------------------------------------------------------------------------
# environment
# ---------------------------------------------------------------------------

def measured_peaks(kind: str = "hbm"):
    """(peak, source): HBM GB/s or dense bf16 TFLOP/s (burst) from the
    measured file, else the fallback figures."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs" if kind == "hbm" else "bf16_tflops"]), "measured"
    except Exception:
        return (6650.0 if kind == "hbm" else 1590.0), "fallback"


PROFILE_FOR = {
    ("decode_gqa", 4, 32): "attend_decode_gqa_b32_ctx4096.md",
    ("decode_gqa", 8, 32): "attend_decode_gqa_b32_ctx4096_8bit.md",
    ("chunk", 4, 32): "attend_chunk_b4_lq64_ctx16384.md",
    ("chunk", 8, 32): "attend_chunk_b4_lq64_ctx16384_8bit.md",
    ("long_context", 4, 32): "attend_decode_long_b8_ctx1000_32768.md",
}


def recorded_traffic(kernel_src: str, workload: str = "decode_gqa", bits: int = 4, group: int = 32,
                     window: int = 0):
    """Per-launch DRAM bytes of the attend kernel from the committed ncu
    summary of this workload, code width and group size, or None when there
    is none (a window is not profiled) or the kernel source changed since
    the capture."""
    import hashlib
    name = None if window else PROFILE_FOR.get((workload, bits, group))
    if name is None:
        return None
    summary = os.path.join(ROOT, "profiles", name)
    try:
        text = open(summary, encoding="utf-8").read()
        src = open(kernel_src, "rb").read()
    except OSError:
        return None
    digest = hashlib.sha256(src).hexdigest()[:16]
    want, traffic = None, None
    for line in text.splitlines():
        if line.startswith("kernel_source_sha256_16:"):
            want = line.split(":", 1)[1].strip()
        if line.startswith("dram_bytes_per_launch:"):
            traffic = int(line.split(":", 1)[1].strip().replace(",", ""))
    return traffic if (want == digest and traffic) else None


class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML on a thread."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, index: int, period_s: float = 0.002):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self.ok = False
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: clocks reported as unavailable
            self.err = str(e)

    def _sample(self):
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            for bit, name in self.REASONS.items():
                if r & bit:
                    self.reasons.add(name)
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        # the region may be shorter than one polling period: one more sample
        # at its end (the caller exits right after its end-of-region sync)
        if self.ok:
            self._stop.set()
            self.t.join()
            self._sample()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "note": "NVML unavailable" if not self.ok else "no samples"}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


def event_times_us(run, n: int, stream, between=None):
    """Device times (µs) of n calls run(i), each bracketed by its own CUDA
    events on `stream`.  between(i), if given, runs before call i outside
    the events (an L2 flush)."""
    import torch
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for i in range(n):
        if between is not None:
            between(i)
        ev[i][0].record(stream)
        run(i)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) * 1e3 for a, b in ev]


def distribution(us):
    """Median, p10 and p90 of a list of observations, and the list itself."""
    a = np.asarray(us, np.float64)
    return {"median": round(float(np.median(a)), 3), "p10": round(float(np.percentile(a, 10)), 3),
            "p90": round(float(np.percentile(a, 90)), 3), "n": int(a.size),
            "all": [round(float(x), 3) for x in a]}


def copy_rows_h2d(dst, src, stream) -> None:
    """Pinned host rows into a strided device view with one pitched copy
    (cudaMemcpy2DAsync: the copy engine alone).  `dst` is the last rows of a
    contiguous [B, H, W, D] device tensor (dst = t[:, :, -L:]), `src` a
    contiguous [B, H, L, D] pinned host tensor.  torch's copy_ into such a
    view stages the rows and runs an elementwise kernel on the copy stream,
    which cannot start while an attend kernel holds every SM."""
    import ctypes
    import torch
    global _CUDART
    if "_CUDART" not in globals():
        fn = None
        names = []
        try:
            import nvidia.cuda_runtime as rt
            names.append(os.path.join(list(rt.__path__)[0], "lib", "libcudart.so.12"))
        except ImportError:
            pass
        names += ["libcudart.so.12", "libcudart.so"]
        for name in names:
            try:
                fn = ctypes.CDLL(name).cudaMemcpy2DAsync
                break
            except (OSError, AttributeError):
                continue
        if fn is not None:
            fn.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_size_t,
                           ctypes.c_size_t, ctypes.c_int, ctypes.c_void_p]
            fn.restype = ctypes.c_int
        _CUDART = fn
    if _CUDART is None:                     # no runtime library found: torch's copy (a staging kernel)
        with torch.cuda.stream(stream):
            dst.copy_(src, non_blocking=True)
        return
    B_, H_, L_, D_ = src.shape
    assert dst.shape == src.shape and src.is_contiguous() and dst.stride(3) == 1
    assert dst.stride(0) == H_ * dst.stride(1) and dst.stride(2) == D_
    es = src.element_size()
    rc = _CUDART(ctypes.c_void_p(dst.data_ptr()), dst.stride(1) * es, ctypes.c_void_p(src.data_ptr()),
                 L_ * D_ * es, L_ * D_ * es, B_ * H_, 1, ctypes.c_void_p(stream.cuda_stream))
    if rc != 0:
        raise RuntimeError(f"cudaMemcpy2DAsync failed: {rc}")


class L2Flush:
    """Writes a buffer twice the size of L2 (at least 256 MB), outside any
    timed region, so the next launch finds none of its inputs in L2."""

    def __init__(self, dev):
        import torch
        l2 = 0
        try:
            l2 = int(torch.cuda.get_device_properties(dev).L2_cache_size)
        except Exception:
            pass
        self.buf = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device=dev)
        self.n = 0

    def __call__(self, *_):
        self.n += 1
        self.buf.fill_(self.n & 0xFF)


# ---------------------------------------------------------------------------
# the oracle on the host (cpu_baseline leg and --impl reference)
# ---------------------------------------------------------------------------

def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_step_sample(heads, q, k, v, lengths, meta, prepacked):
    """One oracle step on the sampled (b, h_kv) heads: pack the group(s) of
    the step's new tokens, decode the head, attend its query heads' rows.
    Returns bytes counted with the same accounting as the GPU step."""
    import oracle as O
    grp = meta["H_q"] // meta["H_kv"]
    bits, g, d, lq = meta["bits"], meta["group"], meta["D"], meta["Lq"]
    uniform = bool(np.all(np.asarray(lengths) == meta["N"]))
    nbytes = 0
    for (b, h) in heads:
        n = int(lengths[b])
        t0 = (n - lq) // g * g
        if uniform:
            O.pack_k(k[b, h, t0:n], bits, g)
            O.pack_v(v[b, h, n - lq:n], bits, g)
        pk, pv = prepacked[(b, h)]
        kh, vh = O.unpack_matrix(pk), O.unpack_matrix(pv)
        rows = q[b, h * grp:(h + 1) * grp].reshape(grp * lq, d)
        O.attend_gqa_heads(rows, kh, vh, n, 1.0)
        nbytes += attend_bytes(1, grp, 1, d, [n], bits, g, lq=lq)
        if uniform:
            nbytes += append_bytes(1, 1, d, n - t0, lq, bits, g)
    return nbytes


def cpu_oracle_rate(q, k, v, lengths, meta, n_heads: int, repeats: int = 1, min_seconds: float = 0.0,
                    max_repeats: int = 30):
    """Bytes and per-pass seconds of the oracle over a sample of n_heads
    (b, h_kv) heads: `repeats` passes, more (up to max_repeats) until the
    passes add up to min_seconds."""
    import oracle as O
    rng = np.random.default_rng(123)
    all_heads = [(b, h) for b in range(meta["B"]) for h in range(meta["H_kv"])]
    idx = rng.choice(len(all_heads), size=min(n_heads, len(all_heads)), replace=False)
    heads = [all_heads[i] for i in sorted(idx)]
    pre = {(b, h): (O.pack_k(k[b, h], meta["bits"], meta["group"]),
                    O.pack_v(v[b, h], meta["bits"], meta["group"])) for (b, h) in heads}
    times, nbytes = [], 0
    oracle_step_sample(heads[:1], q, k, v, lengths, meta, pre)   # warm
    while len(times) < repeats or (sum(times) < min_seconds and len(times) < max_repeats):
        t = time.perf_counter()
        nbytes = oracle_step_sample(heads, q, k, v, lengths, meta, pre)
        times.append(time.perf_counter() - t)
    return nbytes, times, heads


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def run_kvq(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import sm_b200 as K

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    workload = args.workload
    q_np, k_np, v_np, lens_np, meta = W.gqa_case(workload, rank_seed(rank))
    q_np = torch.from_numpy(q_np).to(torch.bfloat16).float().numpy()
    B, H_q, H_kv, D, N, Lq = meta["B"], meta["H_q"], meta["H_kv"], meta["D"], meta["N"], meta["Lq"]
    bits = args.bits if args.bits else (meta["bits"] if isinstance(meta["bits"], int) else 4)
    meta["bits"] = bits
    if args.group:
        meta["group"] = args.group
    g = meta["group"]
    uniform = bool(np.all(lens_np == N))
    # --window W: the last W tokens of each sequence stay unquantized (bf16)
    # in a recent-token window; the packed cache holds the tokens before them
    W_win = int(args.window)
    causal = bool(args.causal)
    append = uniform and not W_win and not causal
    # the step's append: the K group(s) holding the new tokens (re-packed from a
    # float32 recent-token window) and the new tokens' V rows; only when every
    # sequence has the same length, since one kvq_pack call covers one range
    t0 = (N - Lq) // g * g
    v0 = N - Lq

    caches = []
    kd = torch.from_numpy(k_np).to(dev)
    vd = torch.from_numpy(v_np).to(dev)
    for _ in range(2):
        c = K.PackedCache(B, H_kv, N, D, bits, g, dev)
        K.pack(kd, vd, c)
        caches.append(c)
    win_k = kd[:, :, t0:N].contiguous()          # K of the new tokens' groups (recent-token window)
    new_v = vd[:, :, v0:N].contiguous()          # V of the new tokens
    del kd, vd
    qd = torch.from_numpy(q_np).to(dev).to(torch.bfloat16)
    lens = torch.from_numpy(lens_np).to(dev)
    out = torch.empty_like(qd)
    if W_win:
        wl_np = np.minimum(lens_np, W_win).astype(np.int32)
        lens_p_np = (lens_np - wl_np).astype(np.int32)
        kw_np = np.zeros((B, H_kv, W_win, D), np.float32)
        vw_np = np.zeros((B, H_kv, W_win, D), np.float32)
        for b in range(B):
            n, w = int(lens_np[b]), int(wl_np[b])
            kw_np[b, :, :w] = k_np[b, :, n - w:n]
            vw_np[b, :, :w] = v_np[b, :, n - w:n]
        kwin = torch.from_numpy(kw_np).to(dev).to(torch.bfloat16)
        vwin = torch.from_numpy(vw_np).to(dev).to(torch.bfloat16)
        lens = torch.from_numpy(lens_p_np).to(dev)
        wlens = torch.from_numpy(wl_np).to(dev)
        ws_need = K.workspace_size_window(caches[0], H_q, Lq)
    else:
        ws_need = K.workspace_size(caches[0], H_q, Lq)
    ws = torch.empty(max(ws_need, 16), dtype=torch.uint8, device=dev)

    def attend_call(c):
        if W_win:
            K.attend_window(qd, c, lens, kwin, vwin, wlens, 1.0, out=out, workspace=ws)
        else:
            K.attend(qd, c, lens, 1.0, out=out, workspace=ws, causal=causal)
    torch.cuda.synchronize()
    K.check(dev)

    # one decode step per sequence (Lq = 1): kvq_decode_step re-packs the
    # K group of the new token and packs its V row in one kernel, then
    # attends; the multi-query chunk appends its Lq tokens with kvq_pack
    decode_step = append and Lq == 1

    def step(i):
        c = caches[i & 1]
        if decode_step:
            K.decode_step(qd, c, lens, win_k, new_v, 1.0, out=out, workspace=ws)
            return
        if append:
            K.pack(win_k, None, c, t0=t0)
            K.pack(None, new_v, c, t0=v0)
        attend_call(c)

    def attend_only(i):
        attend_call(caches[i & 1])

    stream = torch.cuda.current_stream(dev)
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()

    # The kernel-only region replays CUDA graphs of one step (append + attend
    # on cache 0, then on cache 1), so host launch overhead does not pace it.
    def capture(fn):
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            fn()
        stream.wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        n0 = K.launch_count()
        with torch.cuda.graph(g, stream=side):
            fn()
        torch.cuda.synchronize()
        return g, K.launch_count() - n0

    step_graphs = [capture(lambda i=i: step(i)) for i in range(2)]
    attend_graphs = [capture(lambda i=i: attend_only(i)) for i in range(2)]
    launches_per_step = step_graphs[0][1]
    for i in range(args.warmup):
        step_graphs[i & 1][0].replay()
        attend_graphs[i & 1][0].replay()
    torch.cuda.synchronize()

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with sampler:
        start.record(stream)
        for i in range(args.steps):
            step_graphs[i & 1][0].replay()
        end.record(stream)
        torch.cuda.synchronize()
    launches = launches_per_step * args.steps
    if world > 1:
        dist.barrier()
    K.check(dev)
    ms = start.elapsed_time(end)

    # the attend alone, for the roofline: at least 50 replays, each timed by
    # its own events, the two caches in turn (each larger than L2)
    n_att = max(50, args.steps)
    attend_us = event_times_us(lambda i: attend_graphs[i & 1][0].replay(), n_att, stream)
    attend_dist = distribution(attend_us)
    attend_ms = [attend_dist["median"] / 1e3]

    # end-to-end through the public API (direct calls, no graphs): every step
    # copies its inputs from pinned host buffers and reads its output back,
    # pipelined the way a serving loop runs it -- a copy stream brings step
    # i + 1's inputs into the other of two device input sets while step i
    # computes, and reads step i's output back once it is done.
    q_host = torch.from_numpy(q_np).to(torch.bfloat16).pin_memory()
    kv_host_k = win_k[:, :, -Lq:].cpu().pin_memory()
    kv_host_v = new_v.cpu().pin_memory()
    o_host = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    q_in = [qd, qd.clone()]
    k_in = [win_k, win_k.clone()]
    v_in = [new_v, new_v.clone()]
    o_dev = [out, out.clone()]
    copy_stream = torch.cuda.Stream(dev)

    def e2e_step(i, ready, done, out_read):
        j = i & 1
        c = caches[j]
        stream.wait_event(ready[j])
        if i >= 2:
            stream.wait_event(out_read[j])                # step i - 2's output has been read back
        if decode_step:
            K.decode_step(q_in[j], c, lens, k_in[j], v_in[j], 1.0, out=o_dev[j], workspace=ws)
            done[j].record(stream)
            return
        if append:
            K.pack(k_in[j], None, c, t0=t0)
            K.pack(None, v_in[j], c, t0=v0)
        if W_win:
            K.attend_window(q_in[j], c, lens, kwin, vwin, wlens, 1.0, out=o_dev[j], workspace=ws)
        else:
            K.attend(q_in[j], c, lens, 1.0, out=o_dev[j], workspace=ws, causal=causal)
        done[j].record(stream)

    def e2e_copies(i, n, ready, done, out_read):
        # on the copy stream: read back step i - 1's output, then bring in
        # step i + 1's inputs (its input set was last used by step i - 1)
        with torch.cuda.stream(copy_stream):
            if i >= 1:
                jo = (i - 1) & 1
                copy_stream.wait_event(done[jo])
                o_host[jo].copy_(o_dev[jo], non_blocking=True)
                out_read[jo].record(copy_stream)
            if i + 1 < n:
                jn = (i + 1) & 1
                q_in[jn].copy_(q_host, non_blocking=True)
                if append:
                    copy_rows_h2d(k_in[jn][:, :, -Lq:], kv_host_k, copy_stream)
                    v_in[jn].copy_(kv_host_v, non_blocking=True)
                ready[jn].record(copy_stream)

    def e2e_run(n):
        ready = [torch.cuda.Event(), torch.cuda.Event()]
        done = [torch.cuda.Event(), torch.cuda.Event()]
        out_read = [torch.cuda.Event(), torch.cuda.Event()]
        with torch.cuda.stream(copy_stream):
            q_in[0].copy_(q_host, non_blocking=True)
            if append:
                copy_rows_h2d(k_in[0][:, :, -Lq:], kv_host_k, copy_stream)
                v_in[0].copy_(kv_host_v, non_blocking=True)
            ready[0].record(copy_stream)
        for i in range(n):
            e2e_copies(i, n, ready, done, out_read)
            e2e_step(i, ready, done, out_read)
        with torch.cuda.stream(copy_stream):
            copy_stream.wait_event(done[(n - 1) & 1])
            o_host[(n - 1) & 1].copy_(o_dev[(n - 1) & 1], non_blocking=True)

    # at least 200 timed steps, so the pipeline's fill and drain (the first
    # step's inputs, the last step's read-back) weigh little in the per-step time
    n_e2e = max(args.steps, 200)
    e2e_run(max(3, args.warmup))
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    copy_stream.wait_stream(stream)
    e2e_run(n_e2e)
    stream.wait_stream(copy_stream)
    e_end.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e_start.elapsed_time(e_end)
    h2d = q_host.numel() * 2 + ((kv_host_k.numel() + kv_host_v.numel()) * 4 if append else 0)
    d2h = o_host[0].numel() * 2

    if W_win:
        # packed tokens as usual plus the window's bf16 K and V rows
        abytes = attend_bytes(B, H_q, H_kv, D, lens_p_np, bits, g, lq=Lq) + H_kv * D * 2 * 2 * int(np.sum(wl_np))
    else:
        abytes = attend_bytes(B, H_q, H_kv, D, lens_np, bits, g, lq=Lq)
    step_bytes = abytes + (append_bytes(B, H_kv, D, N - t0, Lq, bits, g) if append else 0)
    if causal:
        # row i of a chunk reads L - Lq + i + 1 keys
        attend_flops = 4 * H_q * D * int(sum(Lq * (int(n) - Lq) + Lq * (Lq + 1) // 2 for n in lens_np))
    else:
        attend_flops = 4 * H_q * Lq * D * int(np.sum(lens_np.astype(np.int64)))
    ms_max, e2e_max = max_over_ranks([ms, e2e_ms], world, dev)

    res = None
    if rank == 0:
        per_step_ms = ms_max / args.steps
        value = whole_job_rate(step_bytes, world, per_step_ms) / 1e9
        e2e_value = whole_job_rate(step_bytes, world, e2e_max / n_e2e) / 1e9
        att_ms = statistics.mean(attend_ms)
        tensor = workload == "chunk"
        if tensor:
            achieved = attend_flops / (att_ms * 1e-3) / 1e12
            peak, peak_kind = measured_peaks("tensor")
        else:
            achieved = abytes / (att_ms * 1e-3) / 1e9
            peak, peak_kind = measured_peaks("hbm")
        kname = K.kernel_name(caches[0], H_q, Lq)
        src = os.path.join(ROOT, "sm_b200", "csrc",
                           "attend_decode.cu" if kname.startswith("decode") else
                           "attend_chunk.cu" if kname.startswith("chunk") else "attend_generic.cu")
        res = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(per_step_ms, 6),
            "us_per_step": round(per_step_ms * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "storage": f"u{bits} codes + f32 scales (group {g}), bf16 Q/O",
            "data": "synthetic",
            "config": {"workload": workload, "B": B, "H_q": H_q, "H_kv": H_kv, "d_h": D,
                       "context": N if uniform else "per-sequence", "lengths_sum": int(np.sum(lens_np)),
                       "bits": bits, "group": g, "lq": Lq,
                       "step": ("kvq_decode_step: append (re-pack the K group of each sequence's new token, "
                                "pack its V row; one kernel) + attend" if decode_step else
                                "append (re-pack the K group(s) of the new tokens, pack their V rows) + attend"
                                if append else
                                f"attend over the packed tokens and a {W_win}-token bf16 window" if W_win else
                                "causal attend (the Lq rows are each sequence's last positions)" if causal else
                                "attend (per-sequence lengths; no shared append range)"),
                       "window": W_win, "causal": causal,
                       "l2": f"inputs larger than L2: 2 packed caches of {caches[0].nbytes() / 1e6:.0f} MB used in turn",
                       "parallelism": f"independent batch per GPU x{world}",
                       "attend_kernel": kname, "step_bytes": step_bytes,
                       "launch": "CUDA graph per step"},
            "pct_of_8tbs": round(100 * value / world / 8000.0, 2),
            "roofline": {"bound": "tensor" if tensor else "hbm", "achieved": round(achieved, 1 if not tensor else 2),
                         "peak": peak, "unit": "TFLOP/s" if tensor else "GB/s",
                         "frac": round(achieved / peak, 4),
                         "peak_source": ("bf16_tflops (burst) of " if tensor else "hbm_gbs of ") + peak_kind,
                         "kernel": f"kvq_attend ({kname})", "attend_us": round(att_ms * 1e3, 3),
                         "attend_us_dist": attend_dist,
                         "timing": f"median of {n_att} attend-only CUDA-graph replays, each timed by its own "
                                   "events, the two caches in turn",
                         "algorithmic_bytes_per_launch": abytes,
                         "algorithmic_flops_per_launch": attend_flops,
                         "attend_gbs": round(abytes / (att_ms * 1e-3) / 1e9, 1),
                         "traffic": recorded_traffic(src, workload, bits, g, W_win or int(causal))},
            "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "us_per_step": round(e2e_max / n_e2e * 1e3, 3), "steps": n_e2e,
                    "pipeline": "inputs copied on a second stream into two alternating device sets, "
                                "outputs read back as each step finishes"},
            "gpu_launches": int(launches),
            "clocks": sampler.summary(),
            "impl": "kvq",
        }
    return res, (q_np, k_np, v_np, lens_np, meta)


# ---------------------------------------------------------------------------
# the other configurations: attend-only device times for the record
# ---------------------------------------------------------------------------

def capture_graph(K, fn, dev, stream):
    """A CUDA graph of fn() (warmed once on a side stream) and the number of
    library kernels it launches."""
    import torch
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        fn()
    stream.wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    n0 = K.launch_count()
    with torch.cuda.graph(g, stream=side):
        fn()
    torch.cuda.synchronize()
    return g, K.launch_count() - n0


def study_gqa(K, dev, stream, flush, workload: str, bits: int, n_rep: int = 50):
    """Attend-only device time of a GQA workload at full size (one cache,
    every replay after an L2 flush) with its roofline fraction: HBM bytes for
    the decode shapes, bf16 tensor FLOPs for the multi-query chunk."""
    import torch
    q_np, k_np, v_np, lens_np, meta = W.gqa_case(workload, SEED)
    B, H_q, H_kv, D, N, Lq, g = meta["B"], meta["H_q"], meta["H_kv"], meta["D"], meta["N"], meta["Lq"], meta["group"]
    cache = K.PackedCache(B, H_kv, N, D, bits, g, dev)
    kd = torch.from_numpy(k_np).to(dev)
    vd = torch.from_numpy(v_np).to(dev)
    K.pack(kd, vd, cache)
    del kd, vd, k_np, v_np
    qd = torch.from_numpy(q_np).to(dev).to(torch.bfloat16)
    lens = torch.from_numpy(lens_np).to(dev)
    out = torch.empty_like(qd)
    ws = torch.empty(max(K.workspace_size(cache, H_q, Lq), 16), dtype=torch.uint8, device=dev)
    graph, launches = capture_graph(K, lambda: K.attend(qd, cache, lens, 1.0, out=out, workspace=ws), dev, stream)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    d = distribution(event_times_us(lambda i: graph.replay(), n_rep, stream, between=flush))
    K.check(dev)
    med_s = d["median"] * 1e-6
    abytes = attend_bytes(B, H_q, H_kv, D, lens_np, bits, g, lq=Lq)
    flops = 4 * H_q * Lq * D * int(np.sum(lens_np.astype(np.int64)))
    src = os.path.join(ROOT, "sm_b200", "csrc", "attend_chunk.cu" if Lq > 1 else "attend_decode.cu")
    res = {"attend_us": d, "kernel": K.kernel_name(cache, H_q, Lq), "launches_per_attend": launches,
           "traffic": recorded_traffic(src, workload, bits, g),
           "bits": bits, "group": g, "B": B, "H_q": H_q, "H_kv": H_kv, "d_h": D, "lq": Lq,
           "lengths_sum": int(np.sum(lens_np)), "algorithmic_bytes": abytes, "flops": flops,
           "gbs": round(abytes / med_s / 1e9, 1)}
    if Lq > 1:
        peak, kind = measured_peaks("tensor")
        tf = flops / med_s / 1e12
        res.update({"tflops": round(tf, 2), "frac": round(tf / peak, 4), "bound": "tensor",
                    "peak": peak, "peak_source": f"bf16_tflops (burst) of {kind}"})
    else:
        peak, kind = measured_peaks("hbm")
        res.update({"frac": round(abytes / med_s / 1e9 / peak, 4), "bound": "hbm", "peak": peak,
                    "peak_source": f"hbm_gbs of {kind}", "pct_of_8tbs": round(100 * abytes / med_s / 8e12, 2)})
    del cache, qd, out, ws, graph
    torch.cuda.empty_cache()
    return res


def study_single_head(K, dev, stream, flush, n_rep: int = 50):
    """The single-head configurations (one head, 4 queries, D 32, N 128 and
    512, every code width and group size): device µs of one attend, each
    replay after an L2 flush.  They are launch-latency bound."""
    import torch
    out = {}
    for n in (128, 512):
        q, k, v = W.single_head(n, 32, 4, SEED, "clean")
        for bits, g in W.FORMATS:
            cache = K.PackedCache(1, 1, n, 32, bits, g, dev)
            K.pack(torch.from_numpy(k[None, None]).to(dev), torch.from_numpy(v[None, None]).to(dev), cache)
            qd = torch.from_numpy(q[None, None]).to(dev)
            lens = torch.tensor([n], dtype=torch.int32, device=dev)
            o = torch.empty_like(qd)
            ws = torch.empty(max(K.workspace_size(cache, 1, 4), 16), dtype=torch.uint8, device=dev)
            graph, _ = capture_graph(K, lambda: K.attend(qd, cache, lens, 1.0 / math.sqrt(32), out=o, workspace=ws),
                                     dev, stream)
            for _ in range(3):
                graph.replay()
            d = distribution(event_times_us(lambda i: graph.replay(), n_rep, stream, between=flush))
            out[f"n{n}_b{bits}_g{g}"] = {"median": d["median"], "p10": d["p10"], "p90": d["p90"], "n": d["n"],
                                         "kernel": K.kernel_name(cache, 1, 4)}
    K.check(dev)
    return out


def oracle_single_head_protocol():
    """The pages' CPU timing protocol on the oracle ("Block KV decoding: less
    workspace, more time", section "CPU timing retains the negative result"):
    the 18 single-head inputs (N 128 and 512, seeds 0-2, clean / early / late)
    at 4-bit g32, three methods -- attention over the float32 cache, decode
    everything then attend, decode and merge 32-token blocks -- each input
    with 3 warm-up and 15 measured rounds in rotated method order; the
    median µs per (N, method) over every observation, which are all kept."""
    import oracle as O
    scale = 1.0 / math.sqrt(32)
    methods = {
        "float32_cache": lambda q, k, v, pk, pv: O.attend_dense(q, k, v, scale),
        "decode_all_then_attend": lambda q, k, v, pk, pv: O.attend_dense(q, O.unpack_matrix(pk),
                                                                         O.unpack_matrix(pv), scale),
        "decode_and_merge_blocks": lambda q, k, v, pk, pv: O.attend_blocked_packed(q, pk, pv, scale, 32),
    }
    names = list(methods)
    obs = {(n, m): [] for n in (128, 512) for m in names}
    for n, seed, dist in W.SINGLE_HEAD_GRID:
        q, k, v = W.single_head(n, 32, 4, seed, dist)
        pk, pv = O.pack_k(k, 4, 32), O.pack_v(v, 4, 32)
        for r in range(3 + 15):
            order = names[r % 3:] + names[:r % 3]
            for m in order:
                t = time.perf_counter()
                methods[m](q, k, v, pk, pv)
                dt = (time.perf_counter() - t) * 1e6
                if r >= 3:
                    obs[(n, m)].append(dt)
    return {f"n{n}": {m: round(float(np.median(obs[(n, m)])), 1) for m in names} for n in (128, 512)} | {
        "observations": sum(len(x) for x in obs.values()), "cores": blas_threads(),
        "protocol": "18 inputs x 3 methods x 15 rounds (after 3 warm-ups), method order rotated each round, "
                    "median per (N, method)"}


def run_studies(K, dev, stream):
    flush = L2Flush(dev)
    res = {"timing": "attend-only CUDA-graph replays, each timed by its own events after an L2 flush"}
    res["long_context"] = study_gqa(K, dev, stream, flush, "long_context", 4)
    res["chunk_4bit"] = study_gqa(K, dev, stream, flush, "chunk", 4)
    res["chunk_8bit"] = study_gqa(K, dev, stream, flush, "chunk", 8)
    res["single_head_us"] = study_single_head(K, dev, stream, flush)
    del flush
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["kvq", "reference"], default="kvq")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-studies", action="store_true",
                    help="skip the attend-only timings of the other configurations (long context, chunk, "
                         "single head) that the default run adds to its JSON line")
    ap.add_argument("--cpu-heads", type=int, default=256,
                    help="(b, h_kv) heads in the oracle's timed sample")
    ap.add_argument("--workload", choices=sorted(W.WORKLOADS), default=WORKLOAD,
                    help="the decode GQA workload is the headline; the others are for study")
    ap.add_argument("--bits", type=int, choices=[4, 8], default=0,
                    help="code width (default: the workload's, 4 for the chunk workload)")
    ap.add_argument("--group", type=int, choices=[8, 32], default=0,
                    help="scale group size (default: the workload's, 32)")
    ap.add_argument("--causal", action="store_true",
                    help="causal rows (kvq_attend_causal): the Lq query rows are each sequence's last "
                         "positions; for the multi-query chunk workload")
    ap.add_argument("--window", type=int, default=0,
                    help="keep the last W tokens of each sequence unquantized (bf16) in a recent-token "
                         "window (kvq_attend_window); 0 = none")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if args.window or args.causal:
            ap.error("--window and --causal are studies of the kvq arm; the reference arm times the "
                     "oracle on the plain workload")
        if rank != 0:
            return 0
        q, k, v, lens, meta = W.gqa_case(args.workload, SEED)
        import torch
        q = torch.from_numpy(q).to(torch.bfloat16).float().numpy()
        if args.bits or not isinstance(meta["bits"], int):
            meta["bits"] = args.bits or 4
        if args.group:
            meta["group"] = args.group
        per_step = max(4, args.cpu_heads // 4)
        total, times = 0, []
        for _ in range(args.warmup):
            cpu_oracle_rate(q, k, v, lens, meta, per_step)
        for _ in range(args.steps):
            nb, ts, heads = cpu_oracle_rate(q, k, v, lens, meta, per_step)
            total += nb
            times.append(sum(ts))
        value = total / sum(times) / 1e9
        line = {
            "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * sum(times) / len(times), 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": args.workload, "B": meta["B"], "H_q": meta["H_q"],
                       "H_kv": meta["H_kv"], "d_h": meta["D"],
                       "context": meta["N"] if bool(np.all(lens == meta["N"])) else "per-sequence",
                       "lengths_sum": int(np.sum(lens)),
                       "bits": meta["bits"], "group": meta["group"], "lq": meta["Lq"]},
            "impl": "reference",
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": blas_threads(),
                             "kind": "oracle",
                             "sample": f"{per_step} of {meta['B'] * meta['H_kv']} (b, h_kv) heads per step"},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line))
        return 0

    import torch
    import torch.distributed as dist
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    res, data = run_kvq(args, rank, world, local_rank)
    plain = not args.window and not args.causal and not args.bits and not args.group
    if rank == 0 and world == 1 and plain and args.workload == WORKLOAD and not args.no_studies:
        dev = torch.device("cuda", local_rank)
        res["studies"] = run_studies(__import__("sm_b200"), dev, torch.cuda.current_stream(dev))
        if not args.no_cpu_baseline:
            res["studies"]["single_head_oracle_host_us"] = oracle_single_head_protocol()
    if rank == 0 and not args.no_cpu_baseline and not args.window and not args.causal:
        q, k, v, lens, meta = data
        nb, ts, heads = cpu_oracle_rate(q, k, v, lens, meta, args.cpu_heads, repeats=3, min_seconds=10.0)
        rate = nb / statistics.median(ts) / 1e9
        res["cpu_baseline"] = {"value": round(rate, 4), "unit": "GB/s", "cores": blas_threads(),
                               "kind": "oracle",
                               "sample": f"{len(heads)} of {meta['B'] * meta['H_kv']} (b, h_kv) heads per pass "
                                         f"(the append + attend of the step for those heads), median of "
                                         f"{len(ts)} passes ({statistics.median(ts):.2f} s each, "
                                         f"{sum(ts):.1f} s in all)"}
    if rank == 0:
        print(json.dumps(res))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
