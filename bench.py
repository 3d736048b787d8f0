"""Benchmark: paged decode attention KV-read GB/s on the Qwen3-4B-shaped decode
batch (64 slots, 32/8 heads, d=128, page 16, lengths U[128,4096]), plus the
other workloads (mixed prefill+decode tokens/s, long-context split-K,
fragmented large batch, tiny decode).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workloads all|none|name,...]

A step is one pass of the hot path over one batch: kv_append of the step's new
K/V rows, then attention (chunked prefill for prompt chunks, decode with its
split-K partition and in-kernel merge for decode rows); a decode-only batch
appends and decodes in one launch (pkv_paged_attn_decode_append).  Inputs are resident in HBM
when the timed region starts; the KV a step reads is larger than the 126 MB
L2, so no flush is needed between steps.  Under torchrun each rank runs its
own batch (requests shard across GPUs with no data-path collective: weak
scaling); the step time is the max over ranks.

--impl reference times the CPU oracle (the plain fp64 definition) on a
bounded sample of the same workload, as the reference arm.
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
sys.path.insert(0, ROOT)

from workloads import make_workload  # noqa: E402

HBM_NOMINAL_GBS = 8000.0
FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS = 6650.0, 1590.0
METRIC = "paged decode attention KV-read GB/s (% of 8 TB/s HBM); mixed-batch tokens/s"
HEADLINE = "qwen3_decode"


def profiled_traffic(key):
    """DRAM bytes (read + write) per launch of a kernel, from the ncu capture
    recorded in profiles/traffic.json -- or None when the kernel's source has
    changed since that capture (its sha256 no longer matches)."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)[key]
        with open(os.path.join(ROOT, rec["source"]), "rb") as f:
            digest = hashlib.sha256(f.read()).hexdigest()
    except (OSError, KeyError, ValueError):
        return None
    return rec["dram_bytes_per_launch"] if digest == rec["source_sha256"] else None


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index):
        self.index, self.samples, self.reasons, self.max_mhz = index, [], set(), None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # NVML missing: record why
            self.nv, self.err = None, str(e)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                mask = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        if self.nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# --------------------------------------------------------------- GPU side
class Packed:
    """Tensors of the given (dtype, shape) as views into one byte buffer, each
    at a 256-byte aligned offset; pinned when on the host."""

    def __init__(self, torch, specs, device):
        offs, n = {}, 0
        for k, (dt, shape) in specs.items():
            offs[k] = n
            nb = int(np.prod(shape)) * torch.empty((), dtype=dt).element_size()
            n += (nb + 255) // 256 * 256
        self.buf = torch.empty(max(n, 256), dtype=torch.uint8, device=device)
        if device == "cpu":
            self.buf = self.buf.pin_memory()
        self.views = {}
        for k, (dt, shape) in specs.items():
            nb = int(np.prod(shape)) * torch.empty((), dtype=dt).element_size()
            self.views[k] = self.buf[offs[k]:offs[k] + nb].view(dt).view(shape)


def fusable_decode_step(w, slots) -> bool:
    """True when a step of workload w is decode only and its new rows (with
    slot mapping `slots`, in request order) are one per request, each at its
    request's position kv_lens - 1: the rows pkv_paged_attn_decode_append
    appends itself."""
    dec, pre = list(w.decode_ids), list(w.prefill_ids)
    if pre or len(dec) != w.B or len(slots) != len(dec) or not bool((w.kv_lens[dec] > 0).all()):
        return False
    last = np.array([int(w.page_table[r][(int(w.kv_lens[r]) - 1) // w.page_size]) * w.page_size
                     + (int(w.kv_lens[r]) - 1) % w.page_size for r in dec], np.int64)
    return bool(np.array_equal(np.asarray(slots, np.int64), last))


class GpuWorkload:
    """Device buffers for one workload: pools with every request's context
    (drawn on the GPU, seeded), and the step's inputs (host-generated)."""

    def __init__(self, pkv, torch, w, seed=4321):
        self.pkv, self.torch, self.w = pkv, torch, w
        dev = "cuda"
        self.k_pool = torch.full(w.pool_shape(), float("nan"), dtype=torch.bfloat16, device=dev)
        self.v_pool = torch.full_like(self.k_pool, float("nan"))
        gen = torch.Generator(device=dev).manual_seed(seed)
        ids = list(range(w.B))
        at = 0
        while at < len(ids):
            grp, toks = [], 0
            while at < len(ids) and (not grp or toks < (1 << 18)):
                grp.append(ids[at]); toks += int(w.ctx_lens[ids[at]]); at += 1
            slots = w.ctx_slots(grp)
            if len(slots):
                k = torch.randn((len(slots), w.num_kv_heads, w.head_dim), generator=gen, device=dev)
                if w.k_rms_norm:
                    k = k / k.pow(2).mean(-1, keepdim=True).sqrt()
                v = torch.randn((len(slots), w.num_kv_heads, w.head_dim), generator=gen, device=dev)
                pkv.pkv_kv_append(k.bfloat16().contiguous(), v.bfloat16().contiguous(),
                                  self.i32(slots), self.k_pool, self.v_pool)
        # step inputs, as host arrays (pinned for the end-to-end leg) and device copies
        k, v, s = w.batch_new()
        dec, pre = list(w.decode_ids), list(w.prefill_ids)
        self.host = {
            "k_new": self.bits(k), "v_new": self.bits(v), "slots": torch.from_numpy(s),
            "pt_dec": torch.from_numpy(np.ascontiguousarray(w.page_table[dec])),
            "len_dec": torch.from_numpy(np.ascontiguousarray(w.kv_lens[dec])),
        }
        if dec:
            self.host["q_dec"] = self.bits(w.batch_q(dec))
        if pre:
            self.host.update({
                "q_pre": self.bits(w.batch_q(pre)),
                "cu_q": torch.from_numpy(w.cu_q_lens(pre)),
                "ctx_pre": torch.from_numpy(np.ascontiguousarray(w.ctx_lens[pre])),
                "pt_pre": torch.from_numpy(np.ascontiguousarray(w.page_table[pre])),
            })
        # every step input lives in one pinned host buffer and in each of two
        # device buffers (views at 256-byte aligned offsets): the end-to-end
        # leg moves a step's inputs with a single copy, double-buffered
        specs = {k: (t.dtype, tuple(t.shape)) for k, t in self.host.items()}
        hin = Packed(torch, specs, "cpu")
        for k, t in self.host.items():
            hin.views[k].copy_(t)
        self.in_host = hin
        self.in_dev = [Packed(torch, specs, dev) for _ in range(2)]
        for d in self.in_dev:
            d.buf.copy_(hin.buf)
        self.host = hin.views
        self.dev = self.in_dev[0].views
        self.dev_sets = [d.views for d in self.in_dev]
        self.dec, self.pre = dec, pre
        # a decode-only step whose new rows are one per request, each at its
        # request's position kv_lens - 1, is appended and decoded in one
        # launch (pkv_paged_attn_decode_append)
        self.fused = fusable_decode_step(w, s)
        self.max_q = int(w.new_lens[pre].max()) if pre else 0
        if dec:
            self.ws = pkv.decode_workspace(len(dec), w.num_q_heads, w.head_dim,
                                           w.max_pages * w.page_size, 0)
        if pre and w.notes.get("attention") == "verify":
            self.vws = pkv.verify_workspace(int(w.new_lens[pre].sum()), w.num_q_heads, w.head_dim,
                                            w.max_pages * w.page_size, 0)
        # outputs: one packed device buffer per set, read back with one copy
        ospecs = {}
        if dec:
            ospecs["dec"] = (torch.bfloat16, tuple(self.dev["q_dec"].shape))
        if pre:
            ospecs["pre"] = (torch.bfloat16, tuple(self.dev["q_pre"].shape))
        self.out_dev = [Packed(torch, ospecs, dev) for _ in range(2)]
        self.out_host = [Packed(torch, ospecs, "cpu") for _ in range(2)]
        self.out_sets = [d.views for d in self.out_dev]
        if dec:
            self.out_dec = self.out_sets[0]["dec"]
        if pre:
            self.out_pre = self.out_sets[0]["pre"]
        torch.cuda.synchronize()

    def bits(self, a):
        return self.torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(self.torch.bfloat16)

    def i32(self, a):
        return self.torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()

    def launches_per_step(self):
        # kv_append, the decode partition kernel (the automatic split merges
        # in-kernel, no combine launch), the prefill kernel; a fused decode
        # step is the partition kernel alone
        if self.fused:
            return 1
        return 1 + (1 if self.dec else 0) + (1 if self.pre else 0)

    def prefill_call(self, d=None, out=None):
        """The chunk rows' attention: chunked prefill, or for the verify
        workload the split-K short-chunk call."""
        d = self.dev if d is None else d
        out = self.out_pre if out is None else out
        if self.w.notes.get("attention") == "verify":
            self.pkv.pkv_paged_attn_verify(d["q_pre"], d["cu_q"], d["ctx_pre"], self.k_pool, self.v_pool,
                                           d["pt_pre"], self.w.scale, self.max_q, 0, workspace=self.vws, out=out)
        else:
            self.pkv.pkv_paged_attn_chunked_prefill(d["q_pre"], d["cu_q"], d["ctx_pre"], self.k_pool,
                                                    self.v_pool, d["pt_pre"], self.w.scale, self.max_q, out=out)

    def decode_call(self, d=None, out=None):
        d = self.dev if d is None else d
        # the kernel just ahead (the append, the prefill or, in the timing
        # loops, another decode) writes neither lengths nor page tables
        self.pkv.pkv_paged_attn_decode_flags(d["q_dec"], self.k_pool, self.v_pool, d["pt_dec"], d["len_dec"],
                                             self.w.scale, 0, workspace=self.ws,
                                             out=self.out_dec if out is None else out,
                                             flags=self.pkv.DECODE_METADATA_READY)

    def mixed_step(self, d=None):
        """kv_append, then the chunk rows and the decode rows in one
        persistent launch (pkv_paged_attn_mixed)."""
        d = self.dev if d is None else d
        self.pkv.pkv_kv_append(d["k_new"], d["v_new"], d["slots"], self.k_pool, self.v_pool)
        self.pkv.pkv_paged_attn_mixed(d["q_pre"], d["cu_q"], d["ctx_pre"], d["pt_pre"], self.max_q, d["q_dec"],
                                      d["pt_dec"], d["len_dec"], self.k_pool, self.v_pool, self.w.scale,
                                      workspace=self.ws, out_pre=self.out_pre, out_dec=self.out_dec)

    def step(self, d, outs=None):
        """One pass of the hot path on device buffers d: kv_append of the
        step's new rows, then the prefill and decode calls (for a decode-only
        step, both in one fused launch); outs picks the output buffers
        (default: the first set)."""
        if self.fused:
            # the kernel just ahead (the previous step's) writes neither
            # lengths nor page tables
            self.pkv.pkv_paged_attn_decode_append(
                d["q_dec"], d["k_new"], d["v_new"], self.k_pool, self.v_pool, d["pt_dec"], d["len_dec"],
                self.w.scale, 0, workspace=self.ws, out=outs["dec"] if outs is not None else self.out_dec,
                flags=self.pkv.DECODE_METADATA_READY)
            return
        self.pkv.pkv_kv_append(d["k_new"], d["v_new"], d["slots"], self.k_pool, self.v_pool)
        if self.pre:
            self.prefill_call(d, outs["pre"] if outs is not None else None)
        if self.dec:
            self.decode_call(d, outs["dec"] if outs is not None else None)

    def run_e2e(self, steps):
        """`steps` steps through the public API from pinned host buffers: every
        step copies its inputs host-to-device, runs the kernels and reads its
        outputs back.  Two buffer sets and a copy stream let the copies of one
        step overlap the kernels of its neighbours: step i+1's inputs are
        queued on the copy stream before step i's read-back (which waits for
        step i's kernels), so they land while step i computes.  The caller
        times the whole run on the current stream (it waits for the copy
        stream at the end)."""
        torch = self.torch
        main = torch.cuda.current_stream()
        cs = self._copy_stream = getattr(self, "_copy_stream", None) or torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        cs.wait_stream(main)

        def load(i):  # on the copy stream
            b = i & 1
            if i >= 2:
                cs.wait_event(ev_done[b])  # the kernels of step i-2 no longer read set b
            self.in_dev[b].buf.copy_(self.in_host.buf, non_blocking=True)
            ev_in[b].record(cs)

        with torch.cuda.stream(cs):
            if steps > 0:
                load(0)
        for i in range(steps):
            b = i & 1
            main.wait_event(ev_in[b])
            if i >= 2:
                main.wait_event(ev_out[b])  # step i-2's outputs have left set b
            self.step(self.dev_sets[b], outs=self.out_sets[b])
            ev_done[b].record(main)
            with torch.cuda.stream(cs):
                if i + 1 < steps:
                    load(i + 1)
                cs.wait_event(ev_done[b])
                self.out_host[b].buf.copy_(self.out_dev[b].buf, non_blocking=True)
                ev_out[b].record(cs)
        main.wait_stream(cs)

    def io_bytes(self):
        """Bytes copied per end-to-end step (packed buffers, alignment included)."""
        return self.in_host.buf.numel(), self.out_dev[0].buf.numel()


def prefill_flops(w):
    """QK^T and PV multiply-adds of the causal chunks (2 flops each)."""
    tot = 0
    for r in w.prefill_ids:
        c, n = int(w.ctx_lens[r]), int(w.new_lens[r])
        keys = n * c + n * (n + 1) // 2  # row i sees c + i + 1 keys
        tot += 4 * keys * w.num_q_heads * w.head_dim
    return tot


def max_over_ranks(dist, x, device="cuda"):
    """The largest of every rank's x (the timing rule for N replicas): an
    all-reduce MAX over the process group, or x itself without one."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([float(x)], device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_gbs(world, bytes_per_rank, ms):
    """Whole-job GB/s of `world` replicas that each move bytes_per_rank in ms."""
    return world * bytes_per_rank / (ms / 1e3) / 1e9


def emit(rank, line):
    """Print the JSON line on rank 0 only; True when printed."""
    if rank != 0:
        return False
    print(json.dumps(line))
    return True


def graph_ms(torch, body, steps, dist=None, clocks=None):
    """Milliseconds for `steps` calls of body(): the calls are captured once as
    one CUDA graph (nothing recorded between the kernels: an event between two
    launches would serialise them and cost the programmatic-dependent-launch
    overlap), replayed once untimed (the graph's upload), then one replay is
    timed with CUDA events, bracketed by a barrier and a synchronize, the max
    over ranks.  Returns (ms, None), or (None, why) when capture is refused."""
    graph = torch.cuda.CUDAGraph()
    try:
        with torch.cuda.graph(graph):
            for _ in range(steps):
                body()
        graph.replay()
        torch.cuda.synchronize()
    except Exception as e:  # noqa: BLE001
        return None, repr(e)[:200]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with (clocks if clocks is not None else _Null()):
        t0.record()
        graph.replay()
        t1.record()
        torch.cuda.synchronize()
    del graph
    return max_over_ranks(dist, t0.elapsed_time(t1)), None


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def eager_ms(torch, body, steps, dist=None, clocks=None):
    """The same as graph_ms with eager launches (where capture is refused)."""
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with (clocks if clocks is not None else _Null()):
        t0.record()
        for _ in range(steps):
            body()
        t1.record()
        torch.cuda.synchronize()
    return max_over_ranks(dist, t0.elapsed_time(t1))


def timed(torch, body, steps, dist=None, clocks=None):
    """(ms per call, how it was timed): one CUDA graph of the calls, else eager."""
    ms, why = graph_ms(torch, body, steps, dist, clocks)
    if ms is not None:
        return ms / steps, "one CUDA graph of the K calls, one replay timed"
    return eager_ms(torch, body, steps, dist, clocks) / steps, f"eager launches ({why})"


def measure(pkv, torch, name, steps, warmup, dist=None, clocks_index=0):
    w = make_workload(name, 0)
    g = GpuWorkload(pkv, torch, w)
    for _ in range(warmup):
        g.step(g.dev)
    torch.cuda.synchronize()
    # the whole step (kv_append, then prefill and/or decode), K times
    clk = ClockSampler(clocks_index)
    step_ms, timing = timed(torch, lambda: g.step(g.dev), steps, dist, clk)
    # each attention kernel alone, K back-to-back calls on the same inputs
    # (their reads exceed the L2, so no flush is needed between calls): the
    # kernel durations behind the rooflines
    dec_ms = pre_ms = None
    if g.dec:
        dec_ms, _ = timed(torch, g.decode_call, steps, dist)
    if g.pre:
        pre_ms, _ = timed(torch, g.prefill_call, steps, dist)
    mixed_ms = None
    if g.pre and g.dec and w.notes.get("attention") != "verify":
        mixed_ms, _ = timed(torch, g.mixed_step, steps, dist)
    # end-to-end through the public API with host buffers
    g.run_e2e(warmup)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    g.run_e2e(steps)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(dist, e0.elapsed_time(e1))
    flags = pkv.pkv_device_error_flags(clear=True)
    if flags:
        raise RuntimeError(f"device error flags {flags:#x} during {name}")
    h2d, d2h = g.io_bytes()
    res = {
        "w": w, "ms_per_step": step_ms, "e2e_ms_per_step": e2e_ms / steps,
        "dec_ms": dec_ms, "pre_ms": pre_ms, "mixed_ms": mixed_ms,
        "kv_bytes_dec": w.kv_bytes_read(w.decode_ids), "kv_bytes_pre": w.kv_bytes_read(w.prefill_ids),
        "tokens": int(w.new_lens.sum()), "flops_pre": prefill_flops(w),
        "launches": g.launches_per_step(), "clocks": clk.summary(), "h2d": h2d, "d2h": d2h,
        "timing": timing,
    }
    del g
    torch.cuda.empty_cache()
    return res


# --------------------------------------------------------------- CPU side
def _request_pool(oracle, w, r):
    """Request r's pages for the oracle: its context plus this step's rows, in
    a pool of just its pages (renumbered 0.. in table order)."""
    pages = w.page_table[r][w.page_table[r] >= 0]
    table = np.arange(len(pages), dtype=np.int32)[None, :]
    P = w.page_size
    kp = np.full((len(pages), w.num_kv_heads, P, w.head_dim), 0x7FC0, np.uint16)
    vp = kp.copy()
    L = int(w.kv_lens[r])
    pos = np.arange(L)
    slots = (pos // P) * P + pos % P
    kc, vc = w.ctx_rows(r)
    kn, vn = w.new_rows(r)
    oracle.kv_append(kp, vp, np.concatenate([kc, kn]), np.concatenate([vc, vn]), slots, P)
    return kp, vp, table


def _oracle_call(oracle, w, r, kind):
    """A closure that runs the oracle, as it stands, on request r: its decode
    attention, or the attention of its prefill chunk."""
    kp, vp, table = _request_pool(oracle, w, r)
    if kind == "decode":
        q, lens = w.q_rows(r)[None, 0], np.array([int(w.kv_lens[r])], np.int32)
        return lambda: oracle.decode_attention(q, kp, vp, table, lens, w.page_size, w.scale)
    q = w.q_rows(r)
    cu = np.array([0, len(q)], np.int32)
    ctx = np.array([int(w.ctx_lens[r])], np.int32)
    return lambda: oracle.chunked_prefill_attention(q, cu, ctx, kp, vp, table, w.page_size, w.scale)


def _crew_worker(name, kind, ids, barrier, conn):
    """One oracle process: builds its requests' inputs (untimed), then on each
    command waits at the barrier with the others and runs the oracle on the
    requests the command names, reporting (start, end) on the shared clock."""
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:  # noqa: BLE001
        pass
    import oracle
    w = make_workload(name, 0)
    calls = [_oracle_call(oracle, w, r, kind) for r in ids]
    conn.send("ready")
    while True:
        sel = conn.recv()
        if sel is None:
            break
        barrier.wait()
        t0 = time.perf_counter()
        for i in sel:
            calls[i]()
        conn.send((t0, time.perf_counter()))


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def work_units(w, r, kind):
    """(KV bytes, flops, query tokens) of request r for the oracle's rates."""
    if kind == "decode":
        return w.kv_bytes_read([r]), 0, 1
    c, n = int(w.ctx_lens[r]), int(w.new_lens[r])
    return w.kv_bytes_read([r]), 4 * (n * c + n * (n + 1) // 2) * w.num_q_heads * w.head_dim, n


class OracleCrew:
    """The CPU oracle, as it stands (never tuned), over whole requests of one
    workload, run by `procs` spawned processes with one numpy thread each.
    Requests are dealt to processes largest first; all processes start each
    run together (a barrier) and the run's time is from the first start to the
    last end."""

    def __init__(self, name, kind, procs):
        import multiprocessing as mp
        ctx = mp.get_context("spawn")
        w = make_workload(name, 0)
        ids = [int(r) for r in (w.decode_ids if kind == "decode" else w.prefill_ids)]
        size = {r: work_units(w, r, kind)[0] + work_units(w, r, kind)[1] for r in ids}
        procs = max(1, min(procs, len(ids)))
        groups, load = [[] for _ in range(procs)], [0] * procs
        for r in sorted(ids, key=lambda r: -size[r]):
            i = load.index(min(load))
            groups[i].append(r)
            load[i] += size[r]
        self.w, self.kind, self.groups = w, kind, groups
        self.barrier = ctx.Barrier(procs)
        self.pipes, self.procs = [], []
        for grp in groups:
            parent, child = ctx.Pipe()
            pr = ctx.Process(target=_crew_worker, args=(name, kind, grp, self.barrier, child), daemon=True)
            pr.start()
            self.pipes.append(parent)
            self.procs.append(pr)
        for c in self.pipes:
            assert c.recv() == "ready"

    def run(self, part=0, nparts=1):
        """Seconds for every process to run its requests (or the part-th of
        nparts slices of them); returns (seconds, units summed over the
        requests run)."""
        sel = [list(range(len(g)))[part::nparts] for g in self.groups]
        for c, sl in zip(self.pipes, sel):
            c.send(sl)
        spans = [c.recv() for c in self.pipes]
        secs = max(t1 for _, t1 in spans) - min(t0 for t0, _ in spans)
        units = np.zeros(3)
        for g, sl in zip(self.groups, sel):
            for i in sl:
                units += work_units(self.w, g[i], self.kind)
        return secs, units

    def close(self):
        for c in self.pipes:
            c.send(None)
        for pr in self.procs:
            pr.join(timeout=30)


def oracle_times(name, kind):
    """The oracle on the whole of one workload's decode or prefill requests,
    on one host thread and on every host core."""
    out = {}
    for label, procs in (("1_thread", 1), ("all_cores", host_cores())):
        crew = OracleCrew(name, kind, procs)
        try:
            secs, (nbytes, flops, toks) = crew.run()
        finally:
            crew.close()
        rec = {"seconds": secs, "processes": len(crew.groups)}
        if kind == "decode":
            rec.update({"kv_gbs": nbytes / secs / 1e9, "tokens_per_s": toks / secs})
        else:
            rec.update({"tflops": flops / secs / 1e12, "tokens_per_s": toks / secs})
        out[label] = rec
    out["sample"] = (f"all {len(make_workload(name, 0).decode_ids if kind == 'decode' else make_workload(name, 0).prefill_ids)}"
                     f" {kind} requests of {name}, whole")
    out["cores"] = host_cores()
    return out


def reference_arm(args):
    """The CPU oracle as the reference arm, on every host core: each step runs
    the oracle over the headline workload's decode requests (all of them, or a
    rotating slice sized so the whole run stays within about two minutes).
    Rank 0 alone runs it; the other ranks of a torchrun launch exit 0."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    steps, warmup = args.steps, args.warmup
    cores = host_cores()
    crew = OracleCrew(HEADLINE, "decode", cores)
    try:
        trial, _ = crew.run()
        nparts = max(1, min(16, math.ceil(trial * (steps + warmup) / 120.0)))
        per = []
        for i in range(warmup + steps):
            secs, units = crew.run(i % nparts, nparts)
            if i >= warmup:
                per.append((secs, units[0]))
    finally:
        crew.close()
    tot_s = sum(t for t, _ in per)
    value = sum(b for _, b in per) / tot_s / 1e9
    w = make_workload(HEADLINE, 0)
    sample = (f"{'all' if nparts == 1 else f'1/{nparts} (rotating) of the'} {len(w.decode_ids)} decode requests "
              f"of {HEADLINE} per step, {len(crew.groups)} processes x 1 thread")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": steps, "warmup": warmup,
        "ms_per_step": 1000 * tot_s / len(per), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": HEADLINE, **{k: v for k, v in w.describe().items() if k != "workload"}},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    emit(rank, line)
    return 0


# -------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workloads", default="all",
                    help="extra workloads to measure besides the headline: all, none, or a list")
    ap.add_argument("--cpu-budget", type=float, default=1.0,
                    help="0 skips the CPU-oracle baseline (any other value runs it)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        return reference_arm(args)

    import torch
    dist = None
    rank, world = int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as tdist
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                 device_id=torch.device("cuda", local))
        dist = tdist
    import paged_kv_attention_37_b200 as pkv

    hbm, tf_burst, tf_sust, peak_src = peaks()
    pre_roof = None
    head = measure(pkv, torch, HEADLINE, args.steps, args.warmup, dist, local)
    extra = {}
    names = [] if args.workloads == "none" else (
        [n for n in ("tiny_decode", "mixed_prefill_decode", "splitk_long", "frag_large", "spec_verify")]
        if args.workloads == "all" else [n for n in args.workloads.split(",") if n])
    for n in names:
        r = measure(pkv, torch, n, args.steps, args.warmup, dist, local)
        e = {"ms_per_step": r["ms_per_step"], "timed_region": r["timing"], "tokens_per_step": r["tokens"],
             "tokens_per_s": world * r["tokens"] / (r["ms_per_step"] / 1e3),
             "e2e_ms_per_step": r["e2e_ms_per_step"]}
        if r["dec_ms"]:
            gbs = r["kv_bytes_dec"] / (r["dec_ms"] / 1e3) / 1e9
            e.update({"decode_kv_bytes": r["kv_bytes_dec"], "decode_ms": r["dec_ms"],
                      "decode_kv_gbs": gbs, "decode_pct_of_8TBs": 100 * gbs / HBM_NOMINAL_GBS,
                      "decode_frac_of_measured_hbm": gbs / hbm})
        if r["pre_ms"] and r["w"].notes.get("attention") == "verify":
            gbs = r["kv_bytes_pre"] / (r["pre_ms"] / 1e3) / 1e9
            e.update({"verify_kv_bytes": r["kv_bytes_pre"], "verify_ms": r["pre_ms"], "verify_kv_gbs": gbs,
                      "verify_pct_of_8TBs": 100 * gbs / HBM_NOMINAL_GBS, "verify_frac_of_measured_hbm": gbs / hbm,
                      "verify_tokens_per_s": world * r["tokens"] / (r["pre_ms"] / 1e3)})
        elif r["pre_ms"]:
            tfs = r["flops_pre"] / (r["pre_ms"] / 1e3) / 1e12
            e.update({"prefill_ms": r["pre_ms"], "prefill_flops": r["flops_pre"],
                      "prefill_tflops": tfs, "prefill_frac_of_measured_bf16": tfs / tf_sust})
        if r["mixed_ms"]:
            e.update({"one_launch_ms_per_step": r["mixed_ms"],
                      "one_launch_tokens_per_s": world * r["tokens"] / (r["mixed_ms"] / 1e3),
                      "one_launch": "kv_append + pkv_paged_attn_mixed (chunks and decode from one work queue)"})
        e["step_kv_gbs"] = (r["kv_bytes_dec"] + r["kv_bytes_pre"]) / (r["ms_per_step"] / 1e3) / 1e9
        e["clocks"] = r["clocks"]
        extra[n] = e
        if r["pre_ms"] and r["w"].notes.get("attention") != "verify":
            pre_roof = {"bound": "tensor", "achieved": r["flops_pre"] / (r["pre_ms"] / 1e3) / 1e12,
                        "peak": tf_sust, "unit": "TFLOP/s",
                        "traffic": profiled_traffic("prefill_mixed_prefill_decode"),
                        "kernel": "chunked prefill (tcgen05), one pkv_paged_attn_chunked_prefill call",
                        "workload": n, "flops_per_launch": r["flops_pre"], "ms": r["pre_ms"],
                        "timing": "one CUDA graph of K back-to-back prefill calls, one replay timed",
                        "peak_source": f"{peak_src} bf16_tflops_sustained (the kernel runs inside a long loop)"}
            pre_roof["frac"] = pre_roof["achieved"] / tf_sust

    w = head["w"]
    kv_bytes = head["kv_bytes_dec"]
    value = aggregate_gbs(world, kv_bytes, head["ms_per_step"])
    achieved = aggregate_gbs(1, kv_bytes, head["dec_ms"])
    e2e_value = aggregate_gbs(world, kv_bytes, head["e2e_ms_per_step"])
    if rank != 0:
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()
        return 0
    cpu = None
    if world == 1 and args.cpu_budget > 0:
        # the oracle on the host cores, whole workloads, 1 thread and all cores
        cpu = {n: oracle_times(n, "prefill" if n == "spec_verify" else "decode")
               for n in [HEADLINE] + [n for n in names if n != "mixed_prefill_decode"]}
        if "mixed_prefill_decode" in names:
            cpu["mixed_prefill_decode"] = {"decode": oracle_times("mixed_prefill_decode", "decode"),
                                           "prefill": oracle_times("mixed_prefill_decode", "prefill")}
        for n, rec in cpu.items():
            if n in extra:
                extra[n]["oracle"] = rec
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "accumulate": "f32",
        "data": "synthetic",
        "config": {"workload": HEADLINE, **{k: v for k, v in w.describe().items() if k != "workload"},
                   "kv_bytes_per_step": kv_bytes, "parallelism": f"replicas{world}",
                   "l2": "inputs larger than L2 (KV read per step > 126 MB), no flush",
                   "timed_region": head["timing"]},
        "pct_of_8TBs": 100 * value / HBM_NOMINAL_GBS,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "traffic": profiled_traffic("decode_partition_qwen3_decode"),
                     "kernel": "decode split-K partition with in-kernel merge (one pkv_paged_attn_decode call)",
                     "bytes_per_launch": kv_bytes, "ms": head["dec_ms"],
                     "timing": "one CUDA graph of K back-to-back decode calls, one replay timed",
                     "peak_source": f"{peak_src} hbm_gbs", "pct_of_8TBs": 100 * achieved / HBM_NOMINAL_GBS},
        "cpu_baseline": None,
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": head["h2d"],
                "d2h_bytes_per_step": head["d2h"], "ms_per_step": head["e2e_ms_per_step"]},
        "gpu_launches": head["launches"] * args.steps,
        "clocks": head["clocks"],
        "workloads": extra,
    }
    if pre_roof is not None:
        line["roofline_prefill"] = pre_roof
    if cpu is not None:
        h = cpu[HEADLINE]
        line["cpu_baseline"] = {
            "value": h["all_cores"]["kv_gbs"], "unit": "GB/s", "cores": h["cores"], "kind": "oracle",
            "sample": h["sample"] + f", {h['all_cores']['processes']} processes x 1 thread",
            "seconds": h["all_cores"]["seconds"],
            "single_thread": {"value": h["1_thread"]["kv_gbs"], "unit": "GB/s", "cores": 1,
                              "seconds": h["1_thread"]["seconds"]}}
    emit(rank, line)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
