#!/usr/bin/env python
"""Benchmark of MLA decode in absorbed latent space on B200.

One step = one pass of the whole decode path over one batch: the split-KV
schedule, the decode kernel and the combine kernel, all through the C ABI
(libmla_b200.so).  The workload is the DeepSeek-V3-shaped decode batch
(b=64, s_q=1, h=128, k=512, p=64, t=4096, 64-token pages, random block
table), synthetic bf16 N(0,1) data.  The metric is TFLOP/s by the page's
cost model (FLOPs = 2 b h s t (2k+p)); the KV GB/s by the same model is
reported beside it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs an independent replica on its own GPU (the
requests shard with no exchange step); the whole-job value sums all ranks'
FLOPs over the slowest rank's time.  `--impl reference` times the fp64 CPU
oracle on a bounded sample of the same workload instead (rank 0 only).
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
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import mla_workloads as mw  # noqa: E402
from mla_workloads import cost  # noqa: E402

METRIC = "MLA decode TFLOPS & KV GB/s vs B200 roofline (h=128,k=512,p=64,t=4096)"
L2_FLUSH_BYTES = 256 << 20
# DRAM bytes (read + write) of one decode launch per workload, from one ncu
# capture of dram__bytes_read.sum + dram__bytes_write.sum each.  Valid only
# for the kernel sources they were taken on: reported as null as soon as any
# of them differs (checked by content hash at run time).
TRAFFIC_SOURCES_SHA1 = {
    "mla_latent_space_b200/csrc/decode_sm100.cu": "183aaa293124ca5522473db1c40c5912bbf84146",
    "mla_latent_space_b200/csrc/sm100_ptx.cuh": "a666c6fb95adecc45850f281b1be3ecacba5d16c",
    "mla_latent_space_b200/csrc/kernel_util.cuh": "9d7c3e48c90d2d444145ab84159f8400e402f999",
    "mla_latent_space_b200/csrc/common.cuh": "7c6e8d72ef32d67aafb386e65a6767fa77f51a7f",
    "mla_latent_space_b200/csrc/decode_launch.cuh": "627872ce2ed746bf011fb893a4fd1851f41ed788",
}
TRAFFIC_BYTES = {
    "dsv3_b64_h128_t4096_paged": 311544064 + 4859648,
    "fp8_b64_h128_t32768": 1374417664 + 22606336,
}


def captured_traffic(workload: str):
    """The capture's bytes per launch for this workload if the kernel sources
    are unchanged since the capture, else None."""
    import hashlib
    if workload not in TRAFFIC_BYTES:
        return None
    for rel, want in TRAFFIC_SOURCES_SHA1.items():
        try:
            with open(os.path.join(ROOT, rel), "rb") as f:
                if hashlib.sha1(f.read()).hexdigest() != want:
                    return None
        except OSError:
            return None
    return TRAFFIC_BYTES[workload]


FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """SM clock, power and clock-event reasons of this process's GPU, sampled
    through NVML while the timed region runs: once as it starts, every 2 ms
    on a background thread, and once as it ends, so that even a region of a
    few milliseconds has several samples (nvidia-smi's own loop is too
    coarse for that)."""

    REASONS = (("hw_slowdown", "HwSlowdown"), ("hw_thermal_slowdown", "HwThermalSlowdown"),
               ("sw_thermal_slowdown", "SwThermalSlowdown"), ("sw_power_cap", "SwPowerCap"))

    def __init__(self, cuda_index: int, period_s: float = 0.002):
        self.cuda_index, self.period = cuda_index, period_s
        self.samples, self.reasons, self.power = [], set(), []
        self.max_mhz, self.err = None, None
        self._stop, self._thread, self._nvml = None, None, None

    def _handle(self):
        import pynvml
        pynvml.nvmlInit()
        self._nvml = pynvml
        try:   # match the CUDA device by UUID (CUDA and NVML may number GPUs differently)
            uuid = str(torch.cuda.get_device_properties(self.cuda_index).uuid)
            return pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(self.cuda_index)

    def start(self):
        import threading
        try:
            h = self._handle()
            nv = self._nvml
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons",
                                  getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons", None))
            bits = {}
            for name, suffix in self.REASONS:
                v = getattr(nv, "nvmlClocksEventReason" + suffix, getattr(nv, "nvmlClocksThrottleReason" + suffix, 0))
                bits[name] = int(v)
        except Exception as e:   # no NVML: the line says so
            self.err = f"nvml unavailable: {type(e).__name__}"
            return
        self._stop = threading.Event()

        def sample():
            try:
                self.samples.append(float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)))
                self.power.append(nv.nvmlDeviceGetPowerUsage(h) / 1000.0)
                r = int(get_reasons(h)) if get_reasons else 0
                for name, bit in bits.items():
                    if bit and r & bit:
                        self.reasons.add(name)
            except Exception:
                pass

        def loop():
            while not self._stop.wait(self.period):
                sample()

        self._sample = sample
        sample()
        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()

    def stop(self):
        if self._thread is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.err or "not sampled"], "samples": 0}
        self._stop.set()
        self._thread.join(timeout=5)
        self._sample()
        try:
            self._nvml.nvmlShutdown()
        except Exception:
            pass
        sm = self.samples
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(sm),
                "power_w_max": max(self.power) if self.power else None, "source": "nvml, 2 ms"}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:   # a host without GPUs (the reference arm): gloo
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 0) for d in threadpool_info() if d.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def run_reference(args, wl, world, rank):
    """The reference arm: the fp64 CPU oracle, as it stands, on the host
    cores; each step is a bounded sample of the workload (whole requests in
    batch order until `--ref-seconds` have passed)."""
    if rank != 0:
        return
    import oracle
    oracle.decode(wl, rows=[(0, 0)])   # warm the BLAS threads (untimed)
    rates, secs, desc = [], [], ""
    budget = min(args.ref_seconds, 120.0 / max(1, args.steps))   # the whole run within about two minutes
    for _ in range(args.steps):
        tf, sec, desc = oracle_timed(wl, budget)
        rates.append(tf)
        secs.append(sec)
    tflops = sum(rates) / len(rates)
    cores = blas_threads()
    line = {"metric": METRIC, "value": tflops, "unit": "TFLOP/s", "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sum(secs) / len(secs) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(wl, world),
            "cpu_baseline": {"value": tflops, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc},
            "e2e": {"value": tflops, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_e2e_pipelined(args, wl, dev, shape, pool, kv_scale, world):
    """Steps per unit time of the whole decode step including its host
    transfers, pipelined over three streams (upload, compute, download).
    With three buffer sets a step's upload never waits for the download of
    the step before last, so uploads and downloads each run back to back on
    their own copy engine.  A step's inputs (query rows, block table,
    lengths) travel as one packed copy and its outputs (O, lse) as one: the
    library takes views into the packed device buffers, so each direction
    pays one copy's fixed cost per step."""
    import mla_latent_space_b200 as mla
    nbuf = args.e2e_buffers

    def layout(parts):   # [(name, nbytes)] -> offsets 256-byte aligned, total
        off, out = 0, {}
        for name, nb in parts:
            out[name] = (off, nb)
            off = (off + nb + 255) // 256 * 256
        return out, off

    oshape = (wl.batch, wl.s_q, wl.num_heads, 512)
    lshape = (wl.batch, wl.s_q, wl.num_heads)
    bt_np, sl_np = np.ascontiguousarray(wl.block_table), np.ascontiguousarray(wl.seqlens)
    lin, nin = layout([("q", wl.q.numel() * 2), ("bt", bt_np.nbytes), ("sl", sl_np.nbytes)])
    lout, nout = layout([("out", int(np.prod(oshape)) * 2), ("lse", int(np.prod(lshape)) * 4)])

    def view(buf, lay, name, dtype, shp):
        o, nb = lay[name]
        return buf[o:o + nb].view(dtype).view(shp)

    h_in = torch.empty(nin, dtype=torch.uint8).pin_memory()
    view(h_in, lin, "q", torch.bfloat16, tuple(wl.q.shape)).copy_(wl.q)
    view(h_in, lin, "bt", torch.int32, bt_np.shape).copy_(torch.from_numpy(bt_np))
    view(h_in, lin, "sl", torch.int32, sl_np.shape).copy_(torch.from_numpy(sl_np))
    h_out = [torch.empty(nout, dtype=torch.uint8).pin_memory() for _ in range(nbuf)]
    d_in = [torch.empty(nin, dtype=torch.uint8, device=dev) for _ in range(nbuf)]
    d_outb = [torch.empty(nout, dtype=torch.uint8, device=dev) for _ in range(nbuf)]
    d_q = [view(d, lin, "q", torch.bfloat16, tuple(wl.q.shape)) for d in d_in]
    d_bt = [view(d, lin, "bt", torch.int32, bt_np.shape) for d in d_in]
    d_sl = [view(d, lin, "sl", torch.int32, sl_np.shape) for d in d_in]
    d_out = [view(d, lout, "out", torch.bfloat16, oshape) for d in d_outb]
    d_lse = [view(d, lout, "lse", torch.float32, lshape) for d in d_outb]
    decs = [mla.Decoder(shape, device=dev) for _ in range(nbuf)]
    s_up, s_comp, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    up_done = [ev() for _ in range(nbuf)]
    comp_done = [ev() for _ in range(nbuf)]
    down_done = [ev() for _ in range(nbuf)]
    used = [False] * nbuf

    def step(k):
        b = k % nbuf
        with torch.cuda.stream(s_up):
            if used[b]:
                s_up.wait_event(down_done[b])       # its previous step is downloaded (so computed)
            d_in[b].copy_(h_in, non_blocking=True)
            up_done[b].record(s_up)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(up_done[b])
            decs[b].schedule(d_sl[b], stream=s_comp)
            decs[b].decode(d_q[b], pool, kv_scale, d_bt[b], d_sl[b], wl.softmax_scale, d_out[b], d_lse[b],
                           stream=s_comp)
            comp_done[b].record(s_comp)
        with torch.cuda.stream(s_down):
            s_down.wait_event(comp_done[b])
            h_out[b].copy_(d_outb[b], non_blocking=True)
            down_done[b].record(s_down)
        used[b] = True

    # warm-up: the host link only reaches its full rate after some hundreds of
    # milliseconds of steady transfers (cold, an upload runs at a quarter of
    # it), as it would in a serving loop; run steps for at least 0.3 s
    k, t_warm = 0, time.perf_counter()
    while k < max(3, args.warmup) or time.perf_counter() - t_warm < 0.3:
        step(k)
        k += 1
        if k % 64 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()
    for dd in decs:
        st = dd.status()
        if st != 0:
            raise RuntimeError(f"device status in the end-to-end loop: {mla.error_string(st)}")
    K = extra_steps(args)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    t0.record(s_up)
    for k in range(K):
        step(k)
    s_up.wait_stream(s_down)
    t1.record(s_up)
    torch.cuda.synchronize()
    barrier(world)
    last = view(h_out[(K - 1) % nbuf], lout, "out", torch.bfloat16, oshape)
    if not bool(torch.isfinite(last.float()).all()):
        raise RuntimeError("non-finite output in the end-to-end loop")
    return max_over_ranks(t0.elapsed_time(t1) / K, world), nin, nout


def extra_steps(args):
    """Timed launches of each secondary measurement (projections, sparse,
    MLAvar6+, the end-to-end loop): the headline's K, at most 100."""
    return max(1, min(args.steps, 100))


def proj_bytes(rows, heads):
    """Algorithmic bytes of the two projections (weights read once, inputs
    read once, outputs written once; bf16)."""
    absorb = 2 * (heads * 512 * 128 + rows * heads * 192 + rows * heads * 576)
    decompress = 2 * (heads * 128 * 512 + rows * heads * 512 + rows * heads * 128)
    return absorb, decompress


def run_projections(args, wl, dev, shape, pool, kv_scale, bt, sl, flush, pk):
    """The per-head projections on either side of the latent decode, timed
    like the decode (L2 flushed before each launch, CUDA events on the
    launching stream), and the whole MLA decode attention they form with it:
    absorb -> schedule -> decode -> combine -> decompress."""
    import mla_latent_space_b200 as mla
    R, h = wl.batch * wl.s_q, wl.num_heads
    p = mw.make_projections(R, h, seed=1)
    q = p.q.to(dev).view(wl.batch, wl.s_q, h, 192)
    wk, wv = p.w_k.to(dev), p.w_kvb2.to(dev)
    o_lat = p.o_lat.to(dev).view(wl.batch, wl.s_q, h, 512)
    qz = torch.empty((wl.batch, wl.s_q, h, 576), dtype=torch.bfloat16, device=dev)
    out = torch.empty((wl.batch, wl.s_q, h, 128), dtype=torch.bfloat16, device=dev)
    lat = torch.empty((wl.batch, wl.s_q, h, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((wl.batch, wl.s_q, h), dtype=torch.float32, device=dev)
    dec = mla.Decoder(shape, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    def absorb():
        mla.mla_absorb_q(q, wk, qz, device_status=status)

    def decompress():
        mla.mla_decompress_o(o_lat, wv, out, device_status=status)

    def chain():
        mla.mla_absorb_q(q, wk, qz, device_status=status)
        dec.schedule(sl)
        dec.decode(qz, pool, kv_scale, bt, sl, wl.softmax_scale, lat, lse)
        mla.mla_decompress_o(lat, wv, out, device_status=status)

    def timed(fn):
        for _ in range(args.warmup):
            flush.zero_()
            fn()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(extra_steps(args))]
        torch.cuda.synchronize()
        for a, b in evs:
            flush.zero_()
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in evs) / len(evs) * 1e3   # us

    # calibration: a one-element torch kernel timed in the same position
    # (after the flush, between an event pair) shows what the event pair
    # itself adds to a short launch
    tiny = torch.zeros(1024, device=dev)
    empty_us = timed(lambda: tiny.add_(1.0))
    ab, db = proj_bytes(R, h)
    res = {"empty_launch_us": empty_us}
    for name, fn, by, kern in [("absorb", absorb, ab, "mla_absorb_q"), ("decompress", decompress, db, "mla_decompress_o")]:
        us = timed(fn)
        gbs = by / (us * 1e-6) / 1e9
        net = max(us - empty_us, 1e-3)
        res[name] = {"kernel": kern, "launch_us": us, "bytes": by, "flops": 2 * R * h * 128 * 512,
                     "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                                  "frac": gbs / pk["hbm_gbs"],
                                  "frac_net_of_empty_launch": by / (net * 1e-6) / 1e9 / pk["hbm_gbs"]}}
    chain_us = timed(chain)
    # the same chain captured once in a CUDA graph and replayed (launch work
    # on the host leaves the timed region; the device work is unchanged)
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        chain()
    stream.wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        chain()
    graph_us = timed(graph.replay)
    del graph
    if int(status.item()) != 0 or dec.status() != 0:
        raise RuntimeError("device status set in the projection timing")
    flops, _ = cost.workload_cost(wl)
    res["whole_step_us"] = chain_us
    res["whole_step_graph_us"] = graph_us
    res["whole_step"] = "absorb -> schedule -> decode -> combine -> decompress, one event pair around it"
    res["whole_step_tflops"] = (flops + 2 * 2 * R * h * 128 * 512) / (chain_us * 1e-6) / 1e12
    res["rows"], res["heads"] = R, h
    if not args.no_cpu_baseline:
        # the fp64 oracle's two projections on the same inputs, on the host cores
        import oracle
        f64 = oracle.bf16_to_f64
        qf, wkf, of, wvf = f64(p.q), f64(p.w_k), f64(p.o_lat), f64(p.w_kvb2)
        t0 = time.perf_counter()
        oracle.absorb(qf, wkf)
        t1 = time.perf_counter()
        oracle.decompress(of, wvf)
        t2 = time.perf_counter()
        res["cpu_baseline"] = {"kind": "oracle", "cores": blas_threads(), "absorb_us": (t1 - t0) * 1e6,
                               "decompress_us": (t2 - t1) * 1e6, "sample": f"all {R} rows x {h} heads"}
    # timed launches: absorb alone, decompress alone, and the chain's five kernels (twice: launched, replayed)
    res["gpu_launches"] = extra_steps(args) * (1 + 1 + 5 + 5)
    return res


SPARSE_SHAPE = dict(batch=64, s_q=1, heads=128, seqlen=32768, topk=2048)


def sparse_cost(b, s, h, topk):
    """FLOPs and the fused-ideal bytes of a sparse decode: every listed row
    read once (1152 B), Q read and O written once."""
    flops = 2 * b * s * h * topk * (2 * 512 + 64)
    nbytes = 2 * (b * s * h * 576 + b * s * h * 512) + b * s * topk * 1152
    return flops, nbytes


def run_sparse(args, dev, flush, pk):
    """Token-level sparse decode on a DeepSeek-V3.2-style batch: 64 requests
    of 32768 cached tokens, 2048 listed positions per query token, timed like
    the decode (L2 flushed before each launch sequence, CUDA events)."""
    import mla_latent_space_b200 as mla
    S = SPARSE_SHAPE
    wl = mw.make(S["batch"], S["s_q"], S["heads"], S["seqlen"], seed=40, name="sparse_b64_h128_t32768_k2048")
    idx = mw.make_sparse_indices(wl.seqlens, S["s_q"], S["topk"], seed=41)
    shape = mla.make_shape(wl.batch, wl.s_q, wl.num_heads, wl.max_pages, wl.num_pages)
    dec = mla.SparseDecoder(shape, S["topk"], device=dev)
    q, pool = wl.q.to(dev), wl.pool.to(dev)
    bt, sl = torch.from_numpy(wl.block_table).to(dev), torch.from_numpy(wl.seqlens).to(dev)
    ix = torch.from_numpy(idx).to(dev)
    out = torch.empty((wl.batch, wl.s_q, wl.num_heads, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((wl.batch, wl.s_q, wl.num_heads), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        flush.zero_()
        dec.decode(q, pool, bt, sl, ix, wl.softmax_scale, out, lse)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(extra_steps(args))]
    torch.cuda.synchronize()
    for a, b in evs:
        flush.zero_()
        a.record(stream)
        dec.decode(q, pool, bt, sl, ix, wl.softmax_scale, out, lse)
        b.record(stream)
    torch.cuda.synchronize()
    if dec.status() != 0:
        raise RuntimeError("device status set in the sparse decode timing")
    us = sum(a.elapsed_time(b) for a, b in evs) / len(evs) * 1e3
    flops, nbytes = sparse_cost(wl.batch, wl.s_q, wl.num_heads, S["topk"])
    gbs = nbytes / (us * 1e-6) / 1e9
    del pool
    cpu = None
    if not args.no_cpu_baseline:
        # the fp64 oracle on the first two requests, scaled to a whole call
        import oracle
        n = 2
        sub = mw.Workload(name="sub", batch=n, s_q=wl.s_q, num_heads=wl.num_heads, causal=False, cache_dtype="bf16",
                          seqlens=wl.seqlens[:n], block_table=wl.block_table[:n], q=wl.q[:n], pool=wl.pool,
                          kv_scale=None, softmax_scale=wl.softmax_scale)
        t0 = time.perf_counter()
        oracle.sparse_decode(sub, idx[:n])
        dt = time.perf_counter() - t0
        cpu = {"kind": "oracle", "cores": blas_threads(), "us_per_call": dt * 1e6 * wl.batch / n,
               "tflops": flops * n / wl.batch / dt / 1e12,
               "sample": f"{n} of {wl.batch} requests (each gathers its whole cache in fp64), scaled to the call"}
    return {"workload": wl.name, "topk": S["topk"], "us_per_call": us, "tflops": flops / (us * 1e-6) / 1e12,
            "kernels": "gather -> schedule -> decode -> combine (4 launches)",
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "bytes": nbytes,
                         "note": "bytes of a fused design (each listed row read once); this composition moves "
                                 "each row three times"},
            "gpu_launches": 4 * extra_steps(args), "cpu_baseline": cpu}


def var6_flops(b, h, s, t, n):
    """The page's MLAvar6+ cost model: 2bhstp + 4bhsnd + 4bhsok (o = t - n)."""
    return 2 * b * h * s * t * 64 + 4 * b * h * s * n * 128 + 4 * b * h * s * (t - n) * 512


def run_var6(args, dev, flush, pk):
    """MLAvar6+ split decode on the speculative workload (b=32, s=16,
    t=4096, causal): n = 16 and 64 newest tokens held decompressed, against
    the latent path with its output decompressed (schedule, decode, combine,
    decompression), both timed like the decode."""
    import mla_latent_space_b200 as mla
    wl = mw.make_config(5, seed=0)
    b, s, h = wl.batch, wl.s_q, wl.num_heads
    g = torch.Generator().manual_seed(7)
    q = torch.randn(b, s, h, 192, generator=g).to(torch.bfloat16).to(dev)
    wv = mw.make_projections(1, h, seed=8).w_kvb2.to(dev)
    shape = mla.make_shape(b, s, h, wl.max_pages, wl.num_pages, wl.cache_dtype, wl.causal)
    qz, pool = wl.q.to(dev), wl.pool.to(dev)
    bt, sl = torch.from_numpy(wl.block_table).to(dev), torch.from_numpy(wl.seqlens).to(dev)
    out = torch.empty((b, s, h, 128), dtype=torch.bfloat16, device=dev)
    lat = torch.empty((b, s, h, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((b, s, h), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def timed(fn):
        for _ in range(args.warmup):
            flush.zero_()
            fn()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(extra_steps(args))]
        torch.cuda.synchronize()
        for a, e in evs:
            flush.zero_()
            a.record(stream)
            fn()
            e.record(stream)
        torch.cuda.synchronize()
        return sum(a.elapsed_time(e) for a, e in evs) / len(evs) * 1e3

    dec = mla.Decoder(shape, device=dev)

    def latent():
        dec.schedule(sl)
        dec.decode(qz, pool, None, bt, sl, wl.softmax_scale, lat, lse)
        mla.mla_decompress_o(lat, wv, out)

    t_lat = timed(latent)
    t = int(wl.seqlens[0])
    res = {"workload": wl.name, "latent_path_us": t_lat,
           "latent_path_tflops": var6_flops(b, h, s, t, 0) / (t_lat * 1e-6) / 1e12, "split": []}
    for n in (16, 64):
        k_new = torch.randn(b, n, h, 128, generator=g).to(torch.bfloat16).to(dev)
        v_new = torch.randn(b, n, h, 128, generator=g).to(torch.bfloat16).to(dev)
        vd = mla.Var6Decoder(shape, n, device=dev)
        us = timed(lambda: vd.decode(qz, q, pool, bt, sl, k_new, v_new, wv, wl.softmax_scale, out, lse))
        if vd.status() != 0:
            raise RuntimeError("device status set in the MLAvar6+ timing")
        res["split"].append({"n_new": n, "us_per_call": us,
                             "tflops": var6_flops(b, h, s, t, n) / (us * 1e-6) / 1e12})
    if dec.status() != 0:
        raise RuntimeError("device status set in the latent-path timing")
    res["gpu_launches"] = extra_steps(args) * (4 + 2 * 6)
    return res


def run_projections_only(args, wl, world, rank):
    """`--projections-only`: the projection timing of run_projections alone,
    on this rank's GPU, printed as its own JSON line."""
    import mla_latent_space_b200 as mla
    from mla_latent_space_b200 import build
    build.build()
    dev = torch.device("cuda", torch.cuda.current_device())
    shape = mla.make_shape(wl.batch, wl.s_q, wl.num_heads, wl.max_pages, wl.num_pages, wl.cache_dtype, wl.causal)
    pool = wl.pool.to(dev)
    kv_scale = None if wl.kv_scale is None else wl.kv_scale.to(dev)
    bt = torch.from_numpy(wl.block_table).to(dev)
    sl = torch.from_numpy(wl.seqlens).to(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    pk, _ = peaks()
    if args.sparse_only:
        res = {"sparse": run_sparse(args, dev, flush, pk)}
    else:
        res = {"workload": wl.name, "mla_attention": run_projections(args, wl, dev, shape, pool, kv_scale, bt, sl,
                                                                     flush, pk)}
    if rank == 0:
        print(json.dumps(res), flush=True)


class DeviceWorkload:
    """One workload's inputs and outputs resident on the GPU, with its
    decoder (schedule and workspace)."""

    def __init__(self, wl, dev):
        import mla_latent_space_b200 as mla
        self.wl = wl
        self.shape = mla.make_shape(wl.batch, wl.s_q, wl.num_heads, wl.max_pages, wl.num_pages, wl.cache_dtype,
                                    wl.causal)
        self.q = wl.q.to(dev)
        self.pool = wl.pool.to(dev)
        self.kv_scale = None if wl.kv_scale is None else wl.kv_scale.to(dev)
        self.bt = torch.from_numpy(wl.block_table).to(dev)
        self.sl = torch.from_numpy(wl.seqlens).to(dev)
        self.out = torch.empty((wl.batch, wl.s_q, wl.num_heads, 512), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((wl.batch, wl.s_q, wl.num_heads), dtype=torch.float32, device=dev)
        self.dec = mla.Decoder(self.shape, device=dev)

    def step(self, ev=None):
        """schedule -> decode -> combine; `ev` brackets the decode launch."""
        import mla_latent_space_b200 as mla
        stream = torch.cuda.current_stream()
        d, wl = self.dec, self.wl
        d.schedule(self.sl)
        if ev is not None:
            ev[0].record(stream)
        mla.mla_decode_fwd(self.shape, self.q, self.pool, self.kv_scale, self.bt, self.sl, wl.softmax_scale,
                           d.sched, d.workspace, self.out, self.lse)
        if ev is not None:
            ev[1].record(stream)
        mla.mla_combine(self.shape, d.sched, d.workspace, self.out, self.lse)

    def status(self):
        return self.dec.status()


def time_steps(args, dw, flush, K, world=1, local=0, sample_clocks=False):
    """W warm-up steps, then K timed steps (L2 flushed before each, outside
    the events), then K more with events around the decode launch alone.
    Returns (step ms list, decode ms list, clocks or None)."""
    import mla_latent_space_b200 as mla
    stream = torch.cuda.current_stream()
    for _ in range(max(3, args.warmup)):
        flush.zero_()
        dw.step()
    torch.cuda.synchronize()
    st = dw.status()
    if st != 0:
        raise RuntimeError(f"{dw.wl.name}: device status after warm-up: {mla.error_string(st)}")
    ev_step = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    ev_dec = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    clocks = ClockSampler(local) if sample_clocks else None
    barrier(world)
    torch.cuda.synchronize()
    if clocks:
        clocks.start()
    # Each iteration runs the step twice: once bracketed by events only at
    # its ends (an event between two of its kernels would stop the next one
    # from launching behind the previous, programmatic dependent launch), and
    # once with events around the decode launch alone, for the roofline.
    # Interleaving them gives both the same clocks and power state.
    for k in range(K):
        flush.zero_()
        ev_step[k][0].record(stream)
        dw.step()
        ev_step[k][1].record(stream)
        flush.zero_()
        dw.step(ev_dec[k])
    torch.cuda.synchronize()
    clk = clocks.stop() if clocks else None
    barrier(world)
    st = dw.status()
    if st != 0:
        raise RuntimeError(f"{dw.wl.name}: device status after timing: {mla.error_string(st)}")
    return [a.elapsed_time(b) for a, b in ev_step], [a.elapsed_time(b) for a, b in ev_dec], clk


def roofline(wl, dec_ms, pk, pk_kind, traffic):
    """The decode kernel against the bound the cost model picks for this
    workload: HBM when its bytes take longer at the measured copy bandwidth
    than its FLOPs at the measured bf16 GEMM rate, else the tensor core."""
    flops, nbytes = cost.workload_cost(wl)
    gbs = nbytes / (dec_ms * 1e-3) / 1e9
    tflops = flops / (dec_ms * 1e-3) / 1e12
    t_hbm = nbytes / (pk["hbm_gbs"] * 1e9)
    t_tc = flops / (pk["bf16_tflops"] * 1e12)
    if t_hbm >= t_tc:
        roof = {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": gbs / pk["hbm_gbs"],
                "traffic": traffic}
    else:
        roof = {"bound": "tensor", "achieved": tflops, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                "frac": tflops / pk["bf16_tflops"], "traffic": traffic}
    roof["kernel"] = "mla_decode_fwd"
    roof["peak_kind"] = f"{pk_kind} (MEASURED_PEAKS.json)" if pk_kind == "measured" else "fallback"
    roof["launch_us"] = dec_ms * 1e3
    roof["roofline_us"] = max(t_hbm, t_tc) * 1e6
    roof["tensor_frac"] = tflops / pk["bf16_tflops"]
    roof["tensor_frac_sustained"] = tflops / pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
    roof["hbm_frac"] = gbs / pk["hbm_gbs"]
    if wl.cache_dtype == "fp8":
        roof["note"] = ("the cost model's bf16 tensor peak, as for the other workloads; the latent scores run "
                        "as FP8 MMAs, the value product as fp16 MMAs")
    return roof


def oracle_timed(wl, budget_s):
    """The fp64 oracle over whole requests (every query token, every head)
    in batch order until `budget_s` seconds have passed (at least one
    request).  Returns (TFLOP/s, seconds, description)."""
    import oracle
    t_tot, fl, n = 0.0, 0.0, 0
    while n < wl.batch and (n == 0 or t_tot < budget_s):
        rows = [(n, i) for i in range(wl.s_q)]
        t0 = time.perf_counter()
        oracle.decode(wl, rows=rows)
        t_tot += time.perf_counter() - t0
        fl += cost.mla_flops(1, wl.num_heads, wl.s_q, None, sum_t=int(wl.seqlens[n]))
        n += 1
    toks = int(wl.seqlens[:n].astype(np.int64).sum())
    return fl / t_tot / 1e12, t_tot, f"requests 0..{n - 1} of {wl.batch} ({toks} cached tokens, all heads)"


def per_config(args, dev, flush, pk, pk_kind, headline=None):
    """The five workloads, each timed like the headline (schedule -> decode
    -> combine with the L2 flushed before every step) with its decode launch
    against its roofline, and the oracle on a bounded sample of it."""
    res = {}
    K = max(5, min(args.steps, args.per_config_steps))
    for cfg in (1, 2, 3, 4, 5):
        if headline is not None and cfg == args.config:
            wl, step_ms, dec_ms, clk = headline
        else:
            wl = mw.make_config(cfg, seed=0)
            dw = DeviceWorkload(wl, dev)
            step_ms, dec_ms, clk = time_steps(args, dw, flush, K, sample_clocks=True)
            del dw
            torch.cuda.empty_cache()
        flops, nbytes = cost.workload_cost(wl)
        us = sum(step_ms) / len(step_ms) * 1e3
        dus = sum(dec_ms) / len(dec_ms) * 1e3
        ent = {"workload": wl.name, "steps": len(step_ms), "us_per_step": us,
               "tflops": flops / (us * 1e-6) / 1e12, "kv_gbs": nbytes / (us * 1e-6) / 1e9,
               "decode_us": dus, "flops": flops, "bytes": nbytes,
               "roofline": roofline(wl, dus * 1e-3, pk, pk_kind, captured_traffic(wl.name)), "clocks": clk}
        if cfg == 1:
            ent["note"] = "0.66 MB and 18 MFLOP: launch-bound, reported only"
        if not args.no_cpu_baseline:
            tf, sec, desc = oracle_timed(wl, args.cpu_seconds)
            ent["cpu_baseline"] = {"value": tf, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                                   "sample": desc, "seconds": sec}
        res[f"config{cfg}"] = ent
        del wl
    return res, 3 * 2 * K * 4   # launches of the timed regions of the four re-timed workloads


def config_dict(wl, world):
    """The `config` of the JSON line; both arms print the same one."""
    return {"workload": wl.name, "batch": wl.batch, "s_q": wl.s_q, "heads": wl.num_heads,
            "seq_len": int(wl.seqlens.max()), "sum_t": wl.total_tokens, "page": 64, "cache": wl.cache_dtype,
            "causal": bool(wl.causal), "parallelism": f"replicas x{world}",
            "l2": "flushed before every timed step (256 MiB write, outside the events)"}


def run_ours(args, wl, world, rank, local):
    import mla_latent_space_b200 as mla
    from mla_latent_space_b200 import build
    build.build()
    dev = torch.device("cuda", torch.cuda.current_device())
    dw = DeviceWorkload(wl, dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    K = args.steps
    step_ms, dec_ms, clk = time_steps(args, dw, flush, K, world=world, local=local, sample_clocks=True)
    my_ms = sum(step_ms) / K
    ms = max_over_ranks(my_ms, world)
    dec_avg_ms = sum(dec_ms) / K

    # End to end through the public API with host buffers.  Every step copies
    # its query, block table and lengths host -> device (pinned memory) and
    # its output and lse device -> host; the KV cache is resident device
    # state.  The steps run as a serving loop would: the copies go on their
    # own streams with double-buffered device tensors, so step k's kernels
    # overlap step k+1's upload and step k-1's download (a step's kernels
    # wait for its upload; a buffer is reused only after the step that last
    # used it has been downloaded).  The cache (302 MB) is larger than L2.
    e2e_ms, h2d, d2h = run_e2e_pipelined(args, wl, dev, dw.shape, dw.pool, dw.kv_scale, world)
    # the extras (the other workloads and the rows around the decode) are
    # timed in single-GPU runs; a multi-GPU run measures the headline step on
    # every replica
    extras = world == 1
    pk, pk_kind = peaks()
    proj = run_projections(args, wl, dev, dw.shape, dw.pool, dw.kv_scale, dw.bt, dw.sl, flush, pk) \
        if extras and not args.no_projections else None
    sparse = run_sparse(args, dev, flush, pk) if extras and not args.no_sparse else None
    var6 = run_var6(args, dev, flush, pk) if extras and not args.no_var6 else None
    del dw
    torch.cuda.empty_cache()
    pcfg, pc_launches = per_config(args, dev, flush, pk, pk_kind, headline=(wl, step_ms, dec_ms, clk)) \
        if extras and not args.no_per_config else (None, 0)

    flops, nbytes = cost.workload_cost(wl)
    value = world * flops / (ms * 1e-3) / 1e12
    traffic = args.traffic if args.traffic is not None else captured_traffic(wl.name)
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_dict(wl, world),
            "kv_gbs": world * nbytes / (ms * 1e-3) / 1e9,
            "us_per_step": ms * 1e3,
            "roofline": roofline(wl, dec_avg_ms, pk, pk_kind, traffic),
            "clocks": clk,
            "e2e": {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                    "pipelining": f"upload / compute / download streams, {args.e2e_buffers} buffers, one packed "
                                  "copy per direction"},
            "gpu_launches": 6 * K,
            "gpu_launches_note": "schedule + decode + combine, twice per timed iteration (the step timed whole, "
                                 "then with events around the decode launch)"}
    if pcfg is not None:
        line["per_config"] = pcfg
    if proj is not None:
        line["mla_attention"] = proj
    if sparse is not None:
        line["sparse_decode"] = sparse
    if var6 is not None:
        line["mlavar6"] = var6
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        if pcfg is not None:
            cb = dict(pcfg[f"config{args.config}"]["cpu_baseline"])
        else:
            tf, sec, desc = oracle_timed(wl, args.cpu_seconds)
            cb = {"value": tf, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle", "sample": desc,
                  "seconds": sec}
        line["cpu_baseline"] = cb
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=2, help="workload 1-5 (2 = the headline decode batch)")
    ap.add_argument("--no-per-config", action="store_true", help="skip the five-workload block")
    ap.add_argument("--per-config-steps", type=int, default=50, help="timed steps of each per-config workload")
    ap.add_argument("--cpu-seconds", type=float, default=3.0, help="oracle seconds per cpu_baseline sample")
    ap.add_argument("--ref-seconds", type=float, default=5.0, help="oracle seconds per reference-arm step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-projections", action="store_true",
                    help="skip the timing of the query absorption / output decompression kernels")
    ap.add_argument("--projections-only", action="store_true",
                    help="time only the query absorption / output decompression kernels and the whole step")
    ap.add_argument("--no-sparse", action="store_true", help="skip the timing of the token-level sparse decode")
    ap.add_argument("--sparse-only", action="store_true", help="time only the token-level sparse decode")
    ap.add_argument("--no-var6", action="store_true", help="skip the timing of the MLAvar6+ split decode")
    ap.add_argument("--e2e-buffers", type=int, default=3, help="buffer sets of the pipelined end-to-end loop")
    ap.add_argument("--traffic", type=float, default=None,
                    help="ncu dram bytes per decode launch for the current kernel (else null)")
    args = ap.parse_args()
    world, rank, local = dist_setup(args.gpus)
    wl = mw.make_config(args.config, seed=0)
    try:
        if args.impl == "reference":
            run_reference(args, wl, world, rank)
        elif args.projections_only or args.sparse_only:
            run_projections_only(args, wl, world, rank)
        else:
            run_ours(args, wl, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
