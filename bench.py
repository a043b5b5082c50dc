"""Benchmark of the KV-cache decode step on B200 (one JSON line on rank 0).

Workload (default): 32-layer GQA decode -- B=16 requests, H_q=32, H_kv=8,
D=128, bf16, contiguous cache, T_past=4096, one new token per request.  A
step is one decode layer-step for all 32 layers: kvc_append_attend per layer
(append, split attend and log-sum-exp merge in one launch on the persistent
path), 8.6 GB of K/V read per step, far above the 126 MB L2, so consecutive
steps cannot hit in L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kvc|reference]

`value` is whole-job KV HBM GB/s: algorithmic bytes of all ranks' steps
(K/V read, q read, out written, appended K/V written) over the max-over-ranks
device time.  `e2e` is the same metric through the C ABI with pinned host
buffers, the host->device copy of q/k_new/v_new and the device->host copy of
out inside the timed region.  `--impl reference` times the fp64 CPU oracle
(the only reference implementation there is) on a bounded sample.
Multi-GPU runs are independent replicas (weak scaling): the decode step has
no cross-request exchange, so no collective is on the data path.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

import workloads as W  # noqa: E402

METRIC = ("decode-attention KV HBM GB/s (% of B200 peak) and tokens/s per layer-step")


# The sources each profiled kernel is compiled from: a committed ncu summary stays
# valid while these files are unchanged.
# The library's default threshold for the tcgen05 combine launch (KVC_TC_COMBINE_MIN_BYTES
# in csrc/kvc_api.cu): segments whose partials average more take a second launch.
TC_COMBINE_MIN_BYTES = 64 * 1024

KERNEL_SOURCES = {
    "attend_streamk_kernel": ("attend_streamk.cuh", "attend_fp8.cuh", "fp8.cuh",
                              "splitk_epilogue.cuh", "device_common.cuh", "params.cuh"),
    "attend_mma_kernel": ("attend_mma.cuh", "splitk_epilogue.cuh", "window.cuh",
                          "device_common.cuh", "params.cuh"),
    "attend_tc_kernel": ("attend_tc.cuh", "splitk_epilogue.cuh", "window.cuh",
                         "device_common.cuh", "params.cuh"),
    "attend_tc_streamk_kernel": ("attend_tc_streamk.cuh", "attend_tc.cuh", "attend_streamk.cuh",
                                 "device_common.cuh", "params.cuh"),
    "attend_fp8_kernel": ("attend_fp8.cuh", "fp8.cuh", "splitk_epilogue.cuh", "window.cuh",
                          "device_common.cuh", "params.cuh"),
    "attend_decode_kernel": ("attend_decode.cuh", "splitk_epilogue.cuh", "window.cuh",
                             "device_common.cuh", "params.cuh"),
}


def kernel_source_sha256(kernel: str = "attend_streamk_kernel") -> str:
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        f = ROOT / "kv_cache_decode_03_b200" / "csrc" / name
        h.update(f.name.encode())
        h.update(f.read_bytes())
    return h.hexdigest()


def profiled_traffic(kernel: str):
    """DRAM bytes per launch from a committed ncu summary, if its sources still match."""
    if kernel.split("<")[0] not in KERNEL_SOURCES:
        return None
    sha = kernel_source_sha256(kernel.split("<")[0])
    for f in sorted((ROOT / "profiles").glob("*.md")):
        kv = {}
        for line in f.read_text().splitlines():
            if ":" in line and not line.startswith(("|", " ", "#")):
                k, _, v = line.partition(":")
                kv[k.strip()] = v.strip()
        if kv.get("kernel") == kernel and kv.get("source_sha256") == sha:
            return int(kv["dram_bytes_per_launch"])
    return None


def peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def tensor_peak():
    """Dense bf16 TFLOP/s: the burst figure (a kernel timed on its own)."""
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        return float(json.loads(p.read_text())["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


L2_BYTES = 126e6


def fp8_algorithmic_bytes(c: W.Case) -> int:
    """Per layer-step on an FP8 cache: codes (1 B) and a K and a V scale (4 B) per
    (token, KV head) read; q in and out in the 16-bit type; the new rows read in the
    16-bit type and written as codes and scales."""
    tokens = c.kv_read_bytes(True) // (2 * c.H_kv * c.D * c.elt)
    kv = tokens * 2 * c.H_kv * (c.D + 4)
    qo = 2 * c.B * c.H_q * c.T_new * c.D * c.elt
    app = c.B * c.H_kv * c.T_new * 2 * (c.D * c.elt + c.D + 4)
    return kv + qo + app


def attend_kernel_name(c: W.Case, kv_format: str, split_tokens: int) -> str:
    rows = (c.H_q // c.H_kv) * c.T_new
    layout = "paged" if c.paged else "contiguous"
    if kv_format == "fp8":
        if split_tokens == 0:  # E4M3 stages in the stream-K kernel
            return f"attend_streamk_kernel<{c.D},1,bf16,{layout},fp8>"
        return f"attend_fp8_kernel<{c.D},{layout}>"
    if rows >= 17 and c.D in (64, 128):
        if split_tokens == 0:
            return f"attend_tc_streamk_kernel<{c.D},{c.dtype},{layout}>"
        return f"attend_tc_kernel<{c.D},{c.dtype},{layout}>"
    if split_tokens == 0:
        nt = 1 if rows <= 8 else 2
        return f"attend_streamk_kernel<{c.D},{nt},{c.dtype},{layout}>"
    if rows >= 3 and c.D in (64, 128):
        return f"attend_mma_kernel<{c.D},{c.dtype},{layout}>"
    return f"attend_decode_kernel<{c.D},{c.dtype},{layout}>"


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.f = None

    def __enter__(self):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict | None:
        if self.proc is None:
            return None
        self.f.flush()
        rows = [r.split(",") for r in Path(self.f.name).read_text().splitlines() if r.strip()]
        os.unlink(self.f.name)
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx = max(mx, float(r[2]))
                for k, name in enumerate(names):
                    if r[5 + k].strip().lower() == "active":
                        reasons.add(name)
            except (ValueError, IndexError):
                continue
        if not sm:
            return None
        busy = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle baseline
# ---------------------------------------------------------------------------

def oracle_sample(case: W.Case, layer: int, requests: list[int]):
    """Inputs for the oracle on a sample of the workload (generated on the host)."""
    import oracle
    sel = np.asarray(requests)
    L = case.seq_lens[sel]
    T_cap = int(L.max()) + case.T_new
    shape = (len(sel), case.H_kv, T_cap, case.D)
    K = W.normal_bits(shape, case.dtype, case.seed, "cpu_k", layer, std=case.kv_std)
    V = W.normal_bits(shape, case.dtype, case.seed, "cpu_v", layer, std=case.kv_std)
    q = W.normal_bits((len(sel), case.H_q, case.T_new, case.D), case.dtype, case.seed,
                      "cpu_q", layer, std=case.q_std)
    return q, K, V, L, oracle.dtype_code(case.dtype)


def sample_bytes(case: W.Case, requests) -> int:
    L = case.seq_lens[np.asarray(requests)]
    kv = int((L.astype(np.int64) + case.T_new).sum()) * 2 * case.H_kv * case.D * case.elt
    qo = 2 * len(requests) * case.H_q * case.T_new * case.D * case.elt
    app = 2 * len(requests) * case.H_kv * case.T_new * case.D * case.elt
    return kv + qo + app


def time_oracle(case: W.Case, requests: list[int], layers: list[int]) -> tuple[float, int]:
    """Wall time of the oracle's attend over the sample (inputs prepared outside)."""
    import oracle
    o = oracle.get()
    total, nbytes = 0.0, 0
    for layer in layers:
        q, K, V, L, dt = oracle_sample(case, layer, requests)
        t0 = time.perf_counter()
        o.attend(q, K, V, L, case.scale, dt)
        total += time.perf_counter() - t0
        nbytes += sample_bytes(case, requests)
    return total, nbytes


def cpu_baseline(case: W.Case, budget_s: float = 12.0, max_elems: float = 6.4e7) -> dict:
    import oracle
    # requests in order while their K/V stays within max_elems host elements (one at least)
    reqs, elems = [], 0
    for b in range(case.B):
        e = (int(case.seq_lens[b]) + case.T_new) * case.H_kv * case.D
        if reqs and elems + e > max_elems:
            break
        reqs.append(b)
        elems += e
    layers, t, nb = [], 0.0, 0
    for layer in range(case.layers):
        dt, b = time_oracle(case, reqs, [layer])
        layers.append(layer)
        t += dt
        nb += b
        if t >= budget_s:
            break
    return {"value": nb / t / 1e9, "unit": "GB/s", "cores": oracle.threads_used(),
            "kind": "oracle",
            "sample": f"{len(layers)} of {case.layers} layers x {len(reqs)} of {case.B} "
                      f"requests ({case.name}), fp64 C oracle, {t:.1f} s"}


def run_reference(args, case: W.Case) -> None:
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    reqs = [0, 1]  # two requests of one layer per step: a bounded sample
    for w in range(args.warmup):
        time_oracle(case, reqs, [w % case.layers])
    tot, nb = 0.0, 0
    for s in range(args.steps):
        dt, b = time_oracle(case, reqs, [s % case.layers])
        tot += dt
        nb += b
    value = nb / tot / 1e9
    cores = oracle.threads_used()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": case.name, "layers": case.layers, "B": case.B,
                   "H_q": case.H_q, "H_kv": case.H_kv, "D": case.D, "T_past": 4096,
                   "T_new": case.T_new, "cache": "contiguous"},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"each step: 2 of {case.B} requests of one layer "
                                   f"({case.name}), fp64 C oracle"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

class Replicas:
    """One process per GPU running an independent replica of the step.

    The decode step has no cross-request exchange, so the only collectives are
    plumbing around the timed region: a barrier on both sides and the max of
    the ranks' device times (the whole job is as slow as its slowest rank)."""

    def __init__(self, backend: str = "nccl", device=None):
        import torch.distributed as dist
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.device = device
        self.dist = dist
        if self.world > 1 and not dist.is_initialized():
            import datetime
            kw = {"device_id": device} if backend == "nccl" else {}
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)

    def barrier(self) -> None:
        if self.world > 1:
            self.dist.barrier()

    def max_over_ranks(self, x: float) -> float:
        if self.world == 1:
            return x
        import torch
        t = torch.tensor([x], dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self) -> None:
        if self.world > 1 and self.dist.is_initialized():
            self.dist.destroy_process_group()


def whole_job_gbs(world: int, bytes_per_rank_step: int, ms_per_step_max: float) -> float:
    """Algorithmic bytes of all replicas' steps over the slowest rank's step time."""
    return world * bytes_per_rank_step / (ms_per_step_max * 1e-3) / 1e9


class Measured(dict):
    pass


def measure(case: W.Case, kv_format: str, steps: int, warmup: int, samples: int,
            reps: "Replicas", pdl_ab: bool = False, e2e: bool = False, clocks: bool = False):
    """Time one workload: a CUDA graph of one step (every layer), K replays between CUDA
    events (max over ranks); the same step eagerly; optionally the step with the
    dependent launch off; the median duration of `samples` event-bracketed calls of
    the step's kernel; and optionally the end-to-end step from pinned host buffers."""
    import torch
    import kv_cache_decode_03_b200 as kvc

    c = case
    fp8 = kv_format == "fp8"
    tdt = {"fp16": torch.float16, "bf16": torch.bfloat16}[c.dtype]
    cache = kvc.KVCache(c.B, c.H_kv, c.D, c.max_T, c.dtype, c.page_size, c.layers,
                        c.num_pages, kv_format=kv_format)
    bt = torch.from_numpy(c.block_table).cuda() if c.paged else None
    max_pages = c.max_pages if c.paged else 0
    gen = torch.Generator(device="cuda")
    gen.manual_seed(c.seed * 1000 + reps.rank)
    for layer in range(c.layers):
        for which in ("k", "v"):
            pool = cache.pool(layer, which)
            if fp8:  # any finite E4M3 codes, positive scales
                pool.random_(0, 0x7E, generator=gen)
                cache.scales(layer, which).uniform_(1e-3, 1e-2, generator=gen)
            else:
                pool.normal_(0.0, c.kv_std, generator=gen)
    qs = torch.randn((c.layers, c.B, c.H_q, c.T_new, c.D), device="cuda", dtype=tdt,
                     generator=gen) * c.q_std
    ks = torch.randn((c.layers, c.B, c.H_kv, c.T_new, c.D), device="cuda", dtype=tdt,
                     generator=gen) * c.kv_std
    vs = torch.randn((c.layers, c.B, c.H_kv, c.T_new, c.D), device="cuda", dtype=tdt,
                     generator=gen) * c.kv_std
    outs = torch.empty((c.layers, c.B, c.H_q, c.T_new, c.D), device="cuda", dtype=tdt)
    seq = torch.from_numpy(c.seq_lens).cuda()
    cache.reserve(c.H_q, c.T_new, max_pages)
    ns, split_tokens = cache.plan(c.H_q, c.T_new, max_pages)
    stream = torch.cuda.Stream()
    scale = c.scale
    # kvc_append_attend is one attend launch on the persistent stream-K kernels (mma.sync
    # with bf16/fp16 or E4M3 stages, tcgen05 for 17+ rows: the append fused into it, a
    # tcgen05 plan's combine launch after it); the fixed-split plans append in a launch of
    # its own first
    fused = split_tokens == 0

    def step(q=qs, k=ks, v=vs, o=outs):
        for layer in range(c.layers):
            cache.append_attend(layer, k[layer], v[layer], q[layer], seq, bt, scale=scale,
                                out=o[layer], stream=stream)

    def capture():
        with torch.cuda.stream(stream):
            for _ in range(max(3, warmup)):
                step()
            stream.synchronize()
            if cache.get_error() != kvc.KVC_OK:
                raise RuntimeError("device error during warm-up")
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                step()
            for _ in range(3):
                g.replay()
            stream.synchronize()
        return g

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def time_graph(g, n, sampler=None):
        reps.barrier()
        torch.cuda.synchronize()
        ctx = sampler if sampler is not None else _Null()
        with ctx:
            with torch.cuda.stream(stream):
                e0.record(stream)
                for _ in range(n):
                    g.replay()
                e1.record(stream)
            e1.synchronize()
        torch.cuda.synchronize()
        reps.barrier()
        return reps.max_over_ranks(e0.elapsed_time(e1) / n)

    # ---- timed region: K graph replays, device time by CUDA events
    graph = capture()
    clk = ClockSampler(torch.cuda.current_device()) if clocks else None
    ms = time_graph(graph, steps, clk)
    res = Measured(ms=ms, clocks=clk.summary() if clk else None)

    # ---- eager (no graph) step time, for reference
    n_eager = max(3, steps // 4)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(n_eager):
            step()
        e1.record(stream)
    e1.synchronize()
    res["ms_eager"] = e0.elapsed_time(e1) / n_eager

    # ---- the same step with the dependent launch off (plain launches)
    if pdl_ab and fused:
        cache.set_dependent_launch(False)
        g_plain = capture()
        res["ms_no_dependent_launch"] = time_graph(g_plain, steps)
        g_plain.reset()
        del g_plain
        cache.set_dependent_launch(True)

    # ---- per-call duration of the step's kernel(s): median of `samples` bracketed calls
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(c.layers)]
    durs = []
    with torch.cuda.stream(stream):
        while len(durs) < samples:
            for layer in range(c.layers):
                evs[layer][0].record(stream)
                cache.append_attend(layer, ks[layer], vs[layer], qs[layer], seq, bt,
                                    scale=scale, out=outs[layer], stream=stream)
                evs[layer][1].record(stream)
            stream.synchronize()
            durs += [a.elapsed_time(b) for a, b in evs]
    res["call_ms_median"] = statistics.median(durs)
    res["call_samples"] = len(durs)
    if cache.get_error() != kvc.KVC_OK:
        raise RuntimeError("device error in the timed region")

    # ---- e2e: pinned host buffers, every step's copies inside the timed region.  Two
    # device buffer sets and a copy stream, as a serving loop runs it: step i+1's inputs
    # go in, and step i's output comes out, while the compute stream runs the step.
    if e2e:
        hq = qs.cpu().pin_memory()
        hk = ks.cpu().pin_memory()
        hv = vs.cpu().pin_memory()
        ho = torch.empty(outs.shape, dtype=tdt).pin_memory()
        bufs = [(torch.empty_like(qs), torch.empty_like(ks), torch.empty_like(vs),
                 torch.empty_like(outs)) for _ in range(2)]
        copy_stream = torch.cuda.Stream()
        e2e_steps = max(3, steps // 4)
        ev_in = [torch.cuda.Event() for _ in range(2)]    # inputs of buffer set landed
        ev_run = [torch.cuda.Event() for _ in range(2)]   # step on buffer set finished
        ev_out = [torch.cuda.Event() for _ in range(2)]   # its output copied out
        def h2d(i):  # step i's inputs into buffer set i % 2 (copy stream, in order)
            dq, dk, dv, _ = bufs[i % 2]
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)
            ev_in[i % 2].record(copy_stream)

        reps.barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        copy_stream.wait_event(e0)
        with torch.cuda.stream(copy_stream):
            h2d(0)
        for i in range(e2e_steps):
            j = i % 2
            dq, dk, dv, do = bufs[j]
            with torch.cuda.stream(stream):
                stream.wait_event(ev_in[j])
                step(dq, dk, dv, do)
                ev_run[j].record(stream)
            with torch.cuda.stream(copy_stream):
                # the next step's inputs go in while this step runs (their set was last
                # used by step i - 1, whose output copy is queued ahead of them) ...
                if i + 1 < e2e_steps:
                    h2d(i + 1)
                # ... and this step's output comes out while the next one runs
                copy_stream.wait_event(ev_run[j])
                ho.copy_(do, non_blocking=True)
                ev_out[j].record(copy_stream)
        stream.wait_event(ev_out[(e2e_steps - 1) % 2])
        e1.record(stream)
        e1.synchronize()
        reps.barrier()
        res["e2e_ms"] = reps.max_over_ranks(e0.elapsed_time(e1) / e2e_steps)
        res["h2d"] = (hq.numel() + hk.numel() + hv.numel()) * c.elt
        res["d2h"] = ho.numel() * c.elt
    graph.reset()
    del graph
    cache.close()

    # ---- derived figures
    layer_bytes = fp8_algorithmic_bytes(c) if fp8 else c.algorithmic_bytes()
    res["layer_bytes"] = layer_bytes
    res["step_bytes"] = c.layers * layer_bytes
    # tcgen05 stream-K (17+ rows) with large segment merges: attend (append fused), combine
    rows = (c.H_q // c.H_kv) * c.T_new
    segs = c.B * c.H_kv * -(-rows // 128)
    combine = (split_tokens == 0 and rows > 16 and not fp8 and
               ns / segs * min(rows, 128) * c.D * 4 > TC_COMBINE_MIN_BYTES)
    res["launches_per_step"] = c.layers * ((1 if fused else 2) + (1 if combine else 0))
    res["ns"], res["split_tokens"] = ns, split_tokens
    # one call's bytes: K/V read + q read + out written + k_new/v_new read + rows written
    # (the FP8 count already holds both sides of the append)
    call_bytes = layer_bytes + (0 if fp8 else 2 * c.B * c.H_kv * c.T_new * c.D * c.elt)
    res["call_bytes"] = call_bytes
    kernel = attend_kernel_name(c, kv_format, split_tokens)
    # attention flops of one call: 4 per (query row, visible position, dimension); new row
    # i of request b sees L_b + i + 1 positions
    seen = float(sum(int(L) * c.T_new + c.T_new * (c.T_new + 1) // 2 for L in c.seq_lens))
    flops = 4.0 * seen * c.H_q * c.D
    call_s = res["call_ms_median"] * 1e-3
    step_call_s = ms * 1e-3 / c.layers  # one layer-step's share of the graph-timed step
    peak, peak_kind = peaks()
    tpeak, tpeak_kind = tensor_peak()
    # the binding roof: the longer of the bytes' time at the HBM peak and the attention
    # flops' time at the dense bf16 peak (the tensor roof binds from about 240 flop/B,
    # i.e. about 240 query rows per KV head)
    if flops / (tpeak * 1e12) > call_bytes / (peak * 1e9):
        roof = {"bound": "tensor", "achieved": flops / call_s / 1e12, "peak": tpeak,
                "unit": "TFLOP/s", "traffic": profiled_traffic(kernel),
                "peak_source": tpeak_kind, "achieved_in_step": flops / step_call_s / 1e12}
    else:
        roof = {"bound": "hbm", "achieved": call_bytes / call_s / 1e9, "peak": peak,
                "unit": "GB/s", "traffic": profiled_traffic(kernel), "peak_source": peak_kind,
                "achieved_in_step": call_bytes / step_call_s / 1e9}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["frac_in_step"] = roof["achieved_in_step"] / roof["peak"]
    roof["kernel"] = (kernel + (", fused: one launch per kvc_append_attend call (append, "
                                "split attend, merge)" if fused and not combine else
                                ", fused: append and split attend in one launch, then the "
                                "combine launch" if fused else ", after the append kernel"))
    roof["duration"] = (f"median of {len(durs)} event-bracketed kvc_append_attend calls "
                        f"({res['call_ms_median'] * 1e3:.2f} us; each call alone, so without "
                        f"the overlap of the dependent launch); achieved_in_step = the "
                        f"graph-timed step / {c.layers} calls")
    res["roofline"] = roof
    res["kernel"] = kernel
    res["tflops_call"] = flops / call_s / 1e12
    res["tflops_step"] = flops / step_call_s / 1e12
    res["peak"] = peak
    return res


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def workload_summary(name: str, case: W.Case, kv_format: str, r: Measured, world: int) -> dict:
    value = whole_job_gbs(world, r["step_bytes"], r["ms"])
    d = {"workload": case.name, "kv_format": kv_format, "layers": case.layers,
         "value_gbs": value, "pct_of_peak": 100.0 * value / world / r["peak"],
         "ms_per_step": r["ms"], "ms_per_step_eager": r["ms_eager"],
         "tokens_per_s_per_layer_step": world * case.B * case.T_new / (r["ms"] * 1e-3 / case.layers),
         "attention_tflops_step": r["tflops_step"],
         "call_us_median": r["call_ms_median"] * 1e3, "call_samples": r["call_samples"],
         "frac": r["roofline"]["frac"], "frac_in_step": r["roofline"]["frac_in_step"],
         "bound": r["roofline"]["bound"], "kernel": r["kernel"],
         "split_k": {"num_splits": r["ns"], "split_tokens": r["split_tokens"]}}
    if "ms_no_dependent_launch" in r:
        d["ms_per_step_no_dependent_launch"] = r["ms_no_dependent_launch"]
    return d


def run_kvc(args, case: W.Case) -> None:
    import torch

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    reps = Replicas("nccl", torch.device("cuda", local))
    world, rank = reps.world, reps.rank
    c = case
    fp8 = args.kv_format == "fp8"
    r = measure(c, args.kv_format, args.steps, args.warmup, args.launch_samples, reps,
                pdl_ab=True, e2e=True, clocks=True)
    ms = r["ms"]
    value = whole_job_gbs(world, r["step_bytes"], ms)
    peak = r["peak"]
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not fp8:
        cpu = cpu_baseline(c)

    # every other named configuration, bounded, on one GPU (the scaling runs time the
    # headline only)
    extra = {}
    if world == 1 and args.workloads == "all":
        for name, kvf in EXTRA_WORKLOADS:
            if name == args.workload and kvf == args.kv_format:
                continue
            wc = sized_case(name, 0)
            torch.cuda.empty_cache()
            wr = measure(wc, kvf, max(5, min(args.steps, 10)), 3, args.launch_samples, reps,
                         pdl_ab=(name.startswith("mha")))
            key = name + ("_fp8" if kvf == "fp8" else "")
            extra[key] = workload_summary(name, wc, kvf, wr, world)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": c.dtype, "data": "synthetic",
            "config": {"workload": c.name, "layers": c.layers, "B": c.B, "H_q": c.H_q,
                       "H_kv": c.H_kv, "D": c.D,
                       "T_past": (int(c.seq_lens[0]) if len(set(c.seq_lens.tolist())) == 1
                                  else [int(c.seq_lens.min()), int(c.seq_lens.max())]),
                       "T_new": c.T_new,
                       "cache": (f"paged P{c.page_size}" if c.paged else "contiguous") +
                                (", FP8 E4M3 + per-row scales" if fp8 else ""),
                       "parallelism": f"replicas x{world}",
                       "l2": (f"inputs larger than L2 ({r['step_bytes'] / 1e9:.2f} GB read per "
                              f"step over {c.layers} layer caches)"),
                       "split_k": {"num_splits": r["ns"], "split_tokens": r["split_tokens"]},
                       "timing": f"CUDA graph of one {c.layers}-layer step, CUDA events"},
            "pct_of_peak": 100.0 * value / world / peak,
            "tokens_per_s_per_layer_step": world * c.B * c.T_new / (ms * 1e-3 / c.layers),
            "ms_per_step_eager": r["ms_eager"],
            "ms_per_step_no_dependent_launch": r.get("ms_no_dependent_launch"),
            "roofline": r["roofline"],
            "attention_tflops": r["tflops_step"],
            "e2e": {"value": whole_job_gbs(world, r["step_bytes"], r["e2e_ms"]), "unit": "GB/s",
                    "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"],
                    "ms_per_step": r["e2e_ms"]},
            "gpu_launches": r["launches_per_step"] * args.steps,
            "clocks": r["clocks"],
            "cpu_baseline": cpu,
            "workloads": extra or None,
        }
        print(json.dumps(line), flush=True)
    reps.close()


WORKLOADS = {
    "gqa_32layer": lambda: W.gqa_32layer(32),
    "paged_gqa": lambda: W.paged_gqa(),
    "mha_b4_L4096": lambda: W.mha_sweep(4096),
    "mha_b4_L8192": lambda: W.mha_sweep(8192),
    **{f"verify_g{g}_hkv{h}": (lambda g=g, h=h: W.spec_verify(g, h))
       for g in (2, 4, 8) for h in (8, 1)},
}

# the named configurations the default run also measures (bounded), beside the headline
EXTRA_WORKLOADS = [("mha_b4_L4096", "native"), ("mha_b4_L8192", "native"),
                   ("paged_gqa", "native"),
                   *[(f"verify_g{g}_hkv{h}", "native") for h in (8, 1) for g in (2, 4, 8)],
                   ("gqa_32layer", "fp8")]


def sized_case(name: str, layers: int) -> W.Case:
    """The named workload with `layers` layer caches, or by default enough independent
    layer caches that a step reads more than 4x L2."""
    case = WORKLOADS[name]()
    if layers:
        case.layers = layers
    else:
        case.layers = max(case.layers, -(-int(4 * L2_BYTES) // case.kv_read_bytes(True)))
    return case


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="kvc", choices=["kvc", "reference"])
    ap.add_argument("--workload", default="gqa_32layer", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=0,
                    help="override the layer count (a smaller case for profiling)")
    ap.add_argument("--kv-format", default="native", choices=["native", "fp8"],
                    help="K/V storage: the 16-bit type, or FP8 E4M3 with per-row scales")
    ap.add_argument("--launch-samples", type=int, default=64,
                    help="event-bracketed calls whose median gives the per-call duration")
    ap.add_argument("--workloads", default="all", choices=["all", "none"],
                    help="also measure every other named configuration (one GPU only)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    args.launch_samples = max(50, args.launch_samples)
    case = sized_case(args.workload, args.layers)
    if args.impl == "reference":
        run_reference(args, case)
    else:
        run_kvc(args, case)


if __name__ == "__main__":
    main()
