"""Benchmark of the RG-LRU block core on B200: prefill tokens/s and HBM GB/s
against the measured roofline, plus batched decode tokens/s at B=256.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one rglru_prefill call over the whole workload (default: the
2B-shaped block, B=8 T=4096 D=2560 bf16), inputs resident in HBM.  Inputs and
outputs (x, g, y: 168 MB each) are larger than the 126 MB L2, so no flush is
needed between steps.  With N>1 (torchrun, one rank per GPU) every rank runs
the same workload on its own GPU with no data-path collective (weak scaling);
the timed region is bracketed by a barrier and a device synchronize, and the
time is the max over ranks.

Rank 0 prints one JSON line.  ``--impl reference`` times the float64 CPU
oracle on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from lm_causal_depthwise_b200 import workloads as W  # noqa: E402

METRIC = "RG-LRU block prefill tokens/s & HBM GB/s vs peak; decode tok/s at B=256"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
E2E_ROWS = 1  # sequences per chunk of the end-to-end (host-buffer) call


def _env_rank():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), \
        int(os.environ.get("LOCAL_RANK", "0"))


def max_over_ranks(value: float, device="cpu") -> float:
    """The maximum of ``value`` over all ranks of the default process group
    (the value itself without one).  Time-like values are reduced this way, so
    the slowest rank sets the job's time."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sharded_throughput(job_units: int, ms_per_step: float) -> float:
    """Throughput of a job whose units are split across the ranks (strong
    scaling): every unit once, divided by the (max-over-ranks) step time."""
    return job_units / (ms_per_step * 1e-3)


def job_throughput(units_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: the units every rank processed in one step, divided
    by the (max-over-ranks) step time."""
    return units_per_rank * world / (ms_per_step * 1e-3)


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# sources the fused prefill kernel is compiled from: its own file and the
# shared headers (the decode and SIMT kernels live in files of their own)
PREFILL_SOURCES = ("prefill_fused.cu", ".h", ".cuh")


def source_digest() -> str:
    """Digest of the fused prefill kernel's sources, which a traffic record is tied to."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "lm_causal_depthwise_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name == PREFILL_SOURCES[0] or name.endswith(PREFILL_SOURCES[1:]):
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(name.encode())
                h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per launch of the dominant kernel from a committed ncu summary,
    only if it was taken on the current kernel sources."""
    p = os.path.join(ROOT, "profiles", f"traffic_{workload}.json")
    try:
        with open(p) as f:
            d = json.load(f)
    except Exception:
        return None
    if d.get("source_digest") != source_digest():
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML (read-only) in a thread."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index: int, period_s: float = 0.005):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], 0
        self._stop = threading.Event()
        self._t = None
        self.ok = False
        self.max_mhz = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
            return self
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        reasons = [n for bit, n in self.REASONS.items() if self.reasons & bit]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples)}


# ----------------------------------------------------------------------------- reference arm

def cpu_sample_run(w: W.Workload, budget_s: float = 12.0):
    """Times the float64 oracle (as it stands) on a bounded sample of workload
    ``w``: whole sequences of the first rows, all heads.  Returns tokens/s,
    threads used and a description of the sample."""
    from oracle import oracle
    inp = W.generate(w.scaled(B=1))
    t0 = time.perf_counter()
    oracle.prefill(**inp)
    one = time.perf_counter() - t0
    rows = int(max(1, min(w.B, budget_s // max(one, 1e-3))))
    if rows > 1:
        inp = W.generate(w.scaled(B=rows))
        t0 = time.perf_counter()
        oracle.prefill(**inp)
        dt = time.perf_counter() - t0
    else:
        dt = one
    tokens = rows * w.T
    return tokens / dt, oracle.threads(), f"{rows} of {w.B} sequences x T={w.T} x D={w.D} " \
                                          f"(all heads), float64 C oracle, {dt:.1f} s"


def run_reference(args, w):
    rank, world, _ = _env_rank()
    if rank != 0:
        return 0
    from oracle import oracle
    inp = W.generate(w.scaled(B=1))
    cores = oracle.threads()
    for _ in range(max(args.warmup, 0)):
        oracle.prefill(**inp)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.prefill(**inp)
        times.append(time.perf_counter() - t0)
    tot = sum(times)
    value = args.steps * w.T / tot
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.describe(), "sample": "1 sequence per step (all heads, full T)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"1 of {w.B} sequences x T={w.T} x D={w.D} per step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- CUDA arm

def count_launches(fns, prefix=("rglru",)):
    """Kernels of this library launched by each function in ``fns`` (one
    profiler session, CUPTI via torch.profiler).  A marker kernel launched
    between the calls splits the device timeline."""
    import torch
    from torch.profiler import ProfilerActivity, profile
    marker = torch.zeros(1, device="cuda")
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        for fn in fns:
            fn()
            torch.cuda.synchronize()
            marker.add_(1.0)
            torch.cuda.synchronize()
    kern = [e for e in prof.events()
            if e.device_type is not None and str(e.device_type).endswith("CUDA")]
    kern.sort(key=lambda e: e.time_range.start)
    groups, cur = [], []
    for e in kern:
        if any(p in e.name for p in prefix):
            cur.append(e.name)
        elif "add" in e.name.lower() or "elementwise" in e.name.lower():
            groups.append(cur)
            cur = []
    while len(groups) < len(fns):
        groups.append([])
    return [(len(g), sorted(set(g))) for g in groups[:len(fns)]]


OTHER_PREFILL = ("prefill-long", "prefill-long-carry", "prefill-9b")
SUSTAINED_S = 1.0  # the sustained run of the headline workload lasts at least this long


def roofline(alg_bytes: int, ms_per_launch: float, peaks: dict, peak_kind: str, traffic, kernels):
    achieved = alg_bytes / (ms_per_launch * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
            "peak_source": f"{peak_kind} copy bandwidth",
            "frac_of_nominal_8tbs": achieved / 8000.0,
            "algorithmic_bytes_per_launch": alg_bytes, "kernel": kernels}


class PrefillCase:
    """Device buffers of one prefill workload and its timed step."""

    def __init__(self, w, dev, inp=None):
        import torch
        from lm_causal_depthwise_b200 import api
        self.w, self.dev = w, dev
        bf = torch.bfloat16 if w.io == "bf16" else torch.float32
        self.bf = bf
        self.inp = W.generate(w) if inp is None else inp
        inp = self.inp
        self.x = torch.from_numpy(inp["x"]).to(dev).to(bf)
        self.g = torch.from_numpy(inp["g"]).to(dev).to(bf)
        self.sp = torch.from_numpy(inp["segpos"]).to(dev)
        self.cs = torch.from_numpy(inp["conv_state"]).to(dev).to(bf)
        self.hs = torch.from_numpy(inp["h_state"]).to(dev)
        self.p = api.Params.from_arrays(inp, bf, dev)
        self.y = torch.empty_like(self.x)
        self.ws = api.new_workspace(api.workspace_size(w.B, w.T, w.D, bf), dev)

    def step(self):
        from lm_causal_depthwise_b200 import api
        api.prefill(self.x, self.g, self.p, self.sp, self.cs, self.hs, workspace=self.ws, y=self.y)

    def status(self):
        from lm_causal_depthwise_b200 import api
        return api.device_status(self.ws)

    def timed(self, steps: int, stream, distributed: bool, sampler_index=None):
        """Time exactly ``steps`` launches on ``stream`` with CUDA events,
        bracketed by a barrier and a device synchronize; max over ranks."""
        import torch
        import torch.distributed as dist
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if distributed:
            dist.barrier()
        torch.cuda.synchronize()
        with ClockSampler(sampler_index if sampler_index is not None else 0) as clk:
            ev0.record(stream)
            for _ in range(steps):
                self.step()
            ev1.record(stream)
            torch.cuda.synchronize()
        if distributed:
            dist.barrier()
        ms = max_over_ranks(ev0.elapsed_time(ev1), stream.device)
        st = self.status()
        if st != 0:
            from lm_causal_depthwise_b200 import api
            raise RuntimeError(f"{self.w.name}: device status {api.status_string(st)}: no valid timing")
        return ms / steps, clk.summary()


def cpu_sample_tokens(w: W.Workload, budget_s: float):
    """The oracle on a bounded sample of ``w``: whole rows while they fit the
    budget, else the first tokens of one row (all heads)."""
    from oracle import oracle
    probe = min(w.T, 1024)
    inp = W.generate(w.scaled(B=1, T=probe))
    t0 = time.perf_counter()
    oracle.prefill(**inp)
    per_tok = (time.perf_counter() - t0) / probe
    tokens = int(max(probe, min(w.B * w.T, budget_s / max(per_tok, 1e-9))))
    if tokens >= w.T:
        rows, T = min(w.B, tokens // w.T), w.T
    else:
        rows, T = 1, tokens
    inp = W.generate(w.scaled(B=rows, T=T))
    t0 = time.perf_counter()
    oracle.prefill(**inp)
    dt = time.perf_counter() - t0
    return rows * T / dt, oracle.threads(), \
        f"{rows} of {w.B} sequences x first {T} of {w.T} tokens x D={w.D} (all heads), " \
        f"float64 C oracle, {dt:.1f} s"


def copy_only_rates(hx, hg, hsp, hy, stream):
    """Host<->device copy rates of the same pinned buffers the end-to-end call
    uses, measured alone: H2D of x, g and segment_pos, D2H of y, each as one
    cudaMemcpyAsync per tensor on ``stream``."""
    import torch
    dx, dg, dsp = (torch.empty_like(t, device=stream.device) for t in (hx, hg, hsp))
    dy = torch.empty_like(hy, device=stream.device)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def h2d():
        dx.copy_(hx, non_blocking=True)
        dg.copy_(hg, non_blocking=True)
        dsp.copy_(hsp, non_blocking=True)

    def d2h():
        hy.copy_(dy, non_blocking=True)

    out = {}
    for name, fn, nbytes in (("h2d", h2d, hx.nbytes + hg.nbytes + hsp.nbytes), ("d2h", d2h, hy.nbytes)):
        fn()
        torch.cuda.synchronize()
        best = None
        for _ in range(3):
            ev0.record(stream)
            fn()
            ev1.record(stream)
            torch.cuda.synchronize()
            ms = ev0.elapsed_time(ev1)
            best = ms if best is None else min(best, ms)
        out[name] = nbytes / (best * 1e-3) / 1e9
    del dx, dg, dsp, dy
    return out


def run_block(args, dev, stream, distributed, peaks, peak_kind):
    """The whole recurrent block on the 2B shape: linear_x and linear_y in one
    GEMM launch, the fused core, linear_out; timed as a whole (K steps) and per
    launch, with the projections' TFLOP/s against the measured bf16 peak and
    the same GEMM shapes through cuBLAS (torch.nn.functional.linear) for context."""
    import torch
    from lm_causal_depthwise_b200 import api
    w = W.PREFILL_2B
    inp = W.generate_block(w)
    bf = torch.bfloat16
    u = torch.from_numpy(inp["u"]).to(dev).to(bf)
    sp = torch.from_numpy(inp["segpos"]).to(dev)
    cs = torch.from_numpy(inp["conv_state"]).to(dev).to(bf)
    hs = torch.from_numpy(inp["h_state"]).to(dev)
    bp = api.BlockParams.from_arrays(inp, dev)
    out = torch.empty_like(u)
    ws = api.new_workspace(api.recurrent_block_workspace_size(w.B, w.T, w.D), dev)
    M, D = w.B * w.T, w.D
    u2 = u.view(M, D)
    x2, g2, y2 = (torch.empty((M, D), dtype=bf, device=dev) for _ in range(3))
    lws = api.linear_workspace(dev)
    core_ws = api.new_workspace(api.workspace_size(w.B, w.T, w.D, bf), dev)
    x3, g3 = x2.view(w.B, w.T, D), g2.view(w.B, w.T, D)

    def block():
        api.recurrent_block_prefill(u, bp, sp, cs, hs, out=out, workspace=ws)

    def pair():
        api.linear_pair(u2, bp.W_lin_x, bp.b_lin_x, bp.W_lin_y, bp.b_lin_y, out0=x2, out1=g2, workspace=lws)

    def core():
        api.prefill(x3, g3, bp.core, sp, cs, hs, workspace=core_ws, y=y2.view(w.B, w.T, D))

    def outp():
        api.linear(y2, bp.W_out, bp.b_out, out=out.view(M, D), workspace=lws)

    bx16, by16 = bp.b_lin_x.to(bf), bp.b_lin_y.to(bf)  # torch's bf16 linear takes a bf16 bias

    def cublas_pair():
        torch.nn.functional.linear(u2, bp.W_lin_x, bx16)
        torch.nn.functional.linear(u2, bp.W_lin_y, by16)

    def timed(fn, n):
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ev0.record(stream)
        for _ in range(n):
            fn()
        ev1.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(ev0.elapsed_time(ev1), dev) / n

    n = max(3, min(args.steps, 20))
    if distributed:
        import torch.distributed as dist
        dist.barrier()
    ms_block = timed(block, n)
    st = api.device_status(ws)
    if st != api.OK:
        raise RuntimeError(f"recurrent block: device status {api.status_string(st)}")
    ms_pair, ms_core, ms_out, ms_cublas = timed(pair, n), timed(core, n), timed(outp, n), timed(cublas_pair, n)
    pair_flops, out_flops = 2 * 2 * M * D * D, 2 * M * D * D
    world = dist.get_world_size() if distributed else 1
    tflops = lambda f, ms: f / (ms * 1e-3) / 1e12
    return {
        "workload": f"recurrent block (linear_x/linear_y, core, linear_out) B={w.B} T={w.T} D={D} bf16",
        "value": job_throughput(w.tokens, world, ms_block), "unit": "tokens/s", "ms_per_step": ms_block,
        "steps": n, "gemm_flops_per_step": W.block_gemm_flops(w),
        "launches": {"linear_pair_ms": ms_pair, "core_ms": ms_core, "linear_out_ms": ms_out},
        "roofline": {"bound": "tensor", "kernel": "rglru_linear_kernel (linear_x + linear_y, one launch)",
                     "achieved": tflops(pair_flops, ms_pair), "peak": peaks.get("bf16_tflops", 1590.0),
                     "unit": "TFLOP/s", "frac": tflops(pair_flops, ms_pair) / peaks.get("bf16_tflops", 1590.0),
                     "peak_source": f"{peak_kind} cuBLAS bf16 burst", "traffic": None},
        "linear_out_tflops": tflops(out_flops, ms_out),
        "cublas_same_pair_tflops": tflops(pair_flops, ms_cublas),
        "core_hbm_frac": W.algorithmic_bytes(w) / (ms_core * 1e-3) / 1e9 / peaks["hbm_gbs"],
    }


def mqa_valid_pairs(segpos, window: int = 2048) -> int:
    """(query, key) pairs the local MQA attends over: for query t the keys from
    max(t - segment_pos[t], t - window + 1, 0) to t (the attention's
    algorithmic work is 4 * 256 flops per pair and head)."""
    import numpy as np
    t = np.arange(segpos.shape[1])[None, :]
    lo = np.maximum(np.maximum(t - segpos.astype(np.int64), t - window + 1), 0)
    return int((t - lo + 1).sum())


def run_mqa(args, dev, stream, distributed, peaks, peak_kind):
    """The local MQA temporal block on the 2B shape (B=8, T=4096, D=2560: 10
    query heads, one key/value head, window 2048, documents of mean length
    1024): the QKV projection, RoPE, the attention kernel and o_proj, timed as a
    whole and per launch; the attention kernel against the measured bf16 peak."""
    import torch
    from lm_causal_depthwise_b200 import api
    w = W.PREFILL_2B
    inp = W.generate_mqa(w)
    bf = torch.bfloat16
    B, T, D = w.B, w.T, w.D
    H, M = D // 256, B * T
    u = torch.from_numpy(inp["u"]).to(dev).to(bf)
    sp = torch.from_numpy(inp["segpos"]).to(dev)
    mp = api.MQAParams.from_arrays(inp, dev)
    out = torch.empty_like(u)
    ws = api.new_workspace(api.mqa_block_workspace_size(B, T, D), dev)
    qkv = torch.empty((B, T, D + 512), dtype=bf, device=dev)
    vt = api.mqa_vt(B, T, dev)
    att = torch.empty((B, T, D), dtype=bf, device=dev)
    lws = api.linear_workspace(dev)
    api.linear(u.view(M, D), mp.W_qkv, None, out=qkv.view(M, D + 512), workspace=lws)
    api.mqa_rope(qkv, sp, vt)

    def block():
        api.mqa_block_prefill(u, mp, sp, out=out, workspace=ws)

    def proj():
        api.linear(u.view(M, D), mp.W_qkv, None, out=qkv.view(M, D + 512), workspace=lws)

    def rope():
        api.mqa_rope(qkv, sp, vt)

    def attention():
        api.mqa_attention(qkv, vt, sp, out=att, workspace=lws)

    def oproj():
        api.linear(att.view(M, D), mp.W_o, mp.b_o, out=out.view(M, D), workspace=lws)

    def timed(fn, n):
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ev0.record(stream)
        for _ in range(n):
            fn()
        ev1.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(ev0.elapsed_time(ev1), dev) / n

    n = max(3, min(args.steps, 20))
    if distributed:
        import torch.distributed as dist
        dist.barrier()
    ms_block = timed(block, n)
    for wsp, what in ((ws, "mqa block"), (lws, "mqa launches")):
        st = api.device_status(wsp)
        if st != api.OK:
            raise RuntimeError(f"{what}: device status {api.status_string(st)}")
    ms_attn = timed(attention, n)
    ms_proj, ms_rope, ms_o = timed(proj, n), timed(rope, n), timed(oproj, n)
    st = api.device_status(lws)
    if st != api.OK:
        raise RuntimeError(f"mqa launches: device status {api.status_string(st)}")
    pairs = mqa_valid_pairs(inp["segpos"])
    attn_flops = 4 * 256 * H * pairs
    peak = peaks.get("bf16_tflops", 1590.0)
    achieved = attn_flops / (ms_attn * 1e-3) / 1e12
    world = dist.get_world_size() if distributed else 1
    rope_bytes = M * (2 * (D + 256) * 2 + 2 * 256 * 2)   # q, k read and written; v read, v_t written
    return {
        "workload": f"local MQA block (QKV projection, RoPE, attention, o_proj) B={B} T={T} D={D} H={H} "
                    f"window 2048, documents of mean length {w.doc_len}, bf16",
        "value": job_throughput(w.tokens, world, ms_block), "unit": "tokens/s", "ms_per_step": ms_block,
        "steps": n,
        "launches": {"qkv_proj_ms": ms_proj, "rope_ms": ms_rope, "attention_ms": ms_attn, "o_proj_ms": ms_o},
        "attention_pairs": pairs, "attention_flops": attn_flops,
        "roofline": {"bound": "tensor", "kernel": "rglru_mqa_attention_kernel", "achieved": achieved, "peak": peak,
                     "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_source": f"{peak_kind} cuBLAS bf16 burst", "traffic": None},
        "qkv_proj_tflops": 2 * M * D * (D + 512) / (ms_proj * 1e-3) / 1e12,
        "o_proj_tflops": 2 * M * D * D / (ms_o * 1e-3) / 1e12,
        "rope_hbm_frac": rope_bytes / (ms_rope * 1e-3) / 1e9 / peaks["hbm_gbs"],
    }


def run_mqa_decode(args, dev, stream, distributed, peaks, peak_kind):
    """One local-MQA decode step for B=256 sequences (10 query heads, window
    2048): RoPE, the cache write, the split-KV attention and the combine, timed
    as a 64-step CUDA graph.  Positions: the decode-2b recipe's document
    positions at its last step; the rings hold synthetic bf16 keys and values.
    HBM roofline: every attended key and value (512 B each) read once, the
    token's qkv read, its cache slot and output written."""
    import numpy as np
    import torch
    from lm_causal_depthwise_b200 import api
    wd = W.DECODE_2B
    B, H, window = wd.B, wd.H, 2048
    rng = np.random.default_rng((wd.seed, 4))
    seg = W.segment_positions(rng, wd)[:, -1].astype(np.int32)
    bf = torch.bfloat16
    g = torch.Generator(device="cpu").manual_seed(wd.seed)
    qkv = torch.randn((B, (H + 2) * 256), generator=g).to(bf).to(dev)
    kc = torch.randn((B, window, 256), generator=g).to(bf).to(dev)
    vc = torch.randn((B, 256, window), generator=g).to(bf).to(dev)
    sp = torch.from_numpy(seg).to(dev)
    out = torch.empty((B, H * 256), dtype=bf, device=dev)
    ws = api.new_workspace(api.mqa_decode_workspace_size(B, H, window), dev)
    steps = 64

    def step():
        api.mqa_decode_step(qkv, sp, kc, vc, out=out, workspace=ws)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    s2 = torch.cuda.Stream(dev)
    s2.wait_stream(torch.cuda.current_stream(dev))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s2):
        step()
        torch.cuda.synchronize()
        with torch.cuda.graph(graph, stream=s2):
            for _ in range(steps):
                step()
    torch.cuda.synchronize()
    graph.replay()
    torch.cuda.synchronize()
    if distributed:
        import torch.distributed as dist
        dist.barrier()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = max(3, min(args.steps, 10))
    ev0.record(stream)
    for _ in range(reps):
        graph.replay()
    ev1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(ev0.elapsed_time(ev1), dev) / (reps * steps)
    del graph
    n = np.minimum(seg.astype(np.int64) + 1, window)
    alg = int(n.sum()) * 2 * 512 + B * (H + 2) * 512 + B * 2 * 512 + B * H * 512
    world = dist.get_world_size() if distributed else 1
    gbs = alg / (ms * 1e-3) / 1e9
    return {
        "workload": f"local MQA decode step B={B} H={H} window {window}, positions of the decode-2b recipe "
                    f"(mean {float(n.mean()):.0f} keys per sequence), bf16",
        "value": job_throughput(B, world, ms), "unit": "tokens/s", "us_per_step": ms * 1e3,
        "graph_steps": steps, "algorithmic_bytes_per_step": alg,
        "roofline": {"bound": "hbm", "kernel": "rglru_mqa_decode_kernel + combine", "achieved": gbs,
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                     "peak_source": "measured copy bandwidth", "traffic": None},
    }


def run_residual_block(args, dev, stream, distributed, peaks, peak_kind):
    """The whole recurrent residual block on the 2B shape (RMSNorm, the
    recurrent block with linear_out's residual add in its epilogue, RMSNorm,
    the GELU-gated MLP up projection, the down projection with the residual
    add): seven launches per step, timed as a whole, plus the MLP GEMMs alone."""
    import torch
    from lm_causal_depthwise_b200 import api
    w = W.PREFILL_2B
    inp = W.generate_residual_block(w)
    bf = torch.bfloat16
    u = torch.from_numpy(inp["u"]).to(dev).to(bf)
    sp = torch.from_numpy(inp["segpos"]).to(dev)
    cs = torch.from_numpy(inp["conv_state"]).to(dev).to(bf)
    hs = torch.from_numpy(inp["h_state"]).to(dev)
    rp = api.ResidualBlockParams.from_arrays(inp, dev)
    F = rp.W_gate.shape[0]
    out = torch.empty_like(u)
    ws = api.new_workspace(api.residual_block_workspace_size(w.B, w.T, w.D, F), dev)
    M, D = w.tokens, w.D
    a2 = u.view(M, D)
    m2 = torch.empty((M, F), dtype=bf, device=dev)
    lws = api.linear_workspace(dev)

    def step():
        api.residual_block_prefill(u, rp, sp, cs, hs, out=out, workspace=ws)

    def up():
        api.linear_geglu(a2, rp.W_gate, rp.b_gate, rp.W_up, rp.b_up, out=m2, workspace=lws)

    def down():
        api.linear_residual(m2, rp.W_down, rp.b_down, a2, out=out.view(M, D), workspace=lws)

    def timed(fn, n):
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ev0.record(stream)
        for _ in range(n):
            fn()
        ev1.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(ev0.elapsed_time(ev1), dev) / n

    n = max(3, min(args.steps, 20))
    ms = timed(step, n)
    st = api.device_status(ws)
    if st != api.OK:
        raise RuntimeError(f"residual block: device status {api.status_string(st)}")
    ms_up, ms_down = timed(up, n), timed(down, n)
    world = torch.distributed.get_world_size() if distributed else 1
    up_flops, down_flops = 2 * 2 * M * D * F, 2 * M * F * D
    return {
        "workload": f"recurrent residual block (RMSNorm, recurrent block, residual, RMSNorm, GELU-gated MLP "
                    f"F={F}, residual) B={w.B} T={w.T} D={D} bf16",
        "value": job_throughput(w.tokens, world, ms), "unit": "tokens/s", "ms_per_step": ms, "steps": n,
        "gemm_flops_per_step": W.residual_block_gemm_flops(w),
        "gemm_tflops_whole_step": W.residual_block_gemm_flops(w) / (ms * 1e-3) / 1e12,
        "mlp_up_geglu_tflops": up_flops / (ms_up * 1e-3) / 1e12, "mlp_up_ms": ms_up,
        "mlp_down_residual_tflops": down_flops / (ms_down * 1e-3) / 1e12, "mlp_down_ms": ms_down,
        "peak_bf16_tflops": peaks.get("bf16_tflops", 1590.0), "peak_source": f"{peak_kind} cuBLAS bf16 burst",
    }


def run_time_sharded(args, w, dev, stream, rank, world, local, distributed):
    """--shard time: each sequence of the workload split along time over the
    ranks, one contiguous chunk of tokens per rank.  A step: the chunk from h = 0
    and from h = 1 (its end states H0, H1), one all-gather of those end states,
    rglru_carry_scan for the state every chunk starts from, the chunk once more
    from its own carried state.  Three passes over each chunk, so the job runs
    at most world / 3 times faster than one GPU (head sharding, where there are
    heads to spread, has no such factor).  Strong scaling: the job's tokens once
    over the max-over-ranks step time."""
    import numpy as np
    import torch
    import torch.distributed as dist
    from lm_causal_depthwise_b200 import api
    from lm_causal_depthwise_b200.sharding import shard_time, shard_time_inputs
    if world > w.T:
        raise SystemExit(f"--shard time needs at least one token per GPU: T = {w.T}, {world} GPUs")
    t0, t1 = shard_time(w.T, world, rank)
    inp = W.generate(w)
    part = w.scaled(T=t1 - t0)
    case = PrefillCase(part, dev, inp=shard_time_inputs(inp, t0, t1))
    h_first = torch.from_numpy(inp["h_state"]).to(dev)
    cs0 = case.cs.clone()
    ends = torch.empty((2, w.B, w.D), dtype=torch.float32, device=dev)  # this chunk's H0, H1
    gathered = torch.empty((world, 2, w.B, w.D), dtype=torch.float32, device=dev)
    H0 = torch.empty((world, w.B, w.D), dtype=torch.float32, device=dev)
    H1 = torch.empty_like(H0)
    h_in = torch.empty_like(H0)

    def step():
        for k, h in enumerate((0.0, 1.0)):
            case.hs.fill_(h)
            case.cs.copy_(cs0)
            case.step()
            ends[k].copy_(case.hs)
        if distributed:
            dist.all_gather_into_tensor(gathered, ends)
        else:
            gathered[0].copy_(ends)
        H0.copy_(gathered[:, 0])
        H1.copy_(gathered[:, 1])
        api.carry_scan(H0, H1, h_first, h_in)
        case.hs.copy_(h_in[rank])
        case.cs.copy_(cs0)
        case.step()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if distributed:
        dist.barrier()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
    if distributed:
        dist.barrier()
    per_step_ms = max_over_ranks(ev0.elapsed_time(ev1) / args.steps, dev)
    st = case.status()
    if st != api.OK:
        raise RuntimeError(f"time-sharded prefill: device status {api.status_string(st)}")
    if distributed:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    peaks, peak_kind = measured_peaks()
    line = {
        "metric": METRIC, "value": sharded_throughput(w.tokens, per_step_ms), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step_ms, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "bf16" if w.io == "bf16" else "f32",
        "data": "synthetic",
        "config": {"workload": w.describe(), "B": w.B, "T": w.T, "D": w.D, "tokens_per_job": w.tokens,
                   "parallelism": f"time split over {world} GPU(s): three passes per chunk and one all-gather "
                                  f"of the chunks' end states; rank 0 has tokens [{t0}, {t1})",
                   "l2": "no flush: on prefill-long a chunk's x, g and y together exceed L2 (126 MB) "
                         "up to 8 GPUs"},
        "roofline": roofline(W.algorithmic_bytes(w), per_step_ms * world, peaks, peak_kind, None, None),
        "roofline_note": "achieved per GPU: the job's algorithmic bytes / world over the step time (each chunk "
                         "is read three times)",
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


def run_head_sharded(args, w, dev, stream, rank, world, local, distributed):
    """--shard heads: the workload's heads split across the ranks (no
    collective on the data path; each rank's output is a column block of the
    whole output).  The job's work is fixed (strong scaling): its tokens once,
    over the max-over-ranks step time."""
    import torch
    import torch.distributed as dist
    from lm_causal_depthwise_b200.sharding import shard_heads, shard_inputs
    h0, h1 = shard_heads(w.H, world, rank)
    ms = 0.0
    clocks = None
    if h1 > h0:
        part = w.scaled(D=(h1 - h0) * W.HEAD)
        case = PrefillCase(part, dev, inp=shard_inputs(W.generate(w), h0, h1))
        for _ in range(args.warmup):
            case.step()
        torch.cuda.synchronize()
        ms, clocks = case.timed(args.steps, stream, False, local)
    if distributed:
        dist.barrier()
    per_step_ms = max_over_ranks(ms, dev)
    if distributed:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    peaks, peak_kind = measured_peaks()
    line = {
        "metric": METRIC, "value": sharded_throughput(w.tokens, per_step_ms), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step_ms, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "bf16" if w.io == "bf16" else "f32",
        "data": "synthetic",
        "config": {"workload": w.describe(), "B": w.B, "T": w.T, "D": w.D, "tokens_per_job": w.tokens,
                   "parallelism": f"heads split over {world} GPU(s), rank 0 has heads [{h0}, {h1})",
                   "l2": "no flush: the shards' x, g, y exceed L2 at the sizes timed"},
        "roofline": roofline(W.algorithmic_bytes(w), per_step_ms * world, peaks, peak_kind, None, None),
        "roofline_note": "achieved per GPU: the job's algorithmic bytes / world over the step time",
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_cuda(args, w):
    import torch
    import torch.distributed as dist
    from lm_causal_depthwise_b200 import api

    rank, world, local = _env_rank()
    distributed = world > 1
    if distributed:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    api.load()

    if args.profile_run and w.decode_steps:
        return profile_decode(args, w, dev, rank, distributed)
    if args.shard != "none" and w.decode_steps:
        raise SystemExit(f"--shard {args.shard} times prefill workloads; {w.name} is a decode workload")
    if args.shard == "time":
        return run_time_sharded(args, w, dev, stream, rank, world, local, distributed)
    if args.shard == "heads":
        return run_head_sharded(args, w, dev, stream, rank, world, local, distributed)
    if args.profile_mqa:
        # only the local MQA block's launches, warm-up then timed
        peaks0, kind0 = measured_peaks()
        r = run_mqa(args, dev, stream, distributed, peaks0, kind0)
        rd = run_mqa_decode(args, dev, stream, distributed, peaks0, kind0)
        if rank == 0:
            print(json.dumps({"profile_mqa": r["workload"], "ms_per_step": r["ms_per_step"],
                              "attention_ms": r["launches"]["attention_ms"], "roofline": r["roofline"],
                              "decode": {"us_per_step": rd["us_per_step"], "roofline": rd["roofline"],
                                         "workload": rd["workload"]}}))
        if distributed:
            dist.destroy_process_group()
        return 0
    if args.profile_block:
        # only the residual block's launches (RMSNorm, projections, core,
        # MLP), warm-up then timed: the command an ncu launch list wraps
        peaks0, kind0 = measured_peaks()
        r = run_residual_block(args, dev, stream, distributed, peaks0, kind0)
        if rank == 0:
            print(json.dumps({"profile_block": r["workload"], "ms_per_step": r["ms_per_step"]}))
        if distributed:
            dist.destroy_process_group()
        return 0
    case = PrefillCase(w, dev)
    for _ in range(args.warmup):
        case.step()
    torch.cuda.synchronize()
    if args.profile_run:
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(args.steps):
            case.step()
        ev1.record(stream)
        torch.cuda.synchronize()
        st = case.status()
        if rank == 0:
            print(json.dumps({"profile_run": w.describe(), "steps": args.steps,
                              "ms_per_step": ev0.elapsed_time(ev1) / args.steps, "device_status": st}))
        if distributed:
            dist.destroy_process_group()
        return 0 if st == 0 else 1
    dec_setup = None if args.no_decode else setup_decode(args, dev)
    fns = [case.step] + ([dec_setup["one"]] if dec_setup else [])
    counts = count_launches(fns)
    launches_per_step, kernel_names = counts[0]

    # ---- the contract's timed region: exactly K steps
    per_step_ms, clocks = case.timed(args.steps, stream, distributed, local)
    value = job_throughput(w.tokens, world, per_step_ms)
    # ---- the same workload sustained for >= SUSTAINED_S (a stable clock record)
    n_sus = int(max(args.steps, math.ceil(SUSTAINED_S / (per_step_ms * 1e-3))))
    if distributed:
        n_sus = int(max_over_ranks(n_sus, dev))
    sus_ms, sus_clocks = case.timed(n_sus, stream, distributed, local)

    # ---- end to end through the public API: rglru_prefill_host reads the
    # pinned host inputs and writes y back to host memory, its copies
    # overlapped with the kernels chunk by chunk (E2E_ROWS sequences each)
    bf = case.bf
    hx = torch.from_numpy(case.inp["x"]).to(bf).pin_memory()
    hg = torch.from_numpy(case.inp["g"]).to(bf).pin_memory()
    hsp = torch.from_numpy(case.inp["segpos"]).pin_memory()
    hy = torch.empty(tuple(case.y.shape), dtype=bf).pin_memory()
    e_steps = max(3, min(args.steps, 20))
    e_rows = min(w.B, E2E_ROWS)
    staging = torch.empty(api.prefill_host_staging_size(w.B, w.T, w.D, bf, e_rows), dtype=torch.uint8,
                          device=dev)
    ws_host = api.new_workspace(api.workspace_size(e_rows, w.T, w.D, bf), dev)

    def e2e_step():
        api.prefill_host(hx, hg, case.p, hsp, case.cs, case.hs, hy, rows_per_chunk=e_rows, staging=staging,
                         workspace=ws_host)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    if distributed:
        dist.barrier()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(e_steps):
        e2e_step()
    ev1.record(stream)
    torch.cuda.synchronize()
    e_ms = max_over_ranks(ev0.elapsed_time(ev1), dev) / e_steps
    e_value = job_throughput(w.tokens, world, e_ms)
    st = api.device_status(ws_host)
    if st != api.OK:
        raise RuntimeError(f"prefill reported device status {api.status_string(st)} in the e2e loop")
    h2d = hx.nbytes + hg.nbytes + hsp.nbytes
    d2h = hy.nbytes
    copy_rates = copy_only_rates(hx, hg, hsp, hy, stream)
    del hx, hg, hy, hsp, staging, ws_host
    del case
    torch.cuda.empty_cache()

    # ---- the other prefill workloads, each timed the same way (K steps)
    others = []
    if not args.headline_only:
        for name in OTHER_PREFILL:
            ow = W.ALL[name]
            oc = PrefillCase(ow, dev)
            for _ in range(args.warmup):
                oc.step()
            torch.cuda.synchronize()
            o_ms, o_clk = oc.timed(max(3, min(args.steps, 20)), stream, distributed, local)
            others.append((ow, o_ms, o_clk, max(3, min(args.steps, 20))))
            del oc
            torch.cuda.empty_cache()

    # ---- batched decode at B=256 (a separate timed loop of single-token steps)
    dec = None
    if dec_setup is not None:
        dec = run_decode(dec_setup, counts[1], stream, distributed)
        del dec_setup
        torch.cuda.empty_cache()

    # ---- the whole recurrent block (projections around the core)
    blk = None
    if not args.headline_only:
        peaks0, kind0 = measured_peaks()
        blk = run_block(args, dev, stream, distributed, peaks0, kind0)
        torch.cuda.empty_cache()
        blk["residual_block"] = run_residual_block(args, dev, stream, distributed, peaks0, kind0)
        torch.cuda.empty_cache()
        blk["mqa_block"] = run_mqa(args, dev, stream, distributed, peaks0, kind0)
        torch.cuda.empty_cache()
        blk["mqa_decode"] = run_mqa_decode(args, dev, stream, distributed, peaks0, kind0)
        torch.cuda.empty_cache()

    if distributed:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks, peak_kind = measured_peaks()
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if w.io == "bf16" else "f32", "data": "synthetic",
        "config": {"workload": w.describe(), "B": w.B, "T": w.T, "D": w.D,
                   "tokens_per_gpu": w.tokens, "parallelism": f"replicas x{world}" if world > 1 else "1 GPU",
                   "l2": "no flush: x, g, y are each larger than L2 (126 MB)"},
        "hbm_gbs": W.algorithmic_bytes(w) / (per_step_ms * 1e-3) / 1e9,
        "roofline": roofline(W.algorithmic_bytes(w), per_step_ms, peaks, peak_kind, recorded_traffic(w.name),
                             kernel_names),
        "e2e": {"value": e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e_steps,
                "api": f"rglru_prefill_host, {e_rows} sequence(s) per chunk",
                "ms_per_step": e_ms,
                "h2d_gbs": h2d / (e_ms * 1e-3) / 1e9, "d2h_gbs": d2h / (e_ms * 1e-3) / 1e9,
                "copy_only_h2d_gbs": copy_rates["h2d"], "copy_only_d2h_gbs": copy_rates["d2h"],
                "h2d_frac_of_copy_only": h2d / (e_ms * 1e-3) / 1e9 / copy_rates["h2d"]},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "sustained": {"steps": n_sus, "seconds": n_sus * sus_ms * 1e-3, "ms_per_step": sus_ms,
                      "value": job_throughput(w.tokens, world, sus_ms), "unit": "tokens/s",
                      "roofline_frac": W.algorithmic_bytes(w) / (sus_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                      "clocks": sus_clocks},
        "source_digest": source_digest(),
    }
    cpu_on = world == 1 and not args.no_cpu_baseline
    if others:
        rows = []
        for ow, o_ms, o_clk, o_steps in others:
            r = {"workload": ow.describe(), "value": job_throughput(ow.tokens, world, o_ms), "unit": "tokens/s",
                 "ms_per_step": o_ms, "steps": o_steps, "tokens_per_gpu": ow.tokens,
                 "hbm_gbs": W.algorithmic_bytes(ow) / (o_ms * 1e-3) / 1e9,
                 "roofline": roofline(W.algorithmic_bytes(ow), o_ms, peaks, peak_kind,
                                      recorded_traffic(ow.name), kernel_names),
                 "tensor_tflops": W.gate_flops(ow) / (o_ms * 1e-3) / 1e12,
                 "clocks": o_clk}
            if cpu_on:
                v, cores, sample = cpu_sample_tokens(ow, 4.0)
                r["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                     "sample": sample}
            rows.append(r)
        line["prefill_workloads"] = rows
    if dec is not None:
        line["decode"] = dec
    if blk is not None:
        mqa = {"prefill_block": blk.pop("mqa_block", None), "decode_step": blk.pop("mqa_decode", None)}
        line["recurrent_block"] = blk
        line["local_mqa"] = mqa
    if cpu_on:
        v, cores, sample = cpu_sample_run(w)
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                "sample": sample}
    print(json.dumps(line), flush=True)
    return 0


def profile_decode(args, w, dev, rank, distributed):
    """--profile-run on a decode workload: warm-up and timed single-token steps
    launched one by one (the command an ncu capture of the decode kernel wraps)."""
    import torch
    import torch.distributed as dist
    args.decode_steps = args.decode_steps or (args.warmup + args.steps)
    d = setup_decode(args, dev)
    for t in range(args.warmup):
        d["one"](t % d["steps"])
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for t in range(args.steps):
        d["one"]((args.warmup + t) % d["steps"])
    ev1.record(stream)
    torch.cuda.synchronize()
    st = d["status"]()
    if rank == 0:
        print(json.dumps({"profile_run": w.describe(), "steps": args.steps,
                          "us_per_step": 1e3 * ev0.elapsed_time(ev1) / args.steps, "device_status": st}))
    if distributed:
        dist.destroy_process_group()
    return 0 if st == 0 else 1


def setup_decode(args, dev):
    """Device buffers of the batched decode workload: B=256 sequences, one
    token per step, inputs of every step resident in HBM."""
    import torch
    from lm_causal_depthwise_b200 import api

    w = W.DECODE_2B
    steps = args.decode_steps or w.decode_steps
    inp = W.generate(w.scaled(T=steps))
    bf = torch.bfloat16
    d = dict(w=w, steps=steps)
    d["xs"] = torch.from_numpy(inp["x"]).to(dev).to(bf).transpose(0, 1).contiguous()
    d["gs"] = torch.from_numpy(inp["g"]).to(dev).to(bf).transpose(0, 1).contiguous()
    d["ss"] = torch.from_numpy(inp["segpos"]).to(dev).t().contiguous()
    d["cs"] = torch.from_numpy(inp["conv_state"]).to(dev).to(bf)
    d["hs"] = torch.from_numpy(inp["h_state"]).to(dev)
    d["p"] = api.Params.from_arrays(inp, bf, dev)
    d["ys"] = torch.empty_like(d["xs"])
    d["ws"] = api.new_workspace(api.decode_workspace_size(w.B, w.D, bf), dev)

    def one(t=0):
        api.decode_step(d["xs"][t], d["gs"][t], d["p"], d["ss"][t], d["cs"], d["hs"],
                        workspace=d["ws"], y=d["ys"][t])

    def loop():
        for t in range(steps):
            one(t)
    d["one"], d["loop"] = one, loop
    d["status"] = lambda: api.device_status(d["ws"])
    return d


def run_decode(d, launch_count, stream, distributed):
    import torch
    import torch.distributed as dist

    w, steps = d["w"], d["steps"]
    d["loop"]()
    torch.cuda.synchronize()
    # the whole step loop as one CUDA graph: one kernel node per step, replayed
    # without host launch overhead between steps
    side = torch.cuda.Stream(device=stream.device)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        d["loop"]()
    stream.wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        d["loop"]()
    torch.cuda.synchronize()
    graph.replay()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if distributed:
        dist.barrier()
    torch.cuda.synchronize()
    ev0.record(stream)
    graph.replay()
    ev1.record(stream)
    torch.cuda.synchronize()
    st = d["status"]()
    del graph
    if st != 0:
        raise RuntimeError(f"decode reported device status {st}: no valid timing")
    ms = max_over_ranks(ev0.elapsed_time(ev1), stream.device)
    world = dist.get_world_size() if distributed else 1
    per_step_us = 1e3 * ms / steps
    step_bytes = W.decode_step_bytes(w)
    n_launch, names = launch_count
    return {"workload": w.scaled(T=steps).describe(), "value": job_throughput(w.B, world, ms / steps),
            "unit": "tokens/s", "us_per_step": per_step_us, "steps": steps,
            "algorithmic_gbs": step_bytes / (per_step_us * 1e-6) / 1e9,
            "algorithmic_bytes_per_step": step_bytes, "gpu_launches": n_launch * steps,
            "kernel": names, "launch": "CUDA graph of the step loop"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=W.PREFILL_2B.name, choices=sorted(W.ALL))
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--decode-steps", type=int, default=0)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-mqa", action="store_true",
                    help="run only the local MQA block's launches (for an ncu launch list)")
    ap.add_argument("--profile-block", action="store_true",
                    help="only the recurrent residual block's steps (the command an ncu launch list of "
                         "the block kernels wraps)")
    ap.add_argument("--shard", default="none", choices=["none", "heads", "time"],
                    help="none: one replica of the workload per GPU (weak scaling); heads: the workload's "
                         "heads split across the GPUs (strong scaling); time: each sequence split along "
                         "time, one all-gather of the chunks' end states per step (strong scaling)")
    ap.add_argument("--headline-only", action="store_true",
                    help="time only the headline prefill workload (not the other prefill workloads)")
    ap.add_argument("--profile-run", action="store_true",
                    help="only the warm-up and timed prefill steps (no profiler, e2e, decode or "
                         "CPU legs): the command an ncu capture wraps")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "cuda":
        args.warmup = 3
    w = W.ALL[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    return run_cuda(args, w)


if __name__ == "__main__":
    sys.exit(main())
