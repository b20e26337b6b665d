"""Benchmark of the MXFP4 MoE layer (one JSON line on stdout from rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one moe_layer_forward call (route -> permute -> grouped gate/up
GEMM + SwiGLU -> grouped down GEMM -> combine) over one batch of seeded
synthetic tokens with the workload's shapes; the MXFP4 weights are quantised
once, before timing, by the library's mxfp4_quantize.  L2 is flushed (a
256 MiB device write) before every timed step, outside the timed events.

The line's own fields are the largest single-GPU workload, the skewed
120B-shaped prefill batch (T 16384, E 128); ``per_workload`` carries the same
fields for the other four workloads (tiny, 20B decode, 20B prefill, 120B
decode), timed in the same run.  ``--workload NAME`` times that one alone.

* value: tokens/s of the whole job (all ranks), inputs resident in HBM, from
  CUDA events around each step on the launching stream, max over ranks.
* e2e: the same metric through the same C-ABI call with host buffers: the
  step's x and logits are copied from pinned host memory and the output is
  copied back inside the timed region.
* roofline: the grouped expert MLP (moe_expert_mlp: the GEMM launches that
  dominate the step, with the tile plan and, on the block-scaled path, the
  split of the input rows), algorithmic bytes (or FLOPs) per call / its event
  time, against the measured HBM copy bandwidth (or the measured bf16 tensor
  rate), whichever roofline term of the call is larger.
* cpu_baseline: the fp64 CPU oracle, as it stands, on the host cores, over
  the first 64 tokens of the batch (all of them when it has fewer), with the
  weights of the experts they route to quantised beforehand (rank 0, one GPU
  only).  The reference arm times the same sample per step.
* router: moe_router_topk (router scores fused with the top-k) on the
  headline workload's tokens against a seeded router matrix.
* unquantised: at the 20B decode batch, the grouped expert MLP on the
  unquantised bf16 weights (moe_expert_mlp_unquantised) beside the MXFP4 one,
  weight bytes streamed and time of each.
* quantize: the quantisers timed on their own (mxfp4_quantize, and
  mxfp4_quantize_sr_rht with the random-sign Hadamard transform and
  stochastic rounding) over the first chunk of the headline workload's bf16
  gate/up weights, GB/s of algorithmic bytes against the HBM copy peak.
Under torchrun each rank runs its own replica of every workload on its own
GPU (independent token batches, no collective on the data path): weak
scaling.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic as syn  # noqa: E402

METRIC = "MoE-layer tokens/s on 1 B200; % of roofline (HBM GB/s decode, TC TFLOP/s prefill)"
UNIT = "tokens/s"
HEADLINE = "120b_skewed_prefill"
OTHERS = ["120b_decode", "20b_decode", "20b_prefill", "tiny"]
FLUSH_BYTES = 256 << 20
CPU_SAMPLE_TOKENS = 64
# the unquantised (bf16 weight) expert MLP is timed beside the MXFP4 one here
UNQUANTISED_AT = "20b_decode"
# kernel launches of one moe_layer_forward call, per GEMM path:
#   block-scaled: route, permute (with the GEMMs' tile list), the split of the
#     rows straight from x into E4M3 pieces, one launch running both GEMMs,
#     combine;
#   bf16-decode: route, permute, the row gather, the gate/up GEMM, the down
#     GEMM, combine
LAUNCHES_PER_LAYER = {"block-scaled": 5, "bf16-decode": 6}
LAUNCH_NOTE = ("step = one replay of a CUDA graph holding one moe_layer_forward call (5 kernels "
               "on the block-scaled path, 6 on the bf16-decode path), captured once per "
               "workload; 'eager' = the same call launched per step")

# dram bytes (read + write) of one moe_expert_mlp call per workload, from ncu
# captures of the GEMM kernels of the source file named beside them, reported
# only while that file's device code (comments and whitespace aside) still
# hashes to the value recorded with them
TRAFFIC: dict[str, tuple[int, str, str]] = {
    # gate/up + down GEMM dram__bytes_read.sum + dram__bytes_write.sum, one
    # launch each, from `ncu --set full` captures of the layer-only benchmark
    "120b_skewed_prefill": (615571200 + 381615104 + 496563968 + 374050048,
                            "expert_mlp_bf16.cu", "0649cf90e608fef6"),
    # the one launch of both GEMMs
    "120b_decode": (1609584640 + 8515584, "expert_mlp.cu", "aa5f9d9df0a4dab7"),
    "20b_decode": (429360128 + 5184000, "expert_mlp.cu", "aa5f9d9df0a4dab7"),
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=None, choices=sorted(syn.WORKLOADS),
                    help="time this workload alone (default: the headline and all others)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layer-only", action="store_true",
                    help="with --workload: only the warm-up and timed layer steps (for profilers)")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def expert_bytes(wl) -> int:
    D, F = wl.d_model, wl.d_ff
    return 2 * F * D // 2 + 2 * F * D // 32 + D * F // 2 + D * F // 32


def code_tokens(src: str) -> str:
    """C/CUDA source with its comments removed and whitespace runs collapsed,
    so an edit of comments or layout leaves the hash below unchanged."""
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


HOST_CODE_MARK = "// ------------------------------------------------------------ host helpers"


def device_code(src: str) -> str:
    """The part of a kernel source file before its host helpers: the kernels
    and their device functions, which alone decide the DRAM traffic."""
    cut = src.find(HOST_CODE_MARK)
    return src if cut < 0 else src[:cut]


def kernel_src_sha(name: str) -> str:
    with open(os.path.join(ROOT, "mxfp4_quantised_mixture_b200", "csrc", name)) as f:
        return hashlib.sha256(code_tokens(device_code(f.read())).encode()).hexdigest()[:16]


def gemm_path(wl) -> str:
    """The GEMM path moe_layer_forward takes for the workload (the library's
    rule: block-scaled when twice the mean routed rows per expert is at most
    64)."""
    S = wl.T * wl.k
    return "block-scaled" if 2 * -(-S // wl.E) <= 64 else "bf16-decode"


def captured_traffic(workload: str):
    rec = TRAFFIC.get(workload)
    if rec is None or rec[0] == 0 or kernel_src_sha(rec[1]) != rec[2]:
        return None
    return rec[0]


# ------------------------------------------------------------------ clocks


class ClockSampler:
    """SM clock and clock-event reasons polled through NVML (every ~2 ms)
    while the timed region runs; nvidia-smi's 100 ms interval is longer than
    a short timed region."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, index: int):
        self.index = index
        self.samples: list[tuple[float, int]] = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self._nvml = None

    def start(self):
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nvml = pynvml
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = self.index
            if vis:
                ids = [v.strip() for v in vis.split(",")]
                if ids[idx].isdigit():
                    idx = int(ids[idx])
            self._h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM))
        except Exception:
            self._nvml = None
            return
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                get = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    nv.nvmlDeviceGetCurrentClocksThrottleReasons
                rs = get(self._h)
                self.samples.append((float(mhz), int(rs)))
            except Exception:
                pass
            time.sleep(0.002)

    def stop(self) -> dict:
        if self._nvml is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"], "samples": 0}
        self._stop.set()
        if self._t:
            self._t.join(timeout=2)
        mhz = [m for m, _ in self.samples]
        bits = 0
        for _, r in self.samples:
            bits |= r
        reasons = sorted(n for n, b in self.REASONS.items() if bits & b)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(mhz)}


# --------------------------------------------------- oracle (CPU baseline)


def oracle_weights(wl, tokens):
    """Oracle-quantised weights [E][...] of the experts the tokens route to
    (the others zero), made before any timing."""
    import oracle

    lg = syn.logits(wl)
    idx, _ = oracle.route(lg[tokens], wl.k)
    need = sorted(set(int(v) for v in idx.ravel()))
    D, F, E = wl.d_model, wl.d_ff, wl.E
    gq = np.zeros((E, 2 * F, D // 2), np.uint8)
    gs = np.zeros((E, 2 * F, D // 32), np.uint8)
    dq = np.zeros((E, D, F // 2), np.uint8)
    ds = np.zeros((E, D, F // 32), np.uint8)
    for e in need:
        q, s = oracle.quantize_experts(syn.w_gate_up(wl, [e]))
        gq[e], gs[e] = q[0], s[0]
        q, s = oracle.quantize_experts(syn.w_down(wl, [e]))
        dq[e], ds[e] = q[0], s[0]
    return gq, gs, dq, ds


def cpu_oracle_sample(wl, n_tokens: int, weights=None, inputs=None):
    """Time the fp64 oracle over the first n_tokens of the workload (the
    whole layer when that is all of them).  Returns (seconds, tokens,
    threads, weights, inputs)."""
    import oracle

    if inputs is None:
        inputs = (syn.activations(wl), syn.logits(wl))
    x, lg = inputs
    tokens = list(range(min(n_tokens, wl.T)))
    if weights is None:
        weights = oracle_weights(wl, tokens)
    t0 = time.perf_counter()
    if len(tokens) == wl.T:
        oracle.layer_forward(x, lg, wl.k, *weights)
    else:
        oracle.layer_tokens(x, lg, wl.k, *weights, tokens)
    dt = time.perf_counter() - t0
    return dt, len(tokens), max(1, min(64, os.cpu_count() or 1)), weights, inputs


def sample_label(wl, n: int) -> str:
    what = f"all {n} tokens of the batch" if n == wl.T else f"first {n} of {wl.T} tokens"
    return (what + "; the oracle's weights of the experts they route to quantised before timing, "
            "their decode to fp64 inside each timed call")


def cpu_baseline(wl) -> dict:
    n = min(wl.T, CPU_SAMPLE_TOKENS)
    dt, tok, threads, weights, inputs = cpu_oracle_sample(wl, n)
    times = [dt]
    while sum(times) < 10.0 and len(times) < 5:  # about 10 s of CPU work
        times.append(cpu_oracle_sample(wl, n, weights, inputs)[0])
    return {"value": tok / statistics.mean(times), "unit": UNIT, "cores": threads,
            "kind": "oracle", "sample": sample_label(wl, tok) + f"; mean of {len(times)} calls"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = syn.WORKLOADS[args.workload or HEADLINE]
    n = min(wl.T, CPU_SAMPLE_TOKENS)
    weights = inputs = None
    for _ in range(args.warmup):
        _, _, _, weights, inputs = cpu_oracle_sample(wl, n, weights, inputs)
    total = 0.0
    threads = 1
    for _ in range(args.steps):
        dt, tok, threads, weights, inputs = cpu_oracle_sample(wl, n, weights, inputs)
        total += dt
    value = args.steps * n / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(wl),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample_label(wl, n) + ", per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_dict(wl):
    return {"workload": wl.name, "T": wl.T, "d_model": wl.d_model, "d_ff": wl.d_ff, "E": wl.E,
            "k": wl.k, "seed": wl.seed, "weights": "MXFP4 (E2M1 + E8M0 per 32), bf16 activations",
            "l2": "flushed before every timed step (256 MiB device write, outside the events)",
            "parallelism": "replica per GPU"}


# ---------------------------------------------------------- rank helpers


def reduce_max(value: float, device=None) -> float:
    """Max of `value` over all ranks of the default process group (the value
    itself when there is none)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, tokens_per_rank: int, steps: int, max_total_ms: float) -> float:
    """Whole-job tokens/s: every rank ran `steps` steps of its own batch; the
    job took as long as the slowest rank."""
    return world * tokens_per_rank * steps / (max_total_ms / 1e3)


# -------------------------------------------------------------------- ours


def quantiser_timings(moe, w, flush, stream, steps, hbm):
    """Mean CUDA-event time of mxfp4_quantize and of mxfp4_quantize_sr_rht
    (both flags) over ``w`` [..., K] bf16, L2 flushed before each call.  The
    algorithmic bytes are 2 read + 17/32 written per element."""
    import torch

    K = w.shape[-1]
    rows = w.numel() // K
    q = torch.empty((rows, K // 2), dtype=torch.uint8, device=w.device)
    sc = torch.empty((rows, K // 32), dtype=torch.uint8, device=w.device)
    signs = torch.from_numpy(np.random.default_rng(7).integers(0, 1 << 32, size=K // 32, dtype=np.uint64)
                             .astype(np.uint32).view(np.int32)).to(w.device)
    elems = rows * K
    nbytes = elems * 2 + elems // 2 + elems // 32
    flags = moe.MOE_QUANT_RHT | moe.MOE_QUANT_SR
    calls = {
        "mxfp4_quantize": lambda i: moe.mxfp4_quantize(w, q, sc, None, stream),
        "mxfp4_quantize_sr_rht": lambda i: moe.mxfp4_quantize_sr_rht(w, flags, signs, 1000 + i, q,
                                                                     sc, None, stream),
    }
    out = {"rows": rows, "K": K, "algorithmic_bytes": nbytes}
    for name, call in calls.items():
        st = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        en = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        for i in range(steps + 2):
            flush.fill_(i & 0xFF)
            if i >= 2:
                st[i - 2].record(stream)
            call(i)
            if i >= 2:
                en[i - 2].record(stream)
        torch.cuda.synchronize()
        ms = statistics.mean(a.elapsed_time(b) for a, b in zip(st, en))
        gbs = nbytes / (ms / 1e3) / 1e9
        out[name] = {"ms": ms, "GB/s": gbs, "frac_of_hbm": gbs / hbm,
                     "Gelem/s": elems / (ms / 1e3) / 1e9}
    out["mxfp4_quantize_sr_rht"]["flags"] = "MOE_QUANT_RHT|MOE_QUANT_SR"
    return out


class Ctx:
    """Device, stream, flush buffer and rank layout shared by the workloads."""

    def __init__(self, args):
        import torch
        import torch.distributed as dist

        self.args = args
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        if self.world > 1:
            import datetime

            torch.cuda.set_device(self.local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", self.local))
        self.dev = torch.device("cuda", self.local)
        torch.cuda.set_device(self.dev)
        self.stream = torch.cuda.current_stream(self.dev)
        self.flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=self.dev)
        self.peaks = peaks()

    def barrier(self):
        import torch.distributed as dist

        if self.world > 1:
            dist.barrier()


def quantised_weights(moe, ctx, wl, keep_first_chunk=False, keep_bf16=False):
    """The workload's MXFP4 weights on the device, quantised by the library
    from the seeded bf16 weights (generated on the host a chunk of experts at
    a time); with keep_bf16 also the bf16 weights themselves."""
    import torch

    dev = ctx.dev
    D, F, E = wl.d_model, wl.d_ff, wl.E
    wgu_q = torch.empty((E, 2 * F, D // 2), dtype=torch.uint8, device=dev)
    wgu_s = torch.empty((E, 2 * F, D // 32), dtype=torch.uint8, device=dev)
    wdn_q = torch.empty((E, D, F // 2), dtype=torch.uint8, device=dev)
    wdn_s = torch.empty((E, D, F // 32), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    chunk = max(1, min(E, (1 << 28) // (2 * F * D)))
    first = None
    if keep_bf16:
        bf_gu = torch.empty((E, 2 * F, D), dtype=torch.bfloat16, device=dev)
        bf_dn = torch.empty((E, D, F), dtype=torch.bfloat16, device=dev)
    for e0 in range(0, E, chunk):
        ex = list(range(e0, min(E, e0 + chunk)))
        gu = torch.from_numpy(syn.w_gate_up(wl, ex).view(np.int16)).to(dev).view(torch.bfloat16)
        dn = torch.from_numpy(syn.w_down(wl, ex).view(np.int16)).to(dev).view(torch.bfloat16)
        moe.mxfp4_quantize(gu, wgu_q[e0:e0 + len(ex)], wgu_s[e0:e0 + len(ex)], status)
        moe.mxfp4_quantize(dn, wdn_q[e0:e0 + len(ex)], wdn_s[e0:e0 + len(ex)], status)
        if e0 == 0 and keep_first_chunk:
            first = gu
        if keep_bf16:
            bf_gu[e0:e0 + len(ex)].copy_(gu)
            bf_dn[e0:e0 + len(ex)].copy_(dn)
        del gu, dn
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError("quantiser reported non-finite weights")
    return (wgu_q, wgu_s, wdn_q, wdn_s), {"first": first,
                                          "bf16": (bf_gu, bf_dn) if keep_bf16 else None}


def captured(torch, fn):
    """A CUDA graph of fn(stream): one call on a side stream first (so any
    one-time set-up of the call happens outside the capture), then the
    capture.  Replaying it launches the same kernels with the same arguments
    on the current stream."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn(side)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn(torch.cuda.current_stream())
    torch.cuda.synchronize()
    return g


def replay_ms(torch, g, flush, stream, steps: int) -> list:
    """Per-replay device ms of graph g, L2 flushed (outside the events) before
    each replay, two untimed replays first."""
    st = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    en = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for i in range(steps + 2):
        flush.fill_(i & 0xFF)
        if i >= 2:
            st[i - 2].record(stream)
        g.replay()
        if i >= 2:
            en[i - 2].record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in zip(st, en)]


def measure_workload(moe, ctx, wl, weights, layer_only=False) -> dict:
    """Time one workload: the layer step, the expert MLP's roofline, e2e
    (with layer_only, the layer step alone)."""
    import torch

    args, dev, stream, flush = ctx.args, ctx.dev, ctx.stream, ctx.flush
    D, F, E, T, k = wl.d_model, wl.d_ff, wl.E, wl.T, wl.k
    S = T * k
    shape = moe.make_shape(T, E, k, D, F)
    wgu_q, wgu_s, wdn_q, wdn_s = weights
    x_np = syn.activations(wl)
    lg_np = syn.logits(wl)
    x = torch.from_numpy(x_np.view(np.int16)).to(dev).view(torch.bfloat16)
    logits = torch.from_numpy(lg_np).to(dev)
    out = torch.empty((T, D), dtype=torch.bfloat16, device=dev)
    ws = moe.alloc_workspace(shape, moe.WS_LAYER, dev)

    def layer(s=stream):
        moe.moe_layer_forward(x, logits, shape, wgu_q, wgu_s, wdn_q, wdn_s, out, ws, s)

    def layer_status():
        st = int(ws[:4].view(torch.int32).item())
        if st != 0:
            raise RuntimeError("layer reported device status %d" % st)

    # the step as a serving loop runs it: moe_layer_forward captured once into
    # a CUDA graph (its five or six kernels, no host work per step), replayed per step
    graph = captured(torch, layer)
    for _ in range(args.warmup):
        flush.fill_(1)
        graph.replay()
    torch.cuda.synchronize()
    layer_status()

    # ---- timed region: K steps, events around each step, L2 flushed between
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    clocks = ClockSampler(ctx.local)
    clocks.start()
    time.sleep(0.3)
    ctx.barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        starts[i].record(stream)
        graph.replay()
        ends[i].record(stream)
    torch.cuda.synchronize()
    ctx.barrier()
    wall = time.perf_counter() - wall0
    clk = clocks.stop()
    layer_status()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = reduce_max(float(sum(step_ms)), dev)
    ms_per_step = total_ms / args.steps
    value = job_throughput(ctx.world, T, args.steps, total_ms)

    # the same steps as eager calls (host planning and the launches per step)
    e_starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e_ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        e_starts[i].record(stream)
        layer()
        e_ends[i].record(stream)
    torch.cuda.synchronize()
    layer_status()
    eager_ms = reduce_max(sum(s.elapsed_time(e) for s, e in zip(e_starts, e_ends)), dev) / args.steps
    eager = {"ms_per_step": eager_ms, "value": ctx.world * T / (eager_ms / 1e3)}
    del graph
    if layer_only:
        return {"value": value, "ms_per_step": ms_per_step, "config": config_dict(wl),
                "launch": LAUNCH_NOTE, "eager": eager,
                "clocks": clk, "gpu_launches": LAUNCHES_PER_LAYER[gemm_path(wl)] * args.steps,
                "step_ms_min": min(step_ms), "step_ms_max": max(step_ms)}

    # ---- roofline of the grouped expert MLP: the same step through the
    #      individual calls: route and permute once, then moe_expert_mlp
    #      captured into a CUDA graph and replayed between events
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    tw = torch.empty((T, k), dtype=torch.float32, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    ss = torch.empty(S, dtype=torch.int32, device=dev)
    sp = torch.empty(S, dtype=torch.int32, device=dev)
    xp = torch.empty((S, D), dtype=torch.bfloat16, device=dev)
    h = torch.empty((S, F), dtype=torch.bfloat16, device=dev)
    yp = torch.empty((S, D), dtype=torch.bfloat16, device=dev)
    ws_mlp = moe.alloc_workspace(shape, moe.WS_EXPERT_MLP, dev)
    moe.moe_route(logits, k, idx, tw, stream)
    moe.moe_permute(idx, x, shape, counts, offsets, ss, sp, xp, None, stream)
    g_mlp = captured(torch, lambda s: moe.moe_expert_mlp(xp, offsets, shape, wgu_q, wgu_s, wdn_q,
                                                         wdn_s, h, yp, ws_mlp, s))
    mlp_ms = statistics.mean(replay_ms(torch, g_mlp, flush, stream, args.steps))
    del g_mlp
    if int(ws_mlp[:4].view(torch.int32).item()) != 0:
        raise RuntimeError("expert MLP reported device status %d" % int(ws_mlp[:4].view(torch.int32).item()))
    touched = int((counts > 0).sum().item())
    mlp_bytes = touched * expert_bytes(wl) + 2 * S * D * 2
    hbm, tc_burst, tc_sust, peak_kind = ctx.peaks
    mlp_flops = 6.0 * S * D * F
    # the bound is whichever roofline term is larger for this call: the bytes
    # at the measured copy bandwidth or the FLOPs at the measured bf16 rate
    # (burst figure: the call is timed on its own)
    tensor_bound = mlp_flops / (tc_burst * 1e12) > mlp_bytes / (hbm * 1e9)
    if tensor_bound:
        roof = {"bound": "tensor", "achieved": mlp_flops / (mlp_ms / 1e3) / 1e12, "peak": tc_burst,
                "unit": "TFLOP/s", "algorithmic_flops": mlp_flops}
    else:
        roof = {"bound": "hbm", "achieved": mlp_bytes / (mlp_ms / 1e3) / 1e9, "peak": hbm,
                "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof.update(traffic=captured_traffic(wl.name),
                kernel="moe_expert_mlp (grouped gate/up+SwiGLU and down GEMMs)",
                algorithmic_bytes=mlp_bytes, ms=mlp_ms, peak_source=peak_kind,
                path=gemm_path(wl))
    layer_bytes = touched * expert_bytes(wl) + T * D * 2 + T * E * 4 + T * D * 2
    layer_flops = 6.0 * S * D * F
    t_roof_meas = max(layer_bytes / (hbm * 1e9), layer_flops / (tc_sust * 1e12))
    t_roof_spec = max(layer_bytes / 8e12, layer_flops / 2.25e15)

    # ---- end to end through the C ABI with host buffers
    x_host = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16).pin_memory()
    lg_host = torch.from_numpy(lg_np).pin_memory()
    out_host = torch.empty((T, D), dtype=torch.bfloat16).pin_memory()
    e_starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e_ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        e_starts[i].record(stream)
        x.copy_(x_host, non_blocking=True)
        logits.copy_(lg_host, non_blocking=True)
        layer()
        out_host.copy_(out, non_blocking=True)
        e_ends[i].record(stream)
        e_ends[i].synchronize()
    e2e_ms = reduce_max(sum(s.elapsed_time(e) for s, e in zip(e_starts, e_ends)) / args.steps, dev)
    e2e = {"value": ctx.world * T / (e2e_ms / 1e3), "unit": UNIT,
           "h2d_bytes_per_step": x_host.numel() * 2 + lg_host.numel() * 4,
           "d2h_bytes_per_step": out_host.numel() * 2}

    cpu = None
    if ctx.rank == 0 and ctx.world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl)

    return {
        "value": value, "ms_per_step": ms_per_step, "config": config_dict(wl),
        "launch": LAUNCH_NOTE, "eager": eager, "roofline": roof,
        "layer_roofline": {"bytes": layer_bytes, "flops": layer_flops,
                           "frac_of_measured": t_roof_meas / (ms_per_step / 1e3),
                           "frac_of_spec_8TBs_2.25PF": t_roof_spec / (ms_per_step / 1e3),
                           "touched_experts": touched},
        "cpu_baseline": cpu, "e2e": e2e, "clocks": clk,
        "gpu_launches": LAUNCHES_PER_LAYER[gemm_path(wl)] * args.steps,
        "wall_s_timed_region": wall, "step_ms_min": min(step_ms), "step_ms_max": max(step_ms),
    }


def unquantised_timing(moe, ctx, wl, weights, bf16_weights) -> dict:
    """The grouped expert MLP on the workload's unquantised bf16 weights
    (moe_expert_mlp_unquantised) beside the same call on the MXFP4 weights
    (moe_expert_mlp), on the same permuted rows, L2 flushed before each call:
    weight bytes streamed and time of each."""
    import torch

    dev, stream, flush, steps = ctx.dev, ctx.stream, ctx.flush, ctx.args.steps
    D, F, E, T, k = wl.d_model, wl.d_ff, wl.E, wl.T, wl.k
    S = T * k
    shape = moe.make_shape(T, E, k, D, F)
    x = torch.from_numpy(syn.activations(wl).view(np.int16)).to(dev).view(torch.bfloat16)
    logits = torch.from_numpy(syn.logits(wl)).to(dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    tw = torch.empty((T, k), dtype=torch.float32, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    ss = torch.empty(S, dtype=torch.int32, device=dev)
    sp = torch.empty(S, dtype=torch.int32, device=dev)
    xp = torch.empty((S, D), dtype=torch.bfloat16, device=dev)
    moe.moe_route(logits, k, idx, tw, stream)
    moe.moe_permute(idx, x, shape, counts, offsets, ss, sp, xp, None, stream)
    h = torch.empty((S, F), dtype=torch.bfloat16, device=dev)
    yp = torch.empty((S, D), dtype=torch.bfloat16, device=dev)
    ws_q = moe.alloc_workspace(shape, moe.WS_EXPERT_MLP, dev)
    ws_u = moe.alloc_workspace(shape, moe.WS_EXPERT_MLP_UNQUANTISED, dev)
    bf_gu, bf_dn = bf16_weights
    calls = {
        "mxfp4": lambda s: moe.moe_expert_mlp(xp, offsets, shape, *weights, h, yp, ws_q, s),
        "bf16": lambda s: moe.moe_expert_mlp_unquantised(xp, offsets, shape, bf_gu, bf_dn, h, yp,
                                                         ws_u, s),
    }
    torch.cuda.synchronize()
    touched = int((counts > 0).sum().item())
    out = {"call": "moe_expert_mlp_unquantised vs moe_expert_mlp (CUDA graph replays)",
           "workload": wl.name}
    for name, call in calls.items():
        g = captured(torch, call)
        ms = statistics.mean(replay_ms(torch, g, flush, stream, steps))
        del g
        wbytes = touched * (expert_bytes(wl) if name == "mxfp4" else 3 * D * F * 2)
        out[name] = {"ms": ms, "weight_bytes": wbytes,
                     "GB/s": (wbytes + 2 * S * D * 2) / (ms / 1e3) / 1e9}
    ws_st = (int(ws_q[:4].view(torch.int32).item()), int(ws_u[:4].view(torch.int32).item()))
    if ws_st != (0, 0):
        raise RuntimeError(f"expert MLP reported device status {ws_st}")
    out["bf16_over_mxfp4_bytes"] = out["bf16"]["weight_bytes"] / out["mxfp4"]["weight_bytes"]
    out["bf16_over_mxfp4_time"] = out["bf16"]["ms"] / out["mxfp4"]["ms"]
    return out


def router_timing(moe, ctx, wl):
    """moe_router_topk on the workload's tokens against a seeded bf16 router
    matrix [E][D], L2 flushed before each call."""
    import torch

    dev, stream, flush, steps = ctx.dev, ctx.stream, ctx.flush, ctx.args.steps
    T, D, E, k = wl.T, wl.d_model, wl.E, wl.k
    x = torch.from_numpy(syn.activations(wl).view(np.int16)).to(dev).view(torch.bfloat16)
    w_router = torch.from_numpy(syn.normal_bf16(wl.seed, 40, (E, D), sigma=1.0 / D ** 0.5)
                                .view(np.int16)).to(dev).view(torch.bfloat16)
    r_idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    r_w = torch.empty((T, k), dtype=torch.float32, device=dev)
    g = captured(torch, lambda s: moe.moe_router_topk(x, w_router, k, r_idx, r_w, None, None, s))
    ms = statistics.mean(replay_ms(torch, g, flush, stream, steps))
    del g
    nbytes = T * D * 2 + E * D * 2 + T * k * 8
    return {"call": "moe_router_topk (CUDA graph replays)", "workload": wl.name, "ms": ms,
            "bytes": nbytes,
            "GB/s": nbytes / (ms / 1e3) / 1e9, "TFLOP/s": 2.0 * T * D * E / (ms / 1e3) / 1e12}


def run_ours(args):
    import torch
    import torch.distributed as dist

    import mxfp4_quantised_mixture_b200 as moe

    ctx = Ctx(args)
    if args.layer_only:
        if not args.workload:
            raise SystemExit("--layer-only needs --workload")
        wl = syn.WORKLOADS[args.workload]
        weights, _ = quantised_weights(moe, ctx, wl)
        r = measure_workload(moe, ctx, wl, weights, layer_only=True)
        if ctx.world > 1:
            dist.barrier()
            dist.destroy_process_group()
        if ctx.rank == 0:
            print(json.dumps(dict(r, metric=METRIC, unit=UNIT, n_gpus=ctx.world, steps=args.steps,
                                  warmup=args.warmup, layer_only=True)), flush=True)
        return 0
    names = [args.workload] if args.workload else [HEADLINE] + OTHERS
    results = {}
    extras = {}
    cache = {}  # weights shared by workloads of the same layer (20B decode and prefill)
    for name in names:
        wl = syn.WORKLOADS[name]
        key = (wl.E, wl.d_model, wl.d_ff, wl.seed, wl.outlier_p, wl.w_sigma)
        if key not in cache:
            cache.clear()
            torch.cuda.empty_cache()
            cache[key] = quantised_weights(moe, ctx, wl, keep_first_chunk=(name == names[0]),
                                           keep_bf16=(name == UNQUANTISED_AT))
        weights, keep = cache[key]
        results[name] = measure_workload(moe, ctx, wl, weights)
        if name == UNQUANTISED_AT:
            extras["unquantised"] = unquantised_timing(moe, ctx, wl, weights, keep["bf16"])
            keep["bf16"] = None
        if name == "20b_decode" and name != names[0]:
            extras["router_decode"] = router_timing(moe, ctx, wl)
        if name == names[0]:
            extras["router"] = router_timing(moe, ctx, wl)
            extras["quantize"] = quantiser_timings(moe, keep["first"], ctx.flush, ctx.stream,
                                                   args.steps, ctx.peaks[0])
            keep["first"] = None
        torch.cuda.empty_cache()
    if ctx.world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if ctx.rank != 0:
        return 0
    head = results[names[0]]
    line = {
        "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": ctx.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": head["config"],
        "roofline": head["roofline"], "layer_roofline": head["layer_roofline"],
        "cpu_baseline": head["cpu_baseline"], "e2e": head["e2e"], "clocks": head["clocks"],
        "gpu_launches": head["gpu_launches"],
        "wall_s_timed_region": head["wall_s_timed_region"],
        "step_ms_min": head["step_ms_min"], "step_ms_max": head["step_ms_max"],
        "launch": head["launch"], "eager": head["eager"],
        "router": extras.get("router"), "router_decode": extras.get("router_decode"),
        "quantize": extras.get("quantize"),
        "unquantised": extras.get("unquantised"),
        "per_workload": {n: r for n, r in results.items() if n != names[0]},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
