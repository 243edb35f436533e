"""Benchmark of the NVFP4 W4A4 linear (run-time activation quantization + block-
scaled FP4 GEMM) on the MLP up-projection of a diffusion transformer:
M = 4096 tokens (64 x 64 latent patches of a 1024 x 1024 image), K = 3072,
N = 12288, bf16 in / bf16 out, synthetic seeded inputs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one nvfp4_linear_laid_out call (the activations' quantization kernel +
the GEMM kernel) on weight scales laid out once at set-up, like the weights' own
quantization; the same step through nvfp4_linear, which lays the weight scales out
in every call, is reported as per_call_weight_layout. Consecutive
steps cycle through buffer sets (x, weights, y, workspace) that together hold at
least four times the L2, so every step reads its operands from HBM; the K timed
steps, each bracketed by CUDA event records, are captured in one CUDA graph and
replayed once, and the value comes from the median step. Several GPUs run independent replicas (weak scaling; the layer has
no exchange step); the time is the max over ranks.

Prints one JSON line (rank 0). Extra keys: step_stats (median / mean / min / max), the same step with a 256 MB flush before
every step (l2_flushed), with warm L2 (l2_warm) and as CUDA graphs over the
rotating sets (l2_rotating_graph); roofline of the GEMM kernel (with the SM clock
the GEMM ran at and the dense FP4 peak at that clock); cpu_baseline (the CPU oracle
on a bounded sample, its CPU model, and one-thread figures); e2e (host buffers,
copies inside the timed region: every step copies its X in and its Y out, the copies
of consecutive steps overlapping the layer on three streams; the back-to-back time
beside it); clocks sampled during the run; and under
"variants" the other layer shapes, the skinny / batched NVFP4 sweep and the W4A16
modulation sweep (rotating-graph timed, against the HBM and FP4 rooflines).
"""
import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "NVFP4 W4A4 linear TFLOPS (quant+GEMM) M4096 K3072 N12288; % dense FP4 peak"
UNIT = "TFLOP/s"
WORKLOAD = dict(M=4096, K=3072, N=12288)
NOMINAL_FP4_OVER_BF16 = 4.0      # dense FP4 : dense bf16 tensor rate (9 : 2.25 PFLOP/s)
NOMINAL_FP8_OVER_BF16 = 2.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- distributed

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max(value: float, device=None) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def aggregate(local_ms: float, units_per_rank: float, world: int, device=None):
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    ms = reduce_max(local_ms, device)
    return ms, units_per_rank * world / (ms / 1e3)


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = [
        ("gpu_idle", 0x1), ("applications_clocks_setting", 0x2), ("sw_power_cap", 0x4),
        ("hw_slowdown", 0x8), ("sync_boost", 0x10), ("sw_thermal_slowdown", 0x20),
        ("hw_thermal_slowdown", 0x40), ("hw_power_brake_slowdown", 0x80),
        ("display_clock_setting", 0x100),
    ]

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.idx = device_index
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self.ok = False

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self._physical_index())
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
            return self
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()
        return self

    def _physical_index(self):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        if vis:
            parts = [p for p in vis.split(",") if p.strip()]
            if self.idx < len(parts) and parts[self.idx].strip().isdigit():
                return int(parts[self.idx])
        return self.idx

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        names = [n for n, bit in self.REASONS if self.reasons & bit]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ----------------------------------------------------------------------------- workloads

def nvfp4_flops(M, K, N):
    return 2.0 * M * K * N


def nvfp4_alg_bytes(M, K, N, bias=False):
    """Algorithmic bytes of one fused NVFP4 linear: read X (bf16), W codes and
    scales, bias; write Y (bf16)."""
    return 2 * M * K + N * K // 2 + N * K // 16 + 2 * M * N + (4 * N if bias else 0)


class Nvfp4Layer:
    """Device-resident NVFP4 layer: W quantized on the GPU (same kernel as the
    activations), input_scale calibrated on the GPU (amax / 2688)."""

    def __init__(self, M, K, N, bias, device, seed=0):
        import torch
        import fp8_rowwise_quantized_b200 as q
        from synthetic import make_linear_inputs
        inp = make_linear_inputs(M, K, N, seed=seed, with_bias=bias)
        self.M, self.K, self.N = M, K, N
        self.x_host = inp.x
        self.x = inp.x.to(device)
        w = inp.w.to(device)
        self.wq, self.ws, self.gw = q.prepare_nvfp4_weight(w)
        del w
        self.gx = q.nvfp4_global_scale(self.x)
        self.bias = None if inp.bias is None else inp.bias.to(device)
        self.y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
        self.work = torch.empty(q.nvfp4_linear_workspace_size(M, K, N), dtype=torch.uint8,
                                device=device)
        self.q = q
        # the weight scales laid out once for the tile width a call of this size uses
        # (a load-time step, like the weight's quantization above); skinny tile widths
        # lay them out inside the GEMM and have no atoms
        self.bn = q.tile_config(M, N, K)[0]
        self.atoms = (q.nvfp4_layout_weight_scales(self.ws, self.bn)
                      if self.bn in (128, 192, 224, 256) else None)

    def step(self):
        self.q.nvfp4_linear(self.x, self.wq, self.ws, self.gw, self.gx, bias=self.bias, y=self.y,
                            workspace=self.work)

    def step_laid_out(self):
        self.q.nvfp4_linear_laid_out(self.x, self.wq, self.atoms, self.bn, self.gw, self.gx,
                                     bias=self.bias, y=self.y, workspace=self.work)

    def prologue(self):
        self.q.nvfp4_linear_prologue(self.x, self.ws, self.gx, self.work)

    def gemm(self):
        self.q.nvfp4_linear_gemm(self.M, self.wq, self.gw, self.gx, self.work, bias=self.bias,
                                 y=self.y)


class Fp8rLayer:
    def __init__(self, M, K, N, bias, device, seed=0):
        import torch
        import fp8_rowwise_quantized_b200 as q
        from synthetic import make_linear_inputs
        inp = make_linear_inputs(M, K, N, seed=seed, with_bias=bias)
        self.M, self.K, self.N = M, K, N
        self.x = inp.x.to(device)
        self.wq, self.wsc = q.prepare_fp8r_weight(inp.w.to(device))
        self.bias = None if inp.bias is None else inp.bias.to(device)
        self.y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
        self.work = torch.empty(q.fp8r_linear_workspace_size(M, K, N), dtype=torch.uint8,
                                device=device)
        self.xq, self.xs = q.fp8r_quantize_rows(self.x)
        self.q = q

    def step(self):
        self.q.fp8r_linear(self.x, self.wq, self.wsc, bias=self.bias, y=self.y,
                           workspace=self.work)

    def gemm(self):
        self.q.fp8r_linear_gemm(self.xq, self.xs, self.wq, self.wsc, bias=self.bias, y=self.y)


class Int4Layer:
    """INT4 W4A4 layer (weights quantized on the GPU by int4_quantize_rows)."""

    def __init__(self, M, K, N, bias, device, seed=0):
        import torch
        import fp8_rowwise_quantized_b200 as q
        from synthetic import make_linear_inputs
        inp = make_linear_inputs(M, K, N, seed=seed, with_bias=bias)
        self.q, self.M, self.K, self.N = q, M, K, N
        self.x = inp.x.to(device)
        self.wq, self.ws = q.prepare_int4_weight(inp.w.to(device))
        self.bias = None if inp.bias is None else inp.bias.to(device)
        self.y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
        self.work = torch.empty(q.int4_linear_workspace_size(M, K, N), dtype=torch.uint8,
                                device=device)
        self.xq, self.xs = q.int4_quantize_rows(self.x)
        self.gwork = torch.empty(q.int4_linear_gemm_workspace_size(M, K, N), dtype=torch.uint8,
                                 device=device)

    def step(self):
        self.q.int4_linear(self.x, self.wq, self.ws, bias=self.bias, y=self.y, workspace=self.work)

    def gemm(self):
        self.q.int4_linear_gemm(self.xq, self.xs, self.wq, self.ws, bias=self.bias, y=self.y,
                                workspace=self.gwork)


class SvdqLayer:
    """svdq_w4a4 NVFP4 layer (smoothing, rank-r bf16 branch, 4-bit residual) with
    synthetic operands of the Nvfp4Layer's shapes."""

    def __init__(self, M, K, N, rank, device, seed=0):
        import torch
        import fp8_rowwise_quantized_b200 as q
        base = Nvfp4Layer(M, K, N, False, device, seed=seed)
        g = torch.Generator().manual_seed(seed + 7)
        self.q, self.base = q, base
        self.down = (torch.randn(rank, K, generator=g) * 0.02).to(torch.bfloat16).to(device)
        self.up = (torch.randn(N, rank, generator=g) * 0.05).to(torch.bfloat16).to(device)
        amax = base.x.float().abs().amax(dim=0).clamp(min=1e-3)
        self.smooth = (1.0 / amax.sqrt()).float().contiguous()
        xs = (base.x.float() * self.smooth).to(torch.bfloat16)
        self.gx = q.nvfp4_global_scale(xs)
        self.work = torch.empty(q.svdq_nvfp4_linear_workspace_size(M, K, N, rank),
                                dtype=torch.uint8, device=device)

    def step(self):
        b = self.base
        self.q.svdq_nvfp4_linear(b.x, b.wq, b.ws, b.gw, self.gx, self.down, self.up,
                                 smooth=self.smooth, y=b.y, workspace=self.work)


class MlpBlock:
    """Diffusion-transformer MLP block on the device: up projection (K -> H), exact
    GELU, down projection (H -> K), both NVFP4. The down projection's input_scale
    is calibrated once, from an unfused run (amax of GELU(up) / 2688), and then
    held fixed, as a deployed model would."""

    def __init__(self, M, K, H, device, seed=0):
        import torch
        import fp8_rowwise_quantized_b200 as q
        self.up = Nvfp4Layer(M, K, H, False, device, seed=seed)
        self.down = Nvfp4Layer(M, H, K, False, device, seed=seed + 1)
        self.q, self.M = q, M
        y = q.nvfp4_linear(self.up.x, self.up.wq, self.up.ws, self.up.gw, self.up.gx)
        self.h = torch.nn.functional.gelu(y.float()).to(torch.bfloat16)
        self.g_down = q.nvfp4_global_scale(self.h)
        self.y = torch.empty((M, K), dtype=torch.bfloat16, device=device)

    def fused(self):
        q = self.q
        q.nvfp4_linear_gelu_quantize(self.up.x, self.up.wq, self.up.ws, self.up.gw, self.up.gx,
                                     self.g_down, self.down.work, workspace=self.up.work)
        q.nvfp4_linear_quantized_input(self.M, self.down.wq, self.down.ws, self.down.gw,
                                       self.g_down, self.down.work, y=self.y)

    def unfused(self):
        import torch
        q = self.q
        q.nvfp4_linear(self.up.x, self.up.wq, self.up.ws, self.up.gw, self.up.gx, y=self.up.y,
                       workspace=self.up.work)
        h = torch.nn.functional.gelu(self.up.y.float()).to(torch.bfloat16)
        q.nvfp4_linear(h, self.down.wq, self.down.ws, self.down.gw, self.g_down, y=self.y,
                       workspace=self.down.work)


def time_events(fn, steps, warmup, flush, stream):
    """Device time (ms) of fn over `steps` calls, each bracketed by CUDA events on
    `stream`, with `flush()` (if given) before every call, outside the events.
    Returns (median, per-call times)."""
    import torch
    for _ in range(warmup):
        if flush:
            flush()
        fn()
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for i in range(steps):
        if flush:
            flush()
        starts[i].record(stream)
        fn()
        ends[i].record(stream)
    torch.cuda.synchronize()
    times = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    return statistics.median(times), times


def time_e2e_pipelined(q, layer, x_pin, steps, warmup, flush, stream):
    """Device time per step (ms) of the layer end to end through the public API, with
    the transfers of consecutive steps overlapped as a serving loop would: step i
    copies X in on one stream, runs the layer on `stream` (after a flush), and copies
    Y out on a third, so the copy-in of step i + 1 and the copy-out of step i - 1 run
    beside step i's layer. X and Y on the device, and the pinned host Y, are
    double-buffered; events order reuse. Total time from an event before the first
    copy to one after the last copy, over `steps`."""
    import torch
    M, K, N = layer.M, layer.K, layer.N
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    xd = [torch.empty((M, K), dtype=torch.bfloat16, device=layer.x.device) for _ in range(2)]
    yd = [torch.empty((M, N), dtype=torch.bfloat16, device=layer.x.device) for _ in range(2)]
    yp = [torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_c = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def run(n):
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_c[b])  # the layer of step i - 2 has read xd[b]
                xd[b].copy_(x_pin, non_blocking=True)
                ev_in[b].record(s_in)
            with torch.cuda.stream(stream):
                stream.wait_event(ev_in[b])
                if i >= 2:
                    stream.wait_event(ev_out[b])  # step i - 2's Y has left yd[b]
                if flush:
                    flush()
                q.nvfp4_linear_laid_out(xd[b], layer.wq, layer.atoms, layer.bn, layer.gw,
                                        layer.gx, y=yd[b], workspace=layer.work)
                ev_c[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_c[b])
                yp[b].copy_(yd[b], non_blocking=True)
                ev_out[b].record(s_out)
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)

    run(warmup)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    s_in.wait_stream(stream)
    s_out.wait_stream(stream)
    run(steps)
    end.record(stream)
    torch.cuda.synchronize()
    # the last step's Y really arrived: compare with the device copy
    assert torch.equal(yp[(steps - 1) % 2], yd[(steps - 1) % 2].cpu())
    return start.elapsed_time(end) / steps


L2_BYTES = 126 << 20
ROTATION_BYTES = 4 * L2_BYTES


class Nvfp4Rotation:
    """R copies of one NVFP4 layer's device buffers (x, weight codes and scales,
    bias, y, workspace), R chosen so that all copies together hold at least four
    times the L2. Stepping through them in turn makes every call find its
    operands in HBM, not in L2, as in a stack of distinct layers; nothing is
    written between calls, so no flush write-back lands in the timed region."""

    def __init__(self, layer, min_bytes=ROTATION_BYTES):
        import torch
        self.L = layer
        per = sum(t.numel() * t.element_size() for t in
                  (layer.x, layer.wq, layer.ws, layer.y, layer.work, layer.atoms) if t is not None)
        if layer.bias is not None:
            per += layer.bias.numel() * 4
        self.R = max(2, -(-min_bytes // per))
        self.bytes_per_set = per

        def clone(t):
            return None if t is None else t.clone()
        self.sets = [(layer.x, layer.wq, layer.ws, layer.bias, layer.y, layer.work)]
        self.atoms = [layer.atoms]
        for _ in range(self.R - 1):
            self.sets.append((clone(layer.x), clone(layer.wq), clone(layer.ws), clone(layer.bias),
                              torch.empty_like(layer.y), torch.empty_like(layer.work)))
            self.atoms.append(clone(layer.atoms))
        self.i = 0

    def _next(self):
        s = self.sets[self.i]
        self.i = (self.i + 1) % self.R
        return s

    def step(self):
        x, wq, ws, b, y, work = self._next()
        self.L.q.nvfp4_linear(x, wq, ws, self.L.gw, self.L.gx, bias=b, y=y, workspace=work)

    def step_laid_out(self):
        atoms = self.atoms[self.i]
        x, wq, ws, b, y, work = self._next()
        self.L.q.nvfp4_linear_laid_out(x, wq, atoms, self.L.bn, self.L.gw, self.L.gx, bias=b, y=y,
                                       workspace=work)

    def prologue_all(self):
        for x, wq, ws, b, y, work in self.sets:
            self.L.q.nvfp4_linear_prologue(x, ws, self.L.gx, work)

    def gemm(self):
        x, wq, ws, b, y, work = self._next()
        self.L.q.nvfp4_linear_gemm(self.L.M, wq, self.L.gw, self.L.gx, work, bias=b, y=y)

    def prologue(self):
        x, wq, ws, b, y, work = self._next()
        self.L.q.nvfp4_linear_prologue(x, ws, self.L.gx, work)

    def quantize_act(self):
        # codes and scales into the set's workspace (row-major, as the call returns them)
        x, wq, ws, b, y, work = self._next()
        M, K = self.L.M, self.L.K
        xq = work[:M * K // 2].view(M, K // 2)
        xs = work[M * K // 2:M * K // 2 + M * K // 16].view(M, K // 16)
        self.L.q.nvfp4_quantize_act(x, self.L.gx, xq, xs)


def time_graph_rotation(fn, calls, reps, stream):
    """Mean device time (ms) of one call of fn, where fn cycles through buffer sets
    larger than L2: `calls` consecutive calls (one per set) are captured in a CUDA
    graph, the graph is replayed `reps` times with CUDA events around each replay,
    and the mean replay time is divided by `calls`. No host launch gap and no
    flush lands inside the timed region."""
    import torch
    for _ in range(calls):  # warm-up: every set once
        fn()
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            for _ in range(calls):
                fn()
    torch.cuda.current_stream().wait_stream(side)
    graph.replay()
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
    for i in range(reps):
        starts[i].record(stream)
        graph.replay()
        ends[i].record(stream)
    torch.cuda.synchronize()
    ms = statistics.fmean(a.elapsed_time(b) for a, b in zip(starts, ends)) / calls
    del graph
    return ms


class W4a16Rotation:
    """W4A16 modulation layer (NVFP4 weight quantized on the GPU, bf16 activations)
    in R copies whose weights together hold at least four times the L2."""

    def __init__(self, M, K, N, device, seed=0, min_bytes=ROTATION_BYTES):
        import torch
        import fp8_rowwise_quantized_b200 as q
        from synthetic import make_linear_inputs
        inp = make_linear_inputs(M, K, N, seed=seed, with_bias=True)
        self.q, self.M, self.K, self.N = q, M, K, N
        x = inp.x.to(device)
        wq, ws, self.gw = q.prepare_nvfp4_weight(inp.w.to(device))
        bias = inp.bias.to(device)
        per = wq.numel() + ws.numel() + x.numel() * 2 + M * N * 2 + N * 4
        self.R = max(2, -(-min_bytes // per))
        self.sets = [(x.clone(), wq.clone(), ws.clone(), bias.clone(),
                      torch.empty((M, N), dtype=torch.bfloat16, device=device))
                     for _ in range(self.R)]
        self.i = 0

    def step(self):
        x, wq, ws, b, y = self.sets[self.i]
        self.i = (self.i + 1) % self.R
        self.q.w4a16_linear(x, wq, ws, self.gw, bias=b, y=y)


def w4a16_bytes(M, K, N):
    """Algorithmic bytes of one W4A16 call: weight codes and scales, x, bias, y."""
    return N * K // 2 + N * K // 16 + 2 * M * K + 4 * N + 2 * M * N


def w4a16_sweep(device, stream, peaks, steps):
    """Modulation projections of a diffusion transformer (hidden 3072): the
    six-way adaptive-norm modulation (N = 6 x 3072) and the three-way one of the
    single-stream blocks (N = 3 x 3072), for batches of 1, 2 and 4 conditioning
    vectors; graph-replayed over rotating weight copies (cold L2 every call)."""
    import torch
    hbm = peaks["hbm_gbs"]
    out = {}
    for N in (18432, 9216):
        for M in (1, 2, 4):
            K = 3072
            L = W4a16Rotation(M, K, N, device)
            reps = max(3, min(steps // L.R, 20))
            ms = time_graph_rotation(L.step, L.R, reps, stream)
            b = w4a16_bytes(M, K, N)
            out[f"M{M}_K{K}_N{N}"] = {"us": ms * 1e3, "gbs": b / (ms / 1e3) / 1e9,
                                      "hbm_frac": b / (ms / 1e3) / 1e9 / hbm,
                                      "alg_bytes": b, "rotation_sets": L.R}
            del L
            torch.cuda.empty_cache()
    return out


# Skinny / batched sweep of the NVFP4 layer (K = 3072): M from a few text tokens
# to four 4096-token latents, N of the attention projection and the MLP up projection.
SKINNY_M = (16, 256, 1024, 8192, 16384)
SKINNY_N = (3072, 12288)


def nvfp4_gemm_alg_bytes(M, K, N):
    """Algorithmic bytes of the GEMM kernel alone: activation codes and scales,
    weight codes and scales in, bf16 Y out."""
    return M * K // 2 + M * K // 16 + N * K // 2 + N * K // 16 + 2 * M * N


def skinny_sweep(device, stream, peaks, steps):
    """Per shape: the nvfp4_linear step, the step on weight scales laid out once
    (nvfp4_linear_laid_out, where the tile width allows) and the GEMM alone, timed over
    rotating buffer sets, against the roofline max(FLOPs / FP4 peak, bytes / HBM peak)."""
    import torch
    fp4_peak = peaks["bf16_tflops"] * NOMINAL_FP4_OVER_BF16
    hbm = peaks["hbm_gbs"]
    out = {}
    for N in SKINNY_N:
        for M in SKINNY_M:
            K = 3072
            L = Nvfp4Layer(M, K, N, False, device)
            rot = Nvfp4Rotation(L)
            reps = max(3, min(steps // rot.R, 20))
            st_ms = time_graph_rotation(rot.step, rot.R, reps, stream)
            # weight scales laid out once (tile widths from 128; the skinny widths lay
            # them out inside the GEMM and have no laid-out call)
            lo_ms = (time_graph_rotation(rot.step_laid_out, rot.R, reps, stream)
                     if L.atoms is not None else None)
            rot.prologue_all()
            g_ms = time_graph_rotation(rot.gemm, rot.R, reps, stream)
            fl = nvfp4_flops(M, K, N)
            b_step = nvfp4_alg_bytes(M, K, N)
            b_gemm = nvfp4_gemm_alg_bytes(M, K, N)
            t_fl = fl / (fp4_peak * 1e12)
            t_gemm_b = b_gemm / (hbm * 1e9)
            t_step_b = b_step / (hbm * 1e9)
            bn, cg = L.q.tile_config(M, N, K)
            out[f"M{M}_N{N}"] = {
                "step_us": st_ms * 1e3, "step_tflops": fl / (st_ms / 1e3) / 1e12,
                "step_gbs": b_step / (st_ms / 1e3) / 1e9,
                "step_roofline_frac": max(t_fl, t_step_b) / (st_ms / 1e3),
                "gemm_us": g_ms * 1e3, "gemm_tflops": fl / (g_ms / 1e3) / 1e12,
                "gemm_gbs": b_gemm / (g_ms / 1e3) / 1e9,
                "gemm_bound": "hbm" if t_gemm_b > t_fl else "tensor",
                "gemm_roofline_frac": max(t_fl, t_gemm_b) / (g_ms / 1e3),
                "tile": f"{128 * cg}x{bn}", "rotation_sets": rot.R,
            }
            if lo_ms is not None:
                out[f"M{M}_N{N}"].update({
                    "step_laid_out_us": lo_ms * 1e3,
                    "step_laid_out_roofline_frac": max(t_fl, t_step_b) / (lo_ms / 1e3)})
            del rot, L
            torch.cuda.empty_cache()
    return out


class _QuietStdout:
    """Sends file descriptor 1 to /dev/null inside the block (library code that prints
    from native code would otherwise break the single JSON line on stdout)."""

    def __enter__(self):
        sys.stdout.flush()
        self._saved = os.dup(1)
        self._null = os.open(os.devnull, os.O_WRONLY)
        os.dup2(self._null, 1)
        return self

    def __exit__(self, *exc):
        sys.stdout.flush()
        os.dup2(self._saved, 1)
        os.close(self._saved)
        os.close(self._null)


def prior_art_flashinfer(M, K, N, device, stream):
    """Context only: the kernels the BFL page names for nvfp4 (FlashInfer's
    nvfp4_quantize and mm_fp4), timed on this GPU on the same shape, over rotating
    operand copies larger than L2 (one CUDA graph per cycle). Library code; none of
    it is on this library's path. Returns a dict, or the reason it could not run."""
    import torch
    try:
        import flashinfer
    except Exception as e:  # pragma: no cover - depends on the image
        return {"unavailable": f"flashinfer import failed: {type(e).__name__}"}
    from synthetic import make_linear_inputs
    inp = make_linear_inputs(M, K, N, seed=0)
    x = inp.x.to(device)
    w = inp.w.to(device)
    # FlashInfer takes the reciprocal global scale: 448 * 6 / amax
    gx = ((448.0 * 6.0) / x.float().abs().amax()).reshape(1).float()
    gw = ((448.0 * 6.0) / w.float().abs().amax()).reshape(1).float()
    alpha = (1.0 / (gx * gw)).float()
    out = {"how": "FlashInfer nvfp4_quantize + mm_fp4 on the same shape; rotating copies, "
                  "one CUDA graph per cycle, mean per call"}
    try:
        xq, xs = flashinfer.nvfp4_quantize(x, gx)
        wq, ws = flashinfer.nvfp4_quantize(w, gw)
        per = xq.numel() + xs.numel() + wq.numel() + ws.numel() + 2 * M * N
        R = max(2, -(-ROTATION_BYTES // per))
        sets = [(xq.clone(), xs.clone(), wq.clone(), ws.clone(),
                 torch.empty(M, N, dtype=torch.bfloat16, device=device)) for _ in range(R)]
        idx = [0]
        for backend in ("cudnn", "cutlass"):
            def gemm(backend=backend):
                a, asf, b, bsf, o = sets[idx[0]]
                idx[0] = (idx[0] + 1) % R
                flashinfer.mm_fp4(a, b.T, asf, bsf.T, alpha, torch.bfloat16, out=o,
                                  backend=backend)
            try:
                ms = time_graph_rotation(gemm, R, 10, stream)
                out[f"mm_fp4_{backend}_us"] = ms * 1e3
                out[f"mm_fp4_{backend}_tflops"] = nvfp4_flops(M, K, N) / (ms / 1e3) / 1e12
            except Exception as e:
                out[f"mm_fp4_{backend}_error"] = f"{type(e).__name__}: {str(e)[:120]}"
        del sets
        xsets = [x.clone() for _ in range(max(2, -(-ROTATION_BYTES // (2 * M * K))))]
        qi = [0]

        def quant():
            xx = xsets[qi[0]]
            qi[0] = (qi[0] + 1) % len(xsets)
            flashinfer.nvfp4_quantize(xx, gx)
        out["nvfp4_quantize_us"] = time_graph_rotation(quant, len(xsets), 10, stream) * 1e3
        del xsets
    except Exception as e:
        out["error"] = f"{type(e).__name__}: {str(e)[:160]}"
    torch.cuda.empty_cache()
    return out


def traffic_from_profiles(kernel_key: str):
    """(per-launch DRAM bytes of a kernel from the committed ncu capture, note): the
    bytes are None, with a note saying so, when there is no capture or the kernel's
    sources changed since it was taken (the counters would describe another kernel)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[kernel_key]
    except (OSError, ValueError, KeyError):
        return None, "no capture recorded in profiles/traffic.json"
    src_hash = source_hash(rec.get("sources", []))
    if src_hash != rec.get("source_sha1"):
        return None, ("stale: the kernel's sources changed since the ncu capture in "
                      "profiles/traffic.json")
    return rec.get("bytes_per_launch"), rec.get("note", "")


def source_hash(files):
    h = hashlib.sha1()
    for rel in files:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


# ----------------------------------------------------------------------------- CPU oracle

def oracle_rows_for(seconds, x, gx, wq, ws, gw, M):
    """Activation rows whose oracle run (quantize + fp64 contraction against the
    whole weight) takes about `seconds`: two timed sizes separate the per-call cost
    (the weight's dequantization) from the per-row cost."""
    import oracle

    def run(rows):
        t0 = time.perf_counter()
        xq, xs = oracle.nvfp4_quantize(x[:rows], gx)
        oracle.nvfp4_linear(xq, xs, wq, ws, gx, gw)
        return time.perf_counter() - t0

    # the oracle spreads rows over its threads: time whole multiples of them
    th = max(1, oracle.get_threads())
    a, b = min(M, 2 * th), min(M, 6 * th)
    t_a = run(a)
    if b == a:
        return a
    t_b = run(b)
    per_row = max((t_b - t_a) / (b - a), 1e-6)
    fixed = max(t_a - a * per_row, 0.0)
    rows = int((seconds - fixed) / per_row) // th * th
    return int(max(1, min(M, max(rows, th))))


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_single_thread():
    """The oracle on one thread for the tiny layer (all of it) and the attention
    projection with bias (a 32-row sample, extrapolated to 4096 rows)."""
    import oracle
    from synthetic import make_linear_inputs
    saved = oracle.get_threads()
    oracle.set_threads(1)
    out = {}
    try:
        for name, (M, K, N, bias, rows) in {
                "tiny_128x256x256": (128, 256, 256, False, 128),
                "attn_proj_4096x3072x3072_bias": (4096, 3072, 3072, True, 32)}.items():
            inp = make_linear_inputs(M, K, N, seed=0, with_bias=bias)
            gw = oracle.nvfp4_global_scale(inp.w)
            wq, ws = oracle.nvfp4_quantize(inp.w, gw)
            gx = oracle.nvfp4_global_scale(inp.x)
            b = None if inp.bias is None else inp.bias.numpy()
            t0 = time.perf_counter()
            xq, xs = oracle.nvfp4_quantize(inp.x[:rows], gx)
            oracle.nvfp4_linear(xq, xs, wq, ws, gx, gw, b)
            t = time.perf_counter() - t0
            out[name] = {"tflops": nvfp4_flops(rows, K, N) / t / 1e12,
                         "seconds_full_layer": t * M / rows,
                         "sample": f"{rows} of {M} rows" + ("" if rows == M else
                                                             ", time extrapolated by rows")}
    finally:
        oracle.set_threads(saved)
    return out


def cpu_oracle_sample(M, K, N, target_s=15.0):
    """Time the oracle (as it stands) on a bounded row sample of the workload:
    activation quantization of the sampled rows + fp64 contraction against the
    whole weight, sized to about `target_s` seconds. Returns (TFLOP/s, threads,
    rows, seconds)."""
    import oracle
    from synthetic import make_linear_inputs
    inp = make_linear_inputs(M, K, N, seed=0)
    gw = oracle.nvfp4_global_scale(inp.w)
    wq, ws = oracle.nvfp4_quantize(inp.w, gw)
    gx = oracle.nvfp4_global_scale(inp.x)
    rows = oracle_rows_for(target_s, inp.x, gx, wq, ws, gw, M)
    t0 = time.perf_counter()
    xq, xs = oracle.nvfp4_quantize(inp.x[:rows], gx)
    oracle.nvfp4_linear(xq, xs, wq, ws, gx, gw)
    t = time.perf_counter() - t0
    return nvfp4_flops(rows, K, N) / t / 1e12, oracle.get_threads(), rows, t


# ----------------------------------------------------------------------------- arms

def run_reference(args):
    """The CPU oracle as the reference arm: each step is a bounded row sample of
    the workload, timed on the host cores."""
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    import numpy as np
    from synthetic import make_linear_inputs
    M, K, N = WORKLOAD["M"], WORKLOAD["K"], WORKLOAD["N"]
    inp = make_linear_inputs(M, K, N, seed=0)
    gw = oracle.nvfp4_global_scale(inp.w)
    wq, ws = oracle.nvfp4_quantize(inp.w, gw)
    gx = oracle.nvfp4_global_scale(inp.x)
    # size one step so that warmup + steps take about two minutes in total
    per_step = 120.0 / max(1, args.steps + args.warmup)
    rows = oracle_rows_for(per_step, inp.x, gx, wq, ws, gw, M)
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        xq, xs = oracle.nvfp4_quantize(inp.x[:rows], gx)
        oracle.nvfp4_linear(xq, xs, wq, ws, gx, gw)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
    sec = statistics.fmean(times)
    value = nvfp4_flops(rows, K, N) / sec / 1e12
    sample = f"{rows} of {M} activation rows per step (all N={N}, K={K}); quantize + fp64 contraction"
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        "config": {"workload": "nvfp4_mlp_up M4096 K3072 N12288", **WORKLOAD},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.get_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    import torch
    import torch.distributed as dist
    world, rank, local = dist_env()
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    stream = torch.cuda.current_stream(device)
    import fp8_rowwise_quantized_b200 as q
    peaks, peak_src = load_peaks()
    M, K, N = WORKLOAD["M"], WORKLOAD["K"], WORKLOAD["N"]

    layer = Nvfp4Layer(M, K, N, bias=False, device=device)
    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)

    def flush():
        # write 256 MB (twice the L2), then read it back: the read evicts the dirty
        # lines of the write, so their write-back happens here, outside the events
        flush_buf.fill_(1)
        flush_buf.view(torch.int32).max()

    flops = nvfp4_flops(M, K, N)
    fp4_peak = peaks["bf16_tflops"] * NOMINAL_FP4_OVER_BF16

    # --------------------------------------------------- headline: timed steps
    # Inputs larger than L2: consecutive steps cycle through R buffer sets (x,
    # weights, y, workspace) that together hold at least four times the L2, so each
    # step reads its operands from HBM, as a stack of distinct layers would. The K
    # timed steps, each bracketed by CUDA event records on the launching stream, are
    # captured in one CUDA graph and replayed once (so no host launch gap lands
    # inside a step); the value is the median step. The clock sampler runs over the
    # warm-up and the timed steps. A step is nvfp4_linear_laid_out: the activations'
    # quantization and the GEMM, on weight scales laid out once at set-up (like the
    # weights' own quantization); the same step laying them out every call is
    # reported beside it (per_call_weight_layout).
    rot = Nvfp4Rotation(layer)
    for _ in range(rot.R):  # every set once before the capture (lazy set-up on the host)
        rot.step_laid_out()
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(args.steps)]
    side = torch.cuda.Stream(device)
    side.wait_stream(stream)
    timed = torch.cuda.CUDAGraph()
    t_host = time.perf_counter()
    with torch.cuda.stream(side):
        with torch.cuda.graph(timed, stream=side):
            for i in range(args.steps):
                starts[i].record(side)
                rot.step_laid_out()
                ends[i].record(side)
    stream.wait_stream(side)
    host_s = time.perf_counter() - t_host
    with ClockSampler(local, period_s=0.002) as clk:
        for _ in range(args.warmup):
            rot.step_laid_out()
        torch.cuda.synchronize()
        barrier(device)
        torch.cuda.synchronize()
        timed.replay()
        torch.cuda.synchronize()
    barrier(device)
    torch.cuda.synchronize()
    step_times = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    del timed
    local_ms = statistics.median(step_times)
    ms, value_flops = aggregate(local_ms, flops, world, device)
    value = value_flops / 1e12
    mean_ms, _ = aggregate(statistics.fmean(step_times), flops, world, device)
    status = q.read_device_status()
    gemm_cycles, gemm_ns = q.read_gemm_clock()     # the last timed step's GEMM
    step_sm_mhz = gemm_cycles / gemm_ns * 1e3 if gemm_ns else None

    # the same step timed two more ways: a 256 MB flush before every step (the
    # operands come from HBM, Y's lines start clean), and warm L2 (the same
    # buffers every step, no flush)
    n_alt = max(20, min(args.steps, 200))
    fl_ms, _ = time_events(layer.step_laid_out, n_alt, 3, flush, stream)
    warm_ms, _ = time_events(layer.step_laid_out, n_alt, 3, None, stream)
    fl_ms, fl_val = aggregate(fl_ms, flops, world, device)
    warm_ms, warm_val = aggregate(warm_ms, flops, world, device)
    # and as one CUDA graph per cycle of buffer sets (no host launch gaps at all)
    graph_ms = time_graph_rotation(rot.step_laid_out, rot.R, max(3, min(args.steps // rot.R, 50)),
                                   stream)
    graph_ms, graph_val = aggregate(graph_ms, flops, world, device)
    # nvfp4_linear, which lays the weight scales out inside every call
    pc_ms = time_graph_rotation(rot.step, rot.R, max(3, min(args.steps // rot.R, 50)), stream)
    pc_ms, pc_val = aggregate(pc_ms, flops, world, device)

    # --------------------------------------------------- roofline of the GEMM kernel
    # the GEMM alone, the prologue alone and the activation quantizer alone, each
    # over the rotating buffer sets, one CUDA graph per cycle of sets (a launch of
    # the short kernels takes less device time than the host needs to issue it, so
    # call-by-call events would time the host)
    tile_bn, tile_cg = q.tile_config(M, N, K)
    reps = max(3, min(args.steps // rot.R, 50))
    rot.prologue_all()
    torch.cuda.synchronize()
    gemm_ms = time_graph_rotation(rot.gemm, rot.R, reps, stream)
    g_cycles, g_ns = q.read_gemm_clock()
    gemm_sm_mhz = g_cycles / g_ns * 1e3 if g_ns else None
    prol_ms = time_graph_rotation(rot.prologue, rot.R, reps, stream)
    quant_ms = time_graph_rotation(rot.quantize_act, rot.R, reps, stream)
    quant_bytes = 2 * M * K + M * K // 2 + M * K // 16
    gemm_tflops = flops / (gemm_ms / 1e3) / 1e12
    prologue_bytes = 2 * M * K + M * K // 2 + M * K // 16 + 2 * (N * K // 16)
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    # dense FP4 MMA rate: 32768 flops per SM per clock (9 PF nominal at 1.855 GHz)
    clock_peak = (sms * 32768 * gemm_sm_mhz * 1e6 / 1e12) if gemm_sm_mhz else None
    traffic, traffic_note = traffic_from_profiles("nvfp4_gemm_mlp_up")
    roofline = {
        "kernel": f"qgemm_kernel<FP4, BN={tile_bn}, {'CTA pair' if tile_cg == 2 else 'one CTA'}> "
                  "(tcgen05 block-scaled FP4 GEMM)",
        "bound": "tensor", "achieved": gemm_tflops, "peak": fp4_peak, "unit": "TFLOP/s",
        "frac": gemm_tflops / fp4_peak,
        "traffic": traffic,
        "traffic_note": traffic_note,
        "peak_source": f"{peak_src} bf16 burst {peaks['bf16_tflops']} TFLOP/s x {NOMINAL_FP4_OVER_BF16} "
                       "(nominal dense FP4:bf16 ratio), of measured",
        "algorithmic": "2*M*K*N flops per launch",
        "gemm_us": gemm_ms * 1e3,
        "gemm_sm_mhz": gemm_sm_mhz,
        "clock_derived_fp4_peak": clock_peak,
        "frac_of_clock_derived_peak": gemm_tflops / clock_peak if clock_peak else None,
        "clock_derived_note": f"{sms} SMs x 32768 flop/clk x the SM clock CTA 0 of the GEMM "
                              "measured over its own run (ql_read_gemm_clock)",
        "frac_of_nominal_9pf": gemm_tflops / 9000.0,
        "prologue_us": prol_ms * 1e3,
        "prologue_gbs": prologue_bytes / (prol_ms / 1e3) / 1e9,
        "prologue_hbm_frac": prologue_bytes / (prol_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
        "quantize_act_us": quant_ms * 1e3,
        "quantize_act_gbs": quant_bytes / (quant_ms / 1e3) / 1e9,
        "quantize_act_hbm_frac": quant_bytes / (quant_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
        "step_frac_of_fp4_peak": value / world / fp4_peak,
        "step_frac_of_nominal_9pf": value / world / 9000.0,
    }

    # --------------------------------------------------- e2e through the public API
    e2e = None
    if not args.no_e2e:
        x_pin = layer.x_host.pin_memory()
        y_pin = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
        x_dev = torch.empty_like(layer.x)

        def e2e_step():
            x_dev.copy_(x_pin, non_blocking=True)
            q.nvfp4_linear_laid_out(x_dev, layer.wq, layer.atoms, layer.bn, layer.gw, layer.gx,
                                    y=layer.y, workspace=layer.work)
            y_pin.copy_(layer.y, non_blocking=True)

        e_steps = max(10, min(args.steps, 50))
        serial_ms, _ = time_events(e2e_step, e_steps, 3, flush, stream)
        serial_ms = reduce_max(serial_ms, device)
        e_ms = time_e2e_pipelined(q, layer, x_pin, e_steps, 3, flush, stream)
        e_ms, e_val = aggregate(e_ms, flops, world, device)
        e2e = {"value": e_val / 1e12, "unit": UNIT, "h2d_bytes_per_step": 2 * M * K,
               "d2h_bytes_per_step": 2 * M * N, "ms_per_step": e_ms,
               "how": "every step copies its X from pinned host memory, runs "
                      "nvfp4_linear_laid_out (256 MB L2 flush before it) and copies its Y to "
                      "pinned host memory; the copy-in, layer and copy-out of consecutive steps "
                      "overlap on three streams (double-buffered X and Y); total time over the "
                      "steps / steps",
               "serial_ms_per_step": serial_ms,
               "serial_how": "the same three steps back to back on one stream, events around "
                             "each; median"}

    # --------------------------------------------------- other layer shapes
    variants = {}
    if not args.no_variants:
        v_steps = max(10, min(args.steps, 100))
        for name, (kind, Mv, Kv, Nv, bias) in {
            "fp8r_4096x3072x3072": ("fp8r", 4096, 3072, 3072, False),
            "nvfp4_attn_proj_4096x3072x3072_bias": ("nvfp4", 4096, 3072, 3072, True),
            "nvfp4_attn_qkv_4096x3072x9216_bias": ("nvfp4", 4096, 3072, 9216, True),
            "nvfp4_mlp_down_4096x12288x3072": ("nvfp4", 4096, 12288, 3072, False),
        }.items():
            L = (Fp8rLayer if kind == "fp8r" else Nvfp4Layer)(Mv, Kv, Nv, bias, device)
            vms, _ = time_events(L.step, v_steps, 3, flush, stream)
            gms, _ = time_events(L.gemm, v_steps, 3, flush, stream)
            fl = nvfp4_flops(Mv, Kv, Nv)
            pk = peaks["bf16_tflops"] * (NOMINAL_FP8_OVER_BF16 if kind == "fp8r" else NOMINAL_FP4_OVER_BF16)
            variants[name] = {"us": vms * 1e3, "tflops": fl / (vms / 1e3) / 1e12,
                              "gemm_us": gms * 1e3, "gemm_tflops": fl / (gms / 1e3) / 1e12,
                              "gemm_frac_of_peak": fl / (gms / 1e3) / 1e12 / pk}
            del L
        torch.cuda.empty_cache()
        # INT4 W4A4 layer on the headline shape: both operands dequantized to f16 (one
        # power-of-two factor per row) and one f16 tensor-core GEMM
        i4 = Int4Layer(M, K, N, False, device)
        i_ms, _ = time_events(i4.step, v_steps, 3, flush, stream)
        ig_ms, _ = time_events(i4.gemm, v_steps, 3, flush, stream)
        f16_peak = peaks["bf16_tflops"]  # f16 and bf16 share the tensor rate
        variants["int4_w4a4_4096x3072x12288"] = {
            "us": i_ms * 1e3, "tops": flops / (i_ms / 1e3) / 1e12,
            "gemm_us": ig_ms * 1e3, "gemm_tops": flops / (ig_ms / 1e3) / 1e12,
            "gemm_frac_of_f16_peak": flops / (ig_ms / 1e3) / 1e12 / f16_peak,
            "tensor_bound_us": flops / (f16_peak * 1e12) * 1e6,
            "note": "int4_linear_gemm = two dequantizations to f16 + one f16 GEMM; "
                    "peak: the measured bf16 rate"}
        del i4
        torch.cuda.empty_cache()
        # svdq_w4a4 NVFP4 layer (rank 32) on the headline shape
        sv = SvdqLayer(M, K, N, 32, device)
        s_ms, _ = time_events(sv.step, v_steps, 3, flush, stream)
        variants["svdq_nvfp4_r32_4096x3072x12288"] = {
            "us": s_ms * 1e3, "tflops": flops / (s_ms / 1e3) / 1e12,
            "lowrank_extra_flops_pct": 100.0 * 2 * 32 * (K + N) / (2 * K * N)}
        del sv
        torch.cuda.empty_cache()
        # MLP block (up 3072 -> 12288, GELU, down 12288 -> 3072): fused GELU + NVFP4
        # requantization epilogue vs up linear, torch GELU, down linear
        mlp = MlpBlock(4096, 3072, 12288, device)
        f_ms, _ = time_events(mlp.fused, v_steps, 3, flush, stream)
        u_ms, _ = time_events(mlp.unfused, v_steps, 3, flush, stream)
        mlp_flops = 2 * nvfp4_flops(4096, 3072, 12288)
        variants["nvfp4_mlp_block_4096x3072x12288"] = {
            "fused_us": f_ms * 1e3, "fused_tflops": mlp_flops / (f_ms / 1e3) / 1e12,
            "unfused_us": u_ms * 1e3, "unfused_tflops": mlp_flops / (u_ms / 1e3) / 1e12}
        del mlp
        torch.cuda.empty_cache()
        # GEMM tile sweep on the headline layer: (128 * cg) x bn output tiles
        sweep = {}
        for bn, cg in [(192, 2), (224, 2), (256, 2), (128, 2), (192, 1)]:
            q.set_tile_override(bn, cg)
            try:
                layer.prologue()
                gms, _ = time_events(layer.gemm, v_steps, 3, flush, stream)
            finally:
                q.set_tile_override(0, 0)
            sweep[f"bn{bn}_cg{cg}"] = {"gemm_us": gms * 1e3,
                                      "gemm_tflops": flops / (gms / 1e3) / 1e12}
        variants["mlp_up_gemm_tile_sweep"] = sweep
        torch.cuda.empty_cache()
        variants["nvfp4_skinny_sweep_K3072"] = skinny_sweep(device, stream, peaks, v_steps)
        variants["w4a16_modulation_sweep"] = w4a16_sweep(device, stream, peaks, v_steps)
    if not args.no_prior_art:
        with _QuietStdout():
            variants["prior_art_flashinfer_mlp_up"] = prior_art_flashinfer(M, K, N, device,
                                                                          stream)

    # --------------------------------------------------- CPU oracle baseline (rank 0, N=1)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tfl, cores, rows, sec = cpu_oracle_sample(M, K, N)
        cpu = {"value": tfl, "unit": UNIT, "cores": cores, "kind": "oracle",
               "cpu_model": cpu_model(),
               "sample": f"{rows} of {M} activation rows, all N={N}, K={K} (quantize + fp64 "
                         f"contraction), {sec:.1f} s",
               "single_thread": oracle_single_thread()}

    clocks = clk.summary()
    clocks["window"] = "NVML samples every 2 ms over the warm-up and the timed steps"
    clocks["gemm_sm_mhz_in_kernel"] = step_sm_mhz
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e2m1xe2m1->f32 (bf16 in/out)", "data": "synthetic",
        "config": {"workload": "nvfp4_mlp_up M4096 K3072 N12288", **WORKLOAD,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": f"inputs larger than L2: {rot.R} buffer sets of "
                         f"{rot.bytes_per_set / 1e6:.0f} MB (x, weights, y, workspace) cycled, "
                         "one per step; value from the median step",
                   "timing": "CUDA events around each step, recorded inside one CUDA graph "
                             "of the K steps (no host launch gaps)",
                   "weight_scales": f"laid out once at set-up for {layer.bn}-row tiles "
                                    "(nvfp4_layout_weight_scales), like the weights' own "
                                    "quantization; a step is nvfp4_linear_laid_out"},
        "frac_of_fp4_peak": value / world / fp4_peak,
        "step_stats": {"median_ms": ms, "mean_ms": mean_ms,
                       "min_ms": min(step_times), "max_ms": max(step_times),
                       "host_capture_us_per_step": host_s / args.steps * 1e6,
                       "how": "the K timed steps captured in one CUDA graph with an event "
                              "record around each step, replayed once"},
        "l2_flushed": {"value": fl_val / 1e12, "ms_per_step": fl_ms,
                       "how": "256 MB written then read before every step, outside the events; "
                              f"median of {n_alt} steps"},
        "l2_warm": {"value": warm_val / 1e12, "ms_per_step": warm_ms,
                    "how": f"the same buffers every step, no flush; median of {n_alt} steps"},
        "l2_rotating_graph": {"value": graph_val / 1e12, "ms_per_step": graph_ms,
                              "how": "the rotating buffer sets, one CUDA graph per cycle of "
                                     "sets; mean over replays"},
        "per_call_weight_layout": {"value": pc_val / 1e12, "ms_per_step": pc_ms,
                                   "how": "nvfp4_linear (the weight scales laid out inside "
                                          "every call), rotating graph as l2_rotating_graph"},
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "clocks": clocks,
        "gpu_launches": 2 * args.steps,
        "device_status": status,
        "variants": variants,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        barrier(device)
        dist.destroy_process_group()
    return 0


def run_profile(args):
    """Short fixed sequence for profilers: `--profile <piece>` runs `--steps` calls
    of one piece of the headline workload (no flushes, no timing): `step` (the
    headline step, nvfp4_linear_laid_out), `step_per_call_layout` (nvfp4_linear),
    `prologue`, `gemm`, `quant` (activation quantization alone), `mlp_fused` (the MLP
    block with the GELU-quantize epilogue), `svdq` (the rank-32 svdq layer), `fp8r_step`,
    `fp8r_quant`, `fp8r_gemm`, `int4` (the INT4 W4A4 layer on the headline shape),
    `w4a16` (the 1 x 3072 x 18432 modulation layer over
    rotating weight copies) or `skinny_<M>_<N>` (nvfp4_linear at K = 3072 over
    rotating copies)."""
    import torch
    torch.cuda.set_device(0)
    device = torch.device("cuda", 0)
    M, K, N = WORKLOAD["M"], WORKLOAD["K"], WORKLOAD["N"]
    if args.profile == "mlp_fused":
        mlp = MlpBlock(4096, 3072, 12288, device)
        fn = mlp.fused
    elif args.profile == "svdq":
        sv = SvdqLayer(4096, 3072, 12288, 32, device)
        fn = sv.step
    elif args.profile == "int4":
        L4 = Int4Layer(M, K, N, False, device)
        fn = L4.step
    elif args.profile == "w4a16":
        W = W4a16Rotation(1, 3072, 18432, device)
        fn = W.step
    elif args.profile.startswith("skinny"):
        # skinny_<M>_<N>: the nvfp4_linear step at K = 3072 over rotating copies
        _, Ms, Ns = args.profile.split("_")
        rot = Nvfp4Rotation(Nvfp4Layer(int(Ms), 3072, int(Ns), False, device))
        fn = rot.step
    elif args.profile.startswith("fp8r"):
        L = Fp8rLayer(4096, 3072, 3072, False, device)
        fn = {"fp8r_step": L.step, "fp8r_gemm": L.gemm,
              "fp8r_quant": lambda: L.q.fp8r_quantize_rows(L.x, L.xq, L.xs)}[args.profile]
    else:
        L = Nvfp4Layer(M, K, N, False, device)
        L.prologue()
        xq = torch.empty((M, K // 2), dtype=torch.uint8, device=device)
        xs = torch.empty((M, K // 16), dtype=torch.uint8, device=device)
        fn = {"step": L.step_laid_out, "step_per_call_layout": L.step, "prologue": L.prologue,
              "gemm": L.gemm,
              "quant": lambda: L.q.nvfp4_quantize_act(L.x, L.gx, xq, xs)}[args.profile]
    for _ in range(args.steps):
        fn()
    torch.cuda.synchronize()
    import fp8_rowwise_quantized_b200 as q
    assert q.read_device_status() == 0
    print(json.dumps({"profile": args.profile, "steps": args.steps, "ok": True}))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-variants", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prior-art", action="store_true",
                    help="skip timing FlashInfer's NVFP4 kernels (context only)")
    ap.add_argument("--profile", choices=["step", "step_per_call_layout", "prologue", "gemm",
                                          "quant", "mlp_fused", "svdq",
                                          "fp8r_step", "fp8r_quant", "fp8r_gemm", "w4a16", "int4",
                                          "skinny_16_3072", "skinny_16_12288",
                                          "skinny_256_12288"], default=None,
                    help="run a short fixed sequence for a profiler instead of the benchmark")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps
    if args.profile:
        return run_profile(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
