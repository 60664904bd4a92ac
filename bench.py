"""Benchmark of the QLoRA NF4 linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one training pass of a LLaMA-7B-shaped decoder layer's seven NF4
projections (q/k/v/o 4096x4096, gate/up 11008x4096, down 4096x11008) at 2048
tokens (batch 4 x seq 512), LoRA r=16, alpha=32: the forward of every
projection (T = X A^T, fused dequant GEMM with the adapter folded in) and the
backward in reverse order (G, fused dX GEMM, dA, dB).  The weights are
quantised once before timing (the pages quantise at load time); the
quantiser, the standalone dequantiser and the decode-shaped forward (70B MLP
weights, M in {1, 4, 16}) are timed as separate sub-measurements of the same
run and reported in the same JSON line.

Metric: algorithmic TFLOP/s = sum over projections of 4*M*N*K + 6*M*r*(N+K)
per step / device time.  Inputs are synthetic (seeded normal draws).
Data-parallel over N GPUs: every rank runs the same per-GPU workload on its
own token shard (weak scaling) and the adapter gradients dA, dB are summed
over ranks with one NCCL all-reduce per step.

--impl reference times the CPU oracle (binary64 numpy + plain C), as it
stands, on a bounded sample of the same step (a slice of the tokens).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from bit_nf4_quantized_21_b200 import inputs  # noqa: E402

METRIC = "QLoRA linear fwd+bwd TFLOP/s; NF4 GEMV weight GB/s; % of roofline"
WL = inputs.LLAMA7B
L2_BYTES = 126 * 1024 * 1024
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# DRAM traffic of one fused-GEMM launch (gate forward) from the ncu capture
# summarised in profiles/k_gemm_nf4_pair_fwd_gate_m2048.md; None once the
# kernel changes and until it is captured again.
GEMM_TRAFFIC_BYTES = 51.67e6


def step_flops(wl=WL, M=None) -> float:
    M = wl.M if M is None else M
    return float(sum(4 * M * N * K + 6 * M * wl.r * (N + K) for _, N, K in wl.shapes))


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int, log_dir: str | None = None):
        """Samples go to <log_dir>/clocks_rank<index>.csv (the system's
        temporary directory when no log_dir is given)."""
        import tempfile
        self.index = index
        self.proc = None
        self.path = os.path.join(log_dir or tempfile.gettempdir(), f"clocks_rank{index}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], 0.0, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                clk, cmax = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            mx = max(mx, cmax)
            sm.append(clk)
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        busy = [c for c in sm if c > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------- our path
def grad_buffer(shapes, r, device):
    """One flat fp32 buffer holding every projection's dA [r, K] and dB [N, r]
    as consecutive views: the kernels write the gradients straight into it and
    the data-parallel sum is one in-place all-reduce.  Returns (flat, [(dA, dB)
    per projection]).  Every view starts on a 16-byte boundary (K % 64 == 0,
    N % 8 == 0)."""
    sizes = []
    for _, N, K in shapes:
        sizes += [(r, K), (N, r)]
    flat = torch.zeros(sum(a * b for a, b in sizes), dtype=torch.float32, device=device)
    views, off = [], 0
    for a, b in sizes:
        views.append(flat[off:off + a * b].view(a, b))
        off += a * b
    return flat, [(views[2 * i], views[2 * i + 1]) for i in range(len(shapes))]


def allreduce_sum(flat, world):
    """Data parallel: every rank ends with the sum of the gradients over all
    ranks (the step's loss is the sum over every rank's tokens)."""
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(flat)


def max_over_ranks(x, world, device):
    """Slowest rank's value of a per-rank time."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# Input each projection reads: in a LLaMA decoder layer q, k and v project
# the same normalised hidden state, and gate and up the same one.
X_SOURCE = {"q": "q", "k": "q", "v": "q", "o": "o", "gate": "gate", "up": "gate", "down": "down"}


# Projections of a decoder layer that do not depend on one another: q, k and
# v read the same input, and so do gate and up.  o needs attention's output
# and down the gated MLP product, so each of those runs alone.
CONCURRENT_GROUPS = (("q", "k", "v"), ("o",), ("gate", "up"), ("down",))


class Layer:
    """Seven NF4 projections of one layer, resident on the device (q/k/v and
    gate/up share their input tensor, as in the model)."""

    def __init__(self, q, wl, M, device, rank):
        self.q = q
        self.wl = wl
        self.M = M
        self.proj = []
        self.grad_flat, grads = grad_buffer(wl.shapes, wl.r, device)
        index = {name: i for i, (name, _, _) in enumerate(wl.shapes)}
        self.x = {}
        for i, (name, N, K) in enumerate(wl.shapes):
            seed = inputs.matrix_seed(wl.base_seed, rank, i)
            xk = X_SOURCE[name]
            if xk not in self.x:
                self.x[xk] = inputs.normal((M, K), 1.0, inputs.matrix_seed(wl.base_seed, rank, index[xk]) * 16 + 1,
                                           device)
            W = inputs.weight((N, K), wl.w_std, seed, device=device)
            Wq = q.empty_nf4(N, K, device)
            p = dict(name=name, N=N, K=K, W_bf16_bytes=W.numel() * 2)
            p["Wq"] = Wq
            p["W_tmp"] = W
            p["X"] = self.x[xk]
            p["xkey"] = xk
            p["dY"] = inputs.normal((M, N), 1.0, seed * 16 + 2, device)
            p["A"] = inputs.normal((wl.r, K), 0.01, seed * 16 + 3, device)
            p["B"] = inputs.normal((N, wl.r), 0.01, seed * 16 + 4, device)
            p["Y"] = torch.empty((M, N), dtype=torch.bfloat16, device=device)
            p["T"] = torch.empty((M, wl.r), dtype=torch.float32, device=device)
            p["dX"] = torch.empty((M, K), dtype=torch.bfloat16, device=device)
            p["dA"], p["dB"] = grads[i]
            self.proj.append(p)
        ws = max(q.qlora_workspace_bytes(M, p["N"], p["K"], wl.r) for p in self.proj)
        self.ws = torch.empty(ws, dtype=torch.uint8, device=device)
        # a workspace per projection, for projections that run concurrently
        self.wss = [torch.empty(q.qlora_workspace_bytes(M, p["N"], p["K"], wl.r), dtype=torch.uint8, device=device)
                    for p in self.proj]
        self.groups = [[index[n] for n in g] for g in CONCURRENT_GROUPS if all(n in index for n in g)]
        self.side = [torch.cuda.Stream(device=device) for _ in range(max(len(g) for g in self.groups))]
        self.status = torch.zeros(1, dtype=torch.int32, device=device)

    def quantize_all(self, events=None):
        for p in self.proj:
            if events is not None:
                events.append((torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)))
                events[-1][0].record()
            self.q.qlora_quantize_nf4(p["W_tmp"], out=p["Wq"], d_status=self.status)
            if events is not None:
                events[-1][1].record()

    def drop_source_weights(self):
        for p in self.proj:
            p.pop("W_tmp", None)

    def _fwd(self, i, ev, ws):
        p = self.proj[i]
        self.q.qlora_linear_fwd(p["X"], p["Wq"], p["A"], p["B"], self.wl.alpha, Y=p["Y"], T_save=p["T"],
                                workspace=ws, d_status=self.status, gemm_events=ev)

    def _bwd(self, i, ev, ws):
        p = self.proj[i]
        self.q.qlora_linear_bwd(p["dY"], p["X"], p["Wq"], p["A"], p["B"], self.wl.alpha, T_saved=p["T"],
                                dX=p["dX"], dA=p["dA"], dB=p["dB"], workspace=ws, d_status=self.status,
                                gemm_events=ev)

    def _group(self, idx, fn, evs):
        """Run fn(i, ev, ws) for the projections idx: alone on the current
        stream, or each on a side stream forked from and joined back into it."""
        main = torch.cuda.current_stream()
        if len(idx) == 1:
            fn(idx[0], evs.get(idx[0]), self.wss[idx[0]])
            return
        fork = torch.cuda.Event()
        fork.record(main)
        joins = []
        for s, i in zip(self.side, idx):
            s.wait_event(fork)
            with torch.cuda.stream(s):
                fn(i, evs.get(i), self.wss[i])
                e = torch.cuda.Event()
                e.record(s)
            joins.append(e)
        for e in joins:
            main.wait_event(e)

    def step_concurrent(self, gemm_events=None):
        """The step with independent projections overlapped (CONCURRENT_GROUPS):
        forward group by group, then backward in reverse group order."""
        n = len(self.proj)
        fev = {i: gemm_events[i] for i in range(n)} if gemm_events else {}
        bev = {i: gemm_events[n + (n - 1 - i)] for i in range(n)} if gemm_events else {}
        for g in self.groups:
            self._group(g, self._fwd, fev)
        for g in reversed(self.groups):
            self._group(list(reversed(g)), self._bwd, bev)

    def step(self, gemm_events=None):
        """Forward of all 7 projections, then backward in reverse order."""
        alpha = self.wl.alpha
        for p in self.proj:
            ev = gemm_events.pop(0) if gemm_events else None
            self.q.qlora_linear_fwd(p["X"], p["Wq"], p["A"], p["B"], alpha, Y=p["Y"], T_save=p["T"],
                                    workspace=self.ws, d_status=self.status, gemm_events=ev)
        for p in reversed(self.proj):
            ev = gemm_events.pop(0) if gemm_events else None
            self.q.qlora_linear_bwd(p["dY"], p["X"], p["Wq"], p["A"], p["B"], alpha, T_saved=p["T"],
                                    dX=p["dX"], dA=p["dA"], dB=p["dB"], workspace=self.ws,
                                    d_status=self.status, gemm_events=ev)

    def step_dense(self, Wd):
        """The same step over dense bf16 weights Wd (one per projection):
        plain LoRA through the same GEMM, the baseline QLoRA is compared to."""
        alpha = self.wl.alpha
        for p, W in zip(self.proj, Wd):
            self.q.qlora_lora_linear_fwd(p["X"], W, p["A"], p["B"], alpha, Y=p["Y"], T_save=p["T"],
                                         workspace=self.ws, d_status=self.status)
        for p, W in zip(reversed(self.proj), reversed(Wd)):
            self.q.qlora_lora_linear_bwd(p["dY"], p["X"], W, p["A"], p["B"], alpha, T_saved=p["T"],
                                         dX=p["dX"], dA=p["dA"], dB=p["dB"], workspace=self.ws,
                                         d_status=self.status)

    def step_e2e(self, hostX, hostdY, hostdA, hostdB, s_h2d, s_d2h, ev, allreduce=None):
        """One step from pinned host buffers: each distinct input X (hostX,
        keyed like self.x) and each dY are copied in on s_h2d while earlier
        projections compute (X in forward order of first use, then dY in
        backward order), each projection waits only for its own inputs, and
        its gradients go back on s_d2h as soon as its backward is done.
        `ev` brackets the whole step on the compute stream."""
        q, alpha = self.q, self.wl.alpha
        comp = torch.cuda.current_stream()
        ev[0].record(comp)
        fork = torch.cuda.Event()      # an ordinary event for the fork: the timing one may be a graph node
        fork.record(comp)
        s_h2d.wait_event(fork)
        ready_x, ready_dy = {}, {}
        with torch.cuda.stream(s_h2d):
            for p in self.proj:
                xk = p["xkey"]
                if xk in ready_x:
                    continue
                self.x[xk].copy_(hostX[xk], non_blocking=True)
                e = torch.cuda.Event()
                e.record(s_h2d)
                ready_x[xk] = e
            for i in reversed(range(len(self.proj))):
                self.proj[i]["dY"].copy_(hostdY[i], non_blocking=True)
                e = torch.cuda.Event()
                e.record(s_h2d)
                ready_dy[i] = e
        for p in self.proj:
            comp.wait_event(ready_x[p["xkey"]])
            q.qlora_linear_fwd(p["X"], p["Wq"], p["A"], p["B"], alpha, Y=p["Y"], T_save=p["T"],
                               workspace=self.ws, d_status=self.status)
        done = {}
        for i in reversed(range(len(self.proj))):
            p = self.proj[i]
            comp.wait_event(ready_dy[i])
            q.qlora_linear_bwd(p["dY"], p["X"], p["Wq"], p["A"], p["B"], alpha, T_saved=p["T"],
                               dX=p["dX"], dA=p["dA"], dB=p["dB"], workspace=self.ws, d_status=self.status)
            e = torch.cuda.Event()
            e.record(comp)
            done[i] = e
        if allreduce is not None:      # data parallel: gradients are summed first
            allreduce()
            e = torch.cuda.Event()
            e.record(comp)
            done = {i: e for i in done}
        for i in reversed(range(len(self.proj))):
            s_d2h.wait_event(done[i])
            with torch.cuda.stream(s_d2h):
                hostdA[i].copy_(self.proj[i]["dA"], non_blocking=True)
                hostdB[i].copy_(self.proj[i]["dB"], non_blocking=True)
        fin = torch.cuda.Event()
        fin.record(s_d2h)
        comp.wait_event(fin)
        ev[1].record(comp)

    def gemm_flops(self):
        """Algorithmic flops of each fused-GEMM launch, in step order."""
        r = self.wl.r
        f = [2 * self.M * p["N"] * p["K"] + 2 * self.M * r * p["N"] for p in self.proj]
        b = [2 * self.M * p["N"] * p["K"] + 2 * self.M * r * p["K"] for p in reversed(self.proj)]
        return f + b


def capture_graph(fn):
    """One CUDA graph of everything fn enqueues (the library's calls validate
    on the host and only enqueue, so they can be captured).  Events fn records
    must already exist (record them once outside the capture)."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def flush_l2(buf):
    buf.add_(1)


def launches_per_step(wl) -> int:
    # this library's kernels per projection: forward T skinny + fused GEMM;
    # backward G skinny (+ T planes) + dX GEMM + one dA/dB skinny (+1 pad of
    # B when r % 8).  The counter clears are memset nodes, not kernels.
    pad = 1 if wl.r % 8 else 0
    return len(wl.shapes) * (2 + 3 + pad)


def run_ours(args):
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import bit_nf4_quantized_21_b200 as q
    q.lib()  # fails loudly when the library is missing
    peaks, peaks_src = load_peaks()

    def barrier():
        if world > 1:
            dist.barrier()

    # ---- setup: draw and quantise the layer (quantiser timed here, after a
    # warm-up call that pays the one-time module load)
    layer = Layer(q, WL, WL.M, dev, rank)
    layer.quantize_all()
    torch.cuda.synchronize()
    # a short device-side spin first, so that all 7 launches are queued before
    # the first event: the events then time the kernels, not the host's
    # launch gaps (each Python call takes longer to issue than its kernel runs)
    qev = []
    torch.cuda._sleep(2_000_000)
    layer.quantize_all(events=qev)
    torch.cuda.synchronize()
    quant_ms = sum(a.elapsed_time(b) for a, b in qev)
    n_params = sum(p["N"] * p["K"] for p in layer.proj)
    quant_bytes = sum(p["W_bf16_bytes"] + p["Wq"].nbytes() for p in layer.proj)
    layer.drop_source_weights()
    torch.cuda.empty_cache()
    assert layer.status.item() == 0, "quantiser reported non-finite weights"

    l2buf = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    def allreduce_grads():
        allreduce_sum(layer.grad_flat, world)

    # ---- warm-up
    for _ in range(args.warmup):
        layer.step()
        allreduce_grads()
    torch.cuda.synchronize()

    # ---- timed device steps (inputs resident), L2 flushed between steps
    nproj = len(layer.proj)
    gemm_ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(2 * nproj)] for _ in range(args.steps)]
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
    graphs = seq_graphs = None
    concurrent = not args.sequential and not args.no_graph
    if not args.no_graph:
        # one graph per timed step: a replay launches the step's 35 kernels
        # and memsets without the host's per-launch gaps between them.  The
        # headline step overlaps the layer's independent projections
        # (q/k/v, gate/up); the roofline pass replays the same calls in
        # sequence, each graph with its own GEMM timing events, so that each
        # fused-GEMM launch is timed alone
        for evs in gemm_ev:
            for a, b in evs:
                a.record(); b.record()
        torch.cuda.synchronize()
        seq_graphs = [capture_graph(lambda i=i: layer.step(gemm_events=list(gemm_ev[i]))) for i in range(args.steps)]
        graphs = ([capture_graph(layer.step_concurrent) for _ in range(args.steps)] if concurrent else seq_graphs)
        graphs[0].replay()
        seq_graphs[0].replay()
        torch.cuda.synchronize()
    clocks = ClockSampler(local, args.clock_log)
    clocks.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush_l2(l2buf)
        step_ev[i][0].record()
        if graphs is not None:
            graphs[i].replay()
        else:
            layer.step(gemm_events=list(gemm_ev[i]))
        allreduce_grads()
        step_ev[i][1].record()
    torch.cuda.synchronize()
    barrier()
    step_ms = [a.elapsed_time(b) for a, b in step_ev]
    seq_ms = step_ms
    if concurrent:
        # roofline pass: the same steps in sequence (L2 flushed likewise)
        seq_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
        for i in range(args.steps):
            flush_l2(l2buf)
            seq_ev[i][0].record()
            seq_graphs[i].replay()
            seq_ev[i][1].record()
        torch.cuda.synchronize()
        seq_ms = [a.elapsed_time(b) for a, b in seq_ev]
    clk = clocks.stop()
    gemm_ms = [[a.elapsed_time(b) for a, b in evs] for evs in gemm_ev]
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    assert layer.status.item() == 0, f"device status {layer.status.item()}"
    flops = step_flops() * args.steps * world
    value = flops / (total_ms * 1e-3) / 1e12

    # ---- roofline of the dominant kernel (fused NF4 GEMM), from the live events
    gflops = layer.gemm_flops()
    g_time = sum(sum(x) for x in gemm_ms) * 1e-3
    g_launches = len(gflops) * args.steps
    g_achieved = sum(gflops) * args.steps / g_time / 1e12
    peak_sus = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
    peak_burst = float(peaks.get("bf16_tflops"))
    gemm_share = g_time * 1e3 / sum(seq_ms)

    # ---- end to end through host buffers (pinned), copies inside the timed region
    e2e = None
    if not args.no_e2e:
        hostX = {k: x.cpu().pin_memory() for k, x in layer.x.items()}
        hostdY = [p["dY"].cpu().pin_memory() for p in layer.proj]
        hostdA = [torch.empty_like(p["dA"], device="cpu").pin_memory() for p in layer.proj]
        hostdB = [torch.empty_like(p["dB"], device="cpu").pin_memory() for p in layer.proj]
        h2d = sum(t.numel() * t.element_size() for t in list(hostX.values()) + hostdY)
        d2h = sum(t.numel() * t.element_size() for t in hostdA + hostdB)
        # external: recorded as event nodes when captured into a graph
        e_ev = [(torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True))
                for _ in range(args.steps)]
        s_h2d, s_d2h = torch.cuda.Stream(), torch.cuda.Stream()
        egraphs = None
        if not args.no_graph and world == 1:
            # the whole end-to-end step -- copies in, kernels, copies out --
            # as one graph per timed step (NCCL stays outside graphs)
            for a, b in e_ev:
                a.record(); b.record()
            torch.cuda.synchronize()
            egraphs = [capture_graph(lambda i=i: layer.step_e2e(hostX, hostdY, hostdA, hostdB, s_h2d, s_d2h,
                                                                e_ev[i]))
                       for i in range(args.steps)]
        barrier()
        torch.cuda.synchronize()
        for i in range(args.steps):
            flush_l2(l2buf)
            if egraphs is not None:
                egraphs[i].replay()
            else:
                layer.step_e2e(hostX, hostdY, hostdA, hostdB, s_h2d, s_d2h, e_ev[i],
                               allreduce_grads if world > 1 else None)
        torch.cuda.synchronize()
        barrier()
        e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in e_ev), world, dev)
        e2e = {"value": round(flops / (e_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": round(e_ms / args.steps, 4)}

    # ---- sub-measurements: standalone dequantiser and decode-shaped forward
    sub = {}
    if not args.no_sub and rank == 0:
        sub = sub_measurements(q, dev, peaks, l2buf, layer, quant_ms, quant_bytes, n_params)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(layer, args.cpu_tokens, dev, legs=not args.no_cpu_legs)

    hbm = float(peaks["hbm_gbs"])
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": "llama7b-layer-7proj-fwd+bwd", "tokens_per_gpu": WL.M,
                   "batch": 4, "seq_len": 512, "lora_r": WL.r, "lora_alpha": WL.alpha,
                   "projections": [[n, N, K] for n, N, K in WL.shapes],
                   "inputs": "q/k/v read one X, gate/up another (as in the decoder layer)",
                   "weights": "NF4 double-quant, block 64, group 256",
                   "flops_per_step": step_flops(), "l2": "flushed between timed steps",
                   "launch": ("each timed step replays a CUDA graph of its library calls; independent "
                              "projections (q/k/v, then gate/up; their backward likewise) overlap on side "
                              "streams, o and down run alone" if concurrent else
                              "each timed step replays a CUDA graph of its library calls, in sequence")
                             if graphs is not None else "library calls launched one by one",
                   "parallelism": f"dp{world}"},
        "roofline": {"bound": "tensor", "kernel": "k_gemm_nf4_pair (fused NF4 dequant + 2-SM tcgen05 GEMM)",
                     "achieved": round(g_achieved, 2), "peak": round(peak_burst, 1), "unit": "TFLOP/s",
                     "frac": round(g_achieved / peak_burst, 4),
                     # the timed region is tens of milliseconds at the maximum
                     # clock (see "clocks"): burst conditions, so the burst peak
                     "peak_source": f"{peaks_src} bf16_tflops (burst)",
                     "frac_of_sustained_peak": round(g_achieved / peak_sus, 4),
                     "launches": g_launches, "avg_launch_us": round(g_time / g_launches * 1e6, 2),
                     "share_of_step": round(gemm_share, 4),
                     "timed_on": ("a sequential replay of the same step graphs right after the timed steps "
                                  f"({round(sum(seq_ms) / len(seq_ms), 4)} ms per step), each launch alone"
                                  if concurrent else "the timed steps"),
                     # DRAM bytes (read + write) of one launch, from the ncu capture in
                     # profiles/k_gemm_nf4_pair_fwd_gate_m2048.md (gate forward,
                     # 2048 x 11008 x 4096); its algorithmic bytes are 85.1 MB, most of
                     # Y still sitting in L2 at the end of the kernel
                     "traffic": GEMM_TRAFFIC_BYTES, "traffic_launch": "gate fwd, M 2048 x N 11008 x K 4096",
                     "traffic_algorithmic": 85.1e6},
        "gpu_launches": launches_per_step(WL) * args.steps,
        "clocks": clk,
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    line.update(sub)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def time_events(fn, reps, flush=None):
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for a, b in evs:
        if flush is not None:
            flush()
        a.record()
        fn()
        b.record()
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def _quantize_model(q, wl, dev, status):
    """Generate every weight of workload `wl` on the device one matrix at a
    time, quantise it into resident NF4 storage and free the bf16 source.
    Returns (nf4 weights [layer][projection], quantiser kernel ms, params)."""
    nf4, evs, params = [], [], 0
    for L in range(wl.layers):
        row = []
        for i, (name, N, K) in enumerate(wl.shapes):
            W = inputs.weight((N, K), wl.w_std, inputs.matrix_seed(wl.base_seed, L, i), device=dev)
            Wq = q.empty_nf4(N, K, dev)
            ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            ev[0].record()
            q.qlora_quantize_nf4(W, out=Wq, d_status=status)
            ev[1].record()
            evs.append(ev)
            del W
            row.append(Wq)
            params += N * K
        nf4.append(row)
    torch.cuda.synchronize()
    return nf4, sum(a.elapsed_time(b) for a, b in evs), params


def _layer_tensors(wl, L, M, dev, x_shared=True):
    """Adapters and activations of one layer.  With x_shared, q/k/v read one
    input and gate/up another, as in a LLaMA decoder layer."""
    index = {name: i for i, (name, _, _) in enumerate(wl.shapes)}
    xs, out = {}, []
    for i, (name, N, K) in enumerate(wl.shapes):
        seed = inputs.matrix_seed(wl.base_seed, L, i)
        k = index[X_SOURCE[name]] if x_shared else i
        if k not in xs:
            xs[k] = inputs.normal((M, K), 1.0, inputs.matrix_seed(wl.base_seed, L, k) * 16 + 1, dev)
        out.append(dict(X=xs[k], dY=inputs.normal((M, N), 1.0, seed * 16 + 2, dev),
                        A=inputs.normal((wl.r, K), 0.01, seed * 16 + 3, dev),
                        B=inputs.normal((N, wl.r), 0.01, seed * 16 + 4, dev),
                        T=torch.empty((M, wl.r), dtype=torch.float32, device=dev),
                        dA=torch.empty((wl.r, K), dtype=torch.float32, device=dev),
                        dB=torch.empty((N, wl.r), dtype=torch.float32, device=dev)))
    return out


def run_concurrent(idx, fn, side):
    """fn(i) for the projections idx: alone on the current stream, or each on a
    side stream forked from and joined back into it."""
    main = torch.cuda.current_stream()
    if len(idx) == 1:
        fn(idx[0])
        return
    fork = torch.cuda.Event()
    fork.record(main)
    joins = []
    for st, i in zip(side, idx):
        st.wait_event(fork)
        with torch.cuda.stream(st):
            fn(i)
            e = torch.cuda.Event()
            e.record(st)
        joins.append(e)
    for e in joins:
        main.wait_event(e)


def _model_step(q, wl, nf4, acts, bufs, wss, status, layers, side):
    """Forward through every projection of `layers`, then backward in reverse;
    within a layer the independent projections (CONCURRENT_GROUPS) overlap."""
    index = {n: i for i, (n, _, _) in enumerate(wl.shapes)}
    groups = [[index[n] for n in g] for g in CONCURRENT_GROUPS if all(n in index for n in g)]

    def fwd(L, i):
        a = acts[L][i]
        q.qlora_linear_fwd(a["X"], nf4[L][i], a["A"], a["B"], wl.alpha, Y=bufs[i]["Y"], T_save=a["T"],
                           workspace=wss[i], d_status=status)

    def bwd(L, i):
        a = acts[L][i]
        q.qlora_linear_bwd(a["dY"], a["X"], nf4[L][i], a["A"], a["B"], wl.alpha, T_saved=a["T"],
                           dX=bufs[i]["dX"], dA=a["dA"], dB=a["dB"], workspace=wss[i], d_status=status)

    for L in layers:
        for g in groups:
            run_concurrent(g, lambda i: fwd(L, i), side)
    for L in reversed(layers):
        for g in reversed(groups):
            run_concurrent(list(reversed(g)), lambda i: bwd(L, i), side)


def _time_model_step(q, wl, nf4, acts, M, dev, layers, steps, warmup):
    """The whole-model step captured once as a CUDA graph and replayed."""
    bufs = [dict(Y=torch.empty((M, N), dtype=torch.bfloat16, device=dev),
                 dX=torch.empty((M, K), dtype=torch.bfloat16, device=dev)) for (_, N, K) in wl.shapes]
    wss = [torch.empty(q.qlora_workspace_bytes(M, N, K, wl.r), dtype=torch.uint8, device=dev)
           for (_, N, K) in wl.shapes]
    side = [torch.cuda.Stream(device=dev) for _ in range(max(len(g) for g in CONCURRENT_GROUPS))]
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    run = lambda: _model_step(q, wl, nf4, acts, bufs, wss, status, layers, side)
    run()                                  # eager once (first-use costs), then capture
    torch.cuda.synchronize()
    g = capture_graph(run)
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    ms = time_events(g.replay, steps)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, "device status set during a config workload"
    t = statistics.median(ms)
    flops = len(layers) * step_flops(wl, M)
    return {"value": round(flops / (t * 1e-3) / 1e12, 2), "unit": "TFLOP/s", "ms_per_step": round(t, 3),
            "tokens": M, "layers": len(layers), "flops_per_step": flops, "steps": steps, "warmup": warmup,
            "launch": "one CUDA graph per step; q/k/v and gate/up overlap within each layer"}


def config_workloads(q, dev, hbm):
    """The 32-layer 7B stack and the 80-layer 65B model: whole-model one-shot
    quantisation on the GPU, then training steps through the resident NF4
    weights (all 224 projections at 4096 tokens; one 65B layer at 8192)."""
    out = {}
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    # 32-layer LLaMA-7B-shaped stack, 4096 tokens, r = 16
    wl = inputs.STACK7B
    nf4, qms, params = _quantize_model(q, wl, dev, status)
    qbytes = params * (2 + 0.5 + 1 / 64 + 4 / 16384)
    acts = [_layer_tensors(wl, L, wl.M, dev) for L in range(wl.layers)]
    torch.cuda.synchronize()
    step = _time_model_step(q, wl, nf4, acts, wl.M, dev, list(range(wl.layers)), steps=10, warmup=3)
    out["stack7b_32layer"] = {
        "quantize": {"params": params, "ms": round(qms, 3), "value": round(qbytes / (qms * 1e-3) / 1e9, 1),
                     "unit": "GB/s (bf16 in + NF4 out)", "frac_of_hbm": round(qbytes / (qms * 1e-3) / 1e9 / hbm, 4),
                     "nf4_resident_gb": round(sum(w.nbytes() for row in nf4 for w in row) / 1e9, 3)},
        "step": step}
    del nf4, acts
    torch.cuda.empty_cache()
    # 80-layer LLaMA-65B-shaped model: all weights quantised and resident,
    # then one layer's 7 projections at 8192 tokens, r = 64
    wl = inputs.LLAMA65B
    nf4, qms, params = _quantize_model(q, wl, dev, status)
    qbytes = params * (2 + 0.5 + 1 / 64 + 4 / 16384)
    resident = sum(w.nbytes() for row in nf4 for w in row)
    acts = {0: _layer_tensors(wl, 0, wl.M, dev)}
    torch.cuda.synchronize()
    step = _time_model_step(q, wl, nf4, acts, wl.M, dev, [0], steps=10, warmup=3)
    assert int(status.item()) == 0
    out["llama65b_80layer"] = {
        "quantize": {"params": params, "ms": round(qms, 3), "value": round(qbytes / (qms * 1e-3) / 1e9, 1),
                     "unit": "GB/s (bf16 in + NF4 out)", "frac_of_hbm": round(qbytes / (qms * 1e-3) / 1e9 / hbm, 4),
                     "nf4_resident_gb": round(resident / 1e9, 3)},
        "layer_step": step}
    del nf4, acts
    torch.cuda.empty_cache()
    return out


def paged_adam(q, master, mom1, mom2, grad, pbf, status, l2buf, hbm):
    """The Adam step over paged optimiser state (CUDA managed memory from
    qlora_paged_alloc), the same n parameters as adam_step: with the state
    resident on the GPU; paged out to the host before each step, which
    faults it back in; and paged out, then prefetched back inside the timed
    region.  Migration bytes per step in the last two: 12 B per parameter."""
    import ctypes
    import numpy as np
    n = master.numel()
    stream = torch.cuda.current_stream()
    ptrs = [q.qlora_paged_alloc(4 * n) for _ in range(3)]
    try:
        for ptr, src in zip(ptrs, (master, mom1, mom2)):
            np.ctypeslib.as_array((ctypes.c_float * n).from_address(ptr))[:] = src.cpu().numpy()
        step_no = [0]

        def step():
            step_no[0] += 1
            rc = q.lib().qlora_adam_step(ptrs[0], ptrs[1], ptrs[2], pbf.data_ptr(), grad.data_ptr(), 0, n,
                                         step_no[0], 1e-4, 0.9, 0.999, 1e-8, 0.01, 1.0, status.data_ptr(),
                                         stream.cuda_stream)
            assert rc == 0

        def page(to_device):
            for ptr in ptrs:
                q.qlora_paged_prefetch(ptr, 4 * n, to_device=to_device, stream=stream)

        res = {}
        page(True)
        torch.cuda.synchronize()
        for _ in range(3):
            step()
        res["resident_us"] = statistics.median(time_events(step, 10, flush=lambda: l2buf.add_(1))) * 1e3
        res["paged_out_fault_in_us"] = statistics.median(
            time_events(step, 5, flush=lambda: (page(False), torch.cuda.synchronize()))) * 1e3
        res["paged_out_prefetch_back_us"] = statistics.median(
            time_events(lambda: (page(True), step()), 5, flush=lambda: (page(False), torch.cuda.synchronize()))) * 1e3
        torch.cuda.synchronize()
        assert status.item() == 0, f"device status {status.item()}"
    finally:
        torch.cuda.synchronize()
        for ptr in ptrs:
            q.qlora_paged_free(ptr)
    return {"unit": "us per step", "params": n, **{k: round(v, 2) for k, v in res.items()},
            "resident_gbs": round(30 * n / (res["resident_us"] * 1e-6) / 1e9, 1),
            "resident_frac_of_hbm": round(30 * n / (res["resident_us"] * 1e-6) / 1e9 / hbm, 4),
            "state": "fp32 master, m, v in CUDA managed memory (qlora_paged_alloc); grad and bf16 copy in device memory"}


def sub_measurements(q, dev, peaks, l2buf, layer, quant_ms, quant_bytes, n_params):
    hbm = float(peaks["hbm_gbs"])
    out = {}
    # quantiser (timed once at setup, 7 projections, bf16 in)
    qgbs = quant_bytes / (quant_ms * 1e-3) / 1e9
    out["quantize"] = {"value": round(qgbs, 1), "unit": "GB/s", "params": n_params,
                       "ms": round(quant_ms, 4), "frac_of_hbm": round(qgbs / hbm, 4),
                       "bytes_per_param": round(quant_bytes / n_params, 4)}
    # standalone dequantiser on the gate projection (11008 x 4096)
    p = layer.proj[4]
    Wout = torch.empty((p["N"], p["K"]), dtype=torch.bfloat16, device=dev)
    f = lambda: q.qlora_dequantize(p["Wq"], out=Wout)
    for _ in range(3):
        f()
    ms = time_events(f, 10, flush=lambda: l2buf.add_(1))
    dbytes = p["Wq"].nbytes() + Wout.numel() * 2
    dgbs = dbytes / (statistics.median(ms) * 1e-3) / 1e9
    out["dequantize"] = {"value": round(dgbs, 1), "unit": "GB/s", "shape": [p["N"], p["K"]],
                         "frac_of_hbm": round(dgbs / hbm, 4)}
    del Wout
    # adapter merge on the gate projection: NF4(W^ + s B A) through an fp32
    # buffer; bytes moved per weight: NF4 read 0.516 + fp32 write 4 + fp32
    # read 4 + NF4 write 0.516
    Wm = torch.empty((p["N"], p["K"]), dtype=torch.float32, device=dev)
    Wnew = q.empty_nf4(p["N"], p["K"], dev)
    f = lambda: q.qlora_merge_nf4(p["Wq"], p["A"], p["B"], layer.wl.alpha, out=Wnew, W_merged=Wm,
                                  d_status=layer.status)
    for _ in range(3):
        f()
    ms = statistics.median(time_events(f, 10, flush=lambda: l2buf.add_(1)))
    mbytes = 2 * p["Wq"].nbytes() + 8 * p["N"] * p["K"]
    out["merge"] = {"value": round(mbytes / (ms * 1e-3) / 1e9, 1), "unit": "GB/s", "shape": [p["N"], p["K"]],
                    "us": round(ms * 1e3, 2), "frac_of_hbm": round(mbytes / (ms * 1e-3) / 1e9 / hbm, 4)}
    assert layer.status.item() == 0, f"device status {layer.status.item()}"
    # the same merge in one pass, merged weights formed in registers (no fp32
    # buffer): bytes per weight NF4 read 0.516 + NF4 write 0.516, plus A and
    # B once; its 2 r fp32 operations per weight for the product B A bound it
    # by arithmetic before bandwidth
    f1 = lambda: q.qlora_merge_nf4(p["Wq"], p["A"], p["B"], layer.wl.alpha, out=Wnew, keep_merged=False,
                                   d_status=layer.status)
    for _ in range(3):
        f1()
    ms1 = statistics.median(time_events(f1, 10, flush=lambda: l2buf.add_(1)))
    fbytes = 2 * p["Wq"].nbytes() + 2 * (p["A"].numel() + p["B"].numel())
    out["merge_fused"] = {"value": round(fbytes / (ms1 * 1e-3) / 1e9, 1), "unit": "GB/s",
                          "shape": [p["N"], p["K"]], "us": round(ms1 * 1e3, 2),
                          "frac_of_hbm": round(fbytes / (ms1 * 1e-3) / 1e9 / hbm, 4),
                          "fp32_ops_per_s": round(4 * p["A"].shape[0] * p["N"] * p["K"] / (ms1 * 1e-3), 1),
                          "time_vs_two_pass": round(ms1 / ms, 4)}
    assert layer.status.item() == 0, f"device status {layer.status.item()}"
    del Wm, Wnew
    # plain LoRA on a bf16 base (the weights' dequantised copies) through the
    # same GEMM, timed with the same harness as the NF4 step beside it: the
    # pages say QLoRA steps are slower than LoRA's without giving a number
    Wd = [q.qlora_dequantize(p["Wq"]) for p in layer.proj]
    for _ in range(3):
        layer.step_dense(Wd)
    ms_d = statistics.median(time_events(lambda: layer.step_dense(Wd), 10, flush=lambda: l2buf.add_(1)))
    ms_q = statistics.median(time_events(layer.step, 10, flush=lambda: l2buf.add_(1)))
    assert layer.status.item() == 0, f"device status {layer.status.item()}"
    out["lora_bf16_baseline"] = {"value": round(step_flops() / (ms_d * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                                 "ms_per_step": round(ms_d, 4), "qlora_ms_per_step": round(ms_q, 4),
                                 "qlora_over_lora_time": round(ms_q / ms_d, 4),
                                 "weights": "bf16 copies of the layer's NF4 weights (dequantised)"}
    del Wd
    torch.cuda.empty_cache()
    # adapter optimiser step (Adam, fp32 master + moments, bf16 copy) over
    # the adapters of the 32-layer 7B stack: 30 bytes moved per parameter
    # (read grad, master, m, v; write master, m, v, bf16 copy)
    wl4 = inputs.STACK7B
    n_ad = wl4.layers * sum(wl4.r * (N + K) for _, N, K in wl4.shapes)
    g = torch.Generator(device=dev).manual_seed(4)
    master = torch.randn(n_ad, generator=g, device=dev) * 0.01
    mom1 = torch.zeros(n_ad, device=dev)
    mom2 = torch.zeros(n_ad, device=dev)
    grad = torch.randn(n_ad, generator=g, device=dev) * 1e-3
    pbf = torch.empty(n_ad, dtype=torch.bfloat16, device=dev)
    step_no = [0]

    def adam():
        step_no[0] += 1
        q.qlora_adam_step(master, mom1, mom2, grad, step_no[0], 1e-4, weight_decay=0.01, param=pbf,
                          d_status=layer.status)
    for _ in range(3):
        adam()
    ms = statistics.median(time_events(adam, 10, flush=lambda: l2buf.add_(1)))
    agbs = 30 * n_ad / (ms * 1e-3) / 1e9
    out["adam_step"] = {"value": round(agbs, 1), "unit": "GB/s", "params": n_ad, "bytes_per_param": 30,
                        "us": round(ms * 1e3, 2), "frac_of_hbm": round(agbs / hbm, 4),
                        "workload": "Adam over the adapters of the 32-layer 7B stack (r = 16)"}
    assert layer.status.item() == 0, f"device status {layer.status.item()}"
    out["adam_step_paged"] = paged_adam(q, master, mom1, mom2, grad, pbf, layer.status, l2buf, hbm)
    del master, mom1, mom2, grad, pbf
    torch.cuda.empty_cache()
    # decode-shaped forward: 70B MLP weights, M in {1, 4, 16}
    wl = inputs.DECODE
    dec = {}
    mats = []
    for i, (name, N, K) in enumerate(wl.shapes):
        seed = inputs.matrix_seed(wl.base_seed, 0, i)
        W = inputs.weight((N, K), wl.w_std, seed, device=dev, outlier_frac=wl.outlier_frac,
                          outlier_scale=wl.outlier_scale)
        Wq = q.qlora_quantize_nf4(W)
        del W
        A = inputs.normal((wl.r, K), 0.01, seed * 16 + 3, dev)
        B = inputs.normal((N, wl.r), 0.01, seed * 16 + 4, dev)
        mats.append((name, N, K, Wq, A, B))
    torch.cuda.empty_cache()
    for M in inputs.DECODE_M:
        res = []
        for name, N, K, Wq, A, B in mats:
            X = inputs.normal((M, K), 1.0, 99 + M, dev)
            Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            ws = torch.empty(q.qlora_workspace_bytes(M, N, K, wl.r), dtype=torch.uint8, device=dev)
            kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(10)]
            it = iter(kev * 2)
            fn = lambda: q.qlora_linear_fwd(X, Wq, A, B, wl.alpha, Y=Y, workspace=ws, gemm_events=next(it))
            for _ in range(3):
                fn()
            it = iter(kev)
            # the flush is followed by a device-side spin so that the call's
            # launches are queued before its start event: the whole-call time
            # is GPU time, not host launch gaps
            ms = statistics.median(time_events(fn, 10, flush=lambda: (l2buf.add_(1), torch.cuda._sleep(400_000))))
            kms = statistics.median(a.elapsed_time(b) for a, b in kev)
            wbytes = Wq.nbytes()
            res.append({"matrix": [N, K], "us": round(ms * 1e3, 2),
                        "weight_gbs": round(wbytes / (ms * 1e-3) / 1e9, 1),
                        "kernel_us": round(kms * 1e3, 2),
                        "kernel_weight_gbs": round(wbytes / (kms * 1e-3) / 1e9, 1)})
        gbs = [r_["weight_gbs"] for r_ in res]
        kgbs = [r_["kernel_weight_gbs"] for r_ in res]
        dec[f"M{M}"] = {"per_matrix": res, "weight_gbs": round(sum(gbs) / len(gbs), 1),
                        "frac_of_hbm": round(sum(gbs) / len(gbs) / hbm, 4),
                        "kernel_weight_gbs": round(sum(kgbs) / len(kgbs), 1),
                        "kernel_frac_of_hbm": round(sum(kgbs) / len(kgbs) / hbm, 4)}
    out["decode_gemv"] = {"unit": "GB/s of NF4 weight (121.17 MB per matrix)", **dec,
                          "peak_hbm_gbs": hbm}
    # a token's pass through one 70B layer's MLP: gate, up and down decoded
    # back to back with no flush -- each matrix was last read two 121 MB
    # matrices earlier, more than L2 holds (L2 defeated by rotating the
    # weights instead of a flush), and each call's launch overlaps the one
    # before it as in a model's decode
    name, N, K = wl.shapes[0]
    seed = inputs.matrix_seed(wl.base_seed, 0, 2)
    Wu = inputs.weight((N, K), wl.w_std, seed, device=dev, outlier_frac=wl.outlier_frac,
                       outlier_scale=wl.outlier_scale)
    up = ("up", N, K, q.qlora_quantize_nf4(Wu), inputs.normal((wl.r, K), 0.01, seed * 16 + 3, dev),
          inputs.normal((N, wl.r), 0.01, seed * 16 + 4, dev))
    del Wu
    seq = [mats[0], up, mats[1]]
    seq_bytes = sum(m[3].nbytes() for m in seq)
    mlp = {}
    for M in inputs.DECODE_M:
        calls = []
        for name, N, K, Wq, A, B in seq:
            X = inputs.normal((M, K), 1.0, 99 + M, dev)
            Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            ws = torch.empty(q.qlora_workspace_bytes(M, N, K, wl.r), dtype=torch.uint8, device=dev)
            calls.append((X, Wq, A, B, Y, ws))

        def token_pass():
            for X, Wq, A, B, Y, ws in calls:
                q.qlora_linear_fwd(X, Wq, A, B, wl.alpha, Y=Y, workspace=ws)
        for _ in range(3):
            token_pass()
        reps = 10
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        torch.cuda._sleep(1_000_000)   # the passes are queued before the start event is reached
        e0.record()
        for _ in range(reps):
            token_pass()
        e1.record()
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / reps
        gbs = seq_bytes / (us * 1e-6) / 1e9
        mlp[f"M{M}"] = {"us_per_pass": round(us, 2), "weight_gbs": round(gbs, 1), "frac_of_hbm": round(gbs / hbm, 4)}
        del calls
    out["decode_mlp_pass"] = {"unit": "GB/s of NF4 weight over gate, up and down (363.5 MB)",
                              "weights": "70B MLP matrices 28672 x 8192 (gate, up) and 8192 x 28672 (down)",
                              "l2": "defeated by rotating the three matrices (no flush)", **mlp}
    del mats, seq, up
    torch.cuda.empty_cache()
    out.update(config_workloads(q, dev, hbm))
    return out


# ------------------------------------------------------------ CPU oracle
def _oracle_sample(layer_np, tokens):
    """One oracle pass over the sample: dequantise (C) + fwd + bwd (numpy f64)."""
    import oracle as O
    wl = WL
    for p in layer_np:
        Wh = O.nf4_dequantize(p["q"])
        O.linear_fwd(p["X"][:tokens], Wh, p["A"], p["B"], wl.alpha, wl.r)
        O.linear_bwd(p["dY"][:tokens], p["X"][:tokens], Wh, p["A"], p["B"], wl.alpha, wl.r)


def _layer_to_host(layer, tokens):
    import numpy as np
    bits = lambda t: t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    out = []
    for p in layer.proj:
        Wq = p["Wq"]
        out.append({"q": {"codes": Wq.codes.cpu().numpy(), "q8": Wq.absmax_q8.cpu().numpy(),
                          "s2": Wq.group_scale.cpu().numpy(), "absmax": None, "rows": p["N"],
                          "cols": p["K"], "double_quant": True},
                    "X": bits(p["X"][:tokens]), "dY": bits(p["dY"][:tokens]),
                    "A": bits(p["A"]), "B": bits(p["B"])})
    return out


def _cores_used():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_legs(dev):
    """The oracle's other legs, as it stands, each on a bounded sample:
    - codec: one-shot quantise and dequantise of the LLaMA-7B layer's seven
      weights in full (202M weights; one layer of the 32-layer stack has the
      same shapes, so this is also that stack's per-layer quantise);
    - decode forward of both 70B MLP matrices in full at 16 tokens
      (dequantise + binary64 forward), in GB/s of NF4 weight like the GPU's;
    - the 65B model's per-layer quantise, measured on its gate projection
      (22016 x 8192) and extrapolated to the layer's 809.5M weights (stated).
    Weights are drawn on the GPU with the bench's seeds and copied to the host."""
    import numpy as np
    import oracle as O
    import bit_nf4_quantized_21_b200 as q
    legs = {}
    # codec, LLaMA-7B layer in full
    tq = td = 0.0
    n = 0
    for i, (name, N, K) in enumerate(WL.shapes):
        W = inputs.weight((N, K), WL.w_std, inputs.matrix_seed(WL.base_seed, 0, i), device=dev)
        Wh = W.float().cpu().numpy()
        del W
        t0 = time.perf_counter()
        qd = O.nf4_quantize(Wh)
        t1 = time.perf_counter()
        O.nf4_dequantize(qd)
        t2 = time.perf_counter()
        tq += t1 - t0
        td += t2 - t1
        n += N * K
        del Wh, qd
    legs["codec_llama7b_layer"] = {
        "weights": n, "quantize_s": round(tq, 3), "dequantize_s": round(td, 3),
        "quantize_elems_per_s": round(n / tq, 1), "dequantize_elems_per_s": round(n / td, 1),
        "stack7b_per_layer_quantize_s": round(tq, 3),
        "sample": "the seven projections in full (bf16 source, NF4 double quant), C oracle, one thread"}
    # decode forward of the 70B MLP matrices in full, 16 tokens
    wl = inputs.DECODE
    tot_s = 0.0
    wbytes = 0
    for i, (name, N, K) in enumerate(wl.shapes):
        seed = inputs.matrix_seed(wl.base_seed, 0, i)
        W = inputs.weight((N, K), wl.w_std, seed, device=dev, outlier_frac=wl.outlier_frac,
                          outlier_scale=wl.outlier_scale)
        Wq = q.qlora_quantize_nf4(W)
        del W
        qd = {"codes": Wq.codes.cpu().numpy(), "q8": Wq.absmax_q8.cpu().numpy(),
              "s2": Wq.group_scale.cpu().numpy(), "absmax": None, "rows": N, "cols": K, "double_quant": True}
        wbytes += Wq.nbytes()
        del Wq
        bits = lambda t: t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
        X = bits(inputs.normal((16, K), 1.0, 99 + 16, dev))
        A = bits(inputs.normal((wl.r, K), 0.01, seed * 16 + 3, dev))
        B = bits(inputs.normal((N, wl.r), 0.01, seed * 16 + 4, dev))
        t0 = time.perf_counter()
        O.linear_fwd(X, O.nf4_dequantize(qd), A, B, wl.alpha, wl.r)
        tot_s += time.perf_counter() - t0
        del qd
    legs["decode_70b_mlp_m16"] = {
        "value": round(wbytes / tot_s / 1e9, 4), "unit": "GB/s of NF4 weight", "s": round(tot_s, 3),
        "sample": "both 70B MLP matrices in full at M = 16: C dequantise + binary64 numpy forward"}
    # 65B per-layer quantise, from its gate projection
    wl = inputs.LLAMA65B
    name, N, K = wl.shapes[4]
    W = inputs.weight((N, K), wl.w_std, inputs.matrix_seed(wl.base_seed, 0, 4), device=dev)
    Wh = W.float().cpu().numpy()
    del W
    t0 = time.perf_counter()
    O.nf4_quantize(Wh)
    dt = time.perf_counter() - t0
    layer_w = sum(N_ * K_ for _, N_, K_ in wl.shapes)
    legs["llama65b_per_layer_quantize"] = {
        "measured_weights": N * K, "measured_s": round(dt, 3), "elems_per_s": round(N * K / dt, 1),
        "layer_weights": layer_w, "layer_s_extrapolated": round(layer_w / (N * K / dt), 2),
        "sample": "gate projection 22016 x 8192 measured; the 7-projection layer extrapolated from its rate"}
    del Wh
    torch.cuda.empty_cache()
    return legs


def cpu_baseline(layer, tokens, dev=None, legs=True):
    host = _layer_to_host(layer, tokens)
    t0 = time.perf_counter()
    _oracle_sample(host, tokens)
    dt = time.perf_counter() - t0
    flops = step_flops(M=tokens)
    out = {"value": round(flops / dt / 1e12, 5), "unit": "TFLOP/s", "cores": _cores_used(),
           "kind": "oracle",
           "sample": f"one step of the same 7 projections on {tokens} of the {WL.M} tokens: "
                     f"C dequantise + binary64 numpy fwd/bwd, {dt:.2f} s"}
    if legs and dev is not None:
        out["legs"] = cpu_legs(dev)
        out["legs_cores"] = "C legs: 1 thread; numpy products: the BLAS threads in cores"
    return out


def run_reference(args):
    """CPU oracle arm: rank 0 only; other ranks exit without work."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np
    import oracle as O
    tokens = args.cpu_tokens
    # the same inputs, drawn on the CPU, quantised by the oracle itself
    host = []
    for i, (name, N, K) in enumerate(WL.shapes):
        seed = inputs.matrix_seed(WL.base_seed, 0, i)
        W = inputs.weight((N, K), WL.w_std, seed, dtype=torch.bfloat16)
        bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
        host.append({"q": O.nf4_quantize(W.float().numpy()),
                     "X": bits(inputs.normal((tokens, K), 1.0, seed * 16 + 1)),
                     "dY": bits(inputs.normal((tokens, N), 1.0, seed * 16 + 2)),
                     "A": bits(inputs.normal((WL.r, K), 0.01, seed * 16 + 3)),
                     "B": bits(inputs.normal((N, WL.r), 0.01, seed * 16 + 4))})
        del W
    for _ in range(args.warmup):
        _oracle_sample(host, tokens)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_sample(host, tokens)
    dt = time.perf_counter() - t0
    value = step_flops(M=tokens) * args.steps / dt / 1e12
    cores = _cores_used()
    sample = (f"each step: the 7 projections on {tokens} of the {WL.M} tokens "
              f"(C dequantise + binary64 numpy fwd/bwd)")
    line = {"metric": METRIC, "value": round(value, 5), "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": "llama7b-layer-7proj-fwd+bwd", "tokens_per_step": tokens,
                       "lora_r": WL.r, "lora_alpha": WL.alpha},
            "cpu_baseline": {"value": round(value, 5), "unit": "TFLOP/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 5), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_only(args):
    """One projection's forward or backward call, repeated: the small case
    for kernel profiles (ncu) of the fused GEMM; with --only decode, the
    decode-shaped forward of one 70B MLP matrix (--proj 0: 28672 x 8192,
    1: 8192 x 28672) at --tokens <= 16; with --only quantize, the quantiser
    over the seven LLaMA-7B projections (bf16), --steps repetitions."""
    import bit_nf4_quantized_21_b200 as q
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if args.only == "quantize":
        Ws, outs = [], []
        for i, (name, N, K) in enumerate(WL.shapes):
            Ws.append(inputs.weight((N, K), WL.w_std, inputs.matrix_seed(WL.base_seed, 0, i), device=dev))
            outs.append(q.empty_nf4(N, K, dev))
        l2 = torch.empty(L2_BYTES // 2, dtype=torch.float32, device=dev)
        params = sum(w.numel() for w in Ws)
        res = []
        for rep in range(args.steps):
            l2.add_(1)
            torch.cuda._sleep(2_000_000)
            evs = []
            for W, o in zip(Ws, outs):
                e = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                e[0].record()
                q.qlora_quantize_nf4(W, out=o)
                e[1].record()
                evs.append(e)
            torch.cuda.synchronize()
            if rep >= 1:
                res.append(sum(a.elapsed_time(b) for a, b in evs))
        ms = statistics.median(res)
        print(json.dumps({"only": "quantize", "params": params, "ms": round(ms, 4),
                          "GBps": round(params * 2.516 / (ms * 1e-3) / 1e9, 1)}), flush=True)
        return
    if args.only == "decode":
        wl = inputs.DECODE
        name, N, K = wl.shapes[args.proj]
        M = args.tokens
        seed = inputs.matrix_seed(wl.base_seed, 0, args.proj)
        W = inputs.weight((N, K), wl.w_std, seed, device=dev, outlier_frac=wl.outlier_frac,
                          outlier_scale=wl.outlier_scale)
        Wq = q.qlora_quantize_nf4(W)
        del W
        X = inputs.normal((M, K), 1.0, 99 + M, dev)
        A = inputs.normal((wl.r, K), 0.01, seed * 16 + 3, dev)
        B = inputs.normal((N, wl.r), 0.01, seed * 16 + 4, dev)
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(q.qlora_workspace_bytes(M, N, K, wl.r), dtype=torch.uint8, device=dev)
        l2 = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)
        evs = []
        for i in range(args.warmup + args.steps):
            l2.add_(1)
            ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            q.qlora_linear_fwd(X, Wq, A, B, wl.alpha, Y=Y, workspace=ws, gemm_events=ev)
            if i >= args.warmup:
                evs.append(ev)
        torch.cuda.synchronize()
        us = statistics.median(a.elapsed_time(b) for a, b in evs) * 1e3
        print(json.dumps({"only": "decode", "shape": [M, N, K], "kernel_us": round(us, 2),
                          "weight_gbs": round(Wq.nbytes() / (us * 1e-6) / 1e9, 1)}))
        return
    name, N, K = WL.shapes[args.proj]
    M = args.tokens
    seed = inputs.matrix_seed(WL.base_seed, 0, args.proj)
    Wq = q.qlora_quantize_nf4(inputs.weight((N, K), WL.w_std, seed, device=dev))
    X = inputs.normal((M, K), 1.0, seed * 16 + 1, dev)
    dY = inputs.normal((M, N), 1.0, seed * 16 + 2, dev)
    A = inputs.normal((WL.r, K), 0.01, seed * 16 + 3, dev)
    B = inputs.normal((N, WL.r), 0.01, seed * 16 + 4, dev)
    T = torch.empty((M, WL.r), dtype=torch.float32, device=dev)
    ws = torch.empty(q.qlora_workspace_bytes(M, N, K, WL.r), dtype=torch.uint8, device=dev)
    q.qlora_linear_fwd(X, Wq, A, B, WL.alpha, T_save=T, workspace=ws)
    evs = []
    for i in range(args.warmup + args.steps):
        ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
        if args.only == "gemm-fwd":
            q.qlora_linear_fwd(X, Wq, A, B, WL.alpha, T_save=T, workspace=ws, gemm_events=ev)
        else:
            q.qlora_linear_bwd(dY, X, Wq, A, B, WL.alpha, T_saved=T, workspace=ws, gemm_events=ev)
        if i >= args.warmup:
            evs.append(ev)
    torch.cuda.synchronize()
    ms = [a.elapsed_time(b) for a, b in evs]
    contraction, outc = (K, N) if args.only == "gemm-fwd" else (N, K)
    flops = 2 * M * N * K + 2 * M * WL.r * outc
    print(json.dumps({"only": args.only, "shape": [M, N, K], "gemm_us": round(statistics.median(ms) * 1e3, 2),
                      "gemm_tflops": round(flops / (statistics.median(ms) * 1e-3) / 1e12, 1)}))


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--cpu-tokens", type=int, default=64)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-sub", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--sequential", action="store_true",
                    help="run the step's projections one after another (default: q/k/v and gate/up overlap)")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch the timed steps call by call instead of replaying a CUDA graph per step")
    ap.add_argument("--no-cpu-legs", action="store_true",
                    help="time only the oracle's layer-step sample, not its codec / decode / quantise legs")
    ap.add_argument("--clock-log", default=None,
                    help="directory for the raw nvidia-smi clock samples (default: the temporary directory)")
    ap.add_argument("--only", choices=("gemm-fwd", "gemm-dx", "decode", "quantize"), default=None,
                    help="profile mode: repeat one projection's call (see --proj, --tokens)")
    ap.add_argument("--proj", type=int, default=4)
    ap.add_argument("--tokens", type=int, default=2048)
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)   # timing rule: at least 3 warm-up steps
    if args.only:
        run_only(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
