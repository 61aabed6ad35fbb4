"""Benchmark of the quantize-once convolution hot path on B200.

One step = one pass of the whole path for one conv layer: quantize X and W
(round-to-nearest-even) and G_Y (Philox stochastic rounding) into square-block
NVFP4/NVFP6 form, then the implicit-GEMM forward, weight-gradient and
input-gradient passes.  `value` is conv TFLOP/s (fwd + wgrad + dgrad FLOPs of
all ranks / device time of the timed steps, max over ranks).  On one GPU the
step is one CUDA graph replay: G_Y's quantization beside X's and W's, the
forward pass after X and W, the two gradient passes after all three, each
pass on its own stream.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the CPU oracle, bounded sample

Under torchrun (N > 1) each rank runs its own batch of the same layer (weak
scaling, data parallel): the per-tensor max|x| of X and G_Y is MAX-all-reduced
before quantizing (so every rank uses the global tensor scale) and G_W is
SUM-all-reduced after the weight-gradient pass, both over NCCL.  With
MQV_DIST_BACKEND=gloo and more ranks than GPUs, ranks share the visible GPUs
(a functional check of this path; its timing is not a measurement).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "quantize GB/s and conv fwd+wgrad+dgrad TFLOP/s at 1 B200, as fraction of roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def pick_layer(name: str) -> workloads.Layer:
    table = {l.name: l for l in [workloads.tiny_layer(), workloads.resnet18_layer2()]
             + workloads.resnet18_body() + workloads.yolov8n_mix()}
    if name not in table:
        raise SystemExit(f"unknown workload {name}; choose from {sorted(table)}")
    return table[name]


def layer_bytes(layer: workloads.Layer):
    """Algorithmic bytes: quantize = 2 fp32 reads + codes + scales written;
    conv pass = both quantized operands read once + fp32 output written once."""
    eb = 0.5 if layer.fmt == "nvfp4" else 0.75
    qb = eb + 1.0 / 16
    x = layer.H * layer.W * layer.Cin * layer.N
    w = layer.Cout * layer.K * layer.K * layer.Cin
    g = layer.Ho * layer.Wo * layer.Cout * layer.N
    quant = {"x": x * (8 + qb), "w": w * (8 + qb), "g": g * (8 + qb)}
    conv = {"fwd": (w + x) * qb + g * 4, "wgrad": (g + x) * qb + w * 4, "dgrad": (w + g) * qb + x * 4}
    return quant, conv, (x, w, g)


class Clocks:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [t.strip() for t in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- GPU arm

def run_gpu(args):
    import torch
    import torch.distributed as dist

    import microscaling_quantized_convolution_b200 as mqv
    from microscaling_quantized_convolution_b200 import dp, naive

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    # one process per GPU; ranks beyond the visible GPUs (a functional check
    # of the multi-rank path on fewer GPUs, host collectives only) share them
    torch.cuda.set_device(local % torch.cuda.device_count())
    if world > 1:
        from datetime import timedelta
        dist.init_process_group(os.environ.get("MQV_DIST_BACKEND", "nccl"), timeout=timedelta(seconds=120))
    mqv.lib()

    layer = pick_layer(args.workload)
    fmt = layer.fmt
    d = mqv.conv_desc(**layer.dims(), fmt=fmt)
    Ho, Wo = layer.Ho, layer.Wo
    xr, xc = layer.H * layer.W * layer.Cin, layer.N
    wr, wc = layer.Cout, layer.K * layer.K * layer.Cin
    gr, gc = Ho * Wo * layer.Cout, layer.N
    dev = torch.device("cuda", local % torch.cuda.device_count())

    # Inputs resident in HBM, rotated over enough sets to exceed the 126 MB L2
    quant_b, conv_b, (nx, nw, ng) = layer_bytes(layer)
    per_set = 4 * (nx + nw + ng) + 4 * (nx + nw + ng)        # fp32 inputs + outputs
    nsets = max(2, min(16, -(-400_000_000 // per_set)))
    sets = []
    for i in range(nsets):
        g = torch.Generator(device=dev)
        g.manual_seed(1000 * rank + i)
        X = torch.randn((layer.H, layer.W, layer.Cin, layer.N), generator=g, device=dev)
        X = torch.relu(X) if layer.x_dist == "relu" else (torch.nn.functional.silu(X) if layer.x_dist == "silu" else X)
        Wt = torch.randn((layer.Cout, layer.K, layer.K, layer.Cin), generator=g, device=dev) * (2.0 / wc) ** 0.5
        G = torch.randn((Ho, Wo, layer.Cout, layer.N), generator=g, device=dev) * layer.gy_std
        sets.append(dict(X=X.view(-1), W=Wt.view(-1), G=G.view(-1),
                         qx=mqv.QTensor.empty(xr, xc, fmt, dev), qw=mqv.QTensor.empty(wr, wc, fmt, dev),
                         qg=mqv.QTensor.empty(gr, gc, fmt, dev),
                         y=torch.empty(Ho * Wo * layer.Cout * layer.N, device=dev),
                         gw=torch.empty(wr * wc, device=dev),
                         gx=torch.empty(xr * xc, device=dev)))
    ws_q = [torch.empty(mqv.quantize_workspace_bytes(r, c), dtype=torch.uint8, device=dev)
            for r, c in ((xr, xc), (wr, wc), (gr, gc))]
    ws_w = mqv.conv_workspace_bytes(d, mqv.OP_WGRAD)
    ws_wgrad = torch.empty(max(ws_w, 16), dtype=torch.uint8, device=dev)
    ws_fwd = torch.empty(max(mqv.conv_workspace_bytes(d, mqv.OP_FWD), 16), dtype=torch.uint8, device=dev)
    ws_dgrad = torch.empty(max(mqv.conv_workspace_bytes(d, mqv.OP_DGRAD), 16), dtype=torch.uint8, device=dev)
    amax_buf = torch.empty(3, dtype=torch.float32, device=dev)
    seed = workloads.sr_seed(layer)
    splits_reduce = 1 if ws_w > 0 else 0

    ws_many = torch.empty(mqv.quantize_many_workspace_bytes(
        [(None, xr, xc, fmt, mqv.RNE, 0), (None, wr, wc, fmt, mqv.RNE, 0), (None, gr, gc, fmt, mqv.SR, 0)]),
        dtype=torch.uint8, device=dev)

    def quantize_all(s, step):
        # X and W round to nearest, G_Y stochastically; one amax pass, one quantize pass
        mqv.quantize_many([(s["X"], xr, xc, fmt, mqv.RNE, 0, s["qx"]),
                           (s["W"], wr, wc, fmt, mqv.RNE, 0, s["qw"]),
                           (s["G"], gr, gc, fmt, mqv.SR, seed + step, s["qg"])], ws=ws_many)

    # the same quantization as two independent calls (X and W for fwd, G_Y
    # for the gradients), each with its own workspace, for the concurrent step
    ws_xw = torch.empty(mqv.quantize_many_workspace_bytes(
        [(None, xr, xc, fmt, mqv.RNE, 0), (None, wr, wc, fmt, mqv.RNE, 0)]), dtype=torch.uint8, device=dev)
    ws_g = torch.empty(mqv.quantize_many_workspace_bytes([(None, gr, gc, fmt, mqv.SR, 0)]),
                       dtype=torch.uint8, device=dev)

    def quantize_xw(s):
        mqv.quantize_many([(s["X"], xr, xc, fmt, mqv.RNE, 0, s["qx"]),
                           (s["W"], wr, wc, fmt, mqv.RNE, 0, s["qw"])], ws=ws_xw)

    def quantize_g(s, step):
        mqv.quantize_many([(s["G"], gr, gc, fmt, mqv.SR, seed + step, s["qg"])], ws=ws_g)

    def fwd(s):
        mqv.conv_fwd(d, s["qw"], s["qx"], y=s["y"], ws=ws_fwd)

    def wgrad(s):
        mqv.conv_wgrad(d, s["qg"], s["qx"], gw=s["gw"], ws=ws_wgrad)

    def dgrad(s):
        mqv.conv_dgrad(d, s["qw"], s["qg"], gx=s["gx"], ws=ws_dgrad)

    class ShardOps:
        """The kernels of the data-parallel step (dp.data_parallel_step, the
        one implementation of the exchange) on input set k's fixed buffers:
        each call runs its library call, or replays the CUDA graph captured
        from that call."""
        RNE, SR = mqv.RNE, mqv.SR

        def __init__(self, k, graphs=None, capture_into=None):
            self.k, self.s, self.g, self.cap = k, sets[k], graphs, capture_into

        def _run(self, name, fn):
            if self.cap is not None:
                self.cap[name] = capture(fn)
            elif self.g is not None:
                self.g[name].replay()
            else:
                fn()

        def amax(self, t, rows, cols):
            x = t is self.s["X"]
            out = amax_buf[0:1] if x else amax_buf[2:3]
            self._run("amax_x" if x else "amax_g", lambda: mqv.amax(t, rows, cols, out=out, ws=ws_q[0 if x else 2]))
            return out

        def quantize_with_amax(self, t, rows, cols, f, rnd, sd, a, c0, tc):
            x = t is self.s["X"]
            q = self.s["qx"] if x else self.s["qg"]
            self._run("quant_x" if x else "quant_g",
                      lambda: mqv.quantize_with_amax(t, rows, cols, f, rnd, sd, a, out=q, sr_col0=c0, sr_cols=tc))
            return q

        def quantize(self, t, rows, cols, f, rnd, sd):
            self._run("quant_w", lambda: mqv.quantize(t, rows, cols, f, rnd, sd, out=self.s["qw"], ws=ws_q[1]))
            return self.s["qw"]

        def fwd(self, dims, qw, qx):
            self._run("fwd", lambda: fwd(self.s))
            return self.s["y"]

        def wgrad(self, dims, qg, qx):
            self._run("wgrad", lambda: wgrad(self.s))
            return self.s["gw"]

        def dgrad(self, dims, qw, qg):
            self._run("dgrad", lambda: dgrad(self.s))
            return self.s["gx"]

    comm = dp.torch_comm() if world > 1 else None

    def dp_step(k, ops, mark=None):
        # this rank's batch is columns [rank·N, (rank+1)·N) of the global batch
        s = sets[k]
        dp.data_parallel_step(ops, comm, s["X"], s["W"], s["G"], layer.dims(), fmt, world * layer.N, rank, world,
                              seed + k, mark=mark)

    def step(i, s=None):
        k = i % nsets if s is None else next(j for j in range(nsets) if sets[j] is s)
        if world > 1:
            dp_step(k, ShardOps(k))
            return
        s = sets[k]
        quantize_all(s, i)
        fwd(s)
        wgrad(s)
        dgrad(s)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    flags = mqv.device_errors()
    if flags:
        raise SystemExit(f"device wait timeout flags {flags:#x}")

    # One CUDA graph per phase and input set, captured through the same ABI
    # calls; the timed loop replays them (collectives stay eager).
    def capture(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        return g

    graphs = []
    for k in range(nsets):
        s = sets[k]
        gk = {"fwd": capture(lambda: fwd(s)), "wgrad": capture(lambda: wgrad(s)),
              "dgrad": capture(lambda: dgrad(s))}
        if world == 1:
            gk["quant"] = capture(lambda: quantize_all(s, k))
            gk["quant_xw"] = capture(lambda: quantize_xw(s))
            gk["quant_g"] = capture(lambda: quantize_g(s, k))
        else:
            # every kernel call of the data-parallel step, captured as the
            # step makes it (the collectives between them run eagerly)
            dp_step(k, ShardOps(k, capture_into=gk))
        graphs.append(gk)
    torch.cuda.synchronize()

    # fwd, wgrad and dgrad read only the quantized operands (and write
    # separate outputs with separate workspaces), so on one GPU they run on
    # three streams after the quantize phase: the ramp and tail of one
    # persistent kernel overlap the others' work.  Across ranks the gradient
    # all-reduce keeps the passes in one stream.
    concurrent = world == 1 and not args.serial
    cur = torch.cuda.current_stream()
    pstreams = {ph: torch.cuda.Stream() for ph in ("fwd", "wgrad", "dgrad")}
    gstream = torch.cuda.Stream()

    def graph_step(i, ev, conc):
        k = i % nsets
        gk, s = graphs[k], sets[k]
        ev[0].record()
        if conc:
            # G_Y's quantization runs beside X's and W's; fwd starts once X and
            # W are done, the gradients once G_Y is too
            gstream.wait_event(ev[0])
            with torch.cuda.stream(gstream):
                gk["quant_g"].replay()
                ev[8].record(gstream)
            gk["quant_xw"].replay()
            ev[1].record()
            for j, ph in enumerate(("fwd", "wgrad", "dgrad")):
                st = pstreams[ph]
                st.wait_event(ev[1])
                if ph != "fwd":
                    st.wait_event(ev[8])
                with torch.cuda.stream(st):
                    ev[2 + 2 * j].record(st)
                    gk[ph].replay()
                    ev[3 + 2 * j].record(st)
            for j in range(3):
                cur.wait_event(ev[3 + 2 * j])
            return
        if world > 1:
            # the data-parallel step replaying its captured calls; its phase
            # boundaries record the events the serial step records below
            marks = {"start": (), "quantized": (ev[1], ev[2]), "fwd": (ev[3], ev[4]), "wgrad": (ev[5], ev[6]),
                     "dgrad": (ev[7],)}
            dp_step(k, ShardOps(k, graphs=gk), mark=lambda nm: [e.record() for e in marks[nm]])
            return
        gk["quant"].replay()
        ev[1].record()
        ev[2].record()
        gk["fwd"].replay()
        ev[3].record()
        ev[4].record()
        gk["wgrad"].replay()
        ev[5].record()
        ev[6].record()
        gk["dgrad"].replay()
        ev[7].record()

    # The concurrent step as one CUDA graph per input set: the fork to the G_Y
    # stream and the three pass streams and the joins are captured as graph
    # edges, so the device resolves the dependencies and one replay a step
    # replaces the per-phase launches and cross-stream event waits.
    def whole_step(s, k):
        cap = torch.cuda.current_stream()
        fork = torch.cuda.Event()
        fork.record(cap)
        gstream.wait_event(fork)
        with torch.cuda.stream(gstream):
            quantize_g(s, k)
            g_done = torch.cuda.Event()
            g_done.record(gstream)
        quantize_xw(s)
        xw_done = torch.cuda.Event()
        xw_done.record(cap)
        joins = []
        for ph, fn in (("fwd", fwd), ("wgrad", wgrad), ("dgrad", dgrad)):
            st = pstreams[ph]
            st.wait_event(xw_done)
            if ph != "fwd":
                st.wait_event(g_done)
            with torch.cuda.stream(st):
                fn(s)
                e = torch.cuda.Event()
                e.record(st)
                joins.append(e)
        for e in joins:
            cap.wait_event(e)

    step_graphs = [capture(lambda: whole_step(sets[k], k)) for k in range(nsets)] if concurrent else []
    torch.cuda.synchronize()

    def timed_whole():
        """K steps, one whole-step graph replay each, between synchronizes."""
        for i in range(3):
            step_graphs[i % nsets].replay()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        t0.record()
        for i in range(args.steps):
            step_graphs[i % nsets].replay()
        t1.record()
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    # The serial step on one GPU: one graph per step with the phase
    # boundaries recorded as event nodes inside it (external events), so the
    # per-phase device times carry no graph launch between phases.  Each of
    # the nk graphs keeps its own events: after the timed loop they hold the
    # last nk steps' phase times, which give the per-kernel durations.
    nk = 4 * nsets
    kev, kgraphs = [], []
    if world == 1:
        kev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(5)] for _ in range(nk)]

        def serial_marked(j):
            k = j % nsets
            s, e = sets[k], kev[j]
            e[0].record()
            quantize_all(s, k)
            e[1].record()
            fwd(s)
            e[2].record()
            wgrad(s)
            e[3].record()
            dgrad(s)
            e[4].record()

        kgraphs = [capture(lambda j=j: serial_marked(j)) for j in range(nk)]
        torch.cuda.synchronize()

    def timed_loop(conc):
        """K steps between a barrier + synchronize on both sides; returns the
        whole-loop time and each phase's mean duration (max over ranks)."""
        if world == 1 and not conc:
            for i in range(nk):
                kgraphs[i].replay()
            torch.cuda.synchronize()
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record()
            for i in range(args.steps):
                kgraphs[i % nk].replay()
            t1.record()
            torch.cuda.synchronize()
            names = ("quantize", "fwd", "wgrad", "dgrad")
            parts = {ph: [e[j].elapsed_time(e[j + 1]) for e in kev] for j, ph in enumerate(names)}
            return t0.elapsed_time(t1), {k: sum(v) / len(v) for k, v in parts.items()}
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(9)] for _ in range(args.steps)]
        for i in range(3):
            graph_step(i, evs[0], conc)
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t0.record()
        for i in range(args.steps):
            graph_step(i, evs[i], conc)
        t1.record()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        total = t0.elapsed_time(t1)
        parts = {"quantize": [], "fwd": [], "wgrad": [], "dgrad": []}
        for e in evs:
            parts["quantize"].append(e[0].elapsed_time(e[1]))
            parts["fwd"].append(e[2].elapsed_time(e[3]))
            parts["wgrad"].append(e[4].elapsed_time(e[5]))
            parts["dgrad"].append(e[6].elapsed_time(e[7]))
        mean = {k: sum(v) / len(v) for k, v in parts.items()}
        if world > 1:
            t = torch.tensor([total] + [mean[k] for k in parts], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            total = t[0].item()
            mean = {k: t[1 + j].item() for j, k in enumerate(parts)}
        return total, mean

    # Each kernel alone (one stream): the per-kernel durations and the
    # roofline.  Then the step as it is run: on one GPU the three passes
    # concurrently; that loop gives the reported throughput.
    clocks = Clocks(local % torch.cuda.device_count())
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.15)
    serial_ms, mean = timed_loop(False)
    phase_ms, conc_mean = timed_loop(True) if concurrent else (serial_ms, mean)
    total_ms = timed_whole() if concurrent else serial_ms
    clk = clocks.stop()
    flags = mqv.device_errors()

    # The baseline the method removes (expand with im2col first, quantize each
    # operand once per GEMM direction), timed the same way on one GPU.
    def run_naive(blocks):
        nb = naive.plan(d, dev, blocks)
        nout = {"y": torch.empty_like(sets[0]["y"]), "gw": torch.empty_like(sets[0]["gw"]),
                "gx": torch.empty_like(sets[0]["gx"])}

        def nphase(k, ph):
            sk = sets[k]
            if ph == "quant":
                naive.quantize_all(nb, sk["X"], sk["W"], sk["G"], seed + k)
            elif ph == "fwd":
                naive.fwd(nb, nout["y"])
            elif ph == "wgrad":
                naive.wgrad(nb, nout["gw"])
            else:
                naive.dgrad(nb, nout["gx"])

        nphases = ("quant", "fwd", "wgrad", "dgrad")
        for k in range(nsets):
            for ph in nphases:
                nphase(k, ph)
        torch.cuda.synchronize()
        ngraphs = [{ph: capture(lambda k=k, ph=ph: nphase(k, ph)) for ph in nphases} for k in range(nsets)]
        nev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.naive_steps)]

        def nstep(i, ev):
            g = ngraphs[i % nsets]
            for j, ph in enumerate(nphases):
                ev[j].record()
                g[ph].replay()
            ev[4].record()

        for i in range(3):
            nstep(i, nev[0])
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for i in range(args.naive_steps):
            nstep(i, nev[i])
        b.record()
        torch.cuda.synchronize()
        n_ms = a.elapsed_time(b) / args.naive_steps
        nparts = {ph: sum(e[j].elapsed_time(e[j + 1]) for e in nev) / len(nev) for j, ph in enumerate(nphases)}
        nbytes = naive.layer_bytes(d)
        Ho_, Wo_ = mqv.out_hw(d)
        ex = Ho_ * Wo_ * d.Kh * d.Kw * d.Cin * d.N          # elements of the expanded X
        once_bytes = sum(quant_b.values()) + sum(conv_b.values())
        naive_res = {"ms_per_step": round(n_ms, 4),
                     "phase_ms": {ph: round(v, 4) for ph, v in nparts.items()},
                     "step_time_ratio": None, "quantize_time_ratio": None,
                     "algorithmic_bytes_ratio": round(sum(nbytes.values()) / once_bytes, 3),
                     "quantized_elements_ratio": round((2 * ex + 2 * nw + 2 * ng) / (nx + nw + ng), 3),
                     "expanded_x_ratio": round(ex / nx, 3),
                     "flow": "im2col, every operand quantized once per GEMM direction, 1x1 GEMMs, col2im",
                     "blocks": ("16-element lines along each GEMM's contraction (x' 16x1 and 1x16, w 1x16 "
                                "and 16x1, g_y 1x16 and 16x1)" if blocks == "line" else
                                "4x4 squares over (kh*kw*ci, n) of the expanded tensor")}
        del ngraphs, nb
        torch.cuda.synchronize()
        return naive_res

    naive_res = naive_sq = None
    if world == 1 and args.naive_steps > 0:
        naive_res = run_naive("line")
        naive_sq = run_naive("square")

    # End to end through the public API with pinned host buffers, pipelined
    # as a training loop would be: step i copies its inputs in on one stream,
    # computes on the current stream and copies its outputs back on a third,
    # alternating between two device slots, so the copies of neighbouring
    # steps overlap each other and the compute.
    e2e = None
    if args.e2e_steps > 0:
        hX = sets[0]["X"].cpu().pin_memory(); hW = sets[0]["W"].cpu().pin_memory()
        hG = sets[0]["G"].cpu().pin_memory()
        hout = [{k: torch.empty(sets[0][k].numel()).pin_memory() for k in ("y", "gw", "gx")} for _ in range(2)]
        cur = torch.cuda.current_stream()
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        ev = [{n: torch.cuda.Event() for n in ("in", "comp", "out")} for _ in range(2)]

        def e2e_step(i):
            k = i % 2
            sk = sets[k]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev[k]["comp"])      # slot k's inputs are consumed
                sk["X"].copy_(hX, non_blocking=True); sk["W"].copy_(hW, non_blocking=True)
                sk["G"].copy_(hG, non_blocking=True)
                ev[k]["in"].record(s_in)
            cur.wait_event(ev[k]["in"])
            if i >= 2:
                cur.wait_event(ev[k]["out"])            # slot k's outputs are back on the host
            step(i, sk)
            ev[k]["comp"].record(cur)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev[k]["comp"])
                for n in ("y", "gw", "gx"):
                    hout[k][n].copy_(sk[n], non_blocking=True)
                ev[k]["out"].record(s_out)

        def drain(last):
            for i in range(max(0, last - 1), last + 1):
                cur.wait_event(ev[i % 2]["out"])

        for i in range(4):
            e2e_step(i)
        drain(3)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for i in range(args.e2e_steps):
            e2e_step(i)
        drain(args.e2e_steps - 1)
        b.record()
        torch.cuda.synchronize()
        e2e_ms = a.elapsed_time(b) / args.e2e_steps
        if world > 1:
            t = torch.tensor([e2e_ms], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e2e_ms = t.item()
        h2d = 4 * (nx + nw + ng)
        d2h = 4 * sum(sets[0][n].numel() for n in ("y", "gw", "gx"))
        e2e = {"value": round(3 * layer.flops() * world / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4),
               "pipeline": "inputs in, compute, outputs out on three streams, two device slots"}

        # The link bound of that pipeline: one step's copies alone in each
        # direction and both directions at once, on the same streams and
        # pinned buffers (no compute).
        def copies_ms(up, down, reps=5):
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            done = [torch.cuda.Event(), torch.cuda.Event()]
            torch.cuda.synchronize()
            t0.record(cur)
            for j, (on, st) in enumerate(((up, s_in), (down, s_out))):
                st.wait_event(t0)
                with torch.cuda.stream(st):
                    for _ in range(reps if on else 0):
                        if st is s_in:
                            for n, h in (("X", hX), ("W", hW), ("G", hG)):
                                sets[0][n].copy_(h, non_blocking=True)
                        else:
                            for n in ("y", "gw", "gx"):
                                hout[0][n].copy_(sets[0][n], non_blocking=True)
                    done[j].record(st)
                cur.wait_event(done[j])
            t1.record(cur)
            torch.cuda.synchronize()
            return t0.elapsed_time(t1) / reps

        up_ms, down_ms, both_ms = copies_ms(True, False), copies_ms(False, True), copies_ms(True, True)
        e2e["link"] = {"h2d_gbs": round(h2d / (up_ms * 1e-3) / 1e9, 1),
                       "d2h_gbs": round(d2h / (down_ms * 1e-3) / 1e9, 1),
                       "both_ms": round(both_ms, 4),
                       "frac": round(both_ms / e2e_ms, 4),
                       "note": "one step's copies in both directions at once, no compute; frac = that "
                               "time / the pipelined step time"}

    del graphs, step_graphs, kgraphs
    torch.cuda.synchronize()
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return

    peaks, peak_src = load_peaks()
    flops = layer.flops()
    ms_step = total_ms / args.steps
    value = 3 * flops * world / (ms_step * 1e-3) / 1e12
    hbm = peaks["hbm_gbs"]
    tc = peaks["bf16_tflops"]              # f16 and bf16 dense MMA have the same nominal rate
    kern = {}
    for name in ("fwd", "wgrad", "dgrad"):
        t = mean[name] * 1e-3
        tflops = flops / t / 1e12
        gbs = conv_b[name] / t / 1e9
        roof_t = max(flops / (tc * 1e12), conv_b[name] / (hbm * 1e9))
        bound = "tensor" if flops / (tc * 1e12) >= conv_b[name] / (hbm * 1e9) else "hbm"
        kern[name] = {"ms": round(mean[name], 5), "tflops": round(tflops, 2), "gbs": round(gbs, 1),
                      "bound": bound, "frac_of_roofline": round(roof_t / t, 4)}
    qbytes = sum(quant_b.values())
    qt = mean["quantize"] * 1e-3
    kern["quantize"] = {"ms": round(mean["quantize"], 5), "gbs": round(qbytes / qt / 1e9, 1),
                        "bound": "hbm", "frac_of_roofline": round(qbytes / qt / 1e9 / hbm, 4),
                        "launches": 2 if world == 1 else 8}
    dom = max(("fwd", "wgrad", "dgrad", "quantize"), key=lambda k: mean[k])
    if dom == "quantize":
        roof = {"kernel": "quantize (amax + block quantizer, X, W, G_Y)", "bound": "hbm",
                "achieved": kern["quantize"]["gbs"], "peak": hbm, "unit": "GB/s",
                "frac": round(kern["quantize"]["gbs"] / hbm, 4)}
    else:
        k = kern[dom]
        if k["bound"] == "tensor":
            roof = {"kernel": f"conv_{dom}", "bound": "tensor", "achieved": k["tflops"], "peak": tc,
                    "unit": "TFLOP/s", "frac": round(k["tflops"] / tc, 4)}
        else:
            roof = {"kernel": f"conv_{dom}", "bound": "hbm", "achieved": k["gbs"], "peak": hbm,
                    "unit": "GB/s", "frac": round(k["gbs"] / hbm, 4)}
    roof["peak_source"] = f"{peak_src} ({'MEASURED_PEAKS.json burst' if peak_src == 'measured' else 'recipe fallback'})"
    roof["traffic"] = args.traffic.get(roof["kernel"]) if args.traffic else None
    # quantize (amax + quantizer per tensor), fwd and dgrad (weight image + conv), wgrad (+ reduce)
    # launches in the loop that gives the value: the quantization (two per
    # quantize_many call, two calls when concurrent), prep + conv for fwd and
    # dgrad, conv + split reduce for wgrad
    launches_per_step = ((4 if concurrent else 2) if world == 1 else 4 + 2 + 2) + 2 + 2 + 1 + splits_reduce
    out = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16", "data": "synthetic",
        "config": {"workload": layer.name, "N": layer.N, "Cin": layer.Cin, "Cout": layer.Cout,
                   "H": layer.H, "W": layer.W, "K": layer.K, "stride": layer.stride, "pad": layer.pad,
                   "storage": f"{layer.fmt} (4x4 blocks, e4m3 block scales, fp32 tensor scale)",
                   "step": "quantize X,W (RNE) and G_Y (SR); conv fwd, wgrad, dgrad",
                   "l2": f"inputs rotated over {nsets} resident sets ({nsets * per_set / 1e6:.0f} MB > 126 MB L2)",
                   "launch": ("the whole step (both quantize launch pairs, the three passes on their "
                              "streams and the joins) replayed as one CUDA graph captured through the C ABI"
                              if concurrent else ("the serial step replayed as one CUDA graph captured through "
                                                  "the C ABI" if world == 1 else
                                                  "each phase replayed as a CUDA graph captured through the C ABI")),
                   "schedule": ("quantize X,W beside quantize G_Y; fwd after X,W; wgrad and dgrad after "
                                "all three; the passes on separate streams" if concurrent
                                else "quantize, fwd, wgrad, dgrad on one stream"),
                   "parallelism": f"dp{world}" if world > 1 else "single"},
        "quantize_gbs": kern["quantize"]["gbs"],
        "kernels": kern,
        "roofline": roof,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
        "device_error_flags": flags,
    }
    out["serial"] = {"ms_per_step": round(serial_ms / args.steps, 5),
                     "value": round(3 * flops * world / (serial_ms / args.steps * 1e-3) / 1e12, 3),
                     "note": ("the same step with quantize, fwd, wgrad, dgrad one after another, one graph per "
                              "step; the per-kernel durations and the roofline come from event nodes inside "
                              f"those graphs (the last {nk} steps of this loop)" if world == 1 else
                              "the same step with fwd, wgrad, dgrad one after another; the per-kernel "
                              "durations and the roofline come from this loop")}
    if concurrent:
        out["kernels_concurrent_ms"] = {k: round(v, 5) for k, v in conc_mean.items()}
        out["phase_graphs"] = {"ms_per_step": round(phase_ms / args.steps, 5),
                               "value": round(3 * flops * world / (phase_ms / args.steps * 1e-3) / 1e12, 3),
                               "note": "the same schedule as one graph per phase with cross-stream event "
                                       "waits between them; the concurrent phase durations come from this loop"}
    if e2e:
        out["e2e"] = e2e
    # against the quantize-once step on one stream, as the baseline runs
    for key, nr in (("naive_baseline", naive_res), ("naive_square_blocks", naive_sq)):
        if nr:
            nr["step_time_ratio"] = round(nr["ms_per_step"] / (serial_ms / args.steps), 3)
            nr["quantize_time_ratio"] = round(nr["phase_ms"]["quant"] / mean["quantize"], 3)
            out[key] = nr
    if world == 1:
        out["mma_form"] = run_mma_form(dev, layer, peaks)
    if world == 1 and not args.no_sweeps:
        # the benchmarked (tensor-bound) layer and an HBM-bound 1 x 1 layer,
        # where the fp32 output is most of the pass's bytes
        hbm_layer = {l.name: l for l in workloads.yolov8n_mix()}["yolov8n_l12_1x1_128_40px"]
        out["fused_epilogue"] = [run_fused(dev, layer, peaks), run_fused(dev, hbm_layer, peaks)]
        out["sweeps"] = run_sweeps(args, dev, peaks)
    if world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(layer, budget_s=args.cpu_budget)
    print(json.dumps(out), flush=True)


# ------------------------------------------------------- sweeps at 1 GPU

def _timed(torch, fn, iters, flush):
    """Mean device ms of fn over `iters` calls, each bracketed by its own
    CUDA events on the current stream, with L2 flushed (a 256 MB write)
    before each call, outside the events."""
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
    for a, b in evs:
        flush.zero_()
        a.record()
        fn()
        b.record()
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in evs) / iters


def run_sweeps(args, dev, peaks):
    """The other measured workloads, each as absolute throughput and as a
    fraction of its roofline:
      - replay_quantize: the quantize-only sweep over the latent-replay
        buffer shapes (1M..1G elements), |N(0,1)| with 0.1 % outliers x100,
        RNE and SR; 8.5625 algorithmic B/element (two fp32 reads, codes,
        scales);
      - replay_form: the magnitude-only replay form of the same quantized
        buffers: pack and unpack (0.5 + 0.375 B moved per element) and
        values read straight back (0.375 + 1/16 B read, 4 B written),
        beside mqv_dequantize of the full codes;
      - depthwise_bf16: the BF16 depthwise passes on YOLOv26n-style
        3x3 layers, against bytes / copy rate;
      - resnet18_body and yolov8n_mix: every layer's step (quantize, fwd,
        wgrad, dgrad) timed phase by phase with L2 flushed before each
        phase; per-network sums against the sum of per-pass rooflines."""
    import torch

    import microscaling_quantized_convolution_b200 as mqv

    hbm, tc = peaks["hbm_gbs"], peaks["bf16_tflops"]
    flush = torch.empty(64 << 20, dtype=torch.float32, device=dev)
    res = {"l2": "256 MB written before every timed call", "timing": "CUDA events per call"}
    launches = 0

    rq, rf = [], []
    for C, H, N in workloads.REPLAY_SHAPES:
        rows, cols = H * H * C, N
        n = rows * cols
        iters = 20 if n < 100_000_000 else 5
        x = workloads.make_replay_input(C, H, N, outliers=True, seed=3, device=dev).view(-1)
        q = mqv.QTensor.empty(rows, cols, "nvfp4", dev)
        ws = torch.empty(mqv.quantize_workspace_bytes(rows, cols), dtype=torch.uint8, device=dev)
        ent = {"C": C, "H": H, "N": N, "elements": n}
        for name, rnd in (("rne", mqv.RNE), ("sr", mqv.SR)):
            def f(rnd=rnd):
                mqv.quantize(x, rows, cols, "nvfp4", rnd, 11, out=q, ws=ws)
            for _ in range(3):
                f()
            ms = _timed(torch, f, iters, flush)
            launches += 2 * (iters + 3)
            gbs = 8.5625 * n / (ms * 1e-3) / 1e9
            ent[name] = {"ms": round(ms, 5), "gbs": round(gbs, 1), "frac": round(gbs / hbm, 4)}
        rq.append(ent)
        del x
        # replay form of the (RNE-rounded last: SR) quantized buffer
        mqv.quantize(workloads.make_replay_input(C, H, N, outliers=True, seed=3, device=dev).view(-1),
                     rows, cols, "nvfp4", mqv.RNE, 0, out=q, ws=ws)
        packed = torch.empty(mqv.replay_bytes(rows, cols, "nvfp4"), dtype=torch.uint8, device=dev)
        vals = torch.empty(n, dtype=torch.float32, device=dev)
        neg = torch.zeros(1, dtype=torch.int32, device=dev)
        codes2 = torch.empty_like(q.codes)
        calls = {"pack": (lambda: mqv.replay_pack(q, out=packed, negatives=neg), 0.875),
                 "unpack": (lambda: mqv.replay_unpack(packed, rows, cols, "nvfp4", codes=codes2), 0.875),
                 "read": (lambda: mqv.replay_dequantize(packed, q.scales, q.tscale, rows, cols, "nvfp4",
                                                        out=vals), 0.375 + 0.0625 + 4),
                 "dequantize_full_codes": (lambda: mqv.dequantize(q, out=vals), 0.5 + 0.0625 + 4)}
        fe = {"C": C, "H": H, "N": N, "elements": n, "bytes": mqv.replay_bytes(rows, cols, "nvfp4"),
              "bits_per_element": 3.5, "bits_per_element_signed": 4.5}
        for name, (fn, bpe) in calls.items():
            for _ in range(3):
                fn()
            ms = _timed(torch, fn, iters, flush)
            launches += iters + 3
            gbs = bpe * n / (ms * 1e-3) / 1e9
            fe[name] = {"ms": round(ms, 5), "gbs": round(gbs, 1), "frac": round(gbs / hbm, 4)}
        fe["negative_codes"] = int(neg.item())
        rf.append(fe)
        del q, ws, packed, vals, codes2
        torch.cuda.empty_cache()
    res["replay_quantize"] = rq
    res["replay_form"] = rf

    # depthwise 3x3 layers in BF16 (outside quantize-once): HBM-bound, so
    # each pass against bytes / copy rate, algorithmic bytes = the two bf16
    # operands read once (2 B/element) + the fp32 output written once
    dw = []
    for C, H, stv in workloads.DEPTHWISE_SHAPES:
        N = workloads.DEPTHWISE_N
        x, w, gy = (t.to(torch.bfloat16).contiguous()
                    for t in workloads.make_depthwise_inputs(C, H, stv, N, seed=C + H, device=dev))
        d = mqv.dw_desc(N, C, H, H, 3, 3, stv, 1)
        ho, _ = mqv.dw_out_hw(d)
        y = torch.empty(ho * ho * C * N, device=dev)
        gx = torch.empty(H * H * C * N, device=dev)
        gw = torch.empty(C * 9, device=dev)
        wsd = torch.empty(max(16, mqv.dw_wgrad_workspace_bytes(d)), dtype=torch.uint8, device=dev)
        nx, ny, nw = H * H * C * N, ho * ho * C * N, C * 9
        calls = {"fwd": (lambda: mqv.dw_fwd(d, w, x, y), 2 * (nw + nx) + 4 * ny),
                 "dgrad": (lambda: mqv.dw_dgrad(d, w, gy, gx), 2 * (nw + ny) + 4 * nx),
                 "wgrad": (lambda: mqv.dw_wgrad(d, gy, x, gw, ws=wsd), 2 * (ny + nx) + 4 * nw)}
        ent = {"C": C, "H": H, "stride": stv, "N": N}
        for name, (fn, nbytes) in calls.items():
            for _ in range(3):
                fn()
            ms = _timed(torch, fn, 10, flush)
            launches += 13 * (2 if name == "wgrad" else 1)
            gbs = nbytes / (ms * 1e-3) / 1e9
            ent[name] = {"ms": round(ms, 5), "gbs": round(gbs, 1), "frac": round(gbs / hbm, 4)}
        dw.append(ent)
        del x, w, gy, y, gx, gw, wsd
    res["depthwise_bf16"] = dw

    for net, layers in (("resnet18_body", workloads.resnet18_body()), ("yolov8n_mix", workloads.yolov8n_mix())):
        tot = {"quantize": 0.0, "fwd": 0.0, "wgrad": 0.0, "dgrad": 0.0}
        roof = {"quantize": 0.0, "conv": 0.0}
        flops_all, per_layer = 0, []
        for layer in layers:
            X, Wt, G = (t.view(-1) for t in workloads.make_layer_inputs(layer, device=dev))
            d = mqv.conv_desc(**layer.dims(), fmt=layer.fmt)
            xr, xc = layer.H * layer.W * layer.Cin, layer.N
            wr, wc = layer.Cout, layer.K * layer.K * layer.Cin
            gr, gc = layer.Ho * layer.Wo * layer.Cout, layer.N
            qx, qw, qg = (mqv.QTensor.empty(r, c, layer.fmt, dev) for r, c in ((xr, xc), (wr, wc), (gr, gc)))
            jobs = [(X, xr, xc, layer.fmt, mqv.RNE, 0, qx), (Wt, wr, wc, layer.fmt, mqv.RNE, 0, qw),
                    (G, gr, gc, layer.fmt, mqv.SR, workloads.sr_seed(layer), qg)]
            wsq = torch.empty(mqv.quantize_many_workspace_bytes([j[:6] for j in jobs]), dtype=torch.uint8,
                              device=dev)
            wss = {op: torch.empty(max(16, mqv.conv_workspace_bytes(d, op)), dtype=torch.uint8, device=dev)
                   for op in (mqv.OP_FWD, mqv.OP_WGRAD, mqv.OP_DGRAD)}
            y = torch.empty(gr * gc, device=dev)
            gw = torch.empty(wr * wc, device=dev)
            gx = torch.empty(xr * xc, device=dev)
            phases = {"quantize": lambda: mqv.quantize_many(jobs, ws=wsq),
                      "fwd": lambda: mqv.conv_fwd(d, qw, qx, y=y, ws=wss[mqv.OP_FWD]),
                      "wgrad": lambda: mqv.conv_wgrad(d, qg, qx, gw=gw, ws=wss[mqv.OP_WGRAD]),
                      "dgrad": lambda: mqv.conv_dgrad(d, qw, qg, gx=gx, ws=wss[mqv.OP_DGRAD])}
            for _ in range(3):
                for fn in phases.values():
                    fn()
            ms = {k: _timed(torch, fn, 5, flush) for k, fn in phases.items()}
            launches += 8 * (2 + 2 + 2 + 1 + (1 if mqv.conv_workspace_bytes(d, mqv.OP_WGRAD) else 0))
            qbytes, cbytes, _ = layer_bytes(layer)
            fl = layer.flops()
            flops_all += 3 * fl
            lr = {"layer": layer.name, "ms": {k: round(v, 5) for k, v in ms.items()}}
            lroof = 0.0
            for k in ("fwd", "wgrad", "dgrad"):
                tot[k] += ms[k]
                rt = max(fl / (tc * 1e12), cbytes[k] / (hbm * 1e9)) * 1e3
                roof["conv"] += rt
                lroof += rt
            tot["quantize"] += ms["quantize"]
            roof["quantize"] += sum(qbytes.values()) / (hbm * 1e9) * 1e3
            lr["conv_frac"] = round(lroof / (ms["fwd"] + ms["wgrad"] + ms["dgrad"]), 4)
            per_layer.append(lr)
            del X, Wt, G, qx, qw, qg, wsq, wss, y, gw, gx
        torch.cuda.empty_cache()
        conv_ms = tot["fwd"] + tot["wgrad"] + tot["dgrad"]
        res[net] = {"layers": len(layers), "conv_ms": round(conv_ms, 4),
                    "conv_tflops": round(flops_all / (conv_ms * 1e-3) / 1e12, 2),
                    "conv_frac_of_roofline": round(roof["conv"] / conv_ms, 4),
                    "quantize_ms": round(tot["quantize"], 4),
                    "quantize_frac_of_roofline": round(roof["quantize"] / tot["quantize"], 4),
                    "phase_ms": {k: round(v, 4) for k, v in tot.items()},
                    "per_layer": per_layer}
    flags = mqv.device_errors()
    if flags:
        raise SystemExit(f"device wait timeout flags {flags:#x} in the sweeps")
    res["launches"] = launches
    return res


def run_mma_form(dev, layer, peaks):
    """The forward pass of the layer in the two MMA forms the square blocks
    allow: fp16 products of dequantized codes (kind::f16, the default) and
    the native block-scaled MMA with each 4-element block row padded to a
    16-element scale group (kind::mxf4nvf4, mqv_conv_fwd_blockscaled).  Each
    call includes its weight image; L2 flushed before each call."""
    import torch

    import microscaling_quantized_convolution_b200 as mqv

    d = mqv.conv_desc(**layer.dims(), fmt=layer.fmt)
    try:
        mqv.conv_workspace_bytes(d, mqv.OP_FWD_BLOCKSCALED)
    except mqv.MqvError as e:
        return {"unsupported": str(e)}
    X, Wt, _ = (t.view(-1) for t in workloads.make_layer_inputs(layer, device=dev))
    xr, wr, wc = layer.H * layer.W * layer.Cin, layer.Cout, layer.K * layer.K * layer.Cin
    qx = mqv.quantize(X, xr, layer.N, layer.fmt, mqv.RNE)
    qw = mqv.quantize(Wt, wr, wc, layer.fmt, mqv.RNE)
    y = torch.empty(layer.Ho * layer.Wo * layer.Cout * layer.N, device=dev)
    ws_f = torch.empty(max(16, mqv.conv_workspace_bytes(d, mqv.OP_FWD)), dtype=torch.uint8, device=dev)
    ws_b = torch.empty(mqv.conv_workspace_bytes(d, mqv.OP_FWD_BLOCKSCALED), dtype=torch.uint8, device=dev)
    flush = torch.empty(64 << 20, dtype=torch.float32, device=dev)
    tc = peaks["bf16_tflops"]
    res = {"layer": layer.name, "note": "same layer, same quantized operands, weight image included, L2 flushed"}
    for name, fn in (("f16_dequantized", lambda: mqv.conv_fwd(d, qw, qx, y=y, ws=ws_f)),
                     ("mxf4nvf4_padded", lambda: mqv.conv_fwd_blockscaled(d, qw, qx, y=y, ws=ws_b))):
        for _ in range(3):
            fn()
        ms = _timed(torch, fn, 20, flush)
        tfl = layer.flops() / (ms * 1e-3) / 1e12
        res[name] = {"ms": round(ms, 5), "tflops": round(tfl, 2), "frac_of_dense_peak": round(tfl / tc, 4)}
    res["winner"] = min(("f16_dequantized", "mxf4nvf4_padded"), key=lambda k: res[k]["ms"])
    return res


def run_fused(dev, layer, peaks):
    """Producer epilogue fused with the next quantization's max pass, on the
    benchmarked layer: fwd writes ReLU(Y) and max|Y| and the next layer's
    X = ReLU(Y) is quantized in one pass (mqv_quantize_with_amax), against
    the plain chain fwd, ReLU written back, amax pass, quantize pass; and
    dgrad with max|G_X| fused, then the SR quantization of G_X, against
    dgrad, amax pass, quantize pass.  Each chain is timed whole, L2 flushed
    before each call."""
    import torch

    import microscaling_quantized_convolution_b200 as mqv

    X, Wt, G = (t.view(-1) for t in workloads.make_layer_inputs(layer, device=dev))
    d = mqv.conv_desc(**layer.dims(), fmt=layer.fmt)
    fmt = layer.fmt
    xr, xc = layer.H * layer.W * layer.Cin, layer.N
    wr, wc = layer.Cout, layer.K * layer.K * layer.Cin
    yr = layer.Ho * layer.Wo * layer.Cout
    qx = mqv.quantize(X, xr, xc, fmt, mqv.RNE)
    qw = mqv.quantize(Wt, wr, wc, fmt, mqv.RNE)
    qg = mqv.quantize(G, yr, xc, fmt, mqv.SR, 3)
    y = torch.empty(yr * xc, device=dev)
    gx = torch.empty(xr * xc, device=dev)
    amax = torch.empty(1, device=dev)
    qy = mqv.QTensor.empty(yr, xc, fmt, dev)
    qgx = mqv.QTensor.empty(xr, xc, fmt, dev)
    wsf = torch.empty(max(16, mqv.conv_workspace_bytes(d, mqv.OP_FWD)), dtype=torch.uint8, device=dev)
    wsd = torch.empty(max(16, mqv.conv_workspace_bytes(d, mqv.OP_DGRAD)), dtype=torch.uint8, device=dev)
    wsy = torch.empty(mqv.quantize_workspace_bytes(yr, xc), dtype=torch.uint8, device=dev)
    wsx = torch.empty(mqv.quantize_workspace_bytes(xr, xc), dtype=torch.uint8, device=dev)
    flush = torch.empty(64 << 20, dtype=torch.float32, device=dev)

    def fwd_plain():
        mqv.conv_fwd(d, qw, qx, y=y, ws=wsf)
        torch.relu_(y)
        mqv.quantize(y, yr, xc, fmt, mqv.RNE, 0, out=qy, ws=wsy)

    def fwd_fused():
        mqv.conv_fwd_fused(d, qw, qx, relu=True, y=y, y_amax=amax, ws=wsf)
        mqv.quantize_with_amax(y, yr, xc, fmt, mqv.RNE, 0, amax, out=qy)

    def dgrad_plain():
        mqv.conv_dgrad(d, qw, qg, gx=gx, ws=wsd)
        mqv.quantize(gx, xr, xc, fmt, mqv.SR, 4, out=qgx, ws=wsx)

    def dgrad_fused():
        mqv.conv_dgrad_fused(d, qw, qg, gx=gx, gx_amax=amax, ws=wsd)
        mqv.quantize_with_amax(gx, xr, xc, fmt, mqv.SR, 4, amax, out=qgx)

    res = {"layer": layer.name, "l2": "256 MB written before every timed chain"}
    for name, fn in (("fwd_relu_quantize", (fwd_plain, fwd_fused)), ("dgrad_quantize", (dgrad_plain, dgrad_fused))):
        plain, fused = fn
        for f in (plain, fused):
            for _ in range(3):
                f()
        tp = _timed(torch, plain, 50, flush)
        tf = _timed(torch, fused, 50, flush)
        res[name] = {"plain_ms": round(tp, 5), "fused_ms": round(tf, 5), "speedup": round(tp / tf, 3)}
    ne = yr * xc
    res["fwd_relu_quantize"]["note"] = ("plain: conv writes Y, a ReLU pass reads and writes it, an amax pass "
                                        "reads it, the quantizer reads it; fused: conv writes ReLU(Y) and its "
                                        "max, the quantizer reads it once")
    res["fwd_relu_quantize"]["bytes_removed"] = 12 * ne
    res["dgrad_quantize"]["bytes_removed"] = 4 * xr * xc
    # quantized producer output: the epilogue writes the next operand's codes
    # and scales with T from a given max (here the previous call's), so no
    # fp32 output goes through HBM at all
    tq = torch.empty(1, device=dev)
    mqv.conv_fwd_fused(d, qw, qx, relu=True, y=y, y_amax=tq, ws=wsf)
    tg = gx.abs().max().reshape(1)

    def fwd_quantized():
        mqv.conv_fwd_quantized(d, qw, qx, tq, relu=1, y_q=qy, y_amax=amax, ws=wsf)

    def dgrad_quantized():
        mqv.conv_dgrad_quantized(d, qw, qg, tg, 4, gx_q=qgx, gx_amax=amax, ws=wsd)

    for name, fn, base in (("fwd_relu_quantize", fwd_quantized, "fused_ms"),
                           ("dgrad_quantize", dgrad_quantized, "fused_ms")):
        try:
            for _ in range(3):
                fn()
        except mqv.MqvError as e:
            res[name]["quantized_output"] = {"unsupported": str(e)}
            continue
        tq_ms = _timed(torch, fn, 50, flush)
        res[name]["quantized_output"] = {
            "ms": round(tq_ms, 5), "speedup_vs_plain": round(res[name]["plain_ms"] / tq_ms, 3),
            "speedup_vs_fused": round(res[name][base] / tq_ms, 3),
            "note": "one pass: the epilogue writes codes and scales (T from a given max, delayed scaling)"}
    flags = mqv.device_errors()
    if flags:
        raise SystemExit(f"device wait timeout flags {flags:#x} in the fused chains")
    return res


# -------------------------------------------------------------- CPU oracle
# -------------------------------------------------------------- CPU oracle

def oracle_sample_layer(layer: workloads.Layer, n_batch: int, hw: int) -> workloads.Layer:
    """The same layer with the batch cut to n_batch and the input to hw x hw."""
    return workloads.Layer(layer.name + f"_sample_n{n_batch}_{hw}px", n_batch, layer.Cin, layer.Cout,
                           hw, hw, layer.K, layer.stride, layer.pad, layer.fmt, layer.x_dist,
                           layer.gy_std, layer.seed, layer.cin_real)


def oracle_step(sample: workloads.Layer):
    from oracle import mqv_oracle as O
    X, Wt, G = workloads.make_layer_inputs(sample)
    s = O.ConvShape(sample.N, sample.Cin, sample.Cout, sample.H, sample.W, sample.K, sample.K,
                    sample.stride, sample.pad)
    f = O.FP4 if sample.fmt == "nvfp4" else O.FP6
    qx, qw, qg = O.quantize_layer(X.numpy(), Wt.numpy(), G.numpy(), s, f, workloads.sr_seed(sample))
    O.layer_outputs(qx, qw, qg, s)


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(layer: workloads.Layer, budget_s: float = 15.0):
    """The oracle as it stands, timed on the host on a bounded sample of the
    same layer: the batch cut to 4 and the input to 14 x 14 pixels."""
    sample = oracle_sample_layer(layer, 4, min(layer.H, 14))
    oracle_step(sample)                      # warm-up
    t0 = time.perf_counter()
    n = 0
    while True:
        oracle_step(sample)
        n += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = (time.perf_counter() - t0) / n
    out = {"value": round(3 * sample.flops() / dt / 1e12, 6), "unit": "TFLOP/s",
           "cores": blas_threads(), "kind": "oracle",
           "sample": f"{sample.name}: quantize X,W,G_Y + fp64 im2col fwd/wgrad/dgrad with |ab| sums, "
                     f"{3 * sample.flops() / 1e9:.3f} GFLOP per step, {n} steps in {n * dt:.1f} s"}
    # the same sample on one core (BLAS limited to one thread), a third of the budget
    try:
        from threadpoolctl import threadpool_limits
    except ImportError:
        out["single_core"] = None
        return out
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        m = 0
        while True:
            oracle_step(sample)
            m += 1
            if time.perf_counter() - t0 > budget_s / 3:
                break
        dt1 = (time.perf_counter() - t0) / m
    out["single_core"] = {"value": round(3 * sample.flops() / dt1 / 1e12, 6), "cores": 1,
                          "steps": m}
    return out


def run_reference(args):
    """The CPU oracle as the reference arm: each step is the bounded sample."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    layer = pick_layer(args.workload)
    total = args.steps + args.warmup
    hw = 8 if total > 200 else 14
    sample = oracle_sample_layer(layer, 4, min(layer.H, hw))
    for _ in range(args.warmup):
        oracle_step(sample)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(sample)
    dt = (time.perf_counter() - t0) / args.steps
    v = round(3 * sample.flops() / dt / 1e12, 6)
    out = {"metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "impl": "reference",
           "config": {"workload": layer.name, "sample": sample.name},
           "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                            "sample": f"{sample.name} per step"},
           "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def run_probe(args):
    """A small fixed case for single-kernel ncu captures: the layer's step
    (quantize X, W, G_Y in one call; fwd in both MMA forms, wgrad, dgrad)
    `args.probe` times through the public API, then a device-error check.
    Prints one line; no timing (numbers taken under a profiler are not
    bench values)."""
    import torch

    import microscaling_quantized_convolution_b200 as mqv

    layer = pick_layer(args.workload)
    dev = torch.device("cuda", 0)
    X, Wt, G = (t.view(-1) for t in workloads.make_layer_inputs(layer, device=dev))
    d = mqv.conv_desc(**layer.dims(), fmt=layer.fmt)
    xr, wr, wc = layer.H * layer.W * layer.Cin, layer.Cout, layer.K * layer.K * layer.Cin
    gr = layer.Ho * layer.Wo * layer.Cout
    try:
        mqv.conv_workspace_bytes(d, mqv.OP_FWD_BLOCKSCALED)
        blockscaled = True
    except mqv.MqvError:
        blockscaled = False
    for i in range(args.probe):
        qx, qw, qg = mqv.quantize_many([(X, xr, layer.N, layer.fmt, mqv.RNE, 0), (Wt, wr, wc, layer.fmt, mqv.RNE, 0),
                                        (G, gr, layer.N, layer.fmt, mqv.SR, 7 + i)])
        mqv.conv_fwd(d, qw, qx)
        if blockscaled:
            mqv.conv_fwd_blockscaled(d, qw, qx)
        mqv.conv_wgrad(d, qg, qx)
        mqv.conv_dgrad(d, qw, qg)
    torch.cuda.synchronize()
    flags = mqv.device_errors()
    print(json.dumps({"probe": layer.name, "iterations": args.probe, "device_error_flags": flags}))
    if flags:
        sys.exit(1)


def run_probe_depthwise(args):
    """The BF16 depthwise passes (fwd, dgrad, wgrad) of one layer of the
    depthwise sweep, `args.probe_depthwise` times, for single-kernel ncu
    captures.  Prints one line; no timing."""
    import torch

    import microscaling_quantized_convolution_b200 as mqv

    C, H, stv = workloads.DEPTHWISE_SHAPES[args.depthwise_shape]
    N = workloads.DEPTHWISE_N
    dev = torch.device("cuda", 0)
    x, w, gy = (t.to(torch.bfloat16).contiguous()
                for t in workloads.make_depthwise_inputs(C, H, stv, N, seed=C + H, device=dev))
    d = mqv.dw_desc(N, C, H, H, 3, 3, stv, 1)
    for _ in range(args.probe_depthwise):
        mqv.dw_fwd(d, w, x)
        mqv.dw_dgrad(d, w, gy)
        mqv.dw_wgrad(d, gy, x)
    torch.cuda.synchronize()
    flags = mqv.device_errors()
    print(json.dumps({"probe": f"depthwise_c{C}_h{H}_s{stv}_n{N}", "iterations": args.probe_depthwise,
                      "device_error_flags": flags}))
    if flags:
        sys.exit(1)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="mine", choices=["mine", "reference"])
    ap.add_argument("--workload", default=workloads.resnet18_layer2().name)
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--serial", action="store_true",
                    help="run fwd, wgrad and dgrad one after another on one stream")
    ap.add_argument("--naive-steps", type=int, default=100,
                    help="steps of the quantize-after-im2col baseline (0: skip)")
    ap.add_argument("--no-sweeps", action="store_true",
                    help="skip the replay-buffer and whole-network sweeps")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--traffic-json", default=os.path.join(ROOT, "profiles", "traffic.json"))
    ap.add_argument("--probe", type=int, default=0,
                    help="run the layer's step this many times for a profiler capture and exit (no timing)")
    ap.add_argument("--probe-depthwise", type=int, default=0,
                    help="run one depthwise sweep layer's three passes this many times and exit (no timing)")
    ap.add_argument("--depthwise-shape", type=int, default=0,
                    help="index into the depthwise sweep shapes for --probe-depthwise")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    args.traffic = None
    if os.path.exists(args.traffic_json):
        with open(args.traffic_json) as f:
            args.traffic = json.load(f).get(args.workload)
    if args.probe > 0:
        run_probe(args)
    elif args.probe_depthwise > 0:
        run_probe_depthwise(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
