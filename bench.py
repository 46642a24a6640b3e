#!/usr/bin/env python
"""Benchmark of the routed-MoE layer on B200: one JSON line on rank 0.

A step is one pass of the whole layer (router, top-k + softmax, permutation, gate_up +
GeGLU, down + combine) over one batch of synthetic inputs, through the C ABI. The headline
workload is the eight-request decode batch (decode_T8: T = 8 tokens, d = 2816, f = 704,
E = 128, k = 8); the same line carries, under "workloads", the single-token layer
(layer_T1), the 4,096-token prefill (prefill_T4096, the tensor-core half of the metric), the
30-layer single-token stack (stack30_T1) and the long prompts of 10,000 and 40,000 tokens
(prefill_T10000, prefill_T40000: chunks of 4,096 tokens) and the decode batch through the
routed experts plus the block's dense MLP (block_T8), each with its own timing, roofline,
end-to-end figure and clocks. Consecutive decode steps rotate over several independent
layers so that the active experts' weights of one step are not L2-resident in the next
(inputs larger than L2); a prefill step reads all 428 MB of a layer's experts, a stack step
all 30 layers.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--extra A,B|none]
                  [--impl ours|reference]

Multi-GPU (torchrun, one rank per GPU): every rank runs an independent replica of the
workload (weak scaling); timing is the max over ranks of the device-timed region.
`--impl reference` times the FP64 CPU oracle on the host cores instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import moe_inputs as mi  # noqa: E402

METRIC = "MoE-layer tokens/s; decode HBM GB/s & prefill TFLOP/s as % of B200 roofline"
EXTRA_DEFAULT = "layer_T1,prefill_T4096,stack30_T1,prefill_T10000,prefill_T40000,block_T8"
# tokens of each workload, and the workspace's token capacity (longer calls run in chunks)
WORKLOAD_T = {"layer_T1": 1, "decode_T8": 8, "stack30_T1": 1, "prefill_T4096": 4096, "skewed_T512": 512,
              "prefill_T10000": 10000, "prefill_T40000": 40000, "block_T8": 8}
CHUNK_TOKENS = 4096


def parse(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--workload", default="decode_T8", choices=mi.WORKLOADS)
    p.add_argument("--extra", default=EXTRA_DEFAULT,
                   help="comma-separated workloads measured after the headline one, or 'none'")
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--layers", type=int, default=0, help="layers rotated across decode steps (0: auto)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--load-s", type=float, default=0.6,
                   help="seconds of untimed replays before and after each timed region (clock samples)")
    return p.parse_args(argv)


def extra_workloads(args) -> list:
    if args.extra.strip().lower() in ("", "none"):
        return []
    out = []
    for name in args.extra.split(","):
        name = name.strip()
        if name not in mi.WORKLOADS:
            raise SystemExit(f"unknown workload {name!r} in --extra")
        if name != args.workload and name not in out:
            out.append(name)
    return out


# ----------------------------------------------------------------------------- peaks

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            pk = json.load(fh)
        return {"hbm_gbs": float(pk["hbm_gbs"]), "bf16_tflops": float(pk["bf16_tflops"]),
                "bf16_tflops_sustained": float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms; only the samples taken
    between mark_load_start() and mark_load_end() (the GPU busy with the workload) count."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []
        self.thread = None
        self.t_load = (None, None)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def mark_load_start(self):
        self.t_load = (time.monotonic(), None)

    def mark_load_end(self):
        self.t_load = (self.t_load[0], time.monotonic())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        return summarize_clock_lines(self.lines, *self.t_load)


def summarize_clock_lines(lines, t0=None, t1=None):
    """Median SM clock, max clock and the throttle reasons seen in the (time, csv line)
    samples taken between t0 and t1 (all samples when either is None)."""
    sm, mx, pw, reasons = [], [], [], set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for t, ln in lines:
        if t0 is not None and t1 is not None and not (t0 <= t <= t1):
            continue
        parts = [x.strip() for x in ln.split(",")]
        if len(parts) < 8:
            continue
        try:
            sm.append(float(parts[0]))
            mx.append(float(parts[1]))
        except ValueError:
            continue
        try:
            pw.append(float(parts[2]))
        except ValueError:
            pass
        for nm, v in zip(names, parts[4:8]):
            if v.lower().startswith("active"):
                reasons.add(nm)
    if not sm:
        return None
    return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
            "samples": len(sm), "power_w_max": max(pw) if pw else None}


# ----------------------------------------------------------------------------- helpers

def flops_bytes(lw: mi.LayerWeights, T: int, k: int, counts: np.ndarray):
    """Algorithmic work of one layer call given the per-expert token counts."""
    d, f = lw.d, lw.f
    active = int((counts > 0).sum())
    gu_bytes = active * 2 * f * (d // 32) * 18
    dn_bytes = active * d * (f // 32) * 18
    router_bytes = lw.E * d * 4
    act_bytes = T * d * 2 + T * d * 4          # x in, out
    h_bytes = T * k * f * 4                    # h written by gate_up, read by down
    flops = 2 * T * k * (2 * f * d + d * f) + 2 * T * lw.E * d
    return {"active": active, "gateup_weight_bytes": gu_bytes, "down_weight_bytes": dn_bytes,
            "router_bytes": router_bytes, "act_bytes": act_bytes, "h_bytes": h_bytes,
            "total_bytes": gu_bytes + dn_bytes + router_bytes + act_bytes + 2 * h_bytes,
            "flops": flops, "gateup_flops": 2 * T * k * 2 * f * d, "down_flops": 2 * T * k * d * f}


def strip_c_comments(src: str) -> str:
    """C/C++ source without its comments and blank lines (string and character literals kept
    intact), so that editing a comment does not count as changing a kernel."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":                                   # a literal: copy it to its closing quote
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = (ln.rstrip() for ln in "".join(out).splitlines())
    return "\n".join(ln for ln in lines if ln)


def sources_sha256() -> str:
    """Hash of the CUDA sources' code (comments and blank lines removed); a recorded ncu
    traffic figure is valid only for this hash."""
    import glob
    import hashlib
    h = hashlib.sha256()
    for p in sorted(glob.glob(os.path.join(ROOT, "mixture_experts_gemv_b200", "csrc", "*"))):
        with open(p, encoding="utf-8") as fh:
            code = strip_c_comments(fh.read())
        h.update(os.path.basename(p).encode() + b"\0" + code.encode())
    return h.hexdigest()


def recorded_traffic(kernel: str, workload: str, units_per_launch: float):
    """DRAM bytes (read + write) per launch of `kernel` from the ncu summary in profiles/,
    scaled to this launch's units when the capture ran a smaller case; None when no summary
    exists or the sources changed since it was captured."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    fields = {}
    with open(path) as fh:
        for ln in fh:
            if ln.startswith("- ") and ":" in ln:
                key, _, val = ln[2:].partition(":")
                val = val.strip()
                if val.startswith("`"):   # the value is the first back-quoted token
                    val = val[1:].partition("`")[0]
                fields[key.strip()] = val
    try:
        if fields.get("sources_sha256") != sources_sha256():
            return None
        traffic = float(fields["dram_bytes_per_launch"])
        units = float(fields.get("units_per_launch", units_per_launch))
        return traffic * units_per_launch / units
    except (KeyError, ValueError):
        return None


def max_over_ranks(vals, device):
    """Element-wise maximum of this rank's timings over all ranks (the slowest rank decides a
    multi-GPU time); the values themselves at one rank."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in vals]
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_throughput(ws: int, units_per_rank_step: float, steps: int, ms_max: float) -> float:
    """Whole-job units per second: every rank's units over the slowest rank's time."""
    return ws * units_per_rank_step * steps / (ms_max / 1e3)


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def decode_launch_roofline(bytes_per_launch, kms, nl, ms_launch_bound, pk, kernel, workload):
    """Roofline of the fused decode kernel: algorithmic bytes per launch over its duration.
    The duration is the per-kernel event time, or, when a step is nothing but these launches,
    the timed region's time per launch (an upper bound without the event nodes' overhead)."""
    ms_launch, src = kms / nl, "per-kernel events (a second replay with an event pair per launch)"
    if ms_launch_bound is not None and ms_launch_bound < ms_launch:
        ms_launch, src = ms_launch_bound, "timed region (a step is nothing but these launches)"
    achieved = bytes_per_launch / (ms_launch / 1e3) / 1e9
    return {"kernel": kernel, "bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / pk["hbm_gbs"], "traffic": recorded_traffic(kernel, workload, bytes_per_launch),
            "peak_source": pk["source"] + " (hbm_gbs, copy bandwidth)", "bytes_per_launch": bytes_per_launch,
            "ms_per_launch": ms_launch, "ms_source": src, "ms_per_launch_events": kms / nl}


def gemm_roofline(flops, kms, nl, pk, kernel, workload):
    achieved = flops / (kms / nl / 1e3) / 1e12
    return {"kernel": kernel, "bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"],
            "unit": "TFLOP/s", "frac": achieved / pk["bf16_tflops"],
            "frac_of_sustained": achieved / pk["bf16_tflops_sustained"],
            "traffic": recorded_traffic("k_moe_gemm", workload, flops) if kernel == "k_moe_gemm<gate_up>" else None,
            "peak_source": pk["source"] + " (bf16_tflops, burst)", "flops_per_launch": flops,
            "ms_per_launch": kms / nl}


# ----------------------------------------------------------------------------- reference arm

def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    wl = mi.make_workload(args.workload, n_layers=1 if args.workload == "stack30_T1" else None)
    lw = wl.layers[0]
    k = wl.k
    # size one step: time a single token, then take as many tokens as fit the budget per step
    t0 = time.perf_counter()
    oracle.moe_layer(wl.x[:1], lw.router_w, lw.router_scale, lw.gate_up, lw.down, lw.expert_scale, k)
    one = time.perf_counter() - t0
    budget = 120.0 / max(1, args.steps + args.warmup)
    n_tok = int(max(1, min(wl.T, budget / max(one, 1e-6))))
    xs = wl.x[:n_tok]
    for _ in range(args.warmup):
        oracle.moe_layer(xs, lw.router_w, lw.router_scale, lw.gate_up, lw.down, lw.expert_scale, k)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.moe_layer(xs, lw.router_w, lw.router_scale, lw.gate_up, lw.down, lw.expert_scale, k)
    el = time.perf_counter() - t0
    val = n_tok * args.steps / el
    sample = f"{n_tok} of the {wl.T} tokens of {args.workload} per step (one layer, FP64 oracle)"
    line = {"metric": METRIC, "value": val, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "T": wl.T, "d": lw.d, "f": lw.f, "E": lw.E, "k": k},
            "impl": "reference",
            "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- our arm

class Bench:
    """Device state shared by the workloads of one run: the library, layers on the device
    (generated once, seed 0), the stream and the run's arguments."""

    def __init__(self, args, moe, dev, ws):
        import torch
        self.torch = torch
        self.args, self.moe, self.dev, self.ws = args, moe, dev, ws
        self.host_layers = {}
        self.dev_layers = {}
        self.pk = measured_peaks()

    def layer(self, i):
        if i not in self.host_layers:
            self.host_layers[i] = mi.make_layer(0, i)
        return self.host_layers[i]

    def prefetch_layers(self, idxs):
        todo = [i for i in idxs if i not in self.host_layers]
        for i, lw in zip(todo, mi.make_layers(todo)):
            self.host_layers[i] = lw

    def up(self, a):
        a = np.ascontiguousarray(a)
        if a.dtype == np.uint16:
            a = a.view(np.int16)
        return self.torch.from_numpy(a).to(self.dev)

    def dev_layer(self, key, lw):
        if key not in self.dev_layers:
            self.dev_layers[key] = dict(router_w=self.up(lw.router_w), router_scale=self.up(lw.router_scale),
                                        gate_up=self.up(lw.gate_up), down=self.up(lw.down),
                                        expert_scale=self.up(lw.expert_scale))
        return self.dev_layers[key]

    def barrier(self):
        if self.ws > 1:
            import torch.distributed as dist
            dist.barrier()

    # ------------------------------------------------------------------ one workload
    def measure(self, name):
        torch, moe, args, dev = self.torch, self.moe, self.args, self.dev
        stack = name == "stack30_T1"
        block = name == "block_T8"   # the routed experts plus the block's dense MLP (f_dense = 704)
        T = WORKLOAD_T[name]
        if stack:
            idx = list(range(30))
        else:
            n_rot = args.layers or (6 if T <= 16 else 1)
            idx = list(range(n_rot))
        self.prefetch_layers(idx)
        base = mi.make_workload(name, layer_fn=self.layer)
        k = base.k
        lw0 = base.layers[0]
        d, f, E = lw0.d, lw0.f, lw0.E
        if stack:
            layers = [(("plain", i), self.layer(i)) for i in idx]
        elif name == "skewed_T512":
            layers = [(("skewed", 0), lw0)]
            for i in idx[1:]:
                w = mi.make_workload("skewed_T512", layer_fn=lambda j, i=i: self.layer(i))
                layers.append((("skewed", i), w.layers[0]))
        else:
            layers = [(("plain", i), self.layer(i)) for i in idx]
        dl = [self.dev_layer(key, lw) for key, lw in layers]
        fd = mi.D_FF_DENSE
        dense = []
        if block:
            for key, _ in layers:
                gud, dnd = mi.make_dense(0, key[1], d, fd)
                dense.append((self.up(gud), self.up(dnd)))
        x = self.up(base.x)
        out = torch.empty((T, d), dtype=torch.float32, device=dev)

        def step(i, xin=None, o=None):
            xin = x if xin is None else xin
            o = out if o is None else o
            stream = torch.cuda.current_stream(dev)   # the capture stream while recording a graph
            if stack:
                moe.moe_stack_forward(xin, [q["router_w"] for q in dl], [q["router_scale"] for q in dl],
                                      [q["gate_up"] for q in dl], [q["down"] for q in dl],
                                      [q["expert_scale"] for q in dl], T, d, f, E, k, 1e-6, o, None, stream)
            elif block:
                q, dq = dl[i % len(dl)], dense[i % len(dl)]
                moe.moe_block_forward(xin, q["router_w"], q["router_scale"], q["gate_up"], q["down"],
                                      q["expert_scale"], dq[0], dq[1], T, d, f, fd, E, k, o, stream)
            else:
                q = dl[i % len(dl)]
                moe.moe_layer_forward(xin, q["router_w"], q["router_scale"], q["gate_up"], q["down"],
                                      q["expert_scale"], T, d, f, E, k, o, stream)

        # per-layer algorithmic work, from the GPU's own routing of each layer on this x (a
        # stacked layer reads the previous output instead; at T = 1 every layer has k
        # active experts either way)
        stream = torch.cuda.current_stream(dev)
        work = []
        for (key, lw), q in zip(layers, dl):
            moe.moe_layer_forward(x, q["router_w"], q["router_scale"], q["gate_up"], q["down"],
                                  q["expert_scale"], T, d, f, E, k, out, stream)
            cnt = torch.empty(E, dtype=torch.int32, device=dev)
            moe.moe_debug_get_routing(counts=cnt, stream=stream)
            torch.cuda.synchronize()
            wk = flops_bytes(lw, T, k, cnt.cpu().numpy())
            if block:
                # the dense MLP's pass: its Q4_0 weights, a one-row zero router, x and out again
                dense_w = 2 * fd * (d // 32) * 18 + d * (fd // 32) * 18
                wk["dense_bytes"] = dense_w + d * 4 + T * d * 6
                wk["total_bytes"] += wk["dense_bytes"]
                wk["flops"] += 2 * T * (2 * fd * d + d * fd)
            work.append(wk)
        moe.moe_debug_check(stream)
        avg = {kk: float(np.mean([w[kk] for w in work])) for kk in work[0]}

        for i in range(args.warmup):
            step(i)
        torch.cuda.synchronize()

        # The K steps are captured once into a CUDA graph and replayed: the library only
        # enqueues work, so a replay runs exactly the kernels of K eager steps without host
        # launch gaps between them.
        def capture(fn):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fn()
            return g

        def run_steps():
            for i in range(args.steps):
                step(i)

        graph = capture(run_steps)
        graph.replay()
        torch.cuda.synchronize()

        props = torch.cuda.get_device_properties(dev)
        gpu_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(dev.index)
        sampler = ClockSampler(gpu_id)
        sampler.start()
        time.sleep(0.5)                      # nvidia-smi's first samples

        def load(seconds):                   # untimed replays keep the GPU busy while sampling
            t_end = time.monotonic() + seconds
            while time.monotonic() < t_end:
                graph.replay()
                torch.cuda.synchronize()

        sampler.mark_load_start()
        load(args.load_s)
        # ---- timed region: K steps
        self.barrier()
        torch.cuda.synchronize()
        ev0 = torch.cuda.Event(enable_timing=True)
        ev1 = torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        graph.replay()
        ev1.record(stream)
        torch.cuda.synchronize()
        self.barrier()
        ms = ev0.elapsed_time(ev1)
        load(args.load_s)
        sampler.mark_load_end()
        clocks = sampler.stop()
        moe.moe_debug_check(stream)
        ms = max_over_ranks([ms], dev)[0]
        ms_step = ms / args.steps
        del graph

        # ---- per-kernel timing: the same K steps with CUDA events recorded around every
        # kernel group on the launch stream (captured as event nodes), replayed once
        self.barrier()
        moe.moe_profile_begin()
        pgraph = capture(run_steps)
        kernels = moe.moe_profile_kernel_launches()
        pgraph.replay()
        torch.cuda.synchronize()
        prof = moe.moe_profile_end()
        del pgraph

        # ---- end to end through the C ABI with host buffers: every step copies its x from
        # pinned host memory to the device and its out back to pinned host memory. The steps
        # are independent batches, so the copies are pipelined as a serving loop would: step
        # i + 1's input copy and step i - 1's output copy (two copy streams) run during step
        # i's layer call; device buffers are double-buffered and every reuse waits on the step
        # that last used the buffer.
        xh = torch.from_numpy(np.ascontiguousarray(base.x).view(np.int16)).pin_memory()
        oh = torch.empty((T, d), dtype=torch.float32).pin_memory()
        xd = [torch.empty_like(x) for _ in range(2)]
        od = [torch.empty_like(out) for _ in range(2)]
        h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

        def e2e_steps():
            main = torch.cuda.current_stream(dev)
            K = args.steps
            ev_in = [torch.cuda.Event() for _ in range(K)]
            ev_comp = [torch.cuda.Event() for _ in range(K)]
            ev_out = [torch.cuda.Event() for _ in range(K)]
            h2d_s.wait_stream(main)
            d2h_s.wait_stream(main)
            for i in range(K):
                b = i & 1
                with torch.cuda.stream(h2d_s):
                    if i >= 2:
                        h2d_s.wait_event(ev_comp[i - 2])     # step i - 2 has read xd[b]
                    xd[b].copy_(xh, non_blocking=True)
                    ev_in[i].record(h2d_s)
                main.wait_event(ev_in[i])
                if i >= 2:
                    main.wait_event(ev_out[i - 2])           # od[b] has been read back
                with torch.cuda.stream(main):
                    step(i, xd[b], od[b])
                ev_comp[i].record(main)
                with torch.cuda.stream(d2h_s):
                    d2h_s.wait_event(ev_comp[i])
                    oh.copy_(od[b], non_blocking=True)
                    ev_out[i].record(d2h_s)
            main.wait_stream(h2d_s)
            main.wait_stream(d2h_s)

        e2e_steps()
        torch.cuda.synchronize()
        egraph = capture(e2e_steps)
        egraph.replay()
        torch.cuda.synchronize()
        self.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        egraph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        self.barrier()
        ms_e2e = e0.elapsed_time(e1)
        # the same without a graph: one eager C-ABI call per step from Python
        e0.record(stream)
        e2e_steps()
        e1.record(stream)
        torch.cuda.synchronize()
        self.barrier()
        ms_e2e_eager = e0.elapsed_time(e1)
        del egraph
        ms_e2e, ms_e2e_eager = max_over_ranks([ms_e2e, ms_e2e_eager], dev)
        moe.moe_debug_check(stream)

        # ---- roofline of the dominant kernel
        pk = self.pk
        ws = self.ws
        n_layers = len(layers) if stack else 1
        extra = {}
        if T <= 16 and "fused_decode" in prof:
            # the whole layer is one kernel: its algorithmic bytes are the active experts' Q4_0
            # weights, the router weights, x, out and the scales (the dense MLP's weights too,
            # when it rides in the same launch; when it takes a pass of its own, a step is two
            # launches and the bytes per launch are the step's over two)
            kms, nl = prof["fused_decode"]
            per_launch_bytes = (avg["gateup_weight_bytes"] + avg["down_weight_bytes"] + avg["router_bytes"] +
                                avg["act_bytes"] + 4 * (E + 1))
            launches = n_layers
            if block:
                launches = max(1, round(nl / args.steps))
                dense_b = (avg["dense_bytes"] - T * d * 6 - d * 4) if launches == 1 else avg["dense_bytes"] + 8
                per_launch_bytes = (per_launch_bytes + dense_b) / launches
            only = set(prof) == {"fused_decode"} and nl == args.steps * launches
            roof = decode_launch_roofline(per_launch_bytes, kms, nl, ms_step / launches if only else None, pk,
                                          "k_moe_decode", name)
            dtype = "int16xq4->int32, f32"
        elif T <= 16:
            kms, nl = prof.get("gateup_gemv", (float("nan"), 1))
            per_launch_bytes = avg["gateup_weight_bytes"] + T * d * 4 + T * k * f * 8
            achieved = per_launch_bytes / (kms / nl / 1e3) / 1e9
            roof = {"kernel": "k_gateup_gemv", "bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"],
                    "unit": "GB/s", "frac": achieved / pk["hbm_gbs"],
                    "traffic": recorded_traffic("k_gateup_gemv", name, per_launch_bytes),
                    "peak_source": pk["source"] + " (hbm_gbs, copy bandwidth)",
                    "bytes_per_launch": per_launch_bytes, "ms_per_launch": kms / nl}
            dtype = "int16xq4->int32, f32"
        else:
            # one GEMM launch per chunk of CHUNK_TOKENS tokens: a launch's flops are the step's
            # over the launches per step
            kms, nl = prof.get("gateup_gemm", (float("nan"), 1))
            per_step = max(1, round(nl / args.steps))
            roof = gemm_roofline(avg["gateup_flops"] / per_step, kms, nl, pk, "k_moe_gemm<gate_up>", name)
            if "down_gemm" in prof:
                dms, dnl = prof["down_gemm"]
                extra["roofline_down"] = gemm_roofline(avg["down_flops"] / per_step, dms, dnl, pk, "k_moe_gemm<down>",
                                                       name)
            if per_step > 1:
                extra["chunks_per_step"] = per_step
            extra["tflops_per_step"] = avg["flops"] / (ms_step / 1e3) / 1e12
            dtype = "bf16"
        step_gbs = avg["total_bytes"] * n_layers / (ms_step / 1e3) / 1e9
        res = {"workload": name, "value": job_throughput(ws, T, args.steps, ms), "unit": "tokens/s",
               "ms_per_step": ms_step, "steps": args.steps, "warmup": args.warmup, "dtype": dtype,
               "config": {"workload": name, "T": T, "d": d, "f": f, "E": E, "k": k, "layers_per_step": n_layers,
                          "layers_rotated": 30 if stack else len(dl), "active_experts_mean": avg["active"],
                          "chunk_tokens": CHUNK_TOKENS,
                          "l2": ("inputs larger than L2: 30 layers (12.8 GB) per step" if stack else
                                 "inputs larger than L2: consecutive steps use different layers' weights"
                                 if len(dl) > 1 else
                                 "inputs larger than L2: every step reads the layer's 428 MB of experts"),
                          "parallelism": f"replicas x{ws}"},
               "roofline": roof, **extra,
               "step_bytes": avg["total_bytes"] * n_layers, "step_gbs": step_gbs,
               "step_hbm_frac": step_gbs / pk["hbm_gbs"],
               "kernel_ms_per_step": {kk: v[0] / args.steps for kk, v in prof.items()},
               "gpu_launches": int(kernels),
               "e2e": {"value": job_throughput(ws, T, args.steps, ms_e2e), "unit": "tokens/s",
                       "h2d_bytes_per_step": T * d * 2, "d2h_bytes_per_step": T * d * 4,
                       "launch": "CUDA graph of K steps; copies pipelined on two copy streams, double-buffered",
                       "eager_value": job_throughput(ws, T, args.steps, ms_e2e_eager)},
               "clocks": clocks}
        if stack:
            res["stack_steps_per_s"] = job_throughput(ws, 1, args.steps, ms)
        return res, layers, base


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    ws, rank, local = dist_env()
    if ws > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    from mixture_experts_gemv_b200 import build as moe_build
    moe_build.build()
    import mixture_experts_gemv_b200 as moe

    names = [args.workload] + extra_workloads(args)
    T_max = max(WORKLOAD_T[n] for n in names)
    moe.moe_init(local, min(T_max, CHUNK_TOKENS), mi.D_MODEL, mi.D_FF, mi.N_EXPERTS, mi.TOP_K)
    moe.moe_set_path(moe.MOE_PATH_AUTO, 16)
    b = Bench(args, moe, dev, ws)

    head, layers, base = b.measure(args.workload)
    subs = {}
    for name in names[1:]:
        subs[name] = b.measure(name)[0]

    line = {"metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": head["dtype"], "data": "synthetic",
            "config": head["config"], "roofline": head["roofline"]}
    for kk in ("roofline_down", "chunks_per_step", "tflops_per_step", "step_bytes", "step_gbs", "step_hbm_frac",
               "kernel_ms_per_step", "gpu_launches", "e2e", "clocks", "stack_steps_per_s"):
        if kk in head:
            line[kk] = head[kk]
    if subs:
        line["workloads"] = subs

    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        import oracle
        lw = layers[0][1]
        T = base.T
        n_tok = T if T <= 8 else 2
        t0 = time.perf_counter()
        reps = 0
        while True:
            oracle.moe_layer(base.x[:n_tok], lw.router_w, lw.router_scale, lw.gate_up, lw.down,
                             lw.expert_scale, base.k)
            reps += 1
            if time.perf_counter() - t0 > 10.0:
                break
        el = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": n_tok * reps / el, "unit": "tokens/s", "cores": oracle.num_threads(),
                                "kind": "oracle",
                                "sample": f"{reps} FP64 oracle layer calls on {n_tok} tokens of {args.workload}"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    moe.moe_destroy()
    if ws > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
