#!/usr/bin/env python
"""Benchmark of the routed-expert MoE layer (512 experts, top-10, hidden
3072, expert FFN 1024, SB3 up/gate + NL4 down) on B200.

A step is one whole decode layer -- router + top-k, grouping, expert FFN
with in-kernel dequantisation, combine -- for T tokens (default 3: one token
plus two MTP drafts), through the C ABI (moe_layer_forward).  Steps rotate
over `--layers` distinct layers whose experts are all resident in HBM
(2.19 GB each), so no step finds its expert bytes in L2 (126 MB).

Prints one JSON line (rank 0).  `--impl reference` times the fp64 CPU oracle
on the same workload instead (a bounded sample per step).
Multi-GPU (torchrun): independent replicas, one per GPU ("replicas only":
the decode layer does not shard); max-over-ranks device time.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = ("MoE-layer tokens/s (decode GB/s vs HBM peak; prefill TFLOP/s vs "
          "bf16 peak)")
UP_BYTES = 2 * synth.BIG.up_bytes          # up + gate of one expert
DOWN_BYTES = synth.BIG.down_bytes
BLOB = synth.BIG.blob_bytes
WR_BYTES = synth.BIG.E * synth.BIG.H * 2   # bf16 router of one layer
LAUNCHES_PER_STEP = 1                      # the one-kernel decode layer
SEED = 0                                   # input seed (--seed)


KERNEL_SOURCES = ["quantized_moe_expert_02_b200/csrc/decode_layer.cu",
                  "quantized_moe_expert_02_b200/csrc/decode_pieces.cuh",
                  "quantized_moe_expert_02_b200/csrc/moe_internal.cuh"]


PF_KERNEL_SOURCES = ["quantized_moe_expert_02_b200/csrc/prefill.cu",
                     "quantized_moe_expert_02_b200/csrc/tc_ptx.cuh",
                     "quantized_moe_expert_02_b200/csrc/moe_internal.cuh"]


def profile_values(name: str, sources):
    """The `key: value` lines of a committed ncu summary under profiles/,
    or None when it is missing or the kernel sources changed since it was
    taken (its source_sha is the sha256 of the sources' digest lines)."""
    import hashlib
    prof = os.path.join(ROOT, "profiles", name)
    if not os.path.exists(prof):
        return None
    vals = {}
    for line in open(prof):
        if ":" in line and not line.startswith(("#", "|", " ")):
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip()
    digests = []
    for f in sources:
        digests.append(hashlib.sha256(open(os.path.join(ROOT, f), "rb")
                                      .read()).hexdigest() + "  " + f)
    sha = hashlib.sha256(("\n".join(digests) + "\n").encode()).hexdigest()
    if vals.get("source_sha") != sha[:16]:
        return None
    return vals


def captured_traffic(alg_bytes_per_launch: float):
    """DRAM traffic per launch from the committed ncu capture of the decode
    kernel, scaled from the captured launch's algorithmic bytes to the
    bench's average launch; None when the kernel sources changed since."""
    vals = profile_values("decode_layer_t3.md", KERNEL_SOURCES)
    if vals is None:
        return None
    t = float(vals["traffic_bytes_per_launch"])
    a = float(vals["algorithmic_bytes_of_captured_launch"])
    return t * alg_bytes_per_launch / a


def captured_traffic_prefill():
    """DRAM traffic of one up/gate launch of the prefill chunk from the
    committed ncu capture (same workload); None when stale."""
    vals = profile_values("pf_gemm_prefill_9536.md", PF_KERNEL_SOURCES)
    return None if vals is None else float(vals["traffic_bytes_per_launch"])


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], "measured"
    return 6650.0, 1590.0, "fallback"


# ------------------------------------------------------------ clocks ----
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.p = None

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}",
               "--format=csv,noheader,nounits", "-lms", "200"]
        if self.uuid:
            cmd += ["-i", self.uuid]
        try:
            self.p = subprocess.Popen(cmd, stdout=subprocess.PIPE,
                                      stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        try:
            out, _ = self.p.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
            out, _ = self.p.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                mx.append(float(f[1]))
            except ValueError:
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "samples": len(sm), "reasons": sorted(reasons)}


# ------------------------------------------------------------- oracle ----
def oracle_step(layer: int, step: int, T: int, tokens, n_experts=None):
    """The oracle on one decode step: routing of all T tokens, then the
    expert FFNs and combine of `tokens` (all k experts each, or only the
    first n_experts of one token).  Returns the number of tokens computed
    (fractional when a token is sampled)."""
    import oracle as o
    shp = synth.BIG
    x = o.bf16_to_f64(synth.gen_x(SEED, T, shp.H, step))
    wr = o.bf16_to_f64(synth.gen_router(SEED, layer, shp.E, shp.H))
    src = o.ExpertSource(shp.H, shp.F, shp.fmt_up_gate, shp.fmt_down,
                         lambda e: synth.gen_expert_blob(shp, SEED, layer, e))
    logits = o.router_logits(x, wr, None)
    idx, w = o.route(logits, shp.k)
    done = 0.0
    for t in tokens:
        js = range(shp.k if n_experts is None else n_experts)
        out = np.zeros(shp.H)
        for j in js:
            wu, wg, wd = src.weights(int(idx[t, j]))
            _, y = o.expert_ffn(x[t:t + 1], wu, wg, wd)
            out += w[t, j] * y[0]
        done += len(js) / shp.k
    return done


def cpu_baseline_prefill(n_tokens: int = 4) -> dict:
    """The oracle on a bounded sample of the prefill chunk: routing (with
    the layer's Zipf bias) and the whole expert FFN + combine of its first
    `n_tokens` tokens."""
    import oracle as o
    shp = synth.BIG
    t0 = time.perf_counter()
    x = o.bf16_to_f64(synth.gen_x(SEED, PF_T, shp.H, 0)[:n_tokens])
    wr = o.bf16_to_f64(synth.gen_router(SEED, 0, shp.E, shp.H))
    bias = synth.gen_zipf_bias(SEED, 0, shp.E)[0]
    src = o.ExpertSource(shp.H, shp.F, shp.fmt_up_gate, shp.fmt_down,
                         lambda e: synth.gen_expert_blob(shp, SEED, 0, e))
    o.moe_layer(x, wr, bias, shp.k, src)
    dt = time.perf_counter() - t0
    return {"value": n_tokens / dt, "unit": "tokens/s",
            "cores": blas_threads(), "kind": "oracle",
            "sample": (f"the first {n_tokens} tokens of the {PF_T}-token "
                       f"prefill chunk: fp64 routing with the Zipf bias, "
                       f"dequantisation and fp64 SwiGLU FFN of their chosen "
                       f"experts, combine ({dt:.1f} s)")}


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info()
             if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(T: int, seconds: float = 10.0) -> dict:
    """The oracle on whole T-token decode steps (the layers rotated as in
    the GPU measurement) until about `seconds` of host time have passed."""
    t0 = time.perf_counter()
    done, n = 0.0, 0
    while True:
        done += oracle_step(layer=n % 8, step=n, T=T, tokens=range(T))
        n += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    steps = (f"one whole {T}-token decode step of layer 0" if n == 1 else
             f"{n} whole {T}-token decode steps (layers 0..{min(n, 8) - 1} "
             f"in turn)")
    return {"value": done / dt, "unit": "tokens/s", "cores": blas_threads(),
            "kind": "oracle",
            "sample": (f"{steps}: fp64 routing of all {T} tokens, then "
                       f"dequantisation and fp64 SwiGLU FFN of every chosen "
                       f"expert and the combine ({dt:.1f} s)")}


def run_reference(args) -> None:
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    # bounded sample per step: one token's first n experts, n sized so
    # that warm-up + steps stay within ~3 minutes
    t0 = time.perf_counter()
    oracle_step(0, 0, args.T, tokens=[0], n_experts=1)
    per_expert = time.perf_counter() - t0
    budget = 180.0 / max(1, args.steps + args.warmup)
    n = int(max(1, min(synth.BIG.k, budget // max(per_expert, 1e-3))))
    for i in range(args.warmup):
        oracle_step(i % args.layers, i, args.T, tokens=[i % args.T],
                    n_experts=n)
    t0 = time.perf_counter()
    done = 0.0
    for i in range(args.steps):
        s = args.warmup + i
        done += oracle_step(s % args.layers, s, args.T, tokens=[s % args.T],
                            n_experts=n)
    dt = time.perf_counter() - t0
    v = done / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": workload_config(args),
        "cpu_baseline": {"value": v, "unit": "tokens/s",
                         "cores": blas_threads(), "kind": "oracle",
                         "sample": (f"per step: routing of a {args.T}-token "
                                    f"decode step, then {n} of the k=10 "
                                    f"experts of one token (fp64 dequant + "
                                    f"SwiGLU FFN); counted as {n}/10 token")},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(args) -> dict:
    return {"workload": (f"decode, one MoE layer: {args.T} tokens, hidden "
                         f"3072, expert FFN 1024, 512 experts, top-10, SB3 "
                         f"up/gate + NL4 down"),
            "T": args.T, "H": 3072, "F": 1024, "E": 512, "k": 10,
            "layers_rotated": args.layers,
            "l2": (f"inputs larger than L2: steps rotate over {args.layers} "
                   f"resident layers x {synth.BIG.E * synth.BIG.blob_stride / 1e9:.2f}"
                   f" GB of experts"),
            "parallelism": f"replicas x{args.gpus}", "seed": SEED}


# ---------------------------------------------------------------- GPU ----
class Layers:
    """Resident layers (packed expert pools, router weights) and the
    per-T step buffers."""

    def __init__(self, L: int, n_x: int = 64, shape=None):
        import torch
        from synth.pools import build_pool, dev, layer_desc
        import quantized_moe_expert_02_b200 as moe
        self.moe, self.torch, self.dev = moe, torch, dev
        shp = self.shape = synth.BIG if shape is None else shape
        self.L, self.n_x = L, n_x
        self.pools = [build_pool(shp, SEED, l) for l in range(L)]
        self.descs = [layer_desc(shp, p) for p in self.pools]
        self.wr = [dev(synth.gen_router(SEED, l, shp.E, shp.H))
                   for l in range(L)]
        self.bufs = {}

    def buffers(self, T: int):
        if T in self.bufs:
            return self.bufs[T]
        torch, moe, shp = self.torch, self.moe, self.shape
        b = {}
        b["xs"] = [self.dev(synth.gen_x(SEED, T, shp.H, s))
                   for s in range(self.n_x)]
        b["ws_bytes"] = moe.moe_layer_workspace_bytes(T, shp.k, shp.E, shp.H,
                                                      shp.F)
        b["ws"] = torch.zeros(b["ws_bytes"], dtype=torch.uint8, device="cuda")
        b["idx"] = torch.empty((T, shp.k), dtype=torch.int32, device="cuda")
        b["w"] = torch.empty((T, shp.k), device="cuda")
        b["out"] = torch.empty((T, shp.H), device="cuda")
        b["ffn_ws_bytes"] = moe.moe_ffn_workspace_bytes(T, shp.k, shp.H, shp.F)
        b["ffn_ws"] = torch.zeros(b["ffn_ws_bytes"], dtype=torch.uint8,
                                  device="cuda")
        b["gws_bytes"] = moe.moe_group_workspace_bytes(T, shp.k, shp.E)
        b["gws"] = torch.zeros(b["gws_bytes"], dtype=torch.uint8,
                               device="cuda")
        b["lg"] = torch.empty((T, shp.E), device="cuda")
        b["off"] = torch.empty(shp.E + 1, dtype=torch.int32, device="cuda")
        b["pairs"] = torch.empty(T * shp.k, dtype=torch.int32, device="cuda")
        b["act"] = torch.empty(shp.E, dtype=torch.int32, device="cuda")
        b["na"] = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.bufs[T] = b
        return b

    def step(self, T: int, i: int, x=None, out=None):
        """One decode layer through the C ABI (one launch)."""
        b, shp = self.buffers(T), self.shape
        l = i % self.L
        xx = b["xs"][i % self.n_x] if x is None else x
        self.moe.moe_layer_forward(self.descs[l], xx, T, shp.k, self.wr[l],
                                   None, None, None,
                                   b["out"] if out is None else out, None,
                                   b["idx"], b["w"], None, b["ws"],
                                   b["ws_bytes"])

    def unique_experts(self, T: int, i: int) -> int:
        """Distinct experts of step i (untimed: routing only)."""
        b, shp = self.buffers(T), self.shape
        l = i % self.L
        self.moe.moe_route_topk(b["xs"][i % self.n_x], T, shp.H, self.wr[l],
                                shp.E, None, shp.k, b["idx"], b["w"], b["lg"])
        return int(self.torch.unique(b["idx"]).numel())


def graph_time(steps: int, warmup: int, fn, per_graph: int) -> float:
    """Device time (ms) of `steps` calls fn(i), replayed from CUDA graphs of
    `per_graph` steps, after `warmup` eager steps and one graph warm-up."""
    import torch
    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize()
    G = min(per_graph, steps)
    full, rem = divmod(steps, G)
    graphs = []
    for n, reps in ((G, full), (rem, 1 if rem else 0)):
        if not reps:
            continue
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(n):
                fn(warmup + i)
        graphs.append((g, reps))
    for g, _ in graphs:
        g.replay()
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for g, reps in graphs:
        for _ in range(reps):
            g.replay()
    e1.record(s)
    e1.synchronize()
    ms = e0.elapsed_time(e1)
    del graphs
    return ms


def prefill_e2e_time(pf, steps: int, warmup: int) -> float:
    """Device time (ms) per prefill step end to end through the C ABI:
    every step copies its x (9536 x 3072 bf16) from pinned host memory and
    its output (fp32) back to pinned host memory, on two copy streams
    beside the layer launches (x of step i+1 goes up while step i computes,
    the output of step i comes back while step i+1 computes)."""
    import torch
    H = synth.BIG.H
    xh = [torch.from_numpy(synth.gen_x(SEED, pf.T, H, s).view(np.int16))
          .pin_memory() for s in range(2)]
    oh = [torch.empty((pf.T, H), dtype=torch.float32).pin_memory()
          for _ in range(2)]
    xd = [torch.empty((pf.T, H), dtype=torch.int16, device="cuda")
          for _ in range(2)]
    od = [torch.empty((pf.T, H), device="cuda") for _ in range(2)]
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    cur = torch.cuda.current_stream()

    def run(n: int):
        up.wait_stream(cur)
        down.wait_stream(cur)
        ev_in, ev_k, ev_out = {}, {}, {}
        for j in range(n):
            b = j % 2
            with torch.cuda.stream(up):
                if j >= 2:
                    up.wait_event(ev_k[j - 2])
                xd[b].copy_(xh[b], non_blocking=True)
                ev_in[j] = torch.cuda.Event()
                ev_in[j].record(up)
            cur.wait_event(ev_in[j])
            if j >= 2:
                cur.wait_event(ev_out[j - 2])
            pf.step(x=xd[b], out=od[b])
            ev_k[j] = torch.cuda.Event()
            ev_k[j].record(cur)
            with torch.cuda.stream(down):
                down.wait_event(ev_k[j])
                oh[b].copy_(od[b], non_blocking=True)
                ev_out[j] = torch.cuda.Event()
                ev_out[j].record(down)
        cur.wait_stream(up)
        cur.wait_stream(down)

    run(warmup)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(cur)
    run(steps)
    e1.record(cur)
    e1.synchronize()
    return e0.elapsed_time(e1) / steps


def e2e_time(lay, T: int, steps: int, warmup: int) -> float:
    """Device time (ms) of `steps` decode steps end to end through the C
    ABI: every step copies its x from pinned host memory to the device and
    its output back to pinned host memory.  The copies run on two copy
    streams beside the layer launches (x of step i+1 goes up while step i
    computes; the output of step i comes back while step i+1 computes),
    with triple-buffered device x and output, so a launch waits only on
    copies two steps back.  Replayed from CUDA graphs of 32 steps."""
    import torch
    H = synth.BIG.H
    nh = lay.L * 4
    xh = [torch.from_numpy(synth.gen_x(SEED, T, H, s).view(np.int16))
          .pin_memory() for s in range(nh)]
    oh = [torch.empty((T, H), dtype=torch.float32).pin_memory()
          for _ in range(nh)]
    NB = 3
    xd = [torch.empty((T, H), dtype=torch.int16, device="cuda")
          for _ in range(NB)]
    od = [torch.empty((T, H), device="cuda") for _ in range(NB)]
    up, down = torch.cuda.Stream(), torch.cuda.Stream()

    def body(i0: int, n: int):
        cur = torch.cuda.current_stream()
        up.wait_stream(cur)
        down.wait_stream(cur)
        ev_in, ev_k, ev_out = {}, {}, {}
        for j in range(n):
            i, b = i0 + j, j % NB
            with torch.cuda.stream(up):
                if j >= NB:
                    up.wait_event(ev_k[j - NB])     # step j-NB read xd[b]
                xd[b].copy_(xh[i % nh], non_blocking=True)
                ev_in[j] = torch.cuda.Event()
                ev_in[j].record(up)
            cur.wait_event(ev_in[j])
            if j >= NB:
                cur.wait_event(ev_out[j - NB])      # od[b] is back on host
            lay.step(T, i, x=xd[b], out=od[b])
            ev_k[j] = torch.cuda.Event()
            ev_k[j].record(cur)
            with torch.cuda.stream(down):
                down.wait_event(ev_k[j])
                oh[i % nh].copy_(od[b], non_blocking=True)
                ev_out[j] = torch.cuda.Event()
                ev_out[j].record(down)
        cur.wait_stream(up)
        cur.wait_stream(down)

    body(0, max(warmup, NB))
    torch.cuda.synchronize()
    G = min(32, steps)
    full, rem = divmod(steps, G)
    graphs = []
    for n, reps in ((G, full), (rem, 1 if rem else 0)):
        if not reps:
            continue
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            body(warmup, n)
        graphs.append((g, reps))
    for g, _ in graphs:
        g.replay()
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for g, reps in graphs:
        for _ in range(reps):
            g.replay()
    e1.record(s)
    e1.synchronize()
    ms = e0.elapsed_time(e1)
    del graphs
    return ms


def kernel_timing(lay, T, steps, warmup):
    """Average device time of one layer launch (the one-kernel decode
    layer), timed with CUDA events around its C-ABI call; a spin kernel
    keeps the GPU busy while the host enqueues, so no host latency falls
    between the events."""
    import torch
    s = torch.cuda.current_stream()
    tot = 0.0
    for i in range(warmup + steps):
        torch.cuda._sleep(200000)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        ev[0].record(s)
        lay.step(T, i)
        ev[1].record(s)
        ev[1].synchronize()
        if i >= warmup:
            tot += ev[0].elapsed_time(ev[1])
    return tot / steps


def decode_measure(lay, T, K, W):
    """tokens/s, ms/step and layer GB/s of K decode steps (graph replay)."""
    uniq = [lay.unique_experts(T, W + i) for i in range(min(K, lay.L * 4))]
    u_avg = sum(uniq) / len(uniq)
    ms = graph_time(K, W, lambda i: lay.step(T, i), per_graph=lay.L * 4)
    bytes_step = WR_BYTES + u_avg * lay.shape.blob_bytes + T * 3072 * 6
    hbm, _, _ = peaks()
    gbs = bytes_step / (ms / K * 1e-3) / 1e9
    return {"tokens_per_s": T * K / (ms / 1e3), "ms_per_step": ms / K,
            "layer_gbs": gbs, "frac_of_hbm": gbs / hbm,
            "unique_experts_per_step": u_avg}, ms


def decode_sweep(lay, W: int, steps: int = 2048) -> dict:
    """The one-kernel decode layer at every token count it serves (1..8):
    per-layer time, tokens/s and the fraction of measured HBM bandwidth of
    its algorithmic bytes (same resident layers, graph replay)."""
    out = {}
    for T in range(1, 9):
        d, _ = decode_measure(lay, T, steps, W)
        out[str(T)] = {"us_per_layer": d["ms_per_step"] * 1e3,
                       "tokens_per_s": d["tokens_per_s"],
                       "frac_of_hbm": d["frac_of_hbm"],
                       "unique_experts": d["unique_experts_per_step"]}
    return out


def clock_soak(lay, T: int, ms_per_step: float, seconds: float = 1.0):
    """nvidia-smi clock samples over about `seconds` of the same decode
    steps (graph replays): the timed region itself may be too short for
    the 200 ms sampler."""
    import torch
    props = torch.cuda.get_device_properties(torch.cuda.current_device())
    uuid = getattr(props, "uuid", None)
    clk = ClockSampler(f"GPU-{uuid}" if uuid else None)
    n = max(lay.L * 4, int(seconds / max(ms_per_step * 1e-3, 1e-6)))
    clk.start()
    graph_time(n, 0, lambda i: lay.step(T, i), per_graph=lay.L * 4)
    out = clk.stop()
    if out is not None:
        out["steps"] = n
    return out


ALT_UP_GATE = {"nl3": (synth.NL3_256, "NL3"), "sb2": (synth.SB2_256, "SB2")}


def alt_decode(T: int, K: int, W: int, which: str) -> dict:
    """The decode layer with up/gate in another format -- the 3-bit
    non-uniform-codebook super-block (NL3) or the 2-bit super-block (SB2) --
    at the 512-expert shape: two resident layers rotated."""
    import torch
    fmt, name = ALT_UP_GATE[which]
    shape = dataclasses.replace(synth.BIG, fmt_up_gate=fmt)
    lay = Layers(2, shape=shape)
    d, _ = decode_measure(lay, T, K, W)
    d["workload"] = (f"decode, one MoE layer: {T} tokens, 512 experts "
                     f"top-10, {name} up/gate + NL4 down")
    d["blob_bytes"] = shape.blob_bytes
    del lay
    torch.cuda.empty_cache()
    return d


def prefill_slots_measure(pool, cap: int = 92, borrow: int = 8,
                          l: int = 0) -> dict:
    """The prefill chunk through one layer's slot partition (`cap` slots
    holding the layer's hottest experts, `borrow` of them borrowed), the
    misses streamed from a pinned host store: device time of one call and
    bit-exactness against the all-resident layer."""
    import torch
    from synth.pools import dev, layer_desc
    from synth.prefill_slots import Partition, PrefillSlots
    import quantized_moe_expert_02_b200 as moe
    shp, T = synth.BIG, PF_T
    _, rank = synth.gen_zipf_bias(SEED, l, shp.E)
    part = Partition(shp, pool, synth.hottest_experts(rank, cap), cap)
    store = torch.empty((shp.E, shp.blob_bytes), dtype=torch.uint8)
    store = store.pin_memory()
    for e in range(shp.E):
        o = e * shp.blob_stride
        store[e].copy_(pool[o:o + shp.blob_bytes])
    ps = PrefillSlots(shp, part, store, {e: e for e in range(shp.E)}, T,
                      borrow=borrow)
    pf = Prefill(pool, layer_desc(shp, pool), l)
    pf.step()
    out = torch.empty((T, shp.H), device="cuda")
    ps.forward(pf.x, pf.wr, pf.bias, out)          # warm
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    stats = ps.forward(pf.x, pf.wr, pf.bias, out)
    e1.record()
    e1.synchronize()
    ms = e0.elapsed_time(e1)
    exact = bool(torch.equal(out, pf.out))
    del ps, part, store, pf
    torch.cuda.empty_cache()
    return {"workload": (f"prefill chunk ({T} tokens) through one layer's "
                         f"{cap}-slot partition, {borrow} slots borrowed, "
                         "misses streamed from pinned host memory"),
            "ms_per_step": ms, "tokens_per_s": T / (ms / 1e3),
            "chosen_experts": stats["chosen"], "hits": stats["hits"],
            "misses": stats["misses"], "waves": stats["waves"],
            "h2d_bytes": stats["h2d_bytes"],
            "h2d_gbs": stats["h2d_bytes"] / (ms * 1e-3) / 1e9,
            "bit_exact_vs_resident": exact}


# -------------------------------------------------------------- prefill ---
PF_T = synth.WORKLOADS["prefill"].T


def prefill_flops(T: int) -> dict:
    shp = synth.BIG
    P = T * shp.k
    up = P * 4 * shp.F * shp.H
    down = P * 2 * shp.H * shp.F
    router = 2 * T * shp.E * shp.H
    return {"up": up, "down": down, "router": router,
            "total": up + down + router}


class Prefill:
    """One prefill chunk (9536 tokens, Zipf(1.1)-biased routing) on one
    resident layer, through the C ABI."""

    def __init__(self, pool, desc, l: int = 0, T: int = PF_T):
        import torch
        from synth.pools import dev
        import quantized_moe_expert_02_b200 as moe
        shp = synth.BIG
        self.moe, self.torch, self.T = moe, torch, T
        self.desc = desc
        self.x = dev(synth.gen_x(SEED, T, shp.H, 0))
        self.wr = dev(synth.gen_router(SEED, l, shp.E, shp.H))
        self.bias = dev(synth.gen_zipf_bias(SEED, l, shp.E)[0])
        k, E, H, F = shp.k, shp.E, shp.H, shp.F
        self.ws_bytes = moe.moe_layer_workspace_bytes(T, k, E, H, F)
        self.ws = torch.zeros(self.ws_bytes, dtype=torch.uint8, device="cuda")
        self.idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
        self.w = torch.empty((T, k), device="cuda")
        self.lg = torch.empty((T, E), device="cuda")
        self.out = torch.empty((T, H), device="cuda")
        # pieces
        self.off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
        self.pairs = torch.empty(T * k, dtype=torch.int32, device="cuda")
        self.act = torch.empty(E, dtype=torch.int32, device="cuda")
        self.na = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.gws_bytes = moe.moe_group_workspace_bytes(T, k, E)
        self.gws = torch.zeros(self.gws_bytes, dtype=torch.uint8,
                               device="cuda")
        self.fws_bytes = moe.moe_ffn_workspace_bytes(T, k, H, F)
        self.fws = torch.zeros(self.fws_bytes, dtype=torch.uint8,
                               device="cuda")
        self.y = torch.empty((T * k, H), device="cuda")

    def step(self, x=None, out=None):
        shp = synth.BIG
        self.moe.moe_layer_forward(self.desc, self.x if x is None else x,
                                   self.T, shp.k, self.wr, self.bias, None,
                                   None, self.out if out is None else out,
                                   None, self.idx, self.w, self.lg, self.ws,
                                   self.ws_bytes)

    def piece_fns(self):
        moe, shp, T = self.moe, synth.BIG, self.T
        k, E, H = shp.k, shp.E, shp.H
        return {
            "route": lambda: moe.moe_route_topk(self.x, T, H, self.wr, E,
                                                self.bias, k, self.idx,
                                                self.w, self.lg),
            "group": lambda: moe.moe_group_tokens(self.idx, T, k, E, self.off,
                                                  self.pairs, self.act,
                                                  self.na, self.gws,
                                                  self.gws_bytes),
            "up": lambda: moe.moe_expert_up_q(self.desc, self.x, T, k,
                                              self.off, self.pairs, self.act,
                                              self.na, None, self.fws,
                                              self.fws_bytes),
            "up_gemm": lambda: moe.moe_expert_up_gemm_q(
                self.desc, T, k, self.off, self.pairs, self.act, self.na,
                None, self.fws, self.fws_bytes),
            "down": lambda: moe.moe_expert_down_q(self.desc, T, k, self.off,
                                                  self.pairs, self.act,
                                                  self.na, None, self.y, None,
                                                  None, None, None, self.fws,
                                                  self.fws_bytes),
            "combine": lambda: moe.moe_combine(self.y, self.w, T, k, H, None,
                                               self.out, None),
        }


def events_time(fn, steps: int, warmup: int) -> float:
    """Average device ms of fn() over `steps` back-to-back calls (CUDA
    events on the launching stream, after `warmup` calls)."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(steps):
        fn()
    e1.record(s)
    e1.synchronize()
    return e0.elapsed_time(e1) / steps


def prefill_measure(pf: "Prefill", steps: int, warmup: int) -> dict:
    """Whole prefill layer (tokens/s, TFLOP/s) and its parts."""
    fl = prefill_flops(pf.T)
    ms = events_time(pf.step, steps, warmup)
    parts = {}
    for name, fn in pf.piece_fns().items():
        parts[name] = events_time(fn, max(2, steps // 2), 2)
    _, tf, _ = peaks()
    return {
        "workload": (f"prefill chunk, one MoE layer: {pf.T} tokens, "
                     "Zipf(1.1)-biased routing, 512 experts top-10"),
        "tokens_per_s": pf.T / (ms / 1e3), "ms_per_step": ms,
        "tflops": fl["total"] / (ms * 1e-3) / 1e12,
        "frac_of_bf16_peak": fl["total"] / (ms * 1e-3) / 1e12 / tf,
        "parts_ms": parts,
        "up_tflops": fl["up"] / (parts["up"] * 1e-3) / 1e12,
        "up_gemm_tflops": fl["up"] / (parts["up_gemm"] * 1e-3) / 1e12,
        "up_gemm_frac_of_bf16_peak":
            fl["up"] / (parts["up_gemm"] * 1e-3) / 1e12 / tf,
        "down_tflops": fl["down"] / (parts["down"] * 1e-3) / 1e12,
        "down_frac_of_bf16_peak":
            fl["down"] / (parts["down"] * 1e-3) / 1e12 / tf,
        "expert_gemms_frac_of_bf16_peak":
            (fl["up"] + fl["down"]) /
            ((parts["up_gemm"] + parts["down"]) * 1e-3) / 1e12 / tf,
        "router_tflops": fl["router"] / (parts["route"] * 1e-3) / 1e12,
        "flops_per_step": fl,
    }


def prefill_sweep(pool, sizes=(1024, 2048, 4096, 9536, 16384, 32768),
                  steps: int = 5) -> dict:
    """The prefill layer at other chunk sizes (same layer, same Zipf-biased
    routing): per-layer time, tokens/s and the fraction of the measured
    bf16 peak of its FLOPs (expert GEMMs and router)."""
    import torch
    from synth.pools import layer_desc
    _, tf, _ = peaks()
    out = {}
    for T in sizes:
        pf = Prefill(pool, layer_desc(synth.BIG, pool), T=T)
        ms = events_time(pf.step, steps, 2)
        fl = prefill_flops(T)
        out[str(T)] = {"ms_per_layer": ms, "tokens_per_s": T / (ms / 1e3),
                       "frac_of_bf16_peak":
                           fl["total"] / (ms * 1e-3) / 1e12 / tf}
        del pf
        torch.cuda.empty_cache()
    return out


def run_profile(args) -> None:
    """Launches for ncu: W warm-up steps then K steps, eager (5 kernels
    each), nothing else on the GPU after the pools are built."""
    import torch
    if args.workload == "prefill":
        from synth.pools import build_pool, layer_desc
        pool = build_pool(synth.BIG, SEED, 0)
        pf = Prefill(pool, layer_desc(synth.BIG, pool))
        for i in range(args.warmup + args.steps):
            pf.step()
        torch.cuda.synchronize()
        print("profile run done", flush=True)
        return
    lay = Layers(args.layers)
    for i in range(args.warmup + args.steps):
        lay.step(args.T, i)
    torch.cuda.synchronize()
    print("profile run done", flush=True)


def max_over_ranks(ms: float, dist, device: str) -> float:
    """The job's time: the largest of the ranks' device times (every rank
    calls this at the same point; a no-op for one process)."""
    if dist is None:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank: float, world: int, ms: float) -> float:
    """Whole-job throughput: the units all ranks processed (replicas, so
    each did the same) over the job's time in ms."""
    return units_per_rank * world / (ms / 1e3)


def run_ours(args) -> None:
    import torch
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    lay = Layers(args.layers)
    T, K, W = args.T, args.steps, args.warmup
    uniq = [lay.unique_experts(T, W + i) for i in range(min(K, lay.L * 4))]
    u_avg = sum(uniq) / len(uniq)
    for i in range(W):
        lay.step(T, i)
    torch.cuda.synchronize()

    props = torch.cuda.get_device_properties(local)
    uuid = getattr(props, "uuid", None)
    clk = ClockSampler(f"GPU-{uuid}" if uuid else None)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    clk.start()
    ms = graph_time(K, W, lambda i: lay.step(T, i), per_graph=lay.L * 4)
    clocks = clk.stop()
    ms = max_over_ranks(ms, dist, "cuda")
    tok_s = job_rate(T * K, world, ms)
    bytes_step = WR_BYTES + u_avg * BLOB + T * 3072 * 6

    line = None
    if rank == 0:
        hbm, tf, src = peaks()
        # the step is one launch of the layer kernel: its average launch
        # duration over the timed region is ms / K; a launch timed alone
        # (behind a spin kernel) is reported beside it
        kt = kernel_timing(lay, T, 64, 4)
        k_ms = ms / K
        k_gbs = bytes_step / (k_ms * 1e-3) / 1e9
        ms_e2e = e2e_time(lay, T, K, W)
        t1, _ = decode_measure(lay, 1, K, W)
        line = {
            "metric": METRIC, "value": tok_s, "unit": "tokens/s",
            "n_gpus": world, "steps": K, "warmup": W,
            "ms_per_step": ms / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "int8 mma (s32 accumulate) + f32",
            "data": "synthetic",
            "config": workload_config(args),
            "layer_gbs": bytes_step / (ms / K * 1e-3) / 1e9,
            "layer_frac_of_hbm": bytes_step / (ms / K * 1e-3) / 1e9 / hbm,
            "roofline": {
                "bound": "hbm",
                "kernel": "decode_layer_kernel (the whole layer, one launch)",
                "achieved": k_gbs, "peak": hbm, "unit": "GB/s",
                "frac": k_gbs / hbm, "peak_source": src,
                "traffic": captured_traffic(bytes_step),
                "algorithmic_bytes_per_launch": bytes_step,
                "avg_launch_ms": k_ms, "single_launch_ms": kt},
            "unique_experts_per_step": u_avg,
            "decode_t1": t1,
            "e2e": {"value": T * K / (ms_e2e / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": T * 3072 * 2,
                    "d2h_bytes_per_step": T * 3072 * 4},
            "gpu_launches": LAUNCHES_PER_STEP * K,
            "clocks": clocks,
        }
        line["clocks_soak"] = clock_soak(lay, T, ms / K)
        if world == 1 and not args.no_extras:
            line["decode_sweep"] = decode_sweep(lay, W)
        if not args.no_prefill:
            pf = Prefill(lay.pools[0], lay.descs[0])
            line["prefill"] = prefill_measure(pf, 10, 3)
            del pf
            torch.cuda.empty_cache()
            if world == 1:
                line["prefill"]["through_slots"] = prefill_slots_measure(
                    lay.pools[0])
        if world == 1 and not args.no_extras:
            line["decode_nl3"] = alt_decode(T, 4096, W, "nl3")
            line["decode_sb2"] = alt_decode(T, 4096, W, "sb2")
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(T)
            line["speedup_vs_cpu_baseline"] = \
                tok_s / line["cpu_baseline"]["value"]
        if world == 1 and not args.no_extras:
            del lay
            torch.cuda.empty_cache()
            res = stack_measure(args.stack_steps, 3, 2, 8.0, False)
            line["stack"] = {
                "workload": ("decode, 48-layer MoE stack: 3 tokens per step,"
                             " Zipf(1.1) routing bias, residual add; all "
                             "48 x 512 experts resident, one CUDA graph per"
                             " step"),
                "steps": res["S"], "tokens_per_s": res["tokens_per_s"],
                "ms_per_step": res["ms_per_step"], "layer_gbs": res["gbs"],
                "frac_of_hbm": res["frac"],
                "unique_experts_per_layer_step": res["u_avg"],
                "graph_replay_matches_eager":
                    res["graph_replay_matches_eager"],
                "slot_cache": {
                    "capacities": res["slot_capacities"],
                    "steps": res["slot_cache_in_stream"]["steps"],
                    "in_stream_tokens_per_s":
                        res["slot_cache_in_stream"]["tokens_per_s"],
                    "one_graph_per_step_tokens_per_s":
                        res["slot_cache_in_stream"]["graph"]["tokens_per_s"],
                    "fused_pull_one_graph_per_step_tokens_per_s":
                        res["slot_cache_in_stream"]["fused_graph"][
                            "tokens_per_s"],
                    "bit_exact_vs_resident":
                        res["slot_cache_in_stream"]["bit_exact_vs_resident"]
                        and res["slot_cache_in_stream"]["graph"][
                            "bit_exact_vs_resident"]
                        and res["slot_cache_in_stream"]["fused_graph"][
                            "bit_exact_vs_resident"]},
                "clocks": res["clocks"]}
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


def stack_measure(S: int, W: int, reps: int, store_gb: float,
                  host_roundtrip: bool = True) -> dict:
    """The 48-layer decode stack (3 tokens per step, Zipf-biased routing,
    residual add between layers) over S steps.  All 48 x 512 experts
    resident (105 GB), one CUDA graph per step; then the same steps through
    the expert-slot pool (240 / 92 / 60 slots per layer, 19.9 GB), misses
    from a pinned host store -- after a host round trip per layer (if
    host_roundtrip), pulled in-stream eagerly, and as one captured graph
    per step -- each checked bit-exact against the resident run."""
    import torch
    from synth.stack import SlotPool, Stack
    L, T = 48, 3
    shp = synth.BIG
    t0 = time.perf_counter()
    st = Stack(L, shp, seed=SEED, T=T)
    setup_s = time.perf_counter() - t0
    xs = [st.x0(s) for s in range(S)]
    r = torch.empty_like(xs[0])
    # untimed pass: unique experts per (step, layer) and the resident outputs
    uniq, ref = [], []
    for s in range(S):
        r.copy_(xs[s])
        rec = []
        st.run_resident(r, record=rec)
        uniq.append([int(torch.unique(i).numel()) for i in rec])
        ref.append(r.clone())
    u_avg = float(np.mean(uniq))
    bytes_step = L * WR_BYTES + float(np.sum(uniq)) / S * BLOB + \
        L * T * 3072 * 6
    # resident stack, one CUDA graph per step
    graphs = []
    for s in range(S):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            r.copy_(xs[s])
            st.run_resident(r)
        graphs.append(g)
    for i in range(W):
        graphs[i % S].replay()
    torch.cuda.synchronize()
    props = torch.cuda.get_device_properties(0)
    uuid = getattr(props, "uuid", None)
    clk = ClockSampler(f"GPU-{uuid}" if uuid else None)
    clk.start()
    reps = max(1, reps)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        for g in graphs:
            g.replay()
    e1.record()
    e1.synchronize()
    clocks = clk.stop()
    ms = e0.elapsed_time(e1) / reps
    graphs[-1].replay()
    torch.cuda.synchronize()
    same_resident = bool(torch.equal(r, ref[-1]))
    del graphs
    # slot cache: a discovery run (misses copied from the resident pools)
    # tells which blobs the pinned host store must hold
    caps = [synth.slot_capacity(l) for l in range(L)]
    disc = SlotPool(st, caps, None)
    max_blobs = int(store_gb * 1e9 // shp.blob_bytes)
    S4 = 0   # slot-cache steps: the longest prefix whose misses fit the store
    for s in range(S):
        r.copy_(xs[s])
        before = set(disc.seen_keys)
        disc.run(r, s + 1)
        if len(disc.seen_keys) > max_blobs:
            disc.seen_keys = before
            break
        S4 = s + 1
    keys = sorted(disc.seen_keys)
    del disc
    torch.cuda.empty_cache()
    t0 = time.perf_counter()
    pool = SlotPool(st, caps, keys)
    store_s = time.perf_counter() - t0
    hbm, tf, src = peaks()
    gbs = bytes_step / (ms / S * 1e-3) / 1e9
    res = {"S": S, "ms": ms, "ms_per_step": ms / S,
           "tokens_per_s": T * S / (ms / 1e3), "gbs": gbs,
           "frac": gbs / hbm, "peak": hbm, "peak_source": src,
           "bytes_step": bytes_step, "u_avg": u_avg,
           "graph_replay_matches_eager": same_resident, "setup_s": setup_s,
           "clocks": clocks}
    if host_roundtrip:
        outs = []
        torch.cuda.synchronize()
        e0.record()
        t0 = time.perf_counter()
        for s in range(S4):
            r.copy_(xs[s])
            pool.run(r, s + 1)
            outs.append(r.clone())
        e1.record()
        e1.synchronize()
        slot_ms = e0.elapsed_time(e1)
        slot_wall = time.perf_counter() - t0
        bit_exact = all(torch.equal(a, b) for a, b in zip(outs, ref[:S4]))
        res["slot_cache"] = {
            "steps": S4,
            "tokens_per_s": T * S4 / (slot_ms / 1e3),
            "ms_per_step": slot_ms / max(1, S4), "wall_s": slot_wall,
            "capacities": "240 (layers 0-4), 92 (5-31), 60 (32-47)",
            "misses": pool.misses,
            "miss_rate": pool.misses / float(np.sum(uniq[:S4])),
            "h2d_bytes": pool.misses * shp.blob_bytes,
            "host_store_blobs": len(keys),
            "host_store_build_s": store_s,
            "bit_exact_vs_resident": bit_exact}
        del outs
    # the misses pulled from the pinned host store by the library on the
    # stream itself: no host sync per layer
    pool.reset()
    pool.start_staging()
    for s in range(min(S4, W)):          # untimed: the launch path warm
        r.copy_(xs[s])
        pool.run_staged(r)
    pool.reset()
    torch.cuda.synchronize()
    outs = []
    e0.record()
    for s in range(S4):
        r.copy_(xs[s])
        pool.run_staged(r)
        outs.append(r.clone())
    e1.record()
    e1.synchronize()
    db_ms = e0.elapsed_time(e1)
    db_exact = all(torch.equal(a, b) for a, b in zip(outs, ref[:S4])) and \
        int(pool.err.item()) == 0
    # the same steps, each one replay of one captured CUDA graph (the slot
    # state and the LRU stamps live on the device)
    pool.reset()
    x_in = torch.empty_like(xs[0])
    g = pool.capture_step(x_in, r)
    torch.cuda.synchronize()
    outs = []
    e0.record()
    for s in range(S4):
        x_in.copy_(xs[s])
        g.replay()
        outs.append(r.clone())
    e1.record()
    e1.synchronize()
    gr_ms = e0.elapsed_time(e1)
    gr_exact = all(torch.equal(a, b) for a, b in zip(outs, ref[:S4])) and \
        int(pool.err.item()) == 0
    del outs, g
    # the pull inside each layer's FFN launch, overlapping the hit experts'
    # compute, replayed as one graph per step
    import quantized_moe_expert_02_b200 as moe
    pool.reset()
    g = pool.capture_step(x_in, r, fused=True)
    torch.cuda.synchronize()
    outs = []
    e0.record()
    for s in range(S4):
        x_in.copy_(xs[s])
        g.replay()
        outs.append(r.clone())
    e1.record()
    e1.synchronize()
    fu_ms = e0.elapsed_time(e1)
    fu_exact = all(torch.equal(a, b) for a, b in zip(outs, ref[:S4])) and \
        int(pool.err.item()) == 0 and moe.moe_get_device_status(st.ws) == 0
    del outs, g
    res["slot_cache_in_stream"] = {
        "steps": S4,
        "tokens_per_s": T * S4 / (db_ms / 1e3),
        "ms_per_step": db_ms / max(1, S4),
        "how": ("per layer on one stream: route, resolve, a kernel that "
                "pulls each missed blob from the pinned host store over "
                "PCIe into its slot, FFN; no host sync per layer"),
        "bit_exact_vs_resident": db_exact,
        "graph": {
            "tokens_per_s": T * S4 / (gr_ms / 1e3),
            "ms_per_step": gr_ms / max(1, S4),
            "how": ("the whole step (48 x route, device-stamped "
                    "resolve, pull, FFN) captured once as one CUDA "
                    "graph, one replay per step"),
            "bit_exact_vs_resident": gr_exact},
        "fused_graph": {
            "tokens_per_s": T * S4 / (fu_ms / 1e3),
            "ms_per_step": fu_ms / max(1, S4),
            "how": ("one graph per step; each layer's misses pulled by the "
                    "FFN launch itself (moe_layer_ffn_residual_staged): "
                    "the hit experts compute while every block copies its "
                    "share of the missed blobs"),
            "bit_exact_vs_resident": fu_exact}}
    res["slot_capacities"] = "240 (layers 0-4), 92 (5-31), 60 (32-47)"
    res["host_store_blobs"] = len(keys)
    del pool, st
    torch.cuda.empty_cache()
    return res


def run_stack(args) -> None:
    """`--workload stack`: the 48-layer decode stack as the headline line
    (see stack_measure)."""
    L, T, S, W = 48, 3, args.steps, args.warmup
    res = stack_measure(S, W, args.stack_reps, args.store_gb, True)
    line = {
        "metric": METRIC, "value": res["tokens_per_s"], "unit": "tokens/s",
        "n_gpus": 1, "steps": S, "warmup": W,
        "ms_per_step": res["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8 mma (s32 accumulate) + f32", "data": "synthetic",
        "config": {"workload": ("decode, 48-layer MoE stack: 3 tokens per "
                                "step, 512 experts top-10 per layer, Zipf(1.1)"
                                " routing bias, residual add (pre-norm), all "
                                "48 x 512 experts resident"),
                   "T": T, "layers": L, "H": 3072, "F": 1024, "E": 512,
                   "k": 10, "l2": "inputs larger than L2: 105 GB of experts",
                   "parallelism": "replicas x1", "seed": SEED},
        "layer_gbs": res["gbs"], "layer_frac_of_hbm": res["frac"],
        "roofline": {"bound": "hbm", "kernel": "decode_layer_kernel x 48",
                     "achieved": res["gbs"], "peak": res["peak"],
                     "unit": "GB/s", "frac": res["frac"],
                     "peak_source": res["peak_source"], "traffic": None,
                     "algorithmic_bytes_per_step": res["bytes_step"]},
        "unique_experts_per_layer_step": res["u_avg"],
        "graph_replay_matches_eager": res["graph_replay_matches_eager"],
        "slot_cache": res.get("slot_cache"),
        "slot_cache_in_stream": res["slot_cache_in_stream"],
        "setup_s": res["setup_s"],
        "gpu_launches": L * S,
        "clocks": res["clocks"],
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(T)
    print(json.dumps(line), flush=True)


PF_LAUNCHES_PER_STEP = 12   # route 2, group 3, row-map fill + pair rows + x16 + plan + up, down, combine


def run_prefill(args) -> None:
    """`--workload prefill`: the prefill chunk as the headline line (one
    GPU; other ranks, if any, run the same replica)."""
    import torch
    from synth.pools import build_pool, layer_desc
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    pool = build_pool(synth.BIG, SEED, 0)
    pf = Prefill(pool, layer_desc(synth.BIG, pool))
    K, W = args.steps, args.warmup
    for _ in range(W):
        pf.step()
    torch.cuda.synchronize()
    props = torch.cuda.get_device_properties(local)
    uuid = getattr(props, "uuid", None)
    clk = ClockSampler(f"GPU-{uuid}" if uuid else None)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    clk.start()
    ms = events_time(pf.step, K, 0) * K
    clocks = clk.stop()
    ms = max_over_ranks(ms, dist, "cuda")
    line = None
    if rank == 0:
        hbm, tf, src = peaks()
        m = prefill_measure(pf, max(3, min(K, 10)), 2)
        fl = prefill_flops(pf.T)
        up_ms = m["parts_ms"]["up_gemm"]
        ms_e2e = prefill_e2e_time(pf, max(3, min(K, 10)), 2)
        line = {
            "metric": METRIC, "value": job_rate(pf.T * K, world, ms),
            "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": W,
            "ms_per_step": ms / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "f16 tcgen05 (f32 accumulate) + f32",
            "data": "synthetic",
            "config": {"workload": m["workload"], "T": pf.T, "H": 3072,
                       "F": 1024, "E": 512, "k": 10,
                       "l2": "inputs larger than L2: 2.19 GB of experts, "
                             "1.17 GB y_pairs per step",
                       "parallelism": f"replicas x{world}", "seed": SEED},
            "tflops": fl["total"] / (ms / K * 1e-3) / 1e12,
            "roofline": {
                "bound": "tensor",
                "kernel": ("pf_gemm_kernel<up, SB3> (up/gate + SwiGLU), "
                           "launched alone on the staged activations"),
                "achieved": m["up_gemm_tflops"], "peak": tf,
                "unit": "TFLOP/s", "frac": m["up_gemm_tflops"] / tf,
                "peak_source": src,
                "traffic": captured_traffic_prefill(),
                "algorithmic_flops_per_launch": fl["up"],
                "avg_launch_ms": up_ms,
                "with_activation_pass": {
                    "achieved": m["up_tflops"],
                    "frac": m["up_tflops"] / tf,
                    "avg_call_ms": m["parts_ms"]["up"]},
                "down_gemm_frac": m["down_frac_of_bf16_peak"],
                "expert_gemms_frac": m["expert_gemms_frac_of_bf16_peak"],
                "layer_frac": m["frac_of_bf16_peak"]},
            "prefill": m,
            "e2e": {"value": pf.T / (ms_e2e / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": pf.T * 3072 * 2,
                    "d2h_bytes_per_step": pf.T * 3072 * 4},
            "gpu_launches": PF_LAUNCHES_PER_STEP * K,
            "clocks": clocks,
        }
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline_prefill()
        if world == 1 and not args.no_extras:
            del pf
            torch.cuda.empty_cache()
            line["prefill_sweep"] = prefill_sweep(pool)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


# Named workloads (the tiny 8-token shape is a parity case, not a bench line)
CONFIGS = {"c1": "decode", "c2": "stack", "c3": "prefill", "c4": "stack"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--layers", type=int, default=8)
    ap.add_argument("--T", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", action="store_true",
                    help="eager steps only, for ncu launch lists")
    ap.add_argument("--workload", default="decode",
                    choices=["decode", "prefill", "stack"])
    ap.add_argument("--stack-reps", type=int, default=4,
                    help="stack: timed passes over the steps")
    ap.add_argument("--store-gb", type=float, default=24.0,
                    help="stack: pinned host store limit for slot misses")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the decode T sweep, NL3 / SB2 decode and 48-layer stack "
                         "objects of the default line")
    ap.add_argument("--stack-steps", type=int, default=16,
                    help="steps of the default line's compact stack object")
    ap.add_argument("--no-prefill", action="store_true",
                    help="leave the prefill figures out of the decode line")
    ap.add_argument("--seed", type=int, default=0,
                    help="seed of every synthetic input (activations, "
                         "router, experts, Zipf bias)")
    ap.add_argument("--config", choices=sorted(CONFIGS),
                    help="a named workload: c1 one decode layer (--T tokens),"
                         " c2 / c4 the 48-layer stack, resident and through "
                         "the slot pool (one line), c3 the 9536-token "
                         "prefill chunk")
    args = ap.parse_args()
    if args.config:
        args.workload = CONFIGS[args.config]
    global SEED
    SEED = args.seed
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.profile:
        run_profile(args)
    elif args.workload == "prefill":
        if args.steps == 100000:
            args.steps = 200
        run_prefill(args)
    elif args.workload == "stack":
        if args.steps == 100000:
            args.steps = 64
        run_stack(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
