#!/usr/bin/env python
"""Benchmark: GLA layer forward+backward tokens/s on B200 and the roofline
fraction of the dominant kernel.

One step = gla_fwd + gla_bwd (the backward reuses the forward's workspace) on
the 1.3B-layer shape B=4 H=4 L=2048 d_k=256 d_v=512, bf16 q/k/v/dO with fp32
gates and states, synthetic seeded inputs. Tokens per step = B*L.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank drives one GPU on its own shard of heads (weak
scaling: every rank processes one full workload; no collective on the data
path); the step time is the max over ranks. Prints ONE JSON line on rank 0.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ models
def algorithmic_model(w, C=128):
    """Algorithmic bytes and flops of one fwd+bwd step (the chunk method's
    own work: inputs read once, outputs written once, GEMM flops of the chunk
    form; no materialised states)."""
    BH, L, K, V = w.B * w.H, w.L, w.K, w.V
    th = BH * L  # token-heads
    e = 2  # bf16
    bytes_fwd = th * (e * (2 * K + V) + 4 * K + e * V) + BH * 4 * K * V
    bytes_bwd = th * (e * (2 * K + 2 * V) + 4 * K + e * (2 * K + V) + 4 * K) + BH * 4 * K * V
    flops_fwd = th * (4 * K * V + C * (K + V))
    flops_bwd = th * (8 * K * V + C * (3 * K + 2 * V))
    return {"bytes": bytes_fwd + bytes_bwd, "flops": flops_fwd + flops_bwd, "bytes_fwd": bytes_fwd,
            "bytes_bwd": bytes_bwd, "flops_fwd": flops_fwd, "flops_bwd": flops_bwd}


def kernel_models(w, C):
    """Per-launch algorithmic (bytes, flops, bound) of each kernel, for the
    roofline of the dominant one. Bytes count each input read once and each
    output written once; flops count the chunk form's GEMMs."""
    BH, L, K, V = w.B * w.H, w.L, w.K, w.V
    th = BH * L
    N = math.ceil(L / C)
    e = 2
    st = BH * K * V * 4
    m = {}
    # CUDA-core kernels (fp32 arithmetic)
    m["simt_chunk_cumsum"] = dict(bytes=th * K * 8, flops=th * K, bound="hbm")
    m["simt_intra_P"] = dict(bytes=th * K * (2 * e + 4) + BH * N * C * C * 4, flops=th * C * K * 3, bound="alu")
    m["simt_state_walk"] = dict(bytes=th * (K * e + V * e + K * 4) + BH * (N + 1) * K * V * 4, flops=th * 2 * K * V,
                                bound="alu")
    m["simt_dstate_walk"] = dict(bytes=th * (K * e + V * e + K * 4) + BH * N * K * V * 4, flops=th * 2 * K * V,
                                 bound="alu")
    m["simt_output"] = dict(bytes=th * (K * e + V * e * 2 + K * 4) + BH * N * K * V * 4, flops=th * 2 * (K * V + C * V),
                            bound="alu")
    m["simt_intra_dP"] = dict(bytes=th * V * e * 2 + BH * N * C * C * 4, flops=th * C * V, bound="alu")
    m["simt_dqdk"] = dict(bytes=th * (4 * K * e + 2 * V * e + K * 8) + 2 * BH * N * K * V * 4,
                          flops=th * 4 * K * V, bound="alu")
    m["simt_dv"] = dict(bytes=th * (K * e + 2 * V * e + K * 4) + BH * N * K * V * 4, flops=th * 2 * K * V,
                        bound="alu")
    m["simt_dlog_a"] = dict(bytes=th * K * 8, flops=th * K, bound="hbm")
    m["step"] = dict(bytes=2 * st, flops=4 * BH * K * V, bound="hbm")
    # tensor-core path (bf16 operands, fp32 accumulate); C = 128
    sb = BH * N * K * V * e  # one set of bf16 chunk states
    pb = BH * N * C * C * e  # intra-chunk score matrices
    m["tc_prep"] = dict(bytes=th * (2 * K * e + 4 * K + 2 * K * e) + pb + BH * N * K * 4,
                        flops=th * 2 * C * K, bound="hbm")
    m["tc_walk_states"] = dict(bytes=th * (K * e + V * e) + sb, flops=th * 2 * K * V, bound="hbm")
    m["tc_walk_dstates"] = dict(bytes=th * (K * e + V * e) + sb, flops=th * 2 * K * V, bound="hbm")
    m["tc_output"] = dict(bytes=th * (K * e + 2 * V * e) + pb + sb, flops=th * 2 * (K * V + C * V), bound="hbm")
    m["tc_output_dv"] = dict(bytes=th * (K * e + 2 * V * e) + pb + sb, flops=th * 2 * (K * V + C * V), bound="hbm")
    m["tc_walk_fwd"] = dict(bytes=th * (2 * K * e + 2 * V * e) + pb + 2 * st, flops=th * 2 * (2 * K * V + C * V),
                            bound="hbm")
    m["tc_walk_dv"] = dict(bytes=th * (2 * K * e + 2 * V * e) + pb + 2 * st, flops=th * 2 * (2 * K * V + C * V),
                           bound="hbm")
    # fused chunk backward: reads dO, v, S_[i], D_i, Q~, q, k, log a, e^Gamma; writes dq, dk, dlog a.
    # flops: dP, dO S^T, v D^T and the two intra-chunk GEMMs
    m["tc_bwd_chunk"] = dict(bytes=th * (2 * V * e + K * e + 2 * K * e + 4 * K + 2 * K * e + 4 * K) + 2 * sb
                             + BH * N * K * 4,
                             flops=th * (2 * C * V + 4 * K * V + 4 * C * K), bound="hbm")
    return m


# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one
# ncu capture of the default workload, with the SHA-1 of the kernel's source
# file at capture time: a kernel whose source changed since reports null.
NCU_TRAFFIC = {
    "tc_prep": (74336256, "gla_tc_prep.cu", "13e8d173e1ef24a6ea33660af099850d6e98cfaf"),
    "tc_walk_states": (82829568, "gla_tc_states.cu", "bb8f83f1545289b859a5164c6b67cdc98e708734"),
    "tc_output": (135306240, "gla_tc_out.cu", "285ea49a1a538d922b569c6ed2e3ad1ab5af4341"),
    "tc_walk_dstates": (75097600, "gla_tc_states.cu", "bb8f83f1545289b859a5164c6b67cdc98e708734"),
    "tc_output_dv": (132920832, "gla_tc_out.cu", "285ea49a1a538d922b569c6ed2e3ad1ab5af4341"),
    "tc_bwd_chunk": (327452160, "gla_tc_bwd.cu", "4ebf7e129f463e33f6887504e06f27e8599c0b35"),
}


def measured_traffic(name):
    ent = NCU_TRAFFIC.get(name)
    if not ent:
        return None
    nbytes, src, sha = ent
    try:
        import hashlib

        with open(os.path.join(ROOT, "chunkwise_linear_rnn_gla_b200", "csrc", src), "rb") as f:
            if hashlib.sha1(f.read()).hexdigest() != sha:
                return None
    except OSError:
        return None
    return nbytes


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="gla_clocks_", suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            self.t_start = time.time()
        except Exception:
            self.proc = None

    def wait_first_sample(self, timeout_s=3.0):
        """Block until nvidia-smi has written its first sample, so that sampling is live before the
        timed region starts."""
        if self.proc is None:
            return
        t0 = time.time()
        while time.time() - t0 < timeout_s:
            try:
                if os.path.getsize(self.path) > 0:
                    return
            except OSError:
                return
            time.sleep(0.01)

    def stop(self, keep_busy=None, min_s=0.0):
        """Stop sampling. `keep_busy` (a callable that enqueues work) keeps the GPU on the same step
        until `min_s` seconds have passed since start, so that a short timed region still gets
        samples taken under its own load."""
        if self.proc is None:
            return None
        if keep_busy is not None:
            while time.time() - self.t_start < min_s:
                keep_busy()
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        try:
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        except Exception:
            return None
        finally:
            try:
                os.unlink(self.path)
            except Exception:
                pass
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "", 1).isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "", 1).isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for name, val in zip(names, r[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(rows)}


# ------------------------------------------------------------- CPU baseline
def cpu_baseline(w, budget_s=20.0):
    """The fp64 oracle as it stands, on a bounded sample of the workload: the
    first n heads (n = host cores, at most B*H) over the full L, fwd+bwd."""
    import torch

    import oracle
    from chunkwise_linear_rnn_gla_b200.inputs import make_inputs, to_f64_numpy

    cores = oracle.num_threads()
    inp = make_inputs(w.B, w.H, w.L, w.K, w.V, w.dtype, seed=0)
    nheads = max(1, min(w.B * w.H, cores))
    sel = lambda t: to_f64_numpy(t.reshape(w.B * w.H, *t.shape[2:])[:nheads].unsqueeze(0))  # noqa: E731
    q, k, v, la, dO = (sel(inp[n]) for n in ("q", "k", "v", "log_a", "dO"))
    del torch
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.fwd(q, k, v, la)
        oracle.bwd(q, k, v, la, dO)
        reps += 1
        if time.perf_counter() - t0 > budget_s * 0.5 or reps >= 3:
            break
    dt = (time.perf_counter() - t0) / reps
    tokens = nheads * w.L / w.H  # token-heads / heads-per-token
    return {"value": tokens / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": "%d of %d heads, full L=%d d_k=%d d_v=%d, fwd+bwd fp64 step recurrence, %d rep(s), %.1f s/rep"
                      % (nheads, w.B * w.H, w.L, w.K, w.V, reps, dt)}


# --------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="gla1p3b_fwdbwd")
    ap.add_argument("--kernel-impl", default="auto", choices=["auto", "simt", "tc"])
    ap.add_argument("--state-mode", default="materialized", choices=["auto", "materialized", "nonmaterialized"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-graph", action="store_true",
                    help="launch the timed step eagerly instead of replaying it from a CUDA graph")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    from chunkwise_linear_rnn_gla_b200 import dp

    env = dp.rank_env()
    world, rank, local_rank = env.world, env.rank, env.local_rank

    from chunkwise_linear_rnn_gla_b200.inputs import WORKLOADS

    w = WORKLOADS[args.workload]
    metric = "GLA layer fwd+bwd tokens/s on 1 B200 and achieved fraction of roofline"

    if args.impl == "reference":
        # The reference arm is the fp64 CPU oracle, timed as it stands on this
        # host; only rank 0 works.
        if rank != 0:
            return 0
        cb = cpu_baseline(w, budget_s=60.0 / max(1, args.steps + args.warmup))
        line = {"impl": "reference", "metric": metric, "value": cb["value"], "unit": "tokens/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": w.name, "B": w.B, "H": w.H, "L": w.L, "d_k": w.K, "d_v": w.V},
                "cpu_baseline": cb,
                "e2e": {"value": cb["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    import torch
    import torch.distributed as dist

    import chunkwise_linear_rnn_gla_b200 as gla

    gla.load()
    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", init_method="env://", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local_rank if world > 1 else 0)
    torch.cuda.set_device(dev)

    from chunkwise_linear_rnn_gla_b200.inputs import make_inputs

    inp = make_inputs(w.B, w.H, w.L, w.K, w.V, w.dtype, seed=dp.shard_seed(0, rank))
    d = {k: v.to(dev) for k, v in inp.items()}
    desc = gla.make_desc(w.B, w.H, w.L, w.K, w.V, w.dtype, 0, 0, args.state_mode, args.kernel_impl)
    C, sc, impl_name, mode = gla.gla_resolve(desc)
    ws = torch.empty(gla.gla_bwd_workspace_size(desc), dtype=torch.uint8, device=dev)
    o = torch.empty_like(d["v"])
    hT = torch.empty(w.B, w.H, w.K, w.V, dtype=torch.float32, device=dev)
    outs = {"dq": torch.empty_like(d["q"]), "dk": torch.empty_like(d["k"]), "dv": torch.empty_like(d["v"]),
            "dlog_a": torch.empty_like(d["log_a"]), "dh0": torch.empty(w.B, w.H, w.K, w.V, device=dev)}
    kw = dict(impl=args.kernel_impl, state_mode=args.state_mode)

    def step():
        gla.gla_fwd(d["q"], d["k"], d["v"], d["log_a"], None, o=o, hT=hT, workspace=ws, **kw)
        gla.gla_bwd(d["q"], d["k"], d["v"], d["log_a"], d["dO"], None, None, workspace=ws, ws_from_fwd=True,
                    out=outs, **kw)

    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)

    stream = torch.cuda.current_stream(dev)

    # The step is captured once into a CUDA graph (the library's launches are capture-safe: host-side
    # tensor maps, no allocation or synchronisation) and replayed, as a training loop would; the
    # per-kernel timing pass stays eager because it needs an event pair around every launch.
    graph, graph_launches, graph_note = None, 0, "eager"
    if not args.no_graph:
        try:
            side = torch.cuda.Stream(dev)
            side.wait_stream(stream)
            with torch.cuda.stream(side):
                step()
            stream.wait_stream(side)
            torch.cuda.synchronize(dev)
            graph = torch.cuda.CUDAGraph()
            gla.gla_launch_count_reset()
            with torch.cuda.graph(graph):
                step()
            graph_launches = gla.gla_launch_count()
            for _ in range(max(3, args.warmup)):
                graph.replay()
            torch.cuda.synchronize(dev)
            graph_note = "cuda_graph"
        except Exception as ex:  # capture is an optimisation: report and time the eager step
            graph, graph_note = None, "eager (graph capture failed: %s)" % type(ex).__name__
            torch.cuda.synchronize(dev)

    def timed_pass(kernel_events, use_graph=False):
        """K steps between barriers and synchronisations; L2 flushed before each step. Returns the
        summed step time (CUDA events on the launching stream) and our kernel launches."""
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        gla.gla_profile_reset()
        gla.gla_launch_count_reset()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        gla.gla_profile_enable(kernel_events)
        for i in range(args.steps):
            flush.fill_(float(i))  # evict L2 (126 MB) between timed steps
            ev[i][0].record(stream)
            if use_graph:
                graph.replay()
            else:
                step()
            ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
        gla.gla_profile_enable(False)
        n_launch = graph_launches * args.steps if use_graph else gla.gla_launch_count()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        return sum(a.elapsed_time(b) for a, b in ev), n_launch

    # pass A: the step as a user runs it (headline time, clocks, launch count)
    clocks = ClockSampler(dev.index if world == 1 else local_rank)
    clocks.start()
    clocks.wait_first_sample()
    total_ms, launches = timed_pass(False, use_graph=graph is not None)

    def keep_busy():  # the same step, untimed, so that the clock samples are taken under this load
        for _ in range(20):
            if graph is not None:
                graph.replay()
            else:
                step()
        torch.cuda.synchronize(dev)

    clk = clocks.stop(keep_busy, min_s=0.6)
    if clk is not None:
        clk["window"] = "timed pass A, then the same step replayed untimed until 0.6 s of sampling (100 ms period)"
    eager_ms = timed_pass(False)[0] if graph is not None else total_ms
    # pass B: the same K steps with a CUDA event pair around every kernel launch, for the per-kernel
    # durations of the roofline (the events between kernels lengthen the step, so pass A is the headline)
    prof_total_ms, _ = timed_pass(True)
    prof = gla.gla_profile_read()
    total_ms = dp.max_over_ranks(total_ms)
    eager_ms = dp.max_over_ranks(eager_ms)
    ms_per_step = total_ms / args.steps
    tokens_per_step = w.B * w.L * world
    value = dp.job_throughput(w.B * w.L, world, ms_per_step)

    # ---------------- end to end through the public API, host buffers
    e2e = None
    if not args.no_e2e:
        pin = {k: v.pin_memory() for k, v in inp.items()}
        host_out = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in outs.items()}
        host_o = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        h2d = sum(v.numel() * v.element_size() for v in pin.values())
        d2h = sum(v.numel() * v.element_size() for v in host_out.values()) + host_o.numel() * host_o.element_size()

        def e2e_step():
            for k_, v_ in pin.items():
                d[k_].copy_(v_, non_blocking=True)
            step()
            host_o.copy_(o, non_blocking=True)
            for k_, v_ in outs.items():
                host_out[k_].copy_(v_, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a_.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        b_.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = dp.max_over_ranks(a_.elapsed_time(b_) / args.e2e_steps)
        e2e = {"value": dp.job_throughput(w.B * w.L, world, e2e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "ms_per_step": e2e_ms}

    # ---------------- roofline of the dominant kernel
    peaks, peaks_src = load_peaks()
    models = kernel_models(w, C)
    roof = None
    kernels = {}
    if prof:
        top = max(prof.items(), key=lambda kv: kv[1][1])
        for name, (n, ms) in prof.items():
            kernels[name] = {"launches": n, "total_ms": round(ms, 4), "share": round(ms / sum(x[1] for x in prof.values()), 4)}
        name, (n, ms) = top
        avg_s = ms / n / 1e3
        mdl = models.get(name)
        if mdl is not None:
            if mdl["bound"] == "hbm":
                ach = mdl["bytes"] / avg_s / 1e9
                roof = {"kernel": name, "bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"],
                        "unit": "GB/s", "frac": round(ach / peaks["hbm_gbs"], 4), "traffic": None}
            elif mdl["bound"] == "tensor":
                ach = mdl["flops"] / avg_s / 1e12
                pk = peaks["bf16_tflops_sustained"]
                roof = {"kernel": name, "bound": "tensor", "achieved": round(ach, 2), "peak": pk, "unit": "TFLOP/s",
                        "frac": round(ach / pk, 4), "traffic": None}
            else:  # fp32 CUDA-core arithmetic: 148 SMs x 128 FMA/clk x 2 flop x max SM clock
                pk = 148 * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
                ach = mdl["flops"] / avg_s / 1e12
                roof = {"kernel": name, "bound": "alu", "achieved": round(ach, 2), "peak": round(pk, 1),
                        "unit": "TFLOP/s", "frac": round(ach / pk, 4), "traffic": None}
            roof["peak_source"] = peaks_src
            roof["timing"] = ("CUDA events around each kernel launch over K further timed steps "
                              "(pass B, %.4f ms per step with the events; the headline step time is pass A, "
                              "without them)" % (prof_total_ms / args.steps))
            roof["launch_ms"] = round(ms / n, 4)
            roof["traffic"] = measured_traffic(name)
            roof["alg_bytes"] = mdl["bytes"]

    alg = algorithmic_model(w, C)
    t_roof = max(alg["bytes"] / (peaks["hbm_gbs"] * 1e9), alg["flops"] / (peaks["bf16_tflops"] * 1e12))
    layer_roof = {"roofline_ms": round(t_roof * 1e3, 5), "frac": round(t_roof * 1e3 / ms_per_step, 4),
                  "alg_bytes": alg["bytes"], "alg_flops": alg["flops"],
                  "tflops": round(alg["flops"] / (ms_per_step / 1e3) / 1e12, 2),
                  # the same flops against the sustained (power-capped) bf16 GEMM rate
                  "tflops_frac_of_sustained_bf16": round(alg["flops"] / (ms_per_step / 1e3) / 1e12
                                                         / peaks["bf16_tflops_sustained"], 4),
                  "bound": "hbm" if alg["bytes"] / peaks["hbm_gbs"] / 1e9 > alg["flops"] / peaks["bf16_tflops"] / 1e12
                  else "tensor"}

    cb = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(w)

    if rank == 0:
        line = {"metric": metric, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32",
                "data": "synthetic (seeded N(0,1)/sqrt(d_k) q,k,v; log_a = logsigmoid(N(0,1))/16; dO ~ N(0,1))",
                "config": {"workload": w.name, "B": w.B, "H": w.H, "L": w.L, "d_k": w.K, "d_v": w.V,
                           "global_batch": dp.global_batch(w.B, world), "seq_len": w.L, "chunk": C, "subchunk": sc,
                           "kernel_impl": impl_name, "state_mode": mode, "parallelism": "dp%d" % world,
                           "l2": "flushed between timed steps (512 MB write)", "step_launch": graph_note,
                           "eager_ms_per_step": round(eager_ms / args.steps, 5)},
                "roofline": roof, "layer_roofline": layer_roof, "cpu_baseline": cb, "e2e": e2e,
                "gpu_launches": int(launches), "clocks": clk, "kernels": kernels}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
