#!/usr/bin/env python
"""Benchmark: GLA layer forward+backward tokens/s on B200 and its fraction of
the layer roofline.

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

import numpy as np
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


def method_bytes(w):
    """Per kernel: bytes of the LAYER's own inputs that the kernel reads plus the layer's own outputs
    that it writes (q, k, v, dO, log a, h0/dhT in; o, hT, dq, dk, dv, dlog a, dh0 out), each once.
    The implementation's intermediates (chunk states, rescaled operands, score blocks) are not
    counted: this is the figure a kernel's bandwidth fraction is judged on."""
    BH, L, K, V = w.B * w.H, w.L, w.K, w.V
    th = BH * L
    e = 2
    st = BH * K * V * 4
    return {
        "tc_prep": th * (2 * K * e + 4 * K),                      # q, k, log a
        "tc_walk_states": th * V * e + st,                        # v; hT
        "tc_output": th * V * e * 2,                              # v; o
        "tc_walk_dstates": th * V * e + st,                       # dO; dh0
        "tc_output_dv": th * V * e * 2,                           # dO; dv
        "tc_bwd_chunk": th * (2 * K * e + 4 * K + 2 * V * e + 2 * K * e + 4 * K),  # q k log a v dO; dq dk dlog a
        "tc_walk_fwd": th * (2 * V * e) + st,                     # v; o, hT
        "tc_walk_dv": th * (2 * V * e) + st,                      # dO; dv, dh0
        "step": 2 * st + BH * (2 * K * e + V * e + 4 * K + V * e),
    }


def fwd_model(w, C=128):
    """Algorithmic bytes and flops of the forward alone (o and hT from q, k, v, log a)."""
    m = algorithmic_model(w, C)
    return {"bytes": m["bytes_fwd"], "flops": m["flops_fwd"]}


def layer_roofline(alg_bytes, alg_flops, ms, peaks):
    """The step against max(algorithmic bytes / measured HBM bandwidth, algorithmic flops / measured
    bf16 dense peak)."""
    t_hbm = alg_bytes / (peaks["hbm_gbs"] * 1e9)
    t_flop = alg_flops / (peaks["bf16_tflops"] * 1e12)
    t_roof = max(t_hbm, t_flop)
    return {"roofline_ms": round(t_roof * 1e3, 5), "frac": round(t_roof * 1e3 / ms, 4),
            "bound": "hbm" if t_hbm >= t_flop else "tensor"}


# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one
# ncu capture of the default workload, with the SHA-1 of the kernel's source
# file at capture time: a kernel whose source changed since reports null.
NCU_TRAFFIC = {
    "tc_prep": (74451200, "gla_tc_prep.cu", "50bba1f6b1363e821086631a7d2d5c1d3a961acc"),
    "tc_walk_states": (82471424, "gla_tc_states.cu", "2412bcc17a256403d58ee52850586d71ceeb4601"),
    "tc_output": (132055552, "gla_tc_out.cu", "285ea49a1a538d922b569c6ed2e3ad1ab5af4341"),
    "tc_walk_dstates": (72099328, "gla_tc_states.cu", "2412bcc17a256403d58ee52850586d71ceeb4601"),
    "tc_output_dv": (132318208, "gla_tc_out.cu", "285ea49a1a538d922b569c6ed2e3ad1ab5af4341"),
    "tc_bwd_chunk": (331208960, "gla_tc_bwd.cu", "7a225b8667dab37de39518c25b00451539497f35"),
    "tc_intra_twolevel": (68345344, "gla_tc_twolevel.cu", "a3457917f64458551c35f0e9c74e355a0ad1a3a5"),
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


# ------------------------------------------------------- the other workloads
def oracle_sample(w, passes, n_heads_max, L_max):
    """The fp64 oracle as it stands on a bounded sample of a workload: the first n heads (n = host
    cores, at most B*H) over the first L_max tokens. Returns tokens/s (a token carries H heads)."""
    import oracle
    from chunkwise_linear_rnn_gla_b200.inputs import make_inputs, to_f64_numpy

    cores = oracle.num_threads()
    Ls = min(w.L, L_max)
    nheads = max(1, min(w.B * w.H, cores, n_heads_max))
    inp = make_inputs(1, nheads, Ls, w.K, w.V, w.dtype, seed=0, z_mean=w.z_mean, with_grad=(passes != "fwd"))
    f = {n: to_f64_numpy(t) for n, t in inp.items()}
    t0 = time.perf_counter()
    oracle.fwd(f["q"], f["k"], f["v"], f["log_a"])
    if passes != "fwd":
        oracle.bwd(f["q"], f["k"], f["v"], f["log_a"], f["dO"])
    dt = time.perf_counter() - t0
    return {"value": nheads * Ls / w.H / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": "%d of %d heads, first %d of L=%d tokens, %s fp64 step recurrence, %.2f s"
                      % (nheads, w.B * w.H, Ls, w.L, passes, dt)}


def gsa_model(B, H, L, K, V, m, C=128):
    """Algorithmic work of gated slot attention fwd+bwd (the method's own tensors and the chunk form's
    arithmetic, no state materialisation). Bytes per token-head: forward reads q, k, v (bf16), the gate
    (fp32, m) and writes o; the backward reads q, k, v, dO and the gate and writes dq, dk, dv and the
    gate gradient. FLOPs per token-head: both memories' state updates and reads (4m(d_k + d_v)), the
    causal halves of the intra-chunk products, and in the backward the two GLA backward passes
    (8 K V + C(3K + 2V) each, K = m), the read of the value memory for the softmax backward and layer
    one's forward for dq."""
    th = B * H * L
    e = 2
    fwd_b = e * (2 * K + V) + 4 * m + e * V
    bwd_b = e * (2 * K + 2 * V) + 4 * m + e * (2 * K + V) + 4 * m
    f_fwd = 4 * m * (K + V) + C * (K + 2 * m + V)
    f_bwd = (8 * m * V + C * (3 * m + 2 * V)) + (2 * m * V + C * (V + m)) + (2 * m * K + C * (m + K)) \
        + (8 * m * K + C * (3 * m + 2 * K))
    return {"bytes": th * (fwd_b + bwd_b), "flops": th * (f_fwd + f_bwd),
            "per_token_head": {"bytes": fwd_b + bwd_b, "flops": f_fwd + f_bwd}}


def run_gsa(dev, peaks, med_ms, flush, with_cpu=True):
    """Gated slot attention, 1.3B-layer shape with 128 slots: device time of fwd+bwd (the backward
    reusing the forward's workspace), the layer roofline of the method's own bytes and FLOPs, the
    per-kernel breakdown from the library's event hooks, and the fp64 oracle on a bounded sample."""
    import torch

    import chunkwise_linear_rnn_gla_b200 as gla
    from chunkwise_linear_rnn_gla_b200 import gsa
    from chunkwise_linear_rnn_gla_b200.inputs import GSA_WORKLOAD as W, make_gsa_inputs

    B, H, L, K, V, m = (W[n] for n in ("B", "H", "L", "K", "V", "m"))
    inp = make_gsa_inputs(B, H, L, K, V, m, W["dtype"], seed=0)
    d = {k: v.to(dev) for k, v in inp.items()}
    desc = gla.make_desc(B, H, L, K, V, W["dtype"])
    ws_f, ws_b = gsa.gsa_fwd_workspace_size(desc, m), gsa.gsa_bwd_workspace_size(desc, m)
    ws = torch.empty(ws_b, dtype=torch.uint8, device=dev)

    def fn():
        gsa.gsa_fwd(d["q"], d["k"], d["v"], d["log_a"], workspace=ws)
        gsa.gsa_bwd(d["q"], d["k"], d["v"], d["log_a"], d["dO"], workspace=ws, ws_from_fwd=True)

    ms = med_ms(fn)
    alg = gsa_model(B, H, L, K, V, m)
    lr = layer_roofline(alg["bytes"], alg["flops"], ms, peaks)
    # per-kernel device time (an event pair around every launch; shares, not the headline), L2 flushed
    # before each step as for the GLA step
    fn()
    torch.cuda.synchronize(dev)
    gla.gla_profile_reset()
    gla.gla_profile_enable(True)
    for _ in range(3):
        flush.fill_(1.0)
        fn()
    torch.cuda.synchronize(dev)
    gla.gla_profile_enable(False)
    prof = gla.gla_profile_read()
    gla.gla_profile_reset()
    tot = sum(x[1] for x in prof.values()) or 1.0
    kernels = {n_: {"launches_per_step": c // 3, "us_per_step": round(t / 3 * 1e3, 2), "share": round(t / tot, 4)}
               for n_, (c, t) in sorted(prof.items(), key=lambda kv: -kv[1][1])}
    entry = {"B": B, "H": H, "L": L, "d_k": K, "d_v": V, "slots": m, "passes": "fwd+bwd",
             "route": gsa.gsa_route(desc, m), "ms": round(ms, 5), "tokens_per_s": round(B * L / ms * 1e3, 1),
             "layer_roofline_frac": lr["frac"], "roofline_ms": lr["roofline_ms"], "bound": lr["bound"],
             "alg_bytes": alg["bytes"], "alg_flops": alg["flops"], "per_token_head": alg["per_token_head"],
             "workspace_bytes": {"fwd": ws_f, "fwd+bwd": ws_b}, "kernels": kernels,
             "note": W["note"]}
    # decode: one token per call for a batch of 64 sequences, both memories (fp32) updated in place
    Bd = 64
    st = make_gsa_inputs(Bd, H, 1, K, V, m, W["dtype"], seed=1)
    sd = {n_: st[n_][:, :, 0].contiguous().to(dev) for n_ in ("q", "k", "v", "log_a")}
    hk = torch.zeros(Bd, H, m, K, device=dev)
    hv = torch.zeros(Bd, H, m, V, device=dev)
    step_ms = med_ms(lambda: gsa.gsa_step(sd["q"], sd["k"], sd["v"], sd["log_a"], hk, hv))
    mem_bytes = 2 * Bd * H * m * (K + V) * 4  # both memories read and written
    entry["decode"] = {"B": Bd, "us_per_step": round(step_ms * 1e3, 2), "tokens_per_s": round(Bd / step_ms * 1e3, 1),
                       "memory_GBps": round(mem_bytes / step_ms / 1e6, 1),
                       "hbm_frac": round(mem_bytes / step_ms / 1e6 / peaks["hbm_gbs"], 4),
                       "how": "median of single calls, L2 flushed before each; %.1f MB of memories read and "
                              "written per step" % (mem_bytes / 1e6)}
    del hk, hv, sd
    if with_cpu:
        import oracle
        from chunkwise_linear_rnn_gla_b200.inputs import to_f64_numpy

        cores = oracle.num_threads()
        nh = max(1, min(B * H, cores, 16))
        Ls = min(L, 512)
        smp = make_gsa_inputs(1, nh, Ls, K, V, m, W["dtype"], seed=0)
        f = {n_: to_f64_numpy(t) for n_, t in smp.items()}
        t0 = time.perf_counter()
        oracle.gsa_fwd(f["q"], f["k"], f["v"], f["log_a"])
        oracle.gsa_bwd(f["q"], f["k"], f["v"], f["log_a"], f["dO"])
        dt = time.perf_counter() - t0
        entry["cpu_baseline"] = {"value": nh * Ls / H / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                 "sample": "%d of %d heads, first %d of L=%d tokens, fwd+bwd fp64 step recurrence, "
                                           "%.2f s" % (nh, B * H, Ls, L, dt)}
    del d, ws
    torch.cuda.empty_cache()
    return entry


def run_workloads(dev, peaks, flush, with_cpu=True, reps=10):
    """Device time of every other named workload, eager calls with L2 flushed before each (median of
    `reps` CUDA-event timings after 3 warm-ups): the 340M-layer forward, the long sequence with
    materialised and non-materialised states (with each mode's workspace bytes: the memory
    footprint), the fixed-token sweep, and the decode workload with L2 flushed and with the state
    left in L2."""
    import torch

    import chunkwise_linear_rnn_gla_b200 as gla
    from chunkwise_linear_rnn_gla_b200.inputs import DECODE, WORKLOADS, make_inputs, make_step_inputs

    stream = torch.cuda.current_stream(dev)

    def med_ms(fn):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(reps):
            flush.fill_(1.0)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize(dev)
            ts.append(a.elapsed_time(b))
        return sorted(ts)[len(ts) // 2]

    cases = [("gla340m_fwd", "fwd", ("materialized",), {}, "gla340m_fwd"),
             ("long16k", "fwd+bwd", ("materialized", "nonmaterialized"), {}, "long16k")]
    cases += [("sweep_L%d" % L, "fwd+bwd", ("materialized",), {}, "sweep_L%d" % L) for L in (1024, 2048, 4096, 8192, 16384)]
    # the intra-chunk scores by two-level chunking (sub-chunks of 16) against the default single GEMM
    cases += [("gla1p3b_fwdbwd", "fwd+bwd", ("materialized",), {"subchunk": sc}, "gla1p3b_subchunk%d" % sc)
              for sc in (128, 16)]
    out = {}
    for name, passes, modes, extra, label in cases:
        w = WORKLOADS[name]
        inp = make_inputs(w.B, w.H, w.L, w.K, w.V, w.dtype, seed=0, z_mean=w.z_mean, with_grad=(passes != "fwd"))
        d = {k: v.to(dev) for k, v in inp.items()}
        o = torch.empty_like(d["v"])
        hT = torch.empty(w.B, w.H, w.K, w.V, device=dev)
        outs = None
        if passes != "fwd":
            outs = {"dq": torch.empty_like(d["q"]), "dk": torch.empty_like(d["k"]), "dv": torch.empty_like(d["v"]),
                    "dlog_a": torch.empty_like(d["log_a"]), "dh0": torch.empty(w.B, w.H, w.K, w.V, device=dev)}
        alg = algorithmic_model(w) if passes != "fwd" else fwd_model(w)
        entry = {"B": w.B, "H": w.H, "L": w.L, "d_k": w.K, "d_v": w.V, "passes": passes, "modes": {}, **extra}
        for mode in modes:
            desc = gla.make_desc(w.B, w.H, w.L, w.K, w.V, w.dtype, 0, extra.get("subchunk", 0), mode, "auto")
            ws_f, ws_b = gla.gla_fwd_workspace_size(desc), gla.gla_bwd_workspace_size(desc)
            ws = torch.empty(ws_b if passes != "fwd" else ws_f, dtype=torch.uint8, device=dev)
            kw = dict(state_mode=mode, **extra)

            def fn():
                gla.gla_fwd(d["q"], d["k"], d["v"], d["log_a"], None, o=o, hT=hT, workspace=ws, **kw)
                if outs is not None:
                    gla.gla_bwd(d["q"], d["k"], d["v"], d["log_a"], d["dO"], None, None, workspace=ws,
                                ws_from_fwd=True, out=outs, **kw)

            ms = med_ms(fn)
            lr = layer_roofline(alg["bytes"], alg["flops"], ms, peaks)
            entry["modes"][mode] = {"ms": round(ms, 5), "tokens_per_s": round(w.B * w.L / ms * 1e3, 1),
                                    "layer_roofline_frac": lr["frac"], "roofline_ms": lr["roofline_ms"],
                                    "workspace_bytes": {"fwd": ws_f, "fwd+bwd": ws_b}}
            del ws
        if with_cpu and not extra:
            entry["cpu_baseline"] = oracle_sample(w, passes, 16, 1024)
        out[label] = entry
        del inp, d, o, hT, outs
        torch.cuda.empty_cache()

    out["gsa1p3b_fwdbwd"] = run_gsa(dev, peaks, med_ms, flush, with_cpu)

    # decode: B=64, H=4, d_k=128, d_v=256, one token per call, fp32 state carried
    B, H, K, V = (DECODE[n] for n in ("B", "H", "K", "V"))
    T = 64
    st = make_step_inputs(B, H, K, V, T, DECODE["dtype"], seed=0)
    q, k, v, la = (st[n].to(dev) for n in ("q", "k", "v", "log_a"))
    S = torch.zeros(B, H, K, V, device=dev)
    ob = torch.empty(T, B, H, V, dtype=q.dtype, device=dev)
    for t in range(T):
        gla.gla_step(q[t], k[t], v[t], la[t], S, o=ob[t])
    torch.cuda.synchronize(dev)
    flushed = []
    for t in range(T):
        flush.fill_(1.0)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        gla.gla_step(q[t], k[t], v[t], la[t], S, o=ob[t])
        b.record(stream)
        torch.cuda.synchronize(dev)
        flushed.append(a.elapsed_time(b))
    ms_flushed = sorted(flushed)[T // 2]
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        gla.gla_step(q[0], k[0], v[0], la[0], S, o=ob[0])
    stream.wait_stream(side)
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for t in range(T):
            gla.gla_step(q[t], k[t], v[t], la[t], S, o=ob[t])
    g.replay()
    torch.cuda.synchronize(dev)
    reps_g = DECODE["steps"] // T
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(reps_g):
        g.replay()
    b.record(stream)
    torch.cuda.synchronize(dev)
    ms_res = a.elapsed_time(b) / (reps_g * T)
    del g
    state_bytes = 2 * B * H * K * V * 4
    dec = {"B": B, "H": H, "d_k": K, "d_v": V, "steps": DECODE["steps"],
           "l2_resident": {"us_per_step": round(ms_res * 1e3, 3), "tokens_per_s": round(B / ms_res * 1e3, 1),
                           "state_GBps": round(state_bytes / ms_res / 1e6, 1),
                           "how": "CUDA graph of 64 steps replayed %d times (%d steps); the 33.5 MB state stays in L2"
                                  % (reps_g, reps_g * T)},
           "l2_flushed": {"us_per_step": round(ms_flushed * 1e3, 3), "tokens_per_s": round(B / ms_flushed * 1e3, 1),
                          "state_GBps": round(state_bytes / ms_flushed / 1e6, 1),
                          "hbm_frac": round(state_bytes / ms_flushed / 1e6 / peaks["hbm_gbs"], 4),
                          "how": "median of 64 single calls, each after a 512 MB write"}}
    if with_cpu:
        import oracle
        from chunkwise_linear_rnn_gla_b200.inputs import to_f64_numpy

        f = {n: to_f64_numpy(st[n][0]) for n in ("q", "k", "v", "log_a")}
        S0 = np.zeros((B, H, K, V))
        t0 = time.perf_counter()
        nrep = 4
        for _ in range(nrep):
            oracle.step(f["q"], f["k"], f["v"], f["log_a"], S0)
        dt = (time.perf_counter() - t0) / nrep
        dec["cpu_baseline"] = {"value": B / dt, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                               "sample": "%d decode steps of the full batch, fp64, %.3f s per step" % (nrep, dt)}
    out["decode_b64"] = dec
    return out


def workload_config(w, world):
    """The workload both arms of the benchmark run (identical keys and values in both JSON lines)."""
    from chunkwise_linear_rnn_gla_b200 import dp

    return {"workload": w.name, "B": w.B, "H": w.H, "L": w.L, "d_k": w.K, "d_v": w.V,
            "global_batch": dp.global_batch(w.B, world), "seq_len": w.L, "parallelism": "dp%d" % world,
            "passes": w.passes, "gate": "per key channel, log alpha = logsigmoid(z)/16, z ~ N(%g, 1)" % w.z_mean}


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
    ap.add_argument("--subchunk", type=int, default=0,
                    help="sub-chunk length of the intra-chunk scores (0: the default single GEMM per chunk; "
                         "16: two-level chunking on the tensor-core path)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the timing of the other named workloads and the decode workload")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=8)
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
                "config": workload_config(w, args.gpus),
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
    desc = gla.make_desc(w.B, w.H, w.L, w.K, w.V, w.dtype, 0, args.subchunk, args.state_mode, args.kernel_impl)
    C, sc, impl_name, mode = gla.gla_resolve(desc)
    ws = torch.empty(gla.gla_bwd_workspace_size(desc), dtype=torch.uint8, device=dev)
    o = torch.empty_like(d["v"])
    hT = torch.empty(w.B, w.H, w.K, w.V, dtype=torch.float32, device=dev)
    outs = {"dq": torch.empty_like(d["q"]), "dk": torch.empty_like(d["k"]), "dv": torch.empty_like(d["v"]),
            "dlog_a": torch.empty_like(d["log_a"]), "dh0": torch.empty(w.B, w.H, w.K, w.V, device=dev)}
    kw = dict(impl=args.kernel_impl, state_mode=args.state_mode, subchunk=args.subchunk)

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
    # Every step copies its inputs from pinned host memory and reads every result back. The copies are
    # pipelined across steps as an input pipeline would run them: step i+1's inputs go host -> device on
    # one stream and step i-1's results device -> host on another while step i computes (PCIe carries
    # both directions at once); inputs and outputs are double-buffered on the device and on the host.
    e2e = None
    if not args.no_e2e:
        pin = {k: v.pin_memory() for k, v in inp.items()}
        outs_all = {"o": o, "hT": hT, **outs}
        dins = [d, {k: torch.empty_like(v) for k, v in d.items()}]
        douts = [outs_all, {k: torch.empty_like(v) for k, v in outs_all.items()}]
        hosts = [{k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in outs_all.items()} for _ in range(2)]
        h2d = sum(v.numel() * v.element_size() for v in pin.values())
        d2h = sum(v.numel() * v.element_size() for v in outs_all.values())
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_run(n):
            for j in range(n):
                b = j % 2
                din, dout, host = dins[b], douts[b], hosts[b]
                if j >= 2:
                    s_in.wait_event(ev_comp[b])  # step j-2 has finished reading this input set
                with torch.cuda.stream(s_in):
                    for k_, v_ in pin.items():
                        din[k_].copy_(v_, non_blocking=True)
                    ev_in[b].record(s_in)
                stream.wait_event(ev_in[b])
                if j >= 2:
                    stream.wait_event(ev_out[b])  # step j-2's results have been read out of this output set
                gla.gla_fwd(din["q"], din["k"], din["v"], din["log_a"], None, o=dout["o"], hT=dout["hT"],
                            workspace=ws, **kw)
                gla.gla_bwd(din["q"], din["k"], din["v"], din["log_a"], din["dO"], None, None, workspace=ws,
                            ws_from_fwd=True, out={n_: dout[n_] for n_ in outs}, **kw)
                ev_comp[b].record(stream)
                s_out.wait_event(ev_comp[b])
                with torch.cuda.stream(s_out):
                    for k_, v_ in dout.items():
                        host[k_].copy_(v_, non_blocking=True)
                    ev_out[b].record(s_out)

        e2e_run(2)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a_.record(s_in)
        e2e_run(args.e2e_steps)
        s_out.wait_stream(s_in)
        s_out.wait_stream(stream)
        b_.record(s_out)
        torch.cuda.synchronize(dev)
        e2e_ms = dp.max_over_ranks(a_.elapsed_time(b_) / args.e2e_steps)
        e2e = {"value": dp.job_throughput(w.B * w.L, world, e2e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "ms_per_step": e2e_ms,
               "how": ("%d steps, inputs host->device and results device->host pipelined across steps on two "
                       "copy streams, double-buffered" % args.e2e_steps)}

    # ---------------- roofline of the whole step (the headline) and of the dominant kernel
    peaks, peaks_src = load_peaks()
    models = kernel_models(w, C)
    mbytes = method_bytes(w)
    kroof = None
    kernels = {}
    if prof:
        tot = sum(x[1] for x in prof.values())
        for name, (n, ms) in prof.items():
            kernels[name] = {"launches": n, "total_ms": round(ms, 4), "share": round(ms / tot, 4),
                             "us_per_launch": round(ms / n * 1e3, 2)}
            if name in mbytes:
                kernels[name]["method_frac"] = round(mbytes[name] / (ms / n / 1e3) / 1e9 / peaks["hbm_gbs"], 4)
        name, (n, ms) = max(prof.items(), key=lambda kv: kv[1][1])
        avg_s = ms / n / 1e3
        mdl = models.get(name)
        if mdl is not None and name in mbytes:
            ach = mbytes[name] / avg_s / 1e9
            kroof = {"kernel": name, "bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": round(ach / peaks["hbm_gbs"], 4), "peak_source": peaks_src,
                     "alg_bytes_method": mbytes[name], "alg_bytes_impl": mdl["bytes"],
                     "frac_impl": round(mdl["bytes"] / avg_s / 1e9 / peaks["hbm_gbs"], 4),
                     "launch_ms": round(ms / n, 4), "traffic": measured_traffic(name),
                     "timing": ("CUDA events around each kernel launch over K further timed steps (pass B, "
                                "%.4f ms per step with the events; the headline step time is pass A, without them)"
                                % (prof_total_ms / args.steps)),
                     "bytes_note": ("achieved = the layer's own inputs read and outputs written by this kernel "
                                    "(alg_bytes_method) / its launch time; alg_bytes_impl adds the "
                                    "implementation's chunk states and operand workspace")}

    alg = algorithmic_model(w, C)
    lr = layer_roofline(alg["bytes"], alg["flops"], ms_per_step, peaks)
    step_traffic = None
    if kernels and all(measured_traffic(k) is not None for k in kernels):
        step_traffic = sum(measured_traffic(k) * kernels[k]["launches"] for k in kernels) // max(1, args.steps)
    layer_roof = {"roofline_ms": lr["roofline_ms"], "frac": lr["frac"], "bound": lr["bound"],
                  "achieved_GBps": round(alg["bytes"] / (ms_per_step / 1e3) / 1e9, 1), "peak_GBps": peaks["hbm_gbs"],
                  "alg_bytes": alg["bytes"], "alg_flops": alg["flops"],
                  "tflops": round(alg["flops"] / (ms_per_step / 1e3) / 1e12, 2),
                  # the same flops against the sustained (power-capped) bf16 GEMM rate
                  "tflops_frac_of_sustained_bf16": round(alg["flops"] / (ms_per_step / 1e3) / 1e12
                                                         / peaks["bf16_tflops_sustained"], 4),
                  "traffic_per_step": step_traffic,
                  "definition": "the whole fwd+bwd step against max(algorithmic bytes / measured HBM copy "
                                "bandwidth, algorithmic flops / measured bf16 dense peak); traffic_per_step = "
                                "summed ncu DRAM bytes of the step's launches (null when any kernel changed since)"}

    workloads = None
    if rank == 0 and world == 1 and not args.no_workloads:
        workloads = run_workloads(dev, peaks, flush, with_cpu=not args.no_cpu_baseline)

    cb = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(w)

    if rank == 0:
        line = {"metric": metric, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32",
                "data": "synthetic (seeded N(0,1)/sqrt(d_k) q,k,v; log_a = logsigmoid(N(0,1))/16; dO ~ N(0,1))",
                "config": workload_config(w, world),
                "impl_config": {"chunk": C,
                           # sub-chunk length of the intra-chunk scores: equal to the chunk on the tensor-core
                           # path means one GEMM per chunk (no secondary chunking); 16 is the two-level form
                           "subchunk": sc,
                           "kernel_impl": impl_name, "state_mode": mode,
                           "l2": "flushed between timed steps (512 MB write)", "step_launch": graph_note,
                           "eager_ms_per_step": round(eager_ms / args.steps, 5)},
                "roofline": kroof, "layer_roofline": layer_roof, "cpu_baseline": cb,
                "e2e": e2e, "gpu_launches": int(launches), "clocks": clk, "kernels": kernels, "workloads": workloads}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
