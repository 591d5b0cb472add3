"""Device times of the named workloads on one GPU:

    python -m chunkwise_linear_rnn_gla_b200.time_workloads [--only NAME ...] [--list]

For every bf16 workload of `inputs.WORKLOADS`: the forward and the forward + backward (the backward
reusing the forward's workspace), with materialised and with non-materialised chunk states. Each
case is called eagerly with L2 flushed before every call (a 512 MB write); the figure is the median
of 10 CUDA-event timings around the call, after 3 warm-up calls, followed by the per-kernel split
from the library's own launch timing over 3 more calls.

For gated slot attention (`inputs.GSA_WORKLOAD`, name "gsa1p3b_fwdbwd"): the forward and the forward +
backward the same way (`--reps 1` makes one timed call of each, for a profiler).

For the decode step (`inputs.DECODE`, and the same shape with B=256 whose 134 MB state exceeds L2):
the median of 20 calls with L2 flushed before each, and a CUDA graph of 64 calls replayed 5 times
with the state left in L2 between calls.

One line per case on stdout. This is a measurement utility; the parity tests live in `tests/`.
"""
import argparse
import sys

import torch

from . import gla_bwd, gla_bwd_workspace_size, gla_fwd, gla_profile_enable, gla_profile_read, gla_profile_reset
from . import gla_step, make_desc
from .inputs import DECODE, GSA_WORKLOAD, WORKLOADS, make_gsa_inputs, make_inputs, make_step_inputs

FLUSH_BYTES = 512 * 1024 * 1024


def _median_ms(fn, flush, reps):
    ts = []
    for _ in range(reps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    ts.sort()
    return ts[len(ts) // 2]


def time_layer(w, flush):
    inp = make_inputs(w.B, w.H, w.L, w.K, w.V, w.dtype, seed=0, z_mean=w.z_mean)
    d = {k: v.cuda() for k, v in inp.items() if v is not None}
    for mode in ("materialized", "nonmaterialized"):
        desc = make_desc(w.B, w.H, w.L, w.K, w.V, "bf16", 0, 0, mode, "auto")
        ws = torch.empty(gla_bwd_workspace_size(desc), dtype=torch.uint8, device="cuda")
        kw = dict(impl="auto", state_mode=mode)

        def fwd():
            gla_fwd(d["q"], d["k"], d["v"], d["log_a"], None, workspace=ws, **kw)

        def both():
            fwd()
            gla_bwd(d["q"], d["k"], d["v"], d["log_a"], d["dO"], None, None, workspace=ws, ws_from_fwd=True, **kw)

        for tag, fn in (("fwd", fwd), ("fwd+bwd", both)):
            for _ in range(3):
                fn()
            ms = _median_ms(fn, flush, 10)
            gla_profile_enable(True)
            gla_profile_reset()
            for _ in range(3):
                flush.zero_()
                fn()
            torch.cuda.synchronize()
            gla_profile_enable(False)
            per = {k: round(v[1] / v[0] * 1000, 1) for k, v in gla_profile_read().items()}
            print("%-16s %-15s %-8s %8.1f us  %8.2f Mtok/s  per kernel (us): %s"
                  % (w.name, mode, tag, ms * 1000, w.B * w.L / ms / 1e3, per), flush=True)


def time_gsa(flush, reps=10):
    from . import gsa

    W = GSA_WORKLOAD
    inp = make_gsa_inputs(W["B"], W["H"], W["L"], W["K"], W["V"], W["m"], W["dtype"], seed=0)
    d = {k: v.cuda() for k, v in inp.items()}
    desc = make_desc(W["B"], W["H"], W["L"], W["K"], W["V"], W["dtype"])
    ws = torch.empty(gsa.gsa_bwd_workspace_size(desc, W["m"]), dtype=torch.uint8, device="cuda")

    def fwd():
        gsa.gsa_fwd(d["q"], d["k"], d["v"], d["log_a"], workspace=ws)

    def both():
        fwd()
        gsa.gsa_bwd(d["q"], d["k"], d["v"], d["log_a"], d["dO"], workspace=ws, ws_from_fwd=True)

    for tag, fn in (("fwd", fwd), ("fwd+bwd", both)):
        for _ in range(3 if reps > 1 else 1):
            fn()
        ms = _median_ms(fn, flush, reps)
        per = {}
        if reps > 1:
            gla_profile_enable(True)
            gla_profile_reset()
            for _ in range(3):
                flush.zero_()
                fn()
            torch.cuda.synchronize()
            gla_profile_enable(False)
            per = {k: round(v[1] / v[0] * 1000, 1) for k, v in gla_profile_read().items()}
        print("%-16s %-15s %-8s %8.1f us  %8.2f Mtok/s  per kernel (us): %s"
              % (W["name"], gsa.gsa_route(desc, W["m"]), tag, ms * 1000, W["B"] * W["L"] / ms / 1e3, per), flush=True)


def time_decode(B, H, K, V, flush):
    st = make_step_inputs(B, H, K, V, 1, DECODE["dtype"], seed=0)
    q, k, v, la = (st[n][0].cuda() for n in ("q", "k", "v", "log_a"))
    S = torch.zeros(B, H, K, V, device="cuda")
    o = torch.empty(B, H, V, dtype=q.dtype, device="cuda")
    for _ in range(10):
        gla_step(q, k, v, la, S, o=o)
    torch.cuda.synchronize()
    state_bytes = 8 * B * H * K * V  # fp32 state read and written
    ms = _median_ms(lambda: gla_step(q, k, v, la, S, o=o), flush, 20)
    print("decode B=%-4d H=%d d_k=%d d_v=%d  cold   %8.2f us/step  %6.0f GB/s of state"
          % (B, H, K, V, ms * 1000, state_bytes / ms / 1e6), flush=True)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        gla_step(q, k, v, la, S, o=o)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(64):
            gla_step(q, k, v, la, S, o=o)
    graph.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(5):
        graph.replay()
    b.record()
    torch.cuda.synchronize()
    us = a.elapsed_time(b) / (5 * 64) * 1000
    print("decode B=%-4d H=%d d_k=%d d_v=%d  graph  %8.2f us/step  %6.0f GB/s of state"
          % (B, H, K, V, us, state_bytes / us / 1e3), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--only", nargs="*", default=None, help="workload names (and/or 'decode') to time")
    ap.add_argument("--list", action="store_true", help="list the workloads and exit")
    ap.add_argument("--reps", type=int, default=10, help="timed calls per case (gated slot attention)")
    args = ap.parse_args(argv)
    names = [n for n, w in WORKLOADS.items() if w.dtype == "bf16"] + [GSA_WORKLOAD["name"], "decode"]
    if args.list:
        for n in names:
            print(n, "-", WORKLOADS[n].note if n in WORKLOADS else
                  GSA_WORKLOAD["note"] if n == GSA_WORKLOAD["name"] else "decode step, B=64 and B=256")
        return 0
    if args.only:
        unknown = [n for n in args.only if n not in names]
        if unknown:
            ap.error("unknown workload(s): %s" % ", ".join(unknown))
        names = [n for n in names if n in args.only]
    if not torch.cuda.is_available():
        print("a CUDA device is required", file=sys.stderr)
        return 2
    flush = torch.empty(FLUSH_BYTES // 4, device="cuda")
    for n in names:
        if n == "decode":
            for B in (DECODE["B"], 4 * DECODE["B"]):
                time_decode(B, DECODE["H"], DECODE["K"], DECODE["V"], flush)
        elif n == GSA_WORKLOAD["name"]:
            time_gsa(flush, max(1, args.reps))
        else:
            time_layer(WORKLOADS[n], flush)
    return 0


if __name__ == "__main__":
    sys.exit(main())
