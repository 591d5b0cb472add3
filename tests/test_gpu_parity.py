"""GPU parity: the CUDA path through the C ABI against the fp64 oracle, on the
same seeded inputs, element by element.

Small cases and the full-size named workloads (in the launch configuration
the benchmark times) both compare every output of every head with the oracle.
"""
import numpy as np
import pytest
import torch

import chunkwise_linear_rnn_gla_b200 as gla
from chunkwise_linear_rnn_gla_b200 import build as gbuild
from chunkwise_linear_rnn_gla_b200.inputs import DECODE, WORKLOADS, make_inputs, make_step_inputs, to_f64_numpy
from tests.parity import compare, heads, oracle_bwd, oracle_fwd, to_dev

pytestmark = pytest.mark.gpu

IMPLS = ["simt"]


@pytest.fixture(scope="module", autouse=True)
def _built():
    gbuild.build()
    gla.load()


def run_fwd(d, impl="auto", **kw):
    o, hT = gla.gla_fwd(d["q"], d["k"], d["v"], d["log_a"], d.get("h0"), impl=impl, **kw)
    torch.cuda.synchronize()
    return o, hT


def run_bwd(d, impl="auto", **kw):
    g = gla.gla_bwd(d["q"], d["k"], d["v"], d["log_a"], d["dO"], d.get("h0"), d.get("dhT"), impl=impl, **kw)
    torch.cuda.synchronize()
    return g


def check_fwd(inp, dtype, impl, idx=None, **kw):
    d = to_dev(inp)
    o, hT = run_fwd(d, impl, **kw)
    o_ref, hT_ref = oracle_fwd(inp, idx)
    if idx is not None:
        o, hT = heads(o, idx), heads(hT, idx)
    compare("o", o, o_ref, dtype)
    compare("hT", hT, hT_ref, dtype)


def check_bwd(inp, dtype, impl, idx=None, **kw):
    d = to_dev(inp)
    g = run_bwd(d, impl, **kw)
    ref = oracle_bwd(inp, idx)
    for name in ("dq", "dk", "dv", "dlog_a", "dh0"):
        val = g[name] if idx is None else heads(g[name], idx)
        compare(name, val, ref[name], dtype)


# ------------------------------------------------------------ small, all heads
@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("L", [1, 63, 64, 65, 200])
def test_small_shapes(impl, dtype, L):
    inp = make_inputs(2, 2, L, 64, 64, dtype, seed=L, h0=True, dhT=True)
    check_fwd(inp, dtype, impl)
    check_bwd(inp, dtype, impl)


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("chunk", [16, 32, 64, 128])
def test_chunk_size_invariance(impl, chunk):
    inp = make_inputs(1, 2, 300, 64, 128, "f32", seed=5, h0=True, dhT=True)
    check_fwd(inp, "f32", impl, chunk=chunk)
    check_bwd(inp, "f32", impl, chunk=chunk)


@pytest.mark.parametrize("subchunk", [1, 4, 16, 64])
def test_secondary_chunking_invariance(subchunk):
    """The CUDA-core path's two-level chunking: pairs in different sub-chunks as products of two
    factors <= 1 (rescaled at the end of the earlier sub-chunk), pairs inside one in log space. Every
    sub-chunk length gives the oracle's result (subchunk 64 = one sub-chunk per chunk, all log space),
    also with strong gates and a zero gate."""
    inp = make_inputs(1, 2, 300, 64, 128, "f32", seed=6, h0=True, dhT=True)
    check_fwd(inp, "f32", "simt", chunk=64, subchunk=subchunk)
    check_bwd(inp, "f32", "simt", chunk=64, subchunk=subchunk)
    strong = make_inputs(1, 1, 200, 64, 64, "f32", seed=7, gate_scale=1.0)
    strong["log_a"][0, 0, 100, :] = -1e30  # alpha = 0: exact forgetting
    check_fwd(strong, "f32", "simt", chunk=64, subchunk=subchunk)
    check_bwd(strong, "f32", "simt", chunk=64, subchunk=subchunk)


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("KV", [(32, 48), (128, 256), (96, 64)])
def test_head_dims(impl, KV):
    K, V = KV
    inp = make_inputs(1, 3, 130, K, V, "bf16", seed=K + V, h0=True, dhT=True)
    check_fwd(inp, "bf16", impl)
    check_bwd(inp, "bf16", impl)


@pytest.mark.parametrize("impl", IMPLS)
def test_zero_and_unit_gates(impl):
    inp = make_inputs(1, 2, 150, 64, 64, "f32", seed=11, h0=True, dhT=True)
    la = inp["log_a"].clone()
    la[:, 0] = -1e30  # head 0: alpha = 0 exactly
    la[:, 1] = 0.0  # head 1: alpha = 1 (no decay)
    inp["log_a"] = la
    check_fwd(inp, "f32", impl)
    check_bwd(inp, "f32", impl)


@pytest.mark.parametrize("impl", IMPLS)
def test_strong_mixed_gates(impl):
    # gates down to ~e^-5 per step: exercises the non-overflow guarantee
    inp = make_inputs(1, 2, 256, 64, 64, "bf16", seed=12, h0=True, dhT=True, gate_scale=1.0)
    check_fwd(inp, "bf16", impl)
    check_bwd(inp, "bf16", impl)


def test_ws_reuse_matches_recompute():
    inp = make_inputs(2, 2, 200, 64, 64, "f32", seed=13, h0=True, dhT=True)
    d = to_dev(inp)
    desc = gla.make_desc(2, 2, 200, 64, 64, "f32")
    ws = torch.empty(gla.gla_bwd_workspace_size(desc), dtype=torch.uint8, device="cuda")
    gla.gla_fwd(d["q"], d["k"], d["v"], d["log_a"], d["h0"], workspace=ws)
    g1 = gla.gla_bwd(d["q"], d["k"], d["v"], d["log_a"], d["dO"], d["h0"], d["dhT"], workspace=ws, ws_from_fwd=True)
    g2 = gla.gla_bwd(d["q"], d["k"], d["v"], d["log_a"], d["dO"], d["h0"], d["dhT"])
    torch.cuda.synchronize()
    for key in g1:
        assert torch.equal(g1[key], g2[key]), key


def test_chunk_cumsum_kernel():
    inp = make_inputs(2, 3, 333, 80, 8, "f32", seed=14, with_grad=False)
    la = inp["log_a"].cuda()
    for C in (16, 64, 128):
        out = gla.gla_chunk_cumsum(la, chunk=C)
        torch.cuda.synchronize()
        ref = np.zeros(la.shape)
        x = to_f64_numpy(inp["log_a"])
        for i0 in range(0, 333, C):
            ref[:, :, i0:i0 + C] = np.cumsum(x[:, :, i0:i0 + C], axis=2)
        np.testing.assert_allclose(to_f64_numpy(out), ref, rtol=0, atol=1e-5)


# ------------------------------------------------------------- decode step
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_step_matches_oracle(dtype):
    import oracle

    B, H, K, V, T = 4, 2, 64, 96, 20
    st = make_step_inputs(B, H, K, V, T, dtype, seed=15)
    S = torch.randn(B, H, K, V, generator=torch.Generator().manual_seed(1)) * 0.1
    S_ref = S.double().numpy()
    Sd = S.cuda()
    for t in range(T):
        o = gla.gla_step(st["q"][t].cuda(), st["k"][t].cuda(), st["v"][t].cuda(), st["log_a"][t].cuda(), Sd)
        o_ref, S_ref = oracle.step(to_f64_numpy(st["q"][t]), to_f64_numpy(st["k"][t]), to_f64_numpy(st["v"][t]),
                                   to_f64_numpy(st["log_a"][t]), S_ref)
        torch.cuda.synchronize()
        compare("o_%d" % t, o, o_ref, dtype)
    compare("S", Sd, S_ref, "f32" if dtype == "f32" else "bf16")


@pytest.mark.parametrize("K,V", [(100, 96), (200, 7), (1, 4), (200, 104), (8, 32), (256, 40), (64, 36)])
def test_step_ragged_rows_odd_columns(K, V):
    """Decode step with row counts that leave the last row batch or the last 128-row box partial,
    value widths that leave the last 32-column tile partial or need the scalar column path, and
    one or eight key channels."""
    import oracle

    B, H, T = 3, 2, 5
    st = make_step_inputs(B, H, K, V, T, "bf16", seed=18)
    S = torch.randn(B, H, K, V, generator=torch.Generator().manual_seed(2)) * 0.1
    S_ref = S.double().numpy()
    Sd = S.cuda()
    for t in range(T):
        o = gla.gla_step(st["q"][t].cuda(), st["k"][t].cuda(), st["v"][t].cuda(), st["log_a"][t].cuda(), Sd)
        o_ref, S_ref = oracle.step(to_f64_numpy(st["q"][t]), to_f64_numpy(st["k"][t]), to_f64_numpy(st["v"][t]),
                                   to_f64_numpy(st["log_a"][t]), S_ref)
        torch.cuda.synchronize()
        compare("o_%d" % t, o, o_ref, "bf16")
    compare("S", Sd, S_ref, "bf16")


def test_step_replays_from_cuda_graph():
    """Eight decode steps captured in a CUDA graph and replayed give the eager steps' outputs and
    state bit for bit (the steps are chained by programmatic dependent launch)."""
    B, H, K, V, T = 8, 4, 128, 256, 8
    st = make_step_inputs(B, H, K, V, T, "bf16", seed=20)
    q, k, v, la = (st[n].cuda() for n in ("q", "k", "v", "log_a"))
    S0 = torch.randn(B, H, K, V, generator=torch.Generator().manual_seed(3)).cuda() * 0.1
    S_e = S0.clone()
    outs_e = [gla.gla_step(q[t], k[t], v[t], la[t], S_e).clone() for t in range(T)]
    S_g = S0.clone()
    outs_g = [torch.empty(B, H, V, dtype=torch.bfloat16, device="cuda") for _ in range(T)]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        gla.gla_step(q[0], k[0], v[0], la[0], S0.clone(), o=outs_g[0])
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for t in range(T):
            gla.gla_step(q[t], k[t], v[t], la[t], S_g, o=outs_g[t])
    S_g.copy_(S0)
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(S_g, S_e)
    for t in range(T):
        assert torch.equal(outs_g[t], outs_e[t]), t


def test_step_rejects_a_misaligned_state():
    """A state 4 bytes past a 16-byte boundary is refused before any launch; the state is untouched."""
    B, H, K, V = 2, 2, 64, 96
    st = make_step_inputs(B, H, K, V, 1, "bf16", seed=19)
    buf = torch.ones(B * H * K * V + 4, device="cuda")
    Sd = buf[1:1 + B * H * K * V].view(B, H, K, V)
    with pytest.raises(gla.GlaError) as ei:
        gla.gla_step(st["q"][0].cuda(), st["k"][0].cuda(), st["v"][0].cuda(), st["log_a"][0].cuda(), Sd)
    assert "INVALID_ARG" in str(ei.value)
    torch.cuda.synchronize()
    assert bool((buf == 1).all())


def test_step_iterated_equals_fwd():
    B, H, L, K, V = 2, 2, 70, 64, 64
    inp = make_inputs(B, H, L, K, V, "f32", seed=16, h0=True)
    d = to_dev(inp)
    o, hT = run_fwd(d)
    S = d["h0"].clone()
    outs = []
    for t in range(L):
        outs.append(gla.gla_step(d["q"][:, :, t].contiguous(), d["k"][:, :, t].contiguous(),
                                 d["v"][:, :, t].contiguous(), d["log_a"][:, :, t].contiguous(), S))
    torch.cuda.synchronize()
    torch.testing.assert_close(torch.stack(outs, 2), o, atol=1e-4, rtol=0)
    torch.testing.assert_close(S, hT, atol=1e-4, rtol=0)


def test_decode_workload_sampled():
    """Decode workload shape (B=64, H=4, Dk=128, Dv=256, fp32 state): 16 steps,
    every head against the oracle."""
    import oracle

    B, H, K, V, T = 64, 4, 128, 256, 16
    st = make_step_inputs(B, H, K, V, T, "bf16", seed=17)
    Sd = torch.zeros(B, H, K, V, device="cuda")
    S_ref = np.zeros((B, H, K, V))
    for t in range(T):
        o = gla.gla_step(st["q"][t].cuda(), st["k"][t].cuda(), st["v"][t].cuda(), st["log_a"][t].cuda(), Sd)
        o_ref, S_ref = oracle.step(to_f64_numpy(st["q"][t]), to_f64_numpy(st["k"][t]), to_f64_numpy(st["v"][t]),
                                   to_f64_numpy(st["log_a"][t]), S_ref)
    torch.cuda.synchronize()
    compare("o_last", o, o_ref, "bf16")
    compare("S", Sd, S_ref, "bf16")


# ------------------------------------------------------- the named workloads
# Every named workload runs in the configuration the benchmark times, and every head of every output
# is compared with the oracle (heads are independent, so a wrong tile-to-head mapping anywhere shows).
_ORACLE_CACHE = {}


def _workload_reference(name, passes):
    """Inputs of a named workload (seed 0) and the oracle's outputs, computed once per module."""
    key = (name, passes)
    if key not in _ORACLE_CACHE:
        w = WORKLOADS[name]
        inp = make_inputs(w.B, w.H, w.L, w.K, w.V, w.dtype, seed=0, z_mean=w.z_mean, with_grad=(passes != "fwd"))
        ref_f = oracle_fwd(inp)
        ref_b = oracle_bwd(inp) if passes != "fwd" else None
        _ORACLE_CACHE.clear()  # keep one workload's arrays alive at a time
        _ORACLE_CACHE[key] = (inp, ref_f, ref_b)
    return _ORACLE_CACHE[key]


def check_workload(name, passes, **kw):
    w = WORKLOADS[name]
    inp, (o_ref, hT_ref), ref = _workload_reference(name, passes)
    d = to_dev(inp)
    o, hT = run_fwd(d, "auto", chunk=w.chunk, **kw)
    compare("o", o, o_ref, w.dtype)
    compare("hT", hT, hT_ref, w.dtype)
    del o, hT
    if ref is not None:
        g = run_bwd(d, "auto", chunk=w.chunk, **kw)
        for n in ("dq", "dk", "dv", "dlog_a", "dh0"):
            compare(n, g[n], ref[n], w.dtype)


def test_workload_tiny_f32():
    check_workload("tiny_f32", "fwd+bwd")


def test_workload_340m_fwd():
    """340M-layer shape, forward: all 32 heads."""
    check_workload("gla340m_fwd", "fwd")


def test_workload_340m_fwdbwd():
    """The same shape through the backward as well (all heads)."""
    check_workload("gla340m_fwd", "fwd+bwd")


def test_workload_1p3b_fwdbwd():
    """1.3B-layer shape, forward and backward: all 16 heads of every output."""
    check_workload("gla1p3b_fwdbwd", "fwd+bwd")


@pytest.mark.parametrize("mode", ["materialized", "nonmaterialized"])
def test_workload_long16k(mode):
    """Long sequence (L=16384, slow gates), materialised and non-materialised inter-chunk states: all
    four heads; both modes run the segmented walks at this shape."""
    check_workload("long16k", "fwd+bwd", state_mode=mode)


@pytest.mark.parametrize("L", [1024, 2048, 4096, 8192, 16384])
def test_workload_sweep(L):
    """16384 tokens per batch at every sweep length, forward and backward, all heads."""
    check_workload("sweep_L%d" % L, "fwd+bwd")


def test_decode_workload_4096_steps():
    """The decode workload in full: B=64, H=4, d_k=128, d_v=256, 4096 single-token steps with the fp32
    state carried on the device. Every step's output of every head and the final state are compared
    with the oracle's recurrence, which is run over the same inputs in blocks of 256 steps with its
    own fp64 state carried between blocks (the drift of the fp32 state over 4096 updates shows)."""
    import oracle

    B, H, K, V = (DECODE[n] for n in ("B", "H", "K", "V"))
    steps, blk = DECODE["steps"], 256
    S = torch.zeros(B, H, K, V, device="cuda")
    S_ref = np.zeros((B, H, K, V))
    for b0 in range(0, steps, blk):
        st = make_step_inputs(B, H, K, V, blk, DECODE["dtype"], seed=1000 + b0 // blk)
        dev = {n: st[n].cuda() for n in ("q", "k", "v", "log_a")}
        outs = torch.empty(blk, B, H, V, dtype=torch.bfloat16, device="cuda")
        for t in range(blk):
            gla.gla_step(dev["q"][t], dev["k"][t], dev["v"][t], dev["log_a"][t], S, o=outs[t])
        # the same steps as the oracle's recurrence over a block of length blk: [steps,B,H,.] -> [B,H,steps,.]
        seq = {n: to_f64_numpy(st[n]).transpose(1, 2, 0, 3) for n in ("q", "k", "v", "log_a")}
        o_ref, S_ref = oracle.fwd(seq["q"], seq["k"], seq["v"], seq["log_a"], S_ref)
        torch.cuda.synchronize()
        compare("o, steps %d..%d" % (b0, b0 + blk - 1), outs.permute(1, 2, 0, 3), o_ref, "bf16")
    compare("S after %d steps" % steps, S, S_ref, "bf16")


# ------------------------------------------------ tensor-core forward path
TC_SHAPES = [(1, 2, 1, 128, 64), (1, 2, 100, 128, 128), (2, 1, 128, 256, 64), (1, 2, 129, 128, 256),
             (1, 1, 300, 256, 128), (2, 2, 512, 128, 64)]


@pytest.mark.parametrize("mode", ["nonmaterialized", "materialized"])
@pytest.mark.parametrize("shape", TC_SHAPES)
def test_tc_forward(mode, shape):
    B, H, L, K, V = shape
    inp = make_inputs(B, H, L, K, V, "bf16", seed=L + K + V, h0=True, with_grad=False)
    check_fwd(inp, "bf16", "tc", state_mode=mode)


@pytest.mark.parametrize("mode", ["nonmaterialized", "materialized"])
def test_tc_forward_extreme_gates(mode):
    # head 0: alpha = 0 exactly; head 1: alpha = 1; head 2: strong decays (up to
    # ~e^-6 per step, so sub-chunk spans exceed the factored fp32 range)
    inp = make_inputs(1, 3, 260, 128, 64, "bf16", seed=21, h0=True, with_grad=False, gate_scale=1.0)
    la = inp["log_a"].clone()
    la[:, 0] = -1e30
    la[:, 1] = 0.0
    la[:, 2] = la[:, 2] * 3.0
    inp["log_a"] = la
    check_fwd(inp, "bf16", "tc", state_mode=mode)


def test_tc_matches_simt_forward():
    inp = make_inputs(2, 2, 700, 256, 128, "bf16", seed=22, h0=True, with_grad=False)
    d = to_dev(inp)
    o_tc, hT_tc = run_fwd(d, "tc")
    o_s, hT_s = run_fwd(d, "simt")
    compare("o tc-vs-simt", o_tc, to_f64_numpy(o_s), "bf16")
    compare("hT tc-vs-simt", hT_tc, to_f64_numpy(hT_s), "bf16")


# ----------------------------------------------- tensor-core backward path
@pytest.mark.parametrize("mode", ["nonmaterialized", "materialized"])
@pytest.mark.parametrize("shape", TC_SHAPES)
def test_tc_backward(mode, shape):
    B, H, L, K, V = shape
    inp = make_inputs(B, H, L, K, V, "bf16", seed=L + K + V + 1, h0=True, dhT=True)
    check_bwd(inp, "bf16", "tc", state_mode=mode)


@pytest.mark.parametrize("mode", ["nonmaterialized", "materialized"])
def test_tc_backward_extreme_gates(mode):
    inp = make_inputs(1, 3, 260, 128, 64, "bf16", seed=23, h0=True, dhT=True, gate_scale=1.0)
    la = inp["log_a"].clone()
    la[:, 0] = -1e30
    la[:, 1] = 0.0
    la[:, 2] = la[:, 2] * 3.0
    inp["log_a"] = la
    check_bwd(inp, "bf16", "tc", state_mode=mode)


@pytest.mark.parametrize("mode", ["nonmaterialized", "materialized"])
def test_tc_ws_reuse_matches_recompute(mode):
    inp = make_inputs(2, 2, 300, 256, 128, "bf16", seed=24, h0=True, dhT=True)
    d = to_dev(inp)
    desc = gla.make_desc(2, 2, 300, 256, 128, "bf16", impl="tc", state_mode=mode)
    ws = torch.empty(gla.gla_bwd_workspace_size(desc), dtype=torch.uint8, device="cuda")
    kw = dict(impl="tc", state_mode=mode)
    gla.gla_fwd(d["q"], d["k"], d["v"], d["log_a"], d["h0"], workspace=ws, **kw)
    g1 = gla.gla_bwd(d["q"], d["k"], d["v"], d["log_a"], d["dO"], d["h0"], d["dhT"], workspace=ws, ws_from_fwd=True,
                     **kw)
    g2 = gla.gla_bwd(d["q"], d["k"], d["v"], d["log_a"], d["dO"], d["h0"], d["dhT"], **kw)
    torch.cuda.synchronize()
    for key in g1:
        assert torch.equal(g1[key], g2[key]), key


def test_tc_backward_matches_simt():
    inp = make_inputs(1, 2, 400, 256, 128, "bf16", seed=25, h0=True, dhT=True)
    d = to_dev(inp)
    g_tc = run_bwd(d, "tc")
    g_s = run_bwd(d, "simt")
    for key in ("dq", "dk", "dv", "dlog_a", "dh0"):
        compare(key + " tc-vs-simt", g_tc[key], to_f64_numpy(g_s[key]), "bf16")


@pytest.mark.parametrize("mode", ["materialized", "nonmaterialized"])
def test_tc_step_replays_from_cuda_graph(mode):
    """The fwd+bwd step captured into a CUDA graph and replayed gives the eager results bit for bit
    (the kernels read and write fixed buffers; nothing in the path allocates or synchronises)."""
    B, H, L, K, V = 2, 2, 300, 256, 128
    inp = make_inputs(B, H, L, K, V, "bf16", seed=26, h0=True, dhT=True)
    d = to_dev(inp)
    desc = gla.make_desc(B, H, L, K, V, "bf16", impl="tc", state_mode=mode)
    ws = torch.empty(gla.gla_bwd_workspace_size(desc), dtype=torch.uint8, device="cuda")
    kw = dict(impl="tc", state_mode=mode)
    o = torch.empty_like(d["v"])
    hT = torch.empty(B, H, K, V, device="cuda")
    outs = {"dq": torch.empty_like(d["q"]), "dk": torch.empty_like(d["k"]), "dv": torch.empty_like(d["v"]),
            "dlog_a": torch.empty_like(d["log_a"]), "dh0": torch.empty(B, H, K, V, device="cuda")}

    def step():
        gla.gla_fwd(d["q"], d["k"], d["v"], d["log_a"], d["h0"], o=o, hT=hT, workspace=ws, **kw)
        gla.gla_bwd(d["q"], d["k"], d["v"], d["log_a"], d["dO"], d["h0"], d["dhT"], workspace=ws, ws_from_fwd=True,
                    out=outs, **kw)

    step()
    torch.cuda.synchronize()
    eager = {"o": o.clone(), "hT": hT.clone(), **{k: v.clone() for k, v in outs.items()}}
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for t in [o, hT, *outs.values()]:
        t.zero_()
    g.replay()
    torch.cuda.synchronize()
    got = {"o": o, "hT": hT, **outs}
    for key in eager:
        assert torch.equal(got[key], eager[key]), key



@pytest.mark.parametrize("mode", ["materialized", "nonmaterialized"])
@pytest.mark.parametrize("z_mean", [0.0, 2.0])
def test_tc_segmented_state_walk(z_mean, mode):
    """Few heads and many chunks: the state walks (materialised, and the fused non-materialised walks)
    run as parallel segments (a zero-start pass, a scan over the segment end states, a second pass
    from the true entering states). Ragged last chunk, nonzero h0 and dhT, slow (z_mean=2) and
    ordinary gates; fwd and bwd against the oracle."""
    B, H, L, K, V = 1, 2, 128 * 20 + 37, 128, 128
    inp = make_inputs(B, H, L, K, V, "bf16", seed=28, z_mean=z_mean, h0=True, dhT=True)
    check_fwd(inp, "bf16", "tc", state_mode=mode)
    check_bwd(inp, "bf16", "tc", state_mode=mode)


def test_bounded_wait_timeout_is_reported_and_the_context_survives():
    """Failure detection without a GPU fault: a kernel whose mbarrier wait nothing completes gives up
    after its bound, the host reads GLA_ERR_TIMEOUT (once; the flag is cleared), and the same context
    then runs the layer correctly."""
    torch.cuda.synchronize()
    assert gla.gla_check_device_error() == 0
    gla.gla_selftest_wait_timeout()
    assert gla.gla_check_device_error() == 5  # GLA_ERR_TIMEOUT
    assert gla.gla_check_device_error() == 0
    inp = make_inputs(1, 2, 300, 128, 128, "bf16", seed=29)
    check_fwd(inp, "bf16", "tc", state_mode="materialized")
    assert gla.gla_check_device_error() == 0


@pytest.mark.parametrize("impl", ["simt", "tc"])
def test_single_zero_gate_mid_chunk(impl):
    """A zero gate (alpha = 0, log alpha = -1e30) in the middle of a chunk, ordinary gates after it:
    exact forgetting, and the decay among the later steps of the same chunk must not be lost to the
    huge cumulative sum."""
    dt = "f32" if impl == "simt" else "bf16"
    K, V = (64, 64) if impl == "simt" else (128, 128)
    inp = make_inputs(1, 2, 300, K, V, dt, seed=30, gate_scale=1.0, h0=True, dhT=True)
    inp["log_a"][0, 0, 100, :] = -1e30
    inp["log_a"][0, 1, 170, : K // 2] = -1e30
    kw = dict(state_mode="materialized") if impl == "tc" else {}
    check_fwd(inp, dt, impl, **kw)
    check_bwd(inp, dt, impl, **kw)


# ------------------------------------ two-level (secondary) chunking on the tensor-core path
@pytest.mark.parametrize("shape", [(1, 2, 129, 128, 64), (1, 1, 300, 256, 128), (2, 2, 512, 128, 64)])
def test_tc_two_level_intra_chunks(shape):
    """Sub-chunk length 16 on the tensor-core path: off-diagonal 16-row blocks as bf16 tcgen05 GEMMs
    with both factors rescaled to <= 1 against each key sub-chunk's last row, diagonal blocks in fp32
    log space; forward and backward against the oracle, with strong gates, a zero gate and ragged L."""
    B, H, L, K, V = shape
    inp = make_inputs(B, H, L, K, V, "bf16", seed=L + K + 7, h0=True, dhT=True, gate_scale=1.0)
    inp["log_a"][0, 0, L // 2, : K // 2] = -1e30
    check_fwd(inp, "bf16", "tc", subchunk=16)
    check_bwd(inp, "bf16", "tc", subchunk=16)


def _straddling_gates(B, H, L, K, seed):
    """Gates whose decay over a 128-step chunk, Gamma_c, is spread over [-70, -58] across the key
    channels: both sides of the -64 bound of the single-GEMM form."""
    g = torch.Generator().manual_seed(seed)
    target = -58.0 - 12.0 * torch.rand(B, H, 1, K, generator=g)  # chunk decay per channel
    jitter = 1.0 + 0.5 * (torch.rand(B, H, L, K, generator=g) - 0.5)
    return (target / 128.0 * jitter).float().contiguous()


def test_two_level_vs_single_gemm_accuracy():
    """The accuracy side of the comparison of the two intra-chunk forms on the 1.3B layer shape (one
    batch row): gates straddling the single-GEMM form's range bound. Both forms meet the tolerance;
    the errors against the oracle are printed for the comparison table."""
    w = WORKLOADS["gla1p3b_fwdbwd"]
    B, H, L, K, V = 1, w.H, w.L, w.K, w.V
    inp = make_inputs(B, H, L, K, V, "bf16", seed=70, with_grad=True)
    inp["log_a"] = _straddling_gates(B, H, L, K, seed=71)
    o_ref, hT_ref = oracle_fwd(inp)
    ref = oracle_bwd(inp)
    d = to_dev(inp)
    errs = {}
    for sc in (128, 16):
        o, hT = run_fwd(d, "tc", subchunk=sc)
        g = run_bwd(d, "tc", subchunk=sc)
        e = {"o": compare("o (subchunk %d)" % sc, o, o_ref, "bf16"),
             "hT": compare("hT (subchunk %d)" % sc, hT, hT_ref, "bf16")}
        for n in ("dq", "dk", "dv", "dlog_a", "dh0"):
            e[n] = compare("%s (subchunk %d)" % (n, sc), g[n], ref[n], "bf16")
        errs[sc] = e
    print("\nmax |gpu - oracle| / max |oracle| with straddling gates:")
    for sc, e in errs.items():
        print("  subchunk %3d: " % sc + "  ".join("%s %.3e" % kv for kv in e.items()))
