"""Gate kinds (include/gla.h, gla_gate): the per-head-and-step scalar decay and the fixed per-head
decay that the pages' ablations compare with the per-channel gate ("Gated Linear Attention
Transformers with Hardware-Efficient Training", atlas.scime.ai summary, "Measured effects"), and
the gate's pre-activation applied inside the kernels ("Approach": the gate is a function of the
input). The oracle takes the per-channel log alpha they stand for, computed here in fp64 on the
host; its per-channel gate gradient maps to each kind by the chain rule (sums over the channels
a scalar is shared by, or the factor sigmoid(-z)/tau of the pre-activation)."""
import numpy as np
import pytest
import torch

import chunkwise_linear_rnn_gla_b200 as gla
from chunkwise_linear_rnn_gla_b200 import _lib
from chunkwise_linear_rnn_gla_b200 import build as gbuild
from chunkwise_linear_rnn_gla_b200.inputs import make_inputs, make_step_inputs, to_f64_numpy
from tests.parity import compare

TAU = 16.0


@pytest.fixture(scope="module", autouse=True)
def _built():
    gbuild.build()
    gla.load()


def gate_inputs(kind, B, H, L, K, seed):
    """The caller's gate argument of each kind (fp32) and the per-channel log alpha it stands for (fp64)."""
    g = torch.Generator().manual_seed(seed)
    if kind == "scalar":
        arg = torch.nn.functional.logsigmoid(torch.randn(B, H, L, generator=g)) / TAU
        pc = np.broadcast_to(to_f64_numpy(arg)[..., None], (B, H, L, K))
    elif kind == "head":
        arg = -torch.rand(H, generator=g) * 0.2 - 0.01  # fixed decays gamma_h = e^{arg} in (0.82, 0.99)
        pc = np.broadcast_to(to_f64_numpy(arg)[None, :, None, None], (B, H, L, K))
    elif kind == "preact":
        arg = torch.randn(B, H, L, K, generator=g) * 2.0
        z = to_f64_numpy(arg)
        pc = (np.minimum(z, 0.0) - np.log1p(np.exp(-np.abs(z)))) / TAU  # logsigmoid(z) / tau in fp64
    else:
        raise ValueError(kind)
    return arg.float().contiguous(), np.ascontiguousarray(pc)


def grad_of_kind(kind, arg, dpc):
    """The caller's gate gradient from the oracle's per-channel one (chain rule)."""
    if kind == "scalar":
        return dpc.sum(axis=3)
    if kind == "head":
        return dpc.sum(axis=(0, 2, 3))
    z = to_f64_numpy(arg)
    return dpc / (1.0 + np.exp(z)) / TAU


def compare_f32_reduced(name, gpu, kind, dpc):
    """fp32 tolerance for a gradient that is a SUM of n per-channel terms (scalar: n = d_k per step;
    head: n = B*L*d_k per head): the stated absolute 1e-4 bounds one term's error; independent
    rounding errors of n terms add up as sqrt(n), so the bound for the sum is 1e-4 * sqrt(n)."""
    axes = (3,) if kind == "scalar" else (0, 2, 3)
    ref = dpc.sum(axis=axes)
    n = int(np.prod([dpc.shape[a] for a in axes]))
    g = to_f64_numpy(gpu)
    assert g.shape == ref.shape and np.all(np.isfinite(g))
    err = np.abs(g - ref).max()
    assert err <= 1e-4 * np.sqrt(n), "%s: max abs err %.3e > 1e-4 * sqrt(%d)" % (name, err, n)


def _oracle(inp, pc):
    import oracle

    f = lambda n: None if inp.get(n) is None else to_f64_numpy(inp[n])  # noqa: E731
    o, hT = oracle.fwd(f("q"), f("k"), f("v"), pc, f("h0"))
    g = oracle.bwd(f("q"), f("k"), f("v"), pc, f("dO"), f("h0"), f("dhT"))
    return o, hT, g


def test_gate_kind_validation():
    lib = _lib.load()
    import ctypes

    base = dict(B=1, H=2, L=64, Dk=64, Dv=64, dtype=0, chunk=0, subchunk=0, state_mode=0, impl=0, flags=0)
    ok = lambda **kw: lib.gla_fwd_workspace_size(ctypes.byref(_lib.GlaDesc(**{**base, **kw}))) > 0  # noqa: E731
    assert ok(gate=0) and ok(gate=1) and ok(gate=2) and ok(gate=3, gate_tau=16.0)
    assert not ok(gate=3, gate_tau=0.0) and not ok(gate=3, gate_tau=-1.0) and not ok(gate=4)
    assert not ok(gate=3, gate_tau=float("nan")) and not ok(gate=3, gate_tau=float("inf"))


@pytest.mark.gpu
@pytest.mark.parametrize("impl,dtype,K,V", [("tc", "bf16", 128, 128), ("tc", "bf16", 256, 64),
                                            ("simt", "f32", 64, 64), ("simt", "bf16", 64, 96)])
@pytest.mark.parametrize("kind", ["scalar", "head", "preact"])
def test_gate_kind_matches_oracle(kind, impl, dtype, K, V):
    B, H, L = 2, 2, 300
    inp = make_inputs(B, H, L, K, V, dtype, seed=50 + K, h0=True, dhT=True)
    arg, pc = gate_inputs(kind, B, H, L, K, seed=51)
    o_ref, hT_ref, ref = _oracle(inp, pc)
    d = {n: t.cuda() for n, t in inp.items()}
    a = arg.cuda()
    kw = dict(impl=impl, gate=kind, tau=TAU)
    o, hT = gla.gla_fwd(d["q"], d["k"], d["v"], a, d["h0"], **kw)
    g = gla.gla_bwd(d["q"], d["k"], d["v"], a, d["dO"], d["h0"], d["dhT"], **kw)
    torch.cuda.synchronize()
    compare("o", o, o_ref, dtype)
    compare("hT", hT, hT_ref, dtype)
    for n in ("dq", "dk", "dv", "dh0"):
        compare(n, g[n], ref[n], dtype)
    assert tuple(g["dlog_a"].shape) == tuple(arg.shape)
    if dtype == "f32" and kind in ("scalar", "head"):
        compare_f32_reduced("dlog_a (%s)" % kind, g["dlog_a"], kind, ref["dlog_a"])
    else:
        compare("dlog_a (%s)" % kind, g["dlog_a"], grad_of_kind(kind, arg, ref["dlog_a"]), dtype)


@pytest.mark.gpu
@pytest.mark.parametrize("kind", ["scalar", "head", "preact"])
def test_gate_kind_workspace_reuse(kind):
    """A backward that reuses the forward's workspace (gate expansion included) gives the result of a
    backward that recomputes everything."""
    B, H, L, K, V = 1, 2, 260, 128, 128
    inp = make_inputs(B, H, L, K, V, "bf16", seed=52, h0=True, dhT=True)
    arg, _ = gate_inputs(kind, B, H, L, K, seed=53)
    d = {n: t.cuda() for n, t in inp.items()}
    a = arg.cuda()
    desc = gla.make_desc(B, H, L, K, V, "bf16", gate=kind, tau=TAU)
    ws = torch.empty(gla.gla_bwd_workspace_size(desc), dtype=torch.uint8, device="cuda")
    kw = dict(gate=kind, tau=TAU)
    gla.gla_fwd(d["q"], d["k"], d["v"], a, d["h0"], workspace=ws, **kw)
    g1 = gla.gla_bwd(d["q"], d["k"], d["v"], a, d["dO"], d["h0"], d["dhT"], workspace=ws, ws_from_fwd=True, **kw)
    g2 = gla.gla_bwd(d["q"], d["k"], d["v"], a, d["dO"], d["h0"], d["dhT"], **kw)
    torch.cuda.synchronize()
    for key in g1:
        assert torch.equal(g1[key], g2[key]), key


@pytest.mark.gpu
@pytest.mark.parametrize("kind", ["channel", "scalar", "head", "preact"])
def test_gate_kind_decode_step(kind):
    import oracle

    B, H, K, V, T = 3, 2, 64, 96, 6
    st = make_step_inputs(B, H, K, V, T, "bf16", seed=54)
    S = torch.zeros(B, H, K, V, device="cuda")
    S_ref = np.zeros((B, H, K, V))
    for t in range(T):
        if kind == "channel":
            arg = st["log_a"][t]
            pc = to_f64_numpy(arg)
        else:
            a4, pc4 = gate_inputs(kind, B, H, 1, K, seed=55 + t)
            arg = a4[:, :, 0] if kind in ("scalar", "preact") else a4
            pc = pc4[:, :, 0]
        o = gla.gla_step(st["q"][t].cuda(), st["k"][t].cuda(), st["v"][t].cuda(), arg.contiguous().cuda(), S,
                         gate=kind, tau=TAU)
        o_ref, S_ref = oracle.step(to_f64_numpy(st["q"][t]), to_f64_numpy(st["k"][t]), to_f64_numpy(st["v"][t]),
                                   np.ascontiguousarray(pc), S_ref)
        torch.cuda.synchronize()
        compare("o_%d" % t, o, o_ref, "bf16")
    compare("S", S, S_ref, "bf16")


@pytest.mark.gpu
@pytest.mark.parametrize("kind", ["scalar", "head"])
def test_scalar_gates_beyond_the_range_bound(kind):
    """Scalar decays strong enough that a chunk's decay is far below e^-64 (per-step log decay down to
    -2, and a zero gate mid-chunk for the scalar kind): the tensor-core path weights each intra term by
    its decay in fp32 (factors <= 1) and needs no range bound; forward and backward match the oracle."""
    B, H, L, K, V = 1, 2, 300, 128, 64
    inp = make_inputs(B, H, L, K, V, "bf16", seed=56, h0=True, dhT=True)
    g = torch.Generator().manual_seed(57)
    if kind == "scalar":
        arg = -torch.rand(B, H, L, generator=g) * 2.0
        arg[0, 0, 150] = -1e30  # alpha = 0: exact forgetting
        pc = np.broadcast_to(to_f64_numpy(arg)[..., None], (B, H, L, K))
    else:
        arg = torch.tensor([-1.5, -0.7])
        pc = np.broadcast_to(to_f64_numpy(arg)[None, :, None, None], (B, H, L, K))
    pc = np.ascontiguousarray(pc)
    o_ref, hT_ref, ref = _oracle(inp, pc)
    d = {n: t.cuda() for n, t in inp.items()}
    a = arg.float().contiguous().cuda()
    o, hT = gla.gla_fwd(d["q"], d["k"], d["v"], a, d["h0"], impl="tc", gate=kind)
    gr = gla.gla_bwd(d["q"], d["k"], d["v"], a, d["dO"], d["h0"], d["dhT"], impl="tc", gate=kind)
    torch.cuda.synchronize()
    compare("o", o, o_ref, "bf16")
    compare("hT", hT, hT_ref, "bf16")
    for n in ("dq", "dk", "dv", "dh0"):
        compare(n, gr[n], ref[n], "bf16")
    compare("dlog_a (%s)" % kind, gr["dlog_a"], grad_of_kind(kind, arg, ref["dlog_a"]), "bf16")


@pytest.mark.gpu
@pytest.mark.parametrize("kind", ["scalar", "head", "preact", "channel"])
@pytest.mark.parametrize("L", [1, 131])
def test_gate_kinds_short_and_ragged(kind, L):
    """Every gate kind on the tensor-core path at L = 1 (one partial chunk) and a ragged L, with h0 and
    dhT; the pre-activation and the per-channel kinds also with two-level chunking."""
    B, H, K, V = 1, 2, 128, 64
    inp = make_inputs(B, H, L, K, V, "bf16", seed=58 + L, h0=True, dhT=True)
    if kind == "channel":
        arg = inp["log_a"]
        pc = to_f64_numpy(arg)
    else:
        arg, pc = gate_inputs(kind, B, H, L, K, seed=59 + L)
    o_ref, hT_ref, ref = _oracle(inp, np.ascontiguousarray(pc))
    d = {n: t.cuda() for n, t in inp.items()}
    a = arg.contiguous().cuda()
    for sc in ((0, 16) if kind in ("preact", "channel") else (0,)):
        kw = dict(impl="tc", gate=kind, tau=TAU, subchunk=sc)
        o, hT = gla.gla_fwd(d["q"], d["k"], d["v"], a, d["h0"], **kw)
        g = gla.gla_bwd(d["q"], d["k"], d["v"], a, d["dO"], d["h0"], d["dhT"], **kw)
        torch.cuda.synchronize()
        compare("o", o, o_ref, "bf16")
        compare("hT", hT, hT_ref, "bf16")
        for n in ("dq", "dk", "dv", "dh0"):
            compare(n, g[n], ref[n], "bf16")
        compare("dlog_a (%s)" % kind, g["dlog_a"], grad_of_kind(kind, arg, ref["dlog_a"]) if kind != "channel"
                else ref["dlog_a"], "bf16")
