"""Gated slot attention on the GPU against the fp64 GSA oracle (element by element, every head).

The method: the mlsanity card for "Gated Slot Attention for Efficient Linear-Time Sequence Modeling"
(abstract); the library evaluates it as GLA passes of its own kernels plus elementwise kernels
(include/gla.h, gated slot attention). Tolerances as for the GLA layer: fp32 max |err| <= 1e-4,
bf16 max |err| / max |ref| <= 2e-2, per output tensor.
"""
import numpy as np
import pytest
import torch

import oracle
from chunkwise_linear_rnn_gla_b200 import _lib, make_desc
from chunkwise_linear_rnn_gla_b200 import gsa
from chunkwise_linear_rnn_gla_b200.inputs import GSA_WORKLOAD, make_gsa_inputs, to_f64_numpy
from tests.parity import compare, to_dev

pytestmark = pytest.mark.gpu


def run_oracle(inp, fwd_only=False):
    f = lambda n: None if inp.get(n) is None else to_f64_numpy(inp[n])  # noqa: E731
    o, s, hkT, hvT = oracle.gsa_fwd(f("q"), f("k"), f("v"), f("log_a"), f("hk0"), f("hv0"))
    ref = {"o": o, "hkT": hkT, "hvT": hvT}
    if not fwd_only:
        ref.update(oracle.gsa_bwd(f("q"), f("k"), f("v"), f("log_a"), f("dO"), f("hk0"), f("hv0"), f("dhkT"),
                                  f("dhvT")))
    return ref


def run_gpu(inp, reuse=True, **kw):
    d = to_dev(inp)
    B, H, L, Dk = d["q"].shape
    m = d["log_a"].shape[-1]
    desc = make_desc(B, H, L, Dk, d["v"].shape[-1], "bf16" if d["q"].dtype == torch.bfloat16 else "f32")
    ws = torch.empty(gsa.gsa_bwd_workspace_size(desc, m), dtype=torch.uint8, device="cuda")
    o, hkT, hvT = gsa.gsa_fwd(d["q"], d["k"], d["v"], d["log_a"], d.get("hk0"), d.get("hv0"), want_state=True,
                              workspace=ws, **kw)
    g = gsa.gsa_bwd(d["q"], d["k"], d["v"], d["log_a"], d["dO"], d.get("hk0"), d.get("hv0"), d.get("dhkT"),
                    d.get("dhvT"), want_dh0=True, workspace=ws, ws_from_fwd=reuse, **kw)
    torch.cuda.synchronize()
    return {"o": o, "hkT": hkT, "hvT": hvT, **g}


def check_all(inp, dtype, names=("o", "hkT", "hvT", "dq", "dk", "dv", "dlog_a", "dhk0", "dhv0"), **kw):
    gpu = run_gpu(inp, **kw)
    ref = run_oracle(inp)
    errs = {}
    for n in names:
        errs[n] = compare(n, gpu[n], ref[n], dtype)
    return errs


def route_of(inp):
    B, H, L, Dk = inp["q"].shape
    m = inp["log_a"].shape[-1]
    dt = "bf16" if inp["q"].dtype == torch.bfloat16 else "f32"
    return gsa.gsa_route(make_desc(B, H, L, Dk, inp["v"].shape[-1], dt), m)


# ---------------------------------------------------------------- CUDA-core path (fp32)
@pytest.mark.parametrize("state", [False, True])
def test_gsa_f32_ragged(state):
    inp = make_gsa_inputs(1, 2, 300, 64, 32, 16, "f32", seed=1, q_scale=4.0, h0=state, dhT=state)
    assert route_of(inp) == "simt"
    check_all(inp, "f32")


def test_gsa_f32_one_step():
    inp = make_gsa_inputs(2, 1, 1, 32, 48, 8, "f32", seed=2, q_scale=4.0, h0=True, dhT=True)
    check_all(inp, "f32")


# ---------------------------------------------------------------- tensor-core path (bf16, m = 128 or 256)
@pytest.mark.parametrize("L,Dk,Dv", [(600, 128, 128), (389, 256, 512), (256, 64, 192), (1, 128, 128), (129, 128, 64)])
def test_gsa_bf16_tensor_core(L, Dk, Dv):
    inp = make_gsa_inputs(1, 2, L, Dk, Dv, 128, "bf16", seed=3, q_scale=4.0, h0=True, dhT=True)
    assert route_of(inp) == "tc"
    check_all(inp, "bf16")


def test_gsa_bf16_peaked_softmax_and_extreme_gates():
    """Strongly peaked read weights (q scaled by 16) and a wide gate spread with near-zero gates, so that
    whole chunks decay past the tensor-core path's range bound and take its exact path."""
    inp = make_gsa_inputs(1, 2, 517, 128, 128, 128, "bf16", seed=4, q_scale=16.0, gate_scale=2.0)
    assert route_of(inp) == "tc"
    check_all(inp, "bf16", names=("o", "hkT", "hvT", "dq", "dk", "dv", "dlog_a"))


def test_gsa_bf16_gates_straddling_the_range_bound():
    """Gates whose chunk decays straddle the tensor-core route's range bound: about half of the slots of
    every full chunk pass it, so the masked scores of the next layer, formed in the slot reads, add their
    exact log-space terms to the tensor-core product within the same chunk (L = 389: a ragged last chunk)."""
    inp = make_gsa_inputs(1, 2, 389, 128, 128, 128, "bf16", seed=9, q_scale=4.0, gate_scale=0.62, h0=True,
                          dhT=True)
    la = inp["log_a"][0]
    frac = [(la[:, i:i + 128].sum(1) < -64).float().mean().item() for i in range(0, 384, 128)]
    assert all(0.3 < f < 0.7 for f in frac), frac
    assert route_of(inp) == "tc"
    check_all(inp, "bf16")


@pytest.mark.parametrize("L,Dk,Dv,m", [(333, 128, 64, 64), (256, 64, 192, 256)])
def test_gsa_bf16_cuda_core_slots(L, Dk, Dv, m):
    """Slot counts other than 128: bf16 tensors on the CUDA-core route (fp32 GLA passes)."""
    inp = make_gsa_inputs(1, 2, L, Dk, Dv, m, "bf16", seed=5, q_scale=4.0, h0=True, dhT=True)
    assert route_of(inp) == "simt"
    check_all(inp, "bf16")


def test_gsa_backward_reuse_matches_recompute():
    inp = make_gsa_inputs(1, 2, 300, 128, 128, 128, "bf16", seed=6, q_scale=4.0)
    a = run_gpu(inp, reuse=True)
    b = run_gpu(inp, reuse=False)
    for n in ("dq", "dk", "dv", "dlog_a"):
        assert torch.equal(a[n], b[n]), n


def test_gsa_zero_gate_copies_v():
    """a = 0 everywhere: every slot holds (k_t, v_t), so o_t = v_t (up to the bf16 rounding of the output)."""
    inp = make_gsa_inputs(1, 2, 200, 128, 128, 128, "bf16", seed=7)
    inp["log_a"] = torch.full_like(inp["log_a"], -1e30)
    gpu = run_gpu(inp)
    compare("o", gpu["o"], to_f64_numpy(inp["v"]), "bf16")


def test_gsa_checks_report_bad_gate():
    inp = make_gsa_inputs(1, 1, 130, 128, 128, 128, "bf16", seed=8)
    inp["log_a"][0, 0, 5, 3] = 0.5
    d = to_dev(inp)
    with pytest.raises(_lib.GlaError) as e:
        gsa.gsa_fwd(d["q"], d["k"], d["v"], d["log_a"], checks=True)
    assert e.value.status == _lib.GLA_ERR_INVALID_ARG


# ---------------------------------------------------------------- the named workload, every head
def test_gsa_workload_full_size():
    w = GSA_WORKLOAD
    inp = make_gsa_inputs(w["B"], w["H"], w["L"], w["K"], w["V"], w["m"], w["dtype"], seed=0)
    assert route_of(inp) == "tc"
    errs = check_all(inp, "bf16", names=("o", "dq", "dk", "dv", "dlog_a"))
    print("gsa workload relative errors", {k: "%.2e" % v for k, v in errs.items()})


# ---------------------------------------------------------------- decode step
@pytest.mark.parametrize("dtype,Dk,Dv,m", [("f32", 64, 32, 16), ("f32", 96, 40, 24), ("bf16", 128, 256, 128),
                                           ("bf16", 256, 512, 128), ("f32", 32, 20, 5), ("bf16", 4, 4, 3)])
def test_gsa_step_matches_oracle(dtype, Dk, Dv, m):
    """T single-token steps from given memories equal the oracle over those T tokens (o at every step, the
    final memories)."""
    B, H, T = 2, 2, 12
    inp = make_gsa_inputs(B, H, T, Dk, Dv, m, dtype, seed=9, q_scale=4.0, h0=True)
    d = to_dev(inp)
    hk, hv = d["hk0"].clone(), d["hv0"].clone()
    outs = [gsa.gsa_step(*(d[n][:, :, t].contiguous() for n in ("q", "k", "v", "log_a")), hk, hv) for t in range(T)]
    torch.cuda.synchronize()
    ref = run_oracle(inp, fwd_only=True)
    compare("o", torch.stack(outs, dim=2), ref["o"], dtype)
    compare("hkT", hk, ref["hkT"], dtype)
    compare("hvT", hv, ref["hvT"], dtype)


def test_gsa_step_continues_the_forward():
    """The forward's final memories (tensor-core route) continued by decode steps give the oracle's outputs
    and memories over the whole sequence."""
    B, H, L, T, Dk, Dv, m = 1, 2, 300, 5, 128, 128, 128
    inp = make_gsa_inputs(B, H, L + T, Dk, Dv, m, "bf16", seed=10, q_scale=4.0)
    d = to_dev(inp)
    pre = {n: d[n][:, :, :L].contiguous() for n in ("q", "k", "v", "log_a")}
    assert route_of(pre) == "tc"
    o, hk, hv = gsa.gsa_fwd(pre["q"], pre["k"], pre["v"], pre["log_a"], want_state=True)
    outs = [gsa.gsa_step(*(d[n][:, :, L + t].contiguous() for n in ("q", "k", "v", "log_a")), hk, hv)
            for t in range(T)]
    torch.cuda.synchronize()
    ref = run_oracle(inp, fwd_only=True)
    compare("o (forward)", o, ref["o"][:, :, :L], "bf16")
    compare("o (steps)", torch.stack(outs, dim=2), ref["o"][:, :, L:], "bf16")
    compare("hkT", hk, ref["hkT"], "bf16")
    compare("hvT", hv, ref["hvT"], "bf16")


# ---------------------------------------------------------------- pre-activation gate
@pytest.mark.parametrize("dtype,Dk,Dv,m", [("bf16", 128, 128, 128), ("f32", 64, 32, 16)])
def test_gsa_preact_gate(dtype, Dk, Dv, m):
    """gate="preact": the caller passes z, log a = logsigmoid(z) / tau; the backward returns
    dL/dz = dL/dlog a * sigmoid(-z) / tau. Against the oracle run on log a, on both routes: forward,
    backward and a decode step continuing the forward's memories."""
    tau = 8.0
    inp = make_gsa_inputs(1, 2, 333, Dk, Dv, m, dtype, seed=11, q_scale=4.0, h0=True, dhT=True)
    z = torch.randn(inp["log_a"].shape, generator=torch.Generator().manual_seed(12)) * 2.0
    inp["log_a"] = (torch.nn.functional.logsigmoid(z) / tau).float()  # what the oracle reads
    zz = z.numpy().astype(np.float64)
    ref = run_oracle(inp)
    d = to_dev(inp)
    zd = z.float().contiguous().to("cuda")
    kw = dict(gate="preact", tau=tau)
    o, hkT, hvT = gsa.gsa_fwd(d["q"], d["k"], d["v"], zd, d["hk0"], d["hv0"], want_state=True, **kw)
    g = gsa.gsa_bwd(d["q"], d["k"], d["v"], zd, d["dO"], d["hk0"], d["hv0"], d["dhkT"], d["dhvT"], want_dh0=True,
                    **kw)
    torch.cuda.synchronize()
    for n, got in (("o", o), ("hkT", hkT), ("hvT", hvT), ("dq", g["dq"]), ("dk", g["dk"]), ("dv", g["dv"])):
        compare(n, got, ref[n], dtype)
    compare("dz", g["dlog_a"], ref["dlog_a"] / (1.0 + np.exp(zz)) / tau, dtype)
    # one decode step from the final memories continues it
    hk, hv = hkT.clone(), hvT.clone()
    step = {n: d[n][:, :, -1].contiguous() for n in ("q", "k", "v")}
    o1 = gsa.gsa_step(step["q"], step["k"], step["v"], zd[:, :, -1].contiguous(), hk, hv, **kw)
    torch.cuda.synchronize()
    f = {n: to_f64_numpy(inp[n][:, :, -1:]) for n in ("q", "k", "v", "log_a")}
    ref1 = oracle.gsa_fwd(f["q"], f["k"], f["v"], f["log_a"], ref["hkT"], ref["hvT"])
    compare("o (step)", o1, ref1[0][:, :, 0], dtype)
