"""Checking mode (GLA_FLAG_CHECKS): precondition checks on the gates, finiteness checks on the
outputs, guard blocks after every workspace slice and host-side canaries around the outputs. A
failed check never faults or traps: it sets the device error flag, which the binding turns into a
GlaError after the call. The bad inputs used here (a positive log alpha, a NaN in q) are values,
not addresses: every kernel reads and writes the same locations as for good inputs."""
import ctypes

import pytest
import torch

import chunkwise_linear_rnn_gla_b200 as gla
from chunkwise_linear_rnn_gla_b200 import _lib
from chunkwise_linear_rnn_gla_b200 import build as gbuild
from chunkwise_linear_rnn_gla_b200.inputs import make_inputs, make_step_inputs
from tests.parity import compare, oracle_bwd, oracle_fwd, to_dev


@pytest.fixture(scope="module")
def lib():
    gbuild.build()
    return _lib.load()


def _desc(**kw):
    d = dict(B=1, H=2, L=300, Dk=128, Dv=128, dtype=1, chunk=0, subchunk=0, state_mode=0, impl=0, flags=0)
    d.update(kw)
    return _lib.GlaDesc(**d)


def test_checking_flag_is_accepted_and_adds_guard_blocks(lib):
    for impl in (1, 2):
        plain = _desc(impl=impl)
        chk = _desc(impl=impl, flags=_lib.FLAG_CHECKS)
        for fn in (lib.gla_fwd_workspace_size, lib.gla_bwd_workspace_size):
            a, b = fn(ctypes.byref(plain)), fn(ctypes.byref(chk))
            assert a > 0 and b > a and (b - a) % 256 == 0
        assert lib.gla_bwd_workspace_bytes(ctypes.byref(chk)) == lib.gla_bwd_workspace_size(ctypes.byref(chk))
    assert lib.gla_fwd_workspace_size(ctypes.byref(_desc(flags=0x4))) == 0  # unknown flag: invalid


def test_checking_build_checks_every_call():
    """The library built with -DGLA_CHECKS sizes every workspace with its guard blocks, flag or not."""
    path = gbuild.build(checks=True)
    chk_lib = ctypes.CDLL(path)
    chk_lib.gla_fwd_workspace_size.argtypes = [ctypes.POINTER(_lib.GlaDesc)]
    chk_lib.gla_fwd_workspace_size.restype = ctypes.c_size_t
    plain = _lib.load()
    d = _desc(impl=2)
    dc = _desc(impl=2, flags=_lib.FLAG_CHECKS)
    assert chk_lib.gla_fwd_workspace_size(ctypes.byref(d)) == plain.gla_fwd_workspace_size(ctypes.byref(dc))


@pytest.mark.gpu
@pytest.mark.parametrize("impl", ["tc", "simt"])
def test_checked_call_matches_plain_call(lib, impl):
    inp = make_inputs(1, 2, 300, 128, 128, "bf16", seed=40, h0=True, dhT=True)
    d = to_dev(inp)
    o1, h1 = gla.gla_fwd(d["q"], d["k"], d["v"], d["log_a"], d["h0"], impl=impl)
    o2, h2 = gla.gla_fwd(d["q"], d["k"], d["v"], d["log_a"], d["h0"], impl=impl, checks=True)
    g1 = gla.gla_bwd(d["q"], d["k"], d["v"], d["log_a"], d["dO"], d["h0"], d["dhT"], impl=impl)
    g2 = gla.gla_bwd(d["q"], d["k"], d["v"], d["log_a"], d["dO"], d["h0"], d["dhT"], impl=impl, checks=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(h1, h2)
    for key in g1:
        assert torch.equal(g1[key], g2[key]), key
    o_ref, hT_ref = oracle_fwd(inp)
    compare("o (checking mode)", o2, o_ref, "bf16")
    ref = oracle_bwd(inp)
    compare("dlog_a (checking mode)", g2["dlog_a"], ref["dlog_a"], "bf16")
    assert gla.gla_check_device_error() == 0


@pytest.mark.gpu
@pytest.mark.parametrize("impl", ["tc", "simt"])
def test_positive_gate_is_reported(lib, impl):
    inp = make_inputs(1, 2, 200, 128, 128, "bf16", seed=41)
    inp["log_a"][0, 1, 37, 5] = 0.25  # alpha > 1: outside the gate's domain
    d = to_dev(inp)
    with pytest.raises(gla.GlaError) as ei:
        gla.gla_fwd(d["q"], d["k"], d["v"], d["log_a"], impl=impl, checks=True)
    assert ei.value.status == _lib.GLA_ERR_INVALID_ARG
    assert gla.gla_check_device_error() == 0  # reported once, then cleared
    with pytest.raises(gla.GlaError) as ei:
        gla.gla_bwd(d["q"], d["k"], d["v"], d["log_a"], d["dO"], impl=impl, checks=True)
    assert ei.value.status == _lib.GLA_ERR_INVALID_ARG
    # the same gate without checking mode: no report (the precondition is the caller's)
    gla.gla_fwd(d["q"], d["k"], d["v"], d["log_a"], impl=impl)
    assert gla.gla_check_device_error() == 0


@pytest.mark.gpu
def test_nan_input_gives_a_non_finite_report(lib):
    inp = make_inputs(1, 2, 200, 128, 128, "bf16", seed=42)
    inp["q"][0, 0, 17, 3] = float("nan")
    d = to_dev(inp)
    with pytest.raises(gla.GlaError) as ei:
        gla.gla_fwd(d["q"], d["k"], d["v"], d["log_a"], checks=True)
    assert ei.value.status == _lib.GLA_ERR_INVALID_ARG
    assert gla.gla_check_device_error() == 0


@pytest.mark.gpu
def test_step_checks(lib):
    st = make_step_inputs(2, 2, 64, 64, 1, "bf16", seed=43)
    q, k, v, la = (st[n][0].cuda() for n in ("q", "k", "v", "log_a"))
    S = torch.zeros(2, 2, 64, 64, device="cuda")
    gla.gla_step(q, k, v, la, S, checks=True)
    la[1, 0, 7] = float("nan")
    with pytest.raises(gla.GlaError) as ei:
        gla.gla_step(q, k, v, la, S, checks=True)
    assert ei.value.status == _lib.GLA_ERR_INVALID_ARG
    assert gla.gla_last_device_error() == 0
