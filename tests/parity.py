"""Helpers for GPU-vs-oracle parity tests.

Tolerances (written here once, used by every parity test):
  fp32 inputs : max |gpu - oracle| <= 1e-4 per output tensor
  bf16 inputs : max |gpu - oracle| / max |oracle| <= 2e-2 per output tensor
The oracle reads exactly the (bf16-rounded) values the GPU reads, upcast to
fp64, so the tolerance measures the kernels alone.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from chunkwise_linear_rnn_gla_b200.inputs import to_f64_numpy

TOL_F32_ABS = 1e-4
TOL_BF16_REL = 2e-2


def compare(name, gpu, ref, dtype):
    g = to_f64_numpy(gpu) if isinstance(gpu, torch.Tensor) else np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert g.shape == ref.shape, (name, g.shape, ref.shape)
    assert np.all(np.isfinite(g)), "%s: non-finite values from the GPU" % name
    err = np.abs(g - ref).max() if g.size else 0.0
    if dtype == "f32":
        assert err <= TOL_F32_ABS, "%s: max abs err %.3e > %.1e" % (name, err, TOL_F32_ABS)
        return err
    scale = np.abs(ref).max() if ref.size else 0.0
    rel = err / scale if scale > 0 else err
    assert rel <= TOL_BF16_REL, "%s: max abs err %.3e / max |ref| %.3e = %.3e > %.1e" % (
        name, err, scale, rel, TOL_BF16_REL)
    return rel


def heads(t, idx):
    """Select flattened (b,h) heads `idx` from a [B,H,...] array/tensor -> [1,len(idx),...]."""
    shp = t.shape
    flat = t.reshape((shp[0] * shp[1],) + tuple(shp[2:]))
    sel = flat[list(idx)]
    return sel.reshape((1, len(idx)) + tuple(shp[2:]))


def oracle_fwd(inp, idx=None):
    f = lambda n: None if inp.get(n) is None else to_f64_numpy(inp[n] if idx is None else heads(inp[n], idx))  # noqa: E731
    return oracle.fwd(f("q"), f("k"), f("v"), f("log_a"), f("h0"))


def oracle_bwd(inp, idx=None):
    f = lambda n: None if inp.get(n) is None else to_f64_numpy(inp[n] if idx is None else heads(inp[n], idx))  # noqa: E731
    return oracle.bwd(f("q"), f("k"), f("v"), f("log_a"), f("dO"), f("h0"), f("dhT"))


def to_dev(inp, dev="cuda"):
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
