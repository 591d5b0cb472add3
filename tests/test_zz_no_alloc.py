"""gla_fwd_noalloc: the forward for callers that cannot allocate device memory
(a plugin under a framework or server that owns every device allocation, a
latency-critical loop that must avoid cudaMalloc/cudaFree, a C caller with no
device memory manager). It takes its scratch from a fixed array inside the
library instead of a caller-provided workspace.

Called here through the C ABI (ctypes) and compared with gla_fwd, the
ordinary entry point, and with the fp64 oracle, on two calls in a row with
different inputs (so that anything the first call left in the shared array
would show up in the second), within the parity tolerances of the other
tests; also at the array's size limit. This file is named to be collected
last.
"""
import ctypes

import pytest
import torch

import chunkwise_linear_rnn_gla_b200 as gla
from chunkwise_linear_rnn_gla_b200 import _lib
from chunkwise_linear_rnn_gla_b200 import build as gbuild
from chunkwise_linear_rnn_gla_b200.inputs import make_inputs
from tests.parity import compare, oracle_fwd

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 16 << 20  # GLA_NOALLOC_SCRATCH_BYTES in include/gla.h


@pytest.fixture(scope="module")
def lib():
    gbuild.build()
    return _lib.load()


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(lib, d, o, hT, chunk=0):
    B, H, L, K = d["q"].shape
    V = d["v"].shape[-1]
    desc = gla.make_desc(B, H, L, K, V, "bf16" if d["q"].dtype == torch.bfloat16 else "f32", chunk=chunk)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.gla_fwd_noalloc(ctypes.byref(desc), _p(d["q"]), _p(d["k"]), _p(d["v"]), _p(d["log_a"]),
                               _p(d.get("h0")), _p(o), _p(hT), stream)


@pytest.mark.parametrize("chunk", [16, 64, 128])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_noalloc_matches_gla_fwd_and_oracle_twice(lib, dtype, chunk):
    """Two calls in a row with different inputs (anything the first call left in the shared array would
    show in the second), at chunk lengths 16, 64 and 128 (128 gives the largest per-chunk score
    blocks); each call is checked against gla_fwd and against the fp64 oracle."""
    B, H, L, K, V = 2, 2, 300, 64, 96
    desc = gla.make_desc(B, H, L, K, V, dtype, chunk=chunk, impl="simt")
    assert gla.gla_fwd_workspace_size(desc) <= SCRATCH_BYTES
    for seed in (1, 2):
        inp = make_inputs(B, H, L, K, V, dtype, seed=seed + chunk, h0=(seed == 1), with_grad=False)
        d = {k_: v_.cuda() for k_, v_ in inp.items()}
        o_ref, hT_ref = gla.gla_fwd(d["q"], d["k"], d["v"], d["log_a"], d.get("h0"), chunk=chunk, impl="simt")
        o = torch.full_like(o_ref, float("nan"))
        hT = torch.full_like(hT_ref, float("nan"))
        st = _noalloc(lib, d, o, hT, chunk)
        assert st == 0, _lib.status_string(st)
        torch.cuda.synchronize()
        compare("o vs gla_fwd (call with seed %d)" % seed, o, o_ref.double().cpu().numpy(), dtype)
        compare("hT vs gla_fwd (call with seed %d)" % seed, hT, hT_ref.double().cpu().numpy(), dtype)
        o_or, hT_or = oracle_fwd(inp)
        compare("o vs oracle (call with seed %d)" % seed, o, o_or, dtype)
        compare("hT vs oracle (call with seed %d)" % seed, hT, hT_or, dtype)


def _largest_fitting_L(B, H, K, V, dtype, chunk):
    """Largest L whose CUDA-core forward workspace fits the fixed array (found from the host-side size
    query alone)."""
    size = lambda L: gla.gla_fwd_workspace_size(gla.make_desc(B, H, L, K, V, dtype, chunk=chunk, impl="simt"))
    lo, hi = 1, 1
    while size(hi) <= SCRATCH_BYTES:
        lo, hi = hi, hi * 2
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if size(mid) <= SCRATCH_BYTES:
            lo = mid
        else:
            hi = mid
    return lo, size(lo), hi, size(hi)


def test_noalloc_at_the_size_limit(lib):
    """A problem whose workspace is just under the array runs and matches the oracle; the next length,
    just over it, is refused with GLA_ERR_WORKSPACE before anything is launched."""
    B, H, K, V, dtype, chunk = 1, 2, 64, 64, "bf16", 64
    L_ok, ws_ok, L_big, ws_big = _largest_fitting_L(B, H, K, V, dtype, chunk)
    assert ws_ok <= SCRATCH_BYTES < ws_big and ws_ok > SCRATCH_BYTES - (1 << 20)
    inp = make_inputs(B, H, L_ok, K, V, dtype, seed=3, h0=True, with_grad=False)
    d = {k_: v_.cuda() for k_, v_ in inp.items()}
    o = torch.full(d["v"].shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    hT = torch.full((B, H, K, V), float("nan"), device="cuda")
    for _ in range(2):
        st = _noalloc(lib, d, o, hT, chunk)
        assert st == 0, _lib.status_string(st)
        torch.cuda.synchronize()
        o_or, hT_or = oracle_fwd(inp)
        compare("o at the limit", o, o_or, dtype)
        compare("hT at the limit", hT, hT_or, dtype)
    big = make_inputs(B, H, L_big, K, V, dtype, seed=4, with_grad=False)
    db = {k_: v_.cuda() for k_, v_ in big.items()}
    ob = torch.full(db["v"].shape, 7.0, dtype=torch.bfloat16, device="cuda")
    assert _noalloc(lib, db, ob, None, chunk) == 3  # GLA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((ob == 7.0).all())  # nothing ran


def test_noalloc_rejects_oversize(lib):
    # the CUDA-core workspace of this problem is far beyond the fixed array
    desc = gla.make_desc(8, 4, 8192, 256, 512, "bf16", impl="simt")
    assert gla.gla_fwd_workspace_size(desc) > SCRATCH_BYTES
    st = lib.gla_fwd_noalloc(ctypes.byref(desc), 256, 256, 256, 256, None, 256, None, None)
    assert st == 3  # GLA_ERR_WORKSPACE, returned before any launch
    bad = gla.make_desc(1, 1, 64, 64, 64, "bf16", impl="tc")
    assert lib.gla_fwd_noalloc(ctypes.byref(bad), 256, 256, 256, 256, None, 256, None, None) == 2
