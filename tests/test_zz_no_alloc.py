"""gla_fwd_noalloc: the forward for callers that cannot allocate device memory
(a plugin under a framework or server that owns every device allocation, a
latency-critical loop that must avoid cudaMalloc/cudaFree, a C caller with no
device memory manager). It takes its scratch from a fixed array inside the
library instead of a caller-provided workspace.

Called here through the C ABI (ctypes) and compared with gla_fwd, the
ordinary entry point, on two calls in a row with different inputs (so that
anything the first call left in the shared array would show up in the
second), within the parity tolerances of the other tests. This file is named
to be collected last.
"""
import ctypes

import pytest
import torch

import chunkwise_linear_rnn_gla_b200 as gla
from chunkwise_linear_rnn_gla_b200 import _lib
from chunkwise_linear_rnn_gla_b200 import build as gbuild
from chunkwise_linear_rnn_gla_b200.inputs import make_inputs
from tests.parity import compare

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 16 << 20  # GLA_NOALLOC_SCRATCH_BYTES in include/gla.h


@pytest.fixture(scope="module")
def lib():
    gbuild.build()
    return _lib.load()


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(lib, d, o, hT):
    B, H, L, K = d["q"].shape
    V = d["v"].shape[-1]
    desc = gla.make_desc(B, H, L, K, V, "bf16" if d["q"].dtype == torch.bfloat16 else "f32")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.gla_fwd_noalloc(ctypes.byref(desc), _p(d["q"]), _p(d["k"]), _p(d["v"]), _p(d["log_a"]),
                               _p(d.get("h0")), _p(o), _p(hT), stream)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_noalloc_matches_gla_fwd_twice(lib, dtype):
    B, H, L, K, V = 2, 2, 300, 64, 96
    desc = gla.make_desc(B, H, L, K, V, dtype, impl="simt")
    assert gla.gla_fwd_workspace_size(desc) <= SCRATCH_BYTES
    for seed in (1, 2):  # two calls in a row, different inputs
        inp = make_inputs(B, H, L, K, V, dtype, seed=seed, h0=(seed == 1), with_grad=False)
        d = {k_: v_.cuda() for k_, v_ in inp.items()}
        o_ref, hT_ref = gla.gla_fwd(d["q"], d["k"], d["v"], d["log_a"], d.get("h0"), impl="simt")
        o = torch.full_like(o_ref, float("nan"))
        hT = torch.full_like(hT_ref, float("nan"))
        st = _noalloc(lib, d, o, hT)
        assert st == 0, _lib.status_string(st)
        torch.cuda.synchronize()
        compare("o (call with seed %d)" % seed, o, o_ref.double().cpu().numpy(), dtype)
        compare("hT (call with seed %d)" % seed, hT, hT_ref.double().cpu().numpy(), dtype)


def test_noalloc_rejects_oversize(lib):
    # the CUDA-core workspace of this problem is far beyond the fixed array
    desc = gla.make_desc(8, 4, 8192, 256, 512, "bf16", impl="simt")
    assert gla.gla_fwd_workspace_size(desc) > SCRATCH_BYTES
    st = lib.gla_fwd_noalloc(ctypes.byref(desc), 256, 256, 256, 256, None, 256, None, None)
    assert st == 3  # GLA_ERR_WORKSPACE, returned before any launch
    bad = gla.make_desc(1, 1, 64, 64, 64, "bf16", impl="tc")
    assert lib.gla_fwd_noalloc(ctypes.byref(bad), 256, 256, 256, 256, None, 256, None, None) == 2
