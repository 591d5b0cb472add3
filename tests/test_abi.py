"""C-ABI checks that need no GPU: the library loads, exports every function
include/gla.h declares, and rejects bad arguments on the host before any
launch."""
import ctypes
import os
import re

import pytest

from chunkwise_linear_rnn_gla_b200 import build as gbuild
from chunkwise_linear_rnn_gla_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    gbuild.build()
    return _lib.load()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "gla.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gla_[a-z_0-9]+)\s*\(", src)))


def test_header_and_binding_agree():
    assert sorted(_lib.EXPORTS) == declared_functions()


def test_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_abi_version(lib):
    assert lib.gla_abi_version() == 2


def test_status_strings(lib):
    for s in range(6):
        assert len(lib.gla_status_string(s)) > 0
    assert lib.gla_status_string(99) == b"unknown status"


def desc(**kw):
    d = dict(B=1, H=1, L=64, Dk=64, Dv=64, dtype=0, chunk=0, subchunk=0, state_mode=0, impl=0, flags=0)
    d.update(kw)
    return _lib.GlaDesc(**d)


def test_resolve_defaults(lib):
    c, sc, im, sm = (ctypes.c_int32() for _ in range(4))
    assert lib.gla_resolve(ctypes.byref(desc(dtype=0)), ctypes.byref(c), ctypes.byref(sc), ctypes.byref(im),
                           ctypes.byref(sm)) == 0
    assert (c.value, sc.value, im.value) == (64, 16, 1)  # fp32 -> CUDA-core path, chunk 64, sub-chunks of 16
    # bf16 at a tensor-core shape -> tensor-core path, C = 128, one sub-chunk per chunk (single GEMM), materialised
    assert lib.gla_resolve(ctypes.byref(desc(dtype=1, Dk=256, Dv=512, L=2048)), ctypes.byref(c), ctypes.byref(sc),
                           ctypes.byref(im), ctypes.byref(sm)) == 0
    assert (c.value, sc.value, im.value, sm.value) == (128, 128, 2, 1)


@pytest.mark.parametrize("bad", [dict(B=0), dict(L=0), dict(Dk=0), dict(dtype=7), dict(chunk=48), dict(chunk=-1),
                                 dict(state_mode=9), dict(impl=5), dict(flags=0x100), dict(chunk=16, subchunk=32),
                                 dict(chunk=64, subchunk=24, impl=1)])
def test_bad_descriptor_rejected(lib, bad):
    d = desc(**bad)
    assert lib.gla_fwd_workspace_size(ctypes.byref(d)) == 0
    st = lib.gla_fwd(ctypes.byref(d), 16, 16, 16, 16, None, 16, None, None, 0, None)
    assert st == 1  # GLA_ERR_INVALID_ARG


def test_null_desc(lib):
    assert lib.gla_fwd(None, 16, 16, 16, 16, None, 16, None, None, 0, None) == 1
    assert lib.gla_step(None, 16, 16, 16, 16, 16, 16, None) == 1
    assert lib.gla_fwd_workspace_size(None) == 0


def test_null_and_misaligned_pointers(lib):
    d = desc()
    # null q
    assert lib.gla_fwd(ctypes.byref(d), None, 16, 16, 16, None, 16, None, None, 0, None) == 1
    # misaligned k
    assert lib.gla_fwd(ctypes.byref(d), 16, 18, 16, 16, None, 16, None, None, 0, None) == 1
    # misaligned optional h0
    assert lib.gla_fwd(ctypes.byref(d), 16, 16, 16, 16, 24, 16, None, None, 0, None) == 1
    # backward: null dlog_a
    assert lib.gla_bwd(ctypes.byref(d), 16, 16, 16, 16, None, 16, None, 16, 16, 16, None, None, None, 0, None) == 1


def test_workspace_checks(lib):
    d = desc()
    need = lib.gla_fwd_workspace_size(ctypes.byref(d))
    assert need > 0
    assert lib.gla_bwd_workspace_size(ctypes.byref(d)) >= need
    # missing workspace, too small, misaligned: all GLA_ERR_WORKSPACE before any launch
    assert lib.gla_fwd(ctypes.byref(d), 16, 16, 16, 16, None, 16, None, None, 0, None) == 3
    assert lib.gla_fwd(ctypes.byref(d), 16, 16, 16, 16, None, 16, None, 256, need - 1, None) == 3
    assert lib.gla_fwd(ctypes.byref(d), 16, 16, 16, 16, None, 16, None, 272, need, None) == 3


def test_simt_rejects_nonmaterialized(lib):
    d = desc(impl=1, state_mode=2)
    assert lib.gla_fwd(ctypes.byref(d), 16, 16, 16, 16, None, 16, None, 256, 1 << 30, None) == 2


def test_launch_counter_host_only(lib):
    lib.gla_launch_count_reset()
    assert lib.gla_launch_count() == 0


# ---------------------------------------------------------------- gated slot attention (host logic only)
def gsa_route(lib, slots, **kw):
    im = ctypes.c_int32(-1)
    st = lib.gla_gsa_resolve(ctypes.byref(desc(**kw)), slots, ctypes.byref(im))
    return st, im.value


def test_gsa_route_selection(lib):
    tc, simt = _lib.IMPL["tc"], _lib.IMPL["simt"]
    # bf16, 128 slots, widths that the tensor-core passes take -> tensor cores
    assert gsa_route(lib, 128, dtype=1, L=2048, Dk=256, Dv=512) == (0, tc)
    assert gsa_route(lib, 128, dtype=1, L=300, Dk=64, Dv=192) == (0, tc)
    # other slot counts, fp32, widths off the 64 grid, a two-level sub-chunk or an explicit CUDA-core request
    for slots, kw in ((64, dict(dtype=1, Dk=128, Dv=128)), (256, dict(dtype=1, Dk=128, Dv=128)),
                      (128, dict(dtype=0, Dk=128, Dv=128)), (128, dict(dtype=1, Dk=96, Dv=128)),
                      (128, dict(dtype=1, Dk=128, Dv=128, subchunk=16)), (128, dict(dtype=1, Dk=128, Dv=128, impl=1))):
        assert gsa_route(lib, slots, L=300, **kw) == (0, simt), (slots, kw)
    # an explicit tensor-core request that the route cannot serve
    assert gsa_route(lib, 64, dtype=1, L=300, Dk=128, Dv=128, impl=2)[0] == _lib.GLA_ERR_UNSUPPORTED


def test_gsa_rejects_bad_arguments(lib):
    assert gsa_route(lib, 0, dtype=1)[0] == _lib.GLA_ERR_INVALID_ARG
    assert gsa_route(lib, 128, dtype=1, gate=1)[0] == _lib.GLA_ERR_UNSUPPORTED  # slot gates are per slot
    assert gsa_route(lib, 128, dtype=1, gate=9)[0] == _lib.GLA_ERR_INVALID_ARG
    assert gsa_route(lib, 128, dtype=1, gate=3)[0] == _lib.GLA_ERR_INVALID_ARG  # pre-activation needs tau > 0
    assert gsa_route(lib, 128, dtype=1, gate=3, gate_tau=8.0, Dk=128, Dv=128) == (0, _lib.IMPL["tc"])
    assert gsa_route(lib, 128, dtype=1, flags=0x40)[0] == _lib.GLA_ERR_INVALID_ARG
    d = desc(dtype=1, L=64, Dk=128, Dv=128)
    ptr = ctypes.c_void_p(256)
    # a null required pointer is rejected on the host, before any launch
    assert lib.gla_gsa_fwd(ctypes.byref(d), 128, None, ptr, ptr, ptr, None, None, ptr, None, None, ptr, 1 << 30,
                           None) == _lib.GLA_ERR_INVALID_ARG
    assert lib.gla_gsa_step(ctypes.byref(d), 128, ptr, ptr, ptr, ptr, ptr, None, ptr, None) == _lib.GLA_ERR_INVALID_ARG
    # misaligned pointers
    bad = ctypes.c_void_p(258)
    assert lib.gla_gsa_step(ctypes.byref(d), 128, bad, ptr, ptr, ptr, ptr, ptr, ptr, None) == _lib.GLA_ERR_INVALID_ARG
    # a step whose widths are not multiples of 4
    d3 = desc(dtype=1, L=1, Dk=130, Dv=128)
    assert lib.gla_gsa_step(ctypes.byref(d3), 128, ptr, ptr, ptr, ptr, ptr, ptr, ptr, None) == _lib.GLA_ERR_UNSUPPORTED
    # the forward's workspace check runs before any launch
    assert lib.gla_gsa_fwd(ctypes.byref(d), 128, ptr, ptr, ptr, ptr, None, None, ptr, None, None, ptr, 16,
                           None) == _lib.GLA_ERR_WORKSPACE
    # a forward cannot take the forward's workspace
    dr = desc(dtype=1, L=64, Dk=128, Dv=128, flags=_lib.FLAG_WS_FROM_FWD)
    assert lib.gla_gsa_fwd(ctypes.byref(dr), 128, ptr, ptr, ptr, ptr, None, None, ptr, None, None, ptr, 1 << 30,
                           None) == _lib.GLA_ERR_INVALID_ARG


@pytest.mark.parametrize("dtype,slots", [(1, 128), (1, 64), (0, 32)])
def test_gsa_workspace_prefix(lib, dtype, slots):
    """The backward's workspace extends the forward's (the backward may take the forward's), and both
    grow with the sequence."""
    sizes = []
    for L in (300, 600):
        d = desc(dtype=dtype, L=L, Dk=128, Dv=256)
        f, b = lib.gla_gsa_fwd_workspace_size(ctypes.byref(d), slots), lib.gla_gsa_bwd_workspace_size(ctypes.byref(d), slots)
        assert 0 < f <= b
        sizes.append(b)
    assert sizes[1] > sizes[0]
