"""Chunkwise gated linear attention (GLA) for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI in ``include/gla.h`` (``libgla.so``). Every
step of the layer runs in the library's CUDA kernels; this module only checks
tensors, allocates outputs and workspace with torch, and passes pointers and
the current CUDA stream. There is no CPU fallback: without the built library
every call raises.

Layer (per batch b and head h; "Gated Linear Attention Transformers with
Hardware-Efficient Training", atlas.scime.ai summary, section "Approach"):
    S_t = diag(exp(log_a_t)) S_{t-1} + k_t^T v_t,    o_t = q_t S_t.
Shapes: q, k, log_a [B,H,L,Dk]; v [B,H,L,Dv]; states [B,H,Dk,Dv] (fp32).
"""
from __future__ import annotations

import ctypes
from typing import Optional

import torch

from . import _lib
from ._lib import GlaDesc, GlaError, load  # noqa: F401

__all__ = ["gla_fwd", "gla_bwd", "gla_step", "gla_chunk_cumsum", "gla_fwd_workspace_size", "gla_last_device_error",
           "gla_fwd_final_state", "gla_bwd_initial_grad",
           "gla_bwd_workspace_size", "gla_resolve", "gla_check_device_error", "gla_launch_count",
           "gla_launch_count_reset", "gla_profile_enable", "gla_profile_read", "gla_profile_reset",
           "make_desc", "GlaError"]

_TORCH_DTYPE = {torch.float32: "f32", torch.bfloat16: "bf16"}


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(dev: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _check(status: int, what: str):
    if status != _lib.GLA_OK:
        raise GlaError(status, what)


def _dt(t: torch.Tensor) -> str:
    if t.dtype not in _TORCH_DTYPE:
        raise TypeError("q/k/v/dO must be float32 or bfloat16, got %s" % t.dtype)
    return _TORCH_DTYPE[t.dtype]


def _need(t, name, shape, dtype, dev):
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if t.device != dev:
        raise ValueError("%s is on %s, expected %s" % (name, t.device, dev))
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), tuple(shape)))
    if t.dtype != dtype:
        raise TypeError("%s has dtype %s, expected %s" % (name, t.dtype, dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


def make_desc(B, H, L, Dk, Dv, dtype="bf16", chunk=0, subchunk=0, state_mode="auto", impl="auto",
              flags=0, gate="channel", tau=0.0) -> GlaDesc:
    """Problem descriptor. gate: what log_a holds -- "channel" (log alpha [B,H,L,Dk]), "scalar"
    (one log decay per head and step, [B,H,L]), "head" (one fixed log decay per head, [H]) or
    "preact" (the gate's argument z [B,H,L,Dk], log alpha = logsigmoid(z) / tau)."""
    return GlaDesc(B, H, L, Dk, Dv, _lib.DTYPE[dtype], chunk, subchunk, _lib.STATE_MODE[state_mode],
                   _lib.IMPL[impl], flags, _lib.GATE[gate], float(tau))


def gate_shape(gate, B, H, L, Dk):
    """Shape of the log_a argument (and of dlog_a) for a gate kind; L=None for the decode step."""
    steps = () if L is None else (L,)
    return {"channel": (B, H) + steps + (Dk,), "scalar": (B, H) + steps, "head": (H,),
            "preact": (B, H) + steps + (Dk,)}[gate]


def gla_fwd_workspace_size(desc: GlaDesc) -> int:
    return int(load().gla_fwd_workspace_size(ctypes.byref(desc)))


def gla_bwd_workspace_size(desc: GlaDesc) -> int:
    return int(load().gla_bwd_workspace_size(ctypes.byref(desc)))


def gla_resolve(desc: GlaDesc):
    """(chunk, subchunk, impl, state_mode) the library resolves `desc` to."""
    c, sc, im, sm = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    _check(load().gla_resolve(ctypes.byref(desc), ctypes.byref(c), ctypes.byref(sc), ctypes.byref(im),
                              ctypes.byref(sm)), "gla_resolve")
    inv_impl = {v: k for k, v in _lib.IMPL.items()}
    inv_sm = {v: k for k, v in _lib.STATE_MODE.items()}
    return c.value, sc.value, inv_impl[im.value], inv_sm[sm.value]


def _workspace(nbytes: int, dev, workspace: Optional[torch.Tensor]):
    if nbytes == 0:
        return None, 0
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    if workspace.numel() * workspace.element_size() < nbytes:
        raise ValueError("workspace too small: %d < %d bytes" % (workspace.numel() * workspace.element_size(), nbytes))
    return workspace, workspace.numel() * workspace.element_size()


# ---- checking mode: the library's device-side checks plus host-side canaries around the outputs.
# Every output the binding allocates is carved from a larger buffer whose margins hold NaN; after the
# call (which is then synchronous) the margins must still be NaN and the device error flag clear.
_CANARY = 256  # elements on each side (>= 256 bytes, keeps 16-byte alignment)


def _guarded(shape, dtype, dev, guards):
    n = 1
    for x in shape:
        n *= int(x)
    buf = torch.full((n + 2 * _CANARY,), float("nan"), dtype=dtype, device=dev)
    guards.append((buf, n))
    return buf[_CANARY:_CANARY + n].view(*shape)


def _finish_checks(guards, what):
    st = gla_check_device_error()
    if st != _lib.GLA_OK:
        raise GlaError(st, what + " (checking mode)")
    for buf, n in guards:
        if not (bool(torch.isnan(buf[:_CANARY]).all()) and bool(torch.isnan(buf[_CANARY + n:]).all())):
            raise GlaError(_lib.GLA_ERR_WORKSPACE, what + " (checking mode: an output canary was overwritten)")


def _desc_from(q, v, chunk, subchunk, state_mode, impl, flags=0, gate="channel", tau=0.0):
    B, H, L, Dk = q.shape
    Dv = v.shape[-1]
    return make_desc(B, H, L, Dk, Dv, _dt(q), chunk, subchunk, state_mode, impl, flags, gate, tau)


def gla_fwd(q, k, v, log_a, h0=None, *, chunk=0, subchunk=0, state_mode="auto", impl="auto", o=None, hT=None,
            want_hT=True, workspace=None, checks=False, gate="channel", tau=0.0):
    """Forward. Returns (o, hT); hT is None when want_hT is False and no hT
    buffer is given. `workspace` (uint8 tensor) may be passed to reuse it.
    checks=True runs the library's checking mode (gate domain, finite
    outputs, workspace guards) with canaries around the outputs allocated
    here; the call then synchronises and raises GlaError on any failure."""
    load()
    dev = q.device
    B, H, L, Dk = q.shape
    Dv = v.shape[-1]
    dt = q.dtype
    _need(k, "k", q.shape, dt, dev)
    _need(v, "v", (B, H, L, Dv), dt, dev)
    _need(log_a, "log_a", gate_shape(gate, B, H, L, Dk), torch.float32, dev)
    if h0 is not None:
        _need(h0, "h0", (B, H, Dk, Dv), torch.float32, dev)
    desc = _desc_from(q, v, chunk, subchunk, state_mode, impl, _lib.FLAG_CHECKS if checks else 0, gate, tau)
    guards = []
    alloc = (lambda shp, t: _guarded(shp, t, dev, guards)) if checks else \
        (lambda shp, t: torch.empty(*shp, dtype=t, device=dev))
    if o is None:
        o = alloc((B, H, L, Dv), dt)
    _need(o, "o", (B, H, L, Dv), dt, dev)
    if hT is None and want_hT:
        hT = alloc((B, H, Dk, Dv), torch.float32)
    if hT is not None:
        _need(hT, "hT", (B, H, Dk, Dv), torch.float32, dev)
    ws, nbytes = _workspace(gla_fwd_workspace_size(desc), dev, workspace)
    with torch.cuda.device(dev):
        st = load().gla_fwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(log_a), _ptr(h0), _ptr(o),
                            _ptr(hT), _ptr(ws), nbytes, _stream(dev))
    _check(st, "gla_fwd")
    if checks:
        _finish_checks(guards, "gla_fwd")
    return o, hT


def gla_bwd(q, k, v, log_a, dO, h0=None, dhT=None, *, chunk=0, subchunk=0, state_mode="auto", impl="auto",
            want_dh0=True, workspace=None, ws_from_fwd=False, out=None, checks=False, gate="channel", tau=0.0):
    """Backward of <dO, o> + <dhT, hT>. Returns a dict with dq, dk, dv,
    dlog_a and dh0. With ws_from_fwd=True the workspace must be the one the
    matching gla_fwd call used (same inputs, same options, checks included).
    checks=True: as for gla_fwd."""
    load()
    dev = q.device
    B, H, L, Dk = q.shape
    Dv = v.shape[-1]
    dt = q.dtype
    _need(k, "k", q.shape, dt, dev)
    _need(v, "v", (B, H, L, Dv), dt, dev)
    _need(log_a, "log_a", gate_shape(gate, B, H, L, Dk), torch.float32, dev)
    _need(dO, "dO", (B, H, L, Dv), dt, dev)
    if h0 is not None:
        _need(h0, "h0", (B, H, Dk, Dv), torch.float32, dev)
    if dhT is not None:
        _need(dhT, "dhT", (B, H, Dk, Dv), torch.float32, dev)
    flags = (_lib.FLAG_WS_FROM_FWD if ws_from_fwd else 0) | (_lib.FLAG_CHECKS if checks else 0)
    desc = _desc_from(q, v, chunk, subchunk, state_mode, impl, flags, gate, tau)
    if ws_from_fwd and workspace is None:
        raise ValueError("ws_from_fwd needs the forward's workspace")
    guards = []
    alloc = (lambda shp, t: _guarded(shp, t, dev, guards)) if checks else \
        (lambda shp, t: torch.empty(*shp, dtype=t, device=dev))
    out = dict(out or {})
    dq = out.get("dq")
    if dq is None:
        dq = alloc(q.shape, dt)
    dk = out.get("dk")
    if dk is None:
        dk = alloc(k.shape, dt)
    dv = out.get("dv")
    if dv is None:
        dv = alloc(v.shape, dt)
    dla = out.get("dlog_a")
    if dla is None:
        dla = alloc(log_a.shape, torch.float32)
    _need(dla, "dlog_a", log_a.shape, torch.float32, dev)
    dh0 = out.get("dh0")
    if dh0 is None and want_dh0:
        dh0 = alloc((B, H, Dk, Dv), torch.float32)
    ws, nbytes = _workspace(gla_bwd_workspace_size(desc), dev, workspace)
    with torch.cuda.device(dev):
        st = load().gla_bwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(log_a), _ptr(h0), _ptr(dO),
                            _ptr(dhT), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dla), _ptr(dh0), _ptr(ws), nbytes,
                            _stream(dev))
    _check(st, "gla_bwd")
    if checks:
        _finish_checks(guards, "gla_bwd")
    return {"dq": dq, "dk": dk, "dv": dv, "dlog_a": dla, "dh0": dh0}


def gla_fwd_final_state(q, k, v, log_a, h0=None, *, chunk=0, subchunk=0, state_mode="auto", impl="auto",
                        hT=None, workspace=None, gate="channel", tau=0.0):
    """hT of gla_fwd without o (tensor-core path; GlaError GLA_ERR_UNSUPPORTED elsewhere)."""
    load()
    dev = q.device
    B, H, L, Dk = q.shape
    Dv = v.shape[-1]
    _need(k, "k", q.shape, q.dtype, dev)
    _need(v, "v", (B, H, L, Dv), q.dtype, dev)
    _need(log_a, "log_a", gate_shape(gate, B, H, L, Dk), torch.float32, dev)
    if h0 is not None:
        _need(h0, "h0", (B, H, Dk, Dv), torch.float32, dev)
    desc = _desc_from(q, v, chunk, subchunk, state_mode, impl, 0, gate, tau)
    if hT is None:
        hT = torch.empty(B, H, Dk, Dv, dtype=torch.float32, device=dev)
    _need(hT, "hT", (B, H, Dk, Dv), torch.float32, dev)
    ws, nbytes = _workspace(gla_fwd_workspace_size(desc), dev, workspace)
    with torch.cuda.device(dev):
        st = load().gla_fwd_final_state(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(log_a), _ptr(h0),
                                        _ptr(hT), _ptr(ws), nbytes, _stream(dev))
    _check(st, "gla_fwd_final_state")
    return hT


def gla_bwd_initial_grad(q, k, v, log_a, dO, dhT=None, *, chunk=0, subchunk=0, state_mode="auto", impl="auto",
                         dh0=None, workspace=None, gate="channel", tau=0.0):
    """dh0 of gla_bwd without the other gradients (tensor-core path; GlaError GLA_ERR_UNSUPPORTED
    elsewhere). v only gives the value width."""
    load()
    dev = q.device
    B, H, L, Dk = q.shape
    Dv = v.shape[-1]
    _need(k, "k", q.shape, q.dtype, dev)
    _need(log_a, "log_a", gate_shape(gate, B, H, L, Dk), torch.float32, dev)
    _need(dO, "dO", (B, H, L, Dv), q.dtype, dev)
    if dhT is not None:
        _need(dhT, "dhT", (B, H, Dk, Dv), torch.float32, dev)
    desc = _desc_from(q, v, chunk, subchunk, state_mode, impl, 0, gate, tau)
    if dh0 is None:
        dh0 = torch.empty(B, H, Dk, Dv, dtype=torch.float32, device=dev)
    _need(dh0, "dh0", (B, H, Dk, Dv), torch.float32, dev)
    ws, nbytes = _workspace(gla_bwd_workspace_size(desc), dev, workspace)
    with torch.cuda.device(dev):
        st = load().gla_bwd_initial_grad(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(log_a), _ptr(dO), _ptr(dhT),
                                         _ptr(dh0), _ptr(ws), nbytes, _stream(dev))
    _check(st, "gla_bwd_initial_grad")
    return dh0


def gla_step(q, k, v, log_a, S, o=None, checks=False, gate="channel", tau=0.0):
    """One decode step; S [B,H,Dk,Dv] fp32 is updated in place. Returns o [B,H,Dv].
    checks=True: the library's checking mode (gate domain, finite o and S), synchronous, raises on a
    failure."""
    load()
    dev = q.device
    B, H, Dk = q.shape
    Dv = v.shape[-1]
    dt = q.dtype
    _need(k, "k", q.shape, dt, dev)
    _need(v, "v", (B, H, Dv), dt, dev)
    _need(log_a, "log_a", gate_shape(gate, B, H, None, Dk), torch.float32, dev)
    _need(S, "S", (B, H, Dk, Dv), torch.float32, dev)
    guards = []
    if o is None:
        o = _guarded((B, H, Dv), dt, dev, guards) if checks else torch.empty(B, H, Dv, dtype=dt, device=dev)
    _need(o, "o", (B, H, Dv), dt, dev)
    desc = make_desc(B, H, 1, Dk, Dv, _dt(q), flags=_lib.FLAG_CHECKS if checks else 0, gate=gate, tau=tau)
    with torch.cuda.device(dev):
        st = load().gla_step(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(log_a), _ptr(S), _ptr(o),
                             _stream(dev))
    _check(st, "gla_step")
    if checks:
        _finish_checks(guards, "gla_step")
    return o


def gla_chunk_cumsum(log_a, chunk=64, out=None):
    """Per-chunk inclusive cumsum of log_a along L (restarting every `chunk`)."""
    load()
    dev = log_a.device
    B, H, L, Dk = log_a.shape
    _need(log_a, "log_a", log_a.shape, torch.float32, dev)
    if out is None:
        out = torch.empty_like(log_a)
    desc = make_desc(B, H, L, Dk, 1, "f32", chunk)
    with torch.cuda.device(dev):
        st = load().gla_chunk_cumsum(ctypes.byref(desc), _ptr(log_a), _ptr(out), _stream(dev))
    _check(st, "gla_chunk_cumsum")
    return out


def gla_check_device_error(stream=None) -> int:
    s = ctypes.c_void_p(stream if stream is not None else torch.cuda.current_stream().cuda_stream)
    return int(load().gla_check_device_error(s))


def gla_last_device_error(stream=None) -> int:
    """The same report as gla_check_device_error (the name the layer's scope table uses)."""
    s = ctypes.c_void_p(stream if stream is not None else torch.cuda.current_stream().cuda_stream)
    return int(load().gla_last_device_error(s))


def gla_selftest_wait_timeout(limit_cycles=0, stream=None) -> None:
    """Run the library's bounded-wait self-test kernel (a wait that nothing completes); the next
    gla_check_device_error reports GLA_ERR_TIMEOUT."""
    s = ctypes.c_void_p(stream if stream is not None else torch.cuda.current_stream().cuda_stream)
    _check(load().gla_selftest_wait_timeout(int(limit_cycles), s), "gla_selftest_wait_timeout")


def gla_launch_count() -> int:
    return int(load().gla_launch_count())


def gla_launch_count_reset() -> None:
    load().gla_launch_count_reset()


def gla_profile_enable(on: bool = True) -> None:
    load().gla_profile_enable(1 if on else 0)


def gla_profile_read():
    """{kernel name: (launches, total device ms)} of the recorded launches."""
    lib = load()
    cap = 64
    names = (ctypes.c_char_p * cap)()
    cnt = (ctypes.c_uint64 * cap)()
    ms = (ctypes.c_double * cap)()
    n = lib.gla_profile_read(names, cnt, ms, cap)
    return {names[i].decode(): (int(cnt[i]), float(ms[i])) for i in range(min(n, cap))}


def gla_profile_reset() -> None:
    load().gla_profile_reset()
