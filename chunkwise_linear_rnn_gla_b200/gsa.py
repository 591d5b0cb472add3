"""Gated slot attention (GSA) on the library's GLA kernels: thin binding over ``gla_gsa_fwd`` /
``gla_gsa_bwd`` (include/gla.h). Argument checks, output and workspace allocation and the current
stream only; every step runs in libgla's kernels.

Method (mlsanity card for "Gated Slot Attention for Efficient Linear-Time Sequence Modeling",
abstract: a bounded slot memory forgotten by a GLA-style gate, read by two GLA layers joined by a
softmax over the slots), with a_t = exp(log_a_t) per slot and write weight 1 - a_t:
    Kmem_t = diag(a_t) Kmem_{t-1} + (1 - a_t)^T k_t,   Vmem_t = diag(a_t) Vmem_{t-1} + (1 - a_t)^T v_t,
    o_t = softmax(Kmem_t q_t^T) Vmem_t.
Shapes: q, k [B,H,L,Dk]; v [B,H,L,Dv]; log_a [B,H,L,m] fp32; memories hk [B,H,m,Dk], hv [B,H,m,Dv] fp32.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import torch

from . import _lib, _need, _ptr, _stream, _check, _workspace, make_desc, _dt
from ._lib import load

__all__ = ["gsa_fwd", "gsa_bwd", "gsa_step", "gsa_fwd_workspace_size", "gsa_bwd_workspace_size", "gsa_route"]


def _desc(q, v, chunk, subchunk, state_mode, impl, flags, gate="channel", tau=0.0):
    B, H, L, Dk = q.shape
    return make_desc(B, H, L, Dk, v.shape[-1], _dt(q), chunk, subchunk, state_mode, impl, flags, gate, tau)


def gsa_route(desc, slots: int) -> str:
    """"tc" or "simt": the route gsa_fwd / gsa_bwd take for this descriptor and slot count."""
    im = ctypes.c_int32()
    _check(load().gla_gsa_resolve(ctypes.byref(desc), int(slots), ctypes.byref(im)), "gla_gsa_resolve")
    return {v: k for k, v in _lib.IMPL.items()}[im.value]


def gsa_fwd_workspace_size(desc, slots: int) -> int:
    return int(load().gla_gsa_fwd_workspace_size(ctypes.byref(desc), int(slots)))


def gsa_bwd_workspace_size(desc, slots: int) -> int:
    return int(load().gla_gsa_bwd_workspace_size(ctypes.byref(desc), int(slots)))


def _check_inputs(q, k, v, log_a):
    dev, dt = q.device, q.dtype
    B, H, L, Dk = q.shape
    _need(k, "k", q.shape, dt, dev)
    if v.dim() != 4 or tuple(v.shape[:3]) != (B, H, L):
        raise ValueError("v has shape %s, expected [%d, %d, %d, Dv]" % (tuple(v.shape), B, H, L))
    _need(v, "v", v.shape, dt, dev)
    if log_a.dim() != 4 or tuple(log_a.shape[:3]) != (B, H, L):
        raise ValueError("log_a has shape %s, expected [%d, %d, %d, slots]" % (tuple(log_a.shape), B, H, L))
    _need(log_a, "log_a", log_a.shape, torch.float32, dev)
    return dev, dt, B, H, L, Dk, v.shape[-1], log_a.shape[-1]


def gsa_fwd(q, k, v, log_a, hk0=None, hv0=None, *, chunk=0, subchunk=0, state_mode="auto", impl="auto",
            want_state=False, workspace=None, checks=False, gate="channel", tau=0.0):
    """Forward. Returns (o, hkT, hvT); the final memories are None unless want_state. Pass the same
    `workspace` to gsa_bwd(ws_from_fwd=True) to reuse the read weights and layer two's states.
    gate="preact": log_a holds the gate's argument z, log a = logsigmoid(z) / tau."""
    load()
    dev, dt, B, H, L, Dk, Dv, m = _check_inputs(q, k, v, log_a)
    if hk0 is not None:
        _need(hk0, "hk0", (B, H, m, Dk), torch.float32, dev)
    if hv0 is not None:
        _need(hv0, "hv0", (B, H, m, Dv), torch.float32, dev)
    desc = _desc(q, v, chunk, subchunk, state_mode, impl, _lib.FLAG_CHECKS if checks else 0, gate, tau)
    o = torch.empty(B, H, L, Dv, dtype=dt, device=dev)
    hkT = torch.empty(B, H, m, Dk, dtype=torch.float32, device=dev) if want_state else None
    hvT = torch.empty(B, H, m, Dv, dtype=torch.float32, device=dev) if want_state else None
    ws, nbytes = _workspace(gsa_fwd_workspace_size(desc, m), dev, workspace)
    with torch.cuda.device(dev):
        st = load().gla_gsa_fwd(ctypes.byref(desc), m, _ptr(q), _ptr(k), _ptr(v), _ptr(log_a), _ptr(hk0),
                                _ptr(hv0), _ptr(o), _ptr(hkT), _ptr(hvT), _ptr(ws), nbytes, _stream(dev))
    _check(st, "gla_gsa_fwd")
    if checks:
        _check(load().gla_check_device_error(_stream(dev)), "gla_gsa_fwd (checking mode)")
    return o, hkT, hvT


def gsa_bwd(q, k, v, log_a, dO, hk0=None, hv0=None, dhkT=None, dhvT=None, *, chunk=0, subchunk=0,
            state_mode="auto", impl="auto", want_dh0=False, workspace=None, ws_from_fwd=False, checks=False,
            gate="channel", tau=0.0):
    """Backward of <dO, o> + <dhkT, hkT> + <dhvT, hvT>. Returns a dict with dq, dk, dv, dlog_a (dL/dz for
    gate="preact") and (with want_dh0) dhk0, dhv0. With ws_from_fwd=True `workspace` must be the matching
    gsa_fwd's, sized for the backward (gsa_bwd_workspace_size)."""
    load()
    dev, dt, B, H, L, Dk, Dv, m = _check_inputs(q, k, v, log_a)
    _need(dO, "dO", (B, H, L, Dv), dt, dev)
    for t, n, shp in ((hk0, "hk0", (B, H, m, Dk)), (hv0, "hv0", (B, H, m, Dv)), (dhkT, "dhkT", (B, H, m, Dk)),
                      (dhvT, "dhvT", (B, H, m, Dv))):
        if t is not None:
            _need(t, n, shp, torch.float32, dev)
    if ws_from_fwd and workspace is None:
        raise ValueError("ws_from_fwd needs the forward's workspace")
    flags = (_lib.FLAG_WS_FROM_FWD if ws_from_fwd else 0) | (_lib.FLAG_CHECKS if checks else 0)
    desc = _desc(q, v, chunk, subchunk, state_mode, impl, flags, gate, tau)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dla = torch.empty_like(log_a)
    dhk0 = torch.empty(B, H, m, Dk, dtype=torch.float32, device=dev) if want_dh0 else None
    dhv0 = torch.empty(B, H, m, Dv, dtype=torch.float32, device=dev) if want_dh0 else None
    ws, nbytes = _workspace(gsa_bwd_workspace_size(desc, m), dev, workspace)
    with torch.cuda.device(dev):
        st = load().gla_gsa_bwd(ctypes.byref(desc), m, _ptr(q), _ptr(k), _ptr(v), _ptr(log_a), _ptr(hk0),
                                _ptr(hv0), _ptr(dO), _ptr(dhkT), _ptr(dhvT), _ptr(dq), _ptr(dk), _ptr(dv),
                                _ptr(dla), _ptr(dhk0), _ptr(dhv0), _ptr(ws), nbytes, _stream(dev))
    _check(st, "gla_gsa_bwd")
    if checks:
        _check(load().gla_check_device_error(_stream(dev)), "gla_gsa_bwd (checking mode)")
    return {"dq": dq, "dk": dk, "dv": dv, "dlog_a": dla, "dhk0": dhk0, "dhv0": dhv0}


def gsa_step(q, k, v, log_a, hk, hv, o=None, checks=False, gate="channel", tau=0.0):
    """One decode step: q, k [B,H,Dk], v [B,H,Dv], log_a [B,H,m] fp32 (z for gate="preact"); the memories
    hk [B,H,m,Dk] and hv [B,H,m,Dv] (fp32) are updated in place. Returns o [B,H,Dv]."""
    load()
    dev, dt = q.device, q.dtype
    B, H, Dk = q.shape
    _need(k, "k", q.shape, dt, dev)
    if v.dim() != 3 or tuple(v.shape[:2]) != (B, H):
        raise ValueError("v has shape %s, expected [%d, %d, Dv]" % (tuple(v.shape), B, H))
    _need(v, "v", v.shape, dt, dev)
    Dv = v.shape[-1]
    if log_a.dim() != 3 or tuple(log_a.shape[:2]) != (B, H):
        raise ValueError("log_a has shape %s, expected [%d, %d, slots]" % (tuple(log_a.shape), B, H))
    _need(log_a, "log_a", log_a.shape, torch.float32, dev)
    m = log_a.shape[-1]
    _need(hk, "hk", (B, H, m, Dk), torch.float32, dev)
    _need(hv, "hv", (B, H, m, Dv), torch.float32, dev)
    if o is None:
        o = torch.empty(B, H, Dv, dtype=dt, device=dev)
    _need(o, "o", (B, H, Dv), dt, dev)
    desc = make_desc(B, H, 1, Dk, Dv, _dt(q), flags=_lib.FLAG_CHECKS if checks else 0, gate=gate, tau=tau)
    with torch.cuda.device(dev):
        st = load().gla_gsa_step(ctypes.byref(desc), m, _ptr(q), _ptr(k), _ptr(v), _ptr(log_a), _ptr(hk), _ptr(hv),
                                 _ptr(o), _stream(dev))
    _check(st, "gla_gsa_step")
    if checks:
        _check(load().gla_check_device_error(_stream(dev)), "gla_gsa_step (checking mode)")
    return o
