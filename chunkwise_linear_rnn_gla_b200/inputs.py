"""Seeded synthetic inputs and the named workloads.

This module is shared by the tests (which feed the oracle) and the benchmark
(which feeds the CUDA library). It holds no arithmetic of the layer itself:
only random draws, the gate pre-activation transform used to make inputs, and
dtype rounding.

Value recipe (the pages describe language-model training on datasets that are
not available here, so these synthetic tensors stand in for the activations):
  q, k, v ~ N(0, 1) / sqrt(d_k)
  z ~ N(z_mean, 1);  log_alpha = logsigmoid(z) / 16  (fp32, <= 0)
  dO ~ N(0, 1);  h0 = 0 unless a test asks for one
Draw order is q, k, v, z, dO, all fp32 from one CPU generator seeded with
`seed`; bf16 workloads round q, k, v, dO to bf16 (round-to-nearest-even) and
hand the rounded values to both the oracle and the GPU.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    L: int
    K: int
    V: int
    dtype: str  # "f32" or "bf16": dtype of q, k, v, o, dO and their gradients
    passes: str  # "fwd" or "fwd+bwd"
    chunk: int = 0  # 0 = library default
    z_mean: float = 0.0
    note: str = ""

    @property
    def tokens(self) -> int:
        return self.B * self.L


# The five workloads of the benchmark spec, named by what they are.
WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 1, 1, 256, 64, 64, "f32", "fwd+bwd", chunk=64,
                         note="B=1 H=1 L=256 d_k=d_v=64 fp32, chunk 64"),
    "gla340m_fwd": Workload("gla340m_fwd", 8, 4, 2048, 128, 256, "bf16", "fwd",
                            note="340M-layer shape B=8 H=4 L=2048 d_k=128 d_v=256, forward"),
    "gla1p3b_fwdbwd": Workload("gla1p3b_fwdbwd", 4, 4, 2048, 256, 512, "bf16", "fwd+bwd",
                               note="1.3B-layer shape B=4 H=4 L=2048 d_k=256 d_v=512, fwd+bwd"),
    "long16k": Workload("long16k", 1, 4, 16384, 128, 256, "bf16", "fwd+bwd", z_mean=2.0,
                        note="long sequence B=1 H=4 L=16384 d_k=128 d_v=256, slow decay z~N(2,1)"),
}
for _L in (1024, 2048, 4096, 8192, 16384):
    WORKLOADS["sweep_L%d" % _L] = Workload(
        "sweep_L%d" % _L, 16384 // _L, 4, _L, 128, 256, "bf16", "fwd+bwd",
        note="16384 tokens per batch, L=%d B=%d H=4 d_k=128 d_v=256" % (_L, 16384 // _L))

DECODE = dict(name="decode_b64", B=64, H=4, K=128, V=256, steps=4096, dtype="bf16")


# Gated slot attention: the 1.3B-layer shape with m = 128 slots (the pages give no slot count; 128 keeps
# the compact per-head memory of the method, 128 x (d_k + d_v), and is a width the tensor-core GLA passes
# take).
GSA_WORKLOAD = dict(name="gsa1p3b_fwdbwd", B=4, H=4, L=2048, K=256, V=512, m=128, dtype="bf16",
                    note="gated slot attention, 1.3B-layer shape B=4 H=4 L=2048 d_k=256 d_v=512, 128 slots, fwd+bwd")


def torch_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def make_inputs(B: int, H: int, L: int, K: int, V: int, dtype: str = "bf16", seed: int = 0,
                z_mean: float = 0.0, with_grad: bool = True, h0: bool = False, dhT: bool = False,
                gate_scale: float = 1.0 / 16.0):
    """Return a dict of CPU tensors: q, k, v (dtype), log_a (fp32), dO (dtype),
    and optional h0 / dhT (fp32). Values follow the module docstring."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    s = 1.0 / math.sqrt(K)
    q = torch.randn(B, H, L, K, generator=g) * s
    k = torch.randn(B, H, L, K, generator=g) * s
    v = torch.randn(B, H, L, V, generator=g) * s
    z = torch.randn(B, H, L, K, generator=g) + z_mean
    log_a = torch.nn.functional.logsigmoid(z) * gate_scale
    out = {"q": q, "k": k, "v": v, "log_a": log_a.float().contiguous()}
    if with_grad:
        out["dO"] = torch.randn(B, H, L, V, generator=g)
    if h0:
        out["h0"] = torch.randn(B, H, K, V, generator=g) * 0.1
    if dhT:
        out["dhT"] = torch.randn(B, H, K, V, generator=g) * 0.1
    td = torch_dtype(dtype)
    for name in ("q", "k", "v", "dO"):
        if name in out:
            out[name] = out[name].to(td).contiguous()
    return out


def make_workload_inputs(w: Workload, seed: int = 0, **kw):
    return make_inputs(w.B, w.H, w.L, w.K, w.V, w.dtype, seed=seed, z_mean=w.z_mean,
                       with_grad=(w.passes != "fwd") or kw.pop("with_grad", False), **kw)


def make_step_inputs(B: int, H: int, K: int, V: int, steps: int, dtype: str = "bf16", seed: int = 0,
                     z_mean: float = 0.0):
    """Per-step decode inputs: q, k [steps,B,H,K], v [steps,B,H,V], log_a [steps,B,H,K]."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    s = 1.0 / math.sqrt(K)
    q = torch.randn(steps, B, H, K, generator=g) * s
    k = torch.randn(steps, B, H, K, generator=g) * s
    v = torch.randn(steps, B, H, V, generator=g) * s
    z = torch.randn(steps, B, H, K, generator=g) + z_mean
    log_a = (torch.nn.functional.logsigmoid(z) / 16.0).float().contiguous()
    td = torch_dtype(dtype)
    return {"q": q.to(td).contiguous(), "k": k.to(td).contiguous(), "v": v.to(td).contiguous(), "log_a": log_a}


def to_f64_numpy(t: Optional[torch.Tensor]):
    """Upcast a (possibly bf16-rounded) tensor to a float64 numpy array."""
    if t is None:
        return None
    return t.detach().to("cpu").to(torch.float64).numpy()


def make_gsa_inputs(B: int, H: int, L: int, K: int, V: int, m: int, dtype: str = "bf16", seed: int = 0,
                    q_scale: float = 1.0, z_mean: float = 0.0, gate_scale: float = 1.0 / 16.0, h0: bool = False,
                    dhT: bool = False):
    """Gated slot attention inputs (CPU tensors): q ~ N(0,1) * q_scale (no 1/sqrt(d_k), so that the slot
    logits spread), k, v ~ N(0,1)/sqrt(d_k), per-slot gate log_a = logsigmoid(z) * gate_scale with
    z ~ N(z_mean, 1) [B,H,L,m], dO ~ N(0,1); optional initial memories hk0 [B,H,m,K], hv0 [B,H,m,V] and
    final-memory gradients dhkT, dhvT (N(0,1) * 0.1, fp32). Draw order q, k, v, z, dO, hk0, hv0, dhkT,
    dhvT; bf16 rounds q, k, v and dO."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    s = 1.0 / math.sqrt(K)
    out = {"q": torch.randn(B, H, L, K, generator=g) * q_scale,
           "k": torch.randn(B, H, L, K, generator=g) * s,
           "v": torch.randn(B, H, L, V, generator=g) * s}
    z = torch.randn(B, H, L, m, generator=g) + z_mean
    out["log_a"] = (torch.nn.functional.logsigmoid(z) * gate_scale).float().contiguous()
    out["dO"] = torch.randn(B, H, L, V, generator=g)
    if h0:
        out["hk0"] = torch.randn(B, H, m, K, generator=g) * 0.1
        out["hv0"] = torch.randn(B, H, m, V, generator=g) * 0.1
    if dhT:
        out["dhkT"] = torch.randn(B, H, m, K, generator=g) * 0.1
        out["dhvT"] = torch.randn(B, H, m, V, generator=g) * 0.1
    td = torch_dtype(dtype)
    for name in ("q", "k", "v", "dO"):
        out[name] = out[name].to(td).contiguous()
    return out
