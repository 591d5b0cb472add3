"""Pins for the fp64 oracle: each test checks it against something other than
itself -- a hand-derived worked example, the O(L^2) masked parallel form,
textbook special cases, finite differences, or an identity of the recurrence.

Layer: S_t = diag(alpha_t) S_{t-1} + k_t^T v_t, o_t = q_t S_t with the gate
G_t = alpha_t^T 1 ("Gated Linear Attention Transformers with Hardware-Efficient
Training", atlas.scime.ai summary, section "Approach").
"""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


def rnd(shape, rng, scale=1.0):
    return rng.standard_normal(shape) * scale


def make(B, H, L, K, V, seed=0, h0=False, dhT=False, gate="mixed"):
    rng = np.random.default_rng(seed)
    q = rnd((B, H, L, K), rng, 1 / math.sqrt(K))
    k = rnd((B, H, L, K), rng, 1 / math.sqrt(K))
    v = rnd((B, H, L, V), rng, 1 / math.sqrt(K))
    if gate == "mixed":
        # a wide spread of decays, including near-zero and near-one gates
        log_a = np.log(1 / (1 + np.exp(-rnd((B, H, L, K), rng, 2.0))))
    else:
        log_a = gate(rng, (B, H, L, K))
    dO = rnd((B, H, L, V), rng)
    out = dict(q=q, k=k, v=v, log_a=log_a, dO=dO)
    out["h0"] = rnd((B, H, K, V), rng, 0.3) if h0 else None
    out["dhT"] = rnd((B, H, K, V), rng, 0.3) if dhT else None
    return out


# ---------------------------------------------------------------- brute force
def brute_force_fwd(q, k, v, log_a, h0=None):
    """O(L^2) masked parallel form, written from the definition with explicit
    products of gates: o_t = sum_{s<=t} (q_t * prod_{r=s+1..t} alpha_r) . k_s v_s
    + (q_t * prod_{r=0..t} alpha_r) h0."""
    B, H, L, K = q.shape
    V = v.shape[-1]
    alpha = np.exp(log_a)
    o = np.zeros((B, H, L, V))
    for b in range(B):
        for h in range(H):
            for t in range(L):
                for s in range(t + 1):
                    decay = np.prod(alpha[b, h, s + 1:t + 1, :], axis=0)  # empty product = 1
                    o[b, h, t] += np.dot(q[b, h, t] * decay, k[b, h, s]) * v[b, h, s]
                if h0 is not None:
                    decay0 = np.prod(alpha[b, h, 0:t + 1, :], axis=0)
                    o[b, h, t] += (q[b, h, t] * decay0) @ h0[b, h]
    return o


# ------------------------------------------------------------- worked example
def test_worked_example_forward():
    ex = json.load(open(GOLD))["per_channel_forward"]
    a = np.array(ex["alpha"], float)
    q = np.array(ex["q"], float)[None, None]
    k = np.array(ex["k"], float)[None, None]
    v = np.array(ex["v"], float)[None, None]
    o, hT = oracle.fwd(q, k, v, np.log(a)[None, None])
    np.testing.assert_allclose(o[0, 0], np.array(ex["o"], float), atol=1e-14)
    np.testing.assert_allclose(hT[0, 0], np.array(ex["hT"], float), atol=1e-14)


def test_worked_example_backward():
    ex = json.load(open(GOLD))["scalar_backward"]
    arr = lambda n: np.array(ex[n], float)[None, None]  # noqa: E731
    g = oracle.bwd(arr("q"), arr("k"), arr("v"), np.log(arr("alpha")), arr("dO"))
    o, _ = oracle.fwd(arr("q"), arr("k"), arr("v"), np.log(arr("alpha")))
    np.testing.assert_allclose(o[0, 0], np.array(ex["o"], float), atol=1e-14)
    for name in ("dq", "dk", "dv", "dlog_a"):
        np.testing.assert_allclose(g[name][0, 0], np.array(ex[name], float), atol=1e-13, err_msg=name)
    np.testing.assert_allclose(g["dlog_a_cf"][0, 0], np.array(ex["dlog_a"], float), atol=1e-13)
    np.testing.assert_allclose(g["dh0"][0, 0], np.array(ex["dh0"], float), atol=1e-14)


# ------------------------------------------------------------------- forward
@pytest.mark.parametrize("h0", [False, True])
@pytest.mark.parametrize("shape", [(1, 1, 7, 3, 5), (2, 2, 19, 4, 6), (1, 1, 33, 8, 2)])
def test_brute_force(shape, h0):
    d = make(*shape, seed=sum(shape), h0=h0)
    o, _ = oracle.fwd(d["q"], d["k"], d["v"], d["log_a"], d["h0"])
    ref = brute_force_fwd(d["q"], d["k"], d["v"], d["log_a"], d["h0"])
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)


def test_no_gate_is_causal_linear_attention():
    # alpha == 1: the no-gate ablation (section "Measured effects") is plain
    # causal linear attention, o = tril(Q K^T) V + Q h0.
    d = make(2, 3, 40, 8, 12, seed=3, h0=True)
    la = np.zeros_like(d["log_a"])
    o, hT = oracle.fwd(d["q"], d["k"], d["v"], la, d["h0"])
    for b in range(2):
        for h in range(3):
            Q, Kk, Vv = d["q"][b, h], d["k"][b, h], d["v"][b, h]
            ref = np.tril(Q @ Kk.T) @ Vv + Q @ d["h0"][b, h]
            np.testing.assert_allclose(o[b, h], ref, atol=1e-12)
            np.testing.assert_allclose(hT[b, h], d["h0"][b, h] + Kk.T @ Vv, atol=1e-12)


def test_scalar_constant_decay_is_retnet_form():
    # one data-independent decay gamma on every channel (the RetNet-style
    # ablation): o = ((Q K^T) * D) V + diag(gamma^{t+1}) Q h0, D_ts = gamma^{t-s}
    d = make(1, 2, 50, 6, 7, seed=4, h0=True)
    gamma = 0.93
    la = np.full_like(d["log_a"], math.log(gamma))
    o, _ = oracle.fwd(d["q"], d["k"], d["v"], la, d["h0"])
    L = 50
    t = np.arange(L)
    D = np.where(t[:, None] >= t[None, :], gamma ** (t[:, None] - t[None, :]).clip(min=0), 0.0)
    for h in range(2):
        Q, Kk, Vv = d["q"][0, h], d["k"][0, h], d["v"][0, h]
        ref = ((Q @ Kk.T) * D) @ Vv + (gamma ** (t + 1))[:, None] * (Q @ d["h0"][0, h])
        np.testing.assert_allclose(o[0, h], ref, atol=1e-12)


def test_zero_gate_forgets_everything():
    d = make(1, 2, 20, 5, 4, seed=5, h0=True)
    la = np.full_like(d["log_a"], -1e30)  # alpha = 0 exactly
    o, hT = oracle.fwd(d["q"], d["k"], d["v"], la, d["h0"])
    qk = np.einsum("bhtc,bhtc->bht", d["q"], d["k"])
    np.testing.assert_allclose(o, qk[..., None] * d["v"], atol=1e-14)
    np.testing.assert_allclose(hT, np.einsum("bhc,bhv->bhcv", d["k"][:, :, -1], d["v"][:, :, -1]), atol=1e-14)


def test_linear_in_v_and_h0():
    d1 = make(1, 1, 30, 4, 5, seed=6, h0=True)
    d2 = make(1, 1, 30, 4, 5, seed=7, h0=True)
    o1, _ = oracle.fwd(d1["q"], d1["k"], d1["v"], d1["log_a"], d1["h0"])
    o2, _ = oracle.fwd(d1["q"], d1["k"], d2["v"], d1["log_a"], d2["h0"])
    o3, _ = oracle.fwd(d1["q"], d1["k"], 2 * d1["v"] - 3 * d2["v"], d1["log_a"], 2 * d1["h0"] - 3 * d2["h0"])
    np.testing.assert_allclose(o3, 2 * o1 - 3 * o2, atol=1e-12)


def test_final_state_closed_form():
    # hT = diag(exp(sum log a)) h0 + sum_s diag(exp(b_T - b_s)) k_s^T v_s, b = global cumsum
    d = make(2, 1, 37, 5, 3, seed=8, h0=True)
    _, hT = oracle.fwd(d["q"], d["k"], d["v"], d["log_a"], d["h0"])
    b = np.cumsum(d["log_a"], axis=2)
    bT = b[:, :, -1:, :]
    ref = np.exp(bT[:, :, 0, :])[..., None] * d["h0"]
    ref = ref + np.einsum("bhsc,bhsv->bhcv", d["k"] * np.exp(bT - b), d["v"])
    np.testing.assert_allclose(hT, ref, atol=1e-12)


@pytest.mark.parametrize("L1", [1, 17, 64])
def test_split_sequence_forward(L1):
    d = make(2, 2, 96, 6, 5, seed=9, h0=True)
    o, hT = oracle.fwd(d["q"], d["k"], d["v"], d["log_a"], d["h0"])
    cut = lambda x, a, b: x[:, :, a:b]  # noqa: E731
    oa, ha = oracle.fwd(cut(d["q"], 0, L1), cut(d["k"], 0, L1), cut(d["v"], 0, L1), cut(d["log_a"], 0, L1), d["h0"])
    ob, hb = oracle.fwd(cut(d["q"], L1, 96), cut(d["k"], L1, 96), cut(d["v"], L1, 96), cut(d["log_a"], L1, 96), ha)
    np.testing.assert_allclose(np.concatenate([oa, ob], axis=2), o, atol=1e-12)
    np.testing.assert_allclose(hb, hT, atol=1e-12)


def test_step_iterated_equals_forward():
    d = make(2, 3, 25, 4, 6, seed=10, h0=True)
    o, hT = oracle.fwd(d["q"], d["k"], d["v"], d["log_a"], d["h0"])
    S = d["h0"].copy()
    for t in range(25):
        ot, S = oracle.step(d["q"][:, :, t], d["k"][:, :, t], d["v"][:, :, t], d["log_a"][:, :, t], S)
        np.testing.assert_allclose(ot, o[:, :, t], atol=1e-12)
    np.testing.assert_allclose(S, hT, atol=1e-12)


# ------------------------------------------------------------------ backward
def _loss(d, q=None, k=None, v=None, log_a=None, h0=None):
    q = d["q"] if q is None else q
    k = d["k"] if k is None else k
    v = d["v"] if v is None else v
    log_a = d["log_a"] if log_a is None else log_a
    h0 = d["h0"] if h0 is None else h0
    o, hT = oracle.fwd(q, k, v, log_a, h0)
    val = np.sum(o * d["dO"])
    if d["dhT"] is not None:
        val += np.sum(hT * d["dhT"])
    return val


@pytest.mark.parametrize("seed", [0, 1])
def test_finite_differences(seed):
    d = make(1, 2, 9, 3, 4, seed=20 + seed, h0=True, dhT=True)
    g = oracle.bwd(d["q"], d["k"], d["v"], d["log_a"], d["dO"], d["h0"], d["dhT"], seg=4)
    eps = 1e-6
    for name, grad in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("log_a", "dlog_a"), ("h0", "dh0")):
        x = d[name]
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp = x.copy()
            xp[idx] += eps
            xm = x.copy()
            xm[idx] -= eps
            num[idx] = (_loss(d, **{name: xp}) - _loss(d, **{name: xm})) / (2 * eps)
        np.testing.assert_allclose(g[grad], num, rtol=1e-6, atol=1e-8, err_msg=grad)
    # the closed-form gate gradient must match the same finite differences
    np.testing.assert_allclose(g["dlog_a_cf"], g["dlog_a"], rtol=1e-9, atol=1e-11)


@pytest.mark.parametrize("with_dhT", [False, True])
def test_closed_form_gate_gradient(with_dhT):
    d = make(2, 2, 150, 8, 16, seed=31, h0=True, dhT=with_dhT)
    g = oracle.bwd(d["q"], d["k"], d["v"], d["log_a"], d["dO"], d["h0"], d["dhT"], seg=16)
    scale = np.abs(g["dlog_a"]).max()
    np.testing.assert_allclose(g["dlog_a_cf"], g["dlog_a"], atol=1e-11 * max(scale, 1.0))


def test_checkpoint_spacing_does_not_matter():
    d = make(1, 2, 70, 5, 6, seed=32, h0=True, dhT=True)
    g1 = oracle.bwd(d["q"], d["k"], d["v"], d["log_a"], d["dO"], d["h0"], d["dhT"], seg=1)
    g2 = oracle.bwd(d["q"], d["k"], d["v"], d["log_a"], d["dO"], d["h0"], d["dhT"], seg=64)
    for key in g1:
        np.testing.assert_allclose(g1[key], g2[key], atol=1e-12, err_msg=key)


def test_split_sequence_backward():
    # truncated BPTT reading: the second segment's dh0 is the first segment's dhT
    d = make(1, 2, 80, 5, 6, seed=33, h0=True, dhT=True)
    g = oracle.bwd(d["q"], d["k"], d["v"], d["log_a"], d["dO"], d["h0"], d["dhT"])
    L1 = 29
    c1 = lambda x: x[:, :, :L1]  # noqa: E731
    c2 = lambda x: x[:, :, L1:]  # noqa: E731
    _, h_mid = oracle.fwd(c1(d["q"]), c1(d["k"]), c1(d["v"]), c1(d["log_a"]), d["h0"])
    g2 = oracle.bwd(c2(d["q"]), c2(d["k"]), c2(d["v"]), c2(d["log_a"]), c2(d["dO"]), h_mid, d["dhT"])
    g1 = oracle.bwd(c1(d["q"]), c1(d["k"]), c1(d["v"]), c1(d["log_a"]), c1(d["dO"]), d["h0"], g2["dh0"])
    for key in ("dq", "dk", "dv", "dlog_a", "dlog_a_cf"):
        np.testing.assert_allclose(np.concatenate([g1[key], g2[key]], axis=2), g[key], atol=1e-12, err_msg=key)
    np.testing.assert_allclose(g1["dh0"], g["dh0"], atol=1e-12)


def test_zero_gate_gradients():
    # alpha = 0: o_t = (q_t . k_t) v_t, so dq_t = (do_t . v_t) k_t etc.
    d = make(1, 1, 12, 4, 3, seed=34)
    la = np.full_like(d["log_a"], -1e30)
    g = oracle.bwd(d["q"], d["k"], d["v"], la, d["dO"])
    dov = np.einsum("bhtv,bhtv->bht", d["dO"], d["v"])[..., None]
    qk = np.einsum("bhtc,bhtc->bht", d["q"], d["k"])[..., None]
    np.testing.assert_allclose(g["dq"], dov * d["k"], atol=1e-14)
    np.testing.assert_allclose(g["dk"], dov * d["q"], atol=1e-14)
    np.testing.assert_allclose(g["dv"], qk * d["dO"], atol=1e-14)
    np.testing.assert_allclose(g["dlog_a"], 0.0, atol=1e-14)
