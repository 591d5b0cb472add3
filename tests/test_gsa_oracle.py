"""Pins for the gated slot attention (GSA) oracle (oracle/gsa_oracle.c).

Each test checks it against something other than itself: a hand-derived worked
example, the O(L^2) parallel form with explicit gate products, textbook special
cases (one slot = an exponential moving average; a zero gate = copy of v),
finite differences, invariances, sequence splitting, and the two-layer GLA
reading of the card (the mlsanity card for "Gated Slot Attention for Efficient
Linear-Time Sequence Modeling", abstract: two GLA layers joined by a softmax)
evaluated with the separately pinned GLA oracle.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden", "gsa_worked_example.json")


def make(B, H, L, K, V, m, seed=0, h0=False, dhT=False, qscale=1.0):
    rng = np.random.default_rng(seed)
    d = dict(
        q=rng.standard_normal((B, H, L, K)) * qscale,
        k=rng.standard_normal((B, H, L, K)) / math.sqrt(K),
        v=rng.standard_normal((B, H, L, V)),
        # a wide spread of gates, near-zero and near-one included
        log_a=np.log(1 / (1 + np.exp(-2.0 * rng.standard_normal((B, H, L, m))))),
        dO=rng.standard_normal((B, H, L, V)),
    )
    d["hk0"] = rng.standard_normal((B, H, m, K)) * 0.5 if h0 else None
    d["hv0"] = rng.standard_normal((B, H, m, V)) * 0.5 if h0 else None
    d["dhkT"] = rng.standard_normal((B, H, m, K)) * 0.5 if dhT else None
    d["dhvT"] = rng.standard_normal((B, H, m, V)) * 0.5 if dhT else None
    return d


def softmax(z, axis=-1):
    z = z - z.max(axis=axis, keepdims=True)
    e = np.exp(z)
    return e / e.sum(axis=axis, keepdims=True)


# ------------------------------------------------------------- worked example
def test_worked_example():
    ex = json.load(open(GOLD))
    a = np.array(ex["alpha"])[None, None]
    q = np.array(ex["q"])[None, None]
    k = np.array(ex["k"])[None, None]
    v = np.array(ex["v"])[None, None]
    o, s, hkT, hvT = oracle.gsa_fwd(q, k, v, np.log(a))
    np.testing.assert_allclose(o[0, 0], np.array(ex["o"]), atol=1e-14)
    np.testing.assert_allclose(s[0, 0], np.array(ex["s"]), atol=1e-14)
    np.testing.assert_allclose(hkT[0, 0], np.array(ex["hkT"]), atol=1e-14)
    np.testing.assert_allclose(hvT[0, 0], np.array(ex["hvT"]), atol=1e-14)


# ----------------------------------------------------------- O(L^2) parallel form
def brute_force(q, k, v, log_a, hk0=None, hv0=None):
    """Kmem_t = sum_{s<=t} (prod_{r=s+1..t} a_r) * (1 - a_s) k_s + (prod_{r<=t} a_r) hk0 per slot, the same for
    Vmem; s_t = softmax(Kmem_t q_t); o_t = s_t Vmem_t."""
    B, H, L, K = q.shape
    V, m = v.shape[-1], log_a.shape[-1]
    a = np.exp(log_a)
    o = np.zeros((B, H, L, V))
    for b in range(B):
        for h in range(H):
            for t in range(L):
                Km = np.zeros((m, K))
                Vm = np.zeros((m, V))
                for s_ in range(t + 1):
                    w = np.prod(a[b, h, s_ + 1:t + 1], axis=0) * (1 - a[b, h, s_])  # [m]
                    Km += np.outer(w, k[b, h, s_])
                    Vm += np.outer(w, v[b, h, s_])
                if hk0 is not None:
                    d0 = np.prod(a[b, h, :t + 1], axis=0)
                    Km += d0[:, None] * hk0[b, h]
                    Vm += d0[:, None] * hv0[b, h]
                o[b, h, t] = softmax(Km @ q[b, h, t]) @ Vm
    return o


@pytest.mark.parametrize("h0", [False, True])
def test_matches_parallel_form(h0):
    d = make(2, 2, 13, 5, 3, 4, seed=1, h0=h0, qscale=2.0)
    o, _, _, _ = oracle.gsa_fwd(d["q"], d["k"], d["v"], d["log_a"], d["hk0"], d["hv0"])
    ref = brute_force(d["q"], d["k"], d["v"], d["log_a"], d["hk0"], d["hv0"])
    np.testing.assert_allclose(o, ref, atol=1e-12, rtol=0)


# ------------------------------------------------------------- special cases
def test_one_slot_is_exponential_moving_average():
    """m = 1: the softmax weight is 1, so o_t = Vmem_t; with a constant gate g that is the textbook EMA
    o_t = (1-g) sum_{s<=t} g^{t-s} v_s + g^{t+1} hv0, whatever q and k are."""
    rng = np.random.default_rng(2)
    B, H, L, K, V, g = 1, 2, 20, 3, 4, 0.8
    q, k = rng.standard_normal((2, B, H, L, K))
    v = rng.standard_normal((B, H, L, V))
    hv0 = rng.standard_normal((B, H, 1, V))
    hk0 = rng.standard_normal((B, H, 1, K))
    la = np.full((B, H, L, 1), math.log(g))
    o, s, _, hvT = oracle.gsa_fwd(q, k, v, la, hk0, hv0)
    np.testing.assert_array_equal(s, 1.0)
    ema = np.zeros((B, H, L, V))
    for t in range(L):
        ema[:, :, t] = g ** (t + 1) * hv0[:, :, 0] + sum((1 - g) * g ** (t - s_) * v[:, :, s_] for s_ in range(t + 1))
    np.testing.assert_allclose(o, ema, atol=1e-12)
    np.testing.assert_allclose(hvT[:, :, 0], ema[:, :, -1], atol=1e-12)


def test_zero_gate_copies_v():
    """a_t = 0: every slot holds exactly (k_t, v_t), the logits are equal, the weights uniform, o_t = v_t."""
    d = make(1, 2, 7, 4, 5, 6, seed=3, h0=True)
    la = np.full_like(d["log_a"], -1e30)
    o, s, hkT, hvT = oracle.gsa_fwd(d["q"], d["k"], d["v"], la, d["hk0"], d["hv0"])
    np.testing.assert_allclose(s, 1.0 / 6, atol=1e-15)
    np.testing.assert_allclose(o, d["v"], atol=1e-14)
    np.testing.assert_allclose(hkT, np.repeat(d["k"][:, :, -1:], 6, axis=2), atol=1e-15)


def test_slot_permutation_invariance():
    """Relabelling the slots (gates and initial memories together) leaves o unchanged and permutes the
    final memories."""
    d = make(1, 2, 11, 3, 4, 5, seed=4, h0=True, qscale=2.0)
    perm = np.array([3, 0, 4, 1, 2])
    o1, s1, hk1, hv1 = oracle.gsa_fwd(d["q"], d["k"], d["v"], d["log_a"], d["hk0"], d["hv0"])
    o2, s2, hk2, hv2 = oracle.gsa_fwd(d["q"], d["k"], d["v"], d["log_a"][..., perm], d["hk0"][:, :, perm],
                                      d["hv0"][:, :, perm])
    np.testing.assert_allclose(o2, o1, atol=1e-13)
    np.testing.assert_allclose(s2, s1[..., perm], atol=1e-14)
    np.testing.assert_allclose(hk2, hk1[:, :, perm], atol=1e-14)


# ------------------------------------------------------ the two-layer GLA reading
def two_layer_fwd(q, k, v, log_a, hk0=None, hv0=None):
    """The card's reading as two GLA layers, each evaluated by the GLA oracle. Layer one's state is the key
    memory (GLA key 1-a, value k); its read Kmem_t q_t is the gradient of <q_t, o'_t> with respect to the
    query of that GLA, so the logits are the GLA oracle's dq with dO = q. Layer two is a GLA with query s,
    key 1-a, value v."""
    w = 1.0 - np.exp(log_a)
    logits = oracle.bwd(np.zeros_like(w), w, k, log_a, q, h0=hk0)["dq"]
    s = softmax(logits)
    o, hvT = oracle.fwd(s, w, v, log_a, hv0)
    return o, s, hvT


def test_two_layer_reading_forward():
    d = make(2, 2, 37, 6, 5, 4, seed=5, h0=True, qscale=2.0)
    o, s, _, hvT = oracle.gsa_fwd(d["q"], d["k"], d["v"], d["log_a"], d["hk0"], d["hv0"])
    o2, s2, hvT2 = two_layer_fwd(d["q"], d["k"], d["v"], d["log_a"], d["hk0"], d["hv0"])
    np.testing.assert_allclose(s2, s, atol=1e-13)
    np.testing.assert_allclose(o2, o, atol=1e-12)
    np.testing.assert_allclose(hvT2, hvT, atol=1e-12)


def two_layer_bwd(q, k, v, log_a, dO, hk0=None, hv0=None, dhkT=None, dhvT=None):
    """Backward of the two-layer reading, each step a GLA oracle call: layer two's backward gives ds, the
    gradient of its key 1-a and dv; the softmax backward gives G = dL/dlogits; layer one's gradients are the
    forward (dq) and backward (d(1-a), dk, gate) of the GLA with query G, key 1-a, value k and dO = q."""
    a = np.exp(log_a)
    w = 1.0 - a
    logits = oracle.bwd(np.zeros_like(w), w, k, log_a, q, h0=hk0)["dq"]
    s = softmax(logits)
    g2 = oracle.bwd(s, w, v, log_a, dO, h0=hv0, dhT=dhvT)
    ds = g2["dq"]
    G = s * (ds - (s * ds).sum(-1, keepdims=True))
    dq, _ = oracle.fwd(G, w, k, log_a, hk0)
    g1 = oracle.bwd(G, w, k, log_a, q, h0=hk0, dhT=dhkT)
    return {"dq": dq, "dk": g1["dv"], "dv": g2["dv"],
            "dlog_a": g1["dlog_a"] + g2["dlog_a"] - a * (g1["dk"] + g2["dk"]),
            "dlog_a_cf": g1["dlog_a_cf"] + g2["dlog_a_cf"] - a * (g1["dk"] + g2["dk"]),
            "dhk0": g1["dh0"], "dhv0": g2["dh0"]}


@pytest.mark.parametrize("h0,dhT", [(False, False), (True, True)])
def test_two_layer_reading_backward(h0, dhT):
    d = make(1, 2, 29, 5, 4, 3, seed=6, h0=h0, dhT=dhT, qscale=2.0)
    args = (d["q"], d["k"], d["v"], d["log_a"], d["dO"], d["hk0"], d["hv0"], d["dhkT"], d["dhvT"])
    g = oracle.gsa_bwd(*args, seg=7)
    g2 = two_layer_bwd(*args)
    for n in ("dq", "dk", "dv", "dlog_a"):
        np.testing.assert_allclose(g2[n], g[n], atol=1e-11, err_msg=n)
    np.testing.assert_allclose(g2["dlog_a_cf"], g["dlog_a"], atol=1e-11)
    if h0:
        np.testing.assert_allclose(g2["dhk0"], g["dhk0"], atol=1e-11)
        np.testing.assert_allclose(g2["dhv0"], g["dhv0"], atol=1e-11)


# ---------------------------------------------------------- finite differences
def loss(d, o, hkT, hvT):
    val = float((d["dO"] * o).sum())
    if d["dhkT"] is not None:
        val += float((d["dhkT"] * hkT).sum() + (d["dhvT"] * hvT).sum())
    return val


def test_finite_differences():
    d = make(1, 1, 6, 3, 2, 3, seed=7, h0=True, dhT=True, qscale=2.0)
    names = ("q", "k", "v", "log_a", "hk0", "hv0")
    g = oracle.gsa_bwd(d["q"], d["k"], d["v"], d["log_a"], d["dO"], d["hk0"], d["hv0"], d["dhkT"], d["dhvT"], seg=4)
    grad_of = {"q": "dq", "k": "dk", "v": "dv", "log_a": "dlog_a", "hk0": "dhk0", "hv0": "dhv0"}
    eps = 1e-6
    for n in names:
        x = d[n]
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            vals = []
            for sgn in (1, -1):
                dd = dict(d)
                xx = x.copy()
                xx[idx] += sgn * eps
                dd[n] = xx
                o, _, hkT, hvT = oracle.gsa_fwd(dd["q"], dd["k"], dd["v"], dd["log_a"], dd["hk0"], dd["hv0"])
                vals.append(loss(d, o, hkT, hvT))
            num[idx] = (vals[0] - vals[1]) / (2 * eps)
        np.testing.assert_allclose(g[grad_of[n]], num, atol=1e-7, rtol=1e-6, err_msg=n)


# ------------------------------------------------------------ sequence splits
def test_split_sequence_forward_and_backward():
    """Running [0, L1) then [L1, L) from the first part's final memories gives the whole sequence's outputs;
    chaining the second part's gradients at its entering memories into the first part's dhT gives the whole
    backward."""
    d = make(1, 2, 23, 4, 3, 5, seed=8, qscale=2.0)
    L1 = 9
    part = lambda n, sl: d[n][:, :, sl]  # noqa: E731
    o, _, hk, hv = oracle.gsa_fwd(d["q"], d["k"], d["v"], d["log_a"])
    a = slice(0, L1)
    b = slice(L1, None)
    o1, _, hk1, hv1 = oracle.gsa_fwd(part("q", a), part("k", a), part("v", a), part("log_a", a))
    o2, _, hk2, hv2 = oracle.gsa_fwd(part("q", b), part("k", b), part("v", b), part("log_a", b), hk1, hv1)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=2), o, atol=1e-13)
    np.testing.assert_allclose(hk2, hk, atol=1e-13)
    g = oracle.gsa_bwd(d["q"], d["k"], d["v"], d["log_a"], d["dO"], seg=5)
    g2 = oracle.gsa_bwd(part("q", b), part("k", b), part("v", b), part("log_a", b), part("dO", b), hk1, hv1, seg=5)
    g1 = oracle.gsa_bwd(part("q", a), part("k", a), part("v", a), part("log_a", a), part("dO", a),
                        dhkT=g2["dhk0"], dhvT=g2["dhv0"], seg=5)
    for n in ("dq", "dk", "dv", "dlog_a"):
        np.testing.assert_allclose(np.concatenate([g1[n], g2[n]], axis=2), g[n], atol=1e-12, err_msg=n)


@pytest.mark.parametrize("seg", [1, 3, 64])
def test_checkpoint_spacing_invariance(seg):
    d = make(1, 2, 17, 3, 4, 5, seed=9, h0=True, dhT=True, qscale=2.0)
    args = (d["q"], d["k"], d["v"], d["log_a"], d["dO"], d["hk0"], d["hv0"], d["dhkT"], d["dhvT"])
    ref = oracle.gsa_bwd(*args, seg=17)
    g = oracle.gsa_bwd(*args, seg=seg)
    for n in ref:
        np.testing.assert_allclose(g[n], ref[n], atol=1e-13, err_msg=n)
