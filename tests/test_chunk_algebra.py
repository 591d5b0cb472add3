"""The chunkwise form of the layer, in fp64 numpy, equals the step recurrence.

This pins the algebra that the CUDA path is built on (it is derived, not
printed on the pages): with B_j the inclusive cumsum of log alpha inside a
chunk and Gamma = B at the chunk's last row,
  o_j     = (q_j * e^{B_j}) S_[i] + sum_{s<=j} (sum_c q_jc k_sc e^{B_jc - B_sc}) v_s
  S_[i+1] = diag(e^{Gamma}) S_[i] + sum_j (k_j * e^{Gamma - B_j})^T v_j
and, for the backward with D_i = dL/dS_[i+1] (D_{N-1} = dhT),
  D_{i-1} = (q * e^B)_i^T dO_i + diag(e^{Gamma_i}) D_i,   dh0 = D_{-1}
  dq_j = e^{B_j} * (dO_j S_[i]^T) + sum_{s<=j} dP_js k_s e^{B_j - B_s},   dP_js = dO_j . v_s
  dk_s = e^{Gamma - B_s} * (v_s D_i^T) + sum_{j>=s} dP_js q_j e^{B_j - B_s}
  dv_s = (k_s e^{Gamma - B_s}) D_i + sum_{j>=s} P_js dO_j
  dlog_a_t = sum_{s>=t} (q_s dq_s - k_s dk_s) + sum_v dhT * hT
("Gated Linear Attention Transformers with Hardware-Efficient Training",
atlas.scime.ai summary, section "Approach": chunkwise form, closed-form gate
gradient).
"""
import math

import numpy as np
import pytest

import oracle


def chunk_fwd(q, k, v, la, h0, C):
    L, K = q.shape
    V = v.shape[1]
    S = np.zeros((K, V)) if h0 is None else h0.copy()
    o = np.zeros((L, V))
    states = []
    for i0 in range(0, L, C):
        i1 = min(i0 + C, L)
        Bc = np.cumsum(la[i0:i1], axis=0)
        G = Bc[-1]
        Q, Kc, Vc = q[i0:i1], k[i0:i1], v[i0:i1]
        P = np.einsum("jc,sc,jsc->js", Q, Kc, np.exp(Bc[:, None, :] - Bc[None, :, :]))
        P = np.tril(P)
        states.append(S.copy())
        o[i0:i1] = (Q * np.exp(Bc)) @ S + P @ Vc
        S = np.exp(G)[:, None] * S + (Kc * np.exp(G - Bc)).T @ Vc
    return o, S, states


def chunk_bwd(q, k, v, la, dO, h0, dhT, C):
    L, K = q.shape
    V = v.shape[1]
    _, hT, states = chunk_fwd(q, k, v, la, h0, C)
    D = np.zeros((K, V)) if dhT is None else dhT.copy()
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    starts = list(range(0, L, C))
    for n in reversed(range(len(starts))):
        i0 = starts[n]
        i1 = min(i0 + C, L)
        Bc = np.cumsum(la[i0:i1], axis=0)
        G = Bc[-1]
        Q, Kc, Vc, dOc = q[i0:i1], k[i0:i1], v[i0:i1], dO[i0:i1]
        W = np.exp(Bc[:, None, :] - Bc[None, :, :])  # [j, s, c]
        mask = np.tril(np.ones((i1 - i0, i1 - i0)))
        P = np.einsum("jc,sc,jsc->js", Q, Kc, W) * mask
        dP = (dOc @ Vc.T) * mask
        Sprev = states[n]
        dq[i0:i1] = np.exp(Bc) * (dOc @ Sprev.T) + np.einsum("js,sc,jsc->jc", dP, Kc, W)
        dk[i0:i1] = np.exp(G - Bc) * (Vc @ D.T) + np.einsum("js,jc,jsc->sc", dP, Q, W)
        dv[i0:i1] = (Kc * np.exp(G - Bc)) @ D + P.T @ dOc
        D = (Q * np.exp(Bc)).T @ dOc + np.exp(G)[:, None] * D
    r = q * dq - k * dk
    base = np.zeros(K) if dhT is None else np.sum(dhT * hT, axis=1)
    dla = np.cumsum(r[::-1], axis=0)[::-1] + base
    return dq, dk, dv, dla, D


def _data(L, K, V, seed, strong=False):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((L, K)) / math.sqrt(K)
    k = rng.standard_normal((L, K)) / math.sqrt(K)
    v = rng.standard_normal((L, V)) / math.sqrt(K)
    z = rng.standard_normal((L, K)) * (2.0 if strong else 1.0)
    la = -np.log1p(np.exp(-z)) / (1.0 if strong else 16.0)
    dO = rng.standard_normal((L, V))
    h0 = rng.standard_normal((K, V)) * 0.3
    dhT = rng.standard_normal((K, V)) * 0.3
    return q, k, v, la, dO, h0, dhT


@pytest.mark.parametrize("C", [1, 4, 16, 64])
@pytest.mark.parametrize("L", [64, 77])
def test_chunk_forward_equals_recurrence(C, L):
    q, k, v, la, dO, h0, dhT = _data(L, 8, 6, seed=C + L)
    o_ref, hT_ref = oracle.fwd(q[None, None], k[None, None], v[None, None], la[None, None], h0[None, None])
    o, hT, _ = chunk_fwd(q, k, v, la, h0, C)
    np.testing.assert_allclose(o, o_ref[0, 0], atol=1e-12)
    np.testing.assert_allclose(hT, hT_ref[0, 0], atol=1e-12)


@pytest.mark.parametrize("C", [4, 16, 64])
@pytest.mark.parametrize("strong", [False, True])
def test_chunk_backward_equals_recurrence(C, strong):
    L = 70
    q, k, v, la, dO, h0, dhT = _data(L, 6, 5, seed=C, strong=strong)
    g = oracle.bwd(q[None, None], k[None, None], v[None, None], la[None, None], dO[None, None],
                   h0[None, None], dhT[None, None])
    dq, dk, dv, dla, dh0 = chunk_bwd(q, k, v, la, dO, h0, dhT, C)
    for name, val in (("dq", dq), ("dk", dk), ("dv", dv), ("dlog_a", dla), ("dh0", dh0)):
        ref = g[name][0, 0]
        np.testing.assert_allclose(val, ref, atol=1e-11 * max(1.0, np.abs(ref).max()), err_msg=name)
