"""The pins are sharp enough: each plausible mistake planted in a copy of the oracle's C sources makes at
least one pin fail, while the oracle as it stands passes them all.

Every mutant is a one-line change of the kind a reader could miss (a wrong index or operand order, a
dropped term, a read before the update, a missing factor). It is compiled into a temporary library,
bound with oracle.oracle.with_library, and run through a compact set of the checks of
tests/test_oracle_pins.py and tests/test_gsa_oracle.py:
the O(L^2) parallel forms, the hand-derived worked examples, central finite differences and the two
ways of computing the GLA gate gradient.
"""
import json
import math
import os
import shutil
import subprocess
import tempfile

import numpy as np
import pytest

from oracle import oracle as ora_mod
from tests.test_gsa_oracle import brute_force as gsa_brute_force
from tests.test_oracle_pins import brute_force_fwd as gla_brute_force

HERE = os.path.dirname(os.path.abspath(__file__))
ORACLE_DIR = os.path.join(os.path.dirname(HERE), "oracle")
GSA_GOLD = os.path.join(HERE, "golden", "gsa_worked_example.json")

# (name, file, text in the source, replacement)
MUTANTS = [
    ("gla: output reads the state before the update", "gla_oracle.c",
     "    for (i64 c = 0; c < K; ++c) {\n        const double a = exp(la[c]);",
     "    if (o) { for (i64 x = 0; x < V; ++x) o[x] = 0.0;\n"
     "        for (i64 c = 0; c < K; ++c) for (i64 x = 0; x < V; ++x) o[x] += q[c] * S[c * V + x]; o = NULL; }\n"
     "    for (i64 c = 0; c < K; ++c) {\n        const double a = exp(la[c]);"),
    ("gla: decay applied to the value index", "gla_oracle.c",
     "for (i64 x = 0; x < V; ++x) row[x] = a * row[x] + kc * v[x];",
     "for (i64 x = 0; x < V; ++x) row[x] = exp(la[x % K]) * row[x] + kc * v[x];"),
    ("gla: direct gate gradient without the factor a", "gla_oracle.c",
     "if (dlog_a) dlog_a[rk + c] = exp(log_a[rk + c]) * acc_a;",
     "if (dlog_a) dlog_a[rk + c] = acc_a;"),
    ("gla: closed form without the dhT hT term", "gla_oracle.c",
     "double run = base;", "double run = 0.0 * base;"),
    ("gla: state gradient not decayed between steps", "gla_oracle.c",
     "for (i64 x = 0; x < V; ++x) G[c * V + x] *= a;", "for (i64 x = 0; x < V; ++x) G[c * V + x] *= 1.0 + 0.0 * a;"),
    ("gsa: write weight a instead of 1 - a", "gsa_oracle.c",
     "const double a = exp(la[c]), w = 1.0 - a;\n        double* kr", "const double a = exp(la[c]), w = a;\n        double* kr"),
    ("gsa: value memory written with k", "gsa_oracle.c",
     "for (i64 x = 0; x < V; ++x) vr[x] = a * vr[x] + w * v[x];",
     "for (i64 x = 0; x < V; ++x) vr[x] = a * vr[x] + w * k[x % K];"),
    ("gsa: softmax backward without the <s, ds> term", "gsa_oracle.c",
     "for (i64 c = 0; c < m; ++c) dz[c] = s[c] * (ds[c] - sd);", "for (i64 c = 0; c < m; ++c) dz[c] = s[c] * ds[c];"),
    ("gsa: gate gradient with the write weight's sign flipped", "gsa_oracle.c",
     "dlog_a[rm + c] = a * (da - dw);", "dlog_a[rm + c] = a * (da + dw);"),
    ("gsa: key memory gradient not decayed between steps", "gsa_oracle.c",
     "GK[c * K + d] = a * gk;", "GK[c * K + d] = gk;"),
]


def build_mutant(tmp, fname, old, new):
    srcs = {}
    for f in ("gla_oracle.c", "gsa_oracle.c"):
        text = open(os.path.join(ORACLE_DIR, f)).read()
        if f == fname:
            assert text.count(old) == 1, "mutation site not found once in %s: %r" % (f, old)
            text = text.replace(old, new)
        path = os.path.join(tmp, f)
        open(path, "w").write(text)
        srcs[f] = path
    so = os.path.join(tmp, "libmutant.so")
    subprocess.run(["gcc", "-O1", "-fopenmp", "-shared", "-fPIC", "-std=c99", srcs["gla_oracle.c"], srcs["gsa_oracle.c"],
                    "-o", so, "-lm"], check=True)
    return ora_mod.with_library(so)


# ------------------------------------------------------------------ the checks
def close(a, b, tol):
    return np.allclose(a, b, atol=tol, rtol=0)


def gla_checks(ora):
    """Names of the GLA pins that fail."""
    failed = []
    rng = np.random.default_rng(0)
    B, H, L, K, V = 1, 2, 9, 3, 4
    q, k = rng.standard_normal((2, B, H, L, K)) / math.sqrt(K)
    v = rng.standard_normal((B, H, L, V))
    la = np.log(1 / (1 + np.exp(-2 * rng.standard_normal((B, H, L, K)))))
    h0 = 0.3 * rng.standard_normal((B, H, K, V))
    dO = rng.standard_normal((B, H, L, V))
    dhT = 0.3 * rng.standard_normal((B, H, K, V))
    o, hT = ora.fwd(q, k, v, la, h0)
    if not close(o, gla_brute_force(q, k, v, la, h0), 1e-12):
        failed.append("parallel form")
    g = ora.bwd(q, k, v, la, dO, h0, dhT, seg=4)
    if not close(g["dlog_a"], g["dlog_a_cf"], 1e-10):
        failed.append("direct = closed-form gate gradient")
    # finite differences of <dO, o> + <dhT, hT> in a few coordinates of each input
    eps = 1e-6

    def loss(q_, k_, v_, la_, h0_):
        o_, hT_ = ora.fwd(q_, k_, v_, la_, h0_)
        return float((dO * o_).sum() + (dhT * hT_).sum())

    args = [q, k, v, la, h0]
    for n, gname in enumerate(("dq", "dk", "dv", "dlog_a", "dh0")):
        x = args[n]
        for idx in [(0, 0, 2, 1), (0, 1, 7, 0)] if x.ndim == 4 and n < 4 else [(0, 1, 2, 3)]:
            idx = tuple(i % s for i, s in zip(idx, x.shape))
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            ap, am = list(args), list(args)
            ap[n], am[n] = xp, xm
            num = (loss(*ap) - loss(*am)) / (2 * eps)
            if abs(num - g[gname][idx]) > 1e-6 * max(1.0, abs(num)):
                failed.append("finite differences " + gname)
                break
    return failed


def gsa_checks(ora):
    failed = []
    ex = json.load(open(GSA_GOLD))
    o, s, hkT, hvT = ora.gsa_fwd(np.array(ex["q"])[None, None], np.array(ex["k"])[None, None],
                                 np.array(ex["v"])[None, None], np.log(np.array(ex["alpha"]))[None, None])
    if not (close(o[0, 0], np.array(ex["o"]), 1e-12) and close(s[0, 0], np.array(ex["s"]), 1e-12)):
        failed.append("worked example")
    rng = np.random.default_rng(1)
    B, H, L, K, V, m = 1, 2, 8, 3, 4, 5
    q = 2 * rng.standard_normal((B, H, L, K))
    k = rng.standard_normal((B, H, L, K)) / math.sqrt(K)
    v = rng.standard_normal((B, H, L, V))
    la = np.log(1 / (1 + np.exp(-2 * rng.standard_normal((B, H, L, m)))))
    hk0 = 0.5 * rng.standard_normal((B, H, m, K))
    hv0 = 0.5 * rng.standard_normal((B, H, m, V))
    dO = rng.standard_normal((B, H, L, V))
    o, _, _, _ = ora.gsa_fwd(q, k, v, la, hk0, hv0)
    if not close(o, gsa_brute_force(q, k, v, la, hk0, hv0), 1e-12):
        failed.append("parallel form")
    g = ora.gsa_bwd(q, k, v, la, dO, hk0, hv0, seg=3)
    eps = 1e-6

    def loss(q_, k_, v_, la_):
        return float((dO * ora.gsa_fwd(q_, k_, v_, la_, hk0, hv0)[0]).sum())

    args = [q, k, v, la]
    for n, gname in enumerate(("dq", "dk", "dv", "dlog_a")):
        x = args[n]
        for idx in [(0, 0, 2, 1), (0, 1, 6, 2)]:
            idx = tuple(i % s for i, s in zip(idx, x.shape))
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            ap, am = list(args), list(args)
            ap[n], am[n] = xp, xm
            num = (loss(*ap) - loss(*am)) / (2 * eps)
            if abs(num - g[gname][idx]) > 1e-6 * max(1.0, abs(num)):
                failed.append("finite differences " + gname)
                break
    return failed


@pytest.fixture(scope="module")
def tmpdir():
    d = tempfile.mkdtemp(prefix="oracle_mutants_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_unmutated_oracle_passes_the_checks(tmpdir):
    ora = build_mutant(os.path.join(tmpdir), "none", "", "")
    assert gla_checks(ora) == []
    assert gsa_checks(ora) == []


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
@pytest.mark.parametrize("name,fname,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(tmpdir, name, fname, old, new):
    sub = os.path.join(tmpdir, str(abs(hash(name))))
    os.makedirs(sub, exist_ok=True)
    ora = build_mutant(sub, fname, old, new)
    failed = (gla_checks(ora) if fname == "gla_oracle.c" else gsa_checks(ora))
    assert failed, "the mutant '%s' passed every pin" % name
