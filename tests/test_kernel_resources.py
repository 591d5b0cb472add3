"""Register and spill budgets of the hot kernels, checked from ptxas's own report (no GPU needed).

A kernel's residency follows from its registers: a 512-thread decode block needs at most 64 registers a
thread for two blocks to share an SM's 64 K registers, and a one-CTA-per-SM tensor-core kernel of 576
threads is capped at 96. A change that grows a kernel past such a cap, or makes it spill, changes its
speed without changing its results, so the parity tests cannot see it. These tests compile the sources of
the hot kernels for sm_100a with `-Xptxas -v` (the library's own flags) and hold each kernel to the
budget it was measured at.
"""
import os
import re
import shutil
import subprocess
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "chunkwise_linear_rnn_gla_b200", "csrc")
FILES = ["gla_step", "gla_gsa", "gla_gsa_read", "gla_tc_bwd", "gla_tc_out", "gla_tc_prep", "gla_tc_states",
         "gla_tc_walk"]


def _nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    return None


def _compile(args):
    nvcc, name, out = args
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include"), "-Xptxas", "-v", "-c",
           os.path.join(CSRC, name + ".cu"), "-o", os.path.join(out, name + ".o")]
    r = subprocess.run(cmd, capture_output=True, text=True)
    return name, r.returncode, r.stdout + r.stderr


def _parse(text):
    """{mangled entry name: (registers, spill store bytes, spill load bytes)}"""
    res, cur, spill = {}, None, (0, 0)
    for line in text.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            cur, spill = m.group(1), (0, 0)
            continue
        m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m and cur:
            spill = (int(m.group(1)), int(m.group(2)))
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and cur:
            res[cur] = (int(m.group(1)),) + spill
            cur = None
    return res


@pytest.fixture(scope="module")
def report():
    nvcc = _nvcc()
    if nvcc is None:
        pytest.skip("nvcc not found")
    out = tempfile.mkdtemp(prefix="gla_ptxas_")
    try:
        with ThreadPoolExecutor(max_workers=len(FILES)) as ex:
            results = list(ex.map(_compile, [(nvcc, f, out) for f in FILES]))
    finally:
        shutil.rmtree(out, ignore_errors=True)
    kernels = {}
    for name, rc, text in results:
        assert rc == 0, "nvcc failed on %s:\n%s" % (name, text[-2000:])
        kernels.update(_parse(text))
    return kernels


def _select(report, base, tmpl=""):
    """Entries whose mangled name holds the kernel name (length-prefixed, as the mangling writes it) and,
    optionally, a piece of its template arguments."""
    key = "%d%s" % (len(base), base)
    got = {k: v for k, v in report.items() if key in k and tmpl in k}
    assert got, "no entry function %s%s in the compiled sources" % (base, tmpl)
    return got


@pytest.mark.parametrize("base", ["k_step_rows", "k_gsa_step"])
def test_decode_kernels_fit_two_blocks_per_sm(report, base):
    """512-thread decode blocks, one per head: two per SM keep a 256-head batch in one wave."""
    for name, (regs, st, ld) in _select(report, base).items():
        assert regs <= 64, (name, regs)
        assert st == 0 and ld == 0, (name, st, ld)


@pytest.mark.parametrize("base,tmpl", [("k_bwd_chunk", ""), ("k_states_walk", ""), ("k_chunk_out", ""),
                                       ("k_walk", ""), ("k_tc_prep", "ILi256E"), ("k_gsa_gate_prep", "")])
def test_tensor_core_kernels_do_not_spill(report, base, tmpl):
    for name, (regs, st, ld) in _select(report, base, tmpl).items():
        assert st == 0 and ld == 0, (name, regs, st, ld)


@pytest.mark.parametrize("base,tmpl,cap,spill", [
    # 576 threads, one CTA per SM: five warps on two of the four register-file quarters cap it at 96
    ("k_gsa_slot_read", "", 96, 64),
    ("k_bwd_chunk", "", 96, 0),
    # the d_k = 128 preparation spills a few bytes at its two-CTAs-per-SM cap
    ("k_tc_prep", "ILi128E", 96, 32),
])
def test_register_caps_and_small_spills(report, base, tmpl, cap, spill):
    for name, (regs, st, ld) in _select(report, base, tmpl).items():
        assert regs <= cap, (name, regs)
        assert st <= spill, (name, st)
