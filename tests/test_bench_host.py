"""Host-side checks of the benchmark's accounting (CPU only): the algorithmic byte and flop
model of one fwd+bwd step, the per-kernel byte models behind the roofline, and the rule that a
recorded ncu traffic figure is dropped once the kernel's source has changed."""
import hashlib
import os
import sys
from types import SimpleNamespace

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _shape(B, H, L, K, V):
    return SimpleNamespace(B=B, H=H, L=L, K=K, V=V)


def _io_bytes(B, H, L, K, V):
    """Every tensor the layer reads or writes once, listed one by one (bf16 q, k, v, o, dO, dq, dk,
    dv; fp32 log a, dlog a, hT, dh0)."""
    th, bh = B * H * L, B * H
    fwd = [("q", th * K, 2), ("k", th * K, 2), ("v", th * V, 2), ("log_a", th * K, 4), ("o", th * V, 2),
           ("hT", bh * K * V, 4)]
    bwd = [("q", th * K, 2), ("k", th * K, 2), ("v", th * V, 2), ("dO", th * V, 2), ("log_a", th * K, 4),
           ("dq", th * K, 2), ("dk", th * K, 2), ("dv", th * V, 2), ("dlog_a", th * K, 4),
           ("dh0", bh * K * V, 4)]
    return sum(n * e for _, n, e in fwd), sum(n * e for _, n, e in bwd)


def _gemm_flops(B, H, L, K, V, C):
    """The chunk form's contractions per chunk of C tokens, 2 flops per multiply-add; the
    intra-chunk products count their causal half."""
    n_chunks = B * H * (L // C)
    fwd = [2 * C * K * V,  # state update K~^T V
           2 * C * K * V,  # inter output Q~ S
           C * C * K,      # causal half of Q K^T
           C * C * V]      # causal half of P V
    bwd = [2 * C * K * V] * 4 + [  # D chain, dO S^T, v D^T, K~ D
        C * C * V,  # dP = dO V^T
        C * C * V,  # P^T dO
        C * C * K,  # dP K
        C * C * K,  # dP^T Q
        C * C * K]  # P recomputed
    return n_chunks * sum(fwd), n_chunks * sum(bwd)


def test_layer_model_matches_the_tensor_list():
    for (B, H, L, K, V) in [(4, 4, 2048, 256, 512), (8, 4, 2048, 128, 256), (1, 4, 16384, 128, 256)]:
        m = bench.algorithmic_model(_shape(B, H, L, K, V), C=128)
        bf, bb = _io_bytes(B, H, L, K, V)
        assert (m["bytes_fwd"], m["bytes_bwd"]) == (bf, bb)
        ff, fb = _gemm_flops(B, H, L, K, V, 128)
        assert (m["flops_fwd"], m["flops_bwd"]) == (ff, fb)


def test_layer_roofline_of_the_1p3b_shape():
    m = bench.algorithmic_model(_shape(4, 4, 2048, 256, 512), C=128)
    assert m["bytes"] == 385875968 and m["flops"] == 62277025792
    t_hbm = m["bytes"] / 6551e9
    t_flop = m["flops"] / 1655.1e12
    assert t_hbm > t_flop  # bound by HBM
    assert abs(t_hbm * 1e6 - 58.9) < 0.05


def test_kernel_byte_models_of_the_1p3b_shape():
    """Per-launch algorithmic megabytes of the tensor-core kernels at B=4, H=4, L=2048, d_k=256,
    d_v=512, C=128, as tabulated with the measured kernel times."""
    m = bench.kernel_models(_shape(4, 4, 2048, 256, 512), 128)
    want = {"tc_prep": 109.3, "tc_walk_states": 117.4, "tc_output": 159.4, "tc_walk_dstates": 117.4,
            "tc_output_dv": 159.4, "tc_bwd_chunk": 352.6}
    for name, mb in want.items():
        assert abs(m[name]["bytes"] / 1e6 - mb) < 0.05, name
        assert m[name]["bound"] == "hbm"
    # the decode step streams the fp32 state once in and once out
    d = bench.kernel_models(_shape(64, 4, 1, 128, 256), 128)["step"]
    assert d["bytes"] == 2 * 64 * 4 * 128 * 256 * 4


def test_recorded_traffic_is_dropped_when_the_source_changes(monkeypatch):
    src = "gla_step.cu"
    with open(os.path.join(ROOT, "chunkwise_linear_rnn_gla_b200", "csrc", src), "rb") as f:
        sha = hashlib.sha1(f.read()).hexdigest()
    monkeypatch.setattr(bench, "NCU_TRAFFIC", {"current": (123, src, sha), "stale": (456, src, "0" * 40),
                                               "missing": (789, "no_such_file.cu", sha)})
    assert bench.measured_traffic("current") == 123
    assert bench.measured_traffic("stale") is None
    assert bench.measured_traffic("missing") is None
    assert bench.measured_traffic("unknown") is None


def test_recorded_traffic_entries_name_existing_sources():
    for name, (nbytes, src, sha) in bench.NCU_TRAFFIC.items():
        assert nbytes > 0 and len(sha) == 40
        assert os.path.exists(os.path.join(ROOT, "chunkwise_linear_rnn_gla_b200", "csrc", src)), name


def test_workload_timer_lists_and_validates_without_a_gpu(capsys):
    import pytest

    from chunkwise_linear_rnn_gla_b200 import time_workloads

    assert time_workloads.main(["--list"]) == 0
    listed = [line.split(" - ")[0] for line in capsys.readouterr().out.splitlines()]
    assert "gla1p3b_fwdbwd" in listed and "decode" in listed and "tiny_f32" not in listed
    with pytest.raises(SystemExit):
        time_workloads.main(["--only", "no_such_workload"])


def _gsa_io_bytes(B, H, L, K, V, m):
    """Gated slot attention: every tensor the method reads or writes once (bf16 q, k, v, o, dO, dq, dk, dv;
    fp32 gate and its gradient over the m slots), no memories."""
    th = B * H * L
    fwd = [("q", th * K, 2), ("k", th * K, 2), ("v", th * V, 2), ("log_a", th * m, 4), ("o", th * V, 2)]
    bwd = [("q", th * K, 2), ("k", th * K, 2), ("v", th * V, 2), ("dO", th * V, 2), ("log_a", th * m, 4),
           ("dq", th * K, 2), ("dk", th * K, 2), ("dv", th * V, 2), ("dlog_a", th * m, 4)]
    return sum(n * e for _, n, e in fwd) + sum(n * e for _, n, e in bwd)


def _gsa_flops(B, H, L, K, V, m, C):
    """The method's contractions per chunk of C tokens (2 flops per multiply-add, causal halves for the
    intra-chunk products), as two GLA layers over the slots joined by the softmax."""
    n_chunks = B * H * (L // C)

    def gla_fwd_out(Kg, Vg):  # the output of a GLA with key width Kg and value width Vg, states given
        return [2 * C * Kg * Vg, C * C * Kg, C * C * Vg]

    def gla_bwd(Kg, Vg):  # a GLA backward with key width Kg, value width Vg
        return [2 * C * Kg * Vg] * 4 + [C * C * Vg, C * C * Vg, C * C * Kg, C * C * Kg, C * C * Kg]

    def slot_read(Dx):  # the value-side read of a slot memory with a Dx-wide query: inter, q k^T, P1 Phi
        return [2 * C * Dx * m, C * C * Dx, C * C * m]

    fwd = [2 * C * m * K, 2 * C * m * V]        # both memories' state updates
    fwd += slot_read(K)                          # layer one: the logits
    fwd += gla_fwd_out(m, V)                     # layer two: o
    bwd = gla_bwd(m, V)                          # layer two's backward
    bwd += slot_read(V)                          # the read of the value memory with dO: ds
    bwd += gla_fwd_out(m, K)                     # layer one's forward with query G: dq
    bwd += gla_bwd(m, K)                         # layer one's backward with dO = q
    return n_chunks * (sum(fwd) + sum(bwd))


def test_gsa_model_matches_the_tensor_and_contraction_lists():
    for (B, H, L, K, V, m) in [(4, 4, 2048, 256, 512, 128), (2, 3, 1024, 128, 64, 64)]:
        g = bench.gsa_model(B, H, L, K, V, m, C=128)
        assert g["bytes"] == _gsa_io_bytes(B, H, L, K, V, m)
        assert g["flops"] == _gsa_flops(B, H, L, K, V, m, 128)


def test_gsa_roofline_of_the_1p3b_shape():
    g = bench.gsa_model(4, 4, 2048, 256, 512, 128)
    assert g["per_token_head"] == {"bytes": 9728, "flops": 1933312}
    t_hbm = g["bytes"] / 6551e9
    assert t_hbm > g["flops"] / 1655.1e12  # bound by HBM
    assert abs(t_hbm * 1e6 - 48.66) < 0.01
