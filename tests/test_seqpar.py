"""Sequence-sharded evaluation (chunkwise_linear_rnn_gla_b200.seqpar): a sequence split along L, one
segment per rank, joined by the affine combine of per-segment summaries (decay a, end state U; in the
backward a and W) -- "Gated Linear Attention Transformers with Hardware-Efficient Training",
atlas.scime.ai summary, "Measured effects" (truncated BPTT: the state carried across segments).

- Two gloo ranks on CPU run the host logic (phases, all-gather, rank order, which summaries combine)
  with the per-segment computations supplied by the fp64 oracle and a combine written out here; the
  ranks' outputs put together equal the oracle on the whole sequence.
- On one GPU, three segments run in turn through the library's kernels (gla_fwd, gla_bwd,
  gla_segment_decay, gla_state_combine) with the exchange done by stacking; the result equals the
  oracle on the whole sequence.
"""
import os
import socket
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from chunkwise_linear_rnn_gla_b200.inputs import make_inputs, to_f64_numpy

WORLD = 2
SHAPE = (1, 2, 70, 8, 6)  # B, H, L, Dk, Dv


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _combine(a_all, U_all, r, init, reverse):
    """X_{g+1} = a_g X_g + U_g from X_0 = init (forward), or Y_{g-1} = a_g Y_g + U_g from Y_{G-1} = init."""
    x = np.zeros(U_all.shape[1:]) if init is None else np.array(init, np.float64)
    G = a_all.shape[0]
    order = range(r) if not reverse else range(G - 1, r, -1)
    for g in order:
        x = a_all[g][..., None] * x + U_all[g]
    return x


class _OracleOps:
    """The per-segment computations of seqpar, supplied by the fp64 oracle (CPU, tensors as float64)."""

    @staticmethod
    def _np(*ts):
        return [None if t is None else t.numpy() for t in ts]

    @staticmethod
    def summary_fwd(q, k, v, la):
        import oracle

        q_, k_, v_, la_ = _OracleOps._np(q, k, v, la)
        _, U = oracle.fwd(q_, k_, v_, la_)
        return torch.from_numpy(np.exp(la_.sum(axis=2))), torch.from_numpy(U)

    @staticmethod
    def finish_fwd(q, k, v, la, a_all, U_all, r, h0):
        import oracle

        q_, k_, v_, la_ = _OracleOps._np(q, k, v, la)
        h0_r = _combine(a_all.numpy(), U_all.numpy(), r, None if h0 is None else h0.numpy(), False)
        o, hT = oracle.fwd(q_, k_, v_, la_, h0_r)
        return torch.from_numpy(o), torch.from_numpy(hT), torch.from_numpy(h0_r)

    @staticmethod
    def summary_bwd(q, k, v, la, dO):
        import oracle

        q_, k_, v_, la_, dO_ = _OracleOps._np(q, k, v, la, dO)
        g = oracle.bwd(q_, k_, v_, la_, dO_)
        return torch.from_numpy(np.exp(la_.sum(axis=2))), torch.from_numpy(g["dh0"])

    @staticmethod
    def finish_bwd(q, k, v, la, dO, h0_r, a_all, W_all, r, dhT):
        import oracle

        q_, k_, v_, la_, dO_ = _OracleOps._np(q, k, v, la, dO)
        dhT_r = _combine(a_all.numpy(), W_all.numpy(), r, None if dhT is None else dhT.numpy(), True)
        g = oracle.bwd(q_, k_, v_, la_, dO_, h0_r.numpy(), dhT_r)
        return {n: torch.from_numpy(g[n]) for n in ("dq", "dk", "dv", "dlog_a", "dh0")}


def _whole():
    B, H, L, K, V = SHAPE
    inp = make_inputs(B, H, L, K, V, "f32", seed=60, h0=True, dhT=True)
    return {n: to_f64_numpy(t) for n, t in inp.items()}


def _worker(rank, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(WORLD),
                      LOCAL_RANK=str(rank))
    try:
        from chunkwise_linear_rnn_gla_b200 import seqpar

        dist.init_process_group("gloo", init_method="env://", timeout=timedelta(seconds=60))
        f = _whole()
        lens = seqpar.split_lengths(f["q"].shape[2], WORLD)
        lo = sum(lens[:rank])
        seg = {n: torch.from_numpy(np.ascontiguousarray(f[n][:, :, lo:lo + lens[rank]]))
               for n in ("q", "k", "v", "log_a", "dO")}
        sh = seqpar.SeqShard(ops=_OracleOps())
        o, hT, h0_r = sh.forward(seg["q"], seg["k"], seg["v"], seg["log_a"], torch.from_numpy(f["h0"]))
        g = sh.backward(seg["q"], seg["k"], seg["v"], seg["log_a"], seg["dO"], h0_r, torch.from_numpy(f["dhT"]))
        got = [None] * WORLD
        dist.all_gather_object(got, (rank, o.numpy(), hT.numpy(), {n: t.numpy() for n, t in g.items()}))
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, got))
    except Exception as e:  # report instead of hanging the parent
        q.put((rank, "error: %r" % (e,)))


def test_two_rank_gloo_sequence_shards():
    import oracle

    ctx = mp.get_context("spawn")
    qu = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, qu)) for r in range(WORLD)]
    for p in procs:
        p.start()
    res = [qu.get(timeout=120) for _ in range(WORLD)]
    for p in procs:
        p.join(timeout=60)
    for r, got in res:
        assert not isinstance(got, str), got
    got = sorted(res[0][1], key=lambda x: x[0])
    f = _whole()
    o_ref, hT_ref = oracle.fwd(f["q"], f["k"], f["v"], f["log_a"], f["h0"])
    ref = oracle.bwd(f["q"], f["k"], f["v"], f["log_a"], f["dO"], f["h0"], f["dhT"])
    np.testing.assert_allclose(np.concatenate([x[1] for x in got], axis=2), o_ref, rtol=0, atol=1e-10)
    np.testing.assert_allclose(got[-1][2], hT_ref, rtol=0, atol=1e-10)  # the last segment's end state
    for n in ("dq", "dk", "dv", "dlog_a"):
        np.testing.assert_allclose(np.concatenate([x[3][n] for x in got], axis=2), ref[n], rtol=0, atol=1e-9)
    np.testing.assert_allclose(got[0][3]["dh0"], ref["dh0"], rtol=0, atol=1e-10)  # segment 0's dh0


@pytest.mark.gpu
@pytest.mark.parametrize("impl,dtype,K,V", [("tc", "bf16", 128, 128), ("simt", "f32", 64, 64)])
def test_sequence_shards_on_one_gpu(impl, dtype, K, V):
    """Three segments of unequal length (one ragged chunk each) through the library's kernels, the
    exchange done by stacking the summaries; against the oracle on the whole sequence."""
    from chunkwise_linear_rnn_gla_b200 import seqpar
    from tests.parity import compare

    import oracle

    B, H, L = 1, 2, 700
    inp = make_inputs(B, H, L, K, V, dtype, seed=61, h0=True, dhT=True)
    f = {n: to_f64_numpy(t) for n, t in inp.items()}
    d = {n: t.cuda() for n, t in inp.items()}
    lens = [300, 257, 143]
    cuts = np.cumsum([0] + lens)
    seg = [{n: d[n][:, :, cuts[i]:cuts[i + 1]].contiguous() for n in ("q", "k", "v", "log_a", "dO")}
           for i in range(3)]
    kw = dict(impl=impl)
    summ = [seqpar.summary_fwd(s["q"], s["k"], s["v"], s["log_a"], **kw) for s in seg]
    a_all = torch.stack([x[0] for x in summ]).contiguous()
    U_all = torch.stack([x[1] for x in summ]).contiguous()
    outs = [seqpar.finish_fwd(s["q"], s["k"], s["v"], s["log_a"], a_all, U_all, i, d["h0"], **kw)
            for i, s in enumerate(seg)]
    bsum = [seqpar.summary_bwd(s["q"], s["k"], s["v"], s["log_a"], s["dO"], **kw) for s in seg]
    W_all = torch.stack([x[1] for x in bsum]).contiguous()
    grads = [seqpar.finish_bwd(s["q"], s["k"], s["v"], s["log_a"], s["dO"], outs[i][2], a_all, W_all, i, d["dhT"],
                               **kw) for i, s in enumerate(seg)]
    torch.cuda.synchronize()
    o_ref, hT_ref = oracle.fwd(f["q"], f["k"], f["v"], f["log_a"], f["h0"])
    ref = oracle.bwd(f["q"], f["k"], f["v"], f["log_a"], f["dO"], f["h0"], f["dhT"])
    compare("o", torch.cat([x[0] for x in outs], dim=2), o_ref, dtype)
    compare("hT", outs[-1][1], hT_ref, dtype)
    for n in ("dq", "dk", "dv", "dlog_a"):
        compare(n, torch.cat([g[n] for g in grads], dim=2), ref[n], dtype)
    compare("dh0", grads[0]["dh0"], ref["dh0"], dtype)


@pytest.mark.gpu
@pytest.mark.parametrize("L", [300, 128 * 20 + 37])
def test_summary_entry_points_match_the_full_passes(L):
    """gla_fwd_final_state / gla_bwd_initial_grad (the state walks alone) give the hT / dh0 of the full
    gla_fwd / gla_bwd bit for bit (the same walk kernels; the long case runs the segmented walks), and
    the oracle's."""
    import chunkwise_linear_rnn_gla_b200 as gla
    from tests.parity import compare, oracle_bwd, oracle_fwd

    B, H, K, V = 1, 2, 128, 128
    inp = make_inputs(B, H, L, K, V, "bf16", seed=62, h0=True, dhT=True)
    d = {n: t.cuda() for n, t in inp.items()}
    _, hT = gla.gla_fwd(d["q"], d["k"], d["v"], d["log_a"], d["h0"], impl="tc")
    hT2 = gla.gla_fwd_final_state(d["q"], d["k"], d["v"], d["log_a"], d["h0"], impl="tc")
    g = gla.gla_bwd(d["q"], d["k"], d["v"], d["log_a"], d["dO"], d["h0"], d["dhT"], impl="tc")
    dh02 = gla.gla_bwd_initial_grad(d["q"], d["k"], d["v"], d["log_a"], d["dO"], d["dhT"], impl="tc")
    torch.cuda.synchronize()
    assert torch.equal(hT, hT2)
    assert torch.equal(g["dh0"], dh02)
    compare("hT", hT2, oracle_fwd(inp)[1], "bf16")
    compare("dh0", dh02, oracle_bwd(inp)["dh0"], "bf16")
