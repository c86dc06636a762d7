"""Token data parallelism, world size 2 over gloo on the CPU.

Each rank takes its contiguous share of one batch, computes the adapter
gradient of its tokens with the oracle, and sums it over the ranks through
dp.allreduce_adapter_grad. The result must equal the oracle's gradient of the
whole batch (float64, exact mode: only the summation order differs). A rank
that fails before the collective must make the other one fail within the
process-group timeout instead of hanging.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
from quantized_rl_fine_b200 import dp, synth
from quantized_rl_fine_b200.configs import MoEConfig

CFG = MoEConfig("dp_tiny_int4_adapter", E=4, k=2, d=64, f=64, T=24, fmt="int4", swiglu=True,
                logits="normal", adapter=True, train=True, seed=3101)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_inputs():
    wl = synth.make_workload(CFG, "cpu")

    def qw(w):
        sc = w.scales.view(torch.int16).numpy().view(np.uint16) if w.fmt == "int4" else w.scales.numpy()
        return O.QWeight(w.fmt, w.packed.numpy(), sc)

    return dict(x=wl["x"].float().numpy().astype(np.float64), logits=wl["logits"].numpy(),
                dy=wl["dy"].float().numpy().astype(np.float64), w_gu=qw(wl["w_gu"]), w_d=qw(wl["w_d"]),
                R=wl["adapter"].float().numpy().astype(np.float64))


def _adapter_grad(inp, lo, hi):
    fwd = O.moe_forward(inp["x"][lo:hi], inp["logits"][lo:hi], CFG.k, CFG.chunk_size, inp["w_gu"],
                        inp["w_d"], R=inp["R"], exact=True)
    bwd = O.moe_backward(fwd, inp["dy"][lo:hi], inp["w_gu"], inp["w_d"], R=inp["R"], exact=True)
    return bwd["d_adapter"]


def _worker(rank, world, port, mode, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=10))
    try:
        if mode == "fail" and rank == 1:
            raise RuntimeError("rank 1 fails before the collective")
        inp = _oracle_inputs()
        lo, hi = dp.token_shard(CFG.T, rank, world)
        g = torch.from_numpy(_adapter_grad(inp, lo, hi)).to(torch.float64)
        # the collective runs on the float32 tensor the library produces; the
        # float64 sum is exchanged alongside to check the rows' partition exactly
        g32 = g.to(torch.float32)
        dp.allreduce_adapter_grad(g32)
        dist.all_reduce(g, op=dist.ReduceOp.SUM)
        out[rank] = (g.numpy(), g32.numpy())
    except Exception as exc:  # reported to the parent
        out[rank] = repr(exc)
    finally:
        dist.destroy_process_group()


def _run(mode):
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, mode, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        for p in procs:
            if p.is_alive():
                p.kill()
                pytest.fail("a rank did not finish")
        return dict(out)


def test_token_shards_partition_the_batch():
    for T in (1, 2, 7, 24, 1000):
        for world in (1, 2, 3, 8):
            spans = [dp.token_shard(T, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == T
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1


def test_allreduce_of_shard_gradients_equals_whole_batch_gradient():
    out = _run("ok")
    whole = _adapter_grad(_oracle_inputs(), 0, CFG.T)
    for rank in (0, 1):
        assert not isinstance(out[rank], str), out[rank]
        g64, g32 = out[rank]
        np.testing.assert_allclose(g64, whole, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(g32, whole, rtol=1e-6, atol=1e-6)


def test_a_failing_rank_does_not_hang_the_other():
    out = _run("fail")
    assert "rank 1 fails" in out[1]
    assert isinstance(out[0], str)      # the survivor's collective ended with an error
