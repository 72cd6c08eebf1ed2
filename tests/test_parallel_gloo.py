"""Token sharding across ranks, on CPU with the gloo backend (world size 2).

Each rank runs the estimator (here the CPU oracle, as test infrastructure)
on its token share with token_offset = its first token; the sum all-reduce of
the per-rank G_W must equal a single run over the whole batch, and the
per-token outputs must be the single run's rows.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from zeroth_order_transformer_dust_b200.parallel import allreduce_weight_grad, token_shard


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_token_shard_partitions_the_batch():
    for T in (0, 1, 7, 128, 16385):
        for world in (1, 2, 3, 8):
            spans = [token_shard(T, world, r) for r in range(world)]
            assert spans[0][0] == 0
            for (s0, n0), (s1, _) in zip(spans, spans[1:]):
                assert s1 == s0 + n0
            assert sum(n for _, n in spans) == T
            assert max(n for _, n in spans) - min(n for _, n in spans) <= 1
    with pytest.raises(ValueError):
        token_shard(10, 2, 2)


def _worker(rank, world, port, S, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        import synth
        wl = synth.Workload("gloo", "head", T=10, d=6, V=40, K=8, S=S, sigma=0.05, seed=3,
                            dtype="f32", targets="zipf")
        inp = synth.make_head_inputs(wl)
        t0, n = token_shard(wl.T, world, rank)
        prm = oracle.Params(T=n, d=wl.d, V=wl.V, K=wl.K, S=wl.S, sigma=wl.sigma, seed=wl.seed,
                            token_offset=t0)
        out = oracle.head_grad(inp["H"][t0:t0 + n], inp["W"], inp["targets"][t0:t0 + n], prm)
        G = torch.from_numpy(out["G"])
        allreduce_weight_grad(G)
        q.put((rank, t0, n, G.numpy(), out["rewards"], out["g"]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("S", [0, 5])
def test_sharded_weight_grad_equals_single_run(S):
    import oracle
    import synth
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, S, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    wl = synth.Workload("gloo", "head", T=10, d=6, V=40, K=8, S=S, sigma=0.05, seed=3,
                        dtype="f32", targets="zipf")
    inp = synth.make_head_inputs(wl)
    prm = oracle.Params(T=wl.T, d=wl.d, V=wl.V, K=wl.K, S=wl.S, sigma=wl.sigma, seed=wl.seed)
    ref = oracle.head_grad(inp["H"], inp["W"], inp["targets"], prm)
    for rank, t0, n, G, rewards, g in res:
        np.testing.assert_allclose(G, ref["G"], rtol=0, atol=1e-12)
        np.testing.assert_array_equal(rewards, ref["rewards"][t0:t0 + n])
        np.testing.assert_allclose(g, ref["g"][t0:t0 + n], rtol=0, atol=1e-13)
