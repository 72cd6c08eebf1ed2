"""Token sharding across ranks, on CPU with the gloo backend (world size 2).

Each rank runs the estimator (here the CPU oracle, as test infrastructure)
on its token share with token_offset = its first token; the sum all-reduce of
the per-rank G_W must equal a single run over the whole batch, and the
per-token outputs must be the single run's rows. The same holds for the
MLP up-projection (split by tokens) and for the attention internals, split
by whole sequences because key and value noise reach later tokens of their
own sequence.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from zeroth_order_transformer_dust_b200.parallel import (allreduce_weight_grad, combine_draw_shards,
                                                         draw_shard, token_shard)


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


def test_sequence_shard_keeps_sequences_whole():
    from zeroth_order_transformer_dust_b200.parallel import sequence_shard
    for L in (1, 4, 1024):
        for n_seq in (0, 1, 3, 8, 9):
            for world in (1, 2, 3, 8):
                spans = [sequence_shard(n_seq * L, L, world, r) for r in range(world)]
                assert all(s % L == 0 and n % L == 0 for s, n in spans)
                assert sum(n for _, n in spans) == n_seq * L
                for (s0, n0), (s1, _) in zip(spans, spans[1:]):
                    assert s1 == s0 + n0
    with pytest.raises(ValueError):
        sequence_shard(10, 4, 2, 0)


class _OracleCtx:
    """CPU stand-in for a device context: the context's call signatures, the
    oracle's arithmetic, G returned as a torch tensor for the all-reduce."""

    def mlp_grad(self, X, W_up, W_down, W_head, y, *, token_offset, K, sigma, seed):
        import oracle
        prm = oracle.Params(T=X.shape[0], d=X.shape[1], V=W_head.shape[0], K=K, sigma=sigma,
                            seed=seed, token_offset=token_offset, d_ff=W_up.shape[0])
        o = oracle.mlp_grad(X, W_up, W_down, W_head, y, prm)
        return {"G": torch.from_numpy(o["G"]), "rewards": o["rewards"], "g": o["g"]}

    def attn_grad(self, X, Q, Kc, Vc, E, *, token_offset, seq_len, n_heads, which, K, sigma,
                  seed):
        import oracle
        prm = oracle.Params(T=X.shape[0], d=X.shape[1], V=1, K=K, sigma=sigma, seed=seed,
                            token_offset=token_offset)
        o = oracle.attn_grad(X, Q, Kc, Vc, E, seq_len, n_heads, which, prm)
        return {"G": torch.from_numpy(o["G"]), "rewards": o["rewards"], "g": o["g"]}


def _layer_workload(kind):
    import synth
    if kind == "mlp":
        return synth.CONFIGS["mlp_bf16"].with_(T=7, d=6, V=30, d_ff=10, K=6, sigma=0.05,
                                               seed=12, dtype="f32")
    return synth.CONFIGS["attn_k_bf16"].with_(T=12, d=5, seq_len=4, n_heads=2, head_dim=3,
                                              K=6, sigma=0.3, seed=13, dtype="f32",
                                              variant="attn_" + kind)


def _layer_worker(rank, world, port, kind, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import synth
        from zeroth_order_transformer_dust_b200.parallel import (
            sequence_shard, sharded_attn_grad, sharded_mlp_grad)
        wl = _layer_workload(kind)
        kw = dict(K=wl.K, sigma=wl.sigma, seed=wl.seed)
        if kind == "mlp":
            x = synth.make_mlp_inputs(wl)
            t0, n = token_shard(wl.T, world, rank)
            out = sharded_mlp_grad(_OracleCtx(), x["X"][t0:t0 + n], x["W_up"], x["W_down"],
                                   x["W_head"], x["targets"][t0:t0 + n], t0, **kw)
        else:
            x = synth.make_attn_inputs(wl)
            t0, n = sequence_shard(wl.T, wl.seq_len, world, rank)
            sl = slice(t0, t0 + n)
            out = sharded_attn_grad(_OracleCtx(), x["X"][sl], x["Q"][sl], x["K"][sl], x["V"][sl],
                                    x["E"][sl], t0, seq_len=wl.seq_len, n_heads=wl.n_heads,
                                    which=kind, **kw)
        q.put((rank, t0, n, out["G"].numpy(), out["rewards"], out["g"]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("kind", ["mlp", "k", "v"])
def test_sharded_layer_estimators_equal_single_run(kind):
    # the MLP up-projection split by tokens (7 tokens: 4 + 3) and the key and
    # value noise of attention split by whole sequences (3 sequences of 4:
    # 8 + 4 tokens), whose rewards reach later tokens of the same sequence
    import oracle
    import synth
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_layer_worker, args=(r, world, port, kind, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    wl = _layer_workload(kind)
    if kind == "mlp":
        x = synth.make_mlp_inputs(wl)
        prm = oracle.Params(T=wl.T, d=wl.d, V=wl.V, K=wl.K, sigma=wl.sigma, seed=wl.seed,
                            d_ff=wl.d_ff)
        ref = oracle.mlp_grad(x["X"], x["W_up"], x["W_down"], x["W_head"], x["targets"], prm)
    else:
        x = synth.make_attn_inputs(wl)
        prm = oracle.Params(T=wl.T, d=wl.d, V=1, K=wl.K, sigma=wl.sigma, seed=wl.seed)
        ref = oracle.attn_grad(x["X"], x["Q"], x["K"], x["V"], x["E"], wl.seq_len, wl.n_heads,
                               kind, prm)
    assert sorted(n for _, _, n, _, _, _ in res) == ([3, 4] if kind == "mlp" else [4, 8])
    for rank, t0, n, G, rewards, g in res:
        np.testing.assert_allclose(G, ref["G"], rtol=0, atol=1e-12)
        np.testing.assert_array_equal(rewards, ref["rewards"][t0:t0 + n])
        np.testing.assert_allclose(g, ref["g"][t0:t0 + n], rtol=0, atol=1e-13)


def _max_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        q.put((rank, bench._max_over_ranks(10.0 + 5.0 * (rank == 1) - rank * 0.25, world,
                                           device="cpu")))
    finally:
        dist.destroy_process_group()


def test_bench_times_the_slowest_rank():
    # bench.py reports the max over ranks of the per-step time
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_max_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == {0: 14.75, 1: 14.75}


def _draw_worker(rank, world, port, S, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        import synth
        wl = synth.Workload("gloo", "head", T=6, d=5, V=30, K=7, S=S, sigma=0.05, seed=4,
                            dtype="f32", targets="zipf")
        inp = synth.make_head_inputs(wl)
        i0, k = draw_shard(wl.K, world, rank)
        prm = oracle.Params(T=wl.T, d=wl.d, V=wl.V, K=k, S=wl.S, sigma=wl.sigma, seed=wl.seed,
                            draw_offset=i0)
        out = oracle.head_grad(inp["H"], inp["W"], inp["targets"], prm)
        G = torch.from_numpy(out["G"])
        g = torch.from_numpy(out["g"])
        combine_draw_shards(G, k, wl.K)
        combine_draw_shards(g, k, wl.K)
        q.put((rank, i0, k, G.numpy(), g.numpy(), out["rewards"]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("S", [0, 4])
def test_draw_sharded_estimate_equals_single_run(S):
    """Ranks with disjoint draw ranges (7 draws as 4 + 3), each over every
    token, combine to the single run's G_W and g; their rewards are the
    single run's columns."""
    import oracle
    import synth
    world = 2
    assert [draw_shard(7, world, r) for r in range(world)] == [(0, 4), (4, 3)]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_draw_worker, args=(r, world, port, S, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    wl = synth.Workload("gloo", "head", T=6, d=5, V=30, K=7, S=S, sigma=0.05, seed=4,
                        dtype="f32", targets="zipf")
    inp = synth.make_head_inputs(wl)
    prm = oracle.Params(T=wl.T, d=wl.d, V=wl.V, K=wl.K, S=wl.S, sigma=wl.sigma, seed=wl.seed)
    ref = oracle.head_grad(inp["H"], inp["W"], inp["targets"], prm)
    for rank, i0, k, G, g, rewards in res:
        np.testing.assert_allclose(G, ref["G"], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(g, ref["g"], rtol=1e-12, atol=1e-12)
        np.testing.assert_array_equal(rewards, ref["rewards"][:, i0:i0 + k])


def test_combine_draw_shards_checks_counts():
    with pytest.raises(ValueError):
        combine_draw_shards(torch.zeros(2), 5, 4)
    with pytest.raises(ValueError):
        combine_draw_shards(torch.zeros(2), 1, 0)
    x = torch.ones(3)
    assert torch.equal(combine_draw_shards(x, 2, 4), torch.full((3,), 0.5))  # one process: no reduce


def _clock_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        mine = [{"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 5},
                {"sm_mhz": 1402.5, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                 "samples": 4}][rank]
        q.put((rank, bench._merge_clocks(mine, world, device="cpu")))
    finally:
        dist.destroy_process_group()


def test_bench_clock_record_covers_every_rank():
    """The JSON line's clock record at N > 1: the lowest median SM clock and
    the union of the throttle reasons over the ranks, the same on every rank."""
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_clock_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in range(world):
        assert res[rank] == {"sm_mhz": 1402.5, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                             "samples": 5, "ranks": 2}
