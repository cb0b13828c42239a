"""The expert-parallel exchange on CPU ranks (gloo, world size 2 and 3): each
rank holds its own tokens, marks the experts it does not hold remote
(ep_slot_table), all-gathers x, computes its partial over its experts (here the
oracle stands in for moe_forward_partial, with remote experts as missing
slots), sums the partials across ranks and finishes its own rows.  The result
on every rank must be the single-process layer on all tokens: the gather order,
the owner map, the chunking of the gathered rows and the row slicing of the
reduction are what is under test."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer_inputs(G):
    import moe_synth as S
    cfg = S.config("tiny", E=12, top_k=3, H=64, I=32, T=4 * G, seed=61)
    x = S.gen_x(cfg)
    return cfg, cfg.desc(), S.gen_arena_host(cfg), S.gen_slot_table(cfg), S.gen_router(cfg, 0), S.gen_bias(cfg, 0), x


def _worker(rank, world, port, max_chunk, out):
    import datetime
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle as O
        from quantized_expert_ffn_top10_b200.ep import ep_slot_table, moe_forward_ep
        cfg, desc, arena, table, W, b, x = _layer_inputs(world)
        T = x.shape[0] // world
        mine = x[rank * T:(rank + 1) * T]
        tab = ep_slot_table(torch.from_numpy(table), cfg.L, cfg.E, rank, world).numpy()
        held = set(int(e) for e in range(cfg.E) if tab[e] >= 0)
        assert held == {e for e in range(cfg.E) if e % world == rank}

        chunks = []

        def partial_fn(x_chunk, partial):
            chunks.append(x_chunk.shape[0])
            xb = x_chunk.numpy().view(np.uint16)
            miss = np.where(tab < 0, -1, tab).astype(np.int32)  # remote experts: absent here
            ref = O.moe_layer(desc, arena, miss, cfg.L, 0, xb, W, b, cfg.top_k, residual=False)
            partial.copy_(torch.from_numpy(ref["out_f64"].astype(np.float32)))

        def finish_fn(xr, total, o):
            r = (xr.numpy().view(np.uint16).astype(np.uint32) << 16).view(np.float32) + total.numpy()
            o.copy_(torch.from_numpy(r))

        xt = torch.from_numpy(mine.view(np.int16).copy())
        res = torch.zeros((T, cfg.H), dtype=torch.float32)
        moe_forward_ep(desc, None, None, cfg.L, 0, xt, None, None, cfg.top_k, True, res,
                       partial_fn=partial_fn, finish_fn=finish_fn, max_chunk=max_chunk)
        out[rank] = res.numpy()
        out[(rank, "chunks")] = chunks
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,max_chunk", [(2, 8192), (3, 8192), (3, 5)])
def test_gloo_ranks_reassemble_the_layer(world, max_chunk):
    import oracle as O
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, max_chunk, out), nprocs=world, join=True)
        res = dict(out)
    cfg, desc, arena, table, W, b, x = _layer_inputs(world)
    ref = O.moe_layer(desc, arena, table, cfg.L, 0, x, W, b, cfg.top_k, residual=True)["out_f64"]
    T = x.shape[0] // world
    want_chunks = [min(max_chunk, world * T - c) for c in range(0, world * T, max_chunk)]
    for rank in range(world):
        assert res[(rank, "chunks")] == want_chunks
        got = res[rank]
        want = ref[rank * T:(rank + 1) * T]
        assert got.shape == want.shape
        assert np.allclose(got, want, rtol=1e-5, atol=1e-6), np.max(np.abs(got - want))


def test_slot_table_marks_every_expert_on_exactly_one_rank():
    import torch
    from quantized_expert_ffn_top10_b200 import MOE_SLOT_REMOTE
    from quantized_expert_ffn_top10_b200.ep import ep_slot_table
    L, E, G = 3, 10, 4
    table = torch.arange(L * E, dtype=torch.int32)
    held = np.zeros((L, E), int)
    for r in range(G):
        t = ep_slot_table(table, L, E, r, G).view(L, E).numpy()
        own = t != MOE_SLOT_REMOTE
        assert np.array_equal(t[own], table.view(L, E).numpy()[own])
        assert np.all(own[:, r::G]) and own.sum() == L * len(range(r, E, G))
        held += own
    assert np.all(held == 1)
