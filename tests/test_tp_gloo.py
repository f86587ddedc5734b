"""Tensor parallelism over I on CPU: two gloo ranks each take their slice of
the experts (fp4_block_scaled_route_b200.tp.shard_weights), compute their
partial layer result with the oracle standing in for the GPU, and sum the
partials with the product's all-reduce helper.  The sum must equal the whole
layer up to fp32 summation order, for every weight format."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

CASES = [dict(wfmt=0, n_shared=1), dict(wfmt=2, n_shared=0), dict(wfmt=3, n_shared=1), dict(wfmt=1, n_shared=0),
         dict(wfmt=4, n_shared=1)]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer(case):
    from fp4_block_scaled_route_b200 import synth
    cfg = dict(T=5, H=256, I=256, E=4, k=2, routing="uniform", **case)
    return synth.make_layer(cfg, 91 + case["wfmt"])


def _oracle(L, w13, s13, w2, s2, I, g13=None, g2=None):
    import oracle
    from fp4_block_scaled_route_b200 import synth
    kw = dict(g13=g13.numpy(), g2=g2.numpy()) if g13 is not None else {}
    return oracle.forward(synth.bf16_bits(L.x), L.ids.numpy(), L.topk_w.numpy(), w13.numpy(), s13.numpy(),
                          w2.numpy(), s2.numpy(), H=L.H, I=I, E=L.E, wfmt=L.wfmt, n_shared=L.n_shared,
                          **kw)["out_f32"]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    from fp4_block_scaled_route_b200 import tp
    for ci, case in enumerate(CASES):
        L = _layer(case)
        sh = tp.shard_weights(L.w13, L.s13, L.w2, L.s2, L.wfmt, L.I, rank, world, L.g13, L.g2)
        part = torch.from_numpy(_oracle(L, sh["w13"], sh["s13"], sh["w2"], sh["s2"], L.I // world,
                                        sh.get("g13"), sh.get("g2")).copy())
        tp.allreduce_partial(part)
        out[(rank, ci)] = part.numpy()
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_sum_to_the_whole_layer():
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    for ci, case in enumerate(CASES):
        L = _layer(case)
        full = _oracle(L, L.w13, L.s13, L.w2, L.s2, L.I, L.g13, L.g2)
        for rank in (0, 1):
            got = out[(rank, ci)]
            assert np.abs(got - full).max() <= 2e-5 * np.abs(full).max(), (case, rank)
        assert np.array_equal(out[(0, ci)], out[(1, ci)])  # every rank holds the same sum


@pytest.mark.parametrize("wfmt", [0, 1, 2, 3, 4])
def test_shards_reassemble_the_weights(wfmt):
    from fp4_block_scaled_route_b200 import tp
    L = _layer(dict(wfmt=wfmt, n_shared=0))
    G = 2
    sh = [tp.shard_weights(L.w13, L.s13, L.w2, L.s2, wfmt, L.I, r, G, L.g13, L.g2) for r in range(G)]
    half = lambda t: t.shape[1] // 2
    gate = torch.cat([s["w13"][:, :half(s["w13"])] for s in sh], 1)
    up = torch.cat([s["w13"][:, half(s["w13"]):] for s in sh], 1)
    assert torch.equal(torch.cat([gate, up], 1), L.w13)
    sgate = torch.cat([s["s13"][:, :half(s["s13"])] for s in sh], 1)
    sup = torch.cat([s["s13"][:, half(s["s13"]):] for s in sh], 1)
    assert torch.equal(torch.cat([sgate, sup], 1), L.s13)
    assert torch.equal(torch.cat([s["w2"] for s in sh], 2), L.w2)
    assert torch.equal(torch.cat([s["s2"] for s in sh], 2), L.s2)
    with pytest.raises(ValueError):
        tp.shard_weights(L.w13, L.s13, L.w2, L.s2, wfmt, L.I, 0, 4)  # I/G = 64: not a multiple of 128
