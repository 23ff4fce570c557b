"""Multi-rank path on CPU: two gloo ranks (spawned processes) each take their
block of shots, compute the shot-summed gradient of their block with the
oracle, sum it over ranks through the shard module and take the maximum of a
per-rank time; the result must equal the single-process gradient over all
shots."""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from adjoint_state_gradients_b200 import shard


def test_shot_blocks_cover_every_shot_once():
    for n in (0, 1, 7, 8, 9, 256):
        for world in (1, 2, 3, 8):
            seen = []
            for r in range(world):
                lo, hi = shard.shot_block(n, r, world)
                assert 0 <= lo <= hi <= n
                assert hi - lo in (n // world, n // world + 1)
                seen.extend(range(lo, hi))
            assert seen == list(range(n))
    with pytest.raises(ValueError):
        shard.shot_block(8, 2, 2)


def _case():
    from tests._cases import small_sim
    from adjoint_state_gradients_b200 import synth
    sim, dt, _ = small_sim(4242, 36, 44, 5, 1, 6, 4, 5, round_f32=True)
    g = synth.rng(42)
    nt = 30
    f = g.normal(size=(nt, 5, 1))
    res = g.normal(size=(nt, 5, 6))
    return sim, f, res


def _rank_main(rank, world, port, out_path):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        sim, f, res = _case()
        lo, hi = shard.shot_block(sim.n_shots, rank, world)
        sub = oracle.Sim(ny=sim.ny, nx=sim.nx, order=sim.order, dy=sim.dy, dx=sim.dx, ca=sim.ca,
                         cb=sim.cb, cq=float(sim.cq[0]), prof_y=sim.prof_y, prof_x=sim.prof_x,
                         src_idx=sim.src_idx[lo:hi], rec_idx=sim.rec_idx[lo:hi])
        ck = sub.fwd_adj_ckpt(f[:, lo:hi], res[:, lo:hi], 8)
        gca = torch.tensor(ck["gca"].sum(axis=0))
        gcb = torch.tensor(ck["gcb"].sum(axis=0))
        shard.sum_over_ranks_(gca, gcb)
        t = shard.max_over_ranks(10.0 + rank)
        if rank == 0:
            np.savez(out_path, gca=gca.numpy(), gcb=gcb.numpy(), t=t)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_sum_gradients_over_shot_blocks(tmp_path):
    import oracle
    out = str(tmp_path / "rank0.npz")
    mp.start_processes(_rank_main, args=(2, _free_port(), out), nprocs=2, join=True,
                       start_method="spawn")
    got = np.load(out)
    sim, f, res = _case()
    ck = sim.fwd_adj_ckpt(f, res, 8)
    want_ca = oracle.combine(ck["gca"])
    want_cb = oracle.combine(ck["gcb"])
    assert np.allclose(got["gca"], want_ca, rtol=1e-12, atol=1e-12 * np.abs(want_ca).max())
    assert np.allclose(got["gcb"], want_cb, rtol=1e-12, atol=1e-12 * np.abs(want_cb).max())
    assert float(got["t"]) == 11.0
