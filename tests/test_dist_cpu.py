"""Multi-rank host logic on CPU (world size 2, gloo): head sharding, barrier, max over ranks.

Heads are independent, so a job split over ranks needs no collective on the data path; each rank
computes its share of heads (here with the oracle, on CPU) and only the timing reduction crosses
ranks.  The shares must cover every head exactly once and reproduce the single-process result.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from gated_linear_attention_relu_b200 import dist as ldist


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shard_range_covers_every_item_once():
    for total in (0, 1, 5, 32, 33, 64):
        for world in (1, 2, 3, 8):
            seen = []
            for r in range(world):
                lo, hi = ldist.shard_range(total, r, world)
                assert 0 <= lo <= hi <= total
                seen.extend(range(lo, hi))
                assert hi - lo in (total // world, -(-total // world))
            assert seen == list(range(total))
    with pytest.raises(ValueError):
        ldist.shard_range(4, 2, 2)


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import oracle as orc
    from gated_linear_attention_relu_b200 import workloads as wl

    r, wsz = ldist.init("gloo", timeout_s=60)
    assert (r, wsz) == (rank, world)
    w = wl.custom("dist", B=2, H=3, T=2, Hh=3, W=5, d=16, bands=(4, 6, 6), dtype="f32")
    Q, K, V, G = (t.double().numpy() for t in wl.generate(w, "cpu"))
    flat = lambda x: x.reshape(w.B * w.H, w.N, w.d)
    lo, hi = ldist.shard_range(w.B * w.H, rank, world)
    pos = orc.grid_positions(w.T, w.Hh, w.W)
    outs = [orc.forward_positions(flat(Q)[u], flat(K)[u], flat(V)[u], flat(G)[u], pos, w.bands,
                                  w.rope_base, w.eps) for u in range(lo, hi)]
    np.save(os.path.join(out_dir, f"rank{rank}.npy"), np.array(outs))
    ldist.barrier()
    t = ldist.max_over_ranks(10.0 * (rank + 1))
    np.save(os.path.join(out_dir, f"max{rank}.npy"), np.array([t]))
    ldist.finalize()


def test_two_rank_gloo_sharding_matches_single_process(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    import oracle as orc
    from gated_linear_attention_relu_b200 import workloads as wl

    w = wl.custom("dist", B=2, H=3, T=2, Hh=3, W=5, d=16, bands=(4, 6, 6), dtype="f32")
    Q, K, V, G = (t.double().numpy() for t in wl.generate(w, "cpu"))
    ref = orc.forward_bidir(Q, K, V, G, (w.T, w.Hh, w.W), w.bands, w.rope_base, w.eps)
    got = np.concatenate([np.load(tmp_path / f"rank{r}.npy") for r in range(world)])
    assert got.shape == (w.B * w.H, w.N, w.d)
    assert np.array_equal(got, ref.reshape(w.B * w.H, w.N, w.d))
    for r in range(world):
        assert float(np.load(tmp_path / f"max{r}.npy")[0]) == 20.0
