"""The data-parallel host path on CPU: two gloo ranks, each scoring its own
shard of the tiny workload with the fp64 oracle, combine their losses with the
same all-reduce the bench uses; the result must equal the mean over the
concatenated shards."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist

    import oracle
    from decoder_only_transformer_nc_b200 import dp
    from workloads import SHAPES, TOKEN_SEED, make_tokens, make_weights

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    s = SHAPES["tiny"]
    w = make_weights(s)
    x, y = make_tokens(s, seed=dp.shard_seed(TOKEN_SEED, rank), batch=1, seq_len=64)
    y = y.copy()
    if rank == 1:
        y[0, ::3] = -1  # unequal valid counts across ranks
    cfg = oracle.OracleConfig(s.n_layer, s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.seq_len,
                              s.vocab, short_window=s.short_window)
    res = oracle.forward(cfg, w, x, y, want_logits=False)
    count = int((y != -1).sum())
    g = dp.global_mean_loss(torch.tensor(res["loss"], dtype=torch.float64), count)
    np.save(os.path.join(out_dir, f"rank{rank}.npy"),
            np.array([g.item(), res["token_loss"].sum(), count], dtype=np.float64))
    dist.barrier()
    dist.destroy_process_group()


def test_global_loss_over_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    r = [np.load(tmp_path / f"rank{i}.npy") for i in range(world)]
    want = (r[0][1] + r[1][1]) / (r[0][2] + r[1][2])
    for i in range(world):
        assert abs(r[i][0] - want) <= 1e-12 * abs(want)
    assert r[0][2] != r[1][2]
