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


def _grad_rank_main(rank, world, port, out_dir):
    import torch.distributed as dist

    import oracle
    from oracle.grad import forward_backward
    from decoder_only_transformer_nc_b200 import dp
    from workloads import SHAPES, TOKEN_SEED, make_tokens, make_weights

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    s = SHAPES["tiny"]
    w = make_weights(s)
    x, y = make_tokens(s, seed=dp.shard_seed(TOKEN_SEED, rank), batch=1, seq_len=48)
    y = y.copy()
    if rank == 1:
        y[0, ::4] = -1  # unequal counts
    cfg = oracle.OracleConfig(s.n_layer, s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.seq_len, s.vocab,
                              short_window=s.short_window)
    _, g = forward_backward(cfg, w, x, y)
    t = {"wte": torch.from_numpy(w["wte"]), "lm_head": torch.from_numpy(w["lm_head"]),
         "layers": [{k: torch.from_numpy(v) for k, v in lw.items()} for lw in w["layers"]]}
    flat, grads = dp.grad_bucket(t, device="cpu")
    grads["wte"].copy_(torch.from_numpy(g["wte"]))
    grads["lm_head"].copy_(torch.from_numpy(g["lm_head"]))
    for l, lw in enumerate(g["layers"]):
        for k, v in lw.items():
            grads["layers"][l][k].copy_(torch.from_numpy(v))
    dp.average_grads_(flat, int((y != -1).sum()))
    np.save(os.path.join(out_dir, f"g{rank}.npy"), flat.numpy())
    dist.destroy_process_group()


def test_gradient_average_matches_the_whole_batch(tmp_path):
    """Two gloo ranks, each with the oracle's gradient of its own shard's mean
    loss, average through the bucket; both must hold the gradient of the mean
    over the concatenated batch (oracle, fp64), to fp32 rounding."""
    import oracle
    from oracle.grad import forward_backward
    from decoder_only_transformer_nc_b200 import dp
    from workloads import SHAPES, TOKEN_SEED, make_tokens, make_weights

    world, port = 2, _free_port()
    mp.spawn(_grad_rank_main, args=(world, port, str(tmp_path)), nprocs=world, join=True)
    s = SHAPES["tiny"]
    w = make_weights(s)
    xs, ys = [], []
    for r in range(world):
        x, y = make_tokens(s, seed=dp.shard_seed(TOKEN_SEED, r), batch=1, seq_len=48)
        y = y.copy()
        if r == 1:
            y[0, ::4] = -1
        xs.append(x)
        ys.append(y)
    cfg = oracle.OracleConfig(s.n_layer, s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.seq_len, s.vocab,
                              short_window=s.short_window)
    _, want = forward_backward(cfg, w, np.concatenate(xs), np.concatenate(ys))
    t = {"wte": torch.from_numpy(w["wte"]), "lm_head": torch.from_numpy(w["lm_head"]),
         "layers": [{k: torch.from_numpy(v) for k, v in lw.items()} for lw in w["layers"]]}
    flat, grads = dp.grad_bucket(t, device="cpu")
    for r in range(world):
        flat.copy_(torch.from_numpy(np.load(tmp_path / f"g{r}.npy")))
        np.testing.assert_allclose(grads["wte"].numpy(), want["wte"], rtol=1e-5, atol=1e-9)
        np.testing.assert_allclose(grads["lm_head"].numpy(), want["lm_head"], rtol=1e-5, atol=1e-9)
        for l, lw in enumerate(want["layers"]):
            for k, v in lw.items():
                np.testing.assert_allclose(grads["layers"][l][k].numpy(), v, rtol=1e-4, atol=1e-9)


def test_grad_bucket_layout():
    """Every view 16-byte aligned (the library's rule for gradient pointers),
    shaped like its weight, disjoint, and the whole bucket zeroed."""
    from decoder_only_transformer_nc_b200 import dp
    from workloads import SHAPES, make_weights

    s = SHAPES["tiny"]
    w = make_weights(s)
    t = {"wte": torch.from_numpy(w["wte"]), "lm_head": torch.from_numpy(w["lm_head"]),
         "layers": [{k: torch.from_numpy(v) for k, v in lw.items()} for lw in w["layers"]]}
    flat, grads = dp.grad_bucket(t, device="cpu")
    assert "extras" not in grads
    views = [("wte", grads["wte"], t["wte"]), ("lm_head", grads["lm_head"], t["lm_head"])]
    views += [(f"{l}.{k}", grads["layers"][l][k], t["layers"][l][k]) for l in range(s.n_layer) for k in dp.NAMES]
    _check_views(flat, views)


def test_grad_bucket_layout_with_extras():
    """The further terms' gradients join the bucket; a per-layer list keeps its
    None entries (layers without a value embedding)."""
    from decoder_only_transformer_nc_b200 import dp
    from workloads import SHAPES, make_extras, make_weights

    s = SHAPES["tiny"]
    w = make_weights(s)
    ex = make_extras(s, layers=[1])
    T = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    t = {"wte": T(w["wte"]), "lm_head": T(w["lm_head"]),
         "layers": [{k: T(v) for k, v in lw.items()} for lw in w["layers"]],
         "extras": {"smear_gate": T(ex["smear_gate"]), "resid_lambdas": T(ex["resid_lambdas"]),
                    "x0_lambdas": T(ex["x0_lambdas"]), "backout_lambda": T(np.reshape(ex["backout_lambda"], 1)),
                    "value_embeds": [None, T(ex["value_embeds"][1])], "ve_gates": [None, T(ex["ve_gates"][1])]}}
    flat, grads = dp.grad_bucket(t, device="cpu")
    ge, te = grads["extras"], t["extras"]
    assert ge["value_embeds"][0] is None and ge["ve_gates"][0] is None
    views = [("wte", grads["wte"], t["wte"]), ("lm_head", grads["lm_head"], t["lm_head"])]
    views += [(f"{l}.{k}", grads["layers"][l][k], t["layers"][l][k]) for l in range(s.n_layer) for k in dp.NAMES]
    views += [(k, ge[k], te[k]) for k in ("smear_gate", "resid_lambdas", "x0_lambdas", "backout_lambda")]
    views += [(f"{k}[1]", ge[k][1], te[k][1]) for k in ("value_embeds", "ve_gates")]
    _check_views(flat, views)


def _check_views(flat, views):
    spans = []
    for name, g, ref in views:
        assert g.shape == ref.shape and g.dtype == torch.float32, name
        assert g.data_ptr() % 16 == 0, name
        off = (g.data_ptr() - flat.data_ptr()) // 4
        spans.append((off, off + g.numel()))
    spans.sort()
    assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))
    assert spans[-1][1] <= flat.numel() - 4 and not flat.any()


def test_average_with_no_counted_targets_anywhere(tmp_path):
    """A world whose ranks count no targets keeps zero gradients (no division by zero)."""
    world, port = 1, _free_port()
    import torch.distributed as dist
    from decoder_only_transformer_nc_b200 import dp
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=0, world_size=world)
    try:
        flat = torch.zeros(16 + 4)
        flat[:16] = 3.0
        dp.average_grads_(flat, 0)
        assert torch.isfinite(flat).all() and not flat[:16].any()
    finally:
        dist.destroy_process_group()


def _tensors_with_extras(with_extras):
    from workloads import SHAPES, make_extras, make_weights
    s = SHAPES["tiny"]
    w = make_weights(s)
    T = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    t = {"wte": T(w["wte"]), "lm_head": T(w["lm_head"]),
         "layers": [{k: T(v) for k, v in lw.items()} for lw in w["layers"]]}
    if with_extras:
        ex = make_extras(s, layers=[1])
        t["extras"] = {"smear_gate": T(ex["smear_gate"]), "resid_lambdas": T(ex["resid_lambdas"]),
                       "x0_lambdas": T(ex["x0_lambdas"]),
                       "backout_lambda": T(np.reshape(ex["backout_lambda"], 1)),
                       "value_embeds": [None, T(ex["value_embeds"][1])], "ve_gates": [None, T(ex["ve_gates"][1])]}
    return t


@pytest.mark.parametrize("with_extras", [False, True])
def test_bucket_slices_cover_the_bucket_once_in_backward_order(with_extras):
    """The pieces of the overlapped gradient average: every float of the bucket
    in exactly one piece; each layer's piece holds exactly its six gradients;
    the order is the backward's (lm_head, layers L-1 .. 0, wte, the tail with
    the count slot)."""
    from decoder_only_transformer_nc_b200 import dp
    t = _tensors_with_extras(with_extras)
    flat, grads = dp.grad_bucket(t, device="cpu")
    sl = dp.bucket_slices(t)
    L = len(t["layers"])
    assert [n for n, _, _ in sl] == ["lm_head"] + [f"layer {l}" for l in reversed(range(L))] + ["wte", "tail"]
    cover = np.zeros(flat.numel(), dtype=int)
    for _, a, b in sl:
        assert 0 <= a <= b <= flat.numel()
        cover[a:b] += 1
    assert (cover == 1).all()
    base = flat.data_ptr()
    off = lambda v: (v.data_ptr() - base) // 4
    for name, a, b in sl:
        if name.startswith("layer"):
            l = int(name.split()[1])
            views = [grads["layers"][l][k] for k in dp.NAMES]
            assert min(off(v) for v in views) == a and max(off(v) + v.numel() for v in views) <= b
            assert b - a - sum(v.numel() for v in views) < 4 * len(views)  # padding only
    assert sl[-1][2] == flat.numel()
    if with_extras:
        ge = grads["extras"]
        for v in [ge["smear_gate"], ge["resid_lambdas"], ge["x0_lambdas"], ge["backout_lambda"],
                  ge["value_embeds"][1], ge["ve_gates"][1]]:
            assert sl[-1][1] <= off(v) and off(v) + v.numel() <= flat.numel() - 4


def _backward_kinds(L, extras_untraced=True):
    """The kinds of one traced training step, in the library's launch order."""
    fwd = ["rope_table", "cast", "embedding"]
    for _ in range(L):
        fwd += ["copy", "rmsnorm", "gemm_qkv", "attention", "gemm_attn_proj", "copy", "rmsnorm", "gemm_fc",
                "gemm_mlp_proj"]
    fwd += ["rmsnorm", "gemm_lm_head", "ce_finalize", "loss_mean"]
    bwd = ["ce_bwd", "gemm_wgrad", "gemm_dgrad", "norm_bwd"]
    for _ in range(L):
        bwd += ["gemm_wgrad", "gemm_dgrad", "rmsnorm", "gemm_wgrad", "gemm_dgrad", "norm_bwd", "gemm_wgrad",
                "gemm_dgrad", "attn_bwd", "qk_bwd", "rmsnorm", "gemm_wgrad", "emb_bwd", "gemm_dgrad", "norm_bwd"]
    bwd += ["emb_bwd"]
    return fwd + bwd


def test_backward_finish_entries_follow_the_trace():
    from decoder_only_transformer_nc_b200 import dp
    L = 3
    kinds = _backward_kinds(L)
    e = dp.backward_finish_entries(kinds, L)
    assert len(e) == 1 + L + 2
    assert kinds[e[0]] == "gemm_wgrad" and kinds[e[0] - 1] == "ce_bwd"  # lm_head's weight gradient
    assert all(kinds[i] == "emb_bwd" for i in e[1:])
    assert e[1:L + 1] == sorted(e[1:L + 1]) and e[L + 1] == e[L + 2] == len(kinds) - 1
    # a layer finishes after all of its own weight-gradient products
    for k in range(L):
        prev = e[k]  # lm_head or the layer above
        assert kinds[prev + 1:e[k + 1]].count("gemm_wgrad") == 4
    with pytest.raises(ValueError):
        dp.backward_finish_entries(kinds[:-1], L)
    with pytest.raises(ValueError):
        dp.backward_finish_entries([k for k in kinds if k != "ce_bwd"], L)


def _sliced_rank_main(rank, world, port, out_dir, with_extras):
    import torch.distributed as dist
    from decoder_only_transformer_nc_b200 import dp
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    t = _tensors_with_extras(with_extras)
    flat, _ = dp.grad_bucket(t, device="cpu")
    g = torch.Generator().manual_seed(100 + rank)
    flat[:-4] = torch.randn(flat.numel() - 4, generator=g)
    count = [37.0, 11.0][rank]
    whole = flat.clone()
    dp.average_grads_(whole, count)
    order = []
    sliced = flat.clone()
    dp.average_grads_sliced_(sliced, dp.bucket_slices(t), count, before=order.append)
    np.save(os.path.join(out_dir, f"sliced{rank}.npy"),
            np.stack([whole.numpy(), sliced.numpy()]).astype(np.float64))
    np.save(os.path.join(out_dir, f"order{rank}.npy"), np.array(order))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("with_extras", [False, True])
def test_sliced_average_equals_the_whole_bucket_average(tmp_path, with_extras):
    """Two gloo ranks with unequal target counts: the per-piece average of the
    overlapped schedule gives the same bucket (gradients and count slot) as the
    one all-reduce of the whole bucket, on both ranks."""
    world = 2
    mp.start_processes(_sliced_rank_main, args=(world, _free_port(), str(tmp_path), with_extras), nprocs=world,
                       join=True, start_method="spawn")
    r = [np.load(tmp_path / f"sliced{i}.npy") for i in range(world)]
    for i in range(world):
        whole, sliced = r[i]
        np.testing.assert_allclose(sliced, whole, rtol=1e-6, atol=1e-7)
        assert whole[-4] == 48.0
        np.testing.assert_array_equal(np.load(tmp_path / f"order{i}.npy"), np.arange(len(np.load(
            tmp_path / f"order{i}.npy"))))
    np.testing.assert_array_equal(r[0][1], r[1][1])
