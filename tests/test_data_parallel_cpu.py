"""Host logic of the batch-sharded forward on CPU ranks (gloo, world size 2 and 3).

Each rank computes its shard's row losses with the fp64 oracle (the GPU kernels are not needed
to check the sharding and the loss combination) and the ranks combine them with the same
all-reduce the GPU path uses.  The combined loss must equal the oracle's loss of the whole
batch, including when ignored targets (-1) are spread unevenly over the ranks."""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import seeded
from decoder_only_transformer_causal_b200.data_parallel import (
    allreduce_loss_terms, global_loss, shard_range)

TINY = seeded.WORKLOADS["tiny"].model_dict()


def test_shard_range_partitions():
    for batch in range(0, 13):
        for world in range(1, 6):
            spans = [shard_range(batch, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == batch
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_range(4, 2, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, batch, ignore_frac, out_path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        W = seeded.to_f64(seeded.make_weights(TINY, stress=True))
        idx, tgt = seeded.make_tokens(batch, 32, TINY["vocab_size"], ignore_frac=ignore_frac)
        # uneven ignores: rank 0's slice loses every target of its first sequence
        tgt[0] = -1
        a, b = shard_range(batch, world, rank)
        sc = torch.zeros(2, dtype=torch.float64)
        if b > a:
            out = oracle.forward(W, TINY, idx[a:b].numpy(), tgt[a:b].numpy(), keep_logits=False)
            sc[0] = float(out["row_loss"].sum())
            sc[1] = float(out["count"])
        allreduce_loss_terms(sc)
        if rank == 0:
            full = oracle.forward(W, TINY, idx.numpy(), tgt.numpy(), keep_logits=False)
            np.save(out_path, np.array([global_loss(sc), full["loss"], sc[1].item(), full["count"]]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,batch", [(2, 5), (3, 4), (2, 1)])
def test_sharded_loss_matches_full_batch(tmp_path, world, batch):
    out = tmp_path / "res.npy"
    mp.spawn(_rank_main, args=(world, _free_port(), batch, 0.2, str(out)), nprocs=world, join=True)
    got, want, n_got, n_want = np.load(out)
    assert n_got == n_want
    if math.isnan(want):
        assert math.isnan(got)
    else:
        assert abs(got - want) <= 1e-12 * abs(want)


def _grad_rank_main(rank, world, port, batch, out_path):
    """Data-parallel gradient combination on gloo ranks: each rank's oracle gradient of its shard,
    taken against the all-reduced global count (its own mean scaled by n_r / n_total, which is
    what dividing by the global count gives), SUM-all-reduced with the product's helpers, must equal
    the oracle gradient of the whole batch."""
    import oracle.backward as ob
    from decoder_only_transformer_causal_b200.data_parallel import allreduce_grads
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = dict(TINY, n_layer=1)
        W = seeded.to_f64(seeded.make_weights(cfg, stress=True))
        idx, tgt = seeded.make_tokens(batch, 16, cfg["vocab_size"], ignore_frac=0.3)
        tgt[0, :12] = -1                                    # rank 0's shard has fewer counted rows
        a, b = shard_range(batch, world, rank)
        sc = torch.zeros(2, dtype=torch.float64)
        names = sorted(W)
        flat = torch.zeros(sum(W[n].size for n in names), dtype=torch.float32)
        if b > a:
            g, _ = ob.backward(W, cfg, idx[a:b].numpy(), tgt[a:b].numpy())
            n_r = float((tgt[a:b] != -1).sum())
            sc[1] = n_r
            allreduce_loss_terms(sc)
            scale = n_r / float(sc[1])
            flat = torch.from_numpy(np.concatenate([(g[n] * scale).ravel() for n in names]).astype(np.float32))
        else:
            allreduce_loss_terms(sc)
        allreduce_grads(flat)
        if rank == 0:
            g_full, _ = ob.backward(W, cfg, idx.numpy(), tgt.numpy())
            ref = np.concatenate([g_full[n].ravel() for n in names])
            np.save(out_path, np.array([np.abs(flat.numpy() - ref).max(), np.abs(ref).max()]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,batch", [(2, 3), (3, 5)])
def test_sharded_gradients_match_full_batch(tmp_path, world, batch):
    out = tmp_path / "g.npy"
    mp.spawn(_grad_rank_main, args=(world, _free_port(), batch, str(out)), nprocs=world, join=True)
    err, scale = np.load(out)
    assert err <= 1e-6 * scale                     # fp32 transport of fp64 gradients


def test_gradient_buckets_cover_the_array_in_backward_order():
    """gpt_grad_buckets: n_layer + 1 disjoint ranges covering the flat gradient array once; bucket i
    < n_layer holds every tensor of layer n_layer - 1 - i (bucket 0 also ln_f), the last one wte and
    wpe -- the order in which the backward completes them."""
    from decoder_only_transformer_causal_b200 import native
    from decoder_only_transformer_causal_b200.native import GPTConfig
    for name in ("tiny", "gpt2"):
        cfg = GPTConfig.from_dict(seeded.WORKLOADS[name].model_dict())
        buckets = native.grad_buckets(cfg)
        L = cfg.n_layer
        assert len(buckets) == L + 1
        spans = sorted(buckets)
        assert spans[0][0] == 0 and spans[-1][1] == native.param_elems(cfg)
        assert all(spans[i][1] == spans[i + 1][0] for i in range(len(spans) - 1))
        es = 2 if cfg.dtype == "bf16" else 4
        entries, _ = native.weights_layout(cfg)
        for tname, off, numel in entries:
            a, b = off // es, off // es + numel
            if tname.startswith("h."):
                i = L - 1 - int(tname.split(".")[1])
            elif tname.startswith("ln_f"):
                i = 0
            else:
                i = L
            assert buckets[i][0] <= a and b <= buckets[i][1], (tname, i)


def _bucket_rank_main(rank, world, port, batch, out_path):
    """The bucketed reduction of the packed flat gradient array (the layout gpt_backward writes),
    with the buckets in the backward's order: equal to the whole batch's oracle gradient."""
    import oracle.backward as ob
    from decoder_only_transformer_causal_b200 import native
    from decoder_only_transformer_causal_b200.data_parallel import allreduce_grads_bucketed
    from decoder_only_transformer_causal_b200.native import GPTConfig
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfgd = dict(TINY, n_layer=2)
        cfg = GPTConfig.from_dict(cfgd)
        W = seeded.to_f64(seeded.make_weights(cfgd, stress=True))
        idx, tgt = seeded.make_tokens(batch, 16, cfgd["vocab_size"], ignore_frac=0.3)
        tgt[0, :12] = -1
        a, b = shard_range(batch, world, rank)
        entries, _ = native.weights_layout(cfg)

        def flatten(g, scale):
            flat = torch.zeros(native.param_elems(cfg), dtype=torch.float32)
            for n, off, numel in entries:
                flat[off // 4: off // 4 + numel] = torch.from_numpy((g[n] * scale).ravel().astype(np.float32))
            return flat
        sc = torch.zeros(2, dtype=torch.float64)
        flat = torch.zeros(native.param_elems(cfg), dtype=torch.float32)
        if b > a:
            g, _ = ob.backward(W, cfgd, idx[a:b].numpy(), tgt[a:b].numpy())
            n_r = float((tgt[a:b] != -1).sum())
            sc[1] = n_r
            allreduce_loss_terms(sc)
            flat = flatten(g, n_r / float(sc[1]))
        else:
            allreduce_loss_terms(sc)
        order = []
        allreduce_grads_bucketed(flat, native.grad_buckets(cfg), wait=order.append)
        if rank == 0:
            g_full, _ = ob.backward(W, cfgd, idx.numpy(), tgt.numpy())
            ref = flatten(g_full, 1.0).numpy()
            np.save(out_path, np.array([np.abs(flat.numpy() - ref).max(), np.abs(ref).max(),
                                        float(order == list(range(cfg.n_layer + 1)))]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,batch", [(2, 3), (3, 4)])
def test_bucketed_gradients_match_full_batch(tmp_path, world, batch):
    out = tmp_path / "b.npy"
    mp.spawn(_bucket_rank_main, args=(world, _free_port(), batch, str(out)), nprocs=world, join=True)
    err, scale, in_order = np.load(out)
    assert in_order == 1.0
    assert err <= 1e-6 * scale
