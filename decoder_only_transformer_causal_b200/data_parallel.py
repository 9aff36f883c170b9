"""Batch-sharded forward over several GPUs (one process per GPU).

Sequences of a batch are independent through the whole forward pass ("nanoGPT 全局流程图", §3.2:
every sequence goes through the same Blocks on its own), so each rank runs gpt_forward on its
own contiguous slice of the batch with replicated weights; no activation crosses a device.  The
only exchange is the loss: F.cross_entropy averages over every counted position of the batch
(targets != -1), so the ranks add their {sum of row losses, number of counted rows} and divide
the totals — not the mean of per-rank means, which would weight ranks with many ignored targets
wrongly.  With NCCL over NVLink that is one 16-byte all-reduce per step.

Data-parallel training ("nanoGPT 全局流程图" 3.4-3.7; "nanoGPT 核心代码速查表" 七 per-GPU batch):
each rank runs the training forward on its shard, the {sum, count} pair is all-reduced *before*
the backward so every rank's cross-entropy gradient divides by the global count, and a SUM
all-reduce of the flat fp32 gradients then gives exactly the whole batch's gradient (also when
ignored targets are spread unevenly); every rank applies the same AdamW step.  The gradient
reduction runs per layer bucket on a second stream, each bucket as soon as the backward has
finished it (gpt_grad_buckets, gpt_backward's bucket events), overlapping the backward of the
earlier layers.
"""
from __future__ import annotations

import math

import torch
import torch.distributed as dist


def shard_range(batch: int, world: int, rank: int) -> tuple[int, int]:
    """[start, stop) of the sequences rank `rank` owns: contiguous, sizes differing by at most
    one (the first batch % world ranks take one more)."""
    if world < 1 or not 0 <= rank < world or batch < 0:
        raise ValueError((batch, world, rank))
    base, extra = divmod(batch, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def allreduce_loss_terms(loss_sum_count: torch.Tensor, group=None) -> torch.Tensor:
    """Sums the fp64 {sum of row losses, counted rows} pair over the ranks, in place."""
    if loss_sum_count.dtype != torch.float64 or loss_sum_count.numel() != 2:
        raise ValueError("loss_sum_count must be a float64 tensor of 2 elements")
    dist.all_reduce(loss_sum_count, op=dist.ReduceOp.SUM, group=group)
    return loss_sum_count


def global_loss(loss_sum_count: torch.Tensor) -> float:
    """Mean row loss of the whole batch from the reduced pair (NaN when nothing is counted)."""
    s, n = (float(v) for v in loss_sum_count.detach().cpu())
    return s / n if n > 0 else math.nan


def forward_sharded(model, idx: torch.Tensor, targets: torch.Tensor, group=None):
    """Runs this rank's slice of (idx, targets) [B, T] through `model` (a GPT instance on this
    rank's device) and returns (local logits, global loss).  idx / targets may be the full
    batch on any device; only this rank's rows are copied to the model's device."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    a, b = shard_range(idx.shape[0], world, rank)
    dev = model.device
    sc = torch.zeros(2, dtype=torch.float64, device=dev)
    logits = None
    if b > a:
        logits, _ = model(idx[a:b].to(dev), targets[a:b].to(dev), loss_sum_count=sc)
    allreduce_loss_terms(sc, group)
    return logits, global_loss(sc)


def allreduce_grads(grads: torch.Tensor, group=None) -> torch.Tensor:
    """SUM all-reduce of the flat fp32 gradient array, in place (each rank holds its share of the
    global mean after a backward against the all-reduced count)."""
    if grads.dtype != torch.float32:
        raise ValueError("grads must be float32")
    dist.all_reduce(grads, op=dist.ReduceOp.SUM, group=group)
    return grads


def allreduce_grads_bucketed(grads: torch.Tensor, buckets, wait=None, group=None) -> torch.Tensor:
    """SUM all-reduce of the flat fp32 gradient array one bucket (an element range) at a time, in
    the given order; wait(i), when given, runs before bucket i is reduced (the GPU step makes the
    communication stream wait there for the backward's event of that bucket)."""
    if grads.dtype != torch.float32:
        raise ValueError("grads must be float32")
    for i, (a, b) in enumerate(buckets):
        if wait is not None:
            wait(i)
        dist.all_reduce(grads[a:b], op=dist.ReduceOp.SUM, group=group)
    return grads


class _Overlap:
    """Per-trainer state of the overlapped reduction: the gradient buckets, one CUDA event per
    bucket (recorded by gpt_backward when the bucket is complete) and the communication stream."""

    def __init__(self, trainer):
        from . import native
        dev = trainer.model.device
        self.buckets = native.grad_buckets(trainer.model.cfg)
        self.stream = torch.cuda.Stream(dev)
        self.events = [torch.cuda.Event() for _ in self.buckets]
        main = torch.cuda.current_stream(dev)
        for e in self.events:      # the CUDA events exist from their first record on
            e.record(main)


def train_step_sharded(trainer, idx: torch.Tensor, targets: torch.Tensor, group=None,
                       overlap: bool = True) -> torch.Tensor:
    """One data-parallel training step of a Trainer on this rank's shard [B_r, T] (already on the
    rank's device): training forward, all-reduce of the loss terms, backward against the global
    count, SUM all-reduce of the gradients, AdamW.  With overlap (the default) the gradients are
    reduced per layer on a second stream while the backward of the earlier layers still runs: each
    bucket's all-reduce waits only for the event gpt_backward records when that bucket is complete,
    and the optimizer waits for all of them.  Returns the global mean loss as a device fp64 scalar
    (NaN when no row is counted), so consecutive steps queue without a host round trip."""
    from . import native
    cfg, w = trainer.model.cfg, trainer.model.weights
    B, T = idx.shape
    native.forward_train(cfg, w, idx, targets, trainer.acts, trainer.fws, loss=trainer.loss)
    lt = native.loss_terms(cfg, trainer.acts, B, T)
    allreduce_loss_terms(lt, group)
    trainer.grads.zero_()
    if not overlap:
        native.backward(cfg, w, idx, targets, trainer.acts, trainer.grads, trainer.bws)
        allreduce_grads(trainer.grads, group)
    else:
        ov = getattr(trainer, "_dp_overlap", None)
        if ov is None:
            ov = trainer._dp_overlap = _Overlap(trainer)
        main = torch.cuda.current_stream(trainer.model.device)
        native.backward(cfg, w, idx, targets, trainer.acts, trainer.grads, trainer.bws, stream=main,
                        bucket_events=ov.events)
        with torch.cuda.stream(ov.stream):
            allreduce_grads_bucketed(trainer.grads, ov.buckets, wait=lambda i: ov.stream.wait_event(ov.events[i]),
                                     group=group)
        main.wait_stream(ov.stream)
    trainer.opt.step(trainer.grads)
    return lt[0] / lt[1]

