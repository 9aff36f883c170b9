"""The data-parallel training step (train_step_sharded) on one GPU.

"nanoGPT 全局流程图" 3.4-3.7: the loss of a batch is the mean over every counted position, so a
data-parallel step adds the ranks' {sum of row losses, counted rows} before the backward and the
cross-entropy gradient of every rank divides by the global count.  With a single-rank process
group the step must equal the plain single-GPU step bit for bit, and the backward must read the
count through the loss-terms view that the all-reduce updates in place: doubling that count
between the forward and the backward halves every gradient."""
import socket

import pytest
import torch
import torch.distributed as dist

import seeded
from gpu_helpers import needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]


def _trainer(B, T):
    from decoder_only_transformer_causal_b200 import GPT, GPTConfig, Trainer
    cfgd = dict(seeded.WORKLOADS["gpt2"].model_dict(), n_layer=2)
    W = seeded.make_weights(cfgd, stress=True)
    model = GPT(GPTConfig.from_dict(cfgd), W)
    return Trainer(model, W, B, T, learning_rate=1e-3, warmup_iters=1, lr_decay_iters=10, min_lr=1e-4)


def _tokens(B, T):
    idx, tgt = seeded.make_tokens(B, T, 50257, seed=561, ignore_frac=0.1)
    return idx.cuda(), tgt.cuda()


@pytest.fixture
def single_rank_group():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device("cuda", 0))
    try:
        yield
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("overlap", [True, False])
def test_sharded_step_equals_single_gpu_step(single_rank_group, overlap):
    """With overlap, the gradient buckets are reduced on a second stream as gpt_backward's events
    fire; the result must not depend on it."""
    from decoder_only_transformer_causal_b200.data_parallel import train_step_sharded
    B, T = 2, 128
    idx, tgt = _tokens(B, T)
    a, b = _trainer(B, T), _trainer(B, T)
    for _ in range(2):
        la = a.step(idx, tgt)
        lb = train_step_sharded(b, idx, tgt, overlap=overlap)
        torch.cuda.synchronize()
        assert torch.equal(a.loss, b.loss)
        assert abs(float(lb) - float(la)) <= 1e-6 * abs(float(la))
        assert torch.equal(a.grads, b.grads)
        assert torch.equal(a.opt.params, b.opt.params)
        assert torch.equal(a.model.weights, b.model.weights)


def test_backward_divides_by_the_reduced_count(monkeypatch):
    """A stand-in all-reduce that doubles the count (as if a second rank had counted as many rows
    and contributed zero loss) must halve every gradient of the step."""
    from decoder_only_transformer_causal_b200 import data_parallel, native
    B, T = 2, 128
    idx, tgt = _tokens(B, T)
    ref = _trainer(B, T)
    cfg, w = ref.model.cfg, ref.model.weights
    native.forward_train(cfg, w, idx, tgt, ref.acts, ref.fws, loss=ref.loss)
    ref.grads.zero_()
    native.backward(cfg, w, idx, tgt, ref.acts, ref.grads, ref.bws)

    def fake_all_reduce(t, op=None, group=None):
        if t.dtype == torch.float64 and t.numel() == 2:
            t[1] *= 2            # in place, exactly as the real collective writes its result

    monkeypatch.setattr(data_parallel.dist, "all_reduce", fake_all_reduce)
    tr = _trainer(B, T)
    data_parallel.train_step_sharded(tr, idx, tgt)
    torch.cuda.synchronize()
    assert float(ref.grads.abs().max()) > 0
    assert torch.equal(tr.grads, ref.grads * 0.5)
