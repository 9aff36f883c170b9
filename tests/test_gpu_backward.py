"""The training step through the C ABI: gpt_forward_train's loss and gpt_backward's gradients of
every parameter against the fp64 gradient oracle (oracle/backward.py), and a few optimizer steps
that must lower the loss of a fixed batch."""
import math

import numpy as np
import pytest
import torch

import oracle
import oracle.backward as ob
import seeded
from gpu_helpers import f64, needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]


def run_grads(cfgd, W, idx, tgt, gelu="erf"):
    from decoder_only_transformer_causal_b200 import GPT, native
    from decoder_only_transformer_causal_b200.native import GPTConfig
    cfg = GPTConfig.from_dict(dict(cfgd, gelu=gelu))
    m = GPT(cfg, W)
    B, T = idx.shape
    acts, fws, bws = native.train_buffers(cfg, B, T)
    loss = native.forward_train(cfg, m.weights, idx.cuda(), tgt.cuda(), acts, fws, sync_check=True)
    grads = torch.zeros(native.param_elems(cfg), device="cuda")
    native.backward(cfg, m.weights, idx.cuda(), tgt.cuda(), acts, grads, bws, sync_check=True)
    shapes = {n: tuple(t.shape) for n, t in W.items()}
    g = {n: f64(t) for n, t in native.unflatten(cfg, grads, shapes).items()}
    # determinism: a second backward into a fresh array is bit-identical
    grads2 = torch.zeros_like(grads)
    native.backward(cfg, m.weights, idx.cuda(), tgt.cuda(), acts, grads2, bws, sync_check=True)
    assert torch.equal(grads, grads2)
    return float(loss), g


def rel_fro(got, want):
    return float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30))


@pytest.mark.parametrize("gelu,bias", [("erf", True), ("tanh", True), ("erf", False)])
def test_tiny_fp32_gradients(gelu, bias):
    cfgd = dict(seeded.WORKLOADS["tiny"].model_dict(), n_layer=2, bias=bias)
    W = seeded.make_weights(cfgd, stress=True)
    idx, tgt = seeded.make_tokens(3, 37, cfgd["vocab_size"], seed=555, ignore_frac=0.2)
    loss, g = run_grads(cfgd, W, idx, tgt, gelu)
    W64 = seeded.to_f64(W)
    ref, rloss = ob.backward(W64, cfgd, idx.numpy(), tgt.numpy(), gelu)
    assert abs(loss - rloss) <= 1e-5 * abs(rloss)
    for n in ref:
        err = rel_fro(g[n], ref[n])
        assert err <= 1e-4, (n, err)


@pytest.mark.parametrize("gelu,B,T", [("erf", 2, 64), ("tanh", 2, 64), ("erf", 1, 40)])
def test_gpt2_shape_bf16_gradients(gelu, B, T):
    """2-layer stress model of the GPT-2 124M shape (C 768, 12 heads, V 50304), both GELU forms (the
    training forward stores GELU's derivative and the bf16 backward multiplies it into the c_proj
    product's epilogue); B 1 x T 40 (40 rows, not a multiple of 32) takes the forward's fallback
    that stores the pre-activation and converts it in place.
    Gradients pass through bf16 storage at about ten points (logits, dlogits, activations, the
    products' inputs, dq/dk/dv), each rounding 2^-9 relative; added in quadrature they leave
    ~1e-2 relative (Frobenius) per tensor.  Bound: 3e-2, and 0.9995 cosine similarity."""
    cfgd = dict(seeded.WORKLOADS["gpt2"].model_dict(), n_layer=2)
    W = seeded.make_weights(cfgd, stress=True)
    idx, tgt = seeded.make_tokens(B, T, 50257, seed=556, ignore_frac=0.1)
    loss, g = run_grads(cfgd, W, idx, tgt, gelu)
    W64 = seeded.to_f64(W)
    ref, rloss = ob.backward(W64, cfgd, idx.numpy(), tgt.numpy(), gelu)
    assert abs(loss - rloss) <= 1e-3 * abs(rloss)
    worst = {}
    for n in ref:
        a, b = g[n].ravel(), ref[n].ravel()
        worst[n] = rel_fro(a, b)
        cos = float(a @ b / max(np.linalg.norm(a) * np.linalg.norm(b), 1e-30))
        assert worst[n] <= 3e-2 and cos >= 0.9995, (n, worst[n], cos)
        # element-wise: no single entry (one row of wte, one column of a bias) may be off by more
        # than the same 3e-2 of the tensor's largest gradient
        elem = float(np.max(np.abs(a - b))) / max(float(np.max(np.abs(b))), 1e-30)
        assert elem <= 3e-2, (n, elem)


def test_training_steps_lower_the_loss():
    from decoder_only_transformer_causal_b200 import GPT, Trainer
    from decoder_only_transformer_causal_b200.native import GPTConfig
    cfgd = seeded.WORKLOADS["tiny"].model_dict()
    W = seeded.make_weights(cfgd)
    model = GPT(GPTConfig.from_dict(cfgd), W)
    idx, tgt = seeded.make_tokens(4, 64, cfgd["vocab_size"], seed=557)
    tr = Trainer(model, W, 4, 64, learning_rate=3e-3, warmup_iters=2, lr_decay_iters=100, min_lr=3e-4)
    losses = [float(tr.step(idx.cuda(), tgt.cuda())) for _ in range(12)]
    assert all(math.isfinite(x) for x in losses)
    assert losses[-1] < losses[0] - 0.3, losses
    # the model's packed weights now give the trained loss in the plain forward
    logits, loss = model(idx.cuda(), tgt.cuda())
    assert float(loss) < losses[0]


def test_accumulated_micro_batches_equal_the_full_batch():
    """The page's accumulation (loss / K per micro-batch, gradients summed) equals the full batch's
    mean gradient when the micro-batches count the same number of rows (no ignored targets)."""
    from decoder_only_transformer_causal_b200 import GPT, native
    from decoder_only_transformer_causal_b200.native import GPTConfig
    cfgd = dict(seeded.WORKLOADS["tiny"].model_dict(), n_layer=2)
    W = seeded.make_weights(cfgd, stress=True)
    cfg = GPTConfig.from_dict(cfgd)
    m = GPT(cfg, W)
    idx, tgt = seeded.make_tokens(4, 32, cfgd["vocab_size"], seed=558)
    idx, tgt = idx.cuda(), tgt.cuda()
    full = torch.zeros(native.param_elems(cfg), device="cuda")
    acts, fws, bws = native.train_buffers(cfg, 4, 32)
    native.forward_train(cfg, m.weights, idx, tgt, acts, fws)
    native.backward(cfg, m.weights, idx, tgt, acts, full, bws)
    acc = torch.zeros_like(full)
    acts2, fws2, bws2 = native.train_buffers(cfg, 2, 32)
    for k in range(2):
        sl = slice(2 * k, 2 * k + 2)
        native.forward_train(cfg, m.weights, idx[sl].contiguous(), tgt[sl].contiguous(), acts2, fws2)
        native.backward(cfg, m.weights, idx[sl].contiguous(), tgt[sl].contiguous(), acts2, acc, bws2, loss_scale=0.5)
    torch.cuda.synchronize()
    err = float((acc - full).abs().max()) / float(full.abs().max())
    assert err <= 1e-5, err
