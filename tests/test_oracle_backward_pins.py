"""Pins of the gradient oracle (oracle/backward.py) against facts that do not come from it.

* Central finite differences of oracle.forward's loss (fp64, h = 1e-5) at sampled entries of
  every parameter tensor of a tiny stress model (biases, LayerNorm and both GELU forms).
* torch fp64 autograd of the independent library composition of the forward (F.embedding,
  F.layer_norm, F.scaled_dot_product_attention with is_causal, F.gelu, F.cross_entropy with
  ignore_index): every gradient tensor.
* Closed-form invariants: each counted row of d(loss)/d(logits) sums to 0, its entry at the
  target is -(1 - p_target)/n, and the rows of ignored targets are 0; LayerNorm's input gradient
  sums to 0 over each row.

Planted mistakes in the oracle must each fail a pin.
"""
from contextlib import contextmanager

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import oracle.backward as ob
import seeded

TINY = seeded.WORKLOADS["tiny"].model_dict()
RNG = np.random.default_rng(20240604)


def tiny_case(n_layer=2, B=2, T=9, ignore_frac=0.25, bias=True):
    cfg = dict(TINY, n_layer=n_layer, bias=bias)
    W = seeded.to_f64(seeded.make_weights(cfg, stress=True))
    idx, tgt = seeded.make_tokens(B, T, cfg["vocab_size"], seed=31337, ignore_frac=ignore_frac)
    return cfg, W, idx.numpy(), tgt.numpy()


def loss_of(W, cfg, idx, tgt, gelu_mode):
    return oracle.forward(W, cfg, idx, tgt, gelu_mode=gelu_mode, keep_logits=False)["loss"]


def pin_finite_differences(o=ob):
    for gelu_mode, bias in (("erf", True), ("tanh", True), ("erf", False)):
        cfg, W, idx, tgt = tiny_case(bias=bias)
        g, loss = o.backward(W, cfg, idx, tgt, gelu_mode)
        assert loss == pytest.approx(loss_of(W, cfg, idx, tgt, gelu_mode), rel=1e-14)
        assert set(g) == set(W)
        h = 1e-5
        for name in sorted(W):
            flat = W[name].reshape(-1)
            picks = RNG.choice(flat.size, size=min(4, flat.size), replace=False)
            if name == "wte":  # rows that occur in idx (embedding + head) and rows that do not
                picks = np.concatenate([picks, [int(idx[0, 0]) * W[name].shape[1] + 3]])
            for i in picks:
                old = flat[i]
                flat[i] = old + h
                lp = loss_of(W, cfg, idx, tgt, gelu_mode)
                flat[i] = old - h
                lm = loss_of(W, cfg, idx, tgt, gelu_mode)
                flat[i] = old
                fd = (lp - lm) / (2 * h)
                an = g[name].reshape(-1)[i]
                assert abs(an - fd) <= 1e-7 + 1e-5 * abs(fd), (gelu_mode, bias, name, int(i), an, fd)


def torch_grads(W, cfg, idx, tgt, gelu_mode):
    Wt = {k: torch.tensor(v, requires_grad=True) for k, v in W.items()}
    idx_t = torch.from_numpy(np.asarray(idx))
    B, S = idx_t.shape
    C, nh = cfg["n_embd"], cfg["n_head"]
    x = F.embedding(idx_t, Wt["wte"]) + F.embedding(torch.arange(S), Wt["wpe"])
    appr = "tanh" if gelu_mode == "tanh" else "none"
    for l in range(cfg["n_layer"]):
        p = f"h.{l}."
        u = F.layer_norm(x, (C,), Wt[p + "ln_1.weight"], Wt.get(p + "ln_1.bias"), 1e-5)
        qkv = F.linear(u, Wt[p + "attn.c_attn.weight"], Wt.get(p + "attn.c_attn.bias"))
        q, k, v = qkv.split(C, dim=2)
        sh = lambda z: z.view(B, S, nh, C // nh).transpose(1, 2)
        y = F.scaled_dot_product_attention(sh(q), sh(k), sh(v), is_causal=True).transpose(1, 2).reshape(B, S, C)
        x = x + F.linear(y, Wt[p + "attn.c_proj.weight"], Wt.get(p + "attn.c_proj.bias"))
        u = F.layer_norm(x, (C,), Wt[p + "ln_2.weight"], Wt.get(p + "ln_2.bias"), 1e-5)
        hh = F.gelu(F.linear(u, Wt[p + "mlp.c_fc.weight"], Wt.get(p + "mlp.c_fc.bias")), approximate=appr)
        x = x + F.linear(hh, Wt[p + "mlp.c_proj.weight"], Wt.get(p + "mlp.c_proj.bias"))
    u = F.layer_norm(x, (C,), Wt["ln_f.weight"], Wt.get("ln_f.bias"), 1e-5)
    logits = u @ Wt["wte"].T
    loss = F.cross_entropy(logits.view(-1, logits.size(-1)), torch.from_numpy(np.asarray(tgt)).view(-1),
                           ignore_index=-1)
    loss.backward()
    return {k: t.grad.numpy() for k, t in Wt.items()}, float(loss.detach())


def pin_vs_torch_autograd(o=ob):
    for gelu_mode in ("erf", "tanh"):
        cfg, W, idx, tgt = tiny_case(n_layer=3, B=3, T=17)
        g, loss = o.backward(W, cfg, idx, tgt, gelu_mode)
        tg, tl = torch_grads(W, cfg, idx, tgt, gelu_mode)
        assert loss == pytest.approx(tl, rel=1e-12)
        for name in W:
            assert np.allclose(g[name], tg[name], rtol=1e-9, atol=1e-12), name


def pin_invariants(o=ob):
    cfg, W, idx, tgt = tiny_case(B=3, T=11, ignore_frac=0.3)
    logits = oracle.forward(W, cfg, idx, tgt)["logits"]
    dz = o.cross_entropy_backward(logits, tgt).reshape(-1, logits.shape[-1])
    keep = tgt.reshape(-1) != -1
    assert np.allclose(dz[keep].sum(axis=-1), 0.0, atol=1e-15)
    assert np.all(dz[~keep] == 0.0) and (~keep).any()
    assert np.allclose(dz[keep].min(axis=-1), -(1.0 - np.exp(-oracle.forward(W, cfg, idx, tgt)["row_loss"]
                                                                 .reshape(-1)[keep])) / keep.sum(), atol=1e-14)
    x = RNG.normal(size=(5, 32)) * 3 + 1
    dx, _, _ = o.layer_norm_backward(RNG.normal(size=(5, 32)), x, RNG.normal(size=32))
    assert np.allclose(dx.sum(axis=-1), 0.0, atol=1e-12)


PINS = [pin_finite_differences, pin_vs_torch_autograd, pin_invariants]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()


# --------------------------------------------------------------------------- planted mistakes
@contextmanager
def planted(name, fn):
    old = getattr(ob, name)
    setattr(ob, name, fn)
    try:
        yield
    finally:
        setattr(ob, name, old)


_orig = {n: getattr(ob, n) for n in ("layer_norm_backward", "attention_backward", "cross_entropy_backward",
                                     "gelu_backward", "embed_backward", "linear_backward")}


def _ln_no_mean_term(dy, x, w, eps=1e-5):
    dy, x, w = np.asarray(dy, float), np.asarray(x, float), np.asarray(w, float)
    mean = x.mean(axis=-1, keepdims=True)
    rstd = 1.0 / np.sqrt(((x - mean) ** 2).mean(axis=-1, keepdims=True) + eps)
    xhat = (x - mean) * rstd
    dxhat = dy * w
    dx = rstd * (dxhat - xhat * (dxhat * xhat).mean(axis=-1, keepdims=True))       # drops mean(dxhat)
    dy2 = dy.reshape(-1, dy.shape[-1])
    return dx, (dy2 * xhat.reshape(dy2.shape)).sum(axis=0), dy2.sum(axis=0)


def _attn_no_rowsum(dy, q, k, v):
    import math
    import oracle.gpt as G
    dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    for b in range(q.shape[0]):
        P = G.attention_probs(q[b], k[b])
        dv[b] = np.swapaxes(P, -1, -2) @ dy[b]
        dS = P * (dy[b] @ np.swapaxes(v[b], -1, -2))                                  # no - rowsum(dP P)
        dq[b] = dS @ k[b] / math.sqrt(q.shape[-1])
        dk[b] = np.swapaxes(dS, -1, -2) @ q[b] / math.sqrt(q.shape[-1])
    return dq, dk, dv


def _ce_no_count(logits, targets, ignore_index=-1):
    n = int((np.asarray(targets) != ignore_index).sum())
    return _orig["cross_entropy_backward"](logits, targets, ignore_index) * n         # a sum, not a mean


def _gelu_missing_density(dh, z, mode="erf"):
    import math
    import oracle.gpt as G
    return np.asarray(dh) * 0.5 * (1.0 + G.erf(np.asarray(z) / math.sqrt(2.0)))     # Phi only


def _embed_no_wpe(dx, idx, V, block_size):
    dwte, dwpe = _orig["embed_backward"](dx, idx, V, block_size)
    return dwte, np.zeros_like(dwpe)


def _linear_w_transposed(dy, x, W):
    dx, dW, db = _orig["linear_backward"](dy, x, W)
    return dx, (dW.T if dW.shape[0] == dW.shape[1] else dW * 1.5), db


MISTAKES = {
    "layer_norm_backward:no-mean": ("layer_norm_backward", _ln_no_mean_term),
    "attention_backward:no-rowsum": ("attention_backward", _attn_no_rowsum),
    "cross_entropy_backward:sum": ("cross_entropy_backward", _ce_no_count),
    "gelu_backward:Phi-only": ("gelu_backward", _gelu_missing_density),
    "embed_backward:no-wpe": ("embed_backward", _embed_no_wpe),
    "linear_backward:dW": ("linear_backward", _linear_w_transposed),
}


@pytest.mark.parametrize("mistake", sorted(MISTAKES))
def test_planted_mistakes(mistake):
    name, fn = MISTAKES[mistake]
    failed = []
    with planted(name, fn):
        for pin in PINS:
            try:
                pin(ob)
            except AssertionError:
                failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {mistake}"
