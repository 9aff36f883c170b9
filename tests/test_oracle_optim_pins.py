"""Pins of the optimizer oracle (oracle/optim.py) against facts that do not come from it.

* Closed forms of the schedule printed on "nanoGPT 全局流程图" 3.5: lr(0) = 6e-4/2001, the peak
  6e-4 at the end of warm-up, the midpoint of the cosine at (6e-4 + 6e-5)/2, the floor 6e-5.
* The first AdamW step from zero moments: m = (1-b1) g, v = (1-b2) g^2, so the step is
  lr * g / (|g| + eps) after the decay factor (1 - lr wd).
* Library routines: torch.optim.AdamW with the page's two parameter groups, and
  torch.nn.utils.clip_grad_norm_, in fp64 on CPU, over several steps.
* The grouping: weight decay exactly on the tensors with two or more dimensions.

Planted mistakes (coupled L2 decay, decay on every tensor, missing bias correction, a per-tensor
clip, warm-up off by one) must each fail a pin.
"""
import math
from contextlib import contextmanager

import numpy as np
import pytest
import torch

import oracle.optim as oo
import seeded

TINY = seeded.WORKLOADS["tiny"].model_dict()
RNG = np.random.default_rng(20240603)


def model_tensors(cfg=TINY):
    shapes = seeded.weight_shapes(cfg)
    p = {n: RNG.normal(0, 0.02, s) for n, s in shapes.items()}
    g = {n: RNG.normal(0, 0.05, s) for n, s in shapes.items()}
    return p, g


def pin_schedule(o=oo):
    assert o.lr_at(0) == pytest.approx(6e-4 / 2001, rel=1e-15)
    assert o.lr_at(1999) == pytest.approx(6e-4 * 2000 / 2001, rel=1e-15)
    assert o.lr_at(2000) == pytest.approx(6e-4, rel=1e-15)
    assert o.lr_at(301000) == pytest.approx((6e-4 + 6e-5) / 2, rel=1e-12)
    assert o.lr_at(600000) == pytest.approx(6e-5, rel=1e-12)
    assert o.lr_at(600001) == 6e-5 and o.lr_at(10 ** 7) == 6e-5
    lrs = [o.lr_at(i) for i in range(2000, 600001, 997)]
    assert all(a >= b for a, b in zip(lrs, lrs[1:]))          # the cosine only decreases


def pin_first_step_closed_form(o=oo):
    p, g = model_tensors()
    z = {n: np.zeros_like(a) for n, a in p.items()}
    lr, wd, eps = 3e-4, 0.1, 1e-8
    newp, m, v, total = o.adamw_step(p, g, z, z, 1, lr, weight_decay=wd, eps=eps, max_norm=0)
    for n in p:
        decay = wd if p[n].ndim >= 2 else 0.0
        want = p[n] * (1 - lr * decay) - lr * g[n] / (np.abs(g[n]) + eps)
        assert np.allclose(newp[n], want, rtol=0, atol=1e-15)
        assert np.allclose(m[n], 0.1 * g[n], rtol=1e-14, atol=0)
        assert np.allclose(v[n], 0.05 * g[n] ** 2, rtol=1e-14, atol=0)
    assert total == pytest.approx(math.sqrt(sum((a ** 2).sum() for a in g.values())), rel=1e-14)


def pin_vs_torch(o=oo, steps=4):
    """torch.optim.AdamW with the page's groups and clip_grad_norm_, fp64 CPU, several steps;
    gradients scaled so that clipping is active on some steps and not on others."""
    p, _ = model_tensors()
    names = list(p)
    tp = {n: torch.nn.Parameter(torch.from_numpy(p[n].copy())) for n in names}
    decay = [tp[n] for n in names if tp[n].dim() >= 2]
    nodecay = [tp[n] for n in names if tp[n].dim() < 2]
    opt = torch.optim.AdamW([{"params": decay, "weight_decay": 0.1}, {"params": nodecay, "weight_decay": 0.0}],
                            lr=1.0, betas=(0.9, 0.95), eps=1e-8)
    op = {n: p[n].copy() for n in names}
    om = {n: np.zeros_like(p[n]) for n in names}
    ov = {n: np.zeros_like(p[n]) for n in names}
    for step in range(1, steps + 1):
        scale = 0.01 if step % 2 else 0.5             # global norm below / above 1.0
        g = {n: RNG.normal(0, scale, p[n].shape) for n in names}
        lr = o.lr_at(step * 700)
        for n in names:
            tp[n].grad = torch.from_numpy(g[n].copy())
        tn = float(torch.nn.utils.clip_grad_norm_([tp[n] for n in names], 1.0))
        for grp in opt.param_groups:
            grp["lr"] = lr
        opt.step()
        op, om, ov, total = o.adamw_step(op, g, om, ov, step, lr)
        assert total == pytest.approx(tn, rel=1e-12)
        for n in names:
            assert np.allclose(op[n], tp[n].detach().numpy(), rtol=0, atol=1e-14), (step, n)
            st = opt.state[tp[n]]
            assert np.allclose(om[n], st["exp_avg"].numpy(), rtol=0, atol=1e-16)
            assert np.allclose(ov[n], st["exp_avg_sq"].numpy(), rtol=0, atol=1e-18)


def pin_grouping(o=oo):
    shapes = seeded.weight_shapes(seeded.WORKLOADS["gpt2"].model_dict())
    decayed = {n for n, s in shapes.items() if o.decays(s)}
    want = {"wte", "wpe"} | {f"h.{l}.{t}.weight" for l in range(12)
                             for t in ("attn.c_attn", "attn.c_proj", "mlp.c_fc", "mlp.c_proj")}
    assert decayed == want
    n_decay = sum(int(np.prod(shapes[n])) for n in decayed)
    n_rest = sum(int(np.prod(s)) for n, s in shapes.items() if n not in decayed)
    assert (len(decayed), len(shapes) - len(decayed)) == (50, 98)
    assert n_decay + n_rest == 124475904 and n_rest == 121344


PINS = [pin_schedule, pin_first_step_closed_form, pin_vs_torch, pin_grouping]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()


# --------------------------------------------------------------------------- planted mistakes
@contextmanager
def planted(name, fn):
    old = getattr(oo, name)
    setattr(oo, name, fn)
    try:
        yield
    finally:
        setattr(oo, name, old)


_orig = {n: getattr(oo, n) for n in ("adamw_step", "decays", "lr_at", "grad_norm")}


def _coupled_decay(params, grads, m, v, step, lr, betas=oo.BETAS, eps=oo.EPS, weight_decay=oo.WEIGHT_DECAY,
                   max_norm=oo.GRAD_CLIP):
    g2 = {n: np.asarray(grads[n]) + (weight_decay * np.asarray(params[n]) if oo.decays(np.shape(params[n])) else 0)
          for n in params}
    return _orig["adamw_step"](params, g2, m, v, step, lr, betas, eps, 0.0, max_norm)


def _no_bias_correction(params, grads, m, v, step, lr, betas=oo.BETAS, eps=oo.EPS, weight_decay=oo.WEIGHT_DECAY,
                        max_norm=oo.GRAD_CLIP):
    # pretend every step is late enough for the corrections to vanish
    p, mm, vv, t = _orig["adamw_step"](params, grads, m, v, 10 ** 6, lr, betas, eps, weight_decay, max_norm)
    return p, mm, vv, t


def _per_tensor_norm(grads):
    return max(math.sqrt(float(np.sum(np.asarray(g) ** 2))) for g in grads.values())


def _warmup_off_by_one(it, learning_rate=oo.LEARNING_RATE, min_lr=oo.MIN_LR, warmup_iters=oo.WARMUP_ITERS,
                       lr_decay_iters=oo.LR_DECAY_ITERS):
    if it < warmup_iters:
        return learning_rate * it / warmup_iters
    return _orig["lr_at"](it, learning_rate, min_lr, warmup_iters, lr_decay_iters)


MISTAKES = {
    "adamw:coupled-decay": ("adamw_step", _coupled_decay),
    "adamw:no-bias-correction": ("adamw_step", _no_bias_correction),
    "decays:everything": ("decays", lambda shape: True),
    "grad_norm:per-tensor": ("grad_norm", _per_tensor_norm),
    "lr_at:warmup": ("lr_at", _warmup_off_by_one),
}


@pytest.mark.parametrize("mistake", sorted(MISTAKES))
def test_planted_mistakes(mistake):
    name, fn = MISTAKES[mistake]
    failed = []
    with planted(name, fn):
        for pin in PINS:
            try:
                pin(oo)
            except AssertionError:
                failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {mistake}"
