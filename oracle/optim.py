"""Plain fp64 definition of one nanoGPT optimizer step: the learning-rate schedule, global
gradient-norm clipping and AdamW with weight decay on matrices only.

TEST INFRASTRUCTURE, NOT PRODUCT CODE: only tests, ``smoke()`` and the CPU-baseline leg of
``bench.py`` use this module.  Parameters, gradients and Adam moments are dicts name -> numpy
array, in any order; nothing is fused or reordered beyond the definitions.

Pages (cited by title and section):
  [流程图] "nanoGPT 全局流程图" (devpress.csdn.net): 3.5 学习率调度 (get_lr), 3.6 梯度裁剪 + 参数
           更新 (clip_grad_norm_ with grad_clip 1.0, then the optimizer step), 优化器配置
           (configure_optimizers: weight decay 0.1 on parameters with dim >= 2, none on the
           rest, torch.optim.AdamW with betas (0.9, 0.95)).
  [代码解析] "nanoGPT 代码解析" (liaow.com wiki): configure_optimizers (the same grouping).

Readings taken where the pages leave a step open:
  * get_lr after lr_decay_iters: the page's code stops at the cosine branch but its comment
    (阶段3) and its plot hold the rate at min_lr; that is what is computed here.
  * AdamW is torch.optim.AdamW's algorithm (the page calls it): decoupled decay
    p <- p (1 - lr wd), then m, v updates and the bias-corrected step with eps = 1e-8 (torch's
    default; the page does not set it).
  * clip_grad_norm_ is torch's: total = sqrt(sum of every gradient entry squared),
    coef = max_norm / (total + 1e-6), gradients scaled by min(coef, 1).
  * The GradScaler of the page is for fp16 training; with bf16 or fp32 it is the identity.

Parity pins: ``tests/test_oracle_optim_pins.py``.
"""
from __future__ import annotations

import math

import numpy as np

LEARNING_RATE = 6e-4      # [流程图] 3.5: the plot's peak
MIN_LR = 6e-5             # [流程图] 3.5: the plot's floor
WARMUP_ITERS = 2000       # [流程图] 3.5: 预热（0 → 2000步）
LR_DECAY_ITERS = 600000   # [流程图] 3.5: 余弦衰减（2000 → 600000步）
BETAS = (0.9, 0.95)       # [流程图] 优化器配置
WEIGHT_DECAY = 0.1        # [流程图] 优化器配置
GRAD_CLIP = 1.0           # [流程图] 3.6
EPS = 1e-8                # torch.optim.AdamW default (reading)


def lr_at(it, learning_rate=LEARNING_RATE, min_lr=MIN_LR, warmup_iters=WARMUP_ITERS,
          lr_decay_iters=LR_DECAY_ITERS):
    """get_lr(it) ([流程图] 3.5): linear warm-up, cosine decay, then min_lr."""
    if it < warmup_iters:
        return learning_rate * (it + 1) / (warmup_iters + 1)
    if it > lr_decay_iters:
        return min_lr
    decay_ratio = (it - warmup_iters) / (lr_decay_iters - warmup_iters)
    coeff = 0.5 * (1.0 + math.cos(math.pi * decay_ratio))
    return min_lr + coeff * (learning_rate - min_lr)


def decays(shape):
    """configure_optimizers' grouping ([流程图] 优化器配置): weight decay iff p.dim() >= 2."""
    return len(shape) >= 2


def grad_norm(grads):
    """The global L2 norm of every gradient entry (clip_grad_norm_ with norm_type 2)."""
    return math.sqrt(sum(float(np.sum(np.asarray(g, np.float64) ** 2)) for g in grads.values()))


def clip_coef(total_norm, max_norm=GRAD_CLIP):
    """The factor clip_grad_norm_ scales every gradient by: min(1, max_norm / (total + 1e-6))."""
    return min(1.0, max_norm / (total_norm + 1e-6))


def adamw_step(params, grads, m, v, step, lr, betas=BETAS, eps=EPS, weight_decay=WEIGHT_DECAY,
               max_norm=GRAD_CLIP):
    """One optimizer step ([流程图] 3.6): clip the gradients by their global norm (max_norm None
    or 0 skips clipping), then AdamW on every tensor, decay only where decays(shape).
    ``step`` counts from 1.  Returns (params, m, v, total_norm) as new dicts."""
    total = grad_norm(grads)
    coef = clip_coef(total, max_norm) if max_norm else 1.0
    b1, b2 = betas
    bc1 = 1.0 - b1 ** step
    bc2 = 1.0 - b2 ** step
    out_p, out_m, out_v = {}, {}, {}
    for name, p in params.items():
        p = np.array(p, dtype=np.float64)
        g = np.asarray(grads[name], np.float64) * coef
        wd = weight_decay if decays(p.shape) else 0.0
        p = p * (1.0 - lr * wd)
        mm = b1 * np.asarray(m[name], np.float64) + (1.0 - b1) * g
        vv = b2 * np.asarray(v[name], np.float64) + (1.0 - b2) * g * g
        denom = np.sqrt(vv) / math.sqrt(bc2) + eps
        p = p - (lr / bc1) * mm / denom
        out_p[name], out_m[name], out_v[name] = p, mm, vv
    return out_p, out_m, out_v, total
