"""Plain fp64 definition of GPT.generate: repeated forward passes and a sampling step.

TEST INFRASTRUCTURE, NOT PRODUCT CODE: only tests, ``smoke()`` and the CPU-baseline leg of
``bench.py`` use this module.  There is no key/value cache here: every step runs the whole
forward of ``oracle.gpt`` on the (cropped) sequence, which is the definition the cached
decoding of the CUDA path must reproduce.

Pages (cited by title and section):
  [流程图] "nanoGPT 全局流程图" (devpress.csdn.net): 第五阶段 生成文本 (GPT.generate) and the
           notes under it on temperature and Top-K.
  [速查表] "nanoGPT 核心代码速查表" (pgsm.cn): 七、关键函数签名,
           generate(idx, max_new_tokens, temperature, top_k) -> tokens.

Readings taken where the pages leave a step open:
  * The multinomial draw is inverse-CDF sampling with a uniform u in [0, 1) supplied by the
    caller: the drawn index is the smallest i with p_0 + ... + p_i > u.  The pages call
    torch.multinomial, whose internal random stream they do not define; passing u in makes
    both implementations draw from the same random numbers.
  * top_k None (or <= 0) means no filter; a top_k above V acts as V (the pages take
    min(top_k, V)).  Every logit equal to the k-th largest stays (the pages mask only the
    logits strictly below it), so ties can keep more than k entries.
  * temperature must be positive (the pages divide by it).

Parity pins: ``tests/test_oracle_generate_pins.py`` checks every function here against
closed forms, brute-force frequencies, library routines and invariants, and plants mistakes
that the pins must catch.
"""
from __future__ import annotations

import numpy as np

from . import gpt as _gpt


def scaled_logits(logits, temperature):
    """logits / temperature ([流程图] 第五阶段: 除以温度)."""
    if not temperature > 0:
        raise ValueError("temperature must be positive")
    return np.asarray(logits, dtype=np.float64) / float(temperature)


def top_k_filter(z, top_k):
    """Sets every entry below the top_k-th largest of its row to -inf ([流程图] 第五阶段:
    Top-K 采样); ties with the k-th largest stay."""
    z = np.array(z, dtype=np.float64)
    if top_k is None or top_k <= 0:
        return z
    k = min(int(top_k), z.shape[-1])
    kth = np.sort(z, axis=-1)[..., -k][..., None]   # the k-th largest value of each row
    return np.where(z < kth, -np.inf, z)


def probabilities(logits, temperature=1.0, top_k=None):
    """softmax(top_k_filter(logits / temperature)) over the last axis ([流程图] 第五阶段:
    Softmax -> 概率分布)."""
    z = top_k_filter(scaled_logits(logits, temperature), top_k)
    e = np.exp(z - z.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def draw(p, u):
    """Inverse-CDF draw from one probability row: the smallest i with cumsum(p)[i] > u.  When
    rounding leaves u at or past the last partial sum, the last index with p > 0 is drawn."""
    p = np.asarray(p, dtype=np.float64)
    c = np.cumsum(p)
    hit = np.nonzero(c > u)[0]
    hit = hit[p[hit] > 0] if hit.size else hit
    if hit.size:
        return int(hit[0])
    return int(np.nonzero(p > 0)[0][-1])


def sample(logits, temperature, top_k, u):
    """One sampling step for a batch: logits [B, V], u [B] -> int64 [B]."""
    p = probabilities(logits, temperature, top_k)
    return np.array([draw(p[b], u[b]) for b in range(p.shape[0])], dtype=np.int64)


def crop(idx, block_size):
    """The context the model sees: the last block_size tokens ([流程图] 第五阶段: 截断到 block_size)."""
    idx = np.asarray(idx)
    return idx if idx.shape[1] <= block_size else idx[:, -block_size:]


def generate(W, cfg, idx, max_new_tokens, uniforms, temperature=1.0, top_k=None, gelu_mode="erf"):
    """GPT.generate ([流程图] 第五阶段; [速查表] 七): appends max_new_tokens drawn tokens to idx.

    uniforms [max_new_tokens, B] supplies the draw of every step.  Returns
    dict(tokens=int64 [B, T0 + max_new_tokens], logits=fp64 [max_new_tokens, B, V]) where
    logits holds each step's last-position logits before the temperature.
    """
    idx = np.array(idx, dtype=np.int64)
    uniforms = np.asarray(uniforms, dtype=np.float64)
    steps = []
    for s in range(max_new_tokens):
        logits = _gpt.forward(W, cfg, crop(idx, cfg["block_size"]), None, gelu_mode)["logits"][:, -1, :]
        steps.append(logits)
        nxt = sample(logits, temperature, top_k, uniforms[s])
        idx = np.concatenate([idx, nxt[:, None]], axis=1)
    V = W["wte"].shape[0]
    return {"tokens": idx,
            "logits": np.stack(steps) if steps else np.zeros((0, idx.shape[0], V))}
