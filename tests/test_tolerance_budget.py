"""Error budget of bf16 arithmetic for the deepest model (GPT-2 XL, 48 layers).

The GPU path rounds to bf16 at seven points: both LayerNorm outputs of every Block, the
c_attn output, the attention probabilities fed to the second MMA, the attention output, the
GELU output, the ln_f output and the stored logits (fp32 accumulation and an fp32 residual
stream everywhere else).  Replaying exactly those roundings in fp64 shows how far any
implementation with these storage precisions must land from the exact oracle.  For GPT-2 XL
the replay's maximum logit error exceeds 2e-2, which is why the XL parity test derives its
bar (3e-2) from this replay instead of using 2e-2.  The replay is test infrastructure: it
reuses the oracle's head split / merge and the input generator, nothing of the CUDA path.
"""
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import erf

import oracle
import seeded


def bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).double().numpy()


def _ln(x, w, b):
    m = x.mean(-1, keepdims=True)
    v = ((x - m) ** 2).mean(-1, keepdims=True)
    return (x - m) / np.sqrt(v + 1e-5) * w + b


def _attn_bf16_p(q, k, v):
    T, hs = q.shape[-2:]
    s = q @ np.swapaxes(k, -1, -2) / math.sqrt(hs)
    s = np.where(np.tril(np.ones((T, T), bool)), s, -np.inf)
    p = np.exp(s - s.max(-1, keepdims=True))
    return (bf16(p) @ v) / p.sum(-1, keepdims=True)


def replay(W, cfg, idx):
    """The forward with bf16 rounding at the GPU path's storage points, fp64 elsewhere."""
    T, nh = idx.shape[1], cfg["n_head"]
    x = W["wte"][idx] + W["wpe"][:T]
    for l in range(cfg["n_layer"]):
        p = f"h.{l}."
        u = bf16(_ln(x, W[p + "ln_1.weight"], W[p + "ln_1.bias"]))
        qkv = bf16(u @ W[p + "attn.c_attn.weight"].T + W[p + "attn.c_attn.bias"])
        q, k, v = oracle.split_heads(qkv, nh)
        y = bf16(oracle.merge_heads(_attn_bf16_p(q, k, v)))
        x = x + y @ W[p + "attn.c_proj.weight"].T + W[p + "attn.c_proj.bias"]
        u = bf16(_ln(x, W[p + "ln_2.weight"], W[p + "ln_2.bias"]))
        a = u @ W[p + "mlp.c_fc.weight"].T + W[p + "mlp.c_fc.bias"]
        h = bf16(0.5 * a * (1 + erf(a / math.sqrt(2))))
        x = x + h @ W[p + "mlp.c_proj.weight"].T + W[p + "mlp.c_proj.bias"]
    u = bf16(_ln(x, W["ln_f.weight"], W["ln_f.bias"]))
    return bf16(u @ W["wte"].T)


def _xl_replay_error(positions):
    w = seeded.WORKLOADS["gpt2-xl"]
    cfg = w.model_dict()
    W = seeded.to_f64(seeded.make_weights(cfg))
    idx, _ = seeded.make_tokens(w.batch, w.seq_len, w.token_high)
    seq = idx[2:3, :positions].numpy()
    exact = oracle.lm_head(oracle.final_hidden(W, cfg, seq), W)
    return np.abs(replay(W, cfg, seq) - exact)


def test_xl_bf16_replay_exceeds_2e2():
    """32 positions of the XL parity test's sequence (~20 s, 13 GB of fp64 weights): already
    there the bf16 storage points alone put the logits more than 2e-2 from the exact values."""
    err = _xl_replay_error(32)
    assert err.max() > 2e-2          # the stated bar is out of reach for bf16 storage
    assert err.max() < 3e-2          # the derived XL bar holds for the replay itself
    assert err.mean() < 5e-3


@pytest.mark.slow
@pytest.mark.skipif(not os.environ.get("GPT_SLOW_TESTS"),
                    reason="the same replay over 128 positions (~1 min); set GPT_SLOW_TESTS=1")
def test_xl_bf16_replay_exceeds_2e2_128_positions():
    err = _xl_replay_error(128)
    assert 2e-2 < err.max() < 3e-2
    assert err.mean() < 5e-3
