"""Plain fp64 definition of the nanoGPT / GPT-2 forward pass, written from the pages.

TEST INFRASTRUCTURE, NOT PRODUCT CODE: only tests, ``smoke()`` and the CPU-baseline leg
of ``bench.py`` use this module.  Nothing here is blocked, fused or reordered beyond what
the definitions state; numpy's matrix product is the one library primitive used as a
step, and ``scipy.special.erf`` supplies erf for the exact GELU.

Pages (cited by title and section):
  [流程图]   "nanoGPT 全局流程图" (devpress.csdn.net): §2.1 模型配置, §2.2 创建模型,
             §2.3 权重共享, §2.4 特殊初始化, §2.5 (A) LayerNorm / (B) CausalSelfAttention /
             (C) MLP, §3.2 前向传播, §3.3 算损失.
  [逐步详解] "nanoGPT架构逐步详解" (lzwjava.github.io): 1. Token + 位置嵌入, 2. Block,
             3. 因果自注意力, 4. MLP（FFN）, 5. 输出头, 完整前向传播, 参数数量 table.
  [代码解析] "nanoGPT 代码解析" (liaow.com wiki): GPT 类的方法节选 (forward), 参数量计算.
  [速查表]   "nanoGPT 核心代码速查表" (pgsm.cn): 三、Attention 计算步骤.
  [DummyGPT] "DummyGPTModel" page (paozippq.com): 参数规模分析, DummyLayerNorm comment.

Readings taken where the pages are silent or disagree:
  * GELU is x*Phi(x) with the exact normal CDF ([逐步详解] 4. MLP; nn.GELU() in [流程图]
    §2.5 (C)); the tanh form is offered as an explicit alternative mode.
  * cross-entropy skips targets equal to -1 and averages over the rest ([流程图] §3.2,
    [代码解析] forward); with no counted row the mean is 0/0 = NaN.
  * softmax runs over all vocabulary columns, the padded ones included.
  * pre-LN ([流程图] §2.5, [逐步详解] 2. Block), not the post-LN sketch of [DummyGPT].
  * dropout is the identity (p = 0.0 in [流程图] §2.1, and this is a forward pass).

Parity pins: every function here is checked in ``tests/test_oracle_pins.py`` against
brute force, closed forms, worked values printed on the pages, invariants or an
independent library routine.  No function is "parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import erf

PAGES = {
    "流程图": "nanoGPT 全局流程图 (devpress.csdn.net)",
    "逐步详解": "nanoGPT架构逐步详解 (lzwjava.github.io)",
    "代码解析": "nanoGPT 代码解析 (liaow.com wiki)",
    "速查表": "nanoGPT 核心代码速查表 (pgsm.cn)",
    "DummyGPT": "DummyGPTModel (paozippq.com)",
}

LN_EPS = 1e-5  # F.layer_norm(..., 1e-5) in [流程图] §2.5 (A)


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def embed(wte, wpe, idx):
    """x[b, t] = wte[idx[b, t]] + wpe[t].

    [流程图] §3.2 ① (tok_emb + pos_emb, pos = arange(t)); [逐步详解] 1. Token + 位置嵌入.
    Dropout after the sum is the identity (p = 0.0, [流程图] §2.1).
    """
    idx = np.asarray(idx)
    T = idx.shape[-1]
    return _f64(wte)[idx] + _f64(wpe)[:T]


def layer_norm(x, w, b, eps=LN_EPS):
    """(x - mean) / sqrt(var + eps) * w + b over the last axis, var the population variance.

    [流程图] §2.5 (A) (F.layer_norm with eps 1e-5: mean 0 / variance 1, then weight and
    bias); [DummyGPT] DummyLayerNorm comment (var with unbiased=False).  ``b`` may be None
    (bias=False).
    """
    x = _f64(x)
    mean = x.mean(axis=-1, keepdims=True)
    var = ((x - mean) ** 2).mean(axis=-1, keepdims=True)
    y = (x - mean) / np.sqrt(var + eps) * _f64(w)
    if b is not None:
        y = y + _f64(b)
    return y


def linear(x, W, b=None):
    """nn.Linear: x @ W^T + b with W stored [out, in]."""
    y = _f64(x) @ _f64(W).T
    if b is not None:
        y = y + _f64(b)
    return y


def split_heads(qkv, n_head):
    """Split c_attn's output into q, k, v and view each as [B, nh, T, hs].

    [流程图] §2.5 (B) 步骤1-2: split(n_embd, dim=2) in the order q, k, v, then
    view(B, T, nh, hs).transpose(1, 2): head h owns columns [h*hs, (h+1)*hs).
    """
    B, T, C3 = qkv.shape
    C = C3 // 3
    hs = C // n_head
    q, k, v = qkv[..., :C], qkv[..., C:2 * C], qkv[..., 2 * C:]
    f = lambda z: z.reshape(B, T, n_head, hs).transpose(0, 2, 1, 3)
    return f(q), f(k), f(v)


def merge_heads(y):
    """[B, nh, T, hs] -> [B, T, nh*hs]: transpose(1, 2).contiguous().view(B, T, C),
    [流程图] §2.5 (B) 步骤7."""
    B, nh, T, hs = y.shape
    return y.transpose(0, 2, 1, 3).reshape(B, T, nh * hs)


def attention_probs(q, k):
    """P = softmax(mask(q k^T / sqrt(hs))) for one or more heads ([..., T, hs] inputs).

    [流程图] §2.5 (B) 步骤3-5: scores scaled by 1/sqrt(hs), positions j > i filled with
    -inf by the lower-triangular mask, softmax over the last axis.  The row maximum is
    subtracted before exponentiating (softmax's value does not change).
    """
    q, k = _f64(q), _f64(k)
    T, hs = q.shape[-2], q.shape[-1]
    s = (q @ np.swapaxes(k, -1, -2)) * (1.0 / math.sqrt(hs))
    allowed = np.tril(np.ones((T, T), dtype=bool))
    s = np.where(allowed, s, -np.inf)
    s = s - s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    return p / p.sum(axis=-1, keepdims=True)


def causal_attention(q, k, v):
    """y = P v, P from :func:`attention_probs` ([流程图] §2.5 (B) 步骤6).

    Inputs [B, nh, T, hs]; evaluated one sequence at a time so the [nh, T, T] score
    block stays small.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    if q.ndim == 2:
        return attention_probs(q, k) @ v
    out = np.empty(q.shape[:-1] + (v.shape[-1],))
    for b in range(q.shape[0]):
        out[b] = attention_probs(q[b], k[b]) @ v[b]
    return out


def gelu(z, mode="erf"):
    """GELU.  ``erf``: z * Phi(z) = 0.5 z (1 + erf(z / sqrt 2)) ([逐步详解] 4. MLP: "x·Φ(x)",
    Phi the standard normal CDF; nn.GELU() in [流程图] §2.5 (C)).  ``tanh``: the usual
    approximation 0.5 z (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3))) (offered as a mode)."""
    z = _f64(z)
    if mode == "erf":
        return 0.5 * z * (1.0 + erf(z / math.sqrt(2.0)))
    if mode == "tanh":
        return 0.5 * z * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (z + 0.044715 * z ** 3)))
    raise ValueError(mode)


def _w(W, name):
    return W.get(name)


def causal_self_attention(u, W, layer, n_head):
    """CausalSelfAttention.forward ([流程图] §2.5 (B); [逐步详解] 3. 因果自注意力):
    c_attn (C -> 3C), split into heads, causal attention, merge heads, c_proj."""
    p = f"h.{layer}.attn."
    qkv = linear(u, W[p + "c_attn.weight"], _w(W, p + "c_attn.bias"))
    q, k, v = split_heads(qkv, n_head)
    y = merge_heads(causal_attention(q, k, v))
    return linear(y, W[p + "c_proj.weight"], _w(W, p + "c_proj.bias"))


def mlp(u, W, layer, gelu_mode="erf"):
    """MLP.forward: c_fc (C -> 4C), GELU, c_proj (4C -> C) ([流程图] §2.5 (C);
    [逐步详解] 4. MLP（FFN）)."""
    p = f"h.{layer}.mlp."
    h = gelu(linear(u, W[p + "c_fc.weight"], _w(W, p + "c_fc.bias")), gelu_mode)
    return linear(h, W[p + "c_proj.weight"], _w(W, p + "c_proj.bias"))


def block(x, W, layer, n_head, gelu_mode="erf"):
    """Pre-LN Block: x = x + attn(ln_1(x)); x = x + mlp(ln_2(x))
    ([流程图] §2.5 Block.forward; [逐步详解] 2. Block)."""
    p = f"h.{layer}."
    x = _f64(x)
    x = x + causal_self_attention(layer_norm(x, W[p + "ln_1.weight"], _w(W, p + "ln_1.bias")),
                                  W, layer, n_head)
    x = x + mlp(layer_norm(x, W[p + "ln_2.weight"], _w(W, p + "ln_2.bias")), W, layer, gelu_mode)
    return x


def final_hidden(W, cfg, idx, gelu_mode="erf"):
    """Embedding, all Blocks, then ln_f ([流程图] §3.2 ①-③)."""
    x = embed(W["wte"], W["wpe"], idx)
    for l in range(cfg["n_layer"]):
        x = block(x, W, l, cfg["n_head"], gelu_mode)
    return layer_norm(x, W["ln_f.weight"], _w(W, "ln_f.bias"))


def lm_head(u, W):
    """Tied output head: logits = u @ wte^T, no bias ([流程图] §2.2 ⑥ bias=False,
    §2.3 wte.weight = lm_head.weight)."""
    return _f64(u) @ _f64(W["wte"]).T


def cross_entropy(logits, targets, ignore_index=-1):
    """Mean over counted rows of logsumexp(z) - z[target] (F.cross_entropy,
    [流程图] §3.2 ④ / §3.3; ignore_index=-1 per [代码解析] forward).

    Returns (mean, per-row loss with 0 at ignored rows, number of counted rows).
    """
    z = _f64(logits).reshape(-1, np.shape(logits)[-1])
    t = np.asarray(targets).reshape(-1)
    zmax = z.max(axis=-1)
    lse = zmax + np.log(np.exp(z - zmax[:, None]).sum(axis=-1))
    keep = t != ignore_index
    row = np.zeros(z.shape[0])
    row[keep] = lse[keep] - z[np.nonzero(keep)[0], t[keep]]
    n = int(keep.sum())
    mean = row[keep].sum() / n if n > 0 else float("nan")
    return mean, row, n


def forward(W, cfg, idx, targets=None, gelu_mode="erf", keep_logits=True, row_chunk=512):
    """GPT.forward(idx, targets) ([流程图] §3.2; [代码解析] forward; [逐步详解] 完整前向传播).

    With targets: logits for every position [B, T, V] and the cross-entropy.  Without:
    logits of the last position only, [B, 1, V], and no loss.

    The head and loss are evaluated ``row_chunk`` rows at a time so a [B*T, V] fp64
    array need not exist; ``keep_logits=False`` returns only the loss terms.
    Returns dict(logits=..., loss=..., row_loss=..., count=...).
    """
    idx = np.asarray(idx)
    B, T = idx.shape
    u = final_hidden(W, cfg, idx, gelu_mode)
    if targets is None:
        return {"logits": lm_head(u[:, -1:, :], W), "loss": None}
    targets = np.asarray(targets)
    uf = u.reshape(B * T, -1)
    tf = targets.reshape(-1)
    V = W["wte"].shape[0]
    logits = np.empty((B * T, V)) if keep_logits else None
    row = np.zeros(B * T)
    for r0 in range(0, B * T, row_chunk):
        z = lm_head(uf[r0:r0 + row_chunk], W)
        if keep_logits:
            logits[r0:r0 + row_chunk] = z
        _, row[r0:r0 + row_chunk], _ = cross_entropy(z, tf[r0:r0 + row_chunk])
    keep = tf != -1
    n = int(keep.sum())
    loss = row[keep].sum() / n if n > 0 else float("nan")
    return {"logits": None if logits is None else logits.reshape(B, T, V),
            "loss": loss, "row_loss": row.reshape(B, T), "count": n}


def num_params(cfg, non_embedding=True):
    """get_num_params ([代码解析] 参数量计算): every parameter counted once (wte and
    lm_head are one tensor, [流程图] §2.3), minus wpe when ``non_embedding``."""
    C, V, L, bs = cfg["n_embd"], cfg["vocab_size"], cfg["n_layer"], cfg["block_size"]
    bias = 1 if cfg.get("bias", True) else 0
    ln = C + bias * C
    per_block = (ln + (3 * C * C + bias * 3 * C) + (C * C + bias * C)
                 + ln + (4 * C * C + bias * 4 * C) + (4 * C * C + bias * C))
    n = V * C + bs * C + L * per_block + ln
    if non_embedding:
        n -= bs * C
    return n
