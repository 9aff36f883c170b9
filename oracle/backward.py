"""Plain fp64 definition of the gradients of the nanoGPT loss with respect to every parameter.

TEST INFRASTRUCTURE, NOT PRODUCT CODE: only tests, ``smoke()`` and the CPU-baseline leg of
``bench.py`` use this module.

Pages (cited by title and section):
  [流程图] "nanoGPT 全局流程图" (devpress.csdn.net): 3.4 反向传播 (loss.backward(): the chain rule
           from the loss back through the graph to every parameter), and the forward it
           differentiates (§2.5, §3.2, §3.3; see oracle/gpt.py).

The pages print no gradient formula; each function below is the derivative of the matching
forward definition in oracle/gpt.py, taken by the chain rule, in the forward's notation.  The
forward values the derivatives need are recomputed by ``forward_with_cache`` from oracle/gpt.py's
own functions.  Nothing is fused or reordered beyond the definitions; numpy's matrix product is
the one library primitive used as a step.

Parity pins: ``tests/test_oracle_backward_pins.py`` (central finite differences, torch fp64
autograd of the library composition, closed-form invariants, planted mistakes).
"""
from __future__ import annotations

import math

import numpy as np

from . import gpt as G


def _f64(a):
    return np.asarray(a, dtype=np.float64)


# ----------------------------------------------------------------------------- per operation
def cross_entropy_backward(logits, targets, ignore_index=-1):
    """d(mean loss)/d(logits): (softmax(z_r) - onehot(t_r)) / n for every counted row r (target
    != ignore_index), 0 for ignored rows; n = number of counted rows ([流程图] §3.3, the mean
    over counted positions)."""
    z = _f64(logits)
    t = np.asarray(targets).reshape(-1)
    z2 = z.reshape(-1, z.shape[-1])
    keep = t != ignore_index
    n = int(keep.sum())
    dz = np.zeros_like(z2)
    if n == 0:
        return dz.reshape(z.shape)
    e = np.exp(z2 - z2.max(axis=-1, keepdims=True))
    p = e / e.sum(axis=-1, keepdims=True)
    rows = np.nonzero(keep)[0]
    dz[rows] = p[rows]
    dz[rows, t[rows]] -= 1.0
    return (dz / n).reshape(z.shape)


def linear_backward(dy, x, W):
    """y = x W^T + b: (dx, dW, db) with dx = dy W, dW = sum over rows of dy^T x, db = sum of dy."""
    dy, x, W = _f64(dy), _f64(x), _f64(W)
    dy2 = dy.reshape(-1, dy.shape[-1])
    x2 = x.reshape(-1, x.shape[-1])
    return (dy @ W), dy2.T @ x2, dy2.sum(axis=0)


def layer_norm_backward(dy, x, w, eps=G.LN_EPS):
    """y = xhat w + b, xhat = (x - mean) / sqrt(var + eps), var the population variance over the
    row: (dx, dw, db) with dx = (dxhat - mean(dxhat) - xhat mean(dxhat xhat)) / sqrt(var + eps),
    dxhat = dy w, dw = sum over rows of dy xhat, db = sum of dy."""
    dy, x, w = _f64(dy), _f64(x), _f64(w)
    mean = x.mean(axis=-1, keepdims=True)
    var = ((x - mean) ** 2).mean(axis=-1, keepdims=True)
    rstd = 1.0 / np.sqrt(var + eps)
    xhat = (x - mean) * rstd
    dxhat = dy * w
    dx = rstd * (dxhat - dxhat.mean(axis=-1, keepdims=True) - xhat * (dxhat * xhat).mean(axis=-1, keepdims=True))
    dy2 = dy.reshape(-1, dy.shape[-1])
    return dx, (dy2 * xhat.reshape(dy2.shape)).sum(axis=0), dy2.sum(axis=0)


def gelu_backward(dh, z, mode="erf"):
    """dh * gelu'(z).  erf form: gelu(z) = z Phi(z), gelu'(z) = Phi(z) + z phi(z) with phi the
    standard normal density.  tanh form: with a = sqrt(2/pi) (z + 0.044715 z^3),
    gelu'(z) = 0.5 (1 + tanh a) + 0.5 z (1 - tanh^2 a) sqrt(2/pi) (1 + 3 * 0.044715 z^2)."""
    dh, z = _f64(dh), _f64(z)
    if mode == "erf":
        phi = np.exp(-0.5 * z * z) / math.sqrt(2.0 * math.pi)
        Phi = 0.5 * (1.0 + G.erf(z / math.sqrt(2.0)))
        return dh * (Phi + z * phi)
    if mode == "tanh":
        c = math.sqrt(2.0 / math.pi)
        th = np.tanh(c * (z + 0.044715 * z ** 3))
        return dh * (0.5 * (1.0 + th) + 0.5 * z * (1.0 - th * th) * c * (1.0 + 3 * 0.044715 * z * z))
    raise ValueError(mode)


def attention_backward(dy, q, k, v):
    """y = P v with P = softmax(mask(q k^T / sqrt(hs))) per head ([..., T, hs]):
    dv = P^T dy, dP = dy v^T, dS = P (dP - rowsum(dP P)) (softmax's derivative; masked entries
    have P = 0 and get 0), dq = dS k / sqrt(hs), dk = dS^T q / sqrt(hs)."""
    dy, q, k, v = _f64(dy), _f64(q), _f64(k), _f64(v)
    hs = q.shape[-1]
    dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    for b in range(q.shape[0]):
        P = G.attention_probs(q[b], k[b])
        dv[b] = np.swapaxes(P, -1, -2) @ dy[b]
        dP = dy[b] @ np.swapaxes(v[b], -1, -2)
        dS = P * (dP - (dP * P).sum(axis=-1, keepdims=True))
        dq[b] = dS @ k[b] / math.sqrt(hs)
        dk[b] = np.swapaxes(dS, -1, -2) @ q[b] / math.sqrt(hs)
    return dq, dk, dv


def split_heads_backward(dq, dk, dv):
    """Inverse of split_heads: [B, nh, T, hs] x 3 -> d(qkv) [B, T, 3C] (columns q, k, v)."""
    return np.concatenate([G.merge_heads(dq), G.merge_heads(dk), G.merge_heads(dv)], axis=-1)


def merge_heads_backward(dy, n_head):
    """Inverse of merge_heads: [B, T, C] -> [B, nh, T, hs]."""
    B, T, C = dy.shape
    return dy.reshape(B, T, n_head, C // n_head).transpose(0, 2, 1, 3)


def embed_backward(dx, idx, V, block_size):
    """x[b, t] = wte[idx[b, t]] + wpe[t]: dwte[v] = sum of dx[b, t] over positions with
    idx[b, t] = v; dwpe[t] = sum over the batch of dx[b, t] (rows t >= T get 0)."""
    dx = _f64(dx)
    B, T, C = dx.shape
    dwte = np.zeros((V, C))
    np.add.at(dwte, np.asarray(idx).reshape(-1), dx.reshape(-1, C))
    dwpe = np.zeros((block_size, C))
    dwpe[:T] = dx.sum(axis=0)
    return dwte, dwpe


# ----------------------------------------------------------------------------- the model
def forward_with_cache(W, cfg, idx, targets, gelu_mode="erf"):
    """The forward of oracle/gpt.py, keeping what the derivatives need."""
    nh = cfg["n_head"]
    cache = {"idx": np.asarray(idx), "layers": []}
    x = G.embed(W["wte"], W["wpe"], idx)
    for l in range(cfg["n_layer"]):
        p = f"h.{l}."
        c = {"x_in": x}
        c["u1"] = G.layer_norm(x, W[p + "ln_1.weight"], W.get(p + "ln_1.bias"))
        qkv = G.linear(c["u1"], W[p + "attn.c_attn.weight"], W.get(p + "attn.c_attn.bias"))
        c["q"], c["k"], c["v"] = G.split_heads(qkv, nh)
        c["y"] = G.merge_heads(G.causal_attention(c["q"], c["k"], c["v"]))
        x = x + G.linear(c["y"], W[p + "attn.c_proj.weight"], W.get(p + "attn.c_proj.bias"))
        c["x_mid"] = x
        c["u2"] = G.layer_norm(x, W[p + "ln_2.weight"], W.get(p + "ln_2.bias"))
        c["pre"] = G.linear(c["u2"], W[p + "mlp.c_fc.weight"], W.get(p + "mlp.c_fc.bias"))
        c["h"] = G.gelu(c["pre"], gelu_mode)
        x = x + G.linear(c["h"], W[p + "mlp.c_proj.weight"], W.get(p + "mlp.c_proj.bias"))
        cache["layers"].append(c)
    cache["x_final"] = x
    cache["uf"] = G.layer_norm(x, W["ln_f.weight"], W.get("ln_f.bias"))
    cache["logits"] = G.lm_head(cache["uf"], W)
    B, T = cache["idx"].shape
    _, rows, n = G.cross_entropy(cache["logits"].reshape(B * T, -1), np.asarray(targets).reshape(-1))
    keep = np.asarray(targets).reshape(-1) != -1
    cache["loss"] = rows[keep].sum() / n if n > 0 else float("nan")
    return cache


def backward(W, cfg, idx, targets, gelu_mode="erf"):
    """Gradients of the mean cross-entropy ([流程图] 3.4 loss.backward()) with respect to every
    tensor of W (same names; biases only where W has them).  Returns (grads, loss)."""
    nh = cfg["n_head"]
    c = forward_with_cache(W, cfg, idx, targets, gelu_mode)
    g = {}
    dz = cross_entropy_backward(c["logits"], targets)
    B, T, V = dz.shape
    # tied head: logits = uf wte^T
    duf = dz @ _f64(W["wte"])
    dwte_head = dz.reshape(-1, V).T @ c["uf"].reshape(-1, c["uf"].shape[-1])
    dx, g["ln_f.weight"], dbf = layer_norm_backward(duf, c["x_final"], W["ln_f.weight"])
    if "ln_f.bias" in W:
        g["ln_f.bias"] = dbf
    for l in reversed(range(cfg["n_layer"])):
        p = f"h.{l}."
        L = c["layers"][l]
        # x = x_mid + c_proj(gelu(c_fc(ln_2(x_mid))))
        dh, g[p + "mlp.c_proj.weight"], db = linear_backward(dx, L["h"], W[p + "mlp.c_proj.weight"])
        if p + "mlp.c_proj.bias" in W:
            g[p + "mlp.c_proj.bias"] = db
        dpre = gelu_backward(dh, L["pre"], gelu_mode)
        du2, g[p + "mlp.c_fc.weight"], db = linear_backward(dpre, L["u2"], W[p + "mlp.c_fc.weight"])
        if p + "mlp.c_fc.bias" in W:
            g[p + "mlp.c_fc.bias"] = db
        dxm, g[p + "ln_2.weight"], db = layer_norm_backward(du2, L["x_mid"], W[p + "ln_2.weight"])
        if p + "ln_2.bias" in W:
            g[p + "ln_2.bias"] = db
        dx = dx + dxm
        # x_mid = x_in + c_proj(attn(ln_1(x_in)))
        dy, g[p + "attn.c_proj.weight"], db = linear_backward(dx, L["y"], W[p + "attn.c_proj.weight"])
        if p + "attn.c_proj.bias" in W:
            g[p + "attn.c_proj.bias"] = db
        dq, dk, dv = attention_backward(merge_heads_backward(dy, nh), L["q"], L["k"], L["v"])
        dqkv = split_heads_backward(dq, dk, dv)
        du1, g[p + "attn.c_attn.weight"], db = linear_backward(dqkv, L["u1"], W[p + "attn.c_attn.weight"])
        if p + "attn.c_attn.bias" in W:
            g[p + "attn.c_attn.bias"] = db
        dxi, g[p + "ln_1.weight"], db = layer_norm_backward(du1, L["x_in"], W[p + "ln_1.weight"])
        if p + "ln_1.bias" in W:
            g[p + "ln_1.bias"] = db
        dx = dx + dxi
    dwte_emb, g["wpe"] = embed_backward(dx, c["idx"], W["wte"].shape[0], W["wpe"].shape[0])
    g["wte"] = dwte_head + dwte_emb
    return g, c["loss"]
