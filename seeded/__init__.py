"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module holds workload shapes and random draws only; it contains none of the
forward pass's arithmetic.  Both sides of every parity check receive the very same
bytes from here.

Shapes and distributions follow the five workloads used throughout:

* ``tiny``        - the small nanoGPT override (4 layers, 4 heads, 128 wide, context 64),
                    fp32, vocabulary 65, batch 8, T 64.
* ``attention``   - standalone causal attention, B 12, 12 heads, T 1024, head size 64,
                    q/k/v i.i.d. N(0, 1) stored bf16 in [B, nh, T, hs].
* ``gpt2``        - GPT-2 124M (12/12/768, context 1024, vocabulary 50304), bf16, B 12, T 1024.
* ``gpt2-medium`` - 24/16/1024, bf16, B 8, T 1024.
* ``gpt2-xl``     - 48/25/1600, bf16, B 4, T 1024.

Weights follow the GPT-2 initialisation the pages describe ("nanoGPT 全局流程图",
§2.4 特殊初始化; "nanoGPT 代码解析", 关键设计决策 table): every Linear weight and both
embedding tables N(0, 0.02); every ``c_proj.weight`` N(0, 0.02/sqrt(2*n_layer));
biases 0; LayerNorm weight 1, bias 0.  The padded vocabulary rows get the same draw.
Token ids are uniform over [0, 50257) for the GPT-2 shapes (the real vocabulary, the
table is padded to 50304) and over [0, 65) for the tiny one.

A ``stress`` variant exercises every epilogue term: biases N(0, 0.02), LayerNorm weight
1 + N(0, 0.1), LayerNorm bias N(0, 0.1) and c_proj at the full 0.02.

Seeds: a torch CPU ``Generator`` per tensor, seeded ``seed + k`` with k the tensor's
position in the packed order (base seed 1337).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, asdict

import torch

BASE_SEED = 1337


@dataclass(frozen=True)
class Workload:
    name: str
    n_layer: int
    n_head: int
    n_embd: int
    block_size: int
    vocab_size: int
    batch: int
    seq_len: int
    dtype: str            # "f32" or "bf16"
    token_high: int       # ids drawn uniformly from [0, token_high)
    bias: bool = True

    @property
    def head_size(self) -> int:
        return self.n_embd // self.n_head

    def model_dict(self) -> dict:
        return dict(n_layer=self.n_layer, n_head=self.n_head, n_embd=self.n_embd,
                    block_size=self.block_size, vocab_size=self.vocab_size, bias=self.bias,
                    dtype=self.dtype)


@dataclass(frozen=True)
class AttentionWorkload:
    name: str
    batch: int
    n_head: int
    seq_len: int
    head_size: int


WORKLOADS = {
    "tiny": Workload("tiny", 4, 4, 128, 64, 65, 8, 64, "f32", 65),
    "gpt2": Workload("gpt2", 12, 12, 768, 1024, 50304, 12, 1024, "bf16", 50257),
    "gpt2-medium": Workload("gpt2-medium", 24, 16, 1024, 1024, 50304, 8, 1024, "bf16", 50257),
    "gpt2-xl": Workload("gpt2-xl", 48, 25, 1600, 1024, 50304, 4, 1024, "bf16", 50257),
}
ATTENTION = AttentionWorkload("attention", 12, 12, 1024, 64)


def weight_names(n_layer: int) -> list[str]:
    """Names of the model tensors in packed order (the order of the per-tensor seeds)."""
    names = ["wte", "wpe"]
    for l in range(n_layer):
        p = f"h.{l}."
        names += [p + "ln_1.weight", p + "ln_1.bias",
                  p + "attn.c_attn.weight", p + "attn.c_attn.bias",
                  p + "attn.c_proj.weight", p + "attn.c_proj.bias",
                  p + "ln_2.weight", p + "ln_2.bias",
                  p + "mlp.c_fc.weight", p + "mlp.c_fc.bias",
                  p + "mlp.c_proj.weight", p + "mlp.c_proj.bias"]
    names += ["ln_f.weight", "ln_f.bias"]
    return names


def weight_shapes(m: dict) -> dict[str, tuple]:
    C, V, L, bs = m["n_embd"], m["vocab_size"], m["n_layer"], m["block_size"]
    shapes = {"wte": (V, C), "wpe": (bs, C), "ln_f.weight": (C,), "ln_f.bias": (C,)}
    for l in range(L):
        p = f"h.{l}."
        shapes.update({
            p + "ln_1.weight": (C,), p + "ln_1.bias": (C,),
            p + "attn.c_attn.weight": (3 * C, C), p + "attn.c_attn.bias": (3 * C,),
            p + "attn.c_proj.weight": (C, C), p + "attn.c_proj.bias": (C,),
            p + "ln_2.weight": (C,), p + "ln_2.bias": (C,),
            p + "mlp.c_fc.weight": (4 * C, C), p + "mlp.c_fc.bias": (4 * C,),
            p + "mlp.c_proj.weight": (C, 4 * C), p + "mlp.c_proj.bias": (C,),
        })
    return shapes


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_weights(m: dict, seed: int = BASE_SEED, stress: bool = False,
                 device: str = "cpu") -> dict[str, torch.Tensor]:
    """Random GPT weights in the storage dtype of ``m['dtype']`` (fp32 or bf16).

    bf16 weights are fp32 draws rounded once to nearest-even.  ``device='cuda'`` draws
    with the CUDA generator (different numbers, same distribution) for throughput runs
    that need no oracle comparison.
    """
    L = m["n_layer"]
    out_dtype = torch.float32 if m.get("dtype", "f32") == "f32" else torch.bfloat16
    shapes = weight_shapes(m)
    proj_std = 0.02 if stress else 0.02 / math.sqrt(2 * L)
    out = {}
    for k, name in enumerate(weight_names(L)):
        shape = shapes[name]
        g = _gen(seed + k, device)
        if name.endswith("ln_1.weight") or name.endswith("ln_2.weight") or name == "ln_f.weight":
            t = torch.ones(shape, device=device)
            if stress:
                t = t + 0.1 * torch.randn(shape, generator=g, device=device)
        elif name.endswith(".bias"):
            if stress:
                std = 0.1 if ("ln_" in name) else 0.02
                t = std * torch.randn(shape, generator=g, device=device)
            else:
                t = torch.zeros(shape, device=device)
        elif name.endswith("c_proj.weight"):
            t = proj_std * torch.randn(shape, generator=g, device=device)
        else:
            t = 0.02 * torch.randn(shape, generator=g, device=device)
        out[name] = t.to(out_dtype)
    if not m.get("bias", True):
        # bias=False drops every bias, LayerNorm's included (LayerNorm "带可选偏置").
        out = {k: v for k, v in out.items() if not k.endswith(".bias")}
    return out


def make_tokens(batch: int, seq_len: int, high: int, seed: int = BASE_SEED + 100_000,
                ignore_frac: float = 0.0) -> tuple[torch.Tensor, torch.Tensor]:
    """(idx, targets) int64 [B, T], uniform over [0, high).

    ``ignore_frac`` > 0 sets that fraction of target positions (chosen by the same
    seed) to -1, the ignored class.
    """
    g = _gen(seed)
    idx = torch.randint(0, high, (batch, seq_len), generator=g, dtype=torch.int64)
    targets = torch.randint(0, high, (batch, seq_len), generator=g, dtype=torch.int64)
    if ignore_frac > 0:
        drop = torch.rand((batch, seq_len), generator=g) < ignore_frac
        targets = torch.where(drop, torch.full_like(targets, -1), targets)
    return idx, targets


def make_qkv(batch: int, n_head: int, seq_len: int, head_size: int,
             seed: int = BASE_SEED + 200_000, dtype=torch.bfloat16,
             device: str = "cpu") -> tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """q, k, v i.i.d. N(0, 1) in [B, nh, T, hs], rounded to ``dtype``."""
    out = []
    for k in range(3):
        g = _gen(seed + k, device)
        out.append(torch.randn((batch, n_head, seq_len, head_size), generator=g,
                               device=device).to(dtype))
    return tuple(out)


def make_residual(batch: int, seq_len: int, n_embd: int, seed: int = BASE_SEED + 300_000,
                  std: float = 1.0, device: str = "cpu") -> torch.Tensor:
    """fp32 residual-stream input [B, T, C], N(0, std^2), for single-Block checks."""
    g = _gen(seed, device)
    return std * torch.randn((batch, seq_len, n_embd), generator=g, device=device)


def make_uniforms(steps: int, batch: int, seed: int = BASE_SEED + 400_000) -> torch.Tensor:
    """fp32 [steps, B] uniforms in [0, 1): the random numbers of the sampling draws, supplied
    to both implementations."""
    return torch.rand((steps, batch), generator=_gen(seed), dtype=torch.float32)


def make_logits(batch: int, vocab: int, seed: int = BASE_SEED + 500_000, std: float = 2.0,
                ties: int = 0) -> torch.Tensor:
    """fp32 [B, V] logits N(0, std^2) for the sampling step.  ``ties`` > 0 copies the largest
    value of each row onto that many other (seeded) positions, so the top-k threshold has
    ties."""
    g = _gen(seed)
    z = std * torch.randn((batch, vocab), generator=g)
    if ties:
        for b in range(batch):
            pos = torch.randperm(vocab, generator=g)[:ties]
            z[b, pos] = z[b].max()
    return z


def make_grads(m: dict, seed: int = BASE_SEED + 700_000, scale: float = 1e-3) -> dict[str, torch.Tensor]:
    """fp32 gradients N(0, scale^2), one per parameter tensor of ``make_weights(m)`` (biases
    only when m["bias"]), for the optimizer step."""
    shapes = weight_shapes(m)
    names = [n for n in weight_names(m["n_layer"]) if m.get("bias", True) or not n.endswith(".bias")]
    return {n: scale * torch.randn(shapes[n], generator=_gen(seed + k)) for k, n in enumerate(names)}


def to_f64(weights: dict[str, torch.Tensor]):
    """Widen stored weights to fp64 numpy arrays (what the oracle consumes)."""
    return {k: v.to(torch.float64).numpy() for k, v in weights.items()}
