"""B200-native GPT-2 / nanoGPT causal decoder forward pass.

The compute lives in libgptb200.so (hand-written sm_100a CUDA behind the C ABI of
include/gpt.h); this package is its ctypes binding (``native``) plus a small model wrapper
that owns the packed weights and a workspace.  Importing the package loads the library and
raises if it is missing: there is no CPU path.
"""
from __future__ import annotations

import torch

from . import native
from .native import GPTConfig, GPTError  # noqa: F401

__all__ = ["GPT", "GPTConfig", "GPTError", "AdamW", "Trainer", "native"]


class GPT:
    """A model instance: packed device weights + a cached workspace.

    ``model(idx, targets)`` is GPT.forward(idx, targets) of the pages ("nanoGPT 全局流程图",
    §3.2) on device tensors: (logits [B, T, V], loss) with targets, (logits [B, 1, V], None)
    without.  ``forward_host`` takes CPU tensors and returns the loss as a Python float,
    copying inputs in and the result out (the end-to-end call).
    """

    def __init__(self, cfg: GPTConfig, tensors: dict, device="cuda"):
        self.cfg = cfg
        self.device = torch.device(device)
        self.weights = native.pack_weights(cfg, tensors, self.device)
        self._ws = None
        self._ws_bt = None
        self._host = {}

    def workspace(self, B: int, T: int) -> torch.Tensor:
        need = native.workspace_bytes(self.cfg, B, T)
        if need == 0:
            raise native.GPTError(native.GPT_ERR_BAD_SHAPE, "gpt_workspace_bytes")
        if self._ws is None or self._ws.numel() < need:
            self._ws = native.alloc_workspace(need, self.device)
        return self._ws

    def __call__(self, idx, targets=None, **kw):
        B, T = idx.shape
        return native.forward(self.cfg, self.weights, idx, targets, self.workspace(B, T), **kw)

    def block(self, layer: int, x: torch.Tensor, **kw) -> torch.Tensor:
        B, T, _ = x.shape
        return native.block(self.cfg, self.weights, layer, x, self.workspace(B, T), **kw)

    def forward_host(self, idx_cpu: torch.Tensor, targets_cpu: torch.Tensor) -> float:
        """End-to-end: pinned host inputs -> device, forward, loss -> host."""
        B, T = idx_cpu.shape
        key = (B, T)
        if key not in self._host:
            self._host[key] = (torch.empty((B, T), dtype=torch.int64, device=self.device),
                               torch.empty((B, T), dtype=torch.int64, device=self.device),
                               torch.empty((B, T, self.cfg.vocab_size), dtype=self.cfg.torch_dtype,
                                           device=self.device),
                               torch.empty((), dtype=torch.float32, device=self.device),
                               torch.empty((), dtype=torch.float32).pin_memory())
        d_idx, d_tgt, logits, loss, h_loss = self._host[key]
        d_idx.copy_(idx_cpu, non_blocking=True)
        d_tgt.copy_(targets_cpu, non_blocking=True)
        native.forward(self.cfg, self.weights, d_idx, d_tgt, self.workspace(B, T), logits=logits, loss=loss)
        h_loss.copy_(loss, non_blocking=True)
        torch.cuda.current_stream(self.device).synchronize()
        return float(h_loss)

    def generate(self, idx: torch.Tensor, max_new_tokens: int, temperature: float = 1.0,
                 top_k: int | None = None, uniforms: torch.Tensor | None = None,
                 generator: torch.Generator | None = None, step_logits: torch.Tensor | None = None):
        """GPT.generate of the pages ("nanoGPT 全局流程图", 第五阶段) on device tensors: returns
        int64 [B, T0 + max_new_tokens].  The draw of each step uses one uniform per sequence:
        ``uniforms`` fp32 [max_new_tokens, B] in [0, 1) if given, else drawn here with torch
        (from ``generator`` if given); the library itself generates no random numbers."""
        B, T0 = idx.shape
        if uniforms is None:
            uniforms = torch.rand((max_new_tokens, B), generator=generator, device=self.device,
                                  dtype=torch.float32)
        key = ("gen", B)
        if key not in self._host:
            self._host[key] = native.alloc_kv_cache(self.cfg, B, self.device)
        ws = native.alloc_workspace(native.generate_workspace_bytes(self.cfg, B, T0, max_new_tokens), self.device)
        return native.generate(self.cfg, self.weights, idx, max_new_tokens, uniforms, temperature, top_k,
                               kv_cache=self._host[key], workspace=ws, step_logits=step_logits)


class AdamW:
    """Optimizer state for a GPT's packed parameters ("nanoGPT 全局流程图", 3.5 and 3.6,
    优化器配置): fp32 master parameters and both Adam moments as flat device arrays in the packed
    element layout, the schedule of get_lr, clipping to max_grad_norm, weight decay on the
    two-dimensional tensors.  ``step(grads)`` takes a flat fp32 gradient array in the same layout
    and writes the updated parameters into the model's packed weights."""

    def __init__(self, model: GPT, tensors: dict, learning_rate=6e-4, min_lr=6e-5, warmup_iters=2000,
                 lr_decay_iters=600000, betas=(0.9, 0.95), eps=1e-8, weight_decay=0.1, max_grad_norm=1.0):
        self.model = model
        self.params = native.flat_params(model.cfg, tensors, model.device)
        self.exp_avg = torch.zeros_like(self.params)
        self.exp_avg_sq = torch.zeros_like(self.params)
        self.workspace = native.alloc_workspace(native.LIB.gpt_adamw_workspace_bytes(), model.device)
        self.grad_norm = torch.empty((), dtype=torch.float32, device=model.device)
        self.schedule = (learning_rate, min_lr, warmup_iters, lr_decay_iters)
        self.betas, self.eps, self.weight_decay, self.max_grad_norm = betas, eps, weight_decay, max_grad_norm
        self.it = 0

    def step(self, grads: torch.Tensor) -> torch.Tensor:
        lr = native.lr_schedule(self.it, *self.schedule)
        self.it += 1
        return native.adamw_step(self.model.cfg, self.params, grads, self.exp_avg, self.exp_avg_sq, self.it, lr,
                                 weights=self.model.weights, betas=self.betas, eps=self.eps,
                                 weight_decay=self.weight_decay, max_grad_norm=self.max_grad_norm,
                                 grad_norm=self.grad_norm, workspace=self.workspace)


class Trainer:
    """One training step of the pages ("nanoGPT 全局流程图" 3.2-3.6) on a GPT: forward with targets
    keeping activations, the backward into a flat fp32 gradient array, then the AdamW step
    (clipping, schedule, decay on matrices), which also refreshes the model's packed weights.
    ``step(idx, targets)`` returns the batch's loss as a device scalar."""

    def __init__(self, model: GPT, tensors: dict, B: int, T: int, **adamw):
        self.model = model
        self.opt = AdamW(model, tensors, **adamw)
        self.acts, self.fws, self.bws = native.train_buffers(model.cfg, B, T, model.device)
        self.grads = torch.zeros_like(self.opt.params)
        self.loss = torch.empty((), dtype=torch.float32, device=model.device)

    def step(self, idx: torch.Tensor, targets: torch.Tensor) -> torch.Tensor:
        cfg, w = self.model.cfg, self.model.weights
        native.forward_train(cfg, w, idx, targets, self.acts, self.fws, loss=self.loss)
        self.grads.zero_()
        native.backward(cfg, w, idx, targets, self.acts, self.grads, self.bws)
        self.opt.step(self.grads)
        return self.loss

    def step_accumulated(self, micro_batches) -> list:
        """Gradient accumulation ("nanoGPT 全局流程图" 3.7): the gradients of K micro-batches
        [(idx, targets), ...] each scaled by 1/K (the page's loss / gradient_accumulation_steps),
        summed, then one optimizer step.  Returns the micro-batches' losses (device scalars)."""
        cfg, w = self.model.cfg, self.model.weights
        K = len(micro_batches)
        self.grads.zero_()
        losses = []
        for idx, targets in micro_batches:
            loss = torch.empty((), dtype=torch.float32, device=self.model.device)
            native.forward_train(cfg, w, idx, targets, self.acts, self.fws, loss=loss)
            native.backward(cfg, w, idx, targets, self.acts, self.grads, self.bws, loss_scale=1.0 / K)
            losses.append(loss)
        self.opt.step(self.grads)
        return losses

