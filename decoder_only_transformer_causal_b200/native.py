"""ctypes binding of libgptb200.so (include/gpt.h).

Argument marshalling only: every function here checks Python-side types, turns tensors into
raw device pointers and calls the C entry point of the same name.  PyTorch supplies device
memory and streams; all arithmetic runs in the library's CUDA kernels.  There is no fallback:
if the library cannot be loaded, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libgptb200.so")

GPT_OK = 0
GPT_ERR_NULL = -1
GPT_ERR_BAD_SHAPE = -2
GPT_ERR_BAD_ALIGN = -3
GPT_ERR_WS_TOO_SMALL = -4
GPT_ERR_INDEX = -5
GPT_ERR_TIMEOUT = -6
GPT_ERR_UNSUPPORTED = -7
GPT_ERR_CUDA = -8

GPT_DTYPE_F32 = 0
GPT_DTYPE_BF16 = 1
GPT_GELU_ERF = 0
GPT_GELU_TANH = 1
GPT_FLAG_SYNC_CHECK = 1
GPT_EPI_STORE, GPT_EPI_GELU, GPT_EPI_RESID = 0, 1, 2

DTYPES = {"f32": GPT_DTYPE_F32, "bf16": GPT_DTYPE_BF16}
TORCH_DTYPES = {GPT_DTYPE_F32: torch.float32, GPT_DTYPE_BF16: torch.bfloat16}
GELUS = {"erf": GPT_GELU_ERF, "tanh": GPT_GELU_TANH}


class GPTError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {status_string(status)} (status {status})"
        if status == GPT_ERR_CUDA:
            msg += f": {LIB.gpt_last_cuda_error().decode()}"
        super().__init__(msg)


class gpt_config_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("n_layer", "n_head", "n_embd", "block_size", "vocab_size", "bias", "dtype", "gelu")]


class gpt_adamw_t(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("eps", ctypes.c_float), ("weight_decay", ctypes.c_float), ("max_grad_norm", ctypes.c_float),
                ("step", ctypes.c_int32)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python decoder_only_transformer_causal_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, Z, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_int
    L, F = ctypes.c_longlong, ctypes.c_float
    CFG = ctypes.POINTER(gpt_config_t)
    sig = {
        "gpt_status_string": (ctypes.c_char_p, [I]),
        "gpt_abi_version": (I, []),
        "gpt_last_cuda_error": (ctypes.c_char_p, []),
        "gpt_validate_config": (I, [CFG]),
        "gpt_weights_bytes": (Z, [CFG]),
        "gpt_weights_count": (I, [CFG]),
        "gpt_weights_layout": (I, [CFG, P, P, I]),
        "gpt_workspace_bytes": (Z, [CFG, I, I]),
        "gpt_check_status": (I, [P, P]),
        "gpt_set_wait_limit_ns": (I, [ctypes.c_ulonglong, I]),
        "gpt_forward": (I, [CFG, P, P, P, I, I, P, P, P, P, P, Z, P, I]),
        "gpt_block": (I, [CFG, P, I, P, I, I, P, Z, P, I]),
        "gpt_attention": (I, [P, P, P, P, I, I, I, I, D, P, P]),
        "gpt_embed": (I, [P, P, P, P, I, I, I, I, D, P, P]),
        "gpt_layernorm": (I, [P, P, P, P, I, I, D, P]),
        "gpt_linear": (I, [P, P, P, P, I, I, I, D, I, I, P, P]),
        "gpt_lm_head_workspace_bytes": (Z, [I, I]),
        "gpt_lm_head_loss": (I, [P, P, P, I, I, I, D, P, P, P, P, P, Z, P, I]),
        "gpt_lm_head_loss_noalloc": (I, [P, P, P, I, I, I, D, P, P, P, P, P, I]),
        "gpt_lm_head_last": (I, [P, L, P, P, P, I, I, I, D, P, P, P]),
        "gpt_kv_cache_bytes": (Z, [CFG, I]),
        "gpt_decode_workspace_bytes": (Z, [CFG, I, I]),
        "gpt_generate_workspace_bytes": (Z, [CFG, I, I, I]),
        "gpt_prefill": (I, [CFG, P, P, I, I, P, P, P, Z, P, I]),
        "gpt_decode_step": (I, [CFG, P, P, L, I, P, P, P, Z, P, I]),
        "gpt_sample": (I, [P, I, I, F, I, P, P, L, P]),
        "gpt_generate": (I, [CFG, P, P, I, I, I, F, I, P, P, P, P, P, Z, P, I]),
        "gpt_lr_schedule": (ctypes.c_double, [L, ctypes.c_double, ctypes.c_double, L, L]),
        "gpt_param_elems": (Z, [CFG]),
        "gpt_adamw_workspace_bytes": (Z, []),
        "gpt_adamw_step": (I, [CFG, P, P, P, P, P, ctypes.POINTER(gpt_adamw_t), P, P, Z, P, I]),
        "gpt_cross_entropy_backward": (I, [P, P, P, I, I, D, P, P, P]),
        "gpt_layernorm_backward_workspace_bytes": (Z, [I, I]),
        "gpt_layernorm_backward": (I, [P, P, P, I, I, D, P, I, P, P, I, P, Z, P]),
        "gpt_bias_grad_workspace_bytes": (Z, [I, I]),
        "gpt_bias_grad": (I, [P, I, I, D, P, I, P, Z, P]),
        "gpt_gelu_backward": (I, [P, P, L, D, I, P, P]),
        "gpt_embedding_backward_workspace_bytes": (Z, [I, I]),
        "gpt_embedding_backward": (I, [P, P, I, I, I, I, P, P, P, Z, P, P]),
        "gpt_attention_train": (I, [P, P, P, P, P, I, I, I, I, D, P, P]),
        "gpt_attention_backward_workspace_bytes": (Z, [I, I, I]),
        "gpt_linear_backward_workspace_bytes": (Z, [I, I, I, I]),
        "gpt_linear_backward": (I, [P, P, P, I, I, I, I, P, P, P, Z, P, P]),
        "gpt_attention_backward": (I, [P, P, P, P, P, P, P, P, P, I, I, I, I, D, P, Z, P, P]),
        "gpt_transpose": (I, [P, D, L, P, D, L, I, I, P]),
        "gpt_train_activation_bytes": (Z, [CFG, I, I]),
        "gpt_backward_workspace_bytes": (Z, [CFG, I, I]),
        "gpt_forward_train": (I, [CFG, P, P, P, I, I, P, Z, P, P, Z, P, I]),
        "gpt_backward": (I, [CFG, P, P, P, I, I, P, Z, P, F, P, Z, P, I, P]),
        "gpt_grad_buckets": (I, [CFG, P, P, I]),
        "gpt_train_loss_terms_offset": (Z, [CFG, I, I]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


LIB = _load()

EXPORTED = ("gpt_status_string", "gpt_abi_version", "gpt_last_cuda_error", "gpt_validate_config", "gpt_weights_bytes",
            "gpt_weights_count", "gpt_weights_layout", "gpt_workspace_bytes", "gpt_check_status", "gpt_set_wait_limit_ns",
            "gpt_forward", "gpt_block", "gpt_attention", "gpt_embed", "gpt_layernorm", "gpt_linear",
            "gpt_lm_head_workspace_bytes", "gpt_lm_head_loss", "gpt_lm_head_loss_noalloc", "gpt_lm_head_last",
            "gpt_kv_cache_bytes", "gpt_decode_workspace_bytes", "gpt_generate_workspace_bytes", "gpt_prefill",
            "gpt_decode_step", "gpt_sample", "gpt_generate", "gpt_lr_schedule", "gpt_param_elems",
            "gpt_adamw_workspace_bytes", "gpt_adamw_step", "gpt_cross_entropy_backward",
            "gpt_layernorm_backward_workspace_bytes", "gpt_layernorm_backward", "gpt_bias_grad_workspace_bytes",
            "gpt_bias_grad", "gpt_gelu_backward", "gpt_embedding_backward_workspace_bytes", "gpt_embedding_backward",
            "gpt_attention_train", "gpt_attention_backward_workspace_bytes", "gpt_attention_backward", "gpt_transpose",
            "gpt_linear_backward_workspace_bytes", "gpt_linear_backward",
            "gpt_train_activation_bytes", "gpt_backward_workspace_bytes", "gpt_forward_train", "gpt_backward",
            "gpt_grad_buckets", "gpt_train_loss_terms_offset")


def status_string(status: int) -> str:
    return LIB.gpt_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != GPT_OK:
        raise GPTError(status, where)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        if t.numel() and not t.is_contiguous():
            raise ValueError("tensors passed to the library must be contiguous")
        return t.data_ptr() or None
    return int(t)


def _stream(stream) -> int | None:
    if stream is None:
        if torch.cuda.is_available():
            return torch.cuda.current_stream().cuda_stream or None
        return None
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream or None
    return int(stream) or None


@dataclass(frozen=True)
class GPTConfig:
    """GPTConfig of the pages ("nanoGPT 全局流程图", §2.1) plus storage dtype and GELU form."""
    n_layer: int = 12
    n_head: int = 12
    n_embd: int = 768
    block_size: int = 1024
    vocab_size: int = 50304
    bias: bool = True
    dtype: str = "bf16"
    gelu: str = "erf"

    def c(self) -> gpt_config_t:
        return gpt_config_t(self.n_layer, self.n_head, self.n_embd, self.block_size,
                            self.vocab_size, int(bool(self.bias)), DTYPES[self.dtype],
                            GELUS[self.gelu])

    @property
    def torch_dtype(self):
        return TORCH_DTYPES[DTYPES[self.dtype]]

    @classmethod
    def from_dict(cls, d: dict) -> "GPTConfig":
        keys = cls.__dataclass_fields__
        return cls(**{k: v for k, v in d.items() if k in keys})


def packed_names(n_layer: int) -> list[str]:
    """Tensor names in the packed order documented in gpt.h."""
    names = ["wte", "wpe"]
    for l in range(n_layer):
        p = f"h.{l}."
        names += [p + s for s in ("ln_1.weight", "ln_1.bias", "attn.c_attn.weight", "attn.c_attn.bias",
                                  "attn.c_proj.weight", "attn.c_proj.bias", "ln_2.weight", "ln_2.bias",
                                  "mlp.c_fc.weight", "mlp.c_fc.bias", "mlp.c_proj.weight",
                                  "mlp.c_proj.bias")]
    return names + ["ln_f.weight", "ln_f.bias"]


def validate_config(cfg: GPTConfig) -> int:
    return LIB.gpt_validate_config(ctypes.byref(cfg.c()))


def weights_layout(cfg: GPTConfig) -> tuple[list[tuple[str, int, int]], int]:
    """[(name, byte offset, numel)] in packed order, and the buffer size in bytes."""
    c = cfg.c()
    n = LIB.gpt_weights_count(ctypes.byref(c))
    _check(n if n < 0 else GPT_OK, "gpt_weights_count")
    offs = (ctypes.c_size_t * n)()
    nums = (ctypes.c_size_t * n)()
    got = LIB.gpt_weights_layout(ctypes.byref(c), offs, nums, n)
    _check(got if got < 0 else GPT_OK, "gpt_weights_layout")
    total = LIB.gpt_weights_bytes(ctypes.byref(c))
    return [(nm, offs[i], nums[i]) for i, nm in enumerate(packed_names(cfg.n_layer))], total


def pack_weights(cfg: GPTConfig, tensors: dict, device="cuda") -> torch.Tensor:
    """Copies named parameter tensors into one packed device buffer (bias slots stay zero
    when absent or when cfg.bias is False)."""
    entries, total = weights_layout(cfg)
    buf = torch.zeros(total, dtype=torch.uint8, device=device)
    dt = cfg.torch_dtype
    for name, off, numel in entries:
        t = tensors.get(name)
        if t is None:
            if name.endswith(".bias"):
                continue
            raise KeyError(name)
        if t.numel() != numel:
            raise ValueError(f"{name}: {t.numel()} elements, layout expects {numel}")
        esz = torch.finfo(dt).bits // 8
        buf[off:off + numel * esz].view(dt).copy_(t.reshape(-1).to(dt))
    return buf


def workspace_bytes(cfg: GPTConfig, B: int, T: int) -> int:
    return LIB.gpt_workspace_bytes(ctypes.byref(cfg.c()), B, T)


def alloc_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def check_status(workspace: torch.Tensor, stream=None) -> int:
    return LIB.gpt_check_status(_ptr(workspace), _stream(stream))


def set_wait_limit_ns(ns: int, force_timeout: bool = False) -> None:
    """gpt_set_wait_limit_ns: the pipeline-wait limit of the tensor-core kernels on the current
    device (0 restores the default) and the forced time-out; a testing aid for the time-out path."""
    _check(LIB.gpt_set_wait_limit_ns(int(ns), int(bool(force_timeout))), "gpt_set_wait_limit_ns")


def forward(cfg: GPTConfig, weights: torch.Tensor, idx: torch.Tensor, targets: torch.Tensor | None,
            workspace: torch.Tensor, logits: torch.Tensor | None = None, loss: torch.Tensor | None = None,
            row_loss: torch.Tensor | None = None, loss_sum_count: torch.Tensor | None = None,
            stream=None, sync_check: bool = False):
    """gpt_forward.  Returns (logits, loss) device tensors (loss None without targets)."""
    B, T = idx.shape
    dt = cfg.torch_dtype
    if logits is None:
        shape = (B, T, cfg.vocab_size) if targets is not None else (B, 1, cfg.vocab_size)
        logits = torch.empty(shape, dtype=dt, device=idx.device)
    if targets is not None and loss is None:
        loss = torch.empty((), dtype=torch.float32, device=idx.device)
    rc = LIB.gpt_forward(ctypes.byref(cfg.c()), _ptr(weights), _ptr(idx), _ptr(targets), B, T,
                         _ptr(logits), _ptr(loss) if targets is not None else None, _ptr(row_loss),
                         _ptr(loss_sum_count), _ptr(workspace), workspace.numel(), _stream(stream),
                         GPT_FLAG_SYNC_CHECK if sync_check else 0)
    _check(rc, "gpt_forward")
    return logits, (loss if targets is not None else None)


def block(cfg: GPTConfig, weights: torch.Tensor, layer: int, x: torch.Tensor, workspace: torch.Tensor,
          stream=None, sync_check: bool = False) -> torch.Tensor:
    B, T, _ = x.shape
    rc = LIB.gpt_block(ctypes.byref(cfg.c()), _ptr(weights), layer, _ptr(x), B, T, _ptr(workspace),
                       workspace.numel(), _stream(stream), GPT_FLAG_SYNC_CHECK if sync_check else 0)
    _check(rc, "gpt_block")
    return x


def attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, y: torch.Tensor | None = None,
              status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    B, nh, T, hs = q.shape
    dtype = {torch.bfloat16: GPT_DTYPE_BF16, torch.float32: GPT_DTYPE_F32}[q.dtype]
    if y is None:
        y = torch.empty_like(q)
    rc = LIB.gpt_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(y), B, nh, T, hs, dtype, _ptr(status),
                           _stream(stream))
    _check(rc, "gpt_attention")
    return y


def embed(wte, wpe, idx, x=None, status=None, stream=None):
    B, T = idx.shape
    V, C = wte.shape
    dtype = {torch.bfloat16: GPT_DTYPE_BF16, torch.float32: GPT_DTYPE_F32}[wte.dtype]
    if x is None:
        x = torch.empty((B, T, C), dtype=torch.float32, device=idx.device)
    _check(LIB.gpt_embed(_ptr(wte), _ptr(wpe), _ptr(idx), _ptr(x), B, T, C, V, dtype, _ptr(status),
                         _stream(stream)), "gpt_embed")
    return x


def layernorm(x, w, b=None, out=None, stream=None):
    C = x.shape[-1]
    rows = x.numel() // C
    dtype = {torch.bfloat16: GPT_DTYPE_BF16, torch.float32: GPT_DTYPE_F32}[w.dtype]
    if out is None:
        out = torch.empty(x.shape, dtype=w.dtype, device=x.device)
    _check(LIB.gpt_layernorm(_ptr(x), _ptr(w), _ptr(b), _ptr(out), rows, C, dtype, _stream(stream)),
           "gpt_layernorm")
    return out


def linear(x, W, b=None, out=None, epilogue=GPT_EPI_STORE, gelu=GPT_GELU_ERF, status=None, stream=None):
    M, K = x.shape
    N = W.shape[0]
    dtype = {torch.bfloat16: GPT_DTYPE_BF16, torch.float32: GPT_DTYPE_F32}[x.dtype]
    if out is None:
        odt = torch.float32 if epilogue == GPT_EPI_RESID else x.dtype
        out = torch.zeros((M, N), dtype=odt, device=x.device)
    _check(LIB.gpt_linear(_ptr(x), _ptr(W), _ptr(b), _ptr(out), M, N, K, dtype, epilogue, gelu,
                          _ptr(status), _stream(stream)), "gpt_linear")
    return out


def lm_head_last(x: torch.Tensor, lnf_w: torch.Tensor, lnf_b: torch.Tensor | None, wte: torch.Tensor,
                 logits: torch.Tensor | None = None, status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """gpt_lm_head_last: ln_f and the tied head of the last position of each sequence.  x is the
    fp32 residual stream [B, T, C] (only row T-1 of each sequence is read) or [B, C]; returns
    logits [B, V] in wte's dtype."""
    if x.dtype != torch.float32 or not x.is_contiguous():
        raise ValueError("x must be a contiguous float32 tensor")
    if x.dim() == 3:
        B, T, C = x.shape
        base, ldx = x[:, T - 1].data_ptr(), T * C
    else:
        B, C = x.shape
        base, ldx = x.data_ptr(), C
    V = wte.shape[0]
    if logits is None:
        logits = torch.empty((B, V), dtype=wte.dtype, device=x.device)
    _check(LIB.gpt_lm_head_last(base, ldx, _ptr(lnf_w), _ptr(lnf_b), _ptr(wte), B, C, V, _dt(wte), _ptr(logits),
                                _ptr(status), _stream(stream)), "gpt_lm_head_last")
    return logits


def lm_head_workspace_bytes(rows: int, V: int) -> int:
    return LIB.gpt_lm_head_workspace_bytes(rows, V)


def lm_head_loss_noalloc(u, wte, targets, logits=None, loss=None, row_loss=None, loss_sum_count=None,
                         stream=None, sync_check=False):
    """gpt_lm_head_loss_noalloc: the head and loss with the library's static scratch (no
    workspace); for callers that cannot allocate device memory at this point."""
    rows, C = u.shape
    V = wte.shape[0]
    dtype = {torch.bfloat16: GPT_DTYPE_BF16, torch.float32: GPT_DTYPE_F32}[u.dtype]
    if logits is None:
        logits = torch.empty((rows, V), dtype=u.dtype, device=u.device)
    if loss is None:
        loss = torch.empty((), dtype=torch.float32, device=u.device)
    _check(LIB.gpt_lm_head_loss_noalloc(_ptr(u), _ptr(wte), _ptr(targets), rows, C, V, dtype, _ptr(logits),
                                        _ptr(loss), _ptr(row_loss), _ptr(loss_sum_count), _stream(stream),
                                        GPT_FLAG_SYNC_CHECK if sync_check else 0), "gpt_lm_head_loss_noalloc")
    return logits, loss


def lm_head_loss(u, wte, targets, workspace=None, logits=None, loss=None, row_loss=None,
                 loss_sum_count=None, stream=None, sync_check=False):
    rows, C = u.shape
    V = wte.shape[0]
    dtype = {torch.bfloat16: GPT_DTYPE_BF16, torch.float32: GPT_DTYPE_F32}[u.dtype]
    if workspace is None:
        workspace = alloc_workspace(lm_head_workspace_bytes(rows, V), u.device)
    if logits is None:
        logits = torch.empty((rows, V), dtype=u.dtype, device=u.device)
    if loss is None:
        loss = torch.empty((), dtype=torch.float32, device=u.device)
    _check(LIB.gpt_lm_head_loss(_ptr(u), _ptr(wte), _ptr(targets), rows, C, V, dtype, _ptr(logits),
                                _ptr(loss), _ptr(row_loss), _ptr(loss_sum_count), _ptr(workspace),
                                workspace.numel(), _stream(stream),
                                GPT_FLAG_SYNC_CHECK if sync_check else 0), "gpt_lm_head_loss")
    return logits, loss


# ---------------------------------------------------------------- generation
def kv_cache_bytes(cfg: GPTConfig, B: int) -> int:
    return LIB.gpt_kv_cache_bytes(ctypes.byref(cfg.c()), B)


def decode_workspace_bytes(cfg: GPTConfig, B: int, T_prefill: int) -> int:
    return LIB.gpt_decode_workspace_bytes(ctypes.byref(cfg.c()), B, T_prefill)


def generate_workspace_bytes(cfg: GPTConfig, B: int, T0: int, max_new_tokens: int) -> int:
    return LIB.gpt_generate_workspace_bytes(ctypes.byref(cfg.c()), B, T0, max_new_tokens)


def alloc_kv_cache(cfg: GPTConfig, B: int, device="cuda") -> torch.Tensor:
    n = kv_cache_bytes(cfg, B)
    if n == 0:
        raise GPTError(GPT_ERR_UNSUPPORTED, "gpt_kv_cache_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device)


def prefill(cfg: GPTConfig, weights: torch.Tensor, idx: torch.Tensor, kv_cache: torch.Tensor,
            workspace: torch.Tensor, logits: torch.Tensor | None = None, stream=None, sync_check=False):
    """gpt_prefill: fills the cache for idx [B, T]; returns the last position's logits fp32 [B, V]."""
    B, T = idx.shape
    if logits is None:
        logits = torch.empty((B, cfg.vocab_size), dtype=torch.float32, device=idx.device)
    _check(LIB.gpt_prefill(ctypes.byref(cfg.c()), _ptr(weights), _ptr(idx), B, T, _ptr(kv_cache), _ptr(logits),
                           _ptr(workspace), workspace.numel(), _stream(stream),
                           GPT_FLAG_SYNC_CHECK if sync_check else 0), "gpt_prefill")
    return logits


def decode_step(cfg: GPTConfig, weights: torch.Tensor, tok: torch.Tensor, kv_cache: torch.Tensor,
                workspace: torch.Tensor, logits: torch.Tensor | None = None, stream=None, sync_check=False):
    """gpt_decode_step: tok int64 [B] (a strided column view is allowed); returns logits fp32 [B, V]."""
    if tok.dim() != 1:
        raise ValueError("tok must be 1-D [B]")
    B = tok.shape[0]
    if logits is None:
        logits = torch.empty((B, cfg.vocab_size), dtype=torch.float32, device=tok.device)
    _check(LIB.gpt_decode_step(ctypes.byref(cfg.c()), _ptr(weights), tok.data_ptr(), tok.stride(0), B,
                               _ptr(kv_cache), _ptr(logits), _ptr(workspace), workspace.numel(), _stream(stream),
                               GPT_FLAG_SYNC_CHECK if sync_check else 0), "gpt_decode_step")
    return logits


def sample(logits: torch.Tensor, u: torch.Tensor, temperature: float = 1.0, top_k: int | None = None,
           out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """gpt_sample: logits fp32 [B, V], u fp32 [B] in [0, 1); returns int64 [B] (or writes the
    strided 1-D view `out`)."""
    B, V = logits.shape
    if out is None:
        out = torch.empty(B, dtype=torch.int64, device=logits.device)
    _check(LIB.gpt_sample(_ptr(logits), B, V, float(temperature), int(top_k or 0), _ptr(u), out.data_ptr(),
                          out.stride(0), _stream(stream)), "gpt_sample")
    return out


def generate(cfg: GPTConfig, weights: torch.Tensor, idx: torch.Tensor, max_new_tokens: int, uniforms: torch.Tensor,
             temperature: float = 1.0, top_k: int | None = None, kv_cache: torch.Tensor | None = None,
             workspace: torch.Tensor | None = None, step_logits: torch.Tensor | None = None, out=None,
             stream=None, sync_check=False) -> torch.Tensor:
    """gpt_generate: idx int64 [B, T0]; uniforms fp32 [max_new_tokens, B]; returns
    int64 [B, T0 + max_new_tokens]."""
    B, T0 = idx.shape
    if uniforms.shape != (max_new_tokens, B) or uniforms.dtype != torch.float32:
        raise ValueError("uniforms must be float32 [max_new_tokens, B]")
    if kv_cache is None:
        kv_cache = alloc_kv_cache(cfg, B, idx.device)
    if workspace is None:
        workspace = alloc_workspace(generate_workspace_bytes(cfg, B, T0, max_new_tokens), idx.device)
    if out is None:
        out = torch.empty((B, T0 + max_new_tokens), dtype=torch.int64, device=idx.device)
    _check(LIB.gpt_generate(ctypes.byref(cfg.c()), _ptr(weights), _ptr(idx), B, T0, max_new_tokens,
                            float(temperature), int(top_k or 0), _ptr(uniforms), _ptr(out), _ptr(step_logits),
                            _ptr(kv_cache), _ptr(workspace), workspace.numel(), _stream(stream),
                            GPT_FLAG_SYNC_CHECK if sync_check else 0), "gpt_generate")
    return out


# ---------------------------------------------------------------- optimizer step
def lr_schedule(it: int, learning_rate: float = 6e-4, min_lr: float = 6e-5, warmup_iters: int = 2000,
                lr_decay_iters: int = 600000) -> float:
    """gpt_lr_schedule: get_lr(it) of the pages (host function)."""
    return LIB.gpt_lr_schedule(int(it), float(learning_rate), float(min_lr), int(warmup_iters), int(lr_decay_iters))


def param_elems(cfg: GPTConfig) -> int:
    return LIB.gpt_param_elems(ctypes.byref(cfg.c()))


def flat_params(cfg: GPTConfig, tensors: dict, device="cuda") -> torch.Tensor:
    """fp32 [param_elems] in the packed element layout (tensor i at byte offset / element size);
    absent tensors (biases when cfg.bias is False) and the padding stay zero."""
    entries, _ = weights_layout(cfg)
    es = 2 if cfg.dtype == "bf16" else 4
    buf = torch.zeros(param_elems(cfg), dtype=torch.float32, device=device)
    for name, off, numel in entries:
        t = tensors.get(name)
        if t is None:
            continue
        buf[off // es: off // es + numel].copy_(t.reshape(-1).to(torch.float32))
    return buf


def unflatten(cfg: GPTConfig, flat: torch.Tensor, shapes: dict) -> dict:
    """Views of a flat fp32 array per tensor name (names in `shapes` only)."""
    entries, _ = weights_layout(cfg)
    es = 2 if cfg.dtype == "bf16" else 4
    return {name: flat[off // es: off // es + numel].view(shapes[name])
            for name, off, numel in entries if name in shapes}


def adamw_step(cfg: GPTConfig, params: torch.Tensor, grads: torch.Tensor, exp_avg: torch.Tensor,
               exp_avg_sq: torch.Tensor, step: int, lr: float, weights: torch.Tensor | None = None,
               betas=(0.9, 0.95), eps: float = 1e-8, weight_decay: float = 0.1, max_grad_norm: float = 1.0,
               grad_norm: torch.Tensor | None = None, workspace: torch.Tensor | None = None, stream=None,
               sync_check=False):
    """gpt_adamw_step on flat fp32 arrays; returns the device grad-norm tensor."""
    if workspace is None:
        workspace = alloc_workspace(LIB.gpt_adamw_workspace_bytes(), params.device)
    if grad_norm is None:
        grad_norm = torch.empty((), dtype=torch.float32, device=params.device)
    hp = gpt_adamw_t(float(lr), float(betas[0]), float(betas[1]), float(eps), float(weight_decay),
                     float(max_grad_norm), int(step))
    _check(LIB.gpt_adamw_step(ctypes.byref(cfg.c()), _ptr(params), _ptr(grads), _ptr(exp_avg), _ptr(exp_avg_sq),
                              _ptr(weights), ctypes.byref(hp), _ptr(grad_norm), _ptr(workspace), workspace.numel(),
                              _stream(stream), GPT_FLAG_SYNC_CHECK if sync_check else 0), "gpt_adamw_step")
    return grad_norm


# ---------------------------------------------------------------- backward pieces
def _dt(t: torch.Tensor) -> int:
    return {torch.bfloat16: GPT_DTYPE_BF16, torch.float32: GPT_DTYPE_F32}[t.dtype]


def cross_entropy_backward(logits: torch.Tensor, targets: torch.Tensor, loss_sum_count: torch.Tensor,
                           dlogits: torch.Tensor | None = None, status=None, stream=None) -> torch.Tensor:
    """gpt_cross_entropy_backward: logits [rows, V] (bf16 or fp32), targets int64 [rows],
    loss_sum_count fp64 [2] from the forward."""
    V = logits.shape[-1]
    rows = logits.numel() // V
    if dlogits is None:
        dlogits = torch.empty_like(logits)
    _check(LIB.gpt_cross_entropy_backward(_ptr(logits), _ptr(targets), _ptr(loss_sum_count), rows, V, _dt(logits),
                                          _ptr(dlogits), _ptr(status), _stream(stream)), "gpt_cross_entropy_backward")
    return dlogits


def layernorm_backward(dy: torch.Tensor, x: torch.Tensor, w: torch.Tensor, dx: torch.Tensor | None = None,
                       accumulate=False, dw=None, db=None, accumulate_wb=False, stream=None):
    """gpt_layernorm_backward: dy, x fp32 [rows, C]; w [C] bf16/fp32; returns (dx, dw, db)."""
    C = x.shape[-1]
    rows = x.numel() // C
    if dx is None:
        dx = torch.empty_like(x)
    if dw is None:
        dw = torch.empty(C, dtype=torch.float32, device=x.device)
    ws = alloc_workspace(LIB.gpt_layernorm_backward_workspace_bytes(rows, C), x.device)
    _check(LIB.gpt_layernorm_backward(_ptr(dy), _ptr(x), _ptr(w), rows, C, _dt(w), _ptr(dx), int(accumulate),
                                      _ptr(dw), _ptr(db), int(accumulate_wb), _ptr(ws), ws.numel(), _stream(stream)),
           "gpt_layernorm_backward")
    return dx, dw, db


def bias_grad(dy: torch.Tensor, db: torch.Tensor | None = None, accumulate=False, stream=None) -> torch.Tensor:
    C = dy.shape[-1]
    rows = dy.numel() // C
    if db is None:
        db = torch.empty(C, dtype=torch.float32, device=dy.device)
    ws = alloc_workspace(LIB.gpt_bias_grad_workspace_bytes(rows, C), dy.device)
    _check(LIB.gpt_bias_grad(_ptr(dy), rows, C, _dt(dy), _ptr(db), int(accumulate), _ptr(ws), ws.numel(),
                             _stream(stream)), "gpt_bias_grad")
    return db


def gelu_backward(dh: torch.Tensor, pre: torch.Tensor, gelu=GPT_GELU_ERF, dpre=None, stream=None) -> torch.Tensor:
    if dpre is None:
        dpre = torch.empty_like(pre)
    _check(LIB.gpt_gelu_backward(_ptr(dh), _ptr(pre), pre.numel(), _dt(pre), gelu, _ptr(dpre), _stream(stream)),
           "gpt_gelu_backward")
    return dpre


def embedding_backward(idx: torch.Tensor, dx: torch.Tensor, dwte: torch.Tensor, dwpe: torch.Tensor, status=None,
                       stream=None):
    """gpt_embedding_backward: adds into dwte [V, C] and dwpe [>= T, C] (fp32)."""
    B, T = idx.shape
    C = dx.shape[-1]
    ws = alloc_workspace(LIB.gpt_embedding_backward_workspace_bytes(B, T), dx.device)
    _check(LIB.gpt_embedding_backward(_ptr(idx), _ptr(dx), B, T, C, dwte.shape[0], _ptr(dwte), _ptr(dwpe), _ptr(ws),
                                      ws.numel(), _ptr(status), _stream(stream)), "gpt_embedding_backward")
    return dwte, dwpe


def attention_train(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, status=None, stream=None):
    """gpt_attention_train: returns (y, lse) for q, k, v [B, nh, T, hs]."""
    B, nh, T, hs = q.shape
    y = torch.empty_like(q)
    lse = torch.empty((B, nh, T), dtype=torch.float32, device=q.device)
    _check(LIB.gpt_attention_train(_ptr(q), _ptr(k), _ptr(v), _ptr(y), _ptr(lse), B, nh, T, hs, _dt(q), _ptr(status),
                                   _stream(stream)), "gpt_attention_train")
    return y, lse


def attention_backward(q, k, v, o, dout, lse, stream=None, out=None, workspace=None, status=None):
    """gpt_attention_backward: returns (dq, dk, dv) for [B, nh, T, hs] tensors (into `out`, a
    (dq, dk, dv) triple, and `workspace` when given; `status`: optional device int32)."""
    B, nh, T, hs = q.shape
    dq, dk, dv = out if out is not None else (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    ws = workspace if workspace is not None else alloc_workspace(
        LIB.gpt_attention_backward_workspace_bytes(B, nh, T), q.device)
    _check(LIB.gpt_attention_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                                      _ptr(dv), B, nh, T, hs, _dt(q), _ptr(ws), ws.numel(), _ptr(status),
                                      _stream(stream)),
           "gpt_attention_backward")
    return dq, dk, dv


def linear_backward(dy, x, W, dW=None, status=None, stream=None):
    """gpt_linear_backward: returns (dx fp32, dW fp32); dW is accumulated into when given."""
    rows, n_out = dy.shape
    n_in = x.shape[1]
    dx = torch.empty((rows, n_in), dtype=torch.float32, device=dy.device)
    if dW is None:
        dW = torch.zeros((n_out, n_in), dtype=torch.float32, device=dy.device)
    ws = alloc_workspace(LIB.gpt_linear_backward_workspace_bytes(max(rows, 1), n_out, n_in, _dt(dy)), dy.device)
    _check(LIB.gpt_linear_backward(_ptr(dy), _ptr(x), _ptr(W), rows, n_out, n_in, _dt(dy), _ptr(dx), _ptr(dW), _ptr(ws),
                                   ws.numel(), _ptr(status) if status is not None else None, _stream(stream)),
           "gpt_linear_backward")
    return dx, dW


def transpose(x: torch.Tensor, out_dtype=None, stream=None) -> torch.Tensor:
    """gpt_transpose of a 2-D tensor (optionally converting bf16 <-> fp32)."""
    R, Cc = x.shape
    out = torch.empty((Cc, R), dtype=out_dtype or x.dtype, device=x.device)
    _check(LIB.gpt_transpose(_ptr(x), _dt(x), Cc, _ptr(out), _dt(out), R, R, Cc, _stream(stream)), "gpt_transpose")
    return out


# ---------------------------------------------------------------- training step
def train_buffers(cfg: GPTConfig, B: int, T: int, device="cuda"):
    """(acts, forward workspace, backward workspace) for gpt_forward_train / gpt_backward."""
    c = ctypes.byref(cfg.c())
    na, nb = LIB.gpt_train_activation_bytes(c, B, T), LIB.gpt_backward_workspace_bytes(c, B, T)
    if na == 0 or nb == 0:
        raise GPTError(GPT_ERR_BAD_SHAPE, "gpt_train_activation_bytes")
    return (alloc_workspace(na, device), alloc_workspace(workspace_bytes(cfg, B, T), device),
            alloc_workspace(nb, device))


def forward_train(cfg, weights, idx, targets, acts, workspace, loss=None, stream=None, sync_check=False):
    B, T = idx.shape
    if loss is None:
        loss = torch.empty((), dtype=torch.float32, device=idx.device)
    _check(LIB.gpt_forward_train(ctypes.byref(cfg.c()), _ptr(weights), _ptr(idx), _ptr(targets), B, T, _ptr(acts),
                                 acts.numel(), _ptr(loss), _ptr(workspace), workspace.numel(), _stream(stream),
                                 GPT_FLAG_SYNC_CHECK if sync_check else 0), "gpt_forward_train")
    return loss


def backward(cfg, weights, idx, targets, acts, grads, workspace, loss_scale=1.0, stream=None, sync_check=False,
             bucket_events=None):
    """gpt_backward: adds loss_scale * the gradients into grads (fp32 [param_elems]).  bucket_events:
    optional list of n_layer + 1 torch.cuda.Event (already recorded once, so that the CUDA event
    exists); event i is recorded when gradient bucket i (grad_buckets) is complete."""
    B, T = idx.shape
    evs = None
    if bucket_events is not None:
        if len(bucket_events) != cfg.n_layer + 1:
            raise ValueError("bucket_events needs n_layer + 1 events")
        handles = [e.cuda_event for e in bucket_events]
        if not all(handles):
            raise ValueError("record each event once before passing it (its CUDA event is created then)")
        evs = (ctypes.c_void_p * len(handles))(*handles)
    _check(LIB.gpt_backward(ctypes.byref(cfg.c()), _ptr(weights), _ptr(idx), _ptr(targets), B, T, _ptr(acts),
                            acts.numel(), _ptr(grads), float(loss_scale), _ptr(workspace), workspace.numel(),
                            _stream(stream), GPT_FLAG_SYNC_CHECK if sync_check else 0, evs), "gpt_backward")
    return grads


def grad_buckets(cfg) -> list[tuple[int, int]]:
    """gpt_grad_buckets: the [start, stop) element ranges of the flat gradient array in the order the
    backward completes them (layer n_layer - 1 with ln_f first, ..., layer 0, then wte and wpe)."""
    n = LIB.gpt_grad_buckets(ctypes.byref(cfg.c()), None, None, 0)
    _check(n if n < 0 else GPT_OK, "gpt_grad_buckets")
    a, b = (ctypes.c_size_t * n)(), (ctypes.c_size_t * n)()
    LIB.gpt_grad_buckets(ctypes.byref(cfg.c()), a, b, n)
    return [(int(a[i]), int(b[i])) for i in range(n)]


def loss_terms(cfg, acts: torch.Tensor, B: int, T: int) -> torch.Tensor:
    """The fp64 {sum of row losses, counted rows} pair inside acts (a view: all-reduce it in place
    before gpt_backward for a data-parallel step)."""
    off = LIB.gpt_train_loss_terms_offset(ctypes.byref(cfg.c()), B, T)
    return acts[off: off + 16].view(torch.float64)

