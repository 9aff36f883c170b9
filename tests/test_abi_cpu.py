"""Host-side checks of the C ABI that need no GPU: the library loads, exports every function
include/gpt.h declares, and rejects bad arguments on the host before anything is enqueued."""
import ctypes
import os
import re

import pytest

import oracle
import seeded
from decoder_only_transformer_causal_b200 import native
from decoder_only_transformer_causal_b200.native import GPTConfig

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "gpt.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gpt_\w+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert len(names) >= 16
    lib = ctypes.CDLL(native.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(native.EXPORTED)


def test_abi_version_and_status_strings():
    assert native.LIB.gpt_abi_version() == 1
    for code in range(-8, 1):
        s = native.status_string(code)
        assert s and s != "unknown status"
    assert native.status_string(-99) == "unknown status"


def _cfg(name, **kw):
    return GPTConfig.from_dict(dict(seeded.WORKLOADS[name].model_dict(), **kw))


@pytest.mark.parametrize("name", sorted(seeded.WORKLOADS))
def test_presets_validate(name):
    assert native.validate_config(_cfg(name)) == native.GPT_OK


def test_validate_rejects():
    assert native.validate_config(_cfg("gpt2", n_head=7)) == native.GPT_ERR_BAD_SHAPE      # C % nh
    assert native.validate_config(_cfg("gpt2", n_head=24)) == native.GPT_ERR_UNSUPPORTED   # bf16 hs 32
    assert native.validate_config(_cfg("tiny", n_head=8)) == native.GPT_OK                 # fp32 hs 16
    assert native.validate_config(_cfg("gpt2", n_layer=-1)) == native.GPT_ERR_BAD_SHAPE
    bad = native.gpt_config_t(1, 1, 64, 8, 10, 1, 5, 0)
    assert native.LIB.gpt_validate_config(ctypes.byref(bad)) == native.GPT_ERR_BAD_SHAPE
    assert native.LIB.gpt_validate_config(None) == native.GPT_ERR_NULL


@pytest.mark.parametrize("name", sorted(seeded.WORKLOADS))
def test_weights_layout_counts(name):
    cfg = _cfg(name)
    entries, total = native.weights_layout(cfg)
    # every parameter exactly once (tied head): the element count is get_num_params
    assert sum(n for _, _, n in entries) == oracle.num_params(seeded.WORKLOADS[name].model_dict(), False)
    offs = [o for _, o, _ in entries]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    esz = 2 if cfg.dtype == "bf16" else 4
    last_name, last_off, last_n = entries[-1]
    assert total >= last_off + last_n * esz
    shapes = seeded.weight_shapes(seeded.WORKLOADS[name].model_dict())
    for nm, _, n in entries:
        numel = 1
        for d in shapes[nm]:
            numel *= d
        assert numel == n, nm


def test_workspace_bytes():
    cfg = _cfg("gpt2")
    ws = native.workspace_bytes(cfg, 12, 1024)
    N, C = 12 * 1024, 768
    # x fp32 + ln out + qkv + y + h (bf16) at least
    assert ws >= N * C * 4 + N * C * 2 * (1 + 3 + 1 + 4)
    assert native.workspace_bytes(cfg, 12, 1025) == 0       # T > block_size
    assert native.workspace_bytes(cfg, 0, 16) == 0
    assert native.lm_head_workspace_bytes(12288, 50304) > 12288 * 4


FAKE = 1 << 20  # an aligned non-null address; the calls below must fail before using it


def _fwd(cfg, B, T, weights=FAKE, ws=FAKE, ws_bytes=1 << 40, logits=FAKE, idx=FAKE):
    return native.LIB.gpt_forward(ctypes.byref(cfg.c()), weights, idx, None, B, T, logits, None, None,
                                  None, ws, ws_bytes, None, 0)


def test_forward_host_validation():
    cfg = _cfg("gpt2")
    assert _fwd(cfg, 2, 1025) == native.GPT_ERR_BAD_SHAPE        # T > block_size
    assert _fwd(cfg, 0, 16) == native.GPT_ERR_BAD_SHAPE
    assert _fwd(cfg, 2, 16, weights=None) == native.GPT_ERR_NULL
    assert _fwd(cfg, 2, 16, idx=None) == native.GPT_ERR_NULL
    assert _fwd(cfg, 2, 16, weights=FAKE + 8) == native.GPT_ERR_BAD_ALIGN
    assert _fwd(cfg, 2, 16, ws_bytes=1024) == native.GPT_ERR_WS_TOO_SMALL
    assert _fwd(_cfg("gpt2", n_head=24), 2, 16) == native.GPT_ERR_UNSUPPORTED
    rc = native.LIB.gpt_block(ctypes.byref(cfg.c()), FAKE, 12, FAKE, 1, 8, FAKE, 1 << 40, None, 0)
    assert rc == native.GPT_ERR_BAD_SHAPE                          # layer out of range


def test_kernel_entry_validation():
    L = native.LIB
    assert L.gpt_attention(FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 32, native.GPT_DTYPE_BF16, None, None) \
        == native.GPT_ERR_UNSUPPORTED                              # bf16 needs hs 64
    assert L.gpt_attention(FAKE, FAKE, FAKE, FAKE + 4, 1, 1, 8, 64, native.GPT_DTYPE_BF16, None, None) \
        == native.GPT_ERR_BAD_ALIGN
    assert L.gpt_attention(None, FAKE, FAKE, FAKE, 1, 1, 8, 64, native.GPT_DTYPE_BF16, None, None) \
        == native.GPT_ERR_NULL
    assert L.gpt_linear(FAKE, FAKE, None, FAKE, 8, 12, 64, native.GPT_DTYPE_BF16, 0, 0, None, None) \
        == native.GPT_ERR_UNSUPPORTED                              # N % 8
    assert L.gpt_linear(FAKE, FAKE, None, FAKE, 8, 16, 64, native.GPT_DTYPE_BF16, 9, 0, None, None) \
        == native.GPT_ERR_BAD_SHAPE
    assert L.gpt_layernorm(FAKE, FAKE, None, FAKE, 4, 6, native.GPT_DTYPE_F32, None) == native.GPT_ERR_BAD_SHAPE
    assert L.gpt_embed(FAKE, FAKE, FAKE, FAKE, 1, 1, 6, 10, native.GPT_DTYPE_F32, None, None) \
        == native.GPT_ERR_BAD_SHAPE
    assert L.gpt_lm_head_loss(FAKE, FAKE, FAKE, 4, 64, 128, native.GPT_DTYPE_BF16, FAKE, None, None, None,
                              FAKE, 16, None, 0) == native.GPT_ERR_WS_TOO_SMALL
    assert L.gpt_check_status(None, None) == native.GPT_ERR_NULL
    bf = native.GPT_DTYPE_BF16
    assert L.gpt_lm_head_last(None, 768, FAKE, None, FAKE, 4, 768, 50304, bf, FAKE, None, None) == native.GPT_ERR_NULL
    assert L.gpt_lm_head_last(FAKE, 100, FAKE, None, FAKE, 4, 768, 50304, bf, FAKE, None, None) \
        == native.GPT_ERR_BAD_SHAPE                                # ldx < C
    assert L.gpt_lm_head_last(FAKE, 776, FAKE, None, FAKE, 4, 772, 50304, bf, FAKE, None, None) \
        == native.GPT_ERR_UNSUPPORTED                              # C % 8
    assert L.gpt_lm_head_last(FAKE, 4096, FAKE, None, FAKE, 16, 4096, 50304, bf, FAKE, None, None) \
        == native.GPT_ERR_UNSUPPORTED                              # 16 staged rows of 4096 exceed shared memory
    assert L.gpt_lm_head_last(FAKE + 4, 768, FAKE, None, FAKE, 4, 768, 50304, bf, FAKE, None, None) \
        == native.GPT_ERR_BAD_ALIGN
    assert L.gpt_lm_head_last(FAKE, 770, FAKE, None, FAKE, 4, 768, 50304, bf, FAKE, None, None) \
        == native.GPT_ERR_BAD_ALIGN                                # row stride not a multiple of 16 bytes


def test_generation_sizes():
    cfg = _cfg("gpt2")
    L, B, bs, C = 12, 4, 1024, 768
    assert native.kv_cache_bytes(cfg, B) == L * B * bs * 2 * C * 2
    assert native.kv_cache_bytes(_cfg("tiny"), 2) == 4 * 2 * 64 * 2 * 128 * 4
    assert native.kv_cache_bytes(cfg, 0) == 0
    d1 = native.decode_workspace_bytes(cfg, B, 1)
    assert d1 >= native.workspace_bytes(cfg, B, 1) + B * 50304 * 4
    assert native.decode_workspace_bytes(cfg, B, 1025) == 0
    # generate: a sequence that outgrows the window needs a full-window prefill
    assert native.generate_workspace_bytes(cfg, B, 8, 100) == native.decode_workspace_bytes(cfg, B, 8)
    assert native.generate_workspace_bytes(cfg, B, 1000, 100) == native.decode_workspace_bytes(cfg, B, 1024)
    assert native.generate_workspace_bytes(cfg, B, 2000, 0) == native.decode_workspace_bytes(cfg, B, 1024)
    assert native.generate_workspace_bytes(_cfg("gpt2", n_embd=772, n_head=4), B, 8, 1) == 0   # hs 193


def test_generation_host_validation():
    Lb = native.LIB
    cfg = _cfg("gpt2")
    c = ctypes.byref(cfg.c())
    big = 1 << 40
    # gpt_sample: temperature must be positive and finite; pointers non-null
    assert Lb.gpt_sample(FAKE, 2, 100, 0.0, 0, FAKE, FAKE, 1, None) == native.GPT_ERR_BAD_SHAPE
    assert Lb.gpt_sample(FAKE, 2, 100, -1.0, 0, FAKE, FAKE, 1, None) == native.GPT_ERR_BAD_SHAPE
    assert Lb.gpt_sample(FAKE, 2, 100, float("inf"), 0, FAKE, FAKE, 1, None) == native.GPT_ERR_BAD_SHAPE
    assert Lb.gpt_sample(FAKE, 2, 100, 1.0, 0, None, FAKE, 1, None) == native.GPT_ERR_NULL
    assert Lb.gpt_sample(FAKE, 0, 100, 1.0, 0, FAKE, FAKE, 1, None) == native.GPT_ERR_BAD_SHAPE
    # gpt_prefill / gpt_decode_step
    assert Lb.gpt_prefill(c, FAKE, FAKE, 2, 1025, FAKE, FAKE, FAKE, big, None, 0) == native.GPT_ERR_BAD_SHAPE
    assert Lb.gpt_prefill(c, FAKE, FAKE, 2, 16, None, FAKE, FAKE, big, None, 0) == native.GPT_ERR_NULL
    assert Lb.gpt_prefill(c, FAKE, FAKE, 2, 16, FAKE, FAKE, FAKE, 4096, None, 0) == native.GPT_ERR_WS_TOO_SMALL
    assert Lb.gpt_prefill(c, FAKE, FAKE, 2, 16, FAKE + 8, FAKE, FAKE, big, None, 0) == native.GPT_ERR_BAD_ALIGN
    assert Lb.gpt_decode_step(c, FAKE, None, 1, 2, FAKE, FAKE, FAKE, big, None, 0) == native.GPT_ERR_NULL
    assert Lb.gpt_decode_step(c, FAKE, FAKE, 1, 0, FAKE, FAKE, FAKE, big, None, 0) == native.GPT_ERR_BAD_SHAPE
    assert Lb.gpt_decode_step(c, FAKE, FAKE, 1, 2, FAKE, FAKE + 4, FAKE, big, None, 0) == native.GPT_ERR_BAD_ALIGN
    # gpt_generate
    gen = lambda **k: Lb.gpt_generate(c, k.get("w", FAKE), k.get("idx", FAKE), k.get("B", 2), k.get("T0", 8),
                                      k.get("n", 4), k.get("temp", 1.0), 0, k.get("u", FAKE), FAKE, None,
                                      FAKE, FAKE, k.get("ws", big), None, 0)
    assert gen(u=None) == native.GPT_ERR_NULL
    assert gen(temp=0.0) == native.GPT_ERR_BAD_SHAPE
    assert gen(n=-1) == native.GPT_ERR_BAD_SHAPE
    assert gen(T0=0) == native.GPT_ERR_BAD_SHAPE
    assert gen(ws=4096) == native.GPT_ERR_WS_TOO_SMALL
    assert gen(w=FAKE + 16) == native.GPT_ERR_BAD_ALIGN
    # an unsupported head size for the decode kernels
    c2 = ctypes.byref(_cfg("tiny", n_head=32).c())                                   # hs 4
    assert Lb.gpt_prefill(c2, FAKE, FAKE, 1, 4, FAKE, FAKE, FAKE, big, None, 0) == native.GPT_ERR_UNSUPPORTED


def test_sample_vocab_limit():
    Lb = native.LIB
    assert Lb.gpt_sample(FAKE, 2, 53248 + 1, 1.0, 0, FAKE, FAKE, 1, None) == native.GPT_ERR_UNSUPPORTED
    c = ctypes.byref(_cfg("gpt2", vocab_size=60000).c())
    assert Lb.gpt_generate(c, FAKE, FAKE, 1, 4, 2, 1.0, 0, FAKE, FAKE, None, FAKE, FAKE, 1 << 40, None, 0) \
        == native.GPT_ERR_UNSUPPORTED


def test_lr_schedule_matches_oracle():
    import oracle.optim as oo
    for it in (0, 1, 999, 1999, 2000, 2001, 123456, 301000, 599999, 600000, 600001, 10 ** 7):
        assert native.lr_schedule(it) == pytest.approx(oo.lr_at(it), rel=1e-14, abs=0)
    assert native.lr_schedule(5, 1.0, 0.1, 10, 100) == pytest.approx(oo.lr_at(5, 1.0, 0.1, 10, 100), rel=1e-14)


def test_adamw_host_validation():
    Lb = native.LIB
    cfg = _cfg("gpt2")
    c = ctypes.byref(cfg.c())
    assert native.param_elems(cfg) == native.LIB.gpt_weights_bytes(c) // 2
    ws = Lb.gpt_adamw_workspace_bytes()
    ok = dict(lr=6e-4, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1, max_grad_norm=1.0, step=1)

    def call(ws_bytes=ws, params=FAKE, weights=None, **kw):
        hp = native.gpt_adamw_t(**dict(ok, **kw))
        return Lb.gpt_adamw_step(c, params, FAKE, FAKE, FAKE, weights, ctypes.byref(hp), None, FAKE, ws_bytes,
                                 None, 0)
    assert call(step=0) == native.GPT_ERR_BAD_SHAPE
    assert call(lr=-1.0) == native.GPT_ERR_BAD_SHAPE
    assert call(lr=float("nan")) == native.GPT_ERR_BAD_SHAPE
    assert call(beta1=1.0) == native.GPT_ERR_BAD_SHAPE
    assert call(eps=0.0) == native.GPT_ERR_BAD_SHAPE
    assert call(weight_decay=-0.1) == native.GPT_ERR_BAD_SHAPE
    assert call(ws_bytes=16) == native.GPT_ERR_WS_TOO_SMALL
    assert call(params=None) == native.GPT_ERR_NULL
    assert call(params=FAKE + 4) == native.GPT_ERR_BAD_ALIGN
    assert call(weights=FAKE + 16) == native.GPT_ERR_BAD_ALIGN
    hp = native.gpt_adamw_t(**ok)
    big = ctypes.byref(_cfg("tiny", n_layer=90).c())                                  # > 1024 tensors
    assert Lb.gpt_adamw_step(big, FAKE, FAKE, FAKE, FAKE, None, ctypes.byref(hp), None, FAKE, ws, None, 0) \
        == native.GPT_ERR_UNSUPPORTED


def test_backward_pieces_host_validation():
    Lb = native.LIB
    bf, f32 = native.GPT_DTYPE_BF16, native.GPT_DTYPE_F32
    assert Lb.gpt_cross_entropy_backward(None, FAKE, FAKE, 4, 10, bf, FAKE, None, None) == native.GPT_ERR_NULL
    assert Lb.gpt_cross_entropy_backward(FAKE, FAKE, FAKE, 4, 0, bf, FAKE, None, None) == native.GPT_ERR_BAD_SHAPE
    assert Lb.gpt_cross_entropy_backward(FAKE, FAKE, FAKE, 4, 10, 7, FAKE, None, None) == native.GPT_ERR_BAD_SHAPE
    ws = Lb.gpt_layernorm_backward_workspace_bytes(100, 768)
    assert ws >= ((100 + 31) // 32) * 2 * 768 * 4                                   # one partial per 32 rows
    assert Lb.gpt_layernorm_backward(FAKE, FAKE, FAKE, 100, 768, bf, FAKE, 0, FAKE, None, 0, FAKE, ws - 1, None) \
        == native.GPT_ERR_WS_TOO_SMALL
    assert Lb.gpt_layernorm_backward(FAKE, FAKE, FAKE, 100, 5000, bf, FAKE, 0, FAKE, None, 0, FAKE, 1 << 40, None) \
        == native.GPT_ERR_BAD_SHAPE
    assert Lb.gpt_bias_grad(FAKE, 10, 8, f32, None, 0, FAKE, 1 << 20, None) == native.GPT_ERR_NULL
    assert Lb.gpt_gelu_backward(FAKE, FAKE, 10, bf, 5, FAKE, None) == native.GPT_ERR_BAD_SHAPE
    assert Lb.gpt_embedding_backward_workspace_bytes(16, 1025) == 0                   # > 16384 positions
    assert Lb.gpt_embedding_backward(FAKE, FAKE, 16, 1025, 8, 10, FAKE, FAKE, FAKE, 1 << 30, None, None) \
        == native.GPT_ERR_UNSUPPORTED


def test_training_products_host_validation():
    """Workspace sizes and argument checks of the Linear and attention backward entry points
    (all return before touching a device)."""
    Lb = native.LIB
    bf, f32 = native.GPT_DTYPE_BF16, native.GPT_DTYPE_F32
    # attention backward: D and the negated lse, both padded to 128 rows per (b, h)
    for B, nh, T in ((12, 12, 1024), (2, 3, 300), (1, 1, 1)):
        tp = (T + 127) // 128 * 128
        assert Lb.gpt_attention_backward_workspace_bytes(B, nh, T) == (2 * B * nh * tp * 4 + 255) // 256 * 256
    assert Lb.gpt_attention_backward_workspace_bytes(0, 1, 1) == 0
    assert Lb.gpt_attention_backward(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 48, bf, FAKE,
                                     1 << 20, None, None) == native.GPT_ERR_UNSUPPORTED       # hs 48
    assert Lb.gpt_attention_backward(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 64, bf, FAKE,
                                     16, None, None) == native.GPT_ERR_WS_TOO_SMALL
    assert Lb.gpt_attention_backward(None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 64, bf, FAKE,
                                     1 << 20, None, None) == native.GPT_ERR_NULL
    # Linear backward: bf16 needs room for the split-K partials of narrow weight gradients
    # (GPT-2's attn c_proj: 768 x 768 over 12,288 rows splits its K range), fp32 for the transposes
    ws_split = Lb.gpt_linear_backward_workspace_bytes(12288, 768, 768, bf)
    assert ws_split > 256 and (ws_split - 256) % (768 * 768 * 4) == 0
    assert Lb.gpt_linear_backward_workspace_bytes(12288, 50304, 768, bf) == 256      # the head: enough tiles
    r, o, i = 77, 40, 24
    a = lambda n: (n + 255) // 256 * 256
    assert Lb.gpt_linear_backward_workspace_bytes(r, o, i, f32) == 256 + a(i * o * 4) + a(o * r * 4) + a(i * r * 4)
    assert Lb.gpt_linear_backward_workspace_bytes(0, 8, 8, bf) == 0
    assert Lb.gpt_linear_backward_workspace_bytes(8, 8, 8, 7) == 0
    ws = 1 << 20
    assert Lb.gpt_linear_backward(None, FAKE, FAKE, 8, 8, 8, bf, FAKE, FAKE, FAKE, ws, None, None) == native.GPT_ERR_NULL
    assert Lb.gpt_linear_backward(FAKE, FAKE, FAKE, 8, 0, 8, bf, FAKE, FAKE, FAKE, ws, None, None) \
        == native.GPT_ERR_BAD_SHAPE
    assert Lb.gpt_linear_backward(FAKE, FAKE, FAKE, 8, 12, 8, bf, FAKE, FAKE, FAKE, ws, None, None) \
        == native.GPT_ERR_UNSUPPORTED                                                     # n_out % 8
    assert Lb.gpt_linear_backward(FAKE, FAKE, FAKE, 64, 64, 64, f32, FAKE, FAKE, FAKE, 16, None, None) \
        == native.GPT_ERR_WS_TOO_SMALL
    assert Lb.gpt_linear_backward(FAKE, FAKE, FAKE, 0, 8, 8, bf, FAKE, FAKE, FAKE, ws, None, None) == native.GPT_OK
