"""Causal attention through the C ABI (gpt_attention) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import seeded
from gpu_helpers import BF16_ATOL, f64, max_abs, needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]


def run(q, k, v):
    from decoder_only_transformer_causal_b200 import native
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = native.attention(q.cuda(), k.cuda(), v.cuda(), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return y


def test_attention_full_size():
    """B 12, 12 heads, T 1024, hs 64, q/k/v N(0,1) bf16: every output element."""
    w = seeded.ATTENTION
    q, k, v = seeded.make_qkv(w.batch, w.n_head, w.seq_len, w.head_size)
    y = run(q, k, v)
    ref = oracle.causal_attention(f64(q), f64(k), f64(v))
    err = max_abs(f64(y), ref)
    assert err <= BF16_ATOL, err


@pytest.mark.parametrize("B,nh,T", [(1, 1, 1), (1, 2, 7), (1, 2, 63), (2, 3, 65), (1, 1, 128),
                                    (1, 2, 129), (2, 2, 257), (1, 1, 640), (1, 1, 1000)])
def test_attention_shapes(B, nh, T):
    q, k, v = seeded.make_qkv(B, nh, T, 64, seed=1000 + T)
    y = run(q, k, v)
    err = max_abs(f64(y), oracle.causal_attention(f64(q), f64(k), f64(v)))
    assert err <= BF16_ATOL, err


def test_attention_T1_is_v_exactly():
    q, k, v = seeded.make_qkv(3, 4, 1, 64)
    assert torch.equal(run(q, k, v).cpu(), v)


def test_attention_first_row_is_v0_and_v_ones():
    q, k, v = seeded.make_qkv(2, 2, 300, 64)
    y = run(q, k, v).cpu()
    assert torch.equal(y[:, :, 0], v[:, :, 0])
    ones = torch.ones_like(v)
    y1 = run(q, k, ones).cpu().float()
    assert float((y1 - 1).abs().max()) <= 4e-3


def test_attention_q_zero_prefix_mean():
    q, k, v = seeded.make_qkv(1, 2, 200, 64)
    y = run(torch.zeros_like(q), k, v).cpu()
    vv = f64(v)
    ref = np.cumsum(vv, axis=2) / np.arange(1, 201)[None, None, :, None]
    assert max_abs(f64(y), ref) <= BF16_ATOL


def test_attention_causality_bit_exact():
    q, k, v = seeded.make_qkv(1, 2, 384, 64)
    y = run(q, k, v).cpu()
    for t in (0, 100, 127, 128, 255, 300):
        k2, v2 = k.clone(), v.clone()
        k2[:, :, t + 1:] = -k2[:, :, t + 1:] * 3
        v2[:, :, t + 1:] = v2[:, :, t + 1:] + 1
        y2 = run(q, k2, v2).cpu()
        assert torch.equal(y2[:, :, :t + 1], y[:, :, :t + 1]), t


@pytest.mark.parametrize("hs,T", [(32, 64), (64, 130), (16, 5), (128, 33)])
def test_attention_f32(hs, T):
    q, k, v = seeded.make_qkv(2, 3, T, hs, dtype=torch.float32)
    y = run(q, k, v)
    err = max_abs(f64(y), oracle.causal_attention(f64(q), f64(k), f64(v)))
    assert err <= 1e-5, err
