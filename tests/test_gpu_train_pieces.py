"""Pieces of the training step through the C ABI: the attention's per-row log-sum-exp (from
gpt_attention_train), the attention backward (gpt_attention_backward) against the oracle's
derivative, and the transpose / conversion used to form the backward products' operands."""
import math

import numpy as np
import pytest
import torch

import oracle.backward as ob
import seeded
from gpu_helpers import f64, needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]


def rel_close(got, want, rtol, atol_scale, floor=1e-6):
    """|got - want| <= rtol |want| + atol_scale * max(max|want|, floor).  The floor covers results
    whose exact value is 0 (T = 1: O = v makes dp - D vanish), where only rounding residue is left."""
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    bound = rtol * np.abs(want) + atol_scale * max(float(np.abs(want).max()), floor)
    return not (np.abs(got - want) > bound).any(), float(np.abs(got - want).max())


# bf16 with hs 64 runs the tensor-core kernels (128-row outer tiles, 64-row inner tiles): T = 1,
# 64, 129 (one row in the last outer tile), 300 and 2048 cover single, ragged and many-tile sweeps;
# fp32 (hs 32 and 64) runs the SIMT kernels.
@pytest.mark.parametrize("B,nh,T,hs,dtype", [(2, 3, 300, 64, torch.bfloat16), (1, 2, 1024, 64, torch.bfloat16),
                                             (2, 4, 77, 32, torch.float32), (1, 1, 1, 64, torch.bfloat16),
                                             (3, 2, 130, 64, torch.float32), (3, 5, 129, 64, torch.bfloat16),
                                             (2, 2, 64, 64, torch.bfloat16), (1, 5, 2048, 64, torch.bfloat16)])
def test_attention_lse_and_backward(B, nh, T, hs, dtype):
    from decoder_only_transformer_causal_b200 import native
    q, k, v = seeded.make_qkv(B, nh, T, hs, dtype=dtype)
    dout = (torch.randn(B, nh, T, hs, generator=torch.Generator().manual_seed(17)) * 0.1).to(dtype)
    qd, kd, vd, gd = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    y, lse = native.attention_train(qd, kd, vd)
    # lse: log2 of sum_j exp(q_i . k_j / sqrt(hs)) over j <= i
    s = np.einsum("bhid,bhjd->bhij", f64(q), f64(k)) / math.sqrt(hs)
    s = np.where(np.tril(np.ones((T, T), bool)), s, -np.inf)
    m = s.max(-1)
    ref_lse = (m + np.log(np.exp(s - m[..., None]).sum(-1))) / math.log(2.0)
    assert np.abs(f64(lse) - ref_lse).max() < (2e-3 if dtype == torch.bfloat16 else 1e-5)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dq, dk, dv = native.attention_backward(qd, kd, vd, y, gd, lse, status=status)
    dq2, dk2, dv2 = native.attention_backward(qd, kd, vd, y, gd, lse, status=status)
    assert torch.equal(dq, dq2) and torch.equal(dk, dk2) and torch.equal(dv, dv2)
    assert int(status) == native.GPT_OK  # no pipeline wait expired
    rdq, rdk, rdv = ob.attention_backward(f64(dout), f64(q), f64(k), f64(v))
    # bf16: inputs, the forward output o and the results are bf16 (2^-9 relative each); the
    # recomputed probabilities use the bf16-path lse; fp32: accumulation order only
    rtol, atol = (3e-2, 1e-2) if dtype == torch.bfloat16 else (1e-4, 1e-5)
    for name, got, ref in (("dq", dq, rdq), ("dk", dk, rdk), ("dv", dv, rdv)):
        ok, err = rel_close(f64(got), ref, rtol, atol)
        assert ok, (name, err)


def test_attention_backward_unaligned_operands_use_simt_kernels():
    """A q whose address is 2 bytes off a 16-byte boundary cannot be described by a TMA map: the
    bf16 / hs 64 call then runs the SIMT kernels and must still match the oracle."""
    from decoder_only_transformer_causal_b200 import native
    B, nh, T, hs = 1, 2, 200, 64
    q, k, v = seeded.make_qkv(B, nh, T, hs, dtype=torch.bfloat16)
    dout = (torch.randn(B, nh, T, hs, generator=torch.Generator().manual_seed(3)) * 0.1).to(torch.bfloat16)
    buf = torch.empty(q.numel() + 1, dtype=torch.bfloat16, device="cuda")
    qd = buf[1:].view(B, nh, T, hs)
    qd.copy_(q.cuda())
    assert qd.data_ptr() % 16 != 0
    y, lse = native.attention_train(q.cuda(), k.cuda(), v.cuda())
    dq, dk, dv = native.attention_backward(qd, k.cuda(), v.cuda(), y, dout.cuda(), lse)
    rdq, rdk, rdv = ob.attention_backward(f64(dout), f64(q), f64(k), f64(v))
    for name, got, ref in (("dq", dq, rdq), ("dk", dk, rdk), ("dv", dv, rdv)):
        ok, err = rel_close(f64(got), ref, 3e-2, 1e-2)
        assert ok, (name, err)


@pytest.mark.parametrize("R,Cc,din,dout_", [(12288, 768, torch.bfloat16, torch.bfloat16), (77, 33, torch.float32, torch.bfloat16),
                                            (5, 1000, torch.bfloat16, torch.float32), (64, 64, torch.float32, torch.float32)])
def test_transpose(R, Cc, din, dout_):
    from decoder_only_transformer_causal_b200 import native
    x = torch.randn(R, Cc, generator=torch.Generator().manual_seed(R)).to(din).cuda()
    t = native.transpose(x, dout_)
    assert torch.equal(t, x.t().to(dout_))


# (rows, n_out, n_in): the four Linear shapes of a GPT-2 block at a small row count, plus ragged
# rows (the K tail of dW's product) and column counts that leave partial 128 / 256-wide tiles.
@pytest.mark.parametrize("rows,n_out,n_in,dtype", [(1000, 2304, 768, torch.bfloat16), (777, 768, 3072, torch.bfloat16),
                                                   (130, 72, 200, torch.bfloat16), (64, 1024, 40, torch.bfloat16),
                                                   (77, 40, 24, torch.float32), (300, 96, 130, torch.float32)])
def test_linear_backward(rows, n_out, n_in, dtype):
    from decoder_only_transformer_causal_b200 import native
    g = torch.Generator().manual_seed(rows + n_out)
    dy = (torch.randn(rows, n_out, generator=g) * 0.05).to(dtype)
    x = torch.randn(rows, n_in, generator=g).to(dtype)
    W = (torch.randn(n_out, n_in, generator=g) * 0.02).to(dtype)
    base = torch.randn(n_out, n_in, generator=g) * 0.01
    dx, dW = native.linear_backward(dy.cuda(), x.cuda(), W.cuda(), dW=base.clone().cuda())
    rdx, rdW, _ = ob.linear_backward(f64(dy), f64(x), f64(W))
    # operands are exact in both; only the fp32 accumulation order differs
    ok, err = rel_close(f64(dx), rdx, 1e-3, 1e-4)
    assert ok, ("dx", err)
    ok, err = rel_close(f64(dW) - f64(base), rdW, 1e-3, 1e-4)
    assert ok, ("dW", err)
    dx2, dW2 = native.linear_backward(dy.cuda(), x.cuda(), W.cuda(), dW=base.clone().cuda())
    assert torch.equal(dx, dx2) and torch.equal(dW, dW2)
