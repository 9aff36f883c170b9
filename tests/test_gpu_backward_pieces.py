"""The backward kernels of the non-matrix-product steps (cross-entropy, LayerNorm, GELU, bias,
embedding) through the C ABI against the oracle's derivatives (oracle/backward.py) on seeded
inputs, at the GPT-2 124M shapes and on ragged small ones; each run twice to check that the
results are bit-identical (every reduction runs in a fixed order)."""
import numpy as np
import pytest
import torch

import oracle.backward as ob
import seeded
from gpu_helpers import f64, needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]


def rel_close(got, want, rtol, atol_scale):
    """|got - want| <= rtol |want| + atol_scale * max|want| (rounding of sums that cancel scales
    with the largest term, not with the entry)."""
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    bound = rtol * np.abs(want) + atol_scale * float(np.abs(want).max())
    bad = np.abs(got - want) > bound
    return not bad.any(), float(np.abs(got - want).max())


@pytest.mark.parametrize("rows,V,dtype", [(96, 50304, torch.bfloat16), (37, 65, torch.float32),
                                          (2048, 50304, torch.bfloat16), (5, 1000, torch.float32)])
def test_cross_entropy_backward(rows, V, dtype):
    from decoder_only_transformer_causal_b200 import native
    z = seeded.make_logits(rows, V, std=1.5).to(dtype)
    _, tgt = seeded.make_tokens(1, rows, V, seed=4321, ignore_frac=0.2)
    tgt = tgt.reshape(-1)
    n = int((tgt != -1).sum())
    sc = torch.tensor([0.0, float(n)], dtype=torch.float64, device="cuda")
    dz = native.cross_entropy_backward(z.cuda(), tgt.cuda(), sc)
    dz2 = native.cross_entropy_backward(z.cuda(), tgt.cuda(), sc)
    assert torch.equal(dz, dz2)
    ref = ob.cross_entropy_backward(f64(z), tgt.numpy())
    # bf16 output: one rounding (2^-9 relative); fp32: exp/log intrinsics (~1e-6 relative)
    rtol = 8e-3 if dtype == torch.bfloat16 else 1e-5
    ok, err = rel_close(f64(dz), ref, rtol, 1e-6)
    assert ok, err
    assert np.all(f64(dz)[tgt.numpy() == -1] == 0.0)


@pytest.mark.parametrize("rows,C,wdtype", [(12288, 768, torch.bfloat16), (37, 128, torch.float32),
                                           (300, 1600, torch.bfloat16)])
def test_layernorm_backward(rows, C, wdtype):
    from decoder_only_transformer_causal_b200 import native
    g = torch.Generator().manual_seed(rows + C)
    x = torch.randn(rows, C, generator=g) * 2 + 0.5
    dy = torch.randn(rows, C, generator=g) * 0.01
    w = (1 + 0.1 * torch.randn(C, generator=g)).to(wdtype)
    base = torch.randn(rows, C, generator=g) * 0.001          # accumulate into an existing gradient
    dx = base.clone().cuda()
    db = torch.empty(C, device="cuda")
    _, dw, _ = native.layernorm_backward(dy.cuda(), x.cuda(), w.cuda(), dx=dx, accumulate=True, db=db)
    rdx, rdw, rdb = ob.layer_norm_backward(f64(dy), f64(x), f64(w))
    ok, err = rel_close(f64(dx) - f64(base), rdx, 1e-4, 1e-5)
    assert ok, ("dx", err)
    ok, err = rel_close(f64(dw), rdw, 1e-4, 1e-5)
    assert ok, ("dw", err)
    ok, err = rel_close(f64(db), rdb, 1e-4, 1e-5)
    assert ok, ("db", err)
    dx2 = base.clone().cuda()
    _, dw2, _ = native.layernorm_backward(dy.cuda(), x.cuda(), w.cuda(), dx=dx2, accumulate=True)
    assert torch.equal(dx, dx2) and torch.equal(dw, dw2)


@pytest.mark.parametrize("rows,C,dtype", [(12288, 3072, torch.bfloat16), (12288, 768, torch.float32),
                                          (300, 768, torch.float32), (129, 65, torch.float32),
                                          (77, 65, torch.bfloat16), (1, 100, torch.bfloat16),
                                          (40, 8200, torch.bfloat16), (33, 4100, torch.float32)])
def test_bias_grad(rows, C, dtype):
    """Vector loads or, where C is not a multiple of the vector width, element loads; widths past
    one CTA's column span; one row; a repeat must give the identical sums."""
    from decoder_only_transformer_causal_b200 import native
    dy = (torch.randn(rows, C, generator=torch.Generator().manual_seed(7)) * 0.01).to(dtype)
    start = torch.full((C,), 0.25, device="cuda")
    db = native.bias_grad(dy.cuda(), db=start.clone(), accumulate=True)
    ok, err = rel_close(f64(db) - 0.25, f64(dy).sum(axis=0), 1e-4, 1e-5)
    assert ok, err
    assert torch.equal(db, native.bias_grad(dy.cuda(), db=start.clone(), accumulate=True))


@pytest.mark.parametrize("gelu", ["erf", "tanh"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_gelu_backward(gelu, dtype):
    from decoder_only_transformer_causal_b200 import native
    g = torch.Generator().manual_seed(11)
    pre = (torch.randn(4097, 33, generator=g) * 2).to(dtype)
    dh = torch.randn(4097, 33, generator=g)
    mode = native.GPT_GELU_TANH if gelu == "tanh" else native.GPT_GELU_ERF
    dpre = native.gelu_backward(dh.cuda(), pre.cuda(), mode)
    ref = ob.gelu_backward(f64(dh), f64(pre), gelu)
    rtol = 8e-3 if dtype == torch.bfloat16 else 2e-6
    ok, err = rel_close(f64(dpre), ref, rtol, 1e-6)
    assert ok, err


@pytest.mark.parametrize("B,T,C,V", [(12, 1024, 768, 50304), (3, 17, 128, 65), (2, 5, 64, 3)])
def test_embedding_backward(B, T, C, V):
    from decoder_only_transformer_causal_b200 import native
    idx, _ = seeded.make_tokens(B, T, V, seed=99)
    if V == 3:
        idx[:] = 1                                             # one long run of the same token
    dx = torch.randn(B, T, C, generator=torch.Generator().manual_seed(5)) * 0.01
    dwte = torch.full((V, C), 0.5, device="cuda")
    dwpe = torch.full((T + 3, C), -0.5, device="cuda")
    native.embedding_backward(idx.cuda(), dx.cuda(), dwte, dwpe)
    rwte, rwpe = ob.embed_backward(f64(dx), idx.numpy(), V, T + 3)
    ok, err = rel_close(f64(dwte) - 0.5, rwte, 1e-5, 1e-6)
    assert ok, err
    ok, err = rel_close(f64(dwpe) + 0.5, rwpe, 1e-5, 1e-6)
    assert ok, err
    w2 = torch.full((V, C), 0.5, device="cuda")
    p2 = torch.full((T + 3, C), -0.5, device="cuda")
    native.embedding_backward(idx.cuda(), dx.cuda(), w2, p2)
    assert torch.equal(dwte, w2) and torch.equal(dwpe, p2)


def test_embedding_backward_bad_token_is_reported():
    from decoder_only_transformer_causal_b200 import native
    idx = torch.tensor([[0, 7, 2]], dtype=torch.int64)
    dx = torch.ones(1, 3, 4)
    dwte = torch.zeros(5, 4, device="cuda")
    dwpe = torch.zeros(3, 4, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    native.embedding_backward(idx.cuda(), dx.cuda(), dwte, dwpe, status=status)
    torch.cuda.synchronize()
    assert int(status) == native.GPT_ERR_INDEX
    assert float(dwte[0].sum()) == 4.0 and float(dwte[2].sum()) == 4.0 and float(dwte.sum()) == 8.0
