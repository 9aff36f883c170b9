"""Single kernels of the forward pass through the C ABI against the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
import seeded
from gpu_helpers import BF16_ATOL, F32_ATOL, LOSS_RTOL, f64, max_abs, needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]


def gen(shape, std=1.0, seed=0, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    return (std * torch.randn(shape, generator=g)).to(dtype)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("rows,C", [(1, 128), (37, 768), (1000, 1024), (3, 1600), (8, 2048)])
def test_layernorm(dtype, rows, C):
    from decoder_only_transformer_causal_b200 import native
    x = gen((rows, C), 2.0, 1, torch.float32) + 0.5
    w = gen((C,), 0.3, 2, dtype) + 1
    b = gen((C,), 0.1, 3, dtype)
    out = native.layernorm(x.cuda(), w.cuda(), b.cuda())
    ref = oracle.layer_norm(f64(x), f64(w), f64(b))
    tol = BF16_ATOL if dtype == torch.bfloat16 else 2e-5
    assert max_abs(f64(out), ref) <= tol


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_embed(dtype):
    from decoder_only_transformer_causal_b200 import native
    V, C, bs, B, T = 1000, 768, 64, 3, 50
    wte, wpe = gen((V, C), 0.02, 4, dtype), gen((bs, C), 0.02, 5, dtype)
    idx, _ = seeded.make_tokens(B, T, V)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    x = native.embed(wte.cuda(), wpe.cuda(), idx.cuda(), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert max_abs(f64(x), oracle.embed(f64(wte), f64(wpe), idx.numpy())) <= 1e-7


def test_embed_bad_index_sets_status():
    from decoder_only_transformer_causal_b200 import native
    V, C = 100, 128
    wte, wpe = gen((V, C), 0.02, 4), gen((8, C), 0.02, 5)
    idx = torch.tensor([[3, 100, -1, 7]])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    x = native.embed(wte.cuda(), wpe.cuda(), idx.cuda(), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == native.GPT_ERR_INDEX
    assert torch.isfinite(x).all()


SHAPES = [(128, 256, 64), (300, 200, 136), (1000, 768, 768), (64, 2304, 768), (129, 1600, 1600),
          (257, 4800, 1600), (2048, 3072, 768), (512, 768, 3072)]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("epi", ["store", "gelu_erf", "gelu_tanh", "resid"])
def test_linear_bf16(M, N, K, epi):
    from decoder_only_transformer_causal_b200 import native
    x = gen((M, K), 1.0, 6)
    W = gen((N, K), 1.0 / math.sqrt(K), 7)
    b = gen((N,), 0.1, 8)
    ref = oracle.linear(f64(x), f64(W), f64(b))
    if epi == "resid":
        base = gen((M, N), 1.0, 9, torch.float32)
        out = native.linear(x.cuda(), W.cuda(), b.cuda(), out=base.clone().cuda(), epilogue=native.GPT_EPI_RESID)
        ref = ref + f64(base)
        tol = 1e-3
    elif epi == "store":
        out = native.linear(x.cuda(), W.cuda(), b.cuda())
        tol = BF16_ATOL
    else:
        mode = epi.split("_")[1]
        out = native.linear(x.cuda(), W.cuda(), b.cuda(), epilogue=native.GPT_EPI_GELU,
                            gelu=native.GELUS[mode])
        ref = oracle.gelu(ref, mode)
        tol = BF16_ATOL
    torch.cuda.synchronize()
    err = max_abs(f64(out), ref)
    assert err <= tol, err


def test_linear_bf16_gelu_wide_range():
    """Pre-activations spread over about [-60, 60]: the erf-form GELU epilogue must give x for large
    x and 0 for large negative x (its polynomial's argument is clamped) and stay within bf16's
    relative step everywhere."""
    from decoder_only_transformer_causal_b200 import native
    M, N, K = 512, 512, 64
    x = gen((M, K), 1.0, 16)
    W = gen((N, K), 20.0 / math.sqrt(K), 17)
    b = gen((N,), 1.0, 18)
    ref = oracle.gelu(oracle.linear(f64(x), f64(W), f64(b)), "erf")
    out = native.linear(x.cuda(), W.cuda(), b.cuda(), epilogue=native.GPT_EPI_GELU, gelu=native.GELUS["erf"])
    torch.cuda.synchronize()
    got = f64(out)
    assert float(np.abs(ref).max()) > 40.0
    err = np.abs(got - ref)
    assert float((err - (4e-3 * np.abs(ref) + 1e-4)).max()) <= 0.0, float(err.max())


@pytest.mark.parametrize("M,N,K", [(64, 96, 40), (300, 200, 136), (512, 1536, 128)])
@pytest.mark.parametrize("epi", [0, 1, 2])
def test_linear_f32(M, N, K, epi):
    from decoder_only_transformer_causal_b200 import native
    x = gen((M, K), 1.0, 6, torch.float32)
    W = gen((N, K), 1.0 / math.sqrt(K), 7, torch.float32)
    b = gen((N,), 0.1, 8, torch.float32)
    ref = oracle.linear(f64(x), f64(W), f64(b))
    base = gen((M, N), 1.0, 9, torch.float32)
    out = base.clone().cuda()
    native.linear(x.cuda(), W.cuda(), b.cuda(), out=out, epilogue=epi)
    if epi == 1:
        ref = oracle.gelu(ref)
    if epi == 2:
        ref = ref + f64(base)
    torch.cuda.synchronize()
    assert max_abs(f64(out), ref) <= 1e-5


@pytest.mark.parametrize("rows,C,V", [(300, 768, 50304), (128, 1600, 50304), (77, 768, 1000), (5, 128, 264)])
def test_lm_head_loss_bf16(rows, C, V):
    from decoder_only_transformer_causal_b200 import native
    u = gen((rows, C), 1.0, 10)
    wte = gen((V, C), 0.02, 11)
    _, tgt = seeded.make_tokens(1, rows, V, ignore_frac=0.1)
    tgt = tgt.reshape(-1)
    row_loss = torch.empty(rows, device="cuda")
    sc = torch.empty(2, dtype=torch.float64, device="cuda")
    logits, loss = native.lm_head_loss(u.cuda(), wte.cuda(), tgt.cuda(), row_loss=row_loss,
                                       loss_sum_count=sc, sync_check=True)
    z = oracle.lm_head(f64(u), {"wte": f64(wte)})
    ref_loss, ref_rows, n = oracle.cross_entropy(z, tgt.numpy())
    assert max_abs(f64(logits), z) <= BF16_ATOL
    assert abs(float(loss) - ref_loss) <= LOSS_RTOL * abs(ref_loss)
    assert max_abs(f64(row_loss), ref_rows) <= 1e-3
    assert float(sc[1]) == n
    assert abs(float(sc[0]) - ref_rows.sum()) <= LOSS_RTOL * abs(ref_rows.sum())


def test_lm_head_loss_f32_and_all_ignored():
    from decoder_only_transformer_causal_b200 import native
    rows, C, V = 40, 128, 65
    u = gen((rows, C), 1.0, 12, torch.float32)
    wte = gen((V, C), 0.02, 13, torch.float32)
    _, tgt = seeded.make_tokens(1, rows, V)
    tgt = tgt.reshape(-1)
    logits, loss = native.lm_head_loss(u.cuda(), wte.cuda(), tgt.cuda(), sync_check=True)
    z = oracle.lm_head(f64(u), {"wte": f64(wte)})
    ref_loss, _, _ = oracle.cross_entropy(z, tgt.numpy())
    assert max_abs(f64(logits), z) <= F32_ATOL
    assert abs(float(loss) - ref_loss) <= 1e-5 * abs(ref_loss)
    ign = torch.full_like(tgt, -1)
    _, loss = native.lm_head_loss(u.cuda(), wte.cuda(), ign.cuda(), sync_check=True)
    assert math.isnan(float(loss))


def test_lm_head_bad_target_reports_index():
    from decoder_only_transformer_causal_b200 import native
    rows, C, V = 16, 128, 256
    u, wte = gen((rows, C), 1.0, 14), gen((V, C), 0.02, 15)
    tgt = torch.arange(rows, dtype=torch.int64)
    tgt[3] = V + 5
    with pytest.raises(native.GPTError) as e:
        native.lm_head_loss(u.cuda(), wte.cuda(), tgt.cuda(), sync_check=True)
    assert e.value.status == native.GPT_ERR_INDEX
