"""The time-out path of the tensor-core kernels and of the single-launch decode step, made to run on
purpose without faulting the GPU.

Every pipeline wait in the tensor-core kernels is bounded: when a wait gives up, the kernel records
GPT_ERR_TIMEOUT in its status word, lets the copies and products it already issued finish, frees
its tensor memory and returns.  gpt_set_wait_limit_ns lowers the limit to 1 ms and makes the
kernel's issuing thread first wait for an event that never happens (a barrier nothing arrives
on), so that wait gives up and the whole kernel takes its time-out path; the test then checks the
status, restores the defaults and checks that the next call on the same context computes the
right result."""
import pytest
import torch

from gpu_helpers import needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]


@pytest.fixture
def short_waits():
    from decoder_only_transformer_causal_b200 import native
    torch.cuda.synchronize()
    native.set_wait_limit_ns(1_000_000, force_timeout=True)
    try:
        yield native
    finally:
        torch.cuda.synchronize()
        native.set_wait_limit_ns(0)


def _attention_inputs():
    g = torch.Generator(device="cuda").manual_seed(71)
    return [torch.randn((2, 4, 512, 64), generator=g, device="cuda").to(torch.bfloat16) for _ in range(3)]


def test_attention_wait_limit_gives_timeout_then_recovers(short_waits):
    native = short_waits
    q, k, v = _attention_inputs()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    native.attention(q, k, v, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == native.GPT_ERR_TIMEOUT
    native.set_wait_limit_ns(0)
    st.zero_()
    y = native.attention(q, k, v, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == native.GPT_OK
    ref = torch.nn.functional.scaled_dot_product_attention(q.float(), k.float(), v.float(), is_causal=True)
    assert float((y.float() - ref).abs().max()) <= 2e-2


@pytest.mark.parametrize("M", [128, 512])
def test_gemm_wait_limit_gives_timeout_then_recovers(short_waits, M):
    """M = 128: one CTA per 128-row tile; M = 512: CTA pairs (2-SM products), whose leader waits
    for the peer's copies, counted on the leader's barriers, before the pair exits."""
    native = short_waits
    g = torch.Generator(device="cuda").manual_seed(72)
    x = torch.randn((M, 768), generator=g, device="cuda").to(torch.bfloat16)
    W = (0.02 * torch.randn((2304, 768), generator=g, device="cuda")).to(torch.bfloat16)
    b = (0.02 * torch.randn(2304, generator=g, device="cuda")).to(torch.bfloat16)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.zeros((M, 2304), dtype=torch.bfloat16, device="cuda")
    native.linear(x, W, b, out=out, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == native.GPT_ERR_TIMEOUT
    native.set_wait_limit_ns(0)
    st.zero_()
    native.linear(x, W, b, out=out, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == native.GPT_OK
    ref = x.float() @ W.float().T + b.float()
    assert float((out.float() - ref).abs().max()) <= 2e-2


def test_decode_step_wait_limit_gives_timeout_then_recovers():
    """The single-launch decode step waits at its first grid barrier for an arrival that never
    comes: every CTA gives up after 1 ms, lets its weight copies land and returns, the position stays
    where it was, and the next step (limits restored) gives the logits of an undisturbed step."""
    import seeded
    from decoder_only_transformer_causal_b200 import GPT, GPTConfig, native
    from gpu_helpers import model_inputs
    cfg_d, W, _, _, _ = model_inputs("gpt2", stress=True, n_layer=2)
    m = GPT(GPTConfig.from_dict(cfg_d), W)
    B, T0 = 1, 40
    prompt, _ = seeded.make_tokens(B, T0, 50257, seed=9021)
    tok = torch.tensor([123], dtype=torch.int64, device="cuda")
    runs = []
    for forced in (False, True):
        kv = native.alloc_kv_cache(m.cfg, B)
        ws = native.alloc_workspace(native.decode_workspace_bytes(m.cfg, B, T0))
        native.prefill(m.cfg, m.weights, prompt.cuda(), kv, ws, sync_check=True)
        if forced:
            torch.cuda.synchronize()
            native.set_wait_limit_ns(1_000_000, force_timeout=True)
            try:
                native.decode_step(m.cfg, m.weights, tok, kv, ws)
                assert native.check_status(ws) == native.GPT_ERR_TIMEOUT
            finally:
                torch.cuda.synchronize()
                native.set_wait_limit_ns(0)
        logits = native.decode_step(m.cfg, m.weights, tok, kv, ws, sync_check=True).clone()
        assert native.check_status(ws) == native.GPT_OK
        runs.append(logits)
    assert torch.equal(runs[0], runs[1])
