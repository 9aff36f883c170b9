"""Generation through the C ABI against the fp64 generate oracle: the sampling step
(gpt_sample), the cached forward (gpt_prefill + gpt_decode_step, teacher-forced with seeded
tokens) and whole runs of gpt_generate.

Where floating point decides a token (the draw), the GPU's choice must equal the oracle's,
except where the oracle's own decision sits within the rounding or tolerance band of a
boundary between two tokens; there the test checks that the GPU's token is one that the
band allows, and a generated sequence is compared no further once it has left the
oracle's."""
import math

import numpy as np
import pytest
import torch

import oracle
import seeded
from gpu_helpers import BF16_ATOL, F32_ATOL, f64, max_abs, model_inputs, needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]


def gpu_model(cfg, W, gelu="erf"):
    from decoder_only_transformer_causal_b200 import GPT, GPTConfig
    return GPT(GPTConfig.from_dict(dict(cfg, gelu=gelu)), W)


def allowed_pick(z, u, pick, temperature, top_k, atol, rel=1e-6):
    """True if `pick` is a draw the oracle could make for logits within atol of z (and with the
    sums rounded to `rel`): it is kept by some such logits, and u falls inside its CDF interval
    widened by the largest change such logits can make to a partial-sum ratio."""
    zf = np.asarray(z, np.float64) / temperature
    tol = atol / temperature
    V = zf.shape[0]
    if top_k and 0 < top_k < V:
        kth = np.sort(zf)[-top_k]
        if zf[pick] < kth - 2 * tol:
            return False
        below = zf[zf < kth]
        if below.size and below.max() >= kth - 2 * tol:   # the kept set itself is not decided
            return True
    p = oracle.gen.probabilities(z, temperature, top_k)
    if p[pick] == 0 and tol == 0:
        return False
    c = np.cumsum(p)
    lo = c[pick - 1] if pick > 0 else 0.0
    hi = c[pick]
    f = math.exp(2 * tol)
    return lo / f - rel <= u <= hi * f + rel


# ------------------------------------------------------------------ sampling step
SAMPLE_CASES = [
    # V, B, temperature, top_k, ties
    (65, 16, 1.0, None, 0),
    (65, 16, 0.8, 5, 0),
    (1000, 12, 0.7, 200, 0),
    (50304, 16, 0.8, 200, 0),
    (50304, 8, 1.3, None, 0),
    (50304, 8, 1.0, 1, 0),
    (5000, 8, 0.9, 10, 3),      # the 10th largest value is shared by four entries
    (5000, 8, 0.9, 1, 2),       # argmax shared by three entries: they split the mass
    (3000, 4, 1.0, 3000, 0),    # top_k == V: no filter
    (1, 3, 1.0, 5, 0),          # one class
    (2049, 5, 0.5, 7, 0),       # ragged chunks per thread
]


@pytest.mark.parametrize("V,B,temperature,top_k,ties", SAMPLE_CASES)
def test_sample_matches_oracle(V, B, temperature, top_k, ties):
    from decoder_only_transformer_causal_b200 import native
    base = seeded.make_logits(B, V, ties=ties)
    reps = 16
    logits = base.repeat(reps, 1)                                  # each row with 16 uniforms
    u = seeded.make_uniforms(1, B * reps)[0]
    u[0], u[1] = 0.0, 1.0 - 2.0 ** -24                             # the ends of [0, 1)
    got = native.sample(logits.cuda(), u.cuda(), temperature, top_k).cpu().numpy()
    ref = oracle.gen.sample(f64(logits), temperature, top_k, f64(u))
    bad = [i for i in np.nonzero(got != ref)[0]
           if not allowed_pick(f64(logits[i]), float(u[i]), int(got[i]), temperature, top_k, 0.0)]
    assert not bad, [(i, got[i], ref[i], float(u[i])) for i in bad[:5]]
    assert (got != ref).mean() <= 0.01
    assert got.min() >= 0 and got.max() < V
    if top_k == 1 and ties == 0:
        assert np.array_equal(got, logits.argmax(-1).numpy())


@pytest.mark.parametrize("V,top_k", [(3000, 100), (8192, 100), (50304, 3000)])
def test_sample_crowded_bin(V, top_k):
    """Every logit in [1, 1.2): one bin of the top-11-bit histogram holds the whole row, more
    members than the candidate buffer, so the threshold is found by bisection (over one CTA's row
    for V < 4096, over a cluster's slices otherwise)."""
    from decoder_only_transformer_causal_b200 import native
    g = torch.Generator().manual_seed(V)
    base = 1.0 + 0.2 * torch.rand(3, V, generator=g)
    reps = 8
    logits = base.repeat(reps, 1)
    u = seeded.make_uniforms(1, 3 * reps)[0]
    got = native.sample(logits.cuda(), u.cuda(), 0.9, top_k).cpu().numpy()
    ref = oracle.gen.sample(f64(logits), 0.9, top_k, f64(u))
    bad = [i for i in np.nonzero(got != ref)[0]
           if not allowed_pick(f64(logits[i]), float(u[i]), int(got[i]), 0.9, top_k, 0.0)]
    assert not bad, [(i, got[i], ref[i], float(u[i])) for i in bad[:5]]
    kth = np.sort(logits.numpy(), axis=1)[:, -top_k]
    assert all(logits[i, got[i]].item() >= kth[i] for i in range(len(got)))


def test_sample_strided_output():
    from decoder_only_transformer_causal_b200 import native
    logits = seeded.make_logits(4, 777).cuda()
    u = seeded.make_uniforms(1, 4)[0].cuda()
    seq = torch.full((4, 10), -7, dtype=torch.int64, device="cuda")
    native.sample(logits, u, 0.9, 50, out=seq[:, 6])
    torch.cuda.synchronize()
    alone = native.sample(logits, u, 0.9, 50)
    assert torch.equal(seq[:, 6], alone)
    assert int((seq[:, :6] != -7).sum()) == 0 and int((seq[:, 7:] != -7).sum()) == 0


# ------------------------------------------------------------------ cached forward
def decode_logits_gpu(cfg, W, prompt, forced, gelu="erf"):
    """Logits after the prefill of `prompt` and after each teacher-forced token of `forced`."""
    from decoder_only_transformer_causal_b200 import native
    m = gpu_model(cfg, W, gelu)
    B, T0 = prompt.shape
    kv = native.alloc_kv_cache(m.cfg, B)
    ws = native.alloc_workspace(native.decode_workspace_bytes(m.cfg, B, T0))
    out = [f64(native.prefill(m.cfg, m.weights, prompt.cuda(), kv, ws, sync_check=True))]
    forced_d = forced.cuda()
    for s in range(forced.shape[1]):
        out.append(f64(native.decode_step(m.cfg, m.weights, forced_d[:, s], kv, ws, sync_check=True)))
    return np.stack(out)


def decode_logits_oracle(cfg, W64, prompt, forced, steps, gelu="erf"):
    seq = np.concatenate([prompt.numpy(), forced.numpy()], axis=1)
    T0 = prompt.shape[1]
    return {s: oracle.forward(W64, cfg, seq[:, :T0 + s], None, gelu)["logits"][:, -1, :] for s in steps}


DECODE_CASES = [
    # workload, stress, layers, B, T0, n_forced, steps checked by the oracle, gelu
    ("tiny", True, None, 3, 5, 59, "all", "erf"),          # up to the last position (63)
    ("tiny", True, None, 9, 3, 6, "all", "tanh"),           # rows 9..16 of one product launch
    ("tiny", True, None, 17, 3, 4, "all", "erf"),           # B > 16: the row-chunked products
    ("gpt2", True, 2, 2, 120, 12, "all", "erf"),            # crosses the 128-key split
    ("gpt2", False, None, 4, 1, 8, "all", "erf"),           # the 124M model from one token
    ("gpt2", True, 2, 9, 40, 3, "all", "erf"),
    ("gpt2-xl", True, 2, 2, 30, 4, "all", "erf"),           # C = 1600: two staged K chunks
    ("gpt2", True, 2, 1, 1000, 23, [0, 1, 12, 23], "erf"),  # the end of the window
]


@pytest.mark.parametrize("name,stress,layers,B,T0,n,steps,gelu", DECODE_CASES)
def test_decode_steps_match_forward(name, stress, layers, B, T0, n, steps, gelu):
    over = {"n_layer": layers} if layers else {}
    cfg, W, W64, _, _ = model_inputs(name, stress=stress, **over)
    V = cfg["vocab_size"]
    prompt, _ = seeded.make_tokens(B, T0, min(V, 50257), seed=9001)
    forced, _ = seeded.make_tokens(B, n, min(V, 50257), seed=9002)
    got = decode_logits_gpu(cfg, W, prompt, forced, gelu)
    steps = range(n + 1) if steps == "all" else steps
    ref = decode_logits_oracle(cfg, W64, prompt, forced, steps, gelu)
    tol = F32_ATOL if cfg["dtype"] == "f32" else BF16_ATOL
    for s, r in ref.items():
        err = max_abs(got[s], r)
        assert err <= tol, (s, err)


PLAN_CASES = [
    # workload, layers, B, T0, n_forced, bias, gelu: the single-launch decode step's shared-memory
    # plans (four weight slots for GPT-2 124M; two for C = 1024 with B <= 8; one for C = 1024, B > 8)
    ("gpt2-medium", 2, 2, 70, 3, True, "erf"),
    ("gpt2-medium", 2, 12, 70, 2, True, "erf"),
    ("gpt2", 2, 16, 63, 3, False, "tanh"),        # 16 sequences, no biases; 64 -> 65 keys: a new chunk
]


@pytest.mark.parametrize("name,layers,B,T0,n,bias,gelu", PLAN_CASES)
def test_decode_step_plans_match_forward(name, layers, B, T0, n, bias, gelu):
    cfg, W, W64, _, _ = model_inputs(name, stress=True, n_layer=layers, bias=bias)
    V = cfg["vocab_size"]
    prompt, _ = seeded.make_tokens(B, T0, min(V, 50257), seed=9011)
    forced, _ = seeded.make_tokens(B, n, min(V, 50257), seed=9012)
    got = decode_logits_gpu(cfg, W, prompt, forced, gelu)
    ref = decode_logits_oracle(cfg, W64, prompt, forced, range(n + 1), gelu)
    for s, r in ref.items():
        err = max_abs(got[s], r)
        assert err <= BF16_ATOL, (s, err)


def test_decode_past_window_is_reported_and_writes_nothing():
    from decoder_only_transformer_causal_b200 import native
    cfg, W, _, _, _ = model_inputs("tiny", stress=True)
    m = gpu_model(cfg, W)
    B, bs = 2, cfg["block_size"]
    prompt, _ = seeded.make_tokens(B, bs, cfg["vocab_size"], seed=9003)
    kv = native.alloc_kv_cache(m.cfg, B)
    ws = native.alloc_workspace(native.decode_workspace_bytes(m.cfg, B, bs))
    native.prefill(m.cfg, m.weights, prompt.cuda(), kv, ws, sync_check=True)
    before = kv.clone()
    tok = torch.zeros(B, dtype=torch.int64, device="cuda")
    with pytest.raises(native.GPTError) as e:
        native.decode_step(m.cfg, m.weights, tok, kv, ws, sync_check=True)
    assert e.value.status == native.GPT_ERR_BAD_SHAPE
    assert torch.equal(kv, before)


def test_decode_bad_token_is_reported():
    from decoder_only_transformer_causal_b200 import native
    cfg, W, _, _, _ = model_inputs("tiny")
    m = gpu_model(cfg, W)
    prompt, _ = seeded.make_tokens(1, 4, cfg["vocab_size"], seed=9004)
    kv = native.alloc_kv_cache(m.cfg, 1)
    ws = native.alloc_workspace(native.decode_workspace_bytes(m.cfg, 1, 4))
    native.prefill(m.cfg, m.weights, prompt.cuda(), kv, ws, sync_check=True)
    tok = torch.tensor([cfg["vocab_size"]], dtype=torch.int64, device="cuda")
    with pytest.raises(native.GPTError) as e:
        native.decode_step(m.cfg, m.weights, tok, kv, ws, sync_check=True)
    assert e.value.status == native.GPT_ERR_INDEX


# ------------------------------------------------------------------ whole generations
def compare_generation(got_tok, got_logits, ref, T0, uniforms, temperature, top_k, atol):
    """Token by token while a sequence agrees with the oracle's: its step logits must be within
    atol, and a differing token must be one the tolerance band allows.  Returns the number of
    (sequence, step) pairs compared."""
    n, B = uniforms.shape
    alive = np.ones(B, bool)
    compared = 0
    for s in range(n):
        for b in np.nonzero(alive)[0]:
            z = ref["logits"][s, b]
            err = max_abs(got_logits[s, b], z)
            assert err <= atol, (s, b, err)
            compared += 1
            g, r = int(got_tok[b, T0 + s]), int(ref["tokens"][b, T0 + s])
            if g != r:
                assert allowed_pick(z, float(uniforms[s, b]), g, temperature, top_k, atol), (s, b, g, r)
                alive[b] = False
    return compared


GEN_CASES = [
    # workload, stress, layers, B, T0, max_new, temperature, top_k
    ("tiny", True, None, 3, 50, 20, 0.9, 20),      # outgrows block_size 64 after 14 steps
    ("tiny", True, None, 2, 70, 3, 1.0, None),     # prompt longer than the window
    ("tiny", False, None, 4, 1, 12, 1.0, 1),       # greedy
    ("gpt2", True, 2, 2, 16, 10, 0.8, 200),        # the pages' sampling settings
    ("gpt2", False, None, 2, 1, 6, 0.8, 200),
]


@pytest.mark.parametrize("name,stress,layers,B,T0,max_new,temperature,top_k", GEN_CASES)
def test_generate_matches_oracle(name, stress, layers, B, T0, max_new, temperature, top_k):
    from decoder_only_transformer_causal_b200 import native
    over = {"n_layer": layers} if layers else {}
    cfg, W, W64, _, _ = model_inputs(name, stress=stress, **over)
    V = cfg["vocab_size"]
    prompt, _ = seeded.make_tokens(B, T0, min(V, 50257), seed=9100)
    u = seeded.make_uniforms(max_new, B)
    m = gpu_model(cfg, W)
    step_logits = torch.empty((max_new, B, V), device="cuda")
    toks = native.generate(m.cfg, m.weights, prompt.cuda(), max_new, u.cuda(), temperature, top_k,
                           step_logits=step_logits, sync_check=True).cpu().numpy()
    assert np.array_equal(toks[:, :T0], prompt.numpy())
    assert toks.min() >= 0 and toks.max() < V
    ref = oracle.gen.generate(W64, cfg, prompt.numpy(), max_new, f64(u), temperature, top_k)
    atol = F32_ATOL if cfg["dtype"] == "f32" else BF16_ATOL
    compared = compare_generation(toks, f64(step_logits), ref, T0, f64(u), temperature, top_k, atol)
    assert compared >= B                       # at least every first step
    if cfg["dtype"] == "f32":
        assert np.array_equal(toks, ref["tokens"])


def test_generate_model_wrapper_and_zero_steps():
    cfg, W, _, _, _ = model_inputs("tiny", stress=True)
    m = gpu_model(cfg, W)
    prompt, _ = seeded.make_tokens(2, 7, cfg["vocab_size"], seed=9200)
    same = m.generate(prompt.cuda(), 0)
    assert torch.equal(same.cpu(), prompt)
    u = seeded.make_uniforms(5, 2).cuda()
    a = m.generate(prompt.cuda(), 5, 0.9, 10, uniforms=u)
    b = m.generate(prompt.cuda(), 5, 0.9, 10, uniforms=u)
    assert torch.equal(a, b)                   # deterministic for fixed uniforms
