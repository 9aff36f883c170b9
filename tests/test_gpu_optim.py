"""The optimizer step (gpt_adamw_step) through the C ABI against the fp64 oracle
(oracle/optim.py): global-norm clipping, AdamW with decay on two-dimensional tensors only, the
bias corrections over consecutive steps, the copy into the packed weights, and the padding of
the flat arrays left untouched."""
import math

import numpy as np
import pytest
import torch

import oracle.optim as oo
import seeded
from gpu_helpers import needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]

# per step: gradient scale (global norm above or below max_norm 1.0) and learning rate
STEPS = [(0.05, 1e-3), (1e-5, 2e-3), (0.2, 5e-4)]


@pytest.mark.parametrize("name,layers,bias,max_norm", [
    ("tiny", None, True, 1.0),
    ("tiny", None, False, 1.0),
    ("gpt2", 2, True, 1.0),
    ("gpt2", 2, True, 0.0),          # clipping off
    ("gpt2-xl", 1, True, 1.0),
])
def test_adamw_matches_oracle(name, layers, bias, max_norm):
    from decoder_only_transformer_causal_b200 import native
    from decoder_only_transformer_causal_b200.native import GPTConfig
    over = {"bias": bias}
    if layers:
        over["n_layer"] = layers
    cfgd = dict(seeded.WORKLOADS[name].model_dict(), **over)
    cfg = GPTConfig.from_dict(cfgd)
    W = seeded.make_weights(cfgd)
    shapes = {n: tuple(t.shape) for n, t in W.items()}
    p = native.flat_params(cfg, W)
    pad = torch.ones_like(p, dtype=torch.bool)
    for t in native.unflatten(cfg, pad, shapes).values():
        t.fill_(False)
    p[pad] = float("nan")                                   # the padding must stay untouched
    m = torch.zeros_like(p)
    v = torch.zeros_like(p)
    m[pad] = float("nan")
    v[pad] = float("nan")
    weights = native.pack_weights(cfg, W)
    ref_p = {n: t.to(torch.float64).numpy() for n, t in W.items()}
    ref_m = {n: np.zeros(s) for n, s in shapes.items()}
    ref_v = {n: np.zeros(s) for n, s in shapes.items()}
    ws = native.alloc_workspace(native.LIB.gpt_adamw_workspace_bytes())
    for step, (scale, lr) in enumerate(STEPS, start=1):
        G = seeded.make_grads(cfgd, seed=seeded.BASE_SEED + 700_000 + 1000 * step, scale=scale)
        g = native.flat_params(cfg, G)
        g[pad] = float("nan")
        norm = native.adamw_step(cfg, p, g, m, v, step, lr, weights=weights, max_grad_norm=max_norm,
                                 workspace=ws, sync_check=True)
        ref_p, ref_m, ref_v, ref_norm = oo.adamw_step(ref_p, {n: t.double().numpy() for n, t in G.items()},
                                                      ref_m, ref_v, step, lr, max_norm=max_norm)
        assert float(norm) == pytest.approx(ref_norm, rel=1e-6)
        clipped = max_norm > 0 and ref_norm > max_norm
        assert clipped == (step != 2 and max_norm > 0)
        gp = native.unflatten(cfg, p, shapes)
        gm = native.unflatten(cfg, m, shapes)
        gv = native.unflatten(cfg, v, shapes)
        for n in shapes:
            a = gp[n].double().cpu().numpy()
            assert np.allclose(a, ref_p[n], rtol=1e-6, atol=1e-7), (step, n, float(np.abs(a - ref_p[n]).max()))
            # fp32 moments: each step rounds a few products and a sum (unit roundoff 6e-8), so the
            # error scales with the tensor's magnitude, not with entries that cancel to near zero
            tm = 2e-6 * float(np.abs(ref_m[n]).max())
            tv = 2e-6 * float(np.abs(ref_v[n]).max())
            assert np.allclose(gm[n].double().cpu().numpy(), ref_m[n], rtol=1e-5, atol=tm), (step, n)
            assert np.allclose(gv[n].double().cpu().numpy(), ref_v[n], rtol=1e-5, atol=tv), (step, n)
        assert bool(torch.isnan(p[pad]).all() and torch.isnan(m[pad]).all() and torch.isnan(v[pad]).all())
    # the forward's packed weights hold the updated parameters in the configuration's dtype
    dt = cfg.torch_dtype
    entries, _ = native.weights_layout(cfg)
    es = 2 if cfg.dtype == "bf16" else 4
    wv = weights.view(dt)
    for nme, off, numel in entries:
        if nme not in shapes:
            continue
        got = wv[off // es: off // es + numel]
        want = p[off // es: off // es + numel].to(dt)
        assert torch.equal(got, want), nme


def test_adamw_helper_class_runs_schedule():
    from decoder_only_transformer_causal_b200 import GPT, AdamW, native
    from decoder_only_transformer_causal_b200.native import GPTConfig
    cfgd = seeded.WORKLOADS["tiny"].model_dict()
    W = seeded.make_weights(cfgd)
    model = GPT(GPTConfig.from_dict(cfgd), W)
    opt = AdamW(model, W, warmup_iters=2, lr_decay_iters=10)
    G = native.flat_params(model.cfg, seeded.make_grads(cfgd, scale=0.01))
    before = opt.params.clone()
    for _ in range(3):
        opt.step(G)
    torch.cuda.synchronize()
    assert opt.it == 3 and not torch.equal(before, opt.params)
    assert math.isfinite(float(opt.grad_norm))
