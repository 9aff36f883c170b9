"""Pins of the generate oracle (oracle/generate.py) against facts that do not come from it.

* Closed forms: two-way softmax with temperature (p_1 = sigmoid((z_1 - z_0) / T)); ties at
  the top-k threshold ("nanoGPT 全局流程图", 第五阶段: only logits strictly below the k-th
  largest are masked).
* Brute force: over a fine grid of uniforms the draw lands on index i with frequency p_i, the
  defining property of a multinomial draw; p from scipy's softmax.
* Library special cases: top_k = 1 is argmax (numpy); greedy generation equals repeated argmax
  over an independent composition of torch fp64 library routines.
* Invariants: the crop to block_size (tokens older than the window do not matter), prefix
  consistency of longer generations, and independence of greedy decoding from the uniforms.

A planted-mistakes test swaps in plausible wrong versions and requires a pin to fail.
"""
from contextlib import contextmanager

import numpy as np
import pytest
import torch
from scipy.special import expit, softmax

import oracle
import oracle.generate as og
import seeded
from test_oracle_pins import torch_forward

TINY = seeded.WORKLOADS["tiny"].model_dict()
RNG = np.random.default_rng(20240602)


def tiny_model(stress=True):
    return seeded.to_f64(seeded.make_weights(TINY, stress=stress))


# --------------------------------------------------------------------------- pins
def pin_two_way_temperature(g=og):
    for a, b, T in [(0.3, -0.4, 1.0), (0.3, -0.4, 0.5), (-1.2, 0.7, 2.0), (2.0, 2.5, 0.8)]:
        p1 = expit((b - a) / T)
        p = g.probabilities(np.array([[a, b]]), T)[0]
        assert abs(p[1] - p1) < 1e-15 and abs(p[0] - (1 - p1)) < 1e-15
        p0 = 1 - p1
        assert g.draw(p, p0 - 1e-9) == 0 and g.draw(p, p0 + 1e-9) == 1
        assert g.sample(np.array([[a, b]]), T, None, [0.0])[0] == 0
        assert g.sample(np.array([[a, b]]), T, None, [0.999999999])[0] == 1


def pin_top_k_ties_and_limits(g=og):
    z = np.array([[3.0, 1.0, 3.0, 2.0]])
    for k in (1, 2):   # both 3's are the k-th largest for k = 1 and 2: both kept, nothing else
        p = g.probabilities(z, 1.0, k)[0]
        assert np.allclose(p, [0.5, 0.0, 0.5, 0.0], atol=1e-15)
        assert g.sample(z, 1.0, k, [0.25])[0] == 0 and g.sample(z, 1.0, k, [0.75])[0] == 2
        assert g.sample(z, 1.0, k, [0.0])[0] == 0
    p3 = g.probabilities(z, 1.0, 3)[0]
    assert np.allclose(p3, softmax([3.0, -np.inf, 3.0, 2.0]), atol=1e-15)
    for k in (4, 10, None, 0):   # k >= V or no filter: plain softmax
        assert np.allclose(g.probabilities(z, 1.0, k)[0], softmax(z[0]), atol=1e-15)
    # masked entries are never drawn, whatever u is
    zz = RNG.normal(size=(1, 40))
    keep = np.argsort(zz[0])[-5:]
    for u in np.linspace(0, 0.999999, 101):
        assert g.sample(zz, 0.7, 5, [u])[0] in keep


def pin_top_k_is_argmax(g=og):
    z = RNG.normal(size=(6, 300))
    for u in (0.0, 0.3, 0.999999):
        got = g.sample(z, 0.8, 1, np.full(6, u))
        assert np.array_equal(got, z.argmax(-1))


def pin_draw_frequencies(g=og):
    """Uniforms at the midpoints of M equal cells: index i is drawn for a run of cells whose
    length is p_i M to within one cell."""
    M = 20000
    us = (np.arange(M) + 0.5) / M
    for T, k in [(1.0, None), (0.6, 4), (1.7, 2)]:
        z = RNG.normal(size=7) * 1.5
        zk = np.where(z < np.sort(z)[-k], -np.inf, z) if k else z
        p = softmax(zk / T)
        picks = np.array([g.sample(z[None], T, k, [u])[0] for u in us])
        counts = np.bincount(picks, minlength=7) / M
        assert np.all(np.abs(counts - p) <= 1.0 / M + 1e-12), (counts, p)
        assert np.all(np.diff(picks) >= 0)   # inverse CDF: monotone in u


def pin_greedy_vs_torch(g=og):
    """top_k = 1 generation equals repeated argmax over the torch fp64 composition of the
    forward, with the sequence cropped to the window as it grows past block_size."""
    W = tiny_model()
    bs = TINY["block_size"]
    idx, _ = seeded.make_tokens(2, bs - 3, TINY["vocab_size"], seed=4242)
    idx = idx.numpy()
    n_new = 6                      # crosses block_size after 3 steps
    got = g.generate(W, TINY, idx, n_new, np.zeros((n_new, 2)), 1.0, 1)["tokens"]
    ref = idx.copy()
    for _ in range(n_new):
        ctx = ref[:, -bs:]
        logits, _ = torch_forward(W, TINY, ctx, np.zeros_like(ctx))
        ref = np.concatenate([ref, logits[:, -1, :].argmax(-1)[:, None]], axis=1)
    assert np.array_equal(got, ref)


def pin_generate_invariants(g=og):
    W = tiny_model()
    bs, V = TINY["block_size"], TINY["vocab_size"]
    idx, _ = seeded.make_tokens(2, bs + 5, V, seed=777)
    idx = idx.numpy()
    u = RNG.random((4, 2))
    # crop: tokens older than the window do not change what is drawn
    a = g.generate(W, TINY, idx, 4, u, 0.9, 20)
    b = g.generate(W, TINY, idx[:, -bs:], 4, u, 0.9, 20)
    assert np.array_equal(a["tokens"][:, -4:], b["tokens"][:, -4:])
    assert np.array_equal(a["tokens"][:, :bs + 5], idx)
    assert a["tokens"].min() >= 0 and a["tokens"].max() < V
    # a longer run starts with the shorter one (same uniforms)
    short = g.generate(W, TINY, idx[:, :10], 2, u[:2], 0.9, None)
    long = g.generate(W, TINY, idx[:, :10], 4, u, 0.9, None)
    assert np.array_equal(long["tokens"][:, :12], short["tokens"])
    assert np.allclose(long["logits"][:2], short["logits"], rtol=0, atol=0)
    # greedy decoding does not depend on the uniforms; zero new tokens returns the prompt
    g1 = g.generate(W, TINY, idx[:, :10], 3, np.zeros((3, 2)), 1.0, 1)["tokens"]
    g2 = g.generate(W, TINY, idx[:, :10], 3, np.full((3, 2), 0.99), 1.0, 1)["tokens"]
    assert np.array_equal(g1, g2)
    assert np.array_equal(g.generate(W, TINY, idx[:, :10], 0, np.zeros((0, 2)))["tokens"], idx[:, :10])
    # step logits are the forward's last-position logits of the (cropped) context
    first = oracle.forward(W, TINY, idx[:, -bs:], None)["logits"][:, -1, :]
    assert np.array_equal(a["logits"][0], first)


PINS = [pin_two_way_temperature, pin_top_k_ties_and_limits, pin_top_k_is_argmax, pin_draw_frequencies,
        pin_greedy_vs_torch, pin_generate_invariants]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()


# --------------------------------------------------------------------------- planted mistakes
@contextmanager
def planted(name, fn):
    old = getattr(og, name)
    setattr(og, name, fn)
    try:
        yield
    finally:
        setattr(og, name, old)


_orig = {n: getattr(og, n) for n in ("scaled_logits", "top_k_filter", "draw", "crop")}


def _temperature_multiplied(logits, temperature):
    return np.asarray(logits, dtype=np.float64) * float(temperature)


def _top_k_drops_ties(z, top_k):        # keeps exactly k entries by position, dropping tied ones
    z = np.array(z, dtype=np.float64)
    if top_k is None or top_k <= 0:
        return z
    k = min(int(top_k), z.shape[-1])
    order = np.argsort(-z, axis=-1, kind="stable")[..., :k]
    out = np.full_like(z, -np.inf)
    np.put_along_axis(out, order, np.take_along_axis(z, order, -1), -1)
    return out


def _top_k_off_by_one(z, top_k):        # threshold at the (k+1)-th largest
    return _orig["top_k_filter"](z, None if not top_k else top_k + 1)


def _draw_ge(p, u):                     # >= instead of >: draws a zero-probability index at u = 0
    c = np.cumsum(np.asarray(p, dtype=np.float64))
    return int(np.nonzero(c >= u)[0][0])


def _draw_reversed(p, u):               # cumulative sum from the wrong end
    p = np.asarray(p, dtype=np.float64)
    return len(p) - 1 - _orig["draw"](p[::-1], u)


def _crop_first_window(idx, block_size):
    idx = np.asarray(idx)
    return idx[:, :block_size]


MISTAKES = {
    "scaled_logits:multiply": ("scaled_logits", _temperature_multiplied),
    "top_k_filter:drop-ties": ("top_k_filter", _top_k_drops_ties),
    "top_k_filter:k+1": ("top_k_filter", _top_k_off_by_one),
    "draw:>=": ("draw", _draw_ge),
    "draw:reversed": ("draw", _draw_reversed),
    "crop:first-window": ("crop", _crop_first_window),
}


@pytest.mark.parametrize("mistake", sorted(MISTAKES))
def test_planted_mistakes(mistake):
    name, fn = MISTAKES[mistake]
    failed = []
    with planted(name, fn):
        for pin in PINS:
            try:
                pin(og)
            except AssertionError:
                failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {mistake}"
