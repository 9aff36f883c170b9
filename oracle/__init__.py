"""fp64 CPU oracle of the GPT-2 / nanoGPT causal decoder forward pass.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the tests, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import it.  It shares nothing with the
CUDA path (no kernels, headers, helpers, tables or constants); the two meet only in
the seeded inputs of the ``seeded`` module.

See ``oracle/gpt.py`` (the forward pass), ``oracle/generate.py`` (GPT.generate),
``oracle/optim.py`` (the optimizer step) and ``oracle/backward.py`` (the gradients) for the
definitions and their citations.
"""
from .gpt import (  # noqa: F401
    PAGES, embed, layer_norm, linear, split_heads, merge_heads, attention_probs,
    causal_attention, gelu, causal_self_attention, mlp, block, final_hidden,
    lm_head, cross_entropy, forward, num_params,
)
from . import generate as gen  # noqa: F401,E402
