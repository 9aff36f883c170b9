"""gpt_lm_head_loss_noalloc: the head + loss for callers that cannot allocate device memory
when they need it (a serving process whose GPU memory is all in a fixed pool, a plugin that may
not bypass its host framework's allocator, a loop that cannot pay for cudaMalloc).

It must give what gpt_lm_head_loss gives with a workspace of its own, call after call, even
though its scratch is one static array that keeps the previous call's contents.  This file is
collected last so that a run stopping at the first failure has run every other test before it;
it passes alone in a fresh process too.
"""
import ctypes
import math

import pytest
import torch

import seeded
from gpu_helpers import BF16_ATOL, LOSS_RTOL, f64, max_abs, needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]


def _case(rows, C, V, seed, ignore_frac):
    g = torch.Generator().manual_seed(seed)
    u = torch.randn((rows, C), generator=g).to(torch.bfloat16).cuda()
    wte = (0.02 * torch.randn((V, C), generator=g)).to(torch.bfloat16).cuda()
    _, tgt = seeded.make_tokens(1, rows, V, seed=seed, ignore_frac=ignore_frac)
    return u, wte, tgt.reshape(-1).cuda()


def _compare(native, u, wte, tgt):
    rows, V = u.shape[0], wte.shape[0]
    ref_rows = torch.empty(rows, device="cuda")
    ref_sc = torch.empty(2, dtype=torch.float64, device="cuda")
    ref_logits, ref_loss = native.lm_head_loss(u, wte, tgt, row_loss=ref_rows, loss_sum_count=ref_sc,
                                               sync_check=True)
    rows_na = torch.full((rows,), float("nan"), device="cuda")
    sc_na = torch.full((2,), float("nan"), dtype=torch.float64, device="cuda")
    logits, loss = native.lm_head_loss_noalloc(u, wte, tgt, row_loss=rows_na, loss_sum_count=sc_na,
                                               sync_check=True)
    assert max_abs(f64(logits), f64(ref_logits)) <= BF16_ATOL
    assert abs(float(loss) - float(ref_loss)) <= LOSS_RTOL * abs(float(ref_loss))
    assert max_abs(f64(rows_na), f64(ref_rows)) <= BF16_ATOL
    assert float(sc_na[1]) == float(ref_sc[1])
    assert abs(float(sc_na[0]) - float(ref_sc[0])) <= LOSS_RTOL * abs(float(ref_sc[0]))


def test_noalloc_matches_workspace_entry_point_twice_in_a_row():
    from decoder_only_transformer_causal_b200 import native
    # first call: a large request with ignored targets; second: a smaller one whose rows fall
    # inside what the first left behind in the shared scratch
    _compare(native, *_case(1000, 768, 50304, seed=11, ignore_frac=0.2))
    _compare(native, *_case(77, 768, 1000, seed=12, ignore_frac=0.0))


def test_noalloc_rejects_requests_beyond_its_scratch():
    from decoder_only_transformer_causal_b200 import native
    rows, V = 8192, 50304  # needs about 26 MB of scratch, more than the 16 MiB built in
    assert native.lm_head_workspace_bytes(rows, V) > 16 << 20
    rc = native.LIB.gpt_lm_head_loss_noalloc(1 << 20, 1 << 20, 1 << 20, rows, 768, V, native.GPT_DTYPE_BF16,
                                             1 << 20, None, None, None, None, 0)
    assert rc == native.GPT_ERR_WS_TOO_SMALL


def test_noalloc_all_ignored_gives_nan():
    from decoder_only_transformer_causal_b200 import native
    u, wte, tgt = _case(64, 128, 256, seed=13, ignore_frac=0.0)
    _, loss = native.lm_head_loss_noalloc(u, wte, torch.full_like(tgt, -1), sync_check=True)
    assert math.isnan(float(loss))
