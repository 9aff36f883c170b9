#!/usr/bin/env python
"""Forward-pass throughput of the GPT-2 124M decoder (B 12, T 1024, bf16) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one gpt_forward call with targets: embedding, 12 Blocks, ln_f, the tied lm_head
with the fused cross-entropy, and (with N > 1) the all-reduce of {sum of row losses, count}
that forms the global loss of a batch-sharded run (weak scaling: every rank runs B 12).
Inputs (weights, token ids, targets) are resident in HBM before timing; the step touches
well over the 126 MB L2 (0.25 GB of weights, 1.24 GB of logits), so no flush is needed.
Rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle on the host cores on a bounded sample of the
same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import seeded  # noqa: E402

WORKLOAD = "gpt2"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-kernels", action="store_true", help="skip the per-kernel timings")
    ap.add_argument("--decode-only", action="store_true",
                    help="run only the decode measurement (--steps graph replays after --warmup) and print it; "
                         "with --no-e2e the generate call is skipped (for profiler captures)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--train-only", action="store_true",
                    help="run only the training-step measurement (--steps timed after --warmup) and print it")
    ap.add_argument("--adamw-only", action="store_true",
                    help="run only the optimizer-step measurement (--steps timed after --warmup) and print it")
    ap.add_argument("--profile-kernel", default=None,
                    help="launch only this kernel of the forward (names as in kernels_ms_per_forward): "
                         "--warmup untimed then --steps timed launches; for profiler captures")
    return ap.parse_args()


# ---------------------------------------------------------------- workload accounting
def forward_flops(w) -> float:
    """Algorithmic FLOPs of one forward: 4 GEMMs per layer, the head, and causal attention
    counted over unmasked (i, j) pairs only."""
    N, C, L, V, T, B = w.batch * w.seq_len, w.n_embd, w.n_layer, w.vocab_size, w.seq_len, w.batch
    gemm = 2 * N * (3 * C * C + C * C + 4 * C * C + 4 * C * C) * L
    head = 2 * N * C * V
    attn = 2 * B * C * T * (T + 1) * L
    return float(gemm + head + attn)


def attention_flops(B, nh, T, hs) -> float:
    return float(2 * B * nh * hs * T * (T + 1))


def launches_per_forward(w) -> int:
    return 1 + 7 * w.n_layer + 1 + 3


def workload_desc(w) -> str:
    return (f"GPT-2 124M forward+loss: {w.n_layer} layers, {w.n_head} heads, width {w.n_embd}, "
            f"vocab {w.vocab_size}, B {w.batch}, T {w.seq_len}, bf16")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.02):
        self.samples, self.reasons, self.ok = [], set(), False
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # noqa: BLE001
            self.max_mhz = None

    def _run(self):
        nv = self.nv
        get_r = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = get_r(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": len(self.samples)}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ---------------------------------------------------------------- CPU oracle timing
def host_cores() -> int:
    """CPU cores this process may run on (its affinity mask)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover - non-Linux hosts
        return os.cpu_count() or 1


def oracle_sample(w, T_sample: int, budget_s: float, max_reps: int = 1000, threads: int | None = None, W=None):
    """Times the fp64 oracle on one sequence of T_sample tokens of the workload (full depth,
    full width, full vocabulary), repeated until budget_s has passed.  threads: BLAS thread limit
    (None: the library's default, one per core of the affinity mask).  Returns (times, threads
    used by BLAS)."""
    import oracle
    from threadpoolctl import threadpool_info, threadpool_limits
    cfg = w.model_dict()
    if W is None:
        W = seeded.to_f64(seeded.make_weights(cfg))
    idx, tgt = seeded.make_tokens(1, T_sample, w.token_high)
    idx, tgt = idx.numpy(), tgt.numpy()
    times = []
    with threadpool_limits(limits=threads):
        used = max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
        t_end = time.perf_counter() + budget_s
        while len(times) < max_reps:
            t0 = time.perf_counter()
            oracle.forward(W, cfg, idx, tgt, keep_logits=False)
            times.append(time.perf_counter() - t0)
            if time.perf_counter() > t_end:
                break
    return times, used


CPU_SAMPLE_T = 256   # tokens of the one sequence each oracle repetition runs (both CPU arms)


# ---------------------------------------------------------------- reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = seeded.WORKLOADS[WORKLOAD]
    T_sample = CPU_SAMPLE_T
    import oracle
    from threadpoolctl import threadpool_info
    cfg = w.model_dict()
    W = seeded.to_f64(seeded.make_weights(cfg))
    idx, tgt = seeded.make_tokens(1, T_sample, w.token_high)
    idx, tgt = idx.numpy(), tgt.numpy()
    for _ in range(args.warmup):
        oracle.forward(W, cfg, idx, tgt, keep_logits=False)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.forward(W, cfg, idx, tgt, keep_logits=False)
    dt = time.perf_counter() - t0
    threads = max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
    threads = min(threads, host_cores())
    value = T_sample * args.steps / dt
    sample = (f"one sequence of {T_sample} tokens of the workload (all {w.n_layer} layers, width "
              f"{w.n_embd}, vocab {w.vocab_size}) per step, fp64 numpy oracle")
    line = {
        "impl": "reference", "metric": "forward tokens/sec (GPT-2 124M, T=1024, bf16)",
        "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1000 * dt / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(w), "global_batch": w.batch, "seq_len": w.seq_len,
                   "parallelism": "none (host cores)", "sample_seq_len": T_sample},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- our arm
def time_region(fn, iters: int, stream) -> float:
    """Average ms per call of fn() over iters calls, CUDA events on `stream`."""
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(iters):
        fn()
    end.record(stream)
    torch.cuda.synchronize()
    return start.elapsed_time(end) / iters


def kernel_ops(w, native, dev, stream, only=None):
    """Each kernel of the forward pass as a closure launching it alone through the C ABI on the
    shapes the forward uses: name -> (fn, algorithmic work per launch, bound, launches per
    forward).  Inputs are allocated per kernel (only the one asked for when `only` is set)."""
    N, C, V, L = w.batch * w.seq_len, w.n_embd, w.vocab_size, w.n_layer
    hs = C // w.n_head
    g = torch.Generator(device=dev).manual_seed(7)
    bf = torch.bfloat16

    def rnd(shape, std=1.0, dtype=bf):
        return (std * torch.randn(shape, generator=g, device=dev)).to(dtype)

    def gemm(K, Nout, epi, out_dtype):
        a, Wt, bias = rnd((N, K)), rnd((Nout, K), 0.02), torch.zeros(Nout, device=dev, dtype=bf)
        out = torch.zeros((N, Nout), device=dev, dtype=out_dtype)
        return lambda: native.linear(a, Wt, bias, out=out, epilogue=epi, stream=stream)

    def attention():
        q, k, v = (rnd((w.batch, w.n_head, w.seq_len, hs)) for _ in range(3))
        y = torch.empty_like(q)
        return lambda: native.attention(q, k, v, y=y, stream=stream)

    def lm_head():
        u, wte = rnd((N, C)), rnd((V, C), 0.02)
        _, tgt = seeded.make_tokens(1, N, w.token_high)
        tgt = tgt.reshape(-1).to(dev)
        logits = torch.empty((N, V), device=dev, dtype=bf)
        loss = torch.empty((), device=dev)
        ws = native.alloc_workspace(native.lm_head_workspace_bytes(N, V), dev)
        return lambda: native.lm_head_loss(u, wte, tgt, workspace=ws, logits=logits, loss=loss, stream=stream)

    def layernorm():
        # four input / output pairs (226 MB, more than the 126 MB L2) used in turn, so every
        # launch reads its input from HBM
        xs = [rnd((N, C), 1.0, torch.float32) for _ in range(4)]
        lw, lb = torch.ones(C, device=dev, dtype=bf), torch.zeros(C, device=dev, dtype=bf)
        outs = [torch.empty((N, C), device=dev, dtype=bf) for _ in range(4)]
        turn = [0]

        def run():
            i = turn[0] = (turn[0] + 1) % 4
            native.layernorm(xs[i], lw, lb, out=outs[i], stream=stream)
        return run

    def embed():
        # three (wte, x) sets (~380 MB) used in turn, so every launch reads and writes HBM
        _, wpe = None, rnd((w.seq_len, C), 0.02)
        wtes = [rnd((V, C), 0.02) for _ in range(3)]
        xs = [torch.empty((w.batch, w.seq_len, C), device=dev) for _ in range(3)]
        idx, _ = seeded.make_tokens(w.batch, w.seq_len, w.token_high)
        idx = idx.to(dev)
        turn = [0]

        def run():
            i = turn[0] = (turn[0] + 1) % 3
            native.embed(wtes[i], wpe, idx, x=xs[i], stream=stream)
        return run

    # name -> (factory, work per launch, bound, launches per forward, kernel function)
    specs = {
        "embed": (embed, float(N * 8 + N * C * 2 + w.seq_len * C * 2 + N * C * 4), "hbm", 1),
        "gemm_c_attn": (lambda: gemm(C, 3 * C, native.GPT_EPI_STORE, bf), 2.0 * N * 3 * C * C, "tensor", L),
        "attention": (attention, attention_flops(w.batch, w.n_head, w.seq_len, hs), "tensor", L),
        "gemm_attn_proj_resid": (lambda: gemm(C, C, native.GPT_EPI_RESID, torch.float32), 2.0 * N * C * C,
                                 "tensor", L),
        "gemm_c_fc_gelu": (lambda: gemm(C, 4 * C, native.GPT_EPI_GELU, bf), 2.0 * N * 4 * C * C, "tensor", L),
        "gemm_mlp_proj_resid": (lambda: gemm(4 * C, C, native.GPT_EPI_RESID, torch.float32), 2.0 * N * 4 * C * C,
                                "tensor", L),
        "lm_head_ce": (lm_head, 2.0 * N * C * V, "tensor", 1),
        "layernorm": (layernorm, float(N * C * (4 + 2) + 4 * C), "hbm", 2 * L + 1),
    }
    return {k: (make(), work, bound, per) for k, (make, work, bound, per) in specs.items()
            if only is None or k == only}


# The kernel function (as ncu names it) behind each op of kernel_ops: ops sharing a function
# are one kernel for the roofline, whose work and time add up.
# Template arguments as ncu prints them: <BN, epilogue (0 store, 1 GELU, 2 residual add,
# 3 cross-entropy partials), GELU tanh form, A MN-major, B MN-major, CTA pair>.
KERNEL_OF = {
    "gemm_c_attn": "gemm_bf16_tc<256, 0, 0, 0, 0, 1>",
    "gemm_attn_proj_resid": "gemm_bf16_tc<256, 2, 0, 0, 0, 1>",
    "gemm_mlp_proj_resid": "gemm_bf16_tc<256, 2, 0, 0, 0, 1>",
    "gemm_c_fc_gelu": "gemm_bf16_tc<256, 1, 0, 0, 0, 1>",
    "lm_head_ce": "gemm_bf16_tc<256, 3, 0, 0, 0, 1> (+ ce_rows, loss_finalize)",
    "attention": "attention_fwd_tc",
    "layernorm": "layernorm_kernel<bf16>",
    "embed": "embed_rows_kernel<bf16, 6>",
}


def kernel_timings(w, native, dev, stream):
    """Average duration of each kernel of the forward pass launched alone."""
    ops = kernel_ops(w, native, dev, stream)
    out = {}
    for name, (fn, work, bound, per_fwd) in ops.items():
        for _ in range(3):
            fn()
        iters = 20
        ms = time_region(fn, iters, stream)
        out[name] = {"ms": ms, "work": work, "bound": bound, "per_forward": per_fwd}
    return out


def decode_bench(model, native, dev, stream, peaks, peak_src, steps: int = 64, warmup: int = 8, e2e: bool = True):
    """Incremental decoding of the same model ("nanoGPT 全局流程图", 第五阶段 generate with a key/value
    cache): one step = gpt_decode_step + gpt_sample (temperature 0.8, top_k 200, the pages'
    sample settings) for every sequence of the batch, replayed from a captured CUDA graph after a
    512-token prefill.  Each step streams the 0.25 GB of weights, more than the 126 MB L2, so no
    flush is needed.  The HBM roofline counts the bytes a step must move: every weight once
    (wte once for the head, one wpe row), the cache rows read and the new k/v rows written, and
    the fp32 logits written and read by the sampler."""
    cfg = model.cfg
    C, L, V, bs = cfg.n_embd, cfg.n_layer, cfg.vocab_size, cfg.block_size
    T0 = 512
    out = {"workload": f"GPT-2 124M bf16 decode after a {T0}-token prompt, temperature 0.8, top_k 200, "
                       f"{steps} steps replayed from a CUDA graph (decode step + sampling)"}
    entries, total = native.weights_layout(cfg)
    wpe_bytes = dict((n, k) for n, _, k in entries)["wpe"] * 2
    for B in (1, 16):
        prompt, _ = seeded.make_tokens(B, T0, 50257, seed=seeded.BASE_SEED + 600_000)
        kv = native.alloc_kv_cache(cfg, B, dev)
        ws = native.alloc_workspace(native.decode_workspace_bytes(cfg, B, T0), dev)
        logits = torch.empty((B, V), device=dev)
        tok = torch.zeros(B, dtype=torch.int64, device=dev)
        u = torch.rand(B, device=dev, generator=torch.Generator(device=dev).manual_seed(5))
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        native.prefill(cfg, model.weights, prompt.to(dev), kv, ws, sync_check=True)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side):
                native.decode_step(cfg, model.weights, tok, kv, ws, logits=logits, stream=side)
                native.sample(logits, u, 0.8, 200, out=tok, stream=side)
        torch.cuda.synchronize()
        native.prefill(cfg, model.weights, prompt.to(dev), kv, ws, sync_check=True)
        for _ in range(warmup):
            g.replay()
        torch.cuda.synchronize()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for _ in range(steps):
            g.replay()
        s1.record(stream)
        torch.cuda.synchronize()
        ms = s0.elapsed_time(s1) / steps
        status = native.check_status(ws)
        del g
        # positions T0 + warmup .. T0 + warmup + steps - 1: the mean cache length read per step
        mean_keys = T0 + warmup + (steps - 1) / 2 + 1
        bytes_step = (total - wpe_bytes + C * 2) + B * L * (mean_keys * 2 * C * 2 + 2 * C * 2) + B * V * 4 * 2
        gbs = bytes_step / (ms / 1000.0) / 1e9
        out[f"B{B}"] = {"tokens_per_s": B / (ms / 1000.0), "ms_per_token_step": ms,
                        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                     "frac": gbs / peaks["hbm_gbs"], "bytes_per_step": bytes_step,
                                     "peak_source": peak_src},
                        "status": native.status_string(status)}
    if not e2e:
        return out
    # end to end: the public generate call from host buffers, 500 new tokens ("nanoGPT 核心代码速查表",
    # sample.py settings), one sequence
    B, n_new = 1, 500
    prompt_h = torch.zeros((B, 1), dtype=torch.int64).pin_memory()
    u_h = torch.rand((n_new, B), generator=torch.Generator().manual_seed(7)).pin_memory()
    toks_h = torch.empty((B, 1 + n_new), dtype=torch.int64).pin_memory()
    kv = native.alloc_kv_cache(cfg, B, dev)
    ws = native.alloc_workspace(native.generate_workspace_bytes(cfg, B, 1, n_new), dev)
    p_d = torch.empty((B, 1), dtype=torch.int64, device=dev)
    u_d = torch.empty((n_new, B), device=dev)
    o_d = torch.empty((B, 1 + n_new), dtype=torch.int64, device=dev)

    def gen():
        p_d.copy_(prompt_h, non_blocking=True)
        u_d.copy_(u_h, non_blocking=True)
        native.generate(cfg, model.weights, p_d, n_new, u_d, 0.8, 200, kv_cache=kv, workspace=ws, out=o_d)
        toks_h.copy_(o_d, non_blocking=True)
        stream.synchronize()

    gen()
    t0 = time.perf_counter()
    reps = 3
    for _ in range(reps):
        gen()
    dt = (time.perf_counter() - t0) / reps
    out["generate_e2e"] = {"tokens_per_s": B * n_new / dt, "ms_per_call": dt * 1000.0, "new_tokens": n_new,
                           "batch": B, "prompt": 1,
                           "note": "host wall clock around gpt_generate with pinned host copies in and out; "
                                   "launched eagerly (no graph), one launch sequence per token"}
    return out


def head_last_bench(native, dev, stream, peaks, peak_src, reps: int = 20):
    """The inference branch's head ("nanoGPT 全局流程图", §3.2 ④, logits [B, 1, V]): gpt_lm_head_last,
    ln_f of each sequence's last residual row and the product with the tied wte, at the GPT-2
    124M (B 12) and XL (B 4, the [4, 1, 50304] output of the XL configuration) shapes.  HBM-bound:
    algorithmic bytes = wte once (V C bf16) + the B fp32 rows + ln_f weight and bias + the bf16
    logits.  Two wte copies are used in turn so that no launch finds its table in the L2."""
    out = {}
    V = 50304
    for name, B, C in (("gpt2", 12, 768), ("gpt2-xl", 4, 1600)):
        g = torch.Generator(device=dev).manual_seed(13)
        x = torch.randn((B, 1024, C), device=dev, generator=g)
        wtes = [(0.02 * torch.randn((V, C), device=dev, generator=g)).to(torch.bfloat16) for _ in range(2)]
        lw = torch.ones(C, device=dev, dtype=torch.bfloat16)
        lb = torch.zeros(C, device=dev, dtype=torch.bfloat16)
        logits = torch.empty((B, V), device=dev, dtype=torch.bfloat16)
        turn = [0]

        def run():
            i = turn[0] = (turn[0] + 1) % 2
            native.lm_head_last(x, lw, lb, wtes[i], logits=logits, stream=stream)
        for _ in range(4):
            run()
        ms = time_region(run, reps, stream)
        nbytes = V * C * 2 + B * C * 4 + 2 * C * 2 + B * V * 2
        gbs = nbytes / (ms / 1000.0) / 1e9
        out[name] = {"workload": f"ln_f + tied head of the last position, B {B}, C {C}, V {V}, bf16",
                     "us_per_launch": ms * 1000.0,
                     "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                  "frac": gbs / peaks["hbm_gbs"], "bytes_per_launch": nbytes,
                                  "peak_source": peak_src}}
        del x, wtes
    return out


def adamw_bench(model, native, dev, stream, peaks, peak_src, steps: int = 20, warmup: int = 3):
    """One optimizer step over GPT-2 124M ("nanoGPT 全局流程图" 3.6 and 优化器配置): the global
    gradient norm, clipping to 1.0, AdamW (betas 0.9/0.95, weight decay 0.1 on matrices) on fp32
    master parameters and moments, and the bf16 copy into the packed weights the forward reads.
    Gradients are seeded N(0, 0.05^2) (norm ~560: clipping active).  Algorithmic traffic per
    parameter: 4 B (norm: read g) + 16 B (read p, g, m, v) + 12 B (write p, m, v) + 2 B (bf16
    copy) = 34 B; the 2 GB of fp32 arrays exceed the 126 MB L2, so no flush is needed."""
    cfg = model.cfg
    g = torch.randn(native.param_elems(cfg), device=dev, generator=torch.Generator(device=dev).manual_seed(11))
    g.mul_(0.05)
    entries, _ = native.weights_layout(cfg)
    n_params = sum(k for _, _, k in entries)
    p = torch.zeros_like(g)
    es = 2
    for name, off, numel in entries:       # master copy of the current weights
        p[off // es: off // es + numel] = model.weights[off: off + numel * es].view(torch.bfloat16).float()
    m = torch.zeros_like(g)
    v = torch.zeros_like(g)
    ws = native.alloc_workspace(native.LIB.gpt_adamw_workspace_bytes(), dev)
    norm = torch.empty((), device=dev)
    native.adamw_step(cfg, p, g, m, v, 1, 6e-4, weights=model.weights, grad_norm=norm, workspace=ws,
                      sync_check=True)
    for i in range(warmup):
        native.adamw_step(cfg, p, g, m, v, 2 + i, 6e-4, weights=model.weights, grad_norm=norm, workspace=ws)
    torch.cuda.synchronize()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for i in range(steps):
        native.adamw_step(cfg, p, g, m, v, 2 + warmup + i, 6e-4, weights=model.weights, grad_norm=norm,
                          workspace=ws)
    s1.record(stream)
    torch.cuda.synchronize()
    ms = s0.elapsed_time(s1) / steps
    bytes_step = 34 * n_params
    gbs = bytes_step / (ms / 1000.0) / 1e9
    return {"workload": "AdamW step over GPT-2 124M (124,475,904 fp32 parameters): grad norm + clip 1.0 + "
                        "update + bf16 copy into the packed weights",
            "ms_per_step": ms, "params_per_s": n_params / (ms / 1000.0),
            "grad_norm": float(norm),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "bytes_per_step": bytes_step, "peak_source": peak_src},
            "gpu_launches_per_step": 2}


def backward_pieces_bench(native, dev, stream, peaks, peak_src, reps: int = 10):
    """Backward steps at the GPT-2 124M shapes ("nanoGPT 全局流程图" 3.4): the cross-entropy gradient
    over the full logits [12288, 50304] bf16 (reads the logits twice, writes the gradient:
    3 x 1.24 GB), one LayerNorm backward [12288, 768] (reads dy and x, reads and writes dx:
    4 x 37.7 MB) and the attention backward of one layer.  Inputs exceed the L2."""
    rows, V, C = 12 * 1024, 50304, 768
    g = torch.Generator(device=dev).manual_seed(3)
    z = (torch.randn((rows, V), device=dev, generator=g) * 1.5).to(torch.bfloat16)
    tgt = torch.randint(0, 50257, (rows,), device=dev, generator=g)
    sc = torch.tensor([0.0, float(rows)], dtype=torch.float64, device=dev)
    dz = torch.empty_like(z)
    x = torch.randn((rows, C), device=dev, generator=g)
    dy = torch.randn((rows, C), device=dev, generator=g) * 0.01
    w = torch.ones(C, device=dev, dtype=torch.bfloat16)
    dx = torch.zeros_like(x)
    dw = torch.empty(C, device=dev)
    db = torch.empty(C, device=dev)
    # attention backward at the attention workload (B 12, 12 heads, T 1024, hs 64): algorithmic work
    # = the five products of the flash backward (S recomputed, dP, dV, dQ, dK) over the causal pairs,
    # 5 * 2 * hs * T (T + 1) / 2 per (b, h); the kernels run seven (S and dP in both passes).
    Ba, nh, T, hs = 12, 12, 1024, 64
    q, k, v, do_ = (torch.randn((Ba, nh, T, hs), device=dev, generator=g).to(torch.bfloat16) for _ in range(4))
    y, lse = native.attention_train(q, k, v)
    dqkv = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    aws = native.alloc_workspace(native.LIB.gpt_attention_backward_workspace_bytes(Ba, nh, T), dev)
    attn_flops = 5 * 2 * hs * T * (T + 1) / 2 * Ba * nh
    out = {}
    for name, fn, nbytes in (
            ("cross_entropy_backward", lambda: native.cross_entropy_backward(z, tgt, sc, dlogits=dz), 3 * rows * V * 2),
            ("layernorm_backward", lambda: native.layernorm_backward(dy, x, w, dx=dx, accumulate=True, dw=dw, db=db),
             4 * rows * C * 4),
            ("attention_backward", lambda: native.attention_backward(q, k, v, y, do_, lse, out=dqkv, workspace=aws),
             None)):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / reps
        if nbytes is None:
            tf = attn_flops / (ms / 1000.0) / 1e12
            out[name] = {"ms": ms, "workload": "causal attention backward B 12, 12 heads, T 1024, hs 64, bf16",
                         "roofline": {"bound": "tensor", "achieved": tf, "peak": peaks["bf16_tflops"],
                                      "unit": "TFLOP/s", "frac": tf / peaks["bf16_tflops"], "flops": attn_flops,
                                      "peak_source": peak_src}}
            continue
        gbs = nbytes / (ms / 1000.0) / 1e9
        out[name] = {"ms": ms, "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                            "frac": gbs / peaks["hbm_gbs"], "bytes": nbytes, "peak_source": peak_src}}
    return out


def train_bench(native, dev, stream, world, rank, dist, steps: int = 5, warmup: int = 2):
    """One training step of GPT-2 124M per rank ("nanoGPT 全局流程图" 3.2-3.6), B 12, T 1024 per GPU
    (weak scaling): training forward keeping activations, backward, AdamW (clip 1.0, decay on
    matrices, get_lr); with N > 1 the loss terms and the gradients are all-reduced (NCCL) between
    the backward's start and the optimizer.  Synthetic seeded data, GPT-2-init weights.  Time per
    phase from CUDA events on one extra step."""
    from decoder_only_transformer_causal_b200 import GPT, GPTConfig, Trainer
    from decoder_only_transformer_causal_b200.data_parallel import train_step_sharded
    w = seeded.WORKLOADS[WORKLOAD]
    W = seeded.make_weights(w.model_dict(), seed=seeded.BASE_SEED + 31, device=str(dev))
    model = GPT(GPTConfig.from_dict(w.model_dict()), W, dev)
    tr = Trainer(model, W, w.batch, w.seq_len)
    idx, tgt = seeded.make_tokens(w.batch, w.seq_len, w.token_high, seed=seeded.BASE_SEED + 700 + rank)
    idx, tgt = idx.to(dev), tgt.to(dev)
    step = (lambda: train_step_sharded(tr, idx, tgt)) if world > 1 else (lambda: tr.step(idx, tgt))
    for _ in range(warmup):
        step()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        last = step()
    e1.record(stream)
    torch.cuda.synchronize()
    t = torch.tensor([e0.elapsed_time(e1) / steps], device=dev)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms = float(t)
    out = {"workload": f"GPT-2 124M training step, B {w.batch} x T {w.seq_len} per GPU, bf16 weights/activations, "
                       "fp32 master weights and Adam moments" + (f", data-parallel over {world} GPUs" if world > 1 else ""),
           "tokens_per_s": world * w.batch * w.seq_len / (ms / 1000.0), "ms_per_step": ms}
    if world == 1:
        # phase split of one more step (single GPU only: with N > 1 a step without the two
        # all-reduces would let the replicated weights of the ranks diverge)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        cfg = model.cfg
        ev[0].record(stream)
        native.forward_train(cfg, model.weights, idx, tgt, tr.acts, tr.fws, loss=tr.loss)
        ev[1].record(stream)
        tr.grads.zero_()
        native.backward(cfg, model.weights, idx, tgt, tr.acts, tr.grads, tr.bws)
        ev[2].record(stream)
        tr.opt.step(tr.grads)
        ev[3].record(stream)
        torch.cuda.synchronize()
        out["phase_ms"] = {"forward_train": ev[0].elapsed_time(ev[1]), "backward": ev[1].elapsed_time(ev[2]),
                           "adamw": ev[2].elapsed_time(ev[3])}
        out["loss_after"] = float(tr.loss)
    else:
        out["loss_after"] = float(last)
    del tr, model
    return out


def adamw_only(args):
    from decoder_only_transformer_causal_b200 import GPT, GPTConfig, native
    dev = torch.device("cuda", 0)
    w = seeded.WORKLOADS[WORKLOAD]
    model = GPT(GPTConfig.from_dict(w.model_dict()), seeded.make_weights(w.model_dict(), device=str(dev)), dev)
    peaks, peak_src = load_peaks()
    d = adamw_bench(model, native, dev, torch.cuda.current_stream(dev), peaks, peak_src, steps=args.steps,
                    warmup=max(3, args.warmup))
    print(json.dumps({"adamw": d}), flush=True)
    return 0


def decode_only(args):
    from decoder_only_transformer_causal_b200 import GPT, GPTConfig, native
    dev = torch.device("cuda", 0)
    w = seeded.WORKLOADS[WORKLOAD]
    model = GPT(GPTConfig.from_dict(w.model_dict()), seeded.make_weights(w.model_dict(), device=str(dev)), dev)
    peaks, peak_src = load_peaks()
    d = decode_bench(model, native, dev, torch.cuda.current_stream(dev), peaks, peak_src, steps=args.steps,
                     warmup=max(3, args.warmup), e2e=not args.no_e2e)
    print(json.dumps({"decode": d}), flush=True)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.profile_kernel:
        return profile_kernel(args)
    if args.decode_only:
        return decode_only(args)
    if args.adamw_only:
        return adamw_only(args)
    if args.train_only:
        dev = torch.device("cuda", 0)
        from decoder_only_transformer_causal_b200 import native
        print(json.dumps({"train": train_bench(native, dev, torch.cuda.current_stream(dev), 1, 0, None,
                                               steps=args.steps, warmup=max(1, args.warmup))}), flush=True)
        return 0
    assert args.warmup >= 3, "at least 3 warm-up steps"
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    from decoder_only_transformer_causal_b200 import GPT, GPTConfig, native
    from decoder_only_transformer_causal_b200.data_parallel import allreduce_loss_terms

    w = seeded.WORKLOADS[WORKLOAD]
    cfg = GPTConfig.from_dict(w.model_dict())
    # replicated weights (the same draw on every rank); each rank's batch shard is its own draw
    model = GPT(cfg, seeded.make_weights(w.model_dict(), seed=seeded.BASE_SEED + 17, device=str(dev)), dev)
    idx_h, tgt_h = seeded.make_tokens(w.batch, w.seq_len, w.token_high, seed=seeded.BASE_SEED + 100_000 + rank)
    idx, tgt = idx_h.to(dev), tgt_h.to(dev)
    ws = model.workspace(w.batch, w.seq_len)
    logits = torch.empty((w.batch, w.seq_len, w.vocab_size), dtype=torch.bfloat16, device=dev)
    loss = torch.empty((), dtype=torch.float32, device=dev)
    sc = torch.empty(2, dtype=torch.float64, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        native.forward(cfg, model.weights, idx, tgt, ws, logits=logits, loss=loss, loss_sum_count=sc,
                       stream=stream)
        if dist is not None:
            allreduce_loss_terms(sc)     # global {sum of row losses, counted rows}

    # correctness guard before timing: the status word must be clean
    native.forward(cfg, model.weights, idx, tgt, ws, logits=logits, loss=loss, sync_check=True)
    for _ in range(args.warmup):
        step()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        start.record(stream)
        for _ in range(args.steps):
            step()
        end.record(stream)
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    ms_total = start.elapsed_time(end)
    t = torch.tensor([ms_total], device=dev)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_total = float(t)
    status = native.check_status(ws)
    tokens = world * w.batch * w.seq_len * args.steps
    value = tokens / (ms_total / 1000.0)
    ms_step = ms_total / args.steps

    # end to end through the public call with host buffers (pinned), loss read back each step
    idx_p, tgt_p = idx_h.pin_memory(), tgt_h.pin_memory()
    for _ in range(3):
        model.forward_host(idx_p, tgt_p)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_steps = max(3, args.steps // 2)
    e_start.record(stream)
    for _ in range(e_steps):
        model.forward_host(idx_p, tgt_p)
    e_end.record(stream)
    torch.cuda.synchronize()
    te = torch.tensor([e_start.elapsed_time(e_end)], device=dev)
    if dist is not None:
        dist.all_reduce(te, op=dist.ReduceOp.MAX)
    e2e_value = world * w.batch * w.seq_len * e_steps / (float(te) / 1000.0)

    peaks, peak_src = load_peaks()
    line = None
    if rank == 0:
        fwd_fl = forward_flops(w)
        line = {
            "metric": "forward tokens/sec (GPT-2 124M, T=1024, bf16)",
            "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded GPT-2-init weights, uniform token ids)",
            "config": {"workload": workload_desc(w), "global_batch": w.batch * world, "seq_len": w.seq_len,
                       "parallelism": f"dp{world}",
                       "l2": "no flush: each step touches > 1.4 GB (weights 0.25 GB, logits 1.24 GB) vs 126 MB L2"},
            "status": native.status_string(status),
            "e2e": {"value": e2e_value, "unit": "tokens/s",
                    "h2d_bytes_per_step": int(idx_h.numel() * 8 + tgt_h.numel() * 8),
                    "d2h_bytes_per_step": 4},
            "gpu_launches": launches_per_forward(w) * args.steps,
            "forward": {"tflops": fwd_fl / (ms_step / 1000.0) / 1e12 * world,
                        "flops_per_step_per_gpu": fwd_fl,
                        "frac_of_sustained_bf16": fwd_fl / (ms_step / 1000.0) / 1e12 /
                        peaks["bf16_tflops_sustained"], "peak_source": peak_src},
            "clocks": clocks.summary(),
        }
    if not args.no_kernels and rank == 0:
        kt = kernel_timings(w, native, dev, stream)
        # dominant kernel: the kernel function with the largest time share of one forward
        share = {k: v["ms"] * v["per_forward"] for k, v in kt.items()}
        by_fn = {}
        for k, v in kt.items():
            f = by_fn.setdefault(KERNEL_OF[k], {"ms": 0.0, "work": 0.0, "launches": 0, "bound": v["bound"]})
            f["ms"] += v["ms"] * v["per_forward"]
            f["work"] += v["work"] * v["per_forward"]
            f["launches"] += v["per_forward"]
        dom = max(by_fn, key=lambda f: by_fn[f]["ms"])
        d = by_fn[dom]
        ms_launch = d["ms"] / d["launches"]
        work_launch = d["work"] / d["launches"]
        if d["bound"] == "tensor":
            achieved = work_launch / (ms_launch / 1000.0) / 1e12
            peak = peaks["bf16_tflops"]
            unit = "TFLOP/s"
        else:
            achieved = work_launch / (ms_launch / 1000.0) / 1e9
            peak = peaks["hbm_gbs"]
            unit = "GB/s"
        line["roofline"] = {"kernel": dom, "bound": d["bound"], "achieved": achieved, "peak": peak,
                            "unit": unit, "frac": achieved / peak, "traffic": traffic_for(dom),
                            "peak_source": f"{peak_src} (burst, kernel timed alone)",
                            "work_per_launch": work_launch, "ms_per_launch": ms_launch,
                            "launches_per_forward": d["launches"],
                            "share_of_forward": d["ms"] / sum(share.values())}
        a = kt["attention"]
        a_tf = a["work"] / (a["ms"] / 1000.0) / 1e12
        line["attention"] = {"workload": "causal attention B 12, 12 heads, T 1024, hs 64, bf16",
                             "tflops": a_tf, "ms": a["ms"], "frac_of_bf16_peak": a_tf / peaks["bf16_tflops"],
                             "flops": a["work"], "peak_source": peak_src}
        line["kernels_ms_per_forward"] = {k: round(v, 4) for k, v in share.items()}
        # the HBM-bound kernels against the copy bandwidth (inputs rotated past the L2)
        line["memory_bound"] = {
            k: {"kernel": KERNEL_OF[k], "us_per_launch": v["ms"] * 1000.0,
                "achieved_gbs": v["work"] / (v["ms"] / 1000.0) / 1e9, "peak_gbs": peaks["hbm_gbs"],
                "frac": v["work"] / (v["ms"] / 1000.0) / 1e9 / peaks["hbm_gbs"], "bytes_per_launch": v["work"],
                "peak_source": peak_src}
            for k, v in kt.items() if v["bound"] == "hbm"}
    # Single-GPU measurements (decode, optimizer, backward pieces) run in the N = 1 line only, so
    # that the other ranks of an N > 1 run do not idle in a collective while rank 0 works alone.
    if rank == 0 and world == 1 and not args.no_kernels:
        line["last_position"] = head_last_bench(native, dev, stream, peaks, peak_src)
        line["decode"] = decode_bench(model, native, dev, stream, peaks, peak_src)
        line["adamw"] = adamw_bench(model, native, dev, stream, peaks, peak_src)
        line["backward_pieces"] = backward_pieces_bench(native, dev, stream, peaks, peak_src)
    if not args.no_kernels:
        tr = train_bench(native, dev, stream, world, rank, dist)
        if rank == 0:
            line["train"] = tr
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        W64 = seeded.to_f64(seeded.make_weights(w.model_dict()))
        cores = host_cores()
        times, threads = oracle_sample(w, CPU_SAMPLE_T, budget_s=12.0, threads=cores, W=W64)
        tok_s = CPU_SAMPLE_T * len(times) / sum(times)
        t1, _ = oracle_sample(w, 64, budget_s=6.0, threads=1, W=W64)
        line["cpu_baseline"] = {"value": tok_s, "unit": "tokens/s", "cores": min(threads, cores), "kind": "oracle",
                                "host_cores": cores,
                                "sample": f"{len(times)} x one sequence of {CPU_SAMPLE_T} tokens of the workload (all "
                                          f"{w.n_layer} layers, full vocab), fp64 numpy oracle",
                                "one_core": {"value": 64 * len(t1) / sum(t1), "unit": "tokens/s", "cores": 1,
                                             "sample": f"{len(t1)} x one sequence of 64 tokens, BLAS limited to "
                                                       "one thread"}}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def profile_kernel(args):
    """Launches one kernel of the forward alone (for an ncu capture of a single kernel)."""
    from decoder_only_transformer_causal_b200 import native
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    w = seeded.WORKLOADS[WORKLOAD]
    fn, work, bound, _ = kernel_ops(w, native, dev, stream, only=args.profile_kernel)[args.profile_kernel]
    for _ in range(args.warmup):
        fn()
    ms = time_region(fn, args.steps, stream)
    print(json.dumps({"kernel": args.profile_kernel, "ms": ms, "work": work, "bound": bound}))
    return 0


def traffic_for(kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if it was taken on the
    current source of that kernel; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")  # written from an ncu capture of the current source
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel)
    if not e:
        return None
    src = os.path.join(ROOT, e["source"])
    if not os.path.exists(src):
        return None
    with open(src, "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()[:16]
    return e["bytes_per_launch"] if sha == e.get("source_sha") else None


if __name__ == "__main__":
    sys.exit(main())
