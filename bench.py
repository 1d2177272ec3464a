"""Benchmark of one TwoTower denoiser refinement step on B200 (one process per GPU).

A step is one pass of the whole hot path over one batch: adaLN-single conditioning, modulated
RMSNorm prologue, Eq. (1) layer-aligned denoiser attention, gated residual and ConfidenceSample
over the vocabulary logits (the paper "Nemotron-TwoTower: Diffusion Language Modeling with
Pretrained AR Context", §2.1-§2.2, Algorithm 2). The headline workload is the bf16 batch-generation
step: per GPU 64 sequences with 16384 context tokens + a block of S=16 at step t=8 of T=16
(tau = 9/16), 32 query / 2 kv heads, head dim 128, adaLN width 2048, vocabulary 131072, gamma
0.8, seeded synthetic inputs. Extra keys report the decode step (8 sequences, 4096 context
tokens), the attention alone on every workload, and the block-sweep unmask table (committed
tokens per step for S x temperature x gamma).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-extras]

N > 1 runs under torchrun: every rank processes its own 64 sequences (weak scaling; sequences
are independent, so there is no data-path collective); the elapsed time is the max over ranks.
`--impl reference` times the CPU fp64 oracle on the host cores instead (the comparison arm).
Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "denoise-step attn query-tok/s, KV-read GB/s vs HBM peak; unmask steps/s"
# the headline: the batch-generation workload, the largest configuration that fits one GPU
WORKLOAD = "batch_bf16"
# RefinementStep schedules (how the step's three independent branches go on streams)
SCHEDULE_TEXT = {
    "branches": "each step three concurrent branches on forked streams",
    "attn_then_unmask": "each step: attention then unmask on one forked stream, the modulation alongside",
    "unmask_then_attn": "each step: unmask then attention on one forked stream, the modulation alongside",
    "serial": "each step on one stream",
}


def shard_range(global_batch: int, world: int, rank: int):
    """Sequences [lo, hi) owned by `rank` when `global_batch` sequences are split evenly."""
    base, extra = divmod(global_batch, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a per-rank float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def workload_desc(w) -> str:
    a = w.attn
    return (f"{w.name}: B={a.batch} per GPU, ctx {a.ctx_lens[0]} + S={a.block_size}, {a.num_q_heads} q / "
            f"{a.num_kv_heads} kv heads, d={a.head_dim}, adaLN D={w.hidden}, vocab {w.vocab}, gamma {w.gamma}")


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "of measured"
    return 6650.0, "of fallback"


def measured_tensor_peak():
    """Dense bf16 tensor peak in TFLOP/s for a kernel timed alone (the burst figure), and its source."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        if "bf16_tflops" in d:
            return float(d["bf16_tflops"]), "of measured"
    return 1590.0, "of fallback"


# ------------------------------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons in the background."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period_ms: int = 100):
        self.gpu = gpu_index
        self.period = period_ms
        self.samples = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 f"-lms={self.period}"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), [x.strip() for x in line.split(",")]))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self, t0: float, t1: float):
        win = [s for (t, s) in self.samples if t0 <= t <= t1]
        if not win:
            win = [s for (_, s) in self.samples]
        if not win:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(s[1]) for s in win if s[1].replace(".", "").isdigit()]
        smax = [float(s[2]) for s in win if s[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for s in win for n, v in zip(names, s[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(win)}


# ------------------------------------------------------------------------------------------ oracle arm
def oracle_token_sample(w, inp, ad, logits, b: int, s: int):
    """The oracle's full step for ONE query token (sequence b, block position s): Eq. (1) for all
    query heads of that position over L_b + S keys, adaLN-single for its sequence plus the
    prologue/residual of its token row, and ConfidenceSample statistics of its logits row."""
    import numpy as np
    from oracle import tt_oracle as O
    f64 = lambda t: t.double().numpy()
    O.denoise_attention(f64(inp.q[b:b + 1, s:s + 1]), f64(inp.k_blk[b:b + 1]), f64(inp.v_blk[b:b + 1]),
                        f64(inp.k_ctx[b:b + 1]), f64(inp.v_ctx[b:b + 1]), [int(inp.ctx_lens[b])])
    mod = O.adaln_cond(f64(ad.tau[b:b + 1]), f64(ad.w1), f64(ad.b1), f64(ad.w2), f64(ad.b2), f64(ad.w3),
                       f64(ad.b3), f64(ad.layer_emb))
    O.adaln_norm_modulate(f64(ad.h[b:b + 1, s:s + 1]), f64(ad.norm_w), mod)
    O.adaln_gated_residual(f64(ad.h[b:b + 1, s:s + 1]), f64(ad.f[b:b + 1, s:s + 1]), mod)
    conf, arg = O.confidence_argmax(f64(logits[b:b + 1, s:s + 1]), w.inv_temperature)
    O.confidence_commit(np.full((1, 1), 3), np.ones((1, 1), bool), conf, arg, w.gamma)


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def host_inputs(w, seed_offset: int = 0):
    """Seeded host tensors of one step of workload w: attention inputs, adaLN inputs (tau = the
    workload's fixed time, else 1: the first refinement step, everything masked) and logits."""
    from denoiser_attention_b200 import synth
    inp = synth.attention_inputs(w.attn, seed=w.seed + seed_offset)
    B, S = w.attn.batch, w.attn.block_size
    tau = [w.tau if w.tau is not None else 1.0] * B
    ad = synth.adaln_inputs(B, S, w.hidden, tau, seed=w.seed + 100 + seed_offset, dtype=w.attn.dtype)
    logits = synth.workload_logits(w, seed=w.seed + seed_offset)
    return inp, ad, logits


def run_reference(args):
    """The comparison arm: the CPU fp64 oracle on the host cores, same config/metric/unit."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from denoiser_attention_b200 import synth
    w = synth.workload(args.workload)
    inp, ad, logits = host_inputs(w)
    B, S = w.attn.batch, w.attn.block_size
    # calibrate one token sample, then size each step so that warmup + steps take ~2 minutes
    t0 = time.perf_counter()
    oracle_token_sample(w, inp, ad, logits, 0, 0)
    t_tok = max(time.perf_counter() - t0, 1e-4)
    per_step = max(1, min(B * S, int(120.0 / ((args.steps + args.warmup) * t_tok))))
    k = 0
    for _ in range(args.warmup):
        for _ in range(per_step):
            oracle_token_sample(w, inp, ad, logits, (k // S) % B, k % S)
            k += 1
    t0 = time.perf_counter()
    for _ in range(args.steps):
        for _ in range(per_step):
            oracle_token_sample(w, inp, ad, logits, (k // S) % B, k % S)
            k += 1
    el = time.perf_counter() - t0
    tokens = args.steps * per_step
    value = tokens / el
    cores = blas_threads()
    sample = f"{per_step} query token(s) per step (all heads, adaLN, unmask of that position), {tokens} timed"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "query-tok/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(w), "global_batch": B, "seq_len": w.attn.ctx_lens[0] + S,
                   "parallelism": "cpu oracle"},
        "cpu_baseline": {"value": value, "unit": "query-tok/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "query-tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


# ------------------------------------------------------------------------------------------ our arm
def kv_bytes_of(a) -> int:
    """Algorithmic K/V bytes of one attention launch: (context + block) tokens x kv heads x
    (K + V) x d x 2 bytes (bf16)."""
    return sum(int(L) + a.block_size for L in a.ctx_lens) * a.num_kv_heads * a.head_dim * 2 * 2


def attn_flops_of(a) -> int:
    """Tensor-core FLOPs of one attention launch: 4 G S d per key and kv head (QK^T and PV)."""
    G = a.num_q_heads // a.num_kv_heads
    return sum(int(L) + a.block_size for L in a.ctx_lens) * a.num_kv_heads * 4 * G * a.block_size * a.head_dim


class StepRun:
    """Device buffers of one workload (rotating input sets, more than 4x L2 in total) and its
    RefinementStep, with a CUDA graph of M steps holding per-branch timing events."""

    def __init__(self, w, inp, ad, logits, dev, schedule):
        import torch
        from denoiser_attention_b200 import api
        B, S = w.attn.batch, w.attn.block_size
        self.w = w
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        self.set_bytes = sum(t.numel() * t.element_size() for t in (inp.k_ctx, inp.v_ctx, logits, inp.q, ad.h, ad.f))
        self.n_sets = max(2, math.ceil(4 * l2 / self.set_bytes))
        weights = {k: getattr(ad, k).to(dev) for k in ("w1", "b1", "w2", "b2", "w3", "b3", "layer_emb", "norm_w")}
        self.sets = []
        for _ in range(self.n_sets):
            self.sets.append(api.StepBuffers(
                tau=ad.tau.to(dev), h=ad.h.to(dev), f=ad.f.to(dev), q=inp.q.to(dev), k_blk=inp.k_blk.to(dev),
                v_blk=inp.v_blk.to(dev), k_ctx=inp.k_ctx.to(dev), v_ctx=inp.v_ctx.to(dev),
                ctx_lens=inp.ctx_lens.to(dev),
                page_table=None if inp.page_table is None else inp.page_table.to(dev), logits=logits.to(dev),
                tokens=torch.full((B, S), 3, dtype=torch.int32, device=dev),
                is_masked=torch.ones((B, S), dtype=torch.uint8, device=dev)))
        self.step = api.RefinementStep(weights, gamma=w.gamma, inv_temperature=w.inv_temperature,
                                       page_size=w.attn.page_size, ctx_stride=inp.ctx_stride, schedule=schedule)
        self.outs = [torch.empty_like(s.q) for s in self.sets]
        for i in range(self.n_sets):   # eager warm-up: kernel attributes, workspaces
            self.step.run(self.sets[i], out_attn=self.outs[i])
        torch.cuda.synchronize()
        self.cap_stream = torch.cuda.Stream(device=dev)

    def capture(self, n_steps, with_events):
        import torch
        mk = lambda: torch.cuda.Event(enable_timing=True, external=True)
        ev = [tuple(mk() for _ in range(8)) for _ in range(n_steps)] if with_events else None
        g = torch.cuda.CUDAGraph()
        self.cap_stream.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(self.cap_stream):
            with torch.cuda.graph(g, stream=self.cap_stream):
                for j in range(n_steps):
                    k = j % self.n_sets
                    self.step.run(self.sets[k], out_attn=self.outs[k], events=None if ev is None else ev[j])
        torch.cuda.current_stream().wait_stream(self.cap_stream)
        torch.cuda.synchronize()
        return g, ev


def isolated_ms(op, sets, outs, cap_stream, reps: int = 20):
    """Mean device time of op(buffers, out) from a CUDA graph of one launch per rotating input set,
    replayed back to back (the sets together exceed L2, so each launch reads from HBM)."""
    import torch
    g = torch.cuda.CUDAGraph()
    cap_stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap_stream):
        with torch.cuda.graph(g, stream=cap_stream):
            for b, o in zip(sets, outs):
                op(b, o)
    torch.cuda.current_stream().wait_stream(cap_stream)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / (reps * len(sets))
    del g
    return ms


def attn_op(step):
    from denoiser_attention_b200 import api
    return lambda b, o: api.denoise_attention(b.q, b.k_blk, b.v_blk, b.k_ctx, b.v_ctx, b.ctx_lens,
                                              page_table=b.page_table, page_size=step.page_size,
                                              ctx_stride=step.ctx_stride, softmax_scale=step.softmax_scale, out=o)


def unmask_op(step):
    from denoiser_attention_b200 import api
    return lambda b, o: api.unmask_step(b.logits, b.tokens, b.is_masked, gamma=step.gamma,
                                        inv_temperature=step.inv_temperature, mask_token_id=step.mask_token_id,
                                        want_conf=False)


def run_ours(args):
    import torch
    import torch.distributed as dist
    from denoiser_attention_b200 import api, build, synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    build.build()

    w = synth.workload(args.workload)
    B, S = w.attn.batch, w.attn.block_size
    global_batch = B * world
    lo, hi = shard_range(global_batch, world, rank)
    assert hi - lo == B
    inp, ad, logits = host_inputs(w, seed_offset=lo)     # this rank's sequences
    run = StepRun(w, inp, ad, logits, dev, args.schedule)
    M = 2 * run.n_sets
    # the timed graph holds the steps only; the per-kernel events live in a second graph of the same
    # steps, replayed after the timed region (an event node between two kernels ends the
    # programmatic overlap of the second kernel's start with the first one's end)
    g, _ = run.capture(M, with_events=False)

    # warm-up: at least W steps and about half a second, untimed
    reps_w = max(1, math.ceil(args.warmup / M))
    clocks = ClockSampler(local)
    clocks.start()
    t_w = time.time()
    while True:
        for _ in range(reps_w):
            g.replay()
        torch.cuda.synchronize()
        if time.time() - t_w > 0.5:
            break
    # ---- timed region: exactly K steps (R replays of M steps, then a remainder graph)
    R, rem = divmod(args.steps, M)
    g_rem = run.capture(rem, with_events=False)[0] if rem else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_c0 = time.time()
    start.record()
    for _ in range(R):
        g.replay()
    if g_rem is not None:
        g_rem.replay()
    stop.record()
    torch.cuda.synchronize()
    t_c1 = time.time()
    if world > 1:
        dist.barrier()
    clocks.stop()
    ms = start.elapsed_time(stop)
    ms_max = max_over_ranks(ms, dev)
    ms_per_step = ms_max / args.steps

    # per-kernel durations from the events of a replay of the same M steps with event nodes, run on
    # one stream so that each event pair spans its own kernels only (with concurrent branches the
    # unmask's pair would also span the attention it waits behind)
    del g, g_rem
    schedule = run.step.schedule
    run.step.schedule = "serial"
    g_ev, ev = run.capture(M, with_events=True)
    run.step.schedule = schedule
    for _ in range(3):
        g_ev.replay()
    torch.cuda.synchronize()
    attn_ms = max_over_ranks(statistics.mean(e[0].elapsed_time(e[1]) for e in ev), dev)
    unmask_ms = max_over_ranks(statistics.mean(e[2].elapsed_time(e[3]) for e in ev), dev)
    cond_ms, normres_ms = (max_over_ranks(statistics.mean(e[i].elapsed_time(e[i + 1]) for e in ev), dev)
                           for i in (4, 6))
    del g_ev
    # the same two kernels alone (own graphs over the same rotating input sets), for context: inside
    # the step they share the GPU with the other branches
    attn_iso_ms = max_over_ranks(isolated_ms(attn_op(run.step), run.sets, run.outs, run.cap_stream), dev)
    unmask_iso_ms = max_over_ranks(isolated_ms(unmask_op(run.step), run.sets, run.outs, run.cap_stream), dev)

    a = w.attn
    kv_bytes = kv_bytes_of(a)
    logit_bytes = B * S * w.vocab * 2
    peak, peak_src = measured_peaks()
    attn_gbs = kv_bytes / (attn_ms * 1e-3) / 1e9
    unmask_gbs = logit_bytes / (unmask_ms * 1e-3) / 1e9
    traffic = measured_traffic(args.workload)
    launches_per_step = api.RefinementStep.LAUNCHES

    # ---- end to end through the public API with host buffers (pinned), copies timed
    e2e = run_e2e(run.step, inp, ad, logits, w, dev, args, world)
    del run
    torch.cuda.empty_cache()

    extras = None
    if rank == 0 and world == 1 and not args.no_extras:
        extras = run_extras(args, dev, peak)

    result = None
    if rank == 0:
        value = global_batch * S / (ms_max * 1e-3 / args.steps)
        cpu = cpu_baseline(w, inp, ad, logits) if world == 1 else None
        result = {
            "metric": METRIC, "value": value, "unit": "query-tok/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": workload_desc(w), "global_batch": global_batch,
                       "seq_len": a.ctx_lens[0] + S, "parallelism": f"dp{world} (independent sequences)",
                       "l2": f"{M // 2} rotating input sets of {run_set_mb(inp, ad, logits):.1f} MB (> 4x L2 together)",
                       "schedule": args.schedule,
                       "timing": f"CUDA graph of {M} steps replayed ({SCHEDULE_TEXT[args.schedule]}); per-kernel times from events in a second graph of the same steps run on one stream"},
            "roofline": {"bound": "hbm", "achieved": attn_gbs, "peak": peak, "unit": "GB/s",
                         "frac": attn_gbs / peak, "traffic": traffic, "kernel": "attn_tc_kernel",
                         "peak_source": peak_src, "algorithmic_bytes_per_launch": kv_bytes},
            "attn_us": attn_ms * 1e3, "attn_kv_gbs": attn_gbs, "attn_query_tok_s": B * S / (attn_ms * 1e-3),
            "attn_tflops": attn_flops_of(a) / (attn_ms * 1e-3) / 1e12,
            "attn_isolated_us": attn_iso_ms * 1e3, "attn_isolated_kv_gbs": kv_bytes / (attn_iso_ms * 1e-3) / 1e9,
            "attn_isolated_frac": kv_bytes / (attn_iso_ms * 1e-3) / 1e9 / peak,
            "unmask_isolated_us": unmask_iso_ms * 1e3,
            "unmask_us": unmask_ms * 1e3, "unmask_steps_per_s": 1.0 / (unmask_ms * 1e-3),
            "unmask_logits_gbs": unmask_gbs, "unmask_frac": unmask_gbs / peak,
            "step_breakdown_us": {"adaln_cond": cond_ms * 1e3, "norm_modulate_and_residual": normres_ms * 1e3,
                                  "attention_and_merge": attn_ms * 1e3,
                                  "unmask": unmask_ms * 1e3,
                                  "note": "events around each launch group in a serial replay of the steps"},
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks.summary(t_c0 - 0.3, t_c1 + 0.1),
        }
        if extras is not None:
            result.update(extras)
        print(json.dumps(result))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return result


def lmhead_inputs(dev, B: int = 8, S: int = 16, D: int = 2048, V: int = 131072, seed: int = 5):
    """Hidden states x [B][S][D] ~ N(0, 1) and an LM-head weight W [V][D] ~ N(0, 3^2 / D) (bf16,
    seeded), every position masked: the decode shape of the fused LM head + unmask."""
    import torch
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((B, S, D), generator=g).to(torch.bfloat16).to(dev)
    w = (torch.randn((V, D), generator=g) * (3.0 / D ** 0.5)).to(torch.bfloat16).to(dev)
    tokens = torch.full((B, S), 3, dtype=torch.int32, device=dev)
    masked = torch.ones((B, S), dtype=torch.uint8, device=dev)
    return x, w, tokens, masked


def lmhead_op(gamma: float = 0.8):
    from denoiser_attention_b200 import api
    return lambda b, o: api.lmhead_unmask_step(b[0], b[1], b[2], b[3], gamma=gamma, want_conf=False)


def run_set_mb(inp, ad, logits) -> float:
    return sum(t.numel() * t.element_size() for t in (inp.k_ctx, inp.v_ctx, logits, inp.q, ad.h, ad.f)) / 1e6


def run_extras(args, dev, peak):
    """Numbers beyond the headline, each from CUDA events over graphs of rotating input sets: the
    decode step, the attention alone on every workload, and the block-sweep unmask table."""
    import torch
    from denoiser_attention_b200 import api, synth
    out = {}
    tpeak, tpeak_src = measured_tensor_peak()
    # ---- the decode step (8 sequences, ctx 4096): whole step and its kernels. Its attention leaves
    # SMs idle (528 key tiles over 148 CTAs), so the three branches on forked streams overlap well
    # here (for the batch workload they only take turns)
    w = synth.workload("decode_bf16")
    inp, ad, logits = host_inputs(w)
    run = StepRun(w, inp, ad, logits, dev, "branches")
    M = 2 * run.n_sets
    g, _ = run.capture(M, with_events=False)
    for _ in range(5):
        g.replay()
    torch.cuda.synchronize()
    reps = max(1, math.ceil(2000 / M))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / (reps * M)
    del g
    g, ev = run.capture(M, with_events=True)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    attn_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    unmask_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in ev)
    del g
    kvb = kv_bytes_of(w.attn)
    out["decode_step"] = {
        "workload": workload_desc(w), "value": w.attn.batch * w.attn.block_size / (ms * 1e-3),
        "unit": "query-tok/s", "ms_per_step": ms, "steps": reps * M, "schedule": "branches", "attn_us": attn_ms * 1e3,
        "attn_frac": kvb / (attn_ms * 1e-3) / 1e9 / peak, "unmask_us": unmask_ms * 1e3}
    del run
    # ---- the attention alone on every workload
    attn = {}
    for name, S in (("decode_bf16", None), ("batch_bf16", None), ("ragged_paged", None),
                    ("sweep_bf16", 4), ("sweep_bf16", 8), ("sweep_bf16", 16), ("sweep_bf16", 32), ("sweep_bf16", 64)):
        w = synth.workload(name, block_size=S)
        a = synth.attention_inputs(w.attn, seed=w.seed)
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        nbytes = (a.k_ctx.numel() + a.v_ctx.numel()) * 2
        n_sets = max(2, math.ceil(4 * l2 / nbytes))
        sets = []
        for _ in range(n_sets):
            sets.append(api.StepBuffers(
                tau=None, h=None, f=None, q=a.q.to(dev), k_blk=a.k_blk.to(dev), v_blk=a.v_blk.to(dev),
                k_ctx=a.k_ctx.to(dev), v_ctx=a.v_ctx.to(dev), ctx_lens=a.ctx_lens.to(dev),
                page_table=None if a.page_table is None else a.page_table.to(dev), logits=None, tokens=None,
                is_masked=None))
        outs = [torch.empty_like(s.q) for s in sets]
        step = api.RefinementStep({}, gamma=0.8, page_size=w.attn.page_size, ctx_stride=a.ctx_stride)
        for b, o in zip(sets, outs):
            attn_op(step)(b, o)
        torch.cuda.synchronize()
        ms = isolated_ms(attn_op(step), sets, outs, torch.cuda.Stream(device=dev), reps=max(3, 200 // n_sets))
        kvb = kv_bytes_of(w.attn)
        key = name if S is None else f"{name}_S{S}"
        tflops = attn_flops_of(w.attn) / (ms * 1e-3) / 1e12
        attn[key] = {"us": ms * 1e3, "kv_gbs": kvb / (ms * 1e-3) / 1e9, "frac": kvb / (ms * 1e-3) / 1e9 / peak,
                     "tflops": tflops, "tensor_frac": tflops / tpeak, "kv_bytes": kvb}
        del sets, outs, a
        torch.cuda.empty_cache()
    out["attention"] = attn
    out["attention_peaks"] = {"hbm_gbs": peak, "bf16_tflops": tpeak, "tensor_peak_source": tpeak_src}
    # ---- the block-sweep unmask table: per S the unmask step time, and per (S, temperature,
    # gamma) the mean number of positions committed in the first refinement step (all masked)
    table = []
    times = {}
    for S in (4, 8, 16, 32, 64):
        w = synth.workload("sweep_bf16", block_size=S)
        B = w.attn.batch
        lg = synth.workload_logits(w).to(dev)
        t = torch.full((B, S), 3, dtype=torch.int32, device=dev)
        m = torch.ones((B, S), dtype=torch.uint8, device=dev)
        for inv_temp in (2.0, 1.0, 0.5):
            for gamma in (0.5, 0.7, 0.8, 0.9, 0.95):
                t.fill_(3)
                m.fill_(1)
                nc, _, conf, _ = api.unmask_step(lg, t, m, gamma=gamma, inv_temperature=inv_temp)
                torch.cuda.synchronize()
                table.append({"S": S, "temperature": 1.0 / inv_temp, "gamma": gamma,
                              "committed_per_step": float(nc.float().mean()),
                              "frac_above_gamma": float((conf >= gamma).float().mean())})
        # rotating copies of the logits, more than 4x L2 together, so that each launch reads HBM
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        n_sets = max(2, math.ceil(4 * l2 / (lg.numel() * lg.element_size())))
        bs = [api.StepBuffers(tau=None, h=None, f=None, q=None, k_blk=None, v_blk=None, k_ctx=None, v_ctx=None,
                              ctx_lens=None, page_table=None, logits=lg if k == 0 else lg.clone(), tokens=t.clone(),
                              is_masked=m.clone()) for k in range(n_sets)]
        st = api.RefinementStep({}, gamma=0.8)
        times[S] = isolated_ms(unmask_op(st), bs, [None] * n_sets, torch.cuda.Stream(device=dev),
                               reps=max(5, 200 // n_sets)) * 1e3
        del lg, bs
        torch.cuda.empty_cache()
    out["sweep_unmask"] = {"unmask_us_by_S": times, "cells": table,
                           "note": "unmask time: graph of launches over rotating copies of the logits (more "
                                   "than 4x L2 together); committed tokens per step: mean over the 32 sequences "
                                   "of the first step (every position masked), confidence sampler"}
    # ---- the fused LM head + unmask on the decode shape (128 rows, D 2048, vocabulary 131072):
    # the 537 MB weight stream is the algorithmic traffic (larger than L2 by itself)
    lm = lmhead_inputs(dev)
    lmhead_op()(lm, None)
    torch.cuda.synchronize()
    ms = isolated_ms(lmhead_op(), [lm], [None], torch.cuda.Stream(device=dev), reps=50)
    wbytes = lm[1].numel() * 2
    flops = 2 * lm[0].shape[0] * lm[0].shape[1] * lm[0].shape[2] * lm[1].shape[0]
    out["lmhead_unmask"] = {"shape": "x 8x16x2048, W 131072x2048 bf16", "us": ms * 1e3,
                            "weight_gbs": wbytes / (ms * 1e-3) / 1e9, "frac": wbytes / (ms * 1e-3) / 1e9 / peak,
                            "tflops": flops / (ms * 1e-3) / 1e12}
    del lm
    torch.cuda.empty_cache()
    return out


def measured_traffic(workload: str):
    """DRAM bytes (read + write) per attention launch on `workload` from the ncu capture recorded
    in profiles/attn_tc_kernel_traffic.json, or None when there is none for this workload or it
    was taken on another version of the kernel source (its sha256 differs from attn_tc.cu)."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "attn_tc_kernel_traffic.json")
    src = os.path.join(ROOT, "denoiser_attention_b200", "csrc", "attn_tc.cu")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get(workload)
    if not rec:
        return None
    if hashlib.sha256(open(src, "rb").read()).hexdigest() != rec.get("source_sha256"):
        return None
    return int(rec["dram_bytes_per_launch"])


def run_e2e(step, inp, ad, logits, w, dev, args, world):
    """Same metric through the public host-buffer API: every step copies its inputs from pinned
    host memory to the device, runs the step and copies the results back."""
    import torch
    from denoiser_attention_b200 import api
    B, S = w.attn.batch, w.attn.block_size
    host = {
        "tau": ad.tau, "h": ad.h, "f": ad.f, "q": inp.q, "k_blk": inp.k_blk, "v_blk": inp.v_blk,
        "k_ctx": inp.k_ctx, "v_ctx": inp.v_ctx, "ctx_lens": inp.ctx_lens, "logits": logits,
        "tokens": torch.full((B, S), 3, dtype=torch.int32), "is_masked": torch.ones((B, S), dtype=torch.uint8),
    }
    host = {k: v.pin_memory() for k, v in host.items()}
    runner = api.HostStep(step, host, dev)
    h2d = runner.h2d_bytes
    d2h = runner.d2h_bytes
    steps = max(3, min(args.steps, 20))
    for _ in range(3):
        runner.run()
    torch.cuda.synchronize()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record()
    for _ in range(steps):
        runner.run()
    s1.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(s0.elapsed_time(s1), dev) / steps
    return {"value": B * world * S / (ms * 1e-3), "unit": "query-tok/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms, "steps": steps}


def cpu_baseline(w, inp, ad, logits):
    """The oracle, as it stands, on the host cores: whole query tokens for ~10 s."""
    B, S = w.attn.batch, w.attn.block_size
    t0 = time.perf_counter()
    k = 0
    while True:
        oracle_token_sample(w, inp, ad, logits, (k // S) % B, k % S)
        k += 1
        if time.perf_counter() - t0 > 10.0 and k >= 4:
            break
    el = time.perf_counter() - t0
    return {"value": k / el, "unit": "query-tok/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{k} query tokens of the workload (all heads, adaLN, unmask of that position), {el:.1f} s"}


def run_kernel(args):
    """One kernel alone on one workload, eager launches: --warmup untimed, then --steps timed with
    CUDA events; one JSON line with its mean time (for profiling captures that should hold only
    that kernel's buffers)."""
    import torch
    from denoiser_attention_b200 import api, build, synth
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    build.build()
    if args.kernel == "lmhead":
        bufs, out, op, nbytes = lmhead_inputs(dev), None, lmhead_op(), 131072 * 2048 * 2
        desc = "x 8x16x2048, W 131072x2048 bf16"
    else:
        # "name" or "name:S" (a block size for the sweep workload)
        name, _, bs = args.workload.partition(":")
        w = synth.workload(name, block_size=int(bs) if bs else None)
        if args.kernel == "attn":
            a = synth.attention_inputs(w.attn, seed=w.seed)
            bufs = api.StepBuffers(tau=None, h=None, f=None, q=a.q.to(dev), k_blk=a.k_blk.to(dev),
                                   v_blk=a.v_blk.to(dev), k_ctx=a.k_ctx.to(dev), v_ctx=a.v_ctx.to(dev),
                                   ctx_lens=a.ctx_lens.to(dev),
                                   page_table=None if a.page_table is None else a.page_table.to(dev), logits=None,
                                   tokens=None, is_masked=None)
            out = torch.empty_like(bufs.q)
            op = attn_op(api.RefinementStep({}, gamma=w.gamma, page_size=w.attn.page_size, ctx_stride=a.ctx_stride))
            nbytes = kv_bytes_of(w.attn)
        else:
            B, S = w.attn.batch, w.attn.block_size
            bufs = api.StepBuffers(tau=None, h=None, f=None, q=None, k_blk=None, v_blk=None, k_ctx=None, v_ctx=None,
                                   ctx_lens=None, page_table=None, logits=synth.workload_logits(w).to(dev),
                                   tokens=torch.full((B, S), 3, dtype=torch.int32, device=dev),
                                   is_masked=torch.ones((B, S), dtype=torch.uint8, device=dev))
            out = None
            op = unmask_op(api.RefinementStep({}, gamma=w.gamma, inv_temperature=w.inv_temperature))
            nbytes = bufs.logits.numel() * bufs.logits.element_size()
        desc = workload_desc(w)
    for _ in range(args.warmup):
        op(bufs, out)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        op(bufs, out)
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / args.steps
    print(json.dumps({"kernel": args.kernel, "workload": desc, "us_per_launch": us, "launches": args.steps,
                      "algorithmic_bytes": nbytes, "gbs": nbytes / (us * 1e-6) / 1e9,
                      "note": "eager launches on one buffer set (warm L2 when the data fits it); for profiling"}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD,
                    help="the step's workload (default: the batch-generation workload, the headline); with "
                         "--kernel also name:S, e.g. sweep_bf16:4")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the extra keys (decode step, attention per workload, block-sweep unmask table)")
    ap.add_argument("--schedule", choices=list(SCHEDULE_TEXT), default="branches",
                    help="how the step's three branches are put on streams")
    ap.add_argument("--kernel", choices=["attn", "unmask", "lmhead"], default=None,
                    help="time one kernel alone on --workload (for profiling captures), not the step")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.kernel is not None:
        run_kernel(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
