"""Benchmark of one TwoTower denoiser refinement step on B200 (one process per GPU).

A step is one pass of the whole hot path over one batch: adaLN-single conditioning, modulated
RMSNorm prologue, Eq. (1) layer-aligned denoiser attention, gated residual and ConfidenceSample
over the vocabulary logits (the paper "Nemotron-TwoTower: Diffusion Language Modeling with
Pretrained AR Context", §2.1-§2.2, Algorithm 2). The workload is the bf16 decode step: per GPU
8 sequences with 4096 context tokens + a block of S=16, 32 query / 2 kv heads, head dim 128,
adaLN width 2048, vocabulary 131072, gamma 0.8, seeded synthetic inputs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun: every rank processes its own 8 sequences (weak scaling; sequences
are independent, so there is no data-path collective); the elapsed time is the max over ranks.
`--impl reference` times the CPU fp64 oracle on the host cores instead (the comparison arm).
Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import re
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
WORKLOAD = "decode_bf16"
PER_GPU_BATCH = 8
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
    import torch
    from denoiser_attention_b200 import synth
    inp = synth.attention_inputs(w.attn, seed=w.seed + seed_offset)
    B, S = w.attn.batch, w.attn.block_size
    tau = [1.0] * B   # first refinement step: the whole block is masked (Algorithm 2's time input)
    ad = synth.adaln_inputs(B, S, w.hidden, tau, seed=w.seed + 100 + seed_offset, dtype=w.attn.dtype)
    logits = synth.workload_logits(w, seed=w.seed + seed_offset)
    return inp, ad, logits


def run_reference(args):
    """The comparison arm: the CPU fp64 oracle on the host cores, same config/metric/unit."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from denoiser_attention_b200 import synth
    w = synth.workload(WORKLOAD)
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

    w = synth.workload(WORKLOAD)
    B, S = w.attn.batch, w.attn.block_size
    global_batch = B * world
    lo, hi = shard_range(global_batch, world, rank)
    assert hi - lo == B
    inp, ad, logits = host_inputs(w, seed_offset=lo)     # this rank's sequences

    # ---- rotating input sets on the device (same bytes at distinct addresses): the per-step
    # working set is smaller than L2, so consecutive steps read different sets
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    ws_bytes = sum(t.numel() * t.element_size() for t in (inp.k_ctx, inp.v_ctx, logits, inp.q, ad.h, ad.f))
    n_sets = max(2, math.ceil(4 * l2 / ws_bytes))
    weights = {k: getattr(ad, k).to(dev) for k in ("w1", "b1", "w2", "b2", "w3", "b3", "layer_emb", "norm_w")}
    sets = []
    for i in range(n_sets):
        sets.append(api.StepBuffers(
            tau=ad.tau.to(dev), h=ad.h.to(dev), f=ad.f.to(dev), q=inp.q.to(dev), k_blk=inp.k_blk.to(dev),
            v_blk=inp.v_blk.to(dev), k_ctx=inp.k_ctx.to(dev), v_ctx=inp.v_ctx.to(dev),
            ctx_lens=inp.ctx_lens.to(dev), page_table=None, logits=logits.to(dev),
            tokens=torch.full((B, S), 3, dtype=torch.int32, device=dev),
            is_masked=torch.ones((B, S), dtype=torch.uint8, device=dev)))
    step = api.RefinementStep(weights, gamma=w.gamma, inv_temperature=w.inv_temperature,
                              ctx_stride=inp.ctx_stride, schedule=args.schedule)
    outs = [torch.empty_like(s.q) for s in sets]

    # eager warm-up (sets the kernels' attributes, allocates workspaces), then capture M steps
    for i in range(n_sets):
        step.run(sets[i], out_attn=outs[i])
    torch.cuda.synchronize()
    M = 2 * n_sets
    # events recorded inside the graph must be "external" to become timestamped graph nodes
    mk = lambda: torch.cuda.Event(enable_timing=True, external=True)
    ev = [(mk(), mk(), mk(), mk()) for _ in range(M)]
    g = torch.cuda.CUDAGraph()
    cap_stream = torch.cuda.Stream(device=dev)
    cap_stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap_stream):
        with torch.cuda.graph(g, stream=cap_stream):
            for j in range(M):
                step.run(sets[j % n_sets], out_attn=outs[j % n_sets], events=ev[j])
    torch.cuda.current_stream().wait_stream(cap_stream)
    launches_per_step = api.RefinementStep.LAUNCHES

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
    g_rem = None
    if rem:
        g_rem = torch.cuda.CUDAGraph()
        with torch.cuda.stream(cap_stream):
            with torch.cuda.graph(g_rem, stream=cap_stream):
                for j in range(rem):
                    step.run(sets[j % n_sets], out_attn=outs[j % n_sets])
        torch.cuda.current_stream().wait_stream(cap_stream)
        torch.cuda.synchronize()
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

    # per-kernel durations from the events of the last replay of the M-step graph
    if R == 0:
        for _ in range(1):
            g.replay()
        torch.cuda.synchronize()
    attn_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    unmask_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in ev)
    attn_ms = max_over_ranks(attn_ms, dev)
    unmask_ms = max_over_ranks(unmask_ms, dev)
    # the same two kernels alone (own graphs over the same rotating input sets), for context: inside
    # the step they share the GPU with the other branches
    attn_iso_ms = max_over_ranks(isolated_ms(lambda b, o: api.denoise_attention(
        b.q, b.k_blk, b.v_blk, b.k_ctx, b.v_ctx, b.ctx_lens, page_table=b.page_table,
        page_size=step.page_size, ctx_stride=step.ctx_stride, softmax_scale=step.softmax_scale, out=o),
        sets, outs, cap_stream), dev)
    unmask_iso_ms = max_over_ranks(isolated_ms(lambda b, o: api.unmask_step(
        b.logits, b.tokens, b.is_masked, gamma=step.gamma, inv_temperature=step.inv_temperature,
        mask_token_id=step.mask_token_id, want_conf=False), sets, outs, cap_stream), dev)

    a = w.attn
    kv_bytes = B * (a.ctx_lens[0] + S) * a.num_kv_heads * a.head_dim * 2 * 2
    logit_bytes = B * S * w.vocab * 2
    peak, peak_src = measured_peaks()
    attn_gbs = kv_bytes / (attn_ms * 1e-3) / 1e9
    unmask_gbs = logit_bytes / (unmask_ms * 1e-3) / 1e9
    traffic = measured_traffic()

    # ---- end to end through the public API with host buffers (pinned), copies timed
    e2e = run_e2e(step, inp, ad, logits, w, dev, args, world)

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
                       "l2": f"{n_sets} rotating input sets of {ws_bytes / 1e6:.1f} MB (> 4x L2)",
                       "schedule": args.schedule,
                       "timing": f"CUDA graph of {M} steps replayed ({SCHEDULE_TEXT[args.schedule]}); per-kernel events on the streams the kernels run on"},
            "roofline": {"bound": "hbm", "achieved": attn_gbs, "peak": peak, "unit": "GB/s",
                         "frac": attn_gbs / peak, "traffic": traffic, "kernel": "attn_tc_kernel",
                         "peak_source": peak_src, "algorithmic_bytes_per_launch": kv_bytes},
            "attn_us": attn_ms * 1e3, "attn_kv_gbs": attn_gbs, "attn_query_tok_s": B * S / (attn_ms * 1e-3),
            "attn_isolated_us": attn_iso_ms * 1e3, "attn_isolated_kv_gbs": kv_bytes / (attn_iso_ms * 1e-3) / 1e9,
            "attn_isolated_frac": kv_bytes / (attn_iso_ms * 1e-3) / 1e9 / peak,
            "unmask_isolated_us": unmask_iso_ms * 1e3,
            "unmask_us": unmask_ms * 1e3, "unmask_steps_per_s": 1.0 / (unmask_ms * 1e-3),
            "unmask_logits_gbs": unmask_gbs, "unmask_frac": unmask_gbs / peak,
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks.summary(t_c0 - 0.3, t_c1 + 0.1),
        }
        print(json.dumps(result))
    if world > 1:
        dist.barrier()
        del g
        dist.destroy_process_group()
    return result


def measured_traffic():
    """DRAM bytes (read + write) per attention launch from the committed ncu summary of the decode
    workload, or None when that summary is absent or was taken on another version of the kernel
    source (its recorded sha256 differs from the current attn_tc.cu)."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "attn_tc_kernel_decode_bf16.md")
    src = os.path.join(ROOT, "denoiser_attention_b200", "csrc", "attn_tc.cu")
    if not os.path.exists(p):
        return None
    text = open(p).read()
    m_bytes = re.search(r"dram_bytes_per_launch:\s*([0-9]+)", text)
    m_sha = re.search(r"source_sha256:\s*([0-9a-f]{64})", text)
    if not (m_bytes and m_sha):
        return None
    if hashlib.sha256(open(src, "rb").read()).hexdigest() != m_sha.group(1):
        return None
    return int(m_bytes.group(1))


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
    steps = max(3, min(args.steps, 50))
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


def run_kernel_only(args):
    """Eager launches of one kernel of the step on the workload (for ncu captures): warmup + steps
    launches, one input set, no graph; prints the mean launch time from CUDA events."""
    import torch
    from denoiser_attention_b200 import api, build, synth
    build.build()
    dev = torch.device("cuda", 0)
    w = synth.workload(args.workload)
    inp, ad, logits = host_inputs(w)
    B, S = w.attn.batch, w.attn.block_size
    q, kb, vb = inp.q.to(dev), inp.k_blk.to(dev), inp.v_blk.to(dev)
    kc, vc, lens = inp.k_ctx.to(dev), inp.v_ctx.to(dev), inp.ctx_lens.to(dev)
    table = None if inp.page_table is None else inp.page_table.to(dev)
    lg = logits.to(dev)
    tokens = torch.full((B, S), 3, dtype=torch.int32, device=dev)
    masked = torch.ones((B, S), dtype=torch.uint8, device=dev)
    weights = {k: getattr(ad, k).to(dev) for k in ("w1", "b1", "w2", "b2", "w3", "b3", "layer_emb", "norm_w")}
    tau, h, f = ad.tau.to(dev), ad.h.to(dev), ad.f.to(dev)
    out = torch.empty_like(q)

    if args.kernel == "lmhead":
        # the fused LM head + unmask at the decode shape: hidden states [8][16][2048], W [131072][2048]
        gen = torch.Generator(device=dev).manual_seed(w.seed)
        D, Vh = 2048, 131072
        xh = torch.randn((B, S, D), device=dev, generator=gen).to(torch.bfloat16)
        wh = (torch.randn((Vh, D), device=dev, generator=gen) * (3.0 / D ** 0.5)).to(torch.bfloat16)

    def once():
        if args.kernel == "lmhead":
            api.lmhead_unmask_step(xh, wh, tokens, masked, gamma=w.gamma, want_conf=False)
        elif args.kernel == "attn":
            api.denoise_attention(q, kb, vb, kc, vc, lens, page_table=table, page_size=w.attn.page_size,
                                  ctx_stride=inp.ctx_stride, out=out)
        elif args.kernel == "unmask":
            api.unmask_step(lg, tokens, masked, gamma=w.gamma, want_conf=False)
        else:
            mod = api.adaln_cond(tau, weights["w1"], weights["b1"], weights["w2"], weights["b2"], weights["w3"],
                                 weights["b3"], weights["layer_emb"])
            api.adaln_norm_modulate(h, weights["norm_w"], mod)
            api.adaln_gated_residual(h, f, mod)

    for _ in range(args.warmup):
        once()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        once()
    e1.record()
    torch.cuda.synchronize()
    print(json.dumps({"kernel": args.kernel, "workload": args.workload, "launches": args.steps,
                      "mean_us_incl_host_gaps": 1e3 * e0.elapsed_time(e1) / args.steps}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--kernel", choices=["attn", "unmask", "adaln", "lmhead"], default=None,
                    help="profiling mode: eager launches of one kernel only (not a bench line)")
    ap.add_argument("--workload", default=WORKLOAD, help="workload of the --kernel profiling mode")
    ap.add_argument("--schedule", choices=list(SCHEDULE_TEXT), default="branches",
                    help="how the step's three branches are put on streams")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.kernel:
        run_kernel_only(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
