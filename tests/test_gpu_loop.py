"""Algorithm 2 on the device (RefinementLoop: tau from the mask by tt_block_tau, then the whole
refinement step, T times), eagerly and replayed from one CUDA graph, against the oracle's
refine_block for the tiny fp32 workload: per step the time input tau, the commit counts, the
adaLN modulation, the attention output and the gated residual, and the final tokens / mask.
Step r draws its own inputs (seed r), as there is no model between steps."""
import numpy as np
import pytest
import torch

from denoiser_attention_b200 import api, synth
from oracle import tt_oracle as O
from tests._parity import np64

pytestmark = pytest.mark.gpu

WEIGHTS = ("w1", "b1", "w2", "b2", "w3", "b3", "layer_emb", "norm_w")


def _per_step_inputs(w, T):
    B, S = w.attn.batch, w.attn.block_size
    per = []
    for r in range(1, T + 1):
        inp = synth.attention_inputs(w.attn, seed=r)
        logits = synth.logits_normal(r, B, S, w.vocab, w.logits_std, torch.float32)
        hf = synth.adaln_inputs(B, S, w.hidden, [1.0] * B, seed=100 + r, dtype=w.attn.dtype)
        per.append((inp, logits, hf.h, hf.f))
    return per


def _buffers(per, dev):
    bufs = []
    for inp, logits, h, f in per:
        bufs.append(api.StepBuffers(
            tau=torch.empty(h.shape[0], dtype=torch.float32, device=dev), h=h.to(dev), f=f.to(dev),
            q=inp.q.to(dev), k_blk=inp.k_blk.to(dev), v_blk=inp.v_blk.to(dev), k_ctx=inp.k_ctx.to(dev),
            v_ctx=inp.v_ctx.to(dev), ctx_lens=inp.ctx_lens.to(dev), page_table=None, logits=logits.to(dev),
            tokens=None, is_masked=None))
    return bufs


def _collect(bufs, outs, tokens, masked):
    torch.cuda.synchronize()
    return {
        "tau": [b.tau.cpu().clone() for b in bufs],
        "nc": [o["n_committed"].cpu().clone() for o in outs],
        "mod": [o["mod"].cpu().clone() for o in outs],
        "attn": [o["attn"].cpu().clone() for o in outs],
        "h": [o["h"].cpu().clone() for o in outs],
        "tokens": tokens.cpu().clone(), "masked": masked.cpu().clone(),
    }


def test_block_loop_on_device_matches_oracle(cuda_lib):
    w = synth.workload("tiny_fp32")
    B, S, T = w.attn.batch, w.attn.block_size, w.steps
    dev = "cuda"
    ad = synth.adaln_inputs(B, S, w.hidden, [1.0] * B, seed=0, dtype=w.attn.dtype)
    weights = {k: getattr(ad, k).to(dev) for k in WEIGHTS}
    per = _per_step_inputs(w, T)
    bufs = _buffers(per, dev)
    step = api.RefinementStep(weights, gamma=w.gamma, ctx_stride=per[0][0].ctx_stride)
    loop = api.RefinementLoop(step)

    tokens = torch.full((B, S), 3, dtype=torch.int32, device=dev)
    masked = torch.ones((B, S), dtype=torch.uint8, device=dev)
    eager = _collect(bufs, loop.run(bufs, tokens, masked), tokens, masked)

    # the same T steps captured as one graph and replayed
    tokens.fill_(3)
    masked.fill_(1)
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            outs_g = loop.run(bufs, tokens, masked)
    torch.cuda.current_stream().wait_stream(s)
    tokens.fill_(3)
    masked.fill_(1)
    g.replay()
    graph = _collect(bufs, outs_g, tokens, masked)
    for k in ("tau", "nc", "mod", "attn", "h"):
        for a, b in zip(eager[k], graph[k]):
            assert torch.equal(a, b), k
    assert torch.equal(eager["tokens"], graph["tokens"]) and torch.equal(eager["masked"], graph["masked"])

    # oracle: Algorithm 2 with the same per-step logits, then each step's modulation and attention
    t_or, m_or, rec = O.refine_block(B, S, T, w.gamma, lambda r, tau: np64(per[r - 1][1]))
    np.testing.assert_array_equal(eager["tokens"].numpy(), t_or)
    np.testing.assert_array_equal(eager["masked"].numpy().astype(bool), m_or)
    f64 = np64
    for r in range(T):
        _, tau_or, nc_or = rec[r]
        assert np.array_equal(eager["tau"][r].double().numpy(), tau_or), r   # k/16: exact in fp32
        np.testing.assert_array_equal(eager["nc"][r].numpy(), nc_or)
        mod = O.adaln_cond(tau_or, *(f64(getattr(ad, k)) for k in WEIGHTS[:7]))
        assert np.abs(f64(eager["mod"][r]) - mod).max() <= 1e-5, r
        inp, _, h, f = per[r]
        att = O.denoise_attention(f64(inp.q), f64(inp.k_blk), f64(inp.v_blk), f64(inp.k_ctx), f64(inp.v_ctx),
                                  inp.ctx_lens.tolist())
        assert np.abs(f64(eager["attn"][r]) - att).max() <= 1e-5, r
        hn = O.adaln_gated_residual(f64(h), f64(f), mod)
        assert np.abs(f64(eager["h"][r]) - hn).max() <= 1e-5, r
    # every step commits exactly one position (max probability ~0.1 << gamma): tau runs 16/16 .. 1/16
    assert [float(t[0]) for t in eager["tau"]] == [(S - r) / S for r in range(T)]


@pytest.mark.parametrize("gamma", [0.001, 0.06])
def test_early_exit_once_the_block_is_complete(cuda_lib, gamma):
    # Algorithm 2 completes the block within T steps, here well before: the steps after the one
    # that commits the last position do nothing (tau, attention output untouched), while every
    # step up to it matches the oracle; the graph replay gives the eager result
    w = synth.workload("tiny_fp32")
    B, S, T = w.attn.batch, w.attn.block_size, w.steps
    dev = "cuda"
    ad = synth.adaln_inputs(B, S, w.hidden, [1.0] * B, seed=0, dtype=w.attn.dtype)
    weights = {k: getattr(ad, k).to(dev) for k in WEIGHTS}
    per = _per_step_inputs(w, T)
    bufs = _buffers(per, dev)
    step = api.RefinementStep(weights, gamma=gamma, ctx_stride=per[0][0].ctx_stride)
    loop = api.RefinementLoop(step, early_exit=True)
    t_or, m_or, rec = O.refine_block(B, S, T, gamma, lambda r, tau: np64(per[r - 1][1]))
    left = [int(np.sum(rec[r][1]) * S) for r in range(T)]     # masked positions entering step r + 1
    r_done = next(r for r in range(1, T + 1) if r == T or left[r] == 0)   # the step that completes
    assert r_done < T

    def run_once(graph: bool):
        tokens = torch.full((B, S), 3, dtype=torch.int32, device=dev)
        masked = torch.ones((B, S), dtype=torch.uint8, device=dev)
        outs_attn = [torch.full_like(b.q, 7.0) for b in bufs]
        for b in bufs:
            b.tau.fill_(-1.0)
        if graph:
            g = torch.cuda.CUDAGraph()
            s = torch.cuda.Stream()
            s.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(s):
                with torch.cuda.graph(g, stream=s):
                    outs = loop.run(bufs, tokens, masked, out_attn=outs_attn)
            torch.cuda.current_stream().wait_stream(s)
            tokens.fill_(3)
            masked.fill_(1)
            for b in bufs:
                b.tau.fill_(-1.0)
            for o in outs_attn:
                o.fill_(7.0)
            g.replay()
        else:
            outs = loop.run(bufs, tokens, masked, out_attn=outs_attn)
        torch.cuda.synchronize()
        return tokens.cpu(), masked.cpu(), [b.tau.cpu().clone() for b in bufs], [o.cpu() for o in outs_attn], \
            [o["n_committed"].cpu() for o in outs]

    for graph in (False, True):
        tokens, masked, taus, attn, ncs = run_once(graph)
        np.testing.assert_array_equal(tokens.numpy(), t_or)
        np.testing.assert_array_equal(masked.numpy().astype(bool), m_or)
        assert loop.finished()
        for r in range(1, T + 1):
            if r <= r_done:
                assert np.array_equal(taus[r - 1].double().numpy(), rec[r - 1][1]), r
                np.testing.assert_array_equal(ncs[r - 1].numpy(), rec[r - 1][2])
                inp = per[r - 1][0]
                att = O.denoise_attention(np64(inp.q), np64(inp.k_blk), np64(inp.v_blk), np64(inp.k_ctx),
                                          np64(inp.v_ctx), inp.ctx_lens.tolist())
                assert np.abs(np64(attn[r - 1]) - att).max() <= 1e-5, r
            else:
                assert (taus[r - 1] == -1.0).all(), r               # block_tau skipped
                assert (attn[r - 1] == 7.0).all(), r                # attention skipped


def test_early_exit_shortens_the_loop(cuda_lib):
    # the decode workload with a threshold every position passes: the block completes at step 1,
    # and the 15 steps after it cost only their launches
    w = synth.workload("decode_bf16")
    B, S, T = w.attn.batch, w.attn.block_size, 16
    dev = "cuda"
    ad = synth.adaln_inputs(B, S, w.hidden, [1.0] * B, seed=5, dtype=w.attn.dtype)
    weights = {k: getattr(ad, k).to(dev) for k in WEIGHTS}
    inp = synth.attention_inputs(w.attn, seed=w.seed)
    logits = synth.workload_logits(w).to(dev)
    one = api.StepBuffers(tau=torch.empty(B, device=dev), h=ad.h.to(dev), f=ad.f.to(dev), q=inp.q.to(dev),
                          k_blk=inp.k_blk.to(dev), v_blk=inp.v_blk.to(dev), k_ctx=inp.k_ctx.to(dev),
                          v_ctx=inp.v_ctx.to(dev), ctx_lens=inp.ctx_lens.to(dev), page_table=None, logits=logits,
                          tokens=None, is_masked=None)
    bufs = [api.StepBuffers(**{**one.__dict__, "tau": torch.empty(B, device=dev)}) for _ in range(T)]
    step = api.RefinementStep(weights, gamma=1e-7, ctx_stride=inp.ctx_stride)
    times = {}
    for early in (False, True):
        loop = api.RefinementLoop(step, early_exit=early)
        tokens = torch.full((B, S), 3, dtype=torch.int32, device=dev)
        masked = torch.ones((B, S), dtype=torch.uint8, device=dev)
        loop.run(bufs, tokens, masked)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                tokens.fill_(3)
                masked.fill_(1)
                loop.run(bufs, tokens, masked)
        torch.cuda.current_stream().wait_stream(s)
        for _ in range(3):
            g.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(10):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        times[early] = e0.elapsed_time(e1) / 10
        assert int(masked.sum()) == 0
        del g
    print(f"16-step loop: {times[False] * 1e3:.1f} us full, {times[True] * 1e3:.1f} us with the early exit")
    assert times[True] < 0.6 * times[False]
