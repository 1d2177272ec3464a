"""The whole refinement step (RefinementStep / HostStep, the public API) against the oracle."""
import numpy as np
import pytest
import torch

from denoiser_attention_b200 import api, synth
from oracle import tt_oracle as O
from tests._parity import assert_close_attn, assert_close_bf16_rounded, check_unmask, np64

pytestmark = pytest.mark.gpu


def _workload_inputs(name):
    w = synth.workload(name)
    inp = synth.attention_inputs(w.attn, seed=w.seed)
    B, S = w.attn.batch, w.attn.block_size
    tau = [1.0 - 0.5 * (b % 2) for b in range(B)]
    ad = synth.adaln_inputs(B, S, w.hidden, tau, seed=w.seed + 100, dtype=w.attn.dtype)
    logits = synth.workload_logits(w)
    return w, inp, ad, logits


@pytest.mark.parametrize("name", ["tiny_fp32", "decode_bf16"])
def test_refinement_step_matches_oracle(cuda_lib, name):
    w, inp, ad, logits = _workload_inputs(name)
    B, S = w.attn.batch, w.attn.block_size
    dev = "cuda"
    weights = {k: getattr(ad, k).to(dev) for k in ("w1", "b1", "w2", "b2", "w3", "b3", "layer_emb", "norm_w")}
    tokens = torch.full((B, S), 3, dtype=torch.int32)
    masked = torch.ones((B, S), dtype=torch.uint8)
    host = {"tau": ad.tau, "h": ad.h, "f": ad.f, "q": inp.q, "k_blk": inp.k_blk, "v_blk": inp.v_blk,
            "k_ctx": inp.k_ctx, "v_ctx": inp.v_ctx, "ctx_lens": inp.ctx_lens, "logits": logits,
            "tokens": tokens, "is_masked": masked}
    step = api.RefinementStep(weights, gamma=w.gamma, ctx_stride=inp.ctx_stride)
    out = api.HostStep(step, host, dev).run()
    torch.cuda.synchronize()
    f64 = np64
    mod = O.adaln_cond(f64(ad.tau), f64(ad.w1), f64(ad.b1), f64(ad.w2), f64(ad.b2), f64(ad.w3), f64(ad.b3),
                       f64(ad.layer_emb))
    attn = O.denoise_attention(f64(inp.q), f64(inp.k_blk), f64(inp.v_blk), f64(inp.k_ctx), f64(inp.v_ctx),
                               inp.ctx_lens.tolist())
    h_new = O.adaln_gated_residual(f64(ad.h), f64(ad.f), mod)
    y = O.adaln_norm_modulate(f64(ad.h), f64(ad.norm_w), mod, ad.eps)
    assert_close_attn(out["attn"], attn, w.attn.dtype, name)
    if w.attn.dtype == torch.bfloat16:
        assert_close_bf16_rounded(out["h"], h_new, "residual")
        assert_close_bf16_rounded(out["y"], y, "modulated RMSNorm")
    else:
        assert np.abs(f64(out["h"]) - h_new).max() <= 1e-5
        assert np.abs(f64(out["y"]) - y).max() <= 1e-5
    check_unmask(tokens, masked, logits, w.gamma, 1.0, out["tokens"], out["is_masked"], out["n_committed"],
                 out["n_masked"])


def test_graph_captured_step_matches_eager(cuda_lib):
    # the benchmark replays the step from a CUDA graph; it must give the eager result
    w, inp, ad, logits = _workload_inputs("decode_bf16")
    B, S = w.attn.batch, w.attn.block_size
    dev = "cuda"
    weights = {k: getattr(ad, k).to(dev) for k in ("w1", "b1", "w2", "b2", "w3", "b3", "layer_emb", "norm_w")}
    bufs = api.StepBuffers(tau=ad.tau.to(dev), h=ad.h.to(dev), f=ad.f.to(dev), q=inp.q.to(dev),
                           k_blk=inp.k_blk.to(dev), v_blk=inp.v_blk.to(dev), k_ctx=inp.k_ctx.to(dev),
                           v_ctx=inp.v_ctx.to(dev), ctx_lens=inp.ctx_lens.to(dev), page_table=None,
                           logits=logits.to(dev), tokens=torch.full((B, S), 3, dtype=torch.int32, device=dev),
                           is_masked=torch.ones((B, S), dtype=torch.uint8, device=dev))
    step = api.RefinementStep(weights, gamma=w.gamma, ctx_stride=inp.ctx_stride)
    o_eager = torch.empty_like(bufs.q)
    r = step.run(bufs, out_attn=o_eager)
    tok_eager = bufs.tokens.clone()
    bufs.tokens.fill_(3)
    bufs.is_masked.fill_(1)
    o_graph = torch.empty_like(bufs.q)
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            step.run(bufs, out_attn=o_graph)
    torch.cuda.current_stream().wait_stream(s)
    bufs.tokens.fill_(3)
    bufs.is_masked.fill_(1)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(o_graph, o_eager)
    assert torch.equal(bufs.tokens, tok_eager)


def test_concurrent_branches_match_sequential(cuda_lib):
    # every stream schedule of the three branches gives the bits of the one-stream order
    w, inp, ad, logits = _workload_inputs("decode_bf16")
    B, S = w.attn.batch, w.attn.block_size
    dev = "cuda"
    weights = {k: getattr(ad, k).to(dev) for k in ("w1", "b1", "w2", "b2", "w3", "b3", "layer_emb", "norm_w")}
    results = []
    for schedule in ("serial", "branches", "branches", "attn_then_unmask", "unmask_then_attn"):
        bufs = api.StepBuffers(tau=ad.tau.to(dev), h=ad.h.to(dev), f=ad.f.to(dev), q=inp.q.to(dev),
                               k_blk=inp.k_blk.to(dev), v_blk=inp.v_blk.to(dev), k_ctx=inp.k_ctx.to(dev),
                               v_ctx=inp.v_ctx.to(dev), ctx_lens=inp.ctx_lens.to(dev), page_table=None,
                               logits=logits.to(dev),
                               tokens=torch.full((B, S), 3, dtype=torch.int32, device=dev),
                               is_masked=torch.ones((B, S), dtype=torch.uint8, device=dev))
        step = api.RefinementStep(weights, gamma=w.gamma, ctx_stride=inp.ctx_stride, schedule=schedule)
        r = step.run(bufs)
        torch.cuda.synchronize()
        results.append({k: v.cpu() for k, v in r.items()} | {"tokens": bufs.tokens.cpu(),
                                                               "is_masked": bufs.is_masked.cpu()})
    for other in results[1:]:
        for k, v in results[0].items():
            assert torch.equal(v, other[k]), k
