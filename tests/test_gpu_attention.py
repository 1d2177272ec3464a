"""Eq. (1) attention on the GPU (through the C ABI) against the CPU fp64 oracle.

Cases span several 128-token key tiles with ragged tails, empty contexts (the first block), block
sizes 1..64, grouped-query layouts with 1..128 query heads per kv head, an odd number of query
tiles per group (the last CTA of a team then holds one), paged KV in shuffled page order, the tiny fp32 workload, and the full-size decode, batch and ragged-paged workloads (the
last ones on sampled sequences where the whole batch would be slow for the oracle)."""
import math

import numpy as np
import pytest
import torch

from denoiser_attention_b200 import api, binding, synth
from oracle import tt_oracle as O
from tests._parity import assert_close_attn, np64

pytestmark = pytest.mark.gpu


def _run(inp: synth.AttnInputs, return_lse=False):
    dev = "cuda"
    sh = inp.shape
    args = dict(page_table=None if inp.page_table is None else inp.page_table.to(dev),
                page_size=sh.page_size, ctx_stride=inp.ctx_stride, softmax_scale=inp.softmax_scale,
                return_lse=return_lse)
    r = api.denoise_attention(inp.q.to(dev), inp.k_blk.to(dev), inp.v_blk.to(dev), inp.k_ctx.to(dev),
                              inp.v_ctx.to(dev), inp.ctx_lens.to(dev), **args)
    torch.cuda.synchronize()
    return r


def _oracle(inp: synth.AttnInputs, seqs=None, return_lse=False):
    sh = inp.shape
    table = None if inp.page_table is None else inp.page_table.numpy()
    lens = inp.ctx_lens.tolist()
    if seqs is None:
        return O.denoise_attention(np64(inp.q), np64(inp.k_blk), np64(inp.v_blk), np64(inp.k_ctx), np64(inp.v_ctx),
                                   lens, table, sh.page_size, inp.softmax_scale, return_lse=return_lse)
    outs = []
    for b in seqs:
        if table is None:
            kc, vc, tb = np64(inp.k_ctx[b:b + 1]), np64(inp.v_ctx[b:b + 1]), None
        else:
            kc, vc, tb = np64(inp.k_ctx), np64(inp.v_ctx), table[b:b + 1]
        outs.append(O.denoise_attention(np64(inp.q[b:b + 1]), np64(inp.k_blk[b:b + 1]), np64(inp.v_blk[b:b + 1]),
                                        kc, vc, lens[b:b + 1], tb, sh.page_size, inp.softmax_scale)[0])
    return np.stack(outs)


CASES = [
    # B, S, Hq, Hkv, d, lens, dtype, page_size
    (3, 16, 32, 2, 128, [0, 100, 1000], torch.bfloat16, 0),
    (2, 16, 32, 2, 128, [64, 4096], torch.bfloat16, 0),
    (4, 1, 32, 2, 128, [1, 63, 65, 700], torch.bfloat16, 0),
    (2, 4, 32, 2, 128, [300, 129], torch.bfloat16, 0),
    (2, 8, 16, 2, 128, [513, 0], torch.bfloat16, 0),
    (2, 32, 32, 2, 128, [1000, 200], torch.bfloat16, 0),
    (1, 64, 32, 2, 128, [777], torch.bfloat16, 0),
    (2, 16, 8, 8, 128, [333, 64], torch.bfloat16, 0),
    (2, 16, 64, 1, 128, [250, 10], torch.bfloat16, 0),
    (2, 5, 12, 4, 128, [77, 190], torch.bfloat16, 0),
    (3, 16, 32, 2, 128, [1000, 3000, 17], torch.bfloat16, 256),
    (2, 16, 32, 2, 128, [4100, 64], torch.bfloat16, 128),
    (2, 16, 32, 2, 128, [130, 700], torch.bfloat16, 512),
    (1, 16, 4, 1, 64, [64], torch.float32, 0),
    (3, 7, 8, 2, 128, [0, 90, 300], torch.float32, 0),
    (2, 16, 4, 1, 64, [100, 37], torch.float32, 32),
    # more than 32 groups with the group-aligned partition (on 148 SMs: 74 teams):
    (36, 16, 32, 2, 128, [300] * 36, torch.bfloat16, 0),    # 72 groups of 4 tiles, one team each
    (17, 16, 32, 2, 128, [1024] * 17, torch.bfloat16, 0),   # 34 groups of 9 tiles, chunks of 4 + 5
    # three query tiles per group: G = 16, S = 24 (8 positions per tile); G = 128, S = 3 (one each)
    (2, 24, 32, 2, 128, [300, 50], torch.bfloat16, 0),
    (1, 3, 128, 1, 128, [200], torch.bfloat16, 0),
]


@pytest.mark.parametrize("B,S,Hq,Hkv,d,lens,dtype,ps", CASES)
def test_attention_matches_oracle(cuda_lib, B, S, Hq, Hkv, d, lens, dtype, ps):
    q_std = 1.0 / math.sqrt(d)
    sh = synth.AttnShape(B, S, Hq, Hkv, d, lens, dtype, page_size=ps, q_std=q_std)
    inp = synth.attention_inputs(sh, seed=100 + B * 7 + S)
    out, lse = _run(inp, return_lse=True)
    ref, ref_lse = _oracle(inp, return_lse=True)
    assert_close_attn(out, ref, dtype, f"{B}x{S} {Hq}/{Hkv} lens={lens}")
    np.testing.assert_allclose(np64(lse), ref_lse, atol=1e-4 if dtype == torch.bfloat16 else 1e-5)


@pytest.mark.parametrize("B,S,lens,ps", [
    (3, 16, [0, 100, 1000], 128),
    (2, 16, [4100, 64], 256),
    (2, 24, [300, 50], 128),     # three query tiles per group
])
def test_two_stream_kernel_on_short_contexts(cuda_lib, B, S, lens, ps):
    # Groups of two query tiles run the one-tile kernel when the host's bound on the key tiles
    # (from the page table's width) is small. A page table wider than the contexts need raises the
    # bound above that limit, so these short contexts run the two-stream kernel; the entries past
    # a sequence's pages are never read, and rows past the context end inside the last page hold
    # NaN, which must not reach the output.
    sh = synth.AttnShape(B, S, 32, 2, 128, lens, torch.bfloat16, page_size=ps, q_std=1 / math.sqrt(128))
    inp = synth.attention_inputs(sh, seed=40 + B + S)
    ref = _oracle(inp)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    units = B * 2
    width = math.ceil(32 * sms / units * 128 / ps) + 2
    assert units * (width * ps // 128 + 1) > 32 * sms
    table = torch.full((B, width), -1, dtype=torch.int32)
    table[:, :inp.page_table.shape[1]] = inp.page_table
    for b, L in enumerate(lens):
        if L % ps:
            pg = int(table[b, L // ps])
            inp.k_ctx[pg, L % ps:] = float("nan")
            inp.v_ctx[pg, L % ps:] = float("nan")
    inp.page_table = table
    assert_close_attn(_run(inp), ref, torch.bfloat16, f"two-stream {B}x{S} lens={lens}")


def test_attention_softmax_scale_and_large_logits(cuda_lib):
    # unscaled Q with softmax_scale 1/sqrt(d): logits of std ~1; and a sharp case (scale 1)
    for scale, q_std in ((1 / math.sqrt(128), 1.0), (1.0, 0.5)):
        sh = synth.AttnShape(2, 16, 32, 2, 128, [900, 2000], torch.bfloat16, q_std=q_std)
        inp = synth.attention_inputs(sh, seed=7)
        inp.softmax_scale = scale
        out = _run(inp)
        assert_close_attn(out, _oracle(inp), torch.bfloat16, f"scale={scale}")


def test_attention_garbage_past_context_end_is_ignored(cuda_lib):
    # slab rows past L_b (and the tail of a partial page) may hold anything, even NaN
    sh = synth.AttnShape(2, 16, 32, 2, 128, [100, 1000], torch.bfloat16, q_std=1 / math.sqrt(128))
    inp = synth.attention_inputs(sh, seed=8)
    ref = _oracle(inp)
    inp.k_ctx[0, 100:] = float("nan")
    inp.v_ctx[0, 100:] = float("nan")
    inp.k_ctx[1, 1000:] = float("inf")
    inp.v_ctx[1, 1000:] = float("nan")
    assert_close_attn(_run(inp), ref, torch.bfloat16, "garbage tail")


def test_tiny_fp32_workload(cuda_lib):
    w = synth.workload("tiny_fp32")
    inp = synth.attention_inputs(w.attn, seed=w.seed)
    assert_close_attn(_run(inp), _oracle(inp), torch.float32, "tiny_fp32")


def test_decode_workload_full(cuda_lib):
    w = synth.workload("decode_bf16")
    inp = synth.attention_inputs(w.attn, seed=w.seed)
    err = assert_close_attn(_run(inp), _oracle(inp), torch.bfloat16, "decode_bf16")
    print("decode_bf16 max/mean abs", err)


def test_batch_workload_sampled(cuda_lib):
    w = synth.workload("batch_bf16")
    inp = synth.attention_inputs(w.attn, seed=w.seed)
    out = _run(inp)
    seqs = [0, 17, 40, 63]
    assert_close_attn(out[seqs], _oracle(inp, seqs), torch.bfloat16, "batch_bf16 sampled")


@pytest.mark.parametrize("S", [4, 8, 16, 32, 64])
def test_sweep_workload_sampled(cuda_lib, S):
    w = synth.workload("sweep_bf16", block_size=S)
    inp = synth.attention_inputs(w.attn, seed=w.seed)
    out = _run(inp)
    seqs = [0, 31]
    assert_close_attn(out[seqs], _oracle(inp, seqs), torch.bfloat16, f"sweep S={S}")


def test_ragged_paged_workload(cuda_lib):
    w = synth.workload("ragged_paged")
    inp = synth.attention_inputs(w.attn, seed=w.seed)
    assert_close_attn(_run(inp), _oracle(inp), torch.bfloat16, "ragged_paged")


def test_first_block_is_bidirectional_block_attention(cuda_lib):
    sh = synth.AttnShape(4, 16, 32, 2, 128, [0, 0, 0, 0], torch.bfloat16, q_std=1 / math.sqrt(128))
    inp = synth.attention_inputs(sh, seed=9)
    out = np64(_run(inp))
    G = 16
    for b in range(4):
        for h in range(32):
            qq = np64(inp.q[b, :, h])
            kk = np64(inp.k_blk[b, :, h // G])
            vv = np64(inp.v_blk[b, :, h // G])
            x = qq @ kk.T
            p = np.exp(x - x.max(1, keepdims=True))
            ref = (p / p.sum(1, keepdims=True)) @ vv
            assert np.abs(out[b, :, h] - ref).max() < 1e-2


def test_block_permutation_equivariance_on_gpu(cuda_lib):
    sh = synth.AttnShape(2, 16, 32, 2, 128, [500, 1300], torch.bfloat16, q_std=1 / math.sqrt(128))
    inp = synth.attention_inputs(sh, seed=10)
    base = np64(_run(inp))
    perm = torch.randperm(16, generator=torch.Generator().manual_seed(0))
    inp.k_blk = inp.k_blk[:, perm].contiguous()
    inp.v_blk = inp.v_blk[:, perm].contiguous()
    assert np.abs(np64(_run(inp)) - base).max() < 2e-3
    inp.q = inp.q[:, perm].contiguous()
    assert np.abs(np64(_run(inp)) - base[:, perm.numpy()]).max() < 2e-3


def test_repeated_calls_are_identical(cuda_lib):
    # the merge tickets reset themselves: back-to-back calls give the same bytes
    sh = synth.AttnShape(3, 16, 32, 2, 128, [3000, 100, 5000], torch.bfloat16, q_std=1 / math.sqrt(128))
    inp = synth.attention_inputs(sh, seed=11)
    a = _run(inp).clone()
    for _ in range(3):
        assert torch.equal(_run(inp), a)


def test_bad_page_reports_device_error(cuda_lib):
    sh = synth.AttnShape(2, 16, 32, 2, 128, [600, 300], torch.bfloat16, page_size=256, q_std=1 / math.sqrt(128))
    inp = synth.attention_inputs(sh, seed=12)
    inp.page_table[1, 0] = 10_000          # beyond the pool: the kernel must not read it
    dev = "cuda"
    q = inp.q.to(dev)
    out = torch.empty_like(q)
    args = binding.attn_args(q, inp.k_blk.to(dev), inp.v_blk.to(dev), inp.k_ctx.to(dev), inp.v_ctx.to(dev),
                             inp.ctx_lens.to(dev), out, page_table=inp.page_table.to(dev), page_size=256)
    ws = binding.new_workspace(binding.tt_denoise_attn_workspace_bytes(args))
    binding.tt_denoise_attn(args, ws)
    st, detail = binding.tt_get_device_error(ws)
    assert st == binding.TT_ERR_DEVICE and detail == 1
    st, _ = binding.tt_get_device_error(ws)      # cleared
    assert st == binding.TT_OK


def test_context_longer_than_slab_reports_device_error(cuda_lib):
    sh = synth.AttnShape(2, 16, 32, 2, 128, [200, 100], torch.bfloat16, q_std=1 / math.sqrt(128))
    inp = synth.attention_inputs(sh, seed=13)
    dev = "cuda"
    q = inp.q.to(dev)
    out = torch.empty_like(q)
    lens = torch.tensor([200, 5000], dtype=torch.int32, device=dev)   # slab holds 200 rows
    args = binding.attn_args(q, inp.k_blk.to(dev), inp.v_blk.to(dev), inp.k_ctx.to(dev), inp.v_ctx.to(dev),
                             lens, out)
    ws = binding.new_workspace(binding.tt_denoise_attn_workspace_bytes(args))
    binding.tt_denoise_attn(args, ws)
    st, detail = binding.tt_get_device_error(ws)
    assert st == binding.TT_ERR_DEVICE and detail == 2
