"""Seeded synthetic inputs for one TwoTower denoiser refinement step.

This module is shared by the CUDA path, the CPU oracle tests and the benchmark. It only draws
random numbers and lays them out; it performs none of the step's own arithmetic (attention,
modulation, confidence). Every tensor is produced on the host from NumPy's PCG64 generator,
rounded to its storage dtype by torch (round-to-nearest-even), so the GPU and the oracle read
identical bytes.

Sub-streams are keyed by (seed, stream name) through NumPy's SeedSequence, so adding a stream
never perturbs another one.

Workloads (names describe what they are; sizes follow the TwoTower decoding setting of
"Nemotron-TwoTower: Diffusion Language Modeling with Pretrained AR Context", §2.1-§2.2, with
the block size S=16 / T=16 steps / gamma=0.8 operating point of the model card's generation
example):
  tiny_fp32      B=1, ctx 64 (4 committed blocks) + S=16, 4 q heads / 1 kv head, d=64, fp32
  decode_bf16    B=8, ctx 4096 + S=16, 32 q / 2 kv heads, d=128, bf16, vocab 131072 with
                 injected confident peaks (about 30% of positions above gamma=0.8)
  batch_bf16     B=64, ctx 16384 + S=16, 32/2 heads, d=128, logits N(0, 3^2)
  sweep_bf16     B=32, ctx 8192, S in {4,8,16,32,64}, 32/2 heads, d=128
  ragged_paged   B=4, ctx ~ U[1024, 131072], S=16, 256-token pages in shuffled order
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

# Stable integer ids for the named sub-streams.
_STREAMS = {
    "q": 1, "kblk": 2, "vblk": 3, "kctx": 4, "vctx": 5, "logits": 6, "pages": 7, "lens": 8,
    "h": 9, "f": 10, "normw": 11, "w1": 12, "b1": 13, "w2": 14, "b2": 15, "w3": 16, "b3": 17,
    "emb": 18, "peaks": 19, "gumbel": 20, "tokens": 21,
}


def rng(seed: int, stream: str) -> np.random.Generator:
    """Independent PCG64 generator for (seed, stream)."""
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), _STREAMS[stream]])))


def _to_dtype(x: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(dtype)


def normal(seed: int, stream: str, shape, std: float = 1.0, dtype: torch.dtype = torch.float32) -> torch.Tensor:
    g = rng(seed, stream)
    x = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return _to_dtype(x, dtype)


@dataclasses.dataclass
class AttnShape:
    batch: int
    block_size: int          # S
    num_q_heads: int         # Hq
    num_kv_heads: int        # Hkv
    head_dim: int            # d
    ctx_lens: list           # L_b per sequence
    dtype: torch.dtype
    page_size: int = 0       # 0 => contiguous context
    q_std: float = 1.0
    kv_std: float = 1.0


@dataclasses.dataclass
class AttnInputs:
    shape: AttnShape
    q: torch.Tensor                  # [B][S][Hq][d]
    k_blk: torch.Tensor              # [B][S][Hkv][d]
    v_blk: torch.Tensor
    k_ctx: torch.Tensor              # contiguous [B][ctx_stride][Hkv][d] or paged [P][page][Hkv][d]
    v_ctx: torch.Tensor
    ctx_lens: torch.Tensor           # int32 [B]
    page_table: Optional[torch.Tensor]  # int32 [B][max_pages] (-1 = unused) or None
    ctx_stride: int                  # contiguous: tokens per sequence row; paged: 0
    softmax_scale: float = 1.0


def attention_inputs(shape: AttnShape, seed: int) -> AttnInputs:
    B, S, Hq, Hkv, d = shape.batch, shape.block_size, shape.num_q_heads, shape.num_kv_heads, shape.head_dim
    lens = [int(x) for x in shape.ctx_lens]
    assert len(lens) == B
    q = normal(seed, "q", (B, S, Hq, d), shape.q_std, shape.dtype)
    kb = normal(seed, "kblk", (B, S, Hkv, d), shape.kv_std, shape.dtype)
    vb = normal(seed, "vblk", (B, S, Hkv, d), shape.kv_std, shape.dtype)
    if shape.page_size == 0:
        stride = max(1, max(lens)) if lens else 1
        kc = normal(seed, "kctx", (B, stride, Hkv, d), shape.kv_std, shape.dtype)
        vc = normal(seed, "vctx", (B, stride, Hkv, d), shape.kv_std, shape.dtype)
        table = None
    else:
        ps = shape.page_size
        npages_seq = [(L + ps - 1) // ps for L in lens]
        total = max(1, sum(npages_seq))
        perm = rng(seed, "pages").permutation(total).astype(np.int32)
        maxp = max(1, max(npages_seq))
        table_np = np.full((B, maxp), -1, dtype=np.int32)
        pos = 0
        for b, n in enumerate(npages_seq):
            table_np[b, :n] = perm[pos:pos + n]
            pos += n
        kc = normal(seed, "kctx", (total, ps, Hkv, d), shape.kv_std, shape.dtype)
        vc = normal(seed, "vctx", (total, ps, Hkv, d), shape.kv_std, shape.dtype)
        table = torch.from_numpy(table_np)
        stride = 0
    return AttnInputs(shape=shape, q=q, k_blk=kb, v_blk=vb, k_ctx=kc, v_ctx=vc,
                      ctx_lens=torch.tensor(lens, dtype=torch.int32), page_table=table,
                      ctx_stride=stride)


@dataclasses.dataclass
class AdaLNInputs:
    hidden: int       # D
    freq_dim: int     # F
    mlp_width: int    # W
    tau: torch.Tensor        # fp32 [B]
    w1: torch.Tensor         # fp32 [W][F]
    b1: torch.Tensor         # fp32 [W]
    w2: torch.Tensor         # fp32 [W][W]
    b2: torch.Tensor         # fp32 [W]
    w3: torch.Tensor         # fp32 [3D][W]
    b3: torch.Tensor         # fp32 [3D]
    layer_emb: torch.Tensor  # fp32 [3][D]
    norm_w: torch.Tensor     # fp32 [D]
    h: torch.Tensor          # [B][S][D] (dtype)
    f: torch.Tensor          # [B][S][D] (dtype)
    eps: float = 1e-5


def adaln_inputs(batch: int, block_size: int, hidden: int, tau, seed: int,
                 dtype: torch.dtype, freq_dim: int = 256, mlp_width: int = 256,
                 weight_std: float = 0.02) -> AdaLNInputs:
    D, F, W = hidden, freq_dim, mlp_width
    tau_t = torch.as_tensor(np.asarray(tau, dtype=np.float32).reshape(batch))
    return AdaLNInputs(
        hidden=D, freq_dim=F, mlp_width=W, tau=tau_t,
        w1=normal(seed, "w1", (W, F), weight_std), b1=normal(seed, "b1", (W,), weight_std),
        w2=normal(seed, "w2", (W, W), weight_std), b2=normal(seed, "b2", (W,), weight_std),
        w3=normal(seed, "w3", (3 * D, W), weight_std), b3=normal(seed, "b3", (3 * D,), weight_std),
        layer_emb=normal(seed, "emb", (3, D), weight_std),
        norm_w=(1.0 + normal(seed, "normw", (D,), 0.1)),
        h=normal(seed, "h", (batch, block_size, D), 1.0, dtype),
        f=normal(seed, "f", (batch, block_size, D), 1.0, dtype),
    )


def logits_normal(seed: int, batch: int, block_size: int, vocab: int, std: float,
                  dtype: torch.dtype) -> torch.Tensor:
    """Plain N(0, std^2) vocabulary logits [B][S][V]."""
    return normal(seed, "logits", (batch, block_size, vocab), std, dtype)


def logits_peaked(seed: int, batch: int, block_size: int, vocab: int, dtype: torch.dtype,
                  std: float = 3.0, peak_frac: float = 0.3,
                  conf_lo: float = 0.85, conf_hi: float = 0.99) -> torch.Tensor:
    """Gumbel-perturbed N(0, std^2) logits with a confident peak planted at a seeded subset of
    positions.

    For a chosen position, token j gets the logit that would make its softmax probability equal
    a target c* ~ U(conf_lo, conf_hi) given the other logits: l_j = log(c*/(1-c*)) + log sum_k!=j
    exp(l_k). Bf16 rounding afterwards moves c* slightly; that is part of the input, not an error.
    """
    n = batch * block_size
    x = rng(seed, "logits").standard_normal(size=(n, vocab), dtype=np.float32)
    x *= np.float32(std)
    x += rng(seed, "gumbel").gumbel(size=(n, vocab)).astype(np.float32)
    g = rng(seed, "peaks")
    chosen = g.random(n) < peak_frac
    tok = g.integers(0, vocab, size=n)
    target = g.uniform(conf_lo, conf_hi, size=n)
    for r in np.nonzero(chosen)[0]:
        row = x[r].astype(np.float64)
        j = int(tok[r])
        others = np.delete(row, j)
        m = others.max()
        lse = m + math.log(np.exp(others - m).sum())
        x[r, j] = np.float32(math.log(target[r] / (1.0 - target[r])) + lse)
    return _to_dtype(x.reshape(batch, block_size, vocab), dtype)


@dataclasses.dataclass
class Workload:
    name: str
    attn: AttnShape
    hidden: int
    vocab: int
    gamma: float
    inv_temperature: float
    logits_kind: str          # "normal" or "peaked"
    logits_std: float
    seed: int
    tau: Optional[float]      # fixed tau for fixed-step workloads, None => Alg. 2 tau from the mask
    steps: int = 16           # T


def ragged_lengths(seed: int, batch: int, lo: int, hi: int) -> list:
    return [int(x) for x in rng(seed, "lens").integers(lo, hi + 1, size=batch)]


def workload(name: str, block_size: Optional[int] = None) -> Workload:
    if name == "tiny_fp32":
        a = AttnShape(1, 16, 4, 1, 64, [64], torch.float32, q_std=1 / 8, kv_std=1 / 8)
        return Workload(name, a, hidden=256, vocab=1024, gamma=0.8, inv_temperature=1.0,
                        logits_kind="normal", logits_std=2.0, seed=0, tau=None)
    if name == "decode_bf16":
        a = AttnShape(8, 16, 32, 2, 128, [4096] * 8, torch.bfloat16, q_std=1 / math.sqrt(128))
        return Workload(name, a, hidden=2048, vocab=131072, gamma=0.8, inv_temperature=1.0,
                        logits_kind="peaked", logits_std=3.0, seed=1, tau=None)
    if name == "batch_bf16":
        a = AttnShape(64, 16, 32, 2, 128, [16384] * 64, torch.bfloat16, q_std=1 / math.sqrt(128))
        return Workload(name, a, hidden=2048, vocab=131072, gamma=0.8, inv_temperature=1.0,
                        logits_kind="normal", logits_std=3.0, seed=2, tau=(16 - 8 + 1) / 16)
    if name == "sweep_bf16":
        S = 16 if block_size is None else int(block_size)
        a = AttnShape(32, S, 32, 2, 128, [8192] * 32, torch.bfloat16, q_std=1 / math.sqrt(128))
        return Workload(name, a, hidden=2048, vocab=131072, gamma=0.8, inv_temperature=1.0,
                        logits_kind="peaked", logits_std=3.0, seed=3, tau=None)
    if name == "ragged_paged":
        lens = ragged_lengths(4, 4, 1024, 131072)
        a = AttnShape(4, 16, 32, 2, 128, lens, torch.bfloat16, page_size=256,
                      q_std=1 / math.sqrt(128))
        return Workload(name, a, hidden=2048, vocab=131072, gamma=0.8, inv_temperature=1.0,
                        logits_kind="peaked", logits_std=3.0, seed=4, tau=None)
    raise KeyError(name)


def workload_logits(w: Workload, seed: Optional[int] = None, batch: Optional[int] = None) -> torch.Tensor:
    s = w.seed if seed is None else seed
    B = w.attn.batch if batch is None else batch
    dt = w.attn.dtype
    if w.logits_kind == "peaked":
        return logits_peaked(s, B, w.attn.block_size, w.vocab, dt, std=w.logits_std)
    return logits_normal(s, B, w.attn.block_size, w.vocab, w.logits_std, dt)
