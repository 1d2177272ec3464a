"""CPU fp64 oracle for one TwoTower denoiser refinement step.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this module: only the tests, the
package's smoke check and the benchmark's CPU-baseline leg call it. It shares no code with the
CUDA library and never imports it. Everything is plain NumPy in float64; a library matmul is
used as one step where the definition is a matrix product, with no blocking, fusion or
reordering beyond what the definitions below state.

Source: "Nemotron-TwoTower: Diffusion Language Modeling with Pretrained AR Context"
(arXiv 2606.26493, Kamalu et al.), hereafter "the paper".

  denoise_attention      the paper §2.1 "Bidirectional attention", Eq. (1)
  timestep_embedding,
  adaln_cond,
  adaln_norm_modulate,
  adaln_gated_residual   the paper §2.1 "Time conditioning" (adaLN-single, after PixArt-alpha)
  confidence_argmax,
  confidence_commit      the paper §2.2 "Sampling" and Algorithm 2 (ConfidenceSample)
  refine_block           the paper Algorithm 2 (single-block confidence unmasking loop)
  predict_noise_step     the predict-and-noise sampler (§2.2 "Sampling"), linear schedule
  lmhead_logits          the denoiser's LM head: logits = x W^T (feeds either sampler)
  append_block           the paper Algorithm 1, context update (the committed block joins the context)

Readings of points the paper leaves open (each is also listed in the design notes):
  * attention mask: every block query sees all L_b context keys and all S block keys; the only
    mask is the ragged end of the context (§2.1: bidirectional inside the block, causal w.r.t.
    the past blocks, which all precede the block).
  * adaLN internals: three modulation vectors (shift, scale, gate); sinusoid with x1000 and
    period 10000; MLP F->W->W->3D with SiLU; (1 + scale); RMSNorm eps 1e-5. The paper only
    says "a global MLP maps t to shared scale, shift and gate, plus a per-layer learned
    embedding" -- parity of this part is pinned to the stated definition, not to the model.
  * confidence = max of softmax(inv_temperature * logits); argmax ties -> lowest token id.
  * commit rule: masked positions with confidence >= gamma; if none qualifies, the single most
    confident masked position (lowest position on ties); with remaining_steps > 0, at least
    ceil(n_masked / remaining_steps) of the most confident masked positions.
"""
from __future__ import annotations

import math
from typing import Callable, Optional, Sequence

import numpy as np


# ----------------------------------------------------------------------------------------------
# Eq. (1): layer-aligned denoiser attention
# ----------------------------------------------------------------------------------------------

def gather_context(k_ctx: np.ndarray, v_ctx: np.ndarray, ctx_lens: Sequence[int],
                   page_table: Optional[np.ndarray], page_size: int):
    """Per-sequence context keys/values [L_b][Hkv][d] (the context tower's layer-i KV for the
    past blocks 0..b-1, the paper §2.1).

    Contiguous: k_ctx is [B][ctx_stride][Hkv][d] and sequence b owns rows 0..L_b-1.
    Paged: k_ctx is [num_pages][page_size][Hkv][d]; logical token t of sequence b lives in
    physical page page_table[b][t // page_size], row t % page_size.
    """
    out_k, out_v = [], []
    for b, L in enumerate(ctx_lens):
        L = int(L)
        if page_table is None:
            out_k.append(k_ctx[b, :L])
            out_v.append(v_ctx[b, :L])
        else:
            rows_k, rows_v = [], []
            for t in range(0, L, page_size):
                p = int(page_table[b][t // page_size])
                n = min(page_size, L - t)
                rows_k.append(k_ctx[p, :n])
                rows_v.append(v_ctx[p, :n])
            if rows_k:
                out_k.append(np.concatenate(rows_k, axis=0))
                out_v.append(np.concatenate(rows_v, axis=0))
            else:
                out_k.append(np.zeros((0,) + k_ctx.shape[2:]))
                out_v.append(np.zeros((0,) + v_ctx.shape[2:]))
    return out_k, out_v


def denoise_attention(q: np.ndarray, k_blk: np.ndarray, v_blk: np.ndarray,
                      k_ctx: np.ndarray, v_ctx: np.ndarray, ctx_lens: Sequence[int],
                      page_table: Optional[np.ndarray] = None, page_size: int = 0,
                      softmax_scale: float = 1.0, return_lse: bool = False):
    """Eq. (1): Attn(Q_b, [K_ctx(<b); K_den(b)], [V_ctx(<b); V_den(b)]), float64.

    q      [B][S][Hq][d]     queries of the noisy block (all S positions)
    k_blk  [B][S][Hkv][d]    denoiser's own layer-i keys of block b (v_blk likewise)
    k_ctx  context keys, contiguous or paged (see gather_context); v_ctx likewise
    Query head h uses key/value head h // G with G = Hq / Hkv (grouped-query attention).
    Returns O [B][S][Hq][d] and, if asked, the natural-log log-sum-exp [B][Hq][S].

    For every (b, h, s): x_j = scale * <q, k_j> over j in context(0..L_b) ++ block(0..S);
    O = sum_j softmax(x)_j v_j, with the softmax computed two-pass (max, then exp-sum).
    """
    q = np.asarray(q, dtype=np.float64)
    B, S, Hq, d = q.shape
    Hkv = k_blk.shape[2]
    assert Hq % Hkv == 0
    G = Hq // Hkv
    ks, vs = gather_context(np.asarray(k_ctx, np.float64), np.asarray(v_ctx, np.float64),
                            ctx_lens, page_table, page_size)
    out = np.zeros((B, S, Hq, d), dtype=np.float64)
    lse = np.zeros((B, Hq, S), dtype=np.float64)
    for b in range(B):
        for kh in range(Hkv):
            keys = np.concatenate([ks[b][:, kh, :], np.asarray(k_blk[b, :, kh, :], np.float64)], axis=0)
            vals = np.concatenate([vs[b][:, kh, :], np.asarray(v_blk[b, :, kh, :], np.float64)], axis=0)
            for g in range(G):
                h = kh * G + g
                x = softmax_scale * (q[b, :, h, :] @ keys.T)          # [S][L_b + S]
                m = x.max(axis=1, keepdims=True)
                e = np.exp(x - m)
                z = e.sum(axis=1, keepdims=True)
                out[b, :, h, :] = (e / z) @ vals
                lse[b, h, :] = (m + np.log(z))[:, 0]
    if return_lse:
        return out, lse
    return out


# ----------------------------------------------------------------------------------------------
# adaLN-single time conditioning (the paper §2.1 "Time conditioning")
# ----------------------------------------------------------------------------------------------

def timestep_embedding(tau: np.ndarray, freq_dim: int = 256, max_period: float = 10000.0,
                       t_scale: float = 1000.0) -> np.ndarray:
    """phi(tau) = [cos(t_scale*tau*w_k), sin(t_scale*tau*w_k)], w_k = max_period^(-k/(F/2)),
    k = 0..F/2-1. Returns [B][F]."""
    tau = np.asarray(tau, dtype=np.float64).reshape(-1)
    half = freq_dim // 2
    k = np.arange(half, dtype=np.float64)
    w = max_period ** (-k / half)
    arg = t_scale * tau[:, None] * w[None, :]
    return np.concatenate([np.cos(arg), np.sin(arg)], axis=1)


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def adaln_cond(tau, w1, b1, w2, b2, w3, b3, layer_emb, freq_dim: int = 256) -> np.ndarray:
    """Global MLP t -> (shift, scale, gate), plus this layer's learned embedding.

    mod = W3 . SiLU(W2 . SiLU(W1 . phi(tau) + b1) + b2) + b3, reshaped to [3][D], + E_layer.
    Weights are [out][in]. Returns [B][3][D] with rows (shift, scale, gate).
    """
    w1, b1, w2, b2, w3, b3, emb = (np.asarray(a, np.float64) for a in (w1, b1, w2, b2, w3, b3, layer_emb))
    phi = timestep_embedding(tau, freq_dim)
    a1 = silu(phi @ w1.T + b1)
    a2 = silu(a1 @ w2.T + b2)
    out = a2 @ w3.T + b3                              # [B][3D]
    D = emb.shape[1]
    return out.reshape(-1, 3, D) + emb[None, :, :]


def adaln_norm_modulate(h, norm_w, mod, eps: float = 1e-5) -> np.ndarray:
    """RMSNorm prologue with adaLN modulation:
    y = h / sqrt(mean(h^2) + eps) * w * (1 + scale_b) + shift_b   over the last axis (D)."""
    h = np.asarray(h, np.float64)
    w = np.asarray(norm_w, np.float64)
    mod = np.asarray(mod, np.float64)
    shift = mod[:, 0, :][:, None, :]
    scale = mod[:, 1, :][:, None, :]
    rms = np.sqrt(np.mean(h * h, axis=-1, keepdims=True) + eps)
    return h / rms * w * (1.0 + scale) + shift


def adaln_gated_residual(h, f, mod) -> np.ndarray:
    """Gated residual: h' = h + gate_b * f."""
    h = np.asarray(h, np.float64)
    f = np.asarray(f, np.float64)
    gate = np.asarray(mod, np.float64)[:, 2, :][:, None, :]
    return h + gate * f


# ----------------------------------------------------------------------------------------------
# ConfidenceSample (the paper §2.2 "Sampling", Algorithm 2)
# ----------------------------------------------------------------------------------------------

def confidence_argmax(logits, inv_temperature: float = 1.0, exclude_token: Optional[int] = None):
    """Per position: confidence = max_v softmax(inv_temperature * logits)_v and the argmax token
    (lowest token id among equal maxima). Returns (conf float64 [..], argmax int64 [..]).

    Computed as 1 / sum_v exp(inv_temperature * (l_v - l_max)), which is the softmax value at the
    maximum, in float64. exclude_token (the [MASK] id) removes that entry from both.
    """
    x = np.array(logits, dtype=np.float64, copy=True)
    if exclude_token is not None:
        x[..., exclude_token] = -np.inf
    m = x.max(axis=-1, keepdims=True)
    a = np.argmax(x, axis=-1)                       # first index of the maximum
    z = np.exp(inv_temperature * (x - m)).sum(axis=-1)
    return 1.0 / z, a


def confidence_commit(tokens, is_masked, conf, argmax, gamma: float, remaining_steps: int = 0):
    """Commit step of ConfidenceSample for each sequence of a batch.

    tokens int [B][S], is_masked bool [B][S], conf/argmax [B][S].
    Masked positions with conf >= gamma are committed (token := argmax, mask cleared). If none
    qualifies and any position is still masked, the single most confident masked position is
    committed (lowest position on ties). With remaining_steps > 0 at least
    ceil(n_masked / remaining_steps) of the most confident masked positions are committed.
    Committed positions are never touched again.
    Returns (tokens, is_masked, n_committed [B], n_masked [B]).
    """
    tokens = np.array(tokens, dtype=np.int64, copy=True)
    is_masked = np.array(is_masked, dtype=bool, copy=True)
    B, S = tokens.shape
    n_committed = np.zeros(B, dtype=np.int64)
    for b in range(B):
        masked = [l for l in range(S) if is_masked[b, l]]
        chosen = {l for l in masked if conf[b, l] >= gamma}
        if masked:
            need = 1
            if remaining_steps > 0:
                need = -(-len(masked) // remaining_steps)
            if len(chosen) < need:
                # most confident first, lowest position first among equal confidence
                order = sorted(masked, key=lambda l: (-conf[b, l], l))
                for l in order:
                    if len(chosen) >= need:
                        break
                    chosen.add(l)
        for l in chosen:
            tokens[b, l] = argmax[b, l]
            is_masked[b, l] = False
        n_committed[b] = len(chosen)
    n_masked = is_masked.sum(axis=1).astype(np.int64)
    return tokens, is_masked, n_committed, n_masked


def unmask_step(tokens, is_masked, logits, gamma: float, inv_temperature: float = 1.0,
                exclude_token: Optional[int] = None, remaining_steps: int = 0):
    """ConfidenceSample(z, p, gamma, T - r + 1): confidence + argmax, then commit.
    Returns (tokens, is_masked, n_committed, n_masked, conf, argmax)."""
    conf, arg = confidence_argmax(logits, inv_temperature, exclude_token)
    t, m, nc, nm = confidence_commit(tokens, is_masked, conf, arg, gamma, remaining_steps)
    return t, m, nc, nm, conf, arg


def predict_noise_step(tokens, is_masked, logits, keep_masked: int, inv_temperature: float = 1.0,
                       exclude_token: Optional[int] = None):
    """The predict-and-noise sampler of block diffusion (the paper §2.2 "Sampling"): predict every
    masked position (argmax, confidence as in confidence_argmax, with the same optional removal
    of the [MASK] token's own logit), then re-mask the least confident ones so that
    min(n_masked, keep_masked) stay masked; i.e. commit the (n_masked - keep_masked) most
    confident masked positions, confidence descending and position ascending on ties. Committed
    positions are never changed."""
    conf, arg = confidence_argmax(logits, inv_temperature, exclude_token)
    tokens = np.array(tokens, dtype=np.int64, copy=True)
    is_masked = np.array(is_masked, dtype=bool, copy=True)
    n_committed = np.zeros(tokens.shape[0], dtype=np.int64)
    for b in range(tokens.shape[0]):
        masked = [l for l in range(tokens.shape[1]) if is_masked[b, l]]
        k = max(0, len(masked) - keep_masked)
        # stable sort by confidence, descending: equal confidences keep position order
        order = sorted(masked, key=lambda l: -conf[b, l])
        for l in order[:k]:
            tokens[b, l] = arg[b, l]
            is_masked[b, l] = False
        n_committed[b] = k
    return tokens, is_masked, n_committed, is_masked.sum(axis=1), conf, arg


def linear_schedule_keep(block_size: int, steps: int, r: int) -> int:
    """Masked positions left after step r of T under alpha_t = 1 - t (masked fraction t = (T-r)/T)."""
    return (block_size * (steps - r)) // steps


def lmhead_logits(x, w) -> np.ndarray:
    """The denoiser's LM head (the paper §2.2: p_theta over the vocabulary for every block
    position): logits[b][l][v] = sum_d x[b][l][d] w[v][d], in float64."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    return np.einsum("bld,vd->blv", x, w)


def refine_block(batch: int, block_size: int, steps: int, gamma: float,
                 logits_for_step: Callable[[int, np.ndarray], np.ndarray],
                 mask_token_id: int = 3, inv_temperature: float = 1.0,
                 use_remaining_steps: bool = False):
    """Algorithm 2: single-block confidence unmasking.

    z <- [MASK]^S; for r = 1..T: tau = |{l : z_l = [MASK]}| / S; p <- Denoiser(z, tau, ...);
    z <- ConfidenceSample(z, p, gamma, T - r + 1). The denoiser is a callable
    logits_for_step(r, tau[B]) -> logits [B][S][V] (synthetic here; there is no model).
    Returns (tokens, is_masked, per-step records [(r, tau, n_committed)]).
    """
    tokens = np.full((batch, block_size), mask_token_id, dtype=np.int64)
    is_masked = np.ones((batch, block_size), dtype=bool)
    records = []
    for r in range(1, steps + 1):
        tau = is_masked.sum(axis=1) / block_size
        logits = logits_for_step(r, tau)
        rem = steps - r + 1 if use_remaining_steps else 0
        tokens, is_masked, nc, nm, _, _ = unmask_step(tokens, is_masked, logits, gamma,
                                                      inv_temperature, None, rem)
        records.append((r, tau.copy(), nc.copy()))
    return tokens, is_masked, records


def append_block(ctx_k: Sequence[np.ndarray], ctx_v: Sequence[np.ndarray], k_new: np.ndarray,
                 v_new: np.ndarray):
    """The context update of Algorithm 1: after block b is committed, the context tower's K/V of its S tokens
    follow the sequence's existing context. ctx_k[b] / ctx_v[b] are [L_b][Hkv][d] (the logical
    context, e.g. from gather_context); k_new / v_new are [B][S][Hkv][d]. Returns the new
    per-sequence contexts [L_b + S][Hkv][d] and lengths. Storage (pages) is not modelled: a paged
    implementation must gather back to exactly these arrays."""
    out_k = [np.concatenate([np.asarray(ctx_k[b]), np.asarray(k_new[b])], axis=0) for b in range(len(ctx_k))]
    out_v = [np.concatenate([np.asarray(ctx_v[b]), np.asarray(v_new[b])], axis=0) for b in range(len(ctx_v))]
    return out_k, out_v, [k.shape[0] for k in out_k]


def round_bf16(x) -> np.ndarray:
    """Round float64 values straight to the nearest bfloat16 (8 significant bits, ties to
    even), returned as float64. A bf16 output is defined as the exact value rounded this way.
    Normal range only (|x| >= 2^-126), which covers every value the step produces."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                      # x = m * 2^e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(m * 256.0), e - 8)
