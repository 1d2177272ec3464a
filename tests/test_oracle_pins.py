"""Pins for the CPU fp64 oracle, against things other than the oracle itself.

Each check ties a part of the oracle to a fact the paper or mathematics fixes: hand-derived
closed forms (tests/golden), special cases that reduce to a library routine (torch's
scaled_dot_product_attention, rms_norm, silu, softmax in float64), invariants (permutation
equivariance, grouped-query = repeated-KV multi-head, paged = contiguous) and brute force on tiny
inputs. A plausible slip in the oracle (a dropped term, a wrong sign or head index, a transposed
operand, a wrong tie rule) fails at least one of them; test_oracle_mutants.py checks exactly that
by planting such slips in a copy of the oracle.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import tt_oracle as O
from denoiser_attention_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _num(x):
    if isinstance(x, str):
        try:
            return float(x)
        except ValueError:
            pass
        return {"ln2": math.log(2.0), "ln3": math.log(3.0), "ln4": math.log(4.0),
                "pi/2000": math.pi / 2000, "pi/10": math.pi / 10}[x]
    return float(x)


def _arr(nested):
    if isinstance(nested, list):
        return np.array([_arr(x) for x in nested], dtype=np.float64)
    return _num(nested)


def _rand_attn(rs, B, S, Hq, Hkv, d, lens, page_size=0):
    q = rs.standard_normal((B, S, Hq, d))
    kb = rs.standard_normal((B, S, Hkv, d))
    vb = rs.standard_normal((B, S, Hkv, d))
    Lmax = max(1, max(lens))
    kc = rs.standard_normal((B, Lmax, Hkv, d))
    vc = rs.standard_normal((B, Lmax, Hkv, d))
    return q, kb, vb, kc, vc


def _sdpa_reference(q, kb, vb, kc, vc, lens, scale):
    """torch's scaled_dot_product_attention (float64, CPU) over the explicitly concatenated keys."""
    B, S, Hq, d = q.shape
    Hkv = kb.shape[2]
    out = np.zeros_like(q)
    for b in range(B):
        L = lens[b]
        K = np.concatenate([kc[b, :L], kb[b]], axis=0)          # [L+S][Hkv][d]
        V = np.concatenate([vc[b, :L], vb[b]], axis=0)
        K = torch.from_numpy(np.ascontiguousarray(K.transpose(1, 0, 2)))[None]   # [1][Hkv][n][d]
        V = torch.from_numpy(np.ascontiguousarray(V.transpose(1, 0, 2)))[None]
        Q = torch.from_numpy(np.ascontiguousarray(q[b].transpose(1, 0, 2)))[None]  # [1][Hq][S][d]
        o = F.scaled_dot_product_attention(Q, K, V, scale=scale, enable_gqa=True)
        out[b] = o[0].numpy().transpose(1, 0, 2)
    return out


# ---------------------------------------------------------------- attention (Eq. 1)

def test_attention_golden_closed_forms():
    g = json.load(open(os.path.join(GOLDEN, "attention_closed_forms.json")))
    for c in g["cases"]:
        out = O.denoise_attention(_arr(c["q"]), _arr(c["k_blk"]), _arr(c["v_blk"]), _arr(c["k_ctx"]),
                                  _arr(c["v_ctx"]), c["ctx_lens"], softmax_scale=c.get("softmax_scale", 1.0))
        np.testing.assert_allclose(out, _arr(c["out"]), rtol=0, atol=1e-12, err_msg=c["why"])


@pytest.mark.parametrize("B,S,Hq,Hkv,d,lens,scale", [
    (2, 4, 4, 2, 8, [5, 11], 0.3),
    (1, 16, 8, 1, 16, [64], 1.0),
    (3, 3, 6, 3, 4, [0, 1, 7], 0.7),
])
def test_attention_matches_library_sdpa(B, S, Hq, Hkv, d, lens, scale):
    rs = np.random.default_rng(11)
    q, kb, vb, kc, vc = _rand_attn(rs, B, S, Hq, Hkv, d, lens)
    out = O.denoise_attention(q, kb, vb, kc, vc, lens, softmax_scale=scale)
    ref = _sdpa_reference(q, kb, vb, kc, vc, lens, scale)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_first_block_is_plain_bidirectional_attention():
    # b = 0: no committed context, Eq. (1) is dense bidirectional attention over the S block tokens.
    rs = np.random.default_rng(1)
    B, S, H, d = 2, 8, 2, 16
    q, kb, vb, kc, vc = _rand_attn(rs, B, S, H, H, d, [0, 0])
    out = O.denoise_attention(q, kb, vb, kc, vc, [0, 0], softmax_scale=0.25)
    Q = torch.from_numpy(q.transpose(0, 2, 1, 3).copy())
    K = torch.from_numpy(kb.transpose(0, 2, 1, 3).copy())
    V = torch.from_numpy(vb.transpose(0, 2, 1, 3).copy())
    ref = F.scaled_dot_product_attention(Q, K, V, scale=0.25, is_causal=False).numpy().transpose(0, 2, 1, 3)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_block_of_one_is_decode_attention():
    # S = 1: ordinary single-query decoding attention over L_b + 1 keys; equals the last row of
    # causal attention over the full sequence [context; token].
    rs = np.random.default_rng(2)
    L, H, d = 9, 3, 8
    q, kb, vb, kc, vc = _rand_attn(rs, 1, 1, H, H, d, [L])
    out = O.denoise_attention(q, kb, vb, kc, vc, [L])
    Kfull = np.concatenate([kc[0, :L], kb[0]], axis=0).transpose(1, 0, 2)[None]
    Vfull = np.concatenate([vc[0, :L], vb[0]], axis=0).transpose(1, 0, 2)[None]
    Qfull = np.concatenate([rs.standard_normal((L, H, d)), q[0]], axis=0).transpose(1, 0, 2)[None]
    ref = F.scaled_dot_product_attention(torch.from_numpy(Qfull.copy()), torch.from_numpy(Kfull.copy()),
                                         torch.from_numpy(Vfull.copy()), scale=1.0, is_causal=True)
    np.testing.assert_allclose(out[0, 0], ref[0, :, -1, :].numpy(), rtol=1e-12, atol=1e-12)


def test_permutation_equivariance_in_block():
    rs = np.random.default_rng(3)
    B, S, Hq, Hkv, d = 2, 6, 4, 2, 8
    lens = [7, 3]
    q, kb, vb, kc, vc = _rand_attn(rs, B, S, Hq, Hkv, d, lens)
    base = O.denoise_attention(q, kb, vb, kc, vc, lens)
    perm = rs.permutation(S)
    # jointly permuting the block's keys and values leaves O unchanged
    out_kv = O.denoise_attention(q, kb[:, perm], vb[:, perm], kc, vc, lens)
    np.testing.assert_allclose(out_kv, base, rtol=1e-12, atol=1e-13)
    # permuting the block's queries permutes O the same way
    out_q = O.denoise_attention(q[:, perm], kb, vb, kc, vc, lens)
    np.testing.assert_allclose(out_q, base[:, perm], rtol=1e-12, atol=1e-13)


def test_gqa_equals_mha_with_repeated_kv():
    rs = np.random.default_rng(4)
    B, S, Hq, Hkv, d = 2, 4, 8, 2, 8
    lens = [6, 2]
    q, kb, vb, kc, vc = _rand_attn(rs, B, S, Hq, Hkv, d, lens)
    G = Hq // Hkv
    rep = lambda x: np.repeat(x, G, axis=2)      # kv head j serves q heads j*G .. j*G+G-1
    out = O.denoise_attention(q, kb, vb, kc, vc, lens)
    ref = O.denoise_attention(q, rep(kb), rep(vb), rep(kc), rep(vc), lens)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)
    # and the mapping is h // G, not h % G: a distinct value per kv head shows up in its q heads
    vb2 = np.zeros_like(vb)
    vc2 = np.zeros_like(vc)
    for j in range(Hkv):
        vb2[:, :, j, :] = j + 1.0
        vc2[:, :, j, :] = j + 1.0
    out2 = O.denoise_attention(q, kb, vb2, kc, vc2, lens)
    for h in range(Hq):
        np.testing.assert_allclose(out2[:, :, h, :], h // G + 1.0, atol=1e-12)


def test_paged_equals_contiguous_with_shuffled_pages():
    rs = np.random.default_rng(5)
    B, S, Hq, Hkv, d, ps = 3, 4, 4, 2, 8, 4
    lens = [9, 0, 13]
    q, kb, vb, kc, vc = _rand_attn(rs, B, S, Hq, Hkv, d, lens)
    npg = [(L + ps - 1) // ps for L in lens]
    total = sum(npg)
    perm = rs.permutation(total)
    table = np.full((B, max(npg)), -1, dtype=np.int64)
    kpool = np.zeros((total, ps, Hkv, d))
    vpool = np.zeros((total, ps, Hkv, d))
    pos = 0
    for b in range(B):
        for i in range(npg[b]):
            p = perm[pos]
            pos += 1
            table[b, i] = p
            n = min(ps, lens[b] - i * ps)
            kpool[p, :n] = kc[b, i * ps:i * ps + n]
            vpool[p, :n] = vc[b, i * ps:i * ps + n]
            kpool[p, n:] = 1e3      # garbage past the end of the context must be ignored
            vpool[p, n:] = 1e3
    out = O.denoise_attention(q, kb, vb, kpool, vpool, lens, page_table=table, page_size=ps)
    ref = O.denoise_attention(q, kb, vb, kc, vc, lens)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)


def test_attention_closed_forms_random():
    rs = np.random.default_rng(6)
    B, S, Hq, Hkv, d = 1, 5, 2, 1, 6
    lens = [8]
    q, kb, vb, kc, vc = _rand_attn(rs, B, S, Hq, Hkv, d, lens)
    u = rs.standard_normal(d)
    # all value rows equal to u -> O = u
    out = O.denoise_attention(q, kb, np.broadcast_to(u, vb.shape).copy(), kc, np.broadcast_to(u, vc.shape).copy(), lens)
    np.testing.assert_allclose(out, np.broadcast_to(u, out.shape), atol=1e-13)
    # q = 0 -> O = mean of all L_b + S value rows
    out = O.denoise_attention(np.zeros_like(q), kb, vb, kc, vc, lens)
    mean = np.concatenate([vc[0, :8, 0], vb[0, :, 0]], axis=0).mean(axis=0)
    np.testing.assert_allclose(out[0, :, 0], np.broadcast_to(mean, (S, d)), atol=1e-13)
    # one key with a score 40 above the others -> O is (to exp(-40)) that key's value row
    qq = np.zeros_like(q)
    qq[..., 0] = 1.0
    kk = np.zeros_like(kc)
    kk[0, 3, 0, 0] = 40.0
    out = O.denoise_attention(qq, np.zeros_like(kb), vb, kk, vc, lens)
    np.testing.assert_allclose(out[0, :, 0], np.broadcast_to(vc[0, 3, 0], (S, d)), atol=1e-15 * 1e3)
    # L_b = 0 and S = 1 -> O = v
    out = O.denoise_attention(q[:, :1], kb[:, :1], vb[:, :1], kc, vc, [0])
    np.testing.assert_allclose(out[0, 0, 0], vb[0, 0, 0], atol=1e-15)


def test_attention_brute_force_tiny():
    rs = np.random.default_rng(7)
    B, S, Hq, Hkv, d = 2, 3, 4, 2, 3
    lens = [4, 1]
    q, kb, vb, kc, vc = _rand_attn(rs, B, S, Hq, Hkv, d, lens)
    out = O.denoise_attention(q, kb, vb, kc, vc, lens, softmax_scale=0.9)
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            j = h // G
            keys = [kc[b, t, j] for t in range(lens[b])] + [kb[b, t, j] for t in range(S)]
            vals = [vc[b, t, j] for t in range(lens[b])] + [vb[b, t, j] for t in range(S)]
            for s in range(S):
                w = [math.exp(0.9 * sum(q[b, s, h, i] * k[i] for i in range(d))) for k in keys]
                z = sum(w)
                for i in range(d):
                    ref = sum(wj * v[i] for wj, v in zip(w, vals)) / z
                    assert abs(out[b, s, h, i] - ref) < 1e-12


def test_attention_lse_matches_library_logsumexp():
    rs = np.random.default_rng(8)
    q, kb, vb, kc, vc = _rand_attn(rs, 1, 2, 2, 1, 4, [5])
    _, lse = O.denoise_attention(q, kb, vb, kc, vc, [5], softmax_scale=0.5, return_lse=True)
    from scipy.special import logsumexp
    for h in range(2):
        for s in range(2):
            keys = np.concatenate([kc[0, :5, 0], kb[0, :, 0]], axis=0)
            assert abs(lse[0, h, s] - logsumexp(0.5 * keys @ q[0, s, h])) < 1e-12


# ---------------------------------------------------------------- adaLN-single

def test_timestep_embedding_golden():
    g = json.load(open(os.path.join(GOLDEN, "timestep_closed_forms.json")))
    for c in g["cases"]:
        phi = O.timestep_embedding(np.array([_num(c["tau"])]), c["freq_dim"])
        np.testing.assert_allclose(phi[0], np.array(c["phi"], dtype=np.float64), atol=1e-12, err_msg=c["why"])


def test_timestep_embedding_frequencies():
    # w_k = 10000^(-k/128): the last frequency is 10000^(-127/128); phase of sin/cos halves
    tau = np.array([0.37])
    phi = O.timestep_embedding(tau, 256)
    k = 127
    w = 10000.0 ** (-k / 128.0)
    assert abs(phi[0, k] - math.cos(370.0 * w)) < 1e-12
    assert abs(phi[0, 128 + k] - math.sin(370.0 * w)) < 1e-12
    np.testing.assert_allclose(phi[0, :128] ** 2 + phi[0, 128:] ** 2, 1.0, atol=1e-12)


def test_norm_modulate_identity_mod_is_library_rmsnorm():
    rs = np.random.default_rng(9)
    B, S, D = 2, 3, 16
    h = rs.standard_normal((B, S, D))
    w = 1.0 + 0.1 * rs.standard_normal(D)
    mod = np.zeros((B, 3, D))
    mod[:, 2] = 1.0                       # shift 0, scale 0, gate 1
    y = O.adaln_norm_modulate(h, w, mod, eps=1e-5)
    ref = F.rms_norm(torch.from_numpy(h), (D,), torch.from_numpy(w), eps=1e-5).numpy()
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)
    f = rs.standard_normal((B, S, D))
    np.testing.assert_allclose(O.adaln_gated_residual(h, f, mod), h + f, atol=1e-15)


def test_norm_modulate_uses_each_row_of_mod():
    rs = np.random.default_rng(10)
    B, S, D = 2, 2, 8
    h = rs.standard_normal((B, S, D))
    w = np.ones(D)
    shift = rs.standard_normal((B, D))
    scale = rs.standard_normal((B, D))
    gate = rs.standard_normal((B, D))
    mod = np.stack([shift, scale, gate], axis=1)
    base = F.rms_norm(torch.from_numpy(h), (D,), eps=1e-5).numpy()
    y = O.adaln_norm_modulate(h, w, mod)
    np.testing.assert_allclose(y, base * (1 + scale[:, None]) + shift[:, None], rtol=1e-12, atol=1e-12)
    f = rs.standard_normal((B, S, D))
    np.testing.assert_allclose(O.adaln_gated_residual(h, f, mod), h + gate[:, None] * f, atol=1e-14)


def test_norm_modulate_constant_row():
    # a constant row c: h / rms(h) = sign(c) (up to eps) -> y = sign(c) * w * (1 + scale) + shift
    D = 8
    for c in (3.0, -0.5):
        h = np.full((1, 1, D), c)
        w = np.linspace(0.5, 1.5, D)
        mod = np.zeros((1, 3, D))
        mod[0, 0] = 0.25
        mod[0, 1] = -0.5
        y = O.adaln_norm_modulate(h, w, mod, eps=0.0)
        np.testing.assert_allclose(y[0, 0], np.sign(c) * w * 0.5 + 0.25, atol=1e-14)


def test_adaln_cond_structure():
    rs = np.random.default_rng(12)
    B, F_, D = 3, 8, 8
    W = F_
    tau = np.array([0.0, 0.25, 1.0])
    emb = rs.standard_normal((3, D))
    b3 = rs.standard_normal(3 * D)
    zeros = lambda *s: np.zeros(s)
    # W3 = 0: mod = b3 reshaped (shift, scale, gate) + per-layer embedding
    mod = O.adaln_cond(tau, rs.standard_normal((W, F_)), zeros(W), rs.standard_normal((W, W)), zeros(W),
                       zeros(3 * D, W), b3, emb, freq_dim=F_)
    np.testing.assert_allclose(mod, np.broadcast_to(b3.reshape(3, D) + emb, (B, 3, D)), atol=1e-15)
    # identity W1/W2 and W3 = [I; 2I; 3I]: mod_r = (r+1) * SiLU(SiLU(phi)) (library silu)
    I = np.eye(W)
    mod = O.adaln_cond(tau, I, zeros(W), I, zeros(W), np.concatenate([I, 2 * I, 3 * I], 0), zeros(3 * D),
                       zeros(3, D), freq_dim=F_)
    phi = torch.from_numpy(O.timestep_embedding(tau, F_))
    a = F.silu(F.silu(phi)).numpy()
    for r in range(3):
        np.testing.assert_allclose(mod[:, r, :], (r + 1) * a, rtol=1e-13, atol=1e-14)
    # biases enter before each SiLU
    b1 = rs.standard_normal(W)
    b2 = rs.standard_normal(W)
    mod = O.adaln_cond(tau, I, b1, I, b2, np.concatenate([I, I, I], 0), zeros(3 * D), zeros(3, D), freq_dim=F_)
    a = F.silu(F.silu(phi + torch.from_numpy(b1)) + torch.from_numpy(b2)).numpy()
    np.testing.assert_allclose(mod[:, 1, :], a, rtol=1e-13, atol=1e-14)
    # a general dense case against torch's Linear/SiLU stack in float64
    w1, w2, w3 = rs.standard_normal((W, F_)), rs.standard_normal((W, W)), rs.standard_normal((3 * D, W))
    mod = O.adaln_cond(tau, w1, b1, w2, b2, w3, b3, emb, freq_dim=F_)
    t = lambda x: torch.from_numpy(x)
    ref = F.linear(F.silu(F.linear(F.silu(F.linear(phi, t(w1), t(b1))), t(w2), t(b2))), t(w3), t(b3))
    ref = ref.numpy().reshape(B, 3, D) + emb
    np.testing.assert_allclose(mod, ref, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- ConfidenceSample

def test_confidence_golden():
    g = json.load(open(os.path.join(GOLDEN, "unmask_closed_forms.json")))
    for c in g["confidence"]:
        x = np.array([_num(v) for v in c["logits"].split(",")])
        conf, arg = O.confidence_argmax(x[None], c["inv_temperature"])
        assert abs(conf[0] - c["conf"]) < 1e-14, c["why"]
        assert int(arg[0]) == c["argmax"], c["why"]


def test_commit_golden():
    g = json.load(open(os.path.join(GOLDEN, "unmask_closed_forms.json")))
    for c in g["commit"]:
        t, m, nc, nm = O.confidence_commit(np.array([c["tokens"]]), np.array([c["is_masked"]], bool),
                                           np.array([c["conf"]]), np.array([c["argmax"]]), c["gamma"],
                                           c["remaining_steps"])
        assert t[0].tolist() == c["out_tokens"], c["why"]
        assert m[0].astype(int).tolist() == c["out_is_masked"], c["why"]
        assert int(nc[0]) == c["n_committed"] and int(nm[0]) == c["n_masked"], c["why"]


def test_confidence_uniform_and_peak():
    V = 1000
    conf, arg = O.confidence_argmax(np.zeros((2, V)))
    np.testing.assert_allclose(conf, 1.0 / V, rtol=1e-15)
    assert (arg == 0).all()
    for delta in (0.5, 3.0, 9.0):
        x = np.zeros(V)
        x[417] = delta
        conf, arg = O.confidence_argmax(x[None])
        assert arg[0] == 417
        assert abs(conf[0] - math.exp(delta) / (math.exp(delta) + V - 1)) < 1e-15


def test_confidence_matches_library_softmax():
    rs = np.random.default_rng(13)
    x = 3.0 * rs.standard_normal((4, 5, 64))
    for it in (0.5, 1.0, 10.0):
        conf, arg = O.confidence_argmax(x, it)
        p = torch.softmax(torch.from_numpy(x * it), dim=-1)
        np.testing.assert_allclose(conf, p.max(dim=-1).values.numpy(), rtol=1e-13)
        np.testing.assert_array_equal(arg, torch.from_numpy(x).argmax(dim=-1).numpy())


def test_confidence_excluded_token():
    x = np.zeros((1, 6))
    x[0, 3] = 5.0
    conf, arg = O.confidence_argmax(x, 1.0, exclude_token=3)
    assert arg[0] == 0 and abs(conf[0] - 0.2) < 1e-15


def test_commit_threshold_extremes_and_invariants():
    rs = np.random.default_rng(14)
    B, S, V = 5, 16, 50
    logits = 2.0 * rs.standard_normal((B, S, V))
    tokens = rs.integers(0, V, (B, S))
    is_masked = rs.random((B, S)) < 0.6
    is_masked[0] = False                       # a fully committed sequence
    tokens[is_masked] = 3
    conf, arg = O.confidence_argmax(logits)
    # gamma > 1: exactly one commit per sequence that still has a masked position
    t, m, nc, nm = O.confidence_commit(tokens, is_masked, conf, arg, 1.5)
    np.testing.assert_array_equal(nc, (is_masked.sum(1) > 0).astype(int))
    # gamma <= 1/V: every masked position commits
    t, m, nc, nm = O.confidence_commit(tokens, is_masked, conf, arg, 1.0 / V)
    assert not m.any()
    np.testing.assert_array_equal(t[is_masked], arg[is_masked])
    # committed positions never change; counts add up
    for gamma in (0.05, 0.1, 0.3):
        t, m, nc, nm = O.confidence_commit(tokens, is_masked, conf, arg, gamma)
        np.testing.assert_array_equal(t[~is_masked], tokens[~is_masked])
        assert not (m & ~is_masked).any()
        np.testing.assert_array_equal(nc + nm, is_masked.sum(1))


def test_commit_brute_force_tiny():
    # enumerate the rule literally over all masked subsets sizes for tiny blocks
    rs = np.random.default_rng(15)
    for _ in range(200):
        S = int(rs.integers(1, 6))
        conf = np.round(rs.random((1, S)), 1)          # many ties
        arg = rs.integers(0, 9, (1, S))
        masked = rs.random((1, S)) < 0.7
        toks = np.where(masked, 3, 100)
        gamma = float(rs.choice([0.3, 0.5, 0.8, 1.1]))
        t, m, nc, nm = O.confidence_commit(toks, masked, conf, arg, gamma)
        ml = [l for l in range(S) if masked[0, l]]
        expect = [l for l in ml if conf[0, l] >= gamma]
        if ml and not expect:
            best = max(conf[0, l] for l in ml)
            expect = [min(l for l in ml if conf[0, l] == best)]
        assert sorted(l for l in range(S) if masked[0, l] and not m[0, l]) == sorted(expect)


def test_refinement_loop_closed_behaviour():
    # tiny fp32 workload: logits ~ N(0, 2^2) over 1024 entries give max probability ~0.1 << 0.8,
    # so every step falls back to exactly one commit and the block finishes at r = T = 16 with
    # tau = 16/16, 15/16, ..., 1/16 (Algorithm 2's time input).
    g = json.load(open(os.path.join(GOLDEN, "generation_defaults.json")))
    S, T, mask_id, gamma = g["block_size"], g["steps_per_block"], g["mask_token_id"], g["confidence_threshold"]
    w = synth.workload("tiny_fp32")
    assert (w.attn.block_size, w.steps, w.gamma) == (S, T, gamma)

    def logits_for_step(r, tau):
        return synth.logits_normal(r, 1, S, w.vocab, w.logits_std, torch.float32).double().numpy()

    tokens, is_masked, rec = O.refine_block(1, S, T, gamma, logits_for_step, mask_token_id=mask_id)
    assert not is_masked.any()
    assert [int(nc[0]) for _, _, nc in rec] == [1] * T
    np.testing.assert_allclose([tau[0] for _, tau, _ in rec], [(S - r + 1) / S for r in range(1, T + 1)])


def test_refinement_loop_finishes_within_T_with_schedule():
    # S > T with remaining_steps: the block still completes within T steps (§2.2)
    S, T, V = 32, 8, 64
    rs = np.random.default_rng(16)
    tokens, is_masked, rec = O.refine_block(2, S, T, 0.99, lambda r, tau: rs.standard_normal((2, S, V)),
                                            use_remaining_steps=True)
    assert not is_masked.any()


def test_round_bf16_matches_torch():
    rs = np.random.default_rng(17)
    x = rs.standard_normal(100000) * 10.0 ** rs.integers(-3, 4, 100000)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).double().numpy()
    # torch rounds fp32 -> bf16; values whose fp64 -> fp32 step lands on a bf16 midpoint may
    # differ by one bf16 ulp (double rounding); there must be almost none
    r = O.round_bf16(x)
    diff = r != ref
    assert diff.sum() <= 2
    m, e = np.frexp(r)
    assert np.all(np.rint(m * 256) == m * 256)


# ---------------------------------------------------------------- block commit (Algorithm 1, context update)
def test_append_block_is_concatenation():
    rs = np.random.default_rng(11)
    lens = [0, 5, 17]
    ctx_k = [rs.standard_normal((L, 2, 8)) for L in lens]
    ctx_v = [rs.standard_normal((L, 2, 8)) for L in lens]
    kn, vn = rs.standard_normal((3, 4, 2, 8)), rs.standard_normal((3, 4, 2, 8))
    out_k, out_v, new_lens = O.append_block(ctx_k, ctx_v, kn, vn)
    assert new_lens == [L + 4 for L in lens]
    for b, L in enumerate(lens):
        np.testing.assert_array_equal(out_k[b][:L], ctx_k[b])      # the old context is untouched
        np.testing.assert_array_equal(out_k[b][L:], kn[b])         # the block follows it
        np.testing.assert_array_equal(out_v[b][L:], vn[b])


def test_append_then_attend_sees_the_committed_block():
    # after the commit, the next block's queries attend to context + committed block + own block:
    # the same as one softmax over the three key sets written out directly
    rs = np.random.default_rng(12)
    B, S, Hq, Hkv, d, L = 2, 3, 4, 2, 8, 5
    ctx_k, ctx_v = rs.standard_normal((B, L, Hkv, d)), rs.standard_normal((B, L, Hkv, d))
    kc, vc = rs.standard_normal((B, S, Hkv, d)), rs.standard_normal((B, S, Hkv, d))   # committed block
    q, kb, vb = rs.standard_normal((B, S, Hq, d)), rs.standard_normal((B, S, Hkv, d)), rs.standard_normal((B, S, Hkv, d))
    nk, nv, lens = O.append_block(list(ctx_k), list(ctx_v), kc, vc)
    stride = max(lens)
    k_slab = np.zeros((B, stride, Hkv, d)); v_slab = np.zeros((B, stride, Hkv, d))
    for b in range(B):
        k_slab[b, :lens[b]], v_slab[b, :lens[b]] = nk[b], nv[b]
    got = O.denoise_attention(q, kb, vb, k_slab, v_slab, lens)
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            keys = np.concatenate([ctx_k[b, :, h // G], kc[b, :, h // G], kb[b, :, h // G]])
            vals = np.concatenate([ctx_v[b, :, h // G], vc[b, :, h // G], vb[b, :, h // G]])
            x = q[b, :, h] @ keys.T
            p = np.exp(x - x.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            np.testing.assert_allclose(got[b, :, h], p @ vals, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- predict-and-noise sampler
def test_predict_noise_commits_top_k_by_brute_force():
    rs = np.random.default_rng(21)
    B, S, V = 3, 10, 17
    logits = rs.standard_normal((B, S, V)) * 2
    masked = rs.random((B, S)) < 0.7
    tokens = np.where(masked, 3, rs.integers(0, V, (B, S)))
    conf, arg = O.confidence_argmax(logits)
    for keep in (0, 2, 5, 100):
        t, m, nc, nm, _, _ = O.predict_noise_step(tokens, masked, logits, keep)
        for b in range(B):
            cand = [l for l in range(S) if masked[b, l]]
            k = max(0, len(cand) - keep)
            # brute force: the k positions whose (confidence, -position) is largest
            best = sorted(cand, key=lambda l: (conf[b, l], -l), reverse=True)[:k]
            assert set(np.flatnonzero(masked[b] & ~m[b])) == set(best)
            assert nc[b] == k and nm[b] == len(cand) - k
            for l in best:
                assert t[b, l] == arg[b, l]
            for l in range(S):
                if not masked[b, l]:
                    assert t[b, l] == tokens[b, l] and not m[b, l]   # committed positions untouched


def test_predict_noise_ties_go_to_the_lower_position():
    logits = np.zeros((1, 4, 8))
    logits[0, :, 1] = 5.0                       # four positions with identical confidence
    t, m, nc, _, _, _ = O.predict_noise_step(np.full((1, 4), 3), np.ones((1, 4), bool), logits, 2)
    assert m[0].tolist() == [False, False, True, True] and nc[0] == 2


def _schedule_cases():
    return json.load(open(os.path.join(GOLDEN, "noise_schedule_linear.json")))["cases"]


@pytest.mark.parametrize("case", _schedule_cases(), ids=lambda c: f"S{c['S']}T{c['T']}")
def test_predict_noise_linear_schedule_golden(case):
    # the hand-derived table (alpha_t = 1 - t, the masked fraction after step r is (T - r) / T):
    # the schedule and a whole T-step predict-and-noise loop both follow it, ending with none left
    S, T, want = case["S"], case["T"], case["keep"]
    assert [O.linear_schedule_keep(S, T, r) for r in range(1, T + 1)] == want
    rs = np.random.default_rng(22 + S + T)
    tokens, masked = np.full((2, S), 3), np.ones((2, S), bool)
    left = []
    for r in range(1, T + 1):
        tokens, masked, _, _, _, _ = O.predict_noise_step(tokens, masked, rs.standard_normal((2, S, 32)),
                                                          O.linear_schedule_keep(S, T, r))
        left.append(masked.sum(axis=1).tolist())
    assert left == [[k, k] for k in want] and left[-1] == [0, 0]


def test_predict_noise_excluded_token():
    # with the [MASK] id excluded its logit takes part in neither the confidence nor the argmax
    # (reading R10), so the ranking is the one of the logits with that column removed
    rs = np.random.default_rng(23)
    B, S, V, mask_id = 2, 8, 12, 3
    logits = rs.standard_normal((B, S, V))
    logits[:, :, mask_id] = 30.0
    masked = np.ones((B, S), bool)
    t, m, nc, _, conf, arg = O.predict_noise_step(np.full((B, S), mask_id), masked, logits, 3, exclude_token=mask_id)
    assert (arg != mask_id).all()
    kept = np.delete(logits, mask_id, axis=2)
    p = np.exp(kept - kept.max(axis=2, keepdims=True))
    np.testing.assert_allclose(conf, (p / p.sum(axis=2, keepdims=True)).max(axis=2), rtol=0, atol=1e-15)
    want_arg = np.argmax(kept, axis=2)
    want_arg = want_arg + (want_arg >= mask_id)
    np.testing.assert_array_equal(arg, want_arg)
    for b in range(B):
        top = sorted(range(S), key=lambda l: (conf[b, l], -l), reverse=True)[:S - 3]
        assert set(np.flatnonzero(~m[b])) == set(top) and nc[b] == S - 3
        assert (t[b][~m[b]] == arg[b][~m[b]]).all()
    # without the exclusion every position would predict the [MASK] id with confidence ~1
    _, _, _, _, conf_in, arg_in = O.predict_noise_step(np.full((B, S), mask_id), masked, logits, 3)
    assert (arg_in == mask_id).all() and (conf_in > 0.99).all()


# ---------------------------------------------------------------- LM head
def test_lmhead_logits_pins():
    rs = np.random.default_rng(31)
    x, w = rs.standard_normal((2, 3, 8)), rs.standard_normal((5, 8))
    lg = O.lmhead_logits(x, w)
    # a matrix product written out as nested sums
    for b in range(2):
        for l in range(3):
            for v in range(5):
                assert abs(lg[b, l, v] - sum(x[b, l, d] * w[v, d] for d in range(8))) < 1e-12
    # one-hot hidden state picks a column of W; scaling x scales the logits
    e = np.zeros((1, 1, 8)); e[0, 0, 3] = 1.0
    np.testing.assert_array_equal(O.lmhead_logits(e, w)[0, 0], w[:, 3])
    np.testing.assert_allclose(O.lmhead_logits(2 * x, w), 2 * lg, rtol=0, atol=1e-12)
