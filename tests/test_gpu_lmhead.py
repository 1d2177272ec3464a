"""The unmask step from hidden states with the LM head fused (tt_lmhead_unmask_step) against the
oracle: logits = x W^T in fp64, then the confidence-threshold or predict-and-noise step. The
kernel forms the logits in fp32 on the tensor cores, so an argmax is compared exactly where the
oracle's two largest logits differ by more than 1e-3 (elsewhere the GPU id must be one of the
near-maximal ids), and a commit decision exactly where the oracle confidence is not within the
accumulation error of gamma (or of the next confidence, for the sampler's ranking)."""
import numpy as np
import pytest
import torch

from denoiser_attention_b200 import api
from oracle import tt_oracle as O
from tests._parity import np64

pytestmark = pytest.mark.gpu


def _inputs(B, S, D, V, seed, frac=0.8):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((B, S, D), generator=g).to(torch.bfloat16)
    w = (torch.randn((V, D), generator=g) * (3.0 / D ** 0.5)).to(torch.bfloat16)
    masked = (torch.rand((B, S), generator=g) < frac).to(torch.uint8)
    tokens = torch.randint(0, 1000, (B, S), generator=g, dtype=torch.int32)
    tokens[masked.bool()] = 3
    return x, w, tokens, masked


def _check_reduction(logits, conf, arg, it=1.0, rtol=2e-5):
    conf_or, arg_or = O.confidence_argmax(logits, it)
    assert np.all(np.abs(conf - conf_or) <= rtol * conf_or + 1e-7), np.abs(conf - conf_or).max()
    top2 = np.sort(logits, axis=-1)[..., -2:]
    clear = (top2[..., 1] - top2[..., 0]) > 1e-3
    assert np.array_equal(arg[clear], arg_or[clear])
    # ambiguous rows: the GPU's id is one of the near-maximal logits
    near = logits >= (logits.max(axis=-1, keepdims=True) - 1e-3)
    idx = np.indices(arg.shape)
    assert near[idx[0], idx[1], arg].all()
    return conf_or, arg_or, clear


@pytest.mark.parametrize("B,S,D,V,gamma", [
    (2, 16, 256, 4096, 0.3),
    (8, 16, 2048, 8192, 0.2),        # the decode shape (M = 128 rows) with a reduced vocabulary
    (16, 16, 512, 4096, 0.3),        # two 128-row tiles
    (3, 7, 128, 1024, 0.25),         # rows not a multiple of the tile
])
def test_lmhead_confidence_step_matches_oracle(cuda_lib, B, S, D, V, gamma):
    x, w, tokens, masked = _inputs(B, S, D, V, seed=D + V + B)
    dev = "cuda"
    t, m = tokens.to(dev), masked.to(dev)
    nc, nm, conf, arg = api.lmhead_unmask_step(x.to(dev), w.to(dev), t, m, gamma=gamma)
    torch.cuda.synchronize()
    logits = O.lmhead_logits(np64(x), np64(w))
    conf_or, arg_or, clear = _check_reduction(logits, conf.cpu().double().numpy(), arg.cpu().numpy())
    t_or, m_or, nc_or, nm_or, _, _ = O.unmask_step(tokens.numpy(), masked.numpy().astype(bool), logits, gamma)
    # commits are decided by conf >= gamma (and the fallback ranking): compare where no oracle
    # confidence sits within the fp32 error of gamma and all argmax ids are unambiguous
    band = np.abs(conf_or - gamma) <= 1e-4
    safe = ~band.any(axis=1) & clear.all(axis=1)
    assert safe.sum() >= 1
    np.testing.assert_array_equal(m.cpu().numpy().astype(bool)[safe], m_or[safe])
    np.testing.assert_array_equal(t.cpu().numpy()[safe], t_or[safe])
    np.testing.assert_array_equal(nc.cpu().numpy()[safe], nc_or[safe])
    np.testing.assert_array_equal(nm.cpu().numpy()[safe], nm_or[safe])


def test_lmhead_predict_noise_matches_oracle(cuda_lib):
    B, S, D, V, keep = 4, 16, 512, 4096, 6
    x, w, tokens, masked = _inputs(B, S, D, V, seed=77)
    dev = "cuda"
    t, m = tokens.to(dev), masked.to(dev)
    api.lmhead_unmask_step(x.to(dev), w.to(dev), t, m, gamma=0.8, keep_masked=keep)
    torch.cuda.synchronize()
    logits = O.lmhead_logits(np64(x), np64(w))
    t_or, m_or, _, _, conf_or, _ = O.predict_noise_step(tokens.numpy(), masked.numpy().astype(bool), logits, keep)
    # the ranking is decided by confidence: sequences whose masked confidences are all separated
    # by more than the fp32 error compare exactly
    safe = []
    for b in range(B):
        c = np.sort(conf_or[b][masked.numpy()[b].astype(bool)])
        safe.append(len(c) < 2 or np.min(np.diff(c)) > 1e-4 * c.max())
    safe = np.array(safe)
    assert safe.sum() >= 1
    np.testing.assert_array_equal(m.cpu().numpy().astype(bool)[safe], m_or[safe])
    assert (m.cpu().numpy().sum(axis=1) == np.minimum(masked.numpy().sum(axis=1), keep)).all()


def test_lmhead_full_vocab_sampled_rows(cuda_lib):
    # the decode shape at full size (D = 2048, V = 131072, 128 rows): conf / argmax of a sample of
    # rows against the oracle (the full fp64 product would take minutes on the host)
    B, S, D, V = 8, 16, 2048, 131072
    x, w, tokens, masked = _inputs(B, S, D, V, seed=5)
    dev = "cuda"
    t, m = tokens.to(dev), masked.to(dev)
    _, _, conf, arg = api.lmhead_unmask_step(x.to(dev), w.to(dev), t, m, gamma=0.8)
    torch.cuda.synchronize()
    rows = [(0, 0), (1, 5), (3, 15), (7, 9)]
    xs = np.stack([np64(x)[b, l] for b, l in rows])[None]
    logits = O.lmhead_logits(xs, np64(w))
    _check_reduction(logits, np.array([[conf[b, l].item() for b, l in rows]], dtype=np.float64),
                     np.array([[arg[b, l].item() for b, l in rows]]), rtol=1e-4)


def test_lmhead_excludes_mask_token(cuda_lib):
    B, S, D, V = 2, 8, 128, 1024
    x, w, tokens, masked = _inputs(B, S, D, V, seed=9)
    w[3] = 50.0 / D ** 0.5 * torch.sign(x[0, 0].float()).to(torch.bfloat16)   # token 3 dominates row (0, 0)
    dev = "cuda"
    _, _, conf, arg = api.lmhead_unmask_step(x.to(dev), w.to(dev), tokens.to(dev), masked.to(dev), gamma=0.8,
                                             exclude_mask_token=True)
    torch.cuda.synchronize()
    logits = O.lmhead_logits(np64(x), np64(w))
    conf_or, arg_or = O.confidence_argmax(logits, 1.0, exclude_token=3)
    assert int(arg[0, 0]) == int(arg_or[0, 0]) != 3
    assert np.all(np.abs(conf.cpu().double().numpy() - conf_or) <= 2e-5 * conf_or + 1e-7)


@pytest.mark.parametrize("rem", [1, 3])
def test_lmhead_remaining_steps_matches_oracle(cuda_lib, rem):
    # the confidence sampler with remaining_steps > 0 (the T - r + 1 of Algorithm 2): at least
    # ceil(n_masked / remaining_steps) of the most confident masked positions commit
    B, S, D, V, gamma = 6, 16, 256, 4096, 0.97
    x, w, tokens, masked = _inputs(B, S, D, V, seed=40 + rem)
    dev = "cuda"
    t, m = tokens.to(dev), masked.to(dev)
    nc, nm, conf, arg = api.lmhead_unmask_step(x.to(dev), w.to(dev), t, m, gamma=gamma, remaining_steps=rem)
    torch.cuda.synchronize()
    logits = O.lmhead_logits(np64(x), np64(w))
    conf_or, arg_or, clear = _check_reduction(logits, conf.cpu().double().numpy(), arg.cpu().numpy())
    t_or, m_or, nc_or, nm_or, _, _ = O.unmask_step(tokens.numpy(), masked.numpy().astype(bool), logits, gamma,
                                                   remaining_steps=rem)
    # the schedule's count is exact; the chosen positions compare where the ranking and the
    # threshold are separated by more than the fp32 accumulation error
    n_in = masked.numpy().astype(np.int64).sum(axis=1)
    need = np.where(n_in > 0, -(-n_in // rem), 0)
    assert (nc.cpu().numpy() >= need).all()
    np.testing.assert_array_equal(nc.cpu().numpy() + nm.cpu().numpy(), n_in)
    safe = []
    for b in range(B):
        c = np.sort(conf_or[b][masked.numpy()[b].astype(bool)])
        sep = len(c) < 2 or np.min(np.diff(c)) > 1e-4 * c.max()
        safe.append(sep and not (np.abs(conf_or[b] - gamma) <= 1e-4).any() and clear[b].all())
    safe = np.array(safe)
    assert safe.sum() >= 1
    np.testing.assert_array_equal(m.cpu().numpy().astype(bool)[safe], m_or[safe])
    np.testing.assert_array_equal(t.cpu().numpy()[safe], t_or[safe])
    np.testing.assert_array_equal(nc.cpu().numpy()[safe], nc_or[safe])


def test_lmhead_noise_schedule_in_the_library(cuda_lib):
    # predict-and-noise from hidden states at step r of T of the linear schedule: the library
    # derives keep_masked = floor(S (T - r) / T)
    B, S, D, V, T = 3, 16, 256, 2048, 6
    x, w, _, _ = _inputs(B, S, D, V, seed=61)
    dev = "cuda"
    for r, keep in ((1, 13), (4, 5), (6, 0)):
        t = torch.full((B, S), 3, dtype=torch.int32, device=dev)
        m = torch.ones((B, S), dtype=torch.uint8, device=dev)
        nc, nm, _, _ = api.lmhead_unmask_step(x.to(dev), w.to(dev), t, m, gamma=0.8, noise_schedule=(T, r))
        torch.cuda.synchronize()
        assert nm.cpu().tolist() == [keep] * B and nc.cpu().tolist() == [S - keep] * B
