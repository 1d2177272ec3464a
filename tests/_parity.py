"""Helpers shared by the GPU parity tests: oracle calls on the exact bytes the GPU reads, and
the comparison rules (tolerances from the accuracy bar of the step: bf16 inputs with fp32
accumulation -> max abs <= 1e-2 and mean abs <= 1e-3; fp32 inputs -> <= 1e-5; argmax ids
bit-exact; the committed mask bit-exact except where the oracle confidence is within 1e-5 of
gamma, which is counted)."""
from __future__ import annotations

import numpy as np
import torch

from oracle import tt_oracle as O

BF16_MAX_ABS = 1e-2
BF16_MEAN_ABS = 1e-3
FP32_ABS = 1e-5
GAMMA_BAND = 1e-5


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").double().numpy()


def assert_close_attn(gpu: torch.Tensor, ref: np.ndarray, dtype: torch.dtype, what: str = ""):
    g = np64(gpu)
    assert np.isfinite(g).all(), f"{what}: non-finite GPU output"
    err = np.abs(g - ref)
    if dtype == torch.float32:
        assert err.max() <= FP32_ABS, f"{what}: max abs {err.max():.3g} > {FP32_ABS}"
    else:
        assert err.max() <= BF16_MAX_ABS, f"{what}: max abs {err.max():.3g} > {BF16_MAX_ABS}"
        assert err.mean() <= BF16_MEAN_ABS, f"{what}: mean abs {err.mean():.3g} > {BF16_MEAN_ABS}"
    return float(err.max()), float(err.mean())


def assert_close_bf16_rounded(gpu: torch.Tensor, ref: np.ndarray, what: str = ""):
    """bf16 outputs of elementwise ops: the output is defined as the exact value rounded to bf16,
    so compare against the oracle's value rounded the same way; a difference of one bf16 ulp is
    allowed where the fp32 and fp64 results straddle a rounding boundary."""
    g = np64(gpu)
    r = O.round_bf16(ref)
    ulp = np.ldexp(1.0, np.frexp(np.abs(r))[1] - 8)
    err = np.abs(g - r)
    assert (err <= ulp * 1.0001).all(), f"{what}: {int((err > ulp).sum())} elements beyond 1 bf16 ulp"
    assert np.abs(g - ref).mean() <= BF16_MEAN_ABS * 4, f"{what}: mean abs vs exact too large"
    return float((err > 0).mean())


def check_unmask(tokens_in, masked_in, logits, gamma, inv_temp, tokens_gpu, masked_gpu, nc_gpu, nm_gpu,
                 conf_gpu=None, arg_gpu=None, exclude_token=None, remaining_steps=0, oracle_conf_arg=None):
    """Compares one GPU unmask step with the oracle; returns the number of positions in the
    gamma band (whose commit decision is allowed to differ). oracle_conf_arg: the oracle's
    (confidence, argmax) of these logits when the caller has them already (logits is then
    unused)."""
    if oracle_conf_arg is None:
        conf, arg = O.confidence_argmax(np64(logits), inv_temp, exclude_token)
    else:
        conf, arg = oracle_conf_arg
    tin = tokens_in.cpu().numpy().astype(np.int64)
    min_ = masked_in.cpu().numpy().astype(bool)
    tg = tokens_gpu.cpu().numpy().astype(np.int64)
    mg = masked_gpu.cpu().numpy().astype(bool)
    if arg_gpu is not None:
        np.testing.assert_array_equal(arg_gpu.cpu().numpy(), arg, err_msg="argmax ids differ")
    if conf_gpu is not None:
        err = np.abs(conf_gpu.cpu().double().numpy() - conf).max()
        assert err <= FP32_ABS, f"confidence max abs err {err:.3g}"
    t_or, m_or, nc_or, nm_or = O.confidence_commit(tin, min_, conf, arg, gamma, remaining_steps)
    B, S = tin.shape
    band = 0
    for b in range(B):
        # never touches committed positions, never re-masks
        assert (tg[b][~min_[b]] == tin[b][~min_[b]]).all()
        assert not (mg[b] & ~min_[b]).any()
        newly = min_[b] & ~mg[b]
        assert (tg[b][newly] == arg[b][newly]).all(), "committed token is not the argmax"
        assert (tg[b][mg[b]] == tin[b][mg[b]]).all()
        near = min_[b] & (np.abs(conf[b] - gamma) <= GAMMA_BAND)
        band += int(near.sum())
        ml = np.nonzero(min_[b])[0]
        n_ge = int((conf[b][ml] >= gamma).sum())
        need = 0
        if len(ml):
            need = min(len(ml), -(-len(ml) // remaining_steps) if remaining_steps > 0 else 1)
        srt = np.sort(conf[b][ml])[::-1]
        tie = n_ge < need < len(ml) and srt[need - 1] - srt[need] <= 1e-6
        if not near.any() and not tie:
            np.testing.assert_array_equal(mg[b], m_or[b], err_msg=f"sequence {b}: committed mask differs")
        else:
            # a decision the accuracy bar cannot separate: check the commit set is a valid one
            assert not (min_[b] & (conf[b] >= gamma + GAMMA_BAND) & mg[b]).any(), \
                f"sequence {b}: a position clearly above gamma stayed masked"
            k = int(newly.sum())
            assert k >= need
            low = newly & (conf[b] < gamma - GAMMA_BAND)
            if low.any():
                kth = srt[need - 1]
                assert (conf[b][low] >= kth - 1e-6).all(), f"sequence {b}: fallback picked a non-maximal position"
        assert int(nc_gpu[b]) == int(newly.sum())
        assert int(nm_gpu[b]) == int(mg[b].sum())
    return band
