"""adaLN-single on the GPU (through the C ABI) against the CPU fp64 oracle."""
import numpy as np
import pytest
import torch

from denoiser_attention_b200 import api, synth
from oracle import tt_oracle as O
from tests._parity import assert_close_bf16_rounded, np64

pytestmark = pytest.mark.gpu


def _dev(x):
    return x.to("cuda")


@pytest.mark.parametrize("B,D,F,W,tau", [
    (1, 256, 256, 256, [1.0]),
    (8, 2048, 256, 256, [1.0, 15 / 16, 0.5, 9 / 16, 1 / 16, 0.25, 0.75, 0.125]),
    (3, 96, 64, 100, [0.0, 0.3, 0.999]),
    (64, 2048, 256, 256, [9 / 16] * 32 + [k / 16 for k in range(32)]),   # the batch workload's width
    (70, 64, 128, 1024, [((7 * k) % 17) / 16 for k in range(70)]),       # sequence chunks, widest layer
    (70, 2040, 256, 256, [((5 * k) % 17) / 16 for k in range(70)]),      # 6120 output rows: a ragged last slice
])
def test_cond_matches_oracle(cuda_lib, B, D, F, W, tau):
    a = synth.adaln_inputs(B, 2, D, tau, seed=D + W, dtype=torch.float32, freq_dim=F, mlp_width=W)
    mod = api.adaln_cond(_dev(a.tau), _dev(a.w1), _dev(a.b1), _dev(a.w2), _dev(a.b2), _dev(a.w3), _dev(a.b3),
                         _dev(a.layer_emb))
    ref = O.adaln_cond(np64(a.tau), np64(a.w1), np64(a.b1), np64(a.w2), np64(a.b2), np64(a.w3), np64(a.b3),
                       np64(a.layer_emb), freq_dim=F)
    err = np.abs(np64(mod) - ref).max()
    assert err <= 1e-5, err


@pytest.mark.parametrize("dtype,B,S,D", [(torch.float32, 1, 16, 256), (torch.bfloat16, 8, 16, 2048),
                                         (torch.bfloat16, 2, 3, 8), (torch.float32, 3, 5, 4100)])
def test_norm_modulate_and_gated_residual(cuda_lib, dtype, B, S, D):
    a = synth.adaln_inputs(B, S, D, [0.5] * B, seed=S + D, dtype=dtype)
    g = torch.Generator().manual_seed(D)
    mod = (0.3 * torch.randn((B, 3, D), generator=g)).float()
    y = api.adaln_norm_modulate(_dev(a.h), _dev(a.norm_w), _dev(mod), eps=1e-5)
    hn = api.adaln_gated_residual(_dev(a.h), _dev(a.f), _dev(mod))
    y_ref = O.adaln_norm_modulate(np64(a.h), np64(a.norm_w), np64(mod), 1e-5)
    h_ref = O.adaln_gated_residual(np64(a.h), np64(a.f), np64(mod))
    if dtype == torch.float32:
        # the accuracy bar for fp32 outputs: absolute 1e-5
        assert np.abs(np64(y) - y_ref).max() <= 1e-5, np.abs(np64(y) - y_ref).max()
        assert np.abs(np64(hn) - h_ref).max() <= 1e-5
    else:
        assert_close_bf16_rounded(y, y_ref, "norm_modulate")
        assert_close_bf16_rounded(hn, h_ref, "gated_residual")


@pytest.mark.parametrize("dtype,B,S,D", [(torch.float32, 1, 16, 256), (torch.bfloat16, 8, 16, 2048),
                                         (torch.bfloat16, 2, 3, 8), (torch.float32, 3, 5, 4100),
                                         (torch.bfloat16, 2, 4, 4160)])
def test_norm_modulate_residual_fused(cuda_lib, dtype, B, S, D):
    # one launch for both outputs, against the two oracle functions; D = 4100 (fp32) and 4160 (bf16)
    # are wider than the rows a warp keeps in registers
    a = synth.adaln_inputs(B, S, D, [0.5] * B, seed=S + D + 1, dtype=dtype)
    g = torch.Generator().manual_seed(D + 1)
    mod = (0.3 * torch.randn((B, 3, D), generator=g)).float()
    y, hn = api.adaln_norm_modulate_residual(_dev(a.h), _dev(a.f), _dev(a.norm_w), _dev(mod), eps=1e-5)
    y_ref = O.adaln_norm_modulate(np64(a.h), np64(a.norm_w), np64(mod), 1e-5)
    h_ref = O.adaln_gated_residual(np64(a.h), np64(a.f), np64(mod))
    if dtype == torch.float32:
        assert np.abs(np64(y) - y_ref).max() <= 1e-5, np.abs(np64(y) - y_ref).max()
        assert np.abs(np64(hn) - h_ref).max() <= 1e-5
    else:
        assert_close_bf16_rounded(y, y_ref, "fused norm_modulate")
        assert_close_bf16_rounded(hn, h_ref, "fused gated_residual")
    # the same with the residual written over h (rows both inside and beyond the register cache)
    h = _dev(a.h).clone()
    y2, _ = api.adaln_norm_modulate_residual(h, _dev(a.f), _dev(a.norm_w), _dev(mod), eps=1e-5, out2=h)
    assert torch.equal(y2, y)
    assert torch.equal(h, hn)


def test_gated_residual_in_place(cuda_lib):
    a = synth.adaln_inputs(2, 4, 64, [0.5, 0.5], seed=3, dtype=torch.bfloat16)
    mod = torch.randn((2, 3, 64)).float()
    h = _dev(a.h).clone()
    ref = O.adaln_gated_residual(np64(a.h), np64(a.f), np64(mod))
    api.adaln_gated_residual(h, _dev(a.f), _dev(mod), out=h)
    assert_close_bf16_rounded(h, ref, "in place")
