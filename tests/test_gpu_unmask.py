"""ConfidenceSample on the GPU (through the C ABI) against the CPU fp64 oracle: confidence within
1e-5, argmax ids bit-exact (lowest id on ties), committed tokens/mask bit-exact except at
positions whose oracle confidence is within 1e-5 of gamma (counted)."""
import numpy as np
import pytest
import torch

from denoiser_attention_b200 import api, synth
from tests._parity import check_unmask, np64

pytestmark = pytest.mark.gpu


def _state(B, S, seed, frac_masked=1.0, mask_id=3):
    g = torch.Generator().manual_seed(seed)
    masked = (torch.rand((B, S), generator=g) < frac_masked).to(torch.uint8)
    tokens = torch.randint(0, 1000, (B, S), generator=g, dtype=torch.int32)
    tokens[masked.bool()] = mask_id
    return tokens, masked


def _step(logits, tokens, masked, **kw):
    dev = "cuda"
    t = tokens.to(dev)
    m = masked.to(dev)
    nc, nm, conf, arg = api.unmask_step(logits.to(dev), t, m, **kw)
    torch.cuda.synchronize()
    return t.cpu(), m.cpu(), nc.cpu(), nm.cpu(), conf.cpu(), arg.cpu()


@pytest.mark.parametrize("B,S,V,dtype,std,gamma,it,frac", [
    (1, 16, 1024, torch.float32, 2.0, 0.8, 1.0, 1.0),
    (2, 16, 1000, torch.float32, 0.5, 0.8, 10.0, 0.7),
    (3, 8, 4096 + 8, torch.bfloat16, 3.0, 0.5, 4.0, 0.9),
    (2, 64, 32000, torch.bfloat16, 3.0, 0.3, 3.0, 0.5),
    (4, 16, 131072, torch.bfloat16, 3.0, 0.8, 1.0, 1.0),
    (1, 1024, 256, torch.float32, 1.0, 0.05, 2.0, 0.8),
])
def test_unmask_matches_oracle(cuda_lib, B, S, V, dtype, std, gamma, it, frac):
    logits = synth.logits_normal(V + S, B, S, V, std, dtype)
    tokens, masked = _state(B, S, seed=V, frac_masked=frac)
    t, m, nc, nm, conf, arg = _step(logits, tokens, masked, gamma=gamma, inv_temperature=it)
    check_unmask(tokens, masked, logits, gamma, it, t, m, nc, nm, conf, arg)


def test_decode_workload_logits(cuda_lib):
    w = synth.workload("decode_bf16")
    logits = synth.workload_logits(w)
    tokens, masked = _state(8, 16, seed=1)
    t, m, nc, nm, conf, arg = _step(logits, tokens, masked, gamma=w.gamma)
    band = check_unmask(tokens, masked, logits, w.gamma, 1.0, t, m, nc, nm, conf, arg)
    frac = float((np64(conf) >= w.gamma).mean())
    print(f"positions above gamma: {frac:.2f}, in the 1e-5 band: {band}")
    assert 0.15 < frac < 0.45


def test_ties_take_lowest_token_id(cuda_lib):
    B, S, V = 2, 4, 8192
    logits = torch.zeros((B, S, V), dtype=torch.bfloat16)
    logits[0, 0, [5000, 17, 8000]] = 2.0      # tie across chunks: lowest id 17
    logits[0, 1, :] = 1.0                     # all equal: id 0
    logits[1, 2, [8191, 4096]] = 3.0
    tokens, masked = _state(B, S, seed=3)
    t, m, nc, nm, conf, arg = _step(logits, tokens, masked, gamma=0.9)
    assert arg[0, 0] == 17 and arg[0, 1] == 0 and arg[1, 2] == 4096
    assert abs(float(conf[0, 1]) - 1.0 / V) < 1e-9
    check_unmask(tokens, masked, logits, 0.9, 1.0, t, m, nc, nm, conf, arg)


def test_exclude_mask_token(cuda_lib):
    B, S, V = 2, 8, 2048
    logits = synth.logits_normal(5, B, S, V, 1.0, torch.float32)
    logits[:, :, 3] = 50.0                     # the [MASK] logit dominates unless excluded
    tokens, masked = _state(B, S, seed=4)
    t, m, nc, nm, conf, arg = _step(logits, tokens, masked, gamma=0.8, exclude_mask_token=True, mask_token_id=3)
    assert (arg != 3).all()
    check_unmask(tokens, masked, logits, 0.8, 1.0, t, m, nc, nm, conf, arg, exclude_token=3)


@pytest.mark.parametrize("rem", [1, 2, 5])
def test_remaining_steps_schedule(cuda_lib, rem):
    B, S, V = 4, 32, 4096
    logits = synth.logits_normal(6, B, S, V, 2.0, torch.bfloat16)
    tokens, masked = _state(B, S, seed=5, frac_masked=0.8)
    t, m, nc, nm, conf, arg = _step(logits, tokens, masked, gamma=0.99, remaining_steps=rem)
    check_unmask(tokens, masked, logits, 0.99, 1.0, t, m, nc, nm, conf, arg, remaining_steps=rem)
    n_in = masked.sum(1)
    assert (nc.long() >= torch.clamp((n_in + rem - 1) // rem, max=S)).all()


def test_fully_committed_sequence_unchanged(cuda_lib):
    B, S, V = 3, 16, 1024
    logits = synth.logits_normal(7, B, S, V, 2.0, torch.float32)
    tokens, masked = _state(B, S, seed=6)
    masked[1] = 0
    t, m, nc, nm, conf, arg = _step(logits, tokens, masked, gamma=0.8)
    assert nc[1] == 0 and nm[1] == 0 and torch.equal(t[1], tokens[1])
    check_unmask(tokens, masked, logits, 0.8, 1.0, t, m, nc, nm, conf, arg)


def test_block_loop_tiny_closes_in_T_steps(cuda_lib):
    # Algorithm 2 on the device for the tiny workload: logits redrawn each step (seed r), tau is
    # the masked fraction; with max probability ~0.1 << gamma every step commits exactly one
    # position and the block finishes at r = T = 16 -- the same trajectory as the oracle's loop.
    from oracle import tt_oracle as O
    w = synth.workload("tiny_fp32")
    S, T = w.attn.block_size, w.steps
    dev = "cuda"
    tokens = torch.full((1, S), 3, dtype=torch.int32, device=dev)
    masked = torch.ones((1, S), dtype=torch.uint8, device=dev)
    traj = []
    for r in range(1, T + 1):
        logits = synth.logits_normal(r, 1, S, w.vocab, w.logits_std, torch.float32).to(dev)
        nc, nm, _, _ = api.unmask_step(logits, tokens, masked, gamma=w.gamma)
        traj.append(int(nc.item()))
    assert traj == [1] * T and int(masked.sum()) == 0
    t_or, m_or, _ = O.refine_block(1, S, T, w.gamma, lambda r, tau: synth.logits_normal(
        r, 1, S, w.vocab, w.logits_std, torch.float32).double().numpy())
    np.testing.assert_array_equal(tokens.cpu().numpy(), t_or)


@pytest.mark.parametrize("B,S,V,dtype,keep", [
    (4, 16, 131072, torch.bfloat16, 10),
    (2, 64, 32000, torch.bfloat16, 0),
    (3, 8, 1000, torch.float32, 3),
    (2, 16, 1024, torch.float32, 16),     # keep >= masked: nothing commits
])
def test_predict_noise_matches_oracle(cuda_lib, B, S, V, dtype, keep):
    from oracle import tt_oracle as O
    logits = synth.logits_normal(V + S + keep, B, S, V, 3.0, dtype)
    tokens, masked = _state(B, S, seed=V + keep, frac_masked=0.8)
    dev = "cuda"
    t, m = tokens.to(dev), masked.to(dev)
    nc, nm, conf, arg = api.unmask_step(logits.to(dev), t, m, gamma=0.8, keep_masked=keep)
    torch.cuda.synchronize()
    t_or, m_or, nc_or, nm_or, conf_or, arg_or = O.predict_noise_step(tokens.numpy(), masked.numpy().astype(bool),
                                                                     np64(logits), keep)
    np.testing.assert_array_equal(arg.cpu().numpy(), arg_or)
    assert np.abs(conf.cpu().double().numpy() - conf_or).max() <= 1e-5
    np.testing.assert_array_equal(nc.cpu().numpy(), nc_or)
    np.testing.assert_array_equal(nm.cpu().numpy(), nm_or)
    np.testing.assert_array_equal(t.cpu().numpy(), t_or)
    np.testing.assert_array_equal(m.cpu().numpy().astype(bool), m_or)


def test_predict_noise_schedule_loop(cuda_lib):
    # T steps of the linear schedule on the device: the trajectory (masked count per step, tokens)
    # equals the oracle's, and the block is complete at step T
    from oracle import tt_oracle as O
    B, S, T, V = 2, 16, 5, 4096
    dev = "cuda"
    t = torch.full((B, S), 3, dtype=torch.int32, device=dev)
    m = torch.ones((B, S), dtype=torch.uint8, device=dev)
    t_or, m_or = np.full((B, S), 3), np.ones((B, S), bool)
    for r in range(1, T + 1):
        logits = synth.logits_normal(100 + r, B, S, V, 3.0, torch.bfloat16)
        keep = api.linear_schedule_keep(S, T, r)     # computed by the library (tt_linear_schedule_keep)
        api.unmask_step(logits.to(dev), t, m, gamma=0.8, keep_masked=keep)
        t_or, m_or, _, _, _, _ = O.predict_noise_step(t_or, m_or, np64(logits), O.linear_schedule_keep(S, T, r))
        torch.cuda.synchronize()
        assert int(m.sum()) == B * keep
        np.testing.assert_array_equal(t.cpu().numpy(), t_or)
    assert int(m.sum()) == 0


# ---------------------------------------------------------------- the block-sweep workload's grid
# block sizes S in {4, 8, 16, 32, 64} x softmax temperatures {0.5, 1, 2} (inv_temperature 2, 1,
# 0.5) x gamma in {0.5, 0.7, 0.8, 0.9, 0.95}, on the full batch of 32 sequences with vocabulary
# 131072; the oracle's confidences are computed once per (S, temperature) on the host.
SWEEP_GAMMAS = (0.5, 0.7, 0.8, 0.9, 0.95)


def _oracle_conf_chunked(logits, inv_temp, rows=256, exclude_token=None):
    from oracle import tt_oracle as O
    B, S, V = logits.shape
    flat = logits.reshape(B * S, V)
    conf, arg = [], []
    for i in range(0, B * S, rows):
        c, a = O.confidence_argmax(flat[i:i + rows].double().numpy(), inv_temp, exclude_token)
        conf.append(c)
        arg.append(a)
    return np.concatenate(conf).reshape(B, S), np.concatenate(arg).reshape(B, S)


@pytest.mark.parametrize("S", [4, 8, 16, 32, 64])
def test_block_sweep_grid_matches_oracle(cuda_lib, S):
    from oracle import tt_oracle as O
    w = synth.workload("sweep_bf16", block_size=S)
    B = w.attn.batch
    logits = synth.workload_logits(w)
    dev = "cuda"
    lg = logits.to(dev)
    tokens0 = torch.full((B, S), 3, dtype=torch.int32)
    masked0 = torch.ones((B, S), dtype=torch.uint8)
    band = 0
    for inv_temp in (2.0, 1.0, 0.5):
        conf_or, arg_or = _oracle_conf_chunked(logits, inv_temp)
        for gamma in SWEEP_GAMMAS:
            t, m = tokens0.to(dev), masked0.to(dev)
            nc, nm, conf, arg = api.unmask_step(lg, t, m, gamma=gamma, inv_temperature=inv_temp)
            torch.cuda.synchronize()
            band += check_unmask(tokens0, masked0, None, gamma, inv_temp, t, m, nc, nm, conf, arg,
                                 oracle_conf_arg=(conf_or, arg_or))
    print(f"S={S}: positions in the 1e-5 band around gamma over the grid: {band}")


def test_batch_workload_unmask_full_size(cuda_lib):
    # the batch workload's logits at full size: 64 sequences x 16 positions x 131072 (1024 rows,
    # every CTA range straddles rows and every sequence ticket sees its 16 rows)
    w = synth.workload("batch_bf16")
    B, S = w.attn.batch, w.attn.block_size
    logits = synth.workload_logits(w)
    g = torch.Generator().manual_seed(2)
    masked = (torch.rand((B, S), generator=g) < 9 / 16).to(torch.uint8)   # t = 8 of 16: about 9/16 masked
    tokens = torch.randint(0, 1000, (B, S), generator=g, dtype=torch.int32)
    tokens[masked.bool()] = 3
    t, m, nc, nm, conf, arg = _step(logits, tokens, masked, gamma=w.gamma)
    check_unmask(tokens, masked, logits, w.gamma, 1.0, t, m, nc, nm, conf, arg)


@pytest.mark.parametrize("B,S,V,dtype,keep", [
    (4, 16, 131072, torch.bfloat16, 6),
    (3, 8, 2048, torch.float32, 2),
])
def test_predict_noise_excluding_mask_token(cuda_lib, B, S, V, dtype, keep):
    from oracle import tt_oracle as O
    logits = synth.logits_normal(V + keep + 1, B, S, V, 2.0, dtype)
    logits[:, :, 3] = 40.0                      # the [MASK] logit would win every position unless excluded
    tokens, masked = _state(B, S, seed=V + 1, frac_masked=0.9)
    dev = "cuda"
    t, m = tokens.to(dev), masked.to(dev)
    nc, nm, conf, arg = api.unmask_step(logits.to(dev), t, m, gamma=0.8, keep_masked=keep, exclude_mask_token=True,
                                        mask_token_id=3)
    torch.cuda.synchronize()
    t_or, m_or, nc_or, nm_or, conf_or, arg_or = O.predict_noise_step(
        tokens.numpy(), masked.numpy().astype(bool), np64(logits), keep, exclude_token=3)
    assert (arg.cpu().numpy() != 3).all()
    np.testing.assert_array_equal(arg.cpu().numpy(), arg_or)
    assert np.abs(conf.cpu().double().numpy() - conf_or).max() <= 1e-5
    np.testing.assert_array_equal(nc.cpu().numpy(), nc_or)
    np.testing.assert_array_equal(nm.cpu().numpy(), nm_or)
    np.testing.assert_array_equal(t.cpu().numpy(), t_or)
    np.testing.assert_array_equal(m.cpu().numpy().astype(bool), m_or)


def test_predict_noise_schedule_in_the_library(cuda_lib):
    # noise_schedule=(T, r): the library derives keep_masked from the linear schedule; the T-step
    # trajectory follows the hand-derived table and the oracle
    import json
    import os
    from oracle import tt_oracle as O
    golden = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "noise_schedule_linear.json")))
    case = [c for c in golden["cases"] if c["S"] == 16 and c["T"] == 6][0]
    B, S, T, V = 3, 16, 6, 4096
    dev = "cuda"
    t = torch.full((B, S), 3, dtype=torch.int32, device=dev)
    m = torch.ones((B, S), dtype=torch.uint8, device=dev)
    t_or, m_or = np.full((B, S), 3), np.ones((B, S), bool)
    for r in range(1, T + 1):
        logits = synth.logits_normal(300 + r, B, S, V, 3.0, torch.bfloat16)
        nc, nm, _, _ = api.unmask_step(logits.to(dev), t, m, gamma=0.8, noise_schedule=(T, r))
        t_or, m_or, _, _, _, _ = O.predict_noise_step(t_or, m_or, np64(logits), case["keep"][r - 1])
        torch.cuda.synchronize()
        assert nm.cpu().tolist() == [case["keep"][r - 1]] * B
        np.testing.assert_array_equal(t.cpu().numpy(), t_or)
        np.testing.assert_array_equal(m.cpu().numpy().astype(bool), m_or)
    assert int(m.sum()) == 0
