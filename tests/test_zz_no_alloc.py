"""tt_unmask_step_noalloc (static scratch, no workspace) against tt_unmask_step, through the C ABI.

Same kernel, same partition of the logits: the outputs are compared exactly (conf within 1e-6)
on two calls in a row, and across calls of different sizes, which share the one fixed-layout
scratch. Kept in the last-collected file so that it also runs after every other GPU test has
used the library.
"""
import pytest
import torch

from denoiser_attention_b200 import binding as B
from denoiser_attention_b200 import synth

pytestmark = pytest.mark.gpu


def _inputs(Bn, S, V, dtype, seed, frac=0.8, mask_id=3):
    logits = synth.logits_normal(seed, Bn, S, V, 3.0, dtype).cuda()
    g = torch.Generator().manual_seed(seed)
    masked = (torch.rand((Bn, S), generator=g) < frac).to(torch.uint8)
    tokens = torch.randint(0, 1000, (Bn, S), generator=g, dtype=torch.int32)
    tokens[masked.bool()] = mask_id
    return logits, tokens.cuda(), masked.cuda()


def _run(logits, tokens0, masked0, gamma, noalloc, remaining_steps=0):
    Bn, S, V = logits.shape
    tokens, masked = tokens0.clone(), masked0.clone()
    nc = torch.empty(Bn, dtype=torch.int32, device="cuda")
    nm = torch.empty(Bn, dtype=torch.int32, device="cuda")
    conf = torch.empty((Bn, S), dtype=torch.float32, device="cuda")
    arg = torch.empty((Bn, S), dtype=torch.int32, device="cuda")
    args = B.unmask_args(logits, tokens, masked, nc, nm, gamma=gamma, inv_temperature=1.0, mask_token_id=3,
                         remaining_steps=remaining_steps, conf=conf, argmax=arg)
    if noalloc:
        B.tt_unmask_step_noalloc(args)
    else:
        ws = B.new_workspace(B.tt_unmask_workspace_bytes(args))
        B.tt_unmask_step(args, ws)
    torch.cuda.synchronize()
    return [x.cpu() for x in (tokens, masked, nc, nm, conf, arg)]


def _same(a, b):
    for x, y in zip(a[:4] + a[5:], b[:4] + b[5:]):
        assert torch.equal(x, y)
    assert torch.allclose(a[4], b[4], rtol=0, atol=1e-6)


@pytest.mark.parametrize("Bn,S,V,dtype,gamma", [
    (8, 16, 131072, torch.bfloat16, 0.5),
    (2, 16, 1000, torch.float32, 0.3),
    (64, 64, 1024, torch.float32, 0.2),      # batch * block_size = 4096, the largest supported
])
def test_noalloc_matches_workspace_entry_twice(cuda_lib, Bn, S, V, dtype, gamma):
    logits, tokens, masked = _inputs(Bn, S, V, dtype, seed=Bn * 1000 + S)
    want = _run(logits, tokens, masked, gamma, noalloc=False)
    first = _run(logits, tokens, masked, gamma, noalloc=True)
    second = _run(logits, tokens, masked, gamma, noalloc=True)
    _same(first, want)
    _same(second, want)


def test_noalloc_across_sizes(cuda_lib):
    """Calls of different sizes in a row share the fixed-layout scratch."""
    cases = [(64, 64, 2048, torch.bfloat16), (3, 8, 4104, torch.bfloat16), (16, 32, 512, torch.float32),
             (3, 8, 4104, torch.bfloat16)]
    for i, (Bn, S, V, dtype) in enumerate(cases):
        logits, tokens, masked = _inputs(Bn, S, V, dtype, seed=7 + i, frac=0.6)
        want = _run(logits, tokens, masked, 0.4, noalloc=False, remaining_steps=2)
        got = _run(logits, tokens, masked, 0.4, noalloc=True, remaining_steps=2)
        _same(got, want)


def test_noalloc_rejects_beyond_limit(cuda_lib):
    logits, tokens, masked = _inputs(5, 820, 16, torch.float32, seed=3)   # 4100 rows
    with pytest.raises(B.TTError) as e:
        _run(logits, tokens, masked, 0.5, noalloc=True)
    assert e.value.status == B.TT_ERR_WORKSPACE_TOO_SMALL
