"""C ABI checks that need no GPU: the library loads, exports every function include/*.h
declares, and rejects bad arguments on the host before anything is launched."""
import ctypes
import glob
import os
import re
import subprocess

import pytest

from denoiser_attention_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(tt_\w+)\s*\(", src, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    from denoiser_attention_b200 import build
    build.build()
    return B.lib()


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for n in ("tt_denoise_attn", "tt_adaln_modulate", "tt_unmask_step", "tt_get_device_error"):
        assert n in names
    assert set(names) == set(B.EXPORTED), names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for n in _declared_functions():
        assert n in exported, n
        getattr(lib, n)


def test_status_strings(lib):
    assert B.status_string(0) == "TT_OK"
    assert B.status_string(6) == "TT_ERR_DEVICE_TIMEOUT"
    assert lib.tt_version() >= 100


def _attn_args(**kw):
    a = B.AttnArgs()
    a.batch, a.block_size, a.num_q_heads, a.num_kv_heads, a.head_dim = 2, 16, 32, 2, 128
    a.dtype, a.softmax_scale = B.TT_BF16, 1.0
    for f in ("q", "k_blk", "v_blk", "k_ctx", "v_ctx", "ctx_lens", "out"):
        setattr(a, f, 4096)
    a.ctx_stride = 4096
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,status", [
    (dict(batch=0), B.TT_ERR_INVALID_ARGUMENT),
    (dict(num_q_heads=31), B.TT_ERR_INVALID_ARGUMENT),
    (dict(q=None), B.TT_ERR_INVALID_ARGUMENT),
    (dict(ctx_lens=None), B.TT_ERR_INVALID_ARGUMENT),
    (dict(dtype=7), B.TT_ERR_INVALID_ARGUMENT),
    (dict(softmax_scale=0.0), B.TT_ERR_INVALID_ARGUMENT),
    (dict(block_size=65), B.TT_ERR_UNSUPPORTED),
    (dict(head_dim=96), B.TT_ERR_UNSUPPORTED),
    (dict(page_table=4096, page_size=100, max_pages_per_seq=4, num_pages=8), B.TT_ERR_UNSUPPORTED),
    (dict(page_table=4096, page_size=0, max_pages_per_seq=4, num_pages=8), B.TT_ERR_INVALID_ARGUMENT),
    (dict(q=4098), B.TT_ERR_UNSUPPORTED),
])
def test_attn_host_validation(lib, kw, status):
    a = _attn_args(**kw)
    assert lib.tt_denoise_attn(ctypes.byref(a), 4096, 1 << 30, None) == status
    assert lib.tt_denoise_attn_workspace_bytes(ctypes.byref(a)) == 0


def test_attn_workspace_too_small(lib):
    a = _attn_args()
    need = lib.tt_denoise_attn_workspace_bytes(ctypes.byref(a))
    assert need > 256
    assert lib.tt_denoise_attn(ctypes.byref(a), 4096, need - 1, None) == B.TT_ERR_WORKSPACE_TOO_SMALL
    assert lib.tt_denoise_attn(ctypes.byref(a), None, need, None) == B.TT_ERR_INVALID_ARGUMENT


def _attn_ws_bytes(units, slots):
    # header, the partition's totals, per group its first/last team, the split-KV partials
    # [slots][128][128] and their log-sum-exps [slots][128], each start 256-byte aligned
    off = 256
    for nbytes in (16, 8 * units, 4 * slots * 128 * 128, 4 * slots * 128):
        off = (off + nbytes + 255) // 256 * 256
    return off


@pytest.mark.parametrize("batch,stride,paged,one_tile", [
    (8, 4096, False, True),       # decode shape: 528 key tiles at most, <= 32 per SM
    (32, 8192, False, True),      # block sweep at S = 16: 4160 tiles
    (64, 16384, False, False),    # batch shape: 16512 tiles, the two-stream kernel
    (4, 0, True, False),          # paged, 480 pages of 256 per sequence: 7688 tiles at most
])
def test_attn_plan_picks_kernel_from_capacity(lib, batch, stride, paged, one_tile):
    # Groups of two query tiles (G = 16, S = 16) run the one-tile kernel (teams of two CTAs) when the
    # host's bound on the key tiles, from the context capacity, is at most 32 per SM; otherwise the
    # two-stream kernel (one CTA per team). The workspace holds one partial per (group + team) and
    # query tile, so its size shows the choice (148 SMs when no GPU is present).
    kw = dict(batch=batch, ctx_stride=stride)
    if paged:
        kw.update(page_table=4096, page_size=256, max_pages_per_seq=480, num_pages=2048, ctx_stride=0)
    a = _attn_args(**kw)
    units, sms = batch * 2, 148
    teams = sms // 2 if one_tile else sms
    assert lib.tt_denoise_attn_workspace_bytes(ctypes.byref(a)) == _attn_ws_bytes(units, (units + teams) * 2)


def _unmask_args(**kw):
    a = B.UnmaskArgs()
    a.batch, a.block_size, a.vocab, a.dtype = 2, 16, 1024, B.TT_BF16
    a.logits = a.tokens = a.is_masked = a.n_committed = a.n_masked = 4096
    a.gamma, a.inv_temperature = 0.8, 1.0
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,status", [
    (dict(vocab=0), B.TT_ERR_INVALID_ARGUMENT),
    (dict(tokens=None), B.TT_ERR_INVALID_ARGUMENT),
    (dict(inv_temperature=0.0), B.TT_ERR_INVALID_ARGUMENT),
    (dict(remaining_steps=-1), B.TT_ERR_INVALID_ARGUMENT),
    (dict(exclude_mask_token=1, mask_token_id=5000), B.TT_ERR_INVALID_ARGUMENT),
    (dict(vocab=1001), B.TT_ERR_UNSUPPORTED),
    (dict(block_size=1025), B.TT_ERR_UNSUPPORTED),
])
def test_unmask_host_validation(lib, kw, status):
    a = _unmask_args(**kw)
    assert lib.tt_unmask_step(ctypes.byref(a), 4096, 1 << 30, None) == status


def test_unmask_workspace_sizes(lib):
    a = _unmask_args(batch=8, vocab=131072)
    need = lib.tt_unmask_workspace_bytes(ctypes.byref(a))
    assert need >= 256 + 8 * 16 * (4 + 4 + 4)
    assert lib.tt_unmask_step(ctypes.byref(a), 4096, need - 1, None) == B.TT_ERR_WORKSPACE_TOO_SMALL


def _adaln_args(**kw):
    a = B.AdalnArgs()
    a.op, a.batch, a.block_size, a.hidden, a.freq_dim, a.mlp_width = B.TT_ADALN_COND, 2, 16, 256, 256, 256
    a.dtype, a.eps = B.TT_F32, 1e-5
    for f in ("tau", "w1", "b1", "w2", "b2", "w3", "b3", "layer_emb", "mod", "h", "norm_w", "f", "out"):
        setattr(a, f, 4096)
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,status", [
    (dict(op=9), B.TT_ERR_INVALID_ARGUMENT),
    (dict(freq_dim=255), B.TT_ERR_INVALID_ARGUMENT),
    (dict(w3=None), B.TT_ERR_INVALID_ARGUMENT),
    (dict(mlp_width=2048), B.TT_ERR_UNSUPPORTED),
    (dict(freq_dim=258), B.TT_ERR_UNSUPPORTED),
    (dict(mlp_width=102), B.TT_ERR_UNSUPPORTED),
    (dict(w2=4100), B.TT_ERR_UNSUPPORTED),
    (dict(op=B.TT_ADALN_NORM_MODULATE, norm_w=None), B.TT_ERR_INVALID_ARGUMENT),
    (dict(op=B.TT_ADALN_NORM_MODULATE, hidden=6), B.TT_ERR_UNSUPPORTED),
    (dict(op=B.TT_ADALN_GATED_RESIDUAL, f=None), B.TT_ERR_INVALID_ARGUMENT),
    (dict(op=B.TT_ADALN_GATED_RESIDUAL, dtype=B.TT_BF16, hidden=260), B.TT_ERR_UNSUPPORTED),
    (dict(op=B.TT_ADALN_NORM_MODULATE, norm_w=4100), B.TT_ERR_UNSUPPORTED),      # read as float4
    (dict(op=B.TT_ADALN_GATED_RESIDUAL, mod=4104), B.TT_ERR_UNSUPPORTED),
    # the fused RMSNorm + gated residual: a second output, not the first one, and y not over f
    (dict(op=B.TT_ADALN_NORM_MODULATE_RESIDUAL, f=12288), B.TT_ERR_INVALID_ARGUMENT),           # out2 NULL
    (dict(op=B.TT_ADALN_NORM_MODULATE_RESIDUAL, f=12288, out2=4096), B.TT_ERR_INVALID_ARGUMENT),
    (dict(op=B.TT_ADALN_NORM_MODULATE_RESIDUAL, out2=8192), B.TT_ERR_INVALID_ARGUMENT),          # out == f
    (dict(op=B.TT_ADALN_NORM_MODULATE_RESIDUAL, f=12288, out2=8200), B.TT_ERR_UNSUPPORTED),     # unaligned
    (dict(op=B.TT_ADALN_NORM_MODULATE_RESIDUAL, f=12288, out2=8192, norm_w=None), B.TT_ERR_INVALID_ARGUMENT),
])
def test_adaln_host_validation(lib, kw, status):
    a = _adaln_args(**kw)
    assert lib.tt_adaln_modulate(ctypes.byref(a), 4096, 1 << 30, None) == status


def test_adaln_workspace(lib):
    a = _adaln_args(batch=8, mlp_width=256)
    assert lib.tt_adaln_workspace_bytes(ctypes.byref(a)) == 256 + 2 * 4 * 8 * 256
    assert lib.tt_adaln_modulate(ctypes.byref(a), 4096, 100, None) == B.TT_ERR_WORKSPACE_TOO_SMALL


@pytest.mark.parametrize("ptrs,batch,S", [
    ((None, 0x1000), 2, 16),        # no mask
    ((0x1000, None), 2, 16),        # no output
    ((0x1000, 0x2000), 0, 16),      # empty batch
    ((0x1000, 0x2000), 2, 0),       # empty block
])
def test_block_tau_host_validation(lib, ptrs, batch, S):
    # rejected on the host before any launch (the pointers are never dereferenced)
    assert lib.tt_block_tau(ptrs[0], batch, S, ptrs[1], None, None) == 1   # TT_ERR_INVALID_ARGUMENT


def test_kv_append_host_validation(lib):
    a = B.KvAppendArgs()
    a.batch, a.block_size, a.num_kv_heads, a.head_dim, a.dtype = 2, 16, 2, 128, B.TT_BF16
    for name in ("k_new", "v_new", "k_ctx", "v_ctx", "page_table", "ctx_lens", "free_pages", "free_count"):
        setattr(a, name, 0x1000)
    a.page_size, a.max_pages_per_seq, a.num_pages = 256, 8, 16
    ws = ctypes.c_void_p(0x2000)
    assert lib.tt_kv_append_workspace_bytes(ctypes.byref(a)) == 256
    a.free_count = None
    assert lib.tt_kv_append(ctypes.byref(a), ws, 256, None) == B.TT_ERR_INVALID_ARGUMENT
    a.free_count = 0x1000
    a.head_dim = 4                                   # 8 bytes per row: not a whole 16-byte vector
    assert lib.tt_kv_append(ctypes.byref(a), ws, 256, None) == B.TT_ERR_UNSUPPORTED
    a.head_dim = 128
    a.k_ctx = 0x1008                                 # misaligned pool
    assert lib.tt_kv_append(ctypes.byref(a), ws, 256, None) == B.TT_ERR_UNSUPPORTED
    a.k_ctx = 0x1000
    assert lib.tt_kv_append(ctypes.byref(a), ws, 64, None) == B.TT_ERR_WORKSPACE_TOO_SMALL


def test_unmask_sampler_fields_validated(lib):
    from denoiser_attention_b200 import binding as Bd
    a = Bd.UnmaskArgs()
    a.batch, a.block_size, a.vocab, a.dtype = 2, 16, 1024, Bd.TT_F32
    for name in ("logits", "tokens", "is_masked", "n_committed", "n_masked"):
        setattr(a, name, 0x1000)
    a.gamma, a.inv_temperature = 0.8, 1.0
    assert lib.tt_unmask_workspace_bytes(ctypes.byref(a)) > 0          # default: confidence sampler
    a.sampler = 7
    assert lib.tt_unmask_workspace_bytes(ctypes.byref(a)) == 0
    a.sampler, a.keep_masked = Bd.TT_SAMPLER_PREDICT_NOISE, -1
    assert lib.tt_unmask_workspace_bytes(ctypes.byref(a)) == 0
    a.keep_masked = 4
    assert lib.tt_unmask_workspace_bytes(ctypes.byref(a)) > 0


def test_lmhead_host_validation(lib):
    from denoiser_attention_b200 import binding as Bd
    a = Bd.LmheadUnmaskArgs()
    a.batch, a.block_size, a.hidden, a.vocab, a.dtype = 2, 16, 256, 4096, Bd.TT_BF16
    for name in ("x", "w", "tokens", "is_masked", "n_committed", "n_masked"):
        setattr(a, name, 0x1000)
    a.gamma, a.inv_temperature = 0.8, 1.0
    assert lib.tt_lmhead_unmask_workspace_bytes(ctypes.byref(a)) > 256
    ws = ctypes.c_void_p(0x2000)
    for field, bad, status in (("hidden", 100, Bd.TT_ERR_UNSUPPORTED), ("vocab", 1000, Bd.TT_ERR_UNSUPPORTED),
                               ("dtype", Bd.TT_F32, Bd.TT_ERR_UNSUPPORTED), ("x", None, Bd.TT_ERR_INVALID_ARGUMENT),
                               ("inv_temperature", 0.0, Bd.TT_ERR_INVALID_ARGUMENT),
                               ("sampler", 5, Bd.TT_ERR_INVALID_ARGUMENT)):
        good = getattr(a, field)
        setattr(a, field, bad)
        assert lib.tt_lmhead_unmask_step(ctypes.byref(a), ws, 1 << 20, None) == status, field
        setattr(a, field, good)
    assert lib.tt_lmhead_unmask_step(ctypes.byref(a), ws, 64, None) == Bd.TT_ERR_WORKSPACE_TOO_SMALL


def test_linear_schedule_keep_is_the_golden_table(lib):
    # the library's schedule (a host function) against the hand-derived table
    import json
    cases = json.load(open(os.path.join(ROOT, "tests", "golden", "noise_schedule_linear.json")))["cases"]
    for c in cases:
        got = [lib.tt_linear_schedule_keep(c["S"], c["T"], r) for r in range(1, c["T"] + 1)]
        assert got == c["keep"], c
    for S, T, r in ((0, 4, 1), (16, 0, 1), (16, 4, 0), (16, 4, 5)):
        assert lib.tt_linear_schedule_keep(S, T, r) == -1


def test_noise_schedule_fields_validated(lib):
    from denoiser_attention_b200 import binding as Bd
    a = Bd.UnmaskArgs()
    a.batch, a.block_size, a.vocab, a.dtype = 2, 16, 1024, Bd.TT_F32
    for name in ("logits", "tokens", "is_masked", "n_committed", "n_masked"):
        setattr(a, name, 0x1000)
    a.gamma, a.inv_temperature = 0.8, 1.0
    a.sampler, a.keep_masked = Bd.TT_SAMPLER_PREDICT_NOISE, -1      # ignored once a schedule is given
    for steps, step, ok in ((6, 1, True), (6, 6, True), (6, 0, False), (6, 7, False), (-1, 1, False)):
        a.noise_steps, a.noise_step = steps, step
        assert (lib.tt_unmask_workspace_bytes(ctypes.byref(a)) > 0) == ok, (steps, step)
    m = Bd.LmheadUnmaskArgs()
    m.batch, m.block_size, m.hidden, m.vocab, m.dtype = 2, 16, 256, 4096, Bd.TT_BF16
    for name in ("x", "w", "tokens", "is_masked", "n_committed", "n_masked"):
        setattr(m, name, 0x1000)
    m.gamma, m.inv_temperature = 0.8, 1.0
    m.sampler, m.keep_masked, m.noise_steps, m.noise_step = Bd.TT_SAMPLER_PREDICT_NOISE, -1, 16, 17
    assert lib.tt_lmhead_unmask_workspace_bytes(ctypes.byref(m)) == 0
    m.noise_step = 16
    assert lib.tt_lmhead_unmask_workspace_bytes(ctypes.byref(m)) > 0


def test_sizes_beyond_32_bit_rows_rejected(lib):
    # batch * block_size must fit the kernels' 32-bit row index; rows * vocab their 64-bit cuts
    from denoiser_attention_b200 import binding as Bd
    a = Bd.UnmaskArgs()
    a.dtype, a.gamma, a.inv_temperature = Bd.TT_F32, 0.8, 1.0
    for name in ("logits", "tokens", "is_masked", "n_committed", "n_masked"):
        setattr(a, name, 0x1000)
    a.batch, a.block_size, a.vocab = 1 << 22, 1024, 4                  # 2^32 rows
    assert lib.tt_unmask_step(ctypes.byref(a), ctypes.c_void_p(0x2000), 1 << 40, None) == Bd.TT_ERR_UNSUPPORTED
    assert lib.tt_unmask_step_noalloc(ctypes.byref(a), None) == Bd.TT_ERR_UNSUPPORTED
    a.batch, a.block_size, a.vocab = 1 << 14, 1024, 1 << 20            # 2^44 logits
    assert lib.tt_unmask_workspace_bytes(ctypes.byref(a)) == 0
    m = Bd.LmheadUnmaskArgs()
    m.batch, m.block_size, m.hidden, m.vocab, m.dtype = 1 << 22, 1024, 256, 4096, Bd.TT_BF16
    for name in ("x", "w", "tokens", "is_masked", "n_committed", "n_masked"):
        setattr(m, name, 0x1000)
    m.gamma, m.inv_temperature = 0.8, 1.0
    assert lib.tt_lmhead_unmask_workspace_bytes(ctypes.byref(m)) == 0
    t = _attn_args(batch=1 << 22, block_size=1024)
    assert lib.tt_denoise_attn_workspace_bytes(ctypes.byref(t)) == 0


def test_probe_bounded_wait_host_validation(lib):
    ws = ctypes.c_void_p(0x2000)
    assert lib.tt_probe_bounded_wait(None, 100, None) == B.TT_ERR_INVALID_ARGUMENT
    assert lib.tt_probe_bounded_wait(ws, 0, None) == B.TT_ERR_INVALID_ARGUMENT
    assert lib.tt_probe_bounded_wait(ws, 1000001, None) == B.TT_ERR_INVALID_ARGUMENT
