"""ctypes binding of libtt_denoise.so: argument marshalling only.

Every entry point of include/tt_denoise.h is exposed under the same name. The torch-facing
wrappers take CUDA tensors, fill the C argument struct with their device pointers and sizes,
and call the library on torch's current stream; all arithmetic runs in the library's kernels.
There is no fallback: if the shared library is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libtt_denoise.so")

TT_OK = 0
TT_ERR_INVALID_ARGUMENT = 1
TT_ERR_UNSUPPORTED = 2
TT_ERR_WORKSPACE_TOO_SMALL = 3
TT_ERR_CUDA = 4
TT_ERR_DEVICE = 5
TT_ERR_DEVICE_TIMEOUT = 6

TT_F32 = 0
TT_BF16 = 1

TT_SAMPLER_CONFIDENCE = 0
TT_SAMPLER_PREDICT_NOISE = 1

TT_ADALN_COND = 0
TT_ADALN_NORM_MODULATE = 1
TT_ADALN_GATED_RESIDUAL = 2
TT_ADALN_NORM_MODULATE_RESIDUAL = 3

EXPORTED = [
    "tt_status_string", "tt_version",
    "tt_denoise_attn_workspace_bytes", "tt_denoise_attn",
    "tt_adaln_workspace_bytes", "tt_adaln_modulate",
    "tt_unmask_workspace_bytes", "tt_unmask_step", "tt_unmask_step_noalloc", "tt_block_tau",
    "tt_kv_append_workspace_bytes", "tt_kv_append",
    "tt_lmhead_unmask_workspace_bytes", "tt_lmhead_unmask_step",
    "tt_linear_schedule_keep", "tt_probe_bounded_wait",
    "tt_get_device_error",
]

TT_DETAIL_WAIT_PROBE = 0x1FF

_vp = ctypes.c_void_p
_i32 = ctypes.c_int32
_f32 = ctypes.c_float


class AttnArgs(ctypes.Structure):
    _fields_ = [
        ("batch", _i32), ("block_size", _i32), ("num_q_heads", _i32), ("num_kv_heads", _i32),
        ("head_dim", _i32), ("dtype", _i32), ("softmax_scale", _f32),
        ("q", _vp), ("k_blk", _vp), ("v_blk", _vp), ("k_ctx", _vp), ("v_ctx", _vp),
        ("ctx_lens", _vp), ("page_table", _vp),
        ("page_size", _i32), ("max_pages_per_seq", _i32), ("num_pages", _i32), ("ctx_stride", _i32),
        ("out", _vp), ("lse", _vp), ("skip_if", _vp),
    ]


class AdalnArgs(ctypes.Structure):
    _fields_ = [
        ("op", _i32), ("batch", _i32), ("block_size", _i32), ("hidden", _i32), ("freq_dim", _i32),
        ("mlp_width", _i32), ("dtype", _i32), ("eps", _f32),
        ("tau", _vp), ("w1", _vp), ("b1", _vp), ("w2", _vp), ("b2", _vp), ("w3", _vp), ("b3", _vp),
        ("layer_emb", _vp), ("mod", _vp), ("h", _vp), ("norm_w", _vp), ("f", _vp), ("out", _vp),
        ("skip_if", _vp), ("out2", _vp),
    ]


class UnmaskArgs(ctypes.Structure):
    _fields_ = [
        ("batch", _i32), ("block_size", _i32), ("vocab", _i32), ("dtype", _i32), ("logits", _vp),
        ("gamma", _f32), ("inv_temperature", _f32), ("mask_token_id", _i32), ("exclude_mask_token", _i32),
        ("remaining_steps", _i32), ("tokens", _vp), ("is_masked", _vp), ("conf", _vp), ("argmax", _vp),
        ("n_committed", _vp), ("n_masked", _vp), ("sampler", _i32), ("keep_masked", _i32),
        ("noise_steps", _i32), ("noise_step", _i32), ("skip_if", _vp), ("all_done", _vp),
    ]


class KvAppendArgs(ctypes.Structure):
    _fields_ = [
        ("batch", _i32), ("block_size", _i32), ("num_kv_heads", _i32), ("head_dim", _i32), ("dtype", _i32),
        ("k_new", _vp), ("v_new", _vp), ("k_ctx", _vp), ("v_ctx", _vp), ("page_table", _vp), ("ctx_lens", _vp),
        ("free_pages", _vp), ("free_count", _vp), ("page_size", _i32), ("max_pages_per_seq", _i32),
        ("num_pages", _i32),
    ]


class LmheadUnmaskArgs(ctypes.Structure):
    _fields_ = [
        ("batch", _i32), ("block_size", _i32), ("hidden", _i32), ("vocab", _i32), ("dtype", _i32),
        ("x", _vp), ("w", _vp), ("gamma", _f32), ("inv_temperature", _f32), ("mask_token_id", _i32),
        ("exclude_mask_token", _i32), ("remaining_steps", _i32), ("tokens", _vp), ("is_masked", _vp),
        ("conf", _vp), ("argmax", _vp), ("n_committed", _vp), ("n_masked", _vp), ("sampler", _i32),
        ("keep_masked", _i32), ("noise_steps", _i32), ("noise_step", _i32), ("skip_if", _vp), ("all_done", _vp),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libtt_denoise.so (raises if it is missing: there is no fallback path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with python -m denoiser_attention_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        L.tt_status_string.restype = ctypes.c_char_p
        L.tt_status_string.argtypes = [ctypes.c_int]
        L.tt_version.restype = ctypes.c_int
        L.tt_denoise_attn_workspace_bytes.restype = ctypes.c_size_t
        L.tt_denoise_attn_workspace_bytes.argtypes = [ctypes.POINTER(AttnArgs)]
        L.tt_denoise_attn.restype = ctypes.c_int
        L.tt_denoise_attn.argtypes = [ctypes.POINTER(AttnArgs), _vp, ctypes.c_size_t, _vp]
        L.tt_adaln_workspace_bytes.restype = ctypes.c_size_t
        L.tt_adaln_workspace_bytes.argtypes = [ctypes.POINTER(AdalnArgs)]
        L.tt_adaln_modulate.restype = ctypes.c_int
        L.tt_adaln_modulate.argtypes = [ctypes.POINTER(AdalnArgs), _vp, ctypes.c_size_t, _vp]
        L.tt_unmask_workspace_bytes.restype = ctypes.c_size_t
        L.tt_unmask_workspace_bytes.argtypes = [ctypes.POINTER(UnmaskArgs)]
        L.tt_unmask_step.restype = ctypes.c_int
        L.tt_unmask_step.argtypes = [ctypes.POINTER(UnmaskArgs), _vp, ctypes.c_size_t, _vp]
        L.tt_unmask_step_noalloc.restype = ctypes.c_int
        L.tt_block_tau.restype = ctypes.c_int
        L.tt_lmhead_unmask_workspace_bytes.restype = ctypes.c_size_t
        L.tt_lmhead_unmask_workspace_bytes.argtypes = [ctypes.POINTER(LmheadUnmaskArgs)]
        L.tt_lmhead_unmask_step.restype = ctypes.c_int
        L.tt_lmhead_unmask_step.argtypes = [ctypes.POINTER(LmheadUnmaskArgs), _vp, ctypes.c_size_t, _vp]
        L.tt_kv_append_workspace_bytes.restype = ctypes.c_size_t
        L.tt_kv_append_workspace_bytes.argtypes = [ctypes.POINTER(KvAppendArgs)]
        L.tt_kv_append.restype = ctypes.c_int
        L.tt_kv_append.argtypes = [ctypes.POINTER(KvAppendArgs), _vp, ctypes.c_size_t, _vp]
        L.tt_block_tau.argtypes = [_vp, ctypes.c_int32, ctypes.c_int32, _vp, _vp, _vp]
        L.tt_unmask_step_noalloc.argtypes = [ctypes.POINTER(UnmaskArgs), _vp]
        L.tt_linear_schedule_keep.restype = ctypes.c_int32
        L.tt_linear_schedule_keep.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32]
        L.tt_probe_bounded_wait.restype = ctypes.c_int
        L.tt_probe_bounded_wait.argtypes = [_vp, ctypes.c_uint32, _vp]
        L.tt_get_device_error.restype = ctypes.c_int
        L.tt_get_device_error.argtypes = [_vp, _vp, ctypes.POINTER(ctypes.c_uint32)]
        _lib = L
    return _lib


class TTError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {lib().tt_status_string(status).decode()}")


def _check(status: int, what: str):
    if status != TT_OK:
        raise TTError(status, what)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return TT_BF16
    if dt == torch.float32:
        return TT_F32
    raise ValueError(f"unsupported dtype {dt}")


def _stream(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def status_string(status: int) -> str:
    return lib().tt_status_string(status).decode()


# ------------------------------------------------------------------------------------------ attn
def attn_args(q, k_blk, v_blk, k_ctx, v_ctx, ctx_lens, out, page_table=None, page_size=0,
              ctx_stride=0, softmax_scale=1.0, lse=None, skip_if=None) -> AttnArgs:
    B, S, Hq, d = q.shape
    Hkv = k_blk.shape[2]
    a = AttnArgs()
    a.batch, a.block_size, a.num_q_heads, a.num_kv_heads, a.head_dim = B, S, Hq, Hkv, d
    a.dtype = _dtype_code(q.dtype)
    a.softmax_scale = float(softmax_scale)
    a.q, a.k_blk, a.v_blk = _ptr(q), _ptr(k_blk), _ptr(v_blk)
    a.k_ctx, a.v_ctx = _ptr(k_ctx), _ptr(v_ctx)
    a.ctx_lens = _ptr(ctx_lens)
    a.page_table = _ptr(page_table)
    if page_table is not None:
        a.page_size = int(page_size)
        a.max_pages_per_seq = int(page_table.shape[1])
        a.num_pages = int(k_ctx.shape[0])
    else:
        a.ctx_stride = int(ctx_stride) if ctx_stride else int(k_ctx.shape[1])
    a.out = _ptr(out)
    a.lse = _ptr(lse)
    a.skip_if = _ptr(skip_if)
    return a


def tt_denoise_attn_workspace_bytes(args: AttnArgs) -> int:
    return int(lib().tt_denoise_attn_workspace_bytes(ctypes.byref(args)))


def tt_denoise_attn(args: AttnArgs, workspace: torch.Tensor, stream=None) -> None:
    _check(lib().tt_denoise_attn(ctypes.byref(args), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                 _stream(stream)), "tt_denoise_attn")


# ------------------------------------------------------------------------------------------ adaLN
def adaln_args(op: int, *, batch: int, hidden: int, block_size: int = 0, freq_dim: int = 256,
               mlp_width: int = 256, dtype=torch.float32, eps: float = 1e-5, tau=None, w1=None, b1=None,
               w2=None, b2=None, w3=None, b3=None, layer_emb=None, mod=None, h=None, norm_w=None, f=None,
               out=None, skip_if=None, out2=None) -> AdalnArgs:
    a = AdalnArgs()
    a.op, a.batch, a.block_size, a.hidden = op, batch, block_size, hidden
    a.freq_dim, a.mlp_width, a.dtype, a.eps = freq_dim, mlp_width, _dtype_code(dtype), float(eps)
    a.tau, a.w1, a.b1, a.w2, a.b2 = _ptr(tau), _ptr(w1), _ptr(b1), _ptr(w2), _ptr(b2)
    a.w3, a.b3, a.layer_emb, a.mod = _ptr(w3), _ptr(b3), _ptr(layer_emb), _ptr(mod)
    a.h, a.norm_w, a.f, a.out = _ptr(h), _ptr(norm_w), _ptr(f), _ptr(out)
    a.skip_if, a.out2 = _ptr(skip_if), _ptr(out2)
    return a


def tt_adaln_workspace_bytes(args: AdalnArgs) -> int:
    return int(lib().tt_adaln_workspace_bytes(ctypes.byref(args)))


def tt_adaln_modulate(args: AdalnArgs, workspace: torch.Tensor, stream=None) -> None:
    _check(lib().tt_adaln_modulate(ctypes.byref(args), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream)),
           "tt_adaln_modulate")


# ------------------------------------------------------------------------------------------ unmask
def unmask_args(logits, tokens, is_masked, n_committed, n_masked, *, gamma: float, inv_temperature: float = 1.0,
                mask_token_id: int = 3, exclude_mask_token: bool = False, remaining_steps: int = 0,
                conf=None, argmax=None, keep_masked: Optional[int] = None,
                noise_schedule: Optional[tuple] = None, skip_if=None, all_done=None) -> UnmaskArgs:
    """keep_masked=None and noise_schedule=None: the confidence-threshold sampler; keep_masked=k:
    the predict-and-noise sampler keeping k positions masked; noise_schedule=(T, r): the
    predict-and-noise sampler at step r of T of the linear schedule (the library derives k)."""
    B, S, V = logits.shape
    a = UnmaskArgs()
    a.batch, a.block_size, a.vocab, a.dtype = B, S, V, _dtype_code(logits.dtype)
    a.logits = _ptr(logits)
    a.gamma, a.inv_temperature = float(gamma), float(inv_temperature)
    a.mask_token_id, a.exclude_mask_token, a.remaining_steps = int(mask_token_id), int(bool(exclude_mask_token)), int(remaining_steps)
    a.tokens, a.is_masked = _ptr(tokens), _ptr(is_masked)
    a.conf, a.argmax = _ptr(conf), _ptr(argmax)
    a.n_committed, a.n_masked = _ptr(n_committed), _ptr(n_masked)
    _set_sampler(a, keep_masked, noise_schedule)
    a.skip_if, a.all_done = _ptr(skip_if), _ptr(all_done)
    return a


def _set_sampler(a, keep_masked, noise_schedule):
    if keep_masked is not None and noise_schedule is not None:
        raise ValueError("give keep_masked or noise_schedule, not both")
    a.sampler, a.keep_masked, a.noise_steps, a.noise_step = TT_SAMPLER_CONFIDENCE, 0, 0, 0
    if keep_masked is not None:
        a.sampler, a.keep_masked = TT_SAMPLER_PREDICT_NOISE, int(keep_masked)
    elif noise_schedule is not None:
        a.sampler = TT_SAMPLER_PREDICT_NOISE
        a.noise_steps, a.noise_step = int(noise_schedule[0]), int(noise_schedule[1])


def tt_linear_schedule_keep(block_size: int, steps: int, step: int) -> int:
    """Positions left masked after step `step` of `steps` (linear schedule); -1 if invalid."""
    return int(lib().tt_linear_schedule_keep(int(block_size), int(steps), int(step)))


def tt_probe_bounded_wait(workspace: torch.Tensor, limit_us: int, stream=None) -> None:
    """Runs the library's bounded device wait on a barrier nothing arrives on (diagnostic)."""
    _check(lib().tt_probe_bounded_wait(_ptr(workspace), int(limit_us), _stream(stream)), "tt_probe_bounded_wait")


def tt_unmask_workspace_bytes(args: UnmaskArgs) -> int:
    return int(lib().tt_unmask_workspace_bytes(ctypes.byref(args)))


def tt_unmask_step(args: UnmaskArgs, workspace: torch.Tensor, stream=None) -> None:
    _check(lib().tt_unmask_step(ctypes.byref(args), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                _stream(stream)), "tt_unmask_step")


def tt_unmask_step_noalloc(args: UnmaskArgs, stream=None) -> None:
    """tt_unmask_step with the library's static scratch: no workspace, nothing allocated."""
    _check(lib().tt_unmask_step_noalloc(ctypes.byref(args), _stream(stream)), "tt_unmask_step_noalloc")


def tt_block_tau(is_masked: torch.Tensor, tau: torch.Tensor, stream=None, skip_if=None) -> None:
    """tau[b] = masked positions of sequence b / S, on the device (nothing when *skip_if != 0)."""
    if is_masked.dtype != torch.uint8 or tau.dtype != torch.float32:
        raise ValueError("is_masked must be uint8 and tau float32")
    Bn, S = is_masked.shape
    _check(lib().tt_block_tau(_ptr(is_masked), Bn, S, _ptr(tau), _ptr(skip_if), _stream(stream)), "tt_block_tau")


# ------------------------------------------------------------------------------- LM head + unmask
def lmhead_unmask_args(x, w, tokens, is_masked, n_committed, n_masked, *, gamma: float,
                       inv_temperature: float = 1.0, mask_token_id: int = 3, exclude_mask_token: bool = False,
                       remaining_steps: int = 0, conf=None, argmax=None,
                       keep_masked: Optional[int] = None, noise_schedule: Optional[tuple] = None,
                       skip_if=None, all_done=None) -> LmheadUnmaskArgs:
    B, S, D = x.shape
    a = LmheadUnmaskArgs()
    a.batch, a.block_size, a.hidden, a.vocab, a.dtype = B, S, D, int(w.shape[0]), _dtype_code(x.dtype)
    a.x, a.w = _ptr(x), _ptr(w)
    a.gamma, a.inv_temperature = float(gamma), float(inv_temperature)
    a.mask_token_id, a.exclude_mask_token, a.remaining_steps = int(mask_token_id), int(bool(exclude_mask_token)), int(remaining_steps)
    a.tokens, a.is_masked, a.conf, a.argmax = _ptr(tokens), _ptr(is_masked), _ptr(conf), _ptr(argmax)
    a.n_committed, a.n_masked = _ptr(n_committed), _ptr(n_masked)
    _set_sampler(a, keep_masked, noise_schedule)
    a.skip_if, a.all_done = _ptr(skip_if), _ptr(all_done)
    return a


def tt_lmhead_unmask_workspace_bytes(args: LmheadUnmaskArgs) -> int:
    return int(lib().tt_lmhead_unmask_workspace_bytes(ctypes.byref(args)))


def tt_lmhead_unmask_step(args: LmheadUnmaskArgs, workspace: torch.Tensor, stream=None) -> None:
    _check(lib().tt_lmhead_unmask_step(ctypes.byref(args), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(), _stream(stream)),
           "tt_lmhead_unmask_step")


# ------------------------------------------------------------------------------------ block commit
def kv_append_args(k_new, v_new, k_ctx, v_ctx, page_table, ctx_lens, free_pages, free_count) -> KvAppendArgs:
    B, S, Hkv, d = k_new.shape
    a = KvAppendArgs()
    a.batch, a.block_size, a.num_kv_heads, a.head_dim = B, S, Hkv, d
    a.dtype = _dtype_code(k_new.dtype)
    a.k_new, a.v_new, a.k_ctx, a.v_ctx = _ptr(k_new), _ptr(v_new), _ptr(k_ctx), _ptr(v_ctx)
    a.page_table, a.ctx_lens = _ptr(page_table), _ptr(ctx_lens)
    a.free_pages, a.free_count = _ptr(free_pages), _ptr(free_count)
    a.num_pages, a.page_size = int(k_ctx.shape[0]), int(k_ctx.shape[1])
    a.max_pages_per_seq = int(page_table.shape[1])
    return a


def tt_kv_append_workspace_bytes(args: KvAppendArgs) -> int:
    return int(lib().tt_kv_append_workspace_bytes(ctypes.byref(args)))


def tt_kv_append(args: KvAppendArgs, workspace: torch.Tensor, stream=None) -> None:
    _check(lib().tt_kv_append(ctypes.byref(args), _ptr(workspace), workspace.numel() * workspace.element_size(),
                              _stream(stream)), "tt_kv_append")


def tt_get_device_error(workspace: torch.Tensor, stream=None):
    detail = ctypes.c_uint32(0)
    st = lib().tt_get_device_error(_ptr(workspace), _stream(stream), ctypes.byref(detail))
    return st, detail.value


def new_workspace(nbytes: int, device=None) -> torch.Tensor:
    """Zero-filled device workspace of at least nbytes (256-byte granularity)."""
    n = max(256, (int(nbytes) + 255) // 256 * 256)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")
