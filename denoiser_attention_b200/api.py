"""Torch-facing API of one TwoTower denoiser refinement step (device memory and streams only).

Each function allocates its outputs with torch and calls the matching C-ABI entry point of
libtt_denoise.so through `binding`; every step of the computation runs in the library's CUDA
kernels. Workspaces are cached per (device, size) and zero-filled once, as the ABI requires.

    denoise_attention    Eq. (1), layer-aligned denoiser attention       (tt_denoise_attn)
    adaln_cond           adaLN-single: tau -> (shift, scale, gate)       (tt_adaln_modulate)
    adaln_norm_modulate  modulated RMSNorm prologue                      (tt_adaln_modulate)
    adaln_gated_residual h + gate * f                                    (tt_adaln_modulate)
    unmask_step          ConfidenceSample, Algorithm 2 (its ConfidenceSample step)            (tt_unmask_step)
                         or the predict-and-noise sampler (keep_masked)
    RefinementStep       the whole step a2..a7 (three concurrent branches), device buffers
    HostStep             the same step from pinned host buffers (copies included)
    block_tau            tau_b = masked fraction of sequence b, on the device  (tt_block_tau)
    append_block_kv      block commit: the block's context KV into the paged cache (tt_kv_append)
    lmhead_unmask_step   the unmask step from hidden states, LM head fused (tt_lmhead_unmask_step)
    RefinementLoop       Algorithm 2: T steps of one block, tau from the mask on the device,
                         capturable as one CUDA graph (no host round trip between steps)
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional, Tuple

import torch

from . import binding as B

_WS: Dict[Tuple, torch.Tensor] = {}


def workspace(nbytes: int, device: torch.device, tag: str, signature: Tuple = ()) -> torch.Tensor:
    """A cached zero-initialised workspace of at least nbytes for (device, tag, signature).

    The layout of a workspace (where its merge tickets live) depends on the argument sizes, and
    the kernels only restore the tickets of their own layout to zero, so a workspace is reused
    only by calls with the same signature (the sizes that determine the layout)."""
    dev = torch.device(device)
    key = (dev.index if dev.index is not None else torch.cuda.current_device(), tag, tuple(signature))
    ws = _WS.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = B.new_workspace(nbytes, device=dev)
        _WS[key] = ws
    return ws


def check_device_error(ws: torch.Tensor):
    st, detail = B.tt_get_device_error(ws)
    if st != B.TT_OK:
        raise B.TTError(st, f"device-side error (detail {detail:#x})")


def check_device_errors(device=None):
    """Reads and clears the device error word of every cached workspace on `device` (all devices
    when None) and raises TTError for the first one set. The kernels report device-side errors
    (a page id outside the pool, a context longer than its table, a bounded wait that gave up)
    only through these words, so a caller polls them, e.g. once per refinement loop. It
    synchronises the streams it reads on: call it outside CUDA-graph capture."""
    want = None if device is None else torch.device(device)
    for (dev_index, tag, _), ws in list(_WS.items()):
        if want is not None and want.index is not None and want.index != dev_index:
            continue
        st, detail = B.tt_get_device_error(ws)
        if st != B.TT_OK:
            raise B.TTError(st, f"device-side error in the {tag} workspace (detail {detail:#x})")


def denoise_attention(q, k_blk, v_blk, k_ctx, v_ctx, ctx_lens, page_table=None, page_size: int = 0,
                      ctx_stride: int = 0, softmax_scale: float = 1.0, return_lse: bool = False,
                      out: Optional[torch.Tensor] = None, ws_tag: str = "attn", skip_if=None):
    out = torch.empty_like(q) if out is None else out
    lse = None
    if return_lse:
        Bn, S, Hq, _ = q.shape
        lse = torch.empty((Bn, Hq, S), dtype=torch.float32, device=q.device)
    args = B.attn_args(q, k_blk, v_blk, k_ctx, v_ctx, ctx_lens, out, page_table=page_table, page_size=page_size,
                       ctx_stride=ctx_stride, softmax_scale=softmax_scale, lse=lse, skip_if=skip_if)
    nbytes = B.tt_denoise_attn_workspace_bytes(args)
    if nbytes == 0:
        # invalid or unsupported arguments: let the launch report the exact status
        nbytes = 256
    ws = workspace(nbytes, q.device, ws_tag, (tuple(q.shape), k_blk.shape[2], q.dtype))
    B.tt_denoise_attn(args, ws)
    return (out, lse) if return_lse else out


def adaln_cond(tau, w1, b1, w2, b2, w3, b3, layer_emb, ws_tag: str = "adaln", skip_if=None):
    Bn = tau.shape[0]
    D = layer_emb.shape[1]
    mod = torch.empty((Bn, 3, D), dtype=torch.float32, device=tau.device)
    args = B.adaln_args(B.TT_ADALN_COND, batch=Bn, hidden=D, freq_dim=w1.shape[1], mlp_width=w1.shape[0],
                        tau=tau, w1=w1, b1=b1, w2=w2, b2=b2, w3=w3, b3=b3, layer_emb=layer_emb, mod=mod,
                        skip_if=skip_if)
    ws = workspace(max(256, B.tt_adaln_workspace_bytes(args)), tau.device, ws_tag)
    B.tt_adaln_modulate(args, ws)
    return mod


def adaln_norm_modulate(h, norm_w, mod, eps: float = 1e-5, out=None, ws_tag: str = "adaln", skip_if=None):
    Bn, S, D = h.shape
    out = torch.empty_like(h) if out is None else out
    args = B.adaln_args(B.TT_ADALN_NORM_MODULATE, batch=Bn, block_size=S, hidden=D, dtype=h.dtype, eps=eps,
                        h=h, norm_w=norm_w, mod=mod, out=out, skip_if=skip_if)
    ws = workspace(256, h.device, ws_tag)
    B.tt_adaln_modulate(args, ws)
    return out


def adaln_gated_residual(h, f, mod, out=None, ws_tag: str = "adaln", skip_if=None):
    Bn, S, D = h.shape
    out = torch.empty_like(h) if out is None else out
    args = B.adaln_args(B.TT_ADALN_GATED_RESIDUAL, batch=Bn, block_size=S, hidden=D, dtype=h.dtype, h=h, f=f,
                        mod=mod, out=out, skip_if=skip_if)
    ws = workspace(256, h.device, ws_tag)
    B.tt_adaln_modulate(args, ws)
    return out


def adaln_norm_modulate_residual(h, f, norm_w, mod, eps: float = 1e-5, out=None, out2=None, ws_tag: str = "adaln",
                                 skip_if=None):
    """(adaln_norm_modulate(h, norm_w, mod), adaln_gated_residual(h, f, mod)) in one launch that
    reads h once."""
    Bn, S, D = h.shape
    out = torch.empty_like(h) if out is None else out
    out2 = torch.empty_like(h) if out2 is None else out2
    args = B.adaln_args(B.TT_ADALN_NORM_MODULATE_RESIDUAL, batch=Bn, block_size=S, hidden=D, dtype=h.dtype,
                        eps=eps, h=h, norm_w=norm_w, f=f, mod=mod, out=out, out2=out2, skip_if=skip_if)
    ws = workspace(256, h.device, ws_tag)
    B.tt_adaln_modulate(args, ws)
    return out, out2


def unmask_step(logits, tokens, is_masked, *, gamma: float, inv_temperature: float = 1.0, mask_token_id: int = 3,
                exclude_mask_token: bool = False, remaining_steps: int = 0, want_conf: bool = True,
                ws_tag: str = "unmask", n_committed: Optional[torch.Tensor] = None,
                n_masked: Optional[torch.Tensor] = None, keep_masked: Optional[int] = None,
                noise_schedule: Optional[Tuple[int, int]] = None, skip_if=None, all_done=None):
    """Updates tokens / is_masked in place; returns (n_committed, n_masked, conf, argmax).
    With keep_masked and noise_schedule both None this is the confidence-threshold sampler.
    keep_masked=k runs the predict-and-noise sampler, which commits all but k of the masked
    positions (the least confident stay masked); noise_schedule=(T, r) runs it at step r of T of
    the linear schedule, the library deriving k (see linear_schedule_keep)."""
    Bn, S, V = logits.shape
    dev = logits.device
    if n_committed is None:
        n_committed = torch.empty(Bn, dtype=torch.int32, device=dev)
    if n_masked is None:
        n_masked = torch.empty(Bn, dtype=torch.int32, device=dev)
    conf = torch.empty((Bn, S), dtype=torch.float32, device=dev) if want_conf else None
    argmax = torch.empty((Bn, S), dtype=torch.int32, device=dev) if want_conf else None
    args = B.unmask_args(logits, tokens, is_masked, n_committed, n_masked, gamma=gamma,
                         inv_temperature=inv_temperature, mask_token_id=mask_token_id,
                         exclude_mask_token=exclude_mask_token, remaining_steps=remaining_steps, conf=conf,
                         argmax=argmax, keep_masked=keep_masked, noise_schedule=noise_schedule,
                         skip_if=skip_if, all_done=all_done)
    ws = workspace(max(256, B.tt_unmask_workspace_bytes(args)), dev, ws_tag, (tuple(logits.shape), logits.dtype))
    B.tt_unmask_step(args, ws)
    return n_committed, n_masked, conf, argmax


def lmhead_unmask_step(x, w, tokens, is_masked, *, gamma: float, inv_temperature: float = 1.0,
                       mask_token_id: int = 3, exclude_mask_token: bool = False, remaining_steps: int = 0,
                       want_conf: bool = True, keep_masked: Optional[int] = None,
                       noise_schedule: Optional[Tuple[int, int]] = None, ws_tag: str = "lmhead",
                       skip_if=None, all_done=None):
    """unmask_step from the final hidden states x [B][S][D] and the LM-head weight w [V][D] (bf16):
    the logits x w^T are reduced on the fly and never stored. Returns (n_committed, n_masked,
    conf, argmax) and updates tokens / is_masked in place."""
    Bn, S, _ = x.shape
    dev = x.device
    n_committed = torch.empty(Bn, dtype=torch.int32, device=dev)
    n_masked = torch.empty(Bn, dtype=torch.int32, device=dev)
    conf = torch.empty((Bn, S), dtype=torch.float32, device=dev) if want_conf else None
    argmax = torch.empty((Bn, S), dtype=torch.int32, device=dev) if want_conf else None
    args = B.lmhead_unmask_args(x, w, tokens, is_masked, n_committed, n_masked, gamma=gamma,
                                inv_temperature=inv_temperature, mask_token_id=mask_token_id,
                                exclude_mask_token=exclude_mask_token, remaining_steps=remaining_steps, conf=conf,
                                argmax=argmax, keep_masked=keep_masked, noise_schedule=noise_schedule,
                                skip_if=skip_if, all_done=all_done)
    ws = workspace(max(256, B.tt_lmhead_unmask_workspace_bytes(args)), dev, ws_tag,
                   (tuple(x.shape), int(w.shape[0])))
    B.tt_lmhead_unmask_step(args, ws)
    return n_committed, n_masked, conf, argmax


def linear_schedule_keep(block_size: int, steps: int, r: int) -> int:
    """Positions left masked after step r (1..T) under the linear schedule alpha_t = 1 - t
    (tt_linear_schedule_keep: the library computes it)."""
    k = B.tt_linear_schedule_keep(block_size, steps, r)
    if k < 0:
        raise ValueError("need block_size >= 1, steps >= 1 and 1 <= r <= steps")
    return k


@dataclasses.dataclass
class StepBuffers:
    """Device tensors of one refinement step (inputs and outputs)."""
    tau: torch.Tensor
    h: torch.Tensor
    f: torch.Tensor
    q: torch.Tensor
    k_blk: torch.Tensor
    v_blk: torch.Tensor
    k_ctx: torch.Tensor
    v_ctx: torch.Tensor
    ctx_lens: torch.Tensor
    page_table: Optional[torch.Tensor]
    logits: torch.Tensor
    tokens: torch.Tensor
    is_masked: torch.Tensor


class RefinementStep:
    """One denoiser refinement step of TwoTower decoding on one GPU.

    a2  mod = adaLN-single(tau)                 (tau = masked fraction: the time input of Algorithm 2)
    a3  y = modulated RMSNorm(h)                (prologue; y feeds the out-of-scope QKV projection)
    a4  O = Eq. (1) attention(q, [K_ctx; K_blk], [V_ctx; V_blk])
    a5  h' = h + gate * f                       (f: the mixer output after its out-projection)
    a6/a7  ConfidenceSample on the vocabulary logits (tokens / mask updated in place)
    The weights (adaLN MLP, per-layer embedding, norm weight) live on the device.

    The step has three independent branches: a2 -> a3 -> a5 (modulation), a4 (attention) and
    a6/a7 (unmask). schedule says how they are put on streams:
      "branches"          attention and unmask on two side streams forked from the caller's stream,
                          the modulation on the caller's stream: all three overlap on the device
      "attn_then_unmask"  attention, then unmask, on one side stream; the modulation alongside
      "unmask_then_attn"  the same with the unmask first
      "serial"            everything on the caller's stream (also concurrent=False)
    Side streams are joined back into the caller's stream before run() returns, so a CUDA graph
    captured around run() holds the same branches. Every output is allocated on the caller's
    stream before the fork. The outputs do not depend on the schedule.

    Device-side errors (a bad page id, a context longer than its table, a bounded wait inside a
    kernel that gave up after one second, e.g. on a GPU time-sliced with other work) are only
    recorded in the workspaces' error words: with check_errors=True every run() reads them after
    the join (it synchronises, so not under graph capture); otherwise call check_device_errors()
    yourself, e.g. once per RefinementLoop.
    """

    SCHEDULES = ("branches", "attn_then_unmask", "unmask_then_attn", "serial")

    # kernel launches per step: adaLN COND (3, one per MLP layer), RMSNorm prologue with the gated
    # residual, attention and its split-KV merge, unmask
    LAUNCHES = 7

    def __init__(self, weights: Dict[str, torch.Tensor], *, gamma: float, inv_temperature: float = 1.0,
                 mask_token_id: int = 3, page_size: int = 0, ctx_stride: int = 0, softmax_scale: float = 1.0,
                 eps: float = 1e-5, remaining_steps: int = 0, concurrent: bool = True,
                 schedule: str = "branches", check_errors: bool = False):
        self.w = weights
        self.gamma = gamma
        self.inv_temperature = inv_temperature
        self.mask_token_id = mask_token_id
        self.page_size = page_size
        self.ctx_stride = ctx_stride
        self.softmax_scale = softmax_scale
        self.eps = eps
        self.remaining_steps = remaining_steps
        if schedule not in self.SCHEDULES:
            raise ValueError(f"schedule must be one of {self.SCHEDULES}")
        self.schedule = schedule if concurrent else "serial"
        self.check_errors = check_errors
        self._streams = {}

    def _side(self, dev):
        key = dev.index if dev.index is not None else torch.cuda.current_device()
        if key not in self._streams:
            mk = lambda: torch.cuda.Event()
            self._streams[key] = (torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev), mk(), mk(), mk())
        return self._streams[key]

    def run(self, b: StepBuffers, out_attn: Optional[torch.Tensor] = None, events=None, skip_if=None,
            all_done=None):
        """Runs the step on the current stream. events: optional timing events recorded around
        the attention (0, 1) and the unmask (2, 3) launches, on the streams they run on, and, when
        8 are given, around the COND (4, 5) and the RMSNorm + gated-residual (6, 7) launches.
        skip_if / all_done: optional int32 device words of a multi-step loop's early exit (every
        kernel of the step does nothing when *skip_if != 0; the unmask sets *all_done = 1 once no
        sequence has a masked position left). all_done must not be the word skip_if points to:
        the unmask runs concurrently with the step's other kernels."""
        w = self.w
        dev = b.q.device
        main = torch.cuda.current_stream(dev)
        out_attn = torch.empty_like(b.q) if out_attn is None else out_attn
        Bn = b.q.shape[0]
        nc = torch.empty(Bn, dtype=torch.int32, device=dev)
        nm = torch.empty(Bn, dtype=torch.int32, device=dev)
        forked = self.schedule != "serial"
        if forked:
            s_a, s_b, fork, join_a, join_u = self._side(dev)
            fork.record(main)
            s_a.wait_event(fork)
            s_attn = s_a
            s_unm = s_b if self.schedule == "branches" else s_a
            if s_unm is not s_attn:
                s_unm.wait_event(fork)
        else:
            s_attn = s_unm = main

        def attention():
            with torch.cuda.stream(s_attn):
                if events is not None:
                    events[0].record(s_attn)
                denoise_attention(b.q, b.k_blk, b.v_blk, b.k_ctx, b.v_ctx, b.ctx_lens, page_table=b.page_table,
                                  page_size=self.page_size, ctx_stride=self.ctx_stride,
                                  softmax_scale=self.softmax_scale, out=out_attn, skip_if=skip_if)
                if events is not None:
                    events[1].record(s_attn)

        def unmask():
            with torch.cuda.stream(s_unm):
                if events is not None:
                    events[2].record(s_unm)
                unmask_step(b.logits, b.tokens, b.is_masked, gamma=self.gamma,
                            inv_temperature=self.inv_temperature, mask_token_id=self.mask_token_id,
                            remaining_steps=self.remaining_steps, want_conf=False, n_committed=nc, n_masked=nm,
                            skip_if=skip_if, all_done=all_done)
                if events is not None:
                    events[3].record(s_unm)

        if self.schedule == "unmask_then_attn":
            unmask()
            attention()
        else:
            attention()
            unmask()
        mark = (lambda i: events[i].record(main)) if events is not None and len(events) >= 8 else (lambda i: None)
        mark(4)
        mod = adaln_cond(b.tau, w["w1"], w["b1"], w["w2"], w["b2"], w["w3"], w["b3"], w["layer_emb"], skip_if=skip_if)
        mark(5)
        mark(6)
        y, h_new = adaln_norm_modulate_residual(b.h, b.f, w["norm_w"], mod, eps=self.eps, skip_if=skip_if)
        mark(7)
        if forked:
            join_a.record(s_attn)
            main.wait_event(join_a)
            if s_unm is not s_attn:
                join_u.record(s_unm)
                main.wait_event(join_u)
        if self.check_errors:
            check_device_errors(dev)
        return {"mod": mod, "y": y, "attn": out_attn, "h": h_new, "n_committed": nc, "n_masked": nm}


def block_tau(is_masked: torch.Tensor, out: Optional[torch.Tensor] = None, skip_if=None) -> torch.Tensor:
    """tau[b] = |{l : is_masked[b, l]}| / S on the device (the time input of Algorithm 2)."""
    tau = torch.empty(is_masked.shape[0], dtype=torch.float32, device=is_masked.device) if out is None else out
    B.tt_block_tau(is_masked, tau, skip_if=skip_if)
    return tau


def append_block_kv(k_new, v_new, k_ctx, v_ctx, page_table, ctx_lens, free_pages, free_count,
                    ws_tag: str = "kv_append") -> torch.Tensor:
    """Appends the committed block's context K/V [B][S][Hkv][d] after each sequence's context in the
    paged pool [num_pages][page_size][Hkv][d], taking pages from the free stack; page_table,
    ctx_lens and free_count are updated in place. Returns the workspace (its error word reports a
    sequence that could not be given pages)."""
    args = B.kv_append_args(k_new, v_new, k_ctx, v_ctx, page_table, ctx_lens, free_pages, free_count)
    ws = workspace(max(256, B.tt_kv_append_workspace_bytes(args)), k_new.device, ws_tag)
    B.tt_kv_append(args, ws)
    return ws


class RefinementLoop:
    """Algorithm 2 on the device: the T refinement steps of one block.

    for r = 1..T:  tau = masked fraction (tt_block_tau, on the device)
                   the RefinementStep with tau and step r's inputs
                   (ConfidenceSample updates the shared tokens / mask in place)
    Every step's inputs (q, K/V, logits, h, f) are the caller's, one StepBuffers per step; tokens
    and is_masked are shared by all steps, and each step's tau buffer is written by the loop.
    run() only enqueues work, so the whole loop can be captured in one CUDA graph and replayed
    with no host synchronisation between steps. The per-step outputs (attention, modulation,
    residual, commit counts) are returned for inspection.

    Early exit (early_exit=True): the block is complete as soon as no sequence has a masked
    position left, usually before step T. Two int32 device words alternate: step r reads word
    r % 2 as every kernel's skip_if and its unmask raises word (r + 1) % 2 once everything is
    committed (a skipped unmask raises it again, so the flag carries forward). The steps after
    completion then do nothing but launch: their outputs are left as they were. The words are
    cleared at the start of run() (stream-ordered, capturable). finished() reads, on the host,
    whether the block completed.
    """

    def __init__(self, step: RefinementStep, early_exit: bool = True):
        self.step = step
        self.early_exit = early_exit
        self.flags = None

    def run(self, steps: "list[StepBuffers]", tokens: torch.Tensor, is_masked: torch.Tensor,
            out_attn: "Optional[list]" = None):
        outs = []
        flags = None
        if self.early_exit:
            if self.flags is None or self.flags.device != tokens.device:
                self.flags = torch.zeros(2, dtype=torch.int32, device=tokens.device)
            flags = self.flags
            flags.zero_()
        for r, b in enumerate(steps, start=1):
            skip = None if flags is None else flags[r % 2]
            done = None if flags is None else flags[(r + 1) % 2]
            block_tau(is_masked, out=b.tau, skip_if=skip)
            b.tokens, b.is_masked = tokens, is_masked
            o = self.step.run(b, out_attn=None if out_attn is None else out_attn[r - 1], skip_if=skip, all_done=done)
            outs.append(o)
        return outs

    def finished(self) -> bool:
        """Whether the last run() completed its block (host read; synchronises)."""
        return self.flags is not None and bool(self.flags.max().item())


class HostStep:
    """RefinementStep driven from host buffers: each run() copies the step's inputs from (pinned)
    host memory to the device, runs the step on the device and copies its results back -- the
    attention output, the modulated RMSNorm output, the updated tokens and mask, the commit
    counts and the new residual."""

    INPUTS = ("tau", "h", "f", "q", "k_blk", "v_blk", "k_ctx", "v_ctx", "ctx_lens", "logits", "tokens", "is_masked")

    def __init__(self, step: RefinementStep, host: Dict[str, torch.Tensor], device, page_table=None):
        self.step = step
        self.host = {k: host[k] for k in self.INPUTS}
        self.dev = {k: torch.empty(v.shape, dtype=v.dtype, device=device) for k, v in self.host.items()}
        self.page_table = None if page_table is None else page_table.to(device)
        self.out_attn = torch.empty_like(self.dev["q"])
        pin = torch.cuda.is_available()
        Bn = self.host["q"].shape[0]
        self.out_host = {
            "attn": torch.empty(self.host["q"].shape, dtype=self.host["q"].dtype, pin_memory=pin),
            "h": torch.empty(self.host["h"].shape, dtype=self.host["h"].dtype, pin_memory=pin),
            "y": torch.empty(self.host["h"].shape, dtype=self.host["h"].dtype, pin_memory=pin),
            "tokens": torch.empty(self.host["tokens"].shape, dtype=torch.int32, pin_memory=pin),
            "is_masked": torch.empty(self.host["is_masked"].shape, dtype=torch.uint8, pin_memory=pin),
            "n_committed": torch.empty(Bn, dtype=torch.int32, pin_memory=pin),
            "n_masked": torch.empty(Bn, dtype=torch.int32, pin_memory=pin),
        }
        self.h2d_bytes = sum(v.numel() * v.element_size() for v in self.host.values())
        self.d2h_bytes = sum(v.numel() * v.element_size() for v in self.out_host.values())

    def run(self) -> Dict[str, torch.Tensor]:
        for k, v in self.host.items():
            self.dev[k].copy_(v, non_blocking=True)
        d = self.dev
        bufs = StepBuffers(tau=d["tau"], h=d["h"], f=d["f"], q=d["q"], k_blk=d["k_blk"], v_blk=d["v_blk"],
                           k_ctx=d["k_ctx"], v_ctx=d["v_ctx"], ctx_lens=d["ctx_lens"], page_table=self.page_table,
                           logits=d["logits"], tokens=d["tokens"], is_masked=d["is_masked"])
        r = self.step.run(bufs, out_attn=self.out_attn)
        o = self.out_host
        o["attn"].copy_(self.out_attn, non_blocking=True)
        o["h"].copy_(r["h"], non_blocking=True)
        o["y"].copy_(r["y"], non_blocking=True)
        o["tokens"].copy_(d["tokens"], non_blocking=True)
        o["is_masked"].copy_(d["is_masked"], non_blocking=True)
        o["n_committed"].copy_(r["n_committed"], non_blocking=True)
        o["n_masked"].copy_(r["n_masked"], non_blocking=True)
        return o
