"""ctypes binding of libkda (include/kda.h), same names as the C ABI.

Argument marshalling only: every step of the computation runs in the CUDA
kernels inside libkda.so.  Tensors are torch CUDA tensors (device memory and
streams come from PyTorch); their data pointers are passed straight through.
If libkda.so is missing or cannot be loaded, every call raises: there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkda.so")

KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED, KDA_ERR_CUDA, KDA_ERR_TIMEOUT, KDA_ERR_INPUT_RANGE = range(6)
KDA_F32, KDA_BF16 = 0, 1
KDA_PREP_GATE_LOGIT, KDA_PREP_L2NORM_QK = 1, 2
_DTYPE = {torch.float32: KDA_F32, torch.bfloat16: KDA_BF16}

# Every symbol the public header declares.
EXPORTED = (
    "kda_chunk_prefill_workspace_bytes",
    "kda_chunk_prefill",
    "kda_chunk_prefill_checkpointed",
    "kda_chunk_prefill_ex",
    "kda_prefill_checkpoint_count",
    "kda_decode_step",
    "kda_decode_step_indexed",
    "kda_backward_workspace_bytes",
    "kda_backward",
    "kda_check_device_error",
    "kda_selftest_bounded_wait",
    "kda_profile_enable",
    "kda_profile_last",
    "kda_chunk_prefill_static_scratch",
    "kda_prefill_host_workspace_bytes",
    "kda_chunk_prefill_host",
    "kda_status_string",
)


class KDAError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} ({code})")


_lib = None


def load(path: str = LIB_PATH):
    """Load libkda.so (raises if it is missing: build it first)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"libkda.so not found at {path}; build it with "
            "`python -m kda_delta_rule_chunkwise_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    lib.kda_chunk_prefill_workspace_bytes.argtypes = [i64, i32, i32, i32, i32, i32]
    lib.kda_chunk_prefill_workspace_bytes.restype = sz
    lib.kda_chunk_prefill.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, i32,
                                      i32, vp, vp, vp, sz, vp]
    lib.kda_chunk_prefill.restype = i32
    lib.kda_chunk_prefill_checkpointed.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32,
                                                   i32, i32, i32, vp, vp, i64, vp, i64, vp, sz,
                                                   vp]
    lib.kda_chunk_prefill_checkpointed.restype = i32
    lib.kda_chunk_prefill_ex.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, i32,
                                         i32, ctypes.c_uint32, vp, vp, i64, vp, i64, vp, sz, vp]
    lib.kda_chunk_prefill_ex.restype = i32
    lib.kda_prefill_checkpoint_count.argtypes = [vp, i32, i64, i32, i64]
    lib.kda_prefill_checkpoint_count.restype = i64
    lib.kda_backward_workspace_bytes.argtypes = [i64, i32, i32, i32, i32]
    lib.kda_backward_workspace_bytes.restype = sz
    lib.kda_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, i32, i32,
                                 vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.kda_backward.restype = i32
    lib.kda_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, vp, vp]
    lib.kda_decode_step.restype = i32
    lib.kda_decode_step_indexed.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                                            i32, vp, vp]
    lib.kda_decode_step_indexed.restype = i32
    lib.kda_check_device_error.argtypes = [vp]
    lib.kda_check_device_error.restype = i32
    lib.kda_selftest_bounded_wait.argtypes = [i64, vp]
    lib.kda_selftest_bounded_wait.restype = i32
    lib.kda_profile_enable.argtypes = [i32]
    lib.kda_profile_enable.restype = i32
    lib.kda_profile_last.argtypes = [ctypes.POINTER(ctypes.c_float), i32, ctypes.POINTER(i32)]
    lib.kda_profile_last.restype = i32
    lib.kda_chunk_prefill_static_scratch.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i64, i32,
                                                     i32, i32, i32, i32, vp, vp, vp]
    lib.kda_chunk_prefill_static_scratch.restype = i32
    lib.kda_prefill_host_workspace_bytes.argtypes = [i32, i64, i32, i32, i32, i32, i64]
    lib.kda_prefill_host_workspace_bytes.restype = sz
    lib.kda_chunk_prefill_host.argtypes = [vp, vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, i32,
                                           vp, vp, i64, vp, sz, vp]
    lib.kda_chunk_prefill_host.restype = i32
    lib.kda_status_string.argtypes = [i32]
    lib.kda_status_string.restype = ctypes.c_char_p
    _lib = lib
    return lib


def status_string(code: int) -> str:
    return load().kda_status_string(int(code)).decode()


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(code: int, where: str):
    if code != KDA_OK:
        raise KDAError(code, where)


def kda_chunk_prefill_workspace_bytes(rows: int, N: int, H: int, dk: int, dv: int,
                                      dtype: torch.dtype) -> int:
    return int(load().kda_chunk_prefill_workspace_bytes(rows, N, H, dk, dv, _DTYPE[dtype]))


def _contig(name, t):
    if t is not None and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def kda_chunk_prefill(q, k, v, g, beta, state_in=None, cu_seqlens=None, *, o=None,
                      state_out=None, workspace=None, want_state=True, stream=None):
    """Chunked prefill.  Shapes follow include/kda.h; returns (o, state_out).

    q, k, g: [B, T, H, dk]; v: [B, T, H, dv]; beta: [B, T, H] (all one dtype,
    bf16 or fp32); state_in: [N, H, dk, dv] fp32 or None; cu_seqlens: int32
    [N+1] on the device or None.  o [B, T, H, dv] and the state are fp32.
    Output buffers are allocated if not given.
    """
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    N = B if cu_seqlens is None else cu_seqlens.numel() - 1
    for name, t in (("q", q), ("k", k), ("v", v), ("g", g), ("beta", beta),
                    ("state_in", state_in), ("cu_seqlens", cu_seqlens)):
        _contig(name, t)
    if cu_seqlens is not None and cu_seqlens.dtype != torch.int32:
        raise ValueError("cu_seqlens must be int32")
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=torch.float32, device=q.device)
    if state_out is None and want_state:
        state_out = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    need = kda_chunk_prefill_workspace_bytes(B * T, N, H, dk, dv, q.dtype)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    code = load().kda_chunk_prefill(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state_in), _ptr(cu_seqlens),
        B, T, N, H, dk, dv, _DTYPE[q.dtype], _ptr(o), _ptr(state_out),
        _ptr(workspace) if need else None, ws_bytes if need else 0, _stream(stream))
    _check(code, "kda_chunk_prefill")
    return o, state_out


def kda_prefill_host_workspace_bytes(B: int, T: int, H: int, dk: int, dv: int,
                                     dtype: torch.dtype, segment: int = 0) -> int:
    return int(load().kda_prefill_host_workspace_bytes(B, T, H, dk, dv, _DTYPE[dtype], segment))


def kda_chunk_prefill_host(q, k, v, g, beta, state_in=None, *, o=None, state_out=None,
                           segment=0, workspace=None, want_state=True, device=None,
                           stream=None):
    """Prefill of B sequences from HOST tensors (pinned for overlap); returns (o, state_out).

    Same shapes as kda_chunk_prefill without cu_seqlens; o and state_out are
    host fp32 tensors (pinned ones are allocated if not given).  The library
    copies segments of `segment` tokens in and out while it computes; the
    outputs are complete once `stream` (default: the current stream of
    `device`, default cuda:0's) has passed the call.
    """
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    for name, t in (("q", q), ("k", k), ("v", v), ("g", g), ("beta", beta),
                    ("state_in", state_in), ("o", o), ("state_out", state_out)):
        _contig(name, t)
        if t is not None and t.is_cuda:
            raise ValueError(f"{name} must be a host tensor")
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else \
        torch.device(device)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=torch.float32, pin_memory=True)
    if state_out is None and want_state:
        state_out = torch.empty((B, H, dk, dv), dtype=torch.float32, pin_memory=True)
    need = kda_prefill_host_workspace_bytes(B, T, H, dk, dv, q.dtype, segment)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(device):
        code = load().kda_chunk_prefill_host(
            _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state_in), B, T, H, dk, dv,
            _DTYPE[q.dtype], _ptr(o), _ptr(state_out), segment,
            _ptr(workspace) if need else None, ws_bytes if need else 0, _stream(stream))
    _check(code, "kda_chunk_prefill_host")
    return o, state_out


def kda_prefill_checkpoint_count(cu_seqlens, B: int, T: int, interval: int) -> int:
    """Snapshots kda_chunk_prefill_checkpointed writes (cu_seqlens: int32 tensor or None;
    a device tensor is copied to the host)."""
    if cu_seqlens is None:
        n = load().kda_prefill_checkpoint_count(None, B, T, B, int(interval))
    else:
        host = cu_seqlens.to("cpu", torch.int32).contiguous()
        n = load().kda_prefill_checkpoint_count(_ptr(host), 1, T, host.numel() - 1, int(interval))
    if n < 0:
        raise KDAError(KDA_ERR_INVALID_ARG, "kda_prefill_checkpoint_count")
    return int(n)


def kda_chunk_prefill_checkpointed(q, k, v, g, beta, state_in=None, cu_seqlens=None, *,
                                   interval: int, ckpt=None, o=None, state_out=None,
                                   workspace=None, stream=None):
    """kda_chunk_prefill plus the state every `interval` tokens inside each sequence.

    Returns (o, state_out, ckpt) with ckpt [count, H, dk, dv] fp32 (allocated if not
    given), entries in sequence order (see include/kda.h)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    N = B if cu_seqlens is None else cu_seqlens.numel() - 1
    for name, t in (("q", q), ("k", k), ("v", v), ("g", g), ("beta", beta),
                    ("state_in", state_in), ("cu_seqlens", cu_seqlens), ("ckpt", ckpt)):
        _contig(name, t)
    if ckpt is None:
        cnt = kda_prefill_checkpoint_count(cu_seqlens, B, T, interval)
        ckpt = torch.empty((cnt, H, dk, dv), dtype=torch.float32, device=q.device)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=torch.float32, device=q.device)
    if state_out is None:
        state_out = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    need = kda_chunk_prefill_workspace_bytes(B * T, N, H, dk, dv, q.dtype)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    code = load().kda_chunk_prefill_checkpointed(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state_in), _ptr(cu_seqlens),
        B, T, N, H, dk, dv, _DTYPE[q.dtype], _ptr(o), _ptr(state_out), int(interval),
        _ptr(ckpt) if ckpt.numel() else None, ckpt.shape[0],
        _ptr(workspace) if need else None, ws_bytes if need else 0, _stream(stream))
    _check(code, "kda_chunk_prefill_checkpointed")
    return o, state_out, ckpt


def kda_chunk_prefill_ex(q, k, v, g, beta, state_in=None, cu_seqlens=None, *, flags=0,
                         ckpt_interval=0, ckpt=None, o=None, state_out=None, workspace=None,
                         stream=None):
    """The general prefill: preprocessing `flags` (KDA_PREP_*) and, with ckpt_interval > 0,
    intermediate states.  Returns (o, state_out, ckpt or None)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    N = B if cu_seqlens is None else cu_seqlens.numel() - 1
    for name, t in (("q", q), ("k", k), ("v", v), ("g", g), ("beta", beta),
                    ("state_in", state_in), ("cu_seqlens", cu_seqlens), ("ckpt", ckpt)):
        _contig(name, t)
    if ckpt_interval and ckpt is None:
        cnt = kda_prefill_checkpoint_count(cu_seqlens, B, T, ckpt_interval)
        ckpt = torch.empty((cnt, H, dk, dv), dtype=torch.float32, device=q.device)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=torch.float32, device=q.device)
    if state_out is None:
        state_out = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    need = kda_chunk_prefill_workspace_bytes(B * T, N, H, dk, dv, q.dtype)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    has_ck = ckpt is not None and ckpt.numel() > 0
    code = load().kda_chunk_prefill_ex(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state_in), _ptr(cu_seqlens),
        B, T, N, H, dk, dv, _DTYPE[q.dtype], int(flags), _ptr(o), _ptr(state_out),
        int(ckpt_interval), _ptr(ckpt) if has_ck else None, ckpt.shape[0] if has_ck else 0,
        _ptr(workspace) if need else None, ws_bytes if need else 0, _stream(stream))
    _check(code, "kda_chunk_prefill_ex")
    return o, state_out, ckpt


def kda_backward(q, k, v, g, beta, state_in, cu_seqlens, dout, dstate_out=None, *,
                 want_dstate_in=True, workspace=None, stream=None):
    """Gradients of the recurrence: returns (dq, dk, dv, dg, dbeta, dstate_in), all fp32
    (dstate_in None unless want_dstate_in).  Inputs as for kda_chunk_prefill; dout like o."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    N = B if cu_seqlens is None else cu_seqlens.numel() - 1
    for name, t in (("q", q), ("k", k), ("v", v), ("g", g), ("beta", beta), ("state_in", state_in),
                    ("cu_seqlens", cu_seqlens), ("dout", dout), ("dstate_out", dstate_out)):
        _contig(name, t)
    f32 = lambda shape: torch.zeros(shape, dtype=torch.float32, device=q.device)
    dq, dk_, dg = f32(q.shape), f32(k.shape), f32(g.shape)
    dv_, db = f32(v.shape), f32(beta.shape)
    ds0 = f32((N, H, dk, dv)) if want_dstate_in else None
    need = int(load().kda_backward_workspace_bytes(B * T, N, H, dk, dv))
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    code = load().kda_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state_in), _ptr(cu_seqlens), B, T, N,
        H, dk, dv, _DTYPE[q.dtype], _ptr(dout), _ptr(dstate_out), _ptr(dq), _ptr(dk_), _ptr(dv_),
        _ptr(dg), _ptr(db), _ptr(ds0), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream))
    _check(code, "kda_backward")
    return dq, dk_, dv_, dg, db, ds0


class KDAPrefill(torch.autograd.Function):
    """The prefill as a differentiable op: forward is kda_chunk_prefill, backward
    is kda_backward (the exact gradients of the recurrence, fp32, cast to each
    input's dtype).  Returns (o, state_out); cu_seqlens gets no gradient."""

    @staticmethod
    def forward(ctx, q, k, v, g, beta, state_in=None, cu_seqlens=None):
        o, s = kda_chunk_prefill(q, k, v, g, beta, state_in, cu_seqlens)
        ctx.save_for_backward(q, k, v, g, beta, state_in, cu_seqlens)
        return o, s

    @staticmethod
    def backward(ctx, do, dstate):
        q, k, v, g, beta, state_in, cu = ctx.saved_tensors
        grads = kda_backward(q, k, v, g, beta, state_in, cu, do.contiguous().float(),
                             None if dstate is None else dstate.contiguous().float(),
                             want_dstate_in=state_in is not None)
        dq, dk_, dv_, dg, db, ds0 = grads
        return (dq.to(q.dtype), dk_.to(k.dtype), dv_.to(v.dtype), dg.to(g.dtype),
                db.to(beta.dtype), ds0, None)


def kda_prefill_autograd(q, k, v, g, beta, state_in=None, cu_seqlens=None):
    """Differentiable prefill (see KDAPrefill): (o, state_out)."""
    return KDAPrefill.apply(q, k, v, g, beta, state_in, cu_seqlens)


def kda_decode_step(q, k, v, g, beta, state, *, o=None, stream=None):
    """One decode step; `state` [N, H, dk, dv] fp32 is updated in place.  Returns o (fp32)."""
    N, H, dk = q.shape
    dv = v.shape[-1]
    for name, t in (("q", q), ("k", k), ("v", v), ("g", g), ("beta", beta), ("state", state)):
        _contig(name, t)
    if o is None:
        o = torch.empty((N, H, dv), dtype=torch.float32, device=q.device)
    code = load().kda_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state),
                                  N, H, dk, dv, _DTYPE[q.dtype], _ptr(o), _stream(stream))
    _check(code, "kda_decode_step")
    return o


def kda_decode_step_indexed(q, k, v, g, beta, state_pool, slots, *, o=None, stream=None):
    """One decode step on pool entries `slots` (int32 [N], distinct) of `state_pool`
    [P, H, dk, dv] fp32, updated in place.  Returns o (fp32)."""
    N, H, dk = q.shape
    dv = v.shape[-1]
    for name, t in (("q", q), ("k", k), ("v", v), ("g", g), ("beta", beta),
                    ("state_pool", state_pool), ("slots", slots)):
        _contig(name, t)
    if slots.dtype != torch.int32 or slots.numel() != N:
        raise ValueError("slots must be an int32 tensor with one entry per request")
    if o is None:
        o = torch.empty((N, H, dv), dtype=torch.float32, device=q.device)
    code = load().kda_decode_step_indexed(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state_pool), _ptr(slots), N,
        state_pool.shape[0], H, dk, dv, _DTYPE[q.dtype], _ptr(o), _stream(stream))
    _check(code, "kda_decode_step_indexed")
    return o


def kda_check_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error status code."""
    return int(load().kda_check_device_error(_stream(stream)))


def kda_selftest_bounded_wait(timeout_us: int, stream=None):
    _check(load().kda_selftest_bounded_wait(int(timeout_us), _stream(stream)),
           "kda_selftest_bounded_wait")


def kda_profile_enable(enable: bool = True):
    _check(load().kda_profile_enable(1 if enable else 0), "kda_profile_enable")


def kda_profile_last(capacity: int = 8):
    """Device milliseconds of each kernel of the most recent call (launch order)."""
    buf = (ctypes.c_float * capacity)()
    cnt = ctypes.c_int(0)
    _check(load().kda_profile_last(buf, capacity, ctypes.byref(cnt)), "kda_profile_last")
    return [float(buf[i]) for i in range(cnt.value)]


# ---------------------------------------------------------------- raw C-ABI access

def raw_prefill(args: dict) -> int:
    """Call kda_chunk_prefill with raw integers/pointers (for ABI-level tests)."""
    lib = load()
    return int(lib.kda_chunk_prefill(
        args.get("q"), args.get("k"), args.get("v"), args.get("g"), args.get("beta"),
        args.get("state_in"), args.get("cu_seqlens"), args["B"], args["T"], args["N"],
        args["H"], args["dk"], args["dv"], args["dtype"], args.get("o"), args.get("state_out"),
        args.get("workspace"), args.get("workspace_bytes", 0), args.get("stream")))


def raw_prefill_checkpointed(args: dict) -> int:
    lib = load()
    return int(lib.kda_chunk_prefill_checkpointed(
        args.get("q"), args.get("k"), args.get("v"), args.get("g"), args.get("beta"),
        args.get("state_in"), args.get("cu_seqlens"), args["B"], args["T"], args["N"],
        args["H"], args["dk"], args["dv"], args["dtype"], args.get("o"), args.get("state_out"),
        args["interval"], args.get("ckpt"), args.get("ckpt_capacity", 0),
        args.get("workspace"), args.get("workspace_bytes", 0), args.get("stream")))


def raw_prefill_host(args: dict) -> int:
    lib = load()
    return int(lib.kda_chunk_prefill_host(
        args.get("q"), args.get("k"), args.get("v"), args.get("g"), args.get("beta"),
        args.get("state_in"), args["B"], args["T"], args["H"], args["dk"], args["dv"],
        args["dtype"], args.get("o"), args.get("state_out"), args.get("segment", 0),
        args.get("workspace"), args.get("workspace_bytes", 0), args.get("stream")))


def raw_decode_indexed(args: dict) -> int:
    lib = load()
    return int(lib.kda_decode_step_indexed(
        args.get("q"), args.get("k"), args.get("v"), args.get("g"), args.get("beta"),
        args.get("state"), args.get("slots"), args["N"], args["P"], args["H"], args["dk"],
        args["dv"], args["dtype"], args.get("o"), args.get("stream")))


def raw_decode(args: dict) -> int:
    lib = load()
    return int(lib.kda_decode_step(
        args.get("q"), args.get("k"), args.get("v"), args.get("g"), args.get("beta"),
        args.get("state"), args["N"], args["H"], args["dk"], args["dv"], args["dtype"],
        args.get("o"), args.get("stream")))
