"""fp64 CPU oracle for the Kimi Delta Attention recurrence.

TEST INFRASTRUCTURE ONLY.  The tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module; the library's
product path never does, and this module imports nothing from it.

The forward arithmetic lives in ``kda_oracle.c`` (plain C, fp64, one token
at a time); this wrapper compiles it with gcc, converts the caller's arrays to
contiguous fp64 (an exact conversion from bf16/fp32), and calls it.  Two
helpers are written here: ``preprocess`` (the gate-from-logit and q/k
normalisation a fused prefill applies, fp64 numpy) and ``backward`` (the
gradients, by PyTorch autograd in fp64 over the token recurrence written out).

Recurrence (the delta rule with per-channel retention described in words in
neurohive.io "Kimi K3 ... overview", section "Sequence length: hybrid KDA and
Gated MLA attention", and best.xiaohu.ai "Kimi K3 tech report", section
"Sequence length: replacing most attention layers with fixed-size memory"):

    S_t = (I - beta_t k_t k_t^T) Diag(exp g_t) S_{t-1} + beta_t k_t v_t^T
    o_t = S_t^T q_t,   with g clamped as max(g, -5)

Every function here is pinned by ``tests/test_oracle_pins.py`` against
closed forms, invariants and brute-force matrix products; see that file.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libkda_oracle.so")
_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile ``kda_oracle.c`` into a shared library (gcc, -O2, no fast-math)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-pthread",
           "-fno-fast-math", "-ffp-contract=off", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = load_library(build())
    return _lib


def _f64(x) -> np.ndarray:
    """Exact conversion of a numpy array or torch tensor (bf16/fp32/fp64) to fp64."""
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor; bf16 -> fp64 is exact
        import torch
        x = x.detach().to("cpu", torch.float64).contiguous().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def load_library(path: str):
    """Load an oracle shared library built from ``kda_oracle.c`` at ``path``.

    Used by the tests that compile deliberately broken copies of the oracle
    to show that the pins catch them.
    """
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    lib.kda_oracle_recurrence.argtypes = [
        dp, dp, dp, dp, dp, dp, ctypes.POINTER(ctypes.c_int64),
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        dp, dp, ctypes.c_int]
    lib.kda_oracle_recurrence.restype = ctypes.c_int
    return lib


def recurrence(q, k, v, g, beta, state_in=None, cu_seqlens=None,
               n_threads: int | None = None, lib=None):
    """Run the fp64 token recurrence.

    Shapes (B equal-length sequences, or one packed batch with cu_seqlens):
      q, k, g: [B, T, H, dk]   v: [B, T, H, dv]   beta: [B, T, H]
      state_in: [N, H, dk, dv] or None (zeros)
      cu_seqlens: int array [N+1] of row offsets into the B*T rows, or None
                  (then N = B and sequence b owns rows b*T .. b*T+T-1).
    Returns (o [B, T, H, dv] fp64, state_out [N, H, dk, dv] fp64).
    """
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    if q.ndim != 4:
        raise ValueError("q must be [B, T, H, dk]")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or g.shape != q.shape or v.shape[:3] != q.shape[:3] \
            or beta.shape != q.shape[:3]:
        raise ValueError("inconsistent shapes")
    if cu_seqlens is None:
        cu = np.arange(B + 1, dtype=np.int64) * T
    else:
        if hasattr(cu_seqlens, "detach"):
            cu_seqlens = cu_seqlens.detach().cpu().numpy()
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
        if cu[0] != 0 or cu[-1] > B * T or np.any(np.diff(cu) < 0):
            raise ValueError("bad cu_seqlens")
    N = len(cu) - 1
    s_in = _f64(state_in)
    if s_in is not None and s_in.shape != (N, H, dk, dv):
        raise ValueError("state_in must be [N, H, dk, dv]")
    o = np.zeros((B, T, H, dv), dtype=np.float64)
    s_out = np.zeros((N, H, dk, dv), dtype=np.float64)
    nt = default_threads() if n_threads is None else int(n_threads)
    rc = (lib or _load()).kda_oracle_recurrence(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(s_in),
        cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
        N, H, dk, dv, _ptr(o), _ptr(s_out), max(1, min(nt, N * H)))
    if rc != 0:
        raise RuntimeError(f"oracle returned {rc}")
    return o, s_out


GATE_LOGIT = 1     # g holds logits x; the log-decay is -5 sigmoid(x)
L2NORM_QK = 2      # q and k are scaled to unit L2 norm over dk per (token, head)


def preprocess(q, k, g, flags: int):
    """The input preprocessing a fused prefill applies, in fp64, before the recurrence.

    GATE_LOGIT: g <- -5 / (1 + exp(-x)), the lower bound -5 on the log-decay of
    neurohive.io "Kimi K3 ... overview", section "Sequence length: hybrid KDA and
    Gated MLA attention", written as a parametrisation (the form the synthetic
    inputs use).  L2NORM_QK: x <- x / ||x||_2 over the last axis; a zero vector
    stays zero.  Returns fp64 (q, k, g).
    """
    q, k, g = _f64(q), _f64(k), _f64(g)
    if flags & GATE_LOGIT:
        g = -5.0 / (1.0 + np.exp(-g))
    if flags & L2NORM_QK:
        def unit(x):
            n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
            return np.divide(x, n, out=np.zeros_like(x), where=n > 0)
        q, k = unit(q), unit(k)
    return q, k, g


def backward(q, k, v, g, beta, state_in, dout, dstate_out=None, cu_seqlens=None):
    """Gradients of L = sum(o * dout) + sum(S_final * dstate_out) with respect to
    q, k, v, g, beta and the initial state, by reverse-mode differentiation
    (PyTorch autograd on CPU, fp64) of the recurrence written out token by token:
        a = exp(clamp(g, min=-5)),  S' = Diag(a) S,  p = S'^T k,
        S = S' + beta k (v - p)^T,  o = S^T q
    the same recurrence as kda_oracle.c (the clamp passes no gradient below -5).
    Shapes as in recurrence(); dout like o, dstate_out like the final state (or
    None).  Returns fp64 numpy arrays (dq, dk, dv, dg, dbeta, dstate_in).
    """
    import torch
    t64 = lambda x: torch.from_numpy(_f64(x))
    q, k, v, g, beta = (t64(x).requires_grad_(True) for x in (q, k, v, g, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is None:
        spans = [(b, 0, T) for b in range(B)]
    else:
        cu = np.asarray(cu_seqlens, dtype=np.int64)
        spans = [(0, int(cu[n]), int(cu[n + 1])) for n in range(len(cu) - 1)]
    N = len(spans)
    S0 = (t64(state_in) if state_in is not None else torch.zeros((N, H, dk, dv), dtype=torch.float64))
    S0.requires_grad_(True)
    dout_t = t64(dout)
    loss = torch.zeros((), dtype=torch.float64)
    for n, (b, t0, t1) in enumerate(spans):
        S = S0[n]
        for t in range(t0, t1):
            a = torch.exp(torch.clamp(g[b, t], min=-5.0))                      # [H, dk]
            Sp = a[:, :, None] * S
            p = torch.einsum("hcj,hc->hj", Sp, k[b, t])
            S = Sp + beta[b, t][:, None, None] * k[b, t][:, :, None] * (v[b, t] - p)[:, None, :]
            o = torch.einsum("hcj,hc->hj", S, q[b, t])
            loss = loss + (o * dout_t[b, t]).sum()
        if dstate_out is not None:
            loss = loss + (S * t64(dstate_out)[n]).sum()
    loss.backward()
    return tuple(x.grad.numpy() for x in (q, k, v, g, beta, S0))


def decode_step(q, k, v, g, beta, state, n_threads: int | None = None, lib=None):
    """One decode step: the same recurrence with a single token per sequence.

    q, k, g: [N, H, dk]; v: [N, H, dv]; beta: [N, H]; state: [N, H, dk, dv].
    Returns (o [N, H, dv], new_state [N, H, dk, dv]), both fp64.
    """
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    N = q.shape[0]
    o, s = recurrence(q[:, None], k[:, None], v[:, None], g[:, None],
                      beta[:, None], state_in=state,
                      cu_seqlens=np.arange(N + 1, dtype=np.int64),
                      n_threads=n_threads, lib=lib)
    # packed as B=N, T=1: row n belongs to sequence n
    return o[:, 0], s
