"""Seeded synthetic inputs for KDA prefill and decode.

This module holds no KDA arithmetic: it only draws random tensors with the
shapes and value distributions of the benchmark workloads, so that the CUDA
path and the fp64 oracle can be fed the very same values.

Draw order (fixed so that a seed names one input set):
  1. q, k, v ~ N(0, 1) in fp32
  2. q and k L2-normalised per (token, head) in fp32 (the caller's job in the
     library contract; the library itself does not normalise)
  3. g_raw ~ N(0, 1) -> g = -5 * sigmoid(g_raw)        (g in (-5, 0))
     or, for the "split" decay mode, channels [0, dk/2) get
     g = -5 + 0.25 * sigmoid(g_raw) (fast decay, near -5) and channels
     [dk/2, dk) get g = -0.01 * sigmoid(g_raw) (slow retention, near 0)
  4. beta_raw ~ N(0, 1) -> beta = sigmoid(beta_raw)
  5. initial state ~ N(0, 0.1^2) in fp32 when requested, else zeros
  6. cast q, k, v, g, beta to the compute dtype last; the state stays fp32.

Everything is generated with ``torch.Generator(device).manual_seed(seed)``
on the requested device; CPU and CUDA generators give different streams, so
a consumer that needs the values on both sides copies them across.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import torch

DTYPES = {"bf16": torch.bfloat16, "f32": torch.float32}


@dataclass
class PrefillInputs:
    q: torch.Tensor          # [B, T, H, dk]
    k: torch.Tensor          # [B, T, H, dk]
    v: torch.Tensor          # [B, T, H, dv]
    g: torch.Tensor          # [B, T, H, dk]
    beta: torch.Tensor       # [B, T, H]
    state_in: Optional[torch.Tensor]   # [N, H, dk, dv] fp32 or None
    cu_seqlens: Optional[torch.Tensor]  # int32 [N+1] or None
    dtype: str = "bf16"
    meta: dict = field(default_factory=dict)

    @property
    def B(self) -> int:
        return self.q.shape[0]

    @property
    def T(self) -> int:
        return self.q.shape[1]

    @property
    def H(self) -> int:
        return self.q.shape[2]

    @property
    def dk(self) -> int:
        return self.q.shape[3]

    @property
    def dv(self) -> int:
        return self.v.shape[3]

    @property
    def N(self) -> int:
        return self.B if self.cu_seqlens is None else self.cu_seqlens.numel() - 1

    def to(self, device) -> "PrefillInputs":
        mv = lambda x: None if x is None else x.to(device)
        return PrefillInputs(mv(self.q), mv(self.k), mv(self.v), mv(self.g),
                             mv(self.beta), mv(self.state_in),
                             mv(self.cu_seqlens), self.dtype, dict(self.meta))


@dataclass
class DecodeInputs:
    q: torch.Tensor      # [steps, N, H, dk]
    k: torch.Tensor
    v: torch.Tensor      # [steps, N, H, dv]
    g: torch.Tensor
    beta: torch.Tensor   # [steps, N, H]
    state: torch.Tensor  # [N, H, dk, dv] fp32
    dtype: str = "bf16"


def _normal(shape, gen, device, std=1.0):
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    return x if std == 1.0 else x * std


def _unit(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)


def _decay(shape, gen, device, mode: str) -> torch.Tensor:
    z = _normal(shape, gen, device)
    if mode == "uniform":
        return -5.0 * torch.sigmoid(z)
    if mode == "split":
        dk = shape[-1]
        g = torch.empty_like(z)
        h = dk // 2
        g[..., :h] = -5.0 + 0.25 * torch.sigmoid(z[..., :h])
        g[..., h:] = -0.01 * torch.sigmoid(z[..., h:])
        return g
    raise ValueError(f"unknown decay mode {mode!r}")


def prefill_inputs(B: int, T: int, H: int, dk: int, dv: int, dtype: str = "bf16",
                   seed: int = 0, decay: str = "uniform", state: str = "zero",
                   lengths=None, device="cpu") -> PrefillInputs:
    """Equal-length batch [B, T] or, with ``lengths``, one packed batch.

    With ``lengths`` (a list of N sequence lengths), B must be 1 and T must
    equal sum(lengths); cu_seqlens is returned as int32 [N+1].
    """
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    tdt = DTYPES[dtype]
    q = _unit(_normal((B, T, H, dk), gen, device))
    k = _unit(_normal((B, T, H, dk), gen, device))
    v = _normal((B, T, H, dv), gen, device)
    g = _decay((B, T, H, dk), gen, device, decay)
    beta = torch.sigmoid(_normal((B, T, H), gen, device))
    if lengths is not None:
        if B != 1 or sum(lengths) != T:
            raise ValueError("packed inputs need B == 1 and T == sum(lengths)")
        cu = torch.zeros(len(lengths) + 1, dtype=torch.int64)
        cu[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0)
        cu_seqlens = cu.to(torch.int32).to(device)
        N = len(lengths)
    else:
        cu_seqlens = None
        N = B
    if state == "zero":
        s0 = None
    elif state == "normal":
        s0 = _normal((N, H, dk, dv), gen, device, std=0.1)
    else:
        raise ValueError(f"unknown state mode {state!r}")
    cast = lambda x: x.to(tdt).contiguous()
    return PrefillInputs(cast(q), cast(k), cast(v), cast(g), cast(beta), s0,
                         cu_seqlens, dtype,
                         dict(seed=seed, decay=decay, state=state))


def prefill_raw_inputs(B: int, T: int, H: int, dk: int, dv: int, dtype: str = "bf16",
                       seed: int = 0, state: str = "normal", lengths=None,
                       device="cpu") -> PrefillInputs:
    """Like prefill_inputs, but q and k are raw projections (N(0, 1) scaled by a random
    per-(token, head) norm in [0.5, 4], not normalised) and g holds gate logits
    ~ N(0, 1), for a prefill that normalises q, k and forms the gate itself."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    tdt = DTYPES[dtype]
    scale = lambda: 0.5 + 3.5 * torch.rand((B, T, H, 1), generator=gen, device=device)
    q = _normal((B, T, H, dk), gen, device) * scale()
    k = _normal((B, T, H, dk), gen, device) * scale()
    v = _normal((B, T, H, dv), gen, device)
    g = _normal((B, T, H, dk), gen, device)
    beta = torch.sigmoid(_normal((B, T, H), gen, device))
    if lengths is not None:
        if B != 1 or sum(lengths) != T:
            raise ValueError("packed inputs need B == 1 and T == sum(lengths)")
        cu = torch.zeros(len(lengths) + 1, dtype=torch.int64)
        cu[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0)
        cu_seqlens = cu.to(torch.int32).to(device)
        N = len(lengths)
    else:
        cu_seqlens = None
        N = B
    s0 = _normal((N, H, dk, dv), gen, device, std=0.1) if state == "normal" else None
    cast = lambda x: x.to(tdt).contiguous()
    return PrefillInputs(cast(q), cast(k), cast(v), cast(g), cast(beta), s0, cu_seqlens, dtype,
                         dict(seed=seed, decay="logits", state=state))


def varlen_lengths(n_seqs: int, lo: int, hi: int, seed: int = 0) -> list:
    """Integer-uniform sequence lengths in [lo, hi], inclusive, seeded (CPU)."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    return torch.randint(lo, hi + 1, (n_seqs,), generator=gen).tolist()


def decode_inputs(steps: int, N: int, H: int, dk: int, dv: int, dtype: str = "bf16",
                  seed: int = 0, device="cpu") -> DecodeInputs:
    """``steps`` consecutive single-token inputs per sequence plus a random state."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    tdt = DTYPES[dtype]
    q = _unit(_normal((steps, N, H, dk), gen, device))
    k = _unit(_normal((steps, N, H, dk), gen, device))
    v = _normal((steps, N, H, dv), gen, device)
    g = _decay((steps, N, H, dk), gen, device, "uniform")
    beta = torch.sigmoid(_normal((steps, N, H), gen, device))
    s0 = _normal((N, H, dk, dv), gen, device, std=0.1)
    cast = lambda x: x.to(tdt).contiguous()
    return DecodeInputs(cast(q), cast(k), cast(v), cast(g), cast(beta), s0, dtype)


# The benchmark workloads, by what they are.
WORKLOADS = {
    "tiny_f32_h2_t256_d64": dict(kind="prefill", B=1, T=256, H=2, dk=64, dv=64,
                                 dtype="f32", decay="uniform", state="zero"),
    "prefill_h32_t8192_d128": dict(kind="prefill", B=1, T=8192, H=32, dk=128,
                                   dv=128, dtype="bf16", decay="uniform",
                                   state="zero"),
    "prefill_h32_t65536_d128_split": dict(kind="prefill", B=1, T=65536, H=32,
                                          dk=128, dv=128, dtype="bf16",
                                          decay="split", state="normal"),
    "decode_n256_h32_d128": dict(kind="decode", N=256, H=32, dk=128, dv=128,
                                 dtype="bf16", steps=1000),
    "varlen_64seq_128to16384_h32_d128": dict(kind="varlen", n_seqs=64, lo=128,
                                             hi=16384, H=32, dk=128, dv=128,
                                             dtype="bf16", decay="uniform",
                                             state="normal"),
}


def workload_inputs(name: str, seed: int = 0, device="cpu"):
    """Inputs for one named workload (prefill/varlen -> PrefillInputs)."""
    w = WORKLOADS[name]
    if w["kind"] == "prefill":
        return prefill_inputs(w["B"], w["T"], w["H"], w["dk"], w["dv"], w["dtype"],
                              seed, w["decay"], w["state"], device=device)
    if w["kind"] == "varlen":
        lens = varlen_lengths(w["n_seqs"], w["lo"], w["hi"], seed)
        return prefill_inputs(1, sum(lens), w["H"], w["dk"], w["dv"], w["dtype"],
                              seed, w["decay"], w["state"], lengths=lens,
                              device=device)
    raise ValueError(f"{name} is a decode workload; use decode_inputs")
