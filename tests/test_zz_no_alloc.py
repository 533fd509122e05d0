"""The allocation-free prefill entry point, kda_chunk_prefill_static_scratch.

It exists for callers that cannot allocate device memory: a serving step
whose device memory is fully reserved up front (a cudaMalloc there can fail
under memory pressure and synchronises the device), or a plugin whose host
runtime owns all allocation.  Its scratch is a fixed array inside libkda.

The test calls it through the C ABI (ctypes, raw device pointers) twice in a
row, on different inputs, and checks each result against the regular entry
point kda_chunk_prefill (which uses a caller-allocated workspace).  Both run
the same kernels on the same inputs and every accumulation has a fixed order,
so the results must be equal bit for bit: a scratch-aliasing fault that the
parity tolerance could hide would show here.  It also checks that a call needing more scratch than the
array holds is refused before anything is launched.  This file is named so
that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from kda_delta_rule_chunkwise_b200 import binding
from kda_delta_rule_chunkwise_b200 import inputs as kin

pytestmark = pytest.mark.gpu

STATIC_SCRATCH_BYTES = 128 << 20


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def call_static(d, o, s_out):
    lib = binding.load()
    N = d.N
    code = lib.kda_chunk_prefill_static_scratch(
        _p(d.q), _p(d.k), _p(d.v), _p(d.g), _p(d.beta), _p(d.state_in), _p(d.cu_seqlens),
        d.B, d.T, N, d.H, d.dk, d.dv, binding.KDA_BF16, _p(o), _p(s_out),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return code


def test_static_scratch_matches_workspace_entry_two_calls():
    cases = [
        kin.prefill_inputs(1, 1000, 4, 128, 128, "bf16", seed=31, state="normal"),
        kin.prefill_inputs(1, 1065, 8, 128, 128, "bf16", seed=32, decay="split", state="normal",
                           lengths=[300, 0, 700, 65]),
    ]
    for i, inp in enumerate(cases):
        d = inp.to("cuda")
        need = binding.kda_chunk_prefill_workspace_bytes(d.B * d.T, d.N, d.H, 128, 128,
                                                         torch.bfloat16)
        assert 0 < need <= STATIC_SCRATCH_BYTES
        o = torch.full((d.B, d.T, d.H, 128), float("nan"), dtype=torch.float32, device="cuda")
        s = torch.full((d.N, d.H, 128, 128), float("nan"), dtype=torch.float32, device="cuda")
        assert call_static(d, o, s) == binding.KDA_OK
        torch.cuda.synchronize()
        assert binding.kda_check_device_error() == binding.KDA_OK
        o_ref, s_ref = binding.kda_chunk_prefill(d.q, d.k, d.v, d.g, d.beta, d.state_in,
                                                 d.cu_seqlens)
        torch.cuda.synchronize()
        if d.cu_seqlens is not None:
            # rows outside every sequence are not written by either entry point
            cu = d.cu_seqlens.cpu().numpy()
            rows = torch.as_tensor(np.concatenate([np.arange(cu[n], cu[n + 1]) for n in range(d.N)]),
                                   device="cuda")
            got, want = o[0, rows], o_ref[0, rows]
        else:
            got, want = o, o_ref
        assert torch.isfinite(got).all() and torch.isfinite(s).all(), f"call {i}"
        assert torch.equal(got, want), f"call {i}: output differs from kda_chunk_prefill"
        assert torch.equal(s, s_ref), f"call {i}: state differs from kda_chunk_prefill"


def test_static_scratch_refuses_oversized_calls():
    lib = binding.load()
    # T large enough that the bound exceeds the array; nothing is dereferenced
    code = lib.kda_chunk_prefill_static_scratch(
        ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(16),
        ctypes.c_void_p(16), None, None, 1, 1 << 20, 1, 32, 128, 128, binding.KDA_BF16,
        ctypes.c_void_p(16), None, None)
    assert code == binding.KDA_ERR_UNSUPPORTED
