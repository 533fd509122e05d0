"""GPU parity: kda_chunk_prefill_host (host buffers, segmented and overlapped).

The call cuts T into segments that each start from the previous segment's
final state; the recurrence is sequential in tokens, so the results are those
of the whole sequence: checked against the oracle, and against
kda_chunk_prefill on device copies of the same inputs.
"""
import numpy as np
import pytest
import torch

from _util import TOL_BF16, TOL_F32, compare_units, oracle_prefill, rel_err, to_np
from kda_delta_rule_chunkwise_b200 import binding
from kda_delta_rule_chunkwise_b200 import inputs as kin

pytestmark = pytest.mark.gpu


def host_units(inp, o, s, units):
    res = {}
    for (n, h) in units:
        res[(n, h)] = (to_np(o[n, :, h]), None if s is None else to_np(s[n, h]))
    return res


def run(inp, segment, pinned=True):
    pin = (lambda x: None if x is None else x.contiguous().pin_memory()) if pinned else \
        (lambda x: None if x is None else x.contiguous())
    hq, hk, hv, hg, hb, hs = (pin(x) for x in (inp.q, inp.k, inp.v, inp.g, inp.beta,
                                               inp.state_in))
    o = torch.full((inp.B, inp.T, inp.H, inp.dv), float("nan"), pin_memory=pinned)
    s = torch.full((inp.B, inp.H, inp.dk, inp.dv), float("nan"), pin_memory=pinned)
    binding.kda_chunk_prefill_host(hq, hk, hv, hg, hb, hs, o=o, state_out=s, segment=segment)
    torch.cuda.synchronize()
    assert binding.kda_check_device_error() == binding.KDA_OK
    return o, s


def device_call(inp):
    d = inp.to("cuda")
    o, s = binding.kda_chunk_prefill(d.q, d.k, d.v, d.g, d.beta, d.state_in)
    torch.cuda.synchronize()
    return o.cpu(), s.cpu()


@pytest.mark.parametrize("B,T,segment,state", [(2, 1000, 256, "normal"), (1, 640, 64, "zero"),
                                               (3, 200, 0, "normal")])
def test_host_bf16_against_oracle_and_device_call(B, T, segment, state):
    inp = kin.prefill_inputs(B, T, 4, 128, 128, "bf16", seed=61 + T, state=state)
    o, s = run(inp, segment)
    units = [(n, h) for n in range(B) for h in range(inp.H)]
    compare_units(oracle_prefill(inp), host_units(inp, o, s, units), TOL_BF16,
                  f"host bf16 B{B} T{T} seg{segment}")
    o_dev, s_dev = device_call(inp)
    eo, es = rel_err(to_np(o), to_np(o_dev)), rel_err(to_np(s), to_np(s_dev))
    print(f"host vs device call: o {eo:.3e}, state {es:.3e}, "
          f"bit-exact {torch.equal(o, o_dev) and torch.equal(s, s_dev)}")
    assert eo <= 1e-5 and es <= 1e-5


def test_host_f32_pageable_ragged_d64():
    inp = kin.prefill_inputs(2, 131, 3, 64, 64, "f32", seed=67, state="normal")
    o, s = run(inp, 64, pinned=False)
    units = [(n, h) for n in range(2) for h in range(3)]
    compare_units(oracle_prefill(inp), host_units(inp, o, s, units), TOL_F32,
                  "host fp32 d64 T131 seg64 pageable")


def test_host_without_state_buffers():
    inp = kin.prefill_inputs(1, 300, 2, 128, 128, "bf16", seed=71, state="zero")
    hq, hk, hv, hg, hb = (x.contiguous().pin_memory() for x in (inp.q, inp.k, inp.v, inp.g,
                                                                inp.beta))
    o, s = binding.kda_chunk_prefill_host(hq, hk, hv, hg, hb, None, segment=128,
                                          want_state=False)
    torch.cuda.synchronize()
    assert s is None
    units = [(0, 0), (0, 1)]
    ref = oracle_prefill(inp)
    got = {u: (to_np(o[0, :, u[1]]), ref[u][1]) for u in units}
    compare_units(ref, got, TOL_BF16, "host bf16 no state buffers")


def test_host_full_size_matches_device_call():
    """H = 32, d = 128, T = 65536, one sequence, the default segment: the
    end-to-end configuration; compared with the device-resident call, which the
    prefill parity tests pin to the oracle at this size."""
    d = kin.prefill_inputs(1, 65536, 32, 128, 128, "bf16", seed=5, state="zero",
                           decay="uniform", device="cuda")
    o_dev, s_dev = device_call(d)
    o, s = run(d.to("cpu"), 0)
    eo, es = rel_err(to_np(o), to_np(o_dev)), rel_err(to_np(s), to_np(s_dev))
    print(f"full size host vs device: o {eo:.3e}, state {es:.3e}")
    assert np.isfinite(eo) and eo <= 1e-5 and es <= 1e-5
