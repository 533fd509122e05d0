"""The device error word: per-launch timeouts, reporting order, the debug input
scan, and malformed cu_seqlens handled alike by every prefill path."""
import numpy as np
import pytest
import torch

from _util import TOL_BF16, TOL_F32, compare_units, gather_gpu, oracle_prefill
from kda_delta_rule_chunkwise_b200 import binding
from kda_delta_rule_chunkwise_b200 import inputs as kin

pytestmark = pytest.mark.gpu


def _drain():
    for _ in range(8):
        if binding.kda_check_device_error() == binding.KDA_OK:
            return
    raise AssertionError("error word does not drain")


def test_stale_timeout_does_not_cut_short_a_later_prefill():
    """A timeout left in the error word (nobody called kda_check_device_error after
    the self test) must not make a later prefill's waits give up: the prefill runs
    in full and matches the oracle, and the old timeout is still reported."""
    _drain()
    binding.kda_selftest_bounded_wait(2000)          # records a timeout, not checked
    torch.cuda.synchronize()
    inp = kin.prefill_inputs(1, 1500, 4, 128, 128, "bf16", seed=41, decay="split", state="normal")
    d = inp.to("cuda")
    o, s = binding.kda_chunk_prefill(d.q, d.k, d.v, d.g, d.beta, d.state_in, None)
    torch.cuda.synchronize()
    ref = oracle_prefill(inp)
    compare_units(ref, gather_gpu(inp, o, s, list(ref)), TOL_BF16, "after a stale timeout")
    assert binding.kda_check_device_error() == binding.KDA_ERR_TIMEOUT   # the self test's
    assert binding.kda_check_device_error() == binding.KDA_OK


def test_error_word_reports_each_condition_once_most_severe_first():
    _drain()
    binding.kda_selftest_bounded_wait(1000)
    # an out-of-range pool entry: skipped on the device and recorded as a bad index
    inp = kin.decode_inputs(1, 2, 2, 128, 128, "bf16", seed=42)
    pool = torch.zeros((2, 2, 128, 128), device="cuda")
    slots = torch.tensor([0, 5], dtype=torch.int32, device="cuda")
    c = lambda x: x[0].contiguous().cuda()
    binding.kda_decode_step_indexed(c(inp.q), c(inp.k), c(inp.v), c(inp.g), c(inp.beta), pool, slots)
    assert binding.kda_check_device_error() == binding.KDA_ERR_TIMEOUT
    assert binding.kda_check_device_error() == binding.KDA_ERR_INVALID_ARG
    assert binding.kda_check_device_error() == binding.KDA_OK


# ------------------------------------------------------------------ debug input scan

def _prefill(d, **kw):
    return binding.kda_chunk_prefill(d.q, d.k, d.v, d.g, d.beta, d.state_in, d.cu_seqlens, **kw)


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
def test_debug_scan_reports_out_of_range_decay(monkeypatch, dtype, d):
    _drain()
    inp = kin.prefill_inputs(1, 300, 3, d, d, dtype, seed=43, state="normal")
    dd = inp.to("cuda")
    o_plain, s_plain = _prefill(dd)
    torch.cuda.synchronize()
    monkeypatch.setenv("KDA_DEBUG_CHECKS", "1")
    o_chk, s_chk = _prefill(dd)
    assert binding.kda_check_device_error() == binding.KDA_OK          # clean inputs
    # the scan changes no result
    assert torch.equal(o_plain, o_chk) and torch.equal(s_plain, s_chk)
    for bad in (0.25, -7.0, float("nan")):
        g = dd.g.clone()
        g[0, 123, 1, 5] = bad
        binding.kda_chunk_prefill(dd.q, dd.k, dd.v, g, dd.beta, dd.state_in, None)
        assert binding.kda_check_device_error() == binding.KDA_ERR_INPUT_RANGE, bad
        assert binding.kda_check_device_error() == binding.KDA_OK
    # off: nothing is scanned
    monkeypatch.setenv("KDA_DEBUG_CHECKS", "0")
    g = dd.g.clone()
    g[0, 7, 0, 0] = 1.0
    binding.kda_chunk_prefill(dd.q, dd.k, dd.v, g, dd.beta, dd.state_in, None)
    assert binding.kda_check_device_error() == binding.KDA_OK


def test_debug_scan_covers_sequences_only_and_decode(monkeypatch):
    _drain()
    monkeypatch.setenv("KDA_DEBUG_CHECKS", "1")
    lens = [100, 0, 100]
    inp = kin.prefill_inputs(1, 200, 2, 128, 128, "bf16", seed=44, state="normal", lengths=lens)
    inp.cu_seqlens[-1] = 170          # rows 170..199 belong to no sequence
    d = inp.to("cuda")
    g = d.g.clone()
    g[0, 190, 0, 3] = 3.0             # outside every sequence: not an input
    binding.kda_chunk_prefill(d.q, d.k, d.v, g, d.beta, d.state_in, d.cu_seqlens)
    assert binding.kda_check_device_error() == binding.KDA_OK
    g[0, 150, 1, 3] = 3.0             # inside sequence 2
    binding.kda_chunk_prefill(d.q, d.k, d.v, g, d.beta, d.state_in, d.cu_seqlens)
    assert binding.kda_check_device_error() == binding.KDA_ERR_INPUT_RANGE
    # gate logits are not log-decays: never reported
    binding.kda_chunk_prefill_ex(d.q, d.k, d.v, g * 10, d.beta, d.state_in, d.cu_seqlens,
                                 flags=binding.KDA_PREP_GATE_LOGIT)
    assert binding.kda_check_device_error() == binding.KDA_OK
    dec = kin.decode_inputs(1, 3, 2, 128, 128, "bf16", seed=45)
    S = dec.state.cuda()
    gd = dec.g[0].clone().cuda()
    binding.kda_decode_step(dec.q[0].cuda(), dec.k[0].cuda(), dec.v[0].cuda(), gd,
                            dec.beta[0].cuda(), S)
    assert binding.kda_check_device_error() == binding.KDA_OK
    gd[2, 1, 100] = 0.5
    binding.kda_decode_step(dec.q[0].cuda(), dec.k[0].cuda(), dec.v[0].cuda(), gd,
                            dec.beta[0].cuda(), S)
    assert binding.kda_check_device_error() == binding.KDA_ERR_INPUT_RANGE
    _drain()


# ------------------------------------------------------------------ malformed offsets

def test_out_of_order_offsets_give_the_same_sequences_on_every_path():
    """cu_seqlens = [0, 300, 200, 500]: every path clamps the offsets and raises each
    to the running maximum, so the sequences are rows [0, 300), [300, 300) (empty)
    and [300, 500), and no two CTAs write the same rows."""
    _drain()
    T, H = 500, 2
    inp = kin.prefill_inputs(1, T, H, 128, 128, "bf16", seed=46, state="normal",
                             lengths=[300, 0, 200])
    want = kin.prefill_inputs(1, T, H, 128, 128, "bf16", seed=46, state="normal",
                              lengths=[300, 0, 200])
    inp.cu_seqlens = torch.tensor([0, 300, 200, 500], dtype=torch.int32)
    ref = oracle_prefill(want)
    for dtype, tol in (("bf16", TOL_BF16), ("f32", TOL_F32)):
        d = inp.to("cuda")
        if dtype == "f32":   # the same values as fp32 inputs take the fp32 SIMT kernel
            for name in ("q", "k", "v", "g", "beta"):
                setattr(d, name, getattr(d, name).float())
        o, s = binding.kda_chunk_prefill(d.q, d.k, d.v, d.g, d.beta, d.state_in, d.cu_seqlens)
        torch.cuda.synchronize()
        assert binding.kda_check_device_error() == binding.KDA_OK
        got = gather_gpu(want, o, s, list(ref))
        compare_units(ref, got, tol, f"out-of-order {dtype}")
