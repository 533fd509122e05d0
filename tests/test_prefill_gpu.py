"""GPU parity: kda_chunk_prefill (through the C ABI) against the fp64 oracle.

Tolerance metric: max|delta| / rms(reference) over the compared tensor;
2e-2 for bf16 inputs with fp32 state, 1e-4 for the fp32 path.
"""
import numpy as np
import pytest
import torch

from _util import (TOL_BF16, TOL_F32, compare_all_units, compare_units, gather_gpu,
                   oracle_prefill, rel_err, to_np)
from kda_delta_rule_chunkwise_b200 import binding
from kda_delta_rule_chunkwise_b200 import inputs as kin

pytestmark = pytest.mark.gpu


def run(inp_cpu, **kw):
    d = inp_cpu.to("cuda")
    o, s = binding.kda_chunk_prefill(d.q, d.k, d.v, d.g, d.beta, d.state_in, d.cu_seqlens, **kw)
    torch.cuda.synchronize()
    assert binding.kda_check_device_error() == binding.KDA_OK
    return o, s


def check(inp, tol, heads=None, seqs=None, what=""):
    o, s = run(inp)
    ref = oracle_prefill(inp, heads=heads, seqs=seqs)
    got = gather_gpu(inp, o, s, list(ref))
    return compare_units(ref, got, tol, what)


# ------------------------------------------------------------------ fp32 path

def test_f32_tiny_config():
    """H=2, T=256, d=64, fp32, zero initial state (the reference-precision workload)."""
    inp = kin.workload_inputs("tiny_f32_h2_t256_d64", seed=0)
    check(inp, TOL_F32, what="tiny fp32")


@pytest.mark.parametrize("d,T,state", [(64, 131, "normal"), (128, 77, "normal"), (128, 1, "zero")])
def test_f32_ragged(d, T, state):
    inp = kin.prefill_inputs(2, T, 3, d, d, "f32", seed=1, state=state)
    check(inp, TOL_F32, what=f"fp32 d{d} T{T}")


def test_f32_varlen():
    lens = [0, 1, 64, 65, 100, 7]
    inp = kin.prefill_inputs(1, sum(lens), 2, 64, 64, "f32", seed=2, state="normal", lengths=lens)
    check(inp, TOL_F32, what="fp32 varlen")


# ------------------------------------------------------------------ bf16 path

@pytest.mark.parametrize("T", [64, 200, 1000])
@pytest.mark.parametrize("state", ["zero", "normal"])
def test_bf16_small(T, state):
    inp = kin.prefill_inputs(1, T, 4, 128, 128, "bf16", seed=3, state=state)
    check(inp, TOL_BF16, what=f"bf16 T{T} {state}")


def test_bf16_split_decay_many_chunks():
    inp = kin.prefill_inputs(2, 777, 3, 128, 128, "bf16", seed=4, decay="split", state="normal")
    check(inp, TOL_BF16, what="bf16 split decay")


def test_bf16_strong_decay_everywhere():
    """g = -5 exactly on every channel: the extreme of the rescaling range."""
    inp = kin.prefill_inputs(1, 300, 2, 128, 128, "bf16", seed=5, state="normal")
    inp.g.fill_(-5.0)
    check(inp, TOL_BF16, what="bf16 g=-5")


def test_bf16_no_decay():
    inp = kin.prefill_inputs(1, 300, 2, 128, 128, "bf16", seed=6, state="normal")
    inp.g.zero_()
    check(inp, TOL_BF16, what="bf16 g=0")


def test_bf16_decay_below_bound_is_clamped():
    inp = kin.prefill_inputs(1, 150, 2, 128, 128, "bf16", seed=7, state="normal")
    inp.g[..., ::7] = -11.0
    check(inp, TOL_BF16, what="bf16 g<-5")


def test_bf16_varlen_edge_lengths():
    lens = [0, 1, 63, 64, 65, 128, 130, 0, 5, 300]
    inp = kin.prefill_inputs(1, sum(lens), 3, 128, 128, "bf16", seed=8, state="normal",
                             lengths=lens)
    check(inp, TOL_BF16, what="bf16 varlen")


def test_bf16_many_short_sequences():
    """1500 packed sequences of 0..9 tokens (more sequences than the chunk table's
    1024 threads, many empty ones), 2 heads."""
    lens = kin.varlen_lengths(1500, 0, 9, seed=12)
    inp = kin.prefill_inputs(1, sum(lens), 2, 128, 128, "bf16", seed=12, state="normal",
                             lengths=lens)
    check(inp, TOL_BF16, what="bf16 1500 short sequences")


@pytest.mark.parametrize("H", [1, 37, 38, 48, 100, 150])
def test_bf16_slice_layouts(H):
    """(sequence, head) counts that select each form of the bf16 prefill: one launch
    for both phases (up to 37 units: H = 1, 37), and the two-kernel form with its
    three state-pass slice widths (32 columns up to 74 units: H = 38, 48; 64 up to
    148: H = 100; 128 beyond: H = 150)."""
    inp = kin.prefill_inputs(1, 130, H, 128, 128, "bf16", seed=9, state="normal")
    check(inp, TOL_BF16, heads=sorted({0, H // 2, H - 1}), what=f"bf16 H{H}")


def test_bf16_state_in_place():
    inp = kin.prefill_inputs(2, 150, 2, 128, 128, "bf16", seed=10, state="normal")
    d = inp.to("cuda")
    s = d.state_in.clone()
    o, s2 = binding.kda_chunk_prefill(d.q, d.k, d.v, d.g, d.beta, s, None, state_out=s)
    torch.cuda.synchronize()
    assert s2.data_ptr() == s.data_ptr()
    ref = oracle_prefill(inp)
    got = gather_gpu(inp, o, s, list(ref))
    compare_units(ref, got, TOL_BF16, "in-place state")


def test_bf16_no_state_out():
    inp = kin.prefill_inputs(1, 100, 2, 128, 128, "bf16", seed=11)
    d = inp.to("cuda")
    o, s = binding.kda_chunk_prefill(d.q, d.k, d.v, d.g, d.beta, None, None, want_state=False)
    torch.cuda.synchronize()
    assert s is None
    ref = oracle_prefill(inp)
    got = np.concatenate([to_np(o[0, :, h]).ravel() for h in range(2)])
    want = np.concatenate([ref[(0, h)][0].ravel() for h in range(2)])
    assert rel_err(got, want) <= TOL_BF16


def test_bf16_prefill_then_decode_matches_long_prefill():
    """Resumability: prefill(T1) then token-by-token decode == prefill(T1 + T2)."""
    T1, T2 = 130, 5
    inp = kin.prefill_inputs(1, T1 + T2, 2, 128, 128, "bf16", seed=12, state="normal")
    d = inp.to("cuda")
    o_full, s_full = binding.kda_chunk_prefill(d.q, d.k, d.v, d.g, d.beta, d.state_in, None)
    o1, s = binding.kda_chunk_prefill(d.q[:, :T1].contiguous(), d.k[:, :T1].contiguous(),
                                      d.v[:, :T1].contiguous(), d.g[:, :T1].contiguous(),
                                      d.beta[:, :T1].contiguous(), d.state_in, None)
    outs = [o1[0]]
    for t in range(T1, T1 + T2):
        outs.append(binding.kda_decode_step(d.q[:, t].contiguous(), d.k[:, t].contiguous(),
                                            d.v[:, t].contiguous(), d.g[:, t].contiguous(),
                                            d.beta[:, t].contiguous(), s)[None, 0])
    o_cat = torch.cat([x.reshape(-1, 2, 128) for x in outs], 0)
    assert rel_err(to_np(o_cat), to_np(o_full[0])) <= TOL_BF16
    assert rel_err(to_np(s), to_np(s_full)) <= TOL_BF16


# ------------------------------------------------------------------ full-size workloads

@pytest.mark.slow
def test_bf16_full_h32_t8192():
    """B=1, H=32, T=8192, d=128, zero state: every head against the oracle."""
    inp = kin.workload_inputs("prefill_h32_t8192_d128", seed=0, device="cuda")
    o, s = run(inp)
    compare_all_units(inp.to("cpu"), o, s, TOL_BF16, what="H32 T8192")


@pytest.mark.slow
def test_bf16_full_h32_t65536_split():
    """B=1, H=32, T=65536, split fast/slow decay, nonzero state: every head."""
    inp = kin.workload_inputs("prefill_h32_t65536_d128_split", seed=0, device="cuda")
    o, s = run(inp)
    compare_all_units(inp.to("cpu"), o, s, TOL_BF16, what="H32 T65536")


@pytest.mark.slow
def test_bf16_full_varlen_64_sequences():
    """64 packed sequences of 128..16384 tokens, H=32: all 64 x 32 (sequence, head) units."""
    inp = kin.workload_inputs("varlen_64seq_128to16384_h32_d128", seed=0, device="cuda")
    o, s = run(inp)
    compare_all_units(inp.to("cpu"), o, s, TOL_BF16, what="varlen 64 seqs")


def test_bf16_prefill_is_deterministic():
    """Two identical calls give the same bits (one issuing thread per accumulator)."""
    inp = kin.prefill_inputs(1, 1065, 8, 128, 128, "bf16", seed=33, decay="split", state="normal",
                             lengths=[300, 0, 700, 65])
    d = inp.to("cuda")
    o1, s1 = binding.kda_chunk_prefill(d.q, d.k, d.v, d.g, d.beta, d.state_in, d.cu_seqlens)
    o2, s2 = binding.kda_chunk_prefill(d.q, d.k, d.v, d.g, d.beta, d.state_in, d.cu_seqlens)
    torch.cuda.synchronize()
    rows = torch.cat([torch.arange(0, 300), torch.arange(300, 1000), torch.arange(1000, 1065)])
    assert torch.equal(o1[0, rows], o2[0, rows]) and torch.equal(s1, s2)


def test_bf16_d64_prefill_uses_the_simt_kernel():
    """bf16 inputs at d = 64 (no tensor-core path at that size) through the fp32 SIMT kernel."""
    inp = kin.prefill_inputs(2, 333, 3, 64, 64, "bf16", seed=34, state="normal")
    check(inp, TOL_BF16, what="bf16 d64")
