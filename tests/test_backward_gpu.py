"""GPU parity: kda_backward (through the C ABI) against the fp64 oracle's
reverse-mode gradients (oracle.backward, pinned by central differences of the
C recurrence in tests/test_oracle_pins.py).

Two paths.  fp32 inputs, and bf16 at d = 64, take the fp32 kernel that walks
the token recurrence from the exact input values: the fp32 bar (1e-4) applies
to every gradient.  bf16 at d = 128 goes through the chunked form on top of the
tensor-core forward (its fp16 per-chunk factors and fp32 chunk-start states,
then fp32 products per chunk): the bf16 bar (2e-2), as for the forward."""
import numpy as np
import pytest
import torch

import oracle
from _util import TOL_BF16, TOL_F32, rel_err, to_np
from kda_delta_rule_chunkwise_b200 import binding
from kda_delta_rule_chunkwise_b200 import inputs as kin

pytestmark = pytest.mark.gpu

NAMES = ("dq", "dk", "dv", "dg", "dbeta", "dstate_in")


def tol_for(inp):
    return TOL_BF16 if (inp.q.dtype == torch.bfloat16 and inp.dk == 128) else TOL_F32


def check(inp, seed, with_ds=True, rows=None):
    gen = torch.Generator().manual_seed(seed)
    N = inp.N
    do = torch.randn(inp.v.shape, generator=gen, dtype=torch.float32)
    ds = torch.randn((N, inp.H, inp.dk, inp.dv), generator=gen) if with_ds else None
    d = inp.to("cuda")
    got = binding.kda_backward(d.q, d.k, d.v, d.g, d.beta, d.state_in, d.cu_seqlens, do.cuda(),
                               None if ds is None else ds.cuda())
    torch.cuda.synchronize()
    assert binding.kda_check_device_error() == binding.KDA_OK
    cu = None if inp.cu_seqlens is None else inp.cu_seqlens.numpy().astype(np.int64)
    ref = oracle.backward(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.state_in, do, ds, cu_seqlens=cu)
    errs = {}
    for name, x, y in zip(NAMES, got, ref):
        gx = to_np(x)
        if rows is not None and name != "dstate_in":
            gx, y = gx[:, rows], y[:, rows]
        errs[name] = rel_err(gx, y)
    print({k_: f"{v_:.2e}" for k_, v_ in errs.items()})
    tol = tol_for(inp)
    for name, e in errs.items():
        assert e <= tol, f"{name}: {e:.3e} > {tol}"


@pytest.mark.parametrize("dtype,d", [("f32", 64), ("f32", 128), ("bf16", 128), ("bf16", 64)])
def test_backward_dense(dtype, d):
    inp = kin.prefill_inputs(2, 150, 2, d, d, dtype, seed=61, state="normal")
    check(inp, seed=1)


def test_backward_varlen_with_empty_and_ragged_sequences_no_state():
    inp = kin.prefill_inputs(1, 200, 2, 128, 128, "bf16", seed=62, decay="split",
                             lengths=[65, 0, 64, 71])
    check(inp, seed=2, with_ds=False)


def test_backward_clamped_decay_passes_no_gradient():
    inp = kin.prefill_inputs(1, 70, 1, 64, 64, "f32", seed=63, state="normal")
    inp.g[0, 10:20, 0, :8] = -7.0          # below the bound
    check(inp, seed=3)
    d = inp.to("cuda")
    grads = binding.kda_backward(d.q, d.k, d.v, d.g, d.beta, d.state_in, None,
                                 torch.ones(inp.v.shape, device="cuda"))
    assert not grads[3][0, 10:20, 0, :8].any()


@pytest.mark.parametrize("B,H", [(1, 40), (2, 40)])
def test_backward_column_slices(B, H):
    """40 units: the value columns go to two CTAs per (sequence, head) and the
    cross-column sums through partials; 80 units: one CTA, direct writes."""
    inp = kin.prefill_inputs(B, 70, H, 64, 64, "bf16", seed=64 + B, state="normal")
    check(inp, seed=4)


def test_backward_column_slices_are_deterministic():
    inp = kin.prefill_inputs(1, 130, 3, 128, 128, "bf16", seed=65, state="normal").to("cuda")
    do = torch.randn(inp.v.shape, generator=torch.Generator().manual_seed(5)).cuda()
    a = binding.kda_backward(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.state_in, None, do)
    b = binding.kda_backward(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.state_in, None, do)
    torch.cuda.synchronize()
    for name, x, y in zip(NAMES, a, b):
        assert torch.equal(x, y), name


def test_backward_full_size_sampled_heads():
    """The configuration the benchmark times (one sequence, T = 8192, H = 32, bf16,
    the chunked path): all heads run on the GPU, heads 0 and 31 are checked against
    the oracle (heads are independent, so this is exact)."""
    inp = kin.workload_inputs("prefill_h32_t8192_d128", seed=7)
    do = torch.randn(inp.v.shape, generator=torch.Generator().manual_seed(8), dtype=torch.float32)
    d = inp.to("cuda")
    got = binding.kda_backward(d.q, d.k, d.v, d.g, d.beta, d.state_in, None, do.cuda())
    torch.cuda.synchronize()
    assert binding.kda_check_device_error() == binding.KDA_OK
    heads = [0, 31]
    pick = lambda x: x[:, :, heads].contiguous()
    s0 = None if inp.state_in is None else inp.state_in[:, heads].contiguous()
    ref = oracle.backward(pick(inp.q), pick(inp.k), pick(inp.v), pick(inp.g), pick(inp.beta), s0,
                          pick(do), None)
    errs = {}
    for name, x, y in zip(NAMES, got, ref):
        if x is None:
            continue
        gx = to_np(x[:, heads] if name == "dstate_in" else x[:, :, heads])
        errs[name] = rel_err(gx, y)
    print({k_: f"{v_:.2e}" for k_, v_ in errs.items()})
    for name, e in errs.items():
        assert e <= TOL_BF16, f"{name}: {e:.3e}"


def test_backward_many_units_d128():
    """80 (sequence, head) units at d = 128: one CTA of 256 threads per unit over
    all 128 value columns (the unsliced kernel)."""
    inp = kin.prefill_inputs(2, 70, 40, 128, 128, "bf16", seed=66, state="normal")
    check(inp, seed=6)


def test_backward_many_short_sequences():
    """300 packed sequences of 0..9 tokens (many empty ones), 2 heads."""
    lengths = kin.varlen_lengths(300, 0, 9, seed=67)
    inp = kin.prefill_inputs(1, sum(lengths), 2, 64, 64, "f32", seed=67, state="normal",
                             lengths=lengths)
    check(inp, seed=7)


def test_autograd_wrapper_matches_the_backward_call():
    """KDAPrefill through torch.autograd gives kda_backward's gradients exactly, and
    they match the oracle."""
    inp = kin.prefill_inputs(2, 90, 2, 64, 64, "f32", seed=68, state="normal").to("cuda")
    leaves = [x.clone().requires_grad_(True) for x in (inp.q, inp.k, inp.v, inp.g, inp.beta,
                                                       inp.state_in)]
    o, s = binding.kda_prefill_autograd(*leaves)
    gen = torch.Generator(device="cuda").manual_seed(9)
    wo = torch.randn(o.shape, generator=gen, device="cuda")
    ws = torch.randn(s.shape, generator=gen, device="cuda")
    ((o * wo).sum() + (s * ws).sum()).backward()
    direct = binding.kda_backward(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.state_in, None, wo, ws)
    torch.cuda.synchronize()
    for name, leaf, ref in zip(NAMES, leaves, direct):
        assert torch.equal(leaf.grad, ref), name
    c = inp.to("cpu")
    want = oracle.backward(c.q, c.k, c.v, c.g, c.beta, c.state_in, wo.cpu(), ws.cpu())
    for name, leaf, y in zip(NAMES, leaves, want):
        assert rel_err(to_np(leaf.grad), y) <= TOL_F32, name


@pytest.mark.parametrize("decay,state,T", [("split", "normal", 1000), ("uniform", "zero", 333)])
def test_backward_chunked_path_decays(decay, state, T):
    """The chunked path on the strong/weak split decay with a state, and on a ragged
    length without one, both heads against the oracle."""
    inp = kin.prefill_inputs(1, T, 2, 128, 128, "bf16", seed=69, decay=decay, state=state)
    check(inp, seed=10)


def test_backward_chunked_path_clamp_and_strong_decay():
    """g = -5 on some channels, below the clamp on others (no gradient there)."""
    inp = kin.prefill_inputs(1, 200, 2, 128, 128, "bf16", seed=70, state="normal")
    inp.g[0, :, :, :16] = -5.0
    inp.g[0, 40:90, 1, 20:30] = -8.0
    check(inp, seed=11)
    d = inp.to("cuda")
    grads = binding.kda_backward(d.q, d.k, d.v, d.g, d.beta, d.state_in, None,
                                 torch.ones(inp.v.shape, device="cuda"))
    torch.cuda.synchronize()
    assert not grads[3][0, 40:90, 1, 20:30].any()


def test_backward_chunked_path_packed_sequences():
    """Packed sequences with empty, one-token and chunk-boundary lengths, 3 heads."""
    lens = [0, 1, 63, 64, 65, 130, 0, 7]
    inp = kin.prefill_inputs(1, sum(lens), 3, 128, 128, "bf16", seed=71, state="normal",
                             lengths=lens)
    check(inp, seed=12)


def test_backward_chunked_path_strongest_decay_everywhere():
    """g = -5 on every channel: the decay-rescaled factors reach e^80 inside each
    16-row block, the edge of their range."""
    inp = kin.prefill_inputs(1, 150, 2, 128, 128, "bf16", seed=72, state="normal")
    inp.g.fill_(-5.0)
    check(inp, seed=13)

