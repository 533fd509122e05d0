"""GPU parity: kda_decode_step (through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from _util import TOL_BF16, TOL_F32, rel_err, to_np
from kda_delta_rule_chunkwise_b200 import binding
from kda_delta_rule_chunkwise_b200 import inputs as kin

pytestmark = pytest.mark.gpu


def run_steps(inp, steps, n_sel=None):
    """Run `steps` decode steps on the GPU and in the oracle; compare all outputs/states."""
    S = inp.state.clone().cuda()
    S_ref = inp.state.double().numpy()
    if n_sel is not None:
        S_ref = S_ref[n_sel]
    errs_o, got_o, want_o = [], [], []
    for t in range(steps):
        cu = lambda x: x[t].contiguous().cuda()
        o = binding.kda_decode_step(cu(inp.q), cu(inp.k), cu(inp.v), cu(inp.g), cu(inp.beta), S)
        sel = (lambda x: x[t]) if n_sel is None else (lambda x: x[t][n_sel])
        o_ref, S_ref = oracle.decode_step(sel(inp.q), sel(inp.k), sel(inp.v), sel(inp.g),
                                          sel(inp.beta), S_ref)
        og = to_np(o) if n_sel is None else to_np(o[n_sel])
        got_o.append(og)
        want_o.append(o_ref)
    torch.cuda.synchronize()
    assert binding.kda_check_device_error() == binding.KDA_OK
    Sg = to_np(S) if n_sel is None else to_np(S[n_sel])
    return np.stack(got_o), np.stack(want_o), Sg, S_ref


@pytest.mark.parametrize("dtype,d,tol", [("bf16", 128, TOL_BF16), ("bf16", 64, TOL_BF16),
                                         ("f32", 128, TOL_F32), ("f32", 64, TOL_F32)])
def test_decode_small(dtype, d, tol):
    inp = kin.decode_inputs(6, 5, 3, d, d, dtype, seed=1)
    go, wo, gs, ws = run_steps(inp, 6)
    assert rel_err(go, wo) <= tol
    assert rel_err(gs, ws) <= tol


def test_decode_beta_zero_g_zero_is_identity_on_state():
    inp = kin.decode_inputs(1, 4, 2, 128, 128, "f32", seed=2)
    inp.beta.zero_()
    inp.g.zero_()
    S0 = inp.state.clone()
    go, wo, gs, ws = run_steps(inp, 1)
    np.testing.assert_array_equal(gs, S0.double().numpy())
    assert rel_err(go, wo) <= TOL_F32


@pytest.mark.slow
def test_decode_full_n256_h32_sampled():
    """N=256 sequences, H=32, d=128, bf16: 20 consecutive steps on the full state,
    oracle on a sample of 8 sequences (all 32 heads)."""
    inp = kin.decode_inputs(20, 256, 32, 128, 128, "bf16", seed=0)
    sel = np.array([0, 1, 77, 128, 200, 253, 254, 255])
    go, wo, gs, ws = run_steps(inp, 20, n_sel=sel)
    assert rel_err(go, wo) <= TOL_BF16
    assert rel_err(gs, ws) <= TOL_BF16
