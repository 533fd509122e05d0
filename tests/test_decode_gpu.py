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
def test_decode_full_n256_h32_1000_steps():
    """The decode workload as specified: N=256 sequences, H=32, d=128, bf16, 1000
    consecutive steps in place on the full state, each step with fresh inputs.  The
    oracle follows 8 of the sequences (all 32 heads) through all 1000 steps: every
    step's output and their final states are compared."""
    steps = 1000
    inp = kin.decode_inputs(steps, 256, 32, 128, 128, "bf16", seed=0, device="cuda")
    sel = torch.tensor([0, 1, 77, 128, 200, 253, 254, 255], device="cuda")
    S = inp.state.clone()
    o = torch.empty((256, 32, 128), dtype=torch.float32, device="cuda")
    o_sel = torch.empty((steps, len(sel), 32, 128), dtype=torch.float32, device="cuda")
    for t in range(steps):
        binding.kda_decode_step(inp.q[t], inp.k[t], inp.v[t], inp.g[t], inp.beta[t], S, o=o)
        o_sel[t] = o.index_select(0, sel)
    torch.cuda.synchronize()
    assert binding.kda_check_device_error() == binding.KDA_OK
    assert torch.isfinite(S).all()
    pick = lambda x: x.index_select(1, sel).cpu()
    q, k, v, g, b = (pick(x) for x in (inp.q, inp.k, inp.v, inp.g, inp.beta))
    S_ref = inp.state.index_select(0, sel).double().cpu().numpy()
    want = np.empty((steps, len(sel), 32, 128))
    for t in range(steps):
        want[t], S_ref = oracle.decode_step(q[t], k[t], v[t], g[t], b[t], S_ref)
    eo = rel_err(to_np(o_sel), want)
    es = rel_err(to_np(S.index_select(0, sel)), S_ref)
    print(f"decode 1000 steps, 8 x 32 units: output error {eo:.3e}, final-state error {es:.3e}")
    assert eo <= TOL_BF16
    assert es <= TOL_BF16


# ---------------------------------------------------------------- pooled (indexed) state

def _pool_case(P, N, H, d, dtype, seed):
    gen = np.random.default_rng(seed)
    inp = kin.decode_inputs(3, N, H, d, d, dtype, seed=seed)
    pool = torch.randn((P, H, d, d), generator=torch.Generator().manual_seed(seed)) * 0.1
    slots = torch.as_tensor(gen.permutation(P)[:N].astype(np.int32))
    return inp, pool, slots


@pytest.mark.parametrize("dtype,d,tol", [("bf16", 128, TOL_BF16), ("f32", 64, TOL_F32)])
def test_decode_indexed_matches_oracle_and_leaves_other_entries(dtype, d, tol):
    P, N, H = 24, 10, 3
    inp, pool, slots = _pool_case(P, N, H, d, dtype, seed=5)
    pool_g = pool.clone().cuda()
    slots_g = slots.cuda()
    S_ref = pool.double().numpy()[slots.numpy()]
    for t in range(3):
        cu = lambda x: x[t].contiguous().cuda()
        o = binding.kda_decode_step_indexed(cu(inp.q), cu(inp.k), cu(inp.v), cu(inp.g),
                                            cu(inp.beta), pool_g, slots_g)
        o_ref, S_ref = oracle.decode_step(inp.q[t], inp.k[t], inp.v[t], inp.g[t], inp.beta[t],
                                          S_ref)
        assert rel_err(to_np(o), o_ref) <= tol, f"step {t}: output"
    assert binding.kda_check_device_error() == binding.KDA_OK
    got = to_np(pool_g)
    assert rel_err(got[slots.numpy()], S_ref) <= tol, "touched entries"
    untouched = np.setdiff1d(np.arange(P), slots.numpy())
    np.testing.assert_array_equal(got[untouched], pool.double().numpy()[untouched])


def test_decode_indexed_identity_slots_equal_the_dense_step():
    """slots = 0..N-1 over a pool of exactly N entries is the dense step, bit for bit."""
    inp = kin.decode_inputs(1, 6, 4, 128, 128, "bf16", seed=9)
    dense = inp.state.clone().cuda()
    pooled = inp.state.clone().cuda()
    cu = lambda x: x[0].contiguous().cuda()
    o1 = binding.kda_decode_step(cu(inp.q), cu(inp.k), cu(inp.v), cu(inp.g), cu(inp.beta), dense)
    o2 = binding.kda_decode_step_indexed(cu(inp.q), cu(inp.k), cu(inp.v), cu(inp.g), cu(inp.beta),
                                         pooled, torch.arange(6, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(dense, pooled)


def test_decode_indexed_out_of_range_slot_is_skipped_and_reported():
    P, N, H = 8, 4, 2
    inp, pool, slots = _pool_case(P, N, H, 128, "bf16", seed=6)
    slots[2] = P          # outside the pool: this request is skipped on the device
    pool_g = pool.clone().cuda()
    o = torch.full((N, H, 128), float("nan"), device="cuda")
    cu = lambda x: x[0].contiguous().cuda()
    binding.kda_decode_step_indexed(cu(inp.q), cu(inp.k), cu(inp.v), cu(inp.g), cu(inp.beta),
                                    pool_g, slots.cuda(), o=o)
    assert binding.kda_check_device_error() == binding.KDA_ERR_INVALID_ARG
    assert binding.kda_check_device_error() == binding.KDA_OK      # cleared
    ok = [0, 1, 3]
    o_ref, S_ref = oracle.decode_step(inp.q[0][ok], inp.k[0][ok], inp.v[0][ok], inp.g[0][ok],
                                      inp.beta[0][ok], pool.double().numpy()[slots.numpy()[ok]])
    assert rel_err(to_np(o)[ok], o_ref) <= TOL_BF16
    assert torch.isnan(o[2]).all()                                  # not written
    got = to_np(pool_g)
    assert rel_err(got[slots.numpy()[ok]], S_ref) <= TOL_BF16
    untouched = np.setdiff1d(np.arange(P), slots.numpy()[ok])
    np.testing.assert_array_equal(got[untouched], pool.double().numpy()[untouched])
