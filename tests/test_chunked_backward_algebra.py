"""CPU: the chunked (WY-form) backward equals the oracle's gradients.

The per-chunk adjoint in _chunked_backward_emulation is what a chunk-parallel
tensor-core backward evaluates (a reverse pass over chunk states, then every
chunk's input gradients independently).  The WY-slot form splits the same adjoint into a chain that needs only the
forward's per-chunk factors (T, R, W, P, Khat, Gamma_L) and a pull-back of
those factors' gradients to q, k, g, beta that needs no state.  Both are pinned
here against oracle.backward
(autograd over the token recurrence, fp64) for several chunk sizes, ragged
tails and decays below the clamp, so the algebra is exact before any kernel
follows it.
"""
import numpy as np
import pytest

import oracle
from _chunked_backward_emulation import backward as chunked_backward, wy_backward
from _util import rel_err
from kda_delta_rule_chunkwise_b200 import inputs as kin


@pytest.mark.parametrize("form", ["chunk", "wy_slot"])
@pytest.mark.parametrize("T,d,C", [(150, 16, 64), (130, 32, 64), (64, 8, 16), (77, 8, 10), (5, 4, 64)])
def test_chunked_backward_equals_the_oracle(T, d, C, form):
    inp = kin.prefill_inputs(1, T, 1, d, d, "f32", seed=3, state="normal")
    f64 = lambda x: x.double().numpy()
    q, k, v, g, b = (f64(x[0, :, 0]) for x in (inp.q, inp.k, inp.v, inp.g, inp.beta))
    g[::7, ::3] = -6.0                 # below the clamp: no gradient there
    S0 = f64(inp.state_in[0, 0])
    rng = np.random.default_rng(T * 100 + d)
    dout, dS_final = rng.normal(size=(T, d)), rng.normal(size=(d, d))
    got = (chunked_backward if form == "chunk" else wy_backward)(q, k, v, g, b, S0, dout, dS_final, C=C)
    want = oracle.backward(q[None, :, None], k[None, :, None], v[None, :, None], g[None, :, None],
                           b[None, :, None], S0[None, None], dout[None, :, None], dS_final[None, None])
    for name, x, w in zip(["dq", "dk", "dv", "dg", "dbeta", "dS0"], got, want):
        assert rel_err(x, np.reshape(w, x.shape)) < 1e-10, name


def test_upper_triangles_of_dR_and_dT_reach_no_output():
    """T, R, X and Aqk are lower triangular, so only the lower parts (diagonal
    included) of dR' = dR - dP (K Gamma)^T and dT' reach dAkk, dAqk and dbeta.
    The chunked backward leaves the 16 x 16 blocks above the diagonal of dT, dR
    and of those two products at 0; here large noise in every strictly upper
    entry must leave all gradients unchanged."""
    inp = kin.prefill_inputs(1, 150, 1, 16, 16, "f32", seed=5, state="normal")
    f64 = lambda x: x.double().numpy()
    q, k, v, g, b = (f64(x[0, :, 0]) for x in (inp.q, inp.k, inp.v, inp.g, inp.beta))
    S0 = f64(inp.state_in[0, 0])
    rng = np.random.default_rng(11)
    dout, dS_final = rng.normal(size=(150, 16)), rng.normal(size=(16, 16))
    want = wy_backward(q, k, v, g, b, S0, dout, dS_final, C=64)
    noise = np.random.default_rng(12)
    got = wy_backward(q, k, v, g, b, S0, dout, dS_final, C=64, upper=lambda shp: 1e3 * noise.normal(size=shp))
    for name, x, w in zip(["dq", "dk", "dv", "dg", "dbeta", "dS0"], got, want):
        assert rel_err(x, w) < 1e-10, name
