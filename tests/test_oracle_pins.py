"""Pins for the fp64 oracle: each check ties it to something other than itself.

The pages print no worked example, so the pins are mathematics:
  * an independently written chunked closed form (numpy, any chunk size),
  * the recurrence as a literal product of dense matrices,
  * beta = 0: pure per-channel decay, S_t = Diag(exp G_t) S_0,
  * g = 0, beta = 1: delta-rule overwrite of orthonormal keys, S^T k_j = v_j,
  * a scalar (dk = dv = 1) case evaluated by hand with exact rationals,
  * linearity in (S_0, V), sequence isolation in packed batches,
  * prefill then token-by-token decode = one long prefill,
  * the lower bound g >= -5 (values below behave as -5).
"""
import numpy as np
import pytest
import torch

import oracle
from _closed_form import chunked, product_form_unit
from kda_delta_rule_chunkwise_b200 import inputs as kin

TOL = 1e-11


def _rand(B, T, H, dk, dv, seed, state=True, decay="uniform"):
    inp = kin.prefill_inputs(B, T, H, dk, dv, "f32", seed=seed, decay=decay,
                             state="normal" if state else "zero")
    f = lambda x: None if x is None else x.double().numpy()
    return f(inp.q), f(inp.k), f(inp.v), f(inp.g), f(inp.beta), f(inp.state_in)


def _rel(a, b):
    return np.max(np.abs(a - b)) / max(1e-300, np.sqrt(np.mean(b * b)))


@pytest.mark.parametrize("C", [1, 2, 3, 16, 64])
def test_chunked_closed_form(C):
    q, k, v, g, b, s0 = _rand(2, 83, 2, 8, 6, seed=1)
    o, s = oracle.recurrence(q, k, v, g, b, s0)
    cu = np.arange(3) * 83
    rs = lambda x: x.reshape((-1,) + x.shape[2:])
    oc, sc = chunked(rs(q), rs(k), rs(v), rs(g), rs(b), s0, cu, C)
    assert _rel(o.reshape(oc.shape), oc) < TOL
    assert _rel(s, sc) < TOL


def test_chunked_closed_form_strong_decay_dk64():
    """Fast-decay channels (g near -5) over a full 64-token chunk."""
    q, k, v, g, b, s0 = _rand(1, 150, 1, 16, 16, seed=2, decay="split")
    o, s = oracle.recurrence(q, k, v, g, b, s0)
    rs = lambda x: x.reshape((-1,) + x.shape[2:])
    oc, sc = chunked(rs(q), rs(k), rs(v), rs(g), rs(b), s0, np.array([0, 150]), 64)
    assert _rel(o.reshape(oc.shape), oc) < TOL
    assert _rel(s, sc) < TOL


def test_literal_product_form():
    q, k, v, g, b, s0 = _rand(1, 40, 3, 5, 7, seed=3)
    o, s = oracle.recurrence(q, k, v, g, b, s0)
    for h in range(3):
        O, S = product_form_unit(q[0, :, h], k[0, :, h], v[0, :, h], g[0, :, h],
                                 b[0, :, h], s0[0, h])
        assert _rel(o[0, :, h], O) < TOL
        assert _rel(s[0, h], S) < TOL


def test_beta_zero_is_pure_decay():
    q, k, v, g, b, s0 = _rand(1, 50, 2, 6, 4, seed=4)
    b = np.zeros_like(b)
    o, s = oracle.recurrence(q, k, v, g, b, s0)
    G = np.cumsum(g[0], axis=0)  # [T, H, dk], no clamping needed (g > -5)
    for h in range(2):
        for t in range(50):
            St = np.exp(G[t, h])[:, None] * s0[0, h]
            np.testing.assert_allclose(o[0, t, h], St.T @ q[0, t, h], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(s[0, h], np.exp(G[-1, h])[:, None] * s0[0, h],
                                   rtol=1e-12, atol=1e-300)


def test_beta_zero_g_zero_keeps_state():
    q, k, v, g, b, s0 = _rand(1, 9, 1, 4, 4, seed=5)
    o, s = oracle.recurrence(q, k, v, np.zeros_like(g), np.zeros_like(b), s0)
    np.testing.assert_array_equal(s, s0)


def test_overwrite_orthonormal_keys():
    """g = 0, beta = 1: writing orthonormal keys in turn stores exactly v_j."""
    rng = np.random.default_rng(6)
    dk, dv, m = 8, 5, 6
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Qm[:, :m].T                           # m orthonormal rows
    k = keys[None, :, None, :]
    v = rng.standard_normal((1, m, 1, dv))
    q = keys[None, :, None, :].copy()            # read back with the key itself
    g = np.zeros((1, m, 1, dk))
    b = np.ones((1, m, 1))
    o, s = oracle.recurrence(q, k, v, g, b, None)
    S = s[0, 0]
    for j in range(m):
        np.testing.assert_allclose(S.T @ keys[j], v[0, j, 0], atol=1e-12)
        # each step's readout with q_t = k_t returns v_t (S_t^T k_t = v_t)
        np.testing.assert_allclose(o[0, j, 0], v[0, j, 0], atol=1e-12)


def test_overwrite_erases_previous_value():
    """beta = 1, unit k, g = 0: a second write along the same key replaces v."""
    dk, dv = 4, 3
    kk = np.array([0.5, 0.5, 0.5, 0.5])
    k = np.stack([kk, kk])[None, :, None, :]
    v = np.array([[1.0, 2.0, 3.0], [-4.0, 0.5, 7.0]])[None, :, None, :]
    o, s = oracle.recurrence(k, k, v, np.zeros((1, 2, 1, dk)), np.ones((1, 2, 1)), None)
    np.testing.assert_allclose(s[0, 0].T @ kk, v[0, 1, 0], atol=1e-14)
    np.testing.assert_allclose(o[0, 1, 0], v[0, 1, 0], atol=1e-14)


def test_scalar_case_by_hand():
    """dk = dv = 1 with exact rationals; worked by hand from the recurrence.

    s_t = (1 - beta_t k_t^2) a_t s_{t-1} + beta_t k_t v_t,  o_t = s_t q_t.
    t=1: k=1, beta=1/2, a=1, v=2, s0=4:  s1 = (1/2)(4) + 1   = 3
    t=2: k=1, beta=1/4, a=1, v=8:        s2 = (3/4)(3) + 2   = 17/4
    t=3: k=1/2, beta=1, a=1, v=-2:       s3 = (3/4)(17/4) - 1 = 35/16
    readout q = (1, 2, -1/2): o = (3, 17/2, -35/32).
    """
    k = np.array([1.0, 1.0, 0.5]).reshape(1, 3, 1, 1)
    b = np.array([0.5, 0.25, 1.0]).reshape(1, 3, 1)
    v = np.array([2.0, 8.0, -2.0]).reshape(1, 3, 1, 1)
    q = np.array([1.0, 2.0, -0.5]).reshape(1, 3, 1, 1)
    g = np.zeros((1, 3, 1, 1))
    s0 = np.array([[[[4.0]]]])
    o, s = oracle.recurrence(q, k, v, g, b, s0)
    assert o.ravel().tolist() == [3.0, 17.0 / 2.0, -35.0 / 32.0]
    assert s.ravel().tolist() == [35.0 / 16.0]


def test_scalar_case_with_decay_closed_form():
    """dk = dv = 1, decay on: s_T = prod(m_t) s0 + sum_t prod_{u>t}(m_u) beta_t k_t v_t,
    with m_t = (1 - beta_t k_t^2) exp(g_t) (expanded by hand, not the loop)."""
    rng = np.random.default_rng(7)
    T = 5
    k = rng.uniform(-1, 1, T)
    b = rng.uniform(0, 1, T)
    v = rng.standard_normal(T)
    g = rng.uniform(-5, 0, T)
    s0 = 0.3
    m = (1 - b * k * k) * np.exp(g)
    expect = np.prod(m) * s0 + sum(np.prod(m[t + 1:]) * b[t] * k[t] * v[t] for t in range(T))
    _, s = oracle.recurrence(np.ones((1, T, 1, 1)), k.reshape(1, T, 1, 1),
                             v.reshape(1, T, 1, 1), g.reshape(1, T, 1, 1),
                             b.reshape(1, T, 1), np.array([[[[s0]]]]))
    assert abs(s.item() - expect) < 1e-14


def test_superposition():
    q, k, v, g, b, s0 = _rand(1, 30, 2, 6, 5, seed=8)
    _, _, v2, _, _, s02 = _rand(1, 30, 2, 6, 5, seed=9)
    a1, a2 = 0.7, -1.9
    o1, s1 = oracle.recurrence(q, k, v, g, b, s0)
    o2, s2 = oracle.recurrence(q, k, v2, g, b, s02)
    o3, s3 = oracle.recurrence(q, k, a1 * v + a2 * v2, g, b, a1 * s0 + a2 * s02)
    assert _rel(o3, a1 * o1 + a2 * o2) < TOL
    assert _rel(s3, a1 * s1 + a2 * s2) < TOL


@pytest.mark.parametrize("T1", [0, 1, 63, 64, 65, 99])
def test_prefill_then_decode_equals_long_prefill(T1):
    T = 100
    q, k, v, g, b, s0 = _rand(1, T, 2, 6, 5, seed=10)
    o_full, s_full = oracle.recurrence(q, k, v, g, b, s0)
    o_a, s = oracle.recurrence(q[:, :T1], k[:, :T1], v[:, :T1], g[:, :T1], b[:, :T1], s0)
    outs = [o_a[0]]
    for t in range(T1, T):
        ot, s = oracle.decode_step(q[:, t], k[:, t], v[:, t], g[:, t], b[:, t], s)
        outs.append(ot)
    o_cat = np.concatenate([x.reshape(-1, 2, 5) for x in outs], axis=0)
    assert _rel(o_cat, o_full[0]) < TOL
    assert _rel(s, s_full) < TOL


def test_packed_sequences_are_isolated():
    lens = [5, 0, 70, 1, 33]
    inp = kin.prefill_inputs(1, sum(lens), 2, 4, 3, "f32", seed=11,
                             state="normal", lengths=lens)
    f = lambda x: x.double().numpy()
    o, s = oracle.recurrence(f(inp.q), f(inp.k), f(inp.v), f(inp.g), f(inp.beta),
                             f(inp.state_in), inp.cu_seqlens.numpy())
    cu = inp.cu_seqlens.numpy()
    for n in range(len(lens)):
        a, e = cu[n], cu[n + 1]
        on, sn = oracle.recurrence(f(inp.q)[:, a:e], f(inp.k)[:, a:e], f(inp.v)[:, a:e],
                                   f(inp.g)[:, a:e], f(inp.beta)[:, a:e],
                                   f(inp.state_in)[n:n + 1])
        np.testing.assert_array_equal(o[:, a:e], on)
        np.testing.assert_array_equal(s[n], sn[0])
    # a zero-length sequence passes its state through unchanged
    np.testing.assert_array_equal(s[1], f(inp.state_in)[1])


def test_decay_lower_bound():
    """log-decay below -5 acts as -5 (the library's reading of the bound)."""
    q, k, v, g, b, s0 = _rand(1, 20, 1, 4, 4, seed=12)
    g_low = g.copy()
    g_low[0, ::3, 0, 1] = -9.0
    g_at = g.copy()
    g_at[0, ::3, 0, 1] = -5.0
    o1, s1 = oracle.recurrence(q, k, v, g_low, b, s0)
    o2, s2 = oracle.recurrence(q, k, v, g_at, b, s0)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(s1, s2)
    # and it does change the result relative to the unclamped -9 product form
    O, S = product_form_unit(q[0, :, 0], k[0, :, 0], v[0, :, 0], g_at[0, :, 0],
                             b[0, :, 0], s0[0, 0])
    assert _rel(s1[0, 0], S) < TOL


def test_bf16_inputs_are_taken_exactly():
    inp = kin.prefill_inputs(1, 17, 1, 8, 8, "bf16", seed=13, state="normal")
    o1, s1 = oracle.recurrence(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.state_in)
    f = lambda x: x.float().double().numpy()
    o2, s2 = oracle.recurrence(f(inp.q), f(inp.k), f(inp.v), f(inp.g), f(inp.beta),
                               inp.state_in.double().numpy())
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(s1, s2)


def test_thread_count_does_not_change_bits():
    q, k, v, g, b, s0 = _rand(3, 40, 4, 8, 8, seed=14)
    r1 = oracle.recurrence(q, k, v, g, b, s0, n_threads=1)
    r8 = oracle.recurrence(q, k, v, g, b, s0, n_threads=8)
    np.testing.assert_array_equal(r1[0], r8[0])
    np.testing.assert_array_equal(r1[1], r8[1])


# ---------------------------------------------------------------- input preprocessing

def test_preprocess_gate_is_minus_five_sigmoid():
    x = np.array([[-40.0, -3.0, 0.0, 3.0, 40.0]])
    _, _, g = oracle.preprocess(np.ones((1, 2)), np.ones((1, 2)), x, oracle.GATE_LOGIT)
    assert g[0, 2] == -2.5                                   # sigmoid(0) = 1/2
    assert np.all(g <= 0) and np.all(g >= -5)                 # inside the bound
    assert np.all(np.diff(g[0]) < 0)                          # more decay for larger logits
    np.testing.assert_allclose(g + g[:, ::-1], -5.0, rtol=0, atol=1e-15)   # s(x) + s(-x) = 1
    np.testing.assert_allclose(g[0, 3], -5.0 / (1.0 + np.exp(-3.0)), rtol=1e-15)


def test_preprocess_l2norm_gives_unit_rows_and_keeps_zero_rows():
    rng = np.random.default_rng(0)
    q = rng.normal(size=(4, 3, 128)) * 7.0
    k = rng.normal(size=(4, 3, 128))
    k[1, 2] = 0.0
    qn, kn, g = oracle.preprocess(q, k, np.zeros((4, 3, 128)), oracle.L2NORM_QK)
    np.testing.assert_allclose(np.linalg.norm(qn, axis=-1), 1.0, rtol=1e-14)
    assert not kn[1, 2].any()
    np.testing.assert_allclose(qn * np.linalg.norm(q, axis=-1, keepdims=True), q, rtol=1e-13)
    assert not g.any()                                        # gate untouched without the flag


def test_preprocess_then_recurrence_equals_recurrence_on_preprocessed_inputs():
    """Scale invariance: scaling q by c > 0 changes nothing once q is normalised."""
    rng = np.random.default_rng(1)
    T, H, d = 37, 2, 8
    q, k, v = (rng.normal(size=(1, T, H, d)) for _ in range(3))
    x = rng.normal(size=(1, T, H, d))
    b = 1 / (1 + np.exp(-rng.normal(size=(1, T, H))))
    flags = oracle.GATE_LOGIT | oracle.L2NORM_QK
    out1 = oracle.recurrence(*oracle.preprocess(q, k, x, flags)[:2], v,
                             oracle.preprocess(q, k, x, flags)[2], b)
    out2 = oracle.recurrence(*oracle.preprocess(3.0 * q, 0.5 * k, x, flags)[:2], v,
                             oracle.preprocess(3.0 * q, 0.5 * k, x, flags)[2], b)
    np.testing.assert_allclose(out1[0], out2[0], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(out1[1], out2[1], rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- backward

def _loss(q, k, v, g, b, s0, do, ds, cu=None):
    o, s = oracle.recurrence(q, k, v, g, b, state_in=s0, cu_seqlens=cu)
    return float(np.sum(o * do) + np.sum(s * ds))


def test_backward_matches_central_differences_of_the_c_oracle():
    """Every gradient entry against (L(x+e) - L(x-e)) / 2e, L evaluated by the C
    recurrence (independent of the autograd graph); includes g below -5."""
    rng = np.random.default_rng(11)
    B, T, H, d = 1, 6, 2, 3
    q, k, v = (rng.normal(size=(B, T, H, d)) for _ in range(3))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    g = -5.0 / (1.0 + np.exp(-rng.normal(size=(B, T, H, d))))
    g[0, 2, 1, 0] = -6.5                                      # clamped: no gradient
    b = 1 / (1 + np.exp(-rng.normal(size=(B, T, H))))
    s0 = rng.normal(size=(B, H, d, d)) * 0.3
    do = rng.normal(size=(B, T, H, d))
    ds = rng.normal(size=(B, H, d, d))
    grads = oracle.backward(q, k, v, g, b, s0, do, ds)
    eps = 1e-6
    for arr, gr in zip((q, k, v, g, b, s0), grads):
        num = np.zeros_like(arr)
        it = np.nditer(arr, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            old = arr[i]
            arr[i] = old + eps
            lp = _loss(q, k, v, g, b, s0, do, ds)
            arr[i] = old - eps
            lm = _loss(q, k, v, g, b, s0, do, ds)
            arr[i] = old
            num[i] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(gr, num, rtol=1e-6, atol=1e-7)
    assert grads[3][0, 2, 1, 0] == 0.0


def test_backward_packed_sequences_are_independent():
    rng = np.random.default_rng(12)
    T, H, d = 9, 1, 4
    q, k, v, g, do = (rng.normal(size=(1, T, H, d)) for _ in range(5))
    g = -np.abs(g)
    b = rng.uniform(0.1, 0.9, size=(1, T, H))
    cu = np.array([0, 4, 4, 9])
    s0 = rng.normal(size=(3, H, d, d))
    full = oracle.backward(q, k, v, g, b, s0, do, None, cu_seqlens=cu)
    part = oracle.backward(q[:, 4:], k[:, 4:], v[:, 4:], g[:, 4:], b[:, 4:], s0[2:], do[:, 4:])
    for x, y in zip(full[:5], part[:5]):
        np.testing.assert_allclose(x[:, 4:], y, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(full[5][2], part[5][0], rtol=1e-12, atol=1e-14)
    # the empty sequence's state passes through: its gradient is dL/dS_final = 0
    assert not full[5][1].any()
