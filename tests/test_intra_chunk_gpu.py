"""GPU check of the intra-chunk (phase A) products on their own.

After a bf16 prefill the caller's workspace holds, per (chunk, head), the
matrices the state pass consumes.  This test decodes them from their
documented shared-memory layouts and compares each with its fp64 definition
written out here from the chunked form of the recurrence:

    G = cumsum(max(g, -5)),  Akk[r,s] = beta_r sum_c k_r k_s e^{G_r-G_s} (s<r)
    Aqk[r,s] = sum_c q_r k_s e^{G_r-G_s} (s<=r),  T = (I+Akk)^{-1} Diag(beta)
    R = Aqk T,  W = T (K e^G),  P = Q e^G - R (K e^G),  Khat = K e^{G_L-G},
    Gamma_L = e^{G_L}

Layouts (fp16): [-W; P] 128x128 K-major 128B-swizzled in two 64-column
blocks 16 KiB apart (slot offset 0); [T; R] 128x64 K-major swizzled (offset
32 KiB); Khat MN-major swizzled (channel contiguous) in two 64-channel blocks
8 KiB apart (offset 48 KiB); Gamma_L fp32 (offset 64 KiB).
"""
import numpy as np
import pytest
import torch

from _precision_emulation import chunk_factors
from _util import rel_err
from kda_delta_rule_chunkwise_b200 import binding
from kda_delta_rule_chunkwise_b200 import inputs as kin

pytestmark = pytest.mark.gpu

SLOT = 66560


def header_bytes(N):
    return ((N + 1) * 16 + 1023) & ~1023


def kmajor_off(row, col, kblock):
    kb, c = col >> 6, col & 63
    return kb * kblock + (row >> 3) * 1024 + (row & 7) * 128 + (((c >> 3) ^ (row & 7)) * 16) + (c & 7) * 2


def mnmajor_off(mn, k, mnblock):
    mb, m = mn >> 6, mn & 63
    return mb * mnblock + (k >> 3) * 1024 + (k & 7) * 128 + (((m >> 3) ^ (k & 7)) * 16) + (m & 7) * 2


def f16_at(buf_u16, offs):
    return buf_u16[offs // 2].view(np.float16).astype(np.float64)


def decode_slot(slot):
    u16 = slot.view(np.uint16)
    rows = np.arange(128)[:, None]
    WP = f16_at(u16, kmajor_off(rows, np.arange(128)[None, :], 16384))
    TR = f16_at(u16, 32768 + kmajor_off(rows, np.arange(64)[None, :], 0))
    s = np.arange(64)[:, None]
    Kh = f16_at(u16, 49152 + mnmajor_off(np.arange(128)[None, :], s, 8192))
    Gam = slot[65536:65536 + 512].view(np.float32).astype(np.float64)
    return WP, TR, Kh, Gam


def reference(q, k, g, b):
    """fp64 definitions for one chunk: q, k, g [L, 128]; b [L]."""
    L = q.shape[0]
    G = np.cumsum(np.maximum(g, -5.0), axis=0)
    E = np.exp(G[:, None, :] - G[None, :, :])
    Akk = np.tril(np.einsum("rc,sc,rsc->rs", k, k, E), -1) * b[:, None]
    Aqk = np.tril(np.einsum("rc,sc,rsc->rs", q, k, E))
    T = np.linalg.inv(np.eye(L) + Akk) * b[None, :]
    R = Aqk @ T
    Kt = k * np.exp(G)
    W = T @ Kt
    P = q * np.exp(G) - R @ Kt
    Kh = k * np.exp(G[-1][None, :] - G)
    return T, R, W, P, Kh, np.exp(G[-1])


@pytest.mark.parametrize("L,decay", [(64, "uniform"), (37, "uniform"), (64, "split")])
def test_intra_chunk_products(L, decay):
    H = 2
    inp = kin.prefill_inputs(1, 64 + L, H, 128, 128, "bf16", seed=20, decay=decay)
    d = inp.to("cuda")
    need = binding.kda_chunk_prefill_workspace_bytes(64 + L, 1, H, 128, 128, torch.bfloat16)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    # one packed sequence, so that the chunk table is built (equal-length batches skip it)
    cu = torch.tensor([0, 64 + L], dtype=torch.int32, device="cuda")
    binding.kda_chunk_prefill(d.q, d.k, d.v, d.g, d.beta, None, cu, workspace=ws)
    torch.cuda.synchronize()
    wsh = ws.cpu().numpy()
    hb = header_bytes(1)
    chunk_off = wsh[:8].view(np.int32)
    assert chunk_off[0] == 0 and chunk_off[1] == 2          # chunk_off[N], N = 1
    f = lambda x: x.double().numpy()
    for c, (t0, n) in enumerate([(0, 64), (64, L)]):
        for h in range(H):
            slot = wsh[hb + (c * H + h) * SLOT: hb + (c * H + h + 1) * SLOT]
            WP, TR, Kh, Gam = decode_slot(slot)
            T, R, W, P, Khr, Gr = reference(f(inp.q[0, t0:t0 + n, h]), f(inp.k[0, t0:t0 + n, h]),
                                            f(inp.g[0, t0:t0 + n, h]), f(inp.beta[0, t0:t0 + n, h]))
            tag = f"chunk {c} head {h}"
            errs = {"T": rel_err(TR[:n, :n], T), "R": rel_err(TR[64:64 + n, :n], R),
                    "W": rel_err(-WP[:n], W), "P": rel_err(WP[64:64 + n], P),
                    "Khat": rel_err(Kh[:n], Khr)}
            # Bar per matrix, derived from the precision scheme rather than fixed: the
            # same factors evaluated in fp64 with every operand rounded as the kernel
            # stores it (tf32 Akk/Aqk operands, fp32 accumulation, fp16 storage; see
            # _precision_emulation) have an error e_emul against the definitions
            # above.  The kernel differs from that emulation only in the order of its
            # fp32 sums and in its exp / reciprocal, so it must stay within a small
            # multiple of it: bar = 4 e_emul, at least 4e-3 (a few fp16 ulps of the
            # largest element).  The end-to-end outputs are held to the 2e-2 bar in
            # test_prefill_gpu.py.
            em = chunk_factors(f(inp.q[0, t0:t0 + n, h]), f(inp.k[0, t0:t0 + n, h]),
                               f(inp.g[0, t0:t0 + n, h]), f(inp.beta[0, t0:t0 + n, h]))
            emul = {"T": rel_err(em["T"], T), "R": rel_err(em["R"], R), "W": rel_err(em["W"], W),
                    "P": rel_err(em["P"], P), "Khat": rel_err(em["Khat"], Khr)}
            print(tag, {k_: f"{v_:.2e} (emulated {emul[k_]:.2e})" for k_, v_ in errs.items()})
            for name, e in errs.items():
                bar = max(4 * emul[name], 4e-3)
                assert e < bar, f"{tag} {name}: {e:.3e} > {bar:.3e}"
            # Gamma_L = exp(G_L) <= 1 in fp32: absolute error (values below the fp32
            # range, e.g. e^-160 after a fast-decaying chunk, are 0)
            assert np.max(np.abs(Gam - Gr)) < 1e-6, tag + " Gamma"
            # masked tails are exactly zero
            assert not TR[n:64].any() and not TR[:, n:64].any(), tag + " T/R tail"
            assert not WP[n:64].any() and not WP[64 + n:].any(), tag + " W/P tail"
            assert not Kh[n:].any(), tag + " Khat tail"
