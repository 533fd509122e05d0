"""Shared helpers for the GPU parity tests (no KDA arithmetic here)."""
from __future__ import annotations

import numpy as np
import torch

import oracle

TOL_BF16 = 2e-2    # max|delta| / rms(reference), bf16 inputs, fp32 state
TOL_F32 = 1e-4     # same metric, fp32 path


def rel_err(got, ref) -> float:
    """max |got - ref| / rms(ref) over the whole tensor (fp64)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rms = float(np.sqrt(np.mean(ref * ref)))
    if rms == 0.0:
        return float(np.max(np.abs(got - ref)))
    return float(np.max(np.abs(got - ref)) / rms)


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def oracle_prefill(inp, heads=None, seqs=None, n_threads=None):
    """Oracle outputs for the given PrefillInputs (CPU tensors), optionally a subset.

    Returns dict (n, h) -> (o [len, dv], S [dk, dv]) for every requested unit.
    """
    H = inp.H
    heads = list(range(H)) if heads is None else list(heads)
    if inp.cu_seqlens is None:
        cu = np.arange(inp.B + 1) * inp.T
        rows = lambda x: x.reshape((inp.B * inp.T,) + tuple(x.shape[2:]))
    else:
        cu = inp.cu_seqlens.cpu().numpy().astype(np.int64)
        rows = lambda x: x[0]
    seqs = list(range(len(cu) - 1)) if seqs is None else list(seqs)
    q, k, v, g, b = (rows(x) for x in (inp.q, inp.k, inp.v, inp.g, inp.beta))
    out = {}
    # one oracle call: requested sequences packed, requested heads side by side
    sel = [(int(cu[n]), int(cu[n + 1])) for n in seqs]
    idx = np.concatenate([np.arange(a, e) for a, e in sel]) if sel else np.zeros(0, int)
    lens = [e - a for a, e in sel]
    cu_s = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    it = torch.as_tensor(idx, dtype=torch.long, device=q.device)
    ht = torch.as_tensor(heads, dtype=torch.long, device=q.device)
    pick = lambda x: x.index_select(0, it).index_select(1, ht).unsqueeze(0)
    s_in = None
    if inp.state_in is not None:
        st = torch.as_tensor(seqs, dtype=torch.long, device=inp.state_in.device)
        s_in = inp.state_in.index_select(0, st).index_select(1, ht.to(st.device))
    o, s = oracle.recurrence(pick(q), pick(k), pick(v), pick(g), pick(b),
                             state_in=s_in, cu_seqlens=cu_s, n_threads=n_threads)
    for i, n in enumerate(seqs):
        for hi, h in enumerate(heads):
            out[(n, h)] = (o[0, cu_s[i]:cu_s[i + 1], hi], s[i, hi])
    return out


def gather_gpu(inp_cpu, o_gpu, s_gpu, units):
    """Pick the same (n, h) units out of the GPU results (copied to host)."""
    if inp_cpu.cu_seqlens is None:
        cu = np.arange(inp_cpu.B + 1) * inp_cpu.T
    else:
        cu = inp_cpu.cu_seqlens.cpu().numpy().astype(np.int64)
    o_rows = o_gpu.reshape((-1,) + tuple(o_gpu.shape[2:]))
    res = {}
    for (n, h) in units:
        a, e = int(cu[n]), int(cu[n + 1])
        res[(n, h)] = (to_np(o_rows[a:e, h]), to_np(s_gpu[n, h]) if s_gpu is not None else None)
    return res


def compare_units(ref, got, tol, what=""):
    o_ref = np.concatenate([ref[u][0].reshape(-1) for u in ref])
    o_got = np.concatenate([got[u][0].reshape(-1) for u in ref])
    s_ref = np.concatenate([ref[u][1].reshape(-1) for u in ref])
    s_got = np.concatenate([got[u][1].reshape(-1) for u in ref])
    eo, es = rel_err(o_got, o_ref), rel_err(s_got, s_ref)
    print(f"{what}: output error {eo:.3e}, final-state error {es:.3e} (bar {tol})")
    assert np.all(np.isfinite(o_got)) and np.all(np.isfinite(s_got)), f"{what}: non-finite output"
    assert eo <= tol, f"{what}: output error {eo:.3e} > {tol}"
    assert es <= tol, f"{what}: final-state error {es:.3e} > {tol}"
    return eo, es


def compare_all_units(inp, o_gpu, s_gpu, tol, what="", budget=1 << 21, n_threads=None):
    """Every (sequence, head) unit of a call against the oracle, element by element.

    The oracle runs on groups of units of at most `budget` token-heads (whole
    sequences, all heads or a slice of them) so that host memory stays
    bounded; the error metric max|delta| / rms(reference) is taken over the
    whole output tensor and over all final states, as for a single comparison.
    """
    if inp.cu_seqlens is None:
        cu = np.arange(inp.B + 1) * inp.T
    else:
        cu = inp.cu_seqlens.cpu().numpy().astype(np.int64)
    N, H = len(cu) - 1, inp.H
    o_rows = o_gpu.reshape((-1,) + tuple(o_gpu.shape[2:])).cpu()
    s_all = s_gpu.cpu()
    acc = {"o": [0.0, 0.0, 0], "s": [0.0, 0.0, 0]}   # max|delta|, sum ref^2, count

    def add(key, got, ref):
        a = acc[key]
        got = np.asarray(got, np.float64)
        assert np.all(np.isfinite(got)), f"{what}: non-finite {key}"
        a[0] = max(a[0], float(np.max(np.abs(got - ref))) if ref.size else 0.0)
        a[1] += float(np.sum(ref * ref))
        a[2] += ref.size

    def run(seqs, heads):
        ref = oracle_prefill(inp, heads=heads, seqs=seqs, n_threads=n_threads)
        for (n, h), (o_ref, s_ref) in ref.items():
            a, e = int(cu[n]), int(cu[n + 1])
            add("o", to_np(o_rows[a:e, h]), o_ref)
            add("s", to_np(s_all[n, h]), s_ref)

    group, tok = [], 0
    for n in range(N):
        ln = int(cu[n + 1] - cu[n])
        if ln * H > budget:                 # one long sequence: slices of heads
            hs = max(1, budget // max(ln, 1))
            for h0 in range(0, H, hs):
                run([n], list(range(h0, min(H, h0 + hs))))
            continue
        if group and (tok + ln) * H > budget:
            run(group, list(range(H)))
            group, tok = [], 0
        group.append(n)
        tok += ln
    if group:
        run(group, list(range(H)))
    errs = {}
    for key, (mx, ss, cnt) in acc.items():
        rms = np.sqrt(ss / max(cnt, 1))
        errs[key] = mx / rms if rms > 0 else mx
    print(f"{what}: all {N} x {H} units: output error {errs['o']:.3e}, "
          f"final-state error {errs['s']:.3e} (bar {tol})")
    assert errs["o"] <= tol, f"{what}: output error {errs['o']:.3e} > {tol}"
    assert errs["s"] <= tol, f"{what}: final-state error {errs['s']:.3e} > {tol}"
    return errs["o"], errs["s"]
