"""GPU parity: kda_chunk_prefill_checkpointed (through the C ABI).

Snapshot m of sequence n is, by definition, the state of the recurrence after
the first m * interval tokens of that sequence: the oracle's final state on
that prefix.  The outputs o and state_out are those of kda_chunk_prefill,
bit for bit (the same kernels run; the snapshots are extra stores).
"""
import numpy as np
import pytest
import torch

import oracle
from _util import TOL_BF16, rel_err, to_np
from kda_delta_rule_chunkwise_b200 import binding
from kda_delta_rule_chunkwise_b200 import inputs as kin

pytestmark = pytest.mark.gpu


def prefix_state(inp, a, length, n, heads):
    """Oracle state of sequence n (rows a .. a+length of the packed inputs) after `length` tokens."""
    rows = lambda x: x.reshape((-1,) + tuple(x.shape[2:]))[a:a + length][:, heads].unsqueeze(0)
    s_in = None if inp.state_in is None else inp.state_in[n:n + 1][:, heads]
    _, s = oracle.recurrence(rows(inp.q), rows(inp.k), rows(inp.v), rows(inp.g), rows(inp.beta),
                             state_in=s_in)
    return s[0]


def check(inp, interval, heads, capacity=None):
    d = inp.to("cuda")
    o_ref, s_ref = binding.kda_chunk_prefill(d.q, d.k, d.v, d.g, d.beta, d.state_in, d.cu_seqlens)
    cnt = binding.kda_prefill_checkpoint_count(d.cu_seqlens, d.B, d.T, interval)
    ckpt = None
    if capacity is not None:
        ckpt = torch.full((capacity, d.H, 128, 128), float("nan"), device="cuda")
    o, s, ck = binding.kda_chunk_prefill_checkpointed(d.q, d.k, d.v, d.g, d.beta, d.state_in,
                                                      d.cu_seqlens, interval=interval, ckpt=ckpt)
    torch.cuda.synchronize()
    status = binding.kda_check_device_error()
    assert torch.equal(o, o_ref) and torch.equal(s, s_ref), "o / state_out differ from kda_chunk_prefill"
    if inp.cu_seqlens is None:
        cu = np.arange(inp.B + 1) * inp.T
    else:
        cu = inp.cu_seqlens.cpu().numpy()
    e, errs = 0, []
    for n in range(len(cu) - 1):
        length = int(cu[n + 1] - cu[n])
        m = 1
        while m * interval < length:
            if e < ck.shape[0]:
                want = prefix_state(inp, int(cu[n]), m * interval, n, heads)
                errs.append(rel_err(to_np(ck[e][heads]), want))
            e += 1
            m += 1
    assert e == cnt, (e, cnt)
    return status, errs


def test_ckpt_dense_every_two_chunks():
    inp = kin.prefill_inputs(2, 1000, 3, 128, 128, "bf16", seed=41, state="normal")
    status, errs = check(inp, 128, heads=[0, 1, 2])
    assert status == binding.KDA_OK
    assert len(errs) == 14 and max(errs) <= TOL_BF16, max(errs)


def test_ckpt_varlen_every_chunk_ragged_and_empty_sequences():
    inp = kin.prefill_inputs(1, 1194, 2, 128, 128, "bf16", seed=42, decay="split", state="normal",
                             lengths=[300, 0, 700, 65, 129])
    status, errs = check(inp, 64, heads=[0, 1])
    assert status == binding.KDA_OK
    assert len(errs) == 4 + 0 + 10 + 1 + 2 and max(errs) <= TOL_BF16, max(errs)


def test_ckpt_capacity_too_small_is_reported_and_the_rest_is_written():
    inp = kin.prefill_inputs(2, 640, 2, 128, 128, "bf16", seed=43, state="normal")
    status, errs = check(inp, 128, heads=[0, 1], capacity=5)   # 8 snapshots needed
    assert status == binding.KDA_ERR_INVALID_ARG
    assert len(errs) == 5 and max(errs) <= TOL_BF16


@pytest.mark.slow
def test_ckpt_full_h32_t8192():
    inp = kin.workload_inputs("prefill_h32_t8192_d128", seed=0, device="cpu")
    status, errs = check(inp, 2048, heads=[0, 31])
    assert status == binding.KDA_OK
    assert len(errs) == 3 and max(errs) <= TOL_BF16, max(errs)
