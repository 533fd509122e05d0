"""GPU parity: kda_chunk_prefill_ex with input preprocessing inside the prefill
(gate from logits g = -5 sigmoid(x); unit-L2 q, k), against the fp64 oracle
applied to the same preprocessing (oracle.preprocess) of the same raw inputs."""
import numpy as np
import pytest
import torch

import oracle
from _util import TOL_BF16, rel_err, to_np
from kda_delta_rule_chunkwise_b200 import binding
from kda_delta_rule_chunkwise_b200 import inputs as kin

pytestmark = pytest.mark.gpu


def oracle_run(inp, flags, rows=None):
    q, k, g = oracle.preprocess(inp.q, inp.k, inp.g, flags)
    cu = None if inp.cu_seqlens is None else inp.cu_seqlens.cpu().numpy().astype(np.int64)
    o, s = oracle.recurrence(q, k, inp.v, g, inp.beta, state_in=inp.state_in, cu_seqlens=cu)
    return o, s


@pytest.mark.parametrize("flags", [binding.KDA_PREP_GATE_LOGIT | binding.KDA_PREP_L2NORM_QK,
                                   binding.KDA_PREP_L2NORM_QK])
def test_prep_raw_inputs(flags):
    inp = kin.prefill_raw_inputs(1, 1065, 4, 128, 128, "bf16", seed=51,
                                 lengths=[300, 0, 700, 65])
    if not flags & binding.KDA_PREP_GATE_LOGIT:
        # gate already formed: use a valid log-decay
        inp.g = (-5.0 * torch.sigmoid(inp.g.float())).to(torch.bfloat16)
    d = inp.to("cuda")
    o, s, _ = binding.kda_chunk_prefill_ex(d.q, d.k, d.v, d.g, d.beta, d.state_in, d.cu_seqlens,
                                           flags=flags)
    torch.cuda.synchronize()
    assert binding.kda_check_device_error() == binding.KDA_OK
    o_ref, s_ref = oracle_run(inp, flags)
    eo, es = rel_err(to_np(o), o_ref), rel_err(to_np(s), s_ref)
    print(f"flags {flags}: output error {eo:.3e}, final-state error {es:.3e}")
    assert eo <= TOL_BF16 and es <= TOL_BF16


def test_prep_gate_only_on_unit_keys():
    inp = kin.prefill_inputs(2, 500, 3, 128, 128, "bf16", seed=52, state="normal")
    inp.g = (2.0 * torch.randn(inp.g.shape, generator=torch.Generator().manual_seed(7))).to(torch.bfloat16)
    d = inp.to("cuda")
    o, s, _ = binding.kda_chunk_prefill_ex(d.q, d.k, d.v, d.g, d.beta, d.state_in, None,
                                           flags=binding.KDA_PREP_GATE_LOGIT)
    o_ref, s_ref = oracle_run(inp, binding.KDA_PREP_GATE_LOGIT)
    assert rel_err(to_np(o), o_ref) <= TOL_BF16 and rel_err(to_np(s), s_ref) <= TOL_BF16


def test_ex_without_flags_is_the_plain_prefill_bit_for_bit():
    inp = kin.prefill_inputs(1, 700, 4, 128, 128, "bf16", seed=53, state="normal")
    d = inp.to("cuda")
    o1, s1 = binding.kda_chunk_prefill(d.q, d.k, d.v, d.g, d.beta, d.state_in, None)
    o2, s2, _ = binding.kda_chunk_prefill_ex(d.q, d.k, d.v, d.g, d.beta, d.state_in, None)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_prep_with_intermediate_states():
    flags = binding.KDA_PREP_GATE_LOGIT | binding.KDA_PREP_L2NORM_QK
    inp = kin.prefill_raw_inputs(1, 640, 2, 128, 128, "bf16", seed=54)
    d = inp.to("cuda")
    o, s, ck = binding.kda_chunk_prefill_ex(d.q, d.k, d.v, d.g, d.beta, d.state_in, None,
                                            flags=flags, ckpt_interval=256)
    torch.cuda.synchronize()
    assert binding.kda_check_device_error() == binding.KDA_OK
    assert ck.shape[0] == 2                       # after 256 and 512 of 640 tokens
    q, k, g = oracle.preprocess(inp.q, inp.k, inp.g, flags)
    for m, t in enumerate((256, 512)):
        _, s_ref = oracle.recurrence(q[:, :t], k[:, :t], inp.v[:, :t], g[:, :t], inp.beta[:, :t],
                                     state_in=inp.state_in)
        assert rel_err(to_np(ck[m]), s_ref[0]) <= TOL_BF16
