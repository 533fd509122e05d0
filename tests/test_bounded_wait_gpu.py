"""Failure detection without a GPU fault: a device-side wait that can never be
satisfied gives up after its poll limit, the kernel returns normally, the host
reads KDA_ERR_TIMEOUT, and the context stays usable."""
import pytest
import torch

from kda_delta_rule_chunkwise_b200 import binding
from kda_delta_rule_chunkwise_b200 import inputs as kin

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    assert binding.kda_check_device_error() == binding.KDA_OK
    binding.kda_selftest_bounded_wait(2000)   # 2 ms
    assert binding.kda_check_device_error() == binding.KDA_ERR_TIMEOUT
    # the word is cleared by the read
    assert binding.kda_check_device_error() == binding.KDA_OK
    # and the context still runs work correctly afterwards
    inp = kin.decode_inputs(1, 2, 2, 64, 64, "f32", seed=3)
    S = inp.state.cuda()
    o = binding.kda_decode_step(inp.q[0].cuda(), inp.k[0].cuda(), inp.v[0].cuda(),
                                inp.g[0].cuda(), inp.beta[0].cuda(), S)
    torch.cuda.synchronize()
    assert torch.isfinite(o).all()
    assert binding.kda_check_device_error() == binding.KDA_OK
