"""GPU: a bounded in-kernel wait that runs out is reported through the device
status word as GMLA_ERR_TIMEOUT, and the CUDA context stays usable after it."""
import numpy as np
import pytest
import torch

import oracle as orc
from synth_inputs import prefill_qkv
from tests.gpu_util import assert_parity, f64, to_dev

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_context_survives():
    import causal_head_latent_b200 as g
    assert g.gmla_get_device_status(raise_on_error=False) == 0
    g.gmla_selftest_wait_timeout(20)
    assert g.STATUS[g.gmla_get_device_status(raise_on_error=False)] == "GMLA_ERR_TIMEOUT"
    # reading the status cleared it
    assert g.gmla_get_device_status(raise_on_error=False) == 0
    # the context still runs kernels correctly
    inp = prefill_qkv(31, 1, 200, 2)
    Q, K, V = to_dev(inp["Q"]), to_dev(inp["K"]), to_dev(inp["V"])
    O = torch.empty_like(Q)
    g.gmla_attend_prefill(Q, K, V, O)
    g.gmla_get_device_status()
    assert_parity(f64(O), orc.attention(inp["Q"], inp["K"], inp["V"]), "O after a timeout")
