"""The device-side failure path: bounded waits that run out.

Every mbarrier wait in the kernels is bounded by %globaltimer; when a bound
runs out the kernel records KDA_ERR_TIMEOUT in the device status word
(instead of trapping) and gives up. kda_selftest_wait_timeout makes two such
waits (CTA and cluster scope) on an mbarrier that nothing arrives on, with a
2 ms bound. The test reads the status word through the C ABI, checks that the
context is still usable (a chunked prefill afterwards matches the oracle),
and that the word reads clean once reset. Nothing faults, traps or hangs.
"""
import pytest
import torch

import oracle
from gated_delta_rule_61_b200 import kda
from gated_delta_rule_61_b200.inputs import prefill_inputs
from tests.parity import TOL_BF16_O, TOL_BF16_STATE, assert_close


def test_selftest_rejects_out_of_range_bounds():
    assert kda.lib().kda_selftest_wait_timeout(10, None) == kda.KDA_ERR_INVALID_ARG
    assert kda.lib().kda_selftest_wait_timeout(5_000_000_000, None) == kda.KDA_ERR_INVALID_ARG


@pytest.mark.gpu
def test_bounded_waits_report_timeout_and_the_context_survives():
    st, _ = kda.device_status(reset=True)          # start from a clean word
    assert st == kda.KDA_OK
    assert kda.selftest_wait_timeout(2_000_000) == kda.KDA_OK
    st, detail = kda.device_status(reset=True)
    assert st == kda.KDA_ERR_TIMEOUT
    assert detail == 9091                          # the CTA-scope wait, then the cluster-scope one
    st, detail = kda.device_status(reset=True)
    assert st == kda.KDA_OK and detail == 0        # reset cleared it

    inp = prefill_inputs(2, 130, 3, 128, 128, dtype=torch.bfloat16, seed=5, init_std=0.1)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    o, s = kda.prefill(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"],
                       init_state=g["init_state"], chunk=64)
    o_ref, s_ref = oracle.kda_forward(inp["q"], inp["k"], inp["v"],
                                      inp["log_alpha"].double().clamp(min=kda.CHUNK_LOG_ALPHA_MIN),
                                      inp["beta"], init_state=inp["init_state"])
    assert_close(o, o_ref, TOL_BF16_O, "o after the timeout self-test")
    assert_close(s, s_ref, TOL_BF16_STATE, "state after the timeout self-test")
    st, detail = kda.device_status(reset=True)
    assert st == kda.KDA_OK and detail == 0
