"""Failure detection on the GPU without a fault: a decode launch whose
producer withholds one tile's copies (gqa_debug_decode_withhold) must give up
its bounded wait, report GQA_ERR_TIMEOUT through gqa_device_status, leave the
workspace zeroed, and leave the library usable: the next call is checked
against the oracle."""
import numpy as np
import pytest
import torch

from gpu_util import assert_bf16_parity, bf16_inputs, oracle_bf16, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gqa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import grouped_query_attention_fwd_b200 as m
    return m


@pytest.mark.parametrize("unit", [0, 100, 383])
def test_decode_wait_runs_out_and_is_reported(gqa, unit):
    # 4 x 4 groups of 24 tiles: 384 units over the SMs, so groups are split
    # and the aborted CTA's partners still merge through the ticket counters.
    bits, (q, k, v) = bf16_inputs(61, 4, 16, 4, 1, 3000, 128)
    plan = gqa.query(q, k, v)
    assert plan["kernel_name"] == "decode" and plan["work_units"] == 384
    ws = torch.zeros(plan["workspace_bytes"], dtype=torch.uint8, device="cuda")
    gqa.debug_decode_withhold(unit, 200_000)  # 200 us limit, this launch only
    gqa.forward(q, k, v, workspace=ws)
    assert gqa.device_status(ws) == gqa.GQA_ERR_TIMEOUT
    assert torch.count_nonzero(ws).item() == 0
    out = gqa.forward(q, k, v, workspace=ws)
    assert gqa.device_status(ws) == gqa.GQA_OK
    assert_bf16_parity(to_np(out), oracle_bf16(*bits), "after a timeout")


def test_withhold_setting_is_checked(gqa):
    with pytest.raises(gqa.GQAError):
        gqa.debug_decode_withhold(0, 10)          # limit below 1 us
    with pytest.raises(gqa.GQAError):
        gqa.debug_decode_withhold(-2, 200_000)    # no such unit
