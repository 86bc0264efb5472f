"""Failure detection without a GPU fault: a bounded wait that runs out (a
barrier nothing arrives on) reports BL_ERR_TIMEOUT through the status word,
and the context keeps working."""
import time

import pytest
import torch

import oracle as O
import ternary_weight_bitlinear_b200 as B
from ternary_weight_bitlinear_b200 import workloads as WL
from gpu_util import assert_f32_output, bf16_dev

pytestmark = pytest.mark.gpu


def test_expired_wait_reports_timeout_and_context_survives():
    assert B.bitlinear_device_status() == 0
    t0 = time.perf_counter()
    B.bitlinear_selftest_wait_timeout(50_000_000)  # 50 ms
    assert B.bitlinear_device_status() == 7        # BL_ERR_TIMEOUT, and the word is cleared
    assert time.perf_counter() - t0 >= 0.045
    assert B.bitlinear_device_status() == 0
    # the same context still computes correctly
    c = WL.config1()
    P_d, beta = B.bitlinear_pack(torch.from_numpy(c["W"]).cuda())
    P_o, beta_o = O.pack_master(c["W"])
    y = B.bitlinear_forward(bf16_dev(c["x"]), P_d, float(beta.item()), out_dtype=torch.float32)
    assert_f32_output(y.cpu().numpy(), O.forward(c["x"], P_o, beta_o, norm=False)["y"], "after timeout")
    assert B.bitlinear_device_status() == 0
