"""The bounded-wait timeout path of a real kernel, exercised without a GPU
fault: a test hook makes the summaries kernel skip the bulk copy its wait is
for, with a wait limit of a millisecond.  The kernel records HGA_ERR_TIMEOUT
(hga_device_status reads it), returns with nothing in flight, and the next
call, hooks off, runs normally with correct results on the same context."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from tests.parity import row_rel_err
from workloads import WORKLOADS, make_prefill_inputs

pytestmark = pytest.mark.gpu


def test_summaries_wait_runs_out_then_recovers(gpu_lib):
    w = WORKLOADS["qwen3_30b_a3b_bf16_prefill_32k"].replace(T=1024)
    dev = torch.device("cuda")
    q, k, v, pos, _ = make_prefill_inputs(w, seed=3)
    kd, pd = k.to(dev), pos.to(dev)
    hp = gpu_lib.HGAParams(C=w.C, g_s=w.g_s, F=w.F, L=w.L, K_c=w.K_c, K_g=w.K_g,
                           rope_theta=w.theta)
    lib = gpu_lib.load()
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert gpu_lib.hga_device_status(clear=True) == 0
    assert lib.hga_set_test_hooks(1, 1_000_000, st) == 0          # 1 ms limit, no copy
    try:
        gpu_lib.hga_build_summaries(kd, pd, hp)
        assert gpu_lib.hga_device_status(clear=True) == 4          # HGA_ERR_TIMEOUT
    finally:
        assert lib.hga_set_test_hooks(0, 0, st) == 0
    # the same context, hooks off: a normal call, no status, correct summaries
    k_rot, s_c, s_g = gpu_lib.hga_build_summaries(kd, pd, hp)
    torch.cuda.synchronize()
    assert gpu_lib.hga_device_status(clear=True) == 0
    S_c, S_g = oracle.build_summaries(k, pos, oracle.Params.of(w))
    assert row_rel_err(s_c.cpu().numpy(), S_c) < 2e-6
    assert row_rel_err(s_g.cpu().numpy(), S_g) < 2e-6
