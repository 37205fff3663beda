"""Failure detection without a GPU fault: a bounded device wait on a barrier that nothing
completes runs out, the kernel records it in the device error word and returns, the host
reads FA_ERR_TIMEOUT, and the context stays usable for the next attention call."""
import numpy as np
import pytest
import torch

import exact_attention_101_b200 as fa
import workloads
from parity_util import compare_bf16, oracle_rows, run_cuda

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives(cuda_ok):
    stream = torch.cuda.current_stream().cuda_stream
    assert fa.fa_check_device_error(stream) == fa.FA_OK           # clean to start with
    assert fa.fa_selftest_bounded_wait(2000, stream) == fa.FA_OK   # 2 ms limit
    assert fa.fa_check_device_error(stream) == fa.FA_ERR_TIMEOUT
    assert fa.fa_check_device_error(stream) == fa.FA_OK           # the word was cleared
    # the next real call runs normally
    w = workloads.WORKLOADS["tiny"]
    inp = workloads.make_inputs(w)
    o, lse = run_cuda(inp, True, w.scale, torch.float32)
    o_ref, lse_ref = oracle_rows(inp, True, w.scale)
    compare_bf16(o.reshape(-1, w.d), lse.reshape(-1), o_ref, lse_ref)
