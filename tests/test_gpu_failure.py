"""The failure path of the kernels' bounded waits, exercised without faulting the GPU.

Every wait inside a kernel (for a tile, a product, a free buffer) has a time limit.  A wait
that runs out records ATTN_ERR_DEVICE_TIMEOUT and the site that gave up in the library's
device error word, the kernel unwinds (its teardown still waits, with the full limit, for the
copies and products it started) and exits; the host reads the status with
attn_get_device_status.  The pages ask for exactly this ("3.7 어텐션 II", 3.7.3): a failure
is reported, never hidden behind a silent fallback.

Here the pipeline waits' limit is lowered to one nanosecond, so the first wait that is not
already satisfied runs out; the test checks the status, the recorded site, and that the next
call with the normal limit is correct.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from io_aware_softmax_b200 import (attn_decode, attn_fwd, attn_last_error_site,
                                   attn_set_wait_limit_ns, device_status)
from tests.gpu_common import compare, f64

pytestmark = pytest.mark.gpu

ATTN_ERR_DEVICE_TIMEOUT = -5


def _run_with_tiny_limit(call):
    assert device_status() == 0
    attn_set_wait_limit_ns(1)
    try:
        call()
        status = device_status()
    finally:
        attn_set_wait_limit_ns(0)
    return status


def test_prefill_wait_that_runs_out_is_reported_and_the_next_call_is_clean():
    q, k, v = (workloads.randn_bf16((1, 4, 700, 128), 51, i).cuda() for i in range(3))
    status = _run_with_tiny_limit(lambda: attn_fwd(q, k, v, mask="causal"))
    assert status == ATTN_ERR_DEVICE_TIMEOUT
    assert attn_last_error_site() != 0
    o, lse = attn_fwd(q, k, v, mask="causal")
    assert device_status() == 0
    O_ref, L_ref = oracle.attention(f64(q), f64(k), f64(v), mask_kind=1)
    compare(o, lse, O_ref, L_ref, "prefill after a timed-out call")


def test_decode_wait_that_runs_out_is_reported_and_the_next_call_is_clean():
    # one sequence, one split: a single CTA streams 1024 cache stages through its three-stage
    # ring, so its consumers wait for a copy from memory at almost every stage (the device
    # timer advances in steps of up to a microsecond; waits this long always see it move)
    q = workloads.randn_bf16((1, 4, 1, 128), 52, 0).cuda()
    kc = workloads.randn_bf16((1, 1, 65536, 128), 52, 1).cuda()
    vc = workloads.randn_bf16((1, 1, 65536, 128), 52, 2).cuda()
    status = _run_with_tiny_limit(lambda: attn_decode(q, kc, vc, num_splits=1))
    assert status == ATTN_ERR_DEVICE_TIMEOUT
    assert attn_last_error_site() != 0
    o, lse = attn_decode(q, kc, vc, num_splits=1)
    assert device_status() == 0
    O_ref, L_ref = oracle.attention(f64(q), f64(kc), f64(vc))
    compare(o, lse, O_ref, L_ref, "decode after a timed-out call")


def test_status_is_cleared_once_read():
    q, k, v = (workloads.randn_bf16((1, 2, 300, 64), 53, i).cuda() for i in range(3))
    assert _run_with_tiny_limit(lambda: attn_fwd(q, k, v)) == ATTN_ERR_DEVICE_TIMEOUT
    assert device_status() == 0
    o1, l1 = attn_fwd(q, k, v)
    o2, l2 = attn_fwd(q, k, v)
    assert device_status() == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2) and np.isfinite(f64(l1)).all()
