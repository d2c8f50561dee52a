"""Failure detection on the GPU without a fault: a device-side wait is made to run out
(a barrier that nothing arrives on, short limit); the kernel records the time-out in
the device status word and returns, the host reads ATTN_ERR_TIMEOUT, and the context
stays usable for ordinary work afterwards."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from parity_util import compare, to_np
from workloads import randn_bf16

pytestmark = pytest.mark.gpu


def test_wait_that_runs_out_is_reported_and_the_device_stays_usable():
    import online_softmax_exact_b200 as osx

    assert osx.attn_device_status(reset=True) == osx.ATTN_OK
    osx.attn_debug_wait_timeout(2_000_000)          # about a millisecond of SM cycles
    assert osx.attn_device_status() == osx.ATTN_ERR_TIMEOUT
    assert osx.attn_device_status(reset=True) == osx.ATTN_ERR_TIMEOUT   # read, then clear
    assert osx.attn_device_status() == osx.ATTN_OK

    q = randn_bf16((1, 2, 300, 64), 5, 0)
    k = randn_bf16((1, 2, 300, 64), 5, 1)
    v = randn_bf16((1, 2, 300, 64), 5, 2)
    o, lse = osx.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True, scale=0.125)
    assert osx.attn_device_status() == osx.ATTN_OK
    o_ref, l_ref = oracle.attention(q, k, v, causal=True, scale=0.125)
    compare(to_np(o), to_np(lse), o_ref, l_ref)


def test_wait_limit_is_validated():
    import online_softmax_exact_b200 as osx

    with pytest.raises(osx.AttnError):
        osx.attn_debug_wait_timeout(0)
    with pytest.raises(osx.AttnError):
        osx.attn_debug_wait_timeout(1 << 40)
