"""Failure detection on the GPU without a fault: a kernel whose single wait can never be
satisfied (a barrier nothing arrives on) gives up after the wait limit, records the timeout,
and returns; the host reads FA_ERR_TIMEOUT, and the context stays usable for the next call."""
import math
import time

import numpy as np
import pytest
import torch

import oracle as oracle_mod
import synth_inputs as si
from exact_io_aware_97_b200 import binding as fa
from parity import check_out, dev_bf16, host64

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    assert fa.fa_last_device_error() == fa.FA_OK  # nothing pending
    t0 = time.monotonic()
    fa.fa_selftest_wait_timeout()
    status = fa.fa_last_device_error()  # synchronises
    elapsed = time.monotonic() - t0
    assert status == fa.FA_ERR_TIMEOUT
    assert 3.0 <= elapsed < 60.0, elapsed
    assert fa.fa_last_device_error() == fa.FA_OK  # the record was cleared
    # the context is usable: a forward still matches the oracle
    q = si.normal(9601, si.Q, (1, 130, 2, 64))
    k = si.normal(9601, si.K, (1, 130, 1, 64))
    v = si.normal(9601, si.V, (1, 130, 1, 64))
    o, _ = fa.forward(dev_bf16(q), dev_bf16(k), dev_bf16(v), causal=True, scale=0.125)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    o_ref, _ = oracle_mod.get().attention(q, k, v, 0.125, causal=True)
    check_out(host64(o), o_ref)
