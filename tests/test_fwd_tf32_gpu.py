"""GPU parity of the tf32 forward path (fa_fwd with FA_TF32: fp32 q, k, v, d = 64, rounded to
tf32 on the device, products on the tf32 tensor-core path, fp32 output) against the fp64 oracle
fed the same tf32-rounded values (as the bf16 path is checked against bf16-rounded values): the
products of tf32 values are exact in fp32, so the forward's stated bounds (1e-2 per element,
1e-3 mean, lse 1e-3) apply as they stand, with fp32 output.  The distance to the unrounded
problem is reported loosely (< 2e-2)."""
import math

import numpy as np
import pytest
import torch

import oracle as oracle_mod
import synth_inputs as si
from exact_io_aware_97_b200 import binding as fa
from parity import check_lse, check_out, dev_f32, host64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def orc():
    return oracle_mod.get()


CASES = [
    # B, Nq, Nk, Hq, Hkv, causal, seed
    (1, 128, 128, 1, 1, 0, 1001),   # the single-head fp32 workload (scale 1/8)
    (2, 300, 300, 4, 2, 1, 9501),
    (1, 257, 130, 2, 1, 1, 9502),
    (1, 1, 5, 1, 1, 0, 9503),
    (1, 1000, 1000, 8, 8, 1, 9504),
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_tf32_forward(orc, case):
    B, Nq, Nk, Hq, Hkv, causal, seed = case
    d = 64
    q = si.normal(seed, si.Q, (B, Nq, Hq, d), "f32")
    k = si.normal(seed, si.K, (B, Nk, Hkv, d), "f32")
    v = si.normal(seed, si.V, (B, Nk, Hkv, d), "f32")
    scale = 1.0 / math.sqrt(d)
    o, lse = fa.forward(dev_f32(q), dev_f32(k), dev_f32(v), causal=bool(causal), scale=scale, tf32=True)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    assert o.dtype == torch.float32
    qr, kr, vr = (si.round_tf32(x) for x in (q, k, v))
    o_ref, lse_ref = orc.attention(qr, kr, vr, scale, causal=bool(causal))
    check_out(host64(o), o_ref, bf16_out=False)
    check_lse(host64(lse), lse_ref)
    o_raw, _ = orc.attention(q, k, v, scale, causal=bool(causal))
    assert np.abs(host64(o) - o_raw).max() < 2e-2


def test_tf32_rejects_unsupported():
    q = torch.zeros(1, 8, 1, 128, device="cuda")
    with pytest.raises(fa.FaError) as e:
        fa.forward(q, q, q, tf32=True)
    assert e.value.status == fa.FA_ERR_UNSUPPORTED
