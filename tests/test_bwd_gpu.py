"""GPU parity of fa_bwd (through the C ABI) against the fp64 oracle's backward on the same
bf16 inputs.  The forward that fa_bwd needs (o, lse) is fa_fwd's, as a caller would run it."""
import math

import numpy as np
import pytest
import torch

import oracle as oracle_mod
import synth_inputs as si
from exact_io_aware_97_b200 import binding as fa
from parity import check_grad, dev_bf16, host64

pytestmark = pytest.mark.gpu

DOUT = 9  # tensor id of the upstream gradient's stream


@pytest.fixture(scope="module")
def orc():
    return oracle_mod.get()


def _inputs(seed, B, Nq, Nk, Hq, Hkv, d):
    q = si.normal(seed, si.Q, (B, Nq, Hq, d))
    k = si.normal(seed, si.K, (B, Nk, Hkv, d))
    v = si.normal(seed, si.V, (B, Nk, Hkv, d))
    do = si.normal(seed, DOUT, (B, Nq, Hq, d))
    return q, k, v, do


def _gpu_bwd(q, k, v, do, causal, scale):
    tq, tk, tv, tdo = dev_bf16(q), dev_bf16(k), dev_bf16(v), dev_bf16(do)
    o, lse = fa.forward(tq, tk, tv, causal=causal, scale=scale)
    dq, dk, dv = fa.backward(tq, tk, tv, o, lse, tdo, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    return host64(dq), host64(dk), host64(dv)


CASES = [
    # B, Nq, Nk, Hq, Hkv, d, causal
    (1, 128, 128, 2, 1, 64, 1),
    (2, 300, 300, 4, 2, 128, 1),
    (1, 513, 513, 8, 2, 128, 0),
    (2, 200, 330, 3, 3, 64, 1),
    (1, 300, 100, 4, 1, 128, 1),
    (1, 1024, 1024, 16, 16, 64, 1),
    (1, 1, 1, 1, 1, 128, 0),
    (3, 77, 1, 2, 1, 64, 0),
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_bwd_small(orc, case):
    B, Nq, Nk, Hq, Hkv, d, causal = case
    q, k, v, do = _inputs(7000 + Nq + Nk + d, B, Nq, Nk, Hq, Hkv, d)
    scale = 1.0 / math.sqrt(d)
    dq, dk, dv = _gpu_bwd(q, k, v, do, causal, scale)
    rq, rk, rv = orc.attention_bwd(q, k, v, do, scale, causal=bool(causal))
    check_grad(dq, rq, "dQ")
    check_grad(dk, rk, "dK")
    check_grad(dv, rv, "dV")


def test_bwd_repeatable_bitwise():
    """dK and dV are accumulated in one CTA in a fixed order: bitwise repeatable.  dQ is summed
    with fp32 reductions from several CTAs, whose order varies: close, not bitwise."""
    q, k, v, do = _inputs(7101, 1, 640, 640, 8, 2, 128)
    a = _gpu_bwd(q, k, v, do, True, 1 / math.sqrt(128))
    b = _gpu_bwd(q, k, v, do, True, 1 / math.sqrt(128))
    assert np.array_equal(a[1], b[1]) and np.array_equal(a[2], b[2])
    assert np.abs(a[0] - b[0]).max() <= 1e-2 * np.abs(a[0]).max()


def test_bwd_gqa_causal_8k_one_group(orc):
    """B=1, Hq=64, Hkv=8, N=8192, d=128, causal (the forward benchmark workload), gradients
    of the whole problem on the GPU; the oracle checks one K/V group (8 query heads), which
    is an independent problem of its own."""
    w = si.WORKLOADS["gqa_causal_8k"]
    B, N, Hq, Hkv, d = w["B"], w["N"], w["Hq"], w["Hkv"], w["d"]
    q, k, v, do = _inputs(w["seed"], B, N, N, Hq, Hkv, d)
    scale = 1.0 / math.sqrt(d)
    dq, dk, dv = _gpu_bwd(q, k, v, do, True, scale)
    G = Hq // Hkv
    g = 5
    hs = slice(g * G, (g + 1) * G)
    rq, rk, rv = orc.attention_bwd(q[:, :, hs], k[:, :, g:g + 1], v[:, :, g:g + 1], do[:, :, hs], scale, causal=True)
    check_grad(dq[:, :, hs], rq, "dQ")
    check_grad(dk[:, :, g:g + 1], rk, "dK")
    check_grad(dv[:, :, g:g + 1], rv, "dV")


def test_bwd_mha_causal_2k_full(orc):
    """B=2, H=12, N=2048, d=64, causal (the pages' packed example shape): every gradient
    element against the oracle (the d = 64 kernel)."""
    w = si.WORKLOADS["mha_causal_2k"]
    B, N, Hq, Hkv, d = w["B"], w["N"], w["Hq"], w["Hkv"], w["d"]
    q, k, v, do = _inputs(w["seed"], B, N, N, Hq, Hkv, d)
    scale = 1.0 / math.sqrt(d)
    dq, dk, dv = _gpu_bwd(q, k, v, do, True, scale)
    rq, rk, rv = orc.attention_bwd(q, k, v, do, scale, causal=True)
    check_grad(dq, rq, "dQ")
    check_grad(dk, rk, "dK")
    check_grad(dv, rv, "dV")
