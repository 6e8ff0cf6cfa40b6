"""GPU parity of fa_fwd_fp8 (e4m3 inputs, P rounded to e4m3) against the fp64 oracle on the
dequantised inputs.

Tolerance, from the arithmetic: the products S = q k^T of e4m3 values are exact in the fp32
accumulator and l sums the unrounded P, so lse keeps the forward's 1e-3.  O differs from the
exact result by the rounding of P to e4m3 (3 mantissa bits: relative error at most 2^-4 per
element in the normal range), i.e. by at most 2^-4 * sum_j p_j |v_j| / l = 2^-4 * A, where A is
attention(q, k, |v|) (computed by the oracle), plus the forward's 1e-2 for accumulation and bf16
output rounding.  The mean error is also bounded (1e-2)."""
import math

import numpy as np
import pytest
import torch

import oracle as oracle_mod
import synth_inputs as si
from exact_io_aware_97_b200 import binding as fa
from parity import check_lse, host64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def orc():
    return oracle_mod.get()


def _fp8_problem(seed, B, Nq, Nk, Hq, Hkv, d=128):
    q = si.normal(seed, si.Q, (B, Nq, Hq, d), "f32")
    k = si.normal(seed, si.K, (B, Nk, Hkv, d), "f32")
    v = si.normal(seed, si.V, (B, Nk, Hkv, d), "f32")
    return [si.to_e4m3(x) for x in (q, k, v)]


def _run(q8, k8, v8, causal, scale):
    dev = lambda t: torch.from_numpy(t[0]).cuda()
    o, lse = fa.forward_fp8(dev(q8), dev(k8), dev(v8), q8[2], k8[2], v8[2], causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    return host64(o), host64(lse)


def _check(o, o_ref, a_ref, what="O"):
    assert np.all(np.isfinite(o)), f"{what}: non-finite"
    err = np.abs(o - o_ref)
    tol = 2.0 ** -4 * a_ref + 1e-2
    bad = err > tol
    assert not bad.any(), f"{what}: {int(bad.sum())} elements out of tolerance, worst {float((err - tol).max())}"
    assert float(err.mean()) <= 1e-2, f"{what}: mean error {float(err.mean())}"
    return float(err.max()), float(err.mean())


CASES = [(1, 128, 128, 2, 1, 1), (2, 300, 300, 4, 2, 0), (1, 200, 333, 8, 8, 1), (1, 1, 1, 1, 1, 0),
         (2, 700, 700, 16, 2, 1)]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_fp8_small(orc, case):
    B, Nq, Nk, Hq, Hkv, causal = case
    q8, k8, v8 = _fp8_problem(9300 + Nq + Nk, B, Nq, Nk, Hq, Hkv)
    scale = 1.0 / math.sqrt(128)
    o, lse = _run(q8, k8, v8, bool(causal), scale)
    o_ref, lse_ref = orc.attention(q8[1], k8[1], v8[1], scale, causal=bool(causal))
    a_ref, _ = orc.attention(q8[1], k8[1], np.abs(v8[1]), scale, causal=bool(causal))
    _check(o, o_ref, a_ref)
    check_lse(lse, lse_ref)


def test_fp8_gqa_causal_8k_sampled(orc):
    """B=1, Hq=64, Hkv=8, N=8192, d=128, causal, e4m3 inputs: 4096 sampled rows (all heads,
    first and last tiles included) against the oracle, and a bitwise repeat."""
    w = si.WORKLOADS["gqa_causal_8k"]
    B, N, Hq, Hkv, d = w["B"], w["N"], w["Hq"], w["Hkv"], w["d"]
    q8, k8, v8 = _fp8_problem(w["seed"], B, N, N, Hq, Hkv, d)
    scale = 1.0 / math.sqrt(d)
    o, lse = _run(q8, k8, v8, True, scale)
    o2, lse2 = _run(q8, k8, v8, True, scale)
    assert np.array_equal(o, o2) and np.array_equal(lse, lse2)
    u = si.uniform_ints(77, 13, 2 * 4096, 0, (1 << 30))
    rows = np.stack([np.zeros(4096, np.int64), u[0::2] % Hq, u[1::2] % N], 1)
    rows[:64, 2] = np.arange(64)
    rows[64:128, 2] = N - 1 - np.arange(64)
    o_ref, lse_ref = orc.attention_rows(q8[1], k8[1], v8[1], scale, rows, causal=True)
    a_ref, _ = orc.attention_rows(q8[1], k8[1], np.abs(v8[1]), scale, rows, causal=True)
    o_s = o[rows[:, 0], rows[:, 2], rows[:, 1]]
    lse_s = lse[rows[:, 0], rows[:, 1], rows[:, 2]]
    _check(o_s, o_ref, a_ref)
    check_lse(lse_s, lse_ref)
