"""GPU parity of fa_bwd_varlen (through the C ABI): packed variable-length sequences against
the fp64 oracle's varlen backward on the same bf16 inputs, and, at the size of the varlen
forward workload, against per-sequence runs of the fixed-length backward (attention, and so
every gradient, stays inside its sequence).  The forward that the backward needs (o, lse)
is fa_fwd's varlen forward, as a caller would run it."""
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


def _inputs(seed, lengths, Hq, Hkv, d, total=None):
    cu = si.cu_seqlens(lengths)
    T = int(cu[-1]) if total is None else total
    q = si.normal(seed, si.Q, (T, Hq, d))
    k = si.normal(seed, si.K, (T, Hkv, d))
    v = si.normal(seed, si.V, (T, Hkv, d))
    do = si.normal(seed, DOUT, (T, Hq, d))
    return cu, q, k, v, do


def _gpu_bwd_varlen(cu, q, k, v, do, causal, scale):
    tq, tk, tv, tdo = dev_bf16(q), dev_bf16(k), dev_bf16(v), dev_bf16(do)
    cud = torch.from_numpy(cu).cuda()
    o, lse = fa.forward(tq, tk, tv, causal=causal, scale=scale, cu_seqlens=cud)
    dq, dk, dv = fa.backward_varlen(tq, tk, tv, o, lse, tdo, cud, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    return dq, dk, dv


CASES = [
    # lengths, Hq, Hkv, d, causal
    ([1, 130, 256, 257, 511, 3], 4, 2, 128, 1),
    ([600, 0, 17, 1024, 255], 8, 2, 64, 1),
    ([300, 129], 4, 4, 128, 0),
    ([77, 0, 0, 64], 2, 1, 64, 0),
    ([2000], 2, 1, 128, 1),
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_bwd_varlen_small(orc, case):
    lengths, Hq, Hkv, d, causal = case
    cu, q, k, v, do = _inputs(9300 + sum(lengths) + d, lengths, Hq, Hkv, d)
    scale = 1.0 / math.sqrt(d)
    dq, dk, dv = _gpu_bwd_varlen(cu, q, k, v, do, causal, scale)
    rq, rk, rv = orc.attention_bwd(q, k, v, do, scale, causal=bool(causal), cu_seqlens=cu)
    check_grad(host64(dq), rq, "dQ")
    check_grad(host64(dk), rk, "dK")
    check_grad(host64(dv), rv, "dV")


def test_bwd_varlen_rows_outside_sequences():
    """Rows past cu_seqlens[B] belong to no sequence: their dq is 0; the sequences' own
    gradients are those of the same call without the extra rows."""
    lengths, Hq, Hkv, d = [200, 0, 70], 4, 2, 128
    cu, q, k, v, do = _inputs(9401, lengths, Hq, Hkv, d, total=300)
    scale = 1.0 / math.sqrt(d)
    dq, dk, dv = _gpu_bwd_varlen(cu, q, k, v, do, True, scale)
    n = int(cu[-1])
    dq2, dk2, dv2 = _gpu_bwd_varlen(cu, q[:n], k[:n], v[:n], do[:n], True, scale)
    assert torch.count_nonzero(dq[n:]).item() == 0
    for a, b in ((dq, dq2), (dk, dk2), (dv, dv2)):
        x, y = host64(a[:n]), host64(b)
        assert np.abs(x - y).max() <= 1e-2 * max(np.abs(y).max(), 1e-30)


def test_bwd_varlen_bad_seqlens_reported():
    """A cu_seqlens that decreases is found on the device: nothing is computed (dq = 0) and
    fa_last_device_error reports FA_ERR_INVALID_ARG; the next valid call is unaffected."""
    Hq, Hkv, d, T = 2, 1, 64, 256
    _, q, k, v, do = _inputs(9501, [T], Hq, Hkv, d)
    tq, tk, tv, tdo = dev_bf16(q), dev_bf16(k), dev_bf16(v), dev_bf16(do)
    good = torch.tensor([0, 100, T], dtype=torch.int32, device="cuda")
    o, lse = fa.forward(tq, tk, tv, causal=True, cu_seqlens=good)
    torch.cuda.synchronize()
    bad = torch.tensor([0, 200, 100], dtype=torch.int32, device="cuda")
    dq, _, _ = fa.backward_varlen(tq, tk, tv, o, lse, tdo, bad, causal=True)
    assert fa.fa_last_device_error() == fa.FA_ERR_INVALID_ARG
    assert torch.count_nonzero(dq).item() == 0
    over = torch.tensor([0, 100, T + 1], dtype=torch.int32, device="cuda")
    fa.backward_varlen(tq, tk, tv, o, lse, tdo, over, causal=True)
    assert fa.fa_last_device_error() == fa.FA_ERR_INVALID_ARG
    fa.backward_varlen(tq, tk, tv, o, lse, tdo, good, causal=True)
    assert fa.fa_last_device_error() == fa.FA_OK


def test_bwd_varlen_gqa_causal_workload(orc):
    """16 sequences, lengths U[256, 8192] from the seed, Hq=32, Hkv=8, d=128, causal, packed
    (the varlen forward workload), in one launch.  Every sequence's gradients equal a
    fixed-length backward of that sequence alone (dQ within rounding of the order of its
    fp32 reductions), and the oracle checks one K/V group of each of the two shortest
    sequences element by element."""
    w = si.WORKLOADS["varlen_gqa_causal"]
    lengths = si.varlen_lengths(w["seed"], w["nseq"], w["len_lo"], w["len_hi"])
    Hq, Hkv, d = w["Hq"], w["Hkv"], w["d"]
    cu, q, k, v, do = _inputs(w["seed"], lengths, Hq, Hkv, d)
    scale = 1.0 / math.sqrt(d)
    dq, dk, dv = _gpu_bwd_varlen(cu, q, k, v, do, True, scale)
    tq, tk, tv, tdo = dev_bf16(q), dev_bf16(k), dev_bf16(v), dev_bf16(do)
    for b in range(len(lengths)):
        s = slice(int(cu[b]), int(cu[b + 1]))
        qb, kb, vb, dob = (t[s].unsqueeze(0).contiguous() for t in (tq, tk, tv, tdo))
        o, lse = fa.forward(qb, kb, vb, causal=True, scale=scale)
        gq, gk, gv = fa.backward(qb, kb, vb, o, lse, dob, causal=True, scale=scale)
        torch.cuda.synchronize()
        for name, a, ref in (("dQ", dq[s], gq[0]), ("dK", dk[s], gk[0]), ("dV", dv[s], gv[0])):
            x, y = host64(a), host64(ref)
            assert np.abs(x - y).max() <= 1e-2 * np.abs(y).max(), (b, name)
    G = Hq // Hkv
    for b, g in zip(np.argsort(lengths)[:2], (3, 6)):
        s = slice(int(cu[b]), int(cu[b + 1]))
        hs = slice(g * G, (g + 1) * G)
        rq, rk, rv = orc.attention_bwd(q[s][None, :, hs], k[s][None, :, g:g + 1], v[s][None, :, g:g + 1],
                                       do[s][None, :, hs], scale, causal=True)
        check_grad(host64(dq[s][:, hs]), rq[0], "dQ")
        check_grad(host64(dk[s][:, g:g + 1]), rk[0], "dK")
        check_grad(host64(dv[s][:, g:g + 1]), rv[0], "dV")
