"""GPU parity of fa_fwd_qkvpacked (q, k, v read in place from one packed [B, N, 3, H, d]
tensor) against the fp64 oracle, and bitwise agreement with fa_fwd on the unpacked slices."""
import math

import numpy as np
import pytest
import torch

import oracle as oracle_mod
import synth_inputs as si
from exact_io_aware_97_b200 import binding as fa
from parity import check_lse, check_out, dev_bf16, host64

pytestmark = pytest.mark.gpu

QKV = 10  # stream id of the packed tensor


@pytest.fixture(scope="module")
def orc():
    return oracle_mod.get()


@pytest.mark.parametrize("B,N,H,d,causal", [(2, 2048, 12, 64, 1), (1, 300, 4, 128, 0), (3, 129, 2, 64, 1)])
def test_qkvpacked_matches_oracle_and_unpacked(orc, B, N, H, d, causal):
    w = si.WORKLOADS["mha_causal_2k"]
    seed = w["seed"] if (B, N, H, d) == (w["B"], w["N"], w["Hq"], w["d"]) else 8800 + N
    qkv = si.normal(seed, QKV, (B, N, 3, H, d))
    scale = 1.0 / math.sqrt(d)
    t = dev_bf16(qkv)
    o, lse = fa.forward_qkvpacked(t, causal=bool(causal), scale=scale)
    o2, lse2 = fa.forward(t[:, :, 0].contiguous(), t[:, :, 1].contiguous(), t[:, :, 2].contiguous(),
                          causal=bool(causal), scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    o_ref, lse_ref = orc.attention(qkv[:, :, 0], qkv[:, :, 1], qkv[:, :, 2], scale, causal=bool(causal))
    check_out(host64(o), o_ref)
    check_lse(host64(lse), lse_ref)


def test_qkvpacked_varlen(orc):
    lens = [100, 257, 1]
    cu = si.cu_seqlens(lens)
    total, H, d = int(cu[-1]), 4, 128
    qkv = si.normal(8901, QKV, (total, 3, H, d))
    scale = 1.0 / math.sqrt(d)
    o, lse = fa.forward_qkvpacked(dev_bf16(qkv), causal=True, scale=scale,
                                  cu_seqlens=torch.from_numpy(cu).cuda())
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    o_ref, lse_ref = orc.attention(qkv[:, 0], qkv[:, 1], qkv[:, 2], scale, causal=True, cu_seqlens=cu)
    check_out(host64(o), o_ref)
    check_lse(host64(lse), lse_ref)
