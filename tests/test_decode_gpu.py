"""GPU parity of fa_decode (split-KV kernel + merge kernel, through the C ABI) against the
fp64 oracle's plain single-row definition (which never merges)."""
import math

import numpy as np
import pytest
import torch

import oracle as oracle_mod
import synth_inputs as si
from exact_io_aware_97_b200 import binding as fa
from parity import check_lse, check_out, dev_bf16, host64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def orc():
    return oracle_mod.get()


def _cache(seed, B, Hq, Hkv, L, d):
    q = si.normal(seed, si.Q, (B, Hq, d))
    kc = si.normal(seed, si.KCACHE, (B, L, Hkv, d))
    vc = si.normal(seed, si.VCACHE, (B, L, Hkv, d))
    return q, kc, vc


CASES = [
    # B, Hq, Hkv, Lmax, d, split, seqlens (None = all Lmax)
    (3, 8, 2, 1000, 128, 256, [1000, 1, 513]),
    (3, 8, 2, 1000, 64, 256, [999, 64, 65]),
    (2, 16, 1, 2048, 128, 512, None),
    (4, 4, 4, 300, 128, 64, [300, 0, 129, 64]),
    (1, 12, 3, 5000, 64, 1024, [4097]),
    (2, 64, 8, 4096, 128, 1024, [4096, 2500]),
]


@pytest.mark.parametrize("case", CASES, ids=[str(c[:6]) for c in CASES])
def test_decode_small(orc, case):
    B, Hq, Hkv, L, d, split, lens = case
    q, kc, vc = _cache(9000 + L + d + Hq, B, Hq, Hkv, L, d)
    scale = 1.0 / math.sqrt(d)
    lens_np = np.full(B, L, np.int32) if lens is None else np.array(lens, np.int32)
    lens_d = None if lens is None else torch.from_numpy(lens_np).cuda()
    o, lse = fa.decode(dev_bf16(q), dev_bf16(kc), dev_bf16(vc), lens_d, scale=scale, split_len=split)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    o_ref, lse_ref = orc.decode(q, kc, vc, lens_np, scale)
    check_out(host64(o), o_ref)
    check_lse(host64(lse), lse_ref)
    empty = lens_np == 0
    if empty.any():
        assert np.all(host64(o)[empty] == 0) and np.all(np.isneginf(host64(lse)[empty]))


@pytest.mark.parametrize("seed_off", [0, 10000, 20000])
def test_decode_split_kv_full(orc, seed_off):
    """B=8, Hq=64, Hkv=8, d=128, cache 32768, splits of 1024 (the benchmark workload, same
    launch), three seeds: every (sequence, head) against the oracle, plus bitwise
    repeatability."""
    w = si.WORKLOADS["decode_split_kv"]
    B, Hq, Hkv, L, d, split = w["B"], w["Hq"], w["Hkv"], w["L"], w["d"], w["split"]
    q, kc, vc = _cache(w["seed"] + seed_off, B, Hq, Hkv, L, d)
    scale = 1.0 / math.sqrt(d)
    qd, kd, vd = dev_bf16(q), dev_bf16(kc), dev_bf16(vc)
    o1, l1 = fa.decode(qd, kd, vd, None, scale=scale, split_len=split)
    o2, l2 = fa.decode(qd, kd, vd, None, scale=scale, split_len=split)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    o_ref, lse_ref = orc.decode(q, kc, vc, np.full(B, L, np.int32), scale)
    check_out(host64(o1), o_ref)
    check_lse(host64(l1), lse_ref)


def test_decode_rejects_large_group():
    q = torch.zeros(1, 32, 128, dtype=torch.bfloat16, device="cuda")
    c = torch.zeros(1, 64, 1, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fa.FaError) as e:
        fa.decode(q, c, c, split_len=64)
    assert e.value.status == fa.FA_ERR_UNSUPPORTED
