"""fa_decode_noalloc, the decode entry point for callers that cannot allocate device memory
(its scratch is a static device array inside the library).  Checked through the C ABI
against the regular fa_decode entry point on the same inputs, on two calls in a row with
different problems, so that the shared scratch's leftover contents cannot leak into a
result.  Collected last on purpose."""
import math

import numpy as np
import pytest
import torch

import synth_inputs as si
from exact_io_aware_97_b200 import binding as fa
from parity import check_lse, check_out, dev_bf16, host64

pytestmark = pytest.mark.gpu


def _problem(seed, B, Hq, Hkv, L, d, lens):
    q = dev_bf16(si.normal(seed, si.Q, (B, Hq, d)))
    kc = dev_bf16(si.normal(seed, si.KCACHE, (B, L, Hkv, d)))
    vc = dev_bf16(si.normal(seed, si.VCACHE, (B, L, Hkv, d)))
    return q, kc, vc, torch.tensor(lens, dtype=torch.int32, device="cuda")


def _noalloc(q, kc, vc, lens, split):
    B, Hq, d = q.shape
    L, Hkv = kc.shape[1], kc.shape[2]
    o = torch.full((B, Hq, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device="cuda")
    fa.fa_decode_noalloc(q, kc, vc, lens, o, lse, B, Hq, Hkv, L, d, 1.0 / math.sqrt(d), split)
    return o, lse


def test_noalloc_decode_matches_regular_decode_twice():
    """Two problems in a row through the shared scratch.  The static-scratch entry point runs
    the same kernels as fa_decode, so the results must be bitwise equal; the first problem is
    also checked against the oracle, and the second holds an empty sequence (length 0), whose
    row must come out as o = 0 and lse = -inf even though the scratch holds the first
    problem's partials."""
    import oracle as oracle_mod
    orc = oracle_mod.get()
    problems = [
        (2101, 4, 32, 4, 5000, 128, [5000, 1, 2600, 4097], 512),
        (2102, 3, 16, 2, 3000, 64, [1500, 0, 3000], 256),
    ]
    for n, (seed, B, Hq, Hkv, L, d, lens, split) in enumerate(problems):
        q, kc, vc, ld = _problem(seed, B, Hq, Hkv, L, d, lens)
        o, lse = _noalloc(q, kc, vc, ld, split)
        o_ref, lse_ref = fa.decode(q, kc, vc, ld, scale=1.0 / math.sqrt(d), split_len=split)
        torch.cuda.synchronize()
        assert fa.fa_last_device_error() == fa.FA_OK
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref), f"problem {n}: differs from fa_decode"
        if n == 0:
            o64, l64 = orc.decode(host64(q), host64(kc), host64(vc), np.array(lens, np.int32), 1.0 / math.sqrt(d))
            check_out(host64(o), o64, what="noalloc O vs oracle")
            check_lse(host64(lse), l64, what="noalloc lse vs oracle")
        for b, n_b in enumerate(lens):
            if n_b == 0:
                assert np.all(host64(o)[b] == 0) and np.all(np.isneginf(host64(lse)[b]))


def test_noalloc_decode_rejects_problems_beyond_its_scratch():
    # 32 sequences x 16 heads x 128 splits of 64 rows, d=64: 17.3 MB of partials > 16 MiB
    B, Hq, Hkv, L, d, split = 32, 16, 1, 8192, 64, 64
    assert fa.fa_decode_workspace_size(B, Hq, L, d, split) > fa.FA_DECODE_NOALLOC_SCRATCH_BYTES
    q = torch.zeros(B, Hq, d, dtype=torch.bfloat16, device="cuda")
    c = torch.zeros(B, L, Hkv, d, dtype=torch.bfloat16, device="cuda")
    o = torch.zeros(B, Hq, d, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fa.FaError) as e:
        fa.fa_decode_noalloc(q, c, c, None, o, None, B, Hq, Hkv, L, d, 0.125, split)
    assert e.value.status == fa.FA_ERR_WORKSPACE
    assert np.all(host64(o) == 0)  # nothing was launched
