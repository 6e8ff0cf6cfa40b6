"""GPU parity of fa_decode_paged (paged split-KV decode with the merge done by the last
split of each group, through the C ABI) against the fp64 oracle, which gathers each
sequence's cache through the block table and applies the plain single-row definition."""
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


def _problem(seed, B, Hq, Hkv, d, ps, lens, extra, poison=True):
    """Host arrays of a paged problem.  With `poison`, rows past each sequence's end in its
    last page and every spare page hold NaN: a correct kernel never lets them into O."""
    table, num_pages = si.page_layout(seed, lens, ps, extra_pages=extra)
    q = si.normal(seed, si.Q, (B, Hq, d))
    kp = si.normal(seed, si.KCACHE, (num_pages, ps, Hkv, d))
    vp = si.normal(seed, si.VCACHE, (num_pages, ps, Hkv, d))
    if poison:
        used = np.zeros(num_pages, bool)
        for b, n in enumerate(lens):
            npg = (n + ps - 1) // ps
            used[table[b, :npg]] = True
            if n % ps:
                kp[table[b, npg - 1], n % ps:] = np.nan
                vp[table[b, npg - 1], n % ps:] = np.nan
        kp[~used] = np.nan
        vp[~used] = np.nan
    return q, kp, vp, table, np.array(lens, np.int32)


def _run(q, kp, vp, table, lens, scale, split, ws=None):
    return fa.decode_paged(dev_bf16(q), dev_bf16(kp), dev_bf16(vp), torch.from_numpy(table).cuda(),
                           torch.from_numpy(lens).cuda(), scale=scale, split_len=split, workspace=ws)


CASES = [
    # seed, B, Hq, Hkv, d, page_size, seqlens, split_len, spare pages
    (3001, 4, 32, 4, 128, 16, [1000, 1, 0, 333], 256, 3),
    (3002, 3, 16, 2, 64, 32, [64, 65, 700], 128, 0),
    (3003, 2, 8, 8, 128, 64, [4096, 4095], 1024, 2),
    (3004, 5, 64, 4, 128, 128, [1, 127, 128, 129, 2000], 512, 1),
    (3005, 2, 16, 2, 128, 256, [5000, 300], 1024, 0),
    (3006, 3, 8, 1, 64, 512, [512, 513, 1], 64, 4),
    (3007, 2, 12, 3, 64, 16, [16, 17], 64, 1),
]


@pytest.mark.parametrize("case", CASES, ids=[f"ps{c[5]}_G{c[2] // c[3]}_d{c[4]}" for c in CASES])
def test_decode_paged_small(orc, case):
    seed, B, Hq, Hkv, d, ps, lens, split, extra = case
    q, kp, vp, table, lens_np = _problem(seed, B, Hq, Hkv, d, ps, lens, extra)
    scale = 1.0 / math.sqrt(d)
    # a workspace full of garbage bytes: nothing in it needs initialising
    ws = torch.full((fa.fa_decode_paged_workspace_size(B, Hq, Hkv, table.shape[1], ps, d, split),), 0xFF,
                    dtype=torch.uint8, device="cuda")
    o, lse = _run(q, kp, vp, table, lens_np, scale, split, ws)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    o_ref, lse_ref = orc.decode_paged(q, kp, vp, table, lens_np, ps, scale)
    check_out(host64(o), o_ref)
    check_lse(host64(lse), lse_ref)
    empty = lens_np == 0
    if empty.any():
        assert np.all(host64(o)[empty] == 0) and np.all(np.isneginf(host64(lse)[empty]))
    # the same workspace, reused, gives the same bits again
    o2, lse2 = _run(q, kp, vp, table, lens_np, scale, split, ws)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(lse, lse2)


def test_decode_paged_workspace_reused_across_problems(orc):
    """One workspace serves a sequence of different problems."""
    ws = torch.zeros(8 << 20, dtype=torch.uint8, device="cuda")
    for seed, B, Hq, Hkv, d, ps, lens, split, extra in [CASES[0], CASES[3], CASES[1], CASES[0]]:
        q, kp, vp, table, lens_np = _problem(seed, B, Hq, Hkv, d, ps, lens, extra)
        assert fa.fa_decode_paged_workspace_size(B, Hq, Hkv, table.shape[1], ps, d, split) <= ws.numel()
        scale = 1.0 / math.sqrt(d)
        o, lse = _run(q, kp, vp, table, lens_np, scale, split, ws)
        torch.cuda.synchronize()
        o_ref, lse_ref = orc.decode_paged(q, kp, vp, table, lens_np, ps, scale)
        check_out(host64(o), o_ref)
        check_lse(host64(lse), lse_ref)


def test_decode_paged_reports_bad_page_index():
    seed, B, Hq, Hkv, d, ps, lens, split, extra = CASES[1]
    q, kp, vp, table, lens_np = _problem(seed, B, Hq, Hkv, d, ps, lens, extra, poison=False)
    table = table.copy()
    table[2, 3] = kp.shape[0] + 1000   # a used entry outside the pool
    o, lse = _run(q, kp, vp, table, lens_np, 0.125, split)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_ERR_INVALID_ARG
    assert torch.isfinite(o.float()).all()
    assert fa.fa_last_device_error() == fa.FA_OK    # the record was cleared


def test_decode_paged_ragged_full(orc):
    """16 sequences of U{1..32768} tokens in a shuffled pool of 16-token pages, Hq=64,
    Hkv=8, d=128, splits of 1024 (the benchmark's paged workload, same launch): every
    (sequence, head) against the oracle."""
    w = si.WORKLOADS["decode_paged_ragged"]
    lens = si.uniform_ints(w["seed"], si.LENGTHS, w["B"], w["len_lo"], w["len_hi"]).tolist()
    q, kp, vp, table, lens_np = _problem(w["seed"], w["B"], w["Hq"], w["Hkv"], w["d"], w["page_size"], lens, 0,
                                         poison=False)
    scale = 1.0 / math.sqrt(w["d"])
    o, lse = _run(q, kp, vp, table, lens_np, scale, w["split"])
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    o_ref, lse_ref = orc.decode_paged(q, kp, vp, table, lens_np, w["page_size"], scale)
    check_out(host64(o), o_ref)
    check_lse(host64(lse), lse_ref)
