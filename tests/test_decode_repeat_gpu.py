"""Repeatability of fa_decode when two split CTAs share an SM: the split partials of many
back-to-back calls on one problem must be bitwise identical.  A missing cross-proxy fence
between the warps' shared-memory reads and the next TMA refill of the same stage once let a
refill overwrite V under a reader, only when a late CTA joined a running one on its SM."""
import math

import pytest
import torch

import synth_inputs as si
from exact_io_aware_97_b200 import binding as fa
from parity import dev_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("lens", [[5000, 1, 2600, 4097], [4097, 5000, 2600, 1]])
def test_decode_partials_repeat_bitwise(lens):
    seed, B, Hq, Hkv, L, d, split = 2101, 4, 32, 4, 5000, 128, 512
    q = dev_bf16(si.normal(seed, si.Q, (B, Hq, d)))
    kc = dev_bf16(si.normal(seed, si.KCACHE, (B, L, Hkv, d)))
    vc = dev_bf16(si.normal(seed, si.VCACHE, (B, L, Hkv, d)))
    ld = torch.tensor(lens, dtype=torch.int32, device="cuda")
    nsplit = (L + split - 1) // split
    wsb = fa.fa_decode_workspace_size(B, Hq, L, d, split)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    o = torch.empty((B, Hq, d), dtype=torch.bfloat16, device="cuda")
    nacc = B * Hq * nsplit * d
    first = None
    for _ in range(200):
        fa.fa_decode(q, kc, vc, ld, o, None, B, Hq, Hkv, L, d, 1 / math.sqrt(d), split, ws, wsb)
        part = ws[: nacc * 4].view(torch.float32).view(B, Hq, nsplit, d)
        # only the splits that hold keys are written
        live = torch.zeros(B, 1, nsplit, 1, dtype=torch.bool, device="cuda")
        for b, n in enumerate(lens):
            live[b, 0, : (n + split - 1) // split] = True
        cur = torch.where(live, part, torch.zeros_like(part))
        if first is None:
            first = cur.clone()
        else:
            assert torch.equal(cur, first)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
