"""Pins of the oracle's paged decode ("LLM basics: from Attention to FlashAttention",
chapter 2 section 8, PagedAttention: fixed-size pages of the KV cache, found through a
per-sequence block table) to facts that do not come from the oracle itself:

* a pool that is the contiguous cache cut into pages, with the identity table, gives the
  contiguous decode;
* shuffling the physical pages and the table with them changes nothing;
* sequences that share their first pages (a shared prefix) and their query agree exactly;
* a brute force over the page table on tiny inputs (Python floats, explicit loops).

Planted mistakes in the page gather (swapped page/row index, an off-by-one page) must fail
at least one of them.
"""
import math

import numpy as np
import pytest

import oracle as oracle_mod
import synth_inputs as si

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _rand(shape, seed, tid):
    return si.normal(seed, tid, shape, dtype="f32").astype(np.float32)


def _cut_into_pages(cache, ps):
    """[B, L, H, d] (L a multiple of ps) -> pool [B*L/ps, ps, H, d] and the identity table."""
    B, L, H, d = cache.shape
    pool = cache.reshape(B * (L // ps), ps, H, d)
    table = np.arange(B * (L // ps), dtype=np.int32).reshape(B, L // ps)
    return pool, table


def pin_identity_table(orc):
    B, Hq, Hkv, d, ps, L = 3, 4, 2, 16, 8, 40
    q = _rand((B, Hq, d), 7001, si.Q)
    kc = _rand((B, L, Hkv, d), 7001, si.KCACHE)
    vc = _rand((B, L, Hkv, d), 7001, si.VCACHE)
    lens = np.array([40, 13, 1], dtype=np.int32)
    kp, table = _cut_into_pages(kc, ps)
    vp, _ = _cut_into_pages(vc, ps)
    o, lse = orc.decode_paged(q, kp, vp, table, lens, ps, 0.25)
    o_ref, lse_ref = orc.decode(q, kc, vc, lens, 0.25)
    return np.array_equal(o, o_ref) and np.array_equal(lse, lse_ref)


def pin_shuffled_pool(orc):
    B, Hq, Hkv, d, ps, L = 2, 2, 1, 8, 4, 24
    q = _rand((B, Hq, d), 7002, si.Q)
    kc = _rand((B, L, Hkv, d), 7002, si.KCACHE)
    vc = _rand((B, L, Hkv, d), 7002, si.VCACHE)
    lens = np.array([23, 9], dtype=np.int32)
    kp, table = _cut_into_pages(kc, ps)
    vp, _ = _cut_into_pages(vc, ps)
    perm = si.permutation(7002, si.PAGES, kp.shape[0])  # physical slot of each page
    kp2, vp2 = np.empty_like(kp), np.empty_like(vp)
    kp2[perm], vp2[perm] = kp, vp
    table2 = perm[table].astype(np.int32)
    o, lse = orc.decode_paged(q, kp2, vp2, table2, lens, ps, 0.5)
    o_ref, lse_ref = orc.decode(q, kc, vc, lens, 0.5)
    return np.array_equal(o, o_ref) and np.array_equal(lse, lse_ref)


def pin_shared_prefix(orc):
    # sequences 0 and 1 share pages 0..2 (12 tokens) and their query; sequence 1 then
    # diverges on its own page, sequence 2 is the shared prefix alone.
    ps, Hkv, d = 4, 1, 8
    pool_k = _rand((6, ps, Hkv, d), 7003, si.KCACHE)
    pool_v = _rand((6, ps, Hkv, d), 7003, si.VCACHE)
    q1 = _rand((1, 2, d), 7003, si.Q)
    q = np.concatenate([q1, q1, q1])
    table = np.array([[0, 1, 2, 3], [0, 1, 2, 5], [0, 1, 2, -1]], dtype=np.int32)
    lens = np.array([12, 15, 12], dtype=np.int32)
    o, lse = orc.decode_paged(q, pool_k, pool_v, table, lens, ps, 0.3)
    prefix_ok = np.array_equal(o[0], o[2]) and np.array_equal(lse[0], lse[2])
    diverged = not np.allclose(o[0], o[1])
    return prefix_ok and diverged


def pin_brute_force(orc):
    ps, Hq, Hkv, d = 2, 4, 2, 3
    pool_k = _rand((7, ps, Hkv, d), 7004, si.KCACHE)
    pool_v = _rand((7, ps, Hkv, d), 7004, si.VCACHE)
    q = _rand((2, Hq, d), 7004, si.Q)
    table = np.array([[6, 2, 0, 4], [1, 3, 5, -1]], dtype=np.int32)
    lens = np.array([7, 5], dtype=np.int32)
    scale = 0.7
    o, lse = orc.decode_paged(q, pool_k, pool_v, table, lens, ps, scale)
    G = Hq // Hkv
    for b in range(2):
        for h in range(Hq):
            kv = h // G
            s = []
            for j in range(int(lens[b])):
                page, row = int(table[b][j // ps]), j % ps
                s.append(scale * sum(float(q[b, h, c]) * float(pool_k[page, row, kv, c]) for c in range(d)))
            m = max(s)
            w = [math.exp(x - m) for x in s]
            z = sum(w)
            for c in range(d):
                ref = sum(w[j] * float(pool_v[int(table[b][j // ps]), j % ps, kv, c]) for j in range(len(s))) / z
                if abs(o[b, h, c] - ref) > 1e-12:
                    return False
            if abs(lse[b, h] - (m + math.log(z))) > 1e-12:
                return False
    return True


PINS = [pin_identity_table, pin_shuffled_pool, pin_shared_prefix, pin_brute_force]


@pytest.fixture(scope="module")
def orc():
    return oracle_mod.get()


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_paged_pin(orc, pin):
    assert pin(orc)


def _gather_swapped(pages, block_table, seqlens, page_size):
    pages, table = np.asarray(pages), np.asarray(block_table)
    B, maxp = table.shape
    out = np.zeros((B, maxp * page_size) + pages.shape[2:], dtype=pages.dtype)
    for b in range(B):
        for j in range(int(seqlens[b])):
            out[b, j] = pages[table[b, min(j % page_size, maxp - 1)], min(j // page_size, page_size - 1)]
    return out


def _gather_next_page(pages, block_table, seqlens, page_size):
    pages, table = np.asarray(pages), np.asarray(block_table)
    B, maxp = table.shape
    out = np.zeros((B, maxp * page_size) + pages.shape[2:], dtype=pages.dtype)
    for b in range(B):
        for j in range(int(seqlens[b])):
            t = min(j // page_size + 1, int((seqlens[b] - 1) // page_size))
            out[b, j] = pages[table[b, t], j % page_size]
    return out


@pytest.mark.parametrize("wrong", [_gather_swapped, _gather_next_page], ids=lambda f: f.__name__)
def test_paged_pins_catch_planted_gather(orc, monkeypatch, wrong):
    monkeypatch.setattr(oracle_mod.Oracle, "gather_pages", staticmethod(wrong))
    assert not all(pin(orc) for pin in PINS)


def test_page_layout_is_a_valid_placement():
    lens = [33, 0, 16, 1, 100]
    table, num_pages = si.page_layout(11, lens, 16, extra_pages=5)
    used = [int(p) for b, n in enumerate(lens) for p in table[b, :(n + 15) // 16]]
    assert len(used) == len(set(used)) and all(0 <= p < num_pages for p in used)
    assert num_pages == sum((n + 15) // 16 for n in lens) + 5
    assert (table[1] == -1).all() and (table[3, 1:] == -1).all()
