"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each pin is a function of an oracle instance.  The real oracle must pass every pin, and
for each planted mistake (a copy of oracle.cpp built with one ORACLE_PLANT_* switch) at
least one pin must fail, so the pins are shown to catch a dropped scale, a flipped sign,
swapped K/V operands, an lse missing its max term, a causal off-by-one and a wrong GQA map.

Sources: the printed values of "LLM basics: from Attention to FlashAttention"
(tests/golden/*.json, each with its citation), closed forms, invariances the pages state,
and a 40-digit brute force on tiny inputs.
"""
import json
import math
import os
from decimal import Decimal, getcontext

import numpy as np
import pytest
from scipy.special import expit, softmax as sp_softmax

import oracle as oracle_mod
import synth_inputs as si

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def orc():
    return oracle_mod.get()


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rand(shape, seed, tid):
    return si.normal(seed, tid, shape, dtype="f32").astype(np.float32)


# --------------------------------------------------------------------------- pins
def pin_worked_example(orc):
    """The page's hand-worked 3-token example: printed scores, softmax and output (2 d.p.),
    plus the exact closed form O = [2e^a, 2+e^a] / (2e^a + 1), a = 1/sqrt(2)."""
    g = _load("worked_example.json")
    q = np.array(g["q"], dtype=np.float32).reshape(1, 1, 1, 2)
    k = np.array(g["k"], dtype=np.float32).reshape(1, 3, 1, 2)
    v = np.array(g["v"], dtype=np.float32).reshape(1, 3, 1, 2)
    scale = 1.0 / math.sqrt(g["d_k"])
    o, lse = orc.attention(q, k, v, scale)
    pr = g["printed"]
    dec = pr["decimals"]
    tol = 0.5 * 10.0 ** (-dec) + 1e-12
    assert np.all(np.abs(o.reshape(2) - np.array(pr["output"])) <= tol), o
    p = orc.softmax(np.array(pr["scores_qkT"]) * scale)
    assert np.all(np.abs(p - np.array(pr["softmax"])) <= tol), p
    # printed exp-sum 5.06 (2 d.p.) bounds lse = ln(sum exp(s))
    lo, hi = math.log(pr["exp_sum"] - 0.005), math.log(pr["exp_sum"] + 0.005)
    assert lo <= float(lse.reshape(())) <= hi, lse
    a = 1.0 / math.sqrt(2.0)
    ea = math.exp(a)
    exact = np.array([2 * ea, 2 + ea]) / (2 * ea + 1)
    assert np.allclose(o.reshape(2), exact, rtol=0, atol=1e-14)
    assert abs(float(lse.reshape(())) - math.log(2 * ea + 1)) < 1e-14


def pin_softmax_printed(orc):
    g = _load("softmax_examples.json")
    for case in g["cases"]:
        p = orc.softmax(np.array(case["x"]))
        tol = 0.5 * 10.0 ** (-case["decimals"]) + 1e-15
        assert np.all(np.abs(p - np.array(case["printed"])) <= tol), (case, p)
        # library routine: scipy's softmax
        assert np.allclose(p, sp_softmax(np.array(case["x"])), rtol=1e-14, atol=0)


def pin_rows_sum_to_one(orc):
    rng_x = _rand((64, 37), 11, 1).astype(np.float64) * 7.0
    for row in rng_x:
        p = orc.softmax(row)
        assert abs(p.sum() - 1.0) <= 1e-12
        assert np.all(p >= 0)


def pin_safe_softmax_no_overflow(orc):
    """exp(x) overflows fp32 above x ~ 88.7 and fp16 above ~11.1 (printed table); the safe
    softmax of scores at and beyond those points stays finite and exact."""
    g = _load("softmax_examples.json")["overflow"]
    assert abs(math.log(g["fp16_max"]) - g["fp16_x"]) < 0.05
    assert abs(math.log(g["fp32_max"]) - g["fp32_x"]) < 0.05
    with np.errstate(over="ignore", invalid="ignore"):
        naive32 = np.exp(np.float32(89.0)) / np.exp(np.float32(89.0))
        naive16 = np.exp(np.float16(12.0))
    assert not np.isfinite(naive32) and not np.isfinite(naive16)
    x = np.array([89.0, 100.0, 1000.0, 999.0])
    p = orc.softmax(x)
    assert np.all(np.isfinite(p))
    assert abs(p[3] / p[2] - math.exp(-1.0)) < 1e-14
    # as attention: one key with a huge score dominates; o equals that key's value
    q = np.array([1.0, 0.0], dtype=np.float32).reshape(1, 1, 1, 2)
    k = np.array([[1000.0, 0.0], [0.0, 0.0], [500.0, 0.0]], dtype=np.float32).reshape(1, 3, 1, 2)
    v = np.array([[3.0, -1.0], [7.0, 7.0], [5.0, 5.0]], dtype=np.float32).reshape(1, 3, 1, 2)
    o, lse = orc.attention(q, k, v, 1.0)
    assert np.allclose(o.reshape(2), [3.0, -1.0], atol=1e-14)
    assert abs(float(lse.reshape(())) - 1000.0) < 1e-12


def pin_online_merge_equals_standard(orc):
    """'FlashAttention notes' section 4: merging blocks with m_new = max(m1, m2),
    l_new = e^(m1-m_new) l1 + e^(m2-m_new) l2 gives the statistics of the whole row, for
    any split.  Checked against a library logsumexp and against unsplit rows."""
    from scipy.special import logsumexp
    x_all = _rand((40, 33), 12, 1).astype(np.float64) * 5.0
    rs = si.uniform_ints(12, 9, 400, 1, 32)
    t = 0
    for row in x_all:
        m_full, l_full = orc.row_stats(row)
        assert abs((m_full + math.log(l_full)) - logsumexp(row)) < 1e-12
        # random split points
        cuts = sorted(set(int(c) for c in rs[t:t + 4]))
        t += 4
        bounds = [0] + cuts + [len(row)]
        M, L = -math.inf, 0.0
        for a, b in zip(bounds[:-1], bounds[1:]):
            m2, l2 = orc.row_stats(row[a:b])
            M, L = orc.merge_stats(M, L, m2, l2)
        assert M == m_full
        assert abs(L - l_full) <= 1e-12 * l_full
    # block size 1..N with partial accumulators (the split-KV merge)
    v = _rand((33, 5), 12, 2).astype(np.float64)
    row = x_all[0]
    w = np.exp(row - row.max())
    ref = (w[:, None] * v).sum(0) / w.sum()
    for bs in range(1, 34):
        ms, ls, accs = [], [], []
        for a in range(0, 33, bs):
            blk = row[a:a + bs]
            m, l = orc.row_stats(blk)
            ms.append(m)
            ls.append(l)
            accs.append((np.exp(blk - m)[:, None] * v[a:a + bs]).sum(0))
        M, L, o = orc.merge_partials(ms, ls, np.array(accs))
        assert M == row.max()
        assert np.allclose(o, ref, rtol=1e-12, atol=1e-14)
    # empty block (m = -inf, l = 0) has weight 0
    M, L, o = orc.merge_partials([-math.inf, 0.5], [0.0, 2.0], np.array([[9.0, 9.0], [4.0, 6.0]]))
    assert M == 0.5 and L == 2.0 and np.allclose(o, [2.0, 3.0])


def pin_constant_v(orc):
    """softmax rows sum to 1, so V rows all equal to c give O = c everywhere."""
    B, N, Hq, Hkv, d = 2, 19, 4, 2, 8
    q = _rand((B, N, Hq, d), 13, 1)
    k = _rand((B, N, Hkv, d), 13, 2)
    c = _rand((d,), 13, 3)
    v = np.broadcast_to(c, (B, N, Hkv, d)).copy()
    for causal in (False, True):
        o, _ = orc.attention(q, k, v, 0.3, causal=causal)
        assert np.allclose(o, np.broadcast_to(c, o.shape), rtol=0, atol=1e-12)


def pin_q_zero_means(orc):
    """Q = 0 makes every allowed score 0: O is the mean of the allowed V rows and
    lse = ln(#allowed).  Causal row i of an (Nq, Nk) problem sees keys j <= i + Nk - Nq."""
    B, Hq, Hkv, d = 2, 2, 1, 4
    for Nq, Nk in ((7, 7), (3, 9), (9, 4)):
        q = np.zeros((B, Nq, Hq, d), dtype=np.float32)
        k = _rand((B, Nk, Hkv, d), 14, 1)
        v = _rand((B, Nk, Hkv, d), 14, 2).astype(np.float32)
        for causal in (False, True):
            o, lse = orc.attention(q, k, v, 0.5, causal=causal)
            for b in range(B):
                for h in range(Hq):
                    for i in range(Nq):
                        n_allowed = min(Nk, i + Nk - Nq + 1) if causal else Nk
                        if n_allowed <= 0:
                            assert np.all(o[b, i, h] == 0) and lse[b, h, i] == -math.inf
                            continue
                        mean = v[b, :n_allowed, 0].astype(np.float64).mean(0)
                        assert np.allclose(o[b, i, h], mean, atol=1e-13)
                        assert abs(lse[b, h, i] - math.log(n_allowed)) < 1e-13


def pin_varlen_q_zero(orc):
    """Varlen with Q = 0: each row averages only its own sequence's causal prefix."""
    lens = [5, 1, 8, 3]
    cu = si.cu_seqlens(lens)
    T, Hq, Hkv, d = int(cu[-1]), 2, 2, 3
    q = np.zeros((T, Hq, d), dtype=np.float32)
    k = _rand((T, Hkv, d), 15, 1)
    v = _rand((T, Hkv, d), 15, 2)
    o, lse = orc.attention(q, k, v, 1.0, causal=True, cu_seqlens=cu)
    for b, L in enumerate(lens):
        for i in range(L):
            rows = v[cu[b]:cu[b] + i + 1].astype(np.float64)
            for h in range(Hq):
                assert np.allclose(o[cu[b] + i, h], rows[:, h].mean(0), atol=1e-13)
                assert abs(lse[h, cu[b] + i] - math.log(i + 1)) < 1e-13


def pin_decode_lengths_q_zero(orc):
    B, Hq, Hkv, L, d = 3, 4, 2, 10, 4
    q = np.zeros((B, Hq, d), dtype=np.float32)
    kc = _rand((B, L, Hkv, d), 16, 1)
    vc = _rand((B, L, Hkv, d), 16, 2)
    lens = np.array([10, 1, 6], dtype=np.int32)
    o, lse = orc.decode(q, kc, vc, lens, 0.7)
    for b in range(B):
        for h in range(Hq):
            g = h // (Hq // Hkv)
            assert np.allclose(o[b, h], vc[b, :lens[b], g].astype(np.float64).mean(0), atol=1e-13)
            assert abs(lse[b, h] - math.log(lens[b])) < 1e-13


def pin_two_keys_closed_form(orc):
    """Two keys: O = sigmoid(s0 - s1) v0 + sigmoid(s1 - s0) v1 and lse = logaddexp(s0, s1)."""
    d = 6
    q = _rand((1, 1, 1, d), 17, 1)
    k = _rand((1, 2, 1, d), 17, 2)
    v = _rand((1, 2, 1, d), 17, 3)
    scale = 0.37
    o, lse = orc.attention(q, k, v, scale)
    s = scale * (k[0, :, 0].astype(np.float64) @ q[0, 0, 0].astype(np.float64))
    w0 = expit(s[0] - s[1])
    ref = w0 * v[0, 0, 0] + (1 - w0) * v[0, 1, 0]
    assert np.allclose(o.reshape(d), ref, atol=1e-14)
    assert abs(float(lse.reshape(())) - np.logaddexp(s[0], s[1])) < 1e-14


def pin_single_key(orc):
    d = 5
    q = _rand((1, 1, 1, d), 18, 1)
    k = _rand((1, 1, 1, d), 18, 2)
    v = _rand((1, 1, 1, d), 18, 3)
    o, lse = orc.attention(q, k, v, 0.25)
    assert np.array_equal(o.reshape(d), v.reshape(d).astype(np.float64))
    assert abs(float(lse.reshape(())) - 0.25 * float(q.reshape(d).astype(np.float64) @ k.reshape(d))) < 1e-14


def pin_shift_invariance(orc):
    """'LLM basics' chapter 3 section 1: adding c to every score of a row leaves softmax
    unchanged.  Append a coordinate (1 in q, c/scale in every k): O unchanged, lse + c."""
    B, N, H, d = 1, 11, 2, 4
    scale = 0.5
    q = _rand((B, N, H, d), 19, 1)
    k = _rand((B, N, H, d), 19, 2)
    v = _rand((B, N, H, d), 19, 3)
    c = 3.0
    q2 = np.concatenate([q, np.ones((B, N, H, 1), np.float32)], -1)
    k2 = np.concatenate([k, np.full((B, N, H, 1), c / scale, np.float32)], -1)
    for causal in (False, True):
        o1, l1 = orc.attention(q, k, v, scale, causal=causal)
        o2, l2 = orc.attention(q2, k2, np.concatenate([v, np.zeros((B, N, H, 1), np.float32)], -1),
                               scale, causal=causal)
        assert np.allclose(o2[..., :d], o1, atol=1e-13)
        assert np.allclose(l2, l1 + c, atol=1e-12)


def pin_scale_equals_scaled_q(orc):
    B, N, H, d = 1, 9, 1, 4
    q = _rand((B, N, H, d), 20, 1)
    k = _rand((B, N, H, d), 20, 2)
    v = _rand((B, N, H, d), 20, 3)
    o1, l1 = orc.attention(q, k, v, 2.0)
    o2, l2 = orc.attention(2.0 * q, k, v, 1.0)
    assert np.allclose(o1, o2, atol=1e-13) and np.allclose(l1, l2, atol=1e-12)


def pin_key_permutation(orc):
    """'LLM basics' chapter 1: attention itself has no notion of order (non-causal)."""
    B, N, H, d = 2, 13, 2, 4
    q = _rand((B, N, H, d), 21, 1)
    k = _rand((B, N, H, d), 21, 2)
    v = _rand((B, N, H, d), 21, 3)
    perm = np.argsort(si.words(si.stream_key(21, 7), 0, N))
    o1, l1 = orc.attention(q, k, v, 0.4)
    o2, l2 = orc.attention(q, k[:, perm], v[:, perm], 0.4)
    assert np.allclose(o1, o2, atol=1e-13) and np.allclose(l1, l2, atol=1e-12)


def pin_causal_rows(orc):
    """Causal row i equals non-causal attention over keys 0..i; the last row equals the
    non-causal result ('LLM basics' chapter 1 section 7)."""
    B, N, H, d = 1, 12, 2, 4
    q = _rand((B, N, H, d), 22, 1)
    k = _rand((B, N, H, d), 22, 2)
    v = _rand((B, N, H, d), 22, 3)
    oc, lc = orc.attention(q, k, v, 0.5, causal=True)
    on, ln = orc.attention(q, k, v, 0.5, causal=False)
    assert np.allclose(oc[:, -1], on[:, -1], atol=1e-13)
    for i in range(N):
        oi, li = orc.attention(q[:, i:i + 1], k[:, :i + 1], v[:, :i + 1], 0.5)
        assert np.allclose(oc[:, i], oi[:, 0], atol=1e-13)
        assert np.allclose(lc[:, :, i], li[:, :, 0], atol=1e-12)


def pin_gqa_equals_repeated_mha(orc):
    """'LLM basics' chapter 2 section 7: G query heads share one K/V head; read as
    contiguous groups, head h uses K/V head h // G.  Equals MHA with K/V repeated."""
    B, N, Hq, Hkv, d = 1, 10, 6, 2, 4
    G = Hq // Hkv
    q = _rand((B, N, Hq, d), 23, 1)
    k = _rand((B, N, Hkv, d), 23, 2)
    v = _rand((B, N, Hkv, d), 23, 3)
    o1, l1 = orc.attention(q, k, v, 0.5, causal=True)
    o2, l2 = orc.attention(q, np.repeat(k, G, axis=2), np.repeat(v, G, axis=2), 0.5, causal=True)
    assert np.allclose(o1, o2, atol=1e-14) and np.allclose(l1, l2, atol=1e-14)


def pin_varlen_equals_independent(orc):
    lens = [4, 9, 1, 6]
    cu = si.cu_seqlens(lens)
    T, Hq, Hkv, d = int(cu[-1]), 4, 2, 4
    q = _rand((T, Hq, d), 24, 1)
    k = _rand((T, Hkv, d), 24, 2)
    v = _rand((T, Hkv, d), 24, 3)
    o, lse = orc.attention(q, k, v, 0.5, causal=True, cu_seqlens=cu)
    for b, L in enumerate(lens):
        s = slice(cu[b], cu[b + 1])
        ob, lb = orc.attention(q[s][None], k[s][None], v[s][None], 0.5, causal=True)
        assert np.allclose(o[s], ob[0], atol=1e-14)
        assert np.allclose(lse[:, s], lb[0], atol=1e-14)


def pin_decode_equals_prefill_last_row(orc):
    """Decode over a cache equals the last row of a causal prefill over the same keys
    ('LLM basics' chapter 2 section 4: the new token attends to every cached token)."""
    B, L, Hq, Hkv, d = 2, 9, 4, 2, 4
    x_q = _rand((B, L, Hq, d), 25, 1)
    kc = _rand((B, L, Hkv, d), 25, 2)
    vc = _rand((B, L, Hkv, d), 25, 3)
    o_pre, l_pre = orc.attention(x_q, kc, vc, 0.5, causal=True)
    o_dec, l_dec = orc.decode(np.ascontiguousarray(x_q[:, -1]), kc, vc, np.full(B, L, np.int32), 0.5)
    assert np.allclose(o_dec, o_pre[:, -1], atol=1e-14)
    assert np.allclose(l_dec, l_pre[:, :, -1], atol=1e-14)


def pin_rows_api_matches_full(orc):
    B, N, Hq, Hkv, d = 2, 7, 4, 2, 8
    q = _rand((B, N, Hq, d), 26, 1)
    k = _rand((B, N, Hkv, d), 26, 2)
    v = _rand((B, N, Hkv, d), 26, 3)
    o, lse = orc.attention(q, k, v, 0.3, causal=True)
    rows = np.array([[1, 3, 6], [0, 0, 0], [1, 2, 4]])
    orr, lr = orc.attention_rows(q, k, v, 0.3, rows, causal=True)
    for t, (b, h, i) in enumerate(rows):
        assert np.array_equal(orr[t], o[b, i, h]) and lr[t] == lse[b, h, i]


def pin_bruteforce_decimal(orc):
    """40-digit brute force on tiny inputs: naive exp (no max shift), explicit sums."""
    getcontext().prec = 40
    for case in range(4):
        B, Nq, Nk, Hq, Hkv, d = 1, 3 + case, 5 + case, 2, 1, 3
        causal = case % 2 == 1
        q = _rand((B, Nq, Hq, d), 27 + case, 1)
        k = _rand((B, Nk, Hkv, d), 27 + case, 2)
        v = _rand((B, Nk, Hkv, d), 27 + case, 3)
        scale = 1.0 / math.sqrt(d)
        o, lse = orc.attention(q, k, v, scale, causal=causal)
        S = Decimal(scale)
        for h in range(Hq):
            for i in range(Nq):
                jmax = min(Nk, i + Nk - Nq + 1) if causal else Nk
                if jmax <= 0:
                    continue
                es = []
                for j in range(jmax):
                    dot = sum(Decimal(float(q[0, i, h, c])) * Decimal(float(k[0, j, 0, c])) for c in range(d))
                    es.append((S * dot).exp())
                tot = sum(es)
                for c in range(d):
                    num = sum(e * Decimal(float(v[0, j, 0, c])) for j, e in enumerate(es))
                    assert abs(float(num / tot) - o[0, i, h, c]) < 1e-14
                assert abs(float(tot.ln()) - lse[0, h, i]) < 1e-14


PINS = [pin_worked_example, pin_softmax_printed, pin_rows_sum_to_one, pin_safe_softmax_no_overflow,
        pin_online_merge_equals_standard, pin_constant_v, pin_q_zero_means, pin_varlen_q_zero,
        pin_decode_lengths_q_zero, pin_two_keys_closed_form, pin_single_key, pin_shift_invariance,
        pin_scale_equals_scaled_q, pin_key_permutation, pin_causal_rows, pin_gqa_equals_repeated_mha,
        pin_varlen_equals_independent, pin_decode_equals_prefill_last_row, pin_rows_api_matches_full,
        pin_bruteforce_decimal]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(orc, pin):
    pin(orc)


PLANTS = ["ORACLE_PLANT_NO_SCALE", "ORACLE_PLANT_SIGN", "ORACLE_PLANT_QV_SWAP",
          "ORACLE_PLANT_LSE_NO_MAX", "ORACLE_PLANT_CAUSAL_OFF_BY_ONE", "ORACLE_PLANT_GQA_MODULO",
          "ORACLE_PLANT_VARLEN_SHORT_KEYS"]


@pytest.mark.parametrize("plant", PLANTS)
def test_pins_catch_planted_mistake(plant):
    broken = oracle_mod.build_planted(plant)
    failed = []
    for pin in PINS:
        try:
            pin(broken)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught {plant}"


def test_oracle_threads_agree(orc):
    """Threading over (b, h) does not change any value."""
    B, N, Hq, Hkv, d = 2, 33, 4, 2, 16
    q = _rand((B, N, Hq, d), 30, 1)
    k = _rand((B, N, Hkv, d), 30, 2)
    v = _rand((B, N, Hkv, d), 30, 3)
    o1, l1 = orc.attention(q, k, v, 0.25, causal=True, nthreads=1)
    o4, l4 = orc.attention(q, k, v, 0.25, causal=True, nthreads=4)
    assert np.array_equal(o1, o4) and np.array_equal(l1, l4)


def test_generator_is_counter_based():
    """Any slice of a stream can be produced on its own (the GPU-side tests rely on it)."""
    a = si.normal(5, si.Q, (1000,), dtype="f32")
    key = si.stream_key(5, si.Q)
    b = si._normals_chunk(key, 400, 200).astype(np.float32)
    assert np.array_equal(a[400:600], b)
    x = si.normal(5, si.K, (4096,), dtype="bf16")
    assert np.all((x.view(np.uint32) & 0xFFFF) == 0)
    assert abs(x.mean()) < 0.06 and abs(x.std() - 1) < 0.05
