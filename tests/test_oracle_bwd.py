"""Pins of the oracle's attention backward (the gradients of o with respect to q, k, v for an
upstream gradient dO; "FlashAttention notes", section 5.2 backward) to facts that do not
come from the oracle's backward itself:

* central finite differences of the oracle's *forward* (a separate code path) on
  f(q, k, v) = sum(o * dO);
* torch.autograd (fp64, CPU) on the plain formula softmax(scale q k^T + mask) v, with GQA
  written as repeating each key/value head over its group;
* invariants: sum_j dV_j = sum_i dO_i over a group (rows of P sum to 1); dQ does not change
  when one vector is added to every key (rows of dS sum to 0); dQ = 0 when all keys are equal;
* packed variable-length sequences give each sequence's own gradients (no attention, hence
  no gradient, crosses a sequence boundary).

Planted mistakes (a dropped D term, dK built from P instead of dS, dQ without the scale, the
GQA and causal mistakes of the forward pins, a packed sequence that loses its last key) must
each fail at least one pin.
"""
import numpy as np
import pytest
import torch

import oracle as oracle_mod
import synth_inputs as si


def _rand(shape, seed, tid):
    return si.normal(seed, tid, shape, dtype="f32").astype(np.float32)


def _problem(seed, B=1, N=6, Hq=4, Hkv=2, d=5, Nk=None):
    Nk = N if Nk is None else Nk
    q = _rand((B, N, Hq, d), seed, si.Q)
    k = _rand((B, Nk, Hkv, d), seed, si.K)
    v = _rand((B, Nk, Hkv, d), seed, si.V)
    do = _rand((B, N, Hq, d), seed, 9)
    return q, k, v, do


def pin_finite_differences(orc):
    ok = True
    for causal, Nk in ((False, 6), (True, 6), (True, 8)):
        q, k, v, do = _problem(8101 + Nk + causal, Nk=Nk)
        scale = 0.6
        dq, dk, dv = orc.attention_bwd(q, k, v, do, scale, causal=causal)

        def f(qq, kk, vv):
            o, _ = orc.attention(qq, kk, vv, scale, causal=causal)
            return float(np.sum(o * do.astype(np.float64)))

        # float32 inputs: perturb by a power of two so x +- h is exact
        h = 2.0 ** -12
        for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
            flat = x.reshape(-1)
            for idx in range(0, flat.size, 7):
                xp, xm = x.copy(), x.copy()
                xp.reshape(-1)[idx] += h
                xm.reshape(-1)[idx] -= h
                args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
                args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
                fd = (f(*args_p) - f(*args_m)) / (2 * h)
                ok &= abs(fd - g.reshape(-1)[idx]) <= 1e-6 * max(1.0, abs(fd))
    return ok


def pin_autograd(orc):
    ok = True
    for causal, seed in ((False, 8201), (True, 8202)):
        q, k, v, do = _problem(seed, B=2, N=7, Hq=6, Hkv=2, d=4)
        scale = 0.45
        dq, dk, dv = orc.attention_bwd(q, k, v, do, scale, causal=causal)
        tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
        G = q.shape[2] // k.shape[2]
        kr = tk.repeat_interleave(G, dim=2)
        vr = tv.repeat_interleave(G, dim=2)
        s = torch.einsum("bihc,bjhc->bhij", tq, kr) * scale
        if causal:
            n = q.shape[1]
            s = s.masked_fill(torch.ones(n, n, dtype=torch.bool).triu(1), float("-inf"))
        o = torch.einsum("bhij,bjhc->bihc", torch.softmax(s, dim=-1), vr)
        (o * torch.tensor(do, dtype=torch.float64)).sum().backward()
        for ours, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
            ok &= np.allclose(ours, ref.numpy(), rtol=1e-10, atol=1e-12)
    return ok


def pin_invariants(orc):
    q, k, v, do = _problem(8301, B=1, N=9, Hq=4, Hkv=2, d=6)
    scale = 0.5
    dq, dk, dv = orc.attention_bwd(q, k, v, do, scale, causal=True)
    G = 2
    # sum over keys of dV equals the sum over queries of dO, per group
    ok = np.allclose(dv.sum(axis=1), do.astype(np.float64).reshape(1, 9, 2, G, 6).sum(axis=(1, 3)), atol=1e-12)
    # adding one vector to every key leaves dQ unchanged
    c = _rand((1, 1, 2, 6), 8302, si.K)
    dq2, _, _ = orc.attention_bwd(q, k + c, v, do, scale, causal=True)
    ok &= np.allclose(dq, dq2, atol=1e-9)
    # equal keys: every row of P is uniform, dS rows sum to 0 and dQ vanishes
    ke = np.broadcast_to(k[:, :1], k.shape).copy()
    dq3, _, _ = orc.attention_bwd(q, ke, v, do, scale, causal=False)
    ok &= np.abs(dq3).max() < 1e-12
    return ok


def pin_varlen_equals_independent(orc):
    """Packed sequences (an empty one included) give the gradients of each sequence run on
    its own: attention never crosses a sequence boundary, so neither does a gradient."""
    lens = [4, 9, 1, 0, 6]
    cu = si.cu_seqlens(lens)
    T, Hq, Hkv, d = int(cu[-1]), 4, 2, 4
    q = _rand((T, Hq, d), 8401, si.Q)
    k = _rand((T, Hkv, d), 8401, si.K)
    v = _rand((T, Hkv, d), 8401, si.V)
    do = _rand((T, Hq, d), 8401, 9)
    ok = True
    for causal in (False, True):
        dq, dk, dv = orc.attention_bwd(q, k, v, do, 0.5, causal=causal, cu_seqlens=cu)
        for b in range(len(lens)):
            s = slice(int(cu[b]), int(cu[b + 1]))
            if lens[b] == 0:
                continue
            gq, gk, gv = orc.attention_bwd(q[s][None], k[s][None], v[s][None], do[s][None], 0.5, causal=causal)
            ok &= np.allclose(dq[s], gq[0], atol=1e-14) and np.allclose(dk[s], gk[0], atol=1e-14)
            ok &= np.allclose(dv[s], gv[0], atol=1e-14)
    return bool(ok)


PINS = [pin_finite_differences, pin_autograd, pin_invariants, pin_varlen_equals_independent]


@pytest.fixture(scope="module")
def orc():
    return oracle_mod.get()


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_bwd_pin(orc, pin):
    assert pin(orc)


@pytest.mark.parametrize("plant", ["ORACLE_PLANT_BWD_NO_D", "ORACLE_PLANT_BWD_DK_FROM_P",
                                   "ORACLE_PLANT_BWD_DQ_NO_SCALE", "ORACLE_PLANT_GQA_MODULO",
                                   "ORACLE_PLANT_CAUSAL_OFF_BY_ONE", "ORACLE_PLANT_VARLEN_SHORT_KEYS"])
def test_bwd_pins_catch_planted_mistake(plant):
    broken = oracle_mod.build_planted(plant)
    assert not all(pin(broken) for pin in PINS)
