"""Helpers shared by the GPU parity tests: device transfer and the comparison rule.

Tolerance (bf16 inputs, fp32 accumulation): every output element within
max(1e-2, one bf16 ulp of the reference value) and the mean absolute error at most 1e-3;
every lse within 1e-3, with -inf exactly where the reference is -inf.  The per-element
bound is the stated 1e-2, widened only where the bf16 output itself cannot resolve 1e-2:
for |O_ref| >= 2 a bf16 ulp exceeds 1e-2, and a correctly rounded result may sit one ulp
from the fp64 reference when the unrounded value lies near a rounding midpoint.
"""
from __future__ import annotations

import numpy as np
import torch

MAX_ABS = 1e-2
MEAN_ABS = 1e-3
LSE_ABS = 1e-3


def dev_bf16(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to("cuda").to(torch.bfloat16)


def dev_f32(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to("cuda")


def host64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    ax = np.abs(x)
    e = np.floor(np.log2(np.maximum(ax, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def check_out(o_gpu: np.ndarray, o_ref: np.ndarray, what: str = "O", bf16_out: bool = True) -> dict:
    assert o_gpu.shape == o_ref.shape, (o_gpu.shape, o_ref.shape)
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite output"
    err = np.abs(o_gpu - o_ref)
    tol = np.maximum(MAX_ABS, bf16_ulp(o_ref)) if bf16_out else MAX_ABS
    bad = err > tol
    stats = {"max_abs": float(err.max()) if err.size else 0.0, "mean_abs": float(err.mean()) if err.size else 0.0}
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(f"{what}: {int(bad.sum())} elements out of tolerance, first {idx.tolist()}: "
                             f"gpu {o_gpu[tuple(idx[0])]} ref {o_ref[tuple(idx[0])]} stats {stats}")
    assert stats["mean_abs"] <= MEAN_ABS, f"{what}: mean abs error {stats['mean_abs']}"
    return stats


def check_lse(l_gpu: np.ndarray, l_ref: np.ndarray, what: str = "lse") -> float:
    assert l_gpu.shape == l_ref.shape
    ninf = np.isneginf(l_ref)
    assert np.array_equal(np.isneginf(l_gpu), ninf), f"{what}: -inf pattern differs"
    fin = ~ninf
    assert np.all(np.isfinite(l_gpu[fin])), f"{what}: non-finite lse"
    err = np.abs(l_gpu[fin] - l_ref[fin])
    m = float(err.max()) if err.size else 0.0
    assert m <= LSE_ABS, f"{what}: max lse error {m}"
    return m


# Gradients (backward).  No tolerance is stated for them; this one follows from the
# arithmetic: P and dS are rounded to bf16 (relative 2^-9) before the tensor-core products
# and every gradient is rounded to bf16 on output, so each element may carry a few bf16
# rounding errors of the terms it sums.  Bound: the relative Frobenius error of each tensor
# at most 1e-2, and every element within 2e-2 of the tensor's largest reference magnitude.
GRAD_REL_FRO = 1e-2
GRAD_MAX_REL = 2e-2
GRAD_ZERO_ABS = 1e-4


def check_grad(g_gpu: np.ndarray, g_ref: np.ndarray, what: str) -> dict:
    assert g_gpu.shape == g_ref.shape, (g_gpu.shape, g_ref.shape)
    assert np.all(np.isfinite(g_gpu)), f"{what}: non-finite gradient"
    err = np.abs(g_gpu - g_ref)
    scale = float(np.abs(g_ref).max()) if g_ref.size else 0.0
    fro = float(np.linalg.norm(g_ref))
    stats = {"rel_fro": float(np.linalg.norm(err)) / fro if fro > 0 else float(np.linalg.norm(err)),
             "max_rel": float(err.max()) / scale if scale > 0 else float(err.max()) if err.size else 0.0}
    if fro == 0.0:
        # an exactly-zero gradient (e.g. dQ with a single key: dP - D cancels) comes out of the
        # fp32 arithmetic as rounding noise of the cancelled terms, which are O(1) for N(0,1)
        # inputs
        assert float(np.abs(g_gpu).max()) <= GRAD_ZERO_ABS, f"{what}: reference is zero, gpu is {stats}"
        return stats
    assert stats["rel_fro"] <= GRAD_REL_FRO, f"{what}: relative Frobenius error {stats}"
    assert stats["max_rel"] <= GRAD_MAX_REL, f"{what}: largest element error {stats}"
    return stats
