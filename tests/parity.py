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
