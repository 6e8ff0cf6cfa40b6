"""ctypes binding of libfa.so: the functions of include/fa.h under the same names.

Argument marshalling only: pointers come from torch tensors (``data_ptr()``) or plain
integers, the stream defaults to torch's current stream, and a non-OK status raises
``FaError``.  Every step of the computation runs in the library's CUDA kernels; there is no
fallback.  If libfa.so is missing this module raises on first use.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libfa.so")

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_WORKSPACE, FA_ERR_CUDA, FA_ERR_TIMEOUT = range(6)
FA_BF16, FA_F32, FA_TF32 = 0, 1, 2

EXPORTED = ("fa_fwd", "fa_fwd_workspace_size", "fa_decode", "fa_decode_workspace_size", "fa_decode_noalloc",
            "fa_decode_paged", "fa_decode_paged_workspace_size", "fa_bwd", "fa_bwd_workspace_size", "fa_bwd_varlen",
            "fa_bwd_varlen_workspace_size", "fa_fwd_qkvpacked",
            "fa_fwd_fp8", "fa_fwd_fp8_workspace_size", "fa_selftest_wait_timeout",
            "fa_last_device_error", "fa_status_string", "fa_device_sm_count")
FA_DECODE_NOALLOC_SCRATCH_BYTES = 16 << 20


class FaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


_lib: Optional[ctypes.CDLL] = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libfa.so (once).  Raises if the CUDA library has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libfa.so not found at {path}; build it with `python -m exact_io_aware_97_b200.build`")
    L = ctypes.CDLL(path)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    L.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp, i, vp, sz, vp]
    L.fa_fwd.restype = i
    L.fa_fwd_workspace_size.argtypes = [i, i, i, i, i, i, i, i]
    L.fa_fwd_workspace_size.restype = sz
    L.fa_decode.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp, sz, vp]
    L.fa_decode.restype = i
    L.fa_decode_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp]
    L.fa_decode_noalloc.restype = i
    L.fa_decode_workspace_size.argtypes = [i, i, i, i, i]
    L.fa_decode_workspace_size.restype = sz
    L.fa_decode_paged.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, i, vp, sz, vp]
    L.fa_decode_paged.restype = i
    L.fa_decode_paged_workspace_size.argtypes = [i, i, i, i, i, i, i]
    L.fa_decode_paged_workspace_size.restype = sz
    L.fa_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, f, f, f, i, vp, sz, vp]
    L.fa_fwd_fp8.restype = i
    L.fa_fwd_fp8_workspace_size.argtypes = [i, i, i, i]
    L.fa_fwd_fp8_workspace_size.restype = sz
    L.fa_fwd_qkvpacked.argtypes = [vp, vp, vp, i, i, i, i, f, i, vp, vp]
    L.fa_fwd_qkvpacked.restype = i
    L.fa_bwd.argtypes = [vp] * 9 + [i] * 6 + [f, i, vp, sz, vp]
    L.fa_bwd.restype = i
    L.fa_bwd_workspace_size.argtypes = [i, i, i, i]
    L.fa_bwd_workspace_size.restype = sz
    L.fa_bwd_varlen.argtypes = [vp] * 9 + [i] * 5 + [f, i, vp, vp, sz, vp]
    L.fa_bwd_varlen.restype = i
    L.fa_bwd_varlen_workspace_size.argtypes = [i, i, i, i]
    L.fa_bwd_varlen_workspace_size.restype = sz
    L.fa_selftest_wait_timeout.argtypes = [vp]
    L.fa_selftest_wait_timeout.restype = i
    L.fa_last_device_error.argtypes = [vp]
    L.fa_last_device_error.restype = i
    L.fa_status_string.argtypes = [i]
    L.fa_status_string.restype = ctypes.c_char_p
    L.fa_device_sm_count.argtypes = []
    L.fa_device_sm_count.restype = i
    _lib = L
    return L


def _ptr(x) -> Optional[int]:
    """Device address of a tensor argument (an int is taken as a raw address).  The library
    reads every tensor as a dense row-major block of device memory, so a host tensor or a
    strided view is refused here rather than handed to a kernel."""
    if x is None:
        return None
    if isinstance(x, int):
        return x or None
    if not x.is_cuda:
        raise ValueError(f"expected a CUDA tensor, got one on {x.device}")
    if not x.is_contiguous():
        raise ValueError(f"expected a contiguous tensor, got strides {tuple(x.stride())} for shape {tuple(x.shape)}")
    return x.data_ptr() or None


def _ptr_i32(x, what: str) -> Optional[int]:
    """Device address of an int32 index tensor (offsets, lengths, block table): the kernels
    read these as int32, so another integer width would be misread as other offsets."""
    if x is not None and not isinstance(x, int) and str(x.dtype) != "torch.int32":
        raise ValueError(f"{what}: expected an int32 tensor, got {x.dtype}")
    return _ptr(x)


def _expect(t, shape, dtype: str, what: str) -> None:
    """A caller-provided output must have exactly the shape and dtype the kernels write."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape) or str(t.dtype) != dtype:
        raise ValueError(f"{what}: expected {dtype} {tuple(shape)}, got {t.dtype} {tuple(t.shape)}")


def _same(what: str, *ts) -> None:
    """Tensors that the kernels read with one shape and one element type."""
    a = ts[0]
    for t in ts[1:]:
        if tuple(t.shape) != tuple(a.shape) or t.dtype != a.dtype:
            raise ValueError(f"{what}: shapes/dtypes differ: {tuple(a.shape)} {a.dtype} vs {tuple(t.shape)} {t.dtype}")


def _require(what: str, ok: bool, expected: str) -> None:
    """A relation between tensors that the kernels rely on: they size every read from q's
    batch and head dimension, so a smaller k or cache would be read past its end."""
    if not ok:
        raise ValueError(f"{what}: expected {expected}")


def _lengths(seqlens, B: int, what: str) -> None:
    """Per-sequence lengths are read as B int32 entries."""
    if seqlens is not None and not isinstance(seqlens, int):
        _require(what, seqlens.dim() == 1 and seqlens.numel() == B, f"{B} entries, got shape {tuple(seqlens.shape)}")


def _bf16(what: str, *ts) -> None:
    """Paths that read bf16 only (the backward, the decodes)."""
    for t in ts:
        if str(t.dtype) != "torch.bfloat16":
            raise ValueError(f"{what}: expected bf16 tensors, got {t.dtype}")


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream or None
    if isinstance(stream, int):
        return stream or None
    return stream.cuda_stream or None


def _check(status: int, where: str) -> None:
    if status != FA_OK:
        raise FaError(status, where)


def status_string(status: int) -> str:
    return load().fa_status_string(int(status)).decode()


def fa_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, cu_seqlens=None, in_dtype=FA_BF16,
           workspace=None, workspace_bytes=0, stream=None) -> None:
    st = load().fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), int(B), int(Hq), int(Hkv), int(Nq), int(Nk),
                       int(d), float(scale), int(bool(causal)), _ptr_i32(cu_seqlens, "cu_seqlens"), int(in_dtype), _ptr(workspace),
                       int(workspace_bytes), _stream(stream))
    _check(st, "fa_fwd")


def fa_fwd_workspace_size(B, Hq, Hkv, Nq, Nk, d, in_dtype=FA_BF16, varlen=False) -> int:
    return int(load().fa_fwd_workspace_size(int(B), int(Hq), int(Hkv), int(Nq), int(Nk), int(d), int(in_dtype),
                                            int(bool(varlen))))


def fa_decode(q, kcache, vcache, seqlens, o, lse, B, Hq, Hkv, Lmax, d, scale, split_len, workspace,
              workspace_bytes, stream=None) -> None:
    st = load().fa_decode(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr_i32(seqlens, "seqlens"), _ptr(o), _ptr(lse), int(B), int(Hq),
                          int(Hkv), int(Lmax), int(d), float(scale), int(split_len), _ptr(workspace),
                          int(workspace_bytes), _stream(stream))
    _check(st, "fa_decode")


def fa_decode_noalloc(q, kcache, vcache, seqlens, o, lse, B, Hq, Hkv, Lmax, d, scale, split_len,
                      stream=None) -> None:
    """fa_decode with its scratch in the library's static device array (no allocation).
    For callers that cannot allocate device memory; calls that overlap on the GPU race, and
    the first call on a device should come before any stream capture (see include/fa.h)."""
    st = load().fa_decode_noalloc(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr_i32(seqlens, "seqlens"), _ptr(o), _ptr(lse), int(B),
                                  int(Hq), int(Hkv), int(Lmax), int(d), float(scale), int(split_len),
                                  _stream(stream))
    _check(st, "fa_decode_noalloc")


def fa_decode_workspace_size(B, Hq, Lmax, d, split_len) -> int:
    return int(load().fa_decode_workspace_size(int(B), int(Hq), int(Lmax), int(d), int(split_len)))


def fa_decode_paged(q, k_pages, v_pages, block_table, seqlens, o, lse, B, Hq, Hkv, num_pages, page_size,
                    max_pages_per_seq, d, scale, split_len, workspace, workspace_bytes, stream=None) -> None:
    st = load().fa_decode_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr_i32(block_table, "block_table"), _ptr_i32(seqlens, "seqlens"), _ptr(o),
                                _ptr(lse), int(B), int(Hq), int(Hkv), int(num_pages), int(page_size),
                                int(max_pages_per_seq), int(d), float(scale), int(split_len), _ptr(workspace),
                                int(workspace_bytes), _stream(stream))
    _check(st, "fa_decode_paged")


def fa_decode_paged_workspace_size(B, Hq, Hkv, max_pages_per_seq, page_size, d, split_len) -> int:
    return int(load().fa_decode_paged_workspace_size(int(B), int(Hq), int(Hkv), int(max_pages_per_seq),
                                                     int(page_size), int(d), int(split_len)))


def fa_fwd_fp8(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, descale_q, descale_k, descale_v, causal, workspace,
               workspace_bytes, stream=None) -> None:
    st = load().fa_fwd_fp8(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), int(B), int(Hq), int(Hkv), int(Nq),
                           int(Nk), int(d), float(scale), float(descale_q), float(descale_k), float(descale_v),
                           int(bool(causal)), _ptr(workspace), int(workspace_bytes), _stream(stream))
    _check(st, "fa_fwd_fp8")


def fa_fwd_fp8_workspace_size(B, Hkv, Nk, d) -> int:
    return int(load().fa_fwd_fp8_workspace_size(int(B), int(Hkv), int(Nk), int(d)))


def fa_fwd_qkvpacked(qkv, o, lse, B, H, N, d, scale, causal, cu_seqlens=None, stream=None) -> None:
    st = load().fa_fwd_qkvpacked(_ptr(qkv), _ptr(o), _ptr(lse), int(B), int(H), int(N), int(d), float(scale),
                                 int(bool(causal)), _ptr_i32(cu_seqlens, "cu_seqlens"), _stream(stream))
    _check(st, "fa_fwd_qkvpacked")


def fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, scale, causal, workspace, workspace_bytes,
           stream=None) -> None:
    st = load().fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
                       int(B), int(Hq), int(Hkv), int(Nq), int(Nk), int(d), float(scale), int(bool(causal)),
                       _ptr(workspace), int(workspace_bytes), _stream(stream))
    _check(st, "fa_bwd")


def fa_bwd_workspace_size(B, Hq, Nq, d) -> int:
    return int(load().fa_bwd_workspace_size(int(B), int(Hq), int(Nq), int(d)))


def fa_bwd_varlen(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, total, d, scale, causal, cu_seqlens, workspace,
                  workspace_bytes, stream=None) -> None:
    st = load().fa_bwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                              _ptr(dv), int(B), int(Hq), int(Hkv), int(total), int(d), float(scale),
                              int(bool(causal)), _ptr_i32(cu_seqlens, "cu_seqlens"), _ptr(workspace), int(workspace_bytes),
                              _stream(stream))
    _check(st, "fa_bwd_varlen")


def fa_bwd_varlen_workspace_size(B, Hq, total, d) -> int:
    return int(load().fa_bwd_varlen_workspace_size(int(B), int(Hq), int(total), int(d)))


def fa_selftest_wait_timeout(stream=None) -> None:
    """Launch the self-test whose bounded wait must run out (see include/fa.h)."""
    _check(load().fa_selftest_wait_timeout(_stream(stream)), "fa_selftest_wait_timeout")


def fa_last_device_error(stream=None) -> int:
    return int(load().fa_last_device_error(_stream(stream)))


def fa_device_sm_count() -> int:
    return int(load().fa_device_sm_count())


# ------------------------------------------------------------------ tensor-level helpers
def forward(q, k, v, causal=False, scale=None, cu_seqlens=None, out=None, lse=None, workspace=None, stream=None,
            tf32=False):
    """O, lse for q [B,Nq,Hq,d] / k,v [B,Nk,Hkv,d] (or packed [total,H,d] with cu_seqlens).

    bf16 inputs give bf16 O; fp32 inputs (fixed length) are rounded to bf16 on the device and
    give fp32 O.  Outputs and workspace are allocated with torch unless passed in."""
    import torch
    varlen = cu_seqlens is not None
    _same("k, v", k, v)
    if q.dtype != k.dtype or q.shape[-1] != k.shape[-1] or q.dim() != k.dim():
        raise ValueError(f"q {q.dtype} {tuple(q.shape)} does not match k {k.dtype} {tuple(k.shape)}")
    if varlen:
        _require("q", q.dim() == 3, f"packed [total, Hq, d] with cu_seqlens, got shape {tuple(q.shape)}")
        total, Hq, d = q.shape
        Hkv = k.shape[1]
        _require("k", k.shape[0] == total, f"{total} packed rows like q, got {k.shape[0]}")
        _require("cu_seqlens", cu_seqlens.dim() == 1 and cu_seqlens.numel() >= 2,
                 f"[B + 1] offsets, got shape {tuple(cu_seqlens.shape)}")
        B, Nq, Nk = cu_seqlens.numel() - 1, total, total
        lse_shape = (Hq, total)
    else:
        _require("q", q.dim() == 4, f"[B, Nq, Hq, d], got shape {tuple(q.shape)}")
        B, Nq, Hq, d = q.shape
        Nk, Hkv = k.shape[1], k.shape[2]
        _require("k", k.shape[0] == B, f"batch {B} like q, got {k.shape[0]}")
        lse_shape = (B, Hq, Nq)
    _require("heads", Hkv > 0 and Hq % Hkv == 0, f"Hq ({Hq}) a multiple of Hkv ({Hkv})")
    in_dtype = (FA_TF32 if tf32 else FA_F32) if q.dtype == torch.float32 else FA_BF16
    if scale is None:
        scale = d ** -0.5
    _expect(out, q.shape, "torch.bfloat16" if in_dtype == FA_BF16 else "torch.float32", "out")
    _expect(lse, lse_shape, "torch.float32", "lse")
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16 if in_dtype == FA_BF16 else torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty(lse_shape, dtype=torch.float32, device=q.device)
    ws_bytes = fa_fwd_workspace_size(B, Hq, Hkv, Nq, Nk, d, in_dtype, varlen)
    if ws_bytes and workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    fa_fwd(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, cu_seqlens, in_dtype, workspace,
           ws_bytes if workspace is not None else 0, stream)
    return out, lse


def decode(q, kcache, vcache, seqlens=None, scale=None, split_len=1024, out=None, lse=None, workspace=None,
           stream=None):
    """O [B,Hq,d], lse [B,Hq] for one query token per sequence over caches [B,Lmax,Hkv,d]."""
    import torch
    _require("q", q.dim() == 3, f"[B, Hq, d], got shape {tuple(q.shape)}")
    B, Hq, d = q.shape
    _same("kcache, vcache", kcache, vcache)
    _bf16("decode", q, kcache)
    _require("kcache", kcache.dim() == 4 and kcache.shape[0] == B and kcache.shape[3] == d,
             f"[B={B}, Lmax, Hkv, d={d}], got shape {tuple(kcache.shape)}")
    Lmax, Hkv = kcache.shape[1], kcache.shape[2]
    _require("heads", Hkv > 0 and Hq % Hkv == 0, f"Hq ({Hq}) a multiple of Hkv ({Hkv})")
    _lengths(seqlens, B, "seqlens")
    if scale is None:
        scale = d ** -0.5
    _expect(out, (B, Hq, d), "torch.bfloat16", "out")
    _expect(lse, (B, Hq), "torch.float32", "lse")
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    ws_bytes = fa_decode_workspace_size(B, Hq, Lmax, d, split_len)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    fa_decode(q, kcache, vcache, seqlens, out, lse, B, Hq, Hkv, Lmax, d, scale, split_len, workspace, ws_bytes,
              stream)
    return out, lse


def decode_paged(q, k_pages, v_pages, block_table, seqlens, scale=None, split_len=1024, out=None, lse=None,
                 workspace=None, stream=None):
    """O [B,Hq,d], lse [B,Hq] for one query token per sequence over a page pool
    [num_pages, page_size, Hkv, d] addressed by block_table [B, max_pages] (int32) and
    seqlens [B] (int32)."""
    import torch
    _require("q", q.dim() == 3, f"[B, Hq, d], got shape {tuple(q.shape)}")
    B, Hq, d = q.shape
    _same("k_pages, v_pages", k_pages, v_pages)
    _bf16("decode_paged", q, k_pages)
    _require("k_pages", k_pages.dim() == 4 and k_pages.shape[3] == d,
             f"[num_pages, page_size, Hkv, d={d}], got shape {tuple(k_pages.shape)}")
    num_pages, page_size, Hkv = k_pages.shape[0], k_pages.shape[1], k_pages.shape[2]
    _require("heads", Hkv > 0 and Hq % Hkv == 0, f"Hq ({Hq}) a multiple of Hkv ({Hkv})")
    _lengths(seqlens, B, "seqlens")
    if block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError(f"block_table: expected [B={B}, max_pages], got {tuple(block_table.shape)}")
    maxp = block_table.shape[1]
    if scale is None:
        scale = d ** -0.5
    _expect(out, (B, Hq, d), "torch.bfloat16", "out")
    _expect(lse, (B, Hq), "torch.float32", "lse")
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    ws_bytes = fa_decode_paged_workspace_size(B, Hq, Hkv, maxp, page_size, d, split_len)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    fa_decode_paged(q, k_pages, v_pages, block_table, seqlens, out, lse, B, Hq, Hkv, num_pages, page_size, maxp, d,
                    scale, split_len, workspace, ws_bytes, stream)
    return out, lse


def backward(q, k, v, o, lse, dout, causal=False, scale=None, workspace=None, stream=None):
    """dq, dk, dv for q [B,Nq,Hq,d], k/v [B,Nk,Hkv,d], the forward's o and lse, and dout."""
    import torch
    _require("q", q.dim() == 4, f"[B, Nq, Hq, d], got shape {tuple(q.shape)}")
    B, Nq, Hq, d = q.shape
    _same("q, o, dout", q, o, dout)
    _same("k, v", k, v)
    _bf16("backward", q, k)
    _require("k", k.dim() == 4 and k.shape[0] == B and k.shape[3] == d,
             f"[B={B}, Nk, Hkv, d={d}], got shape {tuple(k.shape)}")
    Nk, Hkv = k.shape[1], k.shape[2]
    _require("heads", Hkv > 0 and Hq % Hkv == 0, f"Hq ({Hq}) a multiple of Hkv ({Hkv})")
    _expect(lse, (B, Hq, Nq), "torch.float32", "lse")
    if scale is None:
        scale = d ** -0.5
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_bytes = fa_bwd_workspace_size(B, Hq, Nq, d)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, scale, causal, workspace, ws_bytes, stream)
    return dq, dk, dv


def backward_varlen(q, k, v, o, lse, dout, cu_seqlens, causal=False, scale=None, workspace=None, stream=None):
    """dq, dk, dv for packed sequences: q, o, dout [total,Hq,d], k/v [total,Hkv,d], lse [Hq,total]
    from the varlen forward, cu_seqlens int32 [B+1] on the device."""
    import torch
    _require("q", q.dim() == 3, f"packed [total, Hq, d], got shape {tuple(q.shape)}")
    total, Hq, d = q.shape
    _same("q, o, dout", q, o, dout)
    _same("k, v", k, v)
    _bf16("backward_varlen", q, k)
    _require("k", k.dim() == 3 and k.shape[0] == total and k.shape[2] == d,
             f"[total={total}, Hkv, d={d}], got shape {tuple(k.shape)}")
    _require("cu_seqlens", cu_seqlens.dim() == 1 and cu_seqlens.numel() >= 2,
             f"[B + 1] offsets, got shape {tuple(cu_seqlens.shape)}")
    Hkv = k.shape[1]
    _require("heads", Hkv > 0 and Hq % Hkv == 0, f"Hq ({Hq}) a multiple of Hkv ({Hkv})")
    B = cu_seqlens.numel() - 1
    _expect(lse, (Hq, total), "torch.float32", "lse")
    if scale is None:
        scale = d ** -0.5
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_bytes = fa_bwd_varlen_workspace_size(B, Hq, total, d)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    fa_bwd_varlen(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, total, d, scale, causal, cu_seqlens, workspace,
                  ws_bytes, stream)
    return dq, dk, dv


def forward_qkvpacked(qkv, causal=False, scale=None, cu_seqlens=None):
    """O, lse for qkv [B,N,3,H,d] (or [total,3,H,d] with cu_seqlens), bf16."""
    import torch
    if cu_seqlens is not None:
        _require("qkv", qkv.dim() == 4 and qkv.shape[1] == 3, f"[total, 3, H, d], got shape {tuple(qkv.shape)}")
        total, _, H, d = qkv.shape
        B, N = cu_seqlens.numel() - 1, total
        out = torch.empty((total, H, d), dtype=torch.bfloat16, device=qkv.device)
        lse = torch.empty((H, total), dtype=torch.float32, device=qkv.device)
    else:
        _require("qkv", qkv.dim() == 5 and qkv.shape[2] == 3, f"[B, N, 3, H, d], got shape {tuple(qkv.shape)}")
        B, N, _, H, d = qkv.shape
        out = torch.empty((B, N, H, d), dtype=torch.bfloat16, device=qkv.device)
        lse = torch.empty((B, H, N), dtype=torch.float32, device=qkv.device)
    if scale is None:
        scale = d ** -0.5
    fa_fwd_qkvpacked(qkv, out, lse, B, H, N, d, scale, causal, cu_seqlens)
    return out, lse


def forward_fp8(q8, k8, v8, descale_q, descale_k, descale_v, causal=False, scale=None, workspace=None):
    """O (bf16), lse for e4m3 q8 [B,Nq,Hq,128], k8/v8 [B,Nk,Hkv,128] (uint8 or float8 tensors)."""
    import torch
    _require("q8", q8.dim() == 4, f"[B, Nq, Hq, d], got shape {tuple(q8.shape)}")
    B, Nq, Hq, d = q8.shape
    _same("k8, v8", k8, v8)
    _require("k8", k8.dim() == 4 and k8.shape[0] == B and k8.shape[3] == d,
             f"[B={B}, Nk, Hkv, d={d}], got shape {tuple(k8.shape)}")
    Nk, Hkv = k8.shape[1], k8.shape[2]
    _require("heads", Hkv > 0 and Hq % Hkv == 0, f"Hq ({Hq}) a multiple of Hkv ({Hkv})")
    if scale is None:
        scale = d ** -0.5
    o = torch.empty((B, Nq, Hq, d), dtype=torch.bfloat16, device=q8.device)
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q8.device)
    ws_bytes = fa_fwd_fp8_workspace_size(B, Hkv, Nk, d)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q8.device)
    fa_fwd_fp8(q8, k8, v8, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, descale_q, descale_k, descale_v, causal, workspace,
               ws_bytes)
    return o, lse
