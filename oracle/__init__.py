"""fp64 CPU oracle for exact attention (ctypes wrapper over oracle.cpp).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline may use this package; the library and its binding never import it.  It shares
no code with the CUDA path.

What each function computes, and the passage it follows, is documented in oracle.cpp.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import tempfile

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")

_c_double_p = ctypes.POINTER(ctypes.c_double)


def build(out_path: str = _LIB, defines: tuple[str, ...] = (), force: bool = False) -> str:
    """Compile oracle.cpp into a shared library (g++ -O2, fp64, no fast-math)."""
    if (not force and os.path.exists(out_path)
            and os.path.getmtime(out_path) >= os.path.getmtime(_SRC) and not defines):
        return out_path
    cmd = ["g++", "-std=c++17", "-O2", "-fPIC", "-shared", "-pthread", "-fno-fast-math",
           "-ffp-contract=off", _SRC, "-o", out_path] + [f"-D{d}" for d in defines]
    subprocess.run(cmd, check=True)
    return out_path


class Oracle:
    def __init__(self, lib_path: str | None = None):
        path = lib_path or build()
        self.lib = ctypes.CDLL(path)
        L = self.lib
        L.oracle_softmax.argtypes = [_c_double_p, ctypes.c_int64, _c_double_p]
        L.oracle_row_stats.argtypes = [_c_double_p, ctypes.c_int64, _c_double_p, _c_double_p]
        L.oracle_merge_stats.argtypes = [ctypes.c_double] * 4 + [_c_double_p, _c_double_p]
        L.oracle_merge_stats.restype = None
        L.oracle_merge_partials.argtypes = [_c_double_p, _c_double_p, _c_double_p, ctypes.c_int64,
                                            ctypes.c_int, _c_double_p, _c_double_p, _c_double_p]
        common = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 6 + [ctypes.c_double, ctypes.c_int,
                                                                ctypes.c_void_p, ctypes.c_void_p]
        L.oracle_attention.argtypes = common + [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
        L.oracle_attention_rows.argtypes = common + [ctypes.c_void_p, ctypes.c_int64,
                                                     ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
        L.oracle_attention_bwd.argtypes = ([ctypes.c_void_p] * 4 + [ctypes.c_int] * 6 +
                                           [ctypes.c_double, ctypes.c_int, ctypes.c_void_p] +
                                           [ctypes.c_void_p] * 3 + [ctypes.c_int])
        L.oracle_hardware_threads.restype = ctypes.c_int

    # -- softmax statistics and the merge rule -------------------------------------------
    def softmax(self, x) -> np.ndarray:
        x = np.ascontiguousarray(x, dtype=np.float64)
        p = np.empty_like(x)
        assert self.lib.oracle_softmax(x.ctypes.data_as(_c_double_p), x.size,
                                       p.ctypes.data_as(_c_double_p)) == 0
        return p

    def row_stats(self, x) -> tuple[float, float]:
        x = np.ascontiguousarray(x, dtype=np.float64)
        m, l = ctypes.c_double(), ctypes.c_double()
        assert self.lib.oracle_row_stats(x.ctypes.data_as(_c_double_p), x.size,
                                         ctypes.byref(m), ctypes.byref(l)) == 0
        return m.value, l.value

    def merge_stats(self, m1, l1, m2, l2) -> tuple[float, float]:
        m, l = ctypes.c_double(), ctypes.c_double()
        self.lib.oracle_merge_stats(m1, l1, m2, l2, ctypes.byref(m), ctypes.byref(l))
        return m.value, l.value

    def merge_partials(self, m, l, acc):
        m = np.ascontiguousarray(m, dtype=np.float64)
        l = np.ascontiguousarray(l, dtype=np.float64)
        acc = np.ascontiguousarray(acc, dtype=np.float64)
        n, d = acc.shape
        mo, lo = ctypes.c_double(), ctypes.c_double()
        o = np.empty(d, dtype=np.float64)
        assert self.lib.oracle_merge_partials(m.ctypes.data_as(_c_double_p), l.ctypes.data_as(_c_double_p),
                                              acc.ctypes.data_as(_c_double_p), n, d, ctypes.byref(mo),
                                              ctypes.byref(lo), o.ctypes.data_as(_c_double_p)) == 0
        return mo.value, lo.value, o

    # -- attention ------------------------------------------------------------------------
    @staticmethod
    def _f32(a):
        return np.ascontiguousarray(a, dtype=np.float32)

    def attention(self, q, k, v, scale, causal=False, cu_seqlens=None, kv_lens=None, nthreads=0):
        """Full attention.

        Fixed length: q [B,Nq,Hq,d], k/v [B,Nk,Hkv,d] -> o [B,Nq,Hq,d], lse [B,Hq,Nq].
        Varlen: q [total,Hq,d], k/v [total,Hkv,d], cu_seqlens [B+1] -> o [total,Hq,d], lse [Hq,total].
        kv_lens [B] (fixed length only): batch b attends to keys j < kv_lens[b].
        """
        q, k, v = self._f32(q), self._f32(k), self._f32(v)
        if cu_seqlens is not None:
            cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
            total, Hq, d = q.shape
            Hkv = k.shape[1]
            B, Nq, Nk = len(cu) - 1, total, total
            o = np.zeros((total, Hq, d), dtype=np.float64)
            lse = np.zeros((Hq, total), dtype=np.float64)
        else:
            cu = None
            B, Nq, Hq, d = q.shape
            Nk, Hkv = k.shape[1], k.shape[2]
            o = np.zeros((B, Nq, Hq, d), dtype=np.float64)
            lse = np.zeros((B, Hq, Nq), dtype=np.float64)
        kl = None if kv_lens is None else np.ascontiguousarray(kv_lens, dtype=np.int32)
        rc = self.lib.oracle_attention(
            q.ctypes.data, k.ctypes.data, v.ctypes.data, B, Hq, Hkv, Nq, Nk, d, float(scale), int(bool(causal)),
            None if cu is None else cu.ctypes.data, None if kl is None else kl.ctypes.data,
            o.ctypes.data, lse.ctypes.data, int(nthreads))
        if rc != 0:
            raise ValueError("oracle_attention rejected its arguments")
        return o, lse

    def attention_rows(self, q, k, v, scale, rows, causal=False, cu_seqlens=None, kv_lens=None, nthreads=0):
        """Selected rows (b, h, i) of the same problem as attention(): o [n,d], lse [n]."""
        q, k, v = self._f32(q), self._f32(k), self._f32(v)
        rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 3)
        if cu_seqlens is not None:
            cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
            total, Hq, d = q.shape
            Hkv = k.shape[1]
            B, Nq, Nk = len(cu) - 1, total, total
        else:
            cu = None
            B, Nq, Hq, d = q.shape
            Nk, Hkv = k.shape[1], k.shape[2]
        kl = None if kv_lens is None else np.ascontiguousarray(kv_lens, dtype=np.int32)
        n = rows.shape[0]
        o = np.zeros((n, d), dtype=np.float64)
        lse = np.zeros(n, dtype=np.float64)
        rc = self.lib.oracle_attention_rows(
            q.ctypes.data, k.ctypes.data, v.ctypes.data, B, Hq, Hkv, Nq, Nk, d, float(scale), int(bool(causal)),
            None if cu is None else cu.ctypes.data, None if kl is None else kl.ctypes.data,
            rows.ctypes.data, n, o.ctypes.data, lse.ctypes.data, int(nthreads))
        if rc != 0:
            raise ValueError("oracle_attention_rows rejected its arguments")
        return o, lse

    def decode(self, q, kcache, vcache, seqlens, scale, nthreads=0):
        """Single-token decode over a cache: q [B,Hq,d], caches [B,Lmax,Hkv,d], seqlens [B]
        -> o [B,Hq,d], lse [B,Hq].  The plain definition with Nq = 1, non-causal, keys j < seqlens[b]."""
        B, Hq, d = q.shape
        o, lse = self.attention(q.reshape(B, 1, Hq, d), kcache, vcache, scale, causal=False,
                                kv_lens=seqlens, nthreads=nthreads)
        return o.reshape(B, Hq, d), lse.reshape(B, Hq)

    @staticmethod
    def gather_pages(pages, block_table, seqlens, page_size):
        """Contiguous per-sequence cache [B, Lmax, H, d] from a page pool [P, page_size, H, d]
        ("LLM basics: from Attention to FlashAttention", chapter 2 section 8, PagedAttention:
        a sequence's logical page t is the physical page block_table[b, t]; token j of the
        sequence is row j % page_size of its logical page j // page_size).  Rows at or past
        seqlens[b] are left zero (decode never reads them)."""
        pages = np.asarray(pages)
        table = np.asarray(block_table)
        B, maxp = table.shape
        H, d = pages.shape[2], pages.shape[3]
        out = np.zeros((B, maxp * page_size, H, d), dtype=pages.dtype)
        for b in range(B):
            for j in range(int(seqlens[b])):
                out[b, j] = pages[table[b, j // page_size], j % page_size]
        return out

    def decode_paged(self, q, k_pages, v_pages, block_table, seqlens, page_size, scale, nthreads=0):
        """Decode over a paged cache: each sequence's cache is read through its block table
        (gather_pages), then the plain decode definition applies."""
        kc = self.gather_pages(k_pages, block_table, seqlens, page_size)
        vc = self.gather_pages(v_pages, block_table, seqlens, page_size)
        return self.decode(q, kc, vc, np.asarray(seqlens), scale, nthreads=nthreads)

    def attention_bwd(self, q, k, v, dout, scale, causal=False, cu_seqlens=None, nthreads=0):
        """Gradients (dq, dk, dv) of o = attention(q, k, v) for an upstream gradient dout of o
        (layouts as in attention(); see oracle_attention_bwd in oracle.cpp)."""
        q, k, v, dout = self._f32(q), self._f32(k), self._f32(v), self._f32(dout)
        if cu_seqlens is not None:
            cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
            total, Hq, d = q.shape
            Hkv = k.shape[1]
            B, Nq, Nk = len(cu) - 1, total, total
        else:
            cu = None
            B, Nq, Hq, d = q.shape
            Nk, Hkv = k.shape[1], k.shape[2]
        dq = np.zeros(q.shape, dtype=np.float64)
        dk = np.zeros(k.shape, dtype=np.float64)
        dv = np.zeros(v.shape, dtype=np.float64)
        rc = self.lib.oracle_attention_bwd(
            q.ctypes.data, k.ctypes.data, v.ctypes.data, dout.ctypes.data, B, Hq, Hkv, Nq, Nk, d, float(scale),
            int(bool(causal)), None if cu is None else cu.ctypes.data, dq.ctypes.data, dk.ctypes.data,
            dv.ctypes.data, int(nthreads))
        if rc != 0:
            raise ValueError("oracle_attention_bwd rejected its arguments")
        return dq, dk, dv

    def hardware_threads(self) -> int:
        return int(self.lib.oracle_hardware_threads())


_default: Oracle | None = None


def get() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def build_planted(define: str) -> Oracle:
    """A copy of the oracle built with one planted mistake (for the pin-coverage test)."""
    d = tempfile.mkdtemp(prefix="oracle_plant_")
    path = build(os.path.join(d, f"liboracle_{define}.so"), defines=(define,), force=True)
    return Oracle(path)
