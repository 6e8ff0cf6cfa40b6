"""Seeded synthetic inputs for the attention workloads.

This module is shared by the CUDA-path tests, the oracle tests, the benchmark and the
smoke check.  It holds no attention arithmetic: it only turns (seed, stream, index)
into numbers.

Generator (counter-based, so any element can be produced on its own):

* splitmix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014): word i of stream `key` is
  ``mix(key + (i + 1) * 0x9E3779B97F4A7C15)`` with the published finaliser
  ``z ^= z >> 30; z *= 0xBF58476D1CE4E5B9; z ^= z >> 27; z *= 0x94D049BB133111EB;
  z ^= z >> 31``.
* uniforms in (0, 1): ``((w >> 11) + 0.5) * 2**-53``.
* N(0, 1) by the Box-Muller transform (Box and Muller, 1958): words 2p and 2p+1
  give u1, u2 and normals ``r cos(2 pi u2)``, ``r sin(2 pi u2)`` with
  ``r = sqrt(-2 ln u1)``, for elements 2p and 2p+1.
* storage: the float64 normal is rounded to float32 (round to nearest even) and,
  for bf16 storage, that float32 is rounded to bf16 (round to nearest even on the
  bit pattern).  The returned array is float32 holding exactly the stored values.

Each tensor of a workload has its own stream key: ``mix(seed * 2**20 + tensor_id)``.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# tensor ids of the streams
Q, K, V, KCACHE, VCACHE, LENGTHS, PAGES = 1, 2, 3, 4, 5, 6, 7


def _mix(z: np.ndarray) -> np.ndarray:
    z = z ^ (z >> np.uint64(30))
    z = z * _M1
    z = z ^ (z >> np.uint64(27))
    z = z * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, tensor_id: int) -> int:
    with np.errstate(over="ignore"):
        z = np.array([(seed * (1 << 20) + tensor_id) & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64)
        return int(_mix(z)[0])


def words(key: int, start: int, count: int) -> np.ndarray:
    """splitmix64 words start..start+count-1 of stream `key` (uint64)."""
    with np.errstate(over="ignore"):
        i = np.arange(start + 1, start + count + 1, dtype=np.uint64)
        return _mix(np.uint64(key) + i * _GOLDEN)


def _normals_chunk(key: int, start: int, count: int) -> np.ndarray:
    """float64 normals for elements start..start+count-1 (start, count even)."""
    w = words(key, start, count)
    u = ((w >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)
    u1, u2 = u[0::2], u[1::2]
    r = np.sqrt(-2.0 * np.log(u1))
    t = 2.0 * np.pi * u2
    out = np.empty(count, dtype=np.float64)
    out[0::2] = r * np.cos(t)
    out[1::2] = r * np.sin(t)
    return out


def round_bf16(x32: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest even), returned as float32."""
    b = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32)
    lsb = (b >> np.uint32(16)) & np.uint32(1)
    r = (b + np.uint32(0x7FFF) + lsb) & np.uint32(0xFFFF0000)
    return r.view(np.float32)


def round_tf32(x32: np.ndarray) -> np.ndarray:
    """Round float32 values to tf32 (10 mantissa bits, nearest even), returned as float32."""
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    finite = (u & 0x7F800000) != 0x7F800000
    r = (u + 0x0FFF + ((u >> 13) & 1)) & ~np.uint64(0x1FFF)
    return np.where(finite, r, u).astype(np.uint32).view(np.float32)


def normal(seed: int, tensor_id: int, shape, dtype: str = "bf16", threads: int | None = None) -> np.ndarray:
    """N(0,1) tensor of `shape` stored as `dtype` ('bf16' or 'f32'), as float32 values."""
    n = int(np.prod(shape))
    key = stream_key(seed, tensor_id)
    out = np.empty(n, dtype=np.float32)
    chunk = 1 << 22
    starts = list(range(0, n + (n & 1), chunk))

    def fill(s):
        cnt = min(chunk, n + (n & 1) - s)
        vals = _normals_chunk(key, s, cnt).astype(np.float32)
        if dtype == "bf16":
            vals = round_bf16(vals)
        e = min(s + cnt, n)
        out[s:e] = vals[: e - s]

    if threads is None:
        threads = min(32, os.cpu_count() or 1)
    if len(starts) == 1 or threads <= 1:
        for s in starts:
            fill(s)
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(fill, starts))
    return out.reshape(shape)


def uniform_ints(seed: int, tensor_id: int, count: int, lo: int, hi: int) -> np.ndarray:
    """`count` integers uniform on [lo, hi] inclusive (multiply-shift on the top 32 bits)."""
    w = words(stream_key(seed, tensor_id), 0, count)
    top = (w >> np.uint64(32)).astype(np.uint64)
    span = np.uint64(hi - lo + 1)
    return (lo + ((top * span) >> np.uint64(32))).astype(np.int64)


def varlen_lengths(seed: int, nseq: int, lo: int, hi: int) -> np.ndarray:
    return uniform_ints(seed, LENGTHS, nseq, lo, hi)


def cu_seqlens(lengths) -> np.ndarray:
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return cu


def to_e4m3(x: np.ndarray):
    """Per-tensor e4m3 storage of float32 values: the scale maps the largest magnitude to 448
    (the largest finite e4m3 value); returns (bytes uint8, dequantised float32 values, scale),
    with value = e4m3(byte) * scale.  Conversion: torch's float8_e4m3fn cast (round to nearest
    even, saturating)."""
    import torch
    x = np.ascontiguousarray(x, dtype=np.float32)
    amax = float(np.abs(x).max()) if x.size else 0.0
    scale = amax / 448.0 if amax > 0 else 1.0
    f8 = torch.from_numpy(x / np.float32(scale)).to(torch.float8_e4m3fn)
    return f8.view(torch.uint8).numpy().copy(), (f8.to(torch.float32).numpy() * np.float32(scale)), scale


def permutation(seed: int, tensor_id: int, n: int) -> np.ndarray:
    """A permutation of 0..n-1: the indices that sort n words of the stream (stable)."""
    return np.argsort(words(stream_key(seed, tensor_id), 0, n), kind="stable").astype(np.int64)


def page_layout(seed: int, lengths, page_size: int, extra_pages: int = 0, max_pages: int | None = None):
    """Physical page placement for a paged KV cache.

    Sequence b needs ceil(lengths[b] / page_size) pages.  All needed pages plus
    `extra_pages` spare ones form the pool; the pool is shuffled by `permutation` (stream
    PAGES) and handed out in order, sequence by sequence.  Returns (block_table int32
    [B, max_pages] with -1 in entries a sequence does not use, num_pages)."""
    lengths = np.asarray(lengths, dtype=np.int64)
    need = (lengths + page_size - 1) // page_size
    if max_pages is None:
        max_pages = max(1, int(need.max()) if len(need) else 1)
    num_pages = int(need.sum()) + extra_pages
    perm = permutation(seed, PAGES, max(num_pages, 1))
    table = np.full((len(lengths), max_pages), -1, dtype=np.int32)
    nxt = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[nxt:nxt + n]
        nxt += int(n)
    return table, max(num_pages, 1)


# The benchmark workloads: every tensor is i.i.d. N(0,1); config k uses seed 1000 + k.
WORKLOADS = {
    "single_head_f32": dict(B=1, Hq=1, Hkv=1, N=128, d=64, causal=0, dtype="f32", seed=1001),
    "mha_causal_2k": dict(B=2, Hq=12, Hkv=12, N=2048, d=64, causal=1, dtype="bf16", seed=1002),
    "gqa_causal_8k": dict(B=1, Hq=64, Hkv=8, N=8192, d=128, causal=1, dtype="bf16", seed=1003),
    "varlen_gqa_causal": dict(nseq=16, len_lo=256, len_hi=8192, Hq=32, Hkv=8, d=128, causal=1,
                              dtype="bf16", seed=1004),
    "decode_split_kv": dict(B=8, Hq=64, Hkv=8, L=32768, d=128, split=1024, dtype="bf16", seed=1005),
    # paged, ragged decode: 16 sequences of U{1..32768} tokens in 16-token pages, shuffled pool
    "decode_paged_ragged": dict(B=16, Hq=64, Hkv=8, len_lo=1, len_hi=32768, page_size=16, d=128, split=1024,
                                dtype="bf16", seed=1006),
}
