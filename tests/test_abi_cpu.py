"""CPU-side checks of the C-ABI library: it builds, loads without a GPU, exports every
function include/fa.h declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

from exact_io_aware_97_b200 import binding as fa
from exact_io_aware_97_b200 import build as fa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    fa_build.build()
    return fa.load()


def _declared():
    src = open(os.path.join(ROOT, "include", "fa.h")).read()
    return sorted(set(re.findall(r"FA_EXPORT\s+[\w\s\*]+?\b(fa_\w+)\s*\(", src)))


def test_header_declares_the_binding_names():
    assert _declared() == sorted(fa.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name
    # nothing else leaks out of the library under an fa_ name
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", fa.LIB_PATH], capture_output=True, text=True).stdout
    exported = sorted(set(re.findall(r" T (fa_\w+)", out)))
    assert exported == _declared()


def test_status_strings(lib):
    for s in range(6):
        assert fa.status_string(s)
    assert fa.status_string(99) == "unknown status"


def test_workspace_sizes(lib):
    assert fa.fa_fwd_workspace_size(2, 12, 12, 2048, 2048, 64, fa.FA_BF16, False) == 0
    n = fa.fa_fwd_workspace_size(1, 1, 1, 128, 128, 64, fa.FA_F32, False)
    assert n >= 3 * 128 * 64 * 2
    # varlen fp32: Nq = Nk = the packed row count (not multiplied by B)
    nv = fa.fa_fwd_workspace_size(4, 2, 1, 300, 300, 64, fa.FA_F32, True)
    assert 300 * 2 * 64 * 2 + 2 * 300 * 64 * 2 <= nv < 4 * 300 * 2 * 64 * 2
    ws = fa.fa_decode_workspace_size(8, 64, 32768, 128, 1024)
    assert ws >= 8 * 64 * 32 * (128 + 2) * 4
    assert fa.fa_decode_workspace_size(0, 64, 32768, 128, 1024) == 0


def _fwd_status(lib, **kw):
    args = dict(q=256, k=256, v=256, o=256, lse=None, B=1, Hq=2, Hkv=1, Nq=8, Nk=8, d=64, scale=0.125, causal=1,
                cu=None, dt=0, ws=None, wsb=0, st=None)
    args.update(kw)
    return lib.fa_fwd(args["q"], args["k"], args["v"], args["o"], args["lse"], args["B"], args["Hq"], args["Hkv"],
                      args["Nq"], args["Nk"], args["d"], ctypes.c_float(args["scale"]), args["causal"], args["cu"],
                      args["dt"], args["ws"], args["wsb"], args["st"])


def test_fwd_rejects_before_launch(lib):
    assert _fwd_status(lib, q=None) == fa.FA_ERR_INVALID_ARG
    assert _fwd_status(lib, k=258) == fa.FA_ERR_INVALID_ARG          # misaligned
    assert _fwd_status(lib, d=96) == fa.FA_ERR_UNSUPPORTED
    assert _fwd_status(lib, Hq=3, Hkv=2) == fa.FA_ERR_UNSUPPORTED
    assert _fwd_status(lib, scale=0.0) == fa.FA_ERR_INVALID_ARG
    assert _fwd_status(lib, scale=float("nan")) == fa.FA_ERR_INVALID_ARG
    assert _fwd_status(lib, B=-1) == fa.FA_ERR_INVALID_ARG
    assert _fwd_status(lib, cu=512, Nq=8, Nk=9) == fa.FA_ERR_INVALID_ARG   # varlen needs Nq == Nk
    assert _fwd_status(lib, cu=512, dt=1) == fa.FA_ERR_WORKSPACE           # fp32 varlen needs its bf16 copies
    assert _fwd_status(lib, cu=512, dt=2) == fa.FA_ERR_UNSUPPORTED         # tf32 is fixed length only
    assert _fwd_status(lib, cu=514) == fa.FA_ERR_INVALID_ARG               # misaligned offsets
    assert _fwd_status(lib, dt=1) == fa.FA_ERR_WORKSPACE                   # fp32 needs workspace
    assert _fwd_status(lib, dt=7) == fa.FA_ERR_INVALID_ARG


def _dec_status(lib, **kw):
    args = dict(q=256, kc=256, vc=256, sl=None, o=256, lse=None, B=2, Hq=8, Hkv=2, L=128, d=128, scale=0.1,
                split=64, ws=256, wsb=1 << 30, st=None)
    args.update(kw)
    return lib.fa_decode(args["q"], args["kc"], args["vc"], args["sl"], args["o"], args["lse"], args["B"],
                         args["Hq"], args["Hkv"], args["L"], args["d"], ctypes.c_float(args["scale"]),
                         args["split"], args["ws"], args["wsb"], args["st"])


def test_decode_rejects_before_launch(lib):
    assert _dec_status(lib, o=None) == fa.FA_ERR_INVALID_ARG
    assert _dec_status(lib, vc=264) == fa.FA_ERR_INVALID_ARG
    assert _dec_status(lib, Hq=48, Hkv=2) == fa.FA_ERR_UNSUPPORTED   # group of 24 > 16
    assert _dec_status(lib, split=100) == fa.FA_ERR_UNSUPPORTED      # not a multiple of 64
    assert _dec_status(lib, d=80) == fa.FA_ERR_UNSUPPORTED
    assert _dec_status(lib, ws=None) == fa.FA_ERR_WORKSPACE
    assert _dec_status(lib, wsb=16) == fa.FA_ERR_WORKSPACE
    assert _dec_status(lib, L=0) == fa.FA_ERR_INVALID_ARG
    assert _dec_status(lib, sl=258) == fa.FA_ERR_INVALID_ARG


def _paged_status(lib, **kw):
    args = dict(q=256, kp=256, vp=256, bt=512, sl=768, o=256, lse=None, B=2, Hq=8, Hkv=2, P=10, ps=16, maxp=4,
                d=128, scale=0.1, split=64, ws=256, wsb=1 << 30, st=None)
    args.update(kw)
    return lib.fa_decode_paged(args["q"], args["kp"], args["vp"], args["bt"], args["sl"], args["o"], args["lse"],
                               args["B"], args["Hq"], args["Hkv"], args["P"], args["ps"], args["maxp"], args["d"],
                               ctypes.c_float(args["scale"]), args["split"], args["ws"], args["wsb"], args["st"])


def test_decode_paged_rejects_before_launch(lib):
    assert _paged_status(lib, bt=None) == fa.FA_ERR_INVALID_ARG      # block table required
    assert _paged_status(lib, sl=None) == fa.FA_ERR_INVALID_ARG      # lengths required
    assert _paged_status(lib, bt=514) == fa.FA_ERR_INVALID_ARG       # misaligned table
    assert _paged_status(lib, kp=264) == fa.FA_ERR_INVALID_ARG
    assert _paged_status(lib, ps=24) == fa.FA_ERR_UNSUPPORTED        # not a power of two
    assert _paged_status(lib, ps=8) == fa.FA_ERR_UNSUPPORTED         # below 16
    assert _paged_status(lib, ps=0) == fa.FA_ERR_INVALID_ARG
    assert _paged_status(lib, P=0) == fa.FA_ERR_INVALID_ARG
    assert _paged_status(lib, maxp=0) == fa.FA_ERR_INVALID_ARG
    assert _paged_status(lib, split=96) == fa.FA_ERR_UNSUPPORTED
    assert _paged_status(lib, Hq=34, Hkv=2) == fa.FA_ERR_UNSUPPORTED
    assert _paged_status(lib, P=1 << 27, ps=16) == fa.FA_ERR_UNSUPPORTED    # pool rows >= 2^31
    assert _paged_status(lib, ws=None) == fa.FA_ERR_WORKSPACE
    assert _paged_status(lib, wsb=64) == fa.FA_ERR_WORKSPACE
    assert _paged_status(lib, B=0) == fa.FA_OK


def test_decode_paged_workspace_holds_the_partials(lib):
    B, Hq, Hkv, maxp, ps, d, split = 16, 64, 8, 2048, 16, 128, 1024
    n = fa.fa_decode_paged_workspace_size(B, Hq, Hkv, maxp, ps, d, split)
    nsplit = (maxp * ps + split - 1) // split
    assert n >= B * Hq * nsplit * (d + 2) * 4
    assert n == fa.fa_decode_workspace_size(B, Hq, maxp * ps, d, split)
    assert fa.fa_decode_paged_workspace_size(0, Hq, Hkv, maxp, ps, d, split) == 0


def test_empty_problems_are_noops(lib):
    # B == 0 or Nq == 0: valid, nothing launched
    assert _fwd_status(lib, B=0) == fa.FA_OK
    assert _fwd_status(lib, Nq=0) == fa.FA_OK
    assert _dec_status(lib, B=0) == fa.FA_OK


def test_binding_raises_fa_error(lib):
    with pytest.raises(fa.FaError) as e:
        fa.fa_fwd(256, 256, 256, 256, None, 1, 2, 1, 8, 8, 96, 0.1, 1, stream=0)
    assert e.value.status == fa.FA_ERR_UNSUPPORTED


def test_binding_refuses_host_and_strided_tensors(lib):
    """The binding hands the library only dense device memory: a host tensor or a strided
    view raises before any call (the library itself cannot tell a host pointer from a device
    one)."""
    import torch
    host = torch.zeros(1, 8, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        fa.fa_fwd(host, 256, 256, 256, None, 1, 2, 1, 8, 8, 64, 0.1, 1, stream=0)
    with pytest.raises(ValueError, match="CUDA tensor"):
        fa.forward(host, host, host, stream=0)
    with pytest.raises(ValueError, match="CUDA tensor"):
        fa.fa_decode(256, 256, 256, torch.zeros(2, dtype=torch.int32), 256, None, 2, 8, 2, 64, 64, 0.1, 64, 256,
                     1 << 20, stream=0)

    class FakeStrided:  # a device tensor whose layout is not dense
        is_cuda = True
        shape, device = (8, 64), "cuda:0"

        def is_contiguous(self):
            return False

        def stride(self):
            return (1, 8)

        def data_ptr(self):
            raise AssertionError("a strided tensor's address must not be taken")
    with pytest.raises(ValueError, match="contiguous"):
        fa.fa_fwd(FakeStrided(), 256, 256, 256, None, 1, 2, 1, 8, 8, 64, 0.1, 1, stream=0)


def test_binding_checks_index_types_and_output_shapes(lib):
    """Index tensors must be int32 and caller-provided outputs must match what the kernels
    write; the binding says so before anything is called."""
    import torch
    bf = torch.bfloat16
    q = torch.zeros(2, 16, 4, 64, dtype=bf)
    k = torch.zeros(2, 16, 2, 64, dtype=bf)
    with pytest.raises(ValueError, match="int32"):
        fa.fa_fwd(256, 256, 256, 256, None, 2, 4, 2, 16, 16, 64, 0.1, 1, cu_seqlens=torch.zeros(3, dtype=torch.int64),
                  stream=0)
    with pytest.raises(ValueError, match="int32"):
        fa.fa_decode(256, 256, 256, torch.zeros(2, dtype=torch.int64), 256, None, 2, 8, 2, 64, 64, 0.1, 64, 256,
                     1 << 20, stream=0)
    with pytest.raises(ValueError, match="int32"):
        fa.fa_decode_paged(256, 256, 256, torch.zeros(2, 4, dtype=torch.int64), None, 256, None, 2, 8, 2, 16, 16,
                           4, 64, 0.1, 64, 256, 1 << 20, stream=0)
    with pytest.raises(ValueError, match="out"):
        fa.forward(q, k, k, out=torch.zeros(2, 16, 4, 64, dtype=torch.float32), stream=0)
    with pytest.raises(ValueError, match="lse"):
        fa.forward(q, k, k, lse=torch.zeros(2, 16, 4, dtype=torch.float32), stream=0)
    with pytest.raises(ValueError, match="k, v"):
        fa.forward(q, k, torch.zeros(2, 15, 2, 64, dtype=bf), stream=0)
    with pytest.raises(ValueError, match="does not match"):
        fa.forward(q, k.float(), k.float(), stream=0)
    with pytest.raises(ValueError, match="lse"):
        fa.backward(q, k, k, q, torch.zeros(2, 4, 15, dtype=torch.float32), q, stream=0)
    with pytest.raises(ValueError, match="q, o, dout"):
        fa.backward(q, k, k, q.float(), torch.zeros(2, 4, 16, dtype=torch.float32), q, stream=0)
    with pytest.raises(ValueError, match="bf16"):
        qf, kf = q.float(), k.float()
        fa.backward(qf, kf, kf, qf, torch.zeros(2, 4, 16, dtype=torch.float32), qf, stream=0)
    with pytest.raises(ValueError, match="bf16"):
        fa.decode(torch.zeros(2, 4, 64), torch.zeros(2, 32, 2, 64), torch.zeros(2, 32, 2, 64), stream=0)
    with pytest.raises(ValueError, match="block_table"):
        fa.decode_paged(torch.zeros(2, 4, 64, dtype=bf), torch.zeros(8, 16, 2, 64, dtype=bf),
                        torch.zeros(8, 16, 2, 64, dtype=bf), torch.zeros(3, 4, dtype=torch.int32),
                        torch.zeros(2, dtype=torch.int32), stream=0)


def test_binding_checks_shapes_across_tensors(lib):
    """The kernels size every read from q's batch, heads and head dimension: a k, cache or
    length vector that does not match q is refused by the binding with a ValueError (a
    smaller tensor would otherwise be read past its end on the device)."""
    import torch
    bf, i32 = torch.bfloat16, torch.int32
    q = torch.zeros(2, 16, 4, 64, dtype=bf)
    with pytest.raises(ValueError, match="batch 2"):
        fa.forward(q, torch.zeros(1, 16, 2, 64, dtype=bf), torch.zeros(1, 16, 2, 64, dtype=bf), stream=0)
    with pytest.raises(ValueError, match="multiple of Hkv"):
        fa.forward(q, torch.zeros(2, 16, 3, 64, dtype=bf), torch.zeros(2, 16, 3, 64, dtype=bf), stream=0)
    qp = torch.zeros(40, 4, 64, dtype=bf)
    with pytest.raises(ValueError, match="packed rows"):
        fa.forward(qp, torch.zeros(39, 2, 64, dtype=bf), torch.zeros(39, 2, 64, dtype=bf),
                   cu_seqlens=torch.tensor([0, 40], dtype=i32), stream=0)
    with pytest.raises(ValueError, match="cu_seqlens"):
        fa.forward(qp, torch.zeros(40, 2, 64, dtype=bf), torch.zeros(40, 2, 64, dtype=bf),
                   cu_seqlens=torch.tensor([40], dtype=i32), stream=0)
    qd = torch.zeros(2, 8, 128, dtype=bf)
    with pytest.raises(ValueError, match="kcache"):   # cache of one sequence for two queries
        fa.decode(qd, torch.zeros(1, 64, 2, 128, dtype=bf), torch.zeros(1, 64, 2, 128, dtype=bf), stream=0)
    with pytest.raises(ValueError, match="kcache"):   # head dimension differs from q's
        fa.decode(qd, torch.zeros(2, 64, 2, 64, dtype=bf), torch.zeros(2, 64, 2, 64, dtype=bf), stream=0)
    with pytest.raises(ValueError, match="seqlens"):
        fa.decode(qd, torch.zeros(2, 64, 2, 128, dtype=bf), torch.zeros(2, 64, 2, 128, dtype=bf),
                  seqlens=torch.zeros(1, dtype=i32), stream=0)
    with pytest.raises(ValueError, match="multiple of Hkv"):
        fa.decode(qd, torch.zeros(2, 64, 3, 128, dtype=bf), torch.zeros(2, 64, 3, 128, dtype=bf), stream=0)
    with pytest.raises(ValueError, match="k_pages"):
        fa.decode_paged(qd, torch.zeros(8, 16, 2, 64, dtype=bf), torch.zeros(8, 16, 2, 64, dtype=bf),
                        torch.zeros(2, 4, dtype=i32), torch.zeros(2, dtype=i32), stream=0)
    with pytest.raises(ValueError, match="seqlens"):
        fa.decode_paged(qd, torch.zeros(8, 16, 2, 128, dtype=bf), torch.zeros(8, 16, 2, 128, dtype=bf),
                        torch.zeros(2, 4, dtype=i32), torch.zeros(3, dtype=i32), stream=0)
    lse = torch.zeros(2, 4, 16, dtype=torch.float32)
    with pytest.raises(ValueError, match="k"):
        fa.backward(q, torch.zeros(1, 16, 2, 64, dtype=bf), torch.zeros(1, 16, 2, 64, dtype=bf), q, lse, q, stream=0)
    with pytest.raises(ValueError, match="d=64"):
        fa.backward(q, torch.zeros(2, 16, 2, 128, dtype=bf), torch.zeros(2, 16, 2, 128, dtype=bf), q, lse, q,
                    stream=0)
    with pytest.raises(ValueError, match="total=40"):
        fa.backward_varlen(qp, torch.zeros(39, 2, 64, dtype=bf), torch.zeros(39, 2, 64, dtype=bf), qp,
                           torch.zeros(4, 40), qp, torch.tensor([0, 40], dtype=i32), stream=0)
    with pytest.raises(ValueError, match="qkv"):
        fa.forward_qkvpacked(torch.zeros(2, 16, 2, 4, 64, dtype=bf))
    u8 = torch.uint8
    with pytest.raises(ValueError, match="k8"):
        fa.forward_fp8(torch.zeros(2, 16, 4, 128, dtype=u8), torch.zeros(1, 16, 2, 128, dtype=u8),
                       torch.zeros(1, 16, 2, 128, dtype=u8), 1.0, 1.0, 1.0)


def test_bwd_rejects_before_launch(lib):
    def st(**kw):
        a = dict(q=256, k=256, v=256, o=256, do=256, lse=512, dq=256, dk=256, dv=256, B=1, Hq=2, Hkv=1, Nq=8, Nk=8,
                 d=128, scale=0.1, causal=1, ws=256, wsb=1 << 30)
        a.update(kw)
        return lib.fa_bwd(a["q"], a["k"], a["v"], a["o"], a["do"], a["lse"], a["dq"], a["dk"], a["dv"], a["B"],
                          a["Hq"], a["Hkv"], a["Nq"], a["Nk"], a["d"], ctypes.c_float(a["scale"]), a["causal"],
                          a["ws"], a["wsb"], None)
    assert st(do=None) == fa.FA_ERR_INVALID_ARG
    assert st(lse=None) == fa.FA_ERR_INVALID_ARG
    assert st(dk=264) == fa.FA_ERR_INVALID_ARG       # misaligned
    assert st(lse=514) == fa.FA_ERR_INVALID_ARG      # misaligned lse
    assert st(d=96) == fa.FA_ERR_UNSUPPORTED
    assert st(Hq=3, Hkv=2) == fa.FA_ERR_UNSUPPORTED
    assert st(scale=-1.0) == fa.FA_ERR_INVALID_ARG
    assert st(ws=None) == fa.FA_ERR_WORKSPACE
    assert st(B=0) == fa.FA_OK
    assert fa.fa_bwd_workspace_size(1, 64, 8192, 128) >= 8192 * 64 * 128 * 4


def test_bwd_varlen_rejects_before_launch(lib):
    def st(**kw):
        a = dict(q=256, k=256, v=256, o=256, do=256, lse=512, dq=256, dk=256, dv=256, B=2, Hq=2, Hkv=1, total=8,
                 d=128, scale=0.1, causal=1, cu=1024, ws=256, wsb=1 << 30)
        a.update(kw)
        return lib.fa_bwd_varlen(a["q"], a["k"], a["v"], a["o"], a["do"], a["lse"], a["dq"], a["dk"], a["dv"],
                                 a["B"], a["Hq"], a["Hkv"], a["total"], a["d"], ctypes.c_float(a["scale"]),
                                 a["causal"], a["cu"], a["ws"], a["wsb"], None)
    assert st(cu=None) == fa.FA_ERR_INVALID_ARG
    assert st(cu=1026) == fa.FA_ERR_INVALID_ARG      # misaligned cu_seqlens
    assert st(dv=None) == fa.FA_ERR_INVALID_ARG
    assert st(q=264) == fa.FA_ERR_INVALID_ARG        # misaligned
    assert st(total=-1) == fa.FA_ERR_INVALID_ARG
    assert st(d=96) == fa.FA_ERR_UNSUPPORTED
    assert st(Hq=3, Hkv=2) == fa.FA_ERR_UNSUPPORTED
    assert st(scale=float("nan")) == fa.FA_ERR_INVALID_ARG
    assert st(ws=None) == fa.FA_ERR_WORKSPACE
    assert st(wsb=fa.fa_bwd_varlen_workspace_size(2, 2, 8, 128) - 1) == fa.FA_ERR_WORKSPACE
    assert st(B=0) == fa.FA_OK
    assert st(total=0) == fa.FA_OK
    assert fa.fa_bwd_varlen_workspace_size(0, 2, 8, 128) == 0
    # the row vectors hold one 128-row tile per sequence even when every sequence is one row
    # long (the most tiles per row), next to the fp32 dq accumulator
    for B, Hq, d in ((1, 1, 64), (16, 32, 128), (1000, 8, 128)):
        assert fa.fa_bwd_varlen_workspace_size(B, Hq, B, d) >= 2 * Hq * B * 128 * 4 + B * Hq * d * 4
    assert fa.fa_bwd_varlen_workspace_size(16, 32, 67584, 128) >= 67584 * 32 * 128 * 4


def test_fp8_and_packed_reject_before_launch(lib):
    def st8(**kw):
        a = dict(q=256, k=256, v=256, o=256, lse=None, B=1, Hq=2, Hkv=1, Nq=8, Nk=8, d=128, scale=0.1, dq=1.0,
                 dk=1.0, dv=1.0, causal=1, ws=256, wsb=1 << 20)
        a.update(kw)
        return lib.fa_fwd_fp8(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"], a["Hkv"], a["Nq"], a["Nk"],
                              a["d"], ctypes.c_float(a["scale"]), ctypes.c_float(a["dq"]), ctypes.c_float(a["dk"]),
                              ctypes.c_float(a["dv"]), a["causal"], a["ws"], a["wsb"], None)
    assert st8(d=64) == fa.FA_ERR_UNSUPPORTED        # e4m3 path is d = 128 only
    assert st8(dv=0.0) == fa.FA_ERR_INVALID_ARG
    assert st8(dq=float("inf")) == fa.FA_ERR_INVALID_ARG
    assert st8(ws=None) == fa.FA_ERR_WORKSPACE
    assert st8(B=0) == fa.FA_OK
    assert fa.fa_fwd_fp8_workspace_size(1, 8, 8192, 128) == 8 * 128 * 8192
    assert fa.fa_fwd_fp8_workspace_size(1, 8, 8192, 64) == 0

    def stp(**kw):
        a = dict(qkv=256, o=256, lse=None, B=2, H=12, N=2048, d=64, scale=0.125, causal=1, cu=None)
        a.update(kw)
        return lib.fa_fwd_qkvpacked(a["qkv"], a["o"], a["lse"], a["B"], a["H"], a["N"], a["d"],
                                    ctypes.c_float(a["scale"]), a["causal"], a["cu"], None)
    assert stp(qkv=None) == fa.FA_ERR_INVALID_ARG
    assert stp(o=264) == fa.FA_ERR_INVALID_ARG
    assert stp(d=80) == fa.FA_ERR_UNSUPPORTED
    assert stp(cu=514) == fa.FA_ERR_INVALID_ARG
    assert stp(N=0) == fa.FA_OK


def test_tf32_workspace_and_rejects(lib):
    assert fa.fa_fwd_workspace_size(1, 1, 1, 128, 128, 64, fa.FA_TF32, False) >= 3 * 128 * 64 * 4
    assert fa.fa_fwd_workspace_size(1, 1, 1, 128, 128, 128, fa.FA_TF32, False) == 0
    assert _fwd_status(lib, dt=fa.FA_TF32, d=128) == fa.FA_ERR_UNSUPPORTED
    assert _fwd_status(lib, dt=fa.FA_TF32, cu=512) == fa.FA_ERR_UNSUPPORTED
    assert _fwd_status(lib, dt=fa.FA_TF32) == fa.FA_ERR_WORKSPACE
