"""Benchmark of the exact-attention hot path on B200.

One step = one pass of the whole path: the tiled forward on the GQA causal long-context
workload (B=1, Hq=64, Hkv=8, N=8192, d=128, bf16) and the split-KV decode on the decode
workload (B=8, Hq=64, Hkv=8, cache 32768, d=128, splits of 1024).  The headline value is the
forward's TFLOP/s (4 B Hq N^2 d, halved for causal); the decode's HBM GB/s (K and V bytes
read once) is reported in the "decode" object.  Inputs are synthetic i.i.d. N(0,1) from the
seeded generator, resident in HBM before timing; L2 is flushed before every timed launch,
outside its events: a 256 MiB write, then a read of another 256 MiB buffer, so that the
write's dirty lines are written back before the launch rather than during it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

With N > 1 (launched by torch.distributed.run) every rank runs its own replica of the
workload (the units are independent: no collective on the data path); times are the max
over ranks.  --impl reference times the fp64 CPU oracle on bounded samples of the same
workloads instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth_inputs as si  # noqa: E402

METRIC = "attention fwd TFLOP/s & % of BF16 tensor peak; decode HBM GB/s & % of peak"
SPEC_BF16_TFLOPS = 2250.0
SPEC_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0

FWD = si.WORKLOADS["gqa_causal_8k"]
DEC = si.WORKLOADS["decode_split_kv"]
PAGED = si.WORKLOADS["decode_paged_ragged"]
MHA2K = si.WORKLOADS["mha_causal_2k"]
VARLEN = si.WORKLOADS["varlen_gqa_causal"]
DOUT_ID = 9  # stream id of the backward's upstream gradient


def fwd_flops(w=FWD) -> float:
    f = 4.0 * w["B"] * w["Hq"] * w["N"] * w["N"] * w["d"]
    return f / 2 if w["causal"] else f


def fwd_bytes(w=FWD) -> float:
    B, N, Hq, Hkv, d = w["B"], w["N"], w["Hq"], w["Hkv"], w["d"]
    return 2.0 * B * N * Hq * d * 2 + 2.0 * 2 * B * N * Hkv * d + 4.0 * B * Hq * N


def dec_kv_bytes(w=DEC) -> float:
    return 2.0 * w["B"] * w["L"] * w["Hkv"] * w["d"] * 2


def paged_lengths(seed: int, w=PAGED) -> np.ndarray:
    return si.uniform_ints(seed, si.LENGTHS, w["B"], w["len_lo"], w["len_hi"])


def paged_kv_bytes(lengths, w=PAGED) -> float:
    return 2.0 * float(np.sum(lengths)) * w["Hkv"] * w["d"] * 2


def varlen_lengths(seed: int, w=VARLEN) -> np.ndarray:
    return si.varlen_lengths(seed, w["nseq"], w["len_lo"], w["len_hi"])


def varlen_flops(lengths, w=VARLEN) -> float:
    """Forward FLOPs of packed causal sequences: sum over sequences of 4 Hq L^2 d, halved."""
    return float(sum(4.0 * w["Hq"] * float(L) * float(L) * w["d"] for L in lengths)) / 2.0


def dec_flops(w=DEC) -> float:
    return 4.0 * w["B"] * w["Hq"] * w["L"] * w["d"]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm": j["hbm_gbs"], "bf16": j["bf16_tflops"], "bf16_sustained": j["bf16_tflops_sustained"],
                "source": "measured"}
    return {"hbm": FALLBACK_HBM_GBS, "bf16": FALLBACK_BF16_TFLOPS, "bf16_sustained": 1400.0, "source": "fallback"}


def kernel_src_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "exact_io_aware_97_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(key: str):
    """DRAM bytes per launch from a committed ncu summary, if taken on the current kernels."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        j = json.load(f)
    e = j.get(key)
    if not e or e.get("src_sha") != kernel_src_hash():
        return None
    return e.get("bytes_per_launch")


# ----------------------------------------------------------------------------- ranks
def replica_seed(base_seed: int, rank: int) -> int:
    """Each rank runs its own replica of the workload on its own seeded inputs."""
    return base_seed + 100000 * rank


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank time over the process group (identity without one)."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(units_per_replica: float, world: int, max_ms: float) -> float:
    """Whole-job rate: the units all ranks processed over the slowest rank's time (per second)."""
    return world * units_per_replica / (max_ms * 1e-3)


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.marks = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100", "-i", str(self.gpu)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, ValueError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, on: bool):
        self.marks.append((time.time(), on))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.lines:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        # samples inside timed windows
        wins, cur = [], None
        for t, on in self.marks:
            if on:
                cur = t
            elif cur is not None:
                wins.append((cur, t))
                cur = None
        inside = [l for t, l in self.lines if any(a - 0.15 <= t <= b + 0.15 for a, b in wins)] or [l for _, l in self.lines]
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in inside:
            parts = [x.strip() for x in l.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- device arm
def run_device(args):
    import torch
    import torch.distributed as dist

    from exact_io_aware_97_b200 import binding as fa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    fa.load()
    peaks = load_peaks()
    st = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_rd = torch.ones(64 << 20, dtype=torch.float32, device=dev)  # 256 MiB

    def l2_flush():
        # write a buffer larger than L2, then read another one: L2 holds neither the previous
        # launch's data nor dirty lines whose write-back would land inside the timed launch
        flush.fill_(1)
        flush_rd.sum()

    # ---- inputs (each rank its own replica, seeded by the workload seed + rank)
    w = FWD
    B, N, Hq, Hkv, d = w["B"], w["N"], w["Hq"], w["Hkv"], w["d"]
    seed = replica_seed(w["seed"], rank)
    h_q = torch.from_numpy(inputs("fwd", seed, si.Q, (B, N, Hq, d))).to(torch.bfloat16).pin_memory()
    h_k = torch.from_numpy(inputs("fwd", seed, si.K, (B, N, Hkv, d))).to(torch.bfloat16).pin_memory()
    h_v = torch.from_numpy(inputs("fwd", seed, si.V, (B, N, Hkv, d))).to(torch.bfloat16).pin_memory()
    q, k, v = h_q.to(dev), h_k.to(dev), h_v.to(dev)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=dev)
    h_o = torch.empty(o.shape, dtype=torch.bfloat16).pin_memory()
    h_lse = torch.empty(lse.shape, dtype=torch.float32).pin_memory()
    scale = 1.0 / math.sqrt(d)

    do_fwd = args.only in ("all", "fwd")
    do_dec = args.only in ("all", "dec")
    do_paged = args.only in ("all", "paged")
    do_bwd = args.only in ("all", "bwd")
    do_fp8 = args.only in ("all", "fp8")
    do_tf32 = args.only in ("all", "tf32")
    do_bwdv = args.only == "bwd_varlen"  # on request only: its inputs take about a minute to draw
    do_mha2k = args.only in ("all", "mha2k")
    do_varlen = args.only in ("all", "varlen")
    if do_bwd:
        h_do_f = torch.from_numpy(inputs("fwd", seed, DOUT_ID, (B, N, Hq, d))).to(torch.bfloat16)
        b_do = h_do_f.to(dev)
        b_dq, b_dk, b_dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        b_ws_bytes = fa.fa_bwd_workspace_size(B, Hq, N, d)
        b_ws = torch.empty(b_ws_bytes, dtype=torch.uint8, device=dev)
    if not do_fwd and not do_bwd:
        del q, k, v, o, lse
    wd = DEC
    dseed = replica_seed(wd["seed"], rank)
    dB, dHq, dHkv, L, dd, split = wd["B"], wd["Hq"], wd["Hkv"], wd["L"], wd["d"], wd["split"]
    if not do_dec:
        dB = 1  # a token-sized decode problem keeps the code below uniform
        dq = kc = vc = None
    h_dq = torch.from_numpy(inputs("dec", dseed, si.Q, (dB, dHq, dd))).to(torch.bfloat16).pin_memory()
    h_kc = torch.from_numpy(inputs("dec", dseed, si.KCACHE, (dB, L, dHkv, dd))).to(torch.bfloat16).pin_memory()
    h_vc = torch.from_numpy(inputs("dec", dseed, si.VCACHE, (dB, L, dHkv, dd))).to(torch.bfloat16).pin_memory()
    dq, kc, vc = h_dq.to(dev), h_kc.to(dev), h_vc.to(dev)
    do = torch.empty((dB, dHq, dd), dtype=torch.bfloat16, device=dev)
    dlse = torch.empty((dB, dHq), dtype=torch.float32, device=dev)
    ws_bytes = fa.fa_decode_workspace_size(dB, dHq, L, dd, split)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    h_do = torch.empty(do.shape, dtype=torch.bfloat16).pin_memory()
    dscale = 1.0 / math.sqrt(dd)

    # ---- paged ragged decode: shuffled pool of 16-token pages, block table, lengths
    wp = PAGED
    pseed = replica_seed(wp["seed"], rank)
    # the lengths are the workload's shape, the same on every rank (so N ranks do N times the
    # work of one); the values and the page placement are each rank's own
    p_len = paged_lengths(wp["seed"]) if do_paged else np.ones(1, np.int64)
    pB = len(p_len)
    pps, pHq, pHkv, pd, psplit = wp["page_size"], wp["Hq"], wp["Hkv"], wp["d"], wp["split"]
    table_np, npages = si.page_layout(pseed, p_len, pps)
    p_q = torch.from_numpy(inputs("paged", pseed, si.Q, (pB, pHq, pd))).to(torch.bfloat16).to(dev)
    p_k = torch.from_numpy(inputs("paged", pseed, si.KCACHE, (npages, pps, pHkv, pd))).to(torch.bfloat16).to(dev)
    p_v = torch.from_numpy(inputs("paged", pseed, si.VCACHE, (npages, pps, pHkv, pd))).to(torch.bfloat16).to(dev)
    p_table = torch.from_numpy(table_np).to(dev)
    p_lens = torch.from_numpy(p_len.astype(np.int32)).to(dev)
    p_o = torch.empty((pB, pHq, pd), dtype=torch.bfloat16, device=dev)
    p_lse = torch.empty((pB, pHq), dtype=torch.float32, device=dev)
    p_ws_bytes = fa.fa_decode_paged_workspace_size(pB, pHq, pHkv, table_np.shape[1], pps, pd, psplit)
    p_ws = torch.empty(p_ws_bytes, dtype=torch.uint8, device=dev)

    if do_fp8:
        f8 = [si.to_e4m3(inputs("fwd", seed, tid, shp)) for tid, shp in
              ((si.Q, (B, N, Hq, d)), (si.K, (B, N, Hkv, d)), (si.V, (B, N, Hkv, d)))]
        f8_q, f8_k, f8_v = (torch.from_numpy(t[0]).to(dev) for t in f8)
        f8_desc = [t[2] for t in f8]
        f8_o = torch.empty((B, N, Hq, d), dtype=torch.bfloat16, device=dev)
        f8_lse = torch.empty((B, Hq, N), dtype=torch.float32, device=dev)
        f8_ws_bytes = fa.fa_fwd_fp8_workspace_size(B, Hkv, N, d)
        f8_ws = torch.empty(f8_ws_bytes, dtype=torch.uint8, device=dev)

    if do_tf32:
        wt = MHA2K
        tB, tN, tH, td = wt["B"], wt["N"], wt["Hq"], wt["d"]
        tq, tk, tv = (torch.from_numpy(inputs("tf32", wt["seed"] + 100000 * rank, tid, (tB, tN, tH, td)))
                      .to(dev) for tid in (si.Q, si.K, si.V))
        t_o = torch.empty((tB, tN, tH, td), dtype=torch.float32, device=dev)
        t_lse = torch.empty((tB, tH, tN), dtype=torch.float32, device=dev)
        t_ws_bytes = fa.fa_fwd_workspace_size(tB, tH, tH, tN, tN, td, fa.FA_TF32, False)
        t_ws = torch.empty(t_ws_bytes, dtype=torch.uint8, device=dev)

    if do_bwdv:
        vseed = replica_seed(VARLEN["seed"], rank)
        v_len = varlen_lengths(VARLEN["seed"])  # the same lengths on every rank, own values
        v_cu_np = si.cu_seqlens(v_len)
        vT, vB = int(v_cu_np[-1]), len(v_len)
        vHq, vHkv, vd = VARLEN["Hq"], VARLEN["Hkv"], VARLEN["d"]
        v_q, v_k, v_v, v_do = (torch.from_numpy(inputs("varlen", vseed, tid, (vT, hh, vd))).to(torch.bfloat16).to(dev)
                               for tid, hh in ((si.Q, vHq), (si.K, vHkv), (si.V, vHkv), (DOUT_ID, vHq)))
        v_cu = torch.from_numpy(v_cu_np).to(dev)
        v_o = torch.empty_like(v_q)
        v_lse = torch.empty((vHq, vT), dtype=torch.float32, device=dev)
        vscale = 1.0 / math.sqrt(vd)
        fa.fa_fwd(v_q, v_k, v_v, v_o, v_lse, vB, vHq, vHkv, vT, vT, vd, vscale, 1, v_cu, fa.FA_BF16, None, 0, st)
        v_dq, v_dk, v_dv = torch.empty_like(v_q), torch.empty_like(v_k), torch.empty_like(v_v)
        v_ws_bytes = fa.fa_bwd_varlen_workspace_size(vB, vHq, vT, vd)
        v_ws = torch.empty(v_ws_bytes, dtype=torch.uint8, device=dev)

    if do_mha2k:
        wm = MHA2K
        mB, mN, mH, md = wm["B"], wm["N"], wm["Hq"], wm["d"]
        mseed = replica_seed(wm["seed"], rank)
        m_q, m_k, m_v = (torch.from_numpy(inputs("mha2k", mseed, tid, (mB, mN, mH, md))).to(torch.bfloat16).to(dev)
                         for tid in (si.Q, si.K, si.V))
        m_o = torch.empty_like(m_q)
        m_lse = torch.empty((mB, mH, mN), dtype=torch.float32, device=dev)

    if do_varlen:
        fseed = replica_seed(VARLEN["seed"], rank)
        f_len = varlen_lengths(VARLEN["seed"])  # the same lengths on every rank, own values
        f_cu_np = si.cu_seqlens(f_len)
        fT, fB = int(f_cu_np[-1]), len(f_len)
        fHq, fHkv, fd = VARLEN["Hq"], VARLEN["Hkv"], VARLEN["d"]
        f_q, f_k, f_v = (torch.from_numpy(inputs("varlen", fseed, tid, (fT, hh, fd))).to(torch.bfloat16).to(dev)
                         for tid, hh in ((si.Q, fHq), (si.K, fHkv), (si.V, fHkv)))
        f_cu = torch.from_numpy(f_cu_np).to(dev)
        f_o = torch.empty_like(f_q)
        f_lse = torch.empty((fHq, fT), dtype=torch.float32, device=dev)

    def call_mha2k():
        fa.fa_fwd(m_q, m_k, m_v, m_o, m_lse, mB, mH, mH, mN, mN, md, 1.0 / math.sqrt(md), 1, None, fa.FA_BF16, None, 0,
                  st)

    def call_varlen():
        fa.fa_fwd(f_q, f_k, f_v, f_o, f_lse, fB, fHq, fHkv, fT, fT, fd, 1.0 / math.sqrt(fd), 1, f_cu, fa.FA_BF16,
                  None, 0, st)

    def call_bwdv():
        fa.fa_bwd_varlen(v_q, v_k, v_v, v_o, v_do, v_lse, v_dq, v_dk, v_dv, vB, vHq, vHkv, vT, vd, vscale, 1, v_cu,
                         v_ws, v_ws_bytes, st)

    def call_tf32():
        fa.fa_fwd(tq, tk, tv, t_o, t_lse, tB, tH, tH, tN, tN, td, 1.0 / math.sqrt(td), 1, None, fa.FA_TF32, t_ws,
                  t_ws_bytes, st)

    def call_fp8():
        fa.fa_fwd_fp8(f8_q, f8_k, f8_v, f8_o, f8_lse, B, Hq, Hkv, N, N, d, scale, f8_desc[0], f8_desc[1], f8_desc[2],
                      1, f8_ws, f8_ws_bytes, st)

    def call_bwd():
        fa.fa_bwd(q, k, v, o, b_do, lse, b_dq, b_dk, b_dv, B, Hq, Hkv, N, N, d, scale, 1, b_ws, b_ws_bytes, st)

    def call_paged():
        fa.fa_decode_paged(p_q, p_k, p_v, p_table, p_lens, p_o, p_lse, pB, pHq, pHkv, npages, pps,
                           table_np.shape[1], pd, 1.0 / math.sqrt(pd), psplit, p_ws, p_ws_bytes, st)

    def call_fwd():
        fa.fa_fwd(q, k, v, o, lse, B, Hq, Hkv, N, N, d, scale, 1, None, fa.FA_BF16, None, 0, st)

    def call_dec(qq=None, kk=None, vv=None):
        fa.fa_decode(qq if qq is not None else dq, kk if kk is not None else kc, vv if vv is not None else vc, None,
                     do, dlse, dB, dHq, dHkv, L, dd, dscale, split, ws, ws_bytes, st)

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)

    def timed_launches(fn, steps, warmup):
        for _ in range(warmup):
            l2_flush()
            fn()
        barrier()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        clocks.mark(True)
        for a, b in evs:
            l2_flush()
            a.record(st)
            fn()
            b.record(st)
        barrier()
        clocks.mark(False)
        ms = [a.elapsed_time(b) for a, b in evs]
        return ms

    fwd_ms = timed_launches(call_fwd, args.steps, args.warmup) if do_fwd else [float("nan")]
    dec_ms = timed_launches(call_dec, args.steps, args.warmup) if do_dec else [float("nan")]
    paged_ms = timed_launches(call_paged, args.steps, args.warmup) if do_paged else [float("nan")]
    if do_bwd and not do_fwd:
        call_fwd()  # the backward consumes the forward's o and lse
    bwd_ms = timed_launches(call_bwd, args.steps, args.warmup) if do_bwd else [float("nan")]
    fp8_ms = timed_launches(call_fp8, args.steps, args.warmup) if do_fp8 else [float("nan")]
    tf32_ms = timed_launches(call_tf32, args.steps, args.warmup) if do_tf32 else [float("nan")]
    bwdv_ms = timed_launches(call_bwdv, args.steps, args.warmup) if do_bwdv else [float("nan")]
    mha2k_ms = timed_launches(call_mha2k, args.steps, args.warmup) if do_mha2k else [float("nan")]
    varlen_ms = timed_launches(call_varlen, args.steps, args.warmup) if do_varlen else [float("nan")]
    if fa.fa_last_device_error(st) != fa.FA_OK:
        raise RuntimeError("device-side timeout recorded during the benchmark")

    # ---- end to end through the C ABI with host buffers (copies inside the timed region)
    def e2e(steps, warmup, body):
        for _ in range(warmup):
            body()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        clocks.mark(True)
        a.record(st)
        for _ in range(steps):
            body()
        b.record(st)
        barrier()
        clocks.mark(False)
        return a.elapsed_time(b) / steps

    def fwd_e2e_body():
        q.copy_(h_q, non_blocking=True)
        k.copy_(h_k, non_blocking=True)
        v.copy_(h_v, non_blocking=True)
        call_fwd()
        h_o.copy_(o, non_blocking=True)
        h_lse.copy_(lse, non_blocking=True)

    def dec_e2e_body():
        dq.copy_(h_dq, non_blocking=True)
        kc.copy_(h_kc, non_blocking=True)
        vc.copy_(h_vc, non_blocking=True)
        call_dec()
        h_do.copy_(do, non_blocking=True)

    e2e_steps = max(3, args.steps // 4)
    fwd_e2e_ms = e2e(e2e_steps, 1, fwd_e2e_body) if (do_fwd and not args.no_e2e) else float("nan")
    dec_e2e_ms = e2e(e2e_steps, 1, dec_e2e_body) if (do_dec and not args.no_e2e) else float("nan")
    torch.cuda.synchronize()
    clocks.stop()

    # ---- reduce over ranks (max time)
    fwd_mean = max_over_ranks(sum(fwd_ms) / len(fwd_ms), dev)
    dec_mean = max_over_ranks(sum(dec_ms) / len(dec_ms), dev)
    paged_mean = max_over_ranks(sum(paged_ms) / len(paged_ms), dev)
    bwd_mean = max_over_ranks(sum(bwd_ms) / len(bwd_ms), dev)
    fp8_mean = max_over_ranks(sum(fp8_ms) / len(fp8_ms), dev)
    tf32_mean = max_over_ranks(sum(tf32_ms) / len(tf32_ms), dev)
    bwdv_mean = max_over_ranks(sum(bwdv_ms) / len(bwdv_ms), dev)
    mha2k_mean = max_over_ranks(sum(mha2k_ms) / len(mha2k_ms), dev)
    varlen_mean = max_over_ranks(sum(varlen_ms) / len(varlen_ms), dev)
    fwd_e2e_ms = max_over_ranks(fwd_e2e_ms, dev)
    dec_e2e_ms = max_over_ranks(dec_e2e_ms, dev)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    F = fwd_flops()
    tflops = aggregate_rate(F, world, fwd_mean) / 1e12
    kv = dec_kv_bytes()
    gbs = aggregate_rate(kv, world, dec_mean) / 1e9
    h2d_fwd = h_q.numel() * 2 + h_k.numel() * 2 + h_v.numel() * 2
    d2h_fwd = h_o.numel() * 2 + h_lse.numel() * 4
    h2d_dec = h_dq.numel() * 2 + h_kc.numel() * 2 + h_vc.numel() * 2
    d2h_dec = h_do.numel() * 2
    burst = (args.steps * fwd_mean) < 1000.0
    tc_peak = peaks["bf16"] if burst else peaks["bf16_sustained"]
    per_launch_tflops = F / (fwd_mean * 1e-3) / 1e12
    per_launch_gbs = kv / (dec_mean * 1e-3) / 1e9
    bwd_flops = 2.5 * F
    bwd_tflops = bwd_flops / (bwd_mean * 1e-3) / 1e12
    bwd_peak = peaks["bf16"] if (args.steps * bwd_mean) < 1000.0 else peaks["bf16_sustained"]
    fp8_tflops = F / (fp8_mean * 1e-3) / 1e12
    fp8_peak = 2.0 * (peaks["bf16"] if (args.steps * fp8_mean) < 1000.0 else peaks["bf16_sustained"])
    F2k = fwd_flops(MHA2K)
    tf32_tflops = F2k / (tf32_mean * 1e-3) / 1e12
    tf32_peak = peaks["bf16"] * 1100.0 / 2250.0
    pkv = paged_kv_bytes(p_len)
    paged_gbs = pkv / (paged_mean * 1e-3) / 1e9
    cpu = cpu_baseline_fwd(args.cpu_seconds) if not args.no_cpu else None
    dec_cpu = cpu_baseline_dec(args.cpu_seconds) if not args.no_cpu else None
    line = {
        "metric": METRIC,
        "value": round(tflops, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(fwd_mean + dec_mean, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic: i.i.d. N(0,1) from seeded splitmix64 + Box-Muller, rounded to bf16",
        "config": {"workload": "gqa_causal_8k: B=1, Hq=64, Hkv=8, N=8192, d=128, causal, layout [B,N,H,d]",
                   "decode_workload": "decode_split_kv: B=8, Hq=64, Hkv=8, cache 32768, d=128, split 1024",
                   "parallelism": f"replicas x{world} (independent units, no collective)",
                   "l2": "flushed before every timed launch, outside the events (256 MiB write, then a 256 MiB read of "
                              "another buffer so the write-back happens before the launch)",
                   "timing": "CUDA events around each launch on the launching stream; mean over steps; max over ranks"},
        "roofline": {"bound": "tensor", "achieved": round(per_launch_tflops, 2), "peak": tc_peak, "unit": "TFLOP/s",
                     "frac": round(per_launch_tflops / tc_peak, 4),
                     "peak_kind": ("measured burst" if burst else "measured sustained") + f" ({peaks['source']})",
                     "frac_of_spec_2250": round(per_launch_tflops / SPEC_BF16_TFLOPS, 4),
                     "traffic": ncu_traffic("fa_fwd/gqa_causal_8k"),
                     "kernel": "fa_fwd_kernel<128,false>", "algorithmic_flops_per_launch": F,
                     "algorithmic_bytes_per_launch": fwd_bytes()},
        "decode": {"value": round(gbs, 1), "unit": "GB/s", "ms": round(dec_mean, 4),
                   "roofline": {"bound": "hbm", "achieved": round(per_launch_gbs, 1), "peak": peaks["hbm"],
                                "unit": "GB/s", "frac": round(per_launch_gbs / peaks["hbm"], 4),
                                "peak_kind": f"measured copy ({peaks['source']})",
                                "frac_of_spec_8000": round(per_launch_gbs / SPEC_HBM_GBS, 4),
                                "traffic": ncu_traffic("fa_decode/decode_split_kv"),
                                "kernels": "fa_decode_split_kernel<128> + fa_decode_combine_kernel<128>",
                                "algorithmic_bytes_per_launch": kv,
                                "tflops": round(dec_flops() / (dec_mean * 1e-3) / 1e12, 2)},
                   "e2e": {"value": round(world * kv / (dec_e2e_ms * 1e-3) / 1e9, 1), "unit": "GB/s",
                           "h2d_bytes_per_step": h2d_dec, "d2h_bytes_per_step": d2h_dec},
                   "cpu_baseline": dec_cpu},
        "decode_paged": {"value": round(aggregate_rate(pkv, world, paged_mean) / 1e9, 1), "unit": "GB/s",
                         "ms": round(paged_mean, 4),
                         "workload": "decode_paged_ragged: B=16, lengths U{1..32768} (seed 1006), Hq=64, Hkv=8, "
                                     "d=128, 16-token pages in a shuffled pool, split 1024",
                         "roofline": {"bound": "hbm", "achieved": round(paged_gbs, 1), "peak": peaks["hbm"],
                                      "unit": "GB/s", "frac": round(paged_gbs / peaks["hbm"], 4),
                                      "peak_kind": f"measured copy ({peaks['source']})",
                                      "traffic": ncu_traffic("fa_decode_paged/decode_paged_ragged"),
                                      "kernels": "fa_decode_split_kernel<128,paged> + fa_decode_combine_kernel<128>",
                                      "algorithmic_bytes_per_launch": pkv}},
        "forward_fp8": {"value": round(aggregate_rate(F, world, fp8_mean) / 1e12, 2), "unit": "TFLOP/s",
                        "ms": round(fp8_mean, 4),
                        "workload": "gqa_causal_8k with e4m3 q, k, v (per-tensor scales), P in e4m3, O bf16",
                        "roofline": {"bound": "tensor", "achieved": round(fp8_tflops, 2), "peak": round(fp8_peak, 1),
                                     "unit": "TFLOP/s", "frac": round(fp8_tflops / fp8_peak, 4),
                                     "peak_kind": f"measured bf16 x 2 (nominal fp8/bf16 ratio; {peaks['source']})",
                                     "traffic": ncu_traffic("fa_fwd_fp8/gqa_causal_8k"),
                                     "kernels": "transpose_v_e4m3_kernel + fa_fwd_kernel<128,false,fp8>",
                                     "algorithmic_flops_per_launch": F}},
        "forward_tf32": {"value": round(aggregate_rate(F2k, world, tf32_mean) / 1e12, 2), "unit": "TFLOP/s",
                         "ms": round(tf32_mean, 4),
                         "workload": "mha_causal_2k (B=2, H=12, N=2048, d=64, causal) with fp32 q, k, v on the tf32 path",
                         "roofline": {"bound": "tensor", "achieved": round(tf32_tflops, 2), "peak": round(tf32_peak, 1),
                                      "unit": "TFLOP/s", "frac": round(tf32_tflops / tf32_peak, 4),
                                      "peak_kind": f"measured bf16 x 1100/2250 (nominal tf32/bf16 ratio; {peaks['source']})",
                                      "kernels": "round_tf32_kernel x2 + transpose_v_f32_kernel + fa_fwd_kernel<64,true,tf32>",
                                      "algorithmic_flops_per_launch": F2k}},
        "backward": {"value": round(aggregate_rate(bwd_flops, world, bwd_mean) / 1e12, 2), "unit": "TFLOP/s",
                     "ms": round(bwd_mean, 4),
                     "workload": "gqa_causal_8k backward (dQ, dK, dV from the forward's O and lse; dO seeded N(0,1))",
                     "flops_convention": "2.5 x forward FLOPs (five products of the forward's two sizes)",
                     "roofline": {"bound": "tensor", "achieved": round(bwd_tflops, 2), "peak": bwd_peak,
                                  "unit": "TFLOP/s", "frac": round(bwd_tflops / bwd_peak, 4),
                                  "peak_kind": f"measured ({peaks['source']})",
                                  "traffic": ncu_traffic("fa_bwd/gqa_causal_8k"),
                                  "kernels": "fa_bwd_pre_kernel<128> + fa_bwd2_kernel + fa_bwd_dq_kernel<128>",
                                  "algorithmic_flops_per_launch": bwd_flops}},
        "e2e": {"value": round(world * F / (fwd_e2e_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d_fwd, "d2h_bytes_per_step": d2h_fwd},
        "cpu_baseline": cpu,
        "gpu_launches": args.steps * (int(do_fwd) * 1 + int(do_dec) * 2 + int(do_paged) * 2 + int(do_bwd) * 3 + int(do_fp8) * 2 + int(do_tf32) * 4
                                     + int(do_bwdv) * 4 + int(do_mha2k) + int(do_varlen))
        + (0 if args.no_e2e else e2e_steps * (int(do_fwd) * 1 + int(do_dec) * 2)),
        "clocks": clocks.summary(),
        "impl": "b200",
    }
    if do_mha2k:
        mF = fwd_flops(MHA2K)
        m_tflops = mF / (mha2k_mean * 1e-3) / 1e12
        m_peak = peaks["bf16"] if (args.steps * mha2k_mean) < 1000.0 else peaks["bf16_sustained"]
        line["forward_mha2k"] = {
            "value": round(aggregate_rate(mF, world, mha2k_mean) / 1e12, 2), "unit": "TFLOP/s",
            "ms": round(mha2k_mean, 4),
            "workload": "mha_causal_2k: B=2, H=12, N=2048, d=64, causal, bf16, layout [B,N,H,d] "
                        "(latency-sized: 384 query tiles for 148 SMs; reported, no target)",
            "roofline": {"bound": "tensor", "achieved": round(m_tflops, 2), "peak": m_peak, "unit": "TFLOP/s",
                         "frac": round(m_tflops / m_peak, 4), "peak_kind": f"measured ({peaks['source']})",
                         "frac_of_spec_2250": round(m_tflops / SPEC_BF16_TFLOPS, 4),
                         "traffic": ncu_traffic("fa_fwd/mha_causal_2k"),
                         "kernel": "fa_fwd_kernel<64,false>", "algorithmic_flops_per_launch": mF,
                         "algorithmic_bytes_per_launch": fwd_bytes(MHA2K)}}
    if do_varlen:
        fF = varlen_flops(f_len)
        fbytes = float(fT) * (2.0 * 2 * fHq * fd + 2.0 * 2 * fHkv * fd + 4.0 * fHq)
        f_tflops = fF / (varlen_mean * 1e-3) / 1e12
        f_peak = peaks["bf16"] if (args.steps * varlen_mean) < 1000.0 else peaks["bf16_sustained"]
        line["forward_varlen"] = {
            "value": round(aggregate_rate(fF, world, varlen_mean) / 1e12, 2), "unit": "TFLOP/s",
            "ms": round(varlen_mean, 4),
            "workload": f"varlen_gqa_causal: {fB} packed sequences, lengths U[256, 8192] (seed {VARLEN['seed']}), "
                        f"{fT} rows, Hq=32, Hkv=8, d=128, causal within each sequence",
            "flops_convention": "sum over sequences of 4 Hq L^2 d / 2",
            "roofline": {"bound": "tensor", "achieved": round(f_tflops, 2), "peak": f_peak, "unit": "TFLOP/s",
                         "frac": round(f_tflops / f_peak, 4), "peak_kind": f"measured ({peaks['source']})",
                         "frac_of_spec_2250": round(f_tflops / SPEC_BF16_TFLOPS, 4),
                         "traffic": ncu_traffic("fa_fwd/varlen_gqa_causal"),
                         "kernel": "fa_fwd_kernel<128,false> (varlen schedule)",
                         "algorithmic_flops_per_launch": fF, "algorithmic_bytes_per_launch": fbytes}}
    if do_bwdv:
        vF = 2.5 * varlen_flops(v_len)
        v_tflops = vF / (bwdv_mean * 1e-3) / 1e12
        v_peak = peaks["bf16"] if (args.steps * bwdv_mean) < 1000.0 else peaks["bf16_sustained"]
        line["backward_varlen"] = {
            "value": round(aggregate_rate(vF, world, bwdv_mean) / 1e12, 2), "unit": "TFLOP/s",
            "ms": round(bwdv_mean, 4),
            "workload": "varlen_gqa_causal backward: 16 packed sequences, lengths U[256, 8192] (seed 1004), "
                        "Hq=32, Hkv=8, d=128, causal",
            "flops_convention": "2.5 x the sequences' causal forward FLOPs",
            "roofline": {"bound": "tensor", "achieved": round(v_tflops, 2), "peak": v_peak, "unit": "TFLOP/s",
                         "frac": round(v_tflops / v_peak, 4), "peak_kind": f"measured ({peaks['source']})",
                         "kernels": "fa_bwd_tiles_kernel + fa_bwd_pre_kernel<128> + fa_bwd2_kernel + "
                                    "fa_bwd_dq_kernel<128>",
                         "algorithmic_flops_per_launch": vF}}
    print(json.dumps(_nan_to_null(line)), flush=True)


def _nan_to_null(x):
    """Phases left out with --only have no number: report null rather than NaN (not JSON)."""
    if isinstance(x, float) and math.isnan(x):
        return None
    if isinstance(x, dict):
        return {k: _nan_to_null(v) for k, v in x.items()}
    if isinstance(x, list):
        return [_nan_to_null(v) for v in x]
    return x


# ----------------------------------------------------------------------------- CPU oracle
_INPUTS = {}


def inputs(key, seed, tid, shape):
    """Seeded host inputs (float32 holding bf16 values), generated once per process."""
    k = (key, seed, tid, tuple(shape))
    if k not in _INPUTS:
        _INPUTS[k] = si.normal(seed, tid, shape)
    return _INPUTS[k]


def _oracle_rows_fwd(orc, rows_target, threads, seed):
    """Time the oracle on `rows_target` random rows of the forward workload."""
    w = FWD
    B, N, Hq, Hkv, d = w["B"], w["N"], w["Hq"], w["Hkv"], w["d"]
    q = inputs("fwd", seed, si.Q, (B, N, Hq, d))
    k = inputs("fwd", seed, si.K, (B, N, Hkv, d))
    v = inputs("fwd", seed, si.V, (B, N, Hkv, d))
    u = si.uniform_ints(seed, 13, 2 * rows_target, 0, (1 << 30))
    rows = np.stack([np.zeros(rows_target, np.int64), u[0::2] % Hq, u[1::2] % N], 1)
    t = time.perf_counter()
    orc.attention_rows(q, k, v, 1.0 / math.sqrt(d), rows, causal=True, nthreads=threads)
    dt = time.perf_counter() - t
    flops = float(np.sum(4.0 * (rows[:, 2] + 1) * d))
    return dt, flops, rows_target


def cpu_baseline_fwd(seconds: float):
    import oracle
    orc = oracle.get()
    threads = orc.hardware_threads()
    dt, fl, n = _oracle_rows_fwd(orc, 256, threads, FWD["seed"])
    target = max(256, int(n * seconds / max(dt, 1e-3)))
    dt, fl, n = _oracle_rows_fwd(orc, target, threads, FWD["seed"])
    return {"value": round(fl / dt / 1e12, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"{n} random causal rows of the gqa_causal_8k workload (fp64, materialised rows), "
                      f"{dt:.1f} s on {threads} threads"}


def _oracle_dec(orc, pairs, threads, seed):
    w = DEC
    B, Hq, Hkv, L, d = w["B"], w["Hq"], w["Hkv"], w["L"], w["d"]
    G = Hq // Hkv
    # the first `pairs` (sequence, kv-head) groups: each group's G query heads read its K/V once
    q = inputs("dec", seed, si.Q, (B, Hq, d))
    kc = inputs("dec", seed, si.KCACHE, (B, L, Hkv, d))
    vc = inputs("dec", seed, si.VCACHE, (B, L, Hkv, d))
    rows = []
    for p in range(pairs):
        b, g = p // Hkv, p % Hkv
        rows += [(b, g * G + j, 0) for j in range(G)]
    rows = np.array(rows, np.int64)
    t = time.perf_counter()
    orc.attention_rows(q.reshape(B, 1, Hq, d), kc, vc, 1.0 / math.sqrt(d), rows, causal=False,
                       kv_lens=np.full(B, L, np.int32), nthreads=threads)
    dt = time.perf_counter() - t
    return dt, pairs * L * d * 2 * 2


def cpu_baseline_dec(seconds: float):
    import oracle
    orc = oracle.get()
    threads = orc.hardware_threads()
    dt, by = _oracle_dec(orc, 1, threads, DEC["seed"])
    pairs = int(min(DEC["B"] * DEC["Hkv"], max(1, seconds / max(dt, 1e-3))))
    dt, by = _oracle_dec(orc, pairs, threads, DEC["seed"])
    return {"value": round(by / dt / 1e9, 3), "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"{pairs} of 64 (sequence, kv-head) groups of the decode workload, all 8 query heads each, "
                      f"{dt:.1f} s on {threads} threads"}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    orc = oracle.get()
    threads = orc.hardware_threads()
    per_step = max(0.5, args.cpu_seconds / max(1, args.steps))
    dt0, _, n0 = _oracle_rows_fwd(orc, 64, threads, FWD["seed"])
    rows = max(64, int(n0 * per_step / max(dt0, 1e-3)))
    for _ in range(args.warmup):
        _oracle_rows_fwd(orc, rows, threads, FWD["seed"])
    tot_t, tot_f = 0.0, 0.0
    for _ in range(args.steps):
        dt, fl, _ = _oracle_rows_fwd(orc, rows, threads, FWD["seed"])
        tot_t += dt
        tot_f += fl
    val = tot_f / tot_t / 1e12
    line = {
        "metric": METRIC, "value": round(val, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(1e3 * tot_t / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "gqa_causal_8k: B=1, Hq=64, Hkv=8, N=8192, d=128, causal, layout [B,N,H,d]"},
        "impl": "reference",
        "cpu_baseline": {"value": round(val, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": f"{rows} random causal rows per step (fp64 oracle, materialised rows)"},
        "e2e": {"value": round(val, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(_nan_to_null(line)), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end phases")
    ap.add_argument("--only", default="all", choices=["all", "fwd", "dec", "paged", "bwd", "fp8", "tf32", "bwd_varlen",
                                                       "mha2k", "varlen"],
                    help="profiling: run one kernel family")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_device(args)


if __name__ == "__main__":
    main()
