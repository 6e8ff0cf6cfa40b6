// Forward attention kernel for sm_100a.
//
// The method ("FlashAttention notes", sections 3-4; "LLM basics: from Attention to
// FlashAttention", chapter 3 sections 2 and 5): a tile of query rows stays on chip while
// tiles of K and V stream past it; for each K/V tile the scores S = Q K^T are formed on
// chip, the running row max m and row sum l are updated with
//   m_new = max(m_old, rowmax(S)),  l_new = e^(m_old - m_new) l_old + sum_j e^(s_j - m_new),
// the output accumulator is rescaled by the same factor and P V is added to it.  Only O
// and the per-row logsumexp are written to device memory.
//
// B200 mapping (one persistent CTA per SM, 384 threads):
//   warps 0-3   softmax for query tile 0 (thread = row), then its epilogue (O / l; bf16 O
//               goes out through shared memory by TMA stores)
//   warps 4-7   the same for query tile 1
//   warp  8     tcgen05.mma issuer and TMEM owner
//   warp  9     TMA producer
//   warps 10-11 idle (they complete the control warpgroup for the register split)
// The issuing warps run converged and let one elected lane issue each group of instructions.
// A work unit is two 128-row query tiles that share their K/V tiles: 256 rows of one
// (sequence, query head), or (hpair) 128 rows of two query heads of one K/V group, which see
// exactly the same keys, so no causal step runs with one tile.  Units are ordered
// longest-first (causal cost grows with the query tile index) and dealt to CTAs in a snake
// order.  K and V tiles (128 keys each) flow through a shared-memory ring
// of full/empty mbarriers.  TMEM (512 columns): S0 | S1 (128 fp32 columns each, P is
// written back over the first 64 columns of its S as packed bf16) | O0 | O1 (d columns).
// The MMA order S0(j+1) after O0 += P0(j) V(j) and S1(j+1) after O1 += P1(j) V(j) lets the
// tensor core work on one tile while the softmax warps work on the other.
//
// Scores are handled in base 2: t = s * scale * log2(e), p = 2^(t - m).  The output is
// rescaled lazily: the reference max m only moves when the tile max exceeds it by more than
// 8 (a factor 256), which is exact because O and l always share the same reference
// ("LLM basics", chapter 3 section 1: subtracting any constant leaves softmax unchanged).
// Once a row has a reference, its exponentials start right after the scores are loaded and
// the tile max, formed alongside, only confirms before publishing that no row moved past
// the threshold (else the tile is redone against the new max), so the max is off the
// critical path S(j) -> P(j) -> O += P V -> S(j+1) of each tile.
#pragma once

#include "fa_device.cuh"

namespace fa {

struct FwdParams {
  void* o;
  float* lse;
  const int32_t* cu;  // varlen offsets [B+1] or null
  int B, Hq, Hkv, G, Nq, Nk;
  int causal;
  float tau;      // scale * log2(e) (fp8: times the q and k dequantisation factors)
  float o_scale;  // multiplies O at the end (fp8: the v dequantisation factor; else 1)
  int T;          // fixed length: 256-row units per (sequence, head)
  int o_tma;      // bf16 O written through shared memory by TMA stores (tmO describes o)
  int hpair;      // 1: a unit is 128 rows of two query heads of one K/V group (else 256 rows of one)
};

constexpr int kBM = 128;        // query rows per tile
constexpr int kBN = 128;        // keys per K/V tile
constexpr int kUnitRows = 256;  // two query tiles per work unit (128 rows x 2 heads with hpair)
constexpr int kFwdThreads = 384;
// Register split by warpgroup, set with setmaxnreg after the common prologue.  The launch
// gives 384 threads x 168 registers = 64512; softmax warpgroups take 2 x 128 x 208 and the
// control warpgroup (MMA, TMA, two idle warps) 128 x 88, the same total (and the same per
// SM sub-partition: two softmax warps and one control warp each).  (A fourth warpgroup
// for the epilogue leaves the softmax 192 registers at most, which spills: measured slower.)
constexpr int kSoftmaxRegs = 208;
constexpr int kControlRegs = 88;
constexpr int kMaxVarlenB = 1024;
constexpr int kMaxVarlenT = 1024;
constexpr float kRescaleThreshold = 8.0f;
// P is published to the MMA warp in chunks of 64 keys (one mbarrier each, one arrival per
// softmax warp), so O += P V starts on the first chunk while the softmax still makes the
// second.  (Smaller chunks add a barrier wait per chunk to the MMA warp, which shares its
// SM sub-partition with two softmax warps; measured slower.)
constexpr int kPChunks = 2;
constexpr int kChunkKeys = kBN / kPChunks;
// FP8 only: column pairs (bit e of each group of 8 pairs) whose 2^x runs on the FMA pipe (a
// polynomial) instead of the special-function unit, in tiles without masked keys.  With its
// products halved, the fp8 forward is bound by the ex2 rate of the two tiles' softmax steps.
constexpr uint32_t kFp8FmaExpPairs = 0x11;


// Operand kinds of the forward: bf16 (kind::f16); FP8: q, k, v in e4m3 (d = 128 only), the
// S and P V products on the kind::f8f6f4 tensor-core path with P rounded to e4m3; TF32: fp32
// q, k, v (d = 64 only) on the kind::tf32 path with P kept in fp32 (read as tf32).  FP8 and
// TF32 read V from a [d, keys] transposed copy so that both operands of P V are K-major.
constexpr int kKindBF16 = 0, kKindFP8 = 1, kKindTF32 = 2;

template <int D, int KIND = kKindBF16>
struct FwdCfg {
  static constexpr int kElemBytes = KIND == kKindFP8 ? 1 : (KIND == kKindTF32 ? 4 : 2);
  static constexpr int kTileBytes = kBM * D * kElemBytes;  // one 128 x D tile
  static constexpr int kChunkBytes = kBM * 128;            // one 128-row x 128-byte swizzle panel
  static constexpr int kPanels = kTileBytes / kChunkBytes;
  static constexpr int kPanelCols = 128 / kElemBytes;      // elements per 128-byte panel row
  static constexpr int kVtPanelBytes = D * 128;            // V^T tile: D rows x 128 bytes of keys
  static constexpr int kStages = KIND == kKindTF32 ? 4 : ((KIND == kKindFP8 || D == 64) ? 8 : 4);
  static constexpr int kQBytes = 2 * kTileBytes;
  static constexpr int kRingBytes = kStages * kTileBytes;
  // Epilogue staging: per softmax warp two 1 KB boxes of 32 rows x 16 bf16 columns (32-byte
  // swizzle), each stored to O by TMA while the warp fills the other.
  static constexpr int kStageBoxBytes = 32 * 32;
  static constexpr int kStageBytes = 8 * 2 * kStageBoxBytes;
  static constexpr int kNumBars = 2 + 2 * kStages + 6 + 2 * kPChunks;
  static constexpr int kBarBytes = kNumBars * 8 + 16;
  static constexpr int kSchedBytes = kMaxVarlenB * 2 + kMaxVarlenT * 4 + 16;
  static constexpr int kSmemBytes = 1024 + kQBytes + kRingBytes + kStageBytes + kBarBytes + kSchedBytes;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColO = 256;
};

// Geometry of one work unit as every role sees it.
struct Unit {
  int b, h, kvh;         // h: query head of tile 0
  int rstep, hstep;      // tile 1 = tile 0 moved by rstep rows and hstep heads
  int q_start, k_start;  // first row of the sequence in q/o and in k/v
  int nq, nk;
  int row0;   // first query row of the unit within the sequence
  int n[2];   // K/V tiles each query tile attends to (0: tile empty or sees no key)
  int valid[2];
  int nmax;
};

struct SchedShared {
  int T;          // number of levels (query-tile indices)
  int U;          // total units
  uint16_t* sigma;  // varlen: sequences sorted by tile count, descending
  int* cnt;         // varlen: cnt[t] = number of sequences with more than t unit rows-tiles
};

// Walks the units of one CTA in increasing order.
struct UnitWalker {
  int level = 0;
  int level_start = 0;
};

__device__ __forceinline__ int kv_tiles_for(int last_row, int nq, int nk, int causal) {
  int kv_end = nk;
  if (causal) kv_end = min(nk, last_row + (nk - nq) + 1);
  if (kv_end <= 0) return 0;
  return (kv_end + kBN - 1) / kBN;
}

__device__ __forceinline__ void decode_unit(const FwdParams& p, const SchedShared& s, UnitWalker& w, int u,
                                            Unit& out) {
  int b, t, h;
  const int hp = p.hpair;
  const int hunits = p.Hq >> hp;  // units per (sequence, level)
  if (p.cu == nullptr) {
    const int per_level = p.B * hunits;
    const int level = u / per_level;
    const int off = u - level * per_level;
    b = off / hunits;
    h = (off - b * hunits) << hp;
    t = s.T - 1 - level;
    out.q_start = b * p.Nq;
    out.k_start = b * p.Nk;
    out.nq = p.Nq;
    out.nk = p.Nk;
  } else {
    for (;;) {
      const int sz = s.cnt[s.T - 1 - w.level] * hunits;
      if (u < w.level_start + sz) break;
      w.level_start += sz;
      ++w.level;
    }
    const int off = u - w.level_start;
    const int r = off / hunits;
    h = (off - r * hunits) << hp;
    b = s.sigma[r];
    t = s.T - 1 - w.level;
    const int c0 = __ldg(p.cu + b), c1 = __ldg(p.cu + b + 1);
    out.q_start = c0;
    out.k_start = c0;
    out.nq = c1 - c0;
    out.nk = c1 - c0;
  }
  out.b = b;
  out.h = h;
  out.kvh = h / p.G;
  out.row0 = t * (kUnitRows >> hp);
  out.rstep = hp ? 0 : kBM;
  out.hstep = hp;
  for (int i = 0; i < 2; ++i) {
    const int r0 = out.row0 + i * out.rstep;
    out.valid[i] = r0 < out.nq;
    out.n[i] = out.valid[i] ? kv_tiles_for(min(r0 + kBM - 1, out.nq - 1), out.nq, out.nk, p.causal) : 0;
  }
  out.nmax = max(out.n[0], out.n[1]);
}

// The u-th unit handled by CTA c (snake order over rounds of gridDim.x units); -1 when done.
struct UnitIter {
  int round = 0;
  __device__ __forceinline__ int next(int U) {
    const int G = gridDim.x, c = blockIdx.x;
    for (;;) {
      if (round * G >= U) return -1;
      const int u = round * G + ((round & 1) ? (G - 1 - c) : c);
      ++round;
      if (u < U) return u;
    }
  }
};

// Maximum of 128 scores: 16 independent chains of three-input max, then a three-level tree.
__device__ __forceinline__ float row_max128(const float (&s)[128]) {
  float mx[16];
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    mx[q] = fmax3(s[q], s[q + 16], s[q + 32]);
    mx[q] = fmax3(mx[q], s[q + 48], s[q + 64]);
    mx[q] = fmax3(mx[q], s[q + 80], s[q + 96]);
    mx[q] = fmaxf(mx[q], s[q + 112]);
  }
  float my[6];
#pragma unroll
  for (int q = 0; q < 5; ++q) my[q] = fmax3(mx[3 * q], mx[3 * q + 1], mx[3 * q + 2]);
  my[5] = mx[15];
  return fmaxf(fmax3(my[0], my[1], my[2]), fmax3(my[3], my[4], my[5]));
}

template <int D, bool OUT_F32, int KIND = kKindBF16>
__global__ void __launch_bounds__(kFwdThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                  const FwdParams p) {
  constexpr bool FP8 = KIND == kKindFP8, TF32 = KIND == kKindTF32;
  static_assert(!FP8 || (D == 128 && !OUT_F32), "fp8 forward: d = 128, bf16 output");
  static_assert(!TF32 || (D == 64 && OUT_F32), "tf32 forward: d = 64, fp32 output");
  using C = FwdCfg<D, KIND>;
  constexpr int NS = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sRing = smem + C::kQBytes;
  uint8_t* sStage = sRing + C::kRingBytes;  // 1024-byte aligned (Q and ring are multiples of 1 KB)
  uint64_t* bars = reinterpret_cast<uint64_t*>(sStage + C::kStageBytes);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* full = bars + 2;
  uint64_t* empty = bars + 2 + NS;
  uint64_t* s_full = bars + 2 + 2 * NS;   // [tile]
  uint64_t* p_chunk = s_full + 2;         // [tile][chunk]: P of keys 32c .. 32c+31 written
  uint64_t* pv_done = p_chunk + 2 * kPChunks;  // [tile]
  uint64_t* o_free = pv_done + 2;         // [tile]: O read out by the epilogue
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  int* sched_misc = reinterpret_cast<int*>(tmem_slot + 2);  // [0] = T, [1] = total tiles
  uint8_t* sched_mem = reinterpret_cast<uint8_t*>(bars) + C::kBarBytes;
  uint16_t* sigma = reinterpret_cast<uint16_t*>(sched_mem);
  int* cnt = reinterpret_cast<int*>(sched_mem + kMaxVarlenB * 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full + i, 1);
      for (int c = 0; c < kPChunks; ++c) mbar_init(p_chunk + kPChunks * i + c, kBM / 32);  // one per warp
      mbar_init(pv_done + i, 1);
      mbar_init(o_free + i, kBM / 32);  // one per softmax warp
    }
    sched_misc[0] = 0;
    sched_misc[1] = 0;
    fence_barrier_init();
  }
  if (warp == 9 && lane == 0) {
    prefetch_tensormap(&tmQ);
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
  }
  if (!OUT_F32 && p.o_tma && warp == 0 && lane == 0) prefetch_tensormap(&tmO);
  if (warp == 8) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }

  // ---- schedule: fixed length is arithmetic; varlen sorts sequences by tile count
  SchedShared sch;
  sch.sigma = sigma;
  sch.cnt = cnt;
  if (p.cu == nullptr) {
    sch.T = p.T;
    sch.U = p.T * p.B * (p.Hq >> p.hpair);
    __syncthreads();
  } else {
    __syncthreads();  // sched_misc initialised
    // cu_seqlens must start at or above 0, never decrease and end at or below the packed row
    // count; otherwise no unit is scheduled (nothing is read or written) and the error word
    // records it for fa_last_device_error.
    int bad = 0;
    for (int b = threadIdx.x; b < p.B; b += blockDim.x) {
      const int c0 = __ldg(p.cu + b), c1 = __ldg(p.cu + b + 1);
      bad |= (c1 < c0) | (b == 0 && c0 < 0) | (b == p.B - 1 && c1 > p.Nq);
      const int len = c1 - c0;
      const int ur = kUnitRows >> p.hpair;
      const int nt = len > 0 ? (len + ur - 1) / ur : 0;
      atomicMax(&sched_misc[0], nt);
      atomicAdd(&sched_misc[1], nt);
    }
    if (__syncthreads_or(bad)) {
      if (threadIdx.x == 0) atomicOr(&g_error_word, kErrBadSeqlens);
      sched_misc[1] = 0;  // (every thread writes the same value)
    }
    __syncthreads();
    const int T = min(sched_misc[0], kMaxVarlenT);
    for (int b = threadIdx.x; b < p.B; b += blockDim.x) {
      const int lb = __ldg(p.cu + b + 1) - __ldg(p.cu + b);
      const int ur = kUnitRows >> p.hpair;
      const int nb = lb > 0 ? (lb + ur - 1) / ur : 0;
      int rank = 0;
      for (int b2 = 0; b2 < p.B; ++b2) {
        const int l2 = __ldg(p.cu + b2 + 1) - __ldg(p.cu + b2);
        const int n2 = l2 > 0 ? (l2 + ur - 1) / ur : 0;
        rank += (n2 > nb) || (n2 == nb && b2 < b);
      }
      sigma[rank] = (uint16_t)b;
    }
    for (int t = threadIdx.x; t < T; t += blockDim.x) {
      int c = 0;
      for (int b2 = 0; b2 < p.B; ++b2) {
        const int l2 = __ldg(p.cu + b2 + 1) - __ldg(p.cu + b2);
        const int n2 = l2 > 0 ? (l2 + (kUnitRows >> p.hpair) - 1) / (kUnitRows >> p.hpair) : 0;
        c += n2 > t;
      }
      cnt[t] = c;
    }
    __syncthreads();
    sch.T = T;
    sch.U = sched_misc[1] * (p.Hq >> p.hpair);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kControlRegs));
  if (warp == 9) {
    // ================================================================ TMA producer
    {
      const uint64_t kv_policy = policy_evict_last();
      uint32_t g = 0, qcount = 0;
      UnitIter it;
      UnitWalker wk;
      bool ok = true;
      for (int u = it.next(sch.U); u >= 0 && ok; u = it.next(sch.U)) {
        Unit un;
        decode_unit(p, sch, wk, u, un);
        if (qcount > 0 && !warp_wait(q_empty, (qcount - 1) & 1)) break;
        const int ntile = un.valid[1] ? 2 : 1;
        mbar_arrive_expect_tx_elect(q_full, ntile * C::kTileBytes);
        for (int i = 0; i < ntile; ++i)
          for (int c = 0; c < C::kPanels; ++c)
            tma_load_3d_elect(sQ + i * C::kTileBytes + c * C::kChunkBytes, &tmQ, c * C::kPanelCols,
                              un.h + i * un.hstep, un.q_start + un.row0 + i * un.rstep, q_full);
        for (int j = 0; j < un.nmax && ok; ++j) {
          for (int kv = 0; kv < 2; ++kv) {
            const uint32_t slot = g % NS;
            if (g >= (uint32_t)NS && !warp_wait(empty + slot, ((g / NS) - 1) & 1)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx_elect(full + slot, C::kTileBytes);
            if ((FP8 || TF32) && kv) {
              // V^T tile: d rows of 128 keys from the [B * Hkv, d, keys] transposed copy, in
              // 128-byte panels of keys (one for e4m3, four for fp32)
              for (int c = 0; c < C::kTileBytes / C::kVtPanelBytes; ++c)
                tma_load_3d_hint_elect(sRing + slot * C::kTileBytes + c * C::kVtPanelBytes, &tmV,
                                       j * kBN + c * C::kPanelCols, 0, un.b * p.Hkv + un.kvh, full + slot,
                                       kv_policy);
            } else {
              for (int c = 0; c < C::kPanels; ++c)
                tma_load_3d_hint_elect(sRing + slot * C::kTileBytes + c * C::kChunkBytes, kv ? &tmV : &tmK,
                                       c * C::kPanelCols, un.kvh, un.k_start + j * kBN, full + slot, kv_policy);
            }
            ++g;
          }
        }
        ++qcount;
      }
    }
    __syncwarp();
  } else if (warp == 8) {
    // ================================================================ MMA issuer
    {
      constexpr uint32_t idS = FP8 ? idesc_e4m3_f32(kBM, kBN)
                                   : (TF32 ? idesc_tf32_f32(kBM, kBN) : idesc_bf16_f32(kBM, kBN, false));
      constexpr uint32_t idPV = FP8 ? idesc_e4m3_f32(kBM, D) : (TF32 ? idesc_tf32_f32(kBM, D) : idesc_bf16_f32(kBM, D, true));
      const uint32_t qbase = smem_u32(sQ);
      const uint32_t rbase = smem_u32(sRing);
      uint32_t g = 0, qcount = 0;
      uint32_t pcnt[2] = {0, 0}, ounits[2] = {0, 0};
      UnitIter it;
      UnitWalker wk;
      bool ok = true;

      // Shared-memory descriptors are built once; a k-step or a ring slot only moves the
      // start address (the low 14 bits, in 16-byte units, never carry: shared addresses are
      // below 2^18 bytes).  The MMAs of one group are issued by one elected lane.
      const uint64_t dQ = smem_desc_sw128(qbase, 16, 1024);  // K-major, 128-byte swizzle
      const uint64_t dR = smem_desc_sw128(rbase, 16, 1024);  // ring slots read K-major (K, V^T)
      const uint64_t dV = smem_desc_sw128(rbase, C::kChunkBytes, 1024);  // bf16 V read MN-major
      auto slot_off = [](uint32_t slot) -> uint64_t { return (uint64_t)((slot * C::kTileBytes) >> 4); };
      // S_i = Q_i K^T: k-steps of 32 bytes along d (16 bf16, 32 e4m3 or 8 tf32 elements),
      // four per 128-byte panel; then commit to the tile's s_full barrier.
      auto issue_S = [&](int i, uint32_t slot) {
        const uint64_t a0 = dQ + (uint64_t)((i * C::kTileBytes) >> 4), b0 = dR + slot_off(slot);
        if (elect_one_lane()) {
#pragma unroll
          for (int kk = 0; kk < D * C::kElemBytes / 32; ++kk) {
            const uint32_t off = ((kk >> 2) * C::kChunkBytes + (kk & 3) * 32) >> 4;
            mma_ss<KIND>(tmem + i * kBN, a0 + off, b0 + off, idS, kk > 0 ? 1u : 0u);
          }
          umma_commit(s_full + i);
        }
        __syncwarp();
      };
      // O_i (+)= P_i V for the 32 keys of chunk c.  P sits in the S columns of its tile:
      // bf16 two keys per column (k-steps of 16 keys = 8 columns), e4m3 four keys per column
      // (one k-step of 32 keys = 8 columns), fp32 one key per column (k-steps of 8 keys).
      auto issue_PV_chunk = [&](int i, uint32_t slot, int c, bool acc) {
        const uint32_t dO = tmem + C::kColO + i * D, aP = tmem + i * kBN;
        if (elect_one_lane()) {
          if constexpr (TF32) {
            const uint64_t b0 = dR + slot_off(slot);
#pragma unroll
            for (int k8 = 0; k8 < kChunkKeys / 8; ++k8) {
              const int kk = c * (kChunkKeys / 8) + k8;  // 8 keys = 32 bytes of each V^T row
              const uint32_t off = ((kk >> 2) * C::kVtPanelBytes + (kk & 3) * 32) >> 4;
              mma_ts<KIND>(dO, aP + kk * 8, b0 + off, idPV, (acc || kk > 0) ? 1u : 0u);
            }
          } else if constexpr (FP8) {
            const uint64_t b0 = dR + slot_off(slot);
#pragma unroll
            for (int k32 = 0; k32 < kChunkKeys / 32; ++k32) {
              const int kk = c * (kChunkKeys / 32) + k32;  // 32 keys = 32 bytes of each V^T row
              mma_ts<KIND>(dO, aP + kk * 8, b0 + (uint32_t)((kk * 32) >> 4), idPV, (acc || kk > 0) ? 1u : 0u);
            }
          } else {
            const uint64_t b0 = dV + slot_off(slot);
#pragma unroll
            for (int k2 = 0; k2 < kChunkKeys / 16; ++k2) {
              const int kk = c * (kChunkKeys / 16) + k2;  // 16 keys = 16 rows of 128 bytes
              mma_ts<KIND>(dO, aP + kk * 8, b0 + (uint32_t)((kk * 16 * 128) >> 4), idPV, (acc || kk > 0) ? 1u : 0u);
            }
          }
        }
        __syncwarp();
      };
      auto wait_full = [&](uint32_t gi) -> bool {
        if (!warp_wait(full + (gi % NS), (gi / NS) & 1)) return false;
        tc_fence_after();
        return true;
      };
      auto pv_step = [&](int i, int j, uint32_t vslot) -> bool {
        if (j == 0 && ounits[i] > 0 && !warp_wait(o_free + i, (ounits[i] - 1) & 1)) return false;
        // each chunk of P is consumed while the softmax still writes the next
        for (int c = 0; c < kPChunks; ++c) {
          if (!warp_wait(p_chunk + kPChunks * i + c, pcnt[i] & 1)) return false;
          tc_fence_after();
          issue_PV_chunk(i, vslot, c, j > 0);
        }
        ++pcnt[i];
        umma_commit_elect(pv_done + i);
        return true;
      };

      for (int u = it.next(sch.U); u >= 0 && ok; u = it.next(sch.U)) {
        Unit un;
        decode_unit(p, sch, wk, u, un);
        if (!warp_wait(q_full, qcount & 1)) break;
        tc_fence_after();
        const int nmax = un.nmax;
        if (nmax == 0) {
          umma_commit_elect(q_empty);
          ++qcount;
          continue;
        }
        // prologue: S_i(0)
        if (!wait_full(g)) break;
        for (int i = 0; i < 2; ++i)
          if (un.n[i] > 0) issue_S(i, g % NS);
        umma_commit_elect(empty + (g % NS));
        if (nmax == 1) umma_commit_elect(q_empty);
        // per K/V tile j: O_0 += P_0(j) V(j), S_0(j+1), O_1 += P_1(j) V(j), S_1(j+1), so the
        // tensor core works on one tile while the softmax warps work on the other.  (One
        // issuing warp per tile lets the tensor core interleave both tiles' products, which
        // stretches both chains: measured slower.)
        for (int j = 0; j < nmax && ok; ++j) {
          const uint32_t gv = g + 2 * j + 1;
          const uint32_t gk = g + 2 * j + 2;
          // both K/V tiles of the step are waited for here, so no data wait sits between the
          // products of a tile (the producer runs ahead; these waits rarely block)
          if (!wait_full(gv)) { ok = false; break; }
          if (j + 1 < nmax && !wait_full(gk)) { ok = false; break; }
          if (j < un.n[0] && !pv_step(0, j, gv % NS)) { ok = false; break; }
          if (j + 1 < nmax && j + 1 < un.n[0]) issue_S(0, gk % NS);
          if (j < un.n[1] && !pv_step(1, j, gv % NS)) { ok = false; break; }
          umma_commit_elect(empty + (gv % NS));
          if (j + 1 < nmax) {
            if (j + 1 < un.n[1]) issue_S(1, gk % NS);
            umma_commit_elect(empty + (gk % NS));
            if (j + 2 == nmax) umma_commit_elect(q_empty);
          }
        }
        g += 2 * nmax;
        ++qcount;
        for (int i = 0; i < 2; ++i)
          if (un.n[i] > 0) ++ounits[i];
      }
    }
    __syncwarp();
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
    // ================================================================ softmax + epilogue
    const int i = warp >> 2;            // query tile of this warpgroup
    const int r = threadIdx.x & 127;    // row within the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + i * kBN;
    const uint32_t tO = tmem + lane_off + C::kColO + i * D;
    const float tau = p.tau;
    uint32_t scnt = 0, pvcnt = 0;
    UnitIter it;
    UnitWalker wk;
    bool ok = true;

    for (int u = it.next(sch.U); u >= 0 && ok; u = it.next(sch.U)) {
      Unit un;
      decode_unit(p, sch, wk, u, un);
      const int my_valid = i ? un.valid[1] : un.valid[0];
      if (!my_valid) continue;
      const int n = i ? un.n[1] : un.n[0];
      const int row = un.row0 + i * un.rstep + r;                  // row within the sequence
      const int warp_row_min = un.row0 + i * un.rstep + (warp & 3) * 32;
      const int head = un.h + i * un.hstep;                        // query head of this tile
      const int diag = un.nk - un.nq;                              // causal offset
      float m_ref = -INFINITY, l = 0.f;

      // P of keys 32c .. 32c+31 from the scores s (exponent reference ms, as -ms in both halves
      // of nms2) into pk, with the row sum of the unrounded values added to lsum.
      constexpr int kW = FP8 ? kChunkKeys / 4 : (TF32 ? kChunkKeys : kChunkKeys / 2);  // TMEM words
      const uint64_t tau2 = f2(tau, tau);
      auto make_chunk = [&](const float (&sc)[128], int c, uint64_t nms2, uint32_t (&pk)[kW], uint64_t (&lsum)[2],
                            bool unmasked) {
#pragma unroll
        for (int e = 0; e < kChunkKeys / 2; ++e) {
          const int g = c * (kChunkKeys / 2) + e;  // column pair
          float x0, x1, p0, p1;
          f2_split(f2_fma(f2(sc[2 * g], sc[2 * g + 1]), tau2, nms2), x0, x1);
          if (FP8 && ((kFp8FmaExpPairs >> (g & 7)) & 1u) && unmasked) {
            exp2_poly_x2(x0, x1, p0, p1);
          } else {
            p0 = ex2_approx(x0);
            p1 = ex2_approx(x1);
          }
          lsum[e & 1] = f2_add(lsum[e & 1], f2(p0, p1));
          if (TF32) {
            pk[2 * e] = __float_as_uint(p0);
            pk[2 * e + 1] = __float_as_uint(p1);
          } else if (FP8) {
            // four keys per word: pairs e (even) and e + 1 share one
            if (e & 1) pk[e >> 1] |= pack_e4m3x2_hi(p0, p1);
            else pk[e >> 1] = pack_e4m3x2_lo(p0, p1);
          } else {
            pk[e] = pack_bf16x2(p0, p1);
          }
        }
      };
      // Writes chunk c of P over the S columns of its tile and tells the MMA warp (one arrival
      // per warp, after every lane's store has completed).
      auto publish = [&](int c, const uint32_t (&pk)[kW]) {
        const uint32_t col = (uint32_t)(c * kW);
        if constexpr (kW >= 32) {
#pragma unroll
          for (int w0 = 0; w0 < kW; w0 += 32)
            tmem_st32(tS + col + w0, reinterpret_cast<const uint32_t(&)[32]>(pk[w0]));
        } else if constexpr (kW == 16) {
          tmem_st16(tS + col, pk);
        } else {
          tmem_st8(tS + col, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_chunk + kPChunks * i + c);
      };

      for (int j = 0; j < n; ++j) {
        if (!mbar_wait(s_full + i, scnt & 1)) { ok = false; break; }
        ++scnt;
        tc_fence_after();
        uint32_t sv[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, sv[c]);
        tmem_wait_ld();
        float s[128];
#pragma unroll
        for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(sv[c >> 5][c & 31]);

        const int key0 = j * kBN;
        const bool need_mask = (key0 + kBN > un.nk) || (p.causal && key0 + kBN - 1 > warp_row_min + diag);
        uint64_t lsum[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
        float m_tile;
        bool have_max = false;
        // Speculative step: once every row of the warp has a finite reference max and no key
        // of this tile is masked, exponentiate against the reference at once.  The tile max,
        // computed alongside the first chunk's exponentials, then only has to confirm that no
        // row rose above the lazy threshold before anything is published; if one did, the
        // chunk is dropped and the full step below runs (the exact result is the same either
        // way: O and l always share the reference).
        if (!need_mask && __all_sync(0xffffffffu, m_ref != -INFINITY)) {
          m_tile = row_max128(s) * tau;
          const uint64_t nms2 = f2(-m_ref, -m_ref);
          uint32_t pk[kW];
          make_chunk(s, 0, nms2, pk, lsum, true);
          if (!__any_sync(0xffffffffu, m_tile - m_ref > kRescaleThreshold)) {
            publish(0, pk);
#pragma unroll
            for (int c = 1; c < kPChunks; ++c) {
              make_chunk(s, c, nms2, pk, lsum, true);
              publish(c, pk);
            }
            float la, lb, lc, ld;
            f2_split(lsum[0], la, lb);
            f2_split(lsum[1], lc, ld);
            l += (la + lb) + (lc + ld);
            continue;
          }
          lsum[0] = lsum[1] = f2(0.f, 0.f);
          have_max = true;
        }
        if (need_mask) {
          int lim = un.nk - key0;
          if (p.causal) lim = min(lim, row + diag + 1 - key0);
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= lim) s[c] = -INFINITY;
        }
        if (!have_max) m_tile = row_max128(s) * tau;
        const float m_new = fmaxf(m_ref, m_tile);
        const bool need = m_new - m_ref > kRescaleThreshold;  // false when both are -inf
        const bool warp_need = __any_sync(0xffffffffu, need);
        const float alpha = need ? ex2_approx(m_ref - m_new) : 1.f;
        if (need) m_ref = m_new;
        l *= alpha;
        if (warp_need && j > 0) {
          // O holds P V up to tile j-1 (complete: S(j) was committed after that product);
          // bring it to the new reference max before this tile's P is published.
          if (!mbar_wait(pv_done + i, (pvcnt + j - 1) & 1)) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int cc = 0; cc < D / 16; ++cc) {
            uint32_t ov[16];
            tmem_ld16(tO + 16 * cc, ov);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
            tmem_st16(tO + 16 * cc, ov);
          }
          tmem_wait_st();
        }
        // P = 2^(t - m_ref), chunk by chunk, each published as soon as it is written
        const float ms = (m_ref == -INFINITY) ? 0.f : m_ref;
        const uint64_t nms2 = f2(-ms, -ms);
#pragma unroll
        for (int c = 0; c < kPChunks; ++c) {
          uint32_t pk[kW];
          make_chunk(s, c, nms2, pk, lsum, !need_mask);
          publish(c, pk);
        }
        float la, lb, lc, ld;
        f2_split(lsum[0], la, lb);
        f2_split(lsum[1], lc, ld);
        l += (la + lb) + (lc + ld);
      }
      if (!ok) break;

      // ---- epilogue: O / l (times the output scale) -> HBM, lse = (m + log2 l) ln 2
      if (n > 0) {
        if (!mbar_wait(pv_done + i, (pvcnt + n - 1) & 1)) { ok = false; break; }
        tc_fence_after();
      }
      pvcnt += n;
      const bool row_ok = row < un.nq;
      const float inv_l = l > 0.f ? p.o_scale / l : 0.f;
      const size_t orow = ((size_t)(un.q_start + row) * p.Hq + head) * D;
      // A warp whose 32 rows all lie in the sequence writes O by TMA: its rows go to a 1 KB
      // box of shared memory 16 columns at a time (two boxes in turn, the 32-byte swizzle
      // keeps the row-per-lane writes free of bank conflicts) and one lane stores each box.
      // Per-lane global stores would put 32 rows' partial sectors into every instruction.
      const bool tma_o = !OUT_F32 && p.o_tma && __all_sync(0xffffffffu, row_ok);
      // One copy of the chunk code: the epilogue runs once per unit, its instructions cold in
      // the instruction cache, so a rolled loop fetches them once rather than D / 32 times.
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        if (n > 0) {
          tmem_ld32(tO + 32 * c, ov);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = 0u;
        }
        if (c == D / 32 - 1 && n > 0) {
          // every column of O is in registers: the next unit's products may overwrite it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(o_free + i);
        }
        if (tma_o) {
#pragma unroll
          for (int hb = 0; hb < 2; ++hb) {
            uint8_t* box = sStage + ((warp & 7) * 2 + hb) * C::kStageBoxBytes;
            if (lane == 0) bulk_wait_group_read1();  // this box's previous store has read it
            __syncwarp();
            uint4 w0, w1;
            const int e0 = 16 * hb;
            w0.x = pack_bf16x2(__uint_as_float(ov[e0 + 0]) * inv_l, __uint_as_float(ov[e0 + 1]) * inv_l);
            w0.y = pack_bf16x2(__uint_as_float(ov[e0 + 2]) * inv_l, __uint_as_float(ov[e0 + 3]) * inv_l);
            w0.z = pack_bf16x2(__uint_as_float(ov[e0 + 4]) * inv_l, __uint_as_float(ov[e0 + 5]) * inv_l);
            w0.w = pack_bf16x2(__uint_as_float(ov[e0 + 6]) * inv_l, __uint_as_float(ov[e0 + 7]) * inv_l);
            w1.x = pack_bf16x2(__uint_as_float(ov[e0 + 8]) * inv_l, __uint_as_float(ov[e0 + 9]) * inv_l);
            w1.y = pack_bf16x2(__uint_as_float(ov[e0 + 10]) * inv_l, __uint_as_float(ov[e0 + 11]) * inv_l);
            w1.z = pack_bf16x2(__uint_as_float(ov[e0 + 12]) * inv_l, __uint_as_float(ov[e0 + 13]) * inv_l);
            w1.w = pack_bf16x2(__uint_as_float(ov[e0 + 14]) * inv_l, __uint_as_float(ov[e0 + 15]) * inv_l);
            // row = lane, 32 bytes; 16-byte half h sits at h ^ bit 2 of the row (32-byte swizzle)
            const int sw = (lane >> 2) & 1;
            *reinterpret_cast<uint4*>(box + lane * 32 + (sw << 4)) = w0;
            *reinterpret_cast<uint4*>(box + lane * 32 + ((sw ^ 1) << 4)) = w1;
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_3d(&tmO, box, 32 * c + e0, head, un.q_start + row);
              bulk_commit_group();
            }
          }
        } else if (row_ok) {
          if (OUT_F32) {
            float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.o) + orow + 32 * c);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              dst[e] = make_float4(__uint_as_float(ov[4 * e]) * inv_l, __uint_as_float(ov[4 * e + 1]) * inv_l,
                                   __uint_as_float(ov[4 * e + 2]) * inv_l, __uint_as_float(ov[4 * e + 3]) * inv_l);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.o) + orow + 32 * c);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(ov[8 * e + 0]) * inv_l, __uint_as_float(ov[8 * e + 1]) * inv_l);
              w.y = pack_bf16x2(__uint_as_float(ov[8 * e + 2]) * inv_l, __uint_as_float(ov[8 * e + 3]) * inv_l);
              w.z = pack_bf16x2(__uint_as_float(ov[8 * e + 4]) * inv_l, __uint_as_float(ov[8 * e + 5]) * inv_l);
              w.w = pack_bf16x2(__uint_as_float(ov[8 * e + 6]) * inv_l, __uint_as_float(ov[8 * e + 7]) * inv_l);
              dst[e] = w;
            }
          }
        }
      }
      if (row_ok && p.lse != nullptr) {
        const float v = l > 0.f ? (m_ref + log2f(l)) * kLn2 : -INFINITY;
        const size_t li = (p.cu != nullptr) ? (size_t)head * p.Nq + un.q_start + row
                                             : ((size_t)un.b * p.Hq + head) * p.Nq + row;
        p.lse[li] = v;
      }
    }
    if (lane == 0) bulk_wait_group0();  // O boxes stored before the CTA's shared memory goes
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace fa
