// Backward attention kernels for sm_100a.
//
// The method ("FlashAttention notes", section 5.2, backward; "LLM basics: from Attention to
// FlashAttention", chapter 3 section 6): the N x N matrices are not kept from the forward.
// The backward rebuilds P tile by tile from Q, K and the saved per-row logsumexp,
//   P = exp(scale * Q K^T - lse),
// and forms the gradients with it on chip:
//   dV = P^T dO,  dP = dO V^T,  dS = P o (dP - D)  with  D_i = sum_c dO_ic O_ic,
//   dQ = scale * dS K,  dK = scale * dS^T Q.
// Only dQ, dK and dV (and two vectors per row) reach device memory.
//
// Three launches:
//   fa_bwd_pre_kernel   D_i and lse_i * log2(e) per query row (padded to whole tiles, with
//                       +inf where no key is allowed so that P = 0 there), and zeroes the
//                       fp32 dQ accumulator.
//   fa_bwd_kernel       one CTA per (128-key tile, K/V head, sequence): K and V stay in
//                       shared memory while (query head of the group, 128-query tile) pairs
//                       stream past; dK and dV accumulate in TMEM over all of them (the group
//                       sum of GQA included), dQ of each pair is added to the fp32 accumulator
//                       with vector reductions.
//   fa_bwd_dq_kernel    dQ = scale * accumulator, rounded to bf16.
//
// B200 mapping of fa_bwd_kernel (384 threads, one CTA per SM):
//   warp 0      TMA producer (K, V once; Q, dO and the row vectors per pair, double-buffered)
//   warp 1      tcgen05.mma issuer and TMEM owner
//   warps 2-3   idle
//   warps 4-11  two elementwise warpgroups; thread = key row = TMEM lane, warpgroup w takes
//               query columns 64w..64w+63 of each pair, then dQ columns of its half.
// Per pair, with the key tile as the M side (TMEM lanes = keys):
//   S^T = K Q^T -> TMEM[0,128)      dP^T = V dO^T -> TMEM[128,256)       (tcgen05, SS)
//   P^T = 2^(S^T tau - lse2), dS^T = P^T o (dP^T - D)                    (elementwise)
//   P^T (bf16) over TMEM[0,64), dS^T (bf16) over TMEM[128,192), dS^T also to shared memory
//   dV += P^T dO,  dK += dS^T Q               (tcgen05, A from TMEM; TMEM[256,256+2d))
//   dQ = dS K -> TMEM[64,128) and TMEM[192,256) (two 64-column halves; A = dS from shared
//   memory, query-major)
// Every operand tile is stored once (128 rows, 64-column panels, 128-byte swizzle) and read
// either K-major or MN-major through its descriptor.
#pragma once

#include "fa_device.cuh"

namespace fa {

struct BwdParams {
  const __nv_bfloat16* o;     // [B, Nq, Hq, D]
  const __nv_bfloat16* dout;  // [B, Nq, Hq, D]
  const float* lse;           // [B, Hq, Nq] (natural log)
  float* lse2;                // [B, Hq, NqPad] lse * log2(e); +inf where P must be 0
  float* dvec;                // [B, Hq, NqPad] D_i = sum_c dO_ic O_ic
  float* dq_acc;              // [B, Nq, Hq, D] fp32
  __nv_bfloat16* dq;          // [B, Nq, Hq, D]
  __nv_bfloat16* dk;          // [B, Nk, Hkv, D]
  __nv_bfloat16* dv;          // [B, Nk, Hkv, D]
  int B, Hq, Hkv, G, Nq, Nk, NqPad;
  int causal;
  float tau;    // scale * log2(e)
  float scale;
  // packed variable-length sequences (null cu: fixed length).  Sequence b holds rows
  // [cu[b], cu[b+1]) of q, k, v, o, dO and their gradients; lse is [Hq, total].  Key tiles
  // of all sequences are numbered in order: tiles[b] = 128-row tiles of sequences before b.
  // The row vectors hold, per head, ntiles * 128 entries; sequence b's queries start at
  // entry tiles[b] * 128, padded to whole tiles.
  const int32_t* cu;  // [B + 1]
  int32_t* tiles;     // [B + 1], written by fa_bwd_tiles_kernel
  int ntiles;         // bound on tiles[B]: the CTA index space and the vector stride / 128
  int total;          // packed rows
};

constexpr int kBwdThreads = 384;
constexpr int kBwdTile = 128;            // keys per CTA tile and queries per pair
constexpr int kBwdMaxSmem = 232448;      // sm_100 per-block limit

template <int D>
struct BwdCfg {
  static constexpr int kTileBytes = kBwdTile * D * 2;
  static constexpr int kChunkBytes = kBwdTile * 128;  // 128 rows x one 64-column panel
  static constexpr int kVecBytes = kBwdTile * 4;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kTileBytes;
  static constexpr int kOffQ = 2 * kTileBytes;   // [2]
  static constexpr int kOffDO = 4 * kTileBytes;  // [2]
  static constexpr int kOffDS = 6 * kTileBytes;  // 128 keys x 128 queries bf16
  static constexpr int kOffVec = kOffDS + kBwdTile * kBwdTile * 2;  // [slot][lse2, D]
  static constexpr int kOffBar = kOffVec + 4 * kVecBytes;
  static constexpr int kNumBars = 16;
  static constexpr int kUsed = kOffBar + kNumBars * 8 + 16;
  static constexpr int kSmemBytes = (kUsed + 1024 < kBwdMaxSmem) ? kUsed + 1024 : kBwdMaxSmem;
  // TMEM columns
  static constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + D;
};

// Where one CTA's 128-key tile lies.  Fixed length: sequence z, tile x.  Varlen: x numbers
// the tiles of all sequences in order; the sequence is found by bisection over the tile
// prefix sums, and an index at or past the last tile has no work.
struct BwdSeq {
  int tile;        // the tile within its sequence
  int nq, nk;      // query and key rows of the sequence
  int rowq, rowk;  // its first row in the q-side (q, o, dO, dQ) and k-side (k, v, dK, dV) rows
  long long vec0;  // row-vector entry of (head 0, query 0); head h adds h * vech
  long long vech;
};

// Largest b in [0, B] with tiles[b] <= x (B: x is at or past the last tile).
__device__ __forceinline__ int bwd_find_seq(const BwdParams& p, int x) {
  int lo = 0, hi = p.B;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(p.tiles + mid) <= x) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ bool bwd_locate(const BwdParams& p, int x, int z, BwdSeq& s) {
  if (p.cu == nullptr) {
    s.tile = x;
    s.nq = p.Nq;
    s.nk = p.Nk;
    s.rowq = z * p.Nq;
    s.rowk = z * p.Nk;
    s.vech = p.NqPad;
    s.vec0 = (long long)z * p.Hq * p.NqPad;
    return true;
  }
  const int b = bwd_find_seq(p, x);
  if (b >= p.B) return false;
  const int t0 = __ldg(p.tiles + b);
  const int c0 = __ldg(p.cu + b);
  s.tile = x - t0;
  s.nq = s.nk = __ldg(p.cu + b + 1) - c0;
  s.rowq = s.rowk = c0;
  s.vech = (long long)p.ntiles * kBwdTile;
  s.vec0 = (long long)t0 * kBwdTile;
  return true;
}

// CTA index -> (key tile number x, K/V head, sequence z) of the main kernels' 1-D grid.
// K/V heads go in groups of kBwdHeadGroup; within a group the order is tile-major with the
// group's heads (and at fixed length the sequences) varying fastest.  In a causal backward
// the first key tiles of a sequence see the most query tiles, so each group launches its
// longest CTAs first (close to a longest-first list schedule), while the CTAs in flight
// share few heads, so that their Q, dO and fp32 dQ-accumulator rows mostly stay in L2.
// Measured on the 8K GQA causal backward (Hkv = 8), groups of 1 (head-major) / 2 / 4 / 8:
// 3.72 / 3.21 / 3.16 / 3.22 ms with 1.19 / 1.77 / 3.74 / 6.48 GB of DRAM traffic.
constexpr int kBwdHeadGroup = 2;
__device__ __forceinline__ void bwd_cta_coords(const BwdParams& p, int& x, int& kvh, int& z) {
  const int Z = p.cu == nullptr ? p.B : 1;
  const int X = p.cu == nullptr ? (p.Nk + kBwdTile - 1) / kBwdTile : p.ntiles;
  const int hg = min(kBwdHeadGroup, p.Hkv);
  const int L = (int)blockIdx.x;
  const int gi = L / (X * hg * Z);
  const int r = L - gi * (X * hg * Z);
  const int sz = min(hg, p.Hkv - gi * hg);  // heads in this group (the last may be short)
  x = r / (sz * Z);
  const int r2 = r - x * (sz * Z);
  kvh = gi * hg + r2 % sz;
  z = r2 / sz;
}

// ------------------------------------------------------------------ varlen: tile prefix sums
// One block: tiles[b] = sum over sequences before b of ceil(len / 128).  cu must start at or
// above 0, never decrease and end at or below total; otherwise every entry is 0 (no CTA of
// the main kernel has work) and kErrBadSeqlens is recorded.
constexpr int kTilesThreads = 1024;
__global__ void __launch_bounds__(kTilesThreads) fa_bwd_tiles_kernel(const BwdParams p) {
  __shared__ int warp_sum[kTilesThreads / 32];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int per = (p.B + kTilesThreads - 1) / kTilesThreads;
  const int b0 = min(p.B, t * per), b1 = min(p.B, b0 + per);
  int sum = 0, bad = 0;
  for (int b = b0; b < b1; ++b) {
    const int c0 = __ldg(p.cu + b), c1 = __ldg(p.cu + b + 1);
    bad |= (c1 < c0) | (b == 0 && c0 < 0) | (b == p.B - 1 && c1 > p.total);
    sum += (max(c1 - c0, 0) + kBwdTile - 1) / kBwdTile;
  }
  // exclusive prefix of the per-thread sums: within the warp, then over the warp totals
  int incl = sum;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) warp_sum[warp] = incl;
  bad = __syncthreads_or(bad);
  if (warp == 0) {
    int w = warp_sum[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, off);
      if (lane >= off) w += y;
    }
    warp_sum[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  int run = incl - sum + (warp > 0 ? warp_sum[warp - 1] : 0);
  const int grand = warp_sum[kTilesThreads / 32 - 1];
  bad |= grand > p.ntiles;
  if (bad) {
    for (int b = t; b <= p.B; b += kTilesThreads) p.tiles[b] = 0;
    if (t == 0) atomicOr(&g_error_word, kErrBadSeqlens);
    return;
  }
  for (int b = b0; b < b1; ++b) {
    p.tiles[b] = run;
    run += (__ldg(p.cu + b + 1) - __ldg(p.cu + b) + kBwdTile - 1) / kBwdTile;
  }
  if (t == 0) p.tiles[p.B] = grand;
}

// ------------------------------------------------------------------ pre: D and lse2, zero dQ
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(const BwdParams p) {
  const int warps = blockDim.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr int E = D / 32;  // elements per lane
  const bool varlen = p.cu != nullptr;
  const long long per_head = (long long)p.ntiles * kBwdTile;  // varlen vector entries per head
  const long long rows = varlen ? per_head * p.Hq : (long long)p.B * p.Hq * p.NqPad;
  if (varlen) {
    // the accumulator as one flat range (rows outside every sequence included)
    const size_t n4 = (size_t)p.total * p.Hq * D / 4;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x)
      reinterpret_cast<float4*>(p.dq_acc)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (long long w = (long long)blockIdx.x * warps + (threadIdx.x >> 5); w < rows; w += (long long)gridDim.x * warps) {
    // vector entry w -> row of o / dO (units of D; -1: padding) and lse index
    long long row = -1, li = 0;
    if (!varlen) {
      const int q = (int)(w % p.NqPad);
      const long long bh = w / p.NqPad;
      const int h = (int)(bh % p.Hq);
      const int b = (int)(bh / p.Hq);
      if (q < p.Nq) {
        row = ((long long)b * p.Nq + q) * p.Hq + h;
        li = ((long long)b * p.Hq + h) * p.Nq + q;
      }
    } else {
      const int h = (int)(w / per_head);
      const int pos = (int)(w - h * per_head);
      const int b = bwd_find_seq(p, pos / kBwdTile);
      if (b < p.B) {
        const int c0 = __ldg(p.cu + b);
        const int q = pos - __ldg(p.tiles + b) * kBwdTile;
        if (q < __ldg(p.cu + b + 1) - c0) {
          row = ((long long)c0 + q) * p.Hq + h;
          li = (long long)h * p.total + c0 + q;
        }
      }
    }
    float dsum = 0.f, l2 = INFINITY;
    if (row >= 0) {
      const __nv_bfloat16* orow = p.o + row * D + lane * E;
      const __nv_bfloat16* drow = p.dout + row * D + lane * E;
#pragma unroll
      for (int e = 0; e < E; e += 2) {
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(orow + e));
        const float2 g = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(drow + e));
        dsum = fmaf(a.x, g.x, fmaf(a.y, g.y, dsum));
      }
      if (!varlen) {
        float* acc = p.dq_acc + row * D + lane * E;
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = 0.f;
      }
      const float l = p.lse[li];
      l2 = (l == -INFINITY) ? INFINITY : l * 1.4426950408889634f;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, off);
    if (lane == 0) {
      p.dvec[w] = dsum;
      p.lse2[w] = l2;
    }
  }
}

// ------------------------------------------------------------------ post: dQ to bf16
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_dq_kernel(const BwdParams p) {
  const size_t rows = p.cu != nullptr ? (size_t)p.total : (size_t)p.B * p.Nq;
  const size_t n4 = rows * p.Hq * D / 4;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
    const float4 x = reinterpret_cast<const float4*>(p.dq_acc)[i];
    uint2 w;
    w.x = pack_bf16x2(x.x * p.scale, x.y * p.scale);
    w.y = pack_bf16x2(x.z * p.scale, x.w * p.scale);
    reinterpret_cast<uint2*>(p.dq)[i] = w;
  }
}

// ------------------------------------------------------------------ main
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                  const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  {
    uint32_t dyn;
    asm volatile("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
    if ((uint32_t)(smem - smem_raw) + (uint32_t)C::kUsed > dyn) {
      if (threadIdx.x == 0) atomicOr(&g_error_word, kErrSmem);
      return;
    }
  }
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sDO = smem + C::kOffDO;
  uint8_t* sDS = smem + C::kOffDS;
  float* sVec = reinterpret_cast<float*>(smem + C::kOffVec);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* kv_full = bars + 0;
  uint64_t* q_full = bars + 1;     // [2]
  uint64_t* q_empty = bars + 3;    // [2]
  uint64_t* sdp_full = bars + 5;   // S^T and dP^T in TMEM
  uint64_t* ld_done = bars + 6;    // both warpgroups have read S^T and dP^T
  uint64_t* pds_ready = bars + 7;  // P^T, dS^T in TMEM and dS in shared memory
  uint64_t* dq_full = bars + 8;    // dQ in TMEM
  uint64_t* dq_free = bars + 9;    // dQ read out
  uint64_t* acc_done = bars + 10;  // last dK/dV product complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  BwdSeq sq;
  int cta_x, kvh, cta_z;
  bwd_cta_coords(p, cta_x, kvh, cta_z);
  if (!bwd_locate(p, cta_x, cta_z, sq)) return;  // varlen: no tile of this index
  const int Nq = sq.nq, Nk = sq.nk;
  const int n0 = sq.tile * kBwdTile;
  const int diag = Nk - Nq;  // causal: key j is allowed for query i iff j <= i + diag
  const int nq_tiles = (Nq + kBwdTile - 1) / kBwdTile;
  int i_lo = 0;
  if (p.causal) {
    const int need = n0 - diag - (kBwdTile - 1);  // first tile whose last query sees key n0
    i_lo = need <= 0 ? 0 : (need + kBwdTile - 1) / kBwdTile;
  }
  const int ntq = max(0, nq_tiles - i_lo);
  const int T = ntq * p.G;  // (query head, query tile) pairs; heads outer

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(q_full + s, 1);
      mbar_init(q_empty + s, 1);
    }
    mbar_init(sdp_full, 1);
    mbar_init(ld_done, 8);
    mbar_init(pds_ready, 8);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, 8);
    mbar_init(acc_done, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ============================================================ TMA producer
    if (T > 0) {
      mbar_arrive_expect_tx_elect(kv_full, 2 * C::kTileBytes);
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d_elect(sK + c * C::kChunkBytes, &tmK, c * 64, kvh, sq.rowk + n0, kv_full);
        tma_load_3d_elect(sV + c * C::kChunkBytes, &tmV, c * 64, kvh, sq.rowk + n0, kv_full);
      }
      for (int t = 0; t < T; ++t) {
        const int slot = t & 1;
        if (t >= 2 && !warp_wait(q_empty + slot, ((t >> 1) - 1) & 1)) break;
        const int h = kvh * p.G + t / ntq;
        const int q0 = (i_lo + t % ntq) * kBwdTile;
        mbar_arrive_expect_tx_elect(q_full + slot, 2 * C::kTileBytes + 2 * C::kVecBytes);
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d_elect(sQ + slot * C::kTileBytes + c * C::kChunkBytes, &tmQ, c * 64, h, sq.rowq + q0,
                            q_full + slot);
          tma_load_3d_elect(sDO + slot * C::kTileBytes + c * C::kChunkBytes, &tmDO, c * 64, h, sq.rowq + q0,
                            q_full + slot);
        }
        const size_t voff = (size_t)(sq.vec0 + h * sq.vech + q0);
        bulk_load_elect(sVec + (slot * 2 + 0) * kBwdTile, p.lse2 + voff, C::kVecBytes, q_full + slot);
        bulk_load_elect(sVec + (slot * 2 + 1) * kBwdTile, p.dvec + voff, C::kVecBytes, q_full + slot);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    if (T > 0) {
      constexpr uint32_t idS = idesc_bf16_f32(kBwdTile, kBwdTile, false);  // K-major A and B
      constexpr uint32_t idAcc = idesc_bf16_f32(kBwdTile, D, true);        // B MN-major
      constexpr uint32_t idQ = idesc_bf16_f32_mn(kBwdTile, 64, true, true);
      const uint32_t kb = smem_u32(sK), vb = smem_u32(sV), qb = smem_u32(sQ), dob = smem_u32(sDO);
      const uint32_t dsb = smem_u32(sDS);
      bool ok = warp_wait(kv_full, 0);
      tc_fence_after();
      for (int t = 0; t < T && ok; ++t) {
        const int slot = t & 1;
        if (!warp_wait(q_full + slot, (t >> 1) & 1)) break;
        if (t > 0 && !warp_wait(dq_free, (t - 1) & 1)) break;
        tc_fence_after();
        const uint32_t qs = qb + slot * C::kTileBytes, ds = dob + slot * C::kTileBytes;
        // S^T = K Q^T and dP^T = V dO^T (k-steps of 16 along d)
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kChunkBytes + (kk & 3) * 32;
          umma_ss_elect(tmem + C::kColS, smem_desc_sw128(kb + off, 16, 1024), smem_desc_sw128(qs + off, 16, 1024),
                        idS, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kChunkBytes + (kk & 3) * 32;
          umma_ss_elect(tmem + C::kColDP, smem_desc_sw128(vb + off, 16, 1024), smem_desc_sw128(ds + off, 16, 1024),
                        idS, kk > 0 ? 1u : 0u);
        }
        umma_commit_elect(sdp_full);
        if (!warp_wait(pds_ready, t & 1)) break;
        tc_fence_after();
        // dV += P^T dO, dK += dS^T Q (k-steps of 16 queries; A from TMEM)
#pragma unroll
        for (int kk = 0; kk < kBwdTile / 16; ++kk) {
          const uint32_t acc = (t > 0 || kk > 0) ? 1u : 0u;
          umma_ts_elect(tmem + C::kColDV, tmem + C::kColS + kk * 8,
                        smem_desc_sw128(ds + kk * 16 * 128, C::kChunkBytes, 1024), idAcc, acc);
          umma_ts_elect(tmem + C::kColDK, tmem + C::kColDP + kk * 8,
                        smem_desc_sw128(qs + kk * 16 * 128, C::kChunkBytes, 1024), idAcc, acc);
        }
        // dQ = dS K in 64-column halves (k-steps of 16 keys; A query-major from shared memory)
#pragma unroll
        for (int hh = 0; hh < D / 64; ++hh) {
#pragma unroll
          for (int kk = 0; kk < kBwdTile / 16; ++kk)
            umma_ss_elect(tmem + (hh ? C::kColDP : C::kColS) + 64,
                          smem_desc_sw128(dsb + kk * 16 * 128, C::kChunkBytes, 1024),
                          smem_desc_sw128(kb + hh * C::kChunkBytes + kk * 16 * 128, C::kChunkBytes, 1024), idQ,
                          kk > 0 ? 1u : 0u);
        }
        umma_commit_elect(dq_full);
        umma_commit_elect(q_empty + slot);
      }
      umma_commit_elect(acc_done);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ============================================================ elementwise warpgroups
    const int wg = (warp - 4) >> 2;
    const int r = (warp & 3) * 32 + lane;  // key row of the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const int key = n0 + r;
    const bool key_ok = key < Nk;
    const float tau = p.tau;
    bool ok = true;
    for (int t = 0; t < T && ok; ++t) {
      const int slot = t & 1;
      const int h = kvh * p.G + t / ntq;
      const int q0 = (i_lo + t % ntq) * kBwdTile;
      if (!warp_wait(q_full + slot, (t >> 1) & 1) || !warp_wait(sdp_full, t & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float* l2 = sVec + (slot * 2 + 0) * kBwdTile + 64 * wg;
      const float* dd = sVec + (slot * 2 + 1) * kBwdTile + 64 * wg;
      uint32_t pk[32], dsk[32];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t sv[32], dpv[32];
        tmem_ld32(tmem + lane_off + C::kColS + 64 * wg + 32 * c, sv);
        tmem_ld32(tmem + lane_off + C::kColDP + 64 * wg + 32 * c, dpv);
        tmem_wait_ld();
        // allowed iff key_ok and (not causal or key <= q + diag), q = q0 + 64 wg + 32 c + e
        const int qfirst = q0 + 64 * wg + 32 * c;
        int lim = 0;  // columns e < lim are masked
        if (!key_ok) lim = 32;
        else if (p.causal) lim = min(32, max(0, key - diag - qfirst));
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float4 lv = *reinterpret_cast<const float4*>(l2 + 32 * c + 4 * (e >> 1));
          const float4 dv4 = *reinterpret_cast<const float4*>(dd + 32 * c + 4 * (e >> 1));
          const float la = (e & 1) ? lv.z : lv.x, lb = (e & 1) ? lv.w : lv.y;
          const float da = (e & 1) ? dv4.z : dv4.x, db = (e & 1) ? dv4.w : dv4.y;
          float p0 = ex2_approx(fmaf(__uint_as_float(sv[2 * e]), tau, -la));
          float p1 = ex2_approx(fmaf(__uint_as_float(sv[2 * e + 1]), tau, -lb));
          if (2 * e < lim) p0 = 0.f;
          if (2 * e + 1 < lim) p1 = 0.f;
          const float ds0 = p0 * (__uint_as_float(dpv[2 * e]) - da);
          const float ds1 = p1 * (__uint_as_float(dpv[2 * e + 1]) - db);
          pk[16 * c + e] = pack_bf16x2(p0, p1);
          dsk[16 * c + e] = pack_bf16x2(ds0, ds1);
        }
      }
      // dS row r (queries 64 wg .. 64 wg + 63) into the query-major A tile: panel wg, row r,
      // 16-byte unit u stored at u ^ (r % 8) (128-byte swizzle)
      {
        uint8_t* row = sDS + wg * C::kChunkBytes + r * 128;
#pragma unroll
        for (int u = 0; u < 8; ++u)
          *reinterpret_cast<uint4*>(row + ((u ^ (r & 7)) << 4)) =
              make_uint4(dsk[4 * u], dsk[4 * u + 1], dsk[4 * u + 2], dsk[4 * u + 3]);
      }
      // P^T and dS^T go over the first 64 columns of their regions, which the other
      // warpgroup may still be reading: wait until both have read S^T and dP^T
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(ld_done);
      if (!warp_wait(ld_done, t & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      tmem_st32(tmem + lane_off + C::kColS + 32 * wg, pk);
      tmem_st32(tmem + lane_off + C::kColDP + 32 * wg, dsk);
      tmem_wait_st();
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // dS tile -> tensor core
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(pds_ready);
      // dQ of this pair: TMEM lane r = query q0 + r; this warpgroup adds its half of d
      if (!warp_wait(dq_full, t & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      {
        constexpr int kCols = D / 2;  // columns of d per warpgroup
        const uint32_t src = (D == 128) ? (tmem + lane_off + (wg ? C::kColDP : C::kColS) + 64)
                                        : (tmem + lane_off + C::kColS + 64 + 32 * wg);
        const int q = q0 + r;
        float* dst = p.dq_acc + (((size_t)sq.rowq + q) * p.Hq + h) * D + wg * kCols;
        uint32_t a0[32], a1[32];
        tmem_ld32(src, a0);
        if (kCols == 64) tmem_ld32(src + 32, a1);
        tmem_wait_ld();
        // TMEM is free again as soon as the values are in registers: release it before the
        // reductions, so the next pair's products start while they drain
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(dq_free);
        if (q < Nq) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            red_add_v4(dst + e, __uint_as_float(a0[e]), __uint_as_float(a0[e + 1]), __uint_as_float(a0[e + 2]),
                       __uint_as_float(a0[e + 3]));
          if (kCols == 64) {
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              red_add_v4(dst + 32 + e, __uint_as_float(a1[e]), __uint_as_float(a1[e + 1]),
                         __uint_as_float(a1[e + 2]), __uint_as_float(a1[e + 3]));
          }
        }
      }
    }
    // ---- epilogue: dV (warpgroup 0) and dK = scale * acc (warpgroup 1), rows of this key tile
    // (T is uniform over the CTA, so every warp takes the same path to the collective loads)
    const bool have = T > 0 && ok && warp_wait(acc_done, 0);
    tc_fence_after();
    __nv_bfloat16* dst = (wg ? p.dk : p.dv) + (((size_t)sq.rowk + key) * p.Hkv + kvh) * D;
    const float mul = wg ? p.scale : 1.f;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t a[32];
      if (have) {
        tmem_ld32(tmem + lane_off + (wg ? C::kColDK : C::kColDV) + 32 * c, a);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) a[e] = 0u;
      }
      if (key_ok) {
        uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          d4[e] = make_uint4(pack_bf16x2(__uint_as_float(a[8 * e]) * mul, __uint_as_float(a[8 * e + 1]) * mul),
                             pack_bf16x2(__uint_as_float(a[8 * e + 2]) * mul, __uint_as_float(a[8 * e + 3]) * mul),
                             pack_bf16x2(__uint_as_float(a[8 * e + 4]) * mul, __uint_as_float(a[8 * e + 5]) * mul),
                             pack_bf16x2(__uint_as_float(a[8 * e + 6]) * mul, __uint_as_float(a[8 * e + 7]) * mul));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ main, d = 128: two pairs in flight
//
// Same method as fa_bwd_kernel, arranged so that the tensor core and the elementwise
// warpgroups work on different pairs at once: pairs of 64 queries, two TMEM buffers
//   S_b = TMEM[128 b, 128 b + 64), DP_b = TMEM[128 b + 64, 128 b + 128)   (b = pair & 1)
// dV = TMEM[256, 384), dK = TMEM[384, 512).  Per pair t (buffer b):
//   S^T = K Q^T -> S_b, dP^T = V dO^T -> DP_b                        (tcgen05, N = 64)
//   elementwise: P^T, dS^T (bf16) of warpgroup w's 32 queries over S_b[32w, 32w+16) and
//                S_b[32w+16, 32w+32) (the columns it read), dS to shared memory
//   dV += P^T dO, dK += dS^T Q                                        (A from TMEM)
//   dQ^T = K^T dS -> DP_b   (M = d on the TMEM lanes, so each warp's dQ read-out covers 32
//                            consecutive d: coalesced fp32 reductions)
// The MMA warp issues S(t) and dP(t) before the gradient products of pair t-1, so the
// elementwise step of pair t overlaps those products; the warpgroups read dQ^T(t-1) out after
// the elementwise step of pair t.
constexpr int kBwdQ = 64;  // queries per pair
constexpr int kBwdSlots = 3;

struct Bwd2Cfg {
  static constexpr int D = 128;
  static constexpr int kKTile = kBwdTile * D * 2;       // 32 KB: 128 keys, 2 panels of 16 KB
  static constexpr int kKPanel = kBwdTile * 128;
  static constexpr int kQTile = kBwdQ * D * 2;          // 16 KB: 64 queries, 2 panels of 8 KB
  static constexpr int kQPanel = kBwdQ * 128;
  static constexpr int kDSTile = kBwdTile * kBwdQ * 2;  // 16 KB: 128 keys x 64 queries
  static constexpr int kVecBytes = kBwdQ * 4;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kKTile;
  static constexpr int kOffQ = 2 * kKTile;                          // [slots]
  static constexpr int kOffDO = kOffQ + kBwdSlots * kQTile;         // [slots]
  static constexpr int kOffDS = kOffDO + kBwdSlots * kQTile;        // [2]
  static constexpr int kStageBytes = kBwdQ * D * 4;                 // dQ of one pair, [64 q][128 d] fp32
  static constexpr int kOffStage = kOffDS + 2 * kDSTile;
  static constexpr int kOffVec = kOffStage + kStageBytes;           // [slots][lse2, D]
  static constexpr int kOffBar = kOffVec + kBwdSlots * 2 * kVecBytes;
  static constexpr int kNumBars = 24;
  static constexpr int kUsed = kOffBar + kNumBars * 8 + 16;
  static constexpr int kSmemBytes = kUsed + 1024;
  static_assert(kSmemBytes <= kBwdMaxSmem, "shared memory");
  static constexpr uint32_t kColDV = 256, kColDK = 384;
};

__global__ void __launch_bounds__(kBwdThreads, 1)
    fa_bwd2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                   const __grid_constant__ CUtensorMap tmDQ, const BwdParams p) {
  using C = Bwd2Cfg;
  constexpr int D = C::D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  {
    uint32_t dyn;
    asm volatile("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
    if ((uint32_t)(smem - smem_raw) + (uint32_t)C::kUsed > dyn) {
      if (threadIdx.x == 0) atomicOr(&g_error_word, kErrSmem);
      return;
    }
  }
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sDO = smem + C::kOffDO;
  uint8_t* sDS = smem + C::kOffDS;
  float* sStage = reinterpret_cast<float*>(smem + C::kOffStage);
  float* sVec = reinterpret_cast<float*>(smem + C::kOffVec);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* kv_full = bars + 0;
  uint64_t* q_full = bars + 1;     // [slots]
  uint64_t* q_empty = bars + 4;    // [slots]
  uint64_t* sdp_full = bars + 7;   // [2] S^T in TMEM
  uint64_t* dp_full = bars + 9;    // [2] dP^T in TMEM
  uint64_t* pds_ready = bars + 11; // [2]
  uint64_t* dq_full = bars + 13;   // [2]
  uint64_t* buf_free = bars + 15;  // [2]
  uint64_t* acc_done = bars + 17;
  uint64_t* stage_full = bars + 18;  // the warpgroups wrote dQ of a pair into the staging tile
  uint64_t* stage_free = bars + 19;  // its reduction has read the staging tile
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  BwdSeq sq;
  int cta_x, kvh, cta_z;
  bwd_cta_coords(p, cta_x, kvh, cta_z);
  if (!bwd_locate(p, cta_x, cta_z, sq)) return;  // varlen: no tile of this index
  const int Nq = sq.nq, Nk = sq.nk;
  const int n0 = sq.tile * kBwdTile;
  const int diag = Nk - Nq;
  const int nq_tiles = (Nq + kBwdQ - 1) / kBwdQ;
  int i_lo = 0;
  if (p.causal) {
    const int need = n0 - diag - (kBwdQ - 1);  // first 64-query tile whose last query sees key n0
    i_lo = need <= 0 ? 0 : (need + kBwdQ - 1) / kBwdQ;
  }
  const int ntq = max(0, nq_tiles - i_lo);
  const int T = ntq * p.G;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < kBwdSlots; ++s) {
      mbar_init(q_full + s, 1);
      mbar_init(q_empty + s, 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(sdp_full + x, 1);
      mbar_init(dp_full + x, 1);
      mbar_init(pds_ready + x, 8);
      mbar_init(dq_full + x, 1);
      mbar_init(buf_free + x, 8);
    }
    mbar_init(acc_done, 1);
    mbar_init(stage_full, 8);
    mbar_init(stage_free, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 2) {
    // ============================================================ dQ reductions
    // One TMA reduce-add per pair: the staging tile [64 queries][128 d] into the fp32
    // accumulator rows of that pair's (query head, query tile).  Queries past Nq add zeros
    // (their dS is 0), into rows that exist or lie beyond the tensor (then skipped).
    if (lane == 0) {
      for (int tp = 0; tp < T; ++tp) {
        if (!mbar_wait(stage_full, tp & 1)) break;
        const int h = kvh * p.G + tp / ntq;
        const int q0 = (i_lo + tp % ntq) * kBwdQ;
        tma_reduce_add_3d(&tmDQ, sStage, 0, h, sq.rowq + q0);
        bulk_commit_group();
        bulk_wait_group_read0();
        mbar_arrive(stage_free);
      }
      bulk_wait_group0();
    }
    __syncwarp();
  } else if (warp == 0) {
    // ============================================================ TMA producer
    if (T > 0) {
      mbar_arrive_expect_tx_elect(kv_full, 2 * C::kKTile);
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d_elect(sK + c * C::kKPanel, &tmK, c * 64, kvh, sq.rowk + n0, kv_full);
        tma_load_3d_elect(sV + c * C::kKPanel, &tmV, c * 64, kvh, sq.rowk + n0, kv_full);
      }
      for (int t = 0; t < T; ++t) {
        const int slot = t % kBwdSlots;
        if (t >= kBwdSlots && !warp_wait(q_empty + slot, ((t / kBwdSlots) - 1) & 1)) break;
        const int h = kvh * p.G + t / ntq;
        const int q0 = (i_lo + t % ntq) * kBwdQ;
        mbar_arrive_expect_tx_elect(q_full + slot, 2 * C::kQTile + 2 * C::kVecBytes);
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d_elect(sQ + slot * C::kQTile + c * C::kQPanel, &tmQ, c * 64, h, sq.rowq + q0, q_full + slot);
          tma_load_3d_elect(sDO + slot * C::kQTile + c * C::kQPanel, &tmDO, c * 64, h, sq.rowq + q0,
                            q_full + slot);
        }
        const size_t voff = (size_t)(sq.vec0 + h * sq.vech + q0);
        bulk_load_elect(sVec + (slot * 2 + 0) * kBwdQ, p.lse2 + voff, C::kVecBytes, q_full + slot);
        bulk_load_elect(sVec + (slot * 2 + 1) * kBwdQ, p.dvec + voff, C::kVecBytes, q_full + slot);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    if (T > 0) {
      constexpr uint32_t idS = idesc_bf16_f32(kBwdTile, kBwdQ, false);
      constexpr uint32_t idAcc = idesc_bf16_f32(kBwdTile, D, true);
      constexpr uint32_t idQ = idesc_bf16_f32_mn(D, kBwdQ, true, true);
      const uint32_t kb = smem_u32(sK), vb = smem_u32(sV), qb = smem_u32(sQ), dob = smem_u32(sDO);
      const uint32_t dsb = smem_u32(sDS);
      const uint64_t dK0 = smem_desc_sw128(kb, 16, 1024), dV0 = smem_desc_sw128(vb, 16, 1024);
      const uint64_t dKmn = smem_desc_sw128(kb, C::kKPanel, 1024);  // K read d-major (A of dQ^T)
      bool ok = warp_wait(kv_full, 0);
      tc_fence_after();
      for (int t = 0; t <= T && ok; ++t) {
        if (t < T) {
          const int slot = t % kBwdSlots, bb = t & 1;
          if (!warp_wait(q_full + slot, (t / kBwdSlots) & 1)) break;
          if (t >= 2 && !warp_wait(buf_free + bb, ((t >> 1) - 1) & 1)) break;
          tc_fence_after();
          const uint32_t qs = qb + slot * C::kQTile, ds = dob + slot * C::kQTile;
          const uint32_t cS = 128 * bb, cDP = 128 * bb + 64;
          // descriptors built once per pair; a k-step only moves the start address (16-byte
          // units, no carry: shared addresses are below 2^18 bytes); one elected lane issues
          // each group of products and its commit
          const uint64_t dQs = smem_desc_sw128(qs, 16, 1024), dDOs = smem_desc_sw128(ds, 16, 1024);
          if (elect_one_lane()) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t ka = ((kk >> 2) * C::kKPanel + (kk & 3) * 32) >> 4;
              const uint32_t kq = ((kk >> 2) * C::kQPanel + (kk & 3) * 32) >> 4;
              mma_ss<0>(tmem + cS, dK0 + ka, dQs + kq, idS, kk > 0 ? 1u : 0u);
            }
            umma_commit(sdp_full + bb);  // the exponentials start while dP^T is formed
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t ka = ((kk >> 2) * C::kKPanel + (kk & 3) * 32) >> 4;
              const uint32_t kq = ((kk >> 2) * C::kQPanel + (kk & 3) * 32) >> 4;
              mma_ss<0>(tmem + cDP, dV0 + ka, dDOs + kq, idS, kk > 0 ? 1u : 0u);
            }
            umma_commit(dp_full + bb);
          }
          __syncwarp();
        }
        if (t >= 1) {
          const int tp = t - 1, slot = tp % kBwdSlots, bb = tp & 1;
          if (!warp_wait(pds_ready + bb, (tp >> 1) & 1)) break;
          tc_fence_after();
          const uint32_t qs = qb + slot * C::kQTile, ds = dob + slot * C::kQTile;
          const uint32_t cS = 128 * bb, cDP = 128 * bb + 64;
          const uint64_t dDOmn = smem_desc_sw128(ds, C::kQPanel, 1024), dQmn = smem_desc_sw128(qs, C::kQPanel, 1024);
          const uint64_t dDS = smem_desc_sw128(dsb + bb * C::kDSTile, C::kDSTile, 1024);
          if (elect_one_lane()) {
#pragma unroll
            for (int kk = 0; kk < kBwdQ / 16; ++kk) {
              const uint32_t acc = (tp > 0 || kk > 0) ? 1u : 0u;
              // queries 16 kk .. 16 kk + 15: warpgroup kk / 2, P^T at 32 (kk / 2) + 8 (kk % 2), dS^T 16 further
              const uint32_t pc = cS + 32 * (kk >> 1) + 8 * (kk & 1);
              const uint32_t off = (kk * 16 * 128) >> 4;
              mma_ts<0>(tmem + C::kColDV, tmem + pc, dDOmn + off, idAcc, acc);
              mma_ts<0>(tmem + C::kColDK, tmem + pc + 16, dQmn + off, idAcc, acc);
            }
            // dQ^T = K^T dS: A = K (keys x d) read d-major, B = dS (keys x queries) query-major
#pragma unroll
            for (int kk = 0; kk < kBwdTile / 16; ++kk) {
              const uint32_t off = (kk * 16 * 128) >> 4;
              mma_ss<0>(tmem + cDP, dKmn + off, dDS + off, idQ, kk > 0 ? 1u : 0u);
            }
            umma_commit(dq_full + bb);
            umma_commit(q_empty + slot);
          }
          __syncwarp();
        }
      }
      umma_commit_elect(acc_done);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ============================================================ elementwise warpgroups
    const int wg = (warp - 4) >> 2;
    const int r = (warp & 3) * 32 + lane;  // TMEM lane: key row (S, dP) or d (dQ^T)
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const int key = n0 + r;
    const bool key_ok = key < Nk;
    const float tau = p.tau;
    bool ok = true;

    auto read_dq = [&](int tp) -> bool {
      const int bb = tp & 1;
      if (!warp_wait(dq_full + bb, (tp >> 1) & 1)) return false;
      tc_fence_after();
      uint32_t a[32];
      tmem_ld32(tmem + lane_off + 128 * bb + 64 + 32 * wg, a);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(buf_free + bb);
      // stage row q = 32 wg + e, column d = r (lanes write consecutive d: no bank conflicts),
      // once the previous pair's reduction has read the tile
      if (tp >= 1 && !warp_wait(stage_free, (tp - 1) & 1)) return false;
#pragma unroll
      for (int e = 0; e < 32; ++e) sStage[(32 * wg + e) * D + r] = __uint_as_float(a[e]);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(stage_full);
      return true;
    };

    for (int t = 0; t < T && ok; ++t) {
      const int slot = t % kBwdSlots, bb = t & 1;
      const int q0 = (i_lo + t % ntq) * kBwdQ;
      if (!warp_wait(q_full + slot, (t / kBwdSlots) & 1) || !warp_wait(sdp_full + bb, (t >> 1) & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t cS = 128 * bb, cDP = 128 * bb + 64;
      const float* l2 = sVec + (slot * 2 + 0) * kBwdQ + 32 * wg;
      const float* dd = sVec + (slot * 2 + 1) * kBwdQ + 32 * wg;
      uint32_t pk[16], dsk[16];
      {
        uint32_t sv[32];
        tmem_ld32(tmem + lane_off + cS + 32 * wg, sv);
        // the row vectors of this warpgroup's 32 queries (broadcast reads), while TMEM loads
        float4 lv[8], dv4[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          lv[e] = reinterpret_cast<const float4*>(l2)[e];
          dv4[e] = reinterpret_cast<const float4*>(dd)[e];
        }
        tmem_wait_ld();
        const int qfirst = q0 + 32 * wg;
        int lim = 0;  // columns e < lim are masked
        if (!key_ok) lim = 32;
        else if (p.causal) lim = min(32, max(0, key - diag - qfirst));
        const uint64_t tau2 = f2(tau, tau);
        uint64_t pp[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float4 L = lv[e >> 1];
          const uint64_t nl = (e & 1) ? f2(-L.z, -L.w) : f2(-L.x, -L.y);
          float x0, x1;
          f2_split(f2_fma(f2(__uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1])), tau2, nl), x0, x1);
          float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
          if (2 * e < lim) p0 = 0.f;
          if (2 * e + 1 < lim) p1 = 0.f;
          pk[e] = pack_bf16x2(p0, p1);
          pp[e] = f2(p0, p1);
        }
        // dP^T of the pair (its products were issued after S^T's)
        if (!warp_wait(dp_full + bb, (t >> 1) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t dpv[32];
        tmem_ld32(tmem + lane_off + cDP + 32 * wg, dpv);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float4 Dv = dv4[e >> 1];
          const uint64_t nd = (e & 1) ? f2(-Dv.z, -Dv.w) : f2(-Dv.x, -Dv.y);
          const uint64_t g2 = f2_add(f2(__uint_as_float(dpv[2 * e]), __uint_as_float(dpv[2 * e + 1])), nd);
          float g0, g1;
          f2_split(f2_fma(pp[e], g2, f2(0.f, 0.f)), g0, g1);
          dsk[e] = pack_bf16x2(g0, g1);
        }
      }
      // dS row r: 64 queries = one 128-byte row of the query-major tile; this warpgroup's 32
      // queries are units 4 wg .. 4 wg + 3 (stored at u ^ (r % 8))
      {
        uint8_t* row = sDS + bb * C::kDSTile + r * 128;
#pragma unroll
        for (int u = 0; u < 4; ++u)
          *reinterpret_cast<uint4*>(row + (((4 * wg + u) ^ (r & 7)) << 4)) =
              make_uint4(dsk[4 * u], dsk[4 * u + 1], dsk[4 * u + 2], dsk[4 * u + 3]);
      }
      // P^T and dS^T of this warpgroup's 32 queries go over the 32 S columns it has just read
      // (P^T in the first 16, dS^T in the next 16), so no other warpgroup is waited for
      tmem_st16(tmem + lane_off + cS + 32 * wg, pk);
      tmem_st16(tmem + lane_off + cS + 32 * wg + 16, dsk);
      tmem_wait_st();
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(pds_ready + bb);
      if (t >= 1 && !read_dq(t - 1)) {
        ok = false;
        break;
      }
    }
    if (ok && T > 0) ok = read_dq(T - 1);
    // ---- epilogue: dV (warpgroup 0) and dK = scale * acc (warpgroup 1), rows of this key tile
    const bool have = T > 0 && ok && warp_wait(acc_done, 0);
    tc_fence_after();
    __nv_bfloat16* dst = (wg ? p.dk : p.dv) + (((size_t)sq.rowk + key) * p.Hkv + kvh) * D;
    const float mul = wg ? p.scale : 1.f;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t a[32];
      if (have) {
        tmem_ld32(tmem + lane_off + (wg ? C::kColDK : C::kColDV) + 32 * c, a);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) a[e] = 0u;
      }
      if (key_ok) {
        uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          d4[e] = make_uint4(pack_bf16x2(__uint_as_float(a[8 * e]) * mul, __uint_as_float(a[8 * e + 1]) * mul),
                             pack_bf16x2(__uint_as_float(a[8 * e + 2]) * mul, __uint_as_float(a[8 * e + 3]) * mul),
                             pack_bf16x2(__uint_as_float(a[8 * e + 4]) * mul, __uint_as_float(a[8 * e + 5]) * mul),
                             pack_bf16x2(__uint_as_float(a[8 * e + 6]) * mul, __uint_as_float(a[8 * e + 7]) * mul));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fa
