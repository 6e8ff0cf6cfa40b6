// Split-KV decode kernels for sm_100a.
//
// One new query token per sequence attends to its whole KV cache ("LLM basics: from
// Attention to FlashAttention", chapter 2 section 4: decode reads every cached K, V and is
// memory-bound).  The cache is cut into splits; each CTA streams one split of one
// (sequence, KV head) and produces, for every query head of that KV head's group
// (chapter 2 section 7), the partial statistics (m_s, l_s) and the un-normalised
// accumulator acc_s = sum_j 2^(t_j - m_s) v_j.  A second kernel merges the splits with the
// rule of "FlashAttention notes" section 4 (m = max m_s, l = sum 2^(m_s - m) l_s, and the
// accumulators with the same weights) ("FlashAttention-3 (FA-3)", section 4, FlashDecoding).
// (Merging in the split kernel instead, by the last CTA of each (sequence, KV head) to finish,
// measured slower: those merges run serially at the end of the grid, while the combine kernel
// spreads them over all SMs.)
//
// Paged caches ("LLM basics: from Attention to FlashAttention", chapter 2 section 8,
// PagedAttention): the cache is a pool of fixed-size pages, and a per-sequence block table
// maps logical page t / page_size of a sequence to a physical page, so token t sits at row
// t % page_size of that page.  The paged kernel fetches each 64-row stage as whole pages
// (or one 64-row part of a larger page) through the table.
//
// The split kernel is bound by HBM bandwidth: K and V are read once.  Tiles of 64 cache rows
// arrive by TMA (128-byte swizzle, evict-first) in a 3- or 4-stage ring fed by a producer
// warp; four compute warps each take 16 of the 64 rows.  The G <= 16 query heads of the
// group form the M = 16 side of bf16 m16n8k16 tensor-core products, so the small products
// S = q K^T and acc += P V run on tensor cores while the kernel waits on memory.
#pragma once

#include "fa_device.cuh"

namespace fa {

struct DecParams {
  const __nv_bfloat16* q;
  const int32_t* seqlens;  // [B] or null (all Lmax)
  __nv_bfloat16* o;
  float* lse;
  float* ws_acc;  // [B, Hq, nsplit, D]
  float* ws_ml;   // [B, Hq, nsplit, 2]  (m in base-2 units, l)
  // paged caches only
  const int32_t* block_table;  // [B, max_pages]
  int max_pages, page_shift, page_box, num_pages;
  int B, Hq, Hkv, G, Lmax, split_len, nsplit;
  float tau;
};


constexpr int kDecKeys = 64;  // cache rows per stage
constexpr int kDecComputeWarps = 4;
constexpr int kDecThreads = (kDecComputeWarps + 1) * 32;

template <int D>
struct DecCfg {
  static constexpr int kPanelBytes = kDecKeys * 128;   // 64 rows x 64 bf16
  static constexpr int kHalfBytes = kDecKeys * D * 2;  // the K (or V) part of a stage
  static constexpr int kStageBytes = 2 * kHalfBytes;
  static constexpr int kStages = (D == 128) ? 3 : 4;
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + 2 * kStages * 8 + 64;
  static_assert(kStages * kStageBytes >= (kDecComputeWarps * 16 * D + 2 * kDecComputeWarps * 16 + 32) * 4,
                "the merge scratch must fit in the ring");
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Byte offset of (row, column) in a tile stored as 64-column panels of 128-byte rows with
// the 128-byte swizzle (16-byte unit u of row r lives at unit u ^ (r % 8)).
__device__ __forceinline__ uint32_t sw128_offset(int row, int col, int panel_bytes) {
  const int panel = col >> 6;
  const int unit = (col & 63) >> 3;
  return panel * panel_bytes + row * 128 + ((unit ^ (row & 7)) << 4) + ((col & 7) << 1);
}

__device__ __forceinline__ int dec_seqlen(const DecParams& p, int b) {
  int L = p.seqlens ? __ldg(p.seqlens + b) : p.Lmax;
  return max(0, min(L, p.Lmax));
}

// PAGED = false: contiguous caches [B, Lmax, Hkv, D].  PAGED = true: page pool
// [num_pages, page_size, Hkv, D] through the block table.  Either way the partial of every
// split goes to the workspace and fa_decode_combine_kernel merges them.
template <int D, bool PAGED>
__global__ void __launch_bounds__(kDecThreads)
    fa_decode_split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                           const DecParams p) {
  using C = DecCfg<D>;
  constexpr int NS = C::kStages;
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int seqlen = dec_seqlen(p, b);
  const int key_begin = split * p.split_len;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.G;
  const int h0 = kvh * G;
  if (key_begin >= seqlen) return;  // empty split: the combine kernel never reads it
  const int nkeys = min(p.split_len, seqlen - key_begin);
  const int nst = (nkeys + kDecKeys - 1) / kDecKeys;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + NS * C::kStageBytes);
  uint64_t* empty = full + NS;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, kDecComputeWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kDecComputeWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      const uint64_t pol = policy_evict_first();
      const int row_base = b * p.Lmax + key_begin;
      // paged: page_box = min(page_size, 64) rows per copy, so a stage takes at most four
      // copies and no copy straddles a page.  Copies past the sequence end re-read its last
      // page (those rows are masked and their V rows zeroed before use).  The block-table
      // entries of stage s + 1 are loaded while stage s is waited for and issued, so the
      // table's latency stays off the copy stream.
      const int box = PAGED ? p.page_box : kDecKeys;
      const int ps = PAGED ? (1 << p.page_shift) : 1;
      auto stage_tok = [&](int s, int t) {
        const int tok = key_begin + s * kDecKeys + t;
        return tok < seqlen ? tok : ((seqlen - 1) & ~(box - 1));
      };
      const int* bt = PAGED ? p.block_table + (size_t)b * p.max_pages : nullptr;
      int pages[4] = {0, 0, 0, 0};
      if (PAGED) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (k * box < kDecKeys) pages[k] = __ldg(bt + (stage_tok(0, k * box) >> p.page_shift));
      }
      for (int s = 0; s < nst; ++s) {
        const int cur[4] = {pages[0], pages[1], pages[2], pages[3]};
        if (PAGED && s + 1 < nst) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            if (k * box < kDecKeys) pages[k] = __ldg(bt + (stage_tok(s + 1, k * box) >> p.page_shift));
        }
        const int slot = s % NS;
        if (s >= NS && !mbar_wait(empty + slot, ((s / NS) - 1) & 1)) break;
        mbar_arrive_expect_tx(full + slot, C::kStageBytes);
        uint8_t* st = ring + slot * C::kStageBytes;
        if (!PAGED) {
          for (int c = 0; c < D / 64; ++c) {
            tma_load_3d_hint(st + c * C::kPanelBytes, &tmK, c * 64, kvh, row_base + s * kDecKeys, full + slot, pol);
            tma_load_3d_hint(st + C::kHalfBytes + c * C::kPanelBytes, &tmV, c * 64, kvh, row_base + s * kDecKeys,
                             full + slot, pol);
          }
        } else {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int t = k * box;
            if (t >= kDecKeys) break;
            const int tok = stage_tok(s, t);
            int page = cur[k];
            if (page < 0 || page >= p.num_pages) {
              atomicOr(&g_error_word, kErrBadPage);
              page = 0;
            }
            const int row = page * ps + (tok & (ps - 1));
            for (int c = 0; c < D / 64; ++c) {
              tma_load_3d_hint(st + c * C::kPanelBytes + t * 128, &tmK, c * 64, kvh, row, full + slot, pol);
              tma_load_3d_hint(st + C::kHalfBytes + c * C::kPanelBytes + t * 128, &tmV, c * 64, kvh, row,
                               full + slot, pol);
            }
          }
        }
      }
    }
    return;  // the producer takes no part in the merge below
  }

  // -------------------------------------------------------------- compute warps
  const int g = lane >> 2, tig = lane & 3;
  // A fragments of q (rows = the group's query heads, zero beyond G)
  uint32_t qa[D / 16][4];
  {
    const uint32_t* q32 = reinterpret_cast<const uint32_t*>(p.q + ((size_t)b * p.Hq + h0) * D);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int c0 = kk * 16 + 2 * tig;
      qa[kk][0] = (g < G) ? __ldg(q32 + (g * D + c0) / 2) : 0u;
      qa[kk][1] = (g + 8 < G) ? __ldg(q32 + ((g + 8) * D + c0) / 2) : 0u;
      qa[kk][2] = (g < G) ? __ldg(q32 + (g * D + c0 + 8) / 2) : 0u;
      qa[kk][3] = (g + 8 < G) ? __ldg(q32 + ((g + 8) * D + c0 + 8) / 2) : 0u;
    }
  }
  float acc[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
  const float tau = p.tau;
  const int key_lo = 16 * warp;  // this warp's 16 rows within each 64-row stage
  const int mi = lane >> 3, rr = lane & 7;
  bool ok = true;

  for (int s = 0; s < nst; ++s) {
    const int slot = s % NS;
    if (!mbar_wait(full + slot, (s / NS) & 1)) {
      ok = false;
      break;
    }
    const uint32_t kb = smem_u32(ring + slot * C::kStageBytes);
    const uint32_t vb = kb + C::kHalfBytes;
    float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t b0, b1, b2, b3;
      const int key = key_lo + (mi >> 1) * 8 + rr;
      const int col = kk * 16 + (mi & 1) * 8;
      ldsm_x4(kb + sw128_offset(key, col, C::kPanelBytes), b0, b1, b2, b3);
      mma_bf16_16816(sc[0], qa[kk], b0, b1);
      mma_bf16_16816(sc[1], qa[kk], b2, b3);
    }
    // Mask rows of the cache at or beyond the sequence length, and zero their V rows: those
    // rows are unused cache slots whose contents are arbitrary (0 * NaN would poison O).
    // Each warp reads only its own 16 V rows, so a warp-local barrier orders the zeroing.
    const int kglob0 = key_begin + s * kDecKeys + key_lo;
    if (kglob0 + 16 > seqlen) {
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (kglob0 + nt * 8 + 2 * tig + (e & 1) >= seqlen) sc[nt][e] = -INFINITY;
      uint8_t* vrows = ring + slot * C::kStageBytes + C::kHalfBytes;
#pragma unroll
      for (int u = lane; u < 16 * (D / 64) * 8; u += 32) {
        const int r = u & 15, c = u >> 4;  // row within the warp's 16, 16-byte unit of the row
        if (kglob0 + r >= seqlen)
          *reinterpret_cast<uint4*>(vrows + (c >> 3) * C::kPanelBytes + (key_lo + r) * 128 + (c & 7) * 16) =
              make_uint4(0u, 0u, 0u, 0u);
      }
      __syncwarp();
    }
    // online softmax update for rows g (e = 0, 1) and g + 8 (e = 2, 3)
    float alpha[2], ms[2];
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      float mx = fmaxf(fmaxf(sc[0][2 * hr], sc[0][2 * hr + 1]), fmaxf(sc[1][2 * hr], sc[1][2 * hr + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m_r[hr], mx * tau);
      alpha[hr] = (m_r[hr] == -INFINITY) ? 0.f : ex2_approx(m_r[hr] - m_new);
      if (m_new == -INFINITY) alpha[hr] = 1.f;
      m_r[hr] = m_new;
      ms[hr] = (m_new == -INFINITY) ? 0.f : m_new;
    }
    float pr[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) pr[nt][e] = ex2_approx(fmaf(sc[nt][e], tau, -ms[e >> 1]));
#pragma unroll
    for (int hr = 0; hr < 2; ++hr)
      l_r[hr] = l_r[hr] * alpha[hr] + pr[0][2 * hr] + pr[0][2 * hr + 1] + pr[1][2 * hr] + pr[1][2 * hr + 1];
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      acc[n][0] *= alpha[0];
      acc[n][1] *= alpha[0];
      acc[n][2] *= alpha[1];
      acc[n][3] *= alpha[1];
    }
    const uint32_t pa[4] = {pack_bf16x2(pr[0][0], pr[0][1]), pack_bf16x2(pr[0][2], pr[0][3]),
                            pack_bf16x2(pr[1][0], pr[1][1]), pack_bf16x2(pr[1][2], pr[1][3])};
#pragma unroll
    for (int qd = 0; qd < D / 16; ++qd) {
      uint32_t b0, b1, b2, b3;
      const int key = key_lo + (mi & 1) * 8 + rr;
      const int col = qd * 16 + (mi >> 1) * 8;
      ldsm_x4_t(vb + sw128_offset(key, col, C::kPanelBytes), b0, b1, b2, b3);
      mma_bf16_16816(acc[2 * qd], pa, b0, b1);
      mma_bf16_16816(acc[2 * qd + 1], pa, b2, b3);
    }
    // The slot is refilled by TMA (the async proxy) once every warp has arrived.  The warp's
    // ldmatrix reads of it are generic-proxy accesses, so a cross-proxy fence orders them
    // before that refill; without it a refill was seen to overwrite V while a warp still
    // read it (two CTAs per SM, about one run in a few hundred).
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
    if (lane == 0) mbar_arrive(empty + slot);
  }

  // row sums over the quad
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    l_r[hr] += __shfl_xor_sync(0xffffffffu, l_r[hr], 1);
    l_r[hr] += __shfl_xor_sync(0xffffffffu, l_r[hr], 2);
  }

  // merge the four warps' partials through shared memory (the ring is free now: every
  // stage was consumed and the producer issues nothing more)
  asm volatile("bar.sync 1, %0;" ::"n"(kDecComputeWarps * 32) : "memory");
  float* sm_o = reinterpret_cast<float*>(ring);                  // [4][16][D]
  float* sm_m = sm_o + kDecComputeWarps * 16 * D;                // [4][16]
  float* sm_l = sm_m + kDecComputeWarps * 16;                    // [4][16]
  {
    float* ow = sm_o + warp * 16 * D;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      const int col = n * 8 + 2 * tig;
      ow[g * D + col] = acc[n][0];
      ow[g * D + col + 1] = acc[n][1];
      ow[(g + 8) * D + col] = acc[n][2];
      ow[(g + 8) * D + col + 1] = acc[n][3];
    }
    if (tig == 0) {
      sm_m[warp * 16 + g] = ok ? m_r[0] : -INFINITY;
      sm_m[warp * 16 + g + 8] = ok ? m_r[1] : -INFINITY;
      sm_l[warp * 16 + g] = l_r[0];
      sm_l[warp * 16 + g + 8] = l_r[1];
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kDecComputeWarps * 32) : "memory");
  const size_t part0 = ((size_t)b * p.Hq + h0) * p.nsplit + split;  // partial of head h0
  for (int idx = threadIdx.x; idx < G * (D / 4); idx += kDecComputeWarps * 32) {
    const int row = idx / (D / 4), col = 4 * (idx - row * (D / 4));
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecComputeWarps; ++w) M = fmaxf(M, sm_m[w * 16 + row]);
    float L = 0.f;
    float4 A = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < kDecComputeWarps; ++w) {
      const float mw = sm_m[w * 16 + row];
      const float e = (mw == -INFINITY) ? 0.f : ex2_approx(mw - M);
      L += e * sm_l[w * 16 + row];
      const float4 x = *reinterpret_cast<const float4*>(sm_o + (w * 16 + row) * D + col);
      A.x += e * x.x;
      A.y += e * x.y;
      A.z += e * x.z;
      A.w += e * x.w;
    }
    const size_t part = part0 + (size_t)row * p.nsplit;
    *reinterpret_cast<float4*>(p.ws_acc + part * D + col) = A;
    if (col == 0) {
      p.ws_ml[part * 2] = M;
      p.ws_ml[part * 2 + 1] = L;
    }
  }
}

// Merge of the splits of one (sequence, query head) per warp.
template <int D>
__global__ void __launch_bounds__(128) fa_decode_combine_kernel(const DecParams p) {
  const int bh = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (bh >= p.B * p.Hq) return;
  const int b = bh / p.Hq;
  const int seqlen = dec_seqlen(p, b);
  const int ns = (seqlen + p.split_len - 1) / p.split_len;
  const size_t base = (size_t)bh * p.nsplit;
  constexpr int V = D / 32;  // columns per lane
  float M = -INFINITY;
  for (int s = lane; s < ns; s += 32) M = fmaxf(M, p.ws_ml[(base + s) * 2]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  float L = 0.f;
  float a[V];
#pragma unroll
  for (int v = 0; v < V; ++v) a[v] = 0.f;
  for (int s = 0; s < ns; ++s) {
    const float ms = p.ws_ml[(base + s) * 2];
    const float e = (ms == -INFINITY) ? 0.f : ex2_approx(ms - M);
    L += e * p.ws_ml[(base + s) * 2 + 1];
    const float* src = p.ws_acc + (base + s) * D + lane * V;
    if (V == 4) {
      const float4 x = *reinterpret_cast<const float4*>(src);
      a[0] += e * x.x;
      a[1] += e * x.y;
      a[2] += e * x.z;
      a[3] += e * x.w;
    } else {
#pragma unroll
      for (int v = 0; v < V; ++v) a[v] += e * src[v];
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  __nv_bfloat16* dst = p.o + (size_t)bh * D + lane * V;
#pragma unroll
  for (int v = 0; v < V; v += 2) *reinterpret_cast<uint32_t*>(dst + v) = pack_bf16x2(a[v] * inv, a[v + 1] * inv);
  if (lane == 0 && p.lse != nullptr) p.lse[bh] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
}

}  // namespace fa
