// Host side of the C ABI declared in include/fa.h: argument checks, TMA descriptors,
// workspace carving and kernel launches.  No device memory is allocated here.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/fa.h"
#include "fa_bwd_sm100.cuh"
#include "fa_decode_sm100.cuh"
#include "fa_fwd_sm100.cuh"

namespace fa {

// fp32 -> bf16 (round to nearest even), used when the forward is called with fp32 inputs.
__global__ void cast_f32_bf16_kernel(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst, size_t n) {
  const size_t n4 = n / 4;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
    const float4 x = reinterpret_cast<const float4*>(src)[i];
    uint2 w;
    w.x = pack_bf16x2(x.x, x.y);
    w.y = pack_bf16x2(x.z, x.w);
    reinterpret_cast<uint2*>(dst)[i] = w;
  }
  for (size_t i = n4 * 4 + (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
    dst[i] = __float2bfloat16_rn(src[i]);
}

// V^T for the fp8 forward: vt[(b*Hkv + h)*128 + c][n] = v[b][n][h][c] for n < Nk, 0 up to
// NkPad (so that padded keys hold finite values; they are masked).  One block per (64-key
// chunk, head, sequence), staged through shared memory so both sides are coalesced.
__global__ void __launch_bounds__(256) transpose_v_e4m3_kernel(const uint8_t* __restrict__ v, uint8_t* __restrict__ vt,
                                                               int Nk, int Hkv, int NkPad) {
  __shared__ uint32_t tile[64][33];  // 64 keys x 128 bytes (32 words), padded
  const int n0 = blockIdx.x * 64, h = blockIdx.y, b = blockIdx.z;
  for (int idx = threadIdx.x; idx < 64 * 32; idx += 256) {
    const int r = idx >> 5, w = idx & 31;
    const int n = n0 + r;
    tile[r][w] = (n < Nk) ? reinterpret_cast<const uint32_t*>(v + (((size_t)b * Nk + n) * Hkv + h) * 128)[w] : 0u;
  }
  __syncthreads();
  // each thread writes 4 consecutive keys (one word) of one column c
  for (int idx = threadIdx.x; idx < 128 * 16; idx += 256) {
    const int c = idx >> 4, kq = idx & 15;  // column, group of four keys
    const int n = n0 + 4 * kq;
    if (n >= NkPad) continue;
    uint32_t word = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) word |= ((tile[4 * kq + e][c >> 2] >> (8 * (c & 3))) & 0xFFu) << (8 * e);
    *reinterpret_cast<uint32_t*>(vt + (((size_t)b * Hkv + h) * 128 + c) * NkPad + n) = word;
  }
}

// fp32 -> the nearest tf32 value (10 mantissa bits, ties to even), kept in fp32 storage.
// Integer rounding on the bit pattern; infinities and NaN pass through.
__device__ __forceinline__ float round_tf32(float x) {
  uint32_t u = __float_as_uint(x);
  if ((u & 0x7F800000u) != 0x7F800000u) {
    u += 0x0FFFu + ((u >> 13) & 1u);
    u &= ~0x1FFFu;
  }
  return __uint_as_float(u);
}

__global__ void round_tf32_kernel(const float* __restrict__ src, float* __restrict__ dst, size_t n) {
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) dst[i] = round_tf32(src[i]);
}

// V^T for the tf32 forward (d = 64, fp32, rounded to tf32): vt[(b*Hkv + h)*64 + c][n] =
// v[b][n][h][c] for n < Nk, 0 up to NkPad.  One block per (32-key chunk, head, sequence).
__global__ void __launch_bounds__(256) transpose_v_f32_kernel(const float* __restrict__ v, float* __restrict__ vt,
                                                              int Nk, int Hkv, int NkPad) {
  __shared__ float tile[32][65];
  const int n0 = blockIdx.x * 32, h = blockIdx.y, b = blockIdx.z;
  for (int idx = threadIdx.x; idx < 32 * 64; idx += 256) {
    const int r = idx >> 6, c = idx & 63;
    const int n = n0 + r;
    tile[r][c] = (n < Nk) ? round_tf32(v[(((size_t)b * Nk + n) * Hkv + h) * 64 + c]) : 0.f;
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < 64 * 32; idx += 256) {
    const int c = idx >> 5, r = idx & 31;
    const int n = n0 + r;
    if (n < NkPad) vt[(((size_t)b * Hkv + h) * 64 + c) * NkPad + n] = tile[r][c];
  }
}

// Reads and clears the error word in one atomic step, so that a record made by a kernel on
// another stream between a read and a separate clear cannot be lost.
__global__ void take_error_word_kernel() { g_error_taken = atomicExch(&g_error_word, 0u); }

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// [rows, heads, D] bf16 tensor (D innermost) seen as a 3-D map {D, heads, rows}; box of
// 64 columns x 1 head x box_rows rows with the 128-byte swizzle.  Consecutive rows are
// row_stride elements apart (heads * D when the tensor is dense; 3 * heads * D for one of
// q, k, v inside a packed [rows, 3, heads, D] tensor).
bool make_map(CUtensorMap* map, const void* base, int D, int heads, int64_t rows, int box_rows,
              int64_t row_stride = 0) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  if (row_stride <= 0) row_stride = (int64_t)heads * D;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)row_stride * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Byte tensor (e4m3 stored as bytes) of three dimensions with the 128-byte swizzle.
bool make_map_u8(CUtensorMap* map, const void* base, const cuuint64_t (&dims)[3], const cuuint64_t (&strides)[2],
                 const cuuint32_t (&box)[3]) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 tensor of three dimensions with the 128-byte swizzle (box inner extent 32 elements).
bool make_map_f32(CUtensorMap* map, const void* base, const cuuint64_t (&dims)[3], const cuuint64_t (&strides)[2],
                  const cuuint32_t (&box)[3]) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Dense bf16 output [rows, heads, D] as the TMA store target of the forward epilogue: box of
// 16 columns x 1 head x 32 rows (one softmax warp's rows) with the 32-byte swizzle.
bool make_map_o(CUtensorMap* map, const void* base, int D, int heads, int64_t rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc || rows <= 0 || (reinterpret_cast<uintptr_t>(base) & 15u) != 0) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)heads * D * 2};
  cuuint32_t box[3] = {16, 1, 32};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Work units of the forward: 256 query rows of one head, or, at fixed length when the query
// heads of every K/V group come in pairs, 128 rows of two heads of one group: both tiles of a
// unit then see the same keys, so a causal unit has no step with one tile (8K GQA causal:
// 1259 -> 1286 TFLOP/s, FP8 1415 -> 1473, same box).  Packed varlen inputs keep 256-row
// units (measured 1124 against 1114 TFLOP/s with pairs on the 16-sequence workload; the
// kernel supports both).  Sets prm.hpair and prm.T; returns the number of units (fixed
// length) or 0 (varlen: counted on the device).
int64_t fwd_units(FwdParams& prm, bool varlen, int64_t rows_q) {
  (void)rows_q;
  prm.hpair = (prm.G % 2 == 0 && !varlen) ? 1 : 0;
  const int ur = kUnitRows >> prm.hpair;
  prm.T = varlen ? 0 : (prm.Nq + ur - 1) / ur;
  return varlen ? 0 : (int64_t)prm.T * prm.B * (prm.Hq >> prm.hpair);
}

int sm_count_cached() {
  static int counts[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (counts[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    counts[dev] = n;
  }
  return counts[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

template <class K>
cudaError_t set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <int D, bool F32>
fa_status launch_fwd(const void* q, const void* k, const void* v, const FwdParams& prm, int64_t rows_q,
                     int64_t rows_k, int units, cudaStream_t st, int64_t q_stride = 0, int64_t kv_stride = 0) {
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, D, prm.Hq, rows_q, kBM, q_stride) || !make_map(&mk, k, D, prm.Hkv, rows_k, kBN, kv_stride) ||
      !make_map(&mv, v, D, prm.Hkv, rows_k, kBN, kv_stride))
    return FA_ERR_CUDA;
  // bf16 O goes out through TMA stores when it can be described (16-byte aligned base); the
  // kernel writes per lane otherwise (and always for fp32 O)
  FwdParams p2 = prm;
  CUtensorMap mo = mq;
  p2.o_tma = (!F32 && make_map_o(&mo, prm.o, D, prm.Hq, rows_q)) ? 1 : 0;
  auto kern = fa_fwd_kernel<D, F32>;
  const int smem = FwdCfg<D>::kSmemBytes;
  if (set_smem(kern, smem) != cudaSuccess) return FA_ERR_CUDA;
  const int sms = sm_count_cached();
  if (sms <= 0) return FA_ERR_CUDA;
  const int grid = (units > 0) ? std::min(units, sms) : sms;
  kern<<<grid, kFwdThreads, smem, st>>>(mq, mk, mv, mo, p2);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <int D>
fa_status launch_decode(const void* kc, const void* vc, const DecParams& prm, cudaStream_t st) {
  CUtensorMap mk, mv;
  const int64_t rows = (int64_t)prm.B * prm.Lmax;
  if (!make_map(&mk, kc, D, prm.Hkv, rows, kDecKeys) || !make_map(&mv, vc, D, prm.Hkv, rows, kDecKeys))
    return FA_ERR_CUDA;
  auto ks = fa_decode_split_kernel<D, false>;
  const int smem = DecCfg<D>::kSmemBytes;
  if (set_smem(ks, smem) != cudaSuccess) return FA_ERR_CUDA;
  dim3 grid(prm.nsplit, prm.Hkv, prm.B);
  ks<<<grid, kDecThreads, smem, st>>>(mk, mv, prm);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  const int nbh = prm.B * prm.Hq;
  fa_decode_combine_kernel<D><<<(nbh + 3) / 4, 128, 0, st>>>(prm);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <int D>
fa_status launch_decode_paged(const void* kp, const void* vp, const DecParams& prm, cudaStream_t st) {
  CUtensorMap mk, mv;
  const int64_t rows = (int64_t)prm.num_pages << prm.page_shift;
  if (!make_map(&mk, kp, D, prm.Hkv, rows, prm.page_box) || !make_map(&mv, vp, D, prm.Hkv, rows, prm.page_box))
    return FA_ERR_CUDA;
  auto ks = fa_decode_split_kernel<D, true>;
  const int smem = DecCfg<D>::kSmemBytes;
  if (set_smem(ks, smem) != cudaSuccess) return FA_ERR_CUDA;
  dim3 grid(prm.nsplit, prm.Hkv, prm.B);
  ks<<<grid, kDecThreads, smem, st>>>(mk, mv, prm);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  const int nbh = prm.B * prm.Hq;
  fa_decode_combine_kernel<D><<<(nbh + 3) / 4, 128, 0, st>>>(prm);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// Fixed length (prm.cu null) or packed varlen rows (prm.cu, prm.total, prm.ntiles set).
template <int D>
fa_status launch_bwd(const void* q, const void* k, const void* v, const BwdParams& prm, cudaStream_t st) {
  CUtensorMap mq, mk, mv, mdo;
  const bool varlen = prm.cu != nullptr;
  const int64_t rows_q = varlen ? (int64_t)prm.total : (int64_t)prm.B * prm.Nq;
  const int64_t rows_k = varlen ? (int64_t)prm.total : (int64_t)prm.B * prm.Nk;
  if (!make_map(&mq, q, D, prm.Hq, rows_q, kBwdTile) || !make_map(&mdo, prm.dout, D, prm.Hq, rows_q, kBwdTile) ||
      !make_map(&mk, k, D, prm.Hkv, rows_k, kBwdTile) || !make_map(&mv, v, D, prm.Hkv, rows_k, kBwdTile))
    return FA_ERR_CUDA;
  const int sms = sm_count_cached();
  if (sms <= 0) return FA_ERR_CUDA;
  if (varlen) fa_bwd_tiles_kernel<<<1, kTilesThreads, 0, st>>>(prm);
  const long long pre_rows =
      varlen ? (long long)prm.Hq * prm.ntiles * kBwdTile : (long long)prm.B * prm.Hq * prm.NqPad;
  const int pre_blocks = (int)std::min<long long>((pre_rows + 7) / 8, (long long)sms * 16);
  if (pre_blocks > 0) fa_bwd_pre_kernel<D><<<pre_blocks, 256, 0, st>>>(prm);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  if (rows_k > 0 && (varlen || prm.Nk > 0)) {
    // one CTA per (key tile, K/V head, sequence), tile-major (the kernels' bwd_cta_coords);
    // varlen: a tile number over all sequences (bounded by ntiles; the kernels find the
    // sequence and leave numbers past the last tile idle)
    const long long ctas = varlen ? (long long)prm.ntiles * prm.Hkv
                                  : (long long)((prm.Nk + kBwdTile - 1) / kBwdTile) * prm.Hkv * prm.B;
    if (ctas >= (1ll << 31)) return FA_ERR_UNSUPPORTED;
    const dim3 grid((unsigned)ctas);
    if (D == 128) {
      // pairs of 64 queries, two in flight: Q and dO maps with 64-row boxes
      CUtensorMap mq64, mdo64;
      if (!make_map(&mq64, q, D, prm.Hq, rows_q, kBwdQ) || !make_map(&mdo64, prm.dout, D, prm.Hq, rows_q, kBwdQ))
        return FA_ERR_CUDA;
      // the fp32 dQ accumulator as a TMA reduce target: {d, Hq, rows}, box 128 x 1 x 64, no swizzle
      CUtensorMap mdq;
      const cuuint64_t ddq[3] = {(cuuint64_t)D, (cuuint64_t)prm.Hq, (cuuint64_t)rows_q};
      const cuuint64_t sdq[2] = {(cuuint64_t)D * 4, (cuuint64_t)prm.Hq * D * 4};
      const cuuint32_t bdq[3] = {(cuuint32_t)D, 1, (cuuint32_t)kBwdQ};
      const cuuint32_t edq[3] = {1, 1, 1};
      EncodeTiledFn enc = get_encode_fn();
      if (!enc || enc(&mdq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, prm.dq_acc, ddq, sdq, bdq, edq,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return FA_ERR_CUDA;
      const int smem = Bwd2Cfg::kSmemBytes;
      if (set_smem(fa_bwd2_kernel, smem) != cudaSuccess) return FA_ERR_CUDA;
      fa_bwd2_kernel<<<grid, kBwdThreads, smem, st>>>(mq64, mk, mv, mdo64, mdq, prm);
    } else {
      auto kern = fa_bwd_kernel<D>;
      const int smem = BwdCfg<D>::kSmemBytes;
      if (set_smem(kern, smem) != cudaSuccess) return FA_ERR_CUDA;
      kern<<<grid, kBwdThreads, smem, st>>>(mq, mk, mv, mdo, prm);
    }
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  const size_t n4 = (size_t)rows_q * prm.Hq * D / 4;
  if (n4 > 0) fa_bwd_dq_kernel<D><<<(int)std::min<size_t>((n4 + 255) / 256, (size_t)sms * 8), 256, 0, st>>>(prm);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace
}  // namespace fa

using namespace fa;

extern "C" {

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported configuration";
    case FA_ERR_WORKSPACE: return "workspace missing or too small";
    case FA_ERR_CUDA: return "CUDA error";
    case FA_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

int fa_device_sm_count(void) { return sm_count_cached(); }

size_t fa_fwd_workspace_size(int B, int Hq, int Hkv, int Nq, int Nk, int d, fa_dtype in_dtype, int varlen) {
  if (in_dtype == FA_TF32) {
    // tf32-rounded copies of q and k, then the rounded, transposed v
    if (varlen || B <= 0 || Hq <= 0 || Hkv <= 0 || Nq < 0 || Nk < 0 || d != 64) return 0;
    const size_t pad = (size_t)(Nk + 3) / 4 * 4;
    return align_up((size_t)B * Nq * Hq * d * 4, 256) + align_up((size_t)B * Nk * Hkv * d * 4, 256) +
           align_up((size_t)B * Hkv * d * pad * 4, 256);
  }
  if (in_dtype != FA_F32) return 0;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq < 0 || Nk < 0 || d <= 0) return 0;
  // bf16 copies of q, k, v (varlen: Nq = Nk = the packed row count)
  const size_t rq = varlen ? (size_t)Nq : (size_t)B * Nq, rk = varlen ? (size_t)Nk : (size_t)B * Nk;
  const size_t nq = rq * Hq * d, nk = rk * Hkv * d;
  return align_up(nq * 2, 256) + 2 * align_up(nk * 2, 256);
}

}  // extern "C"

namespace fa {
namespace {

// fp32 q, k, v (d = 64, fixed length) on the tf32 tensor-core path; O written as fp32.
fa_status fwd_tf32(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Nq,
                   int Nk, float scale, int causal, void* workspace, size_t workspace_bytes, cudaStream_t st) {
  constexpr int D = 64;
  const int64_t rows_q = (int64_t)B * Nq, rows_k = (int64_t)B * Nk;
  const int pad = (Nk + 3) / 4 * 4;
  const size_t need = fa_fwd_workspace_size(B, Hq, Hkv, Nq, Nk, D, FA_TF32, 0);
  if (need > 0 && (!workspace || workspace_bytes < need || !aligned16(workspace))) return FA_ERR_WORKSPACE;
  if (B > 65535 || Hkv > 65535) return FA_ERR_UNSUPPORTED;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t nq = (size_t)rows_q * Hq * D, nk = (size_t)rows_k * Hkv * D;
  float* qr = reinterpret_cast<float*>(ws);
  float* kr = reinterpret_cast<float*>(ws + align_up(nq * 4, 256));
  float* vt = reinterpret_cast<float*>(ws + align_up(nq * 4, 256) + align_up(nk * 4, 256));
  const int sms0 = std::max(sm_count_cached(), 1);
  round_tf32_kernel<<<sms0 * 4, 256, 0, st>>>(static_cast<const float*>(q), qr, nq);
  if (Nk > 0) {
    round_tf32_kernel<<<sms0 * 4, 256, 0, st>>>(static_cast<const float*>(k), kr, nk);
    dim3 g((pad + 31) / 32, Hkv, B);
    transpose_v_f32_kernel<<<g, 256, 0, st>>>(static_cast<const float*>(v), vt, Nk, Hkv, pad);
  }
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  FwdParams prm{};
  prm.o = o;
  prm.lse = lse;
  prm.cu = nullptr;
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.G = Hq / Hkv;
  prm.Nq = Nq;
  prm.Nk = Nk;
  prm.causal = causal ? 1 : 0;
  prm.tau = (float)((double)scale * 1.4426950408889634074);
  prm.o_scale = 1.f;
  const int64_t units64 = fwd_units(prm, false, rows_q);
  if (units64 >= (int64_t(1) << 31)) return FA_ERR_UNSUPPORTED;
  CUtensorMap mq, mk, mv;
  const cuuint64_t dq3[3] = {D, (cuuint64_t)Hq, (cuuint64_t)rows_q};
  const cuuint64_t sq2[2] = {D * 4, (cuuint64_t)Hq * D * 4};
  const cuuint64_t dk3[3] = {D, (cuuint64_t)Hkv, (cuuint64_t)std::max<int64_t>(rows_k, 1)};
  const cuuint64_t sk2[2] = {D * 4, (cuuint64_t)Hkv * D * 4};
  const int vp = std::max(pad, 4);
  const cuuint64_t dv3[3] = {(cuuint64_t)vp, D, (cuuint64_t)B * Hkv};
  const cuuint64_t sv2[2] = {(cuuint64_t)vp * 4, (cuuint64_t)vp * 4 * D};
  const cuuint32_t box_rows[3] = {32, 1, (cuuint32_t)kBM};
  const cuuint32_t box_vt[3] = {32, D, 1};
  if (!make_map_f32(&mq, qr, dq3, sq2, box_rows) || !make_map_f32(&mk, Nk > 0 ? kr : qr, dk3, sk2, box_rows) ||
      !make_map_f32(&mv, Nk > 0 ? (const void*)vt : qr, dv3, sv2, box_vt))
    return FA_ERR_CUDA;
  auto kern = fa_fwd_kernel<D, true, kKindTF32>;
  const int smem = FwdCfg<D, kKindTF32>::kSmemBytes;
  if (set_smem(kern, smem) != cudaSuccess) return FA_ERR_CUDA;
  const int sms = sm_count_cached();
  if (sms <= 0) return FA_ERR_CUDA;
  kern<<<std::min((int)units64, sms), kFwdThreads, smem, st>>>(mq, mk, mv, mq, prm);  // fp32 O: per-lane stores
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace
}  // namespace fa

extern "C" {

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Nq,
                 int Nk, int d, float scale, int causal, const int32_t* cu_seqlens, fa_dtype in_dtype,
                 void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !o) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return FA_ERR_INVALID_ARG;
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Nq < 0 || Nk < 0) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (in_dtype != FA_BF16 && in_dtype != FA_F32 && in_dtype != FA_TF32) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (in_dtype == FA_TF32 && (d != 64 || cu_seqlens != nullptr)) return FA_ERR_UNSUPPORTED;
  const bool varlen = cu_seqlens != nullptr;
  if (varlen) {
    if (Nq != Nk) return FA_ERR_INVALID_ARG;
    if (B > kMaxVarlenB || (int64_t)Nq > (int64_t)kMaxVarlenT * kUnitRows) return FA_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0) return FA_ERR_INVALID_ARG;
  }
  const int64_t rows_q = varlen ? (int64_t)Nq : (int64_t)B * Nq;
  const int64_t rows_k = varlen ? (int64_t)Nk : (int64_t)B * Nk;
  if (rows_q >= (int64_t(1) << 31) || rows_k >= (int64_t(1) << 31)) return FA_ERR_UNSUPPORTED;
  if (B == 0 || Nq == 0) return FA_OK;

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (in_dtype == FA_TF32) return fwd_tf32(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, causal, workspace,
                                           workspace_bytes, st);
  const void *qb = q, *kb = k, *vb = v;
  if (in_dtype == FA_F32) {
    const size_t need = fa_fwd_workspace_size(B, Hq, Hkv, Nq, Nk, d, in_dtype, varlen ? 1 : 0);
    if (!workspace || workspace_bytes < need || !aligned16(workspace)) return FA_ERR_WORKSPACE;
    const size_t nq = (size_t)rows_q * Hq * d, nk = (size_t)rows_k * Hkv * d;
    uint8_t* w = static_cast<uint8_t*>(workspace);
    __nv_bfloat16* q16 = reinterpret_cast<__nv_bfloat16*>(w);
    __nv_bfloat16* k16 = reinterpret_cast<__nv_bfloat16*>(w + align_up(nq * 2, 256));
    __nv_bfloat16* v16 = reinterpret_cast<__nv_bfloat16*>(w + align_up(nq * 2, 256) + align_up(nk * 2, 256));
    const int sms = std::max(sm_count_cached(), 1);
    cast_f32_bf16_kernel<<<sms * 4, 256, 0, st>>>(static_cast<const float*>(q), q16, nq);
    if (nk > 0) {
      cast_f32_bf16_kernel<<<sms * 4, 256, 0, st>>>(static_cast<const float*>(k), k16, nk);
      cast_f32_bf16_kernel<<<sms * 4, 256, 0, st>>>(static_cast<const float*>(v), v16, nk);
    }
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
    qb = q16;
    kb = k16;
    vb = v16;
  }

  FwdParams prm{};
  prm.o = o;
  prm.lse = lse;
  prm.cu = cu_seqlens;
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.G = Hq / Hkv;
  prm.Nq = Nq;
  prm.Nk = Nk;
  prm.causal = causal ? 1 : 0;
  prm.tau = (float)((double)scale * 1.4426950408889634074);
  prm.o_scale = 1.f;
  const int64_t units64 = fwd_units(prm, varlen, rows_q);
  if (units64 >= (int64_t(1) << 31)) return FA_ERR_UNSUPPORTED;
  const int units = (int)units64;
  const bool f32out = in_dtype == FA_F32;
  // rows_k may be 0 (no keys); the map still needs a non-zero extent
  const int64_t rk = std::max<int64_t>(rows_k, 1);
  if (d == 64)
    return f32out ? launch_fwd<64, true>(qb, kb, vb, prm, rows_q, rk, units, st)
                  : launch_fwd<64, false>(qb, kb, vb, prm, rows_q, rk, units, st);
  return f32out ? launch_fwd<128, true>(qb, kb, vb, prm, rows_q, rk, units, st)
                : launch_fwd<128, false>(qb, kb, vb, prm, rows_q, rk, units, st);
}

size_t fa_fwd_fp8_workspace_size(int B, int Hkv, int Nk, int d) {
  if (B <= 0 || Hkv <= 0 || Nk <= 0 || d != 128) return 0;
  const size_t pad = (size_t)(Nk + 15) / 16 * 16;
  return align_up((size_t)B * Hkv * d * pad, 256);
}

fa_status fa_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                     int Nq, int Nk, int d, float scale, float descale_q, float descale_k, float descale_v,
                     int causal, void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !o) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return FA_ERR_INVALID_ARG;
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Nq < 0 || Nk < 0) return FA_ERR_INVALID_ARG;
  for (float x : {scale, descale_q, descale_k, descale_v})
    if (!(x > 0.f) || !std::isfinite(x)) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_UNSUPPORTED;
  if (d != 128) return FA_ERR_UNSUPPORTED;
  const int64_t rows_q = (int64_t)B * Nq, rows_k = (int64_t)B * Nk;
  if (rows_q >= (int64_t(1) << 31) || rows_k >= (int64_t(1) << 31)) return FA_ERR_UNSUPPORTED;
  if (B > 65535 || Hkv > 65535) return FA_ERR_UNSUPPORTED;
  if (B == 0 || Nq == 0) return FA_OK;
  const int pad = (Nk + 15) / 16 * 16;
  const size_t need = fa_fwd_fp8_workspace_size(B, Hkv, Nk, d);
  if (need > 0 && (!workspace || workspace_bytes < need || !aligned16(workspace))) return FA_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* vt = static_cast<uint8_t*>(workspace);
  if (Nk > 0) {
    dim3 g((pad + 63) / 64, Hkv, B);
    transpose_v_e4m3_kernel<<<g, 256, 0, st>>>(static_cast<const uint8_t*>(v), vt, Nk, Hkv, pad);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  FwdParams prm{};
  prm.o = o;
  prm.lse = lse;
  prm.cu = nullptr;
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.G = Hq / Hkv;
  prm.Nq = Nq;
  prm.Nk = Nk;
  prm.causal = causal ? 1 : 0;
  prm.tau = (float)((double)scale * descale_q * descale_k * 1.4426950408889634074);
  prm.o_scale = descale_v;
  const int64_t units64 = fwd_units(prm, false, rows_q);
  if (units64 >= (int64_t(1) << 31)) return FA_ERR_UNSUPPORTED;
  CUtensorMap mq, mk, mv;
  const cuuint64_t dq3[3] = {128, (cuuint64_t)Hq, (cuuint64_t)rows_q};
  const cuuint64_t sq2[2] = {128, (cuuint64_t)Hq * 128};
  const cuuint64_t dk3[3] = {128, (cuuint64_t)Hkv, (cuuint64_t)std::max<int64_t>(rows_k, 1)};
  const cuuint64_t sk2[2] = {128, (cuuint64_t)Hkv * 128};
  const cuuint64_t dv3[3] = {(cuuint64_t)std::max(pad, 16), 128, (cuuint64_t)B * Hkv};
  const cuuint64_t sv2[2] = {(cuuint64_t)std::max(pad, 16), (cuuint64_t)std::max(pad, 16) * 128};
  const cuuint32_t box_rows[3] = {128, 1, (cuuint32_t)kBM};
  const cuuint32_t box_vt[3] = {(cuuint32_t)kBN, 128, 1};
  if (!make_map_u8(&mq, q, dq3, sq2, box_rows) || !make_map_u8(&mk, k, dk3, sk2, box_rows) ||
      !make_map_u8(&mv, Nk > 0 ? (const void*)vt : k, dv3, sv2, box_vt))
    return FA_ERR_CUDA;
  CUtensorMap mo = mq;
  prm.o_tma = make_map_o(&mo, o, 128, Hq, rows_q) ? 1 : 0;
  auto kern = fa_fwd_kernel<128, false, kKindFP8>;
  const int smem = FwdCfg<128, kKindFP8>::kSmemBytes;
  if (set_smem(kern, smem) != cudaSuccess) return FA_ERR_CUDA;
  const int sms = sm_count_cached();
  if (sms <= 0) return FA_ERR_CUDA;
  const int units = (int)units64;
  kern<<<std::min(units, sms), kFwdThreads, smem, st>>>(mq, mk, mv, mo, prm);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_fwd_qkvpacked(const void* qkv, void* o, float* lse, int B, int H, int N, int d, float scale, int causal,
                           const int32_t* cu_seqlens, void* stream) {
  if (!qkv || !o) return FA_ERR_INVALID_ARG;
  if (!aligned16(qkv) || !aligned16(o)) return FA_ERR_INVALID_ARG;
  if (B < 0 || H <= 0 || N < 0) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  const bool varlen = cu_seqlens != nullptr;
  if (varlen) {
    if (B > kMaxVarlenB || (int64_t)N > (int64_t)kMaxVarlenT * kUnitRows) return FA_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0) return FA_ERR_INVALID_ARG;
  }
  const int64_t rows = varlen ? (int64_t)N : (int64_t)B * N;
  if (rows >= (int64_t(1) << 31)) return FA_ERR_UNSUPPORTED;
  if (B == 0 || N == 0) return FA_OK;
  FwdParams prm{};
  prm.o = o;
  prm.lse = lse;
  prm.cu = cu_seqlens;
  prm.B = B;
  prm.Hq = H;
  prm.Hkv = H;
  prm.G = 1;
  prm.Nq = N;
  prm.Nk = N;
  prm.causal = causal ? 1 : 0;
  prm.tau = (float)((double)scale * 1.4426950408889634074);
  prm.o_scale = 1.f;
  const int64_t units64 = fwd_units(prm, varlen, rows);
  if (units64 >= (int64_t(1) << 31)) return FA_ERR_UNSUPPORTED;
  const __nv_bfloat16* base = static_cast<const __nv_bfloat16*>(qkv);
  const int64_t hd = (int64_t)H * d, stride = 3 * hd;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (d == 64)
    return launch_fwd<64, false>(base, base + hd, base + 2 * hd, prm, rows, rows, (int)units64, st, stride, stride);
  return launch_fwd<128, false>(base, base + hd, base + 2 * hd, prm, rows, rows, (int)units64, st, stride, stride);
}

size_t fa_decode_workspace_size(int B, int Hq, int Lmax, int d, int split_len) {
  if (B <= 0 || Hq <= 0 || Lmax <= 0 || d <= 0 || split_len <= 0) return 0;
  const size_t ns = (size_t)((Lmax + split_len - 1) / split_len);
  const size_t parts = (size_t)B * Hq * ns;
  return align_up(parts * d * 4, 256) + align_up(parts * 2 * 4, 256);
}

fa_status fa_decode(const void* q, const void* kcache, const void* vcache, const int32_t* seqlens, void* o,
                    float* lse, int B, int Hq, int Hkv, int Lmax, int d, float scale, int split_len,
                    void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !kcache || !vcache || !o) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned16(o)) return FA_ERR_INVALID_ARG;
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Lmax <= 0 || split_len <= 0) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (seqlens && (reinterpret_cast<uintptr_t>(seqlens) & 3u) != 0) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_UNSUPPORTED;
  if (Hq / Hkv > 16) return FA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (split_len % kDecKeys != 0) return FA_ERR_UNSUPPORTED;
  if ((int64_t)B * Lmax >= (int64_t(1) << 31)) return FA_ERR_UNSUPPORTED;
  if (B == 0) return FA_OK;
  const int nsplit = (Lmax + split_len - 1) / split_len;
  if (nsplit > 65535 || Hkv > 65535 || B > 65535) return FA_ERR_UNSUPPORTED;
  const size_t need = fa_decode_workspace_size(B, Hq, Lmax, d, split_len);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return FA_ERR_WORKSPACE;
  const size_t parts = (size_t)B * Hq * nsplit;
  DecParams prm{};
  prm.q = static_cast<const __nv_bfloat16*>(q);
  prm.seqlens = seqlens;
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.lse = lse;
  prm.ws_acc = static_cast<float*>(workspace);
  prm.ws_ml = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + align_up(parts * d * 4, 256));
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.G = Hq / Hkv;
  prm.Lmax = Lmax;
  prm.split_len = split_len;
  prm.nsplit = nsplit;
  prm.tau = (float)((double)scale * 1.4426950408889634074);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return d == 64 ? launch_decode<64>(kcache, vcache, prm, st) : launch_decode<128>(kcache, vcache, prm, st);
}

size_t fa_decode_paged_workspace_size(int B, int Hq, int Hkv, int max_pages_per_seq, int page_size, int d,
                                      int split_len) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || max_pages_per_seq <= 0 || page_size <= 0 || d <= 0 || split_len <= 0)
    return 0;
  const int64_t lmax = (int64_t)max_pages_per_seq * page_size;
  if (lmax >= (int64_t(1) << 31)) return 0;
  return fa_decode_workspace_size(B, Hq, (int)lmax, d, split_len);  // the split partials
}

fa_status fa_decode_paged(const void* q, const void* k_pages, const void* v_pages, const int32_t* block_table,
                          const int32_t* seqlens, void* o, float* lse, int B, int Hq, int Hkv, int num_pages,
                          int page_size, int max_pages_per_seq, int d, float scale, int split_len, void* workspace,
                          size_t workspace_bytes, void* stream) {
  if (!q || !k_pages || !v_pages || !block_table || !seqlens || !o) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(o)) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(block_table) & 3u) != 0 || (reinterpret_cast<uintptr_t>(seqlens) & 3u) != 0)
    return FA_ERR_INVALID_ARG;
  if (B < 0 || Hq <= 0 || Hkv <= 0 || num_pages <= 0 || page_size <= 0 || max_pages_per_seq <= 0 || split_len <= 0)
    return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if ((page_size & (page_size - 1)) != 0) return FA_ERR_UNSUPPORTED;
  if (page_size < 16) return FA_ERR_UNSUPPORTED;
  if (Hq % Hkv != 0) return FA_ERR_UNSUPPORTED;
  if (Hq / Hkv > 16) return FA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (split_len % kDecKeys != 0) return FA_ERR_UNSUPPORTED;
  if ((int64_t)num_pages * page_size >= (int64_t(1) << 31)) return FA_ERR_UNSUPPORTED;
  const int64_t lmax = (int64_t)max_pages_per_seq * page_size;
  if (lmax >= (int64_t(1) << 31)) return FA_ERR_UNSUPPORTED;
  if (B == 0) return FA_OK;
  const int nsplit = (int)((lmax + split_len - 1) / split_len);
  if (nsplit > 65535 || Hkv > 65535 || B > 65535) return FA_ERR_UNSUPPORTED;
  const size_t need = fa_decode_paged_workspace_size(B, Hq, Hkv, max_pages_per_seq, page_size, d, split_len);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return FA_ERR_WORKSPACE;
  const size_t parts = (size_t)B * Hq * nsplit;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  DecParams prm{};
  prm.q = static_cast<const __nv_bfloat16*>(q);
  prm.seqlens = seqlens;
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.lse = lse;
  prm.ws_acc = reinterpret_cast<float*>(ws);
  prm.ws_ml = reinterpret_cast<float*>(ws + align_up(parts * d * 4, 256));
  prm.block_table = block_table;
  prm.max_pages = max_pages_per_seq;
  prm.page_shift = __builtin_ctz((unsigned)page_size);
  prm.page_box = std::min(page_size, kDecKeys);
  prm.num_pages = num_pages;
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.G = Hq / Hkv;
  prm.Lmax = (int)lmax;
  prm.split_len = split_len;
  prm.nsplit = nsplit;
  prm.tau = (float)((double)scale * 1.4426950408889634074);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return d == 64 ? launch_decode_paged<64>(k_pages, v_pages, prm, st)
                 : launch_decode_paged<128>(k_pages, v_pages, prm, st);
}

size_t fa_bwd_workspace_size(int B, int Hq, int Nq, int d) {
  if (B <= 0 || Hq <= 0 || Nq <= 0 || d <= 0) return 0;
  const size_t pad = (size_t)(Nq + kBwdTile - 1) / kBwdTile * kBwdTile;
  return 2 * align_up((size_t)B * Hq * pad * 4, 256) + align_up((size_t)B * Nq * Hq * d * 4, 256);
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                 void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                 void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv) || (reinterpret_cast<uintptr_t>(lse) & 3u) != 0)
    return FA_ERR_INVALID_ARG;
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Nq < 0 || Nk < 0) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  const int64_t rows_q = (int64_t)B * Nq, rows_k = (int64_t)B * Nk;
  if (rows_q >= (int64_t(1) << 31) || rows_k >= (int64_t(1) << 31)) return FA_ERR_UNSUPPORTED;
  if (B > 65535 || Hkv > 65535) return FA_ERR_UNSUPPORTED;
  if (B == 0 || (Nq == 0 && Nk == 0)) return FA_OK;
  const size_t need = fa_bwd_workspace_size(B, Hq, Nq, d);
  if (need > 0 && (!workspace || workspace_bytes < need || !aligned16(workspace))) return FA_ERR_WORKSPACE;
  BwdParams prm{};
  const int pad = (Nq + kBwdTile - 1) / kBwdTile * kBwdTile;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  prm.lse2 = reinterpret_cast<float*>(ws);
  prm.dvec = reinterpret_cast<float*>(ws + align_up((size_t)B * Hq * pad * 4, 256));
  prm.dq_acc = reinterpret_cast<float*>(ws + 2 * align_up((size_t)B * Hq * pad * 4, 256));
  prm.o = static_cast<const __nv_bfloat16*>(o);
  prm.dout = static_cast<const __nv_bfloat16*>(dout);
  prm.lse = lse;
  prm.dq = static_cast<__nv_bfloat16*>(dq);
  prm.dk = static_cast<__nv_bfloat16*>(dk);
  prm.dv = static_cast<__nv_bfloat16*>(dv);
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.G = Hq / Hkv;
  prm.Nq = Nq;
  prm.Nk = Nk;
  prm.NqPad = pad;
  prm.causal = causal ? 1 : 0;
  prm.scale = scale;
  prm.tau = (float)((double)scale * 1.4426950408889634074);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (Nq == 0) {
    // no query: every gradient is zero
    if (cudaMemsetAsync(dk, 0, (size_t)rows_k * Hkv * d * 2, st) != cudaSuccess ||
        cudaMemsetAsync(dv, 0, (size_t)rows_k * Hkv * d * 2, st) != cudaSuccess)
      return FA_ERR_CUDA;
    return FA_OK;
  }
  return d == 64 ? launch_bwd<64>(q, k, v, prm, st) : launch_bwd<128>(q, k, v, prm, st);
}

// Varlen backward: the tile bound and the workspace carve (tile prefix sums, two row vectors,
// the fp32 dq accumulator).
static int64_t bwd_varlen_ntiles(int B, int total) { return std::max<int64_t>(1, ((int64_t)total + 127 * (int64_t)B) / kBwdTile); }

size_t fa_bwd_varlen_workspace_size(int B, int Hq, int total, int d) {
  if (B <= 0 || Hq <= 0 || total <= 0 || d <= 0) return 0;
  const size_t vec = (size_t)Hq * bwd_varlen_ntiles(B, total) * kBwdTile * 4;
  return align_up((size_t)(B + 1) * 4, 256) + 2 * align_up(vec, 256) + align_up((size_t)total * Hq * d * 4, 256);
}

fa_status fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                        void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int total, int d, float scale,
                        int causal, const int32_t* cu_seqlens, void* workspace, size_t workspace_bytes,
                        void* stream) {
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !cu_seqlens) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv) || (reinterpret_cast<uintptr_t>(lse) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0)
    return FA_ERR_INVALID_ARG;
  if (B < 0 || Hq <= 0 || Hkv <= 0 || total < 0) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (Hkv > 65535) return FA_ERR_UNSUPPORTED;
  if (B == 0 || total == 0) return FA_OK;
  const int64_t ntiles = bwd_varlen_ntiles(B, total);
  if (ntiles * kBwdTile >= (int64_t(1) << 31)) return FA_ERR_UNSUPPORTED;
  const size_t need = fa_bwd_varlen_workspace_size(B, Hq, total, d);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return FA_ERR_WORKSPACE;
  const size_t vec = align_up((size_t)Hq * ntiles * kBwdTile * 4, 256);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  BwdParams prm{};
  prm.tiles = reinterpret_cast<int32_t*>(ws);
  ws += align_up((size_t)(B + 1) * 4, 256);
  prm.lse2 = reinterpret_cast<float*>(ws);
  prm.dvec = reinterpret_cast<float*>(ws + vec);
  prm.dq_acc = reinterpret_cast<float*>(ws + 2 * vec);
  prm.o = static_cast<const __nv_bfloat16*>(o);
  prm.dout = static_cast<const __nv_bfloat16*>(dout);
  prm.lse = lse;
  prm.dq = static_cast<__nv_bfloat16*>(dq);
  prm.dk = static_cast<__nv_bfloat16*>(dk);
  prm.dv = static_cast<__nv_bfloat16*>(dv);
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.G = Hq / Hkv;
  prm.Nq = total;
  prm.Nk = total;
  prm.NqPad = 0;
  prm.causal = causal ? 1 : 0;
  prm.scale = scale;
  prm.tau = (float)((double)scale * 1.4426950408889634074);
  prm.cu = cu_seqlens;
  prm.ntiles = (int)ntiles;
  prm.total = total;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return d == 64 ? launch_bwd<64>(q, k, v, prm, st) : launch_bwd<128>(q, k, v, prm, st);
}

fa_status fa_last_device_error(void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // one host thread at a time uses g_error_taken
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  take_error_word_kernel<<<1, 1, 0, st>>>();
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return FA_ERR_CUDA;
  unsigned int w = 0;
  if (cudaMemcpyFromSymbol(&w, g_error_taken, sizeof(w)) != cudaSuccess) return FA_ERR_CUDA;
  if (w & kErrTimeout) return FA_ERR_TIMEOUT;
  if (w & kErrSmem) return FA_ERR_CUDA;
  if (w != 0) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------------------
// Self-test of the bounded waits: one barrier that nothing arrives on.
namespace fa {
namespace {

__global__ void selftest_wait_kernel() {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  // phase 0 never completes: the wait gives up after its limit, records the timeout and returns
  if (threadIdx.x == 0) (void)mbar_wait(&bar, 0);
}

}  // namespace
}  // namespace fa

extern "C" fa_status fa_selftest_wait_timeout(void* stream) {
  fa::selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>();
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// ---------------------------------------------------------------------------------------
// fa_decode_noalloc: fa_decode with its scratch in a static device array, for callers that
// cannot allocate device memory (see include/fa.h).
namespace fa {
namespace {

// The split partials of fa_decode_noalloc.  In host code this name is only a stand-in for
// the symbol; its device address comes from cudaGetSymbolAddress (per device).
static __device__ __align__(256) unsigned char g_decode_noalloc_scratch[FA_DECODE_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {};

// Device address of the scratch array on the current device, looked up once per device.
fa_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_noalloc_scratch) != cudaSuccess || p == nullptr) return FA_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return FA_OK;
}

}  // namespace
}  // namespace fa

extern "C" fa_status fa_decode_noalloc(const void* q, const void* kcache, const void* vcache, const int32_t* seqlens,
                                       void* o, float* lse, int B, int Hq, int Hkv, int Lmax, int d, float scale,
                                       int split_len, void* stream) {
  // Argument checks of fa_decode, without a workspace: a valid non-empty problem stops at the
  // workspace check (nothing launched); anything else is returned as is.
  const fa_status pre = fa_decode(q, kcache, vcache, seqlens, o, lse, B, Hq, Hkv, Lmax, d, scale, split_len,
                                  nullptr, 0, stream);
  if (pre != FA_ERR_WORKSPACE) return pre;
  if (fa_decode_workspace_size(B, Hq, Lmax, d, split_len) > (size_t)FA_DECODE_NOALLOC_SCRATCH_BYTES)
    return FA_ERR_WORKSPACE;
  void* scratch = nullptr;
  const fa_status st = fa::noalloc_scratch(&scratch);
  if (st != FA_OK) return st;
  return fa_decode(q, kcache, vcache, seqlens, o, lse, B, Hq, Hkv, Lmax, d, scale, split_len, scratch,
                   (size_t)FA_DECODE_NOALLOC_SCRATCH_BYTES, stream);
}
