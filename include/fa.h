/* Exact IO-aware attention for NVIDIA B200 (sm_100a): C ABI.
 *
 * Exact attention O = softmax(Q K^T * scale) V with the per-row logsumexp, computed tile by
 * tile with the online-softmax running max m and sum l, so the N x N score and probability
 * matrices never reach device memory; its backward; and the decode step over a KV cache:
 *
 *   fa_fwd     the tiled forward ("FlashAttention notes", section 3 "Tiling" and section 4
 *              "Online Softmax": m_new = max(m1, m2), l_new = e^(m1-m_new) l1 + e^(m2-m_new) l2;
 *              "LLM basics: from Attention to FlashAttention", chapter 3 section 5), with
 *              causal masking (same tutorial, chapter 1 section 7), grouped-query heads
 *              (chapter 2 section 7) and variable-length packed batches ("FlashAttention-3
 *              (FA-3)", section 2 feature table: MQA, GQA, variable-length).
 *   fa_decode  single-token decode over a KV cache, split along the cache; the partial
 *              results are merged with the same m/l rule ("FlashAttention-3 (FA-3)",
 *              section 4 "FlashDecoding"; "FlashAttention notes", section 4).
 *   fa_decode_paged  the same decode over a paged cache addressed through a block table.
 *   fa_bwd     the backward of fa_fwd by recomputation from the saved logsumexp;
 *              fa_bwd_varlen the same over packed variable-length sequences.
 *   fa_fwd_qkvpacked  fa_fwd reading q, k, v from one packed [.., 3, H, d] tensor.
 *   fa_fwd_fp8 the forward on e4m3 inputs with per-tensor scales.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The library never
 *     allocates or frees device memory and never synchronises, except in
 *     fa_last_device_error.  Every launch is asynchronous on `stream` (a cudaStream_t
 *     passed as void*; NULL is the legacy default stream).
 *   - Tensors are contiguous with the head dimension d innermost (fa_fwd_qkvpacked reads
 *     its three slices with a row stride of 3 H d).  bf16 is IEEE bfloat16.
 *   - Arguments are validated on the host before anything is launched; a rejected call
 *     returns FA_ERR_INVALID_ARG or FA_ERR_UNSUPPORTED and touches no memory.
 *   - A failed launch returns FA_ERR_CUDA.  A device-side wait that exceeded its time
 *     limit (it never should) is recorded on the device and reported by
 *     fa_last_device_error as FA_ERR_TIMEOUT; the kernel then returns instead of hanging.
 */
#ifndef FA_H
#define FA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FA_EXPORT __attribute__((visibility("default")))
#else
#define FA_EXPORT
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, bad scale */
  FA_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. d not in {64, 128}) */
  FA_ERR_WORKSPACE = 3,   /* workspace missing or smaller than the *_workspace_size() value */
  FA_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed */
  FA_ERR_TIMEOUT = 5      /* a device wait gave up (reported by fa_last_device_error) */
} fa_status;

typedef enum { FA_BF16 = 0, FA_F32 = 1, FA_TF32 = 2 } fa_dtype;

/* Forward attention.
 *
 * Fixed length (cu_seqlens == NULL):
 *   q [B, Nq, Hq, d], k and v [B, Nk, Hkv, d], o [B, Nq, Hq, d], lse [B, Hq, Nq].
 * Variable length (cu_seqlens != NULL, device int32 [B+1]):
 *   Nq == Nk == total packed rows; q and o [total, Hq, d], k and v [total, Hkv, d],
 *   lse [Hq, total]; sequence b owns rows [cu_seqlens[b], cu_seqlens[b+1]) of q, k and v and
 *   attends only within itself.  cu_seqlens must start at or above 0, never decrease and end
 *   at or below total; it is read on the device only, and one that breaks this is found
 *   there: nothing is read or written and fa_last_device_error reports FA_ERR_INVALID_ARG.
 *   Rows outside every sequence are not written.  B <= 1024.
 *
 * in_dtype FA_BF16: q, k, v, o are bf16.  FA_F32: q, k, v are fp32, rounded to bf16 (nearest
 *   even) into the workspace first, and o is written as fp32 (fixed or variable length).
 *   FA_TF32: q, k,
 *   v are fp32, rounded to tf32 (10 mantissa bits, nearest even) into the workspace, and the
 *   products run on the tf32 tensor-core path with P kept in fp32; o fp32; fixed length,
 *   d = 64 (the workspace also holds v transposed).
 * Accumulation is fp32; P is rounded to bf16 before the P*V product.
 * scale: the score multiplier, > 0 (1/sqrt(d) in "LLM basics", chapter 1 section 3).
 * causal: query i of a sequence with nq queries and nk keys sees keys j <= i + nk - nq
 *   (bottom-right aligned; the usual lower triangle when nq == nk).  A row that sees no
 *   key gets o = 0 and lse = -inf.
 * lse: natural-log logsumexp of the scaled scores, fp32; may be NULL.
 * Hq must be a multiple of Hkv; query head h uses key/value head h / (Hq / Hkv).
 * d must be 64 or 128.  q, k, v, o must be 16-byte aligned.
 * workspace: device memory of at least fa_fwd_workspace_size(...) bytes (may be NULL when
 *   that size is 0).
 */
FA_EXPORT fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                 int Nq, int Nk, int d, float scale, int causal, const int32_t* cu_seqlens, fa_dtype in_dtype,
                 void* workspace, size_t workspace_bytes, void* stream);

FA_EXPORT size_t fa_fwd_workspace_size(int B, int Hq, int Hkv, int Nq, int Nk, int d, fa_dtype in_dtype, int varlen);

/* FP8 forward ("Attention is All You Need부터 FlashAttention-3까지", FlashAttention-3 section:
 * FP8 support for higher throughput; "FlashAttention-3 (FA-3)", section 2 feature table: FP8):
 * q, k, v are e4m3 (OCP FP8, stored one byte each) with per-tensor dequantisation factors:
 * the value of an element is (its e4m3 value) * descale_x.  Computes the same O and lse as
 * fa_fwd for the dequantised inputs: S = q k^T on the e4m3 tensor-core path (fp32
 * accumulation, exact products), softmax in fp32, P rounded to e4m3 (nearest even, values
 * <= 256 by the lazy rescale) for the P V product, l summed from the unrounded P; O is written
 * as bf16, lse as in fa_fwd.  Fixed length; d must be 128.
 * q [B, Nq, Hq, 128], k and v [B, Nk, Hkv, 128] (bytes), o [B, Nq, Hq, 128] bf16,
 * lse [B, Hq, Nq] fp32 (may be NULL).  Same causal rule and head grouping as fa_fwd.
 * workspace: at least fa_fwd_fp8_workspace_size(B, Hkv, Nk, 128) bytes; it receives a
 * transposed copy of v ([B, Hkv, 128, Nk rounded up to 16]) so that both operands of P V are
 * K-major. */
FA_EXPORT fa_status fa_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                               int Hkv, int Nq, int Nk, int d, float scale, float descale_q, float descale_k,
                               float descale_v, int causal, void* workspace, size_t workspace_bytes, void* stream);

FA_EXPORT size_t fa_fwd_fp8_workspace_size(int B, int Hkv, int Nk, int d);

/* Forward attention on a packed qkv tensor (the flash_attn_qkvpacked_func interface of
 * "Attention is All You Need부터 FlashAttention-3까지", section "practical implementation: using
 * FlashAttention in PyTorch", whose example is qkv [2, 2048, 3, 12, 64], causal): q, k and v
 * are the three slices of qkv [B, N, 3, H, d] bf16 (fixed length) or [total, 3, H, d] with
 * cu_seqlens (variable length, as in fa_fwd, N = total rows).  H query heads and H key/value
 * heads; o [B, N, H, d] (or [total, H, d]) bf16; lse as in fa_fwd (may be NULL).  Read in
 * place through strided tensor maps: no copy, no workspace.  d 64 or 128; qkv and o 16-byte
 * aligned. */
FA_EXPORT fa_status fa_fwd_qkvpacked(const void* qkv, void* o, float* lse, int B, int H, int N, int d, float scale,
                                     int causal, const int32_t* cu_seqlens, void* stream);

/* Backward of fa_fwd (fixed length): gradients dq, dk, dv of o = attention(q, k, v) for an
 * upstream gradient dout of o ("FlashAttention notes", section 5.2 backward: P is rebuilt on
 * chip from q, k and the saved logsumexp instead of being stored; dV = P^T dO, dP = dO V^T,
 * dS = P o (dP - D) with D_i = sum_c dO_ic O_ic, dQ = scale dS K, dK = scale dS^T Q).
 *
 * q, o, dout, dq [B, Nq, Hq, d] bf16; k, v, dk, dv [B, Nk, Hkv, d] bf16; lse [B, Hq, Nq] fp32,
 * the natural-log logsumexp that fa_fwd wrote for (q, k, v, scale, causal), and o the output
 * it wrote.  Same scale, causal rule and head grouping as fa_fwd; dk and dv sum over the
 * query heads of each group.  Accumulation is fp32; P and dS are rounded to bf16 for the
 * tensor-core products; dq, dk, dv are rounded to bf16 (nearest even).
 * d 64 or 128; pointers 16-byte aligned (lse 4-byte aligned).
 * workspace: at least fa_bwd_workspace_size(B, Hq, Nq, d) bytes (two padded fp32 row vectors
 * and an fp32 dq accumulator); its contents need not be initialised. */
FA_EXPORT fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                           const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq, int Nk,
                           int d, float scale, int causal, void* workspace, size_t workspace_bytes, void* stream);

FA_EXPORT size_t fa_bwd_workspace_size(int B, int Hq, int Nq, int d);

/* Backward of fa_fwd on packed variable-length sequences ("FlashAttention-3 (FA-3)", feature
 * table: variable-length batches; the method is that of fa_bwd, within each sequence).
 *
 * Sequence b owns rows [cu_seqlens[b], cu_seqlens[b+1]) of q, o, dout, dq [total, Hq, d] and
 * of k, v, dk, dv [total, Hkv, d] (bf16); lse [Hq, total] fp32 as fa_fwd wrote it with the same
 * cu_seqlens.  No attention, and so no gradient, crosses a sequence boundary; causal is
 * within each sequence.  cu_seqlens: device int32 [B + 1], starting at or above 0, never
 * decreasing, ending at or below total; a cu_seqlens that breaks this is found on the
 * device: nothing is computed and fa_last_device_error reports FA_ERR_INVALID_ARG.  Rows
 * outside every sequence get dq = 0 and their dk, dv are not written; rows of q, k, v and
 * dout past cu_seqlens[B] are read as padding of the last sequence's last tile and must hold
 * finite values.
 * d 64 or 128; pointers 16-byte aligned (lse and cu_seqlens 4-byte aligned).
 * workspace: at least fa_bwd_varlen_workspace_size(B, Hq, total, d) bytes (tile prefix sums,
 * two fp32 row vectors padded per sequence to 128-row tiles, an fp32 dq accumulator); its
 * contents need not be initialised. */
FA_EXPORT fa_status fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const void* dout,
                                  const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int total,
                                  int d, float scale, int causal, const int32_t* cu_seqlens, void* workspace,
                                  size_t workspace_bytes, void* stream);

FA_EXPORT size_t fa_bwd_varlen_workspace_size(int B, int Hq, int total, int d);

/* Split-KV decode: one query token per sequence against its KV cache.
 *
 * q [B, Hq, d] bf16; kcache and vcache [B, Lmax, Hkv, d] bf16; o [B, Hq, d] bf16;
 * lse [B, Hq] fp32 (may be NULL); seqlens: device int32 [B] with 0 <= seqlens[b] <= Lmax,
 * or NULL meaning every sequence holds Lmax tokens.  Sequence b attends (non-causally) to
 * cache rows j < seqlens[b]; an empty sequence gets o = 0 and lse = -inf.
 * The cache is cut into splits of split_len rows (a multiple of 64); each split's partial
 * (m, l, unnormalised acc) goes to the workspace and a second kernel merges them with the
 * m/l rule.  Hq / Hkv <= 16.  d must be 64 or 128.  Pointers 16-byte aligned.
 */
FA_EXPORT fa_status fa_decode(const void* q, const void* kcache, const void* vcache, const int32_t* seqlens, void* o,
                    float* lse, int B, int Hq, int Hkv, int Lmax, int d, float scale, int split_len,
                    void* workspace, size_t workspace_bytes, void* stream);

FA_EXPORT size_t fa_decode_workspace_size(int B, int Hq, int Lmax, int d, int split_len);

/* Largest scratch, in bytes, that fa_decode_noalloc can use (16 MiB). */
#define FA_DECODE_NOALLOC_SCRATCH_BYTES (16u << 20)

/* fa_decode for callers that cannot allocate device memory.
 *
 * Some callers have no way to call cudaMalloc on this path: a host program that only
 * receives its input and output buffers from someone else (a plugin inside another
 * framework's memory pool), or a latency-critical loop where an allocation, which can
 * synchronise the device, is not allowed.  This entry point takes the same arguments as
 * fa_decode minus the workspace and allocates nothing.  The pages describe no such entry
 * point; it exists only for these callers.
 *
 * Scratch: the split partials live in one static device array of
 * FA_DECODE_NOALLOC_SCRATCH_BYTES in this library, which every GPU that loads the library
 * holds until the process exits.  Problems whose scratch need (fa_decode_workspace_size)
 * exceeds it are rejected with FA_ERR_WORKSPACE before anything is launched; the decode
 * workload B=8, Hq=64, d=128, cache 32768, splits of 1024 needs about 8.7 MB.
 * No part of the scratch has to start at zero: every partial the merge reads is written by
 * the same call.  All calls share the array, so calls that overlap on the GPU (on
 * different streams, or on one stream from different threads without ordering) race and
 * give wrong results; order them on one stream.
 * The first call on each device looks up the array's device address (with that device
 * current) and caches it; make that first call before any stream capture.  The cached
 * address belongs to that device's context: a process that resets the device
 * (cudaDeviceReset) or otherwise tears its primary context down must not call this entry
 * point on that device again, since the library's device memory may then sit elsewhere.
 * Other arguments, results and errors are those of fa_decode. */
FA_EXPORT fa_status fa_decode_noalloc(const void* q, const void* kcache, const void* vcache, const int32_t* seqlens,
                                      void* o, float* lse, int B, int Hq, int Hkv, int Lmax, int d, float scale,
                                      int split_len, void* stream);

/* Split-KV decode over a paged KV cache ("LLM basics: from Attention to FlashAttention",
 * chapter 2 section 8, PagedAttention: fixed-size pages of the cache, mapped from each
 * sequence's logical pages by a block table); the splits are merged as in fa_decode.
 *
 * q [B, Hq, d] bf16; k_pages and v_pages [num_pages, page_size, Hkv, d] bf16 (the page
 * pool); block_table: device int32 [B, max_pages_per_seq], entry (b, t) = the physical page
 * holding tokens t*page_size .. (t+1)*page_size - 1 of sequence b; seqlens: device int32 [B],
 * required, 0 <= seqlens[b] <= max_pages_per_seq * page_size (larger values are clamped).
 * Only the first ceil(seqlens[b] / page_size) entries of row b are read; pages may be
 * shared between sequences and appear in any order.  o [B, Hq, d] bf16; lse [B, Hq] fp32
 * (may be NULL).  Token j of sequence b takes part iff j < seqlens[b]; an empty sequence gets
 * o = 0 and lse = -inf.  Rows of a page beyond a sequence's length may hold anything
 * (NaN included): they are masked and never multiply into o.
 * page_size: a power of two >= 16.  split_len: a multiple of 64.  Hq / Hkv <= 16; d 64 or
 * 128; q, the pages and o 16-byte aligned; block_table and seqlens 4-byte aligned;
 * num_pages * page_size < 2^31.
 * A block-table entry outside [0, num_pages) is read as page 0 and recorded on the device;
 * fa_last_device_error then returns FA_ERR_INVALID_ARG.
 * workspace: at least fa_decode_paged_workspace_size(...) bytes (the split partials); its
 * contents need not be initialised.  Calls sharing a workspace must not overlap on the GPU. */
FA_EXPORT fa_status fa_decode_paged(const void* q, const void* k_pages, const void* v_pages,
                                    const int32_t* block_table, const int32_t* seqlens, void* o, float* lse, int B,
                                    int Hq, int Hkv, int num_pages, int page_size, int max_pages_per_seq, int d,
                                    float scale, int split_len, void* workspace, size_t workspace_bytes,
                                    void* stream);

FA_EXPORT size_t fa_decode_paged_workspace_size(int B, int Hq, int Hkv, int max_pages_per_seq, int page_size, int d,
                                                int split_len);

/* Takes the device-side error record (read and cleared in one atomic exchange, on `stream`),
 * waits for `stream`, and returns FA_ERR_TIMEOUT if any kernel of this library recorded a
 * device-side timeout since the previous call, else FA_ERR_CUDA if a kernel found its shared
 * memory carve-out too small, else FA_ERR_INVALID_ARG if a kernel recorded an invalid
 * device-side input (a block-table entry out of range, a cu_seqlens that fa_fwd or
 * fa_bwd_varlen cannot use); FA_ERR_CUDA if the stream reports an error; else FA_OK.
 * The record is shared by all kernels of the library on the device (all streams); a timeout
 * stops only the kernel whose wait ran out, and later launches run normally whether or not
 * the record has been taken. */
FA_EXPORT fa_status fa_last_device_error(void* stream);

/* Test support for the failure detection: launches one kernel whose single wait can never be
 * satisfied (nothing arrives on its barrier).  The wait is bounded like every wait of the
 * library: after its time limit (4 s) it records a timeout and the kernel returns, so nothing
 * hangs and the context stays usable; the next fa_last_device_error reports FA_ERR_TIMEOUT. */
FA_EXPORT fa_status fa_selftest_wait_timeout(void* stream);

/* Static description of a status code. */
FA_EXPORT const char* fa_status_string(fa_status s);

/* Number of streaming multiprocessors of the current device (0 on failure); the forward
 * kernel's persistent grid uses one CTA per SM. */
FA_EXPORT int fa_device_sm_count(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_H */
