/*
 * ta23.h - C ABI of the B200 (sm_100a) tiled attention library libta23.so.
 *
 * The library computes exact attention O = softmax(scale * Q K^T + mask) V tile
 * by tile with an online softmax, never materialising the score matrix, and a
 * split-KV decode whose chunk results are merged through their log-sum-exp.
 *
 * Sources of the operation (cited by page title and section):
 *  - "FlashAttention in Ascend CANN ops-transformer" (ai6s.net), section 二:
 *    Q/K/V cut into blocks (step 1); per block the running max and running
 *    sum are updated, giving exactly the standard attention result (step 2);
 *    O and the log-sum-exp L are accumulated block by block and written back
 *    (step 3).  Section 四: tensors are [batch, seq_len, num_heads, head_dim],
 *    softmax_scale defaults to 1/sqrt(head_dim), is_causal selects the causal
 *    mask.  Section 五: the causal flag removes keys after the query from the
 *    softmax (bidirectional attention must leave it off); head_dim 64/128/256
 *    are supported.
 *  - "FlashAttention-2 (TH)" (systems-analysis.info): exact result (no
 *    approximation); parallelism over query blocks within a head.
 *  - MNN attention_mode page (lpnh.cn): fused flash-attention prefill for
 *    head_dim in {64,128,256} and GQA group in {1,2,4,8} with a causal mask.
 *  - "5 years, 10K stars: how xformers redefines Transformer acceleration with
 *    the Bias protocol" (developer.cloud.tencent.com): masks are expressed by
 *    structure, never as a dense tensor in memory; a split-K decode backend.
 *
 * Conventions for every entry point:
 *  - Tensors are caller-owned, contiguous, row-major DEVICE memory, base
 *    addresses 16-byte aligned.  bf16 means IEEE bfloat16; fp32 means float.
 *  - G = Hq / Hkv query heads share one K/V head: query head h reads K/V head
 *    h / G (contiguous groups).
 *  - Causal masking is bottom-right aligned: query row i may attend key j iff
 *    j <= i + (Lk - Lq).  Masked scores are -infinity (an additive mask), so
 *    they carry zero probability.
 *  - lse is the natural-log log-sum-exp of the scaled, masked scores of each
 *    query row, in fp32.
 *  - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream).  No call synchronises and no call allocates
 *    device memory.
 *  - Validation failures return before anything is enqueued.
 *  - The library is thread-safe: it keeps no per-call host state.
 */
#ifndef TA23_H
#define TA23_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define TA23_API __attribute__((visibility("default")))
#else
#define TA23_API
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, Hq % Hkv != 0, ... */
  FA_ERR_UNSUPPORTED = 2, /* head_dim not in {64,128,256} or group not in {1,2,4,8} */
  FA_ERR_CUDA = 3,        /* a CUDA runtime error while enqueuing */
  FA_ERR_TIMEOUT = 4,     /* a bounded device-side wait gave up (fa_device_status) */
  FA_ERR_NO_SPACE = 5     /* fa_decode_splitkv_noalloc: the request needs more scratch
                             than its fixed buffer (FA_NOALLOC_SCRATCH_BYTES) holds */
} fa_status;

/*
 * fa_fwd - attention forward (prefill).
 *
 * Computes, for every batch b, query head h, query row i:
 *   O[b,i,h,:] = sum_j softmax_j(scale * q[b,i,h,:] . k[b,j,h/G,:] + mask_ij) v[b,j,h/G,:]
 *   lse[b,h,i] = ln sum_j exp(scale * q . k + mask_ij)
 * (ops-transformer page, section 二 steps 1-3; section 四 for the layout.)
 *
 *   q    [B, Lq, Hq,  D] bf16, device, read only
 *   k    [B, Lk, Hkv, D] bf16, device, read only
 *   v    [B, Lk, Hkv, D] bf16, device, read only
 *   o    [B, Lq, Hq,  D] bf16, device, written (must not overlap the inputs)
 *   lse  [B, Hq, Lq]     fp32, device, written; may be NULL (not written)
 *   scale  multiplies Q K^T before the mask; finite and >= 0
 *   causal 0 = bidirectional, nonzero = causal (bottom-right aligned)
 *
 * Errors: FA_ERR_INVALID_ARG for a NULL q/k/v/o, a base address not 16-byte
 * aligned, any size <= 0, Hq % Hkv != 0, a non-finite or negative scale, causal
 * with Lq > Lk (a row would have no key), or sizes whose element offsets do not
 * fit the tensor-map limits (each dimension < 2^31, B*Lq*Hq*D < 2^40);
 * FA_ERR_UNSUPPORTED for D not in {64,128,256} or Hq/Hkv not in {1,2,4,8};
 * FA_ERR_CUDA if the launch fails (the CUDA error is left set for the caller).
 */
TA23_API fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int Lq, int Lk, int Hq, int Hkv, int D,
                          float scale, int causal, void* stream);

/*
 * fa_fwd_varlen - attention forward over a packed batch of variable-length
 * sequences (block-diagonal attention: a query token attends only keys of its
 * own sequence; the "block diagonal" structured bias of the xformers page,
 * read by structure and never materialised as a mask).  Sequence b is
 * computed exactly as fa_fwd would compute a batch of one with
 * Lq = cu_seqlens_q[b+1] - cu_seqlens_q[b] and Lk = cu_seqlens_k[b+1] -
 * cu_seqlens_k[b], including the bottom-right causal alignment.
 *
 *   q    [total_q, Hq,  D] bf16, device, read only (sequences packed back to back)
 *   k    [total_k, Hkv, D] bf16, device, read only
 *   v    [total_k, Hkv, D] bf16, device, read only
 *   o    [total_q, Hq,  D] bf16, device, written
 *   lse  [Hq, total_q]     fp32, device, written; may be NULL
 *   cu_seqlens_q, cu_seqlens_k  [B+1] int32, device: cumulative token offsets,
 *        cu[0] = 0, non-decreasing, cu_seqlens_q[B] = total_q,
 *        cu_seqlens_k[B] = total_k (device data, not checked on the host)
 *   max_seqlen_q  an upper bound of every query length (sizes the launch);
 *        query rows of a sequence beyond it are not computed
 *
 * A query row with no allowed key (an empty key sequence, or causal with more
 * queries than keys) is written as O = 0, lse = -infinity.  Rows outside
 * [0, total_q) are never written, whatever cu_seqlens_q holds.
 * Errors: FA_ERR_INVALID_ARG for NULL or misaligned pointers, B,
 * max_seqlen_q, total_q, total_k, Hq, Hkv or D <= 0, max_seqlen_q > total_q,
 * Hq % Hkv != 0, or a non-finite/negative scale; FA_ERR_UNSUPPORTED and
 * FA_ERR_CUDA as for fa_fwd.
 */
TA23_API fa_status fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                                 const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int max_seqlen_q,
                                 int total_q, int total_k, int Hq, int Hkv, int D, float scale, int causal,
                                 void* stream);

/*
 * fa_fwd_fp8 - attention forward on 8-bit floating-point inputs (the FP8
 * support of FlashAttention-3, "FlashAttention-2 (TH)" page, section
 * "FlashAttention-3" under the comparison with later versions).
 *
 * Q, K and V are e4m3 codes (OCP 8-bit float: 1 sign, 4 exponent bits with
 * bias 7, 3 mantissa bits; no infinities, S.1111.111 is NaN, largest finite
 * 448) with one dequantisation factor per (batch, head): the operand value is
 * code * descale.  The result is the fa_fwd definition on those values:
 *   O[b,i,h,:] = sum_j softmax_j(scale * qd[b,h] kd[b,h/G] q8 . k8 + mask_ij) vd[b,h/G] v8[b,j,h/G,:]
 * Scores and the softmax run in fp32; the probabilities enter the P V
 * product rounded to e4m3 (relative error <= 2^-4 each), so O carries up to
 * 2^-4 of sum_j p_ij |v_j| of error where fa_fwd carries 2^-9.
 *
 *   q    [B, Lq, Hq,  D] e4m3 codes (one byte each), device, read only
 *   k    [B, Lk, Hkv, D] e4m3 codes, device, read only
 *   v    [B, Lk, Hkv, D] e4m3 codes, device, read only
 *   q_descale [B, Hq], k_descale [B, Hkv], v_descale [B, Hkv]  fp32, device
 *   o    [B, Lq, Hq,  D] bf16, device, written
 *   lse  [B, Hq, Lq]     fp32, device, written; may be NULL
 *   scale, causal as for fa_fwd
 *
 * Errors as for fa_fwd (NULL descale pointers or descale pointers not 4-byte
 * aligned are FA_ERR_INVALID_ARG); FA_ERR_UNSUPPORTED for D not in
 * {64,128,256} or Hq/Hkv not in {1,2,4,8}.  Codes that are NaN give
 * unspecified results.
 */
TA23_API fa_status fa_fwd_fp8(const void* q, const void* k, const void* v, const float* q_descale,
                              const float* k_descale, const float* v_descale, void* o, float* lse,
                              int B, int Lq, int Lk, int Hq, int Hkv, int D, float scale, int causal,
                              void* stream);

/*
 * fa_quantize_fp8 - per-head e4m3 quantisation of a bf16 tensor, the input
 * side of fa_fwd_fp8.  For each (b, h), over the L x D slice x[b, :, h, :]:
 *   amax = max |x|;  inv = 448 / amax in fp32;
 *   code = e4m3(x * inv)  (fp32 product, round to nearest even, saturating
 *                          at +-448);
 *   descale[b, h] = amax / 448 in fp32;
 * a slice with amax < 2^-110 (all zero, or too small for 448 / amax to stay
 * in the fp32 range) takes inv = descale = 1.
 *
 *   x        [B, L, H, D] bf16, device, read only (finite values)
 *   x_fp8    [B, L, H, D] e4m3 codes, device, written
 *   descale  [B, H] fp32, device, written (also used as scratch during the call)
 *
 * Errors: FA_ERR_INVALID_ARG for NULL or misaligned pointers or sizes <= 0;
 * FA_ERR_UNSUPPORTED for D not in {64,128,256}.  Non-finite inputs give
 * unspecified codes and factors.
 */
TA23_API fa_status fa_quantize_fp8(const void* x, void* x_fp8, float* descale, int B, int L, int H, int D,
                                   void* stream);

/*
 * fa_bwd_workspace_bytes - bytes of device workspace fa_bwd needs (one fp32
 * per (b, query head, query row)).  Returns 0 for invalid sizes.
 */
TA23_API size_t fa_bwd_workspace_bytes(int B, int Hq, int Lq);

/*
 * fa_bwd - attention backward: the gradients of fa_fwd's O with respect to q,
 * k and v for an upstream gradient dO (the backward operator the xformers page
 * pairs with each forward operator; training throughput on the
 * FlashAttention-2 page).  With P = softmax(scale q k^T + mask) recomputed from
 * the forward's lse:
 *   dV = P^T dO,  dP = dO V^T,  dS = P o (dP - rowsum(dO o O)),
 *   dQ = scale dS K,  dK = scale dS^T Q   (GQA heads summed into their K/V head)
 *
 *   q, k, v, scale, causal  as passed to fa_fwd
 *   o      [B, Lq, Hq, D] bf16, device: fa_fwd's output
 *   lse    [B, Hq, Lq]    fp32, device: fa_fwd's lse (required)
 *   dout   [B, Lq, Hq, D] bf16, device: the upstream gradient
 *   dq     [B, Lq, Hq, D] bf16, device, written
 *   dk, dv [B, Lk, Hkv, D] bf16, device, written
 *   workspace  at least fa_bwd_workspace_bytes(B, Hq, Lq) bytes, 16-byte aligned
 *
 * Errors: those of fa_fwd, plus FA_ERR_INVALID_ARG for a NULL o, lse, dout,
 * dq, dk, dv or workspace, a misaligned one, or a short workspace;
 * FA_ERR_UNSUPPORTED for D not in {64, 128, 256} or Hq/Hkv not in {1, 2, 4, 8}.
 */
TA23_API fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                          const void* dout, void* dq, void* dk, void* dv, int B, int Lq, int Lk, int Hq,
                          int Hkv, int D, float scale, int causal, void* workspace, size_t workspace_bytes,
                          void* stream);

/*
 * fa_decode_workspace_bytes - bytes of device workspace fa_decode_splitkv needs:
 * num_splits partial outputs of D fp32 values plus one fp32 LSE per split, for
 * every (b, query head).  Returns 0 for invalid sizes.  The pages name split-KV
 * decoding (the xformers page's split-K backend) but not how its partial
 * results are stored; this layout is the library's reading.
 */
TA23_API size_t fa_decode_workspace_bytes(int B, int Hq, int D, int num_splits);

/*
 * fa_decode_splitkv - one query token per sequence against a KV cache, with the
 * keys of each sequence split into num_splits chunks whose partial results
 * (O_c, L_c) are merged through their log-sum-exp:
 *   L = ln sum_c exp(L_c),  O = sum_c exp(L_c - L) O_c
 * (split-K decode backend named on the xformers page; the merge rule is the
 * same running-max/running-sum algebra as step 2 of the ops-transformer page).
 *
 *   q        [B, 1, Hq, D]       bf16, device, read only
 *   k_cache  [B, max_seqlen, Hkv, D] bf16, device, read only
 *   v_cache  [B, max_seqlen, Hkv, D] bf16, device, read only
 *   seqlens  [B] int32, device: sequence b uses keys 0 .. seqlens[b]-1; each
 *            value must lie in [1, max_seqlen] (not checked on the host: the
 *            kernel clamps to that range)
 *   o        [B, 1, Hq, D] bf16, device, written
 *   lse      [B, Hq] fp32, device, written; may be NULL
 *   num_splits  1 .. 64; chunk size per sequence is 64 * ceil(ceil(len/num_splits)/64)
 *   workspace   device scratch of at least fa_decode_workspace_bytes(B,Hq,D,num_splits)
 *               bytes, 16-byte aligned, owned by the caller; overwritten
 *
 * Errors: FA_ERR_INVALID_ARG for NULL q/k_cache/v_cache/seqlens/o/workspace,
 * misalignment, sizes <= 0, Hq % Hkv != 0, num_splits outside [1, 64], a short
 * workspace, or a non-finite/negative scale; FA_ERR_UNSUPPORTED for D not in
 * {64,128,256} or Hq/Hkv not in {1,2,4,8}; FA_ERR_CUDA on a launch failure.
 */
TA23_API fa_status fa_decode_splitkv(const void* q, const void* k_cache, const void* v_cache,
                                     const int* seqlens, void* o, float* lse,
                                     int B, int Hq, int Hkv, int D, int max_seqlen,
                                     int num_splits, float scale,
                                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_decode_paged - fa_decode_splitkv against a paged KV cache.  The keys and
 * values of all sequences live in a shared pool of fixed-size pages, and a
 * per-sequence block table maps logical positions to pages: key j of
 * sequence b is row j % page_size of page block_table[b * max_pages_per_seq +
 * j / page_size].  (The xformers page lists "paged" among the structured
 * attention-bias layouts that a kernel reads by structure instead of from a
 * dense mask; the result is the same as fa_decode_splitkv on the gathered
 * cache, including the chunking into num_splits and the LSE merge.)
 *
 *   q          [B, 1, Hq, D] bf16, device, read only
 *   k_pages    [num_pages, page_size, Hkv, D] bf16, device, read only
 *   v_pages    [num_pages, page_size, Hkv, D] bf16, device, read only
 *   block_table [B, max_pages_per_seq] int32, device: physical page of each
 *              logical page; only entries for pages that hold keys of the
 *              sequence (j < seqlens[b]) are read.  Entries outside
 *              [0, num_pages) are not checked: the copy engine returns zeros
 *              for them (a wrong result, not a fault).
 *   seqlens    [B] int32, device: in [1, max_pages_per_seq * page_size]
 *              (clamped to that range on the device)
 *   o, lse, num_splits, scale, workspace: as fa_decode_splitkv (the same
 *              fa_decode_workspace_bytes(B, Hq, D, num_splits) suffices)
 *   page_size  a multiple of 16 in [16, 65536]
 *
 * Errors: those of fa_decode_splitkv, plus FA_ERR_INVALID_ARG for a NULL or
 * misaligned block_table, num_pages or max_pages_per_seq <= 0, or a page_size
 * that is not a multiple of 16 in [16, 65536].
 */
TA23_API fa_status fa_decode_paged(const void* q, const void* k_pages, const void* v_pages,
                                   const int* block_table, const int* seqlens, void* o, float* lse,
                                   int B, int Hq, int Hkv, int D, int num_pages, int page_size,
                                   int max_pages_per_seq, int num_splits, float scale,
                                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_quantize_kv_int8 - writes an int8 KV cache from bf16 rows (the KV-INT8
 * cache of the MNN attention_mode page, "almost lossless" there; the page fixes
 * no granularity, so here: symmetric, one fp32 scale per (b, token, head)
 * vector of D values).  For every row x of D values, in fp32:
 *   scale = max|x| / 127,  code_d = round-half-even(x_d / scale) clamped to
 *   [-127, 127]   (an all-zero row: scale 0, codes 0)
 * IEEE division and rintf; the codes are bit-exact to that definition.
 *
 *   x       [B, L, H, D] bf16, device, read only
 *   codes   [B, L, H, D] int8, device, written
 *   scales  [B, H, L]    fp32, device, written (head-major: one head's tokens
 *           are contiguous, the layout fa_decode_int8 reads)
 * Errors: FA_ERR_INVALID_ARG for NULL or misaligned pointers (x, codes 16-byte;
 * scales 4-byte) or sizes <= 0; FA_ERR_UNSUPPORTED for D not in {64,128,256};
 * FA_ERR_CUDA on a launch failure.
 */
TA23_API fa_status fa_quantize_kv_int8(const void* x, void* codes, float* scales, int B, int L, int H, int D,
                                       void* stream);

/*
 * fa_decode_int8 - fa_decode_splitkv against an int8 KV cache written by
 * fa_quantize_kv_int8: K is int8, and V is int8 too (v_scales non-NULL) or bf16
 * (v_scales NULL) - the two KV-INT8 modes of the MNN attention_mode page.  The
 * result is the decode of the dequantised cache (value = scale * code):
 *   O = sum_j softmax_j(scale * q . (ks_j * kcode_j)) (vs_j * vcode_j or v_j)
 * with the same chunking into num_splits and LSE merge as fa_decode_splitkv.
 *
 *   q         [B, 1, Hq, D] bf16, device; |q| <= 65280 (the products run in fp16:
 *             q converts exactly for 2^-17 <= |q| <= 65280; smaller values lose
 *             low bits in fp16 subnormals, under 2^-25 they become 0)
 *   k_codes   [B, max_seqlen, Hkv, D] int8, device
 *   k_scales  [B, Hkv, max_seqlen] fp32, device
 *   v_cache   [B, max_seqlen, Hkv, D] int8 (with v_scales) or bf16 (without)
 *   v_scales  [B, Hkv, max_seqlen] fp32, device, or NULL
 *   seqlens, o, lse, num_splits, scale, workspace: as fa_decode_splitkv
 *   max_seqlen  a multiple of 4 (rows of the scale tensors are 16-byte aligned)
 * With int8 V, p * v_scale is rounded to fp16 before P V, so V scales must keep
 * 256 * v_scale below 65504.
 * Errors: those of fa_decode_splitkv, plus FA_ERR_INVALID_ARG for a NULL
 * k_scales, a misaligned scale tensor or max_seqlen not a multiple of 4.
 */
TA23_API fa_status fa_decode_int8(const void* q, const void* k_codes, const float* k_scales,
                                  const void* v_cache, const float* v_scales, const int* seqlens,
                                  void* o, float* lse, int B, int Hq, int Hkv, int D, int max_seqlen,
                                  int num_splits, float scale, void* workspace, size_t workspace_bytes,
                                  void* stream);

/*
 * fa_decode_splitkv_noalloc - fa_decode_splitkv for callers that cannot
 * allocate device memory.  The pages describe no such variant; it exists for
 * callers such as a plug-in inside a host process whose own allocator has
 * reserved the GPU's memory up front (so a private cudaMalloc would fail or
 * fragment it), or a latency-critical decode loop that must not call cudaMalloc
 * because it can synchronise the device.  Such callers still pass q, the caches,
 * seqlens, o and lse, but no workspace: the split partials go to a fixed
 * scratch buffer of FA_NOALLOC_SCRATCH_BYTES that the library holds in device
 * memory (a file-scope __device__ array), on every GPU that loads the library,
 * until the process exits.  This call allocates nothing itself (no cudaMalloc,
 * cudaFree or allocating library routine).
 *
 * Arguments, layouts and results are those of fa_decode_splitkv.
 * - The first call on a device looks up the buffer's device address on the
 *   current device (cudaGetSymbolAddress) and caches it; make that first call
 *   before any stream capture.  The current device must be the device of
 *   `stream` and of the tensors.
 * - Every call on a device shares the one buffer, which keeps the last call's
 *   contents (nothing in it needs to start at zero: every partial a call reads
 *   is written by that call first).  Calls whose execution overlaps on the GPU
 *   (different streams, or more than one host thread) race on the buffer and
 *   give wrong results; serialise them.
 * Errors: those of fa_decode_splitkv; FA_ERR_NO_SPACE when
 * fa_decode_workspace_bytes(B, Hq, D, num_splits) > FA_NOALLOC_SCRATCH_BYTES;
 * FA_ERR_CUDA when the buffer address cannot be obtained.
 */
#define FA_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
TA23_API fa_status fa_decode_splitkv_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                             const int* seqlens, void* o, float* lse,
                                             int B, int Hq, int Hkv, int D, int max_seqlen,
                                             int num_splits, float scale, void* stream);

/*
 * fa_device_status - synchronises the current device, then returns FA_OK, or
 * FA_ERR_TIMEOUT if any kernel of this library gave up a bounded wait since the
 * last call (and clears that record), or FA_ERR_CUDA if synchronising failed.
 * For diagnostics and tests; never called on the hot path.
 */
TA23_API fa_status fa_device_status(void);

/*
 * fa_selftest_wait_timeout - self-test of the bounded device-side waits, for
 * tests and diagnostics (never on the hot path).  The pages describe no failure
 * detection; bounded waits reported through fa_device_status are this
 * library's reading of the operator's error path (a status instead of the
 * ops-transformer page's section 五 fallback).
 *
 * Enqueues on `stream` one kernel whose single warp waits on a barrier that
 * nothing completes, with a limit of limit_us microseconds instead of the
 * kernels' 2 s: the wait gives up, records FA_ERR_TIMEOUT for the next
 * fa_device_status() call and sets its block's abort flag, so a second wait
 * returns at once and the kernel exits.  No memory is touched; the device
 * stays usable.
 * Errors: FA_ERR_INVALID_ARG for limit_us outside [1, 1000000]; FA_ERR_CUDA on a
 * launch error.
 */
TA23_API fa_status fa_selftest_wait_timeout(unsigned int limit_us, void* stream);

/* Human-readable name of a status code (static string).  The codes and their
 * names are this library's reading: the pages define no error interface. */
TA23_API const char* fa_status_string(fa_status s);

/* Build description: target architecture, flags, supported D and groups
 * (static string).  Cf. the build-information report on the xformers page. */
TA23_API const char* fa_build_info(void);

#ifdef __cplusplus
}
#endif

#endif /* TA23_H */
