// C-ABI layer of libta23.so (declared in include/ta23.h): argument checks,
// TMA tensor-map encoding and kernel launch on the caller's stream.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cmath>
#include <cstdint>
#include <climits>
#include <mutex>

#include "ta23.h"
#include "fa_kernels.h"

#define TA23_STR2(x) #x
#define TA23_STR(x) TA23_STR2(x)

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

// The driver entry point is fetched through the runtime, so the library does
// not link libcuda directly.
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool supported_group(int g) { return g == 1 || g == 2 || g == 4 || g == 8; }
bool supported_dim(int d) { return d == 64 || d == 128 || d == 256; }

// A bf16 tensor [n3, n2, n1, D] viewed by TMA as 4-D (D fastest), boxes of
// 64 (one 128-byte swizzle row) x 1 x rows x 1.
bool encode_bhd(CUtensorMap* m, const void* base, int D, int n1, int n2, int n3, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)n1, (cuuint64_t)n2, (cuuint64_t)n3};
  const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)n1 * D * 2, (cuuint64_t)n2 * n1 * D * 2};
  const cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
  const cuuint32_t elem_strides[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, elem_strides,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A tensor of one-byte codes [n3, n2, n1, D] (int8 KV cache, or e4m3 Q/K/V)
// viewed as 4-D (D fastest), boxes of min(D, 128) bytes x 1 x rows x 1 with the
// 128-byte swizzle (64-byte for 64-byte rows): the layout the tcgen05 shared-
// memory descriptors and the decode's ldmatrix reads expect.
bool encode_i8(CUtensorMap* m, const void* base, int D, int n1, int n2, int n3, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)n1, (cuuint64_t)n2, (cuuint64_t)n3};
  const cuuint64_t strides[3] = {(cuuint64_t)D, (cuuint64_t)n1 * D, (cuuint64_t)n2 * n1 * D};
  const cuuint32_t box[4] = {(cuuint32_t)(D < 128 ? D : 128), 1, (cuuint32_t)box_rows, 1};
  const cuuint32_t elem_strides[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box, elem_strides,
             CU_TENSOR_MAP_INTERLEAVE_NONE, D < 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 scales [n3, n2, n1] viewed as 3-D (n1 fastest), boxes of rows x 1 x 1.
bool encode_scales(CUtensorMap* m, const float* base, int n1, int n2, int n3, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)n1, (cuuint64_t)n2, (cuuint64_t)n3};
  const cuuint64_t strides[2] = {(cuuint64_t)n1 * 4, (cuuint64_t)n2 * n1 * 4};
  const cuuint32_t box[3] = {(cuuint32_t)box_rows, 1, 1};
  const cuuint32_t elem_strides[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box, elem_strides,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Element-count limits of the tensor maps: the outermost stride must stay
// below 2^40 bytes.
bool fits_tma(int64_t inner_rows, int64_t heads, int D, int64_t batch) {
  const int64_t per_batch = inner_rows * heads * D * 2;
  return per_batch < (int64_t(1) << 40) && per_batch * batch < (int64_t(1) << 48);
}

}  // namespace

extern "C" {

TA23_API fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Lq,
                          int Lk, int Hq, int Hkv, int D, float scale, int causal, void* stream) {
  if (!q || !k || !v || !o) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return FA_ERR_INVALID_ARG;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return FA_ERR_INVALID_ARG;
  if (B <= 0 || Lq <= 0 || Lk <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || scale < 0.f) return FA_ERR_INVALID_ARG;
  if (causal && Lq > Lk) return FA_ERR_INVALID_ARG;
  if (!supported_dim(D) || !supported_group(Hq / Hkv)) return FA_ERR_UNSUPPORTED;
  if (B > 65535 || Hq > 65535) return FA_ERR_INVALID_ARG;   // grid y/z limits
  if (!fits_tma(Lq, Hq, D, B) || !fits_tma(Lk, Hkv, D, B)) return FA_ERR_INVALID_ARG;

  const int BN = ta23::fwd_block_n(D);
  CUtensorMap tq, tk, tv;
  if (!encode_bhd(&tq, q, D, Hq, Lq, B, 128) || !encode_bhd(&tk, k, D, Hkv, Lk, B, BN) ||
      !encode_bhd(&tv, v, D, Hkv, Lk, B, BN))
    return FA_ERR_CUDA;

  ta23::FwdParams p{};
  p.o = o;
  p.lse = lse;
  p.B = B;
  p.Lq = Lq;
  p.Lk = Lk;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.n_qtiles = (Lq + 127) / 128;
  p.causal_off = Lk - Lq;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.cu_q = p.cu_k = nullptr;
  p.total_q = 0;
  const cudaError_t e =
      ta23::launch_fa_fwd(D, causal != 0, false, tq, tk, tv, p, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

TA23_API fa_status fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                                 const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int max_seqlen_q,
                                 int total_q, int total_k, int Hq, int Hkv, int D, float scale, int causal,
                                 void* stream) {
  if (!q || !k || !v || !o || !cu_seqlens_q || !cu_seqlens_k) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u) || (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return FA_ERR_INVALID_ARG;
  if (B <= 0 || max_seqlen_q <= 0 || total_q <= 0 || total_k <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0)
    return FA_ERR_INVALID_ARG;
  if (max_seqlen_q > total_q) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || scale < 0.f) return FA_ERR_INVALID_ARG;
  if (!supported_dim(D) || !supported_group(Hq / Hkv)) return FA_ERR_UNSUPPORTED;
  if (B > 65535 || Hq > 65535) return FA_ERR_INVALID_ARG;
  if (!fits_tma(total_q, Hq, D, 1) || !fits_tma(total_k, Hkv, D, 1)) return FA_ERR_INVALID_ARG;

  const int BN = ta23::fwd_block_n(D);
  CUtensorMap tq, tk, tv;
  if (!encode_bhd(&tq, q, D, Hq, total_q, 1, 128) || !encode_bhd(&tk, k, D, Hkv, total_k, 1, BN) ||
      !encode_bhd(&tv, v, D, Hkv, total_k, 1, BN))
    return FA_ERR_CUDA;

  ta23::FwdParams p{};
  p.o = o;
  p.lse = lse;
  p.B = B;
  p.Lq = max_seqlen_q;   // sizes the grid; each CTA reads its sequence's lengths
  p.Lk = 0;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.n_qtiles = 0;
  p.causal_off = 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.cu_q = cu_seqlens_q;
  p.cu_k = cu_seqlens_k;
  p.total_q = total_q;
  const cudaError_t e = ta23::launch_fa_fwd(D, causal != 0, true, tq, tk, tv, p, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

TA23_API fa_status fa_fwd_fp8(const void* q, const void* k, const void* v, const float* q_descale,
                              const float* k_descale, const float* v_descale, void* o, float* lse, int B, int Lq,
                              int Lk, int Hq, int Hkv, int D, float scale, int causal, void* stream) {
  if (!q || !k || !v || !o || !q_descale || !k_descale || !v_descale) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(q_descale) & 3u) || (reinterpret_cast<uintptr_t>(k_descale) & 3u) ||
      (reinterpret_cast<uintptr_t>(v_descale) & 3u) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return FA_ERR_INVALID_ARG;
  if (B <= 0 || Lq <= 0 || Lk <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || scale < 0.f) return FA_ERR_INVALID_ARG;
  if (causal && Lq > Lk) return FA_ERR_INVALID_ARG;
  if (!supported_dim(D) || !supported_group(Hq / Hkv)) return FA_ERR_UNSUPPORTED;
  if (B > 65535 || Hq > 65535) return FA_ERR_INVALID_ARG;
  if (!fits_tma(Lq, Hq, D, B) || !fits_tma(Lk, Hkv, D, B)) return FA_ERR_INVALID_ARG;

  const int BN = ta23::fwd_block_n(D);
  CUtensorMap tq, tk, tv;   // min(D, 128)-byte swizzled rows (64-byte swizzle at head_dim 64)
  if (!encode_i8(&tq, q, D, Hq, Lq, B, 128) || !encode_i8(&tk, k, D, Hkv, Lk, B, BN) ||
      !encode_i8(&tv, v, D, Hkv, Lk, B, BN))
    return FA_ERR_CUDA;

  ta23::FwdParams p{};
  p.o = o;
  p.lse = lse;
  p.B = B;
  p.Lq = Lq;
  p.Lk = Lk;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.n_qtiles = (Lq + 127) / 128;
  p.causal_off = Lk - Lq;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.q_descale = q_descale;
  p.k_descale = k_descale;
  p.v_descale = v_descale;
  const cudaError_t e = ta23::launch_fa_fwd_fp8(D, causal != 0, tq, tk, tv, p, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

TA23_API fa_status fa_quantize_fp8(const void* x, void* x_fp8, float* descale, int B, int L, int H, int D,
                                   void* stream) {
  if (!x || !x_fp8 || !descale) return FA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(x_fp8) || (reinterpret_cast<uintptr_t>(descale) & 3u)) return FA_ERR_INVALID_ARG;
  if (B <= 0 || L <= 0 || H <= 0 || D <= 0) return FA_ERR_INVALID_ARG;
  if (!supported_dim(D)) return FA_ERR_UNSUPPORTED;
  if (B > 65535 || H > 65535 || (int64_t)B * H > INT_MAX) return FA_ERR_INVALID_ARG;
  const cudaError_t e = ta23::launch_quantize_fp8(D, x, x_fp8, descale, B, L, H, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

TA23_API size_t fa_bwd_workspace_bytes(int B, int Hq, int Lq) {
  if (B <= 0 || Hq <= 0 || Lq <= 0) return 0;
  return (((size_t)B * Hq * Lq * sizeof(float)) + 255) & ~size_t(255);
}

TA23_API fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                          const void* dout, void* dq, void* dk, void* dv, int B, int Lq, int Lk, int Hq, int Hkv,
                          int D, float scale, int causal, void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !workspace) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv) || !aligned16(workspace) || (reinterpret_cast<uintptr_t>(lse) & 3u))
    return FA_ERR_INVALID_ARG;
  if (B <= 0 || Lq <= 0 || Lk <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || scale < 0.f) return FA_ERR_INVALID_ARG;
  if (causal && Lq > Lk) return FA_ERR_INVALID_ARG;
  if (!supported_dim(D) || !supported_group(Hq / Hkv)) return FA_ERR_UNSUPPORTED;
  if (B > 65535 || Hq > 65535) return FA_ERR_INVALID_ARG;
  if (!fits_tma(Lq, Hq, D, B) || !fits_tma(Lk, Hkv, D, B)) return FA_ERR_INVALID_ARG;
  if (workspace_bytes < fa_bwd_workspace_bytes(B, Hq, Lq)) return FA_ERR_INVALID_ARG;

  // head_dim 256 moves 64-row tiles (two boxes make a 128-row one)
  const int box = D == 256 ? 64 : 128;
  CUtensorMap tq, tk, tv, tdo;
  if (!encode_bhd(&tq, q, D, Hq, Lq, B, box) || !encode_bhd(&tk, k, D, Hkv, Lk, B, box) ||
      !encode_bhd(&tv, v, D, Hkv, Lk, B, box) || !encode_bhd(&tdo, dout, D, Hq, Lq, B, box))
    return FA_ERR_CUDA;
  ta23::BwdParams p;
  p.o = o;
  p.dout = dout;
  p.lse = lse;
  p.delta = static_cast<float*>(workspace);
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.B = B;
  p.Lq = Lq;
  p.Lk = Lk;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.n_qtiles = (Lq + 127) / 128;
  p.causal_off = Lk - Lq;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  const cudaError_t e = ta23::launch_fa_bwd(D, causal != 0, tq, tk, tv, tdo, p, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

TA23_API size_t fa_decode_workspace_bytes(int B, int Hq, int D, int num_splits) {
  if (B <= 0 || Hq <= 0 || D <= 0 || num_splits <= 0) return 0;
  const size_t rows = (size_t)B * Hq * num_splits;
  const size_t o_bytes = rows * D * sizeof(float);
  const size_t l_bytes = rows * sizeof(float);
  return ((o_bytes + 255) & ~size_t(255)) + ((l_bytes + 255) & ~size_t(255));
}

TA23_API fa_status fa_decode_splitkv(const void* q, const void* k_cache, const void* v_cache, const int* seqlens,
                                     void* o, float* lse, int B, int Hq, int Hkv, int D, int max_seqlen,
                                     int num_splits, float scale, void* workspace, size_t workspace_bytes,
                                     void* stream) {
  if (!q || !k_cache || !v_cache || !seqlens || !o || !workspace) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) || !aligned16(workspace))
    return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(seqlens) & 3u) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return FA_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || max_seqlen <= 0) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (num_splits < 1 || num_splits > 64) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || scale < 0.f) return FA_ERR_INVALID_ARG;
  if (!supported_dim(D) || !supported_group(Hq / Hkv)) return FA_ERR_UNSUPPORTED;
  if (B > 65535 || Hkv > 65535) return FA_ERR_INVALID_ARG;
  if (!fits_tma(max_seqlen, Hkv, D, B)) return FA_ERR_INVALID_ARG;
  const size_t need = fa_decode_workspace_bytes(B, Hq, D, num_splits);
  if (workspace_bytes < need) return FA_ERR_INVALID_ARG;

  const int TK = ta23::decode_tile_keys(D);
  CUtensorMap tk, tv;
  if (!encode_bhd(&tk, k_cache, D, Hkv, max_seqlen, B, TK) || !encode_bhd(&tv, v_cache, D, Hkv, max_seqlen, B, TK))
    return FA_ERR_CUDA;

  ta23::DecodeParams p;
  const size_t rows = (size_t)B * Hq * num_splits;
  p.q = q;
  p.seqlens = seqlens;
  p.o = o;
  p.lse = lse;
  p.ws_o = static_cast<float*>(workspace);
  p.ws_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) + ((rows * D * sizeof(float) + 255) & ~size_t(255)));
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.Lmax = max_seqlen;
  p.S = num_splits;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.block_table = nullptr;
  p.page_size = 0;
  p.max_pages = 0;
  p.k_scale = p.v_scale = nullptr;
  const cudaError_t e = ta23::launch_fa_decode(D, false, tk, tv, p, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

TA23_API fa_status fa_decode_paged(const void* q, const void* k_pages, const void* v_pages, const int* block_table,
                                   const int* seqlens, void* o, float* lse, int B, int Hq, int Hkv, int D,
                                   int num_pages, int page_size, int max_pages_per_seq, int num_splits, float scale,
                                   void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k_pages || !v_pages || !block_table || !seqlens || !o || !workspace) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(o) || !aligned16(workspace))
    return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(seqlens) & 3u) || (reinterpret_cast<uintptr_t>(block_table) & 3u) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return FA_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || num_pages <= 0 || max_pages_per_seq <= 0) return FA_ERR_INVALID_ARG;
  if (page_size < ta23::kPagedBoxRows || page_size % ta23::kPagedBoxRows != 0 || page_size > (1 << 16))
    return FA_ERR_INVALID_ARG;
  if ((int64_t)max_pages_per_seq * page_size > INT32_MAX) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (num_splits < 1 || num_splits > 64) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || scale < 0.f) return FA_ERR_INVALID_ARG;
  if (!supported_dim(D) || !supported_group(Hq / Hkv)) return FA_ERR_UNSUPPORTED;
  if (B > 65535 || Hkv > 65535) return FA_ERR_INVALID_ARG;
  if (!fits_tma(page_size, Hkv, D, num_pages)) return FA_ERR_INVALID_ARG;
  if (workspace_bytes < fa_decode_workspace_bytes(B, Hq, D, num_splits)) return FA_ERR_INVALID_ARG;

  CUtensorMap tk, tv;
  if (!encode_bhd(&tk, k_pages, D, Hkv, page_size, num_pages, ta23::kPagedBoxRows) ||
      !encode_bhd(&tv, v_pages, D, Hkv, page_size, num_pages, ta23::kPagedBoxRows))
    return FA_ERR_CUDA;

  ta23::DecodeParams p;
  const size_t rows = (size_t)B * Hq * num_splits;
  p.q = q;
  p.seqlens = seqlens;
  p.o = o;
  p.lse = lse;
  p.ws_o = static_cast<float*>(workspace);
  p.ws_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) + ((rows * D * sizeof(float) + 255) & ~size_t(255)));
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.Lmax = max_pages_per_seq * page_size;
  p.S = num_splits;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.block_table = block_table;
  p.page_size = page_size;
  p.max_pages = max_pages_per_seq;
  p.k_scale = p.v_scale = nullptr;
  const cudaError_t e = ta23::launch_fa_decode(D, true, tk, tv, p, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

TA23_API fa_status fa_quantize_kv_int8(const void* x, void* codes, float* scales, int B, int L, int H, int D,
                                       void* stream) {
  if (!x || !codes || !scales) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(codes) & 15u) ||
      (reinterpret_cast<uintptr_t>(scales) & 3u))
    return FA_ERR_INVALID_ARG;
  if (B <= 0 || L <= 0 || H <= 0 || D <= 0) return FA_ERR_INVALID_ARG;
  if (!supported_dim(D)) return FA_ERR_UNSUPPORTED;
  if ((int64_t)B * L * H >= (int64_t(1) << 34)) return FA_ERR_INVALID_ARG;
  const cudaError_t e = ta23::launch_quantize_kv_int8(x, codes, scales, B, L, H, D, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

TA23_API fa_status fa_decode_int8(const void* q, const void* k_codes, const float* k_scales, const void* v_cache,
                                  const float* v_scales, const int* seqlens, void* o, float* lse, int B, int Hq,
                                  int Hkv, int D, int max_seqlen, int num_splits, float scale, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  if (!q || !k_codes || !k_scales || !v_cache || !seqlens || !o || !workspace) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_codes) || !aligned16(k_scales) || !aligned16(v_cache) || !aligned16(o) ||
      !aligned16(workspace) || (v_scales && !aligned16(v_scales)))
    return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(seqlens) & 3u) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return FA_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || max_seqlen <= 0) return FA_ERR_INVALID_ARG;
  if (max_seqlen % 4 != 0) return FA_ERR_INVALID_ARG;   // 16-byte rows of the scale tensors
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (num_splits < 1 || num_splits > 64) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || scale < 0.f) return FA_ERR_INVALID_ARG;
  if (!supported_dim(D) || !supported_group(Hq / Hkv)) return FA_ERR_UNSUPPORTED;
  if (B > 65535 || Hkv > 65535) return FA_ERR_INVALID_ARG;
  if (!fits_tma(max_seqlen, Hkv, D, B)) return FA_ERR_INVALID_ARG;
  if (workspace_bytes < fa_decode_workspace_bytes(B, Hq, D, num_splits)) return FA_ERR_INVALID_ARG;

  const bool v_int8 = v_scales != nullptr;
  const int TK = ta23::decode_int8_tile_keys(D);
  CUtensorMap tk, tv, tks, tvs;
  if (!encode_i8(&tk, k_codes, D, Hkv, max_seqlen, B, TK) ||
      !(v_int8 ? encode_i8(&tv, v_cache, D, Hkv, max_seqlen, B, TK)
               : encode_bhd(&tv, v_cache, D, Hkv, max_seqlen, B, TK)) ||
      !encode_scales(&tks, k_scales, max_seqlen, Hkv, B, TK) ||
      !encode_scales(&tvs, v_int8 ? v_scales : k_scales, max_seqlen, Hkv, B, TK))
    return FA_ERR_CUDA;

  ta23::DecodeParams p;
  const size_t rows = (size_t)B * Hq * num_splits;
  p.q = q;
  p.seqlens = seqlens;
  p.o = o;
  p.lse = lse;
  p.ws_o = static_cast<float*>(workspace);
  p.ws_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) + ((rows * D * sizeof(float) + 255) & ~size_t(255)));
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.Lmax = max_seqlen;
  p.S = num_splits;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.block_table = nullptr;
  p.page_size = 0;
  p.max_pages = 0;
  p.k_scale = k_scales;
  p.v_scale = v_scales;
  const cudaError_t e =
      ta23::launch_fa_decode_int8(D, v_int8, tk, tv, tks, tvs, p, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

TA23_API fa_status fa_decode_splitkv_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                             const int* seqlens, void* o, float* lse, int B, int Hq, int Hkv,
                                             int D, int max_seqlen, int num_splits, float scale, void* stream) {
  const size_t need = fa_decode_workspace_bytes(B, Hq, D, num_splits);
  if (need == 0) return FA_ERR_INVALID_ARG;
  if (need > FA_NOALLOC_SCRATCH_BYTES) return FA_ERR_NO_SPACE;
  void* scratch = nullptr;
  size_t bytes = 0;
  if (ta23::noalloc_scratch(&scratch, &bytes) != cudaSuccess) return FA_ERR_CUDA;
  return fa_decode_splitkv(q, k_cache, v_cache, seqlens, o, lse, B, Hq, Hkv, D, max_seqlen, num_splits, scale,
                           scratch, bytes, stream);
}

TA23_API fa_status fa_device_status(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return FA_ERR_CUDA;
  const unsigned a = ta23::fwd_read_and_clear_status();
  const unsigned b = ta23::decode_read_and_clear_status();
  const unsigned c = ta23::decode_int8_read_and_clear_status();
  const unsigned d = ta23::bwd_read_and_clear_status();
  if (a == 0xFFFFFFFFu || b == 0xFFFFFFFFu || c == 0xFFFFFFFFu || d == 0xFFFFFFFFu) return FA_ERR_CUDA;
  return (a | b | c | d) ? FA_ERR_TIMEOUT : FA_OK;
}

TA23_API fa_status fa_selftest_wait_timeout(unsigned int limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 1000000) return FA_ERR_INVALID_ARG;
  if (ta23::launch_wait_selftest(1000ull * limit_us, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return FA_ERR_CUDA;
  return FA_OK;
}

TA23_API const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
    case FA_ERR_NO_SPACE: return "FA_ERR_NO_SPACE";
  }
  return "FA_ERR_UNKNOWN";
}

TA23_API const char* fa_build_info(void) {
  return "libta23: arch sm_100a (tcgen05 + TMA prefill, fixed-shape and packed variable-length; TMA + mma.sync "
         "split-KV decode, contiguous, paged and int8 KV caches); "
         "head_dim {64,128,256}; GQA group {1,2,4,8}; masks {bidirectional, causal bottom-right}; "
         "bf16 in/out, fp32 accumulation and LSE; nvcc " TA23_STR(__CUDACC_VER_MAJOR__) "." TA23_STR(
             __CUDACC_VER_MINOR__);
}

}  // extern "C"
