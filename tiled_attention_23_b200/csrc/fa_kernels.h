// Internal interface between the C-ABI layer (fa_api.cu) and the kernels.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace ta23 {

// Attention forward: one CTA per (128-row query tile, query head, batch).
struct FwdParams {
  void* o;            // [B, Lq, Hq, D] bf16
  float* lse;         // [B, Hq, Lq] fp32 or nullptr
  int B, Lq, Lk, Hq, Hkv, G;
  int n_qtiles;       // query tiles (pairs of tiles for the head_dim 64/128 kernel)
  int sched;          // head_dim 64/128 kernel: 0 = one work item per CTA, 1 = persistent CTAs
  int causal_off;     // Lk - Lq (bottom-right causal alignment)
  float scale_log2;   // scale * log2(e)
  // packed variable-length batch only: sequence b holds query tokens
  // [cu_q[b], cu_q[b+1]) and key tokens [cu_k[b], cu_k[b+1]); q/o are
  // [total_q, Hq, D], k/v [total_k, Hkv, D], lse [Hq, total_q]
  const int* cu_q;
  const int* cu_k;
  int total_q;
  // e4m3 inputs only: dequantisation factors, q [B, Hq], k and v [B, Hkv]
  const float* q_descale;
  const float* k_descale;
  const float* v_descale;
};

int fwd_block_n(int D);   // keys per K/V tile for head_dim D
cudaError_t launch_fa_fwd(int D, bool causal, bool varlen, const CUtensorMap& q, const CUtensorMap& k,
                          const CUtensorMap& v, const FwdParams& p, cudaStream_t stream);
// Attention forward on e4m3 Q, K, V (head_dim 64, 128 or 256, fixed-shape batch).
cudaError_t launch_fa_fwd_fp8(int D, bool causal, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                              const FwdParams& p, cudaStream_t stream);
unsigned int fwd_read_and_clear_status();
// One warp waiting on a barrier that nothing completes, with the given limit.
cudaError_t launch_wait_selftest(unsigned long long limit_ns, cudaStream_t stream);
// Per-head e4m3 quantisation of a bf16 [B, L, H, D] tensor; descale [B, H].
cudaError_t launch_quantize_fp8(int D, const void* x, void* out, float* descale, int B, int L, int H,
                                cudaStream_t stream);

// Attention backward: Delta = rowsum(dO o O), then dQ (per query tile) and
// dK, dV (per K/V tile); D in {64, 128}.
struct BwdParams {
  const void* o;      // [B, Lq, Hq, D] bf16, the forward's output
  const void* dout;   // [B, Lq, Hq, D] bf16
  const float* lse;   // [B, Hq, Lq] fp32, the forward's natural-log LSE
  float* delta;       // [B, Hq, Lq] fp32 workspace
  void* dq;           // [B, Lq, Hq, D] bf16
  void* dk;           // [B, Lk, Hkv, D] bf16
  void* dv;           // [B, Lk, Hkv, D] bf16
  int B, Lq, Lk, Hq, Hkv, G;
  int n_qtiles;
  int causal_off;     // Lk - Lq
  float scale, scale_log2;
};

cudaError_t launch_fa_bwd(int D, bool causal, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                          const CUtensorMap& dout, const BwdParams& p, cudaStream_t stream);
unsigned int bwd_read_and_clear_status();

// Split-KV decode: split kernel over (split, kv head, batch) + LSE combine.
struct DecodeParams {
  const void* q;          // [B, 1, Hq, D] bf16
  const int* seqlens;     // [B] int32
  void* o;                // [B, 1, Hq, D] bf16
  float* lse;             // [B, Hq] or nullptr
  float* ws_o;            // [B, Hq, S, D] fp32 partial outputs (normalised)
  float* ws_lse;          // [B, Hq, S] fp32 partial LSE (natural log; -inf when empty)
  int B, Hq, Hkv, G, Lmax, S;
  float scale_log2;
  // paged cache only: sequence b's key j lives in page block_table[b * max_pages
  // + j / page_size], row j % page_size, of a [num_pages, page_size, Hkv, D] pool
  const int* block_table;
  int page_size, max_pages;
  // int8 cache only: per-(b, kv head, token) scales, [B, Hkv, Lmax] fp32
  const float* k_scale;
  const float* v_scale;   // nullptr when V is bf16
};

int decode_tile_keys(int D);   // keys per K/V tile for head_dim D
constexpr int kPagedBoxRows = 16;   // keys per TMA box of a paged cache (page_size is a multiple)
cudaError_t launch_fa_decode(int D, bool paged, const CUtensorMap& k, const CUtensorMap& v, const DecodeParams& p,
                             cudaStream_t stream);
unsigned int decode_read_and_clear_status();

// The LSE combine of the split partials in p.ws_o / p.ws_lse into p.o / p.lse.
cudaError_t launch_decode_combine(int D, const DecodeParams& p, cudaStream_t stream);

// Split-KV decode against an int8 cache (K int8; V int8 or bf16).
int decode_int8_tile_keys(int D);   // keys per tile: 4096 / D
cudaError_t launch_fa_decode_int8(int D, bool v_int8, const CUtensorMap& k, const CUtensorMap& v,
                                  const CUtensorMap& ks, const CUtensorMap& vs, const DecodeParams& p,
                                  cudaStream_t stream);
unsigned int decode_int8_read_and_clear_status();

// Symmetric int8 quantisation of [B, L, H, D] bf16 rows into codes and
// per-(b, h, token) scales [B, H, L].
cudaError_t launch_quantize_kv_int8(const void* x, void* codes, float* scales, int B, int L, int H, int D,
                                    cudaStream_t stream);

// Device address (on the current device) and size of the fixed scratch buffer
// used by fa_decode_splitkv_noalloc; looked up once per device.
cudaError_t noalloc_scratch(void** ptr, size_t* bytes);

}  // namespace ta23
