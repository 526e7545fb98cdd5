// Attention backward for sm_100a: dQ, dK, dV of the tiled forward, from the
// forward's O and log-sum-exp L and the upstream gradient dO.
//
// The xformers page pairs every forward operator with a backward operator,
// and the FlashAttention-2 page reports training throughput; the method's
// backward recomputes the probabilities tile by tile from L instead of
// storing the N x N matrix:
//     P = exp(scale Q K^T - L)            (masked entries 0)
//     dV = P^T dO,  dP = dO V^T,  dS = P o (dP - Delta),  Delta = rowsum(dO o O)
//     dQ = scale dS K,  dK = scale dS^T Q
// Three kernels, each with one owner per output element (no atomics):
//  * fa_bwd_delta_kernel: Delta[b, h, i] = sum_d dO o O (fp32), one warp a row;
//  * fa_bwd_dq_kernel: one CTA per (128-row query tile, head, batch) walks the
//    K/V tiles: S = Q K_j^T and dP = dO V_j^T into tensor memory, the softmax
//    warps form dS, then dQ += dS K_j (A = dS from tensor memory);
//  * fa_bwd_dkdv_kernel: one CTA per (128-key K/V tile, kv head, batch) walks
//    the query tiles of all G heads of its group: S^T = K Q_i^T and
//    dP^T = V dO_i^T, the softmax warps form P^T and dS^T, then
//    dV += P^T dO_i and dK += dS^T Q_i.
// The products are tcgen05 MMAs of the forward's kinds: shared-memory
// operands K-major (S, dP, S^T, dP^T), the second operand read MN-major from
// the same tiles (dQ, dV, dK), the first operand from tensor memory.  S and
// dP are recomputed in both walks (seven 128x128xD products per tile pair
// instead of five) in exchange for no atomics and no extra buffers.
// Load, MMA and softmax roles follow the forward's warp specialisation; every
// mbarrier wait is bounded.  Overlap within a walk: the next S (S^T) product
// is issued as soon as the softmax warps have read the current one, so it
// runs while they form dS; in the dQ walk dP alternates between two
// tensor-memory buffers so dP_j+1 can follow S_j+1 without waiting for dQ_j.
// K and V (Q and dO) stream through separate TMA rings sized by when each
// tile is released.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
#include "fa_kernels.h"

namespace ta23 {
namespace {

constexpr int BM = 128;   // query rows per tile, and keys per K/V tile
constexpr float kLog2e = 1.4426950408889634f;

constexpr uint32_t kDescHi = (uint32_t)((1024u >> 4) | (1u << 14) | (2u << 29));
__device__ __forceinline__ uint64_t desc_from_lo(uint32_t lo) { return ((uint64_t)kDescHi << 32) | lo; }

// Time-bounded wait that ignores the abort flag (used only to drain).
__device__ __forceinline__ void wait_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > FA_WAIT_LIMIT_NS) {
      atomicOr(&g_device_status, kStatusWaitTimeout);
      return;
    }
  }
}

// D[tmem] (+)= A B^T for a 128 x N x DC product, A (128 rows) and B (N rows)
// K-major 128-byte swizzled tiles in blocks of 64 columns (A's blocks 128*128
// bytes apart, B's N*128); a_lo / b_lo: start address >> 4.
template <int DC, int N = BM>
__device__ __forceinline__ void mma_kmajor(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo) {
  constexpr uint32_t id = idesc_bf16_f32(BM, N, 0, 0);
  constexpr uint32_t kABlock = BM * 128, kBBlock = N * 128;
  constexpr uint32_t kLbo = 1u << 16;
#pragma unroll
  for (int kk = 0; kk < DC / 16; ++kk) {
    const uint32_t ao = ((kk >> 2) * kABlock + (kk & 3) * 32) >> 4;
    const uint32_t bo = ((kk >> 2) * kBBlock + (kk & 3) * 32) >> 4;
    mma_bf16_ss(d_tmem, desc_from_lo((a_lo + ao) | kLbo), desc_from_lo((b_lo + bo) | kLbo), id, kk > 0 ? 1u : 0u);
  }
}

// D[tmem] (+)= A B for a 128 x D x KC product: A (128 x KC, bf16) from tensor
// memory at a_tmem (two values per column), B a KC-row tile read MN-major
// (rows = the contraction, D columns in 64-column blocks KC*128 bytes apart).
template <int D, int KC = BM>
__device__ __forceinline__ void mma_tmem_mn(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, bool first) {
  constexpr uint32_t id = idesc_bf16_f32(BM, D, 0, 1);
  constexpr uint32_t kLbo = (uint32_t)((KC * 128) >> 4) << 16;   // next 64-column block
#pragma unroll
  for (int kk = 0; kk < KC / 16; ++kk)
    mma_bf16_ts(d_tmem, a_tmem + kk * 8, desc_from_lo((b_lo + ((kk * 16 * 128) >> 4)) | kLbo), id,
                (!first || kk > 0) ? 1u : 0u);
}

// Loads this thread's N fp32 columns of tensor memory at taddr with a single
// wait.
template <int N = BM>
__device__ __forceinline__ void load_row128(uint32_t taddr, float (&x)[N]) {
#pragma unroll
  for (int c = 0; c < N; c += 32) {
    uint32_t r[32];
    tmem_ld32(taddr + c, r);
#pragma unroll
    for (int e = 0; e < 32; ++e) x[c + e] = __uint_as_float(r[e]);
  }
  tmem_wait_ld();
#pragma unroll
  for (int e = 0; e < N; ++e) asm volatile("" : "+f"(x[e]));
}

// dS = P o (dP - Delta) over a row of N dP columns at taddr, written as bf16
// pairs over the first N/2 of those columns (each chunk of 32 lands behind
// the columns already read).  Delta is `dlt`, or per column from drow
// (PER_COL).  The next chunk's load is in flight while one is computed.
template <bool PER_COL, int N = BM>
__device__ __forceinline__ void ds_pass(uint32_t taddr, const float (&pf)[N], float dlt, const float* drow) {
  uint32_t cur[32], nxt[32];
  tmem_ld32(taddr, cur);
  tmem_wait_ld();
#pragma unroll
  for (int c = 0; c < N; c += 32) {
    if (c + 32 < N) tmem_ld32(taddr + c + 32, nxt);
#pragma unroll
    for (int e = 0; e < 32; ++e) asm volatile("" : "+r"(cur[e]));
    float dc[32];
    if (PER_COL) {
#pragma unroll
      for (int e = 0; e < 32; e += 4) *reinterpret_cast<float4*>(&dc[e]) = *reinterpret_cast<const float4*>(&drow[c + e]);
    }
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float d0 = PER_COL ? dc[2 * e] : dlt, d1 = PER_COL ? dc[2 * e + 1] : dlt;
      pk[e] = pack_bf16x2(pf[c + 2 * e] * (__uint_as_float(cur[2 * e]) - d0),
                          pf[c + 2 * e + 1] * (__uint_as_float(cur[2 * e + 1]) - d1));
    }
    tmem_st16(taddr + c / 2, pk);
    if (c + 32 < N) {
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e) cur[e] = nxt[e];
    }
  }
}

// Writes a row of D fp32 columns of tensor memory, times `mul`, as bf16.
template <int D>
__device__ __forceinline__ void store_row_bf16(uint32_t taddr, float mul, __nv_bfloat16* row, bool ok) {
#pragma unroll 1
  for (int c = 0; c < D; c += 32) {
    uint32_t r[32];
    tmem_ld32(taddr + c, r);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 32; ++e) asm volatile("" : "+r"(r[e]));
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e)
      pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * mul, __uint_as_float(r[2 * e + 1]) * mul);
    if (ok) {
      uint4* dst = reinterpret_cast<uint4*>(row + c);
#pragma unroll
      for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
    }
  }
}

// TMA load of a tile of `rows` rows x D columns (row `row0` of a [B, L, H, D]
// tensor, head h, batch b) into D/64 swizzled blocks of rows x 128 bytes, in
// boxes of BOX rows (the tensor map's box height).
template <int D, int BOX>
__device__ __forceinline__ void load_tile(unsigned char* dst, const CUtensorMap* tm, uint64_t* bar, int rows, int h,
                                          int row0, int b, uint64_t pol) {
#pragma unroll
  for (int db = 0; db < D / 64; ++db)
    for (int r0 = 0; r0 < rows; r0 += BOX)
      tma_load_4d_hint(dst + db * rows * 128 + r0 * 128, tm, bar, db * 64, h, row0 + r0, b, pol);
}

// ===========================================================================
// Delta = rowsum(dO o O)
// ===========================================================================
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_delta_kernel(const __nv_bfloat16* __restrict__ o,
                                                           const __nv_bfloat16* __restrict__ dout,
                                                           float* __restrict__ delta, BwdParams p) {
  const int64_t row = (int64_t)blockIdx.x * 8 + threadIdx.x / 32;   // (b * Lq + i) * Hq + h
  const int lane = threadIdx.x % 32;
  if (row >= (int64_t)p.B * p.Lq * p.Hq) return;
  constexpr int PER = D / 32;
  const __nv_bfloat16* orow = o + row * D + lane * PER;
  const __nv_bfloat16* drow = dout + row * D + lane * PER;
  float acc = 0.f;
#pragma unroll
  for (int e = 0; e < PER; ++e) acc = fmaf(__bfloat162float(orow[e]), __bfloat162float(drow[e]), acc);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) {
    const int h = (int)(row % p.Hq);
    const int64_t bi = row / p.Hq;
    const int i = (int)(bi % p.Lq);
    const int64_t b = bi / p.Lq;
    delta[(b * p.Hq + h) * p.Lq + i] = acc;
  }
}

// ===========================================================================
// dQ: one CTA per (query tile, head, batch)
// ===========================================================================
// BN keys per K/V tile: 128, or 64 at head_dim 256 (where a 128-row tile of
// Q or dO alone is 64 KB and dQ fills 256 tensor-memory columns).
template <int D, int BN>
struct DqCfg {
  static constexpr int kDBlocks = D / 64;
  static constexpr int kQTileBytes = kDBlocks * BM * 128;    // Q or dO: 128 rows of D columns
  static constexpr int kKVTileBytes = kDBlocks * BN * 128;   // K or V: BN rows
  static constexpr int kBox = D == 256 ? 64 : 128;           // rows per TMA box of the tensor maps
  // K and V rings: K_j is read by S_j and, a step later, by dQ_j; V_j only
  // by dP_j, so V needs the shallower ring.
  static constexpr int kKSlots = D == 64 ? 6 : D == 128 ? 3 : 2;
  static constexpr int kVSlots = D == 64 ? 4 : D == 128 ? 2 : 1;
  static constexpr int kThreads = 192;                     // load, MMA, 4 softmax warps
  // tensor-memory columns: S, dQ, and dP in two buffers (dP_j in buffer j % 2;
  // dS_j is written over the first BN/2 columns of its dP)
  static constexpr int kS = 0, kDQ = 256, kDP0 = BN, kDP1 = BN == 128 ? 384 : 2 * BN;
  static constexpr int kSmemBytes = 2 * kQTileBytes + (kKSlots + kVSlots) * kKVTileBytes + 512 + 1024;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static_assert(kDQ + D <= 512 && (BN == 128 || kDP1 + BN <= kDQ), "tensor-memory budget");
};

struct DqBarriers {
  uint64_t qd_full;     // Q and dO
  uint64_t s_full;      // S_j in tensor memory
  uint64_t s_free;      // S_j read by the softmax warps (4 warps)
  uint64_t dp_full[2];  // dP_j in its buffer (one barrier per buffer)
  uint64_t ds_full[2];  // dS_j in its buffer (4 warps)
  uint64_t o_full;      // the last dQ product has landed
  uint64_t drain;
  uint64_t k_full[6];
  uint64_t k_empty[6];
  uint64_t v_full[4];
  uint64_t v_empty[4];
  uint32_t tmem_base;
  int abort_flag;
};

template <int D, int BN, bool CAUSAL>
__global__ void __launch_bounds__(DqCfg<D, BN>::kThreads, 1)
fa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO, BwdParams p) {
  using Cfg = DqCfg<D, BN>;
  constexpr int KS = Cfg::kKSlots, VS = Cfg::kVSlots, BOX = Cfg::kBox;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sQ = base;
  unsigned char* sDO = base + Cfg::kQTileBytes;
  unsigned char* sK = base + 2 * Cfg::kQTileBytes;         // K ring
  unsigned char* sV = sK + KS * Cfg::kKVTileBytes;         // V ring
  DqBarriers& bar = *reinterpret_cast<DqBarriers*>(sV + VS * Cfg::kKVTileBytes);
  volatile int* abortf = &bar.abort_flag;

  const int warp = __shfl_sync(0xffffffffu, (int)threadIdx.x / 32, 0), lane = threadIdx.x % 32;
  const int q_tile = p.n_qtiles - 1 - blockIdx.x;   // longest causal rows first
  const int h = blockIdx.y, b = blockIdx.z, hkv = h / p.G;
  const int q0 = q_tile * BM;
  int n_kv = (p.Lk + BN - 1) / BN;
  if (CAUSAL) n_kv = min(n_kv, (min(q0 + BM, p.Lq) - 1 + p.causal_off) / BN + 1);

  if (threadIdx.x == 0) {
    bar.abort_flag = 0;
    mbar_init(&bar.qd_full, 1);
    mbar_init(&bar.s_full, 1);
    mbar_init(&bar.s_free, 4);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar.dp_full[i], 1);
      mbar_init(&bar.ds_full[i], 4);
    }
    mbar_init(&bar.o_full, 1);
    mbar_init(&bar.drain, 1);
    for (int i = 0; i < KS; ++i) {
      mbar_init(&bar.k_full[i], 1);
      mbar_init(&bar.k_empty[i], 1);
    }
    for (int i = 0; i < VS; ++i) {
      mbar_init(&bar.v_full[i], 1);
      mbar_init(&bar.v_empty[i], 1);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bar.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar.tmem_base;

  if (warp == 0) {
    // ---------------------------------------------------------- load warp
    const uint64_t pol_kv = l2_policy_evict_last();
    const uint64_t pol_q = l2_policy_evict_first();
    if (elect_one()) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      mbar_arrive_expect_tx(&bar.qd_full, 2 * Cfg::kQTileBytes);
      load_tile<D, BOX>(sQ, &tmQ, &bar.qd_full, BM, h, q0, b, pol_q);
      load_tile<D, BOX>(sDO, &tmDO, &bar.qd_full, BM, h, q0, b, pol_q);
    }
    __syncwarp();
    int k_issued = 0, v_issued = 0;
    bool ok = true;
    for (int j = 0; j < n_kv && ok; ++j) {   // K_j then V_j, each into its own ring
      if (j >= KS) ok = __all_sync(0xffffffffu, mbar_wait(&bar.k_empty[j % KS], (j / KS - 1) & 1, abortf));
      if (!ok) break;
      if (elect_one()) {
        mbar_arrive_expect_tx(&bar.k_full[j % KS], Cfg::kKVTileBytes);
        load_tile<D, BOX>(sK + (j % KS) * Cfg::kKVTileBytes, &tmK, &bar.k_full[j % KS], BN, hkv, j * BN, b, pol_kv);
      }
      __syncwarp();
      ++k_issued;
      if (j >= VS) ok = __all_sync(0xffffffffu, mbar_wait(&bar.v_empty[j % VS], (j / VS - 1) & 1, abortf));
      if (!ok) break;
      if (elect_one()) {
        mbar_arrive_expect_tx(&bar.v_full[j % VS], Cfg::kKVTileBytes);
        load_tile<D, BOX>(sV + (j % VS) * Cfg::kKVTileBytes, &tmV, &bar.v_full[j % VS], BN, hkv, j * BN, b, pol_kv);
      }
      __syncwarp();
      ++v_issued;
    }
    if (!ok) {
      wait_drain(&bar.qd_full, 0);
      for (int j = (k_issued > KS ? k_issued - KS : 0); j < k_issued; ++j) wait_drain(&bar.k_full[j % KS], (j / KS) & 1);
      for (int j = (v_issued > VS ? v_issued - VS : 0); j < v_issued; ++j) wait_drain(&bar.v_full[j % VS], (j / VS) & 1);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA warp
    // S_j+1 goes in as soon as the softmax warps have read S_j (s_free), so
    // it runs while they form dS_j; dP_j+1 overwrites the columns dS_j was
    // read from and follows dQ_j.
    const uint32_t q_lo = smem_u32(sQ) >> 4, do_lo = smem_u32(sDO) >> 4;
    const uint32_t k_lo0 = smem_u32(sK) >> 4, v_lo0 = smem_u32(sV) >> 4;
    auto k_lo = [&](int j) { return k_lo0 + (uint32_t)((j % KS) * Cfg::kKVTileBytes >> 4); };
    auto v_lo = [&](int j) { return v_lo0 + (uint32_t)((j % VS) * Cfg::kKVTileBytes >> 4); };
    auto wait_k = [&](int j) { return mbar_wait(&bar.k_full[j % KS], (j / KS) & 1, abortf); };
    auto wait_v = [&](int j) { return mbar_wait(&bar.v_full[j % VS], (j / VS) & 1, abortf); };
    bool ok = __all_sync(0xffffffffu, mbar_wait(&bar.qd_full, 0, abortf));
    if (ok && n_kv > 0) {
      ok = __all_sync(0xffffffffu, wait_k(0) && wait_v(0));
      if (ok) {
        tc_fence_after();
        if (elect_one()) {
          mma_kmajor<D, BN>(tmem + Cfg::kS, q_lo, k_lo(0));        // S_0 = Q K_0^T
          tc_commit(&bar.s_full);
          mma_kmajor<D, BN>(tmem + Cfg::kDP0, do_lo, v_lo(0));     // dP_0 = dO V_0^T
          tc_commit(&bar.dp_full[0]);
          tc_commit(&bar.v_empty[0]);                          // V_0 read
        }
        __syncwarp();
      }
    }
    // dP_j+1 goes into the other buffer right behind S_j+1 (its previous
    // contents, dS_j-1, were read by dQ_j-1, issued before), so the softmax
    // warps find it ready after their pass 1 and dQ_j stays off their path.
    for (int j = 0; j < n_kv && ok; ++j) {
      const bool more = j + 1 < n_kv;
      if (more) {
        ok = __all_sync(0xffffffffu, wait_k(j + 1) && mbar_wait(&bar.s_free, j & 1, abortf) && wait_v(j + 1));
        if (!ok) break;
        tc_fence_after();
        if (elect_one()) {
          mma_kmajor<D, BN>(tmem + Cfg::kS, q_lo, k_lo(j + 1));   // S_j+1 = Q K_j+1^T
          tc_commit(&bar.s_full);
          mma_kmajor<D, BN>(tmem + ((j + 1) & 1 ? Cfg::kDP1 : Cfg::kDP0), do_lo, v_lo(j + 1));   // dP_j+1
          tc_commit(&bar.dp_full[(j + 1) & 1]);
          tc_commit(&bar.v_empty[(j + 1) % VS]);              // V_j+1 read
        }
        __syncwarp();
      }
      ok = __all_sync(0xffffffffu, mbar_wait(&bar.ds_full[j & 1], (j >> 1) & 1, abortf));
      if (!ok) break;
      tc_fence_after();
      if (elect_one()) {
        mma_tmem_mn<D, BN>(tmem + Cfg::kDQ, tmem + (j & 1 ? Cfg::kDP1 : Cfg::kDP0), k_lo(j), j == 0);   // dQ += dS_j K_j
        tc_commit(&bar.k_empty[j % KS]);                                                         // K_j read
        if (!more) tc_commit(&bar.o_full);
      }
      __syncwarp();
    }
    if (!ok) {
      if (elect_one()) tc_commit(&bar.drain);
      __syncwarp();
      wait_drain(&bar.drain, 0);
    }
  } else {
    // ---------------------------------------------------------- softmax warps (one query row each)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int qi = q0 + r;
    const bool row_ok = qi < p.Lq;
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    const int64_t lrow = ((int64_t)b * p.Hq + h) * p.Lq + qi;
    const float lse2 = row_ok ? p.lse[lrow] * kLog2e : 0.f;
    const float dlt = row_ok ? p.delta[lrow] : 0.f;
    const float sl2 = p.scale_log2;
    int key_limit = p.Lk - 1;
    if (CAUSAL) key_limit = min(key_limit, qi + p.causal_off);
    bool ok = true;
    for (int j = 0; j < n_kv && ok; ++j) {
      // Pass 1: P = 2^(S scale log2e - L) in fp32 (the whole row loaded with
      // one wait), then S is released.
      ok = mbar_wait(&bar.s_full, j & 1, abortf);
      if (!ok) break;
      tc_fence_after();
      float pf[BN];
      load_row128<BN>(tmem + lane_addr + Cfg::kS, pf);
      const int lim = row_ok ? key_limit - j * BN : -1;   // columns e <= lim are allowed keys
#pragma unroll
      for (int e = 0; e < BN; e += 2) {
        const float2 x = __ffma2_rn(make_float2(pf[e], pf[e + 1]), make_float2(sl2, sl2),
                                    make_float2(-lse2, -lse2));
        const float2 pv = make_float2(ex2_approx(x.x), ex2_approx(x.y));
        pf[e] = e <= lim ? pv.x : 0.f;
        pf[e + 1] = e + 1 <= lim ? pv.y : 0.f;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.s_free);
      // Pass 2: dS = P o (dP - Delta), over the dP columns already read.
      ok = mbar_wait(&bar.dp_full[j & 1], (j >> 1) & 1, abortf);
      if (!ok) break;
      tc_fence_after();
      ds_pass<false, BN>(tmem + lane_addr + (j & 1 ? Cfg::kDP1 : Cfg::kDP0), pf, dlt, nullptr);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.ds_full[j & 1]);
    }
    if (ok && n_kv > 0) ok = mbar_wait(&bar.o_full, 0, abortf);
    if (ok) {
      __nv_bfloat16* row = reinterpret_cast<__nv_bfloat16*>(p.dq) + (((int64_t)b * p.Lq + qi) * p.Hq + h) * D;
      if (n_kv > 0) {
        tc_fence_after();
        store_row_bf16<D>(tmem + lane_addr + Cfg::kDQ, p.scale, row, row_ok);
      } else if (row_ok) {
        for (int c = 0; c < D; c += 8) *reinterpret_cast<uint4*>(row + c) = make_uint4(0, 0, 0, 0);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ===========================================================================
// dK, dV: one CTA per (K/V tile, kv head, batch), over the group's query tiles
// ===========================================================================
// PASS 0 computes dV and dK in one walk (head_dim 64 and 128).  At head_dim
// 256, dV and dK fill all 512 tensor-memory columns by themselves, so they
// take one walk each over BQ = 64-row query tiles: PASS 1 forms P^T and
// dV += P^T dO; PASS 2 forms dP^T, dS^T and dK += dS^T Q (S^T is recomputed
// in both).
template <int D, int BQ, int PASS>
struct DkvCfg {
  static constexpr int kDBlocks = D / 64;
  static constexpr int kKTileBytes = kDBlocks * BM * 128;    // K or V: 128 keys of D columns
  static constexpr int kQTileBytes = kDBlocks * BQ * 128;    // Q or dO: BQ query rows
  static constexpr int kBox = D == 256 ? 64 : 128;           // rows per TMA box of the tensor maps
  static constexpr bool kNeedV = PASS != 1;
  static constexpr int kThreads = 192;
  // tensor-memory columns: S^T (BQ), then dP^T (BQ; dS^T over its first BQ/2
  // and, in PASS 0, P^T over the other BQ/2), or in PASS 1 P^T (BQ/2); dV, dK
  static constexpr int kST = 0, kDPT = BQ, kPT = BQ;
  static constexpr int kDV = 256, kDK = PASS == 0 ? 256 + D : 256;
  // Separate rings for Q_i and dO_i.  Q_i+1 is needed one MMA group before
  // dO_i+1 (S^T_i+1 is issued ahead of dP^T_i+1), so Q gets the deeper ring.
  static constexpr int kQStages = D == 64 ? 4 : D == 128 ? 3 : 2;
  static constexpr int kDOStages = D == 64 ? 4 : D == 128 ? 2 : (PASS == 1 ? 2 : 1);
  static constexpr int kRowBytes = 2 * BQ * 4;                         // L and Delta of one step
  static constexpr int kSmemBytes = (kNeedV ? 2 : 1) * kKTileBytes + (kQStages + kDOStages) * kQTileBytes +
                                    kRowBytes + 512 + 1024;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static_assert(PASS == 0 ? kDK + D <= 512 : (kDV + D <= 512 && kDPT + BQ <= kDV), "tensor-memory budget");
};

struct DkvBarriers {
  uint64_t kv_full;         // K and V
  uint64_t q_full[4];       // Q_i per ring slot
  uint64_t q_empty[4];
  uint64_t do_full[4];      // dO_i per ring slot
  uint64_t do_empty[4];
  uint64_t st_full;         // S^T in tensor memory
  uint64_t st_free;         // S^T read by the softmax warps (4 warps)
  uint64_t dpt_full;        // dP^T in tensor memory
  uint64_t p_full;          // P^T and/or dS^T in tensor memory (4 warps)
  uint64_t pt_free;         // PASS 1: the dV product has read P^T
  uint64_t o_full;          // the last dV / dK products have landed
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <int D, int BQ, int PASS, bool CAUSAL>
__global__ void __launch_bounds__(DkvCfg<D, BQ, PASS>::kThreads, 1)
fa_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO, BwdParams p) {
  using Cfg = DkvCfg<D, BQ, PASS>;
  constexpr int BOX = Cfg::kBox;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sK = base;
  unsigned char* sV = base + Cfg::kKTileBytes;                              // unused in PASS 1
  unsigned char* sQr = base + (Cfg::kNeedV ? 2 : 1) * Cfg::kKTileBytes;     // Q ring
  unsigned char* sDOr = sQr + Cfg::kQStages * Cfg::kQTileBytes;             // dO ring
  float* sRow = reinterpret_cast<float*>(sDOr + Cfg::kDOStages * Cfg::kQTileBytes);   // [L2, Delta][BQ]
  DkvBarriers& bar = *reinterpret_cast<DkvBarriers*>(reinterpret_cast<unsigned char*>(sRow) + Cfg::kRowBytes);
  volatile int* abortf = &bar.abort_flag;

  const int warp = __shfl_sync(0xffffffffu, (int)threadIdx.x / 32, 0), lane = threadIdx.x % 32;
  const int kv_tile = blockIdx.x, hkv = blockIdx.y, b = blockIdx.z;
  const int k0 = kv_tile * BM;
  const int n_qt = (p.Lq + BQ - 1) / BQ;
  // causal: query tiles whose last row reaches this tile's first key
  const int i_start = CAUSAL ? min(n_qt, max(0, k0 - p.causal_off) / BQ) : 0;
  const int per_head = n_qt - i_start;
  const int T = p.G * per_head;   // steps: (head of the group, query tile)

  if (threadIdx.x == 0) {
    bar.abort_flag = 0;
    mbar_init(&bar.kv_full, 1);
    for (int s = 0; s < 4; ++s) {
      mbar_init(&bar.q_full[s], 1);
      mbar_init(&bar.q_empty[s], 1);
      mbar_init(&bar.do_full[s], 1);
      mbar_init(&bar.do_empty[s], 1);
    }
    mbar_init(&bar.st_full, 1);
    mbar_init(&bar.st_free, 4);
    mbar_init(&bar.dpt_full, 1);
    mbar_init(&bar.p_full, 4);
    mbar_init(&bar.pt_free, 1);
    mbar_init(&bar.o_full, 1);
    mbar_init(&bar.drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bar.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar.tmem_base;

  if (warp == 0) {
    // ---------------------------------------------------------- load warp
    const uint64_t pol_kv = l2_policy_evict_first();
    const uint64_t pol_q = l2_policy_evict_last();
    if (elect_one()) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      mbar_arrive_expect_tx(&bar.kv_full, (Cfg::kNeedV ? 2 : 1) * Cfg::kKTileBytes);
      load_tile<D, BOX>(sK, &tmK, &bar.kv_full, BM, hkv, k0, b, pol_kv);
      if (Cfg::kNeedV) load_tile<D, BOX>(sV, &tmV, &bar.kv_full, BM, hkv, k0, b, pol_kv);
    }
    __syncwarp();
    constexpr int QS = Cfg::kQStages, DS = Cfg::kDOStages;
    int q_issued = 0, do_issued = 0;
    bool ok = true;
    // Q_t then dO_t for every step; each waits for its own ring slot.
    for (int t = 0; t < T && ok; ++t) {
      const int h = hkv * p.G + t / per_head, qt = i_start + t % per_head;
      if (t >= QS) ok = __all_sync(0xffffffffu, mbar_wait(&bar.q_empty[t % QS], (t / QS - 1) & 1, abortf));
      if (!ok) break;
      if (elect_one()) {
        mbar_arrive_expect_tx(&bar.q_full[t % QS], Cfg::kQTileBytes);
        load_tile<D, BOX>(sQr + (t % QS) * Cfg::kQTileBytes, &tmQ, &bar.q_full[t % QS], BQ, h, qt * BQ, b, pol_q);
      }
      __syncwarp();
      ++q_issued;
      if (t >= DS) ok = __all_sync(0xffffffffu, mbar_wait(&bar.do_empty[t % DS], (t / DS - 1) & 1, abortf));
      if (!ok) break;
      if (elect_one()) {
        mbar_arrive_expect_tx(&bar.do_full[t % DS], Cfg::kQTileBytes);
        load_tile<D, BOX>(sDOr + (t % DS) * Cfg::kQTileBytes, &tmDO, &bar.do_full[t % DS], BQ, h, qt * BQ, b,
                          pol_q);
      }
      __syncwarp();
      ++do_issued;
    }
    if (!ok) {
      wait_drain(&bar.kv_full, 0);
      for (int t = (q_issued > QS ? q_issued - QS : 0); t < q_issued; ++t) wait_drain(&bar.q_full[t % QS], (t / QS) & 1);
      for (int t = (do_issued > DS ? do_issued - DS : 0); t < do_issued; ++t)
        wait_drain(&bar.do_full[t % DS], (t / DS) & 1);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA warp
    // S^T_t+1 goes in as soon as the softmax warps have read S^T_t (st_free)
    // and runs while they form the step's P^T / dS^T.  PASS 0 and 2: dP^T_t+1
    // overwrites the columns dS^T_t (and P^T_t) were read from, so it follows
    // the step's dV / dK products.
    constexpr int QS = Cfg::kQStages, DS = Cfg::kDOStages;
    const uint32_t k_lo = smem_u32(sK) >> 4, v_lo = smem_u32(sV) >> 4;
    const uint32_t q_lo0 = smem_u32(sQr) >> 4, do_lo0 = smem_u32(sDOr) >> 4;
    auto q_of = [&](int t) { return q_lo0 + (uint32_t)((t % QS) * Cfg::kQTileBytes >> 4); };
    auto do_of = [&](int t) { return do_lo0 + (uint32_t)((t % DS) * Cfg::kQTileBytes >> 4); };
    auto wait_q = [&](int t) { return mbar_wait(&bar.q_full[t % QS], (t / QS) & 1, abortf); };
    auto wait_do = [&](int t) { return mbar_wait(&bar.do_full[t % DS], (t / DS) & 1, abortf); };
    bool ok = __all_sync(0xffffffffu, mbar_wait(&bar.kv_full, 0, abortf));
    if (ok && T > 0) {
      ok = __all_sync(0xffffffffu, wait_q(0) && (PASS == 1 || wait_do(0)));
      if (ok) {
        tc_fence_after();
        if (elect_one()) {
          mma_kmajor<D, BQ>(tmem + Cfg::kST, k_lo, q_of(0));     // S^T_0 = K Q_0^T
          tc_commit(&bar.st_full);
          if (PASS == 1) tc_commit(&bar.q_empty[0]);              // Q_0 read (PASS 1: by S^T only)
          if (PASS != 1) {
            mma_kmajor<D, BQ>(tmem + Cfg::kDPT, v_lo, do_of(0));   // dP^T_0 = V dO_0^T
            tc_commit(&bar.dpt_full);
            if (PASS == 2) tc_commit(&bar.do_empty[0]);            // dO_0 read (PASS 2: by dP^T only)
          }
        }
        __syncwarp();
      }
    }
    for (int t = 0; t < T && ok; ++t) {
      const bool more = t + 1 < T;
      if (more) {
        ok = __all_sync(0xffffffffu, wait_q(t + 1) && mbar_wait(&bar.st_free, t & 1, abortf));
        if (!ok) break;
        tc_fence_after();
        if (elect_one()) {
          mma_kmajor<D, BQ>(tmem + Cfg::kST, k_lo, q_of(t + 1));   // S^T_t+1
          tc_commit(&bar.st_full);
          if (PASS == 1) tc_commit(&bar.q_empty[(t + 1) % QS]);
        }
        __syncwarp();
      }
      ok = __all_sync(0xffffffffu, mbar_wait(&bar.p_full, t & 1, abortf) && (PASS != 1 || wait_do(t)));
      if (!ok) break;
      tc_fence_after();
      if (elect_one()) {
        if (PASS == 0) {
          mma_tmem_mn<D, BQ>(tmem + Cfg::kDV, tmem + Cfg::kDPT + BQ / 2, do_of(t), t == 0);   // dV += P^T dO_t
          mma_tmem_mn<D, BQ>(tmem + Cfg::kDK, tmem + Cfg::kDPT, q_of(t), t == 0);             // dK += dS^T Q_t
          tc_commit(&bar.q_empty[t % QS]);
          tc_commit(&bar.do_empty[t % DS]);
        } else if (PASS == 1) {
          mma_tmem_mn<D, BQ>(tmem + Cfg::kDV, tmem + Cfg::kPT, do_of(t), t == 0);   // dV += P^T dO_t
          tc_commit(&bar.do_empty[t % DS]);
          tc_commit(&bar.pt_free);
        } else {
          mma_tmem_mn<D, BQ>(tmem + Cfg::kDK, tmem + Cfg::kDPT, q_of(t), t == 0);   // dK += dS^T Q_t
          tc_commit(&bar.q_empty[t % QS]);
        }
        if (!more) tc_commit(&bar.o_full);
      }
      __syncwarp();
      if (PASS != 1 && more) {
        ok = __all_sync(0xffffffffu, wait_do(t + 1));
        if (!ok) break;
        tc_fence_after();
        if (elect_one()) {
          mma_kmajor<D, BQ>(tmem + Cfg::kDPT, v_lo, do_of(t + 1));   // dP^T_t+1
          tc_commit(&bar.dpt_full);
          if (PASS == 2) tc_commit(&bar.do_empty[(t + 1) % DS]);
        }
        __syncwarp();
      }
    }
    if (!ok) {
      if (elect_one()) tc_commit(&bar.drain);
      __syncwarp();
      wait_drain(&bar.drain, 0);
    }
  } else {
    // ---------------------------------------------------------- softmax warps (one key row each)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;        // 0..127 within the softmax warps
    const int key = k0 + r;
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    const float sl2 = p.scale_log2;
    // Every thread passes the named barrier once per step, also after a failed
    // wait (it then skips the work), so no thread waits on a barrier another
    // one has left.
    bool ok = true;
    // L (base 2) and Delta of the query rows of step t (thread r < BQ loads
    // row r): loaded one step ahead, so their global-memory latency stays off
    // the step.
    auto fetch_rows = [&](int t, float& l2, float& dl) {
      l2 = 0.f;
      dl = 0.f;
      if (t >= T || r >= BQ) return;
      const int h = hkv * p.G + t / per_head, qi = (i_start + t % per_head) * BQ + r;
      if (qi < p.Lq) {   // raw values: nothing waits on the loads until the next step
        const int64_t lrow = ((int64_t)b * p.Hq + h) * p.Lq + qi;
        l2 = __ldg(p.lse + lrow);
        if (PASS != 1) dl = __ldg(p.delta + lrow);
      }
    };
    float next_l2, next_dl;
    fetch_rows(0, next_l2, next_dl);
    for (int t = 0; t < T; ++t) {
      const int qt = i_start + t % per_head;
      const int i0 = qt * BQ;
      // the tile's L and Delta, staged for all 128 threads (one buffer: the
      // second barrier below keeps the next step's writes behind every read)
      float* rows = sRow;
      if (r < BQ) {
        rows[r] = next_l2 * kLog2e;
        rows[BQ + r] = next_dl;
      }
      fetch_rows(t + 1, next_l2, next_dl);
      named_barrier_sync(1, 128);
      // Pass 1: P^T from S^T, kept in fp32 until dS^T is formed; S^T released.
      ok = ok && mbar_wait(&bar.st_full, t & 1, abortf);
      if (!ok) {
        named_barrier_sync(1, 128);
        continue;
      }
      tc_fence_after();
      // query q (column) may be attended by this key iff q < Lq and, causal, key <= q + off
      float pf[BQ];
      load_row128<BQ>(tmem + lane_addr + Cfg::kST, pf);
      // the columns' L in chunks of 32 (eight 128-bit shared loads issued
      // together), so no exponential waits on a load of its own
      // allowed columns: lo <= column < lo + span (q < Lq and, causal, key <= q + off)
      const int lo = CAUSAL ? max(key - p.causal_off - i0, 0) : 0;
      const int hi = min(p.Lq - i0, BQ);
      const uint32_t span = hi > lo ? (uint32_t)(hi - lo) : 0u;
#pragma unroll
      for (int c = 0; c < BQ; c += 32) {
        float lc[32];
#pragma unroll
        for (int e = 0; e < 32; e += 4) *reinterpret_cast<float4*>(&lc[e]) = *reinterpret_cast<const float4*>(&rows[c + e]);
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const float2 x = __ffma2_rn(make_float2(pf[c + e], pf[c + e + 1]), make_float2(sl2, sl2),
                                      make_float2(-lc[e], -lc[e + 1]));
          const float p0 = ex2_approx(x.x), p1 = ex2_approx(x.y);
          pf[c + e] = (uint32_t)(c + e - lo) < span ? p0 : 0.f;
          pf[c + e + 1] = (uint32_t)(c + e + 1 - lo) < span ? p1 : 0.f;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.st_free);
      if constexpr (PASS == 1) {
        // P^T into its own columns, once the previous dV product has read them.
        named_barrier_sync(1, 128);   // every thread has read this step's rows
        ok = t == 0 || mbar_wait(&bar.pt_free, (t - 1) & 1, abortf);
        if (!ok) continue;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < BQ; c += 32) {
          uint32_t pp[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) pp[e] = pack_bf16x2(pf[c + 2 * e], pf[c + 2 * e + 1]);
          tmem_st16(tmem + lane_addr + Cfg::kPT + c / 2, pp);
        }
      } else {
        // Pass 2: dS^T = P^T o (dP^T - Delta) into dP^T columns 0..BQ/2 (behind
        // the reads), then (PASS 0) P^T into the other half once every column
        // is read.
        ok = mbar_wait(&bar.dpt_full, t & 1, abortf);
        if (!ok) {
          named_barrier_sync(1, 128);
          continue;
        }
        tc_fence_after();
        ds_pass<true, BQ>(tmem + lane_addr + Cfg::kDPT, pf, 0.f, rows + BQ);
        named_barrier_sync(1, 128);   // every thread has read this step's rows
        if constexpr (PASS == 0) {
#pragma unroll
          for (int c = 0; c < BQ; c += 32) {
            uint32_t pp[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) pp[e] = pack_bf16x2(pf[c + 2 * e], pf[c + 2 * e + 1]);
            tmem_st16(tmem + lane_addr + Cfg::kDPT + BQ / 2 + c / 2, pp);
          }
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.p_full);
    }
    if (ok && T > 0) ok = mbar_wait(&bar.o_full, 0, abortf);
    if (ok) {
      const bool row_ok = key < p.Lk;
      const int64_t off = (((int64_t)b * p.Lk + key) * p.Hkv + hkv) * D;
      __nv_bfloat16* dvrow = reinterpret_cast<__nv_bfloat16*>(p.dv) + off;
      __nv_bfloat16* dkrow = reinterpret_cast<__nv_bfloat16*>(p.dk) + off;
      if (T > 0) {
        tc_fence_after();
        if (PASS != 2) store_row_bf16<D>(tmem + lane_addr + Cfg::kDV, 1.f, dvrow, row_ok);
        if (PASS != 1) store_row_bf16<D>(tmem + lane_addr + Cfg::kDK, p.scale, dkrow, row_ok);
      } else if (row_ok) {
        for (int c = 0; c < D; c += 8) {
          if (PASS != 2) *reinterpret_cast<uint4*>(dvrow + c) = make_uint4(0, 0, 0, 0);
          if (PASS != 1) *reinterpret_cast<uint4*>(dkrow + c) = make_uint4(0, 0, 0, 0);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int D, int BQ, int PASS, bool CAUSAL>
cudaError_t launch_dkdv(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, const CUtensorMap& dout,
                        const BwdParams& p, cudaStream_t s) {
  using Cfg = DkvCfg<D, BQ, PASS>;
  auto kern = fa_bwd_dkdv_kernel<D, BQ, PASS, CAUSAL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
  if (e != cudaSuccess) return e;
  kern<<<dim3((p.Lk + BM - 1) / BM, p.Hkv, p.B), Cfg::kThreads, Cfg::kSmemBytes, s>>>(q, k, v, dout, p);
  return cudaGetLastError();
}

template <int D, bool CAUSAL>
cudaError_t launch_bwd_t(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, const CUtensorMap& dout,
                         BwdParams p, cudaStream_t s) {
  constexpr int BN = D == 256 ? 64 : 128;   // keys per K/V tile of the dQ walk, query rows per tile of the dK/dV walk
  const int64_t rows = (int64_t)p.B * p.Lq * p.Hq;
  fa_bwd_delta_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(static_cast<const __nv_bfloat16*>(p.o),
                                                                    static_cast<const __nv_bfloat16*>(p.dout),
                                                                    p.delta, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  {
    using Cfg = DqCfg<D, BN>;
    auto kern = fa_bwd_dq_kernel<D, BN, CAUSAL>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
    if (e != cudaSuccess) return e;
    p.n_qtiles = (p.Lq + BM - 1) / BM;
    kern<<<dim3(p.n_qtiles, p.Hq, p.B), Cfg::kThreads, Cfg::kSmemBytes, s>>>(q, k, v, dout, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if constexpr (D == 256) {
    e = launch_dkdv<D, BN, 1, CAUSAL>(q, k, v, dout, p, s);
    if (e != cudaSuccess) return e;
    return launch_dkdv<D, BN, 2, CAUSAL>(q, k, v, dout, p, s);
  } else {
    return launch_dkdv<D, BN, 0, CAUSAL>(q, k, v, dout, p, s);
  }
}

}  // namespace

cudaError_t launch_fa_bwd(int D, bool causal, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                          const CUtensorMap& dout, const BwdParams& p, cudaStream_t stream) {
  switch (D) {
    case 64: return causal ? launch_bwd_t<64, true>(q, k, v, dout, p, stream) : launch_bwd_t<64, false>(q, k, v, dout, p, stream);
    case 128:
      return causal ? launch_bwd_t<128, true>(q, k, v, dout, p, stream) : launch_bwd_t<128, false>(q, k, v, dout, p, stream);
    case 256:
      return causal ? launch_bwd_t<256, true>(q, k, v, dout, p, stream) : launch_bwd_t<256, false>(q, k, v, dout, p, stream);
    default: return cudaErrorInvalidValue;
  }
}

unsigned int bwd_read_and_clear_status() {
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof v) != cudaSuccess) return 0xFFFFFFFFu;
  cudaMemcpyToSymbol(g_device_status, &zero, sizeof zero);
  return v;
}

}  // namespace ta23
