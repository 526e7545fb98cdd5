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
// mbarrier wait is bounded.
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

// D[tmem] (+)= A B^T for a 128 x 128 x D product, A and B K-major 128-byte
// swizzled tiles of 128 rows (blocks of 64 columns at `block_bytes` apart);
// a_lo / b_lo: start address >> 4.
template <int D>
__device__ __forceinline__ void mma_kmajor(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo) {
  constexpr uint32_t id = idesc_bf16_f32(BM, BM, 0, 0);
  constexpr uint32_t kBlock = BM * 128;
  constexpr uint32_t kLbo = 1u << 16;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t o = ((kk >> 2) * kBlock + (kk & 3) * 32) >> 4;
    mma_bf16_ss(d_tmem, desc_from_lo((a_lo + o) | kLbo), desc_from_lo((b_lo + o) | kLbo), id, kk > 0 ? 1u : 0u);
  }
}

// D[tmem] (+)= A B for a 128 x D x 128 product: A (128 x 128, bf16) from
// tensor memory at a_tmem (two values per column), B a 128-row tile read
// MN-major (rows = the contraction, D columns in 64-column blocks).
template <int D>
__device__ __forceinline__ void mma_tmem_mn(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, bool first) {
  constexpr uint32_t id = idesc_bf16_f32(BM, D, 0, 1);
  constexpr uint32_t kLbo = (uint32_t)((BM * 128) >> 4) << 16;   // next 64-column block
#pragma unroll
  for (int kk = 0; kk < BM / 16; ++kk)
    mma_bf16_ts(d_tmem, a_tmem + kk * 8, desc_from_lo((b_lo + ((kk * 16 * 128) >> 4)) | kLbo), id,
                (!first || kk > 0) ? 1u : 0u);
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
template <int D>
struct DqCfg {
  static constexpr int kDBlocks = D / 64;
  static constexpr int kTileBytes = kDBlocks * BM * 128;   // one 128-row tile of D columns
  static constexpr int kSlots = D == 64 ? 10 : 5;          // K/V ring
  static constexpr int kThreads = 192;                     // load, MMA, 4 softmax warps
  static constexpr int kS = 0, kDP = 128, kDQ = 256;       // tensor-memory columns
  static constexpr int kSmemBytes = 2 * kTileBytes + kSlots * kTileBytes + 512 + 1024;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

struct DqBarriers {
  uint64_t qd_full;     // Q and dO
  uint64_t s_full;      // S_j in tensor memory
  uint64_t s_free;      // S_j read by the softmax warps (4 warps)
  uint64_t dp_full;     // dP_j in tensor memory
  uint64_t ds_full;     // dS_j in tensor memory (4 warps)
  uint64_t o_full;      // the last dQ product has landed
  uint64_t drain;
  uint64_t kv_full[10];
  uint64_t kv_empty[10];
  uint32_t tmem_base;
  int abort_flag;
};

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(DqCfg<D>::kThreads, 1)
fa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO, BwdParams p) {
  using Cfg = DqCfg<D>;
  constexpr int NS = Cfg::kSlots;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sQ = base;
  unsigned char* sDO = base + Cfg::kTileBytes;
  unsigned char* sKV = base + 2 * Cfg::kTileBytes;
  DqBarriers& bar = *reinterpret_cast<DqBarriers*>(sKV + NS * Cfg::kTileBytes);
  volatile int* abortf = &bar.abort_flag;

  const int warp = __shfl_sync(0xffffffffu, (int)threadIdx.x / 32, 0), lane = threadIdx.x % 32;
  const int q_tile = p.n_qtiles - 1 - blockIdx.x;   // longest causal rows first
  const int h = blockIdx.y, b = blockIdx.z, hkv = h / p.G;
  const int q0 = q_tile * BM;
  int n_kv = (p.Lk + BM - 1) / BM;
  if (CAUSAL) n_kv = min(n_kv, (min(q0 + BM, p.Lq) - 1 + p.causal_off) / BM + 1);

  if (threadIdx.x == 0) {
    bar.abort_flag = 0;
    mbar_init(&bar.qd_full, 1);
    mbar_init(&bar.s_full, 1);
    mbar_init(&bar.s_free, 4);
    mbar_init(&bar.dp_full, 1);
    mbar_init(&bar.ds_full, 4);
    mbar_init(&bar.o_full, 1);
    mbar_init(&bar.drain, 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(&bar.kv_full[i], 1);
      mbar_init(&bar.kv_empty[i], 1);
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
      mbar_arrive_expect_tx(&bar.qd_full, 2 * Cfg::kTileBytes);
      for (int db = 0; db < Cfg::kDBlocks; ++db) {
        tma_load_4d_hint(sQ + db * BM * 128, &tmQ, &bar.qd_full, db * 64, h, q0, b, pol_q);
        tma_load_4d_hint(sDO + db * BM * 128, &tmDO, &bar.qd_full, db * 64, h, q0, b, pol_q);
      }
    }
    __syncwarp();
    int issued = 0;
    bool ok = true;
    for (int i = 0; i < 2 * n_kv && ok; ++i) {   // K_0, V_0, K_1, V_1, ...
      const int slot = i % NS, round = i / NS;
      if (round > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bar.kv_empty[slot], (round - 1) & 1, abortf));
      if (!ok) break;
      const CUtensorMap* tm = (i & 1) ? &tmV : &tmK;
      if (elect_one()) {
        mbar_arrive_expect_tx(&bar.kv_full[slot], Cfg::kTileBytes);
        for (int db = 0; db < Cfg::kDBlocks; ++db)
          tma_load_4d_hint(sKV + slot * Cfg::kTileBytes + db * BM * 128, tm, &bar.kv_full[slot], db * 64, hkv,
                           (i >> 1) * BM, b, pol_kv);
      }
      __syncwarp();
      ++issued;
    }
    if (!ok) {
      wait_drain(&bar.qd_full, 0);
      for (int i = (issued > NS ? issued - NS : 0); i < issued; ++i) wait_drain(&bar.kv_full[i % NS], (i / NS) & 1);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA warp
    // S_j+1 goes in as soon as the softmax warps have read S_j (s_free), so
    // it runs while they form dS_j; dP_j+1 overwrites the columns dS_j was
    // read from and follows dQ_j.
    const uint32_t q_lo = smem_u32(sQ) >> 4, do_lo = smem_u32(sDO) >> 4, kv_lo = smem_u32(sKV) >> 4;
    auto slot_lo = [&](int fill) { return kv_lo + (uint32_t)((fill % NS) * Cfg::kTileBytes >> 4); };
    auto wait_fill = [&](int fill) { return mbar_wait(&bar.kv_full[fill % NS], (fill / NS) & 1, abortf); };
    bool ok = __all_sync(0xffffffffu, mbar_wait(&bar.qd_full, 0, abortf));
    if (ok && n_kv > 0) {
      ok = __all_sync(0xffffffffu, wait_fill(0) && wait_fill(1));
      if (ok) {
        tc_fence_after();
        if (elect_one()) {
          mma_kmajor<D>(tmem + Cfg::kS, q_lo, slot_lo(0));     // S_0 = Q K_0^T
          tc_commit(&bar.s_full);
          mma_kmajor<D>(tmem + Cfg::kDP, do_lo, slot_lo(1));   // dP_0 = dO V_0^T
          tc_commit(&bar.dp_full);
          tc_commit(&bar.kv_empty[1 % NS]);                    // V_0 read
        }
        __syncwarp();
      }
    }
    for (int j = 0; j < n_kv && ok; ++j) {
      const bool more = j + 1 < n_kv;
      if (more) {
        ok = __all_sync(0xffffffffu, wait_fill(2 * j + 2) && mbar_wait(&bar.s_free, j & 1, abortf));
        if (!ok) break;
        tc_fence_after();
        if (elect_one()) {
          mma_kmajor<D>(tmem + Cfg::kS, q_lo, slot_lo(2 * j + 2));   // S_j+1 = Q K_j+1^T
          tc_commit(&bar.s_full);
        }
        __syncwarp();
      }
      ok = __all_sync(0xffffffffu, mbar_wait(&bar.ds_full, j & 1, abortf) && (!more || wait_fill(2 * j + 3)));
      if (!ok) break;
      tc_fence_after();
      if (elect_one()) {
        mma_tmem_mn<D>(tmem + Cfg::kDQ, tmem + Cfg::kDP, slot_lo(2 * j), j == 0);   // dQ += dS_j K_j
        tc_commit(&bar.kv_empty[(2 * j) % NS]);                                     // K_j read
        if (!more) tc_commit(&bar.o_full);
        if (more) {
          mma_kmajor<D>(tmem + Cfg::kDP, do_lo, slot_lo(2 * j + 3));   // dP_j+1 = dO V_j+1^T
          tc_commit(&bar.dp_full);
          tc_commit(&bar.kv_empty[(2 * j + 3) % NS]);                  // V_j+1 read
        }
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
      // Pass 1: P = 2^(S scale log2e - L) as bf16 pairs, then S is released.
      ok = mbar_wait(&bar.s_full, j & 1, abortf);
      if (!ok) break;
      tc_fence_after();
      float pf[BM];
#pragma unroll
      for (int c = 0; c < BM; c += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_addr + Cfg::kS + c, r);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int key = j * BM + c + e;
          pf[c + e] = (row_ok && key <= key_limit) ? ex2_approx(fmaf(__uint_as_float(r[e]), sl2, -lse2)) : 0.f;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.s_free);
      // Pass 2: dS = P o (dP - Delta), over the dP columns already read.
      ok = mbar_wait(&bar.dp_full, j & 1, abortf);
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < BM; c += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_addr + Cfg::kDP + c, r);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(pf[c + 2 * e] * (__uint_as_float(r[2 * e]) - dlt),
                              pf[c + 2 * e + 1] * (__uint_as_float(r[2 * e + 1]) - dlt));
        tmem_st16(tmem + lane_addr + Cfg::kDP + c / 2, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.ds_full);
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
template <int D>
struct DkvCfg {
  static constexpr int kDBlocks = D / 64;
  static constexpr int kTileBytes = kDBlocks * BM * 128;
  static constexpr int kThreads = 192;
  static constexpr int kST = 0, kDPT = 128, kDV = 256, kDK = 256 + D;   // tensor-memory columns
  static constexpr int kStageBytes = 2 * kTileBytes;                    // Q_i and dO_i
  static constexpr int kStages = 2;
  static constexpr int kRowBytes = 2 * 2 * BM * 4;                     // L and Delta, double-buffered
  static constexpr int kSmemBytes = 2 * kTileBytes + kStages * kStageBytes + kRowBytes + 512 + 1024;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static_assert(kDK + D <= 512, "tensor-memory budget");
};

struct DkvBarriers {
  uint64_t kv_full;         // K and V
  uint64_t qd_full[2];      // Q_i and dO_i per stage
  uint64_t qd_empty[2];
  uint64_t st_full;         // S^T in tensor memory
  uint64_t st_free;         // S^T read by the softmax warps (4 warps)
  uint64_t dpt_full;        // dP^T in tensor memory
  uint64_t p_full;          // P^T and dS^T in tensor memory (4 warps)
  uint64_t o_full;          // the last dV / dK products have landed
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(DkvCfg<D>::kThreads, 1)
fa_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO, BwdParams p) {
  using Cfg = DkvCfg<D>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sK = base;
  unsigned char* sV = base + Cfg::kTileBytes;
  unsigned char* sQD = base + 2 * Cfg::kTileBytes;                          // [stage][Q, dO]
  float* sRow = reinterpret_cast<float*>(sQD + Cfg::kStages * Cfg::kStageBytes);   // [parity][L2, Delta][128]
  DkvBarriers& bar = *reinterpret_cast<DkvBarriers*>(reinterpret_cast<unsigned char*>(sRow) + Cfg::kRowBytes);
  volatile int* abortf = &bar.abort_flag;

  const int warp = __shfl_sync(0xffffffffu, (int)threadIdx.x / 32, 0), lane = threadIdx.x % 32;
  const int kv_tile = blockIdx.x, hkv = blockIdx.y, b = blockIdx.z;
  const int k0 = kv_tile * BM;
  const int n_qt = (p.Lq + BM - 1) / BM;
  // causal: query tiles whose last row reaches this tile's first key
  const int i_start = CAUSAL ? min(n_qt, max(0, k0 - p.causal_off) / BM) : 0;
  const int per_head = n_qt - i_start;
  const int T = p.G * per_head;   // steps: (head of the group, query tile)

  if (threadIdx.x == 0) {
    bar.abort_flag = 0;
    mbar_init(&bar.kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar.qd_full[s], 1);
      mbar_init(&bar.qd_empty[s], 1);
    }
    mbar_init(&bar.st_full, 1);
    mbar_init(&bar.st_free, 4);
    mbar_init(&bar.dpt_full, 1);
    mbar_init(&bar.p_full, 4);
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
      mbar_arrive_expect_tx(&bar.kv_full, 2 * Cfg::kTileBytes);
      for (int db = 0; db < Cfg::kDBlocks; ++db) {
        tma_load_4d_hint(sK + db * BM * 128, &tmK, &bar.kv_full, db * 64, hkv, k0, b, pol_kv);
        tma_load_4d_hint(sV + db * BM * 128, &tmV, &bar.kv_full, db * 64, hkv, k0, b, pol_kv);
      }
    }
    __syncwarp();
    int issued = 0;
    bool ok = true;
    for (int t = 0; t < T && ok; ++t) {
      const int st = t & 1;
      if (t >= 2) ok = __all_sync(0xffffffffu, mbar_wait(&bar.qd_empty[st], ((t >> 1) - 1) & 1, abortf));
      if (!ok) break;
      const int h = hkv * p.G + t / per_head, qt = i_start + t % per_head;
      unsigned char* dst = sQD + st * Cfg::kStageBytes;
      if (elect_one()) {
        mbar_arrive_expect_tx(&bar.qd_full[st], Cfg::kStageBytes);
        for (int db = 0; db < Cfg::kDBlocks; ++db) {
          tma_load_4d_hint(dst + db * BM * 128, &tmQ, &bar.qd_full[st], db * 64, h, qt * BM, b, pol_q);
          tma_load_4d_hint(dst + Cfg::kTileBytes + db * BM * 128, &tmDO, &bar.qd_full[st], db * 64, h, qt * BM, b,
                           pol_q);
        }
      }
      __syncwarp();
      ++issued;
    }
    if (!ok) {
      wait_drain(&bar.kv_full, 0);
      for (int t = (issued > 2 ? issued - 2 : 0); t < issued; ++t) wait_drain(&bar.qd_full[t & 1], (t >> 1) & 1);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA warp
    // S^T_t+1 goes in as soon as the softmax warps have read S^T_t (st_free)
    // and runs while they form dS^T_t; dP^T_t+1 overwrites the columns that
    // P^T_t and dS^T_t were read from, so it follows dV_t and dK_t.
    const uint32_t k_lo = smem_u32(sK) >> 4, v_lo = smem_u32(sV) >> 4, qd_lo = smem_u32(sQD) >> 4;
    auto q_of = [&](int t) { return qd_lo + (uint32_t)((t & 1) * Cfg::kStageBytes >> 4); };
    auto wait_qd = [&](int t) { return mbar_wait(&bar.qd_full[t & 1], (t >> 1) & 1, abortf); };
    constexpr uint32_t kDoOff = (uint32_t)(Cfg::kTileBytes >> 4);
    bool ok = __all_sync(0xffffffffu, mbar_wait(&bar.kv_full, 0, abortf));
    if (ok && T > 0) {
      ok = __all_sync(0xffffffffu, wait_qd(0));
      if (ok) {
        tc_fence_after();
        if (elect_one()) {
          mma_kmajor<D>(tmem + Cfg::kST, k_lo, q_of(0));             // S^T_0 = K Q_0^T
          tc_commit(&bar.st_full);
          mma_kmajor<D>(tmem + Cfg::kDPT, v_lo, q_of(0) + kDoOff);   // dP^T_0 = V dO_0^T
          tc_commit(&bar.dpt_full);
        }
        __syncwarp();
      }
    }
    for (int t = 0; t < T && ok; ++t) {
      const bool more = t + 1 < T;
      if (more) {
        ok = __all_sync(0xffffffffu, wait_qd(t + 1) && mbar_wait(&bar.st_free, t & 1, abortf));
        if (!ok) break;
        tc_fence_after();
        if (elect_one()) {
          mma_kmajor<D>(tmem + Cfg::kST, k_lo, q_of(t + 1));   // S^T_t+1
          tc_commit(&bar.st_full);
        }
        __syncwarp();
      }
      ok = __all_sync(0xffffffffu, mbar_wait(&bar.p_full, t & 1, abortf));
      if (!ok) break;
      tc_fence_after();
      if (elect_one()) {
        const uint32_t q_lo = q_of(t), do_lo = q_lo + kDoOff;
        mma_tmem_mn<D>(tmem + Cfg::kDV, tmem + Cfg::kDPT + 64, do_lo, t == 0);   // dV += P^T dO_t
        mma_tmem_mn<D>(tmem + Cfg::kDK, tmem + Cfg::kDPT, q_lo, t == 0);         // dK += dS^T Q_t
        tc_commit(&bar.qd_empty[t & 1]);
        if (!more) tc_commit(&bar.o_full);
        if (more) {
          mma_kmajor<D>(tmem + Cfg::kDPT, v_lo, q_of(t + 1) + kDoOff);   // dP^T_t+1
          tc_commit(&bar.dpt_full);
        }
      }
      __syncwarp();
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
    for (int t = 0; t < T; ++t) {
      const int h = hkv * p.G + t / per_head, qt = i_start + t % per_head;
      const int i0 = qt * BM;
      // the tile's L (base 2) and Delta, staged for all 128 threads
      float* rows = sRow + (t & 1) * 2 * BM;
      {
        const int qi = i0 + r;
        const int64_t lrow = ((int64_t)b * p.Hq + h) * p.Lq + qi;
        rows[r] = qi < p.Lq ? p.lse[lrow] * kLog2e : 0.f;
        rows[BM + r] = qi < p.Lq ? p.delta[lrow] : 0.f;
      }
      named_barrier_sync(1, 128);
      // Pass 1: P^T from S^T, kept in fp32 until dS^T is formed; S^T released.
      ok = ok && mbar_wait(&bar.st_full, t & 1, abortf);
      if (!ok) continue;
      tc_fence_after();
      // query q (column) may be attended by this key iff q < Lq and, causal, key <= q + off
      float pf[BM];
#pragma unroll
      for (int c = 0; c < BM; c += 32) {
        uint32_t sv[32];
        tmem_ld32(tmem + lane_addr + Cfg::kST + c, sv);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int q = i0 + c + e;
          const bool allowed = q < p.Lq && (!CAUSAL || key <= q + p.causal_off);
          pf[c + e] = allowed ? ex2_approx(fmaf(__uint_as_float(sv[e]), sl2, -rows[c + e])) : 0.f;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.st_free);
      // Pass 2: dS^T = P^T o (dP^T - Delta) into dP^T columns 0..63 (behind
      // the reads), then P^T into columns 64..127 once every column is read.
      ok = mbar_wait(&bar.dpt_full, t & 1, abortf);
      if (!ok) continue;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < BM; c += 32) {
        uint32_t dv[32];
        tmem_ld32(tmem + lane_addr + Cfg::kDPT + c, dv);
        tmem_wait_ld();
        uint32_t pd[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pd[e] = pack_bf16x2(pf[c + 2 * e] * (__uint_as_float(dv[2 * e]) - rows[BM + c + 2 * e]),
                              pf[c + 2 * e + 1] * (__uint_as_float(dv[2 * e + 1]) - rows[BM + c + 2 * e + 1]));
        tmem_st16(tmem + lane_addr + Cfg::kDPT + c / 2, pd);
      }
#pragma unroll
      for (int c = 0; c < BM; c += 32) {
        uint32_t pp[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) pp[e] = pack_bf16x2(pf[c + 2 * e], pf[c + 2 * e + 1]);
        tmem_st16(tmem + lane_addr + Cfg::kDPT + 64 + c / 2, pp);
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
        store_row_bf16<D>(tmem + lane_addr + Cfg::kDV, 1.f, dvrow, row_ok);
        store_row_bf16<D>(tmem + lane_addr + Cfg::kDK, p.scale, dkrow, row_ok);
      } else if (row_ok) {
        for (int c = 0; c < D; c += 8) {
          *reinterpret_cast<uint4*>(dvrow + c) = make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4*>(dkrow + c) = make_uint4(0, 0, 0, 0);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int D, bool CAUSAL>
cudaError_t launch_bwd_t(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, const CUtensorMap& dout,
                         BwdParams p, cudaStream_t s) {
  const int64_t rows = (int64_t)p.B * p.Lq * p.Hq;
  fa_bwd_delta_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(static_cast<const __nv_bfloat16*>(p.o),
                                                                    static_cast<const __nv_bfloat16*>(p.dout),
                                                                    p.delta, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  {
    using Cfg = DqCfg<D>;
    auto kern = fa_bwd_dq_kernel<D, CAUSAL>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
    if (e != cudaSuccess) return e;
    p.n_qtiles = (p.Lq + BM - 1) / BM;
    kern<<<dim3(p.n_qtiles, p.Hq, p.B), Cfg::kThreads, Cfg::kSmemBytes, s>>>(q, k, v, dout, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  {
    using Cfg = DkvCfg<D>;
    auto kern = fa_bwd_dkdv_kernel<D, CAUSAL>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
    if (e != cudaSuccess) return e;
    kern<<<dim3((p.Lk + BM - 1) / BM, p.Hkv, p.B), Cfg::kThreads, Cfg::kSmemBytes, s>>>(q, k, v, dout, p);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace

cudaError_t launch_fa_bwd(int D, bool causal, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                          const CUtensorMap& dout, const BwdParams& p, cudaStream_t stream) {
  switch (D) {
    case 64: return causal ? launch_bwd_t<64, true>(q, k, v, dout, p, stream) : launch_bwd_t<64, false>(q, k, v, dout, p, stream);
    case 128:
      return causal ? launch_bwd_t<128, true>(q, k, v, dout, p, stream) : launch_bwd_t<128, false>(q, k, v, dout, p, stream);
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
