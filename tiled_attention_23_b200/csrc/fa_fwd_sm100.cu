// Attention forward (prefill) for sm_100a: TMA-staged Q/K/V tiles, QK^T and
// PV on the 5th-generation tensor cores (tcgen05) with fp32 accumulators in
// tensor memory, and an online softmax in registers.
//
// The method ("FlashAttention in Ascend CANN ops-transformer", section 二):
//   1. Q, K and V are cut into blocks that live in on-chip memory;
//   2. after each K/V block the running row max and running row sum are
//      updated, so the result equals standard attention exactly;
//   3. O and the log-sum-exp L accumulate block by block and are written once.
// "FlashAttention-2 (TH)" adds: minimise non-matmul work, parallelise over
// query blocks, split work across warps.  Here that becomes a warp-specialised
// CTA on one SM:
//
//   warp 0      TMA producer: Q tile once, then K_j / V_j into a ring of slots
//   warp 1      TMEM allocator and MMA issuer (one thread):
//                 S_j = Q K_j^T            (A, B from shared memory)
//                 O  += P_j V_j            (A = P from tensor memory)
//   warps 2..5  softmax: thread = query row (tensor-memory lane); row max,
//               exp2, row sum, P_j -> tensor memory as bf16, occasional
//               rescale of O, and the epilogue (O / l, L = ln of the row sum).
//
// One CTA owns a 128-row query tile of one (batch, query head).  S is double
// buffered in tensor memory so that S_{j+1} is computed while the softmax
// warps work on S_j, and PV_{j-1} runs alongside as well.
//
// Online-softmax bookkeeping (base 2): t = s * scale * log2(e).  Each row keeps
// a reference max m and the sum l of 2^(t - m).  A new tile only moves m when
// its max exceeds m by more than 8 (a factor of 256); then O and l are
// rescaled by 2^(m_old - m_new).  Otherwise the exponentials are taken
// against the stale m, which is exact algebra and keeps P <= 256 in bf16.
//
// Causal masking is computed from indices (bottom-right aligned: key j is
// allowed for query i iff j <= i + Lk - Lq); K/V tiles wholly above the
// diagonal are never loaded, and only tiles that straddle it or the end of the
// keys are masked element by element.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
#include "fa_kernels.h"

namespace ta23 {
namespace {

constexpr int BM = 128;          // query rows per CTA (one tensor-memory lane each)
constexpr int kThreads = 192;    // 6 warps
constexpr float kRescaleThreshold = 8.0f;

template <int D, int BN>
struct FwdCfg {
  static constexpr int kDBlocks = D / 64;                   // 128-byte swizzle blocks along D
  static constexpr int kQBlockBytes = BM * 128;             // one 64-wide block of the Q tile
  static constexpr int kKVBlockBytes = BN * 128;            // one 64-wide block of a K or V tile
  static constexpr int kSlotBytes = kDBlocks * kKVBlockBytes;
  static constexpr int kQBytes = kDBlocks * kQBlockBytes;
  static constexpr int kSlots = (D == 64) ? 8 : (D == 128 ? 4 : 4);
  // tensor-memory columns
  static constexpr int kSCol0 = 0;
  static constexpr int kOCol = 256;
  static constexpr int kPCol0 = (D <= 128) ? 384 : 2 * BN;
  static constexpr int kSmemBytes = kQBytes + kSlots * kSlotBytes + 1024 /*barriers*/ + 1024 /*align*/;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static_assert(2 * BN <= 256 && kPCol0 + BN <= 512 && kOCol + D <= 512, "tensor-memory budget");
  static_assert(kPCol0 >= 2 * BN && (D > 128 || kPCol0 >= kOCol + D), "tensor-memory overlap");
};

struct Barriers {
  uint64_t q_full;
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t pv_done[2];   // PV_t completes phase t/2 of pv_done[t % 2]
  uint64_t drain;
  uint64_t kv_full[8];
  uint64_t kv_empty[8];
  uint32_t tmem_base;
  int abort_flag;
};

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

template <int D, int BN, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, FwdParams p) {
  using Cfg = FwdCfg<D, BN>;
  constexpr int NS = Cfg::kSlots;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sQ = base;
  unsigned char* sKV = base + Cfg::kQBytes;
  Barriers& bar = *reinterpret_cast<Barriers*>(sKV + NS * Cfg::kSlotBytes);
  volatile int* abortf = &bar.abort_flag;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int q_tile = p.n_qtiles - 1 - blockIdx.x;   // longest causal rows first
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int hkv = h / p.G;
  const int q0 = q_tile * BM;

  // Number of K/V tiles this query tile needs.
  int n_kv = (p.Lk + BN - 1) / BN;
  if (CAUSAL) {
    const int last_row = min(q0 + BM, p.Lq) - 1;
    const int last_key = min(last_row + p.causal_off, p.Lk - 1);
    n_kv = min(n_kv, last_key / BN + 1);
  }

  if (threadIdx.x == 0) {
    bar.abort_flag = 0;
    mbar_init(&bar.q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar.s_full[i], 1);
      mbar_init(&bar.p_full[i], 4);   // one arrival per softmax warp
    }
    mbar_init(&bar.pv_done[0], 1);
    mbar_init(&bar.pv_done[1], 1);
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
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const uint64_t pol_kv = l2_policy_evict_last();
      const uint64_t pol_q = l2_policy_evict_first();
      mbar_arrive_expect_tx(&bar.q_full, Cfg::kQBytes);
      for (int db = 0; db < Cfg::kDBlocks; ++db)
        tma_load_4d_hint(sQ + db * Cfg::kQBlockBytes, &tmQ, &bar.q_full, db * 64, h, q0, b, pol_q);
      int issued = 0;
      bool ok = true;
      for (int i = 0; i < 2 * n_kv && ok; ++i) {
        const int slot = i % NS, round = i / NS;
        if (round > 0) ok = mbar_wait(&bar.kv_empty[slot], (round - 1) & 1, abortf);
        if (!ok) break;
        const int key0 = (i >> 1) * BN;
        const CUtensorMap* tm = (i & 1) ? &tmV : &tmK;
        unsigned char* dst = sKV + slot * Cfg::kSlotBytes;
        mbar_arrive_expect_tx(&bar.kv_full[slot], Cfg::kSlotBytes);
        for (int db = 0; db < Cfg::kDBlocks; ++db)
          tma_load_4d_hint(dst + db * Cfg::kKVBlockBytes, tm, &bar.kv_full[slot], db * 64, hkv, key0, b,
                           pol_kv);
        ++issued;
      }
      if (!ok) {
        // Let every copy already in flight land before the CTA exits.
        wait_drain(&bar.q_full, 0);
        for (int i = (issued > NS ? issued - NS : 0); i < issued; ++i)
          wait_drain(&bar.kv_full[i % NS], (i / NS) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(BM, BN, 0, 0);
      constexpr uint32_t idPV = idesc_bf16_f32(BM, D, 0, 1);
      const uint64_t descQ0 = smem_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t descKV0 = smem_desc_sw128(smem_u32(sKV), 16, 1024);
      const uint64_t descV0 = smem_desc_sw128(smem_u32(sKV), Cfg::kKVBlockBytes, 1024);
      bool ok = mbar_wait(&bar.q_full, 0, abortf);

      auto issue_pv = [&](int t) -> bool {
        if (!mbar_wait(&bar.p_full[t & 1], (t >> 1) & 1, abortf)) return false;
        const int i = 2 * t + 1, slot = i % NS;
        if (!mbar_wait(&bar.kv_full[slot], (i / NS) & 1, abortf)) return false;
        tc_fence_after();
        const uint64_t dv = descV0 + ((uint64_t)(slot * Cfg::kSlotBytes) >> 4);
        const uint32_t pcol = tmem + Cfg::kPCol0 + (t & 1) * (BN / 2);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          mma_bf16_ts(tmem + Cfg::kOCol, pcol + kk * 8, dv + ((uint64_t)(kk * 16 * 128) >> 4), idPV,
                      (t > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&bar.kv_empty[slot]);
        tc_commit(&bar.pv_done[t & 1]);
        return true;
      };

      for (int j = 0; j < n_kv && ok; ++j) {
        const int i = 2 * j, slot = i % NS;
        ok = mbar_wait(&bar.kv_full[slot], (i / NS) & 1, abortf);
        if (!ok) break;
        tc_fence_after();
        const uint64_t dk = descKV0 + ((uint64_t)(slot * Cfg::kSlotBytes) >> 4);
        const uint32_t scol = tmem + Cfg::kSCol0 + (j & 1) * BN;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk & 3) * 32;   // 16 bf16 = 32 bytes along the swizzled row
          const uint64_t dq = descQ0 + ((uint64_t)((kk >> 2) * Cfg::kQBlockBytes + off) >> 4);
          const uint64_t dkk = dk + ((uint64_t)((kk >> 2) * Cfg::kKVBlockBytes + off) >> 4);
          mma_bf16_ss(scol, dq, dkk, idS, kk > 0 ? 1u : 0u);
        }
        tc_commit(&bar.s_full[j & 1]);
        tc_commit(&bar.kv_empty[slot]);
        if (j >= 1) ok = issue_pv(j - 1);
      }
      if (ok && n_kv > 0) ok = issue_pv(n_kv - 1);
      if (!ok) {
        tc_commit(&bar.drain);   // wait for every MMA already issued
        wait_drain(&bar.drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int quarter = warp & 3;                    // tensor-memory lane quarter of this warp
    const int r = quarter * 32 + lane;               // row within the tile
    const int qi = q0 + r;                           // query index
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    const float sl2 = p.scale_log2;
    int key_limit = p.Lk - 1;                        // last allowed key for this row
    if (CAUSAL) key_limit = min(key_limit, qi + p.causal_off);

    float m_ref = -INFINITY;   // reference max (base-2 scaled units)
    float l = 0.f;             // running sum of 2^(t - m_ref)
    // PV completions are observed strictly in order.  Two barriers keep the
    // parity waits unambiguous: while PV_t is awaited, PV_{t+1} may already be
    // done, but PV_{t+2} cannot (it needs P_{t+2}, which this thread has not
    // produced yet).
    int pv_seen = 0;           // PV completions observed so far
    bool ok = true;
    auto wait_pv = [&](int t) -> bool {
      while (pv_seen <= t) {
        if (!mbar_wait(&bar.pv_done[pv_seen & 1], (pv_seen >> 1) & 1, abortf)) return false;
        ++pv_seen;
      }
      return true;
    };

    for (int j = 0; j < n_kv && ok; ++j) {
      ok = mbar_wait(&bar.s_full[j & 1], (j >> 1) & 1, abortf);
      if (!ok) break;
      tc_fence_after();
      float s[BN];
      {
        const uint32_t scol = tmem + lane_addr + Cfg::kSCol0 + (j & 1) * BN;
#pragma unroll
        for (int c = 0; c < BN; c += 32) {
          uint32_t rr[32];
          tmem_ld32(scol + c, rr);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) s[c + e] = __uint_as_float(rr[e]);
        }
      }
      const int key0 = j * BN;
      const bool need_mask = (key0 + BN > p.Lk) || (CAUSAL && key0 + BN - 1 > q0 + p.causal_off);
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (key0 + c > key_limit) s[c] = -INFINITY;
      }
      float mx = s[0];
#pragma unroll
      for (int c = 1; c < BN; ++c) mx = fmaxf(mx, s[c]);
      const float t_max = (mx == -INFINITY) ? -INFINITY : mx * sl2;

      float m_new = m_ref, alpha = 1.f;
      bool rescale = false;
      if (m_ref == -INFINITY) {
        m_new = t_max;                       // nothing accumulated yet: O holds zeros/garbage only
      } else if (t_max > m_ref + kRescaleThreshold) {
        m_new = t_max;
        alpha = ex2_approx(m_ref - m_new);
        rescale = true;
      }
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;

      // P_j must not overwrite P_{j-2} before PV_{j-2} has read it.
      if (j >= 2) ok = wait_pv(j - 2);
      if (!ok) break;
      float rowsum = 0.f;
      {
        const uint32_t pcol = tmem + lane_addr + Cfg::kPCol0 + (j & 1) * (BN / 2);
#pragma unroll
        for (int c = 0; c < BN; c += 64) {
          uint32_t pk[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            float p0 = ex2_approx(fmaf(s[c + 2 * e], sl2, -m_use));
            float p1 = ex2_approx(fmaf(s[c + 2 * e + 1], sl2, -m_use));
            if (need_mask) {
              if (key0 + c + 2 * e > key_limit) p0 = 0.f;
              if (key0 + c + 2 * e + 1 > key_limit) p1 = 0.f;
            }
            rowsum += p0 + p1;
            pk[e] = pack_bf16x2(p0, p1);
          }
          tmem_st32(pcol + c / 2, pk);
        }
      }
      // Rescale O (rows whose max moved) once PV_{j-1} has landed in it.
      if (__any_sync(0xffffffffu, rescale) && j >= 1) {
        ok = wait_pv(j - 1);
        if (!ok) break;
        tc_fence_after();
        const uint32_t ocol = tmem + lane_addr + Cfg::kOCol;
        const float a = rescale ? alpha : 1.f;
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
          uint32_t rr[32];
          tmem_ld32(ocol + c, rr);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) rr[e] = __float_as_uint(__uint_as_float(rr[e]) * a);
          tmem_st32(ocol + c, rr);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.p_full[j & 1]);
      l = (rescale ? l * alpha : l) + rowsum;
      m_ref = m_new;
    }

    // ------------------------------------------------------------ epilogue
    if (ok) ok = wait_pv(n_kv - 1);
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      const bool row_ok = qi < p.Lq;
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) +
                            (((int64_t)b * p.Lq + qi) * p.Hq + h) * D;
      const uint32_t ocol = tmem + lane_addr + Cfg::kOCol;
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        uint32_t rr[32];
        tmem_ld32(ocol + c, rr);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(__uint_as_float(rr[2 * e]) * inv_l, __uint_as_float(rr[2 * e + 1]) * inv_l);
        if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
      }
      if (row_ok && p.lse) {
        const float m_fin = (m_ref == -INFINITY) ? 0.f : m_ref;
        p.lse[((int64_t)b * p.Hq + h) * p.Lq + qi] = (m_fin + log2f(l)) * 0.69314718055994530942f;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int D, int BN, bool CAUSAL>
cudaError_t launch_fwd(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                       const FwdParams& p, cudaStream_t stream) {
  using Cfg = FwdCfg<D, BN>;
  auto kern = fa_fwd_kernel<D, BN, CAUSAL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(p.n_qtiles, p.Hq, p.B);
  kern<<<grid, kThreads, Cfg::kSmemBytes, stream>>>(q, k, v, p);
  return cudaGetLastError();
}

}  // namespace

int fwd_block_n(int D) { return D == 256 ? 64 : 128; }

cudaError_t launch_fa_fwd(int D, bool causal, const CUtensorMap& q, const CUtensorMap& k,
                          const CUtensorMap& v, const FwdParams& p, cudaStream_t stream) {
  switch (D) {
    case 64:
      return causal ? launch_fwd<64, 128, true>(q, k, v, p, stream) : launch_fwd<64, 128, false>(q, k, v, p, stream);
    case 128:
      return causal ? launch_fwd<128, 128, true>(q, k, v, p, stream)
                    : launch_fwd<128, 128, false>(q, k, v, p, stream);
    case 256:
      return causal ? launch_fwd<256, 64, true>(q, k, v, p, stream) : launch_fwd<256, 64, false>(q, k, v, p, stream);
    default:
      return cudaErrorInvalidValue;
  }
}

unsigned int fwd_read_and_clear_status() {
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof v) != cudaSuccess) return 0xFFFFFFFFu;
  cudaMemcpyToSymbol(g_device_status, &zero, sizeof zero);
  return v;
}

}  // namespace ta23
