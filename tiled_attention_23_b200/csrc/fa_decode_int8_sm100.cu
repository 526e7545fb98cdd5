// Split-KV decode against an int8 KV cache for sm_100a, and the quantiser
// that writes such a cache.
//
// The MNN attention_mode page offers KV-cache int8 quantisation next to
// FlashAttention, in two forms: key int8 with value unquantised, and key and
// value int8, and calls the int8 cache almost lossless.  It fixes no
// granularity; here every (sequence, token, kv head) vector of D values has
// one fp32 scale: scale = max|x| / 127, code = round-half-even(x / scale) in
// [-127, 127], both decided in fp32.  Scales are stored [B, Hkv, Lmax], so the
// scales of one head's consecutive tokens are contiguous and arrive with the
// tile through the same TMA transaction.
//
// The decode keeps the bf16 split kernel's design (one CTA per (split, kv
// head, sequence) serving all G query heads; four warps each streaming their
// own tiles through a per-warp TMA ring; two small products per tile on
// mma.sync) with half the K/V bytes.  The products run in fp16:
//  * an int8 code converts exactly to fp16 with integer and half2 operations
//    only: the byte x + 128 becomes the low byte of the fp16 pattern 0x64xx,
//    whose value is 1024 + (x + 128), and subtracting 1152 leaves x;
//  * S = Q K^T uses q converted to fp16 against the K codes, then multiplies
//    each fp32 score by its key's scale.  The conversion is exact for bf16
//    values with 2^-17 <= |q| <= 65280 (and 0); below 2^-17 the fp16
//    subnormals drop low bits (under 2^-25 to zero), which a dot product does
//    not notice, and bf16 values from 65536 up overflow fp16;
//  * with int8 V, each p is multiplied by its key's V scale (p stays <= 256 by
//    the stale-max rule) and rounded to fp16, and P V runs on the V codes;
//    with bf16 V, P V is the bf16 product of the bf16 kernel.
// V codes enter the product biased by +1152 (the 0x64xx pattern without the
// subtraction); 1152 times the row's sum of the fp16 P values is removed once
// at the end (the bias is 24x the codes' range, far inside fp32 precision).
// Fragment layouts.  ldmatrix moves 16-bit elements, so on int8 rows each
// element is a pair of adjacent bytes.  For S, a plain ldmatrix gives lane
// (g, t) the four codes d = 4t..4t+3 of key g in a 16-code chunk; the q
// fragment uses the same d order, which leaves the dot product unchanged.
// For P V, a transposing ldmatrix gives lane (g, t) codes (d 2g, 2g+1) of keys
// 2t and 2t+1; splitting the even and odd d into two n-tiles makes every
// fragment regular, and the accumulator of n-tile (chunk c, parity q) holds
// output columns d = 16c + 4t + 2e + q.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "ptx.cuh"
#include "ta23.h"
#include "fa_kernels.h"

namespace ta23 {
namespace {

constexpr int kWarps = 4;
// Per-warp ring depth.  Two buffers (one tile in flight while the other is
// computed) keep the ring at 74 KB, so three CTAs (12 warps) share an SM at
// head_dim <= 128; three buffers (two CTAs per SM) measured 15 % slower.
#ifndef TA23_I8_BUFS
#define TA23_I8_BUFS 2
#endif
constexpr int kBufs = TA23_I8_BUFS;
constexpr float kRescaleThreshold = 8.0f;

constexpr int round_up(int x, int m) { return (x + m - 1) / m * m; }

template <int D, bool V_INT8>
struct Dec8Cfg {
  static constexpr int TK = 4096 / D;                   // keys per tile (4 KB of K codes)
  static constexpr int RB = D < 128 ? D : 128;          // bytes per row of one int8 box
  static constexpr int kNBlk = D / RB;                  // int8 boxes per row
  static constexpr int kKBytes = TK * D;
  static constexpr int kVBytes = V_INT8 ? TK * D : TK * D * 2;
  static constexpr int kScBytes = TK * 4;
  // a tensor copy lands on a 128-byte aligned shared-memory address
  static constexpr int kScStride = round_up(kScBytes, 128);
  static constexpr int kTxBytes = kKBytes + kVBytes + (V_INT8 ? 2 : 1) * kScBytes;
  static constexpr int kSlotBytes = round_up(kKBytes + kVBytes + 2 * kScStride, 1024);
  static constexpr int kRingBytes = kWarps * kBufs * kSlotBytes;
  static constexpr int kMergeBytes = kWarps * 8 * (D + 2) * 4;
  static constexpr int kSmemBytes = kRingBytes + 256 + 1024;
  static constexpr int NT = TK / 8;                     // n-tiles of 8 keys
  static constexpr int KC = D / 16;                     // 16-byte chunks of a K code row
  static_assert(kMergeBytes <= kRingBytes, "merge area must fit in the ring");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static_assert(TK % 16 == 0 && KC % 4 == 0, "tile shape");
  static_assert(kKBytes % 1024 == 0 && kVBytes % 1024 == 0, "swizzled boxes start on 1024-byte boundaries");
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// D = A(16x16, rows >= 8 zero) * B(16x8) + C, fp32 accumulate; fp16 or bf16 operands.
__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

// Two int8 codes picked out of u = w ^ 0x80808080 (each byte x + 128) by the
// byte selector `sel` (0x4x4x pattern: code byte low, 0x64 high in each half)
// -> fp16x2 of x + 1152 (the pattern 0x64xx is 1024 + byte), exactly.
__device__ __forceinline__ uint32_t i8pair_biased(uint32_t u, uint32_t sel) {
  return __byte_perm(u, 0x64646464u, sel);
}
// The same, minus 1152: fp16x2 of the codes themselves, exactly.
__device__ __forceinline__ uint32_t i8pair_exact(uint32_t u, uint32_t sel) {
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(i8pair_biased(u, sel)), "r"(0x64806480u));
  return r;
}
constexpr float kCodeBias = 1152.f;

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Byte offset of 16-byte chunk `cc` of row `row` in a swizzled box of rows of
// RB bytes (128-byte swizzle for 128-byte rows, 64-byte swizzle for 64).
template <int RB>
__device__ __forceinline__ uint32_t swz(int row, int cc) {
  if (RB == 128) return (uint32_t)(row * 128 + ((cc ^ (row & 7)) << 4));
  return (uint32_t)(row * 64 + ((cc ^ ((row >> 1) & 3)) << 4));
}

template <int D, bool V_INT8>
__global__ void __launch_bounds__(kWarps * 32)
fa_decode_split_i8_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                          const __grid_constant__ CUtensorMap tmKS, const __grid_constant__ CUtensorMap tmVS,
                          DecodeParams p) {
  using Cfg = Dec8Cfg<D, V_INT8>;
  constexpr int TK = Cfg::TK, NT = Cfg::NT, KC = Cfg::KC, DN = D / 8, RB = Cfg::RB;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* merge = reinterpret_cast<float*>(base);   // reused once every warp is done with its ring
  uint64_t* full = reinterpret_cast<uint64_t*>(base + Cfg::kRingBytes);   // [kWarps][kBufs]

  const int split = blockIdx.x, hkv = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int g = lane >> 2, t = lane & 3;
  const int G = p.G;

  int n = p.seqlens[b];
  n = n < 1 ? 1 : (n > p.Lmax ? p.Lmax : n);
  const int per = (n + p.S - 1) / p.S;
  const int C = ((per + 63) / 64) * 64;
  const int j0 = split * C;
  const int j1 = min(j0 + C, n);
  const int64_t ws_row0 = ((int64_t)b * p.Hq + (int64_t)hkv * G) * p.S + split;

  if (j0 >= j1) {   // empty chunk: zero weight in the merge
    for (int i = threadIdx.x; i < G * D; i += blockDim.x)
      p.ws_o[(ws_row0 + (int64_t)(i / D) * p.S) * D + (i % D)] = 0.f;
    if (threadIdx.x < G) p.ws_lse[ws_row0 + (int64_t)threadIdx.x * p.S] = -INFINITY;
    return;
  }
  const int ntiles = (j1 - j0 + TK - 1) / TK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kWarps * kBufs; ++i) mbar_init(&full[i], 1);
    fence_barrier_init();
  }
  __syncthreads();

  unsigned char* my_ring = base + warp * kBufs * Cfg::kSlotBytes;
  uint64_t* my_full = full + warp * kBufs;
  const uint64_t pol = l2_policy_evict_first();
  auto issue = [&](int u) {   // local tile u of this warp -> buffer u % kBufs
    const int tile = warp + u * kWarps;
    if (tile >= ntiles) return;
    unsigned char* buf = my_ring + (u % kBufs) * Cfg::kSlotBytes;
    uint64_t* bar = &my_full[u % kBufs];
    const int key0 = j0 + tile * TK;
    mbar_arrive_expect_tx(bar, Cfg::kTxBytes);
#pragma unroll
    for (int blk = 0; blk < Cfg::kNBlk; ++blk)
      tma_load_4d_hint(buf + blk * TK * RB, &tmK, bar, blk * RB, hkv, key0, b, pol);
    if (V_INT8) {
#pragma unroll
      for (int blk = 0; blk < Cfg::kNBlk; ++blk)
        tma_load_4d_hint(buf + Cfg::kKBytes + blk * TK * RB, &tmV, bar, blk * RB, hkv, key0, b, pol);
    } else {
#pragma unroll
      for (int db = 0; db < D / 64; ++db)
        tma_load_4d_hint(buf + Cfg::kKBytes + db * TK * 128, &tmV, bar, db * 64, hkv, key0, b, pol);
    }
    unsigned char* sc = buf + Cfg::kKBytes + Cfg::kVBytes;
    tma_load_3d_hint(sc, &tmKS, bar, key0, hkv, b, pol);
    if (V_INT8) tma_load_3d_hint(sc + Cfg::kScStride, &tmVS, bar, key0, hkv, b, pol);
  };
  if (lane == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmKS);
    if (V_INT8) tma_prefetch_desc(&tmVS);
    for (int u = 0; u < kBufs - 1; ++u) issue(u);
  }

  // q as fp16 in the d order of the K fragments: chunk c gives a0 = (d 16c+4t,
  // +1) and a2 = (d 16c+4t+2, +3); rows g >= G are zero.  Loaded after the
  // first copies are issued, so the latencies overlap.
  uint32_t qa0[KC], qa2[KC];
  {
    const __nv_bfloat16* qrow = reinterpret_cast<const __nv_bfloat16*>(p.q) + ((int64_t)b * p.Hq + hkv * G + g) * D;
#pragma unroll
    for (int c = 0; c < KC; ++c) {
      if (g < G) {
        const uint2 w = *reinterpret_cast<const uint2*>(qrow + 16 * c + 4 * t);
        const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&w.x);
        const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&w.y);
        qa0[c] = pack_f16x2(__low2float(lo), __high2float(lo));
        qa2[c] = pack_f16x2(__low2float(hi), __high2float(hi));
      } else {
        qa0[c] = qa2[c] = 0u;
      }
    }
  }

  float o[DN][4];
#pragma unroll
  for (int i = 0; i < DN; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_ref = -INFINITY, l = 0.f;
  float p_sum = 0.f;   // int8 V: this thread's sum of the fp16 P values fed to PV (for the code bias)
  const float sl2 = p.scale_log2;
  int issued_last = kBufs - 2;
  bool ok = true;

  for (int u = 0;; ++u) {
    const int tile = warp + u * kWarps;
    if (tile >= ntiles) break;
    if (lane == 0) { issue(u + kBufs - 1); issued_last = u + kBufs - 1; }
    ok = mbar_wait(&my_full[u % kBufs], (u / kBufs) & 1, nullptr);
    if (!ok) break;
    unsigned char* buf = my_ring + (u % kBufs) * Cfg::kSlotBytes;
    const uint32_t sK = smem_u32(buf);
    const uint32_t sV = sK + Cfg::kKBytes;
    const float* ksc = reinterpret_cast<const float*>(buf + Cfg::kKBytes + Cfg::kVBytes);
    const float* vsc = ksc + Cfg::kScStride / 4;
    const int key0 = j0 + tile * TK;
    const bool tail = key0 + TK > j1;
    if (!V_INT8 && tail) {
      // bf16 V rows past the sequence end may hold inf or NaN: zero them
      const int first = j1 - key0;
      uint4* vbuf = reinterpret_cast<uint4*>(buf + Cfg::kKBytes);
      for (int i = lane; i < (D / 64) * (TK - first) * 8; i += 32) {
        const int db = i / ((TK - first) * 8), rem = i % ((TK - first) * 8);
        vbuf[(db * TK * 128 + (first + rem / 8) * 128) / 16 + (rem % 8)] = make_uint4(0, 0, 0, 0);
      }
      __syncwarp();
    }

    // S = Q K^T on the K codes (fp16), then each key's scale.
    float s[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
      const int krow = nt * 8 + (lane & 7);
#pragma unroll
      for (int c4 = 0; c4 < KC; c4 += 4) {
        const int chunk = c4 + (lane >> 3);
        const uint32_t addr = sK + (chunk / (RB / 16)) * (TK * RB) + swz<RB>(krow, chunk % (RB / 16));
        uint32_t r[4];
        ldsm_x4(addr, r[0], r[1], r[2], r[3]);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const uint32_t u = r[m] ^ 0x80808080u;
          mma_f16(s[nt], qa0[c4 + m], qa2[c4 + m], i8pair_exact(u, 0x4140), i8pair_exact(u, 0x4342));
        }
      }
    }
    float mx = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int kl = nt * 8 + 2 * t + e;
        s[nt][e] = (tail && key0 + kl >= j1) ? -INFINITY : s[nt][e] * ksc[kl];
        mx = fmaxf(mx, s[nt][e]);
      }
    }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float t_max = mx * sl2;   // finite: every tile holds at least one valid key
    float m_new = m_ref;
    if (m_ref == -INFINITY) {
      m_new = t_max;
    } else if (t_max > m_ref + kRescaleThreshold) {
      m_new = t_max;
      const float alpha = ex2_approx(m_ref - m_new);
      l *= alpha;
      p_sum *= alpha;
#pragma unroll
      for (int i = 0; i < DN; ++i) { o[i][0] *= alpha; o[i][1] *= alpha; }
    }
    m_ref = m_new;

    // P = 2^(t - m) (times the V scale for int8 V), packed as the PV A operand.
    uint32_t pa[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float pp[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int kl = nt * 8 + 2 * t + e;
        const bool masked = tail && key0 + kl >= j1;
        const float pv = masked ? 0.f : ex2_approx(fmaf(s[nt][e], sl2, -m_new));
        l += pv;
        pp[e] = V_INT8 ? (masked ? 0.f : pv * vsc[kl]) : pv;
      }
      if (V_INT8) {
        const __half2 h = __floats2half2_rn(pp[0], pp[1]);
        p_sum += __low2float(h) + __high2float(h);   // exactly the values the product sees
        pa[nt] = *reinterpret_cast<const uint32_t*>(&h);
      } else {
        pa[nt] = pack_bf16x2(pp[0], pp[1]);
      }
    }

    // O += P V: k-steps of 16 keys.
#pragma unroll
    for (int kt = 0; kt < NT / 2; ++kt) {
      const int vrow = kt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
      if (V_INT8) {
        // two 16-code chunks per transposing load -> four n-tiles (chunk, parity)
#pragma unroll
        for (int cp = 0; cp < KC; cp += 2) {
          const int chunk = cp + (lane >> 4);
          const uint32_t addr = sV + (chunk / (RB / 16)) * (TK * RB) + swz<RB>(vrow, chunk % (RB / 16));
          uint32_t r0, r1, r2, r3;
          ldsm_x4_t(addr, r0, r1, r2, r3);
          // V codes enter biased by +1152 (no subtraction); the bias times the
          // row's sum of P is taken off once at the end.
          r0 ^= 0x80808080u;
          r1 ^= 0x80808080u;
          r2 ^= 0x80808080u;
          r3 ^= 0x80808080u;
          mma_f16(o[2 * cp + 0], pa[2 * kt], pa[2 * kt + 1], i8pair_biased(r0, 0x4240), i8pair_biased(r1, 0x4240));
          mma_f16(o[2 * cp + 1], pa[2 * kt], pa[2 * kt + 1], i8pair_biased(r0, 0x4341), i8pair_biased(r1, 0x4341));
          mma_f16(o[2 * cp + 2], pa[2 * kt], pa[2 * kt + 1], i8pair_biased(r2, 0x4240), i8pair_biased(r3, 0x4240));
          mma_f16(o[2 * cp + 3], pa[2 * kt], pa[2 * kt + 1], i8pair_biased(r2, 0x4341), i8pair_biased(r3, 0x4341));
        }
      } else {
        // bf16 V (128-byte swizzled boxes of 64 columns): n-tiles of 8 columns
#pragma unroll
        for (int dp = 0; dp < DN / 2; ++dp) {
          const int chunk = 2 * dp + (lane >> 4);
          const uint32_t addr = sV + (chunk >> 3) * (TK * 128) + swz<128>(vrow, chunk & 7);
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(addr, b0, b1, b2, b3);
          mma_bf16(o[2 * dp], pa[2 * kt], pa[2 * kt + 1], b0, b1);
          mma_bf16(o[2 * dp + 1], pa[2 * kt], pa[2 * kt + 1], b2, b3);
        }
      }
    }
    __syncwarp();
  }
  if (!ok && lane == 0) {
    // Let copies already issued by this warp land before the CTA exits.
    for (int u = 0; u <= issued_last; ++u) {
      if (warp + u * kWarps >= ntiles) break;
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(&my_full[u % kBufs], (u / kBufs) & 1))
        if (globaltimer_ns() - t0 > FA_WAIT_LIMIT_NS) break;
    }
  }

  l += __shfl_xor_sync(0xffffffffu, l, 1);
  l += __shfl_xor_sync(0xffffffffu, l, 2);
  if (V_INT8) {
    // remove the +1152 code bias: every column of row g gained 1152 * sum_k P[g][k]
    p_sum += __shfl_xor_sync(0xffffffffu, p_sum, 1);
    p_sum += __shfl_xor_sync(0xffffffffu, p_sum, 2);
#pragma unroll
    for (int i = 0; i < DN; ++i) {
      o[i][0] -= kCodeBias * p_sum;
      o[i][1] -= kCodeBias * p_sum;
    }
  }

  // Merge the warps' partial states: merge[w][g][0..D) = O, [D] = m, [D+1] = l.
  __syncthreads();
  if (g < G) {
    float* mw = merge + (warp * 8 + g) * (D + 2);
#pragma unroll
    for (int i = 0; i < DN; ++i) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        // int8 V: n-tile i = (chunk i/2, parity i%2) holds d = 16(i/2) + 4t + 2e + i%2
        const int d = V_INT8 ? 16 * (i >> 1) + 4 * t + 2 * e + (i & 1) : 8 * i + 2 * t + e;
        mw[d] = o[i][e];
      }
    }
    if (t == 0) { mw[D] = m_ref; mw[D + 1] = l; }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
    const int gg = idx / D, d = idx % D;
    float m = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) m = fmaxf(m, merge[(w * 8 + gg) * (D + 2) + D]);
    float lt = 0.f, acc = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float* mw = merge + (w * 8 + gg) * (D + 2);
      if (mw[D] == -INFINITY) continue;   // warp had no tile
      const float sc = ex2_approx(mw[D] - m);
      lt += mw[D + 1] * sc;
      acc += mw[d] * sc;
    }
    const int64_t row = ws_row0 + (int64_t)gg * p.S;
    p.ws_o[row * D + d] = acc / lt;
    if (d == 0) p.ws_lse[row] = (m + log2f(lt)) * 0.69314718055994530942f;
  }
}

template <int D, bool V_INT8>
cudaError_t launch_i8(const CUtensorMap& k, const CUtensorMap& v, const CUtensorMap& ks, const CUtensorMap& vs,
                      const DecodeParams& p, cudaStream_t s) {
  using Cfg = Dec8Cfg<D, V_INT8>;
  auto kern = fa_decode_split_i8_kernel<D, V_INT8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
  if (e != cudaSuccess) return e;
  kern<<<dim3(p.S, p.Hkv, p.B), kWarps * 32, Cfg::kSmemBytes, s>>>(k, v, ks, vs, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_decode_combine(D, p, s);
}

// One warp per row of D values: codes = round-half-even(x / scale) with
// scale = max|x| / 127, both in fp32 (IEEE division, rintf).
template <int D>
__global__ void __launch_bounds__(256) quantize_kv_int8_kernel(const __nv_bfloat16* __restrict__ x,
                                                               int8_t* __restrict__ codes, float* __restrict__ scales,
                                                               int64_t rows, int L, int H) {
  constexpr int PER = D / 32;   // values per lane
  const int64_t row = (int64_t)blockIdx.x * 8 + threadIdx.x / 32;   // (b * L + j) * H + h
  const int lane = threadIdx.x % 32;
  if (row >= rows) return;
  float v[PER];
  const __nv_bfloat16* xr = x + row * D + lane * PER;
#pragma unroll
  for (int i = 0; i < PER; ++i) v[i] = __bfloat162float(xr[i]);
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < PER; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const float sc = __fdiv_rn(amax, 127.f);
  int8_t* cr = codes + row * D + lane * PER;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    float r = amax == 0.f ? 0.f : rintf(__fdiv_rn(v[i], sc));
    r = fminf(fmaxf(r, -127.f), 127.f);
    cr[i] = (int8_t)(int)r;
  }
  if (lane == 0) {
    const int h = (int)(row % H);
    const int64_t bj = row / H;
    const int j = (int)(bj % L);
    const int64_t bb = bj / L;
    scales[(bb * H + h) * L + j] = sc;
  }
}

}  // namespace

int decode_int8_tile_keys(int D) { return 4096 / D; }

cudaError_t launch_fa_decode_int8(int D, bool v_int8, const CUtensorMap& k, const CUtensorMap& v,
                                  const CUtensorMap& ks, const CUtensorMap& vs, const DecodeParams& p,
                                  cudaStream_t stream) {
  switch (D) {
    case 64: return v_int8 ? launch_i8<64, true>(k, v, ks, vs, p, stream) : launch_i8<64, false>(k, v, ks, vs, p, stream);
    case 128:
      return v_int8 ? launch_i8<128, true>(k, v, ks, vs, p, stream) : launch_i8<128, false>(k, v, ks, vs, p, stream);
    case 256:
      return v_int8 ? launch_i8<256, true>(k, v, ks, vs, p, stream) : launch_i8<256, false>(k, v, ks, vs, p, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_quantize_kv_int8(const void* x, void* codes, float* scales, int B, int L, int H, int D,
                                    cudaStream_t stream) {
  const int64_t rows = (int64_t)B * L * H;
  const unsigned grid = (unsigned)((rows + 7) / 8);
  const auto* xx = static_cast<const __nv_bfloat16*>(x);
  auto* cc = static_cast<int8_t*>(codes);
  switch (D) {
    case 64: quantize_kv_int8_kernel<64><<<grid, 256, 0, stream>>>(xx, cc, scales, rows, L, H); break;
    case 128: quantize_kv_int8_kernel<128><<<grid, 256, 0, stream>>>(xx, cc, scales, rows, L, H); break;
    case 256: quantize_kv_int8_kernel<256><<<grid, 256, 0, stream>>>(xx, cc, scales, rows, L, H); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

unsigned int decode_int8_read_and_clear_status() {
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof v) != cudaSuccess) return 0xFFFFFFFFu;
  cudaMemcpyToSymbol(g_device_status, &zero, sizeof zero);
  return v;
}

}  // namespace ta23
