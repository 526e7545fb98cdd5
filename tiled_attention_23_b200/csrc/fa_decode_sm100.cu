// Split-KV decode for sm_100a: one query token per sequence against a KV
// cache, the keys of each sequence cut into chunks whose partial results
// (O_c, L_c) are merged through their log-sum-exp in a second, tiny kernel.
//
// The split-K decode backend is named on the xformers page ("5 years, 10K
// stars: how xformers redefines Transformer acceleration with the Bias
// protocol"); the merge is the running-max / running-sum algebra of step 2 in
// section 二 of "FlashAttention in Ascend CANN ops-transformer", applied to
// chunk results instead of blocks.
//
// The path is bound by HBM bandwidth (every valid K and V row is read once;
// about 4 FLOP per byte at GQA group 4), so the design is about moving bytes:
//  * one CTA per (split, kv head, batch) serves all G query heads of the group,
//    so each K/V byte is read from HBM exactly once;
//  * each warp streams its own K/V tiles (round-robin over the chunk) with TMA
//    bulk-tensor copies into a private 3-deep ring of 128-byte-swizzled shared
//    memory buffers, two tiles always in flight per warp;
//  * the math is two small matrix products per tile done with warp-level
//    mma.sync (m16n8k16, bf16 in, fp32 accumulate): the G <= 8 query rows are
//    padded to 16, which costs tensor-pipe slots that are idle anyway here and
//    keeps the issue slots free for the memory stream.
// Each warp keeps its own online-softmax state; the warps of a CTA merge
// theirs in shared memory and write one normalised partial per (b, h, split).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>
#include <mutex>

#include "ptx.cuh"
#include "ta23.h"
#include "fa_kernels.h"

namespace ta23 {
namespace {

constexpr int kWarps = 4;
constexpr int kBufs = 3;
constexpr float kRescaleThreshold = 8.0f;

template <int D>
struct DecCfg {
  static constexpr int TK = D == 64 ? 32 : 16;              // keys per tile (16-key k-steps)
  static constexpr int kDBlocks = D / 64;
  static constexpr int kBoxBytes = TK * 128;                // one 64-wide block of TK keys
  static constexpr int kTileBytes = kDBlocks * kBoxBytes;   // K (or V) tile
  static constexpr int kBufBytes = 2 * kTileBytes;          // K then V
  static constexpr int kRingBytes = kWarps * kBufs * kBufBytes;
  static constexpr int kMergeBytes = kWarps * 8 * (D + 2) * 4;   // aliases the ring at the end
  static constexpr int kSmemBytes = kRingBytes + 256 + 1024;
  static_assert(kMergeBytes <= kRingBytes, "merge area must fit in the ring");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static constexpr int NT = TK / 8;                         // n-tiles of 8 keys
  static_assert(TK % 16 == 0, "a tile must hold whole 16-key k-steps");
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
// D = A(16x16 bf16, rows >= 8 zero: a1 = a3 = 0) * B(16x8 bf16) + C, fp32.
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

// Byte offset, inside a 128-byte-swizzled box of rows of 64 bf16, of the
// 16-byte chunk `chunk` (0..7) of row `row`.
__device__ __forceinline__ uint32_t sw128(int row, int chunk) {
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// PAGED: the cache is a pool of pages ([num_pages, page_size, Hkv, D]) and a
// per-sequence block table maps key j to page block_table[b][j / page_size],
// row j % page_size (the paged layout the xformers page lists among its
// structured attention biases).  Each 16-key box of a tile is fetched from its
// own page, so page_size only has to be a multiple of 16.
template <int D, bool PAGED>
__global__ void __launch_bounds__(kWarps * 32)
fa_decode_split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       DecodeParams p) {
  using Cfg = DecCfg<D>;
  constexpr int TK = Cfg::TK, NT = Cfg::NT, KS = D / 16, DN = D / 8;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* ring = base;
  float* merge = reinterpret_cast<float*>(base);   // reused once every warp is done with its ring
  uint64_t* full = reinterpret_cast<uint64_t*>(base + Cfg::kRingBytes);  // [kWarps][kBufs]

  const int split = blockIdx.x, hkv = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int g = lane >> 2, t = lane & 3;   // mma fragment coordinates
  const int G = p.G;

  int n = p.seqlens[b];
  n = n < 1 ? 1 : (n > p.Lmax ? p.Lmax : n);
  const int per = (n + p.S - 1) / p.S;
  const int C = ((per + 63) / 64) * 64;
  const int j0 = split * C;
  const int j1 = min(j0 + C, n);
  const int64_t ws_row0 = ((int64_t)b * p.Hq + (int64_t)hkv * G) * p.S + split;  // (b, h = hkv*G, split)

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

  unsigned char* my_ring = ring + warp * kBufs * Cfg::kBufBytes;
  uint64_t* my_full = full + warp * kBufs;
  const uint64_t pol = l2_policy_evict_first();
  auto issue = [&](int u) {   // local tile u of this warp -> buffer u % kBufs
    const int tile = warp + u * kWarps;
    if (tile >= ntiles) return;
    unsigned char* buf = my_ring + (u % kBufs) * Cfg::kBufBytes;
    uint64_t* bar = &my_full[u % kBufs];
    const int key0 = j0 + tile * TK;
    mbar_arrive_expect_tx(bar, Cfg::kBufBytes);
    if (PAGED) {
      // Boxes of 16 keys; a box past the sequence end (only in the last tile)
      // re-reads the last page in use, whose rows are masked below.
      const int last_page = (n - 1) / p.page_size;
#pragma unroll
      for (int sb = 0; sb < TK / kPagedBoxRows; ++sb) {
        const int key = key0 + sb * kPagedBoxRows;
        const int pg = min(key / p.page_size, last_page);
        const int phys = __ldg(p.block_table + (int64_t)b * p.max_pages + pg);
        const int row = key - pg * p.page_size;
        const int r = key < n ? row : 0;
#pragma unroll
        for (int db = 0; db < Cfg::kDBlocks; ++db) {
          const int off = db * Cfg::kBoxBytes + sb * kPagedBoxRows * 128;
          tma_load_4d_hint(buf + off, &tmK, bar, db * 64, hkv, r, phys, pol);
          tma_load_4d_hint(buf + Cfg::kTileBytes + off, &tmV, bar, db * 64, hkv, r, phys, pol);
        }
      }
    } else {
#pragma unroll
      for (int db = 0; db < Cfg::kDBlocks; ++db) {
        tma_load_4d_hint(buf + db * Cfg::kBoxBytes, &tmK, bar, db * 64, hkv, key0, b, pol);
        tma_load_4d_hint(buf + Cfg::kTileBytes + db * Cfg::kBoxBytes, &tmV, bar, db * 64, hkv, key0, b, pol);
      }
    }
  };
  if (lane == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    for (int u = 0; u < kBufs - 1; ++u) issue(u);
  }

  // Query fragments (rows g < G hold query heads hkv*G + g; other rows are
  // zero), loaded after the first copies are issued so the latencies overlap.
  uint32_t qa0[KS], qa2[KS];
  {
    const __nv_bfloat16* qrow = reinterpret_cast<const __nv_bfloat16*>(p.q) + ((int64_t)b * p.Hq + hkv * G + g) * D;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      qa0[ks] = (g < G) ? *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 2 * t) : 0u;
      qa2[ks] = (g < G) ? *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 8 + 2 * t) : 0u;
    }
  }

  float o[DN][4];
#pragma unroll
  for (int i = 0; i < DN; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_ref = -INFINITY, l = 0.f;   // row g (base-2 units); l is this thread's partial sum
  const float sl2 = p.scale_log2;
  int issued_last = kBufs - 2;
  bool ok = true;

  for (int u = 0;; ++u) {
    const int tile = warp + u * kWarps;
    if (tile >= ntiles) break;
    if (lane == 0) { issue(u + kBufs - 1); issued_last = u + kBufs - 1; }
    ok = mbar_wait(&my_full[u % kBufs], (u / kBufs) & 1, nullptr);
    if (!ok) break;
    const uint32_t sK = smem_u32(my_ring + (u % kBufs) * Cfg::kBufBytes);
    const uint32_t sV = sK + Cfg::kTileBytes;
    const int key0 = j0 + tile * TK;
    const bool tail = key0 + TK > j1;
    if (tail) {
      // Cache rows past the sequence end hold arbitrary data: zero them in V so
      // that 0 * garbage cannot reach the accumulator.
      const int first = j1 - key0;   // first invalid row of the tile
      uint4* vbuf = reinterpret_cast<uint4*>(my_ring + (u % kBufs) * Cfg::kBufBytes + Cfg::kTileBytes);
      for (int i = lane; i < Cfg::kDBlocks * (TK - first) * 8; i += 32) {
        const int db = i / ((TK - first) * 8), rem = i % ((TK - first) * 8);
        vbuf[(db * Cfg::kBoxBytes + (first + rem / 8) * 128) / 16 + (rem % 8)] = make_uint4(0, 0, 0, 0);
      }
      __syncwarp();
    }

    // S = Q K^T for NT n-tiles of 8 keys.
    float s[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
      const int krow = nt * 8 + (lane & 7);   // key row supplying this lane's ldmatrix address
#pragma unroll
      for (int ks = 0; ks < KS; ks += 2) {
        // 4 matrices: d chunks 2ks, 2ks+1, 2ks+2, 2ks+3 (8 d each) for keys nt*8..+7
        const int chunk = 2 * ks + (lane >> 3);          // 16-byte chunk along D (0..D/8-1)
        const uint32_t addr = sK + (chunk >> 3) * Cfg::kBoxBytes + sw128(krow, chunk & 7);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(addr, b0, b1, b2, b3);
        mma16816(s[nt], qa0[ks], qa2[ks], b0, b1);
        mma16816(s[nt], qa0[ks + 1], qa2[ks + 1], b2, b3);
      }
    }
    // Keys past the end of the chunk take no part (only in the last tile).
    float mx = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        if (tail && key0 + nt * 8 + 2 * t + e >= j1) s[nt][e] = -INFINITY;
        mx = fmaxf(mx, s[nt][e]);
      }
    }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float t_max = mx * sl2;   // finite: every tile holds at least one valid key
    float m_new = m_ref, alpha = 1.f;
    if (m_ref == -INFINITY) {
      m_new = t_max;
    } else if (t_max > m_ref + kRescaleThreshold) {
      m_new = t_max;
      alpha = ex2_approx(m_ref - m_new);
      l *= alpha;
#pragma unroll
      for (int i = 0; i < DN; ++i) { o[i][0] *= alpha; o[i][1] *= alpha; }
    }
    m_ref = m_new;
    // P = 2^(t - m), packed as the A operand of the PV product.
    uint32_t pa[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float p0 = ex2_approx(fmaf(s[nt][0], sl2, -m_new));
      float p1 = ex2_approx(fmaf(s[nt][1], sl2, -m_new));
      if (tail) {
        if (key0 + nt * 8 + 2 * t >= j1) p0 = 0.f;
        if (key0 + nt * 8 + 2 * t + 1 >= j1) p1 = 0.f;
      }
      l += p0 + p1;
      pa[nt] = pack_bf16x2(p0, p1);
    }
    // O += P V: k-steps of 16 keys (two n-tiles of P), n-tiles of 8 along D.
#pragma unroll
    for (int kt = 0; kt < NT / 2; ++kt) {
      // matrices: (keys 16kt..+7, d 16i..+7), (keys +8..+15, same d), (keys 16kt..+7, d +8), (keys +8.., d +8)
      const int vrow = kt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int dp = 0; dp < DN / 2; ++dp) {
        const int chunk = 2 * dp + (lane >> 4);
        const uint32_t addr = sV + (chunk >> 3) * Cfg::kBoxBytes + sw128(vrow, chunk & 7);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(addr, b0, b1, b2, b3);
        mma16816(o[2 * dp], pa[2 * kt], pa[2 * kt + 1], b0, b1);
        mma16816(o[2 * dp + 1], pa[2 * kt], pa[2 * kt + 1], b2, b3);
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

  // Row sums: the four threads of a quad hold disjoint keys of the same row.
  l += __shfl_xor_sync(0xffffffffu, l, 1);
  l += __shfl_xor_sync(0xffffffffu, l, 2);

  // Merge the warps' partial states: merge[w][g][0..D) = O, [D] = m, [D+1] = l.
  __syncthreads();   // every warp is done reading its ring: reuse it
  if (g < G) {
    float* mw = merge + (warp * 8 + g) * (D + 2);
#pragma unroll
    for (int i = 0; i < DN; ++i) {
      mw[i * 8 + 2 * t] = o[i][0];
      mw[i * 8 + 2 * t + 1] = o[i][1];
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

// O = sum_c exp(L_c - L) O_c with L = ln sum_c exp(L_c), chunks in order c = 0..S-1.
template <int D>
__global__ void __launch_bounds__(128) fa_decode_combine_kernel(DecodeParams p) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t bh = (int64_t)blockIdx.x * 4 + warp;
  if (bh >= (int64_t)p.B * p.Hq) return;
  const float* lse_c = p.ws_lse + bh * p.S;
  float m = -INFINITY;
  for (int c = 0; c < p.S; ++c) m = fmaxf(m, lse_c[c]);
  float sum = 0.f;
  for (int c = 0; c < p.S; ++c) sum += (lse_c[c] == -INFINITY) ? 0.f : expf(lse_c[c] - m);
  const float L = m + logf(sum);
  constexpr int PER = D / 32;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  for (int c = 0; c < p.S; ++c) {
    if (lse_c[c] == -INFINITY) continue;
    const float w = expf(lse_c[c] - L);
    const float* oc = p.ws_o + (bh * p.S + c) * D;
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] += w * oc[lane + 32 * e];
  }
  __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) + bh * D;
#pragma unroll
  for (int e = 0; e < PER; ++e) orow[lane + 32 * e] = __float2bfloat16_rn(acc[e]);
  if (p.lse && lane == 0) p.lse[bh] = L;
}

template <int D, bool PAGED>
cudaError_t launch_decode(const CUtensorMap& k, const CUtensorMap& v, const DecodeParams& p, cudaStream_t s) {
  using Cfg = DecCfg<D>;
  auto kern = fa_decode_split_kernel<D, PAGED>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
  if (e != cudaSuccess) return e;
  kern<<<dim3(p.S, p.Hkv, p.B), kWarps * 32, Cfg::kSmemBytes, s>>>(k, v, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t rows = (int64_t)p.B * p.Hq;
  fa_decode_combine_kernel<D><<<(unsigned)((rows + 3) / 4), 128, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

int decode_tile_keys(int D) { return D == 64 ? 32 : 16; }

cudaError_t launch_decode_combine(int D, const DecodeParams& p, cudaStream_t s) {
  const int64_t rows = (int64_t)p.B * p.Hq;
  const unsigned grid = (unsigned)((rows + 3) / 4);
  switch (D) {
    case 64: fa_decode_combine_kernel<64><<<grid, 128, 0, s>>>(p); break;
    case 128: fa_decode_combine_kernel<128><<<grid, 128, 0, s>>>(p); break;
    case 256: fa_decode_combine_kernel<256><<<grid, 128, 0, s>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_fa_decode(int D, bool paged, const CUtensorMap& k, const CUtensorMap& v, const DecodeParams& p,
                             cudaStream_t stream) {
  switch (D) {
    case 64: return paged ? launch_decode<64, true>(k, v, p, stream) : launch_decode<64, false>(k, v, p, stream);
    case 128: return paged ? launch_decode<128, true>(k, v, p, stream) : launch_decode<128, false>(k, v, p, stream);
    case 256: return paged ? launch_decode<256, true>(k, v, p, stream) : launch_decode<256, false>(k, v, p, stream);
    default: return cudaErrorInvalidValue;
  }
}

// Fixed scratch of fa_decode_splitkv_noalloc: every GPU that loads this
// library holds it until the process exits.  In host code the name is only a
// host-side stand-in, so the device address is looked up per device below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

cudaError_t noalloc_scratch(void** ptr, size_t* bytes) {
  constexpr int kMaxDevices = 256;
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);   // with device `dev` current
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *ptr = addr[dev];
  *bytes = sizeof(g_noalloc_scratch);
  return cudaSuccess;
}

unsigned int decode_read_and_clear_status() {
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof v) != cudaSuccess) return 0xFFFFFFFFu;
  cudaMemcpyToSymbol(g_device_status, &zero, sizeof zero);
  return v;
}

}  // namespace ta23
