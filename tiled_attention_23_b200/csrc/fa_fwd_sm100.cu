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
// query blocks, split the work of a block across warps.  On sm_100a that
// becomes a warp-specialised CTA:
//
//   load warp      TMA: the CTA's query tiles once, then K_j / V_j through a
//                  ring of shared-memory slots (128-byte swizzle; 64-byte
//                  for the 64-byte rows of e4m3 at head_dim 64)
//   MMA warp       allocates tensor memory; one thread issues
//                    S = Q K_j^T   (A = Q, B = K_j from shared memory)
//                    O += P V_j    (A = P from tensor memory, B = V_j)
//   wait warp      (pair kernel) waits for the tiles the next products read
//                  while the MMA warp's issue is blocked on the tensor pipe,
//                  and hands each group over at a named barrier
//   softmax warps  one thread per query row (= tensor-memory lane): row max,
//                  exp2, row sum, P -> tensor memory as bf16, the rare O
//                  rescale, and the epilogue (O / l and L).
//
// head_dim 64 and 128 ("pair" kernel): a CTA owns two 128-row query tiles of
// one (batch, head) that share every K/V tile.  Tensor memory holds S0, S1
// (128 columns each), O0, O1; P_w is written over the columns of S_w it was
// computed from.  The MMA thread issues, per K/V tile j,
//     S0_j, PV1_{j-1}, S1_j, PV0_j
// so each softmax warpgroup works on its S while the tensor core runs the
// other tile's products.  Writing S_w again after PV_w has read P_w from the
// same columns relies on tcgen05.mma operations of one thread executing in
// issue order.
//
// Large batches run the pair kernel persistently: one CTA per SM walks a
// list of work items (pairs of query tiles), pairing the heavy and the light
// causal pair of a head so that every CTA gets the same amount of work.  The
// load warp fetches the next item's query tiles as soon as the current
// item's last S products have read theirs, and the next item's first PV of a
// query tile waits only for that tile's epilogue, so the per-CTA start-up
// (launch, barrier and tensor-memory set-up, the first query load) is paid
// once per SM instead of once per item.
//
// head_dim 256 ("single" kernel): O needs 256 columns, so a CTA owns one
// query tile, uses 64-key K/V tiles and double-buffers S, with P in columns
// of its own.
//
// FP8 mode (both kernels): Q, K, V as e4m3 codes with per-head dequantisation
// factors (FlashAttention-3's FP8 support, named on "FlashAttention-2 (TH)"),
// products on tcgen05 kind::f8f6f4, and P written to tensor memory as e4m3.
// The factors fold into the exponent scale and the epilogue; P is scaled by
// 2^6 under a reference-max slack of 2, so a row's largest p lies in
// [2^6, 2^8], inside e4m3's range and far above its subnormals.
//
// Online softmax (base 2): t = s * scale * log2(e).  A row keeps a reference
// max m and the sum l of 2^(t - m).  m moves only when a tile's max exceeds
// it by more than 8, and then O and l are rescaled by 2^(m_old - m_new);
// otherwise exponentials are taken against the stale m (exact algebra; P stays
// <= 256 in bf16).  Causal masks are computed from indices (bottom-right:
// key j allowed for query i iff j <= i + Lk - Lq); tiles wholly above the
// diagonal are never loaded and only tiles crossing it or the end of the keys
// are masked element by element.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cstdint>

#include "ptx.cuh"
#include "fa_kernels.h"

namespace ta23 {
namespace {

constexpr int BM = 128;                  // query rows per tile (one tensor-memory lane each)
constexpr float kRescaleThreshold = 8.0f;

// ---------------------------------------------------------------------------
// Per-row softmax pieces shared by both kernels (one thread = one row).
// ---------------------------------------------------------------------------
// Pretend-writes the registers so the compiler cannot use them before the
// preceding tcgen05.wait::ld has retired.
template <int N>
__device__ __forceinline__ void reg_fence(float (&s)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+f"(s[i]));
}

// Loads N fp32 columns of this thread's row starting at taddr.
template <int N>
__device__ __forceinline__ void load_row(uint32_t taddr, float (&s)[N]) {
  static_assert(N % 32 == 0, "rows load in chunks of 32 columns");
#pragma unroll
  for (int c = 0; c < N; c += 32) {
    uint32_t r[32];
    tmem_ld32(taddr + c, r);
#pragma unroll
    for (int e = 0; e < 32; ++e) s[c + e] = __uint_as_float(r[e]);
  }
  tmem_wait_ld();
  reg_fence(s);
}

template <int N>
__device__ __forceinline__ float row_max(const float (&s)[N]) {
  static_assert(N % 16 == 0, "row length");
  float m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = fmaxf(s[i], s[i + 8]);
#pragma unroll
  for (int c = 16; c < N; c += 16)
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = fmax3(m[i], s[c + i], s[c + 8 + i]);
  return fmaxf(fmax3(m[0], m[1], m[2]), fmax3(fmax3(m[3], m[4], m[5]), m[6], m[7]));
}

#ifndef TA23_POLY_NUM
#define TA23_POLY_NUM 1
#define TA23_POLY_DEN 3
#endif
// The last kPolyNum of every kPolyDen column pairs take their exponentials
// from exp2_poly2, the others from the MUFU (kPolyNum = 0: all on the MUFU).
constexpr int kPolyNum = TA23_POLY_NUM, kPolyDen = TA23_POLY_DEN;
#ifndef TA23_F8_POLY_NUM
#define TA23_F8_POLY_NUM 1
#define TA23_F8_POLY_DEN 3
#define TA23_F8_POLY_DEG 2
#endif
// The split for e4m3 P (whose rounding allows the cheaper degree-2 fit).
constexpr int kF8PolyNum = TA23_F8_POLY_NUM, kF8PolyDen = TA23_F8_POLY_DEN, kF8PolyDeg = TA23_F8_POLY_DEG;

// p = 2^(s * sl2 - m) as bf16 pairs into tensor memory (N/2 columns at
// taddr); returns the fp32 row sum.  With MASK, keys past key_limit get p = 0.
// The exponent argument and the row sum use the packed two-lane fp32 FMA/ADD
// of sm_100 (one instruction per column pair).
template <int N, bool MASK>
__device__ __forceinline__ float exp_store_row(const float (&s)[N], float sl2, float m, uint32_t taddr,
                                               int key0, int key_limit) {
  const float2 scale2 = make_float2(sl2, sl2), neg_m2 = make_float2(-m, -m);
  float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
  for (int c = 0; c < N; c += 64) {
    uint32_t pk[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const float2 x = __ffma2_rn(make_float2(s[c + 2 * e], s[c + 2 * e + 1]), scale2, neg_m2);
      float p0, p1;
      if (e % kPolyDen >= kPolyDen - kPolyNum) {
        const float2 pp = exp2_poly2(x);
        p0 = pp.x;
        p1 = pp.y;
      } else {
        p0 = ex2_approx(x.x);
        p1 = ex2_approx(x.y);
      }
      if (MASK) {
        if (key0 + c + 2 * e > key_limit) p0 = 0.f;
        if (key0 + c + 2 * e + 1 > key_limit) p1 = 0.f;
      }
      acc[e & 3] = __fadd2_rn(acc[e & 3], make_float2(p0, p1));
      pk[e] = pack_bf16x2(p0, p1);
    }
    tmem_st32(taddr + c / 2, pk);
  }
  const float2 t = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
  return t.x + t.y;
}

// The same for 8-bit P: p = 2^(s * sl2 - m) rounded to e4m3 (round to
// nearest even, saturating), four keys to a tensor-memory column (N/4
// columns at taddr, lower key in the lower byte); the fp32 row sum is of the
// unrounded values.
template <int N, bool MASK>
__device__ __forceinline__ float exp_store_row_e4m3(const float (&s)[N], float sl2, float m, uint32_t taddr,
                                                    int key0, int key_limit) {
  const float2 scale2 = make_float2(sl2, sl2), neg_m2 = make_float2(-m, -m);
  float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
  for (int c = 0; c < N; c += 64) {
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const float2 x = __ffma2_rn(make_float2(s[c + 2 * e], s[c + 2 * e + 1]), scale2, neg_m2);
      float p0, p1;
      if (e % kF8PolyDen >= kF8PolyDen - kF8PolyNum) {
        const float2 pp = kF8PolyDeg == 2 ? exp2_poly2_deg2(x) : exp2_poly2(x);
        p0 = pp.x;
        p1 = pp.y;
      } else {
        p0 = ex2_approx(x.x);
        p1 = ex2_approx(x.y);
      }
      if (MASK) {
        if (key0 + c + 2 * e > key_limit) p0 = 0.f;
        if (key0 + c + 2 * e + 1 > key_limit) p1 = 0.f;
      }
      acc[e & 3] = __fadd2_rn(acc[e & 3], make_float2(p0, p1));
      const uint32_t two = __nv_cvt_float2_to_fp8x2(make_float2(p0, p1), __NV_SATFINITE, __NV_E4M3);
      pk[e / 2] = (e & 1) ? (pk[e / 2] | (two << 16)) : two;
    }
    tmem_st16(taddr + c / 4, pk);
  }
  const float2 t = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
  return t.x + t.y;
}

template <int D>
__device__ __forceinline__ void rescale_o(uint32_t taddr, float a) {
#pragma unroll 1
  for (int c = 0; c < D; c += 32) {
    uint32_t r[32];
    tmem_ld32(taddr + c, r);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 32; ++e) asm volatile("" : "+r"(r[e]));
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      const float2 v = __fmul2_rn(make_float2(__uint_as_float(r[e]), __uint_as_float(r[e + 1])), make_float2(a, a));
      r[e] = __float_as_uint(v.x);
      r[e + 1] = __float_as_uint(v.y);
    }
    tmem_st32(taddr + c, r);
  }
}

// O / l -> bf16 row of the output; L = (m + log2 l) ln 2.  The row's
// columns are loaded from tensor memory up to 128 at a time behind one wait,
// and written with 32-byte stores.
template <int D>
__device__ __forceinline__ void epilogue_row(uint32_t taddr, float m, float l, bool row_ok, __nv_bfloat16* orow,
                                             float* lse_ptr, float out_mul = 1.f) {
  const float inv_l = l > 0.f ? out_mul / l : 0.f;   // l == 0 only for a row without keys
  constexpr int CH = D < 128 ? D : 128;                // columns per wait
#pragma unroll 1
  for (int c0 = 0; c0 < D; c0 += CH) {
    uint32_t r[CH];
#pragma unroll
    for (int c = 0; c < CH; c += 32) tmem_ld32(taddr + c0 + c, *reinterpret_cast<uint32_t(*)[32]>(&r[c]));
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < CH; ++e) asm volatile("" : "+r"(r[e]));
#pragma unroll
    for (int c = 0; c < CH; c += 16) {
      uint32_t pk[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float2 v = __fmul2_rn(make_float2(__uint_as_float(r[c + 2 * e]), __uint_as_float(r[c + 2 * e + 1])),
                                    make_float2(inv_l, inv_l));
        pk[e] = pack_bf16x2(v.x, v.y);
      }
      if (row_ok) st_global_v8(orow + c0 + c, pk);
    }
  }
  if (row_ok && lse_ptr) {
    const float m_fin = (m == -INFINITY) ? 0.f : m;
    *lse_ptr = l > 0.f ? (m_fin + log2f(l)) * 0.69314718055994530942f : -INFINITY;
  }
}

// Row state of the online softmax.
struct RowState {
  float m = -INFINITY;   // reference max (base-2 units)
  float l = 0.f;         // sum of 2^(t - m)
};

// Decides the reference max for a tile whose max is t_max; returns the factor
// O and l must be multiplied by (1 when m does not move).
__device__ __forceinline__ float update_max(RowState& st, float t_max, bool& rescale,
                                            float threshold = kRescaleThreshold) {
  rescale = false;
  if (st.m == -INFINITY) {
    st.m = t_max;          // nothing accumulated yet
    return 1.f;
  }
  if (t_max > st.m + threshold) {
    const float a = ex2_approx(st.m - t_max);
    st.m = t_max;
    rescale = true;
    return a;
  }
  return 1.f;
}

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

// Number of K/V tiles of BN keys a query tile starting at row q0 needs.
__device__ __forceinline__ int kv_tiles(int q0, int Lq, int Lk, int off, int BN, bool causal) {
  if (q0 >= Lq) return 0;
  int n = (Lk + BN - 1) / BN;
  if (causal) {
    const int last_row = min(q0 + BM, Lq) - 1;
    const int last_key = min(last_row + off, Lk - 1);
    n = min(n, last_key / BN + 1);
  }
  return n;
}

// The problem one CTA works on: batch entry b of a fixed-shape batch, or
// sequence b of a packed variable-length batch (block-diagonal attention: a
// query token sees only keys of its own sequence, the "block diagonal"
// structured bias of the xformers page).
struct SeqView {
  int Lq, Lk, causal_off;
  int q_row0, k_row0;   // first row of the sequence in the Q and K/V tensor maps
  int tma_b;            // batch coordinate of the tensor maps
  int64_t o_tok0;       // output token index of query row 0
  int64_t lse0;         // lse index of query row 0 of head h (add h * lse_head_stride)
  int64_t lse_hs;       // lse stride between heads
};

template <bool VARLEN>
__device__ __forceinline__ SeqView seq_view(const FwdParams& p, int b) {
  SeqView v;
  if (VARLEN) {
    v.q_row0 = __ldg(p.cu_q + b);
    v.k_row0 = __ldg(p.cu_k + b);
    v.Lq = __ldg(p.cu_q + b + 1) - v.q_row0;
    v.Lk = __ldg(p.cu_k + b + 1) - v.k_row0;
    v.tma_b = 0;
    v.o_tok0 = v.q_row0;
    v.lse0 = v.q_row0;
    v.lse_hs = p.total_q;
  } else {
    v.Lq = p.Lq;
    v.Lk = p.Lk;
    v.q_row0 = v.k_row0 = 0;
    v.tma_b = b;
    v.o_tok0 = (int64_t)b * p.Lq;
    v.lse0 = (int64_t)b * p.Hq * p.Lq;
    v.lse_hs = p.Lq;
  }
  v.causal_off = v.Lk - v.Lq;
  return v;
}

// Whether query row qi of the sequence is written: inside the sequence and,
// for a packed batch, inside the packed tensor (cu_seqlens are device data).
template <bool VARLEN>
__device__ __forceinline__ bool row_in_range(const SeqView& sv, const FwdParams& p, int qi) {
  if (qi >= sv.Lq) return false;
  return !VARLEN || (uint32_t)(sv.q_row0 + qi) < (uint32_t)p.total_q;
}

// A row with no allowed key (only a packed batch can have one: an empty key
// sequence, or causal with more queries than keys) gets O = 0 and L = -inf.
template <int D>
__device__ __forceinline__ void write_empty_row(__nv_bfloat16* orow, float* lse_ptr) {
#pragma unroll
  for (int c = 0; c < D; c += 8) *reinterpret_cast<uint4*>(orow + c) = make_uint4(0, 0, 0, 0);
  if (lse_ptr) *lse_ptr = -INFINITY;
}

// ===========================================================================
// Pair kernel: head_dim 64 / 128, two query tiles per CTA, 128-key K/V tiles.
// ===========================================================================
// FP8: Q, K, V in e4m3 (one byte an element, so a 128-byte swizzle row holds
// 128 columns) and P in e4m3 in tensor memory.
template <int D, bool FP8 = false>
struct PairCfg {
  static constexpr int BN = 128;
  static constexpr int kRowBytes = FP8 ? D : 2 * D;
  // Tiles are stored as blocks of kSwz-byte rows with the kSwz-byte swizzle:
  // 128 bytes, or 64 for the 64-byte rows of e4m3 at head_dim 64.
  static constexpr int kSwz = kRowBytes < 128 ? kRowBytes : 128;
  static constexpr int kBlockCols = FP8 ? kSwz : kSwz / 2;      // columns per block row
  static constexpr int kDBlocks = D / kBlockCols;
  static_assert(kDBlocks >= 1 && D % kBlockCols == 0 && (kSwz == 64 || kSwz == 128), "head_dim");
  static constexpr int kQBlockBytes = BM * kSwz;
  static constexpr int kKVBlockBytes = BN * kSwz;
  static constexpr int kQBytes = kDBlocks * kQBlockBytes;      // one query tile
  static constexpr int kSlotBytes = kDBlocks * kKVBlockBytes;  // one K or V tile
#ifndef TA23_PAIR_SLOTS128
#define TA23_PAIR_SLOTS128 5
#endif
  static constexpr int kSlots = FP8 ? (D == 64 ? 12 : 10) : D == 64 ? 12 : TA23_PAIR_SLOTS128;
  // Three warpgroups: WG0 = load warp, MMA warp and two idle warps; WG1 and
  // WG2 = the softmax warpgroups of query tiles 0 and 1.  Launched at 168
  // registers a thread; setmaxnreg (a warpgroup-wide instruction) moves WG0 to
  // 56 and the softmax warpgroups to 224: 128*56 + 256*224 = 64512 = 384*168,
  // and per sub-partition (warps w, w+4, w+8) 56 + 224 + 224 = 504 <= 512.
  static constexpr int kThreads = 384;
  static constexpr int kRegsSoftmax = 224, kRegsOther = 56;
  // tensor memory columns: S0, S1, O0, O1; P_w at S_w + kPOff (64 columns of
  // bf16 pairs, or 32 of e4m3 quadruples)
  static constexpr int kS0 = 0, kS1 = 128, kO0 = 256, kO1 = 256 + D;
  static constexpr int kPOff = FP8 ? 96 : 64;
  // Reference-max slack (base 2) and, for e4m3 P, the exponent offset that
  // puts the largest p of a row in [2^6, 2^8] (so p <= 256 < 448, the e4m3
  // maximum, and only p below 2^-12 of the row max is subnormal).
  static constexpr float kThreshold = FP8 ? 2.f : kRescaleThreshold;
  static constexpr float kPExp = FP8 ? 6.f : 0.f;
  static constexpr int kSmemBytes = 2 * kQBytes + kSlots * kSlotBytes + 512 + 1024;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static_assert(256 + 2 * D <= 512, "tensor-memory budget");
};

struct PairBarriers {
  uint64_t q_full[2];       // query tile w of the current item has landed
  uint64_t q_empty[2];      // every S product of the item that reads query tile w is done
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_full[2];       // the item's last PV_w has landed in O_w
  uint64_t o_empty[2];      // the item's epilogue has read O_w
  uint64_t drain;
  uint64_t kv_full[12];
  uint64_t kv_empty[12];
  uint32_t tmem_base;
  int abort_flag;
  int handoff_ok[2];        // outcome of the wait warp's waits, by hand-off parity
};

// Work items of the pair kernel: a pair of 128-row query tiles of one (batch,
// head) starting at query row q0.  n0 / n1 = K/V tiles of query tile 0 / 1
// (n1 == 0 for a tail pair, else n1 >= n0).  An item with n0 == n1 == 0 has
// no products: q0 >= 0 for a packed sequence without keys (its rows get
// O = 0, L = -inf), q0 = -1 for no rows at all (a CTA past its sequence's
// queries, or the missing partner of an odd couple).
struct PairItem {
  int q0, h, b, n0, n1;
};

// The k-th item of this CTA (false after the last one).
//  sched 0: one item per CTA: pair (heaviest first) blockIdx.x of head
//           blockIdx.y, batch entry blockIdx.z.
//  sched 1: persistent CTAs over "couples" of pairs (n-1-c, c) of one head:
//           under a causal mask the two carry complementary work, so every
//           couple costs about the same and CTA g taking couples g, g + G, ...
//           (heavier pair first) is balanced; the CTAs running together cover
//           about G / (n/2) heads, whose K/V stay in L2.
template <bool CAUSAL, bool VARLEN>
__device__ __forceinline__ bool pair_item(const FwdParams& p, int k, PairItem& it, SeqView& sv) {
  int pr;
  it.n0 = it.n1 = 0;
  if (p.sched == 0) {
    if (k > 0) return false;
    it.h = blockIdx.y;
    it.b = blockIdx.z;
    sv = seq_view<VARLEN>(p, it.b);
    const int n_pairs = VARLEN ? (sv.Lq + 2 * BM - 1) / (2 * BM) : p.n_qtiles;
    it.q0 = -1;
    if ((int)blockIdx.x >= n_pairs) return true;   // past this sequence's queries: no work
    pr = n_pairs - 1 - blockIdx.x;
  } else {
    const int n = p.n_qtiles, nc = (n + 1) / 2;
    const long long u = blockIdx.x + (long long)(k >> 1) * gridDim.x;
    if (u >= (long long)p.Hq * p.B * nc) return false;
    const int hb = (int)(u / nc), c = (int)(u % nc);
    it.h = hb % p.Hq;
    it.b = hb / p.Hq;
    sv = seq_view<VARLEN>(p, it.b);
    it.q0 = -1;
    if ((k & 1) && c == n - 1 - c) return true;    // middle pair of an odd count: no partner
    pr = (k & 1) ? c : n - 1 - c;
  }
  it.q0 = pr * 2 * BM;
  it.n0 = kv_tiles(it.q0, sv.Lq, sv.Lk, sv.causal_off, 128, CAUSAL);
  it.n1 = kv_tiles(it.q0 + BM, sv.Lq, sv.Lk, sv.causal_off, 128, CAUSAL);
  return true;
}


// Shared-memory descriptor of a tile of SWZ-byte rows from its low word (start
// address >> 4, leading byte offset >> 4): stride byte offset 8 * SWZ (the
// next 8 rows), version 1, layout 128-byte swizzle (code 2) or 64-byte swizzle
// (code 4).
template <int SWZ>
__device__ __forceinline__ uint64_t desc_swz(uint32_t lo) {
  constexpr uint32_t hi = (uint32_t)(((8u * SWZ) >> 4) | (1u << 14) | ((SWZ == 128 ? 2u : 4u) << 29));
  return ((uint64_t)hi << 32) | lo;
}

// The MMAs of S = Q K^T for one 128-row query tile (A and B K-major, swizzled
// blocks of kSwz-byte rows); q_lo / k_lo: start address >> 4 of the tile's
// first block.  Called by the one elected lane of the MMA warp.
// Each instruction takes 32 bytes of the contraction: 16 bf16 or 32 e4m3 columns.
template <int D, bool FP8 = false>
__device__ __forceinline__ void pair_mma_s(uint32_t s_tmem, uint32_t q_lo, uint32_t k_lo) {
  using Cfg = PairCfg<D, FP8>;
  constexpr uint32_t idS = FP8 ? idesc_e4m3_f32(BM, Cfg::BN, 0, 0) : idesc_bf16_f32(BM, Cfg::BN, 0, 0);
  constexpr uint32_t kLbo = 1u << 16;   // leading byte offset field (unused for this layout)
  constexpr int kSteps = Cfg::kSwz / 32;   // 32-byte contraction steps per block row
#pragma unroll
  for (int kk = 0; kk < Cfg::kRowBytes / 32; ++kk) {
    const uint32_t qo = ((kk / kSteps) * Cfg::kQBlockBytes + (kk % kSteps) * 32) >> 4;
    const uint32_t ko = ((kk / kSteps) * Cfg::kKVBlockBytes + (kk % kSteps) * 32) >> 4;
    const uint64_t da = desc_swz<Cfg::kSwz>((q_lo + qo) | kLbo), db = desc_swz<Cfg::kSwz>((k_lo + ko) | kLbo);
    if (FP8)
      mma_f8_ss(s_tmem, da, db, idS, kk > 0 ? 1u : 0u);
    else
      mma_bf16_ss(s_tmem, da, db, idS, kk > 0 ? 1u : 0u);
  }
}

// The MMAs of O += P V_j (A = P from tensor memory, B = V_j MN-major); `first`
// overwrites O instead of accumulating.  Called by the elected lane.
// An instruction covers 16 keys (bf16) or 32 keys (e4m3): 8 columns of P and
// that many rows of V (kSwz bytes each).
template <int D, bool FP8 = false>
__device__ __forceinline__ void pair_mma_pv(uint32_t o_tmem, uint32_t p_tmem, uint32_t v_lo, bool first) {
  using Cfg = PairCfg<D, FP8>;
  constexpr int KK = FP8 ? 32 : 16;
  constexpr uint32_t idPV = FP8 ? idesc_e4m3_f32(BM, D, 0, 1) : idesc_bf16_f32(BM, D, 0, 1);
  constexpr uint32_t kLbo = (uint32_t)(Cfg::kKVBlockBytes >> 4) << 16;   // next block of V columns
#pragma unroll
  for (int kk = 0; kk < Cfg::BN / KK; ++kk) {
    const uint64_t bd = desc_swz<Cfg::kSwz>((v_lo + ((kk * KK * Cfg::kSwz) >> 4)) | kLbo);
    if (FP8)
      mma_f8_ts(o_tmem, p_tmem + kk * 8, bd, idPV, (!first || kk > 0) ? 1u : 0u);
    else
      mma_bf16_ts(o_tmem, p_tmem + kk * 8, bd, idPV, (!first || kk > 0) ? 1u : 0u);
  }
}

// One issue group for query tile W and K/V tile j of an item whose K/V fills
// start at f0: O_W += P_W V_j, then (when tile W has a next K/V tile)
// S_W,j+1 = Q_W K_j+1^T.  The wait warp first waits (the whole warp) for O_W
// to be free (the previous item's epilogue; first tile only), for V_j and for
// K_j+1 (pair_group_wait), which are usually ready long before P; then the
// MMA warp waits for P_W,j itself (at that point the tensor pipe is usually
// idle, so the wait is short) and its elected lane issues the two products
// back to back (pair_group_issue).  S_W,j+1 overwrites the columns P_W,j was
// read from, so it must follow PV_W,j; from the one issuer it enters the
// tensor pipe right behind it.  A K/V slot is released by a commit after the
// last product that reads it: V_j by PV1_j when tile 1 reads V_j, else by
// PV0_j; K_j+1 by S1_j+1 when tile 1 has it, else by S0_j+1.
template <int D, int NS, int W>
__device__ __forceinline__ bool pair_group_wait(PairBarriers& bar, int j, int nw, int f0, int oe,
                                                volatile int* abortf) {
  const int fk = f0 + 2 * j + 2, fv = f0 + 2 * j + 1;   // fills of K_j+1 and V_j
  bool got = true;
  if (j == 0 && oe >= 0) got = mbar_wait(&bar.o_empty[W], oe & 1, abortf);
  got = got && mbar_wait(&bar.kv_full[fv % NS], (fv / NS) & 1, abortf);
  if (j + 1 < nw) got = got && mbar_wait(&bar.kv_full[fk % NS], (fk / NS) & 1, abortf);
  return __all_sync(0xffffffffu, got) && !*abortf;
}

template <int D, int NS, int W, bool FP8>
__device__ __forceinline__ void pair_group_issue(PairBarriers& bar, int j, int nw, int n1, int f0, uint32_t tmem,
                                                 uint32_t q_lo, uint32_t kv_lo) {
  using Cfg = PairCfg<D, FP8>;
  const int fk = f0 + 2 * j + 2, fv = f0 + 2 * j + 1;
  const bool more = j + 1 < nw;
  const bool last_v = W == 1 || j >= n1;
  const bool last_k = W == 1 || j + 1 >= n1;
  if (elect_one()) {
    const uint32_t s_col = tmem + (W ? Cfg::kS1 : Cfg::kS0);
    pair_mma_pv<D, FP8>(tmem + (W ? Cfg::kO1 : Cfg::kO0), s_col + Cfg::kPOff,
                        kv_lo + (uint32_t)((fv % NS) * Cfg::kSlotBytes >> 4), j == 0);
    if (!more) tc_commit(&bar.o_full[W]);
    if (last_v) tc_commit(&bar.kv_empty[fv % NS]);
    if (more) {
      pair_mma_s<D, FP8>(s_col, q_lo + (uint32_t)(W * (Cfg::kQBytes >> 4)),
                         kv_lo + (uint32_t)((fk % NS) * Cfg::kSlotBytes >> 4));
      tc_commit(&bar.s_full[W]);
      if (j + 2 == nw) tc_commit(&bar.q_empty[W]);   // the last S product of tile W
      if (last_k) tc_commit(&bar.kv_empty[fk % NS]);
    }
  }
  __syncwarp();
}

// Hand-off c from the wait warp to the MMA warp: both warps meet at a named
// barrier once per issue group, in the same order (bar.sync on both sides, so
// neither runs ahead), and the wait warp's verdict travels in a flag
// double-buffered by hand-off parity.  The wait warp stops after sending a
// failed verdict, the MMA warp after receiving one, so every barrier use is
// matched.  A failed wait of the MMA warp itself raises the abort flag, after
// which the wait warp's next verdict is a failure: until then the MMA warp
// keeps taking hand-offs without issuing.
constexpr uint32_t kHandoffBar = 1;
__device__ __forceinline__ void handoff_send(PairBarriers& bar, int c, bool ok) {
  if (lane_id() == 0) bar.handoff_ok[c & 1] = ok ? 1 : 0;
  __syncwarp();
  named_barrier_sync(kHandoffBar, 64);
}
__device__ __forceinline__ bool handoff_recv(PairBarriers& bar, int c) {
  named_barrier_sync(kHandoffBar, 64);
  return *reinterpret_cast<volatile int*>(&bar.handoff_ok[c & 1]) != 0;
}

template <int D, bool CAUSAL, bool VARLEN, bool FP8 = false>
__global__ void __launch_bounds__(PairCfg<D, FP8>::kThreads, 1)
fa_fwd_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, FwdParams p) {
  using Cfg = PairCfg<D, FP8>;
  constexpr int BN = Cfg::BN, NS = Cfg::kSlots;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sQ = base;                                   // [2][kQBytes]
  unsigned char* sKV = base + 2 * Cfg::kQBytes;               // [NS][kSlotBytes]
  PairBarriers& bar = *reinterpret_cast<PairBarriers*>(sKV + NS * Cfg::kSlotBytes);
  volatile int* abortf = &bar.abort_flag;

  // warp index broadcast from lane 0, so the compiler knows it is warp-uniform
  // (required for the per-role register counts below)
  const int warp = __shfl_sync(0xffffffffu, (int)threadIdx.x / 32, 0), lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    bar.abort_flag = 0;
    for (int w = 0; w < 2; ++w) {
      mbar_init(&bar.q_full[w], 1);
      mbar_init(&bar.q_empty[w], 1);
      mbar_init(&bar.s_full[w], 1);
      mbar_init(&bar.p_full[w], 4);   // one arrival per warp of the softmax warpgroup
      mbar_init(&bar.o_full[w], 1);
      mbar_init(&bar.o_empty[w], 4);
    }
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

  // Every role walks the same sequence of items (pair_item) and keeps its own
  // running counts of the barrier phases it has seen, so the pipeline runs on
  // from one item into the next: the load warp fetches the next item's query
  // tiles as soon as the current item's S products no longer read them, the
  // MMA warp issues the next item's first S products right behind the current
  // item's last PV products, and a softmax warpgroup writes its output rows
  // while the next item's first scores are computed.
  // Each warpgroup sets its register count at the top of its own branch and
  // never re-joins the other branch (the final barrier is repeated in both).
  if (warp < 4) {
    reg_dealloc<Cfg::kRegsOther>();
    if (warp == 0) {
    // ------------------------------------------------------------ load warp
    // The whole warp runs the loop (waits are warp-wide); one elected lane
    // issues each TMA copy.
      const uint64_t pol_kv = l2_policy_evict_last();
      const uint64_t pol_q = l2_policy_evict_first();
      if (elect_one()) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
      }
      __syncwarp();
      int fill = 0, qc[2] = {0, 0};
      bool ok = true;
      PairItem it;
      SeqView sv;
      for (int k = 0; ok && pair_item<CAUSAL, VARLEN>(p, k, it, sv); ++k) {
        const int N = max(it.n0, it.n1);
        if (N == 0) continue;
        const int hkv = it.h / p.G;
        {
          // the next item's query tiles into L2 now, so that their loads
          // (issued once this item's last S products are done) are short
          PairItem nx;
          SeqView nsv;
          for (int kk = k + 1; pair_item<CAUSAL, VARLEN>(p, kk, nx, nsv); ++kk) {
            if (max(nx.n0, nx.n1) == 0) continue;
            if (elect_one())
              for (int w = 0; w < 2; ++w)
                if ((w ? nx.n1 : nx.n0) > 0)
                  for (int db = 0; db < Cfg::kDBlocks; ++db)
                    tma_prefetch_l2_4d(&tmQ, db * Cfg::kBlockCols, nx.h, nsv.q_row0 + nx.q0 + w * BM, nsv.tma_b);
            __syncwarp();
            break;
          }
        }
        // query tile w of this item, once the previous item's S products no
        // longer read its buffer
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          if ((w ? it.n1 : it.n0) == 0) continue;
          if (qc[w] > 0) ok = ok && __all_sync(0xffffffffu, mbar_wait(&bar.q_empty[w], (qc[w] - 1) & 1, abortf));
          if (!ok) break;
          if (elect_one()) {
            mbar_arrive_expect_tx(&bar.q_full[w], Cfg::kQBytes);
            for (int db = 0; db < Cfg::kDBlocks; ++db)
              tma_load_4d_hint(sQ + w * Cfg::kQBytes + db * Cfg::kQBlockBytes, &tmQ, &bar.q_full[w],
                               db * Cfg::kBlockCols, it.h, sv.q_row0 + it.q0 + w * BM, sv.tma_b, pol_q);
          }
          __syncwarp();
          ++qc[w];
        }
        for (int i = 0; i < 2 * N && ok; ++i, ++fill) {   // K_0, V_0, K_1, V_1, ...
          const int slot = fill % NS, round = fill / NS;
          if (round > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bar.kv_empty[slot], (round - 1) & 1, abortf));
          if (!ok) break;
          const CUtensorMap* tm = (i & 1) ? &tmV : &tmK;
          unsigned char* dst = sKV + slot * Cfg::kSlotBytes;
          if (elect_one()) {
            mbar_arrive_expect_tx(&bar.kv_full[slot], Cfg::kSlotBytes);
            for (int db = 0; db < Cfg::kDBlocks; ++db)
              tma_load_4d_hint(dst + db * Cfg::kKVBlockBytes, tm, &bar.kv_full[slot], db * Cfg::kBlockCols, hkv,
                               sv.k_row0 + (i >> 1) * BN, sv.tma_b, pol_kv);
          }
          __syncwarp();
        }
      }
      if (!ok) {
        // drain the copies still in flight before the CTA exits
        for (int w = 0; w < 2; ++w)
          if (qc[w] > 0) wait_drain(&bar.q_full[w], (qc[w] - 1) & 1);
        for (int i = (fill > NS ? fill - NS : 0); i < fill; ++i) wait_drain(&bar.kv_full[i % NS], (i / NS) & 1);
      }
    } else if (warp == 1) {
    // ------------------------------------------------------------ MMA warp
    // Issues every product.  An issue blocks while the tensor pipe is busy,
    // and mbarrier waits are slow while the tensor core streams its operands
    // from shared memory, so every wait but the one for P runs in the wait
    // warp during the previous group's products; the MMA warp takes the
    // hand-off (a named barrier) and then waits only for P.
    // The whole warp runs the loop, so every descriptor operand is
    // warp-uniform; one elected lane (always the same one) issues.
    // Descriptors are rebuilt per instruction from a constant high word and a
    // 32-bit low word (start address >> 4, leading offset >> 4).
    // Per item: the prologue issues S0_0 and S1_0; then per K/V tile j the
    // groups {PV0_j, S0_j+1} and {PV1_j, S1_j+1}.
      const uint32_t q_lo = smem_u32(sQ) >> 4;
      const uint32_t kv_lo = smem_u32(sKV) >> 4;
      int f0 = 0, c = 0, pc[2] = {0, 0};
      bool ok = true, failed = false;
      PairItem it;
      SeqView sv;
      for (int k = 0; ok && pair_item<CAUSAL, VARLEN>(p, k, it, sv); ++k) {
        const int n0 = it.n0, n1 = it.n1, N = max(n0, n1);
        if (N == 0) continue;
        ok = handoff_recv(bar, c++);
        if (!ok) break;
        tc_fence_after();
        if (!failed && elect_one()) {
          if (n0 > 0) {
            pair_mma_s<D, FP8>(tmem + Cfg::kS0, q_lo, kv_lo + (uint32_t)((f0 % NS) * Cfg::kSlotBytes >> 4));
            tc_commit(&bar.s_full[0]);
            if (n0 == 1) tc_commit(&bar.q_empty[0]);
          }
          if (n1 > 0) {
            pair_mma_s<D, FP8>(tmem + Cfg::kS1, q_lo + (uint32_t)(Cfg::kQBytes >> 4),
                               kv_lo + (uint32_t)((f0 % NS) * Cfg::kSlotBytes >> 4));
            tc_commit(&bar.s_full[1]);
            if (n1 == 1) tc_commit(&bar.q_empty[1]);
          }
          tc_commit(&bar.kv_empty[f0 % NS]);   // K_0
        }
        __syncwarp();
        for (int j = 0; j < N && ok; ++j) {
          if (j < n0) {
            ok = handoff_recv(bar, c++);
            if (ok && !failed) {
              failed = !__all_sync(0xffffffffu, mbar_wait(&bar.p_full[0], (pc[0] + j) & 1, abortf));
              if (!failed) {
                tc_fence_after();
                pair_group_issue<D, NS, 0, FP8>(bar, j, n0, n1, f0, tmem, q_lo, kv_lo);
              }
            }
          }
          if (ok && j < n1) {
            ok = handoff_recv(bar, c++);
            if (ok && !failed) {
              failed = !__all_sync(0xffffffffu, mbar_wait(&bar.p_full[1], (pc[1] + j) & 1, abortf));
              if (!failed) {
                tc_fence_after();
                pair_group_issue<D, NS, 1, FP8>(bar, j, n1, n1, f0, tmem, q_lo, kv_lo);
              }
            }
          }
        }
        pc[0] += n0;
        pc[1] += n1;
        f0 += 2 * N;
      }
      if (!ok || failed) {
        if (elect_one()) tc_commit(&bar.drain);
        __syncwarp();
        wait_drain(&bar.drain, 0);
      }
    } else if (warp == 2) {
    // ------------------------------------------------------------ wait warp
    // Walks the same items and groups as the MMA warp, one group ahead: waits
    // for the query and K/V tiles a group's products read and for the output
    // tile it overwrites, then hands the group to the MMA warp.
      int f0 = 0, c = 0, qf[2] = {0, 0}, oe[2] = {-1, -1};
      bool ok = true;
      PairItem it;
      SeqView sv;
      for (int k = 0; ok && pair_item<CAUSAL, VARLEN>(p, k, it, sv); ++k) {
        const int n0 = it.n0, n1 = it.n1, N = max(n0, n1);
        if (N == 0) continue;
        bool got = true;
        if (n0 > 0) got = mbar_wait(&bar.q_full[0], qf[0] & 1, abortf);
        if (n1 > 0) got = got && mbar_wait(&bar.q_full[1], qf[1] & 1, abortf);
        got = got && mbar_wait(&bar.kv_full[f0 % NS], (f0 / NS) & 1, abortf);
        ok = __all_sync(0xffffffffu, got) && !*abortf;
        handoff_send(bar, c++, ok);
        for (int j = 0; j < N && ok; ++j) {
          if (j < n0) {
            ok = pair_group_wait<D, NS, 0>(bar, j, n0, f0, oe[0], abortf);
            handoff_send(bar, c++, ok);
          }
          if (ok && j < n1) {
            ok = pair_group_wait<D, NS, 1>(bar, j, n1, f0, oe[1], abortf);
            handoff_send(bar, c++, ok);
          }
        }
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          const int nw = w ? n1 : n0;
          if (nw == 0) continue;
          ++qf[w];
          ++oe[w];   // the next item's first PV_w waits for this item's epilogue
        }
        f0 += 2 * N;
      }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
  } else {
    reg_alloc<Cfg::kRegsSoftmax>();
    // ------------------------------------------------------------ softmax warpgroups
    const int w = (warp - 4) / 4;                    // query tile of this warpgroup
    const int quarter = warp & 3;                    // tensor-memory lane quarter
    const int r = quarter * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    const uint32_t s_addr = tmem + lane_addr + (w ? Cfg::kS1 : Cfg::kS0);
    const uint32_t o_addr = tmem + lane_addr + (w ? Cfg::kO1 : Cfg::kO0);
    int sc = 0, oc = 0;   // s_full and o_full phases seen
    bool ok = true;
    PairItem it;
    SeqView sv;
    for (int k = 0; ok && pair_item<CAUSAL, VARLEN>(p, k, it, sv); ++k) {
      const int nw = w ? it.n1 : it.n0;
      const int h = it.h, b = it.b, hkv = h / p.G;
      const int qw0 = it.q0 + w * BM;
      const int qi = qw0 + r;
      const bool row_ok = row_in_range<VARLEN>(sv, p, qi);
      if (nw == 0) {
        if (VARLEN && row_ok && it.q0 >= 0) {
          __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) + ((sv.o_tok0 + qi) * p.Hq + h) * D;
          write_empty_row<D>(orow, p.lse ? p.lse + sv.lse0 + (int64_t)h * sv.lse_hs + qi : nullptr);
        }
        continue;
      }
      // e4m3 inputs: S and O carry the per-head dequantisation factors.
      const float sl2 = FP8 ? p.scale_log2 * __ldg(p.q_descale + (int64_t)b * p.Hq + h) *
                                  __ldg(p.k_descale + (int64_t)b * p.Hkv + hkv)
                            : p.scale_log2;
      int key_limit = sv.Lk - 1;
      if (CAUSAL) key_limit = min(key_limit, qi + sv.causal_off);

      // A tcgen05.commit signals once every MMA the issuing thread issued before
      // it is complete, and PV_w,j-1 is issued before S_w,j: so once S_w,j is
      // seen, O_w holds PV_w,j-1 and may be rescaled without a further wait.
      RowState st;
      for (int j = 0; j < nw && ok; ++j, ++sc) {
        // S_w,j is on the warpgroup's critical path: poll for it rather than
        // suspend (measured: 0.98 of the time, causal; bidirectional unchanged)
        ok = mbar_wait_spin(&bar.s_full[w], sc & 1, abortf);
        if (!ok) break;
        tc_fence_after();
        float s[BN];
        load_row(s_addr, s);
        const int key0 = j * BN;
        const bool need_mask = (key0 + BN > sv.Lk) || (CAUSAL && key0 + BN - 1 > qw0 + sv.causal_off);
        if (need_mask) {
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (key0 + c > key_limit) s[c] = -INFINITY;
        }
        const float mx = row_max(s);
        const float t_max = (mx == -INFINITY) ? -INFINITY : mx * sl2;
        bool rescale;
        const float alpha = update_max(st, t_max, rescale, Cfg::kThreshold);
        const float m_use = ((st.m == -INFINITY) ? 0.f : st.m) - Cfg::kPExp;
        // P_w,j goes over S_w,j.  The previous P_w in these columns was read by
        // PV_w,j-1, which completed before S_w,j did (issue order).
        float rowsum;
        if constexpr (FP8)
          rowsum = need_mask ? exp_store_row_e4m3<BN, true>(s, sl2, m_use, s_addr + Cfg::kPOff, key0, key_limit)
                             : exp_store_row_e4m3<BN, false>(s, sl2, m_use, s_addr + Cfg::kPOff, key0, key_limit);
        else
          rowsum = need_mask ? exp_store_row<BN, true>(s, sl2, m_use, s_addr + Cfg::kPOff, key0, key_limit)
                             : exp_store_row<BN, false>(s, sl2, m_use, s_addr + Cfg::kPOff, key0, key_limit);
        if (__any_sync(0xffffffffu, rescale) && j >= 1) rescale_o<D>(o_addr, rescale ? alpha : 1.f);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar.p_full[w]);
        st.l = st.l * alpha + rowsum;
      }
      if (!ok) break;
      ok = mbar_wait(&bar.o_full[w], oc & 1, abortf);
      ++oc;
      if (!ok) break;
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) + ((sv.o_tok0 + qi) * p.Hq + h) * D;
      float* lse_ptr = p.lse ? p.lse + sv.lse0 + (int64_t)h * sv.lse_hs + qi : nullptr;
      tc_fence_after();
      if constexpr (FP8)
        epilogue_row<D>(o_addr, st.m - Cfg::kPExp, st.l, row_ok, orow, lse_ptr,
                        __ldg(p.v_descale + (int64_t)b * p.Hkv + hkv));
      else
        epilogue_row<D>(o_addr, st.m, st.l, row_ok, orow, lse_ptr);
      // O_w has been read (epilogue_row waits for its tensor-memory loads):
      // the next item's first PV_w may overwrite it.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.o_empty[w]);
    }
    tc_fence_before();
    __syncthreads();
  }
}

// ===========================================================================
// Single kernel: head_dim 256, one query tile per CTA, 64-key K/V tiles.
// ===========================================================================
template <int D, int BN, bool FP8 = false>
struct SingleCfg {
  static constexpr int kBlockCols = FP8 ? 128 : 64;   // columns per 128-byte row
  static constexpr int kDBlocks = D / kBlockCols;
  static constexpr int kRowBytes = FP8 ? D : 2 * D;
  static constexpr int kQBlockBytes = BM * 128;
  static constexpr int kKVBlockBytes = BN * 128;
  static constexpr int kSlotBytes = kDBlocks * kKVBlockBytes;
  static constexpr int kQBytes = kDBlocks * kQBlockBytes;
  static constexpr int kSlots = FP8 ? 8 : 4;
  // as PairCfg: reference-max slack and the e4m3 P exponent offset
  static constexpr float kThreshold = FP8 ? 2.f : kRescaleThreshold;
  static constexpr float kPExp = FP8 ? 6.f : 0.f;
  static constexpr int kThreads = 192;   // load, MMA, 4 softmax warps
  static constexpr int kSCol0 = 0;       // S0, S1 at 0, BN
  static constexpr int kPCol0 = 2 * BN;  // P0, P1 at 2BN, 2BN + BN/2
  static constexpr int kOCol = 256;
  static constexpr int kSmemBytes = kQBytes + kSlots * kSlotBytes + 1024 + 1024;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static_assert(3 * BN <= 256 && kOCol + D <= 512, "tensor-memory budget");
};

struct SingleBarriers {
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

template <int D, int BN, bool CAUSAL, bool VARLEN, bool FP8 = false>
__global__ void __launch_bounds__(SingleCfg<D, BN, FP8>::kThreads, 1)
fa_fwd_single_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, FwdParams p) {
  using Cfg = SingleCfg<D, BN, FP8>;
  constexpr int NS = Cfg::kSlots;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sQ = base;
  unsigned char* sKV = base + Cfg::kQBytes;
  SingleBarriers& bar = *reinterpret_cast<SingleBarriers*>(sKV + NS * Cfg::kSlotBytes);
  volatile int* abortf = &bar.abort_flag;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int h = blockIdx.y, b = blockIdx.z, hkv = h / p.G;
  const SeqView sv = seq_view<VARLEN>(p, b);
  const int n_tiles = VARLEN ? (sv.Lq + BM - 1) / BM : p.n_qtiles;
  if ((int)blockIdx.x >= n_tiles) return;          // past this sequence's queries (whole CTA)
  const int q_tile = n_tiles - 1 - blockIdx.x;
  const int q0 = q_tile * BM;
  const int n_kv = kv_tiles(q0, sv.Lq, sv.Lk, sv.causal_off, BN, CAUSAL);

  if (threadIdx.x == 0) {
    bar.abort_flag = 0;
    mbar_init(&bar.q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar.s_full[i], 1);
      mbar_init(&bar.p_full[i], 4);
      mbar_init(&bar.pv_done[i], 1);
    }
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
    // load warp: warp-wide waits, one elected lane issues the copies
    const uint64_t pol_kv = l2_policy_evict_last();
    const uint64_t pol_q = l2_policy_evict_first();
    if (elect_one()) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(&bar.q_full, Cfg::kQBytes);
      for (int db = 0; db < Cfg::kDBlocks; ++db)
        tma_load_4d_hint(sQ + db * Cfg::kQBlockBytes, &tmQ, &bar.q_full, db * Cfg::kBlockCols, h, sv.q_row0 + q0,
                         sv.tma_b, pol_q);
    }
    __syncwarp();
    int issued = 0;
    bool ok = true;
    for (int i = 0; i < 2 * n_kv && ok; ++i) {
      const int slot = i % NS, round = i / NS;
      if (round > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bar.kv_empty[slot], (round - 1) & 1, abortf));
      if (!ok) break;
      const CUtensorMap* tm = (i & 1) ? &tmV : &tmK;
      unsigned char* dst = sKV + slot * Cfg::kSlotBytes;
      if (elect_one()) {
        mbar_arrive_expect_tx(&bar.kv_full[slot], Cfg::kSlotBytes);
        for (int db = 0; db < Cfg::kDBlocks; ++db)
          tma_load_4d_hint(dst + db * Cfg::kKVBlockBytes, tm, &bar.kv_full[slot], db * Cfg::kBlockCols, hkv,
                           sv.k_row0 + (i >> 1) * BN, sv.tma_b, pol_kv);
      }
      __syncwarp();
      ++issued;
    }
    if (!ok) {
      wait_drain(&bar.q_full, 0);
      for (int i = (issued > NS ? issued - NS : 0); i < issued; ++i) wait_drain(&bar.kv_full[i % NS], (i / NS) & 1);
    }
  } else if (warp == 1) {
    // MMA warp: warp-wide waits, one elected lane (always the same) issues
    constexpr uint32_t idS = FP8 ? idesc_e4m3_f32(BM, BN, 0, 0) : idesc_bf16_f32(BM, BN, 0, 0);
    constexpr uint32_t idPV = FP8 ? idesc_e4m3_f32(BM, D, 0, 1) : idesc_bf16_f32(BM, D, 0, 1);
    constexpr int KK = FP8 ? 32 : 16;   // keys (contraction) per PV instruction
    const uint64_t descQ = smem_desc_sw128(smem_u32(sQ), 16, 1024);
    const uint64_t descK = smem_desc_sw128(smem_u32(sKV), 16, 1024);
    const uint64_t descV = smem_desc_sw128(smem_u32(sKV), Cfg::kKVBlockBytes, 1024);
    bool ok = __all_sync(0xffffffffu, mbar_wait(&bar.q_full, 0, abortf));
    auto issue_pv = [&](int t) -> bool {
      const int i = 2 * t + 1, slot = i % NS;
      bool got = mbar_wait(&bar.p_full[t & 1], (t >> 1) & 1, abortf);
      got = got && mbar_wait(&bar.kv_full[slot], (i / NS) & 1, abortf);
      if (!__all_sync(0xffffffffu, got)) return false;
      tc_fence_after();
      const uint64_t dv = descV + ((uint64_t)(slot * Cfg::kSlotBytes) >> 4);
      const uint32_t pcol = tmem + Cfg::kPCol0 + (t & 1) * (BN / 2);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < BN / KK; ++kk) {
          const uint64_t bd = dv + ((uint64_t)(kk * KK * 128) >> 4);
          if (FP8)
            mma_f8_ts(tmem + Cfg::kOCol, pcol + kk * 8, bd, idPV, (t > 0 || kk > 0) ? 1u : 0u);
          else
            mma_bf16_ts(tmem + Cfg::kOCol, pcol + kk * 8, bd, idPV, (t > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&bar.kv_empty[slot]);
        tc_commit(&bar.pv_done[t & 1]);
      }
      __syncwarp();
      return true;
    };
    for (int j = 0; j < n_kv && ok; ++j) {
      const int i = 2 * j, slot = i % NS;
      ok = __all_sync(0xffffffffu, mbar_wait(&bar.kv_full[slot], (i / NS) & 1, abortf));
      if (!ok) break;
      tc_fence_after();
      const uint64_t dk = descK + ((uint64_t)(slot * Cfg::kSlotBytes) >> 4);
      const uint32_t scol = tmem + Cfg::kSCol0 + (j & 1) * BN;
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < Cfg::kRowBytes / 32; ++kk) {   // 32 bytes of the contraction each
          const uint32_t offq = (kk >> 2) * Cfg::kQBlockBytes + (kk & 3) * 32;
          const uint32_t offk = (kk >> 2) * Cfg::kKVBlockBytes + (kk & 3) * 32;
          if (FP8)
            mma_f8_ss(scol, descQ + (offq >> 4), dk + (offk >> 4), idS, kk > 0 ? 1u : 0u);
          else
            mma_bf16_ss(scol, descQ + (offq >> 4), dk + (offk >> 4), idS, kk > 0 ? 1u : 0u);
        }
        tc_commit(&bar.s_full[j & 1]);
        tc_commit(&bar.kv_empty[slot]);
      }
      __syncwarp();
      if (j >= 1) ok = issue_pv(j - 1);
    }
    if (ok && n_kv > 0) ok = issue_pv(n_kv - 1);
    if (!ok) {
      if (elect_one()) tc_commit(&bar.drain);
      __syncwarp();
      wait_drain(&bar.drain, 0);
    }
  } else {
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int qi = q0 + r;
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    const float sl2 = FP8 ? p.scale_log2 * __ldg(p.q_descale + (int64_t)b * p.Hq + h) *
                                __ldg(p.k_descale + (int64_t)b * p.Hkv + hkv)
                          : p.scale_log2;
    int key_limit = sv.Lk - 1;
    if (CAUSAL) key_limit = min(key_limit, qi + sv.causal_off);

    RowState st;
    int pv_seen = 0;
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
      load_row(tmem + lane_addr + Cfg::kSCol0 + (j & 1) * BN, s);
      const int key0 = j * BN;
      const bool need_mask = (key0 + BN > sv.Lk) || (CAUSAL && key0 + BN - 1 > q0 + sv.causal_off);
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (key0 + c > key_limit) s[c] = -INFINITY;
      }
      const float mx = row_max(s);
      const float t_max = (mx == -INFINITY) ? -INFINITY : mx * sl2;
      bool rescale;
      const float alpha = update_max(st, t_max, rescale, Cfg::kThreshold);
      const float m_use = ((st.m == -INFINITY) ? 0.f : st.m) - Cfg::kPExp;
      if (j >= 2) ok = wait_pv(j - 2);   // P_j reuses the columns PV_{j-2} read
      if (!ok) break;
      const uint32_t pcol = tmem + lane_addr + Cfg::kPCol0 + (j & 1) * (BN / 2);
      float rowsum;
      if constexpr (FP8)
        rowsum = need_mask ? exp_store_row_e4m3<BN, true>(s, sl2, m_use, pcol, key0, key_limit)
                           : exp_store_row_e4m3<BN, false>(s, sl2, m_use, pcol, key0, key_limit);
      else
        rowsum = need_mask ? exp_store_row<BN, true>(s, sl2, m_use, pcol, key0, key_limit)
                           : exp_store_row<BN, false>(s, sl2, m_use, pcol, key0, key_limit);
      if (__any_sync(0xffffffffu, rescale) && j >= 1) {
        ok = wait_pv(j - 1);
        if (!ok) break;
        tc_fence_after();
        rescale_o<D>(tmem + lane_addr + Cfg::kOCol, rescale ? alpha : 1.f);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.p_full[j & 1]);
      st.l = st.l * alpha + rowsum;
    }
    if (ok && n_kv > 0) ok = wait_pv(n_kv - 1);
    if (ok) {
      const bool row_ok = row_in_range<VARLEN>(sv, p, qi);
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) + ((sv.o_tok0 + qi) * p.Hq + h) * D;
      float* lse_ptr = p.lse ? p.lse + sv.lse0 + (int64_t)h * sv.lse_hs + qi : nullptr;
      if (n_kv > 0) {
        tc_fence_after();
        if constexpr (FP8)
          epilogue_row<D>(tmem + lane_addr + Cfg::kOCol, st.m - Cfg::kPExp, st.l, row_ok, orow, lse_ptr,
                          __ldg(p.v_descale + (int64_t)b * p.Hkv + hkv));
        else
          epilogue_row<D>(tmem + lane_addr + Cfg::kOCol, st.m, st.l, row_ok, orow, lse_ptr);
      } else if (VARLEN && row_ok) {
        write_empty_row<D>(orow, lse_ptr);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  return n;
}

template <int D, bool CAUSAL, bool VARLEN, bool FP8 = false>
cudaError_t launch_pair(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, FwdParams p,
                        cudaStream_t stream) {
  using Cfg = PairCfg<D, FP8>;
  auto kern = fa_fwd_pair_kernel<D, CAUSAL, VARLEN, FP8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
  if (e != cudaSuccess) return e;
  // pairs of query tiles (for a packed batch: of the longest sequence, p.Lq)
  p.n_qtiles = (p.Lq + 2 * BM - 1) / (2 * BM);
  // Persistent CTAs (one per SM) once every SM gets a couple of items or
  // more; otherwise one CTA per item and the block scheduler balances.
  const long long couples = (long long)((p.n_qtiles + 1) / 2) * p.Hq * p.B;
  const int sms = sm_count();
  p.sched = (!VARLEN && sms > 0 && couples >= 2LL * sms) ? 1 : 0;
  if (p.sched)
    kern<<<sms, Cfg::kThreads, Cfg::kSmemBytes, stream>>>(q, k, v, p);
  else
    kern<<<dim3(p.n_qtiles, p.Hq, p.B), Cfg::kThreads, Cfg::kSmemBytes, stream>>>(q, k, v, p);
  return cudaGetLastError();
}

template <int D, int BN, bool CAUSAL, bool VARLEN, bool FP8 = false>
cudaError_t launch_single(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, FwdParams p,
                          cudaStream_t stream) {
  using Cfg = SingleCfg<D, BN, FP8>;
  auto kern = fa_fwd_single_kernel<D, BN, CAUSAL, VARLEN, FP8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
  if (e != cudaSuccess) return e;
  p.n_qtiles = (p.Lq + BM - 1) / BM;
  kern<<<dim3(p.n_qtiles, p.Hq, p.B), Cfg::kThreads, Cfg::kSmemBytes, stream>>>(q, k, v, p);
  return cudaGetLastError();
}

template <bool VARLEN>
cudaError_t launch_fwd(int D, bool causal, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                       const FwdParams& p, cudaStream_t stream) {
  switch (D) {
    case 64:
      return causal ? launch_pair<64, true, VARLEN>(q, k, v, p, stream)
                    : launch_pair<64, false, VARLEN>(q, k, v, p, stream);
    case 128:
      return causal ? launch_pair<128, true, VARLEN>(q, k, v, p, stream)
                    : launch_pair<128, false, VARLEN>(q, k, v, p, stream);
    case 256:
      return causal ? launch_single<256, 64, true, VARLEN>(q, k, v, p, stream)
                    : launch_single<256, 64, false, VARLEN>(q, k, v, p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

int fwd_block_n(int D) { return D == 256 ? 64 : 128; }

cudaError_t launch_fa_fwd(int D, bool causal, bool varlen, const CUtensorMap& q, const CUtensorMap& k,
                          const CUtensorMap& v, const FwdParams& p, cudaStream_t stream) {
  return varlen ? launch_fwd<true>(D, causal, q, k, v, p, stream) : launch_fwd<false>(D, causal, q, k, v, p, stream);
}

cudaError_t launch_fa_fwd_fp8(int D, bool causal, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                              const FwdParams& p, cudaStream_t stream) {
  switch (D) {
    case 64:
      return causal ? launch_pair<64, true, false, true>(q, k, v, p, stream)
                    : launch_pair<64, false, false, true>(q, k, v, p, stream);
    case 128:
      return causal ? launch_pair<128, true, false, true>(q, k, v, p, stream)
                    : launch_pair<128, false, false, true>(q, k, v, p, stream);
    case 256:
      return causal ? launch_single<256, 64, true, false, true>(q, k, v, p, stream)
                    : launch_single<256, 64, false, false, true>(q, k, v, p, stream);
    default: return cudaErrorInvalidValue;
  }
}

// Self-test of the bounded waits: one warp waits on an mbarrier that nothing
// arrives on.  The first wait gives up after limit_ns, records the timeout in
// the status word and sets the block's abort flag; the second returns at once
// because of that flag.  Nothing else is in flight, so the kernel just exits.
__global__ void __launch_bounds__(32, 1) wait_selftest_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  const bool first = mbar_wait(&bar, 0, &abort_flag, limit_ns);
  const bool second = mbar_wait(&bar, 0, &abort_flag, limit_ns);
  if (first || second) atomicOr(&g_device_status, 2u);   // cannot happen: nothing completes the phase
}

cudaError_t launch_wait_selftest(unsigned long long limit_ns, cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(limit_ns);
  return cudaGetLastError();
}

unsigned int fwd_read_and_clear_status() {
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof v) != cudaSuccess) return 0xFFFFFFFFu;
  cudaMemcpyToSymbol(g_device_status, &zero, sizeof zero);
  return v;
}

}  // namespace ta23
