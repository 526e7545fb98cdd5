// Per-head e4m3 quantisation of a bf16 tensor [B, L, H, D] for the FP8
// attention forward (FlashAttention-3's FP8 path, "FlashAttention-2 (TH)"
// section on later versions: e4m3 operands with per-head dequantisation
// factors).
//
// For each (b, h):  amax = max |x| over the L x D slice,
//                   inv = 448 / amax (fp32, round to nearest),
//                   code = e4m3(x * inv) (fp32 product, round to nearest even,
//                          saturating at +-448),
//                   descale = amax / 448,
// so that x ~ code * descale and the largest |x| of the slice maps to 448.
// A slice with amax < 2^-110 (all zero, or so small that 448 / amax could
// leave the fp32 range) takes inv = descale = 1: its codes are e4m3(x), +-0.
//
// Three launches: an HBM-bound amax pass (row blocks, atomicMax on the fp32
// bit pattern, which orders like the value for non-negative floats), the
// quantising pass, and a [B, H] finalise that turns amax into descale.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cstdint>

#include "fa_kernels.h"

namespace ta23 {
namespace {

constexpr int kThreads = 256;
constexpr int kRowsPerBlock = 64;
constexpr float kTinyAmax = 0x1p-110f;   // below it: inv = descale = 1

// Thread t of the block handles 8 consecutive elements (16 bytes) of row
// r = t / (D / 8) in each pass over kThreads / (D / 8) rows.
template <int D>
__global__ void __launch_bounds__(kThreads) amax_kernel(const __nv_bfloat16* __restrict__ x, float* amax, int L,
                                                        int H) {
  constexpr int kPerRow = D / 8, kRowsPerPass = kThreads / kPerRow;
  const int h = blockIdx.y, b = blockIdx.z;
  const int r0 = blockIdx.x * kRowsPerBlock;
  const int sub = threadIdx.x % kPerRow, rr = threadIdx.x / kPerRow;
  float m = 0.f;
  for (int r = r0 + rr; r < min(r0 + kRowsPerBlock, L); r += kRowsPerPass) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(x + (((int64_t)b * L + r) * H + h) * D) + sub);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
      m = fmaxf(m, fmaxf(fabsf(__low2float(v)), fabsf(__high2float(v))));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float wmax[kThreads / 32];
  if (threadIdx.x % 32 == 0) wmax[threadIdx.x / 32] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = wmax[0];
#pragma unroll
    for (int i = 1; i < kThreads / 32; ++i) t = fmaxf(t, wmax[i]);
    atomicMax(reinterpret_cast<unsigned int*>(amax) + (int64_t)b * H + h, __float_as_uint(t));
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads) quantize_kernel(const __nv_bfloat16* __restrict__ x,
                                                            const float* __restrict__ amax, uint8_t* __restrict__ out,
                                                            int L, int H) {
  constexpr int kPerRow = D / 8, kRowsPerPass = kThreads / kPerRow;
  const int h = blockIdx.y, b = blockIdx.z;
  const int r0 = blockIdx.x * kRowsPerBlock;
  const int sub = threadIdx.x % kPerRow, rr = threadIdx.x / kPerRow;
  const float a = __ldg(amax + (int64_t)b * H + h);
  const float inv = a >= kTinyAmax ? __fdiv_rn(448.f, a) : 1.f;
  for (int r = r0 + rr; r < min(r0 + kRowsPerBlock, L); r += kRowsPerPass) {
    const int64_t e0 = (((int64_t)b * L + r) * H + h) * D;
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(x + e0) + sub);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    uint32_t q[2];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
      const float2 y = make_float2(__fmul_rn(__low2float(v), inv), __fmul_rn(__high2float(v), inv));
      const uint32_t two = __nv_cvt_float2_to_fp8x2(y, __NV_SATFINITE, __NV_E4M3);
      if (i & 1)
        q[i / 2] |= two << 16;
      else
        q[i / 2] = two;
    }
    *reinterpret_cast<uint2*>(out + e0 + sub * 8) = make_uint2(q[0], q[1]);
  }
}

__global__ void finalize_kernel(float* amax_to_descale, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    const float a = amax_to_descale[i];
    amax_to_descale[i] = a >= kTinyAmax ? __fdiv_rn(a, 448.f) : 1.f;
  }
}

template <int D>
cudaError_t launch_t(const void* x, void* out, float* descale, int B, int L, int H, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(descale, 0, sizeof(float) * (size_t)B * H, s);
  if (e != cudaSuccess) return e;
  const dim3 grid((L + kRowsPerBlock - 1) / kRowsPerBlock, H, B);
  amax_kernel<D><<<grid, kThreads, 0, s>>>(static_cast<const __nv_bfloat16*>(x), descale, L, H);
  quantize_kernel<D><<<grid, kThreads, 0, s>>>(static_cast<const __nv_bfloat16*>(x), descale,
                                               static_cast<uint8_t*>(out), L, H);
  finalize_kernel<<<(B * H + 255) / 256, 256, 0, s>>>(descale, B * H);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize_fp8(int D, const void* x, void* out, float* descale, int B, int L, int H,
                                cudaStream_t stream) {
  switch (D) {
    case 64: return launch_t<64>(x, out, descale, B, L, H, stream);
    case 128: return launch_t<128>(x, out, descale, B, L, H, stream);
    case 256: return launch_t<256>(x, out, descale, B, L, H, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace ta23
