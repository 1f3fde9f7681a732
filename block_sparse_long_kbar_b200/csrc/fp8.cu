// FP8 storage of the KV cache (mo.ai.kr, "Step 5 Preview agentic work design", section
// "long-horizon RL and run cost": the KV cache is trained for FP8 storage). Format read from the
// pages' statement: every (token, group) row of K or V holds its d values as FP8 E4M3 codes and
// one power-of-two scale s = 2^e, e the smallest integer with max |x| <= 448 s (448 is E4M3's
// largest finite value); a code is the E4M3 rounding (to nearest, ties to even) of x / s. A
// dequantized value code * s has at most 4 significant bits, so it is exact in bf16 and the
// attention kernels multiply it back in without error.
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace sgqa {
namespace {

// e of the row scale from the bits of max |x| (a non-negative float): amax = m 2^E with m in
// [1, 2) and 448 = 1.75 2^8, so e = E - 8, plus one when m > 1.75 (mantissa field above 0x600000).
__device__ __forceinline__ int scale_exponent(uint32_t amax_bits) {
  if (amax_bits == 0u) return 0;
  int E = (int)(amax_bits >> 23) - 127;
  uint32_t mant = amax_bits & 0x7FFFFFu;
  if ((amax_bits >> 23) == 0u) {  // subnormal: normalise
    const int p = 31 - __clz((int)mant);
    E = p - 149;
    mant = (mant << (23 - p)) & 0x7FFFFFu;
  }
  return E - 8 + (mant > 0x600000u ? 1 : 0);
}

// One warp per (token, group) row of 128 values (four per lane).
__global__ void __launch_bounds__(256) quantize_fp8_kernel(const uint16_t* __restrict__ src, uint8_t* __restrict__ dst8,
                                                           float* __restrict__ dscale, int batch, int n_t, int G,
                                                           int T, int t0) {
  const long w = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long nrows = (long)batch * n_t * G;
  if (w >= nrows) return;  // warp-uniform
  const long per_seq = (long)n_t * G;
  const long b = w / per_seq, rem = w % per_seq;
  const long dst_row = (b * T + t0) * G + rem;  // rows (t, g) are contiguous in both layouts
  const uint2 v = reinterpret_cast<const uint2*>(src + w * 128)[lane];
  const float x[4] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y)};
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) m = max(m, __float_as_uint(fabsf(x[i])));
  m = __reduce_max_sync(0xFFFFFFFFu, m);  // non-negative floats order like their bits
  const int e = scale_exponent(m);
  uint32_t packed = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_fp8_storage_t c = __nv_cvt_float_to_fp8(ldexpf(x[i], -e), __NV_SATFINITE, __NV_E4M3);
    packed |= (uint32_t)c << (8 * i);
  }
  reinterpret_cast<uint32_t*>(dst8 + dst_row * 128)[lane] = packed;
  if (lane == 0) dscale[dst_row] = ldexpf(1.f, e);
}

}  // namespace

cudaError_t launch_quantize_fp8(const uint16_t* src, uint8_t* dst8, float* dscale, int batch, int n_t, int G, int T,
                                int t0, cudaStream_t s) {
  const long rows = (long)batch * n_t * G;
  if (rows <= 0) return cudaSuccess;
  const long threads = rows * 32;
  quantize_fp8_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(src, dst8, dscale, batch, n_t, G, T, t0);
  return cudaGetLastError();
}

}  // namespace sgqa
