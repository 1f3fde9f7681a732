// K1: block-mean compression of the shared index keys (Step 5 Preview pages: mo.ai.kr,
// "Step 5 Preview agentic work design", section "model structure and training stability" —
// shared index keys are compressed per block of B = 8 tokens; the compression is read as the
// mean of the block's keys).
//
// One thread per (sequence, block, 8-wide column chunk): B coalesced 16-byte loads, the sum
// taken in fp64 in token order (exact unless a block's keys span more than 2^40 in magnitude:
// at most 16 terms of 8 significant bits), one multiply by 1/B (a power of two, exact), then
// one RNE rounding to fp32. kbar is therefore the correctly rounded block mean. The same
// thread also writes the bf16 hi/lo split of kbar that the tensor-core indexer consumes
// (hi = bf16(kbar), lo = bf16(kbar - hi); kbar - hi is exact in fp32).
#include "common.cuh"
#include "kernels.h"

namespace sgqa {
namespace {

__global__ void __launch_bounds__(256) compress_kernel(const uint16_t* __restrict__ k_idx, float* __restrict__ kbar,
                                                       uint16_t* __restrict__ hi, uint16_t* __restrict__ lo,
                                                       int batch, int T, int d_idx, int B, int j0, int nj) {
  const int chunks = d_idx / 8;
  const long total = (long)batch * nj * chunks;
  const long e = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= total) return;
  const int c = (int)(e % chunks);
  const long bj = e / chunks;
  const int j = j0 + (int)(bj % nj);
  const long b = bj / nj;
  const int nblk = T / B;
  double acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.0;
  const uint16_t* src = k_idx + ((b * T) + (long)j * B) * d_idx + c * 8;
  for (int r = 0; r < B; ++r) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(src + (long)r * d_idx));
    const uint32_t p[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] += (double)bf16_lo(p[i]);
      acc[2 * i + 1] += (double)bf16_hi(p[i]);
    }
  }
  const double inv = 1.0 / (double)B;
  float m[8];
  uint16_t h[8], l[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    m[i] = __double2float_rn(acc[i] * inv);
    h[i] = f32_to_bf16_rne(m[i]);
    l[i] = f32_to_bf16_rne(m[i] - bf16_to_f32(h[i]));
  }
  const long o = ((b * nblk) + j) * (long)d_idx + c * 8;
  float4* kd = reinterpret_cast<float4*>(kbar + o);
  kd[0] = make_float4(m[0], m[1], m[2], m[3]);
  kd[1] = make_float4(m[4], m[5], m[6], m[7]);
  if (hi) {
    uint4 hv, lv;
    hv.x = h[0] | ((uint32_t)h[1] << 16); hv.y = h[2] | ((uint32_t)h[3] << 16);
    hv.z = h[4] | ((uint32_t)h[5] << 16); hv.w = h[6] | ((uint32_t)h[7] << 16);
    lv.x = l[0] | ((uint32_t)l[1] << 16); lv.y = l[2] | ((uint32_t)l[3] << 16);
    lv.z = l[4] | ((uint32_t)l[5] << 16); lv.w = l[6] | ((uint32_t)l[7] << 16);
    *reinterpret_cast<uint4*>(hi + o) = hv;
    *reinterpret_cast<uint4*>(lo + o) = lv;
  }
}

__global__ void __launch_bounds__(256) split_planes_kernel(const float* __restrict__ kbar, uint16_t* __restrict__ hi,
                                                           uint16_t* __restrict__ lo, long n4) {
  const long e = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n4) return;
  const float4 v = reinterpret_cast<const float4*>(kbar)[e];
  const float x[4] = {v.x, v.y, v.z, v.w};
  uint16_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    h[i] = f32_to_bf16_rne(x[i]);
    l[i] = f32_to_bf16_rne(x[i] - bf16_to_f32(h[i]));
  }
  reinterpret_cast<uint2*>(hi)[e] = make_uint2(h[0] | ((uint32_t)h[1] << 16), h[2] | ((uint32_t)h[3] << 16));
  reinterpret_cast<uint2*>(lo)[e] = make_uint2(l[0] | ((uint32_t)l[1] << 16), l[2] | ((uint32_t)l[3] << 16));
}

}  // namespace

cudaError_t launch_compress(const uint16_t* k_idx, float* kbar, uint16_t* hi, uint16_t* lo, int batch, int T,
                            int d_idx, int B, int j0, int j1, cudaStream_t s) {
  const int nj = j1 - j0;
  if (nj <= 0) return cudaSuccess;
  const long total = (long)batch * nj * (d_idx / 8);
  const unsigned grid = (unsigned)((total + 255) / 256);
  compress_kernel<<<grid, 256, 0, s>>>(k_idx, kbar, hi, lo, batch, T, d_idx, B, j0, nj);
  return cudaGetLastError();
}

cudaError_t launch_split_planes(const float* kbar, uint16_t* hi, uint16_t* lo, long n, cudaStream_t s) {
  const long n4 = n / 4;
  if (n4 <= 0) return cudaSuccess;
  split_planes_kernel<<<(unsigned)((n4 + 255) / 256), 256, 0, s>>>(kbar, hi, lo, n4);
  return cudaGetLastError();
}

}  // namespace sgqa
