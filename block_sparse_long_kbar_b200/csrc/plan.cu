// Query scheduling for the tiled gather attention: group queries whose selections overlap.
//
// The Step 5 Preview pages (mo.ai.kr, "Step 5 Preview agentic work design", section "model
// structure and training stability") note that adjacent tokens select largely the same blocks
// and that batching them raises GPU utilisation. This step generalises "adjacent": within each
// (sequence, KV group) the query rows are ordered by a MinHash signature of their selected
// blocks (own block excluded), ties kept in token order, so that rows with the same or similar
// selections land in the same attention tile and share every K/V block load. The order is a
// pure function of the selection (a stable sort), so results are run-to-run identical.
//
//   signature_kernel: one warp per row; sig = min over selected j != own of mix32(j); the sort
//                     key is its top 24 bits.
//   radix passes:     stable LSD radix sort of (key, row) per segment, 8 bits per pass:
//                     per-CTA digit histograms, a per-segment scan, and a scatter that ranks
//                     equal digits in input order with warp match + per-warp prefix counts.
#include "common.cuh"
#include "kernels.h"

namespace sgqa {
namespace {

constexpr int kSortTile = 2048;
constexpr int kSortThreads = 256;
constexpr int kKeyBits = 24;

__device__ __forceinline__ uint32_t mix32(uint32_t x) {
  x ^= x >> 16;
  x *= 0x7FEB352Du;
  x ^= x >> 15;
  x *= 0x846CA68Bu;
  x ^= x >> 16;
  return x;
}

__global__ void __launch_bounds__(256) signature_kernel(const int32_t* __restrict__ sel, int sel_T, int sel_t0, int G,
                                                        int Kb, int B, int t_begin, int n, int n_seg,
                                                        uint32_t* __restrict__ keys, uint32_t* __restrict__ vals) {
  const int lane = threadIdx.x & 31;
  const long u = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (u >= (long)n * n_seg) return;
  const int seg = (int)(u / n), i = (int)(u % n);
  const int b = seg / G, g = seg % G;
  const int t = t_begin + i;
  const int c = t / B;
  const int32_t* row = sel + (((long)b * sel_T + (t - sel_t0)) * G + g) * (long)Kb;
  uint32_t h = 0xFFFFFFFFu;
  for (int e = lane; e < Kb; e += 32) {
    const int j = __ldg(row + e);
    if (j >= 0 && j != c) h = min(h, mix32((uint32_t)j));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) h = min(h, __shfl_xor_sync(0xFFFFFFFFu, h, o));
  if (lane == 0) {
    keys[u] = h >> (32 - kKeyBits);
    vals[u] = (uint32_t)i;
  }
}

__global__ void __launch_bounds__(kSortThreads) radix_hist_kernel(const uint32_t* __restrict__ keys, int n, int shift,
                                                                  int n_cta, uint32_t* __restrict__ hist) {
  __shared__ uint32_t h[256];
  const int seg = blockIdx.y, cta = blockIdx.x;
  h[threadIdx.x] = 0;
  __syncthreads();
  const uint32_t* k = keys + (long)seg * n;
  const int e0 = cta * kSortTile, e1 = min(n, e0 + kSortTile);
  for (int e = e0 + threadIdx.x; e < e1; e += kSortThreads) atomicAdd(&h[(k[e] >> shift) & 255u], 1u);
  __syncthreads();
  hist[((long)seg * 256 + threadIdx.x) * n_cta + cta] = h[threadIdx.x];
}

// exclusive scan of one segment's 256 * n_cta counts (digit-major), in place
__global__ void __launch_bounds__(1024) radix_scan_kernel(uint32_t* __restrict__ hist, int n_cta) {
  __shared__ uint32_t warp_sums[32];
  const int L = 256 * n_cta;
  uint32_t* h = hist + (long)blockIdx.x * L;
  const int per = (L + 1023) / 1024;
  const int i0 = min(L, threadIdx.x * per), i1 = min(L, i0 + per);
  uint32_t local = 0;
  for (int i = i0; i < i1; ++i) local += h[i];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, w, o);
      if (lane >= o) w += y;
    }
    warp_sums[lane] = w;
  }
  __syncthreads();
  uint32_t run = (warp > 0 ? warp_sums[warp - 1] : 0u) + x - local;
  for (int i = i0; i < i1; ++i) {
    const uint32_t v = h[i];
    h[i] = run;
    run += v;
  }
}

__global__ void __launch_bounds__(kSortThreads) radix_scatter_kernel(const uint32_t* __restrict__ kin,
                                                                     const uint32_t* __restrict__ vin,
                                                                     uint32_t* __restrict__ kout,
                                                                     uint32_t* __restrict__ vout, int n, int shift,
                                                                     int n_cta, const uint32_t* __restrict__ hist) {
  constexpr int W = kSortThreads / 32;
  __shared__ uint32_t wc[W][256];
  __shared__ uint32_t wp[W][256];
  __shared__ uint32_t run[256];
  __shared__ uint32_t off[256];
  const int seg = blockIdx.y, cta = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int w = 0; w < W; ++w) wc[w][tid] = 0;
  run[tid] = 0;
  off[tid] = hist[((long)seg * 256 + tid) * n_cta + cta];
  __syncthreads();
  const long base = (long)seg * n;
  const unsigned lt = (1u << lane) - 1u;
  for (int it = 0; it < kSortTile / kSortThreads; ++it) {
    const int e = cta * kSortTile + it * kSortThreads + tid;
    const bool valid = e < n;
    const uint32_t key = valid ? kin[base + e] : 0u;
    const uint32_t val = valid ? vin[base + e] : 0u;
    const uint32_t digit = (key >> shift) & 255u;
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, valid ? digit : 0x100u + lane);
    const int rank = __popc(peers & lt);
    if (valid && rank == 0) wc[warp][digit] = __popc(peers);
    __syncthreads();
    {
      uint32_t pre = run[tid];
#pragma unroll
      for (int w = 0; w < W; ++w) {
        wp[w][tid] = pre;
        pre += wc[w][tid];
        wc[w][tid] = 0;
      }
      run[tid] = pre;
    }
    __syncthreads();
    if (valid) {
      const uint32_t pos = off[digit] + wp[warp][digit] + (uint32_t)rank;
      kout[base + pos] = key;
      vout[base + pos] = val;
    }
    __syncthreads();
  }
}

}  // namespace

size_t plan_bytes(long units, int n_seg, int n_per_seg) {
  const int n_cta = (n_per_seg + kSortTile - 1) / kSortTile;
  return 4 * align256((size_t)units * 4) + align256((size_t)n_seg * 256 * n_cta * 4);
}

cudaError_t launch_plan(const int32_t* sel, int sel_T, int sel_t0, int batch, int G, int Kb, int B, int t_begin,
                        int t_end, void* ws, const uint32_t** perm_out, cudaStream_t s) {
  const int n = t_end - t_begin;
  const int n_seg = batch * G;
  const long units = (long)n * n_seg;
  const int n_cta = (n + kSortTile - 1) / kSortTile;
  uint8_t* p = static_cast<uint8_t*>(ws);
  uint32_t* k0 = reinterpret_cast<uint32_t*>(p);
  p += align256((size_t)units * 4);
  uint32_t* v0 = reinterpret_cast<uint32_t*>(p);
  p += align256((size_t)units * 4);
  uint32_t* k1 = reinterpret_cast<uint32_t*>(p);
  p += align256((size_t)units * 4);
  uint32_t* v1 = reinterpret_cast<uint32_t*>(p);
  p += align256((size_t)units * 4);
  uint32_t* hist = reinterpret_cast<uint32_t*>(p);
  const long threads = units * 32;
  signature_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(sel, sel_T, sel_t0, G, Kb, B, t_begin, n, n_seg,
                                                                     k0, v0);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  for (int pass = 0; pass < kKeyBits / 8; ++pass) {
    const int shift = 8 * pass;
    radix_hist_kernel<<<dim3(n_cta, n_seg), kSortThreads, 0, s>>>(k0, n, shift, n_cta, hist);
    radix_scan_kernel<<<n_seg, 1024, 0, s>>>(hist, n_cta);
    radix_scatter_kernel<<<dim3(n_cta, n_seg), kSortThreads, 0, s>>>(k0, v0, k1, v1, n, shift, n_cta, hist);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    uint32_t* tk = k0; k0 = k1; k1 = tk;
    uint32_t* tv = v0; v0 = v1; v1 = tv;
  }
  *perm_out = v0;
  return cudaSuccess;
}

}  // namespace sgqa
