// K2: per-(token, KV group) block selection (Step 5 Preview pages: mo.ai.kr, "Step 5 Preview
// agentic work design", section "model structure and training stability" — each KV group picks
// its own relevant past blocks; k = 4096 tokens = 512 blocks with B = 8).
//
// Definition implemented: c = floor(t/B); candidates j < c with score s_j = q_idx[t,g] . kbar[j];
// keep the best m = min(k/B - 1, c) by (s desc, j asc), then the own block c; ascending.
//
// Design (first version, CUDA cores). A CTA owns 128 rows = (128/G) adjacent queries x G
// groups, one row per thread. kbar tiles are staged in shared memory and shared by all 128 rows
// (the rows of one tile need the same candidate blocks). Per row, an exact radix select on the
// order-preserving 32-bit score key finds the m-th largest key tau: each pass recomputes the
// row's scores and fills a private 256-bin histogram of the next 8 key bits among the keys that
// still match the resolved prefix; a row stops as soon as its threshold bucket is taken whole.
// A final pass streams the candidates in ascending j and emits key > tau, plus the first ties
// at tau (lower block index wins), so the output is ascending without a sort. Scores are fp32
// dot products with a fixed FMA order, recomputed bit-identically in every pass.
#include "common.cuh"
#include "kernels.h"

namespace sgqa {
namespace {

constexpr int kRows = 128;
constexpr int kTile = 64;          // candidate blocks per shared-memory tile
constexpr int kHistStride = 257;   // padded histogram row (bank spread)

template <int DI>
__device__ __forceinline__ float dot_row(const float (&q)[DI], const float* __restrict__ kb) {
  float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
  for (int i = 0; i < DI; i += 8) {
    const float4 a = *reinterpret_cast<const float4*>(kb + i);
    const float4 b = *reinterpret_cast<const float4*>(kb + i + 4);
    acc0 = fmaf(q[i + 0], a.x, acc0);
    acc1 = fmaf(q[i + 1], a.y, acc1);
    acc0 = fmaf(q[i + 2], a.z, acc0);
    acc1 = fmaf(q[i + 3], a.w, acc1);
    acc0 = fmaf(q[i + 4], b.x, acc0);
    acc1 = fmaf(q[i + 5], b.y, acc1);
    acc0 = fmaf(q[i + 6], b.z, acc0);
    acc1 = fmaf(q[i + 7], b.w, acc1);
  }
  return acc0 + acc1;
}

template <int DI>
__device__ __forceinline__ void load_tile(float* ktile, const float* __restrict__ kb_seq, int j0, int n) {
  // n blocks of DI floats, as float4, by 128 threads
  const int total4 = n * (DI / 4);
  const float4* src = reinterpret_cast<const float4*>(kb_seq + (long)j0 * DI);
  float4* dst = reinterpret_cast<float4*>(ktile);
  for (int i = threadIdx.x; i < total4; i += kRows) dst[i] = __ldg(src + i);
}

template <int DI>
__global__ void __launch_bounds__(kRows, 1) select_kernel(SelectArgs a) {
  extern __shared__ __align__(16) uint32_t smem[];
  uint32_t* hist = smem;
  float* ktile = reinterpret_cast<float*>(smem + kRows * kHistStride);

  const int G = a.G;
  const int TQ = kRows / G;
  const int n_tiles = (a.t_end - a.t_begin + TQ - 1) / TQ;
  const int tile = n_tiles - 1 - (int)(blockIdx.x / a.batch);  // heaviest tiles first
  const int b = (int)(blockIdx.x % a.batch);
  const int r = threadIdx.x;
  const int tq0 = a.t_begin + tile * TQ;
  const int t = tq0 + r / G;
  const int g = r % G;
  const bool valid = t < a.t_end;
  const int c = valid ? t / a.B : 0;
  const int m = valid ? min(a.Kb - 1, c) : 0;
  const int t_last = min(a.t_end - 1, tq0 + TQ - 1);
  const int n_cand = t_last / a.B;  // the tile's largest candidate count
  const int nblk = a.T / a.B;
  const float* kb_seq = a.kbar + (long)b * nblk * DI;

  float q[DI];
  if (valid) {
    const uint4* qp = reinterpret_cast<const uint4*>(a.q_idx + (((long)b * a.T + t) * G + g) * DI);
#pragma unroll
    for (int i = 0; i < DI / 8; ++i) {
      const uint4 w = __ldg(qp + i);
      q[8 * i + 0] = bf16_lo(w.x); q[8 * i + 1] = bf16_hi(w.x);
      q[8 * i + 2] = bf16_lo(w.y); q[8 * i + 3] = bf16_hi(w.y);
      q[8 * i + 4] = bf16_lo(w.z); q[8 * i + 5] = bf16_hi(w.z);
      q[8 * i + 6] = bf16_lo(w.w); q[8 * i + 7] = bf16_hi(w.w);
    }
  } else {
#pragma unroll
    for (int i = 0; i < DI; ++i) q[i] = 0.f;
  }

  // Radix state: keys with (key & mask) == prefix form the threshold bucket; rem of them are
  // still to be taken, nb is the bucket's size. done <=> the bucket is taken whole or fully
  // resolved (32 bits).
  uint32_t prefix = 0, mask = 0;
  int rem = m, nb = c;
  bool done = (rem == nb);
  if (rem == 0) { prefix = 0xFFFFFFFFu; mask = 0xFFFFFFFFu; done = true; }
  uint32_t* my_hist = hist + r * kHistStride;

  for (int pass = 0; pass < 4; ++pass) {
    if (!__syncthreads_or(!done)) break;
    const int shift = 24 - 8 * pass;
    for (int i = 0; i < 256; ++i) my_hist[i] = 0;
    for (int j0 = 0; j0 < n_cand; j0 += kTile) {
      const int n = min(kTile, n_cand - j0);
      __syncthreads();
      load_tile<DI>(ktile, kb_seq, j0, n);
      __syncthreads();
      if (!done) {
        const int jn = min(n, c - j0);
        for (int jj = 0; jj < jn; ++jj) {
          const uint32_t key = score_key(dot_row<DI>(q, ktile + jj * DI));
          if ((key & mask) == prefix) my_hist[(key >> shift) & 255u]++;
        }
      }
    }
    if (!done) {
      int above = 0;
      for (int bin = 255; bin >= 0; --bin) {
        const int h = (int)my_hist[bin];
        if (above + h >= rem) {
          prefix |= (uint32_t)bin << shift;
          mask |= 255u << shift;
          rem -= above;
          nb = h;
          break;
        }
        above += h;
      }
      done = (rem == nb) || (mask == 0xFFFFFFFFu);
    }
  }

  // Emit: ascending j; key above the bucket -> taken; in the bucket -> the first rem taken.
  int32_t* out = a.sel + (((long)b * a.sel_T + (t - a.sel_t0)) * G + g) * (long)a.Kb;
  int pos = 0, eq_taken = 0;
  for (int j0 = 0; j0 < n_cand; j0 += kTile) {
    const int n = min(kTile, n_cand - j0);
    __syncthreads();
    load_tile<DI>(ktile, kb_seq, j0, n);
    __syncthreads();
    if (valid) {
      const int jn = min(n, c - j0);
      for (int jj = 0; jj < jn; ++jj) {
        const uint32_t key = score_key(dot_row<DI>(q, ktile + jj * DI)) & mask;
        bool take = key > prefix;
        if (key == prefix) take = (eq_taken++ < rem);
        if (take && pos < m) out[pos++] = j0 + jj;
      }
    }
  }
  if (valid) {
    if (pos != m) report(a.status, SGQA_ERR_DEVICE_CHECK);
    out[pos++] = c;
    for (; pos < a.Kb; ++pos) out[pos] = -1;
  }
}

}  // namespace

cudaError_t launch_select(const SelectArgs& a, cudaStream_t s) {
  if (a.t_end <= a.t_begin) return cudaSuccess;
  const int TQ = kRows / a.G;
  const int n_tiles = (a.t_end - a.t_begin + TQ - 1) / TQ;
  const size_t shmem = (size_t)kRows * kHistStride * 4 + (size_t)kTile * a.d_idx * 4;
  const dim3 grid((unsigned)(n_tiles * a.batch));
  cudaError_t e;
  if (a.d_idx == 64) {
    e = cudaFuncSetAttribute(select_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shmem);
    if (e != cudaSuccess) return e;
    select_kernel<64><<<grid, kRows, shmem, s>>>(a);
  } else if (a.d_idx == 32) {
    e = cudaFuncSetAttribute(select_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shmem);
    if (e != cudaSuccess) return e;
    select_kernel<32><<<grid, kRows, shmem, s>>>(a);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace sgqa
