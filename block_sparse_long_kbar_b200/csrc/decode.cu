// Decode-step kernels: cache append, K4 indexer scores over a long cache, K5 exact top-m select.
//
// A decode step appends n_new tokens to each sequence's caches and computes the layer for them
// exactly as a prefill of the concatenated sequence would (orcarouter.ai, "Step 5 Preview NVFP4
// checkpoint", serving recipe: 1M-token context, MTP with 3 speculative tokens, so 4 query
// tokens per step). With a 1M-token cache a row has up to 131072 candidate blocks, too many
// for one CTA's shared memory, so the select is split in two kernels:
//   K4: grid over (sequence, 256-block chunk); each thread owns one candidate block, keeps its
//       kbar row in registers and scores it against all n_new * G rows of the sequence (fp32,
//       fixed FMA order), writing scores [seq, row, block] with coalesced stores.
//   K5: one CTA per row: an exact radix select of the m-th largest order-preserving key over the
//       row's scores (256-bin shared histograms, 8 bits per pass, early exit), then an ordered
//       emit: per-thread contiguous segments, block scans of the tie and pick counts, so the
//       output is ascending and ties at the threshold go to the lower block index.
#include "common.cuh"
#include "kernels.h"

namespace sgqa {
namespace {

__global__ void __launch_bounds__(256) append_kernel(uint16_t* __restrict__ dst, const uint16_t* __restrict__ src,
                                                     long n8_per_seq, long dst_seq_stride8, long dst_off8, int batch) {
  const long e = (long)blockIdx.x * blockDim.x + threadIdx.x;
  const long total = n8_per_seq * batch;
  if (e >= total) return;
  const long b = e / n8_per_seq, i = e % n8_per_seq;
  reinterpret_cast<uint4*>(dst)[b * dst_seq_stride8 + dst_off8 + i] = __ldg(reinterpret_cast<const uint4*>(src) + e);
}

constexpr int kMaxRows = 32;

template <int DI>
__global__ void __launch_bounds__(256) decode_scores_kernel(const uint16_t* __restrict__ qidx_new,
                                                            const float* __restrict__ kbar, float* __restrict__ scores,
                                                            int n_new, int G, int B, int nblk, int t0) {
  __shared__ float qs[kMaxRows][DI];
  const int b = blockIdx.y;
  const int rows = n_new * G;
  for (int i = threadIdx.x; i < rows * DI; i += blockDim.x) {
    const int r = i / DI, c = i % DI;
    qs[r][c] = bf16_to_f32(qidx_new[((long)b * rows + r) * DI + c]);
  }
  __syncthreads();
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  const int c_max = (t0 + n_new - 1) / B;  // candidates of the last new token
  if (j >= c_max) return;
  float kv[DI];
  const float4* kp = reinterpret_cast<const float4*>(kbar + ((long)b * nblk + j) * DI);
#pragma unroll
  for (int i = 0; i < DI / 4; ++i) {
    const float4 w = __ldg(kp + i);
    kv[4 * i] = w.x; kv[4 * i + 1] = w.y; kv[4 * i + 2] = w.z; kv[4 * i + 3] = w.w;
  }
  for (int r = 0; r < rows; ++r) {
    const int t = t0 + r / G;
    if (j >= t / B) continue;
    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
    for (int i = 0; i < DI; i += 2) {
      acc0 = fmaf(qs[r][i], kv[i], acc0);
      acc1 = fmaf(qs[r][i + 1], kv[i + 1], acc1);
    }
    scores[((long)b * rows + r) * nblk + j] = acc0 + acc1;
  }
}

constexpr int kSelThreads = 512;

// exclusive block scan of one int per thread (512 threads); returns the exclusive prefix and
// writes the total to *total
__device__ int block_exclusive_scan(int v, int* scratch, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kSelThreads / 32 ? scratch[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < kSelThreads / 32) scratch[32 + lane] = w;  // inclusive warp totals
  }
  __syncthreads();
  const int before = (warp > 0 ? scratch[32 + warp - 1] : 0) + x - v;
  *total = scratch[32 + kSelThreads / 32 - 1];
  __syncthreads();
  return before;
}

__global__ void __launch_bounds__(kSelThreads) decode_select_kernel(const float* __restrict__ scores,
                                                                    int32_t* __restrict__ sel, int n_new, int G, int B,
                                                                    int Kb, int nblk, int t0, int* status) {
  __shared__ int hist[256];
  __shared__ int scratch[64];
  __shared__ uint32_t s_prefix, s_mask;
  __shared__ int s_rem, s_nb;
  const int rows = n_new * G;
  const int b = blockIdx.x / rows, r = blockIdx.x % rows;
  const int t = t0 + r / G;
  const int c = t / B;
  const int m = min(Kb - 1, c);
  const float* row = scores + ((long)b * rows + r) * nblk;
  if (threadIdx.x == 0) {
    s_prefix = 0; s_mask = 0; s_rem = m; s_nb = c;
    if (m == 0) { s_prefix = 0xFFFFFFFFu; s_mask = 0xFFFFFFFFu; }
  }
  __syncthreads();
  for (int pass = 0; pass < 4; ++pass) {
    const bool done = (s_rem == s_nb) || (s_mask == 0xFFFFFFFFu);
    if (done) break;
    const int shift = 24 - 8 * pass;
    const uint32_t prefix = s_prefix, mask = s_mask;
    for (int i = threadIdx.x; i < 256; i += kSelThreads) hist[i] = 0;
    __syncthreads();
    for (int j = threadIdx.x; j < c; j += kSelThreads) {
      const uint32_t key = score_key(__ldg(row + j));
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int above = 0;
      const int rem = s_rem;
      for (int bin = 255; bin >= 0; --bin) {
        const int h = hist[bin];
        if (above + h >= rem) {
          s_prefix = prefix | ((uint32_t)bin << shift);
          s_mask = mask | (255u << shift);
          s_rem = rem - above;
          s_nb = h;
          break;
        }
        above += h;
      }
    }
    __syncthreads();
  }
  const uint32_t prefix = s_prefix, mask = s_mask;
  const int rem = s_rem;
  // ordered emit: contiguous segments, counts, scans, then writes
  const int seg = (c + kSelThreads - 1) / kSelThreads;
  const int j_lo = min(c, threadIdx.x * seg), j_hi = min(c, j_lo + seg);
  int n_gt = 0, n_eq = 0;
  for (int j = j_lo; j < j_hi; ++j) {
    const uint32_t key = score_key(__ldg(row + j)) & mask;
    n_gt += key > prefix;
    n_eq += key == prefix;
  }
  int tot;
  const int eq_before = block_exclusive_scan(n_eq, scratch, &tot);
  const int eq_take = max(0, min(n_eq, rem - eq_before));
  const int pos0 = block_exclusive_scan(n_gt + eq_take, scratch, &tot);
  int32_t* out = sel + ((long)b * rows + r) * Kb;
  int pos = pos0, eq_seen = 0;
  for (int j = j_lo; j < j_hi; ++j) {
    const uint32_t key = score_key(__ldg(row + j)) & mask;
    bool take = key > prefix;
    if (key == prefix) take = eq_seen++ < eq_take;
    if (take && pos < m) out[pos++] = j;
  }
  if (threadIdx.x == 0) {
    if (tot != m) report(status, SGQA_ERR_DEVICE_CHECK);
    out[m] = c;
  }
  for (int i = m + 1 + threadIdx.x; i < Kb; i += kSelThreads) out[i] = -1;
}

}  // namespace

cudaError_t launch_append(uint16_t* dst, const uint16_t* src, int batch, long row_elems, long dst_seq_stride,
                          long dst_off, long n_elems_per_seq, cudaStream_t s) {
  (void)row_elems;
  if (n_elems_per_seq <= 0) return cudaSuccess;
  const long n8 = n_elems_per_seq / 8;
  const long total = n8 * batch;
  append_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(dst, src, n8, dst_seq_stride / 8, dst_off / 8, batch);
  return cudaGetLastError();
}

cudaError_t launch_decode_scores(const uint16_t* qidx_new, const float* kbar, float* scores, int batch, int n_new,
                                 int G, int d_idx, int B, int nblk, int t0, cudaStream_t s) {
  if (n_new * G > kMaxRows) return cudaErrorInvalidValue;
  const int c_max = (t0 + n_new - 1) / B;
  if (c_max <= 0) return cudaSuccess;
  const dim3 grid((unsigned)((c_max + 255) / 256), (unsigned)batch);
  if (d_idx == 64) decode_scores_kernel<64><<<grid, 256, 0, s>>>(qidx_new, kbar, scores, n_new, G, B, nblk, t0);
  else if (d_idx == 32) decode_scores_kernel<32><<<grid, 256, 0, s>>>(qidx_new, kbar, scores, n_new, G, B, nblk, t0);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_decode_select(const float* scores, int32_t* sel, int batch, int n_new, int G, int B, int Kb,
                                 int nblk, int t0, int* status, cudaStream_t s) {
  decode_select_kernel<<<(unsigned)(batch * n_new * G), kSelThreads, 0, s>>>(scores, sel, n_new, G, B, Kb, nblk, t0,
                                                                             status);
  return cudaGetLastError();
}

}  // namespace sgqa
