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

// Exact selection of one row over its scores in global memory: radix passes of 8 key bits
// (256-bin shared histograms, early exit), then an ordered emit over per-thread contiguous
// segments with block scans of the tie and pick counts, so the output is ascending and ties at the
// threshold go to the lower block index. Called by all kSelThreads threads of the block.
__device__ void select_row_radix(const float* __restrict__ row, int c, int m, int Kb, int32_t* __restrict__ out,
                                 int* status) {
  __shared__ int hist[256];
  __shared__ int scratch[64];
  __shared__ uint32_t s_prefix, s_mask;
  __shared__ int s_rem, s_nb;
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
  const int j_lo = min(c, (int)threadIdx.x * seg), j_hi = min(c, j_lo + seg);
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

__global__ void __launch_bounds__(kSelThreads) decode_select_kernel(const float* __restrict__ scores,
                                                                    int32_t* __restrict__ sel, int n_new, int G, int B,
                                                                    int Kb, int nblk, int t0, int* status) {
  const int rows = n_new * G;
  const int b = blockIdx.x / rows, r = blockIdx.x % rows;
  const int c = (t0 + r / G) / B;
  select_row_radix(scores + ((long)b * rows + r) * nblk, c, min(Kb - 1, c), Kb,
                   sel + ((long)b * rows + r) * Kb, status);
}

// ---- K5 with a threshold bound ------------------------------------------------------------------
// The largest key of every 32 consecutive candidates (written by K4) gives m distinct candidates
// whose keys are >= the m-th largest of those maxima, L: so the row's m-th largest key is >= L and
// every candidate below L can be dropped. Index keys cluster by topic, so L alone can still leave
// tens of thousands of candidates; one stream over the row's scores therefore histograms the top
// 12 bits of every key >= L (4096 bins), which locates the bin holding the m-th largest key, and
// a second stream collects the candidates at or above that bin (typically a few thousand) with
// their block ids in shared memory. The exact selection is then made among them: radix passes
// over their keys for the threshold key K*, and among the candidates equal to K* the lowest block
// ids (radix passes over ~j); the chosen ids are sorted (bitonic) and written ascending. A row
// whose threshold bin alone holds more than kCap candidates takes the full radix path instead.
constexpr int kCap = 7168;
constexpr int kHBits = 12;
constexpr int kHBins = 1 << kHBits;
constexpr int kGl = 4096;  // groups listed at a time

// Warp-aggregated histogram increment of bin `bin` (lanes with want == false add nothing).
__device__ __forceinline__ void hist_add(int* hist, uint32_t bin, bool want) {
  const unsigned act = __ballot_sync(0xFFFFFFFFu, want);
  if (!want) return;
  const unsigned peers = __match_any_sync(act, bin);
  if ((threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
}

// m-th largest (1-based, 1 <= m <= number of valid entries) of get(i) over valid(i), i < n; all
// threads of the block call it. Returns the key; *rem_out = m - (number of valid keys above it).
template <class Get, class Valid>
__device__ uint32_t kth_largest(int n, int m, Get get, Valid valid, int* rem_out) {
  __shared__ int hist[256];
  __shared__ uint32_t s_prefix, s_mask;
  __shared__ int s_rem;
  if (threadIdx.x == 0) { s_prefix = 0; s_mask = 0; s_rem = m; }
  __syncthreads();
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    const uint32_t prefix = s_prefix, mask = s_mask;
    for (int i = threadIdx.x; i < 256; i += kSelThreads) hist[i] = 0;
    __syncthreads();
    const int n_pad = (n + 31) & ~31;
    for (int i = threadIdx.x; i < n_pad; i += kSelThreads) {
      bool want = false;
      uint32_t key = 0;
      if (i < n && valid(i)) {
        key = get(i);
        want = (key & mask) == prefix;
      }
      hist_add(hist, (key >> shift) & 255u, want);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // warp 0 locates the bin: lane l holds bins 255 - 8l .. 248 - 8l, counts above by a scan
      const int ln = threadIdx.x;
      const int rem = s_rem;
      __syncwarp();
      int cnt[8], local = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        cnt[i] = hist[255 - 8 * ln - i];
        local += cnt[i];
      }
      int x = local;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
        if (ln >= o) x += y;
      }
      int acc = x - local;  // keys in the bins above this lane's
      if (acc < rem && acc + local >= rem) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (acc + cnt[i] >= rem) {
            s_prefix = prefix | ((uint32_t)(255 - 8 * ln - i) << shift);
            s_mask = mask | (255u << shift);
            s_rem = rem - acc;
            break;
          }
          acc += cnt[i];
        }
      }
    }
    __syncthreads();
  }
  *rem_out = s_rem;
  const uint32_t res = s_prefix;
  __syncthreads();
  return res;
}

__global__ void __launch_bounds__(kSelThreads, 3) decode_select_bound_kernel(const float* __restrict__ scores,
                                                                          const uint32_t* __restrict__ tmax,
                                                                          int32_t* __restrict__ sel, int n_new, int G,
                                                                          int B, int Kb, int nblk, int tstride, int t0,
                                                                          int sort_n, int* status) {
  extern __shared__ uint32_t sm[];
  uint32_t* skey = sm;               // [kCap]
  uint32_t* sj = sm + kCap;          // [kCap]
  uint32_t* sorted = sm + 2 * kCap;  // [sort_n]
  uint16_t* glist = reinterpret_cast<uint16_t*>(sorted + sort_n);  // [kGl] groups that reach L
  int* hist = reinterpret_cast<int*>(sm);  // [kHBins], before the survivors are collected
  uint32_t* stm = sj;                      // [n32] the row's group maxima while L is found
  __shared__ int s_cnt, s_pick, s_bin, s_total, s_ng;
  __shared__ int scratch[64];
  const int rows = n_new * G;
  const int b = blockIdx.x / rows, r = blockIdx.x % rows;
  const int c = (t0 + r / G) / B;
  const int m = min(Kb - 1, c);
  const float* row = scores + ((long)b * rows + r) * nblk;
  int32_t* out = sel + ((long)b * rows + r) * Kb;
  const int tid = threadIdx.x, lane = tid & 31;
  if (m == c) {  // every candidate is taken
    for (int i = tid; i < Kb; i += kSelThreads) out[i] = i <= c ? i : -1;
    return;
  }
  if (m == 0) {  // a budget of one block: the own block alone
    for (int i = tid; i < Kb; i += kSelThreads) out[i] = i == 0 ? c : -1;
    return;
  }
  // 1. the bound L from the maxima of 32 candidates (staged in shared memory when they fit)
  const int n32 = (c + 31) / 32;
  const uint32_t* tm = tmax + ((long)b * rows + r) * tstride;
  uint32_t L = 0;
  int rem_dummy;
  if (n32 >= m) {
    if (n32 <= kCap) {
      for (int i = tid; i < n32; i += kSelThreads) stm[i] = __ldg(tm + i);
      __syncthreads();
      L = kth_largest(n32, m, [&](int i) { return stm[i]; }, [](int) { return true; }, &rem_dummy);
    } else {
      L = kth_largest(n32, m, [&](int i) { return __ldg(tm + i); }, [](int) { return true; }, &rem_dummy);
    }
  }
  // Both passes below read only the 32-candidate groups whose maximum reaches L (a group below
  // it holds no key >= L). Those groups are first listed in shared memory, kGl at a time, so that
  // a warp then loads 8 listed groups at once (lane = candidate) with no dependent load in front.
  const int warp = tid >> 5;
  constexpr int kWarps = kSelThreads / 32;
  auto list_groups = [&](int g_begin) {  // all threads; returns the number listed
    if (tid == 0) s_ng = 0;
    __syncthreads();
    const int g_end = min(n32, g_begin + kGl);
    for (int g0 = g_begin; g0 < g_end; g0 += kSelThreads) {
      const int gi = g0 + tid;
      const bool keep = gi < g_end && __ldg(tm + gi) >= L;
      const unsigned bal = __ballot_sync(0xFFFFFFFFu, keep);
      int pos = 0;
      if (lane == 0 && bal) pos = atomicAdd(&s_ng, __popc(bal));
      pos = __shfl_sync(0xFFFFFFFFu, pos, 0) + __popc(bal & ((1u << lane) - 1u));
      if (keep) glist[pos] = (uint16_t)(gi - g_begin);
    }
    __syncthreads();
    return s_ng;
  };
  // f(j, key, ok) for every candidate of the listed groups (ok: j < c and key >= L); all threads
  auto for_listed = [&](int g_begin, int ng, auto&& f) {
    for (int e0 = warp * 8; e0 < ng; e0 += 8 * kWarps) {
      float v[8];
      int j[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        j[u] = e0 + u < ng ? (g_begin + (int)glist[e0 + u]) * 32 + lane : c;
        v[u] = j[u] < c ? __ldg(row + j[u]) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint32_t key = score_key(v[u]);
        f(j[u], key, j[u] < c && key >= L);
      }
    }
  };
  // 2. histogram of the top 12 key bits of the keys >= L
  for (int i = tid; i < kHBins; i += kSelThreads) hist[i] = 0;
  if (tid == 0) { s_cnt = 0; s_pick = 0; }
  __syncthreads();
  int ng_first = 0;
  for (int gb = 0; gb < n32; gb += kGl) {
    const int ng = list_groups(gb);
    if (gb == 0) ng_first = ng;
    for_listed(gb, ng, [&](int, uint32_t key, bool ok) { hist_add(hist, key >> (32 - kHBits), ok); });
    __syncthreads();  // the list is rebuilt for the next chunk
  }
  // the bin of the m-th largest key: suffix sums over 8 bins per thread, scanned from the top
  {
    constexpr int kPer = kHBins / kSelThreads;
    const int top = kHBins - 1 - kPer * tid;  // this thread's bins: top, top - 1, ..., top - kPer + 1
    int local = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) local += hist[top - i];
    int tot;
    const int above = block_exclusive_scan(local, scratch, &tot);  // keys in all higher threads' bins
    if (above < m && above + local >= m) {
      int acc = above;
      for (int i = 0; i < kPer; ++i) {
        const int h = hist[top - i];
        if (acc + h >= m) {
          s_bin = top - i;
          s_total = acc + h;  // keys at or above the threshold bin
          break;
        }
        acc += h;
      }
    }
  }
  __syncthreads();
  const int total = s_total;
  if (total > kCap) {
    select_row_radix(row, c, m, Kb, out, status);
    return;
  }
  const uint32_t lo = (uint32_t)s_bin << (32 - kHBits);
  __syncthreads();  // the histogram area is reused for the survivors below
  // 3. the survivors (keys at or above the threshold bin), any order; the list of the first
  // chunk is still in place when it was the only one
  auto keep_survivor = [&](int j, uint32_t key, bool ok) {
    const bool keep = ok && key >= lo;
    const unsigned bal = __ballot_sync(0xFFFFFFFFu, keep);
    if (bal == 0u) return;
    int pos = 0;
    if (lane == __ffs(bal) - 1) pos = atomicAdd(&s_cnt, __popc(bal));
    pos = __shfl_sync(0xFFFFFFFFu, pos, __ffs(bal) - 1) + __popc(bal & ((1u << lane) - 1u));
    if (keep && pos < kCap) {
      skey[pos] = key;
      sj[pos] = (uint32_t)j;
    }
  };
  if (n32 <= kGl) {
    for_listed(0, ng_first, keep_survivor);
  } else {
    for (int gb = 0; gb < n32; gb += kGl) {
      const int ng = list_groups(gb);
      for_listed(gb, ng, keep_survivor);
      __syncthreads();
    }
  }
  __syncthreads();
  const int ns = s_cnt;
  if (ns != total) report(status, SGQA_ERR_DEVICE_CHECK);
  // 4. the threshold key among the survivors, then the lowest block ids among its ties
  int rem = 0;
  const uint32_t kstar = kth_largest(ns, m, [&](int i) { return skey[i]; }, [](int) { return true; }, &rem);
  // among the keys equal to K*, the rem lowest block ids (all of them when there are just rem)
  if (tid == 0) s_pick = 0;
  __syncthreads();
  {
    int eq = 0;
    for (int i = tid; i < ns; i += kSelThreads) eq += skey[i] == kstar;
    eq = __reduce_add_sync(0xFFFFFFFFu, eq);
    if (lane == 0 && eq) atomicAdd(&s_pick, eq);
  }
  __syncthreads();
  const int n_eq = s_pick;
  __syncthreads();
  if (tid == 0) s_pick = 0;
  uint32_t jstar = 0xFFFFFFFFu;
  if (n_eq > rem) {
    int rem2 = 0;
    jstar = ~kth_largest(ns, rem, [&](int i) { return ~sj[i]; }, [&](int i) { return skey[i] == kstar; }, &rem2);
  }
  __syncthreads();
  // 5. the chosen ids, sorted ascending (bitonic, padded with 0xFFFFFFFF)
  for (int i = tid; i < sort_n; i += kSelThreads) sorted[i] = 0xFFFFFFFFu;
  __syncthreads();
  for (int i = tid; i < ns; i += kSelThreads) {
    const uint32_t key = skey[i];
    if (key > kstar || (key == kstar && sj[i] <= jstar)) {
      const int p = atomicAdd(&s_pick, 1);
      if (p < sort_n) sorted[p] = sj[i];
    }
  }
  __syncthreads();
  for (int k = 2; k <= sort_n; k <<= 1) {
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      for (int i = tid; i < sort_n; i += kSelThreads) {
        const int ixj = i ^ jj;
        if (ixj > i) {
          const uint32_t x = sorted[i], y = sorted[ixj];
          const bool asc = (i & k) == 0;
          if ((x > y) == asc) {
            sorted[i] = y;
            sorted[ixj] = x;
          }
        }
      }
      __syncthreads();
    }
  }
  if (tid == 0 && s_pick != m) report(status, SGQA_ERR_DEVICE_CHECK);
  for (int i = tid; i < Kb; i += kSelThreads) out[i] = i < m ? (int32_t)sorted[i] : i == m ? c : -1;
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

cudaError_t launch_decode_select_bound(const float* scores, const uint32_t* tmax, int32_t* sel, int batch, int n_new,
                                       int G, int B, int Kb, int nblk, int tstride, int t0, int* status,
                                       cudaStream_t s) {
  int sort_n = 1;
  while (sort_n < Kb) sort_n <<= 1;
  const size_t shmem = (size_t)(2 * kCap + sort_n) * 4 + kGl * sizeof(uint16_t);
  cudaError_t e = cudaFuncSetAttribute(decode_select_bound_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)shmem);
  if (e != cudaSuccess) return e;
  decode_select_bound_kernel<<<(unsigned)(batch * n_new * G), kSelThreads, shmem, s>>>(
      scores, tmax, sel, n_new, G, B, Kb, nblk, tstride, t0, sort_n, status);
  return cudaGetLastError();
}

cudaError_t launch_decode_select(const float* scores, int32_t* sel, int batch, int n_new, int G, int B, int Kb,
                                 int nblk, int t0, int* status, cudaStream_t s) {
  decode_select_kernel<<<(unsigned)(batch * n_new * G), kSelThreads, 0, s>>>(scores, sel, n_new, G, B, Kb, nblk, t0,
                                                                             status);
  return cudaGetLastError();
}

}  // namespace sgqa
