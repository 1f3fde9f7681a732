// Backward of the gated attention through a fixed selection: dq, dk, dv and dgate.
//
// The 1M-context model is trained with this layer (mo.ai.kr, "Step 5 Preview agentic work
// design", section "model structure and training stability"); the selection is a discrete choice
// and carries no gradient. For every query row (b, t), head h of group g = h / R, over the
// selected tokens u <= t:
//   z_u = q . k_u / sqrt(d),  p = softmax(z),  o = sum p_u v_u,  s = sigmoid(gate),  y = o * s
//   dgate = dy * o * s * (1 - s),  do = dy * s,  D = do . o,  dp_u = do . v_u,
//   dz_u = p_u (dp_u - D),  dq = sum_u dz_u k_u / sqrt(d),
//   dk_u = sum over rows of dz_u q / sqrt(d),  dv_u = sum over rows of p_u do.
//
// Deterministic, no floating-point atomics:
//   BQ  (row-centric, one CTA per (b, t, g); a warp per head, four dims per lane): an online-softmax
//       pass for the row's max and sum (stored as lse) and o, then dgate and D, then a second pass
//       for dq. Tokens are taken NT at a time (a selected block, or half of a 16-token one): their
//       dot products and warp reductions are independent of one another, and the running maximum
//       is updated once per group.
//   reverse index (per (b, g)): for every block j, the rows that selected it, in increasing t
//       (per-chunk counts, scans over the chunks and the blocks, then every chunk of rows fills
//       its entries walking its rows in order).
//   BKV (key-centric, one CTA per (b, g, block j); the block's tokens split over the threads, a
//       slice of the head dims each): walks the block's selecting rows in order and, per head,
//       recomputes p_u and dz_u from lse, D and do (stored by BQ), accumulating dk and dv in
//       registers.
// Both compute kernels run on the CUDA cores in fp32 (the selection-sparse backward is
// memory-and-latency bound at these shapes; a tensor-core version is the next step).
#include <cmath>

#include "common.cuh"
#include "kernels.h"

namespace sgqa {
namespace {

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, o);
  return x;
}

__device__ __forceinline__ float sigmoidf_acc(float x) { return 1.f / (1.f + expf(-x)); }

// BQ: R heads of one (b, t, g) unit; warp w takes heads w, w + 4, ... (up to 4 per warp); NT
// tokens of a selected block per step.
template <int D, int NT>
__global__ void __launch_bounds__(128) backward_q_kernel(BackwardArgs a) {
  constexpr int DPL = D / 32;  // dims per lane
  constexpr int HPW = 4;       // at most 4 heads per warp (R <= 16)
  const int R = a.Hq / a.G;
  const int unit = blockIdx.x;
  const int g = unit % a.G;
  const long bt = unit / a.G;
  const int t = (int)(bt % a.T);
  const long b = bt / a.T;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nh = (R - warp + 3) / 4;  // heads of this warp
  if (nh <= 0) return;
  const float sc = 1.f / sqrtf((float)D);
  float q[HPW][DPL], o[HPW][DPL], m[HPW], l[HPW];
#pragma unroll
  for (int i = 0; i < HPW; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.f;
#pragma unroll
    for (int e = 0; e < DPL; ++e) q[i][e] = o[i][e] = 0.f;
    if (i < nh) {
      const long row = (bt * a.Hq + (long)g * R + warp + 4 * i) * D + lane * DPL;
#pragma unroll
      for (int e = 0; e < DPL; ++e) q[i][e] = bf16_to_f32(a.q[row + e]);
    }
  }
  const int32_t* srow = a.sel + (bt * a.G + g) * (long)a.Kb;
  const uint16_t* kseq = a.k + ((b * a.T) * a.G + g) * (long)D;
  const uint16_t* vseq = a.v + ((b * a.T) * a.G + g) * (long)D;
  const long kv_stride = (long)a.G * D;
  // pass 1: online max and sum, and o
  for (int i = 0; i < a.Kb; ++i) {
    const int j = __ldg(srow + i);
    if (j < 0) break;
    if (j > t / a.B) {
      if (lane == 0 && warp == 0) report(a.status, SGQA_ERR_DEVICE_CHECK);
      continue;
    }
    const int u_hi = min(j * a.B + a.B - 1, t);
    for (int u0 = j * a.B; u0 <= u_hi; u0 += NT) {
      float kv[NT][DPL], vv[NT][DPL];
#pragma unroll
      for (int s2 = 0; s2 < NT; ++s2) {
        const bool ok = u0 + s2 <= u_hi;
        const int u = ok ? u0 + s2 : u0;
#pragma unroll
        for (int e = 0; e < DPL; ++e) {
          kv[s2][e] = bf16_to_f32(__ldg(kseq + u * kv_stride + lane * DPL + e));
          vv[s2][e] = bf16_to_f32(__ldg(vseq + u * kv_stride + lane * DPL + e));
        }
      }
#pragma unroll
      for (int hh = 0; hh < HPW; ++hh) {
        if (hh >= nh) break;
        float z[NT];
#pragma unroll
        for (int s2 = 0; s2 < NT; ++s2) {
          float acc = 0.f;
#pragma unroll
          for (int e = 0; e < DPL; ++e) acc = fmaf(q[hh][e], kv[s2][e], acc);
          z[s2] = acc;
        }
#pragma unroll
        for (int s2 = 0; s2 < NT; ++s2) z[s2] = warp_sum(z[s2]) * sc;
        float mn = m[hh];
#pragma unroll
        for (int s2 = 0; s2 < NT; ++s2)
          if (u0 + s2 <= u_hi) mn = fmaxf(mn, z[s2]);
        const float corr = expf(m[hh] - mn);
        float ps = 0.f;
#pragma unroll
        for (int e = 0; e < DPL; ++e) o[hh][e] *= corr;
#pragma unroll
        for (int s2 = 0; s2 < NT; ++s2) {
          const float pz = u0 + s2 <= u_hi ? expf(z[s2] - mn) : 0.f;
          ps += pz;
#pragma unroll
          for (int e = 0; e < DPL; ++e) o[hh][e] = fmaf(pz, vv[s2][e], o[hh][e]);
        }
        l[hh] = l[hh] * corr + ps;
        m[hh] = mn;
      }
    }
  }
  // dgate, do, D; lse
  float dov[HPW][DPL], Dsum[HPW], lse[HPW];
#pragma unroll
  for (int hh = 0; hh < HPW; ++hh) {
    Dsum[hh] = 0.f;
    lse[hh] = 0.f;
#pragma unroll
    for (int e = 0; e < DPL; ++e) dov[hh][e] = 0.f;
    if (hh >= nh) continue;
    const int h = g * R + warp + 4 * hh;
    const long row = (bt * a.Hq + h) * D + lane * DPL;
    const float inv = l[hh] > 0.f ? 1.f / l[hh] : 0.f;
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < DPL; ++e) {
      const float oe = o[hh][e] * inv;
      const float s = sigmoidf_acc(bf16_to_f32(a.gate[row + e]));
      const float dye = bf16_to_f32(a.dy[row + e]);
      a.dgate[row + e] = dye * oe * s * (1.f - s);
      dov[hh][e] = dye * s;
      a.dov[row + e] = dov[hh][e];  // kept for the key-centric pass
      acc = fmaf(dov[hh][e], oe, acc);
    }
    Dsum[hh] = warp_sum(acc);
    lse[hh] = m[hh] + logf(l[hh]);
    if (lane == 0) {
      a.lse[bt * a.Hq + h] = lse[hh];
      a.dsum[bt * a.Hq + h] = Dsum[hh];
    }
  }
  // pass 2: dq
  float dq[HPW][DPL];
#pragma unroll
  for (int hh = 0; hh < HPW; ++hh)
#pragma unroll
    for (int e = 0; e < DPL; ++e) dq[hh][e] = 0.f;
  for (int i = 0; i < a.Kb; ++i) {
    const int j = __ldg(srow + i);
    if (j < 0) break;
    if (j > t / a.B) continue;
    const int u_hi = min(j * a.B + a.B - 1, t);
    for (int u0 = j * a.B; u0 <= u_hi; u0 += NT) {
      float kv[NT][DPL], vv[NT][DPL];
#pragma unroll
      for (int s2 = 0; s2 < NT; ++s2) {
        const bool ok = u0 + s2 <= u_hi;
        const int u = ok ? u0 + s2 : u0;
#pragma unroll
        for (int e = 0; e < DPL; ++e) {
          kv[s2][e] = bf16_to_f32(__ldg(kseq + u * kv_stride + lane * DPL + e));
          vv[s2][e] = bf16_to_f32(__ldg(vseq + u * kv_stride + lane * DPL + e));
        }
      }
#pragma unroll
      for (int hh = 0; hh < HPW; ++hh) {
        if (hh >= nh) break;
        float z[NT], dp[NT];
#pragma unroll
        for (int s2 = 0; s2 < NT; ++s2) {
          float az = 0.f, ap = 0.f;
#pragma unroll
          for (int e = 0; e < DPL; ++e) {
            az = fmaf(q[hh][e], kv[s2][e], az);
            ap = fmaf(dov[hh][e], vv[s2][e], ap);
          }
          z[s2] = az;
          dp[s2] = ap;
        }
#pragma unroll
        for (int s2 = 0; s2 < NT; ++s2) {
          z[s2] = warp_sum(z[s2]) * sc;
          dp[s2] = warp_sum(dp[s2]);
        }
#pragma unroll
        for (int s2 = 0; s2 < NT; ++s2) {
          if (u0 + s2 > u_hi) continue;
          const float p = expf(z[s2] - lse[hh]);
          const float dz = p * (dp[s2] - Dsum[hh]) * sc;
#pragma unroll
          for (int e = 0; e < DPL; ++e) dq[hh][e] = fmaf(dz, kv[s2][e], dq[hh][e]);
        }
      }
    }
  }
#pragma unroll
  for (int hh = 0; hh < HPW; ++hh) {
    if (hh >= nh) break;
    const long row = (bt * a.Hq + g * R + warp + 4 * hh) * D + lane * DPL;
#pragma unroll
    for (int e = 0; e < DPL; ++e) a.dq[row + e] = dq[hh][e];
  }
}

// Reverse index. Rows are taken in chunks of a.rchunk consecutive t. Step 1: how many rows of each
// chunk select each block (ccount [seg][chunk][block]).
__global__ void __launch_bounds__(256) rev_count_kernel(BackwardArgs a) {
  const long units = (long)a.batch * a.T * a.G;
  const long w = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= units) return;
  const int g = (int)(w % a.G);
  const long bt = w / a.G;
  const int t = (int)(bt % a.T);
  const long b = bt / a.T;
  const int32_t* srow = a.sel + w * a.Kb;
  int* cnt = a.ccount + ((b * a.G + g) * (long)a.nchunk + t / a.rchunk) * a.nblkc;
  for (int i = lane; i < a.Kb; i += 32) {
    const int j = __ldg(srow + i);
    if (j >= 0 && j <= t / a.B) atomicAdd(cnt + j, 1);
  }
}

// Step 2: per (seg, block), the exclusive prefix of the chunk counts (in place) and the total.
__global__ void __launch_bounds__(256) rev_chunk_scan_kernel(BackwardArgs a) {
  const long e = (long)blockIdx.x * blockDim.x + threadIdx.x;
  const long segs = (long)a.batch * a.G;
  if (e >= segs * a.nblkc) return;
  const long seg = e / a.nblkc;
  const int j = (int)(e % a.nblkc);
  int* col = a.ccount + seg * a.nchunk * (long)a.nblkc + j;
  int run = 0;
  for (int c = 0; c < a.nchunk; ++c) {
    const int v = col[(long)c * a.nblkc];
    col[(long)c * a.nblkc] = run;
    run += v;
  }
  a.rcount[seg * a.nblkc + j] = run;
}

// Step 3: exclusive scan of the totals of one (b, g) over the blocks (one CTA): the list offsets.
__global__ void __launch_bounds__(1024) rev_scan_kernel(BackwardArgs a) {
  __shared__ int warp_tot[32];
  __shared__ int carry;
  const long seg = blockIdx.x;
  const int* cnt = a.rcount + seg * a.nblkc;
  int* off = a.roff + seg * (a.nblkc + 1);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < a.nblkc; base += 1024) {
    const int i = base + threadIdx.x;
    const int v = i < a.nblkc ? cnt[i] : 0;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int w = warp_tot[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, w, o);
        if (lane >= o) w += y;
      }
      warp_tot[lane] = w;  // inclusive
    }
    __syncthreads();
    if (i < a.nblkc) off[i] = carry + (warp > 0 ? warp_tot[warp - 1] : 0) + x - v;
    __syncthreads();
    if (threadIdx.x == 0) carry += warp_tot[31];
    __syncthreads();
  }
  if (threadIdx.x == 0) off[a.nblkc] = carry;
}

// Step 4: one CTA per (seg, chunk) walks its rows in increasing t; the entries of one row name
// distinct blocks, so each block's chunk cursor moves by one thread per row; rows are separated
// by barriers. Row t lands at off[j] + (rows of earlier chunks) + (earlier rows of this chunk):
// every block's list is in increasing t.
__global__ void __launch_bounds__(512) rev_fill_kernel(BackwardArgs a) {
  const long seg = blockIdx.x / a.nchunk;
  const int chunk = (int)(blockIdx.x % a.nchunk);
  const long b = seg / a.G;
  const int g = (int)(seg % a.G);
  const int* off = a.roff + seg * (a.nblkc + 1);
  int* cur = a.ccount + (seg * a.nchunk + chunk) * (long)a.nblkc;
  int* list = a.rlist + seg * (long)a.T * a.Kb;  // this segment's slice
  const int t1 = min(a.T, (chunk + 1) * a.rchunk);
  for (int t = chunk * a.rchunk; t < t1; ++t) {
    const int32_t* srow = a.sel + ((b * a.T + t) * a.G + g) * (long)a.Kb;
    for (int i = threadIdx.x; i < a.Kb; i += blockDim.x) {
      const int j = __ldg(srow + i);
      if (j >= 0 && j <= t / a.B) {
        const int at = off[j] + cur[j]++;
        if (SGQA_CHECK(at < off[j + 1], a.status)) list[at] = t;  // inside the block's slice
      }
    }
    __syncthreads();
  }
}

// BKV: one CTA per (b, g, block j): TPT threads per token of the block, DPT head dims per thread.
template <int D, int B>
__global__ void __launch_bounds__(128) backward_kv_kernel(BackwardArgs a) {
  constexpr int TPT = 128 / B;  // threads per token (a power of two <= 32)
  constexpr int DPT = D / TPT;  // dims per thread
  static_assert(TPT <= 32 && DPT >= 1, "token groups within a warp");
  const int R = a.Hq / a.G;
  const long seg = blockIdx.x / a.nblkc;
  const int j = (int)(blockIdx.x % a.nblkc);
  const long b = seg / a.G;
  const int g = (int)(seg % a.G);
  const int ti = threadIdx.x / TPT, part = threadIdx.x % TPT;
  const int u = j * B + ti;
  const bool live = u < a.T;
  const int d0 = part * DPT;
  const float sc = 1.f / sqrtf((float)D);
  float kv[DPT], vv[DPT], dk[DPT], dv[DPT];
  const long kvrow = ((b * a.T + (live ? u : 0)) * a.G + g) * (long)D + d0;
#pragma unroll
  for (int e = 0; e < DPT; ++e) {
    kv[e] = live ? bf16_to_f32(a.k[kvrow + e]) : 0.f;
    vv[e] = live ? bf16_to_f32(a.v[kvrow + e]) : 0.f;
    dk[e] = dv[e] = 0.f;
  }
  const int* off = a.roff + seg * (a.nblkc + 1);
  const int* list = a.rlist + seg * (long)a.T * a.Kb;
  const int r0 = off[j], r1 = off[j + 1];
  for (int ri = r0; ri < r1; ++ri) {
    int t = __ldg(list + ri);
    if (!SGQA_CHECK(t >= 0 && t < a.T, a.status)) t = 0;  // a query position of the sequence
    const bool vis = live && u <= t;
    const long bt = b * a.T + t;
    for (int hr = 0; hr < R; ++hr) {
      const int h = g * R + hr;
      const long qrow = (bt * a.Hq + h) * D + d0;
      float qv[DPT], dov[DPT];
      float z = 0.f, dp = 0.f;
      if constexpr (DPT % 8 == 0) {  // 16-byte loads: 8 bf16 of q, 2 x 4 fp32 of do
#pragma unroll
        for (int c = 0; c < DPT / 8; ++c) {
          const uint4 w = __ldg(reinterpret_cast<const uint4*>(a.q + qrow) + c);
          const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            qv[8 * c + 2 * i] = bf16_lo(ww[i]);
            qv[8 * c + 2 * i + 1] = bf16_hi(ww[i]);
          }
          const float4 d0v = __ldg(reinterpret_cast<const float4*>(a.dov + qrow) + 2 * c);
          const float4 d1v = __ldg(reinterpret_cast<const float4*>(a.dov + qrow) + 2 * c + 1);
          dov[8 * c] = d0v.x; dov[8 * c + 1] = d0v.y; dov[8 * c + 2] = d0v.z; dov[8 * c + 3] = d0v.w;
          dov[8 * c + 4] = d1v.x; dov[8 * c + 5] = d1v.y; dov[8 * c + 6] = d1v.z; dov[8 * c + 7] = d1v.w;
        }
      } else {
#pragma unroll
        for (int e = 0; e < DPT; ++e) {
          qv[e] = bf16_to_f32(__ldg(a.q + qrow + e));
          dov[e] = __ldg(a.dov + qrow + e);
        }
      }
#pragma unroll
      for (int e = 0; e < DPT; ++e) {
        z = fmaf(qv[e], kv[e], z);
        dp = fmaf(dov[e], vv[e], dp);
      }
#pragma unroll
      for (int o = TPT / 2; o > 0; o >>= 1) {
        z += __shfl_xor_sync(0xFFFFFFFFu, z, o);
        dp += __shfl_xor_sync(0xFFFFFFFFu, dp, o);
      }
      const float p = vis ? expf(z * sc - __ldg(a.lse + bt * a.Hq + h)) : 0.f;
      const float dz = p * (dp - __ldg(a.dsum + bt * a.Hq + h)) * sc;
#pragma unroll
      for (int e = 0; e < DPT; ++e) {
        dk[e] = fmaf(dz, qv[e], dk[e]);
        dv[e] = fmaf(p, dov[e], dv[e]);
      }
    }
  }
  if (live) {
#pragma unroll
    for (int e = 0; e < DPT; ++e) {
      a.dk[kvrow + e] = dk[e];
      a.dv[kvrow + e] = dv[e];
    }
  }
}

template <int D>
cudaError_t launch_kv_d(const BackwardArgs& a, cudaStream_t s) {
  const unsigned grid = (unsigned)((long)a.batch * a.G * a.nblkc);
  switch (a.B) {
    case 4: backward_kv_kernel<D, 4><<<grid, 128, 0, s>>>(a); break;
    case 8: backward_kv_kernel<D, 8><<<grid, 128, 0, s>>>(a); break;
    case 16: backward_kv_kernel<D, 16><<<grid, 128, 0, s>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

bool backward_supported(int Hq, int G, int d, int B) {
  return (d == 64 || d == 128) && (B == 4 || B == 8 || B == 16) && Hq / G <= 16;
}

cudaError_t launch_backward(const BackwardArgs& a, cudaStream_t s) {
  const long units = (long)a.batch * a.T * a.G;
  const long segs = (long)a.batch * a.G;
  cudaError_t e;
  if ((e = cudaMemsetAsync(a.ccount, 0, (size_t)segs * a.nchunk * a.nblkc * sizeof(int), s)) != cudaSuccess)
    return e;
  // NT: a whole block of 4 or 8 tokens, or half of a 16-token block, per step
  if (a.d == 128) {
    if (a.B == 4) backward_q_kernel<128, 4><<<(unsigned)units, 128, 0, s>>>(a);
    else backward_q_kernel<128, 8><<<(unsigned)units, 128, 0, s>>>(a);
  } else {
    if (a.B == 4) backward_q_kernel<64, 4><<<(unsigned)units, 128, 0, s>>>(a);
    else backward_q_kernel<64, 8><<<(unsigned)units, 128, 0, s>>>(a);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  rev_count_kernel<<<(unsigned)((units * 32 + 255) / 256), 256, 0, s>>>(a);
  rev_chunk_scan_kernel<<<(unsigned)((segs * a.nblkc + 255) / 256), 256, 0, s>>>(a);
  rev_scan_kernel<<<(unsigned)segs, 1024, 0, s>>>(a);
  rev_fill_kernel<<<(unsigned)(segs * a.nchunk), 512, 0, s>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return a.d == 128 ? launch_kv_d<128>(a, s) : launch_kv_d<64>(a, s);
}

}  // namespace sgqa
