// K4 for decode on the 5th-generation tensor cores: indexer scores of the n_new * G rows of a
// decode step against every candidate block of a long cache.
//
// Step 5 Preview pages (mo.ai.kr, "Step 5 Preview agentic work design", section "model structure
// and training stability"): every KV group scores the compressed blocks of the shared index keys
// and keeps its top k/B; with a 1M-token cache (orcarouter.ai serving recipe, 1M context, four
// query tokens per step) a row has up to 131072 candidates, and the step streams every block mean
// of every sequence once. The contraction has few rows and many candidates, so the candidates are
// the MMA's M dimension:
//     D[128 candidates x NR] (fp32, TMEM) = (kbar_hi + kbar_lo)[128 x d_idx] . q_idx[NR x d_idx]^T
// with the rows of the sequence (row n = query n / G, group n % G) as the N columns (zero beyond
// n_new * G). kbar is fp32 in the cache; converter warps split each staged tile into bf16 planes
// hi = bf16(kbar), lo = bf16(kbar - hi) (the prefill indexer's operands), so the contraction runs
// at the bf16 tensor rate with fp32-accurate scores, hi products first, then lo, as in prefill.
//
// Pipeline (one CTA per (sequence, range of 128-candidate tiles)): warp 0 TMA-loads fp32 tiles
// (32 KB) into a 2-stage ring; warps 2-5 convert a staged tile into the two bf16 operand planes
// (128B-swizzled K-major); warp 1 allocates TMEM and issues the MMAs into two accumulators;
// warps 6-9 (one per TMEM lane quadrant, a candidate per lane) write each row's fp32
// scores for the candidates it has, and per row the largest order-preserving key of every 32
// consecutive candidates (a lower bound on the row's selection threshold comes from these). Two
// CTAs run per SM, so one's hand-offs overlap the other's work. Every
// wait is bounded by %globaltimer: on expiry the kernel records SGQA_ERR_TIMEOUT, drains its
// copies and MMAs, frees TMEM and returns.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace sgqa {
namespace {

constexpr int kCand = 128;                 // candidates per tile (MMA M)
constexpr int kDI = 64;                    // indexer dim of this kernel
constexpr int kStg = 2;                    // fp32 staging stages
constexpr int kNOp = 1;                    // bf16 operand buffers (hi + lo planes)
constexpr int kCtasPerSm = 2;              // two pipelines per SM hide each other's hand-offs
constexpr int kStgBytes = kCand * kDI * 4; // 32 KB
constexpr int kPlane = kCand * kDI * 2;    // one bf16 plane: 16 KB
constexpr int kOp = 2 * kPlane;            // hi then lo
constexpr int kConvWarps = 4;              // converter warps (2 .. 5); epilogue warps 6 .. 9
constexpr int kThr = (2 + kConvWarps + 4) * 32;

struct ScShared {
  uint64_t full[kStg], empty[kStg], op_full[kNOp], op_empty[kNOp], acc_full[2], acc_empty[2];
  uint32_t tmem;
  volatile int abort_flag;
};

template <int NR>
struct ScCfg {
  static constexpr int kQ = NR * 128;
  static constexpr int kSmem = 1024 + kStg * kStgBytes + kNOp * kOp + kQ + (int)sizeof(ScShared) + 64;
  static_assert(kCtasPerSm * (kSmem + 1024) <= 233472, "shared memory of the resident CTAs");
};

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, const int* gstatus) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = tc::mbar_wait(bar, parity, abort, gstatus) ? 1 : 0;
  return __shfl_sync(0xFFFFFFFFu, ok, 0) != 0;
}

template <int NR>
__global__ void __launch_bounds__(kThr, kCtasPerSm)
    decode_scores_tc_kernel(const __grid_constant__ CUtensorMap map_kbar, DecodeScoreArgs a) {
  using C = ScCfg<NR>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align<1024>(smem_raw);
  uint8_t* sStg = smem;
  uint8_t* sOp = sStg + kStg * kStgBytes;  // [kNOp][hi | lo]
  uint8_t* sQ = sOp + kNOp * kOp;
  ScShared* sh = reinterpret_cast<ScShared*>(sQ + C::kQ);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.x / a.cps, cta = blockIdx.x % a.cps;
  const int rows = a.n_new * a.G;
  const int c_max = (a.t0 + a.n_new - 1) / a.B;  // candidates of the last new token
  const int ntile = (c_max + kCand - 1) / kCand;
  const int tpc = (ntile + a.cps - 1) / a.cps;
  const int i0 = min(ntile, cta * tpc), i1 = min(ntile, i0 + tpc);
  const int n = i1 - i0;

  // a timeout recorded by another CTA (this launch or an earlier one sharing the status word):
  // do nothing (the decision is the CTA's, before any barrier or TMEM is set up)
  if (__syncthreads_or(tid == 0 && tc::grid_timed_out(a.status))) return;
  if (tid == 0) {
    for (int s = 0; s < kStg; ++s) {
      tc::mbar_init(&sh->full[s], 1);
      tc::mbar_init(&sh->empty[s], kConvWarps);
    }
    for (int s = 0; s < kNOp; ++s) {
      tc::mbar_init(&sh->op_full[s], kConvWarps);
      tc::mbar_init(&sh->op_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&sh->acc_full[s], 1);
      tc::mbar_init(&sh->acc_empty[s], 4);
    }
    sh->abort_flag = 0;
    tc::fence_mbar_init();
  }
  // q_idx rows of the sequence: 16-byte chunk c of row r at r * 128 + ((c ^ (r & 7)) * 16)
  for (int idx = tid; idx < NR * 8; idx += kThr) {
    const int r = idx >> 3, c = idx & 7;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < rows) v = __ldg(reinterpret_cast<const uint4*>(a.qidx + ((long)b * rows + r) * kDI) + c);
    *reinterpret_cast<uint4*>(sQ + r * 128 + ((c ^ (r & 7)) * 16)) = v;
  }
  if (warp == 1) tc::tmem_alloc(&sh->tmem, 64);
  tc::fence_proxy_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = sh->tmem;

  if (warp == 0) {
    if (lane == 0 && n > 0) {
      tc::prefetch_tensormap(&map_kbar);
      int k = 0;
      for (; k < n && !sh->abort_flag; ++k) {
        const int st = k % kStg;
        if (k >= kStg && !tc::mbar_wait(&sh->empty[st], (uint32_t)(((k / kStg) - 1) & 1), &sh->abort_flag, a.status)) {
          if (!sh->abort_flag) report(a.status, SGQA_ERR_TIMEOUT);
          sh->abort_flag = 1;
          break;
        }
        tc::mbar_arrive_expect_tx(&sh->full[st], kStgBytes);
        tc::tma_load_2d(sStg + st * kStgBytes, &map_kbar, &sh->full[st], 0, b * a.nblk + (i0 + k) * kCand);
      }
      for (int kk = k - kStg; kk < k; ++kk) {  // the last copies land before the CTA exits
        if (kk < 0) continue;
        volatile int no_abort = 0;
        tc::mbar_wait(&sh->full[kk % kStg], (uint32_t)((kk / kStg) & 1), &no_abort);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && n > 0) {
      const uint32_t idesc = tc::idesc_bf16_f32(kCand, NR);
      int k = 0;
      for (; k < n && !sh->abort_flag; ++k) {
        const int op = k % kNOp, ab = k & 1;
        if (!tc::mbar_wait(&sh->op_full[op], (uint32_t)((k / kNOp) & 1), &sh->abort_flag, a.status) ||
            (k >= 2 && !tc::mbar_wait(&sh->acc_empty[ab], (uint32_t)(((k >> 1) - 1) & 1), &sh->abort_flag, a.status))) {
          if (!sh->abort_flag) report(a.status, SGQA_ERR_TIMEOUT);
          sh->abort_flag = 1;
          break;
        }
        tc::fence_after_sync();
        const uint8_t* hi = sOp + op * kOp;
        const uint32_t d = tmem + (uint32_t)(ab * NR);
#pragma unroll
        for (int kk = 0; kk < kDI / 16; ++kk)
          tc::mma_bf16_ss(d, tc::smem_desc_kmajor(hi + kk * 32, 128), tc::smem_desc_kmajor(sQ + kk * 32, 128), idesc,
                          kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < kDI / 16; ++kk)
          tc::mma_bf16_ss(d, tc::smem_desc_kmajor(hi + kPlane + kk * 32, 128), tc::smem_desc_kmajor(sQ + kk * 32, 128),
                          idesc, 1u);
        tc::mma_commit(&sh->op_empty[op]);
        tc::mma_commit(&sh->acc_full[ab]);
      }
      if (k > 0) {  // the last MMAs complete before TMEM is freed
        volatile int no_abort = 0;
        tc::mbar_wait(&sh->acc_full[(k - 1) & 1], (uint32_t)(((k - 1) >> 1) & 1), &no_abort);
      }
    }
  } else if (warp < 2 + kConvWarps) {
    // ---- converters: fp32 tile -> bf16 hi and lo planes (128B-swizzled K-major rows) ----
    const int ct = tid - 64;
    for (int k = 0; k < n; ++k) {
      const int st = k % kStg, op = k % kNOp;
      if (!warp_wait(&sh->full[st], (uint32_t)((k / kStg) & 1), &sh->abort_flag, a.status) ||
          (k >= kNOp && !warp_wait(&sh->op_empty[op], (uint32_t)(((k / kNOp) - 1) & 1), &sh->abort_flag, a.status))) {
        if (lane == 0 && !sh->abort_flag) report(a.status, SGQA_ERR_TIMEOUT);
        sh->abort_flag = 1;
        break;
      }
      const float4* src = reinterpret_cast<const float4*>(sStg + st * kStgBytes);
      uint8_t* hi = sOp + op * kOp;
#pragma unroll
      for (int e = 0; e < kCand * kDI / 4 / (32 * kConvWarps); ++e) {
        const int idx = ct + 32 * kConvWarps * e;
        const int row = idx >> 4, c4 = idx & 15;
        const float4 f = src[idx];
        // hi = bf16(x) two at a time; lo = bf16(x - hi), where x - hi is exact in fp32
        const uint32_t h01 = pack_bf16x2(f.x, f.y), h23 = pack_bf16x2(f.z, f.w);
        const uint32_t l01 = pack_bf16x2(f.x - bf16_lo(h01), f.y - bf16_hi(h01));
        const uint32_t l23 = pack_bf16x2(f.z - bf16_lo(h23), f.w - bf16_hi(h23));
        const int off = row * 128 + (((c4 >> 1) ^ (row & 7)) * 16) + (c4 & 1) * 8;
        *reinterpret_cast<uint2*>(hi + off) = make_uint2(h01, h23);
        *reinterpret_cast<uint2*>(hi + kPlane + off) = make_uint2(l01, l23);
      }
      tc::fence_proxy_async();
      __syncwarp();
      if (lane == 0) {
        tc::mbar_arrive(&sh->empty[st]);
        tc::mbar_arrive(&sh->op_full[op]);
      }
    }
  } else {
    // ---- epilogue: thread = candidate (TMEM lane) of the tile ----
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_base = (uint32_t)(32 * quad) << 16;
    // per row: the own block (candidates are j < c_row), hoisted out of the tile loop
    int c_row[NR];
#pragma unroll
    for (int rr = 0; rr < NR; ++rr) c_row[rr] = rr < rows ? (a.t0 + rr / a.G) / a.B : 0;
    float* sbase = a.scores + (long)b * rows * a.nblk;
    uint32_t* tbase = a.tmax + (long)b * rows * a.tstride;
    for (int k = 0; k < n; ++k) {
      const int acc = k & 1;
      if (!warp_wait(&sh->acc_full[acc], (uint32_t)((k >> 1) & 1), &sh->abort_flag, a.status)) {
        if (lane == 0 && !sh->abort_flag) report(a.status, SGQA_ERR_TIMEOUT);
        sh->abort_flag = 1;
        break;
      }
      tc::fence_after_sync();
      uint32_t v[NR];
      if constexpr (NR == 16) tc::tmem_ld16(tmem + lane_base + (uint32_t)(acc * NR), v);
      else tc::tmem_ld32(tmem + lane_base + (uint32_t)(acc * NR), v);
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&sh->acc_empty[acc]);
      const int j = (i0 + k) * kCand + r;
      const int j_warp = j - lane;
      if (j_warp >= c_max) continue;  // warp-uniform
      const bool in_range = j < c_max;
#pragma unroll
      for (int rr = 0; rr < NR; ++rr) {
        if (rr >= rows) break;
        const float s = __uint_as_float(v[rr]);
        if (in_range) sbase[rr * a.nblk + j] = s;
        const uint32_t wmax = __reduce_max_sync(0xFFFFFFFFu, j < c_row[rr] ? score_key(s) : 0u);
        if (lane == 0) tbase[rr * a.tstride + (j_warp >> 5)] = wmax;
      }
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 64);
  }
}

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled get_encode() {
  static EncodeTiled fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(p);
  }
  return fn;
}

// 2-D map over kbar [rows = batch * nblk][64] fp32: box = 64 x 128 rows (one tile, 32 KB).
bool make_kbar_map(CUtensorMap* map, const float* kbar, long rows) {
  EncodeTiled enc = get_encode();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)kDI, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)kDI * 4};
  const cuuint32_t box[2] = {(cuuint32_t)kDI, (cuuint32_t)kCand};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(kbar), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NR>
cudaError_t launch_nr(const DecodeScoreArgs& a, cudaStream_t s) {
  using C = ScCfg<NR>;
  CUtensorMap m;
  if (!make_kbar_map(&m, a.kbar, (long)a.batch * a.nblk)) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(decode_scores_tc_kernel<NR>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  decode_scores_tc_kernel<NR><<<(unsigned)(a.batch * a.cps), kThr, C::kSmem, s>>>(m, a);
  return cudaGetLastError();
}

}  // namespace

bool decode_scores_tc_supported(int d_idx, int n_new, int G) { return d_idx == kDI && n_new * G <= 32; }

int decode_scores_ctas(int batch, int c_max) {
  // two CTAs per SM, one wave over all sequences
  const int ntile = (c_max + kCand - 1) / kCand;
  int cps = kCtasPerSm * 148 / (batch > 0 ? batch : 1);
  if (cps > ntile) cps = ntile;
  if (cps < 1) cps = 1;
  return cps;
}

cudaError_t launch_decode_scores_tc(const DecodeScoreArgs& a, cudaStream_t s) {
  const int c_max = (a.t0 + a.n_new - 1) / a.B;
  if (c_max <= 0) return cudaSuccess;
  if ((uintptr_t)a.kbar & 15u) return cudaErrorInvalidValue;
  return a.n_new * a.G <= 16 ? launch_nr<16>(a, s) : launch_nr<32>(a, s);
}

}  // namespace sgqa
