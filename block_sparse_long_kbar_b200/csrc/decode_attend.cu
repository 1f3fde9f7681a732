// K6 for decode on the 5th-generation tensor cores: gated attention of the few new query tokens of
// a decode step over their selected blocks of a long KV cache.
//
// A decode step (orcarouter.ai, "Step 5 Preview NVFP4 checkpoint", serving recipe: 1M-token
// context, MTP with three speculative tokens, so four query tokens per step) attends, for every
// (sequence, KV group), n_new queries x R heads to the blocks each query selected (mo.ai.kr, "Step
// 5 Preview agentic work design", section "model structure and training stability": every KV group
// attends only to its own selected blocks). The queries of one (sequence, group) share most of
// their context, so the kernel streams the UNION of their selections once: that is the HBM stream
// this step is bound by.
//
// Roles of the tensor-core contraction are the transpose of the prefill kernel's, because a decode
// tile has many tokens and few query rows:
//   S^T[128 tokens x 64 columns] = K_tile[128 x d] . Q[64 x d]^T       (tcgen05, M = 128 tokens)
//   O^T[d x 64]                 += V_tile^T[d x 128] . P^T[128 x 64]    (tcgen05, A = V MN-major)
//   l[64]                       += 1[128 x 128] . P^T                   (row sums of the same bf16 P)
// Column n is query n / R, head n % R of the group (n_new * R <= 64 columns; the rest are zero).
// Every probability is taken against a per-column reference maximum computed up front from the
// query's own block (always selected), so there is no rescaling of O^T: a column whose sum of P
// exceeds 2^60 or is not finite makes the CTA stream its tiles again for exact maxima and repeat
// the main pass. The union of a (sequence, group) is split over `splits` CTAs, each writing a
// partial (m, l, O) that a fixed-order merge combines (one CTA per (sequence, group) writes the
// output directly when splits == 1).
//
// Data movement: K and V tiles of 128 token slots (128/B whole blocks of the union) arrive by 3-D
// TMA boxes (64 dims x 1 group x B tokens, 128B swizzle) into one K and one V stage per CTA, two
// CTAs per SM; slots past the union are loaded from out of bounds (zero fill) and masked. Warp roles: warp 0 issues TMA, warp
// 1 allocates TMEM and issues MMAs, warps 2-5 (one per TMEM lane quadrant: a token slot per lane,
// later a head dimension per lane) compute P and the epilogue. Every wait is bounded by
// %globaltimer: on expiry the kernel records SGQA_ERR_TIMEOUT, drains its copies and MMAs, frees
// TMEM and returns.
#include <cmath>
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace sgqa {
namespace {

constexpr int kTok = 128;                 // token slots per tile
constexpr int kNQ = 64;                   // query-head columns
constexpr int kD = 128;                   // head dim of this kernel
constexpr int kNK = 1;                    // bf16 caches: K tile stages (free once S^T is issued)
constexpr int kNV = 1;                    // bf16 caches: V tile stages (free once P V is issued)
constexpr int kSmWarps = 4;
constexpr int kThreads = (2 + kSmWarps) * 32;
constexpr int kHalf = kTok * 128;         // one 64-dim half of a K or V tile: [128 tokens][128 B]
constexpr int kKV = 2 * kHalf;            // K (or V) of one tile
constexpr int kStage = 2 * kKV;           // K then V
constexpr int kQ = 2 * kNQ * 128;         // Q: [half][64 columns][128 B]
constexpr int kP = kTok * 128;            // P^T: [128 tokens][64 columns] bf16, 128B swizzle
constexpr int kOnes = 16 * 256;           // 128 x 16 bf16 ones (K-major core matrices)
constexpr int kTmemCols = 256;            // S^T x 2, O^T, l: 64 columns each
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRiskSum = 1.152921504606846976e18f;  // 2^60

constexpr int kS8 = 3;                    // fp8 caches: staging stages of 8-bit K and V rows
constexpr int kRow8 = kTok * 128;         // 8-bit K (or V) of one tile: [128 tokens][128 B]
constexpr int kThreads8 = (2 + kSmWarps + 4) * 32;  // fp8 caches: + 4 converter warps

struct DecShared {
  // bf16 caches: kf / ke per K stage and vf / ve per V stage (TMA into the operand tiles). fp8
  // caches: st8_full / st8_empty per staging stage (TMA), k_full / k_empty and v_full / v_empty
  // for the single K and V operand tiles (converter warps write them).
  uint64_t kf[kNK], ke[kNK], vf[kNV], ve[kNV], st8_full[kS8], st8_empty[kS8], k_full, k_empty, v_full, v_empty;
  uint64_t s_full[2], s_empty[2], p_full[2], p_empty[2], o_done;
  uint32_t tmem;
  volatile int abort_flag;
  float base[kNQ];         // reference maximum of each column, times the exp2 scale
  float ref_part[2][kNQ];  // the own block's maxima, two halves of its tokens
  uint32_t maxkey[kNQ];    // exact maxima (order-preserving keys) for the fallback pass
};
// operand tiles (bf16: the K ring, then the V ring; fp8: one K and one V tile) then, for fp8
// caches, the staging ring
// bf16 caches: two CTAs per SM, each with one K stage, one V stage and one P buffer (about 102 KB
// of shared memory), so that one CTA's hand-offs overlap the other's work; fp8 caches: one CTA
// per SM with the staging ring and two P buffers.
template <bool F8>
struct DaCfg {
  static constexpr int kRingK = kNK;           // K stages (bf16 caches only)
  static constexpr int kRingV = kNV;           // V stages (bf16 caches only)
  static constexpr int kPB = F8 ? 2 : 1;       // P buffers
  static constexpr int kCtas = F8 ? 1 : 2;     // CTAs per SM
  static constexpr int kOps = F8 ? kStage : (kRingK + kRingV) * kKV;
  static constexpr int kStaging = F8 ? kS8 * 2 * kRow8 : 0;
  static constexpr int kSmem = 1024 + kQ + kOps + kStaging + kPB * kP + kOnes + (int)sizeof(DecShared) + 64;
  static constexpr int kThr = F8 ? kThreads8 : kThreads;
  static_assert(kCtas * (kSmem + 1024) <= 233472, "shared memory of the resident CTAs");
  static_assert(kCtas * kTmemCols <= 512, "TMEM of the resident CTAs");
};

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, const int* gstatus) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = tc::mbar_wait(bar, parity, abort, gstatus) ? 1 : 0;
  return __shfl_sync(0xFFFFFFFFu, ok, 0) != 0;
}

__device__ __forceinline__ float key_to_score(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Instruction descriptor, kind::f16, BF16 x BF16 -> F32, M x N, with the A and/or B operand
// MN-major.
__host__ __device__ constexpr uint32_t idesc_mn(int M, int N, bool a_mn, bool b_mn) {
  return tc::idesc_bf16_f32(M, N, b_mn) | (a_mn ? (1u << 15) : 0u);
}

// Four E4M3 codes (one 32-bit word) times a power-of-two scale as four bf16 (exact: a code has at
// most 4 significant bits), packed two per word.
__device__ __forceinline__ uint2 e4m3x4_to_bf16(uint32_t w, float scale) {
  const __half2_raw h01 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w & 0xFFFFu), __NV_E4M3);
  const __half2_raw h23 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w >> 16), __NV_E4M3);
  const float2 f01 = __half22float2(*reinterpret_cast<const __half2*>(&h01));
  const float2 f23 = __half22float2(*reinterpret_cast<const __half2*>(&h23));
  return make_uint2(pack_bf16x2(f01.x * scale, f01.y * scale), pack_bf16x2(f23.x * scale, f23.y * scale));
}

template <int B, bool F8>
__global__ void __launch_bounds__(DaCfg<F8>::kThr, DaCfg<F8>::kCtas)
    decode_attend_tc_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                            DecodeAttendArgs a) {
  using C = DaCfg<F8>;
  constexpr int NB = kTok / B;  // whole blocks per tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align<1024>(smem_raw);
  uint8_t* sQ = smem;
  uint8_t* sKV = sQ + kQ;  // [stage][K|V][half][128 tokens][128 B] (one stage for fp8 caches)
  uint8_t* s8 = sKV + C::kOps;  // fp8: [stage][K|V][128 tokens][128 B], 128B swizzle
  uint8_t* sP = s8 + C::kStaging;
  uint8_t* sOnes = sP + C::kPB * kP;
  DecShared* sh = reinterpret_cast<DecShared*>(sOnes + kOnes);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int unit = blockIdx.x / a.splits, split = blockIdx.x % a.splits;
  const int b = unit / a.G, g = unit % a.G;
  const int R = a.Hq / a.G;
  const int NQ = a.n_new * R;
  const int count = __ldg(a.ucount + unit);
  const int ntile = (count + NB - 1) / NB;
  const int tps = (ntile + a.splits - 1) / a.splits;
  const int tile0 = min(ntile, split * tps), tile1 = min(ntile, tile0 + tps);
  const int32_t* ublk = a.ublk + (long)unit * a.ucap;
  const uint32_t* umask = a.umask + (long)unit * a.ucap;
  const float sc = kLog2e / sqrtf((float)kD);

  // a timeout recorded by another CTA (this launch or an earlier one sharing the status word):
  // do nothing (the decision is the CTA's, before any barrier or TMEM is set up)
  if (__syncthreads_or(tid == 0 && tc::grid_timed_out(a.status))) return;
  if (tid == 0) {
    for (int i = 0; i < C::kRingK; ++i) {
      tc::mbar_init(&sh->kf[i], 1);
      tc::mbar_init(&sh->ke[i], 1);
    }
    for (int i = 0; i < C::kRingV; ++i) {
      tc::mbar_init(&sh->vf[i], 1);
      tc::mbar_init(&sh->ve[i], 1);
    }
    for (int i = 0; i < kS8; ++i) {
      tc::mbar_init(&sh->st8_full[i], 1);
      tc::mbar_init(&sh->st8_empty[i], 4);
    }
    tc::mbar_init(&sh->k_full, 4);
    tc::mbar_init(&sh->k_empty, 1);
    tc::mbar_init(&sh->v_full, 4);
    tc::mbar_init(&sh->v_empty, 1);
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&sh->s_full[i], 1);
      tc::mbar_init(&sh->s_empty[i], kSmWarps);
    }
    for (int i = 0; i < C::kPB; ++i) {
      tc::mbar_init(&sh->p_full[i], kSmWarps);
      tc::mbar_init(&sh->p_empty[i], 1);
    }
    tc::mbar_init(&sh->o_done, 1);
    sh->abort_flag = 0;
    tc::fence_mbar_init();
  }
  // P buffers start at zero (columns >= NQ are never written), the ones tile is constant
  for (int i = tid; i < C::kPB * kP / 16; i += C::kThr) reinterpret_cast<uint4*>(sP)[i] = make_uint4(0, 0, 0, 0);
  for (int i = tid; i < kOnes / 4; i += C::kThr) reinterpret_cast<uint32_t*>(sOnes)[i] = 0x3F803F80u;
  if (tid < kNQ) sh->maxkey[tid] = 0u;
  // Q columns: n = query * R + head (zero beyond NQ); 16-byte chunk c of half h of column n at
  // h * 8 KB + n * 128 + ((c ^ (n & 7)) * 16) (128B-swizzled K-major)
  for (int idx = tid; idx < kNQ * (kD / 8); idx += C::kThr) {
    const int n = idx / (kD / 8), cc = idx % (kD / 8);
    const int h = cc >> 3, c = cc & 7;
    const bool live = n < NQ;
    const long row = live ? ((long)b * a.n_new + n / R) * a.Hq + (long)g * R + (n % R) : 0;
    cp_async16(smem_u32(sQ + h * (kNQ * 128) + n * 128 + ((c ^ (n & 7)) * 16)), a.q + row * kD + cc * 8,
               live ? 16 : 0);
  }
  cp_async_commit();
  if (warp == 1) tc::tmem_alloc(&sh->tmem, kTmemCols);
  cp_async_wait<0>();
  tc::fence_proxy_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = sh->tmem;
  const uint32_t tmem_o = tmem + 128;
  const uint32_t tmem_l = tmem + 192;

  const bool is_sm = warp >= 2 && warp < 2 + kSmWarps;
  // reference maximum of every column: the query's scores against its own block's tokens
  // (always selected, u <= t), on the CUDA cores from the same K values the tensor cores see
  if (is_sm) {
    const int i = tid - 64;
    const int n = i & (kNQ - 1), part = i >> 6;
    float mx = -INFINITY;
    if (n < NQ) {
      const int tq = a.t0 + n / R;
      const uint8_t* qrow = sQ + n * 128;
      for (int u = (tq / B) * B + part; u <= tq; u += 2) {
        const long krow_i = ((long)b * a.T_kv + u) * a.G + g;
        float acc = 0.f;
        if constexpr (F8) {
          const float ks = __ldg(a.k_scale + krow_i);
          const uint8_t* krow = a.k8 + krow_i * kD;
#pragma unroll
          for (int cc = 0; cc < kD / 16; ++cc) {
            const uint4 kv = __ldg(reinterpret_cast<const uint4*>(krow + cc * 16));
            const uint32_t kw8[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const int c8 = 2 * cc + hh;  // 16-byte chunk of bf16 values (8 dims)
              const int h = c8 >> 3, c = c8 & 7;
              const uint4 qv = *reinterpret_cast<const uint4*>(qrow + h * (kNQ * 128) + ((c ^ (n & 7)) * 16));
              const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
              const uint2 k01 = e4m3x4_to_bf16(kw8[2 * hh], ks), k23 = e4m3x4_to_bf16(kw8[2 * hh + 1], ks);
              const uint32_t kw[4] = {k01.x, k01.y, k23.x, k23.y};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                acc = fmaf(bf16_lo(qw[e]), bf16_lo(kw[e]), acc);
                acc = fmaf(bf16_hi(qw[e]), bf16_hi(kw[e]), acc);
              }
            }
          }
        } else {
          const uint16_t* krow = a.k + krow_i * kD;
#pragma unroll
          for (int cc = 0; cc < kD / 8; ++cc) {
            const int h = cc >> 3, c = cc & 7;
            const uint4 qv = *reinterpret_cast<const uint4*>(qrow + h * (kNQ * 128) + ((c ^ (n & 7)) * 16));
            const uint4 kv = __ldg(reinterpret_cast<const uint4*>(krow + cc * 8));
            const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w}, kw[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              acc = fmaf(bf16_lo(qw[e]), bf16_lo(kw[e]), acc);
              acc = fmaf(bf16_hi(qw[e]), bf16_hi(kw[e]), acc);
            }
          }
        }
        mx = fmaxf(mx, acc);
      }
    }
    sh->ref_part[part][n] = mx;
  }
  __syncthreads();
  if (tid < kNQ) {
    const float m = fmaxf(sh->ref_part[0][tid], sh->ref_part[1][tid]);
    sh->base[tid] = m == -INFINITY ? 0.f : m * sc;
  }
  __syncthreads();

  const int quad = warp & 3;
  const uint32_t lane_base = (uint32_t)(32 * quad) << 16;
  const int r = quad * 32 + lane;  // token slot (softmax, converters) / head dim (epilogue) of this thread
  const uint32_t idesc_s = tc::idesc_bf16_f32(kTok, kNQ);
  const uint32_t idesc_o = idesc_mn(kD, kNQ, true, true);
  const uint32_t idesc_l = idesc_mn(kTok, kNQ, false, true);
  const uint64_t d_ones = tc::smem_desc_kmajor_noswz(sOnes, 128, 256);
  long kc = 0, vc = 0, scnt = 0, pcnt = 0;  // tiles, V tiles (fp8), S and P buffer uses
  bool rerun = false, any_pv = false, o_ok = false;
  int o_commits = 0, o_phase = 0;

  for (int pass = 0; pass < 3; ++pass) {
    if (pass == 1 && !rerun) break;
    const bool main_pass = pass != 1;
    if (pass == 2) {
      // the columns' exact maxima over this CTA's tiles replace the reference maxima
      if (tid < kNQ && sh->maxkey[tid] != 0u) sh->base[tid] = key_to_score(sh->maxkey[tid]) * sc;
      __syncthreads();
    }
    if (warp == 0) {
      // ---- TMA producer: the tile's blocks of the union (out of bounds past it: zero fill) ----
      // (a CTA named by the failure-detection test hook issues nothing: its issuer's first wait
      // then runs out, with no copy in flight)
      if (lane == 0 && (int)blockIdx.x != a.stall_cta) {
        // the tile's token coordinates, loaded together before any copy is issued
        auto coords = [&](int i, int (&zs)[NB]) {
#pragma unroll
          for (int e = 0; e < NB; ++e) {
            const int idx = i * NB + e;
            zs[e] = idx < count ? b * a.T_kv + __ldg(ublk + idx) * B : 0x7FFFFFF0;
          }
        };
        auto fail = [&]() {
          if (!sh->abort_flag) report(a.status, SGQA_ERR_TIMEOUT);
          sh->abort_flag = 1;
        };
        if constexpr (F8) {
          for (int i = tile0; i < tile1 && !sh->abort_flag; ++i, ++kc) {
            const int st = (int)(kc % kS8);
            if (kc >= kS8 &&
                !tc::mbar_wait(&sh->st8_empty[st], (uint32_t)(((kc / kS8) - 1) & 1), &sh->abort_flag, a.status)) {
              fail();
              break;
            }
            int zs[NB];
            coords(i, zs);
            uint64_t* ful = &sh->st8_full[st];
            uint8_t* dst = s8 + st * 2 * kRow8;
            tc::mbar_arrive_expect_tx(ful, main_pass ? 2 * kRow8 : kRow8);
#pragma unroll
            for (int e = 0; e < NB; ++e) {
              tc::tma_load_3d(dst + e * (B * 128), &map_k, ful, 0, g, zs[e]);
              if (main_pass) tc::tma_load_3d(dst + kRow8 + e * (B * 128), &map_v, ful, 0, g, zs[e]);
            }
          }
        } else {
          // K of tile i, then V of tile i - 1: a K stage frees as soon as its S^T is issued, so
          // K runs up to three tiles ahead while V waits for the P V two tiles back
          int zk[NB], zv[NB];
          for (int i = tile0; i <= tile1 && !sh->abort_flag; ++i) {
            if (i < tile1) {
              const int st = (int)(kc % C::kRingK);
              if (kc >= C::kRingK && !tc::mbar_wait(&sh->ke[st], (uint32_t)(((kc / C::kRingK) - 1) & 1), &sh->abort_flag, a.status)) {
                fail();
                break;
              }
              coords(i, zk);
              uint8_t* dst = sKV + st * kKV;
              tc::mbar_arrive_expect_tx(&sh->kf[st], kKV);
#pragma unroll
              for (int e = 0; e < NB; ++e)
#pragma unroll
                for (int h = 0; h < 2; ++h) tc::tma_load_3d(dst + h * kHalf + e * (B * 128), &map_k, &sh->kf[st], h * 64, g, zk[e]);
              ++kc;
            }
            if (main_pass && i > tile0) {
              const int st = (int)(vc % C::kRingV);
              if (vc >= C::kRingV && !tc::mbar_wait(&sh->ve[st], (uint32_t)(((vc / C::kRingV) - 1) & 1), &sh->abort_flag, a.status)) {
                fail();
                break;
              }
              uint8_t* dst = sKV + C::kRingK * kKV + st * kKV;
              tc::mbar_arrive_expect_tx(&sh->vf[st], kKV);
#pragma unroll
              for (int e = 0; e < NB; ++e)
#pragma unroll
                for (int h = 0; h < 2; ++h) tc::tma_load_3d(dst + h * kHalf + e * (B * 128), &map_v, &sh->vf[st], h * 64, g, zv[e]);
              ++vc;
            }
#pragma unroll
            for (int e = 0; e < NB; ++e) zv[e] = zk[e];
          }
        }
      }
    } else if (warp == 1) {
      // ---- MMA issuer ----
      if (lane == 0) {
        long pend = -1;
        bool first = true;
        auto issue_pv = [&](long) -> bool {
          const int pb = (int)(pcnt % C::kPB);
          if (!tc::mbar_wait(&sh->p_full[pb], (uint32_t)((pcnt / C::kPB) & 1), &sh->abort_flag, a.status)) return false;
          if (F8 ? !tc::mbar_wait(&sh->v_full, (uint32_t)(vc & 1), &sh->abort_flag, a.status)
                 : !tc::mbar_wait(&sh->vf[vc % C::kRingV], (uint32_t)((vc / C::kRingV) & 1), &sh->abort_flag, a.status))
            return false;
          tc::fence_after_sync();
          const uint8_t* vbase = F8 ? sKV + kKV : sKV + C::kRingK * kKV + (vc % C::kRingV) * kKV;
          const uint8_t* pbase = sP + pb * kP;
#pragma unroll
          for (int kk = 0; kk < kTok / 16; ++kk) {
            const uint64_t da = tc::smem_desc_mnmajor_sw128(vbase + kk * 2048, kHalf, 1024);
            const uint64_t db = tc::smem_desc_mnmajor_sw128(pbase + kk * 2048, kP, 1024);
            const uint32_t acc = first ? 0u : 1u;
            tc::mma_bf16_ss(tmem_o, da, db, idesc_o, acc);
            tc::mma_bf16_ss(tmem_l, d_ones, db, idesc_l, acc);
            first = false;
          }
          tc::mma_commit(F8 ? &sh->v_empty : &sh->ve[vc % C::kRingV]);
          ++vc;
          tc::mma_commit(&sh->p_empty[pb]);
          ++pcnt;
          return true;
        };
        bool ok = true;
        for (int i = tile0; i < tile1 && ok && !sh->abort_flag; ++i, ++kc, ++scnt) {
          const int st = F8 ? 0 : (int)(kc % C::kRingK);
          const int sb = (int)(scnt & 1);
          uint64_t* kfull = F8 ? &sh->k_full : &sh->kf[st];
          const uint32_t kpar = F8 ? (uint32_t)(kc & 1) : (uint32_t)((kc / C::kRingK) & 1);
          if (!tc::mbar_wait(kfull, kpar, &sh->abort_flag, a.status) ||
              (scnt >= 2 && !tc::mbar_wait(&sh->s_empty[sb], (uint32_t)(((scnt >> 1) - 1) & 1), &sh->abort_flag, a.status))) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint8_t* kst = sKV + st * kKV;
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const int h = kk >> 2, off = (kk & 3) * 32;
            const uint64_t da = tc::smem_desc_kmajor(kst + h * kHalf + off, 128);
            const uint64_t db = tc::smem_desc_kmajor(sQ + h * (kNQ * 128) + off, 128);
            tc::mma_bf16_ss(tmem + (uint32_t)(sb * kNQ), da, db, idesc_s, kk > 0 ? 1u : 0u);
          }
          tc::mma_commit(&sh->s_full[sb]);
          tc::mma_commit(F8 ? &sh->k_empty : &sh->ke[st]);  // the K tile is free once S^T is computed
          if (main_pass) {
            if (pend >= 0 && !issue_pv(pend)) { ok = false; break; }
            pend = kc;
          }
        }
        if (ok && main_pass && pend >= 0 && !sh->abort_flag) ok = issue_pv(pend);
        if (!ok) {
          if (!sh->abort_flag) report(a.status, SGQA_ERR_TIMEOUT);
          sh->abort_flag = 1;
        }
      }
    } else if (!is_sm) {
      // ---- fp8 converters: thread = token slot r; the staged 8-bit rows times their row
      // scales into the bf16 K and V operand tiles (exact). K runs one tile ahead of V: K(i+1)
      // needs only S^T(i) to be done with the K tile, V(i) needs P V(i-1), so the next S^T
      // overlaps this tile's softmax. ----
      if constexpr (F8) {
        const int e = r / B;
        const long st_base = kc;  // staging uses before this pass
        // (row of the cache, K scale, V scale) of a tile's token slot r
        auto meta = [&](int i, long& srow, float& ks, float& vs) {
          const int idx = i * NB + e;
          srow = -1;
          if (i < tile1 && idx < count) {
            // tokens of a partial last block past the cache capacity do not exist (their slots
            // are masked): no scale is read for them
            const int blk = __ldg(ublk + idx);
            const int u = blk * B + (r % B);
            if (SGQA_CHECK(blk >= 0 && blk * B < a.T_kv, a.status) && u < a.T_kv) srow = ((long)b * a.T_kv + u) * a.G + g;
          }
          ks = srow >= 0 ? __ldg(a.k_scale + srow) : 0.f;
          vs = (srow >= 0 && main_pass) ? __ldg(a.v_scale + srow) : 0.f;
        };
        auto convert = [&](int i, int part, float scale) -> bool {
          const long use = st_base + (i - tile0);
          const int st = (int)(use % kS8);
          if (part == 0 &&
              !warp_wait(&sh->st8_full[st], (uint32_t)((use / kS8) & 1), &sh->abort_flag, a.status))
            return false;
          uint64_t* emp = part ? &sh->v_empty : &sh->k_empty;
          const long uses = part ? vc : kc;
          if (uses >= 1 && !warp_wait(emp, (uint32_t)((uses - 1) & 1), &sh->abort_flag, a.status)) return false;
          const uint8_t* src = s8 + st * 2 * kRow8 + part * kRow8 + r * 128;
          uint8_t* dst = sKV + part * kKV + r * 128;
#pragma unroll
          for (int c8 = 0; c8 < 8; ++c8) {  // 16 codes = 16 dims = two 16-byte bf16 chunks
            const uint4 w = *reinterpret_cast<const uint4*>(src + ((c8 ^ (r & 7)) * 16));
            const uint2 x0 = e4m3x4_to_bf16(w.x, scale), x1 = e4m3x4_to_bf16(w.y, scale);
            const uint2 x2 = e4m3x4_to_bf16(w.z, scale), x3 = e4m3x4_to_bf16(w.w, scale);
            const int ca = 2 * c8, cb = 2 * c8 + 1;  // bf16 chunk index 0..15 over the 128 dims
            *reinterpret_cast<uint4*>(dst + (ca >> 3) * kHalf + (((ca & 7) ^ (r & 7)) * 16)) =
                make_uint4(x0.x, x0.y, x1.x, x1.y);
            *reinterpret_cast<uint4*>(dst + (cb >> 3) * kHalf + (((cb & 7) ^ (r & 7)) * 16)) =
                make_uint4(x2.x, x2.y, x3.x, x3.y);
          }
          tc::fence_proxy_async();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(part ? &sh->v_full : &sh->k_full);
          if (part) ++vc;
          else ++kc;
          return true;
        };
        long srow_c, srow_n;
        float ks_c, vs_c, ks_n, vs_n;
        meta(tile0, srow_c, ks_c, vs_c);
        bool ok = tile0 >= tile1 || convert(tile0, 0, ks_c);
        for (int i = tile0; ok && i < tile1; ++i) {
          meta(i + 1, srow_n, ks_n, vs_n);  // in flight while this step waits and converts
          if (i + 1 < tile1 && !convert(i + 1, 0, ks_n)) { ok = false; break; }
          if (main_pass && !convert(i, 1, vs_c)) { ok = false; break; }
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&sh->st8_empty[(int)((st_base + (i - tile0)) % kS8)]);
          srow_c = srow_n;
          ks_c = ks_n;
          vs_c = vs_n;
        }
        if (!ok) {
          if (lane == 0 && !sh->abort_flag) report(a.status, SGQA_ERR_TIMEOUT);
          sh->abort_flag = 1;
        }
        kc = st_base + (tile1 - tile0);  // the staging ring position, as the producer counts it
      }
    } else {
      // ---- probabilities: thread = token slot r of the tile ----
      // the union entry of this thread's token slot, one tile ahead
      auto entry = [&](int i, uint32_t& qm, int& blk) {
        const int idx = i * NB + r / B;
        const bool in = i < tile1 && idx < count;
        qm = in ? __ldg(umask + idx) : 0u;
        blk = in ? __ldg(ublk + idx) : 0;
      };
      uint32_t qm_n;
      int blk_n;
      entry(tile0, qm_n, blk_n);
      for (int i = tile0; i < tile1; ++i, ++scnt) {
        const uint32_t qm = qm_n;
        const int blk = blk_n;
        entry(i + 1, qm_n, blk_n);
        const int sb = (int)(scnt & 1);
        if (!warp_wait(&sh->s_full[sb], (uint32_t)((scnt >> 1) & 1), &sh->abort_flag, a.status)) {
          if (lane == 0 && !sh->abort_flag) report(a.status, SGQA_ERR_TIMEOUT);
          sh->abort_flag = 1;
          break;
        }
        tc::fence_after_sync();
        uint32_t v[kNQ];
        tc::tmem_ld64(tmem + lane_base + (uint32_t)(sb * kNQ), v);
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&sh->s_empty[sb]);
        // columns this token counts for: its block is in the query's selection and u <= t_q
        uint64_t cm = 0;
        if (qm != 0u) {
          const int u = blk * B + (r % B);
          for (int q = 0; q < a.n_new; ++q)
            if (((qm >> q) & 1u) && u <= a.t0 + q) cm |= ((R >= 64 ? ~0ull : ((1ull << R) - 1ull)) << (q * R));
        }
        if (!main_pass) {
#pragma unroll
          for (int n = 0; n < kNQ; ++n)
            if ((cm >> n) & 1ull) atomicMax(&sh->maxkey[n], score_key(__uint_as_float(v[n])));
          continue;
        }
        const int pb = (int)(pcnt % C::kPB);
        if (pcnt >= C::kPB && !warp_wait(&sh->p_empty[pb], (uint32_t)(((pcnt / C::kPB) - 1) & 1), &sh->abort_flag, a.status)) {
          if (lane == 0 && !sh->abort_flag) report(a.status, SGQA_ERR_TIMEOUT);
          sh->abort_flag = 1;
          break;
        }
        uint8_t* prow = sP + pb * kP + r * 128;
        const int nchunk = NQ > 32 ? 8 : 4;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          if (c >= nchunk) break;
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int n0 = 8 * c + 2 * e;
            const float p0 = ((cm >> n0) & 1ull) ? ex2_approx(fmaf(__uint_as_float(v[n0]), sc, -sh->base[n0])) : 0.f;
            const float p1 =
                ((cm >> (n0 + 1)) & 1ull) ? ex2_approx(fmaf(__uint_as_float(v[n0 + 1]), sc, -sh->base[n0 + 1])) : 0.f;
            pk[e] = pack_bf16x2(p0, p1);
          }
          *reinterpret_cast<uint4*>(prow + ((c ^ (r & 7)) * 16)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        tc::fence_proxy_async();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&sh->p_full[pb]);
        ++pcnt;
      }
    }
    if (main_pass) {
      any_pv = tile1 > tile0;
      if (warp == 1 && lane == 0) {
        tc::mma_commit(&sh->o_done);
        ++o_commits;
      }
      if (is_sm) {
        o_ok = warp_wait(&sh->o_done, (uint32_t)o_phase, &sh->abort_flag, a.status);
        if (!o_ok && lane == 0 && !sh->abort_flag) report(a.status, SGQA_ERR_TIMEOUT);
        if (!o_ok) sh->abort_flag = 1;
      }
      o_phase ^= 1;
    }
    __syncthreads();
    if (pass == 0) {
      bool risky = false;
      if (is_sm && o_ok && any_pv) {
        tc::fence_after_sync();
        uint32_t lv[kNQ];
        tc::tmem_ld64(tmem_l + lane_base, lv);
#pragma unroll
        for (int n = 0; n < kNQ; ++n) risky |= n < NQ && !(__uint_as_float(lv[n]) <= kRiskSum);
      }
      rerun = __syncthreads_or(risky) != 0;
    }
  }

  // ---- epilogue: thread = head dimension r; columns in chunks of 32 ----
  if (is_sm && o_ok) {
    float* rec = a.splits > 1 ? a.part + ((long)unit * a.splits + split) * (2 * kNQ + kNQ * kD) : nullptr;
    for (int c0 = 0; c0 < NQ; c0 += 32) {
      uint32_t lv[32], ov[32];
      if (any_pv) {
        tc::fence_after_sync();
        tc::tmem_ld32(tmem_l + lane_base + (uint32_t)c0, lv);
        tc::tmem_ld32(tmem_o + lane_base + (uint32_t)c0, ov);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) lv[i] = ov[i] = 0u;
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int n = c0 + i;
        if (n >= NQ) break;
        const float l = __uint_as_float(lv[i]), o = __uint_as_float(ov[i]);
        if (rec == nullptr) {
          const long off = (((long)b * a.n_new + n / R) * a.Hq + (long)g * R + (n % R)) * kD + r;
          const float y = l > 0.f ? o / l : 0.f;
          a.out[off] = f32_to_bf16_rne(y * sigmoid_fast(bf16_to_f32(__ldg(a.gate + off))));
        } else {
          // partial record of (unit, split): the scaled maximum each column's P was taken
          // against (-inf for a split without tiles), l[64], o[64][d]
          rec[2 * kNQ + n * kD + r] = o;
          if (r == 0) {
            rec[n] = any_pv ? sh->base[n] : -INFINITY;
            rec[kNQ + n] = l;
          }
        }
      }
    }
  }

  // ---- drain and release ----
  if (warp == 0 && lane == 0) {
    // every copy issued lands before the CTA exits
    volatile int no_abort = 0;
    if constexpr (F8) {
      for (long k2 = kc - kS8; k2 < kc; ++k2)
        if (k2 >= 0) tc::mbar_wait(&sh->st8_full[k2 % kS8], (uint32_t)((k2 / kS8) & 1), &no_abort);
    } else {
      for (long k2 = kc - C::kRingK; k2 < kc; ++k2)
        if (k2 >= 0) tc::mbar_wait(&sh->kf[k2 % C::kRingK], (uint32_t)((k2 / C::kRingK) & 1), &no_abort);
      for (long v2 = vc - C::kRingV; v2 < vc; ++v2)
        if (v2 >= 0) tc::mbar_wait(&sh->vf[v2 % C::kRingV], (uint32_t)((v2 / C::kRingV) & 1), &no_abort);
    }
  }
  if (warp == 1 && lane == 0 && o_commits > 0) {
    volatile int no_abort = 0;
    tc::mbar_wait(&sh->o_done, (uint32_t)((o_commits - 1) & 1), &no_abort);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// Union of the selections of the n_new queries of one (sequence, group): ascending block ids and,
// per block, the mask of the queries that selected it. Each list is ascending; an element is
// written by the lowest list that holds it, at the rank given by counting, in every list, the
// elements below it that their lowest lists own (binary searches; no sort).
__global__ void __launch_bounds__(1024) decode_union_kernel(const int32_t* __restrict__ sel, int n_new, int G, int Kb,
                                                           int32_t* __restrict__ ublk, uint32_t* __restrict__ umask,
                                                           int* __restrict__ ucount, int ucap, int* status) {
  extern __shared__ int su[];
  int* lists = su;                 // [n_new][Kb]
  int* incl = su + n_new * Kb;     // [n_new][Kb]: owners among the first i + 1 entries
  uint32_t* msk = reinterpret_cast<uint32_t*>(incl + n_new * Kb);
  __shared__ int len[32];
  const int unit = blockIdx.x, b = unit / G, g = unit % G;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = n_new * Kb;
  if (tid < 32) len[tid] = 0;
  for (int idx = tid; idx < n; idx += blockDim.x) {
    const int q = idx / Kb, i = idx % Kb;
    lists[idx] = __ldg(sel + (((long)b * n_new + q) * G + g) * Kb + i);
  }
  __syncthreads();
  for (int idx = tid; idx < n; idx += blockDim.x) {
    const int q = idx / Kb, i = idx % Kb;
    if (lists[idx] >= 0 && (i == Kb - 1 || lists[idx + 1] < 0)) len[q] = i + 1;
  }
  __syncthreads();
  for (int idx = tid; idx < n; idx += blockDim.x) {
    const int q = idx / Kb, i = idx % Kb;
    int own = 0;
    uint32_t m = 0;
    if (i < len[q]) {
      const int x = lists[idx];
      own = 1;
      m = 1u << q;
      for (int q2 = 0; q2 < n_new; ++q2) {
        if (q2 == q) continue;
        const int* L = lists + q2 * Kb;
        int lo = 0, hi = len[q2];
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (L[mid] < x) lo = mid + 1;
          else hi = mid;
        }
        if (lo < len[q2] && L[lo] == x) {
          m |= 1u << q2;
          if (q2 < q) own = 0;
        }
      }
    }
    incl[idx] = own;
    msk[idx] = m;
  }
  __syncthreads();
  for (int q = warp; q < n_new; q += blockDim.x / 32) {
    int run = 0;
    for (int base = 0; base < len[q]; base += 32) {
      const int i = base + lane;
      const int f = i < len[q] ? incl[q * Kb + i] : 0;
      const unsigned bal = __ballot_sync(0xFFFFFFFFu, f != 0);
      if (i < len[q]) incl[q * Kb + i] = run + __popc(bal & ((2u << lane) - 1u));
      run += __popc(bal);
    }
  }
  __syncthreads();
  for (int idx = tid; idx < n; idx += blockDim.x) {
    const int q = idx / Kb, i = idx % Kb;
    if (i >= len[q]) continue;
    const int own = incl[idx] - (i > 0 ? incl[idx - 1] : 0);
    if (!own) continue;
    const int x = lists[idx];
    int rank = 0;
    for (int q2 = 0; q2 < n_new; ++q2) {
      const int* L = lists + q2 * Kb;
      int lo = 0, hi = len[q2];
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (L[mid] < x) lo = mid + 1;
        else hi = mid;
      }
      rank += lo > 0 ? incl[q2 * Kb + lo - 1] : 0;
    }
    if (!SGQA_CHECK(rank < ucap, status)) continue;
    ublk[(long)unit * ucap + rank] = x;
    umask[(long)unit * ucap + rank] = msk[idx];
  }
  if (tid == 0) {
    int tot = 0;
    for (int q = 0; q < n_new; ++q) tot += len[q] > 0 ? incl[q * Kb + len[q] - 1] : 0;
    ucount[unit] = tot;
  }
}

// Fixed-order merge of the splits' partial records, then the gate: block = (unit, column),
// thread = head dimension.
__global__ void __launch_bounds__(kD) decode_merge_kernel(DecodeAttendArgs a) {
  if (tc::grid_timed_out(a.status)) return;  // the partial records of a stopped launch are incomplete
  const int unit = blockIdx.x, n = blockIdx.y, b = unit / a.G, g = unit % a.G;
  const int R = a.Hq / a.G;
  const int r = threadIdx.x;
  constexpr long kRec = 2 * kNQ + kNQ * kD;
  const float* base = a.part + (long)unit * a.splits * kRec;
  float mstar = -INFINITY;
  for (int s = 0; s < a.splits; ++s) mstar = fmaxf(mstar, __ldg(base + s * kRec + n));
  float den = 0.f, num = 0.f;
  for (int s = 0; s < a.splits; ++s) {
    const float* rec = base + s * kRec;
    const float ms = __ldg(rec + n);
    const float w = ms == -INFINITY ? 0.f : exp2f(ms - mstar);
    den += w * __ldg(rec + kNQ + n);
    num += w * __ldg(rec + 2 * kNQ + n * kD + r);
  }
  const long off = (((long)b * a.n_new + n / R) * a.Hq + (long)g * R + (n % R)) * kD + r;
  const float y = den > 0.f ? num / den : 0.f;
  a.out[off] = f32_to_bf16_rne(y * sigmoid_fast(bf16_to_f32(__ldg(a.gate + off))));
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

// 3-D map over a cache [batch * T_kv tokens][G][d] bf16: box = 64 dims x 1 group x B tokens (one
// block), 128B swizzle.
bool make_cache_map(CUtensorMap* map, const void* base, long tokens, int G, int B) {
  EncodeTiled enc = get_encode();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)G, (cuuint64_t)tokens};
  const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)G * kD * 2};
  const cuuint32_t box[3] = {64, 1, (cuuint32_t)B};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over an fp8 cache [batch * T_kv tokens][G][128] bytes: box = 128 codes x 1 group x B
// tokens (one block), 128B swizzle.
bool make_cache8_map(CUtensorMap* map, const void* base, long tokens, int G, int B) {
  EncodeTiled enc = get_encode();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)G, (cuuint64_t)tokens};
  const cuuint64_t strides[2] = {(cuuint64_t)kD, (cuuint64_t)G * kD};
  const cuuint32_t box[3] = {(cuuint32_t)kD, 1, (cuuint32_t)B};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int B, bool F8>
cudaError_t launch_b(const DecodeAttendArgs& a, cudaStream_t s) {
  using C = DaCfg<F8>;
  CUtensorMap mk, mv;
  const long tokens = (long)a.batch * a.T_kv;
  const bool ok = F8 ? make_cache8_map(&mk, a.k8, tokens, a.G, B) && make_cache8_map(&mv, a.v8, tokens, a.G, B)
                     : make_cache_map(&mk, a.k, tokens, a.G, B) && make_cache_map(&mv, a.v, tokens, a.G, B);
  if (!ok) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(decode_attend_tc_kernel<B, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::kSmem);
  if (e != cudaSuccess) return e;
  decode_attend_tc_kernel<B, F8><<<(unsigned)(a.batch * a.G * a.splits), C::kThr, C::kSmem, s>>>(mk, mv, a);
  return cudaGetLastError();
}

}  // namespace

bool decode_attend_tc_supported(int Hq, int G, int d, int B, int n_new, int Kb) {
  return d == kD && (B == 8 || B == 16) && n_new >= 1 && n_new <= 32 && n_new * (Hq / G) <= kNQ &&
         n_new * Kb <= kUnionMax;
}

int decode_attend_splits(int units, int n_new, int Kb, int B, bool f8) {
  const int max_tiles = (n_new * Kb + kTok / B - 1) / (kTok / B);
  // one wave: 148 SMs x the resident CTAs of the variant
  const int slots = 148 * (f8 ? DaCfg<true>::kCtas : DaCfg<false>::kCtas);
  int s = slots / (units > 0 ? units : 1);
  if (s < 1) s = 1;
  if (s > max_tiles) s = max_tiles;
  return s;
}

size_t decode_part_bytes(int units, int splits) {
  return splits > 1 ? (size_t)units * splits * (2 * kNQ + kNQ * kD) * sizeof(float) : 0;
}

cudaError_t launch_decode_union(const int32_t* sel, int batch, int n_new, int G, int Kb, int32_t* ublk,
                                uint32_t* umask, int* ucount, int ucap, int* status, cudaStream_t s) {
  const size_t shmem = (size_t)n_new * Kb * 12;
  cudaError_t e = cudaFuncSetAttribute(decode_union_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shmem);
  if (e != cudaSuccess) return e;
  // one CTA per (sequence, group): 1024 threads, two or so entries each, so that the binary
  // searches of many threads overlap
  decode_union_kernel<<<(unsigned)(batch * G), 1024, shmem, s>>>(sel, n_new, G, Kb, ublk, umask, ucount, ucap, status);
  return cudaGetLastError();
}

cudaError_t launch_decode_attend_tc(const DecodeAttendArgs& a, cudaStream_t s) {
  const bool f8 = a.k8 != nullptr;
  cudaError_t e = a.B == 8 ? (f8 ? launch_b<8, true>(a, s) : launch_b<8, false>(a, s))
                  : a.B == 16 ? (f8 ? launch_b<16, true>(a, s) : launch_b<16, false>(a, s))
                              : cudaErrorInvalidValue;
  if (e != cudaSuccess || a.splits == 1) return e;
  decode_merge_kernel<<<dim3((unsigned)(a.batch * a.G), (unsigned)(a.n_new * (a.Hq / a.G))), kD, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace sgqa
