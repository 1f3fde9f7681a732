// K2 on the 5th-generation tensor cores: indexer scores q_idx . kbar as a tcgen05 contraction
// with the exact per-row top-(k/B) selection fused into the accumulator epilogue.
//
// Step 5 Preview pages (mo.ai.kr, "Step 5 Preview agentic work design", section "model
// structure and training stability"): every KV group scores the compressed blocks of the shared
// index keys and keeps its top k/B = 512 blocks; blocks of 8 make this eightfold cheaper.
// Selection rule implemented: candidates j < c = floor(t/B); the best m = min(k/B - 1, c) by
// (fp32 score desc, j asc), then the own block c; output ascending, -1 padded.
//
// One CTA owns 128 rows = (128/G) adjacent queries x G groups (the rows are consecutive rows of
// q_idx, so one TMA box loads them). Scores for N = 128 candidate blocks at a time are
//     D[128 x 128] (fp32, TMEM) = q_idx[128 x d_idx] . (kbar_hi + kbar_lo)[128 x d_idx]^T
// issued by one thread as 2 * d_idx/16 tcgen05.mma (kind::f16, bf16 operands, K-major, 128B or
// 64B swizzle) over two TMA-fed shared-memory stages, into two TMEM accumulators. kbar is
// fp32; splitting it into bf16 hi + lo planes keeps the product exact to ~2^-17 relative, and
// q_idx is exactly bf16, so the contraction runs at the bf16 tensor rate.
//
// Warp roles: warp 4 issues TMA loads, warp 5 allocates TMEM and issues MMAs, warps 0-3 own one
// row each per thread (TMEM lane = row). The epilogue performs an exact radix select of the
// m-th largest order-preserving 32-bit score key per row: every pass re-streams the same score
// tiles (recomputed, bit-identical) and fills the row's 256-bin shared histogram of the next 8
// key bits among keys that still match the resolved prefix; once every row's threshold bucket
// is resolved (or taken whole), a final pass streams the candidates in ascending j and emits
// keys above the threshold plus the first ties at it, so ties go to the lower block index and
// the output is ascending without a sort. The epilogue tells the producer and MMA warps at the
// start of each pass whether another pass follows, so they run up to one pass ahead.
//
// Every wait is bounded (globaltimer): on timeout the kernel records SGQA_ERR_TIMEOUT, stops all
// roles, waits (bounded) for its own copies and MMAs in flight, frees TMEM and returns.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace sgqa {
namespace {

constexpr int kRows = 128;
constexpr int kN = 128;          // candidate blocks per MMA tile
constexpr int kStages = 2;
constexpr int kHistStride = 257;
constexpr int kEpiWarps = 8;     // two per TMEM lane quadrant: each histograms half the columns
constexpr int kThreads = (kEpiWarps + 2) * 32;
constexpr int kProducerWarp = kEpiWarps, kMmaWarp = kEpiWarps + 1;
constexpr int kMaxPasses = 5;
constexpr int kCap = 128;        // bucket keys a row may collect for an early exact finish (8 B each)

template <int DI>
struct SelCfg {
  static constexpr int kRowBytes = DI * 2;
  static constexpr int kA = kRows * kRowBytes;
  static constexpr int kBPlane = kN * kRowBytes;
  static constexpr int kStage = 2 * kBPlane;
  static constexpr int kHist = kRows * kHistStride * 4;
  static constexpr int kSmem = 1024 + kA + kStages * kStage + kHist + 256;
};

struct SelShared {
  uint64_t full[kStages], empty[kStages], acc_full[2], acc_empty[2], a_full;
  uint32_t tmem;
  volatile int signals;
  volatile int abort_flag;
  int more[kMaxPasses + 1];
  int vote_cnt[4 * kMaxPasses];
  int vote_any[4 * kMaxPasses];
};

// Bounded barrier + "any" vote among the epilogue warps (slot = a fresh index per use): every
// epilogue warp adds its vote and waits (bounded, abort-aware) until all have voted. Returns 1/0,
// or -1 on giving up.
__device__ __forceinline__ int epi_vote_any(SelShared* sh, int slot, bool v) {
  const int lane = threadIdx.x & 31;
  const unsigned any = __any_sync(0xFFFFFFFFu, v);
  int res = 0;
  if (lane == 0) {
    if (any) atomicOr(&sh->vote_any[slot], 1);
    __threadfence_block();
    atomicAdd(&sh->vote_cnt[slot], 1);
    const uint64_t t0 = tc::globaltimer();
    volatile int* cnt = &sh->vote_cnt[slot];
    res = 1;
    while (*cnt < kEpiWarps) {
      if (sh->abort_flag || tc::globaltimer() - t0 > tc::kWaitLimitNs) { res = -1; break; }
      __nanosleep(32);
    }
    if (res > 0) {
      __threadfence_block();
      res = *(volatile int*)&sh->vote_any[slot] ? 1 : 0;
    }
  }
  return __shfl_sync(0xFFFFFFFFu, res, 0);
}

// Warp-uniform bounded wait: lane 0 polls, the verdict is broadcast to the warp.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = tc::mbar_wait(bar, parity, abort) ? 1 : 0;
  return __shfl_sync(0xFFFFFFFFu, ok, 0) != 0;
}

// Wait until the epilogue has announced pass p-1 (and with it whether pass p exists).
__device__ __forceinline__ int pass_exists(SelShared* sh, int p) {
  if (p == 0) return 1;
  const uint64_t t0 = tc::globaltimer();
  while (sh->signals < p) {
    if (sh->abort_flag) return 0;
    if (tc::globaltimer() - t0 > tc::kWaitLimitNs) return -1;
    __nanosleep(64);
  }
  __threadfence_block();
  return sh->more[p - 1];
}

// ---- branch-free per-key epilogue steps (64 consecutive candidates of one row per call) ----
// Shared-memory histogram increment / pair store, predicated in PTX so that the per-key loop
// has no branches.
__device__ __forceinline__ void red_shared_inc(uint32_t addr) {
  asm volatile("red.shared.add.u32 [%0], 1;" ::"r"(addr) : "memory");
}
__device__ __forceinline__ void red_shared_inc_if_eq(uint32_t addr, uint32_t a, uint32_t b) {
  asm volatile("{ .reg .pred p; setp.eq.u32 p, %1, %2; @p red.shared.add.u32 [%0], 1; }" ::"r"(addr), "r"(a),
               "r"(b)
               : "memory");
}
// (addr is only 4-byte aligned: row histograms are 257 words apart)
__device__ __forceinline__ void st_shared_pair_if(uint32_t addr, uint32_t x, uint32_t y, uint32_t pred) {
  asm volatile("{ .reg .pred p; setp.ne.u32 p, %3, 0; @p st.shared.u32 [%0], %1; @p st.shared.u32 [%0+4], %2; }" ::"r"(
                   addr),
               "r"(x), "r"(y), "r"(pred)
               : "memory");
}

// Histogram pass: count, in the row's 256 bins, the next 8 key bits (at `shift`) of the keys
// whose resolved bits (mask) equal prefix. kFull: all 64 candidates exist (else only q < lim).
template <bool kFull, bool kFirst>
__device__ __forceinline__ void hist_chunk(const uint32_t (&v)[64], int lim, uint32_t mask, uint32_t prefix, int shift,
                                           uint32_t hbase) {
#pragma unroll
  for (int q = 0; q < 64; ++q) {
    const uint32_t key = score_key(__uint_as_float(v[q]));
    const uint32_t addr = hbase + (((key >> shift) & 255u) << 2);
    if (kFull) {
      if (kFirst) red_shared_inc(addr);
      else red_shared_inc_if_eq(addr, key & mask, prefix);
    } else {
      red_shared_inc_if_eq(addr, (q < lim && (kFirst || (key & mask) == prefix)) ? 1u : 0u, 1u);
    }
  }
}

// Emit pass: mark (bits of tb) the candidates taken: keys >= thr, plus, among the keys of the
// bucket [blo, blo + bw], the first tie_lim in j order; the first col_lim bucket keys are also
// stored as (key, j) pairs at cbase. eqn counts the bucket keys seen so far in this row.
template <bool kFull>
__device__ __forceinline__ void emit_chunk(const uint32_t (&v)[64], int lim, uint32_t thr, uint32_t blo, uint32_t bw,
                                           int tie_lim, int col_lim, uint32_t cbase, int j0, int& eqn,
                                           uint32_t (&tb)[2]) {
#pragma unroll
  for (int q = 0; q < 64; ++q) {
    const uint32_t key = score_key(__uint_as_float(v[q]));
    const bool in = kFull || q < lim;
    const bool inb = in && key - blo <= bw;
    const bool take = in && (key >= thr || (inb && eqn < tie_lim));
    st_shared_pair_if(cbase + 8u * (uint32_t)eqn, key, (uint32_t)(j0 + q), (inb && eqn < col_lim) ? 1u : 0u);
    eqn += inb ? 1 : 0;
    tb[q >> 5] |= take ? (1u << (q & 31)) : 0u;
  }
}

template <int DI>
__global__ void __launch_bounds__(kThreads, 1)
    select_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_hi,
                     const __grid_constant__ CUtensorMap map_lo, SelectArgs a) {
  using C = SelCfg<DI>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align<1024>(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = sA + C::kA;                                               // [stage][hi|lo][kN][DI]
  uint32_t* hist = reinterpret_cast<uint32_t*>(sB + kStages * C::kStage);
  SelShared* sh = reinterpret_cast<SelShared*>(reinterpret_cast<uint8_t*>(hist) + C::kHist);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.G, TQ = kRows / G;
  const int n_tiles = (a.t_end - a.t_begin + TQ - 1) / TQ;
  const int tile = n_tiles - 1 - (int)(blockIdx.x / a.batch);  // heaviest tiles first
  const int b = (int)(blockIdx.x % a.batch);
  const int tq0 = a.t_begin + tile * TQ;
  const int t_last = min(a.t_end - 1, tq0 + TQ - 1);
  const int n_cand = t_last / a.B;
  const int n_nt = (n_cand + kN - 1) / kN;
  const int nblk = a.T / a.B;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&sh->full[s], 1);
      tc::mbar_init(&sh->empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&sh->acc_full[s], 1);
      tc::mbar_init(&sh->acc_empty[s], kEpiWarps);
    }
    tc::mbar_init(&sh->a_full, 1);
    sh->signals = 0;
    sh->abort_flag = 0;
    for (int p = 0; p < 4 * kMaxPasses; ++p) sh->vote_cnt[p] = sh->vote_any[p] = 0;
    tc::fence_mbar_init();
  }
  if (warp == kMmaWarp) tc::tmem_alloc(&sh->tmem, 256);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = sh->tmem;

  if (warp == kProducerWarp) {
    // ---------------- TMA producer ----------------
    if (lane == 0 && n_nt > 0) {
      tc::prefetch_tensormap(&map_q);
      tc::prefetch_tensormap(&map_hi);
      tc::prefetch_tensormap(&map_lo);
      tc::mbar_arrive_expect_tx(&sh->a_full, C::kA);
      tc::tma_load_2d(sA, &map_q, &sh->a_full, 0, (int)(((long)b * a.T + tq0) * G));
      long k = 0;
      bool ok = true;
      for (int pass = 0; ok && pass < kMaxPasses; ++pass) {
        const int ex = pass_exists(sh, pass);
        if (ex < 0) { report(a.status, SGQA_ERR_TIMEOUT); sh->abort_flag = 1; ok = false; break; }
        if (ex == 0) break;
        for (int i = 0; i < n_nt; ++i, ++k) {
          const int st = (int)(k % kStages);
          const uint32_t ph = (uint32_t)((k / kStages) & 1);
          if (k >= kStages && !tc::mbar_wait(&sh->empty[st], ph ^ 1u, &sh->abort_flag)) {
            if (!sh->abort_flag) report(a.status, SGQA_ERR_TIMEOUT);
            sh->abort_flag = 1;
            ok = false;
            break;
          }
          uint8_t* dst = sB + st * C::kStage;
          tc::mbar_arrive_expect_tx(&sh->full[st], C::kStage);
          const int row = b * nblk + i * kN;
          tc::tma_load_2d(dst, &map_hi, &sh->full[st], 0, row);
          tc::tma_load_2d(dst + C::kBPlane, &map_lo, &sh->full[st], 0, row);
        }
      }
      // drain: the copies issued last must land before the CTA can exit
      for (long kk = k - kStages; kk < k; ++kk) {
        if (kk < 0) continue;
        const int st = (int)(kk % kStages);
        volatile int no_abort = 0;
        tc::mbar_wait(&sh->full[st], (uint32_t)((kk / kStages) & 1), &no_abort);
      }
      if (k == 0) {
        volatile int no_abort = 0;
        tc::mbar_wait(&sh->a_full, 0, &no_abort);
      }
    }
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issuer ----------------
    if (lane == 0 && n_nt > 0) {
      const uint32_t idesc = tc::idesc_bf16_f32(kRows, kN);
      bool ok = tc::mbar_wait(&sh->a_full, 0, &sh->abort_flag);
      if (!ok) {
        if (!sh->abort_flag) report(a.status, SGQA_ERR_TIMEOUT);
        sh->abort_flag = 1;
      }
      const uint64_t da = tc::smem_desc_kmajor(sA, C::kRowBytes);
      long k = 0;
      for (int pass = 0; ok && pass < kMaxPasses; ++pass) {
        const int ex = pass_exists(sh, pass);
        if (ex < 0) { report(a.status, SGQA_ERR_TIMEOUT); sh->abort_flag = 1; ok = false; break; }
        if (ex == 0) break;
        for (int i = 0; i < n_nt; ++i, ++k) {
          const int st = (int)(k % kStages);
          const uint32_t ph = (uint32_t)((k / kStages) & 1);
          const int buf = (int)(k & 1);
          if (!tc::mbar_wait(&sh->full[st], ph, &sh->abort_flag) ||
              (k >= 2 && !tc::mbar_wait(&sh->acc_empty[buf], (uint32_t)(((k >> 1) - 1) & 1), &sh->abort_flag))) {
            if (!sh->abort_flag) report(a.status, SGQA_ERR_TIMEOUT);
            sh->abort_flag = 1;
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint8_t* bst = sB + st * C::kStage;
          const uint64_t dhi = tc::smem_desc_kmajor(bst, C::kRowBytes);
          const uint64_t dlo = tc::smem_desc_kmajor(bst + C::kBPlane, C::kRowBytes);
          const uint32_t d = tmem + (uint32_t)(buf * kN);
#pragma unroll
          for (int kk = 0; kk < DI / 16; ++kk)
            tc::mma_bf16_ss(d, da + 2 * kk, dhi + 2 * kk, idesc, kk > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < DI / 16; ++kk) tc::mma_bf16_ss(d, da + 2 * kk, dlo + 2 * kk, idesc, 1u);
          tc::mma_commit(&sh->empty[st]);
          tc::mma_commit(&sh->acc_full[buf]);
        }
      }
      // drain: the last MMAs must complete before TMEM is freed
      if (k > 0) {
        volatile int no_abort = 0;
        tc::mbar_wait(&sh->acc_full[(k - 1) & 1], (uint32_t)(((k - 1) >> 1) & 1), &no_abort);
      }
    }
  } else {
    // ---------------- epilogue: one row per thread pair ----------------
    // Warps w and w + 4 read TMEM lane quadrant w % 4 (row r = 32 * (w % 4) + lane); in histogram
    // passes each takes half of every tile's columns (atomics on the row's shared histogram); in
    // the emit pass the lower warp streams all columns in order and the upper one only releases
    // the accumulators.
    const int quad = warp & 3, half = warp >> 2;
    const int r = quad * 32 + lane;
    const int t = tq0 + r / G, g = r % G;
    const bool valid = t <= t_last;
    const int c = valid ? t / a.B : 0;
    const int m = valid ? min(a.Kb - 1, c) : 0;
    uint32_t prefix = 0, mask = 0;
    int rem = m, nb = c;
    bool done = (rem == nb);
    if (rem == 0) { prefix = 0xFFFFFFFFu; mask = 0xFFFFFFFFu; done = true; }
    uint32_t* my_hist = hist + r * kHistStride;
    int32_t* out = a.sel + (((long)b * a.sel_T + (t - a.sel_t0)) * G + g) * (long)a.Kb;
    const uint32_t lane_base = (uint32_t)(32 * quad) << 16;
    const uint32_t hbase = smem_u32(my_hist);
    long k = 0;
    int pos = 0;
    bool aborted = false;
    for (int pass = 0; pass < kMaxPasses; ++pass) {
      // zero the histograms for this pass, then a barrier+vote: is any row still unresolved?
      if (half == 0 && !done && pass < kMaxPasses - 1)
        for (int i = 0; i < 256; ++i) my_hist[i] = 0;
      const int vote = epi_vote_any(sh, 4 * pass, !done);
      // from the third pass on, if every unresolved row's threshold bucket is small, this pass is
      // the last: it also collects those buckets' keys, which are then resolved exactly
      const int vote_big = (pass >= 2 && vote > 0) ? epi_vote_any(sh, 4 * pass + 3, !done && nb > kCap) : 1;
      if (vote < 0 || vote_big < 0) {
        if (lane == 0 && !sh->abort_flag) report(a.status, SGQA_ERR_TIMEOUT);
        sh->abort_flag = 1;
        break;
      }
      const bool is_emit = vote == 0 || vote_big == 0 || pass == kMaxPasses - 1;
      if (warp == 0 && lane == 0) {
        sh->more[pass] = is_emit ? 0 : 1;
        __threadfence_block();
        sh->signals = pass + 1;
      }
      // emit rule of this row: take keys >= thr; bucket [blo, blo + bw] handled by ties or collection
      uint32_t thr = 0xFFFFFFFFu, blo = 0xFFFFFFFFu, bw = 0u;
      int tie_lim = 0, col_lim = 0;
      if (!done) {  // collecting: everything above the bucket, the bucket's keys kept aside
        const uint32_t pend = prefix | ~mask;
        thr = pend == 0xFFFFFFFFu ? 0xFFFFFFFFu : pend + 1u;
        blo = prefix;
        bw = ~mask;
        col_lim = kCap;
      } else if (rem == nb) {  // the whole bucket is taken
        thr = prefix;
      } else {  // fully resolved key with ties: the first rem of them in j order
        thr = prefix == 0xFFFFFFFFu ? 0xFFFFFFFFu : prefix + 1u;
        blo = prefix;
        tie_lim = rem;
      }
      int eqn = 0;
      const int shift = 24 - 8 * pass;
      for (int i = 0; i < n_nt; ++i, ++k) {
        const int buf = (int)(k & 1);
        if (!warp_wait(&sh->acc_full[buf], (uint32_t)((k >> 1) & 1), &sh->abort_flag)) {
          if (lane == 0 && !sh->abort_flag) report(a.status, SGQA_ERR_TIMEOUT);
          sh->abort_flag = 1;
          aborted = true;
          break;
        }
        tc::fence_after_sync();
        if (!is_emit) {
          uint32_t v[64];
          tc::tmem_ld64(tmem + lane_base + (uint32_t)(buf * kN + half * 64), v);
          const int j0 = i * kN + half * 64;
          const int lim = c - j0;
          // a resolved row matches nothing (its histogram is not read; in the first pass it may
          // count, harmlessly)
          const uint32_t mk = done ? 0u : mask, pf = done ? 1u : prefix;
          if (__all_sync(0xFFFFFFFFu, lim >= 64)) {
            if (pass == 0) hist_chunk<true, true>(v, lim, mk, pf, shift, hbase);
            else hist_chunk<true, false>(v, lim, mk, pf, shift, hbase);
          } else if (lim > 0) {
            if (pass == 0) hist_chunk<false, true>(v, lim, mk, pf, shift, hbase);
            else hist_chunk<false, false>(v, lim, mk, pf, shift, hbase);
          }
        } else if (half == 0) {
#pragma unroll 1
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t v[64];
            tc::tmem_ld64(tmem + lane_base + (uint32_t)(buf * kN + hh * 64), v);
            const int j0 = i * kN + hh * 64;
            const int lim = valid ? c - j0 : 0;
            uint32_t tb[2] = {0u, 0u};
            if (__all_sync(0xFFFFFFFFu, lim >= 64))
              emit_chunk<true>(v, lim, thr, blo, bw, tie_lim, col_lim, hbase, j0, eqn, tb);
            else if (lim > 0)
              emit_chunk<false>(v, lim, thr, blo, bw, tie_lim, col_lim, hbase, j0, eqn, tb);
#pragma unroll
            for (int w = 0; w < 2; ++w) {
              uint32_t bits = tb[w];
              while (bits) {
                const int q = __ffs(bits) - 1;
                bits &= bits - 1u;
                if (pos < m) out[pos++] = j0 + 32 * w + q;
              }
            }
          }
        }
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&sh->acc_empty[buf]);
      }
      if (aborted) break;
      if (is_emit) {
        if (half == 0 && valid && !done) {
          // the collected bucket (ascending j): candidate i ranks behind every larger key and every
          // equal key of lower j, and is chosen when fewer than rem rank ahead of it
          const uint32_t* cand = my_hist;
          uint32_t* cj = my_hist;
          int nch = 0;
          if (eqn > kCap) report(a.status, SGQA_ERR_DEVICE_CHECK);
          const int ncand = min(eqn, kCap);
          for (int ci = 0; ci < ncand; ++ci) {
            const uint32_t key = cand[2 * ci];
            int ahead = 0;
            for (int c2 = 0; c2 < ncand; ++c2) {
              const uint32_t k2 = cand[2 * c2];
              ahead += (k2 > key || (k2 == key && c2 < ci)) ? 1 : 0;
            }
            if (ahead < rem) cj[2 * nch++ + 1] = cand[2 * ci + 1];  // keys stay; only j slots move down
          }
          if (pos + nch > m) {
            report(a.status, SGQA_ERR_DEVICE_CHECK);
            nch = m - pos;
          }
          // merge the chosen (ascending j) into the row written so far, from the back
          int rd = pos - 1, wr = pos + nch - 1;
          for (int kk = nch - 1; kk >= 0 && wr >= 0; --wr) {
            const int jc = (int)cj[2 * kk + 1];
            if (rd >= 0 && out[rd] > jc) out[wr] = out[rd--];
            else { out[wr] = jc; --kk; }
          }
          pos += nch;
        }
        if (half == 0 && valid) {
          if (pos != m) report(a.status, SGQA_ERR_DEVICE_CHECK);
          out[pos++] = c;
          for (; pos < a.Kb; ++pos) out[pos] = -1;
        }
        break;
      }
      // both halves' histogram updates are complete before either reads the histogram
      if (epi_vote_any(sh, 4 * pass + 1, false) < 0) {
        if (lane == 0 && !sh->abort_flag) report(a.status, SGQA_ERR_TIMEOUT);
        sh->abort_flag = 1;
        break;
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
      // both halves have read the histogram before the next pass zeroes it
      if (epi_vote_any(sh, 4 * pass + 2, false) < 0) {
        if (lane == 0 && !sh->abort_flag) report(a.status, SGQA_ERR_TIMEOUT);
        sh->abort_flag = 1;
        break;
      }
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 256);
  }
}

// rows with no complete past block (T < B): only the own block is selected
__global__ void own_block_only_kernel(SelectArgs a) {
  const long n = (long)a.batch * (a.t_end - a.t_begin) * a.G;
  for (long e = (long)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (long)gridDim.x * blockDim.x) {
    const int g = (int)(e % a.G);
    const long bt = e / a.G;
    const int t = a.t_begin + (int)(bt % (a.t_end - a.t_begin));
    const int b = (int)(bt / (a.t_end - a.t_begin));
    int32_t* out = a.sel + (((long)b * a.sel_T + (t - a.sel_t0)) * a.G + g) * (long)a.Kb;
    out[0] = t / a.B;
    for (int i = 1; i < a.Kb; ++i) out[i] = -1;
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

// 2D map over a row-major [rows, cols] bf16 matrix, box {cols, box_rows}, swizzle matching the
// row width (128 bytes -> 128B, 64 bytes -> 64B).
bool make_map(CUtensorMap* map, const void* base, long rows, int cols, int box_rows) {
  EncodeTiled enc = get_encode();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {(cuuint32_t)cols, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw = cols * 2 == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DI>
cudaError_t launch_di(const SelectArgs& a, cudaStream_t s) {
  using C = SelCfg<DI>;
  const int nblk = a.T / a.B;
  CUtensorMap mq, mh, ml;
  if (!make_map(&mq, a.q_idx, (long)a.batch * a.T * a.G, DI, kRows) ||
      !make_map(&mh, a.kbar_hi, (long)a.batch * nblk, DI, kN) || !make_map(&ml, a.kbar_lo, (long)a.batch * nblk, DI, kN))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(select_tc_kernel<DI>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  const int TQ = kRows / a.G;
  const int n_tiles = (a.t_end - a.t_begin + TQ - 1) / TQ;
  select_tc_kernel<DI><<<(unsigned)(n_tiles * a.batch), kThreads, C::kSmem, s>>>(mq, mh, ml, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_select(const SelectArgs& a, cudaStream_t s) {
  if (a.t_end <= a.t_begin) return cudaSuccess;
  if (a.T / a.B == 0) {
    own_block_only_kernel<<<148, 256, 0, s>>>(a);
    return cudaGetLastError();
  }
  if (a.d_idx == 64) return launch_di<64>(a, s);
  if (a.d_idx == 32) return launch_di<32>(a, s);
  return cudaErrorInvalidValue;
}

}  // namespace sgqa
