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
// Warp roles: warp 16 issues TMA loads, warp 17 allocates TMEM and issues MMAs, warps 0-15 are
// the epilogue, four per TMEM lane quadrant (TMEM lane = row); each of the four takes a quarter
// (32 columns) of every tile, so that every scheduler interleaves four epilogue warps. The
// epilogue performs an exact radix select of the m-th largest order-preserving 32-bit score key
// per row: every pass re-streams the same score tiles (recomputed, bit-identical); in a histogram
// pass each thread adds its scores that still match the resolved prefix to the row's 256-bin
// shared histogram of the next 8 bits, counted on the raw float bits and read back in key order
// (scores that do not match go to a spare slot of the row, so the shared-memory reductions stay
// branch-free and free of bank conflicts). Once every row's threshold bucket is resolved or taken whole, the emit pass
// marks the taken candidates of each 32-column quarter-tile in one 32-bit word and stores it to
// the row's bitmap in global memory: keys above the threshold; bucket keys taken whole; exact ties
// in j order (the four threads of a row exchange their tie counts through shared memory, so ties
// go to the lower block index); or, when every unresolved row's bucket is small (from the third
// pass on), the bucket keys are collected and resolved exactly afterwards, their bits set with
// atomics. A separate kernel expands every row's bitmap into the ascending block list, appends
// the own block and pads with -1. The epilogue tells the producer and MMA warps at the start of
// each pass whether another pass follows, so they run up to one pass ahead.
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
constexpr int kHistStride = 257;  // words per row (256 bins + spare slot); stored bin-major, below
constexpr int kParts = 4;        // epilogue warps per TMEM lane quadrant, each takes kCols columns
constexpr int kCols = kN / kParts;
constexpr int kEpiWarps = 4 * kParts;
static_assert(kCols == 32, "one bitmap word per part and tile");
constexpr int kThreads = (kEpiWarps + 2) * 32;
constexpr int kProducerWarp = kEpiWarps, kMmaWarp = kEpiWarps + 1;
constexpr int kMaxPasses = 5;
constexpr int kCap = 31;         // bucket keys a row may collect for an early exact finish (2 words each)
constexpr int kCandWords = 2 * kCap;  // words of one part's collected keys
constexpr int kTrash = 256;      // the row's spare histogram slot: target of the keys that do not count
constexpr int kCntBase = kParts * kCandWords;  // parts 1..: collected count and taken count (emit pass)
constexpr int kTieWords = 2 * kParts;          // tie-count slots [part][tile parity]
static_assert(kCntBase + 2 * (kParts - 1) <= kTrash, "per-row words of the emit pass");

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
__device__ __forceinline__ int epi_vote_any(SelShared* sh, int slot, bool v, const int* gstatus) {
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
    for (uint32_t it = 1; *cnt < kEpiWarps; ++it) {
      if (sh->abort_flag || tc::globaltimer() - t0 > tc::kWaitLimitNs) { res = -1; break; }
      if ((it & 1023u) == 0u && tc::grid_timed_out(gstatus)) { sh->abort_flag = 1; res = -1; break; }
      __nanosleep(32);
    }
    if (res > 0) {
      __threadfence_block();
      res = *(volatile int*)&sh->vote_any[slot] ? 1 : 0;
    }
  }
  return __shfl_sync(0xFFFFFFFFu, res, 0);
}

// Warp-uniform bounded wait: lane 0 polls, the outcome is broadcast to the warp.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, const int* gstatus) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = tc::mbar_wait(bar, parity, abort, gstatus) ? 1 : 0;
  return __shfl_sync(0xFFFFFFFFu, ok, 0) != 0;
}

// Wait until the epilogue has announced pass p-1 (and with it whether pass p exists).
__device__ __forceinline__ int pass_exists(SelShared* sh, int p, const int* gstatus) {
  if (p == 0) return 1;
  const uint64_t t0 = tc::globaltimer();
  for (uint32_t it = 1; sh->signals < p; ++it) {
    if (sh->abort_flag) return 0;
    if (tc::globaltimer() - t0 > tc::kWaitLimitNs) return -1;
    if ((it & 1023u) == 0u && tc::grid_timed_out(gstatus)) {
      sh->abort_flag = 1;
      return 0;
    }
    __nanosleep(64);
  }
  __threadfence_block();
  return sh->more[p - 1];
}

// ---- branch-free per-key epilogue steps (64 consecutive candidates of one row per call) ----
// Shared-memory histogram updates for the branch-free per-key loops.
__device__ __forceinline__ void red_shared_inc(uint32_t addr) {
  asm volatile("red.shared.add.u32 [%0], 1;" ::"r"(addr) : "memory");
}

// Histogram pass over the raw float bits (kCols consecutive candidates of a row per call) (the order-preserving key is applied to the bins, once
// per row, when the histogram is read): count, in the row's 256 bins, the 8 raw bits at `shift`
// of the scores whose resolved raw bits equal prefix (whose other bits are zero). With
// x = (raw ^ prefix) >> shift, a matching score has x = its bin and any other x > 255, so
// min(x, 256) sends the others to the row's spare slot: every lane stays active. Adding +0.0
// first makes -0.0 the same score as +0.0. kFull: all 64 candidates exist (else only q < lim).
template <bool kFull, bool kFirst>
__device__ __forceinline__ void hist_chunk(const uint32_t (&v)[kCols], int lim, uint32_t prefix, int shift,
                                           uint32_t hbase) {
#pragma unroll
  for (int q = 0; q < kCols; ++q) {
    const uint32_t raw = __float_as_uint(__uint_as_float(v[q]) + 0.0f);
    uint32_t x = kFirst ? raw >> 24 : min((raw ^ prefix) >> shift, (uint32_t)kTrash);
    if (!kFull) x = q < lim ? x : (uint32_t)kTrash;
    red_shared_inc(hbase + x * (kRows * 4u));
  }
}

// Raw-bits view of a key prefix: the resolved raw bits, and whether the digits run in reverse
// (negative scores: raw = ~key). The sign is the key's top bit, resolved with the first digit.
__device__ __forceinline__ uint32_t raw_prefix(uint32_t prefix, uint32_t mask) {
  return (prefix & 0x80000000u) ? (prefix ^ 0x80000000u) : (~prefix & mask);
}

// The raw bin holding key bin kb of the digit at this level: the first digit maps key top bytes
// 128..255 (non-negative scores) to raw 0..127 and 0..127 (negative) to raw 255..128; later
// digits of a negative prefix run in reverse.
__device__ __forceinline__ int raw_bin(int kb, bool first, bool neg) {
  return first ? (kb >= 128 ? kb - 128 : 255 - kb) : (neg ? 255 - kb : kb);
}

// v[q] for a run-time q, keeping the array in registers (used only for the rare bucket keys)
__device__ __forceinline__ uint32_t pick32(const uint32_t (&v)[kCols], int q) {
  switch (q) {
    case 0: return v[0];
    case 1: return v[1];
    case 2: return v[2];
    case 3: return v[3];
    case 4: return v[4];
    case 5: return v[5];
    case 6: return v[6];
    case 7: return v[7];
    case 8: return v[8];
    case 9: return v[9];
    case 10: return v[10];
    case 11: return v[11];
    case 12: return v[12];
    case 13: return v[13];
    case 14: return v[14];
    case 15: return v[15];
    case 16: return v[16];
    case 17: return v[17];
    case 18: return v[18];
    case 19: return v[19];
    case 20: return v[20];
    case 21: return v[21];
    case 22: return v[22];
    case 23: return v[23];
    case 24: return v[24];
    case 25: return v[25];
    case 26: return v[26];
    case 27: return v[27];
    case 28: return v[28];
    case 29: return v[29];
    case 30: return v[30];
    case 31: return v[31];
    default: return 0u;
  }
}

// Emit pass, kCols consecutive candidates of a row: bits of the taken keys (key >= thr) in tb and,
// with kBucket, of the bucket keys (blo <= key <= blo + bw) in bb. ALU only. kPos (thr above the
// key of +0.0, and blo at or above it): the comparisons run on the raw float bits, which order
// the non-negative scores as their keys do and put every negative score (and -0.0) below thr and
// outside the bucket.
template <bool kFull, bool kBucket, bool kPos>
__device__ __forceinline__ void emit_bits(const uint32_t (&v)[kCols], int lim, uint32_t thr, uint32_t blo, uint32_t bw,
                                          uint32_t& tb, uint32_t& bb) {
  const int thr_raw = (int)(thr ^ 0x80000000u);
  const uint32_t blo_raw = blo ^ 0x80000000u;
#pragma unroll
  for (int q = 0; q < kCols; ++q) {
    const bool in = kFull || q < lim;
    if (kPos) {
      tb |= (in && (int)v[q] >= thr_raw) ? (1u << q) : 0u;
      if (kBucket) bb |= (in && v[q] - blo_raw <= bw) ? (1u << q) : 0u;
    } else {
      const uint32_t key = score_key(__uint_as_float(v[q]));
      tb |= (in && key >= thr) ? (1u << q) : 0u;
      if (kBucket) bb |= (in && key - blo <= bw) ? (1u << q) : 0u;
    }
  }
}

__device__ __forceinline__ bool act_row(bool valid, int m) { return valid && m > 0; }

// The lowest n set bits of x (all of them if n >= popc(x), none if n <= 0).
__device__ __forceinline__ uint32_t first_bits(uint32_t x, int n) {
  if (n <= 0) return 0u;
  if (n >= __popc(x)) return x;
  return x & ((1u << __fns(x, 0u, n + 1)) - 1u);
}

// Per-lane bounded wait for another part's tie count of a tile: the slot holds
// (tile + 1) << 8 | count once written. Returns the count, or -1 on giving up.
__device__ __forceinline__ int wait_tie_count(volatile uint32_t* slot, uint32_t tag, SelShared* sh,
                                              const int* gstatus) {
  const uint64_t t0 = tc::globaltimer();
  for (uint32_t it = 1;; ++it) {
    const uint32_t v = *slot;
    if ((v >> 8) == tag) return (int)(v & 255u);
    if (sh->abort_flag || tc::globaltimer() - t0 > tc::kWaitLimitNs) return -1;
    if ((it & 1023u) == 0u && tc::grid_timed_out(gstatus)) {
      sh->abort_flag = 1;
      return -1;
    }
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

  // a timeout recorded by another CTA (this launch or an earlier one sharing the status word):
  // do nothing (the decision is the CTA's, before any barrier or TMEM is set up)
  if (__syncthreads_or(tid == 0 && tc::grid_timed_out(a.status))) return;
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
      tc::tma_load_2d(sA, &map_q, &sh->a_full, 0, (int)(((long)b * a.q_T + (tq0 - a.q_t0)) * G));
      long k = 0;
      bool ok = true;
      for (int pass = 0; ok && pass < kMaxPasses; ++pass) {
        const int ex = pass_exists(sh, pass, a.status);
        if (ex < 0) { report(a.status, SGQA_ERR_TIMEOUT); sh->abort_flag = 1; ok = false; break; }
        if (ex == 0) break;
        for (int i = 0; i < n_nt; ++i, ++k) {
          const int st = (int)(k % kStages);
          const uint32_t ph = (uint32_t)((k / kStages) & 1);
          if (k >= kStages && !tc::mbar_wait(&sh->empty[st], ph ^ 1u, &sh->abort_flag, a.status)) {
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
      bool ok = tc::mbar_wait(&sh->a_full, 0, &sh->abort_flag, a.status);
      if (!ok) {
        if (!sh->abort_flag) report(a.status, SGQA_ERR_TIMEOUT);
        sh->abort_flag = 1;
      }
      const uint64_t da = tc::smem_desc_kmajor(sA, C::kRowBytes);
      long k = 0;
      for (int pass = 0; ok && pass < kMaxPasses; ++pass) {
        const int ex = pass_exists(sh, pass, a.status);
        if (ex < 0) { report(a.status, SGQA_ERR_TIMEOUT); sh->abort_flag = 1; ok = false; break; }
        if (ex == 0) break;
        for (int i = 0; i < n_nt; ++i, ++k) {
          const int st = (int)(k % kStages);
          const uint32_t ph = (uint32_t)((k / kStages) & 1);
          const int buf = (int)(k & 1);
          if (!tc::mbar_wait(&sh->full[st], ph, &sh->abort_flag, a.status) ||
              (k >= 2 && !tc::mbar_wait(&sh->acc_empty[buf], (uint32_t)(((k >> 1) - 1) & 1), &sh->abort_flag, a.status))) {
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
    // ---------------- epilogue: one row per four threads ----------------
    // Warps w, w + 4, w + 8, w + 12 read TMEM lane quadrant w % 4 (row r = 32 * (w % 4) + lane);
    // warp w takes columns 32 * (w / 4) .. + 31 of every tile, in the histogram passes and in
    // the emit pass.
    const int quad = warp & 3, part = warp >> 2;
    const int r = quad * 32 + lane;
    const int t = tq0 + r / G, g = r % G;
    const bool valid = t <= t_last;
    const int c = valid ? t / a.B : 0;
    const int m = valid ? min(a.Kb - 1, c) : 0;
    uint32_t prefix = 0, mask = 0;
    int rem = m, nb = c;
    bool done = (rem == nb);
    if (rem == 0) { prefix = 0xFFFFFFFFu; mask = 0xFFFFFFFFu; done = true; }
    // the row's words are stored bin-major: word w of row r at hist[w * kRows + r], so the lanes of
    // a warp (32 consecutive rows) always address 32 different banks, whatever bins their keys
    // fall in (row-major rows collided whenever neighbouring rows' keys fell in nearby bins)
    uint32_t* my_hist = hist + r;
    // the row's bitmap of taken candidates (bit j of word j / 32)
    uint32_t* brow = a.bits + (((long)b * (a.t_end - a.t_begin) + (t - a.t_begin)) * G + g) * (long)a.bstride;
    const uint32_t lane_base = (uint32_t)(32 * quad) << 16;
    const uint32_t hbase = smem_u32(my_hist);
    long k = 0;
    bool aborted = false, emitted = false, collect = false;
    int eqn = 0, taken = 0;
    for (int pass = 0; pass < kMaxPasses; ++pass) {
      // zero the histograms for this pass (a resolved row: its tie-count slots), then a
      // barrier+vote: is any row still unresolved?
      if (part == 0 && !done && pass < kMaxPasses - 1)
        for (int i = 0; i < 256; ++i) my_hist[i * kRows] = 0;
      if (part == 0 && done)
        for (int i = 0; i < kTieWords; ++i) my_hist[i * kRows] = 0;
      const int vote = epi_vote_any(sh, 4 * pass, !done, a.status);
      // from the third pass on, if every unresolved row's threshold bucket is small, this pass is
      // the last: it also collects those buckets' keys, which are then resolved exactly
      const int vote_big = (pass >= 2 && vote > 0) ? epi_vote_any(sh, 4 * pass + 3, !done && nb > kCap, a.status) : 1;
      if (vote < 0 || vote_big < 0) {
        if (lane == 0 && !sh->abort_flag) report(a.status, SGQA_ERR_TIMEOUT);
        sh->abort_flag = 1;
        aborted = true;
        break;
      }
      const bool is_emit = vote == 0 || vote_big == 0 || pass == kMaxPasses - 1;
      if (warp == 0 && lane == 0) {
        sh->more[pass] = is_emit ? 0 : 1;
        __threadfence_block();
        sh->signals = pass + 1;
      }
      if (!is_emit) {
        const int shift = 24 - 8 * pass;
        // a resolved row counts too, harmlessly: its histogram is not read, and its tie-count
        // slots are zeroed at the start of the emit pass
        const uint32_t pf = raw_prefix(prefix, mask);
        for (int i = 0; i < n_nt; ++i, ++k) {
          const int buf = (int)(k & 1);
          if (!warp_wait(&sh->acc_full[buf], (uint32_t)((k >> 1) & 1), &sh->abort_flag, a.status)) {
            if (lane == 0 && !sh->abort_flag) report(a.status, SGQA_ERR_TIMEOUT);
            sh->abort_flag = 1;
            aborted = true;
            break;
          }
          tc::fence_after_sync();
          uint32_t v[kCols];
          tc::tmem_ld32(tmem + lane_base + (uint32_t)(buf * kN + part * kCols), v);
          tc::fence_before_sync();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&sh->acc_empty[buf]);
          const int lim = c - (i * kN + part * kCols);
          if (__all_sync(0xFFFFFFFFu, lim >= kCols)) {
            if (pass == 0) hist_chunk<true, true>(v, lim, pf, shift, hbase);
            else hist_chunk<true, false>(v, lim, pf, shift, hbase);
          } else if (lim > 0) {
            if (pass == 0) hist_chunk<false, true>(v, lim, pf, shift, hbase);
            else hist_chunk<false, false>(v, lim, pf, shift, hbase);
          }
        }
        if (aborted) break;
        // every part's histogram updates are complete before any reads the histogram
        if (epi_vote_any(sh, 4 * pass + 1, false, a.status) < 0) {
          if (lane == 0 && !sh->abort_flag) report(a.status, SGQA_ERR_TIMEOUT);
          sh->abort_flag = 1;
          aborted = true;
          break;
        }
        if (!done) {
          int above = 0;
          for (int bin = 255; bin >= 0; --bin) {
            const int h = (int)my_hist[raw_bin(bin, pass == 0, (prefix & 0x80000000u) == 0u) * kRows];
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
        // every part has read the histogram before the next pass zeroes it
        if (epi_vote_any(sh, 4 * pass + 2, false, a.status) < 0) {
          if (lane == 0 && !sh->abort_flag) report(a.status, SGQA_ERR_TIMEOUT);
          sh->abort_flag = 1;
          aborted = true;
          break;
        }
        continue;
      }

      // ---- emit pass: this part's kCols columns of every tile become one bitmap word ----
      // rule of this row: take keys >= thr; the bucket [blo, blo + bw] is collected (unresolved
      // row), taken whole (thr = prefix), or holds exact ties taken in j order up to rem
      const bool act = valid && m > 0;
      uint32_t thr = 0xFFFFFFFFu, blo = 0xFFFFFFFFu, bw = 0u;
      bool ties = false;
      if (act) {
        if (!done) {
          const uint32_t pend = prefix | ~mask;
          thr = pend == 0xFFFFFFFFu ? 0xFFFFFFFFu : pend + 1u;
          blo = prefix;
          bw = ~mask;
          collect = true;
        } else if (rem == nb) {
          thr = prefix;
        } else {
          thr = prefix == 0xFFFFFFFFu ? 0xFFFFFFFFu : prefix + 1u;
          blo = prefix;
          ties = true;
        }
      }
      // identical in the kParts warps of a row group (same rows, same state)
      const bool any_bucket = __any_sync(0xFFFFFFFFu, collect || ties);
      // every row of the warp has a positive threshold (and bucket): raw-bit comparisons
      const bool pos = __all_sync(0xFFFFFFFFu, thr > 0x80000000u && blo >= 0x80000000u);
      const bool any_ties = __any_sync(0xFFFFFFFFu, ties);
      uint32_t* cand = my_hist + part * kCandWords * kRows;  // this part's collected (key, j) pairs (stride kRows)
      volatile uint32_t* slot = my_hist;                     // tie counts: [part][tile parity] (stride kRows)
      int run = 0;  // exact ties before this part's columns of the tile
      for (int i = 0; i < n_nt; ++i, ++k) {
        const int buf = (int)(k & 1);
        if (!warp_wait(&sh->acc_full[buf], (uint32_t)((k >> 1) & 1), &sh->abort_flag, a.status)) {
          if (lane == 0 && !sh->abort_flag) report(a.status, SGQA_ERR_TIMEOUT);
          sh->abort_flag = 1;
          aborted = true;
          break;
        }
        tc::fence_after_sync();
        const int j0 = i * kN + part * kCols;
        const int lim = act ? c - j0 : 0;
        uint32_t tb = 0u, bb = 0u;
        if (__any_sync(0xFFFFFFFFu, lim > 0)) {
          uint32_t v[kCols];
          tc::tmem_ld32(tmem + lane_base + (uint32_t)(buf * kN + part * kCols), v);
          const bool full = __all_sync(0xFFFFFFFFu, lim >= kCols);
          if (any_bucket) {
            if (full && pos) emit_bits<true, true, true>(v, lim, thr, blo, bw, tb, bb);
            else if (full) emit_bits<true, true, false>(v, lim, thr, blo, bw, tb, bb);
            else emit_bits<false, true, false>(v, lim, thr, blo, bw, tb, bb);
          } else {
            if (full && pos) emit_bits<true, false, true>(v, lim, thr, blo, bw, tb, bb);
            else if (full) emit_bits<true, false, false>(v, lim, thr, blo, bw, tb, bb);
            else emit_bits<false, false, false>(v, lim, thr, blo, bw, tb, bb);
          }
          if (collect) {  // the few bucket keys of an unresolved row, kept as (key, j) pairs
            uint32_t bits = bb;
            while (bits) {
              const int q = __ffs(bits) - 1;
              bits &= bits - 1u;
              if (eqn < kCap) {
                cand[(2 * eqn) * kRows] = score_key(__uint_as_float(pick32(v, q)));
                cand[(2 * eqn + 1) * kRows] = (uint32_t)(j0 + q);
              }
              ++eqn;
            }
          }
        }
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&sh->acc_empty[buf]);
        if (any_ties) {
          // exact ties in j order: in tile i the parts' columns run part 0, 1, ..., so a part
          // counts the ties of the lower parts in tile i and of the higher parts in tile i - 1
          // (its own and all earlier tiles are already in run). Each part publishes its count
          // for tile i before it waits, so the waits only reach back to earlier publications.
          const int cnt = ties ? __popc(bb) : 0;
          int got = 0;
          if (ties) {
            slot[(2 * part + (i & 1)) * kRows] = ((uint32_t)(i + 1) << 8) | (uint32_t)cnt;
            for (int q = 0; q < kParts && got >= 0; ++q) {
              if (q == part || (q > part && i == 0)) continue;
              const int ti = q < part ? i : i - 1;
              const int x = wait_tie_count(slot + (2 * q + (ti & 1)) * kRows, (uint32_t)(ti + 1), sh, a.status);
              if (x < 0) got = -1;
              else run += x;
            }
          }
          if (__any_sync(0xFFFFFFFFu, got < 0)) {
            if (lane == 0 && !sh->abort_flag) report(a.status, SGQA_ERR_TIMEOUT);
            sh->abort_flag = 1;
            aborted = true;
            break;
          }
          if (ties) {
            tb |= first_bits(bb, rem - run);
            run += cnt;
          }
        }
        if (lim > 0 && SGQA_CHECK((j0 >> 5) < a.bstride && t < a.t_end, a.status)) brow[j0 >> 5] = tb;
        taken += __popc(tb);
      }
      if (!aborted && part > 0 && act) {
        my_hist[(kCntBase + 2 * (part - 1)) * kRows] = (uint32_t)eqn;
        my_hist[(kCntBase + 2 * (part - 1) + 1) * kRows] = (uint32_t)taken;
      }
      emitted = !aborted;
      break;
    }
    // every epilogue warp gets here (all waits above are bounded): the bitmap words and the
    // collected keys of all parts are complete
    asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory");
    if (emitted && part == 0 && act_row(valid, m) && !sh->abort_flag) {
      int total = taken;
      int ncol[kParts];
      ncol[0] = eqn;
#pragma unroll
      for (int p = 1; p < kParts; ++p) {
        total += (int)my_hist[(kCntBase + 2 * (p - 1) + 1) * kRows];
        ncol[p] = (int)my_hist[(kCntBase + 2 * (p - 1)) * kRows];
      }
      if (collect) {
        // the collected bucket keys of all parts: key x ranks behind every larger key and every
        // equal key of lower j, and is taken when fewer than rem rank ahead of it
#pragma unroll
        for (int p = 0; p < kParts; ++p) {
          if (ncol[p] > kCap) report(a.status, SGQA_ERR_DEVICE_CHECK);
          ncol[p] = min(ncol[p], kCap);
        }
        for (int px = 0; px < kParts; ++px) {
          for (int x = 0; x < ncol[px]; ++x) {
            const uint32_t* cx = my_hist + (px * kCandWords + 2 * x) * kRows;
            const uint32_t kx = cx[0], jx = cx[kRows];
            int ahead = 0;
            for (int py = 0; py < kParts; ++py) {
              for (int y = 0; y < ncol[py]; ++y) {
                const uint32_t* cy = my_hist + (py * kCandWords + 2 * y) * kRows;
                ahead += (cy[0] > kx || (cy[0] == kx && cy[kRows] < jx)) ? 1 : 0;
              }
            }
            if (ahead < rem && SGQA_CHECK(jx < (uint32_t)c && (int)(jx >> 5) < a.bstride, a.status)) {
              atomicOr(brow + (jx >> 5), 1u << (jx & 31u));
              ++total;
            }
          }
        }
      }
      if (total != m) report(a.status, SGQA_ERR_DEVICE_CHECK);
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

// The selection from the bitmaps: per (token, group) row, the set bits of words [0, ceil(c/32))
// in ascending order (m of them), then the own block c, then -1 up to Kb. One warp per row: the
// lanes load 32 words at a time and a warp scan of their population counts gives each word's
// output position; then the warp expands the non-zero words one at a time, lane b writing the
// index of bit b when it is set (one coalesced store per word, no per-lane loops over bits).
__global__ void __launch_bounds__(256) sel_from_bits_kernel(SelectArgs a) {
  const long row = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int nq = a.t_end - a.t_begin;
  if (row >= (long)a.batch * nq * a.G) return;
  const int g = (int)(row % a.G);
  const long bt = row / a.G;
  const int t = a.t_begin + (int)(bt % nq);
  const int b = (int)(bt / nq);
  const int c = t / a.B, m = min(a.Kb - 1, c);
  const uint32_t* bits = a.bits + row * (long)a.bstride;
  int32_t* out = a.sel + (((long)b * a.sel_T + (t - a.sel_t0)) * a.G + g) * (long)a.Kb;
  const int nw = m > 0 && SGQA_CHECK(((c + 31) >> 5) <= a.bstride, a.status) ? (c + 31) >> 5 : 0;
  const uint32_t below = (1u << lane) - 1u;
  int pos = 0;
  for (int w0 = 0; w0 < nw && pos < m; w0 += 32) {
    const int w = w0 + lane;
    const uint32_t x = w < nw ? __ldg(bits + w) : 0u;
    const int n = __popc(x);
    int inc = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, inc, o);
      if (lane >= o) inc += y;
    }
    const int start = pos + inc - n;  // output position of this lane's word
    unsigned nz = __ballot_sync(0xFFFFFFFFu, x != 0u);
    while (nz) {
      const int L = __ffs(nz) - 1;
      nz &= nz - 1u;
      const uint32_t xw = __shfl_sync(0xFFFFFFFFu, x, L);
      const int p = __shfl_sync(0xFFFFFFFFu, start, L) + __popc(xw & below);
      if (((xw >> lane) & 1u) && p < m) out[p] = 32 * (w0 + L) + lane;
    }
    pos += __shfl_sync(0xFFFFFFFFu, inc, 31);
  }
  if (pos != m && lane == 0) report(a.status, SGQA_ERR_DEVICE_CHECK);
  for (int i = min(pos, m) + lane; i < a.Kb; i += 32) out[i] = i == m ? c : -1;
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
  if (!make_map(&mq, a.q_idx, (long)a.batch * a.q_T * a.G, DI, kRows) ||
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

void select_bits_dims(int batch, int T, int G, int B, size_t budget, int* bstride, int* bits_q) {
  const long nblk = T / B;
  *bstride = (int)(4 * ((nblk + kN - 1) / kN));  // whole tiles: a tile's word per part stays in the row
  const size_t per_q = (size_t)batch * G * (size_t)*bstride * 4;
  long q = per_q ? (long)(budget / per_q) : (long)T;
  q = q / 128 * 128;  // whole K2 tiles (128 / G tokens) per range
  if (q < 128) q = 128;
  if (q > T) q = T;
  *bits_q = (int)q;
}

cudaError_t launch_select(const SelectArgs& a, cudaStream_t s) {
  if (a.t_end <= a.t_begin) return cudaSuccess;
  if (a.T / a.B == 0) {
    own_block_only_kernel<<<148, 256, 0, s>>>(a);
    return cudaGetLastError();
  }
  if ((a.d_idx != 64 && a.d_idx != 32) || !a.bits || a.bits_q <= 0) return cudaErrorInvalidValue;
  // query ranges of at most bits_q rows, each: scores + select into the bitmaps, then the lists
  for (int t0 = a.t_begin; t0 < a.t_end; t0 += a.bits_q) {
    SelectArgs p = a;
    p.t_begin = t0;
    p.t_end = a.t_end - t0 > a.bits_q ? t0 + a.bits_q : a.t_end;
    cudaError_t e = a.d_idx == 64 ? launch_di<64>(p, s) : launch_di<32>(p, s);
    if (e != cudaSuccess) return e;
    const long rows = (long)p.batch * (p.t_end - p.t_begin) * p.G;
    sel_from_bits_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace sgqa
