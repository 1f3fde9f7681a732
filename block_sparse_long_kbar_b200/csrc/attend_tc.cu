// K3 on the 5th-generation tensor cores: gated attention for a tile of 128 query rows (128/R
// queries x R heads of one KV group) over the union of their selected blocks.
//
// Step 5 Preview pages (mo.ai.kr, "Step 5 Preview agentic work design", section "model
// structure and training stability"): the full-context layer is Sparse GQA on top of Gated GQA;
// every KV group attends only to its selected blocks, and queries whose selections overlap are
// batched for GPU utilisation. The rows of a tile come from the scheduling permutation (plan.cu)
// that puts rows with similar selections together.
//
// Data movement and math:
//   * Q tile: 128 rows x d bf16 in shared memory (K-major, 128B swizzle), loaded once.
//   * The union of the tile's selections is built window by window over block ids (a shared
//     bitmap of 32-bit query masks per block) and consumed as 16-token superblocks aligned on
//     block ids, four per chunk. Each chunk's K and V rows of the group arrive by 3-D TMA boxes
//     (64 dims x 16, 32 or 64 tokens, 128B swizzle) into a 2-stage K ring and a 2-stage V ring
//     (a K stage is reused as soon as Q K^T has read it). A run of consecutive superblock ids in
//     a chunk (the common case: selections cluster) is fetched by one box per 64-dim half, since
//     every box costs the issuing thread about 100 cycles whatever its size; a missing
//     superblock of the last chunk is loaded from out of bounds, which fills zeros.
//   * S[128 x 64] = Q K^T per chunk: tcgen05.mma (kind::f16, M=128, N=64) into TMEM, double
//     buffered.
//   * Softmax: two threads per row (TMEM lane); the thread with shalf = (superblock id & 1)
//     takes a superblock. Masks from the bitmap (the query selected the block, token <= query
//     position). Every row is scaled by a reference maximum computed up front on the CUDA cores
//     from its own block (always selected), so there is a single streaming pass and no rescaling
//     of O: P = exp2((S - m_ref) log2(e) / sqrt(d)), rounded to bf16 and written back into TMEM
//     over the superblock's first 8 S columns. A row whose sum of P exceeds 2^60 or is not finite
//     is flagged, and if any row is, the tile streams the union again for exact maxima and then
//     repeats the main pass (flagged rows with their exact maximum, the others with exactly the
//     same arithmetic as before).
//   * O[128 x d] += P V with tcgen05.mma, P read from TMEM (A operand) and V from shared memory
//     (an MN-major operand), one K=16 step per superblock. The row sums l add the fp32 values of
//     P (before their rounding to bf16, which changes l by at most 2^-9 relative) on the CUDA
//     cores: each thread sums its superblocks (one id parity) in ascending id order and
//     l = l_even + l_odd. Because superblocks are aligned on block ids, each is one K=16
//     accumulation step and one parity class, and unselected slots contribute exact zeros, every
//     row's arithmetic is the same whatever rows share its tile (bitwise causal, chunk-invariant).
//   * Epilogue: O / l times sigmoid(gate_logits), bf16.
// Warp roles: warp 0 issues TMA, warp 1 allocates TMEM and issues MMAs (Q K^T of a chunk and
// P V of an earlier one, whichever is ready first; neither role blocks on one barrier while the
// other kind of work could proceed; an S/P buffer is refilled only after the P V that reads it
// has been issued, and MMAs of one thread execute in issue order), warps 2-9 run the softmax and
// the epilogue; all ten build the union. Two tiles are resident per SM (shared memory and TMEM
// are sized for it), so one tile's union, setup and epilogue overlap the other's chunks. Every
// wait is bounded by %globaltimer: on expiry the kernel records SGQA_ERR_TIMEOUT, drains its own
// copies and MMAs, frees TMEM and returns.
#include <cmath>
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace sgqa {
namespace {

constexpr int kUnit = 16;    // tokens per superblock
constexpr int kCH = 4;       // superblocks per chunk (one handshake between MMA and softmax)
constexpr int kCT = kCH * kUnit;  // token slots per chunk
constexpr int kWin = 1024;   // block ids per union window
constexpr int kWinWords = 16;     // occupancy bits for up to 512 windows
constexpr int kNK = 2;       // K chunk stages
constexpr int kNV = 2;       // V chunk stages
constexpr int kSmWarps = 8;  // softmax warps: two per TMEM lane quadrant
constexpr int kThreads = (2 + kSmWarps) * 32;
constexpr int kCtasPerSm = 2;  // two tiles resident per SM: one's union, setup and epilogue overlap
                               // the other's chunk loop
constexpr int kM = 128;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRiskSum = 1.152921504606846976e18f;  // 2^60: a row whose sum of P (scaled by its
                                                     // reference maximum) exceeds this, or is not
                                                     // finite, is recomputed with its exact maximum

template <int D>
struct AtcCfg {
  static constexpr int kHalves = D / 64;
  static constexpr int kQ = kM * D * 2;                 // [half][128 rows][128 B]
  static constexpr int kHalfRows = kCT * 128;           // one 64-dim half of a chunk: [kCT tokens][128 B]
  static constexpr int kKc = kHalves * kHalfRows;       // K (or V) of one chunk: [half][kCT][128 B]
  static constexpr int kSmem = 1024 + kQ + (kNK + kNV) * kKc + 2 * kWin * 4 + 4096;
  static_assert(kCtasPerSm * (kSmem + 1024) <= 233472, "shared memory for the resident tiles");
  static constexpr int kSCols = 2 * kCT;                // TMEM: two S/P buffers, then O (D)
  static constexpr int kTmemCols = kSCols + D <= 256 ? 256 : 512;
  static_assert(kCtasPerSm * kTmemCols <= 512, "TMEM for the resident tiles");
};

// K and V maps with boxes of 16, 32 and 64 tokens (one, two or four superblocks); boxes longer
// than the tensor's token count are not encoded and not used (max_run).
struct KvMaps {
  CUtensorMap k[3], v[3];
  int max_run;  // largest usable box: 16 << max_run tokens
};

struct AtcShared {
  uint64_t k_full[kNK], k_empty[kNK], v_full[kNV], v_empty[kNV], s_full[2], p_full[2], o_done;
  float ref_part[2][kM];  // per-row reference maxima from the own block (two halves of its tokens)
  float max_part[2][kM];  // per-row exact maxima by superblock parity (fallback pass)
  float l_part[2][kM];    // per-row sums of P by superblock parity
  uint32_t wbits[kWinWords];
  uint32_t tmem;
  volatile int abort_flag;
  int t[32];
  int scan[kThreads / 32];
  int nu, maxc, all_windows;
};
static_assert(sizeof(AtcShared) <= 4096, "the shared-memory budget reserves 4 KB for AtcShared");

// Idle step of a polling role (producer, MMA issuer): sleep briefly; every 256 idle rounds check
// for a grid-wide timeout and for no progress within the wait limit (then record the timeout and
// raise the CTA's abort flag). Returns false when the role must stop.
__device__ __forceinline__ bool poll_idle(uint32_t spins, uint64_t t_prog, AtcShared* sh, int* gstatus) {
  if ((spins & 255u) == 0u) {
    if (tc::grid_timed_out(gstatus)) {
      sh->abort_flag = 1;
      return false;
    }
    if (tc::globaltimer() - t_prog > tc::kWaitLimitNs) {
      if (!sh->abort_flag) report(gstatus, SGQA_ERR_TIMEOUT);
      sh->abort_flag = 1;
      return false;
    }
  }
  __nanosleep(20);
  return true;
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, const int* gstatus) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = tc::mbar_wait(bar, parity, abort, gstatus) ? 1 : 0;
  return __shfl_sync(0xFFFFFFFFu, ok, 0) != 0;
}

// Visit every valid entry of a query's selection row (strictly ascending block ids <= cq, then -1
// padding), 512 entries per batch with all loads in flight; fn(j) per valid entry. Entries that
// break the format are skipped (and reported when `report_errors`). Must be called by a whole warp.
template <class Fn>
__device__ __forceinline__ void for_each_selected(const int32_t* row, int Kb, int cq, int stop_at, bool report_errors,
                                                  int* status, Fn fn) {
  const int lane = threadIdx.x & 31;
  int before_batch = -1;
  for (int base = 0; base < Kb; base += 512) {
    int jv[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int e = base + i * 32 + lane;
      jv[i] = e < Kb ? __ldg(row + e) : -1;
    }
    bool stop = false;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      int j = jv[i];
      // both shuffles are warp-collective: every lane executes them
      const int prev = __shfl_up_sync(0xFFFFFFFFu, j, 1);
      const int last_prev = __shfl_sync(0xFFFFFFFFu, i > 0 ? jv[i > 0 ? i - 1 : 0] : before_batch, 31);
      const int before = lane > 0 ? prev : last_prev;
      if (j > cq || j < -1 || (j >= 0 && j <= before)) {
        if (report_errors) report(status, SGQA_ERR_DEVICE_CHECK);
        j = -1;
      }
      if (j >= 0 && j < stop_at) fn(j);
      jv[i] = j;
      stop |= __any_sync(0xFFFFFFFFu, j < 0 || j >= stop_at);
    }
    before_batch = __shfl_sync(0xFFFFFFFFu, jv[15], 31);
    if (stop) break;
  }
}

template <int D, int R>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    attend_tc_kernel(const __grid_constant__ KvMaps maps, AttendArgs a, const uint32_t* __restrict__ perm,
                     int n_per_seg, int tiles_per_seg, int lb) {
  using C = AtcCfg<D>;
  constexpr int QT = kM / R;  // queries per tile (<= 32)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align<1024>(smem_raw);
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + C::kQ;                              // [kNK][half][kCT tokens][128 B]
  uint8_t* sV = sK + kNK * C::kKc;                       // [kNV][half][kCT tokens][128 B]
  uint32_t* wmask = reinterpret_cast<uint32_t*>(sV + kNV * C::kKc);
  int32_t* usb = reinterpret_cast<int32_t*>(wmask + kWin);
  AtcShared* sh = reinterpret_cast<AtcShared*>(usb + kWin);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int B = a.B, G = a.G;
  const int seg = blockIdx.x / tiles_per_seg, tile = blockIdx.x % tiles_per_seg;
  const int b = seg / G, g = seg % G;

  // a timeout recorded by another CTA (this launch or an earlier one sharing the status word):
  // do nothing (the decision is the CTA's, before any barrier or TMEM is set up)
  if (__syncthreads_or(tid == 0 && tc::grid_timed_out(a.status))) return;
  if (tid == 0) {
    for (int i = 0; i < kNK; ++i) {
      tc::mbar_init(&sh->k_full[i], 1);
      tc::mbar_init(&sh->k_empty[i], 1);
    }
    for (int i = 0; i < kNV; ++i) {
      tc::mbar_init(&sh->v_full[i], 1);
      tc::mbar_init(&sh->v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&sh->s_full[i], 1);
      tc::mbar_init(&sh->p_full[i], kSmWarps);
    }
    tc::mbar_init(&sh->o_done, 1);
    sh->abort_flag = 0;
    sh->maxc = -1;
    sh->all_windows = 0;
    tc::fence_mbar_init();
  }
  if (tid < kWinWords) sh->wbits[tid] = 0;
  for (int i = tid; i < kWin; i += kThreads) wmask[i] = 0;
  __syncthreads();
  if (tid < QT) {
    const int idx = tile * QT + tid;
    int t = idx < n_per_seg ? a.t_begin + (int)__ldg(perm + (long)seg * n_per_seg + idx) : -1;
    // the permutation maps the tile's slots onto the query range, and q rows exist for it
    if (t >= 0 && !SGQA_CHECK(t < a.t_end && t - a.q_t0 >= 0 && t - a.q_t0 < a.nQ, a.status)) t = -1;
    sh->t[tid] = t;
    if (t >= 0) atomicMax(&sh->maxc, t / B);
  }
  if (warp == 1) tc::tmem_alloc(&sh->tmem, C::kTmemCols);

  // Q tile: row r = query r / R, head r % R; 16-byte chunk c of half h at
  // h * 16 KB + r * 128 + ((c ^ (r & 7)) * 16) (the 128B-swizzled K-major layout).
  __syncthreads();
  for (int idx = tid; idx < kM * (D / 8); idx += kThreads) {
    const int r = idx / (D / 8), cc = idx % (D / 8);
    const int h = cc >> 3, c = cc & 7;
    const int tq = sh->t[r / R];
    const long row = tq >= 0 ? ((long)b * a.nQ + (tq - a.q_t0)) * a.Hq + (long)g * R + (r % R) : 0;
    cp_async16(smem_u32(sQ + h * (kM * 128) + r * 128 + ((c ^ (r & 7)) * 16)), a.q + row * D + cc * 8,
               tq >= 0 ? 16 : 0);
  }
  cp_async_commit();
  // which windows hold any selected block (each row read once; format errors reported here)
  const int nwin = sh->maxc < 0 ? 0 : sh->maxc / kWin + 1;
  if (nwin > 32 * kWinWords) {
    if (tid == 0) sh->all_windows = 1;
  } else {
    for (int q = warp; q < QT; q += kThreads / 32) {
      const int t = sh->t[q];
      if (t < 0) continue;
      const int32_t* row = a.sel + (((long)b * a.sel_T + (t - a.sel_t0)) * G + g) * (long)a.Kb;
      for_each_selected(row, a.Kb, t / B, 0x7FFFFFFF, true, a.status, [&](int j) {
        // most entries fall in a window already marked: read first (lanes reading one word are
        // served at once), so that only the first entries of a window pay for an atomic
        const int w = j / kWin;
        const uint32_t bit = 1u << (w & 31);
        if (!(*reinterpret_cast<volatile uint32_t*>(&sh->wbits[w >> 5]) & bit)) atomicOr(&sh->wbits[w >> 5], bit);
      });
    }
  }
  cp_async_wait<0>();
  tc::fence_proxy_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = sh->tmem;
  const uint32_t tmem_o = tmem + C::kSCols;  // O: D columns after the two S/P buffers

  // softmax role state (warps 2..9): TMEM lane quadrant warp % 4; `shalf` also picks the
  // half of every chunk (superblocks 2 shalf, 2 shalf + 1) and the own-block tokens this thread
  // handles
  const bool is_sm = warp >= 2;
  const int quad = warp & 3;
  const int shalf = is_sm ? (warp - 2) / 4 : 0;
  const int r = quad * 32 + lane;
  const int q_r = r / R, h_r = r % R;
  const int t_r = is_sm ? sh->t[q_r] : -1;
  // lowest key position the row may attend to (Gated SWA); -1 (below every key) without a window,
  // so that lo_r - u0 cannot overflow
  const int lo_r = (a.window > 0 && t_r >= 0) ? t_r - a.window + 1 : -1;
  const float sc = kLog2e / sqrtf((float)D);
  const uint32_t lane_base = (uint32_t)(32 * quad) << 16;

  // reference maximum of the row: its scores against its own block (always selected, u <= t),
  // computed on the CUDA cores from the same bf16 operands; a function of the row alone
  if (is_sm) {
    float mx = -INFINITY;
    if (t_r >= 0) {
      const int u_lo = (t_r / B) * B;
      const uint8_t* qrow = sQ + r * 128;
      for (int u = u_lo + shalf; u <= t_r; u += 2) {
        const uint16_t* krow = a.k + (((long)b * a.T_kv + u) * G + g) * D;
        float acc = 0.f;
#pragma unroll
        for (int cc = 0; cc < D / 8; ++cc) {
          const int h = cc >> 3, c = cc & 7;
          const uint4 qv = *reinterpret_cast<const uint4*>(qrow + h * (kM * 128) + ((c ^ (r & 7)) * 16));
          const uint4 kv = __ldg(reinterpret_cast<const uint4*>(krow + cc * 8));
          const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w}, kw[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            acc = fmaf(bf16_lo(qw[i]), bf16_lo(kw[i]), acc);
            acc = fmaf(bf16_hi(qw[i]), bf16_hi(kw[i]), acc);
          }
        }
        mx = fmaxf(mx, acc);
      }
    }
    sh->ref_part[shalf][r] = mx;
  }
  __syncthreads();
  const float m_ref = is_sm ? fmaxf(sh->ref_part[0][r], sh->ref_part[1][r]) : -INFINITY;
  float m_use = m_ref, m_exact = -INFINITY;
  bool risky = false;  // this row's P sum exceeds kRiskSum (some exponent is near the fp32 range)
  bool o_ok = false;   // this thread saw the last main pass's MMAs complete
  int o_phase = 0, o_commits = 0;

  const int spb = kUnit >> lb;  // blocks per superblock
  long kck = 0, kcv = 0;        // K and V ring positions (producer & MMA: chunks loaded / consumed)
  long scnt = 0;                // S/P buffer uses (MMA: Q K^T issued; softmax: chunks processed)
  long pcnt = 0;                // S/P buffer uses whose P (or exact-max pass) the MMA issuer consumed
  const uint32_t idesc_s = tc::idesc_bf16_f32(kM, kCT);
  const uint32_t idesc_pv = tc::idesc_bf16_f32(kM, D, true);
  bool rerun = false;
  float l_sum = 0.f;            // this thread's sum of P (its superblock parity), per main pass

  // pass 0: main (P V with the reference maximum); passes 1-2 only if some row was risky:
  // exact maxima, then the main pass again (risky rows use their exact maximum, all other rows
  // repeat exactly the same arithmetic as in pass 0).
  for (int pass = 0; pass < 3; ++pass) {
    if (pass == 1 && !rerun) break;
    const bool main_pass = pass != 1;
    bool first_pv = true;
    if (main_pass && pass == 2) m_use = risky ? m_exact : m_ref;
    l_sum = 0.f;
    for (int win = 0; win < nwin; ++win) {
      if (!sh->all_windows && !((sh->wbits[win >> 5] >> (win & 31)) & 1u)) continue;  // uniform
      const int w0 = win * kWin, w1 = w0 + kWin;
      // ---- union of this window (all warps) ----
      for (int q = warp; q < QT; q += kThreads / 32) {
        const int t = sh->t[q];
        if (t < 0) continue;
        const int32_t* row = a.sel + (((long)b * a.sel_T + (t - a.sel_t0)) * G + g) * (long)a.Kb;
        for_each_selected(row, a.Kb, t / B, w1, false, a.status, [&](int j) {
          if (j >= w0) atomicOr(&wmask[j - w0], 1u << q);
        });
      }
      __syncthreads();
      {
        const int nsb_win = kWin / spb;
        const int per = (nsb_win + kThreads - 1) / kThreads;
        const int sb0 = min(nsb_win, tid * per), sb1 = min(nsb_win, sb0 + per);
        int cnt = 0;
        for (int sb = sb0; sb < sb1; ++sb) {
          uint32_t any = 0;
          for (int i = 0; i < spb; ++i) any |= wmask[sb * spb + i];
          cnt += any != 0u;
        }
        int x = cnt;
#pragma unroll
        for (int o2 = 1; o2 < 32; o2 <<= 1) {
          const int y = __shfl_up_sync(0xFFFFFFFFu, x, o2);
          if (lane >= o2) x += y;
        }
        if (lane == 31) sh->scan[warp] = x;
        __syncthreads();
        if (tid == 0) {
          int run = 0;
          for (int w = 0; w < kThreads / 32; ++w) {
            const int v = sh->scan[w];
            sh->scan[w] = run;
            run += v;
          }
          sh->nu = run;
        }
        __syncthreads();
        int pos = sh->scan[warp] + x - cnt;
        for (int sb = sb0; sb < sb1; ++sb) {
          uint32_t any = 0;
          for (int i = 0; i < spb; ++i) any |= wmask[sb * spb + i];
          if (any) {
            // a superblock holding a selected block starts inside the sequence (recorded only:
            // the TMA fetch of any coordinate is safe, out-of-range tokens read zeros)
            (void)SGQA_CHECK(((w0 >> (4 - lb)) + sb) * kUnit < a.T_kv, a.status);
            usb[pos++] = (w0 >> (4 - lb)) + sb;
          }
        }
      }
      __syncthreads();
      const int nu = sh->nu;
      const int nch = (nu + kCH - 1) / kCH;

      if (warp == 0) {
        // ---- TMA producer: one chunk = kCH superblocks; missing ones (partial last chunk) are
        // loaded from out of bounds, which fills zeros. K and V have rings of their own (a K
        // stage is free once Q K^T has read it, a V stage once P V has), and the thread issues
        // whichever load has a free stage, never blocking on one ring while the other could
        // move. ----
        if (lane == 0) {
          int nk = 0, nv = 0;
          uint64_t t_prog = tc::globaltimer();
          uint32_t spins = 0;
          // one chunk of K or V: a box per run of consecutive superblock ids (4, 2 or 1 of them,
          // aligned in the chunk) and 64-dim half
          auto load_chunk = [&](uint8_t* dst, const CUtensorMap* m, uint64_t* bar, int chunk) {
            const int e0 = chunk * kCH;
            for (int i = 0; i < kCH;) {
              const int e = e0 + i;
              int mi = 0;  // box of 16 << mi tokens
              if (e < nu) {
                if (maps.max_run >= 2 && i == 0 && e + 3 < nu && usb[e + 3] == usb[e] + 3) mi = 2;
                else if (maps.max_run >= 1 && (i & 1) == 0 && e + 1 < nu && usb[e + 1] == usb[e] + 1) mi = 1;
              }
              const int z = e < nu ? b * a.T_kv + usb[e] * kUnit : 0x7FFFFFF0;
#pragma unroll
              for (int h = 0; h < C::kHalves; ++h)
                tc::tma_load_3d(dst + h * C::kHalfRows + i * (kUnit * 128), &m[mi], bar, h * 64, g, z);
              i += 1 << mi;
            }
          };
          while (!sh->abort_flag && (nk < nch || (main_pass && nv < nch))) {
            bool prog = false;
            if (nk < nch && (kck < kNK || tc::mbar_try_wait(&sh->k_empty[kck % kNK], (uint32_t)(((kck / kNK) - 1) & 1)))) {
              const int st = (int)(kck % kNK);
              uint8_t* dst = sK + st * C::kKc;
              tc::mbar_arrive_expect_tx(&sh->k_full[st], C::kKc);
              load_chunk(dst, maps.k, &sh->k_full[st], nk);
              ++nk;
              ++kck;
              prog = true;
            }
            if (main_pass && nv < nk &&
                (kcv < kNV || tc::mbar_try_wait(&sh->v_empty[kcv % kNV], (uint32_t)(((kcv / kNV) - 1) & 1)))) {
              const int st = (int)(kcv % kNV);
              uint8_t* dst = sV + st * C::kKc;
              tc::mbar_arrive_expect_tx(&sh->v_full[st], C::kKc);
              load_chunk(dst, maps.v, &sh->v_full[st], nv);
              ++nv;
              ++kcv;
              prog = true;
            }
            if (prog) {
              t_prog = tc::globaltimer();
              spins = 0;
            } else if (!poll_idle(++spins, t_prog, sh, a.status)) {
              break;
            }
          }
        }
      } else if (warp == 1) {
        // ---- MMA issuer: Q K^T of the next chunk as soon as its K is there and the S/P buffer it
        // reuses has been read (its softmax done and, in a main pass, its P V issued: MMAs of this
        // thread execute in issue order), and P V of the oldest chunk whose P and V are there,
        // whichever is ready first ----
        if (lane == 0) {
          int nq = 0, np = 0;
          uint64_t t_prog = tc::globaltimer();
          uint32_t spins = 0;
          while (!sh->abort_flag && np < nch) {
            bool prog = false;
            if (nq < nch && nq < np + 2) {
              const int st = (int)(kck % kNK);
              const int sb = (int)(scnt & 1);
              if (tc::mbar_try_wait(&sh->k_full[st], (uint32_t)((kck / kNK) & 1))) {
                tc::fence_after_sync();
                const uint8_t* kst = sK + st * C::kKc;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                  const int h = kk >> 2, off = (kk & 3) * 32;
                  const uint64_t da = tc::smem_desc_kmajor(sQ + h * (kM * 128) + off, 128);
                  const uint64_t db = tc::smem_desc_kmajor(kst + h * C::kHalfRows + off, 128);
                  tc::mma_bf16_ss(tmem + (uint32_t)(sb * kCT), da, db, idesc_s, kk > 0 ? 1u : 0u);
                }
                tc::mma_commit(&sh->s_full[sb]);
                tc::mma_commit(&sh->k_empty[st]);
                ++nq;
                ++kck;
                ++scnt;
                prog = true;
              }
            }
            if (np < nq) {
              // chunk np: its S/P buffer is (pcnt & 1); pcnt counts buffer uses like scnt
              const int pb = (int)(pcnt & 1);
              const int st = (int)(kcv % kNV);
              if (tc::mbar_try_wait(&sh->p_full[pb], (uint32_t)((pcnt >> 1) & 1)) &&
                  (!main_pass || tc::mbar_try_wait(&sh->v_full[st], (uint32_t)((kcv / kNV) & 1)))) {
                tc::fence_after_sync();
                if (main_pass) {
                  const uint8_t* vbase = sV + st * C::kKc;
#pragma unroll
                  for (int i = 0; i < kCH; ++i) {
                    if (np * kCH + i >= nu) break;  // missing superblocks: P and V are zero
                    const uint32_t pa = tmem + (uint32_t)(pb * kCT + i * kUnit);
                    const uint64_t dv = tc::smem_desc_mnmajor_sw128(vbase + i * (kUnit * 128), C::kHalfRows, 1024);
                    tc::mma_bf16_ts(tmem_o, pa, dv, idesc_pv, first_pv ? 0u : 1u);
                    first_pv = false;
                  }
                  tc::mma_commit(&sh->v_empty[st]);
                  ++kcv;
                }
                ++np;
                ++pcnt;
                prog = true;
              }
            }
            if (prog) {
              t_prog = tc::globaltimer();
              spins = 0;
            } else if (!poll_idle(++spins, t_prog, sh, a.status)) {
              break;
            }
          }
        }
      } else {
        // ---- softmax: one row per thread pair; the thread with shalf = (superblock id & 1) takes
        // a superblock: its 16 S columns become 8 columns of bf16 P in place (TMEM) and the fp32
        // values are added to the thread's row sum, in token order ----
        for (int ch = 0; ch < nch; ++ch, ++scnt) {
          const int sb = (int)(scnt & 1);
          if (!warp_wait(&sh->s_full[sb], (uint32_t)((scnt >> 1) & 1), &sh->abort_flag, a.status)) {
            if (lane == 0 && !sh->abort_flag) report(a.status, SGQA_ERR_TIMEOUT);
            sh->abort_flag = 1;
            break;
          }
          tc::fence_after_sync();
          const float base = m_use * sc;
#pragma unroll 1
          for (int i = 0; i < kCH; ++i) {
            const int e = ch * kCH + i;
            if (e >= nu) break;                 // warp-uniform
            const int sbid = usb[e];
            if ((sbid & 1) != shalf) continue;  // warp-uniform
            const uint32_t col = tmem + lane_base + (uint32_t)(sb * kCT + i * kUnit);
            uint32_t v[kUnit];
            tc::tmem_ld16(col, v);
            const int u0 = sbid * kUnit;
            const bool live = t_r >= 0;
            uint32_t pk[8];
            if (main_pass && lb >= 3 && live && u0 + (kUnit - 1) <= t_r && u0 >= lo_r) {
              // blocks of 8 or 16 tokens wholly before the row's token (and inside its window, if
              // any): the selection bit of each half superblock becomes the additive term of the
              // exponent (-inf when unselected, whose exp2 is an exact 0); no per-token mask
              const int jb = (u0 >> lb) - w0;
              const float bias0 = ((wmask[jb] >> q_r) & 1u) ? -base : -INFINITY;
              const float bias1 = ((wmask[jb + spb - 1] >> q_r) & 1u) ? -base : -INFINITY;
#pragma unroll
              for (int k2 = 0; k2 < 8; ++k2) {
                const float bias = k2 < 4 ? bias0 : bias1;
                const float pa = ex2_approx(fmaf(__uint_as_float(v[2 * k2]), sc, bias));
                const float pb = ex2_approx(fmaf(__uint_as_float(v[2 * k2 + 1]), sc, bias));
                pk[k2] = pack_bf16x2(pa, pb);
                l_sum += pa;
                l_sum += pb;
              }
            } else {
              uint32_t vmask = 0;  // bit k: token sbid * 16 + k is valid for this row
              if (live) {
                for (int blk = 0; blk < spb; ++blk) {
                  const int j = (u0 >> lb) + blk;
                  if ((wmask[j - w0] >> q_r) & 1u) vmask |= ((1u << (1 << lb)) - 1u) << (blk << lb);
                }
                const int lim = t_r - u0;
                if (lim < 15) vmask &= lim < 0 ? 0u : ((2u << lim) - 1u);
                const int below = lo_r - u0;  // tokens of this superblock before the window
                if (below > 0) vmask &= below >= kUnit ? 0u : ~((1u << below) - 1u);
              }
              if (!main_pass) {
#pragma unroll
                for (int k2 = 0; k2 < kUnit; ++k2)
                  if ((vmask >> k2) & 1u) m_exact = fmaxf(m_exact, __uint_as_float(v[k2]));
                continue;
              }
              // masked slots get -inf, whose exp2 is an exact 0
#pragma unroll
              for (int k2 = 0; k2 < 8; ++k2) {
                const bool va = (vmask >> (2 * k2)) & 1u, vb = (vmask >> (2 * k2 + 1)) & 1u;
                const float pa = ex2_approx(va ? fmaf(__uint_as_float(v[2 * k2]), sc, -base) : -INFINITY);
                const float pb = ex2_approx(vb ? fmaf(__uint_as_float(v[2 * k2 + 1]), sc, -base) : -INFINITY);
                pk[k2] = pack_bf16x2(pa, pb);
                l_sum += pa;
                l_sum += pb;
              }
            }
            tc::tmem_st8(col, pk);
          }
          // P of this chunk is in TMEM (or, in the exact-maximum pass, S has been read): the MMA
          // issuer may take the buffer
          tc::tmem_wait_st();
          tc::fence_before_sync();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&sh->p_full[sb]);
        }
      }
      __syncthreads();
      // clear this window's bitmap words through its union list
      for (int e = tid; e < nu; e += kThreads)
        for (int i = 0; i < spb; ++i) wmask[(usb[e] * spb + i) - w0] = 0u;
      __syncthreads();
    }
    if (main_pass) {
      // all of this pass's MMAs have completed once o_done arrives (at once if none was issued);
      // after the first pass the row sums tell which rows need their exact maximum
      if (warp == 1 && lane == 0) {
        tc::mma_commit(&sh->o_done);
        ++o_commits;
      }
      if (is_sm) {
        o_ok = warp_wait(&sh->o_done, (uint32_t)o_phase, &sh->abort_flag, a.status);
        if (!o_ok) {
          if (lane == 0 && !sh->abort_flag) report(a.status, SGQA_ERR_TIMEOUT);
          sh->abort_flag = 1;
        }
        sh->l_part[shalf][r] = l_sum;
      }
      o_phase ^= 1;
      __syncthreads();
      if (is_sm && pass == 0) risky = !(sh->l_part[0][r] + sh->l_part[1][r] <= kRiskSum);
    }
    if (pass == 0) {
      rerun = __syncthreads_or(is_sm && risky) != 0;
    } else if (pass == 1) {
      if (is_sm) sh->max_part[shalf][r] = m_exact;
      __syncthreads();
      if (is_sm) m_exact = fmaxf(sh->max_part[0][r], sh->max_part[1][r]);
    }
  }

  // ---- epilogue ----
  if (is_sm) {
    if (o_ok) {
      tc::fence_after_sync();
      const float l_r = sh->l_part[0][r] + sh->l_part[1][r];
      const float inv = l_r > 0.f ? 1.f / l_r : 0.f;
      const long orow = t_r >= 0 ? ((long)b * a.nQ + (t_r - a.q_t0)) * a.Hq + (long)g * R + h_r : -1;
#pragma unroll 1
      for (int h = shalf; h < D / 32; h += 2) {
        uint32_t o[32];
        tc::tmem_ld32(tmem_o + lane_base + (uint32_t)(h * 32), o);
        if (orow >= 0) {
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            const long off = orow * D + h * 32 + c8 * 8;
            const uint4 gv = __ldg(reinterpret_cast<const uint4*>(a.gate + off));
            const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
            uint32_t ov[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float o0 = inv > 0.f ? __uint_as_float(o[c8 * 8 + 2 * i]) * inv : 0.f;
              const float o1 = inv > 0.f ? __uint_as_float(o[c8 * 8 + 2 * i + 1]) * inv : 0.f;
              const float y0 = o0 * sigmoid_fast(bf16_lo(gw[i]));
              const float y1 = o1 * sigmoid_fast(bf16_hi(gw[i]));
              ov[i] = pack_bf16x2(y0, y1);
            }
            *reinterpret_cast<uint4*>(a.out + off) = make_uint4(ov[0], ov[1], ov[2], ov[3]);
          }
        }
      }
    }
  }

  // ---- drain and release ----
  if (warp == 0 && lane == 0) {
    // copies issued for the last stages must land before the CTA exits
    for (long k2 = kck - kNK; k2 < kck; ++k2) {
      if (k2 < 0) continue;
      volatile int no_abort = 0;
      tc::mbar_wait(&sh->k_full[k2 % kNK], (uint32_t)((k2 / kNK) & 1), &no_abort);
    }
    for (long k2 = kcv - kNV; k2 < kcv; ++k2) {
      if (k2 < 0) continue;
      volatile int no_abort = 0;
      tc::mbar_wait(&sh->v_full[k2 % kNV], (uint32_t)((k2 / kNV) & 1), &no_abort);
    }
  }
  if (warp == 1 && lane == 0 && o_commits > 0) {  // every MMA issued must finish before TMEM is freed
    volatile int no_abort = 0;
    tc::mbar_wait(&sh->o_done, (uint32_t)((o_commits - 1) & 1), &no_abort);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, C::kTmemCols);
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

// 3-D map over k or v [batch * T_kv tokens][G][d] bf16: box = 64 dims x 1 group x box_tokens
// tokens, 128B swizzle (one 128-byte row per token).
bool make_kv_map(CUtensorMap* map, const void* base, long tokens, int G, int d, int box_tokens) {
  EncodeTiled enc = get_encode();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)G, (cuuint64_t)tokens};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)G * d * 2};
  const cuuint32_t box[3] = {64, 1, (cuuint32_t)box_tokens};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int R>
cudaError_t launch_dr(const AttendArgs& a, const uint32_t* perm, cudaStream_t s) {
  using C = AtcCfg<D>;
  constexpr int QT = kM / R;
  const int n = a.t_end - a.t_begin;
  const int tiles = (n + QT - 1) / QT;
  const int n_seg = a.batch * a.G;
  int lb = 0;
  while ((1 << lb) < a.B) ++lb;
  KvMaps maps;
  const long tokens = (long)a.batch * a.T_kv;
  maps.max_run = tokens >= 4 * kUnit ? 2 : (tokens >= 2 * kUnit ? 1 : 0);
  for (int i = 0; i < 3; ++i) {
    const int box = kUnit << (i <= maps.max_run ? i : 0);
    if (!make_kv_map(&maps.k[i], a.k, tokens, a.G, D, box) || !make_kv_map(&maps.v[i], a.v, tokens, a.G, D, box))
      return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaFuncSetAttribute(attend_tc_kernel<D, R>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  attend_tc_kernel<D, R><<<(unsigned)((long)tiles * n_seg), kThreads, C::kSmem, s>>>(maps, a, perm, n, tiles, lb);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const AttendArgs& a, const uint32_t* perm, cudaStream_t s) {
  switch (a.Hq / a.G) {
    case 4: return launch_dr<D, 4>(a, perm, s);
    case 8: return launch_dr<D, 8>(a, perm, s);
    case 16: return launch_dr<D, 16>(a, perm, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

bool attend_tc_supported(int Hq, int G, int B, int d) {
  const int R = Hq / G;
  return (R == 4 || R == 8 || R == 16) && B <= kUnit && (d == 64 || d == 128);
}

cudaError_t launch_attend_tc(const AttendArgs& a, const uint32_t* perm, cudaStream_t s) {
  if (a.t_end <= a.t_begin) return cudaSuccess;
  if (a.d == 128) return launch_d<128>(a, perm, s);
  if (a.d == 64) return launch_d<64>(a, perm, s);
  return cudaErrorInvalidValue;
}

}  // namespace sgqa
