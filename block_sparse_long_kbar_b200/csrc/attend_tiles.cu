// K3 (tiled): gated attention for a tile of query rows over the union of their selected blocks.
//
// Step 5 Preview pages (mo.ai.kr, "Step 5 Preview agentic work design", section "model
// structure and training stability"): Sparse GQA attends only to the selected blocks, and the
// developers batch queries whose selections overlap to raise GPU utilisation. Here a tile holds
// Q query rows of one (sequence, KV group) — the rows are given by the scheduling permutation
// (plan.cu), which puts rows with similar selections together — and every K/V block that any
// of them selected is gathered into shared memory once and used by all of them. Per-query
// masks (did this query select the block; is the token <= the query's position) keep every
// query's result exactly its own: the union only changes which loads are shared.
//
// Layout of the work:
//   * 16-row warp MMA tiles (bf16 mma.sync m16n8k16, fp32 accumulate): a warp owns 16/R query
//     rows x R heads of the group (GQA: the heads share the gathered rows), so each warp holds
//     its rows' Q fragments, online-softmax state (exp2 domain) and O accumulators to the end;
//   * the union is built window by window over block ids: every query's ascending selection is
//     scattered as a query-bit into a shared bitmap (one cursor per query, each entry read
//     once), then compacted into the ascending list of 16-token superblocks (16/B blocks,
//     aligned on block ids) that hold a selected block;
//   * superblocks are consumed four per 64-slot chunk, double-buffered with cp.async into
//     XOR-swizzled shared memory (slots of unselected blocks are zero-filled, not read); a warp
//     skips a superblock none of its queries selected;
//   * per superblock: S (two n-tiles), per-row max update with rescaling only when a max grows,
//     P in bf16, O += P V as one k = 16 step. Because superblocks are aligned on block ids and
//     unselected slots add exact zeros, every query's arithmetic is the same whatever rows share
//     its tile: results are bitwise causal and do not depend on the scheduling;
//   * epilogue: O / l times sigmoid(gate_logits), bf16 round-to-nearest-even.
// The union order (ascending blocks, chunk boundaries) is a function of the tile's selections
// only, so results are deterministic.
#include <cmath>

#include "common.cuh"
#include "kernels.h"

namespace sgqa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kChunk = 64;   // token slots per K/V chunk
constexpr int kWin = 2048;   // block ids per union window

template <int D, int R>
struct TileCfg {
  static constexpr int QW = 16 / R;                         // queries per warp
  static constexpr int kWarps = (32 / QW) < 8 ? (32 / QW) : 8;
  static constexpr int Q = kWarps * QW;                     // queries per tile (<= 32: one mask bit each)
  static constexpr int NT = kWarps * 32;
  static constexpr int kRowBytes = D * 2;
  static constexpr int kStage = 2 * kChunk * kRowBytes;    // K and V rows of one chunk
  static constexpr int kKV = 2 * kStage;                    // double buffered
  static constexpr int kSmem = kKV + 2 * kWin * 4 + 2 * kChunk * 8;
};

__device__ __forceinline__ uint32_t ld_u32(const uint16_t* p) { return __ldg(reinterpret_cast<const uint32_t*>(p)); }

template <int D, int R>
__global__ void __launch_bounds__(TileCfg<D, R>::NT, 1)
    attend_tiles_kernel(AttendArgs a, const uint32_t* __restrict__ perm, int n_per_seg, int tiles_per_seg, int lb) {
  using C = TileCfg<D, R>;
  constexpr int CH = D / 8;
  extern __shared__ __align__(128) uint8_t smem[];
  uint32_t* wmask = reinterpret_cast<uint32_t*>(smem + C::kKV);  // [kWin] query bits per block
  int32_t* usb = reinterpret_cast<int32_t*>(wmask + kWin);         // union superblocks, ascending
  int32_t* slot_u = reinterpret_cast<int32_t*>(usb + kWin);        // [2][kChunk]
  uint32_t* slot_m = reinterpret_cast<uint32_t*>(slot_u + 2 * kChunk);  // [2][kChunk]
  __shared__ int s_t[32];
  __shared__ int s_cur[32];
  __shared__ int s_scan[32];
  __shared__ int s_nu, s_maxc;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int B = a.B, G = a.G;
  const int seg = blockIdx.x / tiles_per_seg, tile = blockIdx.x % tiles_per_seg;
  const int b = seg / G, g = seg % G;

  if (tid == 0) s_maxc = -1;
  __syncthreads();
  if (tid < C::Q) {
    const int idx = tile * C::Q + tid;
    const int t = idx < n_per_seg ? a.t_begin + (int)__ldg(perm + (long)seg * n_per_seg + idx) : -1;
    s_t[tid] = t;
    s_cur[tid] = 0;
    if (t >= 0) atomicMax(&s_maxc, t / B);
  }
  __syncthreads();

  // rows of this warp: r -> query warp*QW + r/R, head r%R; this thread owns rows gid and gid + 8
  const int qa = warp * C::QW + gid / R, ha = gid % R;
  const int qb = warp * C::QW + (gid + 8) / R, hb = (gid + 8) % R;
  const int ta = s_t[qa], tb = s_t[qb];
  const long rowa = ta >= 0 ? ((long)b * a.nQ + (ta - a.q_t0)) * a.Hq + (long)g * R + ha : -1;
  const long rowb = tb >= 0 ? ((long)b * a.nQ + (tb - a.q_t0)) * a.Hq + (long)g * R + hb : -1;
  uint32_t qf[D / 16][4];
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    const int c0 = ks * 16 + tig * 2;
    qf[ks][0] = rowa >= 0 ? ld_u32(a.q + rowa * D + c0) : 0u;
    qf[ks][1] = rowb >= 0 ? ld_u32(a.q + rowb * D + c0) : 0u;
    qf[ks][2] = rowa >= 0 ? ld_u32(a.q + rowa * D + c0 + 8) : 0u;
    qf[ks][3] = rowb >= 0 ? ld_u32(a.q + rowb * D + c0 + 8) : 0u;
  }
  float o[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const float sc = kLog2e / sqrtf((float)D);
  const unsigned wq = ((1u << C::QW) - 1u) << (warp * C::QW);  // this warp's query bits (QW < 32)

  const long seq_off = (long)b * a.T_kv * G * D;
  const uint16_t* kseq = a.k + seq_off;
  const uint16_t* vseq = a.v + seq_off;
  // Work unit: a superblock of 16 token slots aligned on block ids (16/B blocks; B <= 16), so a
  // token's slot, and the grouping of its products in the MMA k-steps, depend only on its own
  // block id, never on which other rows share the tile.
  constexpr int kUnit = 16, kUnitsPerChunk = kChunk / kUnit;

  auto slot_token = [&](int ch, int nu, int s, int w0, uint32_t& msk) -> int {
    const int e = ch * kUnitsPerChunk + s / kUnit;
    msk = 0;
    if (e >= nu) return -1;
    const int u = usb[e] * kUnit + (s % kUnit);
    if (u >= a.T_kv) return -1;
    msk = wmask[(u >> lb) - w0];
    return msk ? u : -1;
  };
  auto issue = [&](int ch, int nu, int w0, int stage) {
    uint8_t* kd = smem + stage * C::kStage;
    uint8_t* vd = kd + kChunk * C::kRowBytes;
    if (tid < kChunk) {
      uint32_t msk;
      const int u = slot_token(ch, nu, tid, w0, msk);
      slot_u[stage * kChunk + tid] = u;
      slot_m[stage * kChunk + tid] = msk;
    }
#pragma unroll
    for (int it = 0; it < 2 * kChunk * CH / C::NT; ++it) {
      const int idx = it * C::NT + tid;
      const int kv = idx / (kChunk * CH);
      const int r = idx % (kChunk * CH);
      const int s = r / CH, c16 = r % CH;
      uint32_t msk;
      const int u = slot_token(ch, nu, s, w0, msk);
      const long off = u >= 0 ? ((long)u * G + g) * D + c16 * 8 : 0;
      const int sw = s * C::kRowBytes + ((c16 ^ (s & 7)) * 16);
      cp_async16(smem_u32((kv ? vd : kd) + sw), (kv ? vseq : kseq) + off, u >= 0 ? 16 : 0);
    }
    cp_async_commit();
  };

  const int nwin = s_maxc < 0 ? 0 : s_maxc / kWin + 1;
  for (int win = 0; win < nwin; ++win) {
    const int w0 = win * kWin, w1 = w0 + kWin;
    for (int i = tid; i < kWin; i += C::NT) wmask[i] = 0;
    __syncthreads();
    // scatter this window's entries of every query (ascending rows: a cursor per query)
    for (int q = warp; q < C::Q; q += C::kWarps) {
      const int t = s_t[q];
      if (t < 0) continue;
      const int cq = t / B;
      const int32_t* row = a.sel + (((long)b * a.sel_T + (t - a.sel_t0)) * G + g) * (long)a.Kb;
      int cur = s_cur[q];
      while (cur < a.Kb) {
        const int e = cur + lane;
        int j = e < a.Kb ? __ldg(row + e) : -1;
        // rows must be strictly ascending block ids <= the own block, then -1 padding
        const int prev = __shfl_up_sync(0xFFFFFFFFu, j, 1);
        const int before = lane > 0 ? prev : (cur > 0 ? __ldg(row + cur - 1) : -1);
        if (j > cq || j < -1 || (j >= 0 && j <= before) || (j >= 0 && j < w0)) {
          report(a.status, SGQA_ERR_DEVICE_CHECK);
          j = -1;
        }
        const bool in = j >= w0 && j < w1;
        const bool past = j < 0 || j >= w1;  // end of row, or beyond this window
        if (in) atomicOr(&wmask[j - w0], 1u << q);
        const unsigned stop = __ballot_sync(0xFFFFFFFFu, past);
        const int adv = stop ? __ffs(stop) - 1 : 32;
        cur += adv;
        if (stop) {
          // an entry of -1 ends the row; entries beyond the window wait for the next window
          const int first = __shfl_sync(0xFFFFFFFFu, j, adv);
          if (first < 0) cur = a.Kb;
          break;
        }
      }
      if (lane == 0) s_cur[q] = cur;
    }
    __syncthreads();
    // compact the window into its ascending list of superblocks holding any selected block
    {
      const int spb = kUnit >> lb;                 // blocks per superblock
      const int nsb_win = kWin / spb;
      const int per = (nsb_win + C::NT - 1) / C::NT;
      const int sb0 = tid * per, sb1 = min(nsb_win, sb0 + per);
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
      if (lane == 31) s_scan[warp] = x;
      __syncthreads();
      if (tid == 0) {
        int run = 0;
        for (int w = 0; w < C::kWarps; ++w) {
          const int v = s_scan[w];
          s_scan[w] = run;
          run += v;
        }
        s_nu = run;
      }
      __syncthreads();
      int pos = s_scan[warp] + x - cnt;
      for (int sb = sb0; sb < sb1; ++sb) {
        uint32_t any = 0;
        for (int i = 0; i < spb; ++i) any |= wmask[sb * spb + i];
        if (any) usb[pos++] = (w0 >> (4 - lb)) + sb;
      }
    }
    __syncthreads();
    const int nu = s_nu;
    const int nch = (nu + kUnitsPerChunk - 1) / kUnitsPerChunk;
    int stage = 0;
    if (nch > 0) issue(0, nu, w0, 0);
    for (int ch = 0; ch < nch; ++ch) {
      if (ch + 1 < nch) {
        issue(ch + 1, nu, w0, stage ^ 1);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();
      const uint8_t* kd = smem + stage * C::kStage;
      const uint8_t* vd = kd + kChunk * C::kRowBytes;
      const int32_t* su = slot_u + stage * kChunk;
      const uint32_t* smk = slot_m + stage * kChunk;
      // One 16-slot unit at a time: a warp skips units none of its queries selected; otherwise
      // S for the unit (two n-tiles, independent accumulators), the per-row max update
      // (rescaling only when some row's max grows), P in bf16 and O += P V (one k = 16 step).
      // Unselected slots contribute exact zeros and leave the max unchanged, so every query's
      // arithmetic is the same sequence of operations whatever other rows share its tile.
#pragma unroll 1
      for (int unit = 0; unit < kUnitsPerChunk; ++unit) {
        const int slot0 = unit * kUnit;
        const uint32_t um = (lane < kUnit ? smk[slot0 + lane] : 0u) & wq;
        if (__reduce_or_sync(0xFFFFFFFFu, um) == 0u) continue;
        float sacc[2][4];
#pragma unroll
        for (int i = 0; i < 2; ++i) sacc[i][0] = sacc[i][1] = sacc[i][2] = sacc[i][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          // x4: (n-tile 0: k lo, k hi), (n-tile 1: k lo, k hi) of k-step ks
          const int mat = lane >> 3;
          const int tok = slot0 + (mat >> 1) * 8 + (lane & 7);
          const int chk = ks * 2 + (mat & 1);
          uint32_t r0, r1, r2, r3;
          ldmatrix_x4(r0, r1, r2, r3, smem_u32(kd + tok * C::kRowBytes + ((chk ^ (tok & 7)) * 16)));
          mma_bf16_16816(sacc[0], qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], r0, r1);
          mma_bf16_16816(sacc[1], qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], r2, r3);
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int slot = slot0 + nt * 8 + tig * 2 + e;
            const int u = su[slot];
            const uint32_t mk = smk[slot];
            if (!(((mk >> qa) & 1u) && u <= ta)) sacc[nt][e] = -INFINITY;
            if (!(((mk >> qb) & 1u) && u <= tb)) sacc[nt][2 + e] = -INFINITY;
          }
        }
        float bm0 = fmaxf(fmaxf(sacc[0][0], sacc[0][1]), fmaxf(sacc[1][0], sacc[1][1]));
        float bm1 = fmaxf(fmaxf(sacc[0][2], sacc[0][3]), fmaxf(sacc[1][2], sacc[1][3]));
        bm0 = fmaxf(bm0, __shfl_xor_sync(0xFFFFFFFFu, bm0, 1));
        bm0 = fmaxf(bm0, __shfl_xor_sync(0xFFFFFFFFu, bm0, 2));
        bm1 = fmaxf(bm1, __shfl_xor_sync(0xFFFFFFFFu, bm1, 1));
        bm1 = fmaxf(bm1, __shfl_xor_sync(0xFFFFFFFFu, bm1, 2));
        const float mn0 = fmaxf(m0, bm0), mn1 = fmaxf(m1, bm1);
        if (__any_sync(0xFFFFFFFFu, mn0 > m0 || mn1 > m1)) {
          const float al0 = m0 == -INFINITY ? 0.f : exp2f((m0 - mn0) * sc);
          const float al1 = m1 == -INFINITY ? 0.f : exp2f((m1 - mn1) * sc);
#pragma unroll
          for (int i = 0; i < D / 8; ++i) {
            o[i][0] *= al0; o[i][1] *= al0;
            o[i][2] *= al1; o[i][3] *= al1;
          }
          l0 *= al0;
          l1 *= al1;
          m0 = mn0;
          m1 = mn1;
        }
        const float base0 = m0 == -INFINITY ? 0.f : m0 * sc;
        const float base1 = m1 == -INFINITY ? 0.f : m1 * sc;
        uint32_t pa[4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          pa[2 * nt] = pack_bf16x2(ex2_approx(fmaf(sacc[nt][0], sc, -base0)), ex2_approx(fmaf(sacc[nt][1], sc, -base0)));
          pa[2 * nt + 1] = pack_bf16x2(ex2_approx(fmaf(sacc[nt][2], sc, -base1)), ex2_approx(fmaf(sacc[nt][3], sc, -base1)));
        }
        l0 += (bf16_lo(pa[0]) + bf16_hi(pa[0])) + (bf16_lo(pa[2]) + bf16_hi(pa[2]));
        l1 += (bf16_lo(pa[1]) + bf16_hi(pa[1])) + (bf16_lo(pa[3]) + bf16_hi(pa[3]));
#pragma unroll
        for (int ndp = 0; ndp < D / 16; ++ndp) {
          // x4.trans: (tokens lo, dims 2ndp), (tokens hi, dims 2ndp), (lo, 2ndp+1), (hi, 2ndp+1)
          const int mat = lane >> 3;
          const int tok = slot0 + (mat & 1) * 8 + (lane & 7);
          const int chk = ndp * 2 + (mat >> 1);
          uint32_t r0, r1, r2, r3;
          ldmatrix_x4_trans(r0, r1, r2, r3, smem_u32(vd + tok * C::kRowBytes + ((chk ^ (tok & 7)) * 16)));
          mma_bf16_16816(o[2 * ndp], pa[0], pa[1], pa[2], pa[3], r0, r1);
          mma_bf16_16816(o[2 * ndp + 1], pa[0], pa[1], pa[2], pa[3], r2, r3);
        }
      }
      __syncthreads();
      stage ^= 1;
    }
  }

  // epilogue: normalise, gate, bf16
  l0 += __shfl_xor_sync(0xFFFFFFFFu, l0, 1);
  l0 += __shfl_xor_sync(0xFFFFFFFFu, l0, 2);
  l1 += __shfl_xor_sync(0xFFFFFFFFu, l1, 1);
  l1 += __shfl_xor_sync(0xFFFFFFFFu, l1, 2);
  const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f;
  const float inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
#pragma unroll
  for (int nt = 0; nt < D / 8; ++nt) {
    const int col = nt * 8 + tig * 2;
    if (rowa >= 0) {
      const uint32_t gw = ld_u32(a.gate + rowa * D + col);
      const float y0 = o[nt][0] * inv0 * (1.f / (1.f + expf(-bf16_lo(gw))));
      const float y1 = o[nt][1] * inv0 * (1.f / (1.f + expf(-bf16_hi(gw))));
      *reinterpret_cast<uint32_t*>(a.out + rowa * D + col) = pack_bf16x2(y0, y1);
    }
    if (rowb >= 0) {
      const uint32_t gw = ld_u32(a.gate + rowb * D + col);
      const float y0 = o[nt][2] * inv1 * (1.f / (1.f + expf(-bf16_lo(gw))));
      const float y1 = o[nt][3] * inv1 * (1.f / (1.f + expf(-bf16_hi(gw))));
      *reinterpret_cast<uint32_t*>(a.out + rowb * D + col) = pack_bf16x2(y0, y1);
    }
  }
}

template <int D, int R>
cudaError_t launch_dr(const AttendArgs& a, const uint32_t* perm, cudaStream_t s) {
  using C = TileCfg<D, R>;
  const int n = a.t_end - a.t_begin;
  const int tiles = (n + C::Q - 1) / C::Q;
  const int n_seg = a.batch * a.G;
  int lb = 0;
  while ((1 << lb) < a.B) ++lb;
  cudaError_t e = cudaFuncSetAttribute(attend_tiles_kernel<D, R>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  attend_tiles_kernel<D, R><<<(unsigned)((long)tiles * n_seg), C::NT, C::kSmem, s>>>(a, perm, n, tiles, lb);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const AttendArgs& a, const uint32_t* perm, cudaStream_t s) {
  switch (a.Hq / a.G) {
    case 1: return launch_dr<D, 1>(a, perm, s);
    case 2: return launch_dr<D, 2>(a, perm, s);
    case 4: return launch_dr<D, 4>(a, perm, s);
    case 8: return launch_dr<D, 8>(a, perm, s);
    case 16: return launch_dr<D, 16>(a, perm, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

bool attend_tiles_supported(int Hq, int G, int B) {
  const int R = Hq / G;
  return (R == 1 || R == 2 || R == 4 || R == 8 || R == 16) && B <= 16;
}

cudaError_t launch_attend_tiles(const AttendArgs& a, const uint32_t* perm, cudaStream_t s) {
  if (a.t_end <= a.t_begin) return cudaSuccess;
  if (a.d == 128) return launch_d<128>(a, perm, s);
  if (a.d == 64) return launch_d<64>(a, perm, s);
  return cudaErrorInvalidValue;
}

}  // namespace sgqa
