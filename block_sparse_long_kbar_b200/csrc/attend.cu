// K3: gated attention over the selected blocks (Step 5 Preview pages: mo.ai.kr, "Step 5 Preview
// agentic work design", section "model structure and training stability" — the full-context
// layer is Sparse GQA on top of Gated GQA; every KV group attends only to its selected blocks).
//
// Definition implemented: for each head h of group g, over U = {u <= t : floor(u/B) in S(t,g)},
// o = softmax_U(q[t,h] . k[u,g] / sqrt(d)) . v[u,g]; out = o * sigmoid(gate_logits[t,h]).
//
// Design (first version). One CTA per (sequence, group, query) unit and, for split-K, per split
// of the unit's selection. The R heads of the group share every gathered K/V row (GQA): they are
// the rows of a 16-row warp MMA tile (rows >= R are zero). The selected tokens are cut into
// chunks of 32 token slots (32/B blocks); the 4 warps take chunks round-robin, each with its own
// double-buffered cp.async gather of the chunk's K and V rows into XOR-swizzled shared memory,
// S = Q K^T and O += P V on bf16 mma.sync (fp32 accumulate), and an online softmax in the exp2
// domain. Slots past the causal limit or past the selection are zero-filled and masked. The
// warps' (max, sum, O) states are merged in a fixed order (deterministic), then either the
// sigmoid gate is applied and bf16 written, or the split's partial state is stored for
// launch_attend_merge (split-K decode).
#include <cmath>

#include "common.cuh"
#include "kernels.h"

namespace sgqa {
namespace {

constexpr int kWarps = 4;
constexpr int kChunk = 32;  // token slots per chunk
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ uint32_t ld_u32(const uint16_t* p) { return __ldg(reinterpret_cast<const uint32_t*>(p)); }

template <int D>
struct AttendSmem {
  static constexpr int kRowBytes = D * 2;
  static constexpr int kStage = 2 * kChunk * kRowBytes;  // K and V rows of one chunk
  static constexpr int kStaging = kWarps * 2 * kStage;
  static constexpr int kMerge = kWarps * 16 * (D + 2) * 4;
  static_assert(kMerge <= kStaging, "merge area reuses the staging buffers");
};

template <int D>
__global__ void __launch_bounds__(kWarps * 32) attend_kernel(AttendArgs a) {
  using L = AttendSmem<D>;
  constexpr int CH = D / 8;  // 16-byte chunks per row
  extern __shared__ __align__(128) uint8_t smem[];
  int32_t* s_sel = reinterpret_cast<int32_t*>(smem + L::kStaging);
  __shared__ int s_nsel;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int G = a.G, R = a.Hq / a.G, B = a.B;
  const int nT = a.t_end - a.t_begin;
  const int unit = blockIdx.x;
  const int g = unit / (a.batch * nT);
  const int rem = unit % (a.batch * nT);
  const int b = rem / nT;
  const int t = a.t_end - 1 - rem % nT;
  const int split = blockIdx.y;
  const int c_own = t / B;

  // ---- the unit's selection, validated --------------------------------------------------------
  const int32_t* srow = a.sel + (((long)b * a.sel_T + (t - a.sel_t0)) * G + g) * (long)a.Kb;
  if (tid == 0) s_nsel = 0;
  __syncthreads();
  int last = -1;
  // the format: strictly ascending block ids in [0, c_own], then -1 padding. An entry out of
  // range, not above the entry before it, or after the padding began is reported and skipped
  // (each thread compares with the previous entry as stored, so no ordering between threads)
  for (int i = tid; i < a.Kb; i += kWarps * 32) {
    int j = __ldg(srow + i);
    if (j > c_own || j < -1) {
      report(a.status, SGQA_ERR_DEVICE_CHECK);
      j = -1;
    }
    if (j >= 0 && i > 0) {
      const int p = __ldg(srow + i - 1);
      if (p < 0 || p > c_own || j <= p) {
        report(a.status, SGQA_ERR_DEVICE_CHECK);
        j = -1;
      }
    }
    s_sel[i] = j;
    if (j >= 0) last = i;
  }
  if (last >= 0) atomicMax(&s_nsel, last + 1);
  __syncthreads();
  const int nsel = s_nsel;
  const int bpc = kChunk / B;
  const int n_chunks = (nsel + bpc - 1) / bpc;
  const int cps = (n_chunks + a.splits - 1) / a.splits;
  const int c_begin = min(n_chunks, split * cps), c_end = min(n_chunks, c_begin + cps);

  // ---- Q fragments (rows = heads of the group, zero beyond R) --------------------------------
  const long qrow = ((long)b * a.nQ + (t - a.q_t0)) * a.Hq + (long)g * R;
  const uint16_t* qp = a.q + qrow * D;
  uint32_t qa[D / 16][4];
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    const int c0 = ks * 16 + tig * 2;
    qa[ks][0] = gid < R ? ld_u32(qp + gid * D + c0) : 0u;
    qa[ks][1] = gid + 8 < R ? ld_u32(qp + (gid + 8) * D + c0) : 0u;
    qa[ks][2] = gid < R ? ld_u32(qp + gid * D + c0 + 8) : 0u;
    qa[ks][3] = gid + 8 < R ? ld_u32(qp + (gid + 8) * D + c0 + 8) : 0u;
  }

  float o[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const float sc = kLog2e / sqrtf((float)D);

  uint8_t* wbase = smem + warp * 2 * L::kStage;
  const long seq_off = (long)b * a.T_kv * G * D;
  const uint16_t* kseq = a.k + seq_off;
  const uint16_t* vseq = a.v + seq_off;

  // token of slot s of chunk ci, or -1
  auto slot_token = [&](int ci, int s) -> int {
    const int e = ci * bpc + s / B;
    if (e >= nsel) return -1;
    const int j = s_sel[e];
    if (j < 0) return -1;
    const int u = j * B + s % B;
    return (u <= t && SGQA_CHECK(u < a.T_kv, a.status)) ? u : -1;
  };
  auto issue = [&](int ci, int stage) {
    uint8_t* kd = wbase + stage * L::kStage;
    uint8_t* vd = kd + kChunk * L::kRowBytes;
#pragma unroll
    for (int it = 0; it < kChunk * CH / 32; ++it) {
      const int idx = it * 32 + lane;
      const int s = idx / CH, ch = idx % CH;
      const int u = slot_token(ci, s);
      const long off = u >= 0 ? ((long)u * G + g) * D + ch * 8 : 0;
      const int sw = s * L::kRowBytes + ((ch ^ (s & 7)) * 16);
      cp_async16(smem_u32(kd + sw), kseq + off, u >= 0 ? 16 : 0);
      cp_async16(smem_u32(vd + sw), vseq + off, u >= 0 ? 16 : 0);
    }
    cp_async_commit();
  };

  int stage = 0;
  int ci = c_begin + warp;
  if (ci < c_end) issue(ci, 0);
  for (; ci < c_end; ci += kWarps) {
    if (ci + kWarps < c_end) {
      issue(ci + kWarps, stage ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncwarp();
    const unsigned vmask = __ballot_sync(0xFFFFFFFFu, slot_token(ci, lane) >= 0);
    const uint8_t* kd = wbase + stage * L::kStage;
    const uint8_t* vd = kd + kChunk * L::kRowBytes;

    // S = Q K^T for 32 tokens (4 n-tiles of 8)
    float sacc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) sacc[i][0] = sacc[i][1] = sacc[i][2] = sacc[i][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        const int mat = lane >> 3;
        const int tok = (np * 2 + (mat >> 1)) * 8 + (lane & 7);
        const int chk = ks * 2 + (mat & 1);
        uint32_t r0, r1, r2, r3;
        ldmatrix_x4(r0, r1, r2, r3, smem_u32(kd + tok * L::kRowBytes + ((chk ^ (tok & 7)) * 16)));
        mma_bf16_16816(sacc[2 * np], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], r0, r1);
        mma_bf16_16816(sacc[2 * np + 1], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], r2, r3);
      }
    }
    // online softmax (exp2 domain); rows gid (m0, l0) and gid + 8 (m1, l1)
    float mx0 = m0, mx1 = m1;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int slot = nt * 8 + tig * 2 + e;
        if (!((vmask >> slot) & 1u)) {
          sacc[nt][e] = -INFINITY;
          sacc[nt][2 + e] = -INFINITY;
        }
        mx0 = fmaxf(mx0, sacc[nt][e]);
        mx1 = fmaxf(mx1, sacc[nt][2 + e]);
      }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xFFFFFFFFu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xFFFFFFFFu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xFFFFFFFFu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xFFFFFFFFu, mx1, 2));
    const float base0 = mx0 == -INFINITY ? 0.f : mx0 * sc;
    const float base1 = mx1 == -INFINITY ? 0.f : mx1 * sc;
    const float alpha0 = exp2f(m0 * sc - base0);
    const float alpha1 = exp2f(m1 * sc - base1);
    m0 = mx0;
    m1 = mx1;
    uint32_t pa[2][4];
    float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int nt = 2 * kk + h;
        const uint32_t lo = pack_bf16x2(ex2_approx(fmaf(sacc[nt][0], sc, -base0)), ex2_approx(fmaf(sacc[nt][1], sc, -base0)));
        const uint32_t hi = pack_bf16x2(ex2_approx(fmaf(sacc[nt][2], sc, -base1)), ex2_approx(fmaf(sacc[nt][3], sc, -base1)));
        pa[kk][2 * h] = lo;       // row gid
        pa[kk][2 * h + 1] = hi;   // row gid + 8
        ps0 += bf16_lo(lo) + bf16_hi(lo);
        ps1 += bf16_lo(hi) + bf16_hi(hi);
      }
    }
    l0 = l0 * alpha0 + ps0;
    l1 = l1 * alpha1 + ps1;
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      o[i][0] *= alpha0; o[i][1] *= alpha0;
      o[i][2] *= alpha1; o[i][3] *= alpha1;
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
      // A fragment: a0 = row gid, tokens lo; a1 = row gid+8, tokens lo; a2/a3 = tokens hi
      const uint32_t a0 = pa[kk][0], a1 = pa[kk][1], a2 = pa[kk][2], a3 = pa[kk][3];
#pragma unroll
      for (int ndp = 0; ndp < D / 16; ++ndp) {
        const int mat = lane >> 3;
        const int tok = kk * 16 + (mat & 1) * 8 + (lane & 7);
        const int chk = ndp * 2 + (mat >> 1);
        uint32_t r0, r1, r2, r3;
        ldmatrix_x4_trans(r0, r1, r2, r3, smem_u32(vd + tok * L::kRowBytes + ((chk ^ (tok & 7)) * 16)));
        mma_bf16_16816(o[2 * ndp], a0, a1, a2, a3, r0, r1);
        mma_bf16_16816(o[2 * ndp + 1], a0, a1, a2, a3, r2, r3);
      }
    }
    __syncwarp();
    stage ^= 1;
  }
  l0 += __shfl_xor_sync(0xFFFFFFFFu, l0, 1);
  l0 += __shfl_xor_sync(0xFFFFFFFFu, l0, 2);
  l1 += __shfl_xor_sync(0xFFFFFFFFu, l1, 1);
  l1 += __shfl_xor_sync(0xFFFFFFFFu, l1, 2);

  // ---- merge the 4 warps in a fixed order ---------------------------------------------------
  __syncthreads();
  float* mg = reinterpret_cast<float*>(smem);               // [warp][16][D] then m, l
  float* mg_m = mg + kWarps * 16 * D;                        // [warp][16]
  float* mg_l = mg_m + kWarps * 16;                          // [warp][16]
#pragma unroll
  for (int nt = 0; nt < D / 8; ++nt) {
    const int col = nt * 8 + tig * 2;
    float* r0p = mg + (warp * 16 + gid) * D + col;
    float* r1p = mg + (warp * 16 + gid + 8) * D + col;
    r0p[0] = o[nt][0]; r0p[1] = o[nt][1];
    r1p[0] = o[nt][2]; r1p[1] = o[nt][3];
  }
  if (tig == 0) {
    mg_m[warp * 16 + gid] = m0;
    mg_m[warp * 16 + gid + 8] = m1;
    mg_l[warp * 16 + gid] = l0;
    mg_l[warp * 16 + gid + 8] = l1;
  }
  __syncthreads();
  const int items = R * (D / 8);
  for (int it = tid; it < items; it += kWarps * 32) {
    const int h = it / (D / 8), e0 = (it % (D / 8)) * 8;
    float mstar = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) mstar = fmaxf(mstar, mg_m[w * 16 + h]);
    float den = 0.f, num[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) num[e] = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float mw = mg_m[w * 16 + h];
      const float wt = mw == -INFINITY ? 0.f : exp2f((mw - mstar) * sc);
      den += wt * mg_l[w * 16 + h];
      const float* ow = mg + (w * 16 + h) * D + e0;
#pragma unroll
      for (int e = 0; e < 8; ++e) num[e] += wt * ow[e];
    }
    if (a.splits == 1) {
      const long orow = (qrow + h) * D + e0;
      const uint4 gv = __ldg(reinterpret_cast<const uint4*>(a.gate + orow));
      const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
      const float inv = den > 0.f ? 1.f / den : 0.f;
      uint32_t ov[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float g0 = bf16_lo(gw[i]), g1 = bf16_hi(gw[i]);
        const float y0 = num[2 * i] * inv * (1.f / (1.f + expf(-g0)));
        const float y1 = num[2 * i + 1] * inv * (1.f / (1.f + expf(-g1)));
        ov[i] = pack_bf16x2(y0, y1);
      }
      *reinterpret_cast<uint4*>(a.out + orow) = make_uint4(ov[0], ov[1], ov[2], ov[3]);
    } else {
      // partial record of (unit, split): m[16], l[16], o[16][D]
      float* rec = a.part + ((long)unit * a.splits + split) * (32 + 16 * D);
      if (e0 == 0) {
        rec[h] = mstar;
        rec[16 + h] = den;
      }
      float* ro = rec + 32 + h * D + e0;
#pragma unroll
      for (int e = 0; e < 8; ++e) ro[e] = num[e];
    }
  }
}

template <int D>
__global__ void __launch_bounds__(128) attend_merge_kernel(AttendArgs a) {
  const int R = a.Hq / a.G;
  const int nT = a.t_end - a.t_begin;
  const int unit = blockIdx.x;
  const int g = unit / (a.batch * nT);
  const int rem = unit % (a.batch * nT);
  const int b = rem / nT;
  const int t = a.t_end - 1 - rem % nT;
  const float sc = kLog2e / sqrtf((float)D);
  const long qrow = ((long)b * a.nQ + (t - a.q_t0)) * a.Hq + (long)g * R;
  const float* base = a.part + (long)unit * a.splits * (32 + 16 * D);
  const int items = R * (D / 8);
  for (int it = threadIdx.x; it < items; it += blockDim.x) {
    const int h = it / (D / 8), e0 = (it % (D / 8)) * 8;
    float mstar = -INFINITY;
    for (int s = 0; s < a.splits; ++s) mstar = fmaxf(mstar, base[s * (32 + 16 * D) + h]);
    float den = 0.f, num[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) num[e] = 0.f;
    for (int s = 0; s < a.splits; ++s) {
      const float* rec = base + s * (32 + 16 * D);
      const float ms = rec[h];
      const float wt = ms == -INFINITY ? 0.f : exp2f((ms - mstar) * sc);
      den += wt * rec[16 + h];
#pragma unroll
      for (int e = 0; e < 8; ++e) num[e] += wt * rec[32 + h * D + e0 + e];
    }
    const long orow = (qrow + h) * D + e0;
    const uint4 gv = __ldg(reinterpret_cast<const uint4*>(a.gate + orow));
    const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
    const float inv = den > 0.f ? 1.f / den : 0.f;
    uint32_t ov[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float g0 = bf16_lo(gw[i]), g1 = bf16_hi(gw[i]);
      ov[i] = pack_bf16x2(num[2 * i] * inv * (1.f / (1.f + expf(-g0))),
                          num[2 * i + 1] * inv * (1.f / (1.f + expf(-g1))));
    }
    *reinterpret_cast<uint4*>(a.out + orow) = make_uint4(ov[0], ov[1], ov[2], ov[3]);
  }
}

template <int D>
cudaError_t launch_d(const AttendArgs& a, cudaStream_t s) {
  using L = AttendSmem<D>;
  const size_t shmem = (size_t)L::kStaging + (size_t)a.Kb * 4;
  cudaError_t e = cudaFuncSetAttribute(attend_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shmem);
  if (e != cudaSuccess) return e;
  const long units = (long)a.batch * a.G * (a.t_end - a.t_begin);
  attend_kernel<D><<<dim3((unsigned)units, (unsigned)a.splits), kWarps * 32, shmem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

size_t attend_part_bytes(int units, int splits, int R, int d) {
  (void)R;
  return (size_t)units * splits * (32 + 16 * (size_t)d) * sizeof(float);
}

cudaError_t launch_attend(const AttendArgs& a, cudaStream_t s) {
  if (a.t_end <= a.t_begin) return cudaSuccess;
  if (a.d == 128) return launch_d<128>(a, s);
  if (a.d == 64) return launch_d<64>(a, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_attend_merge(const AttendArgs& a, cudaStream_t s) {
  if (a.t_end <= a.t_begin || a.splits <= 1) return cudaSuccess;
  const long units = (long)a.batch * a.G * (a.t_end - a.t_begin);
  if (a.d == 128) attend_merge_kernel<128><<<(unsigned)units, 128, 0, s>>>(a);
  else if (a.d == 64) attend_merge_kernel<64><<<(unsigned)units, 128, 0, s>>>(a);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace sgqa
