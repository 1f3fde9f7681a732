// C ABI of libsgqa: argument validation, workspace layout and the kernel sequence of every
// entry point declared in include/sgqa.h. No allocation, no host synchronisation (except the
// explicit status read), no global state.
#include <cstdint>
#include <cstring>

#include "common.cuh"
#include "kernels.h"

using namespace sgqa;

namespace {

constexpr int kSelChunkT = 32768;  // query rows per selection chunk when sel stays in ws
constexpr size_t kSelBitsBudget = 256ull << 20;  // bitmaps of the taken candidates (K2 -> block lists)
int g_test_stall_cta = -1;         // sgqa_test_stall_decode_cta (failure-detection tests only)

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_dims(const sgqa_dims* d) {
  if (!d) return SGQA_ERR_INVALID_ARG;
  if (d->batch <= 0 || d->T <= 0 || d->Hq <= 0 || d->G <= 0 || d->d <= 0 || d->d_idx <= 0 || d->B <= 0 ||
      d->k <= 0)
    return SGQA_ERR_INVALID_ARG;
  if (d->T >= (1 << 28) || d->batch > 65535) return SGQA_ERR_UNSUPPORTED;
  // row indices of q, gate, out and q_idx (and TMA coordinates) are 32-bit
  if ((long)d->batch * d->T * (d->Hq > d->G ? d->Hq : d->G) >= (1L << 31)) return SGQA_ERR_UNSUPPORTED;
  if (d->d != 64 && d->d != 128) return SGQA_ERR_UNSUPPORTED;
  if (d->d_idx != 32 && d->d_idx != 64) return SGQA_ERR_UNSUPPORTED;
  if (d->B != 1 && d->B != 2 && d->B != 4 && d->B != 8 && d->B != 16) return SGQA_ERR_UNSUPPORTED;
  if (d->k % d->B != 0) return SGQA_ERR_UNSUPPORTED;
  if (d->Hq % d->G != 0 || d->Hq / d->G > 16 || 128 % d->G != 0) return SGQA_ERR_UNSUPPORTED;
  if (d->k / d->B > 16384) return SGQA_ERR_UNSUPPORTED;
  return SGQA_OK;
}

struct PrefillWs {
  int* status;
  void* plan;
  float* kbar;
  uint16_t* hi;
  uint16_t* lo;
  uint32_t* bits;
  int bstride, bits_q;
  int32_t* sel;
  size_t bytes;
};

PrefillWs prefill_layout(const sgqa_dims* d, void* ws) {
  PrefillWs w{};
  const size_t nblk = (size_t)(d->T / d->B);
  const size_t nk = (size_t)d->batch * nblk * d->d_idx;
  const size_t chunk = (size_t)(d->T < kSelChunkT ? d->T : kSelChunkT);
  size_t off = kStatusBytes;
  uint8_t* base = static_cast<uint8_t*>(ws);
  w.status = reinterpret_cast<int*>(base);
  w.plan = base + off;
  off += plan_bytes((long)d->batch * d->T * d->G, d->batch * d->G, d->T);
  w.kbar = reinterpret_cast<float*>(base + off);
  off += align256(nk * 4);
  w.hi = reinterpret_cast<uint16_t*>(base + off);
  off += align256(nk * 2);
  w.lo = reinterpret_cast<uint16_t*>(base + off);
  off += align256(nk * 2);
  select_bits_dims(d->batch, d->T, d->G, d->B, kSelBitsBudget, &w.bstride, &w.bits_q);
  w.bits = reinterpret_cast<uint32_t*>(base + off);
  off += align256((size_t)d->batch * w.bits_q * d->G * (size_t)w.bstride * 4);
  w.sel = reinterpret_cast<int32_t*>(base + off);
  off += align256((size_t)d->batch * chunk * d->G * (d->k / d->B) * 4);
  w.bytes = off;
  return w;
}

int decode_splits(long units) {
  long s = 4096 / (units > 0 ? units : 1);
  if (s < 1) s = 1;
  if (s > 16) s = 16;
  return (int)s;
}

struct DecodeWs {
  int* status;
  float* scores;
  uint32_t* tmax;   // per row, the largest key of every 32 candidates (tcgen05 scoring path)
  int tstride;
  bool tc_scores;   // tcgen05 scoring and the bound-based select run (else the CUDA-core K4/K5)
  int32_t* sel;
  int32_t* ublk;    // union of the n_new selections per (sequence, group) (tcgen05 path)
  uint32_t* umask;
  int* ucount;
  float* part;      // split-K partial records
  int splits;
  bool tc;          // the tcgen05 attention runs (else the per-row kernel)
  size_t bytes;
};

DecodeWs decode_layout(const sgqa_dims* d, int n_new, void* ws) {
  DecodeWs w{};
  const size_t nblk = (size_t)(d->T / d->B);
  const int Kb = d->k / d->B;
  const long units = (long)d->batch * n_new * d->G;
  const int ug = d->batch * d->G;
  uint8_t* base = static_cast<uint8_t*>(ws);
  size_t off = kStatusBytes;
  w.status = reinterpret_cast<int*>(base);
  w.scores = reinterpret_cast<float*>(base + off);
  off += align256((size_t)units * nblk * 4);
  w.tc_scores = decode_scores_tc_supported(d->d_idx, n_new, d->G);
  w.tstride = (int)((nblk + 31) / 32);
  if (w.tc_scores) {
    w.tmax = reinterpret_cast<uint32_t*>(base + off);
    off += align256((size_t)units * w.tstride * 4);
  }
  w.sel = reinterpret_cast<int32_t*>(base + off);
  off += align256((size_t)units * Kb * 4);
  w.tc = decode_attend_tc_supported(d->Hq, d->G, d->d, d->B, n_new, Kb);
  if (w.tc) {
    const size_t ucap = (size_t)n_new * Kb;
    w.ublk = reinterpret_cast<int32_t*>(base + off);
    off += align256((size_t)ug * ucap * 4);
    w.umask = reinterpret_cast<uint32_t*>(base + off);
    off += align256((size_t)ug * ucap * 4);
    w.ucount = reinterpret_cast<int*>(base + off);
    off += align256((size_t)ug * 4);
    w.splits = decode_attend_splits(ug, n_new, Kb, d->B, false);  // the larger of the two variants
    w.part = reinterpret_cast<float*>(base + off);
    off += align256(decode_part_bytes(ug, w.splits));
  } else {
    w.splits = decode_splits(units);
    w.part = reinterpret_cast<float*>(base + off);
    off += align256(attend_part_bytes((int)units, w.splits, d->Hq / d->G, d->d));
  }
  w.bytes = off;
  return w;
}

struct BackwardWs {
  int* status;
  float* lse;
  float* dsum;
  float* dov;
  int* rcount;
  int* ccount;
  int* roff;
  int* rlist;
  int nblkc, rchunk, nchunk;
  size_t bytes;
};

BackwardWs backward_layout(const sgqa_dims* d, void* ws) {
  BackwardWs w{};
  uint8_t* base = static_cast<uint8_t*>(ws);
  const size_t rows = (size_t)d->batch * d->T;
  const size_t segs = (size_t)d->batch * d->G;
  w.nblkc = (d->T + d->B - 1) / d->B;
  // chunks of at least 256 rows, at most 256 chunks (bounds the per-chunk count table)
  w.rchunk = 256;
  while ((d->T + w.rchunk - 1) / w.rchunk > 256) w.rchunk *= 2;
  w.nchunk = (d->T + w.rchunk - 1) / w.rchunk;
  size_t off = kStatusBytes;
  w.status = reinterpret_cast<int*>(base);
  w.lse = reinterpret_cast<float*>(base + off);
  off += align256(rows * d->Hq * 4);
  w.dsum = reinterpret_cast<float*>(base + off);
  off += align256(rows * d->Hq * 4);
  w.dov = reinterpret_cast<float*>(base + off);
  off += align256(rows * d->Hq * (size_t)d->d * 4);
  w.rcount = reinterpret_cast<int*>(base + off);
  off += align256(segs * w.nblkc * 4);
  w.roff = reinterpret_cast<int*>(base + off);
  off += align256(segs * (w.nblkc + 1) * 4);
  w.ccount = reinterpret_cast<int*>(base + off);
  off += align256(segs * (size_t)w.nchunk * w.nblkc * 4);
  w.rlist = reinterpret_cast<int*>(base + off);
  off += align256(segs * (size_t)d->T * (d->k / d->B) * 4);
  w.bytes = off;
  return w;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? SGQA_OK : SGQA_ERR_CUDA; }

// Prefill attention for query rows [a.t_begin, a.t_end): schedule the rows by selection
// similarity, then the tiled union kernel; shapes it does not cover use the per-row kernel.
cudaError_t launch_prefill_attend(const AttendArgs& a, void* plan_ws, cudaStream_t s) {
  if (!attend_tiles_supported(a.Hq, a.G, a.B)) return launch_attend(a, s);
  const uint32_t* perm = nullptr;
  cudaError_t e = launch_plan(a.sel, a.sel_T, a.sel_t0, a.batch, a.G, a.Kb, a.B, a.t_begin, a.t_end, plan_ws, &perm, s);
  if (e != cudaSuccess) return e;
  if (attend_tc_supported(a.Hq, a.G, a.B, a.d)) return launch_attend_tc(a, perm, s);
  return launch_attend_tiles(a, perm, s);
}

}  // namespace

extern "C" {

const char* sgqa_status_string(int status) {
  switch (status) {
    case SGQA_OK: return "ok";
    case SGQA_ERR_INVALID_ARG: return "invalid argument";
    case SGQA_ERR_UNSUPPORTED: return "unsupported shape";
    case SGQA_ERR_WORKSPACE: return "workspace too small or misaligned";
    case SGQA_ERR_CUDA: return "CUDA error";
    case SGQA_ERR_TIMEOUT: return "device wait timed out";
    case SGQA_ERR_DEVICE_CHECK: return "device-side check failed";
    default: return "unknown status";
  }
}

const char* sgqa_version(void) { return "sgqa 0.1 sm_100a"; }

size_t sgqa_workspace_size(const sgqa_dims* dims) {
  if (check_dims(dims) != SGQA_OK) return 0;
  return prefill_layout(dims, nullptr).bytes;
}

size_t sgqa_decode_workspace_size(const sgqa_dims* dims, int n_new) {
  if (check_dims(dims) != SGQA_OK || n_new <= 0 || n_new * dims->G > 32) return 0;
  return decode_layout(dims, n_new, nullptr).bytes;
}

int sgqa_reset_device_status(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < kStatusBytes) return SGQA_ERR_WORKSPACE;
  return cuda_status(cudaMemsetAsync(ws, 0, sizeof(int), static_cast<cudaStream_t>(stream)));
}

int sgqa_get_device_status(const void* ws, size_t ws_bytes, int* status) {
  if (!ws || ws_bytes < kStatusBytes || !status) return SGQA_ERR_INVALID_ARG;
  int v = 0;
  const cudaError_t e = cudaMemcpy(&v, ws, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return SGQA_ERR_CUDA;
  *status = v;
  return SGQA_OK;
}

int sgqa_compress_keys(const sgqa_dims* dims, const uint16_t* k_idx, float* kbar, void* ws, size_t ws_bytes,
                       void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (dims->T / dims->B == 0) return SGQA_OK;  // no complete block: nothing to write
  if (!aligned16(k_idx) || !aligned16(kbar)) return SGQA_ERR_INVALID_ARG;
  (void)ws;
  (void)ws_bytes;
  return cuda_status(launch_compress(k_idx, kbar, nullptr, nullptr, dims->batch, dims->T, dims->d_idx, dims->B, 0,
                                     dims->T / dims->B, static_cast<cudaStream_t>(stream)));
}

int sgqa_select(const sgqa_dims* dims, const uint16_t* q_idx, const float* kbar, int32_t* sel, void* ws,
                size_t ws_bytes, void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (!aligned16(q_idx) || (dims->T >= dims->B && !aligned16(kbar)) || !aligned16(sel)) return SGQA_ERR_INVALID_ARG;
  const PrefillWs w = prefill_layout(dims, ws);
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < (size_t)((uint8_t*)w.sel - (uint8_t*)ws))
    return SGQA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  SelectArgs a{};
  a.q_idx = q_idx; a.q_T = dims->T; a.q_t0 = 0; a.kbar = kbar; a.kbar_hi = w.hi; a.kbar_lo = w.lo; a.sel = sel;
  a.batch = dims->batch; a.T = dims->T; a.G = dims->G; a.d_idx = dims->d_idx; a.B = dims->B;
  a.Kb = dims->k / dims->B; a.t_begin = 0; a.t_end = dims->T; a.sel_T = dims->T; a.sel_t0 = 0;
  a.bits = w.bits; a.bstride = w.bstride; a.bits_q = w.bits_q;
  a.status = w.status;
  if (launch_split_planes(kbar, w.hi, w.lo, (long)dims->batch * (dims->T / dims->B) * dims->d_idx, s) !=
      cudaSuccess)
    return SGQA_ERR_CUDA;
  return cuda_status(launch_select(a, s));
}

static AttendArgs prefill_attend_args(const sgqa_dims* d, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                      const uint16_t* gate, uint16_t* out, int* status) {
  AttendArgs a{};
  a.q = q; a.gate = gate; a.out = out; a.k = k; a.v = v;
  a.batch = d->batch; a.nQ = d->T; a.q_t0 = 0; a.T_kv = d->T; a.Hq = d->Hq; a.G = d->G; a.d = d->d;
  a.B = d->B; a.Kb = d->k / d->B; a.splits = 1; a.status = status;
  return a;
}

int sgqa_attend(const sgqa_dims* dims, const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* gate,
                const int32_t* sel, uint16_t* out, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(gate) || !aligned16(sel) || !aligned16(out))
    return SGQA_ERR_INVALID_ARG;
  const PrefillWs w = prefill_layout(dims, ws);
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < w.bytes) return SGQA_ERR_WORKSPACE;
  AttendArgs a = prefill_attend_args(dims, q, k, v, gate, out, w.status);
  a.sel = sel; a.sel_T = dims->T; a.sel_t0 = 0; a.t_begin = 0; a.t_end = dims->T;
  return cuda_status(launch_prefill_attend(a, w.plan, static_cast<cudaStream_t>(stream)));
}

// The layer for query rows [t_begin, t_end) of every sequence: q, gate, q_idx, out (and sel_out)
// hold those rows only; k, v, k_idx hold whole sequences.
static int forward_rows_impl(const sgqa_dims* dims, int t_begin, int t_end, const uint16_t* q, const uint16_t* k,
                             const uint16_t* v, const uint16_t* q_idx, const uint16_t* k_idx, const uint16_t* gate,
                             uint16_t* out, int32_t* sel_out, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (t_begin < 0 || t_end > dims->T || t_begin > t_end) return SGQA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q_idx) || !aligned16(k_idx) ||
      !aligned16(gate) || !aligned16(out) || (sel_out && !aligned16(sel_out)))
    return SGQA_ERR_INVALID_ARG;
  const PrefillWs w = prefill_layout(dims, ws);
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < w.bytes) return SGQA_ERR_WORKSPACE;
  if (t_end == t_begin) return SGQA_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int nq = t_end - t_begin;
  if (launch_compress(k_idx, w.kbar, w.hi, w.lo, dims->batch, dims->T, dims->d_idx, dims->B, 0, dims->T / dims->B,
                      s) != cudaSuccess)
    return SGQA_ERR_CUDA;
  SelectArgs sa{};
  sa.q_idx = q_idx; sa.q_T = nq; sa.q_t0 = t_begin; sa.kbar = w.kbar; sa.kbar_hi = w.hi; sa.kbar_lo = w.lo;
  sa.batch = dims->batch; sa.T = dims->T; sa.G = dims->G; sa.d_idx = dims->d_idx; sa.B = dims->B;
  sa.Kb = dims->k / dims->B; sa.status = w.status;
  sa.bits = w.bits; sa.bstride = w.bstride; sa.bits_q = w.bits_q;
  AttendArgs aa = prefill_attend_args(dims, q, k, v, gate, out, w.status);
  aa.nQ = nq; aa.q_t0 = t_begin;
  const int chunk = sel_out ? nq : (nq < kSelChunkT ? nq : kSelChunkT);
  for (int t0 = t_begin; t0 < t_end; t0 += chunk) {
    const int t1 = t0 + chunk < t_end ? t0 + chunk : t_end;
    sa.sel = sel_out ? sel_out : w.sel;
    sa.sel_T = sel_out ? nq : chunk;
    sa.sel_t0 = sel_out ? t_begin : t0;
    sa.t_begin = t0; sa.t_end = t1;
    if (launch_select(sa, s) != cudaSuccess) return SGQA_ERR_CUDA;
    aa.sel = sa.sel; aa.sel_T = sa.sel_T; aa.sel_t0 = sa.sel_t0; aa.t_begin = t0; aa.t_end = t1;
    if (launch_prefill_attend(aa, w.plan, s) != cudaSuccess) return SGQA_ERR_CUDA;
  }
  return SGQA_OK;
}

int sgqa_forward(const sgqa_dims* dims, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                 const uint16_t* q_idx, const uint16_t* k_idx, const uint16_t* gate, uint16_t* out,
                 int32_t* sel_out, void* ws, size_t ws_bytes, void* stream) {
  if (!dims) return SGQA_ERR_INVALID_ARG;
  return forward_rows_impl(dims, 0, dims->T, q, k, v, q_idx, k_idx, gate, out, sel_out, ws, ws_bytes, stream);
}

int sgqa_forward_rows(const sgqa_dims* dims, int t_begin, int t_end, const uint16_t* q_rows, const uint16_t* k,
                      const uint16_t* v, const uint16_t* q_idx_rows, const uint16_t* k_idx,
                      const uint16_t* gate_rows, uint16_t* out_rows, int32_t* sel_out_rows, void* ws,
                      size_t ws_bytes, void* stream) {
  return forward_rows_impl(dims, t_begin, t_end, q_rows, k, v, q_idx_rows, k_idx, gate_rows, out_rows, sel_out_rows,
                           ws, ws_bytes, stream);
}

int sgqa_gated_swa(const sgqa_dims* dims, int window, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                   const uint16_t* gate, uint16_t* out, int32_t* sel_out, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (window < dims->B || (long)dims->k < (long)window + dims->B) return SGQA_ERR_INVALID_ARG;
  if (!attend_tc_supported(dims->Hq, dims->G, dims->B, dims->d)) return SGQA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(gate) || !aligned16(out) ||
      (sel_out && !aligned16(sel_out)))
    return SGQA_ERR_INVALID_ARG;
  const PrefillWs w = prefill_layout(dims, ws);
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < w.bytes) return SGQA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  AttendArgs aa = prefill_attend_args(dims, q, k, v, gate, out, w.status);
  aa.window = window;
  const int Kb = dims->k / dims->B;
  const int chunk = sel_out ? dims->T : (dims->T < kSelChunkT ? dims->T : kSelChunkT);
  for (int t0 = 0; t0 < dims->T; t0 += chunk) {
    const int t1 = t0 + chunk < dims->T ? t0 + chunk : dims->T;
    aa.sel = sel_out ? sel_out : w.sel;
    aa.sel_T = sel_out ? dims->T : chunk;
    aa.sel_t0 = sel_out ? 0 : t0;
    aa.t_begin = t0; aa.t_end = t1;
    if (launch_window_select(const_cast<int32_t*>(aa.sel), aa.sel_T, aa.sel_t0, dims->batch, dims->G, Kb, dims->B,
                             window, t0, t1, s) != cudaSuccess)
      return SGQA_ERR_CUDA;
    if (launch_prefill_attend(aa, w.plan, s) != cudaSuccess) return SGQA_ERR_CUDA;
  }
  return SGQA_OK;
}

}  // extern "C"

namespace {

// K/V caches of a decode step: bf16 (k, v) or fp8 (k8, v8 with row scales)
struct KvCaches {
  uint16_t* k;
  uint16_t* v;
  uint8_t* k8;
  uint8_t* v8;
  float* k_scale;
  float* v_scale;
};

int decode_impl(const sgqa_dims* dims, int cache_len, int n_new, const KvCaches& kv, uint16_t* kidx_cache,
                float* kbar_cache, const uint16_t* q_new, const uint16_t* k_new, const uint16_t* v_new,
                const uint16_t* qidx_new, const uint16_t* kidx_new, const uint16_t* gate_new, uint16_t* out,
                int32_t* sel_out, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (n_new <= 0 || cache_len < 0 || (long)cache_len + n_new > dims->T || n_new * dims->G > 32)
    return SGQA_ERR_INVALID_ARG;
  const bool f8 = kv.k8 != nullptr;
  if (f8 ? (!aligned16(kv.k8) || !aligned16(kv.v8) || !aligned16(kv.k_scale) || !aligned16(kv.v_scale))
         : (!aligned16(kv.k) || !aligned16(kv.v)))
    return SGQA_ERR_INVALID_ARG;
  if (!aligned16(kidx_cache) || !aligned16(kbar_cache) || !aligned16(q_new) || !aligned16(k_new) ||
      !aligned16(v_new) || !aligned16(qidx_new) || !aligned16(kidx_new) || !aligned16(gate_new) || !aligned16(out) ||
      (sel_out && !aligned16(sel_out)))
    return SGQA_ERR_INVALID_ARG;
  const DecodeWs w = decode_layout(dims, n_new, ws);
  if (f8 && !w.tc) return SGQA_ERR_UNSUPPORTED;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < w.bytes) return SGQA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int T = dims->T, G = dims->G, d = dims->d, di = dims->d_idx, B = dims->B, Kb = dims->k / dims->B;
  const int nblk = T / B;
  cudaError_t e = cudaSuccess;
  // 1. append the new rows (quantized for fp8 caches)
  if (f8) {
    if ((e = launch_quantize_fp8(k_new, kv.k8, kv.k_scale, dims->batch, n_new, G, T, cache_len, s)) != cudaSuccess ||
        (e = launch_quantize_fp8(v_new, kv.v8, kv.v_scale, dims->batch, n_new, G, T, cache_len, s)) != cudaSuccess)
      return SGQA_ERR_CUDA;
  } else {
    if ((e = launch_append(kv.k, k_new, dims->batch, (long)G * d, (long)T * G * d, (long)cache_len * G * d,
                           (long)n_new * G * d, s)) != cudaSuccess)
      return SGQA_ERR_CUDA;
    if ((e = launch_append(kv.v, v_new, dims->batch, (long)G * d, (long)T * G * d, (long)cache_len * G * d,
                           (long)n_new * G * d, s)) != cudaSuccess)
      return SGQA_ERR_CUDA;
  }
  if ((e = launch_append(kidx_cache, kidx_new, dims->batch, di, (long)T * di, (long)cache_len * di, (long)n_new * di,
                         s)) != cudaSuccess)
    return SGQA_ERR_CUDA;
  // 2. block means of the blocks the new rows complete
  const int j0 = cache_len / B, j1 = (cache_len + n_new) / B;
  if (j1 > j0 && (e = launch_compress(kidx_cache, kbar_cache, nullptr, nullptr, dims->batch, T, di, B, j0, j1, s)) !=
                     cudaSuccess)
    return SGQA_ERR_CUDA;
  // 3. indexer scores and selection
  int32_t* sel = sel_out ? sel_out : w.sel;
  if (w.tc_scores) {
    DecodeScoreArgs sa{};
    sa.qidx = qidx_new; sa.kbar = kbar_cache; sa.scores = w.scores; sa.tmax = w.tmax; sa.batch = dims->batch;
    sa.n_new = n_new; sa.G = G; sa.B = B; sa.nblk = nblk; sa.tstride = w.tstride; sa.t0 = cache_len;
    sa.cps = decode_scores_ctas(dims->batch, (cache_len + n_new - 1) / B); sa.status = w.status;
    if ((e = launch_decode_scores_tc(sa, s)) != cudaSuccess) return SGQA_ERR_CUDA;
    if ((e = launch_decode_select_bound(w.scores, w.tmax, sel, dims->batch, n_new, G, B, Kb, nblk, w.tstride,
                                        cache_len, w.status, s)) != cudaSuccess)
      return SGQA_ERR_CUDA;
  } else {
    if ((e = launch_decode_scores(qidx_new, kbar_cache, w.scores, dims->batch, n_new, G, di, B, nblk, cache_len,
                                  s)) != cudaSuccess)
      return SGQA_ERR_CUDA;
    if ((e = launch_decode_select(w.scores, sel, dims->batch, n_new, G, B, Kb, nblk, cache_len, w.status, s)) !=
        cudaSuccess)
      return SGQA_ERR_CUDA;
  }
  // 4. gated attention over the selection
  if (w.tc) {
    if (launch_decode_union(sel, dims->batch, n_new, G, Kb, w.ublk, w.umask, w.ucount, n_new * Kb, w.status, s) != cudaSuccess)
      return SGQA_ERR_CUDA;
    DecodeAttendArgs da{};
    da.q = q_new; da.gate = gate_new; da.out = out; da.k = kv.k; da.v = kv.v;
    da.k8 = kv.k8; da.v8 = kv.v8; da.k_scale = kv.k_scale; da.v_scale = kv.v_scale;
    da.ublk = w.ublk; da.umask = w.umask; da.ucount = w.ucount; da.ucap = n_new * Kb; da.part = w.part;
    da.batch = dims->batch; da.n_new = n_new; da.t0 = cache_len; da.T_kv = T; da.Hq = dims->Hq; da.G = G; da.d = d;
    da.B = B; da.status = w.status; da.stall_cta = g_test_stall_cta;
    da.splits = decode_attend_splits(dims->batch * G, n_new, Kb, B, kv.k8 != nullptr);  // <= w.splits
    if (launch_decode_attend_tc(da, s) != cudaSuccess) return SGQA_ERR_CUDA;
    return SGQA_OK;
  }
  AttendArgs a{};
  a.q = q_new; a.gate = gate_new; a.out = out; a.k = kv.k; a.v = kv.v; a.sel = sel; a.part = w.part;
  a.batch = dims->batch; a.nQ = n_new; a.q_t0 = cache_len; a.T_kv = T; a.Hq = dims->Hq; a.G = G; a.d = d; a.B = B;
  a.Kb = Kb; a.sel_T = n_new; a.sel_t0 = cache_len; a.t_begin = cache_len; a.t_end = cache_len + n_new;
  a.splits = w.splits;
  a.status = w.status;
  if ((e = launch_attend(a, s)) != cudaSuccess) return SGQA_ERR_CUDA;
  if ((e = launch_attend_merge(a, s)) != cudaSuccess) return SGQA_ERR_CUDA;
  return SGQA_OK;
}


}  // namespace

extern "C" {

int sgqa_decode(const sgqa_dims* dims, int cache_len, int n_new, uint16_t* k_cache, uint16_t* v_cache,
                uint16_t* kidx_cache, float* kbar_cache, const uint16_t* q_new, const uint16_t* k_new,
                const uint16_t* v_new, const uint16_t* qidx_new, const uint16_t* kidx_new, const uint16_t* gate_new,
                uint16_t* out, int32_t* sel_out, void* ws, size_t ws_bytes, void* stream) {
  KvCaches kv{};
  kv.k = k_cache;
  kv.v = v_cache;
  return decode_impl(dims, cache_len, n_new, kv, kidx_cache, kbar_cache, q_new, k_new, v_new, qidx_new, kidx_new,
                     gate_new, out, sel_out, ws, ws_bytes, stream);
}

int sgqa_decode_fp8(const sgqa_dims* dims, int cache_len, int n_new, uint8_t* k8_cache, float* k_scale,
                    uint8_t* v8_cache, float* v_scale, uint16_t* kidx_cache, float* kbar_cache, const uint16_t* q_new,
                    const uint16_t* k_new, const uint16_t* v_new, const uint16_t* qidx_new, const uint16_t* kidx_new,
                    const uint16_t* gate_new, uint16_t* out, int32_t* sel_out, void* ws, size_t ws_bytes,
                    void* stream) {
  if (!k8_cache || !v8_cache || !k_scale || !v_scale) return SGQA_ERR_INVALID_ARG;
  KvCaches kv{};
  kv.k8 = k8_cache;
  kv.v8 = v8_cache;
  kv.k_scale = k_scale;
  kv.v_scale = v_scale;
  return decode_impl(dims, cache_len, n_new, kv, kidx_cache, kbar_cache, q_new, k_new, v_new, qidx_new, kidx_new,
                     gate_new, out, sel_out, ws, ws_bytes, stream);
}

size_t sgqa_backward_workspace_size(const sgqa_dims* dims) {
  if (check_dims(dims) != SGQA_OK || !backward_supported(dims->Hq, dims->G, dims->d, dims->B)) return 0;
  return backward_layout(dims, nullptr).bytes;
}

int sgqa_attend_backward(const sgqa_dims* dims, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                         const uint16_t* gate, const int32_t* sel, const uint16_t* dout, float* dq, float* dk,
                         float* dv, float* dgate, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (!backward_supported(dims->Hq, dims->G, dims->d, dims->B)) return SGQA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(gate) || !aligned16(sel) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(dgate))
    return SGQA_ERR_INVALID_ARG;
  const BackwardWs w = backward_layout(dims, ws);
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < w.bytes) return SGQA_ERR_WORKSPACE;
  BackwardArgs a{};
  a.q = q; a.k = k; a.v = v; a.gate = gate; a.dy = dout; a.sel = sel;
  a.dq = dq; a.dk = dk; a.dv = dv; a.dgate = dgate; a.lse = w.lse; a.dsum = w.dsum; a.dov = w.dov;
  a.rcount = w.rcount; a.ccount = w.ccount; a.roff = w.roff; a.rlist = w.rlist;
  a.batch = dims->batch; a.T = dims->T; a.Hq = dims->Hq; a.G = dims->G; a.d = dims->d; a.B = dims->B;
  a.Kb = dims->k / dims->B; a.nblkc = w.nblkc; a.rchunk = w.rchunk; a.nchunk = w.nchunk; a.status = w.status;
  return cuda_status(launch_backward(a, static_cast<cudaStream_t>(stream)));
}

int sgqa_test_stall_decode_cta(int cta) {
  if (cta < -1) return SGQA_ERR_INVALID_ARG;
  g_test_stall_cta = cta;
  return SGQA_OK;
}

int sgqa_quantize_kv_fp8(const sgqa_dims* dims, int t0, int n_t, const uint16_t* src, uint8_t* dst8, float* dst_scale,
                         void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (dims->d != 128) return SGQA_ERR_UNSUPPORTED;
  if (t0 < 0 || n_t < 0 || (long)t0 + n_t > dims->T) return SGQA_ERR_INVALID_ARG;
  if (n_t == 0) return SGQA_OK;
  if (!aligned16(src) || !aligned16(dst8) || !aligned16(dst_scale)) return SGQA_ERR_INVALID_ARG;
  return cuda_status(launch_quantize_fp8(src, dst8, dst_scale, dims->batch, n_t, dims->G, dims->T, t0,
                                         static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
