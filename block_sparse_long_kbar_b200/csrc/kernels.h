// Internal launchers of libsgqa (host side). Not part of the C ABI.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace sgqa {

// K1: block means of k_idx for blocks [j0, j1) of every sequence.
//   k_idx [batch, T, d_idx] bf16; kbar [batch, T/B, d_idx] fp32; hi/lo planes (optional, may be
//   null) [batch, T/B, d_idx] bf16 with hi = bf16(kbar), lo = bf16(kbar - hi).
cudaError_t launch_compress(const uint16_t* k_idx, float* kbar, uint16_t* hi, uint16_t* lo, int batch,
                            int T, int d_idx, int B, int j0, int j1, cudaStream_t s);

// hi/lo bf16 planes of an fp32 kbar [batch, nblk, d_idx].
cudaError_t launch_split_planes(const float* kbar, uint16_t* hi, uint16_t* lo, long n, cudaStream_t s);

// K2: block selection for query rows t in [t_begin, t_end) of every sequence.
//   q_idx rows (b, t) at ((b * q_T + (t - q_t0)) * G + g) * d_idx (q_T = T, q_t0 = 0 for whole
//   sequences); kbar [batch, T/B, d_idx] fp32;
//   sel rows (b, t) at sel + ((b * sel_T + (t - sel_t0)) * G + g) * Kb.
struct SelectArgs {
  const uint16_t* q_idx;
  int q_T, q_t0;
  const float* kbar;
  const uint16_t* kbar_hi;
  const uint16_t* kbar_lo;
  int32_t* sel;
  int batch, T, G, d_idx, B, Kb;
  int t_begin, t_end;
  int sel_T, sel_t0;
  // bitmaps of the taken candidates, one row of bstride words per (token, group) of a query range
  // of at most bits_q tokens: row ((b * n + (t - range start)) * G + g), n the range's length
  uint32_t* bits;
  int bstride, bits_q;
  int* status;
};
cudaError_t launch_select(const SelectArgs& a, cudaStream_t s);
// bitmap row stride (words) and the query rows per range for a workspace budget of `budget` bytes
void select_bits_dims(int batch, int T, int G, int B, size_t budget, int* bstride, int* bits_q);

// K3: gated attention over selected blocks for query positions [t_begin, t_end).
//   q, gate rows (b, t) at ((b * nQ + (t - q_t0)) * Hq + h) * d; out likewise;
//   k, v [batch, T_kv, G, d]; sel rows (b, t) at ((b * sel_T + (t - sel_t0)) * G + g) * Kb.
//   splits > 1: partial (m, l, o) per split into `part`, combined by launch_attend_merge.
struct AttendArgs {
  const uint16_t* q;
  const uint16_t* gate;
  uint16_t* out;
  const uint16_t* k;
  const uint16_t* v;
  const int32_t* sel;
  float* part;
  int batch, nQ, q_t0, T_kv, Hq, G, d, B, Kb, sel_T, sel_t0;
  int t_begin, t_end;
  int splits;
  int* status;
  int window;  // > 0: only keys u > t - window count (Gated SWA); 0: no lower bound (tcgen05 path only)
};
cudaError_t launch_attend(const AttendArgs& a, cudaStream_t s);
cudaError_t launch_attend_merge(const AttendArgs& a, cudaStream_t s);
size_t attend_part_bytes(int units, int splits, int R, int d);

// Query scheduling for the tiled attention: per (sequence, group) segment, the rows of
// [t_begin, t_end) ordered by a MinHash signature of their selection (stable in t).
// *perm_out receives [batch * G][t_end - t_begin] row offsets (t - t_begin), inside ws.
size_t plan_bytes(long units, int n_seg, int n_per_seg);
cudaError_t launch_plan(const int32_t* sel, int sel_T, int sel_t0, int batch, int G, int Kb, int B, int t_begin,
                        int t_end, void* ws, const uint32_t** perm_out, cudaStream_t s);
// K3 tiled: tiles of consecutive rows of perm, union of their selections (requires ascending rows).
bool attend_tiles_supported(int Hq, int G, int B);
// Gated SWA: the selection of the blocks a window of `window` tokens ending at t overlaps
// (ascending, -1 padded), rows [t_begin, t_end) into sel (row t at sel_T offset t - sel_t0).
cudaError_t launch_window_select(int32_t* sel, int sel_T, int sel_t0, int batch, int G, int Kb, int B, int window,
                                 int t_begin, int t_end, cudaStream_t s);
cudaError_t launch_attend_tiles(const AttendArgs& a, const uint32_t* perm, cudaStream_t s);

// K3 on tcgen05 (R in {4, 8, 16}): same contract as launch_attend_tiles.
bool attend_tc_supported(int Hq, int G, int B, int d);
cudaError_t launch_attend_tc(const AttendArgs& a, const uint32_t* perm, cudaStream_t s);

// Decode helpers.
cudaError_t launch_append(uint16_t* dst, const uint16_t* src, int batch, long row_elems, long dst_seq_stride,
                          long dst_off, long n_elems_per_seq, cudaStream_t s);
// K4: fp32 scores of n_rows = n_new * G rows per sequence against every candidate block,
//   written to scores [batch, n_rows, nblk]; row r = i * G + g, query position t = t0 + i.
cudaError_t launch_decode_scores(const uint16_t* qidx_new, const float* kbar, float* scores, int batch,
                                 int n_new, int G, int d_idx, int B, int nblk, int t0, cudaStream_t s);
// K5: exact top-m select over the score rows; sel [batch, n_new, G, Kb].
// K4 on tcgen05 (d_idx = 64, n_new * G <= 32): scores as launch_decode_scores (row stride nblk,
// candidates j < c_max written) plus tmax [batch, n_new * G, tstride]: the largest order-preserving
// key of each 32 consecutive candidates j < t/B of the row (0 where there are none).
struct DecodeScoreArgs {
  const uint16_t* qidx;  // [batch, n_new, G, 64]
  const float* kbar;     // [batch, nblk, 64]
  float* scores;
  uint32_t* tmax;
  int batch, n_new, G, B, nblk, tstride, t0, cps;
  int* status;
};
bool decode_scores_tc_supported(int d_idx, int n_new, int G);
int decode_scores_ctas(int batch, int c_max);
cudaError_t launch_decode_scores_tc(const DecodeScoreArgs& a, cudaStream_t s);
// K5 with the bound from tmax (exact; falls back to the full radix select per row when needed).
cudaError_t launch_decode_select_bound(const float* scores, const uint32_t* tmax, int32_t* sel, int batch, int n_new,
                                       int G, int B, int Kb, int nblk, int tstride, int t0, int* status,
                                       cudaStream_t s);
cudaError_t launch_decode_select(const float* scores, int32_t* sel, int batch, int n_new, int G, int B, int Kb,
                                 int nblk, int t0, int* status, cudaStream_t s);

// K6 for decode on tcgen05 (d = 128, B in {8, 16}, n_new * Hq/G <= 64, n_new * Kb <= kUnionMax):
// per (sequence, group) the union of the n_new queries' selections (ascending block ids and the
// mask of the queries that selected each), then gated attention over it, split over `splits` CTAs
// per (sequence, group) with a fixed-order merge (part: decode_part_bytes).
constexpr int kUnionMax = 4096;
struct DecodeAttendArgs {
  const uint16_t* q;     // [batch, n_new, Hq, d]
  const uint16_t* gate;  // [batch, n_new, Hq, d]
  uint16_t* out;         // [batch, n_new, Hq, d]
  const uint16_t* k;     // caches [batch, T_kv, G, d] (bf16; unused for fp8 caches)
  const uint16_t* v;
  const uint8_t* k8;     // fp8 caches [batch, T_kv, G, d] e4m3 (NULL for bf16 caches)
  const uint8_t* v8;
  const float* k_scale;  // fp8 caches: [batch, T_kv, G] power-of-two row scales
  const float* v_scale;
  const int32_t* ublk;   // [batch * G][ucap]
  const uint32_t* umask; // [batch * G][ucap]
  const int* ucount;     // [batch * G]
  int ucap;
  float* part;
  int batch, n_new, t0, T_kv, Hq, G, d, B, splits;
  int* status;
  int stall_cta;         // failure-detection test hook: this CTA issues no loads (-1: none)
};
bool decode_attend_tc_supported(int Hq, int G, int d, int B, int n_new, int Kb);
// splits per (sequence, group) unit: one wave of the variant's resident CTAs (f8: FP8 caches);
// the bf16 variant's count is the larger and sizes the workspace
int decode_attend_splits(int units, int n_new, int Kb, int B, bool f8);
size_t decode_part_bytes(int units, int splits);
cudaError_t launch_decode_union(const int32_t* sel, int batch, int n_new, int G, int Kb, int32_t* ublk,
                                uint32_t* umask, int* ucount, int ucap, int* status, cudaStream_t s);
cudaError_t launch_decode_attend_tc(const DecodeAttendArgs& a, cudaStream_t s);

// FP8 KV storage: rows (b, t, g) of src [batch, n_t, G, 128] bf16 -> dst8 [batch, T, G, 128] e4m3
// codes and dscale [batch, T, G] power-of-two scales at positions t0 + t.
cudaError_t launch_quantize_fp8(const uint16_t* src, uint8_t* dst8, float* dscale, int batch, int n_t, int G, int T,
                                int t0, cudaStream_t s);

// Backward through a fixed selection (d in {64, 128}, B in {4, 8, 16}, Hq/G <= 16). dq, dgate
// [batch, T, Hq, d], dk, dv [batch, T, G, d] fp32; lse, dsum [batch, T, Hq]; the reverse index:
// rcount [batch * G][nblkc], ccount [batch * G][nchunk][nblkc] (rows of each chunk of rchunk rows
// that select each block, then their prefixes), roff [batch * G][nblkc + 1],
// rlist [batch * G][T * Kb].
struct BackwardArgs {
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  const uint16_t* gate;
  const uint16_t* dy;
  const int32_t* sel;
  float* dq;
  float* dk;
  float* dv;
  float* dgate;
  float* lse;
  float* dsum;
  float* dov;  // dy * sigmoid(gate) [batch, T, Hq, d] fp32, written by the row-centric pass
  int* rcount;
  int* ccount;
  int* roff;
  int* rlist;
  int batch, T, Hq, G, d, B, Kb, nblkc, rchunk, nchunk;
  int* status;
};
bool backward_supported(int Hq, int G, int d, int B);
cudaError_t launch_backward(const BackwardArgs& a, cudaStream_t s);

}  // namespace sgqa
