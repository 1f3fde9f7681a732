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
//   q_idx [batch, T, G, d_idx]; kbar [batch, T/B, d_idx] fp32;
//   sel rows (b, t) at sel + ((b * sel_T + (t - sel_t0)) * G + g) * Kb.
struct SelectArgs {
  const uint16_t* q_idx;
  const float* kbar;
  const uint16_t* kbar_hi;
  const uint16_t* kbar_lo;
  int32_t* sel;
  int batch, T, G, d_idx, B, Kb;
  int t_begin, t_end;
  int sel_T, sel_t0;
  int* status;
};
cudaError_t launch_select(const SelectArgs& a, cudaStream_t s);

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
cudaError_t launch_decode_select(const float* scores, int32_t* sel, int batch, int n_new, int G, int B, int Kb,
                                 int nblk, int t0, int* status, cudaStream_t s);

}  // namespace sgqa
