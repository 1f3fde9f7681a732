// Gated SWA selection: the blocks a sliding window of keys overlaps, in the selection format the
// attention kernels read (ascending block ids, -1 padded).
//
// Step 5 Preview pages (mo.ai.kr, "Step 5 Preview agentic work design", section "model
// structure and training stability"; ai.info, "StepFun illustrates the 92-block architecture of
// Step 5 Preview", section "Why StepFun chose 92 transformer blocks"): three efficient layers of
// Gated Sliding Window Attention alternate with every Sparse GQA full-context layer. The pages
// give no window size; it is a parameter here. A query at t attends to the keys t - window < u <= t,
// which lie in the blocks floor(max(0, t - window + 1) / B) .. floor(t / B); the attention kernel
// masks the tokens of the first block that fall before the window.
#include "common.cuh"
#include "kernels.h"

namespace sgqa {
namespace {

__global__ void __launch_bounds__(256) window_select_kernel(int32_t* __restrict__ sel, int sel_T, int sel_t0, int batch,
                                                            int G, int Kb, int B, int window, int t_begin, int t_end) {
  const long n_rows = (long)batch * (t_end - t_begin) * G;
  const long total = n_rows * Kb;
  for (long e = (long)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (long)gridDim.x * blockDim.x) {
    const int i = (int)(e % Kb);
    const long row = e / Kb;
    const int g = (int)(row % G);
    const long bt = row / G;
    const int t = t_begin + (int)(bt % (t_end - t_begin));
    const int b = (int)(bt / (t_end - t_begin));
    const int lo = t - window + 1 > 0 ? t - window + 1 : 0;
    const int first = lo / B, c = t / B;
    sel[(((long)b * sel_T + (t - sel_t0)) * G + g) * (long)Kb + i] = first + i <= c ? first + i : -1;
  }
}

}  // namespace

cudaError_t launch_window_select(int32_t* sel, int sel_T, int sel_t0, int batch, int G, int Kb, int B, int window,
                                 int t_begin, int t_end, cudaStream_t s) {
  const long total = (long)batch * (t_end - t_begin) * G * Kb;
  if (total <= 0) return cudaSuccess;
  long blocks = (total + 255) / 256;
  if (blocks > 148L * 64) blocks = 148L * 64;
  window_select_kernel<<<(unsigned)blocks, 256, 0, s>>>(sel, sel_T, sel_t0, batch, G, Kb, B, window, t_begin, t_end);
  return cudaGetLastError();
}

}  // namespace sgqa
