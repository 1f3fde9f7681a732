// sgqa_decode_noalloc: a decode step whose scratch lives in a fixed, library-owned device array.
//
// Some callers cannot call cudaMalloc at all: a plugin loaded into a serving process whose
// allocator owns every device byte, code that must not touch the CUDA allocator while another
// component is capturing or replaying work, or an embedder with a fixed memory budget set at
// start-up. For them this entry point takes the same inputs and outputs as sgqa_decode but no
// workspace: the scratch sgqa_decode would need (device status word, per-row indexer scores,
// the selection, split-K partials) is carved out of one file-scope __device__ array of
// SGQA_NOALLOC_SCRATCH_BYTES bytes. Every GPU on which the library's code is loaded holds that
// array until the process exits.
//
// Host code cannot use the array's name as a device address (on the host it names a shadow
// variable). The first call on each device therefore asks the runtime for the array's device
// address with cudaGetSymbolAddress, with that device current, checks the result and caches it
// per device; later calls reuse the cached address. Because the first call on a device does
// that set-up, make it before any stream capture. The cached address is only valid for the
// context it was taken in: a device reset (cudaDeviceReset, or resetting the primary context)
// unloads the module and frees the array, so calls after such a reset are not supported.
//
// Every call uses the same array and the array keeps the last call's contents. The call zeroes
// the status word itself (asynchronously, on the caller's stream) and every other scratch byte
// it reads was written earlier in the same call. Calls whose work overlaps on the GPU (two
// streams, two host threads) race on the array: serialise them.
#include <mutex>

#include "common.cuh"

namespace {

__device__ __align__(256) unsigned char g_decode_scratch[SGQA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

}  // namespace

extern "C" int sgqa_decode_noalloc(const sgqa_dims* dims, int cache_len, int n_new, uint16_t* k_cache,
                                   uint16_t* v_cache, uint16_t* kidx_cache, float* kbar_cache,
                                   const uint16_t* q_new, const uint16_t* k_new, const uint16_t* v_new,
                                   const uint16_t* qidx_new, const uint16_t* kidx_new, const uint16_t* gate_new,
                                   uint16_t* out, int32_t* sel_out, void* stream) {
  const size_t need = sgqa_decode_workspace_size(dims, n_new);
  if (need == 0) return SGQA_ERR_INVALID_ARG;
  if (need > (size_t)SGQA_NOALLOC_SCRATCH_BYTES) return SGQA_ERR_WORKSPACE;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return SGQA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SGQA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return SGQA_ERR_CUDA;
      g_scratch_addr[dev] = p;
    }
    scratch = g_scratch_addr[dev];
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(scratch, 0, sizeof(int), s) != cudaSuccess) return SGQA_ERR_CUDA;
  return sgqa_decode(dims, cache_len, n_new, k_cache, v_cache, kidx_cache, kbar_cache, q_new, k_new, v_new,
                     qidx_new, kidx_new, gate_new, out, sel_out, scratch, (size_t)SGQA_NOALLOC_SCRATCH_BYTES,
                     stream);
}
