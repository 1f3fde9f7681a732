// Device twin of the seeded input generator defined in sgqa_inputs/__init__.py.
//
// Holds none of the Sparse GQA arithmetic: it writes the bf16 bit patterns of the synthetic
// workload tensors (q, k, v, gate_logits, q_idx, k_idx) as a pure function of
// (seed, tensor, position), using the same counter-based splitmix64 + fp64 Box-Muller
// definition as the host generator, so that workloads too large to build on the host
// (the 1M-token decode caches) can be made in device memory.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

__device__ __forceinline__ uint64_t splitmix64(uint64_t x) {
  x += 0x9E3779B97F4A7C15ull;
  uint64_t z = x;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__host__ __device__ inline uint64_t splitmix64_h(uint64_t x) {
  x += 0x9E3779B97F4A7C15ull;
  uint64_t z = x;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

inline uint64_t stream_key(uint64_t seed, uint64_t stream) {
  return splitmix64_h(splitmix64_h(seed) ^ (stream * 0xD1B54A32D192ED03ull));
}

__device__ __forceinline__ double normal_at(uint64_t key, uint64_t i) {
  uint64_t w1 = splitmix64(key + 2 * i);
  uint64_t w2 = splitmix64(key + 2 * i + 1);
  double u1 = __dmul_rn(__dadd_rn((double)(w1 >> 11), 0.5), 0x1.0p-53);
  double u2 = __dmul_rn((double)(w2 >> 11), 0x1.0p-53);
  double r = sqrt(__dmul_rn(-2.0, log(u1)));
  return __dmul_rn(r, cos(__dmul_rn(6.283185307179586, u2)));
}

__device__ __forceinline__ uint16_t to_bf16_bits(double v) {
  float f = __double2float_rn(v);
  uint32_t u = __float_as_uint(f);
  u = (u + 0x7FFFu + ((u >> 16) & 1u)) >> 16;
  return (uint16_t)u;
}

// kind: 0 q, 1 k, 2 v, 3 gate, 4 q_idx, 5 k_idx (streams 1..6); topics stream 7, r stream 8
__global__ void gen_fill_kernel(int kind, uint64_t key, uint64_t topic_key, uint64_t r_key,
                                int span, int G, int d_idx, int W, int batch, int t0, int n_t,
                                int dst_t0, int64_t batch_stride, uint16_t* __restrict__ out) {
  const int64_t total = (int64_t)batch * n_t * W;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int w = (int)(e % W);
    const int64_t bt = e / W;
    const int tt = (int)(bt % n_t);
    const int b = (int)(bt / n_t);
    const uint64_t t = (uint64_t)(t0 + tt);
    const uint64_t row = ((uint64_t)b << 32) + t;
    double v = normal_at(key, row * (uint64_t)W + (uint64_t)w);
    if (kind == 5) {  // k_idx[b,t,i] += 2 * topic[b, t // span, i]
      const uint64_t s = t / (uint64_t)span;
      v = __dadd_rn(v, 2.0 * normal_at(topic_key, ((((uint64_t)b) << 32) + s) * (uint64_t)d_idx + (uint64_t)w));
    } else if (kind == 4) {  // q_idx[b,t,g,i] += 2 * topic[b, r(b,t,g), i]
      const int g = w / d_idx, i = w % d_idx;
      const uint64_t wr = splitmix64(r_key + row * (uint64_t)G + (uint64_t)g);
      const uint64_t r = wr % (t / (uint64_t)span + 1);
      v = __dadd_rn(v, 2.0 * normal_at(topic_key, ((((uint64_t)b) << 32) + r) * (uint64_t)d_idx + (uint64_t)i));
    }
    out[(int64_t)b * batch_stride + (int64_t)(dst_t0 + tt) * W + w] = to_bf16_bits(v);
  }
}

}  // namespace

// Fills out[b, dst_t0 + i, :] (rows W wide, sequences batch_stride elements apart) with the
// values of positions t0 + i, i < n_t, of tensor `kind` of every sequence b < batch.
extern "C" int sgqa_gen_fill(int kind, uint64_t seed, int span, int G, int d_idx, int W, int batch,
                             int t0, int n_t, int dst_t0, int64_t batch_stride, void* out, void* stream) {
  if (kind < 0 || kind > 5 || W <= 0 || batch <= 0 || n_t < 0 || span <= 0) return (int)cudaErrorInvalidValue;
  if (n_t == 0) return 0;
  const uint64_t key = stream_key(seed, (uint64_t)kind + 1);
  const uint64_t topic_key = stream_key(seed, 7);
  const uint64_t r_key = stream_key(seed, 8);
  const int64_t total = (int64_t)batch * n_t * W;
  int64_t blocks = (total + 255) / 256;
  if (blocks > 148 * 64) blocks = 148 * 64;
  gen_fill_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(
      kind, key, topic_key, r_key, span, G, d_idx, W, batch, t0, n_t, dst_t0, batch_stride, (uint16_t*)out);
  return (int)cudaGetLastError();
}
