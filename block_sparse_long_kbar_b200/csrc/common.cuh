// Shared device helpers of libsgqa (sm_100a): bf16 bit handling, the device status word,
// cp.async / ldmatrix / mma.sync wrappers, and the order-preserving float key.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "../../include/sgqa.h"

namespace sgqa {

constexpr int kStatusBytes = 256;

// Device status word (first int of the workspace). First error wins; sticky until reset.
__device__ __forceinline__ void report(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// Debug bounds checks. The library built with -DSGQA_CHECKS (libsgqa_checks.so) tests the
// indices and coordinates its kernels compute from data (selections, union lists, permutations,
// cache positions) against their buffers before use: a failed check records
// SGQA_ERR_DEVICE_CHECK and the access is skipped, so a logic error shows as a status instead of
// a fault. Without the flag every check compiles to `true`.
__device__ __forceinline__ bool check_or_report(bool ok, int* status) {
  if (!ok) report(status, SGQA_ERR_DEVICE_CHECK);
  return ok;
}
#ifdef SGQA_CHECKS
#define SGQA_CHECK(cond, status) (::sgqa::check_or_report((cond), (status)))
#else
#define SGQA_CHECK(cond, status) (true)
#endif

__device__ __forceinline__ float bf16_lo(uint32_t packed) { return __uint_as_float(packed << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t packed) { return __uint_as_float(packed & 0xFFFF0000u); }
__device__ __forceinline__ float bf16_to_f32(uint16_t u) { return __uint_as_float((uint32_t)u << 16); }

// fp32 -> bf16 round-to-nearest-even (finite inputs), as a bit pattern.
__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// 2^x with the hardware's approximate base-2 exponential (relative error ~2^-22, subnormal
// results flushed to zero); used for attention probabilities, which are rounded to bf16 next.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// Gate of the Gated-GQA epilogue, sigmoid(x) = 1 / (1 + 2^(-x log2 e)), from the hardware
// exp2 approximation and a fast divide; both errors are far below the bf16 rounding of the
// output it multiplies. Saturates to 0 (2^.. = inf) and 1 (2^.. = 0) at the ends.
__device__ __forceinline__ float sigmoid_fast(float x) {
  return __fdividef(1.f, 1.f + ex2_approx(-1.4426950408889634f * x));
}

// Order-preserving map of an fp32 score to uint32 (larger score -> larger key). -0 is first
// folded into +0 so that equal scores give equal keys.
__device__ __forceinline__ uint32_t score_key(float s) {
  s = s + 0.0f;
  const uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---- async copies -----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
// Round a dynamic shared-memory base up to A bytes by pointer arithmetic on the shared array
// itself, so pointers derived from it stay in the shared state space (ld/st/atom.shared rather
// than generic accesses).
template <int A>
__device__ __forceinline__ uint8_t* smem_align(uint8_t* base) {
  return base + ((A - (smem_u32(base) & (A - 1))) & (A - 1));
}
// 16-byte global->shared copy; src_bytes = 0 zero-fills the destination without reading.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

// ---- warp-level tensor core ops (m16n8k16, bf16 in, fp32 accumulate) ----------------------------
__device__ __forceinline__ void ldmatrix_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__host__ __device__ constexpr inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace sgqa
