// Shared device helpers for the spattn kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace spattn {

// Device error word codes (workspace control block, word 0).
enum : int { DEV_OK = 0, DEV_BAD_INDEX = 1, DEV_TIMEOUT = 2 };

// Control block layout inside the workspace (int32 words).
enum : int {
  CTRL_ERROR = 0,      // first device error code seen (atomicCAS from 0)
  CTRL_ERROR_AUX = 1,  // where it happened (kernel specific)
  CTRL_WORK = 2,       // persistent attention: next work ticket
  CTRL_DONE = 3,       // persistent attention: CTAs retired (the last one resets both)
  CTRL_NNZ = 4,        // total kept blocks of the last route
  CTRL_WORDS = 64
};

__device__ __forceinline__ void flag_error(int* ctrl, int code, int aux) {
  if (atomicCAS(ctrl + CTRL_ERROR, 0, code) == 0) ctrl[CTRL_ERROR_AUX] = aux;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- Ampere-style async copies (16 B per thread) ----
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

// ---- warp-level MMA (legacy tensor path, bf16 m16n8k16, fp32 accumulate) ----
__device__ __forceinline__ void ldmatrix_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                            uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                                  uint32_t& r3, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float* c, const uint32_t* a, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Swizzled byte offset of 16-byte chunk `c` of row `r` in a tile whose rows
// are `row_bytes` long (multiple of 128): chunk index XOR (row mod 8), so that
// eight consecutive rows read through ldmatrix hit eight different banks.
__device__ __forceinline__ uint32_t swz(int r, int c, int row_bytes) {
  return r * row_bytes + ((c ^ (r & 7)) << 4);
}

}  // namespace spattn
