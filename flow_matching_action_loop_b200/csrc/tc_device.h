// Device helpers shared by the tensor-core kernels (tc_kernels.cu, persistent.cu): status
// latching, number-format packing, GeLU, and the warp-level copy / matrix-multiply wrappers
// written from the PTX ISA.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <math.h>

#include "sm100.h"
#include "tc_kernels.h"

namespace fr {
namespace tc {

using fr::sm100::smem_u32;

// Checked builds: an index at or past its buffer's extent latches the bounds bit and, for the first
// such index, the site's where-code and the index (low 32 bits) in the status word; the access is
// skipped.  The
// product build compiles every check to true.
__device__ __forceinline__ bool in_bounds(unsigned* status, uint64_t idx, uint64_t extent, uint32_t where) {
#ifdef FR_DEVICE_CHECKS
  if (idx < extent) return true;
  if (status && !(atomicOr(status, ST_BOUNDS_BIT) & ST_BOUNDS_BIT)) {   // the first failing check reports
    atomicExch(status + 1, where);
    atomicExch(status + 2, static_cast<unsigned>(idx));
  }
  return false;
#else
  (void)status;
  (void)idx;
  (void)extent;
  (void)where;
  return true;
#endif
}

__device__ __forceinline__ void report_timeout(unsigned* status, uint32_t where) {
  if (status) {
    atomicOr(status, ST_TIMEOUT_BIT);
    atomicExch(status + 1, where);
    atomicExch(status + 2, blockIdx.x | (blockIdx.y << 8) | (blockIdx.z << 20));
  }
}

// GeLU in its tanh form, 0.5·g·(1 + tanh z) with z = sqrt(2/pi)·(g + 0.044715·g³), evaluated as
// g·σ(2z) = g / (1 + e^{-2z}) (the identity 1 + tanh z = 2 / (1 + e^{-2z})): one exponential and one
// fast division instead of a full tanh. The exponent is capped at 80 so the denominator stays far
// below the range where the fast division returns 0 for a finite quotient; there the result is
// already below 1e-33·|g|.
__device__ __forceinline__ float gelu_tanh(float g) {
  const float c0 = 0.7978845608028654f;   // sqrt(2/pi)
  const float t = fminf(-2.f * c0 * (g + 0.044715f * g * g * g), 80.f);
  return __fdividef(g, 1.f + __expf(t));
}

// 2^x by the multi-function unit's approximation (relative error about 2^-22, subnormal results
// flushed to zero, 2^-inf = 0); softmax weights are rounded to bf16 right after.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// two e4m3 codes (saturating, round to nearest even) in one conversion: a in the low byte
__device__ __forceinline__ uint32_t pack_e4m3x2(float a, float b) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  return pack_e4m3x2(a, b) | (pack_e4m3x2(c, d) << 16);
}


constexpr int ATT_PAD = 8;        // bf16 elements of row padding (16 bytes) against bank conflicts

__device__ __forceinline__ void cp_async16(void* sdst, const void* gsrc, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(sdst)), "l"(gsrc), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2_t(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}
__device__ __forceinline__ void mma16816(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}


}  // namespace tc
}  // namespace fr
