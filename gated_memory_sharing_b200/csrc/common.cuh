// Shared device helpers for the SambaY scan + GMU kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sambay {

// Per-device status word.  A kernel that detects a fault (a bounded wait that
// ran out) records the first code here; sambay_device_status reads and
// clears it.  Module-scope storage, not an allocation.
__device__ int g_status;

__device__ __forceinline__ void record_status(int code) { atomicCAS(&g_status, 0, code); }

constexpr int kStatusTimeout = 5;  // == SAMBAY_ERR_TIMEOUT

typedef __nv_bfloat16 bf16;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(bf16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float x) { return __float2bfloat16_rn(x); }

// 2^x on the special-function unit (PTX ex2.approx.ftz.f32).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// SiLU(x) = x / (1 + e^-x), the GMU gate activation and Mamba's post-conv one.
__device__ __forceinline__ float silu(float x) {
  return __fdividef(x, 1.0f + ex2_approx(-x * kLog2e));
}

// log2(x) on the special-function unit (PTX lg2.approx.f32).
__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// softplus(x) = log(1 + e^x) = max(x, 0) + log1p(y),  y = e^-|x| in (0, 1].
// log1p(y): for y < 1/16 its Taylor series y - y^2/2 + y^3/3 - y^4/4 + y^5/5
// (the first omitted term is below 2e-7 of the sum); otherwise
// log2(1 + y) * ln 2 with 1 + y >= 1.0625, where the SFU's absolute error in
// log2 is a few 1e-7 of the result.  Both are evaluated and one selected, so
// a warp whose lanes straddle 1/16 does not run the two paths one after the
// other.  For large x, y underflows towards 0 and the series returns y.
__device__ __forceinline__ float softplus(float x) {
  const float y = ex2_approx(-fabsf(x) * kLog2e);
  const float series = y * fmaf(-y, fmaf(-y, fmaf(-y, fmaf(-y, 0.2f, 0.25f), 0.33333334f), 0.5f), 1.0f);
  const float viaLog = lg2_approx(1.0f + y) * kLn2;
  return fmaxf(x, 0.0f) + (y < 0.0625f ? series : viaLog);
}

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialization may start while the kernel before it on the stream is still
// running; pdl_wait() returns once that kernel has finished and its writes are
// visible, so every global access that can depend on it comes after the wait.
// pdl_launch_dependents() lets the next such kernel start launching (its CTAs
// then sit in their own pdl_wait until this grid has finished).  Both are
// no-ops for a kernel launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// 16-byte load through L2 (no L1 allocation) of p when `pred`, else zeros.
// Written as a predicated load rather than a branch so a run of these stays
// independent and the compiler keeps them all in flight at once.
__device__ __forceinline__ float4 ldcg_or_zero(const float* p, bool pred) {
  float4 v;
  asm("{\n\t.reg .pred q;\n\t"
      "setp.ne.b32 q, %5, 0;\n\t"
      "mov.b32 %0, 0;\n\tmov.b32 %1, 0;\n\tmov.b32 %2, 0;\n\tmov.b32 %3, 0;\n\t"
      "@q ld.global.cg.v4.f32 {%0, %1, %2, %3}, [%4];\n\t}"
      : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
      : "l"(p), "r"(static_cast<int>(pred)));
  return v;
}

// Loads from shared memory by a shared-space address (ld.shared), whatever
// the compiler can prove about the generic pointer: a generic load may be
// ordered behind the thread's earlier global stores, a shared one is not.
__device__ __forceinline__ uint32_t shared_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ float4 ld_shared_f4(const void* p) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(shared_addr(p))
               : "memory");
  return v;
}
__device__ __forceinline__ float ld_shared_f32(const void* p) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(shared_addr(p)) : "memory");
  return v;
}
__device__ __forceinline__ float ld_shared_bf16(const void* p) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(shared_addr(p)) : "memory");
  return __uint_as_float(static_cast<uint32_t>(v) << 16);
}

// Pack / unpack helpers for 16-byte vector access.
union Pack16 {
  uint4 u;
  float f[4];
  bf16 h[8];
  __nv_bfloat162 h2[4];
};

}  // namespace sambay
