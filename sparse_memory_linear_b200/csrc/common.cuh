// common.cuh -- device helpers shared by the SDM kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sdm.h"

namespace sdm {

constexpr unsigned FULL_MASK = 0xffffffffu;
constexpr int KMAX = 128;   // largest W or R
constexpr int SMAX = 4096;  // largest half length

// Status bits recorded by kernels in the per-device status word.
constexpr unsigned STATUS_BAD_INDEX = 1u;
constexpr unsigned STATUS_TIMEOUT = 2u;

// The per-device status word (one instance per device that loads the library).
__device__ unsigned int g_status;

__device__ __forceinline__ void record_status(unsigned bits) { atomicOr(&g_status, bits); }

// Order-preserving 32-bit key of an fp32 score: a larger score has a larger key, and
// -0 and +0 share one key.
__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7fffffffu) == 0u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_score(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  return __uint_as_float(u);
}

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

__device__ __forceinline__ float load_in(const void* p, size_t i, bool bf16) {
  return bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i])
              : reinterpret_cast<const float*>(p)[i];
}

// Eight consecutive inputs starting at element i (i a multiple of 8, 16-byte aligned).
__device__ __forceinline__ void load8_in(const void* p, size_t i, bool bf16, float out[8]) {
  if (bf16) {
    uint4 raw = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p) + i);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float2 f = __bfloat1622float2(h[j]);
      out[2 * j] = f.x;
      out[2 * j + 1] = f.y;
    }
  } else {
    const float4* q = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p) + i);
    float4 a = q[0], b = q[1];
    out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
    out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
  }
}

__device__ __forceinline__ float gate_act(float g, int act) {
  if (act == SDM_GATE_SILU) return g / (1.0f + expf(-g));
  if (act == SDM_GATE_SIGMOID) return 1.0f / (1.0f + expf(-g));
  return g;
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem) : "memory");
}

// Programmatic dependent launch: a grid launched with programmatic stream serialisation
// can start before the grid ahead of it in the stream has finished.  wait blocks until that
// grid has completed and its memory is visible (a no-op without the launch attribute);
// launch_dependents lets the next grid be scheduled.
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" :::);
}

__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

}  // namespace sdm
