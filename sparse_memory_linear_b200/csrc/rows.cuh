// rows.cuh -- low-precision copies of state rows (state checkpoints) and back.
//
// The m.163.com article on SDM (section 八, the memory-efficiency paragraph) stores the state
// checkpoints of long-context fine-tuning as fp8 or int4, and reports no loss from either.
// A row of d_v fp32 values becomes
//   bf16: d_v codes, each the value rounded to nearest-even bf16 (no scale);
//   E4M3: d_v codes and one fp32 scale s = amax / 448: the OCP FP8 E4M3 value nearest to
//         q = x * (1 / s) (ties to even, saturating; a zero result is the code of +0);
//   int4: d_v / 2 bytes of 4-bit two's-complement codes (element 2i in the low nibble) and
//         one fp32 scale s = amax / 7: q rounded to nearest-even, clamped to [-7, 7];
// amax being the row's largest |x|.  s, 1 / s, q and code * s are single fp32 operations
// rounded to nearest (IEEE division for s and 1 / s, once per row); a scale below the
// smallest normal fp32 is stored as 0 with all-zero codes, which keeps 1 / s finite.  Both
// kernels stream: each row is read and written once, one warp per row, 16-byte loads.
#pragma once

#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"

namespace sdm {

constexpr int ROWS_FMT_BF16 = 1;
constexpr int ROWS_FMT_E4M3 = 2;
constexpr int ROWS_FMT_INT4 = 3;
constexpr int ROWS_MAX_Q = 4;  // float4 per lane: d_v <= 512

__device__ __forceinline__ float abs_max4(float4 v) {
  return fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
}

__device__ __forceinline__ uint32_t e4m3_code(float q) {
  uint32_t c = __nv_cvt_float_to_fp8(q, __NV_SATFINITE, __NV_E4M3);
  return (c & 0x7fu) == 0u ? 0u : c;  // zero is always +0
}

__device__ __forceinline__ uint32_t int4_code(float q) {
  float k = rintf(q);
  k = fminf(fmaxf(k, -7.0f), 7.0f);
  return static_cast<uint32_t>(static_cast<int>(k)) & 0xfu;
}

__device__ __forceinline__ float e4m3_value(uint32_t c) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(c), __NV_E4M3);
  return __half2float(__half(h));  // both conversions are exact
}

__device__ __forceinline__ float int4_value(uint32_t nib) {
  return static_cast<float>(static_cast<int>(nib << 28) >> 28);
}

// M [rows, d_v] fp32 -> codes (+ scales).
template <int FMT>
__global__ void __launch_bounds__(256) rows_pack_kernel(const float* __restrict__ M,
                                                        long long rows, int d_v,
                                                        void* __restrict__ codes,
                                                        float* __restrict__ scales) {
  // wait for the kernel ahead in the stream (programmatic launch), then let the next one in
  grid_dependency_wait();
  grid_launch_dependents();
  const int lane = threadIdx.x & 31;
  const long long wid = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
  const int d4 = d_v / 4;
  for (long long r = wid; r < rows; r += nw) {
    const float4* src = reinterpret_cast<const float4*>(M + r * d_v);
    float4 x[ROWS_MAX_Q];
    float amax = 0.0f;
#pragma unroll
    for (int k = 0; k < ROWS_MAX_Q; ++k) {
      const int c = lane + 32 * k;
      x[k] = c < d4 ? __ldcs(src + c) : make_float4(0.f, 0.f, 0.f, 0.f);
      amax = fmaxf(amax, abs_max4(x[k]));
    }
    if constexpr (FMT == ROWS_FMT_BF16) {
      uint2* dst = reinterpret_cast<uint2*>(codes) + r * d4;
#pragma unroll
      for (int k = 0; k < ROWS_MAX_Q; ++k) {
        const int c = lane + 32 * k;
        if (c >= d4) continue;
        const __nv_bfloat162 lo = __floats2bfloat162_rn(x[k].x, x[k].y);
        const __nv_bfloat162 hi = __floats2bfloat162_rn(x[k].z, x[k].w);
        __stcs(dst + c, make_uint2(*reinterpret_cast<const uint32_t*>(&lo),
                                   *reinterpret_cast<const uint32_t*>(&hi)));
      }
    } else {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      const float s0 = amax / (FMT == ROWS_FMT_E4M3 ? 448.0f : 7.0f);
      const float s = s0 >= 1.17549435e-38f ? s0 : 0.0f;  // 2^-126, the smallest normal
      const float inv = s != 0.0f ? 1.0f / s : 0.0f;
      if (lane == 0) scales[r] = s;
#pragma unroll
      for (int k = 0; k < ROWS_MAX_Q; ++k) {
        const int c = lane + 32 * k;
        if (c >= d4) continue;
        // inv = 0 for a zero row: every q is +-0 and codes to 0
        const float q[4] = {__fmul_rn(x[k].x, inv), __fmul_rn(x[k].y, inv),
                            __fmul_rn(x[k].z, inv), __fmul_rn(x[k].w, inv)};
        if constexpr (FMT == ROWS_FMT_E4M3) {
          const uint32_t w = e4m3_code(q[0]) | (e4m3_code(q[1]) << 8) |
                             (e4m3_code(q[2]) << 16) | (e4m3_code(q[3]) << 24);
          __stcs(reinterpret_cast<unsigned int*>(codes) + r * d4 + c, w);
        } else {
          const uint32_t w = int4_code(q[0]) | (int4_code(q[1]) << 4) | (int4_code(q[2]) << 8) |
                             (int4_code(q[3]) << 12);
          reinterpret_cast<uint16_t*>(codes)[r * d4 + c] = static_cast<uint16_t>(w);
        }
      }
    }
  }
}

// codes (+ scales) -> M [rows, d_v] fp32.
template <int FMT>
__global__ void __launch_bounds__(256) rows_unpack_kernel(const void* __restrict__ codes,
                                                          const float* __restrict__ scales,
                                                          long long rows, int d_v,
                                                          float* __restrict__ M) {
  // wait for the kernel ahead in the stream (programmatic launch), then let the next one in
  grid_dependency_wait();
  grid_launch_dependents();
  const int lane = threadIdx.x & 31;
  const long long wid = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
  const int d4 = d_v / 4;
  for (long long r = wid; r < rows; r += nw) {
    float4* dst = reinterpret_cast<float4*>(M + r * d_v);
    const float s = FMT == ROWS_FMT_BF16 ? 1.0f : __ldg(scales + r);
#pragma unroll
    for (int k = 0; k < ROWS_MAX_Q; ++k) {
      const int c = lane + 32 * k;
      if (c >= d4) continue;
      float4 v;
      if constexpr (FMT == ROWS_FMT_BF16) {
        const uint2 w = __ldcs(reinterpret_cast<const uint2*>(codes) + r * d4 + c);
        v = make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xffff0000u),
                        __uint_as_float(w.y << 16), __uint_as_float(w.y & 0xffff0000u));
      } else if constexpr (FMT == ROWS_FMT_E4M3) {
        const uint32_t w = __ldcs(reinterpret_cast<const unsigned int*>(codes) + r * d4 + c);
        v = make_float4(e4m3_value(w & 0xffu) * s, e4m3_value((w >> 8) & 0xffu) * s,
                        e4m3_value((w >> 16) & 0xffu) * s, e4m3_value(w >> 24) * s);
      } else {
        const uint32_t w = reinterpret_cast<const uint16_t*>(codes)[r * d4 + c];
        v = make_float4(int4_value(w & 0xfu) * s, int4_value((w >> 4) & 0xfu) * s,
                        int4_value((w >> 8) & 0xfu) * s, int4_value((w >> 12) & 0xfu) * s);
      }
      dst[c] = v;
    }
  }
}

}  // namespace sdm
