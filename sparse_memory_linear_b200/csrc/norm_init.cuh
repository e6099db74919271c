// norm_init.cuh -- step 4 (RMSNorm + output gate) and the M0 broadcast of the SDM pass.
#pragma once

#include "common.cuh"

namespace sdm {

// Step 4 ["Sparse Delta Memory: Scaling the State of Linear RNNs through Sparsity",
// paper.rainbus.top summary, method step 4; ai-paper-analysis.pages.dev SDM write-up,
// 步骤 4]: o = y * rsqrt(mean(y^2) + eps) * gamma * act(g), one warp per row of d_v.
__global__ void __launch_bounds__(256) norm_gate_kernel(const float* __restrict__ y,
                                                        const void* __restrict__ gate,
                                                        int gate_bf16,
                                                        const float* __restrict__ gamma,
                                                        float eps, int act, long long rows,
                                                        int d_v, float* o) {
  // wait for the kernel ahead in the stream (programmatic launch), then let the next one in
  grid_dependency_wait();
  grid_launch_dependents();
  const int lane = threadIdx.x & 31;
  const long long wid = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
  const int d4 = d_v / 4;
  for (long long r = wid; r < rows; r += nw) {
    const float4* yr = reinterpret_cast<const float4*>(y + r * d_v);
    float ss = 0.0f;
    for (int c = lane; c < d4; c += 32) {
      const float4 t = yr[c];
      ss = fmaf(t.x, t.x, ss);
      ss = fmaf(t.y, t.y, ss);
      ss = fmaf(t.z, t.z, ss);
      ss = fmaf(t.w, t.w, ss);
    }
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) ss += __shfl_xor_sync(FULL_MASK, ss, s);
    const float inv = rsqrtf(ss / static_cast<float>(d_v) + eps);
    for (int c = lane; c < d4; c += 32) {
      const float4 t = yr[c];
      float f[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = 4 * c + e;
        const float gm = gamma ? gamma[col] : 1.0f;
        const float gt = gate ? gate_act(load_in(gate, (size_t)r * d_v + col, gate_bf16 != 0), act)
                              : 1.0f;
        f[e] = f[e] * inv * gm * gt;
      }
      reinterpret_cast<float4*>(o + r * d_v)[c] = make_float4(f[0], f[1], f[2], f[3]);
    }
  }
}

// Learnable initial memory [ai-paper-analysis.pages.dev SDM write-up, learned initial
// state section]: M[b, h] = M0[h] for every sequence b.  Grid-stride float4 copy.
__global__ void __launch_bounds__(256) state_init_kernel(const float4* __restrict__ M0,
                                                         float4* __restrict__ M, int B, int H,
                                                         long long per_head4) {
  // wait for the kernel ahead in the stream (programmatic launch), then let the next one in
  grid_dependency_wait();
  grid_launch_dependents();
  const long long total = (long long)B * H * per_head4;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long bh = i / per_head4;
    const long long w = i - bh * per_head4;
    const int h = static_cast<int>(bh % H);
    M[i] = __ldg(M0 + (long long)h * per_head4 + w);
  }
}

}  // namespace sdm
