// undo.cuh -- undoing a pass's in-place writes from its undo log.
//
// The m.163.com article on SDM (section 八, the memory-efficiency paragraph) trains with the
// state updated in place and the updates undone during backpropagation, which keeps one
// state plus the rows each token overwrote (O(N d + T W d)) instead of a state per chunk.  A
// logged pass (sdm_scan_forward_logged) stores, for write j of token row r, the row as that
// write found it.  Replaying the log from the last token to the first puts every written row
// back; the row left in the end is the one logged by the slot's first write in the pass, so
// the undo restores exactly those entries, in parallel:
//   1. first[(b, h, slot)] = the smallest token that wrote the slot (atomicMin);
//   2. every write whose token is its slot's first copies its log entry into M.
// Within a token the write slots are distinct, so each written slot has exactly one first
// write and the result does not depend on the order of the copies.
#pragma once

#include "common.cuh"

namespace sdm {

__global__ void __launch_bounds__(256) undo_first_kernel(const int32_t* __restrict__ sel_w,
                                                         long long n_writes, int T, int H,
                                                         int W, int N,
                                                         uint32_t* __restrict__ first) {
  // wait for the kernel ahead in the stream (programmatic launch), then let the next one in
  grid_dependency_wait();
  grid_launch_dependents();
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n_writes;
       e += stride) {
    const int slot = sel_w[e];
    if (static_cast<unsigned>(slot) >= static_cast<unsigned>(N)) {
      record_status(STATUS_BAD_INDEX);
      continue;
    }
    const long long r = e / W;  // token row (b * T + t) * H + h
    const int h = static_cast<int>(r % H);
    const long long bt = r / H;
    const int t = static_cast<int>(bt % T);
    const long long b = bt / T;
    atomicMin(first + ((size_t)b * H + h) * N + slot, static_cast<uint32_t>(t));
  }
}

// One warp per token row: the row's writes that are their slot's first copy the logged row
// back into M (lanes over the row's float4s).
__global__ void __launch_bounds__(256) undo_restore_kernel(float* __restrict__ M,
                                                           const int32_t* __restrict__ sel_w,
                                                           const float* __restrict__ wlog,
                                                           long long rows, int T, int H, int W,
                                                           int N, int d_v,
                                                           const uint32_t* __restrict__ first) {
  // wait for the kernel ahead in the stream (programmatic launch), then let the next one in
  grid_dependency_wait();
  grid_launch_dependents();
  const int lane = threadIdx.x & 31;
  const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
  const int d4 = d_v / 4;
  for (long long r = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows;
       r += nw) {
    const int h = static_cast<int>(r % H);
    const long long bt = r / H;
    const int t = static_cast<int>(bt % T);
    const long long b = bt / T;
    const size_t base = ((size_t)b * H + h) * N;
    for (int j0 = 0; j0 < W; j0 += 32) {
      const int j = j0 + lane;
      int slot = -1;
      bool mine = false;
      if (j < W) {
        slot = sel_w[r * W + j];
        mine = static_cast<unsigned>(slot) < static_cast<unsigned>(N) &&
               first[base + slot] == static_cast<uint32_t>(t);
      }
      unsigned todo = __ballot_sync(FULL_MASK, mine);
      while (todo) {
        const int src = __ffs(todo) - 1;
        todo &= todo - 1;
        const int s = __shfl_sync(FULL_MASK, slot, src);
        const float4* from = reinterpret_cast<const float4*>(wlog + ((size_t)r * W + j0 + src) * d_v);
        float4* to = reinterpret_cast<float4*>(M + (base + s) * d_v);
        for (int c = lane; c < d4; c += 32) to[c] = __ldcs(from + c);
      }
    }
  }
}

}  // namespace sdm
