// select_group.cuh -- top-K selection by a group of warps, laid out for latency (one token's
// selection on the critical path of a decode step) rather than for throughput.
//
// Method: "Sparse Delta Memory: Scaling the State of Linear RNNs through Sparsity"
// (paper.rainbus.top summary), method step 1; ai-paper-analysis.pages.dev SDM write-up,
// 步骤 1.  The result is the one the warp-per-row paths of select.cuh and select_fast.cuh
// give: the K largest keys, equal keys in ascending index order, listed in that order.
//
// A group of NT threads holds NK keys per thread (0 = no key; every real key is >= 1):
//   1. cut: shared-memory histograms of 256 bins over the key range [lo, hi] locate the bin
//      that holds the K-th largest key; the bin's lower edge is a cut with at least K keys at
//      or above it.  A bin still holding too many keys is split again (at most 4 levels for
//      32-bit keys, 2 for 16-bit keys);
//   2. the keys at or above the cut are appended to a shared list as composites that order
//      exactly as the selection order (key, then the inverted index);
//   3. each listed composite's rank is the number of listed composites above it: ranks
//      below K place the composite at its final position.
// Every step is a few shared-memory round trips apart from one named barrier, instead of
// the dozens of dependent shuffle stages of a sorting network.
#pragma once

#include "common.cuh"

namespace sdm {

// Named barrier `id` (1..7) over nthreads threads.  The id reaches the instruction as a
// literal, so the compiler reserves only the barriers in use (a register id reserves all 16
// for the CTA, which can cost resident CTAs per SM).
__device__ __forceinline__ void group_bar(int id, int nthreads) {
  switch (id) {
    case 1: asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory"); break;
    case 2: asm volatile("bar.sync 2, %0;" ::"r"(nthreads) : "memory"); break;
    case 3: asm volatile("bar.sync 3, %0;" ::"r"(nthreads) : "memory"); break;
    case 4: asm volatile("bar.sync 4, %0;" ::"r"(nthreads) : "memory"); break;
    case 5: asm volatile("bar.sync 5, %0;" ::"r"(nthreads) : "memory"); break;
    case 6: asm volatile("bar.sync 6, %0;" ::"r"(nthreads) : "memory"); break;
    default: asm volatile("bar.sync 7, %0;" ::"r"(nthreads) : "memory"); break;
  }
}

// Control words of one group, in shared memory.
struct GroupCtl {
  uint32_t wmax[4];  // per-warp maximum key
  uint32_t wmin[4];  // per-warp bracket key (candidate groups: per-warp softmax sums)
  uint32_t bin, run, cnt_bin;
  uint32_t count;    // list append counter, zero before the group starts
  uint32_t kth;      // key of the K-th ranked composite (set by the caller's emit)
};

// Group-wide bracket [lo, hi]: hi is the largest key, lo the smallest of the warps' bracket
// keys (at least K keys are >= lo by construction of the caller's bracket keys).  One
// barrier.
template <int NT>
__device__ __forceinline__ void group_bracket(uint32_t vmax, uint32_t vlo, GroupCtl* ctl,
                                              int gt, int bar_id, uint32_t& lo, uint32_t& hi) {
  constexpr int NW = NT / 32;
  vmax = __reduce_max_sync(FULL_MASK, vmax);
  vlo = __reduce_min_sync(FULL_MASK, vlo);
  if ((gt & 31) == 0) {
    ctl->wmax[gt >> 5] = vmax;
    ctl->wmin[gt >> 5] = vlo;
  }
  group_bar(bar_id, NT);
  hi = ctl->wmax[0];
  lo = ctl->wmin[0];
#pragma unroll
  for (int w = 1; w < NW; ++w) {
    hi = max(hi, ctl->wmax[w]);
    lo = min(lo, ctl->wmin[w]);
  }
  lo = max(lo, 1u);
}

// Outcome of step 1: keys >= cut are the n survivors.
struct CutResult {
  uint32_t cut;
  int n;
};

// Step 1: a cut with need <= n, and n <= cap unless a bin of width one holds more.  Entry:
// at least `need` keys are >= lo, none is > hi, `hist` (256 words) is zero; it is zero again
// on return.
template <int NK, int NT>
__device__ __forceinline__ CutResult group_cut(const uint32_t (&key)[NK], uint32_t lo,
                                               uint32_t hi, int need, int cap, uint32_t* hist,
                                               GroupCtl* ctl, int gt, int bar_id) {
  int above = 0;  // keys > hi
  for (;;) {
    const uint32_t range = hi - lo;
    const int sh = range >= 256u ? 24 - __clz(static_cast<int>(range)) : 0;
#pragma unroll
    for (int i = 0; i < NK; ++i) {
      const uint32_t k = key[i];
      if (k >= lo && k <= hi) atomicAdd(&hist[(k - lo) >> sh], 1u);
    }
    group_bar(bar_id, NT);
    if (gt < 32) {
      // lane l scans bins 255 - 8l down to 248 - 8l
      uint4* h4 = reinterpret_cast<uint4*>(hist);
      const uint4 hh = h4[63 - 2 * gt], hl = h4[62 - 2 * gt];
      const uint32_t c[8] = {hh.w, hh.z, hh.y, hh.x, hl.w, hl.z, hl.y, hl.x};
      uint32_t pre[8];  // keys in this lane's bins above bin i
      uint32_t local = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        pre[i] = local;
        local += c[i];
      }
      uint32_t incl = local;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(FULL_MASK, incl, o);
        if (gt >= o) incl += t;
      }
      const uint32_t excl = incl - local;
      const uint32_t want = static_cast<uint32_t>(need - above);
      const bool crossing = excl < want && want <= incl;
      uint32_t run = 0, cb = 0;
      int bi = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (excl + pre[i] < want && want <= excl + pre[i] + c[i]) {
          bi = i;
          run = excl + pre[i];
          cb = c[i];
        }
      }
      h4[63 - 2 * gt] = make_uint4(0u, 0u, 0u, 0u);
      h4[62 - 2 * gt] = make_uint4(0u, 0u, 0u, 0u);
      if (crossing) {
        ctl->bin = static_cast<uint32_t>(255 - 8 * gt - bi);
        ctl->run = run;
        ctl->cnt_bin = cb;
      }
      // fewer than `want` keys in range can only come from inputs outside the contract (NaN
      // or infinite scores): take the bottom bin with every key in range, so the range still
      // shrinks and the loop ends
      if (__ballot_sync(FULL_MASK, crossing) == 0u && gt == 31) {
        ctl->bin = 0u;
        ctl->run = 0u;
        ctl->cnt_bin = incl;
      }
    }
    group_bar(bar_id, NT);
    const uint32_t b = ctl->bin;
    above += static_cast<int>(ctl->run);
    const int n_ge = above + static_cast<int>(ctl->cnt_bin);
    const uint32_t nlo = lo + (b << sh);
    const uint32_t span = (1u << sh) - 1u;
    hi = (hi - nlo > span) ? nlo + span : hi;
    lo = nlo;
    if (n_ge <= cap || sh == 0) return CutResult{nlo, n_ge};
  }
}

// Steps 2 and 3: the survivors of `cr` in selection order.  emit(r, comp) is called once per
// survivor with its rank r (0 = first); ranks >= K are not part of the top K.  The
// survivors are listed in any order, then each counts the listed survivors above it.
// `list` holds every key of the group plus 4 entries; `counter` is zero on entry.
template <int NK, int NT, typename T, typename Comp, typename Emit>
__device__ __forceinline__ void group_order(const uint32_t (&key)[NK], const CutResult& cr,
                                            Comp comp, T* list, uint32_t* counter, int gt,
                                            int lane, int bar_id, Emit emit) {
  int m = 0;
#pragma unroll
  for (int i = 0; i < NK; ++i) m += key[i] >= cr.cut ? 1 : 0;
  int incl = m;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(FULL_MASK, incl, o);
    if (lane >= o) incl += t;
  }
  int base = 0;
  if (lane == 31 && incl > 0) base = static_cast<int>(atomicAdd(counter, static_cast<uint32_t>(incl)));
  base = __shfl_sync(FULL_MASK, base, 31);
  int pos = base + incl - m;
#pragma unroll
  for (int i = 0; i < NK; ++i)
    if (key[i] >= cr.cut) list[pos++] = comp(i);
  group_bar(bar_id, NT);
  // the survivors listed (cr.n of them for inputs inside the contract), padded with zeros
  // (below every composite) to a multiple of 4
  const int n = static_cast<int>(*counter);
  if (gt < 4 && (n & ~3) + gt >= n) list[(n & ~3) + gt] = T(0);
  group_bar(bar_id, NT);
  const int n4 = (n + 3) >> 2;
  for (int j = gt; j < n; j += NT) {
    const T x = list[j];
    int r0 = 0, r1 = 0;
    if constexpr (sizeof(T) == 4) {
      const uint4* l4 = reinterpret_cast<const uint4*>(list);
#pragma unroll 4
      for (int q = 0; q < n4; ++q) {
        const uint4 y = l4[q];
        r0 += (y.x > x ? 1 : 0) + (y.y > x ? 1 : 0);
        r1 += (y.z > x ? 1 : 0) + (y.w > x ? 1 : 0);
      }
    } else {
      const ulonglong2* l2 = reinterpret_cast<const ulonglong2*>(list);
#pragma unroll 4
      for (int q = 0; q < 2 * n4; q += 2) {
        const ulonglong2 y0 = l2[q], y1 = l2[q + 1];
        r0 += (y0.x > x ? 1 : 0) + (y0.y > x ? 1 : 0);
        r1 += (y1.x > x ? 1 : 0) + (y1.y > x ? 1 : 0);
      }
    }
    emit(r0 + r1, x);
  }
}

}  // namespace sdm
