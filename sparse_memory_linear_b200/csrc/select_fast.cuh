// select_fast.cuh -- register-resident product-key selection for bf16 score halves of up to
// 1024 values and K <= 128 (the selection of select.cuh, same order and same result).
//
// Method: "Sparse Delta Memory: Scaling the State of Linear RNNs through Sparsity"
// (paper.rainbus.top summary), method step 1; ai-paper-analysis.pages.dev SDM write-up,
// 步骤 1.  Per half, per warp:
//   1. 16-byte loads; lane l holds elements r*256 + 8l + i as 16-bit order keys;
//   2. every lane keeps its P = ceil(K/32) largest keys; the K-th largest key T is at least
//      the smallest of the lanes' P-th largest keys (every lane has P keys at or above it),
//      and at most the largest key;
//   3. keys in that bracket are compacted to shared memory in index order; histogram levels
//      (256 bins over the bracket, then over the bin that holds T) find T, and the top K are
//      the keys > T plus the lowest-index ties;
//   4. a register bitonic sort (shuffles) orders them: (key desc, index asc).
// Candidates: the rank pairs with (r1+1)(r2+1) <= K; their K-th largest sum is at least
// both A[K-1] + B[0] and A[0] + B[K-1] (K candidate sums reach each), which brackets the same
// histogram search; equal sums at the threshold take the lowest flat slot indices.  When the
// halves' exponents span more than 15, fp32 sums can round together and the ties at the K-th
// sum are checked against all K*K pairs (repair_ties_at_kth, select.cuh).
#pragma once

#include "select.cuh"

namespace sdm {

// 16-bit order key of a bf16 score from its raw bits; -0 and +0 share one key, and every
// non-NaN value has a key >= 1.
__device__ __forceinline__ uint32_t bf16_key16(uint32_t h) {
  h &= 0xffffu;
  if ((h & 0x7fffu) == 0u) h = 0u;
  return (h & 0x8000u) ? (~h & 0xffffu) : (h | 0x8000u);
}

__device__ __forceinline__ float key16_value(uint32_t k) {
  const uint32_t h = (k & 0x8000u) ? (k & 0x7fffu) : (~k & 0xffffu);
  return __uint_as_float(h << 16);
}

__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(FULL_MASK, v, o);
    if (lane >= o) v += t;
  }
  return v;
}

// The K-th largest key of a warp's keys, by histogram levels: 256 bins of 2^sh keys over
// [lo, hi] locate the bin that holds it; the next level splits that bin, until a bin holds a
// single key value T.  Entry: at least K keys are >= lo and none is > hi; `hist` (256 words)
// is zero, and zero again on return.  for_each(f) calls f(key) on each of this lane's keys.
struct WarpKth {
  uint32_t T;  // the K-th largest key
  int ngt;     // keys > T
  int neq;     // keys == T
};

template <typename ForEach>
__device__ __forceinline__ WarpKth warp_kth_key(ForEach for_each, uint32_t lo, uint32_t hi, int K,
                                                uint32_t* hist, int lane) {
  int above = 0;
  while (true) {
    const uint32_t range = hi - lo;
    const int sh = range >= 256u ? 24 - __clz(static_cast<int>(range)) : 0;
    for_each([&](uint32_t k) {
      if (k >= lo && k <= hi) atomicAdd(&hist[(k - lo) >> sh], 1u);
    });
    __syncwarp();
    // lane l reads bins 255 - 8l down to 248 - 8l and clears them for the next level
    uint4* h4 = reinterpret_cast<uint4*>(hist);
    const uint4 hh = h4[63 - 2 * lane], hl = h4[62 - 2 * lane];
    h4[63 - 2 * lane] = make_uint4(0u, 0u, 0u, 0u);
    h4[62 - 2 * lane] = make_uint4(0u, 0u, 0u, 0u);
    const uint32_t c[8] = {hh.w, hh.z, hh.y, hh.x, hl.w, hl.z, hl.y, hl.x};
    uint32_t pre[8], local = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      pre[i] = local;
      local += c[i];
    }
    const uint32_t incl = static_cast<uint32_t>(warp_incl_scan(static_cast<int>(local), lane));
    const uint32_t excl = incl - local;
    const uint32_t want = static_cast<uint32_t>(K - above);
    uint32_t bin = 0, run = 0, cb = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (excl + pre[i] < want && want <= excl + pre[i] + c[i]) {
        bin = static_cast<uint32_t>(255 - 8 * lane - i);
        run = excl + pre[i];
        cb = c[i];
      }
    }
    const unsigned cm = __ballot_sync(FULL_MASK, excl < want && want <= incl);
    if (cm == 0u) {
      // fewer than K keys in range: only inputs outside the contract (NaN scores) get here;
      // stop with every key in range taken
      __syncwarp();
      return WarpKth{lo, above, static_cast<int>(__shfl_sync(FULL_MASK, incl, 31))};
    }
    const int cl = __ffs(cm) - 1;
    bin = __shfl_sync(FULL_MASK, bin, cl);
    above += static_cast<int>(__shfl_sync(FULL_MASK, run, cl));
    cb = __shfl_sync(FULL_MASK, cb, cl);
    const uint32_t nlo = lo + (bin << sh);
    const uint32_t span = (1u << sh) - 1u;
    hi = (hi - nlo > span) ? nlo + span : hi;
    lo = nlo;
    __syncwarp();  // the cleared bins land before the next level counts
    if (sh == 0) return WarpKth{lo, above, static_cast<int>(cb)};
  }
}

// Compare-exchange of register pairs (q, q | QS) for the stages whose stride spans whole
// registers (stride = 32 QS); QS is a constant so the array stays in registers.
template <typename V, int NPL, int QS>
__device__ __forceinline__ void bitonic_cross_regs(V (&v)[NPL], int size, int lane) {
#pragma unroll
  for (int q = 0; q < NPL; ++q) {
    if ((q & QS) == 0 && (q | QS) < NPL) {
      const int p = q * 32 + lane;
      const bool desc = (p & size) == 0;
      const V a = v[q], b = v[q | QS];
      const bool sw = desc ? (a < b) : (a > b);
      v[q] = sw ? b : a;
      v[q | QS] = sw ? a : b;
    }
  }
}

// Descending bitonic sort of 32*NPL values held NPL per lane (position q*32 + lane), NPL <=
// 4.  The stage loops stay rolled (small code); the per-lane element loops are unrolled.
template <typename V, int NPL>
__device__ __forceinline__ void bitonic_desc_reg(V (&v)[NPL], int lane) {
  static_assert(NPL == 1 || NPL == 2 || NPL == 4, "one, two or four values per lane");
  constexpr int P2 = 32 * NPL;
#pragma unroll 1
  for (int size = 2; size <= P2; size <<= 1) {
#pragma unroll 1
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      if (stride >= 32) {
        if (stride == 32) bitonic_cross_regs<V, NPL, 1>(v, size, lane);
        else bitonic_cross_regs<V, NPL, 2>(v, size, lane);
      } else {
        const bool lower = (lane & stride) == 0;
#pragma unroll
        for (int q = 0; q < NPL; ++q) {
          const int p = q * 32 + lane;
          const bool desc = (p & size) == 0;
          const V o = __shfl_xor_sync(FULL_MASK, v[q], stride);
          const bool take_max = lower == desc;
          v[q] = take_max ? (v[q] > o ? v[q] : o) : (v[q] < o ? v[q] : o);
        }
      }
    }
  }
}

// Shared scratch of one warp of the fast path (6.5 KB for halves of 1024: four warps'
// CTAs of 8 warps fit one SM).
struct FastScratch {
  uint32_t* hist;   // [256] threshold histogram, zero between uses
  uint32_t* surv;   // [max(S1, S2)] bracket survivors of one half (composites)
  uint32_t* a;      // [KMAX] first half: sorted composites key16 << 16 | (0xffff - idx)
  uint32_t* b;      // [KMAX] second half
  uint32_t* stage;  // [KMAX] unsorted winners of a half (u32)
  // candidate phase, over the survivors of the halves (no longer needed by then):
  float* pv;         // [4 * KMAX] half values and scaled indices
  uint64_t* cstage;  // [KMAX] unsorted winners of the candidates
};

__host__ __device__ inline size_t fast_surv_bytes(int S1, int S2) {
  const int smax = S1 > S2 ? S1 : S2;
  const size_t surv = (size_t)smax * 4;
  const size_t cand = 4 * (size_t)KMAX * 4 + (size_t)KMAX * 8;
  return ((surv > cand ? surv : cand) + 15) / 16 * 16;
}

__host__ __device__ inline size_t fast_scratch_bytes(int S1, int S2, int K) {
  (void)K;
  return 256 * 4 + fast_surv_bytes(S1, S2) + 2 * (size_t)KMAX * 4 + (size_t)KMAX * 4;
}

__device__ inline FastScratch carve_fast_scratch(unsigned char* p, int S1, int S2, int K) {
  FastScratch s;
  s.hist = reinterpret_cast<uint32_t*>(p);
  p += 256 * 4;
  s.surv = reinterpret_cast<uint32_t*>(p);
  s.pv = reinterpret_cast<float*>(p);
  s.cstage = reinterpret_cast<uint64_t*>(p + 4 * (size_t)KMAX * 4);
  p += fast_surv_bytes(S1, S2);
  s.a = reinterpret_cast<uint32_t*>(p);
  p += KMAX * 4;
  s.b = reinterpret_cast<uint32_t*>(p);
  p += KMAX * 4;
  s.stage = reinterpret_cast<uint32_t*>(p);
  return s;
}

// Top-K of one bf16 half of S values (S <= 256 * R8), written sorted to out[0..K).
template <int R8, int KC>
__device__ __forceinline__ void half_topk_bf16(const __nv_bfloat16* src, int S, int K, int lane,
                                               uint32_t* surv, uint32_t* stage, uint32_t* hist,
                                               uint32_t* out) {
  constexpr int P = KC / 32;  // enough per-lane leaders for any K <= KC
  const unsigned lt = lanemask_lt();
  uint32_t k[R8][8];
  const bool vec = (reinterpret_cast<uintptr_t>(src) & 15u) == 0;
  const uint16_t* raw16 = reinterpret_cast<const uint16_t*>(src);
#pragma unroll
  for (int r = 0; r < R8; ++r) {
    const int e0 = r * 256 + lane * 8;
    if (vec && e0 + 8 <= S) {
      // read once: streamed (evict-first), so that a selection running beside the slot
      // engine's scan leaves the scan's L2-resident rows in place
      const uint4 raw = __ldcs(reinterpret_cast<const uint4*>(src + e0));
      const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        k[r][2 * j] = bf16_key16(w[j]);
        k[r][2 * j + 1] = bf16_key16(w[j] >> 16);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) k[r][i] = (e0 + i < S) ? bf16_key16(raw16[e0 + i]) : 0u;
    }
  }
  // per-lane P largest keys (descending)
  uint32_t t[P];
#pragma unroll
  for (int q = 0; q < P; ++q) t[q] = 0u;
#pragma unroll
  for (int r = 0; r < R8; ++r) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      uint32_t x = k[r][i];
#pragma unroll
      for (int q = 0; q < P; ++q) {
        const uint32_t hi = max(t[q], x);
        x = min(t[q], x);
        t[q] = hi;
      }
    }
  }
  const int pe = (K + 31) / 32;  // leaders that bracket the K-th key
  uint32_t lead = t[0];
#pragma unroll
  for (int q = 1; q < P; ++q)
    if (q == pe - 1) lead = t[q];
  const uint32_t lo = max(__reduce_min_sync(FULL_MASK, lead), 1u);
  const uint32_t hi = __reduce_max_sync(FULL_MASK, t[0]);  // the largest key
  // bracket survivors, index order, as composites
  int base = 0;
#pragma unroll
  for (int r = 0; r < R8; ++r) {
    int c = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) c += k[r][i] >= lo ? 1 : 0;
    const int incl = warp_incl_scan(c, lane);
    int pos = base + incl - c;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (k[r][i] >= lo)
        surv[pos++] = (k[r][i] << 16) | (0xffffu - (uint32_t)(r * 256 + lane * 8 + i));
    }
    base += __shfl_sync(FULL_MASK, incl, 31);
  }
  __syncwarp();
  const int ns = base;
  const WarpKth kth = warp_kth_key(
      [&](auto f) {
        for (int s = lane; s < ns; s += 32) f(surv[s] >> 16);
      },
      lo, hi, K, hist, lane);
  const uint32_t T = kth.T;
  const int need = K - kth.ngt;
  int tb = 0, ob = 0;
  for (int s0 = 0; s0 < ns; s0 += 32) {
    const int s = s0 + lane;
    const uint32_t c = s < ns ? surv[s] : 0u;
    const uint32_t key = c >> 16;
    const bool tie = s < ns && key == T;
    const bool gt = s < ns && key > T;
    const unsigned tm = __ballot_sync(FULL_MASK, tie);
    const bool take = gt || (tie && tb + __popc(tm & lt) < need);
    const unsigned sm = __ballot_sync(FULL_MASK, take);
    if (take && ob + __popc(sm & lt) < K) stage[ob + __popc(sm & lt)] = c;
    ob += __popc(sm);
    tb += __popc(tm);
  }
  __syncwarp();
  constexpr int NPL = KC / 32;
  uint32_t v[NPL];
#pragma unroll
  for (int q = 0; q < NPL; ++q) {
    const int p = q * 32 + lane;
    v[q] = p < K ? stage[p] : 0u;
  }
  bitonic_desc_reg<uint32_t, NPL>(v, lane);
#pragma unroll
  for (int q = 0; q < NPL; ++q) {
    const int p = q * 32 + lane;
    if (p < K) out[p] = v[q];
  }
  __syncwarp();
}

__device__ __forceinline__ float comp16_value(uint32_t c) { return key16_value(c >> 16); }
__device__ __forceinline__ int comp16_index(uint32_t c) { return (int)(0xffffu - (c & 0xffffu)); }

// Top-K of the rank-pair candidate sums of two sorted halves A, B (composites), written as
// slot indices and softmax weights in selection order.  The candidates stay in registers;
// sums of bf16 halves leave the low bits of their fp32 patterns zero, so the threshold
// search runs on keys shifted right by the bits every candidate has clear.
template <int KC>
__device__ __forceinline__ void cand_topk_bf16(const uint32_t* A, const uint32_t* B, int K,
                                               int S2, const uint16_t* ctab, int lane,
                                               float* pv, uint64_t* stage, uint32_t* hist,
                                               int32_t* out_idx, float* out_wt) {
  constexpr int CPL = (cand_count(KC) + 31) / 32;
  const unsigned lt = lanemask_lt();
  const int C = cand_count_dev(K);
  float* av = pv;                                   // [KMAX] first-half values
  float* bv = pv + KMAX;                            // [KMAX] second-half values
  int* ai = reinterpret_cast<int*>(pv + 2 * KMAX);  // [KMAX] first-half index * S2
  int* bi = reinterpret_cast<int*>(pv + 3 * KMAX);  // [KMAX] second-half index
  for (int j = lane; j < K; j += 32) {
    av[j] = comp16_value(A[j]);
    ai[j] = comp16_index(A[j]) * S2;
    bv[j] = comp16_value(B[j]);
    bi[j] = comp16_index(B[j]);
  }
  __syncwarp();
  uint32_t ck[CPL];
  uint32_t cf[CPL];
  uint32_t orbits = 0u;
#pragma unroll
  for (int q = 0; q < CPL; ++q) {
    const int c = lane + 32 * q;
    ck[q] = 0u;  // no candidate (every real score has a key >= 1)
    cf[q] = 0u;
    if (c < C) {
      const int e = ctab[c];
      const int r1 = e >> 7, r2 = e & 127;
      const float s = __fadd_rn(av[r1], bv[r2]);
      orbits |= __float_as_uint(s) & 0x7fffffffu;
      ck[q] = score_key(s);
      cf[q] = (uint32_t)(ai[r1] + bi[r2]);
    }
  }
  // bracket of the K-th largest sum: the K sums A[i] + B[0] and the K sums A[0] + B[i] are
  // candidates, so both K-th largest bound it from below; A[0] + B[0] is the largest
  const uint32_t hi = score_key(__fadd_rn(av[0], bv[0]));
  const uint32_t lo = max(score_key(__fadd_rn(av[K - 1], bv[0])),
                          score_key(__fadd_rn(av[0], bv[K - 1])));
  orbits = __reduce_or_sync(FULL_MASK, orbits);
  const int tz = orbits ? __ffs(orbits) - 1 : 0;
  const WarpKth kth = warp_kth_key(
      [&](auto f) {
#pragma unroll
        for (int q = 0; q < CPL; ++q)
          if (ck[q] != 0u) f(ck[q] >> tz);
      },
      lo >> tz, hi >> tz, K, hist, lane);
  const uint32_t T = kth.T;  // shifted key of the K-th largest sum
  const int ngt = kth.ngt;
  const int need = K - ngt;
  const int nties = kth.neq;
  int ob = 0;
#pragma unroll
  for (int q = 0; q < CPL; ++q) {
    const uint32_t sk = ck[q] >> tz;
    const bool take = ck[q] != 0u && (sk > T || (sk == T && nties == need));
    const unsigned sm = __ballot_sync(FULL_MASK, take);
    if (take && ob + __popc(sm & lt) < K)
      stage[ob + __popc(sm & lt)] = (static_cast<uint64_t>(ck[q]) << 32) | (0xffffffffu - cf[q]);
    ob += __popc(sm);
  }
  if (nties != need) {
    // equal sums at the threshold: the lowest flat indices (the largest composites) win
    uint64_t floor_c = 0xffffffffffffffffull;
    for (int r = 0; r < need; ++r) {
      uint64_t best = 0ull;
#pragma unroll
      for (int q = 0; q < CPL; ++q) {
        const uint64_t c = (static_cast<uint64_t>(ck[q]) << 32) | (0xffffffffu - cf[q]);
        if (ck[q] != 0u && (ck[q] >> tz) == T && c < floor_c && c > best) best = c;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const uint64_t t2 = __shfl_xor_sync(FULL_MASK, best, o);
        best = t2 > best ? t2 : best;
      }
      if (lane == 0 && ob < K) stage[ob] = best;
      floor_c = best;
      ++ob;
    }
  }
  __syncwarp();
  constexpr int NPL = KC / 32;
  uint64_t v[NPL];
#pragma unroll
  for (int q = 0; q < NPL; ++q) {
    const int p = q * 32 + lane;
    v[q] = p < K ? stage[p] : 0ull;
  }
  bitonic_desc_reg<uint64_t, NPL>(v, lane);
  // ties at the K-th sum beyond the pruning: only when rounding can merge unequal sums
  if (!warp_bf16_sums_exact([&](int j) { return j < K ? av[j] : bv[j - K]; }, K, lane)) {
    uint64_t vk = 0ull;
#pragma unroll
    for (int q = 0; q < NPL; ++q)
      if (q == ((K - 1) >> 5)) vk = v[q];
    const uint32_t Tk = static_cast<uint32_t>(__shfl_sync(FULL_MASK, vk, (K - 1) & 31) >> 32);
#pragma unroll
    for (int q = 0; q < NPL; ++q)
      if (q * 32 + lane < K) stage[q * 32 + lane] = v[q];
    __syncwarp();
    const bool fixed = repair_ties_at_kth(
        [&](int r1, int r2) { return score_key(__fadd_rn(av[r1], bv[r2])); },
        [&](int r1, int r2) { return static_cast<uint32_t>(ai[r1] + bi[r2]); }, K, Tk, lane,
        [&](int r, uint32_t f) {
          stage[r] = (static_cast<uint64_t>(Tk) << 32) | (0xffffffffu - f);
        });
    if (fixed) {
#pragma unroll
      for (int q = 0; q < NPL; ++q) v[q] = q * 32 + lane < K ? stage[q * 32 + lane] : 0ull;
    }
    __syncwarp();
  }
  const float s0 = key_score(static_cast<uint32_t>(__shfl_sync(FULL_MASK, v[0], 0) >> 32));
  float e[NPL];
  float part = 0.0f;
#pragma unroll
  for (int q = 0; q < NPL; ++q) {
    const int p = q * 32 + lane;
    e[q] = p < K ? expf(key_score(static_cast<uint32_t>(v[q] >> 32)) - s0) : 0.0f;
    part += e[q];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(FULL_MASK, part, o);
  const float inv = 1.0f / part;
#pragma unroll
  for (int q = 0; q < NPL; ++q) {
    const int p = q * 32 + lane;
    if (p < K) {
      out_idx[p] = static_cast<int32_t>(0xffffffffu - static_cast<uint32_t>(v[q]));
      out_wt[p] = e[q] * inv;
    }
  }
  __syncwarp();
}

// Full selection of one bf16 score row by one warp (fast path).
template <int R8, int KC>
__device__ __forceinline__ void select_row_fast(const __nv_bfloat16* row, int S1, int S2, int K,
                                                const uint16_t* ctab, FastScratch& sc, int lane,
                                                int32_t* out_idx, float* out_wt) {
  half_topk_bf16<R8, KC>(row, S1, K, lane, sc.surv, sc.stage, sc.hist, sc.a);
  half_topk_bf16<R8, KC>(row + S1, S2, K, lane, sc.surv, sc.stage, sc.hist, sc.b);
  cand_topk_bf16<KC>(sc.a, sc.b, K, S2, ctab, lane, sc.pv, sc.cstage, sc.hist, out_idx, out_wt);
}

// Whether a row shape takes the fast path, and its template parameters.
__host__ __device__ inline bool fast_select_ok(int bf16, int S1, int S2, int K) {
  return bf16 && S1 <= 1024 && S2 <= 1024 && K <= 128;
}
__host__ __device__ inline int fast_r8(int S1, int S2) {
  const int s = S1 > S2 ? S1 : S2;
  return s <= 256 ? 1 : (s <= 512 ? 2 : 4);
}
__host__ __device__ inline int fast_kc(int K) { return K <= 32 ? 32 : (K <= 64 ? 64 : 128); }

// Persistent fast selection kernel over rows of job0 followed by rows of job1.
template <int R8, int KC>
__global__ void __launch_bounds__(256, 4) sel_fast_kernel(SelJob job0, SelJob job1, long long n_rows,
                                                       int njobs, int S1, int S2) {
  // wait for the kernel ahead in the stream (programmatic launch), then let the next one in
  grid_dependency_wait();
  grid_launch_dependents();
  extern __shared__ __align__(16) unsigned char smem[];
  // the jobs' candidate tables, copied once per CTA: every row of a job reads the same one
  __shared__ uint16_t ctab_s[2][cand_count(KC)];
  const int K1 = njobs > 1 ? job1.K : job0.K;
  for (int i = threadIdx.x; i < cand_count_dev(job0.K); i += blockDim.x)
    ctab_s[0][i] = cand_table(job0.K)[i];
  for (int i = threadIdx.x; i < cand_count_dev(K1); i += blockDim.x)
    ctab_s[1][i] = cand_table(K1)[i];
  __syncthreads();
  unsigned char* scratch_base = smem;
  const uint16_t* tab0 = ctab_s[0];
  const uint16_t* tab1 = ctab_s[1];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wpc = blockDim.x >> 5;
  FastScratch sc = carve_fast_scratch(scratch_base + (size_t)warp * fast_scratch_bytes(S1, S2, KC),
                                      S1, S2, KC);
  reinterpret_cast<uint4*>(sc.hist)[2 * lane] = make_uint4(0u, 0u, 0u, 0u);
  reinterpret_cast<uint4*>(sc.hist)[2 * lane + 1] = make_uint4(0u, 0u, 0u, 0u);
  __syncwarp();
  const long long total = n_rows * njobs;
  const int S = S1 + S2;
  for (long long r = (long long)blockIdx.x * wpc + warp; r < total;
       r += (long long)gridDim.x * wpc) {
    const bool second = r >= n_rows;
    const SelJob& J = second ? job1 : job0;
    const long long row = sel_job_row(J, second ? r - n_rows : r);
    const __nv_bfloat16* src = reinterpret_cast<const __nv_bfloat16*>(J.halves) + (size_t)row * S;
    select_row_fast<R8, KC>(src, S1, S2, J.K, second ? tab1 : tab0, sc, lane,
                            J.idx + (size_t)row * J.ld, J.wt + (size_t)row * J.ld);
  }
}

inline size_t sel_fast_smem_bytes(int S1, int S2, int K0, int K1, int warps) {
  const int kc = fast_kc(K0 > K1 ? K0 : K1);
  return (size_t)warps * fast_scratch_bytes(S1, S2, kc);
}

}  // namespace sdm
