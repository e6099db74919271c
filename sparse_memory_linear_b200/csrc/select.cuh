// select.cuh -- step 1 of the SDM pass: product-key top-K slot selection, one warp per
// score row.
//
// Method: "Sparse Delta Memory: Scaling the State of Linear RNNs through Sparsity"
// (paper.rainbus.top summary), method step 1, and the SDM write-up on
// ai-paper-analysis.pages.dev, 步骤 1: the outer sum of two half-score vectors scores the
// N = S1*S2 slots; the top-K of each half, then the top-K of the candidate sums gives the
// top-K slots.  Order everywhere: score descending, slot index ascending.
//
// The warp works in shared memory:
//   1. both halves -> order-preserving 32-bit keys;
//   2. per half, a most-significant-digit radix select (8-bit digits, 256-bin histogram)
//      finds the bin of the K-th key; keys above it and the lowest-index keys inside it
//      form the half's top-K, then a bitonic sort gives their ranks;
//   3. candidates are the rank pairs (r1, r2) with (r1+1)(r2+1) <= K: every other pair is
//      preceded by at least K pairs with a larger-or-equal sum, so the pruned set holds all
//      pairs above the K-th largest sum T and T itself;
//   4. radix select over the candidate sums; ties at the threshold take the lowest flat
//      slot indices; bitonic sort of the K winners;
//   5. ties at T beyond the pruning (repair_ties_at_kth): when fp32 rounding can merge
//      unequal sums, a pair the pruning dropped may sum to T with a lower slot index than a
//      tie it kept; if one does, the ties at T are refilled from all K*K pairs;
//   6. softmax weights.
#pragma once

#include "common.cuh"

namespace sdm {

// Number of rank pairs (r1, r2) with (r1 + 1) * (r2 + 1) <= K.
__host__ __device__ constexpr inline int cand_count(int K) {
  int c = 0;
  for (int r = 1; r <= K; ++r) c += K / r;
  return c;
}

__host__ __device__ constexpr inline int pow2_at_least(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

// The rank pairs of every K in [1, KMAX], packed as r1 << 7 | r2 in (r1, r2) order,
// computed at compile time: table K starts at off[K] and holds off[K + 1] - off[K] pairs.
constexpr int cand_total() {
  int s = 0;
  for (int K = 1; K <= KMAX; ++K) s += cand_count(K);
  return s;
}
constexpr int CAND_TOTAL = cand_total();

struct CandTables {
  uint16_t e[CAND_TOTAL];
  int off[KMAX + 2];
};

constexpr CandTables make_cand_tables() {
  CandTables t{};
  int p = 0;
  for (int K = 1; K <= KMAX; ++K) {
    t.off[K] = p;
    for (int r1 = 0; r1 < K; ++r1)
      for (int r2 = 0; r2 < K / (r1 + 1); ++r2) t.e[p++] = static_cast<uint16_t>((r1 << 7) | r2);
  }
  t.off[KMAX + 1] = p;
  return t;
}

__device__ const CandTables g_cand_tables = make_cand_tables();

__device__ __forceinline__ const uint16_t* cand_table(int K) {
  return g_cand_tables.e + g_cand_tables.off[K];
}
__device__ __forceinline__ int cand_count_dev(int K) {
  return g_cand_tables.off[K + 1] - g_cand_tables.off[K];
}

// Shared scratch of one selecting warp.
struct SelScratch {
  uint32_t* keys;   // [S1 + S2]
  uint32_t* hist;   // [256]
  uint32_t* a_key;  // [KMAX] first-half top-K, sorted
  int32_t* a_idx;
  uint32_t* b_key;  // [KMAX] second-half top-K, sorted
  int32_t* b_idx;
  uint32_t* c_key;  // [C] candidate sums
  int32_t* c_flat;
  uint64_t* sortbuf;  // [pow2(KMAX)]
};

// Bytes of SelScratch for halves S1 + S2, top-K up to K (candidate table excluded).
__host__ __device__ inline size_t sel_scratch_bytes(int S1, int S2, int K) {
  const int C = cand_count(K);
  size_t b = 0;
  b += ((size_t)(S1 + S2) * 4 + 15) / 16 * 16;
  b += 256 * 4;
  b += 4 * (size_t)KMAX * 4;
  b += ((size_t)C * 8 + 15) / 16 * 16;
  b += (size_t)pow2_at_least(KMAX) * 8;
  return b;
}

__device__ inline SelScratch carve_sel_scratch(unsigned char* p, int S1, int S2, int K) {
  SelScratch s;
  const int C = cand_count_dev(K);  // K <= KMAX: the table's count, no division loop
  s.keys = reinterpret_cast<uint32_t*>(p);
  p += ((size_t)(S1 + S2) * 4 + 15) / 16 * 16;
  s.hist = reinterpret_cast<uint32_t*>(p);
  p += 256 * 4;
  s.a_key = reinterpret_cast<uint32_t*>(p);
  p += KMAX * 4;
  s.a_idx = reinterpret_cast<int32_t*>(p);
  p += KMAX * 4;
  s.b_key = reinterpret_cast<uint32_t*>(p);
  p += KMAX * 4;
  s.b_idx = reinterpret_cast<int32_t*>(p);
  p += KMAX * 4;
  s.c_key = reinterpret_cast<uint32_t*>(p);
  s.c_flat = reinterpret_cast<int32_t*>(p + (size_t)C * 4);
  p += ((size_t)C * 8 + 15) / 16 * 16;
  s.sortbuf = reinterpret_cast<uint64_t*>(p);
  return s;
}

// MSD radix select over n keys key(i): finds the 8-bit-digit bin that holds the K-th
// largest key.  On return, keys with (k & pmask) > prefix are above the bin, keys with
// (k & pmask) == prefix are in it; `krem` of the in-bin keys belong to the top-K and the
// bin holds `bin_count` keys.  min_shift stops the descent early (16 for bf16-derived
// keys, whose low 16 bits carry no information).
template <typename KeyAt>
__device__ inline void radix_select(KeyAt key, int n, int K, int min_shift, uint32_t* hist,
                                    int lane, uint32_t& prefix, uint32_t& pmask, int& krem,
                                    int& bin_count) {
  prefix = 0u;
  pmask = 0u;
  krem = K;
  bin_count = n;
  for (int shift = 24; shift >= min_shift; shift -= 8) {
    for (int b = lane; b < 256; b += 32) hist[b] = 0u;
    __syncwarp();
    for (int i = lane; i < n; i += 32) {
      const uint32_t k = key(i);
      if ((k & pmask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1u);
    }
    __syncwarp();
    // lane l owns bins 255-8l ... 248-8l, scanned from the top
    int c[8];
    int sum = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      c[j] = static_cast<int>(hist[255 - 8 * lane - j]);
      sum += c[j];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(FULL_MASK, incl, o);
      if (lane >= o) incl += t;
    }
    const int excl = incl - sum;
    const bool mine = excl < krem && krem <= incl;
    const unsigned ball = __ballot_sync(FULL_MASK, mine);
    const int src = __ffs(ball) - 1;
    int digit = 0, above = 0, cnt = 0;
    if (mine) {
      int run = excl;
      bool done = false;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (!done && run + c[j] >= krem) {
          digit = 255 - 8 * lane - j;
          above = run;
          cnt = c[j];
          done = true;
        }
        run += c[j];
      }
    }
    digit = __shfl_sync(FULL_MASK, digit, src);
    above = __shfl_sync(FULL_MASK, above, src);
    cnt = __shfl_sync(FULL_MASK, cnt, src);
    krem -= above;
    prefix |= static_cast<uint32_t>(digit) << shift;
    pmask |= 255u << shift;
    bin_count = cnt;
    __syncwarp();
    if (cnt == krem) break;  // the whole bin is taken: no need to split it further
  }
}

// Descending bitonic sort of n (a power of two) 64-bit values in shared memory.
__device__ inline void warp_bitonic_desc(uint64_t* s, int n, int lane) {
  for (int size = 2; size <= n; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = lane; i < (n >> 1); i += 32) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const uint64_t a = s[lo], b = s[hi];
        const bool desc = (lo & size) == 0;
        if ((a < b) == desc) {
          s[lo] = b;
          s[hi] = a;
        }
      }
      __syncwarp();
    }
  }
}

// Composite sort key: score key high, inverted index low, so that a larger value comes
// first in (score descending, index ascending) order.
__device__ __forceinline__ uint64_t composite(uint32_t key, int32_t idx) {
  return (static_cast<uint64_t>(key) << 32) | static_cast<uint64_t>(0xffffffffu - static_cast<uint32_t>(idx));
}

// ------------------------------------------------------------------------------------
// Ties at the K-th candidate sum beyond the rank-pair pruning.
//
// Let T be the K-th largest of the K*K candidate sums.  The pruned set P (rank pairs with
// (r1+1)(r2+1) <= K) holds every pair whose sum is above T (such a pair has fewer than K
// pairs at or above it, so its rank rectangle is smaller than K + 1) and at least K pairs at
// or above T, so T and the pairs above it are found exactly from P.  Only the ties at T can
// differ: with exact sums, a tie outside P has at least K pairs of its rank rectangle ahead
// of it (equal sums there mean equal half scores, hence lower indices), but when fp32
// rounding merges unequal sums, a dropped pair can sum to T with a lower slot index than a
// tie P kept.  Sums fall weakly along a rank row and no dropped pair is above T, so such a
// pair exists only if the first pair P drops in some rank row r1 >= 1, (r1, K/(r1+1)),
// sums to T.  The result is then repaired: ranks from the first tie on are refilled with
// the lowest slot indices among all K*K pairs whose sum is T.

// Whether every fp32 sum of two of the bf16 values val(0 .. 2K) is exact: the nonzero values'
// exponent fields (a subnormal's counted as 1) span at most 15 and stay below 254, so a sum
// needs at most 24 significant bits and cannot overflow.  Warp-wide.
template <typename Val>
__device__ __forceinline__ bool warp_bf16_sums_exact(Val val, int K, int lane) {
  uint32_t emin = 255u, emax = 0u;
  for (int j = lane; j < 2 * K; j += 32) {
    const uint32_t u = __float_as_uint(val(j)) & 0x7fffffffu;
    if (u != 0u) {
      const uint32_t e = max(u >> 23, 1u);
      emin = min(emin, e);
      emax = max(emax, e);
    }
  }
  emin = __reduce_min_sync(FULL_MASK, emin);
  emax = __reduce_max_sync(FULL_MASK, emax);
  return emax == 0u || (emax - emin <= 15u && emax < 254u);
}

// Warp-wide repair of a selection whose K-th key is Tk.  sum_key(r1, r2) is the order key of
// the fp32 sum of ranks r1, r2 (weakly decreasing in each), flat(r1, r2) the pair's slot
// index.  If some rank row's first dropped pair sums to Tk, emit(r, flat) is called for the
// ranks r = ngt .. K-1 (ngt: the pairs above Tk) with the lowest slot indices, ascending,
// among all pairs whose key is Tk, and true is returned; otherwise nothing is emitted.
// Emission happens on lane 0.
template <typename SumKey, typename Flat, typename Emit>
__device__ inline bool repair_ties_at_kth(SumKey sum_key, Flat flat, int K, uint32_t Tk,
                                          int lane, Emit emit) {
  bool hit = false;
  for (int r1 = 1 + lane; r1 < K; r1 += 32)
    if (sum_key(r1, K / (r1 + 1)) == Tk) hit = true;
  if (!__any_sync(FULL_MASK, hit)) return false;
  // per rank row, the columns [cs, ce) whose key is Tk, by binary search
  constexpr int RPL = KMAX / 32;
  int cs[RPL], ce[RPL];
  int ngt = 0;
#pragma unroll
  for (int q = 0; q < RPL; ++q) {
    const int r1 = lane + 32 * q;
    cs[q] = 0;
    ce[q] = 0;
    if (r1 < K) {
      int lo = 0, hi = K;
      while (lo < hi) {
        const int m = (lo + hi) >> 1;
        if (sum_key(r1, m) > Tk) lo = m + 1;
        else hi = m;
      }
      cs[q] = lo;
      hi = K;
      while (lo < hi) {
        const int m = (lo + hi) >> 1;
        if (sum_key(r1, m) >= Tk) lo = m + 1;
        else hi = m;
      }
      ce[q] = lo;
      ngt += cs[q];
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ngt += __shfl_xor_sync(FULL_MASK, ngt, o);
  // the lowest slot indices among the ties, one per round (slot indices are below 2^24)
  int floor_f = -1;
  for (int r = ngt; r < K; ++r) {
    uint32_t best = 0xffffffffu;
#pragma unroll
    for (int q = 0; q < RPL; ++q) {
      const int r1 = lane + 32 * q;
      for (int c = cs[q]; c < ce[q]; ++c) {
        const uint32_t f = flat(r1, c);
        if (static_cast<int>(f) > floor_f && f < best) best = f;
      }
    }
    best = __reduce_min_sync(FULL_MASK, best);
    if (best == 0xffffffffu) break;  // unreachable: P's own ties are among the pairs
    if (lane == 0) emit(r, best);
    floor_f = static_cast<int>(best);
  }
  __syncwarp();
  return true;
}

// Top-K of one half (keys[0..n), index = position), written sorted to out_key/out_idx.
__device__ inline void half_topk(const uint32_t* keys, int n, int K, int min_shift,
                                 SelScratch& sc, int lane, uint32_t* out_key,
                                 int32_t* out_idx) {
  uint32_t prefix, pmask;
  int krem, bin_count;
  radix_select([&](int i) { return keys[i]; }, n, K, min_shift, sc.hist, lane, prefix, pmask,
               krem, bin_count);
  const int P = pow2_at_least(K);
  int base = 0, tbase = 0;
  const unsigned lt = lanemask_lt();
  for (int i0 = 0; i0 < n; i0 += 32) {
    const int i = i0 + lane;
    const uint32_t k = i < n ? keys[i] : 0u;
    const uint32_t mk = k & pmask;
    const bool inb = i < n && mk == prefix;
    const bool abv = i < n && mk > prefix;
    const unsigned tb = __ballot_sync(FULL_MASK, inb);
    const int trank = tbase + __popc(tb & lt);
    const bool take = abv || (inb && trank < krem);
    const unsigned sb = __ballot_sync(FULL_MASK, take);
    if (take) sc.sortbuf[base + __popc(sb & lt)] = composite(k, i);
    base += __popc(sb);
    tbase += __popc(tb);
  }
  for (int j = K + lane; j < P; j += 32) sc.sortbuf[j] = 0ull;
  __syncwarp();
  warp_bitonic_desc(sc.sortbuf, P, lane);
  for (int j = lane; j < K; j += 32) {
    const uint64_t c = sc.sortbuf[j];
    out_key[j] = static_cast<uint32_t>(c >> 32);
    out_idx[j] = static_cast<int32_t>(0xffffffffu - static_cast<uint32_t>(c));
  }
  __syncwarp();
}

// Selects the top-K slots of one score row (first half S1 values, then S2 values) and
// writes flat slot indices and softmax weights to out_idx[j], out_wt[j], j < K.
// ctab holds the cand_count(K) rank pairs of K.  Every lane of the warp must call it.
__device__ inline void select_row(const void* row, bool bf16, int S1, int S2, int K,
                                  const uint16_t* ctab, SelScratch& sc, int lane,
                                  int32_t* out_idx, float* out_wt) {
  const int S = S1 + S2;
  const bool vec = (S & 7) == 0 && (reinterpret_cast<uintptr_t>(row) & 15u) == 0;
  if (vec) {
    for (int i = lane * 8; i < S; i += 256) {
      float f[8];
      load8_in(row, i, bf16, f);
#pragma unroll
      for (int j = 0; j < 8; ++j) sc.keys[i + j] = score_key(f[j]);
    }
  } else {
    for (int i = lane; i < S; i += 32) sc.keys[i] = score_key(load_in(row, i, bf16));
  }
  __syncwarp();
  const int min_shift = bf16 ? 16 : 0;
  half_topk(sc.keys, S1, K, min_shift, sc, lane, sc.a_key, sc.a_idx);
  half_topk(sc.keys + S1, S2, K, min_shift, sc, lane, sc.b_key, sc.b_idx);

  // candidate sums of the rank pairs
  const int C = cand_count_dev(K);
  for (int c = lane; c < C; c += 32) {
    const int e = __ldg(ctab + c);
    const int r1 = e >> 7, r2 = e & 127;
    const float s = __fadd_rn(key_score(sc.a_key[r1]), key_score(sc.b_key[r2]));
    sc.c_key[c] = score_key(s);
    sc.c_flat[c] = sc.a_idx[r1] * S2 + sc.b_idx[r2];
  }
  __syncwarp();

  uint32_t prefix, pmask;
  int krem, bin_count;
  radix_select([&](int i) { return sc.c_key[i]; }, C, K, 0, sc.hist, lane, prefix, pmask, krem,
               bin_count);
  const bool take_bin = bin_count == krem;
  int base = 0;
  const unsigned lt = lanemask_lt();
  for (int i0 = 0; i0 < C; i0 += 32) {
    const int i = i0 + lane;
    const uint32_t k = i < C ? sc.c_key[i] : 0u;
    const uint32_t mk = k & pmask;
    const bool take = i < C && (mk > prefix || (take_bin && mk == prefix));
    const unsigned sb = __ballot_sync(FULL_MASK, take);
    if (take) sc.sortbuf[base + __popc(sb & lt)] = composite(k, sc.c_flat[i]);
    base += __popc(sb);
  }
  __syncwarp();
  if (!take_bin) {
    // equal sums at the threshold: the lowest flat slot indices win, one at a time
    for (int r = 0; r < krem; ++r) {
      unsigned best = 0xffffffffu;
      for (int i = lane; i < C; i += 32) {
        if ((sc.c_key[i] & pmask) == prefix && sc.c_flat[i] >= 0) {
          best = min(best, static_cast<unsigned>(sc.c_flat[i]));
        }
      }
      best = __reduce_min_sync(FULL_MASK, best);
      for (int i = lane; i < C; i += 32) {
        if ((sc.c_key[i] & pmask) == prefix && static_cast<unsigned>(sc.c_flat[i]) == best) {
          sc.sortbuf[base] = composite(sc.c_key[i], sc.c_flat[i]);
          sc.c_flat[i] = -1;
        }
      }
      ++base;
      __syncwarp();
    }
  }
  const int P = pow2_at_least(K);
  for (int j = K + lane; j < P; j += 32) sc.sortbuf[j] = 0ull;
  __syncwarp();
  warp_bitonic_desc(sc.sortbuf, P, lane);

  // ties at the K-th sum beyond the pruning (exact bf16 sums cannot merge)
  if (!bf16 || !warp_bf16_sums_exact(
                   [&](int j) { return key_score(j < K ? sc.a_key[j] : sc.b_key[j - K]); }, K,
                   lane)) {
    const uint32_t Tk = static_cast<uint32_t>(sc.sortbuf[K - 1] >> 32);
    repair_ties_at_kth(
        [&](int r1, int r2) {
          return score_key(__fadd_rn(key_score(sc.a_key[r1]), key_score(sc.b_key[r2])));
        },
        [&](int r1, int r2) { return static_cast<uint32_t>(sc.a_idx[r1] * S2 + sc.b_idx[r2]); },
        K, Tk, lane, [&](int r, uint32_t f) { sc.sortbuf[r] = composite(Tk, static_cast<int32_t>(f)); });
  }

  // softmax over the selected scores
  const float s0 = key_score(static_cast<uint32_t>(sc.sortbuf[0] >> 32));
  float e[KMAX / 32];
  float part = 0.0f;
#pragma unroll
  for (int q = 0; q < KMAX / 32; ++q) {
    const int j = lane + 32 * q;
    e[q] = 0.0f;
    if (j < K) {
      const float s = key_score(static_cast<uint32_t>(sc.sortbuf[j] >> 32));
      e[q] = expf(s - s0);
      part += e[q];
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(FULL_MASK, part, o);
  const float inv = 1.0f / part;
#pragma unroll
  for (int q = 0; q < KMAX / 32; ++q) {
    const int j = lane + 32 * q;
    if (j < K) {
      out_idx[j] = static_cast<int32_t>(0xffffffffu - static_cast<uint32_t>(sc.sortbuf[j]));
      out_wt[j] = e[q] * inv;
    }
  }
  __syncwarp();
}

// One selection job: rows of `halves` ([rows, S1+S2], in_dtype) -> idx/wt with row
// stride ld (>= K).
struct SelJob {
  const void* halves;
  int32_t* idx;
  float* wt;
  int K;
  int ld;
  // Rows of a strided window (0: none).  Row r of the job is row
  // (r / seg_rows) * seg_stride + r % seg_rows of halves, idx and wt: a time chunk of every
  // sequence, when the pointers start at the chunk's first row of sequence 0.
  int seg_rows;
  long long seg_stride;
};

__device__ __forceinline__ long long sel_job_row(const SelJob& J, long long r) {
  if (J.seg_rows == 0) return r;
  const long long q = r / J.seg_rows;
  return q * J.seg_stride + (r - q * J.seg_rows);
}

// Persistent selection kernel over rows of job0 followed by rows of job1.
__global__ void __launch_bounds__(256) sel_kernel(SelJob job0, SelJob job1, long long n_rows,
                                                  int njobs, int S1, int S2, int bf16,
                                                  int kmax_all) {
  // wait for the kernel ahead in the stream (programmatic launch), then let the next one in
  grid_dependency_wait();
  grid_launch_dependents();
  extern __shared__ __align__(16) unsigned char smem[];
  unsigned char* scratch_base = smem;
  const uint16_t* tab0 = cand_table(job0.K);
  const uint16_t* tab1 = cand_table(njobs > 1 ? job1.K : job0.K);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wpc = blockDim.x >> 5;
  SelScratch sc = carve_sel_scratch(
      scratch_base + (size_t)warp * sel_scratch_bytes(S1, S2, kmax_all), S1, S2, kmax_all);
  const long long total = n_rows * njobs;
  const int S = S1 + S2;
  const size_t esz = bf16 ? 2 : 4;
  for (long long r = (long long)blockIdx.x * wpc + warp; r < total;
       r += (long long)gridDim.x * wpc) {
    const bool second = r >= n_rows;
    const SelJob& J = second ? job1 : job0;
    const long long row = sel_job_row(J, second ? r - n_rows : r);
    const void* src = reinterpret_cast<const unsigned char*>(J.halves) + (size_t)row * S * esz;
    select_row(src, bf16 != 0, S1, S2, J.K, second ? tab1 : tab0, sc, lane,
               J.idx + (size_t)row * J.ld, J.wt + (size_t)row * J.ld);
  }
}

inline size_t sel_smem_bytes(int S1, int S2, int K0, int K1, int warps) {
  const int kmax = K0 > K1 ? K0 : K1;
  return (size_t)warps * sel_scratch_bytes(S1, S2, kmax);
}

}  // namespace sdm
