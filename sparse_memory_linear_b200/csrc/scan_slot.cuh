// scan_slot.cuh -- the slot-parallel engine of steps 2 and 3 of the SDM pass.
//
// Method: "Sparse Delta Memory: Scaling the State of Linear RNNs through Sparsity"
// (paper.rainbus.top summary), method steps 2 and 3.  A write touches one slot, so every
// slot follows its own first-order recurrence over the tokens that select it,
//   M[i] <- a_t M[i] + b_t v_t,   a_t = alpha_t (1 - beta_t k_i),  b_t = beta_t k_i,
// and a read of slot i at token t needs M[i] after the writes of tokens <= t.
//
// Design.  The selections of every token are turned into events (slot, token, kind,
// weight) and sorted, stably, by (time chunk, sequence, head, slot) -- bit fields of a
// 32-bit key -- with an LSD radix sort; events of one slot inside one chunk are then
// contiguous and in token order, writes before reads at equal tokens.  Chunks run one
// after another (a slot's state carries over); inside a chunk every slot is independent.
//   * A warp takes the events of one slot ("segment"): the row is loaded once (a cp.async
//     ring keeps PF rows in flight per warp), the writes are applied in registers (the v
//     rows of a chunk are L2 resident), every read adds q * row into y with vector atomics
//     (the y rows of a chunk are L2 resident), and the row is stored once.
//   * A segment of at least SLOT_LONG events (a hot slot under skewed access) is taken by a
//     whole CTA: each warp composes the affine map of its slice of the events
//     (s -> A s + B), the maps are chained to give every slice its exact start state, and
//     each warp then re-walks its slice to produce the reads.
// Rows hit by many tokens cost one HBM round trip per chunk instead of one per token.
#pragma once

#include "common.cuh"

namespace sdm {

constexpr int RS_THREADS = 256;
constexpr int RS_WARPS = RS_THREADS / 32;
constexpr int RS_IPT = 16;                       // items per thread
constexpr int RS_TILE = RS_THREADS * RS_IPT;     // 4096 items per tile
constexpr int RS_BINS = 256;
constexpr uint32_t EV_SENTINEL = 0xffffffffu;
constexpr int SLOT_LONG = 256;  // events of a segment taken by a whole CTA

// Bit layout of an event key: chunk | sequence | head | slot (most significant first).
struct KeyBits {
  int nbits, hbits, bbits, cbits;
  __host__ __device__ int total() const { return nbits + hbits + bbits + cbits; }
  __host__ __device__ int chunk_shift() const { return nbits + hbits + bbits; }
};

__host__ __device__ inline int bits_for(long long n) {
  int b = 0;
  while ((1LL << b) < n) ++b;
  return b;
}

// ---------------------------------------------------------------- event construction
struct EventArgs {
  const int32_t* idx_w;  // [rows, ldw]
  const float* wt_w;
  const int32_t* idx_r;  // [rows, ldr]
  const float* wt_r;
  uint32_t* keys;        // [chunk rows * (W + R)]
  uint2* vals;
  float* y;              // [rows, d_v]: the chunk's rows are zeroed here
  uint32_t* offs;        // {0, events of the chunk}
  uint32_t* counters;    // {long segments, span queue}, zeroed here
  int B, T, H, N, W, R, ldw, ldr, d_v;
  int t0, ct;            // the chunk: tokens [t0, t0 + ct)
  KeyBits kb;
};

// Events of one time chunk, one warp per chunk row.  Chunk row r = (b * ct + tc) * H + h is
// token t0 + tc of sequence b, head h; its event e = r * (W + R) + j: j < W is write j of
// the row, else read j - W.  key = (b, h, slot) bit fields; val = {t << 8 | kind << 7 | j,
// weight bits}.
__global__ void __launch_bounds__(256) slot_events_kernel(EventArgs a) {
  // wait for the kernel ahead in the stream (programmatic launch), then let the next one in
  grid_dependency_wait();
  grid_launch_dependents();
  const int lane = threadIdx.x & 31;
  const long long crow = (long long)a.B * a.ct * a.H;
  const int per = a.W + a.R;
  const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long r = gw; r < crow; r += nw) {
    const int h = static_cast<int>(r % a.H);
    const long long bt = r / a.H;
    const int tc = static_cast<int>(bt % a.ct);
    const int b = static_cast<int>(bt / a.ct);
    const int t = a.t0 + tc;
    const long long row = ((long long)b * a.T + t) * a.H + h;
    const uint32_t kbase = ((static_cast<uint32_t>(b) << a.kb.hbits) | (uint32_t)h) << a.kb.nbits;
    const int32_t* iw = a.idx_w + row * a.ldw;
    const float* ww = a.wt_w + row * a.ldw;
    const int32_t* ir = a.idx_r + row * a.ldr;
    const float* wr = a.wt_r + row * a.ldr;
    uint32_t* keys = a.keys + r * per;
    uint2* vals = a.vals + r * per;
    for (int j = lane; j < per; j += 32) {
      const bool rd = j >= a.W;
      const int jj = rd ? j - a.W : j;
      int slot = rd ? ir[jj] : iw[jj];
      const float w = rd ? wr[jj] : ww[jj];
      if (static_cast<unsigned>(slot) >= static_cast<unsigned>(a.N)) {
        record_status(STATUS_BAD_INDEX);
        slot = 0;
      }
      keys[j] = kbase | (uint32_t)slot;
      vals[j] = make_uint2((static_cast<uint32_t>(t) << 8) | (rd ? 128u : 0u) | jj,
                           __float_as_uint(w));
    }
  }
  // the chunk's y rows: contiguous per sequence
  const long long tid0 = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long stride = (long long)gridDim.x * blockDim.x;
  const long long d4 = a.d_v / 4;
  const long long ny = (long long)a.ct * a.H * d4;
  float4* y4 = reinterpret_cast<float4*>(a.y);
  for (int b = 0; b < a.B; ++b) {
    const long long base = ((long long)b * a.T + a.t0) * a.H * d4;
    for (long long i = tid0; i < ny; i += stride) y4[base + i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  if (tid0 < 2) {
    a.counters[tid0] = 0u;
    a.offs[tid0] = tid0 == 0 ? 0u : static_cast<uint32_t>(crow * per);
  }
}

// --------------------------------------------------------------------- radix sort
// Per-tile histogram of one 8-bit digit: hist[digit * ntiles + tile].
__global__ void __launch_bounds__(RS_THREADS) radix_hist_kernel(const uint32_t* __restrict__ keys,
                                                                long long n, int shift,
                                                                uint32_t* __restrict__ hist,
                                                                int ntiles) {
  // wait for the kernel ahead in the stream (programmatic launch), then let the next one in
  grid_dependency_wait();
  grid_launch_dependents();
  __shared__ uint32_t h[RS_WARPS][RS_BINS];
  const int tid = threadIdx.x, warp = tid >> 5;
  for (int i = tid; i < RS_WARPS * RS_BINS; i += RS_THREADS) (&h[0][0])[i] = 0u;
  __syncthreads();
  const long long base = (long long)blockIdx.x * RS_TILE;
  // all of this thread's keys are loaded before the first count
  uint32_t k16[RS_IPT];
#pragma unroll
  for (int k = 0; k < RS_IPT; ++k) {
    const long long i = base + (long long)k * RS_THREADS + tid;
    k16[k] = i < n ? keys[i] : EV_SENTINEL;
  }
#pragma unroll
  for (int k = 0; k < RS_IPT; ++k)
    if (base + (long long)k * RS_THREADS + tid < n) atomicAdd(&h[warp][(k16[k] >> shift) & 255u], 1u);
  __syncthreads();
  uint32_t s = 0;
#pragma unroll
  for (int w = 0; w < RS_WARPS; ++w) s += h[w][tid];
  hist[(size_t)tid * ntiles + blockIdx.x] = s;
}

// Exclusive scan of one digit's per-tile counts (one CTA of 1024 threads per digit);
// totals[digit] receives the digit's count.
__global__ void __launch_bounds__(1024) radix_scan_kernel(uint32_t* __restrict__ hist, int ntiles,
                                                          uint32_t* __restrict__ totals) {
  // wait for the kernel ahead in the stream (programmatic launch), then let the next one in
  grid_dependency_wait();
  grid_launch_dependents();
  __shared__ uint32_t part[1024];
  const int d = blockIdx.x, tid = threadIdx.x;
  uint32_t* row = hist + (size_t)d * ntiles;
  const int per = (ntiles + 1023) / 1024;
  const int lo = tid * per;
  const int hi = min(lo + per, ntiles);
  uint32_t s = 0;
  for (int i = lo; i < hi; ++i) s += row[i];
  part[tid] = s;
  __syncthreads();
  for (int o = 1; o < 1024; o <<= 1) {
    const uint32_t v = tid >= o ? part[tid - o] : 0u;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  uint32_t run = part[tid] - s;  // exclusive prefix of this thread's range
  for (int i = lo; i < hi; ++i) {
    const uint32_t c = row[i];
    row[i] = run;
    run += c;
  }
  if (tid == 1023) totals[d] = part[1023];
}

// Exclusive prefix sum of one value per thread over a CTA of RS_THREADS threads (warp
// shuffles, one exchange through shared memory); `tot` receives the CTA total.
__device__ __forceinline__ uint32_t rs_block_excl(uint32_t v, uint32_t* warp_tot, uint32_t& tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(FULL_MASK, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  uint32_t before = 0;
  tot = 0;
#pragma unroll
  for (int w = 0; w < RS_WARPS; ++w) {
    const uint32_t c = warp_tot[w];
    before += w < warp ? c : 0u;
    tot += c;
  }
  return before + incl - v;
}

// Stable scatter of one digit.  Every tile ranks its items in order (warp by warp, 32 items
// at a time, peers found with match.any) and places their keys and tile positions in shared
// memory in digit order; then each digit's run is written to digit_base + tile_prefix, the
// values gathered from the tile by their staged positions: consecutive threads write
// consecutive addresses of one run.
constexpr size_t RS_SCATTER_SMEM = (size_t)RS_TILE * 6;  // staged keys and tile positions

__global__ void __launch_bounds__(RS_THREADS, 3) radix_scatter_kernel(
    const uint32_t* __restrict__ kin, const uint2* __restrict__ vin, uint32_t* __restrict__ kout,
    uint2* __restrict__ vout, long long n, int shift, const uint32_t* __restrict__ hist,
    const uint32_t* __restrict__ totals, int ntiles) {
  // wait for the kernel ahead in the stream (programmatic launch), then let the next one in
  grid_dependency_wait();
  grid_launch_dependents();
  extern __shared__ __align__(16) unsigned char rs_smem[];
  uint32_t* skey = reinterpret_cast<uint32_t*>(rs_smem);                        // [RS_TILE]
  uint16_t* sidx = reinterpret_cast<uint16_t*>(rs_smem + (size_t)RS_TILE * 4);  // [RS_TILE]
  __shared__ uint32_t wcnt[RS_WARPS][RS_BINS];
  __shared__ uint32_t dbase[RS_BINS];  // global position of the tile's first item of a digit
  __shared__ uint32_t lbase[RS_BINS];  // staged position of the tile's first item of a digit
  __shared__ uint32_t wtot[2][RS_WARPS];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long tile0 = (long long)blockIdx.x * RS_TILE;
  const long long base = tile0 + (long long)warp * (RS_TILE / RS_WARPS);
  // this thread's keys and its digit's counts, loads first
  uint32_t key[RS_IPT];
#pragma unroll
  for (int r = 0; r < RS_IPT; ++r) {
    const long long i = base + r * 32 + lane;
    key[r] = i < n ? kin[i] : 0u;
  }
  const uint32_t my_total = totals[tid];
  const uint32_t my_prefix = hist[(size_t)tid * ntiles + blockIdx.x];
  for (int i = tid; i < RS_WARPS * RS_BINS; i += RS_THREADS) (&wcnt[0][0])[i] = 0u;
  __syncthreads();
  const unsigned lt = lanemask_lt();
  uint32_t rank2[RS_IPT / 2];  // two in-warp ranks (< 512) per register
#pragma unroll
  for (int r = 0; r < RS_IPT; ++r) {
    const long long i = base + r * 32 + lane;
    const bool ok = i < n;
    const uint32_t d = ok ? ((key[r] >> shift) & 255u) : (256u + lane);
    const unsigned m = __match_any_sync(FULL_MASK, d);
    uint32_t before = 0;
    if (ok) before = wcnt[warp][d];
    const uint32_t rk = before + __popc(m & lt);
    if (r & 1) rank2[r >> 1] |= rk << 16;
    else rank2[r >> 1] = rk;
    __syncwarp();
    if (ok && (m & lt) == 0) wcnt[warp][d] = before + __popc(m);
    __syncwarp();
  }
  __syncthreads();
  // per digit (one per thread): the counts of the warps before each warp, the tile's count
  uint32_t run = 0;
#pragma unroll
  for (int w = 0; w < RS_WARPS; ++w) {
    const uint32_t c = wcnt[w][tid];
    wcnt[w][tid] = run;
    run += c;
  }
  uint32_t all;
  dbase[tid] = rs_block_excl(my_total, wtot[0], all) + my_prefix;
  lbase[tid] = rs_block_excl(run, wtot[1], all);
  __syncthreads();
#pragma unroll
  for (int r = 0; r < RS_IPT; ++r) {
    const long long i = base + r * 32 + lane;
    if (i < n) {
      const uint32_t d = (key[r] >> shift) & 255u;
      const uint32_t lp = lbase[d] + wcnt[warp][d] + ((rank2[r >> 1] >> (16 * (r & 1))) & 0xffffu);
      skey[lp] = key[r];
      sidx[lp] = static_cast<uint16_t>(i - tile0);
    }
  }
  __syncthreads();
  const int tn = static_cast<int>(min((long long)RS_TILE, n - tile0));
  for (int i = tid; i < tn; i += RS_THREADS) {
    const uint32_t k = skey[i];
    const uint32_t d = (k >> shift) & 255u;
    const uint32_t pos = dbase[d] + (static_cast<uint32_t>(i) - lbase[d]);
    kout[pos] = k;
    vout[pos] = vin[tile0 + sidx[i]];
  }
}

// Segments of at least SLOT_LONG events, listed as {first event, length}.  Any such segment
// holds two events 128 apart at a multiple of 128, p and p + 128 (its first 256 events
// contain a multiple of 128 no later than its 128th): one thread per multiple of 128 tests
// that pair and reports the segment only from the first multiple of 128 inside it, after
// finding its two ends by binary searches.
__global__ void __launch_bounds__(256) slot_long_segments_kernel(
    const uint32_t* __restrict__ keys, long long n, uint32_t* hot_count, uint2* hot_list,
    int hot_cap) {
  // wait for the kernel ahead in the stream (programmatic launch), then let the next one in
  grid_dependency_wait();
  grid_launch_dependents();
  static_assert(SLOT_LONG >= 256, "two samples 128 apart must fit in a long segment");
  const long long nsamp = (n + 127) / 128;
  for (long long si = (long long)blockIdx.x * blockDim.x + threadIdx.x; si < nsamp;
       si += (long long)gridDim.x * blockDim.x) {
    const long long p = si * 128;
    if (p + 128 >= n) continue;
    const uint32_t K = keys[p];
    if (keys[p + 128] != K) continue;
    if (p >= 128 && keys[p - 128] == K) continue;  // an earlier sample lies in the segment
    // first event: in (p - 128, p]
    long long lo = p >= 127 ? p - 127 : 0, hi = p;  // keys[hi] == K
    while (lo < hi) {
      const long long mid = (lo + hi) >> 1;
      if (keys[mid] == K) hi = mid;
      else lo = mid + 1;
    }
    const long long first = lo;
    // one past the last event: gallop from p + 128, then bisect
    long long good = p + 128, step = 128;
    while (good + step < n && keys[good + step] == K) {
      good += step;
      step *= 2;
    }
    long long bad = good + step < n ? good + step : n;  // keys[bad] != K or bad == n
    while (bad - good > 1) {
      const long long mid = (good + bad) >> 1;
      if (keys[mid] == K) good = mid;
      else bad = mid;
    }
    const long long len = bad - first;
    if (len >= SLOT_LONG) {
      const uint32_t pos = atomicAdd(hot_count, 1u);
      if (pos < (uint32_t)hot_cap)
        hot_list[pos] = make_uint2(static_cast<uint32_t>(first), static_cast<uint32_t>(len));
    }
  }
}

// ------------------------------------------------------------- chunk processing
struct SlotArgs {
  const uint32_t* keys;  // sorted
  const uint2* vals;
  const uint32_t* offs;  // chunk offsets
  const float* alpha;    // [rows]
  const float* beta;
  const void* v;         // [rows, d_v]
  float* M;              // [B*H, N, d_v]
  float* y;              // [rows, d_v]
  const uint32_t* hot_count;  // [n_chunks]
  const uint2* hot_list;      // [n_chunks, hot_cap]
  uint32_t* span_next;        // [n_chunks] dynamic span queue
  int hot_cap;
  int B, T, H, N, d_v, v_bf16;
  KeyBits kb;
  unsigned long long* cta_stats;  // [SDM_SLOT_STATS_CTAS][4] work per CTA, or null
  float* wlog;  // [rows, W, d_v] undo log (each written row as its write found it), or null
  int W;
};

// Stores the lane's part of a written row, as the write found it, to the undo log entry of
// write j of token row r (streamed: the log is read back only by an undo).
template <int NQ>
__device__ __forceinline__ void log_old_row(const SlotArgs& a, uint32_t r, uint32_t j, int lane,
                                            const float4 (&m)[NQ]) {
  float4* lg = reinterpret_cast<float4*>(a.wlog + ((size_t)r * a.W + j) * a.d_v);
  const int d4 = a.d_v / 4;
#pragma unroll
  for (int q = 0; q < NQ; ++q) {
    const int c = lane + 32 * q;
    if (c < d4) __stcs(lg + c, m[q]);
  }
}

// Per-CTA work of the chunk kernel (load-balance analysis), added while enabled:
// [0] events applied from short segments, [1] events of the long segments taken,
// [2] spans taken, [3] summed busy nanoseconds of the CTA's warps.
__device__ unsigned long long g_slot_cta_stats[SDM_SLOT_STATS_CTAS * 4];

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

constexpr int SLOT_THREADS = 256;
constexpr int SLOT_WARPS = SLOT_THREADS / 32;
constexpr int SLOT_SPAN = 256;

// Loads lane's part of a v row (NQ chunks of 4 values) as fp32.
template <int NQ>
__device__ __forceinline__ void load_v(const void* v, size_t off, bool bf16, int lane, int d4,
                                       float4 out[NQ]) {
#pragma unroll
  for (int q = 0; q < NQ; ++q) {
    const int c = lane + 32 * q;
    if (c < d4) {
      if (bf16) {
        const uint2 raw = *reinterpret_cast<const uint2*>(
            reinterpret_cast<const __nv_bfloat16*>(v) + off + 4 * c);
        const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&raw);
        const float2 f0 = __bfloat1622float2(p[0]), f1 = __bfloat1622float2(p[1]);
        out[q] = make_float4(f0.x, f0.y, f1.x, f1.y);
      } else {
        out[q] = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(v) + off + 4 * c);
      }
    }
  }
}

// Applies the events [first, last) of one slot of sequence b, head h to the lane's part of
// the row, m.  compose == false: writes update m, reads add q * m into y.  compose == true:
// m starts at 0 and accumulates the affine map's additive part, A_acc its multiplicative
// part; reads are skipped.  Returns whether any write was applied.
template <int NQ, int G, bool LOG>
__device__ __forceinline__ bool walk_events(const SlotArgs& a, uint32_t first, uint32_t last, int b,
                                            int h, int lane, float4 (&m)[NQ], bool compose,
                                            float& A_acc) {
  const int d4 = a.d_v / 4;
  const bool bf16 = a.v_bf16 != 0;
  bool wrote = false;
  for (uint32_t e = first; e < last; e += 32) {
    const int cnt = static_cast<int>(min(32u, last - e));
    uint32_t r32 = 0u, jl = 0u;
    float ca = 0.f, cb = 0.f;
    if (lane < cnt) {
      const uint2 pv = a.vals[e + lane];
      jl = pv.x & 127u;
      const uint32_t t = pv.x >> 8;
      const uint32_t kind = (pv.x >> 7) & 1u;
      const uint32_t r = ((uint32_t)b * a.T + t) * a.H + (uint32_t)h;
      const float w = __uint_as_float(pv.y);
      if (kind == 0u) {
        const float kb = a.beta[r] * w;
        ca = a.alpha[r] * (1.0f - kb);
        cb = kb;
      } else {
        ca = w;
      }
      r32 = r | (kind << 31);
    }
    for (int i0 = 0; i0 < cnt; i0 += G) {
      float4 vv[G][NQ];
      uint32_t rr[G];
#pragma unroll
      for (int i = 0; i < G; ++i) {
        rr[i] = __shfl_sync(FULL_MASK, r32, (i0 + i) & 31);
        if (i0 + i < cnt && (rr[i] >> 31) == 0u)
          load_v<NQ>(a.v, (size_t)(rr[i] & 0x7fffffffu) * a.d_v, bf16, lane, d4, vv[i]);
      }
#pragma unroll
      for (int i = 0; i < G; ++i) {
        const float A = __shfl_sync(FULL_MASK, ca, (i0 + i) & 31);
        const float Bc = __shfl_sync(FULL_MASK, cb, (i0 + i) & 31);
        if (i0 + i < cnt) {
          if ((rr[i] >> 31) == 0u) {
            if (LOG && !compose)
              log_old_row<NQ>(a, rr[i], __shfl_sync(FULL_MASK, jl, (i0 + i) & 31), lane, m);
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
              m[q].x = fmaf(A, m[q].x, Bc * vv[i][q].x);
              m[q].y = fmaf(A, m[q].y, Bc * vv[i][q].y);
              m[q].z = fmaf(A, m[q].z, Bc * vv[i][q].z);
              m[q].w = fmaf(A, m[q].w, Bc * vv[i][q].w);
            }
            A_acc *= A;
            wrote = true;
          } else if (!compose) {
            float* yrow = a.y + (size_t)(rr[i] & 0x7fffffffu) * a.d_v;
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
              const int c = lane + 32 * q;
              if (c < d4)
                atomicAdd(reinterpret_cast<float4*>(yrow) + c,
                          make_float4(A * m[q].x, A * m[q].y, A * m[q].z, A * m[q].w));
            }
          }
        }
      }
    }
  }
  return wrote;
}

__host__ __device__ constexpr inline size_t slot_warp_smem(int NQ, int PF) {
  return (size_t)PF * 128 * NQ * 4 + (size_t)SLOT_SPAN * 4;
}

// One chunk.  CTAs first take the chunk's long segments, one CTA each (see the file
// comment); then every warp takes spans of SLOT_SPAN sorted events from a queue and handles
// each shorter segment that starts in its span, streaming the segments' state rows through
// a ring of PF shared-memory rows with cp.async.
// LOG: also store each written row, as its write finds it, to the undo log a.wlog (a
// separate instantiation, so that the plain pass keeps its registers).
template <int NQ, int G, int PF, bool LOG>
__global__ void __launch_bounds__(SLOT_THREADS, (NQ <= 2 ? 4 : 1)) slot_chunk_kernel(SlotArgs a, int chunk) {
  // wait for the kernel ahead in the stream (programmatic launch), then let the next one in
  grid_dependency_wait();
  grid_launch_dependents();
  extern __shared__ __align__(16) unsigned char smem[];
  const uint32_t e0 = a.offs[chunk], e1 = a.offs[chunk + 1];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned long long* stats =
      a.cta_stats && blockIdx.x < SDM_SLOT_STATS_CTAS ? a.cta_stats + 4 * blockIdx.x : nullptr;
  const unsigned long long t_start = stats ? global_ns() : 0ull;
  unsigned long long n_short = 0, n_long = 0, n_spans = 0;
  const int d4 = a.d_v / 4;
  const bool bf16 = a.v_bf16 != 0;
  const unsigned lt = lanemask_lt();
  const uint32_t nmask = (1u << a.kb.nbits) - 1u;
  const uint32_t hmask = (1u << a.kb.hbits) - 1u;
  const uint32_t bmask = (1u << a.kb.bbits) - 1u;
  auto row_of = [&](uint32_t K, int& b, int& h) -> float* {
    const uint32_t slot = K & nmask;
    h = static_cast<int>((K >> a.kb.nbits) & hmask);
    b = static_cast<int>((K >> (a.kb.nbits + a.kb.hbits)) & bmask);
    return a.M + (((size_t)b * a.H + h) * a.N + slot) * a.d_v;
  };

  // ---- long segments: one CTA per segment
  {
    float* coefA = reinterpret_cast<float*>(smem);  // [SLOT_WARPS] (32 reserved)
    float* coefB = coefA + 32;                      // [SLOT_WARPS][128 * NQ]
    const uint32_t nh = min(a.hot_count[chunk], (uint32_t)a.hot_cap);
    for (uint32_t hs = blockIdx.x; hs < nh; hs += gridDim.x) {
      const uint2 seg = a.hot_list[(size_t)chunk * a.hot_cap + hs];
      const uint32_t first = seg.x, n = seg.y;
      if (warp == 0) n_long += n;
      int b, h;
      float* row = row_of(a.keys[first], b, h);
      const uint32_t per = (n + SLOT_WARPS - 1) / SLOT_WARPS;
      const uint32_t s0 = first + min(n, per * warp), s1 = first + min(n, per * (warp + 1));
      // 1. this slice's affine map s -> A s + m
      float4 m[NQ];
#pragma unroll
      for (int q = 0; q < NQ; ++q) m[q] = make_float4(0.f, 0.f, 0.f, 0.f);
      float A = 1.0f;
      walk_events<NQ, G, LOG>(a, s0, s1, b, h, lane, m, true, A);
      if (lane == 0) coefA[warp] = A;
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const int c = lane + 32 * q;
        if (c < d4) reinterpret_cast<float4*>(coefB + warp * 128 * NQ)[c] = m[q];
      }
      __syncthreads();
      // 2. start state of this slice: the row after the slices before it
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const int c = lane + 32 * q;
        if (c < d4) m[q] = reinterpret_cast<const float4*>(row)[c];
      }
      for (int k = 0; k < warp; ++k) {
        const float Ak = coefA[k];
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          const int c = lane + 32 * q;
          if (c < d4) {
            const float4 Bk = reinterpret_cast<const float4*>(coefB + k * 128 * NQ)[c];
            m[q].x = fmaf(Ak, m[q].x, Bk.x);
            m[q].y = fmaf(Ak, m[q].y, Bk.y);
            m[q].z = fmaf(Ak, m[q].z, Bk.z);
            m[q].w = fmaf(Ak, m[q].w, Bk.w);
          }
        }
      }
      __syncthreads();  // every warp has read the row before the last one rewrites it
      // 3. re-walk the slice from its exact start state: the reads, and the final row
      float unused = 1.0f;
      walk_events<NQ, G, LOG>(a, s0, s1, b, h, lane, m, false, unused);
      if (warp == SLOT_WARPS - 1) {
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          const int c = lane + 32 * q;
          if (c < d4) reinterpret_cast<float4*>(row)[c] = m[q];
        }
      }
      __syncthreads();  // coefficients are reused by the next long segment
    }
  }

  // ---- the other segments, span by span
  float* ring = reinterpret_cast<float*>(smem + (size_t)warp * slot_warp_smem(NQ, PF));
  uint32_t* heads = reinterpret_cast<uint32_t*>(ring + (size_t)PF * 128 * NQ);
  while (true) {
    uint32_t span_id = 0;
    if (lane == 0) span_id = atomicAdd(&a.span_next[chunk], 1u);
    span_id = __shfl_sync(FULL_MASK, span_id, 0);
    if (span_id >= (e1 - e0 + SLOT_SPAN - 1) / SLOT_SPAN) break;
    ++n_spans;
    const uint32_t span = e0 + span_id * (uint32_t)SLOT_SPAN;
    const uint32_t span_end = min(e1, span + (uint32_t)SLOT_SPAN);
    // heads of the short segments starting in the span, in event order
    int nh = 0;
    for (uint32_t tile = span; tile < span_end; tile += 32) {
      const uint32_t ei = tile + lane;
      const uint32_t k = ei < span_end ? a.keys[ei] : EV_SENTINEL;
      uint32_t kprev = __shfl_up_sync(FULL_MASK, k, 1);
      if (lane == 0) kprev = tile > e0 ? a.keys[tile - 1] : EV_SENTINEL;
      bool head = ei < span_end && k != kprev;
      if (head && ei + SLOT_LONG - 1 < e1 && a.keys[ei + SLOT_LONG - 1] == k) head = false;
      const unsigned hm = __ballot_sync(FULL_MASK, head);
      if (head) heads[nh + __popc(hm & lt)] = ei;
      nh += __popc(hm);
    }
    __syncwarp();
    if (nh == 0) continue;
    // The warp's events: [first, stop), every event of the short segments that start in the
    // span (a long segment can only be the span's last head, and then no head follows it).
    const uint32_t first = heads[0];
    uint32_t stop = heads[nh - 1];
    {
      const uint32_t K = a.keys[stop];
      while (true) {
        const uint32_t ek = stop + lane;
        const unsigned m2 = __ballot_sync(FULL_MASK, ek < e1 && a.keys[ek] == K);
        if (m2 == FULL_MASK) {
          stop += 32;
          continue;
        }
        stop += __ffs(~m2) - 1;
        break;
      }
    }

    n_short += stop - first;
    auto issue = [&](int i) {
      if (i < nh) {
        int bb, hh;
        const float* src = row_of(a.keys[heads[i]], bb, hh);
        float* dst = ring + (size_t)(i % PF) * 128 * NQ;
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          const int c = lane + 32 * q;
          if (c < d4) cp_async16(dst + 4 * c, src + 4 * c);
        }
      }
      cp_async_commit();
    };
#pragma unroll
    for (int i = 0; i < PF - 1; ++i) issue(i);

    // Events stream in batches of 32, one per lane: the batch's key and value were loaded
    // while the batch before it was processed, and its coefficients take one round trip
    // (alpha, beta) issued before the batch's first state row is waited for.
    int seg = -1;
    float* row = nullptr;
    bool dirty = false;
    float4 m[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) m[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    auto close_segment = [&]() {
      if (seg >= 0 && dirty) {
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          const int c = lane + 32 * q;
          if (c < d4) reinterpret_cast<float4*>(row)[c] = m[q];
        }
      }
      __syncwarp();  // the ring slot is refilled by the next issue()
    };
    uint32_t nk = EV_SENTINEL;
    uint2 npv = make_uint2(0u, 0u);
    if (first + lane < stop) {
      nk = a.keys[first + lane];
      npv = a.vals[first + lane];
    }
    uint32_t kcarry = EV_SENTINEL;  // the key before the batch (first is a head)
    for (uint32_t b0 = first; b0 < stop; b0 += 32) {
      const int cnt = static_cast<int>(min(32u, stop - b0));
      const uint32_t ck = nk;
      const uint2 pv = npv;
      if (b0 + 32 + lane < stop) {
        nk = a.keys[b0 + 32 + lane];
        npv = a.vals[b0 + 32 + lane];
      }
      uint32_t kp = __shfl_up_sync(FULL_MASK, ck, 1);
      if (lane == 0) kp = kcarry;
      kcarry = __shfl_sync(FULL_MASK, ck, cnt - 1);
      const bool head = lane < cnt && ck != kp;
      // this lane's event: state row coefficients and token row
      uint32_t r32 = 0u, jl = 0u;
      float ca = 0.f, cb = 0.f;
      if (lane < cnt) {
        jl = pv.x & 127u;
        const uint32_t t = pv.x >> 8;
        const uint32_t kind = (pv.x >> 7) & 1u;
        const uint32_t eh = (ck >> a.kb.nbits) & hmask;
        const uint32_t eb = (ck >> (a.kb.nbits + a.kb.hbits)) & bmask;
        const uint32_t r = (eb * a.T + t) * a.H + eh;
        const float w = __uint_as_float(pv.y);
        if (kind == 0u) {
          const float kb = a.beta[r] * w;
          ca = a.alpha[r] * (1.0f - kb);
          cb = kb;
        } else {
          ca = w;
        }
        r32 = r | (kind << 31);
      }
      for (int i0 = 0; i0 < cnt; i0 += G) {
        float4 vv[G][NQ];
        uint32_t rr[G];
#pragma unroll
        for (int i = 0; i < G; ++i) {
          rr[i] = __shfl_sync(FULL_MASK, r32, (i0 + i) & 31);
          if (i0 + i < cnt && (rr[i] >> 31) == 0u)
            load_v<NQ>(a.v, (size_t)(rr[i] & 0x7fffffffu) * a.d_v, bf16, lane, d4, vv[i]);
        }
#pragma unroll
        for (int i = 0; i < G; ++i) {
          const bool hd = __shfl_sync(FULL_MASK, head, (i0 + i) & 31) != 0;
          const float A = __shfl_sync(FULL_MASK, ca, (i0 + i) & 31);
          const float Bc = __shfl_sync(FULL_MASK, cb, (i0 + i) & 31);
          if (i0 + i < cnt) {
            if (hd) {
              close_segment();
              ++seg;
              issue(seg + PF - 1);
              cp_async_wait<PF - 1>();
              __syncwarp();
              int bb, hh;
              row = row_of(a.keys[heads[seg]], bb, hh);
              const float* slot_row = ring + (size_t)(seg % PF) * 128 * NQ;
#pragma unroll
              for (int q = 0; q < NQ; ++q) {
                const int c = lane + 32 * q;
                if (c < d4) m[q] = reinterpret_cast<const float4*>(slot_row)[c];
              }
              dirty = false;
            }
            if ((rr[i] >> 31) == 0u) {
              if (LOG)
                log_old_row<NQ>(a, rr[i], __shfl_sync(FULL_MASK, jl, (i0 + i) & 31), lane, m);
#pragma unroll
              for (int q = 0; q < NQ; ++q) {
                m[q].x = fmaf(A, m[q].x, Bc * vv[i][q].x);
                m[q].y = fmaf(A, m[q].y, Bc * vv[i][q].y);
                m[q].z = fmaf(A, m[q].z, Bc * vv[i][q].z);
                m[q].w = fmaf(A, m[q].w, Bc * vv[i][q].w);
              }
              dirty = true;
            } else {
              float* yrow = a.y + (size_t)(rr[i] & 0x7fffffffu) * a.d_v;
#pragma unroll
              for (int q = 0; q < NQ; ++q) {
                const int c = lane + 32 * q;
                if (c < d4)
                  atomicAdd(reinterpret_cast<float4*>(yrow) + c,
                            make_float4(A * m[q].x, A * m[q].y, A * m[q].z, A * m[q].w));
              }
            }
          }
        }
      }
    }
    close_segment();
    cp_async_wait<0>();
    __syncwarp();
  }
  if (stats && lane == 0) {
    atomicAdd(stats + 0, n_short);
    atomicAdd(stats + 1, n_long);
    atomicAdd(stats + 2, n_spans);
    atomicAdd(stats + 3, global_ns() - t_start);
  }
}

}  // namespace sdm
