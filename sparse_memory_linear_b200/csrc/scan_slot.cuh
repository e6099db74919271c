// scan_slot.cuh -- the slot-parallel engine of steps 2 and 3 of the SDM pass.
//
// Method: "Sparse Delta Memory: Scaling the State of Linear RNNs through Sparsity"
// (paper.rainbus.top summary), method steps 2 and 3.  A write touches one slot, so every
// slot follows its own first-order recurrence over the tokens that select it,
//   M[i] <- a_t M[i] + b_t v_t,   a_t = alpha_t (1 - beta_t k_i),  b_t = beta_t k_i,
// and a read of slot i at token t needs M[i] after the writes of tokens <= t.
//
// Design.  The selections of every token are turned into events (slot, token, kind,
// weight) and sorted, stably, by (time chunk, sequence, head, slot) with an LSD radix
// sort; events of one slot inside one chunk are then contiguous and in token order,
// writes before reads at equal tokens.  Chunks run one after another (a slot's state
// carries over); inside a chunk every slot is independent.  A warp takes the events of
// one slot, loads the row once, applies the writes in registers (v rows of the chunk are
// L2 resident), adds q * row into y for every read (y rows of the chunk are L2
// resident), and stores the row once.  Rows hit by many tokens (skewed access) cost one
// HBM round trip per chunk instead of one per token.
#pragma once

#include "common.cuh"

namespace sdm {

constexpr int RS_THREADS = 256;
constexpr int RS_WARPS = RS_THREADS / 32;
constexpr int RS_IPT = 16;                       // items per thread
constexpr int RS_TILE = RS_THREADS * RS_IPT;     // 4096 items per tile
constexpr int RS_BINS = 256;
constexpr uint32_t EV_SENTINEL = 0xffffffffu;

// ---------------------------------------------------------------- event construction
struct EventArgs {
  const int32_t* idx_w;  // [rows, ldw]
  const float* wt_w;
  const int32_t* idx_r;  // [rows, ldr]
  const float* wt_r;
  uint32_t* keys;        // [rows * (W + R)]
  uint2* vals;
  float* y;              // [rows, d_v], zeroed here
  int B, T, H, N, W, R, ldw, ldr, d_v, chunk;
};

// Event e = row * (W + R) + j: j < W is write j of the row, else read j - W.
// key = ((chunk * B + b) * H + h) * N + slot; val = {t << 8 | kind << 7 | j, weight bits}.
__global__ void __launch_bounds__(256) slot_events_kernel(EventArgs a) {
  const long long rows = (long long)a.B * a.T * a.H;
  const int per = a.W + a.R;
  const long long n = rows * per;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += stride) {
    const long long row = e / per;
    const int j = static_cast<int>(e - row * per);
    const int h = static_cast<int>(row % a.H);
    const long long bt = row / a.H;
    const int t = static_cast<int>(bt % a.T);
    const int b = static_cast<int>(bt / a.T);
    const bool rd = j >= a.W;
    const int jj = rd ? j - a.W : j;
    int slot = rd ? a.idx_r[row * a.ldr + jj] : a.idx_w[row * a.ldw + jj];
    const float w = rd ? a.wt_r[row * a.ldr + jj] : a.wt_w[row * a.ldw + jj];
    if (static_cast<unsigned>(slot) >= static_cast<unsigned>(a.N)) {
      record_status(STATUS_BAD_INDEX);
      slot = 0;
    }
    const int c = t / a.chunk;
    const uint32_t g = static_cast<uint32_t>((c * a.B + b) * a.H + h);
    a.keys[e] = g * static_cast<uint32_t>(a.N) + static_cast<uint32_t>(slot);
    a.vals[e] = make_uint2((static_cast<uint32_t>(t) << 8) | (rd ? 128u : 0u) | jj,
                           __float_as_uint(w));
  }
  const long long ny = rows * a.d_v / 4;
  float4* y4 = reinterpret_cast<float4*>(a.y);
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < ny; i += stride)
    y4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// --------------------------------------------------------------------- radix sort
// Per-tile histogram of one 8-bit digit: hist[digit * ntiles + tile].
__global__ void __launch_bounds__(RS_THREADS) radix_hist_kernel(const uint32_t* __restrict__ keys,
                                                                long long n, int shift,
                                                                uint32_t* __restrict__ hist,
                                                                int ntiles) {
  __shared__ uint32_t h[RS_WARPS][RS_BINS];
  const int tid = threadIdx.x, warp = tid >> 5;
  for (int i = tid; i < RS_WARPS * RS_BINS; i += RS_THREADS) (&h[0][0])[i] = 0u;
  __syncthreads();
  const long long base = (long long)blockIdx.x * RS_TILE;
#pragma unroll 4
  for (int k = 0; k < RS_IPT; ++k) {
    const long long i = base + (long long)k * RS_THREADS + tid;
    if (i < n) atomicAdd(&h[warp][(keys[i] >> shift) & 255u], 1u);
  }
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

// Stable scatter of one digit: every tile ranks its items in order (warp by warp, 32
// items at a time, peers found with match.any), then writes them at
// digit_base + tile_prefix + rank.
__global__ void __launch_bounds__(RS_THREADS) radix_scatter_kernel(
    const uint32_t* __restrict__ kin, const uint2* __restrict__ vin, uint32_t* __restrict__ kout,
    uint2* __restrict__ vout, long long n, int shift, const uint32_t* __restrict__ hist,
    const uint32_t* __restrict__ totals, int ntiles) {
  __shared__ uint32_t wcnt[RS_WARPS][RS_BINS];
  __shared__ uint32_t dbase[RS_BINS];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < RS_WARPS * RS_BINS; i += RS_THREADS) (&wcnt[0][0])[i] = 0u;
  // digit bases: exclusive prefix of the totals (one digit per thread)
  {
    __shared__ uint32_t sc[RS_BINS];
    sc[tid] = totals[tid];
    __syncthreads();
    for (int o = 1; o < RS_BINS; o <<= 1) {
      const uint32_t v = tid >= o ? sc[tid - o] : 0u;
      __syncthreads();
      sc[tid] += v;
      __syncthreads();
    }
    dbase[tid] = sc[tid] - totals[tid] + hist[(size_t)tid * ntiles + blockIdx.x];
  }
  __syncthreads();
  const long long base = (long long)blockIdx.x * RS_TILE + (long long)warp * (RS_TILE / RS_WARPS);
  const unsigned lt = lanemask_lt();
  uint32_t key[RS_IPT];
  uint32_t rank[RS_IPT];
#pragma unroll
  for (int r = 0; r < RS_IPT; ++r) {
    const long long i = base + r * 32 + lane;
    const bool ok = i < n;
    key[r] = ok ? kin[i] : 0u;
    const uint32_t d = ok ? ((key[r] >> shift) & 255u) : (256u + lane);
    const unsigned m = __match_any_sync(FULL_MASK, d);
    uint32_t before = 0;
    if (ok) before = wcnt[warp][d];
    rank[r] = before + __popc(m & lt);
    __syncwarp();
    if (ok && (m & lt) == 0) wcnt[warp][d] = before + __popc(m);
    __syncwarp();
  }
  __syncthreads();
  // per digit: the counts of the warps before this one
  {
    uint32_t run = 0;
#pragma unroll
    for (int w = 0; w < RS_WARPS; ++w) {
      const uint32_t c = wcnt[w][tid];
      wcnt[w][tid] = run;
      run += c;
    }
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < RS_IPT; ++r) {
    const long long i = base + r * 32 + lane;
    if (i < n) {
      const uint32_t d = (key[r] >> shift) & 255u;
      const uint32_t pos = dbase[d] + wcnt[warp][d] + rank[r];
      kout[pos] = key[r];
      vout[pos] = vin[i];
    }
  }
}

// First event of every chunk in the sorted keys (binary search); offs[n_chunks] = n.
__global__ void slot_chunk_offsets_kernel(const uint32_t* __restrict__ keys, long long n,
                                          int n_chunks, uint32_t per_chunk_keys,
                                          uint32_t* __restrict__ offs) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c > n_chunks) return;
  if (c == n_chunks) {
    offs[c] = static_cast<uint32_t>(n);
    return;
  }
  const unsigned long long target = (unsigned long long)c * per_chunk_keys;
  long long lo = 0, hi = n;
  while (lo < hi) {
    const long long mid = (lo + hi) >> 1;
    if ((unsigned long long)keys[mid] < target) lo = mid + 1;
    else hi = mid;
  }
  offs[c] = static_cast<uint32_t>(lo);
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
  int B, T, H, N, d_v, v_bf16;
};

constexpr int SLOT_THREADS = 256;

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

// Per-warp shared memory of slot_chunk_kernel: a ring of PF state rows (128*NQ floats each)
// and the segment heads of one span of events.
constexpr int SLOT_SPAN = 256;

__host__ __device__ constexpr inline size_t slot_warp_smem(int NQ, int PF) {
  return (size_t)PF * 128 * NQ * 4 + (size_t)SLOT_SPAN * 4;
}

// One chunk.  Warps take spans of SLOT_SPAN sorted events; a warp handles every slot segment
// that starts in its span, to the segment's end.  It first lists the span's segment heads,
// then streams the segments' state rows into a ring of PF shared-memory rows with cp.async,
// PF - 1 segments ahead of the one it applies, so that every warp keeps several HBM row
// reads in flight.  G write events have their v rows (L2 resident) loaded together.
template <int NQ, int G, int PF>
__global__ void __launch_bounds__(SLOT_THREADS) slot_chunk_kernel(SlotArgs a, int chunk) {
  extern __shared__ __align__(16) unsigned char smem[];
  const uint32_t e0 = a.offs[chunk], e1 = a.offs[chunk + 1];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gw = (blockIdx.x * SLOT_THREADS + threadIdx.x) >> 5;
  const int nw = (gridDim.x * SLOT_THREADS) >> 5;
  const int d4 = a.d_v / 4;
  const bool bf16 = a.v_bf16 != 0;
  const unsigned lt = lanemask_lt();
  const uint32_t per_g = static_cast<uint32_t>(a.N);
  float* ring = reinterpret_cast<float*>(smem + (size_t)warp * slot_warp_smem(NQ, PF));
  uint32_t* heads = reinterpret_cast<uint32_t*>(ring + (size_t)PF * 128 * NQ);

  auto row_of = [&](uint32_t K) -> float* {
    const uint32_t g = K / per_g;
    const uint32_t slot = K - g * per_g;
    const uint32_t h = g % a.H;
    const uint32_t b = (g / a.H) % a.B;
    return a.M + (((size_t)b * a.H + h) * a.N + slot) * a.d_v;
  };

  for (uint32_t span = e0 + (uint32_t)SLOT_SPAN * gw; span < e1; span += (uint32_t)SLOT_SPAN * nw) {
    const uint32_t span_end = min(e1, span + (uint32_t)SLOT_SPAN);
    // segment heads of the span, in event order
    int nh = 0;
    for (uint32_t tile = span; tile < span_end; tile += 32) {
      const uint32_t ei = tile + lane;
      const uint32_t k = ei < span_end ? a.keys[ei] : EV_SENTINEL;
      uint32_t kprev = __shfl_up_sync(FULL_MASK, k, 1);
      if (lane == 0) kprev = tile > e0 ? a.keys[tile - 1] : EV_SENTINEL;
      const bool head = ei < span_end && k != kprev;
      const unsigned hm = __ballot_sync(FULL_MASK, head);
      if (head) heads[nh + __popc(hm & lt)] = ei;
      nh += __popc(hm);
    }
    __syncwarp();

    auto issue = [&](int i) {
      if (i < nh) {
        const float* src = row_of(a.keys[heads[i]]);
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

    for (int si = 0; si < nh; ++si) {
      issue(si + PF - 1);
      cp_async_wait<PF - 1>();
      __syncwarp();
      const uint32_t hpos = heads[si];
      const uint32_t K = a.keys[hpos];
      const uint32_t g = K / per_g;
      const int h = static_cast<int>(g % a.H);
      const int b = static_cast<int>((g / a.H) % a.B);
      float* row = row_of(K);
      const float* slot_row = ring + (size_t)(si % PF) * 128 * NQ;
      float4 m[NQ];
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const int c = lane + 32 * q;
        if (c < d4) m[q] = reinterpret_cast<const float4*>(slot_row)[c];
      }
      bool dirty = false;
      uint32_t e = hpos;
      while (true) {
        // next batch of up to 32 events of this slot
        const uint32_t ej = e + lane;
        const uint32_t kj = ej < e1 ? a.keys[ej] : EV_SENTINEL;
        const unsigned match = __ballot_sync(FULL_MASK, kj == K);
        const int cnt = match == FULL_MASK ? 32 : __ffs(~match) - 1;
        float ca = 0.f, cb = 0.f;
        size_t rowoff = 0;
        int kind = 1;
        if (lane < cnt) {
          const uint2 pv = a.vals[ej];
          const int t = static_cast<int>(pv.x >> 8);
          kind = (pv.x >> 7) & 1;
          const size_t r = ((size_t)b * a.T + t) * a.H + h;
          rowoff = r * a.d_v;
          const float w = __uint_as_float(pv.y);
          if (kind == 0) {
            const float kb = a.beta[r] * w;
            ca = a.alpha[r] * (1.0f - kb);
            cb = kb;
          } else {
            ca = w;
          }
        }
        for (int i0 = 0; i0 < cnt; i0 += G) {
          const int ng = min(G, cnt - i0);
          float4 vv[G][NQ];
#pragma unroll
          for (int i = 0; i < G; ++i) {
            const int src = (i0 + i) & 31;
            const int kd = __shfl_sync(FULL_MASK, kind, src);
            const size_t ro = __shfl_sync(FULL_MASK, rowoff, src);
            if (i < ng && kd == 0) load_v<NQ>(a.v, ro, bf16, lane, d4, vv[i]);
          }
#pragma unroll
          for (int i = 0; i < G; ++i) {
            const int src = (i0 + i) & 31;
            const int kd = __shfl_sync(FULL_MASK, kind, src);
            const size_t ro = __shfl_sync(FULL_MASK, rowoff, src);
            const float A = __shfl_sync(FULL_MASK, ca, src);
            const float Bc = __shfl_sync(FULL_MASK, cb, src);
            if (i < ng) {
              if (kd == 0) {
#pragma unroll
                for (int q = 0; q < NQ; ++q) {
                  m[q].x = fmaf(A, m[q].x, Bc * vv[i][q].x);
                  m[q].y = fmaf(A, m[q].y, Bc * vv[i][q].y);
                  m[q].z = fmaf(A, m[q].z, Bc * vv[i][q].z);
                  m[q].w = fmaf(A, m[q].w, Bc * vv[i][q].w);
                }
                dirty = true;
              } else {
#pragma unroll
                for (int q = 0; q < NQ; ++q) {
                  const int c = lane + 32 * q;
                  if (c < d4) {
                    float4* dst = reinterpret_cast<float4*>(a.y + ro) + c;
                    atomicAdd(dst, make_float4(A * m[q].x, A * m[q].y, A * m[q].z, A * m[q].w));
                  }
                }
              }
            }
          }
        }
        e += cnt;
        if (cnt < 32) break;
      }
      if (dirty) {
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          const int c = lane + 32 * q;
          if (c < d4) reinterpret_cast<float4*>(row)[c] = m[q];
        }
      }
      __syncwarp();  // the ring slot is refilled by the next iteration's issue()
    }
    cp_async_wait<0>();
    __syncwarp();
  }
}

}  // namespace sdm
