// scan_chunk.cuh -- the chunk-wise prefill engine: steps 2 and 3 of the SDM pass over chunks
// of C tokens, parallel inside a chunk and recurrent from one chunk to the next.
//
// The m.163.com article on SDM (section 八, the paragraph on the training implementation)
// cuts the sequence into fixed-size chunks, computes inside a chunk in parallel and carries
// the state from chunk to chunk; the interaction of two tokens goes through the slots both
// selected, found by a two-pointer merge of their sorted slot lists in O(W) instead of O(W^2)
// (also the ai-feeds.com summary, section 方法).  Restated for the per-slot rule of the
// paper.rainbus.top summary (method steps 2-3): a write of slot i at token s maps
// M[i] -> a_s M[i] + b_s v_s with a_s = alpha_s (1 - beta_s k_s(i)), b_s = beta_s k_s(i), and
// slots not written keep their rows.  Inside a chunk that starts from state M0, with
// L(t, i) = sum of ln a_u(i) over the writes of slot i at tokens u <= t of the chunk,
//   M_t[i] = exp(L(t, i)) M0[i] + sum over writes of i at s <= t of
//            b_s(i) exp(L(t, i) - L(s, i)) v_s,
// so the read y_t = sum over read slots i of q_t(i) M_t[i] is
//   y_t = sum_i q_t(i) exp(L(t, i)) M0[i]  +  sum_{s <= t} A[t, s] v_s,
//   A[t, s] = sum over i in I_r(t) and I_w(s) of q_t(i) b_s(i) exp(L(t, i) - L(s, i)),
// A lower-triangular C x C matrix whose entries are sparse inner products of token t's read
// list and token s's write list (the two-pointer merge).  The chunk's end state is each
// written slot's writes applied to its M0 row.  ln a is floored at ln 1e-30, so a write with
// a = 0 (beta k = 1) stays finite; its later terms then carry e^-69 where the recurrence has
// 0.
//
// One CTA per (sequence, head, column slice of CW <= 128 values); the slices of a unit repeat
// the chunk's index work and split the rows.  Per chunk, in shared memory: the index lists
// and weights, each token's lists sorted by slot (rank by counting), L of every write and
// read (tokens in order, through a hash table of the chunk's written slots), A (a thread per
// (t, s) pair, two-pointer merge), v's slice; then y (a thread per (token, float4 column),
// the R read rows of M0 gathered from HBM), and the end state (a warp per slot whose last
// write in the chunk is this one, lanes over the slice, walking the slot's writes from the
// last to the first through a per-write link to the slot's previous write:
// M = (prod a) M0 + sum_s b_s (prod of the a after s) v_s).
#pragma once

#include "common.cuh"

namespace sdm {

constexpr int CHUNK_THREADS = 256;
constexpr int CHUNK_EMPTY = -1;
constexpr float CHUNK_LN_FLOOR = -69.0775528f;  // ln 1e-30

struct ChunkArgs {
  const int32_t* idx_w;  // [B*T*H, ldw] selection pre-pass
  const float* wt_w;
  const int32_t* idx_r;  // [B*T*H, ldr]
  const float* wt_r;
  const float* alpha;  // [B*T*H]
  const float* beta;
  const void* v;  // [B*T*H, d_v]
  float* M;       // [B*H, N, d_v]
  float* y;       // [B*T*H, d_v]
  int B, T, H, N, W, R, ldw, ldr, d_v, v_bf16;
  int C;   // tokens per chunk
  int CW;  // columns per slice (multiple of 4, divides d_v, <= 128)
  int hash_size;  // power of two >= 2 * C * W
};

// Shared-memory layout of one CTA (host and device agree on it).
struct ChunkLayout {
  size_t off_iw, off_ir, off_kw, off_qr, off_sw, off_sr, off_lw, off_lr, off_bb, off_aw,
      off_prev, off_A, off_v, off_ab, off_hkey, off_hl, off_hpos, total;
};

__host__ __device__ inline ChunkLayout chunk_layout(int C, int W, int R, int CW, int hash_size) {
  ChunkLayout L;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o += (bytes + 15) / 16 * 16;
    return at;
  };
  L.off_iw = take((size_t)C * W * 4);
  L.off_ir = take((size_t)C * R * 4);
  L.off_kw = take((size_t)C * W * 4);
  L.off_qr = take((size_t)C * R * 4);
  L.off_sw = take((size_t)C * W);  // sorted order of a token's writes (W <= 128)
  L.off_sr = take((size_t)C * R);
  L.off_lw = take((size_t)C * W * 4);
  L.off_lr = take((size_t)C * R * 4);
  L.off_bb = take((size_t)C * W * 4);
  L.off_aw = take((size_t)C * W * 4);
  L.off_prev = take((size_t)C * W * 4);
  L.off_A = take((size_t)C * C * 4);
  L.off_v = take((size_t)C * CW * 4);
  L.off_ab = take((size_t)C * 2 * 4);
  L.off_hkey = take((size_t)hash_size * 4);
  L.off_hl = take((size_t)hash_size * 4);
  L.off_hpos = take((size_t)hash_size * 4);
  L.total = o;
  return L;
}

__device__ __forceinline__ int chunk_hash(int s, int mask) {
  return static_cast<int>((static_cast<uint32_t>(s) * 2654435761u) >> 7) & mask;
}

// Slot s's entry of the chunk's hash table, inserted when absent (distinct threads insert
// distinct slots: the write slots of one token are distinct).
__device__ __forceinline__ int chunk_find_or_insert(int* key, int s, int mask) {
  int h = chunk_hash(s, mask);
  while (true) {
    const int k = atomicCAS(key + h, CHUNK_EMPTY, s);
    if (k == CHUNK_EMPTY || k == s) return h;
    h = (h + 1) & mask;
  }
}

__device__ __forceinline__ int chunk_find(const int* key, int s, int mask) {
  int h = chunk_hash(s, mask);
  while (true) {
    const int k = key[h];
    if (k == s) return h;
    if (k == CHUNK_EMPTY) return -1;
    h = (h + 1) & mask;
  }
}

__global__ void __launch_bounds__(CHUNK_THREADS) chunk_scan_kernel(ChunkArgs a) {
  // wait for the kernel ahead in the stream (programmatic launch), then let the next one in
  grid_dependency_wait();
  grid_launch_dependents();
  extern __shared__ __align__(16) unsigned char smem[];
  const int nslices = a.d_v / a.CW;
  const int slice = blockIdx.x % nslices;
  const int bh = blockIdx.x / nslices;
  const int b = bh / a.H, h = bh % a.H;
  const int col0 = slice * a.CW;
  const int C = a.C, W = a.W, R = a.R, CW = a.CW, cw4 = a.CW / 4;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int mask = a.hash_size - 1;
  const ChunkLayout L = chunk_layout(C, W, R, CW, a.hash_size);
  int* iw = reinterpret_cast<int*>(smem + L.off_iw);
  int* ir = reinterpret_cast<int*>(smem + L.off_ir);
  float* kw = reinterpret_cast<float*>(smem + L.off_kw);
  float* qr = reinterpret_cast<float*>(smem + L.off_qr);
  uint8_t* sw = smem + L.off_sw;
  uint8_t* sr = smem + L.off_sr;
  float* lw = reinterpret_cast<float*>(smem + L.off_lw);
  float* lr = reinterpret_cast<float*>(smem + L.off_lr);
  float* bb = reinterpret_cast<float*>(smem + L.off_bb);
  float* aw = reinterpret_cast<float*>(smem + L.off_aw);
  int* prev = reinterpret_cast<int*>(smem + L.off_prev);  // the slot's previous write, or -1
  float* A = reinterpret_cast<float*>(smem + L.off_A);
  float* vs = reinterpret_cast<float*>(smem + L.off_v);
  float* ab = reinterpret_cast<float*>(smem + L.off_ab);
  int* hkey = reinterpret_cast<int*>(smem + L.off_hkey);
  float* hl = reinterpret_cast<float*>(smem + L.off_hl);
  int* hpos = reinterpret_cast<int*>(smem + L.off_hpos);  // the slot's last write t * W + j
  float* Mbh = a.M + (size_t)bh * a.N * a.d_v;
  const size_t row0 = (size_t)b * a.T * a.H + h;  // (b, t = 0, h) row of [B,T,H]

  for (int c0 = 0; c0 < a.T; c0 += C) {
    const int n = min(C, a.T - c0);
    // 1. the chunk's index lists, weights, gates and v slice; an empty hash table
    for (int e = tid; e < n * W; e += CHUNK_THREADS) {
      const int t = e / W, j = e - t * W;
      const size_t r = row0 + (size_t)(c0 + t) * a.H;
      int s = a.idx_w[r * a.ldw + j];
      if (static_cast<unsigned>(s) >= static_cast<unsigned>(a.N)) {
        record_status(STATUS_BAD_INDEX);
        s = 0;
      }
      iw[e] = s;
      kw[e] = a.wt_w[r * a.ldw + j];
    }
    for (int e = tid; e < n * R; e += CHUNK_THREADS) {
      const int t = e / R, j = e - t * R;
      const size_t r = row0 + (size_t)(c0 + t) * a.H;
      int s = a.idx_r[r * a.ldr + j];
      if (static_cast<unsigned>(s) >= static_cast<unsigned>(a.N)) {
        record_status(STATUS_BAD_INDEX);
        s = 0;
      }
      ir[e] = s;
      qr[e] = a.wt_r[r * a.ldr + j];
    }
    for (int t = tid; t < n; t += CHUNK_THREADS) {
      const size_t r = row0 + (size_t)(c0 + t) * a.H;
      ab[2 * t] = a.alpha[r];
      ab[2 * t + 1] = a.beta[r];
    }
    for (int e = tid; e < n * cw4; e += CHUNK_THREADS) {
      const int t = e / cw4, c4 = e - t * cw4;
      const size_t off = (row0 + (size_t)(c0 + t) * a.H) * a.d_v + col0 + 4 * c4;
      float4 x;
      if (a.v_bf16) {
        const uint2 raw = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(a.v) + off);
        x = make_float4(__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xffff0000u),
                        __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xffff0000u));
      } else {
        x = *reinterpret_cast<const float4*>(static_cast<const float*>(a.v) + off);
      }
      reinterpret_cast<float4*>(vs)[e] = x;
    }
    for (int e = tid; e < a.hash_size; e += CHUNK_THREADS) {
      hkey[e] = CHUNK_EMPTY;
      hpos[e] = -1;
    }
    __syncthreads();

    // 2. each token's lists in slot order (rank by counting; a token's slots are distinct)
    for (int e = tid; e < n * W; e += CHUNK_THREADS) {
      const int t = e / W, j = e - t * W;
      const int s = iw[e];
      int rank = 0;
      for (int k = 0; k < W; ++k) rank += iw[t * W + k] < s;
      sw[t * W + rank] = static_cast<uint8_t>(j);
    }
    for (int e = tid; e < n * R; e += CHUNK_THREADS) {
      const int t = e / R, j = e - t * R;
      const int s = ir[e];
      int rank = 0;
      for (int k = 0; k < R; ++k) rank += ir[t * R + k] < s;
      sr[t * R + rank] = static_cast<uint8_t>(j);
    }
    // 3. L of every write and read, token after token through the hash table of written
    //    slots; the write coefficients a and b
    for (int t = 0; t < n; ++t) {
      const float al = ab[2 * t], be = ab[2 * t + 1];
      for (int j = tid; j < W; j += CHUNK_THREADS) {
        const float k = kw[t * W + j];
        const float kb = be * k;
        const float aa = al * (1.0f - kb);
        const float la = fmaxf(logf(fmaxf(aa, 0.0f)), CHUNK_LN_FLOOR);
        const int hs = chunk_find_or_insert(hkey, iw[t * W + j], mask);
        const int last = hpos[hs];
        const float lsum = (last < 0 ? 0.0f : hl[hs]) + la;  // first write: L = ln a
        hl[hs] = lsum;
        hpos[hs] = t * W + j;
        prev[t * W + j] = last;
        lw[t * W + j] = lsum;
        bb[t * W + j] = kb;
        aw[t * W + j] = aa;
      }
      __syncthreads();
      for (int j = tid; j < R; j += CHUNK_THREADS) {
        const int hs = chunk_find(hkey, ir[t * R + j], mask);
        lr[t * R + j] = hs >= 0 ? hl[hs] : 0.0f;
      }
      __syncthreads();
    }
    // 4. A[t, s], s <= t: sparse inner products by a two-pointer merge of the sorted lists
    for (int p = tid; p < n * n; p += CHUNK_THREADS) {
      const int t = p / n, s = p - t * n;
      float acc = 0.0f;
      if (s <= t) {
        int x = 0, z = 0;
        while (x < R && z < W) {
          const int jr = sr[t * R + x], jw = sw[s * W + z];
          const int rs = ir[t * R + jr], ws = iw[s * W + jw];
          if (rs < ws) {
            ++x;
          } else if (rs > ws) {
            ++z;
          } else {
            acc = fmaf(qr[t * R + jr] * bb[s * W + jw],
                       expf(lr[t * R + jr] - lw[s * W + jw]), acc);
            ++x;
            ++z;
          }
        }
      }
      A[t * C + s] = acc;
    }
    __syncthreads();
    // 5. y_t = sum_i q_t(i) e^{L(t,i)} M0[i] + sum_{s <= t} A[t, s] v_s, a thread per
    //    (token, float4 column) of the slice
    for (int e = tid; e < n * cw4; e += CHUNK_THREADS) {
      const int t = e / cw4, c4 = e - t * cw4;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int j = 0; j < R; ++j) {
        const float w = qr[t * R + j] * expf(lr[t * R + j]);
        const float4 m = __ldg(reinterpret_cast<const float4*>(
            Mbh + (size_t)ir[t * R + j] * a.d_v + col0) + c4);
        acc.x = fmaf(w, m.x, acc.x);
        acc.y = fmaf(w, m.y, acc.y);
        acc.z = fmaf(w, m.z, acc.z);
        acc.w = fmaf(w, m.w, acc.w);
      }
      for (int s = 0; s <= t; ++s) {
        const float w = A[t * C + s];
        const float4 x = reinterpret_cast<const float4*>(vs)[s * cw4 + c4];
        acc.x = fmaf(w, x.x, acc.x);
        acc.y = fmaf(w, x.y, acc.y);
        acc.z = fmaf(w, x.z, acc.z);
        acc.w = fmaf(w, x.w, acc.w);
      }
      reinterpret_cast<float4*>(a.y + (row0 + (size_t)(c0 + t) * a.H) * a.d_v + col0)[c4] = acc;
    }
    __syncthreads();  // every read of M0 is done before the chunk's rows are rewritten
    // 6. end state: the warp of a slot's last write in the chunk walks the slot's writes
    //    back to the first (lanes over the slice's float4 columns):
    //    M = P M0 + acc, acc = sum_s b_s (prod of the a after s) v_s, P = prod a
    for (int e = warp; e < n * W; e += CHUNK_THREADS / 32) {
      const int s = iw[e];
      if (hpos[chunk_find(hkey, s, mask)] != e) continue;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      float P = 1.0f;
      for (int p = e; p >= 0; p = prev[p]) {
        const float Bp = P * bb[p];
        if (lane < cw4) {
          const float4 x = reinterpret_cast<const float4*>(vs)[(p / W) * cw4 + lane];
          acc.x = fmaf(Bp, x.x, acc.x);
          acc.y = fmaf(Bp, x.y, acc.y);
          acc.z = fmaf(Bp, x.z, acc.z);
          acc.w = fmaf(Bp, x.w, acc.w);
        }
        P *= aw[p];
      }
      if (lane < cw4) {
        float4* row = reinterpret_cast<float4*>(Mbh + (size_t)s * a.d_v + col0);
        const float4 m0 = row[lane];
        row[lane] = make_float4(fmaf(P, m0.x, acc.x), fmaf(P, m0.y, acc.y),
                                fmaf(P, m0.z, acc.z), fmaf(P, m0.w, acc.w));
      }
    }
    __syncthreads();  // the next chunk reads the rows written here and reuses the buffers
  }
}

}  // namespace sdm
