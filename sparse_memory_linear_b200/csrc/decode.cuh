// decode.cuh -- one decode step of the SDM pass for every (sequence, head), fused.
//
// Method: "Sparse Delta Memory: Scaling the State of Linear RNNs through Sparsity"
// (paper.rainbus.top summary), method steps 1-4, applied to a single token; the m.163.com
// article on SDM (section 八) reports decode as the setting where the HBM-resident
// memory costs most.  One CTA per (b, h):
//   four warps select the four score halves (write and read, first and second half) and
//   two of them then combine the candidate sums (step 1), while the other warps stage v,
//   alpha, beta and the gate;
//   every warp then rewrites its share of the W write rows (step 2) and, in the same
//   pass, reads the read rows that this token does not write; after a barrier the read
//   rows inside the write set are read back (this CTA's own stores) (step 3);
//   the CTA sums the R weighted rows, then normalises and gates them (step 4).
// About 33 KB of shared memory per CTA keeps a 64 x 8 batch in one wave.
#pragma once

#include "common.cuh"
#include "select.cuh"
#include "select_fast.cuh"

namespace sdm {

struct DecodeArgs {
  const void* kp;  // [B*H, S1+S2]
  const void* qp;
  const void* v;     // [B*H, d_v]
  const float* alpha;  // [B*H]
  const float* beta;
  float* M;            // [B*H, N, d_v]
  float* y;            // [B*H, d_v]
  const void* gate;    // [B*H, d_v] or null
  const float* gamma;  // [d_v] or null
  float* o;            // [B*H, d_v] or null
  int32_t* sel_out;    // [B*H*W] then [B*H*R], or null
  float eps;
  int act;
  int BH, S1, S2, W, R, N, d_v, in_bf16;
};

constexpr int DEC_THREADS = 256;
constexpr int DEC_WARPS = DEC_THREADS / 32;

struct DecLayout {
  size_t off_tab_w, off_tab_r, off_sel, sel_stride, off_list, off_vec, off_part, total;
  bool fast;
};

// Shared-memory plan: the two candidate tables, four selection scratch areas (fast path:
// one per score half; general path: one per selection), the selected lists, v / gate /
// gates and the per-warp partial reads.
__host__ __device__ inline DecLayout dec_layout(int S1, int S2, int W, int R, int d_v, bool fast,
                                                int kc) {
  DecLayout L;
  const int kmax = W > R ? W : R;
  L.fast = fast;
  L.off_tab_w = 0;
  L.off_tab_r = L.off_tab_w + (size_t)((cand_count(W) + 7) / 8) * 16;
  L.off_sel = L.off_tab_r + (size_t)((cand_count(R) + 7) / 8) * 16;
  L.sel_stride = fast ? fast_scratch_bytes(S1, S2, kc) : sel_scratch_bytes(S1, S2, kmax);
  L.sel_stride = (L.sel_stride + 15) / 16 * 16;
  L.off_list = L.off_sel + (L.fast ? 4 : 2) * L.sel_stride;
  // idx_w[KMAX], wt_w[KMAX], idx_r[KMAX], wt_r[KMAX]
  L.off_vec = L.off_list + 4 * (size_t)KMAX * 4;
  // v[d_v], act(gate)[d_v], alpha, beta, ssq partials
  L.off_part = L.off_vec + ((size_t)(2 * d_v + 16 + DEC_WARPS) * 4 + 15) / 16 * 16;
  L.total = L.off_part + (size_t)DEC_WARPS * d_v * 4;
  return L;
}

// Step 1 of one token on the CTA's warps.  Fast path: warps 0-3 take the four score halves
// (write first, write second, read first, read second), then warps 0 and 2 combine the
// candidates of the write and the read selection.  General path: warps 0 and 1.
template <int R8, int KC>
__device__ __forceinline__ void decode_select_fast(const DecodeArgs& a, const DecLayout& L,
                                                   unsigned char* smem, int warp, int lane,
                                                   int32_t* idx_w, float* wt_w, int32_t* idx_r,
                                                   float* wt_r) {
  const int S = a.S1 + a.S2;
  if (warp < 4) {
    const bool rd = warp >= 2;
    const bool second = warp & 1;
    const __nv_bfloat16* row =
        reinterpret_cast<const __nv_bfloat16*>(rd ? a.qp : a.kp) + (size_t)blockIdx.x * S;
    const int K = rd ? a.R : a.W;
    FastScratch own = carve_fast_scratch(smem + L.off_sel + warp * L.sel_stride, a.S1, a.S2, KC);
    FastScratch pair =
        carve_fast_scratch(smem + L.off_sel + (rd ? 2 : 0) * L.sel_stride, a.S1, a.S2, KC);
    half_topk_bf16<R8, KC>(second ? row + a.S1 : row, second ? a.S2 : a.S1, K, lane, own.surv,
                           own.stage, second ? pair.b : pair.a);
  }
  __syncthreads();
  if (warp == 0 || warp == 2) {
    const bool rd = warp == 2;
    FastScratch pair = carve_fast_scratch(smem + L.off_sel + warp * L.sel_stride, a.S1, a.S2, KC);
    cand_topk_bf16<KC>(pair.a, pair.b, rd ? a.R : a.W, a.S2,
                       reinterpret_cast<const uint16_t*>(smem + (rd ? L.off_tab_r : L.off_tab_w)),
                       lane, pair.pv, reinterpret_cast<uint64_t*>(pair.stage),
                       rd ? idx_r : idx_w, rd ? wt_r : wt_w);
  }
}

// R8 == 0 takes the general selection (fp32 halves, halves longer than 1024 values);
// otherwise the fast path for halves of up to 256*R8 values and K <= KC.  NQ float4 columns
// per lane: d_v <= 128*NQ.
template <int R8, int KC, int NQ>
__global__ void __launch_bounds__(DEC_THREADS, 4) decode_kernel(DecodeArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int bh = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool bf16 = a.in_bf16 != 0;
  const DecLayout L = dec_layout(a.S1, a.S2, a.W, a.R, a.d_v, R8 > 0, KC);
  const int kmax = a.W > a.R ? a.W : a.R;
  const int S = a.S1 + a.S2;
  const int d4 = a.d_v / 4;
  const size_t esz = bf16 ? 2 : 4;

  uint16_t* tab_w = reinterpret_cast<uint16_t*>(smem + L.off_tab_w);
  uint16_t* tab_r = reinterpret_cast<uint16_t*>(smem + L.off_tab_r);
  int32_t* idx_w = reinterpret_cast<int32_t*>(smem + L.off_list);
  float* wt_w = reinterpret_cast<float*>(idx_w + KMAX);
  int32_t* idx_r = reinterpret_cast<int32_t*>(wt_w + KMAX);
  float* wt_r = reinterpret_cast<float*>(idx_r + KMAX);
  float* vs = reinterpret_cast<float*>(smem + L.off_vec);  // [d_v]
  float* gs = vs + a.d_v;                                  // [d_v]
  float* ab = gs + a.d_v;                                  // alpha, beta
  float* ssq = ab + 16;                                    // [DEC_WARPS]
  float* part = reinterpret_cast<float*>(smem + L.off_part);  // [DEC_WARPS][d_v]

  build_cand_table(tab_w, a.W, tid, DEC_THREADS);
  build_cand_table(tab_r, a.R, tid, DEC_THREADS);
  // the per-token vectors, staged by the warps that do not select
  const int first_free = R8 > 0 ? 4 : 2;
  if (warp >= first_free) {
    const int t0 = tid - 32 * first_free, nt = DEC_THREADS - 32 * first_free;
    for (int c = t0; c < a.d_v; c += nt) {
      vs[c] = load_in(a.v, (size_t)bh * a.d_v + c, bf16);
      gs[c] = a.gate ? gate_act(load_in(a.gate, (size_t)bh * a.d_v + c, bf16), a.act) : 1.0f;
    }
    if (t0 == 0) {
      ab[0] = a.alpha[bh];
      ab[1] = a.beta[bh];
    }
  }
  __syncthreads();

  // step 1
  if (R8 > 0) {
    decode_select_fast<(R8 > 0 ? R8 : 1), KC>(a, L, smem, warp, lane, idx_w, wt_w, idx_r, wt_r);
  } else if (warp < 2) {
    SelScratch sc = carve_sel_scratch(smem + L.off_sel + warp * L.sel_stride, a.S1, a.S2, kmax);
    const void* src = reinterpret_cast<const unsigned char*>(warp == 0 ? a.kp : a.qp) +
                      (size_t)bh * S * esz;
    select_row(src, bf16, a.S1, a.S2, warp == 0 ? a.W : a.R, warp == 0 ? tab_w : tab_r, sc,
               lane, warp == 0 ? idx_w : idx_r, warp == 0 ? wt_w : wt_r);
  }
  __syncthreads();

  if (a.sel_out) {
    for (int j = tid; j < a.W; j += DEC_THREADS) a.sel_out[(size_t)bh * a.W + j] = idx_w[j];
    for (int j = tid; j < a.R; j += DEC_THREADS)
      a.sel_out[(size_t)a.BH * a.W + (size_t)bh * a.R + j] = idx_r[j];
  }

  float* Mbh = a.M + (size_t)bh * a.N * a.d_v;
  const float al = ab[0], be = ab[1];
  float4 acc[NQ];
#pragma unroll
  for (int q = 0; q < NQ; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);

  // step 2: this warp's write rows (warp, warp + 8, ...), RB at a time: every row load is
  // issued before any update, so a warp waits for one memory latency per RB rows
  constexpr int RB = 8 / NQ;
  for (int j0 = warp; j0 < a.W; j0 += DEC_WARPS * RB) {
    float4 old[RB][NQ];
    int slot[RB];
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      const int j = j0 + r * DEC_WARPS;
      slot[r] = j < a.W ? idx_w[j] : -1;
      if (j < a.W && static_cast<unsigned>(slot[r]) < static_cast<unsigned>(a.N)) {
        const float4* row = reinterpret_cast<const float4*>(Mbh + (size_t)slot[r] * a.d_v);
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          const int c = lane + 32 * q;
          if (c < d4) old[r][q] = row[c];
        }
      }
    }
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      const int j = j0 + r * DEC_WARPS;
      if (j >= a.W) continue;
      if (static_cast<unsigned>(slot[r]) >= static_cast<unsigned>(a.N)) {
        if (lane == 0) record_status(STATUS_BAD_INDEX);
        continue;
      }
      const float kb = be * wt_w[j];
      const float ka = al * (1.0f - kb);
      float4* row = reinterpret_cast<float4*>(Mbh + (size_t)slot[r] * a.d_v);
      const float4* v4 = reinterpret_cast<const float4*>(vs);
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const int c = lane + 32 * q;
        if (c < d4) {
          const float4 vv = v4[c];
          float4 nw;
          nw.x = fmaf(ka, old[r][q].x, kb * vv.x);
          nw.y = fmaf(ka, old[r][q].y, kb * vv.y);
          nw.z = fmaf(ka, old[r][q].z, kb * vv.z);
          nw.w = fmaf(ka, old[r][q].w, kb * vv.w);
          row[c] = nw;
        }
      }
    }
  }
  // step 3 for the read rows this token does not write (no dependence on step 2), RB at a
  // time in the same way
  for (int j0 = warp; j0 < a.R; j0 += DEC_WARPS * RB) {
    float4 val[RB][NQ];
    bool use[RB];
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      const int j = j0 + r * DEC_WARPS;
      const int s = j < a.R ? idx_r[j] : -1;
      bool in_w = false;
      if (j < a.R)
        for (int e = lane; e < a.W; e += 32) in_w |= (idx_w[e] == s);
      in_w = __any_sync(FULL_MASK, in_w);
      use[r] = j < a.R && !in_w;
      if (use[r] && static_cast<unsigned>(s) >= static_cast<unsigned>(a.N)) {
        if (lane == 0) record_status(STATUS_BAD_INDEX);
        use[r] = false;
      }
      if (use[r]) {
        const float4* row = reinterpret_cast<const float4*>(Mbh + (size_t)s * a.d_v);
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          const int c = lane + 32 * q;
          if (c < d4) val[r][q] = row[c];
        }
      }
    }
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      if (!use[r]) continue;
      const float q = wt_r[j0 + r * DEC_WARPS];
#pragma unroll
      for (int qq = 0; qq < NQ; ++qq) {
        const int c = lane + 32 * qq;
        if (c < d4) {
          acc[qq].x = fmaf(q, val[r][qq].x, acc[qq].x);
          acc[qq].y = fmaf(q, val[r][qq].y, acc[qq].y);
          acc[qq].z = fmaf(q, val[r][qq].z, acc[qq].z);
          acc[qq].w = fmaf(q, val[r][qq].w, acc[qq].w);
        }
      }
    }
  }
  __syncthreads();
  // step 3 for read rows inside the write set: this CTA's own stores, visible after the
  // barrier
  for (int j = warp; j < a.R; j += DEC_WARPS) {
    const int s = idx_r[j];
    bool in_w = false;
    for (int e = lane; e < a.W; e += 32) in_w |= (idx_w[e] == s);
    if (!__any_sync(FULL_MASK, in_w)) continue;
    const float q = wt_r[j];
    const float4* row = reinterpret_cast<const float4*>(Mbh + (size_t)s * a.d_v);
#pragma unroll
    for (int qq = 0; qq < NQ; ++qq) {
      const int c = lane + 32 * qq;
      if (c < d4) {
        const float4 val = row[c];
        acc[qq].x = fmaf(q, val.x, acc[qq].x);
        acc[qq].y = fmaf(q, val.y, acc[qq].y);
        acc[qq].z = fmaf(q, val.z, acc[qq].z);
        acc[qq].w = fmaf(q, val.w, acc[qq].w);
      }
    }
  }
#pragma unroll
  for (int qq = 0; qq < NQ; ++qq) {
    const int c = lane + 32 * qq;
    if (c < d4) reinterpret_cast<float4*>(part + (size_t)warp * a.d_v)[c] = acc[qq];
  }
  __syncthreads();

  // y and step 4
  float yv[4];
  float ss = 0.0f;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int c = tid + DEC_THREADS * q;
    yv[q] = 0.0f;
    if (c < a.d_v) {
      float s = 0.0f;
      for (int w = 0; w < DEC_WARPS; ++w) s += part[(size_t)w * a.d_v + c];
      yv[q] = s;
      a.y[(size_t)bh * a.d_v + c] = s;
      ss = fmaf(s, s, ss);
    }
  }
  if (a.o) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(FULL_MASK, ss, o);
    if (lane == 0) ssq[warp] = ss;
    __syncthreads();
    float tot = 0.0f;
    for (int w = 0; w < DEC_WARPS; ++w) tot += ssq[w];
    const float inv = rsqrtf(tot / static_cast<float>(a.d_v) + a.eps);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = tid + DEC_THREADS * q;
      if (c < a.d_v) {
        const float gm = a.gamma ? a.gamma[c] : 1.0f;
        a.o[(size_t)bh * a.d_v + c] = yv[q] * inv * gm * gs[c];
      }
    }
  }
}

}  // namespace sdm
