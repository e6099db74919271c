// decode.cuh -- one decode step of the SDM pass for every (sequence, head), fused.
//
// Method: "Sparse Delta Memory: Scaling the State of Linear RNNs through Sparsity"
// (paper.rainbus.top summary), method steps 1-4, applied to a single token; the m.163.com
// article on SDM (section 八) reports decode as the setting where the HBM-resident
// memory costs most.  One CTA per (b, h):
//   warps 0 and 1 select the write and the read slots (step 1) while the other warps
//   stage v, alpha, beta and the gate;
//   every warp then rewrites its share of the W write rows (step 2) and keeps the new
//   rows in shared memory; read rows outside the write set are loaded in the same pass;
//   after a barrier, read rows inside the write set come from shared memory (step 3);
//   the CTA sums the R weighted rows, then normalises and gates them (step 4).
#pragma once

#include "common.cuh"
#include "select.cuh"

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
  size_t off_tab_w, off_tab_r, off_sel_w, off_sel_r, off_list, off_vec, off_wrows, off_part,
      total;
};

__host__ __device__ inline DecLayout dec_layout(int S1, int S2, int W, int R, int d_v) {
  DecLayout L;
  const int kmax = W > R ? W : R;
  L.off_tab_w = 0;
  L.off_tab_r = L.off_tab_w + (size_t)((cand_count(W) + 7) / 8) * 16;
  L.off_sel_w = L.off_tab_r + (size_t)((cand_count(R) + 7) / 8) * 16;
  L.off_sel_r = L.off_sel_w + sel_scratch_bytes(S1, S2, kmax);
  L.off_list = L.off_sel_r + sel_scratch_bytes(S1, S2, kmax);
  // idx_w[KMAX], wt_w[KMAX], idx_r[KMAX], wt_r[KMAX]
  L.off_vec = L.off_list + 4 * (size_t)KMAX * 4;
  // v[d_v], gate[d_v] as fp32, alpha, beta, ssq partials
  L.off_wrows = L.off_vec + ((size_t)(2 * d_v + 16 + DEC_WARPS) * 4 + 15) / 16 * 16;
  L.off_part = L.off_wrows + (size_t)W * d_v * 4;
  L.total = L.off_part + (size_t)DEC_WARPS * d_v * 4;
  return L;
}

__global__ void __launch_bounds__(DEC_THREADS) decode_kernel(DecodeArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int bh = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const DecLayout L = dec_layout(a.S1, a.S2, a.W, a.R, a.d_v);
  const int kmax = a.W > a.R ? a.W : a.R;
  const int S = a.S1 + a.S2;
  const int d4 = a.d_v / 4;
  const bool bf16 = a.in_bf16 != 0;
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
  float* wrows = reinterpret_cast<float*>(smem + L.off_wrows);  // [W][d_v]
  float* part = reinterpret_cast<float*>(smem + L.off_part);    // [DEC_WARPS][d_v]

  build_cand_table(tab_w, a.W, tid, DEC_THREADS);
  build_cand_table(tab_r, a.R, tid, DEC_THREADS);
  __syncthreads();

  // step 1 on warps 0 (write) and 1 (read); the rest stage the per-token vectors
  if (warp < 2) {
    SelScratch sc = carve_sel_scratch(smem + (warp == 0 ? L.off_sel_w : L.off_sel_r), a.S1,
                                      a.S2, kmax);
    const void* src = reinterpret_cast<const unsigned char*>(warp == 0 ? a.kp : a.qp) +
                      (size_t)bh * S * esz;
    select_row(src, bf16, a.S1, a.S2, warp == 0 ? a.W : a.R, warp == 0 ? tab_w : tab_r, sc,
               lane, warp == 0 ? idx_w : idx_r, warp == 0 ? wt_w : wt_r);
  } else {
    for (int c = tid - 64; c < a.d_v; c += DEC_THREADS - 64) {
      vs[c] = load_in(a.v, (size_t)bh * a.d_v + c, bf16);
      gs[c] = a.gate ? gate_act(load_in(a.gate, (size_t)bh * a.d_v + c, bf16), a.act) : 1.0f;
    }
    if (tid == 64) {
      ab[0] = a.alpha[bh];
      ab[1] = a.beta[bh];
    }
  }
  __syncthreads();

  if (a.sel_out) {
    for (int j = tid; j < a.W; j += DEC_THREADS) a.sel_out[(size_t)bh * a.W + j] = idx_w[j];
    for (int j = tid; j < a.R; j += DEC_THREADS)
      a.sel_out[(size_t)a.BH * a.W + (size_t)bh * a.R + j] = idx_r[j];
  }

  float* Mbh = a.M + (size_t)bh * a.N * a.d_v;
  const float al = ab[0], be = ab[1];

  // step 2: every warp rewrites write rows warp, warp + 8, ...; its read rows that are
  // not in the write set are loaded alongside and accumulated right away.
  constexpr int NQ = 8;  // float4 columns per lane: d_v <= 1024
  float4 acc[NQ];
#pragma unroll
  for (int q = 0; q < NQ; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = warp; j < a.W; j += DEC_WARPS) {
    const int s = idx_w[j];
    if (static_cast<unsigned>(s) >= static_cast<unsigned>(a.N)) {
      if (lane == 0) record_status(STATUS_BAD_INDEX);
      continue;
    }
    const float kb = be * wt_w[j];
    const float ka = al * (1.0f - kb);
    float4* row = reinterpret_cast<float4*>(Mbh + (size_t)s * a.d_v);
    float4* keep = reinterpret_cast<float4*>(wrows + (size_t)j * a.d_v);
    const float4* v4 = reinterpret_cast<const float4*>(vs);
    for (int c = lane; c < d4; c += 32) {
      const float4 old = row[c];
      const float4 vv = v4[c];
      float4 nw;
      nw.x = fmaf(ka, old.x, kb * vv.x);
      nw.y = fmaf(ka, old.y, kb * vv.y);
      nw.z = fmaf(ka, old.z, kb * vv.z);
      nw.w = fmaf(ka, old.w, kb * vv.w);
      row[c] = nw;
      keep[c] = nw;
    }
  }
  // read rows outside the write set
  for (int j = warp; j < a.R; j += DEC_WARPS) {
    const int s = idx_r[j];
    bool in_w = false;
    for (int e = lane; e < a.W; e += 32) in_w |= (idx_w[e] == s);
    if (__any_sync(FULL_MASK, in_w)) continue;
    if (static_cast<unsigned>(s) >= static_cast<unsigned>(a.N)) {
      if (lane == 0) record_status(STATUS_BAD_INDEX);
      continue;
    }
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
  __syncthreads();
  // step 3 for read rows inside the write set: the rows this token just wrote
  for (int j = warp; j < a.R; j += DEC_WARPS) {
    const int s = idx_r[j];
    int pos = -1;
    for (int e = lane; e < a.W; e += 32)
      if (idx_w[e] == s) pos = e;
    const unsigned m = __ballot_sync(FULL_MASK, pos >= 0);
    if (!m) continue;
    pos = __shfl_sync(FULL_MASK, pos, __ffs(m) - 1);
    const float q = wt_r[j];
    const float4* row = reinterpret_cast<const float4*>(wrows + (size_t)pos * a.d_v);
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
