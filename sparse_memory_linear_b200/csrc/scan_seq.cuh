// scan_seq.cuh -- the token-sequential engine of steps 2 and 3 of the SDM pass.
//
// Method: "Sparse Delta Memory: Scaling the State of Linear RNNs through Sparsity"
// (paper.rainbus.top summary), method steps 2 and 3; ai-paper-analysis.pages.dev SDM
// write-up, 步骤 2 and 步骤 3.  For token t, on each selected write slot i only:
//   M~[i] = alpha_t M[i];  M[i] = M~[i] + beta_t k_i (v_t - M~[i])
// which is M[i] = a M[i] + b v_t with a = alpha_t (1 - beta_t k_i), b = beta_t k_i; then
// y_t = sum over the read slots of q_i M[i], after the write.
//
// Design.  Every value column of M evolves independently (alpha, beta and the weights
// are scalars), so one CTA owns a (sequence, head, column slice of CW floats) and walks
// the tokens in order.  The selection of every token is known before the pass starts
// (it never depends on M), so the CTA gathers the rows of token u + D into shared memory
// with cp.async while it works on token u, and the index lists of token u + 2D one stage
// earlier still.  A prefetched row is stale if one of the D tokens in between wrote the
// same slot; a small table (slot hash -> last token that wrote a slot of that hash)
// flags those rows, and the flagged rows take their value from the writer's stage,
// which stays in shared memory for D more tokens.  The same forwarding gives the read
// of token u the rows that token u itself has just written.
#pragma once

#include "common.cuh"

namespace sdm {

struct SeqArgs {
  const int32_t* idx_w;  // [B*T*H, ldw]
  const float* wt_w;
  const int32_t* idx_r;  // [B*T*H, ldr]
  const float* wt_r;
  const float* alpha;  // [B*T*H]
  const float* beta;
  const void* v;       // [B*T*H, d_v]
  float* M;            // [B*H, N, d_v]
  float* y;            // [B*T*H, d_v]
  int B, T, H, N, W, R, ldw, ldr, d_v, v_bf16;
  int coupled;  // 1: the coupled delta rule (one prediction shared by the written rows)
  float* wlog;  // [B*T*H, W, d_v] undo log of the per-slot rule (each written row as its
                // write found it), or null
};

constexpr int SEQ_THREADS = 256;
constexpr int SEQ_HASH_BITS = 13;
constexpr int SEQ_HASH = 1 << SEQ_HASH_BITS;

__device__ __forceinline__ int seq_hash(int s) {
  return static_cast<int>((static_cast<uint32_t>(s) * 2654435761u) >> (32 - SEQ_HASH_BITS));
}

// Shared-memory layout of the engine (host and device agree on it).
struct SeqLayout {
  int meta_bytes;  // one token's index lists, weights, gates and v slice
  int off_idx_r, off_wt_w, off_wt_r, off_ab, off_v;
  int stage_bytes;  // one token's gathered rows
  int NM, NR;
  size_t off_meta, off_stage, off_hash, off_red, total;
};

__host__ __device__ inline SeqLayout seq_layout(int ldw, int ldr, int CW, int v_esz, int D) {
  SeqLayout L;
  L.off_idx_r = ldw * 4;
  L.off_wt_w = L.off_idx_r + ldr * 4;
  L.off_wt_r = L.off_wt_w + ldw * 4;
  L.off_ab = L.off_wt_r + ldr * 4;
  L.off_v = L.off_ab + 16;
  L.meta_bytes = (L.off_v + CW * v_esz + 15) / 16 * 16;
  L.stage_bytes = (ldw + ldr) * CW * 4;
  L.NM = 3 * D;
  L.NR = 2 * D;
  L.off_meta = 0;
  L.off_stage = L.off_meta + (size_t)L.NM * L.meta_bytes;
  L.off_hash = L.off_stage + (size_t)L.NR * L.stage_bytes;
  L.off_red = L.off_hash + (size_t)SEQ_HASH * 4;
  L.total = L.off_red + (size_t)(SEQ_THREADS / 32) * CW * 4;
  return L;
}

template <int CW, int D>
__global__ void __launch_bounds__(SEQ_THREADS, 1) seq_scan_kernel(SeqArgs a) {
  // wait for the kernel ahead in the stream (programmatic launch), then let the next one in
  grid_dependency_wait();
  grid_launch_dependents();
  constexpr int LPR = CW / 4;             // lanes per row, one float4 each
  constexpr int NG = SEQ_THREADS / LPR;   // row groups
  constexpr int NW = SEQ_THREADS / 32;
  extern __shared__ __align__(16) unsigned char smem[];

  const int nslices = a.d_v / CW;
  const int slice = blockIdx.x % nslices;
  const int bh = blockIdx.x / nslices;
  const int b = bh / a.H, h = bh % a.H;
  const int col0 = slice * CW;
  const int tid = threadIdx.x;
  const int g = tid / LPR, lig = tid % LPR;
  const int lane = tid & 31, warp = tid >> 5;
  const unsigned gmask = (LPR == 32 ? FULL_MASK : ((1u << LPR) - 1u)) << (lane / LPR * LPR);
  const int v_esz = a.v_bf16 ? 2 : 4;
  const SeqLayout L = seq_layout(a.ldw, a.ldr, CW, v_esz, D);
  const int NM = L.NM, NR = L.NR;

  unsigned char* meta_base = smem + L.off_meta;
  float* stage_base = reinterpret_cast<float*>(smem + L.off_stage);
  int* tok_tab = reinterpret_cast<int*>(smem + L.off_hash);
  float* red = reinterpret_cast<float*>(smem + L.off_red);

  auto meta = [&](int t) { return meta_base + (size_t)(t % NM) * L.meta_bytes; };
  auto stage = [&](int t) { return stage_base + (size_t)(t % NR) * (L.stage_bytes / 4); };

  float* Mbh = a.M + (size_t)bh * a.N * a.d_v;
  const size_t tok_row0 = (size_t)b * a.T * a.H + h;  // (b, t=0, h) row of [B,T,H]

  for (int i = tid; i < SEQ_HASH; i += SEQ_THREADS) tok_tab[i] = -(1 << 30);

  // cp.async of token t's index lists, weights, gates and v slice into its meta slot
  auto issue_meta = [&](int t) {
    unsigned char* m = meta(t);
    const size_t row = tok_row0 + (size_t)t * a.H;
    const int cw = a.ldw / 4, cr = a.ldr / 4;  // 16-byte chunks
    const int cv = CW * v_esz / 16;
    const int total = 2 * (cw + cr) + cv;
    for (int c = tid; c < total; c += SEQ_THREADS) {
      const void* src;
      void* dst;
      if (c < cw) {
        src = a.idx_w + row * a.ldw + 4 * c;
        dst = m + 16 * c;
      } else if (c < cw + cr) {
        src = a.idx_r + row * a.ldr + 4 * (c - cw);
        dst = m + L.off_idx_r + 16 * (c - cw);
      } else if (c < 2 * cw + cr) {
        src = a.wt_w + row * a.ldw + 4 * (c - cw - cr);
        dst = m + L.off_wt_w + 16 * (c - cw - cr);
      } else if (c < 2 * (cw + cr)) {
        src = a.wt_r + row * a.ldr + 4 * (c - 2 * cw - cr);
        dst = m + L.off_wt_r + 16 * (c - 2 * cw - cr);
      } else {
        const int q = c - 2 * (cw + cr);
        src = reinterpret_cast<const unsigned char*>(a.v) +
              (row * a.d_v + col0) * v_esz + 16 * q;
        dst = m + L.off_v + 16 * q;
      }
      cp_async16(dst, src);
    }
    if (tid == 0) {
      unsigned s0 = static_cast<unsigned>(__cvta_generic_to_shared(m + L.off_ab));
      asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(s0), "l"(a.alpha + row)
                   : "memory");
      asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(s0 + 4), "l"(a.beta + row)
                   : "memory");
    }
  };

  // cp.async of token t's W write rows and R read rows (this slice) into its stage
  auto issue_rows = [&](int t) {
    const unsigned char* m = meta(t);
    const int32_t* iw = reinterpret_cast<const int32_t*>(m);
    const int32_t* ir = reinterpret_cast<const int32_t*>(m + L.off_idx_r);
    float* st = stage(t);
    for (int j = g; j < a.W + a.R; j += NG) {
      int s = j < a.W ? iw[j] : ir[j - a.W];
      if (static_cast<unsigned>(s) >= static_cast<unsigned>(a.N)) s = 0;  // flagged later
      const float* src = Mbh + (size_t)s * a.d_v + col0 + 4 * lig;
      const int srow = j < a.W ? j : a.ldw + (j - a.W);
      cp_async16(st + (size_t)srow * CW + 4 * lig, src);
    }
  };

  // latest token in [t_lo, t_hi] that wrote slot s, and the write row it used
  auto find_writer = [&](int s, int t_hi, int t_lo, int& tw, int& jw) -> bool {
    for (int t = t_hi; t >= t_lo && t >= 0; --t) {
      const int32_t* lst = reinterpret_cast<const int32_t*>(meta(t));
      int hit = -1;
      for (int e = lig; e < a.W; e += LPR)
        if (lst[e] == s) hit = e;
      const unsigned m = __ballot_sync(gmask, hit >= 0);
      if (m) {
        jw = __shfl_sync(gmask, hit, __ffs(m) - 1);
        tw = t;
        return true;
      }
    }
    return false;
  };

  // prologue: meta of tokens [0, D), then rows of [0, D) with meta of [D, 2D)
  for (int t = 0; t < D && t < a.T; ++t) issue_meta(t);
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();
  for (int i = 0; i < D; ++i) {
    if (i < a.T) issue_rows(i);
    if (D + i < a.T) issue_meta(D + i);
    cp_async_commit();
  }

  for (int u = 0; u < a.T; ++u) {
    cp_async_wait<D - 1>();
    __syncthreads();
    const unsigned char* m = meta(u);
    const int32_t* iw = reinterpret_cast<const int32_t*>(m);
    const int32_t* ir = reinterpret_cast<const int32_t*>(m + L.off_idx_r);
    const float* ww = reinterpret_cast<const float*>(m + L.off_wt_w);
    const float* wr = reinterpret_cast<const float*>(m + L.off_wt_r);
    const float al = reinterpret_cast<const float*>(m + L.off_ab)[0];
    const float be = reinterpret_cast<const float*>(m + L.off_ab)[1];
    float4 vv;
    if (a.v_bf16) {
      const __nv_bfloat162* vb = reinterpret_cast<const __nv_bfloat162*>(m + L.off_v) + 2 * lig;
      const float2 p0 = __bfloat1622float2(vb[0]), p1 = __bfloat1622float2(vb[1]);
      vv = make_float4(p0.x, p0.y, p1.x, p1.y);
    } else {
      vv = reinterpret_cast<const float4*>(m + L.off_v)[lig];
    }
    float* st = stage(u);

    if (a.coupled) {
      // step 2, coupled reading: pass 1 gathers this thread's old rows (forwarded where a
      // token of the window wrote them) and its share of the prediction
      // p = sum_j k_j alpha M[j]; the shares meet through shuffles and shared memory; pass 2
      // writes alpha M[j] + beta k_j (v - p)
      constexpr int RPT = (KMAX + NG - 1) / NG;  // write rows per thread
      float4 olds[RPT];
      float4 pp = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int i = 0; i < RPT; ++i) {
        const int j = g + i * NG;
        olds[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (j >= a.W) continue;
        const int s = iw[j];
        if (static_cast<unsigned>(s) >= static_cast<unsigned>(a.N)) continue;
        float4 old = reinterpret_cast<const float4*>(st + (size_t)j * CW)[lig];
        if (tok_tab[seq_hash(s)] >= u - D) {
          int tw, jw;
          if (find_writer(s, u - 1, u - D, tw, jw))
            old = reinterpret_cast<const float4*>(stage(tw) + (size_t)jw * CW)[lig];
        }
        olds[i] = old;
        const float kw = ww[j] * al;
        pp.x = fmaf(kw, old.x, pp.x);
        pp.y = fmaf(kw, old.y, pp.y);
        pp.z = fmaf(kw, old.z, pp.z);
        pp.w = fmaf(kw, old.w, pp.w);
      }
#pragma unroll
      for (int o = LPR; o < 32; o <<= 1) {
        pp.x += __shfl_xor_sync(FULL_MASK, pp.x, o);
        pp.y += __shfl_xor_sync(FULL_MASK, pp.y, o);
        pp.z += __shfl_xor_sync(FULL_MASK, pp.z, o);
        pp.w += __shfl_xor_sync(FULL_MASK, pp.w, o);
      }
      if (lane < LPR) reinterpret_cast<float4*>(red + warp * CW)[lane] = pp;
      __syncthreads();
      float4 pr = reinterpret_cast<const float4*>(red)[lig];
#pragma unroll
      for (int w = 1; w < NW; ++w) {
        const float4 t = reinterpret_cast<const float4*>(red + w * CW)[lig];
        pr.x += t.x;
        pr.y += t.y;
        pr.z += t.z;
        pr.w += t.w;
      }
      const float4 dv = make_float4(vv.x - pr.x, vv.y - pr.y, vv.z - pr.z, vv.w - pr.w);
#pragma unroll
      for (int i = 0; i < RPT; ++i) {
        const int j = g + i * NG;
        if (j >= a.W) continue;
        const int s = iw[j];
        if (static_cast<unsigned>(s) >= static_cast<unsigned>(a.N)) {
          if (lig == 0) record_status(STATUS_BAD_INDEX);
          continue;
        }
        const float kb = be * ww[j];
        float4 nw;
        nw.x = fmaf(al, olds[i].x, kb * dv.x);
        nw.y = fmaf(al, olds[i].y, kb * dv.y);
        nw.z = fmaf(al, olds[i].z, kb * dv.z);
        nw.w = fmaf(al, olds[i].w, kb * dv.w);
        reinterpret_cast<float4*>(st + (size_t)j * CW)[lig] = nw;
        *reinterpret_cast<float4*>(Mbh + (size_t)s * a.d_v + col0 + 4 * lig) = nw;
        if (lig == 0) tok_tab[seq_hash(s)] = u;
      }
    }

    // step 2: gated delta write
    for (int j = g; j < a.W && !a.coupled; j += NG) {
      int s = iw[j];
      if (static_cast<unsigned>(s) >= static_cast<unsigned>(a.N)) {
        if (lig == 0) record_status(STATUS_BAD_INDEX);
        continue;
      }
      float4 old = reinterpret_cast<const float4*>(st + (size_t)j * CW)[lig];
      if (tok_tab[seq_hash(s)] >= u - D) {
        int tw, jw;
        if (find_writer(s, u - 1, u - D, tw, jw))
          old = reinterpret_cast<const float4*>(stage(tw) + (size_t)jw * CW)[lig];
      }
      if (a.wlog)
        __stcs(reinterpret_cast<float4*>(a.wlog + ((tok_row0 + (size_t)u * a.H) * a.W + j) *
                                                      a.d_v + col0) + lig, old);
      const float kb = be * ww[j];
      const float ka = al * (1.0f - kb);
      float4 nw;
      nw.x = fmaf(ka, old.x, kb * vv.x);
      nw.y = fmaf(ka, old.y, kb * vv.y);
      nw.z = fmaf(ka, old.z, kb * vv.z);
      nw.w = fmaf(ka, old.w, kb * vv.w);
      reinterpret_cast<float4*>(st + (size_t)j * CW)[lig] = nw;
      *reinterpret_cast<float4*>(Mbh + (size_t)s * a.d_v + col0 + 4 * lig) = nw;
      if (lig == 0) tok_tab[seq_hash(s)] = u;
    }
    __syncthreads();

    // step 3: sparse read after the write
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = g; j < a.R; j += NG) {
      const int s = ir[j];
      if (static_cast<unsigned>(s) >= static_cast<unsigned>(a.N)) {
        if (lig == 0) record_status(STATUS_BAD_INDEX);
        continue;
      }
      float4 val = reinterpret_cast<const float4*>(st + (size_t)(a.ldw + j) * CW)[lig];
      if (tok_tab[seq_hash(s)] >= u - D) {
        int tw, jw;
        if (find_writer(s, u, u - D, tw, jw))
          val = reinterpret_cast<const float4*>(stage(tw) + (size_t)jw * CW)[lig];
      }
      const float q = wr[j];
      acc.x = fmaf(q, val.x, acc.x);
      acc.y = fmaf(q, val.y, acc.y);
      acc.z = fmaf(q, val.z, acc.z);
      acc.w = fmaf(q, val.w, acc.w);
    }
#pragma unroll
    for (int o = LPR; o < 32; o <<= 1) {
      acc.x += __shfl_xor_sync(FULL_MASK, acc.x, o);
      acc.y += __shfl_xor_sync(FULL_MASK, acc.y, o);
      acc.z += __shfl_xor_sync(FULL_MASK, acc.z, o);
      acc.w += __shfl_xor_sync(FULL_MASK, acc.w, o);
    }
    if (lane < LPR) reinterpret_cast<float4*>(red + warp * CW)[lane] = acc;
    __syncthreads();
    if (tid < LPR) {
      float4 sum = reinterpret_cast<const float4*>(red)[tid];
#pragma unroll
      for (int w = 1; w < NW; ++w) {
        const float4 p = reinterpret_cast<const float4*>(red + w * CW)[tid];
        sum.x += p.x;
        sum.y += p.y;
        sum.z += p.z;
        sum.w += p.w;
      }
      *reinterpret_cast<float4*>(a.y + (tok_row0 + (size_t)u * a.H) * a.d_v + col0 + 4 * tid) =
          sum;
    }
    // refill: rows of token u + D (their writers up to u are done), meta of u + 2D
    if (u + D < a.T) issue_rows(u + D);
    if (u + 2 * D < a.T) issue_meta(u + 2 * D);
    cp_async_commit();
  }
  cp_async_wait<0>();
}

}  // namespace sdm
