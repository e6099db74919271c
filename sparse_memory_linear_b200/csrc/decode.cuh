// decode.cuh -- one decode step of the SDM pass for every (sequence, head), fused.
//
// Method: "Sparse Delta Memory: Scaling the State of Linear RNNs through Sparsity"
// (paper.rainbus.top summary), method steps 1-4, applied to a single token; the m.163.com
// article on SDM (section 八) reports decode as the setting where the HBM-resident
// memory costs most.  One CTA of 8 warps per (b, h), in one wave for a 64 x 8 batch:
//   step 1 (bf16 halves of up to 1024 scores, K <= 128): two warps per score half (write
//   and read selection, first and second half) find the half's top K with the group
//   selection of select_group.cuh; four warps per selection then take the top K of the
//   rank-pair candidate sums the same way and write slot indices and softmax weights (when
//   the halves' exponents span more than 15, the first of the four checks the ties at the
//   K-th sum against all K*K pairs, as select.cuh describes).
//   Other shapes: warps 0 and 1 run the warp-per-row selection of select.cuh.
//   CTAs 0 .. 127 also prefetch into L2 the inputs of the CTAs dispatched after them;
//   steps 2 and 3 issue every row load of the token at once: each warp's write rows go to
//   shared memory (over the dead selection scratch) by cp.async and its first read rows to
//   registers, so the step waits for one memory latency;
//   step 2: every warp rewrites its share of the W write rows; a write row that the token
//   also reads is added to the warp's read sum straight from the registers that hold its
//   new value;
//   step 3: every warp adds its share of the read rows that the token does not write;
//   step 4: warp 0 sums the eight partial reads, normalises and gates them.
#pragma once

#include "common.cuh"
#include "select.cuh"
#include "select_fast.cuh"
#include "select_group.cuh"

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
// Largest write-row set staged in shared memory (W * d_v * 4 bytes); larger sets are loaded
// into registers a batch at a time.
constexpr size_t DEC_ROWS_SMEM_MAX = 64 * 1024;

struct DecLayout {
  uint32_t off_lists, off_vec, off_part;
  // group selection
  uint32_t off_hist, off_ctl, off_list, list_stride, off_clist, clist_stride, off_sorted, off_ev;
  uint32_t off_bits;  // 2048-bit membership filters of the write and the read slots
  uint32_t off_pred;  // coupled rule: per-warp shares of the prediction [DEC_WARPS][d_v]
  // warp-per-row selection
  uint32_t off_sel, sel_stride;
  // write rows staged over the selection scratch (dead once the selection is done)
  uint32_t off_rows;
  int rows_smem;
  uint32_t total;
  int C_w, C_r;  // candidate counts of W and R
};

// Shared-memory plan.  `group` selects the group selection (histograms, control words, four
// half lists, two candidate lists, the sorted halves, softmax numerators); otherwise two
// warp selection scratch areas.
inline DecLayout dec_layout(int S1, int S2, int W, int R, int d_v, bool group,
                            bool coupled = false) {
  DecLayout L{};
  size_t p = 0;
  auto take = [&p](size_t bytes) {
    const size_t o = p;
    p += (bytes + 15) / 16 * 16;
    return static_cast<uint32_t>(o);
  };
  L.C_w = cand_count(W);
  L.C_r = cand_count(R);
  const int kmax = W > R ? W : R;
  const int smax = S1 > S2 ? S1 : S2;
  L.off_lists = take(4 * (size_t)KMAX * 4);  // idx_w, wt_w, idx_r, wt_r
  L.off_vec = take((2 * (size_t)d_v + 4) * 4);  // v, act(gate), alpha, beta
  L.off_part = take((size_t)DEC_WARPS * d_v * 4);
  L.off_bits = take(2 * 64 * 4);
  L.off_pred = coupled ? take((size_t)DEC_WARPS * d_v * 4) : 0u;
  const size_t scratch = p;
  if (group) {
    L.off_hist = take(6 * 256 * 4);  // four halves, two candidate sets
    L.off_ctl = take(6 * sizeof(GroupCtl));
    L.list_stride = ((size_t)(smax + 4) * 4 + 15) / 16 * 16;
    L.off_list = take(4 * L.list_stride);
    L.clist_stride = ((size_t)(cand_count(kmax) + 4) * 8 + 15) / 16 * 16;
    L.off_clist = take(2 * L.clist_stride);
    L.off_sorted = take(4 * (size_t)KMAX * 4);
    L.off_ev = take(2 * (size_t)KMAX * 4);
  } else {
    L.sel_stride = (sel_scratch_bytes(S1, S2, kmax) + 15) / 16 * 16;
    L.off_sel = take(2 * L.sel_stride);
  }
  const size_t rows_bytes = (size_t)W * d_v * 4;
  L.rows_smem = rows_bytes <= DEC_ROWS_SMEM_MAX;
  L.off_rows = static_cast<uint32_t>(scratch);
  if (L.rows_smem && scratch + rows_bytes > p) p = scratch + rows_bytes;
  L.total = static_cast<uint32_t>(p);
  return L;
}

// CTAs 0 .. DEC_PF_CTAS - 1 are dispatched first and prefetch for the others.  Measured on
// a 64 x 8 batch (us per chained step): none 17.2, 32 CTAs 16.3, 64 16.5, 128 15.7.
constexpr int DEC_PF_CTAS = 128;

// L2 prefetch of the 128-byte lines of [p, p + bytes) by the lanes of one warp; every
// address prefetched lies inside the span.
__device__ __forceinline__ void prefetch_l2_span(const void* p, size_t bytes, int lane) {
  const uintptr_t s = reinterpret_cast<uintptr_t>(p);
  const uintptr_t first = s & ~static_cast<uintptr_t>(127);
  const int nl = static_cast<int>((s + bytes - first + 127) >> 7);
  for (int l = lane; l < nl; l += 32) {
    const uintptr_t ad = l == 0 ? s : first + (static_cast<uintptr_t>(l) << 7);
    asm volatile("prefetch.global.L2 [%0];" ::"l"(ad));
  }
}

// The CTAs dispatched first warm L2 with the step inputs (score halves, v, gate, alpha,
// beta) of units bh + DEC_PF_CTAS, bh + 2 DEC_PF_CTAS, ...  Under programmatic launch the
// later CTAs of a step start only as the previous step's CTAs leave the SMs, and their
// score loads would otherwise add a DRAM round trip to the step's critical path.
__device__ __forceinline__ void dec_prefetch_later_units(const DecodeArgs& a, int bh, int warp,
                                                         int lane) {
  if (bh >= DEC_PF_CTAS) return;
  const size_t esz = a.in_bf16 ? 2 : 4;
  const size_t srow = static_cast<size_t>(a.S1 + a.S2) * esz;
  const size_t vrow = static_cast<size_t>(a.d_v) * esz;
  const int nu = (a.BH - 1 - bh) / DEC_PF_CTAS;
  for (int t = warp; t < 4 * nu; t += DEC_WARPS) {
    const int u = bh + DEC_PF_CTAS * (1 + (t >> 2));
    switch (t & 3) {
      case 0: prefetch_l2_span(static_cast<const char*>(a.kp) + u * srow, srow, lane); break;
      case 1: prefetch_l2_span(static_cast<const char*>(a.qp) + u * srow, srow, lane); break;
      case 2:
        prefetch_l2_span(static_cast<const char*>(a.v) + u * vrow, vrow, lane);
        if (lane == 0) {
          asm volatile("prefetch.global.L2 [%0];" ::"l"(a.alpha + u));
          asm volatile("prefetch.global.L2 [%0];" ::"l"(a.beta + u));
        }
        break;
      default:
        if (a.gate) prefetch_l2_span(static_cast<const char*>(a.gate) + u * vrow, vrow, lane);
        break;
    }
  }
}

// Step 1 by the group selection: warps 2g, 2g + 1 take half g (0 write first, 1 write second,
// 2 read first, 3 read second); warps 4s .. 4s + 3 then take the candidates of selection s.
// E: bf16 scores per thread in units of 8 (halves of up to 512 E scores).  KC: largest K.
template <int E, int KC>
__device__ __forceinline__ void decode_select_group(const DecodeArgs& a, const DecLayout& L,
                                                    unsigned char* smem, int tid,
                                                    const uint32_t (&key)[E * 8],
                                                    int32_t* idx_w, float* wt_w, int32_t* idx_r,
                                                    float* wt_r) {
  constexpr int NK = E * 8;
  constexpr int CPT = (cand_count(KC) + 127) / 128;
  const int lane = tid & 31, warp = tid >> 5;
  const int g = warp >> 1, gt = tid & 63;
  const int s = g >> 1, st = tid & 127;
  const int K = s ? a.R : a.W;
  // this thread's rank pairs of the candidate table, loaded before the half selections so
  // that the loads are long done when the candidates need them (read late, these loads of a
  // table every CTA shares sat on the critical path, by up to 6 % of the step)
  uint32_t tpre[CPT];
  {
    const uint16_t* tp = cand_table(K);
    const int Cp = s ? L.C_r : L.C_w;
#pragma unroll
    for (int j = 0; j < CPT; ++j) tpre[j] = st + 128 * j < Cp ? __ldg(tp + st + 128 * j) : 0u;
  }
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + L.off_hist);
  GroupCtl* ctl = reinterpret_cast<GroupCtl*>(smem + L.off_ctl);
  uint32_t* sorted = reinterpret_cast<uint32_t*>(smem + L.off_sorted);

  // half g: bracket from every thread's P-th largest key, P = ceil(K / 64)
  uint32_t t1 = 0u, t2 = 0u;
#pragma unroll
  for (int i = 0; i < NK; ++i) {
    const uint32_t x = key[i];
    t2 = max(t2, min(t1, x));
    t1 = max(t1, x);
  }
  uint32_t lo, hi;
  group_bracket<64>(t1, K > 64 ? t2 : t1, ctl + g, gt, 1 + g, lo, hi);
  const CutResult cr =
      group_cut<NK, 64>(key, lo, hi, K, 2 * K, hist + 256 * g, ctl + g, gt, 1 + g);
  uint32_t* list = reinterpret_cast<uint32_t*>(smem + L.off_list + g * L.list_stride);
  uint32_t* out_half = sorted + KMAX * g;
  group_order<NK, 64>(
      key, cr,
      [&](int i) {
        const int idx = (i >> 3) * 512 + gt * 8 + (i & 7);
        return (key[i] << 16) | (0xffffu - static_cast<uint32_t>(idx));
      },
      list, &ctl[g].count, gt, lane, 1 + g, [&](int r, uint32_t c) {
        if (r < K) out_half[r] = c;
      });
  group_bar(5 + s, 128);

  // candidates of selection s
  const uint32_t* A = sorted + KMAX * (2 * s);
  const uint32_t* B = sorted + KMAX * (2 * s + 1);
  const int C = s ? L.C_r : L.C_w;
  uint32_t ck[CPT], cf[CPT];
#pragma unroll
  for (int j = 0; j < CPT; ++j) {
    const int c = st + 128 * j;
    ck[j] = 0u;
    cf[j] = 0u;
    if (c < C) {
      const int e = static_cast<int>(tpre[j]);
      const uint32_t ca = A[e >> 7], cb = B[e & 127];
      ck[j] = score_key(__fadd_rn(key16_value(ca >> 16), key16_value(cb >> 16)));
      cf[j] = (0xffffu - (ca & 0xffffu)) * static_cast<uint32_t>(a.S2) + (0xffffu - (cb & 0xffffu));
    }
  }
  // the K sums A[i] + B[0] and the K sums A[0] + B[i] are candidates: both K-th largest
  // bound the K-th largest candidate from below
  const float a0 = key16_value(A[0] >> 16), b0 = key16_value(B[0] >> 16);
  const uint32_t chi = score_key(__fadd_rn(a0, b0));
  const uint32_t clo = max(max(score_key(__fadd_rn(key16_value(A[K - 1] >> 16), b0)),
                               score_key(__fadd_rn(a0, key16_value(B[K - 1] >> 16)))), 1u);
  GroupCtl* cctl = ctl + 4 + s;
  const CutResult cc =
      group_cut<CPT, 128>(ck, clo, chi, K, 2 * K, hist + 256 * (4 + s), cctl, st, 5 + s);
  uint64_t* clist = reinterpret_cast<uint64_t*>(smem + L.off_clist + s * L.clist_stride);
  float* ev = reinterpret_cast<float*>(smem + L.off_ev) + KMAX * s;
  int32_t* out_idx = s ? idx_r : idx_w;
  float* out_wt = s ? wt_r : wt_w;
  uint32_t* bits = reinterpret_cast<uint32_t*>(smem + L.off_bits) + 64 * s;
  const float s0 = key_score(chi);
  group_order<CPT, 128>(
      ck, cc, [&](int j) { return (static_cast<uint64_t>(ck[j]) << 32) | (0xffffffffu - cf[j]); },
      clist, &cctl->count, st, lane, 5 + s, [&](int r, uint64_t c) {
        if (r < K) {
          const uint32_t flat = 0xffffffffu - static_cast<uint32_t>(c);
          out_idx[r] = static_cast<int32_t>(flat);
          ev[r] = expf(key_score(static_cast<uint32_t>(c >> 32)) - s0);
          atomicOr(&bits[(flat >> 5) & 63u], 1u << (flat & 31u));
          if (r == K - 1) cctl->kth = static_cast<uint32_t>(c >> 32);
        }
      });
  group_bar(5 + s, 128);
  if (st < 32 && !warp_bf16_sums_exact(
                     [&](int j) { return key16_value((j < K ? A[j] : B[j - K]) >> 16); }, K, st)) {
    // fp32 rounding may have merged unequal sums: the ties at the K-th sum are checked
    // against all K*K pairs (a refilled slot keeps the K-th key, so its weight is unchanged;
    // a replaced slot's filter bit stays set, which the exact membership checks allow)
    const uint32_t Tk = cctl->kth;
    repair_ties_at_kth(
        [&](int r1, int r2) {
          return score_key(__fadd_rn(key16_value(A[r1] >> 16), key16_value(B[r2] >> 16)));
        },
        [&](int r1, int r2) {
          return (0xffffu - (A[r1] & 0xffffu)) * static_cast<uint32_t>(a.S2) +
                 (0xffffu - (B[r2] & 0xffffu));
        },
        K, Tk, st, [&](int r, uint32_t f) {
          out_idx[r] = static_cast<int32_t>(f);
          atomicOr(&bits[(f >> 5) & 63u], 1u << (f & 31u));
        });
  }
  // the softmax denominator: a butterfly sum within each of the group's four warps, then the
  // four warp sums in a fixed order (the same sum on every thread)
  const float e_own = st < K ? ev[st] : 0.0f;
  float esum = e_own;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) esum += __shfl_xor_sync(FULL_MASK, esum, o);
  if (lane == 0) cctl->wmin[st >> 5] = __float_as_uint(esum);
  group_bar(5 + s, 128);
  const float total = (__uint_as_float(cctl->wmin[0]) + __uint_as_float(cctl->wmin[1])) +
                      (__uint_as_float(cctl->wmin[2]) + __uint_as_float(cctl->wmin[3]));
  if (st < K) out_wt[st] = e_own * (1.0f / total);
}

// E == 0: warp-per-row selection (fp32 halves, halves longer than 1024 scores); otherwise
// the group selection for bf16 halves of up to 512 E scores and K <= KC.  NQ float4
// columns per lane: d_v <= 128 NQ.
template <int E, int KC, int NQ, bool CP>
__global__ void __launch_bounds__(DEC_THREADS, 4) decode_kernel(DecodeArgs a, DecLayout L) {
  extern __shared__ __align__(16) unsigned char smem[];
  // the next step may be scheduled at once: its CTAs take the SM slots this step frees, and
  // their selection overlaps this step's row traffic
  grid_launch_dependents();
  const int bh = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool bf16 = a.in_bf16 != 0;
  const int S = a.S1 + a.S2;
  const int d4 = a.d_v / 4;

  int32_t* idx_w = reinterpret_cast<int32_t*>(smem + L.off_lists);
  float* wt_w = reinterpret_cast<float*>(idx_w + KMAX);
  int32_t* idx_r = reinterpret_cast<int32_t*>(wt_w + KMAX);
  float* wt_r = reinterpret_cast<float*>(idx_r + KMAX);
  float* vs = reinterpret_cast<float*>(smem + L.off_vec);  // [d_v]
  float* gs = vs + a.d_v;                                  // [d_v]
  float* ab = gs + a.d_v;                                  // alpha, beta
  float* part = reinterpret_cast<float*>(smem + L.off_part);  // [DEC_WARPS][d_v]

  if constexpr (E > 0) {
    // issue this thread's score loads first: everything else overlaps their latency
    const int g = warp >> 1, gt = tid & 63;
    const int Sh = (g & 1) ? a.S2 : a.S1;
    const __nv_bfloat16* src = reinterpret_cast<const __nv_bfloat16*>((g >> 1) ? a.qp : a.kp) +
                               (size_t)bh * S + ((g & 1) ? a.S1 : 0);
    const bool vec = (reinterpret_cast<uintptr_t>(src) & 15u) == 0;
    const uint16_t* raw16 = reinterpret_cast<const uint16_t*>(src);
    uint32_t key[E * 8];
#pragma unroll
    for (int r = 0; r < E; ++r) {
      const int e0 = r * 512 + gt * 8;
      if (vec && e0 + 8 <= Sh) {
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(src + e0));
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          key[r * 8 + 2 * j] = ww[j];
          key[r * 8 + 2 * j + 1] = ww[j] >> 16;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) key[r * 8 + i] = (e0 + i < Sh) ? raw16[e0 + i] : 0u;
      }
    }
    // this thread's v, gate, alpha, beta loads (d_v <= 128 NQ: at most VQ of each)
    constexpr int VQ = NQ <= 2 ? 1 : NQ / 2;
    float vr[VQ], gr[VQ], abr = 0.0f;
#pragma unroll
    for (int q = 0; q < VQ; ++q) {
      const int c = tid + DEC_THREADS * q;
      vr[q] = c < a.d_v ? load_in(a.v, (size_t)bh * a.d_v + c, bf16) : 0.0f;
      gr[q] = c < a.d_v && a.gate ? load_in(a.gate, (size_t)bh * a.d_v + c, bf16) : 0.0f;
    }
    if (tid < 2) abr = tid == 0 ? a.alpha[bh] : a.beta[bh];
    dec_prefetch_later_units(a, bh, warp, lane);
    // shared state of the group selection: this group's histogram and control words
    uint32_t* hist = reinterpret_cast<uint32_t*>(smem + L.off_hist);
    GroupCtl* ctl = reinterpret_cast<GroupCtl*>(smem + L.off_ctl);
    reinterpret_cast<uint4*>(hist + 256 * g)[gt] = make_uint4(0u, 0u, 0u, 0u);
    if (gt == 0) ctl[g].count = 0u;
    if ((tid & 127) == 0) ctl[4 + (tid >> 7)].count = 0u;
    {
      // this selection group's candidate histogram, filter words and softmax tail
      const int s = tid >> 7, st = tid & 127;
      reinterpret_cast<uint2*>(hist + 256 * (4 + s))[st] = make_uint2(0u, 0u);
      if (st < 64) reinterpret_cast<uint32_t*>(smem + L.off_bits)[64 * s + st] = 0u;
      const int K = s ? a.R : a.W;
      float* ev = reinterpret_cast<float*>(smem + L.off_ev) + KMAX * s;
      if (K + st < ((K + 3) & ~3)) ev[K + st] = 0.0f;
    }
#pragma unroll
    for (int q = 0; q < VQ; ++q) {
      const int c = tid + DEC_THREADS * q;
      if (c < a.d_v) {
        vs[c] = vr[q];
        gs[c] = a.gate ? gate_act(gr[q], a.act) : 1.0f;
      }
    }
    if (tid < 2) ab[tid] = abr;
#pragma unroll
    for (int i = 0; i < E * 8; ++i)
      key[i] = (i >> 3) * 512 + gt * 8 + (i & 7) < Sh ? bf16_key16(key[i]) : 0u;
    decode_select_group<E, KC>(a, L, smem, tid, key, idx_w, wt_w, idx_r, wt_r);
  } else {
    dec_prefetch_later_units(a, bh, warp, lane);
    const int kmax = a.W > a.R ? a.W : a.R;
    const size_t esz = bf16 ? 2 : 4;
    if (tid < 128) reinterpret_cast<uint32_t*>(smem + L.off_bits)[tid] = 0u;
    if (warp >= 2) {
      const int t0 = tid - 64, nt = DEC_THREADS - 64;
      for (int c = t0; c < a.d_v; c += nt) {
        vs[c] = load_in(a.v, (size_t)bh * a.d_v + c, bf16);
        gs[c] = a.gate ? gate_act(load_in(a.gate, (size_t)bh * a.d_v + c, bf16), a.act) : 1.0f;
      }
      if (t0 == 0) {
        ab[0] = a.alpha[bh];
        ab[1] = a.beta[bh];
      }
    } else {
      SelScratch sc = carve_sel_scratch(smem + L.off_sel + warp * L.sel_stride, a.S1, a.S2, kmax);
      const void* src = reinterpret_cast<const unsigned char*>(warp == 0 ? a.kp : a.qp) +
                        (size_t)bh * S * esz;
      select_row(src, bf16, a.S1, a.S2, warp == 0 ? a.W : a.R, cand_table(warp == 0 ? a.W : a.R), sc,
                 lane, warp == 0 ? idx_w : idx_r, warp == 0 ? wt_w : wt_r);
    }
  }
  __syncthreads();
  if constexpr (E == 0) {
    uint32_t* bits = reinterpret_cast<uint32_t*>(smem + L.off_bits);
    for (int j = tid; j < a.W; j += DEC_THREADS) {
      const uint32_t sl = static_cast<uint32_t>(idx_w[j]);
      atomicOr(&bits[(sl >> 5) & 63u], 1u << (sl & 31u));
    }
    for (int j = tid; j < a.R; j += DEC_THREADS) {
      const uint32_t sl = static_cast<uint32_t>(idx_r[j]);
      atomicOr(&bits[64 + ((sl >> 5) & 63u)], 1u << (sl & 31u));
    }
    __syncthreads();
  }

  // Everything above reads only this step's inputs.  A step launched with programmatic
  // stream serialisation may have started while the step before it still ran: wait for that
  // grid (and its memory) before touching anything it writes (sel_out, M, y, o).
  grid_dependency_wait();

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
  constexpr int RB = NQ >= 8 ? 1 : 8 / NQ;
  float* wrow = reinterpret_cast<float*>(smem + L.off_rows);  // [W][d_v] when rows_smem
  // 2048-bit filters of the write and the read slots: a clear bit rules a slot out
  const uint32_t* wbits = reinterpret_cast<const uint32_t*>(smem + L.off_bits);
  const uint32_t* rbits = wbits + 64;

  // Every row load of the step is issued before any is used: this warp's write rows
  // (warp, warp + 8, ...) go to shared memory by cp.async, its first RB read rows to
  // registers.  A read row that the token also writes is loaded too but not used: its
  // writer adds the new value (step 3 after step 2).
  // the variant's largest write-row set (W <= KC, d_v <= 128 NQ) always fits shared memory
  constexpr bool kRowsSmem = (size_t)KC * 128 * NQ * 4 <= DEC_ROWS_SMEM_MAX;
  const bool rows_smem = kRowsSmem || L.rows_smem;
  if (rows_smem) {
    for (int j = warp; j < a.W; j += DEC_WARPS) {
      const int sl = idx_w[j];
      if (static_cast<unsigned>(sl) >= static_cast<unsigned>(a.N)) continue;
      const float* src = Mbh + (size_t)sl * a.d_v;
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const int c = lane + 32 * q;
        if (c < d4) cp_async16(wrow + (size_t)j * a.d_v + 4 * c, src + 4 * c);
      }
    }
    cp_async_commit();
  }
  float4 val[RB][NQ];
  int rslot[RB];
  auto load_reads = [&](int j0) {
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      const int j = j0 + r * DEC_WARPS;
      rslot[r] = j < a.R ? idx_r[j] : -1;
      if (static_cast<unsigned>(rslot[r]) < static_cast<unsigned>(a.N)) {
        const float4* row = reinterpret_cast<const float4*>(Mbh + (size_t)rslot[r] * a.d_v);
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          const int c = lane + 32 * q;
          if (c < d4) val[r][q] = row[c];
        }
      }
    }
  };
  auto add_reads = [&](int j0) {
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      const int j = j0 + r * DEC_WARPS;
      if (j >= a.R) continue;
      if (static_cast<unsigned>(rslot[r]) >= static_cast<unsigned>(a.N)) {
        if (lane == 0) record_status(STATUS_BAD_INDEX);
        continue;
      }
      const uint32_t rs = static_cast<uint32_t>(rslot[r]);
      if ((wbits[(rs >> 5) & 63u] >> (rs & 31u)) & 1u) {
        // the filter admits the slot: an exact check against the write list
        bool in_w = false;
        for (int e = lane; e < a.W; e += 32) in_w |= (idx_w[e] == rslot[r]);
        if (__any_sync(FULL_MASK, in_w)) continue;
      }
      const float q = wt_r[j];
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
  };
  if (rows_smem) {
    // step 3 for this warp's first read rows, before the write loop: they are in flight with
    // the write rows, and their registers are free again before the loop needs its own
    load_reads(warp);
    add_reads(warp);
  }

  // v of this lane's columns, held in registers for the write loop when it is one float4
  // (wider rows read it from shared memory per row: registers are short there)
  constexpr bool kVReg = NQ == 1;
  float4 vreg = make_float4(0.f, 0.f, 0.f, 0.f);
  if (kVReg && lane < d4) vreg = reinterpret_cast<const float4*>(vs)[lane];

  // coupled rule (CP): the prediction p = sum_j k_j alpha M[j] over the write rows, shared by
  // all of them; each warp sums its rows' share, the shares meet in shared memory
  float4 pred[NQ];
#pragma unroll
  for (int q = 0; q < NQ; ++q) pred[q] = make_float4(0.f, 0.f, 0.f, 0.f);
  if constexpr (CP) {
    if (rows_smem) {
      cp_async_wait<0>();  // this warp's write rows (its own lanes' chunks) have landed
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const int c = lane + 32 * q;
        float4 pp = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = warp; j < a.W; j += DEC_WARPS) {
          if (static_cast<unsigned>(idx_w[j]) >= static_cast<unsigned>(a.N) || c >= d4) continue;
          const float kw = wt_w[j] * al;
          const float4 o4 = reinterpret_cast<const float4*>(wrow + (size_t)j * a.d_v)[c];
          pp.x = fmaf(kw, o4.x, pp.x);
          pp.y = fmaf(kw, o4.y, pp.y);
          pp.z = fmaf(kw, o4.z, pp.z);
          pp.w = fmaf(kw, o4.w, pp.w);
        }
        if (c < d4) reinterpret_cast<float4*>(smem + L.off_pred + (size_t)warp * a.d_v * 4)[c] = pp;
      }
      __syncthreads();
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const int c = lane + 32 * q;
        if (c >= d4) continue;
#pragma unroll
        for (int w = 0; w < DEC_WARPS; ++w) {
          const float4 t = reinterpret_cast<const float4*>(smem + L.off_pred + (size_t)w * a.d_v * 4)[c];
          pred[q].x += t.x;
          pred[q].y += t.y;
          pred[q].z += t.z;
          pred[q].w += t.w;
        }
      }
    }
  }

  // step 2 on one write row whose old value is `old`: store the new row, and add it to the
  // read sum if the token also reads the slot.  Per-slot rule: alpha (1 - beta k) M[i] +
  // beta k v; coupled rule: alpha M[i] + beta k (v - p).
  auto write_row = [&](int j, int sl, const float4 (&old)[NQ]) {
    int rpos = -1;
    const uint32_t us = static_cast<uint32_t>(sl);
    if ((rbits[(us >> 5) & 63u] >> (us & 31u)) & 1u) {
      for (int e0 = 0; e0 < a.R; e0 += 32) {
        const unsigned m = __ballot_sync(FULL_MASK, e0 + lane < a.R && idx_r[e0 + lane] == sl);
        if (m && rpos < 0) rpos = e0 + __ffs(m) - 1;
      }
    }
    const float qr = rpos >= 0 ? wt_r[rpos] : 0.0f;
    const float kb = be * wt_w[j];
    const float ka = CP ? al : al * (1.0f - kb);
    float4* row = reinterpret_cast<float4*>(Mbh + (size_t)sl * a.d_v);
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      const int c = lane + 32 * q;
      if (c < d4) {
        float4 vv = kVReg ? vreg : reinterpret_cast<const float4*>(vs)[c];
        if constexpr (CP) {
          vv.x -= pred[q].x;
          vv.y -= pred[q].y;
          vv.z -= pred[q].z;
          vv.w -= pred[q].w;
        }
        float4 nw;
        nw.x = fmaf(ka, old[q].x, kb * vv.x);
        nw.y = fmaf(ka, old[q].y, kb * vv.y);
        nw.z = fmaf(ka, old[q].z, kb * vv.z);
        nw.w = fmaf(ka, old[q].w, kb * vv.w);
        row[c] = nw;
        if (rpos >= 0) {
          acc[q].x = fmaf(qr, nw.x, acc[q].x);
          acc[q].y = fmaf(qr, nw.y, acc[q].y);
          acc[q].z = fmaf(qr, nw.z, acc[q].z);
          acc[q].w = fmaf(qr, nw.w, acc[q].w);
        }
      }
    }
  };
  if (rows_smem) {
    cp_async_wait<0>();  // this lane's own chunks: each lane rewrites exactly what it loaded
    for (int j = warp; j < a.W; j += DEC_WARPS) {
      const int sl = idx_w[j];
      if (static_cast<unsigned>(sl) >= static_cast<unsigned>(a.N)) {
        if (lane == 0) record_status(STATUS_BAD_INDEX);
        continue;
      }
      float4 old[NQ];
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const int c = lane + 32 * q;
        old[q] = c < d4 ? reinterpret_cast<const float4*>(wrow + (size_t)j * a.d_v)[c]
                        : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      write_row(j, sl, old);
    }
  } else {
    // write rows through registers, RB at a time
    for (int j0 = warp; j0 < a.W; j0 += DEC_WARPS * RB) {
      float4 old[RB][NQ];
      int slot[RB];
#pragma unroll
      for (int r = 0; r < RB; ++r) {
        const int j = j0 + r * DEC_WARPS;
        slot[r] = j < a.W ? idx_w[j] : -1;
        if (static_cast<unsigned>(slot[r]) < static_cast<unsigned>(a.N)) {
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
        write_row(j, slot[r], old[r]);
      }
    }
    load_reads(warp);
  }
  // step 3 for the read rows this token does not write
  if (!rows_smem) add_reads(warp);
  for (int j0 = warp + DEC_WARPS * RB; j0 < a.R; j0 += DEC_WARPS * RB) {
    load_reads(j0);
    add_reads(j0);
  }
#pragma unroll
  for (int qq = 0; qq < NQ; ++qq) {
    const int c = lane + 32 * qq;
    if (c < d4) reinterpret_cast<float4*>(part + (size_t)warp * a.d_v)[c] = acc[qq];
  }
  __syncthreads();

  // y and step 4 on warp 0
  if (warp != 0) return;
  float4 yv[NQ];
  float ss = 0.0f;
#pragma unroll
  for (int qq = 0; qq < NQ; ++qq) {
    const int c = lane + 32 * qq;
    yv[qq] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (c < d4) {
      float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int w = 0; w < DEC_WARPS; ++w) {
        const float4 p = reinterpret_cast<const float4*>(part + (size_t)w * a.d_v)[c];
        t.x += p.x;
        t.y += p.y;
        t.z += p.z;
        t.w += p.w;
      }
      yv[qq] = t;
      reinterpret_cast<float4*>(a.y + (size_t)bh * a.d_v)[c] = t;
      ss = fmaf(t.x, t.x, ss);
      ss = fmaf(t.y, t.y, ss);
      ss = fmaf(t.z, t.z, ss);
      ss = fmaf(t.w, t.w, ss);
    }
  }
  if (!a.o) return;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(FULL_MASK, ss, o);
  const float inv = rsqrtf(ss / static_cast<float>(a.d_v) + a.eps);
#pragma unroll
  for (int qq = 0; qq < NQ; ++qq) {
    const int c = lane + 32 * qq;
    if (c < d4) {
      const float4 g4 = reinterpret_cast<const float4*>(gs)[c];
      const float4 m4 = a.gamma ? reinterpret_cast<const float4*>(a.gamma)[c]
                                : make_float4(1.f, 1.f, 1.f, 1.f);
      float4 r;
      r.x = yv[qq].x * inv * m4.x * g4.x;
      r.y = yv[qq].y * inv * m4.y * g4.y;
      r.z = yv[qq].z * inv * m4.z * g4.z;
      r.w = yv[qq].w * inv * m4.w * g4.w;
      reinterpret_cast<float4*>(a.o + (size_t)bh * a.d_v)[c] = r;
    }
  }
}

}  // namespace sdm
