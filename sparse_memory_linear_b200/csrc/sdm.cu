// sdm.cu -- the C ABI of the SDM memory pass (declared in include/sdm.h): host-side
// validation, scratch layout, launch configuration and dispatch to the sm_100a kernels.
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <cmath>
#include <mutex>
#include <utility>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "decode.cuh"
#include "norm_init.cuh"
#include "rows.cuh"
#include "undo.cuh"
#include "scan_chunk.cuh"
#include "scan_seq.cuh"
#include "scan_slot.cuh"
#include "select.cuh"
#include "select_fast.cuh"

using namespace sdm;

namespace {

constexpr int MAX_DEVICES = 64;

// decode_kernel instantiations, cheapest first: (scores per thread / 8, K class, float4
// columns per lane).  E == 0 is the warp-per-row selection.
#define SDM_DEC_VARIANTS(X) \
  X(1, 64, 1) X(1, 128, 2) X(2, 128, 2) X(2, 128, 8) X(0, 128, 8)
constexpr size_t WS_ALIGN = 256;

#define SDM_CUDA_TRY(expr)                       \
  do {                                           \
    if ((expr) != cudaSuccess) {                 \
      (void)cudaGetLastError();                  \
      return SDM_ERR_CUDA;                       \
    }                                            \
  } while (0)

// An NVTX range around one call of the ABI (visible in Nsight timelines; a few nanoseconds
// when no tool is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Process-wide launch options (sdm_option); 0 everywhere by default.
constexpr int OPT_SLOTS = 16;
std::atomic<int> g_opt[OPT_SLOTS];

inline int opt(int which) { return g_opt[which].load(std::memory_order_relaxed); }

// SDM_OPT_NO_PDL = 1 launches every kernel in plain stream order, sdm_decode_step_chained
// included.
inline bool pdl_enabled() { return opt(SDM_OPT_NO_PDL) == 0; }

// Launches `kernel` in stream order, or with PDL = true with programmatic stream
// serialisation: scheduled while the kernel ahead of it finishes.  Every kernel of this
// library starts with griddepcontrol.wait / launch_dependents, so either launch gives the
// same results; the programmatic one hides launch latency.  It is used where the kernel
// ahead is a short one (inside a chunk's sort chain).  Behind the long persistent kernels
// (selection, chunk scan), dependents that sat waiting on the SMs made the step slower.
template <bool PDL = false, typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = PDL && pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Kernels launched by this library in this process (all devices).
std::atomic<unsigned long long> g_launches{0};

struct DeviceInfo {
  int sms = 0;
  int max_smem_optin = 0;
  bool attrs_set = false;
};

std::mutex g_dev_mu;
DeviceInfo g_dev[MAX_DEVICES];

// Lets `kernel` use all the opt-in shared memory that its static shared memory leaves.
template <typename Kernel>
cudaError_t allow_max_dynamic_smem(Kernel kernel, int optin) {
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kernel);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              optin - (int)fa.sharedSizeBytes);
}

sdm_status device_info(DeviceInfo** out) {
  int dev = 0;
  SDM_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= MAX_DEVICES) return SDM_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.attrs_set) {
    SDM_CUDA_TRY(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev));
    SDM_CUDA_TRY(cudaDeviceGetAttribute(&d.max_smem_optin,
                                        cudaDevAttrMaxSharedMemoryPerBlockOptin, dev));
    const int m = d.max_smem_optin;
    SDM_CUDA_TRY(allow_max_dynamic_smem(sel_kernel, m));
#define SDM_FAST_ATTR(R8, KC) \
  SDM_CUDA_TRY(allow_max_dynamic_smem(sel_fast_kernel<R8, KC>, m));
    SDM_FAST_ATTR(1, 32) SDM_FAST_ATTR(1, 64) SDM_FAST_ATTR(1, 128)
    SDM_FAST_ATTR(2, 32) SDM_FAST_ATTR(2, 64) SDM_FAST_ATTR(2, 128)
    SDM_FAST_ATTR(4, 32) SDM_FAST_ATTR(4, 64) SDM_FAST_ATTR(4, 128)
#undef SDM_FAST_ATTR
#define SDM_DEC_ATTR(R8, KC, NQ) \
  SDM_CUDA_TRY(allow_max_dynamic_smem(decode_kernel<R8, KC, NQ, false>, m)); \
  SDM_CUDA_TRY(allow_max_dynamic_smem(decode_kernel<R8, KC, NQ, true>, m));
    SDM_DEC_VARIANTS(SDM_DEC_ATTR)
#undef SDM_DEC_ATTR
#define SDM_SEQ_ATTR(CW, D) \
  SDM_CUDA_TRY(allow_max_dynamic_smem(seq_scan_kernel<CW, D>, m));
    SDM_SEQ_ATTR(4, 4) SDM_SEQ_ATTR(4, 8) SDM_SEQ_ATTR(8, 4) SDM_SEQ_ATTR(8, 8)
    SDM_SEQ_ATTR(16, 4) SDM_SEQ_ATTR(16, 8) SDM_SEQ_ATTR(32, 4) SDM_SEQ_ATTR(32, 8)
#undef SDM_SEQ_ATTR
    SDM_CUDA_TRY(allow_max_dynamic_smem(chunk_scan_kernel, m));
    SDM_CUDA_TRY(cudaFuncSetAttribute(radix_scatter_kernel,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)RS_SCATTER_SMEM));
#define SDM_SLOT_ATTR(NQ, G, PF) \
  SDM_CUDA_TRY(allow_max_dynamic_smem(slot_chunk_kernel<NQ, G, PF, false>, m)); \
  SDM_CUDA_TRY(allow_max_dynamic_smem(slot_chunk_kernel<NQ, G, PF, true>, m));
    SDM_SLOT_ATTR(1, 4, 6) SDM_SLOT_ATTR(2, 2, 6) SDM_SLOT_ATTR(4, 4, 4) SDM_SLOT_ATTR(8, 2, 2)
#undef SDM_SLOT_ATTR
    d.attrs_set = true;
  }
  *out = &d;
  return SDM_OK;
}

// Kernel timing, off by default: when on, every launch is bracketed by two CUDA events
// recorded on the launch's stream; sdm_profile_read() waits for them and sums per kind.
struct ProfRec {
  int kind;
  cudaEvent_t start, stop;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRec> g_prof_pending;

struct ProfScope {
  bool on = false;
  ProfRec rec{};
  cudaStream_t st;
  ProfScope(int kind, cudaStream_t stream) : st(stream) {
    std::lock_guard<std::mutex> lock(g_prof_mu);
    if (!g_prof_on) return;
    rec.kind = kind;
    if (cudaEventCreate(&rec.start) != cudaSuccess) return;
    if (cudaEventCreate(&rec.stop) != cudaSuccess) {
      cudaEventDestroy(rec.start);
      return;
    }
    on = cudaEventRecord(rec.start, st) == cudaSuccess;
  }
  ~ProfScope() {
    if (!on) return;
    cudaEventRecord(rec.stop, st);
    std::lock_guard<std::mutex> lock(g_prof_mu);
    g_prof_pending.push_back(rec);
  }
};

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Shape rules shared by every entry point (T may be 0 where the caller allows it).
bool shape_ok(const sdm_shape& s, bool allow_t0) {
  if (s.B < 1 || s.H < 1 || s.T < (allow_t0 ? 0 : 1)) return false;
  if (s.S1 < 1 || s.S2 < 1 || s.S1 > SMAX || s.S2 > SMAX) return false;
  if (s.in_dtype != SDM_F32 && s.in_dtype != SDM_BF16) return false;
  const int smin = s.S1 < s.S2 ? s.S1 : s.S2;
  if (s.W < 1 || s.R < 1 || s.W > smin || s.R > smin || s.W > KMAX || s.R > KMAX) return false;
  const int dmul = s.in_dtype == SDM_BF16 ? 8 : 4;
  if (s.d_v < dmul || s.d_v > 1024 || s.d_v % dmul != 0) return false;
  if ((long long)s.S1 * s.S2 > 2147483647LL) return false;
  return true;
}

size_t state_elems(const sdm_shape& s) {
  return (size_t)s.B * s.H * (size_t)s.S1 * s.S2 * s.d_v;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

struct WsLayout {
  int ldw, ldr;
  size_t off_idx_w, off_wt_w, off_idx_r, off_wt_r;
  // slot engine
  int chunk, n_chunks, ntiles, hot_cap;
  long long events;
  KeyBits kb;
  size_t off_k0, off_k1, off_v0, off_v1, off_hist, off_tot, off_offs, off_cnt, off_hot;
  size_t total;
};

// Tokens per chunk of the slot engine: a power of two whose y rows (fp32) and v rows, over
// every (sequence, head), take at most 64 MB, about half the L2.  Longer chunks load and
// store a slot's row fewer times and launch less; past this size y and v stop staying in
// L2.  Measured on the long skewed layer (ms per step at budgets of 16, 32, 64, 128 and
// 256 MB): 73.7, 58.2, 52.2, 55.9, 60.3.
int slot_chunk_tokens(const sdm_shape& s) {
  const size_t per_token = (size_t)s.B * s.H * s.d_v * (4 + (s.in_dtype == SDM_BF16 ? 2 : 4));
  size_t c = ((size_t)64 << 20) / (per_token ? per_token : 1);
  size_t p = 1;
  while (p * 2 <= c) p *= 2;
  if (p > (size_t)s.T) p = s.T > 0 ? (size_t)s.T : 1;
  return (int)p;
}

WsLayout ws_layout(const sdm_shape& s, int engine) {
  WsLayout L;
  L.ldw = (int)round_up((size_t)s.W, 4);
  L.ldr = (int)round_up((size_t)s.R, 4);
  const size_t rows = (size_t)s.B * s.T * s.H;
  L.off_idx_w = 0;
  L.off_wt_w = round_up(L.off_idx_w + rows * L.ldw * 4, WS_ALIGN);
  L.off_idx_r = round_up(L.off_wt_w + rows * L.ldw * 4, WS_ALIGN);
  L.off_wt_r = round_up(L.off_idx_r + rows * L.ldr * 4, WS_ALIGN);
  L.total = round_up(L.off_wt_r + rows * L.ldr * 4, WS_ALIGN);
  L.chunk = slot_chunk_tokens(s);
  L.n_chunks = s.T > 0 ? (s.T + L.chunk - 1) / L.chunk : 0;
  // events and their sort buffers hold one time chunk at a time
  L.events = (long long)L.chunk * s.B * s.H * (s.W + s.R);
  L.ntiles = (int)((L.events + RS_TILE - 1) / RS_TILE);
  L.kb.nbits = bits_for((long long)s.S1 * s.S2);
  L.kb.hbits = bits_for(s.H);
  L.kb.bbits = bits_for(s.B);
  L.kb.cbits = 0;
  L.hot_cap = (int)(L.events / SLOT_LONG + 1);
  L.off_k0 = L.off_k1 = L.off_v0 = L.off_v1 = L.off_hist = L.off_tot = L.off_offs = 0;
  L.off_cnt = L.off_hot = 0;
  if (engine == SDM_ENGINE_SLOT) {
    const size_t E = (size_t)L.events;
    L.off_k0 = L.total;
    L.off_k1 = round_up(L.off_k0 + E * 4, WS_ALIGN);
    L.off_v0 = round_up(L.off_k1 + E * 4, WS_ALIGN);
    L.off_v1 = round_up(L.off_v0 + E * 8, WS_ALIGN);
    L.off_hist = round_up(L.off_v1 + E * 8, WS_ALIGN);
    L.off_tot = round_up(L.off_hist + (size_t)RS_BINS * L.ntiles * 4, WS_ALIGN);
    L.off_offs = round_up(L.off_tot + RS_BINS * 4, WS_ALIGN);
    L.off_cnt = round_up(L.off_offs + 2 * 4, WS_ALIGN);
    L.off_hot = round_up(L.off_cnt + 2 * 4, WS_ALIGN);
    L.total = round_up(L.off_hot + (size_t)L.hot_cap * 8, WS_ALIGN);
  }
  return L;
}

// The slot engine packs (sequence, head, slot) into 31 bits of a key and counts a chunk's
// events and the state rows in 32 bits.
bool slot_engine_fits(const sdm_shape& s) {
  const WsLayout L = ws_layout(s, SDM_ENGINE_SEQ);
  const long long rows = (long long)s.B * s.T * s.H;
  return L.kb.total() <= 31 && (unsigned long long)L.events < 0xffffffffull &&
         rows < (1LL << 31) && s.T < (1 << 24);
}

// Prefill times of both engines, measured on one B200 (CUDA events around one
// sdm_scan_forward with SDM_CONTINUE: selection, engine and norm/gate; bf16 inputs, W = R =
// 64).  AUTO takes the engine that was faster on the measured shape nearest to the request.
struct EngineMeasure {
  int B, H, T, N, d_v;
  float seq_ms, slot_ms;
};
constexpr EngineMeasure kEngineTable[] = {
    {2, 4, 2048, 65536, 64, 12.67f, 0.597f},          // small layer
    {4, 8, 8192, 262144, 128, 29.69f, 10.29f},        // 1.4B-like layer
    {1, 4, 262144, 1048576, 256, 1769.2f, 46.30f},    // long prefill, skewed slots
    {64, 8, 256, 262144, 128, 12.82f, 6.34f},         // many short sequences
};

inline double log2d(double x) { return x > 1.0 ? std::log2(x) : 0.0; }

// Engine of an AUTO request: the sequential engine when the slot engine cannot hold the
// shape (its event keys and counts), otherwise the faster engine of the nearest measured
// shape, by distance over log2 of the (sequence, head) units, tokens, slots and width.
int pick_engine(const sdm_shape& s, int requested, int sms) {
  (void)sms;
  if (requested != SDM_ENGINE_AUTO) return requested;
  if (!slot_engine_fits(s)) return SDM_ENGINE_SEQ;
  double best = 1e30;
  int engine = SDM_ENGINE_SLOT;
  for (const EngineMeasure& m : kEngineTable) {
    const double d = std::fabs(log2d((double)s.B * s.H) - log2d((double)m.B * m.H)) +
                     std::fabs(log2d(s.T) - log2d(m.T)) +
                     std::fabs(log2d((double)s.S1 * s.S2) - log2d(m.N)) +
                     std::fabs(log2d(s.d_v) - log2d(m.d_v));
    if (d < best) {
      best = d;
      engine = m.seq_ms < m.slot_ms ? SDM_ENGINE_SEQ : SDM_ENGINE_SLOT;
    }
  }
  return engine;
}

// Grid of a selection launch over `total_rows` rows: one persistent wave at `per_sm` CTAs per
// SM, or, with rows_per_warp > 0, short-lived CTAs whose warps take that many rows each (the
// chunk-pipelined prefill, where the scan's CTAs take the SM slots that they free).
long long select_grid(long long total_rows, int warps, int per_sm, int rows_per_warp,
                      const DeviceInfo* di) {
  const long long need = (total_rows + warps - 1) / warps;
  if (rows_per_warp > 0) return (need + rows_per_warp - 1) / rows_per_warp;
  const int cap = opt(SDM_OPT_SELECT_CTAS_PER_SM);
  if (cap > 0 && cap < per_sm) per_sm = cap;
  const long long grid = (long long)di->sms * per_sm;
  return grid > need ? need : grid;
}

template <int R8, int KC>
sdm_status launch_select_fast_t(const SelJob& j0, const SelJob* j1, long long rows, int S1, int S2,
                                int rows_per_warp, const DeviceInfo* di, cudaStream_t st) {
  const int K1 = j1 ? j1->K : j0.K;
  int warps = 8;
  size_t smem = sel_fast_smem_bytes(S1, S2, j0.K, K1, warps);
  if (smem > (size_t)di->max_smem_optin) return SDM_ERR_UNSUPPORTED;
  int per_sm = 0;
  SDM_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, sel_fast_kernel<R8, KC>,
                                                             warps * 32, smem));
  if (per_sm < 1) return SDM_ERR_UNSUPPORTED;
  const long long total_rows = rows * (j1 ? 2 : 1);
  const long long grid = select_grid(total_rows, warps, per_sm, rows_per_warp, di);
  SDM_CUDA_TRY(launch_pdl(sel_fast_kernel<R8, KC>, dim3((unsigned)grid), dim3(warps * 32), smem, st,
                          j0, j1 ? *j1 : j0, rows, j1 ? 2 : 1, S1, S2));
  g_launches.fetch_add(1, std::memory_order_relaxed);
  SDM_CUDA_TRY(cudaGetLastError());
  return SDM_OK;
}

sdm_status launch_select_fast(const SelJob& j0, const SelJob* j1, long long rows, int S1, int S2,
                              int rows_per_warp, const DeviceInfo* di, cudaStream_t st) {
  const int K1 = j1 ? j1->K : j0.K;
  const int r8 = fast_r8(S1, S2);
  const int kc = fast_kc(j0.K > K1 ? j0.K : K1);
#define SDM_FAST_CASE(R8, KC) \
  if (r8 == R8 && kc == KC)      \
    return launch_select_fast_t<R8, KC>(j0, j1, rows, S1, S2, rows_per_warp, di, st);
  SDM_FAST_CASE(1, 32) SDM_FAST_CASE(1, 64) SDM_FAST_CASE(1, 128)
  SDM_FAST_CASE(2, 32) SDM_FAST_CASE(2, 64) SDM_FAST_CASE(2, 128)
  SDM_FAST_CASE(4, 32) SDM_FAST_CASE(4, 64) SDM_FAST_CASE(4, 128)
#undef SDM_FAST_CASE
  return SDM_ERR_UNSUPPORTED;
}

// Selection of one or two jobs over `rows` score rows (grid: select_grid).
sdm_status launch_select(const SelJob& j0, const SelJob* j1, long long rows, int S1, int S2,
                         int bf16, cudaStream_t st, int rows_per_warp = 0) {
  DeviceInfo* di;
  sdm_status rc = device_info(&di);
  if (rc != SDM_OK) return rc;
  if (rows == 0) return SDM_OK;
  const int K1 = j1 ? j1->K : j0.K;
  const int kmax_all = j0.K > K1 ? j0.K : K1;
  if (fast_select_ok(bf16, S1, S2, kmax_all) && opt(SDM_OPT_SELECT_GENERAL) == 0)
    return launch_select_fast(j0, j1, rows, S1, S2, rows_per_warp, di, st);
  int warps = 8;
  size_t smem = sel_smem_bytes(S1, S2, j0.K, K1, warps);
  while (warps > 1 && smem > (size_t)di->max_smem_optin / 2) {
    warps >>= 1;
    smem = sel_smem_bytes(S1, S2, j0.K, K1, warps);
  }
  if (smem > (size_t)di->max_smem_optin) return SDM_ERR_UNSUPPORTED;
  int per_sm = 0;
  SDM_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, sel_kernel, warps * 32, smem));
  if (per_sm < 1) return SDM_ERR_UNSUPPORTED;
  const long long total_rows = rows * (j1 ? 2 : 1);
  const long long grid = select_grid(total_rows, warps, per_sm, rows_per_warp, di);
  const int kmax = j0.K > K1 ? j0.K : K1;
  SDM_CUDA_TRY(launch_pdl(sel_kernel, dim3((unsigned)grid), dim3(warps * 32), smem, st,
                          j0, j1 ? *j1 : j0, rows, j1 ? 2 : 1, S1, S2, bf16, kmax));
  g_launches.fetch_add(1, std::memory_order_relaxed);
  SDM_CUDA_TRY(cudaGetLastError());
  return SDM_OK;
}

template <int CW, int D>
sdm_status launch_seq_t(const SeqArgs& a, int grid, size_t smem, cudaStream_t st) {
  SDM_CUDA_TRY(launch_pdl(seq_scan_kernel<CW, D>, dim3(grid), dim3(SEQ_THREADS), smem, st,
                          a));
  g_launches.fetch_add(1, std::memory_order_relaxed);
  SDM_CUDA_TRY(cudaGetLastError());
  return SDM_OK;
}

// Column-slice width CW and prefetch distance D of the sequential engine: one CTA per
// The chunk-wise engine: 32 tokens per chunk (16 or 8 when the shared memory of wide index
// lists needs it), column slices of up to 128 values (the largest multiple of 4 that
// divides d_v), a CTA per (sequence, head, slice).
sdm_status launch_chunk(ChunkArgs a, const DeviceInfo* di, cudaStream_t st) {
  a.CW = 4;
  for (int cw = a.d_v < 128 ? a.d_v : 128; cw >= 4; cw -= 4)
    if (cw % 4 == 0 && a.d_v % cw == 0) {
      a.CW = cw;
      break;
    }
  size_t smem = 0;
  for (a.C = 32; a.C >= 8; a.C /= 2) {
    a.hash_size = 1;
    while (a.hash_size < 2 * a.C * a.W) a.hash_size *= 2;
    smem = chunk_layout(a.C, a.W, a.R, a.CW, a.hash_size).total;
    if (smem <= (size_t)di->max_smem_optin) break;
  }
  if (a.C < 8) return SDM_ERR_UNSUPPORTED;
  const long long grid = (long long)a.B * a.H * (a.d_v / a.CW);
  SDM_CUDA_TRY(launch_pdl(chunk_scan_kernel, dim3((unsigned)grid), dim3(CHUNK_THREADS), smem, st,
                          a));
  g_launches.fetch_add(1, std::memory_order_relaxed);
  SDM_CUDA_TRY(cudaGetLastError());
  return SDM_OK;
}

// (sequence, head, slice) and all CTAs resident at once; wider slices while there are
// enough CTAs to cover the SMs, then narrower ones.
sdm_status launch_seq(const SeqArgs& a, cudaStream_t st) {
  DeviceInfo* di;
  sdm_status rc = device_info(&di);
  if (rc != SDM_OK) return rc;
  const int v_esz = a.v_bf16 ? 2 : 4;
  const int bh = a.B * a.H;
  const int cws[4] = {32, 16, 8, 4};
  int CW = 0;
  const int force_cw = opt(SDM_OPT_SEQ_COLUMNS);
  for (int i = 0; i < 4; ++i) {
    const int c = cws[i];
    if (a.d_v % c != 0 || c * v_esz < 16) continue;
    if (force_cw) {
      if (c == force_cw) CW = c;
      continue;
    }
    CW = c;
    if ((long long)bh * (a.d_v / c) * 5 >= (long long)di->sms * 4) break;
  }
  if (CW == 0) return SDM_ERR_UNSUPPORTED;
  int D = opt(SDM_OPT_SEQ_DEPTH);
  if (D != 4 && D != 8) D = CW >= 32 ? 4 : 8;
  SeqLayout L = seq_layout(a.ldw, a.ldr, CW, v_esz, D);
  if (L.total > (size_t)di->max_smem_optin && D == 8) {
    D = 4;
    L = seq_layout(a.ldw, a.ldr, CW, v_esz, D);
  }
  if (L.total > (size_t)di->max_smem_optin) return SDM_ERR_UNSUPPORTED;
  const int grid = bh * (a.d_v / CW);
  const size_t smem = L.total;
#define SDM_SEQ_CASE(C, DD) \
  if (CW == C && D == DD) return launch_seq_t<C, DD>(a, grid, smem, st);
  SDM_SEQ_CASE(32, 4) SDM_SEQ_CASE(32, 8) SDM_SEQ_CASE(16, 4) SDM_SEQ_CASE(16, 8)
  SDM_SEQ_CASE(8, 4) SDM_SEQ_CASE(8, 8) SDM_SEQ_CASE(4, 4) SDM_SEQ_CASE(4, 8)
#undef SDM_SEQ_CASE
  return SDM_ERR_UNSUPPORTED;
}

sdm_status launch_norm_gate(const float* y, const void* gate, int gate_bf16, const float* gamma,
                            float eps, int act, long long rows, int d_v, float* o,
                            cudaStream_t st) {
  DeviceInfo* di;
  sdm_status rc = device_info(&di);
  if (rc != SDM_OK) return rc;
  if (rows == 0) return SDM_OK;
  long long blocks = (rows + 7) / 8;
  const long long cap = (long long)di->sms * 8;
  if (blocks > cap) blocks = cap;
  SDM_CUDA_TRY(launch_pdl(norm_gate_kernel, dim3((unsigned)blocks), dim3(256), 0, st,
                          y, gate, gate_bf16, gamma, eps, act, rows, d_v, o));
  g_launches.fetch_add(1, std::memory_order_relaxed);
  SDM_CUDA_TRY(cudaGetLastError());
  return SDM_OK;
}

sdm_status launch_state_init(const float* M0, float* M, const sdm_shape& s, cudaStream_t st) {
  DeviceInfo* di;
  sdm_status rc = device_info(&di);
  if (rc != SDM_OK) return rc;
  const long long per_head4 = (long long)s.S1 * s.S2 * s.d_v / 4;
  const long long total = per_head4 * s.B * s.H;
  long long blocks = (total + 255) / 256;
  const long long cap = (long long)di->sms * 16;
  if (blocks > cap) blocks = cap;
  SDM_CUDA_TRY(launch_pdl(state_init_kernel, dim3((unsigned)blocks), dim3(256), 0, st,
                          reinterpret_cast<const float4*>(M0), reinterpret_cast<float4*>(M), s.B, s.H, per_head4));
  g_launches.fetch_add(1, std::memory_order_relaxed);
  SDM_CUDA_TRY(cudaGetLastError());
  return SDM_OK;
}

template <int NQ, int G, int PF, bool LOG>
sdm_status launch_slot_chunk_t(const SlotArgs& a, const DeviceInfo* di, cudaStream_t st) {
  const size_t smem = SLOT_WARPS * slot_warp_smem(NQ, PF);
  int per_sm = 0;
  SDM_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(
      &per_sm, slot_chunk_kernel<NQ, G, PF, LOG>, SLOT_THREADS, smem));
  int ctas = per_sm > 0 ? per_sm : 1;
  const int cap = opt(SDM_OPT_SLOT_CTAS_PER_SM);
  if (cap > 0 && cap < ctas) ctas = cap;
  const int grid = di->sms * ctas;
  SDM_CUDA_TRY(launch_pdl(slot_chunk_kernel<NQ, G, PF, LOG>, dim3(grid), dim3(SLOT_THREADS), smem,
                          st, a, 0));
  g_launches.fetch_add(1, std::memory_order_relaxed);
  SDM_CUDA_TRY(cudaGetLastError());
  return SDM_OK;
}

template <int NQ, int G, int PF>
sdm_status launch_slot_chunk(const SlotArgs& a, const DeviceInfo* di, cudaStream_t st) {
  return a.wlog ? launch_slot_chunk_t<NQ, G, PF, true>(a, di, st)
                : launch_slot_chunk_t<NQ, G, PF, false>(a, di, st);
}

// One time chunk [t0, t0 + ct) of the slot engine on `st`: the chunk's events, their radix
// sort by (sequence, head, slot), its long segments, then the chunk's segments.  The chunk's
// selections must be complete in the workspace (stream order, or an event `st` waits on).
sdm_status launch_slot_chunk_work(const sdm_shape& s, const WsLayout& WL, unsigned char* w,
                                  const SlotArgs& a, int t0, const DeviceInfo* di,
                                  cudaStream_t st) {
  uint32_t* k0 = reinterpret_cast<uint32_t*>(w + WL.off_k0);
  uint32_t* k1 = reinterpret_cast<uint32_t*>(w + WL.off_k1);
  uint2* v0 = reinterpret_cast<uint2*>(w + WL.off_v0);
  uint2* v1 = reinterpret_cast<uint2*>(w + WL.off_v1);
  uint32_t* hist = reinterpret_cast<uint32_t*>(w + WL.off_hist);
  uint32_t* tot = reinterpret_cast<uint32_t*>(w + WL.off_tot);
  uint32_t* offs = reinterpret_cast<uint32_t*>(w + WL.off_offs);
  uint32_t* cnt = reinterpret_cast<uint32_t*>(w + WL.off_cnt);
  uint2* hot = reinterpret_cast<uint2*>(w + WL.off_hot);
  float* y = a.y;
  const int N = a.N;
  const int bits = WL.kb.total();
  const uint32_t* ks = a.keys;
  const int d4 = s.d_v / 4;
  const int ct = s.T - t0 < WL.chunk ? s.T - t0 : WL.chunk;
  const long long E = (long long)ct * s.B * s.H * (s.W + s.R);
  const int ntiles = (int)((E + RS_TILE - 1) / RS_TILE);
  {
    ProfScope ps(SDM_KERNEL_SLOT_SORT, st);
    EventArgs ea;
    ea.idx_w = reinterpret_cast<const int32_t*>(w + WL.off_idx_w);
    ea.wt_w = reinterpret_cast<const float*>(w + WL.off_wt_w);
    ea.idx_r = reinterpret_cast<const int32_t*>(w + WL.off_idx_r);
    ea.wt_r = reinterpret_cast<const float*>(w + WL.off_wt_r);
    ea.keys = k0;
    ea.vals = v0;
    ea.y = y;
    ea.offs = offs;
    ea.counters = cnt;
    ea.B = s.B;
    ea.T = s.T;
    ea.H = s.H;
    ea.N = N;
    ea.W = s.W;
    ea.R = s.R;
    ea.ldw = WL.ldw;
    ea.ldr = WL.ldr;
    ea.d_v = s.d_v;
    ea.t0 = t0;
    ea.ct = ct;
    ea.kb = WL.kb;
    const long long crow = (long long)ct * s.B * s.H;
    long long blocks = (crow + 7) / 8;  // a warp per chunk row
    if (blocks > (long long)di->sms * 16) blocks = (long long)di->sms * 16;
    SDM_CUDA_TRY(launch_pdl(slot_events_kernel, dim3((unsigned)blocks), dim3(256), 0, st,
                            ea));
    g_launches.fetch_add(1, std::memory_order_relaxed);
    SDM_CUDA_TRY(cudaGetLastError());
    // LSD radix sort over the key bits in use
    uint32_t* ka = k0;
    uint32_t* kb = k1;
    uint2* va = v0;
    uint2* vb = v1;
    for (int shift = 0; shift < bits; shift += 8) {
      SDM_CUDA_TRY(launch_pdl<true>(radix_hist_kernel, dim3(ntiles), dim3(RS_THREADS), 0, st,
                              ka, E, shift, hist, ntiles));
      SDM_CUDA_TRY(launch_pdl<true>(radix_scan_kernel, dim3(RS_BINS), dim3(1024), 0, st,
                              hist, ntiles, tot));
      SDM_CUDA_TRY(launch_pdl<true>(radix_scatter_kernel, dim3(ntiles), dim3(RS_THREADS), RS_SCATTER_SMEM, st,
                              ka, va, kb, vb, E, shift, hist, tot, ntiles));
      g_launches.fetch_add(3, std::memory_order_relaxed);
      SDM_CUDA_TRY(cudaGetLastError());
      uint32_t* tk = ka;
      ka = kb;
      kb = tk;
      uint2* tv = va;
      va = vb;
      vb = tv;
    }
    const long long nsamp = (E + 127) / 128;
    long long lblocks = (nsamp + 255) / 256;
    if (lblocks > (long long)di->sms * 8) lblocks = (long long)di->sms * 8;
    if (lblocks < 1) lblocks = 1;
    SDM_CUDA_TRY(launch_pdl<true>(slot_long_segments_kernel, dim3((unsigned)lblocks), dim3(256), 0, st,
                            ks, E, cnt, hot, WL.hot_cap));
    g_launches.fetch_add(1, std::memory_order_relaxed);
    SDM_CUDA_TRY(cudaGetLastError());
  }
  ProfScope ps(SDM_KERNEL_SCAN_SLOT, st);
  sdm_status rc;
  if (d4 <= 32) rc = launch_slot_chunk<1, 4, 6>(a, di, st);
  else if (d4 <= 64) rc = launch_slot_chunk<2, 2, 6>(a, di, st);
  else if (d4 <= 128) rc = launch_slot_chunk<4, 4, 4>(a, di, st);
  else rc = launch_slot_chunk<8, 2, 2>(a, di, st);
  return rc;
}

// The slot engine's arguments for one call: sorted events in k0 / v0 after an even number of
// radix passes, else in k1 / v1.
sdm_status make_slot_args(const sdm_shape& s, const WsLayout& WL, unsigned char* w,
                          const float* alpha, const float* beta, const void* v, float* M,
                          float* y, float* wlog, SlotArgs* out) {
  const int passes = (WL.kb.total() + 7) / 8;
  SlotArgs& a = *out;
  a.keys = reinterpret_cast<uint32_t*>(w + (passes % 2 ? WL.off_k1 : WL.off_k0));
  a.vals = reinterpret_cast<uint2*>(w + (passes % 2 ? WL.off_v1 : WL.off_v0));
  a.offs = reinterpret_cast<uint32_t*>(w + WL.off_offs);
  a.alpha = alpha;
  a.beta = beta;
  a.v = v;
  a.M = M;
  a.y = y;
  uint32_t* cnt = reinterpret_cast<uint32_t*>(w + WL.off_cnt);  // hot count | span queue
  a.hot_count = cnt;
  a.hot_list = reinterpret_cast<uint2*>(w + WL.off_hot);
  a.span_next = cnt + 1;
  a.hot_cap = WL.hot_cap;
  a.B = s.B;
  a.T = s.T;
  a.H = s.H;
  a.N = s.S1 * s.S2;
  a.d_v = s.d_v;
  a.v_bf16 = s.in_dtype == SDM_BF16;
  a.kb = WL.kb;
  a.wlog = wlog;
  a.W = s.W;
  a.cta_stats = nullptr;
  if (opt(SDM_OPT_SLOT_CTA_STATS)) {
    void* p = nullptr;
    SDM_CUDA_TRY(cudaGetSymbolAddress(&p, g_slot_cta_stats));
    a.cta_stats = static_cast<unsigned long long*>(p);
  }
  return SDM_OK;
}

// Steps 2-3 with the slot-parallel engine, one time chunk after another on `st`, after the
// whole selection.  A chunk's events and sort buffers (tens of MB) stay in L2 between the
// steps.
sdm_status launch_slot(const sdm_shape& s, const WsLayout& WL, unsigned char* w,
                       const float* alpha, const float* beta, const void* v, float* M, float* y,
                       float* wlog, const DeviceInfo* di, cudaStream_t st) {
  SlotArgs a;
  sdm_status rc = make_slot_args(s, WL, w, alpha, beta, v, M, y, wlog, &a);
  for (int t0 = 0; rc == SDM_OK && t0 < s.T; t0 += WL.chunk)
    rc = launch_slot_chunk_work(s, WL, w, a, t0, di, st);
  return rc;
}

// Whether SDM_OPT_SELECT_SCHEDULE = 0 pipelines the slot engine's selection with its chunks.
// Long skewed step (32 chunks), ms: whole selection first 52.9, pipelined 46.6.
constexpr bool PIPELINE_BY_DEFAULT = true;

// Rows per warp of a chunk's selection launch in the pipelined schedule: CTAs that live one
// selection per warp, so that the scan's CTAs (on the higher-priority stream) take the SM
// slots they free.  Long skewed step, ms: 1 row 46.6, 2 rows 47.7, 8 rows 49.4, one
// persistent wave 48.8; 2 rows with both streams at the same priority 50.2.
constexpr int PIPE_SEL_ROWS_PER_WARP = 1;

// Streams and events of one device for the pipelined slot engine: chunk work on `hi`
// (greatest priority), selections on `lo` (least priority).  Created on first use; the
// mutex serialises the enqueueing of pipelined calls, whose event ring it protects.
struct PipeStreams {
  bool ready = false;
  cudaStream_t hi = nullptr, lo = nullptr;
  cudaEvent_t fork = nullptr, done = nullptr, sel[2] = {nullptr, nullptr};
};
std::mutex g_pipe_mu;
PipeStreams g_pipe[MAX_DEVICES];

sdm_status pipe_streams(PipeStreams** out) {
  int dev = 0;
  SDM_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= MAX_DEVICES) return SDM_ERR_UNSUPPORTED;
  PipeStreams& P = g_pipe[dev];
  if (!P.ready) {
    int least = 0, greatest = 0;
    SDM_CUDA_TRY(cudaDeviceGetStreamPriorityRange(&least, &greatest));
    SDM_CUDA_TRY(cudaStreamCreateWithPriority(&P.hi, cudaStreamNonBlocking, greatest));
    SDM_CUDA_TRY(cudaStreamCreateWithPriority(&P.lo, cudaStreamNonBlocking, least));
    cudaEvent_t* evs[] = {&P.fork, &P.done, &P.sel[0], &P.sel[1]};
    for (cudaEvent_t* e : evs) SDM_CUDA_TRY(cudaEventCreateWithFlags(e, cudaEventDisableTiming));
    P.ready = true;
  }
  *out = &P;
  return SDM_OK;
}

// The selection of time chunk [t0, t0 + ct) of every sequence, both jobs, on `q`.
sdm_status launch_select_chunk(const sdm_shape& s, const WsLayout& WL, const SelJob& jw,
                               const SelJob& jr, int bf16, int t0, cudaStream_t q) {
  const int ct = s.T - t0 < WL.chunk ? s.T - t0 : WL.chunk;
  const long long first = (long long)t0 * s.H;  // the chunk's first row of sequence 0
  const size_t row_bytes = (size_t)(s.S1 + s.S2) * (bf16 ? 2 : 4);
  SelJob cw = jw, cr = jr;
  for (SelJob* j : {&cw, &cr}) {
    j->halves = static_cast<const unsigned char*>(j->halves) + first * row_bytes;
    j->idx += first * j->ld;
    j->wt += first * j->ld;
    j->seg_rows = ct * s.H;
    j->seg_stride = (long long)s.T * s.H;
  }
  ProfScope ps(SDM_KERNEL_SELECT, q);
  return launch_select(cw, &cr, (long long)s.B * ct * s.H, s.S1, s.S2, bf16, q,
                       PIPE_SEL_ROWS_PER_WARP);
}

// Steps 1-3 with the slot engine, pipelined: chunk c + 1's selection runs on a
// low-priority stream while chunk c's sort and scan run on a high-priority one; its CTAs
// take the SM slots that the chunk work leaves (the scan's load-imbalance tail, the
// sort's narrow kernels).  Forked from and joined back to `st` with events, so `st` sees the
// same order as the serial schedule; a chunk's work waits for its own selection only.
sdm_status launch_slot_pipelined(const sdm_shape& s, const WsLayout& WL, unsigned char* w,
                                 const SelJob& jw, const SelJob& jr, int bf16,
                                 const float* alpha, const float* beta, const void* v,
                                 float* M, float* y, float* wlog, const DeviceInfo* di,
                                 cudaStream_t st) {
  SlotArgs a;
  sdm_status rc = make_slot_args(s, WL, w, alpha, beta, v, M, y, wlog, &a);
  if (rc != SDM_OK) return rc;
  std::lock_guard<std::mutex> lock(g_pipe_mu);
  PipeStreams* P;
  rc = pipe_streams(&P);
  if (rc != SDM_OK) return rc;
  SDM_CUDA_TRY(cudaEventRecord(P->fork, st));
  SDM_CUDA_TRY(cudaStreamWaitEvent(P->hi, P->fork, 0));
  SDM_CUDA_TRY(cudaStreamWaitEvent(P->lo, P->fork, 0));
  // chunk c's selection is recorded in sel[c & 1]; chunk c + 1's record is enqueued before
  // `hi` waits for chunk c, and chunk c + 2's (the same event) only after that wait, which
  // keeps the record it saw
  rc = launch_select_chunk(s, WL, jw, jr, bf16, 0, P->lo);
  if (rc != SDM_OK) return rc;
  SDM_CUDA_TRY(cudaEventRecord(P->sel[0], P->lo));
  for (int c = 0; c < WL.n_chunks; ++c) {
    if (c + 1 < WL.n_chunks) {
      rc = launch_select_chunk(s, WL, jw, jr, bf16, (c + 1) * WL.chunk, P->lo);
      if (rc != SDM_OK) return rc;
      SDM_CUDA_TRY(cudaEventRecord(P->sel[(c + 1) & 1], P->lo));
    }
    SDM_CUDA_TRY(cudaStreamWaitEvent(P->hi, P->sel[c & 1], 0));
    rc = launch_slot_chunk_work(s, WL, w, a, c * WL.chunk, di, P->hi);
    if (rc != SDM_OK) return rc;
  }
  // `hi` has waited for every selection, so `done` covers both streams
  SDM_CUDA_TRY(cudaEventRecord(P->done, P->hi));
  SDM_CUDA_TRY(cudaStreamWaitEvent(st, P->done, 0));
  return SDM_OK;
}

bool act_ok(int act) { return act >= SDM_GATE_SILU && act <= SDM_GATE_IDENTITY; }

}  // namespace

extern "C" {

const char* sdm_status_string(sdm_status status) {
  switch (status) {
    case SDM_OK: return "SDM_OK";
    case SDM_ERR_INVALID_ARG: return "SDM_ERR_INVALID_ARG";
    case SDM_ERR_UNSUPPORTED: return "SDM_ERR_UNSUPPORTED";
    case SDM_ERR_CUDA: return "SDM_ERR_CUDA";
    case SDM_ERR_DEVICE_CHECK: return "SDM_ERR_DEVICE_CHECK";
    case SDM_ERR_TIMEOUT: return "SDM_ERR_TIMEOUT";
  }
  return "SDM_ERR_UNKNOWN";
}

size_t sdm_workspace_size(sdm_shape shape, int32_t engine) {
  if (!shape_ok(shape, true)) return 0;
  if (engine < SDM_ENGINE_AUTO || engine > SDM_ENGINE_CHUNK) return 0;
  if (engine == SDM_ENGINE_SLOT && !slot_engine_fits(shape)) return 0;
  if (engine == SDM_ENGINE_CHUNK) engine = SDM_ENGINE_SEQ;  // the selection's lists only
  // AUTO may pick either engine: size for the larger
  if (engine == SDM_ENGINE_AUTO && slot_engine_fits(shape)) engine = SDM_ENGINE_SLOT;
  return ws_layout(shape, engine).total;
}

sdm_status sdm_select(const void* halves, sdm_shape shape, int32_t K, int32_t* idx, float* wt,
                      void* stream) {
  NvtxRange nvtx_range("sdm_select");
  sdm_shape s = shape;  // only B, T, H, S1, S2 and in_dtype matter here
  s.W = s.R = 1;
  s.d_v = s.in_dtype == SDM_BF16 ? 8 : 4;
  if (!shape_ok(s, true)) return SDM_ERR_INVALID_ARG;
  const int smin = s.S1 < s.S2 ? s.S1 : s.S2;
  if (K < 1 || K > smin || K > KMAX) return SDM_ERR_INVALID_ARG;
  if (!halves || !idx || !wt) return SDM_ERR_INVALID_ARG;
  if (!aligned16(halves) || !aligned16(idx) || !aligned16(wt)) return SDM_ERR_INVALID_ARG;
  SelJob j{halves, idx, wt, K, K, 0, 0};
  ProfScope ps(SDM_KERNEL_SELECT, static_cast<cudaStream_t>(stream));
  return launch_select(j, nullptr, (long long)s.B * s.T * s.H, s.S1, s.S2,
                       s.in_dtype == SDM_BF16, static_cast<cudaStream_t>(stream));
}

sdm_status sdm_state_init(const float* M0, float* M, sdm_shape shape, void* stream) {
  NvtxRange nvtx_range("sdm_state_init");
  // only B, H, N = S1*S2 and d_v matter here
  if (shape.B < 1 || shape.H < 1 || shape.S1 < 1 || shape.S2 < 1) return SDM_ERR_INVALID_ARG;
  if (shape.d_v < 4 || shape.d_v > 1024 || shape.d_v % 4 != 0) return SDM_ERR_INVALID_ARG;
  if ((long long)shape.S1 * shape.S2 > 2147483647LL) return SDM_ERR_INVALID_ARG;
  if (!M0 || !M || !aligned16(M0) || !aligned16(M)) return SDM_ERR_INVALID_ARG;
  const size_t n = state_elems(shape) * 4;
  if (overlaps(M, n, M0, n / shape.B)) return SDM_ERR_INVALID_ARG;
  ProfScope ps(SDM_KERNEL_STATE_INIT, static_cast<cudaStream_t>(stream));
  return launch_state_init(M0, M, shape, static_cast<cudaStream_t>(stream));
}

sdm_status sdm_norm_gate(const float* y, const void* gate, const float* gamma, float eps,
                         int32_t act, sdm_shape shape, float* o, void* stream) {
  NvtxRange nvtx_range("sdm_norm_gate");
  sdm_shape s = shape;  // only B, T, H, d_v and in_dtype matter here
  s.S1 = s.S2 = 1;
  s.W = s.R = 1;
  if (!shape_ok(s, true)) return SDM_ERR_INVALID_ARG;
  if (!y || !o || !act_ok(act) || !(eps >= 0.0f)) return SDM_ERR_INVALID_ARG;
  if (!aligned16(y) || !aligned16(o) || (gate && !aligned16(gate)) ||
      (gamma && !aligned16(gamma)))
    return SDM_ERR_INVALID_ARG;
  ProfScope ps(SDM_KERNEL_NORM_GATE, static_cast<cudaStream_t>(stream));
  return launch_norm_gate(y, gate, s.in_dtype == SDM_BF16, gamma, eps, act,
                          (long long)s.B * s.T * s.H, s.d_v, o,
                          static_cast<cudaStream_t>(stream));
}

// Bytes of the codes of `rows` state rows in `format` (0: invalid arguments).
static size_t rows_code_bytes(int64_t rows, int32_t d_v, int32_t format) {
  if (rows < 0 || d_v < 4 || d_v > 512 || d_v % 4 != 0) return 0;
  switch (format) {
    case SDM_ROWS_BF16: return (size_t)rows * d_v * 2;
    case SDM_ROWS_E4M3: return (size_t)rows * d_v;
    case SDM_ROWS_INT4: return (size_t)rows * d_v / 2;
  }
  return 0;
}

static unsigned rows_grid(int64_t rows, const DeviceInfo* di) {
  long long blocks = (rows + 7) / 8;  // a warp per row
  if (blocks > (long long)di->sms * 16) blocks = (long long)di->sms * 16;
  return (unsigned)(blocks > 0 ? blocks : 1);
}

// Host checks shared by the pack and unpack calls.
static sdm_status rows_check(const void* M, int64_t rows, int32_t d_v, int32_t format,
                             const void* codes, const void* scales) {
  if (rows == 0 && format >= SDM_ROWS_BF16 && format <= SDM_ROWS_INT4 && d_v >= 4 &&
      d_v <= 512 && d_v % 4 == 0)
    return SDM_OK;
  const size_t nc = rows_code_bytes(rows, d_v, format);
  if (nc == 0 || !M || !codes || !aligned16(M) || !aligned16(codes)) return SDM_ERR_INVALID_ARG;
  const size_t nm = (size_t)rows * d_v * 4;
  if (overlaps(M, nm, codes, nc)) return SDM_ERR_INVALID_ARG;
  if (format != SDM_ROWS_BF16) {
    if (!scales || (reinterpret_cast<uintptr_t>(scales) & 3u) != 0) return SDM_ERR_INVALID_ARG;
    if (overlaps(M, nm, scales, (size_t)rows * 4) || overlaps(codes, nc, scales, (size_t)rows * 4))
      return SDM_ERR_INVALID_ARG;
  }
  return SDM_OK;
}

size_t sdm_state_rows_bytes(int64_t rows, int32_t d_v, int32_t format) {
  return rows_code_bytes(rows, d_v, format);
}

sdm_status sdm_state_pack(const float* M, int64_t rows, int32_t d_v, int32_t format,
                          void* codes, float* scales, void* stream) {
  NvtxRange nvtx_range("sdm_state_pack");
  sdm_status rc = rows_check(M, rows, d_v, format, codes, scales);
  if (rc != SDM_OK || rows == 0) return rc;
  DeviceInfo* di;
  rc = device_info(&di);
  if (rc != SDM_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ProfScope ps(SDM_KERNEL_STATE_ROWS, st);
  const dim3 grid(rows_grid(rows, di)), block(256);
  if (format == SDM_ROWS_BF16)
    SDM_CUDA_TRY(launch_pdl(rows_pack_kernel<ROWS_FMT_BF16>, grid, block, 0, st, M,
                            (long long)rows, (int)d_v, codes, scales));
  else if (format == SDM_ROWS_E4M3)
    SDM_CUDA_TRY(launch_pdl(rows_pack_kernel<ROWS_FMT_E4M3>, grid, block, 0, st, M,
                            (long long)rows, (int)d_v, codes, scales));
  else
    SDM_CUDA_TRY(launch_pdl(rows_pack_kernel<ROWS_FMT_INT4>, grid, block, 0, st, M,
                            (long long)rows, (int)d_v, codes, scales));
  g_launches.fetch_add(1, std::memory_order_relaxed);
  SDM_CUDA_TRY(cudaGetLastError());
  return SDM_OK;
}

sdm_status sdm_state_unpack(const void* codes, const float* scales, int64_t rows, int32_t d_v,
                            int32_t format, float* M, void* stream) {
  NvtxRange nvtx_range("sdm_state_unpack");
  sdm_status rc = rows_check(M, rows, d_v, format, codes, scales);
  if (rc != SDM_OK || rows == 0) return rc;
  DeviceInfo* di;
  rc = device_info(&di);
  if (rc != SDM_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ProfScope ps(SDM_KERNEL_STATE_ROWS, st);
  const dim3 grid(rows_grid(rows, di)), block(256);
  if (format == SDM_ROWS_BF16)
    SDM_CUDA_TRY(launch_pdl(rows_unpack_kernel<ROWS_FMT_BF16>, grid, block, 0, st, codes,
                            scales, (long long)rows, (int)d_v, M));
  else if (format == SDM_ROWS_E4M3)
    SDM_CUDA_TRY(launch_pdl(rows_unpack_kernel<ROWS_FMT_E4M3>, grid, block, 0, st, codes,
                            scales, (long long)rows, (int)d_v, M));
  else
    SDM_CUDA_TRY(launch_pdl(rows_unpack_kernel<ROWS_FMT_INT4>, grid, block, 0, st, codes,
                            scales, (long long)rows, (int)d_v, M));
  g_launches.fetch_add(1, std::memory_order_relaxed);
  SDM_CUDA_TRY(cudaGetLastError());
  return SDM_OK;
}

// Prefill; `coupled` selects the coupled delta rule (sequential engine only).
static sdm_status scan_forward(const void* kp, const void* qp, const void* v, const float* alpha,
                               const float* beta, const float* M0, float* M, int32_t init,
                               float* y, const void* gate, const float* gamma, float eps,
                               int32_t act, float* o, int32_t* sel_out, int32_t engine, void* ws,
                               size_t ws_bytes, sdm_shape shape, void* stream, bool coupled,
                               float* wlog = nullptr) {
  const sdm_shape& s = shape;
  if (!shape_ok(s, true)) return SDM_ERR_INVALID_ARG;
  if (init != SDM_INIT_FROM_M0 && init != SDM_CONTINUE) return SDM_ERR_INVALID_ARG;
  if (engine < SDM_ENGINE_AUTO || engine > SDM_ENGINE_CHUNK) return SDM_ERR_INVALID_ARG;
  // the slot engine treats every slot as its own recurrence, which the shared prediction of
  // the coupled rule breaks
  if (coupled && engine == SDM_ENGINE_SLOT) return SDM_ERR_UNSUPPORTED;
  // the chunk-wise engine computes the per-slot rule and keeps no undo log
  if ((coupled || wlog) && engine == SDM_ENGINE_CHUNK) return SDM_ERR_UNSUPPORTED;
  if (!act_ok(act) || !(eps >= 0.0f)) return SDM_ERR_INVALID_ARG;
  if (!M || !aligned16(M)) return SDM_ERR_INVALID_ARG;
  if (init == SDM_INIT_FROM_M0) {
    if (!M0 || !aligned16(M0)) return SDM_ERR_INVALID_ARG;
    const size_t n = state_elems(s) * 4;
    if (overlaps(M, n, M0, n / s.B)) return SDM_ERR_INVALID_ARG;
  }
  if (s.T > 0) {
    if (!kp || !qp || !v || !alpha || !beta || !y) return SDM_ERR_INVALID_ARG;
    const void* ptrs[] = {kp, qp, v, alpha, beta, y, gate, gamma, o, sel_out};
    for (const void* p : ptrs)
      if (p && !aligned16(p)) return SDM_ERR_INVALID_ARG;
    if (engine == SDM_ENGINE_SLOT && !slot_engine_fits(s)) return SDM_ERR_UNSUPPORTED;
    if (wlog) {
      const size_t nlog = (size_t)s.B * s.T * s.H * s.W * s.d_v * 4;
      if (!aligned16(wlog) || overlaps(wlog, nlog, M, state_elems(s) * 4) ||
          overlaps(wlog, nlog, y, (size_t)s.B * s.T * s.H * s.d_v * 4))
        return SDM_ERR_INVALID_ARG;
    }
    const size_t need = sdm_workspace_size(s, engine);
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) % WS_ALIGN) != 0)
      return SDM_ERR_INVALID_ARG;
  }

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  sdm_status rc;
  DeviceInfo* di;
  rc = device_info(&di);
  if (rc != SDM_OK) return rc;
  engine = coupled ? SDM_ENGINE_SEQ : pick_engine(s, engine, di->sms);
  if (init == SDM_INIT_FROM_M0) {
    ProfScope ps(SDM_KERNEL_STATE_INIT, st);
    rc = launch_state_init(M0, M, s, st);
    if (rc != SDM_OK) return rc;
  }
  if (s.T == 0) return SDM_OK;

  const WsLayout WL = ws_layout(s, engine);
  unsigned char* w = static_cast<unsigned char*>(ws);
  int32_t* idx_w = reinterpret_cast<int32_t*>(w + WL.off_idx_w);
  float* wt_w = reinterpret_cast<float*>(w + WL.off_wt_w);
  int32_t* idx_r = reinterpret_cast<int32_t*>(w + WL.off_idx_r);
  float* wt_r = reinterpret_cast<float*>(w + WL.off_wt_r);
  const long long rows = (long long)s.B * s.T * s.H;
  const int bf16 = s.in_dtype == SDM_BF16;

  SelJob jw{kp, idx_w, wt_w, s.W, WL.ldw, 0, 0};
  SelJob jr{qp, idx_r, wt_r, s.R, WL.ldr, 0, 0};
  const int sched = opt(SDM_OPT_SELECT_SCHEDULE);
  const bool pipelined = engine == SDM_ENGINE_SLOT && WL.n_chunks > 1 &&
                         (sched == 2 || (sched == 0 && PIPELINE_BY_DEFAULT));
  if (pipelined) {
    rc = launch_slot_pipelined(s, WL, w, jw, jr, bf16, alpha, beta, v, M, y, wlog, di, st);
    if (rc != SDM_OK) return rc;
  } else {
    ProfScope ps(SDM_KERNEL_SELECT, st);
    rc = launch_select(jw, &jr, rows, s.S1, s.S2, bf16, st);
    if (rc != SDM_OK) return rc;
  }
  if (sel_out) {
    SDM_CUDA_TRY(cudaMemcpy2DAsync(sel_out, (size_t)s.W * 4, idx_w, (size_t)WL.ldw * 4,
                                   (size_t)s.W * 4, (size_t)rows, cudaMemcpyDeviceToDevice, st));
    SDM_CUDA_TRY(cudaMemcpy2DAsync(sel_out + (size_t)rows * s.W, (size_t)s.R * 4, idx_r,
                                   (size_t)WL.ldr * 4, (size_t)s.R * 4, (size_t)rows,
                                   cudaMemcpyDeviceToDevice, st));
  }

  if (engine == SDM_ENGINE_SLOT) {
    if (!pipelined) {
      rc = launch_slot(s, WL, w, alpha, beta, v, M, y, wlog, di, st);
      if (rc != SDM_OK) return rc;
    }
    if (o) {
      ProfScope ps(SDM_KERNEL_NORM_GATE, st);
      rc = launch_norm_gate(y, gate, bf16, gamma, eps, act, rows, s.d_v, o, st);
    }
    return rc;
  }

  SeqArgs a;
  a.idx_w = idx_w;
  a.wt_w = wt_w;
  a.idx_r = idx_r;
  a.wt_r = wt_r;
  a.alpha = alpha;
  a.beta = beta;
  a.v = v;
  a.M = M;
  a.y = y;
  a.B = s.B;
  a.T = s.T;
  a.H = s.H;
  a.N = s.S1 * s.S2;
  a.W = s.W;
  a.R = s.R;
  a.ldw = WL.ldw;
  a.ldr = WL.ldr;
  a.d_v = s.d_v;
  a.v_bf16 = bf16;
  a.coupled = coupled ? 1 : 0;
  a.wlog = wlog;
  if (engine == SDM_ENGINE_CHUNK) {
    ChunkArgs c;
    c.idx_w = idx_w;
    c.wt_w = wt_w;
    c.idx_r = idx_r;
    c.wt_r = wt_r;
    c.alpha = alpha;
    c.beta = beta;
    c.v = v;
    c.M = M;
    c.y = y;
    c.B = s.B;
    c.T = s.T;
    c.H = s.H;
    c.N = s.S1 * s.S2;
    c.W = s.W;
    c.R = s.R;
    c.ldw = WL.ldw;
    c.ldr = WL.ldr;
    c.d_v = s.d_v;
    c.v_bf16 = bf16;
    ProfScope ps(SDM_KERNEL_SCAN_CHUNK, st);
    rc = launch_chunk(c, di, st);
  } else {
    ProfScope ps(SDM_KERNEL_SCAN_SEQ, st);
    rc = launch_seq(a, st);
  }
  if (rc != SDM_OK) return rc;

  if (o) {
    ProfScope ps(SDM_KERNEL_NORM_GATE, st);
    rc = launch_norm_gate(y, gate, bf16, gamma, eps, act, rows, s.d_v, o, st);
    if (rc != SDM_OK) return rc;
  }
  return SDM_OK;
}

sdm_status sdm_scan_forward(const void* kp, const void* qp, const void* v, const float* alpha,
                            const float* beta, const float* M0, float* M, int32_t init,
                            float* y, const void* gate, const float* gamma, float eps,
                            int32_t act, float* o, int32_t* sel_out, int32_t engine, void* ws,
                            size_t ws_bytes, sdm_shape shape, void* stream) {
  NvtxRange nvtx_range("sdm_scan_forward");
  return scan_forward(kp, qp, v, alpha, beta, M0, M, init, y, gate, gamma, eps, act, o,
                      sel_out, engine, ws, ws_bytes, shape, stream, false);
}

sdm_status sdm_scan_forward_coupled(const void* kp, const void* qp, const void* v,
                                    const float* alpha, const float* beta, const float* M0,
                                    float* M, int32_t init, float* y, const void* gate,
                                    const float* gamma, float eps, int32_t act, float* o,
                                    int32_t* sel_out, int32_t engine, void* ws, size_t ws_bytes,
                                    sdm_shape shape, void* stream) {
  NvtxRange nvtx_range("sdm_scan_forward_coupled");
  return scan_forward(kp, qp, v, alpha, beta, M0, M, init, y, gate, gamma, eps, act, o,
                      sel_out, engine, ws, ws_bytes, shape, stream, true);
}

sdm_status sdm_scan_forward_logged(const void* kp, const void* qp, const void* v,
                                   const float* alpha, const float* beta, const float* M0,
                                   float* M, int32_t init, float* y, const void* gate,
                                   const float* gamma, float eps, int32_t act, float* o,
                                   int32_t* sel_out, int32_t engine, void* ws, size_t ws_bytes,
                                   sdm_shape shape, float* wlog, void* stream) {
  NvtxRange nvtx_range("sdm_scan_forward_logged");
  if (!wlog && shape.T > 0) return SDM_ERR_INVALID_ARG;
  return scan_forward(kp, qp, v, alpha, beta, M0, M, init, y, gate, gamma, eps, act, o,
                      sel_out, engine, ws, ws_bytes, shape, stream, false, wlog);
}

size_t sdm_undo_workspace_size(sdm_shape shape) {
  if (!shape_ok(shape, true)) return 0;
  return round_up((size_t)shape.B * shape.H * shape.S1 * shape.S2 * 4, WS_ALIGN);
}

sdm_status sdm_state_undo(float* M, const int32_t* sel_w, const float* wlog, sdm_shape shape,
                          void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("sdm_state_undo");
  const sdm_shape& s = shape;
  if (!shape_ok(s, true)) return SDM_ERR_INVALID_ARG;
  if (s.T == 0) return SDM_OK;
  if (!M || !sel_w || !wlog || !ws || !aligned16(M) || !aligned16(sel_w) || !aligned16(wlog) ||
      (reinterpret_cast<uintptr_t>(ws) % WS_ALIGN) != 0 || ws_bytes < sdm_undo_workspace_size(s))
    return SDM_ERR_INVALID_ARG;
  const long long rows = (long long)s.B * s.T * s.H;
  const size_t nm = state_elems(s) * 4, nsel = (size_t)rows * s.W * 4,
               nlog = (size_t)rows * s.W * s.d_v * 4, nws = sdm_undo_workspace_size(s);
  if (overlaps(M, nm, wlog, nlog) || overlaps(M, nm, sel_w, nsel) || overlaps(M, nm, ws, nws) ||
      overlaps(wlog, nlog, ws, nws) || overlaps(sel_w, nsel, ws, nws))
    return SDM_ERR_INVALID_ARG;
  DeviceInfo* di;
  sdm_status rc = device_info(&di);
  if (rc != SDM_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int N = s.S1 * s.S2;
  uint32_t* first = static_cast<uint32_t*>(ws);
  ProfScope ps(SDM_KERNEL_UNDO, st);
  SDM_CUDA_TRY(cudaMemsetAsync(first, 0xff, (size_t)s.B * s.H * N * 4, st));  // no write yet
  const long long n_writes = rows * s.W;
  long long blocks = (n_writes + 255) / 256;
  if (blocks > (long long)di->sms * 16) blocks = (long long)di->sms * 16;
  SDM_CUDA_TRY(launch_pdl(undo_first_kernel, dim3((unsigned)blocks), dim3(256), 0, st, sel_w,
                          n_writes, s.T, s.H, s.W, N, first));
  blocks = (rows + 7) / 8;  // a warp per token row
  if (blocks > (long long)di->sms * 16) blocks = (long long)di->sms * 16;
  SDM_CUDA_TRY(launch_pdl(undo_restore_kernel, dim3((unsigned)blocks), dim3(256), 0, st, M,
                          sel_w, wlog, rows, s.T, s.H, s.W, N, s.d_v,
                          static_cast<const uint32_t*>(first)));
  g_launches.fetch_add(2, std::memory_order_relaxed);
  SDM_CUDA_TRY(cudaGetLastError());
  return SDM_OK;
}

// One decode step; `chained` launches it with programmatic stream serialisation.
static sdm_status decode_step(const void* kp, const void* qp, const void* v, const float* alpha,
                              const float* beta, float* M, float* y, const void* gate,
                              const float* gamma, float eps, int32_t act, float* o,
                              int32_t* sel_out, sdm_shape shape, void* stream, bool chained,
                              bool coupled) {
  NvtxRange nvtx_range("sdm_decode_step");
  sdm_shape s = shape;
  s.T = 1;
  if (!shape_ok(s, false)) return SDM_ERR_INVALID_ARG;
  if (!act_ok(act) || !(eps >= 0.0f)) return SDM_ERR_INVALID_ARG;
  if (!kp || !qp || !v || !alpha || !beta || !M || !y) return SDM_ERR_INVALID_ARG;
  const void* ptrs[] = {kp, qp, v, alpha, beta, M, y, gate, gamma, o, sel_out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return SDM_ERR_INVALID_ARG;
  DeviceInfo* di;
  sdm_status rc = device_info(&di);
  if (rc != SDM_OK) return rc;
  const bool fast = fast_select_ok(s.in_dtype == SDM_BF16, s.S1, s.S2, s.W > s.R ? s.W : s.R);
  const int need_e = fast ? ((s.S1 > s.S2 ? s.S1 : s.S2) <= 512 ? 1 : 2) : 0;
  const int need_kc = (s.W > s.R ? s.W : s.R) <= 64 ? 64 : 128;
  const int need_nq = (s.d_v / 4 + 31) / 32;
#define SDM_DEC_FITS(E, KC, NQ) \
  ((fast ? (E >= need_e && E > 0) : E == 0) && KC >= need_kc && NQ >= need_nq)
  const DecLayout L = dec_layout(s.S1, s.S2, s.W, s.R, s.d_v, fast, coupled);
  if (L.total > (size_t)di->max_smem_optin) return SDM_ERR_UNSUPPORTED;
  // the coupled rule sums the write rows staged in shared memory
  if (coupled && !L.rows_smem) return SDM_ERR_UNSUPPORTED;
  DecodeArgs a;
  a.kp = kp;
  a.qp = qp;
  a.v = v;
  a.alpha = alpha;
  a.beta = beta;
  a.M = M;
  a.y = y;
  a.gate = gate;
  a.gamma = gamma;
  a.o = o;
  a.sel_out = sel_out;
  a.eps = eps;
  a.act = act;
  a.BH = s.B * s.H;
  a.S1 = s.S1;
  a.S2 = s.S2;
  a.W = s.W;
  a.R = s.R;
  a.N = s.S1 * s.S2;
  a.d_v = s.d_v;
  a.in_bf16 = s.in_dtype == SDM_BF16;
  ProfScope ps(SDM_KERNEL_DECODE, static_cast<cudaStream_t>(stream));
  bool launched = false;
  // Chained: programmatic stream serialisation.  The step's selection (which reads only its
  // inputs) may then overlap the end of the kernel ahead of it; the kernel waits for that
  // kernel before its first state access.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.BH);
  cfg.blockDim = dim3(DEC_THREADS);
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = chained && pdl_enabled() ? 1 : 0;
#define SDM_DEC_LAUNCH(E, KC, NQ)                                                        \
  if (!launched && SDM_DEC_FITS(E, KC, NQ)) {                                             \
    if (coupled)                                                                          \
      SDM_CUDA_TRY(cudaLaunchKernelEx(&cfg, decode_kernel<E, KC, NQ, true>, a, L));      \
    else                                                                                  \
      SDM_CUDA_TRY(cudaLaunchKernelEx(&cfg, decode_kernel<E, KC, NQ, false>, a, L));     \
    g_launches.fetch_add(1, std::memory_order_relaxed);                                   \
    launched = true;                                                                      \
  }
  SDM_DEC_VARIANTS(SDM_DEC_LAUNCH)
#undef SDM_DEC_LAUNCH
#undef SDM_DEC_FITS
  if (!launched) return SDM_ERR_UNSUPPORTED;
  SDM_CUDA_TRY(cudaGetLastError());
  return SDM_OK;
}

sdm_status sdm_decode_step(const void* kp, const void* qp, const void* v, const float* alpha,
                           const float* beta, float* M, float* y, const void* gate,
                           const float* gamma, float eps, int32_t act, float* o,
                           int32_t* sel_out, sdm_shape shape, void* stream) {
  return decode_step(kp, qp, v, alpha, beta, M, y, gate, gamma, eps, act, o, sel_out, shape,
                     stream, false, false);
}

sdm_status sdm_decode_step_chained(const void* kp, const void* qp, const void* v,
                                   const float* alpha, const float* beta, float* M, float* y,
                                   const void* gate, const float* gamma, float eps, int32_t act,
                                   float* o, int32_t* sel_out, sdm_shape shape, void* stream) {
  return decode_step(kp, qp, v, alpha, beta, M, y, gate, gamma, eps, act, o, sel_out, shape,
                     stream, true, false);
}

sdm_status sdm_decode_step_coupled(const void* kp, const void* qp, const void* v,
                                   const float* alpha, const float* beta, float* M, float* y,
                                   const void* gate, const float* gamma, float eps, int32_t act,
                                   float* o, int32_t* sel_out, sdm_shape shape, void* stream) {
  return decode_step(kp, qp, v, alpha, beta, M, y, gate, gamma, eps, act, o, sel_out, shape,
                     stream, false, true);
}

sdm_status sdm_decode_step_coupled_chained(const void* kp, const void* qp, const void* v,
                                           const float* alpha, const float* beta, float* M,
                                           float* y, const void* gate, const float* gamma,
                                           float eps, int32_t act, float* o, int32_t* sel_out,
                                           sdm_shape shape, void* stream) {
  return decode_step(kp, qp, v, alpha, beta, M, y, gate, gamma, eps, act, o, sel_out, shape,
                     stream, true, true);
}

sdm_status sdm_get_device_status(void* stream) {
  SDM_CUDA_TRY(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  unsigned int v = 0, zero = 0;
  SDM_CUDA_TRY(cudaMemcpyFromSymbol(&v, g_status, sizeof(v)));
  SDM_CUDA_TRY(cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)));
  if (v & STATUS_TIMEOUT) return SDM_ERR_TIMEOUT;
  if (v & STATUS_BAD_INDEX) return SDM_ERR_DEVICE_CHECK;
  return SDM_OK;
}

uint64_t sdm_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

sdm_status sdm_set_option(int32_t option, int32_t value) {
  bool ok = false;
  switch (option) {
    case SDM_OPT_NO_PDL:
    case SDM_OPT_SELECT_GENERAL: ok = value == 0 || value == 1; break;
    case SDM_OPT_SELECT_CTAS_PER_SM:
    case SDM_OPT_SLOT_CTAS_PER_SM: ok = value >= 0 && value <= 64; break;
    case SDM_OPT_SEQ_COLUMNS: ok = value == 0 || value == 4 || value == 8 || value == 16 || value == 32; break;
    case SDM_OPT_SEQ_DEPTH: ok = value == 0 || value == 4 || value == 8; break;
    case SDM_OPT_SLOT_CTA_STATS: ok = value == 0 || value == 1; break;
    case SDM_OPT_SELECT_SCHEDULE: ok = value >= 0 && value <= 2; break;
    default: ok = false;
  }
  if (!ok) return SDM_ERR_INVALID_ARG;
  g_opt[option].store(value, std::memory_order_relaxed);
  return SDM_OK;
}

int32_t sdm_get_option(int32_t option) {
  if (option < SDM_OPT_NO_PDL || option > SDM_OPT_SELECT_SCHEDULE) return -1;
  return opt(option);
}

sdm_status sdm_slot_cta_stats(uint64_t* out, int32_t max_ctas, int32_t reset) {
  if (!out || max_ctas < 1 || max_ctas > SDM_SLOT_STATS_CTAS) return SDM_ERR_INVALID_ARG;
  SDM_CUDA_TRY(cudaDeviceSynchronize());
  SDM_CUDA_TRY(cudaMemcpyFromSymbol(out, g_slot_cta_stats, (size_t)max_ctas * 4 * 8));
  if (reset) {
    void* p = nullptr;
    SDM_CUDA_TRY(cudaGetSymbolAddress(&p, g_slot_cta_stats));
    SDM_CUDA_TRY(cudaMemset(p, 0, sizeof(unsigned long long) * 4 * SDM_SLOT_STATS_CTAS));
  }
  return SDM_OK;
}

sdm_status sdm_profile_enable(int32_t on) {
  std::vector<ProfRec> drop;
  {
    std::lock_guard<std::mutex> lock(g_prof_mu);
    g_prof_on = on != 0;
    drop.swap(g_prof_pending);
  }
  for (ProfRec& r : drop) {
    cudaEventSynchronize(r.stop);
    cudaEventDestroy(r.start);
    cudaEventDestroy(r.stop);
  }
  return SDM_OK;
}

sdm_status sdm_profile_read(double* ms, int64_t* launches) {
  if (!ms || !launches) return SDM_ERR_INVALID_ARG;
  std::vector<ProfRec> recs;
  {
    std::lock_guard<std::mutex> lock(g_prof_mu);
    recs.swap(g_prof_pending);
  }
  for (int k = 0; k < SDM_KERNEL_KINDS; ++k) {
    ms[k] = 0.0;
    launches[k] = 0;
  }
  sdm_status rc = SDM_OK;
  for (ProfRec& r : recs) {
    float t = 0.0f;
    if (cudaEventSynchronize(r.stop) != cudaSuccess ||
        cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess) {
      (void)cudaGetLastError();
      rc = SDM_ERR_CUDA;
    } else if (r.kind >= 0 && r.kind < SDM_KERNEL_KINDS) {
      ms[r.kind] += t;
      launches[r.kind] += 1;
    }
    cudaEventDestroy(r.start);
    cudaEventDestroy(r.stop);
  }
  return rc;
}

}  // extern "C"

// ------------------------------------------------------------------------------------
// Prefill without any allocation.
//
// Some callers cannot allocate device memory at the time they run the pass: a host engine
// that hands all device memory to its own pool at start-up, a plugin interface that
// offers no workspace argument, or a real-time loop that must not call the CUDA allocator
// (cudaMalloc and cudaFree can synchronise the device) once it is running.  For them,
// sdm_scan_forward_noalloc takes the scratch of the sequential engine from a fixed
// file-scope device array instead of from a caller buffer.  The array exists once per
// device that loads this library and stays allocated until the process exits.
__device__ __align__(256) unsigned char g_noalloc_scratch[SDM_NOALLOC_SCRATCH_BYTES];

namespace {
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[MAX_DEVICES];  // device address of g_noalloc_scratch, per device

// The device address of the array on the current device.  In host code the array's name
// is only a host-side stand-in, so the address comes from cudaGetSymbolAddress, once per
// device, with that device current.
sdm_status noalloc_scratch(void** out) {
  int dev = 0;
  SDM_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= MAX_DEVICES) return SDM_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      (void)cudaGetLastError();
      return SDM_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return SDM_OK;
}
}  // namespace

extern "C" sdm_status sdm_scan_forward_noalloc(const void* kp, const void* qp, const void* v,
                                               const float* alpha, const float* beta,
                                               const float* M0, float* M, int32_t init,
                                               float* y, const void* gate, const float* gamma,
                                               float eps, int32_t act, float* o,
                                               int32_t* sel_out, sdm_shape shape,
                                               void* stream) {
  NvtxRange nvtx_range("sdm_scan_forward_noalloc");
  if (!shape_ok(shape, true)) return SDM_ERR_INVALID_ARG;
  if (sdm_workspace_size(shape, SDM_ENGINE_SEQ) > (size_t)SDM_NOALLOC_SCRATCH_BYTES)
    return SDM_ERR_INVALID_ARG;
  void* ws = nullptr;
  const sdm_status rc = noalloc_scratch(&ws);
  if (rc != SDM_OK) return rc;
  return sdm_scan_forward(kp, qp, v, alpha, beta, M0, M, init, y, gate, gamma, eps, act, o,
                          sel_out, SDM_ENGINE_SEQ, ws, SDM_NOALLOC_SCRATCH_BYTES, shape,
                          stream);
}
