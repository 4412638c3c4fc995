// Host side of the C ABI: argument checks, workspace layout, kernel selection and launches.
//
// Every check happens before the first CUDA call that could launch work, so a refused call
// launches nothing (the serve predicate of metrale "forward_bf16_grouped_decode.rs": the grouped
// decode launches nothing unless its predicate holds).
#include <cmath>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <cstdlib>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "experts.cuh"
#include "fused.cuh"
#include "router.cuh"
#include "tc.cuh"

using namespace moe;

namespace {

thread_local int g_last_cuda_error = 0;

int cuda_fail(cudaError_t e) {
  g_last_cuda_error = (int)e;
  return MOE_ERR_CUDA;
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

int check_cfg(const moe_cfg* c, int m) {
  if (!c) return MOE_ERR_NULL_POINTER;
  if (m < 1 || m > MOE_MAX_ROWS) return MOE_ERR_BAD_SHAPE;
  if (c->hidden <= 0 || c->hidden % 8) return MOE_ERR_BAD_SHAPE;
  if (c->num_experts < 1 || c->num_experts > MOE_MAX_EXPERTS) return MOE_ERR_BAD_SHAPE;
  if (c->top_k < 1 || c->top_k > MOE_MAX_TOP_K || c->top_k > c->num_experts)
    return MOE_ERR_BAD_SHAPE;
  if (c->moe_inter <= 0 || c->moe_inter % 4 || c->shared_inter < 0) return MOE_ERR_BAD_SHAPE;
  if (c->routing < MOE_ROUTE_SOFTMAX || c->routing > MOE_ROUTE_SQRTSOFTPLUS) return MOE_ERR_BAD_OPTION;
  if (c->activation != MOE_ACT_SWIGLU && c->activation != MOE_ACT_GEGLU) return MOE_ERR_BAD_OPTION;
  auto is01 = [](int v) { return v == 0 || v == 1; };
  if (!is01(c->norm_topk_prob) || !is01(c->select_on_raw_logits) || !is01(c->has_expert_bias) ||
      !is01(c->weight_before_ffn))
    return MOE_ERR_BAD_OPTION;
  if (c->routing == MOE_ROUTE_SOFTMAX && (c->select_on_raw_logits || c->has_expert_bias))
    return MOE_ERR_BAD_OPTION;
  if (c->select_on_raw_logits && c->has_expert_bias) return MOE_ERR_BAD_OPTION;
  if (!std::isfinite(c->routed_scaling_factor)) return MOE_ERR_BAD_OPTION;
  if (c->shared_kind < MOE_SHARED_NONE || c->shared_kind > MOE_SHARED_SIGMOID_GATE)
    return MOE_ERR_BAD_OPTION;
  if (c->shared_kind != MOE_SHARED_NONE && c->shared_inter <= 0) return MOE_ERR_BAD_SHAPE;
  if (c->shared_kind == MOE_SHARED_NONE && c->shared_inter != 0) return MOE_ERR_BAD_OPTION;
  if (c->shared_inter % 4) return MOE_ERR_BAD_SHAPE;
  if (c->x_dtype != MOE_FMT_F32 && c->x_dtype != MOE_FMT_BF16) return MOE_ERR_BAD_FORMAT;
  if (c->out_dtype != MOE_FMT_F32 && c->out_dtype != MOE_FMT_BF16) return MOE_ERR_BAD_FORMAT;
  return MOE_OK;
}

// k-dimension rule of each format: 16-byte packed rows, whole scale groups.
bool k_ok(int fmt, int k) {
  switch (fmt) {
    case MOE_FMT_F32: return k % 4 == 0;
    case MOE_FMT_BF16: return k % 8 == 0;
    case MOE_FMT_Q4_AFFINE_G64: return k % 64 == 0;
    case MOE_FMT_NVFP4: return k % 32 == 0;
    case MOE_FMT_MXFP4: return k % 32 == 0;
    case MOE_FMT_FP8_E4M3: return k % 16 == 0;
    default: return false;
  }
}

int check_matrix(const moe_matrix& M, int n, int k, int E, MatDev* out) {
  if (M.format < MOE_FMT_F32 || M.format > MOE_FMT_FP8_E4M3) return MOE_ERR_BAD_FORMAT;
  if (!k_ok(M.format, k)) return MOE_ERR_BAD_FORMAT;
  if (!M.packed) return MOE_ERR_NULL_POINTER;
  if (!aligned(M.packed, 16)) return MOE_ERR_MISALIGNED;
  const size_t mat_bytes = packed_row_bytes(M.format, k) * (size_t)n;
  if (E > 1 && (M.expert_stride < (int64_t)mat_bytes || M.expert_stride % 16))
    return M.expert_stride % 16 ? MOE_ERR_MISALIGNED : MOE_ERR_BAD_SHAPE;
  size_t scale_bytes = 0;
  if (M.format == MOE_FMT_Q4_AFFINE_G64) {
    if (!M.scales || !M.biases) return MOE_ERR_NULL_POINTER;
    if (!aligned(M.scales, 2) || !aligned(M.biases, 2)) return MOE_ERR_MISALIGNED;
    scale_bytes = (size_t)n * (k / 64) * 2;
  } else if (M.format == MOE_FMT_NVFP4) {
    if (!M.scales || !M.tensor_scale) return MOE_ERR_NULL_POINTER;
    if (!aligned(M.scales, 2) || !aligned(M.tensor_scale, 4)) return MOE_ERR_MISALIGNED;
    scale_bytes = (size_t)n * (k / 16);
  } else if (M.format == MOE_FMT_MXFP4) {
    if (!M.scales) return MOE_ERR_NULL_POINTER;
    scale_bytes = (size_t)n * (k / 32);
  } else if (M.format == MOE_FMT_FP8_E4M3) {
    if (!M.tensor_scale) return MOE_ERR_NULL_POINTER;
    if (!aligned(M.tensor_scale, 4)) return MOE_ERR_MISALIGNED;
  }
  const int64_t salign = M.format == MOE_FMT_MXFP4 ? 1 : 2;  // scale element bytes
  if (scale_bytes && E > 1 && (M.scale_stride < (int64_t)scale_bytes || M.scale_stride % salign))
    return M.scale_stride % salign ? MOE_ERR_MISALIGNED : MOE_ERR_BAD_SHAPE;
  out->packed = (const uint8_t*)M.packed;
  out->scales = (const uint8_t*)M.scales;
  out->biases = (const uint8_t*)M.biases;
  out->tscale = M.tensor_scale;
  out->estride = E > 1 ? M.expert_stride : (long long)mat_bytes;
  out->sstride = E > 1 ? M.scale_stride : (long long)scale_bytes;
  out->fmt = M.format;
  out->n = n;
  out->k = k;
  return MOE_OK;
}

int check_table(const moe_expert_table* t, int inter, int h, int E, MatDev* g, MatDev* u,
                MatDev* d) {
  if (!t) return MOE_ERR_NULL_POINTER;
  if (t->gate.format != t->up.format) return MOE_ERR_BAD_FORMAT;
  int rc;
  if ((rc = check_matrix(t->gate, inter, h, E, g))) return rc;
  if ((rc = check_matrix(t->up, inter, h, E, u))) return rc;
  if ((rc = check_matrix(t->down, h, inter, E, d))) return rc;
  return MOE_OK;
}

int n_tiles_c_of(int h) { return (h + kColsPerCta - 1) / kColsPerCta; }

// ---- tensor-core path: work shape and workspace regions ----------------------------------------

// Split jobs keep their chunk values in the workspace: 32 floats per (activation column, job
// tile, chunk). A phase may split its jobs when that storage stays within this size.
constexpr size_t kSlotCapBytes = 24u << 20;
// Down rows of a call are asked into L2 during gate/up when they total at most this many bytes
// (well inside the 126 MB L2, next to the gate/up stream passing through it).
constexpr long long kDownPrefetchCap = 48LL << 20;

// Everything the tensor-core regions and work split depend on, from (cfg, m) alone.
struct TcShape {
  int ntg, ncg_max, tiles_i, tiles_s, tiles_h, nch_h, nch_i, nch_s;
  int j_gu_max, j_dn_max;
  size_t gu_bytes, dn_bytes;           // chunk-value storage of the two phases
  bool gu_slots, dn_slots;             // within the cap: the phase may split its jobs
};

// fmt: the format whose chunk size counts the chunks; the workspace is sized with bf16's, the
// smallest chunk (the most chunks).
TcShape tc_shape(const moe_cfg& c, int m, int fmt = MOE_FMT_BF16) {
  TcShape t;
  const bool has_shared = c.shared_kind != MOE_SHARED_NONE;
  const int S = has_shared ? c.shared_inter : 0;
  // n-tiles of 8 activation columns per pass. One, so that a CTA runs as many warps as its
  // format allows (16; 8 for NVFP4: more latency hidden, no MMAs on absent columns) even though a slot with many columns (the shared expert)
  // then streams its weight tiles once per 8 columns, mostly from L2. Two for Q4 above 8 rows
  // (its decode and post-scale work per weight byte is the largest) and for bf16 layers with a
  // shared expert above 32 rows (a shared expert as large as Llama-4-Scout's, read 8 times
  // from L2 per call, costs more than the smaller CTA). Measured on the B200 at m = 16..64.
  const bool q4 = fmt == MOE_FMT_Q4_AFFINE_G64;
  t.ntg = q4 ? (m <= 8 ? 1 : 2) : (fmt == MOE_FMT_BF16 && has_shared && m > 32) ? 2 : 1;
  t.ncg_max = tc::ceil_div(m, 8);  // column groups at the smallest width (any format)
  t.tiles_i = tc::ceil_div(c.moe_inter, 16);
  t.tiles_s = S ? tc::ceil_div(S, 16) : 0;
  t.tiles_h = tc::ceil_div(c.hidden, 32);
  t.nch_h = tc::n_chunks(c.hidden, fmt);
  t.nch_i = tc::n_chunks(c.moe_inter, fmt);
  t.nch_s = S ? tc::n_chunks(S, fmt) : 1;
  const int te = m * c.top_k;
  const int cap = te < c.num_experts ? te : c.num_experts;
  t.j_gu_max = cap * t.tiles_i + t.tiles_s;
  t.j_dn_max = (cap + (has_shared ? 1 : 0)) * t.tiles_h;
  t.gu_bytes = ((size_t)te * t.tiles_i + (size_t)m * t.tiles_s) * t.nch_h * 32 * 4;
  t.dn_bytes = ((size_t)te * t.tiles_h * t.nch_i + (has_shared ? (size_t)m * t.tiles_h * t.nch_s : 0)) *
               32 * 4;
  t.gu_slots = t.gu_bytes <= kSlotCapBytes;
  t.dn_slots = t.dn_bytes <= kSlotCapBytes;
  return t;
}

struct TcLayout {
  size_t xb, act, sh_act, slot_beg, slot_n, gu_slots, dn_slots, tk, stamps, end;
  int tk_words;
};

TcLayout tc_layout(const moe_cfg& c, int m, size_t off) {
  const TcShape t = tc_shape(c, m);
  const bool has_shared = c.shared_kind != MOE_SHARED_NONE;
  const int S = has_shared ? c.shared_inter : 0;
  const size_t te = (size_t)m * c.top_k;
  const size_t cap = te < (size_t)c.num_experts ? te : (size_t)c.num_experts;
  TcLayout L;
  auto take = [&](size_t bytes) { size_t at = off; off = align256(off + bytes); return at; };
  L.xb = take((size_t)m * c.hidden * 2);
  L.act = take(te * c.moe_inter * 4);                   // hi and lo halves
  L.sh_act = take((size_t)m * (S > 0 ? S : 1) * 4);
  L.slot_beg = take(cap * 4);
  L.slot_n = take(cap * 4);
  // slot storage: the most any call with at most m rows uses, so that the workspace size only
  // grows with m (a workspace sized for the largest m serves every smaller one)
  size_t gu_bytes = 0, dn_bytes = 0;
  for (int mm = 1; mm <= m; ++mm) {
    const TcShape u = tc_shape(c, mm);
    if (u.gu_slots && u.gu_bytes > gu_bytes) gu_bytes = u.gu_bytes;
    if (u.dn_slots && u.dn_bytes > dn_bytes) dn_bytes = u.dn_bytes;
  }
  L.gu_slots = take(gu_bytes);
  L.dn_slots = take(dn_bytes);
  // job tickets of both phases, column-tile tickets, per-slot ready counters (cap + shared)
  L.tk_words = (t.j_gu_max + t.j_dn_max) * t.ncg_max + t.tiles_h + (int)cap + 1;
  L.tk = take((size_t)L.tk_words * 4);
#ifdef MOE_PHASE_TIMERS
  L.stamps = take((size_t)1024 * 16 * 8);  // [CTA][16] uint64, last region of the workspace
#else
  L.stamps = 0;
#endif
  L.end = off;
  return L;
}

WsLayout base_layout_of(const moe_cfg* c, int m) {
  return make_layout(m, c->hidden, c->num_experts, c->top_k, c->moe_inter, c->shared_inter,
                     n_tiles_c_of(c->hidden));
}

// The whole workspace: the regions every path uses, then the tensor-core path's.
WsLayout layout_of(const moe_cfg* c, int m) {
  WsLayout L = base_layout_of(c, m);
  L.total = tc_layout(*c, m, L.total).end;
  return L;
}

// NVTX range around a library call (visible in Nsight timelines; a few ns when no tool listens).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};

// One line on stderr the first time each (launch path, format, m) combination is dispatched,
// when the environment variable MOE_DECODE_LOG is set to anything but "" or "0" (read once per
// process; it changes nothing but this log).
void log_dispatch_once(const char* path, int fmt, int m, int launches) {
  static const bool on = [] {
    const char* e = std::getenv("MOE_DECODE_LOG");
    return e && *e && std::strcmp(e, "0") != 0;
  }();
  if (!on) return;
  static std::mutex mu;
  static unsigned long long seen[2][8] = {};  // bit m-1 of seen[path is chain][format]
  std::lock_guard<std::mutex> lock(mu);
  const int chain = path[0] == 'c';
  unsigned long long& mask = seen[chain][fmt & 7];
  const unsigned long long bit = 1ull << ((m - 1) & 63);
  if (mask & bit) return;
  mask |= bit;
  std::fprintf(stderr, "[moe_decode] m=%d format=%d: %s (%d launch%s)\n", m, fmt, path, launches,
               launches == 1 ? "" : "es");
}

// Compute capability 10.0 check, cached per device.
int check_device() {
  static std::mutex mu;
  static int state[64] = {0};  // 0 unknown, 1 ok, 2 unsupported
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= 64) return MOE_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lock(mu);
  if (state[dev] == 0) {
    int major = 0, minor = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) ||
        (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)))
      return cuda_fail(e);
    state[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  return state[dev] == 1 ? MOE_OK : MOE_ERR_UNSUPPORTED_DEVICE;
}

// Launch with programmatic stream serialisation (PDL) so a kernel's prologue overlaps the
// previous kernel's tail; smem > 48 KB is opted into once per kernel.
template <typename K>
cudaError_t launch(K kernel, int grid, int block, size_t smem, cudaStream_t st, const Params& p,
                   bool pdl) {
  if (smem > 48 * 1024) {
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, p);
}

// Rows staged per pass: as many (1, 2 or 4) as fit a 80 KB staging budget, never more than m.
int rows_per_pass(int K, int fmt, int m) {
  const size_t per_row = (size_t)K * 4 + (fmt == MOE_FMT_Q4_AFFINE_G64 ? (size_t)K / 8 : 0);
  int rb = 4;
  while (rb > 1 && per_row * rb > 80 * 1024) rb >>= 1;
  while (rb > 1 && rb / 2 >= m) rb >>= 1;
  return rb;
}

size_t staging_bytes(int K, int fmt, int rb) {
  return (size_t)rb * K * 4 + (fmt == MOE_FMT_Q4_AFFINE_G64 ? (size_t)rb * (K / 32) * 4 : 0);
}

template <int FMT, bool XBF16>
cudaError_t launch_gate_up_fmt(int rb, int grid, size_t smem, cudaStream_t st, const Params& p) {
  switch (rb) {
    case 1: return launch(gate_up_swiglu_kernel<FMT, XBF16, 1>, grid, kThreads, smem, st, p, true);
    case 2: return launch(gate_up_swiglu_kernel<FMT, XBF16, 2>, grid, kThreads, smem, st, p, true);
    default: return launch(gate_up_swiglu_kernel<FMT, XBF16, 4>, grid, kThreads, smem, st, p, true);
  }
}

template <bool XBF16>
cudaError_t launch_gate_up(int fmt, int rb, int grid, size_t smem, cudaStream_t st,
                           const Params& p) {
  switch (fmt) {
    case MOE_FMT_F32: return launch_gate_up_fmt<MOE_FMT_F32, XBF16>(rb, grid, smem, st, p);
    case MOE_FMT_BF16: return launch_gate_up_fmt<MOE_FMT_BF16, XBF16>(rb, grid, smem, st, p);
    case MOE_FMT_Q4_AFFINE_G64:
      return launch_gate_up_fmt<MOE_FMT_Q4_AFFINE_G64, XBF16>(rb, grid, smem, st, p);
    case MOE_FMT_NVFP4: return launch_gate_up_fmt<MOE_FMT_NVFP4, XBF16>(rb, grid, smem, st, p);
    case MOE_FMT_MXFP4: return launch_gate_up_fmt<MOE_FMT_MXFP4, XBF16>(rb, grid, smem, st, p);
    default: return launch_gate_up_fmt<MOE_FMT_FP8_E4M3, XBF16>(rb, grid, smem, st, p);
  }
}

template <int FMT>
cudaError_t launch_down_fmt(int rb, int grid, size_t smem, cudaStream_t st, const Params& p) {
  switch (rb) {
    case 1: return launch(down_blend_kernel<FMT, 1>, grid, kThreads, smem, st, p, true);
    case 2: return launch(down_blend_kernel<FMT, 2>, grid, kThreads, smem, st, p, true);
    default: return launch(down_blend_kernel<FMT, 4>, grid, kThreads, smem, st, p, true);
  }
}

cudaError_t launch_down(int fmt, int rb, int grid, size_t smem, cudaStream_t st,
                        const Params& p) {
  switch (fmt) {
    case MOE_FMT_F32: return launch_down_fmt<MOE_FMT_F32>(rb, grid, smem, st, p);
    case MOE_FMT_BF16: return launch_down_fmt<MOE_FMT_BF16>(rb, grid, smem, st, p);
    case MOE_FMT_Q4_AFFINE_G64: return launch_down_fmt<MOE_FMT_Q4_AFFINE_G64>(rb, grid, smem, st, p);
    case MOE_FMT_NVFP4: return launch_down_fmt<MOE_FMT_NVFP4>(rb, grid, smem, st, p);
    case MOE_FMT_MXFP4: return launch_down_fmt<MOE_FMT_MXFP4>(rb, grid, smem, st, p);
    default: return launch_down_fmt<MOE_FMT_FP8_E4M3>(rb, grid, smem, st, p);
  }
}

// ---- persistent single-kernel path (m <= 4) --------------------------------------------------

int sm_count() {
  static std::mutex mu;
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) cudaDeviceGetAttribute(&cache[dev], cudaDevAttrMultiProcessorCount, dev);
  return cache[dev];
}

// Launch-path override for tests (moe_debug_set_path): 0 automatic, 1 the multi-kernel chain.
std::atomic<int> g_forced_path{0};
int forced_path() { return g_forced_path.load(std::memory_order_relaxed); }
// Work-split override for tests (moe_debug_set_split): 0 automatic, 1 whole jobs per warp,
// 2 jobs split by chunk wherever the workspace holds their chunk values.
std::atomic<int> g_forced_split{0};

size_t align16(size_t v) { return (v + 15) & ~size_t(15); }

constexpr long long kSpinLimit = 2000000000LL;  // about a second of SM clock cycles
// Failure-detection test settings (moe_debug_barrier_test); zero in normal use.
std::atomic<int> g_test_bar_extra{0};
std::atomic<long long> g_test_spin_limit{0};
constexpr size_t kFusedSmemBudget = 220 * 1024;

// Shared-memory plan of the persistent kernel; false when the layer does not fit it.
bool plan_fused(const moe_cfg& c, int m, bool has_shared, int fmt, int sms, FusedPlan* fp) {
  if (m > kFusedMaxRows || sms <= 0) return false;
  const int h = c.hidden, I = c.moe_inter, S = has_shared ? c.shared_inter : 0;
  const int te = m * c.top_k, n_rows = te + (has_shared ? m : 0);
  const int kmax = S > I ? S : I;
  const int ld = (kmax + 31) / 32 * 32;
  const int cols = (h + sms - 1) / sms;
  const bool q4 = fmt == MOE_FMT_Q4_AFFINE_G64;
  size_t off = 0;
  fp->xs_off = (int)off;
  off += align16((size_t)m * h * 4);
  fp->xsum_off = (int)off;
  off += q4 ? align16((size_t)m * (h / 32) * 4) : 0;
  fp->act_off = (int)off;
  off += align16((size_t)n_rows * ld * 4);
  fp->actsum_off = (int)off;
  off += q4 ? align16((size_t)n_rows * (ld / 32) * 4) : 0;
  fp->y_off = (int)off;
  off += align16((size_t)n_rows * cols * 4);
  if (off > kFusedSmemBudget) return false;
  // down-row tile: as many phase-E slots (column block of one expert's down rows, with their
  // scale rows) as the rest of the budget holds, up to every slot a call can have
  const size_t prb = packed_row_bytes(fmt, kmax);
  const size_t srb = q4 ? (size_t)(kmax / 64) * 2
                     : fmt == MOE_FMT_NVFP4 ? (size_t)(kmax / 16)
                     : fmt == MOE_FMT_MXFP4 ? (size_t)(kmax / 32) : 0;
  const size_t wblk = align16(cols * prb), sblk = align16(cols * srb);
  const size_t slot_bytes = wblk + (q4 ? 2 * sblk : sblk);
  const int max_slots = (c.top_k * m < c.num_experts ? c.top_k * m : c.num_experts) +
                        (has_shared ? 1 : 0);
  size_t n_fit = (kFusedSmemBudget - off) / slot_bytes;
  if (n_fit > (size_t)max_slots) n_fit = (size_t)max_slots;
  fp->tile_off = (int)off;
  fp->tile_slots = (int)n_fit;
  fp->tile_slot_bytes = (int)slot_bytes;
  fp->tile_sc_off = (int)wblk;
  fp->tile_bi_off = (int)(wblk + sblk);
  off += n_fit * slot_bytes;
  fp->grid = sms;
  fp->cols_per_cta = cols;
  fp->act_ld = ld;
  fp->smem_bytes = (int)off;
  fp->spin_limit = g_test_spin_limit.load() > 0 ? g_test_spin_limit.load() : kSpinLimit;
  fp->tile_limit = kSpinLimit;
  fp->bar_extra = (unsigned)g_test_bar_extra.load();
  fp->l2_prefetch_cap = 48LL << 20;
  return true;
}

template <int FMT, bool XBF16, int RB>
cudaError_t launch_fused_t(const Params& p, const FusedPlan& fp, cudaStream_t st) {
  auto kernel = moe_fused_kernel<FMT, XBF16, RB>;
  static bool attr_done = false;
  {
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    if (!attr_done) {
      const cudaError_t e = cudaFuncSetAttribute(
          kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kFusedSmemBudget);
      if (e != cudaSuccess) return e;
      attr_done = true;
    }
  }
  // every CTA must be resident at once: one CTA per SM, checked for this shared-memory size
  int per_sm = 0;
  cudaError_t oe = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kFusedThreads,
                                                                 fp.smem_bytes);
  if (oe != cudaSuccess) return oe;
  if (per_sm < 1) return cudaErrorCooperativeLaunchTooLarge;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(fp.grid);
  cfg.blockDim = dim3(kFusedThreads);
  cfg.dynamicSmemBytes = fp.smem_bytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, p, fp);
}

template <int FMT, bool XBF16>
cudaError_t launch_fused_rb(int m, const Params& p, const FusedPlan& fp, cudaStream_t st) {
  if (m == 1) return launch_fused_t<FMT, XBF16, 1>(p, fp, st);
  if (m == 2) return launch_fused_t<FMT, XBF16, 2>(p, fp, st);
  return launch_fused_t<FMT, XBF16, 4>(p, fp, st);
}

// Formats with a persistent-kernel instantiation (one format for every projection).
bool fused_formats_ok(int fmt, bool xbf16) {
  return (fmt == MOE_FMT_F32 && !xbf16) ||
         (xbf16 && (fmt == MOE_FMT_BF16 || fmt == MOE_FMT_Q4_AFFINE_G64 ||
                    fmt == MOE_FMT_NVFP4 || fmt == MOE_FMT_MXFP4 || fmt == MOE_FMT_FP8_E4M3));
}

cudaError_t launch_fused(int fmt, bool xbf16, int m, const Params& p, const FusedPlan& fp,
                         cudaStream_t st) {
  switch (fmt) {
    case MOE_FMT_F32: return launch_fused_rb<MOE_FMT_F32, false>(m, p, fp, st);
    case MOE_FMT_BF16: return launch_fused_rb<MOE_FMT_BF16, true>(m, p, fp, st);
    case MOE_FMT_Q4_AFFINE_G64: return launch_fused_rb<MOE_FMT_Q4_AFFINE_G64, true>(m, p, fp, st);
    case MOE_FMT_NVFP4: return launch_fused_rb<MOE_FMT_NVFP4, true>(m, p, fp, st);
    case MOE_FMT_MXFP4: return launch_fused_rb<MOE_FMT_MXFP4, true>(m, p, fp, st);
    default: return launch_fused_rb<MOE_FMT_FP8_E4M3, true>(m, p, fp, st);
  }
}

// The tensor-core path takes a call when one format in {bf16, FP8, NVFP4, MXFP4, Q4} serves
// every projection, the activations are bf16, and (fp16 operand formats) hidden is a multiple of
// 16 (the activations are converted in 16-element blocks).
bool tc_eligible(const moe_cfg& c, const moe_expert_table* routed, const moe_expert_table* shared,
                 bool has_shared) {
  const int fmt = routed->gate.format;
  if (fmt == MOE_FMT_F32 || c.x_dtype != MOE_FMT_BF16) return false;
  if (routed->down.format != fmt) return false;
  if (has_shared && (shared->gate.format != fmt || shared->down.format != fmt)) return false;
  if (fmt != MOE_FMT_BF16 && c.hidden % 16) return false;
  // scale and bias slabs are read as aligned 4-byte words: their bases must be 4-byte aligned
  auto words_ok = [](const moe_matrix& M) {
    return (!M.scales || aligned(M.scales, 4)) && (!M.biases || aligned(M.biases, 4));
  };
  if (!words_ok(routed->gate) || !words_ok(routed->up) || !words_ok(routed->down)) return false;
  if (has_shared && (!words_ok(shared->gate) || !words_ok(shared->up) || !words_ok(shared->down)))
    return false;
  return true;
}

template <typename K>
cudaError_t launch_tc(K kernel, int grid, int block, cudaStream_t st, bool cooperative,
                      const Params& p, const tc::TcExtra& tx, const tc::TcPlan* pl,
                      const int* slot_beg, const int* slot_n) {
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lock(mu);
    const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               tc::kRingCtaBytes);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = tc::kRingCtaBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  if (cooperative) {
    attr[na].id = cudaLaunchAttributeCooperative;
    attr[na].val.cooperative = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  if constexpr (std::is_invocable_v<K, Params, tc::TcExtra, tc::TcPlan>) {
    return cudaLaunchKernelEx(&cfg, kernel, p, tx, *pl);
  } else {
    return cudaLaunchKernelEx(&cfg, kernel, p, tx, slot_beg, slot_n);
  }
}

template <int FMT, int NTG>
cudaError_t tc_run(bool chain, int sms, cudaStream_t st, const Params& p, const tc::TcExtra& tx,
                   const tc::TcPlan& pl, int* slot_beg, int* slot_n) {
  constexpr int kThr = 32 * tc::tc_warps<FMT, NTG>();
  if (!chain) {
    auto kernel = tc::tc_fused_kernel<FMT, NTG>;
    int per_sm = 0;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         tc::kRingCtaBytes);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThr, tc::kRingCtaBytes);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorCooperativeLaunchTooLarge;
    return launch_tc(kernel, sms, kThr, st, true, p, tx, &pl, nullptr, nullptr);
  }
  const int router_grid = p.E + (p.shared_kind == MOE_SHARED_SIGMOID_GATE ? 1 : 0);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(router_grid);
  cfg.blockDim = dim3(kRouterThreads);
  cfg.stream = st;
  cudaError_t e = cudaLaunchKernelEx(&cfg, tc::tc_router_kernel<FMT>, p, tx, slot_beg, slot_n);
  if (e != cudaSuccess) return e;
  e = launch_tc(tc::tc_gate_up_kernel<FMT, NTG>, sms, kThr, st, false, p, tx, nullptr,
                slot_beg, slot_n);
  if (e != cudaSuccess) return e;
  return launch_tc(tc::tc_down_kernel<FMT, NTG>, sms, kThr, st, false, p, tx, nullptr,
                   slot_beg, slot_n);
}

template <int FMT>
cudaError_t tc_run_ntg(int ntg, bool chain, int sms, cudaStream_t st, const Params& p,
                       const tc::TcExtra& tx, const tc::TcPlan& pl, int* sb, int* sn) {
  return ntg == 1 ? tc_run<FMT, 1>(chain, sms, st, p, tx, pl, sb, sn)
                  : tc_run<FMT, 2>(chain, sms, st, p, tx, pl, sb, sn);
}

cudaError_t tc_launch(int fmt, int ntg, bool chain, int sms, cudaStream_t st, const Params& p,
                      const tc::TcExtra& tx, const tc::TcPlan& pl, int* sb, int* sn) {
  switch (fmt) {
    case MOE_FMT_BF16: return tc_run_ntg<MOE_FMT_BF16>(ntg, chain, sms, st, p, tx, pl, sb, sn);
    case MOE_FMT_FP8_E4M3:
      return tc_run_ntg<MOE_FMT_FP8_E4M3>(ntg, chain, sms, st, p, tx, pl, sb, sn);
    case MOE_FMT_NVFP4: return tc_run_ntg<MOE_FMT_NVFP4>(ntg, chain, sms, st, p, tx, pl, sb, sn);
    case MOE_FMT_MXFP4: return tc_run_ntg<MOE_FMT_MXFP4>(ntg, chain, sms, st, p, tx, pl, sb, sn);
    default:
      return tc_run_ntg<MOE_FMT_Q4_AFFINE_G64>(ntg, chain, sms, st, p, tx, pl, sb, sn);
  }
}

}  // namespace

extern "C" int moe_workspace_bytes(const moe_cfg* cfg, int m, size_t* out_bytes) {
  if (!out_bytes) return MOE_ERR_NULL_POINTER;
  const int rc = check_cfg(cfg, m);
  if (rc) return rc;
  *out_bytes = layout_of(cfg, m).total;
  return MOE_OK;
}

extern "C" int moe_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
  if (!workspace) return MOE_ERR_NULL_POINTER;
  if (workspace_bytes < (size_t)kCtrlBytes) return MOE_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return MOE_ERR_MISALIGNED;
  const cudaError_t e = cudaMemsetAsync(workspace, 0, kCtrlBytes, (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

// Host dispatch: one persistent kernel for decode-sized calls when every projection shares a
// format and the call's activations fit in shared memory; the three-kernel chain otherwise.
bool use_fused(const moe_cfg& c, int m, const moe_expert_table* routed,
               const moe_expert_table* shared, bool has_shared, FusedPlan* fp) {
  const int fmt = routed->gate.format;
  const bool one_fmt = routed->down.format == fmt &&
                       (!has_shared || (shared->gate.format == fmt && shared->down.format == fmt));
  return forced_path() != 1 && one_fmt &&
         fused_formats_ok(fmt, c.x_dtype == MOE_FMT_BF16) &&
         plan_fused(c, m, has_shared, fmt, sm_count(), fp);
}

// Launches of the chain: router, gate/up (two when the shared expert has its own format), down
// (likewise).
int chain_launches(const moe_expert_table* routed, const moe_expert_table* shared, bool has_shared) {
  const bool split_gu = has_shared && shared->gate.format != routed->gate.format;
  const bool split_d = has_shared && shared->down.format != routed->down.format;
  return 1 + (split_gu ? 2 : 1) + (split_d ? 2 : 1);
}

extern "C" int moe_decode_forward(const moe_cfg* cfg, int m, const void* x, const void* router_w,
                                  const float* expert_bias, const moe_expert_table* routed,
                                  const moe_expert_table* shared, const void* shared_gate_w,
                                  void* out, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  NvtxRange nvtx("moe_decode_forward");
  int rc = check_cfg(cfg, m);
  if (rc) return rc;
  const moe_cfg& c = *cfg;
  if (!x || !router_w || !routed || !out || !workspace) return MOE_ERR_NULL_POINTER;
  if (!aligned(x, 16) || !aligned(router_w, 16) || !aligned(out, 16) || !aligned(workspace, 256))
    return MOE_ERR_MISALIGNED;
  if (c.has_expert_bias && !expert_bias) return MOE_ERR_NULL_POINTER;
  if (expert_bias && !aligned(expert_bias, 4)) return MOE_ERR_MISALIGNED;
  const bool has_shared = c.shared_kind != MOE_SHARED_NONE;
  if (has_shared && !shared) return MOE_ERR_NULL_POINTER;
  if (c.shared_kind == MOE_SHARED_SIGMOID_GATE) {
    if (!shared_gate_w) return MOE_ERR_NULL_POINTER;
    if (!aligned(shared_gate_w, 16)) return MOE_ERR_MISALIGNED;
  }
  Params p;
  std::memset(&p, 0, sizeof(p));
  if ((rc = check_table(routed, c.moe_inter, c.hidden, c.num_experts, &p.rg, &p.ru, &p.rd)))
    return rc;
  if (has_shared &&
      (rc = check_table(shared, c.shared_inter, c.hidden, 1, &p.sg, &p.su, &p.sd)))
    return rc;
  const WsLayout L = layout_of(&c, m);
  if (workspace_bytes < L.total) return MOE_ERR_WORKSPACE;
  if ((rc = check_device())) return rc;

  p.m = m;
  p.h = c.hidden;
  p.E = c.num_experts;
  p.k = c.top_k;
  p.I = c.moe_inter;
  p.S = has_shared ? c.shared_inter : 0;
  p.routing = c.routing;
  p.norm = c.norm_topk_prob;
  p.raw = c.select_on_raw_logits;
  p.has_bias = c.has_expert_bias;
  p.before_ffn = c.weight_before_ffn;
  p.shared_kind = c.shared_kind;
  p.out_bf16 = c.out_dtype == MOE_FMT_BF16;
  p.act_kind = c.activation;
  p.rsf = c.routed_scaling_factor;
  const int te = m * c.top_k;
  p.cap = te < c.num_experts ? te : c.num_experts;
  p.n_tiles_i = (c.moe_inter + kRowsPerCta - 1) / kRowsPerCta;
  p.n_tiles_s = has_shared ? (p.S + kRowsPerCta - 1) / kRowsPerCta : 0;
  p.n_tiles_c = n_tiles_c_of(c.hidden);
  p.has_shared = has_shared ? 1 : 0;
  p.x = x;
  p.router_w = router_w;
  p.expert_bias = expert_bias;
  p.shared_gate_w = shared_gate_w;
  p.out = out;
  uint8_t* ws = (uint8_t*)workspace;
  p.ctrl = (unsigned*)ws;
  p.logits = (float*)(ws + L.logits);
  p.idx = (int*)(ws + L.idx);
  p.wts = (float*)(ws + L.wts);
  p.gamma = (float*)(ws + L.gamma);
  p.sorted_pairs = (int*)(ws + L.sorted_pairs);
  p.offsets = (int*)(ws + L.offsets);
  p.token_to_perm = (int*)(ws + L.token_to_perm);
  p.active = (int*)(ws + L.active);
  p.active_count = (int*)(ws + L.active_count);
  p.act = (float*)(ws + L.act);
  p.act_sh = (float*)(ws + L.act_sh);
  p.ypart = (float*)(ws + L.ypart);
  p.ysh = (float*)(ws + L.ysh);
  p.tickets = (unsigned*)(ws + L.tickets);

  cudaStream_t st = (cudaStream_t)stream;
  const bool xbf16 = c.x_dtype == MOE_FMT_BF16;

  if (tc_eligible(c, routed, shared, has_shared)) {
    const TcShape ts = tc_shape(c, m, routed->gate.format);
    const TcLayout tl = tc_layout(c, m, base_layout_of(&c, m).total);
    const int sms = sm_count();
    if (sms <= 0) return MOE_ERR_UNSUPPORTED_DEVICE;
    tc::TcExtra tx;
    std::memset(&tx, 0, sizeof(tx));
    tx.W = sms * tc::kMaxWarps;
    const int split = g_forced_split.load(std::memory_order_relaxed);
    // whether a phase splits its jobs by chunk is decided in the kernel from the call's routing
    // (tc::split_jobs); here: whether it may (its chunk values fit the workspace and no test
    // forces whole jobs), and whether a test forces the split
    tx.gu_piece = ts.gu_slots && split != 1;
    tx.dn_piece = ts.dn_slots && split != 1;
    tx.force_split = split == 2;
    tx.tiles_i = ts.tiles_i;
    tx.tiles_s = ts.tiles_s;
    tx.tiles_h = ts.tiles_h;
    tx.nch_h = ts.nch_h;
    tx.nch_i = ts.nch_i;
    tx.nch_s = ts.nch_s;
    tx.xb = ws + tl.xb;
    tx.act = ws + tl.act;
    tx.sh_act = ws + tl.sh_act;
    tx.gu_slots = (float*)(ws + tl.gu_slots);
    tx.dn_slots = (float*)(ws + tl.dn_slots);
    tx.tk_gu = (unsigned*)(ws + tl.tk);
    tx.tk_dn = tx.tk_gu + (size_t)ts.j_gu_max * ts.ncg_max;
    tx.tk_col = tx.tk_dn + (size_t)ts.j_dn_max * ts.ncg_max;
    tx.ready = tx.tk_col + ts.tiles_h;
    tx.tk_words = tl.tk_words;
    tx.stamps = tl.stamps ? (unsigned long long*)(ws + tl.stamps) : nullptr;
    tc::TcPlan pl;
    pl.spin_limit = g_test_spin_limit.load() > 0 ? g_test_spin_limit.load() : kSpinLimit;
    pl.bar_extra = (unsigned)g_test_bar_extra.load();
    pl.l2_prefetch_cap = kDownPrefetchCap;
    const bool chain = forced_path() == 1;
    const int ntg = ts.ntg;
    const cudaError_t e = tc_launch(routed->gate.format, ntg, chain, sms, st, p, tx, pl,
                                    (int*)(ws + tl.slot_beg), (int*)(ws + tl.slot_n));
    if (e != cudaSuccess) return cuda_fail(e);
    log_dispatch_once(chain ? "chain (tensor-core router, gate/up, down)"
                            : "persistent tensor-core kernel",
                      routed->gate.format, m, chain ? 3 : 1);
    return MOE_OK;
  }

  {
    FusedPlan fp;
    if (use_fused(c, m, routed, shared, has_shared, &fp)) {
      const cudaError_t e = launch_fused(routed->gate.format, xbf16, m, p, fp, st);
      if (e != cudaSuccess) return cuda_fail(e);
      log_dispatch_once("persistent kernel", routed->gate.format, m, 1);
      return MOE_OK;
    }
  }

  const int router_grid = c.num_experts + (c.shared_kind == MOE_SHARED_SIGMOID_GATE ? 1 : 0);
  cudaError_t e = xbf16 ? launch(router_topk_group_kernel<true>, router_grid, kRouterThreads, 0,
                                 st, p, false)
                        : launch(router_topk_group_kernel<false>, router_grid, kRouterThreads, 0,
                                 st, p, false);
  if (e != cudaSuccess) return cuda_fail(e);

  // gate + up + SwiGLU: shared tiles first (they need no routing), then routed tiles; one
  // launch when routed and shared experts share a format, else one launch per format.
  const int fmt_gu = routed->gate.format;
  const bool split_gu = has_shared && shared->gate.format != fmt_gu;
  auto gate_up = [&](int fmt, const Params& q, int grid) {
    const int rb = rows_per_pass(c.hidden, fmt, m);
    const size_t smem = staging_bytes(c.hidden, fmt, rb);
    return xbf16 ? launch_gate_up<true>(fmt, rb, grid, smem, st, q)
                 : launch_gate_up<false>(fmt, rb, grid, smem, st, q);
  };
  if (split_gu) {
    Params ps = p;  // shared tiles only
    e = gate_up(shared->gate.format, ps, p.n_tiles_s);
    if (e != cudaSuccess) return cuda_fail(e);
    Params pr = p;  // routed tiles only
    pr.n_tiles_s = 0;
    e = gate_up(fmt_gu, pr, p.cap * p.n_tiles_i);
  } else {
    e = gate_up(fmt_gu, p, p.n_tiles_s + p.cap * p.n_tiles_i);
  }
  if (e != cudaSuccess) return cuda_fail(e);

  // down + blend. The column-tile tickets count routed and shared arrivals across launches, so
  // a shared expert in another format runs as a second launch (its CTAs arrive last).
  const int fmt_d = routed->down.format;
  const bool split_d = has_shared && shared->down.format != fmt_d;
  auto down = [&](int fmt, const Params& q, int grid, int K) {
    const int rb = rows_per_pass(K, fmt, m);
    return launch_down(fmt, rb, grid, staging_bytes(K, fmt, rb), st, q);
  };
  if (split_d) {
    e = down(fmt_d, p, p.n_tiles_c * p.cap, c.moe_inter);
    if (e != cudaSuccess) return cuda_fail(e);
    Params ps = p;
    ps.slot_base = p.cap;
    e = down(shared->down.format, ps, p.n_tiles_c, p.S);
  } else {
    const int kmax = (has_shared && p.S > c.moe_inter) ? p.S : c.moe_inter;
    e = down(fmt_d, p, p.n_tiles_c * (p.cap + p.has_shared), kmax);
  }
  if (e != cudaSuccess) return cuda_fail(e);
  log_dispatch_once("chain (router, gate/up, down)", routed->gate.format, m,
                    chain_launches(routed, shared, has_shared));
  return MOE_OK;
}

extern "C" int moe_decode_launches(const moe_cfg* cfg, int m, const moe_expert_table* routed,
                                   const moe_expert_table* shared, int* launches) {
  int rc = check_cfg(cfg, m);
  if (rc) return rc;
  if (!launches) return MOE_ERR_NULL_POINTER;
  const bool has_shared = cfg->shared_kind != MOE_SHARED_NONE;
  MatDev g, u, d;
  if ((rc = check_table(routed, cfg->moe_inter, cfg->hidden, cfg->num_experts, &g, &u, &d)))
    return rc;
  if (has_shared && (rc = check_table(shared, cfg->shared_inter, cfg->hidden, 1, &g, &u, &d)))
    return rc;
  if ((rc = check_device())) return rc;
  FusedPlan fp;
  if (tc_eligible(*cfg, routed, shared, has_shared)) {
    *launches = forced_path() == 1 ? 3 : 1;
  } else {
    *launches = use_fused(*cfg, m, routed, shared, has_shared, &fp)
                    ? 1 : chain_launches(routed, shared, has_shared);
  }
  return MOE_OK;
}

extern "C" int moe_debug_set_path(int path) {
  if (path != 0 && path != 1) return MOE_ERR_BAD_OPTION;
  g_forced_path.store(path);
  return MOE_OK;
}

extern "C" int moe_debug_set_split(int mode) {
  if (mode < 0 || mode > 2) return MOE_ERR_BAD_OPTION;
  g_forced_split.store(mode);
  return MOE_OK;
}

extern "C" int moe_debug_barrier_test(int extra_arrivals, long long spin_limit_cycles) {
  if (extra_arrivals < 0 || extra_arrivals > 1 || spin_limit_cycles < 0) return MOE_ERR_BAD_OPTION;
  g_test_spin_limit.store(spin_limit_cycles);
  g_test_bar_extra.store(extra_arrivals);
  return MOE_OK;
}

extern "C" int moe_decode_read_routing(const moe_cfg* cfg, int m, const void* workspace,
                                       size_t workspace_bytes, void* stream, int32_t* idx,
                                       float* weights, int32_t* sorted_pairs,
                                       int32_t* expert_offsets, int32_t* token_to_perm,
                                       int32_t* active, int32_t* active_count, float* gamma) {
  int rc = check_cfg(cfg, m);
  if (rc) return rc;
  if (!workspace) return MOE_ERR_NULL_POINTER;
  const WsLayout L = layout_of(cfg, m);
  if (workspace_bytes < L.total) return MOE_ERR_WORKSPACE;
  const uint8_t* ws = (const uint8_t*)workspace;
  cudaStream_t st = (cudaStream_t)stream;
  const size_t te = (size_t)m * cfg->top_k;
  const size_t cap = te < (size_t)cfg->num_experts ? te : (size_t)cfg->num_experts;
  struct Item { void* dst; size_t off, bytes; } items[] = {
      {idx, L.idx, te * 4},
      {weights, L.wts, te * 4},
      {sorted_pairs, L.sorted_pairs, te * 4},
      {expert_offsets, L.offsets, (size_t)(cfg->num_experts + 1) * 4},
      {token_to_perm, L.token_to_perm, te * 4},
      {active, L.active, cap * 4},
      {active_count, L.active_count, 4},
      {gamma, L.gamma, (size_t)m * 4},
  };
  for (const Item& it : items) {
    if (!it.dst) continue;
    const cudaError_t e = cudaMemcpyAsync(it.dst, ws + it.off, it.bytes, cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  const cudaError_t e = cudaStreamSynchronize(st);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

extern "C" int moe_get_device_status(const void* workspace, size_t workspace_bytes, void* stream,
                                     int32_t* status) {
  if (!workspace || !status) return MOE_ERR_NULL_POINTER;
  if (workspace_bytes < (size_t)kCtrlBytes) return MOE_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaMemcpyAsync(status, workspace, 4, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e);
}

extern "C" const char* moe_status_string(int status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_NULL_POINTER: return "a required pointer is NULL";
    case MOE_ERR_BAD_SHAPE: return "invalid shape (m, hidden, experts, top_k or intermediate)";
    case MOE_ERR_BAD_FORMAT: return "invalid or mismatched format";
    case MOE_ERR_BAD_OPTION: return "invalid routing or shared-expert option";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_MISALIGNED: return "pointer or stride misaligned";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case MOE_ERR_UNSUPPORTED_DEVICE: return "device is not compute capability 10.0 (B200)";
    case MOE_ERR_DEVICE_CHECK: return "device-side consistency check failed";
    default: return "unknown status";
  }
}

extern "C" int moe_last_cuda_error(void) { return g_last_cuda_error; }

extern "C" int moe_version(void) { return 200; }
