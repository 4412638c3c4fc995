// One persistent kernel for a whole decode MoE layer call (m <= 4 rows).
//
// All CTAs are co-resident (cooperative launch, one CTA per SM). Phases:
//   A  router logits. Before the programmatic-launch wait each CTA asks L2 for its router rows
//      (the weights do not depend on the previous kernel); after the wait it stages the m
//      activation rows in shared memory as fp32 and computes its rows' logits (and the shared-
//      expert gate logit). Then it arrives at grid barrier 1 without waiting.
//   B  shared expert gate+up (needs no routing): a contiguous slice of the S row pairs per CTA.
//   C  wait at barrier 1; every CTA routes every row and groups the pairs by expert in its own
//      shared memory (m*k <= 32 pairs, so doing it redundantly costs less than a barrier).
//   D  routed gate+up: the U*I row pairs of the U active experts are split into equal contiguous
//      slices, one per CTA. Before streaming them the CTA asks L2 for the down-projection rows it
//      will need in phase E, so those bytes arrive while gate/up streams. Arrive + wait barrier 2.
//   E  down + blend: each CTA owns a contiguous range of output columns for all rows. It stages
//      every act row in shared memory, computes y for each (column, active expert) and the shared
//      expert from the L2-resident down rows, and blends: routed slots in slot order times their
//      weight, then gamma times the shared expert. No atomics; a row's bits do not depend on m.
// Barrier waits are bounded (clock64 budget); on expiry the kernel records
// MOE_ERR_DEVICE_TIMEOUT in the workspace status word and carries on, so it always terminates.
#pragma once

#include "experts.cuh"
#include "router.cuh"

namespace moe {

constexpr int kFusedThreads = 512;
constexpr int kFusedWarps = kFusedThreads / 32;
constexpr int kFusedGroups = kFusedWarps * kRowsPerWarp;  // 64 eight-lane row groups per CTA
constexpr int kFusedMaxRows = 4;
constexpr int kFusedMaxPairs = kFusedMaxRows * MOE_MAX_TOP_K;  // 32

enum FusedCtrl { kBarCount = 2, kBarGen = 3, kDbgCount = 4, kDbgGen = 5, kDbgWant = 6 };

struct FusedPlan {
  int grid;            // CTAs (all co-resident)
  int cols_per_cta;    // output columns owned by one CTA in phase E
  int xs_off;          // dynamic smem byte offsets
  int xsum_off;        // Q4 gate/up: per-32 sums of x
  int act_off;         // staged act rows: [te + m][max(I, S)] fp32 (routed pairs, then shared)
  int actsum_off;      // Q4 down: per-32 sums of the staged act rows
  int y_off;           // y[(te + m) * cols_per_cta]
  int act_ld;          // row pitch (floats) of the staged act rows
  int smem_bytes;
  long long spin_limit;  // clock cycles a barrier wait may spin
};

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Ask L2 for [p, p + bytes) in pieces of at most 32 KB (p and bytes are multiples of 16: packed
// weight rows are 16-byte aligned).
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, size_t bytes) {
  const uint8_t* b = (const uint8_t*)p;
  for (size_t o = 0; o < bytes; o += 32768) {
    const unsigned n = (unsigned)(bytes - o < 32768 ? bytes - o : 32768);
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(b + o), "r"(n) : "memory");
  }
}

__device__ __forceinline__ void prefetch_l2_lines(const uint8_t* p, size_t bytes) {
  const uintptr_t a0 = (uintptr_t)p & ~(uintptr_t)127;
  for (uintptr_t a = a0; a < (uintptr_t)p + bytes; a += 128) {
    const uint8_t* q = (const uint8_t*)(a < (uintptr_t)p ? (uintptr_t)p : a);
    asm volatile("prefetch.global.L2 [%0];" ::"l"(q));
  }
}

// Split arrive/wait grid barrier over all CTAs of the launch. The counter returns to zero after
// every barrier; the generation word only grows, and each CTA reads it before its first arrival
// (no barrier can complete before every CTA has arrived), so waits compare against that value.
struct GridBarrier {
  unsigned* count;
  unsigned* gen;
  unsigned* status;
  unsigned gen0;
  long long limit;

  __device__ void arrive() const {
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      const unsigned old = atomicAdd(count, 1u);
      if (old == gridDim.x - 1) {
        atomicExch(count, 0u);
        __threadfence();
        atomicAdd(gen, 1u);
      }
    }
  }
  __device__ void wait(unsigned passed) const {
    if (threadIdx.x == 0) {
      const long long t0 = clock64();
      while ((int)(ld_acquire_u32(gen) - gen0) < (int)passed) {
        if (clock64() - t0 > limit) {
          // record where the wait gave up: arrivals seen, generation seen, generation expected
          atomicExch(status, (unsigned)MOE_ERR_DEVICE_TIMEOUT);
          atomicExch(status + kDbgCount, ld_acquire_u32(count));
          atomicExch(status + kDbgGen, ld_acquire_u32(gen));
          atomicExch(status + kDbgWant, gen0 + passed);
          break;
        }
        __nanosleep(32);
      }
      __threadfence();
    }
    __syncthreads();
  }
};

// Routing and grouping kept in shared memory by every CTA.
struct FusedRoute {
  int idx[kFusedMaxPairs];
  float w[kFusedMaxPairs];
  float gamma[kFusedMaxRows];
  int sorted[kFusedMaxPairs];     // pair ids by (expert, pair)
  int tp[kFusedMaxPairs];         // position of each pair in `sorted`
  int slot_e[kFusedMaxPairs];     // active experts, ascending
  int slot_beg[kFusedMaxPairs];   // first position of each active expert in `sorted`
  int slot_n[kFusedMaxPairs];     // its number of pairs
  int n_active;
};

// Route row r (one warp): same selection rule as the multi-kernel path.
__device__ void fused_route_row(const Params& p, int r, FusedRoute& R) {
  const int lane = threadIdx.x & 31;
  const int E = p.E, k = p.k;
  const float* lrow = p.logits + (size_t)r * (E + 1);
  float lg[8], key[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int e = lane + 32 * j;
    const bool valid = e < E;
    const float l = valid ? __ldcg(lrow + e) : -INFINITY;
    lg[j] = l;
    float kv = l;
    if (p.routing == MOE_ROUTE_SIGMOID && !p.raw) {
      kv = 1.0f / (1.0f + expf(-l));
      if (p.has_bias && valid) kv += __ldg(p.expert_bias + e);
    }
    key[j] = valid ? kv : -INFINITY;
  }
  float mx = -INFINITY, den = 0.f;
  if (p.routing == MOE_ROUTE_SOFTMAX) {
#pragma unroll
    for (int j = 0; j < 8; ++j) mx = fmaxf(mx, lg[j]);
    mx = warp_max(mx);
#pragma unroll
    for (int j = 0; j < 8; ++j) den += (lane + 32 * j < E) ? expf(lg[j] - mx) : 0.f;
    den = warp_sum(den);
  }
  unsigned taken = 0;
  int my_id = 0;
  float my_l = 0.f;
  bool bad = false;
  for (int s = 0; s < k; ++s) {
    float bk = -INFINITY;
    int bid = 0x7fffffff;
    float bl = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane + 32 * j;
      if (e < E && !((taken >> j) & 1u) && (key[j] > bk || (key[j] == bk && e < bid))) {
        bk = key[j];
        bid = e;
        bl = lg[j];
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ok = __shfl_xor_sync(0xffffffffu, bk, o);
      const int oid = __shfl_xor_sync(0xffffffffu, bid, o);
      const float ol = __shfl_xor_sync(0xffffffffu, bl, o);
      if (ok > bk || (ok == bk && oid < bid)) {
        bk = ok;
        bid = oid;
        bl = ol;
      }
    }
    if (bid >= E) {
      bad = true;
      bid = s;
    }
    if ((bid & 31) == lane) taken |= 1u << (bid >> 5);
    if (lane == s) {
      my_id = bid;
      my_l = bl;
    }
  }
  float wv = 0.f;
  if (lane < k)
    wv = (p.routing == MOE_ROUTE_SOFTMAX) ? expf(my_l - mx) / den : 1.0f / (1.0f + expf(-my_l));
  if (p.norm) {
    const float tot = warp_sum(lane < k ? wv : 0.f);
    wv = wv / tot;
  }
  wv *= p.rsf;
  if (lane < k) {
    R.idx[r * k + lane] = my_id;
    R.w[r * k + lane] = wv;
  }
  if (lane == 0) {
    float g = 1.f;
    if (p.shared_kind == MOE_SHARED_SIGMOID_GATE) g = 1.0f / (1.0f + expf(-__ldcg(lrow + E)));
    R.gamma[r] = g;
    if (bad) atomicExch(p.ctrl + kStatus, (unsigned)MOE_ERR_DEVICE_CHECK);
  }
}

// Stable grouping of te <= 32 pairs by expert, by warp 0: pair p (one lane) lands at
// #(pairs with a smaller expert id) + #(earlier pairs with the same id); the first pair of each
// expert opens its slot, slots ordered by expert id.
__device__ void fused_group(const Params& p, FusedRoute& R) {
  const int lane = threadIdx.x & 31;
  const int te = p.m * p.k;
  if (threadIdx.x >= 32) return;
  const bool live = lane < te;
  const int e = live ? R.idx[lane] : 0x7fffffff;
  int less = 0, eq_before = 0, eq_all = 0;
  for (int q = 0; q < te; ++q) {
    const int eq = __shfl_sync(0xffffffffu, e, q);
    less += eq < e;
    eq_before += (eq == e) && (q < lane);
    eq_all += eq == e;
  }
  const bool leader = live && eq_before == 0;
  const unsigned leaders = __ballot_sync(0xffffffffu, leader);
  int slot = 0;
  for (int q = 0; q < te; ++q) {
    const int eq = __shfl_sync(0xffffffffu, e, q);
    slot += ((leaders >> q) & 1u) && eq < e;
  }
  if (live) {
    const int pos = less + eq_before;
    R.sorted[pos] = lane;
    R.tp[lane] = pos;
    if (leader) {
      R.slot_e[slot] = e;
      R.slot_beg[slot] = less;
      R.slot_n[slot] = eq_all;
    }
  }
  if (lane == 0) R.n_active = __popc(leaders);
}

// CTA 0 publishes the routing and grouping for read-back (moe_decode_read_routing).
__device__ void fused_publish(const Params& p, const FusedRoute& R) {
  const int te = p.m * p.k;
  for (int t = threadIdx.x; t < te; t += blockDim.x) {
    p.idx[t] = R.idx[t];
    p.wts[t] = R.w[t];
    p.sorted_pairs[t] = R.sorted[t];
    p.token_to_perm[t] = R.tp[t];
  }
  for (int e = threadIdx.x; e <= p.E; e += blockDim.x) {
    int less = 0;
    for (int q = 0; q < te; ++q) less += R.idx[q] < e;
    p.offsets[e] = less;
  }
  for (int a = threadIdx.x; a < R.n_active; a += blockDim.x) p.active[a] = R.slot_e[a];
  if (threadIdx.x == 0) *p.active_count = R.n_active;
  if (p.shared_kind == MOE_SHARED_SIGMOID_GATE)
    for (int r = threadIdx.x; r < p.m; r += blockDim.x) p.gamma[r] = R.gamma[r];
}

// Dot products of two weight rows A, B with nb activation rows (pointers xr[j] into shared
// memory, xsr[j] their per-32 sums for Q4), chunk range lg, lg + 8, ... < nch.
template <int FMT, int RB, int U>
__device__ __forceinline__ void fused_two_rows(const RowRef& A, const RowRef& B, int nch, int lg,
                                               const float* const (&xr)[RB],
                                               const float* const (&xsr)[RB], int nb,
                                               float (&acc_a)[RB], float (&acc_b)[RB]) {
  constexpr int kE = Fmt<FMT>::kElems;
  for (int c0 = lg; c0 < nch; c0 += kLanesPerRow * U) {
    uint4 ra[U], rb[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + u * kLanesPerRow;
      if (c < nch) {
        ra[u] = ldg_stream(A.w + (size_t)c * 16);
        rb[u] = ldg_stream(B.w + (size_t)c * 16);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + u * kLanesPerRow;
      if (c < nch) {
        Dec<FMT> da, db;
        decode<FMT>(ra[u], A, c, da);
        decode<FMT>(rb[u], B, c, db);
#pragma unroll
        for (int j = 0; j < RB; ++j) {
          if (j < nb) {
            float s = 0.f;
            if constexpr (FMT == MOE_FMT_Q4_AFFINE_G64) s = xsr[j][c];
            acc_a[j] += dot<FMT>(da, xr[j] + c * kE, s);
            acc_b[j] += dot<FMT>(db, xr[j] + c * kE, s);
          }
        }
      }
    }
  }
}

// One weight row A against nb activation rows.
template <int FMT, int RB, int U>
__device__ __forceinline__ void fused_one_row(const RowRef& A, int nch, int lg,
                                              const float* const (&xr)[RB],
                                              const float* const (&xsr)[RB], int nb,
                                              float (&acc)[RB]) {
  constexpr int kE = Fmt<FMT>::kElems;
  for (int c0 = lg; c0 < nch; c0 += kLanesPerRow * U) {
    uint4 ra[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + u * kLanesPerRow;
      if (c < nch) ra[u] = ldg_stream(A.w + (size_t)c * 16);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + u * kLanesPerRow;
      if (c < nch) {
        Dec<FMT> da;
        decode<FMT>(ra[u], A, c, da);
#pragma unroll
        for (int j = 0; j < RB; ++j) {
          if (j < nb) {
            float s = 0.f;
            if constexpr (FMT == MOE_FMT_Q4_AFFINE_G64) s = xsr[j][c];
            acc[j] += dot<FMT>(da, xr[j] + c * kE, s);
          }
        }
      }
    }
  }
}

template <int FMT>
constexpr int fused_unroll() { return FMT == MOE_FMT_BF16 || FMT == MOE_FMT_F32 ? 8 : 4; }

template <int FMT_GU, int FMT_D, bool XBF16, int RB>
__global__ void __launch_bounds__(kFusedThreads, 1) moe_fused_kernel(
    const __grid_constant__ Params p, const __grid_constant__ FusedPlan fp) {
  extern __shared__ __align__(16) uint8_t fsmem[];
  __shared__ FusedRoute R;
  __shared__ unsigned s_gen0;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int lg = lane & (kLanesPerRow - 1);
  const int G = gridDim.x, cta = blockIdx.x;
  const int m = p.m, h = p.h, k = p.k, te = m * k;
  float* xs = reinterpret_cast<float*>(fsmem + fp.xs_off);
  float* xsum = reinterpret_cast<float*>(fsmem + fp.xsum_off);

  // ---- prologue (may overlap the previous kernel): this CTA's router rows into L2 -----------
  const int esz = XBF16 ? 2 : 4;
  const size_t xrow_bytes = (size_t)h * esz;
  const int e_tot = p.E + (p.shared_kind == MOE_SHARED_SIGMOID_GATE ? 1 : 0);
  auto router_row = [&](int e) {
    return e < p.E ? (const uint8_t*)p.router_w + (size_t)e * xrow_bytes
                   : (const uint8_t*)p.shared_gate_w;
  };
  if (tid == 0)
    for (int e = cta; e < e_tot; e += G) prefetch_l2_bulk(router_row(e), xrow_bytes);
  pdl_wait();
  // the previous grid has completed: its barrier updates are all visible
  if (tid == 0) s_gen0 = ld_acquire_u32(p.ctrl + kBarGen);
  __syncthreads();
  const GridBarrier bar{p.ctrl + kBarCount, p.ctrl + kBarGen, p.ctrl + kStatus, s_gen0,
                        fp.spin_limit};

  // ---- stage x (m rows, fp32, plus per-32 sums for Q4) ---------------------------------------
  stage_rows<FMT_GU, XBF16, kFusedMaxRows>(xs, xsum, h, m, [&](int j) {
    return (const uint8_t*)p.x + (size_t)j * xrow_bytes;
  });
  __syncthreads();

  // ---- A: router logits (one warp per (router row, activation row)) -------------------------
  {
    const int my_rows = cta < e_tot ? (e_tot - cta + G - 1) / G : 0;
    const int nch = (int)(xrow_bytes / 16);
    constexpr int kXE = XBF16 ? 8 : 4;
    for (int d = warp; d < my_rows * m; d += kFusedWarps) {
      const int e = cta + (d / m) * G, r = d % m;
      const float* xr = xs + (size_t)r * h;
      const float acc = router_dot_warp<XBF16>(router_row(e), nch, [&](int c, float* xv) {
        const float4 a = *reinterpret_cast<const float4*>(xr + c * kXE);
        xv[0] = a.x; xv[1] = a.y; xv[2] = a.z; xv[3] = a.w;
        if constexpr (XBF16) {
          const float4 b = *reinterpret_cast<const float4*>(xr + c * kXE + 4);
          xv[4] = b.x; xv[5] = b.y; xv[6] = b.z; xv[7] = b.w;
        }
      });
      if (lane == 0) p.logits[(size_t)r * (p.E + 1) + e] = acc;
    }
  }
  bar.arrive();

  // ---- B: shared expert gate + up (no routing needed) ----------------------------------------
  if (p.has_shared) {
    const int s0 = (int)((long long)cta * p.S / G), s1 = (int)((long long)(cta + 1) * p.S / G);
    const int nch = (int)(packed_row_bytes(FMT_GU, h) / 16);
    const float* xr[RB];
    const float* xsr[RB];
#pragma unroll
    for (int j = 0; j < RB; ++j) {
      xr[j] = xs + (size_t)min(j, m - 1) * h;
      xsr[j] = xsum + (size_t)min(j, m - 1) * (h / 32);
    }
    // warp-uniform trip count: the 4 row groups of a warp always reach the lane shuffles
    // together; a group past the end recomputes the last row and discards it
    for (int base = s0 + warp * kRowsPerWarp; base < s1; base += kFusedGroups) {
      const int i_raw = base + (lane >> 3);
      const bool valid = i_raw < s1;
      const int i = valid ? i_raw : s1 - 1;
      const RowRef A = row_ref<FMT_GU>(p.sg, 0, i), B = row_ref<FMT_GU>(p.su, 0, i);
      float ag[RB], au[RB];
#pragma unroll
      for (int j = 0; j < RB; ++j) ag[j] = au[j] = 0.f;
      fused_two_rows<FMT_GU, RB, fused_unroll<FMT_GU>()>(A, B, nch, lg, xr, xsr, m, ag, au);
#pragma unroll
      for (int j = 0; j < RB; ++j) {
        ag[j] = sum8lanes(ag[j]);
        au[j] = sum8lanes(au[j]);
      }
      if (valid && lg == 0) {
#pragma unroll
        for (int j = 0; j < RB; ++j)
          if (j < m) p.act_sh[(size_t)j * p.S + i] = silu_mul(ag[j] * A.ts, au[j] * B.ts);
      }
    }
  }

  // ---- C: routing + grouping (every CTA, in its own shared memory) ---------------------------
  bar.wait(1);
  if (warp < m) fused_route_row(p, warp, R);
  __syncthreads();
  fused_group(p, R);
  __syncthreads();
  const int U = R.n_active;

  // ---- D: routed gate + up; this CTA's phase-E down rows into L2 ------------------------------
  const int c0 = cta * fp.cols_per_cta;
  const int c1 = min(h, c0 + fp.cols_per_cta);
  const int ncols = c1 > c0 ? c1 - c0 : 0;
  if (ncols > 0 && tid < U + p.has_shared) {
    const bool sh = tid == U;
    const MatDev& D = sh ? p.sd : p.rd;
    const int e = sh ? 0 : R.slot_e[tid];
    const size_t rbytes = packed_row_bytes(FMT_D, D.k);
    prefetch_l2_bulk(D.packed + (size_t)e * D.estride + (size_t)c0 * rbytes, ncols * rbytes);
    if constexpr (FMT_D == MOE_FMT_Q4_AFFINE_G64) {
      const size_t sb = (size_t)(D.k / 64) * 2;
      prefetch_l2_lines(D.scales + (size_t)e * D.sstride + (size_t)c0 * sb, ncols * sb);
      prefetch_l2_lines(D.biases + (size_t)e * D.sstride + (size_t)c0 * sb, ncols * sb);
    } else if constexpr (FMT_D == MOE_FMT_NVFP4) {
      const size_t sb = (size_t)(D.k / 16);
      prefetch_l2_lines(D.scales + (size_t)e * D.sstride + (size_t)c0 * sb, ncols * sb);
    }
  }
  {
    const long long UI = (long long)U * p.I;
    const long long q0 = (long long)cta * UI / G, q1 = (long long)(cta + 1) * UI / G;
    const int nch = (int)(packed_row_bytes(FMT_GU, h) / 16);
    for (long long base = q0 + warp * kRowsPerWarp; base < q1; base += kFusedGroups) {
      const long long q_raw = base + (lane >> 3);
      const bool valid = q_raw < q1;
      const long long q = valid ? q_raw : q1 - 1;
      const int a = (int)(q / p.I), i = (int)(q - (long long)a * p.I);
      const int e = R.slot_e[a], beg = R.slot_beg[a], n = R.slot_n[a];
      const float* xr[RB];
      const float* xsr[RB];
#pragma unroll
      for (int j = 0; j < RB; ++j) {
        const int row = R.sorted[beg + min(j, n - 1)] / k;
        xr[j] = xs + (size_t)row * h;
        xsr[j] = xsum + (size_t)row * (h / 32);
      }
      const RowRef A = row_ref<FMT_GU>(p.rg, e, i), B = row_ref<FMT_GU>(p.ru, e, i);
      float ag[RB], au[RB];
#pragma unroll
      for (int j = 0; j < RB; ++j) ag[j] = au[j] = 0.f;
      fused_two_rows<FMT_GU, RB, fused_unroll<FMT_GU>()>(A, B, nch, lg, xr, xsr, n, ag, au);
#pragma unroll
      for (int j = 0; j < RB; ++j) {
        ag[j] = sum8lanes(ag[j]);
        au[j] = sum8lanes(au[j]);
      }
      if (valid && lg == 0) {
#pragma unroll
        for (int j = 0; j < RB; ++j) {
          if (j < n) {
            float g = ag[j] * A.ts, u = au[j] * B.ts;
            if (p.before_ffn) {
              const float w = R.w[R.sorted[beg + j]];
              g *= w;
              u *= w;
            }
            p.act[(size_t)(beg + j) * p.I + i] = silu_mul(g, u);
          }
        }
      }
    }
  }
  bar.arrive();
  if (cta == 0) fused_publish(p, R);
  bar.wait(2);
  pdl_launch_dependents();

  // ---- E: down + blend for this CTA's output columns ------------------------------------------
  if (ncols == 0) return;
  float* act_s = reinterpret_cast<float*>(fsmem + fp.act_off);
  float* actsum = reinterpret_cast<float*>(fsmem + fp.actsum_off);
  float* ys = reinterpret_cast<float*>(fsmem + fp.y_off);
  const int ld = fp.act_ld;
  const int n_rows = te + (p.has_shared ? m : 0);  // routed pairs (sorted order), then shared rows
  for (int t = tid; t < n_rows * (ld / 4); t += kFusedThreads) {
    const int r = t / (ld / 4), c4 = t - r * (ld / 4);
    const bool sh = r >= te;
    const int K = sh ? p.S : p.I;
    if (c4 * 4 < K) {
      const float* src = sh ? p.act_sh + (size_t)(r - te) * p.S : p.act + (size_t)r * p.I;
      reinterpret_cast<float4*>(act_s + (size_t)r * ld)[c4] =
          __ldcg(reinterpret_cast<const float4*>(src) + c4);
    }
  }
  __syncthreads();
  if constexpr (FMT_D == MOE_FMT_Q4_AFFINE_G64) {
    for (int t = tid; t < n_rows * (ld / 32); t += kFusedThreads) {
      const int r = t / (ld / 32), c = t - r * (ld / 32);
      const float* s = act_s + (size_t)r * ld + c * 32;
      float a = 0.f;
#pragma unroll
      for (int u = 0; u < 32; ++u) a += s[u];
      actsum[(size_t)r * (ld / 32) + c] = a;
    }
    __syncthreads();
  }
  {
    const int n_units = ncols * (U + p.has_shared);
    for (int base = warp * kRowsPerWarp; base < n_units; base += kFusedGroups) {
      const int u_raw = base + (lane >> 3);
      const bool valid = u_raw < n_units;
      const int u = valid ? u_raw : n_units - 1;
      const int slot = u / ncols, col = c0 + (u - slot * ncols);
      const bool sh = slot == U;
      const MatDev& D = sh ? p.sd : p.rd;
      const int e = sh ? 0 : R.slot_e[slot];
      const int beg = sh ? te : R.slot_beg[slot];
      const int n = sh ? m : R.slot_n[slot];
      const int K = sh ? p.S : p.I;
      const float* xr[RB];
      const float* xsr[RB];
#pragma unroll
      for (int j = 0; j < RB; ++j) {
        const int r = beg + min(j, n - 1);
        xr[j] = act_s + (size_t)r * ld;
        xsr[j] = actsum + (size_t)r * (ld / 32);
      }
      const RowRef A = row_ref<FMT_D>(D, e, col);
      const int nch = (int)(packed_row_bytes(FMT_D, K) / 16);
      float acc[RB];
#pragma unroll
      for (int j = 0; j < RB; ++j) acc[j] = 0.f;
      fused_one_row<FMT_D, RB, fused_unroll<FMT_D>()>(A, nch, lg, xr, xsr, n, acc);
#pragma unroll
      for (int j = 0; j < RB; ++j) acc[j] = sum8lanes(acc[j]);
      if (valid && lg == 0) {
#pragma unroll
        for (int j = 0; j < RB; ++j)
          if (j < n) ys[(size_t)(beg + j) * ncols + (col - c0)] = acc[j] * A.ts;
      }
    }
  }
  __syncthreads();
  for (int t = tid; t < m * ncols; t += kFusedThreads) {
    const int r = t / ncols, cl = t - r * ncols;
    float acc = 0.f;
    for (int s = 0; s < k; ++s) {
      const int pair = r * k + s;
      const float om = p.before_ffn ? 1.f : R.w[pair];
      acc = fmaf(om, ys[(size_t)R.tp[pair] * ncols + cl], acc);
    }
    if (p.has_shared) acc = fmaf(R.gamma[r], ys[(size_t)(te + r) * ncols + cl], acc);
    const size_t o = (size_t)r * h + c0 + cl;
    if (p.out_bf16) {
      reinterpret_cast<__nv_bfloat16*>(p.out)[o] = __float2bfloat16_rn(acc);
    } else {
      reinterpret_cast<float*>(p.out)[o] = acc;
    }
  }
}

}  // namespace moe
