// One persistent kernel for a whole decode MoE layer call (m <= 4 rows).
//
// All CTAs are co-resident (cooperative launch, one CTA per SM, 16 warps). Phases:
//   A  router logits: stage the m activation rows in shared memory as fp32, one warp per
//      (router row, activation row) dot product (router rows were asked into L2 before the
//      programmatic-launch wait); arrive at grid barrier 1 without waiting.
//   B  shared expert gate+up (needs no routing): this CTA's slice of the S row pairs.
//   C  wait at barrier 1; every CTA routes every row and groups the pairs by expert in its own
//      shared memory (m*k <= 32 pairs).
//   D  routed gate+up: the U*I row pairs of the U active experts in equal contiguous slices, one
//      per CTA; first the CTA asks L2 for the down rows it will need in phase E (when the whole
//      call's down rows fit comfortably in L2), so they arrive while gate/up streams. Arrive and
//      wait at grid barrier 2.
//   E  down + blend: each CTA owns a contiguous range of output columns for all rows; y for each
//      (column, active expert) and for the shared expert, then the blend: routed slots in slot
//      order times their weight, then gamma times the shared expert. No atomics.
// Every weight row is reduced by one warp with the multi-kernel path's arithmetic (lane l takes
// chunks l, l+32, ..., then a butterfly sum), so both paths give the same bits and a row's bits
// do not depend on m. Each grid-barrier wait is bounded (clock64 budget): on expiry it records
// MOE_ERR_DEVICE_TIMEOUT in the workspace status word and carries on, so the kernel terminates.
#pragma once

#include "experts.cuh"
#include "router.cuh"

namespace moe {

constexpr int kFusedThreads = 512;
constexpr int kFusedWarps = kFusedThreads / 32;
constexpr int kFusedMaxRows = 4;
constexpr int kFusedMaxPairs = kFusedMaxRows * MOE_MAX_TOP_K;  // 32

// control words: [2..3] the 64-bit barrier counter, [4..5] where a timed-out wait gave up
enum FusedCtrl { kBarCounter = 2, kDbgSeen = 4, kDbgWant = 5 };

struct FusedPlan {
  int grid;           // CTAs (all co-resident)
  int cols_per_cta;   // output columns owned by one CTA in phase E
  int xs_off;         // dynamic smem byte offsets
  int xsum_off;       // Q4 gate/up: per-32 sums of x
  int act_off;        // staged act rows: [te + m][act_ld] fp32 (routed pairs, then shared)
  int actsum_off;     // Q4 down: per-32 sums of the staged act rows
  int y_off;          // y[(te + m) * cols_per_cta]
  int act_ld;         // row pitch (floats) of the staged act rows
  int smem_bytes;
  long long spin_limit;       // clock cycles a barrier wait may spin before it gives up
  long long l2_prefetch_cap;  // largest per-call down-projection byte count asked into L2
};


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

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}


// Split arrive/wait grid barrier over all CTAs of the launch, on a 64-bit arrival counter that
// only grows by exactly 2 * grid per launch (grid = number of SMs for every launch on a
// workspace), so it is a multiple of the grid between launches. A CTA may be scheduled after
// other CTAs of its launch already arrived at barrier 1, but fewer than grid arrivals can precede
// its own, so flooring the value it reads to a multiple of the grid gives every CTA the same
// base; barrier b is passed once the counter reaches base + b * grid. Arrival is one
// release-ordered add after a CTA-wide barrier (the CTA's writes happen before it),
// waiting is an acquire poll: no fences, no reset.
struct GridBarrier {
  unsigned long long* ctr;
  unsigned* status;
  unsigned long long base;
  long long limit;

  __device__ void arrive() const {
    __syncthreads();
    if (threadIdx.x == 0)
      asm volatile("red.release.gpu.global.add.u64 [%0], 1;" ::"l"(ctr) : "memory");
  }
  __device__ void wait(unsigned passed) const {
    if (threadIdx.x == 0) {
      const unsigned long long target = base + (unsigned long long)passed * gridDim.x;
      const long long t0 = clock64();
      unsigned long long seen;
      while ((seen = ld_acquire_u64(ctr)) < target) {
        if (clock64() - t0 > limit) {
          // record where the wait gave up: arrivals seen, arrivals expected (since the base)
          atomicExch(status, (unsigned)MOE_ERR_DEVICE_TIMEOUT);
          atomicExch(status + kDbgSeen, (unsigned)(seen - base));
          atomicExch(status + kDbgWant, (unsigned)(target - base));
          break;
        }
      }
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

// Route row r (one warp) into the CTA's shared routing tables (same rule and arithmetic as the
// multi-kernel path).
__device__ void fused_route_row(const Params& p, int r, FusedRoute& R) {
  const int lane = threadIdx.x & 31;
  int id;
  float w, g;
  const bool ok = route_row(p, r, id, w, g);
  if (lane < p.k) {
    R.idx[r * p.k + lane] = id;
    R.w[r * p.k + lane] = w;
  }
  if (lane == 0) {
    R.gamma[r] = g;
    if (!ok) atomicExch(p.ctrl + kStatus, (unsigned)MOE_ERR_DEVICE_CHECK);
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
__device__ void fused_publish(const Params& p, const FusedRoute& R, int nt) {
  const int te = p.m * p.k;
  for (int t = threadIdx.x; t < te; t += nt) {
    p.idx[t] = R.idx[t];
    p.wts[t] = R.w[t];
    p.sorted_pairs[t] = R.sorted[t];
    p.token_to_perm[t] = R.tp[t];
  }
  for (int e = threadIdx.x; e <= p.E; e += nt) {
    int less = 0;
    for (int q = 0; q < te; ++q) less += R.idx[q] < e;
    p.offsets[e] = less;
  }
  for (int a = threadIdx.x; a < R.n_active; a += nt) p.active[a] = R.slot_e[a];
  if (threadIdx.x == 0) *p.active_count = R.n_active;
  if (p.shared_kind == MOE_SHARED_SIGMOID_GATE)
    for (int r = threadIdx.x; r < p.m; r += nt) p.gamma[r] = R.gamma[r];
}


// Optional phase timestamps (build with -DMOE_PHASE_TIMERS): thread 0 of every CTA records
// %globaltimer at each phase boundary into the (otherwise unused) down-partials region of the
// workspace, as uint64 [cta][kPhaseSlots].
constexpr int kPhaseSlots = 12;
#ifdef MOE_PHASE_TIMERS
#define MOE_STAMP(slot)                                                                     \
  do {                                                                                      \
    if (threadIdx.x == 0) {                                                                 \
      unsigned long long t_;                                                                \
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                                \
      reinterpret_cast<unsigned long long*>(p.ypart)[blockIdx.x * kPhaseSlots + (slot)] = t_; \
    }                                                                                       \
  } while (0)
#else
#define MOE_STAMP(slot) \
  do {                  \
  } while (0)
#endif

template <int FMT, bool XBF16, int RB>
__global__ void __launch_bounds__(kFusedThreads, 1) moe_fused_kernel(
    const __grid_constant__ Params p, const __grid_constant__ FusedPlan fp) {
  extern __shared__ __align__(16) uint8_t fsmem[];
  __shared__ FusedRoute R;
  __shared__ unsigned long long s_base;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  const int m = p.m, h = p.h, k = p.k, te = m * k;
  float* xs = reinterpret_cast<float*>(fsmem + fp.xs_off);
  float* xsum = reinterpret_cast<float*>(fsmem + fp.xsum_off);
  float* act_s = reinterpret_cast<float*>(fsmem + fp.act_off);
  float* actsum = reinterpret_cast<float*>(fsmem + fp.actsum_off);
  float* ys = reinterpret_cast<float*>(fsmem + fp.y_off);
  const int esz = XBF16 ? 2 : 4;
  const size_t xrow_bytes = (size_t)h * esz;
  const int e_tot = p.E + (p.shared_kind == MOE_SHARED_SIGMOID_GATE ? 1 : 0);
  auto router_row = [&](int e) {
    return e < p.E ? (const uint8_t*)p.router_w + (size_t)e * xrow_bytes
                   : (const uint8_t*)p.shared_gate_w;
  };
  const int c0 = cta * fp.cols_per_cta;
  const int ncols = min(h, c0 + fp.cols_per_cta) > c0 ? min(h, c0 + fp.cols_per_cta) - c0 : 0;
  const int nch_h = (int)(packed_row_bytes(FMT, h) / 16);
  MOE_STAMP(0);

  // ---- prologue (may overlap the previous kernel): this CTA's router rows into L2 -----------
  if (tid == 0)
    for (int e = cta; e < e_tot; e += G) prefetch_l2_bulk(router_row(e), xrow_bytes);
  pdl_wait();
  MOE_STAMP(1);
  unsigned long long* bar_ctr = reinterpret_cast<unsigned long long*>(p.ctrl + kBarCounter);
  if (tid == 0) s_base = ld_acquire_u64(bar_ctr) / (unsigned long long)G * (unsigned long long)G;
  stage_rows<FMT, XBF16>(xs, xsum, h, h, m, [&](int j) {
    return (const uint8_t*)p.x + (size_t)j * xrow_bytes;
  }, 0, kFusedThreads);
  __syncthreads();
  const GridBarrier bar{bar_ctr, p.ctrl + kStatus, s_base, fp.spin_limit};
  MOE_STAMP(2);

  // ---- A: router logits, one warp per (router row, activation row) ----------------------------
  {
    const int my_rows = cta < e_tot ? (e_tot - cta + G - 1) / G : 0;
    const int nch = (int)(xrow_bytes / 16);
    constexpr int kXE = XBF16 ? 8 : 4;
    for (int d = warp; d < my_rows * m; d += kFusedWarps) {
      const int e = cta + (d / m) * G, r = d % m;
      const float* xr = xs + (size_t)r * h;
      const float acc = router_dot_warp<XBF16>(router_row(e), nch, [&](int c, float* xv) {
        const float4 a = x_load<FMT>(xr, c * kXE / 4);
        xv[0] = a.x; xv[1] = a.y; xv[2] = a.z; xv[3] = a.w;
        if constexpr (XBF16) {
          const float4 b = x_load<FMT>(xr, c * kXE / 4 + 1);
          xv[4] = b.x; xv[5] = b.y; xv[6] = b.z; xv[7] = b.w;
        }
      });
      if (lane == 0) p.logits[(size_t)r * (p.E + 1) + e] = acc;
    }
  }
  MOE_STAMP(3);
  bar.arrive();

  // ---- B: shared expert gate + up (no routing needed) ----------------------------------------
  if (p.has_shared) {
    const int s0 = (int)((long long)cta * p.S / G), s1 = (int)((long long)(cta + 1) * p.S / G);
    const float* xr[RB];
    const float* xsr[RB];
#pragma unroll
    for (int j = 0; j < RB; ++j) {
      xr[j] = xs + (size_t)min(j, m - 1) * h;
      xsr[j] = xsum + (size_t)min(j, m - 1) * (h / 32);
    }
    for (int i = s0 + warp; i < s1; i += kFusedWarps) {
      const RowRef A = row_ref<FMT>(p.sg, 0, i), B = row_ref<FMT>(p.su, 0, i);
      float ag[RB], au[RB];
      rows2_dot<FMT, RB, false>(A, B, nch_h, xr, xsr, m, ag, au);
      if (lane < m) {
        float g = 0.f, u = 0.f;
#pragma unroll
        for (int j = 0; j < RB; ++j)
          if (j == lane) {
            g = ag[j];
            u = au[j];
          }
        p.act_sh[(size_t)lane * p.S + i] = silu_mul(g * A.ts, u * B.ts);
      }
    }
  }
  MOE_STAMP(4);

  // ---- C: routing + grouping (every CTA, in its own shared memory) ---------------------------
  bar.wait(1);
  MOE_STAMP(5);
  if (warp < m) fused_route_row(p, warp, R);
  __syncthreads();
  fused_group(p, R);
  __syncthreads();
  const int U = R.n_active;
  MOE_STAMP(6);

  // ---- D: routed gate + up; this CTA's phase-E down rows into L2 ------------------------------
  {
    const size_t down_bytes =
        ((size_t)U * packed_row_bytes(FMT, p.I) + (p.has_shared ? packed_row_bytes(FMT, p.S) : 0)) *
        (size_t)h;
    if (down_bytes <= (size_t)fp.l2_prefetch_cap && ncols > 0 && tid < U + p.has_shared) {
      const bool sh = tid == U;
      const MatDev& D = sh ? p.sd : p.rd;
      const int e = sh ? 0 : R.slot_e[tid];
      const size_t rbytes = packed_row_bytes(FMT, D.k);
      prefetch_l2_bulk(D.packed + (size_t)e * D.estride + (size_t)c0 * rbytes, ncols * rbytes);
      if constexpr (FMT == MOE_FMT_Q4_AFFINE_G64) {
        const size_t sb = (size_t)(D.k / 64) * 2;
        prefetch_l2_lines(D.scales + (size_t)e * D.sstride + (size_t)c0 * sb, ncols * sb);
        prefetch_l2_lines(D.biases + (size_t)e * D.sstride + (size_t)c0 * sb, ncols * sb);
      } else if constexpr (FMT == MOE_FMT_NVFP4) {
        const size_t sb = (size_t)(D.k / 16);
        prefetch_l2_lines(D.scales + (size_t)e * D.sstride + (size_t)c0 * sb, ncols * sb);
      }
    }
  }
  {
    const long long UI = (long long)U * p.I;
    const long long q0 = (long long)cta * UI / G, q1 = (long long)(cta + 1) * UI / G;
    for (long long q = q0 + warp; q < q1; q += kFusedWarps) {
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
      const RowRef A = row_ref<FMT>(p.rg, e, i), B = row_ref<FMT>(p.ru, e, i);
      float ag[RB], au[RB];
      rows2_dot<FMT, RB, false>(A, B, nch_h, xr, xsr, n, ag, au);
      if (lane < n) {
        float g = 0.f, u = 0.f;
#pragma unroll
        for (int j = 0; j < RB; ++j)
          if (j == lane) {
            g = ag[j];
            u = au[j];
          }
        g *= A.ts;
        u *= B.ts;
        if (p.before_ffn) {
          const float w = R.w[R.sorted[beg + lane]];
          g *= w;
          u *= w;
        }
        p.act[(size_t)(beg + lane) * p.I + i] = silu_mul(g, u);
      }
    }
  }
  MOE_STAMP(7);
  bar.arrive();
  if (cta == 0) fused_publish(p, R, kFusedThreads);
  bar.wait(2);
  MOE_STAMP(8);
  pdl_launch_dependents();

  // ---- E: down + blend for this CTA's output columns ------------------------------------------
  if (ncols == 0) {
    MOE_STAMP(11);
    return;
  }
  const int ld = fp.act_ld;
  stage_rows<FMT, false>(act_s, actsum, p.I, ld, te, [&](int j) {
    return (const uint8_t*)(p.act + (size_t)j * p.I);
  }, 0, kFusedThreads);
  if (p.has_shared) {
    stage_rows<FMT, false>(act_s + (size_t)te * ld, actsum + (size_t)te * (ld / 32), p.S, ld, m,
                           [&](int j) { return (const uint8_t*)(p.act_sh + (size_t)j * p.S); },
                           0, kFusedThreads);
  }
  __syncthreads();
  MOE_STAMP(9);
  {
    // units: column pairs of each slot (the routed slots, then the shared expert)
    const int npair = (ncols + 1) / 2;
    const int n_units = npair * (U + p.has_shared);
    for (int u = warp; u < n_units; u += kFusedWarps) {
      const int slot = u / npair, col = c0 + 2 * (u - slot * npair);
      const bool two = col + 1 < c0 + ncols;
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
      const int nch = (int)(packed_row_bytes(FMT, K) / 16);
      const RowRef A = row_ref<FMT>(D, e, col);
      float a0[RB], a1[RB];
      if (two) {
        const RowRef B = row_ref<FMT>(D, e, col + 1);
        rows2_dot<FMT, RB, false>(A, B, nch, xr, xsr, n, a0, a1);
      } else {
        rows1_dot<FMT, RB, false>(A, nch, xr, xsr, n, a0);
      }
      if (lane < n) {
        float v0 = 0.f, v1 = 0.f;
#pragma unroll
        for (int j = 0; j < RB; ++j)
          if (j == lane) {
            v0 = a0[j];
            if (two) v1 = a1[j];
          }
        ys[(size_t)(beg + lane) * ncols + (col - c0)] = v0 * A.ts;
        if (two) ys[(size_t)(beg + lane) * ncols + (col + 1 - c0)] = v1 * A.ts;
      }
    }
  }
  __syncthreads();
  MOE_STAMP(10);
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
  MOE_STAMP(11);
}

}  // namespace moe
