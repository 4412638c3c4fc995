// One persistent kernel for a whole decode MoE layer call (m <= 4 rows).
//
// All CTAs are co-resident (cooperative launch, one CTA per SM, 16 warps). Phases:
//   A  router logits: stage the m activation rows in shared memory as fp32, one warp per
//      (router row, activation row) dot product (router rows were asked into L2 before the
//      programmatic-launch wait); arrive at grid barrier 1 without waiting.
//   B  shared expert gate+up (needs no routing): this CTA's slice of the S row pairs. Meanwhile
//      one idle warp runs the routing code on throw-away rows, so its instructions are cached
//      when phase C needs them.
//   C  wait at barrier 1; every CTA routes every row and groups the pairs by expert in its own
//      shared memory (m*k <= 32 pairs).
//   D  routed gate+up: the U*I row pairs of the U active experts in equal contiguous slices, one
//      per CTA. The last warp bulk-copies the down rows this CTA needs in phase E into a
//      shared-memory tile (slots that do not fit are asked into L2 instead), so they arrive
//      while gate/up streams. Arrive and wait at grid barrier 2.
//   E  down + blend: each CTA owns a contiguous range of output columns for all rows; y for each
//      (column, active expert) and for the shared expert, from the tile, then the blend: routed
//      slots in slot order times their weight, then gamma times the shared expert. No atomics.
// Every weight row is reduced by one warp with the multi-kernel path's arithmetic (lane l takes
// chunks l, l+32, ..., then a butterfly sum), so both paths give the same bits and a row's bits
// do not depend on m. Every wait is bounded (clock64 budget): on expiry it records
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
  int tile_off;       // down-row tile: slot s of phase E at tile_off + s * tile_slot_bytes
  int tile_slots;     // slots the tile region holds (0: no tile)
  int tile_slot_bytes;
  int tile_sc_off;    // within a slot: scales rows, then (Q4) biases rows at 2 * tile_sc_off -
  int tile_bi_off;    //   packed rows first, each block 16-byte aligned
  int smem_bytes;
  long long spin_limit;       // clock cycles a grid-barrier wait may spin before it gives up
  long long tile_limit;       // the same for the down-row tile's copies
  long long l2_prefetch_cap;  // largest per-call down-projection byte count asked into L2
  unsigned bar_extra;         // arrivals a barrier waits for beyond the grid (0; 1 in tests)
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

// Shared-memory transaction barrier fed by bulk copies (one phase per launch).
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(unsigned long long* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(unsigned long long* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                   smem_addr(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(unsigned long long* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar))
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(unsigned long long* bar, unsigned parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}
// Bounded wait for phase `parity` of bar; false when `limit` clock cycles passed first.
__device__ __forceinline__ bool mbar_wait_bounded(unsigned long long* bar, unsigned parity,
                                                  long long limit) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > limit) return false;
  return true;
}
// Global -> shared bulk copy (addresses 16-byte aligned, bytes a multiple of 16) completing as
// transaction bytes on bar; the source lines are marked evict-first in L2 (read once).
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes,
                                         unsigned long long* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], "
      "%2, [%3], %4;" ::"r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(l2_evict_first())
      : "memory");
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
  unsigned extra;  // 0, or 1 to make every wait run out (failure-detection tests)

  __device__ void arrive() const {
    __syncthreads();
    if (threadIdx.x == 0)
      asm volatile("red.release.gpu.global.add.u64 [%0], 1;" ::"l"(ctr) : "memory");
  }
  __device__ void wait(unsigned passed) const {
    if (threadIdx.x == 0) {
      const unsigned long long target = base + (unsigned long long)passed * gridDim.x + extra;
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
  alignas(16) int idx[kFusedMaxPairs];
  float w[kFusedMaxPairs];
  float gamma[kFusedMaxRows];
  int sorted[kFusedMaxPairs];     // pair ids by (expert, pair)
  int tp[kFusedMaxPairs];         // position of each pair in `sorted`
  int slot_e[kFusedMaxPairs];     // active experts, ascending
  int slot_beg[kFusedMaxPairs];   // first position of each active expert in `sorted`
  int slot_n[kFusedMaxPairs];     // its number of pairs
  int n_active;
  float bias[MOE_MAX_EXPERTS];    // expert biases, staged once per call
  float ts[kFusedMaxPairs + 1];   // NVFP4 / FP8 tensor scale of each phase-E slot's down matrix
};

// Route row r (one warp) into the CTA's shared routing tables (same rule and arithmetic as the
// multi-kernel path). Kept out of line so its per-lane candidate arrays get registers of their
// own instead of competing with the streaming loops of the kernel around it.
// With `dry` set it runs the same instructions on any readable rows and stores nothing: an idle
// warp calls it that way ahead of time, so that the routing code is already in this SM's
// instruction caches when the real call runs (it runs once per call, after the weights
// streamed by the previous calls have pushed it out of L2).
__device__ __noinline__ void fused_route_row(const RouteCfg c, unsigned* status, int r,
                                             FusedRoute& R, bool dry) {
  const int lane = threadIdx.x & 31;
  int id;
  float w, g;
  const bool ok = route_row(c, r, R.bias, id, w, g);
  if (dry) return;
  if (lane < c.k) {
    R.idx[r * c.k + lane] = id;
    R.w[r * c.k + lane] = w;
  }
  if (lane == 0) {
    R.gamma[r] = g;
    if (!ok) atomicExch(status, (unsigned)MOE_ERR_DEVICE_CHECK);
  }
}

// Stable grouping of te <= 32 pairs by expert, by warp 0: pair p (one lane) lands at
// #(pairs with a smaller expert id) + #(earlier pairs with the same id); the first pair of each
// expert opens its slot, slots ordered by expert id. Equal ids come from one match; the counts
// of smaller ids from every lane reading all te ids (broadcast shared loads).
__device__ __forceinline__ void fused_group(int te, FusedRoute& R) {
  constexpr unsigned kFull = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x >= 32) return;
  const bool live = lane < te;
  const int e = live ? R.idx[lane] : 0x7fffffff;
  const unsigned same = __match_any_sync(kFull, e);
  const int eq_before = __popc(same & ((1u << lane) - 1u)), eq_all = __popc(same);
  const bool leader = live && eq_before == 0;
  const unsigned leaders = __ballot_sync(kFull, leader);
  int less = 0, slot = 0;
  for (int q = 0; q < te; q += 4) {
    const int4 v = *reinterpret_cast<const int4*>(&R.idx[q]);
    const int vq[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const bool lt = q + t < te && vq[t] < e;
      less += lt;
      slot += lt && ((leaders >> (q + t)) & 1u);
    }
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
__device__ __forceinline__ void fused_publish(const Params& p, const FusedRoute& R, int nt) {
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


// Row `lc` (column c0 + lc) of a down matrix held in a shared-memory tile slot.
template <int FMT>
__device__ __forceinline__ RowRef tile_row_ref(const MatDev& D, int e, const uint8_t* slot, int K,
                                               const FusedPlan& fp, int lc) {
  RowRef r;
  r.w = slot + (size_t)lc * packed_row_bytes(FMT, K);
  r.sc = nullptr;
  r.bi = nullptr;
  r.ts = 1.f;
  if constexpr (FMT == MOE_FMT_Q4_AFFINE_G64) {
    r.sc = slot + fp.tile_sc_off + (size_t)lc * (K / 64) * 2;
    r.bi = slot + fp.tile_bi_off + (size_t)lc * (K / 64) * 2;
  } else if constexpr (FMT == MOE_FMT_NVFP4) {
    r.sc = slot + fp.tile_sc_off + (size_t)lc * (K / 16);  // ts: the caller's (staged per slot)
  } else if constexpr (FMT == MOE_FMT_MXFP4) {
    r.sc = slot + fp.tile_sc_off + (size_t)lc * (K / 32);
  }
  return r;
}

template <int FMT, bool XBF16, int RB>
__global__ void __launch_bounds__(kFusedThreads, 1) moe_fused_kernel(
    const __grid_constant__ Params p, const __grid_constant__ FusedPlan fp) {
  extern __shared__ __align__(16) uint8_t fsmem[];
  __shared__ FusedRoute R;
  __shared__ unsigned long long s_base;
  __shared__ unsigned long long s_tile_bar;   // the down-row tile's bulk copies
  __shared__ unsigned long long s_tile_mask;  // phase-E slots whose rows sit in the tile
  __shared__ int s_tile_n;                    // slots offered to the tile
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
  MOE_STAMP_GLOBAL();

  // ---- prologue (may overlap the previous kernel): this CTA's router rows into L2 -----------
  if (tid == 0)
    for (int e = cta; e < e_tot; e += G) prefetch_l2_bulk(router_row(e), xrow_bytes);
  pdl_wait();
  MOE_STAMP(1);
  if (p.has_bias)
    for (int e = tid; e < p.E; e += kFusedThreads) R.bias[e] = __ldg(p.expert_bias + e);
  unsigned long long* bar_ctr = reinterpret_cast<unsigned long long*>(p.ctrl + kBarCounter);
  if (tid == 0) s_base = ld_acquire_u64(bar_ctr) / (unsigned long long)G * (unsigned long long)G;
  stage_rows<FMT, XBF16>(xs, xsum, h, h, m, [&](int j) {
    return (const uint8_t*)p.x + (size_t)j * xrow_bytes;
  }, 0, kFusedThreads);
  __syncthreads();
  const GridBarrier bar{bar_ctr, p.ctrl + kStatus, s_base, fp.spin_limit, fp.bar_extra};
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
  if (warp == kFusedWarps - 4) {  // same scheduler partition as warp 0, which routes row 0
    RouteCfg dc = route_cfg(p);
    dc.logits = reinterpret_cast<const float*>(p.router_w);  // >= E + 1 floats, any values
    fused_route_row(dc, p.ctrl + kStatus, 0, R, true);
#ifdef MOE_PHASE_TIMERS
    if (lane == 0) {
      unsigned long long t_;
      asm volatile("mov.u64 %0, %%clock64;" : "=l"(t_)::"memory");
      reinterpret_cast<unsigned long long*>(p.ypart)[blockIdx.x * kPhaseSlots + 18] = t_;
    }
#endif
  }

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
        p.act_sh[(size_t)lane * p.S + i] = act_mul(p.act_kind, g * A.ts, u * B.ts);
      }
    }
  }
  MOE_STAMP(4);

  // ---- C: routing + grouping (every CTA, in its own shared memory) ---------------------------
  bar.wait(1);
  MOE_STAMP(5);
  if (warp < m) fused_route_row(route_cfg(p), p.ctrl + kStatus, warp, R, false);
  MOE_STAMP(12);
  __syncthreads();
  fused_group(te, R);
  if (tid == 0) {  // thread 0 wrote n_active in fused_group
    const int n_slots = R.n_active + p.has_shared;
    const int n_tile = ncols > 0 ? min(n_slots, fp.tile_slots) : 0;
    s_tile_mask = 0;
    s_tile_n = n_tile;
    if (n_tile > 0) mbar_init(&s_tile_bar, (unsigned)n_tile);
  }
  __syncthreads();
  const int U = R.n_active;
  MOE_STAMP(6);

  // ---- D: routed gate + up; this CTA's phase-E down rows on their way ------------------------
  // The last warp takes the phase-E slots (active experts in slot order, then the shared
  // expert), lane s slot s, s + 32: the first tile_slots slots are bulk-copied into this CTA's
  // shared-memory tile (when their addresses allow), the others are asked into L2 (when the
  // whole call's down rows fit comfortably there). Both arrive while gate/up streams. Issuing
  // bulk copies can hold the issuing warp until earlier ones drain, so with a tile the last warp
  // does only this and the gate/up rows go to the other warps.
  const bool tile_call = s_tile_n > 0;
  const int n_gu_warps = tile_call ? kFusedWarps - 1 : kFusedWarps;
  if (warp == kFusedWarps - 1 && ncols > 0) {
    const size_t down_bytes =
        ((size_t)U * packed_row_bytes(FMT, p.I) + (p.has_shared ? packed_row_bytes(FMT, p.S) : 0)) *
        (size_t)h;
    for (int sl = lane; sl < U + p.has_shared; sl += 32) {
      const bool sh = sl == U;
      const MatDev D = pick_mat(sh, p.sd, p.rd);
      const int e = sh ? 0 : R.slot_e[sl];
      const int K = sh ? p.S : p.I;
      const size_t prb = packed_row_bytes(FMT, K);
      const size_t srb = FMT == MOE_FMT_Q4_AFFINE_G64 ? (size_t)(K / 64) * 2
                         : FMT == MOE_FMT_NVFP4        ? (size_t)(K / 16)
                         : FMT == MOE_FMT_MXFP4        ? (size_t)(K / 32)
                                                       : 0;
      const uint8_t* wsrc = D.packed + (size_t)e * D.estride + (size_t)c0 * prb;
      const uint8_t* ssrc = srb ? D.scales + (size_t)e * D.sstride + (size_t)c0 * srb : nullptr;
      const uint8_t* bsrc = FMT == MOE_FMT_Q4_AFFINE_G64
                                ? D.biases + (size_t)e * D.sstride + (size_t)c0 * srb
                                : nullptr;
      const unsigned wb = (unsigned)(ncols * prb), sb = (unsigned)(ncols * srb);
      if (FMT == MOE_FMT_NVFP4 || FMT == MOE_FMT_FP8_E4M3) R.ts[sl] = __ldg(D.tscale + e);
      bool in_tile = false;
      if (sl < s_tile_n) {
        in_tile = sb % 16 == 0 && ((uintptr_t)ssrc | (uintptr_t)bsrc) % 16 == 0;
        if (in_tile) {
          uint8_t* dst = fsmem + fp.tile_off + (size_t)sl * fp.tile_slot_bytes;
          const unsigned tx = wb + (FMT == MOE_FMT_Q4_AFFINE_G64 ? 2 * sb : sb);
          mbar_arrive_expect_tx(&s_tile_bar, tx);
          bulk_g2s(dst, wsrc, wb, &s_tile_bar);
          if (srb) bulk_g2s(dst + fp.tile_sc_off, ssrc, sb, &s_tile_bar);
          if (FMT == MOE_FMT_Q4_AFFINE_G64) bulk_g2s(dst + fp.tile_bi_off, bsrc, sb, &s_tile_bar);
          atomicOr(&s_tile_mask, 1ull << sl);
        } else {
          mbar_arrive(&s_tile_bar);
        }
      }
      if (!in_tile && down_bytes <= (size_t)fp.l2_prefetch_cap) {
        prefetch_l2_bulk(wsrc, wb);
        if (srb) prefetch_l2_lines(ssrc, sb);
        if (bsrc) prefetch_l2_lines(bsrc, sb);
      }
    }
  }
  {
    const long long UI = (long long)U * p.I;
    const long long q0 = (long long)cta * UI / G, q1 = (long long)(cta + 1) * UI / G;
    for (long long q = q0 + warp; warp < n_gu_warps && q < q1; q += n_gu_warps) {
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
        p.act[(size_t)(beg + lane) * p.I + i] = act_mul(p.act_kind, g, u);
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
  // Thread 0 waits for the tile's copies and decides for the whole CTA. When the wait runs out
  // the status records it and every slot is read from global memory instead (same arithmetic);
  // the copies still target this CTA's shared memory, so the CTA waits for them once more, with
  // the same bound, before it exits.
  __shared__ int s_tile_ok;
  if (tid == 0) {
    const bool ok = s_tile_mask == 0 || mbar_wait_bounded(&s_tile_bar, 0, fp.tile_limit);
    if (!ok) atomicExch(p.ctrl + kStatus, (unsigned)MOE_ERR_DEVICE_TIMEOUT);
    s_tile_ok = ok;
  }
  __syncthreads();
  const bool tile_ok = s_tile_ok != 0;
  const unsigned long long tile_mask = tile_ok ? s_tile_mask : 0ull;
  MOE_STAMP_AFTER(16, (unsigned)tile_mask);
  // units: column pairs of each slot (the routed slots, then the shared expert). A CTA with a
  // down-row tile reads every row through plain loads (tile slots from shared memory, the rest
  // from L2); one without streams its rows from global memory. Same arithmetic either way.
  auto down_units = [&](auto plain_tag) {
    constexpr bool kPlain = decltype(plain_tag)::value;
    constexpr int NR = kPlain ? 4 : 2;  // output columns per unit
    const int nblk = (ncols + NR - 1) / NR;
    const int n_units = nblk * (U + p.has_shared);
    for (int u = warp; u < n_units; u += kFusedWarps) {
      const int slot = u / nblk, col = c0 + NR * (u - slot * nblk);
      const int nvalid = min(NR, c0 + ncols - col);
      const bool sh = slot == U;
      const MatDev D = pick_mat(sh, p.sd, p.rd);
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
      const bool in_tile = kPlain && ((tile_mask >> slot) & 1ull);
      const uint8_t* sl = fsmem + fp.tile_off + (size_t)slot * fp.tile_slot_bytes;
      // columns past the CTA's last repeat its last column (results dropped)
      RowRef A[NR];
#pragma unroll
      for (int r = 0; r < NR; ++r) {
        const int cr = col + min(r, nvalid - 1);
        A[r] = in_tile ? tile_row_ref<FMT>(D, e, sl, K, fp, cr - c0) : row_ref<FMT>(D, e, cr);
      }
      const float ts = (FMT == MOE_FMT_NVFP4 || FMT == MOE_FMT_FP8_E4M3) ? R.ts[slot] : 1.f;
      float acc[NR][RB];
      rowsN_dot<FMT, RB, kPlain, NR>(A, nch, xr, xsr, n, acc);
      if (lane < n) {
#pragma unroll
        for (int r = 0; r < NR; ++r) {
          float v = 0.f;
#pragma unroll
          for (int j = 0; j < RB; ++j)
            if (j == lane) v = acc[r][j];
          if (r < nvalid) ys[(size_t)(beg + lane) * ncols + (col + r - c0)] = v * ts;
        }
      }
      if (u == warp) MOE_STAMP_AFTER(17, __float_as_uint(acc[0][0]));  // warp 0's first unit
    }
  };
  if (tile_mask) {
    down_units(std::true_type{});
  } else {
    down_units(std::false_type{});
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
  if (!tile_ok && tid == 0) mbar_wait_bounded(&s_tile_bar, 0, fp.tile_limit);
  MOE_STAMP(11);
}

}  // namespace moe
