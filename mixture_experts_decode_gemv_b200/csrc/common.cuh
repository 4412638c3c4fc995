// Shared definitions of the decode MoE kernels: launch parameters, workspace layout, small PTX
// helpers. Device code targets sm_100a only.
#pragma once

#include <cstdint>
#include <type_traits>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "../../include/moe_decode.h"

namespace moe {

// Work-tile geometry shared by the host launcher and the kernels.
constexpr int kThreads = 256;          // 8 warps per CTA in the expert kernels
constexpr int kWarps = kThreads / 32;
constexpr int kRowsPerWarp = 4;        // gate/up row pairs a warp reduces, one after another
constexpr int kRowsPerCta = kWarps * kRowsPerWarp;  // 32 gate/up row pairs per CTA tile
constexpr int kColsPerCta = 2 * kRowsPerCta;       // 64 down-projection output columns per CTA
constexpr int kRouterThreads = 128;
constexpr int kCtrlBytes = 256;

// Control words at the start of the workspace.
enum CtrlWord { kStatus = 0, kRouterTicket = 1 };

struct MatDev {
  const uint8_t* packed;
  const uint8_t* scales;
  const uint8_t* biases;
  const float* tscale;
  long long estride;   // bytes between experts (packed)
  long long sstride;   // bytes between experts (scales / biases)
  int fmt;
  int n, k;            // rows and columns of one expert matrix
};

// Field-wise choice between two matrix descriptors of the kernel parameters. Each field stays a
// constant-bank read; binding a reference to either descriptor at run time would read the
// fields through a generic pointer, from memory.
__device__ __forceinline__ MatDev pick_mat(bool first, const MatDev& a, const MatDev& b) {
  MatDev r;
  r.packed = first ? a.packed : b.packed;
  r.scales = first ? a.scales : b.scales;
  r.biases = first ? a.biases : b.biases;
  r.tscale = first ? a.tscale : b.tscale;
  r.estride = first ? a.estride : b.estride;
  r.sstride = first ? a.sstride : b.sstride;
  r.fmt = first ? a.fmt : b.fmt;
  r.n = first ? a.n : b.n;
  r.k = first ? a.k : b.k;
  return r;
}

// Byte offsets of the workspace regions (all 256-byte aligned).
struct WsLayout {
  size_t logits, idx, wts, gamma, sorted_pairs, offsets, token_to_perm, active, active_count;
  size_t act, act_sh, ypart, ysh, tickets, total;
};

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

inline WsLayout make_layout(int m, int h, int E, int k, int I, int S, int n_tiles_c) {
  WsLayout L;
  const size_t te = (size_t)m * k;
  const size_t cap = te < (size_t)E ? te : (size_t)E;
  size_t off = kCtrlBytes;
  auto take = [&](size_t bytes) { size_t at = off; off = align256(off + bytes); return at; };
  L.logits = take((size_t)m * (E + 1) * 4);
  L.idx = take(te * 4);
  L.wts = take(te * 4);
  L.gamma = take((size_t)m * 4);
  L.sorted_pairs = take(te * 4);
  L.offsets = take((size_t)(E + 1) * 4);
  L.token_to_perm = take(te * 4);
  L.active = take(cap * 4);
  L.active_count = take(4);
  L.act = take(te * (size_t)I * 4);
  L.act_sh = take((size_t)m * (S > 0 ? S : 1) * 4);
  L.ypart = take(te * (size_t)h * 4);
  L.ysh = take((size_t)m * h * 4);
  L.tickets = take((size_t)n_tiles_c * 4);
  L.total = off;
  return L;
}

struct Params {
  int m, h, E, k, I, S;
  int routing, norm, raw, has_bias, before_ffn, shared_kind, out_bf16, act_kind;
  float rsf;
  int cap;             // min(m*k, E): routed work slots
  int n_tiles_i;       // routed gate/up tiles per expert
  int n_tiles_s;       // shared gate/up tiles
  int n_tiles_c;       // output-column tiles of the down projection
  int has_shared;
  int slot_base;       // first work slot of a down launch (shared-only launches start at cap)
  const void* x;
  const void* router_w;
  const float* expert_bias;
  const void* shared_gate_w;
  MatDev rg, ru, rd;   // routed gate, up, down
  MatDev sg, su, sd;   // shared gate, up, down
  void* out;
  unsigned* ctrl;
  float* logits;
  int* idx;
  float* wts;
  float* gamma;
  int* sorted_pairs;
  int* offsets;
  int* token_to_perm;
  int* active;
  int* active_count;
  float* act;
  float* act_sh;
  float* ypart;
  float* ysh;
  unsigned* tickets;
};

// ---- PTX helpers -------------------------------------------------------------------------------

// Streaming 16-byte load of weights: read-only path, no L1 allocation.
// L2 policy for weights that one call reads once: evict them first, so that streaming them does
// not push out what the next call needs again soon (its code and parameters, the router rows,
// activations, the routing workspace). No side effects: the compiler may hoist or merge it.
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t pol;
  asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p), "l"(l2_evict_first()));
  return r;
}

// Programmatic dependent launch: wait for the preceding grid's completion (no-op without PDL)
// and allow the next grid to start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ float sigmoidf_(float z) { return 1.0f / (1.0f + __expf(-z)); }

__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.0f + __expf(-g)) * u; }

// GELU, tanh form, times u: g/2 * (1 + tanh(sqrt(2/pi) * (g + 0.044715 g^3))) * u.
__device__ __forceinline__ float gelu_tanh_mul(float g, float u) {
  const float t = tanhf(0.7978845608028654f * fmaf(0.044715f * g, g * g, g));
  return 0.5f * g * (1.0f + t) * u;
}

// The expert activation of the call: SwiGLU or GeGLU (moe_activation).
__device__ __forceinline__ float act_mul(int act, float g, float u) {
  return act == MOE_ACT_GEGLU ? gelu_tanh_mul(g, u) : silu_mul(g, u);
}

// Optional phase timestamps (build with -DMOE_PHASE_TIMERS): thread 0 of every CTA records
// the SM cycle counter at each phase boundary into the (otherwise unused) down-partials region
// of the workspace, as uint64 [cta][kPhaseSlots]; slot kPhaseSlots - 1 holds %globaltimer at
// entry, to line the CTAs up. MOE_STAMP_AFTER(slot, v) reads the counter only once the 32-bit
// value v has been computed.
constexpr int kPhaseSlots = 20;
#ifdef MOE_PHASE_TIMERS
#define MOE_STAMP_AFTER(slot, v)                                                            \
  do {                                                                                      \
    if (threadIdx.x == 0) {                                                                 \
      unsigned long long t_;                                                                \
      asm volatile("{ .reg .u32 d_; mov.u32 d_, %1; mov.u64 %0, %%clock64; }"               \
                   : "=l"(t_) : "r"((unsigned)(v)) : "memory");                              \
      reinterpret_cast<unsigned long long*>(p.ypart)[blockIdx.x * kPhaseSlots + (slot)] = t_; \
    }                                                                                       \
  } while (0)
#define MOE_STAMP_GLOBAL()                                                                  \
  do {                                                                                      \
    if (threadIdx.x == 0) {                                                                 \
      unsigned long long t_;                                                                \
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_)::"memory");                      \
      reinterpret_cast<unsigned long long*>(p.ypart)[blockIdx.x * kPhaseSlots + kPhaseSlots - 1] = t_; \
    }                                                                                       \
  } while (0)
#else
#define MOE_STAMP_AFTER(slot, v) \
  do {                           \
  } while (0)
#define MOE_STAMP_GLOBAL() \
  do {                     \
  } while (0)
#endif
#define MOE_STAMP(slot) MOE_STAMP_AFTER(slot, 0u)

}  // namespace moe
