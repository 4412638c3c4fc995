// Router GEMV, top-k routing and grouping of (row, slot) pairs by expert, in one launch.
//
// Every CTA computes the logits of one router row (one expert, or the shared-expert gate vector)
// for all m activation rows. The CTA that finishes last (an atomic ticket, no spinning) then
// routes every row and groups the pairs by expert:
//   - routing per row follows the options of the layer (softmax, or sigmoid with an optional
//     expert bias for selection only, raw-logit selection, norm_topk_prob, routed scaling);
//   - grouping is a stable counting sort of pair ids p = r*k + s by expert id, giving
//     sorted_pairs, expert_offsets, token_to_perm, the ascending active-expert list and its count
//     (the sort step of metrale "forward_bf16_grouped_decode.rs").
#pragma once

#include "common.cuh"

namespace moe {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// One router dot product by one warp: lane l takes 16-byte chunks l, l+32, ... of the router
// row, xchunk(c, xv) supplies the chunk's activations as fp32, then a butterfly warp sum. The
// weight loads of up to 8 chunks are issued before any is used. Both launch paths use this, so a
// logit's bits do not depend on which path (or m) computed it.
template <bool XBF16, typename XChunk>
__device__ __forceinline__ float router_dot_warp(const uint8_t* row, int nch, XChunk xchunk) {
  const int lane = threadIdx.x & 31;
  float acc = 0.f;
  for (int c0 = lane; c0 < nch; c0 += 32 * 8) {
    uint4 w[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (c0 + 32 * u < nch) w[u] = ldg_stream(row + (size_t)(c0 + 32 * u) * 16);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int c = c0 + 32 * u;
      if (c < nch) {
        float xv[8];
        xchunk(c, xv);
        if constexpr (XBF16) {
          acc = fmaf(bf16lo(w[u].x), xv[0], acc);
          acc = fmaf(bf16hi(w[u].x), xv[1], acc);
          acc = fmaf(bf16lo(w[u].y), xv[2], acc);
          acc = fmaf(bf16hi(w[u].y), xv[3], acc);
          acc = fmaf(bf16lo(w[u].z), xv[4], acc);
          acc = fmaf(bf16hi(w[u].z), xv[5], acc);
          acc = fmaf(bf16lo(w[u].w), xv[6], acc);
          acc = fmaf(bf16hi(w[u].w), xv[7], acc);
        } else {
          acc = fmaf(__uint_as_float(w[u].x), xv[0], acc);
          acc = fmaf(__uint_as_float(w[u].y), xv[1], acc);
          acc = fmaf(__uint_as_float(w[u].z), xv[2], acc);
          acc = fmaf(__uint_as_float(w[u].w), xv[3], acc);
        }
      }
    }
  }
  return warp_sum(acc);
}

// The same dot product (same chunk order per lane, same fma order, same butterfly sum) with the
// activation row in global memory: the weight and activation loads of up to 8 chunks per lane
// are issued together before any is used, so a chunk's activations cost no extra round trip.
template <bool XBF16>
__device__ __forceinline__ float router_dot_gx(const uint8_t* row, const uint8_t* xr, int nch) {
  const int lane = threadIdx.x & 31;
  float acc = 0.f;
  for (int c0 = lane; c0 < nch; c0 += 32 * 8) {
    uint4 w[8], x[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (c0 + 32 * u < nch) {
        w[u] = ldg_stream(row + (size_t)(c0 + 32 * u) * 16);
        x[u] = __ldg(reinterpret_cast<const uint4*>(xr) + c0 + 32 * u);
      }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (c0 + 32 * u < nch) {
        if constexpr (XBF16) {
          acc = fmaf(bf16lo(w[u].x), bf16lo(x[u].x), acc);
          acc = fmaf(bf16hi(w[u].x), bf16hi(x[u].x), acc);
          acc = fmaf(bf16lo(w[u].y), bf16lo(x[u].y), acc);
          acc = fmaf(bf16hi(w[u].y), bf16hi(x[u].y), acc);
          acc = fmaf(bf16lo(w[u].z), bf16lo(x[u].z), acc);
          acc = fmaf(bf16hi(w[u].z), bf16hi(x[u].z), acc);
          acc = fmaf(bf16lo(w[u].w), bf16lo(x[u].w), acc);
          acc = fmaf(bf16hi(w[u].w), bf16hi(x[u].w), acc);
        } else {
          acc = fmaf(__uint_as_float(w[u].x), __uint_as_float(x[u].x), acc);
          acc = fmaf(__uint_as_float(w[u].y), __uint_as_float(x[u].y), acc);
          acc = fmaf(__uint_as_float(w[u].z), __uint_as_float(x[u].z), acc);
          acc = fmaf(__uint_as_float(w[u].w), __uint_as_float(x[u].w), acc);
        }
      }
    }
  }
  return warp_sum(acc);
}

// Order-preserving map of a float key to uint32 (NaN ranks as -infinity).
__device__ __forceinline__ uint32_t key_bits(float v) {
  if (v != v) v = -INFINITY;
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Routing of row r by one warp. Lane s < k ends with the s-th selected expert (descending key,
// ties to the lower id) and its weight; every lane gets gamma (shared-expert gate, or 1).
// `bias` holds the expert biases (global memory or a shared-memory copy), read only when the
// keys are biased sigmoid scores. Every load of the row (logits, biases, the shared-gate logit)
// is issued before the first one is used. Each lane then sorts its NJ = E/32 candidates once;
// a selection round is one warp max over the lanes' heads and a ballot of the lanes holding it
// (a second reduction, min id, only when several lanes tie), after which the winning lane pops
// its head. Returns false when a selected key is not a finite number.
// Score of the non-softmax routers: sigmoid(l), or sqrt(softplus(l)) with
// softplus(l) = max(l, 0) + log1p(e^-|l|) (no overflow for large |l|).
__device__ __forceinline__ float router_score(int routing, float l) {
  if (routing == MOE_ROUTE_SQRTSOFTPLUS) return sqrtf(fmaxf(l, 0.f) + log1pf(expf(-fabsf(l))));
  return 1.0f / (1.0f + expf(-l));
}

// The routing options of a call, copied out of the kernel parameters into registers (a routine
// that reads them through a reference to the parameter block would load each one from memory).
struct RouteCfg {
  const float* logits;  // [m, E + 1]
  int E, k, routing, raw, has_bias, norm, gated;
  float rsf;
  unsigned long long* stamps;  // phase timestamps (timer builds only)
};

__device__ __forceinline__ RouteCfg route_cfg(const Params& p) {
  RouteCfg c;
  c.logits = p.logits;
  c.E = p.E;
  c.k = p.k;
  c.routing = p.routing;
  c.raw = p.raw;
  c.has_bias = p.has_bias;
  c.norm = p.norm;
  c.gated = p.shared_kind == MOE_SHARED_SIGMOID_GATE;
  c.rsf = p.rsf;
  c.stamps = reinterpret_cast<unsigned long long*>(p.ypart);
  return c;
}

#ifdef MOE_PHASE_TIMERS
#define MOE_ROUTE_STAMP(slot, v)                                                            \
  do {                                                                                      \
    if (threadIdx.x == 0) {                                                                 \
      unsigned long long t_;                                                                \
      asm volatile("{ .reg .u32 d_; mov.u32 d_, %1; mov.u64 %0, %%clock64; }"               \
                   : "=l"(t_) : "r"((unsigned)(v)) : "memory");                              \
      c.stamps[blockIdx.x * kPhaseSlots + (slot)] = t_;                                      \
    }                                                                                       \
  } while (0)
#else
#define MOE_ROUTE_STAMP(slot, v) \
  do {                           \
  } while (0)
#endif

template <int NJ>
__device__ __forceinline__ bool route_row_nj(const RouteCfg& c, int r, const float* bias,
                                             int& my_id, float& my_w, float& gamma) {
  constexpr unsigned kFull = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  const int E = c.E, k = c.k;
  const float* lrow = c.logits + (size_t)r * (E + 1);
  const bool sig_keys = c.routing != MOE_ROUTE_SOFTMAX && !c.raw;  // keys are router scores
  const bool add_bias = sig_keys && c.has_bias;
  const bool gated = c.gated;
  float lg[NJ], bs[NJ];
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const int e = lane + 32 * j;
    lg[j] = e < E ? __ldcg(lrow + e) : -INFINITY;
    bs[j] = (add_bias && e < E) ? bias[e] : 0.f;
  }
  const float glog = gated ? __ldcg(lrow + E) : 0.f;
  MOE_ROUTE_STAMP(13, __float_as_uint(lg[0]) ^ __float_as_uint(bs[0]) ^ __float_as_uint(glog));
  uint32_t key[NJ];
  int id[NJ];
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const int e = lane + 32 * j;
    float kv = lg[j];
    if (sig_keys) {
      kv = router_score(c.routing, lg[j]);
      if (add_bias) kv += bs[j];
    }
    key[j] = e < E ? key_bits(kv) : 0u;  // a real key is >= key_bits(-inf) > 0
    id[j] = e;
  }
  // sort network: position a ends before position b (descending key, then ascending id)
  auto cx = [&](int a, int b) {
    if (key[b] > key[a] || (key[b] == key[a] && id[b] < id[a])) {
      const uint32_t tk = key[a];
      key[a] = key[b];
      key[b] = tk;
      const int ti = id[a];
      id[a] = id[b];
      id[b] = ti;
      const float tl = lg[a];
      lg[a] = lg[b];
      lg[b] = tl;
    }
  };
  if constexpr (NJ == 2) cx(0, 1);
  if constexpr (NJ == 4) {
    cx(0, 1); cx(2, 3); cx(0, 2); cx(1, 3); cx(1, 2);
  }
  if constexpr (NJ == 8) {
    cx(0, 2); cx(1, 3); cx(4, 6); cx(5, 7); cx(0, 4); cx(1, 5); cx(2, 6); cx(3, 7);
    cx(0, 1); cx(2, 3); cx(4, 5); cx(6, 7); cx(2, 4); cx(3, 5); cx(1, 4); cx(3, 6);
    cx(1, 2); cx(3, 4); cx(5, 6);
  }
  MOE_ROUTE_STAMP(14, key[0] ^ (uint32_t)id[0] ^ __float_as_uint(lg[0]));
  const bool softmax = c.routing == MOE_ROUTE_SOFTMAX;
  bool ok = true;
  my_id = 0;
  float my_l = 0.f, top_l = 0.f, den = 0.f;
#pragma unroll 1
  for (int s = 0; s < k; ++s) {  // kept rolled: the body is fetched once, not k times
    const uint32_t best = __reduce_max_sync(kFull, key[0]);
    const bool mine = key[0] == best;
    const unsigned tied = __ballot_sync(kFull, mine);
    int owner = __ffs(tied) - 1;
    if (tied & (tied - 1u))
      owner = (int)(__reduce_min_sync(kFull, mine ? (uint32_t)id[0] : 0xffffffffu) & 31u);
    const int sid = __shfl_sync(kFull, id[0], owner);
    const float sl = __shfl_sync(kFull, lg[0], owner);
    if (best <= key_bits(-INFINITY)) ok = false;  // -inf or NaN won a slot
    if (s == 0) {
      top_l = sl;  // softmax keys are the logits: the first winner holds the largest one
      if (softmax && !c.norm) {
#pragma unroll
        for (int j = 0; j < NJ; ++j) den += expf(lg[j] - top_l);  // -inf past E adds 0
      }
    }
    if (lane == s) {
      my_id = sid;
      my_l = sl;
    }
    if (lane == owner) {
#pragma unroll
      for (int j = 0; j + 1 < NJ; ++j) {
        key[j] = key[j + 1];
        id[j] = id[j + 1];
        lg[j] = lg[j + 1];
      }
      key[NJ - 1] = 0u;
      id[NJ - 1] = 0x7fffffff;
      lg[NJ - 1] = -INFINITY;
    }
  }
  MOE_ROUTE_STAMP(15, (uint32_t)my_id ^ __float_as_uint(my_l) ^ __float_as_uint(top_l));
  float wv;
  if (softmax) {
    // exp(l - max) / sum over all experts; under renormalisation the full sum cancels
    wv = expf(my_l - top_l);
    if (!c.norm) wv = wv / warp_sum(den);
  } else {
    wv = router_score(c.routing, my_l);
  }
  if (lane >= k) wv = 0.f;
  if (c.norm) {
    // lanes >= k hold 0, so the k-lane sum needs only the xor steps below the next power of 2
    float tot = wv;
    for (int off = (k > 4 ? 4 : k > 2 ? 2 : k > 1 ? 1 : 0); off > 0; off >>= 1)
      tot += __shfl_xor_sync(kFull, tot, off);
    wv = wv / tot;
  }
  my_w = wv * c.rsf;
  gamma = gated ? 1.0f / (1.0f + expf(-glog)) : 1.f;
  return ok;
}

__device__ __forceinline__ bool route_row(const RouteCfg& c, int r, const float* bias, int& my_id,
                                          float& my_w, float& gamma) {
  if (c.E <= 32) return route_row_nj<1>(c, r, bias, my_id, my_w, gamma);
  if (c.E <= 64) return route_row_nj<2>(c, r, bias, my_id, my_w, gamma);
  if (c.E <= 128) return route_row_nj<4>(c, r, bias, my_id, my_w, gamma);
  return route_row_nj<8>(c, r, bias, my_id, my_w, gamma);
}

// Routing of row r for the multi-kernel path: route_row, then the global and shared writes.
__device__ void route_row_warp(const Params& p, int r, int* s_idx) {
  const int lane = threadIdx.x & 31;
  int id;
  float w, g;
  const bool ok = route_row(route_cfg(p), r, p.expert_bias, id, w, g);
  if (lane < p.k) {
    p.idx[r * p.k + lane] = id;
    p.wts[r * p.k + lane] = w;
    s_idx[r * p.k + lane] = id;
  }
  if (lane == 0) {
    if (p.shared_kind == MOE_SHARED_SIGMOID_GATE) p.gamma[r] = g;
    if (!ok) atomicExch(p.ctrl + kStatus, (unsigned)MOE_ERR_DEVICE_CHECK);
  }
}

// Stable counting sort of the te pairs by expert (run by one CTA of kRouterThreads threads).
__device__ void group_pairs(const Params& p, const int* s_idx) {
  __shared__ int s_cnt[MOE_MAX_EXPERTS];
  __shared__ int s_off[MOE_MAX_EXPERTS + 1];
  __shared__ int s_wsum[kRouterThreads / 32][2];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int E = p.E, te = p.m * p.k;
  for (int e = tid; e < MOE_MAX_EXPERTS; e += kRouterThreads) s_cnt[e] = 0;
  __syncthreads();
  for (int q = tid; q < te; q += kRouterThreads) atomicAdd(&s_cnt[s_idx[q]], 1);
  __syncthreads();
  // exclusive scan of counts and of the non-empty flags; thread t owns experts 2t, 2t+1
  const int e0 = 2 * tid, e1 = 2 * tid + 1;
  const int c0 = e0 < E ? s_cnt[e0] : 0, c1 = e1 < E ? s_cnt[e1] : 0;
  const int f0 = c0 > 0, f1 = c1 > 0;
  int cs = c0 + c1, fs = f0 + f1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, cs, o), b = __shfl_up_sync(0xffffffffu, fs, o);
    if (lane >= o) {
      cs += a;
      fs += b;
    }
  }
  if (lane == 31) {
    s_wsum[warp][0] = cs;
    s_wsum[warp][1] = fs;
  }
  __syncthreads();
  int cbase = 0, fbase = 0;
  for (int w = 0; w < warp; ++w) {
    cbase += s_wsum[w][0];
    fbase += s_wsum[w][1];
  }
  const int cexcl = cbase + cs - (c0 + c1), fexcl = fbase + fs - (f0 + f1);
  if (e0 < E) {
    s_off[e0] = cexcl;
    p.offsets[e0] = cexcl;
    if (f0) p.active[fexcl] = e0;
  }
  if (e1 < E) {
    s_off[e1] = cexcl + c0;
    p.offsets[e1] = cexcl + c0;
    if (f1) p.active[fexcl + f0] = e1;
  }
  if (tid == kRouterThreads - 1) {
    p.offsets[E] = te;
    *p.active_count = fbase + fs;
  }
  __syncthreads();
  for (int q = tid; q < te; q += kRouterThreads) {
    const int e = s_idx[q];
    int rank = 0;
    for (int q2 = 0; q2 < q; ++q2) rank += (s_idx[q2] == e);
    const int pos = s_off[e] + rank;
    p.sorted_pairs[pos] = q;
    p.token_to_perm[q] = pos;
  }
}

template <bool XBF16>
__global__ void __launch_bounds__(kRouterThreads) router_topk_group_kernel(
    const __grid_constant__ Params p) {
  pdl_launch_dependents();
  const int erow = blockIdx.x;  // router row; erow == E is the shared-expert gate vector
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int esz = XBF16 ? 2 : 4;
  const size_t row_bytes = (size_t)p.h * esz;
  const int nch = (int)(row_bytes / 16);
  const uint8_t* wrow = erow < p.E ? (const uint8_t*)p.router_w + (size_t)erow * row_bytes
                                   : (const uint8_t*)p.shared_gate_w;
  const uint8_t* xb = (const uint8_t*)p.x;
  __shared__ int s_last;
  __shared__ int s_idx[MOE_MAX_ROWS * MOE_MAX_TOP_K];

  // one warp per activation row; the router row comes from L2 after the first warp's pass
  for (int r = warp; r < p.m; r += kRouterThreads / 32) {
    const uint8_t* xr = xb + (size_t)r * row_bytes;
    const float acc = router_dot_gx<XBF16>(wrow, xr, nch);
    if (lane == 0) p.logits[(size_t)r * (p.E + 1) + erow] = acc;
  }
  __syncthreads();

  if (tid == 0) {
    __threadfence();
    const unsigned t = atomicAdd(p.ctrl + kRouterTicket, 1u);
    s_last = (t == gridDim.x - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  for (int r = warp; r < p.m; r += kRouterThreads / 32) route_row_warp(p, r, s_idx);
  __syncthreads();
  group_pairs(p, s_idx);
  for (int t = tid; t < p.n_tiles_c; t += kRouterThreads) p.tickets[t] = 0u;
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    p.ctrl[kRouterTicket] = 0u;
  }
}

}  // namespace moe
