// Dequant-fused expert kernels of the decode MoE layer (CUDA-core GEMV-style tiles).
//
// gate_up_swiglu_kernel: one CTA = 32 rows i of one expert's gate and up matrices for every pair
//   routed to that expert (or every row, for the shared expert). 8 lanes share one (gate_i, up_i)
//   row pair, each lane streaming 16-byte chunks with non-allocating 128-bit loads and decoding
//   them in registers; the expert's activation rows are staged once in shared memory as fp32 and
//   read by all 32 row pairs (the 4 row pairs of a warp read the same addresses, a broadcast).
//   act[pos, i] = silu(g) * u is written per sorted pair position.
// down_blend_kernel: one CTA = 64 output columns of one active expert's down matrix (or the
//   shared expert's) for every row that uses it, into per-pair partials; the CTA that completes a
//   column tile last (atomic ticket, no spinning) blends the tile for every row: the routed slots
//   in slot order, each times its weight, then gamma times the shared expert.
// Accumulation is fp32 throughout; activations stay fp32 between the two kernels.
// The 8-lane reductions are full-warp shuffles, so every guard around them must be uniform
// across a warp: rows come 4 per warp and I, S (multiples of 4) and h (multiple of 8) keep the
// `i < N` / `col0 < h` guards warp-uniform (the host refuses other shapes).
#pragma once

#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "common.cuh"

namespace moe {

template <int FMT> struct Fmt;
template <> struct Fmt<MOE_FMT_F32> { static constexpr int kElems = 4; };
template <> struct Fmt<MOE_FMT_BF16> { static constexpr int kElems = 8; };
template <> struct Fmt<MOE_FMT_Q4_AFFINE_G64> { static constexpr int kElems = 32; };
template <> struct Fmt<MOE_FMT_NVFP4> { static constexpr int kElems = 32; };

__host__ __device__ constexpr size_t packed_row_bytes(int fmt, int k) {
  return fmt == MOE_FMT_F32 ? (size_t)k * 4 : fmt == MOE_FMT_BF16 ? (size_t)k * 2 : (size_t)k / 2;
}

// One decoded 16-byte chunk of a weight row. For the 4-bit affine format the codes are kept as
// f = 1 + q/16 (exact) and the group's scale s and bias b are folded as
//   sum_j (s q_j + b) x_j = 16 s * sum_j f_j x_j + (b - 16 s) * sum_j x_j.
template <int FMT> struct Dec;
template <> struct Dec<MOE_FMT_F32> { float w[4]; };
template <> struct Dec<MOE_FMT_BF16> { float w[8]; };
template <> struct Dec<MOE_FMT_Q4_AFFINE_G64> { float f[32]; float s16, bm; };
template <> struct Dec<MOE_FMT_NVFP4> { float v[32]; float s0, s1; };

// Row-local pointers of one weight row of one expert matrix.
struct RowRef {
  const uint8_t* w;   // packed row
  const uint8_t* sc;  // scales row (4-bit formats)
  const uint8_t* bi;  // biases row (Q4)
  float ts;           // tensor scale (NVFP4), else 1
};

template <int FMT>
__device__ __forceinline__ RowRef row_ref(const MatDev& M, int e, int row) {
  RowRef r;
  r.w = M.packed + (size_t)e * M.estride + (size_t)row * packed_row_bytes(FMT, M.k);
  r.sc = nullptr;
  r.bi = nullptr;
  r.ts = 1.f;
  if constexpr (FMT == MOE_FMT_Q4_AFFINE_G64) {
    r.sc = M.scales + (size_t)e * M.sstride + (size_t)row * (M.k / 64) * 2;
    r.bi = M.biases + (size_t)e * M.sstride + (size_t)row * (M.k / 64) * 2;
  } else if constexpr (FMT == MOE_FMT_NVFP4) {
    r.sc = M.scales + (size_t)e * M.sstride + (size_t)row * (M.k / 16);
    r.ts = __ldg(M.tscale + e);
  }
  return r;
}

template <int FMT>
__device__ __forceinline__ void decode(uint4 raw, const RowRef& rr, int c, Dec<FMT>& d) {
  const uint32_t q[4] = {raw.x, raw.y, raw.z, raw.w};
  if constexpr (FMT == MOE_FMT_F32) {
#pragma unroll
    for (int t = 0; t < 4; ++t) d.w[t] = __uint_as_float(q[t]);
  } else if constexpr (FMT == MOE_FMT_BF16) {
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      d.w[2 * t] = bf16lo(q[t]);
      d.w[2 * t + 1] = bf16hi(q[t]);
    }
  } else if constexpr (FMT == MOE_FMT_Q4_AFFINE_G64) {
#pragma unroll
    for (int t = 0; t < 4; ++t)
#pragma unroll
      for (int n = 0; n < 8; ++n)
        d.f[8 * t + n] = __uint_as_float(0x3F800000u | (((q[t] >> (4 * n)) & 0xFu) << 19));
    const float s = __half2float(__ldg((const __half*)rr.sc + (c >> 1)));
    const float b = __half2float(__ldg((const __half*)rr.bi + (c >> 1)));
    d.s16 = 16.f * s;
    d.bm = b - 16.f * s;
  } else {  // NVFP4: byte j holds elements 2j (low nibble) and 2j+1 (high nibble)
#pragma unroll
    for (int t = 0; t < 4; ++t)
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const __half2_raw hr = __nv_cvt_fp4x2_to_halfraw2(
            (__nv_fp4x2_storage_t)((q[t] >> (8 * b)) & 0xFFu), __NV_E2M1);
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
        d.v[8 * t + 2 * b] = f.x;
        d.v[8 * t + 2 * b + 1] = f.y;
      }
    const unsigned short s2 = __ldg((const unsigned short*)(rr.sc) + c);
    const __half2_raw hs = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)s2, __NV_E4M3);
    const float2 sf = __half22float2(*reinterpret_cast<const __half2*>(&hs));
    d.s0 = sf.x;
    d.s1 = sf.y;
  }
}

// Dot product of a decoded chunk with the fp32 activations xs[0..kElems) (16-byte aligned).
// xsum: for Q4, the sum of the chunk's 32 activations.
template <int FMT>
__device__ __forceinline__ float dot(const Dec<FMT>& d, const float* xs, float xsum) {
  if constexpr (FMT == MOE_FMT_F32 || FMT == MOE_FMT_BF16) {
    constexpr int N = Fmt<FMT>::kElems;
    float a = 0.f;
#pragma unroll
    for (int t = 0; t < N; t += 4) {
      const float4 x = *reinterpret_cast<const float4*>(xs + t);
      a = fmaf(d.w[t], x.x, a);
      a = fmaf(d.w[t + 1], x.y, a);
      a = fmaf(d.w[t + 2], x.z, a);
      a = fmaf(d.w[t + 3], x.w, a);
    }
    return a;
  } else if constexpr (FMT == MOE_FMT_Q4_AFFINE_G64) {
    float a = 0.f;
#pragma unroll
    for (int t = 0; t < 32; t += 4) {
      const float4 x = *reinterpret_cast<const float4*>(xs + t);
      a = fmaf(d.f[t], x.x, a);
      a = fmaf(d.f[t + 1], x.y, a);
      a = fmaf(d.f[t + 2], x.z, a);
      a = fmaf(d.f[t + 3], x.w, a);
    }
    return fmaf(d.s16, a, d.bm * xsum);
  } else {
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int t = 0; t < 16; t += 4) {
      const float4 x = *reinterpret_cast<const float4*>(xs + t);
      a0 = fmaf(d.v[t], x.x, a0);
      a0 = fmaf(d.v[t + 1], x.y, a0);
      a0 = fmaf(d.v[t + 2], x.z, a0);
      a0 = fmaf(d.v[t + 3], x.w, a0);
    }
#pragma unroll
    for (int t = 16; t < 32; t += 4) {
      const float4 x = *reinterpret_cast<const float4*>(xs + t);
      a1 = fmaf(d.v[t], x.x, a1);
      a1 = fmaf(d.v[t + 1], x.y, a1);
      a1 = fmaf(d.v[t + 2], x.z, a1);
      a1 = fmaf(d.v[t + 3], x.w, a1);
    }
    return fmaf(d.s0, a0, d.s1 * a1);
  }
}

__device__ __forceinline__ float sum8lanes(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  v += __shfl_xor_sync(0xffffffffu, v, 4);
  return v;
}

// Shared-memory staging of up to RB activation rows of length K as fp32, plus (Q4) the sum of
// every 32-element chunk. src(j) gives the global row pointer of staged row j.
template <int FMT, bool SRC_BF16, int RB, typename SrcFn>
__device__ __forceinline__ void stage_rows(float* xs, float* xsum, int K, int nb, SrcFn src) {
  const int tid = threadIdx.x;
  for (int j = 0; j < nb; ++j) {
    const uint8_t* g = src(j);
    float* dst = xs + (size_t)j * K;
    if constexpr (SRC_BF16) {
      for (int c = tid; c < K / 8; c += blockDim.x) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(g) + c);
        float4 a = make_float4(bf16lo(v.x), bf16hi(v.x), bf16lo(v.y), bf16hi(v.y));
        float4 b = make_float4(bf16lo(v.z), bf16hi(v.z), bf16lo(v.w), bf16hi(v.w));
        reinterpret_cast<float4*>(dst)[2 * c] = a;
        reinterpret_cast<float4*>(dst)[2 * c + 1] = b;
      }
    } else {
      for (int c = tid; c < K / 4; c += blockDim.x)
        reinterpret_cast<float4*>(dst)[c] = __ldcg(reinterpret_cast<const float4*>(g) + c);
    }
  }
  if constexpr (FMT == MOE_FMT_Q4_AFFINE_G64) {
    __syncthreads();
    const int nchunk = K / 32;
    for (int t = tid; t < nb * nchunk; t += blockDim.x) {
      const int j = t / nchunk, c = t - j * nchunk;
      const float* s = xs + (size_t)j * K + c * 32;
      float a = 0.f;
#pragma unroll
      for (int u = 0; u < 32; ++u) a += s[u];
      xsum[j * nchunk + c] = a;
    }
  }
}

template <int FMT>
constexpr int unroll_of() { return (FMT == MOE_FMT_F32) ? 4 : 4; }

// Accumulate two weight rows (A, B) against nb staged rows: acc_a[j], acc_b[j].
template <int FMT, int RB>
__device__ __forceinline__ void two_row_dots(const RowRef& A, const RowRef& B, int nch, int lg,
                                             const float* xs, const float* xsum, int K, int nb,
                                             float (&acc_a)[RB], float (&acc_b)[RB]) {
  constexpr int kE = Fmt<FMT>::kElems;
  constexpr int U = unroll_of<FMT>();
  const int nchunk32 = K / 32;
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
            const float* x = xs + (size_t)j * K + c * kE;
            float s = 0.f;
            if constexpr (FMT == MOE_FMT_Q4_AFFINE_G64) s = xsum[j * nchunk32 + c];
            acc_a[j] += dot<FMT>(da, x, s);
            acc_b[j] += dot<FMT>(db, x, s);
          }
        }
      }
    }
  }
}

template <int FMT, bool XBF16, int RB>
__global__ void __launch_bounds__(kThreads) gate_up_swiglu_kernel(const __grid_constant__ Params p) {
  pdl_launch_dependents();
  extern __shared__ __align__(16) float smem[];
  const int K = p.h;
  float* xs = smem;
  float* xsum = smem + (size_t)RB * K;
  const bool is_shared = (int)blockIdx.x < p.n_tiles_s;
  int tile, e = 0, beg = 0, nrows, N;
  const MatDev* G;
  const MatDev* U;
  float* dst;
  if (is_shared) {
    tile = blockIdx.x;
    G = &p.sg;
    U = &p.su;
    N = p.S;
    nrows = p.m;
    dst = p.act_sh;
  } else {
    pdl_wait();
    const int b = blockIdx.x - p.n_tiles_s;
    const int a = b / p.n_tiles_i;
    tile = b - a * p.n_tiles_i;
    if (a >= *(volatile int*)p.active_count) return;
    e = __ldcg(p.active + a);
    beg = __ldcg(p.offsets + e);
    nrows = __ldcg(p.offsets + e + 1) - beg;
    G = &p.rg;
    U = &p.ru;
    N = p.I;
    dst = p.act;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int lg = lane & (kLanesPerRow - 1);
  const int i = tile * kRowsPerCta + warp * kRowsPerWarp + (lane >> 3);
  const int nch = (int)(packed_row_bytes(FMT, K) / 16);
  const size_t xrow_bytes = (size_t)K * (XBF16 ? 2 : 4);
  RowRef A{}, B{};
  if (i < N) {
    A = row_ref<FMT>(*G, e, i);
    B = row_ref<FMT>(*U, e, i);
  }
  for (int rb = 0; rb < nrows; rb += RB) {
    const int nb = min(RB, nrows - rb);
    stage_rows<FMT, XBF16, RB>(xs, xsum, K, nb, [&](int j) {
      const int r = is_shared ? rb + j : __ldcg(p.sorted_pairs + beg + rb + j) / p.k;
      return (const uint8_t*)p.x + (size_t)r * xrow_bytes;
    });
    __syncthreads();
    if (i < N) {
      float ag[RB], au[RB];
#pragma unroll
      for (int j = 0; j < RB; ++j) ag[j] = au[j] = 0.f;
      two_row_dots<FMT, RB>(A, B, nch, lg, xs, xsum, K, nb, ag, au);
#pragma unroll
      for (int j = 0; j < RB; ++j) {
        ag[j] = sum8lanes(ag[j]);
        au[j] = sum8lanes(au[j]);
      }
      if (lg == 0) {
#pragma unroll
        for (int j = 0; j < RB; ++j) {
          if (j < nb) {
            float g = ag[j] * A.ts, u = au[j] * B.ts;
            size_t pos;
            if (is_shared) {
              pos = rb + j;
            } else {
              pos = beg + rb + j;
              if (p.before_ffn) {
                const float w = __ldcg(p.wts + __ldcg(p.sorted_pairs + pos));
                g *= w;
                u *= w;
              }
            }
            dst[pos * N + i] = silu_mul(g, u);
          }
        }
      }
    }
    __syncthreads();
  }
}

template <int FMT, int RB>
__global__ void __launch_bounds__(kThreads) down_blend_kernel(const __grid_constant__ Params p) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ __align__(16) float smem[];
  __shared__ int s_last;
  const int tile = blockIdx.x % p.n_tiles_c;
  const int a = p.slot_base + (int)blockIdx.x / p.n_tiles_c;
  const int cnt = *(volatile int*)p.active_count;
  const bool is_shared = (a == p.cap);
  if (!is_shared && a >= cnt) return;
  const int K = is_shared ? p.S : p.I;
  float* xs = smem;
  float* xsum = smem + (size_t)RB * K;
  const MatDev& D = is_shared ? p.sd : p.rd;
  int e = 0, nrows;
  const float* src;
  float* dst;
  if (is_shared) {
    nrows = p.m;
    src = p.act_sh;
    dst = p.ysh;
  } else {
    e = __ldcg(p.active + a);
    const int beg = __ldcg(p.offsets + e);
    nrows = __ldcg(p.offsets + e + 1) - beg;
    src = p.act + (size_t)beg * K;
    dst = p.ypart + (size_t)beg * p.h;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int lg = lane & (kLanesPerRow - 1);
  // each 8-lane group owns two output columns of the tile: col0 and col0 + 32
  const int col0 = tile * kColsPerCta + warp * kRowsPerWarp + (lane >> 3);
  const int col1 = col0 + kRowsPerCta;
  const bool ok0 = col0 < p.h, ok1 = col1 < p.h;
  const int nch = (int)(packed_row_bytes(FMT, K) / 16);
  RowRef A{}, B{};
  if (ok0) A = row_ref<FMT>(D, e, col0);
  B = ok1 ? row_ref<FMT>(D, e, col1) : A;
  for (int rb = 0; rb < nrows; rb += RB) {
    const int nb = min(RB, nrows - rb);
    stage_rows<FMT, false, RB>(xs, xsum, K, nb, [&](int j) {
      return (const uint8_t*)(src + (size_t)(rb + j) * K);
    });
    __syncthreads();
    if (ok0) {
      float a0[RB], a1[RB];
#pragma unroll
      for (int j = 0; j < RB; ++j) a0[j] = a1[j] = 0.f;
      two_row_dots<FMT, RB>(A, B, nch, lg, xs, xsum, K, nb, a0, a1);
#pragma unroll
      for (int j = 0; j < RB; ++j) {
        a0[j] = sum8lanes(a0[j]);
        a1[j] = sum8lanes(a1[j]);
      }
      if (lg == 0) {
#pragma unroll
        for (int j = 0; j < RB; ++j) {
          if (j < nb) {
            dst[(size_t)(rb + j) * p.h + col0] = a0[j] * A.ts;
            if (ok1) dst[(size_t)(rb + j) * p.h + col1] = a1[j] * B.ts;
          }
        }
      }
    }
    __syncthreads();
  }
  // The CTA that completes this column tile last blends it for every row.
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned t = atomicAdd(p.tickets + tile, 1u);
    s_last = (t == (unsigned)(cnt + p.has_shared - 1));
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int cbase = tile * kColsPerCta;
  for (int q = threadIdx.x; q < p.m * kColsPerCta; q += kThreads) {
    const int r = q / kColsPerCta;
    const int col = cbase + (q - r * kColsPerCta);
    if (col >= p.h) continue;
    float acc = 0.f;
    for (int s = 0; s < p.k; ++s) {
      const int pair = r * p.k + s;
      const int pos = __ldcg(p.token_to_perm + pair);
      const float om = p.before_ffn ? 1.f : __ldcg(p.wts + pair);
      acc = fmaf(om, __ldcg(p.ypart + (size_t)pos * p.h + col), acc);
    }
    if (p.has_shared) {
      const float gm = (p.shared_kind == MOE_SHARED_SIGMOID_GATE) ? __ldcg(p.gamma + r) : 1.f;
      acc = fmaf(gm, __ldcg(p.ysh + (size_t)r * p.h + col), acc);
    }
    if (p.out_bf16) {
      reinterpret_cast<__nv_bfloat16*>(p.out)[(size_t)r * p.h + col] = __float2bfloat16_rn(acc);
    } else {
      reinterpret_cast<float*>(p.out)[(size_t)r * p.h + col] = acc;
    }
  }
  if (threadIdx.x == 0) p.tickets[tile] = 0u;
}

}  // namespace moe
