// Dequant-fused expert kernels of the decode MoE layer (CUDA-core GEMV-style tiles).
//
// Every weight row is reduced by one whole warp: lane l takes the row's 16-byte chunks l, l+32,
// l+64, ... in order, decodes each in registers and accumulates in fp32, then a butterfly warp
// sum finishes the row. The same arithmetic runs whether the chunks are streamed from global
// memory (non-allocating 128-bit loads, L2 evict-first) or read with plain loads from a
// shared-memory tile, so both launch paths give identical bits. Activation rows are staged once
// in shared memory as fp32.
//
// gate_up_swiglu_kernel: one CTA = 32 (gate_i, up_i) row pairs of one active expert (or of the
//   shared expert), 4 per warp, for every pair routed to that expert; act[pos, i] = silu(g) * u
//   (or gelu(g) * u) per sorted pair position.
// down_blend_kernel: one CTA = 64 output columns of one active expert's down matrix (or the
//   shared expert's), 8 per warp taken two at a time, for every row that uses it, into per-pair
//   partials; the CTA that completes a column tile last (atomic ticket, no spinning) blends the
//   tile for every row: routed slots in slot order, each times its weight, then gamma times the
//   shared expert.
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
template <> struct Fmt<MOE_FMT_MXFP4> { static constexpr int kElems = 32; };
template <> struct Fmt<MOE_FMT_FP8_E4M3> { static constexpr int kElems = 16; };

__host__ __device__ constexpr size_t packed_row_bytes(int fmt, int k) {
  return fmt == MOE_FMT_F32 ? (size_t)k * 4
         : fmt == MOE_FMT_BF16 ? (size_t)k * 2
         : fmt == MOE_FMT_FP8_E4M3 ? (size_t)k
                                   : (size_t)k / 2;
}

// One decoded 16-byte chunk of a weight row. For the 4-bit affine format the codes are kept as
// f = 1 + q/16 (exact) and the group's scale s and bias b are folded as
//   sum_j (s q_j + b) x_j = 16 s * sum_j f_j x_j + (b - 16 s) * sum_j x_j.
template <int FMT> struct Dec;
template <> struct Dec<MOE_FMT_F32> { float w[4]; };
template <> struct Dec<MOE_FMT_BF16> { float w[8]; };
template <> struct Dec<MOE_FMT_Q4_AFFINE_G64> { float f[32]; float s16, bm; };
template <> struct Dec<MOE_FMT_NVFP4> { float v[32]; float s0, s1; };
template <> struct Dec<MOE_FMT_MXFP4> { float v[32]; float s; };
template <> struct Dec<MOE_FMT_FP8_E4M3> { float w[16]; };

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
  } else if constexpr (FMT == MOE_FMT_MXFP4) {
    r.sc = M.scales + (size_t)e * M.sstride + (size_t)row * (M.k / 32);
  } else if constexpr (FMT == MOE_FMT_FP8_E4M3) {
    r.ts = __ldg(M.tscale + e);
  }
  return r;
}

// One 16-byte chunk of a weight row plus the scale fields it needs, loaded together so a chunk
// costs one memory round trip. aux: Q4 -> fp16 scale (low half) and fp16 bias (high half) of the
// chunk's 64-element group; NVFP4 -> the two E4M3 block scales of its 32 elements.
struct Chunk {
  uint4 w;
  uint32_t aux;
};

__device__ __forceinline__ uint32_t ldg_u16(const void* p) {
  unsigned short v;
  asm volatile("ld.global.nc.L2::cache_hint.u16 %0, [%1], %2;" : "=h"(v) : "l"(p), "l"(l2_evict_first()));
  return v;
}

__device__ __forceinline__ uint32_t ldg_u8(const void* p) {
  unsigned short v;
  asm volatile("ld.global.nc.L2::cache_hint.u8 %0, [%1], %2;" : "=h"(v) : "l"(p), "l"(l2_evict_first()));
  return v & 0xFFu;
}

// SMEM: plain loads (the row may live in shared memory or in L2-resident global memory);
// else streaming non-allocating global loads.
template <int FMT, bool SMEM>
__device__ __forceinline__ Chunk load_chunk(const RowRef& rr, int c) {
  Chunk k;
  k.aux = 0;
  if constexpr (SMEM) {
    k.w = *reinterpret_cast<const uint4*>(rr.w + (size_t)c * 16);
    if constexpr (FMT == MOE_FMT_Q4_AFFINE_G64) {
      k.aux = (uint32_t)(*reinterpret_cast<const unsigned short*>(rr.sc + (size_t)(c >> 1) * 2)) |
              ((uint32_t)(*reinterpret_cast<const unsigned short*>(rr.bi + (size_t)(c >> 1) * 2))
               << 16);
    } else if constexpr (FMT == MOE_FMT_NVFP4) {
      k.aux = *reinterpret_cast<const unsigned short*>(rr.sc + (size_t)c * 2);
    } else if constexpr (FMT == MOE_FMT_MXFP4) {
      k.aux = rr.sc[c];
    }
  } else {
    k.w = ldg_stream(rr.w + (size_t)c * 16);
    if constexpr (FMT == MOE_FMT_Q4_AFFINE_G64) {
      k.aux = ldg_u16(rr.sc + (size_t)(c >> 1) * 2) | (ldg_u16(rr.bi + (size_t)(c >> 1) * 2) << 16);
    } else if constexpr (FMT == MOE_FMT_NVFP4) {
      k.aux = ldg_u16(rr.sc + (size_t)c * 2);
    } else if constexpr (FMT == MOE_FMT_MXFP4) {
      k.aux = ldg_u8(rr.sc + c);
    }
  }
  return k;
}

// 32 E2M1 codes of a chunk (byte j: element 2j in the low nibble, 2j+1 in the high nibble) to
// floats, by the hardware e2m1x2 -> f16x2 conversion.
__device__ __forceinline__ void decode_e2m1x32(const uint32_t (&q)[4], float (&v)[32]) {
#pragma unroll
  for (int t = 0; t < 4; ++t)
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const __half2_raw hr = __nv_cvt_fp4x2_to_halfraw2(
          (__nv_fp4x2_storage_t)((q[t] >> (8 * b)) & 0xFFu), __NV_E2M1);
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
      v[8 * t + 2 * b] = f.x;
      v[8 * t + 2 * b + 1] = f.y;
    }
}

// OCP E8M0 scale byte c -> 2^(c - 127) as a float, built from its bits (c = 0 is the subnormal
// 2^-127; c = 255 is NaN).
__device__ __forceinline__ float e8m0_to_float(uint32_t c) {
  return __uint_as_float(c == 0u ? 0x00400000u : c == 0xFFu ? 0x7FC00000u : (c << 23));
}

template <int FMT>
__device__ __forceinline__ void decode(const Chunk& ch, Dec<FMT>& d) {
  const uint32_t q[4] = {ch.w.x, ch.w.y, ch.w.z, ch.w.w};
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
    const float s = __half2float(__ushort_as_half((unsigned short)(ch.aux & 0xFFFFu)));
    const float b = __half2float(__ushort_as_half((unsigned short)(ch.aux >> 16)));
    d.s16 = 16.f * s;
    d.bm = b - 16.f * s;
  } else if constexpr (FMT == MOE_FMT_MXFP4) {
    decode_e2m1x32(q, d.v);
    d.s = e8m0_to_float(ch.aux & 0xFFu);
  } else if constexpr (FMT == MOE_FMT_FP8_E4M3) {  // byte j is element j
#pragma unroll
    for (int t = 0; t < 4; ++t)
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(
            (__nv_fp8x2_storage_t)((q[t] >> (16 * b)) & 0xFFFFu), __NV_E4M3);
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
        d.w[4 * t + 2 * b] = f.x;
        d.w[4 * t + 2 * b + 1] = f.y;
      }
  } else {  // NVFP4
    decode_e2m1x32(q, d.v);
    const __half2_raw hs =
        __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(ch.aux & 0xFFFFu), __NV_E4M3);
    const float2 sf = __half22float2(*reinterpret_cast<const __half2*>(&hs));
    d.s0 = sf.x;
    d.s1 = sf.y;
  }
}

// Shared-memory layout of staged activation rows. The lanes of a quarter-warp read the
// activations of 8 consecutive weight chunks at once; stored plainly, those reads sit a whole
// chunk apart and pile onto the same banks (8-way for 4-bit chunks of 32 elements). Each row is
// therefore stored as 4-float quads with the quad index XOR-swizzled per chunk, so a
// quarter-warp's reads hit 8 different bank groups. The arithmetic order is unchanged.
template <int FMT>
__device__ __forceinline__ int x_quad(int q) {  // logical quad -> stored quad
  if constexpr (FMT == MOE_FMT_Q4_AFFINE_G64 || FMT == MOE_FMT_NVFP4 || FMT == MOE_FMT_MXFP4) {
    return (q & ~7) | ((q ^ (q >> 3)) & 7);                // 8 quads per chunk
  } else if constexpr (FMT == MOE_FMT_FP8_E4M3) {
    return (q & ~3) | ((q ^ (q >> 3)) & 3);                // 4 quads per chunk
  } else if constexpr (FMT == MOE_FMT_BF16) {
    return (q & ~1) | ((q ^ (q >> 3)) & 1);                // 2 quads per chunk
  } else {
    return q;                                              // 1 quad per chunk
  }
}

template <int FMT>
__device__ __forceinline__ float4 x_load(const float* row, int q) {
  return *reinterpret_cast<const float4*>(row + 4 * x_quad<FMT>(q));
}

// Dot product of decoded chunk c with the staged fp32 activation row `row` (swizzled layout).
// xsum: for Q4, the sum of the chunk's 32 activations.
template <int FMT>
__device__ __forceinline__ float dot(const Dec<FMT>& d, const float* row, int c, float xsum) {
  constexpr int kQ = Fmt<FMT>::kElems / 4;  // quads per chunk
  if constexpr (FMT == MOE_FMT_F32 || FMT == MOE_FMT_BF16 || FMT == MOE_FMT_FP8_E4M3) {
    float a = 0.f;
#pragma unroll
    for (int i = 0; i < kQ; ++i) {
      const float4 x = x_load<FMT>(row, c * kQ + i);
      a = fmaf(d.w[4 * i], x.x, a);
      a = fmaf(d.w[4 * i + 1], x.y, a);
      a = fmaf(d.w[4 * i + 2], x.z, a);
      a = fmaf(d.w[4 * i + 3], x.w, a);
    }
    return a;
  } else if constexpr (FMT == MOE_FMT_Q4_AFFINE_G64) {
    float a = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 x = x_load<FMT>(row, c * 8 + i);
      a = fmaf(d.f[4 * i], x.x, a);
      a = fmaf(d.f[4 * i + 1], x.y, a);
      a = fmaf(d.f[4 * i + 2], x.z, a);
      a = fmaf(d.f[4 * i + 3], x.w, a);
    }
    return fmaf(d.s16, a, d.bm * xsum);
  } else {
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 x = x_load<FMT>(row, c * 8 + i);
      a0 = fmaf(d.v[4 * i], x.x, a0);
      a0 = fmaf(d.v[4 * i + 1], x.y, a0);
      a0 = fmaf(d.v[4 * i + 2], x.z, a0);
      a0 = fmaf(d.v[4 * i + 3], x.w, a0);
    }
#pragma unroll
    for (int i = 4; i < 8; ++i) {
      const float4 x = x_load<FMT>(row, c * 8 + i);
      a1 = fmaf(d.v[4 * i], x.x, a1);
      a1 = fmaf(d.v[4 * i + 1], x.y, a1);
      a1 = fmaf(d.v[4 * i + 2], x.z, a1);
      a1 = fmaf(d.v[4 * i + 3], x.w, a1);
    }
    if constexpr (FMT == MOE_FMT_MXFP4) {
      return (a0 + a1) * d.s;  // one scale for the chunk's 32 elements
    } else {
      return fmaf(d.s0, a0, d.s1 * a1);  // NVFP4: one scale per 16
    }
  }
}

__device__ __forceinline__ float warp_allsum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Staging of nb activation rows of length K as fp32 into shared memory (destination pitch
// `pitch` floats, swizzled for weight format FMT) and, for Q4 weights, the sum of every
// 32-element chunk (pitch / 32 per row). src(j) is the global address of row j (bf16 or fp32).
// Threads t0 .. t0 + nt - 1 take part (nt a multiple of 32). Each thread issues up to four
// 16-byte loads before storing; a chunk's pieces sit in consecutive lanes, so its sum is a fixed
// shuffle tree over per-piece sequential sums (same bits whichever path or thread count stages).
template <int FMT, bool SRC_BF16, typename SrcFn>
__device__ __forceinline__ void stage_rows(float* xs, float* xsum, int K, int pitch, int nb,
                                           SrcFn src, int t0, int nt) {
  constexpr int kPer = SRC_BF16 ? 8 : 4;  // elements per 16-byte piece
  constexpr int kPieces32 = 32 / kPer;    // pieces per 32-element chunk
  const int npieces = K / kPer;
  const int total = nb * npieces;
  const int me = (int)threadIdx.x - t0;
  for (int base = 0; base < total; base += 4 * nt) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int idx = base + u * nt + me;
      if (idx < total) {
        const int j = idx / npieces, c = idx - j * npieces;
        const uint4* g = reinterpret_cast<const uint4*>(src(j)) + c;
        v[u] = SRC_BF16 ? __ldg(g) : __ldcg(g);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int idx = base + u * nt + me;
      const bool live = idx < total;
      const int j = live ? idx / npieces : 0, c = live ? idx - j * npieces : 0;
      float f[kPer];
      if (live) {
        if constexpr (SRC_BF16) {
          f[0] = bf16lo(v[u].x); f[1] = bf16hi(v[u].x); f[2] = bf16lo(v[u].y);
          f[3] = bf16hi(v[u].y); f[4] = bf16lo(v[u].z); f[5] = bf16hi(v[u].z);
          f[6] = bf16lo(v[u].w); f[7] = bf16hi(v[u].w);
        } else {
          f[0] = __uint_as_float(v[u].x); f[1] = __uint_as_float(v[u].y);
          f[2] = __uint_as_float(v[u].z); f[3] = __uint_as_float(v[u].w);
        }
        float* dst = xs + (size_t)j * pitch;
#pragma unroll
        for (int t = 0; t < kPer; t += 4)
          *reinterpret_cast<float4*>(dst + 4 * x_quad<FMT>((c * kPer + t) / 4)) =
              make_float4(f[t], f[t + 1], f[t + 2], f[t + 3]);
      }
      if constexpr (FMT == MOE_FMT_Q4_AFFINE_G64) {
        // the loop bounds are uniform over the participating threads: all lanes shuffle
        float ps = 0.f;
        if (live) {
#pragma unroll
          for (int t = 0; t < kPer; ++t) ps += f[t];
        }
#pragma unroll
        for (int o = 1; o < kPieces32; o <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
        if (live && (c % kPieces32) == 0) xsum[(size_t)j * (pitch / 32) + c / kPieces32] = ps;
      }
    }
  }
}

// Chunks per lane in flight: deep for streamed rows (latency; shallower when a chunk holds 32
// elements or several activation rows make each chunk's arithmetic longer), shallow for plain
// loads of rows already in shared memory or L2 (short latency, and a smaller loop body).
template <int FMT, bool PLAIN, int RB>
constexpr int row_unroll() {
  return PLAIN ? 2 : (FMT == MOE_FMT_BF16 || FMT == MOE_FMT_F32 ? (RB > 1 ? 4 : 8) : (RB > 1 ? 2 : 4));
}

// Two weight rows A and B (same length, nch chunks) against nb <= RB activation rows, by one
// warp: per-lane partial sums in chunk order, then a butterfly sum. xr[j] / xsr[j]: staged row j
// and (Q4) its chunk sums. acc_a / acc_b receive the full dot products (every lane).
template <int FMT, int RB, bool SMEM>
__device__ __forceinline__ void rows2_dot(const RowRef& A, const RowRef& B, int nch,
                                          const float* const (&xr)[RB],
                                          const float* const (&xsr)[RB], int nb,
                                          float (&acc_a)[RB], float (&acc_b)[RB]) {
  constexpr int U = row_unroll<FMT, SMEM, RB>();
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < RB; ++j) acc_a[j] = acc_b[j] = 0.f;
  for (int c0 = lane; c0 < nch; c0 += 32 * U) {
    Chunk ra[U], rb[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + 32 * u;
      if (c < nch) {
        ra[u] = load_chunk<FMT, SMEM>(A, c);
        rb[u] = load_chunk<FMT, SMEM>(B, c);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + 32 * u;
      if (c < nch) {
        Dec<FMT> da, db;
        decode<FMT>(ra[u], da);
        decode<FMT>(rb[u], db);
#pragma unroll
        for (int j = 0; j < RB; ++j) {
          if (j < nb) {
            float s = 0.f;
            if constexpr (FMT == MOE_FMT_Q4_AFFINE_G64) s = xsr[j][c];
            acc_a[j] += dot<FMT>(da, xr[j], c, s);
            acc_b[j] += dot<FMT>(db, xr[j], c, s);
          }
        }
      }
    }
  }
#pragma unroll
  for (int j = 0; j < RB; ++j) {
    acc_a[j] = warp_allsum(acc_a[j]);
    acc_b[j] = warp_allsum(acc_b[j]);
  }
}

// NR weight rows (same length, nch chunks) against nb <= RB activation rows: rows2_dot for any
// number of rows, with the same per-row arithmetic (chunk order per lane, then a butterfly
// sum), so every row's bits match rows2_dot's. With plain loads from shared memory, one chunk
// per row and lane is in flight (NR >= 4) and the activations are re-read per row from shared
// memory; acc[r][j] receives the full dot product of row r with activation row j.
template <int FMT, int RB, bool PLAIN, int NR>
__device__ __forceinline__ void rowsN_dot(const RowRef (&A)[NR], int nch,
                                          const float* const (&xr)[RB],
                                          const float* const (&xsr)[RB], int nb,
                                          float (&acc)[NR][RB]) {
  constexpr int U = PLAIN ? (NR >= 4 ? 1 : 2) : row_unroll<FMT, false, RB>();
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int r = 0; r < NR; ++r)
#pragma unroll
    for (int j = 0; j < RB; ++j) acc[r][j] = 0.f;
  for (int c0 = lane; c0 < nch; c0 += 32 * U) {
    Chunk ch[U][NR];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + 32 * u;
      if (c < nch) {
#pragma unroll
        for (int r = 0; r < NR; ++r) ch[u][r] = load_chunk<FMT, PLAIN>(A[r], c);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + 32 * u;
      if (c < nch) {
#pragma unroll
        for (int r = 0; r < NR; ++r) {
          Dec<FMT> d;
          decode<FMT>(ch[u][r], d);
#pragma unroll
          for (int j = 0; j < RB; ++j) {
            if (j < nb) {
              float sx = 0.f;
              if constexpr (FMT == MOE_FMT_Q4_AFFINE_G64) sx = xsr[j][c];
              acc[r][j] += dot<FMT>(d, xr[j], c, sx);
            }
          }
        }
      }
    }
  }
#pragma unroll
  for (int r = 0; r < NR; ++r)
#pragma unroll
    for (int j = 0; j < RB; ++j) acc[r][j] = warp_allsum(acc[r][j]);
}

// One weight row (same arithmetic per row as rows2_dot).
template <int FMT, int RB, bool SMEM>
__device__ __forceinline__ void rows1_dot(const RowRef& A, int nch,
                                          const float* const (&xr)[RB],
                                          const float* const (&xsr)[RB], int nb,
                                          float (&acc)[RB]) {
  constexpr int U = row_unroll<FMT, SMEM, RB>();
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < RB; ++j) acc[j] = 0.f;
  for (int c0 = lane; c0 < nch; c0 += 32 * U) {
    Chunk ra[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + 32 * u;
      if (c < nch) ra[u] = load_chunk<FMT, SMEM>(A, c);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + 32 * u;
      if (c < nch) {
        Dec<FMT> da;
        decode<FMT>(ra[u], da);
#pragma unroll
        for (int j = 0; j < RB; ++j) {
          if (j < nb) {
            float s = 0.f;
            if constexpr (FMT == MOE_FMT_Q4_AFFINE_G64) s = xsr[j][c];
            acc[j] += dot<FMT>(da, xr[j], c, s);
          }
        }
      }
    }
  }
#pragma unroll
  for (int j = 0; j < RB; ++j) acc[j] = warp_allsum(acc[j]);
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
  const MatDev G = pick_mat(is_shared, p.sg, p.rg);
  const MatDev U = pick_mat(is_shared, p.su, p.ru);
  float* dst;
  if (is_shared) {
    tile = blockIdx.x;
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
    N = p.I;
    dst = p.act;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nch = (int)(packed_row_bytes(FMT, K) / 16);
  const size_t xrow_bytes = (size_t)K * (XBF16 ? 2 : 4);
  const float* xr[RB];
  const float* xsr[RB];
#pragma unroll
  for (int j = 0; j < RB; ++j) {
    xr[j] = xs + (size_t)j * K;
    xsr[j] = xsum + (size_t)j * (K / 32);
  }
  for (int rb = 0; rb < nrows; rb += RB) {
    const int nb = min(RB, nrows - rb);
    stage_rows<FMT, XBF16>(xs, xsum, K, K, nb, [&](int j) {
      const int r = is_shared ? rb + j : __ldcg(p.sorted_pairs + beg + rb + j) / p.k;
      return (const uint8_t*)p.x + (size_t)r * xrow_bytes;
    }, 0, kThreads);
    __syncthreads();
    // warp w takes row pairs tile*32 + w*4 + t; the guard is warp-uniform
    for (int t = 0; t < kRowsPerWarp; ++t) {
      const int i = tile * kRowsPerCta + warp * kRowsPerWarp + t;
      if (i >= N) break;
      const RowRef A = row_ref<FMT>(G, e, i), B = row_ref<FMT>(U, e, i);
      float ag[RB], au[RB];
      rows2_dot<FMT, RB, false>(A, B, nch, xr, xsr, nb, ag, au);
      if (lane < nb) {
        float g = 0.f, u = 0.f;
#pragma unroll
        for (int j = 0; j < RB; ++j)
          if (j == lane) {
            g = ag[j];
            u = au[j];
          }
        g *= A.ts;
        u *= B.ts;
        size_t pos;
        if (is_shared) {
          pos = rb + lane;
        } else {
          pos = beg + rb + lane;
          if (p.before_ffn) {
            const float w = __ldcg(p.wts + __ldcg(p.sorted_pairs + pos));
            g *= w;
            u *= w;
          }
        }
        dst[pos * N + i] = act_mul(p.act_kind, g, u);
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
  const MatDev D = pick_mat(is_shared, p.sd, p.rd);
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
  const int nch = (int)(packed_row_bytes(FMT, K) / 16);
  const float* xr[RB];
  const float* xsr[RB];
#pragma unroll
  for (int j = 0; j < RB; ++j) {
    xr[j] = xs + (size_t)j * K;
    xsr[j] = xsum + (size_t)j * (K / 32);
  }
  constexpr int kColsPerWarp = kColsPerCta / kWarps;  // 8, taken two at a time
  for (int rb = 0; rb < nrows; rb += RB) {
    const int nb = min(RB, nrows - rb);
    stage_rows<FMT, false>(xs, xsum, K, K, nb, [&](int j) {
      return (const uint8_t*)(src + (size_t)(rb + j) * K);
    }, 0, kThreads);
    __syncthreads();
    for (int t = 0; t < kColsPerWarp; t += 2) {
      const int col0 = tile * kColsPerCta + warp * kColsPerWarp + t, col1 = col0 + 1;
      if (col0 >= p.h) break;  // h is a multiple of 8: col1 < h whenever col0 < h
      const RowRef A = row_ref<FMT>(D, e, col0), B = row_ref<FMT>(D, e, col1);
      float a0[RB], a1[RB];
      rows2_dot<FMT, RB, false>(A, B, nch, xr, xsr, nb, a0, a1);
      if (lane < nb) {
        float v0 = 0.f, v1 = 0.f;
#pragma unroll
        for (int j = 0; j < RB; ++j)
          if (j == lane) {
            v0 = a0[j];
            v1 = a1[j];
          }
        dst[(size_t)(rb + lane) * p.h + col0] = v0 * A.ts;
        dst[(size_t)(rb + lane) * p.h + col1] = v1 * B.ts;
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
