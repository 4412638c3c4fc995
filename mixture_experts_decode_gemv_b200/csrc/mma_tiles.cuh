// Tensor-core gate+up tiles for chain calls (m > 4), where several rows share an expert.
//
// At a handful of rows per expert the CUDA-core kernels are bound by instruction issue: every
// decoded weight costs one FMA per activation row. Here one warp computes 16 (gate_i, up_i) row
// pairs for 8 activation rows per m16n8k16 MMA (bf16 operands, fp32 accumulation). Weights of
// the bf16, FP8 E4M3, NVFP4 and MXFP4 formats convert to bf16 exactly (at most 6 significant
// bits after the block scale), and the activation rows are bf16 already, so every product is
// exact and only the order of the fp32 sums differs from the CUDA-core kernels.
//
// Layout trick: the MMA's A fragment gives lane (g, t) the k positions {2t, 2t+1, 2t+8, 2t+9}
// of rows g and g + 8, and the B fragment the same k positions of column g. Any permutation of
// k applied to both operands leaves the product unchanged, so each lane maps k-step s of its
// 16-byte weight chunk (elements 4s .. 4s+3 of the chunk) onto those four positions: a lane
// reads whole 16-byte chunks of its rows (chunk t of every 4-chunk k-tile) and the matching
// 8 .. 64 bytes of each staged activation row, and decodes in registers.
//
// One CTA = 8 warps x 16 row pairs = 128 row pairs of one active expert (or of the shared
// expert); its rows are taken in passes of 8 * NB, staged in shared memory as bf16 rows.
#pragma once

#include <utility>

#include "experts.cuh"

namespace moe {

constexpr int kMmaWarpRows = 16;                           // row pairs per warp
constexpr int kMmaRowsPerCta = kWarps * kMmaWarpRows;      // 128
constexpr int kMmaPitchPad = 64;                           // bytes after each staged row

__host__ __device__ constexpr size_t mma_row_pitch(int K) { return (size_t)K * 2 + kMmaPitchPad; }

// D += A * B for one m16n8k16 tile: bf16 operands, fp32 accumulators.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Elements 4s .. 4s+3 of a decoded chunk as two bf16 pairs: lo = (4s, 4s+1), hi = (4s+2, 4s+3).
template <int FMT, int S>
__device__ __forceinline__ void chunk_pairs(const Chunk& ch, uint32_t& lo, uint32_t& hi) {
  const uint32_t q[4] = {ch.w.x, ch.w.y, ch.w.z, ch.w.w};
  if constexpr (FMT == MOE_FMT_BF16) {  // 8 elements, two per word
    lo = q[2 * S];
    hi = q[2 * S + 1];
  } else if constexpr (FMT == MOE_FMT_FP8_E4M3) {  // 16 elements, four per word
    const uint32_t wd = q[S];
    const __half2_raw h0 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(wd & 0xFFFFu), __NV_E4M3);
    const __half2_raw h1 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(wd >> 16), __NV_E4M3);
    const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&h0));
    const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&h1));
    lo = pack_bf16x2(f0.x, f0.y);
    hi = pack_bf16x2(f1.x, f1.y);
  } else {  // NVFP4 / MXFP4: 32 elements, eight per word, element 2j in the low nibble of byte j
    const uint32_t wd = q[S >> 1] >> (16 * (S & 1));
    const __half2_raw h0 =
        __nv_cvt_fp4x2_to_halfraw2((__nv_fp4x2_storage_t)(wd & 0xFFu), __NV_E2M1);
    const __half2_raw h1 =
        __nv_cvt_fp4x2_to_halfraw2((__nv_fp4x2_storage_t)((wd >> 8) & 0xFFu), __NV_E2M1);
    const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&h0));
    const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&h1));
    float sc;
    if constexpr (FMT == MOE_FMT_MXFP4) {
      sc = e8m0_to_float(ch.aux & 0xFFu);
    } else {  // one E4M3 scale per 16 elements: k-steps 0..3 use the first, 4..7 the second
      const __half2_raw hs =
          __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(ch.aux & 0xFFFFu), __NV_E4M3);
      const float2 sf = __half22float2(*reinterpret_cast<const __half2*>(&hs));
      sc = S < 4 ? sf.x : sf.y;
    }
    lo = pack_bf16x2(f0.x * sc, f0.y * sc);
    hi = pack_bf16x2(f1.x * sc, f1.y * sc);
  }
}

// One k-step (elements 4S .. 4S+3 of each lane's chunks) for the gate and up tiles and every
// block of 8 activation rows. xrow: this lane's staged row g at its first element.
template <int FMT, int NB, int S>
__device__ __forceinline__ void mma_kstep(const Chunk& g0, const Chunk& g1, const Chunk& u0,
                                          const Chunk& u1, const uint8_t* xrow, size_t pitch,
                                          float (&acc_g)[NB][4], float (&acc_u)[NB][4]) {
  uint32_t ga0, ga1, ga2, ga3, ua0, ua1, ua2, ua3;
  chunk_pairs<FMT, S>(g0, ga0, ga2);
  chunk_pairs<FMT, S>(g1, ga1, ga3);
  chunk_pairs<FMT, S>(u0, ua0, ua2);
  chunk_pairs<FMT, S>(u1, ua1, ua3);
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    const uint2 xv =
        *reinterpret_cast<const uint2*>(xrow + (size_t)b * 8 * pitch + (size_t)(4 * S) * 2);
    mma_bf16_16816(acc_g[b], ga0, ga1, ga2, ga3, xv.x, xv.y);
    mma_bf16_16816(acc_u[b], ua0, ua1, ua2, ua3, xv.x, xv.y);
  }
}

template <int FMT, int NB, int... Ss>
__device__ __forceinline__ void mma_ksteps(std::integer_sequence<int, Ss...>, const Chunk& g0,
                                           const Chunk& g1, const Chunk& u0, const Chunk& u1,
                                           const uint8_t* xrow, size_t pitch,
                                           float (&acc_g)[NB][4], float (&acc_u)[NB][4]) {
  (mma_kstep<FMT, NB, Ss>(g0, g1, u0, u1, xrow, pitch, acc_g, acc_u), ...);
}

template <int FMT>
constexpr bool mma_format() {
  return FMT == MOE_FMT_BF16 || FMT == MOE_FMT_FP8_E4M3 || FMT == MOE_FMT_NVFP4 ||
         FMT == MOE_FMT_MXFP4;
}

template <int FMT, int NB>
__global__ void __launch_bounds__(kThreads) gate_up_mma_kernel(const __grid_constant__ Params p) {
  static_assert(mma_format<FMT>(), "bf16, FP8, NVFP4 or MXFP4 weights");
  pdl_launch_dependents();
  extern __shared__ __align__(16) uint8_t xsb[];
  constexpr int kE = Fmt<FMT>::kElems;  // elements per 16-byte chunk
  constexpr int kSteps = kE / 4;        // MMA k-steps per chunk
  constexpr int kTok = 8 * NB;          // activation rows per pass
  const int K = p.h;
  const size_t pitch = mma_row_pitch(K);
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
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int i0 = tile * kMmaRowsPerCta + warp * kMmaWarpRows;  // this warp's first row pair
  const int r0 = min(i0 + g, N - 1), r1 = min(i0 + g + 8, N - 1);  // rows past N: dropped
  const RowRef Ag0 = row_ref<FMT>(G, e, r0), Ag1 = row_ref<FMT>(G, e, r1);
  const RowRef Au0 = row_ref<FMT>(U, e, r0), Au1 = row_ref<FMT>(U, e, r1);
  const int ntile = K / (4 * kE);  // k-tiles of four chunks
  const int xchunks = K / 8;       // 16-byte pieces of a staged bf16 row
  for (int tb = 0; tb < nrows; tb += kTok) {
    const int nt = min(kTok, nrows - tb);
    // stage this pass's activation rows as bf16 (rows past nt are zero)
    for (int idx = threadIdx.x; idx < kTok * xchunks; idx += kThreads) {
      const int j = idx / xchunks, c = idx - j * xchunks;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (j < nt) {
        const int r = is_shared ? tb + j : __ldcg(p.sorted_pairs + beg + tb + j) / p.k;
        v = __ldg(reinterpret_cast<const uint4*>((const uint8_t*)p.x + (size_t)r * K * 2) + c);
      }
      *reinterpret_cast<uint4*>(xsb + (size_t)j * pitch + (size_t)c * 16) = v;
    }
    __syncthreads();
    if (i0 < N) {  // warp-uniform
      float acc_g[NB][4], acc_u[NB][4];
#pragma unroll
      for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc_g[b][q] = acc_u[b][q] = 0.f;
      for (int kt = 0; kt < ntile; kt += 2) {
        Chunk cg0[2], cg1[2], cu0[2], cu1[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          if (kt + u < ntile) {
            const int c = (kt + u) * 4 + t;
            cg0[u] = load_chunk<FMT, false>(Ag0, c);
            cg1[u] = load_chunk<FMT, false>(Ag1, c);
            cu0[u] = load_chunk<FMT, false>(Au0, c);
            cu1[u] = load_chunk<FMT, false>(Au1, c);
          }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          if (kt + u < ntile) {
            const int k_lane = (kt + u) * 4 * kE + kE * t;  // this lane's first element
            mma_ksteps<FMT, NB>(std::make_integer_sequence<int, kSteps>{}, cg0[u], cg1[u],
                                cu0[u], cu1[u], xsb + (size_t)g * pitch + (size_t)k_lane * 2,
                                pitch, acc_g, acc_u);
          }
        }
      }
      // D fragment: [0], [1] = (row g, pass rows 2t, 2t+1); [2], [3] = (row g+8, same rows)
#pragma unroll
      for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int row = i0 + g + (q >= 2 ? 8 : 0);
          const int j = b * 8 + 2 * t + (q & 1);  // row of this pass
          if (row < N && j < nt) {
            float gv = acc_g[b][q] * (q >= 2 ? Ag1.ts : Ag0.ts);
            float uv = acc_u[b][q] * (q >= 2 ? Au1.ts : Au0.ts);
            size_t pos;
            if (is_shared) {
              pos = tb + j;
            } else {
              pos = beg + tb + j;
              if (p.before_ffn) {
                const float w = __ldcg(p.wts + __ldcg(p.sorted_pairs + pos));
                gv *= w;
                uv *= w;
              }
            }
            dst[pos * N + row] = act_mul(p.act_kind, gv, uv);
          }
        }
    }
    __syncthreads();
  }
}

}  // namespace moe
