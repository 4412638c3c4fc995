// Tensor-core decode path for bf16, FP8 E4M3, NVFP4, MXFP4 and 4-bit affine experts.
//
// Every expert projection is a product of a weight matrix W [N, K] (streamed from HBM once per
// call) with a handful of activation columns (the rows routed to that expert). A warp takes a
// "job" of 32 weight rows (two m16 tiles: for gate/up the 16 gate rows and the 16 up rows of the
// same outputs, for down 32 consecutive output columns) and multiplies it with all of the job's
// activation columns, 8 per n-tile, on mma.sync.m16n8k16 with fp32 accumulation. The weights are
// decoded in registers into the tensor-core operand type: bf16 weights stay bf16 (activations
// bf16), the other formats become fp16 exactly (E4M3 codes; E2M1 codes times their E4M3 block
// scale, at most 6 significant bits; 1 + q/16 for the 4-bit affine codes), against fp16
// activations. Every product is therefore exact and only the order of the fp32 sums is chosen
// here.
//
// Lane layout. The MMA gives lane (g = lane/4, t = lane%4) the k positions {2t, 2t+1, 2t+8,
// 2t+9} of rows g and g+8 (A) and of column g (B). A permutation of k applied to both operands
// leaves the product unchanged, so lane t reads, per "k-tile" of a row, its own contiguous
// BPL-byte piece (piece t of four) and maps each k-step's four elements onto those positions:
//   bf16   16 B = 8 elements,  2 k-steps: pairs (4s, 4s+1), (4s+2, 4s+3)
//   FP8    16 B = 16 elements, 4 k-steps: same pairing
//   NVFP4  16 B = 32 elements, 8 k-steps: same pairing; each pair times its E4M3 block scale
//   MXFP4   4 B = 8 elements,  2 k-steps: same pairing; the k-tile is one 32-element E8M0 block
//   Q4      8 B = 16 elements, 4 k-steps: pairs (s, s+4) and (8+s, 12+s) of the lane's 16 (two
//          shifts and a mask build 1 + q/16 for two nibbles of one word); the k-tile is one
//          64-element scale group
// The activation operand (x for gate/up, the act rows for down) is stored by this library in
// the same element order (plain order, except a 4x4 transpose inside every 16 elements for Q4),
// so each B fragment is one 8-byte load.
//
// Canonical arithmetic (the same for every m, every launch path and every work split): K is cut
// into chunks of eight k-tiles (chunk_elems). A chunk's value is the MMA chain over its k-steps starting from
// zero; for MXFP4 and Q4 every k-tile is its own chain from zero and is scaled into the chunk:
//   MXFP4: chunk = fma(2^e, D_tile, chunk)
//   Q4:    chunk = fma(16 s, D_tile, chunk); chunk = fma(b - 16 s, D_ones, chunk)
// (D_ones = the same chain with all-ones weights = the sum of the group's activations; this is
// w = s q + b = 16 s (1 + q/16) + (b - 16 s)). The result is the fp32 sum of the chunks in
// order, times the per-matrix tensor scale (NVFP4, FP8). The activations of the down projection
// are fp32; they enter as a pair hi + lo (hi = the operand type's rounding, lo = the rounding of
// the remainder), two MMAs per k-step, so the act values reach the product to ~2^-22.
//
// Work split: a job's chunks may be shared by several warps ("pieces"): each then stores its
// chunk values, and the warp that completes the job (an atomic ticket) sums them in order. A
// warp that owns a whole job sums in registers in the same order. So the bits do not depend on
// the split, and a row's bits do not depend on m.
#pragma once

#include <cuda_fp16.h>

#include "fused.cuh"
#include "router.cuh"

namespace moe {
namespace tc {

// Elements of K per canonical chunk: eight k-tiles of the format (256 bf16, 512 FP8, 1024 NVFP4,
// 256 MXFP4, 512 Q4 elements), so a chunk costs about the same instructions in every format and a
// one-row call has as many chunk-sized pieces to spread over the warps as the shapes allow.
// Fixed per format, whatever m.
__host__ __device__ constexpr int chunk_elems(int fmt) {
  return fmt == MOE_FMT_BF16 ? 256
         : fmt == MOE_FMT_FP8_E4M3 ? 512
         : fmt == MOE_FMT_NVFP4 ? 1024
         : fmt == MOE_FMT_MXFP4 ? 256
                                : 512;
}
constexpr int kJobRows = 32;   // weight rows per job (two m16 tiles)
constexpr int kMaxWarps = 16;   // warps per CTA of a tensor-core kernel: 16 or 8 (below)
constexpr int kMaxPairs = MOE_MAX_ROWS * MOE_MAX_TOP_K;  // 512
constexpr unsigned kOnes = 0x3C003C00u;  // fp16 pair (1, 1)

template <int FMT> struct Traits;
// BPL: bytes of a row a lane loads per k-tile; EPL: elements in them; KS: k-steps per k-tile;
// U: k-tiles per load batch; F16: fp16 operands (else bf16); POST: per-k-tile scale after the MMA
template <> struct Traits<MOE_FMT_BF16> {
  static constexpr int BPL = 16, EPL = 8, KS = 2, U = 4;
  static constexpr bool F16 = false, POST = false, PERM = false;
};
template <> struct Traits<MOE_FMT_FP8_E4M3> {
  static constexpr int BPL = 16, EPL = 16, KS = 4, U = 4;
  static constexpr bool F16 = true, POST = false, PERM = false;
};
template <> struct Traits<MOE_FMT_NVFP4> {
  static constexpr int BPL = 16, EPL = 32, KS = 8, U = 2;
  static constexpr bool F16 = true, POST = false, PERM = false;
};
template <> struct Traits<MOE_FMT_MXFP4> {
  static constexpr int BPL = 4, EPL = 8, KS = 2, U = 8;
  static constexpr bool F16 = true, POST = true, PERM = false;
};
template <> struct Traits<MOE_FMT_Q4_AFFINE_G64> {
  static constexpr int BPL = 8, EPL = 16, KS = 4, U = 4;
  static constexpr bool F16 = true, POST = true, PERM = true;
};

// K-tiles per load batch: as many as the format's U while the batch's raw weight words and
// activation fragments stay within about 112 registers (rounded down to a power of two).
template <int FMT, int NTG, bool HILO>
constexpr int batch_tiles() {
  using Tr = Traits<FMT>;
  constexpr bool has_s = FMT == MOE_FMT_NVFP4 || FMT == MOE_FMT_MXFP4 || FMT == MOE_FMT_Q4_AFFINE_G64;
  constexpr int per_kt = 4 * (Tr::BPL / 4 + (has_s ? 1 : 0)) + 2 * Tr::KS * NTG * (HILO ? 2 : 1);
  constexpr int fit = 112 / per_kt > 0 ? 112 / per_kt : 1;
  constexpr int cap = fit < Tr::U ? fit : Tr::U;
  return cap >= 8 ? 8 : cap >= 4 ? 4 : cap >= 2 ? 2 : 1;
}

template <int FMT>
constexpr bool tc_format() {
  return FMT == MOE_FMT_BF16 || FMT == MOE_FMT_FP8_E4M3 || FMT == MOE_FMT_NVFP4 ||
         FMT == MOE_FMT_MXFP4 || FMT == MOE_FMT_Q4_AFFINE_G64;
}

__host__ __device__ constexpr int ceil_div(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ constexpr int n_chunks(int K, int fmt) { return ceil_div(K, chunk_elems(fmt)); }

// Position of element i of a row in this library's stored activation order (Q4: a 4x4 transpose
// inside every 16 elements, so a lane's k-step reads 4 consecutive stored elements).
template <int FMT>
__host__ __device__ __forceinline__ int act_pos(int i) {
  if constexpr (Traits<FMT>::PERM) return (i & ~15) | ((i & 3) << 2) | ((i >> 2) & 3);
  return i;
}

// ---- operand helpers ---------------------------------------------------------------------------

__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                        uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
template <bool F16>
__device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                    uint32_t b1) {
  if constexpr (F16) {
    mma_f16(d, a, b0, b1);
  } else {
    mma_bf16(d, a, b0, b1);
  }
}

// Four E2M1 pairs (the 4 bytes of w; low nibble = lower element) to four fp16 pairs.
__device__ __forceinline__ void e2m1x8_f16(uint32_t w, uint32_t (&h)[4]) {
  asm("{\n .reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %4;\n"
      " cvt.rn.f16x2.e2m1x2 %0, b0;\n cvt.rn.f16x2.e2m1x2 %1, b1;\n"
      " cvt.rn.f16x2.e2m1x2 %2, b2;\n cvt.rn.f16x2.e2m1x2 %3, b3;\n}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
      : "r"(w));
}
// Two E4M3 pairs (the 4 bytes of w; low byte = lower element) to two fp16 pairs.
__device__ __forceinline__ void e4m3x4_f16(uint32_t w, uint32_t (&h)[2]) {
  asm("{\n .reg .b16 l, u;\n mov.b32 {l, u}, %2;\n cvt.rn.f16x2.e4m3x2 %0, l;\n"
      " cvt.rn.f16x2.e4m3x2 %1, u;\n}"
      : "=r"(h[0]), "=r"(h[1])
      : "r"(w));
}
__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
// Nibbles j and j + 4 of w as the fp16 pair (1 + q_j/16, 1 + q_{j+4}/16), exact.
template <int J>
__device__ __forceinline__ uint32_t q4_pair(uint32_t w) {
  const uint32_t v = J < 2 ? (w << (6 - 4 * J)) : (w >> (4 * J - 6));
  return (v & 0x03C003C0u) | 0x3C003C00u;
}

__device__ __forceinline__ uint4 ld_w16(const uint8_t* p) { return ldg_stream(p); }
__device__ __forceinline__ uint2 ld_w8(const uint8_t* p) {
  uint2 r;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v2.u32 {%0,%1}, [%2], %3;"
               : "=r"(r.x), "=r"(r.y)
               : "l"(p), "l"(l2_evict_first()));
  return r;
}
__device__ __forceinline__ uint32_t ld_w4(const uint8_t* p) {
  uint32_t r;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.u32 %0, [%1], %2;"
               : "=r"(r)
               : "l"(p), "l"(l2_evict_first()));
  return r;
}
// Scale bytes are read once per call too, but they share L2 lines with neighbouring rows'
// scales; plain non-coherent loads.
__device__ __forceinline__ uint32_t ld_u16(const uint8_t* p) {
  return (uint32_t)__ldg(reinterpret_cast<const unsigned short*>(p));
}
__device__ __forceinline__ uint32_t ld_u8(const uint8_t* p) { return (uint32_t)__ldg(p); }
// Activation operand: written by this library earlier in the call (possibly by other CTAs), so
// always through L2.
__device__ __forceinline__ uint2 ld_act8(const uint8_t* p) {
  return __ldcg(reinterpret_cast<const uint2*>(p));
}

// One lane's view of a job's 32 weight rows: rows g and g + 8 of each m16 tile
// (r = 0: tile 0 row g, 1: tile 0 row g + 8, 2: tile 1 row g, 3: tile 1 row g + 8).
struct JobRows {
  const uint8_t* w[4];   // packed row, nullptr when the row is past the matrix
  const uint8_t* sc[4];  // scale row (NVFP4, MXFP4, Q4)
  const uint8_t* bi[4];  // bias row (Q4)
  int sc_len;            // bytes of one scale (and bias) row
};

// The activation columns of one column group, for this lane (column g of each n-tile): the
// stored activation row, nullptr past the columns. Gate/up rows hold operand-type elements;
// down rows hold every 4 elements as 4 hi halves followed by their 4 lo halves (16 bytes).
template <int NTG>
struct JobCols {
  const uint8_t* row[NTG];
};

template <int FMT>
__device__ __forceinline__ JobRows job_rows(const MatDev& M, int e, int row0, int row1,
                                            int lane) {
  // row0 / row1: first weight row of m16 tile 0 / 1
  JobRows R;
  const int g = lane >> 2;
  const int rows[4] = {row0 + g, row0 + g + 8, row1 + g, row1 + g + 8};
  const size_t prb = packed_row_bytes(FMT, M.k);
  R.sc_len = FMT == MOE_FMT_NVFP4 ? M.k / 16 : FMT == MOE_FMT_MXFP4 ? M.k / 32
             : FMT == MOE_FMT_Q4_AFFINE_G64 ? (M.k / 64) * 2 : 0;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const bool live = rows[r] < M.n;
    R.w[r] = live ? M.packed + (size_t)e * M.estride + (size_t)rows[r] * prb : nullptr;
    R.sc[r] = nullptr;
    R.bi[r] = nullptr;
    if (live) {
      if constexpr (FMT == MOE_FMT_NVFP4) {
        R.sc[r] = M.scales + (size_t)e * M.sstride + (size_t)rows[r] * (M.k / 16);
      } else if constexpr (FMT == MOE_FMT_MXFP4) {
        R.sc[r] = M.scales + (size_t)e * M.sstride + (size_t)rows[r] * (M.k / 32);
      } else if constexpr (FMT == MOE_FMT_Q4_AFFINE_G64) {
        R.sc[r] = M.scales + (size_t)e * M.sstride + (size_t)rows[r] * (M.k / 64) * 2;
        R.bi[r] = M.biases + (size_t)e * M.sstride + (size_t)rows[r] * (M.k / 64) * 2;
      }
    }
  }
  return R;
}

// Raw data of one row for one k-tile (BPL bytes) and its scale word.
template <int FMT>
struct RawTile {
  uint32_t w[Traits<FMT>::BPL / 4];
  uint32_t s;  // NVFP4: two E4M3 block scales; MXFP4: E8M0 byte; Q4: fp16 scale | fp16 bias << 16
};

template <int FMT>
__device__ __forceinline__ void load_tile(const JobRows& R, int r, int kt, int t, bool in_k,
                                          RawTile<FMT>& x) {
  using Tr = Traits<FMT>;
  const uint8_t* base = R.w[r];
#pragma unroll
  for (int i = 0; i < Tr::BPL / 4; ++i) x.w[i] = 0u;
  x.s = 0u;
  if (base == nullptr || !in_k) return;
  const uint8_t* p = base + (size_t)kt * (4 * Tr::BPL) + t * Tr::BPL;
  if constexpr (Tr::BPL == 16) {
    const uint4 v = ld_w16(p);
    x.w[0] = v.x;
    x.w[1] = v.y;
    x.w[2] = v.z;
    x.w[3] = v.w;
  } else if constexpr (Tr::BPL == 8) {
    const uint2 v = ld_w8(p);
    x.w[0] = v.x;
    x.w[1] = v.y;
  } else {
    x.w[0] = ld_w4(p);
  }
  if constexpr (FMT == MOE_FMT_NVFP4) {
    x.s = ld_u16(R.sc[r] + (size_t)kt * 8 + 2 * t);
  } else if constexpr (FMT == MOE_FMT_MXFP4) {
    x.s = ld_u8(R.sc[r] + kt);
  } else if constexpr (FMT == MOE_FMT_Q4_AFFINE_G64) {
    x.s = ld_u16(R.sc[r] + (size_t)kt * 2) | (ld_u16(R.bi[r] + (size_t)kt * 2) << 16);
  }
}

// NVFP4: the two block scales of a lane's 32 elements as broadcast fp16 pairs (s0, s0) and
// (s1, s1); elements 0..15 use the first, 16..31 the second.
__device__ __forceinline__ void nvfp4_scale_pairs(uint32_t s, uint32_t& s0, uint32_t& s1) {
  uint32_t sc[2];
  e4m3x4_f16(s, sc);
  s0 = __byte_perm(sc[0], 0u, 0x1010);
  s1 = __byte_perm(sc[0], 0u, 0x3232);
}

// The A-operand pairs of k-steps 2W and 2W+1 of a row's raw k-tile: p[step][0] holds k positions
// (2t, 2t+1), p[step][1] positions (2t+8, 2t+9). sp: NVFP4 scale pairs of the row.
template <int FMT, int W>
__device__ __forceinline__ void a_pairs2(const RawTile<FMT>& x, uint32_t s0, uint32_t s1,
                                         uint32_t (&p)[2][2]) {
  if constexpr (FMT == MOE_FMT_BF16) {  // elements 4s .. 4s+3 are words 2s, 2s+1
    p[0][0] = x.w[4 * W];
    p[0][1] = x.w[4 * W + 1];
    p[1][0] = x.w[4 * W + 2];
    p[1][1] = x.w[4 * W + 3];
  } else if constexpr (FMT == MOE_FMT_FP8_E4M3) {  // k-step s: word s
    uint32_t h[2];
    e4m3x4_f16(x.w[2 * W], h);
    p[0][0] = h[0];
    p[0][1] = h[1];
    e4m3x4_f16(x.w[2 * W + 1], h);
    p[1][0] = h[0];
    p[1][1] = h[1];
  } else if constexpr (FMT == MOE_FMT_NVFP4 || FMT == MOE_FMT_MXFP4) {  // k-steps 2W, 2W+1: word W
    uint32_t h[4];
    e2m1x8_f16(x.w[W], h);
    if constexpr (FMT == MOE_FMT_NVFP4) {
      const uint32_t sc = W < 2 ? s0 : s1;
#pragma unroll
      for (int i = 0; i < 4; ++i) h[i] = hmul2(h[i], sc);
    }
    p[0][0] = h[0];
    p[0][1] = h[1];
    p[1][0] = h[2];
    p[1][1] = h[3];
  } else {  // Q4: word 0 holds elements 0..7 of the lane's 16, word 1 elements 8..15
    p[0][0] = q4_pair<2 * W>(x.w[0]);
    p[0][1] = q4_pair<2 * W>(x.w[1]);
    p[1][0] = q4_pair<2 * W + 1>(x.w[0]);
    p[1][1] = q4_pair<2 * W + 1>(x.w[1]);
  }
}

// Per-k-tile scale factors of the POST formats for one row.
template <int FMT>
__device__ __forceinline__ void post_scales(const RawTile<FMT>& x, float& mul, float& add) {
  if constexpr (FMT == MOE_FMT_MXFP4) {
    mul = e8m0_to_float(x.s & 0xFFu);
    add = 0.f;
  } else if constexpr (FMT == MOE_FMT_Q4_AFFINE_G64) {
    const float s = __half2float(__ushort_as_half((unsigned short)(x.s & 0xFFFFu)));
    const float b = __half2float(__ushort_as_half((unsigned short)(x.s >> 16)));
    mul = 16.f * s;
    add = b - 16.f * s;
  } else {
    mul = 1.f;
    add = 0.f;
  }
}

// K-steps 2W and 2W+1 for both m16 tiles and every n-tile.
template <int FMT, int NTG, bool HILO, int W>
__device__ __forceinline__ void kstep2(const RawTile<FMT> (&x)[4], const uint32_t (&s0)[4],
                                       const uint32_t (&s1)[4],
                                       const uint2 (&bh)[Traits<FMT>::KS][NTG],
                                       const uint2 (&bl)[Traits<FMT>::KS][NTG],
                                       float (&d)[2][NTG][4], float (&d1)[NTG][4]) {
  constexpr bool F16 = Traits<FMT>::F16;
  uint32_t pr[4][2][2];
#pragma unroll
  for (int r = 0; r < 4; ++r) a_pairs2<FMT, W>(x[r], s0[r], s1[r], pr[r]);
#pragma unroll
  for (int st = 0; st < 2; ++st) {
    const int S = 2 * W + st;
    // tile 0 = raw rows 0 (row g) and 1 (row g + 8); tile 1 = raw rows 2 and 3
    const uint32_t a0[4] = {pr[0][st][0], pr[1][st][0], pr[0][st][1], pr[1][st][1]};
    const uint32_t a1[4] = {pr[2][st][0], pr[3][st][0], pr[2][st][1], pr[3][st][1]};
#pragma unroll
    for (int n = 0; n < NTG; ++n) {
      mma<F16>(d[0][n], a0, bh[S][n].x, bh[S][n].y);
      mma<F16>(d[1][n], a1, bh[S][n].x, bh[S][n].y);
      if constexpr (HILO) {
        mma<F16>(d[0][n], a0, bl[S][n].x, bl[S][n].y);
        mma<F16>(d[1][n], a1, bl[S][n].x, bl[S][n].y);
      }
      if constexpr (FMT == MOE_FMT_Q4_AFFINE_G64) {
        const uint32_t ones[4] = {kOnes, kOnes, kOnes, kOnes};
        mma<F16>(d1[n], ones, bh[S][n].x, bh[S][n].y);
        if constexpr (HILO) mma<F16>(d1[n], ones, bl[S][n].x, bl[S][n].y);
      }
    }
  }
}

template <int FMT, int NTG, bool HILO, int... Ws>
__device__ __forceinline__ void ksteps(std::integer_sequence<int, Ws...>,
                                       const RawTile<FMT> (&x)[4],
                                       const uint2 (&bh)[Traits<FMT>::KS][NTG],
                                       const uint2 (&bl)[Traits<FMT>::KS][NTG],
                                       float (&d)[2][NTG][4], float (&d1)[NTG][4]) {
  uint32_t s0[4] = {0u, 0u, 0u, 0u}, s1[4] = {0u, 0u, 0u, 0u};
  if constexpr (FMT == MOE_FMT_NVFP4) {
#pragma unroll
    for (int r = 0; r < 4; ++r) nvfp4_scale_pairs(x[r].s, s0[r], s1[r]);
  }
  (kstep2<FMT, NTG, HILO, Ws>(x, s0, s1, bh, bl, d, d1), ...);
}

template <int NTG>
__device__ __forceinline__ void zero(float (&a)[2][NTG][4]) {
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int n = 0; n < NTG; ++n)
#pragma unroll
      for (int q = 0; q < 4; ++q) a[m][n][q] = 0.f;
}

// Where the chunk values of a split job go: value (chunk c, activation column col, weight row r
// of the job's 32) at base + col * col_stride + c * 32 + r, for the job's n live columns.
struct SlotMap {
  float* base;     // nullptr: the warp owns the whole job (no stored values)
  int col_stride;  // floats from one column to the next
  int n;           // live columns of the job
  int col0;        // first column of this column group
};

// ---- the per-warp shared-memory ring ---------------------------------------------------------
//
// Every lane streams its own operand pieces into the warp's ring with cp.async and later reads
// back exactly the bytes it copied, so a per-thread cp.async.wait_group is the only
// synchronisation. A stage holds U k-tiles: the weight pieces [u][row][lane] (BPL bytes each),
// the scale words [u][row][word][lane] (the 4-byte aligned word holding the lane's scale bytes),
// and the activation pieces [u][k-step pair (HILO: k-step)][live column][t] (16 bytes each) of
// the lane's live columns only. 2 to 8 stages, as many as the job's live columns leave room for.
constexpr int kRingCtaBytes = 192 * 1024;  // dynamic shared memory per CTA: the warps' rings

// Weight pieces: evict-first in L2, and a 256-byte L2 fetch on a miss, so the k-tiles that
// follow along the same row (64 bytes each for bf16) find their bytes in L2.
__device__ __forceinline__ void cp16_ef(uint32_t dst, const void* src, int n, uint64_t pol) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint.L2::256B [%0], [%1], 16, %2, %3;" ::"r"(dst),
               "l"(src), "r"(n), "l"(pol)
               : "memory");
}
__device__ __forceinline__ void cp8_ef(uint32_t dst, const void* src, int n, uint64_t pol) {
  asm volatile("cp.async.ca.shared.global.L2::cache_hint [%0], [%1], 8, %2, %3;" ::"r"(dst),
               "l"(src), "r"(n), "l"(pol)
               : "memory");
}
__device__ __forceinline__ void cp4_ef(uint32_t dst, const void* src, int n, uint64_t pol) {
  asm volatile("cp.async.ca.shared.global.L2::cache_hint [%0], [%1], 4, %2, %3;" ::"r"(dst),
               "l"(src), "r"(n), "l"(pol)
               : "memory");
}
// Activation pieces: written earlier in this call, so through L2 only (.cg).
__device__ __forceinline__ void cp16(uint32_t dst, const void* src, int n) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp4(uint32_t dst, const void* src, int n) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// cp_wait with a count known only at run time (1..7; warp-uniform)
__device__ __forceinline__ void cp_wait_n(int n) {
  switch (n) {
    case 1: cp_wait<1>(); break;
    case 2: cp_wait<2>(); break;
    case 3: cp_wait<3>(); break;
    case 4: cp_wait<4>(); break;
    case 5: cp_wait<5>(); break;
    case 6: cp_wait<6>(); break;
    default: cp_wait<7>(); break;
  }
}

template <int FMT>
constexpr int scale_words() {  // aligned scale words per (row, k-tile)
  return FMT == MOE_FMT_Q4_AFFINE_G64 ? 2 : (FMT == MOE_FMT_NVFP4 || FMT == MOE_FMT_MXFP4) ? 1 : 0;
}

// Ring bytes one k-tile takes with `cols` live activation columns.
template <int FMT, bool HILO>
__host__ __device__ constexpr int ring_per_kt(int cols) {
  return 128 * Traits<FMT>::BPL + 128 * 4 * scale_words<FMT>() +
         (HILO ? Traits<FMT>::KS : Traits<FMT>::KS / 2) * cols * 64;
}

// Warps per CTA: 16 when each warp's share of the ring still holds two stages of a k-tile with
// every column live (and one column group is 8 wide), else 8. More warps hide more latency.
template <int FMT, int NTG>
__host__ __device__ constexpr int tc_warps() {
  return NTG == 1 && 2 * ring_per_kt<FMT, true>(8) <= kRingCtaBytes / 16 ? 16 : 8;
}
template <int FMT, int NTG>
__host__ __device__ constexpr int ring_bytes() {
  return kRingCtaBytes / tc_warps<FMT, NTG>();
}

// k-tiles with every column of the group live that a warp's ring holds (at least 2 are needed).
template <int FMT, int NTG, bool HILO>
constexpr int ring_stages() {
  return ring_bytes<FMT, NTG>() / ring_per_kt<FMT, HILO>(8 * NTG);
}

// Address of the scale bytes a lane needs for row r, k-tile kt (word w: Q4 0 = scale, 1 = bias).
template <int FMT>
__device__ __forceinline__ const uint8_t* scale_addr(const JobRows& R, int r, int kt, int t,
                                                     int w) {
  if constexpr (FMT == MOE_FMT_NVFP4) return R.sc[r] + (size_t)kt * 8 + 2 * t;
  if constexpr (FMT == MOE_FMT_MXFP4) return R.sc[r] + kt;
  return (w == 0 ? R.sc[r] : R.bi[r]) + (size_t)kt * 2;
}

// Chunks [c0, c1) of a job (elements [c0 * chunk, min(c1 * chunk, K))). With sm.base null the
// chunk values are added to acc in order (the warp owns the whole job); otherwise each chunk's
// values are stored where sm says. ring: this warp's share of the CTA's ring memory.
template <int FMT, int NTG, bool HILO>
__device__ void run_chunks(const JobRows& R, const JobCols<NTG>& C, int ncols, int K, int c0,
                           int c1, float (&acc)[2][NTG][4], const SlotMap& sm, uint8_t* ring,
                           const void* dummy) {
  using Tr = Traits<FMT>;
  constexpr int KT = 4 * Tr::EPL;            // elements per k-tile
  constexpr int TPC = chunk_elems(FMT) / KT;  // k-tiles per chunk
  constexpr int SW = scale_words<FMT>();
  constexpr int KSB = HILO ? Tr::KS : Tr::KS / 2;  // 16-byte activation pieces per k-tile
  constexpr int kRing = ring_bytes<FMT, NTG>();
  static_assert(ring_stages<FMT, NTG, HILO>() >= 2, "the ring must hold two widest k-tiles");
  const int lane = threadIdx.x & 31, t = lane & 3, g = lane >> 2;
  const int nkt = ceil_div(K, KT);
  const int kt_begin = c0 * TPC, kt_end = min(nkt, c1 * TPC);
  // stage layout for this piece (ncols = live columns of this column group, <= 8 * NTG): U
  // k-tiles of per_kt bytes per stage, U as large as keeps at least four stages (at most 8
  // k-tiles), then as many stages as the ring holds (2 to 8): the fewer live columns, the more
  // weight bytes in flight
  const int a_bytes = 128 * Tr::BPL, s_bytes = 128 * 4 * SW, b_bytes = KSB * ncols * 64;
  const int per_kt = a_bytes + s_bytes + b_bytes;
  if (ncols < 1 || ncols > 8 * NTG || 2 * per_kt > kRing) return;  // unreachable by design
  int U = kRing / (4 * per_kt);
  U = U < 1 ? 1 : U > 8 ? 8 : U;
  int S = kRing / (U * per_kt);
  S = S > 8 ? 8 : S;
  const int SB = U * per_kt;  // a multiple of 16 bytes
  const int s_off = U * a_bytes, b_off = U * (a_bytes + s_bytes);
  const int nb = ceil_div(kt_end - kt_begin, U);
  const uint32_t ring_s = (uint32_t)__cvta_generic_to_shared(ring);
  const uint64_t pol = l2_evict_first();
  int cidx[NTG];  // compact index of this lane's column in each n-tile, -1 if not live
#pragma unroll
  for (int q = 0; q < NTG; ++q) cidx[q] = (C.row[q] != nullptr) ? 8 * q + g : -1;

  auto issue = [&](int b, int stage) {
    const uint32_t st = ring_s + (uint32_t)(stage * SB);
    for (int u = 0; u < U; ++u) {
      const int kt = kt_begin + b * U + u;
      if (kt >= kt_end) break;
      const int e0 = kt * KT + t * Tr::EPL;
      const bool in_k = e0 < K;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const bool live = in_k && R.w[r] != nullptr;
        const uint8_t* src = live ? R.w[r] + (size_t)kt * (4 * Tr::BPL) + t * Tr::BPL
                                  : (const uint8_t*)dummy;
        const uint32_t dst = st + (uint32_t)(((u * 4 + r) * 32 + lane) * Tr::BPL);
        if constexpr (Tr::BPL == 16) {
          cp16_ef(dst, src, live ? 16 : 0, pol);
        } else if constexpr (Tr::BPL == 8) {
          cp8_ef(dst, src, live ? 8 : 0, pol);
        } else {
          cp4_ef(dst, src, live ? 4 : 0, pol);
        }
        if constexpr (SW > 0) {
#pragma unroll
          for (int w = 0; w < SW; ++w) {
            const uint32_t sdst = st + (uint32_t)(s_off + (((u * 4 + r) * SW + w) * 32 + lane) * 4);
            int n = 0;
            const uint8_t* ws = (const uint8_t*)dummy;
            if (live) {
              const uint8_t* a = scale_addr<FMT>(R, r, kt, t, w);
              const uint8_t* row_end = (w == 0 ? R.sc[r] : R.bi[r]) + R.sc_len;
              ws = (const uint8_t*)((uintptr_t)a & ~(uintptr_t)3);
              n = (int)(row_end - ws) < 4 ? (int)(row_end - ws) : 4;
            }
            cp4_ef(sdst, ws, n, pol);
          }
        }
      }
      if (in_k) {
#pragma unroll
        for (int q = 0; q < NTG; ++q) {
          if (cidx[q] < 0) continue;
#pragma unroll
          for (int kb = 0; kb < KSB; ++kb) {
            const size_t off = HILO ? (size_t)(e0 + 4 * kb) * 4 : (size_t)(e0 + 8 * kb) * 2;
            const uint32_t bdst =
                st + (uint32_t)(b_off + (((u * KSB + kb) * ncols + cidx[q]) * 4 + t) * 16);
            cp16(bdst, C.row[q] + off, 16);
          }
        }
      }
    }
  };

  float p[2][NTG][4];   // the current chunk's value (POST formats)
  float d[2][NTG][4];   // the running MMA chain (a k-tile's for POST formats)
  float d1[NTG][4];     // Q4: the all-ones chain
  zero<NTG>(p);
  zero<NTG>(d);
  for (int s = 0; s < S - 1; ++s) {
    if (s < nb) issue(s, s);
    cp_commit();
  }
  int rd = 0, wr = S - 1;  // stages of batch b and of batch b + S - 1
  for (int b = 0; b < nb; ++b) {
    if (b + S - 1 < nb) issue(b + S - 1, wr);
    wr = wr + 1 == S ? 0 : wr + 1;
    cp_commit();
    cp_wait_n(S - 1);  // this lane's copies of batch b have landed
    const uint8_t* st = ring + rd * SB;
    rd = rd + 1 == S ? 0 : rd + 1;
    for (int u = 0; u < U; ++u) {
      const int kt = kt_begin + b * U + u;
      if (kt >= kt_end) break;  // warp-uniform
      const int e0 = kt * KT + t * Tr::EPL;
      const bool in_k = e0 < K;
      RawTile<FMT> x[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const uint8_t* src = st + ((u * 4 + r) * 32 + lane) * Tr::BPL;
        if constexpr (Tr::BPL == 16) {
          const uint4 v = *reinterpret_cast<const uint4*>(src);
          x[r].w[0] = v.x;
          x[r].w[1] = v.y;
          x[r].w[2] = v.z;
          x[r].w[3] = v.w;
        } else if constexpr (Tr::BPL == 8) {
          const uint2 v = *reinterpret_cast<const uint2*>(src);
          x[r].w[0] = v.x;
          x[r].w[1] = v.y;
        } else {
          x[r].w[0] = *reinterpret_cast<const uint32_t*>(src);
        }
        x[r].s = 0u;
        if constexpr (SW > 0) {
          const uint8_t* sp = st + s_off + ((u * 4 + r) * SW * 32 + lane) * 4;
          if (R.w[r] != nullptr && in_k) {
            if constexpr (FMT == MOE_FMT_NVFP4) {
              const uintptr_t a = (uintptr_t)scale_addr<FMT>(R, r, kt, t, 0);
              x[r].s = (*reinterpret_cast<const uint32_t*>(sp) >> (8 * (a & 3))) & 0xFFFFu;
            } else if constexpr (FMT == MOE_FMT_MXFP4) {
              const uintptr_t a = (uintptr_t)scale_addr<FMT>(R, r, kt, t, 0);
              x[r].s = (*reinterpret_cast<const uint32_t*>(sp) >> (8 * (a & 3))) & 0xFFu;
            } else {
              const uintptr_t a0 = (uintptr_t)scale_addr<FMT>(R, r, kt, t, 0);
              const uintptr_t a1 = (uintptr_t)scale_addr<FMT>(R, r, kt, t, 1);
              const uint32_t sv = (*reinterpret_cast<const uint32_t*>(sp) >> (8 * (a0 & 3))) & 0xFFFFu;
              const uint32_t bv =
                  (*reinterpret_cast<const uint32_t*>(sp + 32 * 4) >> (8 * (a1 & 3))) & 0xFFFFu;
              x[r].s = sv | (bv << 16);
            }
          }
        }
      }
      uint2 bh[Tr::KS][NTG], bl[Tr::KS][NTG];
#pragma unroll
      for (int q = 0; q < NTG; ++q) {
        const bool live = cidx[q] >= 0 && in_k;
#pragma unroll
        for (int kb = 0; kb < KSB; ++kb) {
          uint4 v = make_uint4(0u, 0u, 0u, 0u);
          if (live)
            v = *reinterpret_cast<const uint4*>(
                st + b_off + (((u * KSB + kb) * ncols + cidx[q]) * 4 + t) * 16);
          if constexpr (HILO) {
            bh[kb][q] = make_uint2(v.x, v.y);
            bl[kb][q] = make_uint2(v.z, v.w);
          } else {
            bh[2 * kb][q] = make_uint2(v.x, v.y);
            bh[2 * kb + 1][q] = make_uint2(v.z, v.w);
            bl[2 * kb][q] = make_uint2(0u, 0u);
            bl[2 * kb + 1][q] = make_uint2(0u, 0u);
          }
        }
      }
      if constexpr (Tr::POST) {
        zero<NTG>(d);
#pragma unroll
        for (int n = 0; n < NTG; ++n)
#pragma unroll
          for (int q = 0; q < 4; ++q) d1[n][q] = 0.f;
      }
      ksteps<FMT, NTG, HILO>(std::make_integer_sequence<int, Tr::KS / 2>{}, x, bh, bl, d, d1);
      if constexpr (Tr::POST) {
        // fragment q: rows g (q < 2) or g + 8 (q >= 2) of each tile: raw rows 0/1 and 2/3
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          float mul_lo, add_lo, mul_hi, add_hi;
          post_scales<FMT>(x[2 * m], mul_lo, add_lo);
          post_scales<FMT>(x[2 * m + 1], mul_hi, add_hi);
#pragma unroll
          for (int n = 0; n < NTG; ++n)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float mul = q < 2 ? mul_lo : mul_hi, add = q < 2 ? add_lo : add_hi;
              p[m][n][q] = fmaf(mul, d[m][n][q], p[m][n][q]);
              if constexpr (FMT == MOE_FMT_Q4_AFFINE_G64)
                p[m][n][q] = fmaf(add, d1[n][q], p[m][n][q]);
            }
        }
      }
      // last k-tile of a chunk: the chunk's value is complete
      if ((kt + 1) % TPC == 0 || kt + 1 == kt_end) {
        float (&v)[2][NTG][4] = Tr::POST ? p : d;
        const int c = kt / TPC;
        if (sm.base == nullptr) {
#pragma unroll
          for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int n = 0; n < NTG; ++n)
#pragma unroll
              for (int q = 0; q < 4; ++q) acc[m][n][q] += v[m][n][q];
        } else {
#pragma unroll
          for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int n = 0; n < NTG; ++n)
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int col = sm.col0 + 8 * n + 2 * t + (q & 1);
                const int r = 16 * m + g + (q >= 2 ? 8 : 0);
                if (col < sm.n)
                  __stcg(sm.base + (size_t)col * sm.col_stride + (size_t)c * 32 + r, v[m][n][q]);
              }
        }
        zero<NTG>(p);
        zero<NTG>(d);
      }
    }
  }
  cp_wait<0>();  // nothing of this piece stays in flight into the next one's ring stages
}

// Sum of the stored chunk values of a job, in chunk order (the reduction of a split job).
template <int NTG>
__device__ __forceinline__ void sum_slots(const SlotMap& sm, int nch, float (&acc)[2][NTG][4]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  constexpr int kB = NTG == 1 ? 4 : 2;  // chunks whose values are loaded together
  zero<NTG>(acc);
  for (int c0 = 0; c0 < nch; c0 += kB) {
    // every load of the batch first (one round trip to L2), then the adds in chunk order
    float v[kB][2][NTG][4];
#pragma unroll
    for (int b = 0; b < kB; ++b)
#pragma unroll
      for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int n = 0; n < NTG; ++n)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int col = sm.col0 + 8 * n + 2 * t + (q & 1);
            const int r = 16 * m + g + (q >= 2 ? 8 : 0);
            v[b][m][n][q] = (col < sm.n && c0 + b < nch)
                                ? __ldcg(sm.base + (size_t)col * sm.col_stride +
                                         (size_t)(c0 + b) * 32 + r)
                                : 0.f;
          }
#pragma unroll
    for (int b = 0; b < kB; ++b) {
      if (c0 + b >= nch) break;
#pragma unroll
      for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int n = 0; n < NTG; ++n)
#pragma unroll
          for (int q = 0; q < 4; ++q) acc[m][n][q] += v[b][m][n][q];
    }
  }
}

// ---- the call's parameters -------------------------------------------------------------------

// Routing as the tensor-core phases read it (shared memory in the persistent kernel, global
// memory in the multi-kernel path): U active experts in ascending id, then the shared expert.
struct SlotView {
  const int* slot_e;    // [U] expert ids
  const int* slot_beg;  // [U] first sorted position of each
  const int* slot_n;    // [U] pairs of each
  const int* sorted;    // [te] pair ids in sorted order
  const float* wts;     // [te] routing weight of each pair
  const int* tp;        // [te] sorted position of each pair
  const float* gamma;   // [m] shared-expert gate
  int U;
};

struct TcExtra {
  int W;               // warps taking part in a phase (all of the grid)
  int gu_piece;        // 1: gate/up jobs may be split by chunk (their chunk values fit); 0: not
  int dn_piece;        // the same for down
  int force_split;     // 1: split every phase that may split (tests); 0: the rule of split_jobs
  int tiles_i, tiles_s;  // gate/up jobs per routed / shared expert (16 row pairs each)
  int tiles_h;         // down jobs per expert (32 output columns each)
  int nch_h, nch_i, nch_s;  // chunks of h, I, S
  uint8_t* xb;         // activations in the operand type and stored order [m][h] (F16 formats)
  uint8_t* act;        // [te][I / 4][8] operand halves: 4 hi then 4 lo per 4 stored elements
  uint8_t* sh_act;     // the shared expert's [m][S / 4][8]
  float* gu_slots;     // chunk values of split gate/up jobs: [pair][tile][chunk][32] for the
                       // routed pairs, then [row][tile][chunk][32] for the shared expert
  float* dn_slots;     // the same for down jobs
  unsigned* tk_gu;     // per gate/up job: chunks finished
  unsigned* tk_dn;     // per down job: chunks finished
  unsigned* tk_col;    // per 32-column tile: down jobs finished
  unsigned* ready;     // per slot: gate/up jobs whose act rows are written
  int tk_words;        // words of the ticket and ready arrays (zeroed at the start of every call)
  unsigned long long* stamps;  // phase timestamps [CTA][16] (timer builds only, else null)
};

// Optional phase timestamps (library built with -DMOE_PHASE_TIMERS): thread 0 of every CTA
// keeps %globaltimer (ns) at phase boundaries in shared memory and writes them at the end of the
// kernel into a region at the end of the workspace (slot 15: the entry time).
#ifdef MOE_PHASE_TIMERS
// The timer read is predicated on the value a shared-memory atomic returns, so the assembler
// cannot move it above the barrier or the work before it.
#define TC_STAMP(slot)                                                                 \
  do {                                                                                 \
    if (threadIdx.x == 0) {                                                            \
      unsigned long long t_;                                                           \
      const uint32_t a_ = (uint32_t)__cvta_generic_to_shared(&s_stamps[(slot)]);      \
      asm volatile(                                                                    \
          "{ .reg .pred p_; .reg .u32 v_; atom.shared.add.u32 v_, [%1], 0;"            \
          " setp.ne.u32 p_, v_, 0xFFFFFFFF; mov.u64 %0, 0; @p_ mov.u64 %0, %%globaltimer; }" \
          : "=l"(t_) : "r"(a_) : "memory");                                            \
      s_stamps[(slot)] = t_;                                                           \
    }                                                                                  \
  } while (0)
#define TC_STAMP_GLOBAL()                                                              \
  do {                                                                                 \
    if (threadIdx.x == 0) {                                                            \
      unsigned long long t_;                                                           \
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_)::"memory");                 \
      s_stamps[15] = t_;                                                               \
    }                                                                                  \
  } while (0)
#define TC_STAMP_FLUSH()                                                               \
  do {                                                                                 \
    if (threadIdx.x < 16 && tx.stamps != nullptr)                                      \
      tx.stamps[blockIdx.x * 16 + threadIdx.x] = s_stamps[threadIdx.x];                \
  } while (0)
#else
#define TC_STAMP(slot) \
  do {                 \
  } while (0)
#define TC_STAMP_GLOBAL() \
  do {                    \
  } while (0)
#define TC_STAMP_FLUSH() \
  do {                   \
  } while (0)
#endif

// Store an fp32 activation value as the operand-type pair hi + lo at stored position pos of a
// row of 4-element groups: hi at [pos / 4][pos % 4], lo at [pos / 4][4 + pos % 4].
template <bool F16>
__device__ __forceinline__ void split_store(float v, uint8_t* row, int pos, unsigned* status) {
  const size_t ih = (size_t)(pos >> 2) * 8 + (pos & 3), il = ih + 4;
  if constexpr (F16) {
    const __half h = __float2half_rn(v);
    const __half l = __float2half_rn(v - __half2float(h));
    if (!(fabsf(v) <= 65504.f)) atomicExch(status, (unsigned)MOE_ERR_DEVICE_CHECK);
    reinterpret_cast<__half*>(row)[ih] = h;
    reinterpret_cast<__half*>(row)[il] = l;
  } else {
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    const __nv_bfloat16 l = __float2bfloat16_rn(v - __bfloat162float(h));
    reinterpret_cast<__nv_bfloat16*>(row)[ih] = h;
    reinterpret_cast<__nv_bfloat16*>(row)[il] = l;
  }
}

// Activations in the operand type and stored order, for the F16 formats: all threads of the
// launch take 16-element blocks in turn (x is bf16, which fp16 holds exactly for
// 2^-17 <= |x| <= 65504; larger values set MOE_ERR_DEVICE_CHECK).
template <int FMT>
__device__ void convert_x(const Params& p, const TcExtra& tx, int gtid, int nthreads) {
  if constexpr (Traits<FMT>::F16) {
    const int nblk = p.m * p.h / 16;
    const __nv_bfloat16* xs = reinterpret_cast<const __nv_bfloat16*>(p.x);
    __half* xd = reinterpret_cast<__half*>(tx.xb);
    for (int b = gtid; b < nblk; b += nthreads) {
      const uint4 v0 = __ldg(reinterpret_cast<const uint4*>(xs + (size_t)b * 16));
      const uint4 v1 = __ldg(reinterpret_cast<const uint4*>(xs + (size_t)b * 16 + 8));
      const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
      __half o[16];
      bool bad = false;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float f = (i & 1) ? bf16hi(w[i >> 1]) : bf16lo(w[i >> 1]);
        bad |= !(fabsf(f) <= 65504.f);
        o[act_pos<FMT>(i)] = __float2half_rn(f);
      }
      if (bad) atomicExch(p.ctrl + kStatus, (unsigned)MOE_ERR_DEVICE_CHECK);
      uint4* dst = reinterpret_cast<uint4*>(xd + (size_t)b * 16);
      dst[0] = *reinterpret_cast<const uint4*>(&o[0]);
      dst[1] = *reinterpret_cast<const uint4*>(&o[8]);
    }
  }
}

// Work items of a phase: (slot, tile, column group), slot a < U a routed expert and slot U the
// shared expert; a slot's items are tiles(a) * ncg(a), tile-major (the column groups of a tile
// are adjacent, so their re-reads of the tile's rows find them in L2). A unit is an item (whole
// mode) or one 256-element chunk of it (piece mode). The prefix sums of the slots' items and
// units are built once per CTA; warp w of W takes the units [w C / W, (w+1) C / W) of the
// concatenated list, so every warp gets the same number of column-group passes over its rows.
struct PhaseMap {
  int item_pre[kMaxPairs + 2];  // first item of each slot
  int unit_pre[kMaxPairs + 2];  // first unit of each slot
  int piece;                    // 1: the phase's jobs are split by chunk
};

// Whether a phase of J jobs (items) of nch chunks each runs split by chunk on a grid of W warps:
// when there are fewer whole jobs than half the warps (more than half the grid would idle) and a
// job is long enough to be worth cutting: at least four chunks, or any length for the formats
// whose k-tiles are instruction-heavy (MXFP4, Q4: decode plus a post-scaled chain per k-tile).
// A piece restarts its warp's copy pipeline and adds a ticket, which a short bf16, FP8 or NVFP4
// job does not win back. Above half the warps, whole jobs (handed out round-robin and taken
// dynamically by the CTA's warps) are balanced well enough. Measured on the B200 at m = 1..64
// over the published shapes, every format.
__device__ __forceinline__ bool split_jobs(int J, int W, int nch, bool heavy) {
  return J > 0 && J < W / 2 && (heavy || nch >= 4);
}

// By one warp: the prefix map of a phase over nslots slots. One scan gives the items (jobs)
// before each slot and their total J, from which decide(J) says whether the phase splits its jobs
// by chunk; the units before slot a are then its items times the chunks per job (nch_a for every
// slot but the last, which has nch_last: the shared expert's down jobs may differ).
template <typename ItemsOf, typename Decide>
__device__ void build_map(int nslots, int nch_a, int nch_last, ItemsOf items_of, Decide decide,
                          PhaseMap& pm) {
  const int lane = threadIdx.x & 31;
  int ib = 0, last_items = 0;
  for (int a0 = 0; a0 < nslots; a0 += 32) {
    const int a = a0 + lane;
    const int it = a < nslots ? items_of(a) : 0;
    int iti = it;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, iti, o);
      if (lane >= o) iti += x;
    }
    if (a < nslots) pm.item_pre[a] = ib + iti - it;
    if (a == nslots - 1) last_items = it;
    ib += __shfl_sync(0xffffffffu, iti, 31);
  }
  last_items = __reduce_add_sync(0xffffffffu, last_items);  // only one lane holds it
  const bool piece = decide(ib);
  __syncwarp();  // every lane's item_pre entries are written
  for (int a = lane; a <= nslots; a += 32) {
    int up;
    if (!piece) {
      up = a < nslots ? pm.item_pre[a] : ib;
    } else if (a < nslots) {
      up = pm.item_pre[a] * nch_a;  // slots before a are all but the last
    } else {
      up = (ib - last_items) * nch_a + last_items * nch_last;
    }
    pm.unit_pre[a] = up;
  }
  if (lane == 0) {
    pm.item_pre[nslots] = ib;
    pm.piece = piece;
  }
}

// The units of CTA cta of G, taken by the CTA's warps from a shared-memory counter (zeroed before
// the phase), so the warps of a CTA balance among themselves. Split jobs: the range
// [cta C / G, (cta+1) C / G) of the concatenated list, `grab` units at a time, so that a piece
// covers consecutive chunks. Whole jobs: every G-th job from cta on, so that every CTA gets its
// share of each slot's jobs (jobs of a slot with many live columns stream fewer weight bytes per
// ring stage, and a contiguous range would give them all to the last CTAs).
// f(slot, item, c0, c1, whole) runs one piece (one item's chunks [c0, c1)).
template <typename NchOf, typename PieceFn>
__device__ __forceinline__ void for_units(const PhaseMap& pm, int nslots, int cta, int G,
                                          bool piece, int warps, int* counter, NchOf nch_of,
                                          PieceFn f) {
  const long long C = pm.unit_pre[nslots];
  int a = 0;
  if (!piece) {
    for (;;) {
      int k = 0;
      if ((threadIdx.x & 31) == 0) k = atomicAdd(counter, 1);
      k = __shfl_sync(0xffffffffu, k, 0);
      const long long q = cta + (long long)k * G;
      if (q >= C) break;
      while (pm.unit_pre[a + 1] <= q) ++a;
      f(a, (int)(q - pm.unit_pre[a]), 0, nch_of(a), true);
    }
    return;
  }
  const int q0 = (int)((long long)cta * C / G), q1 = (int)((long long)(cta + 1) * C / G);
  // split jobs: about one grab per warp, so pieces stay long (fewer pipeline restarts and
  // tickets); a warp that finishes early takes what a late one has not
  const int grab = max(1, (q1 - q0 + warps - 1) / warps);
  for (;;) {
    int u0 = 0;
    if ((threadIdx.x & 31) == 0) u0 = atomicAdd(counter, grab);
    u0 = q0 + __shfl_sync(0xffffffffu, u0, 0);
    if (u0 >= q1) break;
    const int u1 = min(u0 + grab, q1);
    int q = u0;
    while (pm.unit_pre[a] > q) --a;
    while (q < u1) {
      while (pm.unit_pre[a + 1] <= q) ++a;
      const int nch = nch_of(a);
      const int per = nch;
      const int r = q - pm.unit_pre[a];
      const int item = r / per;
      const int c = r - item * per;
      const int item_end = pm.unit_pre[a] + (item + 1) * per;
      const int c1 = c + ((u1 < item_end ? u1 : item_end) - q);
      f(a, item, c, c1, c == 0 && c1 == nch);
      q += c1 - c;
    }
  }
}

// Finish a split item: add this piece's chunks to the item's ticket; true for the warp that
// completed it (it then reads every chunk value).
__device__ __forceinline__ bool piece_done(unsigned* ticket, int chunks, int nch) {
  __threadfence();
  __syncwarp();
  unsigned old = 0;
  if ((threadIdx.x & 31) == 0) old = atomicAdd(ticket, (unsigned)chunks);
  old = __shfl_sync(0xffffffffu, old, 0);
  const bool last = old + (unsigned)chunks == (unsigned)nch;
  if (last) __threadfence();
  return last;
}

// Slot a's activation columns (its pairs) and their count.
__device__ __forceinline__ int slot_cols(const Params& p, const SlotView& sv, int a) {
  return a == sv.U ? p.m : sv.slot_n[a];
}

// The prefix maps of both phases (one warp builds each), with each phase's split decision taken
// from its job count (split_jobs) on this call's routing.
template <int FMT, int NTG>
__device__ void build_maps(const Params& p, const TcExtra& tx, const SlotView& sv, PhaseMap& gu,
                           PhaseMap& dn, int warp) {
  constexpr bool kHeavy = Traits<FMT>::POST;  // MXFP4, Q4
  const int ns = sv.U + p.has_shared;
  const int W = gridDim.x * tc_warps<FMT, NTG>();
  if (warp == 0) {
    const bool may = tx.gu_piece != 0, force = tx.force_split != 0;
    build_map(
        ns, tx.nch_h, tx.nch_h,
        [&](int a) {
          return (a == sv.U ? tx.tiles_s : tx.tiles_i) * ceil_div(slot_cols(p, sv, a), 8 * NTG);
        },
        [&](int J) { return may && (force || split_jobs(J, W, tx.nch_h, kHeavy)); }, gu);
  } else if (warp == 1) {
    const bool may = tx.dn_piece != 0, force = tx.force_split != 0;
    build_map(
        ns, tx.nch_i, p.has_shared ? tx.nch_s : tx.nch_i,
        [&](int a) { return tx.tiles_h * ceil_div(slot_cols(p, sv, a), 8 * NTG); },
        [&](int J) { return may && (force || split_jobs(J, W, tx.nch_i, kHeavy)); }, dn);
  }
}

// ---- gate/up phase --------------------------------------------------------------------------

template <int FMT, int NTG>
__device__ void gate_up_phase(const Params& p, const TcExtra& tx, const SlotView& sv,
                              const PhaseMap& pm, int* counter, uint8_t* ring) {
  constexpr bool F16 = Traits<FMT>::F16;
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int U = sv.U, ns = U + p.has_shared;
  for_units(pm, ns, blockIdx.x, gridDim.x, pm.piece != 0, tc_warps<FMT, NTG>(), counter,
            [&](int) { return tx.nch_h; },
            [&](int a, int item, int c0, int c1, bool whole) {
    const bool sh = a == U;
    const int n = slot_cols(p, sv, a);
    const int ncg = ceil_div(n, 8 * NTG);
    const int tile = item / ncg, cg = item - tile * ncg;
    const MatDev G = pick_mat(sh, p.sg, p.rg);
    const MatDev Um = pick_mat(sh, p.su, p.ru);
    const int e = sh ? 0 : sv.slot_e[a];
    const int beg = sh ? 0 : sv.slot_beg[a];
    const int N = sh ? p.S : p.I;
    // rows: tile 0 = gate rows [16 tile, +16), tile 1 = up rows of the same outputs
    JobRows Rg = job_rows<FMT>(G, e, 16 * tile, 0, lane);
    const JobRows Ru = job_rows<FMT>(Um, e, 16 * tile, 0, lane);
    Rg.w[2] = Ru.w[0];
    Rg.w[3] = Ru.w[1];
    Rg.sc[2] = Ru.sc[0];
    Rg.sc[3] = Ru.sc[1];
    Rg.bi[2] = Ru.bi[0];
    Rg.bi[3] = Ru.bi[1];
    // the tensor scales now, so their round trip overlaps the job's weight stream
    const float tsg = (FMT == MOE_FMT_NVFP4 || FMT == MOE_FMT_FP8_E4M3) ? __ldg(G.tscale + e) : 1.f;
    const float tsu = (FMT == MOE_FMT_NVFP4 || FMT == MOE_FMT_FP8_E4M3) ? __ldg(Um.tscale + e) : 1.f;
    JobCols<NTG> C;
#pragma unroll
    for (int q = 0; q < NTG; ++q) {
      const int col = cg * 8 * NTG + q * 8 + g;
      C.row[q] = nullptr;
      if (col < n) {
        const int row = sh ? col : sv.sorted[beg + col] / p.k;
        C.row[q] = F16 ? tx.xb + (size_t)row * p.h * 2
                       : reinterpret_cast<const uint8_t*>(p.x) + (size_t)row * p.h * 2;
      }
    }
    const int ncols = min(8 * NTG, n - cg * 8 * NTG);
    float acc[2][NTG][4];
    zero<NTG>(acc);
    SlotMap sm;
    sm.base = nullptr;
    sm.n = n;
    sm.col0 = cg * 8 * NTG;
    if (!whole) {
      const int tiles = sh ? tx.tiles_s : tx.tiles_i;
      sm.col_stride = tiles * tx.nch_h * 32;
      sm.base = tx.gu_slots +
                (sh ? (size_t)p.m * p.k * tx.tiles_i * tx.nch_h * 32 + (size_t)tile * tx.nch_h * 32
                    : ((size_t)beg * tx.tiles_i + tile) * tx.nch_h * 32);
      run_chunks<FMT, NTG, false>(Rg, C, ncols, p.h, c0, c1, acc, sm, ring, p.x);
      if (!piece_done(tx.tk_gu + pm.item_pre[a] + item, c1 - c0, tx.nch_h)) return;
      sum_slots<NTG>(sm, tx.nch_h, acc);
    } else {
      run_chunks<FMT, NTG, false>(Rg, C, ncols, p.h, 0, tx.nch_h, acc, sm, ring, p.x);
    }
    // epilogue: fragment f = rows g (f < 2) / g + 8, columns 2t, 2t + 1
#pragma unroll
    for (int q = 0; q < NTG; ++q)
#pragma unroll
      for (int f = 0; f < 4; ++f) {
        const int i = 16 * tile + g + (f >= 2 ? 8 : 0);
        const int col = cg * 8 * NTG + q * 8 + 2 * t + (f & 1);
        if (i < N && col < n) {
          float gv = acc[0][q][f] * tsg, uv = acc[1][q][f] * tsu;
          if (!sh && p.before_ffn) {
            const float w = sv.wts[sv.sorted[beg + col]];
            gv *= w;
            uv *= w;
          }
          uint8_t* row = sh ? tx.sh_act + (size_t)col * p.S * 4
                            : tx.act + (size_t)(beg + col) * p.I * 4;
          split_store<F16>(act_mul(p.act_kind, gv, uv), row, act_pos<FMT>(i), p.ctrl + kStatus);
        }
      }
    // the job's act rows are written: count it for its slot (down jobs of the slot wait for all)
    __syncwarp();
    if (lane == 0) {
      __threadfence();
      atomicAdd(tx.ready + a, 1u);
    }
  });
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
constexpr long long kChainSpinLimit = 2000000000LL;  // clock cycles (about a second)

// ---- down phase + blend -----------------------------------------------------------------------

template <int FMT, int NTG>
__device__ void down_phase(const Params& p, const TcExtra& tx, const SlotView& sv,
                           const PhaseMap& pm, const PhaseMap& gu, long long spin_limit,
                           unsigned extra, int* counter, uint8_t* ring) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int U = sv.U, ns = U + p.has_shared;
  // (slot, column group) items per column tile: the blend waits for all of them
  unsigned col_target = 0;
  for (int a = lane; a < ns; a += 32) col_target += (unsigned)ceil_div(slot_cols(p, sv, a), 8 * NTG);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) col_target += __shfl_xor_sync(0xffffffffu, col_target, o);
  int ready_slot = -1;  // the last slot whose gate/up jobs this warp saw complete
  for_units(pm, ns, blockIdx.x, gridDim.x, pm.piece != 0, tc_warps<FMT, NTG>(), counter,
            [&](int a) { return a == U ? tx.nch_s : tx.nch_i; },
            [&](int a, int item, int c0, int c1, bool whole) {
    const bool sh = a == U;
    const int n = slot_cols(p, sv, a);
    const int ncg = ceil_div(n, 8 * NTG);
    const int ct = item / ncg, cg = item - ct * ncg;
    if (a != ready_slot) {
      // the slot's act rows: wait (bounded) until every gate/up job of the slot has counted
      if (lane == 0) {
        // extra: 1 in the failure-detection test (the wait then runs out), else 0
        const unsigned want = (unsigned)(gu.item_pre[a + 1] - gu.item_pre[a]) + extra;
        const long long t0 = clock64();
        while (ld_acquire_u32(tx.ready + a) < want) {
          if (clock64() - t0 > spin_limit) {
            atomicExch(p.ctrl + kStatus, (unsigned)MOE_ERR_DEVICE_TIMEOUT);
            break;
          }
        }
      }
      __syncwarp();
      ready_slot = a;
    }
    const MatDev D = pick_mat(sh, p.sd, p.rd);
    const int e = sh ? 0 : sv.slot_e[a];
    const int beg = sh ? 0 : sv.slot_beg[a];
    const int K = sh ? p.S : p.I;
    const int nch = sh ? tx.nch_s : tx.nch_i;
    const JobRows R = job_rows<FMT>(D, e, 32 * ct, 32 * ct + 16, lane);
    const float ts = (FMT == MOE_FMT_NVFP4 || FMT == MOE_FMT_FP8_E4M3) ? __ldg(D.tscale + e) : 1.f;
    JobCols<NTG> C;
#pragma unroll
    for (int q = 0; q < NTG; ++q) {
      const int col = cg * 8 * NTG + q * 8 + g;
      C.row[q] = col < n ? (sh ? tx.sh_act + (size_t)col * K * 4
                               : tx.act + (size_t)(beg + col) * K * 4)
                         : nullptr;
    }
    const int ncols = min(8 * NTG, n - cg * 8 * NTG);
    float acc[2][NTG][4];
    zero<NTG>(acc);
    SlotMap sm;
    sm.base = nullptr;
    sm.n = n;
    sm.col0 = cg * 8 * NTG;
    if (!whole) {
      sm.col_stride = tx.tiles_h * nch * 32;
      sm.base = tx.dn_slots +
                (sh ? (size_t)p.m * p.k * tx.tiles_h * tx.nch_i * 32 + (size_t)ct * nch * 32
                    : ((size_t)beg * tx.tiles_h + ct) * nch * 32);
      run_chunks<FMT, NTG, true>(R, C, ncols, K, c0, c1, acc, sm, ring, p.x);
      if (!piece_done(tx.tk_dn + pm.item_pre[a] + item, c1 - c0, nch)) return;
      sum_slots<NTG>(sm, nch, acc);
    } else {
      run_chunks<FMT, NTG, true>(R, C, ncols, K, 0, nch, acc, sm, ring, p.x);
    }
    // y rows: output columns 32 ct + 16 tile + g (+8); columns: the slot's pairs
#pragma unroll
    for (int m2 = 0; m2 < 2; ++m2)
#pragma unroll
      for (int q = 0; q < NTG; ++q)
#pragma unroll
        for (int f = 0; f < 4; ++f) {
          const int c = 32 * ct + 16 * m2 + g + (f >= 2 ? 8 : 0);
          const int col = cg * 8 * NTG + q * 8 + 2 * t + (f & 1);
          if (c < p.h && col < n) {
            const float y = acc[m2][q][f] * ts;
            if (sh) {
              __stcg(p.ysh + (size_t)col * p.h + c, y);
            } else {
              __stcg(p.ypart + (size_t)(beg + col) * p.h + c, y);
            }
          }
        }
    // the column tile is complete once every (slot, column group) item of it is: the warp whose
    // arrival reaches that count blends it
    __threadfence();
    __syncwarp();
    unsigned old = 0;
    if (lane == 0) old = atomicAdd(tx.tk_col + ct, 1u);
    old = __shfl_sync(0xffffffffu, old, 0);
    if (old + 1u != col_target) return;
    __threadfence();
    // blend the 32 columns of tile ct for every row: lane = column. The values of kBR rows
    // (kBS slots each) are loaded together, one round trip to L2, then added in slot order.
    const int c = 32 * ct + lane;
    if (c >= p.h) return;
    constexpr int kBR = 4, kBS = 8;
    for (int r0 = 0; r0 < p.m; r0 += kBR) {
      float o[kBR];
#pragma unroll
      for (int i = 0; i < kBR; ++i) o[i] = 0.f;
      for (int s0 = 0; s0 < p.k; s0 += kBS) {
        float v[kBR][kBS];
#pragma unroll
        for (int i = 0; i < kBR; ++i)
#pragma unroll
          for (int j = 0; j < kBS; ++j) {
            const int r = r0 + i, s2 = s0 + j;
            v[i][j] = (r < p.m && s2 < p.k)
                          ? __ldcg(p.ypart + (size_t)sv.tp[r * p.k + s2] * p.h + c)
                          : 0.f;
          }
#pragma unroll
        for (int i = 0; i < kBR; ++i)
#pragma unroll
          for (int j = 0; j < kBS; ++j) {
            const int r = r0 + i, s2 = s0 + j;
            if (r < p.m && s2 < p.k)
              o[i] = fmaf(p.before_ffn ? 1.f : sv.wts[r * p.k + s2], v[i][j], o[i]);
          }
      }
      float sh[kBR];
#pragma unroll
      for (int i = 0; i < kBR; ++i)
        sh[i] = (p.has_shared && r0 + i < p.m) ? __ldcg(p.ysh + (size_t)(r0 + i) * p.h + c) : 0.f;
#pragma unroll
      for (int i = 0; i < kBR; ++i) {
        const int r = r0 + i;
        if (r >= p.m) break;
        if (p.has_shared) o[i] = fmaf(sv.gamma[r], sh[i], o[i]);
        const size_t oi = (size_t)r * p.h + c;
        if (p.out_bf16) {
          reinterpret_cast<__nv_bfloat16*>(p.out)[oi] = __float2bfloat16_rn(o[i]);
        } else {
          reinterpret_cast<float*>(p.out)[oi] = o[i];
        }
      }
    }
  });
}

}  // namespace tc
}  // namespace moe

namespace moe {
namespace tc {

// ---- routing and grouping for the tensor-core path ---------------------------------------------

// Routing tables of a call (shared memory of every persistent CTA).
struct TcRoute {
  int idx[kMaxPairs];
  float w[kMaxPairs];
  int sorted[kMaxPairs];     // pair ids by (expert, pair)
  int tp[kMaxPairs];         // sorted position of each pair
  int slot_e[kMaxPairs];     // active experts, ascending
  int slot_beg[kMaxPairs];
  int slot_n[kMaxPairs];
  int lead[kMaxPairs];       // per pair: 1 if it is its expert's first pair
  int less[kMaxPairs];       // per pair: pairs with a smaller expert id
  int cnt[kMaxPairs];        // per pair: pairs with its expert id
  float gamma[MOE_MAX_ROWS];
  float bias[MOE_MAX_EXPERTS];
  int n_active;
};

// Stable grouping of the te pairs by expert in shared memory, by all threads of the CTA: pair p
// lands at #(pairs with a smaller id) + #(earlier pairs with the same id); the first pair of
// each expert opens its slot, slots in ascending expert id.
__device__ void tc_group(int te, TcRoute& R) {
  const int tid = threadIdx.x, nt = blockDim.x;
  for (int p = tid; p < te; p += nt) {
    const int e = R.idx[p];
    int less = 0, before = 0, cnt = 0;
    for (int q = 0; q < te; ++q) {
      const int f = R.idx[q];
      less += f < e;
      cnt += f == e;
      before += (f == e) & (q < p);
    }
    const int pos = less + before;
    R.sorted[pos] = p;
    R.tp[p] = pos;
    R.lead[p] = before == 0;
    R.less[p] = less;
    R.cnt[p] = cnt;
  }
  __syncthreads();
  int leaders = 0;
  for (int p = tid; p < te; p += nt) {
    if (!R.lead[p]) continue;
    const int e = R.idx[p];
    int slot = 0;
    for (int q = 0; q < te; ++q) slot += R.lead[q] & (R.idx[q] < e);
    R.slot_e[slot] = e;
    R.slot_beg[slot] = R.less[p];
    R.slot_n[slot] = R.cnt[p];
  }
  if (tid == 0) {
    for (int q = 0; q < te; ++q) leaders += R.lead[q];
    R.n_active = leaders;
  }
  __syncthreads();
}

// ---- the persistent kernel: the whole call in one launch ------------------------------------------

struct TcPlan {
  long long spin_limit;       // clock cycles a device-side wait may spin before it gives up
  long long l2_prefetch_cap;  // largest per-call down-projection byte count asked into L2
  unsigned bar_extra;         // arrivals the barrier and each ready wait expect beyond the real
                              // ones (0; 1 in the failure-detection test)
};

// Phases (all CTAs co-resident, cooperative launch, one CTA of 8 or 16 warps per SM):
//   A  router logits, one warp per (router row, activation row) over the whole grid; the
//      activations in the operand type and order; zero the call's tickets and ready counters;
//      arrive and wait at the grid barrier (the only one).
//   C  every CTA routes every row and groups the pairs in its shared memory; the last warp asks
//      L2 for this CTA's share of the active experts' down rows; warps 0 and 1 build the two
//      phases' maps and split decisions.
//   D  gate/up jobs over all warps of the grid (tc::gate_up_phase); each job counts in its slot's
//      ready counter.
//   E  down jobs over all warps, each slot's once its ready counter is full; the warp completing
//      a 32-column tile blends it (tc::down_phase).
template <int FMT, int NTG>
__global__ void __launch_bounds__(32 * tc_warps<FMT, NTG>(), 1) tc_fused_kernel(
    const __grid_constant__ Params p, const __grid_constant__ TcExtra tx,
    const __grid_constant__ TcPlan pl) {
  extern __shared__ __align__(16) uint8_t tc_ring[];
  constexpr int kWarps = tc_warps<FMT, NTG>(), kThreads = 32 * kWarps;
  __shared__ TcRoute R;
  __shared__ PhaseMap s_gu, s_dn;
  __shared__ unsigned long long s_base;
  __shared__ int s_next[2];  // units taken so far by this CTA's warps in phases D and E
#ifdef MOE_PHASE_TIMERS
  __shared__ unsigned long long s_stamps[16];
#endif
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  const int m = p.m, k = p.k, te = m * k;
  const int wid = cta * kWarps + warp;
  const size_t xrow_bytes = (size_t)p.h * 2;
  const int e_tot = p.E + (p.shared_kind == MOE_SHARED_SIGMOID_GATE ? 1 : 0);
  auto router_row = [&](int e) {
    return e < p.E ? (const uint8_t*)p.router_w + (size_t)e * xrow_bytes
                   : (const uint8_t*)p.shared_gate_w;
  };
  TC_STAMP(0);
  TC_STAMP_GLOBAL();
  // prologue (may overlap the previous kernel): this CTA's router rows into L2
  if (tid == 0)
    for (int e = cta; e < e_tot; e += G) prefetch_l2_bulk(router_row(e), xrow_bytes);
  pdl_wait();
  TC_STAMP(1);
  unsigned long long* bar_ctr = reinterpret_cast<unsigned long long*>(p.ctrl + kBarCounter);
  if (tid == 0) {
    s_base = ld_acquire_u64(bar_ctr) / (unsigned long long)G * (unsigned long long)G;
    s_next[0] = 0;
    s_next[1] = 0;
  }
  if (p.has_bias)
    for (int e = tid; e < p.E; e += kThreads) R.bias[e] = __ldg(p.expert_bias + e);

  // ---- A: router logits; operand activations; zeroed tickets ------------------------------------
  {
    const int nch = (int)(xrow_bytes / 16);
    for (int d = wid; d < e_tot * m; d += G * kWarps) {
      const int e = d / m, r = d - e * m;
      const uint8_t* xr = (const uint8_t*)p.x + (size_t)r * xrow_bytes;
      const float acc = router_dot_gx<true>(router_row(e), xr, nch);
      if (lane == 0) p.logits[(size_t)r * (p.E + 1) + e] = acc;
    }
  }
  convert_x<FMT>(p, tx, cta * kThreads + tid, G * kThreads);
  for (int i = cta * kThreads + tid; i < tx.tk_words; i += G * kThreads) tx.tk_gu[i] = 0u;
  __syncthreads();
  TC_STAMP(2);
  const GridBarrier bar{bar_ctr, p.ctrl + kStatus, s_base, pl.spin_limit, pl.bar_extra};
  bar.arrive();
  bar.wait(1);
  TC_STAMP(3);

  // ---- C: routing and grouping in every CTA -------------------------------------------------------
  {
    const RouteCfg rc = route_cfg(p);
    for (int r = warp; r < m; r += kWarps) {
      int id;
      float w, gm;
      const bool ok = route_row(rc, r, R.bias, id, w, gm);
      if (lane < k) {
        R.idx[r * k + lane] = id;
        R.w[r * k + lane] = w;
      }
      if (lane == 0) {
        R.gamma[r] = gm;
        if (!ok) atomicExch(p.ctrl + kStatus, (unsigned)MOE_ERR_DEVICE_CHECK);
      }
    }
  }
  __syncthreads();
  tc_group(te, R);
  TC_STAMP(4);
  const int U = R.n_active;
  // this CTA's share of the active experts' (and the shared expert's) down rows into L2
  if (warp == kWarps - 1) {
    const size_t prb_i = packed_row_bytes(FMT, p.I);
    const size_t prb_s = p.has_shared ? packed_row_bytes(FMT, p.S) : 0;
    const size_t total = ((size_t)U * prb_i + prb_s) * (size_t)p.h;
    if (total <= (size_t)pl.l2_prefetch_cap) {
      const int r0 = (int)((long long)cta * p.h / G), r1 = (int)((long long)(cta + 1) * p.h / G);
      for (int sl = lane; sl < U + p.has_shared && r1 > r0; sl += 32) {
        const bool sh = sl == U;
        const MatDev D = pick_mat(sh, p.sd, p.rd);
        const int e = sh ? 0 : R.slot_e[sl];
        const size_t prb = sh ? prb_s : prb_i;
        prefetch_l2_bulk(D.packed + (size_t)e * D.estride + (size_t)r0 * prb,
                         (size_t)(r1 - r0) * prb);
        const int K = sh ? p.S : p.I;
        const size_t srb = FMT == MOE_FMT_Q4_AFFINE_G64 ? (size_t)(K / 64) * 2
                           : FMT == MOE_FMT_NVFP4        ? (size_t)(K / 16)
                           : FMT == MOE_FMT_MXFP4        ? (size_t)(K / 32)
                                                         : 0;
        if (srb) {
          prefetch_l2_lines(D.scales + (size_t)e * D.sstride + (size_t)r0 * srb,
                            (size_t)(r1 - r0) * srb);
          if (FMT == MOE_FMT_Q4_AFFINE_G64)
            prefetch_l2_lines(D.biases + (size_t)e * D.sstride + (size_t)r0 * srb,
                              (size_t)(r1 - r0) * srb);
        }
      }
    }
  }
  SlotView sv;
  sv.slot_e = R.slot_e;
  sv.slot_beg = R.slot_beg;
  sv.slot_n = R.slot_n;
  sv.sorted = R.sorted;
  sv.wts = R.w;
  sv.tp = R.tp;
  sv.gamma = R.gamma;
  sv.U = U;
  TC_STAMP(13);
  build_maps<FMT, NTG>(p, tx, sv, s_gu, s_dn, warp);
  TC_STAMP(14);
  __syncthreads();
  TC_STAMP(12);

  // ---- D: gate/up -------------------------------------------------------------------------------
  gate_up_phase<FMT, NTG>(p, tx, sv, s_gu, &s_next[0], tc_ring + warp * ring_bytes<FMT, NTG>());
  TC_STAMP(10);  // warp 0's own share done
#ifdef MOE_PHASE_TIMERS
  __syncthreads();
#endif
  TC_STAMP(9);
  if (cta == 0) {  // the routing and grouping for read-back
    for (int t = tid; t < te; t += kThreads) {
      p.idx[t] = R.idx[t];
      p.wts[t] = R.w[t];
      p.sorted_pairs[t] = R.sorted[t];
      p.token_to_perm[t] = R.tp[t];
    }
    for (int e = tid; e <= p.E; e += kThreads) {
      int less = 0;
      for (int q = 0; q < te; ++q) less += R.idx[q] < e;
      p.offsets[e] = less;
    }
    for (int a = tid; a < U; a += kThreads) p.active[a] = R.slot_e[a];
    if (tid == 0) *p.active_count = U;
    for (int r = tid; r < m; r += kThreads) p.gamma[r] = R.gamma[r];
  }
  TC_STAMP(5);
  pdl_launch_dependents();

  // ---- E: down + blend (each slot's down jobs start once its gate/up jobs have all counted) ---
  down_phase<FMT, NTG>(p, tx, sv, s_dn, s_gu, pl.spin_limit, pl.bar_extra, &s_next[1],
                       tc_ring + warp * ring_bytes<FMT, NTG>());
  TC_STAMP(11);  // warp 0's own share done
#ifdef MOE_PHASE_TIMERS
  __syncthreads();
#endif
  TC_STAMP(8);
#ifdef MOE_PHASE_TIMERS
  __syncthreads();
#endif
  TC_STAMP_FLUSH();
}

// ---- the multi-kernel path: router, gate/up, down -------------------------------------------------

// Router logits (one CTA per router row), operand activations and zeroed tickets (all CTAs);
// the CTA finishing last routes every row, groups the pairs and writes the slot tables.
template <int FMT>
__global__ void __launch_bounds__(kRouterThreads) tc_router_kernel(
    const __grid_constant__ Params p, const __grid_constant__ TcExtra tx, int* slot_beg,
    int* slot_n) {
  pdl_launch_dependents();
  const int erow = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t row_bytes = (size_t)p.h * 2;
  const int nch = (int)(row_bytes / 16);
  const uint8_t* wrow = erow < p.E ? (const uint8_t*)p.router_w + (size_t)erow * row_bytes
                                   : (const uint8_t*)p.shared_gate_w;
  __shared__ int s_last;
  __shared__ int s_idx[kMaxPairs];
  for (int r = warp; r < p.m; r += kRouterThreads / 32) {
    const uint8_t* xr = (const uint8_t*)p.x + (size_t)r * row_bytes;
    const float acc = router_dot_gx<true>(wrow, xr, nch);
    if (lane == 0) p.logits[(size_t)r * (p.E + 1) + erow] = acc;
  }
  convert_x<FMT>(p, tx, blockIdx.x * kRouterThreads + tid, gridDim.x * kRouterThreads);
  for (int i = blockIdx.x * kRouterThreads + tid; i < tx.tk_words; i += gridDim.x * kRouterThreads)
    tx.tk_gu[i] = 0u;
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const unsigned t = atomicAdd(p.ctrl + kRouterTicket, 1u);
    s_last = (t == gridDim.x - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const RouteCfg rc = route_cfg(p);
  for (int r = warp; r < p.m; r += kRouterThreads / 32) {
    int id;
    float w, gm;
    const bool ok = route_row(rc, r, p.expert_bias, id, w, gm);
    if (lane < p.k) {
      p.idx[r * p.k + lane] = id;
      p.wts[r * p.k + lane] = w;
      s_idx[r * p.k + lane] = id;
    }
    if (lane == 0) {
      p.gamma[r] = gm;
      if (!ok) atomicExch(p.ctrl + kStatus, (unsigned)MOE_ERR_DEVICE_CHECK);
    }
  }
  __syncthreads();
  group_pairs(p, s_idx);
  __syncthreads();
  const int U = *(volatile int*)p.active_count;
  for (int a = tid; a < U; a += kRouterThreads) {
    const int e = p.active[a];
    slot_beg[a] = p.offsets[e];
    slot_n[a] = p.offsets[e + 1] - p.offsets[e];
  }
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    p.ctrl[kRouterTicket] = 0u;
  }
}

__device__ __forceinline__ SlotView global_slots(const Params& p, const int* slot_beg,
                                                 const int* slot_n) {
  SlotView sv;
  sv.slot_e = p.active;
  sv.slot_beg = slot_beg;
  sv.slot_n = slot_n;
  sv.sorted = p.sorted_pairs;
  sv.wts = p.wts;
  sv.tp = p.token_to_perm;
  sv.gamma = p.gamma;
  sv.U = *(volatile int*)p.active_count;
  return sv;
}

template <int FMT, int NTG>
__global__ void __launch_bounds__(32 * tc_warps<FMT, NTG>(), 1) tc_gate_up_kernel(
    const __grid_constant__ Params p, const __grid_constant__ TcExtra tx, const int* slot_beg,
    const int* slot_n) {
  extern __shared__ __align__(16) uint8_t tc_ring[];
  __shared__ PhaseMap s_gu, s_dn;
  __shared__ int s_next;
  pdl_launch_dependents();
  pdl_wait();
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) s_next = 0;
  const SlotView sv = global_slots(p, slot_beg, slot_n);
  build_maps<FMT, NTG>(p, tx, sv, s_gu, s_dn, warp);
  __syncthreads();
  gate_up_phase<FMT, NTG>(p, tx, sv, s_gu, &s_next, tc_ring + warp * ring_bytes<FMT, NTG>());
}

template <int FMT, int NTG>
__global__ void __launch_bounds__(32 * tc_warps<FMT, NTG>(), 1) tc_down_kernel(
    const __grid_constant__ Params p, const __grid_constant__ TcExtra tx, const int* slot_beg,
    const int* slot_n) {
  extern __shared__ __align__(16) uint8_t tc_ring[];
  __shared__ PhaseMap s_gu, s_dn;
  __shared__ int s_next;
  pdl_launch_dependents();
  pdl_wait();
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) s_next = 0;
  const SlotView sv = global_slots(p, slot_beg, slot_n);
  build_maps<FMT, NTG>(p, tx, sv, s_gu, s_dn, warp);
  __syncthreads();
  // the gate/up kernel has finished (programmatic-launch wait): every slot is ready at once
  down_phase<FMT, NTG>(p, tx, sv, s_dn, s_gu, kChainSpinLimit, 0u, &s_next,
                       tc_ring + warp * ring_bytes<FMT, NTG>());
}

}  // namespace tc
}  // namespace moe
