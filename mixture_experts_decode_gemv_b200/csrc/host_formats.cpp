// Host-side pack / quantise / dequantise helpers of the C ABI (no GPU needed).
//
// Minifloat encoders are written from the format definitions: IEEE binary16 (5 exponent bits,
// bias 15, with infinities), OCP FP8 E4M3 (4 exponent bits, bias 7, no infinity, max 448) and OCP
// FP4 E2M1 (2 exponent bits, bias 1, max 6). All round to nearest, ties to even. MXFP4 block
// scales are OCP E8M0 (a biased power of two).
#include <cmath>
#include <cstdint>
#include <cstring>
#include <algorithm>

#include "../../include/moe_decode.h"

namespace moe_host {

struct Minifloat {
  int ebits, mbits, bias;
  double max_finite;
  bool saturate;      // true: out-of-range magnitudes become max_finite (no infinity)
  uint32_t inf_code;  // magnitude code of +inf when !saturate
};

static const Minifloat kF16 = {5, 10, 15, 65504.0, false, 0x7C00u};
static const Minifloat kE4M3 = {4, 3, 7, 448.0, true, 0u};
static const Minifloat kE2M1 = {2, 1, 1, 6.0, true, 0u};

// Magnitude code (no sign bit) of the representable value nearest to a >= 0.
static uint32_t encode_magnitude(double a, const Minifloat& f) {
  const double top = std::ldexp(1.0, f.mbits + 1);
  const double lead = std::ldexp(1.0, f.mbits);
  if (!(a > 0.0)) return 0u;
  if (a > f.max_finite) {
    // the rounding midpoint above max_finite decides overflow for IEEE formats
    const int emax = (int)std::floor(std::log2(f.max_finite));
    const double half_ulp = std::ldexp(1.0, emax - f.mbits - 1);
    if (f.saturate || a < f.max_finite + half_ulp) a = f.max_finite;
    else return f.inf_code;
  }
  int e = (int)std::floor(std::log2(a));
  const int emin = 1 - f.bias;
  if (e < emin) e = emin;
  double n = std::nearbyint(std::ldexp(a, f.mbits - e));  // a / 2^(e - mbits), ties to even
  if (n >= top) {  // rounded up into the next binade
    n = lead;
    e += 1;
  }
  if (n < lead) return (uint32_t)n;  // subnormal (exponent field 0)
  return ((uint32_t)(e + f.bias) << f.mbits) | (uint32_t)(n - lead);
}

static double decode_magnitude(uint32_t code, const Minifloat& f) {
  const uint32_t ef = code >> f.mbits;
  const uint32_t mf = code & ((1u << f.mbits) - 1u);
  if (ef == 0) return std::ldexp((double)mf, 1 - f.bias - f.mbits);
  return std::ldexp(1.0 + std::ldexp((double)mf, -f.mbits), (int)ef - f.bias);
}

static uint16_t f32_to_f16(float x) {
  uint32_t u;
  std::memcpy(&u, &x, 4);
  const uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
  if ((u & 0x7F800000u) == 0x7F800000u) return sign | ((u & 0x7FFFFFu) ? 0x7E00 : 0x7C00);
  return sign | (uint16_t)encode_magnitude(std::fabs((double)x), kF16);
}

static double f16_to_double(uint16_t h) {
  const uint32_t mag = h & 0x7FFFu;
  double v;
  if ((mag >> 10) == 31) v = (mag & 0x3FF) ? NAN : INFINITY;
  else v = decode_magnitude(mag, kF16);
  return (h & 0x8000u) ? -v : v;
}

static uint8_t f64_to_e4m3(double x) {
  const uint8_t sign = std::signbit(x) ? 0x80 : 0x00;
  return sign | (uint8_t)encode_magnitude(std::fabs(x), kE4M3);
}

static double e4m3_to_double(uint8_t c) {
  const uint32_t mag = c & 0x7Fu;
  double v = (mag == 0x7Fu) ? NAN : decode_magnitude(mag, kE4M3);
  return (c & 0x80u) ? -v : v;
}

static uint8_t f64_to_e2m1(double x) {
  const uint8_t sign = std::signbit(x) ? 0x8 : 0x0;
  return sign | (uint8_t)encode_magnitude(std::fabs(x), kE2M1);
}

static double e2m1_to_double(uint8_t c) {
  double v = decode_magnitude(c & 0x7u, kE2M1);
  return (c & 0x8u) ? -v : v;
}

// OCP E8M0: an unsigned biased exponent, value 2^(c - 127); 255 encodes NaN.
static double e8m0_to_double(uint8_t c) { return c == 0xFF ? NAN : std::ldexp(1.0, (int)c - 127); }

static uint16_t f32_to_bf16(float x) {
  uint32_t u;
  std::memcpy(&u, &x, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x7FFFFFu)) return (uint16_t)((u >> 16) | 0x40u);
  const uint32_t lsb = (u >> 16) & 1u;
  return (uint16_t)((u + 0x7FFFu + lsb) >> 16);
}

static float bf16_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

}  // namespace moe_host

using namespace moe_host;

extern "C" int moe_packed_bytes(int format, int n, int k, size_t* packed, size_t* scales,
                                size_t* biases) {
  if (!packed || !scales || !biases) return MOE_ERR_NULL_POINTER;
  if (n <= 0 || k <= 0) return MOE_ERR_BAD_SHAPE;
  const size_t nk = (size_t)n * (size_t)k;
  switch (format) {
    case MOE_FMT_F32: *packed = 4 * nk; *scales = 0; *biases = 0; return MOE_OK;
    case MOE_FMT_BF16: *packed = 2 * nk; *scales = 0; *biases = 0; return MOE_OK;
    case MOE_FMT_Q4_AFFINE_G64:
      if (k % 64) return MOE_ERR_BAD_SHAPE;
      *packed = nk / 2; *scales = 2 * (nk / 64); *biases = 2 * (nk / 64); return MOE_OK;
    case MOE_FMT_NVFP4:
      if (k % 32) return MOE_ERR_BAD_SHAPE;
      *packed = nk / 2; *scales = nk / 16; *biases = 0; return MOE_OK;
    case MOE_FMT_MXFP4:
      if (k % 32) return MOE_ERR_BAD_SHAPE;
      *packed = nk / 2; *scales = nk / 32; *biases = 0; return MOE_OK;
    case MOE_FMT_FP8_E4M3:
      if (k % 16) return MOE_ERR_BAD_SHAPE;
      *packed = nk; *scales = 0; *biases = 0; return MOE_OK;
    default: return MOE_ERR_BAD_FORMAT;
  }
}

extern "C" int moe_pack_bf16(const float* w, int64_t count, uint16_t* out) {
  if (!w || !out) return MOE_ERR_NULL_POINTER;
  if (count < 0) return MOE_ERR_BAD_SHAPE;
  for (int64_t i = 0; i < count; ++i) out[i] = f32_to_bf16(w[i]);
  return MOE_OK;
}

extern "C" int moe_quantize_q4_affine(const float* w, int n, int k, uint8_t* packed,
                                      uint16_t* scales, uint16_t* biases) {
  if (!w || !packed || !scales || !biases) return MOE_ERR_NULL_POINTER;
  if (n <= 0 || k <= 0 || k % 64) return MOE_ERR_BAD_SHAPE;
  const int groups = k / 64;
  for (int r = 0; r < n; ++r) {
    const float* row = w + (size_t)r * k;
    uint8_t* prow = packed + (size_t)r * (k / 2);
    for (int g = 0; g < groups; ++g) {
      const float* grp = row + g * 64;
      float lo = grp[0], hi = grp[0];
      for (int j = 1; j < 64; ++j) {
        lo = std::min(lo, grp[j]);
        hi = std::max(hi, grp[j]);
      }
      const uint16_t s16 = f32_to_f16((float)(((double)hi - (double)lo) / 15.0));
      const uint16_t b16 = f32_to_f16(lo);
      scales[(size_t)r * groups + g] = s16;
      biases[(size_t)r * groups + g] = b16;
      const double sv = f16_to_double(s16), bv = f16_to_double(b16);
      for (int j = 0; j < 64; j += 2) {
        uint8_t q2[2];
        for (int t = 0; t < 2; ++t) {
          double q = sv > 0.0 ? std::nearbyint(((double)grp[j + t] - bv) / sv) : 0.0;
          q = std::min(15.0, std::max(0.0, q));
          q2[t] = (uint8_t)q;
        }
        prow[(g * 64 + j) / 2] = (uint8_t)(q2[0] | (q2[1] << 4));
      }
    }
  }
  return MOE_OK;
}

extern "C" int moe_quantize_nvfp4(const float* w, int n, int k, uint8_t* packed, uint8_t* scales,
                                  float* tensor_scale) {
  if (!w || !packed || !scales || !tensor_scale) return MOE_ERR_NULL_POINTER;
  if (n <= 0 || k <= 0 || k % 32) return MOE_ERR_BAD_SHAPE;
  double amax = 0.0;
  const size_t nk = (size_t)n * k;
  for (size_t i = 0; i < nk; ++i) amax = std::max(amax, std::fabs((double)w[i]));
  const float ts = amax > 0.0 ? (float)(amax / (6.0 * 448.0)) : 1.0f;
  *tensor_scale = ts;
  const int blocks = k / 16;
  for (int r = 0; r < n; ++r) {
    const float* row = w + (size_t)r * k;
    uint8_t* prow = packed + (size_t)r * (k / 2);
    for (int b = 0; b < blocks; ++b) {
      const float* blk = row + b * 16;
      double bmax = 0.0;
      for (int j = 0; j < 16; ++j) bmax = std::max(bmax, std::fabs((double)blk[j]));
      const uint8_t sc = f64_to_e4m3(bmax / 6.0 / (double)ts);
      scales[(size_t)r * blocks + b] = sc;
      const double denom = e4m3_to_double(sc) * (double)ts;
      for (int j = 0; j < 16; j += 2) {
        uint8_t c2[2];
        for (int t = 0; t < 2; ++t)
          c2[t] = denom > 0.0 ? f64_to_e2m1((double)blk[j + t] / denom) : 0;
        prow[(b * 16 + j) / 2] = (uint8_t)(c2[0] | (c2[1] << 4));
      }
    }
  }
  return MOE_OK;
}

extern "C" int moe_quantize_mxfp4(const float* w, int n, int k, uint8_t* packed,
                                  uint8_t* scales) {
  if (!w || !packed || !scales) return MOE_ERR_NULL_POINTER;
  if (n <= 0 || k <= 0 || k % 32) return MOE_ERR_BAD_SHAPE;
  const int blocks = k / 32;
  for (int r = 0; r < n; ++r) {
    const float* row = w + (size_t)r * k;
    uint8_t* prow = packed + (size_t)r * (k / 2);
    for (int b = 0; b < blocks; ++b) {
      const float* blk = row + b * 32;
      double bmax = 0.0;
      for (int j = 0; j < 32; ++j) bmax = std::max(bmax, std::fabs((double)blk[j]));
      int x = bmax > 0.0 ? (int)std::floor(std::log2(bmax)) - 2 : 0;
      x = std::min(127, std::max(-127, x));
      scales[(size_t)r * blocks + b] = (uint8_t)(x + 127);
      for (int j = 0; j < 32; j += 2) {
        uint8_t c2[2];
        for (int t = 0; t < 2; ++t) c2[t] = f64_to_e2m1(std::ldexp((double)blk[j + t], -x));
        prow[(b * 32 + j) / 2] = (uint8_t)(c2[0] | (c2[1] << 4));
      }
    }
  }
  return MOE_OK;
}

extern "C" int moe_quantize_fp8_e4m3(const float* w, int n, int k, uint8_t* packed,
                                     float* tensor_scale) {
  if (!w || !packed || !tensor_scale) return MOE_ERR_NULL_POINTER;
  if (n <= 0 || k <= 0 || k % 16) return MOE_ERR_BAD_SHAPE;
  const size_t nk = (size_t)n * k;
  double amax = 0.0;
  for (size_t i = 0; i < nk; ++i) amax = std::max(amax, std::fabs((double)w[i]));
  const float ts = amax > 0.0 ? (float)(amax / 448.0) : 1.0f;
  *tensor_scale = ts;
  for (size_t i = 0; i < nk; ++i) packed[i] = f64_to_e4m3((double)w[i] / (double)ts);
  return MOE_OK;
}

extern "C" int moe_dequantize(int format, const void* packed, const void* scales,
                              const void* biases, const float* tensor_scale, int n, int k,
                              float* out) {
  if (!packed || !out) return MOE_ERR_NULL_POINTER;
  if (n <= 0 || k <= 0) return MOE_ERR_BAD_SHAPE;
  const size_t nk = (size_t)n * k;
  switch (format) {
    case MOE_FMT_F32:
      std::memcpy(out, packed, nk * 4);
      return MOE_OK;
    case MOE_FMT_BF16: {
      const uint16_t* p = (const uint16_t*)packed;
      for (size_t i = 0; i < nk; ++i) out[i] = bf16_to_f32(p[i]);
      return MOE_OK;
    }
    case MOE_FMT_Q4_AFFINE_G64: {
      if (!scales || !biases) return MOE_ERR_NULL_POINTER;
      if (k % 64) return MOE_ERR_BAD_SHAPE;
      const uint8_t* p = (const uint8_t*)packed;
      const uint16_t* s = (const uint16_t*)scales;
      const uint16_t* b = (const uint16_t*)biases;
      for (int r = 0; r < n; ++r)
        for (int j = 0; j < k; ++j) {
          const uint8_t byte = p[(size_t)r * (k / 2) + j / 2];
          const int q = (j & 1) ? (byte >> 4) : (byte & 0xF);
          const size_t g = (size_t)r * (k / 64) + j / 64;
          out[(size_t)r * k + j] = (float)(f16_to_double(s[g]) * q + f16_to_double(b[g]));
        }
      return MOE_OK;
    }
    case MOE_FMT_NVFP4: {
      if (!scales || !tensor_scale) return MOE_ERR_NULL_POINTER;
      if (k % 32) return MOE_ERR_BAD_SHAPE;
      const uint8_t* p = (const uint8_t*)packed;
      const uint8_t* s = (const uint8_t*)scales;
      const double ts = (double)tensor_scale[0];
      for (int r = 0; r < n; ++r)
        for (int j = 0; j < k; ++j) {
          const uint8_t byte = p[(size_t)r * (k / 2) + j / 2];
          const uint8_t c = (j & 1) ? (byte >> 4) : (byte & 0xF);
          const double sc = e4m3_to_double(s[(size_t)r * (k / 16) + j / 16]);
          out[(size_t)r * k + j] = (float)(e2m1_to_double(c) * sc * ts);
        }
      return MOE_OK;
    }
    case MOE_FMT_MXFP4: {
      if (!scales) return MOE_ERR_NULL_POINTER;
      if (k % 32) return MOE_ERR_BAD_SHAPE;
      const uint8_t* p = (const uint8_t*)packed;
      const uint8_t* s = (const uint8_t*)scales;
      for (int r = 0; r < n; ++r)
        for (int j = 0; j < k; ++j) {
          const uint8_t byte = p[(size_t)r * (k / 2) + j / 2];
          const uint8_t c = (j & 1) ? (byte >> 4) : (byte & 0xF);
          const double sc = e8m0_to_double(s[(size_t)r * (k / 32) + j / 32]);
          out[(size_t)r * k + j] = (float)(e2m1_to_double(c) * sc);
        }
      return MOE_OK;
    }
    case MOE_FMT_FP8_E4M3: {
      if (!tensor_scale) return MOE_ERR_NULL_POINTER;
      if (k % 16) return MOE_ERR_BAD_SHAPE;
      const uint8_t* p = (const uint8_t*)packed;
      const double ts = (double)tensor_scale[0];
      for (size_t i = 0; i < nk; ++i) out[i] = (float)(e4m3_to_double(p[i]) * ts);
      return MOE_OK;
    }
    default:
      return MOE_ERR_BAD_FORMAT;
  }
}
