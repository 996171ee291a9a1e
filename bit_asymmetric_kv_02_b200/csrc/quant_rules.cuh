// The exact code rule of the method, shared by the quantize kernels and the in-launch flush of the
// decode step (sm_100a).
//
// Method: KIVI explainer page "ICML 2024論文解説: KIVI — チューニング不要のKVキャッシュ2bit非対称量子化",
//   section 量子化アルゴリズム (Q equation, s/z equation).
// s = fp16_rn((max - min)/(2^b - 1)) is formed in fp64 (exact range, one rounding), z = min.  A code
// is RNE of the exact rational (x - z)/s with the stored s and z: computed in fp32 as (x - z) * (1/s),
// whose absolute error is below 2^-18 for every reachable value, and re-decided with an fp64
// division when the fp32 value lies within 2^-12 of a half-integer, where that division is exact.
// At 2 bits the same code is a count of three fp16 thresholds (make_thresh2 / codes2_h2), which
// costs a few packed fp16 comparisons per pair of elements.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

#include "common.cuh"

namespace kivi {
namespace {

__device__ __forceinline__ void minmax8(uint4 v, float& lo, float& hi) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a = h2f(static_cast<uint16_t>(w[i] & 0xFFFFu));
    const float b = h2f(static_cast<uint16_t>(w[i] >> 16));
    lo = fminf(lo, fminf(a, b));
    hi = fmaxf(hi, fmaxf(a, b));
  }
}

struct GroupParams {
  float inv_s;     // 1/s in fp32 (0 when s == 0)
  float zf;        // z as fp32
  uint16_t s_bits, z_bits;
};

// s, z of one group from its fp16 extremes (section 量子化アルゴリズム, s/z equation).
__device__ __forceinline__ GroupParams make_group(float lo, float hi, int levels) {
  GroupParams g;
  const double range = static_cast<double>(hi) - static_cast<double>(lo);  // exact
  g.s_bits = f64_to_h_rn(range / static_cast<double>(levels));
  g.zf = __fadd_rn(lo, 0.0f);  // a zero minimum is stored as +0
  g.z_bits = __half_as_ushort(__float2half_rn(g.zf));  // lo is an fp16 value: exact
  const float s = h2f(g.s_bits);
  g.inv_s = s > 0.f ? 1.0f / s : 0.f;
  return g;
}

// Group parameters from a stored (s, z) pair (the prefix-group prefill stores them first).
__device__ __forceinline__ GroupParams group_from_stored(uint16_t s_bits, uint16_t z_bits) {
  GroupParams g;
  g.s_bits = s_bits;
  g.z_bits = z_bits;
  g.zf = h2f(z_bits);
  const float s = h2f(s_bits);
  g.inv_s = s > 0.f ? 1.0f / s : 0.f;
  return g;
}

// Q of one element (section 量子化アルゴリズム, Q equation) with the stored fp16 s and z, taken
// exactly: the fp64 quotient decides (used near ties only).
__device__ __noinline__ uint32_t quantize_exact(float x, const GroupParams& g, int levels) {
  const double r64 = (static_cast<double>(x) - static_cast<double>(g.zf)) / static_cast<double>(h2f(g.s_bits));
  return min(static_cast<uint32_t>(rint(r64)), static_cast<uint32_t>(levels));
}

// Q of two elements at once with packed fp32 pairs.  r = (x - z) * (1/s) has absolute error below
// 2^-18 for every reachable r (< 24); adding 1.5 * 2^23 rounds it to the nearest integer, ties to
// even, exactly like rint.  An element whose r lies within 2^-12 of a half-integer is decided
// again by quantize_exact.
__device__ __forceinline__ void quantize_pair(uint32_t hx2, const GroupParams& g, int levels, uint32_t& qa,
                                              uint32_t& qb) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  const float2 x = __half22float2(*reinterpret_cast<const __half2*>(&hx2));
  const float2 r = __fmul2_rn(__fadd2_rn(x, make_float2(-g.zf, -g.zf)), make_float2(g.inv_s, g.inv_s));
  const float2 t = __fadd2_rn(r, make_float2(kMagic, kMagic));
  const float2 d = __fadd2_rn(r, __fadd2_rn(make_float2(kMagic, kMagic), make_float2(-t.x, -t.y)));
  qa = min(__float_as_uint(t.x) - 0x4B400000u, static_cast<uint32_t>(levels));
  qb = min(__float_as_uint(t.y) - 0x4B400000u, static_cast<uint32_t>(levels));
  if (fabsf(d.x) > 0.499755859375f) qa = quantize_exact(x.x, g, levels);  // within 2^-12 of a tie
  if (fabsf(d.y) > 0.499755859375f) qb = quantize_exact(x.y, g, levels);
  if (g.inv_s == 0.f) qa = qb = 0u;
}

__device__ __forceinline__ uint32_t comp4(const uint4& v, int i) {
  return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

// ---- 2 bits: the code as a count of thresholds ----------------------------------------------
// For s > 0, Q(x) = clamp(rint((x - z)/s), 0, 3) with ties to even is [r > 1/2] + [r >= 3/2] +
// [r > 5/2], r = (x - z)/s, i.e. [x > T0] + [x >= T1] + [x > T2] with T_k = z + (k + 1/2) s.  T_k is
// exact in fp64.  Over fp16 x, x > T equals x > (largest fp16 <= T) and x >= T equals
// x > (largest fp16 < T), so three strict fp16 comparisons decide the code exactly; s = 0 (all
// codes 0) uses +inf.
struct Thresh2 {
  uint32_t t[3];  // each threshold in both halves of a half2
};

__device__ __forceinline__ uint16_t f64_to_h_rd(double x) {
  uint16_t r;
  asm("cvt.rm.f16.f64 %0, %1;" : "=h"(r) : "d"(x));
  return r;
}
// The largest fp16 below the finite fp16 h.
__device__ __forceinline__ uint16_t h_below(uint16_t h) {
  if ((h & 0x7FFFu) == 0) return 0x8001u;  // below +-0: the negative subnormal closest to 0
  return (h & 0x8000u) ? static_cast<uint16_t>(h + 1) : static_cast<uint16_t>(h - 1);
}

__device__ Thresh2 make_thresh2(const GroupParams& g) {
  Thresh2 t;
  const double s = static_cast<double>(h2f(g.s_bits)), z = static_cast<double>(g.zf);
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    uint16_t h = 0x7C00u;  // +inf
    if (s > 0.0) {
      const double T = z + (k + 0.5) * s;  // exact
      h = f64_to_h_rd(T);
      if (k == 1 && static_cast<double>(h2f(h)) == T) h = h_below(h);
    }
    t.t[k] = static_cast<uint32_t>(h) * 0x00010001u;
  }
  return t;
}

// Codes of one half2 as the half2 (1024 + c0, 1024 + c1): byte 0 holds c0 and byte 2 holds c1.
__device__ __forceinline__ uint32_t codes2_h2(uint32_t x2, const Thresh2& t) {
  const __half2 x = *reinterpret_cast<const __half2*>(&x2);
  const __half2 t0 = *reinterpret_cast<const __half2*>(&t.t[0]);
  const __half2 t1 = *reinterpret_cast<const __half2*>(&t.t[1]);
  const __half2 t2 = *reinterpret_cast<const __half2*>(&t.t[2]);
  const __half2 c = __hadd2(__hadd2(__hgt2(x, t0), __hgt2(x, t1)), __hadd2(__hgt2(x, t2), __float2half2_rn(1024.f)));
  return *reinterpret_cast<const uint32_t*>(&c);
}

// Four 2-bit codes held one per byte -> an 8-bit field (byte i at bits 2 i).  The product with
// 2^24 + 2^18 + 2^12 + 2^6 moves byte i to bit 24 + 2 i; every other partial product lands below
// bit 24 (their sum stays below 2^24) or above bit 31.
__device__ __forceinline__ uint32_t gather4x2(uint32_t bytes) { return (bytes * 0x01041040u) >> 24; }

// 16-bit codes of the 8 channels of one token row, channel 8 c + j at bits 2 j.
__device__ __forceinline__ uint32_t row_codes2(const uint4& v, const Thresh2& t) {
  const uint32_t h0 = codes2_h2(v.x, t), h1 = codes2_h2(v.y, t), h2 = codes2_h2(v.z, t), h3 = codes2_h2(v.w, t);
  return gather4x2(__byte_perm(h0, h1, 0x6420)) | (gather4x2(__byte_perm(h2, h3, 0x6420)) << 8);
}

// Codes of the 8 channels of one token row of a tile (bits BITS * j for channel 8 c + j).
template <int BITS>
__device__ __forceinline__ uint32_t quantize_row8(const uint4& v, const GroupParams& g) {
  constexpr int L = (1 << BITS) - 1;
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t r = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    uint32_t qa, qb;
    quantize_pair(w[e], g, L, qa, qb);
    r += (qa << (BITS * 2 * e)) + (qb << (BITS * (2 * e + 1)));
  }
  return r;
}


}  // namespace
}  // namespace kivi
