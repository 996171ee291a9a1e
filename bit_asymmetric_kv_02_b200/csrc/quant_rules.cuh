// The exact code rule of the method, shared by the quantize kernels and the in-launch flush of the
// decode step (sm_100a).
//
// Method: KIVI explainer page "ICML 2024論文解説: KIVI — チューニング不要のKVキャッシュ2bit非対称量子化",
//   section 量子化アルゴリズム (Q equation, s/z equation).
// s = fp16_rn((max - min)/(2^b - 1)) is formed in fp64 (exact range, one rounding), z = min.  A code
// is RNE of the exact rational (x - z)/s with the stored s and z: computed in fp32 as (x - z) * (1/s),
// whose absolute error is below 2^-18 for every reachable value, and re-decided with an fp64
// division when the fp32 value lies within 2^-12 of a half-integer, where that division is exact.
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


}  // namespace
}  // namespace kivi
