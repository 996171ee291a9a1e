// Quantize + pack (prefill and flush) and residual append kernels.
//
// Method: KIVI explainer page "ICML 2024論文解説: KIVI — チューニング不要のKVキャッシュ2bit非対称量子化",
//   section 量子化アルゴリズム (Q, D and s/z equations), Per-Channel量子化（Key Cache）(K groups: g_k
//   consecutive channels), Per-Token量子化（Value Cache）(V groups: g_v consecutive tokens) and
//   残差バッファ（Residual Buffer）(the newest tokens stay fp16 until a block is flushed).
//
// One CTA quantizes one R-token block of K or of V for one (batch, KV head).  Two kernels:
//   R <= 512 (quantize_tiles_kernel): 2R threads hold the whole block in registers (one 128-bit
//     load per thread and token row), reduce the group minima / maxima, and emit the codes from
//     the same registers: the block is read from HBM exactly once.
//   R = 1024 (quantize_blocks_kernel): 256 threads; pass 1 reduces the extremes, pass 2 re-reads
//     the block from L2 and emits the codes.
// s = fp16_rn((max - min)/(2^b - 1)) is formed in fp64 (exact range, one rounding), z = min.
// A code is RNE of the exact rational (x - z)/s.  It is computed in fp32 as (x - z) * (1/s), whose
// relative error is below 3*2^-24, i.e. below 2^-18 absolute for every reachable value; when the
// fp32 value lies within 2^-12 of a half-integer the element is re-decided with an fp64 division,
// which is exact there.  Both sides of a parity test therefore take the exact decision.
#include <cstdint>

#include "common.cuh"
#include "kernels.h"
#include "quant_rules.cuh"

namespace kivi {

namespace {

constexpr int kThreads = 256;
constexpr int kChunks = kHeadDim / 8;  // uint4 chunks per token row

// ---------------------------------------------------------------------------------------------
// K block: groups of `gk` channels over all R tokens of the block.
// ---------------------------------------------------------------------------------------------
template <int BITS>
__device__ void quantize_k_block(const uint16_t* __restrict__ src, int R, int gk, uint32_t* __restrict__ codes,
                                 uint16_t* __restrict__ scale, uint16_t* __restrict__ zero, bool given) {
  constexpr int P = 32 / BITS;
  constexpr int L = (1 << BITS) - 1;
  __shared__ float red_lo[kThreads / 32][kChunks], red_hi[kThreads / 32][kChunks];
  __shared__ GroupParams grp[kHeadDim / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int chunk = tid % kChunks;
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
  if (given) {  // prefix groups: (s, z) already stored for this block
    if (tid < kHeadDim / gk) grp[tid] = group_from_stored(scale[tid], zero[tid]);
  } else {
    float lo = INFINITY, hi = -INFINITY;
    for (int t = tid / kChunks; t < R; t += kThreads / kChunks) minmax8(__ldg(s4 + t * kChunks + chunk), lo, hi);
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, 16));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, 16));
    if (lane < kChunks) {
      red_lo[warp][lane] = lo;
      red_hi[warp][lane] = hi;
    }
    __syncthreads();
    if (warp == 0) {
      // lanes 0..15: one chunk each, then combine the chunks of a group (gk/8 consecutive chunks)
      float a = INFINITY, b = -INFINITY;
      if (lane < kChunks) {
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) {
          a = fminf(a, red_lo[w][lane]);
          b = fmaxf(b, red_hi[w][lane]);
        }
      }
      const int cpg = gk / 8;  // chunks per group: 4, 8 or 16
      for (int off = 1; off < cpg; off <<= 1) {
        a = fminf(a, __shfl_xor_sync(0xffffffffu, a, off));
        b = fmaxf(b, __shfl_xor_sync(0xffffffffu, b, off));
      }
      if (lane < kChunks && lane % cpg == 0) {
        const int g = lane / cpg;
        GroupParams gp = make_group(a, b, L);
        grp[g] = gp;
        scale[g] = gp.s_bits;
        zero[g] = gp.z_bits;
      }
    }
  }
  __syncthreads();

  // pass 2: word (t, i) holds channels P*i + j at bits BITS*j; a word never straddles a group
  // (P <= 16 <= group_k)
  constexpr int WPT = kHeadDim / P;  // words per token
#pragma unroll 4
  for (int w = tid; w < R * WPT; w += kThreads) {
    const int t = w / WPT, i = w % WPT;
    const uint4* p = s4 + t * kChunks + (i * P) / 8;
    const GroupParams g = grp[(i * P) / gk];
    uint32_t word = 0;
#pragma unroll
    for (int c8 = 0; c8 < P / 8; ++c8) {
      const uint4 v = __ldg(p + c8);
      const uint32_t hw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {  // channels j, j + 1 of the word
        const int j = c8 * 8 + 2 * e;
        uint32_t qa, qb;
        quantize_pair(hw[e], g, L, qa, qb);
        word += (qa << (BITS * j)) + (qb << (BITS * (j + 1)));  // disjoint bit fields
      }
    }
    codes[w] = word;
  }
}

// ---------------------------------------------------------------------------------------------
// V block: groups of `gv` consecutive tokens over all channels.
// ---------------------------------------------------------------------------------------------
template <int BITS>
__device__ void quantize_v_block(const uint16_t* __restrict__ src, int R, int gv, uint32_t* __restrict__ codes,
                                 uint16_t* __restrict__ scale, uint16_t* __restrict__ zero) {
  constexpr int P = 32 / BITS;
  constexpr int L = (1 << BITS) - 1;
  constexpr int kMaxSlabs = 1024 / 16;
  __shared__ float slab_lo[kMaxSlabs], slab_hi[kMaxSlabs];
  __shared__ GroupParams grp[1024 / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint4* s4 = reinterpret_cast<const uint4*>(src);

  // pass 1: warp w reduces 16-row slabs 16w, 16w + 128, ... (a slab never straddles a V group
  // because gv is a multiple of 32)
  for (int slab = warp; slab < R / 16; slab += kThreads / 32) {
    float lo = INFINITY, hi = -INFINITY;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int t = slab * 16 + lane / kChunks + 2 * k;
      minmax8(__ldg(s4 + t * kChunks + (lane % kChunks)), lo, hi);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
    }
    if (lane == 0) {
      slab_lo[slab] = lo;
      slab_hi[slab] = hi;
    }
  }
  __syncthreads();
  const int ngroups = R / gv;
  if (tid < ngroups) {
    float a = INFINITY, b = -INFINITY;
    for (int s = tid * (gv / 16); s < (tid + 1) * (gv / 16); ++s) {
      a = fminf(a, slab_lo[s]);
      b = fmaxf(b, slab_hi[s]);
    }
    GroupParams gp = make_group(a, b, L);
    grp[tid] = gp;
    scale[tid] = gp.s_bits;
    zero[tid] = gp.z_bits;
  }
  __syncthreads();

  // pass 2: word (r, c) holds tokens P*r + j of channel c at bits BITS*j; a thread does two
  // adjacent channels with 32-bit loads.
  const uint32_t* s2 = reinterpret_cast<const uint32_t*>(src);
#pragma unroll 2
  for (int w2 = tid; w2 < (R / P) * (kHeadDim / 2); w2 += kThreads) {
    const int r = w2 / (kHeadDim / 2), cp = w2 % (kHeadDim / 2);
    const GroupParams g = grp[(r * P) / gv];
    uint32_t wa = 0, wb = 0;
#pragma unroll
    for (int j = 0; j < P; ++j) {  // channels 2 cp, 2 cp + 1 of token P r + j
      const uint32_t pair = __ldg(s2 + (r * P + j) * (kHeadDim / 2) + cp);
      uint32_t qa, qb;
      quantize_pair(pair, g, L, qa, qb);
      wa += qa << (BITS * j);
      wb += qb << (BITS * j);
    }
    codes[r * kHeadDim + 2 * cp] = wa;
    codes[r * kHeadDim + 2 * cp + 1] = wb;
  }
}

// Debug build: the job's source tokens and destination block lie inside their arrays.
__device__ __forceinline__ bool job_in_bounds(const QuantizeArgs& a, int blk) {
  return dbg_check(blk >= 0 && a.dst_blk0 + blk < a.capacity / a.residual &&
                   a.src_tok0 + static_cast<long long>(blk + 1) * a.residual <= a.src_tokens);
}

// Residual copy: tokens [res_tok0, res_tok0 + res_tokens) of the source -> residual slots 0..
__device__ void copy_residual(const QuantizeArgs& a, int bh) {
  if (!dbg_check(a.res_tok0 + a.res_tokens <= a.src_tokens && a.res_tokens <= a.residual)) return;
  const size_t src_tok = static_cast<size_t>(bh) * a.src_tokens + a.res_tok0;
  const uint4* ks = reinterpret_cast<const uint4*>(a.k_src + src_tok * kHeadDim);
  const uint4* vs = reinterpret_cast<const uint4*>(a.v_src + src_tok * kHeadDim);
  uint4* kd = reinterpret_cast<uint4*>(a.k_res + static_cast<size_t>(bh) * a.residual * kHeadDim);
  uint4* vd = reinterpret_cast<uint4*>(a.v_res + static_cast<size_t>(bh) * a.residual * kHeadDim);
  const int n = a.res_tokens * kChunks;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    kd[i] = __ldg(ks + i);
    vd[i] = __ldg(vs + i);
  }
}

// ---------------------------------------------------------------------------------------------
// Register-staged blocks (R <= 512): a CTA of 2R threads reads its block from HBM once.  Thread
// (token group tg, chunk c) holds tokens 8 tg .. 8 tg + 7 x channels 8 c .. 8 c + 7 in registers.
// Every K group (g_k >= 32 channels) and every V group (g_v >= 32 tokens) is a union of whole
// thread tiles, so a thread quantizes its 64 values with one (s, z).  Group extremes travel as the
// fp16 pair (min, -max), which one packed minimum reduces.
// ---------------------------------------------------------------------------------------------
constexpr int kTileTokens = 8;

__device__ __forceinline__ __half2 tile_min_negmax(const uint4 (&x)[kTileTokens]) {
  __half2 lo = *reinterpret_cast<const __half2*>(&x[0].x), hi = lo;
#pragma unroll
  for (int k = 0; k < kTileTokens; ++k) {
    const uint32_t w[4] = {x[k].x, x[k].y, x[k].z, x[k].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __half2 v = *reinterpret_cast<const __half2*>(&w[i]);
      lo = __hmin2(lo, v);
      hi = __hmax2(hi, v);
    }
  }
  return __halves2half2(__hmin(__low2half(lo), __high2half(lo)), __hneg(__hmax(__low2half(hi), __high2half(hi))));
}

__device__ __forceinline__ __half2 shfl_xor_h2(__half2 v, int off) {
  const uint32_t u = __shfl_xor_sync(0xffffffffu, *reinterpret_cast<uint32_t*>(&v), off);
  return *reinterpret_cast<const __half2*>(&u);
}

__device__ __forceinline__ GroupParams group_from_pair(__half2 m, int levels) {
  return make_group(__low2float(m), -__high2float(m), levels);
}

template <int BITS>
__device__ void quantize_k_tiles(const uint16_t* __restrict__ src, int R, int lg_gk, uint32_t* __restrict__ codes,
                                 uint16_t* __restrict__ scale, uint16_t* __restrict__ zero, bool given) {
  constexpr int L = (1 << BITS) - 1;
  __shared__ __half2 red[1024 / 32][kHeadDim / 32];
  __shared__ GroupParams grp[kHeadDim / 32];
  __shared__ Thresh2 thr[kHeadDim / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
  const int c = tid & 15, tg = tid >> 4;
  const uint4* s4 = reinterpret_cast<const uint4*>(src) + (tg * kTileTokens) * kChunks + c;
  uint4 x[kTileTokens];
#pragma unroll
  for (int k = 0; k < kTileTokens; ++k) x[k] = __ldg(s4 + k * kChunks);

  // K group of chunk c: chunks [cpg * g, cpg * (g + 1)), cpg = g_k / 8; the warp's two token
  // groups (lanes < 16 and >= 16) hold the same chunks
  const int lg_cpg = lg_gk - 3, ngk = kHeadDim >> lg_gk;
  if (!given) {
    __half2 m = tile_min_negmax(x);
    for (int off = 1; off < (1 << lg_cpg); off <<= 1) m = __hmin2(m, shfl_xor_h2(m, off));
    m = __hmin2(m, shfl_xor_h2(m, 16));
    if (lane < 16 && (c & ((1 << lg_cpg) - 1)) == 0) red[warp][c >> lg_cpg] = m;
    __syncthreads();
  }
  if (tid < ngk) {
    GroupParams gp;
    if (given) {  // prefix groups: (s, z) already stored for this block
      gp = group_from_stored(scale[tid], zero[tid]);
    } else {
      __half2 t = red[0][tid];
      for (int w = 1; w < nwarps; ++w) t = __hmin2(t, red[w][tid]);
      gp = group_from_pair(t, L);
      scale[tid] = gp.s_bits;
      zero[tid] = gp.z_bits;
    }
    if constexpr (BITS == 2)
      thr[tid] = make_thresh2(gp);
    else
      grp[tid] = gp;
  }
  __syncthreads();
  const int tok0 = tg * kTileTokens;
  if constexpr (BITS == 4) {  // K word c of a token is exactly the tile's 8 channels
    const GroupParams g = grp[c >> lg_cpg];
#pragma unroll
    for (int k = 0; k < kTileTokens; ++k) codes[(tok0 + k) * (kHeadDim / 8) + c] = quantize_row8<4>(x[k], g);
  } else {  // K word c / 2 of a token: chunk 2i in bits 0..15, chunk 2i + 1 in bits 16..31
    const Thresh2 t = thr[c >> lg_cpg];
    uint32_t h[kTileTokens];
#pragma unroll
    for (int k = 0; k < kTileTokens; ++k) h[k] = row_codes2(x[k], t);
    const bool odd = c & 1;
#pragma unroll
    for (int j = 0; j < 4; ++j) {  // the even chunk stores tokens 0..3 of the tile, the odd one 4..7
      const uint32_t other = __shfl_xor_sync(0xffffffffu, odd ? h[j] : h[4 + j], 1);
      const int k = odd ? 4 + j : j;
      const uint32_t word = odd ? (other | (h[4 + j] << 16)) : (h[j] | (other << 16));
      codes[(tok0 + k) * (kHeadDim / 16) + (c >> 1)] = word;
    }
  }
}

template <int BITS>
__device__ void quantize_v_tiles(const uint16_t* __restrict__ src, int R, int lg_gv, uint32_t* __restrict__ codes,
                                 uint16_t* __restrict__ scale, uint16_t* __restrict__ zero) {
  constexpr int L = (1 << BITS) - 1;
  __shared__ __half2 red[1024 / 32];
  __shared__ GroupParams grp[512 / 32];
  __shared__ Thresh2 thr[512 / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = tid & 15, tg = tid >> 4;
  const uint4* s4 = reinterpret_cast<const uint4*>(src) + (tg * kTileTokens) * kChunks + c;
  uint4 x[kTileTokens];
#pragma unroll
  for (int k = 0; k < kTileTokens; ++k) x[k] = __ldg(s4 + k * kChunks);

  // a warp's 16 tokens lie in one V group (g_v >= 32); group j spans warps [j g_v / 16, ...)
  __half2 m = tile_min_negmax(x);
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) m = __hmin2(m, shfl_xor_h2(m, off));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  const int ngv = R >> lg_gv, wpg = 1 << (lg_gv - 4);
  if (tid < ngv) {
    __half2 t = red[tid * wpg];
    for (int w = 1; w < wpg; ++w) t = __hmin2(t, red[tid * wpg + w]);
    const GroupParams gp = group_from_pair(t, L);
    if constexpr (BITS == 2)
      thr[tid] = make_thresh2(gp);
    else
      grp[tid] = gp;
    scale[tid] = gp.s_bits;
    zero[tid] = gp.z_bits;
  }
  __syncthreads();
  const int gv = (tg * kTileTokens) >> lg_gv;
  // codes of channel 8 c + e for the tile's 8 tokens, token k at bits BITS * k
  uint32_t col[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  if constexpr (BITS == 4) {
    const GroupParams g = grp[gv];
#pragma unroll
    for (int k = 0; k < kTileTokens; ++k) {
      const uint32_t w[4] = {x[k].x, x[k].y, x[k].z, x[k].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        uint32_t qa, qb;
        quantize_pair(w[e], g, L, qa, qb);
        col[2 * e] += qa << (BITS * k);
        col[2 * e + 1] += qb << (BITS * k);
      }
    }
  } else {
    // tokens 2a, 2a + 1 of channels 2e, 2e + 1 -> one word of four byte codes, then per channel
    // the bytes of tokens 0..3 and 4..7 -> two 8-bit fields
    const Thresh2 t = thr[gv];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      uint32_t A[4];
#pragma unroll
      for (int a2 = 0; a2 < 4; ++a2) {
        const uint32_t w0 = comp4(x[2 * a2], e), w1 = comp4(x[2 * a2 + 1], e);
        A[a2] = __byte_perm(codes2_h2(w0, t), codes2_h2(w1, t), 0x6240);
      }
      col[2 * e] = gather4x2(__byte_perm(A[0], A[1], 0x5410)) | (gather4x2(__byte_perm(A[2], A[3], 0x5410)) << 8);
      col[2 * e + 1] = gather4x2(__byte_perm(A[0], A[1], 0x7632)) | (gather4x2(__byte_perm(A[2], A[3], 0x7632)) << 8);
    }
  }
  if constexpr (BITS == 4) {  // V word (tg, 8 c + e) holds exactly the tile's 8 tokens
    uint4* dst = reinterpret_cast<uint4*>(codes + tg * kHeadDim + 8 * c);
    dst[0] = make_uint4(col[0], col[1], col[2], col[3]);
    dst[1] = make_uint4(col[4], col[5], col[6], col[7]);
  } else {  // V word (tg / 2, 8 c + e): the even token group in bits 0..15, the odd one in 16..31
    const bool odd = tg & 1;
    uint32_t word[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {  // the even token group stores channels 0..3, the odd one 4..7
      const uint32_t other = __shfl_xor_sync(0xffffffffu, odd ? col[e] : col[4 + e], 16);
      word[e] = odd ? (other | (col[4 + e] << 16)) : (col[e] | (other << 16));
    }
    *reinterpret_cast<uint4*>(codes + (tg >> 1) * kHeadDim + 8 * c + (odd ? 4 : 0)) =
        make_uint4(word[0], word[1], word[2], word[3]);
  }
}

// ---------------------------------------------------------------------------------------------
// Fine-grained groups with register tiles (R <= 256; section KVキャッシュの分布特性): the tiles of
// quantize_tiles_kernel, with one (s, z) per channel per g_k tokens for K and one per token per g_v
// channels for V.  K: a thread reduces each of its 8 channels over its 8 tokens, the warp's two token
// groups and then the g_k / 16 warps of the K group combine them (shared memory), and every thread
// forms the 8 pairs of its channels.  V: a thread reduces each of its 8 tokens over its 8 channels,
// then the g_v / 8 chunks of the channel group combine them by shuffles within the half warp.
// Codes follow the same exact rules (2 bits: thresholds per channel or per token; 4 bits:
// arithmetic with the fp64 re-decision near ties).
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ __half2 half2_of(const uint4& v, int i) {
  const uint32_t w = comp4(v, i);
  return *reinterpret_cast<const __half2*>(&w);
}
__device__ __forceinline__ uint32_t u32_of(__half2 h) { return *reinterpret_cast<const uint32_t*>(&h); }
__device__ __forceinline__ __half2 h2_from(uint32_t u) { return *reinterpret_cast<const __half2*>(&u); }

// Q of two elements with their own (s, z) (ga for the low half, gb for the high half).
__device__ __forceinline__ void quantize_pair2(uint32_t hx2, const GroupParams& ga, const GroupParams& gb, int levels,
                                               uint32_t& qa, uint32_t& qb) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  const float2 x = __half22float2(*reinterpret_cast<const __half2*>(&hx2));
  const float2 r = __fmul2_rn(__fadd2_rn(x, make_float2(-ga.zf, -gb.zf)), make_float2(ga.inv_s, gb.inv_s));
  const float2 t = __fadd2_rn(r, make_float2(kMagic, kMagic));
  const float2 d = __fadd2_rn(r, __fadd2_rn(make_float2(kMagic, kMagic), make_float2(-t.x, -t.y)));
  qa = min(__float_as_uint(t.x) - 0x4B400000u, static_cast<uint32_t>(levels));
  qb = min(__float_as_uint(t.y) - 0x4B400000u, static_cast<uint32_t>(levels));
  if (fabsf(d.x) > 0.499755859375f) qa = quantize_exact(x.x, ga, levels);  // within 2^-12 of a tie
  if (fabsf(d.y) > 0.499755859375f) qb = quantize_exact(x.y, gb, levels);
  if (ga.inv_s == 0.f) qa = 0u;
  if (gb.inv_s == 0.f) qb = 0u;
}

// The code rules of the channels of the block's K token groups, one array per field ([K token
// group][channel]), so that a thread reads its 8 channels' field with one 16-byte load: (s, z) bits,
// and the 2-bit thresholds (bits = 2) or 1/s and z (bits = 4).  Two channels' 16-bit fields in one
// word are exactly the (channel 2 i, 2 i + 1) pairs the codes and the scale rows use.
template <int BITS>
struct KRules {
  uint16_t s[256 / 32][kHeadDim], z[256 / 32][kHeadDim];
  uint16_t t[BITS == 2 ? 3 : 1][256 / 32][BITS == 2 ? kHeadDim : 1];
  float inv_s[BITS == 4 ? 256 / 32 : 1][BITS == 4 ? kHeadDim : 1], zf[BITS == 4 ? 256 / 32 : 1][BITS == 4 ? kHeadDim : 1];
};

template <int BITS>
__device__ void quantize_k_fine_tiles(const uint16_t* __restrict__ src, int lg_gk, uint32_t* __restrict__ codes,
                                      uint16_t* __restrict__ scale, uint16_t* __restrict__ zero) {
  constexpr int L = (1 << BITS) - 1;
  __shared__ uint4 red_lo[1024 / 32][16], red_hi[1024 / 32][16];
  __shared__ __align__(16) KRules<BITS> kr;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = tid & 15, tg = tid >> 4;
  const uint4* s4 = reinterpret_cast<const uint4*>(src) + (tg * kTileTokens) * kChunks + c;
  uint4 x[kTileTokens];
#pragma unroll
  for (int k = 0; k < kTileTokens; ++k) x[k] = __ldg(s4 + k * kChunks);
  // per-channel extremes over the tile's tokens, then over the warp's other token group
  __half2 lo[4], hi[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    lo[i] = hi[i] = half2_of(x[0], i);
#pragma unroll
    for (int k = 1; k < kTileTokens; ++k) {
      lo[i] = __hmin2(lo[i], half2_of(x[k], i));
      hi[i] = __hmax2(hi[i], half2_of(x[k], i));
    }
    lo[i] = __hmin2(lo[i], shfl_xor_h2(lo[i], 16));
    hi[i] = __hmax2(hi[i], shfl_xor_h2(hi[i], 16));
  }
  if (lane < 16) {
    red_lo[warp][c] = make_uint4(u32_of(lo[0]), u32_of(lo[1]), u32_of(lo[2]), u32_of(lo[3]));
    red_hi[warp][c] = make_uint4(u32_of(hi[0]), u32_of(hi[1]), u32_of(hi[2]), u32_of(hi[3]));
  }
  __syncthreads();
  const int wpg = 1 << (lg_gk - 4);  // warps of one K group (g_k / 16)
  const int w0 = warp & ~(wpg - 1);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    lo[i] = h2_from(comp4(red_lo[w0][c], i));
    hi[i] = h2_from(comp4(red_hi[w0][c], i));
  }
  for (int w = 1; w < wpg; ++w) {
    const uint4 l4 = red_lo[w0 + w][c], h4 = red_hi[w0 + w][c];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      lo[i] = __hmin2(lo[i], h2_from(comp4(l4, i)));
      hi[i] = __hmax2(hi[i], h2_from(comp4(h4, i)));
    }
  }
  // Every thread of the K group's tpg tiles that hold chunk c has the same extremes.  Thread `sub`
  // forms (s, z) and the 2-bit thresholds of channels sub, sub + tpg (< 8) once and shares them.
  const int tpg = 1 << (lg_gk - 3);  // token groups (tiles) of one K group
  const int kg = tg >> (lg_gk - 3), sub = tg & (tpg - 1);
  {
    const uint4 l4 = make_uint4(u32_of(lo[0]), u32_of(lo[1]), u32_of(lo[2]), u32_of(lo[3]));
    const uint4 h4 = make_uint4(u32_of(hi[0]), u32_of(hi[1]), u32_of(hi[2]), u32_of(hi[3]));
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int j = sub + tpg * i;
      if (j < 8) {
        const __half2 lj = h2_from(comp4(l4, j >> 1)), hj = h2_from(comp4(h4, j >> 1));
        const float lf = (j & 1) ? __high2float(lj) : __low2float(lj);
        const float hf = (j & 1) ? __high2float(hj) : __low2float(hj);
        const int ch = 8 * c + j;
        const GroupParams g = make_group(lf, hf, L);
        kr.s[kg][ch] = g.s_bits;
        kr.z[kg][ch] = g.z_bits;
        if constexpr (BITS == 2) {
          const Thresh2 t = make_thresh2(g);
#pragma unroll
          for (int k = 0; k < 3; ++k) kr.t[k][kg][ch] = static_cast<uint16_t>(t.t[k]);
        } else {
          kr.inv_s[kg][ch] = g.inv_s;
          kr.zf[kg][ch] = g.zf;
        }
      }
    }
  }
  __syncthreads();
  if ((tg & (tpg - 1)) == 0) {       // the K group's first tile stores the pairs of its 8 channels
    const size_t row = static_cast<size_t>(tg >> (lg_gk - 3)) * kHeadDim + 8 * c;
    *reinterpret_cast<uint4*>(scale + row) = *reinterpret_cast<const uint4*>(&kr.s[kg][8 * c]);
    *reinterpret_cast<uint4*>(zero + row) = *reinterpret_cast<const uint4*>(&kr.z[kg][8 * c]);
  }
  const int tok0 = tg * kTileTokens;
  if constexpr (BITS == 4) {  // K word c of a token is exactly the tile's 8 channels
    GroupParams gp[8];
    {
      const uint4 sb = *reinterpret_cast<const uint4*>(&kr.s[kg][8 * c]);
      const uint4 zb = *reinterpret_cast<const uint4*>(&kr.z[kg][8 * c]);
      const float4 i0 = *reinterpret_cast<const float4*>(&kr.inv_s[BITS == 4 ? kg : 0][BITS == 4 ? 8 * c : 0]);
      const float4 i1 = *reinterpret_cast<const float4*>(&kr.inv_s[BITS == 4 ? kg : 0][BITS == 4 ? 8 * c + 4 : 0]);
      const float4 z0 = *reinterpret_cast<const float4*>(&kr.zf[BITS == 4 ? kg : 0][BITS == 4 ? 8 * c : 0]);
      const float4 z1 = *reinterpret_cast<const float4*>(&kr.zf[BITS == 4 ? kg : 0][BITS == 4 ? 8 * c + 4 : 0]);
      const float inv[8] = {i0.x, i0.y, i0.z, i0.w, i1.x, i1.y, i1.z, i1.w};
      const float zfs[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        gp[j].inv_s = inv[j];
        gp[j].zf = zfs[j];
        gp[j].s_bits = static_cast<uint16_t>(comp4(sb, j >> 1) >> (16 * (j & 1)));
        gp[j].z_bits = static_cast<uint16_t>(comp4(zb, j >> 1) >> (16 * (j & 1)));
      }
    }
#pragma unroll
    for (int k = 0; k < kTileTokens; ++k) {
      const uint32_t w[4] = {x[k].x, x[k].y, x[k].z, x[k].w};
      uint32_t r = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        uint32_t qa, qb;
        quantize_pair2(w[e], gp[2 * e], gp[2 * e + 1], L, qa, qb);
        r += (qa << (BITS * 2 * e)) + (qb << (BITS * (2 * e + 1)));
      }
      codes[(tok0 + k) * (kHeadDim / 8) + c] = r;
    }
  } else {  // K word c / 2 of a token: chunk 2i in bits 0..15, chunk 2i + 1 in bits 16..31
    Thresh2 tp[4];  // thresholds of channels 2 i (low half) and 2 i + 1 (high half)
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      const uint4 tw = *reinterpret_cast<const uint4*>(&kr.t[BITS == 2 ? k : 0][kg][BITS == 2 ? 8 * c : 0]);
#pragma unroll
      for (int i = 0; i < 4; ++i) tp[i].t[k] = comp4(tw, i);
    }
    uint32_t h[kTileTokens];
#pragma unroll
    for (int k = 0; k < kTileTokens; ++k) {
      const uint32_t h0 = codes2_h2(x[k].x, tp[0]), h1 = codes2_h2(x[k].y, tp[1]);
      const uint32_t h2 = codes2_h2(x[k].z, tp[2]), h3 = codes2_h2(x[k].w, tp[3]);
      h[k] = gather4x2(__byte_perm(h0, h1, 0x6420)) | (gather4x2(__byte_perm(h2, h3, 0x6420)) << 8);
    }
    const bool odd = c & 1;
#pragma unroll
    for (int j = 0; j < 4; ++j) {  // the even chunk stores tokens 0..3 of the tile, the odd one 4..7
      const uint32_t other = __shfl_xor_sync(0xffffffffu, odd ? h[j] : h[4 + j], 1);
      const int k = odd ? 4 + j : j;
      const uint32_t word = odd ? (other | (h[4 + j] << 16)) : (h[j] | (other << 16));
      codes[(tok0 + k) * (kHeadDim / 16) + (c >> 1)] = word;
    }
  }
}

template <int BITS>
__device__ void quantize_v_fine_tiles(const uint16_t* __restrict__ src, int lg_gv, uint32_t* __restrict__ codes,
                                      uint16_t* __restrict__ scale, uint16_t* __restrict__ zero) {
  constexpr int L = (1 << BITS) - 1;
  const int tid = threadIdx.x;
  const int c = tid & 15, tg = tid >> 4;
  const uint4* s4 = reinterpret_cast<const uint4*>(src) + (tg * kTileTokens) * kChunks + c;
  uint4 x[kTileTokens];
#pragma unroll
  for (int k = 0; k < kTileTokens; ++k) x[k] = __ldg(s4 + k * kChunks);
  // per-token extremes over the chunk's 8 channels, then over the g_v / 8 chunks of the channel
  // group (lanes c of one half warp)
  const int cpg = 1 << (lg_gv - 3);
  uint32_t mw[kTileTokens];  // (min, -max) of each token's group, the same in all cpg lanes
#pragma unroll
  for (int k = 0; k < kTileTokens; ++k) {
    __half2 lo = half2_of(x[k], 0), hi = lo;
#pragma unroll
    for (int i = 1; i < 4; ++i) {
      lo = __hmin2(lo, half2_of(x[k], i));
      hi = __hmax2(hi, half2_of(x[k], i));
    }
    __half2 m = __halves2half2(__hmin(__low2half(lo), __high2half(lo)), __hneg(__hmax(__low2half(hi), __high2half(hi))));
    for (int off = 1; off < cpg; off <<= 1) m = __hmin2(m, shfl_xor_h2(m, off));
    mw[k] = u32_of(m);
  }
  const int ngv = kHeadDim >> lg_gv, g = c >> (lg_gv - 3);
  const int tok0 = tg * kTileTokens;
  // Lane ci of the group's cpg lanes forms the rule of tokens ci, ci + cpg (< 8) once, stores their
  // (s, z), and hands the rule to the other lanes by shuffles: 2 bits the three thresholds, 4 bits
  // 1/s, z and the stored (s, z) bits.
  const int ci = c & (cpg - 1);
  const int lane = tid & 31;
  uint32_t pa[2] = {0u, 0u}, pb[2] = {0u, 0u}, pc[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int k = ci + cpg * i;
    if (k < kTileTokens) {
      const uint4 m4 = k < 4 ? make_uint4(mw[0], mw[1], mw[2], mw[3]) : make_uint4(mw[4], mw[5], mw[6], mw[7]);
      const GroupParams gk = group_from_pair(h2_from(comp4(m4, k & 3)), L);
      scale[(tok0 + k) * ngv + g] = gk.s_bits;
      zero[(tok0 + k) * ngv + g] = gk.z_bits;
      if constexpr (BITS == 2) {
        const Thresh2 t = make_thresh2(gk);
        pa[i] = (t.t[0] & 0xFFFFu) | (t.t[1] << 16);
        pb[i] = t.t[2] & 0xFFFFu;
      } else {
        pa[i] = __float_as_uint(gk.inv_s);
        pb[i] = __float_as_uint(gk.zf);
        pc[i] = static_cast<uint32_t>(gk.s_bits) | (static_cast<uint32_t>(gk.z_bits) << 16);
      }
    }
  }
  GroupParams gp[kTileTokens];
  Thresh2 t[kTileTokens];
#pragma unroll
  for (int k = 0; k < kTileTokens; ++k) {
    const int src_lane = (lane & ~(cpg - 1)) | (k & (cpg - 1));
    const bool second = k >= cpg;
    const uint32_t a = __shfl_sync(0xffffffffu, second ? pa[1] : pa[0], src_lane);
    const uint32_t b = __shfl_sync(0xffffffffu, second ? pb[1] : pb[0], src_lane);
    if constexpr (BITS == 2) {
      t[k].t[0] = (a & 0xFFFFu) * 0x00010001u;
      t[k].t[1] = (a >> 16) * 0x00010001u;
      t[k].t[2] = (b & 0xFFFFu) * 0x00010001u;
    } else {
      const uint32_t sz = __shfl_sync(0xffffffffu, second ? pc[1] : pc[0], src_lane);
      gp[k].inv_s = __uint_as_float(a);
      gp[k].zf = __uint_as_float(b);
      gp[k].s_bits = static_cast<uint16_t>(sz & 0xFFFFu);
      gp[k].z_bits = static_cast<uint16_t>(sz >> 16);
    }
  }
  // codes of channel 8 c + e for the tile's 8 tokens, token k at bits BITS * k
  uint32_t col[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  if constexpr (BITS == 4) {
#pragma unroll
    for (int k = 0; k < kTileTokens; ++k) {
      const uint32_t w[4] = {x[k].x, x[k].y, x[k].z, x[k].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        uint32_t qa, qb;
        quantize_pair(w[e], gp[k], L, qa, qb);
        col[2 * e] += qa << (BITS * k);
        col[2 * e + 1] += qb << (BITS * k);
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(codes + tg * kHeadDim + 8 * c);
    dst[0] = make_uint4(col[0], col[1], col[2], col[3]);
    dst[1] = make_uint4(col[4], col[5], col[6], col[7]);
  } else {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      uint32_t A[4];
#pragma unroll
      for (int a2 = 0; a2 < 4; ++a2) {
        const uint32_t w0 = comp4(x[2 * a2], e), w1 = comp4(x[2 * a2 + 1], e);
        A[a2] = __byte_perm(codes2_h2(w0, t[2 * a2]), codes2_h2(w1, t[2 * a2 + 1]), 0x6240);
      }
      col[2 * e] = gather4x2(__byte_perm(A[0], A[1], 0x5410)) | (gather4x2(__byte_perm(A[2], A[3], 0x5410)) << 8);
      col[2 * e + 1] = gather4x2(__byte_perm(A[0], A[1], 0x7632)) | (gather4x2(__byte_perm(A[2], A[3], 0x7632)) << 8);
    }
    const bool odd = tg & 1;
    uint32_t word[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {  // the even token group stores channels 0..3, the odd one 4..7
      const uint32_t other = __shfl_xor_sync(0xffffffffu, odd ? col[e] : col[4 + e], 16);
      word[e] = odd ? (other | (col[4 + e] << 16)) : (col[e] | (other << 16));
    }
    *reinterpret_cast<uint4*>(codes + (tg >> 1) * kHeadDim + 8 * c + (odd ? 4 : 0)) =
        make_uint4(word[0], word[1], word[2], word[3]);
  }
}

// grid: x = batch * kv_heads, y = 2 * nblocks (+1 residual-copy job); block = 2R threads (R <= 256:
// the per-channel and per-token parameters need more than the 64 registers of a 1024-thread block)
// NT = 2R threads: 256 threads (R = 128) are held to 64 registers, so that four CTAs share an SM
// (a few spills; 1.6% faster than three CTAs at 80 registers, 2.6x the two CTAs of 98).
#ifndef KIVI_FG_CTAS
#define KIVI_FG_CTAS 4
#endif
template <int BITS, int NT>
__global__ void __launch_bounds__(NT, NT == 256 ? KIVI_FG_CTAS : 1) quantize_fine_tiles_kernel(QuantizeArgs a) {
  constexpr int P = 32 / BITS;
  const int bh = blockIdx.x;
  const int job = blockIdx.y;
  const int R = a.residual;
  const size_t C = static_cast<size_t>(a.capacity);
  if (job >= 2 * a.nblocks) {
    copy_residual(a, bh);
    return;
  }
  const int blk = job >> 1;
  const bool is_v = job & 1;
  if (a.v_only && !is_v) return;
  if (!job_in_bounds(a, blk)) return;
  const size_t src_tok = static_cast<size_t>(bh) * a.src_tokens + a.src_tok0 + static_cast<size_t>(blk) * R;
  const size_t dst_tok = static_cast<size_t>(a.dst_blk0 + blk) * R;
  if (!is_v) {
    const size_t srow = (static_cast<size_t>(bh) * (C >> a.lg_gk) + (dst_tok >> a.lg_gk)) * kHeadDim;
    quantize_k_fine_tiles<BITS>(a.k_src + src_tok * kHeadDim, a.lg_gk,
                                a.k_codes + (static_cast<size_t>(bh) * C + dst_tok) * (kHeadDim / P), a.k_scale + srow,
                                a.k_zero + srow);
  } else {
    const size_t ngv = kHeadDim >> a.lg_gv;
    const size_t srow = (static_cast<size_t>(bh) * C + dst_tok) * ngv;
    quantize_v_fine_tiles<BITS>(a.v_src + src_tok * kHeadDim, a.lg_gv,
                                a.v_codes + (static_cast<size_t>(bh) * (C / P) + dst_tok / P) * kHeadDim, a.v_scale + srow,
                                a.v_zero + srow);
  }
}

// grid: x = batch * kv_heads, y = 2 * nblocks (+1 residual-copy job); block = 2R threads (R <= 512)
template <int BITS>
__global__ void __launch_bounds__(1024) quantize_tiles_kernel(QuantizeArgs a) {
  constexpr int P = 32 / BITS;
  const int bh = blockIdx.x;
  const int job = blockIdx.y;
  const int R = a.residual;
  const size_t C = static_cast<size_t>(a.capacity);
  if (job < 2 * a.nblocks) {
    const int blk = job >> 1;
    const bool is_v = job & 1;
    if (a.v_only && !is_v) return;
    if (!job_in_bounds(a, blk)) return;
    const size_t src_tok = static_cast<size_t>(bh) * a.src_tokens + a.src_tok0 + static_cast<size_t>(blk) * R;
    const int dst_blk = a.dst_blk0 + blk;
    const size_t dst_tok = static_cast<size_t>(dst_blk) * R;
    if (!is_v) {
      quantize_k_tiles<BITS>(a.k_src + src_tok * kHeadDim, R, a.lg_gk,
                             a.k_codes + (static_cast<size_t>(bh) * C + dst_tok) * (kHeadDim / P),
                             a.k_scale + (static_cast<size_t>(bh) * (C / R) + dst_blk) * (kHeadDim >> a.lg_gk),
                             a.k_zero + (static_cast<size_t>(bh) * (C / R) + dst_blk) * (kHeadDim >> a.lg_gk),
                             a.k_given != 0);
    } else {
      quantize_v_tiles<BITS>(a.v_src + src_tok * kHeadDim, R, a.lg_gv,
                             a.v_codes + (static_cast<size_t>(bh) * (C / P) + dst_tok / P) * kHeadDim,
                             a.v_scale + static_cast<size_t>(bh) * (C >> a.lg_gv) + (dst_tok >> a.lg_gv),
                             a.v_zero + static_cast<size_t>(bh) * (C >> a.lg_gv) + (dst_tok >> a.lg_gv));
    }
  } else {
    copy_residual(a, bh);
  }
}

// grid: x = batch * kv_heads, y = 2 * nblocks (+1 residual-copy job when res_tokens > 0)
template <int BITS>
__global__ void __launch_bounds__(kThreads) quantize_blocks_kernel(QuantizeArgs a) {
  constexpr int P = 32 / BITS;
  const int bh = blockIdx.x;
  const int job = blockIdx.y;
  const int R = a.residual;
  const size_t C = static_cast<size_t>(a.capacity);
  if (job < 2 * a.nblocks) {
    const int blk = job >> 1;
    const bool is_v = job & 1;
    if (a.v_only && !is_v) return;
    if (!job_in_bounds(a, blk)) return;
    const size_t src_tok = static_cast<size_t>(bh) * a.src_tokens + a.src_tok0 + static_cast<size_t>(blk) * R;
    const int dst_blk = a.dst_blk0 + blk;
    const size_t dst_tok = static_cast<size_t>(dst_blk) * R;
    if (!is_v) {
      quantize_k_block<BITS>(a.k_src + src_tok * kHeadDim, R, a.group_k,
                             a.k_codes + (static_cast<size_t>(bh) * C + dst_tok) * (kHeadDim / P),
                             a.k_scale + (static_cast<size_t>(bh) * (C / R) + dst_blk) * (kHeadDim / a.group_k),
                             a.k_zero + (static_cast<size_t>(bh) * (C / R) + dst_blk) * (kHeadDim / a.group_k),
                             a.k_given != 0);
    } else {
      quantize_v_block<BITS>(a.v_src + src_tok * kHeadDim, R, a.group_v,
                             a.v_codes + (static_cast<size_t>(bh) * (C / P) + dst_tok / P) * kHeadDim,
                             a.v_scale + static_cast<size_t>(bh) * (C / a.group_v) + dst_tok / a.group_v,
                             a.v_zero + static_cast<size_t>(bh) * (C / a.group_v) + dst_tok / a.group_v);
    }
  } else {
    copy_residual(a, bh);
  }
}

// one thread per 16-byte chunk of the new K and V rows
__global__ void __launch_bounds__(256) append_kernel(AppendArgs a) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const int n = a.bh * kChunks;
  if (i >= n) return;
  if (!dbg_check(a.slot >= 0 && a.slot < a.residual)) return;
  const int bh = i / kChunks, c = i % kChunks;
  const size_t dst = (static_cast<size_t>(bh) * a.residual + a.slot) * kChunks + c;
  reinterpret_cast<uint4*>(a.k_res)[dst] = __ldg(reinterpret_cast<const uint4*>(a.k_new) + i);
  reinterpret_cast<uint4*>(a.v_res)[dst] = __ldg(reinterpret_cast<const uint4*>(a.v_new) + i);
}

// ---------------------------------------------------------------------------------------------
// Fine-grained groups (section KVキャッシュの分布特性: the K range along each channel, the V range
// along each token).  grid: x = batch * kv_heads, y = 2 * nblocks (+1 residual-copy job); 128
// threads, thread c owns channel c.  K: per group of g_k tokens, thread c reduces its channel, forms
// (s, z) and codes the group's tokens (the P threads of a code word OR their codes together).
// V: per token, the g_v threads of a channel group reduce it (warp shuffles, then shared memory
// across warps for g_v > 32), and thread c shifts its code into its channel's word of P tokens.
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t quantize_one(float x, const GroupParams& g, int levels) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23: rounds r to the nearest integer, ties to even
  const float r = __fmul_rn(__fadd_rn(x, -g.zf), g.inv_s);
  const float t = __fadd_rn(r, kMagic);
  const float dr = __fadd_rn(r, __fadd_rn(kMagic, -t));
  uint32_t q = min(__float_as_uint(t) - 0x4B400000u, static_cast<uint32_t>(levels));
  if (fabsf(dr) > 0.499755859375f) q = quantize_exact(x, g, levels);  // within 2^-12 of a tie
  return g.inv_s == 0.f ? 0u : q;
}

template <int BITS>
__global__ void __launch_bounds__(kHeadDim) quantize_fine_kernel(QuantizeArgs a) {
  constexpr int P = 32 / BITS, L = (1 << BITS) - 1;
  __shared__ float red_lo[8][kHeadDim / 32], red_hi[8][kHeadDim / 32];
  const int bh = blockIdx.x, job = blockIdx.y, c = threadIdx.x, warp = c >> 5;
  const int R = a.residual;
  const size_t C = static_cast<size_t>(a.capacity);
  if (job >= 2 * a.nblocks) {
    copy_residual(a, bh);
    return;
  }
  const int blk = job >> 1;
  const bool is_v = job & 1;
  if (a.v_only && !is_v) return;
  if (!job_in_bounds(a, blk)) return;
  const size_t src_tok = static_cast<size_t>(bh) * a.src_tokens + a.src_tok0 + static_cast<size_t>(blk) * R;
  const size_t dst_tok = static_cast<size_t>(a.dst_blk0 + blk) * R;
  const unsigned word_mask = (P == 32 ? 0xffffffffu : ((1u << P) - 1u)) << ((c & 31) & ~(P - 1));
  if (!is_v) {
    const uint16_t* src = a.k_src + src_tok * kHeadDim + c;
    const int gk = a.group_k;
    for (int u = 0; u < R / gk; ++u) {
      float lo = INFINITY, hi = -INFINITY;
      for (int t = 0; t < gk; ++t) {
        const float x = h2f(__ldg(src + static_cast<size_t>(u * gk + t) * kHeadDim));
        lo = fminf(lo, x);
        hi = fmaxf(hi, x);
      }
      const GroupParams gp = make_group(lo, hi, L);
      const size_t si = (static_cast<size_t>(bh) * (C / gk) + (dst_tok / gk) + u) * kHeadDim + c;
      a.k_scale[si] = gp.s_bits;
      a.k_zero[si] = gp.z_bits;
      for (int t = 0; t < gk; ++t) {
        const int tok = u * gk + t;
        const uint32_t q = quantize_one(h2f(__ldg(src + static_cast<size_t>(tok) * kHeadDim)), gp, L);
        const uint32_t word = __reduce_or_sync(word_mask, q << (BITS * (c & (P - 1))));
        if ((c & (P - 1)) == 0)
          a.k_codes[(static_cast<size_t>(bh) * C + dst_tok + tok) * (kHeadDim / P) + c / P] = word;
      }
    }
  } else {
    const uint16_t* src = a.v_src + src_tok * kHeadDim + c;
    const int gv = a.group_v, wpg = gv >> 5;  // warps per channel group
    const int ngv = kHeadDim / gv, g = c / gv;
    uint32_t word = 0u;
    for (int t0 = 0; t0 < R; t0 += 8) {
      float x[8], lo[8], hi[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        x[i] = h2f(__ldg(src + static_cast<size_t>(t0 + i) * kHeadDim));
        lo[i] = x[i];
        hi[i] = x[i];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          lo[i] = fminf(lo[i], __shfl_xor_sync(0xffffffffu, lo[i], off));
          hi[i] = fmaxf(hi[i], __shfl_xor_sync(0xffffffffu, hi[i], off));
        }
      }
      if (wpg > 1) {
        __syncthreads();  // the previous batch's partials are read
        float mlo = lo[0], mhi = hi[0];  // lane i < 8 publishes token i's warp extremes
#pragma unroll
        for (int i = 1; i < 8; ++i) {
          if ((c & 7) == i) {
            mlo = lo[i];
            mhi = hi[i];
          }
        }
        if ((c & 31) < 8) {
          red_lo[c & 31][warp] = mlo;
          red_hi[c & 31][warp] = mhi;
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          for (int w = g * wpg; w < (g + 1) * wpg; ++w) {
            lo[i] = fminf(lo[i], red_lo[i][w]);
            hi[i] = fmaxf(hi[i], red_hi[i][w]);
          }
        }
      }
      // every lane of a warp holds the same 8 group ranges: lane i % 8 forms token i's (s, z) once and
      // the warp broadcasts it
      float mlo = lo[0], mhi = hi[0];
#pragma unroll
      for (int i = 1; i < 8; ++i) {
        if ((c & 7) == i) {
          mlo = lo[i];
          mhi = hi[i];
        }
      }
      const GroupParams mine = make_group(mlo, mhi, L);
      const uint32_t mine_sz = static_cast<uint32_t>(mine.s_bits) | (static_cast<uint32_t>(mine.z_bits) << 16);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int tok = t0 + i;
        GroupParams gp;
        gp.inv_s = __shfl_sync(0xffffffffu, mine.inv_s, i);
        gp.zf = __shfl_sync(0xffffffffu, mine.zf, i);
        const uint32_t sz = __shfl_sync(0xffffffffu, mine_sz, i);
        gp.s_bits = static_cast<uint16_t>(sz & 0xFFFFu);
        gp.z_bits = static_cast<uint16_t>(sz >> 16);
        if (c % gv == 0) {
          const size_t si = (static_cast<size_t>(bh) * C + dst_tok + tok) * ngv + g;
          a.v_scale[si] = gp.s_bits;
          a.v_zero[si] = gp.z_bits;
        }
        word |= quantize_one(x[i], gp, L) << (BITS * (tok & (P - 1)));
        if ((tok & (P - 1)) == P - 1) {
          a.v_codes[(static_cast<size_t>(bh) * (C / P) + (dst_tok + tok) / P) * kHeadDim + c] = word;
          word = 0u;
        }
      }
    }
  }
}

// Online K (section Per-Channel量子化: a new token's K is quantized at once with the existing scale
// and zero point).  grid: x = batch * kv_heads, y = rows; 128 threads, one per channel.  The code
// is clamp(rint((x - z) / s), 0, L) in fp64, which decides exactly: x - z of two fp16 values is
// exact and the one rounding of the quotient cannot move it across a half-integer (s == 0: 0).
// The P threads of one code word OR their shifted codes together.
template <int BITS>
__global__ void __launch_bounds__(kHeadDim) code_k_online_kernel(OnlineKArgs a) {
  constexpr int P = 32 / BITS, L = (1 << BITS) - 1;
  const int bh = blockIdx.x, row = blockIdx.y, c = threadIdx.x;
  const int lg_gk = __ffs(a.group_k) - 1, ngk = kHeadDim >> lg_gk;
  const size_t C = static_cast<size_t>(a.capacity), nblk = C / static_cast<size_t>(a.residual);
  const size_t sb = (static_cast<size_t>(bh) * nblk + a.blk_src) * ngk;
  if (!dbg_check(a.blk_src >= 0 && a.blk_src + (a.copy_scales ? 1 : 0) < static_cast<long long>(nblk) &&
                 a.dst_row0 + row < a.capacity && a.src_tok0 + row < a.src_tokens &&
                 (a.v_new == nullptr || (a.v_slot >= 0 && a.v_slot < a.residual))))
    return;
  const uint16_t xb = __ldg(a.k_src + (static_cast<size_t>(bh) * a.src_tokens + a.src_tok0 + row) * kHeadDim + c);
  const double s = static_cast<double>(h2f(__ldg(a.k_scale + sb + (c >> lg_gk))));
  const double z = static_cast<double>(h2f(__ldg(a.k_zero + sb + (c >> lg_gk))));
  uint32_t code = 0u;
  if (s > 0.0) code = static_cast<uint32_t>(fmin(fmax(rint((static_cast<double>(h2f(xb)) - z) / s), 0.0), double(L)));
  const unsigned mask = (P == 32 ? 0xffffffffu : ((1u << P) - 1u)) << ((c & 31) & ~(P - 1));
  const uint32_t word = __reduce_or_sync(mask, code << (BITS * (c & (P - 1))));
  if ((c & (P - 1)) == 0)
    a.k_codes[(static_cast<size_t>(bh) * C + a.dst_row0 + row) * (kHeadDim / P) + c / P] = word;
  if (row == 0 && a.copy_scales && c < ngk) {
    a.k_scale[sb + ngk + c] = a.k_scale[sb + c];
    a.k_zero[sb + ngk + c] = a.k_zero[sb + c];
  }
  if (row == 0 && a.v_new != nullptr)
    a.v_res[(static_cast<size_t>(bh) * a.residual + a.v_slot) * kHeadDim + c] =
        __ldg(a.v_new + static_cast<size_t>(bh) * kHeadDim + c);
}

// K (s, z) of channel group blockIdx.y of head blockIdx.x over all nblocks * R source tokens
// (section Per-Channel量子化 read with one group over every quantized token of the prompt), written
// into the slot of every destination block.  256 threads; each warp reads 8 tokens x g_k channels
// per step.
template <int BITS>
__global__ void __launch_bounds__(kThreads) k_prefix_extremes_kernel(QuantizeArgs a) {
  constexpr int L = (1 << BITS) - 1;
  __shared__ __half2 red[kThreads / 32];
  __shared__ uint32_t sz;
  const int bh = blockIdx.x, g = blockIdx.y, tid = threadIdx.x;
  const int lg_cpg = a.lg_gk - 3, cpg = 1 << lg_cpg;  // 16-byte chunks per group
  if (!dbg_check(a.dst_blk0 + a.nblocks <= a.capacity / a.residual &&
                 a.src_tok0 + static_cast<long long>(a.nblocks) * a.residual <= a.src_tokens))
    return;
  const long long ntok = static_cast<long long>(a.nblocks) * a.residual;
  const uint4* src = reinterpret_cast<const uint4*>(a.k_src + (static_cast<size_t>(bh) * a.src_tokens + a.src_tok0) *
                                                                  kHeadDim) + g * cpg;
  const uint32_t kPosInf = 0x7C007C00u, kNegInf = 0xFC00FC00u;
  __half2 lo = *reinterpret_cast<const __half2*>(&kPosInf), hi = *reinterpret_cast<const __half2*>(&kNegInf);
  for (long long i = tid; i < (ntok << lg_cpg); i += kThreads) {
    const uint4 v = __ldg(src + (i >> lg_cpg) * kChunks + (i & (cpg - 1)));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __half2 h = *reinterpret_cast<const __half2*>(&w[e]);
      lo = __hmin2(lo, h);
      hi = __hmax2(hi, h);
    }
  }
  __half2 m = __halves2half2(__hmin(__low2half(lo), __high2half(lo)), __hneg(__hmax(__low2half(hi), __high2half(hi))));
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) m = __hmin2(m, shfl_xor_h2(m, off));
  if ((tid & 31) == 0) red[tid >> 5] = m;
  __syncthreads();
  if (tid == 0) {
    __half2 t = red[0];
    for (int w = 1; w < kThreads / 32; ++w) t = __hmin2(t, red[w]);
    const GroupParams gp = group_from_pair(t, L);
    sz = static_cast<uint32_t>(gp.s_bits) | (static_cast<uint32_t>(gp.z_bits) << 16);
  }
  __syncthreads();
  const int ngk = kHeadDim >> a.lg_gk;
  const size_t C = static_cast<size_t>(a.capacity), R = static_cast<size_t>(a.residual);
  for (int blk = tid; blk < a.nblocks; blk += kThreads) {
    const size_t slot = (static_cast<size_t>(bh) * (C / R) + a.dst_blk0 + blk) * ngk + g;
    a.k_scale[slot] = static_cast<uint16_t>(sz & 0xFFFFu);
    a.k_zero[slot] = static_cast<uint16_t>(sz >> 16);
  }
}

}  // namespace

cudaError_t debug_status_quantize(int32_t* out) { return take_debug_status_tu(out); }

cudaError_t launch_quantize_blocks(const QuantizeArgs& args, int bits, cudaStream_t stream) {
  const int jobs = 2 * args.nblocks + (args.res_tokens > 0 ? 1 : 0);
  if (jobs == 0) return cudaSuccess;
  QuantizeArgs a = args;  // group sizes are powers of two (checked by the caller)
  a.lg_gk = __builtin_ctz(static_cast<unsigned>(a.group_k));
  a.lg_gv = __builtin_ctz(static_cast<unsigned>(a.group_v));
  dim3 grid(a.bh, jobs);
  if (a.fine && a.residual <= 256) {  // one thread per 8 tokens x 8 channels of a block
    if (a.residual == 128) {
      if (bits == 2)
        quantize_fine_tiles_kernel<2, 256><<<grid, 256, 0, stream>>>(a);
      else
        quantize_fine_tiles_kernel<4, 256><<<grid, 256, 0, stream>>>(a);
    } else {
      if (bits == 2)
        quantize_fine_tiles_kernel<2, 512><<<grid, 512, 0, stream>>>(a);
      else
        quantize_fine_tiles_kernel<4, 512><<<grid, 512, 0, stream>>>(a);
    }
  } else if (a.fine) {
    if (bits == 2)
      quantize_fine_kernel<2><<<grid, kHeadDim, 0, stream>>>(a);
    else
      quantize_fine_kernel<4><<<grid, kHeadDim, 0, stream>>>(a);
  } else if (a.residual <= 512) {  // one thread per 8 tokens x 8 channels of a block
    if (bits == 2)
      quantize_tiles_kernel<2><<<grid, 2 * a.residual, 0, stream>>>(a);
    else
      quantize_tiles_kernel<4><<<grid, 2 * a.residual, 0, stream>>>(a);
  } else if (bits == 2) {
    quantize_blocks_kernel<2><<<grid, kThreads, 0, stream>>>(a);
  } else {
    quantize_blocks_kernel<4><<<grid, kThreads, 0, stream>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_k_prefix_extremes(const QuantizeArgs& args, int bits, cudaStream_t stream) {
  if (args.nblocks == 0) return cudaSuccess;
  QuantizeArgs a = args;
  a.lg_gk = __builtin_ctz(static_cast<unsigned>(a.group_k));
  a.lg_gv = __builtin_ctz(static_cast<unsigned>(a.group_v));
  dim3 grid(a.bh, kHeadDim / a.group_k);
  if (bits == 2)
    k_prefix_extremes_kernel<2><<<grid, kThreads, 0, stream>>>(a);
  else
    k_prefix_extremes_kernel<4><<<grid, kThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_code_k_online(const OnlineKArgs& a, int bits, cudaStream_t stream) {
  if (a.rows < 1) return cudaSuccess;
  dim3 grid(a.bh, a.rows);
  if (bits == 2)
    code_k_online_kernel<2><<<grid, kHeadDim, 0, stream>>>(a);
  else
    code_k_online_kernel<4><<<grid, kHeadDim, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_append(const AppendArgs& a, cudaStream_t stream) {
  const int n = a.bh * kChunks;
  append_kernel<<<(n + 255) / 256, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace kivi
