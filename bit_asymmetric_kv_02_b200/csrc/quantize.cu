// Quantize + pack (prefill and flush) and residual append kernels.
//
// Method: KIVI explainer page "ICML 2024論文解説: KIVI — チューニング不要のKVキャッシュ2bit非対称量子化",
//   section 量子化アルゴリズム (Q, D and s/z equations), Per-Channel量子化（Key Cache）(K groups: g_k
//   consecutive channels), Per-Token量子化（Value Cache）(V groups: g_v consecutive tokens) and
//   残差バッファ（Residual Buffer）(the newest tokens stay fp16 until a block is flushed).
//
// One CTA quantizes one R-token block of K or of V for one (batch, KV head):
//   pass 1 reads the block once from HBM (128-bit loads) and reduces the group minima / maxima;
//   s = fp16_rn((max - min)/(2^b - 1)) is formed in fp64 (exact range, one rounding), z = min;
//   pass 2 re-reads the block (L2-resident) and emits codes, 32/b per uint32 word.
// A code is RNE of the exact rational (x - z)/s.  It is computed in fp32 as (x - z) * (1/s), whose
// relative error is below 3*2^-24, i.e. below 2^-18 absolute for every reachable value; when the
// fp32 value lies within 2^-12 of a half-integer the element is re-decided with an fp64 division,
// which is exact there.  Both sides of a parity test therefore take the exact decision.
#include <cstdint>

#include "common.cuh"
#include "kernels.h"

namespace kivi {

namespace {

constexpr int kThreads = 256;
constexpr int kChunks = kHeadDim / 8;  // uint4 chunks per token row

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

// Q of one element (section 量子化アルゴリズム, Q equation) with the stored fp16 s and z, taken
// exactly: the fp64 quotient decides (used near ties only).
__device__ __forceinline__ uint32_t quantize_exact(float x, const GroupParams& g, int levels) {
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

// ---------------------------------------------------------------------------------------------
// K block: groups of `gk` channels over all R tokens of the block.
// ---------------------------------------------------------------------------------------------
template <int BITS>
__device__ void quantize_k_block(const uint16_t* __restrict__ src, int R, int gk, uint32_t* __restrict__ codes,
                                 uint16_t* __restrict__ scale, uint16_t* __restrict__ zero) {
  constexpr int P = 32 / BITS;
  constexpr int L = (1 << BITS) - 1;
  __shared__ float red_lo[kThreads / 32][kChunks], red_hi[kThreads / 32][kChunks];
  __shared__ GroupParams grp[kHeadDim / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int chunk = tid % kChunks;
  const uint4* s4 = reinterpret_cast<const uint4*>(src);

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
    const size_t src_tok = static_cast<size_t>(bh) * a.src_tokens + a.src_tok0 + static_cast<size_t>(blk) * R;
    const int dst_blk = a.dst_blk0 + blk;
    const size_t dst_tok = static_cast<size_t>(dst_blk) * R;
    if (!is_v) {
      quantize_k_block<BITS>(a.k_src + src_tok * kHeadDim, R, a.group_k,
                             a.k_codes + (static_cast<size_t>(bh) * C + dst_tok) * (kHeadDim / P),
                             a.k_scale + (static_cast<size_t>(bh) * (C / R) + dst_blk) * (kHeadDim / a.group_k),
                             a.k_zero + (static_cast<size_t>(bh) * (C / R) + dst_blk) * (kHeadDim / a.group_k));
    } else {
      quantize_v_block<BITS>(a.v_src + src_tok * kHeadDim, R, a.group_v,
                             a.v_codes + (static_cast<size_t>(bh) * (C / P) + dst_tok / P) * kHeadDim,
                             a.v_scale + static_cast<size_t>(bh) * (C / a.group_v) + dst_tok / a.group_v,
                             a.v_zero + static_cast<size_t>(bh) * (C / a.group_v) + dst_tok / a.group_v);
    }
  } else {
    // residual copy: tokens [res_tok0, res_tok0 + res_tokens) of the source -> slots 0..
    const size_t src_tok = static_cast<size_t>(bh) * a.src_tokens + a.res_tok0;
    const uint4* ks = reinterpret_cast<const uint4*>(a.k_src + src_tok * kHeadDim);
    const uint4* vs = reinterpret_cast<const uint4*>(a.v_src + src_tok * kHeadDim);
    uint4* kd = reinterpret_cast<uint4*>(a.k_res + static_cast<size_t>(bh) * R * kHeadDim);
    uint4* vd = reinterpret_cast<uint4*>(a.v_res + static_cast<size_t>(bh) * R * kHeadDim);
    const int n = a.res_tokens * kChunks;
    for (int i = threadIdx.x; i < n; i += kThreads) {
      kd[i] = __ldg(ks + i);
      vd[i] = __ldg(vs + i);
    }
  }
}

// one thread per 16-byte chunk of the new K and V rows
__global__ void __launch_bounds__(256) append_kernel(AppendArgs a) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const int n = a.bh * kChunks;
  if (i >= n) return;
  const int bh = i / kChunks, c = i % kChunks;
  const size_t dst = (static_cast<size_t>(bh) * a.residual + a.slot) * kChunks + c;
  reinterpret_cast<uint4*>(a.k_res)[dst] = __ldg(reinterpret_cast<const uint4*>(a.k_new) + i);
  reinterpret_cast<uint4*>(a.v_res)[dst] = __ldg(reinterpret_cast<const uint4*>(a.v_new) + i);
}

}  // namespace

cudaError_t launch_quantize_blocks(const QuantizeArgs& a, int bits, cudaStream_t stream) {
  const int jobs = 2 * a.nblocks + (a.res_tokens > 0 ? 1 : 0);
  if (jobs == 0) return cudaSuccess;
  dim3 grid(a.bh, jobs);
  if (bits == 2)
    quantize_blocks_kernel<2><<<grid, kThreads, 0, stream>>>(a);
  else
    quantize_blocks_kernel<4><<<grid, kThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_append(const AppendArgs& a, cudaStream_t stream) {
  const int n = a.bh * kChunks;
  append_kernel<<<(n + 255) / 256, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace kivi
