// Fused decode attention over the quantized KV cache plus its fp16 residual (sm_100a).
//
// Method: KIVI explainer page "ICML 2024論文解説: KIVI — チューニング不要のKVキャッシュ2bit非対称量子化",
//   section 残差バッファ（Residual Buffer）, Attention equation:
//     out = softmax(scale * q [D(K_quant); K_res]^T) [D(V_quant); V_res],  D(x^) = s x^ + z.
//
// Work decomposition (stream-K over warps).  Every (batch, KV head) is a sequence of equal-size
// 8 KB "units": quantized units of UT tokens (UT = 128 at 2 bits, 64 at 4 bits; 4 KB of K codes +
// 4 KB of V codes) followed by residual units of 16 fp16 tokens (4 KB K + 4 KB V).  The global
// unit sequence is cut into one contiguous range per warp, so the load is balanced to one unit
// whatever the batch, head count or context length.  The grid is one CTA per SM (16, 12 or 8 warps
// by queries per KV head).  Each warp streams its range as half units K0 V0 K1 V1 ... through a
// ring of two (up to 4 queries per KV head) or three 4 KB shared-memory buffers filled by 1-D TMA
// bulk copies (cp.async.bulk, no multicast) and completed on mbarriers: half h uses buffer h % n
// and is reissued as soon as half h - n is consumed.  Every wait is bounded and reports
// KIVI_ERR_DEVICE_TIMEOUT.  A warp whose range covers a whole head writes the output directly; a
// head split over several warps is merged (log-sum-exp) by the warp that arrives last on the head's
// atomic ticket, which then resets the ticket to zero.  No warp ever waits for another.
// A fused append (kivi_append_decode_attention) hands the new token's rows to the warp that owns
// the residual unit holding its slot; that warp patches its shared-memory copy and the cache.
//
// Arithmetic.  The byte dot products are exact int32 sums.  At 2 bits they run on the tensor cores
// (mma.sync m16n8k32, code bytes x operand digits): dp4a would need 768 issues of the half-rate
// FMA-heavy pipe per 8 KB and query, more than the HBM time of those bytes.  At 4 bits dp4a on the
// CUDA cores forms them (half the dp4a per byte).
//   A6  logit_t = sum_c q_c (s_g code + z_g) = sum_c (q_c s_g) code_tc + sum_g z_g sum_{c in g} q_c.
//       (q_c s_g) for one R-token block is turned into a 24-bit signed fixed-point integer Q (kept
//       while the warp stays in the same block).  At 2 bits a code word enters the tensor core as
//       itself plus three masked copies (raw bytes: see variants2) against operand values built
//       from the Q of each byte's four channels, four balanced signed byte digits each; at 4 bits
//       the codes are unpacked to bytes and multiplied with three byte limbs of Q.  Both are exact
//       in int32.  The block constant sum_g z_g q_g is added in fp32.
//   A8  online softmax in base 2 (q pre-scaled by scale*log2 e), redux.sync warp maxima, lane-local
//       sums.
//   A9  o_c = sum_t (p_t s_g(t)) code_tc + sum_t p_t z_g(t): (p_t s_g(t)) is turned into 24-bit
//       unsigned fixed point relative to a bound of the unit's largest value (at 2 bits: the
//       unit's largest weight times its largest V scale; at 4 bits: the exact maximum) and dotted
//       with the V codes (raw bytes and operand digits at 2 bits, as for A6); the z term is the
//       same for every channel and is one scalar.
//   A7/A9 residual rows: fp32 FMAs on the fp16 values.
//   A10 merge of (m, l, Z, o) states: o / l with o += Z.
// 24-bit fixed point keeps every product relative error below 2^-21, the integer sums are exact, and
// the remaining error is fp32 rounding.
#include <cstdint>

#include "common.cuh"
#include "kernels.h"
#include "quant_rules.cuh"

namespace kivi {

namespace {

// Stream-K workers (warps) per CTA: one CTA per SM.  Two to four queries per KV head run their dot
// products in passes of two queries, which fits 12 warps per SM (16 spill; 8 leave the FMA-heavy
// pipe idle more often).  The warps of one CTA are scheduled fairly;
// warps of separate CTAs on one SM are not (the oldest CTA's warps take precedence and finish
// early, leaving the SM with fewer warps for the rest of the launch).
#ifndef KIVI_GQA_WARPS
#define KIVI_GQA_WARPS 12  // warps per CTA for 2 and 4 queries per KV head (base groups)
#endif
template <int G, bool FG = false>
__host__ __device__ constexpr int warps_per_cta() {
  // fine-grained groups keep P operands per (query, V channel group) and more per-query state
  return FG ? (G == 1 ? 16 : (G == 2 ? 12 : (G == 4 ? 8 : 5))) : (G == 1 ? 16 : (G <= 4 ? KIVI_GQA_WARPS : 8));
}
constexpr int kHalfBytes = 4096;    // one half unit: the K part or the V part of a unit
// The tensor-core path lands a V half as four 1 KB pieces (two V word rows each) 1040 bytes apart,
// so that the four lanes reading one channel from rows 2 t + x (t = 0..3) hit four bank groups.
constexpr int kVPiece = 1024, kVPieceStride = 1040;
template <int G>
__host__ __device__ constexpr int buf_bytes() {
  return 4 * kVPieceStride;
}
// Half-unit buffers per warp: 3 gives the ring K0 V0 K1 | V1 K2 V2 | ..., 2 gives K | V.  Up to 4
// queries per KV head use 2 (1.4% faster than 3 at 16 warps per SM, and 16 warps of 3 would not fit
// in shared memory); 8 queries per KV head (8 warps per SM) use 3.
template <int G>
__host__ __device__ constexpr int ring_buffers() {
  return G <= 4 ? 2 : 3;
}
// Slots for the fp16 queries that land with a head's first K half.  With a ring of 2 the next
// unit's K half is issued only after this unit's K half (the last reader of the raw queries) is
// done, so one slot is enough; with a ring of 3 the K half two units ahead can start a head while
// the next unit's head has yet to read its queries: two slots, taken by head parity.
template <int G>
__host__ __device__ constexpr int q_slots() {
  return ring_buffers<G>() == 2 ? 1 : 2;
}
constexpr int kResTokens = 16;      // tokens per residual unit
constexpr unsigned kFull = 0xffffffffu;
constexpr float kQRange = 8388544.f;   // 2^23 - 64: largest |Q| before rounding (signed 24-bit limbs)
constexpr float kPRange = 16777088.f;  // 2^24 - 128: largest P before rounding (unsigned 24-bit limbs)
// Largest |Q| before rounding for balanced signed limbs (every digit in [-128, 127], so the top
// digit (Q + 32896) >> 16 must stay below 128): 2^23 - 2^16.
constexpr float kQRangeBal = 8323072.f;
// Raw-byte operands (2 bits, base scheme): |Q| <= 2^23 keeps every operand value X below 2^30 in
// magnitude (|X| <= 80 |Q|), inside the range of four balanced signed byte digits.
constexpr float kQRangeRaw = 8388544.f;  // 2^23 - 64

// Limb words per query: 96 (three limbs) for the CUDA-core dot products, 128 for the tensor-core
// path, which keeps a fourth, all-zero limb slot (the B operand columns of no limb read it).
constexpr int kLimbVecs = 32;

// FG (fine-grained groups): qw holds the Q limbs of each K token group of a unit (for the query in
// hand) and pw the P limbs of each (query, V channel group) (4 groups per query); oscr turns the
// output into the residual layout.
template <int G, bool FG = false>
struct __align__(16) WarpSmem {
  uint8_t buf[ring_buffers<G>()][buf_bytes<G>()];
  uint16_t qraw[q_slots<G>()][G][kHeadDim];  // fp16 queries of a head (see q_slots)
  uint4 qw[FG ? 4 : G][kLimbVecs];      // Q operand digits of each query (FG: limbs of each K token group)
  uint4 pw[FG ? 4 * G : G][kLimbVecs];  // P operand digits of each query (FG: limbs per query and V channel group)
  uint4 zero4;                      // the all-zero B operand of the other tile of a pair
  float oscr[FG ? kHeadDim : 4];
  float qs[G > 1 ? G : 1][G > 1 ? kHeadDim : 1];  // several queries: q * scale * log2 e of the head
  uint64_t bar[ring_buffers<G>()];
};

// Maximum over the warp in one instruction (sm_100a redux.sync on f32; NaN inputs are ignored).
__device__ __forceinline__ float warp_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}
__device__ __forceinline__ uint32_t comp(const uint4& v, int i) {
  return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}
// 1/x with the MUFU approximation (relative error < 2^-22).
__device__ __forceinline__ float fast_rcp(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// 2^x with the MUFU approximation (relative error ~2^-22); exp2(-inf) = +0.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// hi * 2^16 + mid * 2^8 + lo.  mid * 2^8 + lo stays below 2^27 for every sum formed here (at most
// 128 products of a byte with a code of at most 15), so it is formed exactly in int32.
__device__ __forceinline__ float combine_limbs(int hi, int mid, int lo) {
  return fmaf(static_cast<float>(hi), 65536.f, static_cast<float>((mid << 8) + lo));
}

// Tensor-core byte dot products: D += A B with A a 16 x 32 tile of codes (unsigned bytes, row-major)
// and B a 32 x 8 tile of limbs (signed or unsigned bytes), D 16 x 8 in int32.  Lane (g, t) =
// (lane / 4, lane % 4) holds A rows g and g + 8, columns 4 t .. 4 t + 3 (a0, a1) and 16 + 4 t ..
// 19 + 4 t (a2, a3); B column g, rows 4 t .. 4 t + 3 (b0) and 16 + 4 t .. (b1); D rows g and g + 8,
// columns 2 t and 2 t + 1.
__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_u8u8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// Byte b of x0 .. x3 packed into one word (byte m from x_m).
__device__ __forceinline__ uint32_t pick_bytes(uint32_t x0, uint32_t x1, uint32_t x2, uint32_t x3, int b) {
  const uint32_t sel = static_cast<uint32_t>(b) | (static_cast<uint32_t>(b + 4) << 4);
  return __byte_perm(__byte_perm(x0, x1, sel), __byte_perm(x2, x3, sel), 0x5410);
}
// Rows g and g + 8 of a tile pair's limb accumulators: lanes 2 t' and 2 t' + 1 (t' = 0, 1) hold
// columns (H, M) and (L, 0) of tile t' of the pair (columns 4 t' .. 4 t' + 2).  After one exchange
// with the partner lane, an even lane holds row g and an odd lane row g + 8, whole.
__device__ __forceinline__ float gather_limbs(const int (&c)[4], bool odd) {
  const int r1 = __shfl_xor_sync(0xffffffffu, odd ? c[0] : c[2], 1);
  const int r2 = __shfl_xor_sync(0xffffffffu, c[3], 1);
  const int hi = odd ? r1 : c[0], mid = odd ? r2 : c[1], lo = odd ? c[2] : r1;
  return fmaf(static_cast<float>(hi), 65536.f, static_cast<float>((mid << 8) + lo));
}

// ---- raw-byte operands of the 2-bit tensor-core path ------------------------------------------
// A byte of a 2-bit code word holds four codes c0 + 4 c1 + 16 c2 + 64 c3 (bits 0, 2, 4, 6).  The A
// operand takes the word and three masked copies of it, whose bytes are
//   V0 = c0 + 4 c1 + 16 c2 + 64 c3,  V1 = 4 c1 + 16 c2 + 64 c3,  V2 = 16 c2 + 64 c3,  V3 = 64 c3,
// against B operand values X0 = 64 Q0, X1 = 16 Q1 - 64 Q0, X2 = 4 Q2 - 16 Q1, X3 = Q3 - 4 Q2 built
// from the fixed-point values Q0..Q3 of the byte's four elements, so that
//   V0 X0 + V1 X1 + V2 X2 + V3 X3 = 64 (c0 Q0 + c1 Q1 + c2 Q2 + c3 Q3)
// exactly: three LOP3 per word instead of a shift and four masks.  Each X (|X| < 2^30) enters the
// tensor core as four balanced signed byte digits, one B column per digit.
__device__ __forceinline__ void variants2(uint32_t w, uint32_t (&v)[4]) {
  v[0] = w;
  v[1] = w & 0xFCFCFCFCu;
  v[2] = w & 0xF0F0F0F0u;
  v[3] = w & 0xC0C0C0C0u;
}
// Balanced signed digits of four operand values: word d holds digit d (weight 256^d) of x[m] in
// byte m.  The digits are the bytes of x + 0x80808080, each minus 128 (= xor 0x80 as an s8), and a
// 4 x 4 byte transpose gathers one digit of the four values into one word.
__device__ __forceinline__ void digit_words(const int (&x)[4], uint32_t (&wd)[4]) {
  uint32_t u[4];
#pragma unroll
  for (int m = 0; m < 4; ++m) u[m] = static_cast<uint32_t>(x[m]) + 0x80808080u;
  const uint32_t t0 = __byte_perm(u[0], u[1], 0x5140), t1 = __byte_perm(u[0], u[1], 0x7362);
  const uint32_t t2 = __byte_perm(u[2], u[3], 0x5140), t3 = __byte_perm(u[2], u[3], 0x7362);
  wd[0] = __byte_perm(t0, t2, 0x5410) ^ 0x80808080u;
  wd[1] = __byte_perm(t0, t2, 0x7632) ^ 0x80808080u;
  wd[2] = __byte_perm(t1, t3, 0x5410) ^ 0x80808080u;
  wd[3] = __byte_perm(t1, t3, 0x7632) ^ 0x80808080u;
}
// Stores the digit words of element variant `var` of operand row `row`: digit d goes to slot 3 - d
// (B column 3 - d of its query or tile), word 16 row + 4 (slot ^ (row / 2 % 4)) + var.
__device__ __forceinline__ void store_digits(uint4* rows, int row, int var, const uint32_t (&wd)[4]) {
  uint32_t* base = reinterpret_cast<uint32_t*>(rows) + 16 * row + var;
  const int sw = (row >> 1) & 3;
  base[4 * (3 ^ sw)] = wd[0];
  base[4 * (2 ^ sw)] = wd[1];
  base[4 * (1 ^ sw)] = wd[2];
  base[4 * (0 ^ sw)] = wd[3];
}
// Digit columns 3 and 2 of a tile (or query) land in even lanes t, columns 1 and 0 in odd lanes:
// each lane forms c0 * 256 + c1 for rows g and g + 8 (exact in int32: every digit sum is below
// 2^22), scales by 2^16 if even, and one exchange with lane ^ 1 leaves row g (even lane) or g + 8
// (odd lane) whole.  sc = 65536 in even lanes, 1 in odd lanes.
__device__ __forceinline__ float gather4(const int (&c)[4], bool odd, float sc) {
  const float fg = static_cast<float>(c[0] * 256 + c[1]) * sc;
  const float fh = static_cast<float>(c[2] * 256 + c[3]) * sc;
  const float r = __shfl_xor_sync(0xffffffffu, odd ? fg : fh, 1);
  return (odd ? fh : fg) + r;
}

// Largest worker whose range starts at or before unit u: start(x) = floor(U x / W).
__device__ __forceinline__ long long worker_of(long long u, long long U, long long W) {
  return ((u + 1) * W + U - 1) / U - 1;
}

// Byte vectors of the 4 sets of a packed 2-bit word (sets 1 and 3 hold four times the codes).
__device__ __forceinline__ void masks2(uint32_t w, uint32_t (&m)[4]) {
  const uint32_t w4 = w >> 4;
  m[0] = w & 0x03030303u;
  m[1] = w & 0x0C0C0C0Cu;
  m[2] = w4 & 0x03030303u;
  m[3] = w4 & 0x0C0C0C0Cu;
}
// Byte vectors of the 2 sets (low and high nibbles) of a packed 4-bit word.
__device__ __forceinline__ void masks4(uint32_t w, uint32_t (&m)[2]) {
  m[0] = w & 0x0F0F0F0Fu;
  m[1] = (w >> 4) & 0x0F0F0F0Fu;
}
// One set of one word against the three limbs of the matching operand bytes.
__device__ __forceinline__ void dot_set(uint32_t m, uint32_t L, uint32_t M, uint32_t H, int& al, int& am, int& ah,
                                        bool signed_hi) {
  al = dp4a_uu(m, L, al);
  am = dp4a_uu(m, M, am);
  ah = signed_hi ? dp4a_us(m, H, ah) : dp4a_uu(m, H, ah);
}

// ---- in-launch flush of a full residual (the decode step) ----------------------------------
// A step whose appended token fills the residual also quantizes it, in the same launch, as block
// flush_blk of the quantized arrays (section 残差バッファ: the full residual becomes one quantized
// block; section 量子化アルゴリズム: Q, s and z, by the rule of quant_rules.cuh, so the codes equal
// those of the flush kernel bit for bit).  Jobs: per KV head each K group (g_k channels over the R
// tokens) and each V group (g_v tokens over all channels); worker w takes jobs w, w + W, ... after
// its decode range.  A job moves its group through the warp's free ring buffers 8 KB at a time
// (16 cp.async of 16 bytes per lane, no registers held while they fly): a pass over the stage
// forms the extremes, a second one the codes; a group larger than 8 KB (R > 128 with g_k = 32,
// g_k > 32, g_v > 32) is staged twice, the second time from L2.  Residual slot new_slot is read
// from k_new / v_new: the warp that attends that slot writes it into the cache in this same launch.
__device__ __forceinline__ float warp_min(float v) {
  float r;
  asm volatile("redux.sync.min.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n cp.async.wait_group 0;" ::: "memory");
}

// fp16 extremes of 8 values, both halves of a half2 (exact: min and max of fp16 values)
__device__ __forceinline__ void minmax_h2(const uint4& v, __half2& lo, __half2& hi) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2 x = *reinterpret_cast<const __half2*>(&w[i]);
    lo = __hmin2(lo, x);
    hi = __hmax2(hi, x);
  }
}

template <int BITS>
struct Flusher {
  static constexpr int L = (1 << BITS) - 1;  // largest code
  static constexpr int P = 32 / BITS;        // codes per word
  static constexpr int kStage = 16;          // 16-byte chunks per lane per stage (8 KB per warp)
  const DecodeArgs& a;
  uint4* stage;  // the warp's ring buffers: slot [k][lane]
  const int lane;

  // Address of 16-byte chunk `chunk` of residual token t of KV head `head` (K or V)
  __device__ __forceinline__ const uint4* res_chunk(bool v, long long head, int t, int chunk) const {
    const uint16_t* row = t == a.new_slot ? (v ? a.v_new : a.k_new) + static_cast<size_t>(head) * kHeadDim
                                          : (v ? a.v_res : a.k_res) +
                                                (static_cast<size_t>(head) * a.residual + t) * kHeadDim;
    return reinterpret_cast<const uint4*>(row) + chunk;
  }
  // (s, z) of a group from the lanes' fp16 extremes
  __device__ __forceinline__ GroupParams group_of(__half2 lo, __half2 hi) const {
    const float l = warp_min(fminf(__low2float(lo), __high2float(lo)));
    const float h = warp_max(fmaxf(__low2float(hi), __high2float(hi)));
    return make_group(l, h, L);
  }
  // stage[k][lane] = chunk `chunk` of token tok(k), k < kStage
  template <typename Tok>
  __device__ __forceinline__ void fill(bool v, long long head, int chunk, Tok tok) const {
    __syncwarp();  // the previous stage is no longer read
#pragma unroll
    for (int k = 0; k < kStage; ++k) cp_async16(stage + k * 32 + lane, res_chunk(v, head, tok(k), chunk));
    cp_async_wait_all();
    __syncwarp();
  }

  // K group gi of `head`: channels [gi g_k, (gi + 1) g_k) over the R tokens.  Lane (s, c) holds
  // chunk c (8 channels) of tokens s, s + slots, ...; a 2-bit code word (16 channels) is the OR of
  // two lanes' halves.
  __device__ void k_group(long long head, int gi) const {
    const int R = a.residual, cpr = (1 << a.lg_gk) >> 3, slots = 32 / cpr;
    const int c = lane % cpr, s = lane / cpr, nt = R / slots;  // nt: the lane's tokens, a multiple of 16
    const int chunk = (gi << (a.lg_gk - 3)) + c;  // chunk of the row (8 channels each)
    __half2 lo = __float2half2_rn(INFINITY), hi = __float2half2_rn(-INFINITY);
    for (int k0 = 0; k0 < nt; k0 += kStage) {
      fill(false, head, chunk, [&](int k) { return s + slots * (k0 + k); });
#pragma unroll
      for (int k = 0; k < kStage; ++k) minmax_h2(stage[k * 32 + lane], lo, hi);
    }
    const GroupParams g = group_of(lo, hi);
    const size_t C = static_cast<size_t>(a.capacity);
    const int ngk = kHeadDim >> a.lg_gk;
    if (lane == 0) {
      const size_t si = (static_cast<size_t>(head) * (C / R) + a.flush_blk) * ngk + gi;
      a.fk_scale[si] = g.s_bits;
      a.fk_zero[si] = g.z_bits;
    }
    uint32_t* dst = a.fk_codes + (static_cast<size_t>(head) * C + static_cast<size_t>(a.flush_blk) * R) * (kHeadDim / P);
    Thresh2 th;
    if constexpr (BITS == 2) th = make_thresh2(g);
    for (int k0 = 0; k0 < nt; k0 += kStage) {
      if (nt > kStage) fill(false, head, chunk, [&](int k) { return s + slots * (k0 + k); });
#pragma unroll 4
      for (int k = 0; k < kStage; ++k) {
        const int t = s + slots * (k0 + k);
        const uint4 v = stage[k * 32 + lane];
        // the chunk's 8 codes at their bits of the word
        uint32_t part = BITS == 2 ? row_codes2(v, th) : quantize_row8<BITS>(v, g);
        if constexpr (BITS == 2) {  // word = chunks 2 w and 2 w + 1
          part <<= 16 * (c & 1);
          part |= __shfl_xor_sync(kFull, part, 1);
          if ((c & 1) == 0) dst[static_cast<size_t>(t) * (kHeadDim / P) + (chunk >> 1)] = part;
        } else {  // word = one chunk
          dst[static_cast<size_t>(t) * (kHeadDim / P) + chunk] = part;
        }
      }
    }
  }

  // V group vg of `head`: tokens [vg g_v, (vg + 1) g_v) over all channels, in slabs of 32 tokens.
  // Lane (h, c) holds chunk c of the slab's tokens 16 h .. 16 h + 15, i.e. whole code words (one
  // word row at 2 bits, two at 4 bits) of its 8 channels.
  __device__ void v_group(long long head, int vg) const {
    const int R = a.residual, gv = 1 << a.lg_gv, nslab = gv >> 5;
    const int c = lane & 15, h = lane >> 4;
    const int t0 = vg * gv + 16 * h;
    __half2 lo = __float2half2_rn(INFINITY), hi = __float2half2_rn(-INFINITY);
    for (int sl = 0; sl < nslab; ++sl) {
      fill(true, head, c, [&](int k) { return t0 + 32 * sl + k; });
#pragma unroll
      for (int k = 0; k < kStage; ++k) minmax_h2(stage[k * 32 + lane], lo, hi);
    }
    const GroupParams g = group_of(lo, hi);
    const size_t C = static_cast<size_t>(a.capacity);
    const size_t T0 = static_cast<size_t>(a.flush_blk) * R;  // first token of the block
    if (lane == 0) {
      const size_t si = static_cast<size_t>(head) * (C >> a.lg_gv) + ((T0 + vg * gv) >> a.lg_gv);
      a.fv_scale[si] = g.s_bits;
      a.fv_zero[si] = g.z_bits;
    }
    Thresh2 th;
    if constexpr (BITS == 2) th = make_thresh2(g);
    for (int sl = 0; sl < nslab; ++sl) {
      if (nslab > 1) fill(true, head, c, [&](int k) { return t0 + 32 * sl + k; });
      uint32_t w[16 / P][8];
#pragma unroll
      for (int r = 0; r < 16 / P; ++r)
#pragma unroll
        for (int e = 0; e < 8; ++e) w[r][e] = 0u;
      if constexpr (BITS == 2) {
        // tokens 2 a, 2 a + 1 of channels 2 e, 2 e + 1 -> one word of four byte codes; then per
        // channel the bytes of four tokens -> one 8-bit field (token k at bits 2 k)
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {  // tokens 4 q4 .. 4 q4 + 3
          uint4 v[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) v[i] = stage[(4 * q4 + i) * 32 + lane];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t A0 = __byte_perm(codes2_h2(comp(v[0], e), th), codes2_h2(comp(v[1], e), th), 0x6240);
            const uint32_t A1 = __byte_perm(codes2_h2(comp(v[2], e), th), codes2_h2(comp(v[3], e), th), 0x6240);
            w[0][2 * e] |= gather4x2(__byte_perm(A0, A1, 0x5410)) << (8 * q4);
            w[0][2 * e + 1] |= gather4x2(__byte_perm(A0, A1, 0x7632)) << (8 * q4);
          }
        }
      } else {
#pragma unroll
        for (int k = 0; k < kStage; ++k) {
          const uint4 v = stage[k * 32 + lane];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            uint32_t qa, qb;
            quantize_pair(comp(v, e), g, L, qa, qb);
            w[k / P][2 * e] |= qa << (BITS * (k % P));
            w[k / P][2 * e + 1] |= qb << (BITS * (k % P));
          }
        }
      }
#pragma unroll
      for (int r = 0; r < 16 / P; ++r) {
        const size_t row = (T0 + vg * gv + 32 * sl + 16 * h) / P + r;  // word row of the head
        uint4* dst = reinterpret_cast<uint4*>(a.fv_codes + (static_cast<size_t>(head) * (C / P) + row) * kHeadDim + 8 * c);
        dst[0] = make_uint4(w[r][0], w[r][1], w[r][2], w[r][3]);
        dst[1] = make_uint4(w[r][4], w[r][5], w[r][6], w[r][7]);
      }
    }
  }

  // Not inlined: the flush's registers get their own allocation instead of pushing the decode
  // loop's values into local memory.
  __device__ __noinline__ void run(long long worker) const {
    const int ngk = kHeadDim >> a.lg_gk, nvg = a.residual >> a.lg_gv, per_head = ngk + nvg;
    const long long jobs = static_cast<long long>(a.bh) * per_head;
    if (!dbg_check(a.flush_blk >= 0 && static_cast<long long>(a.flush_blk + 1) * a.residual <= a.capacity &&
                       a.new_slot == a.residual - 1 && a.residual % 128 == 0 && a.lg_gv >= 5,
                   a.status))
      return;
    for (long long j = worker; j < jobs; j += a.workers) {
      const long long head = j / per_head;
      const int r = static_cast<int>(j - head * per_head);
      if (r < ngk)
        k_group(head, r);
      else
        v_group(head, r - ngk);
    }
  }
};

// KC: the residual tokens' K rows are codes (online K); a separate instantiation keeps that path
// out of the register allocation of the others.  FG: fine-grained groups (2 or 4 bits, one to
// eight queries per KV head): K (s, z) per channel per g_k tokens, V (s, z) per token per g_v channels.
// FL: the decode step's in-launch flush of a full residual (base groups only).
template <int BITS, int G, bool KC, bool FG = false, bool FL = false>
struct Decoder {
  static constexpr int P = 32 / BITS;              // codes per word
  static constexpr int UT = BITS == 2 ? 128 : 64;  // tokens per quantized unit (8 KB of codes)
  static constexpr int TPL = UT / 32;              // tokens per lane (K side)
  static constexpr int ROWS = UT / P;              // V word rows per unit (8)
  static_assert(P * BITS == 32 && ROWS * P == UT, "a unit is ROWS V word rows of P tokens");
  static constexpr int kBuffers = ring_buffers<G>();
  static constexpr int GP = G == 1 ? 1 : 2;        // queries per pass over a unit's codes
  // 2 bits: the byte dot products run on the tensor cores (mma.sync); one query per KV head pairs
  // two token (channel) tiles per accumulator, several queries pair two queries per accumulator
  static constexpr bool kMma = BITS == 2;
  static constexpr bool kMma1 = kMma && G == 1;
  static constexpr bool kMmaG = kMma && G > 1 && !FG;
  static constexpr int NBLK = G / 2;  // several queries: n8 blocks of queries (2 p, 2 p + 1)

  const DecodeArgs& a;
  WarpSmem<G, FG>& S;
  const int lane;
  const long long worker, ub, ue;
  const int ngk;  // K groups per head (d / G_k)

  // per-head state.  At 2 bits lane (i, k) = (lane / 4, lane % 4) holds channels 16 i + 4 m + k
  // (m = 0..3: byte m of set k of K word i) and lane j < d / G_k holds the q sum of K group j in
  // qsum[g][0]; at 4 bits lane holds channels lane + 32 j and every lane holds all group sums.
  float qreg[4];        // one query per KV head: its channels of q; several: in shared memory (q_of)
  float qsum[G][4];
  float m[G], l[G], Z[G], o[G][4];
  // per-block state: the Q limbs in S.qw belong to (head, block) == qkey
  long long qkey;
  float invq[G], cblk[G];
  // state handed from the K half to the V half of a unit
  float alpha_[G], invv_[G], pres_[G];
  bool hasv_[G];
  bool omma_;  // o is in the tensor-core layout of several queries (see o_swap_layout)
  // FG: per K token group of the unit, 1 / Q scale and the z constant (of the query in hand); per
  // query and V channel group, the lane's part of sum_t p_t z_(t, group) and (4 bits) 1 / P scale;
  // at 2 bits o is in the FG layout while quantized units run
  float invqf[4], cblkf[4], ZF[FG ? G : 1][4], invvf[FG && BITS == 4 ? G : 1][4];
  bool ofg_;
  // heads whose partials this worker wrote (at most two: the first and the last segment)
  int pend0_, pend1_, npend_;
  // bytes per head of the code arrays and of a residual array; this lane's scale role
  const size_t code_head_bytes, res_head_bytes;
  const bool k_lane, v_lane;

  __device__ Decoder(const DecodeArgs& args, WarpSmem<G, FG>& smem, int ln, long long w, long long b, long long e)
      : a(args), S(smem), lane(ln), worker(w), ub(b), ue(e), ngk(kHeadDim >> args.lg_gk), qkey(-1),
        code_head_bytes(static_cast<size_t>(args.capacity) * (kHeadDim * BITS / 8)),
        res_head_bytes(static_cast<size_t>(args.residual) * kHeadDim * 2),
        k_lane(ln < (kHeadDim >> args.lg_gk)),
        v_lane(ln >= 8 && ln < 8 + ((UT >> args.lg_gv) > 0 ? (UT >> args.lg_gv) : 1)),
        pend0_(-1), pend1_(-1), npend_(0) {}

  // ---- half-unit addressing: half h of the warp's range is the K (h even) or V (h odd) part -----
  // A unit's K half and V half are each 4 KB and contiguous: quantized unit `local` of a head
  // starts at byte local * 4 KB of that head's code arrays, residual unit r at byte r * 4 KB of
  // its residual arrays.
  __device__ void issue_half(int h, long long head, int local) {  // lane 0 only
    const int b = h % kBuffers;
    const bool is_v = h & 1;
    const bool quant = local < a.units_q;
    // the first K half of every head the warp starts also brings the head's queries
    const bool with_q = !is_v && (h == 0 || local == 0);
    const uint32_t qbytes = with_q ? G * kHeadDim * 2 : 0u;
    const char* base = quant ? reinterpret_cast<const char*>(is_v ? a.v_codes : a.k_codes)
                             : reinterpret_cast<const char*>(is_v ? a.v_res : a.k_res);
    const size_t stride = quant ? code_head_bytes : res_head_bytes;
    const int unit = quant ? local : local - a.units_q;
    if constexpr (kDebugBuild) {  // the copy stays inside the head's arrays and the filled tokens
      bool ok = head >= 0 && head < a.bh && local >= 0 && local < a.units;
      if (KC && !quant && !is_v)
        ok = ok && a.n_quant + (unit + 1) * kResTokens <= a.capacity;
      else if (quant)
        ok = ok && (unit + 1) * UT <= a.n_quant && static_cast<size_t>(unit + 1) * kHalfBytes <= code_head_bytes;
      else
        ok = ok && unit * kResTokens < a.n_res && (unit + 1) * kResTokens <= a.residual;
      if (!dbg_check(ok, a.status)) {  // no copy: the phase completes at once on stale data
        mbar_arrive_expect_tx(&S.bar[b], 0);
        return;
      }
    }
    const char* src = base + static_cast<size_t>(head) * stride + static_cast<size_t>(unit) * kHalfBytes;
    if (KC && !quant && !is_v) {  // online K: 16 code rows from token n_quant + 16 unit
      constexpr uint32_t kRowBytes = kHeadDim * BITS / 8;
      src = reinterpret_cast<const char*>(a.k_codes) + static_cast<size_t>(head) * code_head_bytes +
            (static_cast<size_t>(a.n_quant) + static_cast<size_t>(unit) * kResTokens) * kRowBytes;
      mbar_arrive_expect_tx(&S.bar[b], kResTokens * kRowBytes + qbytes + a.debug_extra_tx);
      if (with_q) issue_q(head, b);
      bulk_g2s(S.buf[b], src, kResTokens * kRowBytes, &S.bar[b]);
      return;
    }
    mbar_arrive_expect_tx(&S.bar[b], kHalfBytes + qbytes + a.debug_extra_tx);
    if (with_q) issue_q(head, b);
    if (kMma && is_v) {
#pragma unroll
      for (int c = 0; c < kHalfBytes / kVPiece; ++c)
        bulk_g2s(S.buf[b] + c * kVPieceStride, src + c * kVPiece, kVPiece, &S.bar[b]);
    } else {
      bulk_g2s(S.buf[b], src, kHalfBytes, &S.bar[b]);
    }
  }

  // The G queries of KV head `head` (contiguous fp16 rows, 16-byte aligned) into its q slot.
  __device__ void issue_q(long long head, int b) {
    bulk_g2s(S.qraw[qslot(head)], a.q + static_cast<size_t>(head) * G * kHeadDim, G * kHeadDim * 2, &S.bar[b]);
  }
  static __device__ __forceinline__ int qslot(long long head) { return q_slots<G>() == 1 ? 0 : static_cast<int>(head & 1); }

  // (s, z) pairs of a quantized unit: lanes [0, ngk) hold K groups, lanes [8, 8 + nvg) V groups.
  // Branch-free: every lane forms both candidate indices and at most one lane group loads.
  __device__ uint32_t load_pairs(long long head, int local) const {
    const size_t ik = (static_cast<size_t>(head) * a.blocks_per_head + (local >> a.lg_units_per_blk)) * ngk +
                      (k_lane ? lane : 0);
    const size_t iv = static_cast<size_t>(head) * a.vgroups_per_head + ((local * UT) >> a.lg_gv) +
                      (v_lane ? lane - 8 : 0);
    const uint16_t* ps = k_lane ? a.k_scale + ik : a.v_scale + iv;
    const uint16_t* pz = k_lane ? a.k_zero + ik : a.v_zero + iv;
    uint32_t r = 0u;
    if (!FG && (k_lane || v_lane) && local < a.units_q &&  // FG loads its own scales per unit
        dbg_check(k_lane ? ik < static_cast<size_t>(a.bh) * a.blocks_per_head * ngk
                         : iv < static_cast<size_t>(a.bh) * a.vgroups_per_head, a.status))
      r = static_cast<uint32_t>(__ldg(ps)) | (static_cast<uint32_t>(__ldg(pz)) << 16);
    return r;
  }

  // ---- per-head state ---------------------------------------------------------------------
  __device__ void start_head(long long head) {
    __syncwarp();
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const uint16_t* qp = S.qraw[qslot(head)][g];  // landed with the head's first K half
      if constexpr (BITS == 2) {
        float part = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int c = 16 * (lane >> 2) + 4 * j + (lane & 3);
          const float v = h2f(qp[c]) * a.qscale;
          if (G == 1)
            qreg[j] = v;
          else
            S.qs[g][c] = v;
          part += v;
        }
        // the 2^(lg_gk - 2) consecutive lanes of a K group reduce its sum; lane j takes group j's
        const int span = 1 << (a.lg_gk - 2);
        for (int off = 1; off < span; off <<= 1) part += __shfl_xor_sync(kFull, part, off);
        qsum[g][0] = __shfl_sync(kFull, part, (lane & (ngk - 1)) * span);
      } else {
      float qv[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        qv[j] = h2f(qp[lane + 32 * j]) * a.qscale;
        if (G == 1)
          qreg[j] = qv[j];
        else
          S.qs[g][lane + 32 * j] = qv[j];
      }
#pragma unroll
      for (int gi = 0; gi < 4; ++gi) {
        float part = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (((32 * j) >> a.lg_gk) == gi) part += qv[j];
        qsum[g][gi] = gi < ngk ? warp_sum(part) : 0.f;
      }
      }
      m[g] = -INFINITY;
      l[g] = 0.f;
      Z[g] = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) o[g][e] = 0.f;
    }
    qkey = -1;
    omma_ = kMmaG;  // o is zero: either layout
    ofg_ = FG;
#pragma unroll
    for (int g = 0; g < (FG ? G : 1); ++g)
#pragma unroll
      for (int gc = 0; gc < 4; ++gc) ZF[g][gc] = 0.f;
    __syncwarp();
  }

  // Residual units and the merge read o in the residual layout.
  __device__ __forceinline__ void residual_layout() {
    if constexpr (kMmaG) {
      if (omma_) {
        o_swap_layout();
        omma_ = false;
      }
    }
    if constexpr (FG) {
      if (ofg_) {
        fg_to_residual_layout();
        ofg_ = false;
      }
    }
  }

  // This lane's q channel j of query g (scaled by scale * log2 e): channel 16 (lane / 4) + 4 j +
  // lane % 4 at 2 bits, lane + 32 j at 4 bits.  Several queries per KV head keep it in shared memory
  // (written by start_head) rather than in registers.
  __device__ __forceinline__ float q_of(int g, int j) const {
    if (G == 1) return qreg[j];
    const int c = BITS == 2 ? 16 * (lane >> 2) + 4 * j + (lane & 3) : lane + 32 * j;
    return S.qs[G > 1 ? g : 0][G > 1 ? c : 0];
  }

  // ---- A6 set-up for one K block: fixed-point limbs of q_c * s_g(c) -------------------------
  __device__ void build_q(uint32_t pairs) {
    __syncwarp();  // the previous block's limbs are no longer read
    if constexpr (kMma)
      build_q2_mma(pairs);
    else
      build_q4(pairs);
    __syncwarp();
  }

  // ---- tensor-core path (2 bits), raw-byte operands ------------------------------------------
  // Operand layout in shared memory, Q and P alike: word (row, slot, var) at 16 row + 4 (slot ^
  // (row / 2 % 4)) + var, for row = K code word (Q) or V word row (P) and var = the element variant
  // 0..3 of a byte.  Slot s holds digit 3 - s of the operand values; byte m of the word belongs to
  // byte m of the code words (channels 16 row + 4 m + var of Q, tokens 16 row + 4 m + var of P).  The
  // XOR spreads the four lanes t that read rows 2 t + x of one slot over four bank groups.
  //
  // An m16n8k32 tile contracts 8 code bytes (32 elements) of 16 rows (tokens or channels) against
  // the four digit columns.  With one query per KV head two tiles share one accumulator: the first
  // tile's digits sit in B columns 0..3 and the second's in 4..7, so lane (n, t) with n = lane / 4
  // reads slot n of the first tile's operand (n < 4) or of the second's (n >= 4) and the all-zero
  // operand for the other tile.  With several queries, n8 block p holds queries 2 p (columns 0..3)
  // and 2 p + 1 (columns 4..7).

  // Q operands of one K block: lane (i, k) forms variant k of K word i for bytes m = 0..3 (channels
  // 16 i + 4 m + k); the previous channel's Q is lane - 1's (variant k - 1 of the same word).
  __device__ void build_q2_mma(uint32_t pairs) {
    const int gi = (16 * (lane >> 2)) >> a.lg_gk;  // the K group of all four channels
    const float s = h2f(static_cast<uint16_t>(__shfl_sync(kFull, pairs, gi) & 0xFFFFu));
    const float z_own = k_lane ? h2f(static_cast<uint16_t>(pairs >> 16)) : 0.f;
    const int i = lane >> 2, k = lane & 3;
    const int xa = 64 >> (2 * k), xb = k ? (256 >> (2 * k)) : 0;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float qv[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) qv[j] = q_of(g, j) * s;
      const float mabs = warp_max(fmaxf(fmaxf(fabsf(qv[0]), fabsf(qv[1])), fmaxf(fabsf(qv[2]), fabsf(qv[3]))));
      const float scq = mabs > 0.f ? kQRangeRaw * fast_rcp(mabs) : 0.f;
      invq[g] = mabs * (1.0f / (64.f * kQRangeRaw));  // the operands carry 64 Q
      float c = z_own * qsum[g][0];
      c += __shfl_xor_sync(kFull, c, 1);
      c += __shfl_xor_sync(kFull, c, 2);
      cblk[g] = __shfl_sync(kFull, c, 0);
      int x[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int Q = __float2int_rn(qv[j] * scq);
        const int Qp = __shfl_up_sync(kFull, Q, 1);
        x[j] = Q * xa - Qp * xb;
      }
      uint32_t wd[4];
      digit_words(x, wd);
      store_digits(S.qw[g], i, k, wd);
    }
  }

  // Logits of the unit's 128 tokens.  Tile b of pair j holds on row g + 8 c the token
  // 16 (g / 4 + 2 c + 4 b) + 4 j + g % 4, so that after the exchange lane (g, t) holds in lg[j] the
  // logit of token 16 r + 4 j + v with r = g / 4 + 2 (t % 2) + 4 (t / 2) and v = g % 4: the four
  // tokens whose P operands variant v of word row r needs (see softmax_mma).
  __device__ void k_mma(const uint8_t* kt, float (&lg)[4]) const {
    const int g = lane >> 2, t = lane & 3;
    const int si = 8 * t + ((g & 3) ^ t);
    const uint4* pe = g < 4 ? &S.qw[0][si] : &S.zero4;   // tile 0's operand, or zero
    const uint4* po = g >= 4 ? &S.qw[0][si] : &S.zero4;  // tile 1's
    const uint4 be0 = pe[0], be1 = pe[g < 4 ? 4 : 0], bo0 = po[0], bo1 = po[g >= 4 ? 4 : 0];
    const bool odd = t & 1;
    const float sc = odd ? 1.f : 65536.f;
    const uint8_t* base = kt + (16 * (g >> 2) + (g & 3)) * 32 + 8 * t;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int c[4] = {0, 0, 0, 0};
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        const uint8_t* r0 = base + (4 * j + 64 * b) * 32;
        const uint2 wg = *reinterpret_cast<const uint2*>(r0);
        const uint2 wh = *reinterpret_cast<const uint2*>(r0 + 32 * 32);  // row g + 8: 32 tokens on
        const uint4& B0 = b ? bo0 : be0;
        const uint4& B1 = b ? bo1 : be1;
        uint32_t vg[4], vh[4];
        variants2(wg.x, vg);
        variants2(wh.x, vh);
        mma_u8s8(c, vg[0], vh[0], vg[1], vh[1], B0.x, B0.y);
        mma_u8s8(c, vg[2], vh[2], vg[3], vh[3], B0.z, B0.w);
        variants2(wg.y, vg);
        variants2(wh.y, vh);
        mma_u8s8(c, vg[0], vh[0], vg[1], vh[1], B1.x, B1.y);
        mma_u8s8(c, vg[2], vh[2], vg[3], vh[3], B1.z, B1.w);
      }
      lg[j] = fmaf(gather4(c, odd, sc), invq[0], cblk[0]);
    }
  }

  // Online softmax of the unit and its P operands, P = p s scaled by the bound 2^(mu - m) s_max
  // (reading R16).  Lane (g, t) holds tokens 16 r + 4 m + v (m = 0..3) of word row r, which lie in
  // one V group (V groups span at least 32 tokens); the previous token's P is lane - 4's.
  __device__ void softmax_mma(uint32_t pairs, const float (&lg)[4]) {
    const int g = lane >> 2, t = lane & 3;
    const int r = (g >> 2) + 2 * (t & 1) + 4 * (t >> 1), v = g & 3;
    const float mu = warp_max(fmaxf(fmaxf(lg[0], lg[1]), fmaxf(lg[2], lg[3])));
    const float smax = warp_max(v_lane ? h2f(static_cast<uint16_t>(pairs & 0xFFFFu)) : 0.f);
    const float m_new = fmaxf(m[0], mu);
    const float alpha = fast_exp2(m[0] - m_new);
    const float d = mu - m_new;  // <= 0: the unit's largest weight is 2^d
    const bool hv = d > -64.f && smax > 0.f;
    const uint32_t vp = __shfl_sync(kFull, pairs, 8 + ((16 * r) >> a.lg_gv));
    const float sv = h2f(static_cast<uint16_t>(vp & 0xFFFFu)), zv = h2f(static_cast<uint16_t>(vp >> 16));
    const float f = hv ? (kPRange * fast_rcp(smax)) * fast_exp2(-d) * sv : 0.f;
    const int xa = 64 >> (2 * v), xb = v ? (256 >> (2 * v)) : 0;
    float psum = 0.f;
    int x[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float p = fast_exp2(lg[j] - m_new);
      psum += p;
      const int P = static_cast<int>(__float2uint_rn(p * f));
      const int Pp = __shfl_up_sync(kFull, P, 4);
      x[j] = P * xa - Pp * xb;
    }
    m[0] = m_new;
    l[0] = fmaf(l[0], alpha, psum);
    Z[0] = fmaf(Z[0], alpha, psum * zv);
    alpha_[0] = alpha;
    hasv_[0] = hv;
    invv_[0] = hv ? fast_exp2(d) * smax * (1.0f / (64.f * kPRange)) : 0.f;
    uint32_t wd[4];
    digit_words(x, wd);
    store_digits(S.pw[0], r, v, wd);
  }

  // P . codes of the unit.  Tile pair v holds channels 16 g' + 8 b + 4 c + v (tile 2 v + b, row
  // g' + 8 c) as rows; lane (g, t) reads V word rows 2 t and 2 t + 1 of channels 16 g .. 16 g + 15
  // (four 16-byte loads per row).  After the exchange the lane holds channel 4 lane + v of tile
  // pair v, the channel it accumulates in o[0][v].  Rows 2 t and 2 t + 1 are piece t of the buffer.
  __device__ void v_mma(const uint8_t* vt) {
    static_assert(P == 16 && ROWS == 8, "2-bit units: 8 V word rows of 16 tokens");
    const int g = lane >> 2, t = lane & 3;
    const int si = 8 * t + ((g & 3) ^ t);
    const uint4* pe = g < 4 ? &S.pw[0][si] : &S.zero4;
    const uint4* po = g >= 4 ? &S.pw[0][si] : &S.zero4;
    const uint4 be[2] = {pe[0], pe[g < 4 ? 4 : 0]}, bo[2] = {po[0], po[g >= 4 ? 4 : 0]};
    const bool odd = t & 1;
    const float sc = odd ? 1.f : 65536.f;
    int cv[4][4];
#pragma unroll
    for (int v = 0; v < 4; ++v) cv[v][0] = cv[v][1] = cv[v][2] = cv[v][3] = 0;
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      const uint8_t* rowp = vt + t * kVPieceStride + x * 512 + 64 * g;
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        const uint4 wlo = *reinterpret_cast<const uint4*>(rowp + 32 * b);
        const uint4 whi = *reinterpret_cast<const uint4*>(rowp + 32 * b + 16);
        const uint4& B = b ? bo[x] : be[x];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          uint32_t vg[4], vh[4];
          variants2(comp(wlo, v), vg);
          variants2(comp(whi, v), vh);
          mma_u8s8(cv[v], vg[0], vh[0], vg[1], vh[1], B.x, B.y);
          mma_u8s8(cv[v], vg[2], vh[2], vg[3], vh[3], B.z, B.w);
        }
      }
    }
#pragma unroll
    for (int v = 0; v < 4; ++v) o[0][v] = fmaf(o[0][v], alpha_[0], gather4(cv[v], odd, sc) * invv_[0]);
  }

  // 4 bits: lane holds channels lane + 32 j; each byte of a limb word is stored on its own.
  __device__ void build_q4(uint32_t pairs) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float qv[4], mabs = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int gi = (32 * j) >> a.lg_gk;
        const float s = h2f(static_cast<uint16_t>(__shfl_sync(kFull, pairs, gi) & 0xFFFFu));
        qv[j] = q_of(g, j) * s;
        mabs = fmaxf(mabs, fabsf(qv[j]));
      }
      mabs = warp_max(mabs);
      // |Q| <= 2^23 - 61: the margin keeps the rounded largest element below 2^23, where the
      // signed top limb would wrap (rcp and the product add at most 3 * 2^-22 relative)
      const float scq = mabs > 0.f ? kQRange * fast_rcp(mabs) : 0.f;
      invq[g] = mabs * (1.0f / kQRange);
      float c = 0.f;
#pragma unroll
      for (int gi = 0; gi < 4; ++gi) {
        if (gi < ngk) {
          const float z = h2f(static_cast<uint16_t>(__shfl_sync(kFull, pairs, gi) >> 16));
          c = fmaf(z, qsum[g][gi], c);
        }
      }
      cblk[g] = c;
      uint8_t* qwb = reinterpret_cast<uint8_t*>(S.qw[g]);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int ch = lane + 32 * j;
        const int word = ch >> 3, k = ch & 1, mb = (ch >> 1) & 3;  // word c/8, set c%2, byte (c%8)/2
        const int Q = __float2int_rn(qv[j] * scq);
        uint8_t* base = qwb + ((word * 3) * 2 + k) * 4 + mb;  // limb b of word i: 8 bytes at (3 i + b) * 8
        base[0] = static_cast<uint8_t>(Q & 255);
        base[8] = static_cast<uint8_t>((Q >> 8) & 255);
        base[16] = static_cast<uint8_t>((Q >> 16) & 255);
      }
    }
  }

  // ---- fine-grained groups (FG) -----------------------------------------------------------------
  // Section KVキャッシュの分布特性: the K range is taken along each channel (one (s, z) per channel per
  // g_k tokens: k_scale [bh][C / g_k][128]) and the V range along each token (one (s, z) per token per
  // g_v channels: v_scale [bh][C][128 / g_v]).  K: the Q limbs q_c s_(u, c) and the constant
  // sum_c q_c z_(u, c) are formed for each token group u of the unit.  V: P_(t, gc) = p_t s_(t, gc)
  // per channel group gc, one limb array per (query, group); sum_t p_t z_(t, gc) stays per group (ZF)
  // until fg_to_residual_layout() adds it to the group's channels.  Queries are taken one at a time:
  // each pass over a unit's codes serves one query.
  //
  // 2 bits (tensor cores, three limbs): tile pair j of the K side holds tokens 32 j .. 32 j + 31 (one
  // token group, g_k >= 32).  On the V side tile pair v holds channels 32 v .. 32 v + 31 (group
  // 32 v / g_v) with tile (v, b) row g' + 8 c on channel 32 v + 16 b + 2 g' + c, so after the exchange
  // lane (g, t) holds channel 32 v + 16 (t / 2) + 2 g + t % 2 in o[q][v].
  // 4 bits (dp4a): lane holds tokens lane + 32 j (j = 0, 1: token groups j when g_k = 32, else one)
  // and channels 4 lane .. 4 lane + 3 (one channel group) of the output.

  static __device__ __forceinline__ float sel4(const float (&x)[4], int i) {
    return i == 0 ? x[0] : (i == 1 ? x[1] : (i == 2 ? x[2] : x[3]));
  }

  // K (s, z) index of channel c in token group u of the head (FG layout), bounds-checked in a debug build.
  __device__ __forceinline__ size_t fg_kidx(long long head, size_t u, int c) const {
    const size_t rows = static_cast<size_t>(a.capacity) >> a.lg_gk;
    const size_t i = (static_cast<size_t>(head) * rows + u) * kHeadDim + c;
    return dbg_check(i < static_cast<size_t>(a.bh) * rows * kHeadDim, a.status) ? i : 0;
  }

  __device__ void fg_k(int gq, const uint8_t* kt, long long head, int local) {
    const int ngt = UT >> a.lg_gk;  // K token groups in the unit: 4, 2 or 1
    const size_t u0 = (static_cast<size_t>(local) * UT) >> a.lg_gk;
    const int i = lane >> 2, kk = lane & 3, sw = (i >> 1) & 3;
    __syncwarp();  // the previous pass's limbs are no longer read
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (u < ngt) {
        float qv[4], qz = 0.f;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const size_t ci = fg_kidx(head, u0 + u, 16 * i + 4 * m + kk);
          const float sk = h2f(__ldg(a.k_scale + ci)), zk = h2f(__ldg(a.k_zero + ci));
          const float qm = q_of(gq, m);
          qv[m] = qm * sk;
          qz = fmaf(qm, zk, qz);
        }
        const float mabs = warp_max(fmaxf(fmaxf(fabsf(qv[0]), fabsf(qv[1])), fmaxf(fabsf(qv[2]), fabsf(qv[3]))));
        const float scq = mabs > 0.f ? kQRangeBal * fast_rcp(mabs) : 0.f;
        invqf[u] = mabs * (1.0f / kQRangeBal);
        cblkf[u] = warp_sum(qz);
        const float f = scq * ((lane & 1) ? 0.25f : 1.f);
        uint32_t Q[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) Q[m] = static_cast<uint32_t>(__float2int_rn(qv[m] * f));
        uint32_t* row = reinterpret_cast<uint32_t*>(S.qw[u]) + 16 * i + kk;
        row[4 * (0 ^ sw)] = pick_bytes(Q[0] + 32896u, Q[1] + 32896u, Q[2] + 32896u, Q[3] + 32896u, 2);
        row[4 * (1 ^ sw)] = pick_bytes(Q[0] + 128u, Q[1] + 128u, Q[2] + 128u, Q[3] + 128u, 1);
        row[4 * (2 ^ sw)] = pick_bytes(Q[0], Q[1], Q[2], Q[3], 0);
      }
    }
    __syncwarp();
    const int g = lane >> 2, t = lane & 3;
    const int se = g < 4 ? g : 3, so = g >= 4 ? g - 4 : 3;
    const bool odd = t & 1;
    float lg[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int u = (32 * j) >> a.lg_gk;
      const uint4 be0 = S.qw[u][8 * t + (se ^ t)], be1 = S.qw[u][8 * t + 4 + (se ^ t)];
      const uint4 bo0 = S.qw[u][8 * t + (so ^ t)], bo1 = S.qw[u][8 * t + 4 + (so ^ t)];
      int c[4] = {0, 0, 0, 0};
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        const uint8_t* r0 = kt + (32 * j + 16 * b + g) * 32 + 8 * t;
        const uint2 wg = *reinterpret_cast<const uint2*>(r0);
        const uint2 wh = *reinterpret_cast<const uint2*>(r0 + 8 * 32);
        const uint4& B0 = b ? bo0 : be0;
        const uint4& B1 = b ? bo1 : be1;
        uint32_t mg[4], mh[4];
        masks2(wg.x, mg);
        masks2(wh.x, mh);
        mma_u8s8(c, mg[0], mh[0], mg[1], mh[1], B0.x, B0.y);
        mma_u8s8(c, mg[2], mh[2], mg[3], mh[3], B0.z, B0.w);
        masks2(wg.y, mg);
        masks2(wh.y, mh);
        mma_u8s8(c, mg[0], mh[0], mg[1], mh[1], B1.x, B1.y);
        mma_u8s8(c, mg[2], mh[2], mg[3], mh[3], B1.z, B1.w);
      }
      lg[j] = fmaf(gather_limbs(c, odd), sel4(invqf, u), sel4(cblkf, u));
    }
    softmax_fg(gq, head, local, lg);
  }

  // Online softmax of query gq over the unit and its P limbs for each V channel group.  The lane's
  // token 32 j + 16 (t / 2) + 8 (t % 2) + g has one (s, z) per channel group.
  __device__ void softmax_fg(int gq, long long head, int local, const float (&lg)[4]) {
    const int g = lane >> 2, t = lane & 3;
    const int ngv = kHeadDim >> a.lg_gv;
    float sv[4][4], zv[4][4], smax_l = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const size_t tok = static_cast<size_t>(head) * a.capacity + static_cast<size_t>(local) * UT + 32 * j +
                         16 * (t >> 1) + 8 * (t & 1) + g;
      const bool in = dbg_check(tok < static_cast<size_t>(a.bh) * a.capacity, a.status);
#pragma unroll
      for (int gc = 0; gc < 4; ++gc) {
        sv[j][gc] = gc < ngv && in ? h2f(__ldg(a.v_scale + tok * ngv + gc)) : 0.f;
        zv[j][gc] = gc < ngv && in ? h2f(__ldg(a.v_zero + tok * ngv + gc)) : 0.f;
        smax_l = fmaxf(smax_l, sv[j][gc]);
      }
    }
    const float mu = warp_max(fmaxf(fmaxf(lg[0], lg[1]), fmaxf(lg[2], lg[3])));
    const float smax = warp_max(smax_l);
    const float m_new = fmaxf(m[gq], mu);
    const float alpha = fast_exp2(m[gq] - m_new);
    const float d = mu - m_new;
    const bool hv = d > -64.f && smax > 0.f;
    const float fb = hv ? (kPRange * fast_rcp(smax)) * fast_exp2(-d) * ((g & 1) ? 0.25f : 1.f) : 0.f;
    float psum = 0.f, zl[4] = {0.f, 0.f, 0.f, 0.f};
    const int boff = 64 * (t >> 1) + 4 * (g & 3) + 2 * (t & 1) + (g >> 2);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float p = fast_exp2(lg[j] - m_new);
      psum += p;
#pragma unroll
      for (int gc = 0; gc < 4; ++gc) {
        if (gc < ngv) {
          zl[gc] = fmaf(p, zv[j][gc], zl[gc]);
          const uint32_t P = __float2uint_rn(p * (sv[j][gc] * fb));
          uint8_t* pb = reinterpret_cast<uint8_t*>(S.pw[4 * gq + gc]) + boff + 128 * j;
          pb[16 * (0 ^ j)] = static_cast<uint8_t>(P >> 16);
          pb[16 * (1 ^ j)] = static_cast<uint8_t>(P >> 8);
          pb[16 * (2 ^ j)] = static_cast<uint8_t>(P);
        }
      }
    }
    m[gq] = m_new;
    l[gq] = fmaf(l[gq], alpha, psum);
    Z[gq] *= alpha;
#pragma unroll
    for (int gc = 0; gc < 4; ++gc) ZF[gq][gc] = fmaf(ZF[gq][gc], alpha, zl[gc]);
    alpha_[gq] = alpha;
    hasv_[gq] = hv;
    invv_[gq] = hv ? fast_exp2(d) * smax * (1.0f / kPRange) : 0.f;
  }

  __device__ void v_mma_fg(int gq, const uint8_t* vt) {
    const int g = lane >> 2, t = lane & 3;
    const int se = g < 4 ? g : 3, so = g >= 4 ? g - 4 : 3;
    const bool odd = t & 1;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int gc = (32 * v) >> a.lg_gv;
      int cv[4] = {0, 0, 0, 0};
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        const uint4 be = S.pw[4 * gq + gc][8 * t + 4 * x + (se ^ t)], bo = S.pw[4 * gq + gc][8 * t + 4 * x + (so ^ t)];
        const uint8_t* rowp = vt + t * kVPieceStride + x * 512 + 4 * (32 * v + 2 * g);
        const uint2 w0 = *reinterpret_cast<const uint2*>(rowp);           // tile (v, 0): rows g, g + 8
        const uint2 w1 = *reinterpret_cast<const uint2*>(rowp + 4 * 16);  // tile (v, 1)
        uint32_t mg[4], mh[4];
        masks2(w0.x, mg);
        masks2(w0.y, mh);
        mma_u8u8(cv, mg[0], mh[0], mg[1], mh[1], be.x, be.y);
        mma_u8u8(cv, mg[2], mh[2], mg[3], mh[3], be.z, be.w);
        masks2(w1.x, mg);
        masks2(w1.y, mh);
        mma_u8u8(cv, mg[0], mh[0], mg[1], mh[1], bo.x, bo.y);
        mma_u8u8(cv, mg[2], mh[2], mg[3], mh[3], bo.z, bo.w);
      }
      o[gq][v] = fmaf(o[gq][v], alpha_[gq], gather_limbs(cv, odd) * invv_[gq]);
    }
  }

  // 4 bits: the Q limbs of query gq for the unit's token groups (S.qw[jg], layout of build_q4),
  // then the dot products of the lane's tokens lane + 32 j against their group's limbs.
  __device__ void fg4_k(int gq, const uint8_t* kt, long long head, int local) {
    const int ngt = (UT >> a.lg_gk) > 0 ? (UT >> a.lg_gk) : 1;  // 2 when g_k = 32, else 1
    const size_t u0 = (static_cast<size_t>(local) * UT) >> a.lg_gk;
    __syncwarp();  // the previous pass's limbs are no longer read
#pragma unroll
    for (int jg = 0; jg < 2; ++jg) {
      if (jg < ngt) {
        float qv[4], qz = 0.f, mabs = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const size_t ci = fg_kidx(head, u0 + jg, lane + 32 * j);
          const float qj = q_of(gq, j);
          qv[j] = qj * h2f(__ldg(a.k_scale + ci));
          qz = fmaf(qj, h2f(__ldg(a.k_zero + ci)), qz);
          mabs = fmaxf(mabs, fabsf(qv[j]));
        }
        mabs = warp_max(mabs);
        const float scq = mabs > 0.f ? kQRange * fast_rcp(mabs) : 0.f;
        invqf[jg] = mabs * (1.0f / kQRange);
        cblkf[jg] = warp_sum(qz);
        uint8_t* qwb = reinterpret_cast<uint8_t*>(S.qw[jg]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int ch = lane + 32 * j;
          const int word = ch >> 3, k = ch & 1, mb = (ch >> 1) & 3;
          const int Q = __float2int_rn(qv[j] * scq);
          uint8_t* base = qwb + ((word * 3) * 2 + k) * 4 + mb;
          base[0] = static_cast<uint8_t>(Q & 255);
          base[8] = static_cast<uint8_t>((Q >> 8) & 255);
          base[16] = static_cast<uint8_t>((Q >> 16) & 255);
        }
      }
    }
    __syncwarp();
    int al[TPL], am[TPL], ah[TPL];
#pragma unroll
    for (int j = 0; j < TPL; ++j) al[j] = am[j] = ah[j] = 0;
#pragma unroll 1
    for (int qq = 0; qq < 4; ++qq) {
      const int cq = (qq + (lane >> 1)) & 3;  // bank-conflict-free chunk order
      uint4 kw[TPL];
#pragma unroll
      for (int j = 0; j < TPL; ++j) kw[j] = *reinterpret_cast<const uint4*>(kt + (lane + 32 * j) * 64 + 16 * cq);
#pragma unroll
      for (int ii = 0; ii < 4; ++ii) {
#pragma unroll
        for (int j = 0; j < TPL; ++j) {
          uint32_t mk[2];
          masks4(comp(kw[j], ii), mk);
          const uint2* qrow = reinterpret_cast<const uint2*>(S.qw[ngt == 2 ? j : 0]) + 12 * cq + ii * 3;
          const uint2 QL = qrow[0], QM = qrow[1], QH = qrow[2];
          dot_set(mk[0], QL.x, QM.x, QH.x, al[j], am[j], ah[j], true);
          dot_set(mk[1], QL.y, QM.y, QH.y, al[j], am[j], ah[j], true);
        }
      }
    }
    float lg[TPL];
#pragma unroll
    for (int j = 0; j < TPL; ++j) {  // token group of token j: j when g_k = 32, else 0 (no runtime index)
      const bool own = ngt == 2 && j == 1;
      lg[j] = fmaf(combine_limbs(ah[j], am[j], al[j]), own ? invqf[1] : invqf[0], own ? cblkf[1] : cblkf[0]);
    }
    softmax4_fg(gq, head, local, lg);
  }

  // 4 bits: online softmax of query gq and its P limbs per V channel group (layout of softmax4),
  // each group scaled by its exact maximum.
  __device__ void softmax4_fg(int gq, long long head, int local, const float (&lg)[TPL]) {
    const int ngv = kHeadDim >> a.lg_gv;
    float mu = lg[0];
#pragma unroll
    for (int j = 1; j < TPL; ++j) mu = fmaxf(mu, lg[j]);
    mu = warp_max(mu);
    const float m_new = fmaxf(m[gq], mu);
    const float alpha = fast_exp2(m[gq] - m_new);
    float p[TPL], psum = 0.f;
#pragma unroll
    for (int j = 0; j < TPL; ++j) {
      p[j] = fast_exp2(lg[j] - m_new);
      psum += p[j];
    }
#pragma unroll
    for (int gc = 0; gc < 4; ++gc) {
      float zl = 0.f, mv = 0.f, pp[TPL];
      if (gc < ngv) {
#pragma unroll
        for (int j = 0; j < TPL; ++j) {
          const size_t tok = static_cast<size_t>(head) * a.capacity + static_cast<size_t>(local) * UT + lane + 32 * j;
          const bool in = dbg_check(tok < static_cast<size_t>(a.bh) * a.capacity, a.status);
          const float sv = in ? h2f(__ldg(a.v_scale + tok * ngv + gc)) : 0.f;
          const float zv = in ? h2f(__ldg(a.v_zero + tok * ngv + gc)) : 0.f;
          zl = fmaf(p[j], zv, zl);
          pp[j] = p[j] * sv;
          mv = fmaxf(mv, pp[j]);
        }
      }
      mv = warp_max(mv);  // every lane joins: the group count is warp-uniform
      if (gc < ngv) {
        const float scv = mv > 0.f ? kPRange * fast_rcp(mv) : 0.f;
        invvf[gq][gc] = mv * (1.0f / kPRange);
        uint8_t* pwb = reinterpret_cast<uint8_t*>(S.pw[4 * gq + gc]);
#pragma unroll
        for (int j = 0; j < TPL; ++j) {
          const int t = lane + 32 * j;
          const int row = t >> 3, k = t & 1, mb = (t >> 1) & 3;
          const uint32_t Pq = __float2uint_rn(pp[j] * scv);
          uint8_t* base = pwb + ((row * 3) * 2 + k) * 4 + mb;
          base[0] = static_cast<uint8_t>(Pq & 255u);
          base[8] = static_cast<uint8_t>((Pq >> 8) & 255u);
          base[16] = static_cast<uint8_t>((Pq >> 16) & 255u);
        }
        ZF[gq][gc] = fmaf(ZF[gq][gc], alpha, zl);
      }
    }
    m[gq] = m_new;
    l[gq] = fmaf(l[gq], alpha, psum);
    Z[gq] *= alpha;
    alpha_[gq] = alpha;
  }

  // 4 bits: P . codes of query gq; the lane's channels 4 lane .. 4 lane + 3 lie in one V channel group.
  __device__ void fg4_v(int gq, const uint8_t* vt) {
    const int gcl = (4 * lane) >> a.lg_gv;
    const uint2* pw2 = reinterpret_cast<const uint2*>(S.pw[4 * gq + gcl]);
    int vl[4], vm[4], vh[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) vl[e] = vm[e] = vh[e] = 0;
#pragma unroll 2
    for (int r = 0; r < ROWS; ++r) {
      const uint4 vw = *reinterpret_cast<const uint4*>(vt + r * 512 + 16 * lane);
      const uint2 PL = pw2[r * 3 + 0], PM = pw2[r * 3 + 1], PH = pw2[r * 3 + 2];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        uint32_t mv4[2];
        masks4(comp(vw, e), mv4);
        dot_set(mv4[0], PL.x, PM.x, PH.x, vl[e], vm[e], vh[e], false);
        dot_set(mv4[1], PL.y, PM.y, PH.y, vl[e], vm[e], vh[e], false);
      }
    }
    const float iv = sel4(invvf[gq], gcl);
#pragma unroll
    for (int e = 0; e < 4; ++e) o[gq][e] = fmaf(o[gq][e], alpha_[gq], combine_limbs(vh[e], vm[e], vl[e]) * iv);
  }

  // o to the residual layout (lane l: channels 4 l .. 4 l + 3; at 4 bits it is already there), with
  // each V channel group's z term added to its channels.
  __device__ void fg_to_residual_layout() {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int gq = 0; gq < G; ++gq) {
      float zs[4];
#pragma unroll
      for (int gc = 0; gc < 4; ++gc) zs[gc] = warp_sum(ZF[gq][gc]);
      const float zc = sel4(zs, (4 * lane) >> a.lg_gv);
      if constexpr (BITS == 2) {
        __syncwarp();
#pragma unroll
        for (int v = 0; v < 4; ++v) S.oscr[32 * v + 16 * (t >> 1) + 2 * g + (t & 1)] = o[gq][v];
        __syncwarp();
        const float4 ov = *reinterpret_cast<const float4*>(S.oscr + 4 * lane);
        o[gq][0] = ov.x;
        o[gq][1] = ov.y;
        o[gq][2] = ov.z;
        o[gq][3] = ov.w;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) o[gq][e] += zc;
#pragma unroll
      for (int gc = 0; gc < 4; ++gc) ZF[gq][gc] = 0.f;
    }
    __syncwarp();
  }

  // ---- tensor-core path, several queries per KV head ------------------------------------------
  // B column n of n8 block p reads slot n % 4 of query 2 p + n / 4, so one accumulator holds the
  // four digit columns of queries 2 p (columns 0..3) and 2 p + 1 (columns 4..7) for one 16-row tile.
  // After the exchange a lane holds query 2 p + t / 2 of row g + 8 (t % 2).
  //
  // Output layout while quantized units run: o[2 p + b][v] of lane (g, t) holds query 2 p + t / 2,
  // channel 16 g + 8 b + 4 (t % 2) + v.  o_swap_layout() turns it into the layout of the residual
  // path and the merge (o[q][e]: query q, channel 4 lane + e) and back: it is an involution.

  // Logits of the unit's 128 tokens for every query.  Tile tau holds on row g + 8 c the token
  // 16 (g / 4 + 2 c + 4 (tau / 4)) + 4 (tau % 4) + g % 4; lg[p][tau] is the logit of query
  // 2 p + t / 2 for token 16 (r0 + 4 (tau / 4)) + 4 (tau % 4) + v, r0 = g / 4 + 2 (t % 2), v = g % 4.
  __device__ void k_mma_g(const uint8_t* kt, float (&lg)[NBLK][8]) const {
    const int g = lane >> 2, t = lane & 3, qh = g >> 2, sl = (g & 3) ^ t;
    const bool odd = t & 1;
    const float sc = odd ? 1.f : 65536.f;
    uint4 B[NBLK][2];
#pragma unroll
    for (int p = 0; p < NBLK; ++p) {
      B[p][0] = S.qw[2 * p + qh][8 * t + sl];
      B[p][1] = S.qw[2 * p + qh][8 * t + 4 + sl];
    }
    float iq[NBLK], cb[NBLK];
#pragma unroll
    for (int p = 0; p < NBLK; ++p) {
      iq[p] = (t >> 1) ? invq[2 * p + 1] : invq[2 * p];
      cb[p] = (t >> 1) ? cblk[2 * p + 1] : cblk[2 * p];
    }
    const uint8_t* base = kt + (16 * (g >> 2) + (g & 3)) * 32 + 8 * t;
#pragma unroll
    for (int tau = 0; tau < 8; ++tau) {
      const uint8_t* r0 = base + (64 * (tau >> 2) + 4 * (tau & 3)) * 32;
      const uint2 wg = *reinterpret_cast<const uint2*>(r0);
      const uint2 wh = *reinterpret_cast<const uint2*>(r0 + 32 * 32);  // row g + 8: 32 tokens on
      int c[NBLK][4];
#pragma unroll
      for (int p = 0; p < NBLK; ++p) c[p][0] = c[p][1] = c[p][2] = c[p][3] = 0;
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        uint32_t vg[4], vh[4];
        variants2(w ? wg.y : wg.x, vg);
        variants2(w ? wh.y : wh.x, vh);
#pragma unroll
        for (int p = 0; p < NBLK; ++p) {
          mma_u8s8(c[p], vg[0], vh[0], vg[1], vh[1], B[p][w].x, B[p][w].y);
          mma_u8s8(c[p], vg[2], vh[2], vg[3], vh[3], B[p][w].z, B[p][w].w);
        }
      }
#pragma unroll
      for (int p = 0; p < NBLK; ++p) lg[p][tau] = fmaf(gather4(c[p], odd, sc), iq[p], cb[p]);
    }
  }

  // Online softmax of every query over the unit and the P operands of each query (bound scaling as
  // on the other paths).  Lane (g, t) holds, for query 2 p + t / 2, tokens 16 r + 4 m + v of word
  // rows r = r0 and r0 + 4 (tiles tau = 4 h + m): each row lies in one V group; the previous token's
  // P is lane - 4's.
  __device__ void softmax_mma_g(uint32_t pairs, const float (&lg)[NBLK][8]) {
    const int g = lane >> 2, t = lane & 3, h = t >> 1;
    const int r0 = (g >> 2) + 2 * (t & 1), v = g & 3;
    const int xa = 64 >> (2 * v), xb = v ? (256 >> (2 * v)) : 0;
    const float smax = warp_max(v_lane ? h2f(static_cast<uint16_t>(pairs & 0xFFFFu)) : 0.f);
    const float kinv = smax > 0.f ? kPRange * fast_rcp(smax) : 0.f;
    float sv[2], zv[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const uint32_t vp = __shfl_sync(kFull, pairs, 8 + ((16 * (r0 + 4 * hh)) >> a.lg_gv));
      sv[hh] = h2f(static_cast<uint16_t>(vp & 0xFFFFu));
      zv[hh] = h2f(static_cast<uint16_t>(vp >> 16));
    }
#pragma unroll
    for (int p = 0; p < NBLK; ++p) {
      float mloc = lg[p][0];
#pragma unroll
      for (int tau = 1; tau < 8; ++tau) mloc = fmaxf(mloc, lg[p][tau]);
      float mn_l = 0.f, fb = 0.f;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int q = 2 * p + e;
        const float mu = warp_max(h == e ? mloc : -INFINITY);
        const float m_new = fmaxf(m[q], mu);
        const float d = mu - m_new;
        const bool hv = d > -64.f && smax > 0.f;
        alpha_[q] = fast_exp2(m[q] - m_new);
        hasv_[q] = hv;
        invv_[q] = hv ? fast_exp2(d) * smax * (1.0f / (64.f * kPRange)) : 0.f;
        m[q] = m_new;
        if (h == e) {
          mn_l = m_new;
          fb = hv ? kinv * fast_exp2(-d) : 0.f;
        }
      }
      float psum = 0.f, zsum = 0.f;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const float f = sv[hh] * fb;
        float ph = 0.f;
        int x[4];
#pragma unroll
        for (int mm = 0; mm < 4; ++mm) {
          const float pv = fast_exp2(lg[p][4 * hh + mm] - mn_l);
          ph += pv;
          const int P = static_cast<int>(__float2uint_rn(pv * f));
          const int Pp = __shfl_up_sync(kFull, P, 4);
          x[mm] = P * xa - Pp * xb;
        }
        psum += ph;
        zsum = fmaf(ph, zv[hh], zsum);
        uint32_t wd[4];
        digit_words(x, wd);
        store_digits(S.pw[2 * p + h], r0 + 4 * hh, v, wd);
      }
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int q = 2 * p + e;
        l[q] = fmaf(l[q], alpha_[q], h == e ? psum : 0.f);
        Z[q] = fmaf(Z[q], alpha_[q], h == e ? zsum : 0.f);
      }
    }
  }

  // P . codes of the unit for every query.  Tile (v, b) holds channels 16 g' + 8 b + 4 c + v (row
  // g' + 8 c); lane (g, t) reads V word rows 2 t + x of channels 16 g .. 16 g + 15.  Per tile column b
  // the lane's eight V words are read once and the accumulators live for one v at a time.
  __device__ void v_mma_g(const uint8_t* vt) {
    const int g = lane >> 2, t = lane & 3, qh = g >> 2, sl = (g & 3) ^ t;
    const bool odd = t & 1;
    const float sc = odd ? 1.f : 65536.f;
    uint4 B[NBLK][2];
#pragma unroll
    for (int p = 0; p < NBLK; ++p) {
      B[p][0] = S.pw[2 * p + qh][8 * t + sl];
      B[p][1] = S.pw[2 * p + qh][8 * t + 4 + sl];
    }
    float al[NBLK], iv[NBLK];
#pragma unroll
    for (int p = 0; p < NBLK; ++p) {
      al[p] = (t >> 1) ? alpha_[2 * p + 1] : alpha_[2 * p];
      iv[p] = (t >> 1) ? invv_[2 * p + 1] : invv_[2 * p];
    }
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      uint4 wlo[2], whi[2];
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        const uint8_t* rowp = vt + t * kVPieceStride + x * 512 + 64 * g;
        wlo[x] = *reinterpret_cast<const uint4*>(rowp + 32 * b);
        whi[x] = *reinterpret_cast<const uint4*>(rowp + 32 * b + 16);
      }
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        int acc[NBLK][4];
#pragma unroll
        for (int p = 0; p < NBLK; ++p) acc[p][0] = acc[p][1] = acc[p][2] = acc[p][3] = 0;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          uint32_t vg[4], vh[4];
          variants2(comp(wlo[x], v), vg);
          variants2(comp(whi[x], v), vh);
#pragma unroll
          for (int p = 0; p < NBLK; ++p) {
            mma_u8s8(acc[p], vg[0], vh[0], vg[1], vh[1], B[p][x].x, B[p][x].y);
            mma_u8s8(acc[p], vg[2], vh[2], vg[3], vh[3], B[p][x].z, B[p][x].w);
          }
        }
#pragma unroll
        for (int p = 0; p < NBLK; ++p)
          o[2 * p + b][v] = fmaf(o[2 * p + b][v], al[p], gather4(acc[p], odd, sc) * iv[p]);
      }
    }
  }

  // Swaps o[2 p + 1 - t / 2][v] with lane t ^ 2: the tensor-core layout <-> the residual layout.
  __device__ void o_swap_layout() {
    const bool h = (lane >> 1) & 1;
#pragma unroll
    for (int p = 0; p < NBLK; ++p)
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const float y = __shfl_xor_sync(kFull, h ? o[2 * p][v] : o[2 * p + 1][v], 2);
        if (h)
          o[2 * p][v] = y;
        else
          o[2 * p + 1][v] = y;
      }
  }

  // ---- A6 at 4 bits: integer dot products of TPL tokens per lane, for every query of the KV head
  // (each code word is unpacked once) -----------------------------------------------------------------
  // Queries g0 .. g0 + GP - 1 (the accumulators of one pass).
  __device__ void k_dot(const uint8_t* kt, int g0, int (&al)[GP][TPL], int (&am)[GP][TPL], int (&ah)[GP][TPL]) const {
#pragma unroll
    for (int g = 0; g < GP; ++g)
#pragma unroll
      for (int j = 0; j < TPL; ++j) al[g][j] = am[g][j] = ah[g][j] = 0;
#pragma unroll 1
    for (int qq = 0; qq < 4; ++qq) {
      const int cq = (qq + (lane >> 1)) & 3;  // bank-conflict-free chunk order
      uint4 kw[TPL];
#pragma unroll
      for (int j = 0; j < TPL; ++j) kw[j] = *reinterpret_cast<const uint4*>(kt + (lane + 32 * j) * 64 + 16 * cq);
#pragma unroll
      for (int ii = 0; ii < 4; ++ii) {
        uint32_t mk[TPL][2];
#pragma unroll
        for (int j = 0; j < TPL; ++j) masks4(comp(kw[j], ii), mk[j]);
#pragma unroll
        for (int g = 0; g < GP; ++g) {
          const uint2* qrow = reinterpret_cast<const uint2*>(S.qw[g0 + g]) + 12 * cq + ii * 3;
          const uint2 QL = qrow[0], QM = qrow[1], QH = qrow[2];
#pragma unroll
          for (int j = 0; j < TPL; ++j) dot_set(mk[j][0], QL.x, QM.x, QH.x, al[g][j], am[g][j], ah[g][j], true);
#pragma unroll
          for (int j = 0; j < TPL; ++j) dot_set(mk[j][1], QL.y, QM.y, QH.y, al[g][j], am[g][j], ah[g][j], true);
        }
      }
    }
  }

  // ---- K half of a quantized unit: logits, online softmax, P limbs (A6, A8, A9 set-up) ---------
  __device__ void quantized_k(const uint8_t* kt, long long head, int local, uint32_t pairs) {
    if constexpr (FG) {
#pragma unroll  // the per-query state stays in registers
      for (int gq = 0; gq < G; ++gq) {
        if constexpr (BITS == 2)
          fg_k(gq, kt, head, local);
        else
          fg4_k(gq, kt, head, local);
      }
      return;
    }
    const long long key = head * a.blocks_per_head + (local >> a.lg_units_per_blk);
    if (key != qkey) {
      build_q(pairs);
      qkey = key;
    }
    if constexpr (kMma1) {
      float lg[4];
      k_mma(kt, lg);
      softmax_mma(pairs, lg);
    } else if constexpr (kMmaG) {
      float lg[NBLK][8];
      k_mma_g(kt, lg);
      softmax_mma_g(pairs, lg);
    } else {
#pragma unroll
      for (int g0 = 0; g0 < G; g0 += GP) {
        int al[GP][TPL], am[GP][TPL], ah[GP][TPL];
        k_dot(kt, g0, al, am, ah);
        softmax4(pairs, g0, al, am, ah);
      }
    }
  }

  // 4 bits: lane holds tokens lane + 32 j; each byte of a P limb word is stored on its own.
  __device__ void softmax4(uint32_t pairs, int g0, const int (&al)[GP][TPL], const int (&am)[GP][TPL],
                           const int (&ah)[GP][TPL]) {
#pragma unroll
    for (int gg = 0; gg < GP; ++gg) {
      const int g = g0 + gg;
      float lg[TPL], mu = -INFINITY;
#pragma unroll
      for (int j = 0; j < TPL; ++j) {
        lg[j] = fmaf(combine_limbs(ah[gg][j], am[gg][j], al[gg][j]), invq[g], cblk[g]);
        mu = fmaxf(mu, lg[j]);
      }
      mu = warp_max(mu);
      const float m_new = fmaxf(m[g], mu);
      const float alpha = fast_exp2(m[g] - m_new);
      float psum = 0.f, zsum = 0.f, mv = 0.f, pp[TPL];
#pragma unroll
      for (int j = 0; j < TPL; ++j) {
        const int vg = (32 * j) >> a.lg_gv;  // V group of token lane + 32 j within the unit
        const uint32_t vp = __shfl_sync(kFull, pairs, 8 + vg);
        const float p = fast_exp2(lg[j] - m_new);
        psum += p;
        zsum = fmaf(p, h2f(static_cast<uint16_t>(vp >> 16)), zsum);
        pp[j] = p * h2f(static_cast<uint16_t>(vp & 0xFFFFu));
        mv = fmaxf(mv, pp[j]);
      }
      mv = warp_max(mv);
      m[g] = m_new;
      l[g] = fmaf(l[g], alpha, psum);
      Z[g] = fmaf(Z[g], alpha, zsum);
      alpha_[g] = alpha;
      hasv_[g] = mv > 0.f;
      // P <= 2^24 - 124: the top token must not round to 2^24, where it would wrap to 0
      const float scv = mv > 0.f ? kPRange * fast_rcp(mv) : 0.f;
      invv_[g] = mv * (1.0f / kPRange);
      uint8_t* pwb = reinterpret_cast<uint8_t*>(S.pw[g]);
#pragma unroll
      for (int j = 0; j < TPL; ++j) {
        const int t = lane + 32 * j;
        const int row = t >> 3, k = t & 1, mb = (t >> 1) & 3;  // row t/8, set t%2, byte (t%8)/2
        const uint32_t Pq = __float2uint_rn(pp[j] * scv);
        uint8_t* base = pwb + ((row * 3) * 2 + k) * 4 + mb;  // limb b of row r: 8 bytes at (3 r + b) * 8
        base[0] = static_cast<uint8_t>(Pq & 255u);
        base[8] = static_cast<uint8_t>((Pq >> 8) & 255u);
        base[16] = static_cast<uint8_t>((Pq >> 16) & 255u);
      }
    }
  }

  // ---- V half of a quantized unit: P . codes for every query (A9) ------------------------------
  __device__ void quantized_v(const uint8_t* vt) {
    __syncwarp();  // P limbs of every query are in shared memory
    if constexpr (FG) {
#pragma unroll  // the per-query state stays in registers
      for (int gq = 0; gq < G; ++gq) {
        if constexpr (BITS == 2) {
          if (hasv_[gq]) {
            v_mma_fg(gq, vt);
          } else {  // every weight of the unit is zero for this query: only rescale
#pragma unroll
            for (int e = 0; e < 4; ++e) o[gq][e] *= alpha_[gq];
          }
        } else {
          fg4_v(gq, vt);
        }
      }
    } else if (G == 1 && !hasv_[0]) {  // every weight of the unit is zero: only rescale
#pragma unroll
      for (int e = 0; e < 4; ++e) o[0][e] *= alpha_[0];
    } else if constexpr (kMma1) {
      v_mma(vt);
    } else if constexpr (kMmaG) {
      v_mma_g(vt);
    } else {
      dot_v(vt);
    }
    __syncwarp();  // P limbs are rewritten by the next unit
  }

  // CUDA-core P . codes at 4 bits: dp4a on the three limbs of every query's P.
  __device__ void dot_v(const uint8_t* vt) {
#pragma unroll
    for (int g0 = 0; g0 < G; g0 += GP) {  // queries g0 .. g0 + GP - 1 per pass over the codes
      int vl[GP][4], vm[GP][4], vh[GP][4];
#pragma unroll
      for (int g = 0; g < GP; ++g)
#pragma unroll
        for (int e = 0; e < 4; ++e) vl[g][e] = vm[g][e] = vh[g][e] = 0;
#pragma unroll 2
      for (int r = 0; r < ROWS; ++r) {
        const uint4 vw = *reinterpret_cast<const uint4*>(vt + r * 512 + 16 * lane);
        uint32_t mv4[4][2];
#pragma unroll
        for (int e = 0; e < 4; ++e) masks4(comp(vw, e), mv4[e]);
#pragma unroll
        for (int g = 0; g < GP; ++g) {
          if (G > 1 && !hasv_[g0 + g]) continue;
          const uint2* pw2 = reinterpret_cast<const uint2*>(S.pw[g0 + g]);
          const uint2 PL = pw2[r * 3 + 0], PM = pw2[r * 3 + 1], PH = pw2[r * 3 + 2];
#pragma unroll
          for (int e = 0; e < 4; ++e) dot_set(mv4[e][0], PL.x, PM.x, PH.x, vl[g][e], vm[g][e], vh[g][e], false);
#pragma unroll
          for (int e = 0; e < 4; ++e) dot_set(mv4[e][1], PL.y, PM.y, PH.y, vl[g][e], vm[g][e], vh[g][e], false);
        }
      }
#pragma unroll
      for (int gg = 0; gg < GP; ++gg) {
        const int g = g0 + gg;
        if (hasv_[g]) {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            o[g][e] = fmaf(o[g][e], alpha_[g], combine_limbs(vh[gg][e], vm[gg][e], vl[gg][e]) * invv_[g]);
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) o[g][e] *= alpha_[g];
        }
      }
    }
  }

  // Byte offset of fp16 row tt of a residual V half in its buffer (four rows per 1 KB piece).
  static __device__ __forceinline__ int vrow(int tt) { return tt * 256 + (kMma ? (tt >> 2) * (kVPieceStride - kVPiece) : 0); }

  // ---- K half of a residual unit (16 fp16 rows): logits and softmax weights --------------------
  // q is read in fp16 from global memory (L1-resident: every lane pair reads the same 256 bytes).
  // Fused append: if the new token's slot falls in residual unit r (rows 16 r .. 16 r + 15), copy its
  // row from `src` into the unit's shared-memory copy (which the bulk copy filled from the cache)
  // and into the cache itself.  Each residual unit belongs to one warp, so the row is written once.
  __device__ void insert_new_row(uint8_t* buf, int r, long long head, const uint16_t* src, uint16_t* res, bool v_half) {
    const int row = a.new_slot - r * kResTokens;
    if (a.new_slot < 0 || row < 0 || row >= kResTokens) return;
    if (!dbg_check(a.new_slot < a.residual && head < a.bh, a.status)) return;
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(src + static_cast<size_t>(head) * kHeadDim) + lane);
    *reinterpret_cast<uint2*>(buf + (v_half ? vrow(row) : row * 256) + 8 * lane) = v;
    uint16_t* dst = res + (static_cast<size_t>(head) * a.residual + a.new_slot) * kHeadDim;
    reinterpret_cast<uint2*>(dst)[lane] = v;
    __syncwarp();
  }

  // K half of a residual unit under online K: 16 rows of codes, dequantized with block res_blk's
  // (s, z) (section Per-Channel量子化: the block being filled carries the newest block's pair).
  // Two lanes per token, 64 channels each; a code word lies in one K group (G_k >= 32 >= P).
  __device__ void residual_k_coded(const uint8_t* kt, int nvalid, long long head) {
    constexpr int kRowBytes = kHeadDim * BITS / 8, WPL = 64 / P;
    constexpr uint32_t L = (1u << BITS) - 1u;
    const int t = lane >> 1, hf = lane & 1;
    size_t sb = (static_cast<size_t>(head) * a.blocks_per_head + a.res_blk) * ngk;
    if (!dbg_check(a.res_blk < a.blocks_per_head && head < a.bh, a.status)) sb = 0;
    uint32_t w[WPL];
#pragma unroll
    for (int i = 0; i < WPL; i += 4) {
      const uint4 v4 = *reinterpret_cast<const uint4*>(kt + t * kRowBytes + hf * (kRowBytes / 2) + 4 * i);
      w[i] = v4.x;
      w[i + 1] = v4.y;
      w[i + 2] = v4.z;
      w[i + 3] = v4.w;
    }
#pragma unroll  // the per-query state must stay in registers: no runtime index into it
    for (int g = 0; g < G; ++g) {
      const uint4* qp = reinterpret_cast<const uint4*>(S.qraw[qslot(head)][g] + 64 * hf);
      float dot = 0.f;
#pragma unroll
      for (int i = 0; i < WPL; ++i) {
        const int gi = (64 * hf + P * i) >> a.lg_gk;
        const float sk = h2f(__ldg(a.k_scale + sb + gi)), zk = h2f(__ldg(a.k_zero + sb + gi));
        float acc = 0.f, qs = 0.f;
#pragma unroll
        for (int k8 = 0; k8 < P / 8; ++k8) {
          const uint4 qv = qp[(P * i) / 8 + k8];
          const uint32_t qw4[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 qf = __half22float2(*reinterpret_cast<const __half2*>(&qw4[e]));
            const int j = 8 * k8 + 2 * e;
            acc = fmaf(qf.x, static_cast<float>((w[i] >> (BITS * j)) & L), acc);
            acc = fmaf(qf.y, static_cast<float>((w[i] >> (BITS * (j + 1))) & L), acc);
            qs += qf.x + qf.y;
          }
        }
        dot = fmaf(sk, acc, fmaf(zk, qs, dot));
      }
      dot += __shfl_xor_sync(kFull, dot, 1);
      dot *= a.qscale;
      const bool valid = t < nvalid;
      const float lg = valid ? dot : -INFINITY;
      const float m_new = fmaxf(m[g], warp_max(lg));
      const float alpha = fast_exp2(m[g] - m_new);
      const float p = valid ? fast_exp2(lg - m_new) : 0.f;
      m[g] = m_new;
      l[g] = fmaf(l[g], alpha, hf == 0 ? p : 0.f);
      Z[g] *= alpha;
      alpha_[g] = alpha;
      pres_[g] = p;
    }
  }

  __device__ void residual_k(uint8_t* kt, int nvalid, long long head, int r) {
    if constexpr (KC) {
      residual_k_coded(kt, nvalid, head);
      return;
    }
    insert_new_row(kt, r, head, a.k_new, a.k_res, false);
    const int t = lane >> 1, hf = lane & 1;  // 2 lanes per token, 64 channels each
    float dot[G];
#pragma unroll
    for (int g = 0; g < G; ++g) dot[g] = 0.f;
    if constexpr (G > 1) {
      // several queries: each K chunk is read and converted once for all of them; q (scaled) comes
      // from shared memory (start_head)
#pragma unroll 2
      for (int k = 0; k < 8; ++k) {
        const int cc = (k + lane) & 7;  // bank-conflict-free chunk order
        const int c0 = 64 * hf + 8 * cc;
        const uint4 kv = *reinterpret_cast<const uint4*>(kt + t * 256 + 2 * c0);
        const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w};
        float kf[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&kw[e]));
          kf[2 * e] = f.x;
          kf[2 * e + 1] = f.y;
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float4 qa = *reinterpret_cast<const float4*>(&S.qs[G > 1 ? g : 0][G > 1 ? c0 : 0]);
          const float4 qb = *reinterpret_cast<const float4*>(&S.qs[G > 1 ? g : 0][G > 1 ? c0 + 4 : 0]);
          const float qf[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
#pragma unroll
          for (int e = 0; e < 8; ++e) dot[g] = fmaf(qf[e], kf[e], dot[g]);
        }
      }
    } else {
      const uint4* qp = reinterpret_cast<const uint4*>(S.qraw[qslot(head)][0]);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int cc = (k + lane) & 7;  // bank-conflict-free chunk order
        const int c0 = 64 * hf + 8 * cc;
        const uint4 kv = *reinterpret_cast<const uint4*>(kt + t * 256 + 2 * c0);
        const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w};
        const uint4 qv = qp[c0 >> 3];
        const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 kf = __half22float2(*reinterpret_cast<const __half2*>(&kw[e]));
          const float2 qf = __half22float2(*reinterpret_cast<const __half2*>(&qw[e]));
          dot[0] = fmaf(qf.x, kf.x, dot[0]);
          dot[0] = fmaf(qf.y, kf.y, dot[0]);
        }
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float d = dot[g] + __shfl_xor_sync(kFull, dot[g], 1);
      if (G == 1) d *= a.qscale;  // several queries: q in shared memory is scaled already
      const bool valid = t < nvalid;
      const float lg = valid ? d : -INFINITY;
      const float m_new = fmaxf(m[g], warp_max(lg));
      const float alpha = fast_exp2(m[g] - m_new);
      const float p = valid ? fast_exp2(lg - m_new) : 0.f;
      m[g] = m_new;
      l[g] = fmaf(l[g], alpha, hf == 0 ? p : 0.f);
      Z[g] *= alpha;
      alpha_[g] = alpha;
      pres_[g] = p;
    }
  }

  // ---- V half of a residual unit: p . rows -----------------------------------------------------
  __device__ void residual_v(uint8_t* vt, int nvalid, long long head, int r) {
    insert_new_row(vt, r, head, a.v_new, a.v_res, true);
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[g][e] *= alpha_[g];
    for (int tt = 0; tt < nvalid; ++tt) {  // each row is read and converted once for every query
      const uint2 vv = *reinterpret_cast<const uint2*>(vt + vrow(tt) + 8 * lane);
      const float2 v0 = __half22float2(*reinterpret_cast<const __half2*>(&vv.x));
      const float2 v1 = __half22float2(*reinterpret_cast<const __half2*>(&vv.y));
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float pt = __shfl_sync(kFull, pres_[g], 2 * tt);
        o[g][0] = fmaf(pt, v0.x, o[g][0]);
        o[g][1] = fmaf(pt, v0.y, o[g][1]);
        o[g][2] = fmaf(pt, v1.x, o[g][2]);
        o[g][3] = fmaf(pt, v1.y, o[g][3]);
      }
    }
  }

  // ---- end of a head segment: the output, or a partial ----------------------------------------
  // A segment that covers its head whole writes the output.  Otherwise the segment's partial
  // (m, l, Z, o) goes with plain stores to this worker's slot 0 (the first segment of its range)
  // or slot 1 (the last one); the tickets that choose the worker that merges the head are taken at
  // the end of the range (publish), after one fence that covers both partials, so that no fence or
  // atomic round trip stalls the warp in the middle of its range.
  __device__ void finish_segment(long long head, long long seg_a, long long seg_b) {
    residual_layout();
    const long long h0 = head * a.units, h1 = h0 + a.units;
    float lsum[G], zsum[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      lsum[g] = warp_sum(l[g]);
      zsum[g] = warp_sum(Z[g]);
    }
    if (seg_a == h0 && seg_b == h1) {
#pragma unroll
      for (int g = 0; g < G; ++g) store_out(head, g, o[g], zsum[g], 1.f / lsum[g]);
      return;
    }
    const int slot = seg_a == ub ? 0 : 1;
    if (!dbg_check(worker < a.workers && head < a.bh, a.status)) return;
    float* mine = a.partials + ((worker * 2 + slot) * G) * kPartialStride;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float* p = mine + g * kPartialStride;
      if (lane == 0) {
        p[0] = m[g];
        p[1] = lsum[g];
        p[2] = zsum[g];
      }
      *reinterpret_cast<float4*>(p + 4 + 4 * lane) = make_float4(o[g][0], o[g][1], o[g][2], o[g][3]);
    }
    // only the first and the last segment of a range can be partial
    if (npend_ == 0)
      pend0_ = static_cast<int>(head);
    else
      pend1_ = static_cast<int>(head);
    ++npend_;
  }

  // Workers that hold a part of a head (a contiguous run of them: ranges are contiguous in units).
  __device__ __forceinline__ void head_workers(long long head, long long& wfirst, long long& wlast) const {
    const long long h0 = head * a.units, W = a.workers, U = a.total_units;
    wfirst = worker_of(h0, U, W);
    wlast = worker_of(h0 + a.units - 1, U, W);
  }

  // End of the range: one fence publishes this worker's partials, then one ticket per partial head
  // (both atomics in flight together); the last of a head's workers to arrive merges the head.
  __device__ void publish() {
    if (npend_ == 0) return;
    __threadfence();  // every lane publishes its own slices of the partials before the tickets
    __syncwarp();
    int last = 0;
    if (lane == 0) {
      const int t0 = atomicAdd(a.tickets + pend0_, 1);
      const int t1 = npend_ > 1 ? atomicAdd(a.tickets + pend1_, 1) : -1;
      long long wf, wl;
      head_workers(pend0_, wf, wl);
      if (t0 == static_cast<int>(wl - wf)) last |= 1;
      if (npend_ > 1) {
        head_workers(pend1_, wf, wl);
        if (t1 == static_cast<int>(wl - wf)) last |= 2;
      }
      if (last) __threadfence();  // acquire side: the partials published before the other tickets
    }
    last = __shfl_sync(kFull, last, 0);
    if (!last) return;
    __threadfence();
#pragma unroll 1
    for (int i = 0; i < 2; ++i)
      if ((last >> i) & 1) merge(i ? pend1_ : pend0_);
  }

  // Merge of a head's partials: workers wfirst..wlast each left one.  Only wfirst can have started
  // before the head (its partial is then in its slot 1); every later one starts inside it (slot 0).
  // Lane k reads (m, l, Z) of part k; the o rows follow CH parts at a time, the loads of every query
  // in flight together.
  __device__ void merge(long long head) {
    long long wfirst, wlast;
    head_workers(head, wfirst, wlast);
    const long long W = a.workers, U = a.total_units;
    const int nparts = static_cast<int>(wlast - wfirst + 1);
    const int first_slot = (U * wfirst / W) >= head * a.units ? 0 : 1;
    if (!dbg_check(wfirst >= 0 && wlast < W, a.status)) return;
    auto part = [&](int k, int g) -> const float* {
      const long long x = wfirst + k;
      return a.partials + ((x * 2 + (k == 0 ? first_slot : 0)) * G + g) * kPartialStride;
    };
    constexpr int CH = 8 / G > 0 ? 8 / G : 1;  // o rows of CH parts per query in flight
    float mm[G], ls[G], zs[G], acc[G][4];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      mm[g] = -INFINITY;
      ls[g] = 0.f;
      zs[g] = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[g][e] = 0.f;
    }
    if (nparts > 32) {  // the largest m first; up to 32 parts take it from the pass below
      for (int k = lane; k < nparts; k += 32)
#pragma unroll
        for (int g = 0; g < G; ++g) mm[g] = fmaxf(mm[g], __ldcg(part(k, g)));
#pragma unroll
      for (int g = 0; g < G; ++g) mm[g] = warp_max(mm[g]);
    }
    for (int base = 0; base < nparts; base += 32) {
      const int k = base + lane;
      float mk[G], lk[G], zk[G], wk[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        mk[g] = -INFINITY;
        lk[g] = 0.f;
        zk[g] = 0.f;
        if (k < nparts) {
          const float* p = part(k, g);
          mk[g] = __ldcg(p);
          lk[g] = __ldcg(p + 1);
          zk[g] = __ldcg(p + 2);
        }
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        if (k < nparts && !(lk[g] > 0.f)) report_status(a.status, KIVI_ERR_INTERNAL);  // never written
        if (nparts <= 32) mm[g] = warp_max(mk[g]);
        wk[g] = k < nparts ? fast_exp2(mk[g] - mm[g]) : 0.f;
        ls[g] = fmaf(wk[g], lk[g], ls[g]);
        zs[g] = fmaf(wk[g], zk[g], zs[g]);
      }
      const int n = min(32, nparts - base);
      for (int i = 0; i < n; i += CH) {
        float4 ov[CH][G];
#pragma unroll
        for (int u = 0; u < CH; ++u)
#pragma unroll
          for (int g = 0; g < G; ++g)
            ov[u][g] = i + u < n ? __ldcg(reinterpret_cast<const float4*>(part(base + i + u, g) + 4) + lane)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int u = 0; u < CH; ++u)
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float w = __shfl_sync(kFull, wk[g], (i + u) & 31);
            acc[g][0] = fmaf(w, ov[u][g].x, acc[g][0]);
            acc[g][1] = fmaf(w, ov[u][g].y, acc[g][1]);
            acc[g][2] = fmaf(w, ov[u][g].z, acc[g][2]);
            acc[g][3] = fmaf(w, ov[u][g].w, acc[g][3]);
          }
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) store_out(head, g, acc[g], warp_sum(zs[g]), 1.f / warp_sum(ls[g]));
    if (lane == 0) a.tickets[head] = 0;
  }

  __device__ void store_out(long long head, int g, const float* acc, float z, float inv_l) const {
    __half2 h01 = __floats2half2_rn((acc[0] + z) * inv_l, (acc[1] + z) * inv_l);
    __half2 h23 = __floats2half2_rn((acc[2] + z) * inv_l, (acc[3] + z) * inv_l);
    uint2 v;
    v.x = *reinterpret_cast<uint32_t*>(&h01);
    v.y = *reinterpret_cast<uint32_t*>(&h23);
    *reinterpret_cast<uint2*>(a.out + (static_cast<size_t>(head) * G + g) * kHeadDim + 4 * lane) = v;
  }

  // all lanes wait; the decision is made warp-uniform
  __device__ bool wait_half(int h) {
    const bool ok = mbar_wait_bounded(&S.bar[h % kBuffers], (h / kBuffers) & 1, a.timeout_ns);
    return __all_sync(kFull, ok);
  }

  // After a timeout: wait, each for at most the same limit, until the halves in flight have landed,
  // so that the warp does not exit with bulk copies still writing its shared memory.  A copy that
  // truly never lands outlives the wait; the warp's buffers are then undefined, and so is the
  // output (the status word holds KIVI_ERR_DEVICE_TIMEOUT).
  __device__ void drain_from(int h, int nhalves) {
    for (int x = h; x < h + kBuffers && x < nhalves; ++x)
      (void)mbar_wait_bounded(&S.bar[x % kBuffers], (x / kBuffers) & 1, a.timeout_ns);
    __syncwarp();
  }

  __device__ __forceinline__ void advance(long long& h, int& l) const {
    if (++l == a.units) {
      l = 0;
      ++h;
    }
  }

  __device__ void run() {
    if (lane == 0) {
#pragma unroll
      for (int b = 0; b < kBuffers; ++b) mbar_init(&S.bar[b], 1);
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if constexpr (kMma) {  // FG: slot 3 of every limb row stays zero; the other paths write every word
      for (int i = lane; i < static_cast<int>(sizeof(S.qw) / 4); i += 32) reinterpret_cast<uint32_t*>(S.qw)[i] = 0u;
      for (int i = lane; i < static_cast<int>(sizeof(S.pw) / 4); i += 32) reinterpret_cast<uint32_t*>(S.pw)[i] = 0u;
      if (lane == 0) S.zero4 = make_uint4(0u, 0u, 0u, 0u);
    }
    __syncwarp();
    const int nhalves = static_cast<int>(2 * (ue - ub));
    // (head, local unit) cursors for the current unit and the next two; advanced by increments
    long long head = ub / a.units;
    int local = static_cast<int>(ub - head * a.units);
    long long h1 = head, h2;
    int l1 = local, l2;
    advance(h1, l1);
    h2 = h1;
    l2 = l1;
    advance(h2, l2);
    if (lane == 0) {  // halves 0, 1, 2 = K0, V0, K1
      issue_half(0, head, local);
      issue_half(1, head, local);
      if (kBuffers == 3 && nhalves > 2) issue_half(2, h1, l1);
    }
    uint32_t pairs = load_pairs(head, local);
    long long cur_head = -1, seg_a = ub;
    int hk = 0;
    for (long long u = ub; u < ue; ++u, hk += 2) {
      const bool new_head = head != cur_head;
      if (new_head) {
        if (cur_head >= 0) finish_segment(cur_head, seg_a, u);
        cur_head = head;
        seg_a = u;
      }
      const uint32_t pairs_next = (u + 1 < ue) ? load_pairs(h1, l1) : 0u;
      const bool quant = local < a.units_q;
      const int nvalid = quant ? 0 : min(kResTokens, a.n_res - (local - a.units_q) * kResTokens);
      // K half
      if (!wait_half(hk)) {
        if (lane == 0) report_status(a.status, KIVI_ERR_DEVICE_TIMEOUT);
        drain_from(hk, nhalves);
        return;
      }
      if (new_head) start_head(head);  // the head's queries landed with this K half
      if (quant) {
        quantized_k(S.buf[hk % kBuffers], head, local, pairs);
      } else {
        residual_layout();
        residual_k(S.buf[hk % kBuffers], nvalid, head, local - a.units_q);
      }
      __syncwarp();
      // The bulk copy issued next overwrites the buffer just read.  The reads are complete (their
      // values were consumed before the __syncwarp); a residual unit also wrote the new token's row
      // into it, and that generic-proxy write is ordered before the async-proxy copy by a fence.
      if (!quant) fence_proxy_async_smem();
      // half hk + kBuffers reuses the buffer just consumed: the next unit's V (ring of 3) or K (2)
      if (lane == 0 && hk + kBuffers < nhalves) issue_half(hk + kBuffers, h1, l1);
      // V half
      if (!wait_half(hk + 1)) {
        if (lane == 0) report_status(a.status, KIVI_ERR_DEVICE_TIMEOUT);
        drain_from(hk + 1, nhalves);
        return;
      }
      if (quant)
        quantized_v(S.buf[(hk + 1) % kBuffers]);
      else
        residual_v(S.buf[(hk + 1) % kBuffers], nvalid, head, local - a.units_q);
      __syncwarp();
      if (!quant) fence_proxy_async_smem();
      // the unit after next's K half (ring of 3) or the next unit's V half (2)
      if (lane == 0 && hk + 1 + kBuffers < nhalves) {
        if (kBuffers == 3)
          issue_half(hk + 4, h2, l2);
        else
          issue_half(hk + 3, h1, l1);
      }
      pairs = pairs_next;
      head = h1;
      local = l1;
      h1 = h2;
      l1 = l2;
      advance(h2, l2);
    }
    finish_segment(cur_head, seg_a, ue);
    publish();
    if constexpr (FL) {  // the ring buffers are free: every copy the warp issued has landed and been read
      static_assert(sizeof(S.buf) >= 32 * Flusher<BITS>::kStage * sizeof(uint4), "a flush stage is 8 KB");
      Flusher<BITS>{a, reinterpret_cast<uint4*>(S.buf), lane}.run(worker);
    }
  }
};

// FL: the step whose appended token fills the residual also flushes it (its own instantiation: the
// flush's registers stay out of the allocation of the plain decode).
template <int BITS, int G, bool KC, bool FG = false, bool FL = false>
__global__ void __launch_bounds__(warps_per_cta<G, FG>() * 32, 1) decode_kernel(const __grid_constant__ DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  WarpSmem<G, FG>& S = reinterpret_cast<WarpSmem<G, FG>*>(smem_raw)[warp];
  const long long W = a.workers, U = a.total_units;
  const long long worker = static_cast<long long>(blockIdx.x) * warps_per_cta<G, FG>() + warp;
  if (worker >= W) return;  // the last CTA may hold fewer workers
  const long long ub = U * worker / W, ue = U * (worker + 1) / W;  // non-empty because W <= U
  static_assert(!FL || (!KC && !FG), "the in-launch flush is for the base groups with fp16 residual keys");
  Decoder<BITS, G, KC, FG, FL> d(a, S, lane, worker, ub, ue);
  d.run();
}

template <int BITS, int G, bool FG>
cudaError_t plan_for_kernels(DecodePlan* plan) {
  constexpr int kWarps = warps_per_cta<G, FG>();
  static_assert(kWarps * sizeof(WarpSmem<G, FG>) <= 232448, "a CTA's warps exceed 227 KB of shared memory");
  const int smem = kWarps * static_cast<int>(sizeof(WarpSmem<G, FG>));
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<BITS, G, false, FG>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  if constexpr (!FG) {
    e = cudaFuncSetAttribute(decode_kernel<BITS, G, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(decode_kernel<BITS, G, false, false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem);
    if (e != cudaSuccess) return e;
  }
  int dev = 0, sms = 0, occ = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, decode_kernel<BITS, G, false, FG>, kWarps * 32, smem)) !=
      cudaSuccess)
    return e;
  if (occ < 1) return cudaErrorInvalidConfiguration;
  plan->warps_per_cta = kWarps;
  plan->ctas = sms * occ;
  plan->smem_bytes = smem;
  plan->unit_tokens = Decoder<BITS, G, false, FG>::UT;
  plan->res_unit_tokens = kResTokens;
  return cudaSuccess;
}

template <int BITS, int G>
cudaError_t plan_for(DecodePlan* plan, int fine) {
  if (fine) return plan_for_kernels<BITS, G, true>(plan);
  return plan_for_kernels<BITS, G, false>(plan);
}

template <int BITS, int G>
cudaError_t launch_for(const DecodeArgs& a, const DecodePlan& plan, cudaStream_t stream) {
  if (a.workers < 1 || a.workers > plan.workers() || a.total_units < a.workers) return cudaErrorInvalidValue;
  if (a.flush_blk >= 0 && (a.fine || a.k_res_coded)) return cudaErrorInvalidValue;
  const int ctas = (a.workers + plan.warps_per_cta - 1) / plan.warps_per_cta;
  if (a.fine) {
    decode_kernel<BITS, G, false, true><<<ctas, plan.warps_per_cta * 32, plan.smem_bytes, stream>>>(a);
  } else if (a.k_res_coded) {
    decode_kernel<BITS, G, true><<<ctas, plan.warps_per_cta * 32, plan.smem_bytes, stream>>>(a);
  } else if (a.flush_blk >= 0) {
    decode_kernel<BITS, G, false, false, true><<<ctas, plan.warps_per_cta * 32, plan.smem_bytes, stream>>>(a);
  } else {
    decode_kernel<BITS, G, false><<<ctas, plan.warps_per_cta * 32, plan.smem_bytes, stream>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace

#define KIVI_DISPATCH(BITS_, GQA_, FN, ...)                              \
  do {                                                                   \
    if ((BITS_) == 2) {                                                  \
      switch (GQA_) {                                                    \
        case 1: return FN<2, 1>(__VA_ARGS__);                            \
        case 2: return FN<2, 2>(__VA_ARGS__);                            \
        case 4: return FN<2, 4>(__VA_ARGS__);                            \
        case 8: return FN<2, 8>(__VA_ARGS__);                            \
      }                                                                  \
    } else if ((BITS_) == 4) {                                           \
      switch (GQA_) {                                                    \
        case 1: return FN<4, 1>(__VA_ARGS__);                            \
        case 2: return FN<4, 2>(__VA_ARGS__);                            \
        case 4: return FN<4, 4>(__VA_ARGS__);                            \
        case 8: return FN<4, 8>(__VA_ARGS__);                            \
      }                                                                  \
    }                                                                    \
    return cudaErrorInvalidValue;                                        \
  } while (0)

cudaError_t debug_status_decode(int32_t* out) { return take_debug_status_tu(out); }

cudaError_t decode_plan(int bits, int gqa, int fine, DecodePlan* plan) {
  KIVI_DISPATCH(bits, gqa, plan_for, plan, fine);
}

cudaError_t launch_decode(const DecodeArgs& a, int bits, const DecodePlan& plan, cudaStream_t stream) {
  KIVI_DISPATCH(bits, a.gqa, launch_for, a, plan, stream);
}

}  // namespace kivi
