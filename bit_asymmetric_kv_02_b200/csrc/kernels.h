// Launch arguments of the library's kernels (host <-> device, plain data).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace kivi {

// Quantize `nblocks` R-token blocks of K and V per (batch, KV head) and optionally copy a tail
// into the residual.  Source tensors are fp16 [bh][src_tokens][128]; block j reads tokens
// src_tok0 + j*R .. and is written as quantized block dst_blk0 + j.
struct QuantizeArgs {
  const uint16_t* k_src;
  const uint16_t* v_src;
  uint32_t* k_codes;
  uint32_t* v_codes;
  uint16_t *k_scale, *k_zero, *v_scale, *v_zero;
  uint16_t *k_res, *v_res;
  int bh;          // batch * kv_heads
  int src_tokens;  // tokens per head in the source tensors
  int src_tok0;    // first source token of block 0
  int nblocks;     // blocks to quantize per head
  int dst_blk0;    // destination block index of block 0
  int res_tok0;    // first source token copied into residual slot 0
  int res_tokens;  // tokens copied into the residual (0: none)
  int residual, capacity, group_k, group_v;
  int lg_gk, lg_gv;  // log2(group_k), log2(group_v): set by launch_quantize_blocks
  int k_given;       // 1: the K (s, z) of each block are already in k_scale / k_zero (prefix groups)
  int v_only;        // 1: quantize the V blocks only (online K: the K codes are in place)
  int fine;          // 1: fine-grained groups: K (s, z) per channel per group_k tokens
                     //    ([bh][C/group_k][128]), V (s, z) per token per group_v channels ([bh][C][128/group_v])
};

// Online K: codes `rows` K rows per head (fp16 source rows src_tok0 .. of a [bh][src_tokens][128]
// tensor) with the (s, z) of block blk_src into code rows dst_row0 .. of k_codes; copy_scales
// also copies block blk_src's (s, z) into block blk_src + 1.  v_new != nullptr: also writes the
// V row of each head into residual slot v_slot (an append).
struct OnlineKArgs {
  const uint16_t* k_src;
  int src_tokens, src_tok0, rows;
  uint32_t* k_codes;
  uint16_t *k_scale, *k_zero;
  const uint16_t* v_new;
  uint16_t* v_res;
  int bh, capacity, residual, group_k;
  int blk_src, dst_row0, copy_scales, v_slot;
};

struct AppendArgs {
  const uint16_t* k_new;
  const uint16_t* v_new;
  uint16_t *k_res, *v_res;
  int bh, residual, slot;
};

struct DecodeArgs {
  const uint32_t* k_codes;
  const uint32_t* v_codes;
  const uint16_t *k_scale, *k_zero, *v_scale, *v_zero;
  uint16_t *k_res, *v_res;  // written only by a fused append
  const uint16_t* q;
  uint16_t* out;
  float* partials;    // [workers][2][gqa][kPartialStride]
  int32_t* tickets;   // [bh], zero between calls
  int32_t* status;    // optional device status word
  int bh, gqa, capacity, residual, group_k, group_v;
  int n_quant, n_res;
  int units_q;        // quantized units per head
  int units;          // units per head (quantized + residual)
  long long total_units;
  int blocks_per_head;   // capacity / residual (K scale rows per head)
  int vgroups_per_head;  // capacity / group_v (V scales per head)
  int lg_gk, lg_gv;      // log2(group_k), log2(group_v)
  int lg_units_per_blk;  // log2(residual / tokens per quantized unit)
  int workers;
  float qscale;       // softmax scale * log2(e)
  unsigned long long timeout_ns;
  uint32_t debug_extra_tx;  // test hook: bytes a barrier expects beyond the copy (0 normally)
  // fused append: the token in k_new / v_new ([bh][128] fp16) is residual slot new_slot (< n_res);
  // new_slot < 0: no append
  const uint16_t* k_new;
  const uint16_t* v_new;
  int new_slot;
  // online K: the residual tokens' K rows are code rows n_quant .. of k_codes with the (s, z) of
  // block res_blk (= n_quant / residual); 0: fp16 rows of k_res
  int k_res_coded, res_blk;
  // fine-grained groups (2 or 4 bits, 1-8 queries per KV head): k_scale / k_zero [bh][C >> lg_gk][128]
  // (lg_gk: tokens per K group), v_scale / v_zero [bh][C][128 >> lg_gv] (lg_gv: channels per V group)
  int fine;
  // in-launch flush (decode step whose appended token fills the residual, base groups only): the R
  // residual tokens become quantized block flush_blk (< 0: no flush), written through these
  // pointers to the arrays above.  No unit of the launch reads that block.
  int flush_blk;
  uint32_t *fk_codes, *fv_codes;
  uint16_t *fk_scale, *fk_zero, *fv_scale, *fv_zero;
};

constexpr int kPartialStride = 132;  // m, l, Z, pad, o[128]

cudaError_t launch_quantize_blocks(const QuantizeArgs& a, int bits, cudaStream_t stream);
// K (s, z) of every channel group over all a.nblocks * R source tokens, stored in every
// destination block's slot (the prefix-group prefill); then launch_quantize_blocks with k_given.
cudaError_t launch_k_prefix_extremes(const QuantizeArgs& a, int bits, cudaStream_t stream);
cudaError_t launch_append(const AppendArgs& a, cudaStream_t stream);
cudaError_t launch_code_k_online(const OnlineKArgs& a, int bits, cudaStream_t stream);

// Decode launch plan: warps per CTA, CTAs, dynamic shared memory.
struct DecodePlan {
  int warps_per_cta;
  int ctas;
  int smem_bytes;
  int unit_tokens;      // tokens per quantized unit
  int res_unit_tokens;  // tokens per residual unit
  int workers() const { return warps_per_cta * ctas; }
};
cudaError_t decode_plan(int bits, int gqa, int fine, DecodePlan* plan);
cudaError_t launch_decode(const DecodeArgs& a, int bits, const DecodePlan& plan, cudaStream_t stream);

// Debug build: read and clear the device-side check word of the quantize and the decode kernels
// (always 0 in a release build).
cudaError_t debug_status_quantize(int32_t* out);
cudaError_t debug_status_decode(int32_t* out);

}  // namespace kivi
