// C ABI of the library (include/kivi.h): argument checks, cache counters, launch plans.
// Host code only; every computation runs in the kernels of quantize.cu and decode.cu.
#include <cstdint>
#include <cstdlib>
#include <mutex>

#include <cuda_runtime.h>

#include "kernels.h"
#include "kivi.h"

namespace {

using kivi::DecodeArgs;
using kivi::DecodePlan;

constexpr int kHeadDim = 128;
constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;  // 2 s per bounded device wait

struct DebugState {
  std::mutex mu;
  int mode = 0;
  unsigned long long timeout_ns = kDefaultTimeoutNs;
  long long max_workers = 0;  // 0: no cap
  int units_q_skew = 0;       // debug build: decode sees this many quantized units more than n_quant holds
};
DebugState& debug_state() {
  static DebugState s;
  return s;
}

bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }
int log2i(int x) {
  int r = 0;
  while ((1 << r) < x) ++r;
  return r;
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

int check_cfg(const kivi_config* c) {
  if (c == nullptr) return KIVI_ERR_INVALID_ARG;
  if (c->head_dim != kHeadDim) return KIVI_ERR_UNSUPPORTED;
  if (c->bits != 2 && c->bits != 4) return KIVI_ERR_UNSUPPORTED;
  if (c->batch < 1 || c->num_kv_heads < 1 || c->capacity < 0) return KIVI_ERR_INVALID_ARG;
  if (c->residual < 128 || c->residual > 1024 || !pow2(c->residual)) return KIVI_ERR_INVALID_ARG;
  if (c->capacity % c->residual != 0) return KIVI_ERR_INVALID_ARG;
  if (c->group_k != 32 && c->group_k != 64 && c->group_k != 128) return KIVI_ERR_INVALID_ARG;
  if (c->fine_groups != 0 && c->fine_groups != 1) return KIVI_ERR_INVALID_ARG;
  if (c->fine_groups) {  // group_k: tokens (<= R), group_v: channels
    if (c->group_k > c->residual) return KIVI_ERR_INVALID_ARG;
    if (c->group_v != 32 && c->group_v != 64 && c->group_v != 128) return KIVI_ERR_INVALID_ARG;
  } else if (c->group_v < 32 || !pow2(c->group_v) || c->group_v > c->residual) {
    return KIVI_ERR_INVALID_ARG;
  }
  if (c->online_k != 0 && c->online_k != 1) return KIVI_ERR_INVALID_ARG;
  if (c->online_k && c->fine_groups) return KIVI_ERR_UNSUPPORTED;
  if (static_cast<long long>(c->batch) * c->num_kv_heads > (1ll << 30)) return KIVI_ERR_UNSUPPORTED;
  if (c->capacity / c->residual > 32767) return KIVI_ERR_UNSUPPORTED;  // grid.y limit of a prefill
  return KIVI_OK;
}

int check_state(const kivi_config* c, const kivi_cache* k) {
  if (k == nullptr) return KIVI_ERR_INVALID_ARG;
  if (k->n_quant < 0 || k->n_quant % c->residual != 0 || k->n_quant > c->capacity) return KIVI_ERR_STATE;
  if (k->n_res < 0 || k->n_res > c->residual) return KIVI_ERR_STATE;
  return KIVI_OK;
}

bool cache_ptrs_ok(const kivi_cache* k, bool need_codes) {
  if (!aligned16(k->k_res) || !aligned16(k->v_res)) return false;
  if (!need_codes) return true;
  return aligned16(k->k_codes) && aligned16(k->v_codes) && aligned16(k->k_scale) && aligned16(k->k_zero) &&
         aligned16(k->v_scale) && aligned16(k->v_zero);
}

// Decode plans are cached per (device, bits, gqa).
struct PlanCache {
  std::mutex mu;
  struct Entry {
    int dev, bits, gqa, fine;
    DecodePlan plan;
  };
  Entry entries[64];
  int n = 0;
};
PlanCache& plan_cache() {
  static PlanCache c;
  return c;
}

cudaError_t get_plan(int bits, int gqa, int fine, DecodePlan* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  PlanCache& pc = plan_cache();
  std::lock_guard<std::mutex> lock(pc.mu);
  for (int i = 0; i < pc.n; ++i) {
    if (pc.entries[i].dev == dev && pc.entries[i].bits == bits && pc.entries[i].gqa == gqa &&
        pc.entries[i].fine == fine) {
      *out = pc.entries[i].plan;
      return cudaSuccess;
    }
  }
  DecodePlan p{};
  if ((e = kivi::decode_plan(bits, gqa, fine, &p)) != cudaSuccess) return e;
  if (pc.n < 64) pc.entries[pc.n++] = {dev, bits, gqa, fine, p};
  *out = p;
  return cudaSuccess;
}

bool gqa_supported(int g) { return g == 1 || g == 2 || g == 4 || g == 8; }

// Online K: the residual tokens' K rows are codes (a quantized block exists).
bool k_online(const kivi_config* c, int n_quant) { return c->online_k == 1 && n_quant > 0; }

// Online K coding of `rows` K rows per head from `src` (fp16 [bh][src_tokens][128], rows
// src_tok0 ..) into code rows n_quant + slot0 .. with block n_quant/R - 1's (s, z); slot0 == 0
// also copies that (s, z) into block n_quant/R.  v_new: the V row of an append (or nullptr).
int code_k_online(const kivi_config* cfg, const kivi_cache* cache, const uint16_t* src, int src_tokens, int src_tok0,
                  int rows, int slot0, const uint16_t* v_new, cudaStream_t stream) {
  kivi::OnlineKArgs o{};
  o.k_src = src;
  o.src_tokens = src_tokens;
  o.src_tok0 = src_tok0;
  o.rows = rows;
  o.k_codes = cache->k_codes;
  o.k_scale = cache->k_scale;
  o.k_zero = cache->k_zero;
  o.v_new = v_new;
  o.v_res = cache->v_res;
  o.bh = cfg->batch * cfg->num_kv_heads;
  o.capacity = cfg->capacity;
  o.residual = cfg->residual;
  o.group_k = cfg->group_k;
  o.blk_src = cache->n_quant / cfg->residual - 1;
  o.dst_row0 = cache->n_quant + slot0;
  o.copy_scales = slot0 == 0 ? 1 : 0;
  o.v_slot = slot0;
  return kivi::launch_code_k_online(o, cfg->bits, stream) == cudaSuccess ? KIVI_OK : KIVI_ERR_CUDA;
}

}  // namespace

extern "C" {

int kivi_abi_version(void) { return KIVI_ABI_VERSION; }

const char* kivi_strerror(int s) {
  switch (s) {
    case KIVI_OK: return "ok";
    case KIVI_ERR_INVALID_ARG: return "invalid argument";
    case KIVI_ERR_UNSUPPORTED: return "unsupported configuration";
    case KIVI_ERR_CAPACITY: return "cache capacity exceeded";
    case KIVI_ERR_RESIDUAL_FULL: return "residual buffer full: flush first";
    case KIVI_ERR_RESIDUAL_NOT_FULL: return "residual buffer not full";
    case KIVI_ERR_EMPTY: return "attention over an empty cache";
    case KIVI_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case KIVI_ERR_CUDA: return "CUDA runtime error";
    case KIVI_ERR_DEVICE_TIMEOUT: return "bounded device wait expired";
    case KIVI_ERR_STATE: return "cache counters inconsistent";
    case KIVI_ERR_INTERNAL: return "internal consistency check failed on the device";
    default: return "unknown status";
  }
}

int kivi_check_config(const kivi_config* cfg) { return check_cfg(cfg); }

int kivi_cache_sizes(const kivi_config* cfg, size_t* out) {
  const int st = check_cfg(cfg);
  if (st != KIVI_OK) return st;
  if (out == nullptr) return KIVI_ERR_INVALID_ARG;
  const size_t bh = static_cast<size_t>(cfg->batch) * cfg->num_kv_heads;
  const size_t C = static_cast<size_t>(cfg->capacity), d = kHeadDim;
  const size_t code_bytes = bh * C * d * cfg->bits / 8;
  out[KIVI_BUF_K_CODES] = code_bytes;
  out[KIVI_BUF_V_CODES] = code_bytes;
  if (cfg->fine_groups) {
    out[KIVI_BUF_K_SCALE] = out[KIVI_BUF_K_ZERO] = bh * (C / cfg->group_k) * d * 2;
    out[KIVI_BUF_V_SCALE] = out[KIVI_BUF_V_ZERO] = bh * C * (d / cfg->group_v) * 2;
  } else {
    out[KIVI_BUF_K_SCALE] = out[KIVI_BUF_K_ZERO] = bh * (C / cfg->residual) * (d / cfg->group_k) * 2;
    out[KIVI_BUF_V_SCALE] = out[KIVI_BUF_V_ZERO] = bh * (C / cfg->group_v) * 2;
  }
  out[KIVI_BUF_K_RES] = out[KIVI_BUF_V_RES] = bh * cfg->residual * d * 2;
  return KIVI_OK;
}

namespace {

int prefill_impl(const kivi_config* cfg, kivi_cache* cache, const uint16_t* k_dev, const uint16_t* v_dev,
                 int32_t num_tokens, void* stream, bool prefix_k) {
  int st = check_cfg(cfg);
  if (st != KIVI_OK) return st;
  if (cache == nullptr || num_tokens < 1 || !aligned16(k_dev) || !aligned16(v_dev)) return KIVI_ERR_INVALID_ARG;
  const int R = cfg->residual;
  const int n_res = (num_tokens - 1) % R + 1;
  const int n_quant = num_tokens - n_res;
  if (n_quant > cfg->capacity) return KIVI_ERR_CAPACITY;
  if (prefix_k && (cfg->online_k || cfg->fine_groups)) return KIVI_ERR_UNSUPPORTED;
  if (k_online(cfg, n_quant) && n_quant + R > cfg->capacity) return KIVI_ERR_CAPACITY;
  if (!cache_ptrs_ok(cache, n_quant > 0)) return KIVI_ERR_INVALID_ARG;
  kivi::QuantizeArgs a{};
  a.k_src = k_dev;
  a.v_src = v_dev;
  a.k_codes = cache->k_codes;
  a.v_codes = cache->v_codes;
  a.k_scale = cache->k_scale;
  a.k_zero = cache->k_zero;
  a.v_scale = cache->v_scale;
  a.v_zero = cache->v_zero;
  a.k_res = cache->k_res;
  a.v_res = cache->v_res;
  a.bh = cfg->batch * cfg->num_kv_heads;
  a.src_tokens = num_tokens;
  a.src_tok0 = 0;
  a.nblocks = n_quant / R;
  a.dst_blk0 = 0;
  a.res_tok0 = n_quant;
  a.res_tokens = n_res;
  a.residual = R;
  a.capacity = cfg->capacity;
  a.group_k = cfg->group_k;
  a.group_v = cfg->group_v;
  a.fine = cfg->fine_groups;
  if (prefix_k && a.nblocks > 0) {
    if (kivi::launch_k_prefix_extremes(a, cfg->bits, static_cast<cudaStream_t>(stream)) != cudaSuccess)
      return KIVI_ERR_CUDA;
    a.k_given = 1;
  }
  if (kivi::launch_quantize_blocks(a, cfg->bits, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return KIVI_ERR_CUDA;
  if (k_online(cfg, n_quant)) {  // the tail's K rows become codes (the fp16 copy is left unused)
    kivi_cache after = *cache;
    after.n_quant = n_quant;
    if (code_k_online(cfg, &after, k_dev, num_tokens, n_quant, n_res, 0, nullptr, static_cast<cudaStream_t>(stream)) !=
        KIVI_OK)
      return KIVI_ERR_CUDA;
  }
  cache->n_quant = n_quant;
  cache->n_res = n_res;
  return KIVI_OK;
}

}  // namespace

int kivi_quantize_prefill(const kivi_config* cfg, kivi_cache* cache, const uint16_t* k_dev, const uint16_t* v_dev,
                          int32_t num_tokens, void* stream) {
  return prefill_impl(cfg, cache, k_dev, v_dev, num_tokens, stream, false);
}

int kivi_quantize_prefill_prefix_k(const kivi_config* cfg, kivi_cache* cache, const uint16_t* k_dev,
                                   const uint16_t* v_dev, int32_t num_tokens, void* stream) {
  return prefill_impl(cfg, cache, k_dev, v_dev, num_tokens, stream, true);
}

int kivi_append_token(const kivi_config* cfg, kivi_cache* cache, const uint16_t* k_new_dev,
                      const uint16_t* v_new_dev, void* stream) {
  int st = check_cfg(cfg);
  if (st != KIVI_OK) return st;
  if ((st = check_state(cfg, cache)) != KIVI_OK) return st;
  if (!aligned16(k_new_dev) || !aligned16(v_new_dev) || !cache_ptrs_ok(cache, false)) return KIVI_ERR_INVALID_ARG;
  if (cache->n_res == cfg->residual) return KIVI_ERR_RESIDUAL_FULL;
  if (k_online(cfg, cache->n_quant)) {
    if (cache->n_quant + cfg->residual > cfg->capacity) return KIVI_ERR_CAPACITY;
    if (!cache_ptrs_ok(cache, true)) return KIVI_ERR_INVALID_ARG;
    st = code_k_online(cfg, cache, k_new_dev, 1, 0, 1, cache->n_res, v_new_dev, static_cast<cudaStream_t>(stream));
    if (st == KIVI_OK) cache->n_res += 1;
    return st;
  }
  kivi::AppendArgs a{};
  a.k_new = k_new_dev;
  a.v_new = v_new_dev;
  a.k_res = cache->k_res;
  a.v_res = cache->v_res;
  a.bh = cfg->batch * cfg->num_kv_heads;
  a.residual = cfg->residual;
  a.slot = cache->n_res;
  if (kivi::launch_append(a, static_cast<cudaStream_t>(stream)) != cudaSuccess) return KIVI_ERR_CUDA;
  cache->n_res += 1;
  return KIVI_OK;
}

int kivi_flush_residual(const kivi_config* cfg, kivi_cache* cache, void* stream) {
  int st = check_cfg(cfg);
  if (st != KIVI_OK) return st;
  if ((st = check_state(cfg, cache)) != KIVI_OK) return st;
  if (cache->n_res < cfg->residual) return KIVI_ERR_RESIDUAL_NOT_FULL;
  if (cache->n_quant + cfg->residual > cfg->capacity) return KIVI_ERR_CAPACITY;
  if (!cache_ptrs_ok(cache, true)) return KIVI_ERR_INVALID_ARG;
  const int R = cfg->residual;
  kivi::QuantizeArgs a{};
  a.k_src = cache->k_res;
  a.v_src = cache->v_res;
  a.k_codes = cache->k_codes;
  a.v_codes = cache->v_codes;
  a.k_scale = cache->k_scale;
  a.k_zero = cache->k_zero;
  a.v_scale = cache->v_scale;
  a.v_zero = cache->v_zero;
  a.k_res = cache->k_res;
  a.v_res = cache->v_res;
  a.bh = cfg->batch * cfg->num_kv_heads;
  a.src_tokens = R;
  a.src_tok0 = 0;
  a.nblocks = 1;
  a.dst_blk0 = cache->n_quant / R;
  a.res_tokens = 0;
  a.residual = R;
  a.capacity = cfg->capacity;
  a.group_k = cfg->group_k;
  a.group_v = cfg->group_v;
  a.v_only = k_online(cfg, cache->n_quant) ? 1 : 0;  // online K: the block's K codes are in place
  a.fine = cfg->fine_groups;
  if (kivi::launch_quantize_blocks(a, cfg->bits, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return KIVI_ERR_CUDA;
  cache->n_quant += R;
  cache->n_res = 0;
  return KIVI_OK;
}

size_t kivi_decode_workspace_bytes(const kivi_config* cfg, int32_t num_q_heads) {
  if (check_cfg(cfg) != KIVI_OK || num_q_heads < 1 || num_q_heads % cfg->num_kv_heads != 0) return 0;
  const int gqa = num_q_heads / cfg->num_kv_heads;
  if (!gqa_supported(gqa)) return 0;
  DecodePlan p{};
  if (get_plan(cfg->bits, gqa, cfg->fine_groups, &p) != cudaSuccess) return 0;
  const size_t bh = static_cast<size_t>(cfg->batch) * cfg->num_kv_heads;
  return align256(static_cast<size_t>(p.workers()) * 2 * gqa * kivi::kPartialStride * sizeof(float)) +
         align256(bh * sizeof(int32_t));
}

namespace {

// Decode attention over `cache` (whose counters already include a fused append's token, which
// k_new / v_new hold for residual slot new_slot; new_slot < 0: no append; -2: check the
// arguments only and enqueue nothing).  flush: the appended token fills the residual, and the same
// launch quantizes the residual as block n_quant / R (the caller updates the counters).
int decode_impl(const kivi_config* cfg, const kivi_cache* cache, const uint16_t* q_dev, int32_t num_q_heads,
                float scale, uint16_t* out_dev, void* workspace_dev, size_t workspace_bytes, int32_t* dev_status,
                void* stream, const uint16_t* k_new_dev, const uint16_t* v_new_dev, int new_slot,
                bool flush = false) {
  int st = check_cfg(cfg);
  if (st != KIVI_OK) return st;
  if ((st = check_state(cfg, cache)) != KIVI_OK) return st;
  if (num_q_heads < 1 || num_q_heads % cfg->num_kv_heads != 0) return KIVI_ERR_INVALID_ARG;
  const int gqa = num_q_heads / cfg->num_kv_heads;
  if (!gqa_supported(gqa)) return KIVI_ERR_UNSUPPORTED;
  if (!aligned16(q_dev) || !aligned16(out_dev) || !(scale == scale) || scale > 3.0e38f || scale < -3.0e38f)
    return KIVI_ERR_INVALID_ARG;
  if (cache->n_quant + cache->n_res == 0) return KIVI_ERR_EMPTY;
  if (!cache_ptrs_ok(cache, cache->n_quant > 0)) return KIVI_ERR_INVALID_ARG;
  const bool coded_res = k_online(cfg, cache->n_quant) && cache->n_res > 0;
  if (coded_res && (cache->n_quant + cfg->residual > cfg->capacity || new_slot >= 0)) return KIVI_ERR_STATE;
  if (dev_status != nullptr && (reinterpret_cast<uintptr_t>(dev_status) & 3u) != 0) return KIVI_ERR_INVALID_ARG;
  DecodePlan plan{};
  if (get_plan(cfg->bits, gqa, cfg->fine_groups, &plan) != cudaSuccess) return KIVI_ERR_CUDA;
  const size_t bh = static_cast<size_t>(cfg->batch) * cfg->num_kv_heads;
  const size_t part_bytes = align256(static_cast<size_t>(plan.workers()) * 2 * gqa * kivi::kPartialStride * 4);
  if (workspace_dev == nullptr || (reinterpret_cast<uintptr_t>(workspace_dev) & 255u) != 0 ||
      workspace_bytes < part_bytes + align256(bh * 4))
    return KIVI_ERR_WORKSPACE;

  DecodeArgs a{};
  a.k_codes = cache->k_codes;
  a.v_codes = cache->v_codes;
  a.k_scale = cache->k_scale;
  a.k_zero = cache->k_zero;
  a.v_scale = cache->v_scale;
  a.v_zero = cache->v_zero;
  a.k_res = cache->k_res;
  a.v_res = cache->v_res;
  a.q = q_dev;
  a.out = out_dev;
  a.partials = static_cast<float*>(workspace_dev);
  a.tickets = reinterpret_cast<int32_t*>(static_cast<char*>(workspace_dev) + part_bytes);
  a.status = dev_status;
  a.bh = static_cast<int>(bh);
  a.gqa = gqa;
  a.capacity = cfg->capacity;
  a.residual = cfg->residual;
  a.group_k = cfg->group_k;
  a.group_v = cfg->group_v;
  a.n_quant = cache->n_quant;
  a.n_res = cache->n_res;
  a.units_q = cache->n_quant / plan.unit_tokens;
  a.units = a.units_q + (cache->n_res + plan.res_unit_tokens - 1) / plan.res_unit_tokens;
  a.total_units = static_cast<long long>(bh) * a.units;
  a.blocks_per_head = cfg->capacity / cfg->residual;
  a.vgroups_per_head = cfg->capacity / cfg->group_v;
  a.lg_gk = log2i(cfg->group_k);
  a.lg_gv = log2i(cfg->group_v);
  a.lg_units_per_blk = log2i(cfg->residual / plan.unit_tokens);
  // every worker must own at least one unit: the merge counts all workers that touch a head
  long long workers = a.total_units < plan.workers() ? a.total_units : plan.workers();
  {
    DebugState& d = debug_state();
    std::lock_guard<std::mutex> lock(d.mu);
    if (d.max_workers > 0 && d.max_workers < workers) workers = d.max_workers;
  }
  a.workers = static_cast<int>(workers);
  a.qscale = scale * 1.4426950408889634f;
  {
    DebugState& d = debug_state();
    std::lock_guard<std::mutex> lock(d.mu);
    a.timeout_ns = d.timeout_ns;
    a.debug_extra_tx = d.mode == 1 ? 16u : 0u;
#ifdef KIVI_DEBUG
    // test hook of the debug build: units the kernel's bounds checks must refuse.  The extra units
    // lie inside the capacity (checked here), so even an unguarded copy would stay in bounds.
    if (d.units_q_skew > 0 && !coded_res && !cfg->fine_groups &&
        static_cast<long long>(a.units_q + d.units_q_skew) * plan.unit_tokens <= cfg->capacity) {
      a.units_q += d.units_q_skew;
      a.units += d.units_q_skew;
      a.total_units = static_cast<long long>(bh) * a.units;
      if (a.workers > a.total_units) a.workers = static_cast<int>(a.total_units);
    }
#endif
  }
  a.k_new = k_new_dev;
  a.v_new = v_new_dev;
  a.new_slot = new_slot;
  a.k_res_coded = coded_res ? 1 : 0;
  a.fine = cfg->fine_groups;
  a.res_blk = cache->n_quant / cfg->residual;
  a.flush_blk = -1;
  if (flush) {  // the caller passes only full residuals of the base groups with fp16 residual keys
    if ((new_slot != -2 && new_slot != cfg->residual - 1) || cache->n_res != cfg->residual || coded_res || cfg->fine_groups ||
        cache->n_quant + cfg->residual > cfg->capacity)
      return KIVI_ERR_INTERNAL;
    if (!cache_ptrs_ok(cache, true)) return KIVI_ERR_INVALID_ARG;
    a.flush_blk = cache->n_quant / cfg->residual;
    a.fk_codes = cache->k_codes;
    a.fv_codes = cache->v_codes;
    a.fk_scale = cache->k_scale;
    a.fk_zero = cache->k_zero;
    a.fv_scale = cache->v_scale;
    a.fv_zero = cache->v_zero;
  }
  if (new_slot == -2) return KIVI_OK;  // arguments checked, nothing enqueued
  if (kivi::launch_decode(a, cfg->bits, plan, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return KIVI_ERR_CUDA;
  return KIVI_OK;
}

}  // namespace

int kivi_decode_attention(const kivi_config* cfg, const kivi_cache* cache, const uint16_t* q_dev,
                          int32_t num_q_heads, float scale, uint16_t* out_dev, void* workspace_dev,
                          size_t workspace_bytes, int32_t* dev_status, void* stream) {
  return decode_impl(cfg, cache, q_dev, num_q_heads, scale, out_dev, workspace_dev, workspace_bytes, dev_status,
                     stream, nullptr, nullptr, -1);
}

int kivi_append_decode_attention(const kivi_config* cfg, kivi_cache* cache, const uint16_t* k_new_dev,
                                 const uint16_t* v_new_dev, const uint16_t* q_dev, int32_t num_q_heads, float scale,
                                 uint16_t* out_dev, void* workspace_dev, size_t workspace_bytes, int32_t* dev_status,
                                 void* stream) {
  int st = check_cfg(cfg);
  if (st != KIVI_OK) return st;
  if ((st = check_state(cfg, cache)) != KIVI_OK) return st;
  if (!aligned16(k_new_dev) || !aligned16(v_new_dev) || !cache_ptrs_ok(cache, false)) return KIVI_ERR_INVALID_ARG;
  if (cache->n_res == cfg->residual) return KIVI_ERR_RESIDUAL_FULL;
  if (k_online(cfg, cache->n_quant)) {  // the K row is coded by its own launch before it is attended
    if (cache->n_quant + cfg->residual > cfg->capacity) return KIVI_ERR_CAPACITY;
    kivi_cache after = *cache;
    after.n_res += 1;
    // every argument check of the decode runs before anything is enqueued
    st = decode_impl(cfg, &after, q_dev, num_q_heads, scale, out_dev, workspace_dev, workspace_bytes, dev_status,
                     stream, nullptr, nullptr, -2);
    if (st != KIVI_OK) return st;
    if ((st = kivi_append_token(cfg, cache, k_new_dev, v_new_dev, stream)) != KIVI_OK) return st;
    st = decode_impl(cfg, cache, q_dev, num_q_heads, scale, out_dev, workspace_dev, workspace_bytes, dev_status,
                     stream, nullptr, nullptr, -1);
    if (st != KIVI_OK) cache->n_res -= 1;  // a failed launch: the counters are left as they were
    return st;
  }
  kivi_cache after = *cache;
  after.n_res += 1;
  st = decode_impl(cfg, &after, q_dev, num_q_heads, scale, out_dev, workspace_dev, workspace_bytes, dev_status,
                   stream, k_new_dev, v_new_dev, cache->n_res);
  if (st == KIVI_OK) cache->n_res += 1;
  return st;
}

int kivi_decode_step(const kivi_config* cfg, kivi_cache* cache, const uint16_t* k_new_dev, const uint16_t* v_new_dev,
                     const uint16_t* q_dev, int32_t num_q_heads, float scale, uint16_t* out_dev, void* workspace_dev,
                     size_t workspace_bytes, int32_t* dev_status, void* stream) {
  int st = check_cfg(cfg);
  if (st != KIVI_OK) return st;
  if ((st = check_state(cfg, cache)) != KIVI_OK) return st;
  if (!aligned16(k_new_dev) || !aligned16(v_new_dev) || !cache_ptrs_ok(cache, false)) return KIVI_ERR_INVALID_ARG;
  const int R = cfg->residual;
  // the state the append sees: a residual left full by an earlier call is flushed first
  kivi_cache cur = *cache;
  const bool pre_flush = cur.n_res == R;
  if (pre_flush) {
    if (cur.n_quant + R > cfg->capacity) return KIVI_ERR_CAPACITY;
    if (!cache_ptrs_ok(cache, true)) return KIVI_ERR_INVALID_ARG;
    cur.n_quant += R;
    cur.n_res = 0;
  }
  const bool online = k_online(cfg, cur.n_quant);
  if (online && cur.n_quant + R > cfg->capacity) return KIVI_ERR_CAPACITY;
  const bool flush = cur.n_res + 1 == R && cur.n_quant + R <= cfg->capacity;
  if (flush && !cache_ptrs_ok(cache, true)) return KIVI_ERR_INVALID_ARG;  // the flush writes the block arrays
  // online K past the first block, and fine-grained groups, flush with their own launch
  const bool fused_flush = flush && !online && !cfg->fine_groups;
  // every argument check of the attention, on the state it will see, before anything is enqueued
  kivi_cache after = cur;
  after.n_res += 1;
  st = decode_impl(cfg, &after, q_dev, num_q_heads, scale, out_dev, workspace_dev, workspace_bytes, dev_status, stream,
                   nullptr, nullptr, -2, fused_flush);
  if (st != KIVI_OK) return st;
  if (pre_flush && (st = kivi_flush_residual(cfg, cache, stream)) != KIVI_OK) return st;
  if (!fused_flush) {
    st = kivi_append_decode_attention(cfg, cache, k_new_dev, v_new_dev, q_dev, num_q_heads, scale, out_dev,
                                      workspace_dev, workspace_bytes, dev_status, stream);
    if (st == KIVI_OK && flush) st = kivi_flush_residual(cfg, cache, stream);
    return st;
  }
  after = *cache;
  after.n_res += 1;
  st = decode_impl(cfg, &after, q_dev, num_q_heads, scale, out_dev, workspace_dev, workspace_bytes, dev_status, stream,
                   k_new_dev, v_new_dev, cache->n_res, true);
  if (st == KIVI_OK) {
    cache->n_quant += R;
    cache->n_res = 0;
  }
  return st;
}

int kivi_read_status(const int32_t* dev_status, void* stream) {
  if (dev_status == nullptr) return KIVI_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return KIVI_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpy(&v, dev_status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return KIVI_ERR_CUDA;
  return v;
}

int kivi_debug_inject(int32_t mode, uint64_t value) {
  DebugState& d = debug_state();
  std::lock_guard<std::mutex> lock(d.mu);
  switch (mode) {
    case 0:
      d.mode = 0;
      d.timeout_ns = kDefaultTimeoutNs;
      d.max_workers = 0;
      d.units_q_skew = 0;
      return KIVI_OK;
    case 1:
      d.mode = 1;
      d.timeout_ns = value == 0 ? kDefaultTimeoutNs : value;
      return KIVI_OK;
    case 2:
      d.max_workers = static_cast<long long>(value);
      return KIVI_OK;
    case 3:
#ifdef KIVI_DEBUG
      d.units_q_skew = static_cast<int>(value > 8 ? 8 : value);
      return KIVI_OK;
#else
      return KIVI_ERR_UNSUPPORTED;
#endif
    default:
      return KIVI_ERR_INVALID_ARG;
  }
}

int kivi_debug_status(void) {
#ifdef KIVI_DEBUG
  if (cudaDeviceSynchronize() != cudaSuccess) return KIVI_ERR_CUDA;
  int32_t q = 0, d = 0;
  if (kivi::debug_status_quantize(&q) != cudaSuccess || kivi::debug_status_decode(&d) != cudaSuccess)
    return KIVI_ERR_CUDA;
  return q != 0 ? q : d;
#else
  return KIVI_ERR_UNSUPPORTED;
#endif
}

}  // extern "C"
