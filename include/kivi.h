/*
 * kivi.h - C ABI of the B200 (sm_100a) KIVI-style asymmetric low-bit KV-cache library.
 *
 * Method source: the KIVI explainer page "ICML 2024論文解説: KIVI — チューニング不要のKVキャッシュ2bit
 * 非対称量子化" (arXiv 2402.02750). Section and equation names below refer to that page.
 *
 *   Q(X) = clamp(round((X - z) / s), 0, 2^b - 1)         section 量子化アルゴリズム, Q equation
 *   D(X^) = s * X^ + z                                   section 量子化アルゴリズム, D equation
 *   s = (max X_g - min X_g) / (2^b - 1),  z = min X_g    section 量子化アルゴリズム, s/z equation
 *   K: groups of g_k consecutive channels                section Per-Channel量子化（Key Cache）
 *   V: groups of g_v consecutive tokens                  section Per-Token量子化（Value Cache）
 *   newest tokens stay fp16 in a residual buffer;        section 残差バッファ（Residual Buffer）,
 *   attention = softmax(q [D(Kq); Kres]^T / sqrt(d)) [D(Vq); Vres]   Attention equation
 *
 * Readings this library fixes where the page leaves a step open:
 *   - A K group is one R-token block x g_k consecutive channels (every R-token block gets its own
 *     scale/zero per channel group); a V group is g_v consecutive tokens x all d channels.
 *   - s is stored as fp16, rounded to nearest-even from the exact real (max-min)/(2^b-1);
 *     z = min is stored as fp16 (exact).
 *   - A code is round-half-to-even of the EXACT rational (x - z)/s computed with the stored fp16
 *     s and z, then clamped to [0, 2^b-1].  s == 0 gives code 0 (D reproduces z).
 *   - The residual always holds the newest 1..R tokens once anything is cached; a full residual
 *     is flushed (quantized as one R-token block) before the next append.
 *
 * Every pointer argument named *_dev is DEVICE memory owned by the caller; the library never
 * allocates, frees or retains memory (kivi_decode_attention_noalloc's fixed scratch array is
 * part of the library image, not an allocation).
 * fp16 values are passed as their IEEE binary16 bit patterns (uint16_t).  Every call is
 * asynchronous on `stream` (a cudaStream_t passed as void*; NULL = legacy default stream) and
 * returns a status code synchronously.  On any error return nothing has been enqueued and the
 * cache counters are unchanged.
 *
 * DEVICE LAYOUT (B batch, H = num_kv_heads, d = head_dim, b = bits, P = 32/b codes per uint32,
 * R = residual, C = capacity, G_k = group_k, G_v = group_v; all arrays dense, row-major):
 *   k_codes  uint32 [B][H][C][d/P]   token-major.  Word i of token t holds the codes of channels
 *                                     P*i + j (j = 0..P-1) at bits [b*j, b*j + b).
 *   v_codes  uint32 [B][H][C/P][d]   channel-major within P-token rows.  Word (r, c) holds the
 *                                     codes of tokens P*r + j of channel c at bits [b*j, b*j + b).
 *   k_scale, k_zero  fp16 [B][H][C/R][d/G_k]   one pair per (R-token block, channel group);
 *                    fine_groups: [B][H][C/G_k][d], one pair per (G_k-token group, channel).
 *   v_scale, v_zero  fp16 [B][H][C/G_v]        one pair per G_v-token group;
 *                    fine_groups: [B][H][C][d/G_v], one pair per (token, G_v-channel group).
 *   k_res, v_res     fp16 [B][H][R][d]         residual slots 0..n_res-1 hold the newest tokens.
 *   Token order of a head: quantized tokens 0..n_quant-1, then residual slots 0..n_res-1.
 * Host inputs: k, v fp16 [B][H][T][d]; k_new, v_new fp16 [B][H][d]; q, out fp16 [B][Hq][d].
 * Query head h attends with KV head h / (Hq/H) (contiguous grouped-query mapping).
 *
 * Every device pointer must be 16-byte aligned.
 */
#ifndef KIVI_H
#define KIVI_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KIVI_ABI_VERSION 4

/* Status codes. */
#define KIVI_OK 0
#define KIVI_ERR_INVALID_ARG 1       /* NULL/misaligned pointer or a shape rule below violated */
#define KIVI_ERR_UNSUPPORTED 2       /* bits not in {2,4}, head_dim not 128, or a size limit */
#define KIVI_ERR_CAPACITY 3          /* the call would exceed `capacity` quantized tokens */
#define KIVI_ERR_RESIDUAL_FULL 4     /* append with n_res == R: flush first */
#define KIVI_ERR_RESIDUAL_NOT_FULL 5 /* flush with n_res < R */
#define KIVI_ERR_EMPTY 6             /* attention over an empty cache */
#define KIVI_ERR_WORKSPACE 7         /* workspace NULL, misaligned or too small */
#define KIVI_ERR_CUDA 8              /* a CUDA runtime call or kernel launch failed */
#define KIVI_ERR_DEVICE_TIMEOUT 9    /* a bounded device-side wait expired (reported via status) */
#define KIVI_ERR_STATE 10            /* cache counters inconsistent with the call */
#define KIVI_ERR_INTERNAL 11         /* a device-side consistency check failed (reported via status) */

/*
 * Quantization configuration; mirrors the page's QuantConfig (section アルゴリズム: bits,
 * group_size_k, group_size_v, residual_length) plus the shape and capacity of the cache.
 * Rules: batch >= 1, num_kv_heads >= 1, capacity >= 0, capacity % residual == 0,
 * residual in {128, 256, 512, 1024}, group_k in {32, 64, 128}, group_v a power of two with
 * 32 <= group_v <= residual, online_k in {0, 1}, fine_groups in {0, 1} (KIVI_ERR_INVALID_ARG otherwise);
 * head_dim == 128, bits in {2, 4} (KIVI_ERR_UNSUPPORTED otherwise).
 *
 * online_k = 1 selects online K quantization (section Per-Channel量子化: a new token's K can be
 * quantized at once with the existing scale and zero point).  Once a quantized block exists
 * (n_quant > 0), the K row of every residual token is stored as codes, not fp16: token
 * n_quant + i is code row n_quant + i of k_codes, coded with the (s, z) of block n_quant/R - 1,
 * clamped to [0, 2^b-1], and block n_quant/R holds a copy of that (s, z).  V keeps its fp16
 * residual and its flush.  Before the first block exists K stays fp16 as with online_k = 0.
 * Such a cache needs n_quant + R <= capacity whenever it holds residual tokens (KIVI_ERR_CAPACITY
 * from the prefill or append that would break it).
 *
 * fine_groups = 1 selects fine-grained groups (section KVキャッシュの分布特性: the K range along each
 * channel, the V range along each token): group_k then counts TOKENS (one K (s, z) per channel per
 * group_k consecutive tokens; group_k in {32, 64, 128}, group_k <= residual) and group_v counts
 * CHANNELS (one V (s, z) per token per group_v consecutive channels; group_v in {32, 64, 128}).
 * The scale layouts change (see DEVICE LAYOUT); codes, residual, blocks and flushes do not.
 * Decode attention over such a cache works at both bit widths and every query-head ratio; it is
 * not combined with online_k or the prefix-K prefill (KIVI_ERR_UNSUPPORTED).
 */
typedef struct kivi_config {
  int32_t batch;        /* B */
  int32_t num_kv_heads; /* H */
  int32_t head_dim;     /* d: 128 */
  int32_t bits;         /* b: 2 or 4 */
  int32_t group_k;      /* G_k: channels per K group */
  int32_t group_v;      /* G_v: tokens per V group */
  int32_t residual;     /* R: residual (fp16) capacity in tokens, also the K block length */
  int32_t capacity;     /* C: maximum number of quantized tokens per head */
  int32_t online_k;     /* 0: K residual in fp16; 1: online K quantization (see above) */
  int32_t fine_groups;  /* 0: block / token groups; 1: fine-grained groups (see above) */
} kivi_config;

/* Device buffers of one cache (caller-owned) plus the two host-side counters the calls advance.
 * n_quant is always a multiple of R; 0 <= n_res <= R.  Counters are uniform over (batch, head). */
typedef struct kivi_cache {
  uint32_t *k_codes, *v_codes;
  uint16_t *k_scale, *k_zero, *v_scale, *v_zero;
  uint16_t *k_res, *v_res;
  int32_t n_quant;
  int32_t n_res;
} kivi_cache;

/* Index of each buffer in kivi_cache_sizes' output. */
enum {
  KIVI_BUF_K_CODES = 0, KIVI_BUF_V_CODES, KIVI_BUF_K_SCALE, KIVI_BUF_K_ZERO,
  KIVI_BUF_V_SCALE, KIVI_BUF_V_ZERO, KIVI_BUF_K_RES, KIVI_BUF_V_RES, KIVI_NUM_BUFS
};

/* Writes the byte size of each cache buffer (layout above) into out_bytes[KIVI_NUM_BUFS].
 * Host-only; no CUDA call.  Returns KIVI_OK or KIVI_ERR_INVALID_ARG / KIVI_ERR_UNSUPPORTED. */
int kivi_cache_sizes(const kivi_config* cfg, size_t* out_bytes);

/* Checks cfg against the rules above without touching the device. */
int kivi_check_config(const kivi_config* cfg);

/*
 * Prefill: quantizes a prompt of T tokens per head and resets the cache.
 * Sections 量子化アルゴリズム, Per-Channel量子化, Per-Token量子化 and 残差バッファ.
 * k_dev, v_dev: fp16 [B][H][T][d].  Afterwards n_res = ((T-1) mod R) + 1 and
 * n_quant = T - n_res (so T <= R keeps everything in fp16); tokens [0, n_quant) are quantized
 * as n_quant/R blocks and tokens [n_quant, T) are copied into residual slots 0..n_res-1.
 * With online_k and n_quant > 0 the tail's K rows are coded instead (a second launch).
 * Errors: T < 1 (INVALID_ARG), n_quant > capacity (CAPACITY).  One kernel launch.
 */
int kivi_quantize_prefill(const kivi_config* cfg, kivi_cache* cache, const uint16_t* k_dev,
                          const uint16_t* v_dev, int32_t num_tokens, void* stream);

/*
 * Prefill under the other reading of section Per-Channel量子化, in which one K group spans every
 * quantized token of the prompt instead of one R-token block: the K scale and zero of each
 * channel group are taken over tokens [0, n_quant) and stored in every block's slot, so decode
 * attention, appends and later flushes (which quantize their own R-token blocks) are unchanged.
 * V groups, the residual split, arguments and errors are those of kivi_quantize_prefill.
 * Two kernel launches (the K group extremes over the prefix, then the quantization).
 * online_k = 1 is not combined with this reading (KIVI_ERR_UNSUPPORTED).
 */
int kivi_quantize_prefill_prefix_k(const kivi_config* cfg, kivi_cache* cache, const uint16_t* k_dev,
                                   const uint16_t* v_dev, int32_t num_tokens, void* stream);

/*
 * Append: writes one new token's K and V (fp16 [B][H][d]) into residual slot n_res and
 * increments n_res.  Section 残差バッファ.  With online_k and n_quant > 0 the K row is coded
 * into code row n_quant + n_res instead (section Per-Channel量子化), and the first append after
 * a flush copies block n_quant/R - 1's K (s, z) into block n_quant/R.
 * Errors: n_res == R (RESIDUAL_FULL); online K with n_quant + R > capacity (CAPACITY).  One launch.
 */
int kivi_append_token(const kivi_config* cfg, kivi_cache* cache, const uint16_t* k_new_dev,
                      const uint16_t* v_new_dev, void* stream);

/*
 * Flush: quantizes the full residual (R tokens) as quantized block n_quant/R, then
 * n_quant += R, n_res = 0.  Sections Per-Token量子化 (flush once the group fills) and 残差バッファ.
 * With online_k and n_quant > 0 only V is quantized: the block's K codes and (s, z) are in place.
 * Errors: n_res < R (RESIDUAL_NOT_FULL), n_quant + R > capacity (CAPACITY).  One launch.
 */
int kivi_flush_residual(const kivi_config* cfg, kivi_cache* cache, void* stream);

/* Bytes of scratch workspace kivi_decode_attention needs for this config and query-head count.
 * Returns 0 if the arguments are invalid.  The size does not depend on the cache counters. */
size_t kivi_decode_workspace_bytes(const kivi_config* cfg, int32_t num_q_heads);

/*
 * Decode attention for one query token per query head over the whole cache:
 *   out[b][h] = softmax(scale * q[b][h] . [D(Kq); Kres]^T) [D(Vq); Vres]
 * Section 残差バッファ, Attention equation (scale = 1/sqrt(d_k) there; any finite scale accepted).
 * q_dev, out_dev: fp16 [B][Hq][d]; Hq must be a multiple of H.
 * workspace_dev: kivi_decode_workspace_bytes(cfg, Hq) bytes, 256-byte aligned; it must be ZERO
 * before its first use and is left zero by every call that completes without a device error
 * (after a device error, zero it again).  Calls sharing one workspace must not overlap.
 * dev_status: optional (may be NULL) device int32 that receives KIVI_ERR_DEVICE_TIMEOUT if a
 * bounded wait inside the kernel expires; the caller zeroes it and reads it with kivi_read_status.
 * With online_k and n_quant > 0 the residual tokens' keys are their codes (dequantized with the
 * block's copied (s, z)) and their values the fp16 residual rows.
 * Errors: empty cache (EMPTY), workspace too small (WORKSPACE).  One kernel launch.
 */
int kivi_decode_attention(const kivi_config* cfg, const kivi_cache* cache, const uint16_t* q_dev,
                          int32_t num_q_heads, float scale, uint16_t* out_dev, void* workspace_dev,
                          size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * Append and decode attention in one launch: the same results and cache contents as
 * kivi_append_token(k_new, v_new) followed by kivi_decode_attention(q).  Section 残差バッファ: the
 * newest token joins the fp16 residual and is attended at once.
 * The new token's K and V (fp16 [B][H][d], 16-byte aligned) are written into residual slot n_res
 * by the decode kernel itself: the warp that attends the residual rows of that slot copies the
 * row into its shared-memory tile and into the cache.  On success n_res is incremented; on any
 * error the counters are unchanged (a device error may leave the slot written, as with a failed
 * append).  Arguments and errors are those of the two calls; RESIDUAL_FULL when n_res == R
 * (flush first).  One kernel launch; with online_k and n_quant > 0 the K row must be coded before
 * it is attended, and the call enqueues kivi_append_token and kivi_decode_attention (two launches).
 */
int kivi_append_decode_attention(const kivi_config* cfg, kivi_cache* cache, const uint16_t* k_new_dev,
                                 const uint16_t* v_new_dev, const uint16_t* q_dev, int32_t num_q_heads,
                                 float scale, uint16_t* out_dev, void* workspace_dev, size_t workspace_bytes,
                                 int32_t* dev_status, void* stream);

/*
 * One streaming decode step: append one token, attend, and quantize the residual as soon as it is
 * full.  Section 残差バッファ: the newest tokens stay fp16 and R of them become one quantized block
 * (the quantization of sections 量子化アルゴリズム, Per-Channel量子化 and Per-Token量子化).  The
 * attention output is that of kivi_append_decode_attention(k_new, v_new, q); in addition, when
 * the appended token fills the residual (n_res becomes R) and n_quant + R <= capacity, the same
 * launch quantizes the R residual tokens as block n_quant / R, bit-exactly as kivi_flush_residual
 * would, and on success the counters become n_quant + R and n_res = 0.  The flush is eager (at the
 * step that fills the residual) rather than lazy (at the next step): the outputs of every step are
 * the same either way, since the step that fills the residual attends its tokens in fp16 and the
 * next one attends the new block.
 * Launches: one per step, flush steps included, for the base groups while the residual keys are
 * fp16.  With online_k and n_quant > 0 (and with fine_groups) the step enqueues
 * kivi_append_decode_attention and, on a filling step, kivi_flush_residual.  A residual that is
 * already full when the call starts (left by other calls) is flushed first, by its own launch.
 * Arguments: those of kivi_append_decode_attention.  Errors: those of the calls it stands for,
 * checked before anything is enqueued; CAPACITY when the residual is full at entry and cannot be
 * flushed.  When the residual fills and no block is left (n_quant + R > capacity) the step attends
 * and leaves n_res = R; the next step then returns CAPACITY.
 */
int kivi_decode_step(const kivi_config* cfg, kivi_cache* cache, const uint16_t* k_new_dev, const uint16_t* v_new_dev,
                     const uint16_t* q_dev, int32_t num_q_heads, float scale, uint16_t* out_dev, void* workspace_dev,
                     size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * Largest scratch kivi_decode_attention_noalloc can use, in bytes (see below).
 */
#define KIVI_NOALLOC_SCRATCH_BYTES (16u << 20)

/*
 * Decode attention that allocates nothing.  The paper has no counterpart: this is a variant of
 * kivi_decode_attention for callers that cannot allocate device memory when they decode, for
 * example a serving process that hands all free device memory to its own pool at start-up (a
 * cudaMalloc later would fail or stall the step), or a host that gives this library only the
 * input and output buffers of each call.  Arguments, results and errors are those of
 * kivi_decode_attention without the workspace: the scratch (split partials and per-head tickets)
 * lives in a fixed array of KIVI_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that
 * loads the library holds until the process exits.  The caller still passes q and out.
 *   - Limit: if kivi_decode_workspace_bytes(cfg, num_q_heads) exceeds KIVI_NOALLOC_SCRATCH_BYTES
 *     (very many heads), the call returns KIVI_ERR_WORKSPACE and enqueues nothing; use
 *     kivi_decode_attention with a caller workspace instead.
 *   - Set-up: the first call on each device looks up the array's device address on that device
 *     (cudaGetSymbolAddress); make that first call before any stream capture.
 *   - Sharing: every call uses the same array.  Each call first clears the tickets (an async
 *     memset on `stream`), so the contents left by an earlier call, even a failed one, do not
 *     matter; but calls whose work overlaps on the GPU (different streams, or several host threads
 *     on one device) race on the array and must be serialized by the caller.
 */
int kivi_decode_attention_noalloc(const kivi_config* cfg, const kivi_cache* cache, const uint16_t* q_dev,
                                  int32_t num_q_heads, float scale, uint16_t* out_dev, int32_t* dev_status,
                                  void* stream);

/* Synchronizes `stream` and returns the device-side status word (KIVI_OK if it is 0). */
int kivi_read_status(const int32_t* dev_status, void* stream);

/* Human-readable name of a status code (static string). */
const char* kivi_strerror(int status);

/* KIVI_ABI_VERSION of the loaded library. */
int kivi_abi_version(void);

/*
 * Debug build (nvcc -DKIVI_DEBUG, e.g. python -m bit_asymmetric_kv_02_b200.build --debug, which
 * writes libkivi_debug.so; no counterpart on the page).  Every kernel checks the index ranges of its
 * global-memory accesses (copy sources inside the head's arrays and filled tokens, scale indices,
 * destination blocks, residual slots, partial and ticket slots) and, instead of making an access
 * that fails its check, records KIVI_ERR_INTERNAL (in dev_status too, when given) and skips it; no
 * kernel traps.  kivi_debug_status() synchronizes the device and returns the first such status
 * since the previous call (KIVI_OK if none), then clears it.  A release build returns
 * KIVI_ERR_UNSUPPORTED.
 */
int kivi_debug_status(void);

/*
 * Test hooks (no counterpart on the page); process-wide, not for production use.
 *   mode 0: restore normal operation.
 *   mode 1: every later kivi_decode_attention makes its bulk-copy barriers expect 16 bytes more
 *           than are copied, so each bounded wait runs out after `value` ns (0: the 2 s default)
 *           and the kernel reports KIVI_ERR_DEVICE_TIMEOUT through dev_status and returns (the
 *           output is then undefined).
 *   mode 2: cap the number of decode workers (warps) at `value` (0: no cap), to exercise the
 *           split-and-merge path with chosen splits.
 *   mode 3: debug build only (KIVI_ERR_UNSUPPORTED otherwise): later decode launches see `value`
 *           (at most 8) quantized units more than n_quant holds, when they still fit the capacity,
 *           so that the kernel's bounds checks refuse those units and report KIVI_ERR_INTERNAL.
 */
int kivi_debug_inject(int32_t mode, uint64_t value);

#ifdef __cplusplus
}
#endif

#endif /* KIVI_H */
