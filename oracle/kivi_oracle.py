"""CPU oracle: KIVI-style asymmetric low-bit KV-cache quantization and decode attention.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import or run this module.  The
CUDA library never calls it and shares no code, table or helper with it.

Plain numpy, float64 arithmetic, written for reading rather than speed.  Method source: the KIVI
explainer page "ICML 2024論文解説: KIVI — チューニング不要のKVキャッシュ2bit非対称量子化"
(arXiv 2402.02750).  Each function names the section / equation of that page it follows.

Readings taken where the page leaves a step open (each is pinned by tests/test_oracle_pins.py):
  * K group = one R-token block x G_k consecutive channels; V group = G_v consecutive tokens x
    all d channels (sections Per-Channel量子化 / Per-Token量子化, their K_quant / V_quant equations).
  * z is the group minimum itself (exact in fp16); a minimum of -0 is stored as +0.
  * s is stored in fp16: the exact real (max-min)/(2^b-1) rounded to nearest, ties to even.
    The subtraction of two fp16 values is exact in fp64 and the quotient by 3 or 15 cannot
    fall onto an fp16 rounding midpoint unless it is exactly one, so "fp64 divide, then round to
    fp16" is the correctly rounded value.
  * A code is round-half-to-even of the exact rational (x - z)/s with the STORED fp16 s and z,
    clamped to [0, 2^b-1]; s == 0 gives code 0.  (x - z) is exact in fp64; the fp64 quotient is
    within 2^-50 of the exact value, far closer than any non-tie can be to a half-integer, so
    np.rint of it gives the exact decision.  This is checked against exact rationals.
  * The residual holds the newest 1..R tokens; prefill of T tokens keeps ((T-1) mod R)+1 of them
    in fp16 and quantizes the rest as R-token blocks; a full residual is flushed before an append.
  * Decode attention follows the Attention equation of section 残差バッファ: logits over the
    dequantized quantized tokens followed by the fp16 residual tokens, softmax, weighted sum of
    the matching V rows.  No mask; the query-head -> KV-head map is contiguous (h // (Hq/H)).
  * Fine-grained groups (an opt-in variant, section KVキャッシュの分布特性: K ranges are taken along
    each channel, V ranges along each token): K has one (s, z) per channel per g_k consecutive tokens,
    V one per token per g_v consecutive channels.  Blocks, residual and flushes are as in the base
    scheme; only the group axes (and so the scale layouts) change.
  * Online K (an opt-in variant, section Per-Channel量子化: a new token's K can be quantized at
    once with the existing scale and zero point): once a quantized block exists, every new K row
    is coded at append time with the (s, z) of the newest quantized block, clamped to [0, 2^b-1];
    the block being filled keeps a copy of those (s, z).  No K row stays fp16; V keeps its fp16
    residual and is quantized when the residual fills, as in the base scheme.  Before the first
    block exists there are no scales to reuse and K stays in the fp16 residual.

Parity pinned: every public function below is pinned by at least one test that does not reuse
its code (exact rationals, nearest-grid-point brute force, hand-derived fixtures, closed forms,
textbook attention).
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "OracleError", "levels", "codes_per_word", "fp16_round", "scale_zero", "quantize_values",
    "quantize_k_block", "quantize_v_block", "pack_k", "pack_v", "unpack_k", "unpack_v",
    "dequantize_k", "dequantize_v", "attention", "HeadCache", "OracleCache",
    "quantize_k_block_fine", "quantize_v_block_fine", "dequantize_k_fine", "dequantize_v_fine",
]


class OracleError(Exception):
    """Raised for a call the cache contract forbids; ``.code`` names the matching C status."""

    def __init__(self, code: str, msg: str = ""):
        super().__init__(f"{code}: {msg}")
        self.code = code


def levels(bits: int) -> int:
    """Largest code 2^b - 1 (section 量子化アルゴリズム, clamp bound of the Q equation)."""
    return (1 << bits) - 1


def codes_per_word(bits: int) -> int:
    """Codes packed into one uint32 word of the cache layout."""
    return 32 // bits


def fp16_round(x) -> np.ndarray:
    """Round float64 values to binary16, nearest with ties to even (numpy's direct conversion)."""
    return np.asarray(x, dtype=np.float64).astype(np.float16)


def scale_zero(lo, hi, bits: int):
    """s = (max X_g - min X_g)/(2^b - 1) stored as fp16, z = min X_g (section 量子化アルゴリズム,
    s/z equation).  lo, hi: fp16 group minima and maxima (arrays of equal shape)."""
    lo64 = np.asarray(lo, dtype=np.float16).astype(np.float64)
    hi64 = np.asarray(hi, dtype=np.float16).astype(np.float64)
    s = fp16_round((hi64 - lo64) / levels(bits))
    z = fp16_round(lo64 + 0.0)          # exact; a zero minimum is stored as +0
    return s, z


def quantize_values(x, s, z, bits: int) -> np.ndarray:
    """Q(X) = clamp(round((X - z)/s), 0, 2^b - 1) with round-half-to-even (section 量子化アルゴリズム,
    Q equation).  x, s, z are fp16 and broadcast together; s == 0 yields code 0."""
    x64 = np.asarray(x, dtype=np.float16).astype(np.float64)
    s64 = np.asarray(s, dtype=np.float16).astype(np.float64)
    z64 = np.asarray(z, dtype=np.float16).astype(np.float64)
    safe = np.where(s64 == 0.0, 1.0, s64)
    r = np.rint((x64 - z64) / safe)
    q = np.clip(r, 0, levels(bits))
    q = np.where(s64 == 0.0, 0.0, q)
    return q.astype(np.uint8)


def quantize_k_block(block, group_k: int, bits: int):
    """Per-channel K quantization of one R-token block (section Per-Channel量子化（Key Cache）,
    K_quant[:, j:j+g_k] = Q(K[:, j:j+g_k])): one (s, z) per g_k consecutive channels, taken over
    every token of the block.  block: fp16 [R][d].  Returns codes uint8 [R][d], s and z fp16
    [d/g_k]."""
    block = np.asarray(block, dtype=np.float16)
    n, d = block.shape
    ng = d // group_k
    lo = np.empty(ng, dtype=np.float16)
    hi = np.empty(ng, dtype=np.float16)
    for g in range(ng):
        cols = block[:, g * group_k:(g + 1) * group_k]
        lo[g] = cols.min()
        hi[g] = cols.max()
    s, z = scale_zero(lo, hi, bits)
    s_per_col = np.repeat(s, group_k)[None, :]
    z_per_col = np.repeat(z, group_k)[None, :]
    codes = quantize_values(block, s_per_col, z_per_col, bits)
    return codes, s, z


def quantize_v_block(block, group_v: int, bits: int):
    """Per-token V quantization (section Per-Token量子化（Value Cache）,
    V_quant[i:i+g_v, :] = Q(V[i:i+g_v, :])): one (s, z) per g_v consecutive tokens, taken over
    every channel.  block: fp16 [n][d] with n a multiple of g_v.  Returns codes uint8 [n][d],
    s and z fp16 [n/g_v]."""
    block = np.asarray(block, dtype=np.float16)
    n, d = block.shape
    ng = n // group_v
    lo = np.empty(ng, dtype=np.float16)
    hi = np.empty(ng, dtype=np.float16)
    for u in range(ng):
        rows = block[u * group_v:(u + 1) * group_v, :]
        lo[u] = rows.min()
        hi[u] = rows.max()
    s, z = scale_zero(lo, hi, bits)
    s_per_row = np.repeat(s, group_v)[:, None]
    z_per_row = np.repeat(z, group_v)[:, None]
    codes = quantize_values(block, s_per_row, z_per_row, bits)
    return codes, s, z


def quantize_k_block_fine(block, group_k: int, bits: int):
    """Fine-grained K groups (section KVキャッシュの分布特性: the range of each channel; section
    Per-Channel量子化 for Q): one (s, z) per channel per g_k consecutive tokens.  block: fp16 [n][d]
    with n a multiple of g_k.  Returns codes uint8 [n][d], s and z fp16 [n/g_k][d]."""
    block = np.asarray(block, dtype=np.float16)
    n, d = block.shape
    ng = n // group_k
    lo = np.empty((ng, d), dtype=np.float16)
    hi = np.empty((ng, d), dtype=np.float16)
    for u in range(ng):
        rows = block[u * group_k:(u + 1) * group_k, :]
        lo[u] = rows.min(axis=0)
        hi[u] = rows.max(axis=0)
    s, z = scale_zero(lo, hi, bits)
    codes = quantize_values(block, np.repeat(s, group_k, axis=0), np.repeat(z, group_k, axis=0), bits)
    return codes, s, z


def quantize_v_block_fine(block, group_v: int, bits: int):
    """Fine-grained V groups (section KVキャッシュの分布特性: the range of each token; section
    Per-Token量子化 for Q): one (s, z) per token per g_v consecutive channels.  block: fp16 [n][d].
    Returns codes uint8 [n][d], s and z fp16 [n][d/g_v]."""
    block = np.asarray(block, dtype=np.float16)
    n, d = block.shape
    ng = d // group_v
    lo = np.empty((n, ng), dtype=np.float16)
    hi = np.empty((n, ng), dtype=np.float16)
    for g in range(ng):
        cols = block[:, g * group_v:(g + 1) * group_v]
        lo[:, g] = cols.min(axis=1)
        hi[:, g] = cols.max(axis=1)
    s, z = scale_zero(lo, hi, bits)
    codes = quantize_values(block, np.repeat(s, group_v, axis=1), np.repeat(z, group_v, axis=1), bits)
    return codes, s, z


def pack_k(codes, bits: int) -> np.ndarray:
    """Token-major K packing of the cache layout: word i of token t holds the codes of channels
    P*i + j at bits [b*j, b*j+b), P = 32/b.  codes: uint8 [n][d] -> uint32 [n][d/P]."""
    codes = np.asarray(codes, dtype=np.uint64)
    n, d = codes.shape
    per = codes_per_word(bits)
    out = np.zeros((n, d // per), dtype=np.uint64)
    for j in range(per):
        out |= codes[:, j::per] << np.uint64(bits * j)
    return out.astype(np.uint32)


def pack_v(codes, bits: int) -> np.ndarray:
    """V packing of the cache layout: word (r, c) holds the codes of tokens P*r + j of channel c at
    bits [b*j, b*j+b).  codes: uint8 [n][d], n a multiple of P -> uint32 [n/P][d]."""
    codes = np.asarray(codes, dtype=np.uint64)
    n, d = codes.shape
    per = codes_per_word(bits)
    out = np.zeros((n // per, d), dtype=np.uint64)
    for j in range(per):
        out |= codes[j::per, :] << np.uint64(bits * j)
    return out.astype(np.uint32)


def unpack_k(words, bits: int) -> np.ndarray:
    """Inverse of pack_k: uint32 [n][d/P] -> uint8 [n][d]."""
    words = np.asarray(words, dtype=np.uint32)
    n, nw = words.shape
    per = codes_per_word(bits)
    mask = np.uint32(levels(bits))
    out = np.zeros((n, nw * per), dtype=np.uint8)
    for j in range(per):
        out[:, j::per] = (words >> np.uint32(bits * j)) & mask
    return out


def unpack_v(words, bits: int) -> np.ndarray:
    """Inverse of pack_v: uint32 [n/P][d] -> uint8 [n][d]."""
    words = np.asarray(words, dtype=np.uint32)
    nr, d = words.shape
    per = codes_per_word(bits)
    mask = np.uint32(levels(bits))
    out = np.zeros((nr * per, d), dtype=np.uint8)
    for j in range(per):
        out[j::per, :] = (words >> np.uint32(bits * j)) & mask
    return out


def dequantize_k(codes, s, z, block: int, group_k: int) -> np.ndarray:
    """D(K^) = s*K^ + z in float64 with the (block, channel group) scale of each element (section
    量子化アルゴリズム, D equation).  codes uint8 [n][d]; s, z fp16 [ceil(n/block)][d/group_k] (the
    last block may be partly filled)."""
    codes = np.asarray(codes, dtype=np.float64)
    n = codes.shape[0]
    s64 = np.asarray(s, dtype=np.float16).astype(np.float64)
    z64 = np.asarray(z, dtype=np.float16).astype(np.float64)
    s_full = np.repeat(np.repeat(s64, block, axis=0), group_k, axis=1)[:n]
    z_full = np.repeat(np.repeat(z64, block, axis=0), group_k, axis=1)[:n]
    return s_full * codes + z_full


def dequantize_v(codes, s, z, group_v: int) -> np.ndarray:
    """D(V^) = s*V^ + z in float64 with the token-group scale of each row (D equation).
    codes uint8 [n][d]; s, z fp16 [n/group_v]."""
    codes = np.asarray(codes, dtype=np.float64)
    s64 = np.repeat(np.asarray(s, dtype=np.float16).astype(np.float64), group_v)[:, None]
    z64 = np.repeat(np.asarray(z, dtype=np.float16).astype(np.float64), group_v)[:, None]
    return s64 * codes + z64


def dequantize_k_fine(codes, s, z, group_k: int) -> np.ndarray:
    """D(K^) = s*K^ + z in float64 with the (token group, channel) pair of each element (D equation).
    codes uint8 [n][d]; s, z fp16 [n/g_k][d]."""
    codes = np.asarray(codes, dtype=np.float64)
    s64 = np.repeat(np.asarray(s, dtype=np.float16).astype(np.float64), group_k, axis=0)
    z64 = np.repeat(np.asarray(z, dtype=np.float16).astype(np.float64), group_k, axis=0)
    return s64 * codes + z64


def dequantize_v_fine(codes, s, z, group_v: int) -> np.ndarray:
    """D(V^) = s*V^ + z in float64 with the (token, channel group) pair of each element (D equation).
    codes uint8 [n][d]; s, z fp16 [n][d/g_v]."""
    codes = np.asarray(codes, dtype=np.float64)
    s64 = np.repeat(np.asarray(s, dtype=np.float16).astype(np.float64), group_v, axis=1)
    z64 = np.repeat(np.asarray(z, dtype=np.float16).astype(np.float64), group_v, axis=1)
    return s64 * codes + z64


def attention(q, keys, values, scale: float) -> np.ndarray:
    """softmax(scale * q K^T) V for each query row, in float64 (section 残差バッファ, Attention
    equation).  q: [G][d]; keys, values: [T][d] float64 (dequantized then residual rows).
    Returns float64 [G][d]."""
    q64 = np.asarray(q, dtype=np.float16).astype(np.float64)
    logits = (q64 @ np.asarray(keys, dtype=np.float64).T) * float(scale)   # [G][T]
    logits = logits - logits.max(axis=1, keepdims=True)
    w = np.exp(logits)
    w = w / w.sum(axis=1, keepdims=True)
    return w @ np.asarray(values, dtype=np.float64)


class HeadCache:
    """Quantized cache of one (batch, KV head): quantized blocks plus the fp16 residual.

    Mirrors the library's counters: n_quant (a multiple of R) and n_res in [0, R].  With online_k,
    k_codes also holds the n_res online-coded rows after the n_quant block rows and k_s / k_z
    hold one row for the block being filled.  With fine_groups, g_k counts tokens and g_v channels
    (k_s / k_z [n_quant/g_k][d], v_s / v_z [n_quant][d/g_v])."""

    def __init__(self, head_dim: int, bits: int, group_k: int, group_v: int, residual: int,
                 capacity: int, online_k: bool = False, fine_groups: bool = False):
        self.d, self.bits, self.gk, self.gv = head_dim, bits, group_k, group_v
        self.R, self.capacity = residual, capacity
        self.online_k = bool(online_k)
        self.fine = bool(fine_groups)
        if self.fine and self.online_k:
            raise OracleError("UNSUPPORTED", "online K is not combined with fine-grained groups")
        self.k_codes = np.zeros((0, head_dim), np.uint8)
        self.v_codes = np.zeros((0, head_dim), np.uint8)
        self.k_s = np.zeros((0, head_dim if self.fine else head_dim // group_k), np.float16)
        self.k_z = np.zeros((0, head_dim if self.fine else head_dim // group_k), np.float16)
        self.v_s = np.zeros((0, head_dim // group_v) if self.fine else (0,), np.float16)
        self.v_z = np.zeros((0, head_dim // group_v) if self.fine else (0,), np.float16)
        self.k_res = np.zeros((0, head_dim), np.float16)
        self.v_res = np.zeros((0, head_dim), np.float16)

    @property
    def n_quant(self) -> int:
        return self.v_codes.shape[0]

    @property
    def n_res(self) -> int:
        return self.v_res.shape[0]

    @property
    def k_online(self) -> bool:
        """True when new K rows are coded at append time (online_k and a quantized block exists)."""
        return self.online_k and self.n_quant > 0

    def _code_online(self, rows):
        """Codes K rows with the (s, z) of the newest quantized block (section Per-Channel量子化:
        quantize a new token at once with the existing scale and zero point); the block being
        filled gets a copy of that (s, z) row when its first row arrives."""
        rows = np.asarray(rows, np.float16).reshape(-1, self.d)
        last = self.n_quant // self.R - 1
        s, z = self.k_s[last], self.k_z[last]
        if self.k_s.shape[0] == self.n_quant // self.R:
            self.k_s = np.concatenate([self.k_s, s[None, :]])
            self.k_z = np.concatenate([self.k_z, z[None, :]])
        codes = quantize_values(rows, np.repeat(s, self.gk)[None, :], np.repeat(z, self.gk)[None, :], self.bits)
        self.k_codes = np.concatenate([self.k_codes, codes])

    def _block_parts(self, kblk, vblk):
        """Codes, scales and zero points of one R-token block, rows ready to append."""
        if self.fine:
            kc, ks, kz = quantize_k_block_fine(kblk, self.gk, self.bits)
            vc, vs, vz = quantize_v_block_fine(vblk, self.gv, self.bits)
            return kc, vc, ks, kz, vs, vz
        kc, ks, kz = quantize_k_block(kblk, self.gk, self.bits)
        vc, vs, vz = quantize_v_block(vblk, self.gv, self.bits)
        return kc, vc, ks[None, :], kz[None, :], vs, vz

    def _append_blocks(self, parts):
        """Appends the blocks' rows to the quantized part (one concatenation per array)."""
        if not parts:
            return
        names = ("k_codes", "v_codes", "k_s", "k_z", "v_s", "v_z")
        for i, name in enumerate(names):
            setattr(self, name, np.concatenate([getattr(self, name)] + [p[i] for p in parts]))

    def _quantize_block(self, kblk, vblk):
        self._append_blocks([self._block_parts(kblk, vblk)])

    def prefill(self, k, v):
        """Resets the head and caches a prompt: the newest ((T-1) mod R)+1 tokens stay fp16, the
        older ones are quantized block by block (sections Per-Channel量子化, Per-Token量子化,
        残差バッファ)."""
        k = np.asarray(k, np.float16)
        v = np.asarray(v, np.float16)
        T = k.shape[0]
        if T < 1:
            raise OracleError("INVALID_ARG", "empty prompt")
        n_res = (T - 1) % self.R + 1
        n_quant = T - n_res
        if n_quant > self.capacity:
            raise OracleError("CAPACITY", f"{n_quant} > {self.capacity}")
        self.__init__(self.d, self.bits, self.gk, self.gv, self.R, self.capacity, self.online_k, self.fine)
        self._append_blocks([self._block_parts(k[j * self.R:(j + 1) * self.R], v[j * self.R:(j + 1) * self.R])
                             for j in range(n_quant // self.R)])
        self.v_res = v[n_quant:].copy()
        if self.k_online:
            if n_quant + self.R > self.capacity:
                raise OracleError("CAPACITY", "no block slot for the online K rows")
            self._code_online(k[n_quant:])
        else:
            self.k_res = k[n_quant:].copy()

    def prefill_prefix_k(self, k, v):
        """Prefill under the other reading of section Per-Channel量子化, in which one K group spans
        every quantized token of the prompt (the channel group over tokens [0, n_quant)) instead of
        one R-token block.  The residual split, the V groups (g_v consecutive tokens, section
        Per-Token量子化) and the counters are those of prefill.  The shared K (s, z) is kept once per
        R-token block, so dequantization and later flushes use the same layout as prefill."""
        if self.online_k or self.fine:
            raise OracleError("UNSUPPORTED", "prefix K groups are not combined with online K or fine groups")
        k = np.asarray(k, np.float16)
        v = np.asarray(v, np.float16)
        T = k.shape[0]
        if T < 1:
            raise OracleError("INVALID_ARG", "empty prompt")
        n_res = (T - 1) % self.R + 1
        n_quant = T - n_res
        if n_quant > self.capacity:
            raise OracleError("CAPACITY", f"{n_quant} > {self.capacity}")
        self.__init__(self.d, self.bits, self.gk, self.gv, self.R, self.capacity, self.online_k)
        if n_quant:
            kc, ks, kz = quantize_k_block(k[:n_quant], self.gk, self.bits)
            self.k_codes = kc
            self.k_s = np.tile(ks[None, :], (n_quant // self.R, 1))
            self.k_z = np.tile(kz[None, :], (n_quant // self.R, 1))
            for j in range(n_quant // self.R):
                vc, vs, vz = quantize_v_block(v[j * self.R:(j + 1) * self.R], self.gv, self.bits)
                self.v_codes = np.concatenate([self.v_codes, vc])
                self.v_s = np.concatenate([self.v_s, vs])
                self.v_z = np.concatenate([self.v_z, vz])
        self.k_res = k[n_quant:].copy()
        self.v_res = v[n_quant:].copy()

    def append(self, k_new, v_new):
        """Writes the newest token into the fp16 residual (section 残差バッファ); with online K its
        K row is coded at once instead (section Per-Channel量子化)."""
        if self.n_res == self.R:
            raise OracleError("RESIDUAL_FULL")
        if self.k_online:
            if self.n_quant + self.R > self.capacity:
                raise OracleError("CAPACITY", "no block slot for the online K row")
            self._code_online(k_new)
        else:
            self.k_res = np.concatenate([self.k_res, np.asarray(k_new, np.float16)[None, :]])
        self.v_res = np.concatenate([self.v_res, np.asarray(v_new, np.float16)[None, :]])

    def flush(self):
        """Quantizes a full residual as the next block (section Per-Token量子化: tokens are
        quantized together once a group has accumulated; section 残差バッファ)."""
        if self.n_res < self.R:
            raise OracleError("RESIDUAL_NOT_FULL")
        if self.n_quant + self.R > self.capacity:
            raise OracleError("CAPACITY")
        if self.k_online:  # K rows are coded already; the block keeps its copied (s, z)
            vc, vs, vz = quantize_v_block(self.v_res, self.gv, self.bits)
            self.v_codes = np.concatenate([self.v_codes, vc])
            self.v_s = np.concatenate([self.v_s, vs])
            self.v_z = np.concatenate([self.v_z, vz])
        else:
            self._quantize_block(self.k_res, self.v_res)
        self.k_res = np.zeros((0, self.d), np.float16)
        self.v_res = np.zeros((0, self.d), np.float16)

    def keys(self) -> np.ndarray:
        """[D(K_quant); K_res] as float64 [n_quant + n_res][d] (with online K every row is
        dequantized)."""
        if self.fine:
            kd = dequantize_k_fine(self.k_codes, self.k_s, self.k_z, self.gk)
        else:
            kd = dequantize_k(self.k_codes, self.k_s, self.k_z, self.R, self.gk)
        return np.concatenate([kd, self.k_res.astype(np.float64)])

    def values(self) -> np.ndarray:
        """[D(V_quant); V_res] as float64 [n_quant + n_res][d]."""
        if self.fine:
            vd = dequantize_v_fine(self.v_codes, self.v_s, self.v_z, self.gv)
        else:
            vd = dequantize_v(self.v_codes, self.v_s, self.v_z, self.gv)
        return np.concatenate([vd, self.v_res.astype(np.float64)])

    def attend(self, q, scale: float) -> np.ndarray:
        """Decode attention of the query rows q [G][d] over this head (Attention equation)."""
        if self.n_quant + self.n_res == 0:
            raise OracleError("EMPTY")
        return attention(q, self.keys(), self.values(), scale)

    def packed(self):
        """The head's filled cache in the library's device layout (tokens [0, n_quant))."""
        return {
            "k_codes": pack_k(self.k_codes, self.bits),
            "v_codes": pack_v(self.v_codes, self.bits),
            "k_scale": self.k_s, "k_zero": self.k_z, "v_scale": self.v_s, "v_zero": self.v_z,
            "k_res": self.k_res, "v_res": self.v_res,
        }


class OracleCache:
    """A [batch][kv head] grid of HeadCache objects with the library's calls.  ``heads`` limits the
    work to a subset of (b, h) pairs (the other heads stay empty)."""

    def __init__(self, batch: int, num_kv_heads: int, head_dim: int = 128, bits: int = 2,
                 group_k: int = 32, group_v: int = 32, residual: int = 128, capacity: int = 0,
                 heads=None, online_k: bool = False, fine_groups: bool = False):
        self.B, self.H = batch, num_kv_heads
        self.heads = sorted(heads) if heads is not None else [
            (b, h) for b in range(batch) for h in range(num_kv_heads)]
        self.cache = {bh: HeadCache(head_dim, bits, group_k, group_v, residual, capacity, online_k, fine_groups)
                      for bh in self.heads}

    def _counters(self):
        c = next(iter(self.cache.values()))
        return c.n_quant, c.n_res

    @property
    def n_quant(self) -> int:
        return self._counters()[0]

    @property
    def n_res(self) -> int:
        return self._counters()[1]

    def prefill(self, k_of, v_of):
        """k_of(b, h) / v_of(b, h) return the fp16 [T][d] prompt of one head."""
        for (b, h), c in self.cache.items():
            c.prefill(k_of(b, h), v_of(b, h))

    def append(self, k_new_of, v_new_of):
        if self.n_res == next(iter(self.cache.values())).R:
            raise OracleError("RESIDUAL_FULL")
        for (b, h), c in self.cache.items():
            c.append(k_new_of(b, h), v_new_of(b, h))

    def flush(self):
        for c in self.cache.values():
            c.flush()

    def attend(self, q_of, group: int, scale: float):
        """q_of(b, h) returns the fp16 [group][d] query rows of KV head h (query heads
        h*group .. h*group+group-1).  Returns {(b, h): float64 [group][d]}."""
        return {(b, h): c.attend(q_of(b, h), scale) for (b, h), c in self.cache.items()}
