"""ctypes binding of the CUDA library ``libkivi.so`` (C ABI in include/kivi.h).

Argument marshalling only: every computation runs in the library's kernels.  Functions keep the C
names.  PyTorch is used for device memory and streams: ``KiviCache`` allocates the caller-owned
cache buffers as torch tensors and passes their pointers.  The module raises ``KiviError`` if the
library is missing or a call fails; there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import math
import os

PKG = os.path.dirname(os.path.abspath(__file__))
# KIVI_LIB=debug selects the debug build (libkivi_debug.so: device-side bounds checks); any other
# value is taken as the path of the library to load.
LIB_PATH = {"": os.path.join(PKG, "libkivi.so"), "debug": os.path.join(PKG, "libkivi_debug.so")}.get(
    os.environ.get("KIVI_LIB", ""), os.environ.get("KIVI_LIB", ""))

KIVI_OK = 0
STATUS_NAMES = {
    0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "CAPACITY", 4: "RESIDUAL_FULL",
    5: "RESIDUAL_NOT_FULL", 6: "EMPTY", 7: "WORKSPACE", 8: "CUDA", 9: "DEVICE_TIMEOUT", 10: "STATE",
    11: "INTERNAL",
}
BUFFERS = ("k_codes", "v_codes", "k_scale", "k_zero", "v_scale", "v_zero", "k_res", "v_res")


class KiviError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        self.code = STATUS_NAMES.get(status, str(status))
        super().__init__(f"{where}: {self.code}")


class kivi_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("batch", "num_kv_heads", "head_dim", "bits", "group_k", "group_v", "residual", "capacity",
                 "online_k", "fine_groups")]


class kivi_cache(ctypes.Structure):
    _fields_ = [("k_codes", ctypes.c_void_p), ("v_codes", ctypes.c_void_p),
                ("k_scale", ctypes.c_void_p), ("k_zero", ctypes.c_void_p),
                ("v_scale", ctypes.c_void_p), ("v_zero", ctypes.c_void_p),
                ("k_res", ctypes.c_void_p), ("v_res", ctypes.c_void_p),
                ("n_quant", ctypes.c_int32), ("n_res", ctypes.c_int32)]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libkivi.so (once).  Raises KiviError-like RuntimeError when it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library not built: {path} (run python -m bit_asymmetric_kv_02_b200.build)")
    lib = ctypes.CDLL(path)
    P, I32, U64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint64, ctypes.c_size_t
    cfgp, cachep = ctypes.POINTER(kivi_config), ctypes.POINTER(kivi_cache)
    sig = {
        "kivi_abi_version": (I32, []),
        "kivi_strerror": (ctypes.c_char_p, [I32]),
        "kivi_check_config": (I32, [cfgp]),
        "kivi_cache_sizes": (I32, [cfgp, ctypes.POINTER(SZ)]),
        "kivi_quantize_prefill": (I32, [cfgp, cachep, P, P, I32, P]),
        "kivi_quantize_prefill_prefix_k": (I32, [cfgp, cachep, P, P, I32, P]),
        "kivi_append_token": (I32, [cfgp, cachep, P, P, P]),
        "kivi_flush_residual": (I32, [cfgp, cachep, P]),
        "kivi_decode_workspace_bytes": (SZ, [cfgp, I32]),
        "kivi_decode_attention": (I32, [cfgp, cachep, P, I32, ctypes.c_float, P, P, SZ, P, P]),
        "kivi_append_decode_attention": (I32, [cfgp, cachep, P, P, P, I32, ctypes.c_float, P, P, SZ, P, P]),
        "kivi_decode_step": (I32, [cfgp, cachep, P, P, P, I32, ctypes.c_float, P, P, SZ, P, P]),
        "kivi_decode_attention_noalloc": (I32, [cfgp, cachep, P, I32, ctypes.c_float, P, P, P]),
        "kivi_read_status": (I32, [P, P]),
        "kivi_debug_inject": (I32, [I32, U64]),
        "kivi_debug_status": (I32, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    _lib = lib
    return lib


def _check(status: int, where: str) -> None:
    if status != KIVI_OK:
        raise KiviError(status, where)


# ---- C-ABI functions, same names ------------------------------------------------------------
def kivi_abi_version() -> int:
    return load_library().kivi_abi_version()


def kivi_strerror(status: int) -> str:
    return load_library().kivi_strerror(status).decode()


def kivi_check_config(cfg: kivi_config) -> int:
    return load_library().kivi_check_config(ctypes.byref(cfg))


def kivi_cache_sizes(cfg: kivi_config) -> list[int]:
    out = (ctypes.c_size_t * len(BUFFERS))()
    _check(load_library().kivi_cache_sizes(ctypes.byref(cfg), out), "kivi_cache_sizes")
    return list(out)


def kivi_quantize_prefill(cfg, cache, k_ptr: int, v_ptr: int, num_tokens: int, stream: int) -> None:
    _check(load_library().kivi_quantize_prefill(ctypes.byref(cfg), ctypes.byref(cache), k_ptr, v_ptr,
                                                num_tokens, stream), "kivi_quantize_prefill")


def kivi_quantize_prefill_prefix_k(cfg, cache, k_ptr: int, v_ptr: int, num_tokens: int, stream: int) -> None:
    _check(load_library().kivi_quantize_prefill_prefix_k(ctypes.byref(cfg), ctypes.byref(cache), k_ptr, v_ptr,
                                                         num_tokens, stream), "kivi_quantize_prefill_prefix_k")


def kivi_append_token(cfg, cache, k_new_ptr: int, v_new_ptr: int, stream: int) -> None:
    _check(load_library().kivi_append_token(ctypes.byref(cfg), ctypes.byref(cache), k_new_ptr, v_new_ptr,
                                            stream), "kivi_append_token")


def kivi_flush_residual(cfg, cache, stream: int) -> None:
    _check(load_library().kivi_flush_residual(ctypes.byref(cfg), ctypes.byref(cache), stream),
           "kivi_flush_residual")


def kivi_decode_workspace_bytes(cfg, num_q_heads: int) -> int:
    return load_library().kivi_decode_workspace_bytes(ctypes.byref(cfg), num_q_heads)


def kivi_decode_attention(cfg, cache, q_ptr: int, num_q_heads: int, scale: float, out_ptr: int,
                          ws_ptr: int, ws_bytes: int, status_ptr: int | None, stream: int) -> None:
    _check(load_library().kivi_decode_attention(ctypes.byref(cfg), ctypes.byref(cache), q_ptr, num_q_heads,
                                                scale, out_ptr, ws_ptr, ws_bytes, status_ptr, stream),
           "kivi_decode_attention")


def kivi_append_decode_attention(cfg, cache, k_new_ptr: int, v_new_ptr: int, q_ptr: int, num_q_heads: int,
                                 scale: float, out_ptr: int, ws_ptr: int, ws_bytes: int, status_ptr: int | None,
                                 stream: int) -> None:
    _check(load_library().kivi_append_decode_attention(ctypes.byref(cfg), ctypes.byref(cache), k_new_ptr, v_new_ptr,
                                                       q_ptr, num_q_heads, scale, out_ptr, ws_ptr, ws_bytes,
                                                       status_ptr, stream),
           "kivi_append_decode_attention")


def kivi_decode_step(cfg, cache, k_new_ptr: int, v_new_ptr: int, q_ptr: int, num_q_heads: int, scale: float,
                     out_ptr: int, ws_ptr: int, ws_bytes: int, status_ptr: int | None, stream: int) -> None:
    _check(load_library().kivi_decode_step(ctypes.byref(cfg), ctypes.byref(cache), k_new_ptr, v_new_ptr, q_ptr,
                                           num_q_heads, scale, out_ptr, ws_ptr, ws_bytes, status_ptr, stream),
           "kivi_decode_step")


def kivi_decode_attention_noalloc(cfg, cache, q_ptr: int, num_q_heads: int, scale: float, out_ptr: int,
                                  status_ptr: int | None, stream: int) -> None:
    """Decode attention with the library's fixed scratch array instead of a caller workspace, for
    callers that cannot allocate device memory at decode time (see include/kivi.h)."""
    _check(load_library().kivi_decode_attention_noalloc(ctypes.byref(cfg), ctypes.byref(cache), q_ptr, num_q_heads,
                                                        scale, out_ptr, status_ptr, stream),
           "kivi_decode_attention_noalloc")


def kivi_read_status(status_ptr: int, stream: int) -> int:
    return load_library().kivi_read_status(status_ptr, stream)


def kivi_debug_inject(mode: int, value: int = 0) -> None:
    _check(load_library().kivi_debug_inject(mode, value), "kivi_debug_inject")


def kivi_debug_status() -> int:
    """The first device-side check failure of the debug build since the last call (0: none)."""
    return load_library().kivi_debug_status()


# ---- torch-owned cache --------------------------------------------------------------------------
class KiviCache:
    """Caller-owned device buffers of one cache, allocated as torch tensors, plus the C struct.

    The arguments are the fields of kivi_config (include/kivi.h).  online_k: K rows are coded at
    append with the newest block's (s, z) once a block exists.  fine_groups: group_k counts tokens
    (one K pair per channel per group_k tokens) and group_v channels (one V pair per token per group_v
    channels).  num_q_heads sizes the decode workspace (default: one query head per KV head)."""

    def __init__(self, batch: int, num_kv_heads: int, capacity: int, bits: int = 2, group_k: int = 32,
                 group_v: int = 32, residual: int = 128, head_dim: int = 128, num_q_heads: int | None = None,
                 device=None, online_k: bool = False, fine_groups: bool = False):
        import torch
        self.torch = torch
        self.device = torch.device(device or "cuda")
        self.cfg = kivi_config(batch, num_kv_heads, head_dim, bits, group_k, group_v, residual, capacity,
                               1 if online_k else 0, 1 if fine_groups else 0)
        st = kivi_check_config(self.cfg)
        if st != KIVI_OK:
            raise KiviError(st, "kivi_check_config")
        sizes = kivi_cache_sizes(self.cfg)
        self.buffers = {}
        for name, nbytes in zip(BUFFERS, sizes):
            # uint8 storage padded to 16 bytes so an empty buffer still has an aligned pointer
            self.buffers[name] = torch.empty(max(16, nbytes), dtype=torch.uint8, device=self.device)
        self.c = kivi_cache(*[self.buffers[n].data_ptr() for n in BUFFERS], 0, 0)
        self.num_q_heads = num_q_heads or num_kv_heads
        self.ws_bytes = kivi_decode_workspace_bytes(self.cfg, self.num_q_heads)
        if self.ws_bytes == 0:
            raise KiviError(1, "kivi_decode_workspace_bytes")
        self.workspace = torch.zeros(self.ws_bytes + 256, dtype=torch.uint8, device=self.device)
        off = (-self.workspace.data_ptr()) % 256
        self.ws_ptr = self.workspace.data_ptr() + off
        self.status = torch.zeros(4, dtype=torch.int32, device=self.device)

    # views of the buffers in the layout of include/kivi.h
    def view(self, name: str):
        t = self.torch
        c = self.cfg
        B, H, C, d, R = c.batch, c.num_kv_heads, c.capacity, c.head_dim, c.residual
        P = 32 // c.bits
        shapes = {
            "k_codes": (t.int32, (B, H, C, d // P)), "v_codes": (t.int32, (B, H, C // P, d)),
            "k_scale": (t.float16, (B, H, C // R, d // c.group_k)), "k_zero": (t.float16, (B, H, C // R, d // c.group_k)),
            "v_scale": (t.float16, (B, H, C // c.group_v)), "v_zero": (t.float16, (B, H, C // c.group_v)),
            "k_res": (t.float16, (B, H, R, d)), "v_res": (t.float16, (B, H, R, d)),
        }
        if c.fine_groups:   # K: per channel per group_k tokens; V: per token per group_v channels
            for n_, sh in (("k_scale", (B, H, C // c.group_k, d)), ("k_zero", (B, H, C // c.group_k, d)),
                           ("v_scale", (B, H, C, d // c.group_v)), ("v_zero", (B, H, C, d // c.group_v))):
                shapes[n_] = (t.float16, sh)
        dtype, shape = shapes[name]
        n = math.prod(shape) * (4 if dtype == t.int32 else 2)
        return self.buffers[name][:n].view(dtype).view(shape)

    @property
    def n_quant(self) -> int:
        return self.c.n_quant

    @property
    def n_res(self) -> int:
        return self.c.n_res

    def _stream(self, stream) -> int:
        s = stream if stream is not None else self.torch.cuda.current_stream(self.device)
        return s.cuda_stream

    def prefill(self, k, v, stream=None) -> None:
        """k, v: contiguous fp16 device tensors [B][H][T][d]."""
        assert k.dtype == self.torch.float16 and k.is_contiguous() and v.is_contiguous()
        kivi_quantize_prefill(self.cfg, self.c, k.data_ptr(), v.data_ptr(), k.shape[2], self._stream(stream))

    def prefill_prefix_k(self, k, v, stream=None) -> None:
        """prefill with one K group over the whole quantized prefix (kivi_quantize_prefill_prefix_k)."""
        assert k.dtype == self.torch.float16 and k.is_contiguous() and v.is_contiguous()
        kivi_quantize_prefill_prefix_k(self.cfg, self.c, k.data_ptr(), v.data_ptr(), k.shape[2], self._stream(stream))

    def append(self, k_new, v_new, stream=None) -> None:
        """k_new, v_new: contiguous fp16 device tensors [B][H][d]."""
        kivi_append_token(self.cfg, self.c, k_new.data_ptr(), v_new.data_ptr(), self._stream(stream))

    def flush(self, stream=None) -> None:
        kivi_flush_residual(self.cfg, self.c, self._stream(stream))

    def attend(self, q, out=None, scale: float | None = None, stream=None, status: bool = True):
        """q: contiguous fp16 device tensor [B][Hq][d]; returns out (fp16, same shape)."""
        if out is None:
            out = self.torch.empty_like(q)
        scale = 1.0 / math.sqrt(self.cfg.head_dim) if scale is None else scale
        kivi_decode_attention(self.cfg, self.c, q.data_ptr(), q.shape[1], scale, out.data_ptr(), self.ws_ptr,
                              self.ws_bytes, self.status.data_ptr() if status else None, self._stream(stream))
        return out

    def append_attend(self, k_new, v_new, q, out=None, scale: float | None = None, stream=None,
                      status: bool = True):
        """append(k_new, v_new) then attend(q), in one kernel launch."""
        if out is None:
            out = self.torch.empty_like(q)
        scale = 1.0 / math.sqrt(self.cfg.head_dim) if scale is None else scale
        kivi_append_decode_attention(self.cfg, self.c, k_new.data_ptr(), v_new.data_ptr(), q.data_ptr(), q.shape[1],
                                     scale, out.data_ptr(), self.ws_ptr, self.ws_bytes,
                                     self.status.data_ptr() if status else None, self._stream(stream))
        return out

    def step(self, k_new, v_new, q, out=None, scale: float | None = None, stream=None, status: bool = True):
        """One streaming decode step: append(k_new, v_new), attend(q), and quantize the residual in
        the same launch when this token fills it (kivi_decode_step)."""
        if out is None:
            out = self.torch.empty_like(q)
        scale = 1.0 / math.sqrt(self.cfg.head_dim) if scale is None else scale
        kivi_decode_step(self.cfg, self.c, k_new.data_ptr(), v_new.data_ptr(), q.data_ptr(), q.shape[1], scale,
                         out.data_ptr(), self.ws_ptr, self.ws_bytes, self.status.data_ptr() if status else None,
                         self._stream(stream))
        return out

    def read_status(self, stream=None) -> int:
        return kivi_read_status(self.status.data_ptr(), self._stream(stream))
