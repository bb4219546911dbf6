"""Thin Python binding of libtq's C ABI (include/tq.h): argument marshalling only.

Every computation runs in libtq (CUDA kernels for sm_100a, plus host-side table builders).
PyTorch supplies device memory and the current CUDA stream; nothing here computes on the
data. Importing this module loads libtq.so and raises if it is missing: there is no
fallback path.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np
import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtq.so")

TQ_OK, TQ_ERR_INVALID_ARG, TQ_ERR_UNSUPPORTED, TQ_ERR_WORKSPACE, TQ_ERR_CUDA = 0, 1, 2, 3, 4
TQ_MSE, TQ_PROD, TQ_E2M1 = 0, 1, 2
TQ_F32, TQ_BF16, TQ_F16 = 0, 1, 2

_DTYPES = {torch.float32: TQ_F32, torch.bfloat16: TQ_BF16, torch.float16: TQ_F16}


class TQError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"libtq status {status}: {msg}")
        self.status = status


class tq_qcfg(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int), ("mode", ctypes.c_int), ("qjl_m", ctypes.c_int)]


class tq_cache(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("Hkv", ctypes.c_int), ("T_cap", ctypes.c_int), ("d", ctypes.c_int),
        ("seed", ctypes.c_uint64), ("kc", tq_qcfg), ("vc", tq_qcfg),
        ("k_codes", ctypes.c_void_p), ("v_codes", ctypes.c_void_p),
        ("k_norm", ctypes.c_void_p), ("v_norm", ctypes.c_void_p),
        ("k_signs", ctypes.c_void_p), ("v_signs", ctypes.c_void_p),
        ("k_rnorm", ctypes.c_void_p), ("v_rnorm", ctypes.c_void_p),
        ("k_qjl", ctypes.c_void_p), ("v_qjl", ctypes.c_void_p),
    ]


class tq_paged_cache(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("Hkv", ctypes.c_int), ("d", ctypes.c_int), ("page_size", ctypes.c_int),
        ("num_pages", ctypes.c_int), ("max_pages", ctypes.c_int),
        ("seed", ctypes.c_uint64), ("kc", tq_qcfg), ("vc", tq_qcfg),
        ("k_codes", ctypes.c_void_p), ("v_codes", ctypes.c_void_p),
        ("k_norm", ctypes.c_void_p), ("v_norm", ctypes.c_void_p),
        ("block_table", ctypes.c_void_p),
        ("k_signs", ctypes.c_void_p), ("v_signs", ctypes.c_void_p),
        ("k_rnorm", ctypes.c_void_p), ("v_rnorm", ctypes.c_void_p),
        ("k_qjl", ctypes.c_void_p), ("v_qjl", ctypes.c_void_p),
    ]


EXPORTS = {
    # name: (restype, argtypes)
    "tq_last_error": (ctypes.c_char_p, []),
    "tq_make_codebook": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]),
    "tq_make_signs": (ctypes.c_int, [ctypes.c_uint64, ctypes.c_int, ctypes.c_void_p]),
    "tq_make_qjl_matrix": (ctypes.c_int, [ctypes.c_uint64, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]),
    "tq_code_bytes": (ctypes.c_size_t, [ctypes.c_int, tq_qcfg]),
    "tq_sign_bytes": (ctypes.c_size_t, [ctypes.c_int, tq_qcfg]),
    "tq_record_bytes": (ctypes.c_size_t, [ctypes.c_int, tq_qcfg]),
    "tq_quantize_kv": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_int, ctypes.POINTER(tq_cache), ctypes.c_void_p]),
    "tq_device_faults": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint)]),
    "tq_launch_counts": (ctypes.c_int, [ctypes.POINTER(tq_cache), ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]),
    "tq_decode_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                    ctypes.POINTER(tq_cache)]),
    "tq_decode_attention": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_float, ctypes.POINTER(tq_cache), ctypes.c_void_p,
                                           ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "tq_decode_varlen_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int, ctypes.POINTER(tq_cache),
                                                           ctypes.c_void_p]),
    "tq_decode_attention_varlen": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                                  ctypes.c_void_p, ctypes.c_float, ctypes.POINTER(tq_cache),
                                                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                                  ctypes.c_void_p]),
    "tq_quantize_kv_paged": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int, ctypes.POINTER(tq_paged_cache), ctypes.c_void_p]),
    "tq_decode_paged_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int, ctypes.POINTER(tq_paged_cache),
                                                          ctypes.c_void_p]),
    "tq_decode_attention_paged": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                                 ctypes.c_float, ctypes.POINTER(tq_paged_cache),
                                                 ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                                 ctypes.c_void_p]),
    "tq_decode_attention_noalloc": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                                   ctypes.c_int, ctypes.c_float, ctypes.POINTER(tq_cache),
                                                   ctypes.c_void_p, ctypes.c_void_p]),
    "tq_prefill_attention": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int, ctypes.c_float, ctypes.POINTER(tq_cache),
                                            ctypes.c_void_p, ctypes.c_void_p]),
    "tq_dequantize": (ctypes.c_int, [ctypes.POINTER(tq_cache), ctypes.c_int, ctypes.c_int,
                                     ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]),
    "tq_decode_bf16_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                         ctypes.c_int, ctypes.c_int]),
    "tq_decode_attention_bf16": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                                                ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p,
                                                ctypes.c_size_t, ctypes.c_void_p]),
}


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m quantized_decode_attention_kv_b200.build` "
            "(libtq has no fallback implementation)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in EXPORTS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def last_error() -> str:
    return lib.tq_last_error().decode()


def _check(status: int) -> None:
    if status != TQ_OK:
        raise TQError(status, last_error())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dev(t: torch.Tensor, name: str) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda or not t.is_contiguous():
        raise TQError(TQ_ERR_INVALID_ARG, f"{name} must be a contiguous CUDA tensor")
    return t.data_ptr()


# ------------------------------------------------------------------ host-side helpers
def tq_make_codebook(bits: int, d: int) -> tuple[np.ndarray, np.ndarray]:
    c = np.zeros(1 << bits, dtype=np.float32)
    b = np.zeros(max((1 << bits) - 1, 1), dtype=np.float32)
    _check(lib.tq_make_codebook(bits, d, c.ctypes.data, b.ctypes.data))
    return c, b[: (1 << bits) - 1]


def tq_make_signs(seed: int, d: int) -> np.ndarray:
    out = np.zeros(d // 8, dtype=np.uint8)
    _check(lib.tq_make_signs(seed, d, out.ctypes.data))
    return out


def tq_make_qjl_matrix(seed: int, m: int, d: int) -> np.ndarray:
    out = np.zeros((m, d), dtype=np.float32)
    _check(lib.tq_make_qjl_matrix(seed, m, d, out.ctypes.data))
    return out


def tq_code_bytes(d: int, bits: int, mode: int = TQ_MSE, qjl_m: int = 0) -> int:
    return int(lib.tq_code_bytes(d, tq_qcfg(bits, mode, qjl_m)))


def tq_sign_bytes(d: int, bits: int, mode: int = TQ_MSE, qjl_m: int = 0) -> int:
    return int(lib.tq_sign_bytes(d, tq_qcfg(bits, mode, qjl_m)))


def tq_record_bytes(d: int, bits: int, mode: int = TQ_MSE, qjl_m: int = 0) -> int:
    return int(lib.tq_record_bytes(d, tq_qcfg(bits, mode, qjl_m)))


# ------------------------------------------------------------------ device buffers
@dataclass
class TQCache:
    """One layer's compressed KV cache: torch owns the device buffers, ``struct`` is the
    tq_cache the C ABI reads. Shapes follow include/tq.h."""
    B: int
    Hkv: int
    T_cap: int
    d: int
    k_bits: int
    v_bits: int
    k_mode: int = TQ_MSE
    v_mode: int = TQ_MSE
    k_qjl_m: int = 0
    v_qjl_m: int = 0
    seed: int = 0
    qjl_seed: int = 1
    device: str = "cuda"

    def __post_init__(self):
        dev = torch.device(self.device)
        self.tensors = {}
        for side, bits, mode, m in (("k", self.k_bits, self.k_mode, self.k_qjl_m),
                                    ("v", self.v_bits, self.v_mode, self.v_qjl_m)):
            cb = tq_code_bytes(self.d, bits, mode, m)
            sb = tq_sign_bytes(self.d, bits, mode, m)
            shape = (self.B, self.Hkv, self.T_cap)
            self.tensors[f"{side}_codes"] = torch.zeros(shape + (max(cb, 1),), dtype=torch.uint8, device=dev) if cb else None
            self.tensors[f"{side}_norm"] = torch.zeros(shape, dtype=torch.int16, device=dev)
            if mode == TQ_PROD:
                mm = m or self.d
                self.tensors[f"{side}_signs"] = torch.zeros(shape + (sb,), dtype=torch.uint8, device=dev)
                self.tensors[f"{side}_rnorm"] = torch.zeros(shape, dtype=torch.int16, device=dev)
                self.tensors[f"{side}_qjl"] = torch.from_numpy(
                    tq_make_qjl_matrix(self.qjl_seed, mm, self.d)).to(dev)
            else:
                self.tensors[f"{side}_signs"] = None
                self.tensors[f"{side}_rnorm"] = None
                self.tensors[f"{side}_qjl"] = None
        ptr = lambda t: t.data_ptr() if t is not None else None  # noqa: E731
        self.struct = tq_cache(
            self.B, self.Hkv, self.T_cap, self.d, self.seed,
            tq_qcfg(self.k_bits, self.k_mode, self.k_qjl_m), tq_qcfg(self.v_bits, self.v_mode, self.v_qjl_m),
            ptr(self.tensors["k_codes"]), ptr(self.tensors["v_codes"]),
            ptr(self.tensors["k_norm"]), ptr(self.tensors["v_norm"]),
            ptr(self.tensors["k_signs"]), ptr(self.tensors["v_signs"]),
            ptr(self.tensors["k_rnorm"]), ptr(self.tensors["v_rnorm"]),
            ptr(self.tensors["k_qjl"]), ptr(self.tensors["v_qjl"]))

    def __getitem__(self, key):
        return self.tensors[key]

    def packed_bytes(self, T_len: int) -> int:
        """Stored bytes of positions [0, T_len) for every (b, KV head): codes, signs, norms."""
        per = (tq_record_bytes(self.d, self.k_bits, self.k_mode, self.k_qjl_m)
               + tq_record_bytes(self.d, self.v_bits, self.v_mode, self.v_qjl_m))
        return self.B * self.Hkv * T_len * per


class TQPagedCache:
    """One layer's paged compressed KV cache (head_dim-128 TurboQuant_mse or head_dim-64
    TurboQuant_prod records): torch owns the page pools; ``block_table`` is an int32
    [B][max_pages] device tensor the caller fills with physical page indices (it may be
    rewritten between calls). Shapes follow include/tq.h."""

    def __init__(self, B: int, Hkv: int, d: int, page_size: int, num_pages: int, max_pages: int,
                 k_bits: int, v_bits: int, block_table: torch.Tensor, seed: int = 0, device: str = "cuda",
                 k_mode: int = TQ_MSE, v_mode: int = TQ_MSE, k_qjl_m: int = 0, v_qjl_m: int = 0,
                 qjl_seed: int = 1):
        dev = torch.device(device)
        self.B, self.Hkv, self.d, self.page_size = B, Hkv, d, page_size
        self.num_pages, self.max_pages, self.k_bits, self.v_bits, self.seed = num_pages, max_pages, k_bits, v_bits, seed
        self.k_mode, self.v_mode, self.k_qjl_m, self.v_qjl_m, self.qjl_seed = k_mode, v_mode, k_qjl_m, v_qjl_m, qjl_seed
        if block_table.dtype != torch.int32 or tuple(block_table.shape) != (B, max_pages) or not block_table.is_cuda:
            raise TQError(TQ_ERR_INVALID_ARG, "block_table must be an int32 CUDA tensor [B][max_pages]")
        self.block_table = block_table.contiguous()
        self.tensors = {}
        for side, bits, mode, m in (("k", k_bits, k_mode, k_qjl_m), ("v", v_bits, v_mode, v_qjl_m)):
            cb = tq_code_bytes(d, bits, mode, m)
            shape = (num_pages, Hkv, page_size)
            self.tensors[f"{side}_codes"] = torch.zeros(shape + (max(cb, 1),), dtype=torch.uint8, device=dev) if cb else None
            self.tensors[f"{side}_norm"] = torch.zeros(shape, dtype=torch.int16, device=dev)
            if mode == TQ_PROD:
                self.tensors[f"{side}_signs"] = torch.zeros(shape + (tq_sign_bytes(d, bits, mode, m),),
                                                            dtype=torch.uint8, device=dev)
                self.tensors[f"{side}_rnorm"] = torch.zeros(shape, dtype=torch.int16, device=dev)
                self.tensors[f"{side}_qjl"] = torch.from_numpy(tq_make_qjl_matrix(qjl_seed, m or d, d)).to(dev)
            else:
                for key in ("signs", "rnorm", "qjl"):
                    self.tensors[f"{side}_{key}"] = None
        t = self.tensors
        ptr = lambda x: x.data_ptr() if x is not None else None  # noqa: E731
        self.struct = tq_paged_cache(B, Hkv, d, page_size, num_pages, max_pages, seed,
                                     tq_qcfg(k_bits, k_mode, k_qjl_m), tq_qcfg(v_bits, v_mode, v_qjl_m),
                                     ptr(t["k_codes"]), ptr(t["v_codes"]), ptr(t["k_norm"]), ptr(t["v_norm"]),
                                     self.block_table.data_ptr(),
                                     ptr(t["k_signs"]), ptr(t["v_signs"]), ptr(t["k_rnorm"]), ptr(t["v_rnorm"]),
                                     ptr(t["k_qjl"]), ptr(t["v_qjl"]))

    def __getitem__(self, key):
        return self.tensors[key]


# ------------------------------------------------------------------ device entry points
def tq_quantize_kv(K: torch.Tensor | None, V: torch.Tensor | None, cache: TQCache, t_offset: int = 0,
                   stream=None) -> None:
    ref = K if K is not None else V
    if ref is None:
        raise TQError(TQ_ERR_INVALID_ARG, "K and V are both None")
    T = ref.shape[2]
    dt = _DTYPES.get(ref.dtype)
    if dt is None:
        raise TQError(TQ_ERR_INVALID_ARG, f"unsupported dtype {ref.dtype}")
    kp = _dev(K, "K") if K is not None else None
    vp = _dev(V, "V") if V is not None else None
    _check(lib.tq_quantize_kv(kp, vp, dt, T, t_offset, ctypes.byref(cache.struct), _stream(stream)))


def tq_quantize_kv_paged(K: torch.Tensor | None, V: torch.Tensor | None, cache: TQPagedCache,
                         t_offset: int = 0, stream=None) -> None:
    """Write positions t_offset .. t_offset + T - 1 of every sequence into the paged cache."""
    ref = K if K is not None else V
    if ref is None:
        raise TQError(TQ_ERR_INVALID_ARG, "K and V are both None")
    dt = _DTYPES.get(ref.dtype)
    if dt is None:
        raise TQError(TQ_ERR_INVALID_ARG, f"unsupported dtype {ref.dtype}")
    kp = _dev(K, "K") if K is not None else None
    vp = _dev(V, "V") if V is not None else None
    _check(lib.tq_quantize_kv_paged(kp, vp, dt, ref.shape[2], t_offset, ctypes.byref(cache.struct),
                                    _stream(stream)))


def tq_decode_paged_workspace_bytes(cache: TQPagedCache, Hq: int, T_lens) -> int:
    lens = _lens(T_lens)
    n = int(lib.tq_decode_paged_workspace_bytes(Hq, ctypes.byref(cache.struct), ctypes.cast(lens, ctypes.c_void_p)))
    if n == 0:
        raise TQError(TQ_ERR_INVALID_ARG, last_error())
    return n


def tq_decode_attention_paged(q: torch.Tensor, cache: TQPagedCache, T_lens, scale: float, out: torch.Tensor,
                              ws: torch.Tensor, stream=None) -> None:
    """Decode attention over a paged cache; sequence b attends to its first T_lens[b] positions."""
    dt = _DTYPES.get(q.dtype)
    if dt is None:
        raise TQError(TQ_ERR_INVALID_ARG, f"unsupported dtype {q.dtype}")
    lens = _lens(T_lens)
    _check(lib.tq_decode_attention_paged(_dev(q, "q"), dt, q.shape[1], ctypes.cast(lens, ctypes.c_void_p),
                                         scale, ctypes.byref(cache.struct), _dev(out, "out"), _dev(ws, "ws"),
                                         ws.numel() * ws.element_size(), _stream(stream)))


def tq_launch_counts(cache: TQCache, dtype: torch.dtype, T: int, Hq: int, T_len: int) -> tuple[int, int]:
    """(kernels one tq_quantize_kv of T positions launches, kernels one tq_decode_attention
    over T_len positions launches) for this cache on the current device."""
    dt = _DTYPES.get(dtype)
    if dt is None:
        raise TQError(TQ_ERR_INVALID_ARG, f"unsupported dtype {dtype}")
    nq, nd = ctypes.c_int(0), ctypes.c_int(0)
    _check(lib.tq_launch_counts(ctypes.byref(cache.struct), dt, T, Hq, T_len, ctypes.byref(nq),
                                ctypes.byref(nd)))
    return nq.value, nd.value


def tq_device_faults() -> int:
    """Device-side fault bits recorded since the last call (bit 0: a tensor-core write kernel
    timed out waiting for its MMAs); synchronises the device and clears them."""
    v = ctypes.c_uint(0)
    _check(lib.tq_device_faults(ctypes.byref(v)))
    return v.value


def tq_decode_workspace_bytes(cache: TQCache, Hq: int, T_len: int) -> int:
    n = int(lib.tq_decode_workspace_bytes(cache.B, Hq, T_len, ctypes.byref(cache.struct)))
    if n == 0:
        raise TQError(TQ_ERR_INVALID_ARG, last_error())
    return n


def tq_decode_attention(q: torch.Tensor, cache: TQCache, T_len: int, scale: float, out: torch.Tensor,
                        ws: torch.Tensor, stream=None) -> None:
    dt = _DTYPES.get(q.dtype)
    if dt is None:
        raise TQError(TQ_ERR_INVALID_ARG, f"unsupported dtype {q.dtype}")
    _check(lib.tq_decode_attention(_dev(q, "q"), dt, q.shape[1], T_len, scale, ctypes.byref(cache.struct),
                                   _dev(out, "out"), _dev(ws, "ws"), ws.numel() * ws.element_size(),
                                   _stream(stream)))


def _lens(T_lens) -> ctypes.Array:
    vals = [int(t) for t in T_lens]
    return (ctypes.c_int * len(vals))(*vals)


def tq_decode_varlen_workspace_bytes(cache: TQCache, Hq: int, T_lens) -> int:
    """Workspace bytes of a ragged decode call (T_lens: B per-sequence context lengths)."""
    lens = _lens(T_lens)
    n = int(lib.tq_decode_varlen_workspace_bytes(Hq, ctypes.byref(cache.struct), ctypes.cast(lens, ctypes.c_void_p)))
    if n == 0:
        raise TQError(TQ_ERR_INVALID_ARG, last_error())
    return n


def tq_decode_attention_varlen(q: torch.Tensor, cache: TQCache, T_lens, scale: float, out: torch.Tensor,
                               ws: torch.Tensor, stream=None) -> None:
    """Decode attention where sequence b attends to its first T_lens[b] cached positions."""
    dt = _DTYPES.get(q.dtype)
    if dt is None:
        raise TQError(TQ_ERR_INVALID_ARG, f"unsupported dtype {q.dtype}")
    lens = _lens(T_lens)
    _check(lib.tq_decode_attention_varlen(_dev(q, "q"), dt, q.shape[1], ctypes.cast(lens, ctypes.c_void_p),
                                          scale, ctypes.byref(cache.struct), _dev(out, "out"), _dev(ws, "ws"),
                                          ws.numel() * ws.element_size(), _stream(stream)))


def tq_decode_attention_noalloc(q: torch.Tensor, cache: TQCache, T_len: int, scale: float,
                                out: torch.Tensor, stream=None) -> None:
    """tq_decode_attention without a workspace: libtq keeps the split-K partials in its own
    fixed device scratch (8 MiB), so nothing is allocated. For callers that may not allocate
    device memory; calls that overlap on the GPU must be serialised by the caller."""
    dt = _DTYPES.get(q.dtype)
    if dt is None:
        raise TQError(TQ_ERR_INVALID_ARG, f"unsupported dtype {q.dtype}")
    _check(lib.tq_decode_attention_noalloc(_dev(q, "q"), dt, q.shape[1], T_len, scale,
                                           ctypes.byref(cache.struct), _dev(out, "out"), _stream(stream)))


def tq_prefill_attention(q: torch.Tensor, cache: TQCache, t0: int, scale: float, out: torch.Tensor,
                         stream=None) -> None:
    """Chunked prefill attention: q [B, Lq, Hq, d] at positions t0 .. t0 + Lq - 1 attends causally
    to the compressed cache (the chunk's own K, V already written); out [B, Lq, Hq, d] float32."""
    dt = _DTYPES.get(q.dtype)
    if dt is None:
        raise TQError(TQ_ERR_INVALID_ARG, f"unsupported dtype {q.dtype}")
    if q.dim() != 4:
        raise TQError(TQ_ERR_INVALID_ARG, "q must be [B, Lq, Hq, d]")
    _check(lib.tq_prefill_attention(_dev(q, "q"), dt, q.shape[2], q.shape[1], t0, scale,
                                    ctypes.byref(cache.struct), _dev(out, "out"), _stream(stream)))


def tq_dequantize(cache: TQCache, which: int, T_len: int, out: torch.Tensor, stream=None) -> None:
    dt = _DTYPES.get(out.dtype)
    if dt is None:
        raise TQError(TQ_ERR_INVALID_ARG, f"unsupported dtype {out.dtype}")
    _check(lib.tq_dequantize(ctypes.byref(cache.struct), which, T_len, _dev(out, "out"), dt, _stream(stream)))


def tq_decode_bf16_workspace_bytes(B: int, Hq: int, Hkv: int, T_len: int, d: int) -> int:
    n = int(lib.tq_decode_bf16_workspace_bytes(B, Hq, Hkv, T_len, d))
    if n == 0:
        raise TQError(TQ_ERR_INVALID_ARG, last_error())
    return n


def tq_decode_attention_bf16(q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, T_len: int, scale: float,
                             out: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    B, Hkv, T_cap, d = K.shape
    _check(lib.tq_decode_attention_bf16(_dev(q, "q"), q.shape[1], _dev(K, "K"), _dev(V, "V"), B, Hkv, T_cap,
                                        T_len, d, scale, _dev(out, "out"), _dev(ws, "ws"),
                                        ws.numel() * ws.element_size(), _stream(stream)))


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A caller-owned device workspace of at least ``nbytes`` (16-byte aligned by torch)."""
    return torch.empty((nbytes + 15) // 16 * 4, dtype=torch.float32, device=device)
