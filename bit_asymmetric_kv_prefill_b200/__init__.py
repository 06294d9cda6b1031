"""B200 (sm_100a) KIVI asymmetric 2-bit KV cache: Python binding.

A thin ctypes layer over the C ABI of ``include/kivi.h`` (``libkivi_b200.so``,
built in-tree by ``bit_asymmetric_kv_prefill_b200.build``).  It only marshals
arguments: checks tensor dtype/shape/device, passes raw device pointers and the
current CUDA stream, and turns status codes into exceptions.  Every step of the
hot path runs in the library's CUDA kernels; there is no CPU fallback, and the
calls raise if the library is missing.

    cache = KiviCache(B, H_kv, D, R=128, dtype=torch.bfloat16, T_max=T + steps)
    cache.prefill(K, V)              # K, V [B, H_kv, T, D] on the GPU
    cache.append(k_t, v_t)           # [B, H_kv, D]
    out = cache.decode(q)            # q [B, H_q, D] -> fp32 [B, H_q, D]

    # quantize-dequantize under another grouping (diagnostics, no cache)
    x_hat, sq_err = fake_quant(K, AXIS_PER_TOKEN, G=32, bits=2, symmetric=True)
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# KIVI_LIB selects another build of the same library (e.g. a tuning variant).
LIB_PATH = os.environ.get("KIVI_LIB") or os.path.join(_HERE, "libkivi_b200.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "kivi.h")

KIVI_F16, KIVI_BF16 = 0, 1
AXIS_PER_CHANNEL, AXIS_PER_TOKEN = 0, 1
STATUS = {0: "KIVI_OK", 1: "KIVI_ERR_ARG", 2: "KIVI_ERR_UNSUPPORTED", 3: "KIVI_ERR_CAPACITY",
          4: "KIVI_ERR_STATE", 5: "KIVI_ERR_OOM", 6: "KIVI_ERR_CUDA", 7: "KIVI_ERR_DEVICE"}

_lib = None


class KiviError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {STATUS.get(code, code)} ({status_string(code)})")


class _Config(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H_kv", ctypes.c_int), ("D", ctypes.c_int),
                ("G", ctypes.c_int), ("R", ctypes.c_int), ("dtype", ctypes.c_int),
                ("T_max", ctypes.c_longlong), ("pre_rope", ctypes.c_int),
                ("rope_theta", ctypes.c_float), ("workspace", ctypes.c_void_p),
                ("workspace_bytes", ctypes.c_size_t)]


class _Bytes(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_size_t), ("meta", ctypes.c_size_t),
                ("residual", ctypes.c_size_t), ("scratch", ctypes.c_size_t),
                ("total", ctypes.c_size_t)]


def lib():
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m bit_asymmetric_kv_prefill_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, st = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_int
    P = ctypes.POINTER
    L.kivi_abi_version.restype = i32
    L.kivi_status_string.argtypes = [st]
    L.kivi_status_string.restype = ctypes.c_char_p
    L.kivi_cache_create.argtypes = [i32, i32, i32, i32, i32, i32, i64, P(vp)]
    L.kivi_cache_create_ex.argtypes = [P(_Config), P(vp)]
    L.kivi_cache_required_bytes.argtypes = [P(_Config), P(ctypes.c_size_t)]
    L.kivi_prefill.argtypes = [vp, vp, vp, i64, vp]
    L.kivi_prefill_ragged.argtypes = [vp, vp, vp, i64, P(i64), vp]
    L.kivi_cache_length_at.argtypes = [vp, i32, P(i64), P(i32)]
    L.kivi_append.argtypes = [vp, vp, vp, vp]
    L.kivi_decode_attn.argtypes = [vp, vp, i32, vp, vp]
    L.kivi_append_decode.argtypes = [vp, vp, vp, vp, i32, vp, vp]
    L.kivi_decode_attn_noalloc.argtypes = [vp, vp, i32, vp, vp]
    L.kivi_cache_reset.argtypes = [vp]
    L.kivi_cache_length.argtypes = [vp, P(i64), P(i32)]
    L.kivi_cache_bytes.argtypes = [vp, P(_Bytes)]
    L.kivi_export.argtypes = [vp, i64, i64, vp, vp, vp, vp, vp, vp, vp, vp]
    L.kivi_device_status.argtypes = [vp, P(i32)]
    L.kivi_debug_expire_first_wait.argtypes = [vp, i32]
    L.kivi_cache_destroy.argtypes = [vp]
    L.kivi_decode_split.argtypes = [i64, i64, i32, i32, i32, i64, i64, i64, P(i64)]
    L.kivi_fake_quant.argtypes = [vp, i32, i64, i64, i32, i32, i32, i32, i32, i32, vp, vp, vp]
    L.kivi_fake_quant_levels.argtypes = [vp, i32, i64, i64, i32, i32, i32, i32, P(ctypes.c_double),
                                         vp, vp, vp, vp]
    for name in ("kivi_cache_create", "kivi_cache_create_ex", "kivi_cache_required_bytes",
                 "kivi_prefill", "kivi_prefill_ragged", "kivi_cache_length_at", "kivi_append", "kivi_decode_attn", "kivi_decode_attn_noalloc",
                 "kivi_append_decode",
                 "kivi_cache_reset",
                 "kivi_cache_length", "kivi_cache_bytes", "kivi_export", "kivi_device_status",
                 "kivi_debug_expire_first_wait", "kivi_cache_destroy", "kivi_decode_split",
                 "kivi_fake_quant", "kivi_fake_quant_levels"):
        getattr(L, name).restype = st
    _lib = L
    return L


def declared_symbols():
    """Function names declared in include/kivi.h."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"KIVI_API[^;(]*?\b(kivi_\w+)\s*\(", text)))


def status_string(code: int) -> str:
    return lib().kivi_status_string(code).decode()


def abi_version() -> int:
    return lib().kivi_abi_version()


def _check(code: int, what: str):
    if code != 0:
        raise KiviError(code, what)


def decode_split(seqs, n_groups, r, wg, wr, warps, seq, warp):
    """Host view of the decode work split (see kivi_decode_split)."""
    out = (ctypes.c_longlong * 4)()
    _check(lib().kivi_decode_split(seqs, n_groups, r, wg, wr, warps, seq, warp, out),
           "kivi_decode_split")
    return tuple(out)


def _dtype_code(dtype) -> int:
    if dtype == torch.bfloat16:
        return KIVI_BF16
    if dtype == torch.float16:
        return KIVI_F16
    raise ValueError(f"cache dtype must be bfloat16 or float16, got {dtype}")


def _stream_ptr(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


class KiviCache:
    """One layer's KIVI cache for B sequences x H_kv heads on the current GPU."""

    def __init__(self, B: int, H_kv: int, D: int, G: int = 32, R: int = 128,
                 dtype=torch.bfloat16, T_max: int = 4096, pre_rope: bool = False,
                 rope_theta: float = 10000.0, workspace: torch.Tensor | None = None):
        self.B, self.H_kv, self.D, self.G, self.R = B, H_kv, D, G, R
        self.dtype = dtype
        self.T_max = T_max
        self.pre_rope = bool(pre_rope)
        self._cfg = _Config(B, H_kv, D, G, R, _dtype_code(dtype), T_max, int(pre_rope),
                            float(rope_theta), None, 0)
        self._workspace = workspace
        if workspace is not None:
            if not workspace.is_cuda:
                raise ValueError("workspace must be a CUDA tensor")
            self._cfg.workspace = workspace.data_ptr()
            self._cfg.workspace_bytes = workspace.numel() * workspace.element_size()
        self.device = torch.device("cuda", torch.cuda.current_device())
        h = ctypes.c_void_p()
        _check(lib().kivi_cache_create_ex(ctypes.byref(self._cfg), ctypes.byref(h)),
               "kivi_cache_create_ex")
        self._h = h

    @staticmethod
    def required_bytes(B, H_kv, D, G=32, R=128, dtype=torch.bfloat16, T_max=4096,
                       pre_rope=False, rope_theta=10000.0) -> int:
        cfg = _Config(B, H_kv, D, G, R, _dtype_code(dtype), T_max, int(pre_rope),
                      float(rope_theta), None, 0)
        n = ctypes.c_size_t()
        _check(lib().kivi_cache_required_bytes(ctypes.byref(cfg), ctypes.byref(n)),
               "kivi_cache_required_bytes")
        return n.value

    # -- argument checks (shapes are the C ABI's; the library re-checks sizes)
    def _tensor(self, t: torch.Tensor, shape, name):
        if not isinstance(t, torch.Tensor) or not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if t.dtype != self.dtype:
            raise ValueError(f"{name} must be {self.dtype}, got {t.dtype}")
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        return t.data_ptr()

    def prefill(self, K: torch.Tensor, V: torch.Tensor, stream=None):
        T = K.shape[2]
        shape = (self.B, self.H_kv, T, self.D)
        _check(lib().kivi_prefill(self._h, self._tensor(K, shape, "K"), self._tensor(V, shape, "V"),
                                  T, _stream_ptr(stream)), "kivi_prefill")

    def prefill_ragged(self, K: torch.Tensor, V: torch.Tensor, lengths, stream=None):
        """Prefill with batch element b holding its first lengths[b] tokens of
        K, V [B, H_kv, T_pad, D] (see kivi_prefill_ragged)."""
        T_pad = K.shape[2]
        shape = (self.B, self.H_kv, T_pad, self.D)
        if len(lengths) != self.B:
            raise ValueError(f"lengths must hold {self.B} values")
        arr = (ctypes.c_longlong * self.B)(*[int(t) for t in lengths])
        _check(lib().kivi_prefill_ragged(self._h, self._tensor(K, shape, "K"), self._tensor(V, shape, "V"),
                                         T_pad, arr, _stream_ptr(stream)), "kivi_prefill_ragged")

    def append(self, k: torch.Tensor, v: torch.Tensor, stream=None):
        shape = (self.B, self.H_kv, self.D)
        _check(lib().kivi_append(self._h, self._tensor(k, shape, "k_t"), self._tensor(v, shape, "v_t"),
                                 _stream_ptr(stream)), "kivi_append")

    def decode(self, q: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        H_q = q.shape[1]
        qp = self._tensor(q, (self.B, H_q, self.D), "q")
        if out is None:
            out = torch.empty((self.B, H_q, self.D), dtype=torch.float32, device=q.device)
        elif (out.dtype != torch.float32 or tuple(out.shape) != (self.B, H_q, self.D)
              or not out.is_contiguous() or not out.is_cuda):
            raise ValueError("out must be a contiguous CUDA float32 [B, H_q, D] tensor")
        _check(lib().kivi_decode_attn(self._h, qp, H_q, out.data_ptr(), _stream_ptr(stream)),
               "kivi_decode_attn")
        return out

    def append_decode(self, k: torch.Tensor, v: torch.Tensor, q: torch.Tensor,
                      out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """append(k, v) then decode(q) in one launch (two when a flush is due)."""
        shape = (self.B, self.H_kv, self.D)
        kp, vp_ = self._tensor(k, shape, "k_t"), self._tensor(v, shape, "v_t")
        H_q = q.shape[1]
        qp = self._tensor(q, (self.B, H_q, self.D), "q")
        if out is None:
            out = torch.empty((self.B, H_q, self.D), dtype=torch.float32, device=q.device)
        elif (out.dtype != torch.float32 or tuple(out.shape) != (self.B, H_q, self.D)
              or not out.is_contiguous() or not out.is_cuda):
            raise ValueError("out must be a contiguous CUDA float32 [B, H_q, D] tensor")
        _check(lib().kivi_append_decode(self._h, kp, vp_, qp, H_q, out.data_ptr(), _stream_ptr(stream)),
               "kivi_append_decode")
        return out

    def decode_noalloc(self, q: torch.Tensor, out: torch.Tensor, stream=None) -> torch.Tensor:
        """Decode into a caller-provided `out` without any device allocation:
        the library keeps this call's scratch in a fixed 8 MiB device array
        (see kivi_decode_attn_noalloc), for hosts that may not allocate."""
        H_q = q.shape[1]
        qp = self._tensor(q, (self.B, H_q, self.D), "q")
        if (out.dtype != torch.float32 or tuple(out.shape) != (self.B, H_q, self.D)
                or not out.is_contiguous() or not out.is_cuda):
            raise ValueError("out must be a contiguous CUDA float32 [B, H_q, D] tensor")
        _check(lib().kivi_decode_attn_noalloc(self._h, qp, H_q, out.data_ptr(), _stream_ptr(stream)),
               "kivi_decode_attn_noalloc")
        return out

    def reset(self):
        _check(lib().kivi_cache_reset(self._h), "kivi_cache_reset")

    def length(self):
        n_q, r = ctypes.c_longlong(), ctypes.c_int()
        _check(lib().kivi_cache_length(self._h, ctypes.byref(n_q), ctypes.byref(r)),
               "kivi_cache_length")
        return n_q.value, r.value

    def length_at(self, b: int):
        """(n_q, r) of batch element b."""
        n_q, r = ctypes.c_longlong(), ctypes.c_int()
        _check(lib().kivi_cache_length_at(self._h, b, ctypes.byref(n_q), ctypes.byref(r)),
               "kivi_cache_length_at")
        return n_q.value, r.value

    def nbytes(self) -> dict:
        b = _Bytes()
        _check(lib().kivi_cache_bytes(self._h, ctypes.byref(b)), "kivi_cache_bytes")
        return {f: getattr(b, f) for f, _ in _Bytes._fields_}

    def debug_expire_first_wait(self, on: bool = True):
        """Testing the failure path: later decode launches have each warp's
        first wait give up at once (see kivi_debug_expire_first_wait)."""
        _check(lib().kivi_debug_expire_first_wait(self._h, int(on)), "kivi_debug_expire_first_wait")

    def device_status(self) -> int:
        code = ctypes.c_int()
        _check(lib().kivi_device_status(self._h, ctypes.byref(code)), "kivi_device_status")
        return code.value

    def export(self, seq0: int = 0, nseq: int | None = None) -> dict:
        """Canonical unpacked copy (host numpy arrays) of sequences
        [seq0, seq0 + nseq), sequence = b*H_kv + h."""
        import numpy as np
        nseq = self.B * self.H_kv - seq0 if nseq is None else nseq
        n_q, r = self.length_at(seq0 // self.H_kv)   # the range shares one split
        D, G = self.D, self.G
        a = dict(codesK=np.zeros((nseq, n_q, D), np.uint8), codesV=np.zeros((nseq, n_q, D), np.uint8),
                 sK=np.zeros((nseq, n_q // G, D), np.uint16), zK=np.zeros((nseq, n_q // G, D), np.uint16),
                 sV=np.zeros((nseq, n_q, D // G), np.uint16), zV=np.zeros((nseq, n_q, D // G), np.uint16),
                 resK=np.zeros((nseq, r, D), np.uint16), resV=np.zeros((nseq, r, D), np.uint16))
        ptr = {k: v.ctypes.data_as(ctypes.c_void_p) for k, v in a.items()}
        _check(lib().kivi_export(self._h, seq0, nseq, ptr["codesK"], ptr["codesV"], ptr["sK"],
                                 ptr["zK"], ptr["sV"], ptr["zV"], ptr["resK"], ptr["resV"]),
               "kivi_export")
        return a

    def close(self):
        if getattr(self, "_h", None):
            lib().kivi_cache_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def fake_quant(x: torch.Tensor, axis: int, G: int = 32, bits: int = 2, symmetric: bool = False,
               out: torch.Tensor | None = None, error: bool = True, values: bool = True,
               stream=None, outlier: int = 0):
    """Quantize-dequantize every [T, D] matrix of x ([..., T, D], bf16 or fp16,
    on the GPU) under one grouping (see kivi_fake_quant): ``axis`` is
    AXIS_PER_CHANNEL (groups of G tokens of a channel, the KIVI key rule) or
    AXIS_PER_TOKEN (groups of G channels of a token, the KIVI value rule);
    ``outlier`` = 1 keeps each group's largest-magnitude element exactly.

    Returns (x_hat, sq_err): x_hat fp32 with x's shape (None unless
    ``values``), sq_err fp64 [prod(leading dims)] holding sum (x - x_hat)^2 per
    matrix (None unless ``error``)."""
    if not isinstance(x, torch.Tensor) or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous CUDA tensor")
    if x.dim() < 2:
        raise ValueError("x must have shape [..., T, D]")
    T, D = x.shape[-2], x.shape[-1]
    N = x.numel() // max(T * D, 1)
    xh = None
    if values:
        if out is None:
            out = torch.empty(x.shape, dtype=torch.float32, device=x.device)
        elif (out.dtype != torch.float32 or out.shape != x.shape or not out.is_contiguous()
              or not out.is_cuda):
            raise ValueError("out must be a contiguous CUDA float32 tensor shaped like x")
        xh = out
    err = torch.empty(N, dtype=torch.float64, device=x.device) if error else None
    _check(lib().kivi_fake_quant(x.data_ptr(), _dtype_code(x.dtype), N, T, D, axis, G, bits,
                                 int(symmetric), int(outlier),
                                 xh.data_ptr() if xh is not None else None,
                                 err.data_ptr() if err is not None else None, _stream_ptr(stream)),
           "kivi_fake_quant")
    return xh, err


def fake_quant_levels(x: torch.Tensor, axis: int, G: int, levels, values: bool = True,
                      codes: bool = False, error: bool = True, stream=None):
    """Quantize-dequantize every [T, D] matrix of x ([..., T, D], bf16 or fp16,
    on the GPU) with non-uniform levels per group (see kivi_fake_quant_levels):
    each group's elements are coded by the nearest of the normalized
    ``levels`` on the group's [min, max].

    Returns (x_hat, codes, sq_err): x_hat fp32 with x's shape, codes uint8 with
    x's shape, sq_err fp64 [prod(leading dims)]; each None unless asked for."""
    if not isinstance(x, torch.Tensor) or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous CUDA tensor")
    if x.dim() < 2:
        raise ValueError("x must have shape [..., T, D]")
    T, D = x.shape[-2], x.shape[-1]
    N = x.numel() // max(T * D, 1)
    lev = (ctypes.c_double * len(levels))(*[float(v) for v in levels])
    xh = torch.empty(x.shape, dtype=torch.float32, device=x.device) if values else None
    cc = torch.empty(x.shape, dtype=torch.uint8, device=x.device) if codes else None
    err = torch.empty(N, dtype=torch.float64, device=x.device) if error else None
    _check(lib().kivi_fake_quant_levels(x.data_ptr(), _dtype_code(x.dtype), N, T, D, axis, G,
                                        len(levels), lev,
                                        xh.data_ptr() if xh is not None else None,
                                        cc.data_ptr() if cc is not None else None,
                                        err.data_ptr() if err is not None else None,
                                        _stream_ptr(stream)),
           "kivi_fake_quant_levels")
    return xh, cc, err
