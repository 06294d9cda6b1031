"""Plain CPU oracle for the KIVI asymmetric 2-bit KV cache (test infrastructure).

Only the test-suite, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline leg may import this package.  The arithmetic lives in
``kivi_oracle.c`` (plain C, fp32 quantization rounded once per operation, fp64
attention); this module only builds it, marshals numpy arrays into it and loops
over (batch, kv-head) sequences.  It imports nothing from the CUDA library.

Canonical layouts (row-major, per cache):
  codesK, codesV  [B, H_kv, Tcap, D]    uint8 in {0..3}
  sK, zK          [B, H_kv, Tcap/G, D]  fp16 bit patterns (uint16)
  sV, zV          [B, H_kv, Tcap, D/G]  fp16 bit patterns (uint16)
  resK, resV      [B, H_kv, R, D]       cache dtype bit patterns (uint16)
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kivi_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libkivi_oracle.so")
_lib = None

DTYPE_F16 = 0
DTYPE_BF16 = 1


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no FMA contraction, no fast-math)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=gnu11", "-ffp-contract=off", "-fno-fast-math",
           "-fno-builtin", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _P(t):
    return ctypes.POINTER(t)


def lib():
    global _lib
    if _lib is not None:
        return _lib
    L = ctypes.CDLL(build())
    u8p, u16p, f32p, f64p = _P(ctypes.c_uint8), _P(ctypes.c_uint16), _P(ctypes.c_float), _P(ctypes.c_double)
    i64p, i32p = _P(ctypes.c_longlong), _P(ctypes.c_int)
    c_int, c_ll, c_d = ctypes.c_int, ctypes.c_longlong, ctypes.c_double
    L.oracle_split.argtypes = [c_ll, c_int, i64p, i32p]
    L.oracle_quant_group.argtypes = [f32p, c_int, u8p, u16p, u16p]
    L.oracle_quant_k_group.argtypes = [u16p, c_int, c_int, c_int, u8p, u16p, u16p]
    L.oracle_quant_v_token.argtypes = [u16p, c_int, c_int, c_int, u8p, u16p, u16p]
    L.oracle_prefill_seq.argtypes = [u16p, u16p, c_ll, c_int, c_int, c_int, c_int,
                                     u8p, u16p, u16p, u8p, u16p, u16p, u16p, u16p, i64p, i32p]
    L.oracle_append_seq.argtypes = [u16p, u16p, c_int, c_int, c_int, c_int,
                                    u8p, u16p, u16p, u8p, u16p, u16p, u16p, u16p, i64p, i32p]
    L.oracle_decode_seq.argtypes = [u16p, c_int, c_int, c_int, c_int, c_int, c_int, c_d,
                                    u8p, u16p, u16p, u8p, u16p, u16p, u16p, u16p, c_ll, c_int,
                                    f64p, f32p]
    L.oracle_rope_inv_freq.argtypes = [c_int, c_d, f32p]
    L.oracle_rope_row.argtypes = [f64p, c_int, c_ll, f32p]
    L.oracle_kv_bytes.argtypes = [c_ll, c_ll, c_ll, c_ll, c_ll, c_int, c_int, c_ll, f64p]
    L.oracle_fake_quant.argtypes = [f32p, c_ll, c_int, c_int, c_int, c_int, c_int, c_int, f32p, i32p]
    L.oracle_fake_quant_levels.argtypes = [f32p, c_ll, c_int, c_int, c_int, c_int, f64p, f32p, i32p]
    L.oracle_bf16_to_float.argtypes = [ctypes.c_uint16]
    L.oracle_bf16_to_float.restype = ctypes.c_float
    L.oracle_f16_to_float.argtypes = [ctypes.c_uint16]
    L.oracle_f16_to_float.restype = ctypes.c_float
    L.oracle_float_to_f16.argtypes = [ctypes.c_float]
    L.oracle_float_to_f16.restype = ctypes.c_uint16
    _lib = L
    return L


def workers() -> int:
    """Threads the oracle runs sequences on: the CPUs this process may use
    (``KIVI_ORACLE_THREADS`` overrides).  Each (batch, kv head) sequence is
    one C call, and ctypes releases the GIL for the call's duration, so the
    sequences of a cache run in parallel; none shares memory with another,
    and every result is the same as with one thread."""
    env = os.environ.get("KIVI_ORACLE_THREADS")
    if env:
        return max(1, int(env))
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


_pool = None


def parallel_map(fn, items, threads=None):
    """list(map(fn, items)) on up to `threads` (default workers()) threads."""
    items = list(items)
    n = workers() if threads is None else threads
    if n <= 1 or len(items) <= 1:
        return [fn(x) for x in items]
    global _pool
    if threads is not None:
        with ThreadPoolExecutor(n) as ex:
            return list(ex.map(fn, items))
    if _pool is None:
        _pool = ThreadPoolExecutor(n)
    return list(_pool.map(fn, items))


def _ptr(a: np.ndarray, ct):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(_P(ct))


# ---- scalar / small helpers ------------------------------------------------

def split(T: int, R: int):
    n_q, r = ctypes.c_longlong(), ctypes.c_int()
    lib().oracle_split(T, R, ctypes.byref(n_q), ctypes.byref(r))
    return n_q.value, r.value


def quant_group(x: np.ndarray):
    """One group (fp32 values) -> (codes uint8[n], s_bits, z_bits)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    c = np.zeros(x.size, np.uint8)
    s, z = ctypes.c_uint16(), ctypes.c_uint16()
    lib().oracle_quant_group(_ptr(x, ctypes.c_float), x.size, _ptr(c, ctypes.c_uint8),
                             ctypes.byref(s), ctypes.byref(z))
    return c, s.value, z.value


def f16_to_float(bits):
    L = lib()
    return np.array([L.oracle_f16_to_float(int(b)) for b in np.ravel(bits)], np.float32).reshape(np.shape(bits))


def float_to_f16(x):
    L = lib()
    return np.array([L.oracle_float_to_f16(float(v)) for v in np.ravel(x)], np.uint16).reshape(np.shape(x))


def rope_inv_freq(D: int, theta: float) -> np.ndarray:
    out = np.zeros(D // 2, np.float32)
    lib().oracle_rope_inv_freq(D, theta, _ptr(out, ctypes.c_float))
    return out


def rope_row(x: np.ndarray, pos: int, theta: float) -> np.ndarray:
    x = np.array(x, dtype=np.float64)
    inv = rope_inv_freq(x.size, theta)
    lib().oracle_rope_row(_ptr(x, ctypes.c_double), x.size, pos, _ptr(inv, ctypes.c_float))
    return x


def kv_bytes(layers, heads, head_dim, R, context, bits=2, dtype_bytes=2, G=32):
    out = np.zeros(7, np.float64)
    lib().oracle_kv_bytes(layers, heads, head_dim, R, context, bits, dtype_bytes, G,
                          _ptr(out, ctypes.c_double))
    keys = ["grouped_per_token", "residual_total", "residual_per_token", "sum_per_token",
            "full_per_token", "reduction", "metadata_per_token"]
    return dict(zip(keys, out.tolist()))


AXIS_PER_CHANNEL = 0   # groups of G consecutive tokens of one channel (KIVI keys)
AXIS_PER_TOKEN = 1     # groups of G consecutive channels of one token (KIVI values)


OUTLIER_CODE = -1000   # code reported for a group's sparse (exactly kept) element


def fake_quant(x: np.ndarray, axis: int, G: int = 32, bits: int = 2, sym: bool = False,
               codes: bool = False, outlier: int = 0):
    """Quantize-dequantize every [T, D] matrix of x (fp32, shape [..., T, D])
    under one grouping (see oracle_fake_quant); ``outlier`` = 1 keeps each
    group's largest-magnitude element exactly (dense-and-sparse).  Returns
    x_hat (fp32, same shape), and the integer codes too when ``codes``."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    T, D = x.shape[-2:]
    flat = x.reshape(-1, T, D)
    xh = np.zeros_like(flat)
    cc = np.zeros(flat.shape, np.int32) if codes else None
    L = lib()
    for i in range(flat.shape[0]):
        xi = np.ascontiguousarray(flat[i])
        oi = np.zeros((T, D), np.float32)
        ci = np.zeros((T, D), np.int32) if codes else None
        rc = L.oracle_fake_quant(_ptr(xi, ctypes.c_float), T, D, axis, G, bits, int(sym),
                                 int(outlier), _ptr(oi, ctypes.c_float),
                                 _ptr(ci, ctypes.c_int) if codes else None)
        if rc != 0:
            raise ValueError(f"unsupported fake_quant arguments: T={T} D={D} axis={axis} "
                             f"G={G} bits={bits} sym={sym} outlier={outlier}")
        xh[i] = oi
        if codes:
            cc[i] = ci
    xh = xh.reshape(x.shape)
    return (xh, cc.reshape(x.shape)) if codes else xh


def fake_quant_levels(x: np.ndarray, axis: int, G: int, levels, codes: bool = False):
    """Non-uniform levels (see oracle_fake_quant_levels): every group of x
    (fp32, [..., T, D]) coded by the nearest of the normalized ``levels`` on
    its [min, max].  Returns x_hat, and the codes too when ``codes``."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    lev = np.ascontiguousarray(levels, dtype=np.float64)
    T, D = x.shape[-2:]
    flat = x.reshape(-1, T, D)
    xh = np.zeros_like(flat)
    cc = np.zeros(flat.shape, np.int32) if codes else None
    L = lib()
    for i in range(flat.shape[0]):
        xi = np.ascontiguousarray(flat[i])
        oi = np.zeros((T, D), np.float32)
        ci = np.zeros((T, D), np.int32) if codes else None
        rc = L.oracle_fake_quant_levels(_ptr(xi, ctypes.c_float), T, D, axis, G, lev.size,
                                        _ptr(lev, ctypes.c_double), _ptr(oi, ctypes.c_float),
                                        _ptr(ci, ctypes.c_int) if codes else None)
        if rc != 0:
            raise ValueError(f"unsupported fake_quant_levels arguments: T={T} D={D} axis={axis} "
                             f"G={G} levels={lev.tolist()}")
        xh[i] = oi
        if codes:
            cc[i] = ci
    xh = xh.reshape(x.shape)
    return (xh, cc.reshape(x.shape)) if codes else xh


# ---- the cache --------------------------------------------------------------

class OracleCache:
    """CPU model of one layer's KIVI cache for B sequences x H_kv heads.

    Each batch element b keeps its own split (nqb[b] quantized tokens, rb[b]
    residual tokens), so a prefill may give every batch element its own
    length; the heads of one batch element share it.  ``n_q`` and ``r`` read
    the common split of a uniform batch."""

    def __init__(self, B, H_kv, D, G, R, dtype, T_max, pre_rope=False, rope_theta=10000.0):
        assert D % G == 0 and R % G == 0
        self.B, self.H, self.D, self.G, self.R = B, H_kv, D, G, R
        self.dtype = dtype
        self.pre_rope = bool(pre_rope)
        self.theta = float(rope_theta)
        self.Tcap = -(-T_max // G) * G
        Tc = self.Tcap
        self.codesK = np.zeros((B, H_kv, Tc, D), np.uint8)
        self.codesV = np.zeros((B, H_kv, Tc, D), np.uint8)
        self.sK = np.zeros((B, H_kv, Tc // G, D), np.uint16)
        self.zK = np.zeros((B, H_kv, Tc // G, D), np.uint16)
        self.sV = np.zeros((B, H_kv, Tc, D // G), np.uint16)
        self.zV = np.zeros((B, H_kv, Tc, D // G), np.uint16)
        self.resK = np.zeros((B, H_kv, R, D), np.uint16)
        self.resV = np.zeros((B, H_kv, R, D), np.uint16)
        self.nqb = np.zeros(B, np.int64)
        self.rb = np.zeros(B, np.int64)

    def _uniform(self, a):
        if not (a == a[0]).all():
            raise ValueError("the batch has per-sequence lengths; read nqb / rb")
        return int(a[0])

    @property
    def n_q(self) -> int:
        return self._uniform(self.nqb)

    @property
    def r(self) -> int:
        return self._uniform(self.rb)

    def _seq_ptrs(self, b, h):
        U8, U16 = ctypes.c_uint8, ctypes.c_uint16
        return (_ptr(self.codesK[b, h], U8), _ptr(self.sK[b, h], U16), _ptr(self.zK[b, h], U16),
                _ptr(self.codesV[b, h], U8), _ptr(self.sV[b, h], U16), _ptr(self.zV[b, h], U16),
                _ptr(self.resK[b, h], U16), _ptr(self.resV[b, h], U16))

    def prefill(self, K: np.ndarray, V: np.ndarray, lengths=None):
        """K, V: uint16 bit patterns [B, H_kv, T, D].  ``lengths``: optional
        per-batch-element token counts 1 <= T_b <= T (batch element b uses
        K[b, :, :T_b]); default T for all."""
        K = np.ascontiguousarray(K, dtype=np.uint16)
        V = np.ascontiguousarray(V, dtype=np.uint16)
        T = K.shape[2]
        lengths = [T] * self.B if lengths is None else [int(t) for t in lengths]
        if len(lengths) != self.B or min(lengths) < 1 or max(lengths) > T:
            raise ValueError(f"lengths must be {self.B} values in [1, {T}], got {lengths}")
        L = lib()

        def one(bh):
            b, h = bh
            nq, r = ctypes.c_longlong(), ctypes.c_int()
            kb = np.ascontiguousarray(K[b, h, :lengths[b]])
            vb = np.ascontiguousarray(V[b, h, :lengths[b]])
            L.oracle_prefill_seq(_ptr(kb, ctypes.c_uint16), _ptr(vb, ctypes.c_uint16),
                                 lengths[b], self.D, self.G, self.R, self.dtype,
                                 *self._seq_ptrs(b, h), ctypes.byref(nq), ctypes.byref(r))
            return b, nq.value, r.value

        for b, nq, r in parallel_map(one, [(b, h) for b in range(self.B) for h in range(self.H)]):
            self.nqb[b], self.rb[b] = nq, r

    def append(self, k: np.ndarray, v: np.ndarray):
        """k, v: uint16 bit patterns [B, H_kv, D]."""
        k = np.ascontiguousarray(k, dtype=np.uint16)
        v = np.ascontiguousarray(v, dtype=np.uint16)
        L = lib()
        nq, r = ctypes.c_longlong(), ctypes.c_int()
        for b in range(self.B):
            for h in range(self.H):
                nq.value, r.value = int(self.nqb[b]), int(self.rb[b])
                kb, vb = np.ascontiguousarray(k[b, h]), np.ascontiguousarray(v[b, h])
                L.oracle_append_seq(_ptr(kb, ctypes.c_uint16), _ptr(vb, ctypes.c_uint16),
                                    self.D, self.G, self.R, self.dtype, *self._seq_ptrs(b, h),
                                    ctypes.byref(nq), ctypes.byref(r))
            self.nqb[b], self.rb[b] = nq.value, r.value

    def decode(self, q: np.ndarray, heads=None) -> np.ndarray:
        """q: uint16 bits [B, H_q, D] -> out float32 [B, H_q, D].

        ``heads``: optional list of (b, h_kv) pairs to evaluate; other rows of
        the result are left as NaN (for sampled checks of large caches)."""
        q = np.ascontiguousarray(q, dtype=np.uint16)
        B, H_q, D = q.shape
        HG = H_q // self.H
        out = np.full((B, H_q, D), np.nan, np.float32)
        L = lib()
        pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(self.H)]

        def one(bh):
            b, h = bh
            sc = np.zeros(max(int(self.nqb[b] + self.rb[b]), 1), np.float64)
            qb = np.ascontiguousarray(q[b, h * HG:(h + 1) * HG])
            ob = np.zeros((HG, D), np.float32)
            L.oracle_decode_seq(_ptr(qb, ctypes.c_uint16), HG, D, self.G, self.R, self.dtype,
                                int(self.pre_rope), self.theta, *self._seq_ptrs(b, h),
                                int(self.nqb[b]), int(self.rb[b]), _ptr(sc, ctypes.c_double),
                                _ptr(ob, ctypes.c_float))
            out[b, h * HG:(h + 1) * HG] = ob

        parallel_map(one, pairs)
        return out

    def quantized(self):
        """Canonical quantized store restricted to the first n_q tokens."""
        nq, G = self.n_q, self.G
        return dict(codesK=self.codesK[:, :, :nq], codesV=self.codesV[:, :, :nq],
                    sK=self.sK[:, :, :nq // G], zK=self.zK[:, :, :nq // G],
                    sV=self.sV[:, :, :nq], zV=self.zV[:, :, :nq],
                    resK=self.resK[:, :, :self.r], resV=self.resV[:, :, :self.r])
