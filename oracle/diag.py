"""Errors of the grouping modes that the KIVI pages compare (test infrastructure).

Like the rest of ``oracle``, only tests, the smoke check and the benchmark's CPU
legs may import this module.  It quantizes synthetic keys and values under
each grouping with ``oracle.fake_quant`` and measures, in float64:

  key error      ||K - K_hat||_F of one head's [T, D] keys, mean over heads;
  value error    ||V - V_hat||_F, likewise;
  attention err  100 * ||o - o_hat||_F / ||o||_F over all heads and queries,
                 o = softmax(q K^T / sqrt(D)) V with the exact cache and o_hat
                 the same with K_hat, V_hat (no mask).

The pages print these three kinds of number ("KIVI Quantization Secures
Llama-2 Accuracy at Two Bits", paragraphs 2-3: key error 13.67 per token
against 4.55 per channel; value error 4.57 per token against 3.73 per
channel; attention-output relative error 3.55 against 49.89) without stating
the norm; the Frobenius norm and the percentage above are this module's
reading.  The modes:

  kivi             keys per channel, values per token, asymmetric (the method)
  k_per_token      keys and values per token, asymmetric
  v_per_channel    keys and values per channel, asymmetric
  naive_symmetric  keys and values per token, symmetric absmax (the record
                   kv-efficiency/kivi-2bit-llama2-13b-mha-4k, "Quality" field)
  kivi_sparse      KIVI's grouping, each group dense-and-sparse: its largest-
                   magnitude element kept exactly (KVQuant summary, "Per-Vector
                   Dense-and-Sparse Quantization")
  k_per_token_sparse  keys and values per token, dense-and-sparse
  kivi_nuq         KIVI's grouping with four non-uniform levels per group
                   (KVQuant summary, "Non-Uniform KV Cache Quantization"),
                   fitted by ``fit_levels`` to the keys and to the values

and, for keys stored before or after RoPE (KVQuant summary, "Pre-RoPE Key
Quantization"; KIVI article, paragraph 4), ``rope="pre"`` quantizes K and
rotates K_hat, ``rope="post"`` quantizes the rotated keys; both are compared
with the rotated exact keys.
"""
from __future__ import annotations

import math

import numpy as np

from . import AXIS_PER_CHANNEL, AXIS_PER_TOKEN, fake_quant, fake_quant_levels, rope_row

# mode: ((key axis, symmetric, sparse elements), (value axis, symmetric, sparse))
MODES = {
    "kivi": ((AXIS_PER_CHANNEL, False, 0), (AXIS_PER_TOKEN, False, 0)),
    "k_per_token": ((AXIS_PER_TOKEN, False, 0), (AXIS_PER_TOKEN, False, 0)),
    "v_per_channel": ((AXIS_PER_CHANNEL, False, 0), (AXIS_PER_CHANNEL, False, 0)),
    "naive_symmetric": ((AXIS_PER_TOKEN, True, 0), (AXIS_PER_TOKEN, True, 0)),
    "kivi_sparse": ((AXIS_PER_CHANNEL, False, 1), (AXIS_PER_TOKEN, False, 1)),
    "k_per_token_sparse": ((AXIS_PER_TOKEN, False, 1), (AXIS_PER_TOKEN, False, 1)),
    "kivi_nuq": ((AXIS_PER_CHANNEL, False, "nuq"), (AXIS_PER_TOKEN, False, "nuq")),
}


def group_positions(x: np.ndarray, axis: int, G: int) -> np.ndarray:
    """(x - min)/(max - min) of every element of every non-constant group
    (float64, flattened)."""
    x = np.asarray(x, np.float64)
    T, D = x.shape[-2:]
    flat = x.reshape(-1, T, D)
    if axis == AXIS_PER_CHANNEL:
        g = flat.reshape(flat.shape[0], T // G, G, D).transpose(0, 1, 3, 2).reshape(-1, G)
    else:
        g = flat.reshape(-1, G)
    mn = g.min(axis=1, keepdims=True)
    rg = g.max(axis=1, keepdims=True) - mn
    keep = rg[:, 0] > 0
    return ((g[keep] - mn[keep]) / rg[keep]).ravel()


def fit_levels(x: np.ndarray, axis: int, G: int = 32, nlev: int = 4, iters: int = 40) -> np.ndarray:
    """Normalized levels for ``fake_quant_levels``: Lloyd's algorithm (1-D
    k-means) over the group positions of x, started from their nlev evenly
    spaced quantiles (evenly spaced levels can stall with two clusters on one
    level); each element goes to its nearest level (the lower one on ties) and
    each level moves to the mean of its elements (a level with none stays)."""
    u = np.sort(group_positions(x, axis, G))
    lev = u[np.round(np.linspace(0, u.size - 1, nlev)).astype(np.int64)].copy()
    for _ in range(iters):
        cuts = (lev[1:] + lev[:-1]) / 2.0
        idx = np.searchsorted(cuts, u, side="left")   # u == cut goes to the lower level
        new = lev.copy()
        for k in range(nlev):
            sel = u[idx == k]
            if sel.size:
                new[k] = sel.mean()
        if np.array_equal(new, lev):
            break
        lev = new
    return lev


def _quantize(x, axis, sym, sparse, G, bits):
    if sparse == "nuq":
        return fake_quant_levels(x, axis, G, fit_levels(x, axis, G, 1 << bits))
    return fake_quant(x, axis, G, bits, sym, outlier=sparse)


def rotate(K: np.ndarray, theta: float) -> np.ndarray:
    """RoPE of every row of K [..., T, D] at absolute positions 0..T-1 (float64)."""
    K = np.asarray(K, np.float64)
    out = np.empty_like(K)
    flat_in = K.reshape(-1, K.shape[-2], K.shape[-1])
    flat_out = out.reshape(flat_in.shape)
    for i in range(flat_in.shape[0]):
        for t in range(flat_in.shape[1]):
            flat_out[i, t] = rope_row(flat_in[i, t], t, theta)
    return out


def attention(q: np.ndarray, K: np.ndarray, V: np.ndarray) -> np.ndarray:
    """softmax(q K^T / sqrt(D)) V per head, float64: q [H, M, D], K/V [H, T, D]."""
    q, K, V = (np.asarray(a, np.float64) for a in (q, K, V))
    s = np.einsum("hmd,htd->hmt", q, K) / math.sqrt(q.shape[-1])
    s -= s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=-1, keepdims=True)
    return np.einsum("hmt,htd->hmd", p, V)


def errors(K: np.ndarray, V: np.ndarray, q: np.ndarray, mode: str = "kivi", G: int = 32,
           bits: int = 2, rope: str | None = None, theta: float = 10000.0) -> dict:
    """Errors of one mode.  K, V: exact fp32 values [H, T, D] (keys before RoPE
    when ``rope`` is given); q: [H, M, D] queries (after RoPE)."""
    (ka, ks, ko), (va, vs, vo) = MODES[mode]
    K = np.asarray(K, np.float32)
    V = np.asarray(V, np.float32)
    if rope is None:
        K_ref = K.astype(np.float64)
        K_hat = _quantize(K, ka, ks, ko, G, bits).astype(np.float64)
    elif rope == "pre":
        K_ref = rotate(K, theta)
        K_hat = rotate(_quantize(K, ka, ks, ko, G, bits), theta)
    elif rope == "post":
        K_ref = rotate(K, theta)
        K_hat = _quantize(K_ref.astype(np.float32), ka, ks, ko, G, bits).astype(np.float64)
    else:
        raise ValueError(f"rope must be None, 'pre' or 'post', got {rope!r}")
    V_hat = _quantize(V, va, vs, vo, G, bits).astype(np.float64)
    V_ref = V.astype(np.float64)
    o = attention(q, K_ref, V_ref)
    o_hat = attention(q, K_hat, V_hat)
    return dict(
        key=float(np.mean([np.linalg.norm(K_ref[h] - K_hat[h]) for h in range(K.shape[0])])),
        value=float(np.mean([np.linalg.norm(V_ref[h] - V_hat[h]) for h in range(V.shape[0])])),
        attn=float(100.0 * np.linalg.norm(o - o_hat) / np.linalg.norm(o)),
    )

