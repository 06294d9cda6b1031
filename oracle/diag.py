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

and, for keys stored before or after RoPE (KVQuant summary, "Pre-RoPE Key
Quantization"; KIVI article, paragraph 4), ``rope="pre"`` quantizes K and
rotates K_hat, ``rope="post"`` quantizes the rotated keys; both are compared
with the rotated exact keys.
"""
from __future__ import annotations

import math

import numpy as np

from . import AXIS_PER_CHANNEL, AXIS_PER_TOKEN, fake_quant, rope_row

# mode: ((key axis, symmetric, sparse elements), (value axis, symmetric, sparse))
MODES = {
    "kivi": ((AXIS_PER_CHANNEL, False, 0), (AXIS_PER_TOKEN, False, 0)),
    "k_per_token": ((AXIS_PER_TOKEN, False, 0), (AXIS_PER_TOKEN, False, 0)),
    "v_per_channel": ((AXIS_PER_CHANNEL, False, 0), (AXIS_PER_CHANNEL, False, 0)),
    "naive_symmetric": ((AXIS_PER_TOKEN, True, 0), (AXIS_PER_TOKEN, True, 0)),
    "kivi_sparse": ((AXIS_PER_CHANNEL, False, 1), (AXIS_PER_TOKEN, False, 1)),
    "k_per_token_sparse": ((AXIS_PER_TOKEN, False, 1), (AXIS_PER_TOKEN, False, 1)),
}


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
        K_hat = fake_quant(K, ka, G, bits, ks, outlier=ko).astype(np.float64)
    elif rope == "pre":
        K_ref = rotate(K, theta)
        K_hat = rotate(fake_quant(K, ka, G, bits, ks, outlier=ko), theta)
    elif rope == "post":
        K_ref = rotate(K, theta)
        K_hat = fake_quant(K_ref.astype(np.float32), ka, G, bits, ks, outlier=ko).astype(np.float64)
    else:
        raise ValueError(f"rope must be None, 'pre' or 'post', got {rope!r}")
    V_hat = fake_quant(V, va, G, bits, vs, outlier=vo).astype(np.float64)
    V_ref = V.astype(np.float64)
    o = attention(q, K_ref, V_ref)
    o_hat = attention(q, K_hat, V_hat)
    return dict(
        key=float(np.mean([np.linalg.norm(K_ref[h] - K_hat[h]) for h in range(K.shape[0])])),
        value=float(np.mean([np.linalg.norm(V_ref[h] - V_hat[h]) for h in range(V.shape[0])])),
        attn=float(100.0 * np.linalg.norm(o - o_hat) / np.linalg.norm(o)),
    )
