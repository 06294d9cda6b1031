"""Helpers shared by the GPU parity tests: drive the CUDA library and the CPU
oracle on the same seeded inputs and compare them.

Bars: codes, scales, zeros and residual rows bit-exact; attention output with
relative L2 error <= 5e-3 and max-abs error <= 2e-3 * max|ref| against the
oracle's double-precision attention over the same dequantized cache.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from bit_asymmetric_kv_prefill_b200 import KiviCache, synth

REL_L2 = 5e-3
MAX_ABS = 2e-3


def odtype(w):
    return oracle.DTYPE_BF16 if w.dtype == "bf16" else oracle.DTYPE_F16


def attn_errors(out, ref):
    out = np.asarray(out, np.float64)
    ref = np.asarray(ref, np.float64)
    rel = np.linalg.norm(out - ref) / max(np.linalg.norm(ref), 1e-30)
    mabs = np.abs(out - ref).max() / max(np.abs(ref).max(), 1e-30)
    return rel, mabs


def assert_attn_close(out, ref, what=""):
    assert np.all(np.isfinite(out)), what
    rel, mabs = attn_errors(out, ref)
    assert rel <= REL_L2 and mabs <= MAX_ABS, f"{what}: rel-L2 {rel:.3e}, max-abs/max {mabs:.3e}"
    return rel, mabs


def _runs(seqs, chunk):
    """Consecutive runs (first, count) of the sorted sequence list, at most
    `chunk` long."""
    seqs = sorted(seqs)
    runs, i = [], 0
    while i < len(seqs):
        j = i
        while j + 1 < len(seqs) and seqs[j + 1] == seqs[j] + 1 and j + 1 - i < chunk:
            j += 1
        runs.append((seqs[i], j - i + 1))
        i = j + 1
    return runs


def assert_store_equal(cache: KiviCache, orc: oracle.OracleCache, seqs, chunk=8, orc_index=None):
    """Bit-exact comparison of the quantized store and residual of the given
    flattened sequences (b*H_kv + h) of the GPU cache with an oracle cache.
    The oracle holds every sequence, or (orc_index) maps GPU sequence s to the
    oracle's sequence orc_index[s].  The GPU store is exported in runs of
    `chunk` sequences on the oracle's threads (the export is a C call that
    releases the GIL)."""
    assert cache.length() == (orc.n_q, orc.r)
    ref = orc.quantized()
    keys = ("codesK", "codesV", "sK", "zK", "sV", "zV", "resK", "resV")

    def one(run):
        s0, n = run
        got = cache.export(s0, n)
        for i in range(n):
            s = s0 + i
            o = s if orc_index is None else orc_index[s]
            ob, oh = divmod(o, orc.H)
            for key in keys:
                a, b = got[key][i], ref[key][ob, oh]
                if not np.array_equal(a, b):
                    bad = np.argwhere(a != b)
                    return (f"{key} differs for sequence {s} at {bad[:5].tolist()} "
                            f"({len(bad)} entries): gpu {a[tuple(bad[0])]} oracle {b[tuple(bad[0])]}")
        return None

    errs = [e for e in oracle.parallel_map(one, _runs(seqs, chunk)) if e]
    if errs:
        raise AssertionError(errs[0] + (f" (and {len(errs) - 1} more runs)" if len(errs) > 1 else ""))


class Pair:
    """A GPU cache and an oracle cache fed identical bits.  The oracle holds
    either every sequence or only the sampled ones (`sample`)."""

    def __init__(self, w: synth.Workload, seed=0, sample=None, T_max=None):
        self.w = w
        self.seed = seed
        self.HG = w.H_q // w.H_kv
        self.cache = KiviCache(w.B, w.H_kv, w.D, w.G, w.R, w.torch_dtype,
                               T_max or w.T_max, pre_rope=w.pre_rope, rope_theta=w.rope_theta)
        self.sample = sample
        nb, nh = (w.B, w.H_kv) if sample is None else (len(sample), 1)
        self.orc = oracle.OracleCache(nb, nh, w.D, w.G, w.R, odtype(w), T_max or w.T_max,
                                      pre_rope=w.pre_rope, rope_theta=w.rope_theta)

    def seqs(self):
        return list(range(self.w.B * self.w.H_kv)) if self.sample is None else list(self.sample)

    def _pick(self, t: torch.Tensor):
        """[B, H_kv, ...] -> host bits of the oracle's sequences."""
        if self.sample is None:
            return synth.bits(t)
        rows = [t[s // self.w.H_kv, s % self.w.H_kv] for s in self.sample]
        return synth.bits(torch.stack(rows)[:, None])

    def _pick_q(self, q: torch.Tensor):
        if self.sample is None:
            return synth.bits(q)
        HG = self.HG
        rows = [q[s // self.w.H_kv, (s % self.w.H_kv) * HG:(s % self.w.H_kv + 1) * HG] for s in self.sample]
        return synth.bits(torch.stack(rows))

    def prefill(self, K, V):
        self.cache.prefill(K, V)
        self.orc.prefill(self._pick(K), self._pick(V))

    def append(self, k, v):
        self.cache.append(k, v)
        self.orc.append(self._pick(k), self._pick(v))

    def decode(self, q, seqs=None):
        """GPU output restricted to the oracle's sequences, and the oracle's;
        `seqs` (flattened b*H_kv + h, oracle holding every sequence) restricts
        both to those sequences' query heads."""
        out = self.cache.decode(q)
        torch.cuda.synchronize()
        o = out.cpu().numpy()
        if seqs is not None:
            assert self.sample is None
            H, HG = self.w.H_kv, self.HG
            ref = self.orc.decode(synth.bits(q), heads=[divmod(s, H) for s in seqs])
            rows = lambda a: np.stack([a[s // H, (s % H) * HG:(s % H + 1) * HG] for s in seqs])
            return rows(o), rows(ref)
        ref = self.orc.decode(self._pick_q(q))
        if self.sample is None:
            return o, ref
        HG = self.HG
        got = np.stack([o[s // self.w.H_kv, (s % self.w.H_kv) * HG:(s % self.w.H_kv + 1) * HG]
                        for s in self.sample])
        return got, ref

    def check_store(self, every=1):
        seqs = self.seqs()[::every]
        if self.sample is None:
            assert_store_equal(self.cache, self.orc, seqs)
        else:
            # oracle sequence i <-> GPU sequence sample[i]
            assert_store_equal(self.cache, self.orc, seqs,
                               orc_index={s: i for i, s in enumerate(self.sample)})


def _vals(bits, dtype):
    bits = np.asarray(bits, np.uint16)
    if dtype == "bf16":
        return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return bits.view(np.float16).astype(np.float64)


def value_weight_bound(cache: KiviCache, q_bits, w: synth.Workload):
    """Elementwise bound on |decode - oracle| from the one rounding the decode
    kernel adds to fp32 accumulation: each quantized token's value weight
    p_t * s_t enters the code product as an f16 (relative error <= 2^-11), so
    |d o_c| <= 2^-11 * sum_t w_t s_t c_t,c with w the softmax weights.  Float64
    attention over the exported cache (no pre-RoPE keys)."""
    assert not w.pre_rope
    a = cache.export()
    n_q, r = cache.length()
    D, G, HG = w.D, w.G, w.H_q // w.H_kv
    q = _vals(q_bits, w.dtype)
    bound = np.zeros((w.B, w.H_q, D))
    for s in range(w.B * w.H_kv):
        b, hk = divmod(s, w.H_kv)
        sK = np.repeat(_vals(a["sK"][s], "fp16"), G, axis=0)[:n_q]
        zK = np.repeat(_vals(a["zK"][s], "fp16"), G, axis=0)[:n_q]
        keys = np.concatenate([a["codesK"][s] * sK + zK, _vals(a["resK"][s], w.dtype)])
        sV = np.repeat(_vals(a["sV"][s], "fp16"), G, axis=1)       # [n_q, D]
        for g in range(HG):
            h = hk * HG + g
            sc = keys @ q[b, h] / np.sqrt(D)
            p = np.exp(sc - sc.max())
            p /= p.sum()
            bound[b, h] = 2.0 ** -11 * (p[:n_q, None] * sV * a["codesV"][s]).sum(axis=0)
    return bound
