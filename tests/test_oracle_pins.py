"""Pins for the CPU oracle: facts fixed by the KIVI pages and by mathematics.

Each test ties the oracle to something other than itself: the byte accounting
printed on the Llama-2-13B record, numpy's fp16 conversion, the nearest-level
characterisation of the code, lossless grids where the quantized cache equals
the raw cache (so attention reduces to textbook softmax attention computed with
numpy), RoPE as multiplication by a unit complex number, and the page's
statement that per-channel key grouping beats per-token grouping on keys with
outlier channels.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from bit_asymmetric_kv_prefill_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def to_bits(x, dtype):
    t = torch.from_numpy(np.asarray(x, np.float32))
    t = t.to(torch.bfloat16 if dtype == oracle.DTYPE_BF16 else torch.float16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def from_bits(b, dtype):
    t = torch.from_numpy(np.ascontiguousarray(b).view(np.int16))
    t = t.view(torch.bfloat16 if dtype == oracle.DTYPE_BF16 else torch.float16)
    return t.float().numpy().astype(np.float64)


def f16(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def attn_np(q, K, V):
    """Textbook softmax attention in float64 (numpy): q [HG,D], K/V [T,D]."""
    D = q.shape[1]
    s = K @ q.T / math.sqrt(D)
    s = s - s.max(axis=0, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=0, keepdims=True)
    return p.T @ V


def rope_np(x, pos, theta):
    """RoPE as a complex rotation of (x_i, x_{i+D/2}) by fp32(pos*inv_freq_i)."""
    D = x.shape[-1]
    inv = np.array([np.float32(theta ** (-2.0 * i / D)) for i in range(D // 2)], np.float32)
    ang = (np.float32(pos) * inv).astype(np.float64)
    z = (x[..., :D // 2] + 1j * x[..., D // 2:]) * np.exp(1j * ang)
    return np.concatenate([z.real, z.imag], axis=-1)


# ---- byte accounting (record "KV bytes basis") -------------------------------

def test_kv_bytes_match_printed_record():
    g = json.load(open(os.path.join(GOLDEN, "kv_bytes_llama2_13b.json")))
    i = g["inputs"]
    got = oracle.kv_bytes(i["layers"], i["kv_heads"], i["head_dim"], i["R"], i["context"],
                          i["bits"], i["dtype_bytes"], i["G"])
    for k, v in g["printed"].items():
        assert got[k] == pytest.approx(v, rel=1e-12, abs=0), k


def test_kv_bytes_metadata_equals_the_scale_zero_entries_of_a_cache():
    # The metadata figure (which the record leaves out) is the fp16 scale and
    # zero of every group: count the entries an oracle cache of one layer
    # holds for a 4,096-token capacity (keys: one pair per channel per G
    # tokens; values: one pair per G channels per token), 2 bytes each.
    for heads, D, G, T in ((40, 128, 32, 4096), (8, 64, 32, 1024), (3, 128, 64, 640)):
        c = oracle.OracleCache(1, heads, D, G, 2 * G, oracle.DTYPE_BF16, T)
        entries = c.sK.size + c.zK.size + c.sV.size + c.zV.size
        per_token_layer = 2 * entries / T
        for layers in (1, 40):
            got = oracle.kv_bytes(layers, heads, D, 2 * G, T, G=G)["metadata_per_token"]
            assert got == layers * per_token_layer
    assert oracle.kv_bytes(40, 40, 128, 128, 4096)["metadata_per_token"] == 51200


def test_kv_bytes_falls_toward_8x_with_context():
    # The record notes the reduction falls toward 8x only as context grows.
    r = [oracle.kv_bytes(40, 40, 128, 128, c)["reduction"] for c in (4096, 65536, 1 << 24)]
    assert r[0] < r[1] < r[2] < 8.0 and r[2] > 7.99


# ---- scalar conversion --------------------------------------------------------

def test_fp16_rounding_matches_numpy():
    rng = np.random.default_rng(0)
    vals = [rng.standard_normal(3000) * s for s in (1e-7, 1e-4, 1.0, 300.0, 3e4)]
    # exact halfway points between neighbouring fp16 values, both parities
    h = np.arange(0x0001, 0x7bff, 97, dtype=np.uint16).view(np.float16).astype(np.float32)
    h2 = np.arange(0x0002, 0x7c00, 97, dtype=np.uint16).view(np.float16).astype(np.float32)
    mids = ((h.astype(np.float64) + h2.astype(np.float64)) / 2).astype(np.float32)
    edges = np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, -65520.0, 6.1035156e-05,
                      5.9604645e-08, 2.9802322e-08, 2.9802326e-08, 1e-9], np.float32)
    x = np.concatenate(vals + [mids, -mids, edges]).astype(np.float32)
    ours = oracle.float_to_f16(x)
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    np.testing.assert_array_equal(ours, ref)


# ---- the group code -----------------------------------------------------------

def _random_groups(n_groups=400, G=32, seed=1):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n_groups):
        kind = i % 4
        if kind == 0:
            x = rng.standard_normal(G)
        elif kind == 1:
            x = rng.standard_normal(G) * 0.445
            x[rng.integers(G)] *= 1000
        elif kind == 2:
            x = rng.uniform(-3, 7, G) * 10.0 ** rng.integers(-3, 4)
        else:
            x = rng.standard_normal(G) + 50.0
        out.append(torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).float().numpy())
    return out


def test_code_is_nearest_level():
    """code = argmin_c |x - (z + c s)| over c in {0..3} (ties to the even code),
    wherever the rounded division cannot flip the choice."""
    checked = 0
    for x in _random_groups():
        c, sb, zb = oracle.quant_group(x)
        s, z = f16(sb), f16(zb)
        assert s > 0
        lv = z + s * np.arange(4)
        dist = np.abs(x[:, None].astype(np.float64) - lv[None, :])
        order = np.argsort(dist, axis=1, kind="stable")
        best, second = order[:, 0], order[:, 1]
        gap = dist[np.arange(len(x)), second] - dist[np.arange(len(x)), best]
        clear = gap > 1e-5 * s
        assert np.array_equal(c[clear], best[clear])
        checked += clear.sum()
    assert checked > 10000


def test_group_invariants():
    for x in _random_groups(seed=2):
        c, sb, zb = oracle.quant_group(x)
        s, z = f16(sb), f16(zb)
        mn, mx = float(x.min()), float(x.max())
        assert c.min() >= 0 and c.max() <= 3
        s32 = np.float32(np.float32(mx) - np.float32(mn)) / np.float32(3.0)
        xhat = z + c * s
        bound = s / 2 + 3 * abs(float(s32) - s) + abs(mn - z) + 1e-6 * np.abs(x)
        assert np.all(np.abs(x - xhat) <= bound)
        # a normal-range group uses both extreme codes, and its minimum
        # (fp16-representable here) dequantizes exactly
        if s > 1e-3 and np.float16(mn) == mn:
            assert c[np.argmin(x)] == 0 and z == mn
            assert c[np.argmax(x)] == 3


@pytest.mark.parametrize("e", [-10, -3, 0, 2, 5])
def test_lossless_grid_group(e):
    rng = np.random.default_rng(e + 20)
    for _ in range(50):
        m = int(rng.integers(-60, 60))
        k = rng.integers(0, 4, 32)
        k[rng.integers(32)] = 0
        k[rng.integers(32)] = 3
        k[0] = 3 if k[0] == 0 and (k == 3).sum() == 0 else k[0]
        x = ((m + k) * 2.0 ** e).astype(np.float32)
        c, sb, zb = oracle.quant_group(x)
        assert np.array_equal(c, k)
        assert f16(sb) == 2.0 ** e and f16(zb) == m * 2.0 ** e
        np.testing.assert_array_equal(f16(zb) + c * f16(sb), x)


def test_rint_half_to_even():
    x = np.array([0.0, 3.0, 0.5, 1.5, 2.5, 1.0, 2.0, 0.49, 2.51] + [1.0] * 23, np.float32)
    c, sb, zb = oracle.quant_group(x)
    assert f16(sb) == 1.0 and f16(zb) == 0.0
    assert list(c[:9]) == [0, 3, 0, 2, 2, 1, 2, 0, 3]


def test_constant_and_signed_zero_groups():
    c, sb, zb = oracle.quant_group(np.full(32, 1.25, np.float32))
    assert sb == 0 and f16(zb) == 1.25 and not c.any()
    z = np.zeros(32, np.float32)
    z[::2] = -0.0
    c, sb, zb = oracle.quant_group(z)
    assert sb == 0 and zb == 0 and not c.any()
    c, sb, zb = oracle.quant_group(np.full(32, -0.0, np.float32))
    assert sb == 0 and zb == 0


# ---- axes: keys per channel, values per token ----------------------------------

def test_per_channel_keys_beat_per_token_keys_with_outlier_channels():
    """KIVI article, paragraph 2: per-channel key grouping isolates fixed outlier
    channels and lowers key reconstruction error."""
    w = synth.WORKLOADS["tiny"]
    K, V = synth.prefill_inputs(w, seed=0)
    dt = oracle.DTYPE_F16
    kb = synth.bits(K)
    c = oracle.OracleCache(w.B, w.H_kv, w.D, w.G, w.R, dt, w.T)
    c.prefill(kb, synth.bits(V))
    nq = c.n_q
    G = w.G
    Kf = from_bits(kb, dt)[:, :, :nq]
    sK = f16(c.sK[:, :, :nq // G]).repeat(G, axis=2)
    zK = f16(c.zK[:, :, :nq // G]).repeat(G, axis=2)
    normal = np.ones(w.D, bool)
    normal[list(w.outlier_channels)] = False
    deq_c = c.codesK[:, :, :nq] * sK + zK
    err_channel = np.linalg.norm(Kf - deq_c)
    err_channel_normal = np.linalg.norm((Kf - deq_c)[..., normal])
    # the same keys grouped per token (the value rule applied to keys)
    L = oracle.lib()
    deq_t = np.zeros_like(Kf)
    for h in range(w.H_kv):
        for t in range(nq):
            row = np.ascontiguousarray(kb[0, h, t])
            codes = np.zeros(w.D, np.uint8)
            s = np.zeros(w.D // G, np.uint16)
            z = np.zeros(w.D // G, np.uint16)
            L.oracle_quant_v_token(oracle._ptr(row, oracle.ctypes.c_uint16), w.D, G, dt,
                                   oracle._ptr(codes, oracle.ctypes.c_uint8),
                                   oracle._ptr(s, oracle.ctypes.c_uint16),
                                   oracle._ptr(z, oracle.ctypes.c_uint16))
            deq_t[0, h, t] = codes * f16(s).repeat(G) + f16(z).repeat(G)
    err_token = np.linalg.norm(Kf - deq_t)
    err_token_normal = np.linalg.norm((Kf - deq_t)[..., normal])
    assert err_channel < err_token
    # isolating the outlier channels protects every other channel
    assert err_channel_normal < 0.1 * err_token_normal
    # the outlier channels carry scales ~50x the others
    s_all = f16(c.sK[0, 0, :nq // G])
    assert s_all[:, 3].mean() > 20 * np.median(s_all)


# ---- residual split and flush ---------------------------------------------------

def test_split_counts():
    assert oracle.split(256, 128) == (128, 128)      # 128 quantized + 128 residual
    assert oracle.split(4096, 128) == (3968, 128)
    assert oracle.split(128, 128) == (0, 128)
    assert oracle.split(129, 128) == (128, 1)
    assert oracle.split(1, 128) == (0, 1)
    assert oracle.split(32768, 128) == (32640, 128)


def _lossless_kv(B, H, T, D, G, dtype, seed):
    """K grouped per (G tokens, channel) and V per (token, G channels) on exact
    grids z + k 2^e, with 0 and 3 present in every group."""
    rng = np.random.default_rng(seed)
    K = np.zeros((B, H, T, D))
    V = np.zeros((B, H, T, D))
    for b in range(B):
        for h in range(H):
            for g in range(T // G):
                for d in range(D):
                    e = int(rng.integers(-4, 2))
                    m = int(rng.integers(-40, 40))
                    k = rng.integers(0, 4, G)
                    k[0], k[1] = 0, 3
                    rng.shuffle(k)
                    K[b, h, g * G:(g + 1) * G, d] = (m + k) * 2.0 ** e
            for t in range(T):
                for j in range(D // G):
                    e = int(rng.integers(-4, 2))
                    m = int(rng.integers(-40, 40))
                    k = rng.integers(0, 4, G)
                    k[0], k[1] = 0, 3
                    rng.shuffle(k)
                    V[b, h, t, j * G:(j + 1) * G] = (m + k) * 2.0 ** e
    Kb, Vb = to_bits(K, dtype), to_bits(V, dtype)
    assert np.array_equal(from_bits(Kb, dtype), K) and np.array_equal(from_bits(Vb, dtype), V)
    return Kb, Vb


def test_flush_schedule():
    c = oracle.OracleCache(1, 1, 32, 32, 64, oracle.DTYPE_BF16, 64 * 5 + 200)
    K, V = _lossless_kv(1, 1, 64 * 4, 32, 32, oracle.DTYPE_BF16, 3)
    c.prefill(K, V)
    assert (c.n_q, c.r) == (192, 64)
    seen = []
    for s in range(1, 131):
        c.append(K[:, :, s % 64], V[:, :, s % 64])
        seen.append((c.n_q, c.r))
    assert seen[0] == (256, 1)            # step 1 flushes the full residual
    assert seen[63] == (256, 64)
    assert seen[64] == (320, 1)           # step 65 = R + 1 flushes again
    assert seen[129] == (384, 2)


def test_streaming_equals_batch_prefill():
    w = synth.scaled(synth.WORKLOADS["tiny"], T=160, R=64)
    Kall, Vall = synth.prefill_inputs(w, seed=5, T=160 + 100)
    kb, vb = synth.bits(Kall), synth.bits(Vall)
    dt = oracle.DTYPE_F16
    a = oracle.OracleCache(w.B, w.H_kv, w.D, w.G, w.R, dt, 260)
    a.prefill(kb[:, :, :160], vb[:, :, :160])
    for t in range(160, 260):
        a.append(kb[:, :, t], vb[:, :, t])
    b = oracle.OracleCache(w.B, w.H_kv, w.D, w.G, w.R, dt, 260)
    b.prefill(kb, vb)
    n = min(a.n_q, b.n_q)
    assert n >= 192
    qa, qb = a.quantized(), b.quantized()
    for key in ("codesK", "codesV", "sV", "zV"):
        assert np.array_equal(qa[key][:, :, :n], qb[key][:, :, :n]), key
    for key in ("sK", "zK"):
        assert np.array_equal(qa[key][:, :, :n // w.G], qb[key][:, :, :n // w.G]), key
    assert a.n_q + a.r == b.n_q + b.r == 260


# ---- attention ------------------------------------------------------------------

@pytest.mark.parametrize("dtype", [oracle.DTYPE_F16, oracle.DTYPE_BF16])
def test_residual_only_cache_is_textbook_attention(dtype):
    rng = np.random.default_rng(11)
    B, H, HG, T, D = 2, 2, 2, 100, 64
    K = to_bits(rng.standard_normal((B, H, T, D)) * 3, dtype)
    V = to_bits(rng.standard_normal((B, H, T, D)), dtype)
    q = to_bits(rng.standard_normal((B, H * HG, D)), dtype)
    c = oracle.OracleCache(B, H, D, 32, 128, dtype, 200)
    c.prefill(K, V)
    assert c.n_q == 0 and c.r == T
    out = c.decode(q)
    for b in range(B):
        for hq in range(H * HG):
            h = hq // HG
            ref = attn_np(from_bits(q[b, hq:hq + 1], dtype), from_bits(K[b, h], dtype),
                          from_bits(V[b, h], dtype))
            np.testing.assert_allclose(out[b, hq], ref[0], rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("HG", [1, 2])
def test_lossless_cache_is_textbook_attention(HG):
    dt = oracle.DTYPE_BF16
    B, H, T, D, G, R = 1, 2, 32 * 5 + 7, 64, 32, 64
    K, V = _lossless_kv(B, H, 192, D, G, dt, 7 + HG)
    K, V = K[:, :, :T], V[:, :, :T]
    rng = np.random.default_rng(HG)
    q = to_bits(rng.standard_normal((B, H * HG, D)), dt)
    c = oracle.OracleCache(B, H, D, G, R, dt, T)
    c.prefill(K, V)
    assert c.n_q == 128 and c.r == T - 128
    out = c.decode(q)
    for hq in range(H * HG):
        h = hq // HG   # contiguous GQA groups
        ref = attn_np(from_bits(q[0, hq:hq + 1], dt), from_bits(K[0, h], dt), from_bits(V[0, h], dt))
        np.testing.assert_allclose(out[0, hq], ref[0], rtol=1e-5, atol=1e-6)
    # and the wrong head mapping would be visibly different
    if HG == 2:
        wrong = attn_np(from_bits(q[0, 1:2], dt), from_bits(K[0, 1], dt), from_bits(V[0, 1], dt))
        assert np.abs(out[0, 1] - wrong[0]).max() > 1e-3


def test_constant_values_give_that_constant():
    dt = oracle.DTYPE_F16
    rng = np.random.default_rng(3)
    B, H, T, D = 1, 1, 300, 64
    K = to_bits(rng.standard_normal((B, H, T, D)) * 4, dt)
    V = to_bits(np.full((B, H, T, D), 0.375), dt)
    q = to_bits(rng.standard_normal((B, H, D)) * 3, dt)
    c = oracle.OracleCache(B, H, D, 32, 128, dt, T)
    c.prefill(K, V)
    out = c.decode(q)
    np.testing.assert_allclose(out, 0.375, rtol=0, atol=1e-7)


# ---- RoPE -----------------------------------------------------------------------

def test_rope_is_complex_rotation():
    rng = np.random.default_rng(9)
    for D in (64, 128):
        for pos in (0, 1, 7, 31, 4096, 131071):
            x = rng.standard_normal(D)
            got = oracle.rope_row(x, pos, 10000.0)
            np.testing.assert_allclose(got, rope_np(x, pos, 10000.0), rtol=1e-12, atol=1e-12)
            # norm of every rotated pair is preserved
            n0 = x[:D // 2] ** 2 + x[D // 2:] ** 2
            n1 = got[:D // 2] ** 2 + got[D // 2:] ** 2
            np.testing.assert_allclose(n0, n1, rtol=1e-12)
    x = rng.standard_normal(64)
    np.testing.assert_array_equal(oracle.rope_row(x, 0, 10000.0), x)


def test_pre_rope_decode_rotates_keys_at_absolute_positions():
    dt = oracle.DTYPE_BF16
    B, H, HG, T, D, G, R = 1, 1, 2, 32 * 4 + 9, 64, 32, 64
    K, V = _lossless_kv(B, H, 160, D, G, dt, 21)
    K, V = K[:, :, :T], V[:, :, :T]
    rng = np.random.default_rng(4)
    q = to_bits(rng.standard_normal((B, H * HG, D)), dt)
    c = oracle.OracleCache(B, H, D, G, R, dt, T, pre_rope=True, rope_theta=10000.0)
    c.prefill(K, V)
    assert c.n_q == 128 and c.r == 9
    out = c.decode(q)
    Kr = np.stack([rope_np(from_bits(K[0, 0, t], dt), t, 10000.0) for t in range(T)])
    ref = attn_np(from_bits(q[0], dt), Kr, from_bits(V[0, 0], dt))
    np.testing.assert_allclose(out[0], ref, rtol=1e-5, atol=1e-6)
    # rotating with positions relative to the residual start would differ
    Kbad = Kr.copy()
    for i in range(9):
        Kbad[128 + i] = rope_np(from_bits(K[0, 0, 128 + i], dt), i, 10000.0)
    bad = attn_np(from_bits(q[0], dt), Kbad, from_bits(V[0, 0], dt))
    assert np.abs(bad - ref).max() > 1e-4


# ---- per-sequence lengths in one batch ------------------------------------------

def test_ragged_batch_is_independent_sequences():
    """A batch whose elements have their own lengths (prefill T_b, then common
    appends that flush each residual at its own step) holds, element by element,
    exactly the store and the attention of a one-element cache of that length."""
    w = synth.scaled(synth.WORKLOADS["tiny"], B=3, H_q=4, H_kv=2, T=300)
    dt = oracle.DTYPE_F16
    K, V = synth.prefill_inputs(w, seed=4)
    kb, vb = synth.bits(K), synth.bits(V)
    lengths = [50, 300, 129]
    steps = 140
    c = oracle.OracleCache(w.B, w.H_kv, w.D, w.G, w.R, dt, 300 + steps)
    c.prefill(kb, vb, lengths=lengths)
    singles = []
    for b, T_b in enumerate(lengths):
        s = oracle.OracleCache(1, w.H_kv, w.D, w.G, w.R, dt, 300 + steps)
        s.prefill(kb[b:b + 1, :, :T_b], vb[b:b + 1, :, :T_b])
        singles.append(s)
    assert list(c.nqb) == [0, 256, 128] and list(c.rb) == [50, 44, 1]
    with pytest.raises(ValueError):
        c.n_q
    for step in range(1, steps + 1):
        k, v, q = (synth.bits(t) for t in synth.step_inputs(w, step, seed=4))
        c.append(k, v)
        for b, s in enumerate(singles):
            s.append(k[b:b + 1], v[b:b + 1])
        if step in (1, 78, 79, 84, 85, 127, 128, 140):
            out = c.decode(q)
            for b, s in enumerate(singles):
                assert (c.nqb[b], c.rb[b]) == (s.n_q, s.r)
                np.testing.assert_array_equal(out[b:b + 1], s.decode(q[b:b + 1]))
    for b, s in enumerate(singles):
        n = s.n_q
        np.testing.assert_array_equal(c.codesK[b, :, :n], s.codesK[0, :, :n])
        np.testing.assert_array_equal(c.sV[b, :, :n], s.sV[0, :, :n])
        np.testing.assert_array_equal(c.resK[b, :, :s.r], s.resK[0, :, :s.r])


def test_ragged_lossless_cache_is_textbook_attention_per_sequence():
    dt = oracle.DTYPE_BF16
    B, H, D, G, R = 3, 2, 64, 32, 64
    K, V = _lossless_kv(B, H, 192, D, G, dt, 31)
    lengths = [7, 192, 100]
    rng = np.random.default_rng(5)
    q = to_bits(rng.standard_normal((B, H, D)), dt)
    c = oracle.OracleCache(B, H, D, G, R, dt, 192)
    c.prefill(K, V, lengths=lengths)
    out = c.decode(q)
    for b, T_b in enumerate(lengths):
        for h in range(H):
            ref = attn_np(from_bits(q[b, h:h + 1], dt), from_bits(K[b, h, :T_b], dt),
                          from_bits(V[b, h, :T_b], dt))
            np.testing.assert_allclose(out[b, h], ref[0], rtol=1e-5, atol=1e-6)
    with pytest.raises(ValueError):
        c.prefill(K, V, lengths=[0, 5, 5])
    with pytest.raises(ValueError):
        c.prefill(K, V, lengths=[5, 193, 5])
