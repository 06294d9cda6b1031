"""Pins for the oracle's diagnostic grouping modes (fake quantization).

The generic group quantizer is tied to the 2-bit KIVI codec (itself pinned in
test_oracle_pins.py), to lossless integer grids at every width, to the
nearest-level characterisation of rounding, to the transpose symmetry between
the two grouping axes, and to the error bounds of round-to-nearest.  The error
measures are tied to cases whose answer is known (a lossless cache, a single
attended token), and the KIVI article's directional claims are checked where
the synthetic workloads carry their cause (fixed outlier key channels).
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import diag
from bit_asymmetric_kv_prefill_b200 import synth

PC, PT = oracle.AXIS_PER_CHANNEL, oracle.AXIS_PER_TOKEN


def f16(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def mixed_matrix(T, D, seed):
    """bf16-representable [T, D] matrix with normal, outlier and offset groups."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, D))
    x[:, rng.integers(D, size=3)] *= 300.0
    x[rng.integers(T, size=4)] += 40.0
    x[:, :4] *= 1e-3
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).float().numpy()


# ---- 2 bits, asymmetric: the KIVI codec ----------------------------------------

@pytest.mark.parametrize("dtype", [oracle.DTYPE_F16, oracle.DTYPE_BF16])
def test_two_bit_asymmetric_modes_are_the_kivi_codec(dtype):
    """Per channel = the key rule, per token = the value rule, dequantized as
    code*scale + zero rounded once to fp32."""
    w = synth.scaled(synth.WORKLOADS["tiny"], dtype="bf16" if dtype == oracle.DTYPE_BF16 else "fp16",
                     T=129)
    K, V = synth.prefill_inputs(w, seed=3)
    c = oracle.OracleCache(w.B, w.H_kv, w.D, w.G, w.R, dtype, w.T)
    c.prefill(synth.bits(K), synth.bits(V))
    nq, G = c.n_q, w.G
    assert nq == 128
    sK = f16(c.sK[0, :, :nq // G]).repeat(G, axis=1)
    zK = f16(c.zK[0, :, :nq // G]).repeat(G, axis=1)
    sV = f16(c.sV[0, :, :nq]).repeat(G, axis=2)
    zV = f16(c.zV[0, :, :nq]).repeat(G, axis=2)
    k_codec = (c.codesK[0, :, :nq] * sK + zK).astype(np.float32)
    v_codec = (c.codesV[0, :, :nq] * sV + zV).astype(np.float32)
    Kf = K.float().numpy()[0, :, :nq]
    Vf = V.float().numpy()[0, :, :nq]
    np.testing.assert_array_equal(oracle.fake_quant(Kf, PC, G, 2), k_codec)
    np.testing.assert_array_equal(oracle.fake_quant(Vf, PT, G, 2), v_codec)
    _, codes = oracle.fake_quant(Kf, PC, G, 2, codes=True)
    np.testing.assert_array_equal(codes, c.codesK[0, :, :nq])


@pytest.mark.parametrize("bits,sym", [(2, False), (3, False), (8, False), (2, True), (4, True)])
def test_axes_are_transposes(bits, sym):
    x = mixed_matrix(64, 96, seed=bits + 10 * sym)
    a = oracle.fake_quant(x, PC, 32, bits, sym)
    b = oracle.fake_quant(np.ascontiguousarray(x.T), PT, 32, bits, sym).T
    np.testing.assert_array_equal(a, b)


# ---- lossless grids and closed forms ----------------------------------------------

@pytest.mark.parametrize("bits", range(1, 9))
@pytest.mark.parametrize("axis", [PC, PT])
def test_asymmetric_integer_grid_is_lossless(bits, axis):
    """Values m*2^e + k*2^e with k spanning 0..2^bits-1 in every group come back
    exactly, with codes k."""
    L = (1 << bits) - 1
    rng = np.random.default_rng(bits)
    G, T, D = 32, 64, 64
    k = rng.integers(0, L + 1, (T, D))
    e = int(rng.integers(-6, 3))
    m = int(rng.integers(-20, 20))
    if axis == PC:
        k[0::G, :] = 0
        k[1::G, :] = L
    else:
        k[:, 0::G] = 0
        k[:, 1::G] = L
    x = ((m + k) * 2.0 ** e).astype(np.float32)
    xh, codes = oracle.fake_quant(x, axis, G, bits, codes=True)
    np.testing.assert_array_equal(codes, k)
    np.testing.assert_array_equal(xh, x)


@pytest.mark.parametrize("bits", range(2, 9))
def test_symmetric_integer_grid_is_lossless(bits):
    L = (1 << (bits - 1)) - 1
    rng = np.random.default_rng(100 + bits)
    G = 16
    k = rng.integers(-L, L + 1, (8, 64))
    k[:, 0::G] = L
    e = int(rng.integers(-5, 4))
    x = (k * 2.0 ** e).astype(np.float32)
    xh, codes = oracle.fake_quant(x, PT, G, bits, sym=True, codes=True)
    np.testing.assert_array_equal(codes, k)
    np.testing.assert_array_equal(xh, x)


def test_two_bit_symmetric_levels():
    """Two-bit absmax: levels {-a, 0, a}, rounding half to even at +-a/2."""
    x = np.array([[4.0, -4.0, 2.0, -2.0, 1.9, -2.1, 0.0, 6.0 / 2 + 1e-3] + [0.5] * 8], np.float32)
    x[0, 7] = 4.0 * 0.75
    xh, codes = oracle.fake_quant(x, PT, 16, 2, sym=True, codes=True)
    assert list(codes[0, :8]) == [1, -1, 0, 0, 0, -1, 0, 1]
    assert list(xh[0, :8]) == [4.0, -4.0, 0.0, 0.0, 0.0, -4.0, 0.0, 4.0]


def test_constant_groups():
    x = np.full((32, 8), 1.25, np.float32)
    x[:, 1] = -3.0
    x[:, 2] = 0.0
    np.testing.assert_array_equal(oracle.fake_quant(x, PC, 32, 2), x)
    # symmetric: |c| is the absmax, so c maps to +-L*scale with scale = fp16(|c|/L)
    xh = oracle.fake_quant(x, PC, 32, 3, sym=True)
    s = np.float16(np.float32(1.25) / np.float32(3.0)).astype(np.float32)
    np.testing.assert_array_equal(xh[:, 0], np.float32(3.0) * s)
    assert not xh[:, 2].any()


# ---- rounding: nearest level and error bounds -----------------------------------------

@pytest.mark.parametrize("bits", [1, 2, 3, 4, 8])
def test_asymmetric_code_is_nearest_level(bits):
    L = (1 << bits) - 1
    x = mixed_matrix(32, 256, seed=bits)
    xh, codes = oracle.fake_quant(x, PC, 32, bits, codes=True)
    assert codes.min() >= 0 and codes.max() <= L
    checked = 0
    for d in range(x.shape[1]):
        col = x[:, d].astype(np.float64)
        s = float(np.float16(np.float32(np.float32(col.max()) - np.float32(col.min())) / np.float32(L)))
        z = float(np.float16(np.float32(col.min())))
        if s == 0:
            assert not codes[:, d].any()
            continue
        lv = z + s * np.arange(L + 1)
        dist = np.abs(col[:, None] - lv[None, :])
        order = np.argsort(dist, axis=1, kind="stable")
        gap = dist[np.arange(32), order[:, 1]] - dist[np.arange(32), order[:, 0]]
        clear = gap > 1e-5 * s
        np.testing.assert_array_equal(codes[clear, d], order[clear, 0])
        np.testing.assert_array_equal(xh[:, d], (z + s * codes[:, d]).astype(np.float32))
        checked += clear.sum()
    assert checked > 4000


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_symmetric_error_bound(bits):
    L = (1 << (bits - 1)) - 1
    x = mixed_matrix(16, 512, seed=50 + bits)
    xh, codes = oracle.fake_quant(x, PT, 32, bits, sym=True, codes=True)
    assert codes.min() >= -L - 1 and codes.max() <= L
    g = x.reshape(16, 16, 32)
    amax = np.abs(g).max(axis=2, keepdims=True).astype(np.float64)
    s = (amax / L).astype(np.float16).astype(np.float64)
    err = np.abs(g - xh.reshape(16, 16, 32))
    assert np.all(err <= s / 2 + amax * 2.0 ** -10 + 1e-30)


def test_rejects_unsupported_arguments():
    x = np.zeros((32, 64), np.float32)
    for kw in (dict(axis=PC, G=48), dict(axis=PT, G=48), dict(axis=2, G=32),
               dict(axis=PT, G=32, bits=9), dict(axis=PT, G=32, bits=1, sym=True),
               dict(axis=PT, G=32, bits=0)):
        with pytest.raises(ValueError):
            oracle.fake_quant(x, **kw)


# ---- error measures --------------------------------------------------------------

def test_attention_measure_closed_forms():
    rng = np.random.default_rng(0)
    q = rng.standard_normal((2, 3, 16))
    K = rng.standard_normal((2, 40, 16))
    V = np.ones((2, 40, 16)) * 2.5
    np.testing.assert_allclose(diag.attention(q, K, V), 2.5, rtol=1e-14)
    K[:, 7] = q[:, 0] * 1000.0     # query 0 attends to token 7 alone
    V = rng.standard_normal((2, 40, 16))
    np.testing.assert_allclose(diag.attention(q, K, V)[:, 0], V[:, 7], rtol=1e-12)


def test_lossless_cache_has_zero_error():
    rng = np.random.default_rng(1)
    k = rng.integers(0, 4, (2, 64, 64))
    k[:, 0::32, :] = 0
    k[:, 1::32, :] = 3
    k[:, :, 0::32] = 0
    k[:, :, 1::32] = 3
    x = (k * 0.5 - 1.0).astype(np.float32)
    q = rng.standard_normal((2, 4, 64))
    e = diag.errors(x, x, q, "kivi")
    assert e == dict(key=0.0, value=0.0, attn=0.0)


def _recipe(name, T=512, heads=4, M=8):
    w = synth.scaled(synth.WORKLOADS[name], B=1, H_kv=heads, H_q=heads, T=T)
    K, V = synth.prefill_inputs(w, seed=0)
    q = np.stack([synth.step_inputs(w, s)[2].float().numpy()[0] for s in range(M)], 1)
    return K.float().numpy()[0], V.float().numpy()[0], q


@pytest.mark.parametrize("name", ["tiny", "llama2_7b_layer"])
def test_per_channel_keys_beat_per_token_keys_at_the_output(name):
    """KIVI article, paragraph 2: with fixed outlier key channels, per-channel
    key grouping gives the smaller attention-output error."""
    K, V, q = _recipe(name, heads=2 if name == "tiny" else 4)
    kivi = diag.errors(K, V, q, "kivi")
    per_token = diag.errors(K, V, q, "k_per_token")
    assert kivi["attn"] < per_token["attn"]
    assert kivi["value"] == per_token["value"]
    # per-channel groups keep the outliers' range out of every other channel
    normal = K.std(axis=1) < 10.0
    err_c = np.abs(K - oracle.fake_quant(K, PC))
    err_t = np.abs(K - oracle.fake_quant(K, PT))
    assert np.linalg.norm(err_c * normal[:, None, :]) < 0.1 * np.linalg.norm(err_t * normal[:, None, :])


@pytest.mark.parametrize("name", ["tiny", "llama2_7b_layer", "llama2_13b_cache"])
def test_naive_symmetric_values_lose_to_asymmetric(name):
    """Record kv-efficiency/kivi-2bit-llama2-13b-mha-4k, "Quality": naive
    symmetric 2-bit is the failing baseline.  On outlier-free N(0,1) values,
    three symmetric levels reconstruct worse than four asymmetric ones."""
    K, V, q = _recipe(name, heads=2 if name == "tiny" else 4)
    kivi = diag.errors(K, V, q, "kivi")
    sym = diag.errors(K, V, q, "naive_symmetric")
    assert sym["value"] > 1.3 * kivi["value"]


def test_pre_rope_keys_reconstruct_better_than_post_rope():
    """KVQuant summary, "Pre-RoPE Key Quantization": rotation mixes each outlier
    channel into its partner, so per-channel groups taken after RoPE see wider
    ranges than the same groups taken before it."""
    K, V, q = _recipe("long_context", T=256)
    pre = diag.errors(K, V, q, "kivi", rope="pre")
    post = diag.errors(K, V, q, "kivi", rope="post")
    assert pre["key"] < post["key"]


# ---- dense-and-sparse: one exactly kept element per group ----------------------

@pytest.mark.parametrize("sym,bits", [(False, 2), (False, 4), (True, 2), (True, 3)])
def test_outlier_mode_is_the_plain_code_without_that_element(sym, bits):
    """KVQuant summary, "Per-Vector Dense-and-Sparse Quantization": the group's
    largest-magnitude element is kept exactly and the rest is quantized as a
    group of its own; checked against the plain mode (pinned above) applied to
    the group with that element removed."""
    x = mixed_matrix(40, 33, seed=bits)           # rows are groups of 33
    x[:, 5] = 0.0
    x[3, 7] = x[3, 9] = 1e4                        # equal magnitudes: the first wins
    x[4, 2], x[4, 30] = -7e3, 7e3
    xh, codes = oracle.fake_quant(x, PT, 33, bits, sym, codes=True, outlier=1)
    for t in range(x.shape[0]):
        o = int(np.argmax(np.abs(x[t])))           # numpy takes the first maximum too
        assert codes[t, o] == oracle.OUTLIER_CODE and xh[t, o] == x[t, o]
        rest = np.delete(x[t], o)[None, :]
        ref, ref_codes = oracle.fake_quant(np.ascontiguousarray(rest), PT, 32, bits, sym, codes=True)
        np.testing.assert_array_equal(np.delete(xh[t], o), ref[0])
        np.testing.assert_array_equal(np.delete(codes[t], o), ref_codes[0])
    assert codes[3, 7] == oracle.OUTLIER_CODE and codes[3, 9] != oracle.OUTLIER_CODE
    assert codes[4, 2] == oracle.OUTLIER_CODE


def test_outlier_mode_axes_and_degenerate_groups():
    x = mixed_matrix(64, 96, seed=77)
    a = oracle.fake_quant(x, PC, 32, 2, outlier=1)
    b = oracle.fake_quant(np.ascontiguousarray(x.T), PT, 32, 2, outlier=1).T
    np.testing.assert_array_equal(a, b)
    # one element: kept exactly; two: the smaller-magnitude one alone is a
    # constant group (zero scale, x_hat = fp16(x))
    np.testing.assert_array_equal(oracle.fake_quant(x, PT, 1, 2, outlier=1), x)
    y = np.array([[3.0, 1.1], [-0.3, 9.0]], np.float32)
    yh = oracle.fake_quant(y, PT, 2, 2, outlier=1)
    np.testing.assert_array_equal(yh, np.array([[3.0, np.float16(1.1)], [np.float16(-0.3), 9.0]],
                                               np.float32))
    with pytest.raises(ValueError):
        oracle.fake_quant(x, PT, 32, 2, outlier=2)


def test_outlier_mode_lossless_grid_with_spikes():
    rng = np.random.default_rng(5)
    k = rng.integers(0, 4, (16, 64))
    k[:, 0::32] = 0
    k[:, 1::32] = 3
    x = (k * 0.25 - 1.0).astype(np.float32)
    x[:, 17] = 5e3
    x[:, 40] = -6e3
    np.testing.assert_array_equal(oracle.fake_quant(x, PT, 32, 2, outlier=1), x)


def test_one_sparse_element_rescues_per_token_keys():
    """Per-token key groups hold about one outlier channel each on the
    fixed-outlier workloads; keeping it exactly removes most of the error of
    the other channels."""
    K, _, _ = _recipe("llama2_7b_layer", heads=2)
    plain = np.linalg.norm(K - oracle.fake_quant(K, PT))
    sparse = np.linalg.norm(K - oracle.fake_quant(K, PT, outlier=1))
    assert sparse < 0.6 * plain


def test_per_token_values_win_when_attended_tokens_have_their_own_magnitude():
    """KIVI article, paragraph 3: per-channel value groups spike the
    attention-output error under sparse attention.  On i.i.d. values both
    groupings tie (the workloads' values); the gap appears once tokens carry
    their own value magnitude and attention concentrates on a few of them, as
    in this constructed case (not one of the workloads): per-channel groups then
    quantize a small-magnitude attended token with the scale of the others."""
    rng = np.random.default_rng(0)
    H, T, D, M = 2, 512, 128, 8
    K = rng.standard_normal((H, T, D)).astype(np.float32)
    sigma = (10.0 ** rng.uniform(-2, 0, (H, T, 1))).astype(np.float32)
    V = (rng.standard_normal((H, T, D)) * sigma).astype(np.float32)
    q = np.zeros((H, M, D))
    for h in range(H):
        for m, t in enumerate(np.argsort(sigma[h, :, 0])[:M]):
            q[h, m] = 3.0 * K[h, t]
    per_token = diag.errors(K, V, q, "kivi")
    per_channel = diag.errors(K, V, q, "v_per_channel")
    assert per_channel["attn"] > 10 * per_token["attn"]
    # reconstruction alone does not show it as strongly
    assert per_channel["value"] < 2 * per_token["value"]


# ---- non-uniform levels (KVQuant's non-uniform quantization, fitted here) --------

UNIFORM4 = [0.0, 1.0 / 3.0, 2.0 / 3.0, 1.0]


def _nearest_level_ref(x, axis, G, levels):
    """Brute force in float64: nearest level on each group's [min, max]."""
    x64 = np.asarray(x, np.float64)
    lev = np.asarray(levels, np.float64)
    out = np.empty_like(x64)
    T, D = x.shape
    groups = ([(slice(g * G, (g + 1) * G), d) for d in range(D) for g in range(T // G)]
              if axis == PC else [(t, slice(j * G, (j + 1) * G)) for t in range(T) for j in range(D // G)])
    for idx in groups:
        v = x64[idx]
        mn, mx = v.min(), v.max()
        if mx == mn:
            out[idx] = mn
            continue
        u = (v - mn) / (mx - mn)
        k = np.argmin(np.abs(u[:, None] - lev[None, :]), axis=1)   # first minimum on ties
        out[idx] = mn + (mx - mn) * lev[k]
    return out.astype(np.float32)


@pytest.mark.parametrize("axis", [PC, PT])
@pytest.mark.parametrize("levels", [UNIFORM4, [0.0, 0.1, 0.35, 0.9], [0.05, 0.5, 0.95],
                                    list(np.linspace(0, 1, 16))])
def test_levels_are_nearest_on_each_group_range(axis, levels):
    x = mixed_matrix(64, 96, seed=len(levels) + axis)
    xh = oracle.fake_quant_levels(x, axis, 32, levels)
    np.testing.assert_array_equal(xh, _nearest_level_ref(x, axis, 32, levels))
    t = oracle.fake_quant_levels(np.ascontiguousarray(x.T), 1 - axis, 32, levels).T
    np.testing.assert_array_equal(xh, t)


def test_levels_ties_constant_groups_and_arguments():
    x = np.array([[0.0, 1.0, 0.25, 0.75] + [0.5] * 4, [2.0] * 8], np.float32)
    xh, codes = oracle.fake_quant_levels(x, PT, 8, [0.0, 0.5, 1.0], codes=True)
    assert list(codes[0, :4]) == [0, 2, 0, 1]          # 0.25 and 0.75 are ties: the lower level
    np.testing.assert_array_equal(xh[1], x[1])
    for bad in ([0.0, 1.5], [0.5], [-0.1, 0.5]):
        with pytest.raises(ValueError):
            oracle.fake_quant_levels(x, PT, 8, bad)


def test_levels_on_their_own_grid_are_lossless_and_fitted_exactly():
    """Groups whose elements sit at normalized positions {0, 0.2, 0.5, 1}: those
    levels reproduce them exactly, and Lloyd's algorithm finds them."""
    rng = np.random.default_rng(3)
    pos = np.array([0.0, 0.2, 0.5, 1.0])
    k = rng.integers(0, 4, (64, 64))
    k[0::32, :] = 0
    k[1::32, :] = 3
    base = rng.integers(-20, 20, (2, 64)).repeat(32, axis=0)
    x = (base + 10.0 * pos[k]).astype(np.float32)
    np.testing.assert_array_equal(oracle.fake_quant_levels(x, PC, 32, pos), x)
    np.testing.assert_allclose(diag.fit_levels(x, PC, 32, 4), pos, atol=1e-12)


def test_fitted_levels_lower_the_error_of_even_levels():
    """Lloyd's iterations never raise the squared error; on normal groups the
    fitted four levels beat evenly spaced ones."""
    K, V, _ = _recipe("llama2_7b_layer", heads=2, T=256)
    for X, axis in ((K, PC), (V, PT)):
        lev = diag.fit_levels(X, axis, 32, 4)
        assert np.all(np.diff(lev) > 0) and lev[0] >= 0 and lev[-1] <= 1
        fitted = np.linalg.norm(X - oracle.fake_quant_levels(X, axis, 32, lev))
        even = np.linalg.norm(X - oracle.fake_quant_levels(X, axis, 32, UNIFORM4))
        assert fitted < 0.95 * even
