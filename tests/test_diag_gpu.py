"""GPU parity of kivi_fake_quant (the diagnostic grouping modes) against the oracle.

Dequantized values must be bit-exact (both sides round the same fp32
operations: IEEE division, rint half to even, one rounding of code*scale +
zero).  The per-matrix squared error rounds each difference to fp32 and sums
squares in fp32 over runs of at most 8 elements: each term carries a relative
error of at most 3 * 2^-24 (difference, square) and each run at most 7 * 2^-24
more, all terms being positive, so it is compared with the exact float64 sum to
a relative 10 * 2^-24 < 1e-6.  Shapes span several chunks of work with
ragged tails; the edge cases are single groups, the smallest row, zero-scale
groups and signed zeros.  At full size (every key and value matrix of one
Llama-2-13B layer cache, 16 x 40 heads x 4096 tokens x 128) sampled matrices
are checked one by one, and the per-matrix errors of all matrices against the
values kernel's own output.
"""
import numpy as np
import pytest
import torch

import oracle
import bit_asymmetric_kv_prefill_b200 as kv
from bit_asymmetric_kv_prefill_b200 import synth

pytestmark = pytest.mark.gpu

PC, PT = kv.AXIS_PER_CHANNEL, kv.AXIS_PER_TOKEN
assert (PC, PT) == (oracle.AXIS_PER_CHANNEL, oracle.AXIS_PER_TOKEN)


def check(x, axis, G, bits, sym, outlier=0):
    """Run the GPU path on x (CUDA, bf16/fp16, [..., T, D]) and compare with the oracle."""
    xh, err = kv.fake_quant(x, axis, G, bits, sym, outlier=outlier)
    torch.cuda.synchronize()
    xf = x.float().cpu().numpy()
    ref = oracle.fake_quant(xf, axis, G, bits, sym, outlier=outlier)
    got = xh.cpu().numpy()
    assert got.view(np.uint32).shape == ref.view(np.uint32).shape
    bad = got.view(np.uint32) != ref.view(np.uint32)
    assert not bad.any(), (f"{bad.sum()} mismatches, first at {np.argwhere(bad)[0]}: "
                           f"{got[bad][0]!r} vs {ref[bad][0]!r}")
    T, D = x.shape[-2:]
    d = (xf.astype(np.float64) - ref.astype(np.float64)).reshape(-1, T * D)
    want = (d * d).sum(axis=1)
    np.testing.assert_allclose(err.cpu().numpy(), want, rtol=1e-6, atol=1e-300)
    return xh, err


def recipe(name, B=1, H=3, T=256, dtype=None, seed=0):
    w = synth.WORKLOADS[name]
    w = synth.scaled(w, B=B, H_kv=H, H_q=H, T=T, **({"dtype": dtype} if dtype else {}))
    K, V = synth.prefill_inputs(w, seed=seed, device="cuda")
    return K, V


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("axis", [PC, PT])
@pytest.mark.parametrize("bits,sym", [(1, False), (2, False), (3, False), (4, False), (8, False),
                                      (2, True), (3, True), (4, True), (8, True)])
def test_modes_match_oracle(dtype, axis, bits, sym):
    K, V = recipe("llama2_7b_layer", H=3, T=352, dtype=dtype, seed=bits)
    check(K, axis, 32, bits, sym)
    check(V, axis, 32, bits, sym)


@pytest.mark.parametrize("G", [8, 16, 64, 128])
@pytest.mark.parametrize("axis", [PC, PT])
def test_group_sizes(G, axis):
    K, _ = recipe("llama2_13b_cache", H=2, T=384, seed=G)
    check(K, axis, G, 2, False)
    check(K, axis, G, 4, True)


def test_per_channel_odd_group_and_narrow_rows():
    g = torch.Generator(device="cuda").manual_seed(5)
    x = (torch.randn((2, 3, 105, 24), generator=g, device="cuda") * 3).to(torch.bfloat16)
    check(x, PC, 7, 2, False)
    check(x, PC, 35, 3, True)
    x8 = torch.randn((5, 40, 8), generator=g, device="cuda").to(torch.float16)
    check(x8, PC, 40, 2, False)
    check(x8, PT, 8, 2, False)


def test_ragged_tails_and_single_groups():
    g = torch.Generator(device="cuda").manual_seed(6)
    for shape in [(1, 1, 8), (1, 32, 64), (3, 1, 256), (7, 33, 40), (2, 1000, 72)]:
        x = torch.randn(shape, generator=g, device="cuda").to(torch.bfloat16)
        check(x, PT, 8, 2, False)
        check(x, PC, shape[1], 2, False)


def test_zero_scale_groups_and_signed_zeros():
    x = torch.zeros((2, 64, 64), dtype=torch.float16, device="cuda")
    x[0, :, :32] = 1.5
    x[0, :32, 32:] = -0.0
    x[1, ::2] = -0.0
    x[1, :, 5] = 2.0
    for axis in (PC, PT):
        for bits, sym in ((2, False), (2, True), (8, True)):
            xh, err = check(x, axis, 32, bits, sym)
    xh, _ = kv.fake_quant(x, PT, 32, 2, False)
    assert not torch.signbit(xh[0, :32, 32:]).any()


def test_error_only_and_values_only():
    K, _ = recipe("llama2_13b_cache", H=4, T=512, seed=9)
    xh, err = kv.fake_quant(K, PC)
    none, err2 = kv.fake_quant(K, PC, values=False)
    xh2, none2 = kv.fake_quant(K, PC, error=False)
    assert none is None and none2 is None
    torch.testing.assert_close(err2, err, rtol=1e-12, atol=0)
    assert torch.equal(xh2, xh)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("axis", [PC, PT])
@pytest.mark.parametrize("bits,sym", [(2, False), (3, False), (2, True), (4, True)])
def test_dense_and_sparse_match_oracle(dtype, axis, bits, sym):
    """One exactly kept element per group; bf16/fp16 data has many ties in |x|,
    which exercise the first-element rule across lanes and rows."""
    K, V = recipe("llama2_7b_layer", H=3, T=352, dtype=dtype, seed=20 + bits)
    check(K, axis, 32, bits, sym, outlier=1)
    check(V, axis, 32, bits, sym, outlier=1)
    H, _ = recipe("llama2_13b_cache", H=2, T=256, dtype=dtype, seed=21)
    check(H, axis, 32, bits, sym, outlier=1)


def test_dense_and_sparse_group_sizes_and_ties():
    g = torch.Generator(device="cuda").manual_seed(9)
    x = (torch.randn((3, 96, 128), generator=g, device="cuda") * 4).round().to(torch.bfloat16)
    x[0, :, 5] = 7.0
    x[0, :, 6] = -7.0
    x[1, 3, :] = -9.0
    for G in (8, 16, 64, 128):
        check(x, PT, G, 2, False, outlier=1)
        check(x, PT, G, 3, True, outlier=1)
    for G in (1, 2, 3, 32, 96):
        check(x, PC, G, 2, False, outlier=1)
        check(x, PC, G, 2, True, outlier=1)


def test_two_bit_modes_are_the_cache_codec():
    """At 2 bits, per-channel keys and per-token values reproduce the cache's
    own quantization (exported from kivi_prefill), dequantized."""
    w = synth.scaled(synth.WORKLOADS["llama2_7b_layer"], B=2, H_kv=2, H_q=2, T=257)
    K, V = synth.prefill_inputs(w, seed=1, device="cuda")
    c = kv.KiviCache(w.B, w.H_kv, w.D, R=w.R, dtype=w.torch_dtype, T_max=w.T)
    c.prefill(K, V)
    e = c.export()
    n_q = c.length()[0]
    f16 = lambda b: torch.from_numpy(b.view(np.float16).astype(np.float32))
    sK = f16(e["sK"]).repeat_interleave(32, dim=1)
    zK = f16(e["zK"]).repeat_interleave(32, dim=1)
    sV = f16(e["sV"]).repeat_interleave(32, dim=2)
    zV = f16(e["zV"]).repeat_interleave(32, dim=2)
    k_deq = (torch.from_numpy(e["codesK"]).double() * sK.double() + zK.double()).float()
    v_deq = (torch.from_numpy(e["codesV"]).double() * sV.double() + zV.double()).float()
    kh, _ = kv.fake_quant(K[:, :, :n_q].contiguous(), PC)
    vh, _ = kv.fake_quant(V[:, :, :n_q].contiguous(), PT)
    assert torch.equal(kh.cpu().reshape(k_deq.shape), k_deq)
    assert torch.equal(vh.cpu().reshape(v_deq.shape), v_deq)


@pytest.mark.parametrize("axis,bits,sym", [(PC, 2, False), (PT, 2, False), (PT, 2, True)])
def test_full_size_llama2_13b_layer_sampled(axis, bits, sym):
    """One Llama-2-13B layer cache (16 x 40 heads, 4096 tokens, head_dim 128,
    heavy-tailed keys): sampled matrices element by element against the oracle,
    every matrix's error against the returned values."""
    w = synth.WORKLOADS["llama2_13b_cache"]
    K, V = synth.prefill_inputs(w, seed=0, device="cuda")
    for X in (K, V):
        xh, err = kv.fake_quant(X, axis, 32, bits, sym)
        d = (X.double() - xh.double()).reshape(-1, w.T * w.D)
        torch.testing.assert_close(err, (d * d).sum(dim=1), rtol=1e-6, atol=0)
        flat = X.reshape(-1, w.T, w.D)
        xh_flat = xh.reshape(-1, w.T, w.D)
        for n in (0, 1, 333, flat.shape[0] - 1):
            ref = oracle.fake_quant(flat[n].float().cpu().numpy(), axis, 32, bits, sym)
            got = xh_flat[n].cpu().numpy()
            assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
        del xh, err, d


# ---- non-uniform levels (kivi_fake_quant_levels) ----------------------------------

def check_levels(x, axis, G, levels):
    """GPU non-uniform levels on x against oracle_fake_quant_levels: x_hat and
    codes bit-exact (both sides evaluate the same IEEE fp64 operations), the
    per-matrix squared error against float64 within summation-order rounding."""
    xh, cc, err = kv.fake_quant_levels(x, axis, G, levels, codes=True)
    torch.cuda.synchronize()
    xf = x.float().cpu().numpy()
    ref, rc = oracle.fake_quant_levels(xf, axis, G, levels, codes=True)
    got = xh.cpu().numpy()
    bad = got.view(np.uint32) != ref.view(np.uint32)
    assert not bad.any(), (f"{bad.sum()} x_hat mismatches, first at {np.argwhere(bad)[0]}: "
                           f"{got[bad][0]!r} vs {ref[bad][0]!r}")
    np.testing.assert_array_equal(cc.cpu().numpy().astype(np.int32), rc)
    T, D = x.shape[-2:]
    d = (xf.astype(np.float64) - ref.astype(np.float64)).reshape(-1, T * D)
    np.testing.assert_allclose(err.cpu().numpy(), (d * d).sum(axis=1), rtol=1e-12, atol=1e-300)


LEVELS = [[0.0, 1 / 3, 2 / 3, 1.0], [0.0, 0.1, 0.35, 0.9], [0.05, 0.5, 0.95], [0.9, 0.1, 0.5, 0.0],
          [0.0, 1.0], list(np.linspace(0.0, 1.0, 16)), list(np.sort(np.random.default_rng(3).random(256)))]


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("axis", [PC, PT])
@pytest.mark.parametrize("li", range(len(LEVELS)), ids=[f"lev{len(l)}-{i}" for i, l in enumerate(LEVELS)])
def test_levels_match_oracle(dtype, axis, li):
    K, V = recipe("llama2_7b_layer", H=3, T=352, dtype=dtype, seed=li)
    for x in (K, V):
        check_levels(x, axis, 32, LEVELS[li])


@pytest.mark.parametrize("axis,G", [(PC, 1), (PC, 7), (PC, 11), (PT, 1), (PT, 3), (PT, 64), (PT, 128)])
def test_levels_group_sizes(axis, G):
    T = 77 if axis == PC else 50
    D = 4 * G if axis == PT else 48
    x = (torch.randn(2, T - T % G if axis == PC else T, D, generator=torch.Generator().manual_seed(G)) * 3)
    check_levels(x.to(torch.bfloat16).cuda(), axis, G, [0.0, 0.2, 0.45, 1.0])


def test_levels_ties_grids_and_constant_groups():
    # values on the level grid come back exactly; points halfway between two
    # levels take the first of them; constant groups keep their value
    g = torch.Generator().manual_seed(5)
    T, D = 64, 32
    lev = [0.0, 0.25, 0.5, 1.0]
    base = torch.randint(-8, 8, (T, D), generator=g).float()
    pick = torch.tensor(lev)[torch.randint(0, 4, (T, D), generator=g)]
    x = base + 8.0 * pick
    x[0:32:2, :] = base[0:32:2, :]                      # each group holds its min ...
    x[1:32:2, :] = base[1:32:2, :] + 8.0                # ... and its max
    x[32:64, 3] = 2.5                                   # constant groups
    x[40, 5] = x[32:64, 5].min() + 0.375 * (x[32:64, 5].max() - x[32:64, 5].min())  # tie 0.25 / 0.5
    for dt in (torch.bfloat16, torch.float16):
        check_levels(x.to(dt).cuda()[None], PC, 32, lev)
        check_levels(x.t().contiguous().to(dt).cuda()[None], PT, 32, lev)


def test_levels_rejects_bad_arguments():
    x = torch.zeros(1, 64, 32, dtype=torch.bfloat16, device="cuda")
    for axis, G, lev in [(PC, 32, [0.0]), (PC, 32, [0.0, 1.5]), (PC, 32, [float("nan"), 0.5]),
                         (PC, 30, [0.0, 1.0]), (PT, 5, [0.0, 1.0]), (PC, 32, [0.0] * 257)]:
        with pytest.raises(kv.KiviError) as e:
            kv.fake_quant_levels(x, axis, G, lev)
        assert e.value.code == 1


@pytest.mark.parametrize("axis", [PC, PT])
def test_levels_full_size_llama2_13b_layer_sampled(axis):
    """One full Llama-2-13B layer cache (16 x 40 heads x 4,096 tokens x 128):
    four levels fitted to its keys by Lloyd's algorithm (the oracle's fitting),
    sampled matrices checked one by one and every matrix's error against the
    values the launch returns."""
    from oracle import diag
    w = synth.WORKLOADS["llama2_13b_cache"]
    K, V = synth.prefill_inputs(w, seed=2, device="cuda")
    N, T, D = w.B * w.H_kv, w.T, w.D
    Kn = K.reshape(N, T, D)
    lev = diag.fit_levels(Kn[:4].float().cpu().numpy(), axis, 32, 4)
    xh, cc, err = kv.fake_quant_levels(Kn, axis, 32, lev, codes=True)
    torch.cuda.synchronize()
    for i in (0, 217, N - 1):
        ref, rc = oracle.fake_quant_levels(Kn[i].float().cpu().numpy(), axis, 32, lev, codes=True)
        assert np.array_equal(xh[i].cpu().numpy().view(np.uint32), ref.view(np.uint32)), i
        assert np.array_equal(cc[i].cpu().numpy().astype(np.int32), rc), i
    own = (Kn.double() - xh.double()).pow(2).sum(dim=(1, 2))
    torch.testing.assert_close(err, own, rtol=1e-12, atol=0)
