"""GPU parity of ragged batches: batch elements prefilled with different numbers
of tokens (kivi_prefill_ragged), each flushing its residual at its own steps,
against the oracle's per-sequence lengths (OracleCache.prefill(lengths=...)).

Every element's packed store and residual must be bit-exact after the prefill
and after every step on which some element flushed; decode attention over each
element's own tokens must meet rel-L2 <= 5e-3 and max-abs <= 2e-3*max|ref|.
The cases mix one, two and four query heads per kv head, head_dim 64 and 128,
bf16 and fp16, and keys stored before RoPE; lengths include a single token,
exact multiples of R and lengths one past them.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import bit_asymmetric_kv_prefill_b200 as kivi
from bit_asymmetric_kv_prefill_b200 import KiviCache, KiviError, synth
from tests.parity import assert_attn_close, odtype

pytestmark = pytest.mark.gpu

DEV = "cuda"


def small(name, **kw):
    return synth.scaled(synth.WORKLOADS[name], **kw)


def make(w):
    return KiviCache(w.B, w.H_kv, w.D, w.G, w.R, w.torch_dtype, w.T_max, pre_rope=w.pre_rope,
                     rope_theta=w.rope_theta)


def compare_store(cache, orc, w):
    """Every batch element's store and residual against the oracle's."""
    G = w.G
    for b in range(w.B):
        nq, r = int(orc.nqb[b]), int(orc.rb[b])
        assert cache.length_at(b) == (nq, r), b
        got = cache.export(b * w.H_kv, w.H_kv)
        ref = dict(codesK=orc.codesK[b, :, :nq], codesV=orc.codesV[b, :, :nq],
                   sK=orc.sK[b, :, :nq // G], zK=orc.zK[b, :, :nq // G],
                   sV=orc.sV[b, :, :nq], zV=orc.zV[b, :, :nq],
                   resK=orc.resK[b, :, :r], resV=orc.resV[b, :, :r])
        for key, want in ref.items():
            if not np.array_equal(got[key], want):
                bad = np.argwhere(got[key] != want)
                raise AssertionError(f"element {b} {key} differs at {bad[:4].tolist()} ({len(bad)} entries)")


RAGGED = [
    # (workload, overrides, lengths, decode steps)
    ("tiny", dict(B=4, H_q=2, H_kv=2), [300, 33, 128, 129], 140),
    ("tiny", dict(B=3, H_q=4, H_kv=2, dtype="bf16"), [1, 256, 97], 135),
    ("mistral_gqa", dict(B=3, H_q=8, H_kv=2), [1500, 257, 1], 140),
    ("llama2_7b_layer", dict(B=5, H_q=3, H_kv=3, dtype="fp16"), [611, 4, 128, 256, 900], 130),
    ("long_context", dict(B=3, H_q=8, H_kv=2), [700, 200, 129], 130),
]


@pytest.mark.parametrize("name,kw,lengths,steps", RAGGED,
                         ids=[f"{n}-{'-'.join(map(str, L))}" for n, _, L, _ in RAGGED])
def test_ragged_stream_matches_oracle(name, kw, lengths, steps):
    w = small(name, T=max(lengths), steps=steps, **kw)
    K, V = synth.prefill_inputs(w, 13, device=DEV)
    c = make(w)
    orc = oracle.OracleCache(w.B, w.H_kv, w.D, w.G, w.R, odtype(w), w.T_max, pre_rope=w.pre_rope,
                             rope_theta=w.rope_theta)
    c.prefill_ragged(K, V, lengths)
    orc.prefill(synth.bits(K), synth.bits(V), lengths=lengths)
    compare_store(c, orc, w)
    q0 = synth.step_inputs(w, 0, 13, device=DEV)[2]
    assert_attn_close(c.decode(q0).cpu().numpy(), orc.decode(synth.bits(q0)), "after prefill")
    flushes = 0
    for s in range(1, steps + 1):
        k, v, q = synth.step_inputs(w, s, 13, device=DEV)
        flushed = bool((orc.rb == w.R).any())
        c.append(k, v)
        orc.append(synth.bits(k), synth.bits(v))
        if flushed:
            flushes += 1
            compare_store(c, orc, w)
        if flushed or s % 9 == 0 or s == steps:
            assert_attn_close(c.decode(q).cpu().numpy(), orc.decode(synth.bits(q)), f"step {s}")
        else:
            c.decode(q)
    assert flushes >= 1
    compare_store(c, orc, w)
    assert c.device_status() == 0


@pytest.mark.parametrize("name,kw,lengths,steps", [RAGGED[0], RAGGED[2], RAGGED[4]],
                         ids=["tiny", "gqa", "pre_rope"])
def test_ragged_append_decode_and_noalloc_equal_the_separate_calls(name, kw, lengths, steps):
    """The fused append + decode and the allocation-free decode give the
    separate calls' outputs bit for bit on a ragged batch, flushes included,
    and leave the same caches behind."""
    w = small(name, T=max(lengths), steps=steps, **kw)
    K, V = synth.prefill_inputs(w, 14, device=DEV)
    a, b = make(w), make(w)
    a.prefill_ragged(K, V, lengths)
    b.prefill_ragged(K, V, lengths)
    L = kivi.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for s in range(1, steps + 1):
        k, v, q = synth.step_inputs(w, s, 14, device=DEV)
        a.append(k, v)
        oa = a.decode(q)
        ob = b.append_decode(k, v, q)
        assert [a.length_at(e) for e in range(w.B)] == [b.length_at(e) for e in range(w.B)]
        assert torch.equal(oa, ob), f"step {s}"
        if s % 16 == 0:
            on = torch.full_like(oa, float("nan"))
            assert L.kivi_decode_attn_noalloc(a._h, q.data_ptr(), w.H_q, on.data_ptr(), stream) == 0
            assert torch.equal(on, oa), f"noalloc step {s}"
    for e in range(w.B):
        ea, eb = a.export(e * w.H_kv, w.H_kv), b.export(e * w.H_kv, w.H_kv)
        for key in ea:
            assert np.array_equal(ea[key], eb[key]), (e, key)
    assert a.device_status() == 0 and b.device_status() == 0


def test_equal_lengths_make_a_uniform_cache():
    """A ragged prefill whose lengths agree is the uniform prefill of that
    length (bitwise), and kivi_cache_length answers again."""
    w = small("tiny", B=3, H_q=4, H_kv=2, T=400, steps=3)
    K, V = synth.prefill_inputs(w, 15, device=DEV)
    a, b = make(w), make(w)
    a.prefill_ragged(K, V, [300, 300, 300])
    b.prefill(K[:, :, :300].contiguous(), V[:, :, :300].contiguous())
    assert a.length() == b.length() == (256, 44)
    q = synth.step_inputs(w, 0, 15, device=DEV)[2]
    assert torch.equal(a.decode(q), b.decode(q))
    ea, eb = a.export(), b.export()
    for key in ea:
        assert np.array_equal(ea[key], eb[key]), key


def test_ragged_lengths_and_arguments():
    w = small("tiny", B=2, H_q=2, H_kv=2, T=200, steps=0)
    K, V = synth.prefill_inputs(w, 16, device=DEV)
    c = KiviCache(w.B, w.H_kv, w.D, w.G, w.R, w.torch_dtype, T_max=201)
    for bad in ([0, 10], [201, 10], [10]):
        with pytest.raises((KiviError, ValueError)):
            c.prefill_ragged(K, V, bad)
    c.prefill_ragged(K, V, [200, 129])
    assert c.length_at(0) == (128, 72) and c.length_at(1) == (128, 1)
    with pytest.raises(KiviError) as e:
        c.length()
    assert e.value.code == 4                     # lengths differ: ask per element
    with pytest.raises(KiviError):
        c.export(1, 2)                           # a range across different lengths
    with pytest.raises(KiviError) as e:
        c.prefill_ragged(K, V, [5, 5])
    assert e.value.code == 4                     # prefilled already
    k, v, _ = synth.step_inputs(w, 1, 16, device=DEV)
    c.append(k, v)
    with pytest.raises(KiviError) as e:
        c.append(k, v)                           # element 0 would pass T_max
    assert e.value.code == 3
    assert c.length_at(0) == (128, 73) and c.length_at(1) == (128, 2)
    assert c.device_status() == 0
