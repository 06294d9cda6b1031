"""kivi_decode_attn_noalloc on the GPU, through the C ABI.

Some hosts cannot hand the library device memory beyond the cache and the
call's own inputs and outputs: engines that plan every device byte ahead and
forbid allocation while serving, plugins that only receive pointers, paths that
cannot pay for cudaMalloc's device-wide synchronisation.  For them the library
offers kivi_decode_attn_noalloc, which keeps the decode's scratch in a fixed
8 MiB array inside the library.  These checks compare it with the regular
kivi_decode_attn on the same cache, on two calls in a row (the array keeps
the previous call's contents), after a call on another cache of another shape
has left its own partials in the array, and check that an oversized call is
refused.  Both entry points run the same kernel with the same work split and
merge partials in a fixed order, so their outputs must agree bit for bit.
The file runs last so that a failure here leaves every other test already run.
"""
import ctypes

import pytest
import torch

import bit_asymmetric_kv_prefill_b200 as kivi
from bit_asymmetric_kv_prefill_b200 import KiviCache, synth

pytestmark = pytest.mark.gpu

def _cache(name, steps, seed, **kw):
    """A prefilled cache after `steps` appends, and a decode query."""
    w = synth.scaled(synth.WORKLOADS[name], steps=steps, **kw)
    K, V = synth.prefill_inputs(w, seed, device="cuda")
    c = KiviCache(w.B, w.H_kv, w.D, w.G, w.R, w.torch_dtype, w.T_max)
    c.prefill(K, V)
    for s in range(1, steps + 1):
        k, v, _ = synth.step_inputs(w, s, seed, device="cuda")
        c.append(k, v)
    return w, c, synth.step_inputs(w, steps + 1, seed, device="cuda")[2]


def _call(fn, c, w, q):
    out = torch.full((w.B, w.H_q, w.D), float("nan"), device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert fn(c._h, q.data_ptr(), w.H_q, out.data_ptr(), stream) == 0
    return out


@pytest.mark.parametrize("name,kw,steps", [
    ("mistral_gqa", dict(B=4, H_q=16, H_kv=4, T=3000), 3),
    ("tiny", dict(B=3, H_q=2, H_kv=2, T=700), 130),
    # two sequences over every warp: partials merged in two levels, with the
    # merge blocks' tickets in the shared array too
    ("llama2_7b_layer", dict(B=1, H_q=2, H_kv=2, T=20000), 1),
])
def test_noalloc_matches_decode_attn_on_two_calls(name, kw, steps):
    torch.cuda.set_device(0)
    L = kivi.lib()
    # Another cache of another shape (more sequences, eight query heads per kv
    # head) leaves its tickets and partials in the shared array first.
    wo, co, qo = _cache("mistral_gqa", 0, 5, B=6, H_q=64, H_kv=8, T=2500)
    other = _call(L.kivi_decode_attn_noalloc, co, wo, qo)
    w, c, q = _cache(name, steps, 21, **kw)
    ref = _call(L.kivi_decode_attn, c, w, q)
    a = _call(L.kivi_decode_attn_noalloc, c, w, q)
    b = _call(L.kivi_decode_attn_noalloc, c, w, q)
    torch.cuda.synchronize()
    assert torch.isfinite(ref).all()
    assert torch.equal(a, ref)
    assert torch.equal(b, ref)
    assert torch.equal(other, _call(L.kivi_decode_attn, co, wo, qo))
    assert c.device_status() == 0 and co.device_status() == 0


def test_noalloc_refuses_scratch_beyond_its_array():
    torch.cuda.set_device(0)
    # 4,096 sequences x 8 query heads per kv head need far more than 8 MiB of
    # partials: the call must be refused before any launch.
    B, H_kv, D, T = 512, 8, 128, 32
    K = torch.zeros(B, H_kv, T, D, dtype=torch.bfloat16, device="cuda")
    c = KiviCache(B, H_kv, D, 32, 128, torch.bfloat16, T)
    c.prefill(K, K)
    q = torch.zeros(B, 8 * H_kv, D, dtype=torch.bfloat16, device="cuda")
    out = torch.full((B, 8 * H_kv, D), -7.0, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert kivi.lib().kivi_decode_attn_noalloc(c._h, q.data_ptr(), 8 * H_kv, out.data_ptr(),
                                               stream) == 3   # KIVI_ERR_CAPACITY
    torch.cuda.synchronize()
    assert torch.all(out == -7.0)
