"""GPU parity: the CUDA library against the CPU oracle on identical seeded
inputs.  Codes, scales, zeros and residual rows must be bit-exact; decode
attention must meet rel-L2 <= 5e-3 and max-abs <= 2e-3*max|ref|.

Small cases span several 32-token groups, several residual slices and ragged
tails, every supported head_dim / dtype / GQA ratio, flushes and pre-RoPE keys;
the full-size workloads are run in the launch configuration the benchmark uses
and checked on sampled sequences."""
import numpy as np
import pytest
import torch

import oracle
from bit_asymmetric_kv_prefill_b200 import KiviCache, KiviError, synth
from tests.parity import Pair, assert_attn_close, attn_errors, value_weight_bound

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.set_device(0)
    yield


def small(name, **kw):
    return synth.scaled(synth.WORKLOADS[name], **kw)


def run_stream(w, seed, steps, check_steps=None, store_every=1, sample=None, sampled_steps=(),
               first_decode_sample=False):
    """Prefill + `steps` x (append + decode); compare the store after prefill
    and after each flush, and decode at `check_steps` (default: all) on every
    sequence; at `sampled_steps` decode only on a few sampled sequences (the
    oracle holds every sequence unless `sample` restricts it)."""
    K, V = synth.prefill_inputs(w, seed, device=DEV)
    pr = Pair(w, seed, sample=sample)
    pr.prefill(K, V)
    del K, V
    pr.check_store(store_every)
    few = _sample(w, 4, seed) if sample is None else None
    worst = (0.0, 0.0)
    q0 = synth.step_inputs(w, 0, seed, device=DEV)[2]
    out, ref = pr.decode(q0, seqs=few if first_decode_sample else None)
    worst = max(worst, assert_attn_close(out, ref, "after prefill"))
    for s in range(1, steps + 1):
        k, v, q = synth.step_inputs(w, s, seed, device=DEV)
        flushed = pr.orc.r == w.R
        pr.append(k, v)
        if flushed:
            pr.check_store(store_every)
        if check_steps is None or s in check_steps:
            out, ref = pr.decode(q)
            worst = max(worst, assert_attn_close(out, ref, f"step {s}"))
        elif s in sampled_steps:
            out, ref = pr.decode(q, seqs=few)
            worst = max(worst, assert_attn_close(out, ref, f"step {s} (sampled sequences)"))
        else:
            pr.cache.decode(q)
    pr.check_store(store_every)
    assert pr.cache.device_status() == 0
    return worst


# ---- the tiny workload, exactly as specified ------------------------------------

def test_tiny_workload():
    w = synth.WORKLOADS["tiny"]
    K, V = synth.prefill_inputs(w, 0, device=DEV)
    pr = Pair(w, 0)
    pr.prefill(K, V)
    assert pr.cache.length() == (128, 128)
    pr.check_store()
    q = synth.step_inputs(w, 0, 0, device=DEV)[2]
    out, ref = pr.decode(q)
    assert_attn_close(out, ref, "tiny")
    # Beyond fp32 accumulation the only rounding is that of the f16 value
    # weights: the error stays inside that bound element by element.
    bound = value_weight_bound(pr.cache, synth.bits(q), w)
    err = np.abs(out.astype(np.float64) - ref)
    slack = 1e-5 * np.abs(ref).max()
    assert np.all(err <= bound + slack), float((err - bound).max())
    assert pr.cache.device_status() == 0


# ---- many small shapes: ragged tails, flushes, dtypes, GQA ------------------------

CASES = [
    # (workload, overrides, steps)
    ("tiny", dict(T=1), 3),
    ("tiny", dict(T=31, B=2), 40),
    ("tiny", dict(T=128), 2),
    ("tiny", dict(T=129, H_q=4), 5),
    ("tiny", dict(T=300, B=3, H_q=4, H_kv=2, dtype="bf16"), 90),
    ("tiny", dict(T=700, B=2, H_q=16, H_kv=2), 3),
    ("llama2_7b_layer", dict(B=2, H_q=3, H_kv=3, T=611, dtype="fp16"), 140),
    ("llama2_7b_layer", dict(B=3, H_q=4, H_kv=4, T=1000), 20),
    ("llama2_13b_cache", dict(B=2, H_q=5, H_kv=5, T=517, layers=1), 8),
    ("mistral_gqa", dict(B=3, H_q=8, H_kv=2, T=2000), 131),
    ("mistral_gqa", dict(B=2, H_q=4, H_kv=2, T=257, R=64), 70),
]


@pytest.mark.parametrize("name,kw,steps", CASES,
                         ids=[f"{n}-{'-'.join(f'{k}{v}' for k, v in kw.items())}" for n, kw, _ in CASES])
def test_small_shapes_stream(name, kw, steps):
    w = small(name, steps=steps, **kw)
    run_stream(w, seed=3, steps=steps)


@pytest.mark.parametrize("kw", [dict(T=200, steps=70), dict(T=1100, steps=40, H_q=16, H_kv=4),
                                dict(T=33, steps=130, B=2, H_q=8, H_kv=8)])
def test_pre_rope_small(kw):
    w = small("long_context", B=kw.pop("B", 1), **{"H_q": 8, "H_kv": 2, **kw})
    run_stream(w, seed=4, steps=w.steps)


def test_pre_rope_eight_heads_per_kv_head_and_head_dim_64():
    w = small("long_context", B=2, H_q=16, H_kv=2, T=300, steps=12)
    run_stream(w, seed=7, steps=w.steps)
    w = small("tiny", B=2, H_q=4, H_kv=2, T=333, steps=6, pre_rope=True)
    run_stream(w, seed=8, steps=w.steps)


def test_pre_rope_longest_supported_context():
    """A pre-RoPE cache near its 823,000-token limit (822,000 prefill tokens and
    one append): the largest RoPE angles the decode's exact reduction serves."""
    w = small("long_context", B=1, H_q=1, H_kv=1, T=822000, steps=1)
    run_stream(w, seed=6, steps=1)


# Sequences split over many warps.  A sequence whose work spans more than 16
# warps has its partials merged in two levels (blocks of 8 partials folded by
# the last warp of each block, then the blocks by the last block); at most 16
# are merged in one pass.  The cases put every warp on one sequence (thousands
# of partials), a few hundred partials on each of eight sequences, and 17 or
# 18 per sequence (140 sequences over 148 SMs x 16 warps), just past the
# one-pass limit, where a sequence's last block can hold a single partial.
SPLIT_CASES = [
    ("llama2_7b_layer", dict(B=1, H_q=1, H_kv=1, T=60000), 2),
    ("mistral_gqa", dict(B=1, H_q=32, H_kv=8, T=40000), 2),
    ("llama2_7b_layer", dict(B=35, H_q=4, H_kv=4, T=1500), 2),
    ("long_context", dict(B=1, H_q=8, H_kv=2, T=30000), 2),
]


@pytest.mark.parametrize("name,kw,steps", SPLIT_CASES,
                         ids=["one-sequence", "gqa-8-sequences", "140-sequences", "pre-rope"])
def test_sequences_split_over_many_warps(name, kw, steps):
    w = small(name, steps=steps, **kw)
    run_stream(w, seed=9, steps=steps)


def test_two_level_merge_is_deterministic():
    """The merge reads partials in slot order whichever warp finishes last, so
    repeated decodes of a long sequence agree bit for bit."""
    w = small("llama2_7b_layer", B=1, H_q=2, H_kv=2, T=50000, steps=0)
    K, V = synth.prefill_inputs(w, 10, device=DEV)
    c = KiviCache(w.B, w.H_kv, w.D, w.G, w.R, w.torch_dtype, w.T)
    c.prefill(K, V)
    q = synth.step_inputs(w, 0, 10, device=DEV)[2]
    a = c.decode(q)
    for _ in range(5):
        assert torch.equal(c.decode(q), a)
    assert c.device_status() == 0


def test_head_dim_64_bf16_and_128_fp16():
    run_stream(small("tiny", dtype="bf16", T=400, B=2, steps=10), seed=5, steps=10)
    run_stream(small("llama2_7b_layer", dtype="fp16", T=400, B=1, H_q=2, H_kv=2, steps=10),
               seed=6, steps=10)


# ---- edge values: constant groups, signed zeros, tiny and huge magnitudes -------------

def _edge_inputs(w, device):
    g = torch.Generator(device="cpu").manual_seed(11)
    K = torch.randn(w.B, w.H_kv, w.T, w.D, generator=g)
    V = torch.randn(w.B, w.H_kv, w.T, w.D, generator=g)
    K[:, :, 0:32, 0] = 1.25                       # constant key group
    K[:, :, 32:64, 1] = 0.0
    K[:, :, 32:64:2, 1] = -0.0                    # signed zeros
    K[:, :, 64:96, 2] *= 1e-6                     # subnormal fp16 scales
    K[:, :, 96:128, 3] *= 5e3                     # large magnitudes
    V[:, :, 5, :] = -3.0                          # constant value groups
    V[:, :, 6, :32] = 0.0
    V[:, :, 7, :] *= 1e-7
    V[:, :, 8, :] *= 5e3
    K[:, :, 200, :] = torch.tensor(np.linspace(-60000, 60000, w.D), dtype=torch.float32)
    return K.to(w.torch_dtype).to(device), V.to(w.torch_dtype).to(device)


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_edge_values_bit_exact(dtype):
    w = small("llama2_7b_layer", B=1, H_q=2, H_kv=2, T=300, dtype=dtype, steps=0)
    K, V = _edge_inputs(w, DEV)
    pr = Pair(w)
    pr.prefill(K, V)
    pr.check_store()
    out, ref = pr.decode(synth.step_inputs(w, 0, 0, device=DEV)[2])
    assert_attn_close(out, ref, "edge values")


def test_lossless_cache_matches_textbook_attention():
    """Values on exact grids quantize losslessly: decode equals softmax
    attention on the raw keys and values (computed here in float64)."""
    w = small("tiny", B=1, H_q=4, H_kv=2, T=160, dtype="bf16", steps=0)
    rng = np.random.default_rng(1)
    K = np.zeros((1, 2, 160, 64))
    V = np.zeros((1, 2, 160, 64))
    for h in range(2):
        for g in range(5):
            for d in range(64):
                k = rng.integers(0, 4, 32)
                k[:2] = (0, 3)
                K[0, h, g * 32:(g + 1) * 32, d] = (int(rng.integers(-30, 30)) + k) * 2.0 ** int(rng.integers(-3, 2))
        for t in range(160):
            for j in range(2):
                k = rng.integers(0, 4, 32)
                k[:2] = (0, 3)
                V[0, h, t, j * 32:(j + 1) * 32] = (int(rng.integers(-30, 30)) + k) * 2.0 ** int(rng.integers(-3, 2))
    Kt = torch.tensor(K, dtype=torch.bfloat16, device=DEV)
    Vt = torch.tensor(V, dtype=torch.bfloat16, device=DEV)
    q = torch.randn(1, 4, 64, generator=torch.Generator().manual_seed(2)).to(torch.bfloat16).to(DEV)
    c = KiviCache(1, 2, 64, 32, 128, torch.bfloat16, 160)
    c.prefill(Kt, Vt)
    out = c.decode(q).cpu().numpy().astype(np.float64)
    qf = q.float().cpu().numpy().astype(np.float64)
    for hq in range(4):
        h = hq // 2
        s = K[0, h] @ qf[0, hq] / 8.0
        p = np.exp(s - s.max())
        p /= p.sum()
        ref = p @ V[0, h]
        # Up to fp32 accumulation, the one rounding is that of each token's
        # f16 value weight p_t s_t (relative 2^-11) on its code part
        # V - z = s c, z the value group's minimum.
        z = np.repeat(V[0, h].reshape(160, 2, 32).min(axis=2), 32, axis=1)
        bound = 2.0 ** -11 * (p[:, None] * (V[0, h] - z)).sum(axis=0)
        err = np.abs(out[0, hq] - ref)
        assert np.all(err <= bound + 1e-6 * np.abs(ref).max()), float((err - bound).max())


# ---- fused append + decode -----------------------------------------------------------

FUSED = [
    ("tiny", dict(T=130, B=2, H_q=4, H_kv=2), 140),          # crosses a flush
    ("tiny", dict(T=31, B=1, dtype="bf16"), 40),              # D = 64
    ("llama2_7b_layer", dict(B=2, H_q=2, H_kv=2, T=300), 30),
    ("mistral_gqa", dict(B=2, H_q=8, H_kv=2, T=257, R=64), 70),
    ("long_context", dict(B=1, H_q=8, H_kv=2, T=200), 60),   # pre-RoPE
]


@pytest.mark.parametrize("name,kw,steps", FUSED,
                         ids=[f"{n}-{'-'.join(f'{k}{v}' for k, v in kw.items())}" for n, kw, _ in FUSED])
def test_append_decode_equals_append_then_decode(name, kw, steps):
    """The fused call gives the separate calls' outputs bit for bit and leaves
    the same cache behind, flushes included."""
    w = small(name, steps=steps, **kw)
    K, V = synth.prefill_inputs(w, 9, device=DEV)
    mk = lambda: KiviCache(w.B, w.H_kv, w.D, w.G, w.R, w.torch_dtype, w.T_max,
                           pre_rope=w.pre_rope, rope_theta=w.rope_theta)
    a, b = mk(), mk()
    a.prefill(K, V)
    b.prefill(K, V)
    for s in range(1, steps + 1):
        k, v, q = synth.step_inputs(w, s, 9, device=DEV)
        a.append(k, v)
        oa = a.decode(q)
        ob = b.append_decode(k, v, q)
        assert a.length() == b.length()
        assert torch.equal(oa, ob), f"step {s}"
    ea, eb = a.export(), b.export()
    for key in ea:
        assert np.array_equal(ea[key], eb[key]), key
    assert a.device_status() == 0 and b.device_status() == 0


def test_append_decode_rejects_bad_arguments():
    w = small("tiny", T=40, steps=0)
    K, V = synth.prefill_inputs(w, 0, device=DEV)
    c = KiviCache(w.B, w.H_kv, w.D, w.G, w.R, w.torch_dtype, T_max=41)
    k, v, q = synth.step_inputs(w, 1, 0, device=DEV)
    with pytest.raises(KiviError):
        c.append_decode(k, v, q)                 # before prefill
    c.prefill(K, V)
    with pytest.raises(KiviError):               # 3 query heads over 2 kv heads
        c.append_decode(k, v, torch.zeros(w.B, 3, w.D, dtype=q.dtype, device=DEV))
    assert c.length() == (0, 40)                 # unchanged by the failed call
    c.append_decode(k, v, q)
    assert c.length() == (0, 41)
    with pytest.raises(KiviError):
        c.append_decode(k, v, q)                 # past T_max
    assert c.device_status() == 0


# ---- argument and state errors -----------------------------------------------------

def test_errors_and_capacity():
    w = small("tiny", T=40, steps=0)
    K, V = synth.prefill_inputs(w, 0, device=DEV)
    c = KiviCache(w.B, w.H_kv, w.D, w.G, w.R, w.torch_dtype, T_max=42)
    k, v, q = synth.step_inputs(w, 1, 0, device=DEV)
    with pytest.raises(KiviError) as e:
        c.decode(q)
    assert e.value.code == 4                      # decode before prefill
    with pytest.raises(KiviError) as e:
        c.append(k, v)
    assert e.value.code == 4
    c.prefill(K, V)
    with pytest.raises(KiviError) as e:
        c.prefill(K, V)
    assert e.value.code == 4                      # prefill twice
    c.append(k, v)
    c.append(k, v)
    assert c.length() == (0, 42)
    with pytest.raises(KiviError) as e:
        c.append(k, v)
    assert e.value.code == 3                      # past T_max
    with pytest.raises(KiviError) as e:
        c.decode(torch.zeros(1, 3, 64, dtype=w.torch_dtype, device=DEV))
    assert e.value.code == 1                      # H_q not a multiple of H_kv
    with pytest.raises(KiviError) as e:
        c.decode(torch.zeros(1, 6, 64, dtype=w.torch_dtype, device=DEV))
    assert e.value.code == 2                      # H_q/H_kv = 3 has no kernel
    buf = torch.zeros(2 * 64 + 1, dtype=w.torch_dtype, device=DEV)
    misaligned = buf[1:].view(1, 2, 64)
    with pytest.raises(KiviError) as e:
        c.decode(misaligned)
    assert e.value.code == 1
    c.reset()
    c.prefill(K, V)
    assert c.length() == (0, 40)
    big = KiviCache(w.B, w.H_kv, w.D, w.G, w.R, w.torch_dtype, T_max=10)
    with pytest.raises(KiviError) as e:
        big.prefill(K, V)
    assert e.value.code == 3
    assert c.device_status() == 0


@pytest.mark.skipif(torch.cuda.device_count() < 2, reason="needs a second visible CUDA device")
def test_calls_with_another_device_current_are_refused():
    """A cache belongs to the device current at its creation: calls made with
    another device current are refused before any launch."""
    w = small("tiny", T=40, steps=0)
    K, V = synth.prefill_inputs(w, 0, device="cuda:0")
    k, v, q = synth.step_inputs(w, 1, 0, device="cuda:0")
    c = KiviCache(w.B, w.H_kv, w.D, w.G, w.R, w.torch_dtype, T_max=48)
    c.prefill(K, V)
    torch.cuda.set_device(1)
    try:
        for call in (lambda: c.append(k, v), lambda: c.decode(q), lambda: c.append_decode(k, v, q)):
            with pytest.raises(KiviError) as e:
                call()
            assert e.value.code == 1
    finally:
        torch.cuda.set_device(0)
    assert c.length() == (0, 40)
    c.append(k, v)
    assert c.length() == (0, 41) and c.device_status() == 0


EXPIRE = [("llama2_7b_layer", dict(B=2, H_q=2, H_kv=2, T=700), False),
          ("mistral_gqa", dict(B=3, H_q=8, H_kv=2, T=1500), True),
          ("long_context", dict(B=1, H_q=8, H_kv=2, T=400), True)]


@pytest.mark.parametrize("name,kw,fused", EXPIRE, ids=[n for n, _, _ in EXPIRE])
def test_an_expired_wait_is_reported_and_the_next_call_is_clean(name, kw, fused):
    """A decode whose warps' first waits give up (the test switch) reports the
    failed wait in the status word without faulting or hanging; reading the
    status clears it, and the next call gives the normal result bit for bit."""
    w = small(name, steps=2, **kw)
    K, V = synth.prefill_inputs(w, 12, device=DEV)
    k, v, q = synth.step_inputs(w, 1, 12, device=DEV)
    mk = lambda: KiviCache(w.B, w.H_kv, w.D, w.G, w.R, w.torch_dtype, w.T_max,
                           pre_rope=w.pre_rope, rope_theta=w.rope_theta)
    a, c = mk(), mk()
    for x in (a, c):
        x.prefill(K, V)
    ref = a.append_decode(k, v, q) if fused else a.decode(q)
    c.debug_expire_first_wait(True)
    if fused:
        c.append_decode(k, v, q)
    else:
        c.decode(q)
    torch.cuda.synchronize()
    assert c.device_status() == 1            # KIVI_DEVICE_WAIT_TIMEOUT
    assert c.device_status() == 0            # read and cleared
    c.debug_expire_first_wait(False)
    if fused:
        # the failed launch may not have stored its token: start the cache over
        c.reset()
        c.prefill(K, V)
        assert torch.equal(c.append_decode(k, v, q), ref)
    else:
        assert torch.equal(c.decode(q), ref)
    assert torch.equal(c.decode(q), a.decode(q))
    assert c.device_status() == 0 and a.device_status() == 0


def test_decode_of_many_layers_replays_from_a_cuda_graph():
    """The decode calls allocate nothing and never synchronise, and their
    lengths travel in the launch parameters: the decodes of a stack of layer
    caches captured once into a CUDA graph replay to the eager outputs bit
    for bit, as often as replayed (the merge tickets reset themselves)."""
    w = small("llama2_13b_cache", B=2, H_q=8, H_kv=4, T=700, layers=1)
    layers = 6
    caches, qs = [], []
    for l in range(layers):
        K, V = synth.prefill_inputs(w, 30 + l, device=DEV)
        c = KiviCache(w.B, w.H_kv, w.D, w.G, w.R, w.torch_dtype, w.T)
        c.prefill(K, V)
        caches.append(c)
        qs.append(synth.step_inputs(w, 0, 30 + l, device=DEV)[2])
    eager = [c.decode(q) for c, q in zip(caches, qs)]
    outs = [torch.empty_like(o) for o in eager]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):           # warm-up on the capture stream
        for c, q, o in zip(caches, qs, outs):
            c.decode(q, out=o, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for c, q, o in zip(caches, qs, outs):
            c.decode(q, out=o)
    for _ in range(3):
        for o in outs:
            o.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        for o, e in zip(outs, eager):
            assert torch.equal(o, e)
    assert all(c.device_status() == 0 for c in caches)


def test_caller_workspace_holds_the_whole_cache():
    w = small("tiny", T=300, B=2, steps=0)
    n = KiviCache.required_bytes(w.B, w.H_kv, w.D, w.G, w.R, w.torch_dtype, 300)
    ws = torch.empty(n, dtype=torch.uint8, device=DEV)
    K, V = synth.prefill_inputs(w, 0, device=DEV)
    c = KiviCache(w.B, w.H_kv, w.D, w.G, w.R, w.torch_dtype, 300, workspace=ws)
    ref = KiviCache(w.B, w.H_kv, w.D, w.G, w.R, w.torch_dtype, 300)
    c.prefill(K, V)
    ref.prefill(K, V)
    q = synth.step_inputs(w, 0, 0, device=DEV)[2]
    assert torch.equal(c.decode(q), ref.decode(q))
    small_ws = torch.empty(n // 2, dtype=torch.uint8, device=DEV)
    with pytest.raises(KiviError) as e:
        KiviCache(w.B, w.H_kv, w.D, w.G, w.R, w.torch_dtype, 300, workspace=small_ws)
    assert e.value.code == 5


def test_decode_is_deterministic_and_stream_ordered():
    w = small("mistral_gqa", B=4, H_q=8, H_kv=2, T=3000, steps=0)
    K, V = synth.prefill_inputs(w, 2, device=DEV)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        c = KiviCache(w.B, w.H_kv, w.D, w.G, w.R, w.torch_dtype, w.T)
        c.prefill(K, V, stream=s)
        q = synth.step_inputs(w, 0, 2, device=DEV)[2]
        a = c.decode(q, stream=s)
        b = c.decode(q, stream=s)
    s.synchronize()
    assert torch.equal(a, b)


# ---- full-size workloads -------------------------------------------------------------
# Every sequence's packed store and residual is compared bit for bit after the
# prefill and after every flush, and decode attention on every (batch, kv head)
# at the listed steps (a few more steps on sampled sequences); the oracle runs
# its sequences on all the host's cores.

def _sample(w, n=4, seed=0):
    total = w.B * w.H_kv
    rng = np.random.default_rng(seed)
    picks = {0, total - 1} | set(rng.choice(total, size=min(n, total), replace=False).tolist())
    return sorted(picks)


def test_full_llama2_7b_layer():
    w = synth.WORKLOADS["llama2_7b_layer"]
    run_stream(w, seed=0, steps=w.steps, check_steps={1, 2, 33, 64})


def test_full_llama2_13b_cache_bytes_and_two_layers():
    w = synth.WORKLOADS["llama2_13b_cache"]
    for layer in range(2):
        K, V = synth.prefill_inputs(w, 100 + layer, device=DEV)
        pr = Pair(w)
        pr.prefill(K, V)
        del K, V
        assert pr.cache.length() == (3968, 128)
        pr.check_store()
        out, ref = pr.decode(synth.step_inputs(w, 0, 100 + layer, device=DEV)[2])
        assert_attn_close(out, ref, f"layer {layer}")
        nb = pr.cache.nbytes()
    # record kv-efficiency/kivi-2bit-llama2-13b-mha-4k, "KV bytes basis":
    # 40 layers of this cache at 4,096 tokens -> 128,000 B/token (codes +
    # residual) and 51,200 B/token of fp16 scale/zero metadata.
    per_tok = lambda x: x * w.layers / (w.B * w.T)
    assert per_tok(nb["codes"]) == 102400
    assert per_tok(nb["residual"]) == 25600
    assert per_tok(nb["codes"] + nb["residual"]) == 128000
    ob = oracle.kv_bytes(w.layers, w.H_kv, w.D, w.R, w.T)
    assert per_tok(nb["codes"] + nb["residual"]) == ob["sum_per_token"]
    assert per_tok(nb["meta"]) == ob["metadata_per_token"] == 51200


def test_full_mistral_gqa():
    w = synth.WORKLOADS["mistral_gqa"]
    run_stream(w, seed=0, steps=w.steps, check_steps={1, 129, 256}, sampled_steps={2, 128, 130},
               first_decode_sample=True)


def test_full_long_context_pre_rope():
    w = synth.WORKLOADS["long_context"]
    run_stream(w, seed=0, steps=w.steps, check_steps={1, 2, 16, 32})
