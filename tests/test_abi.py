"""CPU checks of the C-ABI library: it loads, exports every declared symbol,
rejects bad configurations before touching the GPU, and its decode work split
covers every item exactly once."""
import ctypes
import itertools
import subprocess

import numpy as np
import pytest

import bit_asymmetric_kv_prefill_b200 as kivi
from bit_asymmetric_kv_prefill_b200 import build as kbuild


@pytest.fixture(scope="module", autouse=True)
def built():
    kbuild.build()


def test_every_declared_symbol_is_exported():
    declared = kivi.declared_symbols()
    assert len(declared) >= 14
    nm = subprocess.run(["nm", "-D", "--defined-only", kivi.LIB_PATH], capture_output=True,
                        text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in nm.splitlines() if " T " in ln}
    missing = [s for s in declared if s not in exported]
    assert not missing, missing
    L = kivi.lib()
    for s in declared:
        assert getattr(L, s) is not None


def test_status_strings_and_version():
    assert kivi.abi_version() == 1
    names = {kivi.status_string(c) for c in range(8)}
    assert len(names) == 8 and "ok" in names
    assert kivi.status_string(99) == "unknown status"


def _cfg(**kw):
    base = dict(B=1, H_kv=2, D=64, G=32, R=128, dtype=kivi.KIVI_F16, T_max=256, pre_rope=0,
                rope_theta=10000.0, workspace=None, workspace_bytes=0)
    base.update(kw)
    return kivi._Config(*[base[f] for f, _ in kivi._Config._fields_])


@pytest.mark.parametrize("kw,code", [
    (dict(D=96), 2),             # head_dim without a kernel
    (dict(G=16, R=128), 2),      # group size other than 32
    (dict(R=100), 1),            # residual not a multiple of G
    (dict(dtype=5), 1),
    (dict(B=0), 1),
    (dict(T_max=0), 1),
    (dict(pre_rope=1, rope_theta=0.0), 1),
])
def test_bad_configs_are_rejected_before_any_launch(kw, code):
    h = ctypes.c_void_p()
    cfg = _cfg(**kw)
    assert kivi.lib().kivi_cache_create_ex(ctypes.byref(cfg), ctypes.byref(h)) == code
    assert not h.value
    n = ctypes.c_size_t()
    assert kivi.lib().kivi_cache_required_bytes(ctypes.byref(cfg), ctypes.byref(n)) == code


def test_pre_rope_length_limit():
    """Pre-RoPE caches hold at most 823,000 tokens (the decode's exact angle
    reduction); plain caches have no such limit."""
    n = ctypes.c_size_t()
    L = kivi.lib()
    ok = _cfg(pre_rope=1, T_max=823000)
    assert L.kivi_cache_required_bytes(ctypes.byref(ok), ctypes.byref(n)) == 0 and n.value > 0
    over = _cfg(pre_rope=1, T_max=823001)
    assert L.kivi_cache_required_bytes(ctypes.byref(over), ctypes.byref(n)) == 2
    plain = _cfg(pre_rope=0, T_max=4000000)
    assert L.kivi_cache_required_bytes(ctypes.byref(plain), ctypes.byref(n)) == 0


def test_null_handles_are_rejected():
    L = kivi.lib()
    assert L.kivi_prefill(None, None, None, 10, None) == 1
    assert L.kivi_append(None, None, None, None) == 1
    assert L.kivi_decode_attn(None, None, 2, None, None) == 1
    assert L.kivi_cache_destroy(None) == 1
    assert L.kivi_cache_reset(None) == 1
    assert L.kivi_export(None, 0, 1, *([None] * 8)) == 1
    assert L.kivi_cache_length(None, None, None) == 1


# kivi_fake_quant(x, dtype, N, T, D, axis, G, bits, symmetric, xhat, sq_err, stream);
# the pointers below are never dereferenced: every case fails its argument check.
_FQ = dict(x=256, dtype=kivi.KIVI_BF16, N=2, T=64, D=128, axis=kivi.AXIS_PER_TOKEN, G=32,
           bits=2, sym=0, outlier=0, xhat=512, err=None)


@pytest.mark.parametrize("kw,code", [
    (dict(x=None), 1),
    (dict(xhat=None, err=None), 1),
    (dict(x=258), 1),                           # x not 16-byte aligned
    (dict(xhat=520), 1),                        # x_hat not 16-byte aligned
    (dict(err=260), 1),                         # sq_err not 8-byte aligned
    (dict(dtype=3), 1),
    (dict(N=0), 1), (dict(T=0), 1), (dict(D=12), 1), (dict(D=0), 1),
    (dict(axis=2), 1),
    (dict(bits=0), 1), (dict(bits=9), 1), (dict(bits=1, sym=1), 1),
    (dict(outlier=2), 1), (dict(outlier=-1), 1),
    (dict(G=0), 1),
    (dict(G=48), 1),                            # per token: D % G != 0
    (dict(axis=kivi.AXIS_PER_CHANNEL, G=48), 1),  # per channel: T % G != 0
    (dict(G=4, D=128), 2),                      # per-token group below one vector
    (dict(G=512, D=1024), 2),                   # per-token group wider than a warp
    (dict(T=1 << 27, D=128), 2),                # T*D above 2^33
])
def test_fake_quant_rejects_bad_arguments_before_any_launch(kw, code):
    a = dict(_FQ, **kw)
    assert kivi.lib().kivi_fake_quant(a["x"], a["dtype"], a["N"], a["T"], a["D"], a["axis"],
                                      a["G"], a["bits"], a["sym"], a["outlier"], a["xhat"],
                                      a["err"], None) == code


@pytest.mark.parametrize("seqs,n_groups,r,wg,wr,warps", [
    (1, 4, 128, 4, 3, 26),        # tiny workload: 4 groups + 22 residual items
    (256, 128, 1, 4, 3, 2368),    # Llama-2-7B layer after the first flush
    (256, 124, 128, 4, 3, 2368),
    (8, 4092, 128, 4, 3, 2072),   # long context
    (3, 0, 7, 4, 3, 2),           # residual only
    (5, 3, 6, 1, 1, 40),
    (7, 9, 13, 5, 2, 11),
])
def test_decode_split_covers_every_item_once(seqs, n_groups, r, wg, wr, warps):
    n_items = n_groups + -(-r // 6)
    total = seqs * (n_groups * wg + -(-r // 6) * wr)
    warps = min(warps, total)
    for s in range(seqs):
        first, last, _, _ = kivi.decode_split(seqs, n_groups, r, wg, wr, warps, s, 0)
        assert 0 <= first <= last < warps
        covered = []
        for w in range(warps):
            f2, l2, i0, i1 = kivi.decode_split(seqs, n_groups, r, wg, wr, warps, s, w)
            assert (f2, l2) == (first, last)
            if w < first or w > last:
                assert i0 == i1, (s, w)
            covered.extend(range(i0, i1))
        assert covered == list(range(n_items)), s


def test_decode_split_balances_weight():
    seqs, n_groups, r, wg, wr, warps = 256, 128, 64, 4, 3, 2368
    load = [0] * warps
    for s, w in itertools.product(range(0, seqs, 17), range(warps)):
        _, _, i0, i1 = kivi.decode_split(seqs, n_groups, r, wg, wr, warps, s, w)
        load[w] += sum(wg if i < n_groups else wr for i in range(i0, i1))
    per_seq = n_groups * wg + -(-r // 6) * wr
    assert sum(load) == per_seq * len(range(0, seqs, 17))


def _split_reference(seqs, n_groups, r, wg, wr, warps, s, w):
    """The split's definition in exact Python integers."""
    n_res = -(-r // 6)
    n_items = n_groups + n_res
    C = n_groups * wg + n_res * wr
    Tot = C * seqs

    def lo(x):
        return x * Tot // warps

    def owner(pos):
        return ((pos + 1) * warps - 1) // Tot

    def first_item_at(rel):
        gend = n_groups * wg
        if n_groups > 0 and rel <= gend - wg:
            return -(-rel // wg)
        if rel <= gend:
            return n_groups
        return min(n_groups + -(-(rel - gend) // wr), n_items)

    base = s * C
    ra, rb = max(lo(w) - base, 0), min(lo(w + 1) - base, C)
    i0 = i1 = 0
    if ra < rb:
        i0, i1 = first_item_at(ra), first_item_at(rb)
        i1 = max(i1, i0)
    return owner(base), owner(base + C - 1), i0, i1


def test_decode_split_matches_exact_integer_definition():
    """The split runs its divisions as reciprocal multiplies with a one-step
    integer fix-up; on large shapes it must equal exact integer division."""
    rng = np.random.default_rng(5)
    for _ in range(60):
        seqs = int(rng.integers(1, 4097))
        n_groups = int(rng.integers(0, 1 << 20))
        r = int(rng.integers(1, 129))
        wg, wr = int(rng.integers(1, 17)), int(rng.integers(1, 17))
        total = seqs * (n_groups * wg + -(-r // 6) * wr)
        warps = min(int(rng.integers(1, 4737)), total)
        for _ in range(20):
            s, w = int(rng.integers(0, seqs)), int(rng.integers(0, warps))
            got = tuple(kivi.decode_split(seqs, n_groups, r, wg, wr, warps, s, w))
            assert got == _split_reference(seqs, n_groups, r, wg, wr, warps, s, w), \
                (seqs, n_groups, r, wg, wr, warps, s, w)


def test_fake_quant_binding_rejects_host_tensors():
    import torch
    with pytest.raises(ValueError):
        kivi.fake_quant(torch.zeros(4, 64, 128, dtype=torch.bfloat16), kivi.AXIS_PER_CHANNEL)
    with pytest.raises(ValueError):
        kivi.fake_quant(torch.zeros(128, dtype=torch.bfloat16), kivi.AXIS_PER_TOKEN)


@pytest.mark.parametrize("seqs,n_groups,r,warps", [
    (1, 1871, 34, 2368),     # every warp on one sequence
    (8, 1250, 2, 1776),      # a few hundred partials per sequence
    (140, 44, 94, 2368),     # 17 or 18 partials: just past one pass, a last block of one
    (256, 124, 128, 2368),   # Llama-2-7B layer: one pass everywhere
    (3, 0, 7, 2),
    (37, 900, 5, 1184),
])
def test_merge_rows_and_tickets_stay_in_their_arrays(seqs, n_groups, r, warps):
    """Scratch bounds of the decode merge: sequence s's partial of slot k sits
    at row first(s) + s + k, and when the sequence spans more than 16 warps
    its merge blocks of 8 slots take tickets seqs + first(s) + s + kb.  Every
    row lies below warps + seqs (the rows the library reserves), every ticket
    below seqs + warps + seqs, and no row or ticket serves two sequences."""
    F = 8
    warps = min(warps, seqs * (n_groups * 4 + -(-r // 6) * 3))
    rows, tickets = set(), set()
    for s in range(seqs):
        first, last, _, _ = kivi.decode_split(seqs, n_groups, r, 4, 3, warps, s, 0)
        count = last - first + 1
        if count == 1:
            continue   # written directly, no partial
        for k in range(count):
            row = first + s + k
            assert 0 <= row < warps + seqs
            assert row not in rows
            rows.add(row)
        assert s not in tickets
        tickets.add(s)
        if count > 2 * F:
            for kb in range(-(-count // F)):
                t = seqs + first + s + kb
                assert seqs <= t < seqs + warps + seqs
                assert t not in tickets
                tickets.add(t)
